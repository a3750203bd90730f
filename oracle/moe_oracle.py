"""CPU oracle of the fused top-k MoE layer: the Python face of ``moe_oracle.cpp``.

TEST INFRASTRUCTURE ONLY: imported by ``tests/``, ``__graft_entry__.smoke()``
and the CPU-baseline legs of ``bench.py``; never by the product path.  The
oracle shares no code, table or constant generator with the CUDA library.

All of the method's arithmetic is in the C++ file next to this one (plain
loops in double precision, every rounding point of the method explicit, each
function citing its passage).  This module holds none of it: it checks and
converts arguments, picks the experts a call needs, calls the compiled oracle
through ctypes and shapes the results.  The library is compiled with g++ on
first use (``build_oracle.py``) into ``oracle/libmoe_oracle.so``.

Sources: [AWS] "AWS erklärt zwei Kernel-Optimierungen, die den Durchsatz von
SageMaker AI auf H200 steigern" (kinachrichten.com); [PR] the analysis of
vLLM PR #64760, "vLLM, H200 GPU를 위한 FP8 MoE 다운 프로젝션 최적화"
(blog.secrett2633.cloud); [PPLX] "Hosting von Qwen auf Blackwell"
(perplexity.ai).  The readings where the pages are silent are listed at the
top of the C++ file.  Parity pins for every function live in
``tests/test_oracle_*.py``.
"""

from __future__ import annotations

import ctypes
import os
import threading

import numpy as np

from .build_oracle import build

__all__ = [
    "BF16_MAX", "E4M3_MAX", "round_bf16", "e4m3_round", "e4m3_encode", "e4m3_decode", "pow2_ceil",
    "quantize_act_group128", "dequantize_act_group128", "quantize_weight_block128",
    "dequantize_weight_block128", "quantize_mx_group32", "mx_scale", "dequantize_mx_group32", "route",
    "align_capacity", "align", "expert_mlp", "moe_forward", "assignment_outputs", "expert_shards",
    "moe_forward_expert_parallel", "max_threads", "build",
]

_lock = threading.Lock()
_lib = None

_P = ctypes.c_void_p
_I64 = ctypes.c_int64
_I32 = ctypes.c_int32
_D = ctypes.c_double


def _L():
    global _lib
    with _lock:
        if _lib is None:
            # MOE_ORACLE_LIB: load this compiled copy instead (the pins' mutation check runs the pins
            # against copies of the oracle with a planted mistake)
            lib = ctypes.CDLL(os.environ.get("MOE_ORACLE_LIB") or build())
            sig = {
                "orc_last_error": (ctypes.c_char_p, []),
                "orc_bf16_max": (_D, []),
                "orc_e4m3_max": (_D, []),
                "orc_max_threads": (ctypes.c_int, []),
                "orc_round_bf16": (None, [_P, _P, _I64]),
                "orc_e4m3_round": (None, [_P, _P, _I64]),
                "orc_e4m3_encode": (None, [_P, _P, _I64]),
                "orc_e4m3_decode": (None, [_P, _P, _I64]),
                "orc_pow2_ceil": (None, [_P, _P, _I64]),
                "orc_mx_scale": (None, [_P, _P, _I64]),
                "orc_quantize_act_group128": (ctypes.c_int, [_P, _I64, _I64, _P, _P]),
                "orc_dequantize_act_group128": (None, [_P, _P, _I64, _I64, _P]),
                "orc_quantize_weight_block128": (ctypes.c_int, [_P, _I32, _I64, _I64, _I64, _P, _P, _I32]),
                "orc_dequantize_weight_block128": (None, [_P, _P, _I64, _I64, _I64, _P]),
                "orc_quantize_mx_group32": (ctypes.c_int, [_P, _I32, _I64, _I64, _P, _P, _I32]),
                "orc_dequantize_mx_group32": (None, [_P, _P, _I64, _I64, _P]),
                "orc_route": (ctypes.c_int, [_P, _I64, _I32, _I32, _I32, _P, _P]),
                "orc_align_capacity": (_I64, [_I64, _I32, _I32, _I32]),
                "orc_align": (ctypes.c_int, [_P, _I64, _I32, _I32, _I32, _I32, _I32, _P, _P, _P, _P, _P]),
                "orc_expert_mlp": (ctypes.c_int, [_P, _I64, _I64, _I64, _P, _P, _I32, _I32, _D, _P, _P, _P, _P,
                                                  _P, _I32]),
                "orc_moe_forward": (ctypes.c_int, [_P, _I64, _I64, _I64, _I32, _P, _P, _I32, _P, _P, _P, _P, _I32,
                                                   _I32, _I32, _I32, _D, _I32, _P, _P]),
                "orc_assignment_outputs": (ctypes.c_int, [_P, _I64, _I64, _I64, _I32, _P, _P, _I32, _P, _P, _P, _P,
                                                          _I32, _I32, _I32, _I32, _D, _I32, _I64, _P, _P]),
                "orc_expert_shards": (ctypes.c_int, [_I32, _I32, _P, _P]),
                "orc_sum_round_bf16": (None, [_P, _I32, _I64, _P]),
            }
            for name, (res, args) in sig.items():
                f = getattr(lib, name)
                f.restype, f.argtypes = res, args
            _lib = lib
    return _lib


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def _check(rc: int):
    if rc != 0:
        raise ValueError(_L().orc_last_error().decode())


def _f64(x) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(x, dtype=np.float64))


def max_threads() -> int:
    """Threads the oracle's OpenMP loops use by default (all host cores)."""
    return int(_L().orc_max_threads())


BF16_MAX = float(_L().orc_bf16_max())
E4M3_MAX = float(_L().orc_e4m3_max())
MX_GROUP = 32


# ----------------------------------------------------------------------------- number formats
def _elementwise(fn, x, out_dtype, in_dtype=np.float64):
    x = np.ascontiguousarray(np.asarray(x, dtype=in_dtype))
    out = np.empty(x.shape, dtype=out_dtype)
    getattr(_L(), fn)(_ptr(x), _ptr(out), x.size)
    return out


def round_bf16(x) -> np.ndarray:
    """Nearest bfloat16 value, ties to even (float64 result)."""
    return _elementwise("orc_round_bf16", x, np.float64)


def e4m3_round(x) -> np.ndarray:
    """Nearest E4M3 value, ties to even, saturating at +-448 (float64 result)."""
    return _elementwise("orc_e4m3_round", x, np.float64)


def e4m3_encode(x) -> np.ndarray:
    """E4M3 byte codes of ``x`` rounded by :func:`e4m3_round`."""
    return _elementwise("orc_e4m3_encode", x, np.uint8)


def e4m3_decode(codes) -> np.ndarray:
    """E4M3 byte codes -> float64 values."""
    return _elementwise("orc_e4m3_decode", codes, np.float64, np.uint8)


def pow2_ceil(s) -> np.ndarray:
    """Smallest power of two >= s, exactly."""
    return _elementwise("orc_pow2_ceil", s, np.float64)


def mx_scale(e8m0) -> np.ndarray:
    """E8M0 byte -> its power-of-two value."""
    return _elementwise("orc_mx_scale", e8m0, np.float64, np.uint8)


# ----------------------------------------------------------------------------- quantisation rules
def quantize_act_group128(v):
    """[PR] §1.2 per (row, 128 columns), power-of-two fp32 scale.  v [rows, K].
    Returns (codes uint8 [rows, K], scales float32 [rows, K // 128])."""
    v = _f64(v)
    rows, k = v.shape
    codes = np.empty((rows, k), np.uint8)
    scales = np.empty((rows, k // 128), np.float32)
    _check(_L().orc_quantize_act_group128(_ptr(v), rows, k, _ptr(codes), _ptr(scales)))
    return codes, scales


def dequantize_act_group128(codes, scales) -> np.ndarray:
    codes = np.ascontiguousarray(codes, dtype=np.uint8)
    scales = np.ascontiguousarray(scales, dtype=np.float32)
    rows, k = codes.shape
    out = np.empty((rows, k), np.float64)
    _L().orc_dequantize_act_group128(_ptr(codes), _ptr(scales), rows, k, _ptr(out))
    return out


def _values_or_bf16_bits(w):
    """float64 values, or bf16 bit patterns (uint16) passed through as they are."""
    w = np.asarray(w)
    if w.dtype == np.uint16:
        return np.ascontiguousarray(w), 1
    return _f64(w), 0


def quantize_weight_block128(w, threads: int = 0):
    """FP8 E4M3 with one fp32 scale per 128x128 block (the workload's rule).
    w [..., N, K]: bf16 values (float) or bf16 bit patterns (uint16).  Returns
    (codes uint8 [..., N, K], scales float32 [..., N//128, K//128])."""
    w, bits = _values_or_bf16_bits(w)
    *lead, n, k = w.shape
    b = int(np.prod(lead)) if lead else 1
    codes = np.empty(w.shape, np.uint8)
    scales = np.empty((*lead, n // 128, k // 128), np.float32)
    _check(_L().orc_quantize_weight_block128(_ptr(w), bits, b, n, k, _ptr(codes), _ptr(scales), threads))
    return codes, scales


def dequantize_weight_block128(codes, scales) -> np.ndarray:
    codes = np.ascontiguousarray(codes, dtype=np.uint8)
    scales = np.ascontiguousarray(scales, dtype=np.float32)
    *lead, n, k = codes.shape
    b = int(np.prod(lead)) if lead else 1
    out = np.empty(codes.shape, np.float64)
    _L().orc_dequantize_weight_block128(_ptr(codes), _ptr(scales), b, n, k, _ptr(out))
    return out


def quantize_mx_group32(v, threads: int = 0):
    """MXFP8: E4M3 codes with one E8M0 scale per 32 elements of a row.
    v [..., K]: values (float) or bf16 bit patterns (uint16).  Returns
    (codes uint8 [..., K], e8m0 uint8 [..., K // 32])."""
    v, bits = _values_or_bf16_bits(v)
    *lead, k = v.shape
    rows = int(np.prod(lead)) if lead else 1
    codes = np.empty(v.shape, np.uint8)
    e8m0 = np.empty((*lead, k // MX_GROUP), np.uint8)
    _check(_L().orc_quantize_mx_group32(_ptr(v), bits, rows, k, _ptr(codes), _ptr(e8m0), threads))
    return codes, e8m0


def dequantize_mx_group32(codes, e8m0) -> np.ndarray:
    codes = np.ascontiguousarray(codes, dtype=np.uint8)
    e8m0 = np.ascontiguousarray(e8m0, dtype=np.uint8)
    *lead, k = codes.shape
    rows = int(np.prod(lead)) if lead else 1
    out = np.empty(codes.shape, np.float64)
    _L().orc_dequantize_mx_group32(_ptr(codes), _ptr(e8m0), rows, k, _ptr(out))
    return out


# ----------------------------------------------------------------------------- routing and alignment
def route(logits, topk: int, renormalize: bool = True):
    """Top-k softmax router.  logits float32 [T, E] -> (ids int32 [T, k], weights float32 [T, k])."""
    logits = np.ascontiguousarray(logits, dtype=np.float32)
    t, e = logits.shape
    ids = np.empty((t, topk), np.int32)
    w = np.empty((t, topk), np.float32)
    _check(_L().orc_route(_ptr(logits), t, e, topk, int(bool(renormalize)), _ptr(ids), _ptr(w)))
    return ids, w


def align_capacity(T: int, topk: int, E: int, block_m: int) -> int:
    return int(_L().orc_align_capacity(T, topk, E, block_m))


def align(topk_ids, E: int, block_m: int, first_expert: int = 0, num_global_experts=None):
    """[PR] §1.1 expert-sorted, block-padded permutation (dict of the results)."""
    ids = np.ascontiguousarray(np.asarray(topk_ids).astype(np.int32))
    t, k = ids.shape
    n_global = E if num_global_experts is None else int(num_global_experts)
    cap = align_capacity(t, k, E, block_m)
    sorted_ids = np.empty(cap, np.int32)
    expert_ids = np.empty(cap // block_m, np.int32)
    ntpp = np.zeros(1, np.int32)
    counts = np.empty(E, np.int32)
    offsets = np.empty(E + 1, np.int32)
    _check(_L().orc_align(_ptr(ids), t, k, E, block_m, first_expert, n_global, _ptr(sorted_ids),
                          _ptr(expert_ids), _ptr(ntpp), _ptr(counts), _ptr(offsets)))
    return {"sorted_token_ids": sorted_ids, "expert_ids": expert_ids, "num_tokens_post_padded": int(ntpp[0]),
            "expert_counts": counts, "expert_offsets": offsets, "capacity": cap}


# ----------------------------------------------------------------------------- expert MLP and the layer
_REQUANT = {False: 0, True: 1, "mx": 2}


def expert_mlp(x_hat, w13_hat, w2_hat, requant, return_intermediates: bool = False, swiglu_limit=None,
               threads: int = 0):
    """One expert's SiLU-gated MLP on rows ([PR] §1.1/§1.2), double weights.

    requant: False (bf16 path), True (per-(row,128) FP8) or "mx" (per-32 MXFP8).
    x_hat [n, H], w13_hat [2I, H], w2_hat [H, I].  Returns y [n, H] (and the
    intermediates h, p, a2_codes, a2_scales when asked).
    """
    x_hat, w13_hat, w2_hat = _f64(x_hat), _f64(w13_hat), _f64(w2_hat)
    n, hd = x_hat.shape
    i = w13_hat.shape[0] // 2
    rq = _REQUANT[requant if requant == "mx" else bool(requant)]
    y = np.empty((n, hd), np.float64)
    h = np.empty((n, 2 * i), np.float64)
    p = np.empty((n, i), np.float64)
    codes = np.empty((n, i), np.uint8) if rq else None
    scales = None if not rq else (np.empty((n, i // 128), np.float32) if rq == 1 else
                                  np.empty((n, i // MX_GROUP), np.uint8))
    has_lim = swiglu_limit is not None
    _check(_L().orc_expert_mlp(_ptr(x_hat), n, hd, i, _ptr(w13_hat), _ptr(w2_hat), rq, int(has_lim),
                               float(swiglu_limit) if has_lim else 0.0, _ptr(y), _ptr(h), _ptr(p),
                               None if codes is None else _ptr(codes), None if scales is None else _ptr(scales),
                               threads))
    if return_intermediates:
        return y, {"h": h, "p": p, "a2_codes": codes, "a2_scales": scales}
    return y


def _weight_type(w13_e, s13_e, mx):
    if s13_e is None:
        dt = np.asarray(w13_e).dtype
        return 1 if dt == np.uint16 else 0          # bf16 bit patterns, or bf16 values as float64
    if mx is None:
        mx = np.asarray(s13_e).dtype == np.uint8
    return 3 if mx else 2


def _routing(topk, logits, topk_ids, topk_weights, renormalize):
    if logits is not None:
        topk_ids, topk_weights = route(logits, topk, renormalize)
    return np.asarray(topk_ids).astype(np.int32), np.asarray(topk_weights, dtype=np.float32)


def _layer_args(x, w13, w2, topk, tokens, topk_ids, topk_weights, w13_scale, w2_scale, mx,
                router_weight_on_input, swiglu_limit, expert_range, threads):
    """The C arguments of one layer evaluation on the rows ``tokens`` (and the
    arrays that must stay alive while it runs)."""
    fp8 = w13_scale is not None
    if fp8 != (w2_scale is not None):
        raise ValueError("w13_scale and w2_scale go together")
    if router_weight_on_input and topk != 1:
        raise ValueError("router_weight_on_input needs topk == 1")
    h_dim = x.shape[1]
    xs = _f64(x[tokens])
    ids = np.ascontiguousarray(topk_ids[tokens])
    wts = np.ascontiguousarray(topk_weights[tokens])
    if expert_range is None:
        first, count = 0, int(ids.max()) + 1 if ids.size else 1
    else:
        first, count = int(expert_range[0]), int(expert_range[1])
    needed = [int(g) - first for g in np.unique(ids) if 0 <= int(g) - first < count]
    keep = [xs, ids, wts]
    p13, p2, q13, q2 = [None] * count, [None] * count, [None] * count, [None] * count
    wtype, i_dim = (2 if fp8 else 0), 128
    for n, e in enumerate(needed):
        a13, a2 = np.ascontiguousarray(w13[e]), np.ascontiguousarray(w2[e])
        s13 = None if not fp8 else np.ascontiguousarray(w13_scale[e])
        s2 = None if not fp8 else np.ascontiguousarray(w2_scale[e])
        wt = _weight_type(a13, s13, mx)
        if wt == 0:
            a13, a2 = _f64(a13), _f64(a2)
        if n and wt != wtype:
            raise ValueError("experts in different weight formats")
        wtype = wt
        i_dim = a13.shape[0] // 2
        if a13.shape != (2 * i_dim, h_dim) or a2.shape != (h_dim, i_dim):
            raise ValueError(f"expert {e}: w13 {a13.shape} / w2 {a2.shape} do not match H={h_dim}")
        keep += [a13, a2, s13, s2]
        p13[e], p2[e] = _ptr(a13), _ptr(a2)
        if fp8:
            q13[e], q2[e] = _ptr(s13), _ptr(s2)
    arr = ctypes.c_void_p * max(count, 1)
    has_lim = swiglu_limit is not None
    args = (_ptr(xs), len(tokens), h_dim, i_dim, topk, _ptr(ids), _ptr(wts), wtype, arr(*p13), arr(*q13),
            arr(*p2), arr(*q2), first, count, int(bool(router_weight_on_input)), int(has_lim),
            float(swiglu_limit) if has_lim else 0.0, threads)
    return args, keep


def moe_forward(x, w13, w2, topk: int, *, logits=None, topk_ids=None, topk_weights=None,
                w13_scale=None, w2_scale=None, renormalize: bool = True, tokens=None,
                return_y: bool = False, mx=None, router_weight_on_input: bool = False, swiglu_limit=None,
                expert_range=None, threads: int = 0):
    """The fused MoE layer: route -> experts -> top-k weighted combine.

    x [T, H] (bf16 values).  w13 / w2: per-expert weights, indexable by the
    expert (an array [E, ...] or any object with ``__getitem__``), each
    [2I, H] / [H, I] as float64 bf16 values, uint16 bf16 bit patterns, E4M3
    codes with ``w13_scale`` / ``w2_scale`` fp32 [.., N/128, K/128] block
    scales, or E4M3 codes with uint8 E8M0 per-32 scales (MXFP8; ``mx`` or the
    scale dtype says which).  Only the experts the evaluated tokens use are
    read.  Routing: ``logits`` [T, E] float32, or ``topk_ids`` /
    ``topk_weights``.  ``tokens``: the token indices to evaluate (each output
    row depends only on its own token, its routing and the weights).
    ``expert_range = (first, count)``: expert parallelism, the weights hold
    experts [first, first + count) indexed from zero and ``out`` sums only
    their assignments.  ``router_weight_on_input`` (top-1) and
    ``swiglu_limit``: the readings in the C++ file.  ``threads``: OpenMP
    threads (0 = all cores).

    Returns ``out`` [len(tokens), H] (float64 holding bf16 values),
    ``topk_ids``, ``topk_weights`` and, with ``return_y``, ``y``
    [len(tokens), topk, H]: each assignment's expert output before its weight.
    """
    x = np.asarray(x)
    topk_ids, topk_weights = _routing(topk, logits, topk_ids, topk_weights, renormalize)
    tokens = np.arange(x.shape[0]) if tokens is None else np.asarray(tokens, dtype=np.int64)
    args, keep = _layer_args(x, w13, w2, topk, tokens, topk_ids, topk_weights, w13_scale, w2_scale, mx,
                             router_weight_on_input, swiglu_limit, expert_range, threads)
    out = np.empty((tokens.size, x.shape[1]), np.float64)
    y = np.empty((tokens.size, topk, x.shape[1]), np.float64) if return_y else None
    _check(_L().orc_moe_forward(*args, _ptr(out), None if y is None else _ptr(y)))
    del keep
    result = {"out": out, "topk_ids": topk_ids, "topk_weights": topk_weights}
    if return_y:
        result["y"] = y
    return result


def assignment_outputs(x, w13, w2, topk: int, assignments, *, logits=None, topk_ids=None, topk_weights=None,
                       w13_scale=None, w2_scale=None, renormalize: bool = True, mx=None,
                       router_weight_on_input: bool = False, swiglu_limit=None, expert_range=None, threads: int = 0):
    """The unweighted expert output of each listed assignment (flat index
    ``t * topk + j``): y [len(assignments), H], same arguments as
    :func:`moe_forward`.  Only the listed assignments are evaluated."""
    x = np.asarray(x)
    topk_ids, topk_weights = _routing(topk, logits, topk_ids, topk_weights, renormalize)
    assignments = np.asarray(assignments, dtype=np.int64)
    tokens, local = np.unique(assignments // topk, return_inverse=True)
    sel = np.ascontiguousarray(local.reshape(-1) * topk + assignments % topk, dtype=np.int64)
    args, keep = _layer_args(x, w13, w2, topk, tokens, topk_ids, topk_weights, w13_scale, w2_scale, mx,
                             router_weight_on_input, swiglu_limit, expert_range, threads)
    y = np.empty((sel.size, x.shape[1]), np.float64)
    _check(_L().orc_assignment_outputs(*args, sel.size, _ptr(sel), _ptr(y)))
    del keep
    return y


def expert_shards(E: int, world_size: int):
    """Contiguous expert ranges ``(first, count)`` of ``world_size`` ranks (reading of [PPLX])."""
    if world_size < 1:
        raise ValueError("need 1 <= world_size <= E")
    first = np.empty(world_size, np.int32)
    count = np.empty(world_size, np.int32)
    _check(_L().orc_expert_shards(E, world_size, _ptr(first), _ptr(count)))
    return [(int(f), int(c)) for f, c in zip(first, count)]


def moe_forward_expert_parallel(x, w13, w2, topk: int, world_size: int, *, w13_scale=None, w2_scale=None,
                                **kw):
    """The layer under expert parallelism ([PPLX] "Experten-Parallel"): each
    rank's bf16 partial over its own experts, then the all-reduce (exact sum of
    the partials, rounded once).  Returns ``out`` and the list ``partials``."""
    partials = []
    for first, count in expert_shards(len(w13), world_size):
        sl = slice(first, first + count)
        r = moe_forward(x, w13[sl], w2[sl], topk, expert_range=(first, count),
                        w13_scale=None if w13_scale is None else w13_scale[sl],
                        w2_scale=None if w2_scale is None else w2_scale[sl], **kw)
        partials.append(np.ascontiguousarray(r["out"]))
    out = np.empty(partials[0].shape, np.float64)
    arr = ctypes.c_void_p * len(partials)
    _L().orc_sum_round_bf16(arr(*[_ptr(p) for p in partials]), len(partials), out.size, _ptr(out))
    return {"out": out, "partials": partials}
