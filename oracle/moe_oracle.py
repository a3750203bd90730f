"""Plain, slow, obviously correct CPU oracle of the fused top-k MoE layer.

TEST INFRASTRUCTURE ONLY: imported by ``tests/``, ``__graft_entry__.smoke()``
and the CPU-baseline legs of ``bench.py``; never by the product path.  It
shares no code, table or constant generator with the CUDA library.

Arithmetic is numpy float64 except where the method fixes a narrower format;
every rounding point the method names is applied explicitly with the helpers
below, so each function can be read against its source passage.

Sources (web pages the method is taken from):

[AWS]  "AWS erklärt zwei Kernel-Optimierungen, die den Durchsatz von SageMaker
       AI auf H200 steigern" (kinachrichten.com).
[PR]   "[vllm] vLLM, H200 GPU를 위한 FP8 MoE 다운 프로젝션 최적화: TMA 활용 및
       커널 퓨전으로 7.6% 처리량 향상" -- analysis of vLLM PR #64760
       (blog.secrett2633.cloud).
[PPLX] "Hosting von Qwen auf Blackwell" (perplexity.ai).

Readings where the pages are silent:

* route: experts are chosen on the raw logits (softmax is monotone), equal
  logits go to the lower expert index; weights are the softmax over all
  experts, renormalised over the chosen ones.
* align: inside one expert the flat assignment ids ``t*topk + j`` keep their
  ascending order; padding slots hold the sentinel ``T*topk``; empty experts
  own no block; block ids past the used ones are -1.
* the GEMM1 input x is quantised with the same per-(row,128) power-of-two rule
  the page gives for the intermediate.
* weight block scale: ``max(blockmax, 1e-10) / 448`` in fp32, element code
  ``e4m3(fp32(w / scale))``.
* combine: ``out[t] = sum_j w[t,j] * y[t,j]`` exactly (float64 here), rounded
  once to bf16; duplicate expert ids in a row are independent assignments.
* MXFP8: one E8M0 scale per 32 consecutive elements of a row, chosen by the
  same power-of-two rule as the per-(row,128) activation scale.
* expert parallelism: rank r of N holds the contiguous experts
  [floor(r*E/N), floor((r+1)*E/N)); each rank's output is the bf16 rounding of
  its own assignments' sum; the all-reduce is the exact sum of those bf16
  partials, rounded once.

Parity pins for every function live in ``tests/test_oracle_*.py``.
"""

from __future__ import annotations

import numpy as np

__all__ = [
    "BF16_MAX",
    "E4M3_MAX",
    "round_bf16",
    "e4m3_round",
    "e4m3_encode",
    "e4m3_decode",
    "pow2_ceil",
    "quantize_act_group128",
    "dequantize_act_group128",
    "quantize_weight_block128",
    "dequantize_weight_block128",
    "route",
    "align_capacity",
    "align",
    "expert_mlp",
    "moe_forward",
    "expert_shards",
    "moe_forward_expert_parallel",
]

# bfloat16: 1 sign, 8 exponent, 7 stored mantissa bits (8 significant bits).
BF16_MAX = float((2.0 - 2.0 ** -7) * 2.0 ** 127)
# OCP 8-bit floating point, E4M3 ("fn": no infinities, S.1111.111 is NaN).
E4M3_MAX = 448.0
_F32_1E_10 = np.float32(1e-10)
_F32_INV_448 = np.float32(1.0 / 448.0)


# ----------------------------------------------------------------------------
# number formats
# ----------------------------------------------------------------------------

MX_GROUP = 32          # elements per MXFP8 scale
E8M0_BIAS = 127        # E8M0 byte of the scale 2**0


def round_bf16(x) -> np.ndarray:
    """Round to the nearest bfloat16 value, ties to even; result as float64.

    bfloat16 keeps 8 significant bits over the binary32 exponent range, so the
    spacing of values with leading-bit weight 2**(e-1) is 2**(e-8); below the
    smallest normal 2**-126 the spacing is fixed at 2**-133.  Values that
    round past the largest finite bfloat16 become infinite.
    """
    x = np.asarray(x, dtype=np.float64)
    out = np.array(x, dtype=np.float64, copy=True)
    sel = np.isfinite(x) & (x != 0.0)
    if np.any(sel):
        _, e = np.frexp(x[sel])            # x = m * 2**e with 0.5 <= |m| < 1
        q_exp = np.maximum(e - 8, -133)     # exponent of one unit in the last place
        out[sel] = np.ldexp(np.rint(np.ldexp(x[sel], -q_exp)), q_exp)
    big = np.isfinite(out) & (np.abs(out) > BF16_MAX)
    out[big] = np.copysign(np.inf, out[big])
    return out


def e4m3_round(x) -> np.ndarray:
    """Nearest E4M3 value, ties to even, saturating at +-448; float64 result.

    E4M3 has 4 significant bits (1 implicit + 3 stored), exponent bias 7, the
    smallest normal 2**-6 and subnormal spacing 2**-9.  Saturation (instead of
    NaN) matches the clamp to +-448 the fused quantisation kernel applies
    ([PR] §1.2).  The sign of a result that rounds to zero is kept.
    """
    x = np.asarray(x, dtype=np.float64)
    out = np.array(x, dtype=np.float64, copy=True)
    sel = np.isfinite(x) & (x != 0.0)
    if np.any(sel):
        _, e = np.frexp(x[sel])
        q_exp = np.maximum(e - 4, -9)
        out[sel] = np.ldexp(np.rint(np.ldexp(x[sel], -q_exp)), q_exp)
    fin = np.isfinite(out)
    out[fin] = np.clip(out[fin], -E4M3_MAX, E4M3_MAX)
    return out


def _e4m3_value_table() -> np.ndarray:
    """Value of every one of the 256 E4M3 codes, from the format definition."""
    vals = np.empty(256, dtype=np.float64)
    for code in range(256):
        sign = -1.0 if code & 0x80 else 1.0
        exp_field = (code >> 3) & 0xF
        mant = code & 0x7
        if exp_field == 0xF and mant == 0x7:
            vals[code] = np.nan
        elif exp_field == 0:
            vals[code] = sign * mant * 2.0 ** -9
        else:
            vals[code] = sign * (1.0 + mant / 8.0) * 2.0 ** (exp_field - 7)
    return vals


_E4M3_VALUES = _e4m3_value_table()


def e4m3_decode(codes) -> np.ndarray:
    """E4M3 byte codes -> float64 values."""
    return _E4M3_VALUES[np.asarray(codes, dtype=np.uint8)]


def e4m3_encode(x) -> np.ndarray:
    """Round ``x`` with :func:`e4m3_round` and return the uint8 codes."""
    v = e4m3_round(x)
    a = np.abs(v)
    code = np.zeros(v.shape, dtype=np.int64)
    normal = a >= 2.0 ** -6
    if np.any(normal):
        _, e = np.frexp(a[normal])                  # leading bit weight 2**(e-1)
        exp_field = e - 1 + 7
        mant = np.rint((np.ldexp(a[normal], -(e - 1)) - 1.0) * 8.0).astype(np.int64)
        code[normal] = (exp_field << 3) | mant
    sub = (~normal) & (a > 0)
    code[sub] = np.rint(np.ldexp(a[sub], 9)).astype(np.int64)
    code |= np.signbit(v).astype(np.int64) << 7
    return code.astype(np.uint8)


def pow2_ceil(s) -> np.ndarray:
    """Smallest power of two that is >= s (s > 0), computed exactly.

    [PR] §1.2 writes this as ``exp2(ceil(log2(s)))``; here it is taken from
    the binary exponent so that exact powers of two map to themselves.
    """
    s = np.asarray(s, dtype=np.float64)
    m, e = np.frexp(s)                              # s = m * 2**e, 0.5 <= m < 1
    return np.where(m == 0.5, np.ldexp(1.0, e - 1), np.ldexp(1.0, e))


# ----------------------------------------------------------------------------
# FP8 quantisation rules
# ----------------------------------------------------------------------------

def quantize_act_group128(v):
    """Per (row, 128 consecutive columns) FP8 quantisation with a power-of-two scale.

    [PR] §1.2, fused SiLU·mul·quant kernel: ``amax`` over the group, raw scale
    ``max(amax, 1e-10) * (1/448)`` in fp32, scale = the smallest power of two
    at or above it, code = ``e4m3(clamp(v / scale, -448, 448))``.  The same
    rule quantises the GEMM1 input x (reading; the pages do not show it).

    v: float64 [rows, K] holding fp32-representable values, K % 128 == 0.
    Returns (codes uint8 [rows, K], scales float32 [rows, K // 128]).
    """
    v = np.asarray(v, dtype=np.float64)
    rows, k = v.shape
    if k % 128:
        raise ValueError("K must be a multiple of 128")
    g = v.reshape(rows, k // 128, 128)
    amax = np.abs(g).max(axis=-1).astype(np.float32)
    raw = np.maximum(amax, _F32_1E_10) * _F32_INV_448          # one fp32 rounding
    scale = pow2_ceil(raw.astype(np.float64))
    q = np.clip(g / scale[..., None], -E4M3_MAX, E4M3_MAX)     # exact: scale is 2**n
    codes = e4m3_encode(q).reshape(rows, k)
    return codes, scale.astype(np.float32)


def dequantize_act_group128(codes, scales) -> np.ndarray:
    codes = np.asarray(codes)
    rows, k = codes.shape
    vals = e4m3_decode(codes).reshape(rows, k // 128, 128)
    return (vals * np.asarray(scales, dtype=np.float64)[..., None]).reshape(rows, k)


def quantize_weight_block128(w):
    """FP8 E4M3 weights with one fp32 scale per 128x128 block.

    Workload definition: ``scale = blockmax / 448`` (fp32; floored at 1e-10
    as a reading), element code ``e4m3(fp32(w / scale))``.

    w: float64 [..., N, K] (bf16 values), N and K multiples of 128.
    Returns (codes uint8 [..., N, K], scales float32 [..., N//128, K//128]).
    """
    w = np.asarray(w, dtype=np.float64)
    *lead, n, k = w.shape
    if n % 128 or k % 128:
        raise ValueError("N and K must be multiples of 128")
    blocks = w.reshape(*lead, n // 128, 128, k // 128, 128)
    bmax = np.abs(blocks).max(axis=(-3, -1)).astype(np.float32)
    scale = np.maximum(bmax, _F32_1E_10) / np.float32(448.0)    # fp32 division
    ratio = blocks.astype(np.float32) / scale[..., :, None, :, None]  # fp32 division
    codes = e4m3_encode(ratio.astype(np.float64)).reshape(*lead, n, k)
    return codes, scale.astype(np.float32)


def dequantize_weight_block128(codes, scales) -> np.ndarray:
    codes = np.asarray(codes)
    scales = np.asarray(scales, dtype=np.float64)
    vals = e4m3_decode(codes)
    full = np.repeat(np.repeat(scales, 128, axis=-2), 128, axis=-1)
    return vals * full


def quantize_mx_group32(v):
    """MXFP8: E4M3 elements with one power-of-two (E8M0) scale per 32 consecutive
    elements of a row.

    [PPLX] "Quantisierung": Blackwell's micro-scaling formats; Qwen3-235B is
    served with MXFP8 weights.  The page names the scheme but not its scale
    rule.  Reading: the power-of-two rule of [PR] §1.2 (raw scale
    ``max(amax, 1e-10) * (1/448)`` in fp32, scale = the smallest power of two
    at or above it) on 32-element groups -- an E8M0 byte holds exactly the
    powers of two, and this choice never clips the group maximum.  The same
    rule serves weights (groups along K of each row) and activations.

    v: float64 [..., K] holding fp32-representable values, K % 32 == 0.
    Returns (codes uint8 [..., K], e8m0 uint8 [..., K // 32]) with
    scale = 2 ** (e8m0 - 127).
    """
    v = np.asarray(v, dtype=np.float64)
    *lead, k = v.shape
    if k % MX_GROUP:
        raise ValueError("K must be a multiple of 32")
    g = v.reshape(*lead, k // MX_GROUP, MX_GROUP)
    amax = np.abs(g).max(axis=-1).astype(np.float32)
    raw = np.maximum(amax, _F32_1E_10) * _F32_INV_448          # one fp32 rounding
    scale = pow2_ceil(raw.astype(np.float64))
    q = np.clip(g / scale[..., None], -E4M3_MAX, E4M3_MAX)     # exact: scale is 2**n
    codes = e4m3_encode(q).reshape(*lead, k)
    exponent = np.frexp(scale)[1] - 1                           # scale == 2**exponent
    return codes, (exponent + E8M0_BIAS).astype(np.uint8)


def mx_scale(e8m0) -> np.ndarray:
    """E8M0 byte -> its power-of-two value (the NaN byte 0xFF is never produced)."""
    return np.ldexp(1.0, np.asarray(e8m0).astype(np.int64) - E8M0_BIAS)


def dequantize_mx_group32(codes, e8m0) -> np.ndarray:
    codes = np.asarray(codes)
    *lead, k = codes.shape
    vals = e4m3_decode(codes).reshape(*lead, k // MX_GROUP, MX_GROUP)
    return (vals * mx_scale(e8m0)[..., None]).reshape(*lead, k)


# ----------------------------------------------------------------------------
# routing and alignment
# ----------------------------------------------------------------------------

def route(logits, topk: int, renormalize: bool = True):
    """Top-k softmax router.

    [AWS] "Warum MoE-Kernel so wichtig sind" (token routing inside fused MoE)
    and the workload recipe: softmax over the E experts, keep the k largest,
    renormalise them to sum to one.  Experts are picked on the raw logits in
    descending order, equal logits by the lower index.

    logits: float32 [T, E].  Returns (topk_ids int32 [T, k], topk_weights float32 [T, k]).
    """
    logits = np.asarray(logits, dtype=np.float32)
    t, e = logits.shape
    if not 1 <= topk <= e:
        raise ValueError("need 1 <= topk <= E")
    order = np.argsort(-logits, axis=1, kind="stable")          # stable: lower index first on ties
    ids = order[:, :topk].astype(np.int32)
    l64 = logits.astype(np.float64)
    p = np.exp(l64 - l64.max(axis=1, keepdims=True))
    p = p / p.sum(axis=1, keepdims=True)                         # softmax over all experts
    chosen = np.take_along_axis(p, ids.astype(np.int64), axis=1)
    if renormalize:
        chosen = chosen / chosen.sum(axis=1, keepdims=True)
    return ids, chosen.astype(np.float32)


def align_capacity(T: int, topk: int, E: int, block_m: int) -> int:
    """Length of ``sorted_token_ids``: an upper bound of the padded row count.

    Every non-empty expert pads its count up to a multiple of ``block_m``,
    adding at most ``block_m - 1`` slots, and at most ``min(E, T*topk)``
    experts are non-empty.  Rounded up to whole blocks.
    """
    n = T * topk
    if n == 0:
        return 0
    bound = n + min(E, n) * (block_m - 1)
    return -(-bound // block_m) * block_m


def align(topk_ids, E: int, block_m: int, first_expert: int = 0, num_global_experts=None):
    """Expert-sorted, block-padded permutation of the flat assignments.

    [PR] §1.1: ``sorted_token_ids`` (flat ids ``t*topk + j`` grouped by expert,
    each expert's group padded to a multiple of BLOCK_SIZE_M),
    ``num_tokens_post_padded`` and one expert per block.  Readings: stable
    order inside an expert, sentinel ``T*topk`` in padding, -1 past the last
    used block.

    Expert parallelism ([PPLX] "MoE Dispatch - Combine", "Experten-Parallel":
    the dispatch keeps the tokens routed to this rank's experts): the ids are
    global, in ``[0, num_global_experts)``; only those in
    ``[first_expert, first_expert + E)`` are kept, as local experts
    ``id - first_expert``; the others are skipped.
    """
    ids = np.asarray(topk_ids).astype(np.int64)
    t, k = ids.shape
    n_global = E if num_global_experts is None else int(num_global_experts)
    g = ids.reshape(-1)
    n = g.size
    if n and (g.min() < 0 or g.max() >= n_global):
        raise ValueError("expert id out of range")
    flat = g - first_expert                      # local id; outside [0, E) = another rank's expert
    flat = np.where((flat >= 0) & (flat < E), flat, -1)
    counts = np.bincount(flat[flat >= 0], minlength=E).astype(np.int64)
    padded = -(-counts // block_m) * block_m
    offsets = np.zeros(E + 1, dtype=np.int64)
    offsets[1:] = np.cumsum(padded)
    cap = align_capacity(t, k, E, block_m)
    sorted_ids = np.full(cap, n, dtype=np.int32)
    expert_ids = np.full(cap // block_m, -1, dtype=np.int32)
    for e in range(E):
        members = np.nonzero(flat == e)[0]                       # ascending flat order
        sorted_ids[offsets[e]:offsets[e] + members.size] = members
        expert_ids[offsets[e] // block_m:offsets[e + 1] // block_m] = e
    return {
        "sorted_token_ids": sorted_ids,
        "expert_ids": expert_ids,
        "num_tokens_post_padded": int(offsets[E]),
        "expert_counts": counts.astype(np.int32),
        "expert_offsets": offsets.astype(np.int32),
        "capacity": cap,
    }


# ----------------------------------------------------------------------------
# expert MLP and the layer
# ----------------------------------------------------------------------------

def expert_mlp(x_hat, w13_hat, w2_hat, requant, return_intermediates: bool = False, swiglu_limit=None):
    """One expert's SiLU-gated MLP on a batch of rows.

    [PR] §1.1/§1.2: ``h = x · w13ᵀ`` held in bf16 (``intermediate_cache1``);
    gate = columns [0, I), up = columns [I, 2I); ``silu(gate)`` rounded to
    bf16 before it multiplies ``up``; the product rounded to bf16; for the
    FP8 path it is re-quantised per (row, 128) before the down projection
    ``y = a2 · w2ᵀ`` (``requant=True``), for MXFP8 per (row, 32) with an E8M0
    scale (``requant="mx"``), for bf16 kept as is (``requant=False``).

    swiglu_limit L: [PR] names a SwiGLU ``clamp_limit`` (its presence turns the
    fused path off) but not its formula.  Reading: gate = min(gate, L) and
    up = clamp(up, -L, L) on the bf16 values, before the activation.

    x_hat [n, H], w13_hat [2I, H], w2_hat [H, I]: float64.  Returns y [n, H].
    """
    i = w13_hat.shape[0] // 2
    h = round_bf16(x_hat @ w13_hat.T)
    gate, up = h[:, :i], h[:, i:]
    if swiglu_limit is not None:
        lim = float(np.float32(swiglu_limit))
        gate = np.minimum(gate, lim)
        up = np.clip(up, -lim, lim)
    act = round_bf16(gate / (1.0 + np.exp(-gate)))
    p = round_bf16(act * up)
    if requant == "mx":
        codes, scales = quantize_mx_group32(p)
        p_hat = dequantize_mx_group32(codes, scales)
    elif requant:
        codes, scales = quantize_act_group128(p)
        p_hat = dequantize_act_group128(codes, scales)
    else:
        codes = scales = None
        p_hat = p
    y = p_hat @ w2_hat.T
    if return_intermediates:
        return y, {"h": h, "p": p, "a2_codes": codes, "a2_scales": scales}
    return y


def moe_forward(x, w13, w2, topk: int, *, logits=None, topk_ids=None, topk_weights=None,
                w13_scale=None, w2_scale=None, renormalize: bool = True, tokens=None,
                return_y: bool = False, mx=None, router_weight_on_input: bool = False, swiglu_limit=None,
                expert_range=None):
    """The fused MoE layer: route -> experts -> top-k weighted combine.

    [AWS] "Warum MoE-Kernel so wichtig sind": one operation that routes each
    token, runs the chosen experts and combines; [PPLX] "MoE Dispatch -
    Combine": the combine is a weighted accumulation of the expert outputs.

    x:   [T, H] float (bf16 values).
    w13: [E, 2I, H] bf16 values (float) -- or E4M3 codes (uint8) with
         ``w13_scale`` [E, 2I/128, H/128] float32 for the FP8 block-quantised
         path, or ``w13_scale`` [E, 2I, H/32] uint8 (E8M0) for MXFP8, where x
         and the intermediate are MX-quantised too.
    w2:  [E, H, I] likewise with ``w2_scale`` [E, H/128, I/128] or [E, H, I/32].
    Routing: ``logits`` [T, E] float32, or ``topk_ids``/``topk_weights``.
    tokens: optional subset of token indices to evaluate (each output row
    depends only on its own token, its routing and the weights).
    mx: MXFP8 scales (taken from the scale dtype, uint8, when not given).
    router_weight_on_input: [PR]'s test passes ``apply_router_weight_on_input``
    (False there).  Reading: with top-1 routing each token row becomes
    bf16(fp32(x) * w) before the experts and the expert output is not weighted
    again; top-k > 1 is rejected (a non-linear expert cannot take the weight
    on its input without changing the layer).
    swiglu_limit: see :func:`expert_mlp`.
    expert_range: ``(first, count)`` for expert parallelism ([PPLX]
    "Experten-Parallel": each rank accumulates the contributions of its own
    experts before an all-reduce).  ``w13``/``w2`` (and their scales) then
    hold the experts ``[first, first + count)`` only, indexed from zero, the
    routing is over all experts, and ``out`` is the bf16 rounding of the sum
    over the token's assignments to those experts (zero when there are none).

    Returns a dict with ``out`` [len(tokens), H] (float64 holding bf16
    values), ``topk_ids``, ``topk_weights`` and, when asked, ``y``
    [len(tokens), topk, H] before the weights are applied.
    """
    x = np.asarray(x, dtype=np.float64)
    fp8 = w13_scale is not None
    if fp8 != (w2_scale is not None):
        raise ValueError("w13_scale and w2_scale go together")
    mx = fp8 and (bool(mx) if mx is not None else np.asarray(w13_scale).dtype == np.uint8)
    if logits is not None:
        topk_ids, topk_weights = route(logits, topk, renormalize)
    topk_ids = np.asarray(topk_ids).astype(np.int64)
    topk_weights = np.asarray(topk_weights, dtype=np.float32)
    t_all, h_dim = x.shape
    tokens = np.arange(t_all) if tokens is None else np.asarray(tokens, dtype=np.int64)

    xs = x[tokens]
    if router_weight_on_input:
        if topk != 1:
            raise ValueError("router_weight_on_input needs topk == 1")
        w_in = np.asarray(topk_weights, dtype=np.float32)[tokens, 0]
        xs = round_bf16((xs.astype(np.float32) * w_in[:, None]).astype(np.float64))   # one fp32 product
    if mx:
        qx, sx = quantize_mx_group32(xs)
        x_hat = dequantize_mx_group32(qx, sx)
    elif fp8:
        qx, sx = quantize_act_group128(xs)
        x_hat = dequantize_act_group128(qx, sx)
    else:
        x_hat = xs

    ids = topk_ids[tokens]
    base, count = (0, None) if expert_range is None else (int(expert_range[0]), int(expert_range[1]))
    wts = topk_weights[tokens].astype(np.float64)
    acc = np.zeros((tokens.size, h_dim), dtype=np.float64)
    y_all = np.zeros((tokens.size, topk, h_dim), dtype=np.float64) if return_y else None
    for g in np.unique(ids):
        e = g - base                                             # index into the weights given
        if count is not None and not 0 <= e < count:
            continue                                             # another rank's expert
        rows, cols = np.nonzero(ids == g)                        # (token, slot) pairs on expert g
        if mx:
            w13_e = dequantize_mx_group32(w13[e], w13_scale[e])
            w2_e = dequantize_mx_group32(w2[e], w2_scale[e])
        elif fp8:
            w13_e = dequantize_weight_block128(w13[e], w13_scale[e])
            w2_e = dequantize_weight_block128(w2[e], w2_scale[e])
        else:
            w13_e = np.asarray(w13[e], dtype=np.float64)
            w2_e = np.asarray(w2[e], dtype=np.float64)
        y = expert_mlp(x_hat[rows], w13_e, w2_e, requant="mx" if mx else fp8, swiglu_limit=swiglu_limit)
        for r, c, yr in zip(rows, cols, y):
            acc[r] += (1.0 if router_weight_on_input else wts[r, c]) * yr
            if return_y:
                y_all[r, c] = yr
    result = {
        "out": round_bf16(acc),
        "topk_ids": topk_ids.astype(np.int32),
        "topk_weights": topk_weights,
    }
    if return_y:
        result["y"] = y_all
    return result


def expert_shards(E: int, world_size: int):
    """Contiguous expert ranges ``(first, count)`` of ``world_size`` ranks.

    [PPLX] "Hosting von Qwen auf Blackwell" shards 128 experts over EP=4/8/16
    ranks without saying how.  Reading: rank r holds experts
    ``[floor(r*E/N), floor((r+1)*E/N))`` -- contiguous, sizes differing by at
    most one.
    """
    if world_size < 1 or world_size > E:
        raise ValueError("need 1 <= world_size <= E")
    bounds = [(r * E) // world_size for r in range(world_size + 1)]
    return [(bounds[r], bounds[r + 1] - bounds[r]) for r in range(world_size)]


def moe_forward_expert_parallel(x, w13, w2, topk: int, world_size: int, *, w13_scale=None, w2_scale=None,
                                **kw):
    """The layer under expert parallelism ([PPLX] "Experten-Parallel"): x and
    the routing replicated on every rank, each rank's bf16 partial sum over its
    own experts (:func:`moe_forward` with ``expert_range``), then an
    all-reduce (sum) of the partials over the ranks.

    Reading: the all-reduce is the exact sum of the bf16 partials, rounded once
    to bf16 (a collective may round in another order; the difference is within
    bf16 rounding of the summands).  Returns a dict with ``out`` and the list
    ``partials``.
    """
    partials = []
    for first, count in expert_shards(len(w13), world_size):
        sl = slice(first, first + count)
        r = moe_forward(x, w13[sl], w2[sl], topk, expert_range=(first, count),
                        w13_scale=None if w13_scale is None else w13_scale[sl],
                        w2_scale=None if w2_scale is None else w2_scale[sl], **kw)
        partials.append(r["out"])
    return {"out": round_bf16(np.sum(partials, axis=0)), "partials": partials}

