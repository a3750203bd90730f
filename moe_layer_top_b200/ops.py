"""ctypes binding of ``libmoe_b200.so`` (argument marshalling only).

Every function here forwards torch tensors' device pointers and sizes to the C
ABI declared in ``include/moe_b200.h``; all computation happens in the CUDA
kernels.  The library is loaded on first use; if it is missing or cannot be
loaded the call raises ``RuntimeError`` -- there is no fallback path.
"""

from __future__ import annotations

import ctypes
import os
import threading

import torch

_LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libmoe_b200.so")
_lib = None
_lock = threading.Lock()

MOE_OK = 0
MOE_ERR_INVALID = -1
MOE_ERR_UNSUPPORTED = -2
MOE_ERR_WORKSPACE = -3
MOE_ERR_CUDA = -4

MOE_STATUS_OK = 0
MOE_STATUS_BAD_EXPERT_ID = 1
MOE_STATUS_WAIT_TIMEOUT = 0x100

DTYPE_BF16 = 0
DTYPE_FP8_E4M3 = 1
DTYPE_MXFP8_E4M3 = 2

MODE_AUTO = 0
MODE_NORMAL = 1
MODE_SWAP_AB = 2

STAGE_ROUTE, STAGE_ALIGN, STAGE_GATHER, STAGE_GEMM1, STAGE_GEMM2, STAGE_COMBINE = range(6)
NUM_STAGES = 6
STAGE_NAMES = ("route", "align", "gather", "gemm1", "gemm2", "combine")

EXPORTED = (
    "moe_last_error_string", "moe_route", "moe_align_capacity", "moe_align_workspace_size", "moe_align",
    "moe_quantize_weights_fp8", "moe_resolve_problem", "moe_workspace_size", "moe_get_workspace_layout",
    "moe_fused_forward", "moe_forward_stages", "moe_read_status", "moe_version", "moe_align_noalloc",
    "moe_selftest_wait_timeout", "moe_quantize_weights_mxfp8", "moe_combine_allreduce_flag_count",
    "moe_combine_allreduce", "moe_combine_allreduce_emulated", "moe_combine_reduce_scatter_flag_count",
    "moe_combine_reduce_scatter", "moe_combine_reduce_scatter_emulated",
)

MAX_RANKS = 16


class MoeProblem(ctypes.Structure):
    _fields_ = [
        ("T", ctypes.c_int32), ("E", ctypes.c_int32), ("topk", ctypes.c_int32), ("H", ctypes.c_int32),
        ("I", ctypes.c_int32), ("weight_dtype", ctypes.c_int32), ("mode", ctypes.c_int32),
        ("block_m", ctypes.c_int32), ("renormalize", ctypes.c_int32), ("split_k", ctypes.c_int32),
        ("router_weight_on_input", ctypes.c_int32), ("swiglu_limit", ctypes.c_float),
        ("persistent_decode", ctypes.c_int32), ("num_global_experts", ctypes.c_int32),
        ("first_expert", ctypes.c_int32), ("reserved", ctypes.c_int32 * 1),
    ]


class MoeAllreduceRank(ctypes.Structure):
    _fields_ = [("y", ctypes.c_void_p), ("pos_of_flat", ctypes.c_void_p), ("partial", ctypes.c_void_p),
                ("out", ctypes.c_void_p), ("flags", ctypes.c_void_p), ("status", ctypes.c_void_p)]


class MoeWorkspaceLayout(ctypes.Structure):
    _fields_ = [
        ("status", ctypes.c_int64), ("topk_ids", ctypes.c_int64), ("topk_weights", ctypes.c_int64),
        ("sorted_token_ids", ctypes.c_int64), ("expert_ids", ctypes.c_int64),
        ("num_tokens_post_padded", ctypes.c_int64), ("expert_counts", ctypes.c_int64),
        ("expert_offsets", ctypes.c_int64), ("align_scratch", ctypes.c_int64), ("pos_of_flat", ctypes.c_int64),
        ("a1", ctypes.c_int64),
        ("a1_scale", ctypes.c_int64), ("a2", ctypes.c_int64), ("a2_scale", ctypes.c_int64), ("y", ctypes.c_int64),
        ("partials", ctypes.c_int64), ("total_bytes", ctypes.c_int64), ("capacity", ctypes.c_int32), ("block_m", ctypes.c_int32),
        ("mode", ctypes.c_int32), ("align_chunks", ctypes.c_int32),
    ]


def library_path() -> str:
    return _LIB_PATH


def lib():
    """The loaded C library (raises if it is not built or cannot be loaded)."""
    global _lib
    if _lib is not None:
        return _lib
    with _lock:
        if _lib is not None:
            return _lib
        if not os.path.exists(_LIB_PATH):
            raise RuntimeError(f"{_LIB_PATH} is not built: run `python -m moe_layer_top_b200.build`")
        L = ctypes.CDLL(_LIB_PATH)
        vp, i32, i64, sz = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t
        P = ctypes.POINTER(MoeProblem)
        sig = {
            "moe_last_error_string": (ctypes.c_char_p, []),
            "moe_version": (i32, []),
            "moe_route": (ctypes.c_int, [vp, i32, i32, i32, i32, vp, vp, vp]),
            "moe_align_capacity": (i64, [i32, i32, i32, i32]),
            "moe_align_workspace_size": (sz, [i32, i32, i32]),
            "moe_align": (ctypes.c_int, [vp, i32, i32, i32, i32, vp, vp, vp, vp, vp, vp, sz, vp]),
            "moe_align_noalloc": (ctypes.c_int, [vp, i32, i32, i32, i32, vp, vp, vp, vp, vp, vp]),
            "moe_quantize_weights_fp8": (ctypes.c_int, [vp, i64, i32, i32, vp, vp, vp]),
            "moe_quantize_weights_mxfp8": (ctypes.c_int, [vp, i64, i32, i32, vp, vp, vp]),
            "moe_resolve_problem": (ctypes.c_int, [P]),
            "moe_workspace_size": (sz, [P]),
            "moe_get_workspace_layout": (ctypes.c_int, [P, ctypes.POINTER(MoeWorkspaceLayout)]),
            "moe_fused_forward": (ctypes.c_int, [P, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp]),
            "moe_forward_stages": (ctypes.c_int, [P, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, sz, i32, i32, vp]),
            "moe_read_status": (ctypes.c_int, [P, vp, i32, ctypes.POINTER(i32), vp]),
            "moe_selftest_wait_timeout": (ctypes.c_int, [ctypes.c_uint32, vp, vp, vp]),
            "moe_combine_allreduce_flag_count": (i32, [i32, i32]),
            "moe_combine_allreduce": (ctypes.c_int, [i32, i32, i32, i32, i32, ctypes.POINTER(MoeAllreduceRank),
                                                     ctypes.c_uint32, ctypes.c_uint32, vp]),
            "moe_combine_allreduce_emulated": (ctypes.c_int, [i32, i32, i32, i32, ctypes.POINTER(MoeAllreduceRank),
                                                              ctypes.c_uint32, ctypes.c_uint32, vp]),
            "moe_combine_reduce_scatter_flag_count": (i32, [i32, i32]),
            "moe_combine_reduce_scatter": (ctypes.c_int, [i32, i32, i32, i32, i32,
                                                          ctypes.POINTER(MoeAllreduceRank), ctypes.c_uint32,
                                                          ctypes.c_uint32, vp]),
            "moe_combine_reduce_scatter_emulated": (ctypes.c_int, [i32, i32, i32, i32,
                                                                   ctypes.POINTER(MoeAllreduceRank),
                                                                   ctypes.c_uint32, ctypes.c_uint32, vp]),
        }
        for name, (res, args) in sig.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _lib = L
        return L


class MoeError(RuntimeError):
    def __init__(self, code: int, msg: str):
        super().__init__(f"moe error {code}: {msg}")
        self.code = code


def _check(rc: int):
    if rc != MOE_OK:
        raise MoeError(rc, lib().moe_last_error_string().decode(errors="replace"))


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def problem(T, E, topk, H, I, fp8=False, mode=MODE_AUTO, block_m=0, renormalize=True, split_k=True,
            mx=False, router_weight_on_input=False, swiglu_limit=0.0, persistent_decode=False,
            num_global_experts=0, first_expert=0) -> MoeProblem:
    """A moe_problem; ``fp8`` selects E4M3 weights with 128x128 fp32 block scales, ``mx`` MXFP8
    (E4M3 with per-32 E8M0 scales); ``router_weight_on_input`` (top-1 only) scales x by the router
    weight before GEMM1; ``swiglu_limit`` > 0 clamps gate and up before the activation.
    Expert parallelism: ``E`` experts held here, global experts ``[first_expert, first_expert + E)``
    of ``num_global_experts`` that the router scores (0 = ``E``)."""
    p = MoeProblem()
    p.num_global_experts, p.first_expert = int(num_global_experts), int(first_expert)
    p.T, p.E, p.topk, p.H, p.I = int(T), int(E), int(topk), int(H), int(I)
    p.weight_dtype = DTYPE_MXFP8_E4M3 if mx else (DTYPE_FP8_E4M3 if fp8 else DTYPE_BF16)
    p.router_weight_on_input = 1 if router_weight_on_input else 0
    p.swiglu_limit = float(swiglu_limit)
    p.persistent_decode = 1 if persistent_decode else 0
    p.mode, p.block_m, p.renormalize = int(mode), int(block_m), 1 if renormalize else 0
    p.split_k = 0 if split_k else 1
    return p


def resolve_problem(p: MoeProblem) -> MoeProblem:
    q = MoeProblem.from_buffer_copy(p)
    _check(lib().moe_resolve_problem(ctypes.byref(q)))
    return q


def workspace_size(p: MoeProblem) -> int:
    n = lib().moe_workspace_size(ctypes.byref(p))
    if n == 0 and p.T > 0:
        _check(lib().moe_resolve_problem(ctypes.byref(MoeProblem.from_buffer_copy(p))))
    return int(n)


def workspace_layout(p: MoeProblem) -> MoeWorkspaceLayout:
    L = MoeWorkspaceLayout()
    _check(lib().moe_get_workspace_layout(ctypes.byref(p), ctypes.byref(L)))
    return L


def alloc_workspace(p: MoeProblem, device="cuda") -> torch.Tensor:
    """A uint8 device buffer of moe_workspace_size(p) bytes (torch allocations are 256-byte aligned)."""
    return torch.empty(max(workspace_size(p), 256), dtype=torch.uint8, device=device)


def route(logits: torch.Tensor, topk: int, renormalize=True, stream=None):
    T, E = logits.shape
    ids = torch.empty((T, topk), dtype=torch.int32, device=logits.device)
    w = torch.empty((T, topk), dtype=torch.float32, device=logits.device)
    _check(lib().moe_route(_ptr(logits.contiguous()), T, E, topk, 1 if renormalize else 0, _ptr(ids), _ptr(w),
                           _stream(stream)))
    return ids, w


def align_capacity(T, topk, E, block_m) -> int:
    return int(lib().moe_align_capacity(T, topk, E, block_m))


def align(topk_ids: torch.Tensor, E: int, block_m: int, stream=None):
    T, k = topk_ids.shape
    dev = topk_ids.device
    cap = align_capacity(T, k, E, block_m)
    sorted_ids = torch.empty((max(cap, 1),), dtype=torch.int32, device=dev)[:cap]
    expert_ids = torch.empty((max(cap // block_m, 1),), dtype=torch.int32, device=dev)[:cap // block_m]
    ntpp = torch.empty((1,), dtype=torch.int32, device=dev)
    counts = torch.empty((E,), dtype=torch.int32, device=dev)
    offsets = torch.empty((E + 1,), dtype=torch.int32, device=dev)
    ws = torch.empty((max(int(lib().moe_align_workspace_size(T, k, E)), 256),), dtype=torch.uint8, device=dev)
    _check(lib().moe_align(_ptr(topk_ids.contiguous()), T, k, E, block_m, _ptr(sorted_ids), _ptr(expert_ids),
                           _ptr(ntpp), _ptr(counts), _ptr(offsets), _ptr(ws), ws.numel(), _stream(stream)))
    return {"sorted_token_ids": sorted_ids, "expert_ids": expert_ids, "num_tokens_post_padded": ntpp,
            "expert_counts": counts, "expert_offsets": offsets, "capacity": cap, "workspace": ws}


def quantize_weights_fp8(w: torch.Tensor, stream=None):
    """bf16 [..., rows, cols] -> (E4M3 codes as uint8 [..., rows, cols], fp32 scales [..., rows/128, cols/128])."""
    w = w.contiguous()
    *lead, rows, cols = w.shape
    batches = 1
    for d in lead:
        batches *= d
    codes = torch.empty(w.shape, dtype=torch.uint8, device=w.device)
    scales = torch.empty((*lead, rows // 128, cols // 128), dtype=torch.float32, device=w.device)
    _check(lib().moe_quantize_weights_fp8(_ptr(w), batches, rows, cols, _ptr(codes), _ptr(scales), _stream(stream)))
    return codes, scales


def quantize_weights_mxfp8(w: torch.Tensor, stream=None):
    """bf16 [..., rows, cols] -> (E4M3 codes uint8 [..., rows, cols], E8M0 scale factors uint8
    [..., rows * cols / 32] in the SF-atom layout of the header)."""
    w = w.contiguous()
    *lead, rows, cols = w.shape
    batches = 1
    for d in lead:
        batches *= d
    codes = torch.empty(w.shape, dtype=torch.uint8, device=w.device)
    sf = torch.empty((*lead, rows * cols // 32), dtype=torch.uint8, device=w.device)
    _check(lib().moe_quantize_weights_mxfp8(_ptr(w), batches, rows, cols, _ptr(codes), _ptr(sf), _stream(stream)))
    return codes, sf


def sf_atoms_to_rows(sf_atoms: torch.Tensor, rows: int, cols: int) -> torch.Tensor:
    """Re-index SF atoms of [.., rows, cols] into the natural [.., rows, cols/32] order (for tests and tools)."""
    lead = sf_atoms.shape[:-1]
    a = sf_atoms.reshape(*lead, rows // 128, cols // 128, 32, 4, 4)      # [rb, kb, n%32, (n%128)/32, k-group]
    a = a.permute(*range(len(lead)), len(lead), len(lead) + 3, len(lead) + 2, len(lead) + 1, len(lead) + 4)
    return a.reshape(*lead, rows, cols // 32)


def _forward_args(p, x, logits, topk_ids, topk_weights, w13, w2, w13_scale, w2_scale, out, ws):
    return (ctypes.byref(p), _ptr(x), _ptr(logits), _ptr(topk_ids), _ptr(topk_weights), _ptr(w13), _ptr(w2),
            _ptr(w13_scale), _ptr(w2_scale), _ptr(out), _ptr(ws), ws.numel())


def fused_forward(p: MoeProblem, x, w13, w2, *, logits=None, topk_ids=None, topk_weights=None, w13_scale=None,
                  w2_scale=None, out=None, ws=None, stream=None):
    """Run the whole layer; returns ``out`` [T, H] bf16 (allocated if not given)."""
    if out is None:
        out = torch.empty((p.T, p.H), dtype=torch.bfloat16, device=x.device)
    if ws is None:
        ws = alloc_workspace(p, x.device)
    _check(lib().moe_fused_forward(*_forward_args(p, x, logits, topk_ids, topk_weights, w13, w2, w13_scale, w2_scale,
                                                  out, ws), _stream(stream)))
    return out


def forward_stages(p: MoeProblem, x, w13, w2, begin: int, end: int, *, logits=None, topk_ids=None,
                   topk_weights=None, w13_scale=None, w2_scale=None, out=None, ws=None, stream=None):
    _check(lib().moe_forward_stages(*_forward_args(p, x, logits, topk_ids, topk_weights, w13, w2, w13_scale,
                                                   w2_scale, out, ws), begin, end, _stream(stream)))
    return out


def read_status(p: MoeProblem, ws, clear=True, stream=None) -> int:
    st = ctypes.c_int32(-1)
    _check(lib().moe_read_status(ctypes.byref(p), _ptr(ws), 1 if clear else 0, ctypes.byref(st), _stream(stream)))
    return int(st.value)


def workspace_views(p: MoeProblem, ws: torch.Tensor) -> dict:
    """Typed views of the intermediates inside a workspace (for tests and tools)."""
    q = resolve_problem(p)
    L = workspace_layout(q)
    nflat = q.T * q.topk
    cap = L.capacity
    mx = q.weight_dtype == DTYPE_MXFP8_E4M3
    fp8 = q.weight_dtype == DTYPE_FP8_E4M3 or mx
    a1_rows = q.T if q.mode == MODE_SWAP_AB else cap

    def view(off, n, dtype, shape):
        if off < 0:
            return None
        nbytes = n * torch.tensor([], dtype=dtype).element_size()
        return ws[off:off + nbytes].view(dtype).reshape(shape)

    return {
        "status": view(L.status, 1, torch.int32, (1,)),
        "topk_ids": view(L.topk_ids, nflat, torch.int32, (q.T, q.topk)),
        "topk_weights": view(L.topk_weights, nflat, torch.float32, (q.T, q.topk)),
        "sorted_token_ids": view(L.sorted_token_ids, cap, torch.int32, (cap,)),
        "expert_ids": view(L.expert_ids, cap // q.block_m, torch.int32, (cap // q.block_m,)),
        "num_tokens_post_padded": view(L.num_tokens_post_padded, 1, torch.int32, (1,)),
        "expert_counts": view(L.expert_counts, q.E, torch.int32, (q.E,)),
        "expert_offsets": view(L.expert_offsets, q.E + 1, torch.int32, (q.E + 1,)),
        # GEMM1 token rows: sorted copy [cap, H] for normal tiles, one row per token [T, H] for swap-AB
        "a1": view(L.a1, a1_rows * q.H, torch.uint8 if fp8 else torch.bfloat16, (a1_rows, q.H)),
        "pos_of_flat": view(L.pos_of_flat, nflat, torch.int32, (nflat,)),
        "a1_scale_t": None if mx else view(L.a1_scale, cap * (q.H // 128), torch.float32, (q.H // 128, cap)),
        "a1_sf": view(L.a1_scale, cap * q.H // 32, torch.uint8, (cap * q.H // 32,)) if mx else None,
        "a2": view(L.a2, cap * q.I, torch.uint8 if fp8 else torch.bfloat16, (cap, q.I)),
        "a2_scale_t": None if mx else view(L.a2_scale, cap * (q.I // 128), torch.float32, (q.I // 128, cap)),
        "a2_sf": view(L.a2_scale, cap * q.I // 32, torch.uint8, (cap * q.I // 32,)) if mx else None,
        "y": view(L.y, nflat * q.H, torch.bfloat16, (nflat, q.H)),
        "partials": view(L.partials, (L.total_bytes - L.partials) // 4, torch.float32, (-1,)),
        "layout": L,
        "problem": q,
    }


def selftest_wait_timeout(timeout_us: int, stream=None):
    """Run the bounded-wait self-test; returns (status, waited_ns) after a sync."""
    st = torch.zeros((1,), dtype=torch.int32, device="cuda")
    waited = torch.zeros((1,), dtype=torch.int64, device="cuda")
    _check(lib().moe_selftest_wait_timeout(int(timeout_us), _ptr(st), _ptr(waited), _stream(stream)))
    torch.cuda.synchronize()
    return int(st.item()), int(waited.item())


# ----------------------------------------------------------------------------- fused combine + all-reduce
def combine_allreduce_flag_count(T: int, world: int) -> int:
    """int32 entries of each rank's flags array (zero them once before the first call)."""
    return int(lib().moe_combine_allreduce_flag_count(int(T), int(world)))


def _ranks_array(ranks):
    arr = (MoeAllreduceRank * len(ranks))()
    for i, r in enumerate(ranks):
        for name in ("y", "pos_of_flat", "partial", "out", "flags", "status"):
            v = r.get(name)
            setattr(arr[i], name, None if v is None else (v if isinstance(v, int) else v.data_ptr()))
    return arr


def combine_allreduce(T, topk, H, rank, ranks, epoch, timeout_us=2_000_000, stream=None):
    """This rank's fused combine + all-reduce.  ``ranks``: one dict per rank with ``y``,
    ``pos_of_flat``, ``partial``, ``out``, ``flags``, ``status`` -- tensors, or device addresses
    (ints) of peers' buffers as mapped in this process."""
    arr = _ranks_array(ranks)
    _check(lib().moe_combine_allreduce(int(T), int(topk), int(H), len(ranks), int(rank), arr, int(epoch),
                                       int(timeout_us), _stream(stream)))


def combine_allreduce_emulated(T, topk, H, ranks, epoch, timeout_us=2_000_000, stream=None):
    """Every rank's fused combine + all-reduce in one cooperative launch on this GPU (all buffers local)."""
    arr = _ranks_array(ranks)
    _check(lib().moe_combine_allreduce_emulated(int(T), int(topk), int(H), len(ranks), arr, int(epoch),
                                                int(timeout_us), _stream(stream)))


def combine_reduce_scatter_flag_count(T: int, world: int) -> int:
    """int32 entries of each rank's flags array for the reduce-scatter form (T tokens per rank)."""
    return int(lib().moe_combine_reduce_scatter_flag_count(int(T), int(world)))


def combine_reduce_scatter(T, topk, H, rank, ranks, epoch, timeout_us=2_000_000, stream=None):
    """This rank's fused combine + reduce-scatter (T tokens per rank; partial [world*T, H], out [T, H])."""
    arr = _ranks_array(ranks)
    _check(lib().moe_combine_reduce_scatter(int(T), int(topk), int(H), len(ranks), int(rank), arr, int(epoch),
                                            int(timeout_us), _stream(stream)))


def combine_reduce_scatter_emulated(T, topk, H, ranks, epoch, timeout_us=2_000_000, stream=None):
    """Every rank's fused combine + reduce-scatter in one cooperative launch on this GPU."""
    arr = _ranks_array(ranks)
    _check(lib().moe_combine_reduce_scatter_emulated(int(T), int(topk), int(H), len(ranks), arr, int(epoch),
                                                     int(timeout_us), _stream(stream)))

