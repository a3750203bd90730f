"""The C-ABI library loads, exports every symbol the header declares, and
rejects bad arguments on the host before touching the device (no GPU needed)."""

import ctypes
import os
import re

import pytest

from moe_layer_top_b200 import ops

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "moe_b200.h")


def _declared():
    with open(HEADER) as f:
        text = f.read()
    return sorted(set(re.findall(r"^MOE_API\s+[\w\s\*]+?\b(moe_\w+)\(", text, flags=re.M)))


@pytest.fixture(scope="module")
def L():
    if not os.path.exists(ops.library_path()):
        from moe_layer_top_b200 import build
        build.build()
    return ops.lib()


def test_header_declares_the_boundary():
    names = _declared()
    for required in ("moe_route", "moe_align_capacity", "moe_align", "moe_workspace_size", "moe_fused_forward"):
        assert required in names
    assert set(names) == set(ops.EXPORTED)


def test_library_exports_every_declared_symbol(L):
    for name in _declared():
        assert hasattr(L, name), name
    assert L.moe_version() == 200


def test_struct_sizes_match_header():
    assert ctypes.sizeof(ops.MoeProblem) == 16 * 4
    assert ctypes.sizeof(ops.MoeWorkspaceLayout) == 17 * 8 + 4 * 4


def test_align_capacity_formula(L):
    assert ops.align_capacity(1, 8, 128, 16) == 128
    assert ops.align_capacity(0, 8, 128, 16) == 0
    assert ops.align_capacity(16, 2, 8, 128) == 128 * ((32 + 8 * 127 + 127) // 128)
    assert L.moe_align_capacity(-1, 8, 128, 16) == -1
    from oracle import moe_oracle as O
    for args in [(1, 8, 128, 16), (64, 8, 128, 16), (256, 8, 128, 32), (16384, 8, 128, 128), (37, 3, 5, 64)]:
        assert ops.align_capacity(*args) == O.align_capacity(*args)


def test_resolve_problem_auto_modes(L):
    q = ops.resolve_problem(ops.problem(1, 128, 8, 4096, 1536))
    assert q.mode == ops.MODE_SWAP_AB and q.block_m == 16
    q = ops.resolve_problem(ops.problem(16384, 128, 8, 4096, 1536, fp8=True))
    assert q.mode == ops.MODE_NORMAL and q.block_m == 128
    q = ops.resolve_problem(ops.problem(16384, 128, 8, 4096, 1536, fp8=False))
    assert q.mode == ops.MODE_NORMAL and q.block_m == 128
    q = ops.resolve_problem(ops.problem(64, 128, 8, 4096, 1536, mode=ops.MODE_NORMAL))
    assert q.block_m == 128
    q = ops.resolve_problem(ops.problem(64, 128, 8, 4096, 1536, block_m=32))
    assert q.mode == ops.MODE_SWAP_AB and q.block_m == 32


@pytest.mark.parametrize("T,E,H,I,want", [
    (255, 128, 4096, 1536, ("swap", 32)),    # 15.9 expected tokens per expert
    (256, 128, 4096, 1536, ("normal", 128)),  # 16: the switch point
    (128, 128, 4096, 1536, ("swap", 16)),     # 8
    (129, 128, 4096, 1536, ("swap", 32)),     # just above 8
    (511, 256, 7168, 2048, ("swap", 32)),
    (512, 256, 7168, 2048, ("normal", 128)),
    (32, 256, 7168, 2048, ("swap", 16)),
])
def test_resolve_problem_orientation_switch(L, T, E, H, I, want):
    # swap-AB below 16 expected tokens per hit expert (T*k/E under even routing), 128-row tiles from 16 on
    for fp8 in (False, True):
        q = ops.resolve_problem(ops.problem(T, E, 8, H, I, fp8=fp8))
        got = ("swap" if q.mode == ops.MODE_SWAP_AB else "normal", q.block_m)
        assert got == want, (T, E, fp8, got)


def test_resolve_problem_mxfp8_is_normal_128(L):
    for T in (1, 64, 16384):
        q = ops.resolve_problem(ops.problem(T, 128, 8, 4096, 1536, mx=True))
        assert q.weight_dtype == ops.DTYPE_MXFP8_E4M3 and q.mode == ops.MODE_NORMAL and q.block_m == 128
    p = ops.problem(16, 8, 2, 256, 128, mx=True, mode=ops.MODE_SWAP_AB)
    assert L.moe_workspace_size(ctypes.byref(p)) == 0
    p = ops.problem(16, 8, 2, 256, 128, mx=True, block_m=64)
    assert L.moe_workspace_size(ctypes.byref(p)) == 0
    # activation scale regions: the SF atoms take exactly the bytes of the fp32 K-block scales
    lay_mx = ops.workspace_layout(ops.problem(300, 16, 4, 1024, 512, mx=True))
    lay_f8 = ops.workspace_layout(ops.problem(300, 16, 4, 1024, 512, fp8=True, mode=ops.MODE_NORMAL))
    assert lay_mx.total_bytes == lay_f8.total_bytes and lay_mx.a1_scale >= 0 and lay_mx.a2_scale >= 0


def test_normal_tiles_need_h_multiple_of_256(L):
    q = ops.resolve_problem(ops.problem(16384, 8, 2, 384, 128))          # many tokens, but H % 256 == 128
    assert q.mode == ops.MODE_SWAP_AB
    for kw in (dict(mode=ops.MODE_NORMAL), dict(block_m=128), dict(mx=True)):
        p = ops.problem(64, 8, 2, 384, 128, **kw)
        assert L.moe_workspace_size(ctypes.byref(p)) == 0
    assert L.moe_workspace_size(ctypes.byref(ops.problem(64, 8, 2, 512, 128, mode=ops.MODE_NORMAL))) > 0


def test_epilogue_variant_validation(L):
    ok = ops.problem(16, 8, 1, 256, 128, router_weight_on_input=True)
    assert L.moe_workspace_size(ctypes.byref(ok)) > 0
    bad = ops.problem(16, 8, 2, 256, 128, router_weight_on_input=True)      # needs top-1
    assert L.moe_workspace_size(ctypes.byref(bad)) == 0
    assert L.moe_workspace_size(ctypes.byref(ops.problem(16, 8, 2, 256, 128, swiglu_limit=7.0))) > 0
    for lim in (-1.0, float("inf"), float("nan")):
        assert L.moe_workspace_size(ctypes.byref(ops.problem(16, 8, 2, 256, 128, swiglu_limit=lim))) == 0
    p = ops.problem(16, 8, 2, 256, 128)
    p.router_weight_on_input = 2
    assert L.moe_workspace_size(ctypes.byref(p)) == 0


def test_quantize_mxfp8_argument_errors(L):
    g = _fake(1 << 20)
    assert L.moe_quantize_weights_mxfp8(g, 1, 100, 128, g, g, None) == ops.MOE_ERR_INVALID
    assert L.moe_quantize_weights_mxfp8(g, 1, 128, 128, None, g, None) == ops.MOE_ERR_INVALID
    assert L.moe_quantize_weights_mxfp8(g, 1, 128, 128, g, _fake((1 << 20) + 4), None) == ops.MOE_ERR_INVALID
    p = ops.problem(16, 8, 2, 256, 128, mx=True)
    need = ops.workspace_size(p)
    # MXFP8 scale factors must be 16-byte aligned (bulk copies read whole 512-byte atoms)
    assert L.moe_fused_forward(ctypes.byref(p), g, g, None, None, g, g, _fake((1 << 20) + 4), g, g, g, need,
                               None) == ops.MOE_ERR_INVALID


@pytest.mark.parametrize("bad", [
    dict(T=-1), dict(E=0), dict(E=2000), dict(topk=0), dict(topk=9, E=8), dict(H=100), dict(I=0), dict(I=200),
    dict(mode=7), dict(mode=ops.MODE_NORMAL, block_m=16), dict(mode=ops.MODE_SWAP_AB, block_m=128),
    dict(block_m=48), dict(mode=ops.MODE_NORMAL, block_m=256), dict(block_m=256),
    dict(block_m=256, mode=ops.MODE_NORMAL, fp8=True),
])
def test_invalid_problems_are_rejected(L, bad):
    kw = dict(T=16, E=8, topk=2, H=256, I=128)
    kw.update(bad)
    p = ops.problem(kw["T"], kw["E"], kw["topk"], kw["H"], kw["I"], mode=kw.get("mode", 0),
                    block_m=kw.get("block_m", 0), fp8=kw.get("fp8", False))
    assert L.moe_workspace_size(ctypes.byref(p)) == 0
    with pytest.raises(ops.MoeError) as ei:
        ops.resolve_problem(p)
    assert ei.value.code == ops.MOE_ERR_INVALID


def test_workspace_layout_is_aligned_and_ordered(L):
    for fp8 in (False, True):
        p = ops.problem(64, 128, 8, 4096, 1536, fp8=fp8)
        lay = ops.workspace_layout(p)
        offs = [lay.status, lay.topk_ids, lay.topk_weights, lay.sorted_token_ids, lay.expert_ids,
                lay.num_tokens_post_padded, lay.expert_counts, lay.expert_offsets, lay.align_scratch, lay.a1,
                lay.a2, lay.y]
        offs = [o for o in offs if o >= 0]          # -1: a region this problem does not use
        assert all(o % 256 == 0 for o in offs)
        assert offs == sorted(offs)
        assert (lay.a1 >= 0) == fp8 and (lay.pos_of_flat >= 0) == fp8   # bf16 GEMM1 gathers from x itself
        assert (lay.a1_scale >= 0) == fp8 and (lay.a2_scale >= 0) == fp8
        assert lay.total_bytes == ops.workspace_size(p)
        assert lay.y + 64 * 8 * 4096 * 2 <= lay.total_bytes


def _fake(addr):
    return ctypes.c_void_p(addr)


def test_forward_argument_errors_before_any_launch(L):
    p = ops.problem(16, 8, 2, 256, 128)
    need = ops.workspace_size(p)
    good = _fake(1 << 20)
    args = lambda **o: [ctypes.byref(p), o.get("x", good), o.get("logits", good), None, None,
                        o.get("w13", good), o.get("w2", good), None, None, o.get("out", good), o.get("ws", good),
                        o.get("nbytes", need), None]
    assert L.moe_fused_forward(*args(x=None)) == ops.MOE_ERR_INVALID
    assert L.moe_fused_forward(*args(logits=None)) == ops.MOE_ERR_INVALID        # no routing input at all
    assert L.moe_fused_forward(*args(x=_fake((1 << 20) + 8))) == ops.MOE_ERR_INVALID   # misaligned
    assert L.moe_fused_forward(*args(ws=_fake((1 << 20) + 16))) == ops.MOE_ERR_INVALID  # ws not 256-aligned
    assert L.moe_fused_forward(*args(nbytes=need - 1)) == ops.MOE_ERR_WORKSPACE
    assert b"workspace" in L.moe_last_error_string()
    pf = ops.problem(16, 8, 2, 256, 128, fp8=True)
    assert L.moe_fused_forward(ctypes.byref(pf), good, good, None, None, good, good, None, None, good, good,
                               ops.workspace_size(pf), None) == ops.MOE_ERR_INVALID   # FP8 without scales
    bad_stage = L.moe_forward_stages(*args()[:-1], 4, 2, None)
    assert bad_stage == ops.MOE_ERR_INVALID


def test_route_align_quantize_argument_errors(L):
    g = _fake(1 << 20)
    assert L.moe_route(g, 4, 8, 9, 1, g, g, None) == ops.MOE_ERR_INVALID      # topk > E
    assert L.moe_route(g, 4, 8, 2, 3, g, g, None) == ops.MOE_ERR_INVALID      # renormalize not 0/1
    assert L.moe_route(None, 4, 8, 2, 1, g, g, None) == ops.MOE_ERR_INVALID
    ws = int(L.moe_align_workspace_size(4, 2, 8))
    assert ws > 0
    assert L.moe_align(g, 4, 2, 8, 16, g, g, g, None, None, g, ws - 1, None) == ops.MOE_ERR_WORKSPACE
    assert L.moe_align(g, 4, 2, 8, 0, g, g, g, None, None, g, ws, None) == ops.MOE_ERR_INVALID
    assert L.moe_quantize_weights_fp8(g, 1, 100, 128, g, g, None) == ops.MOE_ERR_INVALID
    assert L.moe_quantize_weights_fp8(g, 1, 128, 128, None, g, None) == ops.MOE_ERR_INVALID


def test_product_path_has_no_fallback(tmp_path, monkeypatch):
    """With the library missing, the binding raises instead of computing anything."""
    monkeypatch.setattr(ops, "_LIB_PATH", str(tmp_path / "missing.so"))
    monkeypatch.setattr(ops, "_lib", None)
    with pytest.raises(RuntimeError):
        ops.lib()


def test_selftest_argument_errors(L):
    g = _fake(1 << 20)
    assert L.moe_selftest_wait_timeout(0, g, g, None) == ops.MOE_ERR_INVALID
    assert L.moe_selftest_wait_timeout(2_000_000, g, g, None) == ops.MOE_ERR_INVALID
    assert L.moe_selftest_wait_timeout(100, None, g, None) == ops.MOE_ERR_INVALID


def test_sf_atom_reindex_matches_header_formula():
    """ops.sf_atoms_to_rows is the inverse of the SF-atom layout the header documents."""
    import torch
    rows, cols, batches = 256, 384, 2
    atoms = torch.empty(batches * rows * cols // 32, dtype=torch.long)
    for b in range(batches):
        for n in range(rows):
            for k in range(0, cols, 32):
                nn = b * rows + n
                off = ((nn // 128) * (cols // 128) + k // 128) * 512 + (nn % 32) * 16 + ((nn % 128) // 32) * 4 \
                    + (k % 128) // 32
                atoms[off] = (b * rows + n) * (cols // 32) + k // 32
    back = ops.sf_atoms_to_rows(atoms.reshape(batches, -1), rows, cols)
    assert torch.equal(back.reshape(-1), torch.arange(batches * rows * cols // 32))


def test_expert_parallel_problem_validation(L):
    """Expert ranges: E local experts [first_expert, first_expert + E) of num_global_experts."""
    size = lambda **kw: L.moe_workspace_size(ctypes.byref(ops.problem(64, kw.pop("E", 16), kw.pop("topk", 8), 4096,
                                                                        1536, **kw)))
    assert size(num_global_experts=128, first_expert=112) > 0
    assert size(num_global_experts=128, first_expert=0) > 0
    assert size(E=2, topk=8, num_global_experts=16, first_expert=14) > 0   # topk may exceed the local count
    assert size(num_global_experts=128, first_expert=113) == 0                # range past the last expert
    assert size(num_global_experts=128, first_expert=-1) == 0
    assert size(num_global_experts=8) == 0                                    # fewer global than local
    assert size(num_global_experts=2048) == 0
    assert size(first_expert=1) == 0                                          # no range without num_global_experts
    assert size(E=2, topk=8) == 0                                             # topk <= num_global_experts
    p = ops.problem(64, 16, 8, 4096, 1536)
    p.reserved[0] = 1
    assert L.moe_workspace_size(ctypes.byref(p)) == 0


def test_expert_parallel_plan(L):
    """A rank's tiles are chosen from the tokens its experts expect (T*topk*E/num_global_experts), and
    its workspace keeps the inverse permutation, which masks the combine."""
    full = ops.resolve_problem(ops.problem(4096, 128, 8, 4096, 1536))
    shard = ops.resolve_problem(ops.problem(4096, 16, 8, 4096, 1536, num_global_experts=128, first_expert=32))
    assert full.mode == ops.MODE_NORMAL and shard.mode == ops.MODE_NORMAL
    small = ops.resolve_problem(ops.problem(64, 16, 8, 4096, 1536, num_global_experts=128, first_expert=32))
    assert small.mode == ops.MODE_SWAP_AB and small.block_m == 16               # 64*8/128 = 4 tokens per expert
    assert small.num_global_experts == 128 and small.first_expert == 32
    for fp8 in (False, True):
        lay = ops.workspace_layout(ops.problem(64, 16, 8, 4096, 1536, fp8=fp8, num_global_experts=128,
                                               first_expert=16))
        assert lay.pos_of_flat >= 0
        # capacity bounds the local rows: every assignment may land here
        assert lay.capacity == ops.align_capacity(64, 8, 16, lay.block_m)


def test_combine_allreduce_chunking_and_argument_errors(L):
    """Flag counts follow the chunking rule (at most 64 chunks per rank, at most 1024, whole tokens);
    every argument error is caught before a launch."""
    assert ops.combine_allreduce_flag_count(64, 8) == 2 * 64 + 1        # one token per chunk
    assert ops.combine_allreduce_flag_count(16384, 4) == 2 * 256 + 1    # 64 tokens per chunk
    assert ops.combine_allreduce_flag_count(100000, 16) == 2 * 1021 + 1  # 98 tokens, ceil(100000 / 98) chunks
    assert ops.combine_allreduce_flag_count(0, 2) == 1
    assert ops.combine_allreduce_flag_count(8, 0) == 0 and ops.combine_allreduce_flag_count(8, 17) == 0
    g = 1 << 20
    good = [dict(y=g, pos_of_flat=g, partial=g, out=g, flags=g, status=g) for _ in range(2)]

    def rc(T=8, topk=2, H=256, rank=0, ranks=good, epoch=1, timeout=1000, emulated=False):
        arr = ops._ranks_array(ranks) if ranks is not None else None
        if emulated:
            return L.moe_combine_allreduce_emulated(T, topk, H, len(ranks or []), arr, epoch, timeout, None)
        return L.moe_combine_allreduce(T, topk, H, len(ranks or []), rank, arr, epoch, timeout, None)

    inv = ops.MOE_ERR_INVALID
    assert rc(rank=2) == inv and rc(rank=-1) == inv
    assert rc(H=100) == inv and rc(topk=0) == inv and rc(T=-1) == inv
    assert rc(epoch=0) == inv and rc(timeout=0) == inv and rc(timeout=20_000_000) == inv
    assert rc(ranks=[dict(good[0])] * 17) == inv
    assert rc(ranks=[good[0], dict(good[1], partial=None)]) == inv
    assert rc(ranks=[good[0], dict(good[1], out=g + 8)]) == inv                # out must be 16-byte aligned
    assert rc(ranks=[dict(good[0], y=None), good[1]]) == inv                   # own y is read
    assert rc(ranks=[good[0], dict(good[1], y=None, pos_of_flat=None, status=None)]) != inv  # a peer's are not
    assert rc(ranks=[good[0], dict(good[1], y=None)], emulated=True) == inv     # emulated: every rank's are read
    assert rc(T=0) == ops.MOE_OK                                                # nothing to do
