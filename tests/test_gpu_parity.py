"""CUDA path vs the CPU oracle, through the C ABI.

Bit-exact: routing ids, the alignment (permutation, padding, block experts,
counts, offsets), FP8 weight codes/scales and the FP8 GEMM1 input.  Within
tolerance (normwise 5e-3 bf16 / 2e-2 FP8, max |diff| <= 0.05 max |ref|): the
layer output, on every tile orientation, at small sizes in full and at the
benchmark sizes on sampled tokens."""

import numpy as np
import pytest
import torch

from moe_layer_top_b200 import inputs, ops
from oracle import moe_oracle as O
from tests.gpu_helpers import Case, assert_close, errors

pytestmark = pytest.mark.gpu

MID_BF16 = inputs.make_custom_config("mid_bf16", E=16, topk=4, H=1024, I=512, fp8=False, routing="logits")
MID_FP8 = inputs.make_custom_config("mid_fp8", E=16, topk=4, H=1024, I=512, fp8=True, routing="uniform_ids")
MODES = [(ops.MODE_NORMAL, 128), (ops.MODE_SWAP_AB, 16), (ops.MODE_SWAP_AB, 32), (ops.MODE_SWAP_AB, 64)]


@pytest.fixture(autouse=True, scope="module")
def _built():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from moe_layer_top_b200 import build
    build.build()


# ----------------------------------------------------------------------------- routing
@pytest.mark.parametrize("T,E,k,bias", [(16, 8, 2, 0.0), (64, 128, 8, 0.0), (16384, 128, 8, 0.5), (3, 256, 8, 0.0),
                                        (50, 1000, 32, 0.0)])
def test_route_matches_oracle(T, E, k, bias):
    g = torch.Generator(device="cuda").manual_seed(T * 7 + E)
    logits = torch.randn((T, E), generator=g, device="cuda") + bias * torch.randn((E,), generator=g, device="cuda")
    ids, w = ops.route(logits, k)
    torch.cuda.synchronize()
    ref_ids, ref_w = O.route(logits.cpu().numpy(), k)
    np.testing.assert_array_equal(ids.cpu().numpy(), ref_ids)
    np.testing.assert_allclose(w.cpu().numpy(), ref_w, rtol=1e-5, atol=1e-7)


def test_route_ties_take_lower_index():
    logits = torch.zeros((4, 64), device="cuda")
    logits[1, 10:20] = 1.0
    logits[2] = torch.round(torch.randn(64, device="cuda") * 2) / 2   # many exact ties
    ids, w = ops.route(logits, 8)
    ref_ids, ref_w = O.route(logits.cpu().numpy(), 8)
    np.testing.assert_array_equal(ids.cpu().numpy(), ref_ids)
    np.testing.assert_allclose(w.cpu().numpy(), ref_w, rtol=1e-5)


def test_route_without_renormalisation():
    logits = torch.randn((33, 128), device="cuda")
    ids, w = ops.route(logits, 8, renormalize=False)
    ref_ids, ref_w = O.route(logits.cpu().numpy(), 8, renormalize=False)
    np.testing.assert_array_equal(ids.cpu().numpy(), ref_ids)
    np.testing.assert_allclose(w.cpu().numpy(), ref_w, rtol=1e-5, atol=1e-8)


# ----------------------------------------------------------------------------- alignment
def _ids(T, E, k, dist, seed):
    rng = np.random.default_rng(seed)
    if dist == "uniform":
        return np.stack([rng.permutation(E)[:k] for _ in range(T)]).astype(np.int32)
    if dist == "dup":
        return rng.integers(0, E, (T, k)).astype(np.int32)
    if dist == "one":
        return np.full((T, k), 3 % E, dtype=np.int32)
    return np.minimum(rng.zipf(1.3, (T, k)) - 1, E - 1).astype(np.int32)


@pytest.mark.parametrize("T,E,k,bm,dist", [
    (1, 128, 8, 16, "uniform"), (4, 128, 8, 16, "uniform"), (64, 128, 8, 16, "uniform"),
    (256, 128, 8, 32, "dup"), (1024, 128, 8, 64, "dup"), (16384, 128, 8, 128, "uniform"),
    (8192, 256, 8, 128, "skew"), (33, 256, 8, 16, "skew"), (100, 16, 4, 128, "one"), (7, 1, 1, 16, "uniform"),
    (1000, 1024, 32, 32, "dup"), (3, 8, 8, 64, "uniform"),
])
def test_align_matches_oracle_bit_exact(T, E, k, bm, dist):
    ids = _ids(T, E, k, dist, T + E + bm)
    res = ops.align(torch.from_numpy(ids).cuda(), E, bm)
    torch.cuda.synchronize()
    ref = O.align(ids, E, bm)
    assert res["capacity"] == ref["capacity"]
    np.testing.assert_array_equal(res["sorted_token_ids"].cpu().numpy(), ref["sorted_token_ids"])
    np.testing.assert_array_equal(res["expert_ids"].cpu().numpy(), ref["expert_ids"])
    assert int(res["num_tokens_post_padded"].item()) == ref["num_tokens_post_padded"]
    np.testing.assert_array_equal(res["expert_counts"].cpu().numpy(), ref["expert_counts"])
    np.testing.assert_array_equal(res["expert_offsets"].cpu().numpy(), ref["expert_offsets"])


@pytest.mark.parametrize("name,T,mode,bm", [
    ("tiny", 16, ops.MODE_AUTO, 0), ("decode_bf16", 1, ops.MODE_AUTO, 0), ("decode_bf16", 64, ops.MODE_AUTO, 0),
    ("fp8_uniform", 256, ops.MODE_AUTO, 0), ("fp8_uniform", 1024, ops.MODE_NORMAL, 0),
    ("skewed_fp8", 32, ops.MODE_SWAP_AB, 64), ("prefill_fp8", 16384, ops.MODE_AUTO, 0),
])
def test_forward_routing_and_alignment_bit_exact(name, T, mode, bm):
    """The route/align intermediates of a full forward (single-CTA path for
    small batches, multi-CTA path for large ones) equal the oracle's."""
    cfg = inputs.CONFIGS[name]
    dev = torch.device("cuda")
    x = inputs.make_tokens(cfg, T, 0, device=dev)
    r = inputs.make_routing(cfg, T, 0, device=dev)
    p = ops.problem(T, cfg.E, cfg.topk, cfg.H, cfg.I, fp8=cfg.fp8, mode=mode, block_m=bm)
    q = ops.resolve_problem(p)
    ws = ops.alloc_workspace(p)
    ops.forward_stages(p, x, x, x, ops.STAGE_ROUTE, ops.STAGE_ALIGN + 1, logits=r.get("logits"),
                       topk_ids=r.get("topk_ids"), topk_weights=r.get("topk_weights"),
                       w13_scale=x if cfg.fp8 else None, w2_scale=x if cfg.fp8 else None, out=x, ws=ws)
    torch.cuda.synchronize()
    v = ops.workspace_views(p, ws)
    if "logits" in r:
        ids, w = O.route(r["logits"].cpu().numpy(), cfg.topk)
        np.testing.assert_array_equal(v["topk_ids"].cpu().numpy(), ids)
        np.testing.assert_allclose(v["topk_weights"].cpu().numpy(), w, rtol=1e-5, atol=1e-7)
    else:
        ids = r["topk_ids"].cpu().numpy()
    ref = O.align(ids, cfg.E, q.block_m)
    np.testing.assert_array_equal(v["sorted_token_ids"].cpu().numpy(), ref["sorted_token_ids"])
    np.testing.assert_array_equal(v["expert_ids"].cpu().numpy(), ref["expert_ids"])
    assert int(v["num_tokens_post_padded"].item()) == ref["num_tokens_post_padded"]
    np.testing.assert_array_equal(v["expert_counts"].cpu().numpy(), ref["expert_counts"])
    np.testing.assert_array_equal(v["expert_offsets"].cpu().numpy(), ref["expert_offsets"])
    assert ops.read_status(p, ws) == ops.MOE_STATUS_OK


def test_align_reports_bad_expert_id():
    ids = torch.tensor([[0, 1], [2, 9]], dtype=torch.int32, device="cuda")   # 9 >= E
    res = ops.align(ids, 8, 16)
    torch.cuda.synchronize()
    status = int(res["workspace"][:4].view(torch.int32).item())
    assert status == ops.MOE_STATUS_BAD_EXPERT_ID
    # the three good assignments are still placed, in order
    s = res["sorted_token_ids"].cpu().numpy()
    assert sorted(s[s != 4].tolist()) == [0, 1, 2]


# ----------------------------------------------------------------------------- FP8 preparation
def test_weight_quantisation_bit_exact():
    cfg = inputs.CONFIGS["decode_bf16"]
    w13, w2 = inputs.make_expert_weights(cfg, 5, 0, device="cuda")
    for w in (w13, w2):
        codes, scales = ops.quantize_weights_fp8(w[None])
        torch.cuda.synchronize()
        rc, rs = O.quantize_weight_block128(w.float().cpu().double().numpy())
        np.testing.assert_array_equal(codes[0].cpu().numpy(), rc)
        np.testing.assert_array_equal(scales[0].cpu().numpy(), rs)


def test_weight_quantisation_zero_block_and_extremes():
    w = torch.zeros((1, 256, 256), dtype=torch.bfloat16, device="cuda")
    w[0, 0, 0] = 3.0
    w[0, 200, 130] = -1e-30
    w[0, 130:140, 0:128] = torch.randn((10, 128), device="cuda").to(torch.bfloat16) * 1e4
    codes, scales = ops.quantize_weights_fp8(w)
    rc, rs = O.quantize_weight_block128(w[0].float().cpu().double().numpy())
    np.testing.assert_array_equal(codes[0].cpu().numpy(), rc)
    np.testing.assert_array_equal(scales[0].cpu().numpy(), rs)


@pytest.mark.parametrize("mode,bm", [(ops.MODE_NORMAL, 128), (ops.MODE_SWAP_AB, 32)])
def test_gather_quantises_x_bit_exact(mode, bm):
    """Swap-AB: x is quantised once per token ([T, H] codes) and each scale lands
    on the sorted rows of the token's assignments.  Normal tiles: a sorted copy."""
    c = Case(MID_FP8, 37, seed=3, mode=mode, block_m=bm)
    c.run()
    v = c.views()
    ntpp = int(v["num_tokens_post_padded"].item())
    sorted_ids = v["sorted_token_ids"][:ntpp].cpu().numpy()
    nflat = 37 * MID_FP8.topk
    rows = np.nonzero(sorted_ids < nflat)[0]
    tok = sorted_ids[rows] // MID_FP8.topk
    x = c.x.float().cpu().double().numpy()
    rc, rs = O.quantize_act_group128(x)
    if mode == ops.MODE_NORMAL:
        np.testing.assert_array_equal(v["a1"][:ntpp].cpu().numpy()[rows], rc[tok])
    else:
        np.testing.assert_array_equal(v["a1"].cpu().numpy(), rc)
        pos = v["pos_of_flat"].cpu().numpy()
        np.testing.assert_array_equal(np.sort(pos), np.sort(rows))           # inverse of sorted_token_ids
        np.testing.assert_array_equal(sorted_ids[pos], np.arange(nflat))
    np.testing.assert_array_equal(v["a1_scale_t"][:, :ntpp].cpu().numpy().T[rows], rs[tok])


@pytest.mark.parametrize("mode,bm", [(ops.MODE_NORMAL, 128), (ops.MODE_SWAP_AB, 32)])
def test_fp8_gemm1_intermediate_matches_oracle(mode, bm):
    """The block-FP8 GEMM1 output a2 (E4M3 codes + per-(row,128) power-of-two scales) of every
    real row against the oracle's requantisation of its own bf16 intermediate, for both GEMM1
    epilogues.  The fast exponential of the SiLU and the fp32 accumulation order may move a bf16
    value by one ulp, so codes are compared by value within one E4M3 step, and nearly all codes
    and scales must be equal."""
    c = Case(MID_FP8, 45, seed=8, mode=mode, block_m=bm, split_k=False)
    c.run()
    v = c.views()
    k = MID_FP8.topk
    ntpp = int(v["num_tokens_post_padded"].item())
    sorted_ids = v["sorted_token_ids"][:ntpp].cpu().numpy()
    expert_of_row = np.repeat(v["expert_ids"].cpu().numpy()[:ntpp // bm], bm)
    rows = np.nonzero(sorted_ids < 45 * k)[0]
    x = c.x.float().cpu().double().numpy()
    a2 = v["a2"][:ntpp].cpu().numpy()
    a2_s = v["a2_scale_t"][:, :ntpp].cpu().numpy().T
    got_vals, ref_vals, same_codes, same_scales = [], [], 0, 0
    for e in np.unique(expert_of_row[rows]):
        rr = rows[expert_of_row[rows] == e]
        xq, xs = O.quantize_act_group128(x[sorted_ids[rr] // k])
        w13c, w13s = O.quantize_weight_block128(c.w13_bf16[e].float().cpu().double().numpy())
        w2c, w2s = O.quantize_weight_block128(c.w2_bf16[e].float().cpu().double().numpy())
        _, inter = O.expert_mlp(O.dequantize_act_group128(xq, xs), O.dequantize_weight_block128(w13c, w13s),
                                O.dequantize_weight_block128(w2c, w2s), requant=True, return_intermediates=True)
        got_vals.append(O.dequantize_act_group128(a2[rr], a2_s[rr]))
        ref_vals.append(O.dequantize_act_group128(inter["a2_codes"], inter["a2_scales"]))
        same_codes += int((a2[rr] == inter["a2_codes"]).sum())
        same_scales += int((a2_s[rr] == inter["a2_scales"]).sum())
    got, ref = np.concatenate(got_vals), np.concatenate(ref_vals)
    assert same_codes >= 0.99 * got.size
    assert same_scales >= 0.99 * (got.size // 128)
    step = np.abs(ref) * 2.0 ** -3 + 1e-30
    assert np.all(np.abs(got - ref) <= np.maximum(step, 2.0 ** -9 * np.abs(ref).max()))


# ----------------------------------------------------------------------------- layer output
@pytest.mark.parametrize("mode,bm", [(ops.MODE_AUTO, 0)] + MODES)
def test_tiny_layer_all_modes(mode, bm):
    c = Case(inputs.CONFIGS["tiny"], 16, seed=0, mode=mode, block_m=bm)
    out = c.run()
    assert c.status() == ops.MOE_STATUS_OK
    ref = c.oracle()
    v = c.views()
    np.testing.assert_array_equal(v["topk_ids"].cpu().numpy(), ref["topk_ids"])
    assert_close(out.float().cpu().numpy(), ref["out"], fp8=False)


@pytest.mark.parametrize("cfg", [MID_BF16, MID_FP8], ids=["bf16", "fp8"])
@pytest.mark.parametrize("T", [1, 37, 700])
@pytest.mark.parametrize("mode,bm", MODES)
def test_mid_layer(cfg, T, mode, bm):
    c = Case(cfg, T, seed=T, mode=mode, block_m=bm)
    out = c.run()
    assert c.status() == ops.MOE_STATUS_OK
    ref = c.oracle()
    assert_close(out.float().cpu().numpy(), ref["out"], fp8=cfg.fp8)


@pytest.mark.parametrize("T", [1, 4, 16, 64])
def test_decode_bf16_full_size(T):
    c = Case(inputs.CONFIGS["decode_bf16"], T, seed=0)
    out = c.run()
    assert c.status() == ops.MOE_STATUS_OK
    ref = c.oracle()
    assert_close(out.float().cpu().numpy(), ref["out"], fp8=False)


def _sample(T, n, seed):
    rng = np.random.default_rng(seed)
    return np.unique(np.concatenate([[0, T - 1], rng.choice(T, size=min(n, T), replace=False)]))


# ----------------------------------------------------------------------------- properties
@pytest.mark.parametrize("cfg", [MID_BF16, MID_FP8], ids=["bf16", "fp8"])
def test_run_to_run_bitwise_deterministic(cfg):
    c = Case(cfg, 300, seed=1)
    a = c.run().clone()
    b = c.run().clone()
    assert torch.equal(a, b)


@pytest.mark.parametrize("cfg", [MID_BF16, MID_FP8], ids=["bf16", "fp8"])
def test_block_size_invariance(cfg):
    """Swap-AB with block_m 16/32/64 keeps every element's K order: bitwise equal.
    The normal orientation is within the stated tolerance of it."""
    outs = {}
    w = inputs.make_weights(cfg, 2, device="cuda")
    for mode, bm in MODES:
        c = Case(cfg, 45, seed=2, mode=mode, block_m=bm, weights=w, split_k=False)
        outs[(mode, bm)] = c.run().clone()
    base = outs[(ops.MODE_SWAP_AB, 16)]
    assert torch.equal(base, outs[(ops.MODE_SWAP_AB, 32)])
    assert torch.equal(base, outs[(ops.MODE_SWAP_AB, 64)])
    nr, mr = errors(outs[(ops.MODE_NORMAL, 128)].float().cpu().numpy(), base.float().cpu().numpy())
    assert nr <= (2e-2 if cfg.fp8 else 5e-3) and mr <= 0.05


@pytest.mark.parametrize("name,T", [("mid_bf16", 1), ("mid_bf16", 3), ("mid_fp8", 2), ("mid_fp8", 9),
                                    ("mid_bf16", 5)])
def test_split_k_matches_oracle_and_unsplit(name, T):
    """With at most half as many tiles as SMs the swap-AB GEMMs split K and a reduce kernel
    adds the splits; the result matches the oracle and the unsplit kernel
    within tolerance, and is itself run-to-run deterministic.  The partial-sum
    buffer is written only when a split happened."""
    cfg = {"mid_bf16": MID_BF16, "mid_fp8": MID_FP8}[name]
    w = inputs.make_weights(cfg, 0, device="cuda")
    a = Case(cfg, T, seed=0, weights=w)
    a.views()["partials"].fill_(float("nan"))
    out_split = a.run().clone()
    assert not torch.all(torch.isnan(a.views()["partials"]))   # the GEMMs did split
    assert torch.equal(out_split, a.run())
    b = Case(cfg, T, seed=0, weights=w, split_k=False)
    b.views()["partials"].fill_(float("nan"))
    out_plain = b.run().clone()
    assert torch.all(torch.isnan(b.views()["partials"]))
    ref = a.oracle()
    assert_close(out_split.float().cpu().numpy(), ref["out"], fp8=cfg.fp8)
    assert_close(out_plain.float().cpu().numpy(), ref["out"], fp8=cfg.fp8)
    nr, _ = errors(out_split.float().cpu().numpy(), out_plain.float().cpu().numpy())
    assert nr < (2e-2 if cfg.fp8 else 5e-3)
    assert a.status() == ops.MOE_STATUS_OK


def test_output_canaries_untouched():
    cfg = MID_BF16
    c = Case(cfg, 29, seed=4)
    guard = torch.full((3 * 29 * cfg.H,), 1234.0, dtype=torch.bfloat16, device="cuda")
    out = guard[29 * cfg.H:2 * 29 * cfg.H].view(29, cfg.H)
    c.out = out
    c.run()
    assert torch.all(guard[:29 * cfg.H] == 1234.0) and torch.all(guard[2 * 29 * cfg.H:] == 1234.0)
    assert not torch.any(out == 1234.0)


def test_zero_tokens_is_a_no_op():
    cfg = MID_BF16
    c = Case(cfg, 1, seed=0)
    p = ops.problem(0, cfg.E, cfg.topk, cfg.H, cfg.I)
    out = torch.empty((0, cfg.H), dtype=torch.bfloat16, device="cuda")
    ops.fused_forward(p, c.x[:0], c.w13, c.w2, logits=c.routing["logits"][:0], out=out,
                      ws=torch.empty(256, dtype=torch.uint8, device="cuda"))
    torch.cuda.synchronize()


def test_all_tokens_on_one_expert_and_topk_equals_E():
    cfg = inputs.make_custom_config("hot", E=8, topk=8, H=512, I=256, fp8=True, routing="uniform_ids")
    c = Case(cfg, 200, seed=5)
    c.routing["topk_ids"] = torch.arange(8, dtype=torch.int32, device="cuda").repeat(200, 1)
    c.run()
    ref = c.oracle()
    assert_close(c.out.float().cpu().numpy(), ref["out"], fp8=True)
    cfg1 = inputs.make_custom_config("one", E=4, topk=2, H=256, I=128, fp8=False, routing="uniform_ids")
    c1 = Case(cfg1, 300, seed=6)
    c1.routing["topk_ids"] = torch.full((300, 2), 1, dtype=torch.int32, device="cuda")   # duplicates in each row
    c1.run()
    assert_close(c1.out.float().cpu().numpy(), c1.oracle()["out"], fp8=False)


# ----------------------------------------------------------------------------- epilogue variants
TOP1_BF16 = inputs.make_custom_config("top1_bf16", E=16, topk=1, H=1024, I=512, fp8=False, routing="logits")
TOP1_FP8 = inputs.make_custom_config("top1_fp8", E=16, topk=1, H=1024, I=512, fp8=True, routing="logits")
TOP1_MX = inputs.make_custom_config("top1_mx", E=16, topk=1, H=1024, I=512, fp8=True, mx=True, routing="logits")


@pytest.mark.parametrize("cfg,T,mode,bm", [(TOP1_BF16, 5, ops.MODE_AUTO, 0), (TOP1_BF16, 300, ops.MODE_NORMAL, 128),
                                           (TOP1_FP8, 40, ops.MODE_SWAP_AB, 32), (TOP1_FP8, 300, ops.MODE_AUTO, 0),
                                           (TOP1_MX, 100, ops.MODE_AUTO, 0)],
                         ids=["bf16-swap", "bf16-normal", "fp8-swap", "fp8-normal", "mx"])
def test_router_weight_on_input(cfg, T, mode, bm):
    """Top-1 routing with the weight applied to x before GEMM1 (the gather
    scales each row); GEMM2 then stores the expert output unweighted."""
    c = Case(cfg, T, seed=3, mode=mode, block_m=bm, router_weight_on_input=True)
    out = c.run()
    assert c.status() == ops.MOE_STATUS_OK
    ref = c.oracle()
    assert_close(out.float().cpu().numpy(), ref["out"], fp8=cfg.fp8)
    if not cfg.fp8:   # GEMM1's token rows are bf16(fp32(x) * w) exactly
        v = c.views()
        scaled = (c.x.float() * v["topk_weights"][:, 0][:, None]).bfloat16()
        if c.q.mode == ops.MODE_SWAP_AB:            # one row per token
            assert torch.equal(v["a1"], scaled)
        else:                                       # sorted copy
            ntpp = int(v["num_tokens_post_padded"].item())
            ids = v["sorted_token_ids"][:ntpp]
            rows = torch.nonzero(ids < T).flatten()
            assert torch.equal(v["a1"][rows], scaled[ids[rows].long()])


@pytest.mark.parametrize("cfg,T,mode,bm", [(MID_BF16, 7, ops.MODE_SWAP_AB, 16), (MID_BF16, 300, ops.MODE_NORMAL, 128),
                                           (MID_FP8, 2, ops.MODE_AUTO, 0), (MID_FP8, 500, ops.MODE_NORMAL, 128)],
                         ids=["bf16-swap", "bf16-normal", "fp8-swap-split", "fp8-normal"])
def test_swiglu_clamp(cfg, T, mode, bm):
    """A SwiGLU clamp small enough to bite: gate <= L and |up| <= L before the activation."""
    c = Case(cfg, T, seed=6, mode=mode, block_m=bm, swiglu_limit=0.05)
    out = c.run()
    assert c.status() == ops.MOE_STATUS_OK
    ref = c.oracle()
    assert_close(out.float().cpu().numpy(), ref["out"], fp8=cfg.fp8)
    plain = Case(cfg, T, seed=6, mode=mode, block_m=bm, weights=(c.w13_bf16, c.w2_bf16)).run()
    assert not torch.equal(out, plain)                 # the limit changed the result


def test_swiglu_clamp_mx():
    mx_cfg = inputs.make_custom_config("mid_mx", E=16, topk=4, H=1024, I=512, fp8=True, mx=True, routing="uniform_ids")
    for cfg, bm in ((mx_cfg, 0),):
        c = Case(cfg, 700, seed=7, block_m=bm, swiglu_limit=0.05)
        out = c.run()
        assert c.status() == ops.MOE_STATUS_OK
        assert_close(out.float().cpu().numpy(), c.oracle()["out"], fp8=True)


PR_TEST_SHAPE = inputs.make_custom_config("pr_test_shape", E=256, topk=8, H=4096, I=256, fp8=True,
                                          routing="uniform_ids", tokens=(1024,))


def test_pr_analysis_test_shape():
    """The shape of the PR analysis' own parity test (m = 1024 tokens, E = 256, H = 4096, I = 256,
    top-8, FP8 weights with 128x128 blocks, uniform random ids, softmax weights; our generator, not
    its seed): oracle parity on sampled tokens, and the analysis' point that a change of layout must
    not change the numbers -- swap-AB tiles with 32 and 64 token rows per block are bitwise equal, the
    normal orientation is within the FP8 tolerance."""
    w = inputs.make_weights(PR_TEST_SHAPE, 123, device="cuda")
    a = Case(PR_TEST_SHAPE, 1024, seed=123, weights=w, mode=ops.MODE_SWAP_AB, block_m=32, split_k=False)
    out32 = a.run().clone()
    assert a.status() == ops.MOE_STATUS_OK
    out64 = Case(PR_TEST_SHAPE, 1024, seed=123, weights=w, mode=ops.MODE_SWAP_AB, block_m=64, split_k=False).run()
    assert torch.equal(out32, out64)
    tok = _sample(1024, 10, 123)
    ref = a.oracle(tokens=tok)
    assert_close(out32[torch.from_numpy(tok).cuda()].float().cpu().numpy(), ref["out"], fp8=True)
    normal = Case(PR_TEST_SHAPE, 1024, seed=123, weights=w, mode=ops.MODE_NORMAL, block_m=128).run()
    nr, mr = errors(normal.float().cpu().numpy(), out32.float().cpu().numpy())
    assert nr <= 2e-2 and mr <= 0.05
