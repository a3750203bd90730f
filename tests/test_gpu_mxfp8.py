"""MXFP8 path on the GPU against the oracle: the weight and activation
quantisers bit for bit (codes and E8M0 scale bytes, through the SF-atom
layout), the GEMM1 intermediate, and the layer output within the FP8
tolerance -- small shapes in full, the benchmark shapes on sampled tokens."""

import numpy as np
import pytest
import torch

from moe_layer_top_b200 import inputs, ops
from oracle import moe_oracle as O
from tests.gpu_helpers import Case, assert_close, errors

pytestmark = pytest.mark.gpu

TINY_MX = inputs.make_custom_config("tiny_mx", E=8, topk=2, H=256, I=128, fp8=True, mx=True, routing="logits")
MID_MX = inputs.make_custom_config("mid_mx", E=16, topk=4, H=1024, I=512, fp8=True, mx=True, routing="uniform_ids")


@pytest.fixture(autouse=True, scope="module")
def _built():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from moe_layer_top_b200 import build
    build.build()


def test_mx_weight_quantisation_bit_exact():
    cfg = inputs.CONFIGS["decode_bf16"]
    w13, w2 = inputs.make_expert_weights(cfg, 3, 0, device="cuda")
    for w in (w13, w2):
        codes, sf = ops.quantize_weights_mxfp8(w[None])
        torch.cuda.synchronize()
        rc, re8 = O.quantize_mx_group32(w.float().cpu().double().numpy())
        np.testing.assert_array_equal(codes[0].cpu().numpy(), rc)
        rows, cols = w.shape
        np.testing.assert_array_equal(ops.sf_atoms_to_rows(sf[0], rows, cols).cpu().numpy(), re8)


def test_mx_weight_quantisation_extremes():
    w = torch.zeros((2, 128, 256), dtype=torch.bfloat16, device="cuda")
    w[0, 0, 0] = 3.0                                   # one value in an otherwise zero group
    w[0, 5, 40] = -1e-30                               # tiny value: the 1e-10 floor decides the scale
    w[1, 100:110, 32:64] = torch.randn((10, 32), device="cuda").to(torch.bfloat16) * 1e4
    w[1, 127, 255] = 448.0 * 2.0 ** 20                 # an exact power-of-two multiple of 448
    codes, sf = ops.quantize_weights_mxfp8(w)
    rc, re8 = O.quantize_mx_group32(w.float().cpu().double().numpy())
    np.testing.assert_array_equal(codes.cpu().numpy(), rc)
    np.testing.assert_array_equal(ops.sf_atoms_to_rows(sf, 128, 256).cpu().numpy(), re8)


def test_mx_gather_quantises_x_bit_exact():
    c = Case(MID_MX, 37, seed=3)
    c.run()
    v = c.views()
    ntpp = int(v["num_tokens_post_padded"].item())
    cap = v["sorted_token_ids"].numel()
    sorted_ids = v["sorted_token_ids"][:ntpp].cpu().numpy()
    nflat = 37 * MID_MX.topk
    rows = np.nonzero(sorted_ids < nflat)[0]
    tok = sorted_ids[rows] // MID_MX.topk
    rc, re8 = O.quantize_mx_group32(c.x.float().cpu().double().numpy())
    np.testing.assert_array_equal(v["a1"][:ntpp].cpu().numpy()[rows], rc[tok])   # sorted copy of the codes
    sf_rows = ops.sf_atoms_to_rows(v["a1_sf"], cap, MID_MX.H).cpu().numpy()
    np.testing.assert_array_equal(sf_rows[rows], re8[tok])


def test_mx_gemm1_intermediate_matches_oracle():
    """a2 (E4M3 codes + E8M0 scales) of real rows against the oracle's own MX
    requantisation of its bf16 intermediate.  The SiLU's fast exponential may
    move a bf16 value by one ulp, so codes are compared by value with a
    bound of one E4M3 step, and nearly all must be equal."""
    c = Case(MID_MX, 29, seed=5)
    c.run()
    v = c.views()
    ntpp = int(v["num_tokens_post_padded"].item())
    cap = v["sorted_token_ids"].numel()
    sorted_ids = v["sorted_token_ids"][:ntpp].cpu().numpy()
    expert_of_row = np.repeat(v["expert_ids"].cpu().numpy()[:ntpp // 128], 128)
    nflat = 29 * MID_MX.topk
    rows = np.nonzero(sorted_ids < nflat)[0]
    x = c.x.float().cpu().double().numpy()
    a2 = v["a2"][:ntpp].cpu().numpy()
    a2_sf = ops.sf_atoms_to_rows(v["a2_sf"], cap, MID_MX.I).cpu().numpy()
    got_vals, ref_vals, same = [], [], 0
    for e in np.unique(expert_of_row[rows]):
        rr = rows[expert_of_row[rows] == e]
        xq, xs = O.quantize_mx_group32(x[sorted_ids[rr] // MID_MX.topk])
        w13c, w13s = O.quantize_mx_group32(c.w13_bf16[e].float().cpu().double().numpy())
        w2c, w2s = O.quantize_mx_group32(c.w2_bf16[e].float().cpu().double().numpy())
        _, inter = O.expert_mlp(O.dequantize_mx_group32(xq, xs), O.dequantize_mx_group32(w13c, w13s),
                                O.dequantize_mx_group32(w2c, w2s), requant="mx", return_intermediates=True)
        got_vals.append(O.dequantize_mx_group32(a2[rr], a2_sf[rr]))
        ref_vals.append(O.dequantize_mx_group32(inter["a2_codes"], inter["a2_scales"]))
        same += int((a2[rr] == inter["a2_codes"]).sum())
    got, ref = np.concatenate(got_vals), np.concatenate(ref_vals)
    assert same >= 0.99 * got.size
    step = np.abs(ref) * 2.0 ** -3 + 1e-30
    assert np.all(np.abs(got - ref) <= np.maximum(step, 2.0 ** -9 * np.abs(ref).max()))


@pytest.mark.parametrize("cfg,T", [(TINY_MX, 16), (MID_MX, 1), (MID_MX, 37), (MID_MX, 700)],
                         ids=["tiny16", "mid1", "mid37", "mid700"])
def test_mx_layer_matches_oracle(cfg, T):
    c = Case(cfg, T, seed=1)
    out = c.run()
    assert c.status() == ops.MOE_STATUS_OK
    assert c.q.mode == ops.MODE_NORMAL and c.q.block_m == 128
    ref = c.oracle()
    assert_close(out.float().cpu().numpy(), ref["out"], fp8=True)


def test_mx_layer_run_to_run_deterministic():
    c = Case(MID_MX, 300, seed=2)
    a = c.run().clone()
    assert torch.equal(a, c.run())


def test_mx_and_block_fp8_differ_as_the_oracle_says():
    """Same weights and tokens through the block-128 FP8 path and the MXFP8
    path.  Each is ~6 % (normwise) from the bf16 layer and they differ from
    each other by about as much; the GPU pair must differ as the oracle pair
    does (within 20 %), which checks that the GPU applies each scheme's own
    scales rather than a mix of the two."""
    fp8_cfg = inputs.make_custom_config("mid_fp8", E=16, topk=4, H=1024, I=512, fp8=True, routing="uniform_ids")
    w = inputs.make_weights(MID_MX, 4, device="cuda")
    ca = Case(MID_MX, 64, seed=4, weights=w)
    cb = Case(fp8_cfg, 64, seed=4, weights=w)
    a = ca.run().float().cpu().numpy()
    b = cb.run().float().cpu().numpy()
    gpu_nr, _ = errors(a, b)
    ora_nr, _ = errors(ca.oracle()["out"], cb.oracle()["out"])
    assert 0.8 * ora_nr < gpu_nr < 1.2 * ora_nr
