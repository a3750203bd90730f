"""Pins of the oracle's expert MLP and full layer.

* closed-form special cases with selection-matrix weights (catch a gate/up
  swap, a sign error in SiLU, a transposed operand, a missed rounding point),
  checked against torch's own silu and bf16/float8 casts;
* a brute-force dense evaluation written independently with torch ops
  (every expert on every token, masked by the top-k weights).
"""

import numpy as np
import pytest
import torch
import torch.nn.functional as F

from oracle import moe_oracle as O
from moe_layer_top_b200 import inputs


def _selection_weights(H, I, seed):
    """w13 = a permutation matrix (gate picks x[perm[:I]], up picks x[perm[I:2I]]),
    w2 scatters the I products to output columns perm2[:I]."""
    rng = np.random.default_rng(seed)
    perm = rng.permutation(H)
    w13 = np.zeros((2 * I, H))
    w13[np.arange(2 * I), perm[:2 * I]] = 1.0
    perm2 = rng.permutation(H)
    w2 = np.zeros((H, I))
    w2[perm2[:I], np.arange(I)] = 1.0
    return w13, w2, perm, perm2


def test_expert_mlp_closed_form_bf16():
    H, I = 256, 128
    w13, w2, perm, perm2 = _selection_weights(H, I, 0)
    rng = np.random.default_rng(1)
    x = O.round_bf16(rng.standard_normal((9, H)) * 3)
    x[0, perm[0]] = 0.0            # silu(0) = 0 whatever the up value
    x[1, perm[1]] = 30.0           # silu(30) ~= 30
    x[2, perm[2]] = -30.0          # silu(-30) ~= 0 (tiny negative)
    y = O.expert_mlp(x, w13, w2, requant=False)
    g = torch.from_numpy(x[:, perm[:I]])
    u = torch.from_numpy(x[:, perm[I:2 * I]])
    act = F.silu(g).to(torch.bfloat16).double()
    ref_p = (act * u).to(torch.bfloat16).double().numpy()
    ref = np.zeros_like(y)
    ref[:, perm2[:I]] = ref_p
    np.testing.assert_array_equal(y, ref)
    assert y[0, perm2[0]] == 0.0
    assert y[1, perm2[1]] == O.round_bf16(30.0 * x[1, perm[I + 1]])


def test_expert_mlp_closed_form_fp8_requant():
    H, I = 256, 128
    w13, w2, perm, perm2 = _selection_weights(H, I, 2)
    rng = np.random.default_rng(3)
    x = O.round_bf16(rng.standard_normal((5, H)))
    y = O.expert_mlp(x, w13, w2, requant=True)
    g = torch.from_numpy(x[:, perm[:I]])
    u = torch.from_numpy(x[:, perm[I:2 * I]])
    p = ((F.silu(g).to(torch.bfloat16).double() * u).to(torch.bfloat16)).float()
    raw = torch.clamp(p.abs().amax(-1, keepdim=True), min=1e-10) * torch.tensor(1 / 448.0)
    sc = torch.exp2(torch.ceil(torch.log2(raw.double())))
    q = (p.double() / sc).float().to(torch.float8_e4m3fn).double() * sc
    ref = np.zeros_like(y)
    ref[:, perm2[:I]] = q.numpy()
    np.testing.assert_array_equal(y, ref)


def test_expert_mlp_closed_form_mx_requant():
    H, I = 256, 128
    w13, w2, perm, perm2 = _selection_weights(H, I, 4)
    rng = np.random.default_rng(5)
    x = O.round_bf16(rng.standard_normal((5, H)) * np.exp(rng.uniform(-3, 3, (5, H))))
    y = O.expert_mlp(x, w13, w2, requant="mx")
    g = torch.from_numpy(x[:, perm[:I]])
    u = torch.from_numpy(x[:, perm[I:2 * I]])
    p = ((F.silu(g).to(torch.bfloat16).double() * u).to(torch.bfloat16)).float().reshape(5, I // 32, 32)
    raw = torch.clamp(p.abs().amax(-1, keepdim=True), min=1e-10) * torch.tensor(1 / 448.0)
    sc = torch.exp2(torch.ceil(torch.log2(raw.double())))
    q = ((p.double() / sc).float().to(torch.float8_e4m3fn).double() * sc).reshape(5, I)
    ref = np.zeros_like(y)
    ref[:, perm2[:I]] = q.numpy()
    np.testing.assert_array_equal(y, ref)


def test_expert_mlp_closed_form_swiglu_clamp():
    H, I = 256, 128
    w13, w2, perm, perm2 = _selection_weights(H, I, 6)
    rng = np.random.default_rng(7)
    x = O.round_bf16(rng.standard_normal((6, H)) * 4.0)
    lim = 2.5
    y = O.expert_mlp(x, w13, w2, requant=False, swiglu_limit=lim)
    g = torch.clamp(torch.from_numpy(x[:, perm[:I]]), max=lim)
    u = torch.clamp(torch.from_numpy(x[:, perm[I:2 * I]]), -lim, lim)
    p = (F.silu(g).to(torch.bfloat16).double() * u).to(torch.bfloat16).double()
    ref = np.zeros_like(y)
    ref[:, perm2[:I]] = p.numpy()
    np.testing.assert_array_equal(y, ref)
    assert np.abs(x[:, perm[:2 * I]]).max() > lim          # the clamp is exercised
    # no limit reproduces the unclamped rule
    np.testing.assert_array_equal(O.expert_mlp(x, w13, w2, requant=False),
                                  O.expert_mlp(x, w13, w2, requant=False, swiglu_limit=None))


def test_router_weight_on_input_top1():
    cfg = inputs.make_custom_config("tiny_top1", E=4, topk=1, H=256, I=128, routing="uniform_ids", tokens=(9,))
    w13, w2 = inputs.make_weights(cfg, 8)
    x = inputs.make_tokens(cfg, 9, 8).double().numpy()
    r = inputs.make_routing(cfg, 9, 8)
    ids = r["topk_ids"].numpy()
    wts = (np.random.default_rng(1).uniform(0.2, 1.7, (9, 1))).astype(np.float32)
    a, b = w13.double().numpy(), w2.double().numpy()
    res = O.moe_forward(x, a, b, 1, topk_ids=ids, topk_weights=wts, router_weight_on_input=True)
    # independent path: scale rows with torch's fp32 product and bf16 cast, run each expert, no output weight
    xs = (torch.from_numpy(x).float() * torch.from_numpy(wts)).to(torch.bfloat16).double()
    ref = np.zeros_like(x)
    for t in range(9):
        e = int(ids[t, 0])
        h = (xs[t] @ torch.from_numpy(a[e]).T).to(torch.bfloat16).double()
        p = (F.silu(h[:128]).to(torch.bfloat16).double() * h[128:]).to(torch.bfloat16).double()
        ref[t] = (p @ torch.from_numpy(b[e]).T).to(torch.bfloat16).double().numpy()
    np.testing.assert_array_equal(res["out"], ref)
    # unit weights: identical to weighting the output
    ones = np.ones((9, 1), np.float32)
    np.testing.assert_array_equal(
        O.moe_forward(x, a, b, 1, topk_ids=ids, topk_weights=ones, router_weight_on_input=True)["out"],
        O.moe_forward(x, a, b, 1, topk_ids=ids, topk_weights=ones)["out"])
    with pytest.raises(ValueError):
        O.moe_forward(x, a, b, 2, topk_ids=np.zeros((9, 2), np.int64), topk_weights=np.ones((9, 2), np.float32),
                      router_weight_on_input=True)


def _mx_torch(t, group=32):
    """Independent MX quantise-dequantise of the last dim with torch ops."""
    shp = t.shape
    g = t.reshape(*shp[:-1], shp[-1] // group, group).float()
    raw = torch.clamp(g.abs().amax(-1), min=1e-10) * torch.tensor(1 / 448.0)
    sc = torch.exp2(torch.ceil(torch.log2(raw.double())))
    q = torch.clamp(g.double() / sc[..., None], -448, 448).float().to(torch.float8_e4m3fn).double()
    return (q * sc[..., None]).reshape(shp)


def test_forward_matches_dense_bruteforce_mx_with_duplicate_ids():
    cfg = inputs.make_custom_config("tiny_mx", E=5, topk=3, H=256, I=128, fp8=True,
                                    routing="uniform_ids", tokens=(10,))
    w13, w2 = inputs.make_weights(cfg, 6)
    x = inputs.make_tokens(cfg, 10, 6)
    r = inputs.make_routing(cfg, 10, 6)
    ids = r["topk_ids"].numpy().copy()
    ids[1] = [4, 4, 0]
    wts = r["topk_weights"].numpy()
    q13, s13 = O.quantize_mx_group32(w13.double().numpy())
    q2, s2 = O.quantize_mx_group32(w2.double().numpy())
    assert s13.shape == (5, 256, 8) and s2.shape == (5, 256, 4)
    xn = x.double().numpy()
    res = O.moe_forward(xn, q13, q2, cfg.topk, topk_ids=ids, topk_weights=wts, w13_scale=s13, w2_scale=s2)
    # dense torch evaluation: weights MX-quantised by torch from the same draw
    xt = _mx_torch(torch.from_numpy(xn))
    W13 = _mx_torch(w13.double())
    W2 = _mx_torch(w2.double())
    h = torch.einsum("th,enh->etn", xt, W13).to(torch.bfloat16).double()
    I = 128
    p = (F.silu(h[..., :I]).to(torch.bfloat16).double() * h[..., I:]).to(torch.bfloat16).double()
    y = torch.einsum("eti,ehi->eth", _mx_torch(p), W2)
    mask = torch.zeros(10, 5, dtype=torch.float64)
    mask.scatter_add_(1, torch.from_numpy(ids).long(), torch.from_numpy(wts).double())
    ref = torch.einsum("te,eth->th", mask, y).to(torch.bfloat16).double().numpy()
    np.testing.assert_array_equal(res["out"], ref)
    assert np.abs(res["out"]).max() > 0


def _dense_reference(x, w13, w2, ids, wts, fp8, w13_scale=None, w2_scale=None):
    """Every expert on every token with torch ops, combined through a dense
    [T, E] weight mask; rounding points from torch's casts."""
    xt = torch.from_numpy(np.asarray(x, dtype=np.float64))
    T, H = xt.shape
    E = w13.shape[0]
    if fp8:
        g = xt.reshape(T, H // 128, 128).float()
        raw = torch.clamp(g.abs().amax(-1), min=1e-10) * torch.tensor(1 / 448.0)
        sc = torch.exp2(torch.ceil(torch.log2(raw.double())))
        xq = (g.double() / sc[..., None]).float().to(torch.float8_e4m3fn).double()
        xt = (xq * sc[..., None]).reshape(T, H)
        deq = lambda c, s: torch.from_numpy(c).view(torch.float8_e4m3fn).double() * \
            torch.from_numpy(s).double().repeat_interleave(128, -2).repeat_interleave(128, -1)
        W13 = deq(w13, w13_scale)
        W2 = deq(w2, w2_scale)
    else:
        W13 = torch.from_numpy(np.asarray(w13, dtype=np.float64))
        W2 = torch.from_numpy(np.asarray(w2, dtype=np.float64))
    I = W13.shape[1] // 2
    h = torch.einsum("th,enh->etn", xt, W13).to(torch.bfloat16).double()
    p = (F.silu(h[..., :I]).to(torch.bfloat16).double() * h[..., I:]).to(torch.bfloat16).double()
    if fp8:
        pg = p.reshape(E, T, I // 128, 128).float()
        raw = torch.clamp(pg.abs().amax(-1), min=1e-10) * torch.tensor(1 / 448.0)
        sc = torch.exp2(torch.ceil(torch.log2(raw.double())))
        p = ((pg.double() / sc[..., None]).float().to(torch.float8_e4m3fn).double()
             * sc[..., None]).reshape(E, T, I)
    y = torch.einsum("eti,ehi->eth", p, W2)
    mask = torch.zeros(T, E, dtype=torch.float64)
    ids_t = torch.from_numpy(np.asarray(ids)).long()
    mask.scatter_add_(1, ids_t, torch.from_numpy(np.asarray(wts)).double())
    out = torch.einsum("te,eth->th", mask, y)
    return out.to(torch.bfloat16).double().numpy()


@pytest.mark.parametrize("seed", [0, 1])
def test_forward_matches_dense_bruteforce_tiny_bf16(seed):
    cfg = inputs.CONFIGS["tiny"]
    w13, w2 = inputs.make_weights(cfg, seed)
    x = inputs.make_tokens(cfg, 16, seed)
    r = inputs.make_routing(cfg, 16, seed)
    w13n, w2n, xn = w13.double().numpy(), w2.double().numpy(), x.double().numpy()
    logits = r["logits"].numpy()
    res = O.moe_forward(xn, w13n, w2n, cfg.topk, logits=logits)
    ref = _dense_reference(xn, w13n, w2n, res["topk_ids"], res["topk_weights"], fp8=False)
    np.testing.assert_array_equal(res["out"], ref)
    assert np.abs(res["out"]).max() > 0


def test_forward_matches_dense_bruteforce_fp8_with_duplicate_ids():
    cfg = inputs.make_custom_config("tiny_fp8", E=6, topk=3, H=256, I=256, fp8=True,
                                    routing="uniform_ids", tokens=(12,))
    w13, w2 = inputs.make_weights(cfg, 4)
    x = inputs.make_tokens(cfg, 12, 4)
    r = inputs.make_routing(cfg, 12, 4)
    ids = r["topk_ids"].numpy().copy()
    ids[0] = [2, 2, 2]                       # a row that repeats one expert
    wts = r["topk_weights"].numpy()
    q13, s13 = O.quantize_weight_block128(w13.double().numpy())
    q2, s2 = O.quantize_weight_block128(w2.double().numpy())
    xn = x.double().numpy()
    res = O.moe_forward(xn, q13, q2, cfg.topk, topk_ids=ids, topk_weights=wts,
                        w13_scale=s13, w2_scale=s2)
    ref = _dense_reference(xn, q13, q2, ids, wts, fp8=True, w13_scale=s13, w2_scale=s2)
    np.testing.assert_array_equal(res["out"], ref)


def test_forward_token_subset_matches_full():
    cfg = inputs.CONFIGS["tiny"]
    w13, w2 = inputs.make_weights(cfg, 3)
    x = inputs.make_tokens(cfg, 16, 3).double().numpy()
    logits = inputs.make_routing(cfg, 16, 3)["logits"].numpy()
    full = O.moe_forward(x, w13.double().numpy(), w2.double().numpy(), 2, logits=logits)
    sub = O.moe_forward(x, w13.double().numpy(), w2.double().numpy(), 2, logits=logits,
                        tokens=[3, 0, 15])
    np.testing.assert_array_equal(sub["out"], full["out"][[3, 0, 15]])


def test_forward_zero_weights_give_zero_and_linearity_in_w2():
    cfg = inputs.CONFIGS["tiny"]
    w13, w2 = inputs.make_weights(cfg, 5)
    x = inputs.make_tokens(cfg, 16, 5).double().numpy()
    logits = inputs.make_routing(cfg, 16, 5)["logits"].numpy()
    w13n, w2n = w13.double().numpy(), w2.double().numpy()
    a = O.moe_forward(x, w13n, w2n, 2, logits=logits, return_y=True)
    b = O.moe_forward(x, w13n, 2.0 * w2n, 2, logits=logits, return_y=True)
    np.testing.assert_array_equal(b["y"], 2.0 * a["y"])         # y is linear in w2 (exact in fp64 x2)
    z = O.moe_forward(x, w13n, 0.0 * w2n, 2, logits=logits)
    assert np.all(z["out"] == 0.0)


def test_assignment_outputs_match_dense_per_expert_outputs():
    """One expert's outputs for chosen assignments (used to check every row of an expert on the
    GPU without evaluating the token's other experts) = the dense torch evaluation's unweighted
    output of that expert on that token; FP8 path with duplicate ids."""
    cfg = inputs.make_custom_config("tiny_fp8", E=6, topk=3, H=256, I=256, fp8=True,
                                    routing="uniform_ids", tokens=(12,))
    w13, w2 = inputs.make_weights(cfg, 9)
    xn = inputs.make_tokens(cfg, 12, 9).double().numpy()
    r = inputs.make_routing(cfg, 12, 9)
    ids = r["topk_ids"].numpy().copy()
    ids[3] = [1, 1, 4]
    wts = r["topk_weights"].numpy()
    q13, s13 = O.quantize_weight_block128(w13.double().numpy())
    q2, s2 = O.quantize_weight_block128(w2.double().numpy())
    flat = np.array([3 * 3 + 1, 0, 35, 3 * 3 + 0, 17])          # any order, duplicates' slots included
    got = O.assignment_outputs(xn, q13, q2, 3, flat, topk_ids=ids, topk_weights=wts, w13_scale=s13, w2_scale=s2)
    # dense torch: every expert on every token, unweighted
    g = torch.from_numpy(xn).reshape(12, 2, 128).float()
    raw = torch.clamp(g.abs().amax(-1), min=1e-10) * torch.tensor(1 / 448.0)
    sc = torch.exp2(torch.ceil(torch.log2(raw.double())))
    xt = ((g.double() / sc[..., None]).float().to(torch.float8_e4m3fn).double() * sc[..., None]).reshape(12, 256)
    deq = lambda c, s: torch.from_numpy(c).view(torch.float8_e4m3fn).double() * \
        torch.from_numpy(s).double().repeat_interleave(128, -2).repeat_interleave(128, -1)
    h = torch.einsum("th,enh->etn", xt, deq(q13, s13)).to(torch.bfloat16).double()
    p = (F.silu(h[..., :256]).to(torch.bfloat16).double() * h[..., 256:]).to(torch.bfloat16).double()
    pg = p.reshape(6, 12, 2, 128).float()
    raw = torch.clamp(pg.abs().amax(-1), min=1e-10) * torch.tensor(1 / 448.0)
    sc = torch.exp2(torch.ceil(torch.log2(raw.double())))
    p = ((pg.double() / sc[..., None]).float().to(torch.float8_e4m3fn).double() * sc[..., None]).reshape(6, 12, 256)
    y = torch.einsum("eti,ehi->eth", p, deq(q2, s2)).numpy()
    ref = np.stack([y[ids.reshape(-1)[f], f // 3] for f in flat])
    np.testing.assert_allclose(got, ref, rtol=1e-12, atol=1e-15)
    # and it is the same y the layer evaluation uses
    full = O.moe_forward(xn, q13, q2, 3, topk_ids=ids, topk_weights=wts, w13_scale=s13, w2_scale=s2, return_y=True)
    np.testing.assert_array_equal(got, full["y"].reshape(36, 256)[flat])


def test_parallel_rows_do_not_change_results_and_bf16_bit_patterns():
    """The oracle's OpenMP loops run independent rows: one thread and all threads give the same
    bits.  bf16 weights given as bit patterns (uint16) read as the same values as float64."""
    cfg = inputs.CONFIGS["tiny"]
    w13, w2 = inputs.make_weights(cfg, 11)
    x = inputs.make_tokens(cfg, 16, 11).double().numpy()
    logits = inputs.make_routing(cfg, 16, 11)["logits"].numpy()
    a = O.moe_forward(x, w13.double().numpy(), w2.double().numpy(), 2, logits=logits, threads=1)
    b = O.moe_forward(x, w13.double().numpy(), w2.double().numpy(), 2, logits=logits, threads=0)
    np.testing.assert_array_equal(a["out"], b["out"])
    bits13 = w13.view(torch.int16).numpy().view(np.uint16)
    bits2 = w2.view(torch.int16).numpy().view(np.uint16)
    c = O.moe_forward(x, bits13, bits2, 2, logits=logits)
    np.testing.assert_array_equal(a["out"], c["out"])
