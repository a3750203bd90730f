"""Every benchmark configuration at full size against the oracle, in the launch
configuration bench.py times (automatic tile mode and block size).

For each point:
* routing (when the layer routes from logits) and the whole alignment --
  sorted_token_ids, expert_ids, num_tokens_post_padded, counts, offsets --
  bit-exact for every token;
* the output rows of 512 uniformly drawn tokens (every token when T <= 512)
  and of every token that carries a duplicate expert id;
* every row of the hottest and of the coldest non-empty expert, compared as
  the GEMM2 output y (each assignment's routed-weighted expert output, before
  the combine), which covers all m-blocks and tile waves of the hottest
  expert and the tail block of each.
Tolerances: normwise relative error <= 5e-3 (bf16 weights) / 2e-2 (FP8), and
max |diff| <= 0.05 max |ref|, on each row set.  The model is the PR analysis'
full-size, every-row test of the sorted-A down projection
("test_sorted_a_tma_moe_matches_route_major")."""

import gc

import numpy as np
import pytest
import torch

from moe_layer_top_b200 import inputs, ops
from oracle import moe_oracle as O
from tests.gpu_helpers import Case, assert_close

pytestmark = pytest.mark.gpu

POINTS = [("decode_bf16", 64), ("fp8_uniform", 256), ("fp8_uniform", 1024), ("fp8_uniform", 4096),
          ("prefill_fp8", 16384), ("skewed_fp8", 1), ("skewed_fp8", 32), ("skewed_fp8", 512), ("skewed_fp8", 8192),
          ("prefill_mxfp8", 16384), ("decode_mxfp8", 1), ("decode_mxfp8", 64)]

_weights = {}


@pytest.fixture(autouse=True, scope="module")
def _built():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from moe_layer_top_b200 import build
    build.build()
    yield
    _weights.clear()


def _layer_weights(cfg):
    """bf16 weights of a workload, kept while consecutive points use the same layer."""
    if cfg.name not in _weights:
        _weights.clear()
        gc.collect()
        torch.cuda.empty_cache()
        _weights[cfg.name] = inputs.make_weights(cfg, 0, device="cuda")
    return _weights[cfg.name]


def _sampled_tokens(ids: np.ndarray, n_uniform: int, seed: int) -> np.ndarray:
    T = ids.shape[0]
    if T <= n_uniform:
        return np.arange(T)
    rng = np.random.default_rng(seed)
    uni = rng.choice(T, size=n_uniform, replace=False)
    srt = np.sort(ids, axis=1)
    dup = np.nonzero((srt[:, 1:] == srt[:, :-1]).any(axis=1))[0]
    return np.unique(np.concatenate([uni, dup]))


@pytest.mark.parametrize("name,T", POINTS, ids=[f"{n}-T{t}" for n, t in POINTS])
def test_full_size_point(name, T):
    cfg = inputs.CONFIGS[name]
    c = Case(cfg, T, seed=0, weights=_layer_weights(cfg))
    out = c.run()
    assert c.status() == ops.MOE_STATUS_OK
    v = c.views()
    k = cfg.topk

    # routing and alignment of every token, bit for bit
    if "logits" in c.routing:
        ref_ids, ref_w = O.route(c.routing["logits"].cpu().numpy(), k)
        np.testing.assert_array_equal(v["topk_ids"].cpu().numpy(), ref_ids)
        np.testing.assert_allclose(v["topk_weights"].cpu().numpy(), ref_w, rtol=1e-5, atol=1e-7)
        ids, wts = ref_ids, ref_w
    else:
        ids = c.routing["topk_ids"].cpu().numpy()
        wts = c.routing["topk_weights"].cpu().numpy()
    a = O.align(ids, cfg.E, c.q.block_m)
    for key in ("sorted_token_ids", "expert_ids", "expert_counts", "expert_offsets"):
        np.testing.assert_array_equal(v[key].cpu().numpy(), a[key], err_msg=key)
    assert int(v["num_tokens_post_padded"].item()) == a["num_tokens_post_padded"]

    # output rows: 512 uniform tokens (all when T <= 512) and every token with a duplicate id
    tok = _sampled_tokens(ids, 512, T)
    ref = c.oracle(tokens=tok)
    assert_close(out[torch.from_numpy(tok).cuda()].float().cpu().numpy(), ref["out"], fp8=cfg.fp8)

    # every row of the hottest and of the coldest non-empty expert, as GEMM2 output y
    counts = a["expert_counts"]
    hit = np.nonzero(counts > 0)[0]
    hot = int(hit[np.argmax(counts[hit])])
    cold = int(hit[np.argmin(counts[hit])])
    y = v["y"]
    flat_w = wts.reshape(-1).astype(np.float64)
    for e in sorted({hot, cold}):
        flat = np.nonzero(ids.reshape(-1) == e)[0]
        got = y[torch.from_numpy(flat).cuda()].float().cpu().numpy()
        want = c.oracle_assignments(flat) * flat_w[flat][:, None]
        assert_close(got, want, fp8=cfg.fp8)
