"""Edge shapes of the layer on the GPU against the oracle: the smallest legal
H and I (one 128-deep K block), the largest expert count and top-k, batches
large enough for the multi-CTA alignment, and the un-renormalised router."""

import numpy as np
import pytest
import torch

from moe_layer_top_b200 import inputs, ops
from tests.gpu_helpers import Case, assert_close

pytestmark = pytest.mark.gpu

MODES = [(ops.MODE_NORMAL, 128), (ops.MODE_SWAP_AB, 16), (ops.MODE_SWAP_AB, 32), (ops.MODE_SWAP_AB, 64)]


@pytest.fixture(autouse=True, scope="module")
def _built():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from moe_layer_top_b200 import build
    build.build()


@pytest.mark.parametrize("quant", ["bf16", "fp8", "mx"])
@pytest.mark.parametrize("mode,bm", MODES)
def test_smallest_hidden_and_intermediate(quant, mode, bm):
    """The smallest legal shapes: I = 128 (one K block in GEMM2), H = 128 for
    swap-AB tiles, 256 for normal tiles (one 256-column GEMM2 tile)."""
    if quant == "mx" and mode == ops.MODE_SWAP_AB:
        pytest.skip("MXFP8 runs normal tiles only")
    H = 256 if mode == ops.MODE_NORMAL else 128
    cfg = inputs.make_custom_config(f"min_{quant}", E=4, topk=2, H=H, I=128, fp8=quant != "bf16",
                                    mx=quant == "mx", routing="logits")
    c = Case(cfg, 5, seed=11, mode=mode, block_m=bm)
    out = c.run()
    assert c.status() == ops.MOE_STATUS_OK
    assert_close(out.float().cpu().numpy(), c.oracle()["out"], fp8=cfg.fp8)


@pytest.mark.parametrize("fp8", [False, True], ids=["bf16", "fp8"])
def test_max_experts_and_topk(fp8):
    """E = 1024 experts (multi-CTA route and three-pass align) with top-32."""
    cfg = inputs.make_custom_config("wide", E=1024, topk=32, H=128, I=128, fp8=fp8, routing="logits")
    c = Case(cfg, 9, seed=12)
    out = c.run()
    assert c.status() == ops.MOE_STATUS_OK
    assert_close(out.float().cpu().numpy(), c.oracle()["out"], fp8=fp8)


def test_many_tokens_three_pass_align_sampled():
    """T * topk = 40 000 > 8192: route kernel + three-pass alignment + normal tiles; sampled tokens."""
    cfg = inputs.make_custom_config("tall", E=8, topk=2, H=256, I=128, fp8=True, routing="biased_logits")
    c = Case(cfg, 20000, seed=13)
    out = c.run()
    assert c.status() == ops.MOE_STATUS_OK
    tok = np.unique(np.concatenate([[0, 19999], np.random.default_rng(0).choice(20000, 40, replace=False)]))
    ref = c.oracle(tokens=tok)
    assert_close(out[torch.from_numpy(tok).cuda()].float().cpu().numpy(), ref["out"], fp8=True)


@pytest.mark.parametrize("T", [3, 300])
def test_router_without_renormalisation(T):
    cfg = inputs.make_custom_config("norenorm", E=16, topk=4, H=512, I=256, fp8=False, routing="logits")
    c = Case(cfg, T, seed=14, renormalize=False)
    out = c.run()
    ref = c.oracle()
    assert_close(out.float().cpu().numpy(), ref["out"], fp8=False)
    w = c.views()["topk_weights"].cpu().numpy()
    assert np.all(w.sum(1) < 1.0)          # un-renormalised softmax mass of the chosen experts
