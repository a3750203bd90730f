"""The persistent decode kernel (route + align + GEMM1 + GEMM2 + combine in
one cooperative launch for small bf16 batches) against the oracle and against
the kernel-per-stage pipeline."""

import numpy as np
import pytest
import torch

from moe_layer_top_b200 import inputs, ops
from oracle import moe_oracle as O
from tests.gpu_helpers import Case, assert_close

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True, scope="module")
def _built():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from moe_layer_top_b200 import build
    build.build()


def _eligible(c):
    q = c.q
    return q.mode == ops.MODE_SWAP_AB and q.block_m == 16 and q.T * q.topk <= 256 and q.E <= 256


@pytest.mark.parametrize("name,E,topk,H,I,T,routing", [
    ("tiny", 8, 2, 256, 128, 16, "logits"),
    ("mid", 16, 4, 1024, 512, 3, "logits"),
    ("mid_ids", 16, 4, 1024, 512, 20, "uniform_ids"),     # duplicates inside rows
    ("wide", 256, 8, 512, 256, 32, "logits"),            # E = 256: eight logits per lane
    ("top1", 64, 1, 512, 256, 200, "logits"),
])
def test_persistent_decode_matches_oracle_and_alignment(name, E, topk, H, I, T, routing):
    cfg = inputs.make_custom_config(name, E=E, topk=topk, H=H, I=I, fp8=False, routing=routing)
    c = Case(cfg, T, seed=21, persistent_decode=True)
    assert _eligible(c)
    out = c.run()
    assert c.status() == ops.MOE_STATUS_OK
    ref = c.oracle()
    assert_close(out.float().cpu().numpy(), ref["out"], fp8=False)
    v = c.views()
    if routing == "logits":   # the router's output lands in the workspace
        np.testing.assert_array_equal(v["topk_ids"].cpu().numpy(), ref["topk_ids"])
    al = O.align(ref["topk_ids"], E, 16)
    assert int(v["num_tokens_post_padded"].item()) == al["num_tokens_post_padded"]
    np.testing.assert_array_equal(v["sorted_token_ids"].cpu().numpy(), al["sorted_token_ids"])
    np.testing.assert_array_equal(v["expert_ids"].cpu().numpy(), al["expert_ids"])
    np.testing.assert_array_equal(v["expert_counts"].cpu().numpy(), al["expert_counts"])
    np.testing.assert_array_equal(v["expert_offsets"].cpu().numpy(), al["expert_offsets"])


@pytest.mark.parametrize("T", [1, 4, 16])
def test_persistent_decode_equals_staged_pipeline(T):
    """Same MMAs in the same K order as the per-stage kernels: bitwise equal."""
    cfg = inputs.CONFIGS["decode_bf16"]
    w = inputs.make_weights(cfg, 0, device="cuda")
    a = Case(cfg, T, seed=0, weights=w, persistent_decode=True).run().clone()
    b = Case(cfg, T, seed=0, weights=w).run().clone()
    assert torch.equal(a, b)


def test_persistent_decode_full_size_against_oracle():
    cfg = inputs.CONFIGS["decode_bf16"]
    c = Case(cfg, 16, seed=3, persistent_decode=True)
    out = c.run()
    assert c.status() == ops.MOE_STATUS_OK
    assert_close(out.float().cpu().numpy(), c.oracle()["out"], fp8=False)


def test_persistent_decode_clamp_and_determinism():
    cfg = inputs.make_custom_config("mid", E=16, topk=4, H=1024, I=512, fp8=False, routing="logits")
    c = Case(cfg, 9, seed=5, swiglu_limit=0.05, persistent_decode=True)
    a = c.run().clone()
    assert torch.equal(a, c.run())
    assert_close(a.float().cpu().numpy(), c.oracle()["out"], fp8=False)


def test_persistent_decode_reports_bad_expert_id():
    cfg = inputs.make_custom_config("bad", E=8, topk=2, H=256, I=128, fp8=False, routing="uniform_ids")
    c = Case(cfg, 5, seed=1, persistent_decode=True)
    c.routing["topk_ids"][2, 1] = 99
    c.run()
    assert c.status() == ops.MOE_STATUS_BAD_EXPERT_ID
