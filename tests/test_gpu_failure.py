"""Failure detection on the GPU without a fault: a bounded wait that can
never complete gives up, reports the timeout in the status word, and the
context keeps working afterwards."""

import pytest
import torch

from moe_layer_top_b200 import inputs, ops
from tests.gpu_helpers import Case, assert_close

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True, scope="module")
def _built():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from moe_layer_top_b200 import build
    build.build()


def test_bounded_wait_times_out_and_reports():
    status, waited = ops.selftest_wait_timeout(2000)          # 2 ms limit
    assert status == ops.MOE_STATUS_WAIT_TIMEOUT | 0x7F
    assert 2_000_000 <= waited < 1_000_000_000                 # gave up after the limit, not much later


def test_context_usable_after_timeout():
    ops.selftest_wait_timeout(1000)
    c = Case(inputs.CONFIGS["tiny"], 16, seed=1)
    out = c.run()
    assert c.status() == ops.MOE_STATUS_OK
    assert_close(out.float().cpu().numpy(), c.oracle()["out"], fp8=False)
