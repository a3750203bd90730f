"""moe_align_noalloc: the alignment for callers that may not allocate device
memory (its scratch is a static device array inside the library).

Checked through the C ABI against moe_align (which takes a caller-provided
workspace) on four calls in a row, so that stale contents of the shared
array would show: a large call on the three-pass path (count, scan, scatter
over per-chunk histograms; more than 8192 assignments), a small one on the
single-CTA path, then two more three-pass calls, each smaller than the first
and with another expert count and block size.  Alignment results are
integers, so the comparison is exact, as for moe_align against the oracle.

This file is collected last on purpose: if it fails, every other test has
already run."""

import ctypes

import numpy as np
import pytest
import torch

from moe_layer_top_b200 import ops


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr())


def _noalloc(ids: torch.Tensor, E: int, bm: int):
    T, k = ids.shape
    cap = ops.align_capacity(T, k, E, bm)
    out = {
        "sorted_token_ids": torch.full((cap,), -7, dtype=torch.int32, device="cuda"),
        "expert_ids": torch.full((cap // bm,), -7, dtype=torch.int32, device="cuda"),
        "num_tokens_post_padded": torch.full((1,), -7, dtype=torch.int32, device="cuda"),
        "expert_counts": torch.full((E,), -7, dtype=torch.int32, device="cuda"),
        "expert_offsets": torch.full((E + 1,), -7, dtype=torch.int32, device="cuda"),
    }
    rc = ops.lib().moe_align_noalloc(_ptr(ids), T, k, E, bm, _ptr(out["sorted_token_ids"]),
                                     _ptr(out["expert_ids"]), _ptr(out["num_tokens_post_padded"]),
                                     _ptr(out["expert_counts"]), _ptr(out["expert_offsets"]),
                                     ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert rc == ops.MOE_OK, ops.lib().moe_last_error_string()
    return out


@pytest.mark.gpu
def test_noalloc_align_matches_workspace_align_on_consecutive_calls():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from moe_layer_top_b200 import build
    build.build()
    rng = np.random.default_rng(11)
    cases = [
        (4096, 128, 8, 128, rng.integers(0, 128, (4096, 8))),                         # larger first
        (37, 256, 8, 16, np.minimum(rng.zipf(1.3, (37, 8)) - 1, 255)),                # then smaller, skewed
        (1500, 256, 8, 64, np.minimum(rng.zipf(1.2, (1500, 8)) - 1, 255)),            # three-pass path again,
        (1100, 64, 8, 128, rng.integers(0, 64, (1100, 8))),                           # smaller, other E and BM
    ]
    for T, E, k, bm, ids_np in cases:
        ids = torch.from_numpy(ids_np.astype(np.int32)).cuda()
        ref = ops.align(ids, E, bm)
        got = _noalloc(ids, E, bm)
        torch.cuda.synchronize()
        for key in ("sorted_token_ids", "expert_ids", "num_tokens_post_padded", "expert_counts", "expert_offsets"):
            assert torch.equal(got[key], ref[key]), key


def test_noalloc_align_rejects_oversize_before_touching_the_device():
    L = ops.lib()
    T, k, E = 70000, 8, 128            # needs more than the 1 MiB static scratch
    assert L.moe_align_workspace_size(T, k, E) > (1 << 20)
    fake = ctypes.c_void_p(1 << 20)
    rc = L.moe_align_noalloc(fake, T, k, E, 16, fake, fake, fake, None, None, None)
    assert rc == ops.MOE_ERR_INVALID
    assert b"static" in L.moe_last_error_string()
    assert L.moe_align_noalloc(fake, 4, 2, 8, 16, None, fake, fake, None, None, None) == ops.MOE_ERR_INVALID
