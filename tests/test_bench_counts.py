"""The roofline numerators of bench.py, against hand-worked figures (CPU only)."""

import numpy as np
import pytest

import bench
from moe_layer_top_b200 import inputs


def test_bf16_decode_bytes_per_expert_and_layer():
    cfg = inputs.CONFIGS["decode_bf16"]          # H=4096, I=1536, E=128, top-8, bf16
    counts = np.zeros(cfg.E, dtype=np.int64)
    counts[:8] = 1                                # T = 1: eight experts with one assignment each
    a = bench.algorithmic_counts(cfg, 1, counts, 8 * 16, has_logits=True)
    assert a["w13_bytes_per_expert"] == 25_165_824          # 2 x 1536 x 4096 x 2 B
    assert a["w2_bytes_per_expert"] == 12_582_912           # 4096 x 1536 x 2 B  (37.75 MB per expert)
    assert a["hit_experts"] == 8
    # weights of 8 experts + x and out (4096 x 2 B each) + the logits (128 x 4 B)
    assert a["layer_bytes"] == 8 * 37_748_736 + 2 * 8192 + 512
    assert a["flops"] == 2.0 * 8 * 3 * 4096 * 1536


def test_fp8_block_scales_and_gemm_rows():
    cfg = inputs.CONFIGS["prefill_fp8"]           # FP8 codes + fp32 128x128 block scales
    counts = np.full(cfg.E, 1024, dtype=np.int64)  # 131072 assignments over 128 experts
    a = bench.algorithmic_counts(cfg, 16384, counts, 131072, has_logits=True)
    assert a["w13_bytes_per_expert"] == 3072 * 4096 + (3072 // 128) * (4096 // 128) * 4
    assert a["w2_bytes_per_expert"] == 4096 * 1536 + 32 * 12 * 4
    # GEMM1: weights + sorted token rows (E4M3) + a2 rows (E4M3); GEMM2: weights + a2 rows + y rows (bf16)
    assert a["gemm1_bytes"] == 128 * a["w13_bytes_per_expert"] + 131072 * 4096 + 131072 * 1536
    assert a["gemm2_bytes"] == 128 * a["w2_bytes_per_expert"] + 131072 * 1536 + 131072 * 4096 * 2
    assert a["flops"] == pytest.approx(4.9478e12, rel=1e-4)   # 2 T k 3 H I


def test_mx_scale_bytes_and_routing_ids_input():
    cfg = inputs.CONFIGS["decode_mxfp8"]          # one E8M0 byte per 32 weights
    counts = np.zeros(cfg.E, dtype=np.int64)
    counts[3] = 2
    a = bench.algorithmic_counts(cfg, 2, counts, 128, has_logits=False)
    assert a["w13_bytes_per_expert"] == 3072 * 4096 * 33 / 32
    assert a["hit_experts"] == 1
    # ids + weights input (8 bytes per assignment) instead of logits
    assert a["layer_bytes"] == a["w13_bytes_per_expert"] + a["w2_bytes_per_expert"] + 2 * 4096 * 4 + 2 * 8 * 8
