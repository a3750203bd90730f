"""Pins of the oracle's number formats against the format definitions and
independent library implementations (torch's bf16 / float8_e4m3fn casts)."""

import json
import os

import numpy as np
import pytest
import torch

from oracle import moe_oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _torch_bf16(x):
    return torch.from_numpy(np.asarray(x, dtype=np.float32)).to(torch.bfloat16).to(torch.float64).numpy()


def test_bf16_matches_torch_on_random_and_tie_values():
    rng = np.random.default_rng(1)
    x = np.concatenate([
        rng.standard_normal(200_000).astype(np.float32),
        (rng.standard_normal(50_000) * 1e-30).astype(np.float32),
        (rng.standard_normal(50_000) * 1e30).astype(np.float32),
        np.array([0.0, -0.0, 1.0, -1.0, 3.0e38, -3.0e38, 1e-45, 1e-40], dtype=np.float32),
    ])
    # exact halfway cases between neighbouring bf16 values (low 16 bits = 0x8000)
    bits = (rng.integers(0, 2**15, 20_000, dtype=np.uint32) << 16) | np.uint32(0x8000)
    x = np.concatenate([x, bits.view(np.float32)[np.isfinite(bits.view(np.float32))]])
    ours = O.round_bf16(x.astype(np.float64))
    ref = _torch_bf16(x)
    np.testing.assert_array_equal(ours, ref)


def test_e4m3_decode_matches_golden_table_and_torch():
    with open(os.path.join(GOLDEN, "e4m3_codes.json")) as f:
        gold = json.load(f)
    for code, val in gold["codes"].items():
        got = O.e4m3_decode(np.array([int(code, 16)], dtype=np.uint8))[0]
        assert got == val and np.signbit(got) == np.signbit(val), code
    for code in gold["nan_codes"]:
        assert np.isnan(O.e4m3_decode(np.array([int(code, 16)], dtype=np.uint8))[0])
    codes = np.arange(256, dtype=np.uint8)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    ours = O.e4m3_decode(codes)
    np.testing.assert_array_equal(np.isnan(ours), np.isnan(ref))
    np.testing.assert_array_equal(ours[~np.isnan(ours)], ref[~np.isnan(ref)])


def _brute_nearest_e4m3(v):
    """Nearest finite E4M3 value by exhaustive search; ties -> even code."""
    codes = np.arange(256)
    vals = O.e4m3_decode(codes.astype(np.uint8))
    keep = np.isfinite(vals) & ~((vals == 0) & np.signbit(vals))
    codes, vals = codes[keep], vals[keep]
    out = np.empty_like(v)
    for i, x in enumerate(v):
        x = min(max(x, -448.0), 448.0)
        d = np.abs(vals - x)
        best = np.nonzero(d == d.min())[0]
        if best.size > 1:   # tie: the code with an even mantissa (last bit 0)
            best = best[(codes[best] & 1) == 0]
        out[i] = vals[best[0]]
    return out


def test_e4m3_round_matches_exhaustive_search():
    rng = np.random.default_rng(2)
    vals = O.e4m3_decode(np.arange(0, 0x7F, dtype=np.uint8))
    mids = (vals[1:] + vals[:-1]) / 2.0                      # every positive halfway point
    v = np.concatenate([
        rng.uniform(-470, 470, 3000),
        rng.standard_normal(3000) * 0.01,
        mids, -mids, vals, -vals,
        np.array([448.0, 455.0, 464.0, 470.0, 1000.0, -1000.0]),
    ])
    ours = O.e4m3_round(v)
    ref = _brute_nearest_e4m3(v)
    np.testing.assert_array_equal(np.abs(ours), np.abs(ref))


def test_e4m3_encode_matches_torch_cast():
    rng = np.random.default_rng(3)
    v = np.concatenate([rng.uniform(-448, 448, 100_000), rng.standard_normal(100_000) * 0.02,
                        O.e4m3_decode(np.arange(0, 0x7F, dtype=np.uint8))])
    v32 = v.astype(np.float32)
    ours = O.e4m3_encode(v32.astype(np.float64))
    ref = torch.from_numpy(v32).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    np.testing.assert_array_equal(ours, ref)
    # round trip of every finite code
    codes = np.array([c for c in range(256) if (c & 0x7F) != 0x7F], dtype=np.uint8)
    np.testing.assert_array_equal(O.e4m3_encode(O.e4m3_decode(codes)), codes)


def test_pow2_ceil_matches_exhaustive_search():
    rng = np.random.default_rng(4)
    s = np.concatenate([np.exp(rng.uniform(-60, 20, 2000)), 2.0 ** np.arange(-50, 20)])
    s = s.astype(np.float32).astype(np.float64)
    got = O.pow2_ceil(s)
    for si, gi in zip(s, got):
        k = -200
        while 2.0 ** k < si:
            k += 1
        assert gi == 2.0 ** k


def test_act_quant_properties_and_independent_torch_path():
    rng = np.random.default_rng(5)
    p = O.round_bf16(rng.standard_normal((64, 512)) * np.exp(rng.uniform(-6, 3, (64, 1))))
    p[3, :128] = 0.0                                          # an all-zero group
    codes, scales = O.quantize_act_group128(p)
    s = scales.astype(np.float64)
    m, _ = np.frexp(s)
    assert np.all(m == 0.5), "scales must be powers of two"
    amax = np.abs(p.reshape(64, 4, 128)).max(-1)
    nz = amax > 0
    ratio = amax[nz] / s[nz]
    assert np.all(ratio <= 448.0) and np.all(ratio > 224.0)
    # zero group: scale is the power of two at or above fp32(1e-10) * fp32(1/448)
    floor = np.float32(np.float32(1e-10) * np.float32(1.0 / 448.0))
    assert s[3, 0] >= floor and s[3, 0] < 2 * floor
    deq = O.dequantize_act_group128(codes, scales)
    # independent path: torch computes amax, log2/ceil/exp2 and the float8 cast
    pt = torch.from_numpy(p).reshape(64, 4, 128)
    raw = torch.clamp(pt.abs().amax(-1).float(), min=1e-10) * torch.tensor(1.0 / 448.0, dtype=torch.float32)
    sc = torch.exp2(torch.ceil(torch.log2(raw.double())))
    q = torch.clamp(pt / sc[..., None], -448, 448).float().to(torch.float8_e4m3fn).double()
    ref = (q * sc[..., None]).reshape(64, 512).numpy()
    np.testing.assert_array_equal(deq, ref)
    # error within half a unit in the last place of E4M3 (relative 2**-4) times the scale
    err = np.abs(deq - p).reshape(64, 4, 128)
    assert np.all(err <= np.maximum(np.abs(p).reshape(64, 4, 128) * 2.0 ** -4, 2.0 ** -10 * s[..., None]) + 0)


def test_weight_block_quant_properties_and_torch_path():
    rng = np.random.default_rng(6)
    w = O.round_bf16(rng.standard_normal((2, 256, 384)) * 0.02)
    w[1, 128:, 256:] = 0.0                                    # an all-zero block
    codes, scales = O.quantize_weight_block128(w)
    assert codes.shape == w.shape and scales.shape == (2, 2, 3)
    vals = O.e4m3_decode(codes)
    blk = np.abs(vals).reshape(2, 2, 128, 3, 128).max(axis=(2, 4))
    nz = scales > np.float32(1e-9)
    assert np.all(blk[nz] == 448.0), "the block maximum must map to +-448"
    assert scales[1, 1, 2] == np.float32(np.float32(1e-10) / np.float32(448.0))
    # independent path: torch fp32 division and float8 cast
    wt = torch.from_numpy(w).float().reshape(2, 2, 128, 3, 128)
    st = torch.from_numpy(scales)[:, :, None, :, None]
    ref = (wt / st).to(torch.float8_e4m3fn).view(torch.uint8).reshape(2, 256, 384).numpy()
    np.testing.assert_array_equal(codes, ref)
    deq = O.dequantize_weight_block128(codes, scales)
    # half a unit in the last place: relative 2**-4 for normals, 2**-10 * scale below 2**-6 * scale
    full_s = np.repeat(np.repeat(scales.astype(np.float64), 128, 1), 128, 2)
    bound = np.maximum(np.abs(w) * 2.0 ** -4, 2.0 ** -10 * full_s) * (1 + 1e-6)
    assert np.all(np.abs(deq - w) <= bound)


def test_mx_quant_properties_and_independent_torch_path():
    rng = np.random.default_rng(7)
    p = O.round_bf16(rng.standard_normal((16, 256)) * np.exp(rng.uniform(-6, 3, (16, 1))))
    p[2, 32:64] = 0.0                                         # an all-zero 32-group
    p[5, 100] = 1000.0                                        # one large value: only its group's scale moves
    codes, e8m0 = O.quantize_mx_group32(p)
    assert codes.shape == p.shape and e8m0.shape == (16, 8) and e8m0.dtype == np.uint8
    s = O.mx_scale(e8m0)
    assert np.all(np.frexp(s)[0] == 0.5), "scales must be powers of two"
    amax = np.abs(p.reshape(16, 8, 32)).max(-1)
    nz = amax > 0
    ratio = amax[nz] / s[nz]
    assert np.all(ratio <= 448.0) and np.all(ratio > 224.0)
    assert e8m0[5, 3] > e8m0[5, 2] and e8m0[5, 3] > e8m0[5, 4]
    floor = np.float32(np.float32(1e-10) * np.float32(1.0 / 448.0))
    assert s[2, 1] >= floor and s[2, 1] < 2 * floor
    # the E8M0 byte is the biased exponent of the scale
    np.testing.assert_array_equal(e8m0.astype(np.int64) - 127, np.frexp(s)[1] - 1)
    # independent path: torch amax over 32-groups, log2/ceil/exp2, float8 cast
    pt = torch.from_numpy(p).reshape(16, 8, 32)
    raw = torch.clamp(pt.abs().amax(-1).float(), min=1e-10) * torch.tensor(1.0 / 448.0, dtype=torch.float32)
    sc = torch.exp2(torch.ceil(torch.log2(raw.double())))
    q = torch.clamp(pt / sc[..., None], -448, 448).float().to(torch.float8_e4m3fn)
    np.testing.assert_array_equal(codes, q.view(torch.uint8).reshape(16, 256).numpy())
    np.testing.assert_array_equal(s, sc.numpy())
    deq = O.dequantize_mx_group32(codes, e8m0)
    err = np.abs(deq - p).reshape(16, 8, 32)
    assert np.all(err <= np.maximum(np.abs(p).reshape(16, 8, 32) * 2.0 ** -4, 2.0 ** -10 * s[..., None]))


def test_page_constants_fixture():
    with open(os.path.join(GOLDEN, "pr64760_quant_constants.json")) as f:
        gold = json.load(f)
    assert O.E4M3_MAX == gold["fp8_max"]
    # a group whose amax is exactly 448 * 2**n gets the scale 2**n
    v = np.zeros((1, gold["group_k"]))
    v[0, 5] = 448.0 * 2.0 ** -7
    _, sc = O.quantize_act_group128(v)
    assert sc[0, 0] == 2.0 ** -7
    # below the floor the scale stops shrinking
    v[0, 5] = 1e-20
    _, sc = O.quantize_act_group128(v)
    assert sc[0, 0] == O.pow2_ceil(np.float32(np.float32(gold["amax_floor"]) * np.float32(1 / 448.0)))


def test_quantisers_read_bf16_bit_patterns_as_their_values():
    """The weight quantisers take bf16 weights either as values or as raw bit patterns (what a
    host copy of a bf16 tensor holds); both give the same codes and scales."""
    w = torch.randn(256, 384, generator=torch.Generator().manual_seed(8)).to(torch.bfloat16) * 0.02
    bits = w.view(torch.int16).numpy().view(np.uint16)
    vals = w.double().numpy()
    for quant in (O.quantize_weight_block128, O.quantize_mx_group32):
        a, sa = quant(bits)
        b, sb = quant(vals)
        np.testing.assert_array_equal(a, b)
        np.testing.assert_array_equal(sa, sb)
