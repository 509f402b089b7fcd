"""Pins for oracle/formats.py against torch's conversions (an independent
library) and against values fixed by the format definitions."""

import json
import os

import numpy as np
import torch

from oracle import formats as F

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def test_bf16_decode_exhaustive_vs_torch():
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    ours = F.bf16_to_f64(bits)
    ref = torch.from_numpy(bits.view(np.int16).copy()).view(torch.bfloat16).double().numpy()
    same = (ours == ref) | (np.isnan(ours) & np.isnan(ref))
    assert same.all()


def test_bf16_encode_vs_torch_random_and_midpoints():
    rng = np.random.default_rng(0)
    x = rng.standard_normal(200_000).astype(np.float32) * np.float32(3.0)
    # exact midpoints between neighbouring bf16 values, and their neighbours
    hi = rng.integers(0, 0x7F7F, 50_000, dtype=np.uint32) << np.uint32(16)
    mid = (hi | np.uint32(0x8000)).view(np.float32)
    xs = np.concatenate([x, mid, np.nextafter(mid, np.float32(np.inf)), np.nextafter(mid, np.float32(-np.inf))])
    ours = F.f32_to_bf16(xs)
    ref = torch.from_numpy(xs).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(ours, ref)


def test_f16_encode_vs_torch_on_fp32_exact_values():
    rng = np.random.default_rng(1)
    # fp16 midpoints have 12 significant bits: exact in fp32, so torch's
    # float path and our single rounding from float64 must agree
    h = rng.integers(0, 0x7BFF, 100_000, dtype=np.uint16)
    lo = h.view(np.float16).astype(np.float64)
    hi_ = (h + 1).view(np.float16).astype(np.float64)
    mids = (lo + hi_) / 2
    xs = np.concatenate([mids, -mids, rng.standard_normal(100_000).astype(np.float32).astype(np.float64)])
    ours = F.f64_to_f16(xs)
    ref = torch.from_numpy(xs.astype(np.float32)).to(torch.float16).numpy()
    assert np.array_equal(ours.view(np.uint16), ref.view(np.uint16))


def test_f16_definition_points():
    v = F.f64_to_f16(np.array([65504.0, 2.0 ** -24, 1 + 2.0 ** -11, 1 + 3 * 2.0 ** -11, 2.0 ** -25]))
    assert v[0] == 65504.0  # largest finite
    assert v[1] == 2.0 ** -24  # smallest subnormal
    assert v[2] == 1.0  # tie -> even
    assert v[3] == 1 + 2.0 ** -9  # tie -> even (up)
    assert v[4] == 0.0  # half the smallest subnormal ties to zero


def test_e4m3_decode_exhaustive_vs_torch():
    codes = np.arange(256, dtype=np.uint8)
    ours = F.e4m3_to_f64(codes)
    ref = torch.from_numpy(codes.copy()).view(torch.float8_e4m3fn).double().numpy()
    same = (ours == ref) | (np.isnan(ours) & np.isnan(ref))
    assert same.all()


def test_e4m3_definition_points():
    assert F.E4M3_VALUES[0x7E] == 448.0
    assert F.E4M3_VALUES[0x01] == 2.0 ** -9
    assert F.E4M3_VALUES[0x38] == 1.0
    assert np.isnan(F.E4M3_VALUES[0x7F]) and np.isnan(F.E4M3_VALUES[0xFF])
    # saturation instead of NaN for finite out-of-range values
    assert list(F.f32_to_e4m3(np.array([449.0, 464.0, 500.0, 1e30], np.float32))) == [0x7E] * 4


def test_e4m3_encode_vs_torch_in_range():
    rng = np.random.default_rng(2)
    grid = F.E4M3_VALUES[:0x7F]
    mids = ((grid[:-1] + grid[1:]) / 2).astype(np.float32)
    xs = np.concatenate([
        rng.uniform(0, 448, 100_000).astype(np.float32),
        np.exp(rng.uniform(np.log(1e-4), np.log(448), 100_000)).astype(np.float32),
        mids, np.nextafter(mids, np.float32(0)), np.nextafter(mids, np.float32(1e9)),
    ])
    xs = xs[xs <= 448]
    ours = F.f32_to_e4m3(xs)
    ref = torch.from_numpy(xs).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(ours, ref)


def test_e2m1_values_from_bitfields():
    # E2M1: exponent bias 1, one mantissa bit; the grid of the OCP MX format
    expect = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]
    assert list(F.E2M1_VALUES[:8]) == expect
    assert list(F.E2M1_VALUES[8:]) == [-v for v in expect]


def test_e2m1_round_nearest_even_and_saturate():
    xs = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, 7.0, 100.0, 0.26, 4.9, 5.1], np.float32)
    want = [0.0, 1.0, 1.0, 2.0, 2.0, 4.0, 4.0, 6.0, 6.0, 0.5, 4.0, 6.0]
    assert list(F.e2m1_to_f64(F.f32_to_e2m1(xs))) == want
    neg = F.f32_to_e2m1(-xs)
    assert list(F.e2m1_to_f64(neg)) == [-w for w in want]
    assert F.f32_to_e2m1(np.array([-0.1], np.float32))[0] == 0x8  # sign kept on a zero result


def test_e2m1_grid_is_exact_in_e4m3_and_bf16():
    g = F.E2M1_VALUES.astype(np.float32)
    assert np.array_equal(F.e4m3_to_f64(F.f32_to_e4m3(np.abs(g))), np.abs(g))
    assert np.array_equal(F.bf16_to_f64(F.f32_to_bf16(g)), g.astype(np.float64))


def test_bf16_rounding_of_fp16_scales_within_published_bound():
    bound = json.load(open(os.path.join(GOLDEN, "awq_scale_bf16_bound.json")))["max_relative_change"]
    h = np.arange(0x0400, 0x7C00, dtype=np.uint16)  # every positive normal fp16
    s = h.view(np.float16).astype(np.float32)
    b = F.bf16_to_f64(F.f32_to_bf16(s))
    rel = np.abs(b - s) / s
    assert rel.max() <= bound
    # truncation instead of rounding would break the published bound
    trunc = F.bf16_to_f64((s.view(np.uint32) >> 16).astype(np.uint16))
    assert (np.abs(trunc - s) / s).max() > bound
