"""Pins for the oracle's E2M1 and E4M3 codecs (CPU only).

The oracle writes both codecs from their bit-field definitions and a nearest-
value search.  These tests check them against things that do not share that
code: hand-written value tables (tests/golden), exact rational arithmetic, and
two independent library conversions (ml_dtypes, torch.float8_e4m3fn).
"""
from fractions import Fraction
import math
import os

import ml_dtypes
import numpy as np
import pytest
import torch

from oracle import nvfp4_oracle as o


def _read_table(path):
    rows = []
    with open(path) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            rows.append(line.split())
    return rows


# ---------------------------------------------------------------- E2M1


def test_e2m1_values_match_golden(golden_dir):
    for code, val in _read_table(os.path.join(golden_dir, "e2m1_values.txt")):
        v = o.e2m1_value(int(code))
        assert v == float(val) and math.copysign(1, v) == math.copysign(1, float(val)), code


def test_e2m1_rounding_golden(golden_dir):
    rows = _read_table(os.path.join(golden_dir, "e2m1_rounding.txt"))
    x = np.array([float(r[0]) for r in rows], np.float32)
    want = np.array([int(r[1]) for r in rows], np.uint8)
    np.testing.assert_array_equal(o.e2m1_encode(x), want)


def test_e2m1_roundtrip_all_codes():
    codes = np.arange(16, dtype=np.uint8)
    vals = np.array([o.e2m1_value(int(c)) for c in codes], np.float32)
    np.testing.assert_array_equal(o.e2m1_encode(vals), codes)


def _e2m1_nearest_exact(x: float) -> int:
    """Brute force: exact rational distance to every non-negative value,
    ties to the even code, saturation at 6, sign kept."""
    fx = Fraction(abs(x)) if math.isfinite(x) else None
    if fx is None or fx >= 6:
        best = 7
    else:
        cands = [(abs(fx - Fraction(o.e2m1_value(c))), c % 2, c) for c in range(8)]
        best = min(cands)[2]
    return best + (8 if math.copysign(1.0, x) < 0 else 0)


def test_e2m1_vs_exact_rational_sweep():
    grid = np.arange(-8 * 64, 8 * 64 + 1, dtype=np.float64) / 64.0  # all multiples of 1/64
    rng = np.random.default_rng(0)
    extra = rng.uniform(-7, 7, 2000)
    x = np.concatenate([grid, extra]).astype(np.float32)
    got = o.e2m1_encode(x)
    want = np.array([_e2m1_nearest_exact(float(v)) for v in x], np.uint8)
    np.testing.assert_array_equal(got, want)


def test_e2m1_vs_ml_dtypes():
    rng = np.random.default_rng(1)
    x = np.concatenate([
        rng.standard_normal(200000).astype(np.float32) * 3,
        (np.arange(-1000, 1001) / 128.0).astype(np.float32),
        np.array([0.0, -0.0, 6.0, 6.5, -6.5, 100.0, -1e30], np.float32),
    ])
    ref = x.astype(ml_dtypes.float4_e2m1fn).view(np.uint8) & 15
    np.testing.assert_array_equal(o.e2m1_encode(x), ref)


def test_e2m1_decode_table_vs_ml_dtypes():
    codes = np.arange(16, dtype=np.uint8)
    ref = codes.view(ml_dtypes.float4_e2m1fn).astype(np.float64)
    np.testing.assert_array_equal(o.e2m1_decode(codes), ref)


# ---------------------------------------------------------------- E4M3


def test_e4m3_values_match_golden(golden_dir):
    for code, val in _read_table(os.path.join(golden_dir, "e4m3_values.txt")):
        assert o.e4m3_value(int(code, 16)) == float(val), code


def test_e4m3_rounding_golden(golden_dir):
    rows = _read_table(os.path.join(golden_dir, "e4m3_rounding.txt"))
    x = np.array([float(r[0]) for r in rows], np.float32)
    want = np.array([int(r[1], 16) for r in rows], np.uint8)
    np.testing.assert_array_equal(o.e4m3_encode_nonneg(x), want)


def test_e4m3_decode_all_256_vs_torch():
    codes = torch.arange(256, dtype=torch.uint8)
    ref = codes.view(torch.float8_e4m3fn).to(torch.float64).numpy()
    got = o.e4m3_decode(np.arange(256))
    nan = np.isnan(ref)
    assert np.array_equal(nan, np.isnan(got))
    assert nan.sum() == 2  # 0x7F and 0xFF
    np.testing.assert_array_equal(got[~nan], ref[~nan])


def test_e4m3_roundtrip_and_midpoints():
    codes = np.arange(127)
    vals = o.e4m3_decode(codes).astype(np.float32)
    np.testing.assert_array_equal(o.e4m3_encode_nonneg(vals), codes)
    mids = ((o.E4M3_POS[:-1] + o.E4M3_POS[1:]) / 2).astype(np.float32)
    assert np.all(mids.astype(np.float64) == (o.E4M3_POS[:-1] + o.E4M3_POS[1:]) / 2)  # exact
    want = np.where(codes[:-1] % 2 == 0, codes[:-1], codes[:-1] + 1)
    np.testing.assert_array_equal(o.e4m3_encode_nonneg(mids), want)


def test_e4m3_saturates():
    x = np.array([448.0, 449.0, 464.0, 480.0, 1e6, np.inf], np.float32)
    np.testing.assert_array_equal(o.e4m3_encode_nonneg(x), np.full(6, 0x7E))


def test_e4m3_vs_torch_and_ml_dtypes_in_range():
    rng = np.random.default_rng(2)
    x = np.concatenate([
        rng.uniform(0, 448, 100000), np.exp(rng.uniform(np.log(1e-4), np.log(448), 100000)),
        rng.uniform(0, 2 ** -6, 20000),
    ]).astype(np.float32)
    got = o.e4m3_encode_nonneg(x)
    ref_t = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    ref_m = x.astype(ml_dtypes.float8_e4m3fn).view(np.uint8)
    np.testing.assert_array_equal(got, ref_t)
    np.testing.assert_array_equal(got, ref_m)


def test_e4m3_vs_exact_rational_random():
    rng = np.random.default_rng(3)
    x = np.exp(rng.uniform(np.log(1e-5), np.log(500), 3000)).astype(np.float32)
    vals = [Fraction(float(v)) for v in o.E4M3_POS]
    for xi, ci in zip(x, o.e4m3_encode_nonneg(x)):
        fx = Fraction(float(xi))
        if fx >= 448:
            assert ci == 0x7E
            continue
        best = min((abs(fx - v), c % 2, c) for c, v in enumerate(vals))[2]
        assert ci == best, float(xi)
