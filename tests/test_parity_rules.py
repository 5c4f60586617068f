"""The comparison rules the GPU parity tests apply (tests/gpu_helpers.py),
checked on CPU so that a checker that passes too easily cannot hide a wrong
result: the FP32 accumulation bound, the BF16 one-ulp rule with its
propagated-tolerance fallback, the FP32 ulp, and the un-swizzling of the
tcgen05 block-scale layout (against a layout built here from the
128-row x 4-scale atom description, one byte at a time)."""
import numpy as np
import pytest

from oracle import nvfp4_oracle as o
from tests.gpu_helpers import check_bf16, check_fp32, f32_ulp, unswizzle_sf


def test_fp32_rule_accepts_the_bound_and_rejects_beyond_it():
    y = np.array([1.0, -2.0, 1e3])
    mag = np.array([10.0, 10.0, 1e4])
    tol = 1e-5 * mag
    assert check_fp32(y + 0.99 * tol, y, mag) < 1.0
    with pytest.raises(AssertionError):
        check_fp32(y + np.array([0, 0, 1.01]) * tol, y, mag)


def test_bf16_rule():
    rng = np.random.default_rng(0)
    y = rng.standard_normal(1000) * 10
    yb = o.bf16_round(y)
    ulp = o.bf16_ulp(yb)
    zero_tol = np.zeros_like(y)
    check_bf16(yb, y, zero_tol)              # the correctly rounded value
    check_bf16(yb + ulp, y, zero_tol)        # one ulp away is allowed
    with pytest.raises(AssertionError):      # two ulps away is not, without tolerance
        check_bf16(yb + 2 * ulp, y, zero_tol)
    # the fallback: a propagated tolerance larger than half an ulp admits the value it covers
    big = 3 * ulp
    check_bf16(o.bf16_round(y + 2.5 * ulp), y, big)


def test_f32_ulp():
    assert f32_ulp(1.0) == 2.0 ** -23
    assert f32_ulp(-3.0) == 2.0 ** -22
    assert f32_ulp(0.0) > 0


def test_unswizzle_matches_the_atom_description():
    rows, K = 200, 320  # two row blocks, five 64-wide K chunks
    KA = (K + 63) // 64
    rows_pad = 256
    logical = np.arange(rows_pad * KA * 4, dtype=np.int64).reshape(rows_pad, KA * 4) % 251
    # atoms of 512 bytes: 128 rows x 4 scales, K-chunks fastest within a row block;
    # row r of an atom at (r % 32) * 16 + ((r // 32) % 4) * 4, scale j at + j % 4
    raw = np.zeros(rows_pad * KA * 4, np.int64)
    for r in range(rows_pad):
        for j in range(KA * 4):
            atom = (r // 128) * KA + j // 4
            raw[atom * 512 + (r % 32) * 16 + ((r // 32) % 4) * 4 + j % 4] = logical[r, j]
    assert np.array_equal(unswizzle_sf(raw, rows, K), logical)
