"""Pins for the oracle's NVFP4 quantiser (CPU only).

Invariants the format fixes ("Why Gated DeltaNet Survives 4-Bit Quantization",
ai.info summary, "Methodology in Plain English": E2M1 values, one E4M3 scale
per 16-element block, the block maximum fixes the scale, an outlier degrades
only its own 15 neighbours):
  * the block holding the tensor maximum gets the largest scale, 448 (0x7E);
  * every element is within half a grid step (times S*g) of its dequantised value;
  * zero blocks give scale byte 0 and codes 0;
  * all-equal blocks give code +-6 everywhere;
  * changing one element (global scale held) changes only its own block;
  * sign flips flip only sign bits; power-of-two scaling leaves codes alone.
"""
import numpy as np
import pytest

from oracle import nvfp4_oracle as o


def _rand(shape, seed=0, outliers=()):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal(shape).astype(np.float32)
    for c in outliers:
        x[:, c] *= 50
    return x


def test_global_scale_closed_form():
    x = _rand((8, 64), 1)
    amax = np.float32(np.abs(x).max())
    g = o.global_scale(x)
    assert g == np.float32(amax / np.float32(2688.0))
    assert abs(float(g) * 6 * 448 - float(amax)) <= 1e-6 * float(amax)


def test_tensor_max_block_gets_448():
    x = _rand((16, 128), 2, outliers=(5,))
    codes, sf, g = o.quantize(x)
    r, c = np.unravel_index(np.argmax(np.abs(x)), x.shape)
    assert sf[r, c // 16] == 0x7E
    assert sf.max() == 0x7E
    # the maximum itself is coded as +-6
    assert codes[r, c] & 7 == 7


def test_block_max_maps_to_the_top_code():
    """The largest value of a block fixes its scale: with the scale byte in
    E4M3's normal, unsaturated range, the block maximum lands within E4M3's
    relative rounding (2^-4) of 6, so it is coded as +-6 (code magnitude 7),
    never as 4 or below."""
    x = _rand((32, 256), 9, outliers=(3, 77))
    codes, sf, g = o.quantize(x)
    S = o.e4m3_decode(sf)
    xb = np.abs(x).reshape(32, 16, 16)
    top = np.take_along_axis(codes.reshape(32, 16, 16), np.argmax(xb, axis=2)[:, :, None], axis=2)[:, :, 0]
    normal = (S >= 2.0 ** -6) & (sf < 0x7E)
    assert normal.sum() > 400
    assert np.all(top[normal] & 7 == 7)


def _grid_step(mag):
    return np.where(mag < 2, 0.5, np.where(mag < 4, 1.0, 2.0))


@pytest.mark.parametrize("seed", [0, 1, 2, 3])
def test_per_element_error_bound(seed):
    x = _rand((32, 256), seed, outliers=(3, 77, 200))
    codes, sf, g = o.quantize(x)
    xhat = o.dequantize(codes, sf, g)
    S = o.e4m3_decode(sf)
    normal = np.repeat(S >= 2.0 ** -6, 16, axis=1)
    Sg = np.repeat(S, 16, axis=1) * float(g)
    bound = 0.5 * _grid_step(np.abs(o.e2m1_decode(codes))) * Sg
    err = np.abs(x.astype(np.float64) - xhat)
    slack = 1e-6 * np.abs(x)
    assert np.all(err[normal] <= bound[normal] + slack[normal])
    # subnormal scales still stay inside the saturated range: |x| <= 6.5 S g
    assert np.all(np.abs(x) <= 6.5 * Sg + 1e-30 + slack)


def test_zero_blocks():
    x = _rand((4, 64), 4)
    x[1, 16:32] = 0.0
    x[3, :] = 0.0
    codes, sf, g = o.quantize(x)
    assert sf[1, 1] == 0 and np.all(codes[1, 16:32] == 0)
    assert np.all(sf[3] == 0) and np.all(codes[3] == 0)


def test_all_zero_tensor():
    codes, sf, g = o.quantize(np.zeros((3, 32), np.float32))
    assert g == 0 and not codes.any() and not sf.any()


def test_all_equal_blocks():
    x = _rand((4, 64), 5)
    x[0, 0:16] = 0.37
    x[2, 32:48] = -1.9
    codes, sf, g = o.quantize(x)
    assert np.all(codes[0, 0:16] == 7)
    assert np.all(codes[2, 32:48] == 15)
    S = o.e4m3_decode(sf[0, 0])
    xhat = o.dequantize(codes, sf, g)
    assert np.allclose(np.abs(xhat[0, 0:16] - 0.37), abs(0.37 - 6 * S * float(g)), rtol=0, atol=1e-7)


def test_outlier_isolated_to_its_block():
    x = _rand((4, 128), 6)
    g = o.global_scale(x) * np.float32(4)  # held fixed, with room for the outlier
    c0, s0, _ = o.quantize(x, g)
    y = x.copy()
    y[2, 37] = 9.0 * np.abs(x).max()
    c1, s1, _ = o.quantize(y, g)
    diff_c = np.argwhere(c0 != c1)
    diff_s = np.argwhere(s0 != s1)
    assert len(diff_s) == 1 and tuple(diff_s[0]) == (2, 37 // 16)
    assert np.all(diff_c[:, 0] == 2) and np.all(diff_c[:, 1] // 16 == 37 // 16)
    assert len(diff_c) > 1  # the 15 neighbours were re-coded under the larger scale


def test_sign_symmetry():
    x = _rand((8, 64), 7)
    c0, s0, g0 = o.quantize(x)
    c1, s1, g1 = o.quantize(-x)
    assert g0 == g1
    np.testing.assert_array_equal(s0, s1)
    np.testing.assert_array_equal(c1, c0 ^ 8)


def test_power_of_two_scaling_invariance():
    x = _rand((8, 64), 8)
    c0, s0, g0 = o.quantize(x)
    c1, s1, g1 = o.quantize(x * np.float32(8))
    assert g1 == g0 * 8
    np.testing.assert_array_equal(s0, s1)
    np.testing.assert_array_equal(c0, c1)


def test_static_scale_saturates():
    x = _rand((2, 32), 9)
    g = o.global_scale(x) / np.float32(100)  # calibrated far too small
    codes, sf, _ = o.quantize(x, g)
    assert np.all(sf == 0x7E)
    big = np.abs(x) > 6.5 * 448 * float(g)
    assert np.all(codes[big] & 7 == 7)


def test_pack_unpack_nibble_order():
    codes = np.arange(32, dtype=np.uint8).reshape(2, 16) % 16
    p = o.pack_codes(codes)
    assert p[0, 0] == (codes[0, 0] | (codes[0, 1] << 4))
    np.testing.assert_array_equal(o.unpack_codes(p), codes)


def test_quant_error_magnitude_sane():
    """Soft sanity: N(0,1) activations with outlier channels quantise with a
    relative error of the same order as the pages' A4 figures (7.5-9.2%)."""
    x = _rand((64, 512), 10, outliers=(7, 300))
    codes, sf, g = o.quantize(x)
    xhat = o.dequantize(codes, sf, g)
    rel = np.linalg.norm(x - xhat, axis=1) / np.linalg.norm(x, axis=1)
    assert 0.03 < np.median(rel) < 0.2
