"""Pins for the oracle's activation statistics (CPU only).

What fixes them, independently of the code:
  * hand-computed values on a tiny tensor (moments, amax, dominated blocks,
    per-row and per-column sums) by explicit Python loops;
  * a large Gaussian sample has kurtosis near 3 and max/RMS near its expected
    extreme; a Student-t sample with heavy tails has a much larger kurtosis;
  * a block with one nonzero value is dominated, an all-equal block is not;
  * values that NVFP4 represents exactly have zero A4 error, and the A4 error
    of random data stays below the quantiser's half-step bound;
  * one hot channel x100 gives a hot-channel ratio near 100.
"""
import math

import numpy as np

from oracle import nvfp4_oracle as o


def test_tiny_tensor_by_hand():
    x = np.array([[3.0] + [0.0] * 15 + [1.0] * 16,
                  [-2.0, 2.0] + [0.5] * 14 + [0.0] * 15 + [-8.0]], np.float32)
    st = o.activation_stats(x)
    flat = [float(v) for v in x.ravel()]
    assert st["n"] == 64
    assert math.isclose(st["sum"], sum(flat)) and math.isclose(st["sum_sq"], sum(v * v for v in flat))
    assert math.isclose(st["sum_cube"], sum(v ** 3 for v in flat)) and math.isclose(st["sum_4th"], sum(v ** 4 for v in flat))
    assert st["amax"] == 8.0 and st["blocks"] == 4
    # block 0: 3 > 0 (dominated); block 1: 1 > 15 no; block 2: 2 > 2 + 7 no; block 3: 8 > 0 yes
    assert st["dominated"] == 2
    for r in range(2):
        assert math.isclose(st["row_norm2"][r], sum(float(v) ** 2 for v in x[r]))
    for c in range(32):
        assert math.isclose(st["col_sq"][c], sum(float(x[r, c]) ** 2 for r in range(2)))
        assert st["col_max"][c] == max(abs(float(x[r, c])) for r in range(2))


def test_gaussian_and_heavy_tailed_moments():
    rng = np.random.default_rng(0)
    x = rng.standard_normal((512, 1024)).astype(np.float32)
    s = o.activation_summary(o.activation_stats(x))
    assert abs(s["kurtosis"] - 3.0) < 0.05
    assert 4.0 < s["max_over_rms"] < 6.5  # the largest of 0.5 M normals sits near 5 sigma
    # both are scale-free: x4 (exact in FP32) changes neither
    s4 = o.activation_summary(o.activation_stats(4 * x))
    assert abs(s4["kurtosis"] - s["kurtosis"]) <= 1e-9 * s["kurtosis"]
    assert abs(s4["max_over_rms"] - s["max_over_rms"]) <= 1e-12 * s["max_over_rms"]
    t = rng.standard_t(3, (512, 1024)).astype(np.float32)
    assert o.activation_summary(o.activation_stats(t))["kurtosis"] > 10


def test_dominated_blocks_and_exact_values():
    x = np.zeros((4, 64), np.float32)
    x[:, ::16] = 5.0  # one nonzero per block
    assert o.activation_summary(o.activation_stats(x))["dominated_share"] == 1.0
    y = np.full((4, 64), 0.3, np.float32)
    assert o.activation_summary(o.activation_stats(y))["dominated_share"] == 0.0
    # dominance compares magnitudes: sixteen equal negative values are not
    # dominated, and one large negative value among small ones is
    assert o.activation_summary(o.activation_stats(-y))["dominated_share"] == 0.0
    z = np.full((1, 16), 0.1, np.float32)
    z[0, 3] = -5.0
    assert o.activation_stats(z)["dominated"] == 1.0
    # a tensor NVFP4 represents exactly: every block holds +-6, so S = 448, and
    # the global scale 6 * 0.4375 / 2688 = 2^-10 is exact, as is e2m1 * S * g
    vals = (np.array([0.5, 1, 1.5, 2, 3, 4, 6, -6] * 8, np.float32) * np.float32(0.4375)).reshape(4, 16)
    st = o.activation_stats(vals)
    assert np.all(st["row_err2"] == 0)


def test_a4_error_within_the_half_step_bound_and_hot_channel():
    rng = np.random.default_rng(1)
    x = rng.standard_normal((256, 512)).astype(np.float32)
    x[:, 77] *= 100
    st = o.activation_stats(x)
    s = o.activation_summary(st)
    # the element error is at most half the top grid step (1 * S * g) and S * g <= amax_b / 5.5 or so: well below 25%
    assert 0.0 < s["a4_err_max"] < 0.25 and s["a4_err_min"] > 0.0
    # one channel x100 over N(0, 1) channels: about 100, within the sampling of 256 rows
    assert 92 < s["hot_channel_ratio"] < 112
