"""Pins for the oracle's GEMM, epilogues and fused projection (CPU only)."""
from fractions import Fraction
import math

import numpy as np
import pytest

from oracle import nvfp4_oracle as o


def _q(shape, seed, scale=1.0):
    rng = np.random.default_rng(seed)
    x = (scale * rng.standard_normal(shape)).astype(np.float32)
    return o.quantize(x)


def _brute_force(a_codes, a_sf, w_codes, w_sf):
    """Exact rational dequant-matmul with explicit loops, independent loop
    order (k outermost), no numpy arithmetic."""
    M, K = a_codes.shape
    N = w_codes.shape[0]
    acc = [[Fraction(0)] * N for _ in range(M)]
    for k in range(K):
        for m in range(M):
            av = Fraction(o.e2m1_value(int(a_codes[m, k]))) * Fraction(o.e4m3_value(int(a_sf[m, k // 16])))
            for n in range(N):
                wv = Fraction(o.e2m1_value(int(w_codes[n, k]))) * Fraction(o.e4m3_value(int(w_sf[n, k // 16])))
                acc[m][n] += av * wv
    return acc


def test_gemm_exact_vs_brute_force():
    a = _q((3, 48), 0)
    w = _q((5, 48), 1, 0.02)
    acc, mag = o.gemm(a[0], a[1], w[0], w[1])
    ref = _brute_force(a[0], a[1], w[0], w[1])
    assert acc.shape == (3, 5)
    for m in range(3):
        for n in range(5):
            assert Fraction(float(acc[m, n])) == ref[m][n]  # exact: < 53 bits of range


def test_gemm_is_not_transposed():
    a = _q((2, 32), 2)
    w = _q((4, 32), 3)
    acc, _ = o.gemm(a[0], a[1], w[0], w[1])
    ref = _brute_force(a[0], a[1], w[0], w[1])
    assert acc.shape == (2, 4)
    assert float(ref[1][3]) == acc[1, 3]


def test_magnitude_sum_bounds_accumulation():
    a = _q((4, 64), 4)
    w = _q((6, 64), 5)
    acc, mag = o.gemm(a[0], a[1], w[0], w[1])
    assert np.all(np.abs(acc) <= mag)


def test_linear_global_scales_multiply():
    rng = np.random.default_rng(6)
    x = rng.standard_normal((4, 64)).astype(np.float32)
    w = (0.02 * rng.standard_normal((3, 64))).astype(np.float32)
    y, mag, aq, wq = o.linear(x, w)
    acc, _ = o.gemm(aq[0], aq[1], wq[0], wq[1])
    np.testing.assert_array_equal(y, acc * float(aq[2]) * float(wq[2]))
    # the W4A4 product approximates the exact product within a few percent
    exact = x.astype(np.float64) @ w.T.astype(np.float64)
    assert np.linalg.norm(y - exact) / np.linalg.norm(exact) < 0.2


def test_sigmoid_softplus_closed_forms():
    assert o.sigmoid(0.0) == 0.5
    assert abs(float(o.softplus(0.0)) - math.log(2)) < 1e-16
    t = np.linspace(-30, 30, 121)
    np.testing.assert_allclose(o.sigmoid(t) + o.sigmoid(-t), 1.0, rtol=0, atol=1e-15)
    np.testing.assert_allclose(o.softplus(t) - o.softplus(-t), t, rtol=0, atol=1e-13)
    ref = np.array([1.0 / (1.0 + math.exp(-v)) for v in t])
    np.testing.assert_allclose(o.sigmoid(t), ref, rtol=1e-15, atol=0)
    ref_sp = np.array([math.log1p(math.exp(v)) if v < 0 else v + math.log1p(math.exp(-v)) for v in t])
    np.testing.assert_allclose(o.softplus(t), ref_sp, rtol=1e-14, atol=0)
    assert float(o.softplus(800.0)) == 800.0  # asymptote, no overflow


def test_gdn_decay_closed_form():
    a_log = np.array([0.0, 0.5, -1.0])
    dt = np.array([0.3, -0.2, 1.0])
    y = -dt  # softplus(0) = ln 2
    got = o.gdn_decay(y, a_log, dt)
    np.testing.assert_allclose(got, -np.exp(a_log) * math.log(2), rtol=1e-15)
    assert np.all(o.gdn_decay(np.array([5.0, -5.0, 0.0]), a_log, dt) < 0)
    # large positive pre-activation: softplus -> identity
    np.testing.assert_allclose(o.gdn_decay(np.array([100.0]), np.array([0.0]), np.array([0.0])), -100.0)


def test_swiglu_closed_form():
    assert o.swiglu(0.0, 5.0) == 0.0
    np.testing.assert_allclose(o.swiglu(2.0, 1.0), 2.0 / (1.0 + math.exp(-2.0)), rtol=1e-15)
    np.testing.assert_allclose(o.swiglu(-40.0, 1.0), -40.0 * math.exp(-40.0), rtol=1e-12)


def _fused_case(seed=7):
    rng = np.random.default_rng(seed)
    K = 64
    x = rng.standard_normal((5, K)).astype(np.float32)
    widths = [8, 4, 2, 2]
    scales = [0.02, 0.05, 0.01, 0.03]
    segs = [(s * rng.standard_normal((w, K))).astype(np.float32) for w, s in zip(widths, scales)]
    aq = o.quantize(x)
    wq = [o.quantize(s) for s in segs]
    return x, segs, aq, wq


def test_fused_projection_equals_per_module_linears():
    x, segs, aq, wq = _fused_case()
    a_log = np.array([0.1, -0.3]); dt = np.array([0.2, 0.4])
    epis = ["identity", "identity", "sigmoid", "gdn_decay"]
    outs, pre = o.fused_projection(aq, [(c, s) for c, s, _ in wq], [g for _, _, g in wq], epis, (a_log, dt))
    for s, w in enumerate(segs):
        y, _, _, _ = o.linear(x, w)
        np.testing.assert_array_equal(pre[s][0], y)
    np.testing.assert_array_equal(outs[2], o.sigmoid(pre[2][0]))
    np.testing.assert_array_equal(outs[3], o.gdn_decay(pre[3][0], a_log[None], dt[None]))


def test_common_scale_mismatch_closed_form():
    """One common global scale without rescaling the block scales multiplies
    segment s by g_c / g_s ("Main Findings", fused-GEMM scaling bullet)."""
    x, segs, aq, wq = _fused_case(8)
    g_s = [g for _, _, g in wq]
    g_c = o.common_global_scale(g_s)
    assert g_c == min(g_s)
    epis = ["identity"] * 4
    w_only = [(c, s) for c, s, _ in wq]
    good, pre_good = o.fused_projection(aq, w_only, g_s, epis)
    bad, pre_bad = o.fused_projection(aq, w_only, [g_c] * 4, epis)
    for s in range(4):
        ratio = float(g_c) / float(g_s[s])
        np.testing.assert_allclose(bad[s], good[s] * ratio, rtol=1e-15, atol=0)
    assert any(float(g_c) / float(g) < 1 for g in g_s)


def test_swiglu_pairing_in_fused_projection():
    rng = np.random.default_rng(9)
    x = rng.standard_normal((3, 32)).astype(np.float32)
    gate = (0.02 * rng.standard_normal((4, 32))).astype(np.float32)
    up = (0.05 * rng.standard_normal((4, 32))).astype(np.float32)
    aq = o.quantize(x)
    gq, uq = o.quantize(gate), o.quantize(up)
    outs, pre = o.fused_projection(aq, [gq[:2], uq[:2]], [gq[2], uq[2]], ["swiglu_gate", "swiglu_up"])
    assert set(outs) == {0}
    yg, _, _, _ = o.linear(x, gate)
    yu, _, _, _ = o.linear(x, up)
    np.testing.assert_array_equal(outs[0], o.swiglu(yg, yu))


def test_bf16_round_and_ulp():
    import torch
    rng = np.random.default_rng(10)
    y = rng.standard_normal(100000) * np.exp(rng.uniform(-20, 20, 100000))
    ref = torch.from_numpy(y.astype(np.float32)).to(torch.bfloat16).double().numpy()
    got = o.bf16_round(y)
    # torch rounds via float32 first; they agree except where that double rounding bites
    assert np.mean(got == ref) > 0.999
    assert np.all(np.abs(got - y) <= 0.5 * o.bf16_ulp(y) * (1 + 1e-12))
    assert o.bf16_ulp(1.0) == 2.0 ** -7 and o.bf16_ulp(1.999) == 2.0 ** -7
