"""The seeded input generators shared by the tests, the benchmark and the
oracle follow their stated recipe (CPU only): shapes, BF16-representable
values, the outlier channels, determinism, the reduced-row prefix property the
sampled parity checks rely on, and the recurrence inputs' ranges."""
import numpy as np
import torch

from bit_quantized_linear_nvfp4_b200 import workloads as wl


def test_bf16_rounding_matches_torch_and_is_idempotent():
    rng = np.random.default_rng(0)
    x = (rng.standard_normal(100000) * np.exp(rng.uniform(-20, 20, 100000))).astype(np.float32)
    r = wl.round_to_bf16(x)
    t = torch.from_numpy(x).to(torch.bfloat16).to(torch.float32).numpy()
    assert np.array_equal(r, t)
    assert np.array_equal(wl.round_to_bf16(r), r)


def test_activation_recipe():
    w = wl.OPROJ
    x = wl.make_x(w, rows=512)
    assert x.shape == (512, w.K) and x.dtype == np.float32
    assert np.array_equal(wl.round_to_bf16(x), x)
    rms = np.sqrt((x.astype(np.float64) ** 2).mean(axis=0))
    hot = np.argsort(rms)[-w.n_outlier:]
    assert np.all(rms[hot] > 30) and np.median(rms) < 1.2  # n_outlier channels x100, the rest N(0, 1)
    assert np.count_nonzero(rms > 10) == w.n_outlier
    assert np.array_equal(wl.make_x(w, rows=512), x)  # deterministic


def test_reduced_rows_are_a_prefix_of_the_full_draw():
    w = wl.MLP
    full = wl.make_x(w)
    assert np.array_equal(wl.make_x(w, rows=300), full[:300])


def test_tiny_fixed_outliers_and_fp32():
    x = wl.make_x(wl.TINY)
    assert x.shape == (64, 512)
    rms = np.sqrt((x.astype(np.float64) ** 2).mean(axis=0))
    assert set(np.nonzero(rms > 10)[0]) == {7, 300}


def test_weight_and_gate_recipe():
    w = wl.GDN
    segs = wl.make_w_segments(w)
    assert [s.shape[0] for s in segs] == [sg.width for sg in w.segments]
    for s in segs:
        assert s.shape[1] == w.K and np.array_equal(wl.round_to_bf16(s), s)
        assert abs(float(s.std()) - 0.02) < 0.002
    # each segment has its own generator: no two segments share a draw
    assert not np.array_equal(segs[0][:32], segs[1][:32])
    a_log, dt_bias = wl.make_gate_params(w)
    assert a_log.shape == (w.heads,) and np.all(np.abs(a_log) <= 1.0)
    assert dt_bias.shape == (w.heads,) and 0.2 < float(dt_bias.std()) < 0.9


def test_sample_rows():
    rows = wl.sample_rows(32768, 512)
    assert rows.size == 512 and rows[0] == 0 and rows[-1] == 32767
    assert np.all(np.diff(rows) > 0)
    assert np.array_equal(wl.sample_rows(32768, 512), rows)
    assert np.array_equal(wl.sample_rows(10, 512), np.arange(10))


def test_recurrence_inputs():
    q, k, v, beta, g = wl.make_recurrence_inputs(300, 4, 2, 7, "bf16")
    assert q.shape == (300, 2 * wl.GDN_DK) and k.shape == q.shape and v.shape == (300, 4 * wl.GDN_DV)
    assert beta.shape == (300, 4) and g.shape == (300, 4)
    for a in (q, k, v):
        assert np.array_equal(wl.round_to_bf16(a), a)
    assert np.all((beta >= 0) & (beta <= 1)) and np.all(g < 0)
    _, _, _, _, g_slow = wl.make_recurrence_inputs(300, 4, 2, 7, "bf16", slow=True)
    assert np.median(-g_slow) < np.median(-g)
