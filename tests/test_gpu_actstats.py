"""GPU parity of nvfp4_activation_stats with the oracle's activation_stats:
counts and maxima exact, FP64 moments and FP32 row/column sums within the
bounds of their summation order, accumulation over batches, and the derived
summary."""
import numpy as np
import pytest
import torch

from bit_quantized_linear_nvfp4_b200 import nvfp4 as nv
from bit_quantized_linear_nvfp4_b200 import workloads as wl
from oracle import nvfp4_oracle as o

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


def _x(M, K, seed, dtype="bf16", hot=8):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((M, K)).astype(np.float32)
    x[:, rng.choice(K, size=hot, replace=False)] *= 100
    x[:, :16] = 0.0
    x[0, 5] = 7.0  # a dominated block
    return wl.round_to_bf16(x) if dtype == "bf16" else x


def _dev(x, dtype):
    t = torch.from_numpy(np.ascontiguousarray(x)).to(DEV)
    return t.to(torch.bfloat16) if dtype == "bf16" else t


def _compare(st, ref, x, rel_sum=1e-4):
    m = st["moments"].cpu().numpy()
    a = np.abs(x.astype(np.float64))
    assert m[5] == ref["n"] and m[6] == ref["blocks"] and m[7] == ref["dominated"]
    assert m[4] == ref["amax"]
    assert abs(m[0] - ref["sum"]) <= 1e-6 * a.sum()
    assert abs(m[1] - ref["sum_sq"]) <= 1e-6 * ref["sum_sq"]
    assert abs(m[2] - ref["sum_cube"]) <= 1e-6 * (a ** 3).sum()
    assert abs(m[3] - ref["sum_4th"]) <= 1e-6 * ref["sum_4th"]
    np.testing.assert_allclose(st["row_norm2"].double().cpu().numpy(), ref["row_norm2"], rtol=rel_sum, atol=1e-30)
    np.testing.assert_allclose(st["row_err2"].double().cpu().numpy(), ref["row_err2"], rtol=rel_sum,
                               atol=1e-6 * ref["row_err2"].max())
    np.testing.assert_allclose(st["col_sq"].double().cpu().numpy(), ref["col_sq"], rtol=rel_sum, atol=1e-30)
    assert np.array_equal(st["col_max"].double().cpu().numpy(), ref["col_max"])


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("M,K", [(1, 16), (300, 1040), (257, 5120), (64, 17408)])
def test_stats_match_oracle(dtype, M, K):
    x = _x(M, K, M + K, dtype)
    xd = _dev(x, dtype)
    A, g = nv.nvfp4_quantize(xd)
    st = nv.nvfp4_activation_stats(xd, g)
    torch.cuda.synchronize()
    ref = o.activation_stats(x, np.float32(g.item()))
    _compare(st, ref, x)
    s_gpu = nv.activation_summary(st)
    s_ref = o.activation_summary(ref)
    for k in ("max_over_rms", "kurtosis", "dominated_share", "a4_err_mean", "a4_err_max", "hot_channel_ratio"):
        assert abs(s_gpu[k] - s_ref[k]) <= 1e-4 * max(1.0, abs(s_ref[k])), k


def _host_stats(st):
    """The device accumulators as the oracle's statistics dict, every value
    converted exactly to FP64."""
    m = st["moments"].cpu().numpy()
    return {"sum": m[0], "sum_sq": m[1], "sum_cube": m[2], "sum_4th": m[3], "amax": m[4], "n": m[5],
            "blocks": m[6], "dominated": m[7],
            "row_err2": st["row_err2"].double().cpu().numpy(), "row_norm2": st["row_norm2"].double().cpu().numpy(),
            "col_sq": st["col_sq"].double().cpu().numpy()}


@pytest.mark.parametrize("M,K", [(1, 16), (7, 48), (300, 1040), (257, 5120), (2048, 5120), (64, 17408)])
def test_device_summary_matches_oracle_summary(M, K):
    """nvfp4_activation_summary against oracle.activation_summary on the same
    accumulators: every figure is the same FP64 expression, so they agree to
    a few ulp (the A4 mean sums M terms in a different order: M ulp)."""
    x = _x(M, K, 3 * M + K, "bf16")
    xd = _dev(x, "bf16")
    A, g = nv.nvfp4_quantize(xd)
    st = nv.nvfp4_activation_stats(xd, g)
    dev = nv.nvfp4_activation_summary(st).cpu().numpy()
    ref = o.activation_summary(_host_stats(st))
    for i, k in enumerate(nv.SUMMARY_FIELDS[:7]):
        tol = (4 * M if k == "a4_err_mean" else 8) * np.finfo(np.float64).eps * max(abs(ref[k]), 1e-300)
        assert abs(dev[i] - ref[k]) <= tol, (k, dev[i], ref[k])
    col_rms = np.sqrt(_host_stats(st)["col_sq"] * (1.0 / M))
    assert abs(dev[7] - np.median(col_rms)) <= 8 * np.finfo(np.float64).eps * np.median(col_rms)


def test_device_summary_even_and_odd_channel_counts():
    """The median is the middle channel for an odd count and the mean of the
    two middle ones for an even count; ties and zero channels included."""
    for K in (15, 16, 33, 48):
        rng = np.random.default_rng(K)
        col = rng.integers(0, 5, size=K).astype(np.float32) * 0.5
        st = {"moments": torch.tensor([0, 4, 0, 16, 2, 4, 1, 0], dtype=torch.float64, device=DEV),
              "row_err2": None, "row_norm2": torch.ones(4, device=DEV),
              "col_sq": torch.from_numpy(col).to(DEV)}
        out = nv.nvfp4_activation_summary(st).cpu().numpy()
        rms = np.sqrt(col.astype(np.float64) * 0.25)
        med = np.median(rms)
        assert out[7] == med, (K, out[7], med)
        assert out[6] == (rms.max() / med if med > 0 else 0.0)
        assert np.isnan(out[3]) and np.isnan(out[4]) and np.isnan(out[5])
        assert out[2] == 0.0 and out[0] == 2.0 / 1.0  # amax 2 over sqrt(4 / 4)


def test_accumulates_over_batches_and_strided_rows():
    x = _x(400, 2048, 3)
    big = torch.zeros((400, 2304), dtype=torch.bfloat16, device=DEV)
    big[:, :2048] = _dev(x, "bf16")
    view = big[:, :2048]
    _, g = nv.nvfp4_quantize(view)
    st = nv.nvfp4_activation_stats(view[:150], g)
    # the second batch adds into the same column and moment accumulators
    rest = {"moments": st["moments"], "row_err2": torch.zeros(250, device=DEV), "row_norm2": torch.zeros(250, device=DEV),
            "col_sq": st["col_sq"], "col_max": st["col_max"]}
    nv.nvfp4_activation_stats(view[150:], g, into=rest)
    torch.cuda.synchronize()
    ref = o.activation_stats(x, np.float32(g.item()))
    merged = dict(st)
    merged["row_err2"] = torch.cat([st["row_err2"][:150], rest["row_err2"]])
    merged["row_norm2"] = torch.cat([st["row_norm2"][:150], rest["row_norm2"]])
    _compare(merged, ref, x)


def test_without_global_scale_skips_the_a4_error():
    x = _x(64, 512, 9)
    st = nv.nvfp4_activation_stats(_dev(x, "bf16"))
    torch.cuda.synchronize()
    assert st["row_err2"] is None
    ref = o.activation_stats(x)
    assert st["moments"][7].item() == ref["dominated"]
