"""GPU parity of nvfp4_gemm / nvfp4_fused_proj with the oracle (FP64 GEMM on
the dequantised operands, FP64 epilogues)."""
import numpy as np
import pytest
import torch

from bit_quantized_linear_nvfp4_b200 import nvfp4 as nv
from bit_quantized_linear_nvfp4_b200 import workloads as wl
from oracle import nvfp4_oracle as o
from tests.gpu_helpers import (TOL_ACC, assert_quant_equal, check_bf16, check_fp32, f32_ulp,
                               to_np)

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


def _dev(x, dtype="bf16"):
    t = torch.from_numpy(np.ascontiguousarray(x)).to(DEV)
    return t.to(torch.bfloat16) if dtype == "bf16" else t


def _rand(M, K, seed, scale=1.0, outliers=0, dtype="bf16"):
    rng = np.random.default_rng(seed)
    x = (scale * rng.standard_normal((M, K))).astype(np.float32)
    if outliers:
        x[:, rng.choice(K, size=outliers, replace=False)] *= 50
    return wl.round_to_bf16(x) if dtype == "bf16" else x


def test_tiny_workload_fp32():
    """X[64,512] x W[256,512] FP32 in, FP32 out, every element."""
    w = wl.TINY
    x, wt = wl.make_x(w), wl.make_w_segment(w, 0)
    A, ga = nv.nvfp4_quantize(_dev(x, "f32"))
    W, gw = nv.nvfp4_quantize(_dev(wt, "f32"))
    out = nv.nvfp4_gemm(A, ga, W, gw, out_dtype=torch.float32)
    torch.cuda.synchronize()
    assert_quant_equal(A, ga, x)
    assert_quant_equal(W, gw, wt)
    y, mag, _, _ = o.linear(x, wt)
    check_fp32(to_np(out), y, mag, "tiny")


@pytest.mark.parametrize("M,N,K", [(1, 256, 256), (100, 64, 512), (129, 200, 256), (300, 520, 1024),
                                   (64, 384, 288), (257, 256, 5120)])
@pytest.mark.parametrize("out_dtype", [torch.float32, torch.bfloat16])
def test_ragged_gemm(M, N, K, out_dtype):
    x = _rand(M, K, M + N + K, outliers=2)
    wt = _rand(N, K, 7 * N + K, scale=0.02)
    A, ga = nv.nvfp4_quantize(_dev(x))
    W, gw = nv.nvfp4_quantize(_dev(wt))
    out = nv.nvfp4_gemm(A, ga, W, gw, out_dtype=out_dtype)
    torch.cuda.synchronize()
    y, mag, _, _ = o.linear(x, wt)
    if out_dtype == torch.float32:
        check_fp32(to_np(out), y, mag, f"{M}x{N}x{K}")
    else:
        check_bf16(to_np(out), y, TOL_ACC * mag, f"{M}x{N}x{K}")


def test_output_leading_dimension():
    M, N, K = 70, 256, 256
    x, wt = _rand(M, K, 1), _rand(N, K, 2, 0.02)
    A, ga = nv.nvfp4_quantize(_dev(x))
    W, gw = nv.nvfp4_quantize(_dev(wt))
    big = torch.full((M, N + 64), -7.0, dtype=torch.bfloat16, device=DEV)
    nv.nvfp4_gemm(A, ga, W, gw, out=big[:, 32:32 + N])
    torch.cuda.synchronize()
    y, mag, _, _ = o.linear(x, wt)
    check_bf16(to_np(big[:, 32:32 + N]), y, TOL_ACC * mag)
    assert torch.all(big[:, :32] == -7) and torch.all(big[:, 32 + N:] == -7)


def _gdn_case(M, seed=3, b_a_scale=1.0):
    """GDN in-projection segments with their own global scales (reduced M)."""
    w = wl.GDN
    rng = np.random.default_rng(seed)
    K = w.K
    x = _rand(M, K, seed, outliers=26)
    segs = [wl.make_w_segment(w, s) for s in range(len(w.segments))]
    if b_a_scale != 1.0:
        segs[4] = wl.round_to_bf16(segs[4] * np.float32(b_a_scale))
        segs[5] = wl.round_to_bf16(segs[5] * np.float32(b_a_scale))
    a_log, dt_bias = wl.make_gate_params(w)
    return w, x, segs, a_log, dt_bias


def _run_fused(w, x, segs, a_log, dt_bias, common=False):
    bounds = np.concatenate([[0], np.cumsum([s.width for s in w.segments])])
    wcat = np.concatenate(segs)
    A, ga = nv.nvfp4_quantize(_dev(x))
    W, gw = nv.nvfp4_quantize_segments(_dev(wcat), bounds)
    scales = gw
    if common:
        scales = torch.full_like(gw, float(gw.min().item()))
    M = x.shape[0]
    outs = []
    nsegs = []
    for s, seg in enumerate(w.segments):
        kind = {"identity": "identity_bf16", "sigmoid": "sigmoid", "gdn_decay": "gdn_decay"}[seg.epilogue]
        dt = torch.bfloat16 if kind == "identity_bf16" else torch.float32
        out = torch.empty((M, seg.width), dtype=dt, device=DEV)
        outs.append(out)
        extra = {}
        if kind == "gdn_decay":
            extra = dict(A_log=torch.from_numpy(a_log).to(DEV), dt_bias=torch.from_numpy(dt_bias).to(DEV))
        nsegs.append(nv.Segment(int(bounds[s]), int(bounds[s + 1]), kind, out, **extra))
    nv.nvfp4_fused_proj(A, ga, W, scales, nsegs)
    torch.cuda.synchronize()
    return outs, gw.cpu().numpy(), float(ga.item())


def _oracle_fused(x, segs, g_scales, a_log, dt_bias, w):
    aq = o.quantize(x)
    wq = [o.quantize(s) for s in segs]
    epis = [s.epilogue for s in w.segments]
    outs, pre = o.fused_projection(aq, [(c, s) for c, s, _ in wq], g_scales, epis, (a_log, dt_bias))
    return outs, pre, [g for _, _, g in wq]


def _check_gdn(outs, o_outs, pre, a_log, dt_bias, w):
    for s, seg in enumerate(w.segments):
        gpu = to_np(outs[s])
        y, mag = pre[s]
        tol = TOL_ACC * mag
        if seg.epilogue == "identity":
            check_bf16(gpu, o_outs[s], tol, seg.name)
        elif seg.epilogue == "sigmoid":
            bound = tol / 4 + 4 * f32_ulp(o_outs[s])
            assert np.all(np.abs(gpu - o_outs[s]) <= bound), seg.name
        else:
            t = y + dt_bias[None, :]
            deriv = np.exp(a_log)[None, :] * o.sigmoid(t)
            bound = deriv * (tol + f32_ulp(t)) + 8 * f32_ulp(o_outs[s])
            assert np.all(np.abs(gpu - o_outs[s]) <= bound), seg.name


def test_gdn_fused_projection_reduced_rows():
    w, x, segs, a_log, dt_bias = _gdn_case(300)
    outs, g_gpu, _ = _run_fused(w, x, segs, a_log, dt_bias)
    wq_g = [o.quantize(s)[2] for s in segs]
    np.testing.assert_array_equal(g_gpu, np.array(wq_g, np.float32))
    o_outs, pre, _ = _oracle_fused(x, segs, wq_g, a_log, dt_bias, w)
    _check_gdn(outs, o_outs, pre, a_log, dt_bias, w)


def test_gdn_common_scale_mismatch():
    """One common global scale (the fused serving bug): segment s comes out
    multiplied by g_c / g_s; with the per-segment table it does not."""
    w, x, segs, a_log, dt_bias = _gdn_case(130, seed=11, b_a_scale=2.75)
    good, g_gpu, _ = _run_fused(w, x, segs, a_log, dt_bias)
    bad, _, _ = _run_fused(w, x, segs, a_log, dt_bias, common=True)
    g_c = float(np.min(g_gpu))
    # identity segments: exact ratio up to BF16 rounding of both sides
    for s in range(4):
        ratio = g_c / float(g_gpu[s])
        gd, bd = to_np(good[s]), to_np(bad[s])
        assert np.allclose(bd, gd * ratio, rtol=2 ** -7, atol=1e-6), s
    # oracle with the common scale predicts the corrupted gates
    o_bad, pre_bad, _ = _oracle_fused(x, segs, [g_c] * 6, a_log, dt_bias, w)
    _check_gdn(bad, o_bad, pre_bad, a_log, dt_bias, w)
    assert g_gpu[4] > g_c * 2  # the b/a modules were the mismatched ones


def test_swiglu_reduced():
    M, K, H = 200, 512, 384
    x = _rand(M, K, 21, outliers=3)
    gate = _rand(H, K, 22, 0.02)
    up = _rand(H, K, 23, 0.05)
    A, ga = nv.nvfp4_quantize(_dev(x))
    W, gw = nv.nvfp4_quantize_segments(_dev(np.concatenate([gate, up])), [0, H, 2 * H])
    out = torch.empty((M, H), dtype=torch.bfloat16, device=DEV)
    nv.nvfp4_fused_proj(A, ga, W, gw, [nv.Segment(0, H, "swiglu_gate", out), nv.Segment(H, 2 * H, "swiglu_up")])
    torch.cuda.synchronize()
    aq = o.quantize(x)
    gq, uq = o.quantize(gate), o.quantize(up)
    outs, pre = o.fused_projection(aq, [gq[:2], uq[:2]], [gq[2], uq[2]], ["swiglu_gate", "swiglu_up"])
    yg, mg = pre[0]
    yu, mu = pre[1]
    sg = o.sigmoid(yg)
    dsilu = sg * (1 + yg * (1 - sg))
    tol = np.abs(dsilu * yu) * TOL_ACC * mg + np.abs(yg * sg) * TOL_ACC * mu + 8 * f32_ulp(outs[0])
    check_bf16(to_np(out), outs[0], tol, "swiglu")


@pytest.mark.slow
def test_full_size_oproj_sampled_rows():
    """Prefill o_proj 4096x5120x5120 at full size; 256 sampled rows x all columns."""
    w = wl.OPROJ
    x = wl.make_x(w)
    wt = wl.make_w_segment(w, 0)
    A, ga = nv.nvfp4_quantize(_dev(x))
    W, gw = nv.nvfp4_quantize(_dev(wt))
    out = nv.nvfp4_gemm(A, ga, W, gw)
    torch.cuda.synchronize()
    rows = wl.sample_rows(w.M, 256)
    g_a = o.global_scale(x)
    assert np.float32(ga.item()) == g_a
    aq = o.quantize(x[rows], g_a)
    wq = o.quantize(wt)
    acc, mag = o.gemm(aq[0], aq[1], wq[0], wq[1])
    s = float(g_a) * float(wq[2])
    check_bf16(to_np(out[torch.from_numpy(rows).to(DEV)]), acc * s, TOL_ACC * mag * s, "oproj")


def _check_gdn_sampled(x, segs, a_log, dt_bias, rows, outs_rows, g_gpu, ga_gpu, w):
    """Oracle of the sampled rows of a full-size fused GDN projection, and the
    comparison (outs_rows: the GPU outputs of those rows, per segment)."""
    g_a = o.global_scale(x)
    assert np.float32(ga_gpu) == g_a
    wq = [o.quantize(sg) for sg in segs]
    np.testing.assert_array_equal(g_gpu, np.array([g for _, _, g in wq], np.float32))
    aq = o.quantize(x[rows], g_a)
    o_outs, pre = o.fused_projection(aq, [(c, sf) for c, sf, _ in wq], [g for _, _, g in wq],
                                     [sg.epilogue for sg in w.segments], (a_log, dt_bias))
    _check_gdn(outs_rows, o_outs, pre, a_log, dt_bias, w)


@pytest.mark.slow
def test_full_size_gdn_sampled_rows():
    """The fused GDN in-projection at full size, 32768x12352x5120 (activations
    larger than L2: the grouped rasterisation) in the launch configuration the
    benchmark times; 512 sampled rows (rows 0 and M-1 included) x all columns."""
    w = wl.GDN
    x = wl.make_x(w)
    segs = wl.make_w_segments(w)
    a_log, dt_bias = wl.make_gate_params(w)
    outs, g_gpu, ga = _run_fused(w, x, segs, a_log, dt_bias)
    rows = wl.sample_rows(w.M, 512)
    rows_t = torch.from_numpy(rows).to(DEV)
    _check_gdn_sampled(x, segs, a_log, dt_bias, rows, [t[rows_t] for t in outs], g_gpu, ga, w)


def _check_swiglu_sampled(x, gate, up, rows, out_rows, gw_gpu, ga_gpu, label):
    """Oracle of sampled rows of a fused gate+up projection with SwiGLU, and
    the comparison with the tolerance propagated through silu(g) * u."""
    g_a = o.global_scale(x)
    assert np.float32(ga_gpu) == g_a
    gq, uq = o.quantize(gate), o.quantize(up)
    np.testing.assert_array_equal(gw_gpu, np.array([gq[2], uq[2]], np.float32))
    aq = o.quantize(x[rows], g_a)
    outs, pre = o.fused_projection(aq, [gq[:2], uq[:2]], [gq[2], uq[2]], ["swiglu_gate", "swiglu_up"])
    yg, mg = pre[0]
    yu, mu = pre[1]
    sg = o.sigmoid(yg)
    dsilu = sg * (1 + yg * (1 - sg))
    tol = np.abs(dsilu * yu) * TOL_ACC * mg + np.abs(yg * sg) * TOL_ACC * mu + 8 * f32_ulp(outs[0])
    check_bf16(out_rows, outs[0], tol, label)


@pytest.mark.slow
def test_full_size_mlp_sampled_rows():
    """The fused MLP gate+up with SwiGLU at full size, 8192x34816x5120, in the
    launch configuration the benchmark times; 256 sampled rows x all columns."""
    w = wl.MLP
    x = wl.make_x(w)
    gate, up = wl.make_w_segments(w)
    H = gate.shape[0]
    A, ga = nv.nvfp4_quantize(_dev(x))
    W, gw = nv.nvfp4_quantize_segments(_dev(np.concatenate([gate, up])), [0, H, 2 * H])
    out = torch.empty((w.M, H), dtype=torch.bfloat16, device=DEV)
    nv.nvfp4_fused_proj(A, ga, W, gw, [nv.Segment(0, H, "swiglu_gate", out), nv.Segment(H, 2 * H, "swiglu_up")])
    torch.cuda.synchronize()
    rows = wl.sample_rows(w.M, 256)
    out_rows = to_np(out[torch.from_numpy(rows).to(DEV)])
    del out, W, A
    _check_swiglu_sampled(x, gate, up, rows, out_rows, gw.cpu().numpy(), float(ga.item()), "mlp full size")


# ---------------------------------------------------------------- decode path (M <= 64)

@pytest.mark.parametrize("M", [1, 5, 8, 64])
@pytest.mark.parametrize("N,K", [(640, 2048), (200, 256), (128, 5376)])
def test_decode_path(M, N, K):
    """Few tokens: swap-AB, split-K over a cluster, DSMEM reduction."""
    x = _rand(M, K, 3 * M + N, outliers=2)
    wt = _rand(N, K, 5 * N + K, scale=0.02)
    A, ga = nv.nvfp4_quantize(_dev(x))
    W, gw = nv.nvfp4_quantize(_dev(wt))
    out32 = nv.nvfp4_gemm(A, ga, W, gw, out_dtype=torch.float32)
    out16 = nv.nvfp4_gemm(A, ga, W, gw, out_dtype=torch.bfloat16)
    torch.cuda.synchronize()
    y, mag, _, _ = o.linear(x, wt)
    check_fp32(to_np(out32), y, mag, f"decode f32 {M}x{N}x{K}")
    check_bf16(to_np(out16), y, TOL_ACC * mag, f"decode bf16 {M}x{N}x{K}")


@pytest.mark.parametrize("M", [1, 8, 64])
def test_decode_path_gdn_segments(M):
    """GDN-style segments (identity, write strength, decay) through the decode epilogue."""
    w = wl.GDN
    rng = np.random.default_rng(31 + M)
    K = 1024
    x = _rand(M, K, 40 + M, outliers=3)
    widths = [256, 32, 32]
    segs = [wl.round_to_bf16((0.02 * (i + 1) * rng.standard_normal((n, K))).astype(np.float32)) for i, n in enumerate(widths)]
    a_log, dt_bias = wl.make_gate_params(w)
    bounds = [0, 256, 288, 320]
    A, ga = nv.nvfp4_quantize(_dev(x))
    W, gw = nv.nvfp4_quantize_segments(_dev(np.concatenate(segs)), bounds)
    q = torch.empty((M, 256), dtype=torch.bfloat16, device=DEV)
    beta = torch.empty((M, 32), dtype=torch.float32, device=DEV)
    dec = torch.empty((M, 32), dtype=torch.float32, device=DEV)
    nv.nvfp4_fused_proj(A, ga, W, gw, [
        nv.Segment(0, 256, "identity_bf16", q), nv.Segment(256, 288, "sigmoid", beta),
        nv.Segment(288, 320, "gdn_decay", dec, A_log=torch.from_numpy(a_log).to(DEV),
                   dt_bias=torch.from_numpy(dt_bias).to(DEV))])
    torch.cuda.synchronize()
    aq = o.quantize(x)
    wq = [o.quantize(s) for s in segs]
    outs, pre = o.fused_projection(aq, [(c, s) for c, s, _ in wq], [g for _, _, g in wq],
                                   ["identity", "sigmoid", "gdn_decay"], (a_log, dt_bias))
    check_bf16(to_np(q), outs[0], TOL_ACC * pre[0][1], "q")
    assert np.all(np.abs(to_np(beta) - outs[1]) <= TOL_ACC * pre[1][1] / 4 + 4 * f32_ulp(outs[1]))
    t = pre[2][0] + dt_bias[None, :]
    bound = np.exp(a_log)[None, :] * o.sigmoid(t) * (TOL_ACC * pre[2][1] + f32_ulp(t)) + 8 * f32_ulp(outs[2])
    assert np.all(np.abs(to_np(dec) - outs[2]) <= bound)


@pytest.mark.slow
@pytest.mark.parametrize("M", [1, 8, 64])
def test_full_size_decode(M):
    """Decode down_proj W[5120,17408], every output element."""
    w = wl.decode_workload(M)
    x = wl.make_x(w)
    wt = wl.make_w_segment(w, 0)
    A, ga = nv.nvfp4_quantize(_dev(x))
    W, gw = nv.nvfp4_quantize(_dev(wt))
    out = nv.nvfp4_gemm(A, ga, W, gw)
    torch.cuda.synchronize()
    y, mag, _, _ = o.linear(x, wt)
    check_bf16(to_np(out), y, TOL_ACC * mag, f"decode M={M}")


@pytest.mark.parametrize("M", [8, 64])
def test_full_size_decode_fp32_accumulation(M):
    """Decode down_proj W[5120,17408] with FP32 output, every element: the
    accumulation over K = 17408 against the 1e-5 * sum|a w| bound (the ratio is
    printed; on B200 it measured 4e-4 of the bound)."""
    w = wl.decode_workload(M)
    x = wl.make_x(w)
    wt = wl.make_w_segment(w, 0)
    A, ga = nv.nvfp4_quantize(_dev(x))
    W, gw = nv.nvfp4_quantize(_dev(wt))
    out = nv.nvfp4_gemm(A, ga, W, gw, out_dtype=torch.float32)
    torch.cuda.synchronize()
    y, mag, _, _ = o.linear(x, wt)
    ratio = check_fp32(to_np(out), y, mag, f"decode M={M} fp32")
    print(f"decode M={M} K=17408 FP32: max error / bound = {ratio:.2e}")


def test_wide_tiles_two_segments():
    """A shape that runs the 256-wide overlapped-accumulator kernel for a
    non-SwiGLU projection (one M block, N just above 74 x 192), with a BF16
    and an FP32 segment."""
    M, K, N = 200, 256, 14336
    x = _rand(M, K, 61, outliers=2)
    w0 = _rand(8192, K, 62, 0.02)
    w1 = _rand(N - 8192, K, 63, 0.05)
    A, ga = nv.nvfp4_quantize(_dev(x))
    W, gw = nv.nvfp4_quantize_segments(_dev(np.concatenate([w0, w1])), [0, 8192, N])
    o0 = torch.empty((M, 8192), dtype=torch.bfloat16, device=DEV)
    o1 = torch.empty((M, N - 8192), dtype=torch.float32, device=DEV)
    nv.nvfp4_fused_proj(A, ga, W, gw, [nv.Segment(0, 8192, "identity_bf16", o0), nv.Segment(8192, N, "identity_f32", o1)])
    torch.cuda.synchronize()
    y0, m0, _, _ = o.linear(x, w0)
    y1, m1, _, _ = o.linear(x, w1)
    check_bf16(to_np(o0), y0, TOL_ACC * m0, "wide bf16")
    check_fp32(to_np(o1), y1, m1, "wide f32")


def test_wide_tiles_ragged_segments():
    """The 256-wide kernel (one M block, N above 74 x 192) with BF16 segments
    whose boundaries are off the 8-column grid, one narrower than 64 columns
    and an FP32 one: 64-column groups that cross a boundary or start off the
    grid take the per-lane stores, the rest the staged TMA stores; padded
    output strides; 200 rows, so the last 16-row store box is clipped."""
    M, K = 200, 256
    widths = [100, 8000, 36, 6200]
    kinds = ["identity_bf16", "identity_bf16", "identity_bf16", "identity_f32"]
    N = sum(widths)
    x = _rand(M, K, 71, outliers=2)
    ws = [_rand(w, K, 72 + i, 0.02 * (i + 1)) for i, w in enumerate(widths)]
    bounds = np.concatenate([[0], np.cumsum(widths)])
    A, ga = nv.nvfp4_quantize(_dev(x))
    W, gw = nv.nvfp4_quantize_segments(_dev(np.concatenate(ws)), bounds)
    outs, segs = [], []
    for i, (w, kind) in enumerate(zip(widths, kinds)):
        dt = torch.bfloat16 if kind == "identity_bf16" else torch.float32
        unit = 8 if dt == torch.bfloat16 else 4  # row strides of 16 bytes
        full = torch.full((M, (w // unit + 1) * unit), -7.0, dtype=dt, device=DEV)
        outs.append(full)
        segs.append(nv.Segment(int(bounds[i]), int(bounds[i + 1]), kind, full[:, :w]))
    nv.nvfp4_fused_proj(A, ga, W, gw, segs)
    torch.cuda.synchronize()
    for i, w in enumerate(widths):
        y, mag, _, _ = o.linear(x, ws[i])
        got = to_np(outs[i])
        assert np.all(got[:, w:] == -7.0), f"segment {i} wrote past its width"
        if kinds[i] == "identity_bf16":
            check_bf16(got[:, :w], y, TOL_ACC * mag, f"segment {i}")
        else:
            check_fp32(got[:, :w], y, mag, f"segment {i}")
