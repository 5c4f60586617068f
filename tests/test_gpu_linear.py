"""GPU parity of nvfp4_linear (quantise the activation, then the fused
projection, in one call) with the oracle, and with the two separate calls.

nvfp4_linear launches the quantiser and the GEMM back to back with
programmatic dependent launch, and the weight-streaming GEMM reads W before
the quantiser has finished.  Besides parity, the tests chain layers so that a
quantiser reads the previous GEMM's output and rewrites buffers the previous
GEMM read, to check that every kernel waits where it must."""
import numpy as np
import pytest
import torch

from bit_quantized_linear_nvfp4_b200 import nvfp4 as nv
from bit_quantized_linear_nvfp4_b200 import workloads as wl
from oracle import nvfp4_oracle as o
from tests.gpu_helpers import TOL_ACC, assert_quant_equal, check_bf16, check_fp32, to_np

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


def _rand(M, K, seed, scale=1.0, outliers=0):
    rng = np.random.default_rng(seed)
    x = (scale * rng.standard_normal((M, K))).astype(np.float32)
    if outliers:
        x[:, rng.choice(K, size=outliers, replace=False)] *= 50
    return wl.round_to_bf16(x)


def _bf16(x):
    return torch.from_numpy(np.ascontiguousarray(x)).to(DEV).to(torch.bfloat16)


@pytest.mark.parametrize("M,N,K", [(1, 640, 2048), (5, 200, 256), (64, 384, 4096), (300, 520, 1024)])
@pytest.mark.parametrize("static", [False, True])
def test_linear_matches_oracle_and_separate_calls(M, N, K, static):
    x = _rand(M, K, 11 * M + K, outliers=2)
    wt = _rand(N, K, 13 * N + K, scale=0.02)
    xd = _bf16(x)
    W, gw = nv.nvfp4_quantize(_bf16(wt))
    g_in, gs = None, None
    if static:
        gs = o.global_scale(x)
        g_in = torch.tensor([gs], dtype=torch.float32, device=DEV)
    out = torch.empty((M, N), dtype=torch.bfloat16, device=DEV)
    A, ga = nv.nvfp4_linear(xd, W, gw, [nv.Segment(0, N, "identity_bf16", out)], g_in=g_in)
    A2, ga2 = nv.nvfp4_quantize(xd, g_in)
    out2 = nv.nvfp4_gemm(A2, ga2, W, gw)
    torch.cuda.synchronize()
    assert_quant_equal(A, ga, x, g_in=gs)
    assert torch.equal(A.codes, A2.codes) and torch.equal(A.sf, A2.sf) and torch.equal(ga, ga2)
    assert torch.equal(out, out2)
    y, mag, _, _ = o.linear(x, wt)
    check_bf16(to_np(out), y, TOL_ACC * mag, f"linear {M}x{N}x{K}")


@pytest.mark.parametrize("M", [1, 8])
def test_linear_gate_segments_decode(M):
    """Write-strength and decay segments through the linear entry point."""
    w = wl.GDN
    K = 1024
    rng = np.random.default_rng(90 + M)
    x = _rand(M, K, 91 + M, outliers=3)
    widths = [256, 32, 32]
    segs = [wl.round_to_bf16((0.02 * (i + 1) * rng.standard_normal((n, K))).astype(np.float32))
            for i, n in enumerate(widths)]
    a_log, dt_bias = wl.make_gate_params(w)
    W, gw = nv.nvfp4_quantize_segments(_bf16(np.concatenate(segs)), [0, 256, 288, 320])
    params = dict(A_log=torch.from_numpy(a_log).to(DEV), dt_bias=torch.from_numpy(dt_bias).to(DEV))

    def outs():
        return (torch.empty((M, 256), dtype=torch.bfloat16, device=DEV),
                torch.empty((M, 32), dtype=torch.float32, device=DEV),
                torch.empty((M, 32), dtype=torch.float32, device=DEV))

    def segments(q, b, d):
        return [nv.Segment(0, 256, "identity_bf16", q), nv.Segment(256, 288, "sigmoid", b),
                nv.Segment(288, 320, "gdn_decay", d, **params)]

    r1, r2 = outs(), outs()
    nv.nvfp4_linear(_bf16(x), W, gw, segments(*r1))
    A, ga = nv.nvfp4_quantize(_bf16(x))
    nv.nvfp4_fused_proj(A, ga, W, gw, segments(*r2))
    torch.cuda.synchronize()
    for a, b in zip(r1, r2):
        assert torch.equal(a, b)


@pytest.mark.parametrize("M,width", [(1, 2048), (64, 1024), (200, 512)])
def test_chained_layers_share_buffers(M, width):
    """y_{i+1} = linear(y_i): each quantiser reads the GEMM output before it and
    overwrites the activation buffers that GEMM read; eager, then replayed as a
    CUDA graph, against the same chain with a synchronisation after every call."""
    depth = 4
    x = _rand(M, width, 5 + M)
    ws = [nv.nvfp4_quantize(_bf16(_rand(width, width, 100 + i, scale=1.0 / np.sqrt(width))))
          for i in range(depth)]
    a_codes = torch.empty((M, width // 2), dtype=torch.uint8, device=DEV)
    a_sf = torch.empty(nv.nvfp4_sf_bytes(M, width), dtype=torch.uint8, device=DEV)
    g_a = torch.empty(1, dtype=torch.float32, device=DEV)
    wsp = torch.empty(nv.nvfp4_quantize_workspace_bytes(1), dtype=torch.uint8, device=DEV)
    bufs = [_bf16(x)] + [torch.empty((M, width), dtype=torch.bfloat16, device=DEV) for _ in range(depth)]

    def chain(sync):
        for i, (W, gw) in enumerate(ws):
            nv.nvfp4_linear(bufs[i], W, gw, [nv.Segment(0, width, "identity_bf16", bufs[i + 1])],
                            a_codes=a_codes, a_sf=a_sf, g_a=g_a, workspace=wsp)
            if sync:
                torch.cuda.synchronize()

    chain(True)
    ref = [b.clone() for b in bufs]
    for b in bufs[1:]:
        b.fill_(0)
    chain(False)
    torch.cuda.synchronize()
    for i in range(1, depth + 1):
        assert torch.equal(bufs[i], ref[i]), f"eager layer {i}"
    for b in bufs[1:]:
        b.fill_(0)
    torch.cuda.synchronize()
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        chain(False)  # warm the launch path outside capture
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        chain(False)
    for b in bufs[1:]:
        b.fill_(0)
    graph.replay()
    graph.replay()
    torch.cuda.synchronize()
    for i in range(1, depth + 1):
        assert torch.equal(bufs[i], ref[i]), f"graph layer {i}"
    nv.nvfp4_check()


@pytest.mark.slow
@pytest.mark.parametrize("M", [1, 64])
def test_full_size_decode_linear(M):
    """Decode down_proj shape through nvfp4_linear: same bytes as the separate
    calls, which the decode parity tests compare with the oracle."""
    w = wl.decode_workload(M)
    x = wl.make_x(w)
    W, gw = nv.nvfp4_quantize(_bf16(wl.make_w_segment(w, 0)))
    out = torch.empty((M, w.N), dtype=torch.bfloat16, device=DEV)
    nv.nvfp4_linear(_bf16(x), W, gw, [nv.Segment(0, w.N, "identity_bf16", out)])
    A, ga = nv.nvfp4_quantize(_bf16(x))
    out2 = nv.nvfp4_gemm(A, ga, W, gw)
    torch.cuda.synchronize()
    assert torch.equal(out, out2)
