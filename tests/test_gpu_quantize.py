"""GPU parity of nvfp4_quantize / nvfp4_quantize_segments with the oracle:
codes, scale bytes (after un-swizzling the MMA layout), padding and the
global scale must match bit for bit."""
import numpy as np
import pytest
import torch

from bit_quantized_linear_nvfp4_b200 import nvfp4 as nv
from bit_quantized_linear_nvfp4_b200 import workloads as wl
from oracle import nvfp4_oracle as o
from tests.gpu_helpers import assert_quant_equal, operand_to_logical

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


def _dev(x_np, dtype):
    t = torch.from_numpy(np.ascontiguousarray(x_np)).to(DEV)
    return t.to(torch.bfloat16) if dtype == "bf16" else t


def _rand(M, K, seed, dtype, outliers=0, scale=1.0):
    rng = np.random.default_rng(seed)
    x = (scale * rng.standard_normal((M, K))).astype(np.float32)
    if outliers:
        ch = rng.choice(K, size=outliers, replace=False)
        x[:, ch] *= 100
    return wl.round_to_bf16(x) if dtype == "bf16" else x


def test_tiny_workload_activation_and_weight():
    w = wl.TINY
    x = wl.make_x(w)
    wt = wl.make_w_segment(w, 0)
    for arr in (x, wt):
        op, g = nv.nvfp4_quantize(_dev(arr, "f32"))
        torch.cuda.synchronize()
        assert_quant_equal(op, g, arr)


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("M,K", [(1, 16), (3, 48), (127, 256), (129, 272), (300, 512), (64, 5120), (5, 17408),
                                 # chunks of 512 elements: the one-launch path's limit (512), one row
                                 # past it, and 64 decode tokens (two launches)
                                 (16, 16384), (17, 16384), (64, 17408)])
def test_ragged_shapes(dtype, M, K):
    x = _rand(M, K, M * 7 + K, dtype, outliers=min(3, K // 16))
    op, g = nv.nvfp4_quantize(_dev(x, dtype))
    torch.cuda.synchronize()
    assert_quant_equal(op, g, x)


def test_static_scale_and_saturation():
    x = _rand(40, 128, 1, "bf16")
    for gs in (o.global_scale(x), o.global_scale(x) / np.float32(50), o.global_scale(x) * np.float32(3)):
        g_in = torch.tensor([gs], dtype=torch.float32, device=DEV)
        op, g = nv.nvfp4_quantize(_dev(x, "bf16"), g_in)
        torch.cuda.synchronize()
        assert_quant_equal(op, g, x, g_in=gs)


def test_edge_values():
    x = _rand(8, 128, 2, "f32")
    x[0, :16] = 0.0                      # zero block
    x[0, 16:32] = -0.0                   # negative zeros
    x[1, :16] = 0.37                     # all-equal block
    x[1, 16:32] = -2.5
    x[2, :] *= 1e-3                      # small row
    x[3, 5] = 1e-30                      # tiny next to normal values
    x[4, :16] = np.float32(1e-39)        # FP32 subnormals
    x[5, 40] = 3e4                       # tensor maximum
    x[6, 64:80] = np.linspace(-1, 1, 16)
    op, g = nv.nvfp4_quantize(_dev(x, "f32"))
    torch.cuda.synchronize()
    assert_quant_equal(op, g, x)
    codes, sf, _ = operand_to_logical(op, 8, 128)
    assert sf[0, 0] == 0 and not codes[0, :16].any()
    assert sf[5, 40 // 16] == 0x7E
    assert np.all(codes[1, :16] == 7) and np.all(codes[1, 16:32] == 15)


def test_negative_zero_code_is_0x8():
    """Sign of values that round to magnitude zero is kept (code 0x8)."""
    x = np.zeros((2, 32), np.float32)
    x[0, 0] = 100.0
    x[0, 1] = -1e-3     # rounds to -0
    x[0, 2] = -0.0
    x[1, :] = -0.0      # whole block of negative zeros under a positive scale elsewhere
    op, g = nv.nvfp4_quantize(_dev(x, "f32"))
    torch.cuda.synchronize()
    codes, sf, _ = operand_to_logical(op, 2, 32)
    assert codes[0, 1] == 8 and codes[0, 2] == 8
    assert_quant_equal(op, g, x)


def test_all_zero_tensor():
    x = np.zeros((130, 64), np.float32)
    op, g = nv.nvfp4_quantize(_dev(x, "bf16"))
    torch.cuda.synchronize()
    assert float(g.item()) == 0.0
    assert_quant_equal(op, g, x)


def test_empty_rows():
    x = torch.zeros((0, 64), dtype=torch.bfloat16, device=DEV)
    codes = torch.zeros((0, 32), dtype=torch.uint8, device=DEV)
    sf = torch.zeros(512, dtype=torch.uint8, device=DEV)
    op, g = nv.nvfp4_quantize(x, codes=codes, sf=sf)
    torch.cuda.synchronize()
    assert float(g.item()) == 0.0


def test_row_stride():
    x = _rand(33, 96, 5, "bf16")
    big = torch.zeros((33, 128), dtype=torch.bfloat16, device=DEV)
    big[:, :96] = _dev(x, "bf16")
    op, g = nv.nvfp4_quantize(big[:, :96])
    torch.cuda.synchronize()
    assert_quant_equal(op, g, x)


def test_segments_per_module_scales():
    """Stacked modules, each with its own global scale (rows not 128-aligned)."""
    widths = [64, 200, 32, 32, 1]
    K = 320
    parts = [(0.02 * (s + 1)) * np.random.default_rng(s).standard_normal((wd, K)).astype(np.float32)
             for s, wd in enumerate(widths)]
    parts = [wl.round_to_bf16(p) for p in parts]
    w = np.concatenate(parts)
    bounds = np.concatenate([[0], np.cumsum(widths)])
    op, g = nv.nvfp4_quantize_segments(_dev(w, "bf16"), bounds)
    torch.cuda.synchronize()
    codes, sf, full = operand_to_logical(op, w.shape[0], K)
    gs = g.cpu().numpy()
    for s in range(len(widths)):
        oc, osf, og = o.quantize(parts[s])
        assert np.float32(gs[s]) == og
        r0, r1 = bounds[s], bounds[s + 1]
        np.testing.assert_array_equal(codes[r0:r1], oc)
        np.testing.assert_array_equal(sf[r0:r1], osf)
    # static per-segment scales
    g_in = torch.tensor(gs * 2, device=DEV)
    op2, g2 = nv.nvfp4_quantize_segments(_dev(w, "bf16"), bounds, g_in)
    torch.cuda.synchronize()
    codes2, sf2, _ = operand_to_logical(op2, w.shape[0], K)
    for s in range(len(widths)):
        oc, osf, _ = o.quantize(parts[s], np.float32(gs[s] * 2))
        r0, r1 = bounds[s], bounds[s + 1]
        np.testing.assert_array_equal(codes2[r0:r1], oc)
        np.testing.assert_array_equal(sf2[r0:r1], osf)


@pytest.mark.slow
def test_full_size_quantizer_sampled_rows():
    """The standalone quantiser workload [32768, 17408] BF16, launched as the
    benchmark launches it; global scale exact, 384 sampled rows bit-exact."""
    x = wl.make_quant_input()
    xd = _dev(x, "bf16")
    op, g = nv.nvfp4_quantize(xd)
    torch.cuda.synchronize()
    M, K = x.shape
    g_or = o.global_scale(x)
    assert np.float32(g.item()) == g_or
    rows = wl.sample_rows(M, 384)
    codes_all = op.codes[torch.from_numpy(rows).to(DEV)].cpu().numpy()
    from tests.gpu_helpers import unswizzle_sf
    sf_log = unswizzle_sf(op.sf.cpu().numpy(), M, K)
    oc, osf, _ = o.quantize(x[rows], g_or)
    np.testing.assert_array_equal(o.unpack_codes(codes_all), oc)
    np.testing.assert_array_equal(sf_log[rows, : K // 16], osf)
