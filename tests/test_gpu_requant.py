"""GPU parity of nvfp4_requantize_segments (checkpoint-side harmonisation)
with the oracle's requantize: codes and scale bytes bit-exact, padding zero,
out of place and in place; and a harmonised GDN-style weight through the
fused projection with one common scale."""
import numpy as np
import pytest
import torch

from bit_quantized_linear_nvfp4_b200 import nvfp4 as nv
from bit_quantized_linear_nvfp4_b200 import workloads as wl
from oracle import nvfp4_oracle as o
from tests.gpu_helpers import TOL_ACC, check_bf16, operand_to_logical, to_np

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


def _mods(widths, K, seed, gains):
    rng = np.random.default_rng(seed)
    return [wl.round_to_bf16((0.02 * gain * rng.standard_normal((n, K))).astype(np.float32))
            for n, gain in zip(widths, gains)]


def _check(op, g_out, c_ref, s_ref, g_ref, N, K, nseg):
    codes, sf, full = operand_to_logical(op, N, K)
    assert np.array_equal(sf, s_ref), f"{np.argwhere(sf != s_ref)[:5]}"
    assert np.array_equal(codes, c_ref), f"{np.argwhere(codes != c_ref)[:5]}"
    pad = full.copy()
    pad[:N, : K // 16] = 0
    assert not pad.any()
    assert np.all(g_out.cpu().numpy() == np.float32(g_ref)) and g_out.numel() == nseg


@pytest.mark.parametrize("K", [320, 1024])
@pytest.mark.parametrize("in_place", [False, True])
@pytest.mark.parametrize("given", [False, True])
def test_requantize_matches_oracle(K, in_place, given):
    widths, gains = [100, 37, 200], [1.0, 2.75, 0.6]
    mods = _mods(widths, K, 5 + K, gains)
    bounds = np.concatenate([[0], np.cumsum(widths)])
    N = int(bounds[-1])
    W, gw = nv.nvfp4_quantize_segments(torch.from_numpy(np.concatenate(mods)).to(DEV).to(torch.bfloat16), bounds)
    torch.cuda.synchronize()
    c_in, s_in, _ = operand_to_logical(W, N, K)
    g_old = gw.cpu().numpy()
    # given: a smaller common scale (clips the larger modules' top blocks); else the fused tensor's
    g_new = np.float32(g_old.min()) if given else np.float32(g_old.max())
    g_rows = np.repeat(g_old, widths)
    c_ref, s_ref, g_ref = o.requantize(c_in, s_in, g_rows, g_new)
    g_dev = torch.tensor([g_new], dtype=torch.float32, device=DEV) if given else None
    R, g_out = nv.nvfp4_requantize_segments(W, bounds, gw, g_dev, in_place=in_place)
    torch.cuda.synchronize()
    if in_place:
        assert R.codes.data_ptr() == W.codes.data_ptr()
    _check(R, g_out, c_ref, s_ref, g_ref, N, K, len(widths))
    nv.nvfp4_check()


def test_requantize_same_scale_is_identity():
    mods = _mods([256, 64], 512, 9, [1.0, 3.0])
    W, gw = nv.nvfp4_quantize_segments(torch.from_numpy(np.concatenate(mods)).to(DEV).to(torch.bfloat16), [0, 256, 320])
    one = nv.Operand(W.codes[:256], W.sf[: nv.nvfp4_sf_bytes(256, 512)], 256, 512)
    R, g_out = nv.nvfp4_requantize_segments(one, [0, 256], gw[:1])
    torch.cuda.synchronize()
    assert torch.equal(R.codes, one.codes) and torch.equal(R.sf, one.sf)


def test_harmonised_gdn_weight_with_one_common_scale():
    """Segments q, k (gain 1) and b, a (gain 2.75): re-encode under the fused
    scale, then run the fused projection with one common scale for every
    segment, as a single-scale kernel would; compare with the oracle's
    requantize followed by its fused projection."""
    K, M = 1024, 200
    widths = [256, 256, 32, 32]
    mods = _mods(widths, K, 21, [1.0, 1.0, 2.75, 2.75])
    bounds = np.concatenate([[0], np.cumsum(widths)])
    rng = np.random.default_rng(22)
    x = wl.round_to_bf16(rng.standard_normal((M, K)).astype(np.float32))
    W, gw = nv.nvfp4_quantize_segments(torch.from_numpy(np.concatenate(mods)).to(DEV).to(torch.bfloat16), bounds)
    R, g_out = nv.nvfp4_requantize_segments(W, bounds, gw)
    A, ga = nv.nvfp4_quantize(torch.from_numpy(x).to(DEV).to(torch.bfloat16))
    outs = [torch.empty((M, n), dtype=torch.bfloat16, device=DEV) for n in widths]
    nv.nvfp4_fused_proj(A, ga, R, g_out, [nv.Segment(int(bounds[i]), int(bounds[i + 1]), "identity_bf16", outs[i])
                                          for i in range(len(widths))])
    torch.cuda.synchronize()
    assert len(set(g_out.cpu().numpy().tolist())) == 1
    aq = o.quantize(x)
    mq = [o.quantize(m) for m in mods]
    assert np.array_equal(np.array([g for _, _, g in mq], np.float32), gw.cpu().numpy())
    g_c = np.float32(max(g for _, _, g in mq))
    wq = [o.requantize(c, s, g, g_c) for c, s, g in mq]
    ref, pre = o.fused_projection(aq, [(c, s) for c, s, _ in wq], [g_c] * len(widths), ["identity"] * len(widths))
    for i in range(len(widths)):
        check_bf16(to_np(outs[i]), ref[i], TOL_ACC * pre[i][1], f"segment {i}")
