"""GPU parity of the FP8 (E4M3) KV-cache codec with the oracle: codes and
decoded values bit-exact, BF16 and F32, strided rows, saturation, signed
zeros, a non-positive scale, and the benchmark's KV shape."""
import numpy as np
import pytest
import torch

from bit_quantized_linear_nvfp4_b200 import nvfp4 as nv
from bit_quantized_linear_nvfp4_b200 import workloads as wl
from oracle import nvfp4_oracle as o

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


def _kv(rows, cols, seed, dtype="bf16"):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((rows, cols)).astype(np.float32)
    x[:, rng.choice(cols, size=max(1, cols // 64), replace=False)] *= 20
    return wl.round_to_bf16(x) if dtype == "bf16" else x


def _dev(x, dtype="bf16"):
    t = torch.from_numpy(np.ascontiguousarray(x)).to(DEV)
    return t.to(torch.bfloat16) if dtype == "bf16" else t


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("rows,cols", [(1, 8), (300, 1032), (77, 2048), (5, 4104)])
@pytest.mark.parametrize("scale_kind", ["calibrated", "small"])
def test_kv_codec_matches_oracle(dtype, rows, cols, scale_kind):
    x = _kv(rows, cols, rows + cols, dtype)
    amax = np.float32(np.abs(x).max())
    s = np.float32(amax / 448) if scale_kind == "calibrated" else np.float32(amax / 448 / 7)  # the small one saturates
    sd = torch.tensor([s], dtype=torch.float32, device=DEV)
    codes = nv.nvfp4_kv_fp8_quantize(_dev(x, dtype), sd)
    out16 = nv.nvfp4_kv_fp8_dequantize(codes, sd, torch.bfloat16)
    out32 = nv.nvfp4_kv_fp8_dequantize(codes, sd, torch.float32)
    torch.cuda.synchronize()
    ref = o.kv_fp8_quantize(x, s)
    got = codes.cpu().numpy()
    assert np.array_equal(got, ref), f"{np.argwhere(got != ref)[:5]}"
    assert np.array_equal(out16.to(torch.float64).cpu().numpy(), o.kv_fp8_dequantize(ref, s, "bf16"))
    assert np.array_equal(out32.to(torch.float64).cpu().numpy(), o.kv_fp8_dequantize(ref, s, "f32"))
    if scale_kind == "small":
        assert (got & 0x7F == 0x7E).any()  # saturated values present


def test_strided_rows_signed_zero_and_bad_scale():
    x = _kv(40, 256, 9)
    x[0, :8] = [0.0, -0.0, 1e-30, -1e-30, 1e30, -1e30, 0.5, -0.5]
    big = torch.zeros((40, 384), dtype=torch.bfloat16, device=DEV)
    big[:, :256] = _dev(x)
    s = np.float32(0.01)
    sd = torch.tensor([s], dtype=torch.float32, device=DEV)
    out = torch.full((40, 320), 0xAB, dtype=torch.uint8, device=DEV)
    nv.nvfp4_kv_fp8_quantize(big[:, :256], sd, out=out[:, :256])
    torch.cuda.synchronize()
    assert np.array_equal(out[:, :256].cpu().numpy(), o.kv_fp8_quantize(x, s))
    assert torch.all(out[:, 256:] == 0xAB)
    assert out[0, 1].item() == 0x80  # -0 keeps its sign
    for bad in (0.0, -2.0, float("inf")):
        c = nv.nvfp4_kv_fp8_quantize(_dev(x), torch.tensor([bad], dtype=torch.float32, device=DEV))
        torch.cuda.synchronize()
        assert not c.any()


def test_benchmark_kv_shape():
    """The benchmark's K (or V) cache chunk: 32768 tokens x 8 heads x 128."""
    x = _kv(32768, 1024, 77)
    s = np.float32(np.abs(x).max() / 448)
    sd = torch.tensor([s], dtype=torch.float32, device=DEV)
    codes = nv.nvfp4_kv_fp8_quantize(_dev(x), sd)
    torch.cuda.synchronize()
    assert np.array_equal(codes.cpu().numpy(), o.kv_fp8_quantize(x, s))
