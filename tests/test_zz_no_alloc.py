"""nvfp4_quantize_noalloc, the allocation-free activation quantiser.

It serves callers with no device allocator at hand when they quantise
activations, such as a plugin run by an inference runtime that owns all
memory, or code under a fixed memory plan.  Its amax scratch lives in a static
array inside the library instead of a caller workspace.  This test calls it
through the C ABI (ctypes, no Python wrapper) and checks that its codes, scale
bytes and global scale equal those of nvfp4_quantize bit for bit (the
tolerance the quantiser tests use), on calls in a row.

The first two inputs (8192 and 4096 chunks of 512 elements) are larger than
what the one-launch cluster path takes (512 chunks, 512 KB of BF16), so both
go through the two launches that pass the per-block maxima through the static
scratch.  The first has a large amax
(x40) and fills the scratch with large maxima; the second, FP32 with a much
smaller amax (x0.01) and fewer rows (so fewer amax blocks), would show any
scratch word left over from the first call as a wrong global scale.  Two
small inputs (the cluster path, which needs no scratch) follow.
"""
import ctypes

import numpy as np
import pytest
import torch

from bit_quantized_linear_nvfp4_b200 import build as nvbuild
from bit_quantized_linear_nvfp4_b200 import nvfp4 as nv

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


def _noalloc(lib, x: torch.Tensor):
    M, K = x.shape
    codes = torch.full((M, K // 2), 0xAB, dtype=torch.uint8, device=DEV)
    sf = torch.full((nv.nvfp4_sf_bytes(M, K),), 0xCD, dtype=torch.uint8, device=DEV)
    g = torch.full((1,), -1.0, dtype=torch.float32, device=DEV)
    dtype = nv.DTYPE_BF16 if x.dtype == torch.bfloat16 else nv.DTYPE_F32
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    st = lib.nvfp4_quantize_noalloc(ctypes.c_void_p(x.data_ptr()), dtype, M, K, x.stride(0),
                                    ctypes.c_void_p(g.data_ptr()), ctypes.c_void_p(codes.data_ptr()),
                                    ctypes.c_void_p(sf.data_ptr()), stream)
    assert st == 0, lib.nvfp4_status_string(st)
    return codes, sf, g


def test_noalloc_matches_quantize_on_consecutive_calls():
    nvbuild.build(verbose=False)
    lib = nv.library()
    rng = np.random.default_rng(77)
    inputs = [
        torch.from_numpy((rng.standard_normal((4096, 1024)) * 40).astype(np.float32)).to(DEV).to(torch.bfloat16),
        torch.from_numpy(rng.standard_normal((2048, 1024)).astype(np.float32) * 0.01).to(DEV),
        torch.from_numpy((rng.standard_normal((300, 512)) * 40).astype(np.float32)).to(DEV).to(torch.bfloat16),
        torch.from_numpy(rng.standard_normal((129, 272)).astype(np.float32) * 0.01).to(DEV),
    ]
    for x in inputs:
        codes, sf, g = _noalloc(lib, x)
        ref, g_ref = nv.nvfp4_quantize(x)
        torch.cuda.synchronize()
        assert torch.equal(g, g_ref), (g.item(), g_ref.item())
        assert torch.equal(codes, ref.codes)
        assert torch.equal(sf, ref.sf)
    nv.nvfp4_check()


def test_noalloc_rejects_bad_arguments_on_the_host():
    lib = nv.library()
    v = ctypes.c_void_p
    fake = 0x10000
    assert lib.nvfp4_quantize_noalloc(v(fake), 0, 4, 24, 32, v(fake), v(fake), v(fake), None) == 2
    assert lib.nvfp4_quantize_noalloc(None, 0, 4, 32, 32, v(fake), v(fake), v(fake), None) == 1
    assert lib.nvfp4_quantize_noalloc(v(fake + 4), 0, 4, 32, 32, v(fake), v(fake), v(fake), None) == 3
