"""Device-side failure detection on the GPU, without a fault: a bounded wait
inside a kernel is left to run out (a barrier nothing arrives on), the kernel
records the timeout and returns, nvfp4_check reports it once and clears it,
and the context keeps working (a quantisation afterwards matches the oracle)."""
import time

import numpy as np
import pytest
import torch

from bit_quantized_linear_nvfp4_b200 import nvfp4 as nv
from bit_quantized_linear_nvfp4_b200 import workloads as wl
from oracle import nvfp4_oracle as o

pytestmark = pytest.mark.gpu
DEV = "cuda:0"
NVFP4_OK, NVFP4_ERR_DEVICE_TIMEOUT = 0, 5


def test_bounded_wait_times_out_and_context_survives():
    lib = nv.library()
    torch.cuda.synchronize()
    assert lib.nvfp4_check(None) == NVFP4_OK
    t = time.perf_counter()
    assert lib.nvfp4_selftest_bounded_wait(50_000_000, None) == NVFP4_OK  # 50 ms
    assert lib.nvfp4_check(None) == NVFP4_ERR_DEVICE_TIMEOUT
    waited = time.perf_counter() - t
    assert 0.04 <= waited < 5.0, waited  # the wait ran out by its own limit
    assert lib.nvfp4_check(None) == NVFP4_OK  # reported once, then cleared
    # the context is still usable
    x = wl.round_to_bf16(np.random.default_rng(1).standard_normal((64, 256)).astype(np.float32))
    A, g = nv.nvfp4_quantize(torch.from_numpy(x).to(DEV).to(torch.bfloat16))
    nv.nvfp4_check()
    codes, sf, _ = o.quantize(x)
    assert np.array_equal(o.unpack_codes(A.codes.cpu().numpy())[:64, :256], codes)
    assert np.float32(g.item()) == o.global_scale(x)


def test_timeout_enqueued_on_a_side_stream():
    lib = nv.library()
    s = torch.cuda.Stream()
    assert lib.nvfp4_selftest_bounded_wait(20_000_000, s.cuda_stream) == NVFP4_OK
    assert lib.nvfp4_check(s.cuda_stream) == NVFP4_ERR_DEVICE_TIMEOUT
    assert lib.nvfp4_check(None) == NVFP4_OK
