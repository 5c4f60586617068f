"""NVFP4 W4A4 linear layer for B200 (sm_100a): quantiser, block-scaled GEMM and
fused multi-module projection behind the C ABI in include/nvfp4.h.

The compute lives in libnvfp4.so (build with ``build.py``); ``nvfp4`` is the
ctypes binding.  ``workloads`` holds the seeded synthetic inputs.

A fused projection of two modules, each with its own global scale::

    import torch
    from bit_quantized_linear_nvfp4_b200 import nvfp4 as nv

    w = torch.cat([w_q, w_k])                      # [N, K] BF16 on the GPU, module rows stacked
    W, g_w = nv.nvfp4_quantize_segments(w, [0, w_q.shape[0], w.shape[0]])   # once, offline
    q = torch.empty((M, w_q.shape[0]), dtype=torch.bfloat16, device="cuda")
    k = torch.empty((M, w_k.shape[0]), dtype=torch.bfloat16, device="cuda")
    segs = [nv.Segment(0, w_q.shape[0], "identity", q),
            nv.Segment(w_q.shape[0], w.shape[0], "identity", k)]
    nv.nvfp4_linear(x, W, g_w, segs)               # x [M, K] BF16: quantise X, then the GEMM
    nv.nvfp4_check()                               # synchronise and raise on a device-side error

Segments may also apply a sigmoid or the GDN decay gate (FP32 outputs) or
pair into SwiGLU; ``nvfp4_quantize`` and ``nvfp4_gemm`` are the two steps on
their own."""
