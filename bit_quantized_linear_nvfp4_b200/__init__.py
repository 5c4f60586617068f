"""NVFP4 W4A4 linear layer for B200 (sm_100a): quantiser, block-scaled GEMM and
fused multi-module projection behind the C ABI in include/nvfp4.h.

The compute lives in libnvfp4.so (build with ``build.py``); ``nvfp4`` is the
ctypes binding.  ``workloads`` holds the seeded synthetic inputs."""
