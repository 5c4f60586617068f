// Single translation unit of libnvfp4: the kernels share the device error
// word, so they are compiled together without relocatable device code.
#include "quantize.cu"
#include "gemm.cu"
#include "gemm_decode.cu"
#include "api.cu"
#include "noalloc.cu"
#include "kv_fp8.cu"
#include "act_stats.cu"
#include "gdn.cu"
#include "selftest.cu"
