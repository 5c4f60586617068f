// FP8 (E4M3) KV-cache codec with a calibrated static per-tensor scale, sm_100a.
//
// "Why Gated DeltaNet Survives 4-Bit Quantization" (ai.info summary), "Main
// Findings", KV-cache bullet: the FP8 KV cache keeps calibrated scales rather
// than 1.0.  Encoding, in FP32: inv = 1 / scale (once per launch),
// code = E4M3_rn_satfinite(x * inv) with the sign kept (also for zero); a
// scale that is not a positive finite number gives all-zero codes.  Decoding:
// e4m3 * scale rounded to FP32, then to BF16 for a BF16 output.
//
// HBM-bound elementwise kernels: a warp takes a 1024-element span of one row,
// each lane four 8-element vectors (16-byte BF16 or 32-byte F32 loads, 8-byte
// code stores), all loads in flight before the conversions.  Every kernel
// waits on the previous kernel of the stream (griddepcontrol.wait) before it
// touches memory.
#include <cstdint>

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include "internal.h"
#include "ptx.cuh"

namespace nvfp4 {
namespace kv {

constexpr int kThreads = 512;
constexpr int kVec = 8;                 // elements per lane per vector
constexpr int kPerLane = 4;             // vectors per lane per span
constexpr int kSpan = 32 * kVec * kPerLane;  // 1024 elements per warp step

struct KvArgs {
  const uint8_t* src;
  int64_t ld_src_bytes;
  uint8_t* dst;
  int64_t ld_dst_bytes;
  int64_t rows, cols;
  int64_t spans_per_row;
  const float* scale;
};

__device__ __forceinline__ uint32_t e4m3x4(float a, float b, float c, float d) {
  uint16_t lo, hi;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %2, %1;" : "=h"(lo) : "f"(a), "f"(b));
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %2, %1;" : "=h"(hi) : "f"(c), "f"(d));
  return static_cast<uint32_t>(lo) | (static_cast<uint32_t>(hi) << 16);
}

// Two E4M3 bytes (low byte first) -> two floats, exactly (every E4M3 value is
// an FP16 value).
__device__ __forceinline__ float2 e4m3x2_to_f32(uint16_t v) {
  uint32_t h2;
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h2) : "h"(v));
  const __half2 h = *reinterpret_cast<const __half2*>(&h2);
  return __half22float2(h);
}

template <int DTYPE>
__global__ void __launch_bounds__(kThreads) kv_quant_kernel(const __grid_constant__ KvArgs a) {
  constexpr int kEsz = DTYPE == NVFP4_DTYPE_BF16 ? 2 : 4;
  grid_dependency_wait();
  if (threadIdx.x == 0) grid_launch_dependents();
  const float s = __ldg(a.scale);
  const bool ok = s > 0.0f && s <= 3.4028234663852886e38f;
  const float inv = ok ? 1.0f / s : 0.0f;
  const int lane = threadIdx.x & 31;
  const int64_t warps = static_cast<int64_t>(gridDim.x) * (kThreads / 32);
  const int64_t items = a.rows * a.spans_per_row;
  for (int64_t it = static_cast<int64_t>(blockIdx.x) * (kThreads / 32) + (threadIdx.x >> 5); it < items; it += warps) {
    const int64_t row = it / a.spans_per_row;
    const int64_t c0 = (it - row * a.spans_per_row) * kSpan;
    const uint8_t* src = a.src + row * a.ld_src_bytes;
    uint32_t w[kPerLane][kVec * kEsz / 4];
#pragma unroll
    for (int u = 0; u < kPerLane; ++u) {
      const int64_t c = c0 + u * 32 * kVec + lane * kVec;
      if (c < a.cols) {
#pragma unroll
        for (int q = 0; q < kVec * kEsz / 16; ++q) {
          const uint4 v = __ldg(reinterpret_cast<const uint4*>(src + c * kEsz) + q);
          w[u][4 * q] = v.x;
          w[u][4 * q + 1] = v.y;
          w[u][4 * q + 2] = v.z;
          w[u][4 * q + 3] = v.w;
        }
      }
    }
#pragma unroll
    for (int u = 0; u < kPerLane; ++u) {
      const int64_t c = c0 + u * 32 * kVec + lane * kVec;
      if (c >= a.cols) continue;
      float f[kVec];
      if constexpr (DTYPE == NVFP4_DTYPE_BF16) {
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          f[2 * i] = __uint_as_float(w[u][i] << 16);
          f[2 * i + 1] = __uint_as_float(w[u][i] & 0xFFFF0000u);
        }
      } else {
#pragma unroll
        for (int i = 0; i < kVec; ++i) f[i] = __uint_as_float(w[u][i]);
      }
      uint2 out = make_uint2(0u, 0u);
      if (ok) {
        out.x = e4m3x4(f[0] * inv, f[1] * inv, f[2] * inv, f[3] * inv);
        out.y = e4m3x4(f[4] * inv, f[5] * inv, f[6] * inv, f[7] * inv);
      }
      *reinterpret_cast<uint2*>(a.dst + row * a.ld_dst_bytes + c) = out;
    }
  }
}

template <int DTYPE>
__global__ void __launch_bounds__(kThreads) kv_dequant_kernel(const __grid_constant__ KvArgs a) {
  constexpr int kEsz = DTYPE == NVFP4_DTYPE_BF16 ? 2 : 4;
  grid_dependency_wait();
  if (threadIdx.x == 0) grid_launch_dependents();
  const float s = __ldg(a.scale);
  const int lane = threadIdx.x & 31;
  const int64_t warps = static_cast<int64_t>(gridDim.x) * (kThreads / 32);
  const int64_t items = a.rows * a.spans_per_row;
  for (int64_t it = static_cast<int64_t>(blockIdx.x) * (kThreads / 32) + (threadIdx.x >> 5); it < items; it += warps) {
    const int64_t row = it / a.spans_per_row;
    const int64_t c0 = (it - row * a.spans_per_row) * kSpan;
    uint2 q[kPerLane];
#pragma unroll
    for (int u = 0; u < kPerLane; ++u) {
      const int64_t c = c0 + u * 32 * kVec + lane * kVec;
      if (c < a.cols) q[u] = __ldg(reinterpret_cast<const uint2*>(a.src + row * a.ld_src_bytes + c));
    }
#pragma unroll
    for (int u = 0; u < kPerLane; ++u) {
      const int64_t c = c0 + u * 32 * kVec + lane * kVec;
      if (c >= a.cols) continue;
      float f[kVec];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const uint32_t word = i < 2 ? q[u].x : q[u].y;
        const float2 p = e4m3x2_to_f32(static_cast<uint16_t>(word >> (16 * (i & 1))));
        f[2 * i] = p.x * s;
        f[2 * i + 1] = p.y * s;
      }
      uint8_t* dst = a.dst + row * a.ld_dst_bytes + c * kEsz;
      if constexpr (DTYPE == NVFP4_DTYPE_BF16) {
        uint32_t o[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const __nv_bfloat162 b = __floats2bfloat162_rn(f[2 * i], f[2 * i + 1]);
          o[i] = *reinterpret_cast<const uint32_t*>(&b);
        }
        *reinterpret_cast<uint4*>(dst) = make_uint4(o[0], o[1], o[2], o[3]);
      } else {
        *reinterpret_cast<float4*>(dst) = make_float4(f[0], f[1], f[2], f[3]);
        *reinterpret_cast<float4*>(dst + 16) = make_float4(f[4], f[5], f[6], f[7]);
      }
    }
  }
}

int sm_count() {
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  return sms;
}

template <class Kern>
cudaError_t launch(Kern kern, const KvArgs& a, cudaStream_t stream) {
  const int64_t items = a.rows * a.spans_per_row;
  const int64_t per_block = kThreads / 32;
  int64_t grid = (items + per_block - 1) / per_block;
  const int64_t cap = static_cast<int64_t>(sm_count()) * 4;
  if (grid > cap) grid = cap;
  if (grid < 1) grid = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(grid));
  cfg.blockDim = dim3(kThreads);
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, a);
}

}  // namespace kv

cudaError_t launch_kv_fp8(bool encode, int dtype, const void* src, int64_t ld_src, void* dst, int64_t ld_dst,
                          int64_t rows, int64_t cols, const float* scale, cudaStream_t stream) {
  using namespace kv;
  if (rows == 0 || cols == 0) return cudaSuccess;
  const int esz = dtype == NVFP4_DTYPE_BF16 ? 2 : 4;
  KvArgs a{};
  a.src = static_cast<const uint8_t*>(src);
  a.dst = static_cast<uint8_t*>(dst);
  a.ld_src_bytes = encode ? ld_src * esz : ld_src;
  a.ld_dst_bytes = encode ? ld_dst : ld_dst * esz;
  a.rows = rows;
  a.cols = cols;
  a.spans_per_row = (cols + kSpan - 1) / kSpan;
  a.scale = scale;
  if (encode)
    return dtype == NVFP4_DTYPE_BF16 ? launch(kv_quant_kernel<NVFP4_DTYPE_BF16>, a, stream)
                                     : launch(kv_quant_kernel<NVFP4_DTYPE_F32>, a, stream);
  return dtype == NVFP4_DTYPE_BF16 ? launch(kv_dequant_kernel<NVFP4_DTYPE_BF16>, a, stream)
                                   : launch(kv_dequant_kernel<NVFP4_DTYPE_F32>, a, stream);
}

}  // namespace nvfp4
