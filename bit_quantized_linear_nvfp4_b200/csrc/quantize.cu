// NVFP4 activation / weight quantiser for sm_100a.
//
// Format ("Why Gated DeltaNet Survives 4-Bit Quantization", ai.info summary,
// "Methodology in Plain English"): 4-bit E2M1 values, one E4M3 scale per 16
// consecutive elements along K, an FP32 global scale per tensor or module
// ("Main Findings", fused-GEMM bullet).  Per block of 16, in FP32:
//   s = (amax_b / 6) / g;  sf = E4M3_rn_satfinite(s);  S = decode(sf)
//   inv = S*g > 0 ? 1/(S*g) : 0, at most FLT_MAX;  code = E2M1_rn_satfinite(x*inv)
//
// HBM-bound design: a warp takes one row and up to 4 consecutive chunks of 256
// elements; lane l holds elements [8l, 8l+8) of a chunk (one 16-byte load for
// BF16), so a lane pair holds one 16-block and one shuffle gives its amax.
// Each lane stores its 8 codes as one 32-bit word (a warp writes 128
// contiguous bytes); the 4 scales of a 64-element group are gathered by
// shuffles into one 32-bit word stored at its place in the tcgen05 scale
// layout.  The padding of the scale layout (rows up to 128, K/16 up to 4) is
// written with zeros.
#include <cfloat>
#include <cstdint>

#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "internal.h"
#include "ptx.cuh"

namespace nvfp4 {

namespace qk {

constexpr int kChunk = 256;        // elements per warp per chunk
constexpr int kChunksPerItem = 4;  // chunks of one row per warp item
constexpr int kThreads = 256;

struct SegParams {
  int n;
  int64_t begin[kMaxSeg + 1];
};

__device__ __forceinline__ uint4 ld_stream_v4(const void* p) {
  uint4 r;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "l"(p));
  return r;
}

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

template <int DTYPE>
struct Loader;

template <>
struct Loader<NVFP4_DTYPE_BF16> {
  static constexpr int kBytes = 2;
  struct Raw {
    uint4 a;
  };
  __device__ __forceinline__ static Raw load(const uint8_t* p) { return Raw{ld_stream_v4(p)}; }
  __device__ __forceinline__ static void unpack(const Raw& r, float (&v)[8]) {
    v[0] = bf16_lo(r.a.x); v[1] = bf16_hi(r.a.x);
    v[2] = bf16_lo(r.a.y); v[3] = bf16_hi(r.a.y);
    v[4] = bf16_lo(r.a.z); v[5] = bf16_hi(r.a.z);
    v[6] = bf16_lo(r.a.w); v[7] = bf16_hi(r.a.w);
  }
};

template <>
struct Loader<NVFP4_DTYPE_F32> {
  static constexpr int kBytes = 4;
  struct Raw {
    uint4 a, b;
  };
  __device__ __forceinline__ static Raw load(const uint8_t* p) {
    return Raw{ld_stream_v4(p), ld_stream_v4(p + 16)};
  }
  __device__ __forceinline__ static void unpack(const Raw& r, float (&v)[8]) {
    v[0] = __uint_as_float(r.a.x); v[1] = __uint_as_float(r.a.y);
    v[2] = __uint_as_float(r.a.z); v[3] = __uint_as_float(r.a.w);
    v[4] = __uint_as_float(r.b.x); v[5] = __uint_as_float(r.b.y);
    v[6] = __uint_as_float(r.b.z); v[7] = __uint_as_float(r.b.w);
  }
};

// E4M3 (satfinite, round to nearest even) of a non-negative float: low byte.
__device__ __forceinline__ uint32_t to_e4m3(float s) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(0.0f), "f"(s));
  return r & 0xFFu;
}

// Exact value of a non-negative, non-NaN E4M3 byte, from its bit fields:
// exponent field e (bias 7), mantissa m; e == 0 is subnormal (m * 2^-9).
__device__ __forceinline__ float e4m3_value(uint32_t b) {
  const uint32_t e = (b >> 3) & 15u, m = b & 7u;
  return e ? __uint_as_float(((e + 120u) << 23) | (m << 20)) : static_cast<float>(m) * 0.001953125f;
}

// Eight E2M1 codes (satfinite, round to nearest even), element 2j in the low nibble.
__device__ __forceinline__ uint32_t to_e2m1x8(const float (&q)[8]) {
  uint32_t out;
  asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b0, %2, %1;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b1, %4, %3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b2, %6, %5;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b3, %8, %7;\n\t"
      "mov.b32 %0, {b0, b1, b2, b3};\n\t}"
      : "=r"(out)
      : "f"(q[0]), "f"(q[1]), "f"(q[2]), "f"(q[3]), "f"(q[4]), "f"(q[5]), "f"(q[6]), "f"(q[7]));
  return out;
}

__device__ __forceinline__ int find_segment(const SegParams& sp, int64_t row) {
  int s = 0;
#pragma unroll
  for (int i = 1; i < kMaxSeg; ++i)
    if (i < sp.n && row >= sp.begin[i]) s = i;
  return s;
}

// ------------------------------------------------------------------ amax

template <int DTYPE>
__global__ void __launch_bounds__(kThreads) amax_kernel(const uint8_t* __restrict__ x, int64_t K,
                                                        int64_t ld_bytes, int64_t row_begin,
                                                        int64_t rows, unsigned int* __restrict__ out) {
  using L = Loader<DTYPE>;
  const int lane = threadIdx.x & 31;
  const int64_t nchunks = (K + kChunk - 1) / kChunk;
  const int64_t groups = (nchunks + kChunksPerItem - 1) / kChunksPerItem;
  const int64_t items = rows * groups;
  const int64_t warp0 = (static_cast<int64_t>(blockIdx.x) * kThreads + threadIdx.x) >> 5;
  const int64_t nwarps = (static_cast<int64_t>(gridDim.x) * kThreads) >> 5;
  float m = 0.0f;
  for (int64_t item = warp0; item < items; item += nwarps) {
    const int64_t row = row_begin + item / groups;
    const int64_t c0 = (item % groups) * kChunksPerItem;
    const uint8_t* rp = x + row * ld_bytes;
    typename L::Raw raw[kChunksPerItem];
    bool act[kChunksPerItem];
#pragma unroll
    for (int u = 0; u < kChunksPerItem; ++u) {
      const int64_t col = (c0 + u) * kChunk + lane * 8;
      act[u] = col < K;
      if (act[u]) raw[u] = L::load(rp + col * L::kBytes);
    }
#pragma unroll
    for (int u = 0; u < kChunksPerItem; ++u) {
      if (!act[u]) continue;
      float v[8];
      L::unpack(raw[u], v);
#pragma unroll
      for (int i = 0; i < 8; ++i) m = fmaxf(m, fabsf(v[i]));
    }
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
  __shared__ float red[kThreads / 32];
  if (lane == 0) red[threadIdx.x >> 5] = m;
  __syncthreads();
  if (threadIdx.x == 0) {
    float b = 0.0f;
#pragma unroll
    for (int w = 0; w < kThreads / 32; ++w) b = fmaxf(b, red[w]);
    if (b > 0.0f) atomicMax(out, __float_as_uint(b));  // non-negative floats order as integers
  }
}

// -------------------------------------------------------------- quantise

template <int DTYPE>
__global__ void __launch_bounds__(kThreads) quantize_kernel(
    const uint8_t* __restrict__ x, int64_t M, int64_t K, int64_t ld_bytes, SegParams sp,
    const float* __restrict__ g_in, const unsigned int* __restrict__ ws_bits,
    float* __restrict__ g_out, uint8_t* __restrict__ codes, uint8_t* __restrict__ sf) {
  using L = Loader<DTYPE>;
  __shared__ float g_sh[kMaxSeg];
  if (threadIdx.x < sp.n) {
    float g = g_in ? g_in[threadIdx.x] : __uint_as_float(ws_bits[threadIdx.x]) / 2688.0f;
    g_sh[threadIdx.x] = g;
    if (blockIdx.x == 0) g_out[threadIdx.x] = g;
  }
  __syncthreads();

  const int lane = threadIdx.x & 31;
  const int64_t rows_pad = (M + 127) / 128 * 128;
  const int64_t nchunks = (K + kChunk - 1) / kChunk;
  const int64_t groups = (nchunks + kChunksPerItem - 1) / kChunksPerItem;
  const int64_t KA = (K + 63) / 64;  // scale atoms per 128-row block
  const int64_t code_ld = K / 2;
  const int64_t items = rows_pad * groups;
  const int64_t warp0 = (static_cast<int64_t>(blockIdx.x) * kThreads + threadIdx.x) >> 5;
  const int64_t nwarps = (static_cast<int64_t>(gridDim.x) * kThreads) >> 5;

  for (int64_t item = warp0; item < items; item += nwarps) {
    const int64_t row = item / groups;
    const int64_t c0 = (item % groups) * kChunksPerItem;
    const bool real_row = row < M;
    const float g = real_row ? g_sh[find_segment(sp, row)] : 0.0f;
    const bool live = real_row && (g > 0.0f);
    const uint8_t* rp = x + row * ld_bytes;

    typename L::Raw raw[kChunksPerItem];
    bool act[kChunksPerItem];
#pragma unroll
    for (int u = 0; u < kChunksPerItem; ++u) {
      const int64_t col = (c0 + u) * kChunk + lane * 8;
      act[u] = live && col < K;
      if (act[u]) raw[u] = L::load(rp + col * L::kBytes);
    }
    // scale-layout address pieces of this row
    const int64_t rb = row >> 7;
    const uint32_t in_atom = static_cast<uint32_t>((row & 31) * 16 + ((row >> 5) & 3) * 4);

#pragma unroll
    for (int u = 0; u < kChunksPerItem; ++u) {
      const int64_t chunk = c0 + u;
      if (chunk >= nchunks) break;  // uniform across the warp
      const int64_t col = chunk * kChunk + lane * 8;
      float v[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
      if (act[u]) L::unpack(raw[u], v);
      float m = 0.0f;
#pragma unroll
      for (int i = 0; i < 8; ++i) m = fmaxf(m, fabsf(v[i]));
      m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 1));  // the lane pair holds one 16-block
      uint32_t sfb = 0, word = 0;
      if (act[u]) {
        const float s = (m / 6.0f) / g;
        sfb = to_e4m3(s);
        const float denom = e4m3_value(sfb) * g;
        float inv = denom > 0.0f ? 1.0f / denom : 0.0f;
        inv = fminf(inv, FLT_MAX);
        float q[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) q[i] = v[i] * inv;
        word = to_e2m1x8(q);
      }
      if (real_row && col < K) *reinterpret_cast<uint32_t*>(codes + row * code_ld + col / 2) = word;
      // gather the 4 scale bytes of each 64-element group into lane 8a
      const int base = lane & ~7;
      const uint32_t s1 = __shfl_sync(0xffffffffu, sfb, base + 2);
      const uint32_t s2 = __shfl_sync(0xffffffffu, sfb, base + 4);
      const uint32_t s3 = __shfl_sync(0xffffffffu, sfb, base + 6);
      const int64_t kb = chunk * 4 + (lane >> 3);
      if ((lane & 7) == 0 && kb < KA) {
        const uint32_t w4 = sfb | (s1 << 8) | (s2 << 16) | (s3 << 24);
        *reinterpret_cast<uint32_t*>(sf + (rb * KA + kb) * 512 + in_atom) = w4;
      }
    }
  }
}

int grid_for(int64_t warp_items) {
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int64_t want = (warp_items + (kThreads / 32) - 1) / (kThreads / 32);
  const int64_t cap = static_cast<int64_t>(sms) * 8;  // 8 resident blocks of 256 threads
  int64_t g = want < cap ? want : cap;
  return static_cast<int>(g < 1 ? 1 : g);
}

}  // namespace qk

cudaError_t launch_amax(const void* x, int dtype, int64_t K, int64_t ld, const RowSegments& segs,
                        unsigned int* ws_bits, cudaStream_t stream) {
  using namespace qk;
  cudaError_t e = cudaMemsetAsync(ws_bits, 0, sizeof(unsigned int) * segs.n, stream);
  if (e != cudaSuccess) return e;
  const int esz = dtype == NVFP4_DTYPE_BF16 ? 2 : 4;
  const int64_t groups = ceil_div(ceil_div(K, kChunk), kChunksPerItem);
  for (int s = 0; s < segs.n; ++s) {
    const int64_t rows = segs.begin[s + 1] - segs.begin[s];
    if (rows <= 0 || K <= 0) continue;
    const int grid = grid_for(rows * groups);
    if (dtype == NVFP4_DTYPE_BF16)
      amax_kernel<NVFP4_DTYPE_BF16><<<grid, kThreads, 0, stream>>>(
          static_cast<const uint8_t*>(x), K, ld * esz, segs.begin[s], rows, ws_bits + s);
    else
      amax_kernel<NVFP4_DTYPE_F32><<<grid, kThreads, 0, stream>>>(
          static_cast<const uint8_t*>(x), K, ld * esz, segs.begin[s], rows, ws_bits + s);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

cudaError_t launch_quantize(const void* x, int dtype, int64_t M, int64_t K, int64_t ld,
                            const RowSegments& segs, const float* g_in,
                            const unsigned int* ws_bits, float* g_out, uint8_t* codes,
                            uint8_t* sf, cudaStream_t stream) {
  using namespace qk;
  SegParams sp;
  sp.n = segs.n;
  for (int i = 0; i <= kMaxSeg; ++i) sp.begin[i] = i <= segs.n ? segs.begin[i] : segs.begin[segs.n];
  const int esz = dtype == NVFP4_DTYPE_BF16 ? 2 : 4;
  const int64_t groups = ceil_div(ceil_div(K, kChunk), kChunksPerItem);
  const int64_t rows_pad = ceil_div(M, 128) * 128;
  const int grid = grid_for(rows_pad * groups);
  if (dtype == NVFP4_DTYPE_BF16)
    quantize_kernel<NVFP4_DTYPE_BF16><<<grid, kThreads, 0, stream>>>(
        static_cast<const uint8_t*>(x), M, K, ld * esz, sp, g_in, ws_bits, g_out, codes, sf);
  else
    quantize_kernel<NVFP4_DTYPE_F32><<<grid, kThreads, 0, stream>>>(
        static_cast<const uint8_t*>(x), M, K, ld * esz, sp, g_in, ws_bits, g_out, codes, sf);
  return cudaGetLastError();
}

}  // namespace nvfp4
