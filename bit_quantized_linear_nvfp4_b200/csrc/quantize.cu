// NVFP4 activation / weight quantiser for sm_100a.
//
// Format ("Why Gated DeltaNet Survives 4-Bit Quantization", ai.info summary,
// "Methodology in Plain English"): 4-bit E2M1 values, one E4M3 scale per 16
// consecutive elements along K, an FP32 global scale per tensor or module
// ("Main Findings", fused-GEMM bullet).  Per block of 16, in FP32:
//   s = (amax_b / 6) / g;  sf = E4M3_rn_satfinite(s);  S = decode(sf)
//   inv = S*g > 0 ? 1/(S*g) : 0, at most FLT_MAX;  code = E2M1_rn_satfinite(x*inv)
// with g = amax|x| / (6 * 448) per tensor (or per row range) when not given.
//
// HBM-bound design.  A warp takes a chunk of 512 consecutive elements of one
// row; lane l owns the 16-block l of the chunk (one 256-bit load for BF16),
// so the block amax, scale and codes need no cross-lane traffic.  Each lane
// stores its 16 codes as 8 contiguous bytes (a warp writes 256 bytes), and
// four lanes' scale bytes are gathered by shuffles into one 32-bit word
// stored at its place in the tcgen05 block-scale layout; layout padding
// (rows up to 128, K/16 up to 4) is written with zeros.
//
// With a device-computed scale the kernel runs two passes in one cooperative
// launch: amax over the rows, a grid barrier (bounded wait), then the
// quantisation pass, which re-reads x from L2 when x fits there.
#include <cfloat>
#include <cstdint>

#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "internal.h"
#include "ptx.cuh"

namespace nvfp4 {
namespace qk {

constexpr int kChunk = 512;  // elements per warp per chunk (32 lanes x 16)
// Large blocks keep the number of blocks (and so of same-address atomics in
// the amax reduction and the grid barrier) near the SM count; FP32 input
// needs more registers per lane and uses smaller blocks.
template <int DTYPE>
struct Cfg {
  static constexpr int kThreads = DTYPE == NVFP4_DTYPE_BF16 ? 1024 : 256;
  static constexpr int kWarps = kThreads / 32;
};
constexpr int kUnrollQ = 2;  // chunks per warp iteration, quantisation pass
constexpr int kUnrollA = 4;  // chunks per warp iteration, amax pass

struct QuantArgs {
  const uint8_t* x;
  int64_t ld_bytes;
  int32_t M, K, rows_pad, cpr;  // cpr: chunks per row
  int32_t items_q, items_a;     // rows_pad * cpr, M * cpr
  int nseg;
  int32_t seg_begin[kMaxSeg + 1];
  const float* g_in;
  unsigned int* ws;  // [nseg] amax bits, [nseg] grid-barrier counter (dynamic only)
  float* g_out;
  uint8_t* codes;
  uint8_t* sf;
};

__device__ __forceinline__ void ld_v8(const void* p, uint32_t* r) {
  asm volatile("ld.global.nc.L1::no_allocate.v8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]),
                 "=r"(r[6]), "=r"(r[7])
               : "l"(p));
}
__device__ __forceinline__ void ld_v4(const void* p, uint32_t* r) {
  asm volatile("ld.global.nc.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "l"(p));
}

// Raw 16-element block of one lane: 8 words (BF16) or 16 words (F32).
template <int DTYPE>
struct Block {
  static constexpr int kWords = DTYPE == NVFP4_DTYPE_BF16 ? 8 : 16;
  uint32_t w[kWords];
};

template <int DTYPE, bool WIDE>
__device__ __forceinline__ void load_block(const uint8_t* p, Block<DTYPE>& b) {
  if constexpr (DTYPE == NVFP4_DTYPE_BF16) {
    if constexpr (WIDE) {
      ld_v8(p, b.w);
    } else {
      ld_v4(p, b.w);
      ld_v4(p + 16, b.w + 4);
    }
  } else {
    if constexpr (WIDE) {
      ld_v8(p, b.w);
      ld_v8(p + 32, b.w + 8);
    } else {
#pragma unroll
      for (int i = 0; i < 4; ++i) ld_v4(p + 16 * i, b.w + 4 * i);
    }
  }
}

template <int DTYPE>
__device__ __forceinline__ void unpack(const Block<DTYPE>& b, float (&v)[16]) {
  if constexpr (DTYPE == NVFP4_DTYPE_BF16) {
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      v[2 * i] = __uint_as_float(b.w[i] << 16);
      v[2 * i + 1] = __uint_as_float(b.w[i] & 0xFFFF0000u);
    }
  } else {
#pragma unroll
    for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(b.w[i]);
  }
}

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
__device__ __forceinline__ uint32_t to_e2m1x8(const float* q) {
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

__device__ __forceinline__ int find_segment(const QuantArgs& a, int32_t row) {
  int s = 0;
#pragma unroll
  for (int i = 1; i < kMaxSeg; ++i)
    if (i < a.nseg && row >= a.seg_begin[i]) s = i;
  return s;
}

__device__ __forceinline__ unsigned int ld_acquire_u32(const unsigned int* p) {
  unsigned int v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

// Pass 1: per-segment amax of rows [0, M), one atomicMax per block and segment.
template <int DTYPE, bool WIDE>
__device__ __forceinline__ void amax_pass(const QuantArgs& a) {
  constexpr int kWarps = Cfg<DTYPE>::kWarps;
  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  const int32_t gwarp = blockIdx.x * kWarps + warp;
  const int32_t nwarps = gridDim.x * kWarps;
  constexpr int kEsz = DTYPE == NVFP4_DTYPE_BF16 ? 2 : 4;
  float lm[kMaxSeg];
#pragma unroll
  for (int s = 0; s < kMaxSeg; ++s) lm[s] = 0.0f;
  for (int32_t base = gwarp * kUnrollA; base < a.items_a; base += nwarps * kUnrollA) {
    Block<DTYPE> blk[kUnrollA];
    int32_t rows[kUnrollA];
    bool act[kUnrollA];
#pragma unroll
    for (int u = 0; u < kUnrollA; ++u) {
      const int32_t item = base + u;
      const int32_t row = item / a.cpr;
      const int32_t col = (item - row * a.cpr) * kChunk + lane * 16;
      rows[u] = row;
      act[u] = item < a.items_a && col < a.K;
      if (act[u]) load_block<DTYPE, WIDE>(a.x + row * a.ld_bytes + static_cast<int64_t>(col) * kEsz, blk[u]);
    }
#pragma unroll
    for (int u = 0; u < kUnrollA; ++u) {
      if (!act[u]) continue;
      float v[16];
      unpack<DTYPE>(blk[u], v);
      float m = 0.0f;
#pragma unroll
      for (int i = 0; i < 16; ++i) m = fmaxf(m, fabsf(v[i]));
      const int s = find_segment(a, rows[u]);
#pragma unroll
      for (int i = 0; i < kMaxSeg; ++i)
        if (i == s) lm[i] = fmaxf(lm[i], m);
    }
  }
  __shared__ float red[kWarps][kMaxSeg];
#pragma unroll
  for (int s = 0; s < kMaxSeg; ++s) {
    float m = lm[s];
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
    if (lane == 0) red[warp][s] = m;
  }
  __syncthreads();
  if (threadIdx.x < a.nseg) {
    float m = 0.0f;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) m = fmaxf(m, red[w][threadIdx.x]);
    if (m > 0.0f) atomicMax(a.ws + threadIdx.x, __float_as_uint(m));  // non-negative floats order as integers
  }
}

// Pass 2: quantise rows [0, rows_pad) (rows >= M only zero their scale words).
template <int DTYPE, bool WIDE>
__device__ __forceinline__ void quant_pass(const QuantArgs& a, const float* g_sh) {
  constexpr int kWarps = Cfg<DTYPE>::kWarps;
  const int lane = threadIdx.x & 31;
  const int32_t gwarp = blockIdx.x * kWarps + (threadIdx.x >> 5);
  const int32_t nwarps = gridDim.x * kWarps;
  constexpr int kEsz = DTYPE == NVFP4_DTYPE_BF16 ? 2 : 4;
  const int32_t KA = (a.K + 63) / 64;
  const int64_t code_ld = a.K / 2;
  for (int32_t base = gwarp * kUnrollQ; base < a.items_q; base += nwarps * kUnrollQ) {
    Block<DTYPE> blk[kUnrollQ];
    int32_t rows[kUnrollQ], cols[kUnrollQ];
    bool act[kUnrollQ];
    float gs[kUnrollQ];
#pragma unroll
    for (int u = 0; u < kUnrollQ; ++u) {
      const int32_t item = base + u;
      const int32_t row = item / a.cpr;
      const int32_t col = (item - row * a.cpr) * kChunk + lane * 16;
      rows[u] = row;
      cols[u] = col;
      gs[u] = row < a.M ? g_sh[find_segment(a, row)] : 0.0f;
      act[u] = item < a.items_q && row < a.M && col < a.K && gs[u] > 0.0f;
      if (act[u]) load_block<DTYPE, WIDE>(a.x + row * a.ld_bytes + static_cast<int64_t>(col) * kEsz, blk[u]);
    }
#pragma unroll
    for (int u = 0; u < kUnrollQ; ++u) {
      const int32_t item = base + u;
      if (item >= a.items_q) break;  // uniform across the warp
      const int32_t row = rows[u], col = cols[u];
      uint32_t sfb = 0;
      uint2 word = make_uint2(0u, 0u);
      if (act[u]) {
        const float g = gs[u];
        float v[16];
        unpack<DTYPE>(blk[u], v);
        float m = 0.0f;
#pragma unroll
        for (int i = 0; i < 16; ++i) m = fmaxf(m, fabsf(v[i]));
        const float s = (m / 6.0f) / g;
        sfb = to_e4m3(s);
        const float denom = e4m3_value(sfb) * g;
        float inv = denom > 0.0f ? 1.0f / denom : 0.0f;
        inv = fminf(inv, FLT_MAX);
        float q[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) q[i] = v[i] * inv;
        word.x = to_e2m1x8(q);
        word.y = to_e2m1x8(q + 8);
      }
      if (row < a.M && col < a.K)
        *reinterpret_cast<uint2*>(a.codes + row * code_ld + col / 2) = word;
      // four lanes' scale bytes -> one 32-bit word of the block-scale layout
      const uint32_t s1 = __shfl_down_sync(0xffffffffu, sfb, 1);
      const uint32_t s2 = __shfl_down_sync(0xffffffffu, sfb, 2);
      const uint32_t s3 = __shfl_down_sync(0xffffffffu, sfb, 3);
      const int32_t kb = col / 64;
      if ((lane & 3) == 0 && kb < KA) {
        const int64_t off = (static_cast<int64_t>(row >> 7) * KA + kb) * 512 + (row & 31) * 16 + ((row >> 5) & 3) * 4;
        *reinterpret_cast<uint32_t*>(a.sf + off) = sfb | (s1 << 8) | (s2 << 16) | (s3 << 24);
      }
    }
  }
}

template <int DTYPE, bool WIDE, bool DYNAMIC>
__global__ void __launch_bounds__(Cfg<DTYPE>::kThreads) quantize_kernel(const __grid_constant__ QuantArgs a) {
  __shared__ float g_sh[kMaxSeg];
  __shared__ int abort_sh;
  if constexpr (DYNAMIC) {
    amax_pass<DTYPE, WIDE>(a);
    // grid barrier: every block's amax is published before any block reads it
    __syncthreads();
    if (threadIdx.x == 0) {
      abort_sh = 0;
      unsigned int* counter = a.ws + a.nseg;
      __threadfence();
      atomicAdd(counter, 1u);
      const uint64_t t0 = global_timer_ns();
      while (ld_acquire_u32(counter) < gridDim.x) {
        if (global_timer_ns() - t0 > 2000000000ull) {
          atomicOr(&g_device_error, kErrTimeout);
          abort_sh = 1;
          break;
        }
        __nanosleep(64);
      }
    }
    __syncthreads();
    if (abort_sh) return;
    if (threadIdx.x < a.nseg) {
      const float g = __uint_as_float(ld_acquire_u32(a.ws + threadIdx.x)) / 2688.0f;
      g_sh[threadIdx.x] = g;
      if (blockIdx.x == 0) a.g_out[threadIdx.x] = g;
    }
  } else {
    if (threadIdx.x < a.nseg) {
      const float g = a.g_in[threadIdx.x];
      g_sh[threadIdx.x] = g;
      if (blockIdx.x == 0) a.g_out[threadIdx.x] = g;
    }
  }
  __syncthreads();
  quant_pass<DTYPE, WIDE>(a, g_sh);
}

int num_sms() {
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  return sms;
}

template <int DTYPE, bool WIDE, bool DYNAMIC>
cudaError_t launch_t(const QuantArgs& a, cudaStream_t stream) {
  constexpr int kThreads = Cfg<DTYPE>::kThreads;
  constexpr int kWarps = Cfg<DTYPE>::kWarps;
  auto kern = quantize_kernel<DTYPE, WIDE, DYNAMIC>;
  int per_sm = 0;
  cudaError_t e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kThreads, 0);
  if (e != cudaSuccess) return e;
  if (per_sm < 1) per_sm = 1;
  const int64_t cap = static_cast<int64_t>(num_sms()) * per_sm;
  const int64_t want = (static_cast<int64_t>(a.items_q) + kWarps * kUnrollQ - 1) / (kWarps * kUnrollQ);
  int grid = static_cast<int>(want < cap ? want : cap);
  if (grid < 1) grid = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = DYNAMIC ? 1 : 0;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, a);
}

}  // namespace qk

size_t quantize_scratch_words(int nseg) { return static_cast<size_t>(nseg) + 1; }

cudaError_t launch_quantize(const void* x, int dtype, int64_t M, int64_t K, int64_t ld,
                            const RowSegments& segs, const float* g_in, unsigned int* ws,
                            float* g_out, uint8_t* codes, uint8_t* sf, cudaStream_t stream) {
  using namespace qk;
  QuantArgs a{};
  const int esz = dtype == NVFP4_DTYPE_BF16 ? 2 : 4;
  a.x = static_cast<const uint8_t*>(x);
  a.ld_bytes = ld * esz;
  a.M = static_cast<int32_t>(M);
  a.K = static_cast<int32_t>(K);
  a.rows_pad = static_cast<int32_t>(ceil_div(M, 128) * 128);
  a.cpr = static_cast<int32_t>(ceil_div(K, kChunk));
  a.items_q = a.rows_pad * a.cpr;
  a.items_a = a.M * a.cpr;
  a.nseg = segs.n;
  for (int i = 0; i <= kMaxSeg; ++i)
    a.seg_begin[i] = static_cast<int32_t>(i <= segs.n ? segs.begin[i] : segs.begin[segs.n]);
  a.g_in = g_in;
  a.ws = ws;
  a.g_out = g_out;
  a.codes = codes;
  a.sf = sf;
  const bool dynamic = g_in == nullptr;
  if (dynamic) {
    cudaError_t e = cudaMemsetAsync(ws, 0, sizeof(unsigned int) * quantize_scratch_words(segs.n), stream);
    if (e != cudaSuccess) return e;
  }
  const bool wide = (reinterpret_cast<uintptr_t>(x) % 32 == 0) && (a.ld_bytes % 32 == 0);
  if (dtype == NVFP4_DTYPE_BF16) {
    if (dynamic) return wide ? launch_t<NVFP4_DTYPE_BF16, true, true>(a, stream)
                             : launch_t<NVFP4_DTYPE_BF16, false, true>(a, stream);
    return wide ? launch_t<NVFP4_DTYPE_BF16, true, false>(a, stream)
                : launch_t<NVFP4_DTYPE_BF16, false, false>(a, stream);
  }
  if (dynamic) return wide ? launch_t<NVFP4_DTYPE_F32, true, true>(a, stream)
                           : launch_t<NVFP4_DTYPE_F32, false, true>(a, stream);
  return wide ? launch_t<NVFP4_DTYPE_F32, true, false>(a, stream)
              : launch_t<NVFP4_DTYPE_F32, false, false>(a, stream);
}

}  // namespace nvfp4
