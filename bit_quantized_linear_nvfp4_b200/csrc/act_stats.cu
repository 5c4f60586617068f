// Activation statistics at NVFP4 granularity, sm_100a.
//
// "Why Gated DeltaNet Survives 4-Bit Quantization" (ai.info summary), "Main
// Findings", activation bullet: the residual stream's max/RMS, kurtosis, hot
// channels against the median channel, the share of 16-element blocks
// dominated by a single value, and the per-token A4 quantisation error.  One
// pass over X accumulates (the caller zeroes the outputs once; later calls
// add, e.g. over calibration batches):
//   moments[8] (FP64): sum x, sum x^2, sum x^3, sum x^4, max |x|, elements,
//                      16-blocks, dominated 16-blocks (largest magnitude >
//                      the sum of the other fifteen, decided in FP64);
//   row_err2[M], row_norm2[M] (FP32): sum (x - x_hat)^2 and sum x^2 per row,
//                      x_hat the NVFP4 dequantisation under the global scale g
//                      with the quantiser's exact arithmetic;
//   col_sq[K], col_max[K] (FP32): sum x^2 and max |x| per column.
//
// HBM-bound.  A warp owns a unit = (512-column strip, range of rows); lane l
// reads block l of the strip in each row with one 256-bit load; rows stream
// in pairs through two register buffers, the next pair loading while the
// current one is processed.  Per-column sums stay in the lane's registers for
// the whole unit, so the column outputs take one atomic per column and unit;
// the row sums of four rows are reduced together (one reduce-scatter), one
// atomic per row and strip; FP64 moments are block-reduced, one atomic per
// block.
#include <cfloat>
#include <cstdint>

#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include "internal.h"
#include "ptx.cuh"

namespace nvfp4 {
namespace st {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;

struct StatsArgs {
  const uint8_t* x;
  int64_t ld_bytes;
  int32_t M, K, cpr;  // cpr: 512-column strips
  int32_t ranges;     // row ranges per strip
  const float* g;
  double* moments;
  float* row_err2;
  float* row_norm2;
  float* col_sq;
  float* col_max;
};

template <int DTYPE>
struct Raw {
  uint32_t w[DTYPE == NVFP4_DTYPE_BF16 ? 8 : 16];
};

__device__ __forceinline__ void ld_v8(const void* p, uint32_t* r) {
  asm volatile("ld.global.nc.L1::no_allocate.v8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]),
                 "=r"(r[6]), "=r"(r[7])
               : "l"(p));
}

template <int DTYPE, bool WIDE>
__device__ __forceinline__ void load(const uint8_t* p, Raw<DTYPE>& b) {
  constexpr int kW = DTYPE == NVFP4_DTYPE_BF16 ? 8 : 16;
#pragma unroll
  for (int i = 0; i < kW; i += 8) {
    if constexpr (WIDE) {
      ld_v8(p + 4 * i, b.w + i);
    } else {
      const uint4 a = __ldg(reinterpret_cast<const uint4*>(p + 4 * i));
      const uint4 c = __ldg(reinterpret_cast<const uint4*>(p + 4 * i + 16));
      b.w[i] = a.x; b.w[i + 1] = a.y; b.w[i + 2] = a.z; b.w[i + 3] = a.w;
      b.w[i + 4] = c.x; b.w[i + 5] = c.y; b.w[i + 6] = c.z; b.w[i + 7] = c.w;
    }
  }
}

template <int DTYPE>
__device__ __forceinline__ void to_f32(const Raw<DTYPE>& b, float (&v)[16]) {
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

__device__ __forceinline__ float e4m3_val(uint32_t b) {
  const uint32_t e = (b >> 3) & 15u, m = b & 7u;
  return e ? __uint_as_float(((e + 120u) << 23) | (m << 20)) : static_cast<float>(m) * 0.001953125f;
}

// Packed FP32 pairs (sm_100 f32x2 arithmetic; every lane rounds like the
// scalar instruction).
__device__ __forceinline__ uint64_t pk(float a, float b) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(a), "f"(b));
  return r;
}
__device__ __forceinline__ float2 upk(uint64_t v) {
  float2 f;
  asm("mov.b64 {%0, %1}, %2;" : "=f"(f.x), "=f"(f.y) : "l"(v));
  return f;
}
__device__ __forceinline__ uint64_t mul2(uint64_t a, uint64_t b) {
  uint64_t r;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}
__device__ __forceinline__ uint64_t add2(uint64_t a, uint64_t b) {
  uint64_t r;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}
__device__ __forceinline__ uint64_t fma2(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t r;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(a), "l"(b), "l"(c));
  return r;
}

// E2M1 (satfinite, nearest even) of a pair of floats, returned as the pair of
// code values (exact; element a in .x).
__device__ __forceinline__ float2 e2m1_round2(float2 q) {
  uint32_t h2;
  asm("{\n\t.reg .b8 c;\n\tcvt.rn.satfinite.e2m1x2.f32 c, %2, %1;\n\tcvt.rn.f16x2.e2m1x2 %0, c;\n\t}"
      : "=r"(h2) : "f"(q.x), "f"(q.y));
  return __half22float2(*reinterpret_cast<const __half2*>(&h2));
}

__device__ __forceinline__ double warp_sum(double v) {
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
  return v;
}

// Sums over the warp of eight per-lane values in 9 shuffles (a reduce-scatter
// of halves, then a butterfly over groups of four lanes).  Afterwards every
// lane holds the total of value ((l >> 4) & 1) * 4 + ((l >> 3) & 1) * 2 +
// ((l >> 2) & 1), l its lane.
__device__ __forceinline__ float warp_sum8(const float (&v)[8], int lane) {
  const bool b4 = (lane & 16) != 0, b3 = (lane & 8) != 0, b2 = (lane & 4) != 0;
  float h4[4], h2[2];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float send = b4 ? v[i] : v[i + 4];
    h4[i] = (b4 ? v[i + 4] : v[i]) + __shfl_xor_sync(0xffffffffu, send, 16);
  }
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    const float send = b3 ? h4[i] : h4[i + 2];
    h2[i] = (b3 ? h4[i + 2] : h4[i]) + __shfl_xor_sync(0xffffffffu, send, 8);
  }
  float h1 = (b2 ? h2[1] : h2[0]) + __shfl_xor_sync(0xffffffffu, b2 ? h2[0] : h2[1], 4);
  h1 += __shfl_xor_sync(0xffffffffu, h1, 2);
  h1 += __shfl_xor_sync(0xffffffffu, h1, 1);
  return h1;
}

// Statistics of one lane's 16-element block of one row: moments, column
// accumulators, dominance, and the row's sum x^2 (rn2) and sum (x - x_hat)^2
// (re2).
template <int DTYPE>
__device__ __forceinline__ void block_stats(const Raw<DTYPE>& raw, bool quant, float g, float (&csq)[16],
                                            float (&cmx)[16], double& s1, double& s2, double& s3, double& s4,
                                            float& amax, double& blocks, double& dom, float& rn2, float& re2) {
  float v[16];
  to_f32<DTYPE>(raw, v);
  float am = 0.0f, asum = 0.0f;
  uint64_t p1 = 0, p2 = 0, p3 = 0, p4 = 0;  // packed even/odd partial sums
#pragma unroll
  for (int e = 0; e < 16; e += 2) {
    const uint64_t xv = pk(v[e], v[e + 1]);
    const uint64_t x2 = mul2(xv, xv);
    p1 = add2(p1, xv);
    p2 = add2(p2, x2);
    p3 = fma2(x2, xv, p3);
    p4 = fma2(x2, x2, p4);
    const float2 sq = upk(x2);
    csq[e] += sq.x;
    csq[e + 1] += sq.y;
    const float a0 = fabsf(v[e]), a1 = fabsf(v[e + 1]);
    cmx[e] = fmaxf(cmx[e], a0);
    cmx[e + 1] = fmaxf(cmx[e + 1], a1);
    am = fmaxf(am, fmaxf(a0, a1));
    asum += a0 + a1;
  }
  const float2 f1 = upk(p1), f2 = upk(p2), f3 = upk(p3), f4 = upk(p4);
  amax = fmaxf(amax, am);
  s1 += f1.x + f1.y; s2 += f2.x + f2.y; s3 += f3.x + f3.y; s4 += f4.x + f4.y;
  blocks += 1.0;
  // Dominated: am > (sum |x|) - am, decided in FP64 like the definition.  The
  // FP32 sum of 16 non-negative terms is within 2^-20 of the exact sum, so
  // outside a 2^-18 margin the FP32 comparison gives the same answer; inside
  // it the exact FP64 test runs.
  const float two_am = 2.0f * am;
  bool d;
  if (two_am > asum * (1.0f + 0x1p-18f)) {
    d = true;
  } else if (two_am < asum * (1.0f - 0x1p-18f)) {
    d = false;
  } else {
    double asum64 = 0.0;
#pragma unroll
    for (int e = 0; e < 16; ++e) asum64 += static_cast<double>(fabsf(v[e]));
    d = static_cast<double>(am) > asum64 - static_cast<double>(am);
  }
  if (d) dom += 1.0;
  rn2 = f2.x + f2.y;
  re2 = 0.0f;
  if (quant) {
    // the quantiser's arithmetic (block scale, reciprocal, codes)
    const float s = (am / 6.0f) / g;
    uint16_t sr;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(sr) : "f"(0.0f), "f"(s));
    const float S = e4m3_val(sr & 0xFFu);
    const float denom = S * g;
    float inv = denom > 0.0f ? 1.0f / denom : 0.0f;
    inv = fminf(inv, FLT_MAX);
    const uint64_t inv2 = pk(inv, inv), S2 = pk(S, S), g2 = pk(g, g);
    uint64_t e2 = 0;
#pragma unroll
    for (int e = 0; e < 16; e += 2) {
      const uint64_t xv = pk(v[e], v[e + 1]);
      const float2 c = e2m1_round2(upk(mul2(xv, inv2)));
      // x_hat = (e2m1 * S) * g, each product rounded on its own
      const uint64_t xh = mul2(mul2(pk(c.x, c.y), S2), g2);
      const uint64_t dd = add2(xv, xh ^ 0x8000000080000000ull);  // x - x_hat
      e2 = fma2(dd, dd, e2);
    }
    const float2 fe = upk(e2);
    re2 = fe.x + fe.y;
  }
}

template <int DTYPE, bool WIDE>
__global__ void __launch_bounds__(kThreads, 2) stats_kernel(const __grid_constant__ StatsArgs a) {
  constexpr int kEsz = DTYPE == NVFP4_DTYPE_BF16 ? 2 : 4;
  __shared__ double red[kWarps][8];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  grid_dependency_wait();
  if (threadIdx.x == 0) grid_launch_dependents();
  const float g = a.g != nullptr ? __ldg(a.g) : 0.0f;
  const bool quant = a.g != nullptr && g > 0.0f;
  double s1 = 0, s2 = 0, s3 = 0, s4 = 0, blocks = 0, dom = 0;
  float amax = 0.0f;
  const int64_t units = static_cast<int64_t>(a.cpr) * a.ranges;
  const int64_t nwarps = static_cast<int64_t>(gridDim.x) * kWarps;
  for (int64_t u = static_cast<int64_t>(blockIdx.x) * kWarps + warp; u < units; u += nwarps) {
    const int32_t strip = static_cast<int32_t>(u % a.cpr);
    const int32_t rr = static_cast<int32_t>(u / a.cpr);
    const int32_t r0 = static_cast<int32_t>(static_cast<int64_t>(a.M) * rr / a.ranges);
    const int32_t r1 = static_cast<int32_t>(static_cast<int64_t>(a.M) * (rr + 1) / a.ranges);
    const int32_t col = strip * 512 + lane * 16;
    const bool have = col < a.K;
    const uint8_t* xp = a.x + static_cast<int64_t>(col) * kEsz;
    float csq[16], cmx[16];
#pragma unroll
    for (int e = 0; e < 16; ++e) csq[e] = cmx[e] = 0.0f;
    // Rows stream in pairs through two register buffers: the loads of the
    // next pair are issued before the current pair is processed.  Every four
    // rows, their row sums are reduced together and added with one atomic
    // per lane group.
    Raw<DTYPE> ra[2], rb[2];
#pragma unroll
    for (int k = 0; k < 2; ++k)
      if (have && r0 + k < r1) load<DTYPE, WIDE>(xp + static_cast<int64_t>(r0 + k) * a.ld_bytes, ra[k]);
    for (int32_t row0 = r0; row0 < r1; row0 += 4) {
      float sums[8];
#pragma unroll
      for (int k = 0; k < 2; ++k)
        if (have && row0 + 2 + k < r1) load<DTYPE, WIDE>(xp + static_cast<int64_t>(row0 + 2 + k) * a.ld_bytes, rb[k]);
#pragma unroll
      for (int k = 0; k < 2; ++k) {
        sums[k] = sums[4 + k] = 0.0f;
        if (have && row0 + k < r1)
          block_stats<DTYPE>(ra[k], quant, g, csq, cmx, s1, s2, s3, s4, amax, blocks, dom, sums[k], sums[4 + k]);
      }
#pragma unroll
      for (int k = 0; k < 2; ++k)
        if (have && row0 + 4 + k < r1) load<DTYPE, WIDE>(xp + static_cast<int64_t>(row0 + 4 + k) * a.ld_bytes, ra[k]);
#pragma unroll
      for (int k = 0; k < 2; ++k) {
        sums[2 + k] = sums[6 + k] = 0.0f;
        if (have && row0 + 2 + k < r1)
          block_stats<DTYPE>(rb[k], quant, g, csq, cmx, s1, s2, s3, s4, amax, blocks, dom, sums[2 + k], sums[6 + k]);
      }
      const float total = warp_sum8(sums, lane);
      if ((lane & 3) == 0) {
        const int idx = (lane >> 2) & 7;
        const int32_t row = row0 + (idx & 3);
        if (row < r1) {
          if (idx < 4) {
            if (a.row_norm2 != nullptr) atomicAdd(a.row_norm2 + row, total);
          } else if (a.row_err2 != nullptr && quant) {
            atomicAdd(a.row_err2 + row, total);
          }
        }
      }
    }
    if (have) {
#pragma unroll
      for (int e = 0; e < 16; ++e) {
        if (a.col_sq != nullptr) atomicAdd(a.col_sq + col + e, csq[e]);
        if (a.col_max != nullptr) atomicMax(reinterpret_cast<unsigned int*>(a.col_max) + col + e, __float_as_uint(cmx[e]));
      }
    }
  }
  // block reduction of the moments, then one atomic each
  double m[7] = {s1, s2, s3, s4, static_cast<double>(amax), blocks, dom};
#pragma unroll
  for (int i = 0; i < 7; ++i) {
    if (i == 4) {
      double v = m[i];
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) v = fmax(v, __shfl_xor_sync(0xffffffffu, v, off));
      m[i] = v;
    } else {
      m[i] = warp_sum(m[i]);
    }
    if (lane == 0) red[warp][i] = m[i];
  }
  __syncthreads();
  if (threadIdx.x < 7) {
    const int i = threadIdx.x;
    double v = red[0][i];
    for (int w = 1; w < kWarps; ++w) v = i == 4 ? fmax(v, red[w][i]) : v + red[w][i];
    if (i == 4) {
      atomicMax(reinterpret_cast<unsigned long long*>(a.moments + 4), static_cast<unsigned long long>(__double_as_longlong(v)));
    } else {
      atomicAdd(a.moments + (i < 4 ? i : i + 1), v);
    }
  }
  if (threadIdx.x == 0) {
    double nb = 0.0;
    for (int w = 0; w < kWarps; ++w) nb += red[w][5];
    atomicAdd(a.moments + 5, 16.0 * nb);  // elements = 16 per block
  }
}

// Derived figures of the accumulators above, on the device (one block):
//   out[0] max/RMS = max|x| / sqrt(sum x^2 / n)
//   out[1] kurtosis = fourth central moment / variance^2, from the four raw
//          moments: E x^4 - 4 mu E x^3 + 6 mu^2 E x^2 - 3 mu^4 over
//          (E x^2 - mu^2)^2
//   out[2] dominated share = dominated blocks / blocks
//   out[3..5] per-token A4 error sqrt(row_err2) / sqrt(row_norm2) (a row with
//          zero norm divides by 1): mean, min, max over the M rows (NaN when
//          row_err2 is not given)
//   out[6] hot-channel ratio = largest channel RMS / median channel RMS,
//          channel RMS = sqrt(col_sq / M); the median of an even count is the
//          mean of the two middle values
//   out[7] the median channel RMS
// All arithmetic is FP64, with every product and sum rounded on its own (no
// fused multiply-add), in the order written above.  The two middle channel
// values are found by radix selection on the FP32 bit patterns (col_sq is
// non-negative, so its bit patterns order like its values).
constexpr int kSumThreads = 1024;

__device__ __forceinline__ double dmul(double a, double b) { return __dmul_rn(a, b); }
__device__ __forceinline__ double dadd(double a, double b) { return __dadd_rn(a, b); }
__device__ __forceinline__ double dsub(double a, double b) { return __dsub_rn(a, b); }

__global__ void __launch_bounds__(kSumThreads, 1)
    summary_kernel(const double* __restrict__ moments, const float* __restrict__ row_err2,
                   const float* __restrict__ row_norm2, int64_t M, const float* __restrict__ col_sq, int64_t K,
                   double* __restrict__ out) {
  __shared__ double red_sum[kSumThreads / 32], red_min[kSumThreads / 32], red_max[kSumThreads / 32];
  __shared__ uint32_t red_cmax[kSumThreads / 32];
  __shared__ uint32_t hist[2][256];
  __shared__ uint32_t sel_prefix[2], sel_rank[2];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  grid_dependency_wait();  // the accumulators come from the kernel before this one
  if (tid == 0) grid_launch_dependents();

  // per-token A4 error: sum, min, max over the rows (FP64)
  double esum = 0.0, emin = INFINITY, emax = -INFINITY;
  if (row_err2 != nullptr) {
    for (int64_t r = tid; r < M; r += kSumThreads) {
      const double nrm = __dsqrt_rn(static_cast<double>(row_norm2[r]));
      const double e = __ddiv_rn(__dsqrt_rn(static_cast<double>(row_err2[r])), nrm > 0.0 ? nrm : 1.0);
      esum = dadd(esum, e);
      emin = fmin(emin, e);
      emax = fmax(emax, e);
    }
  }
  // largest column sum of squares (bit patterns order like the values)
  uint32_t cmax = 0;
  for (int64_t c = tid; c < K; c += kSumThreads) cmax = max(cmax, __float_as_uint(col_sq[c]));
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) {
    esum = dadd(esum, __shfl_xor_sync(0xffffffffu, esum, off));
    emin = fmin(emin, __shfl_xor_sync(0xffffffffu, emin, off));
    emax = fmax(emax, __shfl_xor_sync(0xffffffffu, emax, off));
    cmax = max(cmax, __shfl_xor_sync(0xffffffffu, cmax, off));
  }
  if (lane == 0) {
    red_sum[warp] = esum;
    red_min[warp] = emin;
    red_max[warp] = emax;
    red_cmax[warp] = cmax;
  }
  // radix selection of ranks (K-1)/2 and K/2 of col_sq, 8 bits per pass
  if (tid < 2) {
    sel_prefix[tid] = 0;
    sel_rank[tid] = static_cast<uint32_t>(tid == 0 ? (K - 1) / 2 : K / 2);
  }
  for (int shift = 24; shift >= 0; shift -= 8) {
    for (int i = tid; i < 512; i += kSumThreads) hist[i >> 8][i & 255] = 0;
    __syncthreads();
    const uint32_t hi_mask = shift == 24 ? 0u : (0xFFFFFFFFu << (shift + 8));
    const uint32_t p0 = sel_prefix[0], p1 = sel_prefix[1];
    for (int64_t c = tid; c < K; c += kSumThreads) {
      const uint32_t key = __float_as_uint(col_sq[c]);
      const uint32_t digit = (key >> shift) & 255u;
      if ((key & hi_mask) == p0) atomicAdd(&hist[0][digit], 1u);
      if ((key & hi_mask) == p1) atomicAdd(&hist[1][digit], 1u);
    }
    __syncthreads();
    if (tid < 2) {
      uint32_t k = sel_rank[tid], d = 0;
      for (; d < 255; ++d) {
        const uint32_t h = hist[tid][d];
        if (k < h) break;
        k -= h;
      }
      sel_rank[tid] = k;
      sel_prefix[tid] |= d << shift;
    }
    __syncthreads();
  }
  if (warp == 0) {
    const int nw = kSumThreads / 32;
    double s = lane < nw ? red_sum[lane] : 0.0;
    double lo = lane < nw ? red_min[lane] : INFINITY;
    double hi = lane < nw ? red_max[lane] : -INFINITY;
    uint32_t cm = lane < nw ? red_cmax[lane] : 0u;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
      s = dadd(s, __shfl_xor_sync(0xffffffffu, s, off));
      lo = fmin(lo, __shfl_xor_sync(0xffffffffu, lo, off));
      hi = fmax(hi, __shfl_xor_sync(0xffffffffu, hi, off));
      cm = max(cm, __shfl_xor_sync(0xffffffffu, cm, off));
    }
    if (lane == 0) {
      const double n = moments[5];
      const double mean = __ddiv_rn(moments[0], n);
      const double m2 = __ddiv_rn(moments[1], n);
      const double mean2 = dmul(mean, mean);
      const double var = dsub(m2, mean2);
      double m4c = dsub(__ddiv_rn(moments[3], n), __ddiv_rn(dmul(dmul(4.0, mean), moments[2]), n));
      m4c = dadd(m4c, dmul(dmul(6.0, mean2), m2));
      m4c = dsub(m4c, dmul(3.0, dmul(mean2, mean2)));
      out[0] = m2 > 0.0 ? __ddiv_rn(moments[4], __dsqrt_rn(m2)) : 0.0;
      out[1] = var > 0.0 ? __ddiv_rn(m4c, dmul(var, var)) : 0.0;
      out[2] = moments[6] != 0.0 ? __ddiv_rn(moments[7], moments[6]) : 0.0;
      const bool have_err = row_err2 != nullptr && M > 0;
      out[3] = have_err ? __ddiv_rn(s, static_cast<double>(M)) : __longlong_as_double(0x7FF8000000000000ll);
      out[4] = have_err ? lo : __longlong_as_double(0x7FF8000000000000ll);
      out[5] = have_err ? hi : __longlong_as_double(0x7FF8000000000000ll);
      const double inv_rows = M > 0 ? __ddiv_rn(1.0, static_cast<double>(M)) : 1.0;
      const double r_lo = __dsqrt_rn(dmul(static_cast<double>(__uint_as_float(sel_prefix[0])), inv_rows));
      const double r_hi = __dsqrt_rn(dmul(static_cast<double>(__uint_as_float(sel_prefix[1])), inv_rows));
      const double med = K > 0 ? __ddiv_rn(dadd(r_lo, r_hi), 2.0) : 0.0;
      const double rmax = __dsqrt_rn(dmul(static_cast<double>(__uint_as_float(cm)), inv_rows));
      out[6] = med > 0.0 ? __ddiv_rn(rmax, med) : 0.0;
      out[7] = med;
    }
  }
}

int sm_count() {
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  return sms;
}

}  // namespace st

cudaError_t launch_act_stats(const void* x, int dtype, int64_t M, int64_t K, int64_t ld, const float* g,
                             double* moments, float* row_err2, float* row_norm2, float* col_sq, float* col_max,
                             cudaStream_t stream) {
  using namespace st;
  if (M == 0) return cudaSuccess;
  StatsArgs a{};
  const int esz = dtype == NVFP4_DTYPE_BF16 ? 2 : 4;
  a.x = static_cast<const uint8_t*>(x);
  a.ld_bytes = ld * esz;
  a.M = static_cast<int32_t>(M);
  a.K = static_cast<int32_t>(K);
  a.cpr = static_cast<int32_t>(ceil_div(K, 512));
  const int64_t blocks = static_cast<int64_t>(sm_count()) * 2;
  const int64_t warps = blocks * kWarps;
  int64_t ranges = warps / a.cpr;
  if (ranges < 1) ranges = 1;
  if (ranges > M) ranges = M;
  a.ranges = static_cast<int32_t>(ranges);
  a.g = g;
  a.moments = moments;
  a.row_err2 = row_err2;
  a.row_norm2 = row_norm2;
  a.col_sq = col_sq;
  a.col_max = col_max;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(blocks));
  cfg.blockDim = dim3(kThreads);
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  const bool wide = (reinterpret_cast<uintptr_t>(x) % 32 == 0) && (a.ld_bytes % 32 == 0);
  if (dtype == NVFP4_DTYPE_BF16)
    return wide ? cudaLaunchKernelEx(&cfg, stats_kernel<NVFP4_DTYPE_BF16, true>, a)
                : cudaLaunchKernelEx(&cfg, stats_kernel<NVFP4_DTYPE_BF16, false>, a);
  return wide ? cudaLaunchKernelEx(&cfg, stats_kernel<NVFP4_DTYPE_F32, true>, a)
              : cudaLaunchKernelEx(&cfg, stats_kernel<NVFP4_DTYPE_F32, false>, a);
}

cudaError_t launch_act_summary(const double* moments, const float* row_err2, const float* row_norm2, int64_t M,
                               const float* col_sq, int64_t K, double* out, cudaStream_t stream) {
  using namespace st;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(1);
  cfg.blockDim = dim3(kSumThreads);
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, summary_kernel, moments, row_err2, row_norm2, M, col_sq, K, out);
}

}  // namespace nvfp4
