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
// HBM-bound design.  The work item is a chunk of 512 consecutive elements of
// one row; lane l of a warp owns 16-element block l of a chunk (one 256-bit
// load for BF16), so the block amax, scale and codes need no cross-lane
// traffic.  Each lane stores its 16 codes as 8 contiguous bytes (a warp writes
// 256 bytes), and four lanes' scale bytes are gathered by shuffles into one
// 32-bit word of the tcgen05 block-scale layout; layout padding (rows up to
// 128, K/16 up to a multiple of 4) is written with zeros.
//
// Large inputs: one block per SM owns a contiguous, balanced range of chunks;
// its 32 warps read it with 256-bit loads straight into registers (several
// chunks in flight per warp; at each step the block's warps cover 32
// consecutive chunks).  A device-computed scale takes two launches: the amax
// kernel stores one maximum per block and segment (plain stores, so no
// scratch clearing) and the quantise kernel reduces them first.  Both are
// launched with programmatic stream serialization and wait
// (griddepcontrol.wait) before they touch global memory, so launch and
// prologue overlap the kernel before.  The quantise kernel walks its range
// backwards, so that when x is larger than L2 it starts on the chunks the
// amax kernel read last.
//
// Small inputs with a device-computed scale (up to 512 chunks, 256 K
// elements: a decode step's activations): one launch of a cluster of up to 8
// small blocks; each block takes the amax of its share with register loads,
// the blocks exchange their maxima through distributed shared memory, and
// each quantises its share reading x again from L2.
#include <cfloat>
#include <cstdint>

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include "internal.h"
#include "ptx.cuh"

namespace nvfp4 {
namespace qk {

constexpr int kChunk = 512;  // elements per chunk (32 lanes x 16)
constexpr int kWarps = 32;   // warps per block
constexpr int kThreads = kWarps * 32;
constexpr int kUnrollQ = 2;  // chunks in flight per warp, quantise kernel

template <int DTYPE>
struct Cfg {
  static constexpr int kEsz = DTYPE == NVFP4_DTYPE_BF16 ? 2 : 4;
  static constexpr int kChunkBytes = kChunk * kEsz;
  static constexpr int kWords = DTYPE == NVFP4_DTYPE_BF16 ? 8 : 16;  // per lane
  static constexpr int kUnrollA = DTYPE == NVFP4_DTYPE_BF16 ? 4 : 2;  // chunks in flight per warp, amax
};

struct QuantArgs {
  const uint8_t* x;
  int64_t ld_bytes;
  int32_t M, K, rows_pad, cpr;  // cpr: chunks per row
  int64_t items;                // M * cpr (< 2^30)
  uint64_t cpr_inv;             // ceil(2^64 / cpr) (0 when cpr == 1): row = mulhi(item, cpr_inv)
  int nseg;
  int32_t seg_begin[kMaxSeg + 1];
  const float* g_in;    // given scales, or nullptr
  float* partial;       // [amax_blocks][nseg] per-block maxima (device-computed scale)
  int amax_blocks;
  float* g_out;
  uint8_t* codes;
  uint8_t* sf;
};

// The raw 16 elements of one lane: 8 words (BF16) or 16 words (F32).
template <int DTYPE>
struct Blk {
  uint32_t w[Cfg<DTYPE>::kWords];
};

__device__ __forceinline__ void ld_v8(const void* p, uint32_t* r) {
  asm volatile("ld.global.nc.L1::no_allocate.v8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]),
                 "=r"(r[6]), "=r"(r[7])
               : "l"(p));
}
__device__ __forceinline__ void ld_v4(const void* p, uint32_t* r) {
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "l"(p));
}

// From global memory; WIDE: 32-byte aligned, so 256-bit loads.
template <int DTYPE, bool WIDE>
__device__ __forceinline__ void load_global(const uint8_t* p, Blk<DTYPE>& b) {
  constexpr int kW = Cfg<DTYPE>::kWords;
#pragma unroll
  for (int i = 0; i < kW; i += 8) {
    if constexpr (WIDE) {
      ld_v8(p + 4 * i, b.w + i);
    } else {
      ld_v4(p + 4 * i, b.w + i);
      ld_v4(p + 4 * i + 16, b.w + i + 4);
    }
  }
}

// From shared memory (16-byte aligned).
template <int DTYPE>
__device__ __forceinline__ void load_shared(const uint8_t* p, Blk<DTYPE>& b) {
  constexpr int kW = Cfg<DTYPE>::kWords;
#pragma unroll
  for (int i = 0; i < kW; i += 4) {
    const uint4 v = *reinterpret_cast<const uint4*>(p + 4 * i);
    b.w[i] = v.x;
    b.w[i + 1] = v.y;
    b.w[i + 2] = v.z;
    b.w[i + 3] = v.w;
  }
}

// max |x| of the block.  BF16: the magnitudes' bit patterns order like their
// values (finite inputs), so a packed 16-bit integer max gives the exact
// maximum.
template <int DTYPE>
__device__ __forceinline__ float block_amax(const Blk<DTYPE>& b) {
  if constexpr (DTYPE == NVFP4_DTYPE_BF16) {
    uint32_t m = 0;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      uint32_t r;
      asm("max.u16x2 %0, %1, %2;" : "=r"(r) : "r"(m), "r"(b.w[i] & 0x7FFF7FFFu));
      m = r;
    }
    const uint32_t hi = m >> 16, lo = m & 0xFFFFu;
    return __uint_as_float((hi > lo ? hi : lo) << 16);
  } else {
    float m = 0.0f;
#pragma unroll
    for (int i = 0; i < 16; ++i) m = fmaxf(m, fabsf(__uint_as_float(b.w[i])));
    return m;
  }
}

template <int DTYPE>
__device__ __forceinline__ void to_float(const Blk<DTYPE>& b, float (&v)[16]) {
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

// Packed FP32 multiply of a pair by s (sm_100 f32x2; each lane rounds to
// nearest even exactly as a scalar multiply does).
__device__ __forceinline__ void mul_f32x2(float& a0, float& a1, float s) {
  uint64_t x, y, k;
  asm("mov.b64 %0, {%1, %2};" : "=l"(x) : "f"(a0), "f"(a1));
  asm("mov.b64 %0, {%1, %1};" : "=l"(k) : "f"(s));
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(y) : "l"(x), "l"(k));
  asm("mov.b64 {%0, %1}, %2;" : "=f"(a0), "=f"(a1) : "l"(y));
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

// Row and first column of chunk `item` without a division: for 32-bit n and
// d, floor(n / d) is the high word of n * ceil(2^64 / d) (Lemire, Kaser and
// Kurz, "Faster remainder by direct computation", 2019).
__device__ __forceinline__ void chunk_pos(const QuantArgs& a, int64_t item, int32_t& row, int32_t& col0) {
  const uint64_t n = static_cast<uint64_t>(item);
  const uint32_t r = a.cpr == 1 ? static_cast<uint32_t>(n) : static_cast<uint32_t>(__umul64hi(a.cpr_inv, n));
  row = static_cast<int32_t>(r);
  col0 = (static_cast<int32_t>(n) - static_cast<int32_t>(r) * a.cpr) * kChunk;
}

__device__ __forceinline__ int find_segment(const QuantArgs& a, int32_t row) {
  int s = 0;
#pragma unroll
  for (int i = 1; i < kMaxSeg; ++i)
    if (i < a.nseg && row >= a.seg_begin[i]) s = i;
  return s;
}

__device__ __forceinline__ void block_range(int64_t items, int64_t& lo, int64_t& hi) {
  lo = items * blockIdx.x / gridDim.x;
  hi = items * (blockIdx.x + 1) / gridDim.x;
}

// Running per-segment maxima of one lane, kept in registers.
struct SegMax {
  float m[kMaxSeg];
  __device__ __forceinline__ SegMax() {
#pragma unroll
    for (int s = 0; s < kMaxSeg; ++s) m[s] = 0.0f;
  }
  __device__ __forceinline__ void add(int seg, float v) {
#pragma unroll
    for (int s = 0; s < kMaxSeg; ++s)
      if (s == seg) m[s] = fmaxf(m[s], v);
  }
  // Block-wide maxima of segments [0, nseg): warp s returns segment s's
  // maximum in every lane (red: kWarps x kMaxSeg shared floats).
  __device__ __forceinline__ float reduce(int nseg, float (*red)[kMaxSeg]) const {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
#pragma unroll
    for (int s = 0; s < kMaxSeg; ++s) {
      if (s >= nseg) break;  // uniform
      float v = m[s];
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, off));
      if (lane == 0) red[warp][s] = v;
    }
    __syncthreads();
    float v = 0.0f;
    if (warp < nseg) {
      v = red[lane][warp];
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, off));
    }
    return v;
  }
};

// Codes and scale bytes of one lane's block of chunk `item` (all 32 lanes of
// a warp call it for the same chunk; `have` is false past K).
template <int DTYPE>
__device__ __forceinline__ void quantize_block(const QuantArgs& a, const float* g_sh, const Blk<DTYPE>& b,
                                               bool have, int32_t row, int32_t col) {
  const int lane = threadIdx.x & 31;
  const int32_t KA = (a.K + 63) / 64;
  const float g = g_sh[find_segment(a, row)];
  uint32_t sfb = 0;
  uint2 word = make_uint2(0u, 0u);
  if (have && g > 0.0f) {
    const float m = block_amax<DTYPE>(b);
    const float s = (m / 6.0f) / g;
    sfb = to_e4m3(s);
    const float denom = e4m3_value(sfb) * g;
    float inv = denom > 0.0f ? 1.0f / denom : 0.0f;
    inv = fminf(inv, FLT_MAX);
    float q[16];
    to_float<DTYPE>(b, q);
#pragma unroll
    for (int i = 0; i < 16; i += 2) mul_f32x2(q[i], q[i + 1], inv);
    word.x = to_e2m1x8(q);
    word.y = to_e2m1x8(q + 8);
  }
  if (have) *reinterpret_cast<uint2*>(a.codes + static_cast<int64_t>(row) * (a.K / 2) + col / 2) = word;
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

// Zero scale words of the layout's padding rows [M, rows_pad).  They all lie
// in the last 128-row block; word w (4 bytes) of a 512-byte atom holds row
// (w / 4) + 32 * (w % 4) of the block, so a warp walks an atom's 128 words in
// order (coalesced 128-byte stores) and writes those of padding rows.  Warps
// of the whole grid take atoms.
__device__ __forceinline__ void zero_padding_rows_n(const QuantArgs& a, int warps_per_block) {
  if (a.rows_pad == a.M) return;
  const int32_t KA = (a.K + 63) / 64;
  const int32_t rb = a.M >> 7;
  const int lane = threadIdx.x & 31;
  const int32_t gw = blockIdx.x * warps_per_block + (threadIdx.x >> 5), nw = gridDim.x * warps_per_block;
  for (int32_t kb = gw; kb < KA; kb += nw) {
    uint32_t* atom = reinterpret_cast<uint32_t*>(a.sf + (static_cast<int64_t>(rb) * KA + kb) * 512);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int w = lane + 32 * i;
      if (rb * 128 + (w >> 2) + 32 * (w & 3) >= a.M) atom[w] = 0u;
    }
  }
}

__device__ __forceinline__ void zero_padding_rows(const QuantArgs& a) { zero_padding_rows_n(a, kWarps); }

// Pass 1 (device-computed scale): per-segment amax of the block's chunks,
// stored to partial[block][segment].
template <int DTYPE, bool WIDE>
__global__ void __launch_bounds__(kThreads, 1) amax_kernel(const __grid_constant__ QuantArgs a) {
  using C = Cfg<DTYPE>;
  __shared__ float red[kWarps][kMaxSeg];
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  grid_dependency_wait();  // x may come from the kernel before this one
  if (threadIdx.x == 0) grid_launch_dependents();
  int64_t lo, hi;
  block_range(a.items, lo, hi);
  SegMax sm;
  constexpr int kUnrollA = C::kUnrollA;
  for (int64_t base = lo; base < hi; base += kWarps * kUnrollA) {
    Blk<DTYPE> b[kUnrollA];
    int32_t rows[kUnrollA];
    bool act[kUnrollA];
#pragma unroll
    for (int u = 0; u < kUnrollA; ++u) {
      const int64_t item = base + u * kWarps + warp;
      act[u] = false;
      rows[u] = 0;
      if (item < hi) {
        int32_t col;
        chunk_pos(a, item, rows[u], col);
        col += lane * 16;
        act[u] = col < a.K;
        if (act[u]) load_global<DTYPE, WIDE>(a.x + rows[u] * a.ld_bytes + static_cast<int64_t>(col) * C::kEsz, b[u]);
      }
    }
#pragma unroll
    for (int u = 0; u < kUnrollA; ++u)
      if (act[u]) sm.add(find_segment(a, rows[u]), block_amax<DTYPE>(b[u]));
  }
  const float m = sm.reduce(a.nseg, red);
  if (warp < a.nseg && lane == 0) a.partial[blockIdx.x * a.nseg + warp] = m;
}

// Pass 2: global scale per segment (given, or the maximum of the amax
// kernel's partials / 2688), then the codes and scale bytes of rows [0, M)
// and zero scale words for the layout's padding rows [M, rows_pad).
template <int DTYPE, bool WIDE>
__global__ void __launch_bounds__(kThreads, 1) quant_kernel(const __grid_constant__ QuantArgs a) {
  using C = Cfg<DTYPE>;
  __shared__ float g_sh[kMaxSeg];
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  // Once every block of this grid has passed this point all of them are
  // resident, so a dependent kernel may start launching (it waits for this
  // grid's completion before touching what it writes).
  if (threadIdx.x == 0) grid_launch_dependents();
  grid_dependency_wait();
  if (a.g_in != nullptr) {
    if (threadIdx.x < a.nseg) g_sh[threadIdx.x] = a.g_in[threadIdx.x];
  } else if (warp < a.nseg) {
    float m = 0.0f;
    for (int b = lane; b < a.amax_blocks; b += 32) m = fmaxf(m, a.partial[b * a.nseg + warp]);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
    if (lane == 0) g_sh[warp] = m / 2688.0f;
  }
  __syncthreads();
  if (blockIdx.x == 0 && threadIdx.x < a.nseg) a.g_out[threadIdx.x] = g_sh[threadIdx.x];

  int64_t lo, hi;
  block_range(a.items, lo, hi);
  // backwards over the range, kWarps * kUnrollQ chunks per step
  for (int64_t end = hi; end > lo; end -= kWarps * kUnrollQ) {
    const int64_t base = end - kWarps * kUnrollQ > lo ? end - kWarps * kUnrollQ : lo;
    Blk<DTYPE> b[kUnrollQ];
    int32_t rows[kUnrollQ], cols[kUnrollQ];
    bool inr[kUnrollQ], act[kUnrollQ];
#pragma unroll
    for (int u = 0; u < kUnrollQ; ++u) {
      const int64_t item = base + u * kWarps + warp;
      inr[u] = item < end;
      act[u] = false;
      rows[u] = cols[u] = 0;
      if (inr[u]) {
        chunk_pos(a, item, rows[u], cols[u]);
        cols[u] += lane * 16;
        act[u] = cols[u] < a.K;
        if (act[u]) load_global<DTYPE, WIDE>(a.x + rows[u] * a.ld_bytes + static_cast<int64_t>(cols[u]) * C::kEsz, b[u]);
      }
    }
#pragma unroll
    for (int u = 0; u < kUnrollQ; ++u)
      if (inr[u]) quantize_block<DTYPE>(a, g_sh, b[u], act[u], rows[u], cols[u]);  // uniform across the warp
  }
  zero_padding_rows(a);
}

// Small inputs with a device-computed scale, in one launch: a cluster of C
// blocks (C <= 8) of 8 warps, as many as give each warp about one chunk (a
// decode token's row of 17408 elements is 34 chunks: 5 blocks).  (Eight
// blocks of 32 warps for up to 2560 chunks were slower than the two-launch
// path at 64 decode tokens, 17.8 against 6.3 us: eight SMs stream the input
// twice.)  Each block
// takes the amax of its share of x with register loads (up to kSmallUnroll
// chunks in flight per warp), reads the other blocks' maxima through
// distributed shared memory after a cluster barrier, and quantises its share,
// reading x again (it is a few hundred KB at most, and still in L2).  No
// shared-memory staging: the blocks need a few KB of shared memory and 256
// threads, so they can run beside the weight-streaming GEMM's CTAs of the
// layer before.
constexpr int kSmallWarps = 8;
constexpr int kSmallThreads = kSmallWarps * 32;
constexpr int kSmallChunksPerBlock = 64;  // the path takes up to 8 blocks of 64 chunks
constexpr int kMaxSmallBlocks = 8;
constexpr int kSmallUnroll = 4;

template <int DTYPE, bool WIDE>
__global__ void __launch_bounds__(kSmallThreads, 1) small_kernel(const __grid_constant__ QuantArgs a) {
  using C = Cfg<DTYPE>;
  __shared__ float red[kSmallWarps][kMaxSeg];
  __shared__ float blk_amax[kMaxSeg];
  __shared__ float g_sh[kMaxSeg];
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  if (threadIdx.x == 0) grid_launch_dependents();
  grid_dependency_wait();  // x may come from the kernel before this one
  int64_t lo, hi;
  block_range(a.items, lo, hi);
  SegMax sm;
  for (int64_t base = lo + warp; base < hi; base += kSmallWarps * kSmallUnroll) {
    Blk<DTYPE> b[kSmallUnroll];
    int32_t rows[kSmallUnroll];
    bool act[kSmallUnroll];
#pragma unroll
    for (int u = 0; u < kSmallUnroll; ++u) {  // every load before the first use
      const int64_t i = base + u * kSmallWarps;
      int32_t col = 0;
      rows[u] = 0;
      act[u] = false;
      if (i < hi) {
        chunk_pos(a, i, rows[u], col);
        col += lane * 16;
        act[u] = col < a.K;
        if (act[u]) load_global<DTYPE, WIDE>(a.x + rows[u] * a.ld_bytes + static_cast<int64_t>(col) * C::kEsz, b[u]);
      }
    }
#pragma unroll
    for (int u = 0; u < kSmallUnroll; ++u)
      if (act[u]) sm.add(find_segment(a, rows[u]), block_amax<DTYPE>(b[u]));
  }
  // block maxima per segment: warp-reduce, then warp s combines segment s
#pragma unroll
  for (int s = 0; s < kMaxSeg; ++s) {
    if (s >= a.nseg) break;  // uniform
    float v = sm.m[s];
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, off));
    if (lane == 0) red[warp][s] = v;
  }
  __syncthreads();
  if (threadIdx.x < a.nseg) {
    float v = 0.0f;
#pragma unroll
    for (int w = 0; w < kSmallWarps; ++w) v = fmaxf(v, red[w][threadIdx.x]);
    blk_amax[threadIdx.x] = v;
  }
  cluster_sync_all();  // every block's maxima are visible to the cluster
  if (threadIdx.x < a.nseg) {
    float v = 0.0f;
    for (uint32_t rk = 0; rk < gridDim.x; ++rk)
      v = fmaxf(v, ld_shared_cluster_f32(map_to_rank(smem_u32(&blk_amax[threadIdx.x]), rk)));
    g_sh[threadIdx.x] = v / 2688.0f;
  }
  __syncthreads();
  if (blockIdx.x == 0 && threadIdx.x < a.nseg) a.g_out[threadIdx.x] = g_sh[threadIdx.x];
  for (int64_t base = lo + warp; base < hi; base += kSmallWarps * kSmallUnroll) {
    Blk<DTYPE> b[kSmallUnroll];
    int32_t rows[kSmallUnroll], cols[kSmallUnroll];
    bool inr[kSmallUnroll], have[kSmallUnroll];
#pragma unroll
    for (int u = 0; u < kSmallUnroll; ++u) {  // every load before the first use
      const int64_t i = base + u * kSmallWarps;
      inr[u] = i < hi;
      have[u] = false;
      rows[u] = cols[u] = 0;
      if (inr[u]) {
        chunk_pos(a, i, rows[u], cols[u]);
        cols[u] += lane * 16;
        have[u] = cols[u] < a.K;
        if (have[u])
          load_global<DTYPE, WIDE>(a.x + rows[u] * a.ld_bytes + static_cast<int64_t>(cols[u]) * C::kEsz, b[u]);
      }
    }
#pragma unroll
    for (int u = 0; u < kSmallUnroll; ++u)
      if (inr[u]) quantize_block<DTYPE>(a, g_sh, b[u], have[u], rows[u], cols[u]);  // uniform across the warp
  }
  zero_padding_rows_n(a, kSmallWarps);
  cluster_sync_all();  // no block leaves while another may read its maxima
}

// Checkpoint-side harmonisation: re-encode an NVFP4 operand whose row ranges
// (modules) carry their own global scales under one common scale.  Each
// element is dequantised with its module's scale and rounded once to FP32
// (x_hat = e2m1 * S * g_old; e2m1 * S is exact), then quantised exactly as
// the quantiser does.  The common scale is given, or the largest module
// scale (the fused tensor's scale, which clips no block).  Works in place:
// a lane reads its 8 code bytes and its scale byte before the warp writes.
struct RequantArgs {
  QuantArgs q;                 // output side: one segment, the common scale
  const uint8_t* in_codes;
  const uint8_t* in_sf;
  const float* g_old;          // device [nseg_old]
  const float* g_new;          // device [1] or nullptr
  int nseg_old;
  int32_t old_begin[kMaxSeg + 1];
};

__global__ void __launch_bounds__(kThreads, 1) requant_kernel(const __grid_constant__ RequantArgs r) {
  const QuantArgs& a = r.q;
  __shared__ float g_sh[kMaxSeg];
  __shared__ float g_old_sh[kMaxSeg];
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  if (threadIdx.x == 0) grid_launch_dependents();
  grid_dependency_wait();
  if (threadIdx.x < r.nseg_old) g_old_sh[threadIdx.x] = r.g_old[threadIdx.x];
  if (threadIdx.x == 0) {
    float g = 0.0f;
    if (r.g_new != nullptr) {
      g = *r.g_new;
    } else {
      for (int i = 0; i < r.nseg_old; ++i) g = fmaxf(g, r.g_old[i]);
    }
    g_sh[0] = g;
  }
  __syncthreads();
  if (blockIdx.x == 0 && threadIdx.x < r.nseg_old) a.g_out[threadIdx.x] = g_sh[0];
  const int32_t KA = (a.K + 63) / 64;
  constexpr int U = 4;  // chunks in flight per warp (9 bytes per lane each)
  int64_t lo, hi;
  block_range(a.items, lo, hi);
  for (int64_t base = lo; base < hi; base += kWarps * U) {
    uint2 c[U];
    uint32_t sfb[U];
    int32_t rows[U], cols[U];
    bool inr[U], have[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int64_t i = base + u * kWarps + warp;
      inr[u] = i < hi;
      have[u] = false;
      rows[u] = cols[u] = 0;
      if (inr[u]) {
        chunk_pos(a, i, rows[u], cols[u]);
        cols[u] += lane * 16;
        have[u] = cols[u] < a.K;
        if (have[u]) {
          const int32_t row = rows[u], col = cols[u], j = col / 16;
          c[u] = *reinterpret_cast<const uint2*>(r.in_codes + static_cast<int64_t>(row) * (a.K / 2) + col / 2);
          sfb[u] = r.in_sf[(static_cast<int64_t>(row >> 7) * KA + (j >> 2)) * 512 + (row & 31) * 16 +
                           ((row >> 5) & 3) * 4 + (j & 3)];
        }
      }
    }
    __syncwarp();  // in place: every lane has read all U chunks before any lane writes
#pragma unroll
    for (int u = 0; u < U; ++u) {
      if (!inr[u]) continue;  // uniform across the warp
      Blk<NVFP4_DTYPE_F32> b;
      if (have[u]) {
        int s = 0;
#pragma unroll
        for (int k = 1; k < kMaxSeg; ++k)
          if (k < r.nseg_old && rows[u] >= r.old_begin[k]) s = k;
        const float S = e4m3_value(sfb[u]), g = g_old_sh[s];
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          // two codes per byte -> an exact FP16 pair (element 2j in the low half)
          uint32_t h2[4];
          asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\tmov.b32 {b0, b1, b2, b3}, %4;\n\t"
              "cvt.rn.f16x2.e2m1x2 %0, b0;\n\tcvt.rn.f16x2.e2m1x2 %1, b1;\n\t"
              "cvt.rn.f16x2.e2m1x2 %2, b2;\n\tcvt.rn.f16x2.e2m1x2 %3, b3;\n\t}"
              : "=r"(h2[0]), "=r"(h2[1]), "=r"(h2[2]), "=r"(h2[3])
              : "r"(h ? c[u].y : c[u].x));
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&h2[q]));
            // e2m1 * S is exact; one rounding for the global scale
            b.w[8 * h + 2 * q] = __float_as_uint(__fmul_rn(f.x * S, g));
            b.w[8 * h + 2 * q + 1] = __float_as_uint(__fmul_rn(f.y * S, g));
          }
        }
      }
      quantize_block<NVFP4_DTYPE_F32>(a, g_sh, b, have[u], rows[u], cols[u]);
    }
  }
  zero_padding_rows(a);
}

int num_sms() {
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  return sms;
}

// One block per SM (at most kMaxAmaxBlocks), at least 32 chunks per block.
int grid_for(int64_t items) {
  int64_t g = (items + kWarps - 1) / kWarps;
  const int sms = num_sms();
  const int64_t cap = sms < kMaxAmaxBlocks ? sms : kMaxAmaxBlocks;
  if (g > cap) g = cap;
  return g < 1 ? 1 : static_cast<int>(g);
}

template <class Kern>
cudaError_t launch_pdl(Kern kern, int grid, int cluster, int smem, const QuantArgs& a, cudaStream_t stream,
                       int threads = kThreads) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(threads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  attr[1].id = cudaLaunchAttributeClusterDimension;
  attr[1].val.clusterDim.x = cluster;
  attr[1].val.clusterDim.y = 1;
  attr[1].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = cluster > 1 ? 2 : 1;
  return cudaLaunchKernelEx(&cfg, kern, a);
}

template <int DTYPE, bool WIDE>
cudaError_t launch_t(QuantArgs a, bool dynamic, cudaStream_t stream) {
  const int64_t nsmall = (a.items + kSmallChunksPerBlock - 1) / kSmallChunksPerBlock;
  if (dynamic && nsmall <= kMaxSmallBlocks) {
    // about one chunk per warp, up to kMaxSmallBlocks blocks
    int64_t nb = (a.items + kSmallWarps - 1) / kSmallWarps;
    if (nb > kMaxSmallBlocks) nb = kMaxSmallBlocks;
    const int blocks = nb < 1 ? 1 : static_cast<int>(nb);
    return launch_pdl(small_kernel<DTYPE, WIDE>, blocks, blocks, 0, a, stream, kSmallThreads);
  }
  const int grid = grid_for(a.items);
  if (dynamic) {
    a.amax_blocks = grid;
    cudaError_t e = launch_pdl(amax_kernel<DTYPE, WIDE>, grid, 1, 0, a, stream);
    if (e != cudaSuccess) return e;
  }
  return launch_pdl(quant_kernel<DTYPE, WIDE>, grid, 1, 0, a, stream);
}

}  // namespace qk

size_t quantize_scratch_bytes(int nseg) { return static_cast<size_t>(kMaxAmaxBlocks) * nseg * sizeof(float); }

cudaError_t launch_requantize(const uint8_t* codes, const uint8_t* sf, int64_t N, int64_t K,
                              const RowSegments& segs, const float* g_old, const float* g_new,
                              uint8_t* codes_out, uint8_t* sf_out, float* g_out, cudaStream_t stream) {
  using namespace qk;
  RequantArgs r{};
  QuantArgs& a = r.q;
  a.M = static_cast<int32_t>(N);
  a.K = static_cast<int32_t>(K);
  a.rows_pad = static_cast<int32_t>(ceil_div(N, 128) * 128);
  a.cpr = static_cast<int32_t>(ceil_div(K, kChunk));
  a.items = static_cast<int64_t>(a.M) * a.cpr;
  a.cpr_inv = a.cpr == 1 ? 0 : ~0ull / static_cast<uint64_t>(a.cpr) + 1;
  a.nseg = 1;
  for (int i = 0; i <= kMaxSeg; ++i) a.seg_begin[i] = i == 0 ? 0 : a.M;
  a.g_out = g_out;
  a.codes = codes_out;
  a.sf = sf_out;
  r.in_codes = codes;
  r.in_sf = sf;
  r.g_old = g_old;
  r.g_new = g_new;
  r.nseg_old = segs.n;
  for (int i = 0; i <= kMaxSeg; ++i)
    r.old_begin[i] = static_cast<int32_t>(i <= segs.n ? segs.begin[i] : segs.begin[segs.n]);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid_for(a.items));
  cfg.blockDim = dim3(kThreads);
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, requant_kernel, r);
}

cudaError_t launch_quantize(const void* x, int dtype, int64_t M, int64_t K, int64_t ld,
                            const RowSegments& segs, const float* g_in, void* ws,
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
  a.items = static_cast<int64_t>(a.M) * a.cpr;
  a.cpr_inv = a.cpr == 1 ? 0 : ~0ull / static_cast<uint64_t>(a.cpr) + 1;
  a.nseg = segs.n;
  for (int i = 0; i <= kMaxSeg; ++i)
    a.seg_begin[i] = static_cast<int32_t>(i <= segs.n ? segs.begin[i] : segs.begin[segs.n]);
  a.g_in = g_in;
  a.partial = static_cast<float*>(ws);
  a.g_out = g_out;
  a.codes = codes;
  a.sf = sf;
  const bool dynamic = g_in == nullptr;
  const bool wide = (reinterpret_cast<uintptr_t>(x) % 32 == 0) && (a.ld_bytes % 32 == 0);
  if (dtype == NVFP4_DTYPE_BF16)
    return wide ? launch_t<NVFP4_DTYPE_BF16, true>(a, dynamic, stream) : launch_t<NVFP4_DTYPE_BF16, false>(a, dynamic, stream);
  return wide ? launch_t<NVFP4_DTYPE_F32, true>(a, dynamic, stream) : launch_t<NVFP4_DTYPE_F32, false>(a, dynamic, stream);
}

}  // namespace nvfp4
