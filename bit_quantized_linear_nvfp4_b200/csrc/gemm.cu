// Block-scaled NVFP4 x NVFP4 GEMM with fused per-segment epilogues, sm_100a.
//
// Computes acc[m, n] = sum_k e2m1(a[m,k]) Sa[m,k/16] * e2m1(w[n,k]) Sw[n,k/16]
// in FP32 on the 5th-generation tensor cores ("Why Gated DeltaNet Survives
// 4-Bit Quantization", ai.info summary, "Methodology in Plain English": W4A4,
// E2M1 values with one E4M3 scale per 16 elements), then, per output column n
// of segment s, y = acc * g_a * g_w[s] ("Main Findings", fused-GEMM scaling
// bullet: each fused module keeps its own global scale) followed by the
// segment's epilogue (identity, sigmoid write strength, log-space decay
// -exp(A_log) * softplus(y + dt_bias), or SwiGLU; "Main Findings",
// gate-parameterisation bullets).
//
// Kernel shape: persistent, one CTA per SM, 320 threads.
//   warp 0      TMA producer: codes (128-byte swizzle) and scale atoms -> smem
//   warp 1      allocates TMEM; one lane issues tcgen05.cp (scales -> TMEM)
//               and tcgen05.mma ... kind::mxf4nvf4.block_scale into TMEM
//   warps 2..9  epilogue: tcgen05.ld TMEM -> registers, release TMEM, then
//               scale, nonlinearity, store
// Tile 128 x 256 (M x N), 256 K-elements (128 bytes per row) per stage,
// 4 stages.  Each stage is 4 MMAs of K = 64.
#include <cfloat>
#include <cstdint>
#include <cstdio>
#include <mutex>

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "internal.h"
#include "ptx.cuh"

namespace nvfp4 {
namespace gk {

constexpr int BM = 128;
constexpr int BN = 256;
constexpr int BK = 256;
constexpr int kStages = 4;
constexpr int kABytes = BM * BK / 2;     // 16 KB
constexpr int kBBytes = BN * BK / 2;     // 32 KB
constexpr int kSFABytes = BM * BK / 16;  // 2 KB
constexpr int kSFBBytes = BN * BK / 16;  // 4 KB
constexpr int kStageBytes = kABytes + kBBytes + kSFABytes + kSFBBytes;
constexpr int kNumEpiWarps = 8;
constexpr int kThreads = 64 + kNumEpiWarps * 32;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColAcc = 0, kColSFA = 256, kColSFB = 272;
constexpr int kSmemBytes = kStages * kStageBytes + 1024 /*align*/ + 256 /*barriers*/;
static_assert(kStageBytes % 1024 == 0, "stage buffers keep 1024-byte alignment");

struct KernelArgs {
  int64_t M, N, K;
  int num_m_blocks, num_n_blocks, num_k_stages, group_m;
  int swiglu;
  int64_t up_row0;  // SwiGLU: first W row of the up half
  int64_t n_out;    // SwiGLU: output width (= N / 2)
  const float* g_a;
  const float* seg_scale;
  int nseg;
  uint32_t tma_mask;  // bit s: segment s has an output tensor map (staged stores)
  EpiSegment seg[kMaxSeg];
};

// Output tensor maps of the segments for the staged epilogue (BF16): box 64
// columns x 16 rows (whole 128-byte lines, 128-byte swizzle) for the fused
// projections, 32 x 32 (64-byte rows, 64-byte swizzle) for SwiGLU, whose
// warps hold 32 output columns.
struct OutMaps {
  CUtensorMap m[kMaxSeg];
};

struct SharedTail {
  uint64_t full[kStages];
  uint64_t empty[kStages];
  uint64_t tmem_full;
  uint64_t tmem_empty;
  uint64_t drain;
  uint32_t tmem_base;
  int abort_flag;
};

__device__ __forceinline__ void tile_coords(const KernelArgs& a, int t, int& m_blk, int& n_blk) {
  const int per_group = a.group_m * a.num_n_blocks;
  const int grp = t / per_group;
  const int first_m = grp * a.group_m;
  int gm = a.num_m_blocks - first_m;
  if (gm > a.group_m) gm = a.group_m;
  const int r = t - grp * per_group;
  m_blk = first_m + r % gm;
  n_blk = r / gm;
}

__device__ __forceinline__ float sigmoid_f(float y) { return 1.0f / (1.0f + expf(-y)); }
__device__ __forceinline__ float softplus_f(float t) {
  return t > 0.0f ? t + log1pf(expf(-t)) : log1pf(expf(t));
}

__device__ __forceinline__ int seg_of(const KernelArgs& a, int64_t n) {
  int s = 0;
#pragma unroll
  for (int i = 1; i < kMaxSeg; ++i)
    if (i < a.nseg && n >= a.seg[i].n_begin) s = i;
  return s;
}

__device__ __forceinline__ float apply_epi(const EpiSegment& sg, float y, int64_t j) {
  switch (sg.kind) {
    case NVFP4_EPI_SIGMOID_F32:
      return sigmoid_f(y);
    case NVFP4_EPI_GDN_DECAY_F32:
      return -expf(__ldg(sg.a_log + j)) * softplus_f(y + __ldg(sg.dt_bias + j));
    default:
      return y;
  }
}

__device__ __forceinline__ bool epi_is_bf16(int kind) {
  return kind == NVFP4_EPI_IDENTITY_BF16 || kind == NVFP4_EPI_SWIGLU_GATE;
}

__device__ __forceinline__ void st_global_v8(void* p, const uint32_t* w) {
  asm volatile("st.global.v8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"l"(p), "r"(w[0]), "r"(w[1]),
               "r"(w[2]), "r"(w[3]), "r"(w[4]), "r"(w[5]), "r"(w[6]), "r"(w[7])
               : "memory");
}

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  const __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&v);
}

// Store 32 consecutive results of one row: columns n0 .. n0+31 (absolute W row index).
__device__ __forceinline__ void store_chunk(const KernelArgs& a, int64_t row, int64_t n0,
                                           const uint32_t (&r)[32]) {
  if (n0 >= a.N) return;
  const int s = seg_of(a, n0);
  const EpiSegment& sg = a.seg[s];
  const int64_t n_last = n0 + 31;
  const bool bf16 = epi_is_bf16(sg.kind);
  const int vec = bf16 ? 8 : 4;
  const bool uniform = n_last < sg.n_end && ((n0 - sg.n_begin) % vec) == 0;
  if (uniform) {
    const float scale = __ldg(a.g_a) * __ldg(a.seg_scale + s);
    const int64_t j0 = n0 - sg.n_begin;
    if (bf16) {
      __nv_bfloat16* dst = static_cast<__nv_bfloat16*>(sg.out) + row * sg.ld_out + j0;
      const bool wide = (reinterpret_cast<uintptr_t>(dst) & 31u) == 0;
#pragma unroll
      for (int g = 0; g < 2; ++g) {  // 16 values = one 32-byte sector per group
        uint32_t w[8];
#pragma unroll
        for (int i = 0; i < 8; ++i)
          w[i] = pack_bf16(__uint_as_float(r[16 * g + 2 * i]) * scale, __uint_as_float(r[16 * g + 2 * i + 1]) * scale);
        if (wide) {
          st_global_v8(dst + 16 * g, w);
        } else {
          *reinterpret_cast<uint4*>(dst + 16 * g) = make_uint4(w[0], w[1], w[2], w[3]);
          *reinterpret_cast<uint4*>(dst + 16 * g + 8) = make_uint4(w[4], w[5], w[6], w[7]);
        }
      }
    } else {
      float* dst = static_cast<float*>(sg.out) + row * sg.ld_out + j0;
      const bool wide = (reinterpret_cast<uintptr_t>(dst) & 31u) == 0;
#pragma unroll
      for (int g = 0; g < 4; ++g) {
        uint32_t w[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) w[i] = __float_as_uint(apply_epi(sg, __uint_as_float(r[8 * g + i]) * scale, j0 + 8 * g + i));
        if (wide) {
          st_global_v8(dst + 8 * g, w);
        } else {
          *reinterpret_cast<uint4*>(dst + 8 * g) = make_uint4(w[0], w[1], w[2], w[3]);
          *reinterpret_cast<uint4*>(dst + 8 * g + 4) = make_uint4(w[4], w[5], w[6], w[7]);
        }
      }
    }
    return;
  }
  // general path: column by column (segment boundaries, N tail, odd alignment)
  const float ga = __ldg(a.g_a);
#pragma unroll
  for (int j = 0; j < 32; ++j) {
    const int64_t n = n0 + j;
    if (n >= a.N) continue;
    const int sj = seg_of(a, n);
    const EpiSegment& q = a.seg[sj];
    const float y = __uint_as_float(r[j]) * (ga * __ldg(a.seg_scale + sj));
    const int64_t jj = n - q.n_begin;
    if (epi_is_bf16(q.kind))
      static_cast<__nv_bfloat16*>(q.out)[row * q.ld_out + jj] = __float2bfloat16_rn(y);
    else
      static_cast<float*>(q.out)[row * q.ld_out + jj] = apply_epi(q, y, jj);
  }
}

// SwiGLU: output columns o0 .. o0+31 from gate values rg and up values ru.
__device__ __forceinline__ void store_swiglu(const KernelArgs& a, int64_t row, int64_t o0,
                                             const uint32_t (&rg)[32], const uint32_t (&ru)[32]) {
  if (o0 >= a.n_out) return;
  const EpiSegment& sg = a.seg[0];
  const float ga = __ldg(a.g_a);
  const float sgate = ga * __ldg(a.seg_scale + 0);
  const float sup = ga * __ldg(a.seg_scale + 1);
  // silu(g) * u = g * sigmoid(g) * u.  The result is rounded to BF16 (8-bit
  // mantissa), so the fast exponential (a few FP32 ulp) and a correctly
  // rounded reciprocal are ample; 1 / (1 + e^-g) stays correct at both ends
  // (e^-g overflowing to inf gives 0).
  float v[32];
#pragma unroll
  for (int j = 0; j < 32; ++j) {
    const float gv = __uint_as_float(rg[j]) * sgate;
    const float uv = __uint_as_float(ru[j]) * sup;
    v[j] = gv * __frcp_rn(1.0f + __expf(-gv)) * uv;
  }
  __nv_bfloat16* dst = static_cast<__nv_bfloat16*>(sg.out) + row * sg.ld_out + o0;
  if (o0 + 31 < a.n_out && (o0 % 8) == 0) {
    uint32_t w[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) w[i] = pack_bf16(v[2 * i], v[2 * i + 1]);
    if ((reinterpret_cast<uintptr_t>(dst) & 31u) == 0) {
      st_global_v8(dst, w);
      st_global_v8(dst + 16, w + 8);
    } else {
#pragma unroll
      for (int q = 0; q < 4; ++q)
        *reinterpret_cast<uint4*>(dst + 8 * q) = make_uint4(w[4 * q], w[4 * q + 1], w[4 * q + 2], w[4 * q + 3]);
    }
  } else {
#pragma unroll
    for (int j = 0; j < 32; ++j)
      if (o0 + j < a.n_out) dst[j] = __float2bfloat16_rn(v[j]);
  }
}

__global__ void __launch_bounds__(kThreads, 1)
    gemm_kernel(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_b,
                const __grid_constant__ CUtensorMap tm_sfa, const __grid_constant__ CUtensorMap tm_sfb,
                const __grid_constant__ KernelArgs args) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  SharedTail* tail = reinterpret_cast<SharedTail*>(smem + kStages * kStageBytes);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int num_tiles = args.num_m_blocks * args.num_n_blocks;
  volatile int* abort_flag = &tail->abort_flag;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&tail->full[s], 1);
      mbar_init(&tail->empty[s], 1);
    }
    mbar_init(&tail->tmem_full, 1);
    mbar_init(&tail->tmem_empty, kNumEpiWarps);
    mbar_init(&tail->drain, 1);
    tail->abort_flag = 0;
    fence_mbarrier_init();
    prefetch_tmap(&tm_a);
    prefetch_tmap(&tm_b);
    prefetch_tmap(&tm_sfa);
    prefetch_tmap(&tm_sfb);
  }
  if (warp == 1) {
    tmem_alloc(&tail->tmem_base, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tail->tmem_base;
  // Everything above may overlap the previous kernel on the stream; operands,
  // scales and outputs are touched only after the wait (the MMA warp reads
  // shared memory and TMEM only).
  if (warp != 1) grid_dependency_wait();
  if (threadIdx.x == 0) grid_launch_dependents();

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (elect_one()) {
      int stage = 0;
      uint32_t phase = 0;
      uint32_t issued_phase[kStages];
      bool issued[kStages];
      for (int s = 0; s < kStages; ++s) issued[s] = false;
      bool ok = true;
      for (int t = blockIdx.x; t < num_tiles && ok; t += gridDim.x) {
        int m_blk, n_blk;
        tile_coords(args, t, m_blk, n_blk);
        const int64_t b_row0 = args.swiglu ? static_cast<int64_t>(n_blk) * 128 : static_cast<int64_t>(n_blk) * BN;
        const int64_t b_row1 = args.swiglu ? args.up_row0 + static_cast<int64_t>(n_blk) * 128 : b_row0 + 128;
        for (int ks = 0; ks < args.num_k_stages; ++ks) {
          if (!mbar_wait_bounded(&tail->empty[stage], phase ^ 1u, abort_flag)) { ok = false; break; }
          uint8_t* st = smem + stage * kStageBytes;
          mbar_arrive_expect_tx(&tail->full[stage], kStageBytes);
          const int32_t kx = ks * (BK / 2);
          tma_load_2d(st, &tm_a, &tail->full[stage], kx, m_blk * BM);
          tma_load_2d(st + kABytes, &tm_b, &tail->full[stage], kx, static_cast<int32_t>(b_row0));
          tma_load_2d(st + kABytes + kBBytes / 2, &tm_b, &tail->full[stage], kx, static_cast<int32_t>(b_row1));
          uint8_t* sfa = st + kABytes + kBBytes;
          uint8_t* sfb = sfa + kSFABytes;
          tma_load_3d(sfa, &tm_sfa, &tail->full[stage], 0, ks * 4, m_blk);
          tma_load_3d(sfb, &tm_sfb, &tail->full[stage], 0, ks * 4, static_cast<int32_t>(b_row0 / 128));
          tma_load_3d(sfb + kSFBBytes / 2, &tm_sfb, &tail->full[stage], 0, ks * 4, static_cast<int32_t>(b_row1 / 128));
          issued[stage] = true;
          issued_phase[stage] = phase;
          if (++stage == kStages) { stage = 0; phase ^= 1u; }
        }
      }
      if (*abort_flag) {
        // let copies already in flight land before the CTA leaves
        for (int s = 0; s < kStages; ++s)
          if (issued[s]) mbar_wait_bounded(&tail->full[s], issued_phase[s], nullptr, 200000000ull);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (elect_one()) {
      // instruction descriptor: E2M1 x E2M1, UE4M3 scales, K-major A and B, M=128, N=256
      const uint32_t idesc = (1u << 7) | (1u << 10) | (static_cast<uint32_t>(BN >> 3) << 17) |
                             (static_cast<uint32_t>(BM >> 4) << 24);
      const uint32_t base = smem_u32(smem);
      int stage = 0;
      uint32_t phase = 0;
      int local = 0;
      bool ok = true;
      bool any_issued = false;
      for (int t = blockIdx.x; t < num_tiles && ok; t += gridDim.x, ++local) {
        if (local > 0) {
          if (!mbar_wait_bounded(&tail->tmem_empty, (local - 1) & 1, abort_flag)) { ok = false; break; }
        }
        tc_fence_after();
        for (int ks = 0; ks < args.num_k_stages; ++ks) {
          if (!mbar_wait_bounded(&tail->full[stage], phase, abort_flag)) { ok = false; break; }
          tc_fence_after();
          const uint32_t sa = base + stage * kStageBytes;
          const uint32_t sb = sa + kABytes;
          const uint32_t ssfa = sb + kBBytes;
          const uint32_t ssfb = ssfa + kSFABytes;
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            tmem_cp_32x128b_warpx4(tmem + kColSFA + 4 * j, make_smem_desc(ssfa + 512 * j, 0, 128, kLayoutSwizzleNone));
            tmem_cp_32x128b_warpx4(tmem + kColSFB + 8 * j, make_smem_desc(ssfb + 512 * j, 0, 128, kLayoutSwizzleNone));
            tmem_cp_32x128b_warpx4(tmem + kColSFB + 8 * j + 4,
                                   make_smem_desc(ssfb + kSFBBytes / 2 + 512 * j, 0, 128, kLayoutSwizzleNone));
          }
          const uint64_t adesc = make_smem_desc(sa, 16, 1024, kLayoutSwizzle128B);
          const uint64_t bdesc = make_smem_desc(sb, 16, 1024, kLayoutSwizzle128B);
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            // advance the start address by j * 32 bytes (64 FP4 elements) inside the swizzle atom
            mma_mxf4nvf4(tmem + kColAcc, adesc + 2 * j, bdesc + 2 * j, idesc, tmem + kColSFA + 4 * j,
                         tmem + kColSFB + 8 * j, (ks | j) != 0 ? 1u : 0u);
          }
          any_issued = true;
          tc_commit(&tail->empty[stage]);
          if (++stage == kStages) { stage = 0; phase ^= 1u; }
        }
        if (!ok) break;
        tc_commit(&tail->tmem_full);
      }
      if (*abort_flag && any_issued) {
        tc_commit(&tail->drain);
        mbar_wait_bounded(&tail->drain, 0, nullptr, 200000000ull);
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int q = warp & 3;            // TMEM lane quadrant this warp may read
    const int h = (warp - 2) >> 2;     // which half of the tile's columns
    int local = 0;
    for (int t = blockIdx.x; t < num_tiles; t += gridDim.x, ++local) {
      int m_blk, n_blk;
      tile_coords(args, t, m_blk, n_blk);
      if (!mbar_wait_bounded(&tail->tmem_full, local & 1, abort_flag)) break;
      tc_fence_after();
      const uint32_t lane_addr = tmem + (static_cast<uint32_t>(q * 32) << 16);
      uint32_t r0[32], r1[32], r2[32], r3[32];
      if (!args.swiglu) {
        tmem_ld_32x32b_x32(lane_addr + kColAcc + h * 128 + 0, r0);
        tmem_ld_32x32b_x32(lane_addr + kColAcc + h * 128 + 32, r1);
        tmem_ld_32x32b_x32(lane_addr + kColAcc + h * 128 + 64, r2);
        tmem_ld_32x32b_x32(lane_addr + kColAcc + h * 128 + 96, r3);
      } else {
        tmem_ld_32x32b_x32(lane_addr + kColAcc + h * 64 + 0, r0);
        tmem_ld_32x32b_x32(lane_addr + kColAcc + h * 64 + 32, r1);
        tmem_ld_32x32b_x32(lane_addr + kColAcc + 128 + h * 64 + 0, r2);
        tmem_ld_32x32b_x32(lane_addr + kColAcc + 128 + h * 64 + 32, r3);
      }
      tmem_ld_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&tail->tmem_empty);

      const int64_t row = static_cast<int64_t>(m_blk) * BM + q * 32 + lane;
      if (row < args.M) {
        if (!args.swiglu) {
          const int64_t n0 = static_cast<int64_t>(n_blk) * BN + h * 128;
          store_chunk(args, row, n0 + 0, r0);
          store_chunk(args, row, n0 + 32, r1);
          store_chunk(args, row, n0 + 64, r2);
          store_chunk(args, row, n0 + 96, r3);
        } else {
          const int64_t o0 = static_cast<int64_t>(n_blk) * 128 + h * 64;
          store_swiglu(args, row, o0, r0, r2);
          store_swiglu(args, row, o0 + 32, r1, r3);
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// ------------------------------------------------------------------ CTA-pair kernel
//
// Same computation on a 256 x 256 tile shared by the two CTAs of a cluster
// pair: each CTA loads 128 rows of A and 128 of the 256 B rows, the even CTA
// issues tcgen05.mma.cta_group::2 with M = 256, and each CTA's TMEM holds its
// own 128 x 256 accumulator.
//
// Each of the 5 stages holds one K-stage (256 K) of everything the MMAs read:
// the codes (two 16 KB boxes) and the scale atoms of this CTA's 128 A rows
// (2 KB) and of all 256 B rows (4 KB; the pair MMA reads each CTA's scales
// for the whole B tile from its own TMEM).  The epilogue stages BF16 output
// chunks in shared memory and writes them with TMA stores.
constexpr int kStages2 = 5;
constexpr int kBHalfBytes = kBBytes / 2;                                  // 16 KB
constexpr int kStageBytes2 = kABytes + kBHalfBytes + kSFABytes + kSFBBytes;  // 38 KB
constexpr int kStageSFA2 = kABytes + kBHalfBytes;                         // offsets in a stage
constexpr int kStageSFB2 = kStageSFA2 + kSFABytes;
static_assert(kStageBytes2 % 1024 == 0, "stage buffers keep 1024-byte alignment");

// The pair kernel's epilogue has 16 warps: warp w (2..17) reads TMEM lane
// quadrant w % 4 and column group (w - 2) / 4, 64 of the tile's 256 columns.
// Twice the 8 warps of the other kernels, so that one tile's epilogue (TMEM
// reads, scaling, nonlinearity, stores) keeps pace with the next tile's
// mainloop and does not hold back its MMAs.
constexpr int kNumEpiWarps2 = 16;
constexpr int kThreads2 = 64 + kNumEpiWarps2 * 32;
// one 32 x 32 BF16 output chunk (2 KB) of staging per epilogue warp
constexpr int kEpiChunkBytes = 2048;
constexpr int kEpiBytes2 = kNumEpiWarps2 * kEpiChunkBytes;
constexpr int kSmemBytes2 = kStages2 * kStageBytes2 + kEpiBytes2 + 1024 + 256;
static_assert(kSmemBytes2 <= 227 * 1024, "shared memory of one CTA");

// Two accumulators that share 64 TMEM columns: buffer 0 is columns
// [0, 256), buffer 1 is [192, 448), scales follow at 448.  The epilogue reads
// the shared columns first and releases them on ovl_free, so the next tile's
// MMAs (which overwrite them) wait for a 64-column read, not the whole drain.
constexpr uint32_t kColSFA2 = 448, kColSFB2 = 464;
__device__ __forceinline__ uint32_t col_acc2(int buf) { return buf ? 192u : 0u; }

struct SharedTail2 {
  uint64_t full[kStages2];
  uint64_t empty[kStages2];
  uint64_t tmem_full[2];
  uint64_t tmem_empty[2];
  uint64_t ovl_free[2];
  uint64_t drain;
  uint32_t tmem_base;
  int abort_flag;
};

// Staged store of one 32 x 32 BF16 chunk (lane l: row row0 + l, columns
// j0 .. j0+31 of segment s): the warp writes it to its 2 KB buffer in the
// map's 64-byte-swizzle layout (16-byte piece c of row r at c ^ ((r / 2) % 4),
// so the shared stores are free of bank conflicts) and one lane issues the
// TMA store; rows past M are not written.  The buffer is reused only after
// the previous store from it has been read.
__device__ __forceinline__ void stage_and_store_bf16(const CUtensorMap* m, uint8_t* buf, const uint32_t (&w)[16],
                                                     int32_t j0, int32_t row0) {
  const int lane = threadIdx.x & 31;
  if (lane == 0) bulk_wait_group_read<0>();
  __syncwarp();
  uint8_t* rowp = buf + lane * 64;
  const int sw = (lane >> 1) & 3;
#pragma unroll
  for (int c = 0; c < 4; ++c)
    *reinterpret_cast<uint4*>(rowp + ((c ^ sw) << 4)) = make_uint4(w[4 * c], w[4 * c + 1], w[4 * c + 2], w[4 * c + 3]);
  fence_proxy_async_smem();
  __syncwarp();
  if (lane == 0) {
    tma_store_2d(m, buf, j0, row0);
    bulk_commit_group();
  }
}

// Columns n0 .. n0+63 of rows row0 .. row0+31 (chunks r0 and r1).  When
// both lie in one BF16 segment with a map, on its 16-byte grid, they leave
// through the staging buffer as two 16-row x 64-column boxes: rows of 128
// bytes, so every global write is a whole line.  Lanes 16h .. 16h+15 place
// their rows for box h (16-byte piece c of box row r at c ^ (r % 8), the
// map's 128-byte swizzle, free of bank conflicts).  Otherwise (FP32
// epilogues, a segment boundary inside the 64 columns) each chunk is stored
// per lane.
__device__ __forceinline__ void store_pair_staged(const KernelArgs& a, const OutMaps& maps, uint8_t* buf,
                                                  int64_t row0, int64_t n0, const uint32_t (&r0)[32],
                                                  const uint32_t (&r1)[32]) {
  if (n0 >= a.N || row0 >= a.M) return;
  const int lane = threadIdx.x & 31;
  const int s = seg_of(a, n0);
  const EpiSegment& sg = a.seg[s];
  const int64_t j0 = n0 - sg.n_begin;
  if (((a.tma_mask >> s) & 1u) == 0 || n0 + 63 >= sg.n_end || (j0 & 7) != 0) {
    if (row0 + lane < a.M) {
      store_chunk(a, row0 + lane, n0, r0);
      store_chunk(a, row0 + lane, n0 + 32, r1);
    }
    return;
  }
  const float scale = __ldg(a.g_a) * __ldg(a.seg_scale + s);
  uint32_t w[32];
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    w[i] = pack_bf16(__uint_as_float(r0[2 * i]) * scale, __uint_as_float(r0[2 * i + 1]) * scale);
    w[16 + i] = pack_bf16(__uint_as_float(r1[2 * i]) * scale, __uint_as_float(r1[2 * i + 1]) * scale);
  }
  const int rr = lane & 15;
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    if (row0 + 16 * h >= a.M) break;  // uniform
    if (lane == 0) bulk_wait_group_read<0>();
    __syncwarp();
    if ((lane >> 4) == h) {
      uint8_t* rowp = buf + rr * 128;
#pragma unroll
      for (int c = 0; c < 8; ++c)
        *reinterpret_cast<uint4*>(rowp + ((c ^ (rr & 7)) << 4)) =
            make_uint4(w[4 * c], w[4 * c + 1], w[4 * c + 2], w[4 * c + 3]);
    }
    fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0) {
      tma_store_2d(&maps.m[s], buf, static_cast<int32_t>(j0), static_cast<int32_t>(row0 + 16 * h));
      bulk_commit_group();
    }
  }
}

// SwiGLU chunk: output columns o0 .. o0+31 of rows row0 .. row0+31.
__device__ __forceinline__ void store_swiglu_staged(const KernelArgs& a, const OutMaps& maps, uint8_t* buf,
                                                    int64_t row0, int64_t o0, const uint32_t (&rg)[32],
                                                    const uint32_t (&ru)[32]) {
  if (o0 >= a.n_out || row0 >= a.M) return;
  const int lane = threadIdx.x & 31;
  if ((a.tma_mask & 1u) == 0 || o0 + 31 >= a.n_out) {
    if (row0 + lane < a.M) store_swiglu(a, row0 + lane, o0, rg, ru);
    return;
  }
  const float ga = __ldg(a.g_a);
  const float sgate = ga * __ldg(a.seg_scale + 0);
  const float sup = ga * __ldg(a.seg_scale + 1);
  uint32_t w[16];
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    float v[2];
#pragma unroll
    for (int k = 0; k < 2; ++k) {
      const float gv = __uint_as_float(rg[2 * i + k]) * sgate;
      const float uv = __uint_as_float(ru[2 * i + k]) * sup;
      v[k] = gv * __frcp_rn(1.0f + __expf(-gv)) * uv;
    }
    w[i] = pack_bf16(v[0], v[1]);
  }
  stage_and_store_bf16(&maps.m[0], buf, w, static_cast<int32_t>(o0), static_cast<int32_t>(row0));
}

template <bool SWIGLU>
__global__ void __launch_bounds__(kThreads2, 1)
    gemm_pair_kernel(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_b,
                     const __grid_constant__ CUtensorMap tm_sfa, const __grid_constant__ CUtensorMap tm_sfb,
                     const __grid_constant__ KernelArgs args, const __grid_constant__ OutMaps out_maps) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint8_t* epi_smem = smem + kStages2 * kStageBytes2;
  SharedTail2* tail = reinterpret_cast<SharedTail2*>(epi_smem + kEpiBytes2);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_rank() & 1u;  // position in the pair
  const bool leader = rank == 0;
  const int pair = blockIdx.x >> 1;
  const int num_pairs = gridDim.x >> 1;
  const int num_tiles = args.num_m_blocks * args.num_n_blocks;  // m blocks of 256 rows
  const int KS = args.num_k_stages;
  volatile int* abort_flag = &tail->abort_flag;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages2; ++s) {
      mbar_init(&tail->full[s], 1);
      mbar_init(&tail->empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&tail->tmem_full[b], 1);
      mbar_init(&tail->tmem_empty[b], 2 * kNumEpiWarps2);
      // the warps of both CTAs that hold the shared columns: 4 per CTA (one
      // column group), 8 for SwiGLU (gate and up halves of two groups)
      mbar_init(&tail->ovl_free[b], SWIGLU ? 16 : 8);
    }
    mbar_init(&tail->drain, 1);
    tail->abort_flag = 0;
    fence_mbarrier_init();
    prefetch_tmap(&tm_a);
    prefetch_tmap(&tm_b);
    prefetch_tmap(&tm_sfa);
    prefetch_tmap(&tm_sfb);
    for (int i = 0; i < args.nseg; ++i)
      if ((args.tma_mask >> i) & 1u) prefetch_tmap(&out_maps.m[i]);
  }
  if (warp == 1) {
    tmem_alloc_pair(&tail->tmem_base, kTmemCols);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  cluster_sync_all();  // both CTAs' barriers exist before any cross-CTA signal
  tc_fence_after();
  const uint32_t tmem = tail->tmem_base;
  // Everything above may overlap the previous kernel on the stream; operands,
  // scales and outputs are touched only after the wait (the MMA warp reads
  // shared memory and TMEM only).
  if (warp != 1) grid_dependency_wait();
  if (threadIdx.x == 0) grid_launch_dependents();

  if (warp == 0) {
    // ------------------------------------------------------------ producer (both CTAs)
    if (elect_one()) {
      int stage = 0;
      uint32_t phase = 0;
      bool issued[kStages2];
      uint32_t issued_phase[kStages2];
      for (int s = 0; s < kStages2; ++s) issued[s] = false;
      bool ok = true;
      for (int t = pair; t < num_tiles && ok; t += num_pairs) {
        int m_blk, n_blk;
        tile_coords(args, t, m_blk, n_blk);
        const int32_t a_row = m_blk * 256 + static_cast<int32_t>(rank) * 128;
        const int64_t b_row0 = SWIGLU ? static_cast<int64_t>(n_blk) * 128 : static_cast<int64_t>(n_blk) * BN;
        const int64_t b_row1 = SWIGLU ? args.up_row0 + static_cast<int64_t>(n_blk) * 128 : b_row0 + 128;
        const int64_t b_mine = rank ? b_row1 : b_row0;
        for (int ks = 0; ks < KS; ++ks) {
          if (!mbar_wait_bounded(&tail->empty[stage], phase ^ 1u, abort_flag)) { ok = false; break; }
          uint8_t* st = smem + stage * kStageBytes2;
          const uint32_t bar = map_to_rank(smem_u32(&tail->full[stage]), 0);  // even CTA of the pair
          if (leader) mbar_arrive_expect_tx(&tail->full[stage], 2 * kStageBytes2);
          const int32_t kx = ks * (BK / 2);
          tma_load_2d_pair(st, &tm_a, bar, kx, a_row);
          tma_load_2d_pair(st + kABytes, &tm_b, bar, kx, static_cast<int32_t>(b_mine));
          tma_load_3d_pair(st + kStageSFA2, &tm_sfa, bar, 0, ks * 4, a_row / 128);
          if (SWIGLU) {
            tma_load_3d_pair(st + kStageSFB2, &tm_sfb, bar, 0, ks * 4, static_cast<int32_t>(b_row0 / 128));
            tma_load_3d_pair(st + kStageSFB2 + kSFBBytes / 2, &tm_sfb, bar, 0, ks * 4, static_cast<int32_t>(b_row1 / 128));
          } else {
            tma_load_3d_pair(st + kStageSFB2, &tm_sfb, bar, 0, ks * 4, static_cast<int32_t>(b_row0 / 128));
          }
          issued[stage] = true;
          issued_phase[stage] = phase;
          if (++stage == kStages2) { stage = 0; phase ^= 1u; }
        }
      }
      if (*abort_flag && leader) {
        for (int s = 0; s < kStages2; ++s)
          if (issued[s]) mbar_wait_bounded(&tail->full[s], issued_phase[s], nullptr, 200000000ull);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer (even CTA)
    if (leader && elect_one()) {
      // E2M1 x E2M1, UE4M3 scales, K-major A and B, M = 256 (pair), N = 256
      const uint32_t idesc = (1u << 7) | (1u << 10) | (static_cast<uint32_t>(BN >> 3) << 17) |
                             (static_cast<uint32_t>(256 >> 4) << 24);
      const uint32_t base = smem_u32(smem);
      int stage = 0;
      uint32_t phase = 0;
      int local = 0;
      bool ok = true;
      bool any_issued = false;
      for (int t = pair; t < num_tiles && ok; t += num_pairs, ++local) {
        const int buf = local & 1;
        // shared columns read by the previous tile's epilogue; own columns drained two tiles ago
        if (local >= 1 &&
            !mbar_wait_bounded(&tail->ovl_free[buf ^ 1], ((local - 1) >> 1) & 1, abort_flag)) { ok = false; break; }
        if (local >= 2 &&
            !mbar_wait_bounded(&tail->tmem_empty[buf], ((local - 2) >> 1) & 1, abort_flag)) { ok = false; break; }
        tc_fence_after();
        for (int ks = 0; ks < KS; ++ks) {
          if (!mbar_wait_bounded(&tail->full[stage], phase, abort_flag)) { ok = false; break; }
          tc_fence_after();
          const uint32_t sa = base + stage * kStageBytes2;
          const uint32_t sb = sa + kABytes;
          const uint32_t ssfa = sa + kStageSFA2;
          const uint32_t ssfb = sa + kStageSFB2;
#pragma unroll
          for (int kb = 0; kb < 4; ++kb) {
            tmem_cp_32x128b_warpx4_pair(tmem + kColSFA2 + 4 * kb, make_smem_desc(ssfa + 512 * kb, 0, 128, kLayoutSwizzleNone));
            tmem_cp_32x128b_warpx4_pair(tmem + kColSFB2 + 8 * kb, make_smem_desc(ssfb + 512 * kb, 0, 128, kLayoutSwizzleNone));
            tmem_cp_32x128b_warpx4_pair(tmem + kColSFB2 + 8 * kb + 4,
                                        make_smem_desc(ssfb + kSFBBytes / 2 + 512 * kb, 0, 128, kLayoutSwizzleNone));
          }
          const uint64_t adesc = make_smem_desc(sa, 16, 1024, kLayoutSwizzle128B);
          const uint64_t bdesc = make_smem_desc(sb, 16, 1024, kLayoutSwizzle128B);
#pragma unroll
          for (int kb = 0; kb < 4; ++kb)
            mma_mxf4nvf4_pair(tmem + col_acc2(buf), adesc + 2 * kb, bdesc + 2 * kb, idesc, tmem + kColSFA2 + 4 * kb,
                              tmem + kColSFB2 + 8 * kb, (ks | kb) != 0 ? 1u : 0u);
          any_issued = true;
          tc_commit_pair_mc(&tail->empty[stage], 0x3);
          if (++stage == kStages2) { stage = 0; phase ^= 1u; }
        }
        if (!ok) break;
        tc_commit_pair_mc(&tail->tmem_full[buf], 0x3);
      }
      if (*abort_flag && any_issued) {
        tc_commit_pair_mc(&tail->drain, 0x1);
        mbar_wait_bounded(&tail->drain, 0, nullptr, 200000000ull);
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue (both CTAs)
    const int q = warp & 3;           // TMEM lane quadrant this warp may read
    const int g = (warp - 2) >> 2;    // column group: 64 of the tile's 256 columns
    uint8_t* buf_smem = epi_smem + (warp - 2) * kEpiChunkBytes;
    uint32_t empty_leader[2], ovl_leader[2];
    for (int b = 0; b < 2; ++b) {
      empty_leader[b] = map_to_rank(smem_u32(&tail->tmem_empty[b]), 0);
      ovl_leader[b] = map_to_rank(smem_u32(&tail->ovl_free[b]), 0);
    }
    // This warp's two 32-column chunks sit at buffer columns c0 and c1: group
    // g's columns [64g, 64g + 64), or for SwiGLU the gate chunk 32g and its up
    // chunk 128 + 32g.  The shared columns are buffer 0's [192, 256) and
    // buffer 1's [0, 64).
    const uint32_t c0 = SWIGLU ? 32u * g : 64u * g;
    const uint32_t c1 = SWIGLU ? 128u + 32u * g : 64u * g + 32u;
    int local = 0;
    for (int t = pair; t < num_tiles; t += num_pairs, ++local) {
      int m_blk, n_blk;
      tile_coords(args, t, m_blk, n_blk);
      const int buf = local & 1;
      if (!mbar_wait_bounded(&tail->tmem_full[buf], (local >> 1) & 1, abort_flag)) break;
      tc_fence_after();
      const uint32_t base = tmem + (static_cast<uint32_t>(q * 32) << 16) + col_acc2(buf);
      uint32_t r0[32], r1[32];
      tmem_ld_32x32b_x32(base + c0, r0);
      tmem_ld_32x32b_x32(base + c1, r1);
      tmem_ld_wait();
      tc_fence_before();
      __syncwarp();
      const bool shared = buf == 0 ? (c1 >= 192u) : (c0 < 64u);
      if (lane == 0) {
        if (shared) mbar_arrive_remote(ovl_leader[buf]);
        mbar_arrive_remote(empty_leader[buf]);
      }
      const int64_t row0 = static_cast<int64_t>(m_blk) * 256 + rank * 128 + q * 32;
      if constexpr (!SWIGLU) {
        store_pair_staged(args, out_maps, buf_smem, row0, static_cast<int64_t>(n_blk) * BN + 64 * g, r0, r1);
      } else {
        store_swiglu_staged(args, out_maps, buf_smem, row0, static_cast<int64_t>(n_blk) * 128 + 32 * g, r0, r1);
      }
    }
    // every TMA store has read its buffer and written global memory
    if (lane == 0) bulk_wait_group_all();
    __syncwarp();
  }

  tc_fence_before();
  cluster_sync_all();  // no pair-wide tcgen05 work remains in either CTA
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem, kTmemCols);
  }
}

// ------------------------------------------------------------------ CTA-pair kernel, N = 192
//
// The 256 x 256 pair kernel holds a single accumulator per CTA (256 of the 512
// TMEM columns, plus 48 for scales), so each tile ends with the MMA pipe
// draining and the epilogue reading TMEM while the tensor cores wait.  With an
// N = 192 tile two accumulators fit (2 x 192 + 16 SFA + 32 SFB columns), and
// the next tile's MMAs run while the epilogue drains the previous one.  Each
// CTA loads 128 A rows and 96 B rows; the B scale atoms are those of the two
// 128-row blocks the 192 rows touch (a tile starts at 0 or 64 within its first
// block), and the MMA's SFB address is shifted by (n0 mod 128) / 32 = 0 or 2
// columns so that row n0 meets its scales (scale addresses stay 2-column
// aligned).  Used for every fused projection except SwiGLU.
constexpr int BN3 = 192;
constexpr int kStages3 = 6;
constexpr int kBRows3 = BN3 / 2;                           // 96 rows per CTA
constexpr int kBBytes3 = kBRows3 * BK / 2;                 // 12 KB
constexpr int kSFBBlocks3 = 2;
constexpr int kSFBBytes3 = kSFBBlocks3 * 4 * 512;          // 2 row blocks x 4 atoms
constexpr int kStageBytes3 = kABytes + kBBytes3 + kSFABytes + kSFBBytes3;  // 34 KB
constexpr int kSmemBytes3 = kStages3 * kStageBytes3 + 1024 + 256;
__device__ __forceinline__ uint32_t col_acc3(int buf) { return buf ? 192u : 0u; }
constexpr uint32_t kColSFA3 = 384, kColSFB3 = 400;
static_assert(kStageBytes3 % 1024 == 0, "stage buffers keep 1024-byte alignment");

struct SharedTail3 {
  uint64_t full[kStages3];
  uint64_t empty[kStages3];
  uint64_t tmem_full[2];
  uint64_t tmem_empty[2];
  uint64_t drain;
  uint32_t tmem_base;
  int abort_flag;
};

__global__ void __launch_bounds__(kThreads, 1)
    gemm_pair_db_kernel(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_b,
                        const __grid_constant__ CUtensorMap tm_sfa, const __grid_constant__ CUtensorMap tm_sfb,
                        const __grid_constant__ KernelArgs args) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  SharedTail3* tail = reinterpret_cast<SharedTail3*>(smem + kStages3 * kStageBytes3);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_rank() & 1u;
  const bool leader = rank == 0;
  const int pair = blockIdx.x >> 1;
  const int num_pairs = gridDim.x >> 1;
  const int num_tiles = args.num_m_blocks * args.num_n_blocks;
  volatile int* abort_flag = &tail->abort_flag;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages3; ++s) {
      mbar_init(&tail->full[s], 1);
      mbar_init(&tail->empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&tail->tmem_full[b], 1);
      mbar_init(&tail->tmem_empty[b], 2 * kNumEpiWarps);
    }
    mbar_init(&tail->drain, 1);
    tail->abort_flag = 0;
    fence_mbarrier_init();
    prefetch_tmap(&tm_a);
    prefetch_tmap(&tm_b);
    prefetch_tmap(&tm_sfa);
    prefetch_tmap(&tm_sfb);
  }
  if (warp == 1) {
    tmem_alloc_pair(&tail->tmem_base, kTmemCols);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  cluster_sync_all();
  tc_fence_after();
  const uint32_t tmem = tail->tmem_base;
  // Everything above may overlap the previous kernel on the stream; operands,
  // scales and outputs are touched only after the wait (the MMA warp reads
  // shared memory and TMEM only).
  if (warp != 1) grid_dependency_wait();
  if (threadIdx.x == 0) grid_launch_dependents();

  if (warp == 0) {
    // ------------------------------------------------------------ producer (both CTAs)
    if (elect_one()) {
      int stage = 0;
      uint32_t phase = 0;
      uint32_t issued_phase[kStages3];
      bool issued[kStages3];
      for (int s = 0; s < kStages3; ++s) issued[s] = false;
      bool ok = true;
      for (int t = pair; t < num_tiles && ok; t += num_pairs) {
        int m_blk, n_blk;
        tile_coords(args, t, m_blk, n_blk);
        const int32_t a_row = m_blk * 256 + static_cast<int32_t>(rank) * 128;
        const int32_t n0 = n_blk * BN3;
        const int32_t b_row = n0 + static_cast<int32_t>(rank) * kBRows3;
        for (int ks = 0; ks < args.num_k_stages; ++ks) {
          if (!mbar_wait_bounded(&tail->empty[stage], phase ^ 1u, abort_flag)) { ok = false; break; }
          uint8_t* st = smem + stage * kStageBytes3;
          const uint32_t bar = map_to_rank(smem_u32(&tail->full[stage]), 0);
          if (leader) mbar_arrive_expect_tx(&tail->full[stage], 2 * kStageBytes3);
          const int32_t kx = ks * (BK / 2);
          tma_load_2d_pair(st, &tm_a, bar, kx, a_row);
          tma_load_2d_pair(st + kABytes, &tm_b, bar, kx, b_row);
          uint8_t* sfa = st + kABytes + kBBytes3;
          tma_load_3d_pair(sfa, &tm_sfa, bar, 0, ks * 4, a_row / 128);
          tma_load_3d_pair(sfa + kSFABytes, &tm_sfb, bar, 0, ks * 4, n0 / 128);
          issued[stage] = true;
          issued_phase[stage] = phase;
          if (++stage == kStages3) { stage = 0; phase ^= 1u; }
        }
      }
      if (*abort_flag && leader) {
        for (int s = 0; s < kStages3; ++s)
          if (issued[s]) mbar_wait_bounded(&tail->full[s], issued_phase[s], nullptr, 200000000ull);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer (even CTA)
    if (leader && elect_one()) {
      // E2M1 x E2M1, UE4M3 scales, K-major A and B, M = 256 (pair), N = 192
      const uint32_t idesc = (1u << 7) | (1u << 10) | (static_cast<uint32_t>(BN3 >> 3) << 17) |
                             (static_cast<uint32_t>(256 >> 4) << 24);
      const uint32_t base = smem_u32(smem);
      int stage = 0;
      uint32_t phase = 0;
      int local = 0;
      bool ok = true;
      bool any_issued = false;
      for (int t = pair; t < num_tiles && ok; t += num_pairs, ++local) {
        int m_blk, n_blk;
        tile_coords(args, t, m_blk, n_blk);
        const uint32_t shift = static_cast<uint32_t>((n_blk * BN3) % 128) / 32;
        const int buf = local & 1;
        if (local >= 2) {
          if (!mbar_wait_bounded(&tail->tmem_empty[buf], ((local >> 1) - 1) & 1, abort_flag)) { ok = false; break; }
        }
        tc_fence_after();
        for (int ks = 0; ks < args.num_k_stages; ++ks) {
          if (!mbar_wait_bounded(&tail->full[stage], phase, abort_flag)) { ok = false; break; }
          tc_fence_after();
          const uint32_t sa = base + stage * kStageBytes3;
          const uint32_t sb = sa + kABytes;
          const uint32_t ssfa = sb + kBBytes3;
          const uint32_t ssfb = ssfa + kSFABytes;
#pragma unroll
          for (int kb = 0; kb < 4; ++kb) {
            tmem_cp_32x128b_warpx4_pair(tmem + kColSFA3 + 4 * kb, make_smem_desc(ssfa + 512 * kb, 0, 128, kLayoutSwizzleNone));
#pragma unroll
            for (int z = 0; z < kSFBBlocks3; ++z)
              tmem_cp_32x128b_warpx4_pair(tmem + kColSFB3 + 4 * kSFBBlocks3 * kb + 4 * z,
                                          make_smem_desc(ssfb + 2048 * z + 512 * kb, 0, 128, kLayoutSwizzleNone));
          }
          const uint64_t adesc = make_smem_desc(sa, 16, 1024, kLayoutSwizzle128B);
          const uint64_t bdesc = make_smem_desc(sb, 16, 1024, kLayoutSwizzle128B);
#pragma unroll
          for (int kb = 0; kb < 4; ++kb)
            mma_mxf4nvf4_pair(tmem + col_acc3(buf), adesc + 2 * kb, bdesc + 2 * kb, idesc, tmem + kColSFA3 + 4 * kb,
                              tmem + kColSFB3 + 4 * kSFBBlocks3 * kb + shift, (ks | kb) != 0 ? 1u : 0u);
          any_issued = true;
          tc_commit_pair_mc(&tail->empty[stage], 0x3);
          if (++stage == kStages3) { stage = 0; phase ^= 1u; }
        }
        if (!ok) break;
        tc_commit_pair_mc(&tail->tmem_full[buf], 0x3);
      }
      if (*abort_flag && any_issued) {
        tc_commit_pair_mc(&tail->drain, 0x1);
        mbar_wait_bounded(&tail->drain, 0, nullptr, 200000000ull);
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue (both CTAs)
    const int q = warp & 3;
    const int h = (warp - 2) >> 2;  // columns [0, 96) or [96, 192)
    uint32_t empty_leader[2];
    empty_leader[0] = map_to_rank(smem_u32(&tail->tmem_empty[0]), 0);
    empty_leader[1] = map_to_rank(smem_u32(&tail->tmem_empty[1]), 0);
    int local = 0;
    for (int t = pair; t < num_tiles; t += num_pairs, ++local) {
      int m_blk, n_blk;
      tile_coords(args, t, m_blk, n_blk);
      const int buf = local & 1;
      if (!mbar_wait_bounded(&tail->tmem_full[buf], (local >> 1) & 1, abort_flag)) break;
      tc_fence_after();
      const uint32_t col = tmem + (static_cast<uint32_t>(q * 32) << 16) + col_acc3(buf) + h * 96;
      uint32_t r0[32], r1[32], r2[32];
      tmem_ld_32x32b_x32(col + 0, r0);
      tmem_ld_32x32b_x32(col + 32, r1);
      tmem_ld_32x32b_x32(col + 64, r2);
      tmem_ld_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_remote(empty_leader[buf]);

      const int64_t row = static_cast<int64_t>(m_blk) * 256 + rank * 128 + q * 32 + lane;
      if (row < args.M) {
        const int64_t n0 = static_cast<int64_t>(n_blk) * BN3 + h * 96;
        store_chunk(args, row, n0 + 0, r0);
        store_chunk(args, row, n0 + 32, r1);
        store_chunk(args, row, n0 + 64, r2);
      }
    }
  }

  tc_fence_before();
  cluster_sync_all();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem, kTmemCols);
  }
}


// ------------------------------------------------------------------ host side

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// Codes [rows, K/2] bytes: box 128 bytes x box_rows rows, 128-byte swizzle.
bool make_codes_map(CUtensorMap* m, const uint8_t* codes, int64_t rows, int64_t K, uint32_t box_rows = 128) {
  const cuuint64_t dims[2] = {static_cast<cuuint64_t>(K / 2), static_cast<cuuint64_t>(rows)};
  const cuuint64_t strides[1] = {static_cast<cuuint64_t>(K / 2)};
  const cuuint32_t box[2] = {128, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  return encode_fn()(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint8_t*>(codes), dims, strides,
                     box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                     CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Scale atoms: [row blocks][K atoms][512 bytes] viewed as u32 {128, KA, RB};
// box = `atoms` atoms of `blocks` consecutive 128-row blocks.
bool make_sf_map(CUtensorMap* m, const uint8_t* sf, int64_t rows, int64_t K, uint32_t atoms = 4, uint32_t blocks = 1) {
  const int64_t KA = ceil_div(K, 64), RB = ceil_div(rows, 128);
  const cuuint64_t dims[3] = {128, static_cast<cuuint64_t>(KA), static_cast<cuuint64_t>(RB)};
  const cuuint64_t strides[2] = {512, static_cast<cuuint64_t>(KA * 512)};
  const cuuint32_t box[3] = {128, atoms, blocks};
  const cuuint32_t estr[3] = {1, 1, 1};
  return encode_fn()(m, CU_TENSOR_MAP_DATA_TYPE_UINT32, 3, const_cast<uint8_t*>(sf), dims, strides,
                     box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                     CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Output maps for the staged epilogue of the pair kernel: one per BF16
// segment (identity or SwiGLU output) at least 64 columns wide, dims
// {segment width, M}, with the box of the kernel's mode (see OutMaps).
// Other segments keep the per-lane stores (mask bit clear).
uint32_t make_out_maps(const GemmProblem& p, OutMaps* maps) {
  uint32_t mask = 0;
  for (int s = 0; s < p.nseg; ++s) {
    const EpiSegment& sg = p.seg[s];
    const bool bf16 = sg.kind == NVFP4_EPI_IDENTITY_BF16 || sg.kind == NVFP4_EPI_SWIGLU_GATE;
    if (!bf16 || sg.out == nullptr) continue;
    const int64_t width = p.swiglu ? p.N / 2 : sg.n_end - sg.n_begin;
    if (width < 64 || p.M < 1 || (sg.ld_out * 2) % 16 != 0) continue;
    const cuuint64_t dims[2] = {static_cast<cuuint64_t>(width), static_cast<cuuint64_t>(p.M)};
    const cuuint64_t strides[1] = {static_cast<cuuint64_t>(sg.ld_out * 2)};
    const cuuint32_t box[2] = {p.swiglu ? 32u : 64u, p.swiglu ? 32u : 16u};
    const cuuint32_t estr[2] = {1, 1};
    if (encode_fn()(&maps->m[s], CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, sg.out, dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, p.swiglu ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_128B,
                    CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS)
      mask |= 1u << s;
  }
  return mask;
}

}  // namespace gk

size_t gemm_workspace_bytes(int64_t, int64_t, int64_t) { return 0; }

// Prefill shapes (M > 128) run on CTA pairs unless switched off for comparison.
#ifndef NVFP4_PAIR_KERNEL
#define NVFP4_PAIR_KERNEL 1
#endif
bool g_use_pair_kernel = NVFP4_PAIR_KERNEL;

bool decode_path_applies(const GemmProblem& p);
cudaError_t launch_gemm_decode(const GemmProblem& p, cudaStream_t stream);

cudaError_t launch_gemm(const GemmProblem& p, void*, size_t, cudaStream_t stream) {
  using namespace gk;
  if (encode_fn() == nullptr) return cudaErrorNotSupported;
  if (decode_path_applies(p)) return launch_gemm_decode(p, stream);
  CUtensorMap tm_a, tm_b, tm_sfa, tm_sfb;
  if (!make_codes_map(&tm_a, p.a_codes, p.M, p.K) || !make_codes_map(&tm_b, p.w_codes, p.N, p.K) ||
      !make_sf_map(&tm_sfa, p.a_sf, p.M, p.K) || !make_sf_map(&tm_sfb, p.w_sf, p.N, p.K))
    return cudaErrorInvalidValue;

  const bool pair_kernel = p.M > 128 && g_use_pair_kernel;
  KernelArgs a{};
  a.M = p.M;
  a.N = p.N;
  a.K = p.K;
  a.swiglu = p.swiglu ? 1 : 0;
  a.n_out = p.swiglu ? p.N / 2 : p.N;
  a.up_row0 = p.swiglu ? p.N / 2 : 0;
  a.num_m_blocks = static_cast<int>(ceil_div(p.M, pair_kernel ? 2 * BM : BM));
  a.num_n_blocks = static_cast<int>(p.swiglu ? ceil_div(p.N / 2, 128) : ceil_div(p.N, BN));
  a.num_k_stages = static_cast<int>(ceil_div(p.K, BK));
  a.group_m = pair_kernel ? 32 : 16;
  if (pair_kernel) {
    // Tiles are walked m-fastest inside groups of group_m row blocks: the
    // group's A panels stay in L2 while W streams through once per group.
    // When all of A fits in L2 with room for the output stream, one group
    // covers every row block, so W is read from DRAM once; otherwise groups
    // of 32 row blocks (8192 rows, about 24 MB of A at K = 5120) read W once
    // per group.  (Measured on the GDN shape: groups of 32 ran 2.5% faster
    // than groups of 8 or 16; one row block per group, keeping W resident,
    // ran slower: every pair then starts the same new A panel at once.)
    const double a_bytes = static_cast<double>(p.M) * static_cast<double>(p.K) * (0.5 + 1.0 / 16);
    constexpr double kResident = 48.0 * 1024 * 1024;
    if (a_bytes <= kResident) a.group_m = a.num_m_blocks;
  }
  a.g_a = p.g_a;
  a.seg_scale = p.seg_scale;
  a.nseg = p.nseg;
  for (int i = 0; i < p.nseg; ++i) a.seg[i] = p.seg[i];

  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int tiles = a.num_m_blocks * a.num_n_blocks;
  if (tiles == 0) return cudaSuccess;
  if (!pair_kernel) {
    static std::atomic<uint64_t> attr_done{0};
    cudaError_t ea = once_per_device(attr_done, [] {
      return cudaFuncSetAttribute(gemm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
    });
    if (ea != cudaSuccess) return ea;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(tiles < sms ? tiles : sms);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = kSmemBytes;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, gemm_kernel, tm_a, tm_b, tm_sfa, tm_sfb, a);
  }
  // Non-SwiGLU projections run either 192-wide double-buffered tiles or
  // 256-wide tiles with overlapping accumulators.  The 256-wide tile moves
  // about 17% fewer operand bytes per MMA clock; the 192-wide tile can fill
  // the last wave better.  Pick the smaller estimated time.
  bool n192 = false;
  if (!p.swiglu) {
    const int64_t pairs_avail = sms / 2;
    const int64_t mb = ceil_div(p.M, 256);
    const double t192 = static_cast<double>(ceil_div(mb * ceil_div(p.N, BN3), pairs_avail)) * 192.0;
    const double t256 = static_cast<double>(ceil_div(mb * ceil_div(p.N, BN), pairs_avail)) * 256.0 * 0.95;
    n192 = t192 < t256;
  }
  if (n192) {
    KernelArgs b = a;
    b.num_n_blocks = static_cast<int>(ceil_div(p.N, BN3));
    CUtensorMap tm_b3, tm_sfb3;
    if (!make_codes_map(&tm_b3, p.w_codes, p.N, p.K, kBRows3) || !make_sf_map(&tm_sfb3, p.w_sf, p.N, p.K, 4, kSFBBlocks3))
      return cudaErrorInvalidValue;
    static std::atomic<uint64_t> attr3_done{0};
    cudaError_t ea = once_per_device(attr3_done, [] {
      return cudaFuncSetAttribute(gemm_pair_db_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes3);
    });
    if (ea != cudaSuccess) return ea;
    const int tiles3 = b.num_m_blocks * b.num_n_blocks;
    const int pairs3 = tiles3 < sms / 2 ? tiles3 : sms / 2;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2 * pairs3);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = kSmemBytes3;
    cfg.stream = stream;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    return cudaLaunchKernelEx(&cfg, gemm_pair_db_kernel, tm_a, tm_b3, tm_sfa, tm_sfb3, b);
  }
  // scale atoms of one K-stage: this CTA's 128 A rows; the tile's 256 B rows
  // (two consecutive 128-row blocks, or for SwiGLU the gate and up blocks,
  // one box each)
  CUtensorMap tm_sfa1, tm_sfb2;
  if (!make_sf_map(&tm_sfa1, p.a_sf, p.M, p.K, 4, 1) || !make_sf_map(&tm_sfb2, p.w_sf, p.N, p.K, 4, p.swiglu ? 1 : 2))
    return cudaErrorInvalidValue;
  OutMaps maps{};
  a.tma_mask = make_out_maps(p, &maps);
  static std::atomic<uint64_t> attr2_done{0};
  cudaError_t ea = once_per_device(attr2_done, [] {
    cudaError_t e = cudaFuncSetAttribute(gemm_pair_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes2);
    return e != cudaSuccess ? e
                            : cudaFuncSetAttribute(gemm_pair_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                   kSmemBytes2);
  });
  if (ea != cudaSuccess) return ea;
  const int pairs = tiles < sms / 2 ? tiles : sms / 2;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2 * pairs);
  cfg.blockDim = dim3(kThreads2);
  cfg.dynamicSmemBytes = kSmemBytes2;
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  if (p.swiglu) return cudaLaunchKernelEx(&cfg, gemm_pair_kernel<true>, tm_a, tm_b, tm_sfa1, tm_sfb2, a, maps);
  return cudaLaunchKernelEx(&cfg, gemm_pair_kernel<false>, tm_a, tm_b, tm_sfa1, tm_sfb2, a, maps);
}

}  // namespace nvfp4
