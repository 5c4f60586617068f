// Weight-streaming NVFP4 GEMM for few tokens (M <= 64), sm_100a.
//
// Same arithmetic as the prefill kernel ("Why Gated DeltaNet Survives 4-Bit
// Quantization", ai.info summary, "Methodology in Plain English"; "Main
// Findings": per-module global scales and gate nonlinearities), shaped for
// decode, where the GEMM is bound by reading W from HBM ("Main Findings",
// efficiency bullet: decode is weight-bandwidth-bound).
//
//  * Swap AB: 128 weight rows fill the MMA M dimension, the (<= 64) tokens sit
//    in N = 64, so out^T[n, m] = W[n, :] . X[m, :] accumulates in TMEM with one
//    TMEM lane per weight row.
//  * Split K over a thread-block cluster: the S CTAs of a cluster share one
//    128-row block of W and each streams 1/S of K, so about S * N/128 CTAs
//    stream W at once.
//  * The S partial accumulators are summed through distributed shared memory:
//    every CTA stages its FP32 partial in its own shared memory; after a
//    cluster barrier each CTA finalises a share of the tokens, adding the
//    ranks' partials in rank order (deterministic), applying the global
//    scales and the segment's epilogue and storing.  A second cluster barrier
//    keeps every CTA alive until the others have read it.  No workspace, no
//    atomics; all mbarrier waits are bounded.
//
// Warps: 0 TMA producer, 1 TMEM owner + MMA issuer, 2..5 epilogue (one TMEM
// lane quadrant each).
#include <cfloat>
#include <cstdint>

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "internal.h"
#include "ptx.cuh"

namespace nvfp4 {
namespace dk {

constexpr int BM = 128;  // weight rows per CTA (MMA M)
constexpr int BK = 256;  // K elements per 128-byte chunk of a row
constexpr int kEpiWarps = 4;
constexpr int kThreads = 64 + kEpiWarps * 32;
constexpr uint32_t kTmemCols = 256;
constexpr int kSmemBudget = 200 * 1024;

// BN token columns (MMA N = 16, 32 or 64; tokens beyond M are zero rows of X)
// and CH K-chunks of 256 per stage.  Each stage is four TMA copies (W codes,
// X codes, W scales, X scales); with CH = 2 one 32 KB weight box carries two
// chunks.  CH > 1 views the codes as 3-D {128 B, rows, K/256} and needs
// K % 256 == 0; CH = 1 uses the row-clipped 2-D view.
template <int BN, int CH>
struct DCfg {
  static constexpr int kWBytes = BM * BK / 2 * CH;
  static constexpr int kXPlane = BN * BK / 2;  // one chunk of X
  static constexpr int kXBytes = kXPlane * CH;
  static constexpr int kSFWBytes = BM * BK / 16 * CH;
  static constexpr int kSFXBytes = 128 * BK / 16 * CH;  // 128-row atoms
  static constexpr int kStageRaw = kWBytes + kXBytes + kSFWBytes + kSFXBytes;
  static constexpr int kStageBytes = (kStageRaw + 1023) / 1024 * 1024;
  static constexpr int kStages = kSmemBudget / kStageBytes;
  static constexpr uint32_t kColAcc = 0, kColSFW = 64, kColSFX = 64 + 16 * CH;
  // FP32 partial staged row-major over the first stages: row r's BN tokens at
  // r * kPartLd floats; the 4-float pad spreads a quarter-warp's 128-bit
  // accesses over all 32 banks.
  static constexpr int kPartLd = BN + 4;
  static constexpr int kPartialBytes = kPartLd * BM * 4;
  static constexpr int kSmemBytes = kStages * kStageBytes + 1024 + 512;
  static_assert(kPartialBytes <= kStages * kStageBytes, "partial fits in the stage buffers");
  static_assert(kColSFX + 16 * CH <= kTmemCols, "scales fit in TMEM");
  static_assert(kStages >= 2, "at least two stages");
};
constexpr int kMaxStages = 12;

struct DecodeArgs {
  int64_t M, N, K;
  int num_k_stages, split;
  int w_prefetch;   // W is not written by the kernel before this one on the stream
  int l2_prefetch;  // W fits in L2: request a CTA's whole W range up front
  const float* g_a;
  const float* seg_scale;
  int nseg;
  EpiSegment seg[kMaxSeg];
};

struct Tail {
  uint64_t full[kMaxStages];
  uint64_t empty[kMaxStages];
  uint64_t tmem_full;
  uint64_t drain;
  uint32_t tmem_base;
  int abort_flag;
};

__device__ __forceinline__ float sigmoid_f(float y) { return 1.0f / (1.0f + expf(-y)); }
__device__ __forceinline__ float softplus_f(float t) {
  return t > 0.0f ? t + log1pf(expf(-t)) : log1pf(expf(t));
}

template <int BN, int CH>
__global__ void __launch_bounds__(kThreads, 1)
    decode_kernel(const __grid_constant__ CUtensorMap tm_w, const __grid_constant__ CUtensorMap tm_x,
                  const __grid_constant__ CUtensorMap tm_sfw, const __grid_constant__ CUtensorMap tm_sfx,
                  const __grid_constant__ DecodeArgs args) {
  using C = DCfg<BN, CH>;
  constexpr int kStages = C::kStages;
  constexpr int kStageBytes = C::kStageBytes;
  constexpr int kWBytes = C::kWBytes;
  constexpr int kXBytes = C::kXBytes;
  constexpr int kSFWBytes = C::kSFWBytes;
  constexpr uint32_t kColAcc = C::kColAcc, kColSFW = C::kColSFW, kColSFX = C::kColSFX;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  Tail* tail = reinterpret_cast<Tail*>(smem + kStages * kStageBytes);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_rank();
  const int S = args.split;
  const int rb = blockIdx.x / S;
  const int ks0 = static_cast<int>((static_cast<int64_t>(rank) * args.num_k_stages) / S);
  const int ks1 = static_cast<int>((static_cast<int64_t>(rank + 1) * args.num_k_stages) / S);
  volatile int* abort_flag = &tail->abort_flag;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&tail->full[s], 1);
      mbar_init(&tail->empty[s], 1);
    }
    mbar_init(&tail->tmem_full, 1);
    mbar_init(&tail->drain, 1);
    tail->abort_flag = 0;
    fence_mbarrier_init();
    prefetch_tmap(&tm_w);
    prefetch_tmap(&tm_x);
    prefetch_tmap(&tm_sfw);
    prefetch_tmap(&tm_sfx);
  }
  if (warp == 1) {
    tmem_alloc(&tail->tmem_base, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  // every CTA of the cluster has initialised its barriers before any remote arrive
  cluster_sync_all();
  tc_fence_after();
  const uint32_t tmem = tail->tmem_base;

  if (warp == 0) {
    if (elect_one()) {
      // W codes + scales, then X codes + scales, of K-stage ks into stage st;
      // one full barrier completes on the bytes of all four copies.
      auto load_w = [&](int stage, int ks) {
        uint8_t* st = smem + stage * kStageBytes;
        if constexpr (CH == 1)
          tma_load_2d(st, &tm_w, &tail->full[stage], ks * (BK / 2), rb * BM);
        else
          tma_load_3d(st, &tm_w, &tail->full[stage], 0, rb * BM, ks * CH);
        tma_load_3d(st + kWBytes + kXBytes, &tm_sfw, &tail->full[stage], 0, ks * 4 * CH, rb);
      };
      auto load_x = [&](int stage, int ks) {
        uint8_t* st = smem + stage * kStageBytes;
        if constexpr (CH == 1)
          tma_load_2d(st + kWBytes, &tm_x, &tail->full[stage], ks * (BK / 2), 0);
        else
          tma_load_3d(st + kWBytes, &tm_x, &tail->full[stage], 0, 0, ks * CH);
        tma_load_3d(st + kWBytes + kXBytes + kSFWBytes, &tm_sfx, &tail->full[stage], 0, ks * 4 * CH, 0);
      };
      int stage = 0;
      uint32_t phase = 0;
      bool issued[kStages] = {};
      uint32_t issued_phase[kStages] = {};
      // Weights may stream before the previous kernel (the activation
      // quantiser) has finished: fill the first stages with W only, and
      // request the rest of this CTA's W range into L2 (when W fits there),
      // so that HBM streams W while the quantiser runs.  (Issued after the
      // wait instead, with nothing to overlap, the L2 requests only compete
      // with the stage loads; standalone calls skip them.)
      const int npre = args.w_prefetch ? min(kStages, ks1 - ks0) : 0;
      for (int i = 0; i < npre; ++i) {
        mbar_arrive_expect_tx(&tail->full[i], C::kStageRaw);
        load_w(i, ks0 + i);
        issued[i] = true;
      }
      if (args.w_prefetch && args.l2_prefetch)
        for (int ks = ks0 + npre; ks < ks1; ++ks) {
          if constexpr (CH == 1)
            tma_prefetch_l2_2d(&tm_w, ks * (BK / 2), rb * BM);
          else
            tma_prefetch_l2_3d(&tm_w, 0, rb * BM, ks * CH);
          tma_prefetch_l2_3d(&tm_sfw, 0, ks * 4 * CH, rb);
        }
      grid_dependency_wait();
      grid_launch_dependents();
      for (int ks = ks0; ks < ks1; ++ks) {
        if (ks - ks0 >= npre) {
          if (!mbar_wait_bounded(&tail->empty[stage], phase ^ 1u, abort_flag)) break;
          mbar_arrive_expect_tx(&tail->full[stage], C::kStageRaw);
          load_w(stage, ks);
        }
        load_x(stage, ks);
        issued[stage] = true;
        issued_phase[stage] = phase;
        if (++stage == kStages) { stage = 0; phase ^= 1u; }
      }
      if (*abort_flag)
        for (int s = 0; s < kStages; ++s)
          if (issued[s]) mbar_wait_bounded(&tail->full[s], issued_phase[s], nullptr, 200000000ull);
    }
  } else if (warp == 1) {
    if (elect_one()) {
      // E2M1 x E2M1, UE4M3 scales, K-major, M = 128 (weights), N = 64 (tokens)
      const uint32_t idesc = (1u << 7) | (1u << 10) | (static_cast<uint32_t>(BN >> 3) << 17) |
                             (static_cast<uint32_t>(BM >> 4) << 24);
      const uint32_t base = smem_u32(smem);
      int stage = 0;
      uint32_t phase = 0;
      bool any = false;
      for (int ks = ks0; ks < ks1; ++ks) {
        if (!mbar_wait_bounded(&tail->full[stage], phase, abort_flag)) break;
        tc_fence_after();
        const uint32_t sw = base + stage * kStageBytes;
        const uint32_t sx = sw + kWBytes;
        const uint32_t ssfw = sx + kXBytes;
        const uint32_t ssfx = ssfw + kSFWBytes;
#pragma unroll
        for (int kb = 0; kb < 4 * CH; ++kb) {
          tmem_cp_32x128b_warpx4(tmem + kColSFW + 4 * kb, make_smem_desc(ssfw + 512 * kb, 0, 128, kLayoutSwizzleNone));
          tmem_cp_32x128b_warpx4(tmem + kColSFX + 4 * kb, make_smem_desc(ssfx + 512 * kb, 0, 128, kLayoutSwizzleNone));
        }
#pragma unroll
        for (int c = 0; c < CH; ++c) {
          const uint64_t wdesc = make_smem_desc(sw + c * (BM * BK / 2), 16, 1024, kLayoutSwizzle128B);
          const uint64_t xdesc = make_smem_desc(sx + c * C::kXPlane, 16, 1024, kLayoutSwizzle128B);
#pragma unroll
          for (int j = 0; j < 4; ++j)
            mma_mxf4nvf4(tmem + kColAcc, wdesc + 2 * j, xdesc + 2 * j, idesc, tmem + kColSFW + 4 * (4 * c + j),
                         tmem + kColSFX + 4 * (4 * c + j), (ks > ks0 || c > 0 || j > 0) ? 1u : 0u);
        }
        any = true;
        tc_commit(&tail->empty[stage]);
        if (++stage == kStages) { stage = 0; phase ^= 1u; }
      }
      if (any) tc_commit(&tail->tmem_full);  // also the drain point on abort
    }
  } else {
    // ------------------------------------------------------------ epilogue
    grid_dependency_wait();  // g_a, the segment scales and the outputs
    const int q = warp & 3;
    const int row_local = q * 32 + lane;
    float acc[BN];
    bool have = (ks1 > ks0) && mbar_wait_bounded(&tail->tmem_full, 0, abort_flag);
    if (have) {
      tc_fence_after();
      const uint32_t lane_addr = tmem + (static_cast<uint32_t>(q * 32) << 16);
      if constexpr (BN == 64) {
        uint32_t r0[32], r1[32];
        tmem_ld_32x32b_x32(lane_addr + kColAcc, r0);
        tmem_ld_32x32b_x32(lane_addr + kColAcc + 32, r1);
        tmem_ld_wait();
#pragma unroll
        for (int t = 0; t < 32; ++t) {
          acc[t] = __uint_as_float(r0[t]);
          acc[32 + t] = __uint_as_float(r1[t]);
        }
      } else if constexpr (BN == 32) {
        uint32_t r0[32];
        tmem_ld_32x32b_x32(lane_addr + kColAcc, r0);
        tmem_ld_wait();
#pragma unroll
        for (int t = 0; t < 32; ++t) acc[t] = __uint_as_float(r0[t]);
      } else {
        uint32_t r0[16];
        tmem_ld_32x32b_x16(lane_addr + kColAcc, r0);
        tmem_ld_wait();
#pragma unroll
        for (int t = 0; t < 16; ++t) acc[t] = __uint_as_float(r0[t]);
      }
    } else {
#pragma unroll
      for (int t = 0; t < BN; ++t) acc[t] = 0.0f;
    }
    tc_fence_before();
    // this CTA's FP32 partial, row-major ([row][token], row stride kPartLd),
    // staged in its stage buffers for the whole cluster to read
    float* partial = reinterpret_cast<float*>(smem) + row_local * C::kPartLd;
#pragma unroll
    for (int t = 0; t < BN; t += 4)
      *reinterpret_cast<float4*>(partial + t) = make_float4(acc[t], acc[t + 1], acc[t + 2], acc[t + 3]);
  }
  // every CTA of the cluster has staged its partial
  cluster_sync_all();
  if (warp >= 2) {
    // This CTA finalises token groups [g0, g1) of 4 tokens: the sum of the
    // ranks' partials in rank order (the same arithmetic whichever CTA does
    // it), then the segment's epilogue.  Tokens >= M are zero rows of X and
    // are never stored.
    const int q = warp & 3;
    const int row_local = q * 32 + lane;
    const int64_t n = static_cast<int64_t>(rb) * BM + row_local;
    constexpr int kG = BN / 4;
    const int G = (static_cast<int>(args.M) + 3) / 4;
    const int g0 = static_cast<int>(rank) * G / S, g1 = (static_cast<int>(rank) + 1) * G / S;
    float4 sum[kG];
#pragma unroll
    for (int i = 0; i < kG; ++i) sum[i] = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
    const uint32_t mine = smem_u32(reinterpret_cast<float*>(smem) + row_local * C::kPartLd);
    for (int p = 0; p < S; ++p) {
      const uint32_t src = map_to_rank(mine, static_cast<uint32_t>(p));
      float4 v[kG];
      // every load of this rank is issued before the first add
#pragma unroll
      for (int i = 0; i < kG; ++i)
        if (g0 + i < g1) v[i] = ld_shared_cluster_f32x4(src + 16u * static_cast<uint32_t>(g0 + i));
#pragma unroll
      for (int i = 0; i < kG; ++i)
        if (g0 + i < g1) {
          sum[i].x += v[i].x;
          sum[i].y += v[i].y;
          sum[i].z += v[i].z;
          sum[i].w += v[i].w;
        }
    }
    if (g1 > g0 && n < args.N) {
      int s = 0;
#pragma unroll
      for (int i = 1; i < kMaxSeg; ++i)
        if (i < args.nseg && n >= args.seg[i].n_begin) s = i;
      // the segment's parameters, loaded once; one tight loop per kind
      const int kind = args.seg[s].kind;
      const int64_t ld = args.seg[s].ld_out;
      const int64_t j = n - args.seg[s].n_begin;
      const float scale = __ldg(args.g_a) * __ldg(args.seg_scale + s);
      const int mt = static_cast<int>(args.M);
      float a_log = 0.0f, dt = 0.0f;
      if (kind == NVFP4_EPI_GDN_DECAY_F32) {
        a_log = -expf(__ldg(args.seg[s].a_log + j));
        dt = __ldg(args.seg[s].dt_bias + j);
      }
#pragma unroll
      for (int i = 0; i < kG; ++i) {
        if (g0 + i >= g1) break;
        const int t0 = 4 * (g0 + i);
        const float y[4] = {sum[i].x * scale, sum[i].y * scale, sum[i].z * scale, sum[i].w * scale};
        if (kind == NVFP4_EPI_IDENTITY_BF16) {
          __nv_bfloat16* o = static_cast<__nv_bfloat16*>(args.seg[s].out) + j;
#pragma unroll
          for (int c = 0; c < 4; ++c)
            if (t0 + c < mt) o[(t0 + c) * ld] = __float2bfloat16_rn(y[c]);
        } else if (kind == NVFP4_EPI_IDENTITY_F32) {
          float* o = static_cast<float*>(args.seg[s].out) + j;
#pragma unroll
          for (int c = 0; c < 4; ++c)
            if (t0 + c < mt) o[(t0 + c) * ld] = y[c];
        } else if (kind == NVFP4_EPI_SIGMOID_F32) {
          float* o = static_cast<float*>(args.seg[s].out) + j;
#pragma unroll
          for (int c = 0; c < 4; ++c)
            if (t0 + c < mt) o[(t0 + c) * ld] = sigmoid_f(y[c]);
        } else {
          float* o = static_cast<float*>(args.seg[s].out) + j;
#pragma unroll
          for (int c = 0; c < 4; ++c)
            if (t0 + c < mt) o[(t0 + c) * ld] = a_log * softplus_f(y[c] + dt);
        }
      }
    }
  }

  // no CTA leaves (or reuses its shared memory) while another may read it
  tc_fence_before();
  cluster_sync_all();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

}  // namespace dk

bool decode_path_applies(const GemmProblem& p) { return p.M >= 1 && p.M <= 64 && !p.swiglu; }

namespace dk {

// Codes [rows, K/2] viewed as {128 B, rows, K/256}: one box spans CH chunks of
// box_rows rows (needs K % 256 == 0 so that every chunk lies inside its row).
bool make_codes_map3(CUtensorMap* m, const uint8_t* codes, int64_t rows, int64_t K, uint32_t box_rows, uint32_t chunks) {
  const cuuint64_t dims[3] = {128, static_cast<cuuint64_t>(rows), static_cast<cuuint64_t>(K / 256)};
  const cuuint64_t strides[2] = {static_cast<cuuint64_t>(K / 2), 128};
  const cuuint32_t box[3] = {128, box_rows, chunks};
  const cuuint32_t estr[3] = {1, 1, 1};
  return gk::encode_fn()(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<uint8_t*>(codes), dims, strides, box, estr,
                         CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                         CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int BN, int CH>
cudaError_t launch_bn(const GemmProblem& p, cudaStream_t stream) {
  using C = DCfg<BN, CH>;
  CUtensorMap tm_w, tm_x, tm_sfw, tm_sfx;
  bool ok;
  if constexpr (CH == 1)
    ok = gk::make_codes_map(&tm_w, p.w_codes, p.N, p.K, BM) && gk::make_codes_map(&tm_x, p.a_codes, p.M, p.K, BN);
  else
    ok = make_codes_map3(&tm_w, p.w_codes, p.N, p.K, BM, CH) && make_codes_map3(&tm_x, p.a_codes, p.M, p.K, BN, CH);
  if (!ok || !gk::make_sf_map(&tm_sfw, p.w_sf, p.N, p.K, 4 * CH, 1) || !gk::make_sf_map(&tm_sfx, p.a_sf, p.M, p.K, 4 * CH, 1))
    return cudaErrorInvalidValue;
  DecodeArgs a{};
  a.M = p.M;
  a.N = p.N;
  a.K = p.K;
  a.w_prefetch = p.w_prefetch ? 1 : 0;
  a.l2_prefetch = static_cast<double>(p.N) * static_cast<double>(p.K) * (0.5 + 1.0 / 16) <= 64.0 * 1024 * 1024;
  a.num_k_stages = static_cast<int>(ceil_div(ceil_div(p.K, BK), CH));
  a.g_a = p.g_a;
  a.seg_scale = p.seg_scale;
  a.nseg = p.nseg;
  for (int i = 0; i < p.nseg; ++i) a.seg[i] = p.seg[i];
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int rbs = static_cast<int>(ceil_div(p.N, BM));
  int S = sms / rbs;
  if (S > 8) S = 8;
  if (S > a.num_k_stages) S = a.num_k_stages;
  if (S < 1) S = 1;
  a.split = S;
  static std::atomic<uint64_t> attr_done{0};
  cudaError_t ea = once_per_device(attr_done, [] {
    return cudaFuncSetAttribute(decode_kernel<BN, CH>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes);
  });
  if (ea != cudaSuccess) return ea;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(rbs * S);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = C::kSmemBytes;
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = S;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  return cudaLaunchKernelEx(&cfg, decode_kernel<BN, CH>, tm_w, tm_x, tm_sfw, tm_sfx, a);
}
}  // namespace dk

cudaError_t launch_gemm_decode(const GemmProblem& p, cudaStream_t stream) {
  const bool wide = p.K % 256 == 0;
  // Stages of two 256-K chunks (44 KB with 16 tokens, four stages) for up to
  // 32 tokens and of one chunk for 64 tokens: measured in chains of
  // launches, finer stages than four chunks (88 KB, two stages) keep more of
  // the weight stream in flight (M = 1: 12.0 -> 11.3 us; M = 64: 16.2 ->
  // 15.9 us).
  if (p.M <= 16) return wide ? dk::launch_bn<16, 2>(p, stream) : dk::launch_bn<16, 1>(p, stream);
  if (p.M <= 32) return wide ? dk::launch_bn<32, 2>(p, stream) : dk::launch_bn<32, 1>(p, stream);
  return dk::launch_bn<64, 1>(p, stream);
}

}  // namespace nvfp4
