// Gated delta-rule recurrence over the fused projection's outputs, sm_100a.
//
// "Why Gated DeltaNet Survives 4-Bit Quantization" (ai.info summary), "Main
// Findings", recurrence bullet: a fixed-size state per head, every write
// overwrites along the current key, with a decay alpha and a write strength
// beta; gate-parameterisation bullet: the decay gate is emitted in log space
// (g = -exp(A_log) softplus(a + dt_bias)), so alpha = exp(g).  Per value head,
// with the state S [d_v, d_k] in FP32 and q, k L2-normalised (q also scaled):
//     S_t = alpha_t S_{t-1} + beta_t (v_t - alpha_t S_{t-1} k_t) k_t^T,
//     o_t = S_t q_t.
//
// Chunked evaluation, C = 64 tokens per chunk.  With S the state entering a
// chunk and gam the inclusive running sum of g inside it:
//     A[t][j] = beta_t e^(gam_t - gam_j) k_t.k_j   (j < t),   L = (I + A)^-1
//     W = L diag(beta e^gam) K,     U~ = L diag(beta) V
//     P[t][j] = e^(gam_t - gam_j) q_t.k_j          (j <= t)
//     Kd = diag(e^(gam_C - gam)) K
//     M = e^gam_C I - W^T Kd,  N = U~^T Kd,  R = diag(e^gam) Q - P W,  Y = P U~
//     S' = S M + N,   O = R S^T + Y.
// (Unrolling the token recurrence over the chunk gives these: the corrections
// u_t written inside the chunk solve (I + A) U = diag(beta) (V - diag(e^gam) K S^T).)
// Only the last line depends on S.  gdn_prep_kernel builds [M^T; R], N and
// Y^T for every (chunk, head) at once; gdn_state_kernel then walks the chunks
// in order, one CTA per (head, 32 state rows) -- rows of S evolve
// independently -- keeping S in shared memory.
//
// The contractions run on the tensor cores as warp-level TF32 MMAs
// (m16n8k8, FP32 accumulate): every product here is a 64-wide tile inside a
// chain of dependent steps (Gram matrix -> triangular solve -> products ->
// state), where register fragments avoid a round trip through tensor memory
// between steps.  Operands are rounded to TF32 (nearest, ties away); the
// state and all sums stay FP32, and the triangular inverse keeps about FP32
// accuracy (FP32 substitution inside the 16 x 16 diagonal blocks, 3xTF32
// products for the blocks below them).
#include <cstdint>

#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "internal.h"
#include "ptx.cuh"

namespace nvfp4 {
namespace gdn {

constexpr int C = 64;        // tokens per chunk
constexpr int DK = 64;       // key / query head dimension
constexpr int DV = 128;      // value head dimension
constexpr int LD64 = 68;     // padded row stride (floats) of 64-wide tiles in shared memory
constexpr int kThreads = 256;
constexpr int kRows = 32;    // state rows per CTA of the state pass
constexpr int kRec = 3 * 128 * 64;  // floats per (chunk, head) record: [M^T; R], N, Y^T

// Element (r, c) of a row-major tile of 64-float rows whose 16-byte pieces are
// XOR-swizzled by the row: piece c / 4 of row r sits at piece (c / 4) ^ (r % 8).
// Eight consecutive rows then place any one piece in eight different bank
// groups, so 8-row fragment loads are conflict-free without padding and a tile
// moves as one contiguous copy.  The records use this layout in global memory.
__device__ __forceinline__ int sw64(int r, int c) { return r * 64 + (((c >> 2) ^ (r & 7)) << 2) + (c & 3); }

struct GdnArgs {
  const uint8_t* q;
  const uint8_t* k;
  const uint8_t* v;
  int64_t ld_q, ld_k, ld_v;  // bytes
  const float* beta;
  const float* g;
  int64_t ld_beta, ld_g;     // elements
  int64_t T;
  int H, rep;                // value heads; value heads per query/key head
  int nchunks;
  float scale, eps;
  const float* h0;           // [H, DV, DK] or null
  float* h_out;              // [H, DV, DK] or null
  uint8_t* o;
  int64_t ld_o;              // bytes
  int out_f32;
  float* ws;                 // nchunks * H records
};

__device__ __forceinline__ uint32_t tf32(float x) {
  uint32_t r;
  asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(r) : "f"(x));
  return r;
}

// D += A B, m16n8k8, A row-major 16x8, B 8x8 (k rows), TF32 in, FP32 accumulate.
__device__ __forceinline__ void mma(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k8.row.col.f32.tf32.tf32.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// d += a b to about FP32 accuracy with three TF32 products (x = hi + lo, both
// TF32; the lo * lo term, below 2^-22 relative, is dropped).
__device__ __forceinline__ void split_tf32(float x, uint32_t& hi, uint32_t& lo) {
  hi = tf32(x);
  lo = tf32(x - __uint_as_float(hi));
}
__device__ __forceinline__ void mma_3xtf32(float (&d)[4], const float (&a)[4], float b0, float b1) {
  uint32_t ah[4], alo[4], bh0, bl0, bh1, bl1;
#pragma unroll
  for (int i = 0; i < 4; ++i) split_tf32(a[i], ah[i], alo[i]);
  split_tf32(b0, bh0, bl0);
  split_tf32(b1, bh1, bl1);
  mma(d, alo, bh0, bh1);
  mma(d, ah, bl0, bl1);
  mma(d, ah, bh0, bh1);
}

// Fragment layouts (gid = lane / 4, tig = lane % 4).  An A fragment holds
// (m0+gid, k0+tig), (m0+gid+8, k0+tig), (m0+gid, k0+tig+4), (m0+gid+8, k0+tig+4);
// a B fragment (k0+tig, n0+gid), (k0+tig+4, n0+gid); the accumulator
// (m0+gid, n0+2tig), (m0+gid, n0+2tig+1), (m0+gid+8, n0+2tig), (m0+gid+8, n0+2tig+1).
//
// Both operand fragments are blocks of 8 rows x 4 consecutive FP32 words of a
// row-major tile (for B, a tile stored with n as the row), which is what
// ldmatrix distributes: four 8 x 8 matrices of 16-bit elements, lane l
// supplying the address of row l % 8 of matrix l / 8 and receiving word
// (row l / 4, column l % 4) of every matrix.  Tiles in shared memory have row
// strides of 68 floats (17 pieces of 16 bytes), so eight consecutive rows hit
// eight different bank groups.
__device__ __forceinline__ void ldsm_x4(uint32_t (&r)[4], uint32_t addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr)
               : "memory");
}
// A[m][k] = X[m][k], rows m0 .. m0+15, columns k0 .. k0+7 (X row-major, stride ld).
__device__ __forceinline__ void lda(uint32_t (&a)[4], const float* X, int ld, int m0, int k0, int lane) {
  const int rr = lane & 7, j = lane >> 3;
  ldsm_x4(a, smem_u32(X + (m0 + rr + 8 * (j & 1)) * ld + k0 + 4 * (j >> 1)));
}
// B[k][n] = X[n][k] for columns n0 .. n0+7 and two k-steps: b[0], b[1] at k0,
// b[2], b[3] at k0 + 8.
__device__ __forceinline__ void ldb2(uint32_t (&b)[4], const float* X, int ld, int n0, int k0, int lane) {
  ldsm_x4(b, smem_u32(X + (n0 + (lane & 7)) * ld + k0 + 4 * (lane >> 3)));
}
template <int N>
__device__ __forceinline__ void round_tf32(uint32_t (&r)[N]) {
#pragma unroll
  for (int i = 0; i < N; ++i) r[i] = tf32(__uint_as_float(r[i]));
}
// B[k][n] = s[k] X[k][n] (X stored with k as the row), rounded to TF32.
__device__ __forceinline__ void frag_b(uint32_t& b0, uint32_t& b1, const float* X, int ld, const float* s, int n0,
                                       int k0, int gid, int tig) {
  b0 = tf32(s[k0 + tig] * X[(k0 + tig) * ld + n0 + gid]);
  b1 = tf32(s[k0 + tig + 4] * X[(k0 + tig + 4) * ld + n0 + gid]);
}

// 16 consecutive elements (BF16 or F32) -> FP32.
template <int DTYPE>
__device__ __forceinline__ void load16(const uint8_t* p, float (&f)[16]) {
  if constexpr (DTYPE == NVFP4_DTYPE_BF16) {
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const uint4 w = *reinterpret_cast<const uint4*>(p + 16 * h);
      const uint32_t u[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        f[8 * h + 2 * i] = __uint_as_float(u[i] << 16);
        f[8 * h + 2 * i + 1] = __uint_as_float(u[i] & 0xFFFF0000u);
      }
    }
  } else {
#pragma unroll
    for (int h = 0; h < 4; ++h) {
      const float4 w = *reinterpret_cast<const float4*>(p + 16 * h);
      f[4 * h] = w.x;
      f[4 * h + 1] = w.y;
      f[4 * h + 2] = w.z;
      f[4 * h + 3] = w.w;
    }
  }
}

struct PrepSmem {
  float q[C * LD64];   // q^ rows (normalised and scaled), FP32
  float k[C * LD64];   // k^ rows, FP32; from step 3 on K_d^T [d_k][token] (TF32)
  float al[C * LD64];  // A, then L (TF32), then W^T [d_k][token] (TF32)
  float p[C * LD64];   // P (TF32)
  float vt[DV * LD64]; // (diag(beta) V)^T [value][token] (TF32), then U~^T
  float gam[C];        // inclusive running sum of g
  float beta[C];
  float bg[C];         // beta e^gam
  float eg[C];         // e^gam
  float kdec[C];       // e^(gam_C - gam)
  float tmp[6 * 144];  // per-warp 16 x 8 parts of T in the triangular inverse (row stride 9)
};

// One CTA per (chunk, value head): the S-independent matrices of the chunk.
// Every operand fragment is read with ldmatrix from a row-major tile, so the
// matrices that are contracted over tokens (W, U~, K_d, diag(beta) V) are kept
// transposed, token index along the row.
template <int DTYPE>
__global__ void __launch_bounds__(kThreads, 2) gdn_prep_kernel(const __grid_constant__ GdnArgs a) {
  extern __shared__ __align__(16) uint8_t smem_raw[];
  PrepSmem& s = *reinterpret_cast<PrepSmem*>(smem_raw);
  constexpr int kEsz = DTYPE == NVFP4_DTYPE_BF16 ? 2 : 4;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int gid = lane >> 2, tig = lane & 3;
  const int c = blockIdx.x, h = blockIdx.y, hq = h / a.rep;
  const int64_t t0 = static_cast<int64_t>(c) * C;

  grid_dependency_wait();
  if (tid == 0) grid_launch_dependents();

  // decay and write strength of tokens 2 lane and 2 lane + 1 (warp 0), loaded
  // together with q, k and v
  float ga = 0.0f, gb = 0.0f, ba = 0.0f, bb = 0.0f;
  if (warp == 0) {
    const int64_t ta = t0 + 2 * lane, tb = ta + 1;
    if (ta < a.T) {
      ga = a.g[ta * a.ld_g + h];
      ba = a.beta[ta * a.ld_beta + h];
    }
    if (tb < a.T) {
      gb = a.g[tb * a.ld_g + h];
      bb = a.beta[tb * a.ld_beta + h];
    }
  }
  {
    // q, k rows: four threads per row, 16 elements each.  v: one token per
    // lane, 32 consecutive values per thread (so the transposed writes below
    // are conflict-free).  Every load is issued before any is used.
    const int row = tid >> 2, part = tid & 3;
    const int64_t t = t0 + row;
    const int vrow = lane + 32 * (warp & 1), vcol = 32 * (warp >> 1);
    const int64_t tv = t0 + vrow;
    float fq[16], fk[16], fv[2][16], bv = 0.0f;
    if (t < a.T) {
      load16<DTYPE>(a.q + t * a.ld_q + (static_cast<int64_t>(hq) * DK + part * 16) * kEsz, fq);
      load16<DTYPE>(a.k + t * a.ld_k + (static_cast<int64_t>(hq) * DK + part * 16) * kEsz, fk);
    } else {
#pragma unroll
      for (int i = 0; i < 16; ++i) fq[i] = fk[i] = 0.0f;
    }
    if (tv < a.T) {
      const uint8_t* src = a.v + tv * a.ld_v + (static_cast<int64_t>(h) * DV + vcol) * kEsz;
      load16<DTYPE>(src, fv[0]);
      load16<DTYPE>(src + 16 * kEsz, fv[1]);
      bv = a.beta[tv * a.ld_beta + h];
    } else {
#pragma unroll
      for (int i = 0; i < 16; ++i) fv[0][i] = fv[1][i] = 0.0f;
    }
    // L2 norms in FP32
    float sq = 0.0f, sk = 0.0f;
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      sq = fmaf(fq[i], fq[i], sq);
      sk = fmaf(fk[i], fk[i], sk);
    }
    sq += __shfl_xor_sync(0xffffffffu, sq, 1);
    sk += __shfl_xor_sync(0xffffffffu, sk, 1);
    sq += __shfl_xor_sync(0xffffffffu, sq, 2);
    sk += __shfl_xor_sync(0xffffffffu, sk, 2);
    const float iq = a.scale / sqrtf(sq + a.eps), ik = 1.0f / sqrtf(sk + a.eps);
#pragma unroll
    for (int i = 0; i < 16; i += 4) {
      *reinterpret_cast<float4*>(&s.q[row * LD64 + part * 16 + i]) =
          make_float4(fq[i] * iq, fq[i + 1] * iq, fq[i + 2] * iq, fq[i + 3] * iq);
      *reinterpret_cast<float4*>(&s.k[row * LD64 + part * 16 + i]) =
          make_float4(fk[i] * ik, fk[i + 1] * ik, fk[i + 2] * ik, fk[i + 3] * ik);
    }
    // V is read only as diag(beta) V, a TF32 operand: scaled, rounded and
    // transposed here once
#pragma unroll
    for (int hh = 0; hh < 2; ++hh)
#pragma unroll
      for (int i = 0; i < 16; ++i) s.vt[(vcol + 16 * hh + i) * LD64 + vrow] = __uint_as_float(tf32(bv * fv[hh][i]));
  }
  // ---- gates: running sum of the log decay inside the chunk (warp 0)
  if (warp == 0) {
    const float pair = ga + gb;
    float run = pair;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const float y = __shfl_up_sync(0xffffffffu, run, off);
      if (lane >= off) run += y;
    }
    const float excl = run - pair;
    const float gma = excl + ga, gmb = excl + ga + gb;
    const float gC = __shfl_sync(0xffffffffu, gmb, 31);
    s.gam[2 * lane] = gma;
    s.gam[2 * lane + 1] = gmb;
    s.beta[2 * lane] = ba;
    s.beta[2 * lane + 1] = bb;
    const float ea = expf(gma), eb = expf(gmb);
    s.eg[2 * lane] = ea;
    s.eg[2 * lane + 1] = eb;
    s.bg[2 * lane] = ba * ea;
    s.bg[2 * lane + 1] = bb * eb;
    s.kdec[2 * lane] = expf(gC - gma);
    s.kdec[2 * lane + 1] = expf(gC - gmb);
  }
  __syncthreads();

  // ---- step 1: Gram matrices K K^T (-> A) and Q K^T (-> P), lower triangle.
  // The 20 tiles (mt, nt) with nt <= 2 mt + 1 of each matrix go five to a
  // warp: w = warp % 4 takes half of the tiles of row block 3 (w < 2) or 2,
  // and half of those of row block 0 or 1.  The five tiles are independent
  // accumulations, interleaved.
  {
    const int mat = warp >> 2, w4 = warp & 3;
    const float* X = mat == 0 ? s.k : s.q;
    float* out = mat == 0 ? s.al : s.p;
    const int mt_big = w4 < 2 ? 3 : 2, mt_small = 3 - mt_big;
    const int nb = mt_big + 1;  // tiles of the big row block; 5 - nb of the small one
    const int nb0 = (w4 & 1) * nb, ns0 = (w4 & 1) * (5 - nb);
    float d[5][4];
#pragma unroll
    for (int i = 0; i < 5; ++i) d[i][0] = d[i][1] = d[i][2] = d[i][3] = 0.0f;
#pragma unroll
    for (int kp = 0; kp < 4; ++kp) {
      uint32_t ab0[4], ab1[4], as0[4], as1[4];
      lda(ab0, X, LD64, 16 * mt_big, 16 * kp, lane);
      lda(ab1, X, LD64, 16 * mt_big, 16 * kp + 8, lane);
      lda(as0, X, LD64, 16 * mt_small, 16 * kp, lane);
      lda(as1, X, LD64, 16 * mt_small, 16 * kp + 8, lane);
      round_tf32(ab0);
      round_tf32(ab1);
      round_tf32(as0);
      round_tf32(as1);
#pragma unroll
      for (int i = 0; i < 5; ++i) {
        const bool big = i < nb;
        const int nt = big ? nb0 + i : ns0 + i - nb;
        uint32_t b[4], a0[4], a1[4];
        ldb2(b, s.k, LD64, 8 * nt, 16 * kp, lane);
        round_tf32(b);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          a0[e] = big ? ab0[e] : as0[e];
          a1[e] = big ? ab1[e] : as1[e];
        }
        mma(d[i], a0, b[0], b[1]);
        mma(d[i], a1, b[2], b[3]);
      }
    }
#pragma unroll
    for (int i = 0; i < 5; ++i) {
      const bool big = i < nb;
      const int mt = big ? mt_big : mt_small, nt = big ? nb0 + i : ns0 + i - nb;
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int t = 16 * mt + gid + (e >= 2 ? 8 : 0), j = 8 * nt + 2 * tig + (e & 1);
        float val = 0.0f;
        if (mat == 0) {
          if (j < t) val = s.beta[t] * __expf(s.gam[t] - s.gam[j]) * d[i][e];
        } else {
          // P is read only as a TF32 MMA operand: rounded here once
          if (j <= t) val = __uint_as_float(tf32(__expf(s.gam[t] - s.gam[j]) * d[i][e]));
        }
        out[t * LD64 + j] = val;
      }
    }
  }
  __syncthreads();

  // ---- step 2: L = (I + A)^-1 with A strictly lower triangular, in 16 x 16
  // blocks: the diagonal blocks by forward substitution (one column per
  // thread, FP32), then one block diagonal at a time
  //     L_ij = -L_ii T,  T = sum_{m=j}^{i-1} A_im L_mj   (i > j)
  // with 3xTF32 tensor products (about FP32 accuracy).  While A is still
  // read, L is built transposed in al's strict upper triangle.
  {
    if (tid < C) {
      const int base = 16 * (tid >> 4), jj = tid & 15;
      float col[16];
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        float acc0 = 0.0f, acc1 = 0.0f;
#pragma unroll
        for (int m = 0; m < i; ++m) {
          const float a = s.al[(base + i) * LD64 + base + m];
          if (m & 1) acc1 = fmaf(a, col[m], acc1);
          else acc0 = fmaf(a, col[m], acc0);
        }
        col[i] = (i == jj ? 1.0f : 0.0f) - (acc0 + acc1);
      }
#pragma unroll
      for (int i = 0; i < 16; ++i)
        if (i > jj) s.al[(base + jj) * LD64 + base + i] = col[i];
    }
    __syncthreads();
    // Off-diagonal blocks, one block diagonal dd at a time; warp w takes
    // block (i, j) = (w / 2 + dd, w / 2) and its 8 columns 8 (w % 2) .. +7:
    // T = sum_{m=j}^{i-1} A_im L_mj, then L_ij = -L_ii T, both on the tensor
    // cores in 3xTF32, even and odd k-steps in separate accumulators.
    // lval(mb, j, r, c) = L[16mb + r][16j + c] (mb >= j), read from the transposed copy.
    auto lval = [&](int mb, int j, int r, int c) -> float {
      if (mb > j) return s.al[(16 * j + c) * LD64 + 16 * mb + r];
      return r > c ? s.al[(16 * j + c) * LD64 + 16 * j + r] : (r == c ? 1.0f : 0.0f);
    };
    for (int dd = 1; dd < 4; ++dd) {
      if (warp < 2 * (4 - dd)) {
        const int j = warp >> 1, i = j + dd, nt = warp & 1;
        float* tw = &s.tmp[warp * 144];  // this warp's 16 x 8 columns of T, row stride 9
        float t[2][4] = {{0.0f, 0.0f, 0.0f, 0.0f}, {0.0f, 0.0f, 0.0f, 0.0f}};
        for (int mb = j; mb < i; ++mb) {
#pragma unroll
          for (int kk = 0; kk < 2; ++kk) {
            const float* arow = &s.al[(16 * i) * LD64 + 16 * mb + 8 * kk];
            const float a[4] = {arow[gid * LD64 + tig], arow[(gid + 8) * LD64 + tig], arow[gid * LD64 + tig + 4],
                                arow[(gid + 8) * LD64 + tig + 4]};
            mma_3xtf32(t[kk], a, lval(mb, j, 8 * kk + tig, 8 * nt + gid), lval(mb, j, 8 * kk + tig + 4, 8 * nt + gid));
          }
        }
        tw[gid * 9 + 2 * tig] = t[0][0] + t[1][0];
        tw[gid * 9 + 2 * tig + 1] = t[0][1] + t[1][1];
        tw[(gid + 8) * 9 + 2 * tig] = t[0][2] + t[1][2];
        tw[(gid + 8) * 9 + 2 * tig + 1] = t[0][3] + t[1][3];
        __syncwarp();
        float l[2][4] = {{0.0f, 0.0f, 0.0f, 0.0f}, {0.0f, 0.0f, 0.0f, 0.0f}};
#pragma unroll
        for (int kk = 0; kk < 2; ++kk) {
          const float a[4] = {lval(i, i, gid, 8 * kk + tig), lval(i, i, gid + 8, 8 * kk + tig),
                              lval(i, i, gid, 8 * kk + tig + 4), lval(i, i, gid + 8, 8 * kk + tig + 4)};
          mma_3xtf32(l[kk], a, tw[(8 * kk + tig) * 9 + gid], tw[(8 * kk + tig + 4) * 9 + gid]);
        }
        // L_ij, negated, into the transposed copy: L[16i + r][16j + c] at al[16j + c][16i + r]
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int r = gid + (e >= 2 ? 8 : 0), c = 8 * nt + 2 * tig + (e & 1);
          s.al[(16 * j + c) * LD64 + 16 * i + r] = -(l[0][e] + l[1][e]);
        }
      }
      __syncthreads();
    }
    // move L to the lower triangle (unit diagonal, zeros above) for the products
    float mv[16];
#pragma unroll
    for (int e = 0; e < 16; ++e) {
      const int idx = tid + e * kThreads, r = idx >> 6, c = idx & 63;
      mv[e] = r > c ? s.al[c * LD64 + r] : (r == c ? 1.0f : 0.0f);
    }
    __syncthreads();
#pragma unroll
    for (int e = 0; e < 16; ++e) {
      const int idx = tid + e * kThreads, r = idx >> 6, c = idx & 63;
      s.al[r * LD64 + c] = __uint_as_float(tf32(mv[e]));  // read only as a TF32 operand
    }
  }
  __syncthreads();

  // ---- step 3: W = L diag(beta e^gam) K  and  U~ = L diag(beta) V.
  // 24 column tiles (0-7: W, 8-23: U~) x 4 row blocks, 2 mt + 2 k-steps each
  // (L is lower triangular).  Warp w takes column tiles 6 (w % 4) .. +5 of row
  // blocks 3 and 0 (w < 4) or 2 and 1: 60 k-steps for every warp, and the two
  // row blocks share each B fragment.
  {
    const int mt_big = warp < 4 ? 3 : 2, mt_small = 3 - mt_big;
    const int nkb = 2 * mt_big + 2, nks = 2 * mt_small + 2;
    const int ntb = 6 * (warp & 3);
    float db[6][4], ds[6][4];
#pragma unroll
    for (int i = 0; i < 6; ++i)
#pragma unroll
      for (int e = 0; e < 4; ++e) db[i][e] = ds[i][e] = 0.0f;
    // k-step pairs outermost: only two A fragments of each row block are live
#pragma unroll
    for (int kp = 0; kp < 4; ++kp) {
      if (2 * kp >= nkb) continue;
      const bool small = 2 * kp < nks;
      uint32_t ab0[4], ab1[4], as0[4], as1[4];
      lda(ab0, s.al, LD64, 16 * mt_big, 16 * kp, lane);
      lda(ab1, s.al, LD64, 16 * mt_big, 16 * kp + 8, lane);
      if (small) {
        lda(as0, s.al, LD64, 16 * mt_small, 16 * kp, lane);
        lda(as1, s.al, LD64, 16 * mt_small, 16 * kp + 8, lane);
      }
#pragma unroll
      for (int i = 0; i < 6; ++i) {
        const int nt = ntb + i;
        uint32_t b[4];
        if (nt < 8) {
          frag_b(b[0], b[1], s.k, LD64, s.bg, 8 * nt, 16 * kp, gid, tig);
          frag_b(b[2], b[3], s.k, LD64, s.bg, 8 * nt, 16 * kp + 8, gid, tig);
        } else {
          ldb2(b, s.vt, LD64, 8 * (nt - 8), 16 * kp, lane);
        }
        mma(db[i], ab0, b[0], b[1]);
        mma(db[i], ab1, b[2], b[3]);
        if (small) {
          mma(ds[i], as0, b[0], b[1]);
          mma(ds[i], as1, b[2], b[3]);
        }
      }
    }
    // K for K_d, read before the barrier (token j = idx % 64, column n = idx / 64)
    float kr[16];
#pragma unroll
    for (int e = 0; e < 16; ++e) {
      const int idx = tid + e * kThreads;
      kr[e] = s.k[(idx & 63) * LD64 + (idx >> 6)];
    }
    __syncthreads();  // L, V and K are read; W^T goes over L, U~^T over V^T, K_d^T over K
    // W and U~ are read only as TF32 operands: rounded here once, stored transposed
#pragma unroll
    for (int i = 0; i < 6; ++i) {
      const int nt = ntb + i;
      float* dst = nt < 8 ? &s.al[(8 * nt + 2 * tig) * LD64] : &s.vt[(8 * (nt - 8) + 2 * tig) * LD64];
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        const float(&d)[4] = half ? ds[i] : db[i];
        const int r = 16 * (half ? mt_small : mt_big) + gid;
        dst[r] = __uint_as_float(tf32(d[0]));
        dst[LD64 + r] = __uint_as_float(tf32(d[1]));
        dst[r + 8] = __uint_as_float(tf32(d[2]));
        dst[LD64 + r + 8] = __uint_as_float(tf32(d[3]));
      }
    }
    // from here on K is read only as K_d^T = (diag(e^(gam_C - gam)) K)^T, a TF32 operand
#pragma unroll
    for (int e = 0; e < 16; ++e) {
      const int idx = tid + e * kThreads, j = idx & 63;
      s.k[(idx >> 6) * LD64 + j] = __uint_as_float(tf32(s.kdec[j] * kr[e]));
    }
  }
  __syncthreads();

  // ---- step 4: the record: [M^T; R] (128 x 64), N (128 x 64), Y^T (128 x 64),
  // rows swizzled (sw64)
  float* rec = a.ws + (static_cast<int64_t>(c) * a.H + h) * kRec;
  {
    const float eC = s.eg[C - 1];
    // M^T = e^gam_C I - K_d^T W (warps 0-3) or R = diag(e^gam) Q - P W (warps 4-7): 16 rows each
    {
      const bool is_r = warp >= 4;
      const int mt = warp & 3;
      const int nks = is_r ? 2 * mt + 2 : 8;  // P is lower triangular
      uint32_t af[8][4];
#pragma unroll
      for (int ks = 0; ks < 8; ++ks)
        if (ks < nks) lda(af[ks], is_r ? s.p : s.k, LD64, 16 * mt, 8 * ks, lane);
      float* dst = rec + (is_r ? 64 : 0) * 64;
#pragma unroll
      for (int nt = 0; nt < 8; ++nt) {
        float d[4] = {0.0f, 0.0f, 0.0f, 0.0f};
#pragma unroll
        for (int kp = 0; kp < 4; ++kp) {
          if (2 * kp >= nks) continue;
          uint32_t b[4];
          ldb2(b, s.al, LD64, 8 * nt, 16 * kp, lane);
          mma(d, af[2 * kp], b[0], b[1]);
          mma(d, af[2 * kp + 1], b[2], b[3]);
        }
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
          const int r = 16 * mt + gid + 8 * hh, col = 8 * nt + 2 * tig;
          float v0, v1;
          if (is_r) {
            v0 = s.eg[r] * s.q[r * LD64 + col] - d[2 * hh];
            v1 = s.eg[r] * s.q[r * LD64 + col + 1] - d[2 * hh + 1];
          } else {
            v0 = (r == col ? eC : 0.0f) - d[2 * hh];
            v1 = (r == col + 1 ? eC : 0.0f) - d[2 * hh + 1];
          }
          // rounded here once: the state pass reads these rows only as TF32 MMA operands
          *reinterpret_cast<float2*>(dst + sw64(r, col)) =
              make_float2(__uint_as_float(tf32(v0)), __uint_as_float(tf32(v1)));
        }
      }
    }
    // N = U~^T K_d and Y^T = U~^T P^T: rows 16*warp .. +16 of both
    {
      const int mt = warp;
      uint32_t af[8][4];
#pragma unroll
      for (int ks = 0; ks < 8; ++ks) lda(af[ks], s.vt, LD64, 16 * mt, 8 * ks, lane);
#pragma unroll
      for (int nt = 0; nt < 16; ++nt) {
        const bool is_y = nt >= 8;
        const int n0 = 8 * (nt & 7);
        float d[4] = {0.0f, 0.0f, 0.0f, 0.0f};
#pragma unroll
        for (int kp = 0; kp < 4; ++kp) {
          if (is_y && 2 * kp > (nt & 7)) continue;  // P[t][j] = 0 for j > t
          uint32_t b[4];
          ldb2(b, is_y ? s.p : s.k, LD64, n0, 16 * kp, lane);
          mma(d, af[2 * kp], b[0], b[1]);
          if (!is_y || 2 * kp + 1 <= (nt & 7)) mma(d, af[2 * kp + 1], b[2], b[3]);
        }
        float* dst = rec + (is_y ? 2 : 1) * 128 * 64;
        const int r = 16 * mt + gid, col = n0 + 2 * tig;
        *reinterpret_cast<float2*>(dst + sw64(r, col)) = make_float2(d[0], d[1]);
        *reinterpret_cast<float2*>(dst + sw64(r + 8, col)) = make_float2(d[2], d[3]);
      }
    }
  }
}

constexpr int kBufs = 3;  // record buffers of the state pass
constexpr int kAhead = kBufs - 1;  // chunks whose records are requested ahead
// floats of one record buffer of the state pass: [M^T; R] (128 rows), then
// this CTA's 32 rows of N and of Y^T
constexpr int kRecCta = (128 + 2 * kRows) * 64;

struct StateSmem {
  float rec[kBufs][kRecCta];  // swizzled rows, as stored by the per-chunk pass
  float st[2][kRows * 64];    // the state rows, current and next (TF32 values but the last), swizzled
  float os[2][C * 36];        // output staging [t][i], two chunks
  uint64_t full[kBufs];
  int abort_flag;
};

// O rows of chunk c from the staging buffer: 64 tokens x 32 values, 8 per thread.
__device__ __forceinline__ void store_out(const GdnArgs& a, const float* os, int c, int h, int i0, int tid) {
  const int t = tid >> 2, part = tid & 3;
  const int64_t tok = static_cast<int64_t>(c) * C + t;
  if (tok >= a.T) return;
  const float* src = &os[t * 36 + 8 * part];
  uint8_t* dst = a.o + tok * a.ld_o;
  const int64_t col = static_cast<int64_t>(h) * DV + i0 + 8 * part;
  if (a.out_f32) {
    float4* p = reinterpret_cast<float4*>(dst + col * 4);
    p[0] = make_float4(src[0], src[1], src[2], src[3]);
    p[1] = make_float4(src[4], src[5], src[6], src[7]);
  } else {
    uint32_t w[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const __nv_bfloat162 b = __floats2bfloat162_rn(src[2 * i], src[2 * i + 1]);
      w[i] = *reinterpret_cast<const uint32_t*>(&b);
    }
    *reinterpret_cast<uint4*>(dst + col * 2) = make_uint4(w[0], w[1], w[2], w[3]);
  }
}

// One CTA per (value head, 32 state rows): the chunks in order, one block
// barrier per chunk.  Chunk c's record (the shared [M^T; R] and this CTA's rows
// of N and Y^T, three bulk copies) lands in buffer c % kBufs, requested kAhead
// chunks ahead; its output goes out from the staging buffer during chunk c + 1.
// Fragments come from shared memory with ldmatrix: the records and the state
// rows are swizzled (sw64), so the loads are free of bank conflicts.
__global__ void __launch_bounds__(kThreads, 1) gdn_state_kernel(const __grid_constant__ GdnArgs a) {
  extern __shared__ __align__(16) uint8_t smem_raw[];
  StateSmem& s = *reinterpret_cast<StateSmem*>(smem_raw);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int gid = lane >> 2, tig = lane & 3;
  const int h = blockIdx.x, i0 = blockIdx.y * kRows;
  volatile int* abort_flag = &s.abort_flag;

  if (tid == 0) {
    for (int b = 0; b < kBufs; ++b) mbar_init(&s.full[b], 1);
    s.abort_flag = 0;
    fence_mbarrier_init();
  }
  __syncthreads();
  grid_dependency_wait();
  if (tid == 0) grid_launch_dependents();

  auto issue = [&](int c) {  // thread 0 only
    const int b = c % kBufs;
    const float* rec = a.ws + (static_cast<int64_t>(c) * a.H + h) * kRec;
    mbar_arrive_expect_tx(&s.full[b], kRecCta * 4);
    bulk_load(s.rec[b], rec, 128 * 64 * 4, &s.full[b]);
    bulk_load(s.rec[b] + 128 * 64, rec + 128 * 64 + i0 * 64, kRows * 64 * 4, &s.full[b]);
    bulk_load(s.rec[b] + (128 + kRows) * 64, rec + 256 * 64 + i0 * 64, kRows * 64 * 4, &s.full[b]);
  };
  if (tid == 0) {
    for (int cc = 0; cc < kAhead && cc < a.nchunks; ++cc) issue(cc);
  }
  // entering state, as the TF32 operand it is used as
  for (int idx = tid; idx < kRows * DK; idx += kThreads) {
    const int r = idx / DK, col = idx % DK;
    const float v = a.h0 ? a.h0[(static_cast<int64_t>(h) * DV + i0 + r) * DK + col] : 0.0f;
    s.st[0][sw64(r, col)] = __uint_as_float(tf32(v));
  }
  // this lane's rows and pieces for ldmatrix: A (state) rows rr + 8 (j & 1),
  // piece 2 ks + (j >> 1); B ([M^T; R]) rows rr + 8 (j >> 1), piece 2 ks + (j & 1)
  const int rr = lane & 7, jm = lane >> 3;
  const int a_row = rr + 8 * (jm & 1), a_pc = jm >> 1;
  const int nbase = 16 * warp;  // warps 0-3: state columns, 4-7: tokens
  const int b_row = nbase + rr + 8 * (jm >> 1), b_pc = jm & 1;
  int cur = 0, c = 0;
  for (; c < a.nchunks; ++c) {
    const int buf = c % kBufs;
    const bool ok = mbar_wait_bounded(&s.full[buf], static_cast<uint32_t>(c / kBufs) & 1u, abort_flag);
    if (__syncthreads_or(!ok)) break;  // a copy did not arrive in time: every thread stops
    // buffer (c + kAhead) % kBufs was last read during chunk c - 1
    if (tid == 0 && c + kAhead < a.nchunks) issue(c + kAhead);
    if (c > 0) store_out(a, s.os[(c - 1) & 1], c - 1, h, i0, tid);
    const float* bc = s.rec[buf];
    const float* nn = bc + 128 * 64;
    const float* yt = bc + (128 + kRows) * 64;
    // D[i][n] = sum_k S[i][k] Bc[n][k]: n < 64 -> (S M)[i][n], n >= 64 -> (S R^T)[i][t = n - 64]
    {
      const uint32_t st_u = smem_u32(s.st[cur]), bc_u = smem_u32(bc);
      uint32_t af[2][8][4];
#pragma unroll
      for (int mt = 0; mt < 2; ++mt)
#pragma unroll
        for (int ks = 0; ks < 8; ++ks)
          ldsm_x4(af[mt][ks], st_u + (16 * mt + a_row) * 256 + (((2 * ks + a_pc) ^ rr) << 4));
      // two accumulators per tile (even and odd k-steps) halve the dependent MMA chain
      float d[2][2][4], d2[2][2][4];
#pragma unroll
      for (int mt = 0; mt < 2; ++mt)
#pragma unroll
        for (int nt = 0; nt < 2; ++nt)
#pragma unroll
          for (int e = 0; e < 4; ++e) d[mt][nt][e] = d2[mt][nt][e] = 0.0f;
#pragma unroll
      for (int ks = 0; ks < 8; ++ks) {
        uint32_t bq[4];  // b0, b1 of columns nbase .. +7, then of nbase + 8 .. +15
        ldsm_x4(bq, bc_u + b_row * 256 + (((2 * ks + b_pc) ^ rr) << 4));
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) {
          mma((ks & 1) ? d2[0][nt] : d[0][nt], af[0][ks], bq[2 * nt], bq[2 * nt + 1]);
          mma((ks & 1) ? d2[1][nt] : d[1][nt], af[1][ks], bq[2 * nt], bq[2 * nt + 1]);
        }
      }
#pragma unroll
      for (int mt = 0; mt < 2; ++mt)
#pragma unroll
        for (int nt = 0; nt < 2; ++nt)
#pragma unroll
          for (int e = 0; e < 4; ++e) d[mt][nt][e] += d2[mt][nt][e];
      if (warp < 4) {
        // the next state: FP32 after the last chunk (it is the result), else the TF32 operand
        const bool last = c + 1 == a.nchunks;
#pragma unroll
        for (int mt = 0; mt < 2; ++mt)
#pragma unroll
          for (int nt = 0; nt < 2; ++nt)
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
              const int r = 16 * mt + gid + 8 * hh, col = nbase + 8 * nt + 2 * tig;
              const float2 n2 = *reinterpret_cast<const float2*>(&nn[sw64(r, col)]);
              float v0 = d[mt][nt][2 * hh] + n2.x, v1 = d[mt][nt][2 * hh + 1] + n2.y;
              if (!last) {
                v0 = __uint_as_float(tf32(v0));
                v1 = __uint_as_float(tf32(v1));
              }
              *reinterpret_cast<float2*>(&s.st[cur ^ 1][sw64(r, col)]) = make_float2(v0, v1);
            }
      } else {
        float* os = s.os[c & 1];
#pragma unroll
        for (int mt = 0; mt < 2; ++mt)
#pragma unroll
          for (int nt = 0; nt < 2; ++nt)
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
              const int r = 16 * mt + gid + 8 * hh;
              const int t = nbase - 64 + 8 * nt + 2 * tig;
              const float2 y2 = *reinterpret_cast<const float2*>(&yt[sw64(r, t)]);
              os[t * 36 + r] = d[mt][nt][2 * hh] + y2.x;
              os[(t + 1) * 36 + r] = d[mt][nt][2 * hh + 1] + y2.y;
            }
      }
    }
    cur ^= 1;
  }
  if (c < a.nchunks) {
    // a record copy did not arrive in time (the error word is set): wait, with
    // a limit, for the copies still in flight into this CTA's buffers, then stop
    if (tid == 0)
      for (int cc = c; cc < a.nchunks && cc < c + kAhead; ++cc)
        mbar_wait_bounded(&s.full[cc % kBufs], static_cast<uint32_t>(cc / kBufs) & 1u, nullptr);
    return;
  }
  __syncthreads();
  if (a.nchunks > 0) store_out(a, s.os[(a.nchunks - 1) & 1], a.nchunks - 1, h, i0, tid);
  if (a.h_out) {
    for (int idx = tid; idx < kRows * DK; idx += kThreads) {
      const int r = idx / DK, col = idx % DK;
      a.h_out[(static_cast<int64_t>(h) * DV + i0 + r) * DK + col] = s.st[cur][sw64(r, col)];
    }
  }
}

template <class Kern>
cudaError_t launch(Kern kern, dim3 grid, int smem, const GdnArgs& a, cudaStream_t stream) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, a);
}

}  // namespace gdn

size_t gdn_workspace_bytes(int64_t T, int64_t H) {
  return static_cast<size_t>(ceil_div(T, gdn::C)) * static_cast<size_t>(H) * gdn::kRec * sizeof(float);
}

cudaError_t launch_gdn(const GdnProblem& p, cudaStream_t stream) {
  using namespace gdn;
  static std::atomic<uint64_t> attr_done{0};
  cudaError_t ea = once_per_device(attr_done, [] {
    cudaError_t e = cudaFuncSetAttribute(gdn_prep_kernel<NVFP4_DTYPE_BF16>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, sizeof(PrepSmem));
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(gdn_prep_kernel<NVFP4_DTYPE_F32>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               sizeof(PrepSmem));
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(gdn_state_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, sizeof(StateSmem));
    return e;
  });
  if (ea != cudaSuccess) return ea;
  const int esz = p.in_dtype == NVFP4_DTYPE_BF16 ? 2 : 4;
  GdnArgs a{};
  a.q = static_cast<const uint8_t*>(p.q);
  a.k = static_cast<const uint8_t*>(p.k);
  a.v = static_cast<const uint8_t*>(p.v);
  a.ld_q = p.ld_q * esz;
  a.ld_k = p.ld_k * esz;
  a.ld_v = p.ld_v * esz;
  a.beta = p.beta;
  a.g = p.g;
  a.ld_beta = p.ld_beta;
  a.ld_g = p.ld_g;
  a.T = p.T;
  a.H = static_cast<int>(p.H);
  a.rep = static_cast<int>(p.H / p.H_k);
  a.nchunks = static_cast<int>(ceil_div(p.T, C));
  a.scale = p.scale;
  a.eps = 1e-6f;
  a.h0 = p.h0;
  a.h_out = p.h_out;
  a.o = static_cast<uint8_t*>(p.o);
  a.out_f32 = p.out_dtype == NVFP4_DTYPE_F32 ? 1 : 0;
  a.ld_o = p.ld_o * (a.out_f32 ? 4 : 2);
  a.ws = static_cast<float*>(p.workspace);
  const dim3 gp(static_cast<unsigned>(a.nchunks), static_cast<unsigned>(a.H));
  cudaError_t e = p.in_dtype == NVFP4_DTYPE_BF16
                      ? launch(gdn_prep_kernel<NVFP4_DTYPE_BF16>, gp, sizeof(PrepSmem), a, stream)
                      : launch(gdn_prep_kernel<NVFP4_DTYPE_F32>, gp, sizeof(PrepSmem), a, stream);
  if (e != cudaSuccess) return e;
  return launch(gdn_state_kernel, dim3(static_cast<unsigned>(a.H), DV / kRows), sizeof(StateSmem), a, stream);
}

}  // namespace nvfp4
