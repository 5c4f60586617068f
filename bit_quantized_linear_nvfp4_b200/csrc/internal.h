// Internal host-side interfaces between the C ABI layer and the kernels.
#pragma once

#include <atomic>
#include <cstddef>
#include <cstdint>
#include <cuda_runtime.h>

#include "../../include/nvfp4.h"

namespace nvfp4 {

constexpr int kMaxSeg = NVFP4_MAX_SEGMENTS;

// Row ranges that share one global scale (modules stacked along rows).
struct RowSegments {
  int n;
  int64_t begin[kMaxSeg + 1];  // begin[n] == total rows
};

inline int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }

// Runs set() -- raising a kernel's dynamic shared-memory limit, which is a
// per-device setting -- once for each device a process launches on.  `done`
// holds one bit per device (devices 64 and up set it on every launch).
template <class F>
cudaError_t once_per_device(std::atomic<uint64_t>& done, F set) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const uint64_t bit = dev < 64 ? (uint64_t{1} << dev) : 0;
  if (bit != 0 && (done.load(std::memory_order_acquire) & bit) != 0) return cudaSuccess;
  e = set();
  if (e == cudaSuccess && bit != 0) done.fetch_or(bit, std::memory_order_acq_rel);
  return e;
}
inline size_t sf_bytes(int64_t rows, int64_t K) {
  return static_cast<size_t>(ceil_div(rows, 128) * 128) * static_cast<size_t>(ceil_div(K, 64) * 4);
}

// Most blocks the amax kernel launches (one per SM, at most this many).
constexpr int kMaxAmaxBlocks = 256;

// Scratch bytes a device-computed scale needs: one maximum per amax block and
// segment.  Every call overwrites what it reads, so the scratch needs no
// clearing.
size_t quantize_scratch_bytes(int nseg);

// Quantise rows [0, M) (scale layout padded to 128 rows).  Global scale of
// segment s: g_in[s] if g_in, else amax over the segment's rows / 2688,
// computed by a first launch into `ws` (quantize_scratch_bytes(segs.n)
// bytes).  Writes g_out[s].
cudaError_t launch_quantize(const void* x, int dtype, int64_t M, int64_t K, int64_t ld,
                            const RowSegments& segs, const float* g_in, void* ws,
                            float* g_out, uint8_t* codes, uint8_t* sf, cudaStream_t stream);

// Re-encode codes/sf of [N, K] (row ranges `segs` quantised with g_old[s])
// under one common scale (*g_new, or the largest g_old when g_new is null);
// writes codes_out / sf_out (may equal the inputs) and g_out[s] = common scale.
cudaError_t launch_requantize(const uint8_t* codes, const uint8_t* sf, int64_t N, int64_t K,
                              const RowSegments& segs, const float* g_old, const float* g_new,
                              uint8_t* codes_out, uint8_t* sf_out, float* g_out, cudaStream_t stream);

// FP8 (E4M3) KV codec with a static scale: encode x [rows, cols] (BF16/F32,
// row stride ld_src elements) into codes (row stride ld_dst bytes), or decode
// codes (row stride ld_src bytes) into BF16/F32 (row stride ld_dst elements).
cudaError_t launch_kv_fp8(bool encode, int dtype, const void* src, int64_t ld_src, void* dst, int64_t ld_dst,
                          int64_t rows, int64_t cols, const float* scale, cudaStream_t stream);

// Activation statistics of x [M, K] (accumulating; see nvfp4_activation_stats).
cudaError_t launch_act_stats(const void* x, int dtype, int64_t M, int64_t K, int64_t ld, const float* g,
                             double* moments, float* row_err2, float* row_norm2, float* col_sq, float* col_max,
                             cudaStream_t stream);

// Derived figures of the statistics' accumulators (see nvfp4_activation_summary).
cudaError_t launch_act_summary(const double* moments, const float* row_err2, const float* row_norm2, int64_t M,
                               const float* col_sq, int64_t K, double* out, cudaStream_t stream);

// Gated delta-rule recurrence (see nvfp4_gdn_recurrence); leading dimensions
// in elements, d_k = 64 and d_v = 128.
struct GdnProblem {
  const void* q;
  const void* k;
  const void* v;
  int in_dtype;
  int64_t T, H, H_k;
  int64_t ld_q, ld_k, ld_v;
  const float* beta;
  const float* g;
  int64_t ld_beta, ld_g;
  float scale;
  const float* h0;
  float* h_out;
  void* o;
  int out_dtype;
  int64_t ld_o;
  void* workspace;
};

size_t gdn_workspace_bytes(int64_t T, int64_t H);

// One kernel whose bounded wait is left to run out (see nvfp4_selftest_bounded_wait).
cudaError_t launch_wait_selftest(uint64_t limit_ns, cudaStream_t stream);
cudaError_t launch_gdn(const GdnProblem& p, cudaStream_t stream);

// GEMM epilogue description handed to the kernels.
struct EpiSegment {
  int64_t n_begin, n_end;
  int32_t kind;
  int32_t scale_index;
  void* out;
  int64_t ld_out;
  const float* a_log;
  const float* dt_bias;
};

struct GemmProblem {
  const uint8_t* a_codes;
  const uint8_t* a_sf;
  const uint8_t* w_codes;
  const uint8_t* w_sf;
  int64_t M, N, K;
  const float* g_a;
  const float* seg_scale;  // device [nseg]
  int nseg;
  EpiSegment seg[kMaxSeg];
  bool swiglu;             // two segments: gate [0, N/2), up [N/2, N)
  // W and its scales are not written by the kernel launched just before the
  // GEMM on the stream, so the weight-streaming kernel may start reading them
  // before that kernel completes.
  bool w_prefetch;
};

size_t gemm_workspace_bytes(int64_t M, int64_t N, int64_t K);
cudaError_t launch_gemm(const GemmProblem& p, void* workspace, size_t workspace_bytes,
                        cudaStream_t stream);

}  // namespace nvfp4
