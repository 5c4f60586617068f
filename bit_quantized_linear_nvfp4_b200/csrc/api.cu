// extern "C" entry points of libnvfp4 (declared in include/nvfp4.h): host-side
// argument checks, then the launches.  No entry point allocates device memory,
// synchronises (except nvfp4_check) or aborts.
#include <cstdint>
#include <cstring>

#include <cuda_runtime.h>

#include "internal.h"
#include "ptx.cuh"

namespace {

thread_local int t_last_cuda_error = 0;

int cuda_fail(cudaError_t e) {
  t_last_cuda_error = static_cast<int>(e);
  return NVFP4_ERR_CUDA;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int check_device() {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e);
  int major = 0, minor = 0;
  cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
  cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev);
  if (major != 10 || minor != 0) return NVFP4_ERR_DEVICE;
  return NVFP4_OK;
}

int check_quant_args(const void* x, int dtype, int64_t M, int64_t K, int64_t ld, float* g_out,
                     uint8_t* codes, uint8_t* sf) {
  if (dtype != NVFP4_DTYPE_BF16 && dtype != NVFP4_DTYPE_F32) return NVFP4_ERR_INVALID_ARG;
  if (M < 0 || K <= 0 || g_out == nullptr) return NVFP4_ERR_INVALID_ARG;
  if (K % 16 != 0) return NVFP4_ERR_UNSUPPORTED_SHAPE;
  if (M > (int64_t(1) << 31) || K > (int64_t(1) << 30)) return NVFP4_ERR_UNSUPPORTED_SHAPE;
  // the kernels index (row, 512-element chunk) work items with 32-bit integers
  if (nvfp4::ceil_div(M, 128) * 128 * nvfp4::ceil_div(K, 512) >= (int64_t(1) << 30))
    return NVFP4_ERR_UNSUPPORTED_SHAPE;
  if (M == 0) return NVFP4_OK;
  if (x == nullptr || codes == nullptr || sf == nullptr) return NVFP4_ERR_INVALID_ARG;
  if (ld < K) return NVFP4_ERR_INVALID_ARG;
  const int esz = dtype == NVFP4_DTYPE_BF16 ? 2 : 4;
  if (!aligned16(x) || (ld * esz) % 16 != 0) return NVFP4_ERR_MISALIGNED;
  if (!aligned16(codes) || !aligned16(sf) || (K / 2) % 4 != 0) return NVFP4_ERR_MISALIGNED;
  if ((reinterpret_cast<uintptr_t>(g_out) & 3u) != 0) return NVFP4_ERR_MISALIGNED;
  return NVFP4_OK;
}

int quantize_impl(const void* x, int dtype, int64_t M, int64_t K, int64_t ld,
                  const nvfp4::RowSegments& segs, const float* g_in, float* g_out, uint8_t* codes,
                  uint8_t* sf, void* ws, size_t ws_bytes, void* stream) {
  int st = check_quant_args(x, dtype, M, K, ld, g_out, codes, sf);
  if (st != NVFP4_OK) return st;
  if (g_in == nullptr && (ws == nullptr || ws_bytes < nvfp4_quantize_workspace_bytes(segs.n) ||
                          !aligned16(ws)))
    return NVFP4_ERR_WORKSPACE;
  st = check_device();
  if (st != NVFP4_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaError_t e = nvfp4::launch_quantize(x, dtype, M, K, ld, segs, g_in, ws, g_out, codes, sf, s);
  if (e != cudaSuccess) return cuda_fail(e);
  return NVFP4_OK;
}

int check_operand(const nvfp4_operand* o) {
  if (o == nullptr || o->codes == nullptr || o->sf == nullptr) return NVFP4_ERR_INVALID_ARG;
  if (o->rows <= 0 || o->K <= 0) return NVFP4_ERR_INVALID_ARG;
  if (o->K % 32 != 0) return NVFP4_ERR_UNSUPPORTED_SHAPE;
  if (o->rows > (int64_t(1) << 31) || o->K > (int64_t(1) << 30)) return NVFP4_ERR_UNSUPPORTED_SHAPE;
  if (!aligned16(o->codes) || !aligned16(o->sf)) return NVFP4_ERR_MISALIGNED;
  return NVFP4_OK;
}

bool epi_is_bf16(int kind) { return kind == NVFP4_EPI_IDENTITY_BF16 || kind == NVFP4_EPI_SWIGLU_GATE; }

}  // namespace

extern "C" {

const char* nvfp4_status_string(int status) {
  switch (status) {
    case NVFP4_OK: return "ok";
    case NVFP4_ERR_INVALID_ARG: return "invalid argument";
    case NVFP4_ERR_UNSUPPORTED_SHAPE: return "unsupported shape";
    case NVFP4_ERR_MISALIGNED: return "misaligned pointer or leading dimension";
    case NVFP4_ERR_CUDA: return "CUDA error";
    case NVFP4_ERR_DEVICE_TIMEOUT: return "device-side wait timed out";
    case NVFP4_ERR_WORKSPACE: return "workspace missing or too small";
    case NVFP4_ERR_DEVICE: return "device is not compute capability 10.0";
    default: return "unknown status";
  }
}

int nvfp4_last_cuda_error(void) { return t_last_cuda_error; }

size_t nvfp4_sf_bytes(int64_t rows, int64_t K) {
  if (rows <= 0 || K <= 0) return 0;
  return nvfp4::sf_bytes(rows, K);
}

size_t nvfp4_quantize_workspace_bytes(int nseg) {
  if (nseg < 1) nseg = 1;
  return 16 * ((nvfp4::quantize_scratch_bytes(nseg) + 15) / 16);
}

int nvfp4_quantize(const void* x, int x_dtype, int64_t M, int64_t K, int64_t ld_x,
                   const float* g_in, float* g_out, uint8_t* codes, uint8_t* sf, void* workspace,
                   size_t workspace_bytes, void* stream) {
  nvfp4::RowSegments segs{};
  segs.n = 1;
  segs.begin[0] = 0;
  segs.begin[1] = M;
  return quantize_impl(x, x_dtype, M, K, ld_x, segs, g_in, g_out, codes, sf, workspace,
                       workspace_bytes, stream);
}

int nvfp4_quantize_segments(const void* w, int w_dtype, int64_t N, int64_t K, int64_t ld_w,
                            const int64_t* row_bounds, int nseg, const float* g_in, float* g_out,
                            uint8_t* codes, uint8_t* sf, void* workspace, size_t workspace_bytes,
                            void* stream) {
  if (row_bounds == nullptr || nseg < 1 || nseg > NVFP4_MAX_SEGMENTS) return NVFP4_ERR_INVALID_ARG;
  if (row_bounds[0] != 0 || row_bounds[nseg] != N) return NVFP4_ERR_INVALID_ARG;
  nvfp4::RowSegments segs{};
  segs.n = nseg;
  for (int i = 0; i <= nseg; ++i) {
    if (i > 0 && row_bounds[i] <= row_bounds[i - 1]) return NVFP4_ERR_INVALID_ARG;
    segs.begin[i] = row_bounds[i];
  }
  return quantize_impl(w, w_dtype, N, K, ld_w, segs, g_in, g_out, codes, sf, workspace,
                       workspace_bytes, stream);
}

size_t nvfp4_gemm_workspace_bytes(int64_t M, int64_t N, int64_t K) {
  return nvfp4::gemm_workspace_bytes(M, N, K);
}

}  // extern "C"

namespace {

// Checks the arguments of one fused projection and describes it in *p.
int build_problem(const nvfp4_operand* A, const float* g_a, const nvfp4_operand* W,
                  const float* seg_global_scale, const nvfp4_segment* segs, int nseg,
                  void* workspace, size_t workspace_bytes, nvfp4::GemmProblem* out) {
  int st = check_operand(A);
  if (st != NVFP4_OK) return st;
  st = check_operand(W);
  if (st != NVFP4_OK) return st;
  if (A->K != W->K) return NVFP4_ERR_INVALID_ARG;
  if (g_a == nullptr || seg_global_scale == nullptr || segs == nullptr) return NVFP4_ERR_INVALID_ARG;
  if (nseg < 1 || nseg > NVFP4_MAX_SEGMENTS) return NVFP4_ERR_INVALID_ARG;

  nvfp4::GemmProblem& p = *out;
  p = nvfp4::GemmProblem{};
  p.a_codes = A->codes;
  p.a_sf = A->sf;
  p.w_codes = W->codes;
  p.w_sf = W->sf;
  p.M = A->rows;
  p.N = W->rows;
  p.K = A->K;
  p.g_a = g_a;
  p.seg_scale = seg_global_scale;
  p.nseg = nseg;
  int n_swiglu = 0;
  for (int i = 0; i < nseg; ++i) {
    const nvfp4_segment& s = segs[i];
    const int64_t expect_begin = i == 0 ? 0 : segs[i - 1].n_end;
    if (s.n_begin != expect_begin || s.n_end <= s.n_begin) return NVFP4_ERR_INVALID_ARG;
    if (s.epilogue < NVFP4_EPI_IDENTITY_BF16 || s.epilogue > NVFP4_EPI_SWIGLU_UP || s.reserved != 0)
      return NVFP4_ERR_INVALID_ARG;
    const int64_t width = s.n_end - s.n_begin;
    if (s.epilogue == NVFP4_EPI_SWIGLU_GATE || s.epilogue == NVFP4_EPI_SWIGLU_UP) ++n_swiglu;
    if (s.epilogue != NVFP4_EPI_SWIGLU_UP) {
      if (s.out == nullptr) return NVFP4_ERR_INVALID_ARG;
      if (!aligned16(s.out)) return NVFP4_ERR_MISALIGNED;
      const int64_t vec = epi_is_bf16(s.epilogue) ? 8 : 4;
      if (s.ld_out < width || s.ld_out % vec != 0) return NVFP4_ERR_MISALIGNED;
    }
    if (s.epilogue == NVFP4_EPI_GDN_DECAY_F32) {
      if (s.A_log == nullptr || s.dt_bias == nullptr) return NVFP4_ERR_INVALID_ARG;
    }
    nvfp4::EpiSegment& e = p.seg[i];
    e.n_begin = s.n_begin;
    e.n_end = s.n_end;
    e.kind = s.epilogue;
    e.scale_index = i;
    e.out = s.out;
    e.ld_out = s.ld_out;
    e.a_log = s.A_log;
    e.dt_bias = s.dt_bias;
  }
  if (segs[nseg - 1].n_end != W->rows) return NVFP4_ERR_INVALID_ARG;
  if (n_swiglu != 0) {
    if (nseg != 2 || segs[0].epilogue != NVFP4_EPI_SWIGLU_GATE ||
        segs[1].epilogue != NVFP4_EPI_SWIGLU_UP)
      return NVFP4_ERR_INVALID_ARG;
    if (segs[0].n_end * 2 != W->rows) return NVFP4_ERR_INVALID_ARG;
    if (segs[0].n_end % 128 != 0) return NVFP4_ERR_UNSUPPORTED_SHAPE;
    p.swiglu = true;
  }
  if (workspace_bytes < nvfp4::gemm_workspace_bytes(p.M, p.N, p.K) ||
      (nvfp4::gemm_workspace_bytes(p.M, p.N, p.K) > 0 && workspace == nullptr))
    return NVFP4_ERR_WORKSPACE;
  return check_device();
}

// [p, p + n) and [q, q + m) share a byte.
bool overlap(const void* p, size_t n, const void* q, size_t m) {
  const uintptr_t a = reinterpret_cast<uintptr_t>(p), b = reinterpret_cast<uintptr_t>(q);
  return n != 0 && m != 0 && a < b + m && b < a + n;
}

}  // namespace

extern "C" {

int nvfp4_fused_proj(const nvfp4_operand* A, const float* g_a, const nvfp4_operand* W,
                     const float* seg_global_scale, const nvfp4_segment* segs, int nseg,
                     void* workspace, size_t workspace_bytes, void* stream) {
  nvfp4::GemmProblem p;
  int st = build_problem(A, g_a, W, seg_global_scale, segs, nseg, workspace, workspace_bytes, &p);
  if (st != NVFP4_OK) return st;
  cudaError_t e = nvfp4::launch_gemm(p, workspace, workspace_bytes, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e);
  return NVFP4_OK;
}

int nvfp4_linear(const void* x, int x_dtype, int64_t M, int64_t K, int64_t ld_x, const float* g_in,
                 uint8_t* a_codes, uint8_t* a_sf, float* g_a, const nvfp4_operand* W,
                 const float* seg_global_scale, const nvfp4_segment* segs, int nseg, void* workspace,
                 size_t workspace_bytes, void* stream) {
  int st = check_quant_args(x, x_dtype, M, K, ld_x, g_a, a_codes, a_sf);
  if (st != NVFP4_OK) return st;
  st = check_operand(W);
  if (st != NVFP4_OK) return st;
  if (W->K != K) return NVFP4_ERR_INVALID_ARG;
  if (M == 0) return NVFP4_OK;
  if (g_in == nullptr && (workspace == nullptr || workspace_bytes < nvfp4_quantize_workspace_bytes(1) ||
                          !aligned16(workspace)))
    return NVFP4_ERR_WORKSPACE;
  // The GEMM may read W while the quantiser still runs: nothing the quantiser
  // writes may share memory with W or the segment scales.
  const size_t wc = static_cast<size_t>(W->rows) * static_cast<size_t>(K / 2);
  const size_t ws = nvfp4::sf_bytes(W->rows, K);
  const size_t nsc = seg_global_scale ? sizeof(float) * static_cast<size_t>(nseg > 0 ? nseg : 0) : 0;
  const size_t ac = static_cast<size_t>(M) * static_cast<size_t>(K / 2), as = nvfp4::sf_bytes(M, K);
  const size_t wsb = g_in == nullptr ? nvfp4_quantize_workspace_bytes(1) : 0;
  const void* written[4] = {a_codes, a_sf, g_a, workspace};
  const size_t wbytes[4] = {ac, as, sizeof(float), wsb};
  for (int i = 0; i < 4; ++i)
    if (overlap(written[i], wbytes[i], W->codes, wc) || overlap(written[i], wbytes[i], W->sf, ws) ||
        overlap(written[i], wbytes[i], seg_global_scale, nsc))
      return NVFP4_ERR_INVALID_ARG;
  nvfp4_operand A{a_codes, a_sf, M, K};
  nvfp4::GemmProblem p;
  st = build_problem(&A, g_a, W, seg_global_scale, segs, nseg, nullptr, 0, &p);
  if (st != NVFP4_OK) return st;
  nvfp4::RowSegments one{};
  one.n = 1;
  one.begin[0] = 0;
  one.begin[1] = M;
  st = quantize_impl(x, x_dtype, M, K, ld_x, one, g_in, g_a, a_codes, a_sf, workspace, workspace_bytes, stream);
  if (st != NVFP4_OK) return st;
  p.w_prefetch = true;  // the kernel before the GEMM is the quantiser, which leaves W alone
  cudaError_t e = nvfp4::launch_gemm(p, nullptr, 0, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e);
  return NVFP4_OK;
}

int nvfp4_requantize_segments(const nvfp4_operand* W, const int64_t* row_bounds, int nseg,
                              const float* g_old, const float* g_new, uint8_t* codes_out, uint8_t* sf_out,
                              float* g_out, void* stream) {
  int st = check_operand(W);
  if (st != NVFP4_OK) return st;
  if (row_bounds == nullptr || nseg < 1 || nseg > NVFP4_MAX_SEGMENTS) return NVFP4_ERR_INVALID_ARG;
  if (row_bounds[0] != 0 || row_bounds[nseg] != W->rows) return NVFP4_ERR_INVALID_ARG;
  nvfp4::RowSegments segs{};
  segs.n = nseg;
  for (int i = 0; i <= nseg; ++i) {
    if (i > 0 && row_bounds[i] <= row_bounds[i - 1]) return NVFP4_ERR_INVALID_ARG;
    segs.begin[i] = row_bounds[i];
  }
  if (g_old == nullptr || codes_out == nullptr || sf_out == nullptr || g_out == nullptr) return NVFP4_ERR_INVALID_ARG;
  if (!aligned16(codes_out) || !aligned16(sf_out) || (reinterpret_cast<uintptr_t>(g_out) & 3u) != 0)
    return NVFP4_ERR_MISALIGNED;
  // in place, or into separate buffers: no partial overlap
  const size_t nc = static_cast<size_t>(W->rows) * static_cast<size_t>(W->K / 2), ns = nvfp4::sf_bytes(W->rows, W->K);
  if ((codes_out != W->codes && overlap(codes_out, nc, W->codes, nc)) || (sf_out != W->sf && overlap(sf_out, ns, W->sf, ns)) ||
      overlap(codes_out, nc, sf_out, ns) || overlap(codes_out, nc, W->sf, ns) || overlap(sf_out, ns, W->codes, nc))
    return NVFP4_ERR_INVALID_ARG;
  st = check_device();
  if (st != NVFP4_OK) return st;
  cudaError_t e = nvfp4::launch_requantize(W->codes, W->sf, W->rows, W->K, segs, g_old, g_new, codes_out, sf_out, g_out,
                                           static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e);
  return NVFP4_OK;
}

int nvfp4_kv_fp8_quantize(const void* x, int x_dtype, int64_t rows, int64_t cols, int64_t ld_x,
                          const float* scale, uint8_t* out, int64_t ld_out, void* stream) {
  if (x_dtype != NVFP4_DTYPE_BF16 && x_dtype != NVFP4_DTYPE_F32) return NVFP4_ERR_INVALID_ARG;
  if (rows < 0 || cols < 0 || scale == nullptr) return NVFP4_ERR_INVALID_ARG;
  if (cols % 8 != 0) return NVFP4_ERR_UNSUPPORTED_SHAPE;
  if (rows == 0 || cols == 0) return NVFP4_OK;
  if (x == nullptr || out == nullptr || ld_x < cols || ld_out < cols) return NVFP4_ERR_INVALID_ARG;
  const int esz = x_dtype == NVFP4_DTYPE_BF16 ? 2 : 4;
  if (!aligned16(x) || (ld_x * esz) % 16 != 0) return NVFP4_ERR_MISALIGNED;
  if ((reinterpret_cast<uintptr_t>(out) & 7u) != 0 || ld_out % 8 != 0 || (reinterpret_cast<uintptr_t>(scale) & 3u) != 0)
    return NVFP4_ERR_MISALIGNED;
  int st = check_device();
  if (st != NVFP4_OK) return st;
  cudaError_t e = nvfp4::launch_kv_fp8(true, x_dtype, x, ld_x, out, ld_out, rows, cols, scale,
                                       static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e);
  return NVFP4_OK;
}

int nvfp4_kv_fp8_dequantize(const uint8_t* codes, int64_t rows, int64_t cols, int64_t ld_codes,
                            const float* scale, void* out, int out_dtype, int64_t ld_out, void* stream) {
  if (out_dtype != NVFP4_DTYPE_BF16 && out_dtype != NVFP4_DTYPE_F32) return NVFP4_ERR_INVALID_ARG;
  if (rows < 0 || cols < 0 || scale == nullptr) return NVFP4_ERR_INVALID_ARG;
  if (cols % 8 != 0) return NVFP4_ERR_UNSUPPORTED_SHAPE;
  if (rows == 0 || cols == 0) return NVFP4_OK;
  if (codes == nullptr || out == nullptr || ld_codes < cols || ld_out < cols) return NVFP4_ERR_INVALID_ARG;
  const int esz = out_dtype == NVFP4_DTYPE_BF16 ? 2 : 4;
  if ((reinterpret_cast<uintptr_t>(codes) & 7u) != 0 || ld_codes % 8 != 0) return NVFP4_ERR_MISALIGNED;
  if (!aligned16(out) || (ld_out * esz) % 16 != 0 || (reinterpret_cast<uintptr_t>(scale) & 3u) != 0)
    return NVFP4_ERR_MISALIGNED;
  int st = check_device();
  if (st != NVFP4_OK) return st;
  cudaError_t e = nvfp4::launch_kv_fp8(false, out_dtype, codes, ld_codes, out, ld_out, rows, cols, scale,
                                       static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e);
  return NVFP4_OK;
}

int nvfp4_activation_stats(const void* x, int x_dtype, int64_t M, int64_t K, int64_t ld_x, const float* g,
                           double* moments, float* row_err2, float* row_norm2, float* col_sq, float* col_max,
                           void* stream) {
  if (x_dtype != NVFP4_DTYPE_BF16 && x_dtype != NVFP4_DTYPE_F32) return NVFP4_ERR_INVALID_ARG;
  if (M < 0 || K <= 0 || moments == nullptr) return NVFP4_ERR_INVALID_ARG;
  if (K % 16 != 0) return NVFP4_ERR_UNSUPPORTED_SHAPE;
  if (M > (int64_t(1) << 31) - 1 || K > (int64_t(1) << 30)) return NVFP4_ERR_UNSUPPORTED_SHAPE;
  if (row_err2 != nullptr && g == nullptr) return NVFP4_ERR_INVALID_ARG;
  if (M == 0) return NVFP4_OK;
  if (x == nullptr || ld_x < K) return NVFP4_ERR_INVALID_ARG;
  const int esz = x_dtype == NVFP4_DTYPE_BF16 ? 2 : 4;
  if (!aligned16(x) || (ld_x * esz) % 16 != 0) return NVFP4_ERR_MISALIGNED;
  if ((reinterpret_cast<uintptr_t>(moments) & 7u) != 0) return NVFP4_ERR_MISALIGNED;
  const void* f32s[5] = {g, row_err2, row_norm2, col_sq, col_max};
  for (const void* q : f32s)
    if ((reinterpret_cast<uintptr_t>(q) & 3u) != 0) return NVFP4_ERR_MISALIGNED;
  int st = check_device();
  if (st != NVFP4_OK) return st;
  cudaError_t e = nvfp4::launch_act_stats(x, x_dtype, M, K, ld_x, g, moments, row_err2, row_norm2, col_sq, col_max,
                                          static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e);
  return NVFP4_OK;
}

int nvfp4_activation_summary(const double* moments, const float* row_err2, const float* row_norm2, int64_t M,
                             const float* col_sq, int64_t K, double* summary, void* stream) {
  if (moments == nullptr || row_norm2 == nullptr || col_sq == nullptr || summary == nullptr)
    return NVFP4_ERR_INVALID_ARG;
  if (M <= 0 || K <= 0) return NVFP4_ERR_INVALID_ARG;
  if (M > (int64_t(1) << 31) - 1 || K > (int64_t(1) << 30)) return NVFP4_ERR_UNSUPPORTED_SHAPE;
  if ((reinterpret_cast<uintptr_t>(moments) & 7u) != 0 || (reinterpret_cast<uintptr_t>(summary) & 7u) != 0)
    return NVFP4_ERR_MISALIGNED;
  const void* f32s[3] = {row_err2, row_norm2, col_sq};
  for (const void* q : f32s)
    if ((reinterpret_cast<uintptr_t>(q) & 3u) != 0) return NVFP4_ERR_MISALIGNED;
  int st = check_device();
  if (st != NVFP4_OK) return st;
  cudaError_t e = nvfp4::launch_act_summary(moments, row_err2, row_norm2, M, col_sq, K, summary,
                                            static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e);
  return NVFP4_OK;
}

int nvfp4_gemm(const nvfp4_operand* A, const float* g_a, const nvfp4_operand* W, const float* g_w,
               void* out, int out_dtype, int64_t ld_out, void* workspace, size_t workspace_bytes,
               void* stream) {
  if (W == nullptr) return NVFP4_ERR_INVALID_ARG;
  if (out_dtype != NVFP4_DTYPE_BF16 && out_dtype != NVFP4_DTYPE_F32) return NVFP4_ERR_INVALID_ARG;
  nvfp4_segment seg{};
  seg.n_begin = 0;
  seg.n_end = W->rows;
  seg.epilogue = out_dtype == NVFP4_DTYPE_BF16 ? NVFP4_EPI_IDENTITY_BF16 : NVFP4_EPI_IDENTITY_F32;
  seg.out = out;
  seg.ld_out = ld_out;
  return nvfp4_fused_proj(A, g_a, W, g_w, &seg, 1, workspace, workspace_bytes, stream);
}

size_t nvfp4_gdn_workspace_bytes(int64_t T, int64_t H) {
  if (T <= 0 || H <= 0) return 0;
  return nvfp4::gdn_workspace_bytes(T, H);
}

int nvfp4_gdn_recurrence(const void* q, const void* k, const void* v, int in_dtype, int64_t T, int64_t H,
                         int64_t H_k, int64_t d_k, int64_t d_v, int64_t ld_q, int64_t ld_k, int64_t ld_v,
                         const float* beta, int64_t ld_beta, const float* g, int64_t ld_g, float scale,
                         const float* h0, float* h_out, void* o, int out_dtype, int64_t ld_o,
                         void* workspace, size_t workspace_bytes, void* stream) {
  if (in_dtype != NVFP4_DTYPE_BF16 && in_dtype != NVFP4_DTYPE_F32) return NVFP4_ERR_INVALID_ARG;
  if (out_dtype != NVFP4_DTYPE_BF16 && out_dtype != NVFP4_DTYPE_F32) return NVFP4_ERR_INVALID_ARG;
  if (T < 0 || H <= 0 || H_k <= 0 || H % H_k != 0) return NVFP4_ERR_INVALID_ARG;
  if (!(scale >= 0.0f) || scale > 3.4028234663852886e38f) return NVFP4_ERR_INVALID_ARG;
  if (d_k != 64 || d_v != 128) return NVFP4_ERR_UNSUPPORTED_SHAPE;
  if (H > 65535 || nvfp4::ceil_div(T, 64) > (int64_t(1) << 31) - 1) return NVFP4_ERR_UNSUPPORTED_SHAPE;
  const size_t state_bytes = static_cast<size_t>(H) * 128 * 64 * sizeof(float);
  if ((reinterpret_cast<uintptr_t>(h0) & 3u) != 0 || (reinterpret_cast<uintptr_t>(h_out) & 3u) != 0)
    return NVFP4_ERR_MISALIGNED;
  if (h_out != nullptr && h0 != nullptr && h_out != h0 && overlap(h_out, state_bytes, h0, state_bytes))
    return NVFP4_ERR_INVALID_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (T == 0) {
    if (h_out == nullptr || h_out == h0) return NVFP4_OK;
    int st = check_device();
    if (st != NVFP4_OK) return st;
    cudaError_t e = h0 ? cudaMemcpyAsync(h_out, h0, state_bytes, cudaMemcpyDeviceToDevice, s)
                       : cudaMemsetAsync(h_out, 0, state_bytes, s);
    if (e != cudaSuccess) return cuda_fail(e);
    return NVFP4_OK;
  }
  if (q == nullptr || k == nullptr || v == nullptr || beta == nullptr || g == nullptr || o == nullptr)
    return NVFP4_ERR_INVALID_ARG;
  if (ld_q < H_k * 64 || ld_k < H_k * 64 || ld_v < H * 128 || ld_o < H * 128 || ld_beta < H || ld_g < H)
    return NVFP4_ERR_INVALID_ARG;
  const int esz = in_dtype == NVFP4_DTYPE_BF16 ? 2 : 4, osz = out_dtype == NVFP4_DTYPE_BF16 ? 2 : 4;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || (ld_q * esz) % 16 != 0 ||
      (ld_k * esz) % 16 != 0 || (ld_v * esz) % 16 != 0 || (ld_o * osz) % 16 != 0)
    return NVFP4_ERR_MISALIGNED;
  if ((reinterpret_cast<uintptr_t>(beta) & 3u) != 0 || (reinterpret_cast<uintptr_t>(g) & 3u) != 0)
    return NVFP4_ERR_MISALIGNED;
  const size_t ws_need = nvfp4::gdn_workspace_bytes(T, H);
  if (workspace == nullptr || workspace_bytes < ws_need || !aligned16(workspace)) return NVFP4_ERR_WORKSPACE;
  // o and the workspace are written: neither may overlap anything read
  const size_t nq = static_cast<size_t>((T - 1) * ld_q + H_k * 64) * esz;
  const size_t nk = static_cast<size_t>((T - 1) * ld_k + H_k * 64) * esz;
  const size_t nv = static_cast<size_t>((T - 1) * ld_v + H * 128) * esz;
  const size_t nb = static_cast<size_t>((T - 1) * ld_beta + H) * sizeof(float);
  const size_t ng = static_cast<size_t>((T - 1) * ld_g + H) * sizeof(float);
  const size_t no = static_cast<size_t>((T - 1) * ld_o + H * 128) * osz;
  const void* written[3] = {o, workspace, h_out};
  const size_t wbytes[3] = {no, ws_need, h_out ? state_bytes : 0};
  for (int i = 0; i < 3; ++i) {
    if (overlap(written[i], wbytes[i], q, nq) || overlap(written[i], wbytes[i], k, nk) ||
        overlap(written[i], wbytes[i], v, nv) || overlap(written[i], wbytes[i], beta, nb) ||
        overlap(written[i], wbytes[i], g, ng))
      return NVFP4_ERR_INVALID_ARG;
    for (int j = i + 1; j < 3; ++j)
      if (overlap(written[i], wbytes[i], written[j], wbytes[j])) return NVFP4_ERR_INVALID_ARG;
    if (i < 2 && overlap(written[i], wbytes[i], h0, h0 ? state_bytes : 0)) return NVFP4_ERR_INVALID_ARG;
  }
  int st = check_device();
  if (st != NVFP4_OK) return st;
  nvfp4::GdnProblem p{};
  p.q = q;
  p.k = k;
  p.v = v;
  p.in_dtype = in_dtype;
  p.T = T;
  p.H = H;
  p.H_k = H_k;
  p.ld_q = ld_q;
  p.ld_k = ld_k;
  p.ld_v = ld_v;
  p.beta = beta;
  p.g = g;
  p.ld_beta = ld_beta;
  p.ld_g = ld_g;
  p.scale = scale == 0.0f ? 0.125f : scale;  // d_k^-1/2 for d_k = 64
  p.h0 = h0;
  p.h_out = h_out;
  p.o = o;
  p.out_dtype = out_dtype;
  p.ld_o = ld_o;
  p.workspace = workspace;
  cudaError_t e = nvfp4::launch_gdn(p, s);
  if (e != cudaSuccess) return cuda_fail(e);
  return NVFP4_OK;
}

int nvfp4_selftest_bounded_wait(uint64_t limit_ns, void* stream) {
  if (limit_ns < 1000000ull || limit_ns > 2000000000ull) return NVFP4_ERR_INVALID_ARG;
  int st = check_device();
  if (st != NVFP4_OK) return st;
  cudaError_t e = nvfp4::launch_wait_selftest(limit_ns, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e);
  return NVFP4_OK;
}

int nvfp4_check(void* stream) {
  cudaError_t e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e);
  unsigned int flag = 0, zero = 0;
  e = cudaMemcpyFromSymbol(&flag, nvfp4::g_device_error, sizeof(flag));
  if (e != cudaSuccess) return cuda_fail(e);
  if (flag != 0) {
    e = cudaMemcpyToSymbol(nvfp4::g_device_error, &zero, sizeof(zero));
    if (e != cudaSuccess) return cuda_fail(e);
    return NVFP4_ERR_DEVICE_TIMEOUT;
  }
  return NVFP4_OK;
}

}  // extern "C"
