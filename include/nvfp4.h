/*
 * nvfp4.h — C ABI of libnvfp4: the NVFP4 W4A4 linear layer on B200 (sm_100a).
 *
 * What it computes.  "Why Gated DeltaNet Survives 4-Bit Quantization: NVFP4
 * W4A4 for the Recurrent Half of a Hybrid 27B LLM" (ai.info summary),
 * "Methodology in Plain English": weights and activations are stored as 4-bit
 * E2M1 values with one E4M3 scale per block of 16 consecutive elements along
 * K; "Main Findings", fused-GEMM scaling bullet: each linear module keeps one
 * FP32 global scale, and a GEMM that fuses several modules must apply each
 * module's own global scale (the repair of the global-scale mismatch);
 * "Main Findings", gate-parameterisation bullets: the GDN write strength is
 * sigmoid(b) and the decay is log-space, -exp(A_log) * softplus(a + dt_bias).
 *
 * Conventions for every entry point
 *   - All pointers named "device" are device memory owned by the caller; the
 *     library allocates no device memory and keeps no pointer after a call.
 *   - Work is enqueued on `stream` (a cudaStream_t; NULL = legacy default
 *     stream) and is asynchronous: no entry point synchronises, except
 *     nvfp4_check.  Arguments are validated on the host before any launch; a
 *     non-zero status means nothing was enqueued (NVFP4_ERR_CUDA: a launch or
 *     driver call failed, see nvfp4_last_cuda_error).  Nothing aborts.
 *   - Global scales are dequantisation multipliers: x ~= e2m1 * S * g with
 *     g = amax / (6 * 448) when the library computes it.
 *   - Codes: row-major [rows, K/2] bytes, element 2j of a row in the low
 *     nibble, 2j+1 in the high nibble.
 *   - Scale bytes (E4M3) use the tcgen05 block-scale layout: rows padded to
 *     a multiple of 128, K/16 padded to a multiple of 4; 512-byte atoms hold
 *     128 rows x 4 scales, scale (r, j) at byte
 *       ((r/128) * KA + j/4) * 512 + (r%32)*16 + ((r/32)%4)*4 + j%4,
 *     KA = ceil(K/64).  Padding bytes are zero (nvfp4_quantize writes them).
 *   - Every kernel that reads or writes an argument buffer is launched with
 *     programmatic stream serialization: it may start while the kernel
 *     before it on the stream is finishing, and waits for that kernel to
 *     complete before it touches any argument buffer.  Only nvfp4_linear
 *     reads a buffer (the weights) before that point, and only while its own
 *     quantiser runs.  (nvfp4_selftest_bounded_wait's kernel touches no
 *     argument buffer and is launched plainly.)
 *   - Devices: compute capability 10.0 (B200) only.
 */
#ifndef NVFP4_H
#define NVFP4_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum nvfp4_status {
  NVFP4_OK = 0,
  NVFP4_ERR_INVALID_ARG = 1,       /* null pointer, bad count or enum value */
  NVFP4_ERR_UNSUPPORTED_SHAPE = 2, /* a size outside what the kernels take */
  NVFP4_ERR_MISALIGNED = 3,        /* pointer or leading dimension alignment */
  NVFP4_ERR_CUDA = 4,              /* a CUDA runtime/driver call failed */
  NVFP4_ERR_DEVICE_TIMEOUT = 5,    /* a bounded device-side wait gave up */
  NVFP4_ERR_WORKSPACE = 6,         /* workspace missing or too small */
  NVFP4_ERR_DEVICE = 7             /* current device is not sm_100 */
} nvfp4_status;

/* Input element types for the quantiser. */
enum { NVFP4_DTYPE_BF16 = 0, NVFP4_DTYPE_F32 = 1 };

/* Largest number of segments (modules) in one fused projection or one
 * segmented weight quantisation. */
#define NVFP4_MAX_SEGMENTS 8

/* A quantised operand in device memory (the struct itself is host memory). */
typedef struct nvfp4_operand {
  const uint8_t* codes; /* device, [rows, K/2], 16-byte aligned */
  const uint8_t* sf;    /* device, nvfp4_sf_bytes(rows, K) bytes, 16-byte aligned */
  int64_t rows;         /* M for activations, N for weights */
  int64_t K;            /* reduction length, a multiple of 32 for the GEMMs */
} nvfp4_operand;

/* Per-segment epilogues of nvfp4_fused_proj.  y = acc * g_a * g_w[segment]. */
typedef enum nvfp4_epilogue {
  NVFP4_EPI_IDENTITY_BF16 = 0, /* out = bf16(y)                                   */
  NVFP4_EPI_IDENTITY_F32 = 1,  /* out = y                                         */
  NVFP4_EPI_SIGMOID_F32 = 2,   /* out = 1 / (1 + exp(-y))   (GDN write strength)  */
  NVFP4_EPI_GDN_DECAY_F32 = 3, /* out = -exp(A_log[h]) * softplus(y + dt_bias[h]),
                                  h = column - n_begin     (GDN log-space decay)  */
  NVFP4_EPI_SWIGLU_GATE = 4,   /* out = bf16(silu(y) * y_up), paired with the
                                  NVFP4_EPI_SWIGLU_UP segment of equal width      */
  NVFP4_EPI_SWIGLU_UP = 5      /* consumed by the gate segment; writes nothing   */
} nvfp4_epilogue;

/* One segment (module) of a fused projection: W rows [n_begin, n_end). */
typedef struct nvfp4_segment {
  int64_t n_begin, n_end;
  int32_t epilogue;      /* nvfp4_epilogue */
  int32_t reserved;      /* must be 0 */
  void* out;             /* device; element (m, j) at out[m * ld_out + j], j = n - n_begin;
                            16-byte aligned; NULL only for NVFP4_EPI_SWIGLU_UP */
  int64_t ld_out;        /* elements; multiple of 8 (BF16) or 4 (F32) */
  const float* A_log;    /* device [n_end - n_begin], GDN decay only, else NULL */
  const float* dt_bias;  /* device [n_end - n_begin], GDN decay only, else NULL */
} nvfp4_segment;

/* Human-readable name of a status code (static storage). */
const char* nvfp4_status_string(int status);

/* The CUDA error (cudaError_t value) behind the last NVFP4_ERR_CUDA on this thread. */
int nvfp4_last_cuda_error(void);

/* Bytes of the scale-factor buffer for a [rows, K] operand (padded layout above). */
size_t nvfp4_sf_bytes(int64_t rows, int64_t K);

/* Workspace bytes nvfp4_quantize / nvfp4_quantize_segments need (dynamic
 * scales only; 0 when every global scale is given). */
size_t nvfp4_quantize_workspace_bytes(int nseg);

/*
 * nvfp4_quantize — on-the-fly NVFP4 quantisation of an activation tensor
 * (the "A4" half of W4A4, "Main Findings", activation-statistics bullet:
 * per-token activation quantisation; format per "Methodology in Plain
 * English").
 *   x       device, [M, K] row-major with row stride ld_x elements; BF16 or F32
 *           (x_dtype); 16-byte aligned base, ld_x * elem_size % 16 == 0.
 *           Values must be finite.
 *   K       multiple of 16.  M >= 0 (M == 0 writes only g_out).
 *   g_in    device float, a calibrated (static) global scale, or NULL to use
 *           g = amax|x| / 2688 computed on the device (two launches, two passes
 *           over x; the second re-reads x from L2 when it fits there).
 *   g_out   device float, receives the global scale used (may equal g_in).
 *   codes   device, [M, K/2] bytes, 16-byte aligned.
 *   sf      device, nvfp4_sf_bytes(M, K) bytes, 16-byte aligned; padding zeroed.
 *   workspace / workspace_bytes: device scratch of at least
 *           nvfp4_quantize_workspace_bytes(1) bytes when g_in == NULL.
 * Per block of 16 (FP32): s = (amax_b / 6) / g; sf = E4M3_rn_satfinite(s);
 * S = decode(sf); inv = 1 / (S * g) (0 if S * g == 0, at most FLT_MAX);
 * code = E2M1_rn_satfinite(x * inv).  g <= 0 gives all-zero codes and scales.
 */
int nvfp4_quantize(const void* x, int x_dtype, int64_t M, int64_t K, int64_t ld_x,
                   const float* g_in, float* g_out, uint8_t* codes, uint8_t* sf,
                   void* workspace, size_t workspace_bytes, void* stream);

/*
 * nvfp4_quantize_segments — the same quantiser over a weight matrix made of
 * nseg modules stacked along rows, each with its own FP32 global scale ("one
 * FP32 global scale per linear module", "Main Findings", fused-GEMM bullet).
 *   row_bounds  host, nseg + 1 increasing row indices, row_bounds[0] == 0,
 *               row_bounds[nseg] == N.
 *   g_in        device float [nseg] or NULL (per-module amax / 2688).
 *   g_out       device float [nseg].
 *   Other arguments as nvfp4_quantize with M -> N; workspace of
 *   nvfp4_quantize_workspace_bytes(nseg) bytes when g_in == NULL.
 */
int nvfp4_quantize_segments(const void* w, int w_dtype, int64_t N, int64_t K, int64_t ld_w,
                            const int64_t* row_bounds, int nseg, const float* g_in, float* g_out,
                            uint8_t* codes, uint8_t* sf, void* workspace, size_t workspace_bytes,
                            void* stream);

/*
 * nvfp4_quantize_noalloc — nvfp4_quantize with the device-computed global
 * scale (g = amax|x| / 2688), for callers that cannot allocate device memory.
 * The paper has no counterpart: it is an interface for this library's users.
 * Some callers have no device allocator at hand at the point where they
 * quantise activations: a plugin enqueued by an inference runtime that owns
 * all memory, code running under a fixed memory plan, or a C caller that only
 * holds the tensors it was given.  The dynamic scale needs a few bytes of
 * device scratch between its two launches; this entry point keeps that scratch
 * in a static array inside the library (NVFP4_NOALLOC_SCRATCH_BYTES bytes,
 * held on every GPU that loads the library until the process exits), so the
 * caller passes only inputs and outputs and nothing is allocated.
 *   Arguments as nvfp4_quantize with g_in = NULL and no workspace.
 *   One call uses nvfp4_quantize_workspace_bytes(1) bytes of the scratch; a
 *   call needing more than NVFP4_NOALLOC_SCRATCH_BYTES is rejected with
 *   NVFP4_ERR_UNSUPPORTED_SHAPE.
 *   The first call on a device looks up the scratch address on that device
 *   (and so does the first call in a new context of the device, after a
 *   cudaDeviceReset or after the primary context was released and created
 *   again); make that first call before any stream capture on the device.
 *   Every call shares the one scratch array (each call writes the scratch it
 *   later reads, so it needs no clearing):
 *   calls whose work overlaps on the GPU, on different streams, race and must
 *   be serialised by the caller.
 */
#define NVFP4_NOALLOC_SCRATCH_BYTES 1024
int nvfp4_quantize_noalloc(const void* x, int x_dtype, int64_t M, int64_t K, int64_t ld_x,
                           float* g_out, uint8_t* codes, uint8_t* sf, void* stream);

/* Workspace bytes nvfp4_gemm / nvfp4_fused_proj need for an [M, N, K]
 * problem (currently 0 for every shape; the argument is kept so that a
 * future path may use scratch). */
size_t nvfp4_gemm_workspace_bytes(int64_t M, int64_t N, int64_t K);

/*
 * nvfp4_gemm — block-scaled FP4 x FP4 GEMM, out = (A . W^T) * g_a * g_w with
 * FP32 accumulation: acc[m, n] = sum_k e2m1(a) Sa * e2m1(w) Sw
 * ("Methodology in Plain English": W4A4 with 16-element E4M3 block scales).
 *   A        host struct, device buffers: activations [M, K].
 *   W        host struct, device buffers: weights [N, K] (same K).
 *   g_a,g_w  device floats.
 *   out      device, [M, N] row-major, stride ld_out elements; out_dtype is
 *            NVFP4_DTYPE_BF16 or NVFP4_DTYPE_F32.
 * Equivalent to nvfp4_fused_proj with one identity segment.
 */
int nvfp4_gemm(const nvfp4_operand* A, const float* g_a, const nvfp4_operand* W,
               const float* g_w, void* out, int out_dtype, int64_t ld_out,
               void* workspace, size_t workspace_bytes, void* stream);

/*
 * nvfp4_fused_proj — one GEMM over nseg weight segments (modules) that keep
 * their own global scales, with a per-segment epilogue: the fused GDN input
 * projection (q, k, v, z identity to BF16; b -> sigmoid; a -> log-space decay)
 * and the fused MLP gate/up projection (SwiGLU).  Column n of segment s is
 * scaled by g_a * seg_global_scale[s] before its epilogue ("Main Findings",
 * fused-GEMM scaling bullet).  Passing the same value for every segment
 * reproduces the mismatch the pages describe.
 *   seg_global_scale  device float [nseg].
 *   segs              host array [nseg]; segments must tile [0, W->rows) in
 *                     increasing order; a SwiGLU call has exactly two segments,
 *                     gate then up, of equal width.
 */
int nvfp4_fused_proj(const nvfp4_operand* A, const float* g_a, const nvfp4_operand* W,
                     const float* seg_global_scale, const nvfp4_segment* segs, int nseg,
                     void* workspace, size_t workspace_bytes, void* stream);

/*
 * nvfp4_linear — the W4A4 linear layer in one call: quantise the activation x
 * (as nvfp4_quantize) into the caller's buffers, then run nvfp4_fused_proj on
 * the result ("Methodology in Plain English": activations are quantised on
 * the fly, weights offline; "Main Findings", fused-GEMM bullets for the
 * segments).  Because the library launches both kernels, the GEMM may start
 * streaming W while the quantiser is still running; for few tokens (the
 * weight-streaming, decode-shaped GEMM) that hides the quantiser.
 *   x, x_dtype, M, K, ld_x, g_in   as nvfp4_quantize (K a multiple of 32).
 *   a_codes, a_sf, g_a   device outputs of the quantiser (as codes, sf, g_out
 *                        of nvfp4_quantize); afterwards they hold the
 *                        quantised activation.  They and the workspace must
 *                        not overlap W's buffers or seg_global_scale.
 *   W, seg_global_scale, segs, nseg   as nvfp4_fused_proj (W->K == K).
 *   workspace / workspace_bytes   as nvfp4_quantize (the GEMM needs none).
 * M == 0 enqueues nothing.  All arguments are checked before either launch.
 */
int nvfp4_linear(const void* x, int x_dtype, int64_t M, int64_t K, int64_t ld_x,
                 const float* g_in, uint8_t* a_codes, uint8_t* a_sf, float* g_a,
                 const nvfp4_operand* W, const float* seg_global_scale,
                 const nvfp4_segment* segs, int nseg, void* workspace,
                 size_t workspace_bytes, void* stream);

/*
 * nvfp4_requantize_segments — checkpoint-side harmonisation of fused modules'
 * global scales ("Methodology in Plain English": the fused modules' scales
 * are made to agree on the checkpoint side, so that a kernel that applies one
 * global scale to the fused GEMM is correct).  Every element of the NVFP4
 * operand W is dequantised with its module's scale (x = e2m1 * S * g_old[s],
 * rounded once to FP32) and quantised again, exactly as nvfp4_quantize does,
 * with one common scale.
 *   W           host struct, device buffers: the operand [N, K] to re-encode.
 *   row_bounds  host, nseg + 1 increasing row indices (as nvfp4_quantize_segments).
 *   g_old       device float [nseg]: the modules' current global scales.
 *   g_new       device float, the common scale, or NULL for the largest of
 *               g_old, which is the scale of the fused (concatenated) weight
 *               and the only choice that clips no block (a smaller common
 *               scale makes the larger modules' top block scales saturate).
 *   codes_out, sf_out  device, [N, K/2] and nvfp4_sf_bytes(N, K) bytes, 16-byte
 *               aligned; either exactly W's buffers (in place) or disjoint
 *               from them.
 *   g_out       device float [nseg], receives the common scale for every
 *               module, so (codes_out, sf_out, g_out) is again an operand with
 *               its per-segment scale table.
 */
int nvfp4_requantize_segments(const nvfp4_operand* W, const int64_t* row_bounds, int nseg,
                              const float* g_old, const float* g_new, uint8_t* codes_out,
                              uint8_t* sf_out, float* g_out, void* stream);

/*
 * nvfp4_kv_fp8_quantize / nvfp4_kv_fp8_dequantize — FP8 (E4M3) KV-cache codec
 * with a calibrated static per-tensor scale ("Main Findings", KV-cache
 * bullet: FP8 KV with calibrated scales instead of 1.0).  The attention that
 * consumes the cache is not part of this library.
 *   Encode: code = E4M3_rn_satfinite(x * inv), inv = 1 / *scale in FP32 (once),
 *     the sign kept (also for zero); *scale not a positive finite number gives
 *     all-zero codes.  x: device [rows, cols] BF16 or F32 (x_dtype), row stride
 *     ld_x elements, 16-byte aligned rows; out: device [rows, cols] bytes, row
 *     stride ld_out, 8-byte aligned.
 *   Decode: out = e4m3(code) * *scale rounded to FP32 (then to BF16 for a BF16
 *     output).  codes: row stride ld_codes bytes, 8-byte aligned; out: device
 *     BF16 or F32 (out_dtype), row stride ld_out elements, 16-byte aligned rows.
 *   cols must be a multiple of 8; scale is a device float (the calibrated
 *   value, typically amax / 448 over calibration data).
 */
int nvfp4_kv_fp8_quantize(const void* x, int x_dtype, int64_t rows, int64_t cols, int64_t ld_x,
                          const float* scale, uint8_t* out, int64_t ld_out, void* stream);
int nvfp4_kv_fp8_dequantize(const uint8_t* codes, int64_t rows, int64_t cols, int64_t ld_codes,
                            const float* scale, void* out, int out_dtype, int64_t ld_out, void* stream);

/*
 * nvfp4_activation_stats — activation statistics at NVFP4 granularity, one
 * pass over x ("Main Findings", activation bullet: max/RMS, kurtosis, hot
 * channels against the median channel, the share of 16-element blocks
 * dominated by one value, per-token A4 error).  Every output ACCUMULATES: the
 * caller zeroes them once, and further calls add (statistics over several
 * calibration batches).
 *   x        device [M, K] BF16 or F32 (x_dtype), row stride ld_x elements,
 *            16-byte aligned rows; K a multiple of 16.
 *   g        device float, the global scale for the A4 error (nvfp4_quantize's
 *            g_out), or NULL (then row_err2 must be NULL).
 *   moments  device double[8]: sum x, sum x^2, sum x^3, sum x^4 (FP64
 *            accumulation), max |x|, elements, 16-blocks, dominated 16-blocks
 *            (largest magnitude > the sum of the other fifteen).
 *   row_err2, row_norm2  device float[M] or NULL: per row, sum (x - x_hat)^2
 *            with x_hat the NVFP4 dequantisation under g (the quantiser's
 *            arithmetic), and sum x^2.
 *   col_sq, col_max  device float[K] or NULL: per column, sum x^2 and max |x|.
 * The derived figures (max/RMS, kurtosis, dominated share, per-token A4
 * error, hot-channel ratio) come from nvfp4_activation_summary.
 */
int nvfp4_activation_stats(const void* x, int x_dtype, int64_t M, int64_t K, int64_t ld_x, const float* g,
                           double* moments, float* row_err2, float* row_norm2, float* col_sq, float* col_max,
                           void* stream);

/*
 * nvfp4_activation_summary — the figures the pages report for the residual
 * stream ("Main Findings", activation bullet: max/RMS, kurtosis, the share of
 * 16-element blocks dominated by one value, the per-token A4 error, hot
 * channels against the median channel), derived on the device from
 * nvfp4_activation_stats' accumulators in one small launch.  FP64 throughout,
 * each product and sum rounded on its own (no fused multiply-add):
 *   summary[0] max/RMS        moments[4] / sqrt(moments[1] / n), n = moments[5]
 *   summary[1] kurtosis       (E x^4 - 4 mu E x^3 + 6 mu^2 E x^2 - 3 mu^4) / var^2,
 *                             mu = E x, var = E x^2 - mu^2 (0 when var <= 0)
 *   summary[2] dominated share   moments[7] / moments[6]
 *   summary[3..5] per-token A4 error e_r = sqrt(row_err2[r]) / sqrt(row_norm2[r])
 *                             (divided by 1 when row_norm2[r] == 0): mean, min,
 *                             max over the M rows; NaN when row_err2 is NULL
 *   summary[6] hot-channel ratio  max_c rms_c / median_c rms_c,
 *                             rms_c = sqrt(col_sq[c] / M); the median of an even
 *                             count is the mean of the two middle values
 *   summary[7] median channel RMS (0 gives summary[6] = 0)
 *   moments    device double[8] as nvfp4_activation_stats writes them.
 *   row_err2, row_norm2  device float[M] (row_err2 may be NULL).
 *   col_sq     device float[K], non-negative.
 *   summary    device double[8], written.
 * M >= 1 and K >= 1.  Enqueued on `stream` after the statistics; the caller
 * reads the 64 bytes back when it needs them.
 */
int nvfp4_activation_summary(const double* moments, const float* row_err2, const float* row_norm2, int64_t M,
                             const float* col_sq, int64_t K, double* summary, void* stream);

/*
 * nvfp4_gdn_recurrence — the gated delta-rule recurrence that consumes the
 * fused GDN projection's q, k, v, beta and g ("Main Findings", recurrence
 * bullet: a fixed-size state in which every write overwrites along the
 * current key, with a decay and a write strength; gate-parameterisation
 * bullet: the decay gate is log-space, alpha = exp(g)).  Per value head h,
 * with the state S [d_v, d_k] in FP32:
 *     S_t = alpha_t S_{t-1} + beta_t (v_t - alpha_t S_{t-1} k_t) k_t^T,
 *     o_t = S_t q_t,   alpha_t = exp(g_t),
 * q and k L2-normalised per head (x / sqrt(sum x^2 + 1e-6)) and q scaled by
 * `scale`.  One sequence of T tokens; value head h reads query/key head
 * h / (H / H_k).  Evaluated in chunks of 64 tokens with TF32 tensor-core
 * products and FP32 state (results differ from an exact evaluation by the
 * rounding of the products' operands to TF32).
 *   q, k     device [T, H_k * d_k] (BF16 or F32, in_dtype), row strides ld_q,
 *            ld_k elements; head j in columns [j d_k, (j+1) d_k).
 *   v        device [T, H * d_v], same dtype, row stride ld_v.
 *   beta, g  device FP32 [T, H] (the projection's sigmoid and decay outputs),
 *            row strides ld_beta, ld_g elements.
 *   scale    query scale; 0 selects d_k^-1/2.  Must be finite and >= 0.
 *   h0       device FP32 [H, d_v, d_k] entering state, or NULL for zeros.
 *   h_out    device FP32 [H, d_v, d_k] receives the final state, or NULL;
 *            may equal h0 (the update is then in place) but no other overlap.
 *   o        device [T, H * d_v] (BF16 or F32, out_dtype), row stride ld_o.
 *   workspace, workspace_bytes   device, 16-byte aligned, at least
 *            nvfp4_gdn_workspace_bytes(T, H) bytes (per-chunk matrices).
 * Shapes: d_k == 64 and d_v == 128 (else NVFP4_ERR_UNSUPPORTED_SHAPE);
 * H_k divides H; q, k, v and o rows 16-byte aligned.  o must not overlap any
 * input or the workspace.  T == 0 only copies h0 (or zeros) to h_out.
 */
size_t nvfp4_gdn_workspace_bytes(int64_t T, int64_t H);
int nvfp4_gdn_recurrence(const void* q, const void* k, const void* v, int in_dtype, int64_t T, int64_t H,
                         int64_t H_k, int64_t d_k, int64_t d_v, int64_t ld_q, int64_t ld_k, int64_t ld_v,
                         const float* beta, int64_t ld_beta, const float* g, int64_t ld_g, float scale,
                         const float* h0, float* h_out, void* o, int out_dtype, int64_t ld_o,
                         void* workspace, size_t workspace_bytes, void* stream);

/*
 * nvfp4_selftest_bounded_wait — exercises the device-side failure path for
 * tests of failure detection.  It enqueues one small kernel whose single
 * thread waits, through the same bounded wait the library's kernels use, on a
 * barrier that nothing arrives on.  The wait gives up after limit_ns
 * nanoseconds (1 ms to 2 s, else NVFP4_ERR_INVALID_ARG), sets the device error
 * word and returns, so the next nvfp4_check on the stream reports
 * NVFP4_ERR_DEVICE_TIMEOUT and the context stays usable.  Nothing faults or
 * hangs.
 */
int nvfp4_selftest_bounded_wait(uint64_t limit_ns, void* stream);

/*
 * nvfp4_check — synchronise `stream`, then report (and clear) the library's
 * device error word: NVFP4_ERR_DEVICE_TIMEOUT if a bounded wait inside a
 * kernel gave up since the last check, NVFP4_ERR_CUDA on a CUDA error.
 */
int nvfp4_check(void* stream);

#ifdef __cplusplus
}
#endif

#endif /* NVFP4_H */
