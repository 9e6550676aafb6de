/*
 * sq.h -- C ABI of libsq, the B200 (sm_100a) SmoothQuant W8A8 linear layer.
 *
 * The method ("SmoothQuant: Accurate and Efficient Post-Training Quantization
 * for Large Language Models", Xiao et al., as explained on the abeam.tech
 * page):
 *   1. calibration   a_j = max_t |X[t,j]|, b_j = max_n |W[n,j]|
 *                    (glossary "Calibration"; section "how is the smoothing
 *                    factor chosen")
 *   2. smoothing     s_j = a_j^alpha / b_j^(1-alpha), folded offline into the
 *                    preceding LayerNorm (gamma/s, beta/s) and into diag(s) W
 *                    (section "what it does mathematically")
 *   3. runtime       per-token dynamic INT8 quantization of the activations
 *                    (section "inference", level O1), INT8 x INT8 -> INT32
 *                    GEMM (glossary "INT8 GEMM") against per-output-channel
 *                    INT8 weights, dequantized to fp16 by multiplying the
 *                    scales back (itmedia quantization tutorial, section 3).
 *
 * Conventions for every entry point:
 *   - All pointers except the sizes are DEVICE pointers on the current CUDA
 *     device, owned by the caller.  The library never allocates or frees.
 *   - fp16 tensors are passed as `const void*` (IEEE binary16).
 *   - Matrices are row-major.  Activations are [tokens, K]; the weight is the
 *     nn.Linear layout [N, K]; the output is [M, N].  K is contiguous.
 *   - Calls are asynchronous on `stream` (a cudaStream_t; NULL = legacy
 *     default stream).  Arguments are checked on the host first: a bad
 *     argument returns an error code and launches nothing.
 *   - Requirements: 1 <= K <= SQ_MAX_K, K % 16 == 0; rows/M/N >= 1;
 *     every pointer 16-byte aligned; leading dimensions (in elements) a
 *     multiple of 8 and >= K.  The device must be compute capability 10.0
 *     (B200); the library is built for sm_100a only and has no CPU path.
 *   - Numerics: every fp32 operation is IEEE round-to-nearest-even in the
 *     order written below, with no fused multiply-add; rint is ties-to-even.
 *     INT8 codes and int32 accumulators are therefore bit-identical to any
 *     implementation that follows the same order.
 *   - Non-finite inputs follow IEEE arithmetic: a NaN never sets a range
 *     (maxima ignore it) and is coded 0; an Inf sets an infinite range (scale
 *     Inf, reciprocal 0, so every code of that row or tensor is 0); a
 *     LayerNorm row holding an Inf or a NaN has NaN mean and rstd, so all of
 *     its values are NaN (scale 0, codes 0, no effect on calibration).  With
 *     a range fixed in advance (level O3, producer-side quantization) +-Inf
 *     saturate to +-127 and NaN is coded 0.
 *   - Device-side waits are bounded (default 2 s, see sq_set_wait_budget_ns).
 *     A wait that runs out records SQ_ERR_TIMEOUT in a per-device status word
 *     and the kernel returns early (its outputs are then undefined); read it
 *     with sq_poll_status.
 */
#ifndef SQ_H
#define SQ_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Largest K for which a sum of K products of two int8 codes in [-127, 127]
 * cannot leave the int32 range: 133144 * 127^2 = 2147479576 <= 2^31 - 1. */
#define SQ_MAX_K 133144

/* Largest token count served by the weight-streaming (swap-AB, stream-K)
 * GEMM kernel (SQ_PATH_SPLITK: tokens in the MMA's N slot, up to 128). */
#define SQ_SPLITK_MAX_M 128

/* Token counts up to which sq_w8a8_linear always streams the weight (the
 * decoding stage), and which the allocation-free entry point serves. */
#define SQ_DECODE_MAX_M 32

typedef enum sq_status {
  SQ_OK = 0,
  SQ_ERR_INVALID_ARG = 1,       /* null pointer, size <= 0, ld < K, bad path */
  SQ_ERR_MISALIGNED = 2,        /* pointer not 16-byte aligned or ld % 8 != 0 */
  SQ_ERR_UNSUPPORTED_SHAPE = 3, /* K % 16 != 0, or M too large for a forced path */
  SQ_ERR_K_OVERFLOW = 4,        /* K > SQ_MAX_K */
  SQ_ERR_WORKSPACE = 5,         /* workspace NULL or smaller than required */
  SQ_ERR_ARCH = 6,              /* current device is not compute capability 10.0 */
  SQ_ERR_CUDA = 7,              /* a CUDA runtime call or launch failed */
  SQ_ERR_TIMEOUT = 8            /* a device-side bounded wait ran out */
} sq_status;

/* A cudaStream_t, passed as an opaque pointer. */
typedef void* sq_stream_t;

/* Human-readable name of a status code (static storage, never NULL). */
const char* sq_status_string(int status);

/* ABI version of this header (major * 100 + minor). */
int sq_abi_version(void);

/*
 * Calibration (step 1): per-input-channel running absmax.
 *   amax_inout[j] = max(amax_inout[j], max_{r < rows} |x_hat[r, j]|)
 * where x_hat = x (ln_gamma == NULL) or the LayerNorm of each row of x:
 *   x_hat = ((x - mu) * rstd) * ln_gamma + ln_beta   (ln_beta may be NULL)
 * with mu, var the exact mean and biased variance of the row (integer sums of
 * the fp16 values scaled by 2^24, converted to fp64 by a fixed sequence of
 * correctly rounded operations) and rstd = 1 / sqrt(var + ln_eps), both
 * rounded to fp32.  Call it on the calibration activations to get a (the
 * LayerNorm output is what feeds the linear), and on W [N, K] (ln_gamma NULL)
 * to get b.
 *   x           fp16 [rows, ld], first K columns used
 *   amax_inout  fp32 [K]; zero-filled before the first batch (by the caller
 *               or sq_calibrate_reset); max is exact, so the result does not
 *               depend on call order
 */
sq_status sq_calibrate_absmax(const void* x_f16, int64_t rows, int64_t K, int64_t ld,
                              const float* ln_gamma, const float* ln_beta, float ln_eps,
                              float* amax_inout, sq_stream_t stream);

/*
 * The start of a calibration run: amax[0 .. n) = 0 (one or several running
 * maxima laid out back to back), on `stream`, ordered with the kernels
 * before and after it like every other call -- the zero-fill that
 * sq_calibrate_absmax expects before its first batch.
 *   amax fp32 [n], n >= 1
 */
sq_status sq_calibrate_reset(float* amax, int64_t n, sq_stream_t stream);

/*
 * Smoothing factor and offline fold (step 2).
 *   s_j     = fp32( pow(max(a_j, 1e-5f), alpha) / pow(max(b_j, 1e-5f), 1 - alpha) )
 *             evaluated in fp64 (1e-5f floors dead channels)
 *   inv_s_j = 1.0f / s_j
 *   gamma_out_j = gamma_j * inv_s_j, beta_out_j = beta_j * inv_s_j      (fp32)
 *   w_out[n, j] = fp16(fp32(w[n, j]) * s_j)                             (fp16)
 * gamma/beta (and their outputs) may be NULL; gamma_out may alias gamma.
 * w may be NULL (then w_out is ignored and N is unused); w_out may alias w.
 *   amax_x, amax_w, s_out, inv_s_out, gamma*, beta*   fp32 [K]
 *   w, w_out                                          fp16 [N, K]
 */
sq_status sq_smooth_fold(const float* amax_x, const float* amax_w, int64_t K, float alpha,
                         float* s_out, float* inv_s_out, const float* gamma, const float* beta,
                         float* gamma_out, float* beta_out, const void* w_f16, void* w_out_f16,
                         int64_t N, sq_stream_t stream);

/*
 * Per-output-channel symmetric INT8 weight quantization (step 2, weight side).
 * With s == NULL the row is w itself; with s given it is the folded weight
 * fp16(fp32(w[n, k]) * s_k), computed on the fly (the fold and the
 * quantization in one pass over w, without writing the folded fp16 weight).
 *   w_scale[n] = max_k |w'[n, k]| / 127
 *   wq[n, k]   = clamp(rint(fp32(w'[n, k]) * (1 / w_scale[n])), -127, 127)
 * An all-zero row gets scale 0 and codes 0.
 *   w   fp16 [N, K]; s fp32 [K] or NULL; wq int8 [N, K]; w_scale fp32 [N]
 */
sq_status sq_quantize_weight(const void* w_f16, int64_t N, int64_t K, const float* s,
                             int8_t* wq, float* w_scale, sq_stream_t stream);

/*
 * Runtime activation path (step 3a): optional LayerNorm, optional smoothing,
 * per-token dynamic INT8 quantization, one pass over h.
 *   x_hat      = gamma ? ((h - mu) * rstd) * gamma + beta : h      (as in calibration)
 *   x_hat      = inv_s ? x_hat * inv_s : x_hat
 *   x_scale[t] = max_k |x_hat[t, k]| / 127
 *   xq[t, k]   = clamp(rint(x_hat[t, k] * (1 / x_scale[t])), -127, 127)
 * With the smoothing folded into the LayerNorm pass gamma' / beta' and
 * inv_s = NULL; for an input with no preceding LayerNorm pass gamma = NULL
 * and inv_s.  beta may be NULL.
 *   h fp16 [M, ld]; gamma, beta, inv_s fp32 [K]; xq int8 [M, K]; x_scale fp32 [M]
 */
sq_status sq_ln_quant_act(const void* h_f16, int64_t M, int64_t K, int64_t ld,
                          const float* gamma, const float* beta, const float* inv_s, float eps,
                          int8_t* xq, float* x_scale, sq_stream_t stream);

/*
 * Per-tensor scales: the efficiency levels of the explainer (section
 * "inference").  O1 quantizes activations per token (sq_ln_quant_act) and the
 * weight per tensor; O2 quantizes both per tensor with dynamic scales; O3 per
 * tensor with static scales fixed offline from calibration.  The quantizer is
 * the same with one range for the whole tensor:
 *   scale = range / 127,  q = clamp(rint(x * (1 / scale)), -127, 127)
 * and the scale is written once per row (w_scale[n] or x_scale[t], all
 * equal), so sq_w8a8_linear serves every level unchanged.  `range_out` /
 * `range_in` point to one fp32 in device memory owned by the caller (16-byte
 * aligned, like every pointer here).
 */

/* Per-tensor weight quantization: range = max_{n,k} |w'[n, k]| over the
 * (optionally folded, as in sq_quantize_weight) weight, written to
 * range_out[0]; w_scale[n] = range / 127 for every n; two passes over w.
 *   w fp16 [N, K]; s fp32 [K] or NULL; wq int8 [N, K]; w_scale fp32 [N] */
sq_status sq_quantize_weight_tensor(const void* w_f16, int64_t N, int64_t K, const float* s,
                                    int8_t* wq, float* w_scale, float* range_out,
                                    sq_stream_t stream);

/* Level O2 activations: one dynamic scale for the whole batch.  range =
 * max_{t,k} |x_hat[t, k]| (x_hat as in sq_ln_quant_act) is written to
 * range_out[0]; x_scale[t] = range / 127 for every t.  Two passes over h
 * (the range must be known before the first code). */
sq_status sq_ln_quant_act_tensor(const void* h_f16, int64_t M, int64_t K, int64_t ld,
                                 const float* gamma, const float* beta, const float* inv_s,
                                 float eps, int8_t* xq, float* x_scale, float* range_out,
                                 sq_stream_t stream);

/* Level O3 activations: the range was fixed offline (range_in[0], e.g. from
 * sq_tensor_range); x_scale[t] = range / 127 for every t, and values beyond
 * the range saturate at -127 / 127.  One pass over h, no per-row max. */
sq_status sq_ln_quant_act_static(const void* h_f16, int64_t M, int64_t K, int64_t ld,
                                 const float* gamma, const float* beta, const float* inv_s,
                                 float eps, const float* range_in, int8_t* xq, float* x_scale,
                                 sq_stream_t stream);

/* The static activation range for level O3 from calibrated per-channel
 * ranges: range_out[0] = max_j amax[j], or max_j fp32(amax[j] * inv_s[j])
 * when inv_s is given.  With the smoothing folded into a LayerNorm, calibrate
 * on the folded gamma' / beta' and pass inv_s = NULL; for an input the runtime
 * multiplies by inv_s, calibrate the raw input and pass inv_s (rounding is
 * monotonic, so both give the largest |x_hat| over the calibration set).
 *   amax, inv_s fp32 [K] (inv_s may be NULL); range_out fp32 [1] */
sq_status sq_tensor_range(const float* amax, const float* inv_s, int64_t K, float* range_out,
                          sq_stream_t stream);

/*
 * Tensor-parallel building blocks (the explainer runs the quantized models
 * sharded over several GPUs: sections "how far speed and memory improved",
 * OPT-175B on 4 GPUs instead of 8, and "does it hold for a 530B model", 8
 * INT8 GPUs instead of 16 FP16).  A rank that
 * holds a slice of K (row-parallel: a slice of every token's channels and of
 * every weight row) must quantize with the ranges of the WHOLE row, so each
 * rank reports its slice's per-row ranges, the ranks max-reduce them, and
 * every rank quantizes its slice with the global ranges; the int32 partial
 * accumulators (sq_w8a8_gemm_s32) are then sum-reduced, exactly, and
 * dequantized once (sq_dequant).  The result equals the unsharded layer bit
 * for bit.
 *
 * Rows are the activation transform of sq_ln_quant_act (gamma, beta, inv_s,
 * eps) or, with s_fold given (and gamma, beta, inv_s NULL), the folded weight
 * fp16(fp32(x) * s_fold[k]) of sq_quantize_weight.
 */

/* range_out[r] = max_k |x_hat[r, k]| over this slice's K columns.
 *   x fp16 [rows, ld]; range_out fp32 [rows] */
sq_status sq_row_ranges(const void* x_f16, int64_t rows, int64_t K, int64_t ld, const float* gamma,
                        const float* beta, const float* inv_s, const float* s_fold, float eps,
                        float* range_out, sq_stream_t stream);

/* INT8 codes with given per-row ranges: scale[r] = range_in[r] / 127,
 * q[r, k] = clamp(rint(x_hat[r, k] * (1 / scale[r])), -127, 127).
 *   x fp16 [rows, ld]; range_in fp32 [rows]; q int8 [rows, K]; scale fp32 [rows] */
sq_status sq_quantize_rows_ranged(const void* x_f16, int64_t rows, int64_t K, int64_t ld,
                                  const float* gamma, const float* beta, const float* inv_s,
                                  const float* s_fold, float eps, const float* range_in, int8_t* q,
                                  float* scale, sq_stream_t stream);

/* The linear's epilogue on its own: y[t, n] = fp16((fp32(acc[t, n]) * x_scale[t]) * w_scale[n]
 * + fp32(bias[n])) (no add when bias is NULL).  acc int32 [M, N]; N % 4 == 0. */
sq_status sq_dequant(const int32_t* acc, const float* x_scale, const float* w_scale,
                     const void* bias_f16, void* y_f16, int64_t M, int64_t N, sq_stream_t stream);

/* Bytes of workspace the stream-K path needs for this shape: nonzero for
 * M <= SQ_SPLITK_MAX_M (needed up to SQ_DECODE_MAX_M tokens, optional above,
 * where it lets sq_w8a8_linear stream the weight of a narrow layer), 0 for
 * larger M or non-positive sizes.  The workspace holds int32 partial sums and
 * per-tile arrival counters of the stream-K path.  The caller zero-fills it once before its first use; every
 * call that completes leaves the counters at zero again.  After a call that
 * reported SQ_ERR_TIMEOUT, zero-fill it again.  Calls that share a workspace
 * must not overlap on the GPU. */
size_t sq_w8a8_workspace_bytes(int64_t M, int64_t N, int64_t K);

/*
 * The W8A8 linear (step 3b): INT8 GEMM with the dequant epilogue fused.
 *   acc[t, n] = sum_k xq[t, k] * wq[n, k]                       (exact int32)
 *   y[t, n]   = fp16( (fp32(acc) * x_scale[t]) * w_scale[n] + fp32(bias[n]) )
 * (no add when bias is NULL).  Per-tensor weight scaling (level O1 of the
 * explainer) is the special case of a w_scale array filled with one value.
 *   xq int8 [M, K]; x_scale fp32 [M]; wq int8 [N, K]; w_scale fp32 [N];
 *   bias fp16 [N] or NULL; y fp16 [M, N]
 * M <= SQ_DECODE_MAX_M runs the weight-streaming stream-K kernel and needs
 * sq_w8a8_workspace_bytes(M, N, K) bytes of workspace.  For
 * SQ_DECODE_MAX_M < M <= SQ_SPLITK_MAX_M the stream-K kernel runs when the
 * workspace given holds sq_w8a8_workspace_bytes(M, N, K) bytes and the layer
 * is narrow (4 * ceil(N / 256) <= the SM count: the tiled kernel's 128 x 256
 * tiles would leave most SMs idle), otherwise the tiled tensor-core kernel
 * (128 x 256 tiles, no workspace; NULL is fine).  M > 128 runs a persistent
 * kernel of 256 x 256 tiles on CTA pairs (tcgen05 cta_group::2), no workspace.
 */
sq_status sq_w8a8_linear(const int8_t* xq, const float* x_scale, const int8_t* wq,
                         const float* w_scale, const void* bias_f16, void* y_f16, int64_t M,
                         int64_t N, int64_t K, void* workspace, size_t ws_bytes,
                         sq_stream_t stream);

/*
 * Producer-side quantization: the linear with the NEXT linear's input
 * quantization fused into its epilogue (the smoothing of the next linear
 * folded into the layer that produces its input -- section "what it does
 * mathematically" -- at level O3 of section "inference": one static
 * activation scale).  Per element, in this order:
 *   y = fp16( (fp32(acc) * x_scale[t]) * w_scale[n] + fp32(bias[n]) )  (as sq_w8a8_linear)
 *   a = relu ? max(y, 0) : y
 *   x = fp32(a) * inv_s_next[n]                  (x = a when inv_s_next is NULL)
 *   xq_next[t, n] = clamp(rint(x * (1 / scale)), -127, 127),  scale = range_next[0] / 127
 * and x_scale_next[t] = scale for every t, so (xq_next, x_scale_next) feed
 * the next sq_w8a8_linear directly: the fp16 y never reaches memory (1 byte
 * written per output instead of 2 written + 3 moved by a separate
 * quantization pass).  range_next is the next linear's static input range
 * (sq_tensor_range).  For the per-token dynamic scale of the next linear
 * see sq_w8a8_linear_quant_dyn.
 *   xq int8 [M, K]; x_scale fp32 [M]; wq int8 [N, K]; w_scale fp32 [N];
 *   bias fp16 [N] or NULL; inv_s_next fp32 [N] or NULL; range_next fp32 [1];
 *   xq_next int8 [M, N]; x_scale_next fp32 [M].  N % 16 == 0 (the next
 *   linear's K).  M <= SQ_DECODE_MAX_M needs the stream-K workspace.
 */
sq_status sq_w8a8_linear_quant(const int8_t* xq, const float* x_scale, const int8_t* wq,
                               const float* w_scale, const void* bias_f16, int relu,
                               const float* inv_s_next, const float* range_next, int8_t* xq_next,
                               float* x_scale_next, int64_t M, int64_t N, int64_t K, void* workspace,
                               size_t ws_bytes, sq_stream_t stream);

/*
 * Producer-side quantization at the next linear's per-token dynamic scale:
 * the linear, an optional ReLU and the next linear's 1/s, then the next
 * linear's default input quantization -- one scale per token, taken from the
 * token's own maximum (the smoothing of the next linear folded into the
 * layer that produces its input: section "what it does mathematically"; the
 * per-token dynamic activation scale: section "inference", level O1).  Per
 * element, in this order:
 *   y = fp16( (fp32(acc) * x_scale[t]) * w_scale[n] + fp32(bias[n]) )  (as sq_w8a8_linear)
 *   a = relu ? max(y, 0) : y                     (a NaN becomes 0)
 *   x = fp32(a) * inv_s_next[n]                  (x = a when inv_s_next is NULL)
 *   x_scale_next[t] = max_n |x[t, n]| / 127      (NaN ignored, as in sq_ln_quant_act)
 *   xq_next[t, n]   = clamp(rint(x * (1 / x_scale_next[t])), -127, 127)
 * -- exactly sq_w8a8_linear, the ReLU, then sq_ln_quant_act with inv_s.  A
 * token's maximum spans every output tile of its row, so the work runs in
 * two launches: the GEMM's epilogue writes a (fp16, into the workspace) and,
 * per token, the maxima of |x| over groups of its columns; a second kernel
 * takes each token's maximum of its groups and writes the codes (no row
 * reduction over the data, no second GEMM).
 *   xq int8 [M, K]; x_scale fp32 [M]; wq int8 [N, K]; w_scale fp32 [N];
 *   bias fp16 [N] or NULL; inv_s_next fp32 [N] or NULL;
 *   xq_next int8 [M, N]; x_scale_next fp32 [M]; N % 16 == 0 (the next
 *   linear's K).  workspace: at least
 *   sq_w8a8_linear_quant_dyn_workspace_bytes(M, N, K) bytes, 16-byte
 *   aligned, zero-filled by the caller once before its first use (for
 *   M <= SQ_DECODE_MAX_M it starts with the stream-K arrival counters, which
 *   every completed call leaves at zero; after a call that reported
 *   SQ_ERR_TIMEOUT zero-fill it again).  Calls sharing a workspace must not
 *   overlap on the GPU.
 */
size_t sq_w8a8_linear_quant_dyn_workspace_bytes(int64_t M, int64_t N, int64_t K);
sq_status sq_w8a8_linear_quant_dyn(const int8_t* xq, const float* x_scale, const int8_t* wq,
                                   const float* w_scale, const void* bias_f16, int relu,
                                   const float* inv_s_next, int8_t* xq_next, float* x_scale_next,
                                   int64_t M, int64_t N, int64_t K, void* workspace, size_t ws_bytes,
                                   sq_stream_t stream);

/*
 * INT8 BMM (the explainer, section "inference": after smoothing, the linear
 * layers and the BMMs of attention run in INT8): `batch` independent
 * products, e.g. one per attention head,
 *   acc[i, m, n] = sum_k a[i, m, k] * b[i, n, k]                      (exact int32)
 *   y[i, m, n]   = fp16( (fp32(acc) * a_scale[i, m]) * b_scale[i, n] )
 * a int8 [batch, M, K] (e.g. Q per head, K contiguous); b int8 [batch, N, K]
 * (K per head for Q K^T; V^T per head for P V, i.e. V stored transposed);
 * a_scale fp32 [batch, M]; b_scale fp32 [batch, N] (per-head scales: every
 * entry of a head equal; per-token scales: one per row); y fp16 [batch, M, N].
 * Items are independent: rows past M or N of one item never mix with the
 * next (3-D tensor maps, out-of-bounds rows read as zero).  Runs the
 * CTA-pair tensor-core kernel over batch x 256 x 256 tiles.
 */
sq_status sq_w8a8_bmm(const int8_t* a, const float* a_scale, const int8_t* b, const float* b_scale,
                      void* y_f16, int64_t batch, int64_t M, int64_t N, int64_t K, sq_stream_t stream);

/* Kernel choice for sq_w8a8_linear_path. */
typedef enum sq_gemm_path {
  SQ_PATH_AUTO = 0,   /* what sq_w8a8_linear does */
  SQ_PATH_TILED = 1,  /* tiled tcgen05 kernel, any M */
  SQ_PATH_SPLITK = 2, /* weight-streaming stream-K kernel, M <= SQ_SPLITK_MAX_M */
  SQ_PATH_PAIR = 3    /* 256 x 256 tiles on CTA pairs (tcgen05 cta_group::2), any M */
} sq_gemm_path;

/* sq_w8a8_linear with the kernel chosen by the caller (testing and
 * benchmarking both kernels on one shape).  Same contract otherwise. */
sq_status sq_w8a8_linear_path(const int8_t* xq, const float* x_scale, const int8_t* wq,
                              const float* w_scale, const void* bias_f16, void* y_f16,
                              int64_t M, int64_t N, int64_t K, void* workspace,
                              size_t ws_bytes, int path, sq_stream_t stream);

/* The INT8 GEMM alone: acc int32 [M, N] = xq @ wq^T, written without the
 * epilogue, through the same kernels (for checking the accumulators). */
sq_status sq_w8a8_gemm_s32(const int8_t* xq, const int8_t* wq, int32_t* acc, int64_t M,
                           int64_t N, int64_t K, void* workspace, size_t ws_bytes, int path,
                           sq_stream_t stream);

/*
 * Allocation-free variant of sq_w8a8_linear for M <= SQ_DECODE_MAX_M (the
 * stream-K decode kernel).  The paper has no counterpart: this entry point
 * exists for callers that cannot allocate device memory -- for example a
 * plug-in inside another runtime that owns every device allocation and hands
 * over only input and output buffers, or a latency-critical path where a
 * cudaMalloc (which may synchronize the whole device) is not acceptable.
 *
 * Instead of a caller workspace it uses one fixed array of
 * SQ_NOALLOC_SCRATCH_BYTES in device global memory, owned by the library;
 * every GPU that loads the library holds that array until the process exits.
 * The call allocates and frees nothing.  Limits: M <= SQ_DECODE_MAX_M
 * (else SQ_ERR_UNSUPPORTED_SHAPE) and at most SQ_NOALLOC_MAX_TILES tiles of
 * 128 output channels, i.e. N <= 524288 (else SQ_ERR_WORKSPACE, the shape
 * needs more scratch than the fixed array holds).  Same numerics and the
 * same output as sq_w8a8_linear.
 *
 * The first call on a device looks up the array's device address (once per
 * device, with that device current); make that first call before any stream
 * capture.  Every call shares the array and it keeps the last call's
 * contents; each call clears the arrival counters it needs before its GEMM
 * kernel runs, on `stream`.  Calls whose kernels overlap on the GPU (on
 * different streams or from different host threads) race on the array and
 * must be serialized by the caller.
 */
#define SQ_NOALLOC_MAX_TILES 4096
#define SQ_NOALLOC_SCRATCH_BYTES (5u * 1024u * 1024u + 4u * SQ_NOALLOC_MAX_TILES)
sq_status sq_w8a8_linear_noalloc(const int8_t* xq, const float* x_scale, const int8_t* wq,
                                 const float* w_scale, const void* bias_f16, void* y_f16,
                                 int64_t M, int64_t N, int64_t K, sq_stream_t stream);

/* Synchronizes `stream`, then reports and clears the current device's status
 * word: SQ_ERR_TIMEOUT if a bounded device wait ran out since the last poll,
 * SQ_ERR_CUDA if the stream reported an error, else SQ_OK. */
sq_status sq_poll_status(sq_stream_t stream);

/* Budget of every device-side bounded wait launched after this call, in
 * nanoseconds (default 2e9; values below 1000 are raised to 1000).  Process
 * wide. */
void sq_set_wait_budget_ns(uint64_t ns);

/* Self-test of the bounded-wait machinery: launches one kernel that waits on
 * a barrier nothing completes, for `budget_ns`; the wait runs out, the kernel
 * records SQ_ERR_TIMEOUT and returns.  Follow with sq_poll_status. */
sq_status sq_selftest_wait_timeout(uint64_t budget_ns, sq_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* SQ_H */
