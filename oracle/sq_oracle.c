/*
 * CPU oracle for the SmoothQuant W8A8 linear layer.
 *
 * TEST INFRASTRUCTURE ONLY.  Only tests, the smoke check and the CPU-baseline
 * leg of the benchmark may load this library.  The product path (the CUDA
 * library) shares no code with it and never calls it.
 *
 * Every function is a plain loop that restates one step of the method in a
 * fixed operation order, written for a reader to check by eye against the
 * sources:
 *   [SQ]  "SmoothQuant: Accurate and Efficient Post-Training Quantization for
 *         Large Language Models" (Xiao et al.), as explained on the abeam.tech
 *         page: sections "Calibration" (glossary), "smoothing factor" (the
 *         formula s_j = max|X_j|^a / max|W_j|^(1-a)), "what it does
 *         mathematically" (Y = (X diag(s)^-1)(diag(s) W), folded offline into
 *         the preceding LayerNorm), "why activations are hard to quantize"
 *         (absmax sets the INT8 range) and "inference" (O1: per-token
 *         activation scale).
 *   [Q]   the itmedia quantization tutorial, section 3: find the range, shrink
 *         it by a scale, round to the nearest level, multiply the scale back
 *         at inference (53 -> 5.3 -> 5 -> 50).
 *
 * Numerics (identical on the CUDA side, each op IEEE round-to-nearest-even,
 * no FMA contraction: build with -ffp-contract=off):
 *   scale = absmax / 127.0f ; inv = scale > 0 ? 1.0f / scale : 0
 *   q = clamp(rint(x * inv), -127, 127), NaN products give 0
 *   acc = exact int32 sum of int8 products
 *   y = fp16( ((float)acc * sx[t]) * sw[n] + (float)bias[n] )   (no add if bias is NULL)
 * LayerNorm statistics are exact integer sums (see ln_stats below), so the
 * LN output does not depend on summation order.
 */
#include <math.h>
#include <stdint.h>
#include <string.h>

#ifdef _OPENMP
#include <omp.h>
#endif

typedef unsigned __int128 u128;
typedef __int128 i128;

/* ---------------------------------------------------------------- fp16 --- */
/* IEEE binary16 <-> binary32 through the compiler's _Float16 type: widening is
 * exact, narrowing rounds to nearest even (overflow to +-inf). */
static float h2f(uint16_t b) {
  _Float16 h;
  memcpy(&h, &b, 2);
  return (float)h;
}

static uint16_t f2h(float f) {
  _Float16 h = (_Float16)f;
  uint16_t b;
  memcpy(&b, &h, 2);
  return b;
}

void oracle_half_to_float(const uint16_t* in, float* out, int64_t n) {
  for (int64_t i = 0; i < n; ++i) out[i] = h2f(in[i]);
}

void oracle_float_to_half(const float* in, uint16_t* out, int64_t n) {
  for (int64_t i = 0; i < n; ++i) out[i] = f2h(in[i]);
}

/* --------------------------------------------------- quantize primitive --- */
/* [Q] section 3 / [SQ] "why activations are hard": the range (absmax) fixes
 * the scale; a value is divided by the scale (here: multiplied by its
 * reciprocal), rounded to the nearest integer level (ties to even) and kept
 * inside the symmetric INT8 range [-127, 127]. */
static int8_t quantize_one(float x, float inv) {
  float p = x * inv;
  if (isnan(p)) return 0;
  float r = rintf(p); /* default rounding mode: nearest, ties to even */
  if (r > 127.0f) r = 127.0f;
  if (r < -127.0f) r = -127.0f;
  return (int8_t)r;
}

static float scale_of(float amax) { return amax / 127.0f; }

static float inv_of(float scale) { return scale > 0.0f ? 1.0f / scale : 0.0f; }

/* Quantize n values with one explicit scale (the [Q] worked example uses a
 * given scale of 10).  Returns nothing; codes land in q. */
void oracle_quantize_with_scale(const float* x, int64_t n, float scale, int8_t* q) {
  float inv = inv_of(scale);
  for (int64_t i = 0; i < n; ++i) q[i] = quantize_one(x[i], inv);
}

/* ------------------------------------------------------------ LayerNorm --- */
/* The pages fold s into "the preceding LayerNorm" but do not define the
 * LayerNorm itself.  Reading: the usual (biased-variance) LayerNorm
 *   x = ((h - mu) * rstd) * gamma + beta,   rstd = 1 / sqrt(var + eps).
 * mu and var come from exact sums: every fp16 value h is v * 2^-24 for an
 * integer v with |v| < 2^40, so S1 = sum v (fits int64) and
 * S2 = sum v^2 (< 2^97, fits 128 bits) are exact.  They are turned into
 * doubles by this fixed sequence of correctly rounded operations:
 *   d(S2) = (double)(S2 >> 64) * 2^64 + (double)(S2 mod 2^64)
 *   mu    = (double)S1 / (K * 2^24)
 *   var   = max(d(S2) / (K * 2^48) - mu * mu, 0)
 *   rstd  = 1 / sqrt(var + (double)eps)
 * and then rounded to float.  A row holding an Inf or a NaN has no finite
 * mean or variance; as in the usual LayerNorm's IEEE arithmetic, both are
 * then NaN (so is every value of the row's LayerNorm output). */
static void ln_stats(const uint16_t* h, int64_t K, float eps, float* mu32, float* rstd32) {
  i128 s1 = 0;
  u128 s2 = 0;
  for (int64_t k = 0; k < K; ++k) {
    if (!isfinite(h2f(h[k]))) {
      *mu32 = NAN;
      *rstd32 = NAN;
      return;
    }
  }
  for (int64_t k = 0; k < K; ++k) {
    double hv = (double)h2f(h[k]);
    int64_t v = (int64_t)(hv * 16777216.0); /* exact: hv * 2^24 is an integer */
    s1 += v;
    s2 += (u128)((i128)v * (i128)v);
  }
  double two64 = 18446744073709551616.0;
  double d_s1 = (double)(int64_t)s1;
  double d_s2 = (double)(uint64_t)(s2 >> 64) * two64 + (double)(uint64_t)s2;
  double mean = d_s1 / ((double)K * 16777216.0);
  double ex2 = d_s2 / ((double)K * 281474976710656.0);
  double var = ex2 - mean * mean;
  if (var < 0.0) var = 0.0;
  double rstd = 1.0 / sqrt(var + (double)eps);
  *mu32 = (float)mean;
  *rstd32 = (float)rstd;
}

/* The smoothed activation row x_hat (fp32) of one token:
 *   gamma given : x = ((h - mu) * rstd) * gamma + beta   (beta NULL -> no add)
 *   otherwise   : x = h
 *   inv_s given : x = x * inv_s                           ([SQ] X diag(s)^-1)
 */
static void act_row(const uint16_t* h, int64_t K, const float* gamma, const float* beta,
                    const float* inv_s, float eps, float* out) {
  if (gamma) {
    float mu, rstd;
    ln_stats(h, K, eps, &mu, &rstd);
    for (int64_t k = 0; k < K; ++k) {
      float d = h2f(h[k]) - mu;
      float t = d * rstd;
      float u = t * gamma[k];
      out[k] = beta ? u + beta[k] : u;
    }
  } else {
    for (int64_t k = 0; k < K; ++k) out[k] = h2f(h[k]);
  }
  if (inv_s)
    for (int64_t k = 0; k < K; ++k) out[k] = out[k] * inv_s[k];
}

/* LayerNorm statistics of each row, exposed so tests can pin them. */
void oracle_ln_stats(const uint16_t* h, int64_t rows, int64_t K, int64_t ld, float eps,
                     float* mu_out, float* rstd_out) {
  for (int64_t r = 0; r < rows; ++r) ln_stats(h + r * ld, K, eps, mu_out + r, rstd_out + r);
}

/* The fp32 activation rows (before quantization), exposed for tests. */
void oracle_act_rows(const uint16_t* h, int64_t rows, int64_t K, int64_t ld, const float* gamma,
                     const float* beta, const float* inv_s, float eps, float* out) {
  for (int64_t r = 0; r < rows; ++r) act_row(h + r * ld, K, gamma, beta, inv_s, eps, out + r * K);
}

/* ---------------------------------------------------------- calibration --- */
/* [SQ] glossary "Calibration" and "smoothing factor": a_j = max over the
 * calibration tokens t of |X[t, j]|, kept as a running maximum across calls.
 * X is either the raw input rows or their LayerNorm output (gamma given).
 * The same routine gives b_j = max_n |W[n, j]| when called on W [N, K]. */
void oracle_calibrate_absmax(const uint16_t* x, int64_t rows, int64_t K, int64_t ld,
                             const float* gamma, const float* beta, float eps, float* amax_inout,
                             float* scratch_row /* K floats */) {
  for (int64_t r = 0; r < rows; ++r) {
    act_row(x + r * ld, K, gamma, beta, 0, eps, scratch_row);
    for (int64_t j = 0; j < K; ++j) {
      float a = fabsf(scratch_row[j]);
      if (a > amax_inout[j]) amax_inout[j] = a;
    }
  }
}

/* ------------------------------------------------------ smoothing factor --- */
/* [SQ] "smoothing factor": s_j = max|X_j|^alpha / max|W_j|^(1 - alpha), both
 * maxima floored at 1e-5 so that a dead channel still gives a finite s.
 * Evaluated in double precision and rounded once to float; inv_s = 1 / s in
 * float. */
void oracle_smooth(const float* amax_x, const float* amax_w, int64_t K, float alpha, float* s,
                   float* inv_s) {
  double a = (double)alpha;
  for (int64_t j = 0; j < K; ++j) {
    double x = amax_x[j] > 1e-5f ? (double)amax_x[j] : (double)1e-5f;
    double w = amax_w[j] > 1e-5f ? (double)amax_w[j] : (double)1e-5f;
    double sj = pow(x, a) / pow(w, 1.0 - a);
    s[j] = (float)sj;
    inv_s[j] = 1.0f / s[j];
  }
}

/* ------------------------------------------------------------------ fold --- */
/* [SQ] "what it does mathematically": the scaling is absorbed offline,
 *   gamma' = gamma * inv_s, beta' = beta * inv_s  (LayerNorm, fp32), and
 *   W'[n, j] = fp16(W[n, j] * s_j)               (the weight, stored fp16). */
void oracle_fold_ln(const float* gamma, const float* beta, const float* inv_s, int64_t K,
                    float* gamma_out, float* beta_out) {
  for (int64_t j = 0; j < K; ++j) {
    if (gamma) gamma_out[j] = gamma[j] * inv_s[j];
    if (beta) beta_out[j] = beta[j] * inv_s[j];
  }
}

void oracle_fold_weight(const uint16_t* w, int64_t N, int64_t K, const float* s, uint16_t* w_out) {
  for (int64_t n = 0; n < N; ++n)
    for (int64_t j = 0; j < K; ++j) w_out[n * K + j] = f2h(h2f(w[n * K + j]) * s[j]);
}

/* --------------------------------------------------- weight quantization --- */
/* Per output channel n: sw[n] = max_k |W'[n, k]| / 127 and
 * wq[n, k] = clamp(rint(W'[n, k] * (1 / sw[n])), -127, 127). */
void oracle_quantize_weight(const uint16_t* w, int64_t N, int64_t K, int8_t* wq, float* sw) {
#pragma omp parallel for schedule(static)
  for (int64_t n = 0; n < N; ++n) {
    const uint16_t* row = w + n * K;
    float amax = 0.0f;
    for (int64_t k = 0; k < K; ++k) {
      float a = fabsf(h2f(row[k]));
      if (a > amax) amax = a;
    }
    float sc = scale_of(amax);
    float inv = inv_of(sc);
    sw[n] = sc;
    for (int64_t k = 0; k < K; ++k) wq[n * K + k] = quantize_one(h2f(row[k]), inv);
  }
}

/* ---------------------------------------- per-token activation quantization --- */
/* [SQ] "inference", level O1: one dynamic scale per token row,
 * sx[t] = max_k |x_hat[t, k]| / 127, xq = clamp(rint(x_hat * (1 / sx)), +-127). */
void oracle_ln_quant_act(const uint16_t* h, int64_t M, int64_t K, int64_t ld, const float* gamma,
                         const float* beta, const float* inv_s, float eps, int8_t* xq, float* sx,
                         float* scratch /* nthreads * K floats */) {
#pragma omp parallel for schedule(static)
  for (int64_t t = 0; t < M; ++t) {
    int tid = 0;
#ifdef _OPENMP
    tid = omp_get_thread_num();
#endif
    float* row = scratch + (int64_t)tid * K;
    act_row(h + t * ld, K, gamma, beta, inv_s, eps, row);
    float amax = 0.0f;
    for (int64_t k = 0; k < K; ++k) {
      float a = fabsf(row[k]);
      if (a > amax) amax = a;
    }
    float sc = scale_of(amax);
    float inv = inv_of(sc);
    sx[t] = sc;
    for (int64_t k = 0; k < K; ++k) xq[t * K + k] = quantize_one(row[k], inv);
  }
}

/* ------------------------------------------ per-tensor levels (O1 - O3) --- */
/* [SQ] "inference": the efficiency levels differ only in how coarse the
 * scales are.  O1: activations per token, dynamic; weights per tensor.
 * O2: activations and weights per tensor, dynamic.  O3: both per tensor,
 * static (the activation scale is fixed offline from calibration).  A
 * per-tensor scale is the same quantizer with one range for the whole tensor:
 *   scale = range / 127, q = clamp(rint(x * (1 / scale)), -127, 127).
 * The scale is returned once per row (sw[n] or sx[t], all equal) so the
 * INT8 GEMM and its dequant epilogue stay exactly as in O1. */

/* Weights, one scale for all of W' [N, K]: range = max_{n,k} |W'[n, k]|. */
void oracle_quantize_weight_tensor(const uint16_t* w, int64_t N, int64_t K, int8_t* wq, float* sw,
                                   float* range_out) {
  float range = 0.0f;
  for (int64_t i = 0; i < N * K; ++i) {
    float a = fabsf(h2f(w[i]));
    if (a > range) range = a;
  }
  float sc = scale_of(range);
  float inv = inv_of(sc);
  for (int64_t n = 0; n < N; ++n) sw[n] = sc;
  for (int64_t i = 0; i < N * K; ++i) wq[i] = quantize_one(h2f(w[i]), inv);
  *range_out = range;
}

/* Level O2 activations: one dynamic range over every token of this batch,
 * range = max_{t,k} |x_hat[t, k]|.  Two passes over the rows (the range must
 * be known before the first code). */
void oracle_ln_quant_act_tensor(const uint16_t* h, int64_t M, int64_t K, int64_t ld,
                                const float* gamma, const float* beta, const float* inv_s, float eps,
                                int8_t* xq, float* sx, float* range_out,
                                float* scratch_row /* K floats */) {
  float range = 0.0f;
  for (int64_t t = 0; t < M; ++t) {
    act_row(h + t * ld, K, gamma, beta, inv_s, eps, scratch_row);
    for (int64_t k = 0; k < K; ++k) {
      float a = fabsf(scratch_row[k]);
      if (a > range) range = a;
    }
  }
  float sc = scale_of(range);
  float inv = inv_of(sc);
  for (int64_t t = 0; t < M; ++t) {
    act_row(h + t * ld, K, gamma, beta, inv_s, eps, scratch_row);
    sx[t] = sc;
    for (int64_t k = 0; k < K; ++k) xq[t * K + k] = quantize_one(scratch_row[k], inv);
  }
  *range_out = range;
}

/* Level O3 activations: the range was fixed offline; values outside it
 * saturate at -127 / 127 (the clamp of quantize_one). */
void oracle_ln_quant_act_static(const uint16_t* h, int64_t M, int64_t K, int64_t ld,
                                const float* gamma, const float* beta, const float* inv_s, float eps,
                                float range, int8_t* xq, float* sx, float* scratch_row /* K floats */) {
  float sc = scale_of(range);
  float inv = inv_of(sc);
  for (int64_t t = 0; t < M; ++t) {
    act_row(h + t * ld, K, gamma, beta, inv_s, eps, scratch_row);
    sx[t] = sc;
    for (int64_t k = 0; k < K; ++k) xq[t * K + k] = quantize_one(scratch_row[k], inv);
  }
}

/* The static per-tensor range of the smoothed activation from calibrated
 * per-channel ranges: max_j amax[j] (amax measured on the runtime transform,
 * e.g. the LayerNorm with the folded gamma' / beta'), or, when the runtime
 * multiplies by inv_s, max_j fp32(amax[j] * inv_s[j]) -- rounding is
 * monotonic, so this is the largest |x * inv_s_j| over the calibration set. */
float oracle_tensor_range(const float* amax, const float* inv_s, int64_t K) {
  float range = 0.0f;
  for (int64_t j = 0; j < K; ++j) {
    float a = inv_s ? amax[j] * inv_s[j] : amax[j];
    if (a > range) range = a;
  }
  return range;
}

/* ------------------------------------------------------------- INT8 GEMM --- */
/* [SQ] glossary "INT8 GEMM": acc[t, n] = sum_k xq[t, k] * wq[n, k], int32.
 * K <= 133144 keeps |acc| <= 133144 * 127^2 < 2^31. */
void oracle_int_gemm(const int8_t* xq, const int8_t* wq, int64_t M, int64_t N, int64_t K,
                     int32_t* acc) {
#pragma omp parallel for schedule(static)
  for (int64_t t = 0; t < M; ++t)
    for (int64_t n = 0; n < N; ++n) {
      int32_t sum = 0;
      for (int64_t k = 0; k < K; ++k) sum += (int32_t)xq[t * K + k] * (int32_t)wq[n * K + k];
      acc[t * N + n] = sum;
    }
}

/* Same sum in int64, to check that the int32 sum never wrapped. */
void oracle_int_gemm64(const int8_t* xq, const int8_t* wq, int64_t M, int64_t N, int64_t K,
                       int64_t* acc) {
#pragma omp parallel for schedule(static)
  for (int64_t t = 0; t < M; ++t)
    for (int64_t n = 0; n < N; ++n) {
      int64_t sum = 0;
      for (int64_t k = 0; k < K; ++k) sum += (int64_t)xq[t * K + k] * (int64_t)wq[n * K + k];
      acc[t * N + n] = sum;
    }
}

/* ------------------------------------------------------ dequant epilogue --- */
/* [Q] "multiply the scale back": y = fp16(((float)acc * sx[t]) * sw[n] + bias[n]). */
void oracle_dequant(const int32_t* acc, const float* sx, const float* sw, const uint16_t* bias,
                    int64_t M, int64_t N, uint16_t* y) {
#pragma omp parallel for schedule(static)
  for (int64_t t = 0; t < M; ++t)
    for (int64_t n = 0; n < N; ++n) {
      float v = (float)acc[t * N + n] * sx[t];
      v = v * sw[n];
      if (bias) v = v + h2f(bias[n]);
      y[t * N + n] = f2h(v);
    }
}

/* The whole runtime linear: INT8 GEMM then the dequant epilogue. */
void oracle_w8a8_linear(const int8_t* xq, const float* sx, const int8_t* wq, const float* sw,
                        const uint16_t* bias, int64_t M, int64_t N, int64_t K, uint16_t* y) {
#pragma omp parallel for schedule(static)
  for (int64_t t = 0; t < M; ++t)
    for (int64_t n = 0; n < N; ++n) {
      int32_t sum = 0;
      for (int64_t k = 0; k < K; ++k) sum += (int32_t)xq[t * K + k] * (int32_t)wq[n * K + k];
      float v = (float)sum * sx[t];
      v = v * sw[n];
      if (bias) v = v + h2f(bias[n]);
      y[t * N + n] = f2h(v);
    }
}

/* ------------------------------------- producer-side quantization (fused) --- */
/* [SQ] "what it does mathematically" folds s into the layer that produces a
 * linear's input; with the next linear at level O3 ("inference": one static
 * activation scale), the producing linear can hand over INT8 codes directly.
 * The result is defined as the plain composition of the steps above:
 *   y    = fp16(((float)acc * sx[t]) * sw[n] + bias[n])     (the linear's output)
 *   a    = relu ? max(y, 0) : y                            (fp16 activation)
 *   x    = (float)a * inv_s_next[n]                        (the next linear's X diag(s)^-1)
 *   q    = clamp(rint(x * (1 / scale)), -127, 127),  scale = range_next / 127
 * and sx_next[t] = scale for every token.  inv_s_next may be NULL (x = a). */
void oracle_w8a8_linear_quant_static(const int8_t* xq, const float* sx, const int8_t* wq,
                                     const float* sw, const uint16_t* bias, int relu,
                                     const float* inv_s_next, float range_next, int64_t M,
                                     int64_t N, int64_t K, int8_t* q_next, float* sx_next) {
  float sc = scale_of(range_next);
  float inv = inv_of(sc);
#pragma omp parallel for schedule(static)
  for (int64_t t = 0; t < M; ++t) {
    sx_next[t] = sc;
    for (int64_t n = 0; n < N; ++n) {
      int32_t sum = 0;
      for (int64_t k = 0; k < K; ++k) sum += (int32_t)xq[t * K + k] * (int32_t)wq[n * K + k];
      float v = (float)sum * sx[t];
      v = v * sw[n];
      if (bias) v = v + h2f(bias[n]);
      float a = h2f(f2h(v));
      if (relu && !(a > 0.0f)) a = 0.0f;
      float x = inv_s_next ? a * inv_s_next[n] : a;
      q_next[t * N + n] = quantize_one(x, inv);
    }
  }
}

/* --------------------------------------------------------------- INT8 BMM --- */
/* [SQ] "inference": with the smoothing in place the attention BMMs run in
 * INT8 too.  `batch` independent products (one per head):
 *   acc[i, m, n] = sum_k a[i, m, k] * b[i, n, k]              (int32)
 *   y[i, m, n]   = fp16((float)acc * a_scale[i, m] * b_scale[i, n])  (in that order) */
void oracle_w8a8_bmm(const int8_t* a, const float* a_scale, const int8_t* b, const float* b_scale,
                     int64_t batch, int64_t M, int64_t N, int64_t K, uint16_t* y) {
  for (int64_t i = 0; i < batch; ++i) {
    const int8_t* ai = a + i * M * K;
    const int8_t* bi = b + i * N * K;
#pragma omp parallel for schedule(static)
    for (int64_t m = 0; m < M; ++m)
      for (int64_t n = 0; n < N; ++n) {
        int32_t sum = 0;
        for (int64_t k = 0; k < K; ++k) sum += (int32_t)ai[m * K + k] * (int32_t)bi[n * K + k];
        float v = (float)sum * a_scale[i * M + m];
        v = v * b_scale[i * N + n];
        y[(i * M + m) * N + n] = f2h(v);
      }
  }
}

int oracle_num_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}

void oracle_set_num_threads(int n) {
#ifdef _OPENMP
  if (n > 0) omp_set_num_threads(n);
#else
  (void)n;
#endif
}
