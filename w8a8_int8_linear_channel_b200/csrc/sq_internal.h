// sq_internal.h -- launchers shared between the C-ABI layer (sq_api.cu) and
// the kernel files.  Not part of the public ABI.
#pragma once

#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace sq {

// Programmatic dependent launch is on unless the environment sets
// SQ_NO_PDL=1 (read once per process).
bool pdl_enabled();

// Launch with programmatic stream serialization (see griddep_wait): the
// kernel's launch and prologue overlap the tail of the previous kernel.
template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                              cudaStream_t stream, Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl_enabled() ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
}

// Per-call launch context filled in by the ABI layer.
struct Ctx {
  int device;
  int num_sms;
  uint32_t* status;    // device address of this device's status word
  uint64_t budget_ns;  // bound of every device-side wait
  cudaStream_t stream;
};

// Row-wise kernels (k_rows.cu).
struct RowArgs {
  const __half* x;  // [rows, ld]
  int64_t rows, K, ld;
  const float* gamma;  // LayerNorm scale or NULL
  const float* beta;   // LayerNorm shift or NULL
  const float* vec;    // inv_s (activation path) or s (weight path) or NULL
  float eps;
  int8_t* q;       // codes [rows, K]
  float* scale;    // per-row scale [rows]
  float* amax;     // calibration running max [K]
  // per-tensor scales (levels O2 / O3 of the explainer, per-tensor weights):
  const float* range_in;  // fixed range [1]: scale = range / 127, codes clamped, no row max
  float* range_out;       // range pass [1]: atomic max of every row's |x_hat|, nothing else written
  int range_per_row;      // range_in / range_out hold one range per row [rows] instead
};

// Elementwise dequantization of int32 accumulators (k_cols.cu).
cudaError_t launch_dequant(const int32_t* acc, const float* sx, const float* sw, const __half* bias, __half* y,
                           int64_t M, int64_t N, const Ctx& c);

cudaError_t launch_ln_quant_act(const RowArgs& a, const Ctx& c);
// Second phase of the per-token producer-side quantization: row t's scale is
// max_g part[t * part_n + g] / 127 and q[t, n] the code of fp32(a[t, n]) *
// inv_s[n] (inv_s NULL: 1) at that scale; N % 8 == 0.
cudaError_t launch_quant_partial_rows(const __half* a, int64_t M, int64_t N, const float* part, int64_t part_n,
                                      const float* inv_s, int8_t* q, float* scale, const Ctx& c);
cudaError_t launch_quantize_weight(const RowArgs& a, const Ctx& c);
cudaError_t launch_calibrate_ln(const RowArgs& a, const Ctx& c);

// Column-wise / elementwise kernels (k_cols.cu).
cudaError_t launch_calib_reset(float* amax, int64_t n, const Ctx& c);
cudaError_t launch_absmax_cols(const __half* x, int64_t rows, int64_t K, int64_t ld, float* amax,
                               const Ctx& c);
cudaError_t launch_smooth(const float* amax_x, const float* amax_w, int64_t K, float alpha,
                          float* s, float* inv_s, const float* gamma, const float* beta,
                          float* gamma_out, float* beta_out, const Ctx& c);
cudaError_t launch_tensor_range(const float* amax, const float* inv_s, int64_t K, float* range,
                                const Ctx& c);
cudaError_t launch_fold_weight(const __half* w, __half* w_out, int64_t N, int64_t K,
                               const float* s, const Ctx& c);

// GEMM kernels (k_gemm_tiled.cu, k_gemm_splitk.cu).
struct GemmArgs {
  const int8_t* xq;  // [M, K]
  const float* sx;   // [M]
  const int8_t* wq;  // [N, K]
  const float* sw;   // [N]
  const __half* bias;  // [N] or NULL
  __half* y;           // [M, N]   (fp16 output) or NULL
  int32_t* acc;        // [M, N]   (int32 output, no epilogue) or NULL
  int64_t M, N, K;
  void* ws;
  size_t ws_bytes;
  // producer-side quantization of the next linear's input at a static
  // per-tensor scale (q_next != NULL; y and acc unused):
  //   a = fp16(y) (ReLU if relu), x = a * inv_s_next[n] (if given),
  //   q_next = clamp(rint(x * (1 / scale)), -127, 127), scale = *range_next / 127
  int8_t* q_next;           // [M, N]
  float* sx_next;           // [M], every entry = scale
  const float* inv_s_next;  // [N] or NULL
  const float* range_next;  // [1]
  int relu;
  // batched GEMM (INT8 BMM): batch items of [M, K] x [N, K]^T -> [M, N], the
  // scales per (item, row) sx [batch, M] and per (item, column) sw [batch, N]
  int64_t batch;  // 0 = not batched
  // producer-side quantization at the next linear's per-token dynamic scale,
  // first phase (part != NULL; y receives a = fp16(y), ReLU if relu): per row
  // the maxima of |fp32(a) * inv_s_next[n]| over consecutive column groups,
  // part[row * part_n + group] (groups of 128 columns on the CTA-pair kernel,
  // 32 on the stream-K kernel); launch_quant_partial_rows then quantizes a
  // with each row's maximum.
  float* part;
  int64_t part_n;
};

cudaError_t launch_gemm_tiled(const GemmArgs& g, const Ctx& c);  // 128 x 256 tiles
cudaError_t launch_gemm_pair(const GemmArgs& g, const Ctx& c);   // 256 x 256 tiles on CTA pairs
cudaError_t launch_bmm_pair(const GemmArgs& g, const Ctx& c);    // the same, batched (g.batch items)
cudaError_t launch_gemm_splitk(const GemmArgs& g, const Ctx& c);
size_t splitk_workspace_bytes(int64_t M, int64_t N, int64_t K, int num_sms);

cudaError_t launch_wait_selftest(uint64_t budget_ns, const Ctx& c);

// Launch context of the current device (arch check, status word, wait
// budget); returns an sq_status code (0 = ok).
int call_context(void* stream, Ctx* ctx);

// Driver entry point for tensor-map encoding (resolved once through the
// runtime, so the library does not link libcuda directly).
void* tensor_map_encoder();

}  // namespace sq
