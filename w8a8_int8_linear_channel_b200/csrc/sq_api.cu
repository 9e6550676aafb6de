// sq_api.cu -- the C ABI declared in include/sq.h: host-side argument checks,
// device / architecture checks, the per-device status word of the bounded
// device waits, and dispatch to the kernels.  No entry point allocates
// device memory.
#include <stdlib.h>

#include <atomic>
#include <mutex>

#include "../../include/sq.h"
#include "sq_internal.h"
#include "sq_ptx.cuh"

namespace sq {

// One status word per device (a bounded wait that ran out writes DEV_TIMEOUT).
__device__ uint32_t g_status_word;

namespace {

constexpr int kMaxDevices = 64;

struct DeviceInfo {
  std::once_flag once;
  sq_status state = SQ_ERR_CUDA;
  int num_sms = 0;
  uint32_t* status = nullptr;
};

DeviceInfo g_dev[kMaxDevices];
std::atomic<uint64_t> g_budget_ns{2000000000ull};

void* g_encoder = nullptr;
std::once_flag g_encoder_once;

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Current device: must exist and be compute capability 10.0.  Resolves the
// device address of the status word once per device.
sq_status current_ctx(sq_stream_t stream, Ctx* ctx) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0) {
    cudaGetLastError();
    return SQ_ERR_CUDA;
  }
  if (dev >= kMaxDevices) return SQ_ERR_CUDA;
  DeviceInfo& d = g_dev[dev];
  std::call_once(d.once, [&] {
    int major = 0, minor = 0, sms = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
      cudaGetLastError();
      d.state = SQ_ERR_CUDA;
      return;
    }
    if (major != 10 || minor != 0) {
      d.state = SQ_ERR_ARCH;
      return;
    }
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_status_word) != cudaSuccess) {
      cudaGetLastError();
      d.state = SQ_ERR_CUDA;
      return;
    }
    d.status = static_cast<uint32_t*>(p);
    d.num_sms = sms;
    d.state = SQ_OK;
  });
  if (d.state != SQ_OK) return d.state;
  ctx->device = dev;
  ctx->num_sms = d.num_sms;
  ctx->status = d.status;
  ctx->budget_ns = g_budget_ns.load(std::memory_order_relaxed);
  ctx->stream = static_cast<cudaStream_t>(stream);
  return SQ_OK;
}

sq_status launched(cudaError_t e) {
  if (e != cudaSuccess) {
    cudaGetLastError();
    return SQ_ERR_CUDA;
  }
  return SQ_OK;
}

sq_status check_k(int64_t K) {
  if (K <= 0) return SQ_ERR_INVALID_ARG;
  if (K > SQ_MAX_K) return SQ_ERR_K_OVERFLOW;
  if (K % 16 != 0) return SQ_ERR_UNSUPPORTED_SHAPE;
  return SQ_OK;
}

sq_status check_ld(int64_t K, int64_t ld) {
  if (ld < K) return SQ_ERR_INVALID_ARG;
  if (ld % 8 != 0) return SQ_ERR_MISALIGNED;
  return SQ_OK;
}

// Optional pointer: NULL is fine, otherwise 16-byte aligned.
bool opt_aligned(const void* p) { return p == nullptr || aligned16(p); }

__global__ void k_wait_selftest(uint32_t* status, uint64_t budget) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ uint32_t abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&bar), 1);
    abort_flag = 0;
    fence_barrier_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    // nothing ever arrives on this barrier: the bounded wait must run out
    mbar_wait(smem_u32(&bar), 0, budget, status, &abort_flag);
  }
  __syncthreads();
}

sq_status linear_impl(const int8_t* xq, const float* x_scale, const int8_t* wq,
                      const float* w_scale, const void* bias_f16, void* y_f16, int32_t* acc,
                      int64_t M, int64_t N, int64_t K, void* workspace, size_t ws_bytes, int path,
                      sq_stream_t stream) {
  const bool i32 = acc != nullptr;
  if (!xq || !wq) return SQ_ERR_INVALID_ARG;
  if (!i32 && (!x_scale || !w_scale || !y_f16)) return SQ_ERR_INVALID_ARG;
  if (M <= 0 || N <= 0) return SQ_ERR_INVALID_ARG;
  sq_status st = check_k(K);
  if (st != SQ_OK) return st;
  if (path < SQ_PATH_AUTO || path > SQ_PATH_PAIR) return SQ_ERR_INVALID_ARG;
  if (!aligned16(xq) || !aligned16(wq) || !opt_aligned(x_scale) || !opt_aligned(w_scale) ||
      !opt_aligned(bias_f16) || !opt_aligned(y_f16) || !opt_aligned(acc))
    return SQ_ERR_MISALIGNED;
  if (M > 0x7fffffffLL || N > 0x7fffffffLL) return SQ_ERR_UNSUPPORTED_SHAPE;
  if (path == SQ_PATH_SPLITK && M > SQ_SPLITK_MAX_M) return SQ_ERR_UNSUPPORTED_SHAPE;

  Ctx ctx;
  st = current_ctx(stream, &ctx);
  if (st != SQ_OK) return st;
  if (path == SQ_PATH_AUTO) {
    if (M <= SQ_DECODE_MAX_M) {
      path = SQ_PATH_SPLITK;
    } else if (M <= SQ_SPLITK_MAX_M && 4 * ((N + 255) / 256) <= ctx.num_sms && workspace != nullptr &&
               aligned16(workspace) && ws_bytes >= splitk_workspace_bytes(M, N, K, ctx.num_sms)) {
      // a narrow layer: 128 x 256 tiles would leave most SMs idle, while the
      // stream-K kernel streams the weight on all of them
      path = SQ_PATH_SPLITK;
    }
  }

  GemmArgs g{};
  g.xq = xq;
  g.sx = x_scale;
  g.wq = wq;
  g.sw = w_scale;
  g.bias = static_cast<const __half*>(bias_f16);
  g.y = static_cast<__half*>(y_f16);
  g.acc = acc;
  g.M = M;
  g.N = N;
  g.K = K;
  g.ws = workspace;
  g.ws_bytes = ws_bytes;
  if (path == SQ_PATH_SPLITK) {
    const size_t need = splitk_workspace_bytes(M, N, K, ctx.num_sms);
    if (workspace == nullptr || ws_bytes < need || !aligned16(workspace)) return SQ_ERR_WORKSPACE;
    return launched(launch_gemm_splitk(g, ctx));
  }
  if (path == SQ_PATH_PAIR) return launched(launch_gemm_pair(g, ctx));
  if (path == SQ_PATH_TILED) return launched(launch_gemm_tiled(g, ctx));
  // automatic: 256 x 256 tiles on CTA pairs once the token count fills them
  // (their double-buffered accumulators hide the epilogue; with two K boxes
  // per stage they also lead the single-CTA 256 x 256 kernel at long K:
  // 8192 x 12288 x 49152 and 4096 x 12288 x 16384 12-14 % faster);
  // single-CTA 128-row tiles below 129 tokens
  if (M <= 128) return launched(launch_gemm_tiled(g, ctx));
  return launched(launch_gemm_pair(g, ctx));
}

}  // namespace

int call_context(void* stream, Ctx* ctx) { return current_ctx(stream, ctx); }

bool pdl_enabled() {
  static const bool on = [] {
    const char* v = getenv("SQ_NO_PDL");
    return !(v && v[0] == '1');
  }();
  return on;
}

void* tensor_map_encoder() {
  std::call_once(g_encoder_once, [] {
    cudaDriverEntryPointQueryResult q;
    void* fn = nullptr;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      g_encoder = fn;
    else
      cudaGetLastError();
  });
  return g_encoder;
}

cudaError_t launch_wait_selftest(uint64_t budget_ns, const Ctx& c) {
  k_wait_selftest<<<1, 32, 0, c.stream>>>(c.status, budget_ns);
  return cudaGetLastError();
}

}  // namespace sq

using namespace sq;

// Argument checks and row arguments shared by the per-tensor activation entry points.
static sq_status act_args(const void* h_f16, int64_t M, int64_t K, int64_t ld, const float* gamma,
                   const float* beta, const float* inv_s, float eps, int8_t* xq, float* x_scale,
                   const float* range, RowArgs* a) {
  if (!h_f16 || !xq || !x_scale || !range || M <= 0) return SQ_ERR_INVALID_ARG;
  if (!gamma && beta) return SQ_ERR_INVALID_ARG;
  sq_status st = check_k(K);
  if (st != SQ_OK) return st;
  if ((st = check_ld(K, ld)) != SQ_OK) return st;
  if (!aligned16(h_f16) || !aligned16(xq) || !aligned16(x_scale) || !aligned16(range) ||
      !opt_aligned(gamma) || !opt_aligned(beta) || !opt_aligned(inv_s))
    return SQ_ERR_MISALIGNED;
  *a = RowArgs{};
  a->x = static_cast<const __half*>(h_f16);
  a->rows = M;
  a->K = K;
  a->ld = ld;
  a->gamma = gamma;
  a->beta = beta;
  a->vec = inv_s;
  a->eps = eps;
  a->q = xq;
  a->scale = x_scale;
  return SQ_OK;
}

// Row arguments of the per-row-range entry points: the weight fold (s_fold)
// or the activation transform (LayerNorm / 1/s), never both.
static sq_status ranged_args(const void* x_f16, int64_t rows, int64_t K, int64_t ld, const float* gamma,
                             const float* beta, const float* inv_s, const float* s_fold, float eps,
                             RowArgs* a) {
  if (!x_f16 || rows <= 0) return SQ_ERR_INVALID_ARG;
  if (!gamma && beta) return SQ_ERR_INVALID_ARG;
  if (s_fold && (gamma || inv_s)) return SQ_ERR_INVALID_ARG;
  sq_status st = check_k(K);
  if (st != SQ_OK) return st;
  if ((st = check_ld(K, ld)) != SQ_OK) return st;
  if (!aligned16(x_f16) || !opt_aligned(gamma) || !opt_aligned(beta) || !opt_aligned(inv_s) ||
      !opt_aligned(s_fold))
    return SQ_ERR_MISALIGNED;
  *a = RowArgs{};
  a->x = static_cast<const __half*>(x_f16);
  a->rows = rows;
  a->K = K;
  a->ld = ld;
  a->gamma = gamma;
  a->beta = beta;
  a->vec = s_fold ? s_fold : inv_s;
  a->eps = eps;
  a->range_per_row = 1;
  return SQ_OK;
}

extern "C" {

const char* sq_status_string(int status) {
  switch (status) {
    case SQ_OK: return "SQ_OK";
    case SQ_ERR_INVALID_ARG: return "SQ_ERR_INVALID_ARG";
    case SQ_ERR_MISALIGNED: return "SQ_ERR_MISALIGNED";
    case SQ_ERR_UNSUPPORTED_SHAPE: return "SQ_ERR_UNSUPPORTED_SHAPE";
    case SQ_ERR_K_OVERFLOW: return "SQ_ERR_K_OVERFLOW";
    case SQ_ERR_WORKSPACE: return "SQ_ERR_WORKSPACE";
    case SQ_ERR_ARCH: return "SQ_ERR_ARCH";
    case SQ_ERR_CUDA: return "SQ_ERR_CUDA";
    case SQ_ERR_TIMEOUT: return "SQ_ERR_TIMEOUT";
    default: return "SQ_ERR_UNKNOWN";
  }
}

int sq_abi_version(void) { return 200; }

sq_status sq_calibrate_reset(float* amax, int64_t n, sq_stream_t stream) {
  if (!amax || n <= 0) return SQ_ERR_INVALID_ARG;
  if (!aligned16(amax)) return SQ_ERR_MISALIGNED;
  Ctx ctx;
  sq_status st = current_ctx(stream, &ctx);
  if (st != SQ_OK) return st;
  return launched(launch_calib_reset(amax, n, ctx));
}

sq_status sq_calibrate_absmax(const void* x_f16, int64_t rows, int64_t K, int64_t ld,
                              const float* ln_gamma, const float* ln_beta, float ln_eps,
                              float* amax_inout, sq_stream_t stream) {
  if (!x_f16 || !amax_inout || rows <= 0) return SQ_ERR_INVALID_ARG;
  if (!ln_gamma && ln_beta) return SQ_ERR_INVALID_ARG;
  sq_status st = check_k(K);
  if (st != SQ_OK) return st;
  if ((st = check_ld(K, ld)) != SQ_OK) return st;
  if (!aligned16(x_f16) || !aligned16(amax_inout) || !opt_aligned(ln_gamma) || !opt_aligned(ln_beta))
    return SQ_ERR_MISALIGNED;
  Ctx ctx;
  if ((st = current_ctx(stream, &ctx)) != SQ_OK) return st;
  const __half* x = static_cast<const __half*>(x_f16);
  if (!ln_gamma) return launched(launch_absmax_cols(x, rows, K, ld, amax_inout, ctx));
  RowArgs a{};
  a.x = x;
  a.rows = rows;
  a.K = K;
  a.ld = ld;
  a.gamma = ln_gamma;
  a.beta = ln_beta;
  a.eps = ln_eps;
  a.amax = amax_inout;
  return launched(launch_calibrate_ln(a, ctx));
}

sq_status sq_smooth_fold(const float* amax_x, const float* amax_w, int64_t K, float alpha,
                         float* s_out, float* inv_s_out, const float* gamma, const float* beta,
                         float* gamma_out, float* beta_out, const void* w_f16, void* w_out_f16,
                         int64_t N, sq_stream_t stream) {
  if (!amax_x || !amax_w || !s_out || !inv_s_out) return SQ_ERR_INVALID_ARG;
  if ((gamma && !gamma_out) || (beta && !beta_out)) return SQ_ERR_INVALID_ARG;
  if (w_f16 && (!w_out_f16 || N <= 0)) return SQ_ERR_INVALID_ARG;
  if (!(alpha >= 0.0f && alpha <= 1.0f)) return SQ_ERR_INVALID_ARG;
  sq_status st = check_k(K);
  if (st != SQ_OK) return st;
  if (!aligned16(amax_x) || !aligned16(amax_w) || !aligned16(s_out) || !aligned16(inv_s_out) ||
      !opt_aligned(gamma) || !opt_aligned(beta) || !opt_aligned(gamma_out) ||
      !opt_aligned(beta_out) || !opt_aligned(w_f16) || !opt_aligned(w_out_f16))
    return SQ_ERR_MISALIGNED;
  Ctx ctx;
  if ((st = current_ctx(stream, &ctx)) != SQ_OK) return st;
  st = launched(launch_smooth(amax_x, amax_w, K, alpha, s_out, inv_s_out, gamma, beta, gamma_out,
                              beta_out, ctx));
  if (st != SQ_OK || !w_f16) return st;
  return launched(launch_fold_weight(static_cast<const __half*>(w_f16),
                                     static_cast<__half*>(w_out_f16), N, K, s_out, ctx));
}

sq_status sq_quantize_weight(const void* w_f16, int64_t N, int64_t K, const float* s, int8_t* wq,
                             float* w_scale, sq_stream_t stream) {
  if (!w_f16 || !wq || !w_scale || N <= 0) return SQ_ERR_INVALID_ARG;
  sq_status st = check_k(K);
  if (st != SQ_OK) return st;
  if (!aligned16(w_f16) || !aligned16(wq) || !aligned16(w_scale) || !opt_aligned(s))
    return SQ_ERR_MISALIGNED;
  Ctx ctx;
  if ((st = current_ctx(stream, &ctx)) != SQ_OK) return st;
  RowArgs a{};
  a.x = static_cast<const __half*>(w_f16);
  a.rows = N;
  a.K = K;
  a.ld = K;
  a.vec = s;
  a.q = wq;
  a.scale = w_scale;
  return launched(launch_quantize_weight(a, ctx));
}

sq_status sq_ln_quant_act(const void* h_f16, int64_t M, int64_t K, int64_t ld, const float* gamma,
                          const float* beta, const float* inv_s, float eps, int8_t* xq,
                          float* x_scale, sq_stream_t stream) {
  if (!h_f16 || !xq || !x_scale || M <= 0) return SQ_ERR_INVALID_ARG;
  if (!gamma && beta) return SQ_ERR_INVALID_ARG;
  sq_status st = check_k(K);
  if (st != SQ_OK) return st;
  if ((st = check_ld(K, ld)) != SQ_OK) return st;
  if (!aligned16(h_f16) || !aligned16(xq) || !aligned16(x_scale) || !opt_aligned(gamma) ||
      !opt_aligned(beta) || !opt_aligned(inv_s))
    return SQ_ERR_MISALIGNED;
  Ctx ctx;
  if ((st = current_ctx(stream, &ctx)) != SQ_OK) return st;
  RowArgs a{};
  a.x = static_cast<const __half*>(h_f16);
  a.rows = M;
  a.K = K;
  a.ld = ld;
  a.gamma = gamma;
  a.beta = beta;
  a.vec = inv_s;
  a.eps = eps;
  a.q = xq;
  a.scale = x_scale;
  return launched(launch_ln_quant_act(a, ctx));
}

sq_status sq_quantize_weight_tensor(const void* w_f16, int64_t N, int64_t K, const float* s,
                                    int8_t* wq, float* w_scale, float* range_out,
                                    sq_stream_t stream) {
  if (!w_f16 || !wq || !w_scale || !range_out || N <= 0) return SQ_ERR_INVALID_ARG;
  sq_status st = check_k(K);
  if (st != SQ_OK) return st;
  if (!aligned16(w_f16) || !aligned16(wq) || !aligned16(w_scale) || !aligned16(range_out) ||
      !opt_aligned(s))
    return SQ_ERR_MISALIGNED;
  Ctx ctx;
  if ((st = current_ctx(stream, &ctx)) != SQ_OK) return st;
  RowArgs a{};
  a.x = static_cast<const __half*>(w_f16);
  a.rows = N;
  a.K = K;
  a.ld = K;
  a.vec = s;
  a.q = wq;
  a.scale = w_scale;
  // pass 1: the range of the (folded) weight; pass 2: codes with one scale
  if (cudaMemsetAsync(range_out, 0, sizeof(float), ctx.stream) != cudaSuccess) return launched(cudaErrorUnknown);
  a.range_out = range_out;
  if ((st = launched(launch_quantize_weight(a, ctx))) != SQ_OK) return st;
  a.range_out = nullptr;
  a.range_in = range_out;
  return launched(launch_quantize_weight(a, ctx));
}


sq_status sq_ln_quant_act_tensor(const void* h_f16, int64_t M, int64_t K, int64_t ld,
                                 const float* gamma, const float* beta, const float* inv_s,
                                 float eps, int8_t* xq, float* x_scale, float* range_out,
                                 sq_stream_t stream) {
  RowArgs a;
  sq_status st = act_args(h_f16, M, K, ld, gamma, beta, inv_s, eps, xq, x_scale, range_out, &a);
  if (st != SQ_OK) return st;
  Ctx ctx;
  if ((st = current_ctx(stream, &ctx)) != SQ_OK) return st;
  if (cudaMemsetAsync(range_out, 0, sizeof(float), ctx.stream) != cudaSuccess) return launched(cudaErrorUnknown);
  a.range_out = range_out;
  if ((st = launched(launch_ln_quant_act(a, ctx))) != SQ_OK) return st;
  a.range_out = nullptr;
  a.range_in = range_out;
  return launched(launch_ln_quant_act(a, ctx));
}

sq_status sq_ln_quant_act_static(const void* h_f16, int64_t M, int64_t K, int64_t ld,
                                 const float* gamma, const float* beta, const float* inv_s,
                                 float eps, const float* range_in, int8_t* xq, float* x_scale,
                                 sq_stream_t stream) {
  RowArgs a;
  sq_status st = act_args(h_f16, M, K, ld, gamma, beta, inv_s, eps, xq, x_scale, range_in, &a);
  if (st != SQ_OK) return st;
  Ctx ctx;
  if ((st = current_ctx(stream, &ctx)) != SQ_OK) return st;
  a.range_in = range_in;
  return launched(launch_ln_quant_act(a, ctx));
}

sq_status sq_row_ranges(const void* x_f16, int64_t rows, int64_t K, int64_t ld, const float* gamma,
                        const float* beta, const float* inv_s, const float* s_fold, float eps,
                        float* range_out, sq_stream_t stream) {
  RowArgs a;
  sq_status st = ranged_args(x_f16, rows, K, ld, gamma, beta, inv_s, s_fold, eps, &a);
  if (st != SQ_OK) return st;
  if (!range_out) return SQ_ERR_INVALID_ARG;
  if (!aligned16(range_out)) return SQ_ERR_MISALIGNED;
  Ctx ctx;
  if ((st = current_ctx(stream, &ctx)) != SQ_OK) return st;
  a.range_out = range_out;
  return launched(s_fold ? launch_quantize_weight(a, ctx) : launch_ln_quant_act(a, ctx));
}

sq_status sq_quantize_rows_ranged(const void* x_f16, int64_t rows, int64_t K, int64_t ld, const float* gamma,
                                  const float* beta, const float* inv_s, const float* s_fold, float eps,
                                  const float* range_in, int8_t* q, float* scale, sq_stream_t stream) {
  RowArgs a;
  sq_status st = ranged_args(x_f16, rows, K, ld, gamma, beta, inv_s, s_fold, eps, &a);
  if (st != SQ_OK) return st;
  if (!range_in || !q || !scale) return SQ_ERR_INVALID_ARG;
  if (!aligned16(range_in) || !aligned16(q) || !aligned16(scale)) return SQ_ERR_MISALIGNED;
  Ctx ctx;
  if ((st = current_ctx(stream, &ctx)) != SQ_OK) return st;
  a.range_in = range_in;
  a.q = q;
  a.scale = scale;
  return launched(s_fold ? launch_quantize_weight(a, ctx) : launch_ln_quant_act(a, ctx));
}

sq_status sq_dequant(const int32_t* acc, const float* x_scale, const float* w_scale, const void* bias_f16,
                     void* y_f16, int64_t M, int64_t N, sq_stream_t stream) {
  if (!acc || !x_scale || !w_scale || !y_f16 || M <= 0 || N <= 0) return SQ_ERR_INVALID_ARG;
  if (N % 4 != 0) return SQ_ERR_UNSUPPORTED_SHAPE;
  if (!aligned16(acc) || !aligned16(x_scale) || !aligned16(w_scale) || !opt_aligned(bias_f16) ||
      !aligned16(y_f16))
    return SQ_ERR_MISALIGNED;
  Ctx ctx;
  sq_status st = current_ctx(stream, &ctx);
  if (st != SQ_OK) return st;
  return launched(launch_dequant(acc, x_scale, w_scale, static_cast<const __half*>(bias_f16),
                                 static_cast<__half*>(y_f16), M, N, ctx));
}

sq_status sq_tensor_range(const float* amax, const float* inv_s, int64_t K, float* range_out,
                          sq_stream_t stream) {
  if (!amax || !range_out || K <= 0) return SQ_ERR_INVALID_ARG;
  if (K > SQ_MAX_K) return SQ_ERR_K_OVERFLOW;
  if (!aligned16(amax) || !aligned16(range_out) || !opt_aligned(inv_s)) return SQ_ERR_MISALIGNED;
  Ctx ctx;
  sq_status st = current_ctx(stream, &ctx);
  if (st != SQ_OK) return st;
  return launched(launch_tensor_range(amax, inv_s, K, range_out, ctx));
}

sq_status sq_w8a8_linear_quant(const int8_t* xq, const float* x_scale, const int8_t* wq,
                               const float* w_scale, const void* bias_f16, int relu,
                               const float* inv_s_next, const float* range_next, int8_t* xq_next,
                               float* x_scale_next, int64_t M, int64_t N, int64_t K, void* workspace,
                               size_t ws_bytes, sq_stream_t stream) {
  if (!xq || !x_scale || !wq || !w_scale || !range_next || !xq_next || !x_scale_next)
    return SQ_ERR_INVALID_ARG;
  if (M <= 0 || N <= 0) return SQ_ERR_INVALID_ARG;
  sq_status st = check_k(K);
  if (st != SQ_OK) return st;
  // the codes are the next linear's input: its K (= N here) follows the same rule
  if (N % 16 != 0 || N > SQ_MAX_K) return SQ_ERR_UNSUPPORTED_SHAPE;
  if (!aligned16(xq) || !aligned16(x_scale) || !aligned16(wq) || !aligned16(w_scale) ||
      !opt_aligned(bias_f16) || !opt_aligned(inv_s_next) || !aligned16(range_next) ||
      !aligned16(xq_next) || !aligned16(x_scale_next))
    return SQ_ERR_MISALIGNED;
  if (M > 0x7fffffffLL) return SQ_ERR_UNSUPPORTED_SHAPE;
  Ctx ctx;
  if ((st = current_ctx(stream, &ctx)) != SQ_OK) return st;
  GemmArgs g{};
  g.xq = xq;
  g.sx = x_scale;
  g.wq = wq;
  g.sw = w_scale;
  g.bias = static_cast<const __half*>(bias_f16);
  g.M = M;
  g.N = N;
  g.K = K;
  g.ws = workspace;
  g.ws_bytes = ws_bytes;
  g.q_next = xq_next;
  g.sx_next = x_scale_next;
  g.inv_s_next = inv_s_next;
  g.range_next = range_next;
  g.relu = relu ? 1 : 0;
  if (M <= SQ_DECODE_MAX_M) {
    const size_t need = splitk_workspace_bytes(M, N, K, ctx.num_sms);
    if (workspace == nullptr || ws_bytes < need || !aligned16(workspace)) return SQ_ERR_WORKSPACE;
    return launched(launch_gemm_splitk(g, ctx));
  }
  return launched(launch_gemm_pair(g, ctx));
}

namespace {

// Workspace of the per-token producer-side quantization: [the stream-K
// scratch for M <= SQ_DECODE_MAX_M] [a fp16 M x N] [row-group maxima fp32 M x part_n],
// each piece 256-byte aligned.
struct DynLayout {
  size_t sk, a_off, part_off, total;
  int64_t part_n;
};

size_t round256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

DynLayout dyn_layout(int64_t M, int64_t N, int64_t K, int num_sms) {
  DynLayout l{};
  const bool decode = M <= SQ_DECODE_MAX_M;
  l.sk = decode ? round256(splitk_workspace_bytes(M, N, K, num_sms)) : 0;
  // one maximum per row and column group: 32 columns (a warp's channels) on the stream-K
  // kernel, 128 (half a 256-column tile) on the CTA-pair kernel
  l.part_n = decode ? (N + 31) / 32 : 2 * ((N + 255) / 256);
  l.a_off = l.sk;
  l.part_off = l.a_off + round256(static_cast<size_t>(M) * static_cast<size_t>(N) * 2);
  l.total = l.part_off + round256(static_cast<size_t>(M) * static_cast<size_t>(l.part_n) * 4);
  return l;
}

int sm_count() {
  int dev = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
    cudaGetLastError();
    sms = 148;
  }
  return sms;
}

}  // namespace

size_t sq_w8a8_linear_quant_dyn_workspace_bytes(int64_t M, int64_t N, int64_t K) {
  if (M <= 0 || N <= 0 || K <= 0 || M > 0x7fffffffLL || N > SQ_MAX_K) return 0;
  return dyn_layout(M, N, K, sm_count()).total;
}

sq_status sq_w8a8_linear_quant_dyn(const int8_t* xq, const float* x_scale, const int8_t* wq,
                                   const float* w_scale, const void* bias_f16, int relu,
                                   const float* inv_s_next, int8_t* xq_next, float* x_scale_next,
                                   int64_t M, int64_t N, int64_t K, void* workspace, size_t ws_bytes,
                                   sq_stream_t stream) {
  if (!xq || !x_scale || !wq || !w_scale || !xq_next || !x_scale_next || !workspace)
    return SQ_ERR_INVALID_ARG;
  if (M <= 0 || N <= 0) return SQ_ERR_INVALID_ARG;
  sq_status st = check_k(K);
  if (st != SQ_OK) return st;
  // the codes are the next linear's input: its K (= N here) follows the same rule
  if (N % 16 != 0 || N > SQ_MAX_K) return SQ_ERR_UNSUPPORTED_SHAPE;
  if (!aligned16(xq) || !aligned16(x_scale) || !aligned16(wq) || !aligned16(w_scale) ||
      !opt_aligned(bias_f16) || !opt_aligned(inv_s_next) || !aligned16(xq_next) ||
      !aligned16(x_scale_next) || !aligned16(workspace))
    return SQ_ERR_MISALIGNED;
  if (M > 0x7fffffffLL) return SQ_ERR_UNSUPPORTED_SHAPE;
  Ctx ctx;
  if ((st = current_ctx(stream, &ctx)) != SQ_OK) return st;
  const DynLayout l = dyn_layout(M, N, K, ctx.num_sms);
  if (ws_bytes < l.total) return SQ_ERR_WORKSPACE;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  GemmArgs g{};
  g.xq = xq;
  g.sx = x_scale;
  g.wq = wq;
  g.sw = w_scale;
  g.bias = static_cast<const __half*>(bias_f16);
  g.y = reinterpret_cast<__half*>(ws + l.a_off);
  g.M = M;
  g.N = N;
  g.K = K;
  g.ws = workspace;
  g.ws_bytes = l.sk;
  g.inv_s_next = inv_s_next;
  g.relu = relu ? 1 : 0;
  g.part = reinterpret_cast<float*>(ws + l.part_off);
  g.part_n = l.part_n;
  cudaError_t e = M <= SQ_DECODE_MAX_M ? launch_gemm_splitk(g, ctx) : launch_gemm_pair(g, ctx);
  if (e != cudaSuccess) return launched(e);
  return launched(launch_quant_partial_rows(g.y, M, N, g.part, g.part_n, inv_s_next, xq_next, x_scale_next, ctx));
}

sq_status sq_w8a8_bmm(const int8_t* a, const float* a_scale, const int8_t* b, const float* b_scale,
                      void* y_f16, int64_t batch, int64_t M, int64_t N, int64_t K, sq_stream_t stream) {
  if (!a || !a_scale || !b || !b_scale || !y_f16) return SQ_ERR_INVALID_ARG;
  if (batch <= 0 || M <= 0 || N <= 0) return SQ_ERR_INVALID_ARG;
  sq_status st = check_k(K);
  if (st != SQ_OK) return st;
  if (!aligned16(a) || !aligned16(a_scale) || !aligned16(b) || !aligned16(b_scale) || !aligned16(y_f16))
    return SQ_ERR_MISALIGNED;
  if (M > 0x7fffffffLL || N > 0x7fffffffLL || batch > 0x7fffffffLL) return SQ_ERR_UNSUPPORTED_SHAPE;
  Ctx ctx;
  if ((st = current_ctx(stream, &ctx)) != SQ_OK) return st;
  GemmArgs g{};
  g.xq = a;
  g.sx = a_scale;
  g.wq = b;
  g.sw = b_scale;
  g.y = static_cast<__half*>(y_f16);
  g.M = M;
  g.N = N;
  g.K = K;
  g.batch = batch;
  return launched(launch_bmm_pair(g, ctx));
}

size_t sq_w8a8_workspace_bytes(int64_t M, int64_t N, int64_t K) {
  if (M <= 0 || N <= 0 || K <= 0 || M > SQ_SPLITK_MAX_M) return 0;
  int dev = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
    cudaGetLastError();
    sms = 148;
  }
  return splitk_workspace_bytes(M, N, K, sms);
}

sq_status sq_w8a8_linear(const int8_t* xq, const float* x_scale, const int8_t* wq,
                         const float* w_scale, const void* bias_f16, void* y_f16, int64_t M,
                         int64_t N, int64_t K, void* workspace, size_t ws_bytes,
                         sq_stream_t stream) {
  return linear_impl(xq, x_scale, wq, w_scale, bias_f16, y_f16, nullptr, M, N, K, workspace,
                     ws_bytes, SQ_PATH_AUTO, stream);
}

sq_status sq_w8a8_linear_path(const int8_t* xq, const float* x_scale, const int8_t* wq,
                              const float* w_scale, const void* bias_f16, void* y_f16, int64_t M,
                              int64_t N, int64_t K, void* workspace, size_t ws_bytes, int path,
                              sq_stream_t stream) {
  return linear_impl(xq, x_scale, wq, w_scale, bias_f16, y_f16, nullptr, M, N, K, workspace,
                     ws_bytes, path, stream);
}

sq_status sq_w8a8_gemm_s32(const int8_t* xq, const int8_t* wq, int32_t* acc, int64_t M, int64_t N,
                           int64_t K, void* workspace, size_t ws_bytes, int path,
                           sq_stream_t stream) {
  if (!acc) return SQ_ERR_INVALID_ARG;
  return linear_impl(xq, nullptr, wq, nullptr, nullptr, nullptr, acc, M, N, K, workspace, ws_bytes,
                     path, stream);
}

sq_status sq_poll_status(sq_stream_t stream) {
  Ctx ctx;
  sq_status st = current_ctx(stream, &ctx);
  if (st != SQ_OK) return st;
  if (cudaStreamSynchronize(ctx.stream) != cudaSuccess) {
    cudaGetLastError();
    return SQ_ERR_CUDA;
  }
  uint32_t v = 0;
  if (cudaMemcpy(&v, ctx.status, sizeof(v), cudaMemcpyDeviceToHost) != cudaSuccess) {
    cudaGetLastError();
    return SQ_ERR_CUDA;
  }
  if (v != 0) {
    const uint32_t zero = 0;
    if (cudaMemcpy(ctx.status, &zero, sizeof(zero), cudaMemcpyHostToDevice) != cudaSuccess) {
      cudaGetLastError();
      return SQ_ERR_CUDA;
    }
    return v == DEV_TIMEOUT ? SQ_ERR_TIMEOUT : SQ_ERR_CUDA;
  }
  return SQ_OK;
}

void sq_set_wait_budget_ns(uint64_t ns) {
  g_budget_ns.store(ns < 1000 ? 1000 : ns, std::memory_order_relaxed);
}

sq_status sq_selftest_wait_timeout(uint64_t budget_ns, sq_stream_t stream) {
  Ctx ctx;
  sq_status st = current_ctx(stream, &ctx);
  if (st != SQ_OK) return st;
  return launched(launch_wait_selftest(budget_ns < 1000 ? 1000 : budget_ns, ctx));
}

}  // extern "C"
