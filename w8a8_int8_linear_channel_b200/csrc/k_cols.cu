// k_cols.cu -- column-wise and elementwise kernels:
//   * per-column absmax of a raw fp16 matrix (calibration of X, and the
//     weight range b_j = max_n |W[n, j]|; glossary "Calibration", section
//     "how is the smoothing factor chosen");
//   * the smoothing factor s_j = a_j^alpha / b_j^(1-alpha), its reciprocal,
//     and the fold into LayerNorm gamma/beta (section "what it does
//     mathematically");
//   * the fold of diag(s) into the fp16 weight.
// All are HBM-bound streams with 16-byte loads; maxima are exact, so the
// cross-CTA merge by integer atomicMax on non-negative floats is
// order-independent.
#include "sq_internal.h"
#include "sq_ptx.cuh"

namespace sq {
namespace {

__device__ __forceinline__ __half2 habs2(__half2 v) {
  const uint32_t b = *reinterpret_cast<uint32_t*>(&v) & 0x7FFF7FFFu;
  return *reinterpret_cast<const __half2*>(&b);
}

__device__ __forceinline__ __half2 as_h2(uint32_t w) { return *reinterpret_cast<__half2*>(&w); }

// Each thread owns one 8-column chunk and walks a strided set of rows; the
// fp16 maxima are exact, merged into amax with atomicMax on the float bits.
__global__ void __launch_bounds__(256) k_absmax_cols(const __half* __restrict__ x, int64_t rows,
                                                     int64_t Kc, int64_t ld,
                                                     float* __restrict__ amax) {
  const int64_t c = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (c >= Kc) return;
  __half2 m0 = __float2half2_rn(0.0f), m1 = m0, m2 = m0, m3 = m0;
  int64_t r = blockIdx.y;
  const int64_t step = gridDim.y;
  for (; r + 3 * step < rows; r += 4 * step) {
    uint4 v[4];
#pragma unroll
    for (int u = 0; u < 4; ++u)
      v[u] = __ldg(reinterpret_cast<const uint4*>(x + (r + u * step) * ld) + c);
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      m0 = __hmax2(m0, habs2(as_h2(v[u].x)));
      m1 = __hmax2(m1, habs2(as_h2(v[u].y)));
      m2 = __hmax2(m2, habs2(as_h2(v[u].z)));
      m3 = __hmax2(m3, habs2(as_h2(v[u].w)));
    }
  }
  for (; r < rows; r += step) {
    const uint4 v = __ldg(reinterpret_cast<const uint4*>(x + r * ld) + c);
    m0 = __hmax2(m0, habs2(as_h2(v.x)));
    m1 = __hmax2(m1, habs2(as_h2(v.y)));
    m2 = __hmax2(m2, habs2(as_h2(v.z)));
    m3 = __hmax2(m3, habs2(as_h2(v.w)));
  }
  int* dst = reinterpret_cast<int*>(amax) + c * 8;
  const __half2 m[4] = {m0, m1, m2, m3};
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    atomicMax(dst + 2 * j, __float_as_int(__low2float(m[j])));
    atomicMax(dst + 2 * j + 1, __float_as_int(__high2float(m[j])));
  }
}

// s_j in fp64 (both maxima floored at 1e-5f), rounded once to fp32.
__global__ void k_smooth(const float* __restrict__ amax_x, const float* __restrict__ amax_w,
                         int64_t K, float alpha, float* __restrict__ s, float* __restrict__ inv_s,
                         const float* gamma, const float* beta, float* gamma_out,
                         float* beta_out) {
  const int64_t j = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (j >= K) return;
  const float ax = amax_x[j], aw = amax_w[j];
  const double x = ax > 1e-5f ? static_cast<double>(ax) : static_cast<double>(1e-5f);
  const double w = aw > 1e-5f ? static_cast<double>(aw) : static_cast<double>(1e-5f);
  const double a = static_cast<double>(alpha);
  const double sj = __ddiv_rn(pow(x, a), pow(w, __dsub_rn(1.0, a)));
  const float s32 = __double2float_rn(sj);
  const float inv = __frcp_rn(s32);
  s[j] = s32;
  inv_s[j] = inv;
  if (gamma) gamma_out[j] = __fmul_rn(gamma[j], inv);
  if (beta) beta_out[j] = __fmul_rn(beta[j], inv);
}

// w_out[n, j] = fp16(fp32(w[n, j]) * s_j), one 8-element chunk per thread and
// iteration (grid-stride).
__global__ void __launch_bounds__(256) k_fold_weight(const __half* __restrict__ w,
                                                     __half* __restrict__ w_out, int64_t total_c,
                                                     int64_t Kc, const float* __restrict__ s) {
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < total_c;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t c = i % Kc;
    uint4 v = __ldg(reinterpret_cast<const uint4*>(w) + i);
    const float4 s0 = __ldg(reinterpret_cast<const float4*>(s + c * 8));
    const float4 s1 = __ldg(reinterpret_cast<const float4*>(s + c * 8 + 4));
    const float sv[8] = {s0.x, s0.y, s0.z, s0.w, s1.x, s1.y, s1.z, s1.w};
    uint32_t* wv = reinterpret_cast<uint32_t*>(&v);
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const __half2 h = as_h2(wv[j]);
      const __half lo = __float2half_rn(__fmul_rn(__low2float(h), sv[2 * j]));
      const __half hi = __float2half_rn(__fmul_rn(__high2float(h), sv[2 * j + 1]));
      const __half2 o = __halves2half2(lo, hi);
      wv[j] = *reinterpret_cast<const uint32_t*>(&o);
    }
    reinterpret_cast<uint4*>(w_out)[i] = v;
  }
}

}  // namespace

cudaError_t launch_absmax_cols(const __half* x, int64_t rows, int64_t K, int64_t ld, float* amax,
                               const Ctx& c) {
  const int64_t Kc = K / 8;
  int threads = static_cast<int>(Kc < 256 ? ((Kc + 31) / 32) * 32 : 256);
  const int64_t gx = (Kc + threads - 1) / threads;
  int64_t gy = (static_cast<int64_t>(c.num_sms) * 2048 + threads * gx - 1) / (threads * gx);
  if (gy > rows) gy = rows;
  if (gy > 65535) gy = 65535;
  if (gy < 1) gy = 1;
  dim3 grid(static_cast<unsigned>(gx), static_cast<unsigned>(gy));
  k_absmax_cols<<<grid, threads, 0, c.stream>>>(x, rows, Kc, ld, amax);
  return cudaGetLastError();
}

cudaError_t launch_smooth(const float* amax_x, const float* amax_w, int64_t K, float alpha,
                          float* s, float* inv_s, const float* gamma, const float* beta,
                          float* gamma_out, float* beta_out, const Ctx& c) {
  const int threads = 256;
  const int64_t blocks = (K + threads - 1) / threads;
  k_smooth<<<static_cast<unsigned>(blocks), threads, 0, c.stream>>>(
      amax_x, amax_w, K, alpha, s, inv_s, gamma, beta, gamma_out, beta_out);
  return cudaGetLastError();
}

cudaError_t launch_fold_weight(const __half* w, __half* w_out, int64_t N, int64_t K,
                               const float* s, const Ctx& c) {
  const int64_t Kc = K / 8;
  const int64_t total = N * Kc;
  int64_t blocks = static_cast<int64_t>(c.num_sms) * 8;
  const int64_t need = (total + 255) / 256;
  if (blocks > need) blocks = need;
  k_fold_weight<<<static_cast<unsigned>(blocks), 256, 0, c.stream>>>(w, w_out, total, Kc, s);
  return cudaGetLastError();
}

}  // namespace sq
