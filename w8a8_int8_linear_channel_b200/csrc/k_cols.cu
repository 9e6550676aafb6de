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

// Column maxima of a row-major fp16 matrix.  A CTA covers 256 columns (32
// chunks of 8) and a band of rows; its 8 warps read 8 rows at a time (each
// warp 512 contiguous bytes per row), 8 independent 16-byte loads in flight
// per thread.  The CTA reduces its 8 row lanes in shared memory and merges
// its 256 maxima with one global atomicMax each (exact: max of non-negative
// floats, ordered as ints); the number of row bands is kept small so each
// column sees only a few dozen atomics.
__global__ void __launch_bounds__(256)
    k_absmax_cols(const __half* __restrict__ x, int64_t rows, int64_t Kc, int64_t ld,
                  int64_t rows_per_cta, float* __restrict__ amax) {
  __shared__ float red[8][257];
  griddep_wait();
  griddep_launch_dependents();
  const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;
  const int64_t c = static_cast<int64_t>(blockIdx.x) * 32 + tx;
  const int64_t r0 = static_cast<int64_t>(blockIdx.y) * rows_per_cta;
  const int64_t r1 = r0 + rows_per_cta < rows ? r0 + rows_per_cta : rows;
  __half2 m0 = __float2half2_rn(0.0f), m1 = m0, m2 = m0, m3 = m0;
  if (c < Kc) {
    const uint4* base = reinterpret_cast<const uint4*>(x) + c;
    const int64_t ldc = ld / 8;  // row stride in 16-byte chunks
    // batches of 8 rows per thread (64 per CTA), all loads of a batch issued
    // before any is used; rows past the band read as zeros
    for (int64_t r = r0 + ty; r < r1; r += 64) {
      uint4 v[8];
#pragma unroll
      for (int u = 0; u < 8; ++u)
        v[u] = (r + 8 * u < r1) ? __ldg(base + (r + 8 * u) * ldc) : make_uint4(0, 0, 0, 0);
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        m0 = __hmax2(m0, habs2(as_h2(v[u].x)));
        m1 = __hmax2(m1, habs2(as_h2(v[u].y)));
        m2 = __hmax2(m2, habs2(as_h2(v[u].z)));
        m3 = __hmax2(m3, habs2(as_h2(v[u].w)));
      }
    }
  }
  const __half2 m[4] = {m0, m1, m2, m3};
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    red[ty][tx * 8 + 2 * j] = __low2float(m[j]);
    red[ty][tx * 8 + 2 * j + 1] = __high2float(m[j]);
  }
  __syncthreads();
  const int col = threadIdx.x;  // 0..255
  const int64_t k = static_cast<int64_t>(blockIdx.x) * 256 + col;
  if (k < Kc * 8) {
    float mm = 0.0f;
#pragma unroll
    for (int y = 0; y < 8; ++y) mm = fmaxf(mm, red[y][col]);
    atomicMax(reinterpret_cast<int*>(amax) + k, __float_as_int(mm));
  }
}

// s_j in fp64 (both maxima floored at 1e-5f), rounded once to fp32.  The
// two powers of a channel are evaluated by a pair of adjacent threads (even:
// a^alpha, odd: b^(1-alpha)) to halve the dependent fp64 latency.
__global__ void k_smooth(const float* __restrict__ amax_x, const float* __restrict__ amax_w,
                         int64_t K, float alpha, float* __restrict__ s, float* __restrict__ inv_s,
                         const float* gamma, const float* beta, float* gamma_out,
                         float* beta_out) {
  griddep_wait();
  griddep_launch_dependents();
  const int64_t t = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  const int64_t j = t >> 1;
  const bool odd = (t & 1) != 0;
  const bool valid = j < K;
  const float av = valid ? (odd ? amax_w[j] : amax_x[j]) : 1.0f;
  // gamma / beta do not depend on the powers: load them now, so their
  // latency overlaps the fp64 work instead of following it
  const bool even_ok = valid && !odd;
  const float gj = (even_ok && gamma) ? gamma[j] : 0.0f;
  const float bj = (even_ok && beta) ? beta[j] : 0.0f;
  const double base = av > 1e-5f ? static_cast<double>(av) : static_cast<double>(1e-5f);
  const double a = static_cast<double>(alpha);
  const double p = pow(base, odd ? __dsub_rn(1.0, a) : a);
  const double den = __shfl_down_sync(0xffffffffu, p, 1);
  if (!even_ok) return;
  const float s32 = __double2float_rn(__ddiv_rn(p, den));
  const float inv = __frcp_rn(s32);
  s[j] = s32;
  inv_s[j] = inv;
  if (gamma) gamma_out[j] = __fmul_rn(gj, inv);
  if (beta) beta_out[j] = __fmul_rn(bj, inv);
}

// w_out[n, j] = fp16(fp32(w[n, j]) * s_j), one 8-element chunk per thread and
// iteration (grid-stride).
__global__ void __launch_bounds__(256) k_fold_weight(const __half* w, __half* w_out,
                                                     int64_t total_c,
                                                     int64_t Kc, const float* __restrict__ s) {
  griddep_wait();
  griddep_launch_dependents();
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < total_c;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t c = i % Kc;
    uint4 v = reinterpret_cast<const uint4*>(w)[i];  // w_out may alias w
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

// The per-tensor range of calibrated per-channel ranges (level O3 of the
// explainer): max_j amax[j], or max_j fp32(amax[j] * inv_s[j]) when the
// runtime multiplies by 1/s.  One CTA (K <= 133144: about 130 values per
// thread).
__global__ void __launch_bounds__(1024) k_tensor_range(const float* __restrict__ amax,
                                                       const float* __restrict__ inv_s, int64_t K,
                                                       float* __restrict__ range) {
  __shared__ float red[32];
  griddep_wait();
  griddep_launch_dependents();
  float m = 0.0f;
  for (int64_t j = threadIdx.x; j < K; j += blockDim.x) {
    const float v = inv_s ? __fmul_rn(amax[j], inv_s[j]) : amax[j];
    m = fmaxf(m, v);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = m;
  __syncthreads();
  if (threadIdx.x < 32) {
    m = threadIdx.x < (blockDim.x >> 5) ? red[threadIdx.x] : 0.0f;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    if (threadIdx.x == 0) range[0] = m;
  }
}

// y[t, n] = fp16(((float)acc[t, n] * sx[t]) * sw[n] + bias[n]): the linear's
// epilogue on its own, for int32 accumulators summed across tensor-parallel
// ranks.  Four outputs per thread and iteration (N % 4 == 0), grid-stride.
__global__ void __launch_bounds__(256) k_dequant(const int32_t* __restrict__ acc, const float* __restrict__ sx,
                                                 const float* __restrict__ sw, const __half* __restrict__ bias,
                                                 __half* __restrict__ y, int64_t M, int64_t N) {
  griddep_wait();
  griddep_launch_dependents();
  const int64_t n4 = N / 4;
  const int64_t total = M * n4;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < total;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t t = i / n4;
    const int64_t n = (i - t * n4) * 4;
    const int4 a = __ldg(reinterpret_cast<const int4*>(acc + t * N + n));
    const float4 w = __ldg(reinterpret_cast<const float4*>(sw + n));
    const float x = sx[t];
    float f[4] = {__fmul_rn(__fmul_rn(__int2float_rn(a.x), x), w.x), __fmul_rn(__fmul_rn(__int2float_rn(a.y), x), w.y),
                  __fmul_rn(__fmul_rn(__int2float_rn(a.z), x), w.z), __fmul_rn(__fmul_rn(__int2float_rn(a.w), x), w.w)};
    if (bias != nullptr) {
#pragma unroll
      for (int j = 0; j < 4; ++j) f[j] = __fadd_rn(f[j], __half2float(bias[n + j]));
    }
    const __half2 lo = __floats2half2_rn(f[0], f[1]);
    const __half2 hi = __floats2half2_rn(f[2], f[3]);
    uint2 o;
    o.x = *reinterpret_cast<const uint32_t*>(&lo);
    o.y = *reinterpret_cast<const uint32_t*>(&hi);
    *reinterpret_cast<uint2*>(y + t * N + n) = o;
  }
}

// The start of a calibration run: every running maximum back to 0.
__global__ void __launch_bounds__(256) k_calib_reset(float* __restrict__ amax, int64_t n) {
  griddep_wait();  // an earlier kernel may still read the previous ranges
  griddep_launch_dependents();
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x)
    amax[i] = 0.0f;
}

}  // namespace

cudaError_t launch_calib_reset(float* amax, int64_t n, const Ctx& c) {
  int64_t blocks = (n + 255) / 256;
  if (blocks > c.num_sms) blocks = c.num_sms;
  return launch_pdl(k_calib_reset, dim3(static_cast<unsigned>(blocks)), dim3(256), 0, c.stream, amax, n);
}

cudaError_t launch_dequant(const int32_t* acc, const float* sx, const float* sw, const __half* bias, __half* y,
                           int64_t M, int64_t N, const Ctx& c) {
  const int64_t total = M * (N / 4);
  int64_t blocks = static_cast<int64_t>(c.num_sms) * 8;
  const int64_t need = (total + 255) / 256;
  if (blocks > need) blocks = need;
  if (blocks < 1) blocks = 1;
  return launch_pdl(k_dequant, dim3(static_cast<unsigned>(blocks)), dim3(256), 0, c.stream, acc, sx, sw, bias, y,
                    M, N);
}

cudaError_t launch_tensor_range(const float* amax, const float* inv_s, int64_t K, float* range,
                                const Ctx& c) {
  return launch_pdl(k_tensor_range, dim3(1), dim3(1024), 0, c.stream, amax, inv_s, K, range);
}

cudaError_t launch_absmax_cols(const __half* x, int64_t rows, int64_t K, int64_t ld, float* amax,
                               const Ctx& c) {
  const int64_t Kc = K / 8;
  const int64_t gx = (Kc + 31) / 32;
  // about three CTAs per SM, at least 128 rows per CTA, at most 64 bands
  int64_t gy = (3 * static_cast<int64_t>(c.num_sms) + gx - 1) / gx;
  const int64_t by_rows = (rows + 127) / 128;
  if (gy > by_rows) gy = by_rows;
  if (gy > 64) gy = 64;
  if (gy < 1) gy = 1;
  const int64_t rows_per_cta = (rows + gy - 1) / gy;
  dim3 grid(static_cast<unsigned>(gx), static_cast<unsigned>(gy));
  return launch_pdl(k_absmax_cols, grid, dim3(256), 0, c.stream, x, rows, Kc, ld, rows_per_cta, amax);
}

cudaError_t launch_smooth(const float* amax_x, const float* amax_w, int64_t K, float alpha,
                          float* s, float* inv_s, const float* gamma, const float* beta,
                          float* gamma_out, float* beta_out, const Ctx& c) {
  const int threads = 64;  // two threads per channel, spread over many SMs
  const int64_t blocks = (2 * K + threads - 1) / threads;
  return launch_pdl(k_smooth, dim3(static_cast<unsigned>(blocks)), dim3(threads), 0, c.stream, amax_x,
                    amax_w, K, alpha, s, inv_s, gamma, beta, gamma_out, beta_out);
}

cudaError_t launch_fold_weight(const __half* w, __half* w_out, int64_t N, int64_t K,
                               const float* s, const Ctx& c) {
  const int64_t Kc = K / 8;
  const int64_t total = N * Kc;
  int64_t blocks = static_cast<int64_t>(c.num_sms) * 8;
  const int64_t need = (total + 255) / 256;
  if (blocks > need) blocks = need;
  return launch_pdl(k_fold_weight, dim3(static_cast<unsigned>(blocks)), dim3(256), 0, c.stream, w, w_out,
                    total, Kc, s);
}

}  // namespace sq
