// k_rows.cu -- row-wise memory-bound kernels of the SmoothQuant W8A8 linear:
//   * LayerNorm (optional) + smoothing (optional) + per-token INT8
//     quantization of the activations (explainer section "inference", O1);
//   * per-output-channel INT8 quantization of the weight, optionally folding
//     diag(s) on the fly (section "what it does mathematically");
//   * calibration absmax of the LayerNorm output (glossary "Calibration").
//
// One CTA of 256 threads owns one row at a time (grid-stride over rows); the
// row is read once from HBM with 16-byte loads and held in registers (8 fp16
// values per chunk, NCH chunks per thread).  Rows too long for registers
// re-read their chunks (the row then sits in L2).  Reductions are warp
// shuffles plus one shared-memory step.
//
// The LayerNorm statistics are exact: every fp16 value h equals v * 2^-24 for
// an integer v (|v| < 2^40); S1 = sum v is kept in int64 and S2 = sum v^2 in
// 128 bits, so the sums -- and hence mu, rstd and every INT8 code -- do not
// depend on the reduction order.
#include "sq_internal.h"
#include "sq_ptx.cuh"

namespace sq {
namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;

enum RowMode { MODE_ACT = 0, MODE_WEIGHT = 1, MODE_CALIB = 2 };

typedef unsigned __int128 u128;

struct RowShared {
  long long s1[kWarps];
  unsigned long long s2_hi[kWarps];
  unsigned long long s2_lo[kWarps];
  float mx[kWarps];
  float mu, rstd, inv;
};

__device__ __forceinline__ void stats_add(uint32_t b, long long& s1, u128& s2) {
  const uint32_t e = (b >> 10) & 31u;
  const uint32_t m = b & 1023u;
  const uint32_t sig = e ? (m | 1024u) : m;
  const uint32_t sh = e ? e - 1u : 0u;
  const unsigned long long mag = static_cast<unsigned long long>(sig) << sh;
  s1 += (b & 0x8000u) ? -static_cast<long long>(mag) : static_cast<long long>(mag);
  s2 += static_cast<u128>(static_cast<unsigned long long>(sig * sig)) << (2u * sh);
}

// mu and rstd from the exact sums, by the fixed sequence of correctly rounded
// fp64 operations documented in sq.h.
__device__ __forceinline__ void ln_finalize(long long s1, u128 s2, int64_t K, float eps,
                                            float& mu, float& rstd) {
  const double two64 = 18446744073709551616.0;
  const double d1 = __ll2double_rn(s1);
  const double d2 = __dadd_rn(
      __dmul_rn(__ull2double_rn(static_cast<unsigned long long>(s2 >> 64)), two64),
      __ull2double_rn(static_cast<unsigned long long>(s2)));
  const double Kd = static_cast<double>(K);
  const double mean = __ddiv_rn(d1, __dmul_rn(Kd, 16777216.0));
  const double ex2 = __ddiv_rn(d2, __dmul_rn(Kd, 281474976710656.0));
  double var = __dsub_rn(ex2, __dmul_rn(mean, mean));
  if (var < 0.0) var = 0.0;
  const double r = __ddiv_rn(1.0, __dsqrt_rn(__dadd_rn(var, static_cast<double>(eps))));
  mu = __double2float_rn(mean);
  rstd = __double2float_rn(r);
}

__device__ __forceinline__ int8_t quant_code(float x, float inv) {
  // cvt.rni: nearest, ties to even; NaN -> 0; saturates, then the symmetric clamp
  int q = __float2int_rn(__fmul_rn(x, inv));
  q = q > 127 ? 127 : q;
  q = q < -127 ? -127 : q;
  return static_cast<int8_t>(q);
}

__device__ __forceinline__ float4 ld_f4(const float* p) {
  return __ldg(reinterpret_cast<const float4*>(p));
}

__device__ __forceinline__ void load8f(const float* p, float (&o)[8]) {
  const float4 a = ld_f4(p), b = ld_f4(p + 4);
  o[0] = a.x; o[1] = a.y; o[2] = a.z; o[3] = a.w;
  o[4] = b.x; o[5] = b.y; o[6] = b.z; o[7] = b.w;
}

__device__ __forceinline__ uint32_t half_bits(const uint4& v, int j) {
  const uint32_t w = (j < 2) ? v.x : (j < 4) ? v.y : (j < 6) ? v.z : v.w;
  return (j & 1) ? (w >> 16) : (w & 0xFFFFu);
}

__device__ __forceinline__ float bits_to_f(uint32_t b) {
  return __half2float(__ushort_as_half(static_cast<unsigned short>(b)));
}

// The 8 transformed fp32 values of chunk c (elements 8c..8c+7) of a row.
template <int MODE>
__device__ __forceinline__ void transform8(const uint4& v, int64_t c, const RowArgs& a, float mu,
                                           float rstd, float (&x)[8]) {
#pragma unroll
  for (int j = 0; j < 8; ++j) x[j] = bits_to_f(half_bits(v, j));
  const int64_t k0 = c * 8;
  if (MODE == MODE_WEIGHT) {
    if (a.vec) {
      float s[8];
      load8f(a.vec + k0, s);
#pragma unroll
      for (int j = 0; j < 8; ++j) x[j] = __half2float(__float2half_rn(__fmul_rn(x[j], s[j])));
    }
    return;
  }
  if (a.gamma) {
    float g[8];
    load8f(a.gamma + k0, g);
#pragma unroll
    for (int j = 0; j < 8; ++j) x[j] = __fmul_rn(__fmul_rn(__fsub_rn(x[j], mu), rstd), g[j]);
    if (a.beta) {
      float b[8];
      load8f(a.beta + k0, b);
#pragma unroll
      for (int j = 0; j < 8; ++j) x[j] = __fadd_rn(x[j], b[j]);
    }
  }
  if (MODE == MODE_ACT && a.vec) {
    float is[8];
    load8f(a.vec + k0, is);
#pragma unroll
    for (int j = 0; j < 8; ++j) x[j] = __fmul_rn(x[j], is[j]);
  }
}

// NCH > 0: the thread's chunks of the row live in registers.
// NCH == 0: chunks are re-read from global memory in every pass.
template <int MODE, int NCH>
__global__ void __launch_bounds__(kThreads) k_rows(const RowArgs a) {
  constexpr bool REG = NCH > 0;
  __shared__ RowShared sh;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int64_t Kc = a.K / 8;
  const int nch = REG ? NCH : static_cast<int>((Kc + kThreads - 1) / kThreads);
  const bool use_ln = (MODE != MODE_WEIGHT) && a.gamma != nullptr;

  // calibration: running column maxima of this thread's chunks
  constexpr bool CALIB_REG = (MODE == MODE_CALIB) && REG && NCH <= 8;
  float cmax[CALIB_REG ? NCH * 8 : 1];
  if (CALIB_REG) {
#pragma unroll
    for (int i = 0; i < (CALIB_REG ? NCH * 8 : 1); ++i) cmax[i] = 0.0f;
  }

  uint4 v[REG ? NCH : 1];
  for (int64_t r = blockIdx.x; r < a.rows; r += gridDim.x) {
    const uint4* src = reinterpret_cast<const uint4*>(a.x + r * a.ld);
    if (REG) {
#pragma unroll
      for (int i = 0; i < (REG ? NCH : 1); ++i) {
        const int64_t c = tid + static_cast<int64_t>(i) * kThreads;
        v[i] = c < Kc ? __ldg(src + c) : make_uint4(0, 0, 0, 0);
      }
    }
    auto chunk = [&](int i, int64_t c) -> uint4 {
      if constexpr (REG) return v[i];
      else return __ldg(src + c);
    };

    float mu = 0.0f, rstd = 0.0f;
    if (use_ln) {
      long long s1 = 0;
      u128 s2 = 0;
#pragma unroll
      for (int i = 0; i < (REG ? NCH : 1); ++i) {
        const int iters = REG ? 1 : nch;
        for (int ii = 0; ii < iters; ++ii) {
          const int ci = REG ? i : ii;
          const int64_t c = tid + static_cast<int64_t>(ci) * kThreads;
          if (c < Kc) {
            const uint4 q = chunk(ci, c);
#pragma unroll
            for (int j = 0; j < 8; ++j) stats_add(half_bits(q, j), s1, s2);
          }
        }
      }
      unsigned long long hi = static_cast<unsigned long long>(s2 >> 64);
      unsigned long long lo = static_cast<unsigned long long>(s2);
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        const long long t1 = __shfl_xor_sync(0xffffffffu, s1, o);
        const unsigned long long th = __shfl_xor_sync(0xffffffffu, hi, o);
        const unsigned long long tl = __shfl_xor_sync(0xffffffffu, lo, o);
        s1 += t1;
        const u128 sum = ((static_cast<u128>(hi) << 64) | lo) + ((static_cast<u128>(th) << 64) | tl);
        hi = static_cast<unsigned long long>(sum >> 64);
        lo = static_cast<unsigned long long>(sum);
      }
      if (lane == 0) {
        sh.s1[warp] = s1;
        sh.s2_hi[warp] = hi;
        sh.s2_lo[warp] = lo;
      }
      __syncthreads();
      if (tid == 0) {
        long long t1 = 0;
        u128 t2 = 0;
        for (int w = 0; w < kWarps; ++w) {
          t1 += sh.s1[w];
          t2 += (static_cast<u128>(sh.s2_hi[w]) << 64) | sh.s2_lo[w];
        }
        float m_, r_;
        ln_finalize(t1, t2, a.K, a.eps, m_, r_);
        sh.mu = m_;
        sh.rstd = r_;
      }
      __syncthreads();
      mu = sh.mu;
      rstd = sh.rstd;
    }

    if (MODE == MODE_CALIB) {
#pragma unroll
      for (int i = 0; i < (REG ? NCH : 1); ++i) {
        const int iters = REG ? 1 : nch;
        for (int ii = 0; ii < iters; ++ii) {
          const int ci = REG ? i : ii;
          const int64_t c = tid + static_cast<int64_t>(ci) * kThreads;
          if (c < Kc) {
            float x[8];
            transform8<MODE>(chunk(ci, c), c, a, mu, rstd, x);
#pragma unroll
            for (int j = 0; j < 8; ++j) {
              const float ax = fabsf(x[j]);
              if constexpr (CALIB_REG) {
                cmax[ci * 8 + j] = fmaxf(cmax[ci * 8 + j], ax);
              } else {
                atomicMax(reinterpret_cast<int*>(a.amax) + c * 8 + j, __float_as_int(ax));
              }
            }
          }
        }
      }
      continue;
    }

    // row absmax of the transformed values
    float amax = 0.0f;
#pragma unroll
    for (int i = 0; i < (REG ? NCH : 1); ++i) {
      const int iters = REG ? 1 : nch;
      for (int ii = 0; ii < iters; ++ii) {
        const int ci = REG ? i : ii;
        const int64_t c = tid + static_cast<int64_t>(ci) * kThreads;
        if (c < Kc) {
          float x[8];
          transform8<MODE>(chunk(ci, c), c, a, mu, rstd, x);
#pragma unroll
          for (int j = 0; j < 8; ++j) amax = fmaxf(amax, fabsf(x[j]));
        }
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
    if (lane == 0) sh.mx[warp] = amax;
    __syncthreads();
    if (tid == 0) {
      float m = 0.0f;
      for (int w = 0; w < kWarps; ++w) m = fmaxf(m, sh.mx[w]);
      const float sc = __fdiv_rn(m, 127.0f);
      sh.inv = sc > 0.0f ? __frcp_rn(sc) : 0.0f;
      a.scale[r] = sc;
    }
    __syncthreads();
    const float inv = sh.inv;

    // quantize and store 8 codes (8 bytes) per chunk
    int8_t* dst = a.q + r * a.K;
#pragma unroll
    for (int i = 0; i < (REG ? NCH : 1); ++i) {
      const int iters = REG ? 1 : nch;
      for (int ii = 0; ii < iters; ++ii) {
        const int ci = REG ? i : ii;
        const int64_t c = tid + static_cast<int64_t>(ci) * kThreads;
        if (c < Kc) {
          float x[8];
          transform8<MODE>(chunk(ci, c), c, a, mu, rstd, x);
          uint32_t w0 = 0, w1 = 0;
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            w0 |= (static_cast<uint32_t>(static_cast<uint8_t>(quant_code(x[j], inv)))) << (8 * j);
            w1 |= (static_cast<uint32_t>(static_cast<uint8_t>(quant_code(x[j + 4], inv)))) << (8 * j);
          }
          *reinterpret_cast<uint2*>(dst + c * 8) = make_uint2(w0, w1);
        }
      }
    }
  }

  if constexpr (CALIB_REG) {
#pragma unroll
    for (int i = 0; i < (CALIB_REG ? NCH : 1); ++i) {
      const int64_t c = tid + static_cast<int64_t>(i) * kThreads;
      if (c < Kc) {
#pragma unroll
        for (int j = 0; j < 8; ++j)
          atomicMax(reinterpret_cast<int*>(a.amax) + c * 8 + j, __float_as_int(cmax[i * 8 + j]));
      }
    }
  }
}

template <int MODE, int NCH>
cudaError_t launch_nch(const RowArgs& a, const Ctx& c) {
  static int occ[64] = {0};  // CTAs per SM, per device
  int dev = c.device < 64 ? c.device : 63;
  if (occ[dev] == 0) {
    int n = 0;
    cudaError_t e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, k_rows<MODE, NCH>, kThreads, 0);
    if (e != cudaSuccess) return e;
    occ[dev] = n > 0 ? n : 1;
  }
  int64_t grid = static_cast<int64_t>(c.num_sms) * occ[dev];
  if (grid > a.rows) grid = a.rows;
  k_rows<MODE, NCH><<<static_cast<unsigned>(grid), kThreads, 0, c.stream>>>(a);
  return cudaGetLastError();
}

template <int MODE>
cudaError_t launch_mode(const RowArgs& a, const Ctx& c) {
  const int64_t per_thread = (a.K / 8 + kThreads - 1) / kThreads;  // chunks per thread
  if (per_thread <= 1) return launch_nch<MODE, 1>(a, c);
  if (per_thread <= 2) return launch_nch<MODE, 2>(a, c);
  if (per_thread <= 4) return launch_nch<MODE, 4>(a, c);
  if (per_thread <= 6) return launch_nch<MODE, 6>(a, c);
  if (per_thread <= 8) return launch_nch<MODE, 8>(a, c);
  if (per_thread <= 12) return launch_nch<MODE, 12>(a, c);
  if (per_thread <= 24) return launch_nch<MODE, 24>(a, c);
  return launch_nch<MODE, 0>(a, c);
}

}  // namespace

cudaError_t launch_ln_quant_act(const RowArgs& a, const Ctx& c) { return launch_mode<MODE_ACT>(a, c); }

cudaError_t launch_quantize_weight(const RowArgs& a, const Ctx& c) {
  return launch_mode<MODE_WEIGHT>(a, c);
}

cudaError_t launch_calibrate_ln(const RowArgs& a, const Ctx& c) {
  return launch_mode<MODE_CALIB>(a, c);
}

}  // namespace sq
