// k_rows.cu -- row-wise memory-bound kernels of the SmoothQuant W8A8 linear:
//   * LayerNorm (optional) + smoothing (optional) + per-token INT8
//     quantization of the activations (explainer section "inference", O1);
//   * per-output-channel INT8 quantization of the weight, optionally folding
//     diag(s) on the fly (section "what it does mathematically");
//   * calibration absmax of the LayerNorm output (glossary "Calibration").
//
// Shapes of the same computation (chosen by K):
//   * K <= 1024: one warp per row (no block barrier at all; many rows in
//     flight per SM).  The row and its transformed values live in registers.
//   * K <= 16384: one CTA of 64 to 256 threads per row, up to 8 16-byte
//     chunks per thread held in registers (converted to fp32 once), the
//     CTA's next row prefetched; warp shuffles plus one shared-memory step
//     per reduction.
//   * larger K: the same CTA shape with 12 or 24 chunks per thread in
//     registers, or (K > 49152) the row re-read from global in every pass.
// Rows are read once from HBM with 16-byte loads (except the last shape).
// A row maximum is taken NaN-propagating; a row whose maximum is not finite
// (it holds a NaN or an Inf) recomputes its NaN-free maximum and quantizes
// through the NaN-safe path.
//
// LayerNorm statistics are exact and order-independent: every fp16 value h
// equals v * 2^-24 for an integer v (|v| < 2^40).  Per 8-element chunk the
// sums of h and of h^2 are formed exactly in fp64 (h^2 has a 22-bit
// significand; it is split exactly into a multiple of 2^-13 and a remainder
// below 2^-13 so both partial sums stay within 53 bits), then converted to
// int64 in units of 2^-24 (S1) and 2^-13 / 2^-48 (S2), and summed as
// integers.  S1 = sum v and S2 = sum v^2 are therefore the exact integers,
// whatever the reduction order.
//
// Calibration merges its per-column maxima across a cluster of 8 CTAs
// through distributed shared memory, so each column receives one global
// atomicMax per cluster instead of one per CTA.
#include <cooperative_groups.h>

#include <type_traits>

#include "sq_internal.h"
#include "sq_ptx.cuh"

namespace cg = cooperative_groups;

namespace sq {
namespace {

constexpr int kCtaThreads = 256;
constexpr int kWarpThreads = 128;  // 4 row-warps per CTA in the warp-per-row kernels
constexpr int kCluster = 8;

enum RowMode { MODE_ACT = 0, MODE_WEIGHT = 1, MODE_CALIB = 2 };

typedef unsigned __int128 u128;

// ------------------------------------------------------- exact LN sums ---
struct Sums {
  long long s1;   // sum v            (units 2^-24 of h)
  long long s2h;  // sum of h^2 parts that are multiples of 2^-13, in units 2^-13
  long long s2l;  // sum of the remainders below 2^-13, in units 2^-48
  int bad;        // the row holds an Inf or a NaN (its statistics are NaN)
};

__device__ __forceinline__ uint32_t half_bits(const uint4& v, int j) {
  const uint32_t w = (j < 2) ? v.x : (j < 4) ? v.y : (j < 6) ? v.z : v.w;
  return (j & 1) ? (w >> 16) : (w & 0xFFFFu);
}

// fp16 bit pattern (low 16 bits of b) -> fp64, exact.
__device__ __forceinline__ double half_to_f64(uint32_t b) {
  double d;
  asm("cvt.f64.f16 %0, %1;" : "=d"(d) : "h"(static_cast<unsigned short>(b)));
  return d;
}

__device__ __forceinline__ float bits_to_f(uint32_t b) {
  return __half2float(__ushort_as_half(static_cast<unsigned short>(b)));
}

__device__ __forceinline__ void chunk_sums(const uint4& v, Sums& s) {
  const double kSplit = 824633720832.0;  // 1.5 * 2^39: (t + kSplit) - kSplit rounds t to 2^-13
  double c1 = 0.0, c2h = 0.0, c2l = 0.0;
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    const double d = static_cast<double>(bits_to_f(half_bits(v, j)));
    c1 = __dadd_rn(c1, d);
    const double t = __dmul_rn(d, d);
    const double th = __dsub_rn(__dadd_rn(t, kSplit), kSplit);
    c2h = __dadd_rn(c2h, th);
    c2l = __dadd_rn(c2l, __dsub_rn(t, th));
  }
  s.s1 += __double2ll_rn(__dmul_rn(c1, 16777216.0));            // * 2^24
  s.s2h += __double2ll_rn(__dmul_rn(c2h, 8192.0));              // * 2^13
  s.s2l += __double2ll_rn(__dmul_rn(c2l, 281474976710656.0));   // * 2^48
  // eight finite fp16 values sum to a finite double; an Inf or a NaN among
  // them leaves c1 infinite or NaN
  s.bad |= !(fabs(c1) <= 1.7976931348623157e308);
}

// Same sums from the 8 values already converted to fp32 (exact conversions).
__device__ __forceinline__ void chunk_sums_f(const float (&x)[8], Sums& s) {
  const double kSplit = 824633720832.0;  // 1.5 * 2^39: (t + kSplit) - kSplit rounds t to 2^-13
  double c1 = 0.0, c2h = 0.0, c2l = 0.0;
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    const double d = static_cast<double>(x[j]);
    c1 = __dadd_rn(c1, d);
    const double t = __dmul_rn(d, d);
    const double th = __dsub_rn(__dadd_rn(t, kSplit), kSplit);
    c2h = __dadd_rn(c2h, th);
    c2l = __dadd_rn(c2l, __dsub_rn(t, th));
  }
  s.s1 += __double2ll_rn(__dmul_rn(c1, 16777216.0));            // * 2^24
  s.s2h += __double2ll_rn(__dmul_rn(c2h, 8192.0));              // * 2^13
  s.s2l += __double2ll_rn(__dmul_rn(c2l, 281474976710656.0));   // * 2^48
  s.bad |= !(fabs(c1) <= 1.7976931348623157e308);
}

__device__ __forceinline__ void warp_sum(Sums& s) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    s.s1 += __shfl_xor_sync(0xffffffffu, s.s1, o);
    s.s2h += __shfl_xor_sync(0xffffffffu, s.s2h, o);
    s.s2l += __shfl_xor_sync(0xffffffffu, s.s2l, o);
  }
  s.bad = __any_sync(0xffffffffu, s.bad);
}

// mu and rstd from the exact sums S1 = s1 and S2 = s2h * 2^35 + s2l, by the
// fixed sequence of correctly rounded fp64 operations documented in sq.h.
// k_log2 >= 0 when K is a power of two: the divisions by K * 2^24 and K * 2^48
// are then exact scalings, done as multiplications by the (exact) reciprocal
// power of two -- the same correctly rounded results, without the division
// sequences.
__device__ __forceinline__ void ln_finalize(const Sums& s, int64_t K, float eps, float& mu,
                                            float& rstd, int k_log2 = -1) {
  if (s.bad) {  // a row with an Inf or a NaN: NaN statistics
    mu = __int_as_float(0x7fc00000);
    rstd = mu;
    return;
  }
  const u128 S2 = (static_cast<u128>(static_cast<unsigned long long>(s.s2h)) << 35) +
                  static_cast<u128>(static_cast<__int128>(s.s2l));
  const double two64 = 18446744073709551616.0;
  const double d1 = __ll2double_rn(s.s1);
  const double d2 = __dadd_rn(
      __dmul_rn(__ull2double_rn(static_cast<unsigned long long>(S2 >> 64)), two64),
      __ull2double_rn(static_cast<unsigned long long>(S2)));
  const double Kd = static_cast<double>(K);
  double mean, ex2;
  if (k_log2 >= 0) {
    const double r1 = __longlong_as_double(static_cast<long long>(1023 - 24 - k_log2) << 52);  // 2^-(24+log2 K)
    const double r2 = __longlong_as_double(static_cast<long long>(1023 - 48 - k_log2) << 52);  // 2^-(48+log2 K)
    mean = __dmul_rn(d1, r1);
    ex2 = __dmul_rn(d2, r2);
  } else {
    mean = __ddiv_rn(d1, __dmul_rn(Kd, 16777216.0));
    ex2 = __ddiv_rn(d2, __dmul_rn(Kd, 281474976710656.0));
  }
  double var = __dsub_rn(ex2, __dmul_rn(mean, mean));
  if (var < 0.0) var = 0.0;
  const double r = __ddiv_rn(1.0, __dsqrt_rn(__dadd_rn(var, static_cast<double>(eps))));
  mu = __double2float_rn(mean);
  rstd = __double2float_rn(r);
}

// ------------------------------------------------------- element math ---
__device__ __forceinline__ void load8f(const float* p, float (&o)[8]) {
  const float4 a = __ldg(reinterpret_cast<const float4*>(p));
  const float4 b = __ldg(reinterpret_cast<const float4*>(p) + 1);
  o[0] = a.x; o[1] = a.y; o[2] = a.z; o[3] = a.w;
  o[4] = b.x; o[5] = b.y; o[6] = b.z; o[7] = b.w;
}

// The 8 transformed fp32 values of chunk c (elements 8c..8c+7) of a row.
__device__ __forceinline__ void unpack8(const uint4& v, float (&x)[8]) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&w[j]));
    x[2 * j] = f.x;
    x[2 * j + 1] = f.y;
  }
}

template <int MODE>
__device__ __forceinline__ void transform8(const uint4& v, int64_t c, const RowArgs& a, float mu,
                                           float rstd, float (&x)[8]) {
  unpack8(v, x);
  const int64_t k0 = c * 8;
  if (MODE == MODE_WEIGHT) {
    if (a.vec) {
      float s[8];
      load8f(a.vec + k0, s);
#pragma unroll
      for (int j = 0; j < 8; j += 2) {
        // fold diag(s) and round once to fp16, two lanes per instruction
        const float2 f = __half22float2(__floats2half2_rn(__fmul_rn(x[j], s[j]), __fmul_rn(x[j + 1], s[j + 1])));
        x[j] = f.x;
        x[j + 1] = f.y;
      }
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

// Eight codes packed into 8 bytes.  p = x * inv (rounded), then
// p + 1.5 * 2^23 rounds p to the nearest integer, ties to even, and leaves
// that integer in the low mantissa bits: the low byte of the sum is the
// two's-complement code (code_bits maps a NaN sum to byte 0).  No clamp is needed:
// inv = RN(1 / RN(amax / 127)) and |x| <= amax bound |p| by 127 (1 + 3 * 2^-24)
// < 127.5, so the rounded value is already inside [-127, 127] -- the same
// codes as clamp(rint(p), -127, 127).
// SAFE: a NaN sum (any NaN bit pattern) is mapped by an unsigned min onto
// 1.5 * 2^23 + 256, whose low byte is 0, while every in-range sum
// (0x4B3FFF81 .. 0x4B40007F) is below it.  Rows whose range is finite have
// no NaN product and skip it.
template <bool SAFE>
__device__ __forceinline__ uint32_t code_bits(float p) {
  const float kMagic = 12582912.0f;  // 1.5 * 2^23
  const uint32_t b = __float_as_uint(__fadd_rn(p, kMagic));
  return SAFE ? min(b, 0x4B400100u) : b;
}

template <bool SAFE>
__device__ __forceinline__ uint32_t quant4(float x0, float x1, float x2, float x3, float inv) {
  const uint32_t b0 = code_bits<SAFE>(__fmul_rn(x0, inv));
  const uint32_t b1 = code_bits<SAFE>(__fmul_rn(x1, inv));
  const uint32_t b2 = code_bits<SAFE>(__fmul_rn(x2, inv));
  const uint32_t b3 = code_bits<SAFE>(__fmul_rn(x3, inv));
  return __byte_perm(__byte_perm(b0, b1, 0x0040), __byte_perm(b2, b3, 0x0040), 0x5410);
}

// transform8 on values already unpacked to fp32, in place.
template <int MODE>
__device__ __forceinline__ void transform8f(float (&x)[8], int64_t c, const RowArgs& a, float mu,
                                            float rstd) {
  const int64_t k0 = c * 8;
  if (MODE == MODE_WEIGHT) {
    if (a.vec) {
      float s[8];
      load8f(a.vec + k0, s);
#pragma unroll
      for (int j = 0; j < 8; j += 2) {
        const float2 f = __half22float2(__floats2half2_rn(__fmul_rn(x[j], s[j]), __fmul_rn(x[j + 1], s[j + 1])));
        x[j] = f.x;
        x[j + 1] = f.y;
      }
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

template <bool SAFE = false>
__device__ __forceinline__ uint2 pack8(const float (&x)[8], float inv) {
  return make_uint2(quant4<SAFE>(x[0], x[1], x[2], x[3], inv), quant4<SAFE>(x[4], x[5], x[6], x[7], inv));
}

// max(a, |b|) for a >= 0 (or NaN), propagating a NaN.  A row maximum taken
// with it is finite exactly when the row holds no NaN and no Inf.
__device__ __forceinline__ float absmax_nan(float a, float b) {
  float d;
  asm("max.NaN.f32 %0, %1, %2;" : "=f"(d) : "f"(a), "f"(fabsf(b)));
  return d;
}

__device__ __forceinline__ bool finite_f(float m) { return fabsf(m) <= 3.402823466e38f; }

// The same codes for a scale fixed in advance (per-tensor levels): x * inv
// may now leave [-127, 127], so it is clamped first (a NaN product passes
// the clamp unchanged and still gives byte 0 as above).
__device__ __forceinline__ float clamp127(float p) {
  p = p > 127.0f ? 127.0f : p;
  return p < -127.0f ? -127.0f : p;
}

__device__ __forceinline__ uint32_t quant4c(float x0, float x1, float x2, float x3, float inv) {
  const uint32_t b0 = code_bits<true>(clamp127(__fmul_rn(x0, inv)));
  const uint32_t b1 = code_bits<true>(clamp127(__fmul_rn(x1, inv)));
  const uint32_t b2 = code_bits<true>(clamp127(__fmul_rn(x2, inv)));
  const uint32_t b3 = code_bits<true>(clamp127(__fmul_rn(x3, inv)));
  return __byte_perm(__byte_perm(b0, b1, 0x0040), __byte_perm(b2, b3, 0x0040), 0x5410);
}

__device__ __forceinline__ uint2 pack8c(const float (&x)[8], float inv) {
  return make_uint2(quant4c(x[0], x[1], x[2], x[3], inv), quant4c(x[4], x[5], x[6], x[7], inv));
}

// Scale and reciprocal of a given range (same op order as per row): one
// range for the tensor, or one per row (range_per_row).
__device__ __forceinline__ void range_scale(const RowArgs& a, int64_t r, float& sc, float& inv) {
  sc = __fdiv_rn(a.range_per_row ? a.range_in[r] : *a.range_in, 127.0f);
  inv = sc > 0.0f ? __frcp_rn(sc) : 0.0f;
}

// Range pass: a row's max goes to its own slot (range_per_row) or is merged
// into the tensor's range (exact and order-free: non-negative floats order
// as their bit patterns).
__device__ __forceinline__ void range_merge(const RowArgs& a, int64_t r, float m) {
  if (a.range_per_row) a.range_out[r] = m;
  else atomicMax(reinterpret_cast<int*>(a.range_out), __float_as_int(m));
}

// =========================================================================
// Warp per row (K <= 32 * 8 * NW).
// =========================================================================
template <int MODE, int NW>
__global__ void __launch_bounds__(kWarpThreads) k_rows_warp(const RowArgs a) {
  griddep_wait();
  griddep_launch_dependents();
  const int lane = threadIdx.x & 31;
  const int64_t wid = (static_cast<int64_t>(blockIdx.x) * kWarpThreads + threadIdx.x) >> 5;
  const int64_t nwarps = (static_cast<int64_t>(gridDim.x) * kWarpThreads) >> 5;
  const int64_t Kc = a.K >> 3;
  const bool use_ln = (MODE == MODE_ACT) && a.gamma != nullptr;
  for (int64_t r = wid; r < a.rows; r += nwarps) {
    const uint4* src = reinterpret_cast<const uint4*>(a.x + r * a.ld);
    uint4 v[NW];
#pragma unroll
    for (int i = 0; i < NW; ++i) {
      const int64_t c = lane + 32 * i;
      v[i] = c < Kc ? ld_stream(src + c) : make_uint4(0, 0, 0, 0);
    }
    float mu = 0.0f, rstd = 0.0f;
    if (use_ln) {
      Sums s{0, 0, 0, 0};
#pragma unroll
      for (int i = 0; i < NW; ++i)
        if (lane + 32 * i < Kc) chunk_sums(v[i], s);
      warp_sum(s);
      ln_finalize(s, a.K, a.eps, mu, rstd);
    }
    float x[NW][8];
    float amax = 0.0f;
#pragma unroll
    for (int i = 0; i < NW; ++i) {
      const int64_t c = lane + 32 * i;
      if (c < Kc) {
        transform8<MODE>(v[i], c, a, mu, rstd, x[i]);
#pragma unroll
        for (int j = 0; j < 8; ++j) amax = absmax_nan(amax, x[i][j]);
      }
    }
    int8_t* dst = a.q + r * a.K;
    if (a.range_in) {  // per-tensor scale fixed in advance: no row max
      float sc, inv;
      range_scale(a, r, sc, inv);
      if (lane == 0) a.scale[r] = sc;
#pragma unroll
      for (int i = 0; i < NW; ++i) {
        const int64_t c = lane + 32 * i;
        if (c < Kc) *reinterpret_cast<uint2*>(dst + c * 8) = pack8c(x[i], inv);
      }
      continue;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) amax = absmax_nan(amax, __shfl_xor_sync(0xffffffffu, amax, o));
    const bool safe = !finite_f(amax);  // warp-uniform
    if (safe) {  // a NaN or an Inf in the row: the range ignores NaN
      amax = 0.0f;
#pragma unroll
      for (int i = 0; i < NW; ++i)
        if (lane + 32 * i < Kc)
#pragma unroll
          for (int j = 0; j < 8; ++j) amax = fmaxf(amax, fabsf(x[i][j]));
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
    }
    amax = fabsf(amax);
    if (a.range_out) {  // range pass only
      if (lane == 0) range_merge(a, r, amax);
      continue;
    }
    const float sc = __fdiv_rn(amax, 127.0f);
    const float inv = sc > 0.0f ? __frcp_rn(sc) : 0.0f;
    if (lane == 0) a.scale[r] = sc;
    auto store = [&](auto safe_t) {
#pragma unroll
      for (int i = 0; i < NW; ++i) {
        const int64_t c = lane + 32 * i;
        if (c < Kc) *reinterpret_cast<uint2*>(dst + c * 8) = pack8<decltype(safe_t)::value>(x[i], inv);
      }
    };
    if (safe) store(std::true_type{});
    else store(std::false_type{});
  }
}

// LayerNorm calibration, warp per row: per-lane running maxima of the
// lane's columns in registers, merged per CTA in shared memory and across
// the cluster of 8 CTAs through distributed shared memory.
template <int NW>
__global__ void __cluster_dims__(kCluster, 1, 1) __launch_bounds__(kWarpThreads)
    k_calib_warp(const RowArgs a) {
  extern __shared__ int colmax_s[];  // K float bits (non-negative floats order as ints)
  cg::cluster_group cluster = cg::this_cluster();
  const int lane = threadIdx.x & 31;
  const int64_t Kc = a.K >> 3;
  for (int64_t j = threadIdx.x; j < a.K; j += kWarpThreads) colmax_s[j] = 0;
  __syncthreads();
  griddep_wait();
  griddep_launch_dependents();

  float cm[NW][8];
#pragma unroll
  for (int i = 0; i < NW; ++i)
#pragma unroll
    for (int j = 0; j < 8; ++j) cm[i][j] = 0.0f;

  const int64_t wid = (static_cast<int64_t>(blockIdx.x) * kWarpThreads + threadIdx.x) >> 5;
  const int64_t nwarps = (static_cast<int64_t>(gridDim.x) * kWarpThreads) >> 5;
  for (int64_t r = wid; r < a.rows; r += nwarps) {
    const uint4* src = reinterpret_cast<const uint4*>(a.x + r * a.ld);
    uint4 v[NW];
#pragma unroll
    for (int i = 0; i < NW; ++i) {
      const int64_t c = lane + 32 * i;
      v[i] = c < Kc ? ld_stream(src + c) : make_uint4(0, 0, 0, 0);
    }
    Sums s{0, 0, 0, 0};
#pragma unroll
    for (int i = 0; i < NW; ++i)
      if (lane + 32 * i < Kc) chunk_sums(v[i], s);
    warp_sum(s);
    float mu, rstd;
    ln_finalize(s, a.K, a.eps, mu, rstd);
#pragma unroll
    for (int i = 0; i < NW; ++i) {
      const int64_t c = lane + 32 * i;
      if (c < Kc) {
        float x[8];
        transform8<MODE_CALIB>(v[i], c, a, mu, rstd, x);
#pragma unroll
        for (int j = 0; j < 8; ++j) cm[i][j] = fmaxf(cm[i][j], fabsf(x[j]));
      }
    }
  }
#pragma unroll
  for (int i = 0; i < NW; ++i) {
    const int64_t c = lane + 32 * i;
    if (c < Kc)
#pragma unroll
      for (int j = 0; j < 8; ++j) atomicMax(colmax_s + c * 8 + j, __float_as_int(cm[i][j]));
  }
  __syncthreads();
  cluster.sync();
  const int64_t slice = (a.K + kCluster - 1) / kCluster;
  const int64_t j0 = static_cast<int64_t>(cluster.block_rank()) * slice;
  const int64_t j1 = j0 + slice < a.K ? j0 + slice : a.K;
  for (int64_t j = j0 + threadIdx.x; j < j1; j += kWarpThreads) {
    int m = 0;
#pragma unroll
    for (int q = 0; q < kCluster; ++q) m = max(m, cluster.map_shared_rank(colmax_s, q)[j]);
    atomicMax(reinterpret_cast<int*>(a.amax) + j, m);
  }
  cluster.sync();  // peers may still be reading this CTA's maxima
}

// =========================================================================
// CTA per row (K > 1024): T threads, NCH 16-byte chunks per thread held in
// registers (NCH == 0: re-read from global in every pass), optionally
// prefetching the CTA's next row while the current one is processed.
// Per-row partial sums and maxima go through shared memory double-buffered
// by row parity, so each row costs one barrier (two with the LayerNorm).
// =========================================================================
template <int T>
struct RowSharedT {
  long long s1[2][T / 32], s2h[2][T / 32], s2l[2][T / 32];
  int bad[2][T / 32];
  float mx[2][T / 32];
  float mx2[2][T / 32];  // NaN-free row maxima (rows holding a NaN or an Inf)
  float mu[2], rstd[2];
};

template <int MODE, int T, int NCH, bool PF, int CM>
__device__ __forceinline__ void cta_rows(const RowArgs& a, RowSharedT<T>& sh, float (&cmax)[CM]) {
  constexpr bool REG = NCH > 0;
  // weights: the folded values stay in registers between the two passes;
  // activations recompute them (registers go to occupancy instead)
  constexpr bool KEEPX = REG && NCH <= 8 && MODE == MODE_WEIGHT;
  constexpr int W = T / 32;
  constexpr bool CALIB_REG = (MODE == MODE_CALIB) && REG && CM == NCH * 8;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int64_t Kc = a.K / 8;
  const int nch = REG ? NCH : static_cast<int>((Kc + T - 1) / T);
  const bool use_ln = (MODE != MODE_WEIGHT) && a.gamma != nullptr;

  uint4 v[REG ? NCH : 1];
  uint4 nv[(REG && PF) ? NCH : 1];
  auto load_row = [&](int64_t row, uint4* dst) {
    const uint4* src = reinterpret_cast<const uint4*>(a.x + row * a.ld);
#pragma unroll
    for (int i = 0; i < (REG ? NCH : 1); ++i) {
      const int64_t c = tid + static_cast<int64_t>(i) * T;
      dst[i] = c < Kc ? ld_stream(src + c) : make_uint4(0, 0, 0, 0);
    }
  };
  if (REG && PF && static_cast<int64_t>(blockIdx.x) < a.rows) load_row(blockIdx.x, v);
  int par = 0;
  for (int64_t r = blockIdx.x; r < a.rows; r += gridDim.x, par ^= 1) {
    if (REG && !PF) load_row(r, v);
    if (REG && PF) {
      const int64_t rn = r + gridDim.x;
      if (rn < a.rows) load_row(rn, nv);
    }
    const uint4* src = reinterpret_cast<const uint4*>(a.x + r * a.ld);
    auto chunk = [&](int i, int64_t c) -> uint4 {
      if constexpr (REG) return v[i];
      else return __ldg(src + c);
    };
    const int iters = REG ? NCH : nch;

    float mu = 0.0f, rstd = 0.0f;
    if (use_ln) {
      Sums s{0, 0, 0, 0};
#pragma unroll
      for (int i = 0; i < iters; ++i) {
        const int64_t c = tid + static_cast<int64_t>(i) * T;
        if (c < Kc) chunk_sums(chunk(i, c), s);
      }
      warp_sum(s);
      if (lane == 0) {
        sh.s1[par][warp] = s.s1;
        sh.s2h[par][warp] = s.s2h;
        sh.s2l[par][warp] = s.s2l;
        sh.bad[par][warp] = s.bad;
      }
      __syncthreads();
      if (warp == 0) {  // one warp turns the sums into mu / rstd and broadcasts them
        Sums t{0, 0, 0, 0};
#pragma unroll
        for (int w = 0; w < W; ++w) {
          t.s1 += sh.s1[par][w];
          t.s2h += sh.s2h[par][w];
          t.s2l += sh.s2l[par][w];
          t.bad |= sh.bad[par][w];
        }
        float m_, r_;
        ln_finalize(t, a.K, a.eps, m_, r_);
        if (lane == 0) {
          sh.mu[par] = m_;
          sh.rstd[par] = r_;
        }
      }
      __syncthreads();
      mu = sh.mu[par];
      rstd = sh.rstd[par];
    }

    if (MODE == MODE_CALIB) {
#pragma unroll
      for (int i = 0; i < iters; ++i) {
        const int64_t c = tid + static_cast<int64_t>(i) * T;
        if (c < Kc) {
          float x[8];
          transform8<MODE>(chunk(i, c), c, a, mu, rstd, x);
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            const float ax = fabsf(x[j]);
            if constexpr (CALIB_REG) cmax[i * 8 + j] = fmaxf(cmax[i * 8 + j], ax);
            else atomicMax(reinterpret_cast<int*>(a.amax) + c * 8 + j, __float_as_int(fmaxf(ax, 0.0f)));  // NaN: 0
          }
        }
      }
    } else if (a.range_in) {  // per-tensor scale fixed in advance: no row max, one pass
      float sc, inv;
      range_scale(a, r, sc, inv);
      if (tid == 0) a.scale[r] = sc;
      int8_t* dst = a.q + r * a.K;
#pragma unroll
      for (int i = 0; i < iters; ++i) {
        const int64_t c = tid + static_cast<int64_t>(i) * T;
        if (c < Kc) {
          float x[8];
          transform8<MODE>(chunk(i, c), c, a, mu, rstd, x);
          *reinterpret_cast<uint2*>(dst + c * 8) = pack8c(x, inv);
        }
      }
    } else {
      float amax = 0.0f;
      float xs[KEEPX ? NCH : 1][8];
#pragma unroll
      for (int i = 0; i < iters; ++i) {
        const int64_t c = tid + static_cast<int64_t>(i) * T;
        if (c < Kc) {
          float x[8];
          transform8<MODE>(chunk(i, c), c, a, mu, rstd, x);
#pragma unroll
          for (int j = 0; j < 8; ++j) amax = absmax_nan(amax, x[j]);
          if constexpr (KEEPX) {
#pragma unroll
            for (int j = 0; j < 8; ++j) xs[i][j] = x[j];
          }
        }
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) amax = absmax_nan(amax, __shfl_xor_sync(0xffffffffu, amax, o));
      if (lane == 0) sh.mx[par][warp] = amax;
      __syncthreads();
      float m = 0.0f;
#pragma unroll
      for (int w = 0; w < W; ++w) m = absmax_nan(m, sh.mx[par][w]);
      const bool safe = !finite_f(m);  // CTA-uniform
      if (safe) {  // a NaN or an Inf in the row: the range ignores NaN
        float a2 = 0.0f;
#pragma unroll
        for (int i = 0; i < iters; ++i) {
          const int64_t c = tid + static_cast<int64_t>(i) * T;
          if (c < Kc) {
            float x[8];
            if constexpr (KEEPX) {
#pragma unroll
              for (int j = 0; j < 8; ++j) x[j] = xs[i][j];
            } else {
              transform8<MODE>(chunk(i, c), c, a, mu, rstd, x);
            }
#pragma unroll
            for (int j = 0; j < 8; ++j) a2 = fmaxf(a2, fabsf(x[j]));
          }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) a2 = fmaxf(a2, __shfl_xor_sync(0xffffffffu, a2, o));
        if (lane == 0) sh.mx2[par][warp] = a2;
        __syncthreads();
        m = 0.0f;
#pragma unroll
        for (int w = 0; w < W; ++w) m = fmaxf(m, sh.mx2[par][w]);
      }
      m = fabsf(m);
      if (a.range_out) {  // range pass only
        if (tid == 0) range_merge(a, r, m);
      } else {
        const float sc = __fdiv_rn(m, 127.0f);
        const float inv = sc > 0.0f ? __frcp_rn(sc) : 0.0f;
        if (tid == 0) a.scale[r] = sc;
        int8_t* dst = a.q + r * a.K;
        auto store = [&](auto safe_t) {
#pragma unroll
          for (int i = 0; i < iters; ++i) {
            const int64_t c = tid + static_cast<int64_t>(i) * T;
            if (c < Kc) {
              float x[8];
              if constexpr (KEEPX) {
#pragma unroll
                for (int j = 0; j < 8; ++j) x[j] = xs[i][j];
              } else {
                transform8<MODE>(chunk(i, c), c, a, mu, rstd, x);
              }
              *reinterpret_cast<uint2*>(dst + c * 8) = pack8<decltype(safe_t)::value>(x, inv);
            }
          }
        };
        if (safe) store(std::true_type{});
        else store(std::false_type{});
      }
    }
    if (REG && PF) {
#pragma unroll
      for (int i = 0; i < (REG ? NCH : 1); ++i) v[i] = nv[i];
    }
  }
}

// Register-resident rows (NCH <= 8): every value is converted to fp32 once;
// the statistics, the transform (in place), the absmax and the quantization
// all work on those registers.
template <int MODE, int T, int NCH, bool PF, int CM>
__device__ __forceinline__ void cta_rows_fast(const RowArgs& a, RowSharedT<T>& sh, float (&cmax)[CM]) {
  constexpr int W = T / 32;
  constexpr bool CALIB_REG = (MODE == MODE_CALIB) && CM == NCH * 8;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int64_t Kc = a.K / 8;
  const bool use_ln = (MODE != MODE_WEIGHT) && a.gamma != nullptr;

  uint4 v[NCH];
  uint4 nv[PF ? NCH : 1];
  auto load_row = [&](int64_t row, uint4* dst) {
    const uint4* src = reinterpret_cast<const uint4*>(a.x + row * a.ld);
#pragma unroll
    for (int i = 0; i < NCH; ++i) {
      const int64_t c = tid + static_cast<int64_t>(i) * T;
      dst[i] = c < Kc ? ld_stream(src + c) : make_uint4(0, 0, 0, 0);
    }
  };
  if (PF && static_cast<int64_t>(blockIdx.x) < a.rows) load_row(blockIdx.x, v);
  int par = 0;
  for (int64_t r = blockIdx.x; r < a.rows; r += gridDim.x, par ^= 1) {
    if (!PF) load_row(r, v);
    if (PF) {
      const int64_t rn = r + gridDim.x;
      if (rn < a.rows) load_row(rn, nv);
    }
    float x[NCH][8];
#pragma unroll
    for (int i = 0; i < NCH; ++i) unpack8(v[i], x[i]);  // chunks past K are zeros

    float mu = 0.0f, rstd = 0.0f;
    if (use_ln) {
      Sums s{0, 0, 0, 0};
#pragma unroll
      for (int i = 0; i < NCH; ++i)
        if (tid + static_cast<int64_t>(i) * T < Kc) chunk_sums_f(x[i], s);
      warp_sum(s);
      if (lane == 0) {
        sh.s1[par][warp] = s.s1;
        sh.s2h[par][warp] = s.s2h;
        sh.s2l[par][warp] = s.s2l;
        sh.bad[par][warp] = s.bad;
      }
      __syncthreads();
      if (warp == 0) {
        Sums t{0, 0, 0, 0};
#pragma unroll
        for (int w = 0; w < W; ++w) {
          t.s1 += sh.s1[par][w];
          t.s2h += sh.s2h[par][w];
          t.s2l += sh.s2l[par][w];
          t.bad |= sh.bad[par][w];
        }
        float m_, r_;
        ln_finalize(t, a.K, a.eps, m_, r_);
        if (lane == 0) {
          sh.mu[par] = m_;
          sh.rstd[par] = r_;
        }
      }
      __syncthreads();
      mu = sh.mu[par];
      rstd = sh.rstd[par];
    }
    float amax = 0.0f;
#pragma unroll
    for (int i = 0; i < NCH; ++i) {
      const int64_t c = tid + static_cast<int64_t>(i) * T;
      if (c < Kc) {
        transform8f<MODE>(x[i], c, a, mu, rstd);
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          if constexpr (MODE == MODE_CALIB) {
            if constexpr (CALIB_REG) cmax[i * 8 + j] = fmaxf(cmax[i * 8 + j], fabsf(x[i][j]));
          } else {
            amax = absmax_nan(amax, x[i][j]);
          }
        }
      }
    }
    if constexpr (MODE != MODE_CALIB) {
      int8_t* dst = a.q + r * a.K;
      if (a.range_in) {  // per-tensor scale fixed in advance: no row max
        float sc, inv;
        range_scale(a, r, sc, inv);
        if (tid == 0) a.scale[r] = sc;
#pragma unroll
        for (int i = 0; i < NCH; ++i) {
          const int64_t c = tid + static_cast<int64_t>(i) * T;
          if (c < Kc) *reinterpret_cast<uint2*>(dst + c * 8) = pack8c(x[i], inv);
        }
      } else {
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) amax = absmax_nan(amax, __shfl_xor_sync(0xffffffffu, amax, o));
        if (lane == 0) sh.mx[par][warp] = amax;
        __syncthreads();
        float m = 0.0f;
#pragma unroll
        for (int w = 0; w < W; ++w) m = absmax_nan(m, sh.mx[par][w]);
        const bool safe = !finite_f(m);  // CTA-uniform
        if (safe) {  // a NaN or an Inf in the row: the range ignores NaN
          float a2 = 0.0f;
#pragma unroll
          for (int i = 0; i < NCH; ++i)
            if (tid + static_cast<int64_t>(i) * T < Kc)
#pragma unroll
              for (int j = 0; j < 8; ++j) a2 = fmaxf(a2, fabsf(x[i][j]));
#pragma unroll
          for (int o = 16; o > 0; o >>= 1) a2 = fmaxf(a2, __shfl_xor_sync(0xffffffffu, a2, o));
          if (lane == 0) sh.mx2[par][warp] = a2;
          __syncthreads();
          m = 0.0f;
#pragma unroll
          for (int w = 0; w < W; ++w) m = fmaxf(m, sh.mx2[par][w]);
        }
        m = fabsf(m);
        if (a.range_out) {  // range pass only
          if (tid == 0) range_merge(a, r, m);
        } else {
          const float sc = __fdiv_rn(m, 127.0f);
          const float inv = sc > 0.0f ? __frcp_rn(sc) : 0.0f;
          if (tid == 0) a.scale[r] = sc;
          auto store = [&](auto safe_t) {
#pragma unroll
            for (int i = 0; i < NCH; ++i) {
              const int64_t c = tid + static_cast<int64_t>(i) * T;
              if (c < Kc) *reinterpret_cast<uint2*>(dst + c * 8) = pack8<decltype(safe_t)::value>(x[i], inv);
            }
          };
          if (safe) store(std::true_type{});
          else store(std::false_type{});
        }
      }
    }
    if (PF) {
#pragma unroll
      for (int i = 0; i < NCH; ++i) v[i] = nv[i];
    }
  }
}

template <int MODE, int T, int NCH, bool PF>
__global__ void __launch_bounds__(T) k_rows_cta(const RowArgs a) {
  __shared__ RowSharedT<T> sh;
  griddep_wait();
  griddep_launch_dependents();
  float none[1];
  if constexpr (NCH > 0 && NCH <= 8) cta_rows_fast<MODE, T, NCH, PF, 1>(a, sh, none);
  else cta_rows<MODE, T, NCH, PF, 1>(a, sh, none);
}

// CTA-per-row calibration with register maxima, merged across a cluster of 8
// CTAs through distributed shared memory.
template <int T, int NCH>
__global__ void __cluster_dims__(kCluster, 1, 1) __launch_bounds__(T) k_calib_cta(const RowArgs a) {
  __shared__ RowSharedT<T> sh;
  extern __shared__ int colmax_s[];
  cg::cluster_group cluster = cg::this_cluster();
  float cmax[NCH * 8];
#pragma unroll
  for (int i = 0; i < NCH * 8; ++i) cmax[i] = 0.0f;
  griddep_wait();
  griddep_launch_dependents();
  cta_rows_fast<MODE_CALIB, T, NCH, true, NCH * 8>(a, sh, cmax);
  const int64_t Kc = a.K / 8;
#pragma unroll
  for (int i = 0; i < NCH; ++i) {
    const int64_t c = threadIdx.x + static_cast<int64_t>(i) * T;
    if (c < Kc)
#pragma unroll
      for (int j = 0; j < 8; ++j) colmax_s[c * 8 + j] = __float_as_int(cmax[i * 8 + j]);
  }
  __syncthreads();
  cluster.sync();
  const int64_t slice = (a.K + kCluster - 1) / kCluster;
  const int64_t j0 = static_cast<int64_t>(cluster.block_rank()) * slice;
  const int64_t j1 = j0 + slice < a.K ? j0 + slice : a.K;
  for (int64_t j = j0 + threadIdx.x; j < j1; j += T) {
    int m = 0;
#pragma unroll
    for (int q = 0; q < kCluster; ++q) m = max(m, cluster.map_shared_rank(colmax_s, q)[j]);
    atomicMax(reinterpret_cast<int*>(a.amax) + j, m);
  }
  cluster.sync();  // peers may still be reading this CTA's maxima
}

// Per-row global atomics: calibration with K too large for register maxima.
__global__ void __launch_bounds__(kCtaThreads) k_calib_cta_atomic(const RowArgs a) {
  __shared__ RowSharedT<kCtaThreads> sh;
  griddep_wait();
  griddep_launch_dependents();
  float none[1];
  cta_rows<MODE_CALIB, kCtaThreads, 0, false, 1>(a, sh, none);
}

// =========================================================================
// LayerNorm / smoothing + per-token quantization, and fold + per-channel
// weight quantization, rows staged by bulk copies.
//
// One CTA of T threads per row, persistent over rows (grid-stride).  One
// thread streams whole rows into a 2-slot shared-memory ring with untiled
// bulk copies (cp.async.bulk, one instruction per row, completion counted on
// an mbarrier), so each CTA has the next row in flight while it works on the
// current one and no register holds prefetched data.  Every thread keeps its
// NCH chunks of 8 values as fp32 in registers from its read of shared memory
// to the codes.  Per element:
//   statistics  exact sums in fp64: h (a multiple of 2^-24, |h| < 2^16) adds
//               exactly into an fp64 accumulator; h*h (exact in fp64) goes
//               into an accumulator A biased by 1.5 * 2^43 (unit in the last
//               place 2^-9 for every partial sum) with one fused multiply-add,
//               A' = fma(h, h, A), and the part that rounding dropped,
//               fma(h, h, A - A') (exact: A - A' is exact and so is the
//               remainder, a multiple of 2^-48 below 2^-10), into a second
//               accumulator.  Two independent sets per thread (even / odd
//               elements), added (exactly) into three fp64 partials per
//               thread.  One warp alone reduces them: per lane the partials
//               of T / 32 threads in fp64, pairwise (exact: at most 512
//               elements), then as int64 across the warp: S1 = sum v and
//               S2 = sum v^2 (v = h * 2^24) exactly, whatever the order.
//   transform   (x - mu) * rstd, then * gamma, in packed fp32 pairs (each lane
//               rounded like the scalar op), + beta in scalar adds (a packed add
//               after a packed multiply can be contracted into a fused
//               multiply-add; a scalar one is not), times inv_s packed; for a
//               weight row (no statistics) w * s packed, rounded to fp16 pairs
//   maximum     three-input NaN-propagating max of absolute values; across
//               lanes and warps an unsigned max of the bit patterns (|x| and a
//               positive NaN order as their bits: NaN above Inf above finite)
//   codes       x * (1 / scale) packed, + 1.5 * 2^23 scalar, low bytes packed
// FULL: K = 8 * NCH * T, every chunk of every thread is inside the row.
// One thread waits for each row (suspended in the mbarrier try-wait, bounded);
// the others wait at the row's first barrier, which also turns a time-out into
// a CTA-wide stop, after which the CTA waits (bounded) for its copies in
// flight before returning.  Rows of up to four warps, one at a time: with a
// LayerNorm two more barriers (statistics from the values in registers, then
// mu / rstd from warp 0) and one for the row maximum.  Rows of eight warps
// with a LayerNorm run one row deep instead: the statistics of row j+1 (read
// again from its slot) and the transform of row j between the same two
// barriers, the finalization of row j+1 by one warp after row j's codes.
// Rows with a non-finite maximum take the NaN-free maximum and the NaN-safe
// codes, as in the kernels above.
// =========================================================================
constexpr double kS2Bias = 13194139533312.0;  // 1.5 * 2^43: unit in the last place 2^-9

// x - mu lane-wise (a subtraction feeding a multiply: nothing to contract)
__device__ __forceinline__ uint64_t f2_sub_rn(uint64_t a, uint64_t b) {
  uint64_t r;
  asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}

__device__ __forceinline__ float absmax3(float m, float a, float b) {
  float d;
  asm("max.NaN.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(m), "f"(fabsf(a)), "f"(fabsf(b)));
  return d;
}

__device__ __forceinline__ void bulk_row_load(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
               ::"r"(dst), "l"(src), "r"(bytes), "r"(bar)
               : "memory");
}

template <int T, bool STATS>
struct ActShared {
  static constexpr int NP = STATS ? T : 1;
  double p1[2][NP], p2h[2][NP], p2l[2][NP];  // per-thread statistics partials (LayerNorm rows)
  alignas(16) uint32_t mx[2][T / 32];     // per-warp row maxima (bit patterns)
  alignas(16) uint32_t mx2[2][T / 32];
  float mu[2], rstd[2];
  alignas(8) uint64_t full[2];
};

// Unsigned max over the warp (redux.sync).
__device__ __forceinline__ uint32_t warp_max_u32(uint32_t v) {
  uint32_t r;
  asm volatile("redux.sync.max.u32 %0, %1, 0xffffffff;" : "=r"(r) : "r"(v));
  return r;
}

template <int MODE, int T, int NCH, bool FULL>
__device__ __forceinline__ void rows_bulk(const RowArgs& a, uint32_t* status, uint64_t budget) {
  constexpr int W = T / 32;
  __shared__ ActShared<T, MODE == MODE_ACT> sh;
  extern __shared__ __align__(128) uint8_t ring[];  // 2 slots of one row (2K bytes each)
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int64_t Kc = a.K >> 3;
  const uint32_t row_bytes = static_cast<uint32_t>(a.K * 2);
  const uint32_t slot0 = smem_u32(ring);
  const uint32_t full0 = smem_u32(&sh.full[0]);
  const bool use_ln = MODE == MODE_ACT && a.gamma != nullptr;
  const int k_log2 = (a.K & (a.K - 1)) == 0 ? __ffsll(a.K) - 1 : -1;  // K a power of two: its log2
  const int64_t G = gridDim.x;
  if (tid == 0) {
    mbar_init(full0, 1);
    mbar_init(full0 + 8, 1);
    fence_barrier_init();
  }
  __syncthreads();
  griddep_wait();  // h (and gamma / beta / inv_s) come from earlier kernels
  griddep_launch_dependents();

  // thread 0: issue the copy of the row of iteration j into slot j & 1
  int64_t issued = 0;  // iterations whose copy has been issued (thread 0)
  auto issue = [&](int64_t j) {
    const int64_t row = blockIdx.x + j * G;
    if (row >= a.rows) return;
    const uint32_t bar = full0 + 8u * static_cast<uint32_t>(j & 1);
    mbar_arrive_expect_tx(bar, row_bytes);
    bulk_row_load(slot0 + static_cast<uint32_t>(j & 1) * row_bytes, a.x + row * a.ld, row_bytes, bar);
    issued = j + 1;
  };
  if (tid == 0) {
    issue(0);
    issue(1);
  }
  int64_t consumed = 0;  // copies whose landing has been waited for (a time-out drains the rest)
  bool aborted = false;

  if constexpr (W < 8) {
    // rows of up to four warps, one row at a time: with a LayerNorm the
    // statistics from the values in registers, one warp finalizes between two
    // barriers, then the transform, the row maximum and the codes
    int par = 0;
    for (int64_t j = 0;; ++j, par ^= 1) {
      const int64_t r = blockIdx.x + j * G;
      if (r >= a.rows) break;
      const uint32_t s = static_cast<uint32_t>(j & 1);
      // one thread waits for the row (the others wait at the barrier, issuing
      // nothing); the barrier also makes a time-out a CTA-wide decision
      bool ok = true;
      if (tid == 0) ok = mbar_wait_bounded(full0 + 8u * s, static_cast<uint32_t>((j >> 1) & 1), budget);
      if (__syncthreads_or(!ok)) {
        aborted = true;
        break;
      }
      float x[NCH][8];
      const uint4* src = reinterpret_cast<const uint4*>(ring + s * row_bytes);
#pragma unroll
      for (int i = 0; i < NCH; ++i) {
        const int64_t c = tid + static_cast<int64_t>(i) * T;
        uint4 v = make_uint4(0, 0, 0, 0);
        if (FULL || c < Kc) v = src[c];
        unpack8(v, x[i]);  // chunks past K are zeros
      }

      float mu = 0.0f, rstd = 0.0f;
      if (use_ln) {
        double s1[2] = {0.0, 0.0}, hi[2] = {kS2Bias, kS2Bias}, lo[2] = {0.0, 0.0};
        int bad;
#pragma unroll
        for (int i = 0; i < NCH; ++i) {
#pragma unroll
          for (int jj = 0; jj < 8; ++jj) {
            const int u = jj & 1;
            const double d = static_cast<double>(x[i][jj]);
            s1[u] = __dadd_rn(s1[u], d);
            const double hn = __fma_rn(d, d, hi[u]);
            lo[u] = __dadd_rn(lo[u], __fma_rn(d, d, __dsub_rn(hi[u], hn)));
            hi[u] = hn;
          }
        }
        // this thread's partials (exact: multiples of 2^-24, 2^-9 and 2^-48 far
        // inside 53 bits); an Inf or a NaN in the row leaves them non-finite
        sh.p1[par][tid] = __dadd_rn(s1[0], s1[1]);
        sh.p2h[par][tid] = __dadd_rn(__dsub_rn(hi[0], kS2Bias), __dsub_rn(hi[1], kS2Bias));
        sh.p2l[par][tid] = __dadd_rn(lo[0], lo[1]);
        __syncthreads();  // every thread has read slot s
        consumed = j + 1;
        if (tid == 0) issue(j + 2);
        if (warp == 0) {
          // pairwise (every partial sum is exact, so any order gives the same)
          double q1[W], q2h[W], q2l[W];
#pragma unroll
          for (int w = 0; w < W; ++w) {
            q1[w] = sh.p1[par][32 * w + lane];
            q2h[w] = sh.p2h[par][32 * w + lane];
            q2l[w] = sh.p2l[par][32 * w + lane];
          }
#pragma unroll
          for (int st = 1; st < W; st *= 2)
#pragma unroll
            for (int w = 0; w + st < W; w += 2 * st) {
              q1[w] = __dadd_rn(q1[w], q1[w + st]);
              q2h[w] = __dadd_rn(q2h[w], q2h[w + st]);
              q2l[w] = __dadd_rn(q2l[w], q2l[w + st]);
            }
          const double t1 = q1[0], t2h = q2h[0], t2l = q2l[0];
          bad = !(fabs(t1) <= 1.7976931348623157e308) || !(fabs(t2h) <= 1.7976931348623157e308);
          Sums t{bad ? 0 : __double2ll_rn(__dmul_rn(t1, 16777216.0)),          // units 2^-24
                 bad ? 0 : __double2ll_rn(__dmul_rn(t2h, 8192.0)),             // units 2^-13
                 bad ? 0 : __double2ll_rn(__dmul_rn(t2l, 281474976710656.0)),  // units 2^-48
                 bad};
          warp_sum(t);
          float m_, r_;
          ln_finalize(t, a.K, a.eps, m_, r_, k_log2);
          if (lane == 0) {
            sh.mu[par] = m_;
            sh.rstd[par] = r_;
          }
        }
        __syncthreads();
        mu = sh.mu[par];
        rstd = sh.rstd[par];
      }

      // transform in place and the row maximum (NaN-propagating)
      float amax = 0.0f;
      {
        const uint64_t mu2 = f2_pack(mu, mu), r2 = f2_pack(rstd, rstd);
#pragma unroll
        for (int i = 0; i < NCH; ++i) {
          const int64_t c = tid + static_cast<int64_t>(i) * T;
          if (FULL || c < Kc) {
            const int64_t k0 = c * 8;
            if (use_ln) {
              const float4 g0 = __ldg(reinterpret_cast<const float4*>(a.gamma + k0));
              const float4 g1 = __ldg(reinterpret_cast<const float4*>(a.gamma + k0) + 1);
              const float gg[8] = {g0.x, g0.y, g0.z, g0.w, g1.x, g1.y, g1.z, g1.w};
              float bb[8] = {0, 0, 0, 0, 0, 0, 0, 0};
              if (a.beta) {
                const float4 b0 = __ldg(reinterpret_cast<const float4*>(a.beta + k0));
                const float4 b1 = __ldg(reinterpret_cast<const float4*>(a.beta + k0) + 1);
                bb[0] = b0.x; bb[1] = b0.y; bb[2] = b0.z; bb[3] = b0.w;
                bb[4] = b1.x; bb[5] = b1.y; bb[6] = b1.z; bb[7] = b1.w;
              }
              // ((x - mu) * rstd) * gamma in packed pairs; the add of beta stays
              // scalar (a packed add right after a packed multiply was seen
              // contracted into one fused multiply-add)
#pragma unroll
              for (int jj = 0; jj < 8; jj += 2) {
                const float2 f = f2_unpack(f2_mul_rn(f2_mul_rn(f2_sub_rn(f2_pack(x[i][jj], x[i][jj + 1]), mu2), r2),
                                                     f2_pack(gg[jj], gg[jj + 1])));
                x[i][jj] = f.x;
                x[i][jj + 1] = f.y;
              }
              if (a.beta) {
#pragma unroll
                for (int jj = 0; jj < 8; ++jj) x[i][jj] = __fadd_rn(x[i][jj], bb[jj]);
              }
            }
            if (a.vec) {
              const float4 i0 = __ldg(reinterpret_cast<const float4*>(a.vec + k0));
              const float4 i1 = __ldg(reinterpret_cast<const float4*>(a.vec + k0) + 1);
              const float is[8] = {i0.x, i0.y, i0.z, i0.w, i1.x, i1.y, i1.z, i1.w};
#pragma unroll
              for (int jj = 0; jj < 8; jj += 2) {
                float2 f = f2_unpack(f2_mul_rn(f2_pack(x[i][jj], x[i][jj + 1]), f2_pack(is[jj], is[jj + 1])));
                // a weight row: x = fp16(w * s), the folded weight rounded once to fp16
                if (MODE == MODE_WEIGHT) f = __half22float2(__floats2half2_rn(f.x, f.y));
                x[i][jj] = f.x;
                x[i][jj + 1] = f.y;
              }
            }
#pragma unroll
            for (int jj = 0; jj < 8; jj += 2) amax = absmax3(amax, x[i][jj], x[i][jj + 1]);
          }
        }
      }
      // amax is >= 0 or a positive NaN (max.NaN of absolute values)
      const uint32_t wmax = warp_max_u32(__float_as_uint(amax));
      if (lane == 0) sh.mx[par][warp] = wmax;
      __syncthreads();  // (without a LayerNorm: every thread has read slot s)
      if (!use_ln) {
        consumed = j + 1;
        if (tid == 0) issue(j + 2);
      }
      uint32_t mb = 0;
#pragma unroll
      for (int w = 0; w < W; ++w) mb = max(mb, sh.mx[par][w]);
      float m = __uint_as_float(mb);
      const bool safe = !finite_f(m);  // CTA-uniform
      if (safe) {  // a NaN or an Inf in the row: the range ignores NaN
        float a2 = 0.0f;
#pragma unroll
        for (int i = 0; i < NCH; ++i)
          if (FULL || tid + static_cast<int64_t>(i) * T < Kc)
#pragma unroll
            for (int jj = 0; jj < 8; ++jj) a2 = fmaxf(a2, fabsf(x[i][jj]));
        const uint32_t w2 = warp_max_u32(__float_as_uint(a2));  // NaN-free, >= 0
        if (lane == 0) sh.mx2[par][warp] = w2;
        __syncthreads();
        mb = 0;
#pragma unroll
        for (int w = 0; w < W; ++w) mb = max(mb, sh.mx2[par][w]);
        m = __uint_as_float(mb);
      }
      const float sc = __fdiv_rn(m, 127.0f);
      const float inv = sc > 0.0f ? __frcp_rn(sc) : 0.0f;
      if (tid == 0) a.scale[r] = sc;
      int8_t* dst = a.q + r * a.K;
      const uint64_t inv2 = f2_pack(inv, inv);
#pragma unroll
      for (int i = 0; i < NCH; ++i) {
        const int64_t c = tid + static_cast<int64_t>(i) * T;
        if (FULL || c < Kc) {
          uint32_t b[8];
          // x * (1 / scale) in packed pairs, then + 1.5 * 2^23 in scalar adds (each rounded)
#pragma unroll
          for (int jj = 0; jj < 8; jj += 2) {
            const float2 p = f2_unpack(f2_mul_rn(f2_pack(x[i][jj], x[i][jj + 1]), inv2));
            b[jj] = __float_as_uint(__fadd_rn(p.x, 12582912.0f));
            b[jj + 1] = __float_as_uint(__fadd_rn(p.y, 12582912.0f));
          }
          if (safe) {
#pragma unroll
            for (int jj = 0; jj < 8; ++jj) b[jj] = min(b[jj], 0x4B400100u);
          }
          const uint32_t lo4 = __byte_perm(__byte_perm(b[0], b[1], 0x0040), __byte_perm(b[2], b[3], 0x0040), 0x5410);
          const uint32_t hi4 = __byte_perm(__byte_perm(b[4], b[5], 0x0040), __byte_perm(b[6], b[7], 0x0040), 0x5410);
          *reinterpret_cast<uint2*>(dst + c * 8) = make_uint2(lo4, hi4);
        }
      }
    }
  } else {
    // rows of eight warps
    // one thread waits for copy j when `has` (the others wait at the barrier,
    // issuing nothing); the barrier also turns a time-out into a CTA-wide stop
    auto wait_copy = [&](int64_t j, bool has) {
      bool ok = true;
      if (tid == 0 && has)
        ok = mbar_wait_bounded(full0 + 8u * static_cast<uint32_t>(j & 1), static_cast<uint32_t>((j >> 1) & 1), budget);
      if (__syncthreads_or(!ok)) return false;
      if (has) consumed = j + 1;
      return true;
    };
    // this thread's NCH chunks of the row in slot s, as fp32 (chunks past K are zeros)
    auto load_x = [&](uint32_t s, float (&x)[NCH][8]) {
      const uint4* src = reinterpret_cast<const uint4*>(ring + s * row_bytes);
#pragma unroll
      for (int i = 0; i < NCH; ++i) {
        const int64_t c = tid + static_cast<int64_t>(i) * T;
        uint4 v = make_uint4(0, 0, 0, 0);
        if (FULL || c < Kc) v = src[c];
        unpack8(v, x[i]);
      }
    };
    // the exact LayerNorm partials of this thread's chunks of the row in slot s
    // (read again from shared memory, each fp16 value converted once to fp64)
    // into sh.p*[pp][tid]: exact, multiples of 2^-24, 2^-9 and 2^-48 far inside
    // 53 bits; an Inf or a NaN in the row leaves them non-finite
    auto stats = [&](uint32_t s, int pp) {
      const uint4* src = reinterpret_cast<const uint4*>(ring + s * row_bytes);
      double s1[2] = {0.0, 0.0}, hi[2] = {kS2Bias, kS2Bias}, lo[2] = {0.0, 0.0};
#pragma unroll
      for (int i = 0; i < NCH; ++i) {
        const int64_t c = tid + static_cast<int64_t>(i) * T;
        uint4 v = make_uint4(0, 0, 0, 0);
        if (FULL || c < Kc) v = src[c];
#pragma unroll
        for (int jj = 0; jj < 8; ++jj) {
          const int u = jj & 1;
          const double d = half_to_f64(half_bits(v, jj));
          s1[u] = __dadd_rn(s1[u], d);
          const double hn = __fma_rn(d, d, hi[u]);
          lo[u] = __dadd_rn(lo[u], __fma_rn(d, d, __dsub_rn(hi[u], hn)));
          hi[u] = hn;
        }
      }
      sh.p1[pp][tid] = __dadd_rn(s1[0], s1[1]);
      sh.p2h[pp][tid] = __dadd_rn(__dsub_rn(hi[0], kS2Bias), __dsub_rn(hi[1], kS2Bias));
      sh.p2l[pp][tid] = __dadd_rn(lo[0], lo[1]);
    };
    // one warp: the row's mu / rstd from the partials sh.p*[pp] into sh.mu[pp], sh.rstd[pp]
    auto finalize = [&](int pp) {
      // pairwise (every partial sum is exact, so any order gives the same)
      double q1[W], q2h[W], q2l[W];
#pragma unroll
      for (int w = 0; w < W; ++w) {
        q1[w] = sh.p1[pp][32 * w + lane];
        q2h[w] = sh.p2h[pp][32 * w + lane];
        q2l[w] = sh.p2l[pp][32 * w + lane];
      }
#pragma unroll
      for (int st = 1; st < W; st *= 2)
#pragma unroll
        for (int w = 0; w + st < W; w += 2 * st) {
          q1[w] = __dadd_rn(q1[w], q1[w + st]);
          q2h[w] = __dadd_rn(q2h[w], q2h[w + st]);
          q2l[w] = __dadd_rn(q2l[w], q2l[w + st]);
        }
      const double t1 = q1[0], t2h = q2h[0], t2l = q2l[0];
      const int bad = !(fabs(t1) <= 1.7976931348623157e308) || !(fabs(t2h) <= 1.7976931348623157e308);
      Sums t{bad ? 0 : __double2ll_rn(__dmul_rn(t1, 16777216.0)),          // units 2^-24
             bad ? 0 : __double2ll_rn(__dmul_rn(t2h, 8192.0)),             // units 2^-13
             bad ? 0 : __double2ll_rn(__dmul_rn(t2l, 281474976710656.0)),  // units 2^-48
             bad};
      warp_sum(t);
      float m_, r_;
      ln_finalize(t, a.K, a.eps, m_, r_, k_log2);
      if (lane == 0) {
        sh.mu[pp] = m_;
        sh.rstd[pp] = r_;
      }
    };
    // this warp's row maximum (bit patterns: amax is >= 0 or a positive NaN)
    auto publish = [&](float amax, int pp) {
      const uint32_t wmax = warp_max_u32(__float_as_uint(amax));
      if (lane == 0) sh.mx[pp][warp] = wmax;
    };
    // the transform in place and this thread's row maximum (NaN-propagating)
    auto transform = [&](float (&x)[NCH][8], float mu, float rstd) {
      float amax = 0.0f;
      {
        const uint64_t mu2 = f2_pack(mu, mu), r2 = f2_pack(rstd, rstd);
#pragma unroll
        for (int i = 0; i < NCH; ++i) {
          const int64_t c = tid + static_cast<int64_t>(i) * T;
          if (FULL || c < Kc) {
            const int64_t k0 = c * 8;
            if (use_ln) {
              const float4 g0 = __ldg(reinterpret_cast<const float4*>(a.gamma + k0));
              const float4 g1 = __ldg(reinterpret_cast<const float4*>(a.gamma + k0) + 1);
              const float gg[8] = {g0.x, g0.y, g0.z, g0.w, g1.x, g1.y, g1.z, g1.w};
              float bb[8] = {0, 0, 0, 0, 0, 0, 0, 0};
              if (a.beta) {
                const float4 b0 = __ldg(reinterpret_cast<const float4*>(a.beta + k0));
                const float4 b1 = __ldg(reinterpret_cast<const float4*>(a.beta + k0) + 1);
                bb[0] = b0.x; bb[1] = b0.y; bb[2] = b0.z; bb[3] = b0.w;
                bb[4] = b1.x; bb[5] = b1.y; bb[6] = b1.z; bb[7] = b1.w;
              }
              // ((x - mu) * rstd) * gamma in packed pairs; the add of beta stays
              // scalar (a packed add right after a packed multiply was seen
              // contracted into one fused multiply-add)
#pragma unroll
              for (int jj = 0; jj < 8; jj += 2) {
                const float2 f = f2_unpack(f2_mul_rn(f2_mul_rn(f2_sub_rn(f2_pack(x[i][jj], x[i][jj + 1]), mu2), r2),
                                                     f2_pack(gg[jj], gg[jj + 1])));
                x[i][jj] = f.x;
                x[i][jj + 1] = f.y;
              }
              if (a.beta) {
#pragma unroll
                for (int jj = 0; jj < 8; ++jj) x[i][jj] = __fadd_rn(x[i][jj], bb[jj]);
              }
            }
            if (a.vec) {
              const float4 i0 = __ldg(reinterpret_cast<const float4*>(a.vec + k0));
              const float4 i1 = __ldg(reinterpret_cast<const float4*>(a.vec + k0) + 1);
              const float is[8] = {i0.x, i0.y, i0.z, i0.w, i1.x, i1.y, i1.z, i1.w};
#pragma unroll
              for (int jj = 0; jj < 8; jj += 2) {
                float2 f = f2_unpack(f2_mul_rn(f2_pack(x[i][jj], x[i][jj + 1]), f2_pack(is[jj], is[jj + 1])));
                // a weight row: x = fp16(w * s), the folded weight rounded once to fp16
                if (MODE == MODE_WEIGHT) f = __half22float2(__floats2half2_rn(f.x, f.y));
                x[i][jj] = f.x;
                x[i][jj + 1] = f.y;
              }
            }
#pragma unroll
            for (int jj = 0; jj < 8; jj += 2) amax = absmax3(amax, x[i][jj], x[i][jj + 1]);
          }
        }
      }
      return amax;
    };
    // row r's scale from the warps' maxima in sh.mx[par], then its codes
    auto codes = [&](int64_t r, float (&x)[NCH][8], int par) {
      uint32_t mb = 0;
#pragma unroll
      for (int w = 0; w < W; ++w) mb = max(mb, sh.mx[par][w]);
      float m = __uint_as_float(mb);
      const bool safe = !finite_f(m);  // CTA-uniform
      if (safe) {  // a NaN or an Inf in the row: the range ignores NaN
        float a2 = 0.0f;
#pragma unroll
        for (int i = 0; i < NCH; ++i)
          if (FULL || tid + static_cast<int64_t>(i) * T < Kc)
#pragma unroll
            for (int jj = 0; jj < 8; ++jj) a2 = fmaxf(a2, fabsf(x[i][jj]));
        const uint32_t w2 = warp_max_u32(__float_as_uint(a2));  // NaN-free, >= 0
        if (lane == 0) sh.mx2[par][warp] = w2;
        __syncthreads();
        mb = 0;
#pragma unroll
        for (int w = 0; w < W; ++w) mb = max(mb, sh.mx2[par][w]);
        m = __uint_as_float(mb);
      }
      const float sc = __fdiv_rn(m, 127.0f);
      const float inv = sc > 0.0f ? __frcp_rn(sc) : 0.0f;
      if (tid == 0) a.scale[r] = sc;
      int8_t* dst = a.q + r * a.K;
      const uint64_t inv2 = f2_pack(inv, inv);
#pragma unroll
      for (int i = 0; i < NCH; ++i) {
        const int64_t c = tid + static_cast<int64_t>(i) * T;
        if (FULL || c < Kc) {
          uint32_t b[8];
          // x * (1 / scale) in packed pairs, then + 1.5 * 2^23 in scalar adds (each rounded)
#pragma unroll
          for (int jj = 0; jj < 8; jj += 2) {
            const float2 p = f2_unpack(f2_mul_rn(f2_pack(x[i][jj], x[i][jj + 1]), inv2));
            b[jj] = __float_as_uint(__fadd_rn(p.x, 12582912.0f));
            b[jj + 1] = __float_as_uint(__fadd_rn(p.y, 12582912.0f));
          }
          if (safe) {
#pragma unroll
            for (int jj = 0; jj < 8; ++jj) b[jj] = min(b[jj], 0x4B400100u);
          }
          const uint32_t lo4 = __byte_perm(__byte_perm(b[0], b[1], 0x0040), __byte_perm(b[2], b[3], 0x0040), 0x5410);
          const uint32_t hi4 = __byte_perm(__byte_perm(b[4], b[5], 0x0040), __byte_perm(b[6], b[7], 0x0040), 0x5410);
          *reinterpret_cast<uint2*>(dst + c * 8) = make_uint2(lo4, hi4);
        }
      }
    };

    if (!use_ln) {
      for (int64_t j = 0;; ++j) {
        const int64_t r = blockIdx.x + j * G;
        if (r >= a.rows) break;
        if (!wait_copy(j, true)) {
          aborted = true;
          break;
        }
        const int pp = static_cast<int>(j & 1);
        float x[NCH][8];
        load_x(static_cast<uint32_t>(pp), x);
        publish(transform(x, 0.0f, 0.0f), pp);
        __syncthreads();  // every thread has read slot pp; the warps' maxima are in
        if (tid == 0) issue(j + 2);
        codes(r, x, pp);
      }
    } else {
      // LayerNorm rows of eight warps, one row deep (the finalization, a reduction
      // over eight warps' partials, then overlaps the other warps' codes): iteration j takes the partials of row j+1
      // (its copy waited for at the iteration's first barrier, which also
      // publishes row j's mu / rstd), transforms row j, and after the second
      // barrier every warp writes row j's codes, one of them (in turn) then
      // finalizing row j+1 while the others go on to the next barrier
      if (static_cast<int64_t>(blockIdx.x) < a.rows) {
        if (!wait_copy(0, true)) {
          aborted = true;
        } else {
          stats(0u, 0);
          __syncthreads();
          if (warp == 0) finalize(0);
        }
      }
      for (int64_t j = 0; !aborted; ++j) {
        const int64_t r = blockIdx.x + j * G;
        if (r >= a.rows) break;
        const bool nxt = r + G < a.rows;
        const int pp = static_cast<int>(j & 1), pn = pp ^ 1;
        if (!wait_copy(j + 1, nxt)) {
          aborted = true;
          break;
        }
        if (nxt) stats(static_cast<uint32_t>(pn), pn);
        float x[NCH][8];
        load_x(static_cast<uint32_t>(pp), x);
        publish(transform(x, sh.mu[pp], sh.rstd[pp]), pp);
        __syncthreads();  // slot pp read; row j's maxima and row j+1's partials are in
        if (tid == 0) issue(j + 2);
        codes(r, x, pp);
        // (after the codes: the row's values are no longer held meanwhile)
        if (nxt && warp == static_cast<int>(j % W)) finalize(pn);
      }
    }
  }
  if (aborted) {
    if (tid == 0) {
      atomicCAS(status, DEV_OK, DEV_TIMEOUT);
      // wait (bounded) for the copies still in flight before shared memory is released
      for (int64_t j = consumed; j < issued; ++j)
        mbar_drain(full0 + 8u * static_cast<uint32_t>(j & 1), static_cast<uint32_t>((j >> 1) & 1), budget);
    }
    __syncthreads();
  }
}

// Activation rows (LayerNorm and / or 1/s, per-token scales) and weight rows
// (fold diag(s) rounded to fp16, per-output-channel scales).
// CTAs per SM the activation kernel is built for: two for rows of eight warps
// (at most 128 registers per thread, which the one-row-deep LayerNorm pipeline
// would otherwise exceed); 0, no bound, otherwise (a bound of one CTA lets the
// compiler spend more registers on the one-row-at-a-time loop, measured slower).
template <int T, int NCH>
constexpr int act_min_ctas() {
  return T >= 256 ? 2 : 0;
}

template <int T, int NCH, bool FULL>
__global__ void __launch_bounds__(T, act_min_ctas<T, NCH>()) k_act_rows_bulk(const RowArgs a, uint32_t* status,
                                                                              uint64_t budget) {
  rows_bulk<MODE_ACT, T, NCH, FULL>(a, status, budget);
}

template <int T, int NCH, bool FULL>
__global__ void __launch_bounds__(T) k_weight_rows_bulk(const RowArgs a, uint32_t* status, uint64_t budget) {
  rows_bulk<MODE_WEIGHT, T, NCH, FULL>(a, status, budget);
}

// =========================================================================
// Second phase of producer-side quantization at the next linear's per-token
// scale.  The producing GEMM wrote a = fp16 y (ReLU applied) and, per row,
// the maxima of |fp32(a) * inv_s| over groups of columns; here a row's range
// is the maximum of its groups (exact, order-free), and every element is
// coded at that scale: x = fp32(a) * inv_s, q = code(x * (1 / scale)) -- the
// same values and the same codes as the activation kernel's inv_s path.  One
// warp per row (grid-stride), no block barrier: each lane issues the loads of
// up to kQChunks chunks of 8 columns (16 bytes of a each) before the warp
// reduces the row's group maxima with one unsigned max of their bit patterns
// (they are >= 0 and NaN-free), so the data is in flight meanwhile; longer
// rows take further batches.  The codes go through the NaN-safe path (a NaN x
// is coded 0; an Inf range gives scale Inf, reciprocal 0, codes 0).
// =========================================================================
constexpr int kQWarps = 8;    // rows in flight per CTA
constexpr int kQChunks = 16;  // 8-column chunks per lane per batch (4096 columns per warp)

__global__ void __launch_bounds__(32 * kQWarps) k_quant_partial_rows(const __half* a, int64_t M, int64_t N,
                                                                     const float* part, int64_t part_n,
                                                                     const float* inv_s, int8_t* q, float* scale) {
  griddep_wait();  // a and the partial maxima come from the GEMM just before
  griddep_launch_dependents();
  const int lane = threadIdx.x & 31;
  const int64_t Nc = N >> 3;
  const int64_t nwarps = static_cast<int64_t>(gridDim.x) * kQWarps;
  for (int64_t r = static_cast<int64_t>(blockIdx.x) * kQWarps + (threadIdx.x >> 5); r < M; r += nwarps) {
    const uint4* src = reinterpret_cast<const uint4*>(a + r * N);
    int8_t* dst = q + r * N;
    uint4 v[kQChunks];
    auto load = [&](int64_t b0) {
#pragma unroll
      for (int i = 0; i < kQChunks; ++i) {
        const int64_t c = b0 + lane + 32 * i;
        v[i] = c < Nc ? ld_stream(src + c) : make_uint4(0, 0, 0, 0);
      }
    };
    load(0);
    uint32_t mb = 0;
    for (int64_t i = lane; i < part_n; i += 32) mb = max(mb, __float_as_uint(__ldg(part + r * part_n + i)));
    const float m = __uint_as_float(warp_max_u32(mb));
    const float sc = __fdiv_rn(m, 127.0f);
    const float inv = sc > 0.0f ? __frcp_rn(sc) : 0.0f;
    if (lane == 0) scale[r] = sc;
    for (int64_t b0 = 0; b0 < Nc; b0 += 32 * kQChunks) {
      if (b0 > 0) load(b0);
#pragma unroll
      for (int i = 0; i < kQChunks; ++i) {
        const int64_t c = b0 + lane + 32 * i;
        if (c < Nc) {
          float x[8];
          unpack8(v[i], x);
          if (inv_s != nullptr) {
            float is[8];
            load8f(inv_s + c * 8, is);
#pragma unroll
            for (int j = 0; j < 8; ++j) x[j] = __fmul_rn(x[j], is[j]);
          }
          *reinterpret_cast<uint2*>(dst + c * 8) = pack8<true>(x, inv);
        }
      }
    }
  }
}

// ------------------------------------------------------------- launch ----
template <typename Kern>
int occupancy(Kern k, int threads, size_t smem) {
  int n = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, k, threads, smem) != cudaSuccess) {
    cudaGetLastError();
    n = 1;
  }
  return n > 0 ? n : 1;
}

template <int MODE, int NW>
cudaError_t launch_warp(const RowArgs& a, const Ctx& c) {
  static int occ[64] = {0};
  const int dev = c.device < 64 ? c.device : 63;
  if (occ[dev] == 0) occ[dev] = occupancy(k_rows_warp<MODE, NW>, kWarpThreads, 0);
  int64_t grid = static_cast<int64_t>(c.num_sms) * occ[dev];
  const int64_t need = (a.rows + 3) / 4;  // 4 row-warps per CTA
  if (grid > need) grid = need;
  return launch_pdl(k_rows_warp<MODE, NW>, dim3(static_cast<unsigned>(grid)), dim3(kWarpThreads), 0,
                    c.stream, a);
}

template <int MODE, int T, int NCH, bool PF>
cudaError_t launch_cta(const RowArgs& a, const Ctx& c) {
  static int occ[64] = {0};
  const int dev = c.device < 64 ? c.device : 63;
  if (occ[dev] == 0) occ[dev] = occupancy(k_rows_cta<MODE, T, NCH, PF>, T, 0);
  int64_t grid = static_cast<int64_t>(c.num_sms) * occ[dev];
  if (grid > a.rows) grid = a.rows;
  return launch_pdl(k_rows_cta<MODE, T, NCH, PF>, dim3(static_cast<unsigned>(grid)), dim3(T), 0, c.stream, a);
}

template <int MODE>
cudaError_t launch_mode(const RowArgs& a, const Ctx& c) {
  const int64_t Kc = a.K / 8;
  if (Kc <= 32) return launch_warp<MODE, 1>(a, c);
  if (Kc <= 64) return launch_warp<MODE, 2>(a, c);
  if (Kc <= 128) return launch_warp<MODE, 4>(a, c);
  if (Kc <= 256) return launch_cta<MODE, 64, 4, true>(a, c);
  if (Kc <= 512) return launch_cta<MODE, 128, 4, true>(a, c);
  if (Kc <= 1024) return launch_cta<MODE, 256, 4, true>(a, c);
  if (Kc <= 1536) return launch_cta<MODE, 256, 6, true>(a, c);
  if (Kc <= 2048) return launch_cta<MODE, 256, 8, true>(a, c);
  if (Kc <= 3072) return launch_cta<MODE, 256, 12, false>(a, c);
  if (Kc <= 6144) return launch_cta<MODE, 256, 24, false>(a, c);
  return launch_cta<MODE, 256, 0, false>(a, c);
}

// Calibration grids: a multiple of the cluster size.
int64_t calib_grid(int64_t want, int64_t cap) {
  cap = (cap / kCluster) * kCluster;
  if (cap < kCluster) cap = kCluster;
  if (want > cap) want = cap;
  return ((want + kCluster - 1) / kCluster) * kCluster;
}

template <int NW>
cudaError_t launch_calib_warp(const RowArgs& a, const Ctx& c) {
  const size_t smem = static_cast<size_t>(a.K) * 4;
  const int64_t grid = calib_grid((a.rows + 3) / 4, 4 * static_cast<int64_t>(c.num_sms));
  return launch_pdl(k_calib_warp<NW>, dim3(static_cast<unsigned>(grid)), dim3(kWarpThreads), smem,
                    c.stream, a);
}

template <int T, int NCH>
cudaError_t launch_calib_cta(const RowArgs& a, const Ctx& c) {
  const size_t smem = static_cast<size_t>(a.K) * 4;
  static bool attr[64] = {false};
  const int dev = c.device < 64 ? c.device : 63;
  if (!attr[dev]) {
    cudaError_t e = cudaFuncSetAttribute(k_calib_cta<T, NCH>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         NCH * 8 * T * 4);
    if (e != cudaSuccess) return e;
    attr[dev] = true;
  }
  // one or two rows per CTA, at most a few CTAs per SM
  const int64_t grid = calib_grid((a.rows + 1) / 2, 4 * static_cast<int64_t>(c.num_sms));
  return launch_pdl(k_calib_cta<T, NCH>, dim3(static_cast<unsigned>(grid)), dim3(T), smem, c.stream, a);
}

}  // namespace

template <int MODE, int T, int NCH, bool FULL>
cudaError_t launch_rows_bulk_k(const RowArgs& a, const Ctx& c) {
  constexpr auto kern = MODE == MODE_ACT ? k_act_rows_bulk<T, NCH, FULL> : k_weight_rows_bulk<T, NCH, FULL>;
  static int occ[64] = {0};
  static int64_t occ_bytes[64] = {0};
  const int dev = c.device < 64 ? c.device : 63;
  const size_t smem = static_cast<size_t>(a.K) * 4;  // two slots of one fp16 row
  if (occ_bytes[dev] != static_cast<int64_t>(smem)) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    occ[dev] = occupancy(kern, T, smem);
    occ_bytes[dev] = static_cast<int64_t>(smem);
  }
  int64_t grid = static_cast<int64_t>(c.num_sms) * occ[dev];
  if (grid > a.rows) grid = a.rows;
  return launch_pdl(kern, dim3(static_cast<unsigned>(grid)), dim3(T), smem, c.stream, a, c.status, c.budget_ns);
}

template <int MODE, int T, int NCH>
cudaError_t launch_rows_bulk(const RowArgs& a, const Ctx& c) {
  if (a.K == 8 * NCH * T) return launch_rows_bulk_k<MODE, T, NCH, true>(a, c);
  return launch_rows_bulk_k<MODE, T, NCH, false>(a, c);
}

// Rows streamed by bulk copies, for per-row dynamic scales (no fixed range, no
// range pass) and 1024 < K <= 16384: 4 to 8 chunks of 8 values per thread and
// as few threads per row as that allows (the per-row reductions and the
// LayerNorm statistics' finalization are amortized over more elements).
template <int MODE>
cudaError_t launch_bulk_or(const RowArgs& a, const Ctx& c) {
  const int64_t Kc = a.K / 8;
  if (a.range_in == nullptr && a.range_out == nullptr && Kc > 128 && Kc <= 2048) {
    if (Kc <= 256) return Kc <= 192 ? launch_rows_bulk<MODE, 32, 6>(a, c) : launch_rows_bulk<MODE, 32, 8>(a, c);
    if (Kc <= 512) return Kc <= 384 ? launch_rows_bulk<MODE, 64, 6>(a, c) : launch_rows_bulk<MODE, 128, 4>(a, c);
    if (Kc <= 1024)
      return Kc <= 768 ? launch_rows_bulk<MODE, 128, 6>(a, c) : launch_rows_bulk<MODE, 128, 8>(a, c);
    return Kc <= 1536 ? launch_rows_bulk<MODE, 256, 6>(a, c) : launch_rows_bulk<MODE, 256, 8>(a, c);
  }
  return launch_mode<MODE>(a, c);
}

cudaError_t launch_ln_quant_act(const RowArgs& a, const Ctx& c) { return launch_bulk_or<MODE_ACT>(a, c); }

cudaError_t launch_quant_partial_rows(const __half* a, int64_t M, int64_t N, const float* part, int64_t part_n,
                                      const float* inv_s, int8_t* q, float* scale, const Ctx& c) {
  int64_t grid = (M + kQWarps - 1) / kQWarps;
  const int64_t cap = 16 * static_cast<int64_t>(c.num_sms);
  if (grid > cap) grid = cap;
  return launch_pdl(k_quant_partial_rows, dim3(static_cast<unsigned>(grid)), dim3(32 * kQWarps), 0, c.stream, a, M,
                    N, part, part_n, inv_s, q, scale);
}

cudaError_t launch_quantize_weight(const RowArgs& a, const Ctx& c) { return launch_bulk_or<MODE_WEIGHT>(a, c); }

cudaError_t launch_calibrate_ln(const RowArgs& a, const Ctx& c) {
  const int64_t Kc = a.K / 8;
  if (Kc <= 32) return launch_calib_warp<1>(a, c);
  if (Kc <= 64) return launch_calib_warp<2>(a, c);
  if (Kc <= 128) return launch_calib_warp<4>(a, c);
  if (Kc <= 256) return launch_calib_cta<64, 4>(a, c);
  if (Kc <= 512) return launch_calib_cta<128, 4>(a, c);
  if (Kc <= 1024) return launch_calib_cta<256, 4>(a, c);
  if (Kc <= 2048) return launch_calib_cta<256, 8>(a, c);
  static int occ[64] = {0};
  const int dev = c.device < 64 ? c.device : 63;
  if (occ[dev] == 0) occ[dev] = occupancy(k_calib_cta_atomic, kCtaThreads, 0);
  int64_t grid = static_cast<int64_t>(c.num_sms) * occ[dev];
  if (grid > a.rows) grid = a.rows;
  return launch_pdl(k_calib_cta_atomic, dim3(static_cast<unsigned>(grid)), dim3(kCtaThreads), 0, c.stream, a);
}

}  // namespace sq
