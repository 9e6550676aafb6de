// k_gemm_splitk.cu -- the W8A8 linear for decode-sized token counts
// (M <= 32), where the layer is bound by streaming the INT8 weight from HBM
// (the explainer's "decoding stage"), and for up to 128 tokens on layers too
// narrow for the tiled kernel's 128 x 256 tiles to cover the SMs.
//
// Swap-AB: the MMA's 128-row M slot takes 128 weight rows (output channels)
// and its N slot takes the BT (16, 32, 64 or 128) zero-padded tokens, so
//   TMEM lane = output channel n,  TMEM column = token t.
// Persistent grid of one CTA per SM; a unit is a (channel tile, 256-byte K
// span).  Each CTA streams its units back to back, so its TMA stream never
// drains at tile boundaries, and the units are balanced across CTAs: equal
// numbers of whole tiles, plus an equal share (stream-K) of the remaining
// tiles, which every CTA processes first.  A tile split between CTAs is summed exactly:
// each contributor writes its int32 partial accumulator to the workspace and
// the last to arrive (per-tile counter, no waiting) adds the others and runs
// the epilogue y = fp16((acc * sx[t]) * sw[n] + bias[n]).  int32 addition is
// associative, so the result is bit-identical to a single-CTA sum.
//
// Roles: warp 0 TMA producer (a 5-deep ring for up to 32 tokens, 4- and 3-deep for 64 and
// 128; a stage is two K-consecutive 16 KB weight boxes + two BT x 128 B token boxes),
// warp 1 TMEM owner + MMA issuer (double-buffered accumulators), warps 2-5 epilogue.
// All waits are bounded.
#include "sq_internal.h"
#include "sq_ptx.cuh"
#include "sq_tmap.h"

namespace sq {
namespace {

constexpr int BW = 128;  // weight rows (output channels) per tile
constexpr int BK = 128;  // K bytes per swizzled box
constexpr int KPS = 2;   // consecutive K boxes per unit (per pipeline stage)
constexpr int kThreads = 192;

template <int BT>
struct SkLayout {
  static constexpr int STAGES = BT <= 32 ? 5 : BT == 64 ? 4 : 3;  // about 192-200 KB of ring
  static constexpr int A_BYTES = BW * BK * KPS;  // 2 x 16 KB weight boxes
  static constexpr int B_BYTES = BT * BK * KPS;  // 2 token boxes
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr int kStages = STAGES;
  static constexpr int CTRL = kStages * STAGE_BYTES;
  static constexpr int NBARS = 2 * kStages + 5;  // full, empty, acc_full[2], acc_empty[2], drain
  static constexpr int SLOT = CTRL + NBARS * 8;  // TMEM address, abort, last, decision[2]
  static constexpr int SX = SLOT + 32;           // sx[BT]
  static constexpr int BYTES = SX + BT * 4;
  static constexpr size_t SMEM = BYTES + 1024;
  static constexpr int TMEM_COLS = 2 * BT < 32 ? 32 : 2 * BT;
  static_assert(BT == 16 || BT == 32 || BT == 64 || BT == 128, "token tile of the MMA's N slot");
  static_assert(SX + BT * 4 + 1024 <= 232448, "shared memory per CTA");
};

// Work split.  With T channel tiles on `grid` CTAs, every CTA owns Wt =
// T / grid whole tiles (the last tiles, processed last); the remaining R
// tiles are cut stream-K style: their U = R * KB units are split into equal
// contiguous ranges over the first G CTAs, which process that share first.
// Tiles shared between CTAs are therefore summed early in the kernel, and
// every CTA ends on whole tiles that need no cross-CTA fix-up.
struct SkGeom {
  int64_t U;   // stream-K units = R * KB
  int KB;      // units (KPS boxes of 128 K bytes) per tile
  int G;       // CTAs sharing the stream-K region (>= 1)
  int R;       // tiles 0 .. R-1 are split stream-K style
  int Wt;      // whole tiles per CTA: tiles R + c * Wt .. R + c * Wt + Wt - 1
  int grid;    // CTAs launched
  __device__ __forceinline__ int64_t u0(int c) const { return (static_cast<int64_t>(c) * U) / G; }
  __device__ __forceinline__ int cta_of(int64_t u) const {
    return static_cast<int>(((u + 1) * G - 1) / U);
  }
};

template <int BT>
__device__ __forceinline__ void tmem_ld_tokens(uint32_t taddr, uint32_t (&v)[BT]);

template <>
__device__ __forceinline__ void tmem_ld_tokens<32>(uint32_t taddr, uint32_t (&v)[32]) {
  tmem_ld_32x32b_x32(taddr, v);
}

template <>
__device__ __forceinline__ void tmem_ld_tokens<16>(uint32_t taddr, uint32_t (&v)[16]) {
  tmem_ld_32x32b_x16(taddr, v);
}

// 64 and 128 tokens: 32-column loads, each chunk's registers tied to the wait
template <>
__device__ __forceinline__ void tmem_ld_tokens<64>(uint32_t taddr, uint32_t (&v)[64]) {
  uint32_t(&a)[32] = *reinterpret_cast<uint32_t(*)[32]>(&v[0]);
  uint32_t(&b)[32] = *reinterpret_cast<uint32_t(*)[32]>(&v[32]);
  tmem_ld_32x32b_x32(taddr, a);
  tmem_ld_32x32b_x32(taddr + 32u, b);
  tmem_ld_wait_regs(a);
  tmem_ld_wait_regs(b);
}

template <>
__device__ __forceinline__ void tmem_ld_tokens<128>(uint32_t taddr, uint32_t (&v)[128]) {
#pragma unroll
  for (int c = 0; c < 4; ++c)
    tmem_ld_32x32b_x32(taddr + 32u * c, *reinterpret_cast<uint32_t(*)[32]>(&v[32 * c]));
#pragma unroll
  for (int c = 0; c < 4; ++c) tmem_ld_wait_regs(*reinterpret_cast<uint32_t(*)[32]>(&v[32 * c]));
}

// EPI: 0 = fp16 y, 1 = int32 accumulators, 2 = the next linear's INT8 codes
// at its static scale (producer-side quantization), 3 = the first phase of
// producer-side quantization at the next linear's per-token scale: fp16
// a = y (ReLU if asked) and per token the maximum of |a * inv_s_next| over
// each warp's 32 channels.
template <int BT, int EPI>
__global__ void __launch_bounds__(kThreads, 1)
    k_gemm_splitk(const __grid_constant__ CUtensorMap tmW, const __grid_constant__ CUtensorMap tmX,
                  const GemmArgs g, const SkGeom geo, uint32_t* counters, int32_t* partials,
                  uint32_t* status, uint64_t budget) {
  constexpr bool OUT_I32 = EPI == 1;
  using L = SkLayout<BT>;
  constexpr int kStages = L::STAGES;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  const uint32_t sbase = smem_u32(smem);
  const uint32_t sA = sbase;
  const uint32_t sB = sbase + kStages * L::A_BYTES;
  const uint32_t bar0 = sbase + L::CTRL;
  auto full_bar = [&](int s) { return bar0 + 8u * s; };
  auto empty_bar = [&](int s) { return bar0 + 8u * (kStages + s); };
  auto accf_bar = [&](int b) { return bar0 + 8u * (2 * kStages + b); };
  auto acce_bar = [&](int b) { return bar0 + 8u * (2 * kStages + 2 + b); };
  const uint32_t drain_bar = bar0 + 8u * (2 * kStages + 4);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::SLOT);
  volatile uint32_t* abort_flag = tmem_slot + 1;
  volatile uint32_t* last_flag = tmem_slot + 2;
  volatile uint32_t* decision = tmem_slot + 3;  // [2]
  float* sx_s = reinterpret_cast<float*>(smem + L::SX);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int cta = blockIdx.x;
  const int64_t ubeg = cta < geo.G ? geo.u0(cta) : 0;
  const int64_t uend = cta < geo.G ? geo.u0(cta + 1) : 0;
  const int KB = geo.KB;
  const int64_t n_sk = uend - ubeg;                                 // stream-K units of this CTA
  const int64_t n_all = n_sk + static_cast<int64_t>(geo.Wt) * KB;  // then its whole tiles
  const int64_t wt0 = geo.R + static_cast<int64_t>(cta) * geo.Wt;  // first whole tile
  // position j of this CTA's unit sequence -> (tile, unit within the tile)
  auto unit_of = [&](int64_t j, int64_t& t, int& kb) {
    if (j < n_sk) {
      const int64_t u = ubeg + j;
      t = u / KB;
      kb = static_cast<int>(u % KB);
    } else {
      const int64_t w = j - n_sk;
      t = wt0 + w / KB;
      kb = static_cast<int>(w % KB);
    }
  };

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(full_bar(s), 1);
      mbar_init(empty_bar(s), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(accf_bar(b), 1);
      mbar_init(acce_bar(b), 4);  // one arrive per epilogue warp
    }
    mbar_init(drain_bar, 1);
    *abort_flag = 0;
    fence_barrier_init();
    tma_prefetch_desc(&tmW);
    tma_prefetch_desc(&tmX);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), L::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  griddep_wait();  // inputs and workspace are written by earlier kernels

  int64_t issued = 0;
  bool mma_any = false;

  if (warp == 0) {
    if (lane == 0) {
      const uint64_t pol_w = l2_policy_evict_first();  // each weight byte is read once
      const uint64_t pol_x = l2_policy_evict_last();   // every CTA re-reads the tokens
      for (int64_t i = 0; i < n_all; ++i) {
        const int s = static_cast<int>(i % kStages);
        const int64_t r = i / kStages;
        if (i >= kStages && !mbar_wait(empty_bar(s), static_cast<uint32_t>((r - 1) & 1), budget, status, abort_flag))
          break;
        int64_t t;
        int kb;
        unit_of(i, t, kb);
        mbar_arrive_expect_tx(full_bar(s), L::STAGE_BYTES);  // boxes past K arrive zero-filled
#pragma unroll
        for (int p = 0; p < KPS; ++p) {
          const int32_t kx = (kb * KPS + p) * BK;
          tma_load_2d_hint(sA + s * L::A_BYTES + p * (BW * BK), &tmW, full_bar(s), kx,
                           static_cast<int32_t>(t * BW), pol_w);
          tma_load_2d_hint(sB + s * L::B_BYTES + p * (BT * BK), &tmX, full_bar(s), kx, 0, pol_x);
        }
        ++issued;
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_i8(BW, BT);
      int seg = 0;
      int b = 0;
      for (int64_t i = 0; i < n_all; ++i) {
        const int s = static_cast<int>(i % kStages);
        const int64_t r = i / kStages;
        int64_t t;
        int kb;
        unit_of(i, t, kb);
        const bool first = i == 0 || i == n_sk || kb == 0;
        const bool last = i == n_sk - 1 || i == n_all - 1 || kb == KB - 1;
        if (first) {
          b = seg & 1;
          if (seg >= 2 && !mbar_wait(acce_bar(b), static_cast<uint32_t>(((seg >> 1) - 1) & 1), budget, status, abort_flag))
            break;
        }
        if (!mbar_wait(full_bar(s), static_cast<uint32_t>(r & 1), budget, status, abort_flag)) break;
        tc_fence_after();
        const uint32_t d = tmem + static_cast<uint32_t>(b * BT);
#pragma unroll
        for (int p = 0; p < KPS; ++p) {
          const uint64_t ad = sdesc_k_sw128(sA + s * L::A_BYTES + p * (BW * BK));
          const uint64_t bd = sdesc_k_sw128(sB + s * L::B_BYTES + p * (BT * BK));
#pragma unroll
          for (int k = 0; k < BK / 32; ++k)
            mma_i8(d, ad + 2u * k, bd + 2u * k, idesc, (first && p == 0 && k == 0) ? 0u : 1u);
        }
        mma_any = true;
        mma_commit(empty_bar(s));
        if (last) {
          mma_commit(accf_bar(b));
          ++seg;
        }
      }
      griddep_launch_dependents();
    }
  } else {
    const int et = threadIdx.x - 64;
    const int q = warp & 3;
    if (!OUT_I32 && et < BT) sx_s[et] = et < g.M ? g.sx[et] : 0.0f;
    float q_inv = 0.0f;
    if constexpr (EPI == 2) {
      const float q_sc = __fdiv_rn(*g.range_next, 127.0f);
      q_inv = q_sc > 0.0f ? __frcp_rn(q_sc) : 0.0f;
      if (blockIdx.x == 0 && et < BT && et < g.M) g.sx_next[et] = q_sc;
    }
    named_bar_sync(1, 128);
    int seg = 0;
    for (int64_t j = 0; j < n_all;) {
      int64_t t, tile_end = 0, seglen;
      bool whole;
      int slot = 0;
      if (j < n_sk) {  // a piece of a stream-K tile
        const int64_t u = ubeg + j;
        t = u / KB;
        tile_end = (t + 1) * KB;
        const int64_t seg_end = uend < tile_end ? uend : tile_end;
        whole = (u == t * KB) && (seg_end == tile_end);
        slot = (j == 0) ? 0 : 1;
        seglen = seg_end - u;
      } else {  // one of this CTA's whole tiles
        t = wt0 + (j - n_sk) / KB;
        whole = true;
        seglen = KB;
      }
      const int b = seg & 1;
      mbar_wait(accf_bar(b), static_cast<uint32_t>((seg >> 1) & 1), budget, status, abort_flag);
      // one thread decides whether to stop and broadcasts it (double-buffered by
      // segment parity), so every epilogue thread leaves the loop at the same point
      if (et == 0) decision[seg & 1] = *abort_flag;
      named_bar_sync(1, 128);
      if (decision[seg & 1]) break;
      tc_fence_after();
      uint32_t v[BT];
      tmem_ld_tokens<BT>(tmem + (static_cast<uint32_t>(32 * q) << 16) + static_cast<uint32_t>(b * BT), v);
      tmem_ld_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(acce_bar(b));

      const int64_t nl = 32 * q + lane;  // channel within the tile
      const int64_t n = t * BW + nl;
      bool emit = whole;
      // a partial slot holds BW x BT int32 as BT/4 groups of [channel][4 tokens]:
      // a warp's 16-byte stores and loads of one group cover 512 contiguous bytes
      auto part = [&](int64_t sl, int j) { return partials + (sl * BT + j) * BW + nl * 4; };
      if (!whole) {
#pragma unroll
        for (int j = 0; j < BT; j += 4)
          *reinterpret_cast<int4*>(part(2 * cta + slot, j)) =
              make_int4(static_cast<int>(v[j]), static_cast<int>(v[j + 1]), static_cast<int>(v[j + 2]),
                        static_cast<int>(v[j + 3]));
        __threadfence();
        named_bar_sync(1, 128);
        const int c_lo = geo.cta_of(t * KB);
        const int c_hi = geo.cta_of(tile_end - 1);
        if (et == 0) {
          const uint32_t prev = atomicAdd(counters + t, 1u);
          const bool is_last = prev == static_cast<uint32_t>(c_hi - c_lo);
          if (is_last) counters[t] = 0;  // every contributor has arrived: reset for the next call
          *last_flag = is_last ? 1u : 0u;
        }
        named_bar_sync(1, 128);
        emit = *last_flag != 0;
        if (emit) {
          __threadfence();
          for (int cc = c_lo; cc <= c_hi; ++cc) {
            if (cc == cta) continue;
            const int first_tile = static_cast<int>(geo.u0(cc) / KB);
            const int sl = (t == first_tile) ? 0 : 1;
#pragma unroll
            for (int j = 0; j < BT; j += 4) {
              const int4 p = __ldcg(reinterpret_cast<const int4*>(part(2 * cc + sl, j)));
              v[j] += p.x;
              v[j + 1] += p.y;
              v[j + 2] += p.z;
              v[j + 3] += p.w;
            }
          }
        }
      }
      if (EPI == 3 && emit) {
        // a = relu ? max(y, 0) : y (a NaN becomes 0), written as fp16; per
        // token the maximum of |fp32(a) * inv_s_next[n]| over this warp's 32
        // channels (NaN-free; channels past N give 0) -> part[m][n / 32]
        const bool in_n = n < g.N;
        const float swn = in_n ? g.sw[n] : 0.0f;
        const bool has_bias = g.bias != nullptr;
        const float bn = (has_bias && in_n) ? __half2float(g.bias[n]) : 0.0f;
        const float isn = !in_n ? 0.0f : g.inv_s_next != nullptr ? g.inv_s_next[n] : 1.0f;
        const int64_t grp = (t * BW + 32 * q) / 32;
#pragma unroll
        for (int m = 0; m < BT; ++m) {
          if (m < g.M) {  // warp-uniform
            float f = dequant_f32(static_cast<int32_t>(v[m]), sx_s[m], swn);
            if (has_bias) f = __fadd_rn(f, bn);
            __half hv = __float2half_rn(f);
            if (g.relu && !(__half2float(hv) > 0.0f)) hv = __float2half_rn(0.0f);
            if (in_n) g.y[m * g.N + n] = hv;
            float p = fabsf(__fmul_rn(__half2float(hv), isn));
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) p = fmaxf(p, __shfl_xor_sync(0xffffffffu, p, o));
            if (lane == 0 && grp < g.part_n) g.part[m * g.part_n + grp] = p;
          }
        }
      } else if (emit && n < g.N) {
        if (OUT_I32) {
          for (int m = 0; m < BT; ++m)
            if (m < g.M) g.acc[m * g.N + n] = static_cast<int32_t>(v[m]);
        } else if (EPI == 2) {
          // y = fp16((acc * sx) * sw + bias), a = relu ? max(y, 0) : y,
          // code = clamp(rint(a * inv_s_next[n] * (1 / scale)), -127, 127)
          const float swn = g.sw[n];
          const bool has_bias = g.bias != nullptr;
          const float bn = has_bias ? __half2float(g.bias[n]) : 0.0f;
          const float isn = g.inv_s_next != nullptr ? g.inv_s_next[n] : 1.0f;
#pragma unroll
          for (int m = 0; m < BT; ++m) {
            if (m < g.M) {
              float f = dequant_f32(static_cast<int32_t>(v[m]), sx_s[m], swn);
              if (has_bias) f = __fadd_rn(f, bn);
              float a = __half2float(__float2half_rn(f));
              if (g.relu && !(a > 0.0f)) a = 0.0f;
              float p = __fmul_rn(__fmul_rn(a, isn), q_inv);
              if (p != p) p = 0.0f;
              p = p > 127.0f ? 127.0f : p;
              p = p < -127.0f ? -127.0f : p;
              g.q_next[m * g.N + n] = static_cast<int8_t>(__float_as_uint(__fadd_rn(p, 12582912.0f)) & 0xFFu);
            }
          }
        } else {
          const float swn = g.sw[n];
          const bool has_bias = g.bias != nullptr;
          const float bn = has_bias ? __half2float(g.bias[n]) : 0.0f;
#pragma unroll
          for (int m = 0; m < BT; ++m) {
            if (m < g.M) {
              float f = dequant_f32(static_cast<int32_t>(v[m]), sx_s[m], swn);
              if (has_bias) f = __fadd_rn(f, bn);
              g.y[m * g.N + n] = __float2half_rn(f);
            }
          }
        }
      }
      j += seglen;
      ++seg;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (*abort_flag) {
    if (warp == 1 && lane == 0 && mma_any) {
      mma_commit(drain_bar);
      mbar_drain(drain_bar, 0, budget);
    }
    if (warp == 0 && lane == 0) {
      for (int s = 0; s < kStages && s < issued; ++s) {
        const int64_t last = ((issued - 1 - s) / kStages) * kStages + s;
        mbar_drain(full_bar(s), static_cast<uint32_t>((last / kStages) & 1), budget);
      }
    }
    __syncthreads();
  }
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, L::TMEM_COLS);
  }
}

int64_t tiles_of(int64_t N) { return (N + BW - 1) / BW; }

SkGeom make_geom(int64_t N, int64_t K, int64_t grid_cap) {
  SkGeom geo;
  geo.KB = static_cast<int>(((K + BK - 1) / BK + KPS - 1) / KPS);
  const int64_t T = tiles_of(N);
  const int64_t total = T * geo.KB;
  // at least half a tile of K per CTA, so a split tile has at most three
  // contributors and its last arrival adds at most two partials (on small
  // layers fewer CTAs then stream the weight; each still keeps a deep ring)
  const int64_t min_units = (geo.KB + 1) / 2;
  const int64_t by_units = (total + min_units - 1) / min_units;
  int64_t grid = total < grid_cap ? total : grid_cap;
  if (grid > by_units) grid = by_units;
  geo.grid = static_cast<int>(grid);
  geo.Wt = static_cast<int>(T / grid);
  geo.R = static_cast<int>(T - static_cast<int64_t>(geo.Wt) * grid);
  geo.U = static_cast<int64_t>(geo.R) * geo.KB;
  geo.G = geo.U > 0 ? static_cast<int>(geo.U < grid ? geo.U : grid) : 1;
  return geo;
}

template <int BT, int EPI>
cudaError_t launch_bt(const GemmArgs& g, const Ctx& c) {
  using L = SkLayout<BT>;
  static bool attr_set[64] = {false};
  const int dev = c.device < 64 ? c.device : 63;
  if (!attr_set[dev]) {
    cudaError_t e = cudaFuncSetAttribute(k_gemm_splitk<BT, EPI>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(L::SMEM));
    if (e != cudaSuccess) return e;
    attr_set[dev] = true;
  }
  CUtensorMap tmW, tmX;
  if (!make_tmap_i8(&tmW, g.wq, g.K, g.N, BK, BW)) return cudaErrorInvalidValue;
  if (!make_tmap_i8(&tmX, g.xq, g.K, g.M, BK, BT)) return cudaErrorInvalidValue;
  const SkGeom geo = make_geom(g.N, g.K, c.num_sms);
  uint8_t* ws = static_cast<uint8_t*>(g.ws);
  const size_t counter_bytes = ((tiles_of(g.N) * 4 + 255) / 256) * 256;
  uint32_t* counters = reinterpret_cast<uint32_t*>(ws);
  int32_t* partials = reinterpret_cast<int32_t*>(ws + counter_bytes);
  return launch_pdl(k_gemm_splitk<BT, EPI>, dim3(geo.grid), dim3(kThreads), L::SMEM, c.stream, tmW, tmX,
                    g, geo, counters, partials, c.status, c.budget_ns);
}

}  // namespace

size_t splitk_workspace_bytes(int64_t M, int64_t N, int64_t K, int num_sms) {
  (void)K;
  const int64_t bt = M <= 16 ? 16 : M <= 32 ? 32 : M <= 64 ? 64 : 128;
  const size_t counter_bytes = ((tiles_of(N) * 4 + 255) / 256) * 256;
  return counter_bytes + static_cast<size_t>(2) * num_sms * BW * bt * 4;
}

cudaError_t launch_gemm_splitk(const GemmArgs& g, const Ctx& c) {
  const int epi = g.acc != nullptr ? 1 : g.q_next != nullptr ? 2 : g.part != nullptr ? 3 : 0;
  if (epi == 3) {  // per-token producer-side quantization: decode token counts only
    if (g.M <= 16) return launch_bt<16, 3>(g, c);
    if (g.M <= 32) return launch_bt<32, 3>(g, c);
    return cudaErrorInvalidValue;
  }
  if (g.M <= 16) return epi == 1 ? launch_bt<16, 1>(g, c) : epi == 2 ? launch_bt<16, 2>(g, c) : launch_bt<16, 0>(g, c);
  if (g.M <= 32) return epi == 1 ? launch_bt<32, 1>(g, c) : epi == 2 ? launch_bt<32, 2>(g, c) : launch_bt<32, 0>(g, c);
  if (g.M <= 64) return epi == 1 ? launch_bt<64, 1>(g, c) : epi == 2 ? launch_bt<64, 2>(g, c) : launch_bt<64, 0>(g, c);
  return epi == 1 ? launch_bt<128, 1>(g, c) : epi == 2 ? launch_bt<128, 2>(g, c) : launch_bt<128, 0>(g, c);
}

}  // namespace sq

// ---------------------------------------------------------------------------
// Allocation-free variant of the stream-K linear.
//
// Some callers cannot allocate device memory at all: a plug-in running inside
// another runtime that owns every device allocation and hands the plug-in
// only its input and output buffers, or a latency-critical path where
// cudaMalloc (which may synchronize the device) is not acceptable.  This
// variant keeps the stream-K scratch (per-tile arrival counters and int32
// partial accumulators) in one fixed array in device global memory, owned by
// the library: every GPU that loads the library holds it until the process
// exits.  Calls share the array and it keeps the last call's contents, so the
// counters are cleared at the start of every call, and two calls whose
// kernels overlap on the GPU (different streams, or different host threads)
// race on it.
#include <mutex>

#include "../../include/sq.h"

namespace sq {
namespace {

constexpr size_t kNoAllocCounterBytes = 4u * SQ_NOALLOC_MAX_TILES;        // one uint32 per tile
constexpr size_t kNoAllocPartialBytes = SQ_NOALLOC_SCRATCH_BYTES - kNoAllocCounterBytes;
static_assert(kNoAllocCounterBytes % 256 == 0, "partials must start 256-byte aligned");

static __device__ __align__(256) uint8_t g_noalloc_scratch[SQ_NOALLOC_SCRATCH_BYTES];

// The counters must start at zero; the array keeps whatever the last call left.
__global__ void k_noalloc_clear_counters(uint32_t n) {
  griddep_wait();  // the previous call's kernels may still be reading them
  griddep_launch_dependents();
  uint32_t* counters = reinterpret_cast<uint32_t*>(g_noalloc_scratch);
  for (uint32_t i = blockIdx.x * blockDim.x + threadIdx.x; i < n; i += gridDim.x * blockDim.x)
    counters[i] = 0;
}

constexpr int kMaxDev = 64;
std::once_flag g_noalloc_once[kMaxDev];
uint8_t* g_noalloc_dev_ptr[kMaxDev];
cudaError_t g_noalloc_setup_err[kMaxDev];

// Device address of the scratch array on the current device.  Host code only
// knows a host-side stand-in for the array's name, so the address is looked
// up once per device (with that device current) and handed to the kernels.
cudaError_t noalloc_scratch(int dev, uint8_t** out) {
  std::call_once(g_noalloc_once[dev], [dev] {
    void* p = nullptr;
    cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess) cudaGetLastError();
    g_noalloc_setup_err[dev] = e;
    g_noalloc_dev_ptr[dev] = static_cast<uint8_t*>(p);
  });
  *out = g_noalloc_dev_ptr[dev];
  return g_noalloc_setup_err[dev];
}

// Same kernel as launch_bt, with the scratch of the fixed array and the grid
// capped to the partial-accumulator slots the array holds.
template <int BT>
cudaError_t launch_noalloc(const GemmArgs& g, const Ctx& c, uint8_t* scratch) {
  using L = SkLayout<BT>;
  static bool attr_set[64] = {false};  // once per device, as in launch_bt
  const int dev = c.device < 64 ? c.device : 63;
  cudaError_t e;
  if (!attr_set[dev]) {
    e = cudaFuncSetAttribute(k_gemm_splitk<BT, 0>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(L::SMEM));
    if (e != cudaSuccess) return e;
    attr_set[dev] = true;
  }
  CUtensorMap tmW, tmX;
  if (!make_tmap_i8(&tmW, g.wq, g.K, g.N, BK, BW)) return cudaErrorInvalidValue;
  if (!make_tmap_i8(&tmX, g.xq, g.K, g.M, BK, BT)) return cudaErrorInvalidValue;
  const int64_t slots = static_cast<int64_t>(kNoAllocPartialBytes / (2ull * BW * BT * 4));
  const SkGeom geo = make_geom(g.N, g.K, c.num_sms < slots ? c.num_sms : slots);
  uint32_t* counters = reinterpret_cast<uint32_t*>(scratch);
  int32_t* partials = reinterpret_cast<int32_t*>(scratch + kNoAllocCounterBytes);
  const uint32_t ntiles = static_cast<uint32_t>(tiles_of(g.N));
  e = launch_pdl(k_noalloc_clear_counters, dim3((ntiles + 255) / 256), dim3(256), 0, c.stream, ntiles);
  if (e != cudaSuccess) return e;
  return launch_pdl(k_gemm_splitk<BT, 0>, dim3(geo.grid), dim3(kThreads), L::SMEM, c.stream, tmW, tmX, g,
                    geo, counters, partials, c.status, c.budget_ns);
}

}  // namespace
}  // namespace sq

extern "C" sq_status sq_w8a8_linear_noalloc(const int8_t* xq, const float* x_scale,
                                            const int8_t* wq, const float* w_scale,
                                            const void* bias_f16, void* y_f16, int64_t M,
                                            int64_t N, int64_t K, sq_stream_t stream) {
  using namespace sq;
  auto a16 = [](const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; };
  if (!xq || !x_scale || !wq || !w_scale || !y_f16) return SQ_ERR_INVALID_ARG;
  if (M <= 0 || N <= 0 || K <= 0) return SQ_ERR_INVALID_ARG;
  if (K > SQ_MAX_K) return SQ_ERR_K_OVERFLOW;
  if (K % 16 != 0 || M > SQ_DECODE_MAX_M) return SQ_ERR_UNSUPPORTED_SHAPE;
  if (tiles_of(N) > SQ_NOALLOC_MAX_TILES) return SQ_ERR_WORKSPACE;  // beyond the fixed scratch
  if (!a16(xq) || !a16(wq) || !a16(x_scale) || !a16(w_scale) || !a16(y_f16) ||
      (bias_f16 && !a16(bias_f16)))
    return SQ_ERR_MISALIGNED;
  Ctx ctx;
  const int st = call_context(stream, &ctx);
  if (st != SQ_OK) return static_cast<sq_status>(st);
  if (ctx.device >= kMaxDev) return SQ_ERR_CUDA;
  uint8_t* scratch = nullptr;
  if (noalloc_scratch(ctx.device, &scratch) != cudaSuccess || scratch == nullptr) return SQ_ERR_CUDA;
  GemmArgs g{};
  g.xq = xq;
  g.sx = x_scale;
  g.wq = wq;
  g.sw = w_scale;
  g.bias = static_cast<const __half*>(bias_f16);
  g.y = static_cast<__half*>(y_f16);
  g.acc = nullptr;
  g.M = M;
  g.N = N;
  g.K = K;
  g.ws = scratch;
  g.ws_bytes = SQ_NOALLOC_SCRATCH_BYTES;
  const cudaError_t e = (M <= 16) ? launch_noalloc<16>(g, ctx, scratch) : launch_noalloc<32>(g, ctx, scratch);
  if (e != cudaSuccess) {
    cudaGetLastError();
    return SQ_ERR_CUDA;
  }
  return SQ_OK;
}
