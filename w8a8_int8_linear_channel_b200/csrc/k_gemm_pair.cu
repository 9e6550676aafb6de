// k_gemm_pair.cu -- the W8A8 linear for large token counts on CTA pairs: INT8
// x INT8 -> INT32 GEMM on the 5th-generation tensor cores (tcgen05.mma
// cta_group::2, kind::i8) with the dequant epilogue fused (glossary "INT8
// GEMM"; section "inference", O1 scales; the quantization tutorial's
// "multiply the scale back").
//
// A cluster of two CTAs (one TPC) computes 256 x 256 output tiles, walking
// them persistently.  Per 128-byte K block each CTA loads 128 token rows of
// xq and 128 of the 256 weight rows of wq (32 KB); one pair MMA of
// 256 x 256 x 32 reads A from both CTAs and B from both halves, so each CTA's
// shared memory serves 64 bytes per tensor-core cycle (half of what a
// single-CTA 128 x 256 MMA reads) and the TMA refill another 64.  Each CTA
// holds its 128 accumulator rows x 256 int32 columns in TMEM, twice (512
// columns), so the epilogue of one tile runs under the MMAs of the next.
//   warp 0      TMA producer of this CTA's halves (a 192 KB ring: 6 stages
//               of one K block, or, for K >= 512, 3 stages of two); the
//               loads of both CTAs complete on the leader's barrier of the
//               stage
//   warp 1      TMEM allocation (both CTAs); in the leader, lane 0 issues the
//               pair MMAs once both CTAs' halves of a stage have landed
//   warps 2-9   epilogue of this CTA's 128 rows: warp w reads TMEM lane
//               quarter w % 4 for column half (w - 2) / 4, computes
//               y = fp16((acc * sx[t]) * sw[n] + bias[n]) and writes 32 x 32
//               blocks through shared memory with TMA stores -- or, for
//               producer-side quantization, turns y into the next linear's
//               INT8 codes at its static scale and writes 32 bytes per row,
//               or (per-token scale) writes fp16 y after the ReLU and each
//               row's maximum of |y * inv_s_next| over its 128 columns
// Every mbarrier wait is bounded; a wait that runs out records a timeout,
// tells the other CTA of the pair to stop, and both CTAs drain what they
// issued, free TMEM and return.
#include <string.h>

#include "sq_internal.h"
#include "sq_ptx.cuh"
#include "sq_tmap.h"

namespace sq {
namespace {

constexpr int BM = 128;  // token rows per CTA (the pair covers 256)
constexpr int BN = 256;  // output channels per tile (each CTA loads 128 weight rows)
constexpr int BNH = BN / 2;
constexpr int BK = 128;  // K bytes per TMA box = one 128-byte swizzle row
constexpr int kEpiWarps = 8;
constexpr int kThreads = 64 + 32 * kEpiWarps;
constexpr int A_BYTES = BM * BK;   // 16 KB
constexpr int B_BYTES = BNH * BK;  // 16 KB
constexpr int RING = 6 * (A_BYTES + B_BYTES);  // 192 KB of pipeline stages
// The ring as 6 stages of one 128-byte K box (short K) or 3 stages of two
// (K >= 512: half the barrier round trips and MMA commits per K byte, which
// measured 5 % faster on 2048 x 4096 x 4096 and 7-8 % on longer grids).  With
// tiles TBN = 128 channels wide (the batched product at N <= 128) each CTA
// loads 64 weight rows per box: 8 stages of one box, 4 of two.
template <int KSUB, int TBN = BN>
struct Ring {
  static constexpr int STAGE_BYTES = KSUB * (A_BYTES + (TBN / 2) * BK);
  static constexpr int STAGES = RING / STAGE_BYTES;
  static_assert(STAGES * STAGE_BYTES == RING && STAGES >= 2 && STAGES <= 8, "ring of whole stages");
};
constexpr int STG = RING;                  // per-epilogue-warp output staging
constexpr int STG_BYTES = 2048;            // one 32 rows x 32 fp16 block, 64-byte swizzle
constexpr int STG_WARP = 2 * STG_BYTES;    // double-buffered per warp
constexpr int CTRL = STG + kEpiWarps * STG_WARP;
// barriers: full[S] (leader: both CTAs' loads landed), empty[S], accf[2],
// acce[2] (leader: both epilogues done), drain; sized for the 8-stage ring
constexpr int NBARS = 2 * 8 + 5;
// TMEM address, abort flag, decision[2], loads issued by the peer
constexpr int SLOT = CTRL + NBARS * 8;
// sw[BN] fp32, bias[BN] fp16 of the current tile, read as 16-byte vectors
constexpr int VEC = (SLOT + 32 + 15) & ~15;
static_assert(VEC % 16 == 0 && (VEC + BN * 4) % 16 == 0, "vector loads of sw and bias");
constexpr int SMEM_BYTES = VEC + BN * 4 + BN * 2;
constexpr size_t SMEM = SMEM_BYTES + 1024;  // slack for 1024-byte alignment
static_assert(SMEM <= 232448, "shared memory per CTA");
constexpr uint32_t TMEM_COLS = 512;

// What the epilogue writes (EPI_BMM: fp16 y of a batched GEMM, 3-D maps;
// EPI_QD: the first phase of the per-token producer-side quantization, fp16
// a = y (ReLU if asked) plus per-row maxima of |a * inv_s_next| per 128
// columns).
enum Epi { EPI_F16 = 0, EPI_I32 = 1, EPI_Q8 = 2, EPI_BMM = 3, EPI_QD = 4 };

// Tile t -> (token tile, channel tile), grouped: groups of kGroupM token
// tiles walk every channel tile, token tile fastest.  The 74 tiles in flight
// at a time then span about 8 token tiles x 9 channel tiles, so each operand
// panel they read is shared by several of them in L2 (token-tile-fastest over
// all token tiles would span 32 x 2.3 tiles for 8192 tokens and re-read every
// token panel from DRAM for each group of channel tiles).
constexpr int kGroupM = 8;

static_assert((kGroupM & (kGroupM - 1)) == 0, "token tiles per group: a power of two");

// n / d for 0 <= n < 2^31 and a divisor d >= 1 fixed for the whole kernel:
// a multiply-high, a subtract, an add and two shifts instead of a division
// sequence (Granlund and Montgomery, "Division by invariant integers using
// multiplication", 1994: the unsigned case with a 33-bit multiplier, m' =
// floor(2^32 (2^l - d) / d) + 1 and l = ceil(log2 d)).
// Built on the host and passed as a kernel parameter (read from the constant
// bank, so it holds no registers).
struct FastDiv {
  uint32_t d, m;
  int l;
  static FastDiv make(uint32_t d_) {
    FastDiv f;
    f.d = d_;
    f.l = 0;
    while (f.l < 32 && (static_cast<uint64_t>(1) << f.l) < d_) ++f.l;  // ceil(log2 d)
    f.m = static_cast<uint32_t>(((static_cast<uint64_t>(1) << 32) * ((static_cast<uint64_t>(1) << f.l) - d_)) / d_ + 1);
    return f;
  }
  __device__ __forceinline__ int div(int n) const {
    if (l == 0) return n;
    const uint32_t u = static_cast<uint32_t>(n);
    const uint32_t t1 = __umulhi(m, u);
    return static_cast<int>((t1 + ((u - t1) >> 1)) >> (l - 1));
  }
};

// Tile t of the grid -> batch item bi (BATCHED only), token tile tm, channel
// tile tn.
struct TileMap {
  FastDiv item;   // tiles per batch item
  FastDiv group;  // tiles per group of kGroupM token tiles (kGroupM * tiles_n)
  int tiles_m;
  static TileMap make(int per_item, int tiles_m_) {
    TileMap t;
    t.item = FastDiv::make(static_cast<uint32_t>(per_item));
    t.group = FastDiv::make(static_cast<uint32_t>(kGroupM * (per_item / tiles_m_)));
    t.tiles_m = tiles_m_;
    return t;
  }
  template <bool BATCHED>
  __device__ __forceinline__ void coords(int t, int& bi, int& tm, int& tn) const {
    bi = BATCHED ? item.div(t) : 0;
    const int u = BATCHED ? t - bi * static_cast<int>(item.d) : t;
    const int gi = group.div(u);
    const int first = gi * kGroupM;
    const int r = u - gi * static_cast<int>(group.d);
    if (tiles_m - first >= kGroupM) {
      tm = first + (r & (kGroupM - 1));
      tn = r / kGroupM;
    } else {  // the last, narrower group
      const int gm = tiles_m - first;
      tm = first + r % gm;
      tn = r / gm;
    }
  }
};

// Bounded wait that, when it runs out, also raises the other CTA's abort
// flag so the pair stops together.  Barriers completed by the other CTA's
// threads (cluster_scope) are polled without suspending.
__device__ __forceinline__ bool pair_wait(uint32_t bar, uint32_t parity, bool cluster_scope,
                                          uint64_t budget_ns, uint32_t* status,
                                          volatile uint32_t* abort, uint32_t peer_abort) {
  auto test = [&]() { return cluster_scope ? mbar_test_wait_cluster(bar, parity) : mbar_try_wait(bar, parity); };
  if (test()) return true;
  const uint64_t t0 = globaltimer_ns();
  while (true) {
    if (test()) return true;
    if (*abort) return false;
    if (globaltimer_ns() - t0 > budget_ns) {
      atomicCAS(status, DEV_OK, DEV_TIMEOUT);
      *abort = 1;
      st_shared_cluster_u32(peer_abort, 1u);
      return false;
    }
  }
}

// TMAS: fp16 blocks leave through TMA stores (rows 16-byte aligned); without
// it they go through the warp's staging, row by row (a separate
// instantiation, so the TMA-store kernel keeps its own registers).
// TBN: channels per tile, 256, or 128 for the batched product at N <= 128
// (P V of attention: a 256-wide tile would be half padding).
template <int EPI, bool TMAS, int KSUB, int TBN = BN>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
    k_gemm_pair(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                const __grid_constant__ CUtensorMap tmY, const GemmArgs g, const TileMap tmap, int tiles,
                uint32_t* status, uint64_t budget) {
  constexpr int STAGES = Ring<KSUB, TBN>::STAGES, STAGE_BYTES = Ring<KSUB, TBN>::STAGE_BYTES;
  static_assert(TBN == BN || (TBN == BN / 2 && EPI == EPI_BMM), "128-wide tiles: the batched product");
  constexpr int TNH = TBN / 2;            // weight rows per CTA
  constexpr int TB_BYTES = TNH * BK;      // one weight box per CTA
  constexpr int CW = TBN / 2;             // columns of a tile per epilogue warp
  constexpr int NB = CW / 32;             // 32-column blocks per epilogue warp
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  const uint32_t sbase = smem_u32(smem);
  const uint32_t bar0 = sbase + CTRL;
  auto full_bar = [&](int s) { return bar0 + 8u * s; };
  auto empty_bar = [&](int s) { return bar0 + 8u * (STAGES + s); };
  auto accf_bar = [&](int b) { return bar0 + 8u * (2 * STAGES + b); };
  auto acce_bar = [&](int b) { return bar0 + 8u * (2 * STAGES + 2 + b); };
  const uint32_t drain_bar = bar0 + 8u * (2 * STAGES + 4);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + SLOT);
  volatile uint32_t* abort_flag = tmem_slot + 1;
  volatile uint32_t* decision = tmem_slot + 2;     // [2]
  volatile uint32_t* peer_issued = tmem_slot + 4;  // leader: loads the peer issued (teardown)
  float* sw_s = reinterpret_cast<float*>(smem + VEC);
  __half* bias_s = reinterpret_cast<__half*>(smem + VEC + BN * 4);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();  // 0 = leader (issues the MMAs), 1 = peer
  const uint32_t peer = rank ^ 1u;
  const uint32_t peer_abort = mapa_shared(smem_u32(tmem_slot + 1), peer);
  const int pair = static_cast<int>(blockIdx.x >> 1);
  const int npairs = static_cast<int>(gridDim.x >> 1);
  const int KB = static_cast<int>((g.K + KSUB * BK - 1) / (KSUB * BK));
  // tiles of one batch item (the whole grid when not batched)

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(full_bar(s), 1);  // the leader's arrive_expect_tx for both halves
      mbar_init(empty_bar(s), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(accf_bar(b), 1);
      mbar_init(acce_bar(b), 2);  // one arrival from each CTA's epilogue
    }
    mbar_init(drain_bar, 1);
    *abort_flag = 0;
    *peer_issued = 0;
    fence_barrier_init();
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
  }
  if (warp == 1) {
    tmem_alloc_pair(smem_u32(tmem_slot), TMEM_COLS);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  // barriers of both CTAs initialised and TMEM allocated before any
  // cross-CTA arrival
  cluster_sync_all();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  griddep_wait();  // inputs of this kernel are written by the previous one

  int64_t issued = 0;    // producer: stages issued by this CTA
  bool mma_any = false;  // leader's MMA thread: issued at least one MMA

  if (warp == 0) {
    if (lane == 0) {
      const uint32_t full_leader0 = mapa_shared(full_bar(0), 0);
      int64_t it = 0;
      bool ok = true;
      for (int t = pair; t < tiles && ok; t += npairs) {
        int bi, tm, tn;  // batch item (0 when not batched), token tile, channel tile
        tmap.coords<EPI == EPI_BMM>(t, bi, tm, tn);
        const int32_t m0 = tm * (2 * BM) + static_cast<int32_t>(rank) * BM;
        const int32_t n0 = tn * TBN + static_cast<int32_t>(rank) * TNH;
        for (int kb = 0; kb < KB; ++kb, ++it) {
          const int s = static_cast<int>(it % STAGES);
          const int64_t r = it / STAGES;
          if (it >= STAGES &&
              !pair_wait(empty_bar(s), static_cast<uint32_t>((r - 1) & 1), false, budget, status, abort_flag, peer_abort)) {
            ok = false;
            break;
          }
          const uint32_t st = sbase + s * STAGE_BYTES;
          if (rank == 0) mbar_arrive_expect_tx(full_bar(s), 2 * STAGE_BYTES);
#pragma unroll
          for (int j = 0; j < KSUB; ++j) {
            const int32_t x = (kb * KSUB + j) * BK;
            const uint32_t sa = st + j * A_BYTES, sb = st + KSUB * A_BYTES + j * TB_BYTES;
            if constexpr (EPI == EPI_BMM) {
              tma_load_3d_pair(sa, &tmA, full_leader0 + 8u * s, x, m0, bi);
              tma_load_3d_pair(sb, &tmB, full_leader0 + 8u * s, x, n0, bi);
            } else {
              tma_load_2d_pair(sa, &tmA, full_leader0 + 8u * s, x, m0);
              tma_load_2d_pair(sb, &tmB, full_leader0 + 8u * s, x, n0);
            }
          }
          ++issued;
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0 && rank == 0) {
      // leader: one pair MMA of 256 x 256 x 32 per 32 bytes of K
      constexpr uint32_t idesc = idesc_i8(2 * BM, TBN);
      int64_t it = 0;
      int tl = 0;
      bool ok = true;
      for (int t = pair; t < tiles && ok; t += npairs, ++tl) {
        const int b = tl & 1;
        if (tl >= 2 &&
            !pair_wait(acce_bar(b), static_cast<uint32_t>(((tl >> 1) - 1) & 1), true, budget, status, abort_flag, peer_abort))
          break;
        tc_fence_after();
        const uint32_t dacc = tmem + static_cast<uint32_t>(b * TBN);
        for (int kb = 0; kb < KB; ++kb, ++it) {
          const int s = static_cast<int>(it % STAGES);
          const uint32_t par = static_cast<uint32_t>((it / STAGES) & 1);
          if (!pair_wait(full_bar(s), par, false, budget, status, abort_flag, peer_abort)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t st = sbase + s * STAGE_BYTES;
#pragma unroll
          for (int j = 0; j < KSUB; ++j) {
            if (j > 0 && static_cast<int64_t>(kb * KSUB + j) * BK >= g.K) break;  // a box wholly past K: zeros
            const uint64_t a = sdesc_k_sw128(st + j * A_BYTES);
            const uint64_t bd = sdesc_k_sw128(st + KSUB * A_BYTES + j * TB_BYTES);
#pragma unroll
            for (int k = 0; k < BK / 32; ++k)
              mma_i8_pair(dacc, a + 2u * k, bd + 2u * k, idesc, (kb | j | k) != 0 ? 1u : 0u);
          }
          mma_any = true;
          mma_commit_pair_mc(empty_bar(s), 0x3);  // frees stage s in both CTAs
        }
        if (ok) mma_commit_pair_mc(accf_bar(b), 0x3);  // accumulator b complete in both CTAs
      }
      griddep_launch_dependents();
    } else if (lane == 0) {
      griddep_launch_dependents();
    }
  } else {
    // epilogue: 256 threads over this CTA's 128 rows x TBN columns
    const int et = threadIdx.x - 64;
    const int q = warp & 3;            // TMEM lane quarter this warp may access
    const int half = (warp - 2) >> 2;  // column half of the tile
    const uint32_t stg0 = sbase + STG + static_cast<uint32_t>(warp - 2) * STG_WARP;
    const uint32_t acce_leader0 = mapa_shared(acce_bar(0), 0);
    int nst = 0;  // blocks this warp has staged (selects the buffer; two stores may be in flight)
    // producer-side quantization: the next linear's 1/s of this tile's columns
    // (in the output staging area, unused in that mode) and its static scale
    float* inv_s_s = reinterpret_cast<float*>(smem + STG);
    float q_inv = 0.0f, q_sc = 0.0f;
    if constexpr (EPI == EPI_Q8) {
      q_sc = __fdiv_rn(*g.range_next, 127.0f);
      q_inv = q_sc > 0.0f ? __frcp_rn(q_sc) : 0.0f;
    }
    // this thread's scale entries of a tile: sw / bias / 1/s of column et and
    // sx of its row; fetched one tile ahead so their global-load latency
    // overlaps the previous tile's epilogue instead of stalling every tile
    struct Vecs {
      float sw, is, sx;
      __half bias;
    };
    auto fetch = [&](int t) {
      Vecs v{0.0f, 1.0f, 0.0f, __float2half_rn(0.0f)};
      if (EPI == EPI_I32 || t >= tiles) return v;
      int bi, tm, tn;
      tmap.coords<EPI == EPI_BMM>(t, bi, tm, tn);
      const int64_t n = static_cast<int64_t>(tn) * TBN + et;
      const int64_t row = static_cast<int64_t>(tm) * (2 * BM) + static_cast<int64_t>(rank) * BM + 32 * q + lane;
      if (et < TBN && n < g.N) {  // thread et < TBN holds column et's entries
        v.sw = g.sw[static_cast<int64_t>(bi) * g.N + n];
        if (g.bias != nullptr) v.bias = g.bias[n];
        if (EPI == EPI_Q8 && g.inv_s_next != nullptr) v.is = g.inv_s_next[n];
      }
      if (row < g.M) v.sx = g.sx[static_cast<int64_t>(bi) * g.M + row];
      return v;
    };
    Vecs nxt = fetch(pair);
    int tl = 0;
    for (int t = pair; t < tiles; t += npairs, ++tl) {
      const int b = tl & 1;
      int bi, tm, tn;  // batch item (0 when not batched), token tile, channel tile
      tmap.coords<EPI == EPI_BMM>(t, bi, tm, tn);
      const int64_t m0 = static_cast<int64_t>(tm) * (2 * BM) + static_cast<int64_t>(rank) * BM;
      const int64_t n0 = static_cast<int64_t>(tn) * TBN;
      const Vecs cur = nxt;
      nxt = fetch(t + npairs);
      if (EPI != EPI_I32 && et < TBN) {
        sw_s[et] = cur.sw;
        bias_s[et] = cur.bias;
        if (EPI == EPI_Q8) inv_s_s[et] = cur.is;
      }
      const float sxr = cur.sx;
      if (EPI == EPI_Q8) {
        const int64_t row = m0 + 32 * q + lane;
        if (tn == 0 && half == 0 && row < g.M) g.sx_next[row] = q_sc;
      }
      pair_wait(accf_bar(b), static_cast<uint32_t>((tl >> 1) & 1), false, budget, status, abort_flag, peer_abort);
      // one thread decides whether to stop and broadcasts it (double-buffered by
      // tile parity), so every epilogue thread leaves the loop at the same point.
      // The same barrier publishes this tile's sw / bias / 1/s above: the
      // barrier that ends the previous tile (below) came after every read of the
      // previous tile's entries, so they were free to overwrite.
      if (et == 0) decision[tl & 1] = *abort_flag;
      named_bar_sync(1, 32 * kEpiWarps);
      if (decision[tl & 1]) break;
      tc_fence_after();

      float pmax = 0.0f;  // EPI_QD: this lane's row maximum over the warp's 128 columns
      auto taddr = [&](int c) {
        return tmem + (static_cast<uint32_t>(32 * q) << 16) +
               static_cast<uint32_t>(TBN * b + CW * half + 32 * c);
      };
      const int64_t row0 = m0 + 32 * q;  // first row of this warp's blocks
      auto emit = [&](int c, uint32_t (&v)[32]) {
        const int cl = CW * half + 32 * c;  // column within the tile
        const int64_t col0 = n0 + cl;
        // rows / columns of this warp's 32 x 32 block inside the output (warp-uniform)
        const int brows = g.M - row0 < 32 ? static_cast<int>(g.M - row0) : 32;
        const int bcols = g.N - col0 < 32 ? static_cast<int>(g.N - col0) : 32;
        if constexpr (EPI == EPI_I32) {
          if (brows > 0 && bcols > 0)  // through the warp's 4 KB staging, row by row
            warp_store_rows_i32(stg0, v, g.acc + row0 * g.N + col0, g.N, brows, bcols);
          return;
        } else if constexpr (EPI == EPI_Q8) {
          // the composition, per element: y = fp16((acc * sx) * sw + bias),
          // a = relu ? max(y, 0) : y, x = a * inv_s_next, then the static
          // quantizer; fp32 pairs, the ReLU on half2 (max with 0 turns a NaN
          // into 0, like the scalar test), codes packed 4 per word, a NaN
          // product coded 0 (q8_code_bits).  With a zero range every code is
          // 0, as the scalar quantizer gives for a zero reciprocal.
          __align__(16) uint32_t qw[8];
          if (q_inv == 0.0f) {
#pragma unroll
            for (int u = 0; u < 8; ++u) qw[u] = 0u;
          } else {
            const uint64_t sx2 = f2_pack(sxr, sxr);
            const uint64_t qi2 = f2_pack(q_inv, q_inv);
            const float4* swv = reinterpret_cast<const float4*>(sw_s + cl);
            const float4* isv = reinterpret_cast<const float4*>(inv_s_s + cl);
            const uint4* bv = reinterpret_cast<const uint4*>(bias_s + cl);
            const __half2 zero2 = __float2half2_rn(0.0f);
#pragma unroll
            for (int j = 0; j < 32; j += 4) {
              const float4 w = swv[j / 4];
              const float4 is = isv[j / 4];
              uint64_t d0 = f2_mul_rn(f2_mul_rn(f2_pack(__int2float_rn(static_cast<int32_t>(v[j])),
                                                        __int2float_rn(static_cast<int32_t>(v[j + 1]))), sx2),
                                      f2_pack(w.x, w.y));
              uint64_t d1 = f2_mul_rn(f2_mul_rn(f2_pack(__int2float_rn(static_cast<int32_t>(v[j + 2])),
                                                        __int2float_rn(static_cast<int32_t>(v[j + 3]))), sx2),
                                      f2_pack(w.z, w.w));
              if (g.bias != nullptr) {
                const uint2 b4 = reinterpret_cast<const uint2*>(bv)[j / 4];
                const float2 b01 = __half22float2(*reinterpret_cast<const __half2*>(&b4.x));
                const float2 b23 = __half22float2(*reinterpret_cast<const __half2*>(&b4.y));
                // the add stays scalar: a packed add after a packed multiply can be
                // contracted into a fused multiply-add
                float2 e0 = f2_unpack(d0), e1 = f2_unpack(d1);
                d0 = f2_pack(__fadd_rn(e0.x, b01.x), __fadd_rn(e0.y, b01.y));
                d1 = f2_pack(__fadd_rn(e1.x, b23.x), __fadd_rn(e1.y, b23.y));
              }
              const float2 f0 = f2_unpack(d0), f1 = f2_unpack(d1);
              __half2 h0 = __floats2half2_rn(f0.x, f0.y), h1 = __floats2half2_rn(f1.x, f1.y);
              if (g.relu) {
                h0 = __hmax2(h0, zero2);
                h1 = __hmax2(h1, zero2);
              }
              const float2 a0 = __half22float2(h0), a1 = __half22float2(h1);
              const float2 p0 = f2_unpack(f2_mul_rn(f2_mul_rn(f2_pack(a0.x, a0.y), f2_pack(is.x, is.y)), qi2));
              const float2 p1 = f2_unpack(f2_mul_rn(f2_mul_rn(f2_pack(a1.x, a1.y), f2_pack(is.z, is.w)), qi2));
              const uint32_t c0 = q8_code_bits(p0.x);
              const uint32_t c1 = q8_code_bits(p0.y);
              const uint32_t c2 = q8_code_bits(p1.x);
              const uint32_t c3 = q8_code_bits(p1.y);
              qw[j / 4] = __byte_perm(__byte_perm(c0, c1, 0x0040), __byte_perm(c2, c3, 0x0040), 0x5410);
            }
          }
          if (row0 + lane < g.M && col0 < g.N) {
            // each lane writes its row's 32 codes, one full 32-byte sector
            int8_t* dst = g.q_next + (row0 + lane) * g.N + col0;
            if ((g.N % 16) == 0 && col0 + 32 <= g.N) {
              reinterpret_cast<uint4*>(dst)[0] = reinterpret_cast<const uint4*>(qw)[0];
              reinterpret_cast<uint4*>(dst)[1] = reinterpret_cast<const uint4*>(qw)[1];
            } else {
              const int8_t* qb = reinterpret_cast<const int8_t*>(qw);
              for (int j = 0; j < 32; ++j)
                if (col0 + j < g.N) dst[j] = qb[j];
            }
          }
          return;
        } else {
          // ((acc * sx) * sw + bias) in packed fp32 pairs, each lane rounded
          // like the scalar sequence; scales and bias read as 16-byte vectors
          __align__(16) __half h[32];
          const uint64_t sx2 = f2_pack(sxr, sxr);
          const float4* swv = reinterpret_cast<const float4*>(sw_s + cl);
          const uint4* bv = reinterpret_cast<const uint4*>(bias_s + cl);
#pragma unroll
          for (int j = 0; j < 32; j += 8) {
            const float4 w0 = swv[j / 4], w1 = swv[j / 4 + 1];
            uint64_t p[4];
            p[0] = f2_mul_rn(f2_mul_rn(f2_pack(__int2float_rn(static_cast<int32_t>(v[j])),
                                              __int2float_rn(static_cast<int32_t>(v[j + 1]))), sx2),
                             f2_pack(w0.x, w0.y));
            p[1] = f2_mul_rn(f2_mul_rn(f2_pack(__int2float_rn(static_cast<int32_t>(v[j + 2])),
                                              __int2float_rn(static_cast<int32_t>(v[j + 3]))), sx2),
                             f2_pack(w0.z, w0.w));
            p[2] = f2_mul_rn(f2_mul_rn(f2_pack(__int2float_rn(static_cast<int32_t>(v[j + 4])),
                                              __int2float_rn(static_cast<int32_t>(v[j + 5]))), sx2),
                             f2_pack(w1.x, w1.y));
            p[3] = f2_mul_rn(f2_mul_rn(f2_pack(__int2float_rn(static_cast<int32_t>(v[j + 6])),
                                              __int2float_rn(static_cast<int32_t>(v[j + 7]))), sx2),
                             f2_pack(w1.z, w1.w));
            if (g.bias != nullptr) {
              const uint4 b8 = bv[j / 8];
              const uint32_t bw[4] = {b8.x, b8.y, b8.z, b8.w};
#pragma unroll
              for (int u = 0; u < 4; ++u) {
                const float2 bf = __half22float2(*reinterpret_cast<const __half2*>(&bw[u]));
                const float2 e = f2_unpack(p[u]);  // scalar adds: never contracted with the multiply
                p[u] = f2_pack(__fadd_rn(e.x, bf.x), __fadd_rn(e.y, bf.y));
              }
            }
#pragma unroll
            for (int u = 0; u < 4; ++u) {
              const float2 f = f2_unpack(p[u]);
              *reinterpret_cast<__half2*>(&h[j + 2 * u]) = __floats2half2_rn(f.x, f.y);
            }
          }
          if constexpr (EPI == EPI_QD) {
            // a = relu ? max(y, 0) : y on half2 (a NaN becomes 0, as in the
            // scalar y > 0 ? y : 0), and this row's running maximum of
            // |fp32(a) * inv_s_next[n]| (NaN-free: fmaxf drops a NaN); the
            // 1/s of these 32 columns are the same for every lane (broadcast
            // loads), columns past N contribute 0
            const __half2 zero2 = __float2half2_rn(0.0f);
#pragma unroll
            for (int j = 0; j < 32; j += 4) {
              __half2* h2 = reinterpret_cast<__half2*>(&h[j]);
              if (g.relu) {
                h2[0] = __hmax2(h2[0], zero2);
                h2[1] = __hmax2(h2[1], zero2);
              }
              float4 is = make_float4(1.0f, 1.0f, 1.0f, 1.0f);
              if (col0 + j >= g.N) is = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
              else if (g.inv_s_next != nullptr) is = __ldg(reinterpret_cast<const float4*>(g.inv_s_next + col0 + j));
              const float2 a01 = __half22float2(h2[0]), a23 = __half22float2(h2[1]);
              pmax = fmaxf(pmax, fabsf(__fmul_rn(a01.x, is.x)));
              pmax = fmaxf(pmax, fabsf(__fmul_rn(a01.y, is.y)));
              pmax = fmaxf(pmax, fabsf(__fmul_rn(a23.x, is.z)));
              pmax = fmaxf(pmax, fabsf(__fmul_rn(a23.y, is.w)));
            }
          }
          if constexpr (TMAS) {
            // stage the 32 x 32 block in the 64-byte-swizzled image; one TMA
            // store writes it (rows/columns outside y are skipped); two buffers
            // per warp, so the previous block's store may still be reading one
            const uint32_t stg = stg0 + static_cast<uint32_t>(nst & 1) * STG_BYTES;
            if (lane == 0 && nst >= 2) bulk_wait_group_read<1>();
            __syncwarp();
            ++nst;
            const uint4* hv = reinterpret_cast<const uint4*>(h);
#pragma unroll
            for (int cc = 0; cc < 4; ++cc) {
              const uint32_t addr = stg + lane * 64 + ((cc ^ ((lane >> 1) & 3)) * 16);
              asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(hv[cc].x), "r"(hv[cc].y),
                           "r"(hv[cc].z), "r"(hv[cc].w)
                           : "memory");
            }
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) {
              if (row0 < g.M && col0 < g.N) {
                if constexpr (EPI == EPI_BMM)
                  tma_store_3d(&tmY, stg, static_cast<int32_t>(col0), static_cast<int32_t>(row0), bi);
                else
                  tma_store_2d(&tmY, stg, static_cast<int32_t>(col0), static_cast<int32_t>(row0));
              }
              bulk_commit_group();
            }
          } else if (brows > 0 && bcols > 0) {
            // rows not 16-byte aligned (N % 8 != 0): through the staging, row by row
            warp_store_rows_f16(stg0, h, g.y + (static_cast<int64_t>(bi) * g.M + row0) * g.N + col0, g.N, brows,
                                bcols);
          }
        }
      };
      uint32_t va[32], vb[32];
      tmem_ld_32x32b_x32(taddr(0), va);
      tmem_ld_wait_regs(va);
      tmem_ld_32x32b_x32(taddr(1), vb);
      emit(0, va);
      tmem_ld_wait_regs(vb);
      if constexpr (NB == 4) {
        tmem_ld_32x32b_x32(taddr(2), va);
        emit(1, vb);
        tmem_ld_wait_regs(va);
        tmem_ld_32x32b_x32(taddr(3), vb);
        emit(2, va);
        tmem_ld_wait_regs(vb);
        emit(3, vb);
      } else {
        emit(1, vb);
      }
      if constexpr (EPI == EPI_QD) {
        const int64_t row = row0 + lane;
        // every group of the row is written (a group wholly past N holds 0), so the
        // codes pass never reads a stale maximum
        if (row < g.M) g.part[row * g.part_n + 2 * tn + half] = pmax;
      }
      // every epilogue thread of this CTA has read accumulator b: tell the leader
      tc_fence_before();
      named_bar_sync(1, 32 * kEpiWarps);
      if (et == 0) mbar_arrive_cluster(acce_leader0 + 8u * b);
    }
    if (lane == 0) bulk_wait_group0();  // this warp's output stores are complete
  }

  // teardown.  The peer tells the leader how many stages it loaded; after
  // the cluster barrier both CTAs see the same abort flag (a wait that runs
  // out raises both).  After an abort the leader waits (bounded) for its
  // MMAs and for the last phase of every stage: a half the peer never loaded
  // is settled with complete_tx, a half the leader never armed is armed now.
  // Without an abort nothing is in flight any more at the first cluster
  // barrier (every load was consumed by an MMA whose completion both
  // epilogues waited for); after one, a second barrier keeps both CTAs
  // resident until the drain is done.  Then TMEM is freed.
  tc_fence_before();
  __syncthreads();
  if (threadIdx.x == 0 && rank == 1)
    st_shared_cluster_u32(mapa_shared(smem_u32(const_cast<uint32_t*>(peer_issued)), 0),
                          static_cast<uint32_t>(issued));
  cluster_sync_all();
  const bool aborted = *abort_flag != 0;  // the same in both CTAs after the barrier
  if (aborted && rank == 0) {
    if (warp == 1 && lane == 0 && mma_any) {
      mma_commit_pair(drain_bar);
      mbar_drain(drain_bar, 0, budget);
    }
    if (threadIdx.x == 0) {
      const int64_t pi = static_cast<int64_t>(*peer_issued);
      for (int s = 0; s < STAGES; ++s) {
        const int64_t lr = issued > s ? (issued - 1 - s) / STAGES + 1 : 0;  // rounds of stage s armed
        const int64_t pr = pi > s ? (pi - 1 - s) / STAGES + 1 : 0;          // rounds the peer loaded
        if (lr == 0 && pr == 0) continue;
        if (lr == pr + 1) mbar_complete_tx(full_bar(s), STAGE_BYTES);
        else if (pr == lr + 1) mbar_arrive_expect_tx(full_bar(s), STAGE_BYTES);
        const int64_t last = (lr > pr ? lr : pr) - 1;
        mbar_drain(full_bar(s), static_cast<uint32_t>(last & 1), budget);
      }
    }
  }
  if (aborted) cluster_sync_all();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem, TMEM_COLS);
  }
}

// Clusters of two CTAs that fit on the device at once (at most one per TPC).
int max_pairs(int device, int num_sms) {
  static int cached[64] = {0};
  const int d = device < 64 ? device : 63;
  if (cached[d] > 0) return cached[d];
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(num_sms & ~1));
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = SMEM;
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, k_gemm_pair<EPI_F16, true, 2>, &cfg) != cudaSuccess || n <= 0) {
    (void)cudaGetLastError();
    n = num_sms / 2;
  }
  if (n > num_sms / 2) n = num_sms / 2;
  cached[d] = n;
  return n;
}

template <int EPI, bool TMAS, int KSUB, int TBN>
cudaError_t smem_attr(int device) {
  static bool attr_set[64] = {};
  const int dev = device < 64 ? device : 63;
  if (!attr_set[dev]) {
    cudaError_t e = cudaFuncSetAttribute(k_gemm_pair<EPI, TMAS, KSUB, TBN>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(SMEM));
    if (e != cudaSuccess) return e;
    attr_set[dev] = true;
  }
  return cudaSuccess;
}

template <int EPI, bool TMAS, int KSUB, int TBN>
cudaError_t launch_kernel(const GemmArgs& g, const Ctx& c, const CUtensorMap& tmA, const CUtensorMap& tmB,
                          const CUtensorMap& tmY, int tiles_m, int tiles, int pairs) {
  cudaError_t e = smem_attr<EPI, TMAS, KSUB, TBN>(c.device);
  if (e != cudaSuccess) return e;
  // tiles of one batch item (the whole grid when not batched)
  const int per_item = EPI == EPI_BMM ? tiles / static_cast<int>(g.batch) : tiles;
  return launch_pdl(k_gemm_pair<EPI, TMAS, KSUB, TBN>, dim3(2 * pairs), dim3(kThreads), SMEM, c.stream, tmA, tmB,
                    tmY, g, TileMap::make(per_item, tiles_m), tiles, c.status, c.budget_ns);
}

template <int EPI, bool TMAS, int TBN = BN>
cudaError_t launch_ring(const GemmArgs& g, const Ctx& c, const CUtensorMap& tmA, const CUtensorMap& tmB,
                        const CUtensorMap& tmY, int tiles_m, int tiles, int pairs) {
  if (g.K >= 512) return launch_kernel<EPI, TMAS, 2, TBN>(g, c, tmA, tmB, tmY, tiles_m, tiles, pairs);
  return launch_kernel<EPI, TMAS, 1, TBN>(g, c, tmA, tmB, tmY, tiles_m, tiles, pairs);
}

template <int EPI>
cudaError_t launch_cfg(const GemmArgs& g, const Ctx& c) {
  CUtensorMap tmA, tmB, tmY;
  const bool bmm = EPI == EPI_BMM;
  const uint64_t items = bmm ? static_cast<uint64_t>(g.batch) : 1;
  // the batched product with at most 128 channels (P V): tiles 128 wide
  const bool narrow = bmm && g.N <= BN / 2;
  const int tbn = narrow ? BN / 2 : BN;
  if (bmm) {
    if (!make_tmap_i8_3d(&tmA, g.xq, g.K, g.M, items, BK, BM)) return cudaErrorInvalidValue;
    if (!make_tmap_i8_3d(&tmB, g.wq, g.K, g.N, items, BK, tbn / 2)) return cudaErrorInvalidValue;
  } else {
    if (!make_tmap_i8(&tmA, g.xq, g.K, g.M, BK, BM)) return cudaErrorInvalidValue;
    if (!make_tmap_i8(&tmB, g.wq, g.K, g.N, BK, BNH)) return cudaErrorInvalidValue;
  }
  // TMA stores of fp16 y need 16-byte row strides (N % 8 == 0); otherwise
  // row-by-row stores through the staging (always for int32 accumulators;
  // int8 codes are written 32 bytes per row)
  const bool tma_store = (EPI == EPI_F16 || EPI == EPI_QD || bmm) && g.N % 8 == 0;
  if (tma_store) {
    const bool ok = bmm ? make_tmap_f16_out_3d(&tmY, g.y, g.N, g.M, items) : make_tmap_f16_out(&tmY, g.y, g.N, g.M);
    if (!ok) return cudaErrorInvalidValue;
  } else {
    memset(&tmY, 0, sizeof(tmY));
  }
  const int tiles_m = static_cast<int>((g.M + 2 * BM - 1) / (2 * BM));
  const int tiles_n = static_cast<int>((g.N + tbn - 1) / tbn);
  const int64_t tiles64 = static_cast<int64_t>(items) * tiles_m * tiles_n;
  if (tiles64 > 0x7fffffffLL) return cudaErrorInvalidValue;
  const int tiles = static_cast<int>(tiles64);
  const int mp = max_pairs(c.device, c.num_sms);
  const int pairs = tiles < mp ? tiles : mp;
  if constexpr (EPI == EPI_QD) {  // N % 16 == 0 here: always TMA stores
    if (!tma_store) return cudaErrorInvalidValue;
    return launch_ring<EPI, true>(g, c, tmA, tmB, tmY, tiles_m, tiles, pairs);
  } else {
    if constexpr (EPI == EPI_BMM) {
      if (narrow)
        return tma_store ? launch_ring<EPI, true, BN / 2>(g, c, tmA, tmB, tmY, tiles_m, tiles, pairs)
                         : launch_ring<EPI, false, BN / 2>(g, c, tmA, tmB, tmY, tiles_m, tiles, pairs);
    }
    if (tma_store) {
      if constexpr (EPI == EPI_F16 || EPI == EPI_BMM)
        return launch_ring<EPI, true>(g, c, tmA, tmB, tmY, tiles_m, tiles, pairs);
    }
    return launch_ring<EPI, false>(g, c, tmA, tmB, tmY, tiles_m, tiles, pairs);
  }
}

}  // namespace

cudaError_t launch_bmm_pair(const GemmArgs& g, const Ctx& c) { return launch_cfg<EPI_BMM>(g, c); }

cudaError_t launch_gemm_pair(const GemmArgs& g, const Ctx& c) {
  if (g.acc != nullptr) return launch_cfg<EPI_I32>(g, c);
  if (g.q_next != nullptr) return launch_cfg<EPI_Q8>(g, c);
  if (g.part != nullptr) return launch_cfg<EPI_QD>(g, c);
  return launch_cfg<EPI_F16>(g, c);
}

}  // namespace sq
