// k_gemm_wide.cu -- the W8A8 linear on single CTAs with 256 x 256 tiles
// (SQ_PATH_WIDE; the automatic choice for M > 128 is the CTA-pair kernel):
// INT8 x INT8 -> INT32 GEMM on the 5th-generation tensor cores with the
// dequant epilogue fused (glossary "INT8 GEMM"; section "inference", O1
// scales; the quantization tutorial's "multiply the scale back").
//
// Persistent: one CTA per SM walks 256 x 256 output tiles.  Per 128-byte K
// block a 64 KB stage holds 256 token rows of xq and 256 weight rows of wq;
// two tcgen05.mma kind::i8 of 128 x 256 x 32 (token rows 0-127 and 128-255)
// share the weight operand, so each byte brought into shared memory feeds
// twice the MMA work of a 128 x 256 tile.  The two int32 accumulators fill
// all 512 TMEM columns.
//   warp 0      TMA producer (3-stage ring); runs ahead into the next tile
//               while the epilogue drains the accumulators
//   warp 1      TMEM allocation; lane 0 issues the MMAs
//   warps 2-9   epilogue: warp w reads TMEM lane quarter w % 4 (32 token
//               rows of each accumulator) for column half (w - 2) / 4, then
//               y = fp16((acc * sx[t]) * sw[n] + bias[n]); each 32 x 32 block
//               is staged in shared memory and written by a TMA store
// Every mbarrier wait is bounded; a wait that runs out records a timeout, the
// CTA drains what it issued, frees TMEM and returns.
#include <string.h>

#include "sq_internal.h"
#include "sq_ptx.cuh"
#include "sq_tmap.h"

namespace sq {
namespace {

constexpr int BM = 256;  // token rows per tile (two 128-lane accumulators)
constexpr int BN = 256;  // output channels per tile
constexpr int BK = 128;  // K bytes per stage = one 128-byte swizzle row
constexpr int STAGES = 3;
constexpr int kEpiWarps = 8;
constexpr int kThreads = 64 + 32 * kEpiWarps;
constexpr int A_BYTES = BM * BK;              // 32 KB
constexpr int B_BYTES = BN * BK;              // 32 KB
constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
constexpr int STG = STAGES * STAGE_BYTES;     // per-epilogue-warp output staging
constexpr int STG_BYTES = 2048;               // one 32 rows x 32 fp16 block, 64-byte swizzle
constexpr int STG_WARP = 2 * STG_BYTES;       // double-buffered per warp
constexpr int CTRL = STG + kEpiWarps * STG_WARP;
constexpr int NBARS = 2 * STAGES + 3;         // full, empty, acc_full, acc_empty, drain
constexpr int SLOT = CTRL + NBARS * 8;        // TMEM address, abort flag, decision[2]
constexpr int VEC = SLOT + 16;                // sw[BN] fp32, bias[BN] fp16 of the current tile
constexpr int SMEM_BYTES = VEC + BN * 4 + BN * 2;
constexpr size_t SMEM = SMEM_BYTES + 1024;    // slack for 1024-byte alignment
constexpr uint32_t TMEM_COLS = 512;

// TMAS: fp16 blocks leave through TMA stores (rows 16-byte aligned); without
// it (and for int32) through the warp's staging, row by row -- a separate
// instantiation, so the TMA-store kernel keeps its own registers.
template <bool OUT_I32, bool TMAS>
__global__ void __launch_bounds__(kThreads, 1)
    k_gemm_wide(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                const __grid_constant__ CUtensorMap tmY, const GemmArgs g, int tiles_m, int tiles,
                uint32_t* status, uint64_t budget) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  const uint32_t sbase = smem_u32(smem);
  const uint32_t bar0 = sbase + CTRL;
  auto full_bar = [&](int s) { return bar0 + 8u * s; };
  auto empty_bar = [&](int s) { return bar0 + 8u * (STAGES + s); };
  const uint32_t accf_bar = bar0 + 8u * (2 * STAGES);
  const uint32_t acce_bar = bar0 + 8u * (2 * STAGES + 1);
  const uint32_t drain_bar = bar0 + 8u * (2 * STAGES + 2);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + SLOT);
  volatile uint32_t* abort_flag = tmem_slot + 1;
  volatile uint32_t* decision = tmem_slot + 2;  // [2]
  float* sw_s = reinterpret_cast<float*>(smem + VEC);
  __half* bias_s = reinterpret_cast<__half*>(smem + VEC + BN * 4);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int KB = static_cast<int>((g.K + BK - 1) / BK);

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(full_bar(s), 1);
      mbar_init(empty_bar(s), 1);
    }
    mbar_init(accf_bar, 1);
    mbar_init(acce_bar, 1);
    mbar_init(drain_bar, 1);
    *abort_flag = 0;
    fence_barrier_init();
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  griddep_wait();  // inputs of this kernel are written by the previous one

  int64_t issued = 0;    // producer: stages issued
  bool mma_any = false;  // MMA thread: issued at least one MMA

  if (warp == 0) {
    if (lane == 0) {
      int64_t it = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < tiles && ok; t += gridDim.x) {
        const int32_t m0 = (t % tiles_m) * BM;
        const int32_t n0 = (t / tiles_m) * BN;
        for (int kb = 0; kb < KB; ++kb, ++it) {
          const int s = static_cast<int>(it % STAGES);
          const int64_t r = it / STAGES;
          if (it >= STAGES && !mbar_wait(empty_bar(s), static_cast<uint32_t>((r - 1) & 1), budget, status, abort_flag)) {
            ok = false;
            break;
          }
          const uint32_t st = sbase + s * STAGE_BYTES;
          mbar_arrive_expect_tx(full_bar(s), STAGE_BYTES);
          tma_load_2d(st, &tmA, full_bar(s), kb * BK, m0);
          tma_load_2d(st + A_BYTES, &tmB, full_bar(s), kb * BK, n0);
          ++issued;
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_i8(128, BN);
      int64_t it = 0;
      int tl = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < tiles && ok; t += gridDim.x, ++tl) {
        if (tl >= 1 && !mbar_wait(acce_bar, static_cast<uint32_t>((tl - 1) & 1), budget, status, abort_flag))
          break;
        tc_fence_after();
        for (int kb = 0; kb < KB; ++kb, ++it) {
          const int s = static_cast<int>(it % STAGES);
          const int64_t r = it / STAGES;
          if (!mbar_wait(full_bar(s), static_cast<uint32_t>(r & 1), budget, status, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t st = sbase + s * STAGE_BYTES;
          const uint64_t a0 = sdesc_k_sw128(st);
          const uint64_t a1 = sdesc_k_sw128(st + A_BYTES / 2);
          const uint64_t b = sdesc_k_sw128(st + A_BYTES);
#pragma unroll
          for (int k = 0; k < BK / 32; ++k) {
            const uint32_t acc = (kb | k) != 0 ? 1u : 0u;
            mma_i8(tmem, a0 + 2u * k, b + 2u * k, idesc, acc);
            mma_i8(tmem + 256u, a1 + 2u * k, b + 2u * k, idesc, acc);
          }
          mma_any = true;
          mma_commit(empty_bar(s));
        }
        if (ok) mma_commit(accf_bar);
      }
      griddep_launch_dependents();
    }
  } else {
    // epilogue: 256 threads
    const int et = threadIdx.x - 64;
    const int q = warp & 3;            // TMEM lane quarter this warp may access
    const int half = (warp - 2) >> 2;  // column half of the tile
    const uint32_t stg0 = sbase + STG + static_cast<uint32_t>(warp - 2) * STG_WARP;
    int nst = 0;  // blocks this warp has staged (selects the buffer; two stores may be in flight)
    int tl = 0;
    for (int t = blockIdx.x; t < tiles; t += gridDim.x, ++tl) {
      const int64_t m0 = static_cast<int64_t>(t % tiles_m) * BM;
      const int64_t n0 = static_cast<int64_t>(t / tiles_m) * BN;
      if (!OUT_I32) {
        const int64_t n = n0 + et;
        sw_s[et] = n < g.N ? g.sw[n] : 0.0f;
        bias_s[et] = (g.bias != nullptr && n < g.N) ? g.bias[n] : __float2half_rn(0.0f);
      }
      float sxr[2] = {0.0f, 0.0f};
      if (!OUT_I32) {
#pragma unroll
        for (int a = 0; a < 2; ++a) {
          const int64_t row = m0 + 128 * a + 32 * q + lane;
          sxr[a] = row < g.M ? g.sx[row] : 0.0f;
        }
      }
      named_bar_sync(1, 32 * kEpiWarps);
      mbar_wait(accf_bar, static_cast<uint32_t>(tl & 1), budget, status, abort_flag);
      // one thread decides whether to stop and broadcasts it (double-buffered by
      // tile parity), so every epilogue thread leaves the loop at the same point
      if (et == 0) decision[tl & 1] = *abort_flag;
      named_bar_sync(1, 32 * kEpiWarps);
      if (decision[tl & 1]) break;
      tc_fence_after();

      // 8 chunks of 32 columns: (accumulator a, column group cc); the TMEM load
      // of the next chunk is in flight while the current one is converted
      auto taddr = [&](int idx) {
        return tmem + (static_cast<uint32_t>(32 * q) << 16) +
               static_cast<uint32_t>(256 * (idx >> 2) + 128 * half + 32 * (idx & 3));
      };
      auto emit = [&](int idx, uint32_t (&v)[32]) {
        const int a = idx >> 2;
        const int cl = 128 * half + 32 * (idx & 3);  // column within the tile
        const int64_t row0 = m0 + 128 * a + 32 * q;  // first row of this warp's block
        const int64_t col0 = n0 + cl;
        // rows / columns of this warp's 32 x 32 block inside the output (warp-uniform)
        const int brows = g.M - row0 < 32 ? static_cast<int>(g.M - row0) : 32;
        const int bcols = g.N - col0 < 32 ? static_cast<int>(g.N - col0) : 32;
        if constexpr (OUT_I32) {
          if (brows > 0 && bcols > 0)  // through the warp's 4 KB staging, row by row
            warp_store_rows_i32(stg0, v, g.acc + row0 * g.N + col0, g.N, brows, bcols);
          return;
        } else {
        __align__(16) __half h[32];
#pragma unroll
        for (int j = 0; j < 32; j += 2) {
          float f0 = dequant_f32(static_cast<int32_t>(v[j]), sxr[a], sw_s[cl + j]);
          float f1 = dequant_f32(static_cast<int32_t>(v[j + 1]), sxr[a], sw_s[cl + j + 1]);
          if (g.bias != nullptr) {
            const float2 b = __half22float2(*reinterpret_cast<const __half2*>(&bias_s[cl + j]));
            f0 = __fadd_rn(f0, b.x);
            f1 = __fadd_rn(f1, b.y);
          }
          // both lanes of the pair rounded to nearest even in one instruction
          *reinterpret_cast<__half2*>(&h[j]) = __floats2half2_rn(f0, f1);
        }
        if constexpr (TMAS) {
          // stage the 32 x 32 block in the 64-byte-swizzled image and let one
          // TMA store write it (rows/columns outside y are skipped by the TMA);
          // two buffers per warp, so the store of the previous block may still
          // be reading the other one
          const uint32_t stg = stg0 + static_cast<uint32_t>(nst & 1) * STG_BYTES;
          if (lane == 0 && nst >= 2) bulk_wait_group_read<1>();  // the store from this buffer is done reading
          __syncwarp();
          ++nst;
          const uint4* hv = reinterpret_cast<const uint4*>(h);
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            const uint32_t addr = stg + lane * 64 + ((c ^ ((lane >> 1) & 3)) * 16);
            asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(hv[c].x), "r"(hv[c].y),
                         "r"(hv[c].z), "r"(hv[c].w)
                         : "memory");
          }
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) {
            if (row0 < g.M && col0 < g.N)
              tma_store_2d(&tmY, stg, static_cast<int32_t>(col0), static_cast<int32_t>(row0));
            bulk_commit_group();  // one group per staged block, empty if nothing was stored
          }
        } else if (brows > 0 && bcols > 0) {
          // rows not 16-byte aligned (N % 8 != 0): through the staging, row by row
          warp_store_rows_f16(stg0, h, g.y + row0 * g.N + col0, g.N, brows, bcols);
        }
        }
      };
      uint32_t va[32], vb[32];
      tmem_ld_32x32b_x32(taddr(0), va);
      tmem_ld_wait_regs(va);
#pragma unroll 1
      for (int idx = 0; idx < 8; idx += 2) {
        tmem_ld_32x32b_x32(taddr(idx + 1), vb);
        emit(idx, va);
        tmem_ld_wait_regs(vb);
        if (idx + 2 < 8) tmem_ld_32x32b_x32(taddr(idx + 2), va);
        emit(idx + 1, vb);
        tmem_ld_wait_regs(va);
      }
      // every epilogue thread has read its TMEM columns: release the accumulators
      tc_fence_before();
      named_bar_sync(1, 32 * kEpiWarps);
      if (et == 0) mbar_arrive(acce_bar);
    }
    if (lane == 0) bulk_wait_group0();  // this warp's output stores are complete
  }

  // teardown: after an abort, wait (bounded) for the MMAs and TMA loads this
  // CTA issued before freeing TMEM.
  tc_fence_before();
  __syncthreads();
  if (*abort_flag) {
    if (warp == 1 && lane == 0 && mma_any) {
      mma_commit(drain_bar);
      mbar_drain(drain_bar, 0, budget);
    }
    if (warp == 0 && lane == 0) {
      for (int s = 0; s < STAGES && s < issued; ++s) {
        const int64_t last = ((issued - 1 - s) / STAGES) * STAGES + s;  // last load into stage s
        mbar_drain(full_bar(s), static_cast<uint32_t>((last / STAGES) & 1), budget);
      }
    }
    __syncthreads();
  }
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, TMEM_COLS);
  }
}

template <bool OUT_I32, bool TMAS>
cudaError_t launch_kernel(const CUtensorMap& tmA, const CUtensorMap& tmB, const CUtensorMap& tmY,
                          const GemmArgs& g, int tiles_m, int tiles, const Ctx& c) {
  static bool attr_set[64] = {false};
  const int dev = c.device < 64 ? c.device : 63;
  if (!attr_set[dev]) {
    cudaError_t e = cudaFuncSetAttribute(k_gemm_wide<OUT_I32, TMAS>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(SMEM));
    if (e != cudaSuccess) return e;
    attr_set[dev] = true;
  }
  const int grid = tiles < c.num_sms ? tiles : c.num_sms;
  return launch_pdl(k_gemm_wide<OUT_I32, TMAS>, dim3(grid), dim3(kThreads), SMEM, c.stream, tmA, tmB, tmY, g,
                    tiles_m, tiles, c.status, c.budget_ns);
}

template <bool OUT_I32>
cudaError_t launch_cfg(const GemmArgs& g, const Ctx& c) {
  CUtensorMap tmA, tmB, tmY;
  if (!make_tmap_i8(&tmA, g.xq, g.K, g.M, BK, BM)) return cudaErrorInvalidValue;
  if (!make_tmap_i8(&tmB, g.wq, g.K, g.N, BK, BN)) return cudaErrorInvalidValue;
  // TMA stores need 16-byte row strides (N % 8 == 0); otherwise row-by-row
  // stores through the staging
  const bool tma_store = !OUT_I32 && g.N % 8 == 0;
  if (tma_store && !make_tmap_f16_out(&tmY, g.y, g.N, g.M)) return cudaErrorInvalidValue;
  if (!tma_store) memset(&tmY, 0, sizeof(tmY));
  const int tiles_m = static_cast<int>((g.M + BM - 1) / BM);
  const int tiles_n = static_cast<int>((g.N + BN - 1) / BN);
  const int tiles = tiles_m * tiles_n;
  if (tma_store) {
    if constexpr (!OUT_I32) return launch_kernel<false, true>(tmA, tmB, tmY, g, tiles_m, tiles, c);
  }
  return launch_kernel<OUT_I32, false>(tmA, tmB, tmY, g, tiles_m, tiles, c);
}

}  // namespace

cudaError_t launch_gemm_wide(const GemmArgs& g, const Ctx& c) {
  if (g.acc != nullptr) return launch_cfg<true>(g, c);
  return launch_cfg<false>(g, c);
}

}  // namespace sq
