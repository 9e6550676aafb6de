// k_gemm_tiled.cu -- the W8A8 linear for large token counts: INT8 x INT8 ->
// INT32 GEMM on the 5th-generation tensor cores with the dequant epilogue
// fused (glossary "INT8 GEMM"; section "inference", O1 scales; the
// quantization tutorial's "multiply the scale back").
//
// One CTA computes one 128 x BN output tile:
//   warp 0      TMA producer: 128-byte-swizzled K-major tiles of xq [M, K]
//               and wq [N, K] into a STAGES-deep shared-memory ring;
//   warp 1      allocates TMEM; lane 0 issues tcgen05.mma.kind::i8
//               (128 x BN x 32 per instruction, 4 per 128-byte K block)
//               into an int32 TMEM accumulator, releasing each stage with
//               tcgen05.commit;
//   warps 2-5   epilogue: tcgen05.ld of the accumulator (each warp owns its
//               32-lane TMEM quarter = 32 token rows), then
//               y = fp16((acc * sx[t]) * sw[n] + bias[n]).
// Every mbarrier wait is bounded (sq_ptx.cuh); a wait that runs out records
// a timeout, the CTA drains what it issued, frees TMEM and returns.
#include "sq_internal.h"
#include "sq_ptx.cuh"
#include "sq_tmap.h"

namespace sq {
namespace {

constexpr int BM = 128;  // token rows per tile (TMEM lanes)
constexpr int BK = 128;  // K bytes per stage = one 128-byte swizzle row
constexpr int kThreads = 192;

template <int BN, int STAGES, bool ROWS>
struct TiledLayout {
  static constexpr int A_BYTES = BM * BK;
  static constexpr int B_BYTES = BN * BK;
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr int CTRL = STAGES * STAGE_BYTES;      // barriers start here
  static constexpr int NBARS = 2 * STAGES + 2;           // full, empty, acc_full, drain
  static constexpr int SLOT = CTRL + NBARS * 8;          // TMEM address, abort flag
  static constexpr int VEC = SLOT + 16;                  // sw[BN], bias[BN]
  static constexpr int STG = VEC + 2 * BN * 4;           // 4 KB output staging per epilogue warp (ROWS)
  static constexpr int BYTES = STG + (ROWS ? 4 * 4096 : 0);
  static constexpr size_t SMEM = BYTES + 1024;           // slack for 1024-byte alignment
  static_assert(STG % 16 == 0 && SMEM <= 232448, "staging alignment, shared memory per CTA");
};

// ROWS: the output blocks go through the warp's staging, row by row (int32,
// or fp16 rows that are not 16-byte aligned); otherwise each lane stores its
// fp16 row as 16-byte vectors.
template <int BN, int STAGES, bool OUT_I32, bool ROWS>
__global__ void __launch_bounds__(kThreads, 1)
    k_gemm_tiled(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                 const GemmArgs g, uint32_t* status, uint64_t budget) {
  using L = TiledLayout<BN, STAGES, ROWS>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  const uint32_t sbase = smem_u32(smem);
  const uint32_t sA = sbase;
  const uint32_t sB = sbase + STAGES * L::A_BYTES;
  const uint32_t bar0 = sbase + L::CTRL;
  auto full_bar = [&](int s) { return bar0 + 8u * s; };
  auto empty_bar = [&](int s) { return bar0 + 8u * (STAGES + s); };
  const uint32_t acc_bar = bar0 + 8u * (2 * STAGES);
  const uint32_t drain_bar = bar0 + 8u * (2 * STAGES + 1);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::SLOT);
  volatile uint32_t* abort_flag = tmem_slot + 1;
  float* sw_s = reinterpret_cast<float*>(smem + L::VEC);
  float* bias_s = sw_s + BN;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t m0 = static_cast<int64_t>(blockIdx.y) * BM;
  const int64_t n0 = static_cast<int64_t>(blockIdx.x) * BN;
  const int KB = static_cast<int>((g.K + BK - 1) / BK);

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(full_bar(s), 1);
      mbar_init(empty_bar(s), 1);
    }
    mbar_init(acc_bar, 1);
    mbar_init(drain_bar, 1);
    *abort_flag = 0;
    fence_barrier_init();
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), BN);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  griddep_wait();  // inputs of this kernel are written by the previous one

  int issued = 0;        // producer: stages issued
  bool mma_any = false;  // MMA thread: issued at least one MMA

  if (warp == 0) {
    if (lane == 0) {
      for (int kb = 0; kb < KB; ++kb) {
        const int s = kb % STAGES;
        const int r = kb / STAGES;
        if (kb >= STAGES && !mbar_wait(empty_bar(s), (r - 1) & 1, budget, status, abort_flag)) break;
        mbar_arrive_expect_tx(full_bar(s), L::STAGE_BYTES);
        tma_load_2d(sA + s * L::A_BYTES, &tmA, full_bar(s), kb * BK, static_cast<int32_t>(m0));
        tma_load_2d(sB + s * L::B_BYTES, &tmB, full_bar(s), kb * BK, static_cast<int32_t>(n0));
        ++issued;
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_i8(BM, BN);
      bool ok = true;
      for (int kb = 0; kb < KB; ++kb) {
        const int s = kb % STAGES;
        const int r = kb / STAGES;
        if (!mbar_wait(full_bar(s), r & 1, budget, status, abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint64_t ad = sdesc_k_sw128(sA + s * L::A_BYTES);
        const uint64_t bd = sdesc_k_sw128(sB + s * L::B_BYTES);
#pragma unroll
        for (int k = 0; k < BK / 32; ++k)
          mma_i8(tmem, ad + 2u * k, bd + 2u * k, idesc, (kb | k) != 0 ? 1u : 0u);
        mma_any = true;
        mma_commit(empty_bar(s));
      }
      if (ok) mma_commit(acc_bar);
      griddep_launch_dependents();
    }
  } else {
    // epilogue warps 2..5: TMEM lane quarter (warp % 4) = token rows 32q .. 32q+31
    const int et = threadIdx.x - 64;
    if (!OUT_I32) {
      for (int i = et; i < BN; i += 128) {
        const int64_t n = n0 + i;
        sw_s[i] = n < g.N ? g.sw[n] : 0.0f;
        bias_s[i] = (g.bias != nullptr && n < g.N) ? __half2float(g.bias[n]) : 0.0f;
      }
    }
    named_bar_sync(1, 128);
    if (mbar_wait(acc_bar, 0, budget, status, abort_flag)) {
      tc_fence_after();
      const int q = warp & 3;
      const int64_t row = m0 + 32 * q + lane;
      const bool row_ok = row < g.M;
      const float sxr = (!OUT_I32 && row_ok) ? g.sx[row] : 0.0f;
      // this warp's 32 x 32 blocks go out through its 4 KB staging, row by
      // row (coalesced row segments instead of one row per lane)
      const uint32_t stg = sbase + L::STG + static_cast<uint32_t>(warp - 2) * 4096u;
      const int64_t row0 = m0 + 32 * q;
      const int brows = g.M - row0 < 32 ? static_cast<int>(g.M - row0) : 32;  // warp-uniform
#pragma unroll 1
      for (int cc = 0; cc < BN / 32; ++cc) {
        uint32_t v[32];
        tmem_ld_32x32b_x32(tmem + (static_cast<uint32_t>(32 * q) << 16) + 32u * cc, v);
        tmem_ld_wait();
        const int64_t col0 = n0 + 32 * cc;
        if (brows <= 0 || col0 >= g.N) continue;  // warp-uniform
        const int bcols = g.N - col0 < 32 ? static_cast<int>(g.N - col0) : 32;
        if constexpr (OUT_I32) {
          warp_store_rows_i32(stg, v, g.acc + row0 * g.N + col0, g.N, brows, bcols);
        } else {
          __align__(16) __half h[32];
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            float f = dequant_f32(static_cast<int32_t>(v[j]), sxr, sw_s[32 * cc + j]);
            if (g.bias != nullptr) f = __fadd_rn(f, bias_s[32 * cc + j]);
            h[j] = __float2half_rn(f);
          }
          if constexpr (ROWS) {
            warp_store_rows_f16(stg, h, g.y + row0 * g.N + col0, g.N, brows, bcols);
          } else if (lane < brows) {
            __half* dst = g.y + (row0 + lane) * g.N + col0;
            if (bcols == 32) {
#pragma unroll
              for (int j = 0; j < 4; ++j)
                reinterpret_cast<uint4*>(dst)[j] = reinterpret_cast<const uint4*>(h)[j];
            } else {
#pragma unroll
              for (int j = 0; j < 32; ++j)
                if (j < bcols) dst[j] = h[j];
            }
          }
        }
      }
    }
  }

  // teardown: every tcgen05.ld completed (wait::ld); after an abort, wait
  // (bounded) for the MMAs and TMA loads this CTA issued before freeing TMEM.
  tc_fence_before();
  __syncthreads();
  if (*abort_flag) {
    if (warp == 1 && lane == 0 && mma_any) {
      mma_commit(drain_bar);
      mbar_drain(drain_bar, 0, budget);
    }
    if (warp == 0 && lane == 0) {
      for (int s = 0; s < STAGES && s < issued; ++s) {
        const int last = ((issued - 1 - s) / STAGES) * STAGES + s;  // last kb issued to stage s
        mbar_drain(full_bar(s), (last / STAGES) & 1, budget);
      }
    }
    __syncthreads();
  }
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, BN);
  }
}

template <int BN, int STAGES, bool OUT_I32, bool ROWS>
cudaError_t launch_cfg(const GemmArgs& g, const Ctx& c) {
  using L = TiledLayout<BN, STAGES, ROWS>;
  static bool attr_set[64] = {false};
  const int dev = c.device < 64 ? c.device : 63;
  if (!attr_set[dev]) {
    cudaError_t e = cudaFuncSetAttribute(k_gemm_tiled<BN, STAGES, OUT_I32, ROWS>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(L::SMEM));
    if (e != cudaSuccess) return e;
    attr_set[dev] = true;
  }
  CUtensorMap tmA, tmB;
  if (!make_tmap_i8(&tmA, g.xq, g.K, g.M, BK, BM)) return cudaErrorInvalidValue;
  if (!make_tmap_i8(&tmB, g.wq, g.K, g.N, BK, BN)) return cudaErrorInvalidValue;
  dim3 grid(static_cast<unsigned>((g.N + BN - 1) / BN), static_cast<unsigned>((g.M + BM - 1) / BM));
  return launch_pdl(k_gemm_tiled<BN, STAGES, OUT_I32, ROWS>, grid, dim3(kThreads), L::SMEM, c.stream, tmA, tmB, g,
                    c.status, c.budget_ns);
}

}  // namespace

cudaError_t launch_gemm_tiled(const GemmArgs& g, const Ctx& c) {
  if (g.acc != nullptr) return launch_cfg<256, 4, true, true>(g, c);
  if (g.N % 8 != 0) return launch_cfg<256, 4, false, true>(g, c);  // fp16 rows not 16-byte aligned
  return launch_cfg<256, 4, false, false>(g, c);
}

}  // namespace sq
