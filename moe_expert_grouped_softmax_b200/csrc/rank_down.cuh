// Rank-r down-projections on their own pass (used with the CTA-pair GEMMs,
// whose weight operand then holds whole weight atoms only): per expert e
// with rows [a, b)
//   V[a:b] = s * U[a:b] F[e]       [M_e, r]
// Backward: (U, F) = (dZ2, B2) -> s dZ2 B2 and (dZ1, B1) -> s dZ1 B1, with
// F[e] [K, r] read in place as an MN-major operand (one r-column atom).
// Forward: (U, F) = (Xp, A1^T) -> s Xp A1^T and (h, A2^T) -> s h A2^T, with
// F[e]^T = A[e] [r, K] read in place as a K-major operand.  U [R, K] is a
// K-major operand.  Written twice: row-major [R, r] (the A operand of the
// up-projection MMA) and transposed [r, ldR] (the saved / LoRA-gradient
// operand).  Memory-bound: U is streamed once.
#pragma once

#include "gemm.cuh"

namespace moe {

template <int RK, bool KMAJ_F>
struct RankDownCfg {
  static constexpr int BM = 128, BK = 64;
  static constexpr int A_BYTES = BM * BK * 2;
  static constexpr int B_BYTES = BK * RK * 2;
  static constexpr int STAGE_BYTES = (A_BYTES + B_BYTES + 1023) / 1024 * 1024;
  // CTAs per SM: two CTAs of four stages keep as many bytes in flight as
  // one of eight, and one CTA's prologue and pipeline fill overlap the
  // other's streaming
#ifndef MOE_RANK_CTAS
#define MOE_RANK_CTAS 2
#endif
  static constexpr int CTAS_PER_SM = MOE_RANK_CTAS;
  static constexpr int NS = 8 / CTAS_PER_SM;
  static constexpr int MISC_BYTES = 256 + 8 * 520;
  static constexpr int SMEM_BYTES = 1024 + NS * STAGE_BYTES + MISC_BYTES;
  static constexpr int ACC_STRIDE = RK < 32 ? 32 : RK;
  static constexpr int TMEM_COLS = 2 * ACC_STRIDE < 32 ? 32 : 2 * ACC_STRIDE;
  // MN-major factor atom: r columns wide (32-, 64- or 128-byte swizzle)
  static constexpr uint32_t FLAYOUT =
      RK == 16 ? kLayoutSW32 : (RK == 32 ? kLayoutSW64 : kLayoutSW128);
  static constexpr uint32_t FSBO = 8 * RK * 2;  // next 8 K-rows
  static_assert(SMEM_BYTES <= kSmemOptin, "rank-down shared memory");
};

struct RankDownArgs {
  const int32_t* offsets;
  int E, R, K;
  int k_rows;               // rows of F per expert (= K)
  float s;
  __nv_bfloat16* out_rm;    // [R, r]
  __nv_bfloat16* out_t;     // [r, ld_t]
  int ld_t;
  uint64_t wait_ns;
};

template <int RK, bool KMAJ_F>
__global__ void __launch_bounds__(192, RankDownCfg<RK, KMAJ_F>::CTAS_PER_SM)
    rank_down_kernel(const __grid_constant__ CUtensorMap tmU,
                     const __grid_constant__ CUtensorMap tmF, const RankDownArgs args) {
  griddep_sync();  // before any global memory access
  using C = RankDownCfg<RK, KMAJ_F>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t* sStage = smem;
  uint64_t* full = reinterpret_cast<uint64_t*>(sStage + C::NS * C::STAGE_BYTES);
  uint64_t* empty = full + C::NS;
  uint64_t* acc_full = empty + C::NS;
  uint64_t* acc_empty = acc_full + 2;
  uint64_t* drain_bar = acc_empty + 2;
  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(drain_bar + 1);
  volatile int* s_abort = reinterpret_cast<volatile int*>(s_tmem + 1);
  int* s_off = reinterpret_cast<int*>(s_tmem + 4);
  int* s_mstart = s_off + 520;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int E = args.E;
  const uint64_t wait_ns = args.wait_ns;

  if (threadIdx.x == 0) {
    for (int i = 0; i < C::NS; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&acc_full[i], 1);
      mbar_init(&acc_empty[i], 4);
    }
    mbar_init(drain_bar, 1);
    *s_abort = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tmU);
    prefetch_tmap(&tmF);
  }
  if (warp == 1) {
    tmem_alloc(s_tmem, C::TMEM_COLS);
    tmem_relinquish();
  }
  if (warp == 2) build_tile_table(args.offsets, E, args.R, s_off, s_mstart, lane);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();

  const uint32_t tmem_base = *s_tmem;
  const int total = s_mstart[E];  // one n-tile: tiles are (expert, 128-row m-tile)
  const int k_iters = (args.K + C::BK - 1) / C::BK;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      const uint64_t pol_u = policy_evict_first();  // streamed once
      int stage = 0;
      uint32_t phase = 0;
      int armed = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < total && ok; tile += gridDim.x) {
        int e, mt, nt;
        decode_tile(tile, 1, s_mstart, E, e, mt, nt);
        const int row0 = s_off[e] + mt * C::BM;
        for (int kt = 0; kt < k_iters; ++kt) {
          if (!mbar_wait(&empty[stage], phase ^ 1, s_abort, wait_ns)) { ok = false; break; }
          uint8_t* st = sStage + stage * C::STAGE_BYTES;
          mbar_arrive_expect_tx(&full[stage], C::A_BYTES + C::B_BYTES);
          tma_load_2d_hint(st, &tmU, &full[stage], kt * C::BK, row0, pol_u);
          if constexpr (KMAJ_F)  // A[e] rows: r rows x 64 K-columns
            tma_load_2d(st + C::A_BYTES, &tmF, &full[stage], kt * C::BK, e * RK);
          else                   // B[e] rows: 64 K-rows x r columns
            tma_load_2d(st + C::A_BYTES, &tmF, &full[stage], 0, e * args.k_rows + kt * C::BK);
          if (armed < C::NS) ++armed;
          if (++stage == C::NS) {
            stage = 0;
            phase ^= 1;
          }
        }
      }
      for (int i = 0; i < armed; ++i) {
        int s = stage - 1 - i;
        uint32_t ph = phase;
        if (s < 0) {
          s += C::NS;
          ph ^= 1;
        }
        drain_wait(&full[s], ph, wait_ns);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    constexpr uint32_t kIdesc = idesc_bf16_f32(128, RK, false, !KMAJ_F);
    int stage = 0;
    uint32_t phase = 0;
    int local = 0;
    bool ok = true;
    for (int tile = blockIdx.x; ok && tile < total; tile += gridDim.x, ++local) {
      const int bb = local & 1;
      const uint32_t use = (local >> 1) & 1;
      const uint32_t t_acc = tmem_base + bb * C::ACC_STRIDE;
      if (!warp_wait(&acc_empty[bb], use ^ 1, s_abort, wait_ns)) { ok = false; break; }
      tc_fence_after();
      for (int kt = 0; kt < k_iters; ++kt) {
        if (!warp_wait(&full[stage], phase, s_abort, wait_ns)) { ok = false; break; }
        if (elect_one()) {
          const uint32_t a0 = smem_u32(sStage + stage * C::STAGE_BYTES);
          const uint32_t b0 = a0 + C::A_BYTES;
#pragma unroll
          for (int kk = 0; kk < C::BK / 16; ++kk)
            umma_bf16(t_acc, smem_desc(a0 + kk * 32, 16, 1024, kLayoutSW128),
                      KMAJ_F ? smem_desc(b0 + kk * 32, 16, 1024, kLayoutSW128)
                             : smem_desc(b0 + kk * 16 * RK * 2, 16, C::FSBO, C::FLAYOUT),
                      kIdesc, (kt | kk) ? 1u : 0u);
          umma_commit(&empty[stage]);
        }
        __syncwarp();
        if (++stage == C::NS) {
          stage = 0;
          phase ^= 1;
        }
      }
      if (!ok) break;
      if (elect_one()) umma_commit(&acc_full[bb]);
      __syncwarp();
    }
    if (elect_one()) umma_commit(drain_bar);
    __syncwarp();
    drain_wait(drain_bar, 0, wait_ns);
  } else {
    // ------------------------------------------------------------ epilogue
    const int ew = warp & 3;
    const int row_in_tile = ew * 32 + lane;
    const uint32_t lane_base = static_cast<uint32_t>(ew * 32) << 16;
    const uint64_t pol = policy_evict_last();  // read again by the next kernels
    int local = 0;
    for (int tile = blockIdx.x; tile < total; tile += gridDim.x, ++local) {
      int e, mt, nt;
      decode_tile(tile, 1, s_mstart, E, e, mt, nt);
      const int grow = s_off[e] + mt * C::BM + row_in_tile;
      const bool rvalid = grow < s_off[e + 1];
      const int bb = local & 1;
      const uint32_t use = (local >> 1) & 1;
      if (!warp_wait(&acc_full[bb], use, s_abort, wait_ns)) break;
      tc_fence_after();
      float v[RK];
#pragma unroll
      for (int c = 0; c < RK; c += 16)
        tmem_ld16(tmem_base + lane_base + bb * C::ACC_STRIDE + c, v + c);
      tmem_ld_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&acc_empty[bb]);
      if (rvalid) {
#pragma unroll
        for (int i = 0; i < RK; ++i) v[i] *= args.s;
        store_row_bf16<RK>(args.out_rm + static_cast<size_t>(grow) * RK, v, RK, pol);
#pragma unroll
        for (int q = 0; q < RK; ++q)
          args.out_t[static_cast<size_t>(q) * args.ld_t + grow] = __float2bfloat16_rn(v[q]);
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem_base, C::TMEM_COLS);
  }
}

}  // namespace moe
