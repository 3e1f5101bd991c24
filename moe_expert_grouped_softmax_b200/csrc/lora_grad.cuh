// a9: per-expert LoRA weight gradients with the base weights frozen.
//
// All four gradients have one shape: for expert e with rows [a, b),
//   G_e[p, q] = sum_{m in [a, b)} U[m, p] * V[m, q]      (p < P, q < r)
// with (U, V) = (Xp, s dZ1 B1) -> dA1^T, (dZ1, s Xp A1^T) -> dB1,
//               (h, s dZ2 B2) -> dA2^T, (dZ2, s h A2^T) -> dB2.
// The rank-r factors V were written transposed ([r, ldR]) by the GEMM
// epilogues, already multiplied by s.  One tcgen05 MMA per 16 rows:
// M = 128 columns p of U (an MN-major operand straight from the row-major
// activations), N = r, K = rows.  The reduction over rows runs in a fixed
// order inside one CTA, so the result is deterministic.  The ragged tail of
// an expert is zeroed in shared memory before its MMA.  Experts with no rows
// get exact zeros.
//
// Tiles are (expert, problem, 128-column block), experts in decreasing order
// of their row counts (power-of-two buckets, expert index inside a bucket),
// so that the long reductions of heavily loaded experts start first and the
// short ones fill in behind them on the persistent CTAs.  Every CTA computes
// the same order, and each tile is still reduced by one CTA in a fixed
// order: the results do not depend on it.
#pragma once

#include "ptx.cuh"
#include "expert_order.cuh"

namespace moe {

struct GradProblem {
  int P;               // columns of U
  int p_tiles;         // ceil(P / 128)
  int tile_begin;      // first tile of this problem inside an expert's tiles
  int transpose_out;   // 1: out[e][q][p]; 0: out[e][p][q]
  __nv_bfloat16* out;
};

struct GradArgs {
  const int32_t* offsets;
  int E, R;
  int tiles_per_expert;  // sum of the problems' p_tiles
  int total_tiles;       // E * tiles_per_expert
  GradProblem prob[4];
  uint64_t wait_ns;
};

// Resident CTAs per SM, each with MOE_GRAD_NS pipeline stages (measured
// against one CTA with 8 stages: 2 CTAs with 4 stages each 214 -> 166 us on
// the gpt-oss-20b shape, 393 -> 332 us on the Qwen3-30B-A3B one; one CTA's
// per-tile hand-off overlaps the other's loads).
#ifndef MOE_GRAD_CTAS_PER_SM
#define MOE_GRAD_CTAS_PER_SM 2
#endif
#ifndef MOE_GRAD_NS
#define MOE_GRAD_NS (8 / MOE_GRAD_CTAS_PER_SM)
#endif

template <int RK>
struct GradCfg {
  static constexpr int U_BYTES = 64 * 128 * 2;   // 64 rows x 128 columns
  static constexpr int V_BYTES = RK * 64 * 2;    // r rows x 64 columns
  static constexpr int STAGE_BYTES = U_BYTES + V_BYTES;
  static constexpr int CTAS_PER_SM = MOE_GRAD_CTAS_PER_SM;
  static constexpr int NS = MOE_GRAD_NS;
  // barriers, then s_off [E + 1], the expert order [E] and 33 bucket cursors
  static constexpr int MISC_BYTES = 256 + 4 * (520 + 520 + 64);
  static constexpr int SMEM_BYTES = 1024 + NS * STAGE_BYTES + MISC_BYTES;
  static constexpr int ACC_COLS = RK;
  static constexpr int TMEM_COLS = (2 * RK) < 32 ? 32 : 2 * RK;
  static_assert(SMEM_BYTES <= kSmemOptin, "grad kernel shared memory");
};

__device__ __forceinline__ void grad_decode(const GradArgs& a, const int* s_eorder, int tile,
                                            int& pi, int& e, int& pt) {
  const int slot = tile / a.tiles_per_expert;
  const int rem = tile - slot * a.tiles_per_expert;
  pi = 0;
#pragma unroll
  for (int i = 1; i < 4; ++i)
    if (rem >= a.prob[i].tile_begin) pi = i;
  pt = rem - a.prob[pi].tile_begin;
  e = s_eorder[slot];
}

template <int RK>
__global__ void __launch_bounds__(192, GradCfg<RK>::CTAS_PER_SM)
    lora_grad_kernel(const __grid_constant__ CUtensorMap tmU0,
                     const __grid_constant__ CUtensorMap tmU1,
                     const __grid_constant__ CUtensorMap tmU2,
                     const __grid_constant__ CUtensorMap tmU3,
                     const __grid_constant__ CUtensorMap tmV0,
                     const __grid_constant__ CUtensorMap tmV1,
                     const __grid_constant__ CUtensorMap tmV2,
                     const __grid_constant__ CUtensorMap tmV3,
                     const GradArgs args) {
  griddep_sync();  // before any global memory access
  using C = GradCfg<RK>;
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
  int* s_eorder = s_off + 520;
  int* s_bcur = s_eorder + 520;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint64_t wait_ns = args.wait_ns;
  const CUtensorMap* tmU[4] = {&tmU0, &tmU1, &tmU2, &tmU3};
  const CUtensorMap* tmV[4] = {&tmV0, &tmV1, &tmV2, &tmV3};

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
    for (int i = 0; i < 4; ++i) {
      prefetch_tmap(tmU[i]);
      prefetch_tmap(tmV[i]);
    }
  }
  if (warp == 1) {
    tmem_alloc(s_tmem, C::TMEM_COLS);
    tmem_relinquish();
  }
  if (warp == 2) {
    bool bad = false;
    for (int e = lane; e <= args.E; e += 32) {
      const int v = args.offsets[e];
      s_off[e] = v;
      if (v < 0 || v > args.R) bad = true;
      if (e > 0 && v < args.offsets[e - 1]) bad = true;
    }
    if (lane == 0 && (args.offsets[0] != 0 || args.offsets[args.E] != args.R)) bad = true;
    if (__any_sync(0xffffffffu, bad)) {
      if (lane == 0) set_status(5);
      for (int e = lane; e <= args.E; e += 32) s_off[e] = 0;  // all experts empty
    }
    __syncwarp();
    expert_load_order(s_off, args.E, s_eorder, s_bcur, lane);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *s_tmem;
  const int total = args.total_tiles;

  if (warp == 0) {
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      int armed = 0;
      for (int tile = blockIdx.x; tile < total; tile += gridDim.x) {
        int pi, e, pt;
        grad_decode(args, s_eorder, tile, pi, e, pt);
        const int a = s_off[e], b = s_off[e + 1];
        const int a8 = a & ~7;  // TMA x coordinate of V must be 16-byte aligned
        const int nk = (b > a) ? ((b - a8 + 63) >> 6) : 0;
        bool ok = true;
        for (int c = 0; c < nk; ++c) {
          if (!mbar_wait(&empty[stage], phase ^ 1, s_abort, wait_ns)) { ok = false; break; }
          uint8_t* st = sStage + stage * C::STAGE_BYTES;
          const int y = a8 + 64 * c;
          mbar_arrive_expect_tx(&full[stage], C::STAGE_BYTES);
          tma_load_2d(st, tmU[pi], &full[stage], pt * 128, y);
          tma_load_2d(st + 8192, tmU[pi], &full[stage], pt * 128 + 64, y);
          tma_load_2d(st + C::U_BYTES, tmV[pi], &full[stage], y, 0);
          if (armed < C::NS) ++armed;
          if (++stage == C::NS) {
            stage = 0;
            phase ^= 1;
          }
        }
        if (!ok) break;
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
    constexpr uint32_t kIdesc = idesc_bf16_f32(128, RK, true, false);
    int stage = 0;
    uint32_t phase = 0;
    int local = 0;
    for (int tile = blockIdx.x; tile < total; tile += gridDim.x, ++local) {
      int pi, e, pt;
      grad_decode(args, s_eorder, tile, pi, e, pt);
      const int a = s_off[e], b = s_off[e + 1];
      const int a8 = a & ~7;
      const int nk = (b > a) ? ((b - a8 + 63) >> 6) : 0;
      const int bb = local & 1;
      const uint32_t use = (local >> 1) & 1;
      const uint32_t t_acc = tmem_base + bb * C::ACC_COLS;
      if (!warp_wait(&acc_empty[bb], use ^ 1, s_abort, wait_ns)) break;
      tc_fence_after();
      bool ok = true;
      for (int c = 0; c < nk; ++c) {
        if (!warp_wait(&full[stage], phase, s_abort, wait_ns)) { ok = false; break; }
        uint8_t* st = sStage + stage * C::STAGE_BYTES;
        // tile rows are [y, y + 64); only [a, b) belong to this expert.
        const int y = a8 + 64 * c;
        const int lo = max(0, a - y), hi = min(64, b - y);
        if (lo > 0 || hi < 64) {
          // zero the other experts' rows in both 64-column halves of the U
          // tile (a row is 128 contiguous bytes; the swizzle only permutes
          // 16-byte chunks inside it).
          for (int h = 0; h < 2; ++h) {
            uint4* z = reinterpret_cast<uint4*>(st + h * 8192);
            for (int i = lane; i < lo * 8; i += 32) z[i] = make_uint4(0, 0, 0, 0);
            for (int i = hi * 8 + lane; i < 64 * 8; i += 32) z[i] = make_uint4(0, 0, 0, 0);
          }
          fence_proxy_async_smem();
        }
        __syncwarp();
        if (lane == 0) {
          tc_fence_after();
          const uint32_t u0 = smem_u32(st);
          const uint32_t v0 = u0 + C::U_BYTES;
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            const uint64_t da = smem_desc(u0 + kk * 2048, 8192, 1024, kLayoutSW128);
            const uint64_t db = smem_desc(v0 + kk * 32, 16, 1024, kLayoutSW128);
            umma_bf16(t_acc, da, db, kIdesc, (c | kk) ? 1u : 0u);
          }
          umma_commit(&empty[stage]);
        }
        __syncwarp();
        if (++stage == C::NS) {
          stage = 0;
          phase ^= 1;
        }
      }
      if (!ok) break;
      if (lane == 0) umma_commit(&acc_full[bb]);
      __syncwarp();
    }
    if (lane == 0) {
      umma_commit(drain_bar);
      drain_wait(drain_bar, 0, wait_ns);
    }
    __syncwarp();
  } else {
    const int ew = warp & 3;
    const int row_in_tile = ew * 32 + lane;
    const uint32_t lane_base = static_cast<uint32_t>(ew * 32) << 16;
    int local = 0;
    for (int tile = blockIdx.x; tile < total; tile += gridDim.x, ++local) {
      int pi, e, pt;
      grad_decode(args, s_eorder, tile, pi, e, pt);
      const GradProblem& pr = args.prob[pi];
      const int nk = (s_off[e + 1] > s_off[e]) ? 1 : 0;  // any rows at all
      const int bb = local & 1;
      const uint32_t use = (local >> 1) & 1;
      if (!warp_wait(&acc_full[bb], use, s_abort, wait_ns)) break;
      tc_fence_after();
      float v[RK];
      if (nk > 0) {
#pragma unroll
        for (int c = 0; c < RK; c += 16)
          tmem_ld16(tmem_base + lane_base + bb * C::ACC_COLS + c, v + c);
        tmem_ld_wait();
      } else {
#pragma unroll
        for (int i = 0; i < RK; ++i) v[i] = 0.f;
      }
      const int p = pt * 128 + row_in_tile;
      if (p < pr.P) {
        if (pr.transpose_out) {
          __nv_bfloat16* o = pr.out + static_cast<size_t>(e) * RK * pr.P + p;
#pragma unroll
          for (int q = 0; q < RK; ++q) o[static_cast<size_t>(q) * pr.P] = __float2bfloat16_rn(v[q]);
        } else {
          __nv_bfloat16* o = pr.out + (static_cast<size_t>(e) * pr.P + p) * RK;
#pragma unroll
          for (int q = 0; q < RK; q += 8)
            *reinterpret_cast<uint4*>(o + q) = make_uint4(
                pack_bf16x2(v[q + 0], v[q + 1]), pack_bf16x2(v[q + 2], v[q + 3]),
                pack_bf16x2(v[q + 4], v[q + 5]), pack_bf16x2(v[q + 6], v[q + 7]));
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&acc_empty[bb]);
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
