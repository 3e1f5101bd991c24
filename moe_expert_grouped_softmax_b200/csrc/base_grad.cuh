// Base-weight gradients for full fine-tuning (the pages list full
// fine-tuning beside LoRA among what their MoE kernels support): with W1, W2
// trainable, each projection y = x W^T also yields dW = dy^T x, so per expert
// e with rows [a, b)
//   dW1[e] = dZ1[a:b]^T Xp[a:b]   [2I, H]
//   dW2[e] = dZ2[a:b]^T h[a:b]    [H, I]
// Both are G[p, q] = sum_m U[m, p] V[m, q] with a ragged K (the expert's
// rows): M = 128 columns p of U, N = BN columns q of V, both operands
// MN-major straight from the row-major activations.  The reduction over rows
// runs in a fixed order inside one CTA (deterministic).  The rows of the next
// expert inside an expert's last 64-row chunk are zeroed in shared memory
// before its MMA; experts with no rows get exact zeros.  Tiles are (expert,
// problem, p-tile, q-tile), experts in decreasing order of their row counts
// (the same order in every CTA; see expert_order.cuh).
#pragma once

#include "expert_order.cuh"
#include "gemm.cuh"

namespace moe {

struct BaseGradProblem {
  int P, Q;            // columns of U (output rows) and of V (output columns)
  int p_tiles, q_tiles;
  int tile_begin;      // first tile of this problem inside an expert's tiles
  __nv_bfloat16* out;  // [E, P, Q]
};

struct BaseGradArgs {
  const int32_t* offsets;
  int E, R;
  int tiles_per_expert;  // both problems' p_tiles * q_tiles
  int total_tiles;       // E * tiles_per_expert
  BaseGradProblem prob[2];
  uint64_t wait_ns;
};

template <int BN>
struct BaseGradCfg {
  static constexpr int BK = 64;                      // rows per stage
  static constexpr int U_BYTES = BK * 128 * 2;       // 64 rows x 128 columns
  static constexpr int V_BYTES = BK * BN * 2;        // 64 rows x BN columns
  static constexpr int STAGE_BYTES = U_BYTES + V_BYTES;
  // barriers, then s_off [E + 1], the expert order [E] and 33 bucket cursors
  static constexpr int MISC_BYTES = 256 + 4 * (520 + 520 + 64);
  static constexpr int NS_FIT = (kSmemOptin - 1024 - MISC_BYTES) / STAGE_BYTES;
  static constexpr int NS = NS_FIT > 8 ? 8 : NS_FIT;
  static constexpr int SMEM_BYTES = 1024 + NS * STAGE_BYTES + MISC_BYTES;
  static constexpr int ACC_STRIDE = 256;
  static constexpr int TMEM_COLS = 512;
  static_assert(BN % 64 == 0 && BN <= 256, "64-column MN-major atoms, N <= 256");
  static_assert(NS >= 3, "base-gradient kernel stages");
};

__device__ __forceinline__ void base_grad_decode(const BaseGradArgs& a, const int* s_eorder,
                                                 int tile, int& pi, int& e, int& pt, int& qt) {
  const int slot = tile / a.tiles_per_expert;
  const int rem = tile - slot * a.tiles_per_expert;
  pi = rem >= a.prob[1].tile_begin ? 1 : 0;
  const BaseGradProblem& p = a.prob[pi];
  const int local = rem - p.tile_begin;
  pt = local / p.q_tiles;       // q-tiles fastest: CTAs at work share U rows
  qt = local - pt * p.q_tiles;
  e = s_eorder[slot];
}

template <int BN>
__global__ void __launch_bounds__(192, 1)
    base_grad_kernel(const __grid_constant__ CUtensorMap tmU0,
                     const __grid_constant__ CUtensorMap tmU1,
                     const __grid_constant__ CUtensorMap tmV0,
                     const __grid_constant__ CUtensorMap tmV1,
                     const __grid_constant__ BaseGradArgs args) {
  griddep_sync();  // before any global memory access
  using C = BaseGradCfg<BN>;
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
    prefetch_tmap(&tmU0);
    prefetch_tmap(&tmU1);
    prefetch_tmap(&tmV0);
    prefetch_tmap(&tmV1);
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
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      const uint64_t pol = policy_evict_normal();
      int stage = 0;
      uint32_t phase = 0;
      int armed = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < total && ok; tile += gridDim.x) {
        int pi, e, pt, qt;
        base_grad_decode(args, s_eorder, tile, pi, e, pt, qt);
        const int a = s_off[e], b = s_off[e + 1];
        const int nk = (b - a + C::BK - 1) / C::BK;
        for (int c = 0; c < nk; ++c) {
          if (!mbar_wait(&empty[stage], phase ^ 1, s_abort, wait_ns)) { ok = false; break; }
          uint8_t* st = sStage + stage * C::STAGE_BYTES;
          const int y = a + C::BK * c;  // a row index: no alignment rule
          mbar_arrive_expect_tx(&full[stage], C::STAGE_BYTES);
          const CUtensorMap* tu = pi ? &tmU1 : &tmU0;
          const CUtensorMap* tv = pi ? &tmV1 : &tmV0;
          tma_load_2d_hint(st, tu, &full[stage], pt * 128, y, pol);
          tma_load_2d_hint(st + 8192, tu, &full[stage], pt * 128 + 64, y, pol);
#pragma unroll
          for (int i = 0; i < BN / 64; ++i)
            tma_load_2d_hint(st + C::U_BYTES + i * kMnAtomBytes, tv, &full[stage],
                             qt * BN + 64 * i, y, pol);
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
    // (whole warp: tail zeroing is shared by the lanes, issue by one)
    constexpr uint32_t kIdesc = idesc_bf16_f32(128, BN, true, true);
    int stage = 0;
    uint32_t phase = 0;
    int local = 0;
    bool ok = true;
    for (int tile = blockIdx.x; ok && tile < total; tile += gridDim.x, ++local) {
      int pi, e, pt, qt;
      base_grad_decode(args, s_eorder, tile, pi, e, pt, qt);
      const int a = s_off[e], b = s_off[e + 1];
      const int nk = (b - a + C::BK - 1) / C::BK;
      const int bb = local & 1;
      const uint32_t use = (local >> 1) & 1;
      const uint32_t t_acc = tmem_base + bb * C::ACC_STRIDE;
      if (!warp_wait(&acc_empty[bb], use ^ 1, s_abort, wait_ns)) { ok = false; break; }
      tc_fence_after();
      for (int c = 0; c < nk; ++c) {
        if (!warp_wait(&full[stage], phase, s_abort, wait_ns)) { ok = false; break; }
        uint8_t* st = sStage + stage * C::STAGE_BYTES;
        const int hi = b - (a + C::BK * c);  // rows of this expert in the chunk
        if (hi < C::BK) {
          // zero the next expert's rows in both 64-column halves of the U
          // tile (a row is 128 contiguous bytes; the swizzle only permutes
          // 16-byte chunks inside it)
          for (int h = 0; h < 2; ++h) {
            uint4* z = reinterpret_cast<uint4*>(st + h * 8192);
            for (int i = hi * 8 + lane; i < C::BK * 8; i += 32) z[i] = make_uint4(0, 0, 0, 0);
          }
          fence_proxy_async_smem();
        }
        __syncwarp();
        if (elect_one()) {
          tc_fence_after();
          const uint32_t u0 = smem_u32(st);
          const uint32_t v0 = u0 + C::U_BYTES;
#pragma unroll
          for (int kk = 0; kk < C::BK / 16; ++kk) {
            const uint64_t da = smem_desc(u0 + kk * 2048, 8192, 1024, kLayoutSW128);
            const uint64_t db = smem_desc(v0 + kk * 2048, kMnAtomBytes, 1024, kLayoutSW128);
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
    const uint64_t pol = policy_evict_first();  // gradients stream out of L2
    int local = 0;
    for (int tile = blockIdx.x; tile < total; tile += gridDim.x, ++local) {
      int pi, e, pt, qt;
      base_grad_decode(args, s_eorder, tile, pi, e, pt, qt);
      const BaseGradProblem& pr = args.prob[pi];
      const bool any = s_off[e + 1] > s_off[e];
      const int bb = local & 1;
      const uint32_t use = (local >> 1) & 1;
      if (!warp_wait(&acc_full[bb], use, s_abort, wait_ns)) break;
      tc_fence_after();
      const int p = pt * 128 + row_in_tile;
      const int q0 = qt * BN;
      __nv_bfloat16* orow = pr.out + (static_cast<size_t>(e) * pr.P + p) * pr.Q + q0;
      const uint32_t t_acc = tmem_base + lane_base + bb * C::ACC_STRIDE;
      for_chunks<BN>([&](int c, auto w) {
        constexpr int W = decltype(w)::value;
        float v[W];
        if (any) {
          tmem_ld<W>(t_acc + c, v);
          tmem_ld_wait();
        } else {
#pragma unroll
          for (int i = 0; i < W; ++i) v[i] = 0.f;
        }
        if (p < pr.P) store_row_bf16<W>(orow + c, v, pr.Q - q0 - c, pol);
      });
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
