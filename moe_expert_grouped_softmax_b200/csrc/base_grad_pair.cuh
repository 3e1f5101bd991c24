// Base-weight gradients of full fine-tuning on CTA pairs: the sums of
// base_grad_kernel (per expert e with rows [a, b): dW1[e] = dZ1[a:b]^T Xp[a:b],
// dW2[e] = dZ2[a:b]^T h[a:b]) with 256 x Nt output tiles on a pair of CTAs
// (tcgen05 cta_group::2: M = 256 output rows p, 128 in each CTA's shared
// memory and TMEM; N = Nt output columns q, Nt / 2 of the V columns in each
// CTA), so that a CTA streams two thirds of the operand bytes per FLOP of the
// single-CTA 128 x 256 tile.  Nt = 256, or 128 for a last column tile with at
// most 128 columns (each CTA still loads two 64-column V atoms, so that every
// stage carries the same bytes).
//
// The loads of both CTAs complete on the leader's barrier of the stage (the
// pair form of the TMA copy), as in the pair GEMMs.  The reduction runs over
// the expert's rows in 64-row chunks, in the same order for every tile
// (deterministic); in an expert's last chunk the rows of the next expert are
// zeroed in both CTAs' U tiles by the leader's MMA warp (its own tile
// directly, the peer's through distributed shared memory) before it issues.
// Experts with no rows get exact zeros.  Tiles are (expert, problem, p-tile,
// q-tile), experts in decreasing order of their row counts.
#pragma once

#include "base_grad.cuh"
#include "gemm_pair.cuh"

namespace moe {

#ifndef MOE_BGP_EPI_WARPS
#define MOE_BGP_EPI_WARPS 4
#endif

struct BaseGradPairCfg {
  static constexpr int BK = 64;                      // rows (K) per stage
  static constexpr int U_BYTES = BK * 128 * 2;       // this CTA's 128 p columns
  static constexpr int V_BYTES = BK * 128 * 2;       // two 64-column q atoms
  static constexpr int STAGE_BYTES = U_BYTES + V_BYTES;
  // barriers and counters, then s_off [E + 1], the expert order [E] and 33
  // bucket cursors
  static constexpr int MISC_BYTES = 512 + 4 * (520 + 520 + 64);
  static constexpr int NS_FIT = (kSmemOptin - 1024 - MISC_BYTES) / STAGE_BYTES;
  static constexpr int NS = NS_FIT > 8 ? 8 : NS_FIT;
  static constexpr int SMEM_BYTES = 1024 + NS * STAGE_BYTES + MISC_BYTES;
  // producer, MMA (leader), epilogue warps: one per TMEM lane quarter (4), or
  // two per quarter draining half the columns each (8)
  static constexpr int EPI_WARPS = MOE_BGP_EPI_WARPS;
  static constexpr int THREADS = 64 + 32 * EPI_WARPS;
  static constexpr int ACC_STRIDE = 256;
  static constexpr int TMEM_COLS = 512;
  static_assert(NS >= 3, "base-gradient pair kernel stages");
  static_assert((2 * NS + 8) * 8 + 32 <= 512, "barrier area");
};

// Output columns of the tile: 256, or 128 when at most 128 remain.
__device__ __forceinline__ int bg_pair_nt(const BaseGradProblem& p, int qt) {
  return p.Q - qt * 256 <= 128 ? 128 : 256;
}

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(BaseGradPairCfg::THREADS, 1)
    base_grad_pair_kernel(const __grid_constant__ CUtensorMap tmU0,
                          const __grid_constant__ CUtensorMap tmU1,
                          const __grid_constant__ CUtensorMap tmV0,
                          const __grid_constant__ CUtensorMap tmV1,
                          const __grid_constant__ BaseGradArgs args) {
  using C = BaseGradPairCfg;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t* sStage = smem;
  uint64_t* full = reinterpret_cast<uint64_t*>(sStage + C::NS * C::STAGE_BYTES);
  uint64_t* empty = full + C::NS;
  uint64_t* acc_full = empty + C::NS;
  uint64_t* acc_empty = acc_full + 2;
  uint64_t* final_bar = acc_empty + 2;
  uint64_t* peer_done = final_bar + 1;  // leader: the peer has finished
  uint64_t* drained = peer_done + 1;    // peer: its copies have landed
  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(drained + 1);
  volatile int* s_abort = reinterpret_cast<volatile int*>(s_tmem + 1);
  // stage copies issued by this CTA's producer ([0]); the peer's count is
  // written into the leader's [2] at teardown
  int* s_issued = reinterpret_cast<int*>(s_tmem + 4);
  int* s_off = reinterpret_cast<int*>(smem + C::NS * C::STAGE_BYTES + 512);
  int* s_eorder = s_off + 520;
  int* s_bcur = s_eorder + 520;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;
  const int pair = blockIdx.x >> 1, npairs = gridDim.x >> 1;
  const uint64_t wait_ns = args.wait_ns;

  if (threadIdx.x == 0) {
    for (int i = 0; i < C::NS; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&acc_full[i], 1);
      mbar_init(&acc_empty[i], 2 * C::EPI_WARPS);  // both CTAs' epilogue warps
    }
    mbar_init(final_bar, 1);
    mbar_init(peer_done, 1);
    mbar_init(drained, 1);
    for (int i = 0; i < 4; ++i) s_issued[i] = 0;
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
    tmem_alloc_pair(s_tmem, C::TMEM_COLS);
    tmem_relinquish_pair();
  }
  // everything above touches only shared memory, TMEM and the kernel's
  // parameters; the preceding kernel's outputs are read from here on
  griddep_sync();
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
  cluster_sync_all();  // both CTAs' barriers initialised, TMEM allocated
  tc_fence_after();
  const uint32_t tmem_base = *s_tmem;
  const int total = args.total_tiles;
  auto lead = [&](const void* p) { return mapa_shared(smem_u32(p), 0); };

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      const uint64_t pol = policy_evict_normal();
      int stage = 0;
      uint32_t phase = 0;
      int n_st = 0;
      bool ok = true;
      for (int tile = pair; tile < total && ok; tile += npairs) {
        int pi, e, pt, qt;
        base_grad_decode(args, s_eorder, tile, pi, e, pt, qt);
        const int a = s_off[e], b = s_off[e + 1];
        const int nk = (b - a + C::BK - 1) / C::BK;
        const int nh = bg_pair_nt(args.prob[pi], qt) >> 1;  // this CTA's q columns
        const int p0 = pt * 256 + static_cast<int>(rank) * 128;
        const int q0 = qt * 256 + static_cast<int>(rank) * nh;
        const CUtensorMap* tu = pi ? &tmU1 : &tmU0;
        const CUtensorMap* tv = pi ? &tmV1 : &tmV0;
        for (int c = 0; c < nk; ++c) {
          if (!mbar_wait(&empty[stage], phase ^ 1, s_abort, wait_ns)) { ok = false; break; }
          uint8_t* st = sStage + stage * C::STAGE_BYTES;
          const int y = a + C::BK * c;  // a row index: no alignment rule
          const uint32_t fb = lead(&full[stage]);
          if (leader) mbar_arrive_expect_tx(&full[stage], 2 * C::STAGE_BYTES);
          tma_load_2d_pair_hint(st, tu, fb, p0, y, pol);
          tma_load_2d_pair_hint(st + 8192, tu, fb, p0 + 64, y, pol);
          tma_load_2d_pair_hint(st + C::U_BYTES, tv, fb, q0, y, pol);
          tma_load_2d_pair_hint(st + C::U_BYTES + kMnAtomBytes, tv, fb, q0 + 64, y, pol);
          ++n_st;
          if (++stage == C::NS) {
            stage = 0;
            phase ^= 1;
          }
        }
      }
      s_issued[0] = n_st;
    }
  } else if (warp == 1) {
    if (leader) {
      // ---------------------------------------------------------- MMA (leader)
      constexpr uint16_t kBoth = 0x3;
      int stage = 0;
      uint32_t phase = 0;
      int local = 0;
      bool ok = true;
      for (int tile = pair; ok && tile < total; tile += npairs, ++local) {
        int pi, e, pt, qt;
        base_grad_decode(args, s_eorder, tile, pi, e, pt, qt);
        const int a = s_off[e], b = s_off[e + 1];
        const int nk = (b - a + C::BK - 1) / C::BK;
        const uint32_t idesc = idesc_bf16_f32(256, bg_pair_nt(args.prob[pi], qt), true, true);
        const int bb = local & 1;
        const uint32_t use = (local >> 1) & 1;
        const uint32_t t_acc = tmem_base + bb * C::ACC_STRIDE;
        if (!warp_wait_cluster(&acc_empty[bb], use ^ 1, s_abort, wait_ns)) { ok = false; break; }
        tc_fence_after();
        for (int c = 0; c < nk; ++c) {
          if (!warp_wait(&full[stage], phase, s_abort, wait_ns)) { ok = false; break; }
          uint8_t* st = sStage + stage * C::STAGE_BYTES;
          const int hi = b - (a + C::BK * c);  // rows of this expert in the chunk
          if (hi < C::BK) {
            // zero rows [hi, BK) of both CTAs' U tiles (two 64-column atoms
            // each; a row is 128 contiguous bytes, the swizzle only permutes
            // 16-byte chunks inside it)
            const uint32_t peer_st = mapa_shared(smem_u32(st), 1);
            const uint4 z4 = make_uint4(0, 0, 0, 0);
            for (int h = 0; h < 2; ++h) {
              uint4* z = reinterpret_cast<uint4*>(st + h * 8192);
              for (int i = hi * 8 + lane; i < C::BK * 8; i += 32) {
                z[i] = z4;
                st_shared_cluster_v4(peer_st + h * 8192 + 16 * i, z4);
              }
            }
            fence_proxy_async_all();
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
              umma_bf16_pair(t_acc, da, db, idesc, (c | kk) ? 1u : 0u);
            }
            umma_commit_pair_mc(&empty[stage], kBoth);
          }
          __syncwarp();
          if (++stage == C::NS) {
            stage = 0;
            phase ^= 1;
          }
        }
        if (!ok) break;
        if (elect_one()) umma_commit_pair_mc(&acc_full[bb], kBoth);
        __syncwarp();
      }
      // all of the leader's MMAs complete -> both CTAs' final_bar
      if (elect_one()) umma_commit_pair_mc(final_bar, kBoth);
      __syncwarp();
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int ew = warp & 3;  // TMEM lane quarter this warp may access
    const int ehalf = C::EPI_WARPS == 8 ? (warp - 2) >> 2 : 0;  // its share of the columns
    const uint32_t lane_base = static_cast<uint32_t>(ew * 32) << 16;
    const uint64_t pol = policy_evict_first();  // gradients stream out of L2
    int local = 0;
    for (int tile = pair; tile < total; tile += npairs, ++local) {
      int pi, e, pt, qt;
      base_grad_decode(args, s_eorder, tile, pi, e, pt, qt);
      const BaseGradProblem& pr = args.prob[pi];
      const bool any = s_off[e + 1] > s_off[e];
      const int nt = bg_pair_nt(pr, qt);
      const int bb = local & 1;
      const uint32_t use = (local >> 1) & 1;
      if (!warp_wait(&acc_full[bb], use, s_abort, wait_ns)) break;
      tc_fence_after();
      const int p = pt * 256 + static_cast<int>(rank) * 128 + ew * 32 + lane;
      const int q0 = qt * 256;
      __nv_bfloat16* orow = pr.out + (static_cast<size_t>(e) * pr.P + p) * pr.Q + q0;
      const uint32_t t_acc = tmem_base + lane_base + bb * C::ACC_STRIDE;
      const int c_lo = C::EPI_WARPS == 8 ? ehalf * (nt >> 1) : 0;
      const int c_hi = C::EPI_WARPS == 8 ? c_lo + (nt >> 1) : nt;
      for_chunks<256>([&](int c, auto w) {
        constexpr int W = decltype(w)::value;
        if (c < c_lo || c >= c_hi) return;
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
      // the accumulator's TMEM reads have completed (tcgen05.wait::ld); the
      // release needs no ordering of the output stores
      if (lane == 0) MOE_ACC_RELEASE(lead(&acc_empty[bb]));
    }
  }

  // ---------------------------------------------------------------- teardown
  tc_fence_before();
  __syncthreads();
  if (threadIdx.x == 0) {
    // the leader's MMAs read this CTA's shared memory and write its TMEM
    drain_wait(final_bar, 0, wait_ns);
    if (!leader) {
      // publish this CTA's copy count (the release orders it before the
      // arrive, after which nothing else arrives from this CTA), then wait
      // for the leader to see every copy land
      st_shared_cluster_s32(lead(&s_issued[2]), s_issued[0]);
      mbar_arrive_cluster(lead(peer_done));
      drain_wait(drained, 0, wait_ns);
    } else {
      drain_wait_cluster(peer_done, 0, wait_ns);
      drain_pair_copies(full, C::NS, C::STAGE_BYTES, s_issued[0], s_issued[2], wait_ns);
      mbar_arrive_cluster(mapa_shared(smem_u32(drained), 1));
    }
  }
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, C::TMEM_COLS);
  }
}

}  // namespace moe
