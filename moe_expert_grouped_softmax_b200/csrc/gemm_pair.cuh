// a3, a4, a7, a8 on CTA pairs: the grouped GEMMs with 256-row tiles on the
// 2-SM tensor-core instruction (tcgen05.mma.cta_group::2).
//
// A cluster of two CTAs on two SMs computes one 256-row x Nt-column tile of
// one expert (Nt <= 256, below).  Each CTA stages its own 128 rows of A and
// half (Nt/2 columns) of the weight operand, so every SM moves a third less
// operand data per FLOP than the single-CTA 128-row tile, through shared
// memory as well as from L2.  The even CTA ("leader") issues the MMAs, which read both CTAs'
// shared memory and write both CTAs' TMEM.
//
// Split LoRA: the rank-r down-products (s Xp A1^T, s h A2^T, s dZ2 B2,
// s dZ1 B1) come from their own pass (rank_down_kernel), so the B operand is
// weight columns only.  Each tile's up-projection operands -- its rows of the
// rank-r product and the up factor rows of its columns, both K-major with
// K = r -- are loaded by TMA beside the tile and accumulated into the same
// TMEM tile right after the mainloop: W + s B A is never formed.
//
// Tile width Nt (the MMA's N), per launch: 256 for gate_up forward; down
// forward: the narrowest multiple of 16 that covers N in as many tiles as
// 256 would (N = 2880: 12 tiles of 240, no padded columns); backward: 128 or
// 256 (whole MN-major atoms; any multiple of 16 computes correctly, but
// partial atoms run slower).  B operand of each CTA (Nt / 2 columns):
//   gate_up fwd: [gate j..j+63 | up j..j+63] with j = 128 nt + 64 rank, so
//                every 128 tile columns hold gate and up of the same 64
//                output columns (the SwiGLU epilogue needs both in one
//                thread, also for half tiles);
//   down fwd:    W2 rows Nt nt + Nt/2 rank .. (K-major);
//   backward:    W read in place as [K, N], two MN-major atoms of 64
//                columns from column Nt nt + Nt/2 rank (the MMA reads the
//                first Nt/2).
// Half tiles: an expert's last tile with at most 128 rows of the expert runs
// on the M = 128 pair instruction (64 rows per CTA); its accumulator sits in
// TMEM as lanes 0-63 = the CTA's 64 rows for tile columns [0, Nt/2) and
// lanes 64-127 = the same rows for [Nt/2, Nt) (measured).
//
// Synchronisation (every wait bounded):
//  * both CTAs' TMA loads of a stage complete on the leader's barrier (the
//    pair form of the tensor copy signals a barrier of either CTA); only the
//    leader arms it, for the bytes of both halves;
//  * the leader's MMA commits are multicast to both CTAs' barriers
//    (stage free, up-projection operands free, accumulator ready);
//  * both CTAs' epilogues arrive on the leader's barriers (accumulator
//    drained);
//  * at exit, each CTA waits for the leader's last MMAs (which touch its
//    shared memory and TMEM); the peer then tells the leader how many copies
//    it issued, the leader balances and waits out every copy either CTA has
//    in flight (all complete on its barriers) and releases the peer, so
//    neither leaves while a copy, an MMA or an arrive can still reach it.
#pragma once

#include "gemm.cuh"

namespace moe {

// Teardown of the leader: every copy of either CTA completes on the
// leader's barriers bars[0..n) (phase q / n of barrier q % n for the q-th
// copy).  The leader armed its first `mine` phases for both halves; the
// peer issued its first `peers` halves.  Arm what only the peer issued,
// balance what the peer never issued, and wait out the last n phases
// (earlier ones completed before any later copy could be issued).
__device__ __forceinline__ void drain_pair_copies(uint64_t* bars, int n, uint32_t bytes,
                                                  int mine, int peers, uint64_t limit_ns) {
  const int hi = mine > peers ? mine : peers;
  const int lo = hi - n > 0 ? hi - n : 0;
  for (int q = lo; q < hi; ++q) {
    uint64_t* bar = &bars[q % n];
    if (q >= mine) {
      mbar_arrive_expect_tx(bar, bytes);
    } else if (q >= peers) {
      mbar_complete_tx(bar, bytes);
    }
    drain_wait(bar, static_cast<uint32_t>(q / n) & 1u, limit_ns);
  }
}

// An expert's last 256-row tile with at most 128 rows of the expert.
__device__ __forceinline__ bool pair_half_tile(const int* s_off, int e, int mt) {
  return s_off[e + 1] - (s_off[e] + mt * 256) <= 128;
}

// L2 policies of the pair kernels' operand loads: 0 = default for both,
// 1 = weights evict-last, 2 = activations evict-last.
#ifndef MOE_PAIR_HINTS
#define MOE_PAIR_HINTS 1
#endif
// Tile order of the pair kernels (see decode_tile): m-tiles fastest.
#ifndef MOE_PAIR_TILE_ORDER
#define MOE_PAIR_TILE_ORDER 1
#endif

// Epilogue stores of the pair kernels: each epilogue warp stages its 32 rows
// of an output column block (SBW bf16 columns) in a swizzled shared-memory
// box and writes it with one TMA store, through a ring of NSTG boxes per
// warp; boxes that would cross a tile's column range or hold rows of another
// expert fall back to per-thread row stores.  (The per-thread stores of 32
// different rows per instruction load the same LSU path as the pipeline's
// barrier polls.)
// MOE_PAIR_TMA_STORE: bit m set = mode m stores through the ring.  Measured
// (same-box A/B): gate_up fwd and gate_up bwd about 1% faster with it; down
// fwd no faster on the gpt-oss-20b shape and 9% slower on the Qwen3-30B-A3B
// one (K = 768: short mainloops leave the staging no slack); down bwd 2%
// slower.
#ifndef MOE_PAIR_TMA_STORE
#define MOE_PAIR_TMA_STORE 0x9
#endif
#ifndef MOE_PAIR_STORE_BOX
#define MOE_PAIR_STORE_BOX 16
#endif
#ifndef MOE_PAIR_NSTG
#define MOE_PAIR_NSTG 3
#endif
#ifndef MOE_PAIR_NSTG8
#define MOE_PAIR_NSTG8 1
#endif
// Epilogue warps of the down-backward pair kernel: 4, one per TMEM lane
// quarter, each draining all of a row's columns (measured against 8, two per
// quarter with half the columns each: 1.5% faster on the gpt-oss-20b shape,
// 2.5% on the Qwen3-30B-A3B one; loading the saved gate / up rows one
// 32-column chunk ahead of their use was 25-45% slower, with either count).
// Down-backward epilogue: the dZ1 stores of whole 32 x 32 chunks go through
// a 2 KB shared staging tile per warp, so that each store instruction
// covers 16 rows x 64 bytes instead of 32 rows x 32 bytes (measured: down
// bwd 4-5% faster on the Qwen3-30B-A3B shape, 2-3% on gpt-oss-20b; staging
// the saved gate / up loads the same way gained nothing more, and 64-column
// chunks stored as 16 rows x 128 bytes were 10% slower).
#ifndef MOE_DBWD_STAGED
#define MOE_DBWD_STAGED 1
#endif
#ifndef MOE_PAIR_DOWN_BWD_WARPS
#define MOE_PAIR_DOWN_BWD_WARPS 4
#endif

template <int MODE, int RK>
struct PairCfg {
  static constexpr bool kSwiGLU = (MODE == kGateUpFwd);
  static constexpr bool kBMN = (MODE == kDownBwd || MODE == kGateUpBwd);
  static constexpr int BM = 128, BK = 64;           // rows per CTA, K per stage
  static constexpr int BN = 256;                    // tile columns (MMA N)
  static constexpr int NH = BN / 2;                 // B columns per CTA
  static constexpr int A_BYTES = BM * BK * 2;
  static constexpr int B_BYTES = NH * BK * 2;
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr int LSPAN = RK * 2;              // bytes per K-major rank-r row
  // this CTA's up-factor block: NH rows of r (K-major, forward) or r rows of
  // NH columns as two 64-column MN-major atoms (backward; the same bytes)
  static constexpr int LB_BYTES = NH * LSPAN;
  static constexpr int LB_ATOM = RK * 128;          // backward: one 64-column atom
  static constexpr int XA_BYTES = BM * LSPAN;       // this CTA's rank-r rows
  static constexpr int UP_BYTES = LB_BYTES + XA_BYTES;
  static constexpr int MISC_BYTES = 512 + 8 * 520;  // barriers, counts, tables
  // epilogue warps: one per TMEM lane quarter (down bwd: above)
  static constexpr int EPI_WARPS = MODE == kDownBwd ? MOE_PAIR_DOWN_BWD_WARPS : 4;
  static constexpr int THREADS = 64 + 32 * EPI_WARPS;
  // epilogue store staging: per warp NSTG boxes of 32 rows x SBW columns
  static constexpr bool kRing = ((MOE_PAIR_TMA_STORE >> MODE) & 1) != 0;
  static constexpr int SBW = MOE_PAIR_STORE_BOX;
  static constexpr int SLOT_BYTES = 32 * SBW * 2;
  static constexpr int NSTG = EPI_WARPS == 8 ? MOE_PAIR_NSTG8 : MOE_PAIR_NSTG;
  // down bwd: one 32-row x 64-byte staging tile per epilogue warp
  static constexpr bool kStg = MODE == kDownBwd && MOE_DBWD_STAGED != 0;
  static constexpr int STG_TILE = 32 * 64;
  static constexpr int RING_BYTES =
      kRing ? EPI_WARPS * NSTG * SLOT_BYTES : (kStg ? EPI_WARPS * STG_TILE : 0);
  static constexpr uint32_t SLOT_SWZ_SPAN = SBW * 2;  // bytes per staged row
  static constexpr int FIXED = 2 * UP_BYTES + MISC_BYTES + RING_BYTES;
  static constexpr int NS_FIT = (kSmemOptin - 1024 - FIXED) / STAGE_BYTES;
  static constexpr int NS = NS_FIT > 8 ? 8 : NS_FIT;
  static constexpr int SMEM_BYTES = 1024 + NS * STAGE_BYTES + FIXED;
  static constexpr uint32_t LLAYOUT =
      RK == 16 ? kLayoutSW32 : (RK == 32 ? kLayoutSW64 : kLayoutSW128);
  static constexpr int TMEM_COLS = 512;
  static constexpr int ACC_STRIDE = 256;
  // rows per TMA box of the K-major weight in gate_up fwd (gate and up
  // blocks of 64; down fwd boxes hold the launch's Nt/2 rows) and of the up
  // factor (gate_up fwd: two blocks of 64; otherwise 128, of which the MMA
  // reads the first Nt/2)
  static constexpr int W_BOX_ROWS = 64;
  static constexpr int LB_BOX_ROWS = kSwiGLU ? 64 : NH;
  static constexpr int MN_BOX = 64 * BK * 2;        // one 64-column MN-major atom
  static_assert(NS >= 3, "not enough shared memory for three stages");
  static_assert(SMEM_BYTES <= kSmemOptin, "shared memory over the opt-in limit");
  static_assert(LB_BYTES % 1024 == 0 && XA_BYTES % 1024 == 0, "swizzle atoms");
  static_assert(SBW == 16 || SBW == 32, "staged box width");
  static_assert(NSTG >= 1 && SLOT_BYTES % 1024 == 0, "staging ring");
};

// One epilogue warp's ring of staged output boxes (32 rows x SBW bf16
// columns each, swizzled with the box's row span).
template <int SBW, int NSTG>
struct StoreRing {
  uint8_t* base;
  int slot;

  // Stores this thread's SBW values (its row of the box) at columns
  // [x, x + SBW) of rows [y, y + 32) of the tensor behind `tm`.  Warp-wide.
  __device__ __forceinline__ void put(const CUtensorMap* tm, const float* v, int x, int y,
                                      uint64_t pol, int lane) {
    constexpr uint32_t SPAN = SBW * 2;
    uint8_t* box = base + slot * (32 * SPAN);
    if (lane == 0) bulk_wait_group_read<NSTG - 1>();  // this slot's last store has read it
    __syncwarp();
#pragma unroll
    for (int ch = 0; ch < SBW / 8; ++ch)
      *reinterpret_cast<uint4*>(box + swz_offset(lane, ch, SPAN)) = pack8(v + 8 * ch);
    fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0) {
      tma_store_2d(tm, box, x, y, pol);
      bulk_commit_group();
    }
    slot = slot + 1 == NSTG ? 0 : slot + 1;
  }

  // Every store issued by this warp has written global memory.
  __device__ __forceinline__ void finish(int lane) {
    if (lane == 0) bulk_wait_group<0>();
    __syncwarp();
  }
};

// Writes this thread's W values v (output columns [col, col + W) of its
// row) of one output: through the staging ring in SBW-column boxes when all
// 32 rows of the warp belong to the tile's expert (rows_all) and the box
// stays inside the tile's columns [.., hi); otherwise with per-thread row
// stores.  Columns at or past nmax (the output's width) are never written;
// a box that reaches past nmax is clipped by the tensor map.
template <int W, bool kRing, int SBW, int NSTG>
__device__ __forceinline__ void pair_out_chunk(StoreRing<SBW, NSTG>& ring, const CUtensorMap* tm,
                                               __nv_bfloat16* rowp, const float* v, int col,
                                               int y0, bool rows_all, bool rvalid, int hi,
                                               int nmax, uint64_t pol, int lane) {
  const int lim = min(hi, nmax);
  if constexpr (W < SBW || !kRing) {
    if (rvalid) store_row_bf16<W>(rowp + col, v, lim - col, pol);
  } else if (rows_all) {
#pragma unroll
    for (int b = 0; b < W; b += SBW) {
      const int x = col + b;
      if (x >= lim) break;
      if (x + SBW <= hi) ring.put(tm, v + b, x, y0, pol, lane);
      else store_row_bf16<SBW>(rowp + x, v + b, lim - x, pol);
    }
  } else if (rvalid) {
    store_row_bf16<W>(rowp + col, v, lim - col, pol);
  }
}

// SwiGLU epilogue of one 64-column gate / up block of a row: gate at TMEM
// column t_gate, up at t_gate + 64; output columns col .. col + 63 of h
// (tmH), of the saved gate (tmG: Z1 columns [0, I)) and of the saved up
// (tmU: Z1 columns [I, 2I)).
template <bool kRing, int SBW, int NSTG>
__device__ __forceinline__ void epi_swiglu_seg64(const GemmArgs& args, StoreRing<SBW, NSTG>& ring,
                                                 const CUtensorMap* tmH, const CUtensorMap* tmG,
                                                 const CUtensorMap* tmU, uint32_t t_gate,
                                                 int grow, int y0, bool rows_all, bool rvalid,
                                                 int col, uint64_t pol, int lane) {
  __nv_bfloat16* hrow = args.out + static_cast<size_t>(grow) * args.ld_out;
  __nv_bfloat16* zrow = args.out2 + static_cast<size_t>(grow) * args.ld_out2;
#pragma unroll 1
  for (int c = 0; c < 64; c += 32) {
    float g[32], u[32], h[32];
    tmem_ld<32>(t_gate + c, g);
    tmem_ld<32>(t_gate + 64 + c, u);
    tmem_ld_wait();
#pragma unroll
    for (int i = 0; i < 32; ++i) h[i] = g[i] * sigmoidf_(g[i]) * u[i];
    const int cc = col + c, hi = col + 64;
    pair_out_chunk<32, kRing>(ring, tmH, hrow, h, cc, y0, rows_all, rvalid, hi, args.N, pol,
                              lane);
    pair_out_chunk<32, kRing>(ring, tmG, zrow, g, cc, y0, rows_all, rvalid, hi, args.N, pol,
                              lane);
    pair_out_chunk<32, kRing>(ring, tmU, zrow + args.I, u, cc, y0, rows_all, rvalid, hi,
                              args.N, pol, lane);
  }
}

// The saved gate and up values of W columns [col, col + W) of one row of
// Z1 (gate at grow_p[col], up at grow_p[I + col]); zeros past nmax and for a
// row outside the expert.  32-byte loads where the addresses allow.
template <int W>
struct SavedGU {
  uint4 g[W / 8], u[W / 8];
};

template <int W>
__device__ __forceinline__ void load_saved_gu(SavedGU<W>& sv, const __nv_bfloat16* grow_p, int I,
                                              int col0, int nmax, bool rvalid) {
  const bool a32 = ((reinterpret_cast<uintptr_t>(grow_p + col0) |
                     reinterpret_cast<uintptr_t>(grow_p + I + col0)) & 31u) == 0;
#pragma unroll
  for (int q = 0; q < W / 8; q += 2) {
    const int col = col0 + 8 * q;
    sv.g[q] = sv.u[q] = make_uint4(0, 0, 0, 0);
    if (q + 1 < W / 8) sv.g[q + 1] = sv.u[q + 1] = make_uint4(0, 0, 0, 0);
    if (!rvalid) continue;
    if (q + 1 < W / 8 && a32 && col + 16 <= nmax) {
      ld_global_nc_v8(grow_p + col, sv.g[q], sv.g[q + 1]);
      ld_global_nc_v8(grow_p + I + col, sv.u[q], sv.u[q + 1]);
    } else {
      if (col < nmax) {
        sv.g[q] = *reinterpret_cast<const uint4*>(grow_p + col);
        sv.u[q] = *reinterpret_cast<const uint4*>(grow_p + I + col);
      }
      if (q + 1 < W / 8 && col + 8 < nmax) {
        sv.g[q + 1] = *reinterpret_cast<const uint4*>(grow_p + col + 8);
        sv.u[q + 1] = *reinterpret_cast<const uint4*>(grow_p + I + col + 8);
      }
    }
  }
}

// Byte offset of 16-byte unit u (columns 8u .. 8u + 7) of row r in a
// 32-row x 64-byte staging tile; the unit index is XORed with bits 1-2 of
// the row, so that a warp's 16-byte accesses, one row per lane or two lanes
// per row, fall in distinct banks within each 8-lane phase.
__device__ __forceinline__ uint32_t stg_off(int r, int u) {
  return static_cast<uint32_t>(r * 64 + ((u ^ ((r >> 1) & 3)) << 4));
}

// Stores 32 bf16 columns [col, col + 32) of the warp's 32 rows y0 .. y0 + 31
// (this thread's row, v, rounded as the per-row stores round it) through the
// warp's staging tile: lane l then writes 32 bytes (half l % 2) of rows l / 2
// and l / 2 + 16, so that each store instruction covers 16 rows x 64 bytes
// instead of 32 rows x 32 bytes.  All 32 rows and columns must be in range
// and every row piece 32-byte aligned.  Warp-wide.
template <class Args>
__device__ __forceinline__ void store_rows_staged32(const Args& args, uint8_t* stg, const float* v,
                                                    int y0, size_t col, uint64_t pol, int lane) {
  __syncwarp();  // the tile's previous reads are done
#pragma unroll
  for (int q = 0; q < 4; ++q) *reinterpret_cast<uint4*>(stg + stg_off(lane, q)) = pack8(v + 8 * q);
  __syncwarp();
  const int rr = lane >> 1, hh = lane & 1;
  const uint4 a0 = *reinterpret_cast<const uint4*>(stg + stg_off(rr, 2 * hh));
  const uint4 a1 = *reinterpret_cast<const uint4*>(stg + stg_off(rr, 2 * hh + 1));
  const uint4 b0 = *reinterpret_cast<const uint4*>(stg + stg_off(rr + 16, 2 * hh));
  const uint4 b1 = *reinterpret_cast<const uint4*>(stg + stg_off(rr + 16, 2 * hh + 1));
  const size_t ra = static_cast<size_t>(y0 + rr);
  st_global_v8_hint(args.out + ra * args.ld_out + col + 16 * hh, a0, a1, pol);
  st_global_v8_hint(args.out + (ra + 16) * args.ld_out + col + 16 * hh, b0, b1, pol);
}

// Epilogue of the other modes for NC accumulator columns (this warp's share
// of them with kSplit): tile column j of the drained range sits at TMEM
// column t_acc + j and is output column col0 + j; nothing at or past hi
// (the end of the tile's columns) or args.N is written.  Plain store (down
// fwd: Z2, gate_up bwd: dXp, through tmO) or SwiGLU backward (down bwd:
// reads the saved gate / up, writes dZ1 = [dg | du] through tmO / tmU).
template <int MODE, int NC, bool kSplit, bool kRing, bool C_STG, int SBW, int NSTG>
__device__ __forceinline__ void epi_pair_drain(const GemmArgs& args, StoreRing<SBW, NSTG>& ring,
                                               uint8_t* stg, const CUtensorMap* tmO,
                                               const CUtensorMap* tmU, uint32_t t_acc, int grow,
                                               int y0, bool rows_all, bool rvalid, int ehalf,
                                               int col0, int hi, uint64_t pol, int lane) {
  const int nmax = min(args.N, hi);
  __nv_bfloat16* orow = args.out + static_cast<size_t>(grow) * args.ld_out;
  if constexpr (MODE == kDownBwd) {
    const __nv_bfloat16* grow_p = args.aux + static_cast<size_t>(grow) * args.ld_aux;
    // staged stores need 32-byte aligned row pieces of dZ1
    bool stg_ok = false;
    if constexpr (C_STG) {
      const __nv_bfloat16* o0 = args.out + static_cast<size_t>(y0) * args.ld_out + col0;
      stg_ok = (reinterpret_cast<uintptr_t>(o0) & 31u) == 0 && ((args.ld_out | args.I) & 15) == 0;
    }
    for_my_chunks<NC, kSplit>(ehalf, [&](int c, auto w) {
      constexpr int W = decltype(w)::value;
      const int col = col0 + c;
      SavedGU<W> sv;  // loads first (in flight during the TMEM read)
      load_saved_gu<W>(sv, grow_p, args.I, col, nmax, rvalid);
      float dh[W];
      tmem_ld<W>(t_acc + c, dh);
      tmem_ld_wait();
      float dg[W], du[W];
#pragma unroll
      for (int q = 0; q < W / 8; ++q) {
        const uint32_t ga[4] = {sv.g[q].x, sv.g[q].y, sv.g[q].z, sv.g[q].w};
        const uint32_t ua[4] = {sv.u[q].x, sv.u[q].y, sv.u[q].z, sv.u[q].w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
#pragma unroll
          for (int h2 = 0; h2 < 2; ++h2) {
            const float gg = h2 ? bf16_hi(ga[i]) : bf16_lo(ga[i]);
            const float uu = h2 ? bf16_hi(ua[i]) : bf16_lo(ua[i]);
            const int j = 8 * q + 2 * i + h2;
            const float sg = sigmoidf_(gg);
            dg[j] = dh[j] * uu * sg * (1.f + gg * (1.f - sg));
            du[j] = dh[j] * gg * sg;
          }
        }
      }
      if constexpr (C_STG && W == 32) {
        // a whole chunk of the warp's 32 rows, all inside the expert
        if (rows_all && col + 32 <= nmax && stg_ok) {
          store_rows_staged32(args, stg, dg, y0, col, pol, lane);
          store_rows_staged32(args, stg, du, y0, static_cast<size_t>(col) + args.I, pol, lane);
          return;
        }
      }
      pair_out_chunk<W, kRing>(ring, tmO, orow, dg, col, y0, rows_all, rvalid, hi, args.N, pol,
                               lane);
      pair_out_chunk<W, kRing>(ring, tmU, orow + args.I, du, col, y0, rows_all, rvalid, hi,
                               args.N, pol, lane);
    });
  } else {
    for_my_chunks<NC, kSplit>(ehalf, [&](int c, auto w) {
      constexpr int W = decltype(w)::value;
      float v[W];
      tmem_ld<W>(t_acc + c, v);
      tmem_ld_wait();
      pair_out_chunk<W, kRing>(ring, tmO, orow, v, col0 + c, y0, rows_all, rvalid, hi, args.N,
                               pol, lane);
    });
  }
}

// Operand maps: tmA = A [R, K] (128-row boxes); tmW = the weight (K-major
// [E * b_rows, K] in boxes of W_BOX_ROWS rows (gate_up fwd) or Nt/2 rows
// (down fwd), or MN-major [E * b_rows, N] in 64 x 64 atoms); tmXA = the rank-r product [R, r] (128-row boxes);
// tmLB = the up factor: forward B [E * lb_rows, r] (LB_BOX_ROWS-row boxes);
// backward A read in place as [E * r, N] (64-column x r-row boxes: the MMA's
// B operand MN-major, so the factor needs no transposed copy).
template <int MODE, int RK>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(PairCfg<MODE, RK>::THREADS, 1)
    grouped_lora_gemm_pair_kernel(const __grid_constant__ CUtensorMap tmA,
                                  const __grid_constant__ CUtensorMap tmW,
                                  const __grid_constant__ CUtensorMap tmXA,
                                  const __grid_constant__ CUtensorMap tmLB,
                                  const __grid_constant__ CUtensorMap tmO,
                                  const __grid_constant__ CUtensorMap tmO2,
                                  const __grid_constant__ CUtensorMap tmO3,
                                  const GemmArgs args) {
  using C = PairCfg<MODE, RK>;
  constexpr bool kSwiGLU = C::kSwiGLU;
  constexpr bool kBMN = C::kBMN;
  constexpr int BN = C::BN;

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t* sStage = smem;
  uint8_t* sRing = sStage + C::NS * C::STAGE_BYTES;  // epilogue store staging
  uint8_t* sLB = sRing + C::RING_BYTES;
  uint8_t* sXA = sLB + 2 * C::LB_BYTES;
  uint64_t* full = reinterpret_cast<uint64_t*>(sXA + 2 * C::XA_BYTES);
  uint64_t* empty = full + C::NS;
  uint64_t* lb_full = empty + C::NS;
  uint64_t* lb_empty = lb_full + 2;
  uint64_t* acc_full = lb_empty + 2;
  uint64_t* acc_empty = acc_full + 2;
  uint64_t* final_bar = acc_empty + 2;
  uint64_t* peer_done = final_bar + 1;       // leader: the peer is done
  uint64_t* drained = peer_done + 1;         // peer: its copies have landed
  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(drained + 1);
  volatile int* s_abort = reinterpret_cast<volatile int*>(s_tmem + 1);
  // copies issued by this CTA's producer: [0] stages, [1] up-operand sets;
  // [2], [3]: the same counts of the peer (written into the leader)
  int* s_issued = reinterpret_cast<int*>(s_tmem + 4);
  int* s_off = s_issued + 4;
  int* s_mstart = s_off + 520;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const bool leader = (rank == 0);
  const int E = args.E;
  const uint64_t wait_ns = args.wait_ns;
  const int pair = blockIdx.x >> 1, npairs = gridDim.x >> 1;

  if (threadIdx.x == 0) {
    for (int i = 0; i < C::NS; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&lb_full[i], 1);
      mbar_init(&lb_empty[i], 1);
      mbar_init(&acc_full[i], 1);
      mbar_init(&acc_empty[i], 2 * C::EPI_WARPS);
    }
    mbar_init(final_bar, 1);
    mbar_init(peer_done, 1);
    mbar_init(drained, 1);
    for (int i = 0; i < 4; ++i) s_issued[i] = 0;
    *s_abort = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tmA);
    prefetch_tmap(&tmW);
    prefetch_tmap(&tmXA);
    prefetch_tmap(&tmLB);
  }
  if (warp == 2 && lane == 0) {
    prefetch_tmap(&tmO);
    prefetch_tmap(&tmO2);
    prefetch_tmap(&tmO3);
  }
  if (warp == 1) {
    tmem_alloc_pair(s_tmem, C::TMEM_COLS);
    tmem_relinquish_pair();
  }
  // everything above touches only shared memory, TMEM and the kernel's
  // parameters; the preceding kernel's outputs are read from here on
  griddep_sync();
  if (warp == 2) build_tile_table(args.offsets, E, args.R, s_off, s_mstart, lane, 8);
  tc_fence_before();
  cluster_sync_all();  // both CTAs' barriers initialised, TMEM allocated
  tc_fence_after();

  const uint32_t tmem_base = *s_tmem;
  const int total_tiles = s_mstart[E] * args.n_tiles;
  const int k_iters = (args.K + C::BK - 1) / C::BK;
  // tile width (MMA N) and this CTA's share of it
  const int Nt = kSwiGLU ? BN : args.tile_n;
  const int NHt = Nt >> 1;
  // bytes of one CTA's half of a stage (down fwd: Nt/2 weight rows)
  const uint32_t stage_bytes = (kSwiGLU || kBMN)
                                   ? static_cast<uint32_t>(C::STAGE_BYTES)
                                   : static_cast<uint32_t>(C::A_BYTES + NHt * C::BK * 2);
  // cluster addresses of the leader's copies of the barriers
  auto lead = [&](const void* p) { return mapa_shared(smem_u32(p), 0); };

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      int n_st = 0, n_lb = 0;
      bool ok = true;
      int local = 0;
      // L2 residency: activations (A, reused by the tile's n-tiles) and
      // weights (reused by the expert's m-tiles), see MOE_PAIR_HINTS
#if MOE_PAIR_HINTS == 1
      const uint64_t pol_a = policy_evict_normal(), pol_w = policy_evict_last();
#elif MOE_PAIR_HINTS == 2
      const uint64_t pol_a = policy_evict_last(), pol_w = policy_evict_normal();
#else
      const uint64_t pol_a = policy_evict_normal(), pol_w = policy_evict_normal();
#endif
      for (int tile = pair; tile < total_tiles && ok; tile += npairs, ++local) {
        int e, mt, nt;
        decode_tile<MOE_PAIR_TILE_ORDER>(tile, args.n_tiles, s_mstart, E, e, mt, nt);
        const int rows_per_cta = pair_half_tile(s_off, e, mt) ? C::BM / 2 : C::BM;
        const int row0 = s_off[e] + mt * 2 * C::BM + static_cast<int>(rank) * rows_per_cta;
        // first weight / up-factor row of this CTA's tile columns
        const int n0 = kSwiGLU ? nt * (BN / 2) + static_cast<int>(rank) * 64
                               : nt * Nt + static_cast<int>(rank) * NHt;
        const int b = local & 1;
        const uint32_t use = (local >> 1) & 1;
        if (!mbar_wait(&lb_empty[b], use ^ 1, s_abort, wait_ns)) { ok = false; break; }
        if (leader) mbar_arrive_expect_tx(&lb_full[b], 2 * C::UP_BYTES);
        {
          // up-projection operands: this CTA's rows of the rank-r product and
          // the up factor rows of its tile columns
          const uint32_t lbb = lead(&lb_full[b]);
          uint8_t* lb = sLB + b * C::LB_BYTES;
          if constexpr (kBMN) {
            // A[e] rows 0..r-1, this CTA's tile columns, as two atoms
            tma_load_2d_pair(lb, &tmLB, lbb, n0, e * RK);
            tma_load_2d_pair(lb + C::LB_ATOM, &tmLB, lbb, n0 + 64, e * RK);
          } else {
            const int lrow = e * args.lb_rows + n0;
            tma_load_2d_pair(lb, &tmLB, lbb, 0, lrow);
            if constexpr (kSwiGLU)
              tma_load_2d_pair(lb + 64 * C::LSPAN, &tmLB, lbb, 0, lrow + args.I);
          }
          tma_load_2d_pair(sXA + b * C::XA_BYTES, &tmXA, lbb, 0, row0);
        }
        ++n_lb;
        for (int kt = 0; kt < k_iters; ++kt) {
          if (!mbar_wait(&empty[stage], phase ^ 1, s_abort, wait_ns)) { ok = false; break; }
          uint8_t* st = sStage + stage * C::STAGE_BYTES;
          uint8_t* sb = st + C::A_BYTES;
          const int kx = kt * C::BK;
          const uint32_t fb = lead(&full[stage]);
          if (leader) mbar_arrive_expect_tx(&full[stage], 2 * stage_bytes);
          tma_load_2d_pair_hint(st, &tmA, fb, kx, row0, pol_a);
          if constexpr (kBMN) {
            // W [K, N] in place: this CTA's Nt/2 tile columns, loaded as two
            // 64-column atoms
            const int krow = e * args.b_rows + kx;
            tma_load_2d_pair_hint(sb, &tmW, fb, n0, krow, pol_w);
            tma_load_2d_pair_hint(sb + C::MN_BOX, &tmW, fb, n0 + 64, krow, pol_w);
          } else if constexpr (kSwiGLU) {
            const int wrow = e * args.b_rows + n0;
            tma_load_2d_pair_hint(sb, &tmW, fb, kx, wrow, pol_w);                 // gate
            tma_load_2d_pair_hint(sb + 64 * 128, &tmW, fb, kx, wrow + args.I, pol_w);  // up
          } else {
            tma_load_2d_pair_hint(sb, &tmW, fb, kx, e * args.b_rows + n0, pol_w);
          }
          ++n_st;
          if (++stage == C::NS) {
            stage = 0;
            phase ^= 1;
          }
        }
      }
      // every copy lands on the leader's barriers; the teardown waits them out
      s_issued[0] = n_st;
      s_issued[1] = n_lb;
    }
  } else if (warp == 1) {
    if (leader) {
      // ---------------------------------------------------------- MMA (leader)
      // The whole warp runs the loop (its state stays warp-uniform); one
      // elected lane issues the tensor-core instructions.
      const uint32_t kIdesc = idesc_bf16_f32(256, Nt, false, kBMN);
      const uint32_t kIdescH = idesc_bf16_f32(128, Nt, false, kBMN);
      const uint32_t kIdescUp = idesc_bf16_f32(256, Nt, false, kBMN);
      const uint32_t kIdescUpH = idesc_bf16_f32(128, Nt, false, kBMN);
      constexpr uint16_t kBoth = 0x3;
      const uint64_t a_desc0 = smem_desc(smem_u32(sStage), 16, 1024, kLayoutSW128);
      // MN-major: LBO = next 64-column atom, SBO = next 8 K-rows (8 x 128 B)
      const uint64_t b_desc0 =
          kBMN ? smem_desc(smem_u32(sStage) + C::A_BYTES, C::MN_BOX, 1024, kLayoutSW128)
               : smem_desc(smem_u32(sStage) + C::A_BYTES, 16, 1024, kLayoutSW128);
      constexpr uint64_t kStageInc = C::STAGE_BYTES >> 4;
      constexpr uint64_t kBStep = kBMN ? (2048 >> 4) : (32 >> 4);  // 16 K
      int stage = 0;
      uint64_t soff = 0;
      uint32_t phase = 0;
      int local = 0;
      bool ok = true;
      if (args.stall_test) ok = warp_wait(final_bar, 0, s_abort, wait_ns);
#ifdef MOE_GEMM_TRACE
      const long long t_role = clock64();
#endif
      for (int tile = pair; ok && tile < total_tiles; tile += npairs, ++local) {
        const int b = local & 1;
        const uint32_t use = (local >> 1) & 1;
        const uint32_t t_acc = tmem_base + b * C::ACC_STRIDE;
        int e, mt, nt;
        decode_tile<MOE_PAIR_TILE_ORDER>(tile, args.n_tiles, s_mstart, E, e, mt, nt);
        const bool half = pair_half_tile(s_off, e, mt);
        const uint32_t idesc = half ? kIdescH : kIdesc;
        const uint32_t idesc_up = half ? kIdescUpH : kIdescUp;
        if (!MOE_TIMED(MODE, 14, warp_wait_cluster(&acc_empty[b], use ^ 1, s_abort, wait_ns))) { ok = false; break; }
        tc_fence_after();
        for (int kt = 0; kt < k_iters; ++kt) {
          if (!MOE_TIMED(MODE, 11, warp_wait(&full[stage], phase, s_abort, wait_ns))) { ok = false; break; }
          const uint64_t da = a_desc0 + soff, db = b_desc0 + soff;
          if (elect_one()) {
            umma_bf16_pair(t_acc, da, db, idesc, kt > 0 ? 1u : 0u);
#pragma unroll
            for (int kk = 1; kk < C::BK / 16; ++kk)
              umma_bf16_pair(t_acc, da + 2 * kk, db + kk * kBStep, idesc, 1u);
            umma_commit_pair_mc(&empty[stage], kBoth);
          }
          __syncwarp();
          soff += kStageInc;
          if (++stage == C::NS) {
            stage = 0;
            soff = 0;
            phase ^= 1;
          }
        }
        if (!ok) break;
        // up-projection (K = r) into the same accumulator
        if (!warp_wait(&lb_full[b], use, s_abort, wait_ns)) { ok = false; break; }
        tc_fence_after();
        if (elect_one()) {
          const uint32_t xa0 = smem_u32(sXA + b * C::XA_BYTES);
          const uint32_t lb0 = smem_u32(sLB + b * C::LB_BYTES);
#pragma unroll
          for (int kk = 0; kk < RK / 16; ++kk)
            umma_bf16_pair(t_acc, smem_desc(xa0 + kk * 32, 16, 8 * C::LSPAN, C::LLAYOUT),
                           kBMN ? smem_desc(lb0 + kk * 2048, C::LB_ATOM, 1024, kLayoutSW128)
                                : smem_desc(lb0 + kk * 32, 16, 8 * C::LSPAN, C::LLAYOUT),
                           idesc_up,
                           1u);
          umma_commit_pair_mc(&lb_empty[b], kBoth);
          umma_commit_pair_mc(&acc_full[b], kBoth);
        }
        __syncwarp();
      }
#ifdef MOE_GEMM_TRACE
      if (lane == 0)
        atomicAdd(&g_gemm_trace[MODE][blockIdx.x % 160][13],
                  static_cast<unsigned long long>(clock64() - t_role));
#endif
      // all of the leader's MMAs complete -> both CTAs' final_bar
      if (elect_one()) umma_commit_pair_mc(final_bar, kBoth);
      __syncwarp();
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int ew = warp & 3;              // TMEM lane quarter
    constexpr bool kSplit = C::EPI_WARPS == 8;
    const int ehalf = (warp - 2) >> 2;    // which share of the columns
    const uint32_t lane_base = static_cast<uint32_t>(ew * 32) << 16;
    const uint64_t pol = policy_evict_first();  // outputs stream out of L2
    StoreRing<C::SBW, C::NSTG> ring{sRing + (warp - 2) * C::NSTG * C::SLOT_BYTES, 0};
    uint8_t* stg = sRing + (warp - 2) * C::STG_TILE;  // down bwd staging (kStg)
    int local = 0;
    for (int tile = pair; tile < total_tiles; tile += npairs, ++local) {
      int e, mt, nt;
      decode_tile<MOE_PAIR_TILE_ORDER>(tile, args.n_tiles, s_mstart, E, e, mt, nt);
      const int b = local & 1;
      const uint32_t use = (local >> 1) & 1;
      const bool half = pair_half_tile(s_off, e, mt);
      // half tile: lane quarters 0-1 hold rows 0-63 for tile columns
      // [0, 128), quarters 2-3 the same rows for [128, 256)
      const int wrow0 = half ? (ew & 1) * 32 : ew * 32;   // the warp's first row
      const int y0 = s_off[e] + mt * 2 * C::BM +
                     static_cast<int>(rank) * (half ? C::BM / 2 : C::BM) + wrow0;
      const int grow = y0 + lane;
      const bool rvalid = grow < s_off[e + 1];
      const bool rows_all = y0 + 32 <= s_off[e + 1];  // the warp's 32 rows are the expert's
      const uint32_t t_acc = tmem_base + lane_base + b * C::ACC_STRIDE;
      const int col0 = nt * Nt;             // first output column of the tile
      // (no L2 prefetch of the saved gate / up rows here: measured 1.5%
      // slower in this kernel)
      if (!warp_wait(&acc_full[b], use, s_abort, wait_ns)) break;
      tc_fence_after();
      if constexpr (kSwiGLU) {
        // 128-column blocks [gate 64 | up 64] of output columns
        // 128 nt + 64 q .. +63, q = the block
        const int oc0 = nt * (BN / 2);
        if (half) {
          epi_swiglu_seg64<C::kRing>(args, ring, &tmO, &tmO2, &tmO3, t_acc, grow, y0, rows_all, rvalid,
                           oc0 + (ew >> 1) * 64, pol, lane);
        } else {
          epi_swiglu_seg64<C::kRing>(args, ring, &tmO, &tmO2, &tmO3, t_acc, grow, y0, rows_all, rvalid,
                           oc0, pol, lane);
          epi_swiglu_seg64<C::kRing>(args, ring, &tmO, &tmO2, &tmO3, t_acc + 128, grow, y0, rows_all,
                           rvalid, oc0 + 64, pol, lane);
        }
      } else {
        // tile columns [0, Nt) = output columns col0 + c; TMEM columns past
        // Nt (or past N) hold nothing of this tile and are not stored
        if (half) {
          const int q = ew >> 1;
          epi_pair_drain<MODE, BN / 2, kSplit, C::kRing, C::kStg>(
              args, ring, stg, &tmO, &tmO3, t_acc, grow, y0, rows_all, rvalid, ehalf,
              col0 + q * NHt, col0 + (q + 1) * NHt, pol, lane);
        } else {
          epi_pair_drain<MODE, BN, kSplit, C::kRing, C::kStg>(args, ring, stg, &tmO, &tmO3, t_acc,
                                                            grow, y0, rows_all, rvalid, ehalf,
                                                            col0, col0 + Nt, pol, lane);
        }
      }
      tc_fence_before();
      __syncwarp();
      // the accumulator's TMEM reads have completed (tcgen05.wait::ld); the
      // release needs no ordering of the output stores
      if (lane == 0) MOE_ACC_RELEASE(lead(&acc_empty[b]));
    }
    if constexpr (C::kRing) ring.finish(lane);  // every staged store has left shared memory
  }

  // ---------------------------------------------------------------- teardown
  tc_fence_before();
  __syncthreads();
  if (threadIdx.x == 0) {
    // the leader's MMAs read this CTA's shared memory and write its TMEM
    drain_wait(final_bar, 0, wait_ns);
    if (!leader) {
      // publish this CTA's copy counts; the release orders them before the
      // arrive, after which nothing else arrives from this CTA
      st_shared_cluster_s32(lead(&s_issued[2]), s_issued[0]);
      st_shared_cluster_s32(lead(&s_issued[3]), s_issued[1]);
      mbar_arrive_cluster(lead(peer_done));
      drain_wait(drained, 0, wait_ns);        // the leader saw every copy land
    } else {
      drain_wait_cluster(peer_done, 0, wait_ns);
      drain_pair_copies(full, C::NS, stage_bytes, s_issued[0], s_issued[2], wait_ns);
      drain_pair_copies(lb_full, 2, C::UP_BYTES, s_issued[1], s_issued[3], wait_ns);
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
