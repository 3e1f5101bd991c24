// a3 / a4 / a7 / a8: persistent grouped GEMM over ragged experts on the
// 5th-generation tensor cores, with the split-LoRA product fused in.
//
// Per output tile (128 rows of one expert x BN columns), with the TMEM
// accumulator D = [acc (BN columns) | lora (r columns)]:
//   mainloop : D += A_k * [B_k ; LA_k]^T   one MMA of N = BN + r per K-slice:
//              the rank-r down-projection factor LA rides in the B operand,
//              so A is read from shared memory once for both products;
//   handoff  : xa = bf16(s * lora)          TMEM -> registers -> shared memory
//   up       : acc += xa * LB^T             the rank-r up-projection, a second
//              accumulate (K = r) into the same TMEM tile, issued while the
//              next tile's mainloop is already running;
//   epilogue : mode-specific (SwiGLU, plain store, SwiGLU backward).
// This is the "split LoRA" order of the Unsloth page "Fine-tune MoE LLMs 12x
// faster with Unsloth" (section "Faster LoRA MoE training"): x W^T +
// s (x A^T) B^T, so W + s B A is never formed.
//
// Roles: warp 0 = TMA producer, warp 1 = MMA issuer (and TMEM owner), then
// 4 or 8 epilogue warps: TMEM lane quarter = warp % 4; with 8, the two warps
// of a quarter split the tile's columns.  TMEM holds
// two accumulators of 256 columns, so the epilogue of one tile overlaps the
// mainloop of the next.  Tiles are enumerated on the device from
// expert_offsets (no host synchronisation): m-tiles of all experts in expert
// order, n fastest.
#pragma once

#include "ptx.cuh"

namespace moe {

enum GemmMode : int {
  kGateUpFwd = 0,  // Z1 = Xp W1^T + s (Xp A1^T) B1^T -> SwiGLU -> h (+ Z1, XA1)
  kDownFwd = 1,    // Z2 = h W2^T + s (h A2^T) B2^T (+ hA2)
  kDownBwd = 2,    // dh = dZ2 W2 + s (dZ2 B2) A2 -> SwiGLU backward -> dZ1
  kGateUpBwd = 3,  // dXp = dZ1 W1 + s (dZ1 B1) A1
};

struct GemmArgs {
  const int32_t* offsets;  // [E+1] expert row offsets (device)
  int E, R, K;
  int N;                   // output columns (I for gate_up fwd / down bwd)
  int n_tiles;             // tiles along N
  int tile_n;              // CTA-pair kernels: columns per tile (MMA N)
  int I;                   // gate/up split
  int b_rows;              // rows per expert in B's 2-D view
  int lb_rows;             // rows per expert in LB's 2-D view
  float s;
  __nv_bfloat16* out;
  int ld_out;
  __nv_bfloat16* out2;     // saved Z1 (gate_up fwd)
  int ld_out2;
  const __nv_bfloat16* aux;  // saved Z1 (down bwd)
  int ld_aux;
  __nv_bfloat16* lora_t;   // [r, ld_lora] s-scaled rank-r product, transposed
  int ld_lora;
  uint64_t wait_ns;
  int stall_test;          // testing: make the MMA warp's first wait run out
};

constexpr int kSmemOptin = 232448;  // max dynamic shared memory per block

// K-slice of one pipeline stage of the single-CTA kernel: 64 bf16 = 128-byte
// rows, 128-byte swizzle for the K-major operands.  (Measured: halving it to
// 32 doubles the TMA requests per FLOP and slows the mainloop.)
constexpr int kGemmBK = 64;
constexpr uint32_t kKmajLayout = kGemmBK == 64 ? kLayoutSW128 : kLayoutSW64;
constexpr int kKmajSBO = 8 * kGemmBK * 2;        // 8 rows of 64 bytes
constexpr int kMnAtomBytes = kGemmBK * 128;      // 64 columns x BK rows (MN-major)
// Epilogue warps per mode: the SwiGLU-backward epilogue (loads of the saved
// gate / up and two stores per element) gets two warps per TMEM lane quarter.
__host__ __device__ constexpr int gemm_epi_warps(int mode) {
  return mode == 2 ? 8 : 4;
}
__host__ __device__ constexpr int gemm_threads(int mode) {
  return 64 + 32 * gemm_epi_warps(mode);
}

// Split of a tile's NC epilogue columns between the two warps of a TMEM lane
// quarter, in multiples of 8 columns.
template <int NC>
struct ColSplit {
  static constexpr int C0 = ((NC / 8 + 1) / 2) * 8;
  static constexpr int C1 = NC - C0;
  static_assert(C1 > 0 && C1 % 8 == 0, "column split");
};

// for_chunks over this warp's share [0, C0) or [C0, NC) of the columns
// (all of them when the quarter has a single warp).
template <int NC, bool SPLIT, typename F>
__device__ __forceinline__ void for_my_chunks(int half, F&& f) {
  using S = ColSplit<NC>;
  if constexpr (!SPLIT) {
    for_chunks<NC>(f);
  } else if (half == 0) {
    for_chunks<S::C0>(f);
  } else {
    for_chunks<S::C1>([&](int c, auto w) { f(S::C0 + c, w); });
  }
}

template <int MODE, int BN, int RK>
struct GemmCfg {
  static constexpr bool kBMN = (MODE == kDownBwd || MODE == kGateUpBwd);
  static constexpr int BM = 128, BK = kGemmBK;
  static constexpr int NMMA = BN + RK;  // N of the fused mainloop MMA
  static constexpr int A_BYTES = BM * BK * 2;
  // K-major: BN weight rows then r factor rows, BK*2 bytes each.  MN-major:
  // BN/64 weight atoms then one 64-column atom holding the (zero-padded)
  // factor.
  static constexpr int B_BYTES = kBMN ? (BN / 64 + 1) * kMnAtomBytes : NMMA * BK * 2;
  // stages start on 1024-byte boundaries (the widest swizzle period)
  static constexpr int STAGE_BYTES = (A_BYTES + B_BYTES + 1023) / 1024 * 1024;
  static constexpr int LB_BYTES = BN * RK * 2;
  static constexpr int XA_BYTES = BM * RK * 2;
  static constexpr int MISC_BYTES = 256 + 8 * 520;  // barriers, flags, tables
  static constexpr int FIXED = 2 * LB_BYTES + 2 * XA_BYTES + MISC_BYTES;
  static constexpr int NS_FIT = (kSmemOptin - 1024 - FIXED) / STAGE_BYTES;
  static constexpr int NS = NS_FIT > 8 ? 8 : NS_FIT;
  static constexpr int SMEM_BYTES = 1024 + NS * STAGE_BYTES + FIXED;
  static constexpr int LSPAN = RK * 2;  // bytes of one LoRA row = swizzle span
  static constexpr uint32_t LLAYOUT =
      RK == 16 ? kLayoutSW32 : (RK == 32 ? kLayoutSW64 : kLayoutSW128);
  static constexpr int TMEM_COLS = 512;
  static constexpr int ACC_STRIDE = 256;
  static_assert(NS >= 2, "not enough shared memory for two stages");
  static_assert(SMEM_BYTES <= kSmemOptin, "shared memory over the opt-in limit");
  static_assert(NMMA <= ACC_STRIDE && NMMA % 16 == 0, "MMA N = BN + r");
  static_assert(BN % 16 == 0, "BN must be a multiple of 16");
  static_assert(!kBMN || BN % 64 == 0, "MN-major B needs 64-column atoms");
  static_assert(RK == 16 || RK == 32 || RK == 64, "rank must be 16, 32 or 64");
};

// Tile order (build-time choice, MOE_TILE_ORDER): tiles are grouped by
// expert (expert e owns tiles [n_tiles * s_mstart[e], n_tiles *
// s_mstart[e + 1])); inside an expert either the n-tile index runs fastest
// (0, default: CTAs that run together share one activation tile and the
// expert's weight panels are reused from L2 by its later m-tiles) or the
// m-tile index does (1: the CTA-pair kernels' order, MOE_PAIR_TILE_ORDER;
// measured -1% per step against 0 on the gpt-oss-20b-shaped layer).
#ifndef MOE_TILE_ORDER
#define MOE_TILE_ORDER 0
#endif
// L2 residency hints for the mainloop loads (MOE_L2_HINTS): 0 none, 1 keep
// weights / stream activations (default), 2 keep activations / stream
// weights.  Measured with the single-CTA kernels on the gpt-oss-20b-shaped
// layer: order 0 with hints 1 is fastest; without hints the step is 5-10%
// slower.
#ifndef MOE_L2_HINTS
#define MOE_L2_HINTS 1
#endif

template <int ORDER = MOE_TILE_ORDER>
__device__ __forceinline__ void decode_tile(int tile, int n_tiles,
                                            const int* s_mstart, int E, int& e,
                                            int& mt, int& nt) {
  const int gm = tile / n_tiles;  // expert boundaries are multiples of n_tiles
  int lo = 0, hi = E;             // s_mstart[lo] <= gm < s_mstart[hi]
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (s_mstart[mid] <= gm) lo = mid; else hi = mid;
  }
  e = lo;
  if constexpr (ORDER == 1) {
    const int me = s_mstart[lo + 1] - s_mstart[lo];  // m-tiles of this expert
    const int local = tile - n_tiles * s_mstart[lo];
    nt = local / me;
    mt = local - nt * me;
  } else {
    nt = tile - gm * n_tiles;
    mt = gm - s_mstart[lo];
  }
}

// warp_wait for a barrier that other CTAs of the cluster arrive on.
__device__ __forceinline__ bool warp_wait_cluster(uint64_t* bar, uint32_t parity,
                                                  volatile int* abort_flag,
                                                  uint64_t limit_ns) {
  const bool ok = mbar_wait_cluster(bar, parity, abort_flag, limit_ns);
  return __all_sync(0xffffffffu, ok);
}

// Lane 0's view of a non-blocking barrier test, for the whole warp.
__device__ __forceinline__ bool warp_uniform(bool v) {
  return __shfl_sync(0xffffffffu, v ? 1 : 0, 0) != 0;
}

// drain_wait for a barrier that other CTAs of the cluster arrive on with
// release semantics (acquire at cluster scope).
__device__ __forceinline__ void drain_wait_cluster(uint64_t* bar, uint32_t parity,
                                                   uint64_t limit_ns) {
  const uint64_t limit = limit_ns > 1000000000ull ? limit_ns : 1000000000ull;
  const uint64_t t0 = globaltimer_ns();
  while (!mbar_try_wait_cluster(bar, parity)) {
    if (globaltimer_ns() - t0 > limit) {
      set_status(4);
      return;
    }
  }
}

// Builds the m-tile table in shared memory (one warp): s_off = offsets,
// s_mstart[e] = first global m-tile (of 2^bm_shift rows) of expert e,
// s_mstart[E] = total.
// Offsets that are not a valid partition of [0, R) give zero tiles.
__device__ __forceinline__ void build_tile_table(const int32_t* offsets, int E,
                                                 int R, int* s_off,
                                                 int* s_mstart, int lane,
                                                 int bm_shift = 7) {
  const int bm_round = (1 << bm_shift) - 1;
  const int per = (E + 31) / 32;
  const int lo = min(E, lane * per), hi = min(E, lo + per);
  bool bad = false;
  int local = 0;
  for (int e = lo; e < hi; ++e) {
    const int a = offsets[e], b = offsets[e + 1];
    if (b < a) bad = true;
    local += (b - a + bm_round) >> bm_shift;
  }
  if (lane == 0 && offsets[0] != 0) bad = true;
  if (lane == 0 && offsets[E] != R) bad = true;
  int incl = local;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, incl, off);
    if (lane >= off) incl += y;
  }
  int run = incl - local;
  for (int e = lo; e < hi; ++e) {
    const int a = offsets[e], b = offsets[e + 1];
    s_off[e] = a;
    s_mstart[e] = run;
    run += (b - a + bm_round) >> bm_shift;
  }
  const bool any_bad = __any_sync(0xffffffffu, bad);
  if (lane == 31) {
    s_mstart[E] = any_bad ? 0 : incl;
    s_off[E] = R;
  }
  if (any_bad && lane == 0) set_status(5);
}

// Optional wait-time instrumentation (compiled in only with MOE_GEMM_TRACE):
// clock cycles per CTA and role spent in each wait, by GEMM mode.
#ifdef MOE_GEMM_TRACE
constexpr int kTraceSlots = 16;
__device__ unsigned long long g_gemm_trace[4][160][kTraceSlots];
#define MOE_TIMED(mode, slot, expr)                                           \
  ([&]() {                                                                    \
    const long long _t = clock64();                                           \
    auto _r = (expr);                                                         \
    if ((threadIdx.x & 31) == 0)                                              \
      atomicAdd(&g_gemm_trace[mode][blockIdx.x % 160][slot],                  \
                static_cast<unsigned long long>(clock64() - _t));             \
    return _r;                                                                \
  }())
#define MOE_TIMED_VOID(mode, slot, stmt)                                      \
  do {                                                                        \
    const long long _t = clock64();                                           \
    stmt;                                                                     \
    if ((threadIdx.x & 31) == 0)                                              \
      atomicAdd(&g_gemm_trace[mode][blockIdx.x % 160][slot],                  \
                static_cast<unsigned long long>(clock64() - _t));             \
  } while (0)
#else
#define MOE_TIMED(mode, slot, expr) (expr)
#define MOE_TIMED_VOID(mode, slot, stmt) stmt
#endif

__device__ __forceinline__ uint4 pack8(const float* v) {
  return make_uint4(pack_bf16x2(v[0], v[1]), pack_bf16x2(v[2], v[3]),
                    pack_bf16x2(v[4], v[5]), pack_bf16x2(v[6], v[7]));
}

// Stores the bf16 roundings of v[0, W) to p[0, W) (a row segment of a
// tile), skipping columns [nvalid, W) (nvalid a multiple of 8, may be <= 0).
// Each thread writes its own row, so 32-byte stores where the address allows
// (whole L2 sectors, half the transactions of 16-byte ones), else 16 bytes.
template <int Q>
__device__ __forceinline__ void store8(__nv_bfloat16* p, const float* v, int nvalid,
                                       uint64_t pol) {
  if (8 * Q < nvalid) st_global_v4_hint(p + 8 * Q, pack8(v + 8 * Q), pol);
}
template <int Q>
__device__ __forceinline__ void store16(__nv_bfloat16* p, const float* v, int nvalid,
                                        uint64_t pol) {
  if (8 * Q + 16 <= nvalid)
    st_global_v8_hint(p + 8 * Q, pack8(v + 8 * Q), pack8(v + 8 * Q + 8), pol);
  else
    store8<Q>(p, v, nvalid, pol);
}
template <int Q, int NQ>
__device__ __forceinline__ void store_pairs(__nv_bfloat16* p, const float* v, int nvalid,
                                            uint64_t pol) {
  if constexpr (Q + 1 < NQ) {
    store16<Q>(p, v, nvalid, pol);
    store_pairs<Q + 2, NQ>(p, v, nvalid, pol);
  } else if constexpr (Q < NQ) {
    store8<Q>(p, v, nvalid, pol);
  }
}

// Stores the bf16 roundings of v[0, W) to p[0, W) (a row segment of a
// tile), skipping columns [nvalid, W) (nvalid a multiple of 8, may be <= 0).
// Each thread writes its own row, so 32-byte stores where the address allows
// (whole L2 sectors, half the transactions of 16-byte ones), else 16 bytes.
template <int W>
__device__ __forceinline__ void store_row_bf16(__nv_bfloat16* p, const float* v, int nvalid,
                                               uint64_t pol) {
  if ((reinterpret_cast<uintptr_t>(p) & 31u) == 0) {
    store_pairs<0, W / 8>(p, v, nvalid, pol);
  } else {
    store8<0>(p, v, nvalid, pol);
    store_pairs<1, W / 8>(p, v, nvalid, pol);
  }
}

// Epilogue step 1: the rank-r product (TMEM columns [BN, BN + r) of this
// thread's row) times s, rounded to bf16, into the swizzled K-major shared
// tile that feeds the up-projection; the first n-tile also saves it
// (transposed) for the backward.
template <int RK>
__device__ __forceinline__ void epi_rank_handoff(const GemmArgs& args, uint32_t t_lora,
                                                 uint8_t* xt, int row_in_tile, int nt,
                                                 bool rvalid, int grow) {
  constexpr uint32_t LSPAN = RK * 2;
  float xa[RK];
#pragma unroll
  for (int c = 0; c < RK; c += 16) tmem_ld16(t_lora + c, xa + c);
  tmem_ld_wait();
#pragma unroll
  for (int i = 0; i < RK; ++i) xa[i] *= args.s;
#pragma unroll
  for (int ch = 0; ch < RK / 8; ++ch)
    *reinterpret_cast<uint4*>(xt + swz_offset(row_in_tile, ch, LSPAN)) = pack8(xa + 8 * ch);
  if (nt == 0 && rvalid && args.lora_t != nullptr) {
#pragma unroll
    for (int q = 0; q < RK; ++q)
      args.lora_t[static_cast<size_t>(q) * args.ld_lora + grow] = __float2bfloat16_rn(xa[q]);
  }
}

// SwiGLU backward: pull this row's saved gate / up segments (this warp's
// share of the columns) into L2 while the up-projection and the next tile's
// mainloop run.
// The tile's columns start at output column col0.
template <int BN>
__device__ __forceinline__ void epi_prefetch_saved(const GemmArgs& args, int grow,
                                                   bool rvalid, int col0, int ehalf) {
  if (!rvalid) return;
  using S = ColSplit<BN>;
  const int c0 = col0 + (ehalf ? S::C0 : 0);
  const int ncol = min(ehalf ? S::C1 : S::C0, args.N - c0);
  if (ncol > 0) {
    const __nv_bfloat16* gp = args.aux + static_cast<size_t>(grow) * args.ld_aux + c0;
    prefetch_l2_bulk(gp, static_cast<uint32_t>(ncol) * 2u);
    prefetch_l2_bulk(gp + args.I, static_cast<uint32_t>(ncol) * 2u);
  }
}

// Epilogue step 2: drain the accumulator of this thread's row with the
// mode's math (SwiGLU; plain store; SwiGLU backward).
// Non-SwiGLU modes can drain a part of the tile: NC columns starting at
// tile column cbase (TMEM column t_acc holds tile column cbase), writing no
// output column at or beyond nlim.
template <int MODE, int BN, bool kSplit, int NC = BN>
__device__ __forceinline__ void epi_drain(const GemmArgs& args, uint32_t t_acc, int grow,
                                          bool rvalid, int nt, int ehalf, int cbase = 0,
                                          int nlim = 0x7fffffff) {
  const int nmax = min(args.N, nlim);
  constexpr bool kSwiGLU = (MODE == kGateUpFwd);
  constexpr int HALF = BN / 2;
  const uint64_t pol = policy_evict_first();  // outputs stream out of L2
  if constexpr (kSwiGLU) {
    // gate columns [0, HALF), up columns [HALF, BN) of the tile
    const int col0 = nt * HALF;
    __nv_bfloat16* hrow = args.out + static_cast<size_t>(grow) * args.ld_out;
    __nv_bfloat16* zrow = args.out2 + static_cast<size_t>(grow) * args.ld_out2;
    for_my_chunks<HALF, kSplit>(ehalf, [&](int c, auto w) {
      constexpr int W = decltype(w)::value;
      float g[W], u[W];
      tmem_ld<W>(t_acc + c, g);
      tmem_ld<W>(t_acc + HALF + c, u);
      tmem_ld_wait();
      if (rvalid) {
        float h[W];
#pragma unroll
        for (int i = 0; i < W; ++i) h[i] = g[i] * sigmoidf_(g[i]) * u[i];
        const int col = col0 + c, nv = args.N - col;
        store_row_bf16<W>(hrow + col, h, nv, pol);
        store_row_bf16<W>(zrow + col, g, nv, pol);
        store_row_bf16<W>(zrow + args.I + col, u, nv, pol);
      }
    });
  } else if constexpr (MODE == kDownBwd) {
    const int col0 = nt * BN + cbase;
    const __nv_bfloat16* grow_p = args.aux + static_cast<size_t>(grow) * args.ld_aux;
    __nv_bfloat16* orow = args.out + static_cast<size_t>(grow) * args.ld_out;
    for_my_chunks<NC, kSplit>(ehalf, [&](int c, auto w) {
      constexpr int W = decltype(w)::value;
      uint4 gv[W / 8], uv[W / 8];
      // loads first (in flight during the TMEM read), 32 bytes at a time
      // where the address allows
      const bool a32 = ((reinterpret_cast<uintptr_t>(grow_p + col0 + c) |
                         reinterpret_cast<uintptr_t>(grow_p + args.I + col0 + c)) & 31u) == 0;
#pragma unroll
      for (int q = 0; q < W / 8; q += 2) {
        const int col = col0 + c + 8 * q;
        gv[q] = uv[q] = make_uint4(0, 0, 0, 0);
        if (q + 1 < W / 8) gv[q + 1] = uv[q + 1] = make_uint4(0, 0, 0, 0);
        if (!rvalid) continue;
        if (q + 1 < W / 8 && a32 && col + 16 <= nmax) {
          ld_global_nc_v8(grow_p + col, gv[q], gv[q + 1]);
          ld_global_nc_v8(grow_p + args.I + col, uv[q], uv[q + 1]);
        } else {
          if (col < nmax) {
            gv[q] = *reinterpret_cast<const uint4*>(grow_p + col);
            uv[q] = *reinterpret_cast<const uint4*>(grow_p + args.I + col);
          }
          if (q + 1 < W / 8 && col + 8 < nmax) {
            gv[q + 1] = *reinterpret_cast<const uint4*>(grow_p + col + 8);
            uv[q + 1] = *reinterpret_cast<const uint4*>(grow_p + args.I + col + 8);
          }
        }
      }
      float dh[W];
      tmem_ld<W>(t_acc + c, dh);
      tmem_ld_wait();
      if (rvalid) {
        float dg[W], du[W];
#pragma unroll
        for (int q = 0; q < W / 8; ++q) {
          const uint32_t ga[4] = {gv[q].x, gv[q].y, gv[q].z, gv[q].w};
          const uint32_t ua[4] = {uv[q].x, uv[q].y, uv[q].z, uv[q].w};
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
        const int col = col0 + c, nv = nmax - col;
        store_row_bf16<W>(orow + col, dg, nv, pol);
        store_row_bf16<W>(orow + args.I + col, du, nv, pol);
      }
    });
  } else {
    const int col0 = nt * BN + cbase;
    __nv_bfloat16* orow = args.out + static_cast<size_t>(grow) * args.ld_out;
    for_my_chunks<NC, kSplit>(ehalf, [&](int c, auto w) {
      constexpr int W = decltype(w)::value;
      float v[W];
      tmem_ld<W>(t_acc + c, v);
      tmem_ld_wait();
      if (rvalid) store_row_bf16<W>(orow + c + col0, v, nmax - col0 - c, pol);
    });
  }
}

template <int MODE, int BN, int RK>
__global__ void __launch_bounds__(gemm_threads(MODE), 1)
    grouped_lora_gemm_kernel(const __grid_constant__ CUtensorMap tmA,
                             const __grid_constant__ CUtensorMap tmB,
                             const __grid_constant__ CUtensorMap tmLA,
                             const __grid_constant__ CUtensorMap tmLB,
                             const GemmArgs args) {
  griddep_sync();  // before any global memory access
  using C = GemmCfg<MODE, BN, RK>;
  constexpr bool kSwiGLU = (MODE == kGateUpFwd);
  constexpr bool kBMN = C::kBMN;
  constexpr int HALF = BN / 2;

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t* sStage = smem;
  uint8_t* sLB = sStage + C::NS * C::STAGE_BYTES;
  uint8_t* sXA = sLB + 2 * C::LB_BYTES;
  uint64_t* full = reinterpret_cast<uint64_t*>(sXA + 2 * C::XA_BYTES);
  uint64_t* empty = full + C::NS;
  uint64_t* lb_full = empty + C::NS;
  uint64_t* lb_empty = lb_full + 2;
  uint64_t* lora_full = lb_empty + 2;
  uint64_t* xa_ready = lora_full + 2;
  uint64_t* acc_full = xa_ready + 2;
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
      mbar_init(&lb_full[i], 1);
      mbar_init(&lb_empty[i], 1);
      mbar_init(&lora_full[i], 1);
      mbar_init(&xa_ready[i], 4);
      mbar_init(&acc_full[i], 1);
      mbar_init(&acc_empty[i], gemm_epi_warps(MODE));
    }
    mbar_init(drain_bar, 1);
    *s_abort = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tmA);
    prefetch_tmap(&tmB);
    prefetch_tmap(&tmLA);
    prefetch_tmap(&tmLB);
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
  const int total_tiles = s_mstart[E] * args.n_tiles;
  const int k_iters = (args.K + C::BK - 1) / C::BK;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      // L2 residency of the operand reused over time (see MOE_L2_HINTS)
#if MOE_L2_HINTS == 2
      const uint64_t pol_w = policy_evict_first();
      const uint64_t pol_a = policy_evict_last();
#elif MOE_L2_HINTS == 1
      const uint64_t pol_w = policy_evict_last();
      const uint64_t pol_a = policy_evict_first();
#else
      const uint64_t pol_w = policy_evict_normal();
      const uint64_t pol_a = policy_evict_normal();
#endif
      int stage = 0;
      uint32_t phase = 0;
      int armed_stages = 0;      // stages armed at least once
      uint32_t lb_armed = 0;     // LB buffers armed at least once
      uint32_t lb_par[2] = {0, 0};
      bool ok = true;
      int local = 0;
      for (int tile = blockIdx.x; tile < total_tiles && ok;
           tile += gridDim.x, ++local) {
        int e, mt, nt;
        decode_tile(tile, args.n_tiles, s_mstart, E, e, mt, nt);
        const int row0 = s_off[e] + mt * C::BM;
        const int b = local & 1;
        const uint32_t use = (local >> 1) & 1;
        if (!MOE_TIMED(MODE, 5, mbar_wait(&lb_empty[b], use ^ 1, s_abort, wait_ns))) { ok = false; break; }
        mbar_arrive_expect_tx(&lb_full[b], C::LB_BYTES);
        lb_armed |= 1u << b;
        lb_par[b] = use;
        uint8_t* lb = sLB + b * C::LB_BYTES;
        if (kSwiGLU) {
          tma_load_2d_hint(lb, &tmLB, &lb_full[b], 0, e * args.lb_rows + nt * HALF, pol_w);
          tma_load_2d_hint(lb + HALF * C::LSPAN, &tmLB, &lb_full[b], 0,
                           e * args.lb_rows + args.I + nt * HALF, pol_w);
        } else {
          tma_load_2d_hint(lb, &tmLB, &lb_full[b], 0, e * args.lb_rows + nt * BN, pol_w);
        }
        for (int kt = 0; kt < k_iters; ++kt) {
          if (!MOE_TIMED(MODE, 4, mbar_wait(&empty[stage], phase ^ 1, s_abort, wait_ns))) { ok = false; break; }
          uint8_t* st = sStage + stage * C::STAGE_BYTES;
          mbar_arrive_expect_tx(&full[stage], C::STAGE_BYTES);
          tma_load_2d_hint(st, &tmA, &full[stage], kt * C::BK, row0, pol_a);
          uint8_t* sb = st + C::A_BYTES;
          if (kBMN) {
#pragma unroll
            for (int i = 0; i < BN / 64; ++i)
              tma_load_2d_hint(sb + i * kMnAtomBytes, &tmB, &full[stage], nt * BN + 64 * i,
                               e * args.b_rows + kt * C::BK, pol_w);
            // factor atom: [K rows, 64 columns] zero-padded past r
            tma_load_2d_hint(sb + (BN / 64) * kMnAtomBytes, &tmLA, &full[stage], 0,
                             e * args.b_rows + kt * C::BK, pol_w);
          } else {
            if (kSwiGLU) {
              tma_load_2d_hint(sb, &tmB, &full[stage], kt * C::BK,
                               e * args.b_rows + nt * HALF, pol_w);
              tma_load_2d_hint(sb + HALF * C::BK * 2, &tmB, &full[stage], kt * C::BK,
                               e * args.b_rows + args.I + nt * HALF, pol_w);
            } else {
              tma_load_2d_hint(sb, &tmB, &full[stage], kt * C::BK, e * args.b_rows + nt * BN,
                               pol_w);
            }
            // factor rows right after the weight rows: one operand of N = BN + r
            tma_load_2d_hint(sb + BN * C::BK * 2, &tmLA, &full[stage], kt * C::BK, e * RK,
                             pol_w);
          }
          if (armed_stages < C::NS) ++armed_stages;
          if (++stage == C::NS) {
            stage = 0;
            phase ^= 1;
          }
        }
      }
      // Wait until every load issued has landed before the CTA may exit.
      for (int i = 0; i < armed_stages; ++i) {
        int s = stage - 1 - i;  // the most recent arming of stage s
        uint32_t ph = phase;
        if (s < 0) {
          s += C::NS;
          ph ^= 1;
        }
        drain_wait(&full[s], ph, wait_ns);
      }
      for (int bb = 0; bb < 2; ++bb)
        if (lb_armed & (1u << bb)) drain_wait(&lb_full[bb], lb_par[bb], wait_ns);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    // The whole warp runs the loop (its state stays warp-uniform); one
    // elected lane issues the tensor-core instructions.
    {
      constexpr uint32_t kIdesc = idesc_bf16_f32(128, C::NMMA, false, kBMN);
      constexpr uint32_t kIdescUp = idesc_bf16_f32(128, BN, false, false);
      // acc[b] += xa[b] * LB[b]^T, then release LB[b] and publish acc[b]
      auto issue_up = [&](int b) {
        const uint32_t t_acc = tmem_base + b * C::ACC_STRIDE;
        const uint32_t xa0 = smem_u32(sXA + b * C::XA_BYTES);
        const uint32_t lb0 = smem_u32(sLB + b * C::LB_BYTES);
#pragma unroll
        for (int kk = 0; kk < RK / 16; ++kk)
          umma_bf16(t_acc, smem_desc(xa0 + kk * 32, 16, 8 * C::LSPAN, C::LLAYOUT),
                    smem_desc(lb0 + kk * 32, 16, 8 * C::LSPAN, C::LLAYOUT), kIdescUp, 1u);
        umma_commit(&lb_empty[b]);
        umma_commit(&acc_full[b]);
      };
      auto up_when_ready = [&](int pb) {
        tc_fence_after();
        if (elect_one()) issue_up(pb);
        __syncwarp();
      };
      // Stage-0 operand descriptors; a stage / K-step moves only the 14-bit
      // start-address field (shared addresses are < 256 KB, so adding the
      // byte offset >> 4 never carries out of it).
      const uint64_t a_desc0 = smem_desc(smem_u32(sStage), 16, kKmajSBO, kKmajLayout);
      const uint64_t b_desc0 =
          kBMN ? smem_desc(smem_u32(sStage) + C::A_BYTES, kMnAtomBytes, 1024, kLayoutSW128)
               : smem_desc(smem_u32(sStage) + C::A_BYTES, 16, kKmajSBO, kKmajLayout);
      constexpr uint64_t kStageInc = C::STAGE_BYTES >> 4;
      constexpr uint64_t kAStep = 32 >> 4;                     // 16 K of K-major
      constexpr uint64_t kBStep = kBMN ? (2048 >> 4) : (32 >> 4);  // 16 K rows / cols
      int stage = 0;
      uint64_t soff = 0;
      uint32_t phase = 0;
      int local = 0;
      int pending = -1;  // local index of the tile whose up-projection is due
      bool ok = true;
      // Testing hook: wait on a barrier that nothing arrives on before the
      // end of the kernel, so the bounded wait runs out and the whole CTA
      // takes its abort path.
      if (args.stall_test) ok = warp_wait(drain_bar, 0, s_abort, wait_ns);
#ifdef MOE_GEMM_TRACE
      const long long t_role = clock64();
#endif
      for (int tile = blockIdx.x; ok && tile < total_tiles; tile += gridDim.x, ++local) {
        const int b = local & 1;
        const uint32_t use = (local >> 1) & 1;
        const uint32_t t_acc = tmem_base + b * C::ACC_STRIDE;
        if (!MOE_TIMED(MODE, 1, warp_wait(&acc_empty[b], use ^ 1, s_abort, wait_ns))) { ok = false; break; }
        tc_fence_after();
        for (int kt = 0; kt < k_iters; ++kt) {
          // (TMA -> MMA ordering comes with the barrier; no tcgen05 fence)
          if (!MOE_TIMED(MODE, 0, warp_wait(&full[stage], phase, s_abort, wait_ns))) { ok = false; break; }
          const uint64_t da = a_desc0 + soff, db = b_desc0 + soff;
          if (elect_one()) {
            umma_bf16(t_acc, da, db, kIdesc, kt > 0 ? 1u : 0u);
#pragma unroll
            for (int kk = 1; kk < C::BK / 16; ++kk)
              umma_bf16(t_acc, da + kk * kAStep, db + kk * kBStep, kIdesc, 1u);
            umma_commit(&empty[stage]);
          }
          __syncwarp();
          soff += kStageInc;
          if (++stage == C::NS) {
            stage = 0;
            soff = 0;
            phase ^= 1;
          }
          if (pending >= 0) {  // previous tile's up-projection, once it is ready
            const int pb = pending & 1;
            const uint32_t pu = (pending >> 1) & 1;
            if (warp_uniform(mbar_test_wait(&xa_ready[pb], pu) &&
                             mbar_test_wait(&lb_full[pb], pu))) {
              up_when_ready(pb);
              pending = -1;
            }
          }
        }
        if (!ok) break;
        if (elect_one()) umma_commit(&lora_full[b]);
        __syncwarp();
        if (pending >= 0) {
          const int pb = pending & 1;
          const uint32_t pu = (pending >> 1) & 1;
          if (!MOE_TIMED(MODE, 2, warp_wait(&xa_ready[pb], pu, s_abort, wait_ns)) ||
              !MOE_TIMED(MODE, 3, warp_wait(&lb_full[pb], pu, s_abort, wait_ns))) { ok = false; break; }
          up_when_ready(pb);
        }
        pending = local;
      }
      if (ok && pending >= 0) {
        const int pb = pending & 1;
        const uint32_t pu = (pending >> 1) & 1;
        if (warp_wait(&xa_ready[pb], pu, s_abort, wait_ns) &&
            warp_wait(&lb_full[pb], pu, s_abort, wait_ns))
          up_when_ready(pb);
      }
#ifdef MOE_GEMM_TRACE
      if (lane == 0)
        atomicAdd(&g_gemm_trace[MODE][blockIdx.x % 160][7],
                  static_cast<unsigned long long>(clock64() - t_role));
#endif
      // every MMA issued by this warp must be complete before TMEM is freed
      if (elect_one()) umma_commit(drain_bar);
      __syncwarp();
      drain_wait(drain_bar, 0, wait_ns);
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int ew = warp & 3;              // TMEM lane quarter
    constexpr bool kSplit = gemm_epi_warps(MODE) == 8;
    const int ehalf = (warp - 2) >> 2;    // which share of the columns
    const int row_in_tile = ew * 32 + lane;
    const uint32_t lane_base = static_cast<uint32_t>(ew * 32) << 16;
    int local = 0;
    for (int tile = blockIdx.x; tile < total_tiles; tile += gridDim.x, ++local) {
      int e, mt, nt;
      decode_tile(tile, args.n_tiles, s_mstart, E, e, mt, nt);
      const int b = local & 1;
      const uint32_t use = (local >> 1) & 1;
      const int grow = s_off[e] + mt * C::BM + row_in_tile;
      const bool rvalid = grow < s_off[e + 1];
      const uint32_t t_acc = tmem_base + lane_base + b * C::ACC_STRIDE;
      const uint32_t t_lora = t_acc + BN;

      // rank-r product: TMEM -> bf16 A operand of the up-projection (done by
      // the first four epilogue warps)
      if (ehalf == 0) {
        if (!MOE_TIMED(MODE, 8, warp_wait(&lora_full[b], use, s_abort, wait_ns))) break;
        tc_fence_after();
        epi_rank_handoff<RK>(args, t_lora, sXA + b * C::XA_BYTES, row_in_tile, nt, rvalid,
                             grow);
        fence_proxy_async_smem();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&xa_ready[b]);
      }
      if constexpr (MODE == kDownBwd) epi_prefetch_saved<BN>(args, grow, rvalid, nt * BN, ehalf);

      if (!MOE_TIMED(MODE, 9, warp_wait(&acc_full[b], use, s_abort, wait_ns))) break;
      tc_fence_after();
      MOE_TIMED_VOID(MODE, 10, (epi_drain<MODE, BN, kSplit>(args, t_acc, grow, rvalid, nt, ehalf)));
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&acc_empty[b]);
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
