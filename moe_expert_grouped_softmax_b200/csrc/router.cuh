// Trainable router (the pages keep the router frozen by default; this is the
// optional variant): the router's linear layer and its backward.
//
//   forward:  logits = X Wr^T                        [T, E] fp32
//   backward: for token t and kept slot j (softmax over the kept logits;
//             the top-k choice itself is piecewise constant)
//               g[t, j] = w[t, j] (dw[t, j] - sum_i w[t, i] dw[t, i])
//             dWr[e]  = sum over the rows of expert e of g * Xp[row]  [E, H]
//             dX[t]  += sum_j g[t, j] Wr[idx[t, j]]  (inside the dX combine)
#pragma once

#include "gemm.cuh"
#include "permute.cuh"

namespace moe {

// ------------------------------------------------------------- logits GEMM
// One CTA per 128 tokens and per BN experts: M = 128 tokens, N = BN experts
// (E rounded up to a multiple of 16, at most 256 per CTA), K = H, on tcgen05
// with TMA-fed 128-byte-swizzled K-major operands; a single accumulator read
// back as fp32.  Warp 0: TMA; warp 1: MMA (one elected lane); warps 2-5:
// epilogue.
template <int BN>
struct RouterCfg {
  static constexpr int BM = 128, BK = 64;
  static constexpr int A_BYTES = BM * BK * 2;
  static constexpr int B_BYTES = BN * BK * 2;
  static constexpr int STAGE_BYTES = (A_BYTES + B_BYTES + 1023) / 1024 * 1024;
  static constexpr int NS = 4;
  static constexpr int SMEM_BYTES = 1024 + NS * STAGE_BYTES + 256;
  static constexpr int TMEM_COLS = BN <= 32 ? 32 : (BN <= 64 ? 64 : (BN <= 128 ? 128 : 256));
  static_assert(BN % 16 == 0 && BN <= 256, "MMA N");
  static_assert(SMEM_BYTES <= kSmemOptin, "router shared memory");
};

template <int BN>
__global__ void __launch_bounds__(192, 1)
    router_logits_kernel(const __grid_constant__ CUtensorMap tmX,
                         const __grid_constant__ CUtensorMap tmW, int T, int H, int E,
                         float* __restrict__ logits, uint64_t wait_ns) {
  griddep_sync();  // before any global memory access
  using C = RouterCfg<BN>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t* sStage = smem;
  uint64_t* full = reinterpret_cast<uint64_t*>(sStage + C::NS * C::STAGE_BYTES);
  uint64_t* empty = full + C::NS;
  uint64_t* acc_full = empty + C::NS;
  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(acc_full + 1);
  volatile int* s_abort = reinterpret_cast<volatile int*>(s_tmem + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int row0 = blockIdx.x * C::BM, n0 = blockIdx.y * BN;
  const int k_iters = (H + C::BK - 1) / C::BK;

  if (threadIdx.x == 0) {
    for (int i = 0; i < C::NS; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 1);
    }
    mbar_init(acc_full, 1);
    *s_abort = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tmX);
    prefetch_tmap(&tmW);
  }
  if (warp == 1) {
    tmem_alloc(s_tmem, C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *s_tmem;

  if (warp == 0) {
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      int armed = 0;
      for (int kt = 0; kt < k_iters; ++kt) {
        if (!mbar_wait(&empty[stage], phase ^ 1, s_abort, wait_ns)) break;
        uint8_t* st = sStage + stage * C::STAGE_BYTES;
        mbar_arrive_expect_tx(&full[stage], C::A_BYTES + C::B_BYTES);
        tma_load_2d(st, &tmX, &full[stage], kt * C::BK, row0);
        tma_load_2d(st + C::A_BYTES, &tmW, &full[stage], kt * C::BK, n0);
        if (armed < C::NS) ++armed;
        if (++stage == C::NS) {
          stage = 0;
          phase ^= 1;
        }
      }
      for (int i = 0; i < armed; ++i) {  // every copy lands before exit
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
    constexpr uint32_t kIdesc = idesc_bf16_f32(128, BN, false, false);
    const uint64_t a_desc0 = smem_desc(smem_u32(sStage), 16, 1024, kLayoutSW128);
    const uint64_t b_desc0 = smem_desc(smem_u32(sStage) + C::A_BYTES, 16, 1024, kLayoutSW128);
    int stage = 0;
    uint32_t phase = 0;
    for (int kt = 0; kt < k_iters; ++kt) {
      if (!warp_wait(&full[stage], phase, s_abort, wait_ns)) break;
      const uint64_t soff = static_cast<uint64_t>(stage) * (C::STAGE_BYTES >> 4);
      if (elect_one()) {
#pragma unroll
        for (int kk = 0; kk < C::BK / 16; ++kk)
          umma_bf16(tmem_base, a_desc0 + soff + 2 * kk, b_desc0 + soff + 2 * kk, kIdesc,
                    (kt | kk) ? 1u : 0u);
        umma_commit(&empty[stage]);
      }
      __syncwarp();
      if (++stage == C::NS) {
        stage = 0;
        phase ^= 1;
      }
    }
    if (elect_one()) umma_commit(acc_full);
    __syncwarp();
    drain_wait(acc_full, 0, wait_ns);  // all MMAs done before TMEM is freed
  } else {
    const int ew = warp & 3;
    const int t = row0 + ew * 32 + lane;
    const uint32_t t_acc = tmem_base + (static_cast<uint32_t>(ew * 32) << 16);
    if (warp_wait(acc_full, 0, s_abort, wait_ns)) {
      tc_fence_after();
      for_chunks<BN>([&](int c, auto w) {
        constexpr int W = decltype(w)::value;
        float v[W];
        tmem_ld<W>(t_acc + c, v);
        tmem_ld_wait();
        if (t < T) {
          float* o = logits + static_cast<size_t>(t) * E;
#pragma unroll
          for (int i = 0; i < W; ++i)
            if (n0 + c + i < E) o[n0 + c + i] = v[i];
        }
      });
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

// ---------------------------------------------------------- logit gradient
// One thread per token: g[t, j] = w_j (dw_j - sum_i w_i dw_i) for its k kept
// slots (fp32, slots in order), also scattered to the token's permuted rows
// (g_row[dest[t, j]]) for the weight gradient.
__global__ void router_dlogit_kernel(const float* __restrict__ w, const float* __restrict__ dw,
                                     const int32_t* __restrict__ dest, int T, int k,
                                     float* __restrict__ g, float* __restrict__ g_row) {
  griddep_sync();  // before any global memory access
  const int R = T * k;
  for (int t = blockIdx.x * blockDim.x + threadIdx.x; t < T; t += gridDim.x * blockDim.x) {
    const size_t b = static_cast<size_t>(t) * k;
    float mean = 0.f;
    for (int j = 0; j < k; ++j) mean = fmaf(w[b + j], dw[b + j], mean);
    for (int j = 0; j < k; ++j) {
      const float gj = w[b + j] * (dw[b + j] - mean);
      g[b + j] = gj;
      const int d = dest[b + j];
      if (d < 0 || d >= R) {
        set_status(5);
        continue;
      }
      g_row[d] = gj;
    }
  }
}

// ----------------------------------------------------------- weight gradient
// dWr[e, c] = sum over the rows of expert e of g_row * Xp[row, c], fp32.
// One CTA per (expert, 256-column chunk), 8 warps: warp w takes rows
// a + w, a + w + 8, ... with each lane owning 8 adjacent columns (one 16-byte
// load per row), and the 8 partial sums are added in warp order at the end,
// so the result does not depend on timing.
constexpr int kRouterWCols = 256;
__global__ void __launch_bounds__(256)
    router_wgrad_kernel(const __nv_bfloat16* __restrict__ Xp, const float* __restrict__ g_row,
                        const int32_t* __restrict__ offsets, int E, int H, int R,
                        float* __restrict__ dWr) {
  griddep_sync();  // before any global memory access
  __shared__ float part[8][kRouterWCols];
  const int e = blockIdx.x;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int c0 = blockIdx.y * kRouterWCols + 8 * lane;
  int a = offsets[e], b = offsets[e + 1];
  if (a < 0 || b > R || a > b) {
    if (threadIdx.x == 0) set_status(5);
    a = b = 0;
  }
  float acc[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) acc[i] = 0.f;
  if (c0 < H) {  // H is a multiple of 16: the 8 columns are all in range
    const __nv_bfloat16* col = Xp + c0;
#pragma unroll 4
    for (int row = a + warp; row < b; row += 8) {
      const float gr = g_row[row];
      const uint4 x = ld_nc_v4(col + static_cast<size_t>(row) * H);
      acc[0] = fmaf(gr, bf16_lo(x.x), acc[0]);
      acc[1] = fmaf(gr, bf16_hi(x.x), acc[1]);
      acc[2] = fmaf(gr, bf16_lo(x.y), acc[2]);
      acc[3] = fmaf(gr, bf16_hi(x.y), acc[3]);
      acc[4] = fmaf(gr, bf16_lo(x.z), acc[4]);
      acc[5] = fmaf(gr, bf16_hi(x.z), acc[5]);
      acc[6] = fmaf(gr, bf16_lo(x.w), acc[6]);
      acc[7] = fmaf(gr, bf16_hi(x.w), acc[7]);
    }
  }
#pragma unroll
  for (int i = 0; i < 8; ++i) part[warp][8 * lane + i] = acc[i];
  __syncthreads();
  const int c = blockIdx.y * kRouterWCols + threadIdx.x;
  if (c < H) {
    float sum = 0.f;
#pragma unroll
    for (int w = 0; w < 8; ++w) sum += part[w][threadIdx.x];
    dWr[static_cast<size_t>(e) * H + c] = sum;
  }
}

}  // namespace moe
