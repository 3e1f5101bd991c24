// a1: fused softmax / top-k router, per-block expert histogram with stable
// in-block ranks, a deterministic cross-block scan, and destination rows.
//
// Routing follows the Unsloth page "Fine-tune MoE LLMs 12x faster with
// Unsloth": each token goes to the k experts its (frozen) router ranks
// highest; the kept probabilities are renormalised to sum to one.  The
// permutation is the grouping of the page's per-expert loop (section "What
// is torch._grouped_mm?"), done as a stable counting sort over t*k + j.
#pragma once

#include "ptx.cuh"

namespace moe {

constexpr int kRouteWarps = 8;          // top-k: one token per warp
constexpr int kRankWarps = 16;          // ranking: 16 warps per CTA
constexpr int kRankPerWarp = 128;       // flat entries per warp
constexpr int kRankChunk = kRankWarps * kRankPerWarp;  // entries per CTA

__device__ __forceinline__ bool better(float va, int ea, float vb, int eb) {
  return va > vb || (va == vb && ea < eb);
}

// One warp per token.  Lane l holds experts l, l+32, ... (EPL of them).
// Writes the k selected experts (logit desc, index asc) and their
// renormalised weights.  Per-warp scratch in shared memory: k values.
template <int EPL>
__global__ void __launch_bounds__(kRouteWarps * 32)
    route_topk_kernel(const float* __restrict__ logits, int T, int E, int k,
                      int32_t* __restrict__ idx_out, float* __restrict__ w_out) {
  griddep_sync();  // before any global memory access
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  extern __shared__ float s_val_all[];
  float* my_val = s_val_all + warp * k;
  const int t = blockIdx.x * kRouteWarps + warp;
  if (t >= T) return;
  float v[EPL];
  uint32_t taken = 0;
#pragma unroll
  for (int q = 0; q < EPL; ++q) {
    const int e = lane + 32 * q;
    if (e < E) {
      const float x = __ldg(logits + static_cast<size_t>(t) * E + e);
      v[q] = (x != x) ? -INFINITY : x;  // NaN never outranks a number
    } else {
      v[q] = -INFINITY;
      taken |= 1u << q;
    }
  }
  for (int j = 0; j < k; ++j) {
    float bv = -INFINITY;
    int be = 0x7fffffff;
#pragma unroll
    for (int q = 0; q < EPL; ++q) {
      const int e = lane + 32 * q;
      if (!((taken >> q) & 1u) && better(v[q], e, bv, be)) {
        bv = v[q];
        be = e;
      }
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
      const float ov = __shfl_xor_sync(0xffffffffu, bv, off);
      const int oe = __shfl_xor_sync(0xffffffffu, be, off);
      if (better(ov, oe, bv, be)) {
        bv = ov;
        be = oe;
      }
    }
    if (be >= E) {  // cannot happen for k <= E; keep indices in range
      set_status(5);
      be = 0;
    }
    if (lane == (be & 31)) taken |= 1u << (be >> 5);
    if (lane == 0) {
      my_val[j] = bv;
      idx_out[static_cast<size_t>(t) * k + j] = be;
    }
  }
  __syncwarp();
  // renormalised softmax over the k kept logits (my_val[0] is the max)
  float denom = 0.f;
  const float vmax = my_val[0];
  for (int j = 0; j < k; ++j) denom += expf(my_val[j] - vmax);
  for (int j = lane; j < k; j += 32)
    w_out[static_cast<size_t>(t) * k + j] = expf(my_val[j] - vmax) / denom;
}

// One CTA per kRankChunk consecutive flat entries f = t*k + j: the stable rank
// of each entry among the chunk's earlier entries of the same expert, and the
// chunk's expert histogram.
__global__ void __launch_bounds__(kRankWarps * 32)
    route_rank_kernel(const int32_t* __restrict__ idx, int R, int E,
                      int32_t* __restrict__ blk_hist,
                      int32_t* __restrict__ local_rank) {
  griddep_sync();  // before any global memory access
  extern __shared__ int s_cnt[];  // [kRankWarps][E]
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int i = threadIdx.x; i < kRankWarps * E; i += blockDim.x) s_cnt[i] = 0;
  __syncthreads();
  const int f0 = blockIdx.x * kRankChunk + warp * kRankPerWarp;
  int* cnt = s_cnt + warp * E;
  int rank[kRankPerWarp / 32];
  int ex[kRankPerWarp / 32];
#pragma unroll
  for (int p = 0; p < kRankPerWarp / 32; ++p) {
    const int f = f0 + p * 32 + lane;
    const bool valid = f < R;
    int e = valid ? idx[f] : -1 - lane;
    if (valid && (e < 0 || e >= E)) {  // defensive: keep shared indices in range
      set_status(5);
      e = 0;
    }
    const uint32_t m = __match_any_sync(0xffffffffu, e);
    rank[p] = valid ? __popc(m & ((1u << lane) - 1u)) + cnt[e] : 0;
    ex[p] = e;
    __syncwarp();
    if (valid && lane == __ffs(m) - 1) cnt[e] += __popc(m);
    __syncwarp();
  }
  __syncthreads();
  // exclusive scan over warps per expert -> chunk histogram
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    int run = 0;
    for (int w = 0; w < kRankWarps; ++w) {
      const int c = s_cnt[w * E + e];
      s_cnt[w * E + e] = run;
      run += c;
    }
    blk_hist[static_cast<size_t>(blockIdx.x) * E + e] = run;
  }
  __syncthreads();
#pragma unroll
  for (int p = 0; p < kRankPerWarp / 32; ++p) {
    const int f = f0 + p * 32 + lane;
    if (f < R) local_rank[f] = rank[p] + cnt[ex[p]];
  }
}

// One CTA: per-expert totals over the blocks (in parallel partitions), the
// exclusive expert offsets, and each block's base row per expert (in place in
// blk_hist).  Deterministic: integer sums in a fixed order.
__global__ void __launch_bounds__(1024)
    route_scan_kernel(int32_t* __restrict__ blk_hist, int nblk, int E, int R,
                      int32_t* __restrict__ counts,
                      int32_t* __restrict__ offsets) {
  griddep_sync();  // before any global memory access
  extern __shared__ int smem_i[];
  const int P = max(1, static_cast<int>(blockDim.x) / E);
  int* s_part = smem_i;              // [P][E]
  int* s_off = s_part + P * E;       // [E + 1]
  const int tid = threadIdx.x;
  const int e = tid % E, p = tid / E;
  const int per = (nblk + P - 1) / P;
  const int b0 = p * per, b1 = min(nblk, b0 + per);
  if (p < P) {
    int sum = 0;
    for (int b = b0; b < b1; ++b) sum += blk_hist[static_cast<size_t>(b) * E + e];
    s_part[p * E + e] = sum;
  }
  __syncthreads();
  if (tid < E) {
    int run = 0;
    for (int q = 0; q < P; ++q) {
      const int c = s_part[q * E + tid];
      s_part[q * E + tid] = run;
      run += c;
    }
    counts[tid] = run;
    s_off[tid] = run;
  }
  __syncthreads();
  if (tid < 32) {  // exclusive scan of the counts by one warp
    const int per_lane = (E + 31) / 32;
    const int lo = tid * per_lane, hi = min(E, lo + per_lane);
    int local = 0;
    for (int i = lo; i < hi; ++i) local += s_off[i];
    int incl = local;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, incl, off);
      if (tid >= off) incl += y;
    }
    int run = incl - local;
    for (int i = lo; i < hi; ++i) {
      const int c = s_off[i];
      s_off[i] = run;
      run += c;
    }
  }
  __syncthreads();
  if (tid <= E) offsets[tid] = (tid == E) ? R : s_off[tid];
  if (tid == E && s_off[E - 1] + counts[E - 1] != R) set_status(5);
  if (p < P) {
    int run = s_off[e] + s_part[p * E + e];
    for (int b = b0; b < b1; ++b) {
      const size_t o = static_cast<size_t>(b) * E + e;
      const int c = blk_hist[o];
      blk_hist[o] = run;
      run += c;
    }
  }
}

// dest[f] = base row of (chunk of f, expert) + in-chunk stable rank.
__global__ void route_dest_kernel(const int32_t* __restrict__ idx,
                                  const int32_t* __restrict__ blk_base,
                                  const int32_t* __restrict__ local_rank,
                                  int R, int E, int32_t* __restrict__ dest) {
  griddep_sync();  // before any global memory access
  for (int f = blockIdx.x * blockDim.x + threadIdx.x; f < R;
       f += gridDim.x * blockDim.x) {
    const int b = f / kRankChunk;
    const int e = idx[f];
    int d = blk_base[static_cast<size_t>(b) * E + e] + local_rank[f];
    if (d < 0 || d >= R) {
      set_status(5);
      d = 0;
    }
    dest[f] = d;
  }
}

}  // namespace moe
