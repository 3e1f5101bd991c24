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

// ------------------------------------------------------- one-launch routing
// The four steps above in one cooperative launch.  CTA b takes the tokens
// [b * tpc, + tpc) and their flat entries [b * tpc * k, ...): top-k and
// weights (a warp per token), then the stable rank of each entry among the
// CTA's earlier entries of its expert and the CTA's expert histogram
// (rounds of kRFThreads entries), published to blk_hist[b].  One grid-wide
// wait (a counter the host zeroes before the launch; bounded by wait_ns)
// makes every histogram visible; then each CTA sums them (integers, so the
// result does not depend on the order) into the expert totals and its own
// base row per expert, and writes dest for its entries.  CTA 0 writes the
// counts and offsets.  Same outputs, bit for bit, as the four kernels.
constexpr int kRFWarps = 16;
constexpr int kRFThreads = kRFWarps * 32;
constexpr int kRFMaxCtas = 256;

__host__ __device__ constexpr size_t route_fused_smem(int E, int k) {
  // s_val [warps][k] f32, s_cnt [warps][E], s_run / s_base / s_off [E + 1]
  return (static_cast<size_t>(kRFWarps) * k + static_cast<size_t>(kRFWarps) * E +
          3 * static_cast<size_t>(E + 1)) * 4;
}

template <int EPL>
__global__ void __launch_bounds__(kRFThreads)
    route_fused_kernel(const float* __restrict__ logits, int T, int E, int k, int tpc,
                       int32_t* __restrict__ idx_out, float* __restrict__ w_out,
                       int32_t* __restrict__ counts, int32_t* __restrict__ offsets,
                       int32_t* __restrict__ dest, int32_t* __restrict__ blk_hist,
                       int32_t* __restrict__ local_rank, unsigned int* __restrict__ arrived,
                       uint64_t wait_ns) {
  extern __shared__ int smem_rf[];
  float* s_val = reinterpret_cast<float*>(smem_rf);     // [warps][k]
  int* s_cnt = smem_rf + kRFWarps * k;                    // [warps][E]
  int* s_run = s_cnt + kRFWarps * E;                      // [E + 1]
  int* s_base = s_run + (E + 1);                          // [E + 1]
  int* s_off = s_base + (E + 1);                          // [E + 1]
  __shared__ int s_ok;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int G = gridDim.x, b = blockIdx.x;
  const int R = T * k;
  const int t0 = min(T, b * tpc), t1 = min(T, t0 + tpc);
  const int f0 = t0 * k, f1 = t1 * k;

  // 1. top-k and renormalised weights, a warp per token
  float* my_val = s_val + warp * k;
  for (int t = t0 + warp; t < t1; t += kRFWarps) {
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
    float denom = 0.f;
    const float vmax = my_val[0];
    for (int j = 0; j < k; ++j) denom += expf(my_val[j] - vmax);
    for (int j = lane; j < k; j += 32)
      w_out[static_cast<size_t>(t) * k + j] = expf(my_val[j] - vmax) / denom;
    __syncwarp();
  }
  for (int e = tid; e < E; e += kRFThreads) s_run[e] = 0;
  __syncthreads();

  // 2. stable ranks within the CTA, rounds of kRFThreads entries (warp w
  // takes the round's entries 32w .. 32w + 31)
  for (int r0 = f0; r0 < f1; r0 += kRFThreads) {
    for (int i = tid; i < kRFWarps * E; i += kRFThreads) s_cnt[i] = 0;
    __syncthreads();
    const int f = r0 + tid;
    const bool valid = f < f1;
    int e = valid ? idx_out[f] : -1 - lane;
    if (valid && (e < 0 || e >= E)) {
      set_status(5);
      e = 0;
    }
    const uint32_t m = __match_any_sync(0xffffffffu, e);
    const int inwarp = __popc(m & ((1u << lane) - 1u));
    if (valid && lane == __ffs(m) - 1) s_cnt[warp * E + e] = __popc(m);
    __syncthreads();
    for (int x = tid; x < E; x += kRFThreads) {
      int run = s_run[x];
      for (int w = 0; w < kRFWarps; ++w) {
        const int c = s_cnt[w * E + x];
        s_cnt[w * E + x] = run;
        run += c;
      }
      s_run[x] = run;
    }
    __syncthreads();
    if (valid) local_rank[f] = s_cnt[warp * E + e] + inwarp;
    __syncthreads();
  }
  for (int e = tid; e < E; e += kRFThreads) blk_hist[static_cast<size_t>(b) * E + e] = s_run[e];

  // 3. every CTA's histogram is published before any CTA reads them
  __threadfence();
  __syncthreads();
  if (tid == 0) {
    atomicAdd(arrived, 1u);
    const uint64_t tstart = globaltimer_ns();
    int ok = 1;
    while (*reinterpret_cast<volatile unsigned int*>(arrived) < static_cast<unsigned int>(G)) {
      if (globaltimer_ns() - tstart > wait_ns) {
        set_status(4 /* MOE_ERR_DEVICE_TIMEOUT */);
        ok = 0;
        break;
      }
    }
    __threadfence();
    s_ok = ok;
  }
  __syncthreads();
  if (!s_ok) return;

  // 4. expert totals (s_off) and this CTA's base row per expert (s_base):
  // the [G, E] histograms read as 16-byte vectors, eight in flight per
  // thread, summed with shared-memory integer atomics (exact in any order)
  for (int e = tid; e < E; e += kRFThreads) {
    s_base[e] = 0;
    s_off[e] = 0;
  }
  __syncthreads();
  {
    const int n = G * E, n4 = n >> 2;
    const int4* h4 = reinterpret_cast<const int4*>(blk_hist);
    auto add = [&](int i, int c) {
      const int q = i / E, e = i - q * E;
      atomicAdd(&s_off[e], c);
      if (q < b) atomicAdd(&s_base[e], c);
    };
    for (int v0 = tid; v0 < n4; v0 += kRFThreads * 8) {
      int4 v[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int x = v0 + kRFThreads * u;
        v[u] = x < n4 ? __ldcg(h4 + x) : make_int4(0, 0, 0, 0);
      }
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int x = v0 + kRFThreads * u;
        if (x < n4) {
          add(4 * x, v[u].x);
          add(4 * x + 1, v[u].y);
          add(4 * x + 2, v[u].z);
          add(4 * x + 3, v[u].w);
        }
      }
    }
    for (int i = 4 * n4 + tid; i < n; i += kRFThreads) add(i, __ldcg(blk_hist + i));
  }
  __syncthreads();
  if (warp == 0) {  // exclusive scan of the totals (in s_off) by one warp
    const int per_lane = (E + 31) / 32;
    const int lo = lane * per_lane, hi = min(E, lo + per_lane);
    int local = 0;
    for (int i = lo; i < hi; ++i) local += s_off[i];
    int incl = local;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, incl, off);
      if (lane >= off) incl += y;
    }
    int run = incl - local;
    for (int i = lo; i < hi; ++i) {
      const int c = s_off[i];
      if (b == 0) counts[i] = c;
      s_off[i] = run;
      run += c;
    }
    if (lane == 31 && run != R) set_status(5);
  }
  __syncthreads();
  if (b == 0)
    for (int e = tid; e <= E; e += kRFThreads) offsets[e] = e == E ? R : s_off[e];

  // 5. destination rows of this CTA's entries
  for (int f = f0 + tid; f < f1; f += kRFThreads) {
    int e = idx_out[f];
    if (e < 0 || e >= E) e = 0;  // recorded in step 2
    int d = s_off[e] + s_base[e] + local_rank[f];
    if (d < 0 || d >= R) {
      set_status(5);
      d = 0;
    }
    dest[f] = d;
  }
}

}  // namespace moe
