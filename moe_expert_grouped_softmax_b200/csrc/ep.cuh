// Expert parallelism: the row reorder on the receiving rank.  With the E
// experts split over N ranks (rank p holds experts [p * EL, (p + 1) * EL)),
// every rank routes and permutes its own tokens into expert-major order,
// which is already the order of destination ranks, so one all-to-all sends
// each rank its experts' rows.  The receive buffer then holds, for each
// source rank s in turn, that source's rows for the local experts in expert
// order (source-major: segment (s, e)).  The local grouped GEMMs want
// expert-major order over all sources (segment (e, s)); within a segment the
// rows keep their order, so the local rows of expert e come in the order of
// the source ranks, then of the source's flat index t * k + j: the order a
// single rank routing the concatenation of all ranks' tokens would give.
#pragma once

#include "ptx.cuh"

namespace moe {

constexpr int kRegroupThreads = 256;
constexpr int kRegroupMaxSegs = 4096;  // N * EL

// Exclusive prefix sum of get(0 .. n-1), written through put(i, prefix), by
// the whole CTA (each thread a contiguous run, then warp and CTA scans).
// s_warp holds one int per warp.
template <class Get, class Put>
__device__ void block_exclusive_scan(int n, Get get, Put put, int* s_warp) {
  const int tid = threadIdx.x, nt = blockDim.x, lane = tid & 31, warp = tid >> 5;
  const int nw = nt >> 5;
  const int per = (n + nt - 1) / nt;
  const int lo = min(n, tid * per), hi = min(n, lo + per);
  int local = 0;
  for (int i = lo; i < hi; ++i) local += get(i);
  int incl = local;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, incl, off);
    if (lane >= off) incl += y;
  }
  if (lane == 31) s_warp[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    const int ws = lane < nw ? s_warp[lane] : 0;
    int wi = ws;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, wi, off);
      if (lane >= off) wi += y;
    }
    __syncwarp();
    if (lane < nw) s_warp[lane] = wi - ws;
  }
  __syncthreads();
  int run = s_warp[warp] + incl - local;
  for (int i = lo; i < hi; ++i) {
    const int c = get(i);
    put(i, run);
    run += c;
  }
  __syncthreads();
}

// dir 0: out[expert-major row] = in[source-major row]; dir 1: the reverse
// (out source-major from in expert-major).  counts [N, EL]: rows source s
// holds for local expert e; rows = their sum.  With dir 0 and offsets !=
// nullptr, CTA 0 also writes offsets[e] = first expert-major row of expert
// e, offsets[EL] = rows.  One warp per source-major row, 16-byte vectors.
__global__ void __launch_bounds__(kRegroupThreads)
    ep_regroup_kernel(const __nv_bfloat16* __restrict__ in, const int32_t* __restrict__ counts,
                      int N, int EL, int rows, int H, int dir,
                      __nv_bfloat16* __restrict__ out, int32_t* __restrict__ offsets) {
  griddep_sync();  // before any global memory access
  extern __shared__ int sm_rg[];
  const int nseg = N * EL;
  int* s_src = sm_rg;              // [nseg + 1]: segment (s, e) start, source-major
  int* s_dst = s_src + nseg + 1;   // [nseg]: segment (s, e) start, expert-major
  int* s_warp = s_dst + nseg;      // [32]
  __shared__ int s_bad;
  if (threadIdx.x == 0) s_bad = 0;
  __syncthreads();
  block_exclusive_scan(
      nseg,
      [&](int i) {
        const int c = counts[i];
        if (c < 0) s_bad = 1;
        return c < 0 ? 0 : c;
      },
      [&](int i, int v) { s_src[i] = v; }, s_warp);
  block_exclusive_scan(
      nseg,
      [&](int m) {  // m = e * N + s
        const int c = counts[(m % N) * EL + m / N];
        return c < 0 ? 0 : c;
      },
      [&](int m, int v) { s_dst[(m % N) * EL + m / N] = v; }, s_warp);
  if (threadIdx.x == 0) {
    const int last = counts[nseg - 1];
    if (s_bad || s_src[nseg - 1] + (last < 0 ? 0 : last) != rows) {
      s_bad = 1;
      set_status(5);
    }
    s_src[nseg] = rows;
  }
  __syncthreads();
  if (s_bad) return;
  if (dir == 0 && offsets != nullptr && blockIdx.x == 0)
    for (int e = threadIdx.x; e <= EL; e += blockDim.x) offsets[e] = e == EL ? rows : s_dst[e];
  const int lane = threadIdx.x & 31;
  const int nvec = H >> 3;
  const int warps = (gridDim.x * blockDim.x) >> 5;
  for (int i = (blockIdx.x * blockDim.x + threadIdx.x) >> 5; i < rows; i += warps) {
    // the last segment starting at or before i (empty segments share the
    // start of the next one, so this is the segment that holds row i)
    int lo = 0, hi = nseg;  // invariant: s_src[lo] <= i < s_src[hi]
    while (hi - lo > 1) {
      const int mid = (lo + hi) >> 1;
      if (s_src[mid] <= i) lo = mid;
      else hi = mid;
    }
    const int j = s_dst[lo] + (i - s_src[lo]);
    const int src_row = dir == 0 ? i : j, dst_row = dir == 0 ? j : i;
    const uint4* a = reinterpret_cast<const uint4*>(in + static_cast<size_t>(src_row) * H);
    uint4* b = reinterpret_cast<uint4*>(out + static_cast<size_t>(dst_row) * H);
    for (int v = lane; v < nvec; v += 32) b[v] = a[v];
  }
}

}  // namespace moe
