// Order of the experts by load for the ragged-K reduction kernels (LoRA and
// base-weight gradients): taking the experts with the most rows first lets
// the long per-expert reductions start first and the short ones fill in
// behind them on the persistent CTAs.
#pragma once

#include "ptx.cuh"

namespace moe {

// s_eorder[0..E) = the experts by decreasing row-count bucket
// (floor(log2(rows)); empty experts last), index order inside a bucket.  One
// warp; deterministic (bucket sizes from a histogram, positions from the
// lanes' ranks among equal keys, chunks of 32 experts in index order).
__device__ __forceinline__ void expert_load_order(const int* s_off, int E, int* s_eorder,
                                                  int* s_bcur, int lane) {
  auto bucket = [&](int e) {  // 0 = empty, 1 + floor(log2(rows)) otherwise
    const int n = s_off[e + 1] - s_off[e];
    return n > 0 ? 32 - __clz(n) : 0;
  };
  for (int b = lane; b < 33; b += 32) s_bcur[b] = 0;
  __syncwarp();
  for (int e = lane; e < E; e += 32) atomicAdd(&s_bcur[bucket(e)], 1);
  __syncwarp();
  if (lane == 0) {  // exclusive prefix, largest bucket first
    int acc = 0;
    for (int b = 32; b >= 0; --b) {
      const int c = s_bcur[b];
      s_bcur[b] = acc;
      acc += c;
    }
  }
  __syncwarp();
  for (int c0 = 0; c0 < E; c0 += 32) {
    const int e = c0 + lane;
    const int key = e < E ? bucket(e) : 33;
    const unsigned peers = __match_any_sync(0xffffffffu, key);
    const int rank = __popc(peers & ((1u << lane) - 1u));
    if (e < E) s_eorder[s_bcur[key] + rank] = e;
    __syncwarp();
    if (e < E && rank == 0) s_bcur[key] += __popc(peers);
    __syncwarp();
  }
}

}  // namespace moe
