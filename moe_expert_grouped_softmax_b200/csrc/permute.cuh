// a2 / a6: gather tokens into expert order (optionally scaled by the routing
// weight, optionally with the routing-weight gradient), and a5 / a10: the
// weighted combine back to token order.  Both are HBM-bound copies: one warp
// per token, 16-byte vector accesses, several loads in flight per lane.
#pragma once

#include "ptx.cuh"

namespace moe {

__device__ __forceinline__ uint4 ld_nc_v4(const void* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

__device__ __forceinline__ uint4 ld_v4(const void* p) {
  uint4 v;
  asm volatile("ld.global.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

__device__ __forceinline__ void st_v4(void* p, uint4 v) {
  asm volatile("st.global.v4.u32 [%0], {%1,%2,%3,%4};" ::"l"(p), "r"(v.x),
               "r"(v.y), "r"(v.z), "r"(v.w)
               : "memory");
}

__device__ __forceinline__ uint32_t scale2(uint32_t v, float c) {
  return pack_bf16x2(bf16_lo(v) * c, bf16_hi(v) * c);
}

__device__ __forceinline__ float dot8(uint4 a, uint4 b) {
  float s = bf16_lo(a.x) * bf16_lo(b.x);
  s = fmaf(bf16_hi(a.x), bf16_hi(b.x), s);
  s = fmaf(bf16_lo(a.y), bf16_lo(b.y), s);
  s = fmaf(bf16_hi(a.y), bf16_hi(b.y), s);
  s = fmaf(bf16_lo(a.z), bf16_lo(b.z), s);
  s = fmaf(bf16_hi(a.z), bf16_hi(b.z), s);
  s = fmaf(bf16_lo(a.w), bf16_lo(b.w), s);
  s = fmaf(bf16_hi(a.w), bf16_hi(b.w), s);
  return s;
}

constexpr int kCopyUnroll = 4;

// The gather's register budget allows 3 resident CTAs of 256 threads per SM
// (measured against 2, the allocation without a minimum: Qwen3-30B-A3B
// shape 108 -> 106 us per launch, gpt-oss-20b shape unchanged; 4 spills).
#ifndef MOE_PERMUTE_MINB
#define MOE_PERMUTE_MINB 3
#endif

// Xp[dest[t,j]] = (scale ? scale[t,j] : 1) * X[t].  The unit of work is a
// part of a row (one of `parts` consecutive vector ranges of the row; the
// host picks parts so that every warp gets several units, which evens out
// the last round of a launch); one warp per unit, grid-stride: the part is
// read once into registers (VPL 16-byte vectors per lane in flight per pass,
// permute_vpl) and written to all k destinations.
template <int kRowVec>
__global__ void __launch_bounds__(256, MOE_PERMUTE_MINB)
    permute_rows_kernel(const __nv_bfloat16* __restrict__ X,
                        const int32_t* __restrict__ dest,
                        const float* __restrict__ scale, int T, int H, int k,
                        __nv_bfloat16* __restrict__ Xp, int parts) {
  griddep_sync();  // before any global memory access
  const int lane = threadIdx.x & 31;
  const int warps = (gridDim.x * blockDim.x) >> 5;
  const int nvec = H >> 3;
  const int nvp = (nvec + parts - 1) / parts;
  const int R = T * k;
  const long long units = static_cast<long long>(T) * parts;
  for (long long q = (blockIdx.x * blockDim.x + threadIdx.x) >> 5; q < units; q += warps) {
    const int t = static_cast<int>(q / parts);
    const int part = static_cast<int>(q - static_cast<long long>(t) * parts);
    const int v_lo = part * nvp, v_hi = min(nvec, v_lo + nvp);
    const char* xrow = reinterpret_cast<const char*>(X + static_cast<size_t>(t) * H);
    for (int v0 = v_lo + lane; v0 < v_hi; v0 += 32 * kRowVec) {
      uint4 x[kRowVec];
#pragma unroll
      for (int u = 0; u < kRowVec; ++u) {
        const int v = v0 + 32 * u;
        if (v < v_hi) x[u] = ld_nc_v4(xrow + 16 * static_cast<size_t>(v));
      }
      for (int j = 0; j < k; ++j) {
        const int d = dest[static_cast<size_t>(t) * k + j];
        if (d < 0 || d >= R) {
          if (lane == 0 && v0 == v_lo) set_status(5);
          continue;
        }
        char* orow = reinterpret_cast<char*>(Xp + static_cast<size_t>(d) * H);
        const float c = scale ? scale[static_cast<size_t>(t) * k + j] : 1.f;
#pragma unroll
        for (int u = 0; u < kRowVec; ++u) {
          const int v = v0 + 32 * u;
          if (v < v_hi) {
            uint4 y = x[u];
            if (scale) {
              y.x = scale2(y.x, c);
              y.y = scale2(y.y, c);
              y.z = scale2(y.z, c);
              y.w = scale2(y.w, c);
            }
            st_v4(orow + 16 * static_cast<size_t>(v), y);
          }
        }
      }
    }
  }
}

// Vectors per lane per pass of permute_rows_kernel for row parts of nvp
// 16-byte vectors: enough for a whole part in one pass up to 512 vectors
// (H = 4096), one of 4, 6, 8, 12, 16 (fewest idle lane slots: 360 vectors,
// H = 2880, take 12, one pass with 94% of the slots used, where 8 took two
// passes at 70%; half of that row takes 6).
inline int permute_vpl(int nvp) {
  const int per_lane = (nvp + 31) / 32;
  return per_lane <= 4 ? 4 : per_lane <= 6 ? 6 : per_lane <= 8 ? 8 : per_lane <= 12 ? 12 : 16;
}

#ifndef MOE_ROW_PARTS_MAX
#define MOE_ROW_PARTS_MAX 2
#endif
#ifndef MOE_ROW_PART_MIN
#define MOE_ROW_PART_MIN 128
#endif
#ifndef MOE_ROW_UNITS_PER_WARP
#define MOE_ROW_UNITS_PER_WARP 4
#endif
// Parts per row for the gather: enough that each of the `warps` resident
// warps gets about four units (T tokens in all), at most MOE_ROW_PARTS_MAX,
// and no part under 128 vectors (measured, gpt-oss-20b shape: 2 parts, 52 ->
// 48 us per launch; the last round of whole rows left SMs idle).
inline int row_parts(int T, int nvec, int warps) {
  int p = 1;
  while (p < MOE_ROW_PARTS_MAX &&
         static_cast<long long>(T) * p < static_cast<long long>(MOE_ROW_UNITS_PER_WARP) * warps &&
         nvec / (p + 1) >= MOE_ROW_PART_MIN)
    ++p;
  return p;
}

// The same sums as permute_kernel (below) for rows of at most 32 * kRowVec
// vectors: the row is read once into registers (kRowVec vectors per lane),
// then for each slot j its Zp row is loaded (all of the lane's vectors in
// flight together), dotted with the row in the lane's vector order, the
// scaled row stored, and the lane sums reduced across the warp in the same
// order as permute_kernel (so dw is the same bits).  k <= 32: lane j holds
// slot j's destination and weight.
template <int kRowVec>
__global__ void __launch_bounds__(256, 2)
    permute_dw_rows_kernel(const __nv_bfloat16* __restrict__ X,
                           const int32_t* __restrict__ dest,
                           const float* __restrict__ scale, int T, int H, int k,
                           __nv_bfloat16* __restrict__ Xp,
                           const __nv_bfloat16* __restrict__ Zp,
                           float* __restrict__ dw) {
  griddep_sync();  // before any global memory access
  const int lane = threadIdx.x & 31;
  const int warps = (gridDim.x * blockDim.x) >> 5;
  const int nvec = H >> 3;
  const int R = T * k;
  for (int t = (blockIdx.x * blockDim.x + threadIdx.x) >> 5; t < T; t += warps) {
    const char* xrow = reinterpret_cast<const char*>(X + static_cast<size_t>(t) * H);
    int my_d = -1;
    float my_c = 1.f;
    if (lane < k) {
      my_d = dest[static_cast<size_t>(t) * k + lane];
      if (scale) my_c = scale[static_cast<size_t>(t) * k + lane];
      if (my_d < 0 || my_d >= R) {
        set_status(5);
        my_d = -1;
      }
    }
    uint4 x[kRowVec];
#pragma unroll
    for (int u = 0; u < kRowVec; ++u) {
      const int v = lane + 32 * u;
      if (v < nvec) x[u] = ld_v4(xrow + 16 * static_cast<size_t>(v));
    }
    for (int j = 0; j < k; ++j) {
      const int d = __shfl_sync(0xffffffffu, my_d, j);
      const float c = __shfl_sync(0xffffffffu, my_c, j);
      if (d < 0) continue;  // recorded above; the same on every lane
      char* orow = reinterpret_cast<char*>(Xp + static_cast<size_t>(d) * H);
      const char* zrow = reinterpret_cast<const char*>(Zp + static_cast<size_t>(d) * H);
      uint4 z[kRowVec];
#pragma unroll
      for (int u = 0; u < kRowVec; ++u) {
        const int v = lane + 32 * u;
        if (v < nvec) z[u] = ld_nc_v4(zrow + 16 * static_cast<size_t>(v));
      }
      float acc = 0.f;
#pragma unroll
      for (int u = 0; u < kRowVec; ++u) {
        const int v = lane + 32 * u;
        if (v < nvec) {
          acc += dot8(x[u], z[u]);
          uint4 y = x[u];
          y.x = scale2(y.x, c);
          y.y = scale2(y.y, c);
          y.z = scale2(y.z, c);
          y.w = scale2(y.w, c);
          st_v4(orow + 16 * static_cast<size_t>(v), y);
        }
      }
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
      if (lane == 0) dw[static_cast<size_t>(t) * k + j] = acc;
    }
  }
}

// Same with the routing-weight gradient dw[t,j] = <X[t], Zp[dest[t,j]]>.
// One warp per token, grid-stride over tokens.
__global__ void __launch_bounds__(256)
    permute_kernel(const __nv_bfloat16* __restrict__ X,
                   const int32_t* __restrict__ dest,
                   const float* __restrict__ scale, int T, int H, int k,
                   __nv_bfloat16* __restrict__ Xp,
                   const __nv_bfloat16* __restrict__ Zp,
                   float* __restrict__ dw) {
  griddep_sync();  // before any global memory access
  const int lane = threadIdx.x & 31;
  const int warps = (gridDim.x * blockDim.x) >> 5;
  const int nvec = H >> 3;
  const int R = T * k;
  for (int t = (blockIdx.x * blockDim.x + threadIdx.x) >> 5; t < T; t += warps) {
    const char* xrow = reinterpret_cast<const char*>(X + static_cast<size_t>(t) * H);
    for (int j = 0; j < k; ++j) {
      const int d = dest[static_cast<size_t>(t) * k + j];
      if (d < 0 || d >= R) {
        if (lane == 0) set_status(5);
        continue;
      }
      const float c = scale ? scale[static_cast<size_t>(t) * k + j] : 1.f;
      char* orow = reinterpret_cast<char*>(Xp + static_cast<size_t>(d) * H);
      const char* zrow =
          Zp ? reinterpret_cast<const char*>(Zp + static_cast<size_t>(d) * H)
             : nullptr;
      float acc = 0.f;
      for (int v0 = lane; v0 < nvec; v0 += 32 * kCopyUnroll) {
        uint4 x[kCopyUnroll];
#pragma unroll
        for (int u = 0; u < kCopyUnroll; ++u) {
          const int v = v0 + 32 * u;
          if (v < nvec) x[u] = ld_v4(xrow + 16 * static_cast<size_t>(v));
        }
        if (dw) {
#pragma unroll
          for (int u = 0; u < kCopyUnroll; ++u) {
            const int v = v0 + 32 * u;
            if (v < nvec) acc += dot8(x[u], ld_nc_v4(zrow + 16 * static_cast<size_t>(v)));
          }
        }
#pragma unroll
        for (int u = 0; u < kCopyUnroll; ++u) {
          const int v = v0 + 32 * u;
          if (v < nvec) {
            uint4 y = x[u];
            if (scale) {
              y.x = scale2(y.x, c);
              y.y = scale2(y.y, c);
              y.z = scale2(y.z, c);
              y.w = scale2(y.w, c);
            }
            st_v4(orow + 16 * static_cast<size_t>(v), y);
          }
        }
      }
      if (dw) {
#pragma unroll
        for (int off = 16; off > 0; off >>= 1)
          acc += __shfl_xor_sync(0xffffffffu, acc, off);
        if (lane == 0) dw[static_cast<size_t>(t) * k + j] = acc;
      }
    }
  }
}

// Y[t] = sum_j (w ? w[t,j] : 1) * Yp[dest[t,j]], fp32 in j order -> bf16.
// With a trained router (Wr != nullptr) the router's part of dX is added
// before the one rounding: + sum_j g[t,j] * Wr[idx[t,j]] (Wr [E, H] bf16).
// One warp per token (splitting rows into parts as the gather does
// measured no faster here).  The token's destination rows and weights are
// read once (lane j holds slot j, broadcast by shuffle) and two source rows'
// kCombVec vectors per lane are loaded before either is accumulated (the sum
// stays in j order).  Measured against one row at a time with dest
// re-read per row: Qwen3-30B-A3B shape (k = 8) 117 -> 103 us, gpt-oss-20b
// shape unchanged.  kCombVec 16-byte vectors per lane and source row per
// pass, kMinB resident CTAs per SM (see combine_vec).
template <int kCombVec, int kMinB>
__global__ void __launch_bounds__(256, kMinB)
    unpermute_kernel(const __nv_bfloat16* __restrict__ Yp,
                     const int32_t* __restrict__ dest,
                     const float* __restrict__ w, int T, int H, int k,
                     __nv_bfloat16* __restrict__ Y,
                     const __nv_bfloat16* __restrict__ Wr = nullptr,
                     const int32_t* __restrict__ idx = nullptr,
                     const float* __restrict__ g = nullptr, int E = 0) {
  griddep_sync();  // before any global memory access
  const int lane = threadIdx.x & 31;
  const int warps = (gridDim.x * blockDim.x) >> 5;
  const int nvec = H >> 3;
  const int R = T * k;
  auto fma8 = [](float* a, float c, uint4 z) {
    a[0] = fmaf(c, bf16_lo(z.x), a[0]);
    a[1] = fmaf(c, bf16_hi(z.x), a[1]);
    a[2] = fmaf(c, bf16_lo(z.y), a[2]);
    a[3] = fmaf(c, bf16_hi(z.y), a[3]);
    a[4] = fmaf(c, bf16_lo(z.z), a[4]);
    a[5] = fmaf(c, bf16_hi(z.z), a[5]);
    a[6] = fmaf(c, bf16_lo(z.w), a[6]);
    a[7] = fmaf(c, bf16_hi(z.w), a[7]);
  };
  const int v_lo = 0, v_hi = nvec;
  for (int t = (blockIdx.x * blockDim.x + threadIdx.x) >> 5; t < T; t += warps) {
    char* yrow = reinterpret_cast<char*>(Y + static_cast<size_t>(t) * H);
    // slots j0 .. j0 + 31 of the token on lanes 0 .. 31 (k <= 32 in one go)
    int my_d = -1;
    float my_c = 1.f;
    if (lane < k) {
      my_d = dest[static_cast<size_t>(t) * k + lane];
      if (w) my_c = w[static_cast<size_t>(t) * k + lane];
      if (my_d < 0 || my_d >= R) {
        set_status(5);
        my_d = -1;
      }
    }
    // the pass loop's trip count is the same on every lane (the shuffles
    // below need the whole warp); vectors past v_hi are masked
    for (int base = v_lo; base < v_hi; base += 32 * kCombVec) {
      const int v0 = base + lane;
      float acc[kCombVec][8];
#pragma unroll
      for (int u = 0; u < kCombVec; ++u)
#pragma unroll
        for (int i = 0; i < 8; ++i) acc[u][i] = 0.f;
      for (int j0 = 0; j0 < k; j0 += 32) {
        int dj = my_d;
        float cj = my_c;
        if (j0 > 0) {  // slots past 32 (k > 32): reload for this group
          dj = -1;
          cj = 1.f;
          if (j0 + lane < k) {
            dj = dest[static_cast<size_t>(t) * k + j0 + lane];
            if (w) cj = w[static_cast<size_t>(t) * k + j0 + lane];
            if (dj < 0 || dj >= R) {
              if (base == v_lo) set_status(5);
              dj = -1;
            }
          }
        }
        const int nj = min(32, k - j0);
        for (int jj = 0; jj < nj; jj += 2) {
          const int da = __shfl_sync(0xffffffffu, dj, jj);
          const float ca = __shfl_sync(0xffffffffu, cj, jj);
          const int db = __shfl_sync(0xffffffffu, dj, jj + 1 < nj ? jj + 1 : jj);
          const float cb = __shfl_sync(0xffffffffu, cj, jj + 1 < nj ? jj + 1 : jj);
          const bool has_b = jj + 1 < nj;
          uint4 za[kCombVec], zb[kCombVec];
#pragma unroll
          for (int u = 0; u < kCombVec; ++u) {
            const int v = v0 + 32 * u;
            za[u] = zb[u] = make_uint4(0, 0, 0, 0);
            if (v < v_hi && da >= 0)
              za[u] = ld_nc_v4(reinterpret_cast<const char*>(Yp + static_cast<size_t>(da) * H) +
                              16 * static_cast<size_t>(v));
            if (v < v_hi && has_b && db >= 0)
              zb[u] = ld_nc_v4(reinterpret_cast<const char*>(Yp + static_cast<size_t>(db) * H) +
                              16 * static_cast<size_t>(v));
          }
#pragma unroll
          for (int u = 0; u < kCombVec; ++u) {
            if (da >= 0) fma8(acc[u], ca, za[u]);
            if (has_b && db >= 0) fma8(acc[u], cb, zb[u]);
          }
        }
      }
      if (Wr != nullptr) {
        for (int j = 0; j < k; ++j) {
          const int e = idx[static_cast<size_t>(t) * k + j];
          if (e < 0 || e >= E) {
            if (lane == 0) set_status(5);
            continue;
          }
          const float c = g[static_cast<size_t>(t) * k + j];
          const char* wrow = reinterpret_cast<const char*>(Wr + static_cast<size_t>(e) * H);
#pragma unroll
          for (int u = 0; u < kCombVec; ++u) {
            const int v = v0 + 32 * u;
            if (v < v_hi)
              fma8(acc[u], c, *reinterpret_cast<const uint4*>(wrow + 16 * static_cast<size_t>(v)));
          }
        }
      }
#pragma unroll
      for (int u = 0; u < kCombVec; ++u) {
        const int v = v0 + 32 * u;
        if (v < v_hi) {
          uint4 o;
          o.x = pack_bf16x2(acc[u][0], acc[u][1]);
          o.y = pack_bf16x2(acc[u][2], acc[u][3]);
          o.z = pack_bf16x2(acc[u][4], acc[u][5]);
          o.w = pack_bf16x2(acc[u][6], acc[u][7]);
          st_v4(yrow + 16 * static_cast<size_t>(v), o);
        }
      }
    }
  }
}

// The backward's operand copies of the LoRA factors in one launch: a list
// of jobs, each either a zero-padding copy (out[row][0:width] = (in[row][0:r],
// zeros); width a multiple of 8, >= r) or a batched transpose
// ([nb, P, Q] -> [nb, Q, P]).  Each CTA (256 threads) works for one job.
struct FactorJob {
  const __nv_bfloat16* in;
  __nv_bfloat16* out;
  int kind;          // 0: pad, 1: transpose
  int blocks;        // CTAs given to this job
  long long rows;    // pad
  int r, width;      // pad
  int nb, P, Q;      // transpose
};
constexpr int kMaxFactorJobs = 4;
struct FactorJobs {
  FactorJob job[kMaxFactorJobs];
  int n;
};

__global__ void __launch_bounds__(256) factor_prep_kernel(const FactorJobs jobs) {
  griddep_sync();  // before any global memory access
  int b = blockIdx.x, ji = 0;
  while (ji < jobs.n && b >= jobs.job[ji].blocks) {
    b -= jobs.job[ji].blocks;
    ++ji;
  }
  if (ji >= jobs.n) return;
  const FactorJob& J = jobs.job[ji];
  if (J.kind == 0) {
    const int chunks = J.width / 8;  // 16-byte chunks per output row
    const long long n = J.rows * chunks;
    for (long long i = b * 256ll + threadIdx.x; i < n; i += static_cast<long long>(J.blocks) * 256) {
      const long long row = i / chunks;
      const int c8 = static_cast<int>(i - row * chunks) * 8;
      uint4 v = make_uint4(0, 0, 0, 0);
      if (c8 < J.r) v = *reinterpret_cast<const uint4*>(J.in + row * J.r + c8);
      *reinterpret_cast<uint4*>(J.out + row * J.width + c8) = v;
    }
  } else {
    __shared__ __nv_bfloat16 tile[32][33];
    const int qt = (J.Q + 31) / 32, pt = (J.P + 31) / 32;
    const int q0 = (b % qt) * 32, p0 = ((b / qt) % pt) * 32;
    const size_t bb = static_cast<size_t>(b / (qt * pt));
    const __nv_bfloat16* src = J.in + bb * static_cast<size_t>(J.P) * J.Q;
    __nv_bfloat16* dst = J.out + bb * static_cast<size_t>(J.P) * J.Q;
    const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;
    for (int i = ty; i < 32; i += 8) {
      const int p = p0 + i, q = q0 + tx;
      if (p < J.P && q < J.Q) tile[i][tx] = src[static_cast<size_t>(p) * J.Q + q];
    }
    __syncthreads();
    for (int i = ty; i < 32; i += 8) {
      const int q = q0 + i, p = p0 + tx;
      if (p < J.P && q < J.Q) dst[static_cast<size_t>(q) * J.P + p] = tile[tx][i];
    }
  }
}

// Vectors per lane per pass of the combine for rows of nvec 16-byte vectors:
// 4 (3 CTAs per SM) when the row is whole 128-vector passes, else 2 (4 CTAs
// per SM: more rows in flight for the ragged last pass).  Measured, per
// launch: H = 2880, 51 us with (4, 2 CTAs) -> 45 us with (2, 4); H = 2048,
// 103 -> 98 us with (4, 3).
inline int combine_vec(int nvec) { return nvec % 128 == 0 ? 4 : 2; }

}  // namespace moe
