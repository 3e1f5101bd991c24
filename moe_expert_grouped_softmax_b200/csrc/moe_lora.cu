// Host side of the C ABI declared in include/moe_lora.h: argument checks,
// tensor-map encoding, tile-shape choice and kernel launches.  Every kernel
// of the block is compiled into this one translation unit (so they share the
// device status word).
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <utility>
#include <atomic>
#include <cstdint>
#include <cstring>
#include <mutex>

#include "moe_lora.h"
#include "ptx.cuh"
#include "route.cuh"
#include "permute.cuh"
#include "gemm.cuh"
#include "gemm_pair.cuh"
#include "lora_grad.cuh"
#include "base_grad.cuh"
#include "base_grad_pair.cuh"
#include "router.cuh"
#include "rank_down.cuh"
#include "ep.cuh"

using namespace moe;

// Scratch of moe_route_topk_noalloc: a fixed array in the library's own device
// memory, so that entry point never needs a caller-provided workspace and never
// allocates.  Every GPU that loads the library holds these bytes until the
// process exits.  In host code `g_route_scratch` is only a host-side stand-in
// for the symbol, never a device address: its device address is looked up
// with cudaGetSymbolAddress, with the caller's device current, on every call
// (see route_scratch_on_current_device).
constexpr size_t kRouteScratchBytes = size_t(4) << 20;  // 4 MiB
static __device__ __align__(256) unsigned char g_route_scratch[kRouteScratchBytes];

namespace {

// Device address of g_route_scratch in the current device's context.  Looked
// up on every call rather than cached: the lookup is a host-side query that
// allocates nothing, and a cached address would go stale after
// cudaDeviceReset (the module is loaded again, possibly elsewhere) or belong
// to another context of the same device.
moe_status_t route_scratch_on_current_device(void** out) {
  void* p = nullptr;
  if (cudaGetSymbolAddress(&p, g_route_scratch) != cudaSuccess || p == nullptr)
    return MOE_ERR_CUDA;
  *out = p;
  return MOE_OK;
}

uint64_t g_wait_limit_ns = 1000000000ull;  // one second per bounded wait
std::atomic<unsigned long long> g_launches{0};  // kernels launched by the library
inline void count_launch() { g_launches.fetch_add(1, std::memory_order_relaxed); }
int g_stall_test = 0;                      // testing hook, see moe_test_inject_stall
int g_cta_pairs = -1;                      // grouped GEMMs on CTA pairs: <0 auto
// Automatic choice (measured): a GEMM runs on CTA pairs when the mean rows
// per expert fill at least one 256-row tile (an expert's ragged last tile
// with at most 128 rows runs as a half tile) and K has at least 12 k-steps.
// Pairs against single CTAs, whole step: 256 rows per expert, K = 2048 to
// 7168: -26%; 1024 rows per expert, K = 768 (down forward): -28% on that
// GEMM.
constexpr int kPairMinRowsPerExpert = 256;
constexpr int kPairMinK = 768;
bool use_pairs(int R, int E, int K) {
  if (g_cta_pairs >= 0) return g_cta_pairs > 0;
  return static_cast<int64_t>(R) >= static_cast<int64_t>(kPairMinRowsPerExpert) * E &&
         K >= kPairMinK;
}

// Launches a kernel on `st`; with MOE_PDL the launch allows programmatic
// dependent launch (the kernel's griddep_sync waits for the preceding kernel
// of the stream before touching global memory, and lets the next one launch
// while this one's CTAs finish).  Errors are left for launch_status().
template <typename... KArgs, typename... Args>
void launch_k(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
              Args&&... args) {
#if MOE_PDL
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
#else
  kern<<<grid, block, smem, st>>>(std::forward<Args>(args)...);
#endif
}

// ------------------------------------------------ optional per-kernel timing
// When enabled, each launch site of a kernel kind records a CUDA event before
// and after its launch on the caller's stream (up to kProfCap pairs per kind).
constexpr int kProfCap = 512;
bool g_prof_on = false;
cudaEvent_t g_prof_ev[MOE_PROF_KINDS][kProfCap][2];
int g_prof_n[MOE_PROF_KINDS];
bool g_prof_created = false;

// Under stream capture the records become event-record nodes of the graph
// (re-recorded by every replay), so that a replayed step can be timed per
// kernel without host launch gaps between the launches.
void prof_record(int kind, int which, cudaStream_t st) {
  if (!g_prof_on || kind < 0 || kind >= MOE_PROF_KINDS) return;
  const int n = g_prof_n[kind];
  if (n >= kProfCap) return;
  cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
  if (cudaStreamIsCapturing(st, &cap) == cudaSuccess && cap == cudaStreamCaptureStatusActive)
    cudaEventRecordWithFlags(g_prof_ev[kind][n][which], st, cudaEventRecordExternal);
  else
    cudaEventRecord(g_prof_ev[kind][n][which], st);
  if (which == 1) g_prof_n[kind] = n + 1;
}

struct ProfScope {
  int kind;
  cudaStream_t st;
  ProfScope(int k, cudaStream_t s) : kind(k), st(s) { prof_record(kind, 0, st); }
  ~ProfScope() { prof_record(kind, 1, st); }
};

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t,
                                  void*, const cuuint64_t*, const cuuint64_t*,
                                  const cuuint32_t*, const cuuint32_t*,
                                  CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion,
                                  CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000,
                                         cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

int num_sms() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 0;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    return 0;
  return n;
}

// 2-D bf16 tensor map: `inner` contiguous elements per row, `outer` rows,
// row pitch `pitch_bytes`; box of box_inner x box_outer elements.
bool tmap_2d(CUtensorMap* m, const void* base, uint64_t inner, uint64_t outer,
             uint64_t pitch_bytes, uint32_t box_inner, uint32_t box_outer,
             CUtensorMapSwizzle swz) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  if ((reinterpret_cast<uintptr_t>(base) & 15u) || (pitch_bytes & 15u)) return false;
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {pitch_bytes};
  cuuint32_t box[2] = {box_inner, box_outer};
  cuuint32_t estr[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims,
            strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, swz,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

CUtensorMapSwizzle lora_swizzle(int r) {
  return r == 16 ? CU_TENSOR_MAP_SWIZZLE_32B
                 : (r == 32 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_128B);
}

inline size_t align256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

// swizzle of the single-CTA kernel's K-major operand boxes (kGemmBK wide)
constexpr CUtensorMapSwizzle kKmajSwz =
    kGemmBK == 64 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B;
inline int ld_rank(int R) { return (R + 63) & ~63; }  // row pitch of [r, R] parts

moe_status_t launch_status() {
  const cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

bool shape_ok(int E, int H, int I, int r) {
  if (E < 1 || E > 512) return false;
  if (H < 64 || I < 64 || (H % 16) || (I % 16)) return false;
  if (!(r == 16 || r == 32 || r == 64)) return false;
  return true;
}

// Tile width along N.  Forward (K-major B): 256 - r, 192 or 128; backward
// (MN-major B, 64-column atoms): 192 or 128.  Picks the smallest estimated
// cost tiles * (BN + r + 48), where 48 stands for the per-tile fixed work.
int pick_bn(int n_cols, bool swiglu, int r, bool backward) {
  const int fwd_c[3] = {256 - r, 192, 128};
  const int bwd_c[2] = {192, 128};
  const int* c = backward ? bwd_c : fwd_c;
  const int nc = backward ? 2 : 3;
  int best = 128;
  double best_cost = 1e300;
  for (int i = 0; i < nc; ++i) {
    const int bn = c[i];
    if (bn + r > 256) continue;
    const int w = swiglu ? bn / 2 : bn;
    const double tiles = (n_cols + w - 1) / w;
    const double cost = tiles * (bn + r + 48);
    if (cost < best_cost) {
      best_cost = cost;
      best = bn;
    }
  }
  return best;
}

template <int MODE, int BN, int RK>
moe_status_t launch_gemm_t(const CUtensorMap& a, const CUtensorMap& b,
                           const CUtensorMap& la, const CUtensorMap& lb,
                           const GemmArgs& args, cudaStream_t st) {
  using C = GemmCfg<MODE, BN, RK>;
  auto kern = grouped_lora_gemm_kernel<MODE, BN, RK>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           C::SMEM_BYTES) != cudaSuccess)
    return MOE_ERR_CUDA;
  const long long max_tiles =
      (static_cast<long long>(args.R) / 128 + args.E) * args.n_tiles;
  const int grid = static_cast<int>(std::min<long long>(num_sms(), max_tiles));
  if (grid <= 0) return MOE_ERR_CUDA;
  ProfScope prof(MODE == kGateUpFwd ? MOE_PROF_GATE_UP_FWD
                 : MODE == kDownFwd ? MOE_PROF_DOWN_FWD
                 : MODE == kDownBwd ? MOE_PROF_DOWN_BWD : MOE_PROF_GATE_UP_BWD, st);
  launch_k(kern, grid, gemm_threads(MODE), C::SMEM_BYTES, st, a, b, la, lb, args);
  count_launch();
  return launch_status();
}

template <int MODE>
moe_status_t launch_gemm(int bn, int r, const CUtensorMap& a, const CUtensorMap& b,
                         const CUtensorMap& la, const CUtensorMap& lb,
                         const GemmArgs& args, cudaStream_t st) {
  constexpr bool kFwd = (MODE == kGateUpFwd || MODE == kDownFwd);
  if constexpr (kFwd) {
    if (r == 16 && bn == 240) return launch_gemm_t<MODE, 240, 16>(a, b, la, lb, args, st);
    if (r == 32 && bn == 224) return launch_gemm_t<MODE, 224, 32>(a, b, la, lb, args, st);
  }
  if (r == 16 && bn == 192) return launch_gemm_t<MODE, 192, 16>(a, b, la, lb, args, st);
  if (r == 16 && bn == 128) return launch_gemm_t<MODE, 128, 16>(a, b, la, lb, args, st);
  if (r == 32 && bn == 192) return launch_gemm_t<MODE, 192, 32>(a, b, la, lb, args, st);
  if (r == 32 && bn == 128) return launch_gemm_t<MODE, 128, 32>(a, b, la, lb, args, st);
  if (r == 64 && bn == 192) return launch_gemm_t<MODE, 192, 64>(a, b, la, lb, args, st);
  if (r == 64 && bn == 128) return launch_gemm_t<MODE, 128, 64>(a, b, la, lb, args, st);
  return MOE_ERR_UNSUPPORTED;
}

// Grouped GEMM on CTA pairs (256 x 256 tiles, weight-only B operand).
// A: [R, K] activations; W: the base weight as [E * b_rows, K] (forward) or
// read in place as [E * b_rows, N] (backward); XA: the s-scaled rank-r
// product [R, r] from the rank pass; LB: the up factor as [E * lb_rows, r].
template <int MODE, int RK>
moe_status_t launch_pair_t(const void* A, const void* W, const void* XA, const void* LB,
                           const GemmArgs& args, cudaStream_t st) {
  using C = PairCfg<MODE, RK>;
  const uint64_t K = static_cast<uint64_t>(args.K);
  const uint64_t EU = static_cast<uint64_t>(args.E);
  CUtensorMap ta, tw, txa, tlb;
  bool ok = tmap_2d(&ta, A, K, args.R, K * 2, 64, 128, CU_TENSOR_MAP_SWIZZLE_128B);
  if constexpr (C::kBMN) {
    // W [E * K, N] in place, 64-column x 64-row boxes (128-byte swizzle)
    const uint64_t N = static_cast<uint64_t>(args.N);
    ok = ok && tmap_2d(&tw, W, N, EU * args.b_rows, N * 2, 64, 64, CU_TENSOR_MAP_SWIZZLE_128B);
  } else {
    // K-major: gate_up fwd loads 64-row gate / up blocks, down fwd the
    // tile's Nt / 2 rows per CTA
    const int wbox = C::kSwiGLU ? C::W_BOX_ROWS : args.tile_n / 2;
    ok = ok && tmap_2d(&tw, W, K, EU * args.b_rows, K * 2, 64, wbox,
                       CU_TENSOR_MAP_SWIZZLE_128B);
  }
  ok = ok && tmap_2d(&txa, XA, RK, args.R, RK * 2ull, RK, C::BM, lora_swizzle(RK));
  if constexpr (C::kBMN) {
    // the up factor A [E, r, N] in place: [E * r, N], 64-column x r-row boxes
    const uint64_t N = static_cast<uint64_t>(args.N);
    ok = ok && tmap_2d(&tlb, LB, N, EU * RK, N * 2, 64, RK, CU_TENSOR_MAP_SWIZZLE_128B);
  } else {
    ok = ok && tmap_2d(&tlb, LB, RK, EU * args.lb_rows, RK * 2ull, RK, C::LB_BOX_ROWS,
                       lora_swizzle(RK));
  }
  // outputs, stored by the epilogue in boxes of 32 rows x SBW columns:
  // gate_up fwd h [R, I], saved gate = Z1 columns [0, I) and saved up = Z1
  // columns [I, 2I) (two views of Z1, so a box never spills from one half
  // into the other); down bwd dZ1 = [dg | du] likewise; otherwise [R, N]
  CUtensorMap to, to2, to3;
  const CUtensorMapSwizzle osw =
      C::SBW == 16 ? CU_TENSOR_MAP_SWIZZLE_32B : CU_TENSOR_MAP_SWIZZLE_64B;
  const uint64_t R = static_cast<uint64_t>(args.R), N = static_cast<uint64_t>(args.N);
  ok = ok && tmap_2d(&to, args.out, N, R, args.ld_out * 2ull, C::SBW, 32, osw);
  to2 = to3 = to;
  if constexpr (MODE == kGateUpFwd) {
    ok = ok && tmap_2d(&to2, args.out2, N, R, args.ld_out2 * 2ull, C::SBW, 32, osw);
    ok = ok && tmap_2d(&to3, args.out2 + args.I, N, R, args.ld_out2 * 2ull, C::SBW, 32, osw);
  } else if constexpr (MODE == kDownBwd) {
    ok = ok && tmap_2d(&to3, args.out + args.I, N, R, args.ld_out * 2ull, C::SBW, 32, osw);
  }
  if (!ok) return MOE_ERR_CUDA;
  auto kern = grouped_lora_gemm_pair_kernel<MODE, RK>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           C::SMEM_BYTES) != cudaSuccess)
    return MOE_ERR_CUDA;
  const long long max_pairs =
      (static_cast<long long>(args.R) / 256 + args.E) * args.n_tiles;
  const int pairs = static_cast<int>(std::min<long long>(num_sms() / 2, max_pairs));
  if (pairs <= 0) return MOE_ERR_CUDA;
  ProfScope prof(MODE == kGateUpFwd   ? MOE_PROF_GATE_UP_FWD
                 : MODE == kDownFwd   ? MOE_PROF_DOWN_FWD
                 : MODE == kDownBwd   ? MOE_PROF_DOWN_BWD
                                      : MOE_PROF_GATE_UP_BWD,
                 st);
  launch_k(kern, 2 * pairs, C::THREADS, C::SMEM_BYTES, st, ta, tw, txa, tlb, to, to2, to3,
           args);
  count_launch();
  return launch_status();
}

// Columns per CTA-pair tile (the MMA's N) for N output columns.  K-major
// weight (down forward): the narrowest multiple of 16 that covers N in as
// many tiles as 256 would (2880 -> 12 tiles of 240; 2048 -> 256).  MN-major
// weight (backward): whole 64-column atoms per CTA, 128 or 256 (measured:
// 240 -- 120-column halves -- slows both backward GEMMs by about 20%).
// Gate_up forward always uses 256 (128 gate + 128 up columns per tile).
constexpr int pair_tile_n(int N, bool mn_major) {
  if (mn_major) return N <= 128 ? 128 : 256;
  const int tiles = (N + 255) / 256;
  return 16 * ((N + 16 * tiles - 1) / (16 * tiles));
}

template <int MODE>
moe_status_t launch_pair(int r, const void* A, const void* W, const void* XA,
                         const void* LB, const GemmArgs& args, cudaStream_t st) {
  if (r == 16) return launch_pair_t<MODE, 16>(A, W, XA, LB, args, st);
  if (r == 32) return launch_pair_t<MODE, 32>(A, W, XA, LB, args, st);
  if (r == 64) return launch_pair_t<MODE, 64>(A, W, XA, LB, args, st);
  return MOE_ERR_UNSUPPORTED;
}

template <int RK>
moe_status_t launch_grad_t(const CUtensorMap* u, const CUtensorMap* v,
                           const GradArgs& args, cudaStream_t st) {
  using C = GradCfg<RK>;
  auto kern = lora_grad_kernel<RK>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           C::SMEM_BYTES) != cudaSuccess)
    return MOE_ERR_CUDA;
  const int grid = std::min(num_sms() * C::CTAS_PER_SM, args.total_tiles);
  if (grid <= 0) return MOE_OK;
  ProfScope prof(MOE_PROF_LORA_GRAD, st);
  launch_k(kern, grid, 192, C::SMEM_BYTES, st, u[0], u[1], u[2], u[3], v[0], v[1], v[2], v[3],
           args);
  count_launch();
  return launch_status();
}

// Saved-activation parts (bytes from the start of `saved`).
constexpr int kSavedParts = 6;
void saved_layout(int R, int H, int I, int r, size_t off[kSavedParts + 1]) {
  (void)H;
  const size_t z1 = static_cast<size_t>(R) * 2 * I * 2;
  const size_t h = static_cast<size_t>(R) * I * 2;
  const size_t xa = static_cast<size_t>(r) * ld_rank(R) * 2;
  const size_t xa_rm = static_cast<size_t>(R) * r * 2;
  off[0] = 0;                          // Z1 [R, 2I]
  off[1] = off[0] + align256(z1);      // h [R, I]
  off[2] = off[1] + align256(h);       // XA1t [r, ldR]
  off[3] = off[2] + align256(xa);      // HA2t [r, ldR]
  off[4] = off[3] + align256(xa);      // XA1 [R, r]
  off[5] = off[4] + align256(xa_rm);   // HA2 [R, r]
  off[6] = off[5] + align256(xa_rm);
}

// Backward scratch parts.
void bwd_layout(int R, int E, int H, int I, int r, size_t off[10]) {
  const size_t dz1 = static_cast<size_t>(R) * 2 * I * 2;
  const size_t vt = static_cast<size_t>(r) * ld_rank(R) * 2;
  off[0] = 0;                                                  // dZ1 [R, 2I]
  off[1] = off[0] + align256(dz1);                             // dZB2t [r, ldR]
  off[2] = off[1] + align256(vt);                              // dZB1t [r, ldR]
  off[3] = off[2] + align256(vt);                              // B2p [E*H, <= 64]
  off[4] = off[3] + align256(static_cast<size_t>(E) * H * 64 * 2);     // A2t [E, I, r]
  off[5] = off[4] + align256(static_cast<size_t>(E) * I * r * 2);      // B1p [E*2I, <= 64]
  off[6] = off[5] + align256(static_cast<size_t>(E) * 2 * I * 64 * 2);  // A1t [E, H, r]
  off[7] = off[6] + align256(static_cast<size_t>(E) * H * r * 2);     // s dZ2 B2 [R, r]
  off[8] = off[7] + align256(static_cast<size_t>(R) * r * 2);          // s dZ1 B1 [R, r]
  off[9] = off[8] + align256(static_cast<size_t>(R) * r * 2);
}

template <typename T>
T* at(void* base, size_t off) {
  return reinterpret_cast<T*>(static_cast<char*>(base) + off);
}
template <typename T>
const T* at(const void* base, size_t off) {
  return reinterpret_cast<const T*>(static_cast<const char*>(base) + off);
}

// zero the padding columns [R, ldR) of an [r, ldR] bf16 part
moe_status_t zero_rank_padding(void* p, int R, int r, cudaStream_t st) {
  const int ld = ld_rank(R);
  if (ld == R) return MOE_OK;
  const cudaError_t e = cudaMemset2DAsync(static_cast<char*>(p) + static_cast<size_t>(R) * 2,
                                          static_cast<size_t>(ld) * 2, 0,
                                          static_cast<size_t>(ld - R) * 2, r, st);
  return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

// out [rows, 64] = in [rows, r] followed by zero columns (one MN-major
// 64-column atom per K-slice for the backward's fused rank-r operand).
// Jobs of factor_prep_kernel, launched together.
struct FactorPrep {
  FactorJobs jobs{};
  int total = 0;
  void pad(const void* in, void* out, long long rows, int r, int width) {
    FactorJob& J = jobs.job[jobs.n++];
    J.in = static_cast<const __nv_bfloat16*>(in);
    J.out = static_cast<__nv_bfloat16*>(out);
    J.kind = 0;
    J.rows = rows;
    J.r = r;
    J.width = width;
    J.blocks = static_cast<int>(std::min<long long>((rows * (width / 8) + 255) / 256, 148ll * 4));
    total += J.blocks;
  }
  void transpose(const void* in, void* out, int nb, int P, int Q) {
    FactorJob& J = jobs.job[jobs.n++];
    J.in = static_cast<const __nv_bfloat16*>(in);
    J.out = static_cast<__nv_bfloat16*>(out);
    J.kind = 1;
    J.nb = nb;
    J.P = P;
    J.Q = Q;
    J.blocks = ((Q + 31) / 32) * ((P + 31) / 32) * nb;
    total += J.blocks;
  }
  moe_status_t launch(cudaStream_t st) {
    if (total == 0) return MOE_OK;
    ProfScope prof(MOE_PROF_TRANSPOSE, st);
    launch_k(factor_prep_kernel, total, 256, 0, st, jobs);
    count_launch();
    return launch_status();
  }
};

template <int BN>
moe_status_t launch_base_grad_t(const CUtensorMap* u, const CUtensorMap* v,
                                BaseGradArgs args, cudaStream_t st) {
  using C = BaseGradCfg<BN>;
  int begin = 0;
  for (int i = 0; i < 2; ++i) {
    BaseGradProblem& p = args.prob[i];
    p.p_tiles = (p.P + 127) / 128;
    p.q_tiles = (p.Q + BN - 1) / BN;
    p.tile_begin = begin;  // inside one expert's tiles
    begin += p.p_tiles * p.q_tiles;
  }
  args.tiles_per_expert = begin;
  args.total_tiles = args.E * begin;
  auto kern = base_grad_kernel<BN>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           C::SMEM_BYTES) != cudaSuccess)
    return MOE_ERR_CUDA;
  const int grid = std::min(num_sms(), args.total_tiles);
  if (grid <= 0) return MOE_OK;
  ProfScope prof(MOE_PROF_BASE_GRAD, st);
  launch_k(kern, grid, 192, C::SMEM_BYTES, st, u[0], u[1], v[0], v[1], args);
  count_launch();
  return launch_status();
}

// The same two problems as 256 x 256 (or 256 x 128) tiles on CTA pairs
// (measured against the single-CTA kernel: gpt-oss-20b shape 1770 -> 1510 us,
// Qwen3-30B-A3B shape 1315 -> 1232 us per launch).
#ifndef MOE_BASE_GRAD_PAIR
#define MOE_BASE_GRAD_PAIR 1
#endif

moe_status_t launch_base_grad_pair(const CUtensorMap* u, const CUtensorMap* v,
                                   BaseGradArgs args, cudaStream_t st) {
  using C = BaseGradPairCfg;
  int begin = 0;
  for (int i = 0; i < 2; ++i) {
    BaseGradProblem& p = args.prob[i];
    p.p_tiles = (p.P + 255) / 256;
    p.q_tiles = (p.Q + 255) / 256;
    p.tile_begin = begin;
    begin += p.p_tiles * p.q_tiles;
  }
  args.tiles_per_expert = begin;
  args.total_tiles = args.E * begin;
  if (cudaFuncSetAttribute(base_grad_pair_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           C::SMEM_BYTES) != cudaSuccess)
    return MOE_ERR_CUDA;
  const int pairs = std::min(num_sms() / 2, args.total_tiles);
  if (pairs <= 0) return MOE_OK;
  ProfScope prof(MOE_PROF_BASE_GRAD, st);
  launch_k(base_grad_pair_kernel, 2 * pairs, C::THREADS, C::SMEM_BYTES, st, u[0], u[1], v[0],
           v[1], args);
  count_launch();
  return launch_status();
}

// dW1 = per-expert dZ1^T Xp, dW2 = dZ2^T h (one launch for both).  On CTA
// pairs where the backward GEMMs run on pairs; otherwise single CTAs with
// the tile width of {256, 192} with the smaller estimated cost
// tiles * (BN + 32) over both problems.
moe_status_t base_grads(const void* dZ1, const void* Xp, const void* dZ2, const void* h,
                        const int32_t* offsets, int E, int H, int I, int R, void* dW1,
                        void* dW2, cudaStream_t st) {
  const void* U[2] = {dZ1, dZ2};
  const void* V[2] = {Xp, h};
  const int P[2] = {2 * I, H}, Q[2] = {H, I};
  CUtensorMap tu[2], tv[2];
  for (int i = 0; i < 2; ++i) {
    bool ok = tmap_2d(&tu[i], U[i], P[i], R, P[i] * 2ull, 64, 64, CU_TENSOR_MAP_SWIZZLE_128B);
    ok = ok && tmap_2d(&tv[i], V[i], Q[i], R, Q[i] * 2ull, 64, 64, CU_TENSOR_MAP_SWIZZLE_128B);
    if (!ok) return MOE_ERR_CUDA;
  }
  BaseGradArgs g{};
  g.offsets = offsets;
  g.E = E;
  g.R = R;
  g.wait_ns = g_wait_limit_ns;
  g.prob[0].P = P[0]; g.prob[0].Q = Q[0]; g.prob[0].out = static_cast<__nv_bfloat16*>(dW1);
  g.prob[1].P = P[1]; g.prob[1].Q = Q[1]; g.prob[1].out = static_cast<__nv_bfloat16*>(dW2);
  if (MOE_BASE_GRAD_PAIR && use_pairs(R, E, 2 * I)) return launch_base_grad_pair(tu, tv, g, st);
  double cost[2] = {0, 0};
  const int bns[2] = {256, 192};
  for (int c = 0; c < 2; ++c)
    for (int i = 0; i < 2; ++i)
      cost[c] += static_cast<double>((P[i] + 127) / 128) * ((Q[i] + bns[c] - 1) / bns[c]) *
                 (bns[c] + 32);
  return cost[0] <= cost[1] ? launch_base_grad_t<256>(tu, tv, g, st)
                            : launch_base_grad_t<192>(tu, tv, g, st);
}

template <int BN>
moe_status_t launch_router_logits_t(const void* X, const void* Wr, int T, int H, int E,
                                    float* logits, cudaStream_t st) {
  using C = RouterCfg<BN>;
  CUtensorMap tx, tw;
  bool ok = tmap_2d(&tx, X, H, T, H * 2ull, 64, 128, CU_TENSOR_MAP_SWIZZLE_128B);
  ok = ok && tmap_2d(&tw, Wr, H, E, H * 2ull, 64, BN, CU_TENSOR_MAP_SWIZZLE_128B);
  if (!ok) return MOE_ERR_CUDA;
  auto kern = router_logits_kernel<BN>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           C::SMEM_BYTES) != cudaSuccess)
    return MOE_ERR_CUDA;
  dim3 grid((T + 127) / 128, (E + BN - 1) / BN);
  ProfScope prof(MOE_PROF_ROUTER_FWD, st);
  launch_k(kern, grid, 192, C::SMEM_BYTES, st, tx, tw, T, H, E, logits, g_wait_limit_ns);
  count_launch();
  return launch_status();
}

template <int RK, bool KMAJ_F>
moe_status_t launch_rank_down_t(const void* U, const void* F, int K, const int32_t* offsets,
                                int E, int R, float s, void* out_rm, void* out_t,
                                cudaStream_t st) {
  using C = RankDownCfg<RK, KMAJ_F>;
  CUtensorMap tu, tf;
  const uint64_t EU = static_cast<uint64_t>(E);
  bool ok = tmap_2d(&tu, U, K, R, K * 2ull, 64, 128, CU_TENSOR_MAP_SWIZZLE_128B);
  if constexpr (KMAJ_F)  // F^T = A [E * r, K]
    ok = ok && tmap_2d(&tf, F, K, EU * RK, K * 2ull, 64, RK, CU_TENSOR_MAP_SWIZZLE_128B);
  else                   // F = B [E * K, r]
    ok = ok && tmap_2d(&tf, F, RK, EU * K, RK * 2ull, RK, 64, lora_swizzle(RK));
  if (!ok) return MOE_ERR_CUDA;
  RankDownArgs a{};
  a.offsets = offsets;
  a.E = E; a.R = R; a.K = K; a.k_rows = K; a.s = s;
  a.out_rm = static_cast<__nv_bfloat16*>(out_rm);
  a.out_t = static_cast<__nv_bfloat16*>(out_t);
  a.ld_t = ld_rank(R);
  a.wait_ns = g_wait_limit_ns;
  auto kern = rank_down_kernel<RK, KMAJ_F>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           C::SMEM_BYTES) != cudaSuccess)
    return MOE_ERR_CUDA;
  const int grid = static_cast<int>(
      std::min<long long>(static_cast<long long>(num_sms()) * C::CTAS_PER_SM, R / 128 + E));
  if (grid <= 0) return MOE_OK;
  ProfScope prof(MOE_PROF_RANK_DOWN, st);
  launch_k(kern, grid, 192, C::SMEM_BYTES, st, tu, tf, a);
  count_launch();
  return launch_status();
}

// s U_e F[e] per expert, row-major [R, r] and transposed [r, ldR]; F is
// B [E, K, r] (backward) or, with kmaj_f, A [E, r, K] (forward: s U A^T).
moe_status_t rank_down(int r, bool kmaj_f, const void* U, const void* F, int K,
                       const int32_t* offsets, int E, int R, float s, void* out_rm,
                       void* out_t, cudaStream_t st) {
#define MOE_RANK_DOWN(RK_)                                                                   \
  return kmaj_f ? launch_rank_down_t<RK_, true>(U, F, K, offsets, E, R, s, out_rm, out_t, st) \
                : launch_rank_down_t<RK_, false>(U, F, K, offsets, E, R, s, out_rm, out_t, st)
  if (r == 16) MOE_RANK_DOWN(16);
  if (r == 32) MOE_RANK_DOWN(32);
  if (r == 64) MOE_RANK_DOWN(64);
#undef MOE_RANK_DOWN
  return MOE_ERR_UNSUPPORTED;
}

}  // namespace

extern "C" {

const char* moe_status_string(moe_status_t s) {
  switch (s) {
    case MOE_OK: return "ok";
    case MOE_ERR_INVALID_ARG: return "invalid argument";
    case MOE_ERR_UNSUPPORTED: return "unsupported shape";
    case MOE_ERR_CUDA: return "CUDA error";
    case MOE_ERR_DEVICE_TIMEOUT: return "device wait timed out";
    case MOE_ERR_DEVICE_BOUNDS: return "device index out of range";
    default: return "unknown status";
  }
}

void moe_set_wait_limit_ns(uint64_t ns) {
  g_wait_limit_ns = ns ? ns : 1000000000ull;
}

void moe_test_inject_stall(int on) { g_stall_test = on ? 1 : 0; }

unsigned long long moe_kernel_launches(void) {
  return g_launches.load(std::memory_order_relaxed);
}

void moe_set_cta_pairs(int mode) { g_cta_pairs = mode > 0 ? 1 : (mode == 0 ? 0 : -1); }

int moe_uses_cta_pairs(int R, int E, int K) { return use_pairs(R, E, K) ? 1 : 0; }

moe_status_t moe_profile_enable(int on) {
  if (on && !g_prof_created) {
    for (int k = 0; k < MOE_PROF_KINDS; ++k)
      for (int i = 0; i < kProfCap; ++i)
        for (int w = 0; w < 2; ++w)
          if (cudaEventCreate(&g_prof_ev[k][i][w]) != cudaSuccess) return MOE_ERR_CUDA;
    g_prof_created = true;
  }
  for (int k = 0; k < MOE_PROF_KINDS; ++k) g_prof_n[k] = 0;
  g_prof_on = on != 0;
  return MOE_OK;
}

int moe_profile_collect(int kind, float* ms, int max_n) {
  if (!g_prof_created || kind < 0 || kind >= MOE_PROF_KINDS) return 0;
  const int n = std::min(g_prof_n[kind], max_n);
  for (int i = 0; i < n; ++i) {
    if (cudaEventSynchronize(g_prof_ev[kind][i][1]) != cudaSuccess ||
        cudaEventElapsedTime(&ms[i], g_prof_ev[kind][i][0], g_prof_ev[kind][i][1]) !=
            cudaSuccess)
      return -1;
  }
  return n;
}

#ifdef MOE_GEMM_TRACE
// Instrumented builds only: copies (and clears) the per-CTA wait counters.
MOE_API int moe_debug_read_trace(unsigned long long* out, int n) {
  const int total = static_cast<int>(sizeof(g_gemm_trace) / sizeof(unsigned long long));
  if (n < total) return -total;
  if (cudaDeviceSynchronize() != cudaSuccess) return -1;
  if (cudaMemcpyFromSymbol(out, g_gemm_trace, sizeof(g_gemm_trace)) != cudaSuccess) return -1;
  static unsigned long long zeros[sizeof(g_gemm_trace) / sizeof(unsigned long long)];
  if (cudaMemcpyToSymbol(g_gemm_trace, zeros, sizeof(g_gemm_trace)) != cudaSuccess) return -1;
  return total;
}
#endif

moe_status_t moe_get_device_status(moe_stream_t stream) {
  if (cudaStreamSynchronize(stream) != cudaSuccess) return MOE_ERR_CUDA;
  int v = 0, zero = 0;
  if (cudaMemcpyFromSymbol(&v, g_status, sizeof(int)) != cudaSuccess) return MOE_ERR_CUDA;
  if (cudaMemcpyToSymbol(g_status, &zero, sizeof(int)) != cudaSuccess) return MOE_ERR_CUDA;
  return v;
}

// ------------------------------------------------------------------ route
size_t moe_route_workspace_bytes(int T, int E, int k) {
  if (T <= 0 || E <= 0 || k <= 0) return 256;
  const size_t R = static_cast<size_t>(T) * k;
  const size_t nblk = (R + kRankChunk - 1) / kRankChunk;
  return align256(nblk * E * 4) + align256(R * 4);
}

moe_status_t moe_route_topk(const float* logits, int T, int E, int k, int32_t* topk_idx,
                            float* topk_w, int32_t* expert_counts,
                            int32_t* expert_offsets, int32_t* dest, void* ws,
                            size_t ws_bytes, moe_stream_t stream) {
  if (T < 0 || E < 1 || E > 512 || k < 1 || k > E) return MOE_ERR_UNSUPPORTED;
  if (static_cast<long long>(T) * k >= (1ll << 31)) return MOE_ERR_UNSUPPORTED;
  if (!expert_counts || !expert_offsets) return MOE_ERR_INVALID_ARG;
  cudaStream_t st = stream;
  if (T == 0) {
    if (cudaMemsetAsync(expert_counts, 0, E * 4, st) != cudaSuccess) return MOE_ERR_CUDA;
    if (cudaMemsetAsync(expert_offsets, 0, (E + 1) * 4, st) != cudaSuccess) return MOE_ERR_CUDA;
    return MOE_OK;
  }
  if (!logits || !topk_idx || !topk_w || !dest || !ws) return MOE_ERR_INVALID_ARG;
  if (ws_bytes < moe_route_workspace_bytes(T, E, k)) return MOE_ERR_INVALID_ARG;
  ProfScope prof(MOE_PROF_ROUTE, st);
  const int R = T * k;
  const int nblk = (R + kRankChunk - 1) / kRankChunk;
  int32_t* blk_hist = static_cast<int32_t*>(ws);
  int32_t* local_rank = at<int32_t>(ws, align256(static_cast<size_t>(nblk) * E * 4));
  // 1. top-k + weights, one token per warp
  const size_t smem1 = static_cast<size_t>(kRouteWarps) * k * 4;
  const int epl = (E + 31) / 32;
  const int grid1 = (T + kRouteWarps - 1) / kRouteWarps;
  auto launch = [&](auto kern) -> moe_status_t {
    if (smem1 > 48 * 1024 &&
        cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(smem1)) != cudaSuccess)
      return MOE_ERR_CUDA;
    launch_k(kern, grid1, kRouteWarps * 32, smem1, st, logits, T, E, k, topk_idx, topk_w);
    count_launch();
    return launch_status();
  };
  moe_status_t s;
  if (epl <= 1) s = launch(route_topk_kernel<1>);
  else if (epl <= 2) s = launch(route_topk_kernel<2>);
  else if (epl <= 4) s = launch(route_topk_kernel<4>);
  else if (epl <= 8) s = launch(route_topk_kernel<8>);
  else s = launch(route_topk_kernel<16>);
  if (s != MOE_OK) return s;
  // 2. stable in-chunk ranks + chunk histograms
  launch_k(route_rank_kernel, nblk, kRankWarps * 32, static_cast<size_t>(kRankWarps) * E * 4,
           st, topk_idx, R, E, blk_hist, local_rank);
  count_launch();
  if ((s = launch_status()) != MOE_OK) return s;
  // 3. expert totals, offsets and per-chunk base rows (one CTA)
  const int P = std::max(1, 1024 / E);
  const size_t smem2 = (static_cast<size_t>(P) * E + E + 1) * 4;
  launch_k(route_scan_kernel, 1, 1024, smem2, st, blk_hist, nblk, E, R, expert_counts,
           expert_offsets);
  count_launch();
  if ((s = launch_status()) != MOE_OK) return s;
  // 4. destination rows
  const int grid = std::min((R + 255) / 256, std::max(1, num_sms()) * 8);
  launch_k(route_dest_kernel, grid, 256, 0, st, topk_idx, blk_hist, local_rank, R, E, dest);
  count_launch();
  return launch_status();
}

// Same routing as moe_route_topk, with the scratch in g_route_scratch instead
// of a caller-provided workspace; allocates nothing.
moe_status_t moe_route_topk_noalloc(const float* logits, int T, int E, int k,
                                    int32_t* topk_idx, float* topk_w,
                                    int32_t* expert_counts, int32_t* expert_offsets,
                                    int32_t* dest, moe_stream_t stream) {
  if (T < 0 || E < 1 || E > 512 || k < 1 || k > E) return MOE_ERR_UNSUPPORTED;
  if (static_cast<long long>(T) * k >= (1ll << 31)) return MOE_ERR_UNSUPPORTED;
  if (moe_route_workspace_bytes(T, E, k) > kRouteScratchBytes) return MOE_ERR_UNSUPPORTED;
  void* scratch = nullptr;
  const moe_status_t st = route_scratch_on_current_device(&scratch);
  if (st != MOE_OK) return st;
  return moe_route_topk(logits, T, E, k, topk_idx, topk_w, expert_counts, expert_offsets,
                        dest, scratch, kRouteScratchBytes, stream);
}

size_t moe_route_noalloc_max_workspace_bytes(void) { return kRouteScratchBytes; }

// ---------------------------------------------------------- permute / combine
#ifndef MOE_DW_ROWS
#define MOE_DW_ROWS 1
#endif
// The combine (unpermute_kernel), its vector width and register budget
// chosen from the row length.
void launch_combine(const __nv_bfloat16* Yp, const int32_t* dest, const float* w, int T, int H,
                    int k, __nv_bfloat16* Y, const __nv_bfloat16* Wr, const int32_t* idx,
                    const float* g, int E, cudaStream_t st) {
  const int warps = 8;
  const int grid = std::min((T + warps - 1) / warps, std::max(1, num_sms()) * 8);
  auto kern = combine_vec(H / 8) == 4 ? unpermute_kernel<4, 3> : unpermute_kernel<2, 4>;
  launch_k(kern, grid, warps * 32, 0, st, Yp, dest, w, T, H, k, Y, Wr, idx, g, E);
}

moe_status_t moe_permute(const void* X, const int32_t* dest, const float* scale, int T,
                         int H, int k, void* Xp, const void* Zp, float* dw,
                         moe_stream_t stream) {
  if (T < 0 || H <= 0 || k < 1 || (H % 8)) return MOE_ERR_UNSUPPORTED;
  if (static_cast<long long>(T) * k >= (1ll << 31)) return MOE_ERR_UNSUPPORTED;
  if (T == 0) return MOE_OK;
  if (!X || !dest || !Xp) return MOE_ERR_INVALID_ARG;
  if ((dw == nullptr) != (Zp == nullptr)) return MOE_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(X) | reinterpret_cast<uintptr_t>(Xp) |
       reinterpret_cast<uintptr_t>(Zp)) & 15u)
    return MOE_ERR_INVALID_ARG;
  const int warps = 8;
  const int sms = std::max(1, num_sms());
  ProfScope prof(MOE_PROF_PERMUTE, stream);
  if (dw == nullptr) {
    const int nvec = H / 8;
    const int parts = row_parts(T, nvec, sms * MOE_PERMUTE_MINB * warps);
    const int vpl = permute_vpl((nvec + parts - 1) / parts);
    auto kern = vpl == 4    ? permute_rows_kernel<4>
                : vpl == 6  ? permute_rows_kernel<6>
                : vpl == 8  ? permute_rows_kernel<8>
                : vpl == 12 ? permute_rows_kernel<12>
                            : permute_rows_kernel<16>;
    const long long units = static_cast<long long>(T) * parts;
    const int grid = static_cast<int>(std::min<long long>((units + warps - 1) / warps, sms * 8));
    launch_k(kern, grid, warps * 32, 0, stream, static_cast<const __nv_bfloat16*>(X), dest,
             scale, T, H, k, static_cast<__nv_bfloat16*>(Xp), parts);
  } else if (MOE_DW_ROWS && k <= 32 && H / 8 <= 32 * 16) {
    // routing-weight gradient with the whole row in registers
    const int vpl = permute_vpl(H / 8);
    auto kern = vpl == 4    ? permute_dw_rows_kernel<4>
                : vpl == 6  ? permute_dw_rows_kernel<6>
                : vpl == 8  ? permute_dw_rows_kernel<8>
                : vpl == 12 ? permute_dw_rows_kernel<12>
                            : permute_dw_rows_kernel<16>;
    const int grid = std::min((T + warps - 1) / warps, sms * 8);
    launch_k(kern, grid, warps * 32, 0, stream, static_cast<const __nv_bfloat16*>(X), dest,
             scale, T, H, k, static_cast<__nv_bfloat16*>(Xp),
             static_cast<const __nv_bfloat16*>(Zp), dw);
  } else {
    const int grid = std::min((T + warps - 1) / warps, sms * 8);
    launch_k(permute_kernel, grid, warps * 32, 0, stream,
        static_cast<const __nv_bfloat16*>(X), dest, scale, T, H, k,
        static_cast<__nv_bfloat16*>(Xp), static_cast<const __nv_bfloat16*>(Zp), dw);
  }
  count_launch();
  return launch_status();
}

moe_status_t moe_unpermute(const void* Yp, const int32_t* dest, const float* w, int T,
                           int H, int k, void* Y, moe_stream_t stream) {
  if (T < 0 || H <= 0 || k < 1 || (H % 8)) return MOE_ERR_UNSUPPORTED;
  if (static_cast<long long>(T) * k >= (1ll << 31)) return MOE_ERR_UNSUPPORTED;
  if (T == 0) return MOE_OK;
  if (!Yp || !dest || !Y) return MOE_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(Yp) | reinterpret_cast<uintptr_t>(Y)) & 15u)
    return MOE_ERR_INVALID_ARG;
  ProfScope prof(MOE_PROF_UNPERMUTE, stream);
  launch_combine(static_cast<const __nv_bfloat16*>(Yp), dest, w, T, H, k,
                 static_cast<__nv_bfloat16*>(Y), nullptr, nullptr, nullptr, 0, stream);
  count_launch();
  return launch_status();
}

// ------------------------------------------------------ expert parallelism
moe_status_t moe_ep_regroup(const void* in, const int32_t* counts, int N, int E_loc, int rows,
                            int H, int dir, void* out, int32_t* offsets, moe_stream_t stream) {
  if (N < 1 || E_loc < 1 || static_cast<long long>(N) * E_loc > kRegroupMaxSegs || rows < 0 ||
      H <= 0 || (H % 8) || (dir != 0 && dir != 1))
    return MOE_ERR_UNSUPPORTED;
  if (!counts) return MOE_ERR_INVALID_ARG;
  if (offsets != nullptr && dir != 0) return MOE_ERR_INVALID_ARG;
  cudaStream_t st = stream;
  if (rows > 0) {
    if (!in || !out) return MOE_ERR_INVALID_ARG;
    if ((reinterpret_cast<uintptr_t>(in) | reinterpret_cast<uintptr_t>(out)) & 15u)
      return MOE_ERR_INVALID_ARG;
  }
  const int nseg = N * E_loc;
  const size_t smem = (2 * static_cast<size_t>(nseg) + 1 + 32) * 4;
  if (smem > 48 * 1024 &&
      cudaFuncSetAttribute(ep_regroup_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(smem)) != cudaSuccess)
    return MOE_ERR_CUDA;
  const int warps = kRegroupThreads / 32;
  const int grid =
      std::max(1, std::min((rows + warps - 1) / warps, std::max(1, num_sms()) * 8));
  launch_k(ep_regroup_kernel, grid, kRegroupThreads, smem, st,
      static_cast<const __nv_bfloat16*>(in), counts, N, E_loc, rows, H, dir,
      static_cast<__nv_bfloat16*>(out), offsets);
  count_launch();
  return launch_status();
}

// ------------------------------------------------------------- trained router
moe_status_t moe_router_fwd(const void* X, const void* Wr, int T, int H, int E,
                            float* logits, moe_stream_t stream) {
  if (T < 0 || H < 64 || (H % 16) || E < 1 || E > 512) return MOE_ERR_UNSUPPORTED;
  if (T == 0) return MOE_OK;
  if (!X || !Wr || !logits) return MOE_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(X) | reinterpret_cast<uintptr_t>(Wr)) & 15u)
    return MOE_ERR_INVALID_ARG;
  if (E <= 16) return launch_router_logits_t<16>(X, Wr, T, H, E, logits, stream);
  if (E <= 32) return launch_router_logits_t<32>(X, Wr, T, H, E, logits, stream);
  if (E <= 64) return launch_router_logits_t<64>(X, Wr, T, H, E, logits, stream);
  if (E <= 128) return launch_router_logits_t<128>(X, Wr, T, H, E, logits, stream);
  return launch_router_logits_t<256>(X, Wr, T, H, E, logits, stream);
}

size_t moe_router_bwd_workspace_bytes(int T, int k) {
  if (T < 0 || k < 1) return 0;
  return 2 * align256(static_cast<size_t>(T) * k * 4);
}

moe_status_t moe_router_bwd(const float* w, const float* dw, const int32_t* topk_idx,
                            const int32_t* dest, const int32_t* expert_offsets,
                            const void* Xp, const void* Wr, const void* dXp, int T, int H,
                            int E, int k, void* dX, float* dWr, void* ws, size_t ws_bytes,
                            moe_stream_t stream) {
  if (T < 0 || H < 64 || (H % 16) || E < 1 || E > 512 || k < 1 || k > E)
    return MOE_ERR_UNSUPPORTED;
  if (static_cast<long long>(T) * k >= (1ll << 31)) return MOE_ERR_UNSUPPORTED;
  if (!dWr) return MOE_ERR_INVALID_ARG;
  cudaStream_t st = stream;
  if (T == 0)
    return cudaMemsetAsync(dWr, 0, static_cast<size_t>(E) * H * 4, st) == cudaSuccess
               ? MOE_OK
               : MOE_ERR_CUDA;
  if (!w || !dw || !topk_idx || !dest || !expert_offsets || !Xp || !Wr || !dXp || !dX || !ws)
    return MOE_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(Xp) | reinterpret_cast<uintptr_t>(Wr) |
       reinterpret_cast<uintptr_t>(dXp) | reinterpret_cast<uintptr_t>(dX)) & 15u)
    return MOE_ERR_INVALID_ARG;
  if (ws_bytes < moe_router_bwd_workspace_bytes(T, k)) return MOE_ERR_INVALID_ARG;
  const int R = T * k;
  float* g = static_cast<float*>(ws);
  float* g_row = at<float>(ws, align256(static_cast<size_t>(R) * 4));
  ProfScope prof(MOE_PROF_ROUTER_BWD, st);
  const int grid0 = std::min((T + 255) / 256, std::max(1, num_sms()) * 4);
  launch_k(router_dlogit_kernel, grid0, 256, 0, st, w, dw, dest, T, k, g, g_row);
  count_launch();
  moe_status_t s;
  if ((s = launch_status()) != MOE_OK) return s;
  launch_k(router_wgrad_kernel, dim3(E, (H + kRouterWCols - 1) / kRouterWCols), 256, 0, st,
      static_cast<const __nv_bfloat16*>(Xp), g_row, expert_offsets, E, H, R, dWr);
  count_launch();
  if ((s = launch_status()) != MOE_OK) return s;
  launch_combine(static_cast<const __nv_bfloat16*>(dXp), dest, nullptr, T, H, k,
                 static_cast<__nv_bfloat16*>(dX), static_cast<const __nv_bfloat16*>(Wr),
                 topk_idx, g, E, st);
  count_launch();
  return launch_status();
}

// ------------------------------------------------------------------ sizes
size_t moe_saved_bytes(int R, int H, int I, int r) {
  if (R < 0 || H <= 0 || I <= 0 || r <= 0) return 0;
  size_t off[kSavedParts + 1];
  saved_layout(R, H, I, r, off);
  return off[kSavedParts];
}

size_t moe_saved_part_offset(int R, int H, int I, int r, int part) {
  if (part < 0 || part > kSavedParts || R < 0) return 0;
  size_t off[kSavedParts + 1];
  saved_layout(R, H, I, r, off);
  return off[part];
}

size_t moe_workspace_bytes(int R, int E, int H, int I, int r) {
  if (R < 0 || E <= 0 || H <= 0 || I <= 0 || r <= 0) return 0;
  size_t off[10];
  bwd_layout(R, E, H, I, r, off);
  return off[9];
}

// ------------------------------------------------------------------ forward
moe_status_t moe_lora_mlp_fwd(const void* Xp, const int32_t* expert_offsets, int E,
                              int H, int I, int r, float s, const void* W1,
                              const void* A1, const void* B1, const void* W2,
                              const void* A2, const void* B2, int R, void* Z2,
                              void* saved, size_t saved_bytes, void* ws,
                              size_t ws_bytes, moe_stream_t stream) {
  (void)ws;
  (void)ws_bytes;
  if (!shape_ok(E, H, I, r) || R < 0) return MOE_ERR_UNSUPPORTED;
  if (R == 0) return MOE_OK;
  if (!Xp || !expert_offsets || !W1 || !A1 || !B1 || !W2 || !A2 || !B2 || !Z2 || !saved)
    return MOE_ERR_INVALID_ARG;
  if (saved_bytes < moe_saved_bytes(R, H, I, r)) return MOE_ERR_INVALID_ARG;
  cudaStream_t st = stream;
  size_t off[kSavedParts + 1];
  saved_layout(R, H, I, r, off);
  __nv_bfloat16* Z1 = at<__nv_bfloat16>(saved, off[0]);
  __nv_bfloat16* h = at<__nv_bfloat16>(saved, off[1]);
  __nv_bfloat16* xa1 = at<__nv_bfloat16>(saved, off[2]);
  __nv_bfloat16* ha2 = at<__nv_bfloat16>(saved, off[3]);
  __nv_bfloat16* xa1_rm = at<__nv_bfloat16>(saved, off[4]);
  __nv_bfloat16* ha2_rm = at<__nv_bfloat16>(saved, off[5]);
  moe_status_t stt;
  if ((stt = zero_rank_padding(xa1, R, r, st)) != MOE_OK) return stt;
  if ((stt = zero_rank_padding(ha2, R, r, st)) != MOE_OK) return stt;
  const CUtensorMapSwizzle lsw = lora_swizzle(r);
  const uint64_t EU = static_cast<uint64_t>(E);

  // gate_up + SwiGLU
  if (use_pairs(R, E, H)) {
    // s Xp A1^T (both layouts) on its own pass, then the GEMM
    if ((stt = rank_down(r, true, Xp, A1, H, expert_offsets, E, R, s, xa1_rm, xa1, st)) !=
        MOE_OK)
      return stt;
    GemmArgs g{};
    g.offsets = expert_offsets;
    g.E = E; g.R = R; g.K = H; g.N = I; g.n_tiles = (I + 127) / 128; g.I = I;
    g.tile_n = 256;
    g.b_rows = 2 * I; g.lb_rows = 2 * I; g.s = s;
    g.out = h; g.ld_out = I; g.out2 = Z1; g.ld_out2 = 2 * I;
    g.lora_t = nullptr; g.ld_lora = ld_rank(R); g.wait_ns = g_wait_limit_ns;
    g.stall_test = g_stall_test;
    if ((stt = launch_pair<kGateUpFwd>(r, Xp, W1, xa1_rm, B1, g, st)) != MOE_OK) return stt;
  } else {
    const int bn = pick_bn(I, true, r, false), half = bn / 2;
    CUtensorMap ta, tb, tla, tlb;
    bool ok = tmap_2d(&ta, Xp, H, R, H * 2ull, kGemmBK, 128, kKmajSwz);
    ok = ok && tmap_2d(&tb, W1, H, EU * 2 * I, H * 2ull, kGemmBK, half, kKmajSwz);
    ok = ok && tmap_2d(&tla, A1, H, EU * r, H * 2ull, kGemmBK, r, kKmajSwz);
    ok = ok && tmap_2d(&tlb, B1, r, EU * 2 * I, r * 2ull, r, half, lsw);
    if (!ok) return MOE_ERR_CUDA;
    GemmArgs g{};
    g.offsets = expert_offsets;
    g.E = E; g.R = R; g.K = H; g.N = I; g.n_tiles = (I + half - 1) / half; g.I = I;
    g.b_rows = 2 * I; g.lb_rows = 2 * I; g.s = s;
    g.out = h; g.ld_out = I; g.out2 = Z1; g.ld_out2 = 2 * I;
    g.lora_t = xa1; g.ld_lora = ld_rank(R); g.wait_ns = g_wait_limit_ns;
    g.stall_test = g_stall_test;
    if ((stt = launch_gemm<kGateUpFwd>(bn, r, ta, tb, tla, tlb, g, st)) != MOE_OK) return stt;
  }
  // down
  if (use_pairs(R, E, I)) {
    if ((stt = rank_down(r, true, h, A2, I, expert_offsets, E, R, s, ha2_rm, ha2, st)) !=
        MOE_OK)
      return stt;
    const int tn = pair_tile_n(H, false);
    GemmArgs g{};
    g.offsets = expert_offsets;
    g.E = E; g.R = R; g.K = I; g.N = H; g.n_tiles = (H + tn - 1) / tn; g.I = I;
    g.tile_n = tn;
    g.b_rows = H; g.lb_rows = H; g.s = s;
    g.out = static_cast<__nv_bfloat16*>(Z2); g.ld_out = H;
    g.lora_t = nullptr; g.ld_lora = ld_rank(R); g.wait_ns = g_wait_limit_ns;
    g.stall_test = g_stall_test;
    if ((stt = launch_pair<kDownFwd>(r, h, W2, ha2_rm, B2, g, st)) != MOE_OK) return stt;
  } else {
    const int bn = pick_bn(H, false, r, false);
    CUtensorMap ta, tb, tla, tlb;
    bool ok = tmap_2d(&ta, h, I, R, I * 2ull, kGemmBK, 128, kKmajSwz);
    ok = ok && tmap_2d(&tb, W2, I, EU * H, I * 2ull, kGemmBK, bn, kKmajSwz);
    ok = ok && tmap_2d(&tla, A2, I, EU * r, I * 2ull, kGemmBK, r, kKmajSwz);
    ok = ok && tmap_2d(&tlb, B2, r, EU * H, r * 2ull, r, bn, lsw);
    if (!ok) return MOE_ERR_CUDA;
    GemmArgs g{};
    g.offsets = expert_offsets;
    g.E = E; g.R = R; g.K = I; g.N = H; g.n_tiles = (H + bn - 1) / bn; g.I = I;
    g.b_rows = H; g.lb_rows = H; g.s = s;
    g.out = static_cast<__nv_bfloat16*>(Z2); g.ld_out = H;
    g.lora_t = ha2; g.ld_lora = ld_rank(R); g.wait_ns = g_wait_limit_ns;
    g.stall_test = g_stall_test;
    if ((stt = launch_gemm<kDownFwd>(bn, r, ta, tb, tla, tlb, g, st)) != MOE_OK) return stt;
  }
  return MOE_OK;
}

// ------------------------------------------------------------------ backward
}  // extern "C"

namespace {

moe_status_t lora_mlp_bwd_impl(const void* dZ2, const void* Xp,
                               const int32_t* expert_offsets, int E, int H, int I, int r,
                               float s, const void* W1, const void* A1, const void* B1,
                               const void* W2, const void* A2, const void* B2,
                               const void* saved, size_t saved_bytes, int R, void* dXp,
                               void* dA1, void* dB1, void* dA2, void* dB2, void* dW1,
                               void* dW2, void* ws, size_t ws_bytes, cudaStream_t st) {
  if (!shape_ok(E, H, I, r) || R < 0) return MOE_ERR_UNSUPPORTED;
  if (!dA1 || !dB1 || !dA2 || !dB2) return MOE_ERR_INVALID_ARG;
  const bool full = dW1 != nullptr;
  if (full && ((reinterpret_cast<uintptr_t>(dW1) | reinterpret_cast<uintptr_t>(dW2)) & 15u))
    return MOE_ERR_INVALID_ARG;
  if (R == 0) {
    const size_t n = static_cast<size_t>(E) * r * 2;
    if (cudaMemsetAsync(dA1, 0, n * H, st) != cudaSuccess ||
        cudaMemsetAsync(dB1, 0, n * 2 * I, st) != cudaSuccess ||
        cudaMemsetAsync(dA2, 0, n * I, st) != cudaSuccess ||
        cudaMemsetAsync(dB2, 0, n * H, st) != cudaSuccess)
      return MOE_ERR_CUDA;
    if (full) {
      const size_t w = static_cast<size_t>(E) * H * I * 2;
      if (cudaMemsetAsync(dW1, 0, 2 * w, st) != cudaSuccess ||
          cudaMemsetAsync(dW2, 0, w, st) != cudaSuccess)
        return MOE_ERR_CUDA;
    }
    return MOE_OK;
  }
  if (!dZ2 || !Xp || !expert_offsets || !W1 || !A1 || !B1 || !W2 || !A2 || !B2 ||
      !saved || !dXp || !ws)
    return MOE_ERR_INVALID_ARG;
  if (saved_bytes < moe_saved_bytes(R, H, I, r)) return MOE_ERR_INVALID_ARG;
  if (ws_bytes < moe_workspace_bytes(R, E, H, I, r)) return MOE_ERR_INVALID_ARG;
  size_t so[kSavedParts + 1], wo[10];
  saved_layout(R, H, I, r, so);
  bwd_layout(R, E, H, I, r, wo);
  const __nv_bfloat16* Z1 = at<__nv_bfloat16>(saved, so[0]);
  const __nv_bfloat16* h = at<__nv_bfloat16>(saved, so[1]);
  const __nv_bfloat16* xa1 = at<__nv_bfloat16>(saved, so[2]);
  const __nv_bfloat16* ha2 = at<__nv_bfloat16>(saved, so[3]);
  __nv_bfloat16* dZ1 = at<__nv_bfloat16>(ws, wo[0]);
  __nv_bfloat16* dzb2 = at<__nv_bfloat16>(ws, wo[1]);
  __nv_bfloat16* dzb1 = at<__nv_bfloat16>(ws, wo[2]);
  const void* B2p = B2;  // [E*H, 64 or 32]: B2 itself when r fills the width
  const void* B1p = B1;  // [E*2I, 64 or 32]
  __nv_bfloat16* A2t = at<__nv_bfloat16>(ws, wo[4]);
  __nv_bfloat16* A1t = at<__nv_bfloat16>(ws, wo[6]);
  moe_status_t stt;
  if ((stt = zero_rank_padding(dzb2, R, r, st)) != MOE_OK) return stt;
  if ((stt = zero_rank_padding(dzb1, R, r, st)) != MOE_OK) return stt;
  // Operand copies of the LoRA factors: the down-projection factors B2, B1
  // zero-padded to one 64-column MN-major atom for the single-CTA kernels
  // (fused into the base MMA; the CTA-pair backward reads them in place in
  // its rank-r pass), the up-projection factors A2, A1 transposed to K-major
  // (both kernels).
  const bool pair_down = use_pairs(R, E, H);
  const bool pair_gate_up = use_pairs(R, E, 2 * I);
  FactorPrep prep;
  if (r < 64 && !pair_down) {
    B2p = at<__nv_bfloat16>(ws, wo[3]);
    prep.pad(B2, const_cast<void*>(B2p), 1ll * E * H, r, 64);
  }
  if (r < 64 && !pair_gate_up) {
    B1p = at<__nv_bfloat16>(ws, wo[5]);
    prep.pad(B1, const_cast<void*>(B1p), 2ll * E * I, r, 64);
  }
  __nv_bfloat16* dzb2_rm = at<__nv_bfloat16>(ws, wo[7]);
  __nv_bfloat16* dzb1_rm = at<__nv_bfloat16>(ws, wo[8]);
  // (the CTA-pair kernels read A2, A1 in place as MN-major operands)
  if (!pair_down) prep.transpose(A2, A2t, E, r, I);
  if (!pair_gate_up) prep.transpose(A1, A1t, E, r, H);
  if ((stt = prep.launch(st)) != MOE_OK) return stt;
  const CUtensorMapSwizzle lsw = lora_swizzle(r);
  const uint64_t EU = static_cast<uint64_t>(E);

  // down backward: dh = dZ2 W2 + s (dZ2 B2) A2, SwiGLU backward -> dZ1
  if (pair_down) {
    const int bn = pair_tile_n(I, true);
    GemmArgs g{};
    g.offsets = expert_offsets;
    g.E = E; g.R = R; g.K = H; g.N = I; g.n_tiles = (I + bn - 1) / bn; g.I = I;
    g.tile_n = bn;
    g.b_rows = H; g.lb_rows = I; g.s = s;
    g.out = dZ1; g.ld_out = 2 * I; g.aux = Z1; g.ld_aux = 2 * I;
    g.lora_t = nullptr; g.ld_lora = ld_rank(R); g.wait_ns = g_wait_limit_ns;
    g.stall_test = g_stall_test;
    // s dZ2 B2 (both layouts) on its own pass, then the GEMM
    if ((stt = rank_down(r, false, dZ2, B2, H, expert_offsets, E, R, s, dzb2_rm, dzb2, st)) !=
        MOE_OK)
      return stt;
    if ((stt = launch_pair<kDownBwd>(r, dZ2, W2, dzb2_rm, A2, g, st)) != MOE_OK) return stt;
  } else {
    const int bn = pick_bn(I, false, r, true);
    CUtensorMap ta, tb, tla, tlb;
    bool ok = tmap_2d(&ta, dZ2, H, R, H * 2ull, kGemmBK, 128, kKmajSwz);
    ok = ok && tmap_2d(&tb, W2, I, EU * H, I * 2ull, 64, kGemmBK, CU_TENSOR_MAP_SWIZZLE_128B);
    ok = ok && tmap_2d(&tla, B2p, 64, EU * H, 128, 64, kGemmBK, CU_TENSOR_MAP_SWIZZLE_128B);
    ok = ok && tmap_2d(&tlb, A2t, r, EU * I, r * 2ull, r, bn, lsw);
    if (!ok) return MOE_ERR_CUDA;
    GemmArgs g{};
    g.offsets = expert_offsets;
    g.E = E; g.R = R; g.K = H; g.N = I; g.n_tiles = (I + bn - 1) / bn; g.I = I;
    g.b_rows = H; g.lb_rows = I; g.s = s;
    g.out = dZ1; g.ld_out = 2 * I; g.aux = Z1; g.ld_aux = 2 * I;
    g.lora_t = dzb2; g.ld_lora = ld_rank(R); g.wait_ns = g_wait_limit_ns;
    g.stall_test = g_stall_test;
    if ((stt = launch_gemm<kDownBwd>(bn, r, ta, tb, tla, tlb, g, st)) != MOE_OK) return stt;
  }
  // LoRA gradients, after the gate_up GEMM (measured: running them before
  // it, right after the s dZ1 B1 pass, makes neither faster)
  auto lora_grads = [&]() -> moe_status_t {
    moe_status_t stt;
    const int ldr = ld_rank(R);
    const void* U[4] = {Xp, dZ1, h, dZ2};
    const void* V[4] = {dzb1, xa1, dzb2, ha2};
    const int P[4] = {H, 2 * I, I, H};
    void* out[4] = {dA1, dB1, dA2, dB2};
    const int tr[4] = {1, 0, 1, 0};
    CUtensorMap tu[4], tv[4];
    GradArgs g{};
    g.offsets = expert_offsets;
    g.E = E; g.R = R; g.wait_ns = g_wait_limit_ns;
    int begin = 0;
    for (int i = 0; i < 4; ++i) {
      bool ok = tmap_2d(&tu[i], U[i], P[i], R, P[i] * 2ull, 64, 64, CU_TENSOR_MAP_SWIZZLE_128B);
      ok = ok && tmap_2d(&tv[i], V[i], ldr, r, ldr * 2ull, 64, r, CU_TENSOR_MAP_SWIZZLE_128B);
      if (!ok) return MOE_ERR_CUDA;
      g.prob[i].P = P[i];
      g.prob[i].p_tiles = (P[i] + 127) / 128;
      g.prob[i].tile_begin = begin;  // inside one expert's tiles
      g.prob[i].transpose_out = tr[i];
      g.prob[i].out = static_cast<__nv_bfloat16*>(out[i]);
      begin += g.prob[i].p_tiles;
    }
    g.tiles_per_expert = begin;
    g.total_tiles = E * begin;
    if (r == 16) stt = launch_grad_t<16>(tu, tv, g, st);
    else if (r == 32) stt = launch_grad_t<32>(tu, tv, g, st);
    else stt = launch_grad_t<64>(tu, tv, g, st);
    return stt;
  };
  // gate_up backward: dXp = dZ1 W1 + s (dZ1 B1) A1
  if (pair_gate_up) {
    const int bn = pair_tile_n(H, true);
    GemmArgs g{};
    g.offsets = expert_offsets;
    g.E = E; g.R = R; g.K = 2 * I; g.N = H; g.n_tiles = (H + bn - 1) / bn; g.I = I;
    g.tile_n = bn;
    g.b_rows = 2 * I; g.lb_rows = H; g.s = s;
    g.out = static_cast<__nv_bfloat16*>(dXp); g.ld_out = H;
    g.lora_t = nullptr; g.ld_lora = ld_rank(R); g.wait_ns = g_wait_limit_ns;
    g.stall_test = g_stall_test;
    if ((stt = rank_down(r, false, dZ1, B1, 2 * I, expert_offsets, E, R, s, dzb1_rm, dzb1, st)) !=
        MOE_OK)
      return stt;
    if ((stt = launch_pair<kGateUpBwd>(r, dZ1, W1, dzb1_rm, A1, g, st)) != MOE_OK) return stt;
    if ((stt = lora_grads()) != MOE_OK) return stt;
  } else {
    const int bn = pick_bn(H, false, r, true);
    CUtensorMap ta, tb, tla, tlb;
    bool ok = tmap_2d(&ta, dZ1, 2 * I, R, 4ull * I, kGemmBK, 128, kKmajSwz);
    ok = ok && tmap_2d(&tb, W1, H, EU * 2 * I, H * 2ull, 64, kGemmBK, CU_TENSOR_MAP_SWIZZLE_128B);
    ok = ok && tmap_2d(&tla, B1p, 64, EU * 2 * I, 128, 64, kGemmBK, CU_TENSOR_MAP_SWIZZLE_128B);
    ok = ok && tmap_2d(&tlb, A1t, r, EU * H, r * 2ull, r, bn, lsw);
    if (!ok) return MOE_ERR_CUDA;
    GemmArgs g{};
    g.offsets = expert_offsets;
    g.E = E; g.R = R; g.K = 2 * I; g.N = H; g.n_tiles = (H + bn - 1) / bn; g.I = I;
    g.b_rows = 2 * I; g.lb_rows = H; g.s = s;
    g.out = static_cast<__nv_bfloat16*>(dXp); g.ld_out = H;
    g.lora_t = dzb1; g.ld_lora = ld_rank(R); g.wait_ns = g_wait_limit_ns;
    g.stall_test = g_stall_test;
    if ((stt = launch_gemm<kGateUpBwd>(bn, r, ta, tb, tla, tlb, g, st)) != MOE_OK) return stt;
    if ((stt = lora_grads()) != MOE_OK) return stt;
  }
  // base-weight gradients (full fine-tuning)
  if (full &&
      (stt = base_grads(dZ1, Xp, dZ2, h, expert_offsets, E, H, I, R, dW1, dW2, st)) != MOE_OK)
    return stt;
  return MOE_OK;
}

}  // namespace

extern "C" {

moe_status_t moe_lora_mlp_bwd(const void* dZ2, const void* Xp,
                              const int32_t* expert_offsets, int E, int H, int I, int r,
                              float s, const void* W1, const void* A1, const void* B1,
                              const void* W2, const void* A2, const void* B2,
                              const void* saved, size_t saved_bytes, int R, void* dXp,
                              void* dA1, void* dB1, void* dA2, void* dB2, void* ws,
                              size_t ws_bytes, moe_stream_t stream) {
  return lora_mlp_bwd_impl(dZ2, Xp, expert_offsets, E, H, I, r, s, W1, A1, B1, W2, A2, B2,
                           saved, saved_bytes, R, dXp, dA1, dB1, dA2, dB2, nullptr,
                           nullptr, ws, ws_bytes, stream);
}

moe_status_t moe_lora_mlp_bwd_full(const void* dZ2, const void* Xp,
                                   const int32_t* expert_offsets, int E, int H, int I,
                                   int r, float s, const void* W1, const void* A1,
                                   const void* B1, const void* W2, const void* A2,
                                   const void* B2, const void* saved, size_t saved_bytes,
                                   int R, void* dXp, void* dA1, void* dB1, void* dA2,
                                   void* dB2, void* dW1, void* dW2, void* ws,
                                   size_t ws_bytes, moe_stream_t stream) {
  if (!dW1 || !dW2) return MOE_ERR_INVALID_ARG;
  return lora_mlp_bwd_impl(dZ2, Xp, expert_offsets, E, H, I, r, s, W1, A1, B1, W2, A2, B2,
                           saved, saved_bytes, R, dXp, dA1, dB1, dA2, dB2, dW1, dW2, ws,
                           ws_bytes, stream);
}

}  // extern "C"
