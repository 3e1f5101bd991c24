/*
 * moe_lora.h -- C ABI of the B200 (sm_100a) MoE split-LoRA expert block.
 *
 * The block (forward and backward) is the Mixture-of-Experts expert MLP used
 * in LoRA fine-tuning, as described on the Unsloth page "Fine-tune MoE LLMs
 * 12x faster with Unsloth":
 *   route (top-k over router logits) -> permute tokens into expert order ->
 *   grouped GEMM over gate_up_proj [E, 2I, H] with SwiGLU -> grouped GEMM over
 *   down_proj [E, H, I] -> routing-weighted unpermute (combine).
 * Every projection carries split LoRA (section "Faster LoRA MoE training"):
 *   y = x W^T + s (x A^T) B^T,   A [E, r, in], B [E, out, r],
 * so W + s B A is never formed.  The backward computes dX and the LoRA
 * gradients dA, dB with the base weights frozen.
 *
 * Conventions (all entry points):
 *  - Every pointer except the status helpers is a DEVICE pointer; every
 *    tensor is dense row-major.  "bf16" means IEEE bfloat16 (16-bit, stored
 *    as uint16).  The caller owns and allocates every buffer, including the
 *    workspace and the saved-activation buffer; the library never allocates,
 *    frees or synchronises (except moe_get_device_status).
 *  - All work is enqueued asynchronously on `stream` (a cudaStream_t; NULL is
 *    the legacy default stream) on the current device.
 *  - Argument errors are detected on the host and returned before anything is
 *    launched.  Errors that only the device can see (a bounded wait that ran
 *    out, an index out of range) are recorded in a per-device status word that
 *    moe_get_device_status() returns and clears; the kernel that saw the error
 *    skips the offending access and returns.
 *  - Shape limits: 1 <= k <= E <= 512; H and I multiples of 16 and >= 64;
 *    r in {16, 32, 64}; T * k < 2^31.  Router logits must be finite.
 *  - R = T * k is the number of routed (token, slot) rows.
 */
#ifndef MOE_LORA_H_
#define MOE_LORA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef int moe_status_t;
#define MOE_OK 0
#define MOE_ERR_INVALID_ARG 1     /* null pointer, bad size, too-small buffer */
#define MOE_ERR_UNSUPPORTED 2     /* shape outside the limits above */
#define MOE_ERR_CUDA 3            /* a CUDA runtime / driver call failed */
#define MOE_ERR_DEVICE_TIMEOUT 4  /* a kernel's bounded wait ran out */
#define MOE_ERR_DEVICE_BOUNDS 5   /* a kernel found an index out of range */

typedef struct CUstream_st* moe_stream_t; /* same type as cudaStream_t */

#if defined(__GNUC__)
#define MOE_API __attribute__((visibility("default")))
#else
#define MOE_API
#endif

/* ---------------------------------------------------------------- a1: route
 * Top-k routing (page section "What is torch._grouped_mm?": each token is sent
 * to the experts its router picks; section "Implementation details": the
 * router is frozen, so logits are an input).
 *   logits        fp32 [T, E]   router logits (finite).
 *   topk_idx      int32 [T, k]  experts by (logit desc, expert index asc).
 *   topk_w        fp32 [T, k]   w_j = exp(l_j - l_max) / sum_sel exp(l - l_max)
 *                               (softmax over E renormalised over the kept k).
 *   expert_counts int32 [E]     rows routed to each expert.
 *   expert_offsets int32 [E+1]  exclusive prefix sum of counts; [E] = T*k.
 *   dest          int32 [T, k]  permuted row of (t, j): offsets[e] + the
 *                               number of earlier flat indices t'*k+j' routed
 *                               to the same expert (stable counting sort).
 *   ws            device scratch of moe_route_workspace_bytes(T, E, k) bytes.
 * Deterministic: the same inputs give the same bytes. */
MOE_API size_t moe_route_workspace_bytes(int T, int E, int k);
MOE_API moe_status_t moe_route_topk(const float* logits, int T, int E, int k,
                            int32_t* topk_idx, float* topk_w,
                            int32_t* expert_counts, int32_t* expert_offsets,
                            int32_t* dest, void* ws, size_t ws_bytes,
                            moe_stream_t stream);

/* Allocation-free variant of moe_route_topk (the pages have no counterpart:
 * this is an interface convenience, not part of the method).
 * Some callers cannot allocate device memory at the time they route: for
 * example a plugin whose enqueue hook runs inside a host engine that owns all
 * device memory and forbids cudaMalloc there, or code running under a fixed
 * memory budget decided at start-up.  This entry point needs no workspace:
 * its scratch is a 4 MiB array inside the library's own device memory (every
 * GPU that loads the library holds it until the process exits).  It computes
 * exactly what moe_route_topk computes; the caller still passes the logits
 * and all outputs.  It calls no cudaMalloc / cudaFree and no allocating
 * library routine.
 *  - Limit: moe_route_workspace_bytes(T, E, k) must not exceed
 *    moe_route_noalloc_max_workspace_bytes() (4 MiB; e.g. T <= 65536 tokens
 *    with k <= 8 and E <= 512); larger sizes return MOE_ERR_UNSUPPORTED
 *    before anything is launched.
 *  - Every call looks up the array's device address with the caller's device
 *    current (cudaGetSymbolAddress, a host-side query that allocates
 *    nothing), so the address stays right after cudaDeviceReset and in any
 *    context.  The first call in a process may load the library's device
 *    code: make one call before any stream capture begins.
 *  - All calls share the one array and it keeps the last call's contents.
 *    Nothing in it needs to start at zero (each call writes every scratch
 *    byte it reads before reading it), but calls whose work overlaps on the
 *    GPU (other streams, other threads) race on it: serialise them. */
MOE_API moe_status_t moe_route_topk_noalloc(const float* logits, int T, int E, int k,
                                            int32_t* topk_idx, float* topk_w,
                                            int32_t* expert_counts,
                                            int32_t* expert_offsets, int32_t* dest,
                                            moe_stream_t stream);
MOE_API size_t moe_route_noalloc_max_workspace_bytes(void);

/* ------------------------------------------------------- a2 / a6: permute
 * Gather into expert order: Xp[dest[t, j]] = scale[t, j] * X[t] (scale NULL
 * means 1; with scale the product is formed in fp32 and rounded to bf16).
 *   X [T, H] bf16 -> Xp [T*k, H] bf16.
 * Optional, for the routing-weight gradient (backward of the combine):
 *   if dw != NULL, dw[t, j] = <X[t], Zp[dest[t, j]]> (fp32 accumulation) with
 *   Zp [T*k, H] bf16 (pass the forward's Z2 and X = dY). */
MOE_API moe_status_t moe_permute(const void* X, const int32_t* dest, const float* scale,
                         int T, int H, int k, void* Xp, const void* Zp,
                         float* dw, moe_stream_t stream);

/* ----------------------------------------------------- a5 / a10: unpermute
 * Weighted combine: Y[t] = sum_j w[t, j] * Yp[dest[t, j]], accumulated in fp32
 * in j order, rounded once to bf16 (w NULL means 1: used for dX).
 *   Yp [T*k, H] bf16 -> Y [T, H] bf16.  No atomics; deterministic. */
MOE_API moe_status_t moe_unpermute(const void* Yp, const int32_t* dest, const float* w,
                           int T, int H, int k, void* Y, moe_stream_t stream);

/* ---------------------------------------------- saved activations / scratch
 * The forward writes what the backward needs into `saved`
 * (moe_saved_bytes(R, H, I, r) bytes, 256-byte aligned parts):
 *   part 0: Z1  bf16 [R, 2I]  gate_up output (gate = cols [0, I), up = [I, 2I))
 *   part 1: h   bf16 [R, I]   silu(gate) * up
 *   part 2: XA1 bf16 [r, R]   s * (Xp A1^T), transposed, row pitch
 *                             round_up(R, 64) elements (padding zeroed)
 *   part 3: HA2 bf16 [r, R]   s * (h A2^T), transposed, same pitch
 *   part 4: XA1 bf16 [R, r]   s * (Xp A1^T), row-major (written when the
 *                             gate_up GEMM runs on CTA pairs)
 *   part 5: HA2 bf16 [R, r]   s * (h A2^T), row-major (likewise, down GEMM)
 * moe_saved_part_offset(R, H, I, r, part) gives each part's byte offset;
 * part 6 is the end (= moe_saved_bytes). */
MOE_API size_t moe_saved_bytes(int R, int H, int I, int r);
MOE_API size_t moe_saved_part_offset(int R, int H, int I, int r, int part);
/* Scratch needed by moe_lora_mlp_fwd / moe_lora_mlp_bwd (device bytes). */
MOE_API size_t moe_workspace_bytes(int R, int E, int H, int I, int r);

/* ------------------------------------------------- a3 + a4: expert forward
 * Per expert e, on its rows Xp[offsets[e] : offsets[e+1]] (page section "What
 * is torch._grouped_mm?": gate, up = chunk(2) of linear(x, gate_up_proj[e])):
 *   Z1 = Xp W1[e]^T + s (Xp A1[e]^T) B1[e]^T             [M_e, 2I]
 *   h  = silu(Z1[:, :I]) * Z1[:, I:]                     [M_e, I]
 *   Z2 = h W2[e]^T + s (h A2[e]^T) B2[e]^T               [M_e, H]
 * Weights: W1 [E, 2I, H], A1 [E, r, H], B1 [E, 2I, r], W2 [E, H, I],
 * A2 [E, r, I], B2 [E, H, r]; all bf16.  Xp [R, H], Z2 [R, H] bf16.
 * expert_offsets is the device array from moe_route_topk (read on the device;
 * no host synchronisation).  Products accumulate in fp32 on the tensor cores;
 * the rank-r intermediates are rounded to bf16 before the second product.
 * `saved` receives the parts listed above; ws / ws_bytes are not used (NULL /
 * 0 allowed). */
MOE_API moe_status_t moe_lora_mlp_fwd(const void* Xp, const int32_t* expert_offsets,
                              int E, int H, int I, int r, float s,
                              const void* W1, const void* A1, const void* B1,
                              const void* W2, const void* A2, const void* B2,
                              int R, void* Z2, void* saved, size_t saved_bytes,
                              void* ws, size_t ws_bytes, moe_stream_t stream);

/* ---------------------------------------- a7 + a8 + a9: expert backward
 * Input dZ2 [R, H] bf16 is the gradient at Z2 already multiplied by the
 * routing weight (moe_permute of dY with scale = topk_w).  With the base
 * weights frozen:
 *   dh   = dZ2 W2[e] + s (dZ2 B2[e]) A2[e]                 [M_e, I]
 *   dZ1  = [dh * up * silu'(gate), dh * silu(gate)]        [M_e, 2I]
 *   dXp  = dZ1 W1[e] + s (dZ1 B1[e]) A1[e]                 [M_e, H]
 *   dA2[e] = s (dZ2 B2)^T h,   dB2[e] = s dZ2^T (h A2^T)
 *   dA1[e] = s (dZ1 B1)^T Xp,  dB1[e] = s dZ1^T (Xp A1^T)
 * with silu'(g) = sigmoid(g) (1 + g (1 - sigmoid(g))).  Outputs dXp [R, H],
 * dA1 [E, r, H], dB1 [E, 2I, r], dA2 [E, r, I], dB2 [E, H, r], all bf16
 * (fp32 accumulation, fixed order: deterministic).  Experts with no rows get
 * exact zeros.  `saved` must hold the forward's saved activations. */
MOE_API moe_status_t moe_lora_mlp_bwd(const void* dZ2, const void* Xp,
                              const int32_t* expert_offsets,
                              int E, int H, int I, int r, float s,
                              const void* W1, const void* A1, const void* B1,
                              const void* W2, const void* A2, const void* B2,
                              const void* saved, size_t saved_bytes, int R,
                              void* dXp, void* dA1, void* dB1, void* dA2,
                              void* dB2, void* ws, size_t ws_bytes,
                              moe_stream_t stream);

/* -------------------------- full fine-tuning: base-weight gradients as well
 * The page lists full fine-tuning beside LoRA among what its MoE kernels
 * support.  Everything moe_lora_mlp_bwd computes, plus, with W1 and W2
 * trainable (dW = dy^T x for each projection y = x W^T), per expert e with
 * rows [a, b):
 *   dW1[e] = dZ1[a:b]^T Xp[a:b]   [2I, H]     dW2[e] = dZ2[a:b]^T h[a:b]   [H, I]
 * Outputs dW1 [E, 2I, H] and dW2 [E, H, I] bf16 (the layouts of W1, W2),
 * accumulated in fp32 over the expert's rows in a fixed order
 * (deterministic); experts with no rows get exact zeros.  dW1 and dW2 must
 * both be non-NULL (MOE_ERR_INVALID_ARG otherwise) and 16-byte aligned.  Same
 * saved activations and workspace as moe_lora_mlp_bwd. */
MOE_API moe_status_t moe_lora_mlp_bwd_full(const void* dZ2, const void* Xp,
                                   const int32_t* expert_offsets,
                                   int E, int H, int I, int r, float s,
                                   const void* W1, const void* A1, const void* B1,
                                   const void* W2, const void* A2, const void* B2,
                                   const void* saved, size_t saved_bytes, int R,
                                   void* dXp, void* dA1, void* dB1, void* dA2,
                                   void* dB2, void* dW1, void* dW2, void* ws,
                                   size_t ws_bytes, moe_stream_t stream);

/* ------------------------------------------ expert parallelism (optional)
 * The pages call multi-GPU training experimental (winningdata.io hands-on
 * blog, section "Limitações"); they give no design.  With the E experts split
 * over N ranks (rank p holds experts [p * E_loc, (p + 1) * E_loc)), each rank
 * routes and permutes its own tokens over all E experts; its expert-major
 * rows are then already ordered by destination rank, and one all-to-all
 * (NCCL, called by the caller) sends each rank its experts' rows.  The
 * receiving rank holds them source-major: for each source s in turn, s's
 * rows for the E_loc local experts in expert order.  moe_ep_regroup moves
 * rows between that order and the expert-major order over all sources that
 * the local grouped GEMMs take (moe_lora_mlp_fwd / _bwd with E = E_loc);
 * within each (source, expert) segment the rows keep their order.
 *   in, out  bf16 [rows, H] device, 16-byte aligned, not overlapping.
 *   counts   int32 [N, E_loc] device: rows source s sent for local expert e
 *            (the all-to-all of moe_route_topk's expert_counts); rows must
 *            equal their sum, else MOE_ERR_DEVICE_BOUNDS is recorded and
 *            nothing is written.
 *   dir      0: out = in reordered source-major -> expert-major (dispatch);
 *            1: expert-major -> source-major (before the return all-to-all).
 *   offsets  int32 [E_loc + 1] device, or NULL; dir 0 only: the local
 *            experts' row offsets in the expert-major order ([E_loc] = rows).
 *   N * E_loc <= 4096, H a multiple of 8.  Nothing is allocated. */
MOE_API moe_status_t moe_ep_regroup(const void* in, const int32_t* counts, int N, int E_loc,
                                    int rows, int H, int dir, void* out, int32_t* offsets,
                                    moe_stream_t stream);

/* ------------------------------------------ trained router (optional)
 * The pages keep the router frozen by default; these two calls make it
 * trainable.  moe_router_fwd: logits [T, E] fp32 = X [T, H] bf16 times
 * Wr [E, H] bf16 transposed (the router's linear layer; fp32 accumulation
 * on the tensor cores), to feed moe_route_topk.
 * moe_router_bwd, from the routing-weight gradient dw [T, k] (moe_permute's
 * optional output) and the routing of the step (topk_w, topk_idx, dest,
 * expert_offsets): with the kept weights a softmax over the kept logits,
 *   g[t, j] = w[t, j] (dw[t, j] - sum_i w[t, i] dw[t, i])   (dlogits)
 *   dWr[e]  = sum over the rows of expert e of g * Xp[row]     [E, H] fp32
 *   dX[t]   = sum_j dXp[dest[t, j]] + sum_j g[t, j] Wr[topk_idx[t, j]]
 * dX replaces the plain dX combine (moe_unpermute of dXp with w = NULL): both
 * sums are accumulated in fp32 and rounded once to bf16.  dWr sums each
 * expert's rows in order (deterministic).  ws: at least
 * moe_router_bwd_workspace_bytes(T, k) device bytes.  H a multiple of 16
 * (>= 64), 1 <= k <= E <= 512; bf16 pointers 16-byte aligned. */
MOE_API moe_status_t moe_router_fwd(const void* X, const void* Wr, int T, int H, int E,
                                    float* logits, moe_stream_t stream);
MOE_API size_t moe_router_bwd_workspace_bytes(int T, int k);
MOE_API moe_status_t moe_router_bwd(const float* topk_w, const float* dw,
                                    const int32_t* topk_idx, const int32_t* dest,
                                    const int32_t* expert_offsets, const void* Xp,
                                    const void* Wr, const void* dXp, int T, int H, int E,
                                    int k, void* dX, float* dWr, void* ws, size_t ws_bytes,
                                    moe_stream_t stream);

/* ---------------------------------------------------------------- status
 * moe_get_device_status synchronises `stream`, returns the first device-side
 * error recorded since the last call (MOE_OK if none) and clears it.
 * moe_status_string never returns NULL. */
MOE_API moe_status_t moe_get_device_status(moe_stream_t stream);
MOE_API const char* moe_status_string(moe_status_t status);

/* Testing hook: caps every bounded device wait at `ns` nanoseconds (0 restores
 * the default of one second).  A cap of 1 makes the first wait that does not
 * succeed immediately give up, which exercises the timeout path. */
MOE_API void moe_set_wait_limit_ns(uint64_t ns);

/* Testing hook: while on, every grouped-GEMM kernel's MMA warp first waits on
 * a barrier that nothing arrives on.  Its bounded wait runs out after the
 * configured limit; the kernel then records MOE_ERR_DEVICE_TIMEOUT, lets the
 * copies already in flight land, frees its tensor memory and returns.  This
 * exercises the timeout path without faulting or hanging the GPU. */
MOE_API void moe_test_inject_stall(int on);

/* Number of kernels this library has launched in this process (all devices,
 * all streams), counted on the host at each launch; for measurement. */
MOE_API unsigned long long moe_kernel_launches(void);

/* Kernel choice for the four grouped GEMMs (not thread-safe; takes effect at
 * the next moe_lora_mlp_fwd / moe_lora_mlp_bwd call): mode > 0 runs them on
 * CTA pairs (256-row tiles on the 2-SM tensor-core instruction), mode == 0
 * on single CTAs (128-row tiles), mode < 0 (the default) chooses per GEMM:
 * pairs when the mean rows per expert R / E is at least 256 (one 256-row
 * tile; an expert's last tile with at most 128 rows runs as a half tile)
 * and the GEMM's K is at least 768 (H for gate_up forward and down
 * backward, I for down forward, 2I for gate_up backward).  A GEMM on pairs takes its rank-r product (s Xp A1^T,
 * s h A2^T, s dZ2 B2 or s dZ1 B1) from a separate memory-bound pass.  All
 * compute the same result to the tolerance of bf16 rounding. */
MOE_API void moe_set_cta_pairs(int mode);
/* 1 when a grouped GEMM over R routed rows, E experts and reduction length
 * K runs on CTA pairs under the current moe_set_cta_pairs setting (and then
 * takes its rank-r product from the separate pass), else 0; for measurement
 * (the bytes that pass moves). */
MOE_API int moe_uses_cta_pairs(int R, int E, int K);

/* Benchmark hook (not thread-safe; for measurement only).
 * moe_profile_enable(1) starts recording, for every kernel kind below, a pair
 * of CUDA events around each of its launches on the launching stream (up to
 * 512 launches per kind; the counts restart at each enable call);
 * moe_profile_enable(0) stops recording.  moe_profile_collect synchronises on
 * the recorded events and writes the durations (ms) of up to max_n launches
 * of `kind` into ms[], returning how many (or -1 on a CUDA error).  Route
 * covers its four kernels together; MOE_PROF_TRANSPOSE is the one launch
 * that makes the backward's operand copies of the LoRA factors. */
#define MOE_PROF_ROUTE 0
#define MOE_PROF_PERMUTE 1
#define MOE_PROF_GATE_UP_FWD 2
#define MOE_PROF_DOWN_FWD 3
#define MOE_PROF_UNPERMUTE 4
#define MOE_PROF_DOWN_BWD 5
#define MOE_PROF_GATE_UP_BWD 6
#define MOE_PROF_LORA_GRAD 7
#define MOE_PROF_TRANSPOSE 8   /* the factor operand copies (one launch) */
#define MOE_PROF_BASE_GRAD 9
#define MOE_PROF_ROUTER_FWD 10
#define MOE_PROF_ROUTER_BWD 11
#define MOE_PROF_RANK_DOWN 12
#define MOE_PROF_KINDS 13
MOE_API moe_status_t moe_profile_enable(int on);
MOE_API int moe_profile_collect(int kind, float* ms, int max_n);

#ifdef __cplusplus
}
#endif
#endif /* MOE_LORA_H_ */
