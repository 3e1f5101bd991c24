"""Algorithmic work of one MoE split-LoRA block step (FLOPs and HBM bytes).

These are the denominators of the roofline figures: unique algorithmic work,
not what a kernel happens to move.

FLOP model.  The Unsloth page "Fine-tune MoE LLMs 12x faster with Unsloth",
section "LoRA in MoE", counts one split-LoRA projection of an (m, n) weight
applied to the s tokens of each of k routed experts as
``2 k (s m n + s m r + s r n)``; summed over routed rows R = k*T this is
``2 R (m n + m r + r n)``.  The block has two projections (gate_up: m = H,
n = 2I; down: m = I, n = H).  The backward of a frozen-base split-LoRA
projection does, per routed row, one base product for dX (2 m n) and four
rank-r products (dX's LoRA path 2 (n r + r m), dA 2 r m, dB 2 n r).
"""

from __future__ import annotations


def lora_params_per_projection(m, n, r):
    """Trainable LoRA parameters of one (m, n) projection: r (m + n)."""
    return r * (m + n)


def split_lora_proj_flops(rows, m, n, r):
    """``2 rows (m n + m r + r n)`` for one split-LoRA projection."""
    return 2 * rows * (m * n + m * r + r * n)


def merged_lora_flops(E, rows, m, n, r):
    """Merged (PEFT-style) cost of one projection over E experts:
    ``E (2 m n r + m n) + 2 rows m n``."""
    return E * (2 * m * n * r + m * n) + 2 * rows * m * n


def base_grad_flops(R, H, I):
    """Base-weight gradients of full fine-tuning: dW1 = dZ1^T Xp [2I, H] and
    dW2 = dZ2^T h [H, I] over all routed rows."""
    return 2 * R * (2 * I * H + H * I)


def router_flops(T, H, E, k):
    """Trained router: logits X Wr^T (2 T E H), and from the k kept logits per
    token dWr (2 T k H) and the router's part of dX (2 T k H)."""
    return 2 * T * E * H + 4 * T * k * H


def block_flops(T, H, I, E, k, r, full_ft=False, train_router=False):
    """Forward + backward algorithmic FLOPs of the block (base frozen, or with
    the base-weight gradients when ``full_ft``; with the router's when
    ``train_router``)."""
    R = T * k
    fwd = (split_lora_proj_flops(R, H, 2 * I, r)
           + split_lora_proj_flops(R, I, H, r))
    # backward, per projection (m -> n): dX base 2mn, dX LoRA 2(nr + rm),
    # dA 2rm, dB 2nr
    def bwd(m, n):
        return 2 * R * (m * n + n * r + r * m + r * m + n * r)
    extra = (base_grad_flops(R, H, I) if full_ft else 0) + (
        router_flops(T, H, E, k) if train_router else 0)
    return dict(fwd=fwd, bwd=bwd(H, 2 * I) + bwd(I, H) + extra,
                total=fwd + bwd(H, 2 * I) + bwd(I, H) + extra,
                base_gemm=2 * R * (H * 2 * I + I * H) * 2)


def gemm_flops(R, H, I, r, pairs=(False, False, False, False)):
    """FLOPs of each tensor-core kernel of the block, by kernel.

    ``pairs`` says, for gate_up fwd, down fwd, down bwd and gate_up bwd,
    whether that GEMM ran on CTA pairs: there the rank-r down-projection of
    the GEMM (s Xp A1^T, s h A2^T, s dZ2 B2, s dZ1 B1) is computed by the
    separate rank pass, so its FLOPs are counted under ``rank_down`` (the
    sum over the passes that ran) and not under the GEMM."""
    down_proj = (2 * R * H * r, 2 * R * I * r, 2 * R * H * r, 2 * R * 2 * I * r)
    full = (split_lora_proj_flops(R, H, 2 * I, r),
            split_lora_proj_flops(R, I, H, r),
            2 * R * (H * I + H * r + r * I),          # dh, with LoRA path
            2 * R * (2 * I * H + 2 * I * r + r * H))
    names = ("gate_up_fwd", "down_fwd", "down_bwd", "gate_up_bwd")
    out = {}
    rank = 0
    for n, f, d, p in zip(names, full, down_proj, pairs):
        out[n] = f - d if p else f
        rank += d if p else 0
    if rank:
        out["rank_down"] = rank
    out["lora_grads"] = 2 * R * r * (H + 2 * I + I + H)
    out["base_grad"] = base_grad_flops(R, H, I)
    return out


def hbm_bytes(T, H, E, k):
    """Unique HBM bytes of the memory-bound steps (bf16 activations)."""
    R = T * k
    return dict(
        route=T * E * 4 + T * k * 12 + E * 8,
        permute=T * H * 2 + R * H * 2 + R * 4,
        unpermute=R * H * 2 + T * H * 2 + R * 8,
        dy_gather=T * H * 2 + R * H * 2 + R * 8,
        dx_unpermute=R * H * 2 + T * H * 2 + R * 4,
    )
