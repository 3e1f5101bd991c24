"""Shared test helpers: tolerance checks and oracle runs on given inputs."""

from __future__ import annotations

import numpy as np
import torch

import oracle as O

# bf16 outputs and gradients: max|err| <= 2e-2 * max|ref| and rel-L2 <= 5e-3
MAX_REL = 2e-2
L2_REL = 5e-3
W_ABS = 1e-6   # routing weights, fp32 kernel vs fp64 oracle


def errs(got, ref):
    g = torch.as_tensor(got).double().cpu().numpy() if not isinstance(got, np.ndarray) else got.astype(np.float64)
    r = torch.as_tensor(ref).double().cpu().numpy() if not isinstance(ref, np.ndarray) else ref.astype(np.float64)
    d = g - r
    mref = np.abs(r).max() if r.size else 0.0
    nref = np.linalg.norm(r)
    m = float(np.abs(d).max() / mref) if mref > 0 else float(np.abs(d).max() if d.size else 0.0)
    l2 = float(np.linalg.norm(d) / nref) if nref > 0 else float(np.linalg.norm(d))
    return m, l2


def assert_bf16_close(got, ref, name):
    m, l2 = errs(got, ref)
    assert m <= MAX_REL and l2 <= L2_REL, (
        f"{name}: max|err|/max|ref| = {m:.3e} (<= {MAX_REL}), rel-L2 = {l2:.3e} (<= {L2_REL})")
    return m, l2


def f32(t):
    """bf16/fp32 torch tensor -> float32 numpy (exact for bf16)."""
    return t.detach().float().cpu().numpy()


def oracle_block(inp, k, base=False):
    """Full fp64 oracle forward + backward on the given (CPU) inputs (with
    ``base``, also the base-weight gradients dW1, dW2)."""
    W = [f32(inp[n]) for n in ("W1", "A1", "B1", "W2", "A2", "B2")]
    Y, ctx = O.block_forward(f32(inp["X"]), inp["logits"].numpy(), k, *W, inp["s"])
    g = O.block_backward(f32(inp["dY"]), ctx, base=base)
    return Y, ctx, g


def oracle_parts(ctx):
    """Forward intermediates from the oracle's per-expert caches (Z1, h)."""
    R = ctx["Xp"].shape[0]
    W1 = ctx["weights"][0]
    I = np.shape(W1)[1] // 2
    Z1 = np.zeros((R, 2 * I))
    h = np.zeros((R, I))
    off = ctx["offsets"]
    for e, c in enumerate(ctx["caches"]):
        if c is None:
            continue
        a, b = int(off[e]), int(off[e + 1])
        Z1[a:b, :I] = c["g"]
        Z1[a:b, I:] = c["u"]
        h[a:b] = c["h"]
    return Z1, h
