"""Plain, slow, fp64 CPU oracle for the MoE split-LoRA expert block.

TEST INFRASTRUCTURE ONLY.  Nothing on the product path imports this module:
only the tests, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` /
``--impl reference`` legs of ``bench.py`` may call it.  It shares no code,
tables or helpers with the CUDA library.

Sources (web pages; cited by title and section):

* [P1] Unsloth docs, "Fine-tune MoE LLMs 12x faster with Unsloth"
  (unsloth.ai/docs/jp/xin-ji-neng/faster-moe).
  - section "What is torch._grouped_mm?": the per-expert loop that gathers the
    tokens routed to one expert and applies ``linear(x, gate_up_proj[e])``
    followed by ``.chunk(2, dim=-1)`` (gate = first half, up = second half),
    and the Transformers-v5 layout ``gate_up_proj = Parameter([E, 2I, H])``.
  - section "Faster LoRA MoE training": split LoRA computes ``X W + (X A) B``
    instead of first materialising the merged ``W + A B``; only the order of
    the products changes (associativity), so outputs, loss and gradients are
    identical.
  - section "Implementation details": a LoRA adapter on an (m, n) weight is a
    pair of (m, r) and (r, n) matrices, the router is not fine-tuned, and the
    recommended ``lora_alpha = 2 r`` gives the standard scale s = alpha / r.
  - the page's opening list of what the kernels support: LoRA and full
    fine-tuning (FFT).  With the base weights trainable, each projection
    ``y = x W^T`` also yields ``dW = dy^T x`` (chain rule; unchanged by the
    split order of the LoRA term).
* [P5] aiflowlearn codex tutorial "Meet Unsloth", section on ``fast_lora.py``
  (``LoRA_MLP``): SwiGLU is ``e = X G; f = e * sigmoid(e); g = X U;
  h = f * g; out = h W``.

Everything is computed in float64 with no intermediate rounding.  Inputs may be
any float dtype; they are widened to float64 on entry.

Readings where the pages are silent (each is listed in the design notes):

* routing: softmax over the E logits of a token, keep the k largest, and
  renormalise the kept probabilities to sum to 1 -- identical to a softmax over
  the k kept logits.  Ties are broken by the lower expert index.
* the routing weight multiplies the expert output after the down projection
  (weighted unpermute / combine); the router is frozen, so logits are an input
  and dX has no path through the router.
* one LoRA adapter on the fused gate_up projection: A1 [E, r, H],
  B1 [E, 2I, r]; one on down: A2 [E, r, I], B2 [E, H, r]; each projection is
  ``y = x W^T + s (x A^T) B^T``.
* permuted order: a stable counting sort of the flat (token, slot) index
  ``t*k + j`` by expert id.

Parity status: every function below is pinned by the ``-m "not gpu"`` tests
(brute force, library special cases, merged-weight identity, dense-MLP special
case, finite differences).  None is "parity unpinned".
"""

from __future__ import annotations

import numpy as np

__all__ = [
    "route_topk",
    "permutation",
    "permute",
    "unpermute",
    "silu",
    "lora_linear",
    "expert_forward",
    "expert_backward",
    "grouped_forward",
    "grouped_backward",
    "expert_base_grads",
    "grouped_base_grads",
    "block_forward",
    "block_backward",
    "router_logits",
    "router_backward",
]


def _f64(a):
    return np.asarray(a, dtype=np.float64)


# --------------------------------------------------------------------------
# router (trainable variant; the pages keep it frozen by default)
# --------------------------------------------------------------------------
def router_logits(X, Wr):
    """The router's linear layer: ``logits = X Wr^T`` [T, E] for Wr [E, H]
    ([P1] "What is torch._grouped_mm?": the gate scores each token against
    every expert before the top-k choice)."""
    return _f64(X) @ _f64(Wr).T


def router_backward(w, dw, idx, X, Wr, E):
    """Gradients through a trained router, from the routing-weight gradient
    ``dw`` [T, k] (of ``<dY, Y>``, see :func:`block_backward`).

    The k kept weights are a softmax over the k kept logits (the selection
    itself is piecewise constant), so for kept slot j of token t
    ``dlogit[t, idx[t, j]] = w_j (dw_j - sum_i w_i dw_i)`` and 0 for the
    experts not kept.  Then ``dWr = dlogit^T X`` [E, H] and the router's part
    of dX is ``dlogit Wr`` [T, H].
    Returns (dlogits [T, E], dWr [E, H], dX_router [T, H]).
    """
    w, dw = _f64(w), _f64(dw)
    T, k = w.shape
    dl = np.zeros((T, E))
    for t in range(T):
        mean = float(w[t] @ dw[t])
        for j in range(k):
            dl[t, int(idx[t, j])] += w[t, j] * (dw[t, j] - mean)
    return dl, dl.T @ _f64(X), dl @ _f64(Wr)


# --------------------------------------------------------------------------
# a1: routing
# --------------------------------------------------------------------------
def route_topk(logits, k):
    """Top-k expert choice per token and renormalised routing weights.

    [P1] "What is torch._grouped_mm?": each token is sent to the experts its
    router selects (``expert_mask``); [P1] "Implementation details": the
    router is frozen, so ``logits`` [T, E] are an input here.

    Selection order is (logit descending, expert index ascending), done with a
    stable sort of the negated logits.  Comparisons of the fp32 logits are
    exact, so the selection does not depend on the precision of any later
    arithmetic.  Weights: ``w_j = exp(l_j - l_max) / sum_sel exp(l - l_max)``
    which equals softmax over all E followed by renormalisation over the k
    kept entries.

    Returns ``idx`` int32 [T, k] and ``w`` float64 [T, k].
    """
    L = _f64(logits)
    T, E = L.shape
    if not 1 <= k <= E:
        raise ValueError("need 1 <= k <= E")
    order = np.argsort(-L, axis=1, kind="stable")
    idx = order[:, :k].astype(np.int32)
    sel = np.take_along_axis(L, idx.astype(np.int64), axis=1)
    lmax = sel[:, :1]
    ex = np.exp(sel - lmax)
    w = ex / ex.sum(axis=1, keepdims=True)
    return idx, w


# --------------------------------------------------------------------------
# permutation (counting sort by expert over the flat index t*k + j)
# --------------------------------------------------------------------------
def permutation(idx, E):
    """Expert histogram, exclusive offsets and destination row of each pair.

    ``counts[e]`` = number of (t, j) with ``idx[t, j] == e``;
    ``offsets`` = exclusive prefix sum of counts, ``offsets[E] = T*k``;
    ``dest[t, j] = offsets[e] + #{(t', j') : t'*k + j' < t*k + j, idx = e}``.

    This is the grouping the per-expert loop of [P1] "What is
    torch._grouped_mm?" performs (all tokens of one expert together, in token
    order), written as a stable counting sort.  A running per-expert counter
    walks the flat index in order.
    """
    idx = np.asarray(idx)
    T, k = idx.shape
    flat = idx.reshape(-1).astype(np.int64)
    if flat.size and (flat.min() < 0 or flat.max() >= E):
        raise ValueError("expert id out of range")
    counts = np.zeros(E, dtype=np.int64)
    for e in flat:
        counts[e] += 1
    offsets = np.zeros(E + 1, dtype=np.int64)
    for e in range(E):
        offsets[e + 1] = offsets[e] + counts[e]
    nxt = offsets[:E].copy()
    dest = np.empty(flat.size, dtype=np.int64)
    for f, e in enumerate(flat):
        dest[f] = nxt[e]
        nxt[e] += 1
    return (counts.astype(np.int32), offsets.astype(np.int32),
            dest.reshape(T, k).astype(np.int32))


# --------------------------------------------------------------------------
# a2 / a6: permute (gather), a5 / a10: unpermute (weighted combine)
# --------------------------------------------------------------------------
def permute(X, dest, scale=None):
    """``Xp[dest[t, j]] = scale[t, j] * X[t]`` (scale = 1 when None)."""
    X = _f64(X)
    dest = np.asarray(dest)
    T, k = dest.shape
    Xp = np.zeros((T * k, X.shape[1]), dtype=np.float64)
    for t in range(T):
        for j in range(k):
            c = 1.0 if scale is None else float(scale[t, j])
            Xp[dest[t, j]] = c * X[t]
    return Xp


def unpermute(Zp, dest, w=None):
    """``Y[t] = sum_j w[t, j] * Zp[dest[t, j]]``, summed in j order."""
    Zp = _f64(Zp)
    dest = np.asarray(dest)
    T, k = dest.shape
    Y = np.zeros((T, Zp.shape[1]), dtype=np.float64)
    for j in range(k):
        c = np.ones(T) if w is None else _f64(w)[:, j]
        Y += c[:, None] * Zp[dest[:, j]]
    return Y


# --------------------------------------------------------------------------
# a3 / a4 / a7 / a8 / a9: one expert's split-LoRA SwiGLU MLP
# --------------------------------------------------------------------------
def sigmoid(x):
    with np.errstate(over="ignore"):
        return 1.0 / (1.0 + np.exp(-x))


def silu(x):
    """[P5] ``fast_lora.py`` SwiGLU: ``f = e * sigmoid(e)``."""
    return x * sigmoid(x)


def lora_linear(X, W, A, B, s):
    """Split-LoRA projection ``X W^T + s (X A^T) B^T``.

    [P1] "Faster LoRA MoE training": the rank-r path is applied to the
    activations (``X A`` then ``(X A) B``) rather than to the weight, so the
    (out, in) matrix ``W + s B A`` is never formed.  Weight layout: W [out, in],
    A [r, in], B [out, r].
    """
    X = _f64(X)
    return X @ _f64(W).T + s * ((X @ _f64(A).T) @ _f64(B).T)


def expert_forward(Xe, W1, A1, B1, W2, A2, B2, s):
    """Forward of one expert on its rows ``Xe`` [M, H].

    gate_up: ``Z1 = Xe W1^T + s (Xe A1^T) B1^T`` [M, 2I]; gate = Z1[:, :I],
    up = Z1[:, I:] ([P1] ``.chunk(2, dim=-1)``); ``h = silu(gate) * up``
    ([P5] SwiGLU); down: ``Z2 = h W2^T + s (h A2^T) B2^T`` [M, H].
    Returns Z2 and a cache for :func:`expert_backward`.
    """
    Xe = _f64(Xe)
    I = _f64(W1).shape[0] // 2
    Z1 = lora_linear(Xe, W1, A1, B1, s)
    g, u = Z1[:, :I], Z1[:, I:]
    h = silu(g) * u
    Z2 = lora_linear(h, W2, A2, B2, s)
    cache = dict(X=Xe, g=g, u=u, h=h)
    return Z2, cache


def expert_backward(dZ2, cache, W1, A1, B1, W2, A2, B2, s):
    """Backward of one expert with the base weights frozen.

    By the chain rule through ``y = x W^T + s (x A^T) B^T``:
    ``dx = dy W + s (dy B) A``, ``dA = s (dy B)^T x``, ``dB = s dy^T (x A^T)``.
    Through SwiGLU: ``dg = dh * u * silu'(g)`` with
    ``silu'(g) = sigmoid(g) (1 + g (1 - sigmoid(g)))`` and ``du = dh * silu(g)``.
    [P1] "Faster LoRA MoE training": the split order leaves these gradients
    equal to those of the merged weight.
    Returns dXe [M, H], dA1 [r, H], dB1 [2I, r], dA2 [r, I], dB2 [H, r].
    """
    dZ2 = _f64(dZ2)
    X, g, u, h = cache["X"], cache["g"], cache["u"], cache["h"]
    W1, A1, B1, W2, A2, B2 = map(_f64, (W1, A1, B1, W2, A2, B2))
    # down projection
    dZB2 = dZ2 @ B2                      # [M, r]
    dh = dZ2 @ W2 + s * (dZB2 @ A2)      # [M, I]
    dA2 = s * (dZB2.T @ h)               # [r, I]
    dB2 = s * (dZ2.T @ (h @ A2.T))       # [H, r]
    # SwiGLU
    sg = sigmoid(g)
    dg = dh * u * sg * (1.0 + g * (1.0 - sg))
    du = dh * g * sg
    dZ1 = np.concatenate([dg, du], axis=1)   # [M, 2I]
    # gate_up projection
    dZB1 = dZ1 @ B1                      # [M, r]
    dX = dZ1 @ W1 + s * (dZB1 @ A1)      # [M, H]
    dA1 = s * (dZB1.T @ X)               # [r, H]
    dB1 = s * (dZ1.T @ (X @ A1.T))       # [2I, r]
    cache["dZ1"] = dZ1                   # for the base-weight gradients
    return dX, dA1, dB1, dA2, dB2


def expert_base_grads(dZ2, cache):
    """Base-weight gradients of one expert when W1, W2 are trainable (full
    fine-tuning, [P1] opening list): for ``y = x W^T``, ``dW = dy^T x``, so
    ``dW2 = dZ2^T h`` [H, I] and ``dW1 = dZ1^T X`` [2I, H].  ``cache`` must have
    been through :func:`expert_backward` (which leaves dZ1 in it)."""
    dZ2 = _f64(dZ2)
    return cache["dZ1"].T @ cache["X"], dZ2.T @ cache["h"]


# --------------------------------------------------------------------------
# grouped over experts (rows of expert e are offsets[e]:offsets[e+1])
# --------------------------------------------------------------------------
def grouped_forward(Xp, offsets, W1, A1, B1, W2, A2, B2, s):
    """Per-expert loop over the permuted rows ([P1] "What is
    torch._grouped_mm?"): expert e owns rows ``offsets[e]:offsets[e+1]``.
    Returns Z2p [R, H] and the per-expert caches."""
    Xp = _f64(Xp)
    E = len(offsets) - 1
    Z2 = np.zeros((Xp.shape[0], _f64(W2[0]).shape[0]), dtype=np.float64)
    caches = []
    for e in range(E):
        a, b = int(offsets[e]), int(offsets[e + 1])
        if b == a:
            caches.append(None)
            continue
        Z2[a:b], c = expert_forward(Xp[a:b], W1[e], A1[e], B1[e],
                                    W2[e], A2[e], B2[e], s)
        caches.append(c)
    return Z2, caches


def grouped_backward(dZ2p, offsets, caches, W1, A1, B1, W2, A2, B2, s):
    """Backward of :func:`grouped_forward`; empty experts get exact zeros."""
    dZ2p = _f64(dZ2p)
    E = len(offsets) - 1
    r, H = np.shape(A1)[1], np.shape(A1)[2]
    I = np.shape(A2)[2]
    dXp = np.zeros((dZ2p.shape[0], H))
    dA1 = np.zeros((E, r, H)); dB1 = np.zeros((E, 2 * I, r))
    dA2 = np.zeros((E, r, I)); dB2 = np.zeros((E, H, r))
    for e in range(E):
        a, b = int(offsets[e]), int(offsets[e + 1])
        if b == a:
            continue
        dXp[a:b], dA1[e], dB1[e], dA2[e], dB2[e] = expert_backward(
            dZ2p[a:b], caches[e], W1[e], A1[e], B1[e], W2[e], A2[e], B2[e], s)
    return dXp, dA1, dB1, dA2, dB2


def grouped_base_grads(dZ2p, offsets, caches, H, I):
    """dW1 [E, 2I, H] and dW2 [E, H, I] over the experts (after
    :func:`grouped_backward` on the same caches); empty experts get exact
    zeros."""
    dZ2p = _f64(dZ2p)
    E = len(offsets) - 1
    dW1 = np.zeros((E, 2 * I, H))
    dW2 = np.zeros((E, H, I))
    for e in range(E):
        a, b = int(offsets[e]), int(offsets[e + 1])
        if b == a:
            continue
        dW1[e], dW2[e] = expert_base_grads(dZ2p[a:b], caches[e])
    return dW1, dW2


# --------------------------------------------------------------------------
# the whole block
# --------------------------------------------------------------------------
def block_forward(X, logits, k, W1, A1, B1, W2, A2, B2, s, route=None):
    """route -> permute -> gate_up+SwiGLU -> down -> weighted unpermute.

    ``route`` may pass a precomputed ``(idx, w)`` (used by finite-difference
    checks on ``w``).  Returns Y [T, H] and a context for
    :func:`block_backward`.
    """
    E = np.shape(W1)[0]
    if route is None:
        idx, w = route_topk(logits, k)
    else:
        idx, w = route
        w = _f64(w)
    counts, offsets, dest = permutation(idx, E)
    Xp = permute(X, dest)
    Z2p, caches = grouped_forward(Xp, offsets, W1, A1, B1, W2, A2, B2, s)
    Y = unpermute(Z2p, dest, w)
    ctx = dict(idx=idx, w=w, counts=counts, offsets=offsets, dest=dest,
               Xp=Xp, Z2p=Z2p, caches=caches,
               weights=(W1, A1, B1, W2, A2, B2), s=s)
    return Y, ctx


def block_backward(dY, ctx, base=False):
    """Gradients of ``<dY, Y>``: dX, dA1, dB1, dA2, dB2 and dw (and, with
    ``base``, the base-weight gradients dW1, dW2).

    weighted dY gather ``dZ2p[dest[t, j]] = w[t, j] dY[t]``;
    ``dw[t, j] = <dY[t], Z2p[dest[t, j]]>``; expert backward;
    ``dX[t] = sum_j dXp[dest[t, j]]``.
    """
    dY = _f64(dY)
    dest, w = ctx["dest"], ctx["w"]
    T, k = dest.shape
    dZ2p = permute(dY, dest, scale=w)
    dw = np.zeros((T, k))
    for t in range(T):
        for j in range(k):
            dw[t, j] = float(dY[t] @ ctx["Z2p"][dest[t, j]])
    W1, A1, B1, W2, A2, B2 = ctx["weights"]
    dXp, dA1, dB1, dA2, dB2 = grouped_backward(
        dZ2p, ctx["offsets"], ctx["caches"], W1, A1, B1, W2, A2, B2, ctx["s"])
    dX = unpermute(dXp, dest, None)
    out = dict(dX=dX, dA1=dA1, dB1=dB1, dA2=dA2, dB2=dB2, dw=dw,
               dZ2p=dZ2p, dXp=dXp)
    if base:
        H, I = np.shape(W2)[1], np.shape(W2)[2]
        out["dW1"], out["dW2"] = grouped_base_grads(dZ2p, ctx["offsets"], ctx["caches"],
                                                    H, I)
    return out
