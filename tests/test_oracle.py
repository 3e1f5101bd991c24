"""Pins of the fp64 oracle against things other than itself.

Each test checks the oracle against a fact fixed by the pages or by the
mathematics: brute force on tiny inputs, a library routine that the step
reduces to, the merged-weight identity of split LoRA, the dense SwiGLU MLP
special case, torch autograd and finite differences.
"""

import itertools

import numpy as np
import pytest
import torch

import oracle as O

RNG = np.random.default_rng(12345)


def _params(E, H, I, r, rng, scale=0.3):
    W1 = rng.normal(0, scale, (E, 2 * I, H))
    A1 = rng.normal(0, scale, (E, r, H))
    B1 = rng.normal(0, scale, (E, 2 * I, r))
    W2 = rng.normal(0, scale, (E, H, I))
    A2 = rng.normal(0, scale, (E, r, I))
    B2 = rng.normal(0, scale, (E, H, r))
    return W1, A1, B1, W2, A2, B2


# ---------------------------------------------------------------- routing
def test_route_bruteforce_with_ties():
    """Top-k by (logit desc, index asc) against a full Python sort."""
    rng = np.random.default_rng(7)
    for T, E, k in [(40, 8, 2), (30, 5, 5), (25, 16, 4), (10, 3, 1)]:
        # small integer logits: many exact ties
        L = rng.integers(-2, 3, size=(T, E)).astype(np.float32)
        idx, w = O.route_topk(L, k)
        for t in range(T):
            want = sorted(range(E), key=lambda e: (-float(L[t, e]), e))[:k]
            assert list(idx[t]) == want
        np.testing.assert_allclose(w.sum(1), 1.0, rtol=0, atol=1e-15)


def test_route_weights_equal_renormalised_full_softmax():
    """Softmax over all E then renormalising the kept k == softmax over k."""
    L = RNG.normal(0, 3, (64, 32)).astype(np.float32)
    idx, w = O.route_topk(L, 4)
    L64 = L.astype(np.float64)
    p = np.exp(L64 - L64.max(1, keepdims=True))
    p /= p.sum(1, keepdims=True)
    kept = np.take_along_axis(p, idx.astype(np.int64), 1)
    np.testing.assert_allclose(w, kept / kept.sum(1, keepdims=True),
                               rtol=1e-13, atol=0)
    # weights are in descending order of logit
    assert np.all(np.diff(w, axis=1) <= 1e-15)


def test_route_closed_form():
    L = np.array([[1.0, 3.0, 3.0, 0.0], [0.0, 0.0, 0.0, 0.0],
                  [-1.0, 2.0, 0.0, 2.0 + np.log(3.0)]], dtype=np.float32)
    idx, w = O.route_topk(L, 2)
    assert idx.tolist() == [[1, 2], [0, 1], [3, 1]]
    np.testing.assert_allclose(w[0], [0.5, 0.5], atol=1e-15)
    np.testing.assert_allclose(w[1], [0.5, 0.5], atol=1e-15)
    d = float(np.float32(2.0 + np.log(3.0))) - 2.0
    np.testing.assert_allclose(w[2], [1 / (1 + np.exp(-d)), 1 / (1 + np.exp(d))],
                               atol=1e-15)


def test_route_rejects_bad_k():
    with pytest.raises(ValueError):
        O.route_topk(np.zeros((2, 3), np.float32), 4)


# ---------------------------------------------------------------- permutation
@pytest.mark.parametrize("T,E,k", [(50, 8, 2), (33, 4, 4), (17, 64, 8), (1, 2, 1)])
def test_permutation_is_stable_argsort(T, E, k):
    rng = np.random.default_rng(T * 100 + E)
    L = rng.normal(size=(T, E)).astype(np.float32)
    idx, _ = O.route_topk(L, k)
    counts, offsets, dest = O.permutation(idx, E)
    flat = idx.reshape(-1)
    np.testing.assert_array_equal(counts, np.bincount(flat, minlength=E))
    assert offsets[0] == 0 and offsets[-1] == T * k
    np.testing.assert_array_equal(np.diff(offsets), counts)
    order = np.argsort(flat, kind="stable")      # library counting-sort twin
    inv = np.empty_like(order)
    inv[order] = np.arange(order.size)
    np.testing.assert_array_equal(dest.reshape(-1), inv)


def test_permutation_invariants_skewed():
    T, E, k = 200, 16, 3
    L = RNG.normal(size=(T, E)).astype(np.float32)
    L[:, :3] += 3.0      # hot experts
    L[:, -4:] -= 30.0    # cold experts, never chosen
    idx, _ = O.route_topk(L, k)
    counts, offsets, dest = O.permutation(idx, E)
    assert (counts[-4:] == 0).all()
    d = dest.reshape(-1)
    assert sorted(d.tolist()) == list(range(T * k))      # bijection
    flat = idx.reshape(-1)
    for e in range(E):
        rows = np.nonzero(flat == e)[0]                  # flat order
        got = d[rows]
        assert (got >= offsets[e]).all() and (got < offsets[e + 1]).all()
        assert (np.diff(got) == 1).all()                 # stable: increasing


def test_permute_unpermute_identity():
    T, H, E, k = 37, 24, 6, 3
    X = RNG.normal(size=(T, H))
    L = RNG.normal(size=(T, E)).astype(np.float32)
    idx, w = O.route_topk(L, k)
    _, _, dest = O.permutation(idx, E)
    Xp = O.permute(X, dest)
    np.testing.assert_allclose(O.unpermute(Xp, dest, w), X, rtol=1e-14, atol=1e-14)
    np.testing.assert_array_equal(O.unpermute(Xp, dest, None), k * X)
    idx1, _ = O.route_topk(L, 1)
    _, _, d1 = O.permutation(idx1, E)
    np.testing.assert_array_equal(O.unpermute(O.permute(X, d1), d1,
                                              np.ones((T, 1))), X)


# ---------------------------------------------------------------- forward
def _merged_token_loop(X, L, k, W1, A1, B1, W2, A2, B2, s, route=None):
    """The pages' per-expert loop (expert mask -> token indices -> linear on
    the merged weight -> chunk(2)), written independently of the oracle's
    permutation, with the merged weight W + s B A."""
    T, H = X.shape
    E = W1.shape[0]
    I = W1.shape[1] // 2
    if route is None:
        order = np.argsort(-L.astype(np.float64), axis=1, kind="stable")[:, :k]
        sel = np.take_along_axis(L.astype(np.float64), order, 1)
        p = np.exp(sel - sel.max(1, keepdims=True))
        w = p / p.sum(1, keepdims=True)
    else:
        order, w = route
    Y = np.zeros((T, H))
    mask = np.zeros((E, k, T), bool)
    for t in range(T):
        for j in range(k):
            mask[order[t, j], j, t] = True
    for e in range(E):
        jj, tok = np.where(mask[e])
        if tok.size == 0:
            continue
        W1m = W1[e] + s * B1[e] @ A1[e]
        W2m = W2[e] + s * B2[e] @ A2[e]
        cur = X[tok]
        z = cur @ W1m.T
        gate, up = z[:, :I], z[:, I:]
        out = (gate / (1 + np.exp(-gate)) * up) @ W2m.T
        Y[tok] += w[tok, jj][:, None] * out
    return Y


@pytest.mark.parametrize("T,H,I,E,k,r,s", [(40, 16, 12, 5, 2, 3, 2.0),
                                           (23, 8, 20, 8, 3, 4, 0.7),
                                           (9, 12, 8, 3, 3, 2, 1.3)])
def test_merged_equals_split(T, H, I, E, k, r, s):
    rng = np.random.default_rng(T + H + I)
    X = rng.normal(size=(T, H))
    L = rng.normal(size=(T, E)).astype(np.float32)
    P = _params(E, H, I, r, rng)
    Y, _ = O.block_forward(X, L, k, *P, s)
    Ym = _merged_token_loop(X, L, k, *P, s)
    np.testing.assert_allclose(Y, Ym, rtol=1e-11, atol=1e-11)


def test_dense_swiglu_special_case():
    """E = 1, k = 1: the block is the dense LoRA SwiGLU MLP with weight 1."""
    rng = np.random.default_rng(3)
    T, H, I, r, s = 11, 10, 14, 3, 2.0
    X = rng.normal(size=(T, H))
    W1, A1, B1, W2, A2, B2 = _params(1, H, I, r, rng)
    Y, ctx = O.block_forward(X, np.zeros((T, 1), np.float32), 1,
                             W1, A1, B1, W2, A2, B2, s)
    assert np.all(ctx["w"] == 1.0)
    G = W1[0, :I] + s * B1[0, :I] @ A1[0]
    U = W1[0, I:] + s * B1[0, I:] @ A1[0]
    D = W2[0] + s * B2[0] @ A2[0]
    e = X @ G.T
    f = e * (1 / (1 + np.exp(-e)))
    g = X @ U.T
    np.testing.assert_allclose(Y, (f * g) @ D.T, rtol=1e-12, atol=1e-12)


def test_zero_scale_and_zero_b_give_base_moe():
    rng = np.random.default_rng(5)
    T, H, I, E, k, r = 30, 12, 10, 4, 2, 3
    X = rng.normal(size=(T, H))
    L = rng.normal(size=(T, E)).astype(np.float32)
    W1, A1, B1, W2, A2, B2 = _params(E, H, I, r, rng)
    Z = np.zeros
    base = _merged_token_loop(X, L, k, W1, Z(A1.shape), Z(B1.shape), W2,
                              Z(A2.shape), Z(B2.shape), 0.0)
    Y0, _ = O.block_forward(X, L, k, W1, A1, B1, W2, A2, B2, 0.0)
    Yb, _ = O.block_forward(X, L, k, W1, A1, Z(B1.shape), W2, A2, Z(B2.shape), 2.0)
    np.testing.assert_allclose(Y0, base, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(Yb, base, rtol=1e-12, atol=1e-12)


def test_lora_scale_from_alpha():
    """lora_alpha = 2 r gives s = alpha / r = 2 (the pages' recommended
    setting); the split term with s must equal merging s * B A."""
    rng = np.random.default_rng(11)
    r = 4
    alpha = r * 2
    s = alpha / r
    assert s == 2.0
    X = rng.normal(size=(5, 6))
    W = rng.normal(size=(7, 6))
    A = rng.normal(size=(r, 6))
    B = rng.normal(size=(7, r))
    np.testing.assert_allclose(O.lora_linear(X, W, A, B, s),
                               X @ (W + s * B @ A).T, rtol=1e-12)


# ---------------------------------------------------------------- backward
def _torch_merged_loss(X, w, idx, P, s, dY):
    W1, A1, B1, W2, A2, B2 = P
    T, k = idx.shape
    I = W1.shape[1] // 2
    Y = torch.zeros_like(X)
    rows = []
    for t in range(T):
        acc = torch.zeros(X.shape[1], dtype=X.dtype)
        for j in range(k):
            e = int(idx[t, j])
            z = X[t] @ (W1[e] + s * B1[e] @ A1[e]).T
            g, u = z[:I], z[I:]
            hh = torch.nn.functional.silu(g) * u
            acc = acc + w[t, j] * (hh @ (W2[e] + s * B2[e] @ A2[e]).T)
        rows.append(acc)
    Y = torch.stack(rows)
    return (Y * dY).sum()


def test_backward_matches_torch_autograd_of_merged_weights():
    rng = np.random.default_rng(21)
    T, H, I, E, k, r, s = 14, 10, 6, 4, 2, 3, 1.7
    X = rng.normal(size=(T, H))
    L = rng.normal(size=(T, E)).astype(np.float32)
    P = _params(E, H, I, r, rng)
    dY = rng.normal(size=(T, H))
    _, ctx = O.block_forward(X, L, k, *P, s)
    g = O.block_backward(dY, ctx, base=True)
    tX = torch.tensor(X, requires_grad=True)
    tw = torch.tensor(ctx["w"], requires_grad=True)
    tP = [torch.tensor(p, requires_grad=True) for p in P]
    loss = _torch_merged_loss(tX, tw, ctx["idx"], tP, s, torch.tensor(dY))
    gX, gw, gW1, gA1, gB1, gW2, gA2, gB2 = torch.autograd.grad(
        loss, [tX, tw] + tP)
    # (the merged weight W + sBA has the base-weight gradient of W itself)
    for name, want in [("dX", gX), ("dw", gw), ("dA1", gA1), ("dB1", gB1),
                       ("dA2", gA2), ("dB2", gB2), ("dW1", gW1), ("dW2", gW2)]:
        np.testing.assert_allclose(g[name], want.numpy(), rtol=1e-10,
                                   atol=1e-10, err_msg=name)


def test_backward_finite_differences():
    rng = np.random.default_rng(99)
    T, H, I, E, k, r, s = 8, 6, 5, 4, 2, 3, 1.3
    X = rng.normal(size=(T, H))
    L = rng.normal(size=(T, E)).astype(np.float32)
    P = list(_params(E, H, I, r, rng, scale=0.5))
    dY = rng.normal(size=(T, H))
    _, ctx = O.block_forward(X, L, k, *P, s)
    grads = O.block_backward(dY, ctx, base=True)
    route = (ctx["idx"], ctx["w"])

    def loss(X_, P_, w_=None):
        Y, _ = O.block_forward(X_, L, k, *P_, s,
                               route=(route[0], route[1] if w_ is None else w_))
        return float((Y * dY).sum())

    eps = 1e-6
    # dX: every entry
    fd = np.zeros_like(X)
    for i, j in itertools.product(range(T), range(H)):
        Xp_, Xm_ = X.copy(), X.copy()
        Xp_[i, j] += eps
        Xm_[i, j] -= eps
        fd[i, j] = (loss(Xp_, P) - loss(Xm_, P)) / (2 * eps)
    np.testing.assert_allclose(grads["dX"], fd, rtol=1e-6, atol=1e-7)
    # LoRA matrices and base weights: every entry
    for pi, name in [(1, "dA1"), (2, "dB1"), (4, "dA2"), (5, "dB2"), (0, "dW1"),
                     (3, "dW2")]:
        fd = np.zeros_like(P[pi])
        for ix in np.ndindex(P[pi].shape):
            Pp = [p.copy() for p in P]
            Pm = [p.copy() for p in P]
            Pp[pi][ix] += eps
            Pm[pi][ix] -= eps
            fd[ix] = (loss(X, Pp) - loss(X, Pm)) / (2 * eps)
        np.testing.assert_allclose(grads[name], fd, rtol=1e-6, atol=1e-7,
                                   err_msg=name)
    # routing weight (treated as an input)
    fd = np.zeros_like(ctx["w"])
    for ix in np.ndindex(fd.shape):
        wp, wm = ctx["w"].copy(), ctx["w"].copy()
        wp[ix] += eps
        wm[ix] -= eps
        fd[ix] = (loss(X, P, wp) - loss(X, P, wm)) / (2 * eps)
    np.testing.assert_allclose(grads["dw"], fd, rtol=1e-6, atol=1e-7)


def test_empty_expert_grads_are_exact_zero():
    rng = np.random.default_rng(4)
    T, H, I, E, k, r = 20, 8, 6, 6, 2, 2
    X = rng.normal(size=(T, H))
    L = rng.normal(size=(T, E)).astype(np.float32)
    L[:, 4:] = -30.0
    P = _params(E, H, I, r, rng)
    _, ctx = O.block_forward(X, L, k, *P, 2.0)
    g = O.block_backward(rng.normal(size=(T, H)), ctx, base=True)
    assert (ctx["counts"][4:] == 0).all()
    for n in ("dA1", "dB1", "dA2", "dB2", "dW1", "dW2"):
        assert np.all(g[n][4:] == 0.0)
        assert np.any(g[n][:4] != 0.0)


def test_base_grads_dense_closed_form():
    """E = 1, k = 1: dW2 = (w dY)^T h and dW1 = dZ1^T X over all tokens, with
    h and dZ1 from the textbook SwiGLU chain written out here."""
    rng = np.random.default_rng(31)
    T, H, I, r, s = 9, 7, 5, 2, 1.5
    X = rng.normal(size=(T, H))
    L = np.zeros((T, 1), dtype=np.float32)
    W1, A1, B1, W2, A2, B2 = _params(1, H, I, r, rng)
    dY = rng.normal(size=(T, H))
    _, ctx = O.block_forward(X, L, 1, W1, A1, B1, W2, A2, B2, s)
    g = O.block_backward(dY, ctx, base=True)
    M1 = W1[0] + s * B1[0] @ A1[0]
    M2 = W2[0] + s * B2[0] @ A2[0]
    Z = X @ M1.T
    gate, up = Z[:, :I], Z[:, I:]
    sig = 1.0 / (1.0 + np.exp(-gate))
    h = gate * sig * up
    dh = dY @ M2
    dZ1 = np.concatenate([dh * up * (sig + gate * sig * (1 - sig)), dh * gate * sig], axis=1)
    np.testing.assert_allclose(g["dW2"][0], dY.T @ h, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(g["dW1"][0], dZ1.T @ X, rtol=1e-12, atol=1e-12)


# ---------------------------------------------------------------- trained router
def _router_case(seed=41):
    rng = np.random.default_rng(seed)
    T, H, I, E, k, r, s = 10, 7, 5, 5, 2, 2, 1.4
    X = rng.normal(size=(T, H))
    Wr = rng.normal(size=(E, H))
    P = list(_params(E, H, I, r, rng, scale=0.5))
    dY = rng.normal(size=(T, H))
    return X, Wr, P, dY, k, s


def _router_loss(X, Wr, P, dY, k, s, route=None):
    L = O.router_logits(X, Wr)
    Y, ctx = O.block_forward(X, L, k, *P, s, route=route)
    return float((Y * dY).sum()), ctx, L


def test_router_backward_matches_torch_autograd():
    """logits = X Wr^T, top-k by torch.topk (no gradient through the choice),
    softmax over the kept logits, merged-weight experts; autograd gives dX
    (expert + router paths) and dWr."""
    X, Wr, P, dY, k, s = _router_case()
    E = Wr.shape[0]
    _, ctx, L = _router_loss(X, Wr, P, dY, k, s)
    g = O.block_backward(dY, ctx)
    dl, dWr, dXr = O.router_backward(ctx["w"], g["dw"], ctx["idx"], X, Wr, E)
    tX = torch.tensor(X, requires_grad=True)
    tWr = torch.tensor(Wr, requires_grad=True)
    tP = [torch.tensor(p) for p in P]
    logits = tX @ tWr.T
    idx = torch.topk(logits.detach(), k, dim=1).indices
    assert np.array_equal(np.sort(idx.numpy(), 1), np.sort(ctx["idx"], 1))
    tw = torch.softmax(torch.gather(logits, 1, idx), dim=1)
    loss = _torch_merged_loss(tX, tw, idx.numpy(), tP, s, torch.tensor(dY))
    gX, gWr = torch.autograd.grad(loss, [tX, tWr])
    np.testing.assert_allclose(g["dX"] + dXr, gX.numpy(), rtol=1e-10, atol=1e-10)
    np.testing.assert_allclose(dWr, gWr.numpy(), rtol=1e-10, atol=1e-10)


def test_router_backward_finite_differences():
    """Central differences of <dY, Y> in every logit (top-k set unchanged by
    the step) and every router weight."""
    X, Wr, P, dY, k, s = _router_case(43)
    E = Wr.shape[0]
    _, ctx, L = _router_loss(X, Wr, P, dY, k, s)
    g = O.block_backward(dY, ctx)
    dl, dWr, _ = O.router_backward(ctx["w"], g["dw"], ctx["idx"], X, Wr, E)
    eps = 1e-6

    def loss_L(L_):
        Y, c = O.block_forward(X, L_, k, *P, s)
        assert np.array_equal(c["idx"], ctx["idx"])
        return float((Y * dY).sum())

    fd = np.zeros_like(L)
    for ix in np.ndindex(L.shape):
        Lp, Lm = L.copy(), L.copy()
        Lp[ix] += eps
        Lm[ix] -= eps
        fd[ix] = (loss_L(Lp) - loss_L(Lm)) / (2 * eps)
    np.testing.assert_allclose(dl, fd, rtol=1e-6, atol=1e-7)
    fd = np.zeros_like(Wr)
    for ix in np.ndindex(Wr.shape):
        Wp, Wm = Wr.copy(), Wr.copy()
        Wp[ix] += eps
        Wm[ix] -= eps
        fd[ix] = (_router_loss(X, Wp, P, dY, k, s)[0] - _router_loss(X, Wm, P, dY, k, s)[0]) / (2 * eps)
    np.testing.assert_allclose(dWr, fd, rtol=1e-6, atol=1e-7)


def test_router_gradient_zero_for_unselected_and_sums_to_zero():
    """Unselected experts get no logit gradient; a shift of all kept logits
    of a token leaves its weights unchanged, so each row of dlogits sums to 0."""
    X, Wr, P, dY, k, s = _router_case(47)
    E = Wr.shape[0]
    _, ctx, _ = _router_loss(X, Wr, P, dY, k, s)
    g = O.block_backward(dY, ctx)
    dl, _, _ = O.router_backward(ctx["w"], g["dw"], ctx["idx"], X, Wr, E)
    for t in range(X.shape[0]):
        kept = set(int(e) for e in ctx["idx"][t])
        for e in range(E):
            if e not in kept:
                assert dl[t, e] == 0.0
    np.testing.assert_allclose(dl.sum(1), 0.0, atol=1e-12)
