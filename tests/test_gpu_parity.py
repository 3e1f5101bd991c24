"""GPU path vs the fp64 oracle on the same seeded inputs (small shapes that
span several tiles and ragged tails).  All calls go through the C ABI."""

import numpy as np
import pytest
import torch

import oracle as O
from moe_expert_grouped_softmax_b200 import ops
from moe_expert_grouped_softmax_b200 import synthetic as S

from _common import W_ABS, assert_bf16_close, errs, f32, oracle_block, oracle_parts

pytestmark = pytest.mark.gpu

DEV = "cuda"


def _cuda(inp):
    return {k: (v.to(DEV) if torch.is_tensor(v) else v) for k, v in inp.items()}


def _weights(g):
    return [g[n] for n in ("W1", "A1", "B1", "W2", "A2", "B2")]


# ------------------------------------------------------------------ routing
ROUTE_CASES = [
    dict(T=512, E=8, k=2, kind="xwr"),
    dict(T=1000, E=32, k=4, kind="normal"),
    dict(T=777, E=128, k=8, kind="bias"),
    dict(T=300, E=256, k=8, kind="hotcold"),
    dict(T=129, E=512, k=16, kind="normal"),
    dict(T=64, E=5, k=5, kind="normal"),
    dict(T=33, E=1, k=1, kind="normal"),
    dict(T=3000, E=64, k=1, kind="normal"),
]


@pytest.mark.parametrize("case", ROUTE_CASES, ids=lambda c: f"T{c['T']}E{c['E']}k{c['k']}")
def test_route_bit_exact(cuda_ok, case):
    cfg = S.make_config(None, T=case["T"], H=64, I=64, E=case["E"], k=case["k"], r=16,
                        logits=case["kind"], seed=7 + case["T"])
    X = torch.randn(case["T"], 64, generator=torch.Generator().manual_seed(1)).to(torch.bfloat16)
    L, _ = S.make_logits(cfg, X)
    idx, w, counts, offsets, dest = ops.route_topk(L.to(DEV), case["k"])
    ridx, rw = O.route_topk(L.numpy(), case["k"])
    rc, ro, rd = O.permutation(ridx, case["E"])
    np.testing.assert_array_equal(idx.cpu().numpy(), ridx)
    np.testing.assert_array_equal(counts.cpu().numpy(), rc)
    np.testing.assert_array_equal(offsets.cpu().numpy(), ro)
    np.testing.assert_array_equal(dest.cpu().numpy(), rd)
    assert np.abs(w.cpu().double().numpy() - rw).max() <= W_ABS
    assert ops.device_status() == 0


def test_route_ties(cuda_ok):
    g = torch.Generator().manual_seed(3)
    L = torch.randint(-2, 3, (2000, 16), generator=g).float()
    idx, w, counts, offsets, dest = ops.route_topk(L.to(DEV), 4)
    ridx, rw = O.route_topk(L.numpy(), 4)
    rc, ro, rd = O.permutation(ridx, 16)
    np.testing.assert_array_equal(idx.cpu().numpy(), ridx)
    np.testing.assert_array_equal(dest.cpu().numpy(), rd)
    assert np.abs(w.cpu().double().numpy() - rw).max() <= W_ABS


def test_route_deterministic(cuda_ok):
    L = torch.randn(5000, 64).to(DEV)
    a = [t.clone() for t in ops.route_topk(L, 6)]
    b = ops.route_topk(L, 6)
    for x, y in zip(a, b):
        assert torch.equal(x, y)


def test_route_empty_tokens(cuda_ok):
    L = torch.zeros((0, 8), device=DEV)
    _, _, counts, offsets, _ = ops.route_topk(L, 2)
    assert counts.cpu().tolist() == [0] * 8 and offsets.cpu().tolist() == [0] * 9


# ------------------------------------------------------------------ permute / combine
def test_permute_and_combine(cuda_ok):
    T, H, E, k = 301, 200, 8, 3
    g = torch.Generator().manual_seed(5)
    X = torch.randn(T, H, generator=g).to(torch.bfloat16)
    L = torch.randn(T, E, generator=g)
    Z = torch.randn(T * k, H, generator=g).to(torch.bfloat16)
    dY = torch.randn(T, H, generator=g).to(torch.bfloat16)
    idx, w, counts, offsets, dest = ops.route_topk(L.to(DEV), k)
    Xp = ops.permute(X.to(DEV), dest)
    rdest = dest.cpu().numpy()
    # the copy is exact
    np.testing.assert_array_equal(f32(Xp), O.permute(f32(X), rdest).astype(np.float32))
    rw = w.cpu().double().numpy()
    # weighted gather (+ routing-weight gradient)
    Sg, dw = ops.permute(dY.to(DEV), dest, scale=w, Zp=Z.to(DEV))
    assert_bf16_close(Sg, O.permute(f32(dY), rdest, scale=rw), "scaled gather")
    ref_dw = np.array([[f32(dY)[t].astype(np.float64) @ f32(Z)[rdest[t, j]] for j in range(k)]
                       for t in range(T)])
    assert_bf16_close(dw, ref_dw, "dw")
    # weighted combine and plain combine
    Y = ops.unpermute(Z.to(DEV), dest, w)
    assert_bf16_close(Y, O.unpermute(f32(Z), rdest, rw), "combine")
    Y1 = ops.unpermute(Z.to(DEV), dest, None)
    assert_bf16_close(Y1, O.unpermute(f32(Z), rdest, None), "combine w=1")
    # permute then combine with the routing weights returns X (sum w = 1)
    assert_bf16_close(ops.unpermute(Xp, dest, w), f32(X), "combine(permute(X))")
    assert ops.device_status() == 0


@pytest.mark.parametrize("H", [2048, 2880, 4104])
def test_permute_and_combine_row_parts(cuda_ok, H):
    """Few tokens and long rows: the gather splits each row into parts (one
    warp per part); results are those of whole rows.  H = 4104 (513 vectors)
    gives the combine a last pass that only some lanes' vectors reach, while
    its shuffles still need the whole warp."""
    T, E, k = 333, 16, 4
    g = torch.Generator().manual_seed(H)
    X = torch.randn(T, H, generator=g).to(torch.bfloat16)
    L = torch.randn(T, E, generator=g)
    Z = torch.randn(T * k, H, generator=g).to(torch.bfloat16)
    dY = torch.randn(T, H, generator=g).to(torch.bfloat16)
    idx, w, counts, offsets, dest = ops.route_topk(L.to(DEV), k)
    rdest = dest.cpu().numpy()
    rw = w.cpu().double().numpy()
    Xp = ops.permute(X.to(DEV), dest)
    np.testing.assert_array_equal(f32(Xp), O.permute(f32(X), rdest).astype(np.float32))
    Sg = ops.permute(dY.to(DEV), dest, scale=w)
    ref = (dY.float().repeat_interleave(k, 0) * w.cpu().flatten()[:, None]).to(torch.bfloat16)
    assert torch.equal(Sg.cpu()[torch.as_tensor(rdest.reshape(-1), dtype=torch.long)], ref)
    assert_bf16_close(ops.unpermute(Z.to(DEV), dest, w), O.unpermute(f32(Z), rdest, rw),
                      "combine")
    assert_bf16_close(ops.unpermute(Z.to(DEV), dest, None), O.unpermute(f32(Z), rdest, None),
                      "combine w=1")
    assert ops.device_status() == 0


# ------------------------------------------------------------------ expert MLP + block
BLOCK_CASES = {
    "tiny": S.make_config("tiny"),
    # ragged everything: K tails (H % 64 != 0), N tails (I % 96 != 0), few rows
    "ragged": S.make_config(None, T=77, H=208, I=80, E=5, k=3, r=16, logits="normal", seed=11),
    "rank32": S.make_config(None, T=300, H=256, I=384, E=16, k=4, r=32, logits="bias",
                            bias_std=1.5, seed=12),
    "rank64": S.make_config(None, T=200, H=192, I=256, E=6, k=2, r=64, logits="normal", seed=13),
    "dense": S.make_config(None, T=150, H=128, I=192, E=1, k=1, r=16, logits="normal", seed=14),
    "skew_empty": S.make_config(None, T=400, H=128, I=128, E=32, k=2, r=16, logits="hotcold",
                                seed=15),
    "many_tiles": S.make_config(None, T=1024, H=512, I=384, E=4, k=2, r=16, logits="normal",
                                seed=16),
}


# every case forced onto the single-CTA GEMM kernels, and again ("/pairs")
# onto the CTA-pair GEMM kernels (the default chooses between them per GEMM
# from the rows per expert and K)
BLOCK_RUNS = [(c, False) for c in BLOCK_CASES] + [(c, True) for c in BLOCK_CASES]


@pytest.fixture(scope="module", params=BLOCK_RUNS,
                ids=lambda p: p[0] + ("/pairs" if p[1] else ""))
def block_run(request, cuda_ok):
    name, pairs = request.param
    cfg = BLOCK_CASES[name]
    inp = S.make_inputs(cfg)
    Y, ctx, grads = oracle_block(inp, cfg["k"], base=True)
    g = _cuda(inp)
    # the full fine-tuning backward: the LoRA outputs plus dW1, dW2 (the
    # LoRA-only entry point is checked against it bit for bit below)
    blk = ops.MoeBlock(cfg["T"], cfg["H"], cfg["I"], cfg["E"], cfg["k"], cfg["r"], cfg["s"],
                       with_dw=True, full_ft=True)
    W = _weights(g)
    ops.set_cta_pairs(pairs)
    try:
        blk.step(g["X"], g["logits"], g["dY"], W)
        torch.cuda.synchronize()
    finally:
        ops.set_cta_pairs(None)
    status = ops.device_status()
    return dict(name=name, pairs=pairs, cfg=cfg, inp=inp, Y=Y, ctx=ctx, grads=grads,
                blk=blk, status=status)


def test_block_status(block_run):
    assert block_run["status"] == 0


def test_block_routing(block_run):
    b, ctx = block_run["blk"], block_run["ctx"]
    np.testing.assert_array_equal(b.idx.cpu().numpy(), ctx["idx"])
    np.testing.assert_array_equal(b.offsets.cpu().numpy(), ctx["offsets"])
    np.testing.assert_array_equal(b.dest.cpu().numpy(), ctx["dest"])


def test_block_forward_parts(block_run):
    b, ctx, cfg = block_run["blk"], block_run["ctx"], block_run["cfg"]
    R, H, I, r, s = b.R, cfg["H"], cfg["I"], cfg["r"], cfg["s"]
    Z1, h = oracle_parts(ctx)
    gZ1, gh, gxa, gha = ops.saved_views(b.saved, R, H, I, r)
    assert_bf16_close(gZ1[:, :I], Z1[:, :I], "gate")
    assert_bf16_close(gZ1[:, I:], Z1[:, I:], "up")
    assert_bf16_close(gh, h, "h")
    # s * (Xp A1^T) and s * (h A2^T) per expert, transposed
    A1 = f32(block_run["inp"]["A1"]).astype(np.float64)
    A2 = f32(block_run["inp"]["A2"]).astype(np.float64)
    off = ctx["offsets"]
    xa = np.zeros((R, r))
    ha = np.zeros((R, r))
    for e in range(cfg["E"]):
        a, bb = int(off[e]), int(off[e + 1])
        xa[a:bb] = s * ctx["Xp"][a:bb] @ A1[e].T
        ha[a:bb] = s * h[a:bb] @ A2[e].T
    assert_bf16_close(gxa[:, :R].T, xa, "s*Xp*A1^T")
    assert_bf16_close(gha[:, :R].T, ha, "s*h*A2^T")
    assert_bf16_close(b.Z2, ctx["Z2p"], "Z2")


def test_block_outputs(block_run):
    b, g = block_run["blk"], block_run["grads"]
    assert_bf16_close(b.Y, block_run["Y"], "Y")
    assert_bf16_close(b.dZ2, g["dZ2p"], "dZ2 (weighted gather)")
    assert_bf16_close(b.dXp, g["dXp"], "dXp")
    assert_bf16_close(b.dX, g["dX"], "dX")
    assert_bf16_close(b.dw, g["dw"], "dw")


@pytest.mark.parametrize("name", ["dA1", "dB1", "dA2", "dB2"])
def test_block_lora_grads(block_run, name):
    b, g, ctx = block_run["blk"], block_run["grads"], block_run["ctx"]
    got = getattr(b, name)
    assert_bf16_close(got, g[name], name)
    empty = np.nonzero(ctx["counts"] == 0)[0]
    if len(empty):
        assert torch.all(got[torch.as_tensor(empty, device=got.device)] == 0)


@pytest.mark.parametrize("name", ["dW1", "dW2"])
def test_block_base_grads(block_run, name):
    """Full fine-tuning: dW1 = dZ1^T Xp and dW2 = dZ2^T h per expert."""
    b, g, ctx = block_run["blk"], block_run["grads"], block_run["ctx"]
    got = getattr(b, name)
    assert_bf16_close(got, g[name], name)
    empty = np.nonzero(ctx["counts"] == 0)[0]
    if len(empty):
        assert torch.all(got[torch.as_tensor(empty, device=got.device)] == 0)


def test_block_lora_only_entry_point_matches(block_run):
    """moe_lora_mlp_bwd (base weights frozen) gives bit-identical LoRA
    gradients and dX to the full fine-tuning entry point."""
    cfg, b = block_run["cfg"], block_run["blk"]
    g = _cuda(block_run["inp"])
    W = _weights(g)
    lo = ops.MoeBlock(cfg["T"], cfg["H"], cfg["I"], cfg["E"], cfg["k"], cfg["r"], cfg["s"])
    ops.set_cta_pairs(block_run["pairs"])
    try:
        lo.step(g["X"], g["logits"], g["dY"], W)
        torch.cuda.synchronize()
    finally:
        ops.set_cta_pairs(None)
    assert ops.device_status() == 0
    for n in ("Y", "dX", "dA1", "dB1", "dA2", "dB2"):
        assert torch.equal(getattr(lo, n), getattr(b, n)), n


def test_block_deterministic(block_run):
    b = block_run["blk"]
    g = _cuda(block_run["inp"])
    W = _weights(g)
    first = [t.clone() for t in (b.Y, b.dX, b.dA1, b.dB1, b.dA2, b.dB2, b.dW1, b.dW2)]
    ops.set_cta_pairs(block_run["pairs"])
    try:
        b.step(g["X"], g["logits"], g["dY"], W)
    finally:
        ops.set_cta_pairs(None)
    for x, y in zip(first, (b.Y, b.dX, b.dA1, b.dB1, b.dA2, b.dB2, b.dW1, b.dW2)):
        assert torch.equal(x, y)
