"""Trained router on the GPU (optional variant; the pages keep the router
frozen): the logits GEMM against the oracle's X Wr^T, and a whole block with
the router trained against the oracle's router backward.

The top-k choice is an integer decision taken from floating-point logits, so
both sides take it from the same logits: the GPU's (checked first against the
oracle's to fp32 accuracy)."""

import numpy as np
import pytest
import torch

import oracle as O
from moe_expert_grouped_softmax_b200 import ops
from moe_expert_grouped_softmax_b200 import synthetic as S

from _common import assert_bf16_close, f32

pytestmark = pytest.mark.gpu

NAMES = ("W1", "A1", "B1", "W2", "A2", "B2")


def _wr(E, H, seed):
    g = torch.Generator().manual_seed(seed)
    return (torch.randn(E, H, generator=g) * 0.05).to(torch.bfloat16)


@pytest.mark.parametrize("T,H,E", [(1000, 2880, 32), (77, 208, 5), (300, 2048, 128),
                                   (129, 512, 256), (64, 256, 300)])
def test_router_logits(cuda_ok, T, H, E):
    g = torch.Generator().manual_seed(T + E)
    X = torch.randn(T, H, generator=g).to(torch.bfloat16)
    Wr = _wr(E, H, T)
    L = ops.router_fwd(X.cuda(), Wr.cuda())
    torch.cuda.synchronize()
    assert ops.device_status() == 0
    ref = O.router_logits(f32(X), f32(Wr))
    err = np.abs(L.cpu().double().numpy() - ref)
    # fp32 accumulation of exact bf16 products over H terms
    assert err.max() <= 1e-5 * np.abs(ref).max() + 1e-6, err.max()


ROUTER_CASES = {
    "tiny": S.make_config("tiny"),
    "ragged": S.make_config(None, T=77, H=208, I=80, E=5, k=3, r=16, logits="normal", seed=21),
    "qwen_like": S.make_config(None, T=512, H=1024, I=384, E=64, k=8, r=32, logits="normal",
                               seed=22),
}


@pytest.fixture(scope="module", params=list(ROUTER_CASES))
def router_run(request, cuda_ok):
    cfg = ROUTER_CASES[request.param]
    inp = S.make_inputs(cfg)
    T, H, I, E, k, r, s = (cfg[x] for x in ("T", "H", "I", "E", "k", "r", "s"))
    Wr = _wr(E, H, 7 + T)
    dev = torch.device("cuda")
    W = [inp[n].to(dev) for n in NAMES]
    blk = ops.MoeBlock(T, H, I, E, k, r, s, device=dev, train_router=True)
    blk.step(inp["X"].to(dev), None, inp["dY"].to(dev), W, Wr=Wr.to(dev))
    torch.cuda.synchronize()
    status = ops.device_status()
    gl = blk.logits.cpu()
    # the oracle routes on the GPU's logits; everything else is its own fp64
    Wf = [f32(inp[n]) for n in NAMES]
    X = f32(inp["X"])
    Y, ctx = O.block_forward(X, gl.numpy(), k, *Wf, s)
    grads = O.block_backward(f32(inp["dY"]), ctx)
    dl, dWr, dXr = O.router_backward(ctx["w"], grads["dw"], ctx["idx"], X, f32(Wr), E)
    return dict(cfg=cfg, blk=blk, status=status, gl=gl, ctx=ctx, Y=Y, grads=grads, dWr=dWr,
                dX=grads["dX"] + dXr, X=X, Wr=f32(Wr))


def test_router_status(router_run):
    assert router_run["status"] == 0


def test_router_logits_in_block(router_run):
    ref = O.router_logits(router_run["X"], router_run["Wr"])
    err = np.abs(router_run["gl"].double().numpy() - ref)
    assert err.max() <= 1e-5 * np.abs(ref).max() + 1e-6


def test_router_routing_bit_exact(router_run):
    b, ctx = router_run["blk"], router_run["ctx"]
    np.testing.assert_array_equal(b.idx.cpu().numpy(), ctx["idx"])
    np.testing.assert_array_equal(b.dest.cpu().numpy(), ctx["dest"])


def test_router_outputs(router_run):
    b = router_run["blk"]
    assert_bf16_close(b.Y, router_run["Y"], "Y")
    assert_bf16_close(b.dw, router_run["grads"]["dw"], "dw")
    assert_bf16_close(b.dX, router_run["dX"], "dX (experts + router)")
    assert_bf16_close(b.dWr, router_run["dWr"], "dWr")


def test_router_deterministic(router_run):
    b, cfg = router_run["blk"], router_run["cfg"]
    inp = S.make_inputs(cfg)
    dev = torch.device("cuda")
    W = [inp[n].to(dev) for n in NAMES]
    Wr = _wr(cfg["E"], cfg["H"], 7 + cfg["T"]).to(dev)
    first = [t.clone() for t in (b.logits, b.dX, b.dWr)]
    b.step(inp["X"].to(dev), None, inp["dY"].to(dev), W, Wr=Wr)
    for x, y in zip(first, (b.logits, b.dX, b.dWr)):
        assert torch.equal(x, y)
