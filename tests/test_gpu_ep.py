"""Expert parallelism on the GPU: the CUDA regroup against a segment-loop
reference (bit-exact: it is a row copy), and the whole expert-parallel block
on real kernels with N ranks as threads of one process (``LoopbackHub``:
stream-ordered copies stand in for the all-to-all, so no kernel waits on
another) against the fp64 oracle's single-rank block on the concatenation of
all ranks' tokens."""

import threading

import numpy as np
import pytest
import torch

import oracle as O
from moe_expert_grouped_softmax_b200 import ops
from moe_expert_grouped_softmax_b200.expert_parallel import ExpertParallelBlock, LoopbackHub

from _common import assert_bf16_close, f32

pytestmark = pytest.mark.gpu

NAMES = ("W1", "A1", "B1", "W2", "A2", "B2")


def _segments(c):
    N, EL = c.shape
    src, dst, o = {}, {}, 0
    for s in range(N):
        for e in range(EL):
            src[s, e] = o
            o += int(c[s, e])
    o = 0
    for e in range(EL):
        for s in range(N):
            dst[s, e] = o
            o += int(c[s, e])
    return src, dst, o


@pytest.mark.parametrize("N,EL,H", [(2, 4, 64), (8, 16, 2880), (3, 5, 200), (1, 1, 8)])
def test_ep_regroup_bit_exact_and_round_trip(cuda_ok, N, EL, H):
    g = np.random.default_rng(N * 100 + EL)
    c = g.integers(0, 40, (N, EL)).astype(np.int32)
    c[g.random((N, EL)) < 0.3] = 0                       # empty segments
    src, dst, rows = _segments(c)
    x = torch.randn(rows, H, generator=torch.Generator().manual_seed(3)).to(torch.bfloat16)
    ref = torch.empty_like(x)
    for (s, e), a in src.items():
        n, b = int(c[s, e]), dst[s, e]
        ref[b:b + n] = x[a:a + n]
    counts = torch.from_numpy(c).cuda()
    offs = torch.full((EL + 1,), -7, dtype=torch.int32, device="cuda")
    y = ops.ep_regroup(x.cuda(), counts, 0, offsets=offs)
    assert torch.equal(y.cpu(), ref)
    assert offs.cpu().tolist() == [dst[0, e] for e in range(EL)] + [rows]
    back = ops.ep_regroup(y, counts, 1)
    assert torch.equal(back.cpu(), x)
    assert ops.device_status() == 0


def test_ep_regroup_rejects_inconsistent_counts(cuda_ok):
    c = torch.tensor([[3, 2], [1, 4]], dtype=torch.int32, device="cuda")  # sum 10
    x = torch.zeros((12, 16), dtype=torch.bfloat16, device="cuda")
    out = torch.full_like(x, 5.0)
    ops.ep_regroup(x, c, 0, out=out)
    assert ops.device_status() == 5
    assert bool((out == 5.0).all())                      # nothing written


def _inputs(world, T, H, I, E, k, r):
    g = torch.Generator().manual_seed(77)
    std = 0.05
    W = dict(W1=torch.randn(E, 2 * I, H, generator=g) * std,
             A1=torch.randn(E, r, H, generator=g) * std,
             B1=torch.randn(E, 2 * I, r, generator=g) * std,
             W2=torch.randn(E, H, I, generator=g) * std,
             A2=torch.randn(E, r, I, generator=g) * std,
             B2=torch.randn(E, H, r, generator=g) * std)
    W = {n: v.to(torch.bfloat16) for n, v in W.items()}
    X = torch.randn(world * T, H, generator=g).to(torch.bfloat16)
    L = torch.randn(world * T, E, generator=g)
    dY = torch.randn(world * T, H, generator=g).to(torch.bfloat16)
    return W, X, L, dY


@pytest.mark.parametrize("world", [2, 4])
def test_expert_parallel_block_in_process_ranks(cuda_ok, world):
    T, H, I, E, k, r, s = 300, 256, 128, 8, 2, 16, 2.0
    W, X, L, dY = _inputs(world, T, H, I, E, k, r)
    hub = LoopbackHub(world)
    res, errors = {}, []

    def rank_main(p):
        try:
            blk = ExpertParallelBlock(T, H, I, E, k, r, s, hub.endpoint(p))
            el = blk.E_loc
            Wl = [W[n][blk.e0:blk.e0 + el].contiguous().cuda() for n in NAMES]
            sl = slice(p * T, (p + 1) * T)
            Y = blk.forward(X[sl].cuda(), L[sl].cuda(), Wl)
            dX, grads = blk.backward(dY[sl].cuda(), Wl)
            torch.cuda.synchronize()
            res[p] = (Y.cpu(), dX.cpu(), [t.cpu() for t in grads])
        except BaseException as e:  # release the other ranks, report below
            errors.append(repr(e))
            hub._barrier.abort()

    threads = [threading.Thread(target=rank_main, args=(p,)) for p in range(world)]
    for t in threads:
        t.start()
    for t in threads:
        t.join(timeout=300)
    assert not errors, errors
    assert ops.device_status() == 0
    Wn = [f32(W[n]) for n in NAMES]
    Yref, c = O.block_forward(f32(X), L.numpy(), k, *Wn, s)
    gref = O.block_backward(f32(dY), c)
    el = E // world
    for p in range(world):
        Y, dX, grads = res[p]
        sl = slice(p * T, (p + 1) * T)
        assert_bf16_close(Y, Yref[sl], f"rank {p} Y")
        assert_bf16_close(dX, gref["dX"][sl], f"rank {p} dX")
        for name, got in zip(("dA1", "dB1", "dA2", "dB2"), grads):
            assert_bf16_close(got, gref[name][p * el:(p + 1) * el], f"rank {p} {name}")
