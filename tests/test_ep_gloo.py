"""Expert parallelism's host logic on CPU with `gloo` ranks.

Each rank runs ``ExpertParallelBlock`` (count and row all-to-alls over
``torch.distributed``, the splits, the regroup directions, the return trip)
with a CPU stand-in for the kernels: the fp64 oracle's own steps (route,
permute, grouped expert MLP and its backward, combine) and a segment-loop
regroup written here.  Each rank's Y and dX, and the LoRA gradients of its
local experts, must equal the oracle's single-rank block on the
concatenation of all ranks' tokens.  (The CUDA regroup and the whole path on
real kernels are checked on the GPU with in-process ranks,
``test_gpu_ep.py``.)
"""

import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import oracle as O  # noqa: E402
from moe_expert_grouped_softmax_b200.expert_parallel import (  # noqa: E402
    ExpertParallelBlock, TorchExchange)

NAMES = ("W1", "A1", "B1", "W2", "A2", "B2")


class CpuKernels:
    """Stand-in for the kernel binding on CPU tensors (fp64 oracle steps)."""

    def route_topk(self, logits, k):
        E = logits.shape[1]
        idx, w = O.route_topk(logits.numpy(), k)
        counts, offsets, dest = O.permutation(idx, E)
        t = lambda a: torch.from_numpy(np.ascontiguousarray(a).astype(np.int32))  # noqa: E731
        return t(idx), torch.from_numpy(w), t(counts), t(offsets), t(dest)

    def permute(self, X, dest, scale=None):
        sc = None if scale is None else scale.numpy()
        return torch.from_numpy(O.permute(X.numpy(), dest.numpy(), scale=sc))

    def unpermute(self, Zp, dest, w=None):
        return torch.from_numpy(O.unpermute(Zp.numpy(), dest.numpy(),
                                            None if w is None else w.numpy()))

    def ep_regroup(self, inp, counts, direction, out=None, offsets=None):
        c = counts.numpy()
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
        out = torch.empty_like(inp)
        for (s, e), a in src.items():
            n, b = int(c[s, e]), dst[s, e]
            if direction == 0:
                out[b:b + n] = inp[a:a + n]
            else:
                out[a:a + n] = inp[b:b + n]
        if offsets is not None:
            for e in range(EL):
                offsets[e] = dst[0, e]
            offsets[EL] = o
        return out

    def lora_mlp_fwd(self, Xl, offs, W1, A1, B1, W2, A2, B2, s):
        Z2, caches = O.grouped_forward(Xl.numpy(), offs.numpy(), W1, A1, B1, W2, A2, B2, s)
        return torch.from_numpy(Z2), caches

    def lora_mlp_bwd(self, dZ2, Xl, offs, W1, A1, B1, W2, A2, B2, s, saved):
        out = O.grouped_backward(dZ2.numpy(), offs.numpy(), saved, W1, A1, B1, W2, A2, B2, s)
        return tuple(torch.from_numpy(np.ascontiguousarray(a)) for a in out)


def _inputs(world, T, H, I, E, k, r, kind):
    g = np.random.default_rng(11)
    W = dict(W1=g.normal(0, 0.3, (E, 2 * I, H)), A1=g.normal(0, 0.3, (E, r, H)),
             B1=g.normal(0, 0.3, (E, 2 * I, r)), W2=g.normal(0, 0.3, (E, H, I)),
             A2=g.normal(0, 0.3, (E, r, I)), B2=g.normal(0, 0.3, (E, H, r)))
    X = g.normal(0, 1, (world * T, H))
    L = g.normal(0, 1, (world * T, E))
    if kind == "skewed":  # no token anywhere picks the last rank's experts
        L[:, E - E // world:] -= 100.0
    dY = g.normal(0, 1, (world * T, H))
    return W, X, L, dY


def _rank_main(rank, world, port, shape, kind, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=__import__("datetime").timedelta(seconds=60))
    try:
        T, H, I, E, k, r, s = shape
        W, X, L, dY = _inputs(world, T, H, I, E, k, r, kind)
        sl = slice(rank * T, (rank + 1) * T)
        ex = TorchExchange()
        blk = ExpertParallelBlock(T, H, I, E, k, r, s, ex, kernels=CpuKernels())
        el = blk.E_loc
        Wl = [W[n][blk.e0:blk.e0 + el] for n in NAMES]
        Y = blk.forward(torch.from_numpy(X[sl]), torch.from_numpy(L[sl]), Wl)
        dX, grads = blk.backward(torch.from_numpy(dY[sl]), Wl)
        q.put((rank, Y.numpy(), dX.numpy(), [g.numpy() for g in grads]))
    finally:
        dist.destroy_process_group()


def _free_port():
    with socket.socket() as sock:
        sock.bind(("127.0.0.1", 0))
        return sock.getsockname()[1]


@pytest.mark.parametrize("world,kind", [(2, "normal"), (2, "skewed"), (4, "normal")])
def test_expert_parallel_block_matches_single_rank_oracle(world, kind):
    shape = (24, 16, 8, 8, 2, 4, 2.0)  # T per rank, H, I, E, k, r, s
    T, H, I, E, k, r, s = shape
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(p, world, port, shape, kind, q))
             for p in range(world)]
    for p in procs:
        p.start()
    res = sorted((q.get(timeout=300) for _ in procs), key=lambda x: x[0])
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    W, X, L, dY = _inputs(world, T, H, I, E, k, r, kind)
    Wn = [W[n] for n in NAMES]
    Yref, c = O.block_forward(X, L, k, *Wn, s)
    gref = O.block_backward(dY, c)
    if kind == "skewed":
        assert int(c["counts"][E - E // world:].sum()) == 0  # the last rank gets no rows
    el = E // world
    for rank, Y, dX, grads in res:
        sl = slice(rank * T, (rank + 1) * T)
        np.testing.assert_allclose(Y, Yref[sl], rtol=1e-12, atol=1e-12)
        np.testing.assert_allclose(dX, gref["dX"][sl], rtol=1e-12, atol=1e-12)
        for name, got in zip(("dA1", "dB1", "dA2", "dB2"), grads):
            np.testing.assert_allclose(got, gref[name][rank * el:(rank + 1) * el],
                                       rtol=1e-12, atol=1e-12, err_msg=name)
