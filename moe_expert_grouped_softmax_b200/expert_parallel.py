"""Expert parallelism for the block: the E experts split over N ranks.

Rank p holds the LoRA-adapted weights of experts [p * E_loc, (p + 1) * E_loc)
(E_loc = E / N) and routes its own T tokens over all E experts.  The pages
only say that multi-GPU training is experimental (winningdata.io hands-on
blog, section "Limitações"), so the layout below is this library's own:

forward
  route + permute over all E (one rank's ``moe_route_topk`` / ``moe_permute``):
  the expert-major rows Xp are already ordered by destination rank;
  all-to-all of the per-expert counts, then of the rows;
  ``moe_ep_regroup`` source-major -> expert-major, with the local offsets;
  the local grouped MLP (``moe_lora_mlp_fwd`` with E_loc experts);
  ``moe_ep_regroup`` back to source-major; the return all-to-all; the
  weighted combine on the rank that owns the tokens.
backward
  the weighted dY gather; the same all-to-all and regroup for dZ2; the local
  ``moe_lora_mlp_bwd`` (the LoRA gradients of the local experts are complete
  on their rank: every row routed to an expert is on its owner); dXp back
  through regroup and the all-to-all; the dX combine.

The rows of a local expert come in the order of the source ranks, then of
each source's flat index t * k + j, which is the order one rank routing the
concatenation of all ranks' tokens would give; the block over N ranks
therefore computes what the single-rank block computes on the concatenated
tokens (same routing per token, same rows per expert in the same order).

The exchange is an object with ``rank``, ``world`` and
``all_to_all(out, inp, out_splits, in_splits)`` (rows along dim 0):
``TorchExchange`` (``torch.distributed``: NCCL between GPUs, gloo on CPU
tensors) or ``LoopbackExchange`` (N ranks as threads of one process, sharing
one stream; no kernel waits on another).  ``kernels`` is the C-ABI binding
(``ops``) by default; the row counts of the all-to-alls are read to the host
once per forward (one synchronisation), as ``torch.distributed`` needs them
as Python integers.
"""

import threading

import torch

from . import ops


class TorchExchange:
    """All-to-all over a ``torch.distributed`` process group."""

    def __init__(self, group=None):
        import torch.distributed as dist
        self._dist = dist
        self.group = group
        self.rank = dist.get_rank(group)
        self.world = dist.get_world_size(group)

    def all_to_all(self, out, inp, out_splits, in_splits):
        self._dist.all_to_all_single(out, inp, output_split_sizes=list(out_splits),
                                     input_split_sizes=list(in_splits), group=self.group)


class LoopbackHub:
    """N ranks as threads of one process: each ``all_to_all`` posts this
    rank's input, waits for all ranks, copies its segments from every
    source's input (stream-ordered copies on the shared current stream), and
    waits again so that no input is reused before every rank has copied."""

    def __init__(self, world, timeout=60.0):
        self.world = world
        self._barrier = threading.Barrier(world, timeout=timeout)
        self._posted = [None] * world

    def endpoint(self, rank):
        return LoopbackExchange(self, rank)


class LoopbackExchange:
    def __init__(self, hub, rank):
        self.hub, self.rank, self.world = hub, rank, hub.world

    def all_to_all(self, out, inp, out_splits, in_splits):
        hub = self.hub
        hub._posted[self.rank] = (inp, list(in_splits))
        hub._barrier.wait()
        o = 0
        for s in range(self.world):
            src, splits = hub._posted[s]
            n = splits[self.rank]
            if n != out_splits[s]:
                raise ValueError(f"rank {self.rank}: expected {out_splits[s]} rows from "
                                 f"rank {s}, it sends {n}")
            a = sum(splits[:self.rank])
            if n:
                out[o:o + n].copy_(src[a:a + n])
            o += n
        hub._barrier.wait()


class ExpertParallelBlock:
    """One rank's share of the block under expert parallelism (see the module
    docstring).  ``forward(X, logits, W_local)`` returns Y [T, H] for this
    rank's tokens; ``backward(dY, W_local)`` returns dX [T, H] and the LoRA
    gradients (dA1, dB1, dA2, dB2) of the local experts.  ``W_local`` =
    (W1, A1, B1, W2, A2, B2) of experts [e0, e0 + E_loc)."""

    def __init__(self, T, H, I, E, k, r, s, exchange, kernels=None):
        if E % exchange.world:
            raise ValueError(f"E = {E} experts do not split over {exchange.world} ranks")
        self.T, self.H, self.I, self.E, self.k, self.r, self.s = T, H, I, E, k, r, s
        self.ex = exchange
        self.K = kernels if kernels is not None else ops
        self.N = exchange.world
        self.E_loc = E // self.N
        self.e0 = exchange.rank * self.E_loc

    def _rows(self, like, n):
        return torch.empty((n, like.shape[1]), dtype=like.dtype, device=like.device)

    def forward(self, X, logits, W_local):
        K, ex, N, EL = self.K, self.ex, self.N, self.E_loc
        idx, w, counts, offsets, dest = K.route_topk(logits, self.k)
        Xp = K.permute(X, dest)
        recv_counts = torch.empty_like(counts)
        ex.all_to_all(recv_counts, counts, [EL] * N, [EL] * N)
        send = counts.view(N, EL).sum(1)
        recv = recv_counts.view(N, EL).sum(1)
        send, recv = send.tolist(), recv.tolist()  # the one host synchronisation
        rows = sum(recv)
        Xr = self._rows(Xp, rows)
        ex.all_to_all(Xr, Xp, recv, send)
        rc = recv_counts.view(N, EL)
        offs = torch.empty((EL + 1,), dtype=torch.int32, device=Xp.device)
        Xl = K.ep_regroup(Xr, rc, 0, offsets=offs)
        Z2l, saved = K.lora_mlp_fwd(Xl, offs, *W_local, self.s)
        Z2r = K.ep_regroup(Z2l, rc, 1)
        Z2p = self._rows(Z2l, Xp.shape[0])
        ex.all_to_all(Z2p, Z2r, send, recv)
        Y = K.unpermute(Z2p, dest, w)
        self._ctx = dict(w=w, dest=dest, send=send, recv=recv, rc=rc, offs=offs, Xl=Xl,
                         saved=saved, R=Xp.shape[0])
        return Y

    def backward(self, dY, W_local):
        K, ex, c = self.K, self.ex, self._ctx
        dZ2 = K.permute(dY, c["dest"], scale=c["w"])
        dZ2r = self._rows(dZ2, sum(c["recv"]))
        ex.all_to_all(dZ2r, dZ2, c["recv"], c["send"])
        dZ2l = K.ep_regroup(dZ2r, c["rc"], 0)
        dXl, dA1, dB1, dA2, dB2 = K.lora_mlp_bwd(dZ2l, c["Xl"], c["offs"], *W_local, self.s,
                                                 c["saved"])
        dXr = K.ep_regroup(dXl, c["rc"], 1)
        dXp = self._rows(dXl, c["R"])
        ex.all_to_all(dXp, dXr, c["send"], c["recv"])
        dX = K.unpermute(dXp, c["dest"], None)
        return dX, (dA1, dB1, dA2, dB2)
