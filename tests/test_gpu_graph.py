"""A whole fwd+bwd step captured in a CUDA graph and replayed gives the same
bytes as the step launched eagerly (the library allocates nothing and
launches only stream-ordered work, so capture records exactly that work),
and a replay on new input values computes on those values."""

import pytest
import torch

from moe_expert_grouped_softmax_b200 import ops
from moe_expert_grouped_softmax_b200 import synthetic as S

from _common import assert_bf16_close, oracle_block

pytestmark = pytest.mark.gpu

NAMES = ("W1", "A1", "B1", "W2", "A2", "B2")
OUTS = ("Y", "dX", "dA1", "dB1", "dA2", "dB2", "Xp", "Z2", "dZ2", "dXp")


@pytest.mark.parametrize("pairs", [False, True], ids=["single", "pairs"])
def test_graph_replay_matches_eager_step(cuda_ok, pairs):
    cfg = S.make_config("tiny")
    inp = S.make_inputs(cfg)
    g = {k: (v.cuda() if torch.is_tensor(v) else v) for k, v in inp.items()}
    W = [g[n] for n in NAMES]
    args = (cfg["T"], cfg["H"], cfg["I"], cfg["E"], cfg["k"], cfg["r"], cfg["s"])
    ops.set_cta_pairs(pairs)
    try:
        eager = ops.MoeBlock(*args)
        eager.step(g["X"], g["logits"], g["dY"], W)
        X, L, dY = g["X"].clone(), g["logits"].clone(), g["dY"].clone()
        graphed = ops.MoeBlock(*args)
        graphed.capture(X, L, dY, W)
        # clobber the outputs, then replay: the graph must recompute them
        for n in OUTS:
            getattr(graphed, n).fill_(0)
        graphed.replay()
        torch.cuda.synchronize()
        assert ops.device_status() == 0
        for n in OUTS:
            assert torch.equal(getattr(graphed, n), getattr(eager, n)), n
        # new values in the captured input buffers: the replay uses them
        inp2 = S.make_inputs(S.make_config("tiny", seed=4242))
        X.copy_(inp2["X"].cuda())
        L.copy_(inp2["logits"].cuda())
        dY.copy_(inp2["dY"].cuda())
        graphed.replay()
        torch.cuda.synchronize()
    finally:
        ops.set_cta_pairs(None)
    assert ops.device_status() == 0
    inp2.update({n: inp[n] for n in NAMES})  # same weights as captured
    Y, _, grads = oracle_block(inp2, cfg["k"])
    assert_bf16_close(graphed.Y, Y, "Y (replay on new inputs)")
    assert_bf16_close(graphed.dX, grads["dX"], "dX (replay on new inputs)")
    assert_bf16_close(graphed.dA1, grads["dA1"], "dA1 (replay on new inputs)")


def test_forward_and_backward_graphs_match_eager_step(cuda_ok):
    """capture_parts: the forward and the backward as two graphs, replayed in
    turn, give the eager step's bytes."""
    cfg = S.make_config("tiny")
    inp = S.make_inputs(cfg)
    g = {k: (v.cuda() if torch.is_tensor(v) else v) for k, v in inp.items()}
    W = [g[n] for n in NAMES]
    args = (cfg["T"], cfg["H"], cfg["I"], cfg["E"], cfg["k"], cfg["r"], cfg["s"])
    eager = ops.MoeBlock(*args)
    eager.step(g["X"], g["logits"], g["dY"], W)
    parts = ops.MoeBlock(*args)
    parts.capture_parts(g["X"].clone(), g["logits"].clone(), g["dY"].clone(), W)
    for n in OUTS:
        getattr(parts, n).fill_(0)
    parts.replay_forward()
    parts.replay_backward()
    torch.cuda.synchronize()
    assert ops.device_status() == 0
    for n in OUTS:
        assert torch.equal(getattr(parts, n), getattr(eager, n)), n
