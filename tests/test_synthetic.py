"""The seeded input recipe: reproducible, right shapes, right skew."""
import numpy as np
import torch

from moe_expert_grouped_softmax_b200 import synthetic as S


def test_tiny_inputs_reproducible_and_bf16():
    cfg = S.make_config("tiny")
    a = S.make_inputs(cfg)
    b = S.make_inputs(cfg)
    for n in ("X", "W1", "A1", "B1", "W2", "A2", "B2", "dY"):
        assert a[n].dtype == torch.bfloat16
        assert torch.equal(a[n], b[n])
    assert a["logits"].dtype == torch.float32
    assert torch.equal(a["logits"], b["logits"])
    assert a["W1"].shape == (8, 1024, 256) and a["B2"].shape == (8, 256, 16)
    # slices regenerate alone
    assert torch.equal(S.expert_slice(cfg, "W2", 5), a["W2"][5])
    assert torch.equal(S.token_rows(cfg, "X", [3, 511, 0]), a["X"][[3, 511, 0]])
    assert abs(float(a["W1"].float().std()) - 0.02) < 1e-3


def test_deepseek_hot_cold_skew():
    cfg = S.make_config("deepseek-v3")
    L, meta = S.make_logits(cfg)
    assert L.shape == (8192, 256)
    assert abs(meta["hot_share"] - 0.5) <= 0.02
    top = np.argpartition(-L.numpy(), 7, axis=1)[:, :8]
    counts = np.bincount(top.reshape(-1), minlength=256)
    assert (counts[256 - meta["n_cold"]:] == 0).all()


def test_qwen_bias_is_skewed():
    cfg = S.make_config("qwen3-30b-a3b")
    L, meta = S.make_logits(cfg)
    top = np.argpartition(-L.numpy(), 7, axis=1)[:, :8]
    st = S.routing_stats(np.bincount(top.reshape(-1), minlength=128))
    assert st["max_over_mean"] > 3.0
