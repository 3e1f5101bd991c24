"""Seeded synthetic inputs for the MoE split-LoRA expert block.

This module only draws random numbers: it holds none of the block's own
arithmetic and is shared, as the single input source, by the tests, the
benchmark and the CPU oracle.

Shapes follow the model families benchmarked on the Unsloth page "Fine-tune
MoE LLMs 12x faster with Unsloth" (sections "Kernel results and benchmarks"
and "LoRA in MoE"): gpt-oss-20b (H = I = 2880, 32 experts, top-4),
Qwen3-30B-A3B (H = 2048, I = 768, 128 experts, top-8) and a DeepSeek-V3-shaped
layer (H = 7168, I = 2048, 256 experts, top-8).  No checkpoint or dataset is
used: only the shapes and the value distributions below.

Recipe (every tensor is drawn as fp32 from a seeded ``torch.Generator`` on the
CPU and rounded to bf16 with round-to-nearest-even):

* X ~ N(0, 1) [T, H]; dY ~ N(0, 1) [T, H]
* W1 [E, 2I, H], W2 [E, H, I], A1 [E, r, H], B1 [E, 2I, r], A2 [E, r, I],
  B2 [E, H, r] ~ N(0, 0.02)
* router logits, fp32 [T, E]:
  - ``xwr``: X @ Wr with Wr ~ N(0, 0.02) [H, E] (bf16), accumulated in fp64
    on the host and rounded once to fp32;
  - ``normal``: N(0, 1) per (t, e);
  - ``bias``: N(0, 1) + b_e with b_e ~ N(0, bias_std) drawn once per layer;
  - ``hotcold``: N(0, 1) + b_e where the first ceil(E/10) experts get +beta,
    the last E/16 experts get -30 (so they receive no tokens) and the rest 0;
    beta is found by bisection so that the hot set takes 50% +- 2% of the
    T*k routed (token, slot) pairs.

Each expert slice of a weight tensor, and each 1024-row chunk of X / dY, has
its own seed, so a slice can be regenerated alone (the oracle does this for
sampled experts of the largest layers) and the draws run in parallel threads.
"""

from __future__ import annotations

import math
import os
from concurrent.futures import ThreadPoolExecutor

import numpy as np
import torch

CONFIGS = {
    "tiny": dict(T=512, H=256, I=512, E=8, k=2, r=16, s=2.0,
                 logits="xwr", seed=1001),
    "gpt-oss-20b": dict(T=8192, H=2880, I=2880, E=32, k=4, r=16, s=2.0,
                        logits="normal", seed=1002),
    "qwen3-30b-a3b": dict(T=16384, H=2048, I=768, E=128, k=8, r=32, s=2.0,
                          logits="bias", bias_std=1.5, seed=1003),
    "gpt-oss-20b-long": dict(T=65536, H=2880, I=2880, E=32, k=4, r=16, s=2.0,
                             logits="normal", seed=1004),
    "deepseek-v3": dict(T=8192, H=7168, I=2048, E=256, k=8, r=16, s=2.0,
                        logits="hotcold", seed=1005),
}

WEIGHT_STD = 0.02
_TENSOR_IDS = {"X": 1, "dY": 2, "W1": 3, "A1": 4, "B1": 5, "W2": 6, "A2": 7,
               "B2": 8, "Wr": 9, "logits": 10, "bias": 11}
_ROW_CHUNK = 1024


def make_config(name=None, **over):
    """A config dict by name, with any field overridden."""
    cfg = dict(CONFIGS[name]) if name is not None else {}
    cfg.update(over)
    cfg.setdefault("s", 2.0)
    cfg.setdefault("logits", "normal")
    cfg.setdefault("seed", 1)
    cfg["name"] = name or "custom"
    return cfg


def _seed(cfg_seed, tensor, part):
    return (int(cfg_seed) * 1_000_003 + _TENSOR_IDS[tensor] * 100_003
            + int(part)) % (2 ** 63)


def _randn(shape, std, seed):
    g = torch.Generator().manual_seed(seed)
    t = torch.randn(shape, generator=g, dtype=torch.float32)
    if std != 1.0:
        t.mul_(std)
    return t


def _threads():
    return max(1, min(32, os.cpu_count() or 1))


def expert_slice(cfg, tensor, e):
    """One expert's slice of a weight tensor (bf16), regenerated alone."""
    H, I, r = cfg["H"], cfg["I"], cfg["r"]
    shape = {"W1": (2 * I, H), "A1": (r, H), "B1": (2 * I, r),
             "W2": (H, I), "A2": (r, I), "B2": (H, r)}[tensor]
    return _randn(shape, WEIGHT_STD, _seed(cfg["seed"], tensor, e)).to(
        torch.bfloat16)


def _weight(cfg, tensor, pool):
    E = cfg["E"]
    first = expert_slice(cfg, tensor, 0)
    out = torch.empty((E,) + tuple(first.shape), dtype=torch.bfloat16)
    out[0] = first

    def fill(e):
        out[e] = expert_slice(cfg, tensor, e)

    list(pool.map(fill, range(1, E)))
    return out


def _rows(cfg, tensor, T, H, pool):
    out = torch.empty((T, H), dtype=torch.bfloat16)
    nchunk = (T + _ROW_CHUNK - 1) // _ROW_CHUNK

    def fill(c):
        a = c * _ROW_CHUNK
        b = min(T, a + _ROW_CHUNK)
        out[a:b] = _randn((b - a, H), 1.0, _seed(cfg["seed"], tensor, c)).to(
            torch.bfloat16)

    list(pool.map(fill, range(nchunk)))
    return out


def token_rows(cfg, tensor, rows):
    """Rows of X or dY (bf16) for the given token indices, regenerated alone."""
    rows = np.asarray(rows, dtype=np.int64)
    out = torch.empty((len(rows), cfg["H"]), dtype=torch.bfloat16)
    for c in np.unique(rows // _ROW_CHUNK):
        a = int(c) * _ROW_CHUNK
        b = min(cfg["T"], a + _ROW_CHUNK)
        blk = _randn((b - a, cfg["H"]), 1.0,
                     _seed(cfg["seed"], tensor, int(c))).to(torch.bfloat16)
        sel = np.nonzero(rows // _ROW_CHUNK == c)[0]
        out[torch.from_numpy(sel)] = blk[torch.from_numpy(rows[sel] - a)]
    return out


def _hot_share(L, k, hot):
    top = np.argpartition(-L, k - 1, axis=1)[:, :k]
    return float(np.isin(top, hot).mean())


def make_logits(cfg, X=None):
    """Router logits fp32 [T, E] by the config's recipe (see module doc).

    Returns ``(logits, meta)``; ``meta`` records the drawn bias or beta.
    """
    T, E, k = cfg["T"], cfg["E"], cfg["k"]
    kind = cfg["logits"]
    meta = {"kind": kind}
    if kind == "xwr":
        if X is None:
            raise ValueError("xwr logits need X")
        Wr = _randn((cfg["H"], E), WEIGHT_STD,
                    _seed(cfg["seed"], "Wr", 0)).to(torch.bfloat16)
        L = (X.double().numpy() @ Wr.double().numpy()).astype(np.float32)
        return torch.from_numpy(L), meta
    base = _randn((T, E), 1.0, _seed(cfg["seed"], "logits", 0)).numpy()
    if kind == "normal":
        return torch.from_numpy(base.copy()), meta
    if kind == "bias":
        b = _randn((E,), cfg.get("bias_std", 1.5),
                   _seed(cfg["seed"], "bias", 0)).numpy()
        meta["bias"] = b
        return torch.from_numpy((base + b[None, :]).astype(np.float32)), meta
    if kind == "hotcold":
        n_hot = int(math.ceil(E / 10))
        n_cold = max(1, E // 16)
        hot = np.arange(n_hot)
        bias = np.zeros(E, dtype=np.float32)
        bias[E - n_cold:] = -30.0
        lo, hi = 0.0, 10.0
        beta = hi
        for _ in range(60):
            beta = 0.5 * (lo + hi)
            bias[:n_hot] = beta
            share = _hot_share(base + bias[None, :], k, hot)
            if abs(share - 0.5) <= 0.005:
                break
            if share < 0.5:
                lo = beta
            else:
                hi = beta
        bias[:n_hot] = np.float32(beta)
        L = (base + bias[None, :]).astype(np.float32)
        meta.update(beta=float(np.float32(beta)), n_hot=n_hot, n_cold=n_cold,
                    hot_share=_hot_share(L, k, hot))
        return torch.from_numpy(L), meta
    raise ValueError(f"unknown logits recipe {kind!r}")


def make_inputs(cfg, weights=True, grad_out=True):
    """All inputs of one config as CPU tensors.

    Returns a dict with X, logits (+ ``logits_meta``), W1, A1, B1, W2, A2, B2
    (when ``weights``), dY (when ``grad_out``) and the scalar ``s``.
    """
    T, H = cfg["T"], cfg["H"]
    with ThreadPoolExecutor(_threads()) as pool:
        out = {"s": float(cfg["s"])}
        out["X"] = _rows(cfg, "X", T, H, pool)
        out["logits"], out["logits_meta"] = make_logits(cfg, out["X"])
        if weights:
            for name in ("W1", "A1", "B1", "W2", "A2", "B2"):
                out[name] = _weight(cfg, name, pool)
        if grad_out:
            out["dY"] = _rows(cfg, "dY", T, H, pool)
    return out


def routing_stats(counts):
    """Max/mean load and empty-expert count of an expert histogram."""
    c = np.asarray(counts, dtype=np.float64)
    return dict(max_load=float(c.max()), mean_load=float(c.mean()),
                max_over_mean=float(c.max() / max(c.mean(), 1e-30)),
                empty_experts=int((c == 0).sum()))
