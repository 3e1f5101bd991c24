"""Full-size layers (the shapes of the pages' model families) through the
exact launch configuration the benchmark times (``MoeBlock.step``).

Routing is checked in full (bit-exact against the oracle).  Outputs are
checked on samples the oracle can compute one by one: Y, dX and Z2 on sampled
tokens (each routed row through the fp64 per-expert MLP), and dA / dB on
sampled whole experts (all of their rows), plus exact zeros for every empty
expert.
"""

import numpy as np
import pytest
import torch

import oracle as O
from moe_expert_grouped_softmax_b200 import ops
from moe_expert_grouped_softmax_b200 import synthetic as S

from _common import W_ABS, assert_bf16_close

pytestmark = pytest.mark.gpu

NAMES = ("W1", "A1", "B1", "W2", "A2", "B2")
FULL = ["gpt-oss-20b", "qwen3-30b-a3b", "gpt-oss-20b-long", "deepseek-v3"]
FULL_FT = ("gpt-oss-20b", "qwen3-30b-a3b")   # also run the full fine-tuning backward


def _expert_weights(inp, e):
    return [inp[n][e].double().numpy() for n in NAMES]


@pytest.fixture(scope="module", params=FULL)
def run(request, cuda_ok):
    cfg = S.make_config(request.param)
    inp = S.make_inputs(cfg)
    dev = torch.device("cuda")
    T, H, I, E, k, r, s = (cfg[x] for x in ("T", "H", "I", "E", "k", "r", "s"))
    W = [inp[n].to(dev) for n in NAMES]
    full_ft = request.param in FULL_FT
    blk = ops.MoeBlock(T, H, I, E, k, r, s, device=dev, full_ft=full_ft)
    Xd, dYd = inp["X"].to(dev), inp["dY"].to(dev)
    blk.step(Xd, inp["logits"].to(dev), dYd, W)
    torch.cuda.synchronize()
    status = ops.device_status()
    # the gather and the weighted dY gather are exact copies / one rounding:
    # every routed row, compared on the device
    dflat = blk.dest.long().flatten()
    xp_exact = torch.equal(blk.Xp[dflat], Xd.repeat_interleave(k, dim=0))
    dz2_ref = (dYd.float().repeat_interleave(k, dim=0) * blk.w.flatten()[:, None]).to(torch.bfloat16)
    dz2_exact = torch.equal(blk.dZ2[dflat], dz2_ref)
    del dflat, dz2_ref, Xd, dYd
    names = ["idx", "w", "counts", "offsets", "dest", "Y", "dX", "Z2",
             "dA1", "dB1", "dA2", "dB2"] + (["dW1", "dW2"] if full_ft else [])
    got = {n: getattr(blk, n).cpu() for n in names}
    del W, blk
    torch.cuda.empty_cache()
    # oracle routing on the full logits (cheap) drives the sampling
    ridx, rw = O.route_topk(inp["logits"].numpy(), k)
    rc, ro, rd = O.permutation(ridx, E)
    yield dict(cfg=cfg, inp=inp, got=got, status=status, ridx=ridx, rw=rw, rc=rc,
               ro=ro, rd=rd, xp_exact=xp_exact, dz2_exact=dz2_exact)


def test_status(run):
    assert run["status"] == 0


def test_gathers_exact_full(run):
    """Xp[dest[t, j]] == X[t] and dZ2[dest[t, j]] == bf16(w[t, j] dY[t]) for
    every routed row of the full-size step (the launch configuration the
    benchmark times, row parts included)."""
    assert run["xp_exact"]
    assert run["dz2_exact"]


def test_routing_full(run):
    g = run["got"]
    np.testing.assert_array_equal(g["idx"].numpy(), run["ridx"])
    np.testing.assert_array_equal(g["counts"].numpy(), run["rc"])
    np.testing.assert_array_equal(g["offsets"].numpy(), run["ro"])
    np.testing.assert_array_equal(g["dest"].numpy(), run["rd"])
    assert np.abs(g["w"].double().numpy() - run["rw"]).max() <= W_ABS


def test_sampled_tokens(run):
    """Y[t], dX[t] and the Z2 rows of sampled tokens, row by row."""
    cfg, inp, g = run["cfg"], run["inp"], run["got"]
    T, k, s = cfg["T"], cfg["k"], cfg["s"]
    rng = np.random.default_rng(cfg["seed"])
    n = 16 if cfg["E"] > 64 else 32
    toks = np.unique(np.concatenate([[0, T - 1], rng.choice(T, n, replace=False)]))
    X = inp["X"][toks].double().numpy()
    dY = inp["dY"][toks].double().numpy()
    idx, w, dest = run["ridx"][toks], run["rw"][toks], run["rd"][toks]
    Z2 = np.zeros((len(toks), k, cfg["H"]))
    dXr = np.zeros((len(toks), k, cfg["H"]))
    for e in np.unique(idx):
        W = _expert_weights(inp, int(e))
        ti, jj = np.nonzero(idx == e)
        z, cache = O.expert_forward(X[ti], *W, s)
        dz2 = w[ti, jj][:, None] * dY[ti]
        dx = O.expert_backward(dz2, cache, *W, s)[0]
        Z2[ti, jj] = z
        dXr[ti, jj] = dx
    Y = (w[:, :, None] * Z2).sum(1)
    dX = dXr.sum(1)
    assert_bf16_close(g["Y"][toks], Y, "Y (sampled tokens)")
    assert_bf16_close(g["dX"][toks], dX, "dX (sampled tokens)")
    gz = g["Z2"][torch.as_tensor(dest.reshape(-1))].reshape(len(toks), k, -1)
    assert_bf16_close(gz, Z2, "Z2 rows (sampled tokens)")


def test_sampled_experts_lora_grads(run):
    """dA / dB of whole experts (smallest non-empty, median, largest)."""
    cfg, inp, g = run["cfg"], run["inp"], run["got"]
    k, s = cfg["k"], cfg["s"]
    counts = run["rc"]
    nz = np.nonzero(counts)[0]
    order = nz[np.argsort(counts[nz], kind="stable")]
    picks = sorted({int(order[0]), int(order[len(order) // 2]), int(order[-1])})
    flat_idx = run["ridx"].reshape(-1)
    for e in picks:
        f = np.nonzero(flat_idx == e)[0]          # flat (t, j) in row order
        t, j = f // k, f % k
        W = _expert_weights(inp, e)
        X = inp["X"][torch.as_tensor(t)].double().numpy()
        dY = inp["dY"][torch.as_tensor(t)].double().numpy()
        dz2 = run["rw"][t, j][:, None] * dY
        _, cache = O.expert_forward(X, *W, s)
        _, dA1, dB1, dA2, dB2 = O.expert_backward(dz2, cache, *W, s)
        for name, ref in (("dA1", dA1), ("dB1", dB1), ("dA2", dA2), ("dB2", dB2)):
            assert_bf16_close(g[name][e], ref, f"{name}[expert {e}, {len(f)} rows]")
        if "dW1" in g:
            dW1, dW2 = O.expert_base_grads(dz2, cache)
            assert_bf16_close(g["dW1"][e], dW1, f"dW1[expert {e}, {len(f)} rows]")
            assert_bf16_close(g["dW2"][e], dW2, f"dW2[expert {e}, {len(f)} rows]")


def test_empty_experts_exact_zero(run):
    g = run["got"]
    empty = np.nonzero(run["rc"] == 0)[0]
    for name in ("dA1", "dB1", "dA2", "dB2", "dW1", "dW2"):
        if len(empty) and name in g:
            assert torch.all(g[name][torch.as_tensor(empty)] == 0), name
