"""Device-side failure detection without faulting the GPU.

* Every wait in the pipelined kernels is bounded.  With the stall hook on,
  each grouped-GEMM kernel (single-CTA or CTA-pair) waits on a barrier that
  nothing arrives on; after
  the (shortened) limit it records MOE_ERR_DEVICE_TIMEOUT, drains its own
  copies and MMAs, frees its tensor memory and returns.  The context must stay
  usable: the next run without the hook is correct.
* Index checks: offsets that are not a partition of [0, R) and destination
  rows out of range are reported as MOE_ERR_DEVICE_BOUNDS and the offending
  access is skipped.
"""

import numpy as np
import pytest
import torch

from moe_expert_grouped_softmax_b200 import ops
from moe_expert_grouped_softmax_b200 import synthetic as S

from _common import assert_bf16_close, oracle_block

pytestmark = pytest.mark.gpu

NAMES = ("W1", "A1", "B1", "W2", "A2", "B2")


def _setup():
    cfg = S.make_config("tiny")
    inp = S.make_inputs(cfg)
    g = {k: (v.cuda() if torch.is_tensor(v) else v) for k, v in inp.items()}
    blk = ops.MoeBlock(cfg["T"], cfg["H"], cfg["I"], cfg["E"], cfg["k"], cfg["r"],
                       cfg["s"])
    return cfg, inp, g, blk


@pytest.mark.parametrize("pairs", [False, True], ids=["single", "pairs"])
def test_wait_timeout_is_reported_and_context_survives(cuda_ok, pairs):
    cfg, inp, g, blk = _setup()
    W = [g[n] for n in NAMES]
    assert ops.device_status() == 0
    ops.set_wait_limit_ns(2_000_000)  # 2 ms
    ops.test_inject_stall(True)
    ops.set_cta_pairs(pairs)
    try:
        blk.step(g["X"], g["logits"], g["dY"], W)
        torch.cuda.synchronize()
        st = ops.device_status()
    finally:
        ops.test_inject_stall(False)
        ops.set_wait_limit_ns(0)
        ops.set_cta_pairs(None)
    assert st == 4, ops.STATUS_NAMES.get(st, st)
    # same process, same context: a normal run is correct
    blk.step(g["X"], g["logits"], g["dY"], W)
    torch.cuda.synchronize()
    assert ops.device_status() == 0
    Y, _, grads = oracle_block(inp, cfg["k"])
    assert_bf16_close(blk.Y, Y, "Y after timeout run")
    assert_bf16_close(blk.dX, grads["dX"], "dX after timeout run")


def test_bad_offsets_are_reported_and_skipped(cuda_ok):
    cfg, inp, g, blk = _setup()
    W = [g[n] for n in NAMES]
    blk.forward(g["X"], g["logits"], W)
    torch.cuda.synchronize()
    bad = blk.offsets.clone()
    bad[-1] += 5                       # no longer ends at R
    sentinel = torch.full_like(blk.Z2, 7.0)
    ops.lora_mlp_fwd(blk.Xp, bad, *W, cfg["s"], out=sentinel)
    torch.cuda.synchronize()
    assert ops.device_status() == 5
    assert torch.all(sentinel == 7.0)  # nothing was written


def test_bad_destination_rows_are_reported_and_skipped(cuda_ok):
    T, H, k = 64, 128, 2
    Yp = torch.randn(T * k, H, device="cuda").to(torch.bfloat16)
    dest = torch.arange(T * k, device="cuda", dtype=torch.int32).view(T, k).contiguous()
    dest[3, 1] = T * k + 100           # out of range
    out = ops.unpermute(Yp, dest, None)
    torch.cuda.synchronize()
    assert ops.device_status() == 5
    ref = Yp.float().view(T, k, H)
    # the bad row is skipped; the others are summed
    assert torch.allclose(out[3].float(), ref[3, 0], atol=1e-2)
    np.testing.assert_allclose(out[5].float().cpu().numpy(),
                               ref[5].sum(0).cpu().numpy(), rtol=1e-2, atol=1e-2)
