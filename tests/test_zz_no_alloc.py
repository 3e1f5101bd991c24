"""The allocation-free router entry point, through the C ABI.

Callers that cannot allocate device memory when they route (a plugin hook
inside an engine that owns all device memory, or code under a fixed memory
budget) use moe_route_topk_noalloc, whose scratch lives in a fixed array
inside the library.  It must give exactly what moe_route_topk gives, call
after call, even though every call reuses the same scratch.

This file is collected last on purpose; it also passes when run alone.
"""

import ctypes

import numpy as np
import pytest
import torch

from moe_expert_grouped_softmax_b200 import ops

from _common import W_ABS

pytestmark = pytest.mark.gpu


def _noalloc(L):
    f = L.moe_route_topk_noalloc
    P, I = ctypes.c_void_p, ctypes.c_int
    f.argtypes = [P, I, I, I, P, P, P, P, P, P]
    f.restype = I
    L.moe_route_noalloc_max_workspace_bytes.restype = ctypes.c_size_t
    L.moe_route_noalloc_max_workspace_bytes.argtypes = []
    return f


def _outs(T, E, k):
    dev = "cuda"
    return (torch.empty((T, k), dtype=torch.int32, device=dev),
            torch.empty((T, k), dtype=torch.float32, device=dev),
            torch.empty((E,), dtype=torch.int32, device=dev),
            torch.empty((E + 1,), dtype=torch.int32, device=dev),
            torch.empty((T, k), dtype=torch.int32, device=dev))


def _p(t):
    return ctypes.c_void_p(t.data_ptr())


@pytest.mark.parametrize("T,E,k", [(8192, 32, 4), (16384, 128, 8), (777, 256, 8)])
def test_noalloc_route_matches_workspace_route_twice(cuda_ok, T, E, k):
    L = ops.lib()
    f = _noalloc(L)
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    g = torch.Generator(device="cpu").manual_seed(T + E + k)
    for call in range(2):  # two calls in a row share (and reuse) the scratch
        logits = (torch.randn(T, E, generator=g) + 0.5 * call).cuda()
        ref = ops.route_topk(logits, k)
        got = _outs(T, E, k)
        rc = f(_p(logits), T, E, k, *[_p(t) for t in got], stream)
        assert rc == 0, ops.STATUS_NAMES.get(rc, rc)
        torch.cuda.synchronize()
        assert ops.device_status() == 0
        for name, a, b in zip(("idx", "counts", "offsets", "dest"),
                              (got[0], got[2], got[3], got[4]),
                              (ref[0], ref[2], ref[3], ref[4])):
            assert torch.equal(a, b), f"call {call}: {name} differs"
        assert float((got[1] - ref[1]).abs().max()) <= W_ABS


def test_noalloc_route_rejects_sizes_over_its_scratch(cuda_ok):
    L = ops.lib()
    f = _noalloc(L)
    cap = L.moe_route_noalloc_max_workspace_bytes()
    T, E, k = 1 << 20, 64, 8  # needs far more than the fixed scratch
    assert ops.route_workspace_bytes(T, E, k) > cap
    # Real buffers of the full size for these T, E, k (about 0.4 GB), so that
    # even if the size check were lost no kernel could reach past a caller's
    # buffer (the scratch itself is guarded a second time by the workspace
    # check of the routing call this entry point forwards to, which would
    # then return 1): the call must be rejected with 2 before any launch.
    logits = torch.zeros((T, E), dtype=torch.float32, device="cuda")
    got = _outs(T, E, k)
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    assert f(_p(logits), T, E, k, *[_p(t) for t in got], stream) == 2
    torch.cuda.synchronize()
    assert ops.device_status() == 0
