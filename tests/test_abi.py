"""The C ABI library: it loads without a GPU, exports every declared entry
point, sizes its buffers sensibly, and rejects bad arguments on the host
before launching anything."""

import ctypes
import os
import re

import pytest

from moe_expert_grouped_softmax_b200 import build, ops

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def L():
    build.build()
    return ops.lib()


def _declared():
    names = []
    inc = os.path.join(ROOT, "include")
    for f in sorted(os.listdir(inc)):
        if f.endswith(".h"):
            src = open(os.path.join(inc, f)).read()
            names += re.findall(r"MOE_API\s+[\w\s\*]+?\b(moe_\w+)\s*\(", src)
    return names


def test_every_declared_symbol_is_exported(L):
    names = _declared()
    assert len(names) >= 12
    for n in names:
        assert hasattr(L, n), n
    assert set(ops.EXPORTS) <= set(names)


def test_status_strings(L):
    for code in range(6):
        assert L.moe_status_string(code)
    assert L.moe_status_string(99) == b"unknown status"


def test_sizes(L):
    R, H, I, r = 1000, 256, 512, 16
    sb = L.moe_saved_bytes(R, H, I, r)
    assert sb >= R * 2 * I * 2 + R * I * 2 + 2 * r * 1024 * 2
    offs = [L.moe_saved_part_offset(R, H, I, r, p) for p in range(7)]
    assert offs == sorted(offs) and offs[0] == 0 and offs[6] == sb
    assert offs[5] - offs[4] >= R * r * 2 and sb - offs[5] >= R * r * 2
    assert all(o % 256 == 0 for o in offs)
    assert L.moe_workspace_bytes(R, 8, H, I, r) >= R * 2 * I * 2
    assert L.moe_route_workspace_bytes(512, 8, 2) >= 512 * 2 * 4


def test_cta_pair_choice(L):
    """The grouped-GEMM kernel choice is host logic: pairs from 256 rows per
    expert and K >= 768 by default, forced either way by moe_set_cta_pairs."""
    try:
        assert L.moe_uses_cta_pairs(32768, 32, 2880) == 1      # gpt-oss-20b shape
        assert L.moe_uses_cta_pairs(65536, 256, 2048) == 1     # 256 rows per expert
        assert L.moe_uses_cta_pairs(131072, 128, 768) == 1     # K = 768
        assert L.moe_uses_cta_pairs(65536, 256, 512) == 0      # K too short
        assert L.moe_uses_cta_pairs(8191, 32, 2880) == 0       # < 256 rows per expert
        L.moe_set_cta_pairs(1)
        assert L.moe_uses_cta_pairs(100, 8, 64) == 1
        L.moe_set_cta_pairs(0)
        assert L.moe_uses_cta_pairs(32768, 32, 2880) == 0
    finally:
        L.moe_set_cta_pairs(-1)
    assert L.moe_uses_cta_pairs(32768, 32, 2880) == 1


class _Buffers:
    """Buffers for the host-side error checks, each sized for the dimensions
    of the call it is passed to.  With a GPU they are real device
    allocations, so that if a host check were lost the call would launch on
    valid memory and the test would fail on its return code, instead of a
    kernel touching a made-up address on a shared GPU.  Without a GPU the
    library cannot launch anything, and host memory of the same size stands
    in."""

    def __init__(self):
        import torch
        self.torch = torch
        self.cuda = torch.cuda.is_available()
        self.keep = []

    def __call__(self, nbytes):
        n = max(1, int(nbytes))
        if self.cuda:
            t = self.torch.zeros(n, dtype=self.torch.uint8, device="cuda")
            self.keep.append(t)
            return ctypes.c_void_p(t.data_ptr())
        b = ctypes.create_string_buffer(n)
        self.keep.append(b)
        return ctypes.c_void_p(ctypes.addressof(b))


def test_host_side_argument_errors(L):
    B = _Buffers()

    def route_bufs(T, E, k, ws_bytes):
        return (B(T * E * 4), B(T * k * 4), B(T * k * 4), B(E * 4), B((E + 1) * 4),
                B(T * k * 4), B(ws_bytes))

    ws = 1 << 20
    # k > E, E > 512: rejected before any launch
    lg, ix, w, c, o, d, wb = route_bufs(4, 3, 4, ws)
    assert L.moe_route_topk(lg, 4, 3, 4, ix, w, c, o, d, wb, ws, None) == 2
    lg, ix, w, c, o, d, wb = route_bufs(4, 513, 1, ws)
    assert L.moe_route_topk(lg, 4, 513, 1, ix, w, c, o, d, wb, ws, None) == 2
    # T*k overflow: no buffer can be that large, so every pointer is null
    # (a lost overflow check would then stop at the null check, with 1)
    assert L.moe_route_topk(None, 1 << 30, 8, 4, None, None, None, None, None, None,
                            ws, None) == 2
    # null output; workspace declared too short (the buffer itself is full size)
    T, E, k = 4, 8, 2
    need = L.moe_route_workspace_bytes(T, E, k)
    lg, ix, w, c, o, d, wb = route_bufs(T, E, k, need)
    assert L.moe_route_topk(lg, T, E, k, None, w, c, o, d, wb, need, None) == 1
    assert L.moe_route_topk(lg, T, E, k, ix, w, c, o, d, wb, 1, None) == 1
    # permute: H not a multiple of 8, null input, dw without Zp
    T, k = 4, 2
    assert L.moe_permute(B(T * 12 * 2), B(T * k * 4), None, T, 12, k, B(T * k * 12 * 2),
                         None, None, None) == 2
    assert L.moe_permute(None, B(T * k * 4), None, T, 16, k, B(T * k * 16 * 2),
                         None, None, None) == 1
    assert L.moe_permute(B(T * 16 * 2), B(T * k * 4), None, T, 16, k, B(T * k * 16 * 2),
                         None, B(T * k * 4), None) == 1
    assert L.moe_unpermute(B(T * k * 16 * 2), B(T * k * 4), None, T, 16, k, None,
                           None) == 1

    # GEMMs: unsupported rank / shape, missing output, short saved buffer and
    # workspace (every buffer sized for the shape it is passed with)
    def gemm_bufs(E, H, I, r, R):
        W = [B(E * 2 * I * H * 2), B(E * r * H * 2), B(E * 2 * I * r * 2),
             B(E * H * I * 2), B(E * r * I * 2), B(E * H * r * 2)]
        return B(R * H * 2), B((E + 1) * 4), W

    E, H, I, R = 8, 256, 512, 64
    xp, off, W = gemm_bufs(E, H, I, 8, R)
    assert L.moe_lora_mlp_fwd(xp, off, E, H, I, 8, 2.0, *W, R, B(R * H * 2), B(1 << 20),
                              1 << 20, None, 0, None) == 2
    xp, off, W = gemm_bufs(E, 200, I, 16, R)
    assert L.moe_lora_mlp_fwd(xp, off, E, 200, I, 16, 2.0, *W, R, B(R * 200 * 2),
                              B(1 << 20), 1 << 20, None, 0, None) == 2
    xp, off, W = gemm_bufs(E, H, I, 16, R)
    sb = L.moe_saved_bytes(R, H, I, 16)
    assert L.moe_lora_mlp_fwd(xp, off, E, H, I, 16, 2.0, *W, R, None, B(sb), sb,
                              None, 0, None) == 1
    assert L.moe_lora_mlp_fwd(xp, off, E, H, I, 16, 2.0, *W, R, B(R * H * 2), B(sb), 16,
                              None, 0, None) == 1
    wsb = L.moe_workspace_bytes(R, E, H, I, 16)
    assert L.moe_lora_mlp_bwd(B(R * H * 2), xp, off, E, H, I, 16, 2.0, *W, B(sb), sb, R,
                              B(R * H * 2), B(E * 16 * H * 2), B(E * 2 * I * 16 * 2),
                              B(E * 16 * I * 2), B(E * H * 16 * 2), B(wsb), 16, None) == 1


def test_ep_regroup_host_side_argument_errors(L):
    """Every rejection returns before a launch (no GPU needed)."""
    B = _Buffers()
    N, EL, rows, H = 2, 4, 10, 16

    def bufs(n, el, h):
        return B(rows * h * 2), B(n * el * 4), B(rows * h * 2), B((el + 1) * 4)

    i, c, o, off = bufs(N, EL, H)
    # unsupported: H not a multiple of 8, too many segments, bad direction
    i12, c12, o12, _ = bufs(N, EL, 12)
    assert L.moe_ep_regroup(i12, c12, N, EL, rows, 12, 0, o12, None, None) == 2
    assert L.moe_ep_regroup(None, None, 65, 64, rows, H, 0, None, None, None) == 2
    assert L.moe_ep_regroup(i, c, N, EL, rows, H, 2, o, None, None) == 2
    assert L.moe_ep_regroup(i, c, 0, EL, rows, H, 0, o, None, None) == 2
    # invalid: null counts, null rows with rows > 0, offsets with direction 1
    assert L.moe_ep_regroup(i, None, N, EL, rows, H, 0, o, None, None) == 1
    assert L.moe_ep_regroup(None, c, N, EL, rows, H, 0, o, None, None) == 1
    assert L.moe_ep_regroup(i, c, N, EL, rows, H, 0, None, None, None) == 1
    assert L.moe_ep_regroup(i, c, N, EL, rows, H, 1, o, off, None) == 1


def test_binding_fails_loudly_without_library(monkeypatch, tmp_path):
    monkeypatch.setattr(ops, "_LIB_PATH", str(tmp_path / "missing.so"))
    monkeypatch.setattr(ops, "_lib", None)
    with pytest.raises(RuntimeError, match="missing"):
        ops.lib()
