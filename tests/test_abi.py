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


def test_host_side_argument_errors(L):
    P = ctypes.c_void_p
    fake = P(256)  # never dereferenced: the call must fail before any launch
    # k > E, E > 512, T*k overflow
    assert L.moe_route_topk(fake, 4, 3, 4, fake, fake, fake, fake, fake, fake, 1 << 20, None) == 2
    assert L.moe_route_topk(fake, 4, 513, 1, fake, fake, fake, fake, fake, fake, 1 << 20, None) == 2
    assert L.moe_route_topk(fake, 1 << 30, 8, 4, fake, fake, fake, fake, fake, fake, 1 << 20, None) == 2
    # null outputs / short workspace
    assert L.moe_route_topk(fake, 4, 8, 2, None, fake, fake, fake, fake, fake, 1 << 20, None) == 1
    assert L.moe_route_topk(fake, 4, 8, 2, fake, fake, fake, fake, fake, fake, 1, None) == 1
    # permute: H not a multiple of 8, null, dw without Zp
    assert L.moe_permute(fake, fake, None, 4, 12, 2, fake, None, None, None) == 2
    assert L.moe_permute(None, fake, None, 4, 16, 2, fake, None, None, None) == 1
    assert L.moe_permute(fake, fake, None, 4, 16, 2, fake, None, fake, None) == 1
    assert L.moe_unpermute(fake, fake, None, 4, 16, 2, None, None) == 1
    # GEMMs: unsupported rank / shape, missing buffers, short saved buffer
    W = [fake] * 6
    assert L.moe_lora_mlp_fwd(fake, fake, 8, 256, 512, 8, 2.0, *W, 64, fake, fake, 1 << 30, None, 0, None) == 2
    assert L.moe_lora_mlp_fwd(fake, fake, 8, 200, 512, 16, 2.0, *W, 64, fake, fake, 1 << 30, None, 0, None) == 2
    assert L.moe_lora_mlp_fwd(fake, fake, 8, 256, 512, 16, 2.0, *W, 64, None, fake, 1 << 30, None, 0, None) == 1
    assert L.moe_lora_mlp_fwd(fake, fake, 8, 256, 512, 16, 2.0, *W, 64, fake, fake, 16, None, 0, None) == 1
    assert L.moe_lora_mlp_bwd(fake, fake, fake, 8, 256, 512, 16, 2.0, *W, fake, 1 << 30, 64,
                              fake, fake, fake, fake, fake, fake, 16, None) == 1


def test_binding_fails_loudly_without_library(monkeypatch, tmp_path):
    monkeypatch.setattr(ops, "_LIB_PATH", str(tmp_path / "missing.so"))
    monkeypatch.setattr(ops, "_lib", None)
    with pytest.raises(RuntimeError, match="missing"):
        ops.lib()
