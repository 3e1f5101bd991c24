"""Python binding of libmoe_lora.so (ctypes).

Argument marshalling only: every step of the block runs in the library's
CUDA kernels.  Tensors are passed by ``data_ptr()`` with the current CUDA
stream.  If the library is missing, every call raises; there is no fallback.
"""

from __future__ import annotations

import ctypes
import os

import torch

_LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libmoe_lora.so")
_lib = None

MOE_OK = 0
STATUS_NAMES = {0: "ok", 1: "invalid argument", 2: "unsupported shape",
                3: "CUDA error", 4: "device wait timed out",
                5: "device index out of range"}

EXPORTS = [
    "moe_route_workspace_bytes", "moe_route_topk", "moe_permute", "moe_unpermute",
    "moe_saved_bytes", "moe_saved_part_offset", "moe_workspace_bytes",
    "moe_lora_mlp_fwd", "moe_lora_mlp_bwd", "moe_lora_mlp_bwd_full", "moe_get_device_status",
    "moe_status_string", "moe_set_wait_limit_ns", "moe_test_inject_stall",
    "moe_set_cta_pairs", "moe_uses_cta_pairs", "moe_kernel_launches", "moe_profile_enable",
    "moe_router_fwd", "moe_router_bwd_workspace_bytes", "moe_router_bwd",
    "moe_profile_collect", "moe_ep_regroup",
]

PROF_KINDS = {"route": 0, "permute": 1, "gate_up_fwd": 2, "down_fwd": 3,
              "unpermute": 4, "down_bwd": 5, "gate_up_bwd": 6, "lora_grad": 7,
              "transpose": 8, "base_grad": 9, "router_fwd": 10, "router_bwd": 11,
              "rank_down": 12}


class MoeError(RuntimeError):
    def __init__(self, code, where):
        super().__init__(f"{where}: {STATUS_NAMES.get(code, code)} ({code})")
        self.code = code


def lib():
    """The loaded library (raises if it was not built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(_LIB_PATH):
            raise RuntimeError(
                f"{_LIB_PATH} is missing: build it with "
                "`python -m moe_expert_grouped_softmax_b200.build`")
        L = ctypes.CDLL(_LIB_PATH)
        P, I, S, F, U64 = (ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t,
                           ctypes.c_float, ctypes.c_uint64)
        L.moe_route_workspace_bytes.argtypes = [I, I, I]
        L.moe_route_workspace_bytes.restype = S
        L.moe_route_topk.argtypes = [P, I, I, I, P, P, P, P, P, P, S, P]
        L.moe_route_topk.restype = I
        L.moe_permute.argtypes = [P, P, P, I, I, I, P, P, P, P]
        L.moe_permute.restype = I
        L.moe_unpermute.argtypes = [P, P, P, I, I, I, P, P]
        L.moe_unpermute.restype = I
        L.moe_router_fwd.argtypes = [P, P, I, I, I, P, P]
        L.moe_router_fwd.restype = I
        L.moe_router_bwd_workspace_bytes.argtypes = [I, I]
        L.moe_router_bwd_workspace_bytes.restype = S
        L.moe_router_bwd.argtypes = [P, P, P, P, P, P, P, P, I, I, I, I, P, P, P, S, P]
        L.moe_router_bwd.restype = I
        L.moe_saved_bytes.argtypes = [I, I, I, I]
        L.moe_saved_bytes.restype = S
        L.moe_saved_part_offset.argtypes = [I, I, I, I, I]
        L.moe_saved_part_offset.restype = S
        L.moe_workspace_bytes.argtypes = [I, I, I, I, I]
        L.moe_workspace_bytes.restype = S
        L.moe_lora_mlp_fwd.argtypes = [P, P, I, I, I, I, F, P, P, P, P, P, P, I, P,
                                       P, S, P, S, P]
        L.moe_lora_mlp_fwd.restype = I
        L.moe_lora_mlp_bwd.argtypes = [P, P, P, I, I, I, I, F, P, P, P, P, P, P, P,
                                       S, I, P, P, P, P, P, P, S, P]
        L.moe_lora_mlp_bwd.restype = I
        L.moe_lora_mlp_bwd_full.argtypes = [P, P, P, I, I, I, I, F, P, P, P, P, P, P, P,
                                            S, I, P, P, P, P, P, P, P, P, S, P]
        L.moe_lora_mlp_bwd_full.restype = I
        L.moe_get_device_status.argtypes = [P]
        L.moe_get_device_status.restype = I
        L.moe_status_string.argtypes = [I]
        L.moe_status_string.restype = ctypes.c_char_p
        L.moe_set_wait_limit_ns.argtypes = [U64]
        L.moe_set_wait_limit_ns.restype = None
        L.moe_set_cta_pairs.argtypes = [I]
        L.moe_set_cta_pairs.restype = None
        L.moe_uses_cta_pairs.argtypes = [I, I, I]
        L.moe_uses_cta_pairs.restype = I
        L.moe_kernel_launches.argtypes = []
        L.moe_kernel_launches.restype = ctypes.c_ulonglong
        L.moe_test_inject_stall.argtypes = [I]
        L.moe_test_inject_stall.restype = None
        L.moe_profile_enable.argtypes = [I]
        L.moe_profile_enable.restype = I
        L.moe_profile_collect.argtypes = [I, ctypes.POINTER(ctypes.c_float), I]
        L.moe_profile_collect.restype = I
        L.moe_ep_regroup.argtypes = [P, P, I, I, I, I, I, P, P, P]
        L.moe_ep_regroup.restype = I
        _lib = L
    return _lib


def _p(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream():
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def _check(code, where):
    if code != MOE_OK:
        raise MoeError(code, where)


def _need(t, dtype, shape, name):
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise ValueError(f"{name}: expected {dtype}, got {t.dtype}")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name}: expected shape {tuple(shape)}, got {tuple(t.shape)}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def device_status():
    """Synchronise, return and clear the device-side status word."""
    return lib().moe_get_device_status(_stream())


def set_wait_limit_ns(ns):
    lib().moe_set_wait_limit_ns(int(ns))


def kernel_launches():
    """Kernels this library has launched in this process (host-side count)."""
    return int(lib().moe_kernel_launches())


def set_cta_pairs(on=True):
    """Grouped GEMMs on CTA pairs (True, 256-row tiles), single CTAs (False)
    or chosen per GEMM from the rows per expert and K (None, the default)."""
    lib().moe_set_cta_pairs(-1 if on is None else (1 if on else 0))


def uses_cta_pairs(R, E, K):
    """Whether a grouped GEMM over R routed rows, E experts and reduction
    length K runs on CTA pairs under the current setting (the library's own
    choice; host-side, no GPU needed)."""
    return bool(lib().moe_uses_cta_pairs(R, E, K))


def test_inject_stall(on=True):
    lib().moe_test_inject_stall(1 if on else 0)


def profile_enable(on=True):
    _check(lib().moe_profile_enable(1 if on else 0), "moe_profile_enable")


def profile_collect(kind):
    """Durations (ms) of the recorded launches of one kernel kind."""
    buf = (ctypes.c_float * 512)()
    n = lib().moe_profile_collect(PROF_KINDS[kind], buf, 512)
    if n < 0:
        raise MoeError(3, "moe_profile_collect")
    return [buf[i] for i in range(n)]


# ------------------------------------------------------------------ sizes
def route_workspace_bytes(T, E, k):
    return lib().moe_route_workspace_bytes(T, E, k)


def saved_bytes(R, H, I, r):
    return lib().moe_saved_bytes(R, H, I, r)


def saved_part_offset(R, H, I, r, part):
    return lib().moe_saved_part_offset(R, H, I, r, part)


def workspace_bytes(R, E, H, I, r):
    return lib().moe_workspace_bytes(R, E, H, I, r)


def ld_rank(R):
    """Row pitch (elements) of the transposed rank-r saved parts."""
    return (R + 63) // 64 * 64


def saved_views(saved, R, H, I, r):
    """Views of the saved-activation buffer: Z1, h, XA1t, HA2t."""
    b = saved
    o = [saved_part_offset(R, H, I, r, i) for i in range(5)]
    ld = ld_rank(R)

    def view(i, shape):
        n = 1
        for d in shape:
            n *= d
        return b[o[i]:o[i] + 2 * n].view(torch.bfloat16).view(*shape)

    return (view(0, (R, 2 * I)), view(1, (R, I)), view(2, (r, ld)), view(3, (r, ld)))


# ------------------------------------------------------------------ ops
def route_topk(logits, k, out=None, ws=None):
    """a1: returns (topk_idx, topk_w, expert_counts, expert_offsets, dest)."""
    T, E = logits.shape
    _need(logits, torch.float32, (T, E), "logits")
    dev = logits.device
    if out is None:
        out = (torch.empty((T, k), dtype=torch.int32, device=dev),
               torch.empty((T, k), dtype=torch.float32, device=dev),
               torch.empty((E,), dtype=torch.int32, device=dev),
               torch.empty((E + 1,), dtype=torch.int32, device=dev),
               torch.empty((T, k), dtype=torch.int32, device=dev))
    idx, w, counts, offsets, dest = out
    nbytes = route_workspace_bytes(T, E, k)
    if ws is None or ws.numel() < nbytes:
        ws = torch.empty(nbytes, dtype=torch.uint8, device=dev)
    _check(lib().moe_route_topk(_p(logits), T, E, k, _p(idx), _p(w), _p(counts),
                                _p(offsets), _p(dest), _p(ws), ws.numel(), _stream()),
           "moe_route_topk")
    return idx, w, counts, offsets, dest


def permute(X, dest, scale=None, Zp=None, out=None, dw=None):
    """a2 / a6: Xp[dest[t, j]] = scale[t, j] * X[t]; optional dw = <X[t], Zp[dest]>."""
    T, H = X.shape
    k = dest.shape[1]
    _need(X, torch.bfloat16, (T, H), "X")
    _need(dest, torch.int32, (T, k), "dest")
    if scale is not None:
        _need(scale, torch.float32, (T, k), "scale")
    if out is None:
        out = torch.empty((T * k, H), dtype=torch.bfloat16, device=X.device)
    if Zp is not None:
        _need(Zp, torch.bfloat16, (T * k, H), "Zp")
        if dw is None:
            dw = torch.empty((T, k), dtype=torch.float32, device=X.device)
    _check(lib().moe_permute(_p(X), _p(dest), _p(scale), T, H, k, _p(out), _p(Zp),
                             _p(dw), _stream()), "moe_permute")
    return (out, dw) if Zp is not None else out


def router_fwd(X, Wr, out=None):
    """Trained router: logits [T, E] fp32 = X Wr^T."""
    T, H = X.shape
    E = Wr.shape[0]
    _need(X, torch.bfloat16, (T, H), "X")
    _need(Wr, torch.bfloat16, (E, H), "Wr")
    if out is None:
        out = torch.empty((T, E), dtype=torch.float32, device=X.device)
    _need(out, torch.float32, (T, E), "logits")
    _check(lib().moe_router_fwd(_p(X), _p(Wr), T, H, E, _p(out), _stream()), "moe_router_fwd")
    return out


def router_bwd(w, dw, idx, dest, offsets, Xp, Wr, dXp, out=None, ws=None):
    """Trained router backward: returns (dX with the router's part, dWr fp32)."""
    T, k = w.shape
    E, H = Wr.shape
    for t, dt, sh, n in ((w, torch.float32, (T, k), "w"), (dw, torch.float32, (T, k), "dw"),
                         (idx, torch.int32, (T, k), "idx"), (dest, torch.int32, (T, k), "dest"),
                         (offsets, torch.int32, (E + 1,), "offsets"),
                         (Xp, torch.bfloat16, (T * k, H), "Xp"), (Wr, torch.bfloat16, (E, H), "Wr"),
                         (dXp, torch.bfloat16, (T * k, H), "dXp")):
        _need(t, dt, sh, n)
    dev = Xp.device
    if out is None:
        out = (torch.empty((T, H), dtype=torch.bfloat16, device=dev),
               torch.empty((E, H), dtype=torch.float32, device=dev))
    dX, dWr = out
    nb = int(lib().moe_router_bwd_workspace_bytes(T, k))
    if ws is None or ws.numel() < nb:
        ws = torch.empty(max(nb, 1), dtype=torch.uint8, device=dev)
    _check(lib().moe_router_bwd(_p(w), _p(dw), _p(idx), _p(dest), _p(offsets), _p(Xp), _p(Wr),
                                _p(dXp), T, H, E, k, _p(dX), _p(dWr), _p(ws), ws.numel(),
                                _stream()),
           "moe_router_bwd")
    return dX, dWr


def unpermute(Yp, dest, w=None, out=None):
    """a5 / a10: Y[t] = sum_j w[t, j] Yp[dest[t, j]]."""
    T, k = dest.shape
    H = Yp.shape[1]
    _need(Yp, torch.bfloat16, (T * k, H), "Yp")
    _need(dest, torch.int32, (T, k), "dest")
    if w is not None:
        _need(w, torch.float32, (T, k), "w")
    if out is None:
        out = torch.empty((T, H), dtype=torch.bfloat16, device=Yp.device)
    _check(lib().moe_unpermute(_p(Yp), _p(dest), _p(w), T, H, k, _p(out), _stream()),
           "moe_unpermute")
    return out


def ep_regroup(inp, counts, direction, out=None, offsets=None):
    """Expert parallelism: rows from N source ranks for this rank's E_loc
    experts (``counts`` [N, E_loc] int32 on the device), source-major ->
    expert-major (``direction`` 0, optionally writing the local ``offsets``
    [E_loc + 1]) or back (1)."""
    rows, H = inp.shape
    N, EL = counts.shape
    _need(inp, torch.bfloat16, (rows, H), "rows")
    _need(counts, torch.int32, (N, EL), "counts")
    if out is None:
        out = torch.empty_like(inp)
    if offsets is not None:
        _need(offsets, torch.int32, (EL + 1,), "offsets")
    _check(lib().moe_ep_regroup(_p(inp), _p(counts), N, EL, rows, H, int(direction), _p(out),
                                _p(offsets), _stream()),
           "moe_ep_regroup")
    return out


def _weights_check(W1, A1, B1, W2, A2, B2):
    E, I2, H = W1.shape
    I = I2 // 2
    r = A1.shape[1]
    for t, shp, n in [(W1, (E, 2 * I, H), "W1"), (A1, (E, r, H), "A1"),
                      (B1, (E, 2 * I, r), "B1"), (W2, (E, H, I), "W2"),
                      (A2, (E, r, I), "A2"), (B2, (E, H, r), "B2")]:
        _need(t, torch.bfloat16, shp, n)
    return E, H, I, r


def lora_mlp_fwd(Xp, offsets, W1, A1, B1, W2, A2, B2, s, out=None, saved=None):
    """a3 + a4: returns (Z2 [R, H], saved uint8 buffer)."""
    E, H, I, r = _weights_check(W1, A1, B1, W2, A2, B2)
    R = Xp.shape[0]
    _need(Xp, torch.bfloat16, (R, H), "Xp")
    _need(offsets, torch.int32, (E + 1,), "offsets")
    if out is None:
        out = torch.empty((R, H), dtype=torch.bfloat16, device=Xp.device)
    nb = saved_bytes(R, H, I, r)
    if saved is None:
        saved = torch.empty(max(nb, 1), dtype=torch.uint8, device=Xp.device)
    _check(lib().moe_lora_mlp_fwd(_p(Xp), _p(offsets), E, H, I, r, float(s), _p(W1),
                                  _p(A1), _p(B1), _p(W2), _p(A2), _p(B2), R, _p(out),
                                  _p(saved), saved.numel(), None, 0, _stream()),
           "moe_lora_mlp_fwd")
    return out, saved


def lora_mlp_bwd(dZ2, Xp, offsets, W1, A1, B1, W2, A2, B2, s, saved, out=None,
                 ws=None, base_out=None):
    """a7 + a8 + a9: returns (dXp, dA1, dB1, dA2, dB2).  With ``base_out`` =
    (dW1 [E, 2I, H], dW2 [E, H, I]) the base-weight gradients of full
    fine-tuning are written there too (``moe_lora_mlp_bwd_full``)."""
    E, H, I, r = _weights_check(W1, A1, B1, W2, A2, B2)
    R = Xp.shape[0]
    _need(dZ2, torch.bfloat16, (R, H), "dZ2")
    _need(Xp, torch.bfloat16, (R, H), "Xp")
    _need(offsets, torch.int32, (E + 1,), "offsets")
    dev = Xp.device
    if out is None:
        out = (torch.empty((R, H), dtype=torch.bfloat16, device=dev),
               torch.empty((E, r, H), dtype=torch.bfloat16, device=dev),
               torch.empty((E, 2 * I, r), dtype=torch.bfloat16, device=dev),
               torch.empty((E, r, I), dtype=torch.bfloat16, device=dev),
               torch.empty((E, H, r), dtype=torch.bfloat16, device=dev))
    dXp, dA1, dB1, dA2, dB2 = out
    nb = workspace_bytes(R, E, H, I, r)
    if ws is None or ws.numel() < nb:
        ws = torch.empty(max(nb, 1), dtype=torch.uint8, device=dev)
    if base_out is None:
        _check(lib().moe_lora_mlp_bwd(_p(dZ2), _p(Xp), _p(offsets), E, H, I, r, float(s),
                                      _p(W1), _p(A1), _p(B1), _p(W2), _p(A2), _p(B2),
                                      _p(saved), saved.numel(), R, _p(dXp), _p(dA1),
                                      _p(dB1), _p(dA2), _p(dB2), _p(ws), ws.numel(),
                                      _stream()),
               "moe_lora_mlp_bwd")
    else:
        dW1, dW2 = base_out
        _need(dW1, torch.bfloat16, (E, 2 * I, H), "dW1")
        _need(dW2, torch.bfloat16, (E, H, I), "dW2")
        _check(lib().moe_lora_mlp_bwd_full(_p(dZ2), _p(Xp), _p(offsets), E, H, I, r,
                                           float(s), _p(W1), _p(A1), _p(B1), _p(W2),
                                           _p(A2), _p(B2), _p(saved), saved.numel(), R,
                                           _p(dXp), _p(dA1), _p(dB1), _p(dA2), _p(dB2),
                                           _p(dW1), _p(dW2), _p(ws), ws.numel(),
                                           _stream()),
               "moe_lora_mlp_bwd_full")
    return dXp, dA1, dB1, dA2, dB2


# ------------------------------------------------------------------ the block
class MoeBlock:
    """Forward + backward of the whole block through the C ABI, with all
    buffers preallocated once for a fixed shape (used by the benchmark and the
    end-to-end tests).  ``step`` runs, on the current stream: route, permute,
    gate_up + SwiGLU, down, weighted unpermute, weighted dY gather, down /
    gate_up backward, LoRA gradients and the dX combine (with ``full_ft``, also
    the base-weight gradients dW1, dW2 of full fine-tuning)."""

    def __init__(self, T, H, I, E, k, r, s, device="cuda", with_dw=False, full_ft=False,
                 train_router=False):
        self.T, self.H, self.I, self.E, self.k, self.r, self.s = T, H, I, E, k, r, s
        self.R = R = T * k
        self.with_dw = with_dw
        dev = torch.device(device)
        bf, i32, f32 = torch.bfloat16, torch.int32, torch.float32
        self.idx = torch.empty((T, k), dtype=i32, device=dev)
        self.w = torch.empty((T, k), dtype=f32, device=dev)
        self.counts = torch.empty((E,), dtype=i32, device=dev)
        self.offsets = torch.empty((E + 1,), dtype=i32, device=dev)
        self.dest = torch.empty((T, k), dtype=i32, device=dev)
        self.route_ws = torch.empty(route_workspace_bytes(T, E, k), dtype=torch.uint8,
                                    device=dev)
        self.Xp = torch.empty((R, H), dtype=bf, device=dev)
        self.Z2 = torch.empty((R, H), dtype=bf, device=dev)
        self.saved = torch.empty(max(1, saved_bytes(R, H, I, r)), dtype=torch.uint8,
                                 device=dev)
        self.Y = torch.empty((T, H), dtype=bf, device=dev)
        self.dZ2 = torch.empty((R, H), dtype=bf, device=dev)
        self.dw = torch.empty((T, k), dtype=f32, device=dev) if with_dw else None
        self.dXp = torch.empty((R, H), dtype=bf, device=dev)
        self.dX = torch.empty((T, H), dtype=bf, device=dev)
        self.dA1 = torch.empty((E, r, H), dtype=bf, device=dev)
        self.dB1 = torch.empty((E, 2 * I, r), dtype=bf, device=dev)
        self.dA2 = torch.empty((E, r, I), dtype=bf, device=dev)
        self.dB2 = torch.empty((E, H, r), dtype=bf, device=dev)
        self.full_ft = full_ft
        # trained router: logits = X Wr^T on the device; dw, dlogits -> dWr and
        # the router's part of dX (needs the routing-weight gradient)
        self.train_router = train_router
        if train_router:
            self.with_dw = True
            self.dw = torch.empty((T, k), dtype=f32, device=dev)
            self.logits = torch.empty((T, E), dtype=f32, device=dev)
            self.dWr = torch.empty((E, H), dtype=f32, device=dev)
            self.router_ws = torch.empty(max(1, int(lib().moe_router_bwd_workspace_bytes(T, k))),
                                         dtype=torch.uint8, device=dev)
        self.dW1 = torch.empty((E, 2 * I, H), dtype=bf, device=dev) if full_ft else None
        self.dW2 = torch.empty((E, H, I), dtype=bf, device=dev) if full_ft else None
        self.ws = torch.empty(max(1, workspace_bytes(R, E, H, I, r)), dtype=torch.uint8,
                              device=dev)

    def forward(self, X, logits, W, Wr=None):
        if self.train_router:
            logits = router_fwd(X, Wr, out=self.logits)
        route_topk(logits, self.k, out=(self.idx, self.w, self.counts, self.offsets,
                                        self.dest), ws=self.route_ws)
        permute(X, self.dest, out=self.Xp)
        lora_mlp_fwd(self.Xp, self.offsets, *W, self.s, out=self.Z2, saved=self.saved)
        unpermute(self.Z2, self.dest, self.w, out=self.Y)
        return self.Y

    def backward(self, dY, W, Wr=None):
        if self.with_dw:
            permute(dY, self.dest, scale=self.w, Zp=self.Z2, out=self.dZ2, dw=self.dw)
        else:
            permute(dY, self.dest, scale=self.w, out=self.dZ2)
        lora_mlp_bwd(self.dZ2, self.Xp, self.offsets, *W, self.s, self.saved,
                     out=(self.dXp, self.dA1, self.dB1, self.dA2, self.dB2), ws=self.ws,
                     base_out=(self.dW1, self.dW2) if self.full_ft else None)
        if self.train_router:
            router_bwd(self.w, self.dw, self.idx, self.dest, self.offsets, self.Xp, Wr,
                       self.dXp, out=(self.dX, self.dWr), ws=self.router_ws)
        else:
            unpermute(self.dXp, self.dest, None, out=self.dX)
        return self.dX

    def step(self, X, logits, dY, W, Wr=None):
        """One fwd+bwd; with a trained router, ``Wr`` [E, H] bf16 replaces
        ``logits`` (which may then be None)."""
        self.forward(X, logits, W, Wr)
        self.backward(dY, W, Wr)

    def capture(self, X, logits, dY, W, Wr=None):
        """Capture one ``step`` on these exact tensors into a CUDA graph;
        ``replay`` then re-runs all of its kernels with one launch.  Inputs
        must be updated in place (the graph holds their addresses).  The
        library launches nothing but its own kernels and stream-ordered
        memsets, and allocates nothing, so the captured step is the same work
        as ``step``."""
        side = torch.cuda.Stream()
        side.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(side):      # one eager step off the capture
            self.step(X, logits, dY, W, Wr)
        torch.cuda.current_stream().wait_stream(side)
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            self.step(X, logits, dY, W, Wr)
        self._graph = graph
        return graph

    def replay(self):
        """Run the captured step on the current stream."""
        self._graph.replay()

    def capture_parts(self, X, logits, dY, W, Wr=None):
        """Capture the forward and the backward of one step on these exact
        tensors into two CUDA graphs (``replay_forward``, ``replay_backward``),
        so that a caller can overlap dY's upload with the forward and Y's
        download with the backward."""
        side = torch.cuda.Stream()
        side.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(side):      # one eager step off the capture
            self.step(X, logits, dY, W, Wr)
        torch.cuda.current_stream().wait_stream(side)
        gf, gb = torch.cuda.CUDAGraph(), torch.cuda.CUDAGraph()
        with torch.cuda.graph(gf):
            self.forward(X, logits, W, Wr)
        with torch.cuda.graph(gb):
            self.backward(dY, W, Wr)
        self._graph_fwd, self._graph_bwd = gf, gb
        return gf, gb

    def replay_forward(self):
        self._graph_fwd.replay()

    def replay_backward(self):
        self._graph_bwd.replay()
