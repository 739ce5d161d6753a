"""ctypes binding of ``libmoe_b200.so`` (the C ABI declared in ``include/moe_b200.h``).

Argument marshalling only: torch tensors provide device memory and the current CUDA stream;
every step of the layer runs in the library's kernels.  Importing this module fails loudly if
the library has not been built, and every call raises :class:`MoeError` on a non-zero status.
There is no CPU path.
"""
from __future__ import annotations

import ctypes
import math
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmoe_b200.so")

MOE_F32, MOE_BF16 = 0, 1
FLAG_RENORMALIZE, FLAG_ARRIVAL_ORDER, FLAG_GATED, FLAG_ROUTER_PREPARED = 1, 2, 4, 8
MOE_OK = 0
MOE_ERR_DEVICE = 5       # the status word holds an error (moe_get_device_status)
DEV_OK, DEV_TIMEOUT, DEV_BAD_INDEX = 0, 1, 2


class MoeError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__("%s failed: %s (status %d)" % (what, _status_string(status), status))


class Problem(ctypes.Structure):
    _fields_ = [("T", ctypes.c_int32), ("d_model", ctypes.c_int32), ("d_ff", ctypes.c_int32),
                ("E", ctypes.c_int32), ("k", ctypes.c_int32),
                ("capacity_factor", ctypes.c_float), ("dtype", ctypes.c_int32),
                ("flags", ctypes.c_uint32)]


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError("libmoe_b200.so is not built (run __graft_entry__.build() or "
                          "python expert_ffn_layer_router_b200/build.py); there is no fallback")
    L = ctypes.CDLL(LIB_PATH)
    P = ctypes.POINTER(Problem)
    vp, sz = ctypes.c_void_p, ctypes.c_size_t
    sig = {
        "moe_capacity": [P, ctypes.POINTER(ctypes.c_int64)],
        "moe_workspace_size": [P, ctypes.POINTER(ctypes.c_size_t)],
        "moe_route": [P, vp, vp, vp, vp, vp, vp, vp, sz, vp],
        "moe_capacity_dispatch": [P, ctypes.c_int64] + [vp] * 8 + [sz, vp],
        "moe_router_logits": [P, vp, vp, vp, vp, vp, sz, vp],
        "moe_prepare_router": [P, vp, vp, sz, vp],
        "moe_dispatch": [P, vp, vp, vp, vp, vp, vp, vp, sz, vp],
        "moe_expert_ffn": [P, vp, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp],
        "moe_combine": [P, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp],
        "moe_forward": [P] + [vp] * 15 + [sz, vp],
        "moe_get_device_status": [vp, sz, vp, ctypes.POINTER(ctypes.c_int32)],
        "moe_reset_device_status": [vp, sz, vp],
        "moe_set_stage_events": [ctypes.POINTER(ctypes.c_void_p), ctypes.c_int32],
        "moe_route_static": [P, vp, vp, vp, vp, vp, vp, vp],
        "moe_selftest_wait_timeout": [vp, sz, ctypes.c_int32, vp],
    }
    for name, args in sig.items():
        fn = getattr(L, name)
        fn.argtypes = args
        fn.restype = ctypes.c_int
    L.moe_status_string.argtypes = [ctypes.c_int]
    L.moe_status_string.restype = ctypes.c_char_p
    L.moe_last_launch_count.argtypes = []
    L.moe_last_launch_count.restype = ctypes.c_int32
    return L


_lib = _load()

EXPORTS = ("moe_capacity", "moe_workspace_size", "moe_route", "moe_dispatch", "moe_expert_ffn",
           "moe_combine", "moe_forward", "moe_get_device_status", "moe_reset_device_status",
           "moe_last_launch_count", "moe_status_string", "moe_set_stage_events",
           "moe_route_static", "moe_selftest_wait_timeout", "moe_capacity_dispatch",
           "moe_router_logits", "moe_prepare_router")

STAGE_EVENTS = 7
STAGE_NAMES = ("router_logits", "route_topk", "capacity_dispatch", "expert_gemm1",
               "expert_gemm2", "combine")


def lib():
    return _lib


def _status_string(s: int) -> str:
    return _lib.moe_status_string(int(s)).decode()


def _check(status: int, what: str):
    if status != MOE_OK:
        raise MoeError(status, what)


def _ptr(t):
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def problem(T, d_model, d_ff, E, k, capacity_factor, dtype, flags=0) -> Problem:
    if isinstance(dtype, str):
        dtype = {"f32": MOE_F32, "bf16": MOE_BF16}[dtype]
    elif isinstance(dtype, torch.dtype):
        dtype = MOE_BF16 if dtype == torch.bfloat16 else MOE_F32
    return Problem(int(T), int(d_model), int(d_ff), int(E), int(k), float(capacity_factor),
                   int(dtype), int(flags))


def moe_capacity(p: Problem) -> int:
    K = ctypes.c_int64()
    _check(_lib.moe_capacity(ctypes.byref(p), ctypes.byref(K)), "moe_capacity")
    return K.value


def moe_workspace_size(p: Problem) -> int:
    n = ctypes.c_size_t()
    _check(_lib.moe_workspace_size(ctypes.byref(p), ctypes.byref(n)), "moe_workspace_size")
    return n.value


def moe_route(p, logits, ids, w, slot, drop, counts, ws, stream=None):
    _check(_lib.moe_route(ctypes.byref(p), _ptr(logits), _ptr(ids), _ptr(w), _ptr(slot),
                          _ptr(drop), _ptr(counts), _ptr(ws), ws.numel() * ws.element_size(),
                          _stream(stream)), "moe_route")


def moe_capacity_dispatch(p, K, ids, w, slot, drop, counts, ws, offsets=None, rowtok=None,
                          stream=None):
    _check(_lib.moe_capacity_dispatch(ctypes.byref(p), int(K), _ptr(ids), _ptr(w), _ptr(slot),
                                      _ptr(drop), _ptr(counts), _ptr(offsets), _ptr(rowtok),
                                      _ptr(ws), ws.numel() * ws.element_size(), _stream(stream)),
           "moe_capacity_dispatch")


def moe_prepare_router(p, Wr, ws, stream=None):
    _check(_lib.moe_prepare_router(ctypes.byref(p), _ptr(Wr), _ptr(ws),
                                   ws.numel() * ws.element_size(), _stream(stream)),
           "moe_prepare_router")


def moe_router_logits(p, x, Wr, br, logits, ws, stream=None):
    _check(_lib.moe_router_logits(ctypes.byref(p), _ptr(x), _ptr(Wr), _ptr(br), _ptr(logits),
                                  _ptr(ws), ws.numel() * ws.element_size(), _stream(stream)),
           "moe_router_logits")


def moe_dispatch(p, ids, slot, offsets, rowtok, ws, x=None, x_perm=None, stream=None):
    _check(_lib.moe_dispatch(ctypes.byref(p), _ptr(ids), _ptr(slot), _ptr(offsets),
                             _ptr(rowtok), _ptr(x), _ptr(x_perm), _ptr(ws),
                             ws.numel() * ws.element_size(), _stream(stream)), "moe_dispatch")


def moe_expert_ffn(p, x, offsets, rowtok, W1, b1, W2, b2, Y, ws, stream=None):
    _check(_lib.moe_expert_ffn(ctypes.byref(p), _ptr(x), _ptr(offsets), _ptr(rowtok), _ptr(W1),
                               _ptr(b1), _ptr(W2), _ptr(b2), _ptr(Y), _ptr(ws),
                               ws.numel() * ws.element_size(), _stream(stream)),
           "moe_expert_ffn")


def moe_combine(p, x, Y, w, ids, slot, offsets, out, ws=None, stream=None):
    nbytes = 0 if ws is None else ws.numel() * ws.element_size()
    _check(_lib.moe_combine(ctypes.byref(p), _ptr(x), _ptr(Y), _ptr(w), _ptr(ids), _ptr(slot),
                            _ptr(offsets), _ptr(out), _ptr(ws), nbytes, _stream(stream)),
           "moe_combine")


def moe_forward(p, x, Wr, br, W1, b1, W2, b2, out, ws, logits_out=None, ids_out=None,
                w_out=None, slot_out=None, drop_out=None, counts_out=None, stream=None):
    _check(_lib.moe_forward(ctypes.byref(p), _ptr(x), _ptr(Wr), _ptr(br), _ptr(W1), _ptr(b1),
                            _ptr(W2), _ptr(b2), _ptr(out), _ptr(logits_out), _ptr(ids_out),
                            _ptr(w_out), _ptr(slot_out), _ptr(drop_out), _ptr(counts_out),
                            _ptr(ws), ws.numel() * ws.element_size(), _stream(stream)),
           "moe_forward")


def moe_get_device_status(ws, stream=None) -> int:
    """Status word of ``ws``; ``ws=None``: that of moe_route_static on the current device."""
    code = ctypes.c_int32()
    nbytes = 0 if ws is None else ws.numel() * ws.element_size()
    rc = _lib.moe_get_device_status(_ptr(ws), nbytes, _stream(stream), ctypes.byref(code))
    if rc not in (MOE_OK, MOE_ERR_DEVICE):
        raise MoeError(rc, "moe_get_device_status")
    return code.value


def moe_reset_device_status(ws, stream=None):
    nbytes = 0 if ws is None else ws.numel() * ws.element_size()
    _check(_lib.moe_reset_device_status(_ptr(ws), nbytes, _stream(stream)),
           "moe_reset_device_status")


def moe_selftest_wait_timeout(ws, limit_us, stream=None):
    _check(_lib.moe_selftest_wait_timeout(_ptr(ws), ws.numel() * ws.element_size(), int(limit_us),
                                          _stream(stream)), "moe_selftest_wait_timeout")


def moe_last_launch_count() -> int:
    return int(_lib.moe_last_launch_count())


def moe_set_stage_events(events):
    """``events``: STAGE_EVENTS torch.cuda.Event objects (or None to turn recording off)."""
    if not events:
        _check(_lib.moe_set_stage_events(None, 0), "moe_set_stage_events")
        return
    arr = (ctypes.c_void_p * len(events))(*[ctypes.c_void_p(e.cuda_event) for e in events])
    _check(_lib.moe_set_stage_events(arr, len(events)), "moe_set_stage_events")


# ----------------------------------------------------------------------------------------------
# Convenience: a layer that owns its workspace (allocated once through torch).
# ----------------------------------------------------------------------------------------------
class MoELayer:
    """Holds a problem description and a workspace; calls the C ABI on torch tensors."""

    def __init__(self, T, d_model, d_ff, E, k, capacity_factor=math.inf, dtype="bf16",
                 device="cuda", flags=0):
        self.p = problem(T, d_model, d_ff, E, k, capacity_factor, dtype, flags)
        self.K = moe_capacity(self.p)
        self.device = torch.device(device)
        nbytes = moe_workspace_size(self.p)
        # int64 elements keep the base 256-byte aligned through the caching allocator.
        self.ws = torch.zeros((nbytes + 7) // 8, dtype=torch.int64, device=self.device)
        self.max_rows = min(T * k, E * self.K)

    @property
    def torch_dtype(self):
        return torch.bfloat16 if self.p.dtype == MOE_BF16 else torch.float32

    def forward(self, x, Wr, br, W1, b1, W2, b2, out=None, want_routing=False, stream=None):
        p = self.p
        out = torch.empty_like(x) if out is None else out
        extra = {}
        if want_routing:
            dev = x.device
            extra = dict(
                logits_out=torch.empty((p.T, p.E), dtype=torch.float32, device=dev),
                ids_out=torch.empty((p.T, p.k), dtype=torch.int32, device=dev),
                w_out=torch.empty((p.T, p.k), dtype=torch.float32, device=dev),
                slot_out=torch.empty((p.T, p.k), dtype=torch.int32, device=dev),
                drop_out=torch.empty((p.T, p.k), dtype=torch.uint8, device=dev),
                counts_out=torch.empty(2 * p.E, dtype=torch.int32, device=dev))
        moe_forward(p, x, Wr, br, W1, b1, W2, b2, out, self.ws, stream=stream, **extra)
        return (out, extra) if want_routing else out

    def route(self, logits, stream=None):
        p, dev = self.p, logits.device
        r = dict(ids=torch.empty((p.T, p.k), dtype=torch.int32, device=dev),
                 w=torch.empty((p.T, p.k), dtype=torch.float32, device=dev),
                 slot=torch.empty((p.T, p.k), dtype=torch.int32, device=dev),
                 drop=torch.empty((p.T, p.k), dtype=torch.uint8, device=dev),
                 counts=torch.empty(2 * p.E, dtype=torch.int32, device=dev))
        moe_route(p, logits, r["ids"], r["w"], r["slot"], r["drop"], r["counts"], self.ws,
                  stream)
        return r

    def prepare_router(self, Wr, stream=None):
        """Splits Wr once into the workspace; later forwards skip the split (the problem's
        MOE_FLAG_ROUTER_PREPARED is set).  Call again after Wr changes."""
        self.p.flags |= FLAG_ROUTER_PREPARED
        moe_prepare_router(self.p, Wr, self.ws, stream)

    def router_logits(self, x, Wr, br, stream=None):
        logits = torch.empty((self.p.T, self.p.E), dtype=torch.float32, device=x.device)
        moe_router_logits(self.p, x, Wr, br, logits, self.ws, stream)
        return logits

    def capacity_dispatch(self, ids, w, K, stream=None):
        """Capacity selection of a given routing (ids, w [T, k]) with capacity K; returns slot,
        drop, counts and the expert-sorted layout (offsets, rowtok)."""
        p, dev = self.p, ids.device
        rows = max(min(p.T * p.k, p.E * int(K)), 1)
        r = dict(slot=torch.empty((p.T, p.k), dtype=torch.int32, device=dev),
                 drop=torch.empty((p.T, p.k), dtype=torch.uint8, device=dev),
                 counts=torch.empty(2 * p.E, dtype=torch.int32, device=dev),
                 offsets=torch.empty(p.E + 1, dtype=torch.int32, device=dev),
                 rowtok=torch.empty(rows, dtype=torch.int32, device=dev))
        moe_capacity_dispatch(p, K, ids, w, r["slot"], r["drop"], r["counts"], self.ws,
                              r["offsets"], r["rowtok"], stream)
        return r

    def dispatch(self, ids, slot, x=None, permute=False, stream=None):
        p, dev = self.p, ids.device
        offsets = torch.empty(p.E + 1, dtype=torch.int32, device=dev)
        rowtok = torch.empty(max(self.max_rows, 1), dtype=torch.int32, device=dev)
        xp = None
        if permute:
            xp = torch.empty((max(self.max_rows, 1), p.d_model), dtype=x.dtype, device=dev)
        moe_dispatch(p, ids, slot, offsets, rowtok, self.ws, x=x, x_perm=xp, stream=stream)
        return offsets, rowtok, xp

    def expert_ffn(self, x, offsets, rowtok, W1, b1, W2, b2, stream=None):
        p = self.p
        Y = torch.empty((max(self.max_rows, 1), p.d_model), dtype=x.dtype, device=x.device)
        moe_expert_ffn(p, x, offsets, rowtok, W1, b1, W2, b2, Y, self.ws, stream)
        return Y

    def combine(self, x, Y, w, ids, slot, offsets, stream=None):
        out = torch.empty_like(x)
        moe_combine(self.p, x, Y, w, ids, slot, offsets, out, self.ws, stream)
        return out
