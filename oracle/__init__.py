"""ctypes view of the CPU oracle (``moe_oracle.cpp``).

TEST INFRASTRUCTURE ONLY: the tests, the package smoke check and the bench's CPU-baseline leg
may import this package; the product path never does.  Arrays are numpy; bfloat16 tensors are
passed as ``np.uint16`` arrays of raw bits (dtype code 1), float32 tensors as ``np.float32``
(dtype code 0).
"""
import ctypes
import os

import numpy as np

from . import build_oracle

_lib = None

_i32p = np.ctypeslib.ndpointer(dtype=np.int32, flags="C_CONTIGUOUS")
_f32p = np.ctypeslib.ndpointer(dtype=np.float32, flags="C_CONTIGUOUS")
_f64p = np.ctypeslib.ndpointer(dtype=np.float64, flags="C_CONTIGUOUS")
_u8p = np.ctypeslib.ndpointer(dtype=np.uint8, flags="C_CONTIGUOUS")
_vp = ctypes.c_void_p


def lib():
    global _lib
    if _lib is None:
        path = build_oracle.build()
        L = ctypes.CDLL(path)
        L.oracle_capacity.restype = ctypes.c_longlong
        L.oracle_capacity.argtypes = [ctypes.c_longlong] * 3 + [ctypes.c_double]
        L.oracle_own_exp.restype = ctypes.c_float
        L.oracle_own_exp.argtypes = [ctypes.c_float]
        L.oracle_own_exp_n.restype = None
        L.oracle_own_exp_n.argtypes = [ctypes.c_longlong, _f32p, _f32p]
        L.oracle_softmax.restype = None
        L.oracle_softmax.argtypes = [ctypes.c_int, ctypes.c_int, _f32p, _f32p]
        L.oracle_logits.restype = None
        L.oracle_logits.argtypes = [ctypes.c_int] * 4 + [_vp, _f32p, _vp, _f32p, ctypes.c_int]
        L.oracle_route.restype = ctypes.c_int
        L.oracle_route.argtypes = [ctypes.c_int] * 3 + [ctypes.c_longlong, _f32p, _i32p, _f32p,
                                                        _i32p, _u8p, _i32p, ctypes.c_int]
        L.oracle_select.restype = ctypes.c_int
        L.oracle_select.argtypes = [ctypes.c_int] * 3 + [ctypes.c_longlong, _i32p, _f32p,
                                                         _i32p, _u8p, _i32p, ctypes.c_int]
        L.oracle_dispatch.restype = ctypes.c_int
        L.oracle_dispatch.argtypes = [ctypes.c_int] * 3 + [_i32p, _i32p, _i32p, _i32p]
        L.oracle_expert_rows.restype = ctypes.c_int
        L.oracle_expert_rows.argtypes = [ctypes.c_int] * 4 + [_vp] * 5 + [
            ctypes.c_int, _i32p, _i32p, _f64p, _vp, ctypes.c_int, ctypes.c_int]
        L.oracle_combine_tokens.restype = ctypes.c_int
        L.oracle_combine_tokens.argtypes = [ctypes.c_int] * 6 + [_vp] * 5 + [
            _i32p, _f32p, _i32p, ctypes.c_int, _i32p, _f64p, _vp, ctypes.c_int, ctypes.c_int]
        L.oracle_combine_given_y.restype = ctypes.c_int
        L.oracle_combine_given_y.argtypes = [ctypes.c_int] * 5 + [_vp, _vp, ctypes.c_longlong,
                                                                  _f32p, _i32p, _i32p, _i32p,
                                                                  _f64p, _vp]
        L.oracle_bf16_from_double.restype = ctypes.c_uint16
        L.oracle_bf16_from_double.argtypes = [ctypes.c_double]
        _lib = L
    return _lib


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _dtype_code(a):
    if a.dtype == np.float32:
        return 0
    if a.dtype == np.uint16:
        return 1
    raise TypeError("oracle takes float32 or bfloat16 bits (uint16), got %s" % a.dtype)


def _c(a, dt):
    return np.ascontiguousarray(a, dtype=dt)


def capacity(T, E, k, C):
    """K = min(T, floor(C*T*k/E)).  The library's interface carries C as a float32, so the
    oracle evaluates that same float32 value (e.g. 0.9 -> 0.89999998 gives 629, not 630, for
    T=700, k=3, E=3)."""
    return int(lib().oracle_capacity(T, E, k, float(np.float32(C))))


def own_exp(x):
    x = _c(np.atleast_1d(x), np.float32)
    y = np.empty_like(x)
    lib().oracle_own_exp_n(x.size, x.reshape(-1), y.reshape(-1))
    return y


def softmax(logits):
    L = _c(logits, np.float32)
    T, E = L.shape
    p = np.empty_like(L)
    lib().oracle_softmax(T, E, L, p)
    return p


def logits(x, Wr, br=None, nthreads=0):
    x = np.ascontiguousarray(x)
    T, d = x.shape
    Wr = _c(Wr, np.float32)
    E = Wr.shape[1]
    out = np.empty((T, E), np.float32)
    brc = None if br is None else _c(br, np.float32)
    lib().oracle_logits(T, d, E, _dtype_code(x), _ptr(x), Wr, _ptr(brc), out, nthreads)
    return out


RENORMALIZE = 1
ARRIVAL_ORDER = 2
GATED = 4


def route(logits_, k, K, flags=0):
    L = _c(logits_, np.float32)
    T, E = L.shape
    ids = np.empty((T, k), np.int32)
    w = np.empty((T, k), np.float32)
    slot = np.empty((T, k), np.int32)
    drop = np.empty((T, k), np.uint8)
    counts = np.empty(2 * E, np.int32)
    rc = lib().oracle_route(T, E, k, int(K), L, ids, w, slot, drop, counts, int(flags))
    if rc != 0:
        raise ValueError("oracle_route rejected its arguments")
    return dict(ids=ids, w=w, slot=slot, drop=drop, received=counts[:E].copy(),
                kept=counts[E:].copy())


def select(ids, w, E, K, flags=0):
    """Capacity selection of a given routing: ids/w [T, k] (pair p = t*k + j); each expert keeps
    at most K pairs by (weight descending, token ascending), or its first K in token order with
    ARRIVAL_ORDER; slots rank the kept tokens in token order."""
    ids = _c(ids, np.int32)
    w = _c(w, np.float32)
    T, k = ids.shape
    slot = np.empty((T, k), np.int32)
    drop = np.empty((T, k), np.uint8)
    counts = np.empty(2 * E, np.int32)
    rc = lib().oracle_select(T, E, k, int(K), ids, w, slot, drop, counts, int(flags))
    if rc != 0:
        raise ValueError("oracle_select rejected its arguments")
    return dict(slot=slot, drop=drop, received=counts[:E].copy(), kept=counts[E:].copy())


def dispatch(ids, slot, E):
    ids = _c(ids, np.int32)
    slot = _c(slot, np.int32)
    T, k = ids.shape
    offsets = np.empty(E + 1, np.int32)
    rowtok = np.full(max(T * k, 1), -1, np.int32)
    lib().oracle_dispatch(T, E, k, ids, slot, offsets, rowtok)
    return offsets, rowtok[: int(offsets[-1])].copy()


def expert_rows(x, W1, b1, W2, b2, row_tok, row_exp, want_h=False, nthreads=0, flags=0):
    """Expert outputs per (token, expert) row.  flags & GATED: W1 is [E, 2F, d] (gate, up)."""
    x = np.ascontiguousarray(x)
    W1 = np.ascontiguousarray(W1)
    W2 = np.ascontiguousarray(W2)
    E, d, F = W2.shape
    row_tok = _c(row_tok, np.int32)
    row_exp = _c(row_exp, np.int32)
    n = row_tok.size
    Y = np.empty((n, d), np.float64)
    H = np.empty((n, F), np.float64) if want_h else None
    b1c = None if b1 is None else _c(b1, np.float32)
    b2c = None if b2 is None else _c(b2, np.float32)
    rc = lib().oracle_expert_rows(d, F, E, _dtype_code(x), _ptr(x), _ptr(W1), _ptr(b1c),
                                  _ptr(W2), _ptr(b2c), n, row_tok, row_exp, Y, _ptr(H), nthreads,
                                  int(flags))
    if rc != 0:
        raise ValueError("oracle_expert_rows rejected its arguments")
    return (Y, H) if want_h else Y


def combine_tokens(x, W1, b1, W2, b2, route_, tokens=None, nthreads=0, flags=0):
    """Layer output for ``tokens`` (all when None) given a routing dict from :func:`route`.

    Returns ``(out_f64, out_x)``: the unrounded double result and the result in x's dtype."""
    x = np.ascontiguousarray(x)
    W1 = np.ascontiguousarray(W1)
    W2 = np.ascontiguousarray(W2)
    T, d = x.shape
    E, _, F = W2.shape
    ids, w, slot = (_c(route_["ids"], np.int32), _c(route_["w"], np.float32),
                    _c(route_["slot"], np.int32))
    k = ids.shape[1]
    tok = np.arange(T, dtype=np.int32) if tokens is None else _c(tokens, np.int32)
    out64 = np.empty((tok.size, d), np.float64)
    outx = np.empty((tok.size, d), x.dtype)
    b1c = None if b1 is None else _c(b1, np.float32)
    b2c = None if b2 is None else _c(b2, np.float32)
    rc = lib().oracle_combine_tokens(T, d, F, E, k, _dtype_code(x), _ptr(x), _ptr(W1), _ptr(b1c),
                                     _ptr(W2), _ptr(b2c), ids, w, slot, tok.size, tok, out64,
                                     _ptr(outx), nthreads, int(flags))
    if rc != 0:
        raise ValueError("oracle_combine_tokens rejected its arguments")
    return out64, outx


def forward(x, Wr, br, W1, b1, W2, b2, k, C, tokens=None, logits_=None, nthreads=0, flags=0):
    """The whole layer: logits (unless given), routing, and outputs for ``tokens``."""
    T = x.shape[0]
    E = W1.shape[0]
    L = logits(x, Wr, br, nthreads) if logits_ is None else _c(logits_, np.float32)
    K = capacity(T, E, k, C)
    r = route(L, k, K, flags & 3)
    out64, outx = combine_tokens(x, W1, b1, W2, b2, r, tokens, nthreads, flags)
    return dict(logits=L, K=K, route=r, out_f64=out64, out=outx)


def combine_given_y(x, Y, route_, offsets):
    """Combine alone from given expert outputs ``Y`` (rows in expert-sorted order)."""
    x = np.ascontiguousarray(x)
    Y = np.ascontiguousarray(Y, dtype=x.dtype)
    T, d = x.shape
    ids, w, slot = (_c(route_["ids"], np.int32), _c(route_["w"], np.float32),
                    _c(route_["slot"], np.int32))
    k = ids.shape[1]
    offsets = _c(offsets, np.int32)
    E = offsets.size - 1
    out64 = np.empty((T, d), np.float64)
    outx = np.empty((T, d), x.dtype)
    rc = lib().oracle_combine_given_y(T, d, E, k, _dtype_code(x), _ptr(x), _ptr(Y), Y.shape[0],
                                      w, ids, slot, offsets, out64, _ptr(outx))
    if rc != 0:
        raise ValueError("oracle_combine_given_y rejected its arguments")
    return out64, outx


def bf16_from_double(v):
    return int(lib().oracle_bf16_from_double(float(v)))
