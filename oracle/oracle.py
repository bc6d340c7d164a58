"""numpy front end of the C++ CPU oracle (test infrastructure only).

Every function takes and returns numpy arrays; floating inputs are widened to
fp64 exactly (bf16 values are passed in as the fp32/fp64 numbers they denote).
The arithmetic lives in ``dms_oracle.cpp``; this file only marshals arguments.
"""
import ctypes as C
import os

import numpy as np

from . import build as _build

_lib = None


def lib():
    global _lib
    if _lib is None:
        path = _build.build()
        L = C.CDLL(path)
        dp = C.POINTER(C.c_double)
        fp = C.POINTER(C.c_float)
        ip = C.POINTER(C.c_int)
        up = C.POINTER(C.c_uint8)
        L.oracle_set_threads.argtypes = [C.c_int]
        L.oracle_set_threads.restype = C.c_int
        L.oracle_e4m3_encode_n.argtypes = [fp, up, C.c_long]
        L.oracle_e4m3_decode_n.argtypes = [up, dp, C.c_long]
        L.oracle_decide_proj.argtypes = [C.c_int] * 4 + [dp] * 5 + [C.c_double, C.c_double, C.c_int, dp]
        L.oracle_decide_neuron.argtypes = [C.c_int] * 6 + [dp, dp, C.c_double, C.c_int, dp]
        L.oracle_decide_score.argtypes = [C.c_int] * 4 + [dp] * 4 + [C.c_int, dp]
        L.oracle_rope.argtypes = [C.c_int] * 4 + [dp, C.c_int, dp, dp]
        L.oracle_round_bf16_n.argtypes = [dp, fp, C.c_long]
        L.oracle_prefill_attention.argtypes = [C.c_int] * 6 + [dp, dp, dp, up, ip, C.c_long, dp]
        L.oracle_cache_new.argtypes = [C.c_int] * 12
        L.oracle_train_gate.argtypes = [C.c_int] * 3 + [dp, dp, C.c_double, dp, dp, dp]
        L.oracle_train_attention.argtypes = [C.c_int] * 6 + [dp] * 4 + [ip, C.c_long, dp]
        L.oracle_cache_new.restype = C.c_void_p
        L.oracle_cache_delete.argtypes = [C.c_void_p]
        L.oracle_cache_clone.argtypes = [C.c_void_p]
        L.oracle_cache_clone.restype = C.c_void_p
        L.oracle_cache_status.argtypes = [C.c_void_p]
        L.oracle_cache_status.restype = C.c_int
        L.oracle_cache_prefill.argtypes = [C.c_void_p, C.c_int, C.c_int, up, fp, fp]
        L.oracle_cache_append.argtypes = [C.c_void_p, C.c_int, up, fp, fp]
        L.oracle_cache_export.argtypes = [C.c_void_p, C.c_int, ip, ip, ip, ip, ip, ip, up, ip]
        L.oracle_cache_pages.argtypes = [C.c_void_p, dp, dp, up, up, fp, fp]
        L.oracle_cache_decode_attention.argtypes = [C.c_void_p, C.c_int, C.c_int, dp, dp]
        L.oracle_cache_prefill_attention.argtypes = [C.c_void_p, C.c_int, C.c_int, C.c_int, dp, dp, dp, up, ip,
                                                     C.c_long, dp]
        _lib = L
    return _lib


def _p(a, ctype):
    if a is None:
        return None
    return a.ctypes.data_as(C.POINTER(ctype))


def _f64(a):
    return np.ascontiguousarray(np.asarray(a, dtype=np.float64))


def _f32(a):
    return np.ascontiguousarray(np.asarray(a, dtype=np.float32))


def _u8(a):
    return np.ascontiguousarray(np.asarray(a, dtype=np.uint8))


def set_threads(n: int) -> int:
    """Set the OpenMP thread count (n <= 0 keeps it); returns the count in use."""
    return lib().oracle_set_threads(int(n))


def e4m3_encode(x):
    x = _f32(x)
    out = np.empty(x.shape, np.uint8)
    lib().oracle_e4m3_encode_n(_p(x, C.c_float), _p(out, C.c_uint8), x.size)
    return out


def e4m3_decode(c):
    c = _u8(c)
    out = np.empty(c.shape, np.float64)
    lib().oracle_e4m3_decode_n(_p(c, C.c_uint8), _p(out, C.c_double), c.size)
    return out


def decide_proj(h, gamma, W, bias, offset, scale=100.0, eps=1e-6, layer_mode=False):
    """alpha[B,Hkv,T] from h[B,T,hidden], RMSNorm weight gamma, Linear W[Hkv,hidden]."""
    h = _f64(h)
    B, T, hidden = h.shape
    W = _f64(W)
    Hkv = W.shape[0]
    off = _f64(np.broadcast_to(np.asarray(offset, np.float64), (B, Hkv)))
    bias = None if bias is None else _f64(bias)
    gamma = _f64(gamma)
    alpha = np.empty((B, Hkv, T), np.float64)
    lib().oracle_decide_proj(B, T, hidden, Hkv, _p(h, C.c_double), _p(gamma, C.c_double),
                             _p(W, C.c_double), _p(bias, C.c_double), _p(off, C.c_double),
                             float(scale), float(eps), int(bool(layer_mode)), _p(alpha, C.c_double))
    return alpha


def decide_score(h, W, bias, threshold, layer_mode=False):
    """alpha[B,Hkv,T] = threshold - (W . h + bias): the importance-score source."""
    h = _f64(h)
    B, T, hidden = h.shape
    W = _f64(W)
    Hkv = W.shape[0]
    thr = _f64(np.broadcast_to(np.asarray(threshold, np.float64), (B, Hkv)))
    bias = None if bias is None else _f64(bias)
    alpha = np.empty((B, Hkv, T), np.float64)
    lib().oracle_decide_score(B, T, hidden, Hkv, _p(h, C.c_double), _p(W, C.c_double), _p(bias, C.c_double),
                              _p(thr, C.c_double), int(bool(layer_mode)), _p(alpha, C.c_double))
    return alpha


def decide_neuron(x, group, Hkv, offset, scale=100.0, layer_mode=False):
    """alpha[B,Hkv,T] from the last element of x[B,T,Hsrc,D] heads 0, group, 2*group, ...

    Returns (alpha, x_zeroed): a copy of x with each decision element set to 0.
    """
    x = _f64(x).copy()
    B, T, Hsrc, D = x.shape
    off = _f64(np.broadcast_to(np.asarray(offset, np.float64), (B, Hkv)))
    alpha = np.empty((B, Hkv, T), np.float64)
    lib().oracle_decide_neuron(B, T, Hsrc, D, int(group), Hkv, _p(x, C.c_double), _p(off, C.c_double),
                               float(scale), int(bool(layer_mode)), _p(alpha, C.c_double))
    return alpha, x


def rope(x, pos0, cos, sin):
    """Half-split rotary embedding of x[B,T,H,D] at positions pos0.. (returns a copy)."""
    x = _f64(x).copy()
    B, T, H, D = x.shape
    cos = _f64(cos)
    sin = _f64(sin)
    lib().oracle_rope(B, T, H, D, _p(x, C.c_double), int(pos0), _p(cos, C.c_double), _p(sin, C.c_double))
    return x


def round_bf16(x):
    """fp64 values rounded once (nearest, ties to even) to bfloat16; returned as fp64."""
    x = _f64(x)
    out = np.empty(x.shape, np.float32)
    lib().oracle_round_bf16_n(_p(x, C.c_double), _p(out, C.c_float), x.size)
    return out.astype(np.float64)


def round_to(x, dtype):
    """fp64 values stored in the activation dtype ("f32" or "bf16"), one rounding."""
    if dtype == "bf16":
        return round_bf16(x)
    return _f64(x).astype(np.float32).astype(np.float64)


def evict_bits(alpha, disable_eviction=False):
    """Inference decision: evict iff alpha > 0 (and eviction is enabled)."""
    a = np.asarray(alpha)
    if disable_eviction:
        return np.zeros(a.shape, np.uint8)
    return (a > 0).astype(np.uint8)


def prefill_attention(q, k, v, evict, window, rows=None):
    """o[B,T,Hq,D] (or o[len(rows),D] for a list of (b, hq, i) rows), fp64."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, T, Hq, D = q.shape
    Hkv = k.shape[2]
    ev = _u8(evict)
    assert ev.shape == (B, Hkv, T)
    if rows is None:
        o = np.empty((B, T, Hq, D), np.float64)
        rp, n = None, 0
    else:
        r = np.ascontiguousarray(np.asarray(rows, np.int32).reshape(-1, 3))
        o = np.empty((r.shape[0], D), np.float64)
        rp, n = _p(r, C.c_int), r.shape[0]
    lib().oracle_prefill_attention(B, T, Hq, Hkv, D, int(window), _p(q, C.c_double), _p(k, C.c_double),
                                   _p(v, C.c_double), _p(ev, C.c_uint8), rp, n, _p(o, C.c_double))
    return o


def train_gate(alpha, noise, tau):
    """(prob, hard, penalty) [B,Hkv,T] of the training path's gate (fp64)."""
    a = _f64(alpha)
    B, H, T = a.shape
    g = None if noise is None else _f64(noise)
    prob, hard, pen = (np.empty((B, H, T), np.float64) for _ in range(3))
    lib().oracle_train_gate(B, H, T, _p(a, C.c_double), _p(g, C.c_double), float(tau), _p(prob, C.c_double),
                            _p(hard, C.c_double), _p(pen, C.c_double))
    return prob, hard, pen


def train_attention(q, k, v, penalty, window, rows=None):
    """The soft-gated training attention, o[B,T,Hq,D] (or o[len(rows),D])."""
    q, k, v, pen = _f64(q), _f64(k), _f64(v), _f64(penalty)
    B, T, Hq, D = q.shape
    Hkv = k.shape[2]
    if rows is None:
        o = np.empty((B, T, Hq, D), np.float64)
        rp, n = None, 0
    else:
        r = np.ascontiguousarray(np.asarray(rows, np.int32).reshape(-1, 3))
        o = np.empty((r.shape[0], D), np.float64)
        rp, n = _p(r, C.c_int), r.shape[0]
    lib().oracle_train_attention(B, T, Hq, Hkv, D, int(window), _p(q, C.c_double), _p(k, C.c_double),
                                 _p(v, C.c_double), _p(pen, C.c_double), rp, n, _p(o, C.c_double))
    return o


class Cache:
    """Sequential simulation of the paged DMS cache (one object per test)."""

    def __init__(self, L, B, Hkv, D, window, block, max_pos, pool_pages, prealloc_tokens=0,
                 fp8=False, store_values=True, shift=0):
        self.L, self.B, self.Hkv, self.D = L, B, Hkv, D
        self.w, self.P, self.max_pos = window, block, max_pos
        self.maxp = (max_pos + block - 1) // block
        self.cap = self.maxp * block
        self.pool_pages = pool_pages
        self.fp8 = bool(fp8)
        self.store_values = bool(store_values)
        self.shift = int(shift)
        self._h = lib().oracle_cache_new(L, B, Hkv, D, window, block, max_pos, pool_pages,
                                         prealloc_tokens, int(self.fp8), int(self.store_values), self.shift)

    def clone(self):
        """An independent copy (state and pages) of this cache."""
        c = Cache.__new__(Cache)
        c.__dict__.update({k: v for k, v in self.__dict__.items() if k != "_h"})
        c._h = lib().oracle_cache_clone(self._h)
        return c

    def __del__(self):
        if getattr(self, "_h", None):
            lib().oracle_cache_delete(self._h)
            self._h = None

    @property
    def status(self):
        return lib().oracle_cache_status(self._h)

    def prefill(self, layer, evict, k=None, v=None):
        ev = _u8(evict)
        T = ev.shape[-1]
        kk = None if k is None else _f32(k)
        vv = None if v is None else _f32(v)
        lib().oracle_cache_prefill(self._h, layer, T, _p(ev, C.c_uint8), _p(kk, C.c_float), _p(vv, C.c_float))

    def append(self, layer, evict, k=None, v=None):
        ev = _u8(evict)
        kk = None if k is None else _f32(k)
        vv = None if v is None else _f32(v)
        lib().oracle_cache_append(self._h, layer, _p(ev, C.c_uint8), _p(kk, C.c_float), _p(vv, C.c_float))

    def export(self, layer):
        B, H = self.B, self.Hkv
        out = dict(
            npos=np.empty((B, H), np.int32), count=np.empty((B, H), np.int32),
            npages=np.empty((B, H), np.int32), page_table=np.empty((B, H, self.maxp), np.int32),
            slot_pos=np.empty((B, H, self.cap), np.int32), ring_slot=np.empty((B, H, self.w), np.int32),
            ring_evict=np.empty((B, H, self.w), np.uint8))
        nxt = np.zeros(1, np.int32)
        lib().oracle_cache_export(self._h, layer, *[_p(out[k], C.c_int) for k in
                                                    ("npos", "count", "npages", "page_table", "slot_pos", "ring_slot")],
                                  _p(out["ring_evict"], C.c_uint8), _p(nxt, C.c_int))
        out["next_page"] = int(nxt[0])
        return out

    def pages(self):
        n = (self.pool_pages, self.P, self.D)
        kv, vv = np.empty(n, np.float64), np.empty(n, np.float64)
        kc, vc = np.zeros(n, np.uint8), np.zeros(n, np.uint8)
        ks, vs = np.zeros(self.pool_pages, np.float32), np.zeros(self.pool_pages, np.float32)
        lib().oracle_cache_pages(self._h, _p(kv, C.c_double), _p(vv, C.c_double), _p(kc, C.c_uint8),
                                 _p(vc, C.c_uint8), _p(ks, C.c_float), _p(vs, C.c_float))
        return dict(kval=kv, vval=vv, kcode=kc, vcode=vc, kscale=ks, vscale=vs)

    def decode_attention(self, layer, q):
        q = _f64(q)
        B, Hq, D = q.shape
        o = np.empty_like(q)
        lib().oracle_cache_decode_attention(self._h, layer, Hq, _p(q, C.c_double), _p(o, C.c_double))
        return o

    def prefill_attention(self, layer, q, k, v, evict, rows=None):
        """Attention of a prefill call's rows against the cache as it is now
        (call before prefill() of the same tokens) plus the call's own keys.
        q [B,T,Hq,D], k/v [B,T,Hkv,D], evict [B,Hkv,T]; returns o[B,T,Hq,D] or
        o[len(rows),D] for (b, hq, i) rows."""
        q, k, v = _f64(q), _f64(k), _f64(v)
        B, T, Hq, D = q.shape
        ev = _u8(evict)
        assert ev.shape == (B, self.Hkv, T)
        if rows is None:
            o = np.empty((B, T, Hq, D), np.float64)
            rp, n = None, 0
        else:
            r = np.ascontiguousarray(np.asarray(rows, np.int32).reshape(-1, 3))
            o = np.empty((r.shape[0], D), np.float64)
            rp, n = _p(r, C.c_int), r.shape[0]
        lib().oracle_cache_prefill_attention(self._h, layer, T, Hq, _p(q, C.c_double), _p(k, C.c_double),
                                             _p(v, C.c_double), _p(ev, C.c_uint8), rp, n, _p(o, C.c_double))
        return o
