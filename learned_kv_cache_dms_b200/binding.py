"""Thin Python binding of libdms (include/dms.h): argument marshalling only.

Every function here forwards to the C entry point of the same name.  PyTorch is
used for device memory and streams: the caller passes torch CUDA tensors, whose
data pointers and the current stream go through the C ABI unchanged.  All
arithmetic of the DMS path runs in libdms's CUDA kernels; there is no fallback.
"""
from __future__ import annotations

import ctypes as C
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
# DMS_LIB_PATH selects another build of the same library (e.g. a tracing build)
LIB_PATH = os.environ.get("DMS_LIB_PATH") or os.path.join(_PKG, "libdms.so")

if not os.path.exists(LIB_PATH):
    raise ImportError("libdms.so is not built: run `python -m learned_kv_cache_dms_b200.build` "
                      "(needs nvcc for sm_100a)")

_lib = C.CDLL(LIB_PATH)

# ---- constants (mirror include/dms.h) ---------------------------------------
DMS_OK, DMS_ERR_INVALID, DMS_ERR_STATE, DMS_ERR_CUDA, DMS_ERR_NOMEM, DMS_ERR_SCRATCH_LIMIT = 0, -1, -2, -3, -4, -5
DMS_ST_POOL_EXHAUSTED, DMS_ST_CAPACITY, DMS_ST_TIMEOUT, DMS_ST_SPLIT_LIMIT = 1, 2, 4, 8
DMS_F32, DMS_BF16, DMS_FP8_E4M3 = 0, 1, 2
DMS_ALPHA_PER_HEAD, DMS_ALPHA_PER_LAYER = 0, 1
DMS_ALPHA_PROJ, DMS_ALPHA_KEY_NEURON, DMS_ALPHA_QUERY_NEURON, DMS_ALPHA_SCORE_LINEAR = 0, 1, 2, 3
DMS_DECODE_AUTO, DMS_DECODE_CLUSTER, DMS_DECODE_FLAT = 0, 1, 2

_ERRORS = {DMS_ERR_INVALID: "DMS_ERR_INVALID", DMS_ERR_STATE: "DMS_ERR_STATE", DMS_ERR_CUDA: "DMS_ERR_CUDA",
           DMS_ERR_NOMEM: "DMS_ERR_NOMEM", DMS_ERR_SCRATCH_LIMIT: "DMS_ERR_SCRATCH_LIMIT"}


class DMSError(RuntimeError):
    def __init__(self, code, where):
        super().__init__("%s returned %s" % (where, _ERRORS.get(code, code)))
        self.code = code


class dms_cache_desc(C.Structure):
    _fields_ = [(n, C.c_int) for n in ("num_layers", "batch", "num_q_heads", "num_kv_heads", "head_dim", "hidden",
                                       "window", "block", "max_positions", "prealloc_tokens", "pool_pages",
                                       "act_dtype", "kv_dtype", "alpha_per", "alpha_source")] + \
              [("alpha_scale", C.c_float), ("rms_eps", C.c_float), ("disable_eviction", C.c_int),
               ("decode_kernel", C.c_int), ("decision_shift", C.c_int)]


class dms_cache_view(C.Structure):
    _fields_ = [(n, C.c_void_p) for n in ("pos", "count", "npages", "page_table", "slot_pos", "ring")]


class dms_cache_layout(C.Structure):
    _fields_ = [(n, C.c_size_t) for n in ("total_bytes", "status", "next_page", "pos", "count", "npages",
                                          "page_table", "slot_pos", "ring", "k_pool", "v_pool", "k_scale",
                                          "v_scale")] + \
              [(n, C.c_int) for n in ("max_pages_per_head", "slot_capacity", "prealloc_pages", "first_free_page")]


class dms_decide_params(C.Structure):
    _fields_ = [("hidden", C.c_void_p), ("norm_weight", C.c_void_p), ("proj_weight", C.c_void_p),
                ("proj_bias", C.c_void_p), ("offset", C.c_void_p), ("offset_batch_stride", C.c_int)]


class dms_prefill_args(C.Structure):
    _fields_ = [("seq_len", C.c_int), ("q", C.c_void_p), ("k", C.c_void_p), ("v", C.c_void_p), ("o", C.c_void_p),
                ("alpha", C.c_void_p), ("decide", C.POINTER(dms_decide_params)), ("rope_cos", C.c_void_p),
                ("rope_sin", C.c_void_p)]


class dms_decode_args(C.Structure):
    _fields_ = [("q", C.c_void_p), ("k", C.c_void_p), ("v", C.c_void_p), ("o", C.c_void_p), ("alpha", C.c_void_p),
                ("decide", C.POINTER(dms_decide_params)), ("rope_cos", C.c_void_p), ("rope_sin", C.c_void_p)]


_P = C.c_void_p
_lib.dms_cache_desc_default.argtypes = [C.POINTER(dms_cache_desc)]
_lib.dms_cache_desc_default.restype = None
_lib.dms_cache_bytes.argtypes = [C.POINTER(dms_cache_desc), C.POINTER(C.c_size_t)]
_lib.dms_cache_alloc.argtypes = [C.POINTER(dms_cache_desc), _P, C.c_size_t, _P, C.POINTER(_P)]
_lib.dms_cache_free.argtypes = [_P]
_lib.dms_cache_reset.argtypes = [_P, _P]
_lib.dms_cache_get_layout.argtypes = [_P, C.POINTER(dms_cache_layout)]
_lib.dms_cache_status.argtypes = [_P, _P, C.POINTER(C.c_int)]
_lib.dms_cache_export.argtypes = [_P, C.c_int, C.POINTER(dms_cache_view), _P]
_lib.dms_decide.argtypes = [_P, C.c_int, C.POINTER(dms_decide_params), _P, _P, _P]
_lib.dms_prefill.argtypes = [_P, C.c_int, C.POINTER(dms_prefill_args), _P]
_lib.dms_decode_step.argtypes = [_P, C.c_int, C.POINTER(dms_decode_args), _P]
_lib.dms_prefill_compact.argtypes = [_P, C.c_int, C.POINTER(dms_prefill_args), _P]
_lib.dms_prefill_attention.argtypes = [_P, C.c_int, C.POINTER(dms_prefill_args), _P]
_lib.dms_decode_append.argtypes = [_P, C.c_int, C.POINTER(dms_decode_args), _P]
_lib.dms_decode_attention.argtypes = [_P, C.c_int, _P, _P, _P]
_lib.dms_decode_attention_noalloc.argtypes = [_P, C.c_int, _P, _P, _P]
_lib.dms_cache_positions.argtypes = [_P, C.c_int]
_lib.dms_selftest_wait_timeout.argtypes = [_P, C.c_int, _P]
_lib.dms_decode_step_layers.argtypes = [_P, C.c_int, C.c_int, C.POINTER(dms_decode_args), _P]
_lib.dms_train_gate.argtypes = [_P, C.c_int, _P, _P, C.c_float, _P, _P, _P, _P]
_lib.dms_train_attention.argtypes = [_P, C.c_int, _P, _P, _P, _P, _P, _P]
for _f in ("dms_cache_bytes", "dms_cache_alloc", "dms_cache_free", "dms_cache_reset", "dms_cache_get_layout",
           "dms_cache_status", "dms_decide", "dms_prefill", "dms_decode_step", "dms_cache_positions",
           "dms_prefill_compact", "dms_prefill_attention", "dms_decode_append", "dms_decode_attention",
           "dms_decode_attention_noalloc", "dms_cache_export", "dms_selftest_wait_timeout",
           "dms_decode_step_layers", "dms_train_gate", "dms_train_attention"):
    getattr(_lib, _f).restype = C.c_int

EXPORTED = ("dms_cache_desc_default", "dms_cache_bytes", "dms_cache_alloc", "dms_cache_free", "dms_cache_reset",
            "dms_cache_get_layout", "dms_cache_status", "dms_decide", "dms_prefill", "dms_decode_step",
            "dms_cache_positions", "dms_prefill_compact", "dms_prefill_attention", "dms_decode_append",
            "dms_decode_attention", "dms_decode_attention_noalloc", "dms_cache_export",
            "dms_selftest_wait_timeout", "dms_decode_step_layers", "dms_train_gate", "dms_train_attention")


def _check(code, where):
    if code < 0:
        raise DMSError(code, where)
    return code


def _ptr(t):
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _stream(stream=None):
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else stream


# ---- the C entry points, one to one -------------------------------------------
def dms_cache_desc_default() -> dms_cache_desc:
    d = dms_cache_desc()
    _lib.dms_cache_desc_default(C.byref(d))
    return d


def dms_cache_bytes(desc: dms_cache_desc) -> int:
    n = C.c_size_t(0)
    _check(_lib.dms_cache_bytes(C.byref(desc), C.byref(n)), "dms_cache_bytes")
    return n.value


def dms_cache_alloc(desc: dms_cache_desc, dev_mem: int, nbytes: int, stream=None) -> int:
    h = C.c_void_p()
    _check(_lib.dms_cache_alloc(C.byref(desc), dev_mem, nbytes, _stream(stream), C.byref(h)), "dms_cache_alloc")
    return h.value


def dms_cache_free(handle: int) -> None:
    _check(_lib.dms_cache_free(handle), "dms_cache_free")


def dms_cache_reset(handle: int, stream=None) -> None:
    _check(_lib.dms_cache_reset(handle, _stream(stream)), "dms_cache_reset")


def dms_cache_get_layout(handle: int) -> dms_cache_layout:
    l = dms_cache_layout()
    _check(_lib.dms_cache_get_layout(handle, C.byref(l)), "dms_cache_get_layout")
    return l


def dms_cache_export(handle: int, layer: int, desc, layout, stream=None) -> dict:
    """Host (numpy int32) copies of one layer's state: pos [B], count and
    npages [B,Hkv], page_table [B,Hkv,maxp], slot_pos [B,Hkv,cap], ring
    [B,Hkv,w] (bit 31: eviction decision)."""
    import numpy as np
    B, H, w = desc.batch, desc.num_kv_heads, desc.window
    maxp, cap = layout.max_pages_per_head, layout.slot_capacity
    out = dict(pos=np.zeros(B, np.int32), count=np.zeros((B, H), np.int32), npages=np.zeros((B, H), np.int32),
               page_table=np.zeros((B, H, maxp), np.int32), slot_pos=np.zeros((B, H, cap), np.int32),
               ring=np.zeros((B, H, w), np.int32))
    v = dms_cache_view(*[out[k].ctypes.data for k in ("pos", "count", "npages", "page_table", "slot_pos", "ring")])
    _check(_lib.dms_cache_export(handle, layer, C.byref(v), _stream(stream)), "dms_cache_export")
    return out


def dms_cache_status(handle: int, stream=None) -> int:
    s = C.c_int(0)
    _check(_lib.dms_cache_status(handle, _stream(stream), C.byref(s)), "dms_cache_status")
    return s.value


def dms_decide(handle: int, seq_len: int, decide: dms_decide_params, neuron_src, alpha, stream=None) -> None:
    _check(_lib.dms_decide(handle, seq_len, C.byref(decide), _ptr(neuron_src), _ptr(alpha), _stream(stream)),
           "dms_decide")


def dms_prefill(handle: int, layer: int, args: dms_prefill_args, stream=None) -> None:
    _check(_lib.dms_prefill(handle, layer, C.byref(args), _stream(stream)), "dms_prefill")


def dms_decode_step(handle: int, layer: int, args: dms_decode_args, stream=None) -> None:
    _check(_lib.dms_decode_step(handle, layer, C.byref(args), _stream(stream)), "dms_decode_step")


def dms_prefill_compact(handle: int, layer: int, args: dms_prefill_args, stream=None) -> None:
    _check(_lib.dms_prefill_compact(handle, layer, C.byref(args), _stream(stream)), "dms_prefill_compact")


def dms_prefill_attention(handle: int, layer: int, args: dms_prefill_args, stream=None) -> None:
    _check(_lib.dms_prefill_attention(handle, layer, C.byref(args), _stream(stream)), "dms_prefill_attention")


def dms_decode_append(handle: int, layer: int, args: dms_decode_args, stream=None) -> None:
    _check(_lib.dms_decode_append(handle, layer, C.byref(args), _stream(stream)), "dms_decode_append")


def dms_decode_attention(handle: int, layer: int, q, o, stream=None) -> None:
    _check(_lib.dms_decode_attention(handle, layer, _ptr(q), _ptr(o), _stream(stream)), "dms_decode_attention")


def dms_decode_attention_noalloc(handle: int, layer: int, q, o, stream=None) -> None:
    """dms_decode_attention with its split-K scratch in the library's fixed
    device array instead of the cache buffer (see include/dms.h)."""
    _check(_lib.dms_decode_attention_noalloc(handle, layer, _ptr(q), _ptr(o), _stream(stream)),
           "dms_decode_attention_noalloc")


def dms_cache_positions(handle: int, layer: int) -> int:
    return _check(_lib.dms_cache_positions(handle, layer), "dms_cache_positions")


def dms_decode_step_layers(handle: int, layer: int, num_layers: int, args: dms_decode_args, stream=None) -> None:
    _check(_lib.dms_decode_step_layers(handle, layer, num_layers, C.byref(args), _stream(stream)),
           "dms_decode_step_layers")


def dms_train_gate(handle: int, seq_len: int, alpha, noise, tau: float, prob, hard, penalty, stream=None) -> None:
    _check(_lib.dms_train_gate(handle, seq_len, _ptr(alpha), _ptr(noise), float(tau), _ptr(prob), _ptr(hard),
                               _ptr(penalty), _stream(stream)), "dms_train_gate")


def dms_train_attention(handle: int, seq_len: int, q, k, v, penalty, o, stream=None) -> None:
    _check(_lib.dms_train_attention(handle, seq_len, _ptr(q), _ptr(k), _ptr(v), _ptr(penalty), _ptr(o),
                                    _stream(stream)), "dms_train_attention")


def dms_selftest_wait_timeout(handle: int, tries: int, stream=None) -> None:
    _check(_lib.dms_selftest_wait_timeout(handle, tries, _stream(stream)), "dms_selftest_wait_timeout")


# ---- convenience wrapper over torch tensors (still marshalling only) ---------
def decide_params(offset, hidden=None, norm_weight=None, proj_weight=None, proj_bias=None):
    """dms_decide_params over torch tensors; offset is [Hkv] or [B, Hkv] fp32."""
    p = dms_decide_params()
    p.hidden, p.norm_weight, p.proj_weight = _ptr(hidden), _ptr(norm_weight), _ptr(proj_weight)
    p.proj_bias, p.offset = _ptr(proj_bias), _ptr(offset)
    p.offset_batch_stride = offset.shape[-1] if offset.dim() == 2 else 0
    return p


class Cache:
    """A DMS cache whose device buffer is a torch uint8 tensor."""

    def __init__(self, desc: dms_cache_desc, device=None, stream=None):
        self.desc = desc
        self.nbytes = dms_cache_bytes(desc)
        self.buffer = torch.empty(self.nbytes, dtype=torch.uint8, device=device or "cuda")
        self.handle = dms_cache_alloc(desc, self.buffer.data_ptr(), self.nbytes, stream)
        self.layout = dms_cache_get_layout(self.handle)
        self._keep = []

    def close(self):
        if self.handle:
            dms_cache_free(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def reset(self, stream=None):
        dms_cache_reset(self.handle, stream)

    def status(self, stream=None) -> int:
        return dms_cache_status(self.handle, stream)

    def positions(self, layer: int) -> int:
        return dms_cache_positions(self.handle, layer)

    @staticmethod
    def prefill_args(q, k, v, o, alpha, decide: dms_decide_params | None = None, rope=None) -> dms_prefill_args:
        a = dms_prefill_args()
        a.seq_len = q.shape[1]
        a.q, a.k, a.v, a.o, a.alpha = _ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(alpha)
        a.decide = C.pointer(decide) if decide is not None else None
        a.rope_cos, a.rope_sin = (_ptr(rope[0]), _ptr(rope[1])) if rope is not None else (None, None)
        return a

    @staticmethod
    def decode_args(q, k, v, o, alpha, decide: dms_decide_params | None = None, rope=None) -> dms_decode_args:
        a = dms_decode_args()
        a.q, a.k, a.v, a.o, a.alpha = _ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(alpha)
        a.decide = C.pointer(decide) if decide is not None else None
        a.rope_cos, a.rope_sin = (_ptr(rope[0]), _ptr(rope[1])) if rope is not None else (None, None)
        return a

    def prefill(self, layer, q, k, v, o, alpha, decide: dms_decide_params | None = None, rope=None, stream=None):
        dms_prefill(self.handle, layer, self.prefill_args(q, k, v, o, alpha, decide, rope), stream)

    def decode_step(self, layer, q, k, v, o, alpha, decide: dms_decide_params | None = None, rope=None,
                    stream=None):
        dms_decode_step(self.handle, layer, self.decode_args(q, k, v, o, alpha, decide, rope), stream)

    # --- state views (for inspection) ---
    def _view(self, off, n, dtype):
        esz = torch.empty(0, dtype=dtype).element_size()
        return self.buffer[off:off + n * esz].view(dtype)

    def state(self, layer):
        d, l = self.desc, self.layout
        B, H, L = d.batch, d.num_kv_heads, d.num_layers
        maxp, cap, w = l.max_pages_per_head, l.slot_capacity, d.window
        nb = B * H
        i32 = torch.int32
        ring = self._view(l.ring, L * nb * w, i32).view(L, B, H, w)[layer]
        return dict(
            pos=self._view(l.pos, L * B, i32).view(L, B)[layer],
            count=self._view(l.count, L * nb, i32).view(L, B, H)[layer],
            npages=self._view(l.npages, L * nb, i32).view(L, B, H)[layer],
            page_table=self._view(l.page_table, L * nb * maxp, i32).view(L, B, H, maxp)[layer],
            slot_pos=self._view(l.slot_pos, L * nb * cap, i32).view(L, B, H, cap)[layer],
            ring_slot=ring & 0x7FFFFFFF,
            ring_evict=((ring >> 31) & 1).to(torch.uint8),
            next_page=self._view(l.next_page, 1, i32),
            status=self._view(l.status, 1, i32),
        )

    def export(self, layer: int, stream=None) -> dict:
        """dms_cache_export of one layer (host numpy copies)."""
        return dms_cache_export(self.handle, layer, self.desc, self.layout, stream)

    def counts(self):
        """Retained lengths of every layer, [L, B, Hkv] int32 (a view of the cache)."""
        d, l = self.desc, self.layout
        nb = d.num_layers * d.batch * d.num_kv_heads
        return self._view(l.count, nb, torch.int32).view(d.num_layers, d.batch, d.num_kv_heads)

    def pages(self):
        d, l = self.desc, self.layout
        shape = (d.pool_pages, d.block, d.head_dim)
        n = d.pool_pages * d.block * d.head_dim
        dt = {DMS_F32: torch.float32, DMS_BF16: torch.bfloat16, DMS_FP8_E4M3: torch.uint8}[d.kv_dtype]
        out = dict(k=self._view(l.k_pool, n, dt).view(shape), v=self._view(l.v_pool, n, dt).view(shape))
        if d.kv_dtype == DMS_FP8_E4M3:
            out["k_scale"] = self._view(l.k_scale, d.pool_pages, torch.float32)
            out["v_scale"] = self._view(l.v_scale, d.pool_pages, torch.float32)
        return out
