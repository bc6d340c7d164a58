"""CPU checks of the C ABI: the library loads, exports every declared symbol, and
rejects bad descriptors on the host (no GPU needed)."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "dms.h")


def declared_functions():
    src = open(HEADER).read()
    return sorted(set(re.findall(r"DMS_API\s+[\w\s\*]+?\b(dms_\w+)\s*\(", src)))


@pytest.fixture(scope="module")
def B():
    from learned_kv_cache_dms_b200 import build
    build.build()
    from learned_kv_cache_dms_b200 import binding
    return binding


def test_header_declares_entry_points():
    names = declared_functions()
    for n in ("dms_cache_bytes", "dms_cache_alloc", "dms_cache_free", "dms_prefill", "dms_decode_step",
              "dms_decide", "dms_cache_status", "dms_cache_reset"):
        assert n in names


def test_library_exports_every_declared_symbol(B):
    lib = ctypes.CDLL(B.LIB_PATH)
    for n in declared_functions():
        assert hasattr(lib, n), n
    assert sorted(B.EXPORTED) == declared_functions()


def good_desc(B):
    d = B.dms_cache_desc_default()
    d.num_layers, d.batch, d.num_q_heads, d.num_kv_heads, d.head_dim, d.hidden = 1, 2, 8, 2, 128, 512
    d.window, d.block, d.max_positions, d.prealloc_tokens = 64, 32, 300, 64
    d.pool_pages = 64
    return d


def test_defaults_follow_config_record(B):
    d = B.dms_cache_desc_default()
    assert (d.window, d.block, d.prealloc_tokens) == (512, 256, 4096)
    assert d.alpha_scale == 100.0 and d.alpha_per == B.DMS_ALPHA_PER_HEAD and d.disable_eviction == 0


def test_cache_bytes_and_validation(B):
    d = good_desc(B)
    n = B.dms_cache_bytes(d)
    assert n > 2 * 64 * 32 * 128 * 2  # at least the two page pools
    bad = [
        ("window", 32),          # window must exceed the block
        ("block", 24),           # block % 16
        ("head_dim", 96),
        ("num_q_heads", 7),      # not a multiple of kv heads
        ("alpha_per", 2),
        ("alpha_source", 4),
        ("kv_dtype", 2),         # FP8 pages need bf16 activations: ok here...
    ]
    for field, val in bad[:-1]:
        e = good_desc(B)
        setattr(e, field, val)
        with pytest.raises(B.DMSError) as ex:
            B.dms_cache_bytes(e)
        assert ex.value.code == B.DMS_ERR_INVALID, field
    e = good_desc(B)
    e.act_dtype, e.kv_dtype = B.DMS_F32, B.DMS_FP8_E4M3  # ...but not fp32 activations
    with pytest.raises(B.DMSError):
        B.dms_cache_bytes(e)
    e = good_desc(B)
    e.pool_pages = 3  # smaller than the preallocation (1*2*2*2 pages)
    with pytest.raises(B.DMSError):
        B.dms_cache_bytes(e)


def test_null_handles_rejected(B):
    assert B._lib.dms_cache_free(None) == 0
    assert B._lib.dms_cache_reset(None, None) == B.DMS_ERR_INVALID
    assert B._lib.dms_prefill(None, 0, None, None) == B.DMS_ERR_INVALID
    assert B._lib.dms_decode_step(None, 0, None, None) == B.DMS_ERR_INVALID


def test_every_entry_point_rejects_bad_arguments(B):
    """Argument checks happen on the host before any CUDA call: null handles,
    null outputs, layers out of range and caller buffers that are missing,
    misaligned or too small all come back as error codes."""
    import ctypes as C
    L = B._lib
    inv = B.DMS_ERR_INVALID
    d = good_desc(B)
    n = C.c_size_t(0)
    assert L.dms_cache_bytes(None, C.byref(n)) == inv
    assert L.dms_cache_bytes(C.byref(d), None) == inv
    # alloc: output handle, descriptor, buffer (never dereferenced: every
    # check below returns before the pointer is used)
    out = C.c_void_p(1)
    need = B.dms_cache_bytes(d)
    fake = 1 << 20  # 256-byte aligned, not a real allocation
    assert L.dms_cache_alloc(C.byref(d), C.c_void_p(fake), need, None, None) == inv
    assert L.dms_cache_alloc(None, C.c_void_p(fake), need, None, C.byref(out)) == inv and out.value is None
    assert L.dms_cache_alloc(C.byref(d), None, need, None, C.byref(out)) == inv
    assert L.dms_cache_alloc(C.byref(d), C.c_void_p(fake + 8), need, None, C.byref(out)) == inv
    assert L.dms_cache_alloc(C.byref(d), C.c_void_p(fake), need - 1, None, C.byref(out)) == B.DMS_ERR_NOMEM
    # every call on a null cache
    lay = B.dms_cache_layout()
    view = B.dms_cache_view()
    st = C.c_int(0)
    alpha = C.c_void_p(fake)
    assert L.dms_cache_get_layout(None, C.byref(lay)) == inv
    assert L.dms_cache_export(None, 0, C.byref(view), None) == inv
    assert L.dms_cache_status(None, None, C.byref(st)) == inv
    assert L.dms_cache_positions(None, 0) == inv
    assert L.dms_decide(None, 16, None, None, alpha, None) == inv
    assert L.dms_prefill_compact(None, 0, None, None) == inv
    assert L.dms_prefill_attention(None, 0, None, None) == inv
    assert L.dms_decode_append(None, 0, None, None) == inv
    assert L.dms_decode_attention(None, 0, alpha, alpha, None) == inv
    assert L.dms_decode_attention_noalloc(None, 0, alpha, alpha, None) == inv

