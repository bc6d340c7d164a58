"""Failure detection on the GPU without any GPU fault.

- Calls made in the wrong state, or with misaligned rows, are refused on the
  host (DMS_ERR_STATE / DMS_ERR_INVALID) before anything is launched.
- A prefill into an undersized page pool sets DMS_ST_POOL_EXHAUSTED in the
  device status word, as the oracle's replay of the same prompt does; the
  kernels skip the rows that have no page.
- A bounded device wait that nothing completes gives up and sets
  DMS_ST_TIMEOUT; the context stays usable and a reset clears the bit.
- A cache emptied by dms_cache_reset and filled again gives the same state and
  outputs as a fresh oracle run of the new inputs.
"""
import dataclasses

import numpy as np
import pytest
import torch

from harness import Case, build, check_case, make_desc
from oracle import oracle as O

SMALL = Case(B=2, T=200, steps=6, Hq=8, Hkv=2, D=64, w=32, P=16, act="bf16", kv="bf16", source="input",
             keep=0.3, seed=41)


def _cache(case):
    from learned_kv_cache_dms_b200 import binding as B_
    return B_, B_.Cache(make_desc(B_, case), torch.device("cuda"))


def _code(B_, fn, *a):
    with pytest.raises(B_.DMSError) as ex:
        fn(*a)
    return ex.value.code


@pytest.mark.gpu
def test_calls_in_the_wrong_state_are_refused():
    B_, cache = _cache(SMALL)
    dev = "cuda"
    B, T, Hq, Hkv, D = SMALL.B, SMALL.T, SMALL.Hq, SMALL.Hkv, SMALL.D
    q1 = torch.zeros(B, Hq, D, dtype=torch.bfloat16, device=dev)
    k1 = torch.zeros(B, Hkv, D, dtype=torch.bfloat16, device=dev)
    a1 = -torch.ones(B, Hkv, dtype=torch.float32, device=dev)
    o1 = torch.empty_like(q1)
    st = B_.DMS_ERR_STATE
    # decode before the layer's prefill, and the staged halves out of order
    assert _code(B_, cache.decode_step, 0, q1, k1, k1, o1, a1) == st
    assert _code(B_, B_.dms_decode_append, cache.handle, 0, B_.Cache.decode_args(q1, k1, k1, None, a1)) == st
    assert _code(B_, B_.dms_decode_attention, cache.handle, 0, q1, o1) == st
    assert _code(B_, B_.dms_decode_attention_noalloc, cache.handle, 0, q1, o1) == st
    # prefill attention before the compaction of the same layer and length
    q = torch.randn(B, T, Hq, D, device=dev).to(torch.bfloat16)
    k = torch.randn(B, T, Hkv, D, device=dev).to(torch.bfloat16)
    v = torch.randn(B, T, Hkv, D, device=dev).to(torch.bfloat16)
    o = torch.empty_like(q)
    alpha = -torch.ones(B, Hkv, T, dtype=torch.float32, device=dev)
    args = B_.Cache.prefill_args(q, k, v, o, alpha)
    assert _code(B_, B_.dms_prefill_attention, cache.handle, 0, args) == st
    B_.dms_prefill_compact(cache.handle, 0, args)
    shorter = B_.Cache.prefill_args(q[:, :T - 1], k[:, :T - 1], v[:, :T - 1], o[:, :T - 1], alpha)
    assert _code(B_, B_.dms_prefill_attention, cache.handle, 0, shorter) == st
    B_.dms_prefill_attention(cache.handle, 0, args)
    # a layer out of range
    assert _code(B_, cache.decode_step, 1, q1, k1, k1, o1, a1) == B_.DMS_ERR_INVALID
    torch.cuda.synchronize()
    assert cache.status() == 0 and cache.positions(0) == T
    cache.close()


@pytest.mark.gpu
def test_misaligned_rows_are_refused():
    """q, k, v, o move as 16-byte vectors: a view 2 bytes off is refused on the host."""
    B_, cache = _cache(SMALL)
    B, T, Hq, Hkv, D = SMALL.B, SMALL.T, SMALL.Hq, SMALL.Hkv, SMALL.D
    n = B * T * Hq * D
    buf = torch.zeros(n + 8, dtype=torch.bfloat16, device="cuda")
    q_off = buf[1:1 + n].view(B, T, Hq, D)
    assert q_off.data_ptr() % 16 != 0
    k = torch.zeros(B, T, Hkv, D, dtype=torch.bfloat16, device="cuda")
    o = torch.empty(B, T, Hq, D, dtype=torch.bfloat16, device="cuda")
    alpha = -torch.ones(B, Hkv, T, dtype=torch.float32, device="cuda")
    inv = B_.DMS_ERR_INVALID
    assert _code(B_, cache.prefill, 0, q_off, k, k, o, alpha) == inv
    kb = torch.zeros(B * T * Hkv * D + 8, dtype=torch.bfloat16, device="cuda")
    k_off = kb[1:1 + B * T * Hkv * D].view(B, T, Hkv, D)
    q = torch.zeros(B, T, Hq, D, dtype=torch.bfloat16, device="cuda")
    assert _code(B_, cache.prefill, 0, q, k_off, k, o, alpha) == inv
    assert _code(B_, cache.prefill, 0, q, k, k_off, o, alpha) == inv
    ob = torch.empty(n + 8, dtype=torch.bfloat16, device="cuda")
    assert _code(B_, cache.prefill, 0, q, k, k, ob[1:1 + n].view(B, T, Hq, D), alpha) == inv
    # nothing was launched: the layer is still empty and can be filled
    cache.prefill(0, q, k, k, o, alpha)
    q1 = torch.zeros(B, Hq, D, dtype=torch.bfloat16, device="cuda")
    q1b = torch.zeros(B * Hq * D + 8, dtype=torch.bfloat16, device="cuda")[1:1 + B * Hq * D].view(B, Hq, D)
    k1 = torch.zeros(B, Hkv, D, dtype=torch.bfloat16, device="cuda")
    a1 = -torch.ones(B, Hkv, dtype=torch.float32, device="cuda")
    assert _code(B_, cache.decode_step, 0, q1b, k1, k1, torch.empty_like(q1), a1) == inv
    assert _code(B_, cache.decode_step, 0, q1, k1, k1, q1b, a1) == inv
    torch.cuda.synchronize()
    assert cache.status() == 0 and cache.positions(0) == T
    cache.close()


@pytest.mark.gpu
@pytest.mark.parametrize("kv", ["bf16", "fp8"])
def test_prefill_into_an_undersized_pool_sets_the_status(kv):
    """Pool exhaustion is a device-side condition: the prefill's page grants run
    out, the status word says so, and the oracle's sequential replay of the same
    prompt into a pool of the same size reports the same bit."""
    case = Case(B=2, T=400, steps=0, Hq=8, Hkv=2, D=64, w=64, P=16, act="bf16", kv=kv, source="input",
                keep=0.5, pool_pages=24, seed=42)
    ins = build(case)
    assert ins["oracle_status"] & 1, "the oracle's pool of 24 pages must run out for this prompt"
    B_, cache = _cache(case)
    dev = torch.device("cuda")
    T = case.T
    q, k, v = (ins[n][:, :T].contiguous().to(dev) for n in ("q", "k", "v"))
    o = torch.empty_like(q)
    alpha = ins["alpha_in"][:, :, :T].contiguous().to(dev)
    cache.prefill(0, q, k, v, o, alpha)
    torch.cuda.synchronize()
    st = cache.status()
    assert st & B_.DMS_ST_POOL_EXHAUSTED
    assert st == ins["oracle_status"]
    # the state of the exhausted cache is unspecified; a reset clears the bit
    cache.reset()
    assert cache.status() == 0
    cache.close()


@pytest.mark.gpu
def test_bounded_wait_gives_up_and_sets_the_status():
    B_, cache = _cache(SMALL)
    B_.dms_selftest_wait_timeout(cache.handle, 1 << 14)
    torch.cuda.synchronize()
    assert cache.status() == B_.DMS_ST_TIMEOUT
    # the context is still usable: a reset clears the bit and a full case runs
    cache.reset()
    assert cache.status() == 0
    errs = check_case(SMALL, cache=cache)
    assert cache.status() == 0
    print(errs)
    cache.close()


@pytest.mark.gpu
@pytest.mark.parametrize("kv", ["bf16", "fp8"])
def test_reset_then_reuse_matches_a_fresh_oracle(kv):
    first = dataclasses.replace(SMALL, kv=kv, prealloc=32, seed=43)
    second = dataclasses.replace(first, seed=44, keep=0.6)
    B_, cache = _cache(first)
    check_case(first, cache=cache)
    cache.reset()
    assert cache.positions(0) == 0 and cache.status() == 0
    errs = check_case(second, cache=cache)   # the oracle side starts from an empty cache
    print(kv, errs)
    cache.close()
