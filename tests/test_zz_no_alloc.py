"""dms_decode_attention_noalloc: the decode attention for callers that cannot
give the library scratch memory (a fixed device-memory pool set up at start,
a decode loop that must never reach cudaMalloc).  Its split-K partials live in
a fixed array inside the library instead of the caller's cache buffer.  Its
output is checked against the oracle's decode attention and against
dms_decode_attention, on two calls in a row (the array keeps the last call's
contents).

This file sorts last so that a run stopping at the first failure has already
run every other test; it also passes on its own in a fresh process.
"""
import numpy as np
import pytest
import torch

from harness import Case, build, make_desc

TOL = 2e-2  # bf16 / FP8 attention tolerance used by the parity tests


def _setup(case):
    from learned_kv_cache_dms_b200 import binding as B_
    ins = build(case)
    dev = torch.device("cuda")
    cache = B_.Cache(make_desc(B_, case), dev)
    T = case.T
    q = ins["q"].to(dev)
    k = ins["k"].to(dev)
    v = ins["v"].to(dev)
    alpha_in = ins["alpha_in"].to(dev)
    o = torch.empty_like(q[:, :T])
    cache.prefill(0, q[:, :T].contiguous(), k[:, :T].contiguous(), v[:, :T].contiguous(), o,
                  alpha_in[:, :, :T].contiguous())
    return B_, ins, cache, q, k, v, alpha_in


def _steps_against_oracle(case, steps):
    B_, ins, cache, q, k, v, alpha_in = _setup(case)
    T = case.T
    worst = 0.0
    for i, t in enumerate(range(T, T + steps)):
        qt, kt, vt = q[:, t].contiguous(), k[:, t].contiguous(), v[:, t].contiguous()
        at = alpha_in[:, :, t].contiguous()
        B_.dms_decode_append(cache.handle, 0, B_.Cache.decode_args(qt, kt, vt, None, at))
        ref = torch.empty_like(qt)
        B_.dms_decode_attention(cache.handle, 0, qt, ref)
        want = ins["o_decode"][i]
        for _ in range(2):  # two calls in a row on the shared fixed array
            out = torch.full_like(qt, float("nan"))
            B_.dms_decode_attention_noalloc(cache.handle, 0, qt, out)
            torch.cuda.synchronize()
            err_o = float(np.max(np.abs(out.double().cpu().numpy() - want)))
            err_r = (out.float() - ref.float()).abs().max().item()
            assert err_o <= TOL, ("against the oracle", err_o)
            assert err_r <= TOL, ("against dms_decode_attention", err_r)
            worst = max(worst, err_o)
    assert cache.status() == 0
    cache.close()
    return worst


@pytest.mark.gpu
@pytest.mark.parametrize("kv", ["bf16", "fp8"])
@pytest.mark.parametrize("D", [64, 128])
def test_noalloc_matches_oracle_two_calls(kv, D):
    case = Case(B=2, T=700, steps=2, Hq=8, Hkv=2, D=D, w=64, P=32, act="bf16", kv=kv, source="input",
                keep=0.3, seed=31 if kv == "bf16" else 32)
    print(kv, D, _steps_against_oracle(case, 2))


@pytest.mark.gpu
def test_noalloc_qwen8b_batch1_step():
    """The Qwen3-8B layer shape at batch 1 (8192-token prompt, keep 1/8): about
    1.35 MB of partials, inside the fixed array; one step against the oracle."""
    case = Case(B=1, T=8192, steps=1, Hq=32, Hkv=8, D=128, w=512, P=256, act="bf16", kv="bf16", source="input",
                keep=1 / 8, prealloc=4096, attn_rows=8, seed=1002)
    print(_steps_against_oracle(case, 1))


@pytest.mark.gpu
def test_noalloc_rejects_caches_beyond_the_limit():
    # batch 32 x 8 kv heads x 68 pages of work items x 4 query heads x 130 floats
    # of partials is far beyond the fixed 4 MiB: rejected before any launch
    from learned_kv_cache_dms_b200 import binding as B_
    case = Case(B=32, T=1024, steps=16384, Hq=32, Hkv=8, D=128, w=512, P=256, act="bf16", kv="bf16",
                source="input", keep=1 / 16)
    d = make_desc(B_, case)
    d.pool_pages = 32 * 8 * 8
    d.max_positions = case.T + case.steps
    cache = B_.Cache(d, torch.device("cuda"))
    q = torch.zeros(32, 32, 128, dtype=torch.bfloat16, device="cuda")
    kv = torch.zeros(32, 8, 128, dtype=torch.bfloat16, device="cuda")
    alpha = -torch.ones(32, 8, 1, dtype=torch.float32, device="cuda")
    o1 = torch.empty(32, 1, 32, 128, dtype=torch.bfloat16, device="cuda")
    cache.prefill(0, q[:, None], kv[:, None], kv[:, None], o1, alpha)
    B_.dms_decode_append(cache.handle, 0, B_.Cache.decode_args(q, kv, kv, None, alpha[:, :, 0].contiguous()))
    out = torch.empty_like(q)
    with pytest.raises(B_.DMSError) as ex:
        B_.dms_decode_attention_noalloc(cache.handle, 0, q, out)
    assert ex.value.code == B_.DMS_ERR_SCRATCH_LIMIT
    cache.close()
