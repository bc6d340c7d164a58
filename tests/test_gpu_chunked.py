"""Chunked prefill ([DMS-Qwen3], advanced options: a long prompt prefilled in
fixed-size chunks, 4096 tokens by default): every chunk is one dms_prefill
into a layer that already holds the earlier chunks, and attends to the cache
plus itself.  Compared with the oracle's chunk-by-chunk replay: decisions,
state and pages bit for bit after the last chunk and after the decode steps
that follow; the chunks' attention rows within the parity tolerance.

Also: chunks of different layers interleaved (the kept list and its K/V copy
are scratch shared by the layers, so each call rebuilds them from its own
layer), and the calls a chunked prefill refuses.
"""
import numpy as np
import pytest
import torch

from harness import Case, build, check_case, marks, compare_pages, compare_state, make_desc, run_gpu

CASES = {
    # three ragged chunks, each spanning several 64-key tiles
    "bf16_d128_three_chunks": Case(B=2, T=900, steps=12, Hq=8, Hkv=2, D=128, w=64, P=32, act="bf16", kv="bf16",
                                   source="input", keep=0.3, chunks=(300, 257, 343), seed=61),
    # chunks shorter than the window, adapter decisions
    "bf16_d64_proj_short_chunks": Case(B=2, T=200, steps=10, Hq=8, Hkv=4, D=64, hidden=256, w=64, P=16,
                                       act="bf16", kv="bf16", source="proj", keep=0.25, chunks=(20, 33, 47, 100),
                                       seed=62),
    # a one-token first chunk
    "bf16_one_token_then_rest": Case(B=1, T=400, steps=8, Hq=4, Hkv=2, D=64, w=48, P=16, act="bf16", kv="bf16",
                                     source="input", keep=0.4, chunks=(1, 399), seed=63),
    # FP8 pages, key-neuron decisions, rotary tables at the chunks' positions
    "fp8_key_rope_chunks": Case(B=2, T=700, steps=20, Hq=8, Hkv=2, D=64, w=64, P=32, act="bf16", kv="fp8",
                                source="key", keep=0.125, rope=True, chunks=(250, 250, 200), seed=64),
    # decision shifts across chunk boundaries: the carried decision (+1) and
    # the previous chunk's last token marked by the next chunk's first (-1)
    "bf16_shift_right_chunks": Case(B=2, T=600, steps=10, Hq=8, Hkv=2, D=128, w=64, P=32, act="bf16", kv="bf16",
                                    source="input", keep=0.3, chunks=(200, 1, 399), shift=1, seed=68),
    "bf16_shift_left_chunks": Case(B=2, T=600, steps=10, Hq=8, Hkv=2, D=64, hidden=256, w=64, P=32, act="bf16",
                                   kv="bf16", source="proj", keep=0.3, chunks=(150, 250, 200), shift=-1, seed=69),
    # per-layer decisions and the query neuron over two chunks
    "bf16_query_layer_chunks": Case(B=1, T=520, steps=6, Hq=8, Hkv=2, D=128, w=96, P=32, act="bf16", kv="bf16",
                                    source="query", per="layer", keep=0.2, chunks=(256, 264), seed=65),
}

FULL = {
    # the Qwen3-8B layer shape: a 12288-token prompt in three chunks of 4096, then 128 steps
    "qwen8b_three_chunks_of_4096": Case(B=1, T=12288, steps=128, Hq=32, Hkv=8, D=128, hidden=4096, w=512, P=256,
                                        act="bf16", kv="bf16", source="proj", keep=1 / 8, prealloc=4096,
                                        attn_rows=256, chunks=(4096, 4096, 4096), seed=1002),
}


@pytest.mark.parametrize("name", sorted(CASES) + sorted(FULL))
def test_chunked_case_builds(name):
    """CPU: the oracle's chunk replay holds the retained-count invariant."""
    case = {**CASES, **FULL}[name]
    if name in FULL:
        pytest.skip("full-size oracle replay runs with the GPU test")
    ins = build(case)
    ev, T, w = marks(ins["evict"][:, :, :case.T], case.shift), case.T, case.w
    expect = min(T, w) + (1 - ev[:, :, : max(0, T - w)]).sum(-1)
    assert np.array_equal(ins["state_prefill"]["count"], expect)


@pytest.mark.gpu
@pytest.mark.parametrize("name", sorted(CASES))
def test_chunked_prefill_parity(name):
    print(name, check_case(CASES[name]))


@pytest.mark.gpu
@pytest.mark.parametrize("name", sorted(FULL))
def test_chunked_prefill_fullsize(name):
    print(name, check_case(FULL[name]))


@pytest.mark.gpu
def test_chunks_of_two_layers_interleaved():
    """Chunk 1 of layer 0, chunk 1 of layer 1, chunk 2 of layer 0, ... as a
    model runs a chunk through every layer before the next: each layer ends
    as its own oracle replay does."""
    from learned_kv_cache_dms_b200 import binding as B_
    base = dict(B=2, T=600, steps=6, Hq=8, Hkv=2, D=64, w=64, P=32, act="bf16", kv="bf16", source="input",
                keep=0.3, layers=2, prealloc=64, chunks=(200, 150, 250))
    cases = [Case(layer=0, seed=66, **base), Case(layer=1, seed=67, **base)]
    ins = [build(c) for c in cases]
    dev = torch.device("cuda")
    cache = B_.Cache(make_desc(B_, cases[0]), dev)
    T = cases[0].T
    outs = [[], []]
    t0 = 0
    for n in cases[0].chunks:
        for l, (c, x) in enumerate(zip(cases, ins)):
            q = x["q"][:, t0:t0 + n].contiguous().to(dev)
            k = x["k"][:, t0:t0 + n].contiguous().to(dev)
            v = x["v"][:, t0:t0 + n].contiguous().to(dev)
            a = x["alpha_in"][:, :, t0:t0 + n].contiguous().to(dev)
            o = torch.empty_like(q)
            cache.prefill(l, q, k, v, o, a)
            outs[l].append(o)
        t0 += n
    torch.cuda.synchronize()
    for l, (c, x) in enumerate(zip(cases, ins)):
        st = {k_: t.cpu().clone() for k_, t in cache.state(l).items()}
        so = x["state_prefill"]
        # page ids interleave across the layers' calls; compare everything else
        assert np.array_equal(so["count"], st["count"].numpy())
        for b in range(c.B):
            for h in range(c.Hkv):
                n_ = so["count"][b, h]
                assert np.array_equal(so["slot_pos"][b, h, :n_], st["slot_pos"].numpy()[b, h, :n_])
        err = float(np.max(np.abs(torch.cat(outs[l], 1).double().cpu().numpy() - x["o_prefill"])))
        assert err <= 2e-2, (l, err)
    assert cache.status() == 0
    cache.close()


@pytest.mark.gpu
def test_chunked_prefill_refusals():
    from learned_kv_cache_dms_b200 import binding as B_
    dev = "cuda"

    def prefill(cache, T, B=1, Hq=4, Hkv=2, D=64, dt=torch.bfloat16):
        q = torch.zeros(B, T, Hq, D, dtype=dt, device=dev)
        k = torch.zeros(B, T, Hkv, D, dtype=dt, device=dev)
        a = -torch.ones(B, Hkv, T, dtype=torch.float32, device=dev)
        cache.prefill(0, q, k, k, torch.empty_like(q), a)

    def code(fn, *a):
        with pytest.raises(B_.DMSError) as ex:
            fn(*a)
        return ex.value.code

    case = Case(B=1, T=100, steps=4, Hq=4, Hkv=2, D=64, w=32, P=16, act="bf16", kv="bf16", source="input")
    cache = B_.Cache(make_desc(B_, case), torch.device(dev))
    prefill(cache, 60)
    prefill(cache, 40)                      # a second chunk is accepted
    assert code(prefill, cache, 5) == B_.DMS_ERR_INVALID  # past max_positions (104)
    q1 = torch.zeros(1, 4, 64, dtype=torch.bfloat16, device=dev)
    k1 = torch.zeros(1, 2, 64, dtype=torch.bfloat16, device=dev)
    cache.decode_step(0, q1, k1, k1, torch.empty_like(q1), -torch.ones(1, 2, dtype=torch.float32, device=dev))
    assert code(prefill, cache, 2) == B_.DMS_ERR_STATE     # after a decode step
    cache.reset()
    prefill(cache, 10)                      # a reset starts a new prompt
    torch.cuda.synchronize()
    assert cache.status() == 0
    cache.close()
    # fp32 activations and GQA groups that are not a power of two have no
    # chunk path (the tcgen05 attention reads the window and kept copies)
    for kw in (dict(act="f32", kv="f32"), dict(Hq=6, Hkv=2)):
        c2 = Case(**{**dict(B=1, T=100, steps=4, Hq=4, Hkv=2, D=64, w=32, P=16, act="bf16", kv="bf16",
                            source="input"), **kw})
        cache = B_.Cache(make_desc(B_, c2), torch.device(dev))
        dt = torch.float32 if c2.act == "f32" else torch.bfloat16
        prefill(cache, 30, Hq=c2.Hq, Hkv=c2.Hkv, dt=dt)
        assert code(prefill, cache, 20, 1, c2.Hq, c2.Hkv, 64, dt) == B_.DMS_ERR_INVALID
        cache.close()
