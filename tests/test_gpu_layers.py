"""dms_decode_step_layers: one decode step of several layers in one launch (a
stack whose layers do not feed each other within a step, like the synthetic
36-layer reasoning stack), on bf16 and FP8 pages.  Against one oracle cache that replays the same
calls in the same order (prefill of each layer, then every step appending to
layer 0, 1, ...): state and page tables bit for bit, stored pages bit for bit,
decision logits within 1e-3 (decisions exact), attention within 2e-2.
"""
import dataclasses

import numpy as np
import pytest
import torch

from harness import Case, build, compare_pages, compare_state, make_desc
from oracle import oracle as O

BASE = Case(B=4, T=300, steps=20, Hq=8, Hkv=4, D=128, hidden=256, w=64, P=32, act="bf16", kv="bf16",
            source="proj", keep=(1 / 16, 1 / 4), layers=3, prealloc=64)


def _stack(ts):
    return torch.stack([t for t in ts]).contiguous()


@pytest.mark.gpu
@pytest.mark.parametrize("variant", ["proj", "input_shift_left", "proj_layer_d64", "fp8_proj", "fp8_input_d64"])
def test_decode_step_layers_matches_the_oracle(variant):
    from learned_kv_cache_dms_b200 import binding as B_
    base = BASE
    if variant == "input_shift_left":
        base = dataclasses.replace(BASE, source="input", shift=-1, keep=0.3)
    elif variant == "proj_layer_d64":
        base = dataclasses.replace(BASE, D=64, per="layer", B=2, Hq=16)
    elif variant == "fp8_proj":
        # FP8 pages: each layer's owner CTA appends (re-encoding the page when
        # its scale grows) before the attention reads the page
        base = dataclasses.replace(BASE, kv="fp8")
    elif variant == "fp8_input_d64":
        base = dataclasses.replace(BASE, kv="fp8", source="input", D=64, B=2, Hq=16, keep=0.3)
    L, B, T, N = base.layers, base.B, base.T, base.N
    cases = [dataclasses.replace(base, layer=l, seed=80 + l) for l in range(L)]
    ins = [build(c) for c in cases]
    # the oracle: one cache, the GPU's call order
    oc = O.Cache(L, B, base.Hkv, base.D, base.w, base.P, N, base.pool, base.prealloc, fp8=base.kv == "fp8",
                 shift=base.shift)
    for l, x in enumerate(ins):
        oc.prefill(l, np.ascontiguousarray(x["evict"][:, :, :T]), x["k_stored"][:, :T].astype(np.float32),
                   x["v"][:, :T].float().numpy())
    dev = torch.device("cuda")
    cache = B_.Cache(make_desc(B_, base), dev)
    keep = []
    for l, (c, x) in enumerate(zip(cases, ins)):
        q, k, v = (x[n][:, :T].contiguous().to(dev) for n in ("q", "k", "v"))
        o = torch.empty_like(q)
        if c.source == "proj":
            alpha = torch.empty(B, c.Hkv, T, dtype=torch.float32, device=dev)
            h = x["h"][:, :T].contiguous().to(dev)
            g, W, off = x["gamma"].to(dev), x["W"].to(dev), x["offset"].to(dev)
            keep += [h, g, W, off]
            cache.prefill(l, q, k, v, o, alpha, decide=B_.decide_params(off, hidden=h, norm_weight=g, proj_weight=W))
        else:
            cache.prefill(l, q, k, v, o, x["alpha_in"][:, :, :T].contiguous().to(dev))
    # layer-stacked decision parameters
    if base.source == "proj":
        gam = _stack([x["gamma"] for x in ins]).to(dev)
        Wst = _stack([x["W"] for x in ins]).to(dev)
        offs = _stack([x["offset"] for x in ins]).to(dev)  # [L, B, Hkv]
    worst = 0.0
    for s in range(base.steps):
        t = T + s
        qs = _stack([x["q"][:, t] for x in ins]).to(dev)
        ks = _stack([x["k"][:, t] for x in ins]).to(dev)
        vs = _stack([x["v"][:, t] for x in ins]).to(dev)
        os_ = torch.empty_like(qs)
        if base.source == "proj":
            hs = _stack([x["h"][:, t] for x in ins]).to(dev)
            dp = B_.decide_params(offs[0], hidden=hs, norm_weight=gam, proj_weight=Wst)
            dp.offset = offs.data_ptr()
            alpha = torch.empty(L, B, base.Hkv, dtype=torch.float32, device=dev)
            args = B_.Cache.decode_args(qs, ks, vs, os_, alpha, dp)
        else:
            alpha = _stack([x["alpha_in"][:, :, t] for x in ins]).to(dev)
            args = B_.Cache.decode_args(qs, ks, vs, os_, alpha)
        B_.dms_decode_step_layers(cache.handle, 0, L, args)
        for l, x in enumerate(ins):
            oc.append(l, np.ascontiguousarray(x["evict"][:, :, t]), np.ascontiguousarray(x["k_stored"][:, t]).astype(np.float32),
                      x["v"][:, t].float().numpy())
        torch.cuda.synchronize()
        for l, x in enumerate(ins):
            want = oc.decode_attention(l, np.ascontiguousarray(x["q_stored"][:, t]))
            err = float(np.max(np.abs(os_[l].double().cpu().numpy() - want)))
            assert err <= 2e-2, (variant, l, t, err)
            worst = max(worst, err)
            if base.source == "proj":
                a_g = alpha[l].double().cpu().numpy()
                a_o = x["alpha_o"][:, :, t]
                assert np.max(np.abs(a_g - a_o)) < 1e-3 * max(1.0, float(np.max(np.abs(a_o))))
                assert np.array_equal(a_g > 0, a_o > 0)
    for l in range(L):
        st = {k_: t_.cpu().clone() for k_, t_ in cache.state(l).items()}
        so = oc.export(l)
        compare_state(cases[l], so, st, N)
    pages = {k_: t_.cpu().clone() for k_, t_ in cache.pages().items()}
    po = oc.pages()
    for l in range(L):
        compare_pages(cases[l], oc.export(l), po, pages)
    assert cache.status() == 0 and oc.status == 0
    print(variant, "max-abs", worst)
    cache.close()


@pytest.mark.gpu
def test_decode_step_layers_refusals():
    from learned_kv_cache_dms_b200 import binding as B_
    dev = torch.device("cuda")
    c = dataclasses.replace(BASE, source="input", steps=2, T=40)
    cache = B_.Cache(make_desc(B_, c), dev)
    L, B = c.layers, c.B
    q = torch.zeros(L, B, c.Hq, c.D, dtype=torch.bfloat16, device=dev)
    k = torch.zeros(L, B, c.Hkv, c.D, dtype=torch.bfloat16, device=dev)
    a = -torch.ones(L, B, c.Hkv, dtype=torch.float32, device=dev)
    args = B_.Cache.decode_args(q, k, k, torch.empty_like(q), a)
    with pytest.raises(B_.DMSError) as ex:
        B_.dms_decode_step_layers(cache.handle, 0, L, args)   # before the prefills
    assert ex.value.code == B_.DMS_ERR_STATE
    for l in range(L):
        qp = torch.zeros(B, 40 - l, c.Hq, c.D, dtype=torch.bfloat16, device=dev)
        kp = torch.zeros(B, 40 - l, c.Hkv, c.D, dtype=torch.bfloat16, device=dev)
        cache.prefill(l, qp, kp, kp, torch.empty_like(qp), -torch.ones(B, c.Hkv, 40 - l, device=dev))
    with pytest.raises(B_.DMSError) as ex:
        B_.dms_decode_step_layers(cache.handle, 0, L, args)   # layers of different lengths
    assert ex.value.code == B_.DMS_ERR_STATE
    with pytest.raises(B_.DMSError) as ex:
        B_.dms_decode_step_layers(cache.handle, 1, L, args)   # past the last layer
    assert ex.value.code == B_.DMS_ERR_INVALID
    B_.dms_decode_step_layers(cache.handle, 2, 1, B_.Cache.decode_args(q[:1], k[:1], k[:1], torch.empty_like(q[:1]),
                                                                         a[:1]))
    torch.cuda.synchronize()
    assert cache.status() == 0 and cache.positions(2) == 39
    cache.close()
