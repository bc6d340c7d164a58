"""GPU: dms_cache_export copies one layer's state (positions, counts, pages,
page table, slot positions, ring) to host buffers; it must equal the device
state read through the cache layout, for a layer that was decoded and for one
that was only prefilled."""
import numpy as np
import pytest
import torch


@pytest.mark.gpu
def test_export_matches_device_state():
    from learned_kv_cache_dms_b200 import binding as B_
    B, T, S, Hq, Hkv, D, w, P = 2, 300, 7, 8, 2, 64, 64, 32
    d = B_.dms_cache_desc_default()
    d.num_layers, d.batch, d.num_q_heads, d.num_kv_heads = 2, B, Hq, Hkv
    d.head_dim, d.window, d.block = D, w, P
    d.max_positions, d.prealloc_tokens = T + S, 64
    d.pool_pages = d.num_layers * B * Hkv * (-(-(T + S) // P))
    d.alpha_source = B_.DMS_ALPHA_KEY_NEURON
    g = torch.Generator(device="cuda")
    g.manual_seed(5)

    def rn(*shape):
        return torch.randn(*shape, generator=g, device="cuda").to(torch.bfloat16)

    cache = B_.Cache(d)
    off = torch.zeros(B, Hkv, dtype=torch.float32, device="cuda")
    for layer in range(2):
        q, k, v = rn(B, T, Hq, D), rn(B, T, Hkv, D), rn(B, T, Hkv, D)
        o = torch.empty_like(q)
        alpha = torch.empty(B, Hkv, T, dtype=torch.float32, device="cuda")
        cache.prefill(layer, q, k, v, o, alpha, decide=B_.decide_params(off))
    for s in range(S):
        qd, kd, vd = rn(B, Hq, D), rn(B, Hkv, D), rn(B, Hkv, D)
        od = torch.empty_like(qd)
        ad = torch.empty(B, Hkv, dtype=torch.float32, device="cuda")
        cache.decode_step(0, qd, kd, vd, od, ad, decide=B_.decide_params(off))
    torch.cuda.synchronize()
    assert cache.status() == 0
    for layer, n in ((0, T + S), (1, T)):
        ex = cache.export(layer)
        st = cache.state(layer)
        assert (ex["pos"] == n).all()
        assert np.array_equal(ex["pos"], st["pos"].cpu().numpy())
        for key in ("count", "npages", "page_table"):
            assert np.array_equal(ex[key], st[key].cpu().numpy()), key
        ring = st["ring_slot"].cpu().numpy().astype(np.int64) | (st["ring_evict"].cpu().numpy().astype(np.int64) << 31)
        assert np.array_equal(ex["ring"].view(np.uint32).astype(np.int64), ring)
        sp = st["slot_pos"].cpu().numpy()
        for b in range(B):
            for h in range(Hkv):
                c = int(ex["count"][b, h])
                assert np.array_equal(ex["slot_pos"][b, h, :c], sp[b, h, :c])
