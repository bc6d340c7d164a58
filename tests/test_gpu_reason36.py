"""The 36-layer long-reasoning decode stress, replayed in full through the C ABI
against the oracle: Qwen3-8B attention-layer shape (32 query / 8 KV heads,
head_dim 128), batch 32, prompt 1024, then 16384 generated tokens in every
layer, keep fraction 1/16, window 512, block 256, bf16 pages.

- The cache state of all 36 layers (positions, retained counts, pages owned,
  page tables, slot positions, ring, page counter) is compared bit for bit
  after the prefill and after every 1024th decode step.
- At those steps the decode attention of layers 0, 17 and 35 is compared with
  the oracle's (max-abs 2e-2), and their stored page rows bit for bit.

Inputs (seeded): decisions are given as logits, fresh for every layer,
sequence, head and position; the prompt's q/k/v rows are shared by the layers
and the decode tokens cycle a bank of 64 rows, so that the inputs fit in host
memory.  The layers are independent (no MLP, no O-projection), and each
layer's retained set follows its own decisions.
"""
import numpy as np
import pytest
import torch

from harness import compare_state
from learned_kv_cache_dms_b200 import inputs as I
from oracle import oracle as O

L, B, HQ, HKV, D, T, STEPS, W, P = 36, 32, 32, 8, 128, 1024, 16384, 512, 256
KEEP = 1 / 16
SAMPLED = (0, 17, 35)
CHECK_EVERY = 1024
NBANK = 64
SEED = 1005
TOL = 2e-2


class _Geom:
    """What harness.compare_state reads from a case."""
    B, Hkv, w = B, HKV, W


def _state(cache, layer):
    return {k: t.cpu().clone() for k, t in cache.state(layer).items()}


def _pages_equal(so, po, pages_gpu, pt_gpu):
    """Stored rows of every retained slot of one layer, bit for bit: the GPU's
    pages through its page table, the oracle's through its own."""
    kg, vg = pages_gpu
    for b in range(B):
        for h in range(HKV):
            c = int(so["count"][b, h])
            npg = -(-c // P)
            ids_g = pt_gpu[b, h, :npg]
            rows_k = kg[ids_g].reshape(-1, D)[:c].double().cpu().numpy()
            rows_v = vg[ids_g].reshape(-1, D)[:c].double().cpu().numpy()
            ids_o = so["page_table"][b, h, :npg]
            assert np.array_equal(rows_k, po["kval"][ids_o].reshape(-1, D)[:c]), ("k rows", b, h)
            assert np.array_equal(rows_v, po["vval"][ids_o].reshape(-1, D)[:c]), ("v rows", b, h)


@pytest.mark.gpu
def test_reason36_full_replay():
    from learned_kv_cache_dms_b200 import binding as B_
    dev = torch.device("cuda")
    N = T + STEPS
    # ---- inputs ----
    qp = I.normal(SEED, (100, 1), (B, T, HQ, D), "bf16")
    kp = I.normal(SEED, (100, 2), (B, T, HKV, D), "bf16")
    vp = I.normal(SEED, (100, 3), (B, T, HKV, D), "bf16")
    qb = I.normal(SEED, (101, 1), (NBANK, B, HQ, D), "bf16")
    kb = I.normal(SEED, (101, 2), (NBANK, B, HKV, D), "bf16")
    vb = I.normal(SEED, (101, 3), (NBANK, B, HKV, D), "bf16")
    alpha = [I.synthetic_alpha(SEED, (l, 5), B, HKV, N, KEEP) for l in range(L)]   # [B, Hkv, N] fp32
    evict = [O.evict_bits(a.numpy()) for a in alpha]

    # ---- oracle: every layer's index state in one cache (one page counter, the
    # GPU's call order), values only for the sampled layers ----
    pages_per_head = 8
    oc = O.Cache(L, B, HKV, D, W, P, N, L * B * HKV * pages_per_head, 0, store_values=False)
    vc = {l: O.Cache(1, B, HKV, D, W, P, N, B * HKV * pages_per_head, 0) for l in SAMPLED}
    kp32, vp32 = kp.float().numpy(), vp.float().numpy()
    kb32, vb32, qb64 = kb.float().numpy(), vb.float().numpy(), qb.double().numpy()

    # ---- GPU ----
    d = B_.dms_cache_desc_default()
    d.num_layers, d.batch, d.num_q_heads, d.num_kv_heads, d.head_dim, d.hidden = L, B, HQ, HKV, D, 4096
    d.window, d.block, d.max_positions, d.prealloc_tokens = W, P, N, 0
    d.pool_pages = L * B * HKV * pages_per_head
    d.act_dtype = d.kv_dtype = B_.DMS_BF16
    cache = B_.Cache(d, dev)
    qpd, kpd, vpd = qp.to(dev), kp.to(dev), vp.to(dev)
    qbd, kbd, vbd = qb.to(dev), kb.to(dev), vb.to(dev)
    o_pre = torch.empty_like(qpd)
    # per-step decision logits of each layer, [STEPS, B, Hkv] (one dense row per step)
    a_dec = [a[:, :, T:].permute(2, 0, 1).contiguous().to(dev) for a in alpha]
    ev_dec = [np.ascontiguousarray(e[:, :, T:].transpose(2, 0, 1)) for e in evict]

    for l in range(L):
        cache.prefill(l, qpd, kpd, vpd, o_pre, alpha[l][:, :, :T].contiguous().to(dev))
        oc.prefill(l, np.ascontiguousarray(evict[l][:, :, :T]))
    for l in SAMPLED:
        vc[l].prefill(0, np.ascontiguousarray(evict[l][:, :, :T]), kp32, vp32)
    torch.cuda.synchronize()
    for l in range(L):
        compare_state(_Geom, oc.export(l), _state(cache, l), T)

    o_scratch = torch.empty(B, HQ, D, dtype=torch.bfloat16, device=dev)
    o_s = {l: torch.empty_like(o_scratch) for l in SAMPLED}
    worst = 0.0
    for s in range(STEPS):
        j = s % NBANK
        for l in range(L):
            cache.decode_step(l, qbd[j], kbd[j], vbd[j], o_s.get(l, o_scratch), a_dec[l][s])
            oc.append(l, ev_dec[l][s])
        for l in SAMPLED:
            vc[l].append(0, ev_dec[l][s], kb32[j], vb32[j])
        if (s + 1) % CHECK_EVERY:
            continue
        torch.cuda.synchronize()
        for l in range(L):
            compare_state(_Geom, oc.export(l), _state(cache, l), T + s + 1)
        pages = cache.pages()
        for l in SAMPLED:
            so, po = vc[l].export(0), vc[l].pages()
            st = cache.state(l)
            _pages_equal(so, po, (pages["k"], pages["v"]), st["page_table"].cpu().numpy())
            want = vc[l].decode_attention(0, qb64[j])
            err = float(np.max(np.abs(o_s[l].double().cpu().numpy() - want)))
            assert err <= TOL, ("decode attention", l, s, err)
            worst = max(worst, err)
    assert cache.status() == 0 and oc.status == 0 and all(vc[l].status == 0 for l in SAMPLED)
    counts = cache.counts().cpu().numpy()
    print("reason36 full replay: retained per head %d..%d, max-abs error %.3g" % (counts.min(), counts.max(), worst))
    cache.close()
