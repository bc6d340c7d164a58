"""Pins for the CPU oracle: each test ties one oracle function to something other
than the oracle itself (a hand-worked example, a closed form, a special case that
reduces to a library routine, an invariant, or exhaustive enumeration)."""
import json
import math
import os

import numpy as np
import pytest
import torch

from oracle import oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# ---------------------------------------------------------------------------
# FP8 E4M3 encoder (OCP FP8 spec) -- pinned to the spec's fixed points and to
# torch's own CPU cast.
# ---------------------------------------------------------------------------
def test_e4m3_spec_points():
    pts = {0.0: 0x00, 1.0: 0x38, -2.0: 0xC0, 448.0: 0x7E, -448.0: 0xFE, 2.0 ** -9: 0x01,
           2.0 ** -6: 0x08, 7 * 2.0 ** -9: 0x07, 1.125: 0x39, 240.0: 0x77, 0.5: 0x30}
    for x, c in pts.items():
        assert O.e4m3_encode(np.array([x], np.float32))[0] == c, x
        assert O.e4m3_decode(np.array([c], np.uint8))[0] == x
    # satfinite: finite overflow clamps to +-448
    assert list(O.e4m3_encode(np.array([500.0, 1e30, -1e30, np.inf], np.float32))) == [0x7E, 0x7E, 0xFE, 0x7E]


def test_e4m3_roundtrip_all_codes():
    codes = np.array([c for c in range(256) if (c & 0x7F) != 0x7F], np.uint8)
    vals = O.e4m3_decode(codes).astype(np.float32)
    back = O.e4m3_encode(vals)
    # +0 and -0 are distinct codes that both decode to zero
    assert np.array_equal(back[codes != 0x80], codes[codes != 0x80])


def test_e4m3_matches_torch_cast():
    rng = np.random.default_rng(0)
    x = np.concatenate([
        rng.standard_normal(200000) * s for s in (1e-3, 0.05, 1.0, 30.0, 200.0)
    ]).astype(np.float32)
    # every midpoint between adjacent finite codes: exercises ties-to-even
    pos = np.sort(O.e4m3_decode(np.arange(0, 0x7F, dtype=np.uint8)))
    mids = ((pos[1:] + pos[:-1]) / 2).astype(np.float32)
    x = np.concatenate([x, mids, -mids, pos.astype(np.float32)])
    x = x[np.abs(x) < 448.0]
    ours = O.e4m3_encode(x)
    ref = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(ours, ref)


# ---------------------------------------------------------------------------
# Decision logits
# ---------------------------------------------------------------------------
def test_decide_proj_hand_example():
    # h = (1,1,1,1): mean square 1, so with eps = 0 the RMSNorm output is gamma.
    h = np.ones((1, 1, 4))
    gamma = np.array([1.0, 2.0, 0.0, -1.0])
    W = np.array([[1.0, 1.0, 1.0, 1.0], [0.0, 0.0, 0.0, 1.0]])
    a = O.decide_proj(h, gamma, W, None, [5.0, 5.0], scale=100.0, eps=0.0)
    assert a[0, 0, 0] == 2.0 * 100 - 5      # W0 . gamma = 2
    assert a[0, 1, 0] == -1.0 * 100 - 5     # W1 . gamma = -1
    # eps enters under the square root: mean square 1 + eps 3 -> 1/2
    a = O.decide_proj(h, gamma, W, None, [0.0, 0.0], scale=1.0, eps=3.0)
    assert a[0, 0, 0] == 1.0 and a[0, 1, 0] == -0.5
    # hidden (3, 4): mean square 12.5
    a = O.decide_proj(np.array([[[3.0, 4.0]]]), np.ones(2), np.array([[1.0, 0.0]]), None, [0.0],
                      scale=1.0, eps=0.0)
    assert a[0, 0, 0] == pytest.approx(3.0 / math.sqrt(12.5), rel=1e-15)


def test_decide_proj_invariants():
    rng = np.random.default_rng(1)
    B, T, hid, H = 2, 5, 16, 3
    h = rng.standard_normal((B, T, hid))
    g = rng.standard_normal(hid)
    W = rng.standard_normal((H, hid))
    off = rng.standard_normal((B, H))
    a = O.decide_proj(h, g, W, None, off, eps=0.0)
    # RMSNorm makes the logit invariant to the scale of h (eps = 0)
    assert np.allclose(O.decide_proj(h * 7.5, g, W, None, off, eps=0.0), a, rtol=1e-12, atol=1e-9)
    # zero projection (the adapter's initial state): alpha = -offset, gate open
    z = O.decide_proj(h, g, np.zeros_like(W), None, off)
    assert np.array_equal(z, np.broadcast_to(-off[:, :, None], z.shape))
    # a bias adds bias * scale
    bias = np.array([0.5, -1.0, 2.0])
    ab = O.decide_proj(h, g, W, bias, off, eps=0.0)
    assert np.allclose(ab - a, 100.0 * bias[None, :, None], atol=1e-9)
    # layer granularity: every head takes head 0's logit
    al = O.decide_proj(h, g, W, None, off, eps=0.0, layer_mode=True)
    for hd in range(H):
        assert np.array_equal(al[:, hd], a[:, 0])


def test_decide_neuron():
    rng = np.random.default_rng(2)
    B, T, Hq, Hkv, D = 2, 4, 8, 2, 8
    x = rng.standard_normal((B, T, Hq, D))
    off = np.array([[1.0, 2.0], [3.0, 4.0]])
    g = Hq // Hkv
    a, xz = O.decide_neuron(x, g, Hkv, off, scale=100.0)
    for b in range(B):
        for hd in range(Hkv):
            assert np.array_equal(a[b, hd], x[b, :, hd * g, D - 1] * 100.0 - off[b, hd])
    # the decision neuron of the first query head of each group is zeroed, nothing else
    diff = xz != x
    assert np.all(xz[:, :, ::g, D - 1] == 0)
    assert not diff[:, :, :, : D - 1].any()
    assert not np.delete(diff[..., D - 1], np.arange(0, Hq, g), axis=2).any()
    al, _ = O.decide_neuron(x, g, Hkv, off, layer_mode=True)
    assert np.array_equal(al[:, 1], al[:, 0]) and np.array_equal(al[:, 0], a[:, 0])


def test_rope_matches_complex_rotation():
    # half-split RoPE is multiplication of (x_i + i x_{i+D/2}) by exp(i * angle)
    rng = np.random.default_rng(3)
    B, T, H, D = 1, 6, 2, 8
    x = rng.standard_normal((B, T, H, D))
    ang = rng.uniform(-3, 3, (10, D // 2))
    y = O.rope(x, 2, np.cos(ang), np.sin(ang))
    z = (x[..., : D // 2] + 1j * x[..., D // 2:]) * np.exp(1j * ang[2:2 + T])[None, :, None, :]
    assert np.allclose(y[..., : D // 2], z.real, rtol=0, atol=1e-12)
    assert np.allclose(y[..., D // 2:], z.imag, rtol=0, atol=1e-12)


def test_rope_fp32_tables_exact_products():
    # bf16 elements times fp32 table entries: both products are exact in fp64,
    # so each rotated value is the exact rotation (rational arithmetic) rounded once
    from fractions import Fraction as F
    rng = np.random.default_rng(5)
    D = 8
    x = O.round_bf16(rng.standard_normal((1, 3, 1, D)) * 3)
    ang = rng.uniform(-3, 3, (3, D // 2))
    c, s = np.cos(ang).astype(np.float32).astype(np.float64), np.sin(ang).astype(np.float32).astype(np.float64)
    y = O.rope(x, 0, c, s)
    for t in range(3):
        for i in range(D // 2):
            a, b = F(x[0, t, 0, i]), F(x[0, t, 0, i + D // 2])
            ex0 = a * F(c[t, i]) - b * F(s[t, i])
            ex1 = b * F(c[t, i]) + a * F(s[t, i])
            assert y[0, t, 0, i] == float(ex0)            # float(Fraction) rounds to nearest
            assert y[0, t, 0, i + D // 2] == float(ex1)


def _bf16_neighbours(v):
    """The two bf16 values bracketing the rational v (exact, by enumeration of the grid)."""
    from fractions import Fraction as F
    import math
    if v == 0:
        return F(0), F(0)
    a = abs(v)
    e = math.floor(math.log2(a))
    while F(2) ** e > a:
        e -= 1
    while F(2) ** (e + 1) <= a:
        e += 1
    q = F(2) ** max(e - 7, -133)          # quantum of bf16 at this magnitude
    lo = (a // q) * q
    hi = lo if lo == a else lo + q
    return (lo, hi) if v > 0 else (-hi, -lo)


def test_round_bf16_definition():
    # nearest bf16, ties to the even mantissa, against exact rational arithmetic
    from fractions import Fraction as F
    rng = np.random.default_rng(6)
    xs = list(rng.standard_normal(3000) * 10.0 ** rng.integers(-6, 6, 3000))
    # exact midpoints and values one fp64 ulp either side of them
    for m in rng.integers(128, 256, 200):
        for e in (-20, -3, 0, 5):
            mid = (float(m) + 0.5) * 2.0 ** (e - 7)
            xs += [mid, np.nextafter(mid, 0), np.nextafter(mid, np.inf), -mid]
    xs += [2.0 ** -130 * 1.37, -(2.0 ** -133) * 0.5, 2.0 ** -133 * 1.5]   # subnormal range
    x = np.array(xs, np.float64)
    r = O.round_bf16(x)
    for xv, rv in zip(x, r):
        v = F(float(xv))
        lo, hi = _bf16_neighbours(v)
        dlo, dhi = v - lo, hi - v
        if dlo < dhi:
            want = lo
        elif dhi < dlo:
            want = hi
        else:   # tie: the neighbour whose last mantissa bit is 0
            q = hi - lo
            want = lo if (lo / q) % 2 == 0 else hi
        assert F(float(rv)) == want, (xv, rv, float(want))


def test_round_bf16_matches_torch_on_fp32_values():
    # for inputs that are fp32 numbers, rounding to bf16 is a single step in torch too
    rng = np.random.default_rng(7)
    x = (rng.standard_normal(200000) * 10.0 ** rng.integers(-8, 8, 200000)).astype(np.float32)
    want = torch.from_numpy(x).to(torch.bfloat16).double().numpy()
    assert np.array_equal(O.round_bf16(x.astype(np.float64)), want)


def test_rope_relative_position():
    # with true rotary tables, <R(m) q, R(n) k> depends only on m - n
    from learned_kv_cache_dms_b200.inputs import rope_tables
    cos, sin = (t.double().numpy() for t in rope_tables(64, 16, theta=10000.0))
    rng = np.random.default_rng(4)
    q = rng.standard_normal((1, 1, 1, 16))
    k = rng.standard_normal((1, 1, 1, 16))
    d1 = np.sum(O.rope(q, 10, cos, sin) * O.rope(k, 7, cos, sin))
    d2 = np.sum(O.rope(q, 40, cos, sin) * O.rope(k, 37, cos, sin))
    assert d1 == pytest.approx(d2, rel=1e-6)


# ---------------------------------------------------------------------------
# Append rule / cache state
# ---------------------------------------------------------------------------
def closed_form_state(evict, w):
    """Parallel characterisation of the append rule (independent of the oracle's
    sequential replay): a token opens a new slot iff it is in the first window or
    the token w earlier is kept; a token that does not open a slot inherits the
    slot of the token w earlier."""
    T = len(evict)
    opens = [t < w or not evict[t - w] for t in range(T)]
    newslot = np.cumsum([0] + opens[:-1]) if T else np.array([])
    slot = []
    for t in range(T):
        r = t
        while not opens[r]:
            r -= w
        slot.append(int(newslot[r]))
    count = int(sum(opens))
    slot_pos = [-1] * count
    for t in range(T):
        if t >= T - w or not evict[t]:
            slot_pos[slot[t]] = t
    return slot, count, slot_pos


def oracle_state(evict, w, P, max_pos=None, prealloc=0, pool=None):
    T = len(evict)
    max_pos = max_pos or max(T, 1)
    pool = pool or (max_pos // P + 2)
    c = O.Cache(1, 1, 1, 4, w, P, max_pos, pool, prealloc, store_values=False)
    c.prefill(0, np.array(evict, np.uint8).reshape(1, 1, T))
    return c, c.export(0)


def test_append_rule_golden():
    g = json.load(open(os.path.join(GOLDEN, "append_rule_w3_p2.json")))
    c, s = oracle_state(g["evict"], g["window"], g["block"], max_pos=12)
    n = g["count"]
    assert s["count"][0, 0] == n
    assert list(s["slot_pos"][0, 0, :n]) == g["slot_pos"]
    assert list(s["ring_slot"][0, 0]) == g["ring_slot"]
    assert list(s["ring_evict"][0, 0]) == g["ring_evict"]
    assert list(s["page_table"][0, 0, :3]) == g["page_table"]
    # token-by-token slots: replay prefixes
    for t in range(len(g["evict"])):
        _, st = oracle_state(g["evict"][: t + 1], g["window"], g["block"], max_pos=12)
        assert st["slot_pos"][0, 0, g["slot_of_token"][t]] == t
    # the retained set equals the visible keys of the last query
    assert sorted(s["slot_pos"][0, 0, :n]) == g["visible_keys_of_query_9"]


@pytest.mark.parametrize("T,w", [(1, 1), (5, 2), (7, 3), (12, 4)])
def test_append_rule_exhaustive(T, w):
    for bits in range(1 << T):
        ev = [(bits >> t) & 1 for t in range(T)]
        slot, count, slot_pos = closed_form_state(ev, w)
        _, s = oracle_state(ev, w, 2)
        assert s["count"][0, 0] == count
        assert list(s["slot_pos"][0, 0, :count]) == slot_pos
        for t in range(max(0, T - w), T):
            assert s["ring_slot"][0, 0, t % w] == slot[t]
            assert s["ring_evict"][0, 0, t % w] == ev[t]


def test_append_rule_random_long():
    rng = np.random.default_rng(5)
    for T, w, P, keep in [(600, 32, 16, 0.5), (2000, 512, 256, 0.125), (3000, 100, 64, 0.9)]:
        ev = (rng.random(T) > keep).astype(int).tolist()
        slot, count, slot_pos = closed_form_state(ev, w)
        _, s = oracle_state(ev, w, P)
        assert s["count"][0, 0] == count
        # the retained count: a full window plus every kept token before it
        assert count == min(T, w) + sum(1 - e for e in ev[: max(0, T - w)])
        assert list(s["slot_pos"][0, 0, :count]) == slot_pos
        assert s["npages"][0, 0] == -(-count // P)


def test_all_keep_and_all_evict():
    T, w, P = 100, 8, 4
    _, s = oracle_state([0] * T, w, P)
    assert s["count"][0, 0] == T and list(s["slot_pos"][0, 0, :T]) == list(range(T))
    assert list(s["page_table"][0, 0, :T // P]) == list(range(T // P))
    _, s = oracle_state([1] * T, w, P)
    assert s["count"][0, 0] == w
    # pure sliding window: slot s holds the last token congruent to s mod w
    assert list(s["slot_pos"][0, 0, :w]) == [T - w + ((sl - T) % w) for sl in range(w)]


def test_prefill_then_appends_equals_longer_prefill():
    rng = np.random.default_rng(6)
    B, H, T, n, w, P = 2, 3, 70, 25, 16, 8
    ev = (rng.random((B, H, T + n)) > 0.4).astype(np.uint8)
    a = O.Cache(1, B, H, 4, w, P, T + n, 200, 0, store_values=False)
    a.prefill(0, ev)
    b = O.Cache(1, B, H, 4, w, P, T + n, 200, 0, store_values=False)
    b.prefill(0, np.ascontiguousarray(ev[:, :, :T]))
    for t in range(T, T + n):
        b.append(0, np.ascontiguousarray(ev[:, :, t]))
    sa, sb = a.export(0), b.export(0)
    for key in ("count", "slot_pos", "ring_slot", "ring_evict", "npos"):
        assert np.array_equal(sa[key], sb[key]), key
    # page ids differ only in allocation order (prefill grants per (b, h) at
    # once, appends interleave heads), never in the number of pages per head
    assert np.array_equal(sa["npages"], sb["npages"])


def test_page_ids_prealloc_and_order():
    # prealloc pages are numbered row-major over (layer, b, h, page); later
    # grants come from one ascending counter in (b, h) row-major order
    B, H, w, P = 2, 2, 4, 4
    L = 2
    c = O.Cache(L, B, H, 4, w, P, 40, 100, prealloc_tokens=8)
    T = 20
    ev = np.zeros((B, H, T), np.uint8)
    c.prefill(1, ev)
    s = c.export(1)
    pre = 2
    for b in range(B):
        for h in range(H):
            base = ((1 * B + b) * H + h) * pre
            assert list(s["page_table"][b, h, :2]) == [base, base + 1]
    first_free = L * B * H * pre
    expect = first_free
    for b in range(B):
        for h in range(H):
            assert list(s["page_table"][b, h, 2:5]) == [expect, expect + 1, expect + 2]
            expect += 3
    assert s["next_page"] == expect


def test_pool_exhaustion_sets_status():
    c = O.Cache(1, 1, 1, 4, 4, 2, 64, 3, 0, store_values=False)
    c.prefill(0, np.zeros((1, 1, 10), np.uint8))
    assert c.status & 1


# ---------------------------------------------------------------------------
# Attention
# ---------------------------------------------------------------------------
def sdpa64(q, k, v, mask):
    """torch SDPA in fp64 on [B,T,H,D] inputs with GQA expansion; mask [T,T] or None."""
    Hq, Hkv = q.shape[2], k.shape[2]
    g = Hq // Hkv
    qt = torch.from_numpy(q).permute(0, 2, 1, 3)
    kt = torch.from_numpy(k).permute(0, 2, 1, 3).repeat_interleave(g, dim=1)
    vt = torch.from_numpy(v).permute(0, 2, 1, 3).repeat_interleave(g, dim=1)
    if mask is None:
        o = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, is_causal=True)
    else:
        o = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, attn_mask=torch.from_numpy(mask))
    return o.permute(0, 2, 1, 3).numpy()


def rand_qkv(seed, B, T, Hq, Hkv, D):
    rng = np.random.default_rng(seed)
    return (rng.standard_normal((B, T, Hq, D)), rng.standard_normal((B, T, Hkv, D)),
            rng.standard_normal((B, T, Hkv, D)))


def test_attention_reduces_to_causal():
    B, T, Hq, Hkv, D = 2, 40, 4, 2, 16
    q, k, v = rand_qkv(7, B, T, Hq, Hkv, D)
    ref = sdpa64(q, k, v, None)
    rng = np.random.default_rng(8)
    ev = (rng.random((B, Hkv, T)) > 0.5).astype(np.uint8)
    # window >= sequence length: every causal key is inside the window
    assert np.allclose(O.prefill_attention(q, k, v, ev, window=T), ref, atol=1e-12)
    # all keep (or eviction disabled): dense causal attention
    assert np.allclose(O.prefill_attention(q, k, v, np.zeros_like(ev), window=3), ref, atol=1e-12)
    assert np.allclose(O.prefill_attention(q, k, v, O.evict_bits(ev, disable_eviction=True), window=3),
                       ref, atol=1e-12)


def test_attention_all_evict_is_sliding_window():
    B, T, Hq, Hkv, D, w = 1, 50, 4, 1, 8, 7
    q, k, v = rand_qkv(9, B, T, Hq, Hkv, D)
    i = np.arange(T)[:, None]
    j = np.arange(T)[None, :]
    band = (j <= i) & (i - j < w)
    ref = sdpa64(q, k, v, band)
    got = O.prefill_attention(q, k, v, np.ones((B, Hkv, T), np.uint8), window=w)
    assert np.allclose(got, ref, atol=1e-12)


def test_attention_single_kept_token():
    # only token 3 is kept: query i >= 3 + w sees token 3 plus its window
    B, T, Hq, Hkv, D, w = 1, 30, 2, 1, 8, 5
    q, k, v = rand_qkv(10, B, T, Hq, Hkv, D)
    ev = np.ones((B, Hkv, T), np.uint8)
    ev[0, 0, 3] = 0
    i = np.arange(T)[:, None]
    j = np.arange(T)[None, :]
    mask = (j <= i) & ((i - j < w) | (j == 3))
    assert np.allclose(O.prefill_attention(q, k, v, ev, window=w), sdpa64(q, k, v, mask), atol=1e-12)


def test_attention_convex_combination_and_rows():
    B, T, Hq, Hkv, D, w = 1, 20, 2, 1, 8, 4
    q, k, _ = rand_qkv(11, B, T, Hq, Hkv, D)
    v = np.tile(np.arange(D, dtype=np.float64), (B, T, Hkv, 1))
    ev = (np.random.default_rng(12).random((B, Hkv, T)) > 0.5).astype(np.uint8)
    o = O.prefill_attention(q, k, v, ev, w)
    assert np.allclose(o, np.arange(D)[None, None, None, :], atol=1e-12)
    q, k, v = rand_qkv(13, B, T, Hq, Hkv, D)
    full = O.prefill_attention(q, k, v, ev, w)
    rows = [(0, 1, 19), (0, 0, 3), (0, 1, 0)]
    part = O.prefill_attention(q, k, v, ev, w, rows=rows)
    for r, (b, hq, i) in enumerate(rows):
        assert np.array_equal(part[r], full[b, i, hq])


def test_decode_attention_equals_prefill_row():
    # decoding token t over the cache equals row t of the masked prefill
    B, T, Hq, Hkv, D, w, P = 2, 60, 4, 2, 16, 8, 4
    q, k, v = rand_qkv(14, B, T, Hq, Hkv, D)
    ev = (np.random.default_rng(15).random((B, Hkv, T)) > 0.5).astype(np.uint8)
    full = O.prefill_attention(q, k, v, ev, w)
    T0 = 40
    c = O.Cache(1, B, Hkv, D, w, P, T, 100, 0)
    c.prefill(0, np.ascontiguousarray(ev[:, :, :T0]), k[:, :T0].astype(np.float32), v[:, :T0].astype(np.float32))
    for t in range(T0, T):
        c.append(0, np.ascontiguousarray(ev[:, :, t]), np.ascontiguousarray(k[:, t]).astype(np.float32),
                 np.ascontiguousarray(v[:, t]).astype(np.float32))
        qt = np.ascontiguousarray(q[:, t])
        # keys are stored as fp32 in the cache: compare with the fp32-rounded inputs
        ref = O.prefill_attention(q, k.astype(np.float32), v.astype(np.float32), ev, w,
                                  rows=[(b, hq, t) for b in range(B) for hq in range(Hq)])
        got = c.decode_attention(0, qt)
        assert np.allclose(got.reshape(-1, D), ref, atol=1e-12)
    assert np.allclose(full[:, T - 1], c.decode_attention(0, np.ascontiguousarray(q[:, T - 1])), atol=1e-6)


def test_cache_clone_is_independent():
    # a clone continues exactly like the original, and appending to one leaves the other unchanged
    B, T, Hq, Hkv, D, w, P = 1, 30, 2, 1, 8, 4, 4
    q, k, v = rand_qkv(16, B, T, Hq, Hkv, D)
    ev = (np.random.default_rng(17).random((B, Hkv, T)) > 0.5).astype(np.uint8)
    c = O.Cache(1, B, Hkv, D, w, P, T, 40, 0)
    c.prefill(0, np.ascontiguousarray(ev[:, :, :20]), k[:, :20].astype(np.float32), v[:, :20].astype(np.float32))
    d = c.clone()
    q20 = np.ascontiguousarray(q[:, 20])
    before = c.decode_attention(0, q20)
    for t in range(20, 25):
        d.append(0, np.ascontiguousarray(ev[:, :, t]), np.ascontiguousarray(k[:, t]).astype(np.float32),
                 np.ascontiguousarray(v[:, t]).astype(np.float32))
    assert np.array_equal(c.decode_attention(0, q20), before)
    for t in range(20, 25):
        c.append(0, np.ascontiguousarray(ev[:, :, t]), np.ascontiguousarray(k[:, t]).astype(np.float32),
                 np.ascontiguousarray(v[:, t]).astype(np.float32))
    q25 = np.ascontiguousarray(q[:, 24])
    assert np.array_equal(c.decode_attention(0, q25), d.decode_attention(0, q25))
    del c
    assert np.isfinite(d.decode_attention(0, q25)).all()


# ---------------------------------------------------------------------------
# FP8 pages
# ---------------------------------------------------------------------------
def test_fp8_prefill_page_scale_and_codes():
    B, H, D, w, P, T = 1, 1, 8, 2, 4, 6
    rng = np.random.default_rng(16)
    k = rng.standard_normal((B, T, H, D)).astype(np.float32)
    v = rng.standard_normal((B, T, H, D)).astype(np.float32)
    ev = np.zeros((B, H, T), np.uint8)  # all kept: slot t holds token t
    c = O.Cache(1, B, H, D, w, P, T, 4, 0, fp8=True)
    c.prefill(0, ev, k, v)
    pg = c.pages()
    for p in range(2):
        rows = k[0, p * P:(p + 1) * P, 0]
        s = np.float32(np.max(np.abs(rows))) / np.float32(448.0)
        assert pg["kscale"][p] == s
        assert np.array_equal(pg["kcode"][p, :len(rows)], O.e4m3_encode(rows / s))


def test_fp8_decode_rescale_rule():
    # row 0 has amax 1; row 1 has amax 2 -> the page scale doubles and row 0 is
    # re-encoded from its decoded value
    D, w, P = 4, 2, 4
    c = O.Cache(1, 1, 1, D, w, P, 8, 2, 0, fp8=True)
    r0 = np.array([[1.0, 0.3, -0.7, 0.1]], np.float32)
    r1 = np.array([[2.0, -1.5, 0.2, 0.9]], np.float32)
    c.prefill(0, np.zeros((1, 1, 1), np.uint8), r0.reshape(1, 1, 1, D), r0.reshape(1, 1, 1, D))
    c.append(0, np.zeros((1, 1), np.uint8), r1, r1)
    pg = c.pages()
    s0 = np.float32(1.0) / np.float32(448.0)
    s1 = np.float32(2.0) / np.float32(448.0)
    assert pg["kscale"][0] == s1
    c0 = O.e4m3_encode(r0[0] / s0)
    dq = (O.e4m3_decode(c0).astype(np.float32) * s0).astype(np.float32)
    assert np.array_equal(pg["kcode"][0, 0], O.e4m3_encode(dq / s1))
    assert np.array_equal(pg["kcode"][0, 1], O.e4m3_encode(r1[0] / s1))


# ---------------------------------------------------------------------------
# Chunked prefill ([DMS-Qwen3], advanced options: the prompt is prefilled in
# fixed-size chunks, each attending to the cache and to itself, and the chunks'
# outputs are concatenated)
# ---------------------------------------------------------------------------
def _chunked(c, layer, q, k, v, ev, splits, rows_per_call=None):
    outs, t0 = [], 0
    for n in splits:
        sl = slice(t0, t0 + n)
        outs.append(c.prefill_attention(layer, np.ascontiguousarray(q[:, sl]), np.ascontiguousarray(k[:, sl]),
                                        np.ascontiguousarray(v[:, sl]), np.ascontiguousarray(ev[:, :, sl])))
        c.prefill(layer, np.ascontiguousarray(ev[:, :, sl]), np.ascontiguousarray(k[:, sl]).astype(np.float32),
                  np.ascontiguousarray(v[:, sl]).astype(np.float32))
        t0 += n
    return np.concatenate(outs, 1)


@pytest.mark.parametrize("splits", [[50], [13, 1, 20, 16], [3, 47], [8, 8, 8, 8, 8, 10], [7, 30, 13]])
def test_chunked_prefill_equals_one_prefill(splits):
    """With exact pages (bf16/fp32 values) a chunked prefill leaves the same
    cache state and pages as one prefill of the whole prompt, and its rows'
    attention equals the whole prompt's masked attention."""
    B, T, Hq, Hkv, D, w, P = 2, 50, 4, 2, 16, 8, 4
    # values the pages hold exactly (fp32 numbers)
    q, k, v = (x.astype(np.float32).astype(np.float64) for x in rand_qkv(21, B, T, Hq, Hkv, D))
    ev = (np.random.default_rng(22).random((B, Hkv, T)) < 0.6).astype(np.uint8)
    one = O.Cache(1, B, Hkv, D, w, P, T + 4, 64, 0)
    one.prefill(0, ev, k.astype(np.float32), v.astype(np.float32))
    ref = O.prefill_attention(q, k, v, ev, w)
    ch = O.Cache(1, B, Hkv, D, w, P, T + 4, 64, 0)
    got = _chunked(ch, 0, q, k, v, ev, splits)
    assert np.allclose(got, ref, rtol=0, atol=1e-12)
    a, b = one.export(0), ch.export(0)
    for key in ("npos", "count", "npages", "ring_slot", "ring_evict", "next_page"):
        assert np.array_equal(a[key], b[key]), key
    # page ids follow each call's grant order (one counter, (b, h) row-major
    # per call), so they differ between one call and several; the pages used
    # and every slot's stored row do not
    pa, pb = one.pages(), ch.pages()
    used_a, used_b = set(), set()
    for bb in range(B):
        for h in range(Hkv):
            n = a["count"][bb, h]
            assert np.array_equal(a["slot_pos"][bb, h, :n], b["slot_pos"][bb, h, :n])
            ida = a["page_table"][bb, h, :a["npages"][bb, h]]
            idb = b["page_table"][bb, h, :b["npages"][bb, h]]
            used_a |= set(ida.tolist())
            used_b |= set(idb.tolist())
            for key in ("kval", "vval"):
                ra = pa[key][ida].reshape(-1, D)[:n]
                rb = pb[key][idb].reshape(-1, D)[:n]
                assert np.array_equal(ra, rb), key
    assert used_a == used_b
    # and the decode steps after it see the same cache
    qd = np.ascontiguousarray(q[:, T - 1])
    assert np.array_equal(one.decode_attention(0, qd), ch.decode_attention(0, qd))


def test_chunk_attention_sees_marked_window_keys_until_they_leave():
    """A marked token of the previous chunk stays visible to the next chunk's
    queries while it is inside their window, then disappears: brute force over
    the visible set, with a single marked token."""
    B, Hq, Hkv, D, w, P = 1, 1, 1, 8, 4, 4
    T0, C = 6, 6
    q, k, v = (x.astype(np.float32).astype(np.float64) for x in rand_qkv(23, B, T0 + C, Hq, Hkv, D))
    ev = np.zeros((B, Hkv, T0 + C), np.uint8)
    ev[0, 0, 4] = 1  # position 4 marked: visible to queries 4..7, gone from query 8 on
    c = O.Cache(1, B, Hkv, D, w, P, T0 + C, 8, 0)
    c.prefill(0, np.ascontiguousarray(ev[:, :, :T0]), k[:, :T0].astype(np.float32), v[:, :T0].astype(np.float32))
    got = c.prefill_attention(0, q[:, T0:], k[:, T0:], v[:, T0:], np.ascontiguousarray(ev[:, :, T0:]))
    sc = 1 / np.sqrt(D)
    for i in range(C):
        qi = T0 + i
        vis = [j for j in range(qi + 1) if not (j == 4 and qi - j >= w)]
        s = np.array([q[0, qi, 0] @ k[0, j, 0] * sc for j in vis])
        p = np.exp(s - s.max())
        want = (p[:, None] * v[0, vis, 0]).sum(0) / p.sum()
        assert np.allclose(got[0, i, 0], want, rtol=0, atol=1e-12), i


def test_fp8_chunk_of_one_token_is_a_decode_append():
    """The FP8 rule for a prefill call whose rows land in a page that already
    holds rows reduces, for a one-token call, to the decode append's rule."""
    B, H, D, w, P, T0 = 1, 2, 8, 4, 4, 9
    rng = np.random.default_rng(24)
    k = (rng.standard_normal((B, T0 + 1, H, D)) * np.linspace(0.5, 4, T0 + 1)[None, :, None, None]).astype(np.float32)
    v = rng.standard_normal((B, T0 + 1, H, D)).astype(np.float32)
    ev = (rng.random((B, H, T0 + 1)) < 0.5).astype(np.uint8)
    a = O.Cache(1, B, H, D, w, P, T0 + 1, 16, 0, fp8=True)
    a.prefill(0, np.ascontiguousarray(ev[:, :, :T0]), np.ascontiguousarray(k[:, :T0]), np.ascontiguousarray(v[:, :T0]))
    b = a.clone()
    a.prefill(0, np.ascontiguousarray(ev[:, :, T0:]), np.ascontiguousarray(k[:, T0:]), np.ascontiguousarray(v[:, T0:]))
    b.append(0, np.ascontiguousarray(ev[:, :, T0]), np.ascontiguousarray(k[:, T0]), np.ascontiguousarray(v[:, T0]))
    pa, pb = a.pages(), b.pages()
    for key in ("kcode", "vcode", "kscale", "vscale", "kval", "vval"):
        assert np.array_equal(pa[key], pb[key]), key
    sa, sb = a.export(0), b.export(0)
    assert np.array_equal(sa["count"], sb["count"]) and np.array_equal(sa["slot_pos"], sb["slot_pos"])


def test_fp8_chunked_scales_cover_every_row():
    """After a chunked FP8 prefill every page's scale is at least each of its
    rows' max |x| / 448, and every stored row decodes to within half a code
    step of its input (the rescale only coarsens the grid)."""
    B, H, D, w, P, T = 1, 2, 8, 6, 4, 40
    rng = np.random.default_rng(25)
    k = (rng.standard_normal((B, T, H, D)) * rng.uniform(0.2, 5, (1, T, 1, 1))).astype(np.float32)
    v = rng.standard_normal((B, T, H, D)).astype(np.float32)
    ev = (rng.random((B, H, T)) < 0.5).astype(np.uint8)
    c = O.Cache(1, B, H, D, w, P, T, 32, 0, fp8=True)
    q = np.zeros((B, T, 2, D))
    _chunked(c, 0, q, k, v, ev, [9, 5, 17, 9])
    s, pg = c.export(0), c.pages()
    for h in range(H):
        for sl in range(s["count"][0, h]):
            t = s["slot_pos"][0, h, sl]
            pid = s["page_table"][0, h, sl // P]
            sc = pg["kscale"][pid]
            assert sc >= np.float32(np.max(np.abs(k[0, t, h]))) / np.float32(448.0)
            # E4M3 has 3 mantissa bits: relative step 2^-3 above the subnormals
            err = np.abs(pg["kval"][pid, sl % P] - k[0, t, h])
            assert np.all(err <= np.maximum(np.abs(k[0, t, h]) * 2.0 ** -3, sc * 2.0 ** -8) + 1e-12)


# ---------------------------------------------------------------------------
# Decision shift ([DMS-Qwen3], attention: the training path shifts the decision
# logits by one position).  +1: token t is marked by token t - 1's decision
# (token 0 by the padding, "keep"); -1: token t's decision marks token t - 1.
# Each reduces to the unshifted rule applied to the correspondingly shifted
# decisions.
# ---------------------------------------------------------------------------
def _shifted_bits(bits, shift):
    out = np.zeros_like(bits)
    if shift == 1:
        out[..., 1:] = bits[..., :-1]
    elif shift == -1:
        out[..., :-1] = bits[..., 1:]   # the last token's mark is still pending (keep)
    else:
        out[:] = bits
    return out


@pytest.mark.parametrize("shift", [1, -1])
@pytest.mark.parametrize("splits", [[40], [11, 17, 12]])
def test_shift_reduces_to_the_unshifted_rule(shift, splits):
    B, H, D, w, P, T, n = 2, 2, 8, 5, 4, 40, 15
    rng = np.random.default_rng(30 + shift)
    bits = (rng.random((B, H, T + n)) < 0.55).astype(np.uint8)
    k = rng.standard_normal((B, T + n, H, D)).astype(np.float32)
    a = O.Cache(1, B, H, D, w, P, T + n, 120, 0, shift=shift)
    t0 = 0
    for m in splits:
        a.prefill(0, np.ascontiguousarray(bits[:, :, t0:t0 + m]), np.ascontiguousarray(k[:, t0:t0 + m]),
                  np.ascontiguousarray(k[:, t0:t0 + m]))
        t0 += m
    for t in range(T, T + n):
        a.append(0, np.ascontiguousarray(bits[:, :, t]), np.ascontiguousarray(k[:, t]), np.ascontiguousarray(k[:, t]))
    ref_bits = _shifted_bits(bits, shift)
    b = O.Cache(1, B, H, D, w, P, T + n, 120, 0)
    b.prefill(0, np.ascontiguousarray(ref_bits[:, :, :T]), np.ascontiguousarray(k[:, :T]), np.ascontiguousarray(k[:, :T]))
    for t in range(T, T + n):
        b.append(0, np.ascontiguousarray(ref_bits[:, :, t]), np.ascontiguousarray(k[:, t]), np.ascontiguousarray(k[:, t]))
    sa, sb = a.export(0), b.export(0)
    for key in ("count", "npages", "ring_slot", "ring_evict", "next_page", "slot_pos"):
        if key == "slot_pos":
            for bb in range(B):
                for h in range(H):
                    c = sa["count"][bb, h]
                    assert np.array_equal(sa[key][bb, h, :c], sb[key][bb, h, :c])
        elif key != "page_table":
            assert np.array_equal(sa[key], sb[key]), key
    if len(splits) == 1:  # one prefill call: the same page ids, so the same pages
        assert np.array_equal(a.pages()["kval"], b.pages()["kval"])


@pytest.mark.parametrize("shift", [1, -1])
def test_shift_attention_reduces_to_masked_attention(shift):
    """A prefill's rows under a shift see exactly the keys the unshifted mask
    gives for the shifted decisions; across a chunk boundary too."""
    B, Hq, Hkv, D, w, P, T = 1, 2, 1, 8, 6, 4, 36
    q, k, v = (x.astype(np.float32).astype(np.float64) for x in rand_qkv(33, B, T, Hq, Hkv, D))
    bits = (np.random.default_rng(34).random((B, Hkv, T)) < 0.6).astype(np.uint8)
    ref = O.prefill_attention(q, k, v, _shifted_bits(bits, shift), w)
    c = O.Cache(1, B, Hkv, D, w, P, T, 40, 0, shift=shift)
    got = _chunked(c, 0, q, k, v, bits, [13, 23])
    assert np.allclose(got, ref, rtol=0, atol=1e-12)


# ---------------------------------------------------------------------------
# Importance-score source (the KVzap-linear page: one Linear per layer from the
# hidden state to a score per KV head; prune below the threshold, keep the
# most recent tokens)
# ---------------------------------------------------------------------------
def test_decide_score_is_threshold_minus_linear_score():
    rng = np.random.default_rng(40)
    B, T, hid, H = 2, 7, 64, 3
    h = rng.standard_normal((B, T, hid))
    W = rng.standard_normal((H, hid)) / 8
    bias = rng.standard_normal(H)
    thr = np.array([[-4.0, 0.5, 1.0], [2.0, -1.0, 0.0]])
    a = O.decide_score(h, W, bias, thr)
    want = thr[:, :, None] - (np.einsum("bti,hi->bht", h, W) + bias[None, :, None])
    assert np.allclose(a, want, rtol=0, atol=1e-12)
    # no normalisation: the score is linear in the hidden state (the adapter's
    # RMSNorm would make it scale-invariant instead)
    a2 = O.decide_score(2 * h, W, None, np.zeros((B, H)))
    assert np.allclose(a2, 2 * O.decide_score(h, W, None, np.zeros((B, H))), rtol=0, atol=1e-12)
    # zero weights: every token scores its bias; layer mode copies head 0
    assert np.array_equal(O.decide_score(h, np.zeros((H, hid)), None, thr), np.broadcast_to(thr[:, :, None], (B, H, T)))
    al = O.decide_score(h, W, bias, thr, layer_mode=True)
    assert np.array_equal(al[:, 1], al[:, 0]) and np.array_equal(al[:, 0], a[:, 0])


def test_score_pruning_keeps_recent_tokens_and_high_scores():
    """With window 128 the delayed-eviction rule keeps exactly what the page's
    pruning keeps: the last 128 tokens and every earlier token whose score is
    not below the threshold."""
    rng = np.random.default_rng(41)
    T, hid, w, P = 700, 32, 128, 64
    h = rng.standard_normal((1, T, hid))
    W = rng.standard_normal((1, hid)) / 6
    a = O.decide_score(h, W, None, np.array([[-0.3]]))
    ev = O.evict_bits(a)
    c = O.Cache(1, 1, 1, 8, w, P, T, 64, 0, store_values=False)
    c.prefill(0, ev)
    s = c.export(0)
    score = (h[0] @ W[0])
    keep = set(range(T - w, T)) | {j for j in range(T - w) if score[j] >= -0.3}
    assert sorted(s["slot_pos"][0, 0, :s["count"][0, 0]]) == sorted(keep)


# ---------------------------------------------------------------------------
# Training mode: Gumbel-sigmoid gate and soft-gated attention ([DMS-Qwen3],
# "Gumbel 噪声与可微门控" and "注意力实现")
# ---------------------------------------------------------------------------
def test_train_gate_definition():
    rng = np.random.default_rng(50)
    a = rng.standard_normal((2, 3, 40)) * 3
    u = rng.random((2, 3, 40))
    g = np.log(u) - np.log1p(-u)
    tau = 0.1
    prob, hard, pen = O.train_gate(a, g, tau)
    l = (a + g) / tau
    assert np.allclose(prob, torch.sigmoid(torch.from_numpy(l)).numpy(), rtol=1e-12, atol=1e-15)
    assert np.array_equal(hard, (a + g > 0).astype(np.float64))
    # penalty: logsigmoid of the negated logit of the previous position; none at 0
    want = torch.nn.functional.logsigmoid(-torch.from_numpy(l)).numpy()
    assert np.all(pen[:, :, 0] == 0)
    assert np.allclose(pen[:, :, 1:], want[:, :, :-1], rtol=1e-12, atol=1e-14)
    # = log(1 - p) of the previous position
    assert np.allclose(np.exp(pen[:, :, 1:]), 1 - prob[:, :, :-1], rtol=1e-9, atol=1e-12)
    # no noise: the gate of the logit itself
    p0, h0, _ = O.train_gate(a, None, tau)
    assert np.array_equal(h0, (a > 0).astype(np.float64))


def test_train_attention_reduces_to_causal_and_window():
    rng = np.random.default_rng(51)
    B, T, Hq, Hkv, D, w = 1, 50, 4, 2, 16, 8
    q, k, v = rand_qkv(52, B, T, Hq, Hkv, D)
    def sdpa(mask):
        qq = torch.from_numpy(q).permute(0, 2, 1, 3)
        kk = torch.from_numpy(k).permute(0, 2, 1, 3).repeat_interleave(Hq // Hkv, 1)
        vv = torch.from_numpy(v).permute(0, 2, 1, 3).repeat_interleave(Hq // Hkv, 1)
        return torch.nn.functional.scaled_dot_product_attention(qq, kk, vv, attn_mask=mask).permute(0, 2, 1, 3).numpy()
    i, j = np.arange(T)[:, None], np.arange(T)[None, :]
    causal = torch.from_numpy(j <= i)
    # no penalty (every gate closed): dense causal attention
    o = O.train_attention(q, k, v, np.zeros((B, Hkv, T)), w)
    assert np.allclose(o, sdpa(causal), rtol=0, atol=1e-12)
    # the window covers the prompt: the penalty is never applied
    o = O.train_attention(q, k, v, rng.standard_normal((B, Hkv, T)) - 5, T)
    assert np.allclose(o, sdpa(causal), rtol=0, atol=1e-12)
    # a huge penalty everywhere: pure sliding-window attention
    o = O.train_attention(q, k, v, np.full((B, Hkv, T), -1e4), w)
    assert np.allclose(o, sdpa(torch.from_numpy((j <= i) & (i - j < w))), rtol=0, atol=1e-12)
    # an additive per-key bias outside the window: SDPA with a float mask
    pen = -np.abs(rng.standard_normal((B, Hkv, T)))
    bias = np.where(i - j < w, 0.0, pen[0, 0][None, :])
    bias = np.where(j <= i, bias, -np.inf)
    o = O.train_attention(q[:, :, :1], k[:, :, :1], v[:, :, :1], pen[:, :1], w)
    qq, kk, vv = (torch.from_numpy(x[:, :, :1]).permute(0, 2, 1, 3) for x in (q, k, v))
    ref = torch.nn.functional.scaled_dot_product_attention(qq, kk, vv, attn_mask=torch.from_numpy(bias)).permute(0, 2, 1, 3)
    assert np.allclose(o, ref.numpy(), rtol=0, atol=1e-12)


def test_train_attention_hard_limit_is_the_inference_mask():
    """As tau -> 0 the gate's penalty is 0 or -inf: the training attention
    becomes the inference DMS mask of the decisions shifted right by one
    (the +1 decision shift)."""
    B, T, Hq, Hkv, D, w = 2, 60, 4, 2, 16, 8
    q, k, v = rand_qkv(53, B, T, Hq, Hkv, D)
    a = np.where(np.random.default_rng(54).random((B, Hkv, T)) < 0.5, -1.0, 1.0)
    _, hard, pen = O.train_gate(a, None, 1e-4)    # |l| = 1e4: penalty 0 or about -1e4
    o = O.train_attention(q, k, v, pen, w)
    marks = np.zeros((B, Hkv, T), np.uint8)
    marks[:, :, 1:] = hard[:, :, :-1]
    assert np.allclose(o, O.prefill_attention(q, k, v, marks, w), rtol=0, atol=1e-12)
