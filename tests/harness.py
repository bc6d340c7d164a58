"""Shared parity harness: one seeded case run through the oracle (CPU) and
through libdms's C ABI (GPU), compared element by element.

Bit-exact: decisions, counts, page tables, slot maps, ring, page counter, stored
bf16/fp32 rows, FP8 codes and scales.  Within tolerance (max-abs vs the fp64
oracle): attention outputs, 2e-3 for fp32 and 2e-2 for bf16 / FP8 pages.
"""
from __future__ import annotations

import dataclasses

import numpy as np
import torch

from learned_kv_cache_dms_b200 import inputs as I
from oracle import oracle as O

TOL = {"f32": 2e-3, "bf16": 2e-2}
ALPHA_SCALE = 100.0
RMS_EPS = 1e-6
MIN_MARGIN = 0.02  # decisions are compared bit for bit only when |alpha| clears this


@dataclasses.dataclass
class Case:
    B: int = 1
    T: int = 256
    steps: int = 8
    Hq: int = 4
    Hkv: int = 2
    D: int = 64
    hidden: int = 256
    w: int = 32
    P: int = 16
    act: str = "f32"
    kv: str = "f32"
    source: str = "input"      # input | proj | key | query | score
    per: str = "head"          # head | layer
    keep: object = 0.5         # float, or (lo, hi) per (b, h)
    disable: bool = False
    rope: bool = False
    prealloc: int = 0
    pool_pages: int | None = None
    layers: int = 1
    layer: int = 0
    seed: int = 1
    attn_rows: int | None = None  # sample this many prefill rows (None: all)
    staged: bool = False          # decode through dms_decode_append + dms_decode_attention
    kernel: str = "auto"          # decode attention kernel: auto | cluster | flat
    chunks: tuple | None = None   # chunked prefill: the prompt's chunk sizes (summing to T)
    shift: int = 0                # decision shift: 0 own, +1 previous token's, -1 next token's decision

    @property
    def N(self):
        return self.T + self.steps

    @property
    def maxp(self):
        return -(-self.N // self.P)

    @property
    def pool(self):
        if self.pool_pages is not None:
            return self.pool_pages
        pre = min(self.maxp, -(-self.prealloc // self.P))
        return self.layers * self.B * self.Hkv * max(pre, self.maxp) + self.layers * self.B * self.Hkv * pre


def _keep(case):
    if isinstance(case.keep, tuple):
        lo, hi = case.keep
        return I.uniform(case.seed, (77,), (case.B, case.Hkv), lo, hi).numpy()
    return np.full((case.B, case.Hkv), float(case.keep))


def _f64(t):
    return t.double().numpy()


def build(case: Case):
    """Inputs (torch CPU tensors in the activation dtype) and the oracle's results."""
    s, B, N, T = case.seed, case.B, case.N, case.T
    q = I.normal(s, (case.layer, 1), (B, N, case.Hq, case.D), case.act)
    k = I.normal(s, (case.layer, 2), (B, N, case.Hkv, case.D), case.act)
    v = I.normal(s, (case.layer, 3), (B, N, case.Hkv, case.D), case.act)
    out = dict(q=q, k=k, v=v)
    keep = _keep(case)
    layer_mode = case.per == "layer"
    if case.source == "input":
        alpha = I.synthetic_alpha(s, (case.layer, 5), B, case.Hkv, N, keep)
        if layer_mode:
            alpha[:] = alpha[:, :1]
        alpha_o = alpha.double().numpy()
        out["alpha_in"] = alpha
        kz, qz = _f64(k), _f64(q)
    elif case.source == "score":
        # the importance score: Linear(hidden -> Hkv) with a bias, no norm;
        # thresholds calibrated per head like the adapter's offsets
        h = I.normal(s, (case.layer, 4), (B, N, case.hidden), case.act)
        W = I.normal(s, (case.layer, 11), (case.Hkv, case.hidden), case.act, std=case.hidden ** -0.5)
        bias = I.normal(s, (case.layer, 12), (case.Hkv,), case.act, std=0.1)
        neg_score = O.decide_score(_f64(h), _f64(W), _f64(bias), np.zeros((B, case.Hkv)), layer_mode)
        off, _ = I.calibrate_offsets(neg_score, keep)
        if layer_mode:
            off[:] = off[:, :1]
        thr = -off.astype(np.float64)
        alpha_o = O.decide_score(_f64(h), _f64(W), _f64(bias), thr, layer_mode)
        out.update(h=h, W=W, bias=bias, offset=torch.from_numpy(thr.astype(np.float32)))
        kz, qz = _f64(k), _f64(q)
    elif case.source == "proj":
        h = I.normal(s, (case.layer, 4), (B, N, case.hidden), case.act)
        gamma = I.normal(s, (case.layer, 10), (case.hidden,), case.act)
        W = I.normal(s, (case.layer, 11), (case.Hkv, case.hidden), case.act, std=case.hidden ** -0.5)
        raw = O.decide_proj(_f64(h), _f64(gamma), _f64(W), None, np.zeros((B, case.Hkv)), ALPHA_SCALE, RMS_EPS,
                            layer_mode)
        # offsets from every token's raw logit (prompt and decode), so that no
        # decision sits within the comparison margin
        off, _ = I.calibrate_offsets(raw, keep)
        if layer_mode:
            off[:] = off[:, :1]
        alpha_o = O.decide_proj(_f64(h), _f64(gamma), _f64(W), None, off, ALPHA_SCALE, RMS_EPS, layer_mode)
        out.update(h=h, gamma=gamma, W=W, offset=torch.from_numpy(off))
        kz, qz = _f64(k), _f64(q)
    else:
        src = k if case.source == "key" else q
        group = 1 if case.source == "key" else case.Hq // case.Hkv
        raw, _ = O.decide_neuron(_f64(src), group, case.Hkv, np.zeros((B, case.Hkv)), ALPHA_SCALE, layer_mode)
        off, _ = I.calibrate_offsets(raw, keep)
        if layer_mode:
            off[:] = off[:, :1]
        alpha_o, zeroed = O.decide_neuron(_f64(src), group, case.Hkv, off, ALPHA_SCALE, layer_mode)
        out["offset"] = torch.from_numpy(off)
        kz = zeroed if case.source == "key" else _f64(k)
        qz = zeroed if case.source == "query" else _f64(q)
    if case.source != "input":
        # the score is not multiplied by alpha_scale: the same margin on the
        # raw dot product as the adapter's (0.02 / 100)
        margin = MIN_MARGIN / ALPHA_SCALE if case.source == "score" else MIN_MARGIN
        m = np.min(np.abs(alpha_o))
        assert m > margin, "decision margin %.3g too small for a bit-exact comparison; change the seed" % m
    if case.rope:
        cos, sin = I.rope_tables(N, case.D)
        out["rope"] = (cos, sin)
        qz = O.rope(qz, 0, cos.double().numpy(), sin.double().numpy())
        kz = O.rope(kz, 0, cos.double().numpy(), sin.double().numpy())
    # the stored (activation-dtype) values of q and k after zeroing and rotation:
    # the fp64 rotation rounded once
    qs = O.round_to(qz, case.act)
    ks = O.round_to(kz, case.act)
    vs = _f64(v)
    evict = O.evict_bits(alpha_o, case.disable)
    out.update(alpha_o=alpha_o, evict=evict, q_stored=qs, k_stored=ks)

    # oracle: prefill attention, cache replay, decode attention
    rows = None
    if case.attn_rows is not None:
        rng = np.random.default_rng(case.seed + 99)
        rows = np.stack([rng.integers(0, B, case.attn_rows), rng.integers(0, case.Hq, case.attn_rows),
                         rng.integers(0, T, case.attn_rows)], 1)
        rows[: min(B, case.attn_rows), 2] = T - 1  # always include the last rows
        out["rows"] = rows
    cache = O.Cache(case.layers, B, case.Hkv, case.D, case.w, case.P, N, case.pool, case.prealloc,
                    fp8=case.kv == "fp8", shift=case.shift)
    if case.chunks is None and case.shift == 0:
        out["o_prefill"] = O.prefill_attention(qs[:, :T], ks[:, :T], vs[:, :T],
                                               np.ascontiguousarray(evict[:, :, :T]), case.w, rows=rows)
        cache.prefill(case.layer, np.ascontiguousarray(evict[:, :, :T]), ks[:, :T].astype(np.float32),
                      vs[:, :T].astype(np.float32))
    else:
        # each chunk attends to the cache as the earlier chunks left it, then is
        # appended (a shifted-decision prompt in one call goes the same way)
        chunks = case.chunks or (T,)
        assert sum(chunks) == T
        outs, t0 = [], 0
        for n in chunks:
            sl = slice(t0, t0 + n)
            ev_c = np.ascontiguousarray(evict[:, :, sl])
            r_c = None
            if rows is not None:
                sel = (rows[:, 2] >= t0) & (rows[:, 2] < t0 + n)
                r_c = rows[sel] - np.array([0, 0, t0])
            o_c = cache.prefill_attention(case.layer, np.ascontiguousarray(qs[:, sl]), np.ascontiguousarray(ks[:, sl]),
                                          np.ascontiguousarray(vs[:, sl]), ev_c, rows=r_c)
            outs.append((sel, o_c) if rows is not None else o_c)
            cache.prefill(case.layer, ev_c, np.ascontiguousarray(ks[:, sl]).astype(np.float32),
                          np.ascontiguousarray(vs[:, sl]).astype(np.float32))
            t0 += n
        if rows is None:
            out["o_prefill"] = np.concatenate(outs, 1)
        else:
            o = np.empty((rows.shape[0], case.D))
            for sel, o_c in outs:
                o[sel] = o_c
            out["o_prefill"] = o
    out["state_prefill"] = cache.export(case.layer)
    out["pages_prefill"] = cache.pages() if case.steps == 0 else None
    o_dec = []
    for t in range(T, N):
        cache.append(case.layer, np.ascontiguousarray(evict[:, :, t]), np.ascontiguousarray(ks[:, t]).astype(np.float32),
                     np.ascontiguousarray(vs[:, t]).astype(np.float32))
        o_dec.append(cache.decode_attention(case.layer, np.ascontiguousarray(qs[:, t])))
    out["o_decode"] = o_dec
    out["state_final"] = cache.export(case.layer)
    out["pages_final"] = cache.pages()
    out["oracle_status"] = cache.status
    return out


def marks(evict, shift):
    """Eviction marks of the tokens from their own decisions under a decision
    shift (+1: the previous token's decision, the first token keeps; -1: the
    next token's, the last token not yet marked)."""
    out = np.zeros_like(evict)
    if shift == 1:
        out[..., 1:] = evict[..., :-1]
    elif shift == -1:
        out[..., :-1] = evict[..., 1:]
    else:
        out[:] = evict
    return out


def make_desc(B_, case: Case):
    d = B_.dms_cache_desc_default()
    d.num_layers, d.batch, d.num_q_heads, d.num_kv_heads = case.layers, case.B, case.Hq, case.Hkv
    d.head_dim, d.hidden, d.window, d.block = case.D, case.hidden, case.w, case.P
    d.max_positions, d.prealloc_tokens, d.pool_pages = case.N, case.prealloc, case.pool
    d.act_dtype = {"f32": B_.DMS_F32, "bf16": B_.DMS_BF16}[case.act]
    d.kv_dtype = {"f32": B_.DMS_F32, "bf16": B_.DMS_BF16, "fp8": B_.DMS_FP8_E4M3}[case.kv]
    d.alpha_per = B_.DMS_ALPHA_PER_LAYER if case.per == "layer" else B_.DMS_ALPHA_PER_HEAD
    d.alpha_source = {"input": B_.DMS_ALPHA_PROJ, "proj": B_.DMS_ALPHA_PROJ, "key": B_.DMS_ALPHA_KEY_NEURON,
                      "query": B_.DMS_ALPHA_QUERY_NEURON, "score": B_.DMS_ALPHA_SCORE_LINEAR}[case.source]
    if case.source in ("key", "query", "input"):
        d.hidden = max(d.hidden, 8)
    d.alpha_scale, d.rms_eps = ALPHA_SCALE, RMS_EPS
    d.disable_eviction = int(case.disable)
    d.decision_shift = case.shift
    d.decode_kernel = {"auto": B_.DMS_DECODE_AUTO, "cluster": B_.DMS_DECODE_CLUSTER,
                       "flat": B_.DMS_DECODE_FLAT}[case.kernel]
    return d


def run_gpu(case: Case, ins, cache=None):
    """Run prefill + decode steps through the C ABI; returns GPU results on the CPU.

    With `cache` (an open binding.Cache of this case's descriptor) the run uses
    it as it is and leaves it open; otherwise a fresh cache is made and closed."""
    from learned_kv_cache_dms_b200 import binding as B_
    dev = torch.device("cuda")
    own = cache is None
    if own:
        cache = B_.Cache(make_desc(B_, case), dev)
    T, N, B = case.T, case.N, case.B
    q = ins["q"].to(dev)
    k = ins["k"].to(dev)
    v = ins["v"].to(dev)
    rope = tuple(t.to(dev) for t in ins["rope"]) if case.rope else None
    decide = None
    keep_alive = []
    gamma = bias = None
    if case.source in ("proj", "score"):
        h = ins["h"].to(dev)
        W = ins["W"].to(dev)
        if case.source == "proj":
            gamma = ins["gamma"].to(dev)
        else:
            bias = ins["bias"].to(dev)
        off = ins["offset"].to(dev)
        keep_alive += [h, gamma, W, off, bias]
    elif case.source in ("key", "query"):
        off = ins["offset"].to(dev)
        keep_alive.append(off)
    chunks = case.chunks or (T,)
    o_parts, a_parts, q_parts, k_parts = [], [], [], []
    t0 = 0
    for n in chunks:
        qp = q[:, t0:t0 + n].contiguous()
        kp = k[:, t0:t0 + n].contiguous()
        vp = v[:, t0:t0 + n].contiguous()
        o = torch.empty_like(qp)
        if case.source == "input":
            alpha = ins["alpha_in"][:, :, t0:t0 + n].contiguous().to(dev)
        else:
            alpha = torch.empty(B, case.Hkv, n, dtype=torch.float32, device=dev)
            if case.source in ("proj", "score"):
                hp = h[:, t0:t0 + n].contiguous()
                keep_alive.append(hp)
                decide = B_.decide_params(off, hidden=hp, norm_weight=gamma, proj_weight=W, proj_bias=bias)
            else:
                decide = B_.decide_params(off)
        cache.prefill(case.layer, qp, kp, vp, o, alpha, decide=decide, rope=rope)
        o_parts.append(o)
        a_parts.append(alpha)
        q_parts.append(qp)
        k_parts.append(kp)
        keep_alive += [vp]
        t0 += n
    torch.cuda.synchronize()
    res = dict(o_prefill=torch.cat(o_parts, 1).cpu(), alpha_prefill=torch.cat(a_parts, 2).cpu(),
               k_prefill=torch.cat(k_parts, 1).cpu(), q_prefill=torch.cat(q_parts, 1).cpu())
    res["state_prefill"] = {k_: t.cpu().clone() for k_, t in cache.state(case.layer).items()}
    if case.steps == 0:
        res["pages_prefill"] = {k_: t.cpu().clone() for k_, t in cache.pages().items()}
    o_dec, a_dec, qk_dec = [], [], []
    for t in range(T, N):
        qt, kt, vt = q[:, t].contiguous(), k[:, t].contiguous(), v[:, t].contiguous()
        ot = torch.empty_like(qt)
        if case.source == "input":
            at = ins["alpha_in"][:, :, t].contiguous().to(dev)
            dd = None
        else:
            at = torch.empty(B, case.Hkv, dtype=torch.float32, device=dev)
            if case.source in ("proj", "score"):
                ht = h[:, t].contiguous()
                dd = B_.decide_params(off, hidden=ht, norm_weight=gamma, proj_weight=W, proj_bias=bias)
                keep_alive.append(ht)
            else:
                dd = B_.decide_params(off)
        if case.staged:
            args = B_.Cache.decode_args(qt, kt, vt, ot, at, dd, rope)
            B_.dms_decode_append(cache.handle, case.layer, args)
            B_.dms_decode_attention(cache.handle, case.layer, qt, ot)
        else:
            cache.decode_step(case.layer, qt, kt, vt, ot, at, decide=dd, rope=rope)
        o_dec.append(ot)
        a_dec.append(at)
        qk_dec.append((qt, kt))
    torch.cuda.synchronize()
    res["o_decode"] = [x.cpu() for x in o_dec]
    res["alpha_decode"] = [x.cpu() for x in a_dec]
    # the decode rows as the step left them (decision element zeroed, rotated)
    res["q_decode"] = torch.stack([x[0].cpu() for x in qk_dec], 1) if qk_dec else None
    res["k_decode"] = torch.stack([x[1].cpu() for x in qk_dec], 1) if qk_dec else None
    res["state_final"] = {k_: t.cpu().clone() for k_, t in cache.state(case.layer).items()}
    res["pages_final"] = {k_: t.cpu().clone() for k_, t in cache.pages().items()}
    res["status"] = cache.status()
    res["positions"] = cache.positions(case.layer)
    if own:
        cache.close()
    return res


def compare_state(case, so, sg, npos):
    """Bit-exact comparison of the oracle's and the GPU's cache state for one layer."""
    B, H, w = case.B, case.Hkv, case.w
    cnt_o = so["count"]
    cnt_g = sg["count"].numpy()
    assert np.array_equal(cnt_o, cnt_g), "count"
    assert np.array_equal(so["npages"], sg["npages"].numpy()), "npages"
    assert so["next_page"] == int(sg["next_page"][0]), "next_page"
    assert np.array_equal(sg["pos"].numpy(), np.full(B, npos)), "pos"
    pt_g = sg["page_table"].numpy()
    sp_g = sg["slot_pos"].numpy()
    for b in range(B):
        for h in range(H):
            n = so["npages"][b, h]
            assert np.array_equal(so["page_table"][b, h, :n], pt_g[b, h, :n]), ("page_table", b, h)
            c = cnt_o[b, h]
            assert np.array_equal(so["slot_pos"][b, h, :c], sp_g[b, h, :c]), ("slot_pos", b, h)
    valid = [t % w for t in range(max(0, npos - w), npos)]
    assert np.array_equal(so["ring_slot"][:, :, valid], sg["ring_slot"].numpy()[:, :, valid]), "ring_slot"
    assert np.array_equal(so["ring_evict"][:, :, valid], sg["ring_evict"].numpy()[:, :, valid]), "ring_evict"


def compare_pages(case, so, po, pg):
    """Stored rows of every retained slot: bit-exact (values, or FP8 codes + scales)."""
    B, H, P = case.B, case.Hkv, case.P
    for b in range(B):
        for h in range(H):
            c = so["count"][b, h]
            ids = so["page_table"][b, h, : -(-c // P)]
            for p, pid in enumerate(ids):
                rows = min(P, c - p * P)
                if case.kv == "fp8":
                    assert np.array_equal(po["kcode"][pid, :rows], pg["k"][pid, :rows].numpy()), ("kcode", b, h, p)
                    assert np.array_equal(po["vcode"][pid, :rows], pg["v"][pid, :rows].numpy()), ("vcode", b, h, p)
                    assert po["kscale"][pid] == pg["k_scale"][pid].item(), ("kscale", b, h, p)
                    assert po["vscale"][pid] == pg["v_scale"][pid].item(), ("vscale", b, h, p)
                else:
                    assert np.array_equal(po["kval"][pid, :rows], pg["k"][pid, :rows].double().numpy()), ("k", b, h, p)
                    assert np.array_equal(po["vval"][pid, :rows], pg["v"][pid, :rows].double().numpy()), ("v", b, h, p)


def check_case(case: Case, ins=None, cache=None):
    ins = ins if ins is not None else build(case)
    res = run_gpu(case, ins, cache)
    tol = TOL[case.act]
    T = case.T
    # decisions
    if case.source != "input":
        a_g = res["alpha_prefill"].double().numpy()
        a_o = ins["alpha_o"][:, :, :T]
        assert np.max(np.abs(a_g - a_o)) < 1e-3 * max(1.0, float(np.max(np.abs(a_o)))), "alpha"
        assert np.array_equal(a_g > 0, a_o > 0), "decisions"
        for i, t in enumerate(range(T, case.N)):
            ad = res["alpha_decode"][i].double().numpy()
            ao = ins["alpha_o"][:, :, t]
            assert np.max(np.abs(ad - ao)) < 1e-3 * max(1.0, float(np.max(np.abs(ao)))), ("decode alpha", t)
            assert np.array_equal(ad > 0, ao > 0), ("decode decisions", t)
    # q and k as stored after the decision element is zeroed and the rotary
    # embedding applied: the oracle's fp64 rotation rounded once into the
    # activation dtype, bit for bit (rows_differing counts the elements that
    # differ; the assertion below requires none)
    rows_differing = compare_rows(case, ins, res)
    # state after prefill and after the decode steps
    compare_state(case, ins["state_prefill"], res["state_prefill"], T)
    compare_state(case, ins["state_final"], res["state_final"], case.N)
    assert res["positions"] == case.N
    compare_pages(case, ins["state_final"], ins["pages_final"], res["pages_final"])
    # attention
    og = res["o_prefill"].double().numpy()
    if ins.get("rows") is not None:
        r = ins["rows"]
        og = og[r[:, 0], r[:, 2], r[:, 1]]
    err_p = float(np.max(np.abs(og - ins["o_prefill"])))
    assert err_p <= tol, "prefill attention max-abs error %.3g > %.3g" % (err_p, tol)
    err_d = 0.0
    for i in range(case.steps):
        err_d = max(err_d, float(np.max(np.abs(res["o_decode"][i].double().numpy() - ins["o_decode"][i]))))
    assert err_d <= tol, "decode attention max-abs error %.3g > %.3g" % (err_d, tol)
    assert res["status"] == 0 and ins["oracle_status"] == 0
    return dict(err_prefill=err_p, err_decode=err_d, rows_differing=rows_differing)


def compare_rows(case, ins, res):
    """Rotated / zeroed q and k rows (prompt and decode) against the oracle, bit for bit."""
    T = case.T
    if not case.rope and case.source not in ("key", "query"):
        return 0
    pairs = [(res["q_prefill"], ins["q_stored"][:, :T]), (res["k_prefill"], ins["k_stored"][:, :T])]
    if res.get("q_decode") is not None:
        pairs += [(res["q_decode"], ins["q_stored"][:, T:]), (res["k_decode"], ins["k_stored"][:, T:])]
    bad = 0
    for g, o in pairs:
        bad += int(np.count_nonzero(g.double().numpy() != o))
    assert bad == 0, "%d rotated or zeroed q/k elements differ from the oracle's single rounding" % bad
    return bad
