"""GPU: a decode run is a pure function of its inputs.  The same prompt and
tokens through a fresh prefill give bit-identical outputs, decisions, cache
state and pages, for both decode attention kernels, at a batch whose heads are
shared by several CTAs (partials merged by whichever CTA finishes last)."""
import numpy as np
import pytest
import torch

from learned_kv_cache_dms_b200 import inputs as I


def _run(B_, desc, x, off, steps):
    cache = B_.Cache(desc)
    o = torch.empty_like(x["q"])
    alpha = torch.empty(desc.batch, desc.num_kv_heads, x["q"].shape[1], dtype=torch.float32, device="cuda")
    pd = B_.decide_params(off, hidden=x["h"], norm_weight=x["gamma"], proj_weight=x["W"])
    cache.prefill(0, x["q"], x["k"], x["v"], o, alpha, decide=pd)
    outs, alphas = [], []
    for s in range(steps):
        od = torch.empty_like(x["qd"][s])
        ad = torch.empty(desc.batch, desc.num_kv_heads, dtype=torch.float32, device="cuda")
        dd = B_.decide_params(off, hidden=x["hd"][s], norm_weight=x["gamma"], proj_weight=x["W"])
        cache.decode_step(0, x["qd"][s], x["kd"][s], x["vd"][s], od, ad, decide=dd)
        outs.append(od)
        alphas.append(ad)
    torch.cuda.synchronize()
    st = {k: v.clone() for k, v in cache.state(0).items()}
    pg = {k: v.clone() for k, v in cache.pages().items()}
    status = cache.status()
    cache.close()
    return torch.stack(outs), torch.stack(alphas), st, pg, status


@pytest.mark.gpu
@pytest.mark.parametrize("kernel", ["flat", "cluster"])
def test_decode_is_deterministic(kernel):
    from learned_kv_cache_dms_b200 import binding as B_
    B, T, S, Hq, Hkv, D, hidden, w, P = 8, 2048, 64, 32, 8, 128, 512, 512, 256
    d = B_.dms_cache_desc_default()
    d.num_layers, d.batch, d.num_q_heads, d.num_kv_heads = 1, B, Hq, Hkv
    d.head_dim, d.hidden, d.window, d.block = D, hidden, w, P
    d.max_positions, d.prealloc_tokens = T + S, 1024
    d.pool_pages = B * Hkv * (-(-(T + S) // P))
    d.decode_kernel = {"flat": B_.DMS_DECODE_FLAT, "cluster": B_.DMS_DECODE_CLUSTER}[kernel]
    g = torch.Generator(device="cuda")
    g.manual_seed(1234)

    def rn(*shape, std=1.0):
        return (torch.randn(*shape, generator=g, device="cuda") * std).to(torch.bfloat16)

    x = dict(q=rn(B, T, Hq, D), k=rn(B, T, Hkv, D), v=rn(B, T, Hkv, D), h=rn(B, T, hidden),
             qd=rn(S, B, Hq, D), kd=rn(S, B, Hkv, D), vd=rn(S, B, Hkv, D), hd=rn(S, B, hidden),
             gamma=rn(hidden), W=rn(Hkv, hidden, std=hidden ** -0.5))
    # offsets for per-(b, h) keep fractions in [1/16, 1/4] from the library's own logits
    probe = B_.Cache(d)
    raw = torch.empty(B, Hkv, T, dtype=torch.float32, device="cuda")
    zero = torch.zeros(B, Hkv, dtype=torch.float32, device="cuda")
    B_.dms_decide(probe.handle, T, B_.decide_params(zero, hidden=x["h"], norm_weight=x["gamma"],
                                                    proj_weight=x["W"]), None, raw)
    torch.cuda.synchronize()
    probe.close()
    keep = I.uniform(7, (77,), (B, Hkv), 1 / 16, 1 / 4).numpy()
    off, _ = I.calibrate_offsets(raw.cpu().numpy(), keep)
    off = torch.from_numpy(off).cuda()

    r1 = _run(B_, d, x, off, S)
    r2 = _run(B_, d, x, off, S)
    assert r1[4] == 0 and r2[4] == 0
    diff = (r1[0].float() - r2[0].float()).abs()
    bad = torch.nonzero(diff.amax(dim=-1))
    assert bad.numel() == 0, "decode outputs differ at (step, b, q head): %s; max %.3g" % (
        bad[:8].tolist(), float(diff.max()))
    assert torch.equal(r1[1], r2[1]), "decision logits differ"
    for k in r1[2]:
        assert torch.equal(r1[2][k], r2[2][k]), "state %s differs" % k
    for k in r1[3]:
        assert torch.equal(r1[3][k], r2[3][k]), "pages %s differ" % k
    assert int(r1[2]["count"].min()) > 2 * P  # several sub-tiles and pages per head
    assert np.isfinite(r1[0].float().cpu().numpy()).all()
