"""Training-mode forward on the GPU ([DMS-Qwen3], "Gumbel 噪声与可微门控" and
"注意力实现"): dms_train_gate (Gumbel-sigmoid gate, straight-through forward
value, shifted logsigmoid penalty) and dms_train_attention (the soft-gated
score_mod attention on the tensor cores), against the fp64 oracle on the same
seeded inputs: probabilities and penalties within fp32 rounding, hard
decisions exactly (away from a zero logit), attention max-abs 2e-2 (bf16).
"""
import numpy as np
import pytest
import torch

from harness import Case, make_desc
from learned_kv_cache_dms_b200 import inputs as I
from oracle import oracle as O

CASES = {
    "d128_g4": dict(B=2, T=700, Hq=8, Hkv=2, D=128, w=64, rows=None, seed=90),
    "d64_g4_w128": dict(B=1, T=1000, Hq=32, Hkv=8, D=64, w=128, rows=None, seed=91),
    "d128_g8_ragged": dict(B=3, T=333, Hq=16, Hkv=2, D=128, w=48, rows=None, seed=92),
    # the Qwen3-8B layer shape, 8192 tokens, window 512 (dense causal work), sampled rows
    "qwen8b_8192": dict(B=1, T=8192, Hq=32, Hkv=8, D=128, w=512, rows=256, seed=1002),
}
TAU = 0.1


@pytest.mark.gpu
@pytest.mark.parametrize("name", sorted(CASES))
def test_train_gate_and_attention(name):
    from learned_kv_cache_dms_b200 import binding as B_
    p = CASES[name]
    B, T, Hq, Hkv, D, w, s = p["B"], p["T"], p["Hq"], p["Hkv"], p["D"], p["w"], p["seed"]
    q = I.normal(s, (0, 1), (B, T, Hq, D), "bf16")
    k = I.normal(s, (0, 2), (B, T, Hkv, D), "bf16")
    v = I.normal(s, (0, 3), (B, T, Hkv, D), "bf16")
    alpha = (I.normal(s, (0, 5), (B, Hkv, T), "f32", std=2.0) - 0.5).float()
    u = I.uniform(s, (0, 6), (B, Hkv, T), 1e-6, 1 - 1e-6)
    noise = (torch.log(u) - torch.log1p(-u)).float()   # logistic noise of the binary Gumbel-sigmoid
    # oracle
    prob_o, hard_o, pen_o = O.train_gate(alpha.double().numpy(), noise.double().numpy(), TAU)
    rows = None
    if p["rows"]:
        rng = np.random.default_rng(s)
        rows = np.stack([rng.integers(0, B, p["rows"]), rng.integers(0, Hq, p["rows"]),
                         rng.integers(0, T, p["rows"])], 1)
        rows[0, 2] = T - 1
    o_o = O.train_attention(q.double().numpy(), k.double().numpy(), v.double().numpy(), pen_o, w, rows=rows)
    # GPU
    case = Case(B=B, T=T, steps=0, Hq=Hq, Hkv=Hkv, D=D, w=w, P=16 if w <= 64 else 64, act="bf16", kv="bf16",
                source="input")
    dev = torch.device("cuda")
    cache = B_.Cache(make_desc(B_, case), dev)
    a_d, n_d = alpha.to(dev), noise.to(dev)
    prob, hard, pen = (torch.empty(B, Hkv, T, dtype=torch.float32, device=dev) for _ in range(3))
    B_.dms_train_gate(cache.handle, T, a_d, n_d, TAU, prob, hard, pen)
    qd, kd, vd = q.to(dev), k.to(dev), v.to(dev)
    o = torch.empty_like(qd)
    B_.dms_train_attention(cache.handle, T, qd, kd, vd, pen, o)
    torch.cuda.synchronize()
    assert cache.status() == 0
    # gate
    g = prob.double().cpu().numpy()
    assert np.max(np.abs(g - prob_o)) < 1e-6
    clear = np.abs(alpha.double().numpy() + noise.double().numpy()) > 1e-5
    assert np.array_equal(hard.cpu().numpy()[clear], hard_o[clear])
    pg = pen.double().cpu().numpy()
    assert np.all(np.abs(pg - pen_o) <= 1e-5 * np.maximum(1.0, np.abs(pen_o)))
    # attention
    og = o.double().cpu().numpy()
    if rows is not None:
        og = og[rows[:, 0], rows[:, 2], rows[:, 1]]
    err = float(np.max(np.abs(og - o_o)))
    assert err <= 2e-2, err
    print(name, "attention max-abs", err)
    cache.close()


@pytest.mark.gpu
def test_train_refusals():
    from learned_kv_cache_dms_b200 import binding as B_
    dev = torch.device("cuda")
    case = Case(B=1, T=64, steps=0, Hq=6, Hkv=2, D=64, w=32, P=16, act="bf16", kv="bf16", source="input")
    cache = B_.Cache(make_desc(B_, case), dev)
    x = torch.zeros(1, 64, 6, 64, dtype=torch.bfloat16, device=dev)
    kv = torch.zeros(1, 64, 2, 64, dtype=torch.bfloat16, device=dev)
    pen = torch.zeros(1, 2, 64, device=dev)
    with pytest.raises(B_.DMSError) as ex:   # g = 3: not a tcgen05 shape
        B_.dms_train_attention(cache.handle, 64, x, kv, kv, pen, torch.empty_like(x))
    assert ex.value.code == B_.DMS_ERR_INVALID
    a = torch.zeros(1, 2, 64, device=dev)
    with pytest.raises(B_.DMSError) as ex:   # tau must be positive
        B_.dms_train_gate(cache.handle, 64, a, None, 0.0, a, a, a)
    assert ex.value.code == B_.DMS_ERR_INVALID
    cache.close()
