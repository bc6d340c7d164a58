"""GPU parity: libdms (through the C ABI) against the CPU oracle on the same
seeded inputs.  Sizes are small enough for the oracle to finish in seconds but
span several tiles, pages and a ragged tail."""
import dataclasses

import numpy as np
import pytest
import torch

from harness import Case, build, check_case, marks

CASES = {
    # the tiny fp32 workload: B1, hidden 256, 4/2 heads, D64, 256 + 16 tokens, w32, P16, keep 1/2
    "tiny_f32_proj": Case(B=1, T=256, steps=16, Hq=4, Hkv=2, D=64, hidden=256, w=32, P=16, act="f32", kv="f32",
                          source="proj", keep=0.5, seed=1001),
    "bf16_d128_input_ragged": Case(B=2, T=600, steps=40, Hq=8, Hkv=2, D=128, w=64, P=32, act="bf16", kv="bf16",
                                   source="input", keep=0.3, prealloc=64, seed=2),
    "bf16_d128_proj": Case(B=2, T=515, steps=24, Hq=8, Hkv=4, D=128, hidden=512, w=96, P=32, act="bf16",
                           kv="bf16", source="proj", keep=(1 / 16, 1 / 4), seed=3),
    # a hidden size that is a multiple of 8 but not of the adapter kernel's chunks
    "bf16_proj_hidden_ragged": Case(B=2, T=300, steps=12, Hq=8, Hkv=4, D=64, hidden=328, w=64, P=32, act="bf16",
                                    kv="bf16", source="proj", keep=0.25, seed=31),
    # the same hidden size (3 chunks) over 157 token tiles: some CTAs take two
    # tiles, the second starting at an odd chunk index
    "bf16_proj_hidden_ragged_multitile": Case(B=2, T=5000, steps=8, Hq=8, Hkv=4, D=64, hidden=328, w=64, P=32,
                                              act="bf16", kv="bf16", source="proj", keep=0.25, attn_rows=64,
                                              seed=32),
    "bf16_d64_proj_layer": Case(B=2, T=333, steps=20, Hq=4, Hkv=4, D=64, hidden=256, w=48, P=16, act="bf16",
                                kv="bf16", source="proj", per="layer", keep=0.25, seed=4),
    "fp8_key_rope_head": Case(B=2, T=700, steps=30, Hq=8, Hkv=2, D=64, w=64, P=32, act="bf16", kv="fp8",
                              source="key", keep=0.125, rope=True, seed=5),
    "fp8_key_rope_layer": Case(B=2, T=700, steps=30, Hq=8, Hkv=2, D=64, w=64, P=32, act="bf16", kv="fp8",
                               source="key", per="layer", keep=0.125, rope=True, seed=6),
    "bf16_query_neuron": Case(B=1, T=400, steps=12, Hq=8, Hkv=2, D=128, w=64, P=32, act="bf16", kv="bf16",
                              source="query", keep=0.2, seed=7),
    "fp8_d128_input": Case(B=2, T=500, steps=20, Hq=4, Hkv=2, D=128, w=64, P=32, act="bf16", kv="fp8",
                           source="input", keep=0.4, seed=8),
    # FP8 pages with 16 query heads per KV head (the query-major decode tiles,
    # codes widened to bf16) and with 8 (key-major f16 tiles), D = 128 and 64
    "fp8_g16_d128_input": Case(B=2, T=450, steps=16, Hq=32, Hkv=2, D=128, w=64, P=32, act="bf16", kv="fp8",
                               source="input", keep=0.3, seed=41),
    "fp8_g8_d64_input_p48": Case(B=2, T=420, steps=16, Hq=16, Hkv=2, D=64, w=64, P=48, act="bf16", kv="fp8",
                                 source="input", keep=0.3, seed=42),
    "f32_rope_input": Case(B=1, T=200, steps=10, Hq=4, Hkv=1, D=128, w=40, P=16, act="f32", kv="f32",
                           source="input", keep=0.5, rope=True, seed=9),
    # degenerate decision patterns
    "all_keep": Case(B=1, T=300, steps=10, Hq=4, Hkv=2, D=64, w=32, P=16, act="bf16", kv="bf16", source="input",
                     keep=1.0, seed=10),
    "all_evict": Case(B=1, T=300, steps=40, Hq=4, Hkv=2, D=64, w=32, P=16, act="bf16", kv="bf16", source="input",
                      keep=0.0, seed=11),
    "disable_eviction": Case(B=1, T=300, steps=10, Hq=4, Hkv=2, D=64, w=32, P=16, act="bf16", kv="bf16",
                             source="input", keep=0.1, disable=True, seed=12),
    # sequences shorter than the window, and a single-token prompt
    "short_prompt": Case(B=2, T=20, steps=60, Hq=4, Hkv=2, D=64, w=32, P=16, act="bf16", kv="bf16", source="input",
                         keep=0.3, seed=13),
    "one_token_prompt": Case(B=1, T=1, steps=40, Hq=4, Hkv=2, D=128, w=32, P=16, act="bf16", kv="bf16",
                             source="input", keep=0.5, seed=14),
    # the staged API (append, then attention) on bf16 pages
    "bf16_proj_staged": Case(B=2, T=515, steps=24, Hq=8, Hkv=4, D=128, hidden=512, w=96, P=32, act="bf16",
                             kv="bf16", source="proj", keep=(1 / 16, 1 / 4), seed=3, staged=True),
    "bf16_d64_key_rope_staged": Case(B=2, T=400, steps=20, Hq=8, Hkv=2, D=64, w=64, P=32, act="bf16", kv="bf16",
                                     source="key", keep=0.2, rope=True, seed=16, staged=True),
    # fused decode over many heads (batch 8: decision logits inside the kernel)
    "bf16_b8_proj": Case(B=8, T=300, steps=40, Hq=16, Hkv=8, D=128, hidden=256, w=64, P=32, act="bf16", kv="bf16",
                         source="proj", keep=(1 / 16, 1 / 4), prealloc=96, seed=17),
    # heads long enough (>= 512 slots per rank of an 8-CTA cluster) that the
    # rank computing the decision logit also attends half a share
    "bf16_proj_long_heads": Case(B=1, T=4100, steps=12, Hq=8, Hkv=2, D=128, hidden=256, w=64, P=32, act="bf16",
                                 kv="bf16", source="proj", keep=0.95, attn_rows=64, seed=19),
    "fp8_proj_long_heads": Case(B=1, T=4100, steps=12, Hq=8, Hkv=2, D=128, hidden=256, w=64, P=32, act="bf16",
                                kv="fp8", source="proj", keep=0.95, attn_rows=64, seed=20),
    # 32 heads of D = 64 with 8 query heads each (two CTAs per SM), pages of 48
    # slots cut into 16-slot sub-tiles, key-major tiles
    "bf16_d64_b8_g8_p48": Case(B=8, T=280, steps=24, Hq=32, Hkv=4, D=64, w=64, P=48, act="bf16", kv="bf16",
                               source="input", keep=(1 / 16, 1 / 4), prealloc=96, seed=18),
    # a prompt large enough for the row-walking rotary kernel (batch x tokens x
    # 8-pair chunks above 148 x 256), 256-slot pages scattered by several CTAs
    # each, the last page ragged
    "bf16_key_rope_p256": Case(B=2, T=2500, steps=16, Hq=8, Hkv=2, D=128, w=320, P=256, act="bf16", kv="bf16",
                               source="key", keep=0.2, rope=True, attn_rows=128, seed=21),
    # fp32 pages of 256 slots: eight 32-row scatter groups per page, the last page ragged
    "f32_p256_scatter": Case(B=1, T=700, steps=10, Hq=4, Hkv=2, D=128, w=320, P=256, act="f32", kv="f32",
                             source="input", keep=0.3, attn_rows=64, seed=33),
    # GQA groups that are not a power of two: the prefill attention takes the
    # mma.sync kernel (the tcgen05 kernel tiles 128 / g positions x g heads)
    "bf16_g3_mma_prefill": Case(B=2, T=450, steps=12, Hq=12, Hkv=4, D=128, w=64, P=32, act="bf16", kv="bf16",
                                source="input", keep=0.3, seed=51),
    "bf16_g6_d64_proj_mma_prefill": Case(B=1, T=380, steps=10, Hq=12, Hkv=2, D=64, hidden=256, w=48, P=16,
                                         act="bf16", kv="bf16", source="proj", keep=0.25, seed=52),
    # decision shifts: +1 (token t marked by token t-1's decision) with the
    # adapter, -1 (token t's decision marks token t-1) on FP8 pages with the
    # key neuron and rotary tables, +1 on fp32 pages
    "bf16_shift_right_proj": Case(B=2, T=515, steps=24, Hq=8, Hkv=4, D=128, hidden=512, w=96, P=32, act="bf16",
                                  kv="bf16", source="proj", keep=(1 / 16, 1 / 4), shift=1, seed=71),
    "fp8_shift_left_key_rope": Case(B=2, T=700, steps=30, Hq=8, Hkv=2, D=64, w=64, P=32, act="bf16", kv="fp8",
                                    source="key", keep=0.125, rope=True, shift=-1, seed=72),
    "f32_shift_right_input": Case(B=1, T=256, steps=16, Hq=4, Hkv=2, D=64, w=32, P=16, act="f32", kv="f32",
                                  source="input", keep=0.5, shift=1, seed=73),
    "bf16_shift_left_layer_b8": Case(B=8, T=300, steps=40, Hq=16, Hkv=8, D=128, hidden=256, w=64, P=32,
                                     act="bf16", kv="bf16", source="proj", per="layer", keep=(1 / 16, 1 / 4),
                                     prealloc=96, shift=-1, seed=74),
    # the importance-score source (KVzap-style: Linear with a bias, no norm,
    # prune below a threshold, keep the last 128 tokens), bf16 and fp32
    "bf16_score_w128": Case(B=2, T=700, steps=20, Hq=32, Hkv=8, D=128, hidden=512, w=128, P=64, act="bf16",
                            kv="bf16", source="score", keep=0.25, seed=75),
    "f32_score_w128_layer": Case(B=1, T=400, steps=12, Hq=8, Hkv=4, D=64, hidden=256, w=128, P=32, act="f32",
                                 kv="f32", source="score", per="layer", keep=0.3, seed=76),
    "fp8_score_w128": Case(B=2, T=600, steps=16, Hq=16, Hkv=4, D=64, hidden=320, w=128, P=64, act="bf16",
                           kv="fp8", source="score", keep=0.2, seed=77),
    # second layer of a two-layer cache with preallocation
    "layer1_of_2": Case(B=2, T=260, steps=12, Hq=4, Hkv=2, D=64, w=32, P=16, act="bf16", kv="bf16",
                        source="input", keep=0.3, layers=2, layer=1, prealloc=64, seed=15),
}


@pytest.mark.parametrize("name", sorted(CASES))
def test_case_inputs_and_oracle(name):
    """CPU: the case's inputs build, its decision margins clear the bound, and
    the oracle's own invariants hold (retained count)."""
    case = CASES[name]
    ins = build(case)
    ev = marks(ins["evict"][:, :, :case.T], case.shift)
    T, w = case.T, case.w
    cnt = ins["state_prefill"]["count"]
    expect = min(T, w) + (1 - ev[:, :, : max(0, T - w)]).sum(-1)
    if case.per == "layer":
        expect = np.broadcast_to(expect[:, :1], expect.shape)
    assert np.array_equal(cnt, expect)


@pytest.mark.gpu
@pytest.mark.parametrize("kernel", ["cluster", "flat"])
@pytest.mark.parametrize("name", sorted(CASES))
def test_gpu_parity(name, kernel):
    """Every case through both decode attention kernels (one cluster per head;
    one CTA per SM over the flat slot list)."""
    case = dataclasses.replace(CASES[name], kernel=kernel)
    errs = check_case(case)
    print(name, kernel, errs)


@pytest.mark.gpu
def test_disable_eviction_is_vanilla_causal():
    """With eviction disabled the GPU output is plain causal attention (torch SDPA, fp64)."""
    case = CASES["disable_eviction"]
    ins = build(case)
    from harness import run_gpu
    res = run_gpu(case, ins)
    T = case.T
    q = torch.from_numpy(ins["q_stored"][:, :T]).permute(0, 2, 1, 3)
    k = torch.from_numpy(ins["k_stored"][:, :T]).permute(0, 2, 1, 3).repeat_interleave(case.Hq // case.Hkv, 1)
    v = torch.from_numpy(ins["v"][:, :T].double().numpy()).permute(0, 2, 1, 3).repeat_interleave(
        case.Hq // case.Hkv, 1)
    ref = torch.nn.functional.scaled_dot_product_attention(q, k, v, is_causal=True).permute(0, 2, 1, 3).numpy()
    assert np.max(np.abs(res["o_prefill"].double().numpy() - ref)) <= 2e-2
    assert res["state_final"]["count"].min().item() == case.N
