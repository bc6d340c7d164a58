"""GPU parity at the workloads' full sizes: the bench's shapes, decision
sources, page formats and decode-kernel choice, through the C ABI, against the
oracle.  Prefill attention is compared on sampled rows (the last position of
every sequence among them), every decode step's outputs in full, and the cache
state (counts, page tables, slot positions, ring) and the stored pages
(values, or FP8 codes and scales) bit for bit.

The 36-layer reasoning stack is sampled: its last layer, in a cache that holds
all 36, over the first 256 of its decode steps, with pages granted on demand
(the oracle's page pool would otherwise hold every layer's preallocation)."""
import pytest

from harness import Case, check_case

FULL = {
    # Qwen3-8B layer shape, batch 1, 8192 + 128, keep 1/8
    "qwen8b_b1": Case(B=1, T=8192, steps=128, Hq=32, Hkv=8, D=128, hidden=4096, w=512, P=256, act="bf16",
                      kv="bf16", source="proj", keep=1 / 8, prealloc=4096, attn_rows=256, seed=1002),
    # batch 8, per-(b, h) keep fractions in [1/16, 1/4]
    "qwen8b_b8": Case(B=8, T=8192, steps=128, Hq=32, Hkv=8, D=128, hidden=4096, w=512, P=256, act="bf16",
                      kv="bf16", source="proj", keep=(1 / 16, 1 / 4), prealloc=4096, attn_rows=256, seed=1003),
    # Llama-3.2-1B layer shape, FP8 pages, key-neuron decisions, rotary tables, 32768 + 256
    "llama1b_head": Case(B=4, T=32768, steps=256, Hq=32, Hkv=8, D=64, hidden=2048, w=512, P=256, act="bf16",
                         kv="fp8", source="key", keep=1 / 8, rope=True, prealloc=4096, attn_rows=256, seed=1004),
    "llama1b_layer": Case(B=4, T=32768, steps=256, Hq=32, Hkv=8, D=64, hidden=2048, w=512, P=256, act="bf16",
                          kv="fp8", source="key", per="layer", keep=1 / 8, rope=True, prealloc=4096,
                          attn_rows=256, seed=1014),
    # the importance-score source on the Llama-3.1-8B attention shape (the
    # KVzap-linear page: hidden 4096 -> 8 KV heads, threshold pruning outside
    # the last 128 tokens), 8192 + 64, keep 1/4
    "kvzap_llama8b_score": Case(B=1, T=8192, steps=64, Hq=32, Hkv=8, D=128, hidden=4096, w=128, P=64,
                                act="bf16", kv="bf16", source="score", keep=1 / 4, prealloc=2048, attn_rows=256,
                                seed=1006),
    # reasoning stack: batch 32, prompt 1024, keep 1/16, last of 36 layers
    "reason36_last_layer": Case(B=32, T=1024, steps=256, Hq=32, Hkv=8, D=128, hidden=4096, w=512, P=256,
                                act="bf16", kv="bf16", source="proj", keep=1 / 16, layers=36, layer=35,
                                prealloc=0, pool_pages=32 * 8 * 8, attn_rows=256, seed=1005),
}


@pytest.mark.gpu
@pytest.mark.parametrize("name", sorted(FULL))
def test_fullsize_parity(name):
    errs = check_case(FULL[name])
    print(name, errs)
