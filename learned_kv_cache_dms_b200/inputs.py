"""Seeded synthetic inputs for the DMS path.

This module is shared by the tests (oracle side and CUDA side) and by the
benchmark.  It draws random numbers and holds the workload shapes; it holds none
of the method's arithmetic (no decision logits, no masks, no cache rules).

Workloads (synthetic stand-ins for the pages' Qwen3-8B and Llama-3.2-1B runs;
no model weights or datasets are used):

  tiny     fp32, B1, hidden 256, 4 q heads / 2 kv heads, D64, prompt 256 + 16
           decode steps, window 32, block 16, keep 1/2 per head.
  qwen8b   bf16, B1, hidden 4096, 32/8, D128, prompt 8192 + 128 steps, w512,
           block 256, keep 1/8 per head.
  qwen8b_c8  as qwen8b with batch 8; per-(sequence, head) keep ~ U[1/16, 1/4];
           4096 tokens preallocated per head.
  llama1b  bf16 activations, FP8 E4M3 KV pages, B4, hidden 2048, 32/8, D64,
           prompt 32768 + 256 steps, w512, block 256, keep 1/8, alpha from the
           last key neuron, rotary tables; run per head and per layer.
  reason36 bf16, 36 independent layers, B32, prompt 1024 + 16384 steps, w512,
           block 256, keep 1/16, decisions online every step.
  kvzap8b  bf16, Llama-3.1-8B attention shape, B1, prompt 8192 + 128 steps,
           importance-score decisions (Linear, no norm, threshold), w128,
           block 64, keep 1/4.
"""
from __future__ import annotations

import dataclasses
import math

import numpy as np
import torch


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    layers: int
    batch: int
    hidden: int
    q_heads: int
    kv_heads: int
    head_dim: int
    prompt: int
    decode_steps: int
    window: int
    block: int
    act_dtype: str          # "f32" | "bf16"
    kv_dtype: str           # "f32" | "bf16" | "fp8"
    keep: float             # mean keep fraction outside the window
    keep_range: tuple | None = None   # per-(b,h) keep ~ U[lo, hi]
    alpha_source: str = "proj"        # "proj" | "key" | "query" | "score"
    alpha_per: str = "head"           # "head" | "layer"
    rope: bool = False
    prealloc_tokens: int = 4096
    seed: int = 1000

    @property
    def gqa(self) -> int:
        return self.q_heads // self.kv_heads

    @property
    def max_positions(self) -> int:
        return self.prompt + self.decode_steps


WORKLOADS = {
    "tiny": Workload("tiny", 1, 1, 256, 4, 2, 64, 256, 16, 32, 16, "f32", "f32", 0.5,
                     prealloc_tokens=0, seed=1001),
    "qwen8b": Workload("qwen8b", 1, 1, 4096, 32, 8, 128, 8192, 128, 512, 256, "bf16", "bf16",
                       1 / 8, seed=1002),
    "qwen8b_c8": Workload("qwen8b_c8", 1, 8, 4096, 32, 8, 128, 8192, 128, 512, 256, "bf16", "bf16",
                          5 / 32, keep_range=(1 / 16, 1 / 4), seed=1003),
    "llama1b": Workload("llama1b", 1, 4, 2048, 32, 8, 64, 32768, 256, 512, 256, "bf16", "fp8",
                        1 / 8, alpha_source="key", rope=True, seed=1004),
    "llama1b_layer": Workload("llama1b_layer", 1, 4, 2048, 32, 8, 64, 32768, 256, 512, 256, "bf16",
                              "fp8", 1 / 8, alpha_source="key", alpha_per="layer", rope=True,
                              seed=1004),
    "reason36": Workload("reason36", 36, 32, 4096, 32, 8, 128, 1024, 16384, 512, 256, "bf16", "bf16",
                         1 / 16, seed=1005),
    # the importance-score source on the Llama-3.1-8B attention shape (the
    # KVzap-linear page: hidden 4096 -> 8 KV-head scores, threshold pruning
    # outside the last 128 tokens), batch 1, 8192 + 128, keep 1/4
    "kvzap8b": Workload("kvzap8b", 1, 1, 4096, 32, 8, 128, 8192, 128, 128, 64, "bf16", "bf16", 1 / 4,
                        alpha_source="score", seed=1006),
}

TORCH_DTYPES = {"f32": torch.float32, "bf16": torch.bfloat16}


def _gen(seed: int, *key: int) -> torch.Generator:
    # One independent stream per (seed, key...) tuple.
    h = seed & 0xFFFFFFFF
    for k in key:
        h = (h * 1000003 + (k & 0xFFFFFFFF) + 0x9E3779B9) & 0xFFFFFFFFFFFF
    g = torch.Generator(device="cpu")
    g.manual_seed(h)
    return g


def normal(seed: int, key: tuple, shape, dtype: str = "f32", std: float = 1.0) -> torch.Tensor:
    """N(0, std^2) samples on the CPU, rounded once to `dtype`."""
    x = torch.randn(*shape, generator=_gen(seed, *key), dtype=torch.float64) * std
    return x.to(TORCH_DTYPES[dtype])


def uniform(seed: int, key: tuple, shape, lo: float = 0.0, hi: float = 1.0) -> torch.Tensor:
    x = torch.rand(*shape, generator=_gen(seed, *key), dtype=torch.float64)
    return x * (hi - lo) + lo


def keep_fractions(wl: Workload, seed: int | None = None) -> np.ndarray:
    """Per-(b, h) keep fraction: constant, or ~U[lo, hi] when keep_range is set."""
    seed = wl.seed if seed is None else seed
    if wl.keep_range is None:
        return np.full((wl.batch, wl.kv_heads), wl.keep, np.float64)
    lo, hi = wl.keep_range
    return uniform(seed, (77,), (wl.batch, wl.kv_heads), lo, hi).numpy()


def synthetic_alpha(seed: int, key: tuple, B: int, H: int, T: int, keep, margin: float = 1.0,
                    spread: float = 8.0) -> torch.Tensor:
    """Decision logits given directly: alpha <= -margin with probability `keep`
    (per (b, h) if `keep` is an array), else alpha >= +margin.  fp32 [B, H, T]."""
    keep = np.broadcast_to(np.asarray(keep, np.float64), (B, H))
    u = uniform(seed, key + (1,), (B, H, T)).numpy()
    mag = margin + spread * uniform(seed, key + (2,), (B, H, T)).numpy()
    sign = np.where(u < keep[:, :, None], -1.0, 1.0)
    return torch.from_numpy((sign * mag).astype(np.float32))


def calibrate_offsets(raw_logits: np.ndarray, keep) -> tuple[np.ndarray, float]:
    """Offsets [B, H] that keep a `keep` fraction of tokens per (b, h).

    raw_logits[B, H, T] are the logits computed with a zero offset; a token is
    kept when raw <= offset.  The offset sits in the middle of the widest gap
    between consecutive sorted raw logits within +-1% of rank k = keep * T, so
    every decision has a margin that floating-point rounding cannot cross; the
    smallest margin is returned too.
    """
    raw = np.asarray(raw_logits, np.float64)
    B, H, T = raw.shape
    keep = np.broadcast_to(np.asarray(keep, np.float64), (B, H))
    off = np.empty((B, H), np.float64)
    margin = math.inf
    win = max(1, T // 100)
    for b in range(B):
        for h in range(H):
            s = np.sort(raw[b, h])
            k = int(round(keep[b, h] * T))
            if k <= 0:
                o = s[0] - 1.0
            elif k >= T:
                o = s[-1] + 1.0
            else:
                lo, hi = max(1, k - win), min(T - 1, k + win)
                j = lo + int(np.argmax(s[lo:hi + 1] - s[lo - 1:hi]))
                o = 0.5 * (s[j - 1] + s[j])
            off[b, h] = o
            margin = min(margin, float(np.min(np.abs(raw[b, h] - o))))
    return off.astype(np.float32), margin


def rope_tables(max_pos: int, head_dim: int, theta: float = 500000.0) -> tuple[torch.Tensor, torch.Tensor]:
    """cos/sin tables [max_pos, head_dim/2] in fp32 for angle pos * theta^(-2i/D)."""
    half = head_dim // 2
    inv = theta ** (-np.arange(half, dtype=np.float64) * 2.0 / head_dim)
    ang = np.arange(max_pos, dtype=np.float64)[:, None] * inv[None, :]
    return (torch.from_numpy(np.cos(ang).astype(np.float32)),
            torch.from_numpy(np.sin(ang).astype(np.float32)))


def layer_inputs(wl: Workload, layer: int, T: int, pos0: int = 0, seed: int | None = None,
                 batch: int | None = None):
    """q[B,T,Hq,D], k/v[B,T,Hkv,D], h[B,T,hidden] for a block of T tokens.

    The stream is keyed by (layer, pos0): a decode step at position p draws
    with T=1, pos0=p, independently of the prompt block drawn at pos0=0.
    """
    seed = wl.seed if seed is None else seed
    B = wl.batch if batch is None else batch
    d = wl.act_dtype
    q = normal(seed, (layer, pos0, 1), (B, T, wl.q_heads, wl.head_dim), d)
    k = normal(seed, (layer, pos0, 2), (B, T, wl.kv_heads, wl.head_dim), d)
    v = normal(seed, (layer, pos0, 3), (B, T, wl.kv_heads, wl.head_dim), d)
    h = normal(seed, (layer, pos0, 4), (B, T, wl.hidden), d)
    return q, k, v, h


def decide_weights(wl: Workload, layer: int, seed: int | None = None):
    """RMSNorm weight gamma[hidden] and Linear W[Hkv, hidden], N(0,1)/sqrt(hidden)."""
    seed = wl.seed if seed is None else seed
    s = 1.0 / math.sqrt(wl.hidden)
    gamma = normal(seed, (layer, 10), (wl.hidden,), wl.act_dtype, std=1.0)
    W = normal(seed, (layer, 11), (wl.kv_heads, wl.hidden), wl.act_dtype, std=s)
    return gamma, W
