#!/usr/bin/env python
"""Benchmark of the DMS hot path on B200: decode tokens/s and retained-KV GB/s.

Decode steps are replayed from CUDA graphs captured once, one graph per step
holding the step's start/end timing events around its kernel(s), as the step
would run inside a whole-model graph.

One bench step = one pass of the whole path over one batch: cache reset,
prefill of the prompt (decision logits, compaction into pages, DMS-masked
attention), then every decode step (decision logit, append with delayed
eviction, split-K attention over the retained pages).  Workload: one Qwen3-8B
attention layer (hidden 4096, 32 q / 8 kv heads, head_dim 128), batch 1,
prompt 8192 + 128 decode steps, window 512, block 256, adapter decisions
calibrated to keep 1/8 of the tokens outside the window; synthetic seeded bf16
inputs resident in HBM.

L2: the decode working set (~6 MB) fits in the 126 MB L2, so a 512 MB buffer
is written before every decode step (outside the timed segments) and the KV
bytes come from DRAM.  Times are CUDA events on the launching stream.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
Multi-GPU (torchrun): every rank runs its own replica (independent sequences,
weak scaling, no collective on the data path); rank 0 prints one JSON line.
"""
import argparse
import json
import os
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

from learned_kv_cache_dms_b200 import inputs as I  # noqa: E402

WL = I.WORKLOADS["qwen8b"]
METRIC = "DMS decode tok/s and retained-KV HBM GB/s (% of B200 peak), Qwen3-8B shape"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def parse():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=5)
    p.add_argument("--warmup", type=int, default=3)
    p.add_argument("--impl", choices=["ours", "reference"], default="ours")
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--cpu-seconds", type=float, default=12.0)
    p.add_argument("--no-e2e", action="store_true", help="skip the host-buffer pass (profiler runs)")
    return p.parse_args()


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    return FALLBACK_PEAKS, "fallback"


# ---------------------------------------------------------------------------
# distributed plumbing
# ---------------------------------------------------------------------------
def dist_setup():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    elif torch.cuda.is_available():
        torch.cuda.set_device(0)
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def allreduce(x, op, world):
    if world == 1:
        return x
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device="cuda")
    dist.all_reduce(t, op=op)
    return float(t.item())


# ---------------------------------------------------------------------------
# clocks during the timed region
# ---------------------------------------------------------------------------
class ClockSampler:
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,clocks_event_reasons.hw_slowdown,"
         "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
         "clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.f = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
        self.idx = gpu_index
        self.p = None

    def __enter__(self):
        try:
            self.p = subprocess.Popen(["nvidia-smi", "-i", str(self.idx), "--query-gpu=" + self.Q,
                                       "--format=csv,noheader,nounits", "-lms", "200"], stdout=self.f,
                                      stderr=subprocess.DEVNULL)
        except OSError:
            self.p = None
        time.sleep(0.3)
        return self

    def __exit__(self, *a):
        if self.p is not None:
            self.p.terminate()
            try:
                self.p.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.p.kill()

    def summary(self):
        self.f.flush()
        self.f.seek(0)
        rows = [r.split(",") for r in self.f.read().strip().splitlines() if r.count(",") >= 8]
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"]}
        sm = [float(r[1]) for r in rows]
        smax = float(rows[0][2])
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].strip().lower() == "active"})
        loaded = [s for s in sm if s > 0.5 * smax] or sm
        return {"sm_mhz": float(np.median(loaded)), "sm_max_mhz": smax, "reasons": reasons, "samples": len(rows)}


# ---------------------------------------------------------------------------
# our implementation
# ---------------------------------------------------------------------------
def make_desc(B_, wl):
    d = B_.dms_cache_desc_default()
    d.num_layers, d.batch, d.num_q_heads, d.num_kv_heads = wl.layers, wl.batch, wl.q_heads, wl.kv_heads
    d.head_dim, d.hidden, d.window, d.block = wl.head_dim, wl.hidden, wl.window, wl.block
    d.max_positions, d.prealloc_tokens = wl.max_positions, wl.prealloc_tokens
    maxp = -(-wl.max_positions // wl.block)
    d.pool_pages = wl.layers * wl.batch * wl.kv_heads * maxp
    d.act_dtype = B_.DMS_BF16
    d.kv_dtype = B_.DMS_BF16
    return d


def gpu_inputs(wl, seed):
    g = torch.Generator(device="cuda")
    g.manual_seed(seed)
    B, T, S = wl.batch, wl.prompt, wl.decode_steps
    bf = torch.bfloat16

    def rn(*shape, std=1.0):
        return (torch.randn(*shape, generator=g, device="cuda", dtype=torch.float32) * std).to(bf)

    x = dict(q=rn(B, T, wl.q_heads, wl.head_dim), k=rn(B, T, wl.kv_heads, wl.head_dim),
             v=rn(B, T, wl.kv_heads, wl.head_dim), h=rn(B, T, wl.hidden),
             qd=rn(S, B, wl.q_heads, wl.head_dim), kd=rn(S, B, wl.kv_heads, wl.head_dim),
             vd=rn(S, B, wl.kv_heads, wl.head_dim), hd=rn(S, B, wl.hidden),
             gamma=rn(wl.hidden), W=rn(wl.kv_heads, wl.hidden, std=wl.hidden ** -0.5))
    return x


def calibrate(B_, cache, wl, x):
    """Offsets that keep a 1/8 fraction per head, from the library's own logits."""
    zero = torch.zeros(wl.batch, wl.kv_heads, dtype=torch.float32, device="cuda")
    raw = torch.empty(wl.batch, wl.kv_heads, wl.prompt, dtype=torch.float32, device="cuda")
    p = B_.decide_params(zero, hidden=x["h"], norm_weight=x["gamma"], proj_weight=x["W"])
    B_.dms_decide(cache.handle, wl.prompt, p, None, raw)
    s, _ = torch.sort(raw, dim=-1)
    k = int(round(wl.keep * wl.prompt))
    return (0.5 * (s[..., k - 1] + s[..., k])).contiguous()


class Runner:
    def __init__(self, B_, wl, seed):
        self.B_, self.wl = B_, wl
        self.cache = B_.Cache(make_desc(B_, wl))
        self.x = gpu_inputs(wl, seed)
        self.off = calibrate(B_, self.cache, wl, self.x)
        x, wl_ = self.x, wl
        self.o = torch.empty_like(x["q"])
        self.alpha = torch.empty(wl_.batch, wl_.kv_heads, wl_.prompt, dtype=torch.float32, device="cuda")
        self.od = torch.empty_like(x["qd"])
        self.ad = torch.empty(wl_.decode_steps, wl_.batch, wl_.kv_heads, dtype=torch.float32, device="cuda")
        self.pdec = B_.decide_params(self.off, hidden=x["h"], norm_weight=x["gamma"], proj_weight=x["W"])
        self.pargs = B_.Cache.prefill_args(x["q"], x["k"], x["v"], self.o, self.alpha, self.pdec)
        self.ddec = [B_.decide_params(self.off, hidden=x["hd"][s], norm_weight=x["gamma"], proj_weight=x["W"])
                     for s in range(wl_.decode_steps)]
        self.dargs = [B_.Cache.decode_args(x["qd"][s], x["kd"][s], x["vd"][s], self.od[s], self.ad[s], self.ddec[s])
                      for s in range(wl_.decode_steps)]
        self.flush = torch.empty(512 << 20, dtype=torch.uint8, device="cuda")
        self.graphs = None

    def capture(self):
        """CUDA graphs of each decode step's append and attention (the decode
        kernels read the token position from device memory, so a replay
        advances the cache exactly like an eager call)."""
        B_, h = self.B_, self.cache.handle
        self.cache.reset()
        B_.dms_prefill(h, 0, self.pargs)
        torch.cuda.synchronize()
        side = torch.cuda.Stream()
        gs = []
        for s in range(self.wl.decode_steps):
            ga = torch.cuda.CUDAGraph()
            ev = (torch.cuda.Event(enable_timing=True, external=True),
                  torch.cuda.Event(enable_timing=True, external=True))
            with torch.cuda.graph(ga, stream=side):
                ev[0].record()
                B_.dms_decode_step(h, 0, self.dargs[s])
                ev[1].record()
            gs.append((ga, ev))
        torch.cuda.synchronize()
        self.graphs = gs

    def step(self, ev=None, counts=None):
        """One bench step.  ev: list of event tuples filled per segment."""
        B_, h = self.B_, self.cache.handle
        self.cache.reset()
        self.flush.fill_(1)
        E = torch.cuda.Event
        e0, e1, e2 = E(enable_timing=True), E(enable_timing=True), E(enable_timing=True)
        e0.record()
        B_.dms_prefill_compact(h, 0, self.pargs)
        e1.record()
        B_.dms_prefill_attention(h, 0, self.pargs)
        e2.record()
        dec = []
        for s in range(self.wl.decode_steps):
            self.flush.fill_(s & 0xFF)
            if self.graphs is not None:
                # the step's graph records its own start/end events around the kernel
                self.graphs[s][0].replay()
            else:
                a, c = E(enable_timing=True), E(enable_timing=True)
                a.record()
                B_.dms_decode_step(h, 0, self.dargs[s])
                c.record()
                dec.append((a, c))
            if counts is not None:
                counts.append(self.cache.state(0)["count"].sum().item())
        if ev is not None:
            # graph events are re-recorded by the next replay: read them now
            torch.cuda.synchronize()
            dec_ms = sum(g[1][0].elapsed_time(g[1][1]) for g in self.graphs) if self.graphs else \
                sum(a.elapsed_time(c) for a, c in dec)
            ev.append(((e0, e1, e2), dec_ms))


def kernel_launches_per_step(wl):
    # reset (1) + compaction (decide, scan, scatter) + prefill attention (1)
    # + per decode step: one fused kernel (decision logit, attention, combine, append)
    return 1 + 3 + 1 + 1 * wl.decode_steps


def visible_pairs(alpha, wl):
    """Sum over (b, h, i) of |V_i| from the prefill decisions (alpha > 0 evicts)."""
    ev = (alpha > 0).cpu().numpy()  # [B,H,T]
    T, w = wl.prompt, wl.window
    keep = ~ev
    keep[:, :, max(0, T - w):] = False
    cum = np.concatenate([np.zeros(ev.shape[:2] + (1,), np.int64), np.cumsum(keep, -1)], -1)  # kept before t
    i = np.arange(T)
    band = np.minimum(i + 1, w)
    upto = np.clip(i - w + 1, 0, T)
    return int((band[None, None, :] + cum[:, :, upto]).sum())


def run_ours(args, world, rank, local):
    from learned_kv_cache_dms_b200 import binding as B_
    wl = WL
    pk, pk_kind = peaks()
    r = Runner(B_, wl, seed=WL.seed + rank)
    # untimed pass: retained counts after each append (identical in every step)
    counts = []
    r.cache.reset()
    B_.dms_prefill(r.cache.handle, 0, r.pargs)
    counts_prefill = r.cache.state(0)["count"].sum().item()
    r.step(counts=counts)
    torch.cuda.synchronize()
    assert r.cache.status() == 0
    pairs = visible_pairs(r.alpha, wl)
    o_eager = r.od.clone()
    r.capture()
    for _ in range(max(1, args.warmup - 1)):
        r.step()
    torch.cuda.synchronize()
    assert r.cache.status() == 0
    # the graph replays must reproduce the eager decode outputs exactly
    assert torch.equal(o_eager, r.od), "graph replay differs from the eager decode"

    barrier(world)
    torch.cuda.synchronize()
    evs = []
    with ClockSampler(local) as clk:
        t0 = torch.cuda.Event(enable_timing=True)
        t1 = torch.cuda.Event(enable_timing=True)
        t0.record()
        for _ in range(args.steps):
            r.step(ev=evs)
        t1.record()
        torch.cuda.synchronize()
    barrier(world)
    region_ms = t0.elapsed_time(t1)

    compact_ms = prefill_attn_ms = decode_ms = 0.0
    for (e0, e1, e2), dec_ms in evs:
        compact_ms += e0.elapsed_time(e1)
        prefill_attn_ms += e1.elapsed_time(e2)
        decode_ms += dec_ms
    K, S, B = args.steps, wl.decode_steps, wl.batch
    prefill_ms = compact_ms + prefill_attn_ms
    hot_ms_per_step = (decode_ms + prefill_ms) / K
    # max over ranks of the device times
    decode_ms_max = allreduce(decode_ms, _op("max"), world)
    prefill_ms_max = allreduce(prefill_ms, _op("max"), world)
    hot_max = allreduce(hot_ms_per_step, _op("max"), world)
    dec_tokens = K * S * B * world
    value = dec_tokens / (decode_ms_max / 1e3)
    prefill_tps = K * B * wl.prompt * world / (prefill_ms_max / 1e3)

    # algorithmic bytes of one fused decode step (one launch): the retained K/V
    # the attention reads (before the append, plus the new row), q and o, the
    # new K/V row written, the hidden row and W of the decision logits, and the
    # page-table entries
    D, elem = wl.head_dim, 2
    BH = B * wl.kv_heads
    per_step_fixed = (2 * B * wl.q_heads * D * elem            # q, o
                      + 2 * BH * D * elem                      # new K/V rows read
                      + 2 * BH * D * elem                      # new K/V rows written
                      + B * wl.hidden * elem + wl.kv_heads * wl.hidden * elem + wl.hidden * elem)  # h, W, gamma
    pre_counts = [counts_prefill] + counts[:-1]
    step_bytes = [cp * D * 2 * elem + (-(-cp // wl.block)) * 4 + per_step_fixed for cp in pre_counts]
    attn_bytes = sum(step_bytes)
    decode_gbs = K * attn_bytes / (decode_ms / 1e3) / 1e9
    attn_gbs = decode_gbs
    prefill_flops = 4.0 * D * wl.gqa * pairs
    prefill_tflops = K * prefill_flops / (prefill_attn_ms / 1e3) / 1e12
    clocks = clk.summary()

    e2e = None if args.no_e2e else run_e2e(B_, r, args, world)
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(wl, args.cpu_seconds)
    roof = {"bound": "hbm", "achieved": round(attn_gbs, 1), "peak": pk["hbm_gbs"], "unit": "GB/s",
            "frac": round(attn_gbs / pk["hbm_gbs"], 4), "traffic": None,
            "kernel": "fused decode step k_decode_attn<128,bf16,fused> (split-K attention, combine, append)",
            "algorithmic_bytes_per_launch": int(attn_bytes / S), "peak_source": pk_kind}
    line = {
        "metric": METRIC, "value": round(value, 1), "unit": "tokens/s", "n_gpus": world, "steps": K,
        "warmup": args.warmup, "ms_per_step": round(hot_max, 4), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": "qwen8b_layer_b1_ctx8192_dec128", "batch": B, "prompt": wl.prompt,
                   "decode_steps": S, "hidden": wl.hidden, "q_heads": wl.q_heads, "kv_heads": wl.kv_heads,
                   "head_dim": D, "window": wl.window, "block": wl.block, "keep": wl.keep,
                   "l2": "512 MB buffer written before every decode step (untimed)",
                   "parallelism": "dp%d replicas" % world},
        "retained_kv_gbps": round(decode_gbs, 1),
        "retained_kv_frac_of_peak": round(decode_gbs / pk["hbm_gbs"], 4),
        "decode_ms_per_token_step": round(decode_ms / (K * S), 5),
        "prefill_tok_s": round(prefill_tps, 1),
        "prefill_ms": round(prefill_ms / K, 4),
        "prefill_compact_ms": round(compact_ms / K, 4),
        "prefill_attention_ms": round(prefill_attn_ms / K, 4),
        "prefill_attention": {"bound": "tensor", "achieved": round(prefill_tflops, 2),
                              "peak": pk["bf16_tflops"], "unit": "TFLOP/s",
                              "frac": round(prefill_tflops / pk["bf16_tflops"], 4),
                              "flops_per_launch": prefill_flops, "visible_pairs": pairs},
        "achieved_cr": round(wl.max_positions / (counts[-1] / (B * wl.kv_heads)), 3),
        "region_ms_per_step_incl_l2_flush": round(region_ms / K, 3),
        "roofline": roof, "e2e": e2e, "gpu_launches": kernel_launches_per_step(wl) * K,
        "clocks": clocks, "cpu_baseline": cpu,
    }
    return line


def _op(name):
    import torch.distributed as dist
    return {"max": dist.ReduceOp.MAX, "sum": dist.ReduceOp.SUM}[name] if dist.is_initialized() else None


def run_e2e(B_, r, args, world):
    """Same workload through the public API with host (pinned) buffers: the
    prompt and every decode token are copied host->device and every output
    device->host inside the timed segments."""
    wl, x = r.wl, r.x
    host = {k: v.cpu().pin_memory() for k, v in x.items() if k in ("q", "k", "v", "h", "qd", "kd", "vd", "hd")}
    o_host = torch.empty(tuple(r.o.shape), dtype=r.o.dtype).pin_memory()
    od_host = torch.empty(tuple(r.od.shape), dtype=r.od.dtype).pin_memory()
    dev = {k: torch.empty_like(x[k]) for k in host}
    pdec = B_.decide_params(r.off, hidden=dev["h"], norm_weight=x["gamma"], proj_weight=x["W"])
    pargs = B_.Cache.prefill_args(dev["q"], dev["k"], dev["v"], r.o, r.alpha, pdec)
    ddec = [B_.decide_params(r.off, hidden=dev["hd"][s], norm_weight=x["gamma"], proj_weight=x["W"])
            for s in range(wl.decode_steps)]
    dargs = [B_.Cache.decode_args(dev["qd"][s], dev["kd"][s], dev["vd"][s], r.od[s], r.ad[s], ddec[s])
             for s in range(wl.decode_steps)]
    E = torch.cuda.Event
    dec_ms = 0.0
    h2d = d2h = 0
    for it in range(args.steps + 1):
        r.cache.reset()
        r.flush.fill_(3)
        e0, e1 = E(enable_timing=True), E(enable_timing=True)
        e0.record()
        for k in ("q", "k", "v", "h"):
            dev[k].copy_(host[k], non_blocking=True)
        B_.dms_prefill(r.cache.handle, 0, pargs)
        o_host.copy_(r.o, non_blocking=True)
        e1.record()
        evs = []
        for s in range(wl.decode_steps):
            r.flush.fill_(s & 0xFF)
            a, c = E(enable_timing=True), E(enable_timing=True)
            a.record()
            for k in ("qd", "kd", "vd", "hd"):
                dev[k][s].copy_(host[k][s], non_blocking=True)
            B_.dms_decode_step(r.cache.handle, 0, dargs[s])
            od_host[s].copy_(r.od[s], non_blocking=True)
            c.record()
            evs.append((a, c))
        torch.cuda.synchronize()
        if it == 0:
            continue  # warm-up
        dec_ms += sum(a.elapsed_time(c) for a, c in evs)
    bpe = 2
    h2d = (sum(host[k].numel() for k in ("q", "k", "v", "h")) + sum(host[k].numel() for k in ("qd", "kd", "vd", "hd"))) * bpe
    d2h = (o_host.numel() + od_host.numel()) * bpe
    dec_ms_max = allreduce(dec_ms, _op("max"), world)
    val = args.steps * wl.decode_steps * wl.batch * world / (dec_ms_max / 1e3)
    return {"value": round(val, 1), "unit": "tokens/s", "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h)}


# ---------------------------------------------------------------------------
# CPU oracle (baseline arm)
# ---------------------------------------------------------------------------
def oracle_decode_sample(wl, seconds, n_steps_max=None):
    """Time the oracle's decode steps (append + decode attention) on the host
    cores after an untimed prefill replay.  Returns (tok/s, cores, steps, secs)."""
    from oracle import oracle as O
    cores = O.set_threads(os.cpu_count() or 1)
    B, T, S = wl.batch, wl.prompt, wl.decode_steps
    s = wl.seed
    k = I.normal(s, (0, 2), (B, T + S, wl.kv_heads, wl.head_dim), "bf16").float().numpy()
    v = I.normal(s, (0, 3), (B, T + S, wl.kv_heads, wl.head_dim), "bf16").float().numpy()
    q = I.normal(s, (0, 1), (B, S, wl.q_heads, wl.head_dim), "bf16").double().numpy()
    alpha = I.synthetic_alpha(s, (0, 5), B, wl.kv_heads, T + S, wl.keep).numpy()
    ev = (alpha > 0).astype(np.uint8)
    maxp = -(-wl.max_positions // wl.block)
    c = O.Cache(1, B, wl.kv_heads, wl.head_dim, wl.window, wl.block, wl.max_positions,
                B * wl.kv_heads * maxp, wl.prealloc_tokens)
    c.prefill(0, np.ascontiguousarray(ev[:, :, :T]), np.ascontiguousarray(k[:, :T]), np.ascontiguousarray(v[:, :T]))
    n = 0
    t0 = time.perf_counter()
    limit = n_steps_max or S
    while n < limit and (time.perf_counter() - t0) < seconds:
        t = T + n
        c.append(0, np.ascontiguousarray(ev[:, :, t]), np.ascontiguousarray(k[:, t]), np.ascontiguousarray(v[:, t]))
        c.decode_attention(0, np.ascontiguousarray(q[:, n]))
        n += 1
    dt = time.perf_counter() - t0
    return n * B / dt, cores, n, dt


def cpu_baseline(wl, seconds):
    tps, cores, n, dt = oracle_decode_sample(wl, seconds)
    return {"value": round(tps, 2), "unit": "tokens/s", "cores": cores, "kind": "oracle",
            "sample": "first %d of %d decode steps (append + fp64 decode attention over the retained slots) after "
                      "an untimed prefill replay of the 8192-token prompt, %.1f s" % (n, wl.decode_steps, dt)}


def run_reference(args, world, rank):
    if rank != 0:
        return None
    wl = WL
    per_step = 4  # decode steps of the oracle per bench step (bounded sample)
    for _ in range(args.warmup):
        oracle_decode_sample(wl, 1e9, n_steps_max=1)
    tot_tok = tot_s = 0.0
    cores = 1
    for _ in range(args.steps):
        tps, cores, n, dt = oracle_decode_sample(wl, 1e9, n_steps_max=per_step)
        tot_tok += n * wl.batch
        tot_s += dt
    val = tot_tok / tot_s
    return {"impl": "reference", "metric": METRIC, "value": round(val, 2), "unit": "tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(1e3 * tot_s / args.steps, 3),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": "qwen8b_layer_b1_ctx8192_dec128", "batch": wl.batch, "prompt": wl.prompt,
                       "decode_steps": wl.decode_steps},
            "cpu_baseline": {"value": round(val, 2), "unit": "tokens/s", "cores": cores, "kind": "oracle",
                             "sample": "%d decode steps per bench step after an untimed prefill replay" % per_step},
            "e2e": {"value": round(val, 2), "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def main():
    args = parse()
    if args.impl == "reference":
        rank = int(os.environ.get("RANK", "0"))
        world = int(os.environ.get("WORLD_SIZE", "1"))
        line = run_reference(args, world, rank)
        if line is not None:
            print(json.dumps(line), flush=True)
        return
    world, rank, local = dist_setup()
    line = run_ours(args, world, rank, local)
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
