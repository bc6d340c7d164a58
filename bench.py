#!/usr/bin/env python
"""Benchmark of the DMS hot path on B200: decode tokens/s and retained-KV GB/s.

Decode steps are replayed from CUDA graphs captured once, one graph per step
holding the step's start/end timing events around its kernel(s), as the step
would run inside a whole-model graph.

One bench step = one pass of the whole path over one batch: cache reset,
prefill of the prompt (decision logits, compaction into pages, DMS-masked
attention) in every layer, then every decode step (decision logit, append with
delayed eviction, split-K attention over the retained pages) through the
layer stack.  Default workload: one Qwen3-8B attention layer (hidden 4096,
32 q / 8 kv heads, head_dim 128), batch 1, prompt 8192 + 128 decode steps,
window 512, block 256, adapter decisions calibrated to keep 1/8 of the tokens
outside the window; synthetic seeded bf16 inputs resident in HBM.  --workload
selects the batch-8 Qwen3-8B layer, the FP8 Llama-3.2-1B layer (32K context,
key-neuron decisions, rotary tables) or the 36-layer batch-32 stack.

L2: a single layer's decode working set (6-60 MB) fits in the 126 MB L2, so
each decode step runs R independent replicas of the cache back to back (R
chosen so that together they hold >= 4x L2): no replica's KV is still in L2
when it is read again, and no flush kernel sits between decode kernels.  The
36-layer stack reads gigabytes per step and runs its steps back to back.
Times are CUDA events on the launching stream.

The JSON line also carries: `e2e` (the whole request -- prompt copies,
prefill, every decode step with its host copies -- through the public API with
host buffers), `decode_step_us_single` (one replica's step, L2 flushed before
it), the prefill attention's fraction on executed tiles, the decision and
compaction kernels on their own, `cpu_baseline` (the oracle on the host cores:
decode on all cores and on one core, and a prefill sample), and `secondary`
records for the other workloads (batch 8, the FP8 Llama-3.2-1B layer, the
first 512 steps of the 36-layer stack).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                  [--workload NAME] [--decode-steps N]
Multi-GPU (torchrun): every rank runs its own replica (independent sequences,
weak scaling, no collective on the data path); rank 0 prints one JSON line.
"""
import argparse
import dataclasses
import hashlib
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
    p.add_argument("--measure", choices=["train_attention", "chunked_prefill"], default=None,
                   help="run one of the extra measurements alone and print its record (profiler captures)")
    p.add_argument("--no-secondary", action="store_true",
                   help="measure only --workload (the default run also measures the other workloads)")
    p.add_argument("--workload", choices=BENCH_WORKLOADS, default="qwen8b",
                   help="qwen8b (default): one Qwen3-8B layer, batch 1; qwen8b_c8: batch 8; llama1b(_layer): "
                        "FP8 pages, key-neuron decisions, 32K context; reason36: 36 layers, batch 32")
    p.add_argument("--decode-steps", type=int, default=None, help="decode only the first N steps")
    p.add_argument("--decode-kernel", choices=["auto", "cluster", "flat"], default="auto",
                   help="decode attention kernel (auto: by the number of heads)")
    p.add_argument("--decode-api", choices=["auto", "step", "layers"], default="auto",
                   help="multi-layer stacks: one dms_decode_step_layers launch per step (auto, layers) or one "
                        "dms_decode_step per layer (step)")
    p.add_argument("--replicas", type=int, default=None,
                   help="cache replicas per step (default: enough that each step's KV is >= 4x L2; 1 gives a "
                        "small case for profiler captures, whose numbers are then not L2-cold)")
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
    """One process per GPU (NCCL; rendezvous from the torchrun environment).
    Without a GPU (host-logic tests) the group is gloo over CPU tensors."""
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        if torch.cuda.is_available():
            torch.cuda.set_device(local)
            dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                    device_id=torch.device("cuda", local))
        else:
            dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=120))
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
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
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
BENCH_WORKLOADS = ("qwen8b", "qwen8b_c8", "llama1b", "llama1b_layer", "reason36", "kvzap8b")
STEP_POOL = 64  # distinct decode-token inputs per layer of a multi-layer stack (cycled)


def workload_label(wl, n_dec):
    if wl.name == "qwen8b" and n_dec == wl.decode_steps:
        return "qwen8b_layer_b1_ctx8192_dec128"
    return "%s_L%d_b%d_ctx%d_dec%d_%s" % (wl.name, wl.layers, wl.batch, wl.prompt, n_dec, wl.kv_dtype)


def make_desc(B_, wl, kernel="auto"):
    d = B_.dms_cache_desc_default()
    d.decode_kernel = {"auto": B_.DMS_DECODE_AUTO, "cluster": B_.DMS_DECODE_CLUSTER,
                       "flat": B_.DMS_DECODE_FLAT}[kernel]
    d.num_layers, d.batch, d.num_q_heads, d.num_kv_heads = wl.layers, wl.batch, wl.q_heads, wl.kv_heads
    d.head_dim, d.hidden, d.window, d.block = wl.head_dim, wl.hidden, wl.window, wl.block
    d.max_positions, d.prealloc_tokens = wl.max_positions, wl.prealloc_tokens
    maxp = -(-wl.max_positions // wl.block)
    pre = min(maxp, -(-wl.prealloc_tokens // wl.block))
    # pages one head can need: the window, the kept tokens at the largest keep
    # fraction with 25% slack, one partly filled page
    hi = wl.keep_range[1] if wl.keep_range else wl.keep
    need = -(-int(wl.window + 1.25 * hi * wl.max_positions + wl.block) // wl.block)
    d.pool_pages = wl.layers * wl.batch * wl.kv_heads * min(maxp, max(pre, need))
    d.act_dtype = B_.DMS_BF16
    d.kv_dtype = {"bf16": B_.DMS_BF16, "fp8": B_.DMS_FP8_E4M3}[wl.kv_dtype]
    d.alpha_source = {"proj": B_.DMS_ALPHA_PROJ, "key": B_.DMS_ALPHA_KEY_NEURON,
                      "score": B_.DMS_ALPHA_SCORE_LINEAR}[wl.alpha_source]
    d.alpha_per = B_.DMS_ALPHA_PER_LAYER if wl.alpha_per == "layer" else B_.DMS_ALPHA_PER_HEAD
    return d


def decode_launches_per_step(wl):
    """Kernels one dms_decode_step launches per layer: the decision neuron /
    rotary pass where needed, then one fused kernel (decision logit,
    attention, combine, append; FP8 pages appended first inside it)."""
    pre = 1 if (wl.alpha_source not in ("proj", "score") or wl.rope) else 0
    return pre + 1


def prefill_launches_per_layer(wl):
    """Kernels one dms_prefill launches: the adapter / score logits or the
    decision neuron and rotary pass, the two scan kernels, the scatter and the
    masked attention."""
    decide = 1 if wl.alpha_source in ("proj", "score") else 0
    rope = 1 if (wl.alpha_source not in ("proj", "score") or wl.rope) else 0
    return decide + rope + 2 + 1 + 1


def kernel_launches_per_step(wl, n_dec, stacked=False):
    # reset (1) + per layer the prefill + the decode steps (with
    # dms_decode_step_layers: each layer's rotary pass where needed, then one
    # launch for the whole stack)
    pre = decode_launches_per_step(wl) - 1
    per_step = wl.layers * pre + 1 if stacked else wl.layers * decode_launches_per_step(wl)
    return 1 + wl.layers * prefill_launches_per_layer(wl) + n_dec * per_step


def decode_label(wl, kern, stacked, layers):
    """What the decode roofline's time covers, for the JSON line."""
    parts = ["split-K attention",
             "on-chip combine" if kern == "k_decode_cluster" else "partials merged by the last CTA of a head"]
    fp8_inside = wl.kv_dtype == "fp8" and kern == "k_decode_cluster"
    if wl.kv_dtype == "bf16" or fp8_inside:
        parts.append("append" + (" first (page re-encode), then the attention" if fp8_inside else ""))
    if wl.alpha_source in ("proj", "score"):
        parts.append("decision logit")
    label = "decode step: %s<%d,%s> (%s)%s%s" % (
        kern, wl.head_dim, wl.kv_dtype, ", ".join(parts),
        " after k_decode_append" if wl.kv_dtype == "fp8" and not fp8_inside else "",
        "; the step's time includes the decision-neuron / rotary pass before it"
        if decode_launches_per_step(wl) > 1 else "")
    if stacked:
        label += ", all %d layers in one launch (dms_decode_step_layers)" % layers
    return label


def decode_kernel_name(wl, choice, num_sms):
    """The decode kernel the library runs for this workload (its AUTO rule:
    the cluster kernel)."""
    if choice == "auto":
        choice = "cluster"
    return "k_decode_" + choice


# Sources of each kernel whose DRAM traffic is recorded in profiles/traffic.txt
TRAFFIC_SOURCES = {
    "k_decode_cluster": ["k_decode_cluster.cu", "decode_common.cuh"],
    "k_decode_flat": ["k_decode_flat.cu", "decode_common.cuh"],
    "k_attn_prefill_tc": ["k_attn_prefill_tc.cu"],
}


def source_digest(kernel):
    h = hashlib.sha256()
    for f in TRAFFIC_SOURCES[kernel]:
        with open(os.path.join(ROOT, "learned_kv_cache_dms_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def recorded_traffic(kernel, workload):
    """DRAM bytes (read + write) per launch of `kernel` on `workload` from the
    ncu capture summarised in profiles/, or None when there is none or the
    kernel's sources changed since it was taken."""
    path = os.path.join(ROOT, "profiles", "traffic.txt")
    if kernel not in TRAFFIC_SOURCES or not os.path.exists(path):
        return None
    digest = source_digest(kernel)
    with open(path) as f:
        for line in f:
            fields = line.split()
            if len(fields) >= 4 and not line.startswith("#") and fields[0] == kernel and fields[1] == workload:
                return int(fields[2]) if fields[3] == digest else None
    return None


def replicas_for(wl, l2_bytes):
    """Independent cache replicas whose decode steps run back to back so that
    each step's KV is evicted from L2 before it is read again: together they
    hold at least 4x L2.  A multi-layer stack is its own rotation."""
    if wl.layers > 1:
        return 1
    keep = sum(wl.keep_range) / 2 if wl.keep_range else wl.keep
    retained = min(wl.prompt, wl.window) + keep * max(0, wl.prompt - wl.window)
    elem = 1 if wl.kv_dtype == "fp8" else 2
    per_step = wl.batch * wl.kv_heads * retained * wl.head_dim * 2 * elem
    return int(min(128, max(1, -(-4 * l2_bytes // per_step))))


class Runner:
    """One workload on one GPU: seeded inputs in HBM, R replicas of its cache
    (each holding every layer), and the decode steps captured as CUDA graphs
    that run every (replica, layer) back to back."""

    def __init__(self, B_, wl, seed, n_dec=None, kernel="auto", replicas=None, api="auto"):
        self.B_, self.wl = B_, wl
        self.S = n_dec or wl.decode_steps
        self.L = wl.layers
        # a single layer draws every decode token; a deep stack cycles a pool
        self.pool = self.S if self.L == 1 else min(self.S, STEP_POOL)
        self.desc = make_desc(B_, wl, kernel)
        l2 = torch.cuda.get_device_properties(0).L2_cache_size
        self.R = replicas or replicas_for(wl, l2)
        self.caches = [B_.Cache(self.desc) for _ in range(self.R)]
        self.cache = self.caches[0]
        self.neuron = wl.alpha_source not in ("proj", "score")
        self.score = wl.alpha_source == "score"
        # the compaction and the decode step rewrite q and k in place (neuron
        # zeroing, rotary): such inputs get a copy per replica, restored from
        # pristine copies outside the timed segments
        self.inplace = self.neuron or wl.rope
        if self.inplace and self.L > 1:
            raise NotImplementedError("in-place inputs on a multi-layer stack")
        self.rope = None
        if wl.rope:
            cos, sin = I.rope_tables(wl.max_positions, wl.head_dim)
            self.rope = (cos.cuda(), sin.cuda())
        B, T, Hq, D = wl.batch, wl.prompt, wl.q_heads, wl.head_dim
        # prefill outputs are not read back: one buffer serves every unit
        self.o = torch.empty(B, T, Hq, D, dtype=torch.bfloat16, device="cuda")
        self.lay = [self._layer(l, seed) for l in range(self.L)]
        # units of decode work: (replica, layer) with their own token outputs
        self.units = [self._unit(r, l) for r in range(self.R) for l in range(self.L)]
        self.od = self.units[0]["od"]
        self.graphs = None
        self.cycled = self.pool < self.S
        # a stack of bf16 layers decodes all its layers in one launch
        # (dms_decode_step_layers) unless asked otherwise
        self.stacked = (api in ("auto", "layers") and self.L > 1 and wl.kv_dtype == "bf16" and not self.inplace)
        if self.stacked:
            self._stack_inputs()

    def _stack_inputs(self):
        """Decode inputs of every layer stacked layer by layer ([pool, L, B, ...])
        and one dms_decode_step_layers argument set per (replica, token)."""
        B_, wl, P = self.B_, self.wl, self.pool
        st = {k_: torch.stack([x[k_] for x in self.lay], 1).contiguous() for k_ in ("qd", "kd", "vd")}
        proj = not self.neuron
        if proj:
            st["hd"] = torch.stack([x["hd"] for x in self.lay], 1).contiguous()
            st["gamma"] = torch.stack([x["gamma"] for x in self.lay]).contiguous()
            st["W"] = torch.stack([x["W"] for x in self.lay]).contiguous()
            st["off"] = torch.stack([x["off"] for x in self.lay]).contiguous()  # [L, B, Hkv]
        self.st = st
        self.sargs = []
        for r in range(self.R):
            ad = torch.empty(P, self.L, wl.batch, wl.kv_heads, dtype=torch.float32, device="cuda")
            od = torch.empty_like(st["qd"])
            args, keep = [], []
            for i in range(P):
                dp = None
                if proj:
                    dp = B_.decide_params(st["off"][0], hidden=st["hd"][i], norm_weight=st["gamma"], proj_weight=st["W"])
                    dp.offset = st["off"].data_ptr()
                    keep.append(dp)
                args.append(B_.Cache.decode_args(st["qd"][i], st["kd"][i], st["vd"][i], od[i], ad[i], dp))
            self.sargs.append(dict(h=self.caches[r].handle, args=args, ad=ad, od=od, keep=keep))
        self.od = self.sargs[0]["od"][:, 0]

    def decode_replica(self, r, i):
        """Decode step i of replica r: every layer."""
        if self.stacked:
            sa = self.sargs[r]
            self.B_.dms_decode_step_layers(sa["h"], 0, self.L, sa["args"][i])
        else:
            for u in self.units[r * self.L:(r + 1) * self.L]:
                self.B_.dms_decode_step(u["h"], u["l"], u["dargs"][i])

    def decode_all(self, i):
        for r in range(self.R):
            self.decode_replica(r, i)

    def _layer(self, l, seed):
        B_, wl = self.B_, self.wl
        g = torch.Generator(device="cuda")
        g.manual_seed(seed * 4099 + l)
        bf = torch.bfloat16
        B, T, P, Hq, H, D = wl.batch, wl.prompt, self.pool, wl.q_heads, wl.kv_heads, wl.head_dim

        def rn(*shape, std=1.0):
            return (torch.randn(*shape, generator=g, device="cuda", dtype=torch.float32) * std).to(bf)

        x = dict(q=rn(B, T, Hq, D), k=rn(B, T, H, D), v=rn(B, T, H, D),
                 qd=rn(P, B, Hq, D), kd=rn(P, B, H, D), vd=rn(P, B, H, D))
        if not self.neuron:
            x.update(h=rn(B, T, wl.hidden), hd=rn(P, B, wl.hidden), gamma=None if self.score else rn(wl.hidden),
                     W=rn(H, wl.hidden, std=wl.hidden ** -0.5))
        # offsets that keep the workload's fraction of tokens per (b, h)
        keep = I.keep_fractions(wl, seed)
        if self.neuron:
            raw = (x["k"][..., -1].float() * self.desc.alpha_scale).permute(0, 2, 1)
        else:
            zero = torch.zeros(B, H, dtype=torch.float32, device="cuda")
            raw = torch.empty(B, H, T, dtype=torch.float32, device="cuda")
            p = B_.decide_params(zero, hidden=x["h"], norm_weight=x["gamma"], proj_weight=x["W"])
            B_.dms_decide(self.cache.handle, T, p, None, raw)
        raw = raw.cpu().numpy()
        if wl.alpha_per == "layer":  # every head follows head 0's logit
            raw = np.broadcast_to(raw[:, :1], raw.shape)
            keep = np.broadcast_to(keep[:, :1], keep.shape)
        off, _ = I.calibrate_offsets(raw, keep)
        # the score source marks a token when threshold - score > 0: with a
        # zero threshold the logit is -score, so the threshold is -offset
        x["off"] = torch.from_numpy(-off if self.score else off).cuda()
        if self.neuron:
            x["pdec"] = B_.decide_params(x["off"])
            x["ddec"] = [x["pdec"]] * P
        else:
            x["pdec"] = B_.decide_params(x["off"], hidden=x["h"], norm_weight=x["gamma"], proj_weight=x["W"])
            x["ddec"] = [B_.decide_params(x["off"], hidden=x["hd"][i], norm_weight=x["gamma"], proj_weight=x["W"])
                         for i in range(P)]
        return x

    def _unit(self, r, l):
        B_, wl, x = self.B_, self.wl, self.lay[l]
        B, T, P, H = wl.batch, wl.prompt, self.pool, wl.kv_heads
        u = dict(r=r, l=l, h=self.caches[r].handle)
        for k_ in ("q", "k", "qd", "kd"):
            # inputs rewritten in place: a working copy per replica
            u[k_] = x[k_].clone() if self.inplace else x[k_]
            u[k_ + "0"] = x[k_]
        u["alpha"] = torch.empty(B, H, T, dtype=torch.float32, device="cuda")
        u["ad"] = torch.empty(P, B, H, dtype=torch.float32, device="cuda")
        u["od"] = torch.empty_like(x["qd"])
        u["pargs"] = B_.Cache.prefill_args(u["q"], u["k"], x["v"], self.o, u["alpha"], x["pdec"], self.rope)
        u["dargs"] = [B_.Cache.decode_args(u["qd"][i], u["kd"][i], x["vd"][i], u["od"][i], u["ad"][i],
                                           x["ddec"][i], self.rope) for i in range(P)]
        return u

    # restores of inputs the library rewrites in place (outside the timed segments)
    def restore_prompt(self):
        if self.inplace:
            for u in self.units:
                u["q"].copy_(u["q0"])
                u["k"].copy_(u["k0"])

    def restore_token(self, i):
        if self.inplace:
            for u in self.units:
                u["qd"][i].copy_(u["qd0"][i])
                u["kd"][i].copy_(u["kd0"][i])

    def reset_all(self):
        for cch in self.caches:
            cch.reset()

    def prefill_all(self):
        for u in self.units:
            self.B_.dms_prefill(u["h"], u["l"], u["pargs"])

    def capture(self):
        """CUDA graphs of the decode steps, one per distinct token input, each
        running every (replica, layer) back to back between the step's
        start/end events (the decode kernels read the token position from
        device memory, so a replay advances the caches exactly like eager
        calls)."""
        B_ = self.B_
        self.reset_all()
        self.restore_prompt()
        self.prefill_all()
        torch.cuda.synchronize()
        side = torch.cuda.Stream()
        gs = []
        for i in range(self.pool):
            self.restore_token(i)
            torch.cuda.synchronize()
            ga = torch.cuda.CUDAGraph()
            ev = (torch.cuda.Event(enable_timing=True, external=True),
                  torch.cuda.Event(enable_timing=True, external=True))
            with torch.cuda.graph(ga, stream=side):
                ev[0].record()
                self.decode_all(i)
                ev[1].record()
            gs.append((ga, ev))
        torch.cuda.synchronize()
        self.graphs = gs

    def step(self, ev=None, counts=None):
        """One bench step: reset, prefill of every unit, every decode step.
        ev: list that receives (prefill segments, decode ms) of this step."""
        B_ = self.B_
        E = torch.cuda.Event
        self.reset_all()
        self.restore_prompt()
        seg = []
        for u in self.units:
            e0, e1, e2 = E(enable_timing=True), E(enable_timing=True), E(enable_timing=True)
            e0.record()
            B_.dms_prefill_compact(u["h"], u["l"], u["pargs"])
            e1.record()
            B_.dms_prefill_attention(u["h"], u["l"], u["pargs"])
            e2.record()
            seg.append((e0, e1, e2))
        if counts is not None:
            counts.append(self.cache.counts().sum(dtype=torch.int64))
        dec = []
        d0, d1 = E(enable_timing=True), E(enable_timing=True)
        d0.record()
        for s in range(self.S):
            i = s % self.pool
            self.restore_token(i)
            if self.graphs is not None:
                self.graphs[i][0].replay()
            else:
                a, c = E(enable_timing=True), E(enable_timing=True)
                a.record()
                self.decode_all(i)
                c.record()
                dec.append((a, c))
            if counts is not None:
                counts.append(self.cache.counts().sum(dtype=torch.int64))
        d1.record()
        if ev is not None:
            torch.cuda.synchronize()
            if self.cycled:
                # steps run back to back: the stack's working set is many times L2
                dec_ms = d0.elapsed_time(d1)
            elif self.graphs is not None:
                dec_ms = sum(g[1][0].elapsed_time(g[1][1]) for g in self.graphs)
            else:
                dec_ms = sum(a.elapsed_time(c) for a, c in dec)
            ev.append((seg, dec_ms))


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


def executed_tile_flops(alpha, wl):
    """Tensor-core flops the tcgen05 prefill attention executes (whole 128 x 64
    tiles, masked elements included), from the prefill decisions: a work item
    is 2 Q tiles of 128 rows (128/g positions x the g query heads of one KV
    head); it runs ceil(nk / 64) kept-prefix tiles (nk = kept tokens before
    position i1 - w) and the band tiles of keys [max(0, i0 - w + 1), i1 - 1],
    each tile 4 * 128 * 64 * D flops (Q K^T and P V) per Q tile."""
    ev = (alpha > 0).cpu().numpy()  # [B,H,T]
    B, H, T = ev.shape
    w, D, g = wl.window, wl.head_dim, wl.gqa
    NP = 128 // g
    span = 2 * NP
    kept = ~ev
    kept[:, :, max(0, T - w):] = False
    cum = np.concatenate([np.zeros((B, H, 1), np.int64), np.cumsum(kept, -1)], -1)  # kept before x
    i0 = np.arange(0, T, span)
    i1 = np.minimum(T, i0 + span)
    nk = cum[:, :, np.clip(i1 - w, 0, T)] * (i1 - w > 0)
    nkt = (nk + 63) // 64
    jlo = np.maximum(0, i0 - w + 1)
    band = (i1 - 1 - jlo + 64) // 64
    tiles = int((nkt + band[None, None, :]).sum())
    return tiles * 2 * 4 * 128 * 64 * D


def decode_step_bytes(wl, retained):
    """Algorithmic HBM bytes of one decode step over the stack, given the
    retained slots summed over (layer, b, h) before the append: the retained
    K/V read, page-table entries (and FP8 page scales), q and o, the new K/V
    row read and written, and the decision inputs (hidden row, W, gamma)."""
    D, B, L = wl.head_dim, wl.batch, wl.layers
    elem = 1 if wl.kv_dtype == "fp8" else 2
    BH = B * wl.kv_heads
    pages = -(-retained // wl.block)  # a lower bound on pages touched
    per_page = 4 + (8 if wl.kv_dtype == "fp8" else 0)
    fixed = L * (2 * B * wl.q_heads * D * 2 + 2 * BH * D * 2 + 2 * BH * D * elem)
    if wl.alpha_source in ("proj", "score"):
        fixed += L * (B * wl.hidden * 2 + wl.kv_heads * wl.hidden * 2 + (wl.hidden * 2 if wl.alpha_source == "proj" else 0))
    return retained * D * 2 * elem + pages * per_page + fixed


def measure_prefill_parts(B_, r, wl, passes=3):
    """The decision logits (dms_decide) and the compaction (dms_prefill_compact)
    of one (replica, layer) timed on their own, each after an L2 flush (a
    512 MB write), the cache reset and the prompt restored before each pass.
    Returns (decide ms or None for neuron sources, compaction ms), medians."""
    u = r.units[0]
    flush = torch.empty(512 << 20, dtype=torch.uint8, device="cuda")
    alpha = torch.empty_like(u["alpha"])
    proj = wl.alpha_source in ("proj", "score")
    dec, comp = [], []
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
    for i in range(passes):
        r.reset_all()
        r.restore_prompt()
        if proj:
            flush.fill_(i)
            ev[0].record()
            B_.dms_decide(u["h"], wl.prompt, u["pargs"].decide.contents, None, alpha)
            ev[1].record()
            torch.cuda.synchronize()
            dec.append(ev[0].elapsed_time(ev[1]))
        flush.fill_(i + 100)
        ev[0].record()
        B_.dms_prefill_compact(u["h"], u["l"], u["pargs"])
        ev[1].record()
        torch.cuda.synchronize()
        comp.append(ev[0].elapsed_time(ev[1]))
    med = lambda x: sorted(x)[len(x) // 2]
    return (med(dec) if proj else None), med(comp)


def measure_single_step(B_, r, steps=32):
    """One replica's decode step on its own: a CUDA graph per step holding
    only that replica's launch(es) between two events, replayed after a 512 MB
    write that evicts its KV from L2.  Returns the median step time in us."""
    wl = r.wl
    units = [u for u in r.units if u["r"] == 0]
    flush = torch.empty(512 << 20, dtype=torch.uint8, device="cuda")
    n = min(steps, r.S)
    r.reset_all()
    r.restore_prompt()
    for u in units:
        B_.dms_prefill(u["h"], u["l"], u["pargs"])
    torch.cuda.synchronize()
    side = torch.cuda.Stream()
    graphs = []
    for i in range(n):
        r.restore_token(i % r.pool)
        torch.cuda.synchronize()
        ga = torch.cuda.CUDAGraph()
        ev = (torch.cuda.Event(enable_timing=True, external=True),
              torch.cuda.Event(enable_timing=True, external=True))
        with torch.cuda.graph(ga, stream=side):
            ev[0].record()
            r.decode_replica(0, i % r.pool)
            ev[1].record()
        graphs.append((ga, ev))
    torch.cuda.synchronize()
    # replays from a fresh prefill: the captures above advanced the caches
    r.reset_all()
    r.restore_prompt()
    for u in units:
        B_.dms_prefill(u["h"], u["l"], u["pargs"])
    times = []
    for i, (ga, ev) in enumerate(graphs):
        r.restore_token(i % r.pool)
        flush.fill_(i & 0xFF)
        ga.replay()
        torch.cuda.synchronize()
        times.append(ev[0].elapsed_time(ev[1]) * 1e3 / wl.layers)
    del graphs
    return float(np.median(times))


def run_ours(args, world, rank, local, primary=True):
    """Measure one workload.  The primary record (the JSON line) carries every
    leg; a secondary record (another workload in the same run) carries the
    device-timed decode and prefill figures and the single-replica latency."""
    from learned_kv_cache_dms_b200 import binding as B_
    wl = I.WORKLOADS[args.workload]
    pk, pk_kind = peaks()
    r = Runner(B_, wl, seed=wl.seed + rank, n_dec=args.decode_steps, kernel=args.decode_kernel, replicas=args.replicas,
               api=args.decode_api)
    S, L = r.S, r.L
    # untimed pass: retained counts after the prefill and after each append
    counts = []
    r.step(counts=counts)
    torch.cuda.synchronize()
    counts = [int(c.item()) for c in torch.stack(counts).cpu()]
    assert r.cache.status() == 0, "cache status %d" % r.cache.status()
    pairs = sum(visible_pairs(u["alpha"], wl) for u in r.units if u["r"] == 0)
    tile_flops = sum(executed_tile_flops(u["alpha"], wl) for u in r.units if u["r"] == 0)
    o_eager = r.od.clone()
    r.capture()
    for _ in range(max(1, args.warmup - 1)):
        r.step()
    torch.cuda.synchronize()
    assert r.cache.status() == 0
    if not r.cycled:
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
    for seg, dec_ms in evs:
        for e0, e1, e2 in seg:
            compact_ms += e0.elapsed_time(e1)
            prefill_attn_ms += e1.elapsed_time(e2)
        decode_ms += dec_ms
    K, B, R = args.steps, wl.batch, r.R
    prefill_ms = compact_ms + prefill_attn_ms
    hot_ms_per_step = (decode_ms + prefill_ms) / K
    # max over ranks of the device times
    decode_ms_max = allreduce(decode_ms, _op("max"), world)
    prefill_ms_max = allreduce(prefill_ms, _op("max"), world)
    hot_max = allreduce(hot_ms_per_step, _op("max"), world)
    dec_tokens = K * S * B * R * world
    value = dec_tokens / (decode_ms_max / 1e3)
    prefill_tps = K * B * R * wl.prompt * world / (prefill_ms_max / 1e3)

    step_bytes = [decode_step_bytes(wl, c) for c in counts[:-1]]  # one replica
    attn_bytes = sum(step_bytes)
    decode_gbs = K * R * attn_bytes / (decode_ms / 1e3) / 1e9
    prefill_flops = 4.0 * wl.head_dim * wl.gqa * pairs  # one replica, every layer
    prefill_tflops = K * R * prefill_flops / (prefill_attn_ms / 1e3) / 1e12
    exec_tflops = K * R * tile_flops / (prefill_attn_ms / 1e3) / 1e12
    clocks = clk.summary()

    # decision logits (A1) and compaction (A2) on their own, L2-cold
    dec_ms1, comp_ms1 = measure_prefill_parts(B_, r, wl)
    T_ = wl.prompt
    ret_prefill = counts[0] / L  # retained slots of one layer after the prefill
    kv_in = 2  # bf16 K/V input rows
    kv_page = 1 if wl.kv_dtype == "fp8" else 2
    dec_bytes = (B * T_ * wl.hidden * 2 + wl.kv_heads * wl.hidden * 2 + B * wl.kv_heads * T_ * 4 +
                 (wl.hidden * 2 if wl.alpha_source == "proj" else 0))
    comp_bytes = B * wl.kv_heads * T_ * 4 + ret_prefill * wl.head_dim * 2 * (kv_in + kv_page)
    neuron_pass = wl.alpha_source not in ("proj", "score")
    if neuron_pass:  # q and k rewritten in place by the neuron/rotary pass, inside the compaction call
        comp_bytes += 2 * B * T_ * (wl.q_heads + wl.kv_heads) * wl.head_dim * 2
    comp_only_ms = comp_ms1 - (dec_ms1 or 0.0)
    decide_roof = None if dec_ms1 is None else {
        "bound": "hbm", "achieved": round(dec_bytes / (dec_ms1 / 1e3) / 1e9, 1), "peak": pk["hbm_gbs"], "unit": "GB/s",
        "frac": round(dec_bytes / (dec_ms1 / 1e3) / 1e9 / pk["hbm_gbs"], 4), "ms": round(dec_ms1, 4),
        "algorithmic_bytes": int(dec_bytes),
        "kernel": "k_decide_proj_tc (%s) via dms_decide, L2-cold"
                  % ("importance score: linear, no norm" if wl.alpha_source == "score" else "adapter RMSNorm + linear")}
    compact_roof = {
        "bound": "hbm", "achieved": round(comp_bytes / (comp_only_ms / 1e3) / 1e9, 1), "peak": pk["hbm_gbs"],
        "unit": "GB/s", "frac": round(comp_bytes / (comp_only_ms / 1e3) / 1e9 / pk["hbm_gbs"], 4),
        "ms": round(comp_only_ms, 4), "algorithmic_bytes": int(comp_bytes),
        "kernel": ("k_neuron_rope8 + " if neuron_pass else "") + "k_prefill_scan_bits + k_prefill_scan_assign + k_prefill_scatter "
                  "(dms_prefill_compact minus dms_decide), L2-cold"}

    single_us = measure_single_step(B_, r)
    e2e = None if (args.no_e2e or not primary) else run_e2e(B_, r, args, world)
    cpu = None
    if primary and rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(wl, args.cpu_seconds)
    kern = ("k_decode_cluster" if r.stacked else
            decode_kernel_name(wl, args.decode_kernel, torch.cuda.get_device_properties(0).multi_processor_count))
    kname = decode_label(wl, kern, r.stacked, L)
    traffic = recorded_traffic(kern, workload_label(wl, S)) if args.replicas is None else None
    roof = {"bound": "hbm", "achieved": round(decode_gbs, 1), "peak": pk["hbm_gbs"], "unit": "GB/s",
            "frac": round(decode_gbs / pk["hbm_gbs"], 4), "traffic": traffic, "kernel": kname,
            "algorithmic_bytes_per_launch": int(attn_bytes / (S * (1 if r.stacked else L))), "peak_source": pk_kind}
    retained_first = counts[0] / (L * B * wl.kv_heads)
    retained_last = counts[-1] / (L * B * wl.kv_heads)
    cfg = {"workload": workload_label(wl, S), "layers": L, "batch": B, "prompt": wl.prompt, "decode_steps": S,
           "hidden": wl.hidden, "q_heads": wl.q_heads, "kv_heads": wl.kv_heads, "head_dim": wl.head_dim,
           "window": wl.window, "block": wl.block, "kv_dtype": wl.kv_dtype, "alpha_source": wl.alpha_source,
           "alpha_per": wl.alpha_per, "keep": list(wl.keep_range) if wl.keep_range else wl.keep,
           "l2": ("decode steps back to back; the stack's retained KV (%.2f GB per step) is many times L2"
                  % (step_bytes[0] / 1e9)) if r.cycled else
                 ("each decode step runs %d independent replicas of the cache back to back (%.0f MB of retained "
                  "KV per step, >= 4x L2), so no replica's KV is in L2 when it is read; no flush"
                  % (R, R * step_bytes[0] / 1e6)),
           "replicas": R,
           "parallelism": "dp%d replicas" % world, "decode_kernel": args.decode_kernel,
           "decode_api": "dms_decode_step_layers" if r.stacked else "dms_decode_step"}
    if r.cycled:
        cfg["decode_inputs"] = "%d distinct token inputs per layer, cycled" % r.pool
    line = {
        "metric": METRIC, "value": round(value, 1), "unit": "tokens/s", "n_gpus": world, "steps": K,
        "warmup": args.warmup, "ms_per_step": round(hot_max, 4), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16" if wl.kv_dtype == "bf16" else "bf16+fp8kv", "data": "synthetic",
        "config": cfg,
        "retained_kv_gbps": round(decode_gbs, 1),
        "retained_kv_frac_of_peak": round(decode_gbs / pk["hbm_gbs"], 4),
        "retained_per_head": [round(retained_first, 1), round(retained_last, 1)],
        "decode_ms_per_token_step": round(decode_ms / (K * S * R), 5),
        "prefill_tok_s": round(prefill_tps, 1),
        "prefill_ms": round(prefill_ms / (K * R), 4),
        "prefill_compact_ms": round(compact_ms / (K * R), 4),
        "prefill_attention_ms": round(prefill_attn_ms / (K * R), 4),
        "prefill_attention": {"bound": "tensor", "achieved": round(prefill_tflops, 2),
                              "peak": pk["bf16_tflops"], "unit": "TFLOP/s",
                              "frac": round(prefill_tflops / pk["bf16_tflops"], 4),
                              "flops_per_launch": prefill_flops / L, "visible_pairs": pairs,
                              "executed_tile_tflops": round(exec_tflops, 2),
                              "frac_executed_tiles": round(exec_tflops / pk["bf16_tflops"], 4),
                              "executed_over_algorithmic": round(tile_flops / prefill_flops, 4),
                              "kernel": "k_attn_prefill_tc<%d> (tcgen05/TMEM)" % wl.head_dim},
        "decode_step_us_single": round(single_us, 3),
        "decide": decide_roof,
        "compaction": compact_roof,
        "achieved_cr": round(wl.max_positions / retained_last, 3) if S == wl.decode_steps else None,
        "region_ms_per_step": round(region_ms / K, 3),
        "roofline": roof, "e2e": e2e, "gpu_launches": kernel_launches_per_step(wl, S, r.stacked) * K * R,
        "clocks": clocks, "cpu_baseline": cpu,
    }
    return line


def _op(name):
    import torch.distributed as dist
    return {"max": dist.ReduceOp.MAX, "sum": dist.ReduceOp.SUM}[name] if dist.is_initialized() else None


def run_e2e(B_, r, args, world):
    """The whole request through the public API with host (pinned) buffers,
    for the R replicas the device-timed measurement uses (R independent
    requests served together; their caches together hold >= 4x L2).  Inside
    the timed region, per request: each replica's prompt (q, k, v, hidden)
    copied host->device and dms_prefill of every layer, the last prompt
    position's outputs copied back; then per decode step one host->device copy
    of every replica's token inputs, one dms_decode_step per (replica, layer),
    one device->host copy of the step's outputs.  Eager calls, no graphs.  A
    multi-layer stack is sampled over its first E2E_STEPS_STACK decode steps."""
    wl = r.wl
    S = r.S if r.L == 1 else min(r.S, E2E_STEPS_STACK)
    R, L = r.R, r.L
    names_p = ("q", "k", "v") + (() if r.neuron else ("h",))
    names_d = ("qd", "kd", "vd") + (() if r.neuron else ("hd",))
    host_p = [{k: x[k].cpu().pin_memory() for k in names_p} for x in r.lay]
    dev_p = [{k: torch.empty_like(x[k]) for k in names_p} for x in r.lay]
    # token inputs: per step, every (replica, layer)'s rows packed in one buffer
    row_elems = [sum(r.lay[l][k][0].numel() for k in names_d) for l in range(L)]
    unit_off = np.cumsum([0] + [row_elems[l] for _ in range(R) for l in range(L)])
    tok_n = int(unit_off[-1])
    one = torch.cat([torch.cat([r.lay[l][k].reshape(r.pool, -1) for k in names_d], 1) for l in range(L)], 1).cpu()
    packed = one.repeat(1, R)  # every replica serves the same token inputs
    assert packed.shape[1] == tok_n
    host_t = torch.empty(S, tok_n, dtype=torch.bfloat16).pin_memory()
    for i in range(S):
        host_t[i].copy_(packed[i % r.pool])
    dev_t = torch.empty(tok_n, dtype=torch.bfloat16, device="cuda")
    od_dev = torch.empty(R, L, *r.od.shape[1:], dtype=r.od.dtype, device="cuda")
    od_host = torch.empty(S, *od_dev.shape, dtype=od_dev.dtype).pin_memory()
    olast_host = torch.empty(R, L, wl.batch, wl.q_heads, wl.head_dim, dtype=r.o.dtype).pin_memory()
    keep, pargs, dargs, alphas = [], [], [], []
    for rr in range(R):
        for l in range(L):
            x, d = r.lay[l], dev_p[l]
            u = r.units[rr * L + l]
            base = int(unit_off[rr * L + l])
            views, o = {}, base
            for k in names_d:
                n = x[k][0].numel()
                views[k] = dev_t[o:o + n].view(x[k][0].shape)
                o += n
            if r.neuron:
                pd = B_.decide_params(x["off"])
                dd = pd
            else:
                pd = B_.decide_params(x["off"], hidden=d["h"], norm_weight=x["gamma"], proj_weight=x["W"])
                dd = B_.decide_params(x["off"], hidden=views["hd"], norm_weight=x["gamma"], proj_weight=x["W"])
            a_tok = torch.empty(wl.batch, wl.kv_heads, dtype=torch.float32, device="cuda")
            keep.append((pd, dd, views, a_tok))
            pargs.append(B_.Cache.prefill_args(d["q"], d["k"], d["v"], r.o, u["alpha"], pd, r.rope))
            dargs.append(B_.Cache.decode_args(views["qd"], views["kd"], views["vd"], od_dev[rr, l], a_tok, dd,
                                              r.rope))
    E = torch.cuda.Event
    total_ms = 0.0
    for it in range(args.steps + 1):
        r.reset_all()
        torch.cuda.synchronize()
        a, c = E(enable_timing=True), E(enable_timing=True)
        a.record()
        for rr in range(R):
            h = r.caches[rr].handle
            for l in range(L):
                for k in names_p:
                    dev_p[l][k].copy_(host_p[l][k], non_blocking=True)
                B_.dms_prefill(h, l, pargs[rr * L + l])
                olast_host[rr, l].copy_(r.o[:, wl.prompt - 1], non_blocking=True)
        for i in range(S):
            dev_t.copy_(host_t[i], non_blocking=True)
            for rr in range(R):
                h = r.caches[rr].handle
                for l in range(L):
                    B_.dms_decode_step(h, l, dargs[rr * L + l])
            od_host[i].copy_(od_dev, non_blocking=True)
        c.record()
        torch.cuda.synchronize()
        if it == 0:
            continue  # warm-up request
        total_ms += a.elapsed_time(c)
    h2d = R * sum(host_p[l][k].numel() * 2 for l in range(L) for k in names_p) + S * tok_n * 2
    d2h = olast_host.numel() * 2 + S * od_dev.numel() * 2
    total_max = allreduce(total_ms, _op("max"), world)
    val = args.steps * R * S * wl.batch * world / (total_max / 1e3)
    out = {"value": round(val, 1), "unit": "tokens/s", "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
           "request_ms": round(total_ms / args.steps, 3),
           "timed": "whole request: %d replica prompts copied in and prefilled, %d decode steps with their "
                    "token copies in and outputs out; generated tokens / request time" % (R, S)}
    if S < r.S:
        out["sample"] = "first %d decode steps" % S
    return out


E2E_STEPS_STACK = 256


# ---------------------------------------------------------------------------
# CPU oracle (baseline arm)
# ---------------------------------------------------------------------------
def oracle_decode_sample(wl, seconds, n_steps_max=None):
    """Time the oracle's decode steps (append + decode attention) of one layer
    on the host cores after an untimed prefill replay; when the workload's
    steps take less than `seconds`, further passes over them start from a copy
    of the prefilled cache (copied outside the timed region).  Returns (tok/s
    over the workload's layer stack, cores, steps, secs, passes)."""
    from oracle import oracle as O
    cores = O.set_threads(os.cpu_count() or 1)
    B, T, S = wl.batch, wl.prompt, wl.decode_steps
    s = wl.seed
    k = I.normal(s, (0, 2), (B, T + S, wl.kv_heads, wl.head_dim), "bf16").float().numpy()
    v = I.normal(s, (0, 3), (B, T + S, wl.kv_heads, wl.head_dim), "bf16").float().numpy()
    q = I.normal(s, (0, 1), (B, S, wl.q_heads, wl.head_dim), "bf16").double().numpy()
    alpha = I.synthetic_alpha(s, (0, 5), B, wl.kv_heads, T + S, I.keep_fractions(wl)).numpy()
    ev = (alpha > 0).astype(np.uint8)
    maxp = -(-wl.max_positions // wl.block)
    c = O.Cache(1, B, wl.kv_heads, wl.head_dim, wl.window, wl.block, wl.max_positions,
                B * wl.kv_heads * maxp, wl.prealloc_tokens, fp8=wl.kv_dtype == "fp8")
    c.prefill(0, np.ascontiguousarray(ev[:, :, :T]), np.ascontiguousarray(k[:, :T]), np.ascontiguousarray(v[:, :T]))
    limit = n_steps_max or S
    n = passes = 0
    dt = 0.0
    while dt < seconds and (passes == 0 or n_steps_max is None):
        cc = c.clone() if n_steps_max is None else c
        t0 = time.perf_counter()
        i = 0
        while i < limit and dt + (time.perf_counter() - t0) < seconds:
            t = T + i
            cc.append(0, np.ascontiguousarray(ev[:, :, t]), np.ascontiguousarray(k[:, t]), np.ascontiguousarray(v[:, t]))
            cc.decode_attention(0, np.ascontiguousarray(q[:, i]))
            i += 1
        dt += time.perf_counter() - t0
        n += i
        passes += 1
    return n * B / (dt * wl.layers), cores, n, dt, passes


def oracle_prefill_sample(wl, seconds):
    """Time the oracle's prefill of one layer on the host cores: the sequential
    replay of the append rule over the whole prompt (slots, pages, stored
    values) and the fp64 masked attention of a sample of prompt rows (b, hq, i)
    drawn uniformly, extrapolated to all B * T * Hq rows.  Returns (prompt
    tok/s over the layer stack, replay s, rows timed, attention s, cores)."""
    from oracle import oracle as O
    cores = O.set_threads(os.cpu_count() or 1)
    B, T, s = wl.batch, wl.prompt, wl.seed
    q = I.normal(s, (0, 1), (B, T, wl.q_heads, wl.head_dim), "bf16").double().numpy()
    k = I.normal(s, (0, 2), (B, T, wl.kv_heads, wl.head_dim), "bf16")
    v = I.normal(s, (0, 3), (B, T, wl.kv_heads, wl.head_dim), "bf16")
    alpha = I.synthetic_alpha(s, (0, 5), B, wl.kv_heads, T, I.keep_fractions(wl)).numpy()
    ev = np.ascontiguousarray((alpha > 0).astype(np.uint8))
    maxp = -(-wl.max_positions // wl.block)
    c = O.Cache(1, B, wl.kv_heads, wl.head_dim, wl.window, wl.block, wl.max_positions,
                B * wl.kv_heads * maxp, wl.prealloc_tokens, fp8=wl.kv_dtype == "fp8")
    k32, v32 = k.float().numpy(), v.float().numpy()
    t0 = time.perf_counter()
    c.prefill(0, ev, k32, v32)
    replay_s = time.perf_counter() - t0
    k64, v64 = k.double().numpy(), v.double().numpy()
    rng = np.random.default_rng(s)
    n, attn_s = 0, 0.0
    batch = 64 * cores
    while attn_s < seconds:
        rows = np.stack([rng.integers(0, B, batch), rng.integers(0, wl.q_heads, batch),
                         rng.integers(0, T, batch)], 1)
        t0 = time.perf_counter()
        O.prefill_attention(q, k64, v64, ev, wl.window, rows=rows)
        attn_s += time.perf_counter() - t0
        n += batch
    total = replay_s + attn_s * (B * T * wl.q_heads) / n
    return B * T / (total * wl.layers), replay_s, n, attn_s, cores


def cpu_baseline(wl, seconds):
    """The oracle as it stands, on the host cores: decode steps on all cores
    (the reported value) and on one core, and a prefill sample on all cores."""
    from oracle import oracle as O
    tps, cores, n, dt, passes = oracle_decode_sample(wl, 0.5 * seconds)
    O.set_threads(1)
    tps1, _, n1, dt1, _ = oracle_decode_sample(wl, 0.2 * seconds)
    O.set_threads(os.cpu_count() or 1)
    ptps, replay_s, prow, pattn_s, pcores = oracle_prefill_sample(wl, 0.3 * seconds)
    return {"value": round(tps, 2), "unit": "tokens/s", "cores": cores, "kind": "oracle", "nproc": os.cpu_count(),
            "sample": "%d decode steps of one layer (append + fp64 decode attention over the retained slots) in %d "
                      "pass(es) over the workload's %d steps, each from the cache after an untimed prefill replay of "
                      "the %d-token prompt, %.1f s timed on %d cores%s"
                      % (n, passes, wl.decode_steps, wl.prompt, dt, cores,
                         "; scaled to the %d-layer stack" % wl.layers if wl.layers > 1 else ""),
            "decode_one_core": {"value": round(tps1, 2), "unit": "tokens/s", "cores": 1,
                                "sample": "%d decode steps, %.1f s" % (n1, dt1)},
            "prefill": {"value": round(ptps, 2), "unit": "prompt tokens/s", "cores": pcores,
                        "sample": "append-rule replay of the %d-token prompt (%.2f s, measured) + fp64 masked "
                                  "attention of %d sampled prompt rows (%.1f s), extrapolated to all %d rows"
                                  % (wl.prompt, replay_s, prow, pattn_s, wl.batch * wl.prompt * wl.q_heads)}}


def _flush_l2(buf, i):
    buf.fill_(i & 0xFF)


def _med(x):
    return sorted(x)[len(x) // 2]


def measure_chunked_prefill(B_, pk, passes=3, chunk=4096, n_chunks=3):
    """Chunked prefill on the Qwen3-8B layer shape: a 12288-token prompt
    prefilled as three calls of 4096 (each dms_prefill_compact, then
    dms_prefill_attention), against the same prompt in one call; adapter
    decisions calibrated for keep 1/8.  L2 flushed before each pass (the chunks
    of a pass run back to back).  Attention flops: 4 * D per visible (query,
    key) pair of the prompt, the same for both."""
    wl = I.WORKLOADS["qwen8b"]
    T = chunk * n_chunks
    g = torch.Generator(device="cuda")
    g.manual_seed(wl.seed * 7 + 1)
    bf = torch.bfloat16
    B, Hq, H, D = wl.batch, wl.q_heads, wl.kv_heads, wl.head_dim

    def rn(*shape, std=1.0):
        return (torch.randn(*shape, generator=g, device="cuda", dtype=torch.float32) * std).to(bf)

    q, k, v, h = rn(B, T, Hq, D), rn(B, T, H, D), rn(B, T, H, D), rn(B, T, wl.hidden)
    gamma, W = rn(wl.hidden), rn(H, wl.hidden, std=wl.hidden ** -0.5)
    d = make_desc(B_, dataclasses.replace(wl, prompt=T, decode_steps=16))
    cache = B_.Cache(d)
    raw = torch.empty(B, H, T, dtype=torch.float32, device="cuda")
    B_.dms_decide(cache.handle, T, B_.decide_params(torch.zeros(B, H, device="cuda"), hidden=h, norm_weight=gamma,
                                                    proj_weight=W), None, raw)
    off, _ = I.calibrate_offsets(raw.cpu().numpy(), I.keep_fractions(wl))
    off = torch.from_numpy(off).cuda()
    o = torch.empty_like(q)
    alpha = torch.empty(B, H, T, dtype=torch.float32, device="cuda")
    parts = []
    for c0 in range(0, T, chunk):
        sl = slice(c0, c0 + chunk)
        qc, kc, vc, hc = (x[:, sl].contiguous() for x in (q, k, v, h))
        oc, ac = torch.empty_like(qc), torch.empty(B, H, chunk, dtype=torch.float32, device="cuda")
        dp = B_.decide_params(off, hidden=hc, norm_weight=gamma, proj_weight=W)
        parts.append(dict(keep=(qc, kc, vc, hc, oc, ac, dp), args=B_.Cache.prefill_args(qc, kc, vc, oc, ac, dp)))
    whole = B_.Cache.prefill_args(q, k, v, o, alpha, B_.decide_params(off, hidden=h, norm_weight=gamma, proj_weight=W))
    flush = torch.empty(512 << 20, dtype=torch.uint8, device="cuda")
    E = lambda: torch.cuda.Event(enable_timing=True)
    ch_comp, ch_attn, one = [], [], []
    for it in range(passes + 1):
        cache.reset()
        _flush_l2(flush, it)
        ev = [(E(), E(), E()) for _ in parts]
        for (e0, e1, e2), pt in zip(ev, parts):
            e0.record()
            B_.dms_prefill_compact(cache.handle, 0, pt["args"])
            e1.record()
            B_.dms_prefill_attention(cache.handle, 0, pt["args"])
            e2.record()
        cache.reset()
        _flush_l2(flush, it + 50)
        a0, a1 = E(), E()
        a0.record()
        B_.dms_prefill(cache.handle, 0, whole)
        a1.record()
        torch.cuda.synchronize()
        if it == 0:
            continue
        ch_comp.append(sum(e0.elapsed_time(e1) for e0, e1, _ in ev))
        ch_attn.append(sum(e1.elapsed_time(e2) for _, e1, e2 in ev))
        one.append(a0.elapsed_time(a1))
    assert cache.status() == 0
    pairs = visible_pairs(alpha, dataclasses.replace(wl, prompt=T))
    flops = 4.0 * D * wl.gqa * pairs
    tot = _med([a + b for a, b in zip(ch_comp, ch_attn)])
    att = _med(ch_attn)
    tf = flops / (att / 1e3) / 1e12
    cache.close()
    return {"workload": "qwen8b_layer_b1_prompt%d_in_%d_chunks_of_%d" % (T, n_chunks, chunk),
            "prefill_tok_s": round(B * T / (tot / 1e3), 1), "ms": round(tot, 4),
            "compact_ms": round(_med(ch_comp), 4), "attention_ms": round(att, 4),
            "one_call_ms": round(_med(one), 4),
            "attention": {"bound": "tensor", "achieved": round(tf, 2), "peak": pk["bf16_tflops"], "unit": "TFLOP/s",
                          "frac": round(tf / pk["bf16_tflops"], 4), "flops": flops,
                          "kernel": "k_attn_prefill_tc<128> with the window copy of the previous chunk"},
            "passes": passes, "l2": "512 MB written before each pass"}


def measure_train_attention(B_, pk, passes=3):
    """The training path on the Qwen3-8B layer shape, 8192 tokens: the gate
    (dms_train_gate) and the soft-gated attention (dms_train_attention), each
    after an L2 flush, median of `passes`.  Algorithmic flops: 4 * D per causal
    (query, key) pair, every key visible (dense causal)."""
    wl = I.WORKLOADS["qwen8b"]
    T, B, Hq, H, D = wl.prompt, wl.batch, wl.q_heads, wl.kv_heads, wl.head_dim
    g = torch.Generator(device="cuda")
    g.manual_seed(wl.seed * 7 + 2)
    bf = torch.bfloat16
    q, k, v = (torch.randn(*s_, generator=g, device="cuda").to(bf) for s_ in ((B, T, Hq, D), (B, T, H, D), (B, T, H, D)))
    alpha = torch.randn(B, H, T, generator=g, device="cuda") * 2 - 0.5
    u = torch.rand(B, H, T, generator=g, device="cuda").clamp(1e-6, 1 - 1e-6)
    noise = torch.log(u) - torch.log1p(-u)
    cache = B_.Cache(make_desc(B_, wl))
    prob, hard, pen = (torch.empty(B, H, T, device="cuda") for _ in range(3))
    o = torch.empty_like(q)
    flush = torch.empty(512 << 20, dtype=torch.uint8, device="cuda")
    E = lambda: torch.cuda.Event(enable_timing=True)
    tg, ta = [], []
    for it in range(passes + 1):
        _flush_l2(flush, it)
        e0, e1, e2, e3 = E(), E(), E(), E()
        e0.record()
        B_.dms_train_gate(cache.handle, T, alpha, noise, 0.1, prob, hard, pen)
        e1.record()
        _flush_l2(flush, it + 50)
        e2.record()
        B_.dms_train_attention(cache.handle, T, q, k, v, pen, o)
        e3.record()
        torch.cuda.synchronize()
        if it:
            tg.append(e0.elapsed_time(e1))
            ta.append(e2.elapsed_time(e3))
    assert cache.status() == 0
    cache.close()
    flops = 4.0 * D * Hq * B * T * (T + 1) / 2
    keep_all = -torch.ones(B, H, T)
    tiles = executed_tile_flops(keep_all, wl)
    att = _med(ta)
    tf = flops / (att / 1e3) / 1e12
    return {"workload": "qwen8b_layer_b1_T%d_dense_causal" % T, "gate_ms": round(_med(tg), 4),
            "attention_ms": round(att, 4), "tok_s": round(B * T / (att / 1e3), 1),
            "attention": {"bound": "tensor", "achieved": round(tf, 2), "peak": pk["bf16_tflops"], "unit": "TFLOP/s",
                          "frac": round(tf / pk["bf16_tflops"], 4), "flops": flops,
                          "frac_executed_tiles": round(tiles / (att / 1e3) / 1e12 / pk["bf16_tflops"], 4),
                          "executed_over_algorithmic": round(tiles / flops, 4),
                          "kernel": "k_attn_prefill_tc<128>, soft mode (penalty on keys outside the window)"},
            "passes": passes, "l2": "512 MB written before each kernel"}


def run_reference(args, world, rank):
    if rank != 0:
        return None
    wl = I.WORKLOADS[args.workload]
    per_step = 4  # decode steps of the oracle per bench step (bounded sample)
    for _ in range(args.warmup):
        oracle_decode_sample(wl, 1e9, n_steps_max=1)[:4]
    tot_tok = tot_s = 0.0
    cores = 1
    for _ in range(args.steps):
        tps, cores, n, dt, _ = oracle_decode_sample(wl, 1e9, n_steps_max=per_step)
        tot_tok += n * wl.batch / wl.layers
        tot_s += dt
    val = tot_tok / tot_s
    return {"impl": "reference", "metric": METRIC, "value": round(val, 2), "unit": "tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(1e3 * tot_s / args.steps, 3),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": workload_label(wl, args.decode_steps or wl.decode_steps), "batch": wl.batch,
                       "prompt": wl.prompt, "decode_steps": wl.decode_steps},
            "cpu_baseline": {"value": round(val, 2), "unit": "tokens/s", "cores": cores, "kind": "oracle",
                             "sample": "%d decode steps per bench step after an untimed prefill replay" % per_step},
            "e2e": {"value": round(val, 2), "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


SECONDARY = (("qwen8b_c8", None), ("llama1b", None), ("llama1b_layer", None), ("reason36", 512), ("kvzap8b", None))
SECONDARY_KEYS = ("value", "unit", "steps", "warmup", "ms_per_step", "config", "roofline", "retained_kv_gbps",
                  "retained_per_head", "decode_ms_per_token_step", "decode_step_us_single", "prefill_tok_s",
                  "prefill_ms", "prefill_compact_ms", "prefill_attention_ms", "prefill_attention", "decide",
                  "compaction", "gpu_launches", "clocks")


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
    if args.measure:
        from learned_kv_cache_dms_b200 import binding as B_
        pk, _ = peaks()
        fn = {"train_attention": measure_train_attention, "chunked_prefill": measure_chunked_prefill}[args.measure]
        print(json.dumps({args.measure: fn(B_, pk)}), flush=True)
        return
    line = run_ours(args, world, rank, local)
    if world == 1 and args.workload == "qwen8b" and not args.no_secondary:
        # the other workloads, measured in the same run (device-timed legs);
        # the 36-layer stack over its first 512 decode steps
        torch.cuda.empty_cache()
        line["secondary"] = {}
        for name, n_dec in SECONDARY:
            sub = argparse.Namespace(**vars(args))
            sub.workload, sub.decode_steps, sub.replicas = name, n_dec, None
            sub.steps = min(args.steps, 3)
            rec = run_ours(sub, world, rank, local, primary=False)
            line["secondary"][name] = {k: rec[k] for k in SECONDARY_KEYS if k in rec}
            torch.cuda.empty_cache()
        # the rows beyond the first prefill-then-decode: chunked prefill and
        # the training path's forward
        from learned_kv_cache_dms_b200 import binding as B_
        pk, _ = peaks()
        line["next"] = {"chunked_prefill": measure_chunked_prefill(B_, pk)}
        torch.cuda.empty_cache()
        line["next"]["train_attention"] = measure_train_attention(B_, pk)
        torch.cuda.empty_cache()
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
