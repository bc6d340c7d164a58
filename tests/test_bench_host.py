"""Host logic of bench.py (no GPU): which decode kernel a workload's line
names, the recorded DRAM traffic, which is reported only while the kernel's
sources are the ones the capture was taken on, and the kernel launches the
line claims."""
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402


@pytest.mark.parametrize("name,kernel", [("qwen8b", "k_decode_cluster"), ("qwen8b_c8", "k_decode_cluster"),
                                         ("llama1b", "k_decode_cluster"), ("reason36", "k_decode_cluster")])
def test_decode_kernel_name_follows_auto_rule(name, kernel):
    wl = bench.I.WORKLOADS[name]
    assert bench.decode_kernel_name(wl, "auto", 148) == kernel
    # an explicit choice is taken as given
    assert bench.decode_kernel_name(wl, "flat", 148) == "k_decode_flat"
    assert bench.decode_kernel_name(wl, "cluster", 148) == "k_decode_cluster"


def test_recorded_traffic_only_for_current_sources(monkeypatch):
    path = os.path.join(ROOT, "profiles", "traffic.txt")
    rows = [ln.split() for ln in open(path) if ln.strip() and not ln.startswith("#")]
    assert rows, "profiles/traffic.txt lists no capture"
    kernel, workload, nbytes, digest = rows[0][:4]
    expect = int(nbytes) if bench.source_digest(kernel) == digest else None
    assert bench.recorded_traffic(kernel, workload) == expect
    # once the sources differ from the captured ones, nothing is reported
    monkeypatch.setattr(bench, "source_digest", lambda k: "0" * 16)
    assert bench.recorded_traffic(kernel, workload) is None
    monkeypatch.undo()
    assert bench.recorded_traffic(kernel, "no_such_workload") is None
    assert bench.recorded_traffic("k_not_recorded", workload) is None



def test_executed_tiles_cover_the_visible_pairs():
    """The tile count of the tcgen05 prefill schedule covers every visible
    (query, key) pair, and with every key kept inside one band it is the
    causal band's tile count."""
    import numpy as np
    import torch
    wl = bench.I.WORKLOADS["qwen8b"]
    rng = np.random.default_rng(0)
    alpha = torch.from_numpy(np.where(rng.random((1, 8, wl.prompt)) < 0.125, -1.0, 1.0).astype(np.float32))
    flops = bench.executed_tile_flops(alpha, wl)
    algo = 4.0 * wl.head_dim * wl.gqa * bench.visible_pairs(alpha, wl)
    assert algo <= flops <= 4 * algo
    # all evicted: only the band; items of 2 * 128 / g positions see keys [i0 - w + 1, i1 - 1]
    allev = torch.ones_like(alpha)
    span = 2 * 128 // wl.gqa
    tiles = 0
    for i0 in range(0, wl.prompt, span):
        i1 = min(wl.prompt, i0 + span)
        tiles += (i1 - 1 - max(0, i0 - wl.window + 1) + 64) // 64
    assert bench.executed_tile_flops(allev, wl) == 8 * tiles * 2 * 4 * 128 * 64 * wl.head_dim


def test_kernel_launch_counts():
    """The launches the bench claims per bench step and replica follow the
    library's launch structure: reset; per layer the logits (adapter / score)
    or the decision neuron and rotary pass, two scan kernels, the scatter and
    the attention; per decode step the rotary pass where needed and one fused
    kernel (one for the whole stack with the layer-range call)."""
    wl = bench.I.WORKLOADS
    assert bench.kernel_launches_per_step(wl["qwen8b"], 128) == 1 + 5 + 128
    assert bench.kernel_launches_per_step(wl["qwen8b_c8"], 128) == 1 + 5 + 128
    assert bench.kernel_launches_per_step(wl["kvzap8b"], 128) == 1 + 5 + 128
    assert bench.kernel_launches_per_step(wl["llama1b"], 256) == 1 + 5 + 256 * 2
    assert bench.kernel_launches_per_step(wl["llama1b_layer"], 256) == 1 + 5 + 256 * 2
    assert bench.kernel_launches_per_step(wl["reason36"], 512, stacked=True) == 1 + 36 * 5 + 512


def test_decode_label_says_what_the_time_covers():
    wl = bench.I.WORKLOADS
    b1 = bench.decode_label(wl["qwen8b"], "k_decode_cluster", False, 1)
    assert "append" in b1 and "decision logit" in b1 and "rotary" not in b1
    fp8 = bench.decode_label(wl["llama1b"], "k_decode_cluster", False, 1)
    assert "append first" in fp8 and "k_decode_append" not in fp8 and "decision logit" not in fp8
    assert "rotary pass" in fp8
    assert "after k_decode_append" in bench.decode_label(wl["llama1b"], "k_decode_flat", False, 1)
    assert "all 36 layers in one launch" in bench.decode_label(wl["reason36"], "k_decode_cluster", True, 36)
