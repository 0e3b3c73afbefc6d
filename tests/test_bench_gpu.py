"""The benchmark's JSON line on a GPU: one short run of `bench.py` (the normal
workload, three timed steps, no CPU baseline and no extra workloads) prints
exactly one line that carries every key of the contract, with values that
are consistent with one another: GB/s from the algorithmic bytes and the step
time, the roofline fraction from its achieved and peak figures, an end-to-end
leg that moved bytes both ways, the launch count of our kernels, and each
phase timed both inside the step (events) and alone (CUDA-graph replay)."""
import json
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_bench_line_carries_the_contract():
    cmd = [sys.executable, os.path.join(ROOT, "bench.py"), "--steps", "3", "--warmup", "3",
           "--no-cpu-baseline", "--no-extra"]
    run = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=600)
    assert run.returncode == 0, run.stderr[-2000:]
    lines = [ln for ln in run.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1, run.stdout[-2000:]
    d = json.loads(lines[0])
    for k in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
              "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config",
              "roofline", "e2e", "gpu_launches", "clocks", "phases_ms", "phases_event_ms",
              "phases_graph_replay_ms", "bytes_per_step"):
        assert k in d, k
    assert d["n_gpus"] == 1 and d["steps"] == 3 and d["warmup"] >= 3
    assert d["unit"] == "GB/s" and d["higher_is_better"] is True
    step_bytes = d["bytes_per_step"]["dispatch"] + d["bytes_per_step"]["combine"]
    assert d["value"] == pytest.approx(step_bytes / (d["ms_per_step"] * 1e-3) / 1e9, rel=1e-6)
    r = d["roofline"]
    assert r["bound"] == "hbm" and r["unit"] == "GB/s"
    assert r["frac"] == pytest.approx(r["achieved"] / r["peak"], rel=1e-9)
    assert 0.0 < r["frac"] < 1.5
    e = d["e2e"]
    assert e["h2d_bytes_per_step"] > 0 and e["d2h_bytes_per_step"] > 0
    assert 0.0 < e["value"] < d["value"]  # the host link is slower than HBM
    assert d["gpu_launches"] == 5 * d["steps"]
    for ph in ("dispatch_notify_with_layout", "dispatch_copy", "combine"):
        assert d["phases_ms"][ph] > 0 and d["phases_graph_replay_ms"][ph] > 0
        assert d["phases_event_ms"][ph] > 0
    # device-timed phases are disjoint spans inside the step that ran them
    dev = d["phases_ms"]
    spans = dev["dispatch_notify_with_layout"] + dev["dispatch_copy"] + dev["combine"]
    assert 0.85 * dev["step_with_phase_timers"] < spans <= 1.001 * dev["step_with_phase_timers"]
    # the three phases alone add up to about one step
    alone = sum(d["phases_graph_replay_ms"].values())
    assert 0.8 * d["ms_per_step"] < alone < 1.2 * d["ms_per_step"]
    assert d["clocks"]["sm_max_mhz"] > 0
