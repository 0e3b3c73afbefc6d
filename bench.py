#!/usr/bin/env python
"""Benchmark: normal-mode MoE token routing (layout -> dispatch -> combine) on
8 simulated ranks x 4096 tokens x 7168 hidden (bf16), top-8 of 256 experts.

One step = ep_notify_dispatch with the fused layout (A1 + A2 in one kernel),
ep_dispatch_cached (the row copy; notify + cached == ep_dispatch) and
ep_combine, over one batch of seeded synthetic input (identity experts:
combine reads the dispatched rows).
Prints ONE JSON line (rank 0).  The headline value is algorithmic HBM GB/s of
dispatch+combine (bytes the method must move, per step, divided by the step
time); tokens/s and the share of 8 TB/s ride along.  The "e2e" figure is the
same metric with every step's inputs uploaded from pinned host memory and its
result downloaded, the copies of neighbouring steps overlapping the compute.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

N > 1 (launched under torchrun) runs N independent replicas, one per GPU:
the routing problem is simulated inside one GPU's HBM, so nothing is
exchanged between GPUs; value = all replicas' bytes / max-over-ranks time.
``--impl reference`` times the CPU oracle on the host (rank 0 only).
"""
from __future__ import annotations

import argparse
import datetime
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time
from typing import Optional

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from workloads import CONFIGS, Workload, make  # noqa: E402

METRIC = "dispatch+combine HBM GB/s (% of 8 TB/s) and tokens/s at 8r×4096×7168 top-8"
UNIT = "GB/s"
SPEC_HBM_GBS = 8000.0
FALLBACK_HBM_GBS = 6650.0


# ---------------------------------------------------------------------------
# algorithmic bytes (bytes the method must move; counts from the seeded run)
# ---------------------------------------------------------------------------

def dispatch_bytes(R, T, H, K, N):
    """x read once, N rows written, top-k ids+weights read, per-copy metadata
    (ids, weights, source index) written, layout/scan metadata."""
    return (R * T * H * 2 + N * H * 2 + R * T * K * (8 + 4) + N * (K * 8 + K * 4 + 4)
            + (R * T * K * 8 + 2 * R * T * R + R * T * R * 4))


def combine_bytes(R, T, H, K, N):
    """N rows read, R*T rows written, received weights read, combined weights
    written, send positions read."""
    return N * H * 2 + R * T * H * 2 + N * K * 4 + R * T * K * 4 + R * T * R * 4


def ll_dispatch_bytes(R, T, H, K, C):
    return R * T * H * 2 + C * H + C * (H // 128) * 4 + R * T * K * (8 + 4) + C * 4


def ll_combine_bytes(R, T, H, K, C):
    return C * H * 2 + R * T * H * 2 + R * T * K * (8 + 4 + 4)


def layout_bytes(S, T, K, E, R):
    return S * T * K * 8 + S * T * R + S * R * 4 + S * E * 4


# ---------------------------------------------------------------------------
# distributed plumbing (also exercised by the CPU gloo tests)
# ---------------------------------------------------------------------------

def dist_env():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", str(rank)))
    return ws, rank, local


def reduce_max(value: float, device=None) -> float:
    """Max of a float over all ranks (identity without a process group)."""
    import torch
    import torch.distributed as dist

    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def reduce_sum(value: float, device=None) -> float:
    import torch
    import torch.distributed as dist

    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return float(t.item())


def aggregate(bytes_per_step_local: float, tokens_per_step_local: float, ms_local: float,
              device=None) -> dict:
    """Whole-job throughput: all ranks' work divided by the slowest rank's time."""
    ms = reduce_max(ms_local, device)
    total_bytes = reduce_sum(bytes_per_step_local, device)
    total_tokens = reduce_sum(tokens_per_step_local, device)
    return {"ms_per_step": ms, "gbs": total_bytes / (ms * 1e-3) / 1e9,
            "tokens_per_s": total_tokens / (ms * 1e-3)}


def barrier(device=None):
    import torch.distributed as dist

    if dist.is_available() and dist.is_initialized() and dist.get_world_size() > 1:
        if dist.get_backend() == "nccl":
            dist.barrier(device_ids=[device.index] if device is not None else None)
        else:
            dist.barrier()


# ---------------------------------------------------------------------------
# clocks during the timed region
# ---------------------------------------------------------------------------

class ClockSampler:
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.f = None

    def start(self):
        try:
            self.f = tempfile.TemporaryFile(mode="w+")
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=self.f, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self) -> dict:
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.f.seek(0)
        rows = [r.strip().split(",") for r in self.f.read().splitlines() if r.strip()]
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in rows:
            try:
                sm.append(float(r[0]))
                mx = float(r[1])
                for nm, v in zip(names, r[4:8]):
                    if v.strip().lower() == "active":
                        reasons.add(nm)
            except (ValueError, IndexError):
                continue
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": mx,
                "reasons": sorted(reasons), "samples": len(sm)}


# ---------------------------------------------------------------------------
# the CPU oracle as a baseline (rank 0, N=1, bounded sample)
# ---------------------------------------------------------------------------

def sample_workload(w: Workload, T_sample: int) -> dict:
    """The first T_sample tokens of every source rank of the seeded workload."""
    full = make(w)
    return {k: np.ascontiguousarray(v[:, :T_sample]) for k, v in full.items()}


def oracle_pass(sample: dict, w: Workload):
    import oracle

    t0 = time.perf_counter()
    res = oracle.normal_path(sample["x"], sample["topk_idx"], sample["topk_weights"], w.E)
    dt = time.perf_counter() - t0
    R, T, H = sample["x"].shape
    N = int(res["recv_count"].sum())
    nbytes = dispatch_bytes(R, T, H, w.K, N) + combine_bytes(R, T, H, w.K, N)
    return dt, nbytes, R * T


def host_cpu() -> dict:
    """The host's CPU model and core counts (the CPU baseline runs on one core)."""
    model = None
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    model = line.split(":", 1)[1].strip()
                    break
    except OSError:
        pass
    nproc = os.cpu_count()
    try:
        avail = len(os.sched_getaffinity(0))
    except (AttributeError, OSError):
        avail = nproc
    return {"cpu_model": model, "nproc": nproc, "cores_available": avail}


def cpu_baseline(w: Workload, T_sample: int = 2048, reps: int = 3) -> dict:
    sample = sample_workload(w, T_sample)
    times = []
    for _ in range(reps):
        dt, nbytes, ntok = oracle_pass(sample, w)
        times.append(dt)
    dt = statistics.median(times)
    host = host_cpu()
    return {"value": nbytes / dt / 1e9, "unit": UNIT, "cores": 1, "kind": "oracle",
            "cores_used": f"1 of {host['cores_available']} cores", **host,
            "sample": (f"first {T_sample} of {w.T} tokens of each of the {w.R} source ranks "
                       f"(same seeded workload), layout+prefix+dispatch+combine, median of "
                       f"{reps} single-threaded runs of the C oracle"),
            "tokens_per_s": ntok / dt, "seconds": dt}


def workload_config(T: int, ws: int) -> dict:
    """The `config` of the JSON line, the same for both arms."""
    w = CONFIGS["normal"]
    return {"workload": f"normal: R={w.R} simulated ranks x T={T} tokens x H={w.H} bf16, "
                        f"E={w.E} experts, top-{w.K} distinct uniform, fp32 softmax weights, "
                        "identity experts",
            "global_batch": w.R * T * ws, "seq_len": None,
            "parallelism": f"replicas x{ws}" if ws > 1 else "single GPU",
            "l2": "inputs larger than L2 (x 470 MB, recv_x 2.5 GB written); no flush"}


def run_reference(args) -> None:
    ws, rank, _ = dist_env()
    if rank != 0:
        return
    w = CONFIGS["normal"]
    T_sample = 512
    sample = sample_workload(w, T_sample)
    for _ in range(args.warmup):
        oracle_pass(sample, w)
    t0 = time.perf_counter()
    tot_bytes, tot_tok = 0, 0
    for _ in range(args.steps):
        _, nb, nt = oracle_pass(sample, w)
        tot_bytes += nb
        tot_tok += nt
    dt = time.perf_counter() - t0
    value = tot_bytes / dt / 1e9
    host = host_cpu()
    config = workload_config(w.T, 1)
    # the CPU arm times a sample of the workload; the rate is per byte and per
    # token of that sample
    config["sample"] = {"tokens_per_rank": T_sample, "of_tokens_per_rank": w.T,
                        "source_ranks": w.R, "global_batch_timed": w.R * T_sample}
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt / args.steps * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic",
        "config": config,
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": 1, "kind": "oracle",
                         "cores_used": f"1 of {host['cores_available']} cores", **host,
                         "sample": (f"each step runs the C oracle single-threaded on the first "
                                    f"{T_sample} of {w.T} tokens of each of the {w.R} source "
                                    "ranks (bytes and tokens counted for that sample)")},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        "tokens_per_s": tot_tok / dt,
    }
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------------------
# GPU arm
# ---------------------------------------------------------------------------

def load_peak():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


# the source files each timed kernel is built from (for staleness checks)
KERNEL_SOURCES = {
    "dispatch_copy_rows_kernel": ["ep_dispatch.cu", "ep_scan.cuh", "ep_common.cuh", "ep_api.cu"],
    "combine_kernel": ["ep_combine.cu", "ep_common.cuh", "ep_api.cu"],
}


def kernel_source_hash(kernel: str) -> str:
    """sha1 of the code of the CUDA sources of `kernel` (comments and blank
    lines removed, so that an edit of a comment keeps it), to tell whether
    recorded counters still describe the kernel that runs."""
    import hashlib
    import re

    h = hashlib.sha1()
    csrc = os.path.join(ROOT, "combine_get_dispatch_06_b200", "csrc")
    for f in KERNEL_SOURCES[kernel]:
        h.update(f.encode())
        with open(os.path.join(csrc, f)) as fh:
            text = re.sub(r"/\*.*?\*/", "", fh.read(), flags=re.S)
        for line in text.splitlines():
            code = line.split("//", 1)[0].rstrip()
            if code:
                h.update(code.encode() + b"\n")
    return h.hexdigest()


def recorded_traffic(kernel: str, T: int):
    """DRAM bytes (read + write) per launch of `kernel` on the normal workload,
    from the ncu capture summarised in profiles/dram_traffic_normal.md -- or
    None if that capture is of another build of the kernel."""
    import re

    path = os.path.join(ROOT, "profiles", "dram_traffic_normal.md")
    try:
        text = open(path).read()
    except OSError:
        return None
    if T != CONFIGS["normal"].T:
        return None
    m = re.search(rf"\|\s*{kernel}\s*\|\s*(\d+)\s*\|\s*([0-9a-f]{{40}})\s*\|", text)
    if not m or m.group(2) != kernel_source_hash(kernel):
        return None
    return int(m.group(1))


def to_dev_bf16(a: np.ndarray, device):
    import torch

    return torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).to(device)


def graph_time_ms(fn, device, iters=20, warm=3) -> float:
    """Mean device time of fn() in ms: `iters` calls captured in one CUDA
    graph and replayed, so host launch overhead does not enter the number.
    fn launches on the current stream (the capture stream while capturing)."""
    import torch

    stream = torch.cuda.current_stream(device)
    for _ in range(warm):
        fn()
    torch.cuda.synchronize(device)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        for _ in range(iters):
            fn()
    g.replay()
    torch.cuda.synchronize(device)
    a = torch.cuda.Event(enable_timing=True)
    b = torch.cuda.Event(enable_timing=True)
    a.record(stream)
    g.replay()
    b.record(stream)
    b.synchronize()
    del g
    return a.elapsed_time(b) / iters


def extra_configs(device, ep) -> dict:
    """Secondary workloads (timed only; parity is the tests' job)."""
    import torch

    out = {}

    def timeit(fn, iters=20, warm=3):
        return graph_time_ms(fn, device, iters=iters, warm=warm)

    # layout only: [4096, 8] of 256 experts, 8 ranks
    w = CONFIGS["layout"]
    inp = make(w, with_x=False)
    idx = torch.from_numpy(inp["topk_idx"][0]).to(device)
    o = {"a": torch.empty((w.R,), dtype=torch.int32, device=device),
         "b": torch.empty((w.E,), dtype=torch.int32, device=device),
         "c": torch.empty((w.T, w.R), dtype=torch.bool, device=device)}

    def lay():
        ep.ep_get_dispatch_layout(idx, w.E, w.R, num_tokens_per_rank=o["a"],
                                  num_tokens_per_expert=o["b"], is_token_in_rank=o["c"])
    ms = timeit(lay, iters=200, warm=10)
    out["layout_4096x8"] = {"us": ms * 1e3,
                            "gbs": layout_bytes(1, w.T, w.K, w.E, w.R) / (ms * 1e-3) / 1e9}

    # skewed routing: dispatch + combine
    w = CONFIGS["skewed"]
    inp = make(w)
    x = to_dev_bf16(inp["x"], device)
    idx = torch.from_numpy(inp["topk_idx"]).to(device)
    wt = torch.from_numpy(inp["topk_weights"]).to(device)
    # the same call sequence as the headline step: layout fused into notify
    d = ep.ep_notify_dispatch(idx, wt, w.T, w.R, w.E, with_layout=True)
    d["recv_x"] = ep.ep_dispatch_cached(x, d["send_pos"])
    cx, cw = ep.ep_combine(d["recv_x"], d["send_pos"], d["recv_topk_weights"])
    wsp = torch.empty(ep.ep_dispatch_workspace_bytes(w.R, w.T, w.E), dtype=torch.uint8,
                      device=device)
    buf = {"d": d}

    def sk():
        ep.ep_notify_dispatch(idx, wt, w.T, w.R, w.E, with_layout=True, out=d, workspace=wsp)
        ep.ep_dispatch_cached(x, d["send_pos"], recv_x=d["recv_x"])
        ep.ep_combine(d["recv_x"], d["send_pos"], d["recv_topk_weights"], combined_x=cx,
                      combined_topk_weights=cw)
    ms = timeit(sk, iters=20)
    N = int(buf["d"]["recv_count"].sum().item())
    nb = dispatch_bytes(w.R, w.T, w.H, w.K, N) + combine_bytes(w.R, w.T, w.H, w.K, N)
    out["skewed"] = {"ms": ms, "gbs": nb / (ms * 1e-3) / 1e9, "copies": N,
                     "tokens_per_s": w.R * w.T / (ms * 1e-3)}
    del x, idx, wt, buf, d, cx, cw, wsp
    torch.cuda.empty_cache()

    # low latency: FP8 dispatch + weighted combine
    w = CONFIGS["ll"]
    inp = make(w)
    R, T, H, E, K = w.R, w.T, w.H, w.E, w.K
    x = to_dev_bf16(inp["x"], device)
    idx = torch.from_numpy(inp["topk_idx"]).to(device)
    wt = torch.from_numpy(inp["topk_weights"]).to(device)
    ws = torch.empty(ep.ep_ll_workspace_bytes(R, T, E), dtype=torch.uint8, device=device)
    d = ep.ep_ll_dispatch(x, idx, E, use_fp8=True, workspace=ws)
    torch.cuda.synchronize(device)
    # synthetic expert outputs: bf16 slab rows (the method does not look at them)
    El = E // R
    y = torch.empty((R, El, R * T, H), dtype=torch.bfloat16, device=device)
    cnt = d["recv_count"].view(-1).cpu()
    yv = y.view(E, R * T, H)
    g = torch.Generator(device=device).manual_seed(1)
    for e in range(E):
        n = int(cnt[e])
        if n:
            yv[e, :n] = torch.randn((n, H), generator=g, device=device).to(torch.bfloat16)
    out_c = torch.empty((R, T, H), dtype=torch.bfloat16, device=device)

    def ll_d():
        ep.ep_ll_dispatch(x, idx, E, use_fp8=True, out=d, workspace=ws)

    def ll_c():
        ep.ep_ll_combine(y, idx, wt, d["ll_pos"], out=out_c)

    ms_d = timeit(ll_d, iters=50)
    ms_c = timeit(ll_c, iters=50)
    # the same back-to-back calls with the full-grid phase timers on: each
    # call's span from its zeroing kernel's earliest block (after the wait for
    # the previous call) to its last block, without the hand-off between calls
    timers = torch.zeros(8 * len(ep.PHASES), dtype=torch.int64, device=device)
    ep.ep_set_phase_timers(timers)
    try:
        timeit(ll_d, iters=50)
        timeit(ll_c, iters=50)
    finally:
        ep.ep_set_phase_timers(None)
    pt = ep.phase_timer_ms(timers)
    span_d, span_c = pt["ll_dispatch"]["ms"], pt["ll_combine"]["ms"]
    C = int(cnt.sum())
    out["low_latency"] = {
        "dispatch_us": ms_d * 1e3, "combine_us": ms_c * 1e3,
        "dispatch_gbs": ll_dispatch_bytes(R, T, H, K, C) / (ms_d * 1e-3) / 1e9,
        "combine_gbs": ll_combine_bytes(R, T, H, K, C) / (ms_c * 1e-3) / 1e9,
        "dispatch_span_us": span_d * 1e3, "combine_span_us": span_c * 1e3,
        "dispatch_span_gbs": ll_dispatch_bytes(R, T, H, K, C) / (span_d * 1e-3) / 1e9,
        "combine_span_gbs": ll_combine_bytes(R, T, H, K, C) / (span_c * 1e-3) / 1e9,
        "span_method": "full-grid phase timers (%globaltimer), mean over the timed calls; "
                       "dispatch_us / combine_us: CUDA-graph replay time per call",
        "copies": C, "tokens_per_s": R * T / ((ms_d + ms_c) * 1e-3)}
    del x, idx, wt, y, d, out_c
    torch.cuda.empty_cache()
    return out


def routing_step(ep, io: dict, out: dict, wsp, status, R: int, T: int, E: int, stream=None,
                 ev=None) -> None:
    """One step of the timed path.

    The layout (A1) is fused into the notify scan (A2): ep_notify_dispatch with
    the layout outputs returns the layout, the handle and the received top-k
    metadata from one kernel.  ep_dispatch_cached moves the rows (ep_dispatch
    == ep_notify_dispatch + ep_dispatch_cached; the halves are called apart so
    that the row copy gets its own events), and ep_combine reduces them back
    with identity experts (y = recv_x).  io: inputs x, idx, wt and combined
    outputs cx, cw; out: handle, layout and receive buffers; ev: five events
    recorded around the phases, or None."""
    if ev is not None:
        ev[0].record(stream)
        ev[1].record(stream)
    ep.ep_notify_dispatch(io["idx"], io["wt"], T, R, E, with_layout=True, out=out,
                          workspace=wsp, status=status, stream=stream)
    if ev is not None:
        ev[2].record(stream)
    ep.ep_dispatch_cached(io["x"], out["send_pos"], recv_x=out["recv_x"], status=status,
                          stream=stream)
    if ev is not None:
        ev[3].record(stream)
    ep.ep_combine(out["recv_x"], out["send_pos"], out["recv_topk_weights"],
                  combined_x=io["cx"], combined_topk_weights=io["cw"], status=status,
                  stream=stream)
    if ev is not None:
        ev[4].record(stream)


def step_buffers(R: int, T: int, H: int, E: int, K: int, device) -> tuple:
    """Device buffers of routing_step: (out, cx, cw, workspace, status)."""
    import torch

    import combine_get_dispatch_06_b200 as ep

    cap = R * T
    out = {
        "recv_x": torch.empty((R, cap, H), dtype=torch.bfloat16, device=device),
        "recv_topk_idx": torch.empty((R, cap, K), dtype=torch.int64, device=device),
        "recv_topk_weights": torch.empty((R, cap, K), dtype=torch.float32, device=device),
        "recv_src_idx": torch.empty((R, cap), dtype=torch.int32, device=device),
        "rank_prefix_matrix": torch.empty((R, R), dtype=torch.int32, device=device),
        "recv_count": torch.empty((R,), dtype=torch.int32, device=device),
        "num_recv_tokens_per_expert": torch.empty((R, E // R), dtype=torch.int32, device=device),
        "send_pos": torch.empty((R, T, R), dtype=torch.int32, device=device),
        "num_tokens_per_rank": torch.empty((R, R), dtype=torch.int32, device=device),
        "num_tokens_per_expert": torch.empty((R, E), dtype=torch.int32, device=device),
        "is_token_in_rank": torch.empty((R, T, R), dtype=torch.bool, device=device),
    }
    cx = torch.empty((R, T, H), dtype=torch.bfloat16, device=device)
    cw = torch.empty((R, T, K), dtype=torch.float32, device=device)
    wsp = torch.empty(ep.ep_dispatch_workspace_bytes(R, T, E), dtype=torch.uint8, device=device)
    return out, cx, cw, wsp, ep.new_status(device)


def run_ours(args) -> None:
    import torch
    import torch.distributed as dist

    ws, rank, local = dist_env()
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)  # before the process group: NCCL binds this device
    if ws > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    import combine_get_dispatch_06_b200 as ep  # fails loudly without libep.so

    w = CONFIGS["normal"]
    R, T, H, E, K = w.R, (args.tokens or w.T), w.H, w.E, w.K
    inp = make(Workload(w.name, R=R, T=T, H=H, E=E, K=K, seed=w.seed + rank))
    stream = torch.cuda.current_stream(device)

    # pinned host copies for the end-to-end leg
    x_h = torch.from_numpy(inp["x"].view(np.int16)).view(torch.bfloat16).pin_memory()
    idx_h = torch.from_numpy(inp["topk_idx"]).pin_memory()
    w_h = torch.from_numpy(inp["topk_weights"]).pin_memory()
    x = x_h.to(device)
    idx = idx_h.to(device)
    wt = w_h.to(device)

    out, cx, cw, wsp, status = step_buffers(R, T, H, E, K, device)

    io0 = {"x": x, "idx": idx, "wt": wt, "cx": cx, "cw": cw}

    def step(ev=None, io=io0):
        routing_step(ep, io, out, wsp, status, R, T, E, stream, ev)

    for _ in range(max(3, args.warmup)):
        step()
    torch.cuda.synchronize(device)
    if int(status.item()) != 0:
        raise RuntimeError(f"device status {int(status.item())} during warm-up")
    N = int(out["recv_count"].sum().item())
    bytes_d = dispatch_bytes(R, T, H, K, N)
    bytes_c = combine_bytes(R, T, H, K, N)
    bytes_step = bytes_d + bytes_c

    # ---- timed region: exactly K steps, device-resident inputs ------------
    # The steps run back to back with no event between their kernels, since an
    # event between two programmatically chained launches keeps the second
    # from starting early.  A second pass of K steps runs the same sequence
    # with the library's full-grid phase timers on (%globaltimer, earliest
    # block start to last block end of each phase): phases_ms.  A third
    # records CUDA events around each phase (phases_event_ms); the roofline's
    # kernel time comes from those events.
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(5)] for _ in range(args.steps)]
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)

    def timed_pass(with_phases: bool) -> float:
        barrier(device)
        torch.cuda.synchronize(device)
        t_start.record(stream)
        for i in range(args.steps):
            step(evs[i] if with_phases else None)
        t_end.record(stream)
        torch.cuda.synchronize(device)
        barrier(device)
        return t_start.elapsed_time(t_end) / args.steps

    sampler = ClockSampler(local)
    sampler.start()
    time.sleep(0.3)
    ms_local = timed_pass(False)
    timers = torch.zeros(24, dtype=torch.int64, device=device)
    ep.ep_set_phase_timers(timers)
    ms_timers = timed_pass(False)
    ep.ep_set_phase_timers(None)
    ms_phased = timed_pass(True)
    clocks = sampler.stop()
    pt = ep.phase_timer_ms(timers)
    for ph in ("notify", "copy", "combine"):
        if pt[ph]["launches"] != args.steps:
            raise RuntimeError(f"phase timer {ph}: {pt[ph]['launches']} of {args.steps} steps")
    phases_dev = {"dispatch_notify_with_layout": pt["notify"]["ms"],
                  "dispatch_copy": pt["copy"]["ms"], "combine": pt["combine"]["ms"]}
    phases_dev["dispatch"] = phases_dev["dispatch_notify_with_layout"] + phases_dev["dispatch_copy"]
    phases_dev["step_with_phase_timers"] = ms_timers
    notify_ms = statistics.mean(e[1].elapsed_time(e[2]) for e in evs)
    copy_ms = statistics.mean(e[2].elapsed_time(e[3]) for e in evs)
    comb_ms = statistics.mean(e[3].elapsed_time(e[4]) for e in evs)
    disp_ms = notify_ms + copy_ms
    agg = aggregate(bytes_step, R * T, ms_local, device)
    if int(status.item()) != 0:
        raise RuntimeError(f"device status {int(status.item())} in the timed region")

    # Each phase alone, replayed from a CUDA graph on the same buffers (outside
    # the timed region): no event sits between the kernels of a phase, so the
    # launch chaining inside it stays, as in the steps of the timed region.
    phases_graph = {
        "dispatch_notify_with_layout": graph_time_ms(
            lambda: ep.ep_notify_dispatch(idx, wt, T, R, E, with_layout=True, out=out,
                                          workspace=wsp, status=status), device, iters=50),
        "dispatch_copy": graph_time_ms(
            lambda: ep.ep_dispatch_cached(x, out["send_pos"], recv_x=out["recv_x"],
                                          status=status), device, iters=10),
        "combine": graph_time_ms(
            lambda: ep.ep_combine(out["recv_x"], out["send_pos"], out["recv_topk_weights"],
                                  combined_x=cx, combined_topk_weights=cw, status=status),
            device, iters=10),
    }
    torch.cuda.synchronize(device)
    if int(status.item()) != 0:
        raise RuntimeError(f"device status {int(status.item())} in the phase replays")

    # ---- end to end: host inputs in, host result out, every step -----------
    # Batches stream the way a serving loop feeds them: while step i computes,
    # the inputs of step i+1 go up on one copy stream and the result of step
    # i-1 comes down on another (the link is full duplex).  Two device sets of
    # inputs and results alternate; events keep a set from being overwritten
    # before the step or the copy that reads it is done.
    cx_h = torch.empty((R, T, H), dtype=torch.bfloat16).pin_memory()
    cw_h = torch.empty((R, T, K), dtype=torch.float32).pin_memory()
    e2e_steps = max(3, min(args.steps, 20))
    io1 = {k: torch.empty_like(v) for k, v in io0.items()}
    ios = (io0, io1)
    s_up = torch.cuda.Stream(device)
    s_down = torch.cuda.Stream(device)
    ev_up = [torch.cuda.Event() for _ in ios]
    ev_done = [torch.cuda.Event() for _ in ios]
    ev_down = [torch.cuda.Event() for _ in ios]

    def e2e_run(nsteps, start=None):
        if start is not None:
            s_up.wait_event(start)
        for i in range(nsteps):
            j = i % 2
            io = ios[j]
            with torch.cuda.stream(s_up):
                if i >= 2:
                    s_up.wait_event(ev_done[j])      # step i-2 has read this set
                io["x"].copy_(x_h, non_blocking=True)
                io["idx"].copy_(idx_h, non_blocking=True)
                io["wt"].copy_(w_h, non_blocking=True)
                ev_up[j].record(s_up)
            stream.wait_event(ev_up[j])
            if i >= 2:
                stream.wait_event(ev_down[j])        # result of step i-2 is on the host
            step(io=io)
            ev_done[j].record(stream)
            with torch.cuda.stream(s_down):
                s_down.wait_event(ev_done[j])
                cx_h.copy_(io["cx"], non_blocking=True)
                cw_h.copy_(io["cw"], non_blocking=True)
                ev_down[j].record(s_down)
        stream.wait_stream(s_down)

    e2e_run(2)
    barrier(device)
    torch.cuda.synchronize(device)
    a = torch.cuda.Event(enable_timing=True)
    b = torch.cuda.Event(enable_timing=True)
    a.record(stream)
    e2e_run(e2e_steps, start=a)
    b.record(stream)
    torch.cuda.synchronize(device)
    barrier(device)
    e2e = aggregate(bytes_step, R * T, a.elapsed_time(b) / e2e_steps, device)
    if int(status.item()) != 0:
        raise RuntimeError(f"device status {int(status.item())} in the end-to-end leg")
    if not torch.equal(cx_h.view(torch.int16), cx.cpu().view(torch.int16)):
        raise RuntimeError("end-to-end result differs from the device-resident step's")
    h2d = x_h.numel() * 2 + idx_h.numel() * 8 + w_h.numel() * 4
    d2h = cx_h.numel() * 2 + cw_h.numel() * 4

    peak, peak_kind = load_peak()
    bytes_copy = R * T * H * 2 + N * H * 2       # rows: read once, written per copy
    if copy_ms >= comb_ms:
        dominant, dom_bytes, dom_ms = "dispatch_copy_rows_kernel", bytes_copy, copy_ms
    else:
        dominant, dom_bytes, dom_ms = "combine_kernel", bytes_c, comb_ms
    achieved = dom_bytes / (dom_ms * 1e-3) / 1e9
    traffic = recorded_traffic(dominant, T)

    line = {
        "metric": METRIC, "value": agg["gbs"], "unit": UNIT, "n_gpus": ws, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": agg["ms_per_step"], "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": workload_config(T, ws),
        "tokens_per_s": agg["tokens_per_s"],
        "pct_of_8TBps": 100.0 * agg["gbs"] / (SPEC_HBM_GBS * ws),
        "phases_ms": phases_dev,
        "phases_method": "device full-grid timers: %globaltimer from the earliest block start "
                         "(after the launch's wait for the previous grid) of a phase's first "
                         "kernel to the last block end of its last kernel, mean of K steps of "
                         "the timed sequence with no events between kernels",
        "phases_event_ms": {"dispatch": disp_ms, "dispatch_notify_with_layout": notify_ms,
                            "dispatch_copy": copy_ms, "combine": comb_ms,
                            "step_with_phase_events": ms_phased},
        "phases_graph_replay_ms": phases_graph,
        "bytes_per_step": {"dispatch": bytes_d, "combine": bytes_c, "copies": N},
        "roofline": {"bound": "hbm", "kernel": dominant, "achieved": achieved, "peak": peak,
                     "unit": "GB/s", "frac": achieved / peak, "traffic": traffic,
                     "algorithmic_bytes": dom_bytes,
                     "peak_source": f"{peak_kind} copy bandwidth (MEASURED_PEAKS.json hbm_gbs)"
                     if peak_kind == "measured" else "fallback 6.65 TB/s"},
        "e2e": {"value": e2e["gbs"], "unit": UNIT, "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "ms_per_step": e2e["ms_per_step"]},
        "gpu_launches": 5 * args.steps,   # zeroing, scan (+layout), pad, copy, combine per step
        "clocks": clocks,
    }
    if ws == 1 and rank == 0 and not args.no_extra and T == CONFIGS["normal"].T:
        line["extra"] = extra_configs(device, ep)
    if ws == 1 and rank == 0 and not args.no_cpu_baseline and T == CONFIGS["normal"].T:
        line["cpu_baseline"] = cpu_baseline(w)
    if rank == 0:
        print(json.dumps(line), flush=True)
    if ws > 1:
        dist.destroy_process_group()


# ---------------------------------------------------------------------------
# one rank per GPU (--mode sharded)
# ---------------------------------------------------------------------------

def shard_bytes(R, T, H, K, N):
    """Algorithmic bytes of one rank's dispatch + combine: its T rows read
    once, its N copies written, its ids and weights read, per-copy metadata
    written, its layout / positions; combine reads the N rows back, writes T
    rows, weights and positions."""
    disp = T * H * 2 + N * H * 2 + T * K * 12 + N * (K * 12 + 4) + T * K * 8 + 2 * T * R + T * R * 4
    comb = N * H * 2 + T * H * 2 + N * K * 4 + T * K * 4 + T * R * 4
    return disp, comb


def sharded_ll(args, device, rank: int, ws: int, timed) -> Optional[dict]:
    """The low-latency pair with one rank per GPU, at the LL workload's shape
    per rank (T = 128 tokens, H = 7168, top-8 of 256 experts, FP8): counts
    exchange, dispatch into the destinations' slabs, identity experts (the
    output slabs are left as they are), combine.  Timed like the normal step
    (CUDA-graph replay when the capture works); None when the experts do not
    divide over the ranks."""
    import torch
    import torch.distributed as dist

    from combine_get_dispatch_06_b200.shard import ShardedBuffer

    w0 = CONFIGS["ll"]
    if w0.E % ws != 0:
        return None
    w = Workload("ll_sharded", R=ws, T=w0.T, H=w0.H, E=w0.E, K=w0.K, seed=w0.seed)
    inp = make(w, ranks=[rank])
    x = to_dev_bf16(inp["x"][0], device)
    idx = torch.from_numpy(inp["topk_idx"][0]).to(device)
    wt = torch.from_numpy(inp["topk_weights"][0]).to(device)
    out = torch.empty((w.T, w.H), dtype=torch.bfloat16, device=device)
    buf = ShardedBuffer(dist.group.WORLD, w.T, w.H, w.K, w.E, device=device)
    buf.enable_low_latency(use_fp8=True)

    def step():
        buf.ll_dispatch(x, idx)
        buf.ll_combine(idx, wt, out=out)

    for _ in range(max(3, args.warmup)):
        step()
    torch.cuda.synchronize(device)
    if int(buf.status.item()) != 0:
        raise RuntimeError(f"device status {int(buf.status.item())} in the LL warm-up")
    C = int(buf._ll["counts"].sum().item())          # rows this rank sends
    nbytes = ll_dispatch_bytes(1, w.T, w.H, w.K, C) + ll_combine_bytes(1, w.T, w.H, w.K, C)
    graph, note = None, None
    try:
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            step()
        torch.cuda.synchronize(device)
        graph = g
    except Exception as e:  # capture refused: time the eager pair only
        note = f"capture failed: {type(e).__name__}: {str(e)[:200]}"
        torch.cuda.synchronize(device)
    ms = timed(graph.replay) if graph is not None else timed(step)
    agg = aggregate(nbytes, w.T, ms, device)
    if int(buf.status.item()) != 0:
        raise RuntimeError(f"device status {int(buf.status.item())} in the LL timed region")
    del graph
    torch.cuda.synchronize(device)
    buf.close()
    return {"workload": f"low latency, one rank per GPU: R={ws} x T={w.T} tokens x H={w.H}, "
                        f"E={w.E}, top-{w.K}, FP8 dispatch, weighted combine",
            "us_per_step": agg["ms_per_step"] * 1e3, "gbs": agg["gbs"],
            "tokens_per_s": agg["tokens_per_s"], "cuda_graph": note is None,
            "cuda_graph_note": note}


def run_sharded(args) -> None:
    """The normal workload with one rank per GPU: rank r holds its own T
    tokens, writes their rows into the destination GPUs' receive buffers
    through peer pointers (CUDA IPC over NVLink) and gathers them back at
    combine; the notify counts travel by an NCCL all-gather and the phases
    are ordered by stream-ordered NCCL all-reduces (no host round trip).
    R = number of GPUs, 32 experts per rank unless 256 divides evenly."""
    import torch
    import torch.distributed as dist

    ws, rank, local = dist_env()
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
    os.environ.setdefault("MASTER_PORT", "29533")
    dist.init_process_group("nccl", rank=rank, world_size=ws,
                            timeout=datetime.timedelta(seconds=120))
    from combine_get_dispatch_06_b200.shard import ShardedBuffer  # fails loudly without libep.so

    w0 = CONFIGS["normal"]
    R, T, H, K = ws, (args.tokens or w0.T), w0.H, w0.K
    E = w0.E if w0.E % R == 0 else 32 * R
    w = Workload("normal_sharded", R=R, T=T, H=H, E=E, K=K, seed=w0.seed)
    inp = make(w, ranks=[rank])
    x = to_dev_bf16(inp["x"][0], device)
    idx = torch.from_numpy(inp["topk_idx"][0]).to(device)
    wt = torch.from_numpy(inp["topk_weights"][0]).to(device)
    cx = torch.empty((T, H), dtype=torch.bfloat16, device=device)
    cw = torch.empty((T, K), dtype=torch.float32, device=device)
    buf = ShardedBuffer(dist.group.WORLD, T, H, K, E, device=device)
    stream = torch.cuda.current_stream(device)

    def step():
        buf.dispatch(x, idx, wt)
        buf.combine(combined_x=cx, combined_topk_weights=cw)

    for _ in range(max(3, args.warmup)):
        step()
    torch.cuda.synchronize(device)
    if int(buf.status.item()) != 0:
        raise RuntimeError(f"device status {int(buf.status.item())} during warm-up")
    sp = buf.send_pos
    N = int((sp >= 0).sum().item())
    remote = torch.ones(R, dtype=torch.bool, device=device)
    remote[rank] = False
    N_remote = int(((sp >= 0) & remote[None, :]).sum().item())
    bd, bc = shard_bytes(R, T, H, K, N)

    a = torch.cuda.Event(enable_timing=True)
    b = torch.cuda.Event(enable_timing=True)

    def timed(run) -> float:
        barrier(device)
        torch.cuda.synchronize(device)
        a.record(stream)
        for _ in range(args.steps):
            run()
        b.record(stream)
        torch.cuda.synchronize(device)
        barrier(device)
        return a.elapsed_time(b) / args.steps

    eager_ms = timed(step)
    # the whole step -- kernels and NCCL collectives -- captured once and
    # replayed, so that host launch overhead does not pace the GPUs
    graph, graph_note = None, None
    try:
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            step()
        torch.cuda.synchronize(device)
        graph = g
    except Exception as e:  # capture refused: time the eager step only
        graph_note = f"capture failed: {type(e).__name__}: {str(e)[:200]}"
        torch.cuda.synchronize(device)
    sampler = ClockSampler(local)
    sampler.start()
    time.sleep(0.3)
    ms_local = timed(graph.replay) if graph is not None else eager_ms
    clocks = sampler.stop()
    agg = aggregate(bd + bc, T, ms_local, device)
    eager = aggregate(bd + bc, T, eager_ms, device)
    if int(buf.status.item()) != 0:
        raise RuntimeError(f"device status {int(buf.status.item())} in the timed region")
    # rows crossing NVLink per step (each way): copies to other ranks, then read back
    link = reduce_max(N_remote * H * 2 * 2, device)

    # end to end: this step's inputs up from pinned host memory, its result down
    x_h = torch.from_numpy(inp["x"][0].view(np.int16)).view(torch.bfloat16).pin_memory()
    idx_h = torch.from_numpy(inp["topk_idx"][0]).pin_memory()
    w_h = torch.from_numpy(inp["topk_weights"][0]).pin_memory()
    cx_h = torch.empty((T, H), dtype=torch.bfloat16).pin_memory()
    e2e_steps = max(3, min(args.steps, 20))
    barrier(device)
    torch.cuda.synchronize(device)
    a.record(stream)
    for _ in range(e2e_steps):
        x.copy_(x_h, non_blocking=True)
        idx.copy_(idx_h, non_blocking=True)
        wt.copy_(w_h, non_blocking=True)
        step()
        cx_h.copy_(cx, non_blocking=True)
    b.record(stream)
    torch.cuda.synchronize(device)
    barrier(device)
    e2e = aggregate(bd + bc, T, a.elapsed_time(b) / e2e_steps, device)
    h2d = x_h.numel() * 2 + idx_h.numel() * 8 + w_h.numel() * 4
    probe = buf.notify_probe.cpu().numpy().astype(np.uint64)
    starts = [None] * ws
    dist.all_gather_object(starts, int(probe[2]))
    low_latency = sharded_ll(args, device, rank, ws, timed)

    line = {
        "metric": METRIC, "value": agg["gbs"], "unit": UNIT, "n_gpus": ws, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": agg["ms_per_step"], "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "mode": "sharded",
        "config": {"workload": f"normal, one rank per GPU: R={R} ranks x T={T} tokens x H={H} "
                               f"bf16, E={E} experts, top-{K} distinct uniform, fp32 softmax "
                               "weights, identity experts",
                   "global_batch": R * T, "seq_len": None,
                   "parallelism": f"ep{R} (one rank per GPU, peer stores over NVLink)",
                   "l2": "inputs larger than L2; no flush"},
        "tokens_per_s": agg["tokens_per_s"],
        "pct_of_8TBps": 100.0 * agg["gbs"] / (SPEC_HBM_GBS * ws),
        "nvlink_bytes_per_step_per_gpu": link,
        "nvlink_gbs_per_gpu": link / (agg["ms_per_step"] * 1e-3) / 1e9,
        "notify_probe": {"launches": int(probe[1]),
                         "mean_full_grid_us": float(probe[0]) / max(int(probe[1]), 1) / 1e3,
                         "arrival_skew_us": (max(starts) - min(starts)) / 1e3},
        "e2e": {"value": e2e["gbs"], "unit": UNIT, "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": cx_h.numel() * 2, "ms_per_step": e2e["ms_per_step"]},
        "gpu_launches": 7 * args.steps,   # layout, zeroing, prefix, scan, pad, copy, combine per step
        "cuda_graph": graph is not None, "cuda_graph_note": graph_note,
        "eager": {"ms_per_step": eager["ms_per_step"], "value": eager["gbs"]},
        "clocks": clocks,
        "low_latency": low_latency,
    }
    if rank == 0:
        print(json.dumps(line), flush=True)
    del graph
    torch.cuda.synchronize(device)
    buf.close()
    dist.destroy_process_group()


# ---------------------------------------------------------------------------
# profiling cases: one entry point of the path, looped, on a named workload
# ---------------------------------------------------------------------------

# Sized for ncu captures: the "_small" and "_scan" cases hold at most ~2 GB on
# the device (inputs still larger than L2 where the kernel streams rows); the
# full-size cases are for the single-pass launch list only.
PROFILE_CASES = {
    "notify_normal": (Workload("normal_routing", R=8, T=4096, H=0, E=256, K=8), "notify"),
    "notify_skewed": (Workload("skewed_routing", R=16, T=2048, H=0, E=128, K=6, routing="zipf",
                               zipf_s=1.2, masked_frac=0.1), "notify"),
    "layout": (CONFIGS["layout"], "layout"),
    "copy_normal_small": (Workload("normal_small", R=8, T=1536, H=7168, E=256, K=8), "copy"),
    "combine_normal_small": (Workload("normal_small", R=8, T=1536, H=7168, E=256, K=8),
                             "combine"),
    "step_skewed_small": (Workload("skewed_small", R=16, T=1024, H=4096, E=128, K=6,
                                   routing="zipf", zipf_s=1.2, masked_frac=0.1), "step"),
    "step_skewed": (CONFIGS["skewed"], "step"),
    "ll_dispatch_small": (Workload("ll_small", R=8, T=512, H=7168, E=64, K=8), "ll_dispatch"),
    "ll_scan": (Workload("ll_routing", R=32, T=128, H=128, E=256, K=8), "ll_dispatch"),
    "ll_dispatch": (CONFIGS["ll"], "ll_dispatch"),
    "ll_combine_small": (Workload("ll_small", R=8, T=256, H=7168, E=64, K=8), "ll_combine"),
}


def run_profile(args) -> None:
    """Loop one entry point on a PROFILE_CASES workload (warm-up, then
    --steps calls) and print its mean time per call as one JSON line."""
    import dataclasses

    import torch

    import combine_get_dispatch_06_b200 as ep

    w, what = PROFILE_CASES[args.profile]
    device = torch.device("cuda", 0)
    torch.cuda.set_device(device)
    inp = make(w)
    R, T, H, E, K = w.R, w.T, w.H, w.E, w.K
    idx = torch.from_numpy(inp["topk_idx"]).to(device)
    wt = torch.from_numpy(inp["topk_weights"]).to(device)
    x = to_dev_bf16(inp["x"], device) if "x" in inp else None
    status = ep.new_status(device)
    stream = torch.cuda.current_stream(device)
    if what == "layout":
        idx1 = idx[0]
        o = ep.ep_get_dispatch_layout(idx1, E, R, status=status)

        def call():
            ep.ep_get_dispatch_layout(idx1, E, R, num_tokens_per_rank=o[0],
                                      num_tokens_per_expert=o[1], is_token_in_rank=o[2],
                                      status=status)
    elif what in ("notify", "copy", "combine", "step"):
        out, cx, cw, wsp, _ = step_buffers(R, T, max(H, 8), E, K, device)
        ep.ep_notify_dispatch(idx, wt, T, R, E, with_layout=True, out=out, workspace=wsp,
                              status=status)
        if x is not None:
            ep.ep_dispatch_cached(x, out["send_pos"], recv_x=out["recv_x"], status=status)
        io = {"x": x, "idx": idx, "wt": wt, "cx": cx, "cw": cw}

        def call():
            if what == "notify":
                ep.ep_notify_dispatch(idx, wt, T, R, E, with_layout=True, out=out,
                                      workspace=wsp, status=status)
            elif what == "copy":
                ep.ep_dispatch_cached(x, out["send_pos"], recv_x=out["recv_x"], status=status)
            elif what == "combine":
                ep.ep_combine(out["recv_x"], out["send_pos"], out["recv_topk_weights"],
                              combined_x=cx, combined_topk_weights=cw, status=status)
            else:
                routing_step(ep, io, out, wsp, status, R, T, E, stream)
    elif what in ("ll_dispatch", "ll_combine"):
        ws = torch.empty(ep.ep_ll_workspace_bytes(R, T, E), dtype=torch.uint8, device=device)
        d = ep.ep_ll_dispatch(x, idx, E, use_fp8=True, workspace=ws, status=status)
        if what == "ll_combine":
            del d["recv_x"], d["recv_scales"]
            g = torch.Generator(device=device).manual_seed(1)
            y = torch.randn((R, E // R, R * T, H), generator=g, device=device,
                            dtype=torch.bfloat16)
            out_c = torch.empty((R, T, H), dtype=torch.bfloat16, device=device)

            def call():
                ep.ep_ll_combine(y, idx, wt, d["ll_pos"], out=out_c, status=status)
        else:
            def call():
                ep.ep_ll_dispatch(x, idx, E, use_fp8=True, out=d, workspace=ws, status=status)
    else:
        raise ValueError(what)
    for _ in range(args.warmup):
        call()
    torch.cuda.synchronize(device)
    a = torch.cuda.Event(enable_timing=True)
    b = torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for _ in range(args.steps):
        call()
    b.record(stream)
    torch.cuda.synchronize(device)
    if int(status.item()) != 0:
        raise RuntimeError(f"device status {int(status.item())}")
    print(json.dumps({"profile": args.profile, "entry": what,
                      "us_per_call": a.elapsed_time(b) / args.steps * 1e3,
                      "steps": args.steps, "warmup": args.warmup,
                      "workload": dataclasses.asdict(w)}), flush=True)


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.splitlines()[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-extra", action="store_true")
    ap.add_argument("--tokens", type=int, default=None,
                    help="tokens per source rank (default 4096; smaller only for profiling)")
    ap.add_argument("--mode", choices=["replicas", "sharded"], default="replicas",
                    help="N > 1: independent single-GPU replicas (default), or one routing "
                         "rank per GPU over NVLink")
    ap.add_argument("--profile", choices=sorted(PROFILE_CASES), default=None,
                    help="loop one entry point on a named small workload (for ncu captures)")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        args.warmup = 3
    if args.profile is not None:
        run_profile(args)
    elif args.impl == "reference":
        run_reference(args)
    elif args.mode == "sharded":
        run_sharded(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
