"""The benchmark's algorithmic byte counts, on the CPU: the number of copies N
of the seeded normal workload comes from the oracle's layout, and the byte
formulas are the per-unit figures of the measurement plan (x read once, each
copy written once, metadata per slot and per copy)."""
import os
import sys

import numpy as np

import oracle
from workloads import CONFIGS, make

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402


def test_normal_workload_copies_and_bytes():
    w = CONFIGS["normal"]
    inp = make(w, with_x=False)
    lay = oracle.layout(inp["topk_idx"], w.E, w.R)
    N = int(lay["is_token_in_rank"].sum())
    # E[n_dest] = R * (1 - C(E - E_l, K) / C(E, K)) = 5.295 for 8 ranks, top-8 of 256
    assert abs(N / (w.R * w.T) - 5.295) < 0.02
    R, T, H, K = w.R, w.T, w.H, w.K
    d = bench.dispatch_bytes(R, T, H, K, N)
    c = bench.combine_bytes(R, T, H, K, N)
    rows = R * T * H * 2 + N * H * 2          # the data movement itself
    assert d - rows == R * T * K * 12 + N * (K * 12 + 4) + R * T * K * 8 + 2 * R * T * R + R * T * R * 4
    assert c - rows == N * K * 4 + R * T * K * 4 + R * T * R * 4
    # the row traffic dominates: metadata is under 1% of each direction
    assert (d - rows) / d < 0.01 and (c - rows) / c < 0.01
    # the roofline kernel's algorithmic bytes (rows only) at the 8 TB/s spec
    assert abs(rows / 8e12 * 1e6 - 369.4) < 1.0


def test_low_latency_bytes():
    w = CONFIGS["ll"]
    inp = make(w, with_x=False)
    C = int((inp["topk_idx"] >= 0).sum())   # distinct experts per token: one copy per slot
    assert C == w.R * w.T * w.K
    b = bench.ll_dispatch_bytes(w.R, w.T, w.H, w.K, C)
    # bf16 rows read once, e4m3 rows + one fp32 scale per 128 channels written per copy
    assert b >= w.R * w.T * w.H * 2 + C * (w.H + w.H // 128 * 4)
    assert bench.ll_combine_bytes(w.R, w.T, w.H, w.K, C) >= C * w.H * 2 + w.R * w.T * w.H * 2


def test_expected_copies_closed_form():
    """The 5.295 used above: probability that a token hits a given rank when K
    distinct experts are drawn uniformly from E, E_l per rank."""
    from math import comb
    R, E, K = 8, 256, 8
    El = E // R
    p_hit = 1 - comb(E - El, K) / comb(E, K)
    assert abs(R * p_hit - 5.295) < 0.001
    # and the sampled workload agrees with it at the configuration's size
    w = CONFIGS["normal"]
    idx = make(w, with_x=False)["topk_idx"]
    ranks = idx // (w.E // w.R)
    hits = np.zeros((w.R, w.T, w.R), bool)
    for k in range(w.K):
        np.put_along_axis(hits, ranks[..., k:k + 1], True, axis=2)
    assert abs(hits.sum(axis=2).mean() - R * p_hit) < 0.02
