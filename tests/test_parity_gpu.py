"""Parity of the CUDA path (through the C ABI) with the CPU oracle.

Integer and byte outputs must match bit for bit; the fp32-accumulated outputs
(combine, low-latency combine) must match bit for bit as well, because both
sides sum in the same order with the same IEEE operations -- the method's
tolerance (<= 1 bf16 ulp) is checked too, as a looser second line.
"""
import numpy as np
import pytest
import torch

import oracle
from workloads import CONFIGS, Workload, make
from tests.helpers import b2f, to_dev, to_host

pytestmark = pytest.mark.gpu

ep = None


def setup_module(module):
    global ep
    import combine_get_dispatch_06_b200 as _ep
    ep = _ep
    ep.ep_set_debug_flags(0)
    ep.ep_set_wait_timeout_ns(10**9)


def ulp_diff_bf16(a_bits, b_bits):
    """Distance in bf16 ulps between two arrays of finite bf16 patterns."""
    def key(b):
        b = b.astype(np.int32)
        return np.where(b & 0x8000, -(b & 0x7FFF), b)
    return np.abs(key(a_bits) - key(b_bits))


# ---------------------------------------------------------------------------
# A1 layout
# ---------------------------------------------------------------------------

LAYOUT_CASES = [
    ("pr1", CONFIGS["pr1"]),
    ("layout_4096x8", CONFIGS["layout"]),
    ("skewed", CONFIGS["skewed"]),
    ("ragged", Workload("ragged", R=5, T=301, H=0, E=40, K=3, masked_frac=0.2, seed=3)),
    ("one_token", Workload("one", R=3, T=1, H=0, E=6, K=2)),
    ("k1_el1", Workload("k1", R=8, T=200, H=0, E=8, K=1, seed=5)),
    ("r64", Workload("r64", R=64, T=130, H=0, E=128, K=8, seed=7)),
    ("r384", Workload("r384", R=384, T=3, H=0, E=384, K=16, seed=9)),
    ("e512_k16", Workload("e512", R=16, T=257, H=0, E=512, K=16, seed=11)),
    # experts per rank not a power of two (the expert -> rank division)
    ("el7", Workload("el7", R=6, T=200, H=0, E=42, K=5, seed=13)),
    ("el511", Workload("el511", R=1, T=150, H=0, E=511, K=9, seed=15)),
    # past one 8-CTA cluster per source rank (4096 tokens): the tile kernel
    ("t5000_tiles", Workload("t5k", R=8, T=5000, H=0, E=64, K=6, masked_frac=0.05, seed=17)),
    ("r33_tiles", Workload("r33", R=33, T=300, H=0, E=66, K=4, seed=18)),
]


@pytest.mark.parametrize("name,w", LAYOUT_CASES, ids=[c[0] for c in LAYOUT_CASES])
def test_layout_parity(name, w):
    inp = make(w, with_x=False)
    idx = inp["topk_idx"]
    ref = oracle.layout(idx, w.E, w.R)
    st = ep.new_status()
    ntpr, ntpe, inr = ep.ep_get_dispatch_layout(to_dev(idx), w.E, w.R, status=st)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(to_host(ntpr), ref["num_tokens_per_rank"])
    np.testing.assert_array_equal(to_host(ntpe), ref["num_tokens_per_expert"])
    np.testing.assert_array_equal(to_host(inr), ref["is_token_in_rank"])
    assert int(st.item()) == 0


@pytest.mark.parametrize("T", [150, 4200], ids=["cluster", "tiles"])
def test_layout_bad_ids_and_duplicates(T):
    rng = np.random.default_rng(1)
    R, K, E = 4, 4, 16
    idx = rng.integers(0, E, size=(R, T, K)).astype(np.int64)
    idx[:, ::7, 1] = idx[:, ::7, 0]          # repeated experts
    idx[:, ::5, 2] = -1
    idx[1, 3, 3] = E                          # invalid ids
    idx[2, 9, 0] = -4
    ref = oracle.layout(idx, E, R)
    st = ep.new_status()
    ntpr, ntpe, inr = ep.ep_get_dispatch_layout(to_dev(idx), E, R, status=st)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(to_host(ntpr), ref["num_tokens_per_rank"])
    np.testing.assert_array_equal(to_host(ntpe), ref["num_tokens_per_expert"])
    np.testing.assert_array_equal(to_host(inr), ref["is_token_in_rank"])
    assert int(st.item()) & ep.EP_STATUS_BAD_EXPERT


def test_layout_empty():
    idx = torch.empty((2, 0, 4), dtype=torch.int64, device="cuda")
    ntpr, ntpe, inr = ep.ep_get_dispatch_layout(idx, 8, 2)
    torch.cuda.synchronize()
    assert (to_host(ntpr) == 0).all() and (to_host(ntpe) == 0).all() and inr.numel() == 0


# ---------------------------------------------------------------------------
# A2 + A3 + A4: full element-wise parity at oracle-friendly sizes
# ---------------------------------------------------------------------------

def check_dispatch(out, ref, R, K, with_meta=True):
    rc = ref["recv_count"]
    np.testing.assert_array_equal(to_host(out["recv_count"]), rc)
    np.testing.assert_array_equal(to_host(out["rank_prefix_matrix"]), ref["rank_prefix_matrix"])
    np.testing.assert_array_equal(to_host(out["send_pos"]), ref["send_pos"])
    cap = out["recv_x"].shape[1]
    rx = to_host(out["recv_x"])
    rsi = to_host(out["recv_src_idx"])
    for d in range(R):
        n = min(int(rc[d]), cap)
        np.testing.assert_array_equal(rx[d, :n], ref["recv_x"][d, :n])
        np.testing.assert_array_equal(rsi[d, :n], ref["recv_src_idx"][d, :n])
    if with_meta:
        ri = to_host(out["recv_topk_idx"])
        rw = to_host(out["recv_topk_weights"])
        for d in range(R):
            n = min(int(rc[d]), cap)
            np.testing.assert_array_equal(ri[d, :n], ref["recv_topk_idx"][d, :n])
            np.testing.assert_array_equal(rw[d, :n], ref["recv_topk_weights"][d, :n])
        np.testing.assert_array_equal(to_host(out["num_recv_tokens_per_expert"]),
                                      ref["num_recv_tokens_per_expert"])


PARITY_CASES = [
    ("pr1", CONFIGS["pr1"], 1),
    ("ragged_tiles", Workload("rt", R=4, T=300, H=264, E=16, K=3, masked_frac=0.15, seed=1), 1),
    ("align8", Workload("a8", R=6, T=129, H=128, E=24, K=4, seed=2), 8),
    ("skew_small", Workload("sk", R=16, T=140, H=256, E=128, K=6, routing="zipf",
                            masked_frac=0.1, seed=4), 1),
    ("r64_multiwarp", Workload("r64", R=64, T=40, H=64, E=128, K=8, seed=6), 1),
    ("k1", Workload("k1", R=3, T=257, H=8, E=3, K=1, seed=8), 1),
    ("big_row_chunks", Workload("br", R=3, T=70, H=12288, E=12, K=3, seed=10), 1),
    ("el3_align4", Workload("e3", R=5, T=150, H=64, E=15, K=4, masked_frac=0.05, seed=14), 4),
    # the largest rank count (12 warps per copy CTA, 384-bit routing masks)
    ("r384_max", Workload("r384", R=384, T=3, H=64, E=384, K=4, seed=16), 1),
    # one and two ranks: a tile's predecessors hold a number of counts that is
    # not a multiple of four (the look-back's last group is partly past the end)
    ("r1_tiles", Workload("r1", R=1, T=700, H=64, E=8, K=3, seed=19), 1),
    ("r2_tiles", Workload("r2", R=2, T=650, H=64, E=10, K=4, masked_frac=0.05, seed=20), 1),
    # seven slots on eight ranks: just past the bound for combine's 6-row shape
    ("k7_r8", Workload("k7", R=8, T=300, H=136, E=32, K=7, masked_frac=0.05, seed=23), 1),
]


@pytest.mark.parametrize("name,w,align", PARITY_CASES, ids=[c[0] for c in PARITY_CASES])
def test_dispatch_combine_parity(name, w, align):
    inp = make(w)
    x, idx, wts = inp["x"], inp["topk_idx"], inp["topk_weights"]
    ref = oracle.normal_path(x, idx, wts, w.E, alignment=align)
    st = ep.new_status()
    xd, idd, wd = to_dev(x), to_dev(idx), to_dev(wts)
    # the pages' sequence: get_dispatch_layout, then dispatch with the layout
    _, _, inr = ep.ep_get_dispatch_layout(idd, w.E, w.R, status=st)
    out = ep.ep_dispatch(xd, idd, wd, w.E, is_token_in_rank=inr, expert_alignment=align,
                         status=st)
    cx, cw = ep.ep_combine(out["recv_x"], out["send_pos"], out["recv_topk_weights"], status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    check_dispatch(out, ref, w.R, w.K)
    np.testing.assert_array_equal(to_host(cx), ref["combined_x"])
    np.testing.assert_array_equal(to_host(cw), ref["combined_topk_weights"])

    # routing computed inside ep_dispatch (no layout given) gives the same
    out2 = ep.ep_dispatch(xd, idd, wd, w.E, expert_alignment=align, status=st)
    torch.cuda.synchronize()
    check_dispatch(out2, ref, w.R, w.K)

    # combine of random expert outputs: bit-exact with the oracle and within
    # 1 bf16 ulp of it (the method's bound)
    g = torch.Generator(device="cuda").manual_seed(5)
    y = torch.randn(out["recv_x"].shape, generator=g, device="cuda").to(torch.bfloat16)
    cy, _ = ep.ep_combine(y, out["send_pos"], status=st)
    ry, _ = oracle.combine(to_host(y), ref["send_pos"])
    torch.cuda.synchronize()
    got = to_host(cy)
    assert ulp_diff_bf16(got, ry).max() <= 1
    np.testing.assert_array_equal(got, ry)


def test_dispatch_from_is_token_in_rank_only():
    """with_topk=False path: routing from a given is_token_in_rank that is not
    derived from any top-k choice; no metadata."""
    rng = np.random.default_rng(21)
    R, T, H = 5, 333, 136
    inr = (rng.random((R, T, R)) < 0.4).astype(np.uint8)
    inr[:, 7] = 0           # tokens with no destination
    inr[:, 8] = 1           # tokens to every rank
    x = make(Workload("x", R=R, T=T, H=H, E=R, K=1, seed=22))["x"]
    pre = oracle.prefix(inr)
    rx = oracle.dispatch_rows(x, pre["send_pos"])
    st = ep.new_status()
    out = ep.ep_dispatch(to_dev(x), None, None, R, is_token_in_rank=to_dev(inr).bool(),
                         status=st)
    cx, _ = ep.ep_combine(out["recv_x"], out["send_pos"])
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    ref = dict(pre)
    ref["recv_x"] = rx
    check_dispatch(out, ref, R, 1, with_meta=False)
    rc, _ = oracle.combine(rx, pre["send_pos"])
    np.testing.assert_array_equal(to_host(cx), rc)
    assert (b2f(to_host(cx))[:, 7] == 0).all()


def test_capacity_overflow_reports_and_stays_in_bounds():
    w = Workload("ovf", R=4, T=200, H=64, E=8, K=2, routing="zipf", seed=3)
    inp = make(w)
    x, idx, wts = inp["x"], inp["topk_idx"], inp["topk_weights"]
    full = oracle.normal_path(x, idx, wts, w.E)
    cap = int(full["recv_count"].max()) - 50
    assert cap > 0
    ref = oracle.normal_path(x, idx, wts, w.E, cap=cap)
    st = ep.new_status()
    # guard elements after the receive buffer: must stay untouched
    n = w.R * cap * w.H
    big = torch.zeros(n + 64 * w.H, dtype=torch.bfloat16, device="cuda")
    recv = big[:n].view(w.R, cap, w.H)
    out = ep.ep_dispatch(to_dev(x), to_dev(idx), to_dev(wts), w.E, capacity=cap,
                         out={"recv_x": recv}, status=st)
    torch.cuda.synchronize()
    assert int(st.item()) & ep.EP_STATUS_CAPACITY
    check_dispatch(out, ref, w.R, w.K)
    assert (to_host(big[n:]) == 0).all()
    st2 = ep.new_status()
    cx, _ = ep.ep_combine(out["recv_x"], out["send_pos"], status=st2)
    rc, _ = oracle.combine(to_host(out["recv_x"]), ref["send_pos"])
    torch.cuda.synchronize()
    assert int(st2.item()) & ep.EP_STATUS_BAD_POSITION
    np.testing.assert_array_equal(to_host(cx), rc)


def test_dispatch_empty_tokens():
    R, H, E, K = 4, 64, 8, 2
    x = torch.empty((R, 0, H), dtype=torch.bfloat16, device="cuda")
    idx = torch.empty((R, 0, K), dtype=torch.int64, device="cuda")
    w = torch.empty((R, 0, K), dtype=torch.float32, device="cuda")
    out = ep.ep_dispatch(x, idx, w, E, capacity=0)
    cx, cw = ep.ep_combine(out["recv_x"], out["send_pos"], out["recv_topk_weights"])
    torch.cuda.synchronize()
    assert (to_host(out["recv_count"]) == 0).all()
    assert (to_host(out["rank_prefix_matrix"]) == 0).all()
    assert (to_host(out["num_recv_tokens_per_expert"]) == 0).all()
    assert cx.numel() == 0


def test_determinism_hash():
    w = Workload("det", R=8, T=512, H=512, E=64, K=8, seed=12)
    inp = make(w)
    xd, idd, wd = to_dev(inp["x"]), to_dev(inp["topk_idx"]), to_dev(inp["topk_weights"])
    hashes = []
    for _ in range(3):
        out = ep.ep_dispatch(xd, idd, wd, w.E)
        cx, cw = ep.ep_combine(out["recv_x"], out["send_pos"], out["recv_topk_weights"])
        torch.cuda.synchronize()
        # rows past recv_count are never written (fresh, uninitialised
        # buffers each call), so only the written rows enter the hash
        rc = to_host(out["recv_count"])
        rx = to_host(out["recv_x"])
        rows = b"".join(rx[d, :rc[d]].tobytes() for d in range(w.R))
        h = (to_host(out["send_pos"]).tobytes(), to_host(cx).tobytes(), to_host(cw).tobytes(),
             rows)
        hashes.append(hash(h))
    assert len(set(hashes)) == 1


def test_lookback_timeout_is_reported_and_recoverable():
    """Failure detection without a GPU fault: scan tiles stop publishing, so
    every look-back wait runs out after its limit; the status word reports it,
    every store stays in bounds, and the next normal call is correct."""
    w = Workload("to", R=4, T=600, H=128, E=16, K=2, seed=13)
    inp = make(w)
    xd, idd, wd = to_dev(inp["x"]), to_dev(inp["topk_idx"]), to_dev(inp["topk_weights"])
    st = ep.new_status()
    try:
        ep.ep_set_wait_timeout_ns(2_000_000)   # 2 ms
        ep.ep_set_debug_flags(ep.EP_DEBUG_SUPPRESS_PUBLISH)
        out = ep.ep_dispatch(xd, idd, wd, w.E, status=st)
        ll = ep.ep_ll_dispatch(xd, idd, w.E, use_fp8=True, status=st)
        torch.cuda.synchronize()
    finally:
        ep.ep_set_debug_flags(0)
        ep.ep_set_wait_timeout_ns(10**9)
    assert int(st.item()) & ep.EP_STATUS_WAIT_TIMEOUT
    st2 = ep.new_status()
    ref = oracle.normal_path(inp["x"], inp["topk_idx"], inp["topk_weights"], w.E)
    out = ep.ep_dispatch(xd, idd, wd, w.E, status=st2)
    torch.cuda.synchronize()
    assert int(st2.item()) == 0
    check_dispatch(out, ref, w.R, w.K)


# ---------------------------------------------------------------------------
# A5 + A6 low latency
# ---------------------------------------------------------------------------

LL_CASES = [
    ("small_fp8", Workload("l1", R=4, T=150, H=384, E=16, K=4, masked_frac=0.1, seed=1), True),
    ("small_bf16", Workload("l2", R=4, T=150, H=392, E=16, K=4, masked_frac=0.1, seed=2), False),
    ("h128_halfwarp", Workload("l3", R=3, T=40, H=128, E=9, K=3, seed=3), True),
    ("h640_scales_unaligned", Workload("l4", R=2, T=130, H=640, E=8, K=2, seed=4), True),
    ("pr1_shape", Workload("l5", R=4, T=64, H=256, E=16, K=2, seed=0), True),
    # 96 scan tiles (6 per source) against ~440 dispatch CTAs: most tokens'
    # rows are read while the scan that writes their positions still runs
    ("many_tiles", Workload("l6", R=16, T=700, H=256, E=64, K=8, masked_frac=0.05, seed=6), True),
]


def _dup_slots(idx, frac, seed):
    rng = np.random.default_rng(seed)
    idx = idx.copy()
    if idx.shape[2] > 1:
        m = rng.random(idx.shape[:2]) < frac
        idx[..., 1][m] = idx[..., 0][m]
    return idx


@pytest.mark.parametrize("name,w,fp8", LL_CASES, ids=[c[0] for c in LL_CASES])
def test_ll_parity(name, w, fp8):
    inp = make(w)
    x, wts = inp["x"], inp["topk_weights"]
    idx = _dup_slots(inp["topk_idx"], 0.1, w.seed)
    R, T, H, E = w.R, w.T, w.H, w.E
    El = E // R
    ref = oracle.ll_layout(idx, E)
    rq, rs = oracle.ll_dispatch_rows(x, idx, ref["ll_pos"], E, use_fp8=fp8)
    st = ep.new_status()
    xd, idd, wd = to_dev(x), to_dev(idx), to_dev(wts)
    out = ep.ep_ll_dispatch(xd, idd, E, use_fp8=fp8, status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    np.testing.assert_array_equal(to_host(out["recv_count"]), ref["recv_count"])
    np.testing.assert_array_equal(to_host(out["layout_range"]), ref["layout_range"])
    np.testing.assert_array_equal(to_host(out["ll_pos"]), ref["ll_pos"])
    q = to_host(out["recv_x"])
    rsi = to_host(out["recv_src_info"])
    sc = to_host(out["recv_scales"]) if fp8 else None
    for d in range(R):
        for j in range(El):
            n = ref["recv_count"][d, j]
            np.testing.assert_array_equal(rsi[d, j, :n], ref["recv_src_info"][d, j, :n])
            np.testing.assert_array_equal(q[d, j, :n], rq[d, j, :n])
            if fp8:
                np.testing.assert_array_equal(sc[d, j, :n], rs[d, j, :n])
    # combine: experts return the (dequantised) received rows; oracle-built input
    y = oracle.dequant_rows(rq, rs) if fp8 else rq
    ro = oracle.ll_combine(y, idx, wts, ref["ll_pos"])
    co = ep.ep_ll_combine(to_dev(y), idd, wd, out["ll_pos"], status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    got = to_host(co)
    assert ulp_diff_bf16(got, ro).max() <= 1
    np.testing.assert_array_equal(got, ro)


# ---------------------------------------------------------------------------
# cached mode and the fixed worst-case receive capacity
# ---------------------------------------------------------------------------

def test_cached_dispatch_replays_the_handle():
    """Re-dispatching with the handle reproduces recv_x; a new payload goes to
    the same rows (legacy-test analysis page, cached dispatch check)."""
    w = Workload("cache", R=6, T=300, H=136, E=24, K=4, masked_frac=0.1, seed=41)
    inp = make(w)
    xd, idd, wd = to_dev(inp["x"]), to_dev(inp["topk_idx"]), to_dev(inp["topk_weights"])
    st = ep.new_status()
    out = ep.ep_dispatch(xd, idd, wd, w.E, status=st)
    first = out["recv_x"].clone()
    again = ep.ep_dispatch_cached(xd, out["send_pos"], status=st)
    x2 = make(Workload("cache2", R=6, T=300, H=136, E=24, K=4, seed=42))["x"]
    other = ep.ep_dispatch_cached(to_dev(x2), out["send_pos"], status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    rc = to_host(out["recv_count"])
    for d in range(w.R):
        assert torch.equal(again[d, :rc[d]].view(torch.int16), first[d, :rc[d]].view(torch.int16))
    ref2 = oracle.dispatch_rows(x2, to_host(out["send_pos"]))
    got2 = to_host(other)
    for d in range(w.R):
        np.testing.assert_array_equal(got2[d, :rc[d]], ref2[d, :rc[d]])


def test_notify_then_cached_equals_dispatch():
    w = Workload("split", R=8, T=260, H=256, E=64, K=8, seed=43)
    inp = make(w)
    xd, idd, wd = to_dev(inp["x"]), to_dev(inp["topk_idx"]), to_dev(inp["topk_weights"])
    ref = ep.ep_dispatch(xd, idd, wd, w.E, expert_alignment=2)
    h = ep.ep_notify_dispatch(idd, wd, w.T, w.R, w.E, expert_alignment=2)
    rx = ep.ep_dispatch_cached(xd, h["send_pos"])
    torch.cuda.synchronize()
    for name in ("send_pos", "rank_prefix_matrix", "recv_count", "num_recv_tokens_per_expert"):
        assert torch.equal(h[name], ref[name]), name
    rc = to_host(ref["recv_count"])
    for d in range(w.R):
        n = rc[d]
        assert torch.equal(rx[d, :n].view(torch.int16), ref["recv_x"][d, :n].view(torch.int16))
        for name in ("recv_src_idx", "recv_topk_idx", "recv_topk_weights"):
            assert torch.equal(h[name][d, :n], ref[name][d, :n]), name


def test_worst_case_capacity_pads_recv_topk_idx():
    """Fixed capacity = the pages' num_worst_tokens mode: rows past the receive
    count hold recv_topk_idx == -1, and the real rows are the same as with an
    exactly sized buffer."""
    w = Workload("worst", R=4, T=200, H=64, E=16, K=3, seed=44)
    inp = make(w)
    xd, idd, wd = to_dev(inp["x"]), to_dev(inp["topk_idx"]), to_dev(inp["topk_weights"])
    ref = oracle.normal_path(inp["x"], inp["topk_idx"], inp["topk_weights"], w.E)
    exact = int(ref["recv_count"].max())
    small = ep.ep_dispatch(xd, idd, wd, w.E, capacity=exact)
    out = {"recv_topk_idx": torch.full((w.R, w.R * w.T, w.K), 7, dtype=torch.int64,
                                       device="cuda")}
    worst = ep.ep_dispatch(xd, idd, wd, w.E, out=out)
    torch.cuda.synchronize()
    rc = ref["recv_count"]
    ri = to_host(worst["recv_topk_idx"])
    for d in range(w.R):
        assert (ri[d, rc[d]:] == -1).all()
        np.testing.assert_array_equal(ri[d, :rc[d]], ref["recv_topk_idx"][d, :rc[d]])
        assert torch.equal(worst["recv_x"][d, :rc[d]].view(torch.int16),
                           small["recv_x"][d, :rc[d]].view(torch.int16))


# ---------------------------------------------------------------------------
# FP8 input to normal dispatch; combine with bias
# ---------------------------------------------------------------------------

FP8_CASES = [
    ("rowmajor_bulk", Workload("f1", R=4, T=300, H=512, E=16, K=3, seed=51), False),
    ("rowmajor_unaligned", Workload("f2", R=5, T=140, H=384, E=20, K=2, seed=52), False),
    ("colmajor", Workload("f3", R=4, T=257, H=512, E=8, K=2, seed=53), True),
    ("colmajor_7168", Workload("f4", R=3, T=130, H=7168, E=12, K=4, seed=54), True),
]


@pytest.mark.parametrize("name,w,colmaj", FP8_CASES, ids=[c[0] for c in FP8_CASES])
def test_fp8_input_dispatch(name, w, colmaj):
    inp = make(w)
    R, T, H = w.R, w.T, w.H
    nb = H // 128
    # realistic FP8 input: the oracle's per-token cast of the bf16 rows
    q = np.zeros((R, T, H), np.uint8)
    sc = np.zeros((R, T, nb), np.float32)
    for s in range(R):
        for t in range(T):
            q[s, t], sc[s, t] = oracle.quantize_row(inp["x"][s, t])
    sc_in = np.ascontiguousarray(sc.transpose(0, 2, 1)) if colmaj else sc
    idd = to_dev(inp["topk_idx"])
    h = ep.ep_notify_dispatch(idd, None, T, R, w.E)
    st = ep.new_status()
    rq, rs = ep.ep_dispatch_cached_fp8(to_dev(q), to_dev(sc_in), h["send_pos"],
                                       scales_col_major=colmaj, status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    sp = to_host(h["send_pos"])
    eq, es = oracle.dispatch_rows_fp8(q, sc_in, sp, col_major=colmaj)
    rc = to_host(h["recv_count"])
    gq, gs = to_host(rq), to_host(rs)
    for d in range(R):
        np.testing.assert_array_equal(gq[d, :rc[d]], eq[d, :rc[d]])
        np.testing.assert_array_equal(gs[d, :rc[d]], es[d, :rc[d]])


def test_combine_with_bias():
    w = Workload("bias", R=6, T=210, H=264, E=24, K=4, masked_frac=0.05, seed=55)
    inp = make(w)
    ref = oracle.normal_path(inp["x"], inp["topk_idx"], inp["topk_weights"], w.E)
    b = make(Workload("b", R=6, T=210, H=264, E=24, K=4, seed=56))["x"]
    b1 = make(Workload("b1", R=6, T=210, H=264, E=24, K=4, seed=57))["x"]
    out = ep.ep_dispatch(to_dev(inp["x"]), to_dev(inp["topk_idx"]), to_dev(inp["topk_weights"]),
                         w.E)
    st = ep.new_status()
    cx, _ = ep.ep_combine(out["recv_x"], out["send_pos"], bias=(to_dev(b), to_dev(b1)), status=st)
    c0, _ = ep.ep_combine(out["recv_x"], out["send_pos"], bias=(to_dev(b), None), status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    e2, _ = oracle.combine(ref["recv_x"], ref["send_pos"], bias=(b, b1))
    e1, _ = oracle.combine(ref["recv_x"], ref["send_pos"], bias=(b, None))
    np.testing.assert_array_equal(to_host(cx), e2)
    np.testing.assert_array_equal(to_host(c0), e1)


# ---------------------------------------------------------------------------
# low-latency variants: power-of-two / UE8M0 scales, failed ranks, statistics
# ---------------------------------------------------------------------------

RS_CASES = [
    ("h384_plain_scales", Workload("r1", R=4, T=70, H=384, E=16, K=4, seed=61)),
    ("h2048_bulk_ue8m0", Workload("r2", R=3, T=130, H=2048, E=12, K=3, seed=62)),
    ("h7168", Workload("r3", R=4, T=40, H=7168, E=16, K=4, seed=63)),
]


@pytest.mark.parametrize("ue8m0", [False, True])
@pytest.mark.parametrize("name,w", RS_CASES, ids=[c[0] for c in RS_CASES])
def test_ll_round_scale(name, w, ue8m0):
    inp = make(w)
    x, idx = inp["x"], inp["topk_idx"]
    R, T, H, E = w.R, w.T, w.H, w.E
    El = E // R
    ref = oracle.ll_layout(idx, E)
    st = ep.new_status()
    out = ep.ep_ll_dispatch(to_dev(x), to_dev(idx), E, use_fp8=True, round_scale=True,
                            use_ue8m0=ue8m0, status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    np.testing.assert_array_equal(to_host(out["ll_pos"]), ref["ll_pos"])
    q = to_host(out["recv_x"])
    sc = to_host(out["recv_scales"])
    for s in range(R):
        for t in range(T):
            qr, sr, ur = oracle.quantize_row_ex(x[s, t], round_scale=True)
            for k in range(w.K):
                e = int(idx[s, t, k])
                p = int(ref["ll_pos"][s, t, k])
                d, j = divmod(e, El)
                np.testing.assert_array_equal(q[d, j, p], qr)
                np.testing.assert_array_equal(sc[d, j, p], ur if ue8m0 else sr)


def test_ll_failed_ranks_and_cumulative_stats():
    w = Workload("mk", R=8, T=150, H=256, E=32, K=4, masked_frac=0.05, seed=64)
    inp = make(w)
    x, idx, wts = inp["x"], inp["topk_idx"], inp["topk_weights"]
    R, E = w.R, w.E
    mask = np.array([0, 1, 0, 0, 0, 1, 0, 0], np.int32)   # ranks 1 and 5 failed
    ref = oracle.ll_layout(idx, E, mask=mask)
    md = to_dev(mask)
    stats = torch.zeros((R, E // R), dtype=torch.int32, device="cuda")
    st = ep.new_status()
    xd, idd, wd = to_dev(x), to_dev(idx), to_dev(wts)
    for _ in range(2):
        out = ep.ep_ll_dispatch(xd, idd, E, use_fp8=False, rank_mask=md,
                                cumulative_local_expert_recv_stats=stats, status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    np.testing.assert_array_equal(to_host(out["recv_count"]), ref["recv_count"])
    np.testing.assert_array_equal(to_host(out["layout_range"]), ref["layout_range"])
    np.testing.assert_array_equal(to_host(out["ll_pos"]), ref["ll_pos"])
    np.testing.assert_array_equal(to_host(stats), 2 * ref["recv_count"])
    slab, _ = oracle.ll_dispatch_rows(x, idx, ref["ll_pos"], E, use_fp8=False)
    ro = oracle.ll_combine(slab, idx, wts, ref["ll_pos"], mask=mask)
    co = ep.ep_ll_combine(to_dev(slab), idd, wd, out["ll_pos"], rank_mask=md, status=st)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(to_host(co), ro)
    assert (to_host(co)[1] == 0).all() and (to_host(co)[5] == 0).all()


# ---------------------------------------------------------------------------
# limits of the ABI: K = 16, E = 512, R > 32 on every path, empty inputs
# ---------------------------------------------------------------------------

def test_dispatch_combine_k16_e512():
    w = Workload("lim", R=16, T=150, H=136, E=512, K=16, masked_frac=0.05, seed=71)
    inp = make(w)
    x, idx, wts = inp["x"], inp["topk_idx"], inp["topk_weights"]
    ref = oracle.normal_path(x, idx, wts, w.E, alignment=4)
    st = ep.new_status()
    out = ep.ep_dispatch(to_dev(x), to_dev(idx), to_dev(wts), w.E, expert_alignment=4, status=st)
    cx, cw = ep.ep_combine(out["recv_x"], out["send_pos"], out["recv_topk_weights"], status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    check_dispatch(out, ref, w.R, w.K)
    np.testing.assert_array_equal(to_host(cx), ref["combined_x"])
    np.testing.assert_array_equal(to_host(cw), ref["combined_topk_weights"])


def test_ll_windowed_lookback():
    """40 scan tiles x 512 experts is past the size at which a tile reads every
    predecessor's counts at once: the windowed decoupled look-back on 64-bit
    descriptors, five tiles per source (row counts added by atomics)."""
    w = Workload("llw", R=8, T=600, H=128, E=512, K=8, masked_frac=0.05, seed=76)
    inp = make(w)
    x = inp["x"]
    idx = _dup_slots(inp["topk_idx"], 0.1, w.seed)
    R, E = w.R, w.E
    El = E // R
    ref = oracle.ll_layout(idx, E)
    rq, rs = oracle.ll_dispatch_rows(x, idx, ref["ll_pos"], E, use_fp8=True)
    st = ep.new_status()
    out = ep.ep_ll_dispatch(to_dev(x), to_dev(idx), E, use_fp8=True, status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    np.testing.assert_array_equal(to_host(out["recv_count"]), ref["recv_count"])
    np.testing.assert_array_equal(to_host(out["layout_range"]), ref["layout_range"])
    np.testing.assert_array_equal(to_host(out["ll_pos"]), ref["ll_pos"])
    q = to_host(out["recv_x"])
    rsi = to_host(out["recv_src_info"])
    sc = to_host(out["recv_scales"])
    for d in range(R):
        for j in range(El):
            n = ref["recv_count"][d, j]
            np.testing.assert_array_equal(rsi[d, j, :n], ref["recv_src_info"][d, j, :n])
            np.testing.assert_array_equal(q[d, j, :n], rq[d, j, :n])
            np.testing.assert_array_equal(sc[d, j, :n], rs[d, j, :n])


def test_ll_k16_e512():
    w = Workload("llim", R=8, T=70, H=256, E=512, K=16, masked_frac=0.05, seed=72)
    inp = make(w)
    x, idx, wts = inp["x"], _dup_slots(inp["topk_idx"], 0.2, 72), inp["topk_weights"]
    ref = oracle.ll_layout(idx, w.E)
    rq, rs = oracle.ll_dispatch_rows(x, idx, ref["ll_pos"], w.E, use_fp8=True)
    st = ep.new_status()
    idd = to_dev(idx)
    out = ep.ep_ll_dispatch(to_dev(x), idd, w.E, use_fp8=True, status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    np.testing.assert_array_equal(to_host(out["ll_pos"]), ref["ll_pos"])
    np.testing.assert_array_equal(to_host(out["recv_count"]), ref["recv_count"])
    np.testing.assert_array_equal(to_host(out["layout_range"]), ref["layout_range"])
    q, sc = to_host(out["recv_x"]), to_host(out["recv_scales"])
    El = w.E // w.R
    for d in range(w.R):
        for j in range(El):
            n = ref["recv_count"][d, j]
            np.testing.assert_array_equal(q[d, j, :n], rq[d, j, :n])
            np.testing.assert_array_equal(sc[d, j, :n], rs[d, j, :n])
    y = oracle.dequant_rows(rq, rs)
    co = ep.ep_ll_combine(to_dev(y), idd, to_dev(wts), out["ll_pos"], status=st)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(to_host(co), oracle.ll_combine(y, idx, wts, ref["ll_pos"]))


@pytest.mark.parametrize("fp8,H_max,H_over", [(True, 57728, 57856), (False, 57792, 57800)])
def test_ll_largest_hidden_and_one_past(fp8, H_max, H_over):
    """LL rows are staged whole in shared memory: the largest hidden size the
    header states runs bit-exact, the next step is refused before launch."""
    w = Workload("llh", R=2, T=5, H=H_max, E=4, K=2, seed=74)
    inp = make(w)
    x, idx = inp["x"], inp["topk_idx"]
    ref = oracle.ll_layout(idx, w.E)
    rq, rs = oracle.ll_dispatch_rows(x, idx, ref["ll_pos"], w.E, use_fp8=fp8)
    st = ep.new_status()
    out = ep.ep_ll_dispatch(to_dev(x), to_dev(idx), w.E, use_fp8=fp8, status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    np.testing.assert_array_equal(to_host(out["ll_pos"]), ref["ll_pos"])
    q = to_host(out["recv_x"])
    sc = to_host(out["recv_scales"]) if fp8 else None
    for d in range(w.R):
        for j in range(w.E // w.R):
            n = ref["recv_count"][d, j]
            np.testing.assert_array_equal(q[d, j, :n], rq[d, j, :n])
            if fp8:
                np.testing.assert_array_equal(sc[d, j, :n], rs[d, j, :n])
    w2 = Workload("llh2", R=2, T=5, H=H_over, E=4, K=2, seed=75)
    inp2 = make(w2)
    with pytest.raises(ep.EPError, match="unsupported"):
        ep.ep_ll_dispatch(to_dev(inp2["x"]), to_dev(inp2["topk_idx"]), w2.E, use_fp8=fp8)


def test_fp8_input_dispatch_r40_multiwarp():
    w = Workload("f40", R=40, T=20, H=256, E=80, K=4, seed=73)
    inp = make(w)
    R, T, H = w.R, w.T, w.H
    q = np.zeros((R, T, H), np.uint8)
    sc = np.zeros((R, T, H // 128), np.float32)
    for s in range(R):
        for t in range(T):
            q[s, t], sc[s, t] = oracle.quantize_row(inp["x"][s, t])
    h = ep.ep_notify_dispatch(to_dev(inp["topk_idx"]), None, T, R, w.E)
    st = ep.new_status()
    rq, rs = ep.ep_dispatch_cached_fp8(to_dev(q), to_dev(sc), h["send_pos"], status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    eq, es = oracle.dispatch_rows_fp8(q, sc, to_host(h["send_pos"]))
    rc = to_host(h["recv_count"])
    for d in range(R):
        np.testing.assert_array_equal(to_host(rq)[d, :rc[d]], eq[d, :rc[d]])
        np.testing.assert_array_equal(to_host(rs)[d, :rc[d]], es[d, :rc[d]])


def test_empty_inputs_everywhere():
    R, H, E, K = 4, 256, 16, 2
    x = torch.empty((R, 0, H), dtype=torch.bfloat16, device="cuda")
    idx = torch.empty((R, 0, K), dtype=torch.int64, device="cuda")
    wt = torch.empty((R, 0, K), dtype=torch.float32, device="cuda")
    ll = ep.ep_ll_dispatch(x, idx, E, use_fp8=True)
    y = torch.empty((R, E // R, 0, H), dtype=torch.bfloat16, device="cuda")
    co = ep.ep_ll_combine(y, idx, wt, ll["ll_pos"])
    sp = torch.empty((R, 0, R), dtype=torch.int32, device="cuda")
    rx = ep.ep_dispatch_cached(x, sp, capacity=0)
    q = torch.empty((R, 0, H), dtype=torch.uint8, device="cuda")
    s = torch.empty((R, 0, H // 128), dtype=torch.float32, device="cuda")
    rq, rs = ep.ep_dispatch_cached_fp8(q, s, sp, capacity=0)
    torch.cuda.synchronize()
    assert (to_host(ll["recv_count"]) == 0).all() and (to_host(ll["layout_range"]) == 0).all()
    assert co.numel() == 0 and rx.numel() == 0 and rq.numel() == 0


# ---------------------------------------------------------------------------
# layout fused into the notify scan
# ---------------------------------------------------------------------------

FUSED_CASES = [
    ("normal_like", Workload("fu1", R=8, T=300, H=64, E=256, K=8, seed=81)),
    ("ragged_masked", Workload("fu2", R=5, T=129, H=64, E=40, K=3, masked_frac=0.2, seed=82)),
    ("r40_unaligned", Workload("fu3", R=40, T=33, H=64, E=80, K=4, seed=83)),
    # sixteen slots (the scan's 16-slot form) on 16 ranks with 512 experts: the
    # per-source expert counts the kernel after the scan writes are 16 x 512
    ("k16_e512", Workload("fu4", R=16, T=140, H=64, E=512, K=16, masked_frac=0.05, seed=84)),
    ("r2_tiles", Workload("fu5", R=2, T=333, H=64, E=6, K=2, seed=85)),
]


@pytest.mark.parametrize("name,w", FUSED_CASES, ids=[c[0] for c in FUSED_CASES])
def test_notify_with_fused_layout(name, w):
    inp = make(w, with_x=False)
    idx, wts = inp["topk_idx"], inp["topk_weights"]
    lay = oracle.layout(idx, w.E, w.R)
    pre = oracle.prefix(lay["is_token_in_rank"])
    st = ep.new_status()
    h = ep.ep_notify_dispatch(to_dev(idx), to_dev(wts), w.T, w.R, w.E, with_layout=True,
                              status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    np.testing.assert_array_equal(to_host(h["num_tokens_per_rank"]), lay["num_tokens_per_rank"])
    np.testing.assert_array_equal(to_host(h["num_tokens_per_expert"]), lay["num_tokens_per_expert"])
    np.testing.assert_array_equal(to_host(h["is_token_in_rank"]), lay["is_token_in_rank"])
    np.testing.assert_array_equal(to_host(h["send_pos"]), pre["send_pos"])
    np.testing.assert_array_equal(to_host(h["num_recv_tokens_per_expert"]),
                                  oracle.expert_recv_counts(lay["num_tokens_per_expert"], w.R))
    np.testing.assert_array_equal(to_host(h["rank_prefix_matrix"]), pre["rank_prefix_matrix"])
    np.testing.assert_array_equal(to_host(h["recv_count"]), pre["recv_count"])
    ri, rw = oracle.dispatch_meta(idx, wts, pre["send_pos"], w.E)
    rsi, gi, gw = (to_host(h[k]) for k in ("recv_src_idx", "recv_topk_idx", "recv_topk_weights"))
    for d in range(w.R):
        n = int(pre["recv_count"][d])
        np.testing.assert_array_equal(rsi[d, :n], pre["recv_src_idx"][d, :n])
        np.testing.assert_array_equal(gi[d, :n], ri[d, :n])
        np.testing.assert_array_equal(gw[d, :n], rw[d, :n])
        assert (gi[d, n:] == -1).all()
