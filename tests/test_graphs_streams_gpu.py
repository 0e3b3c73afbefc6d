"""Launch-order robustness of the C ABI: the kernels are chained with
programmatic dependent launch, and the low-latency scan and dispatch kernels
run concurrently.  These tests check that (1) a CUDA graph captured from the
calls replays to the eager results, (2) ordinary stream work issued right
after a call (no host synchronisation) sees its outputs, and (3) independent
calls on two streams, with their own workspaces, run side by side correctly."""
import numpy as np
import pytest
import torch

import combine_get_dispatch_06_b200 as ep
import oracle
from workloads import Workload, make
from tests.helpers import to_dev, to_host
from tests.test_parity_gpu import check_dispatch

pytestmark = pytest.mark.gpu


def _normal_inputs(w):
    inp = make(w)
    return inp, to_dev(inp["x"]), to_dev(inp["topk_idx"]), to_dev(inp["topk_weights"])


def _normal_buffers(w, dev):
    R, T, H, E, K = w.R, w.T, w.H, w.E, w.K
    cap = R * T
    out = {
        "recv_x": torch.empty((R, cap, H), dtype=torch.bfloat16, device=dev),
        "recv_topk_idx": torch.empty((R, cap, K), dtype=torch.int64, device=dev),
        "recv_topk_weights": torch.empty((R, cap, K), dtype=torch.float32, device=dev),
        "recv_src_idx": torch.empty((R, cap), dtype=torch.int32, device=dev),
        "rank_prefix_matrix": torch.empty((R, R), dtype=torch.int32, device=dev),
        "recv_count": torch.empty((R,), dtype=torch.int32, device=dev),
        "num_recv_tokens_per_expert": torch.empty((R, E // R), dtype=torch.int32, device=dev),
        "send_pos": torch.empty((R, T, R), dtype=torch.int32, device=dev),
        "num_tokens_per_rank": torch.empty((R, R), dtype=torch.int32, device=dev),
        "num_tokens_per_expert": torch.empty((R, E), dtype=torch.int32, device=dev),
        "is_token_in_rank": torch.empty((R, T, R), dtype=torch.bool, device=dev),
    }
    cx = torch.empty((R, T, H), dtype=torch.bfloat16, device=dev)
    cw = torch.empty((R, T, K), dtype=torch.float32, device=dev)
    ws = torch.empty(ep.ep_dispatch_workspace_bytes(R, T, E), dtype=torch.uint8, device=dev)
    return out, cx, cw, ws


def _normal_step(w, xd, idd, wd, out, cx, cw, ws, st):
    ep.ep_notify_dispatch(idd, wd, w.T, w.R, w.E, with_layout=True, out=out, workspace=ws,
                          status=st)
    ep.ep_dispatch_cached(xd, out["send_pos"], recv_x=out["recv_x"], status=st)
    ep.ep_combine(out["recv_x"], out["send_pos"], out["recv_topk_weights"], combined_x=cx,
                  combined_topk_weights=cw, status=st)


def _scramble(tensors):
    for t in tensors:
        if t.dtype == torch.bool:
            t.fill_(True)
        elif t.is_floating_point():
            t.view(torch.int16 if t.element_size() == 2 else torch.int32).fill_(-21846)
        else:
            t.fill_(-7)


def test_graph_replay_equals_eager_normal_path():
    w = Workload("g", R=8, T=300, H=256, E=64, K=8, masked_frac=0.05, seed=21)
    inp, xd, idd, wd = _normal_inputs(w)
    ref = oracle.normal_path(inp["x"], inp["topk_idx"], inp["topk_weights"], w.E)
    dev = xd.device
    out, cx, cw, ws = _normal_buffers(w, dev)
    st = ep.new_status(dev)
    # eager, then a torch op on the same stream with no host sync in between
    _normal_step(w, xd, idd, wd, out, cx, cw, ws, st)
    cx_copy = cx.clone()
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    check_dispatch(out, ref, w.R, w.K)
    np.testing.assert_array_equal(to_host(cx_copy), ref["combined_x"])
    eager = {k: v.clone() for k, v in out.items()}
    eager_cx, eager_cw = cx.clone(), cw.clone()

    g = torch.cuda.CUDAGraph()
    s = torch.cuda.Stream(dev)
    s.wait_stream(torch.cuda.current_stream(dev))
    with torch.cuda.stream(s):  # warm the capture stream
        _normal_step(w, xd, idd, wd, out, cx, cw, ws, st)
    torch.cuda.current_stream(dev).wait_stream(s)
    torch.cuda.synchronize()
    with torch.cuda.graph(g):
        _normal_step(w, xd, idd, wd, out, cx, cw, ws, st)
    for _ in range(2):
        _scramble(list(out.values()) + [cx, cw])
        g.replay()
        torch.cuda.synchronize()
        assert int(st.item()) == 0
        for k in eager:
            if k == "recv_x":  # rows past recv_count are not written
                for d in range(w.R):
                    n = int(ref["recv_count"][d])
                    assert torch.equal(out[k][d, :n].view(torch.int16),
                                       eager[k][d, :n].view(torch.int16)), k
            elif k in ("recv_src_idx", "recv_topk_weights"):
                for d in range(w.R):
                    n = int(ref["recv_count"][d])
                    assert torch.equal(out[k][d, :n], eager[k][d, :n]), k
            else:
                assert torch.equal(out[k], eager[k]), k
        assert torch.equal(cx.view(torch.int16), eager_cx.view(torch.int16))
        assert torch.equal(cw, eager_cw)
    del g


def test_graph_replay_equals_eager_low_latency():
    w = Workload("gl", R=8, T=200, H=512, E=32, K=6, masked_frac=0.05, seed=22)
    inp = make(w)
    xd, idd, wd = to_dev(inp["x"]), to_dev(inp["topk_idx"]), to_dev(inp["topk_weights"])
    ref = oracle.ll_layout(inp["topk_idx"], w.E)
    rq, rs = oracle.ll_dispatch_rows(inp["x"], inp["topk_idx"], ref["ll_pos"], w.E, use_fp8=True)
    dev = xd.device
    ws = torch.empty(ep.ep_ll_workspace_bytes(w.R, w.T, w.E), dtype=torch.uint8, device=dev)
    st = ep.new_status(dev)
    d = ep.ep_ll_dispatch(xd, idd, w.E, use_fp8=True, workspace=ws, status=st)
    y = to_dev(oracle.dequant_rows(rq, rs))
    co = ep.ep_ll_combine(y, idd, wd, d["ll_pos"], status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    eager = {k: v.clone() for k, v in d.items()}
    eager_co = co.clone()

    def step():
        ep.ep_ll_dispatch(xd, idd, w.E, use_fp8=True, out=d, workspace=ws, status=st)
        ep.ep_ll_combine(y, idd, wd, d["ll_pos"], out=co, status=st)

    s = torch.cuda.Stream(dev)
    s.wait_stream(torch.cuda.current_stream(dev))
    with torch.cuda.stream(s):
        step()
    torch.cuda.current_stream(dev).wait_stream(s)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        step()
    for _ in range(2):
        d["ll_pos"].fill_(-7)
        d["recv_count"].fill_(-7)
        d["layout_range"].fill_(-7)
        co.view(torch.int16).fill_(-21846)
        g.replay()
        torch.cuda.synchronize()
        assert int(st.item()) == 0
        for k in ("ll_pos", "recv_count", "layout_range"):
            assert torch.equal(d[k], eager[k]), k
        np.testing.assert_array_equal(to_host(d["ll_pos"]), ref["ll_pos"])
        assert torch.equal(co.view(torch.int16), eager_co.view(torch.int16))
        q, sc, rsi = to_host(d["recv_x"]), to_host(d["recv_scales"]), to_host(d["recv_src_info"])
        El = w.E // w.R
        for r in range(w.R):
            for j in range(El):
                n = ref["recv_count"][r, j]
                np.testing.assert_array_equal(q[r, j, :n], rq[r, j, :n])
                np.testing.assert_array_equal(sc[r, j, :n], rs[r, j, :n])
                np.testing.assert_array_equal(rsi[r, j, :n], ref["recv_src_info"][r, j, :n])
    del g


def test_independent_calls_on_two_streams():
    wa = Workload("sa", R=6, T=400, H=384, E=48, K=6, seed=23)
    wb = Workload("sb", R=4, T=700, H=256, E=16, K=4, masked_frac=0.1, seed=24)
    dev = torch.device("cuda")
    runs = []
    for w in (wa, wb):
        inp, xd, idd, wd = _normal_inputs(w)
        ref = oracle.normal_path(inp["x"], inp["topk_idx"], inp["topk_weights"], w.E)
        out, cx, cw, ws = _normal_buffers(w, dev)
        runs.append((w, ref, xd, idd, wd, out, cx, cw, ws, ep.new_status(dev),
                     torch.cuda.Stream(dev)))
    torch.cuda.synchronize()
    for _ in range(3):  # interleave the two streams' launches
        for (w, ref, xd, idd, wd, out, cx, cw, ws, st, s) in runs:
            with torch.cuda.stream(s):
                _normal_step(w, xd, idd, wd, out, cx, cw, ws, st)
    torch.cuda.synchronize()
    for (w, ref, xd, idd, wd, out, cx, cw, ws, st, s) in runs:
        assert int(st.item()) == 0
        check_dispatch(out, ref, w.R, w.K)
        np.testing.assert_array_equal(to_host(cx), ref["combined_x"])
        np.testing.assert_array_equal(to_host(cw), ref["combined_topk_weights"])


def test_phase_timers_time_each_phase_of_each_step():
    """The opt-in full-grid timers (DeepEP PR #720 page, "Notify full-kernel
    duration"): one timed phase per call, in stream order and disjoint; the
    results stay the oracle's; a captured graph times its replays; turned
    off, nothing more is counted."""
    w = Workload("pt", R=8, T=300, H=256, E=64, K=8, masked_frac=0.05, seed=23)
    inp, xd, idd, wd = _normal_inputs(w)
    ref = oracle.normal_path(inp["x"], inp["topk_idx"], inp["topk_weights"], w.E)
    dev = xd.device
    out, cx, cw, ws = _normal_buffers(w, dev)
    st = ep.new_status(dev)
    timers = torch.zeros(24, dtype=torch.int64, device=dev)
    ep.ep_set_phase_timers(timers)
    try:
        steps = 3
        for _ in range(steps):
            _normal_step(w, xd, idd, wd, out, cx, cw, ws, st)
        torch.cuda.synchronize()
        v = timers.cpu().tolist()
        for p in range(3):
            assert v[8 * p + 0] == 0 and v[8 * p + 1] == 0  # working slots cleared
            assert v[8 * p + 3] == steps
            assert v[8 * p + 2] > 0
            assert 0 < v[8 * p + 4] < v[8 * p + 5]
        # last step: notify, then copy, then combine, no overlap
        assert v[5] <= v[8 + 4] and v[8 + 5] <= v[16 + 4]
        pt = ep.phase_timer_ms(timers)
        assert all(pt[ph]["launches"] == steps and pt[ph]["ms"] > 0
                   for ph in ("notify", "copy", "combine"))

        g = torch.cuda.CUDAGraph()
        s = torch.cuda.Stream(dev)
        s.wait_stream(torch.cuda.current_stream(dev))
        with torch.cuda.stream(s):
            _normal_step(w, xd, idd, wd, out, cx, cw, ws, st)
        torch.cuda.current_stream(dev).wait_stream(s)
        torch.cuda.synchronize()
        with torch.cuda.graph(g):
            _normal_step(w, xd, idd, wd, out, cx, cw, ws, st)
        before = timers.cpu().tolist()
        g.replay()
        g.replay()
        torch.cuda.synchronize()
        after = timers.cpu().tolist()
        for p in range(3):
            assert after[8 * p + 3] == before[8 * p + 3] + 2
        del g
    finally:
        ep.ep_set_phase_timers(None)
    _scramble(list(out.values()) + [cx, cw])
    _normal_step(w, xd, idd, wd, out, cx, cw, ws, st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    check_dispatch(out, ref, w.R, w.K)
    np.testing.assert_array_equal(to_host(cx), ref["combined_x"])
    np.testing.assert_array_equal(to_host(cw), ref["combined_topk_weights"])
    assert timers.cpu().tolist() == after  # off: nothing more counted


def test_phase_timers_time_the_low_latency_pair():
    """Phases 3 and 4 of the full-grid timers: one LL dispatch span (zeroing,
    scan and the dispatch kernel beside it) and one LL combine span per call,
    disjoint and in stream order; results still the oracle's; a 3-phase array
    leaves the LL calls untimed."""
    w = Workload("plt", R=8, T=200, H=512, E=32, K=6, masked_frac=0.05, seed=24)
    inp = make(w)
    xd, idd, wd = to_dev(inp["x"]), to_dev(inp["topk_idx"]), to_dev(inp["topk_weights"])
    ref = oracle.ll_layout(inp["topk_idx"], w.E)
    rq, rs = oracle.ll_dispatch_rows(inp["x"], inp["topk_idx"], ref["ll_pos"], w.E, use_fp8=True)
    yh = oracle.dequant_rows(rq, rs)
    ro = oracle.ll_combine(yh, inp["topk_idx"], inp["topk_weights"], ref["ll_pos"])
    dev = xd.device
    ws = torch.empty(ep.ep_ll_workspace_bytes(w.R, w.T, w.E), dtype=torch.uint8, device=dev)
    st = ep.new_status(dev)
    y = to_dev(yh)
    timers = torch.zeros(40, dtype=torch.int64, device=dev)
    ep.ep_set_phase_timers(timers)
    try:
        steps = 3
        for _ in range(steps):
            d = ep.ep_ll_dispatch(xd, idd, w.E, use_fp8=True, workspace=ws, status=st)
            co = ep.ep_ll_combine(y, idd, wd, d["ll_pos"], status=st)
        torch.cuda.synchronize()
        v = timers.cpu().tolist()
    finally:
        ep.ep_set_phase_timers(None)
    assert int(st.item()) == 0
    for p in (3, 4):
        assert v[8 * p + 0] == 0 and v[8 * p + 1] == 0
        assert v[8 * p + 3] == steps and v[8 * p + 2] > 0
        assert 0 < v[8 * p + 4] < v[8 * p + 5]
    assert v[24 + 5] <= v[32 + 4]  # last dispatch ends before the last combine starts
    assert all(v[8 * p + 3] == 0 for p in range(3))  # no normal-path call was made
    np.testing.assert_array_equal(to_host(d["ll_pos"]), ref["ll_pos"])
    np.testing.assert_array_equal(to_host(d["recv_count"]), ref["recv_count"])
    np.testing.assert_array_equal(to_host(co), ro)
    q, sc = to_host(d["recv_x"]), to_host(d["recv_scales"])
    for r in range(w.R):
        for j in range(w.E // w.R):
            n = ref["recv_count"][r, j]
            np.testing.assert_array_equal(q[r, j, :n], rq[r, j, :n])
            np.testing.assert_array_equal(sc[r, j, :n], rs[r, j, :n])
    # an array with room for the three normal-path phases only
    short = torch.zeros(24, dtype=torch.int64, device=dev)
    ep.ep_set_phase_timers(short)
    try:
        ep.ep_ll_dispatch(xd, idd, w.E, use_fp8=True, out=d, workspace=ws, status=st)
        ep.ep_ll_combine(y, idd, wd, d["ll_pos"], out=co, status=st)
        torch.cuda.synchronize()
    finally:
        ep.ep_set_phase_timers(None)
    assert int(st.item()) == 0 and short.cpu().tolist() == [0] * 24
