"""The one-rank-per-GPU entry points at eight ranks, all driven from one
process on the one test GPU.

To the kernels a peer's buffer is only device memory reached through a table
of pointers, so the eight ranks' receive buffers here are slices of local
allocations, and each rank's calls run in turn on one stream (no kernel waits
for another rank's).  The notify exchange is the stacking of every rank's
count rows, as the all-gather would deliver them.  This reaches the shapes
two processes cannot: R = 8 with top-8 routing, so combine takes its 8-row
form through the peer tables, and the low-latency pair with 8 slabs per
destination.  Every output is compared with the CPU oracle on the stacked
problem (DeepEP legacy-test page: check_data over every received row, the
combine check, low_latency_dispatch / low_latency_combine and their counts).
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle
from tests.helpers import to_dev, to_host
from workloads import Workload, make

import combine_get_dispatch_06_b200 as ep

pytestmark = pytest.mark.gpu

_lib = ep._lib


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _table(t):
    """Device table of the R slices t[0], t[1], ... (one 'peer' buffer each)."""
    return torch.tensor([t[r].data_ptr() for r in range(t.shape[0])], dtype=torch.int64,
                        device=t.device)


def _ok(rc, what):
    assert rc == 0, f"{what}: {ep.ep_status_string(rc)}"


def test_normal_pair_eight_ranks_in_one_process():
    w = Workload("shard8", R=8, T=257, H=512, E=64, K=8, masked_frac=0.05, seed=90)
    R, T, H, K, E = w.R, w.T, w.H, w.K, w.E
    El = E // R
    cap = R * T
    inp = make(w)
    x, idx, wts = inp["x"], inp["topk_idx"], inp["topk_weights"]
    ref = oracle.normal_path(x, idx, wts, E)
    dev = torch.device("cuda")
    stream = torch.cuda.current_stream().cuda_stream
    st = ep.new_status()
    xs, ids, ws_ = to_dev(x), to_dev(idx), to_dev(wts)
    # every rank's receive buffers ("peer" memory) and its own outputs
    recv_x = torch.zeros((R, cap, H), dtype=torch.bfloat16, device=dev)
    recv_idx = torch.zeros((R, cap, K), dtype=torch.int64, device=dev)
    recv_w = torch.zeros((R, cap, K), dtype=torch.float32, device=dev)
    recv_src = torch.zeros((R, cap), dtype=torch.int32, device=dev)
    send_pos = torch.empty((R, T, R), dtype=torch.int32, device=dev)
    P = torch.empty((R, R, R), dtype=torch.int32, device=dev)
    rc = torch.empty((R, 1), dtype=torch.int32, device=dev)
    nrte = torch.empty((R, El), dtype=torch.int32, device=dev)
    ws = torch.empty((R, int(_lib.ep_shard_workspace_bytes(R, T))), dtype=torch.uint8,
                     device=dev)
    # notify exchange: every rank's layout rows, stacked in rank order
    ntpr = torch.empty((R, R), dtype=torch.int32, device=dev)
    ntpe = torch.empty((R, E), dtype=torch.int32, device=dev)
    for r in range(R):
        a, b, _ = ep.ep_get_dispatch_layout(ids[r:r + 1], E, R, status=st)
        ntpr[r].copy_(a[0])
        ntpe[r].copy_(b[0])
    t_rsi, t_idx, t_w, t_x = _table(recv_src), _table(recv_idx), _table(recv_w), _table(recv_x)
    for r in range(R):
        _ok(_lib.ep_shard_notify(_ptr(ids[r]), _ptr(ws_[r]), _ptr(ntpr), _ptr(ntpe), r, R, T, K, E,
                                 1, cap, _ptr(t_rsi), _ptr(t_idx), _ptr(t_w), _ptr(recv_idx[r]),
                                 _ptr(P[r]), _ptr(rc[r]), _ptr(nrte[r]), _ptr(send_pos[r]), None,
                                 _ptr(ws[r]), ws.shape[1], _ptr(st), stream), "ep_shard_notify")
        _ok(_lib.ep_shard_dispatch(_ptr(xs[r]), _ptr(send_pos[r]), R, T, H, cap, _ptr(t_x),
                                   _ptr(st), stream), "ep_shard_dispatch")
    # combine of every rank's tokens, identity experts, through the same tables
    cx = torch.empty((R, T, H), dtype=torch.bfloat16, device=dev)
    cw = torch.empty((R, T, K), dtype=torch.float32, device=dev)
    for r in range(R):
        _ok(_lib.ep_shard_combine(_ptr(t_x), _ptr(t_w), _ptr(send_pos[r]), None, None, R, T, H, K,
                                  cap, _ptr(cx[r]), _ptr(cw[r]), _ptr(st), stream),
            "ep_shard_combine")
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    np.testing.assert_array_equal(to_host(send_pos), ref["send_pos"])
    for r in range(R):
        np.testing.assert_array_equal(to_host(P[r]), ref["rank_prefix_matrix"])
        assert int(rc[r].item()) == int(ref["recv_count"][r])
        np.testing.assert_array_equal(to_host(nrte[r]), ref["num_recv_tokens_per_expert"][r])
        n = int(ref["recv_count"][r])
        np.testing.assert_array_equal(to_host(recv_x[r, :n]), ref["recv_x"][r, :n])
        np.testing.assert_array_equal(to_host(recv_src[r, :n]), ref["recv_src_idx"][r, :n])
        np.testing.assert_array_equal(to_host(recv_idx[r, :n]), ref["recv_topk_idx"][r, :n])
        np.testing.assert_array_equal(to_host(recv_w[r, :n]), ref["recv_topk_weights"][r, :n])
        assert (to_host(recv_idx[r, n:]) == -1).all()
    np.testing.assert_array_equal(to_host(cx), ref["combined_x"])
    np.testing.assert_array_equal(to_host(cw), ref["combined_topk_weights"])


def test_low_latency_pair_eight_ranks_in_one_process():
    w = Workload("shardll8", R=8, T=96, H=256, E=64, K=8, masked_frac=0.05, seed=91)
    R, T, H, K, E = w.R, w.T, w.H, w.K, w.E
    El = E // R
    cap = R * T
    inp = make(w)
    x, idx, wts = inp["x"], inp["topk_idx"], inp["topk_weights"]
    ref = oracle.ll_layout(idx, E)
    rq, rs = oracle.ll_dispatch_rows(x, idx, ref["ll_pos"], E, use_fp8=True)
    y = oracle.dequant_rows(rq, rs)
    ro = oracle.ll_combine(y, idx, wts, ref["ll_pos"])
    dev = torch.device("cuda")
    stream = torch.cuda.current_stream().cuda_stream
    st = ep.new_status()
    xs, ids, ws_ = to_dev(x), to_dev(idx), to_dev(wts)
    slab = torch.zeros((R, El, cap, H), dtype=torch.uint8, device=dev)
    scales = torch.zeros((R, El, cap, H // 128), dtype=torch.float32, device=dev)
    rsi = torch.zeros((R, El, cap), dtype=torch.int32, device=dev)
    lr = torch.zeros((R, El, R, 2), dtype=torch.int32, device=dev)
    ysl = to_dev(y)                                      # the experts' outputs, every slab
    recv_count = torch.empty((R, El), dtype=torch.int32, device=dev)
    ll_pos = torch.empty((R, T, K), dtype=torch.int32, device=dev)
    counts = torch.empty((R, E), dtype=torch.int32, device=dev)
    ws = torch.empty((R, int(_lib.ep_shard_ll_workspace_bytes(R, T, E))), dtype=torch.uint8,
                     device=dev)
    for r in range(R):
        _ok(_lib.ep_shard_ll_counts(_ptr(ids[r]), None, r, R, T, K, E, _ptr(counts[r]), _ptr(st),
                                    stream), "ep_shard_ll_counts")
    t_q, t_s, t_rsi, t_lr, t_y = _table(slab), _table(scales), _table(rsi), _table(lr), _table(ysl)
    for r in range(R):
        _ok(_lib.ep_shard_ll_dispatch(_ptr(xs[r]), _ptr(ids[r]), None, _ptr(counts), r, R, T, H,
                                      K, E, ep.EP_LL_FP8, _ptr(t_q), _ptr(t_s), _ptr(t_rsi),
                                      _ptr(t_lr), _ptr(recv_count[r]), _ptr(ll_pos[r]), None,
                                      _ptr(ws[r]), ws.shape[1], _ptr(st), stream),
            "ep_shard_ll_dispatch")
    out = torch.empty((R, T, H), dtype=torch.bfloat16, device=dev)
    for r in range(R):
        _ok(_lib.ep_shard_ll_combine(_ptr(t_y), _ptr(ids[r]), _ptr(ws_[r]), _ptr(ll_pos[r]), None,
                                     r, R, T, H, K, E, _ptr(out[r]), _ptr(st), stream),
            "ep_shard_ll_combine")
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    np.testing.assert_array_equal(to_host(ll_pos), ref["ll_pos"])
    np.testing.assert_array_equal(to_host(recv_count), ref["recv_count"])
    np.testing.assert_array_equal(to_host(lr), ref["layout_range"])
    q, sc, ri = to_host(slab), to_host(scales), to_host(rsi)
    for d in range(R):
        for j in range(El):
            n = int(ref["recv_count"][d, j])
            np.testing.assert_array_equal(ri[d, j, :n], ref["recv_src_info"][d, j, :n])
            np.testing.assert_array_equal(q[d, j, :n], rq[d, j, :n])
            np.testing.assert_array_equal(sc[d, j, :n], rs[d, j, :n])
    np.testing.assert_array_equal(to_host(out), ro)
