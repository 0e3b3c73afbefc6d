"""Full-size parity with the CPU oracle, every output element, no sampling.

* The benchmark's own step (``bench.routing_step``: layout fused into the
  notify scan, cached row copy, combine with identity experts) at the normal
  shape (R=8 x T=4096 x H=7168, top-8 of 256) and the skewed shape (R=16 x
  T=2048 x H=4096, Zipf 1.2 popularity, 10% masked slots), run twice on the
  same buffers and workspace as the timed loop runs it.
* The pages' own sequence at the same shapes: get_dispatch_layout, then
  dispatch with that is_token_in_rank, then combine (DeepEP legacy-test
  analysis page, the check_data walk over every received row).
* The low-latency pair at R=32 x T=128 x H=7168 (top-8 of 256): every slab
  row (e4m3 payload and fp32 scales), every handle entry, and the weighted
  combine of every token.

Host memory is bounded: the oracle's receive buffers are sized to the largest
receive count instead of R*T rows, received rows are pulled from the device
one destination at a time, and the low-latency oracle is called on groups of
tokens whose slab rows are gathered into a compact problem (the 7.5 GB e4m3
slab and the 15 GB bf16 expert-output slab never exist on the host).
"""
import gc
import os
import sys

import numpy as np
import pytest
import torch

import oracle
from workloads import CONFIGS, make
from tests.helpers import to_dev, to_host

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)
import bench  # noqa: E402

pytestmark = [pytest.mark.gpu, pytest.mark.slow]

eq = np.testing.assert_array_equal


def _ep():
    import combine_get_dispatch_06_b200 as ep
    ep.ep_set_debug_flags(0)
    ep.ep_set_wait_timeout_ns(10**9)
    return ep


def _check_normal(out: dict, cx, cw, ref: dict, R: int, with_layout: bool):
    """Every output of one dispatch + combine against the oracle's."""
    rc = ref["recv_count"]
    if with_layout:
        eq(to_host(out["num_tokens_per_rank"]), ref["num_tokens_per_rank"])
        eq(to_host(out["num_tokens_per_expert"]), ref["num_tokens_per_expert"])
        eq(to_host(out["is_token_in_rank"]), ref["is_token_in_rank"])
    eq(to_host(out["rank_prefix_matrix"]), ref["rank_prefix_matrix"])
    eq(to_host(out["recv_count"]), rc)
    eq(to_host(out["send_pos"]), ref["send_pos"])
    eq(to_host(out["num_recv_tokens_per_expert"]), ref["num_recv_tokens_per_expert"])
    for d in range(R):
        n = int(rc[d])
        eq(to_host(out["recv_src_idx"][d, :n]), ref["recv_src_idx"][d, :n])
        eq(to_host(out["recv_topk_idx"][d, :n]), ref["recv_topk_idx"][d, :n])
        eq(to_host(out["recv_topk_weights"][d, :n]), ref["recv_topk_weights"][d, :n])
        # fixed worst-case capacity: rows past the receive count read -1
        assert bool((out["recv_topk_idx"][d, n:] == -1).all()), d
        eq(to_host(out["recv_x"][d, :n]), ref["recv_x"][d, :n])
    eq(to_host(cx), ref["combined_x"])
    eq(to_host(cw), ref["combined_topk_weights"])


def _oracle_full(x, idx, wts, E: int, R: int) -> dict:
    lay = oracle.layout(idx, E, R)
    rc = oracle.prefix(lay["is_token_in_rank"])["recv_count"]
    # receive buffers as deep as the deepest destination: the positions (all
    # below their destination's count) are the same as with R*T rows
    return oracle.normal_path(x, idx, wts, E, cap=int(rc.max()))


def _random_y_combine(ep, out, ref, R, H, status, seed):
    """Combine of random expert outputs over the received rows, all tokens."""
    capo = int(ref["recv_count"].max())
    g = torch.Generator(device="cuda").manual_seed(seed)
    y = torch.randn((R, capo, H), generator=g, device="cuda", dtype=torch.bfloat16)
    cy, _ = ep.ep_combine(y, out["send_pos"], status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    ry, _ = oracle.combine(to_host(y), ref["send_pos"])
    eq(to_host(cy), ry)


@pytest.mark.parametrize("name", ["normal", "skewed"])
def test_bench_step_full_size(name):
    ep = _ep()
    w = CONFIGS[name]
    R, T, H, E, K = w.R, w.T, w.H, w.E, w.K
    inp = make(w)
    x, idx, wts = inp["x"], inp["topk_idx"], inp["topk_weights"]
    device = torch.device("cuda", torch.cuda.current_device())
    out, cx, cw, wsp, status = bench.step_buffers(R, T, H, E, K, device)
    io = {"x": to_dev(x), "idx": to_dev(idx), "wt": to_dev(wts), "cx": cx, "cw": cw}
    stream = torch.cuda.current_stream()
    for _ in range(2):   # the second step reuses workspace and buffers, as the timed loop does
        bench.routing_step(ep, io, out, wsp, status, R, T, E, stream)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    ref = _oracle_full(x, idx, wts, E, R)
    _check_normal(out, cx, cw, ref, R, with_layout=True)
    del ref["recv_x"]
    gc.collect()
    _random_y_combine(ep, out, ref, R, H, status, seed=9)


@pytest.mark.parametrize("name", ["normal", "skewed"])
def test_pages_sequence_full_size(name):
    """get_dispatch_layout -> dispatch(is_token_in_rank) -> combine."""
    ep = _ep()
    w = CONFIGS[name]
    R, E = w.R, w.E
    inp = make(w)
    x, idx, wts = inp["x"], inp["topk_idx"], inp["topk_weights"]
    st = ep.new_status()
    xd, idd, wd = to_dev(x), to_dev(idx), to_dev(wts)
    ntpr, ntpe, inr = ep.ep_get_dispatch_layout(idd, E, R, status=st)
    out = ep.ep_dispatch(xd, idd, wd, E, is_token_in_rank=inr, status=st)
    cx, cw = ep.ep_combine(out["recv_x"], out["send_pos"], out["recv_topk_weights"], status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    ref = _oracle_full(x, idx, wts, E, R)
    out.update(num_tokens_per_rank=ntpr, num_tokens_per_expert=ntpe, is_token_in_rank=inr)
    _check_normal(out, cx, cw, ref, R, with_layout=True)


def test_ll_full_size():
    ep = _ep()
    w = CONFIGS["ll"]
    R, T, H, E, K = w.R, w.T, w.H, w.E, w.K
    El = E // R
    inp = make(w)
    x, idx, wts = inp["x"], inp["topk_idx"], inp["topk_weights"]
    st = ep.new_status()
    xd, idd, wd = to_dev(x), to_dev(idx), to_dev(wts)
    ws = torch.empty(ep.ep_ll_workspace_bytes(R, T, E), dtype=torch.uint8, device="cuda")
    out = ep.ep_ll_dispatch(xd, idd, E, use_fp8=True, workspace=ws, status=st)
    # again on the same outputs and workspace, as the benchmark repeats it
    out = ep.ep_ll_dispatch(xd, idd, E, use_fp8=True, out=out, workspace=ws, status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0

    ref = oracle.ll_layout(idx, E)
    cnt = ref["recv_count"].reshape(E)
    eq(to_host(out["recv_count"]), ref["recv_count"])
    eq(to_host(out["layout_range"]), ref["layout_range"])
    eq(to_host(out["ll_pos"]), ref["ll_pos"])
    rsi = to_host(out["recv_src_info"]).reshape(E, R * T)
    rsi_ref = ref["recv_src_info"].reshape(E, R * T)
    for e in range(E):
        eq(rsi[e, :cnt[e]], rsi_ref[e, :cnt[e]])

    # (token, expert) pairs: one slab row each (a repeated expert shares it)
    pos = ref["ll_pos"]
    s_, t_, k_ = np.nonzero((idx >= 0) & (idx < E))
    e_ = idx[s_, t_, k_]
    p_ = pos[s_, t_, k_]
    u_ = s_ * T + t_
    _, first = np.unique(u_ * E + e_, return_index=True)
    uu, ee, pp = u_[first], e_[first], p_[first]
    # the rows named are exactly 0 .. count-1 of each expert
    order = np.lexsort((pp, ee))
    eq(pp[order], np.concatenate([np.arange(cnt[e]) for e in range(E)]))
    eq(ee[order], np.repeat(np.arange(E), cnt))

    # every slab row: the oracle's quantisation of its token's row
    xf = x.reshape(R * T, H)
    qo = np.empty((R * T, H), np.uint8)
    so = np.empty((R * T, H // 128), np.float32)
    for u in range(R * T):
        qo[u], so[u] = oracle.quantize_row(xf[u])
    te, tp = torch.from_numpy(ee).cuda(), torch.from_numpy(pp).cuda()
    eq(to_host(out["recv_x"].view(E, R * T, H)[te, tp]), qo[uu])
    eq(to_host(out["recv_scales"].view(E, R * T, H // 128)[te, tp]), so[uu])
    del out["recv_x"], out["recv_scales"], qo, so
    torch.cuda.empty_cache()

    # combine of random expert outputs, every token
    g = torch.Generator(device="cuda").manual_seed(3)
    y = torch.randn((R, El, R * T, H), generator=g, device="cuda", dtype=torch.bfloat16)
    co = ep.ep_ll_combine(y, idd, wd, out["ll_pos"], status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    got = to_host(co).reshape(R * T, H)
    # gather every slot's row once; the oracle then combines groups of n
    # tokens as a one-rank problem [1, E, n, H] whose row i of expert e is the
    # row token i of the group reads from expert e
    yg = to_host(y.view(E, R * T, H)[te, tp])          # [pairs, H], in pair order
    row_of = {}
    for i, (u, e) in enumerate(zip(uu.tolist(), ee.tolist())):
        row_of[(u, e)] = i
    idx_f = idx.reshape(R * T, K)
    w_f = wts.reshape(R * T, K)
    n = 64
    ys = np.zeros((1, E, n, H), np.uint16)
    for g0 in range(0, R * T, n):
        toks = range(g0, min(g0 + n, R * T))
        m = len(toks)
        idx_s = np.full((1, n, K), -1, np.int64)
        pos_s = np.full((1, n, K), -1, np.int32)
        w_s = np.zeros((1, n, K), np.float32)
        for i, u in enumerate(toks):
            idx_s[0, i] = idx_f[u]
            w_s[0, i] = w_f[u]
            for k in range(K):
                e = int(idx_f[u, k])
                if 0 <= e < E:
                    ys[0, e, i] = yg[row_of[(u, e)]]
                    pos_s[0, i, k] = i
        ro = oracle.ll_combine(ys, idx_s, w_s, pos_s)
        eq(got[g0:g0 + m], ro[0, :m])
