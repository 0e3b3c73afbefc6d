"""ep_dispatch_noalloc: dispatch for callers that cannot allocate device
memory when they call (their device memory belongs to another allocator, or
cudaMalloc/cudaFree is too slow or synchronising for their loop).  Its scratch
is a static array inside the library.  This file checks, through the C ABI,
that calls in a row (different shapes, so the array is reused with stale
contents) give exactly what ep_dispatch gives with a workspace the caller
allocated, and exactly what the CPU oracle computes; that a call routed by
is_token_in_rank alone works; that a shape whose scratch nearly fills the
array runs and one that needs more is refused; and that an invalid call is
reported as invalid whatever its size.  Collected last so that a failure here
does not hide the other tests' results."""
import numpy as np
import pytest
import torch

import oracle
from workloads import Workload, make
from tests.helpers import to_dev, to_host

pytestmark = pytest.mark.gpu

SCRATCH_BYTES = 2 << 20


def _outputs_like(ref: dict) -> dict:
    return {k: torch.empty_like(v) for k, v in ref.items() if isinstance(v, torch.Tensor)}


def _compare_gpu(a: dict, b: dict, R: int):
    rc = to_host(b["recv_count"])
    np.testing.assert_array_equal(to_host(a["recv_count"]), rc)
    for name in ("rank_prefix_matrix", "send_pos", "num_recv_tokens_per_expert"):
        if name in b:
            np.testing.assert_array_equal(to_host(a[name]), to_host(b[name]))
    for name in ("recv_x", "recv_src_idx", "recv_topk_idx", "recv_topk_weights"):
        if name not in b:
            continue
        ha, hb = to_host(a[name]), to_host(b[name])
        for d in range(R):
            np.testing.assert_array_equal(ha[d, :rc[d]], hb[d, :rc[d]])


def _compare_oracle(a: dict, ref: dict, R: int, meta: bool = True):
    rc = ref["recv_count"]
    np.testing.assert_array_equal(to_host(a["recv_count"]), rc)
    np.testing.assert_array_equal(to_host(a["rank_prefix_matrix"]), ref["rank_prefix_matrix"])
    np.testing.assert_array_equal(to_host(a["send_pos"]), ref["send_pos"])
    names = [("recv_x", "recv_x"), ("recv_src_idx", "recv_src_idx")]
    if meta:
        np.testing.assert_array_equal(to_host(a["num_recv_tokens_per_expert"]),
                                      ref["num_recv_tokens_per_expert"])
        names += [("recv_topk_idx", "recv_topk_idx"), ("recv_topk_weights", "recv_topk_weights")]
    for got_name, ref_name in names:
        g = to_host(a[got_name])
        for d in range(R):
            np.testing.assert_array_equal(g[d, :rc[d]], ref[ref_name][d, :rc[d]])


def _run_pair(ep, w: Workload, align: int):
    inp = make(w)
    xd = to_dev(inp["x"])
    idd = to_dev(inp["topk_idx"])
    wd = to_dev(inp["topk_weights"])
    st_ref = ep.new_status()
    ref = ep.ep_dispatch(xd, idd, wd, w.E, expert_alignment=align, status=st_ref)
    out = _outputs_like(ref)
    st = ep.new_status()
    got = ep.ep_dispatch_noalloc(xd, idd, wd, w.E, expert_alignment=align, out=out, status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0 and int(st_ref.item()) == 0
    _compare_gpu(got, ref, w.R)
    rc = oracle.prefix(oracle.layout(inp["topk_idx"], w.E, w.R)["is_token_in_rank"])["recv_count"]
    o = oracle.normal_path(inp["x"], inp["topk_idx"], inp["topk_weights"], w.E,
                           alignment=align, cap=max(int(rc.max()), 1))
    _compare_oracle(got, o, w.R)


def test_noalloc_matches_dispatch_and_oracle_in_a_row():
    import combine_get_dispatch_06_b200 as ep

    cases = [Workload("na1", R=8, T=1000, H=512, E=64, K=8, seed=31),
             Workload("na2", R=6, T=333, H=264, E=24, K=4, masked_frac=0.2, seed=32),
             Workload("na1b", R=8, T=1000, H=512, E=64, K=8, seed=33)]
    for w in cases:   # calls in a row, different shapes: the scratch keeps stale contents
        _run_pair(ep, w, align=4)


def test_noalloc_routing_from_is_token_in_rank_only():
    """No top-k ids: E counts as 0 for the scratch size, no metadata."""
    import combine_get_dispatch_06_b200 as ep

    rng = np.random.default_rng(34)
    R, T, H = 5, 400, 136
    inr = (rng.random((R, T, R)) < 0.4).astype(np.uint8)
    x = make(Workload("x", R=R, T=T, H=H, E=R, K=1, seed=35))["x"]
    pre = oracle.prefix(inr)
    rx = oracle.dispatch_rows(x, pre["send_pos"])
    cap = R * T
    out = {"recv_x": torch.empty((R, cap, H), dtype=torch.bfloat16, device="cuda"),
           "recv_src_idx": torch.empty((R, cap), dtype=torch.int32, device="cuda"),
           "rank_prefix_matrix": torch.empty((R, R), dtype=torch.int32, device="cuda"),
           "recv_count": torch.empty((R,), dtype=torch.int32, device="cuda"),
           "send_pos": torch.empty((R, T, R), dtype=torch.int32, device="cuda")}
    st = ep.new_status()
    for _ in range(2):
        got = ep.ep_dispatch_noalloc(to_dev(x), None, None, R,
                                     is_token_in_rank=to_dev(inr).bool(), out=out, status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    ref = dict(pre)
    ref["recv_x"] = rx
    _compare_oracle(got, ref, R, meta=False)


def test_noalloc_near_the_limit_runs_and_past_it_is_refused():
    import combine_get_dispatch_06_b200 as ep

    # 384 ranks, one scan tile per source, 384 experts: 84% of the array
    near = Workload("near", R=384, T=128, H=8, E=384, K=4, seed=36)
    assert 0.8 * SCRATCH_BYTES < ep.ep_dispatch_workspace_bytes(384, 128, 384) <= SCRATCH_BYTES
    _run_pair(ep, near, align=1)
    # one token more per source: two tiles per source, past the array
    over = Workload("over", R=384, T=129, H=8, E=384, K=4, seed=37)
    assert ep.ep_dispatch_workspace_bytes(384, 129, 384) > SCRATCH_BYTES
    inp = make(over)
    cap = over.R * over.T
    out = {"recv_x": torch.empty((over.R, cap, over.H), dtype=torch.bfloat16, device="cuda"),
           "recv_src_idx": torch.empty((over.R, cap), dtype=torch.int32, device="cuda"),
           "rank_prefix_matrix": torch.empty((over.R, over.R), dtype=torch.int32, device="cuda"),
           "recv_count": torch.empty((over.R,), dtype=torch.int32, device="cuda"),
           "send_pos": torch.empty((over.R, over.T, over.R), dtype=torch.int32, device="cuda"),
           "recv_topk_idx": torch.empty((over.R, cap, over.K), dtype=torch.int64, device="cuda"),
           "recv_topk_weights": torch.empty((over.R, cap, over.K), dtype=torch.float32,
                                            device="cuda"),
           "num_recv_tokens_per_expert": torch.empty((over.R, 1), dtype=torch.int32,
                                                     device="cuda")}
    with pytest.raises(ep.EPError, match="unsupported"):
        ep.ep_dispatch_noalloc(to_dev(inp["x"]), to_dev(inp["topk_idx"]),
                               to_dev(inp["topk_weights"]), over.E, out=out)


def test_noalloc_invalid_call_is_invalid_whatever_its_size():
    import combine_get_dispatch_06_b200 as ep

    R, T = 384, 4096          # look-back descriptors alone would need ~150 MB
    assert ep.ep_dispatch_workspace_bytes(R, T, 384) > SCRATCH_BYTES
    # no output pointers at all: an argument error, reported before the size
    rc = ep._lib.ep_dispatch_noalloc(None, None, None, None, R, T, 64, 2, 384, 1, R * T,
                                     None, None, None, None, None, None, None, None, None,
                                     None)
    assert rc == ep.EP_ERR_INVALID_ARG
