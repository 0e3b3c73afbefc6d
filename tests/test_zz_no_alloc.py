"""ep_dispatch_noalloc: dispatch for callers that cannot allocate device
memory when they call (their device memory belongs to another allocator, or
cudaMalloc/cudaFree is too slow or synchronising for their loop).  Its scratch
is a static array inside the library; this file checks that two calls in a
row, through the C ABI, give exactly what ep_dispatch gives with a workspace
the caller allocated.  Collected last so that a failure here does not hide
the other tests' results."""
import numpy as np
import pytest
import torch

from workloads import Workload, make
from tests.helpers import to_dev, to_host

pytestmark = pytest.mark.gpu


def _outputs_like(ref: dict) -> dict:
    return {k: torch.empty_like(v) for k, v in ref.items() if isinstance(v, torch.Tensor)}


def _compare(a: dict, b: dict, R: int):
    rc = to_host(b["recv_count"])
    np.testing.assert_array_equal(to_host(a["recv_count"]), rc)
    for name in ("rank_prefix_matrix", "send_pos", "num_recv_tokens_per_expert"):
        np.testing.assert_array_equal(to_host(a[name]), to_host(b[name]))
    for name in ("recv_x", "recv_src_idx", "recv_topk_idx", "recv_topk_weights"):
        ha, hb = to_host(a[name]), to_host(b[name])
        for d in range(R):
            np.testing.assert_array_equal(ha[d, :rc[d]], hb[d, :rc[d]])


def test_noalloc_matches_dispatch_twice_in_a_row():
    import combine_get_dispatch_06_b200 as ep

    cases = [Workload("na1", R=8, T=1000, H=512, E=64, K=8, seed=31),
             Workload("na2", R=6, T=333, H=264, E=24, K=4, masked_frac=0.2, seed=32)]
    for w in cases:   # two calls in a row, different shapes: the scratch is reused
        inp = make(w)
        xd = to_dev(inp["x"])
        idd = to_dev(inp["topk_idx"])
        wd = to_dev(inp["topk_weights"])
        st_ref = ep.new_status()
        ref = ep.ep_dispatch(xd, idd, wd, w.E, expert_alignment=4, status=st_ref)
        out = _outputs_like(ref)
        st = ep.new_status()
        got = ep.ep_dispatch_noalloc(xd, idd, wd, w.E, expert_alignment=4, out=out, status=st)
        torch.cuda.synchronize()
        assert int(st.item()) == 0 and int(st_ref.item()) == 0
        _compare(got, ref, w.R)


def test_noalloc_rejects_sizes_beyond_its_scratch():
    import combine_get_dispatch_06_b200 as ep

    R, T = 384, 4096          # look-back descriptors alone need ~150 MB
    assert ep.ep_dispatch_workspace_bytes(R, T, 384) > (2 << 20)
    rc = ep._lib.ep_dispatch_noalloc(None, None, None, None, R, T, 64, 2, 384, 1, R * T,
                                     None, None, None, None, None, None, None, None, None,
                                     None)
    assert rc == ep.EP_ERR_UNSUPPORTED
