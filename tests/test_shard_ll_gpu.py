"""The sharded low-latency pair on the GPU: two processes, each one rank of a
2-rank job, both on the one GPU of the test machine.

Each rank counts the rows its tokens send to every expert, the ranks
all-gather the counts (gloo), and each rank writes its quantised rows, their
scales and the handle entries straight into the destinations' slabs through
CUDA IPC peer pointers.  Every output is compared with the CPU oracle on the
stacked (single-GPU) problem: ll_pos of the rank's tokens, and as the
destination of its experts the receive counts, layout_range, recv_src_info,
every e4m3 slab row and its scales (legacy-test page, low_latency_dispatch
and its per-expert count check).  The experts then write the dequantised
rows into the shared output slabs and each rank's weighted combine is
compared with the oracle's (legacy-test page, low_latency_combine).  A second
step on new inputs, with rank 1 marked failed, reuses the buffers and adds to
the cumulative per-expert counter.  A second test covers the other payloads:
bf16 rows with sixteen slots (and their combine), and e4m3 rows with UE8M0
scales (round_scale), each slab row against the oracle's quantiser.
"""
import datetime
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _steps():
    from workloads import Workload
    # T = 150: two scan tiles per source rank; some tokens repeat an expert
    return [(Workload("sll_a", R=2, T=150, H=256, E=16, K=4, masked_frac=0.1, seed=60), None),
            (Workload("sll_b", R=2, T=150, H=256, E=16, K=4, routing="zipf", seed=61),
             np.array([0, 1], np.int32))]


def _inputs(w):
    from workloads import make
    inp = make(w)
    idx = inp["topk_idx"].copy()
    g = np.random.default_rng(w.seed + 100)
    rep = g.random(idx.shape[:2]) < 0.1            # slot 1 repeats slot 0's expert
    idx[..., 1][rep] = idx[..., 0][rep]
    return inp["x"], idx, inp["topk_weights"]


def _expected(w, mask):
    import oracle
    x, idx, wts = _inputs(w)
    ref = oracle.ll_layout(idx, w.E, mask=mask)
    rq, rs = oracle.ll_dispatch_rows(x, idx, ref["ll_pos"], w.E, use_fp8=True)
    y = oracle.dequant_rows(rq, rs)                  # the experts' outputs: [R, El, R*T, H]
    out = oracle.ll_combine(y, idx, wts, ref["ll_pos"], mask=mask)
    return ref, rq, rs, y, out


def _worker(rank, world, port, q):
    sys.path.insert(0, ROOT)
    import torch.distributed as dist

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    torch.cuda.set_device(0)
    try:
        from combine_get_dispatch_06_b200.shard import ShardedBuffer
        from tests.helpers import to_dev, to_host

        w0 = _steps()[0][0]
        El = w0.E // world
        buf = ShardedBuffer(dist.group.WORLD, w0.T, w0.H, w0.K, w0.E)
        buf.enable_low_latency(use_fp8=True)
        stats = torch.zeros((El,), dtype=torch.int32, device="cuda")
        results = []
        for w, mask in _steps():
            x, idx, wts = _inputs(w)
            md = to_dev(mask) if mask is not None else None
            out = buf.ll_dispatch(to_dev(x[rank]), to_dev(idx[rank]), rank_mask=md,
                                  cumulative_local_expert_recv_stats=stats)
            torch.cuda.synchronize()
            res = {k: to_host(out[k]) for k in ("ll_pos", "recv_count", "layout_range",
                                                "recv_src_info", "recv_x", "recv_scales")}
            # the experts write their outputs (the oracle's dequantised rows)
            _, _, _, y, _ = _expected(w, mask)
            out["expert_outputs"].copy_(to_dev(y[rank]))
            co = buf.ll_combine(to_dev(idx[rank]), to_dev(wts[rank]), rank_mask=md)
            torch.cuda.synchronize()
            res["combined"] = to_host(co)
            res["status"] = int(buf.status.item())
            results.append(res)
        res_stats = to_host(stats)
        buf.close()
        q.put((rank, results, res_stats, None))
    except Exception:  # report instead of hanging the parent
        import traceback
        q.put((rank, None, None, traceback.format_exc()))
        raise
    finally:
        dist.destroy_process_group()


def test_two_ranks_low_latency_on_one_gpu_match_the_oracle():
    sys.path.insert(0, ROOT)
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    got = {}
    for _ in procs:
        rank, results, stats, err = q.get(timeout=600)
        assert err is None, f"rank {rank}:\n{err}"
        got[rank] = (results, stats)
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0

    total = {r: 0 for r in range(world)}
    for step, (w, mask) in enumerate(_steps()):
        ref, rq, rs, _, out = _expected(w, mask)
        El = w.E // world
        for r in range(world):
            res = got[r][0][step]
            assert res["status"] == 0
            np.testing.assert_array_equal(res["ll_pos"], ref["ll_pos"][r])
            np.testing.assert_array_equal(res["recv_count"], ref["recv_count"][r])
            np.testing.assert_array_equal(res["layout_range"], ref["layout_range"][r])
            for j in range(El):
                n = int(ref["recv_count"][r, j])
                np.testing.assert_array_equal(res["recv_src_info"][j, :n],
                                              ref["recv_src_info"][r, j, :n])
                np.testing.assert_array_equal(res["recv_x"][j, :n], rq[r, j, :n])
                np.testing.assert_array_equal(res["recv_scales"][j, :n], rs[r, j, :n])
            np.testing.assert_array_equal(res["combined"], out[r])
            total[r] = total[r] + ref["recv_count"][r]
        if mask is not None:  # the failed rank sends nothing and gets nothing back
            assert (got[1][0][step]["combined"] == 0).all()
            assert (ref["recv_count"][1] == 0).all()
    for r in range(world):
        np.testing.assert_array_equal(got[r][1], total[r])


# ---------------------------------------------------------------------------
# the other payloads: bf16 rows with sixteen slots, and FP8 with UE8M0 scales
# ---------------------------------------------------------------------------

def _cases():
    from workloads import Workload
    return {"bf16_k16": Workload("sll_c", R=2, T=140, H=256, E=32, K=16, masked_frac=0.05,
                                 seed=62),
            "ue8m0": Workload("sll_d", R=2, T=70, H=384, E=16, K=4, seed=63)}


def _worker_formats(rank, world, port, q):
    sys.path.insert(0, ROOT)
    import torch.distributed as dist

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    torch.cuda.set_device(0)
    try:
        import oracle
        from combine_get_dispatch_06_b200.shard import ShardedBuffer
        from tests.helpers import to_dev, to_host
        from workloads import make

        results = {}
        for name, w in _cases().items():
            inp = make(w)
            x, idx, wts = inp["x"], inp["topk_idx"], inp["topk_weights"]
            buf = ShardedBuffer(dist.group.WORLD, w.T, w.H, w.K, w.E)
            bf16 = name == "bf16_k16"
            buf.enable_low_latency(use_fp8=not bf16, use_ue8m0=not bf16)
            out = buf.ll_dispatch(to_dev(x[rank]), to_dev(idx[rank]), round_scale=not bf16)
            torch.cuda.synchronize()
            res = {k: to_host(out[k]) for k in ("ll_pos", "recv_count", "layout_range",
                                                "recv_src_info", "recv_x")}
            res["recv_scales"] = None if bf16 else to_host(out["recv_scales"])
            if bf16:  # experts return the received rows; combine reads them back
                ref = oracle.ll_layout(idx, w.E)
                rq, _ = oracle.ll_dispatch_rows(x, idx, ref["ll_pos"], w.E, use_fp8=False)
                out["expert_outputs"].copy_(to_dev(rq[rank]))
                co = buf.ll_combine(to_dev(idx[rank]), to_dev(wts[rank]))
                torch.cuda.synchronize()
                res["combined"] = to_host(co)
            res["status"] = int(buf.status.item())
            buf.close()
            results[name] = res
        q.put((rank, results, None))
    except Exception:  # report instead of hanging the parent
        import traceback
        q.put((rank, None, traceback.format_exc()))
        raise
    finally:
        dist.destroy_process_group()


def test_two_ranks_low_latency_bf16_k16_and_ue8m0_match_the_oracle():
    sys.path.insert(0, ROOT)
    import oracle
    from workloads import make

    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker_formats, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    got = {}
    for _ in procs:
        rank, results, err = q.get(timeout=600)
        assert err is None, f"rank {rank}:\n{err}"
        got[rank] = results
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0

    for name, w in _cases().items():
        inp = make(w)
        x, idx, wts = inp["x"], inp["topk_idx"], inp["topk_weights"]
        ref = oracle.ll_layout(idx, w.E)
        El = w.E // world
        bf16 = name == "bf16_k16"
        if bf16:
            rq, _ = oracle.ll_dispatch_rows(x, idx, ref["ll_pos"], w.E, use_fp8=False)
            co = oracle.ll_combine(rq, idx, wts, ref["ll_pos"])
        for r in range(world):
            res = got[r][name]
            assert res["status"] == 0, name
            np.testing.assert_array_equal(res["ll_pos"], ref["ll_pos"][r])
            np.testing.assert_array_equal(res["recv_count"], ref["recv_count"][r])
            np.testing.assert_array_equal(res["layout_range"], ref["layout_range"][r])
            for j in range(El):
                n = int(ref["recv_count"][r, j])
                np.testing.assert_array_equal(res["recv_src_info"][j, :n],
                                              ref["recv_src_info"][r, j, :n])
                if bf16:
                    np.testing.assert_array_equal(res["recv_x"][j, :n], rq[r, j, :n])
            if bf16:
                np.testing.assert_array_equal(res["combined"], co[r])
        if not bf16:  # every slab row against the oracle's quantiser, row by row
            for s in range(world):
                for t in range(w.T):
                    qr, _, ur = oracle.quantize_row_ex(x[s, t], round_scale=True)
                    for k in range(w.K):
                        e = int(idx[s, t, k])
                        if e < 0:
                            continue
                        p = int(ref["ll_pos"][s, t, k])
                        d, j = divmod(e, El)
                        np.testing.assert_array_equal(got[d][name]["recv_x"][j, p], qr)
                        np.testing.assert_array_equal(got[d][name]["recv_scales"][j, p], ur)
