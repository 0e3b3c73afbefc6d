"""The sharded paths' control plane on CPU ranks (gloo, world size 2 and 4).

Each rank takes its own source rank's layout (the oracle's, on the CPU), and
the rows every rank all-gathers must be the single-GPU layout's rows in rank
order: their inclusive prefix over ranks is then the oracle's rank prefix
matrix, its last row the oracle's receive counts, and the gathered expert
rows give the oracle's per-expert receive counts of every destination
(legacy-test analysis page, the inclusive recv_gbl_rank_prefix_sum that
check_data walks; Python接口 page, num_recv_tokens_per_expert_list).  IPC
handles come back in rank order and every rank computes the same layout of
the shared region.  For the low-latency pair, the gathered per-expert rows
of every rank add up to the oracle's receive counts, and their prefix over
earlier ranks is the first row of each rank's block in the oracle's
layout_range (legacy-test page, the low_latency_dispatch handle).
"""
import datetime
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _workload(world):
    from workloads import Workload
    return Workload("shard_host", R=world, T=300, H=0, E=8 * world, K=4, masked_frac=0.1,
                    seed=40 + world)


def _worker(rank, world, port, q):
    sys.path.insert(0, ROOT)
    import torch.distributed as dist

    import oracle
    from combine_get_dispatch_06_b200.shard import (allgather_rows, exchange_handles,
                                                    region_layout)
    from workloads import make

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        w = _workload(world)
        idx = make(w, with_x=False)["topk_idx"]
        mine = oracle.layout(idx[rank:rank + 1], w.E, w.R)     # this rank's own tokens
        counts = allgather_rows(torch.from_numpy(mine["num_tokens_per_rank"][0]))
        ecounts = allgather_rows(torch.from_numpy(mine["num_tokens_per_expert"][0]))
        # the low-latency pair's exchange: rows this rank sends to each expert
        ll_mine = oracle.ll_layout(idx[rank:rank + 1], w.E)["recv_count"].reshape(w.E)
        llcounts = allgather_rows(torch.from_numpy(ll_mine))
        handles = exchange_handles(bytes([rank + 1]) * 64)
        lay = region_layout(w.R * w.T, 64, w.K, True)
        q.put((rank, counts.numpy(), ecounts.numpy(), handles,
               {k: (v if k == "_bytes" else (v[0], v[1], str(v[2]))) for k, v in lay.items()},
               llcounts.numpy()))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 4])
def test_count_exchange_gives_the_oracle_prefix_matrix(world):
    sys.path.insert(0, ROOT)
    import oracle
    from workloads import make

    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    got = dict((r[0], r[1:]) for r in (q.get(timeout=240) for _ in procs))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0

    w = _workload(world)
    idx = make(w, with_x=False)["topk_idx"]
    full = oracle.layout(idx, w.E, w.R)
    pre = oracle.prefix(full["is_token_in_rank"])
    nrte = oracle.expert_recv_counts(full["num_tokens_per_expert"], w.R)
    El = w.E // w.R
    layouts = set()
    llref = oracle.ll_layout(idx, w.E)
    for rank in range(world):
        counts, ecounts, handles, lay, llcounts = got[rank]
        # the sharded LL prefix: rows of each expert from earlier ranks are the
        # first row of that rank's block in the destination's layout_range
        # (legacy-test page, low_latency_dispatch handle), and every rank's
        # rows add up to the expert's receive count
        np.testing.assert_array_equal(llcounts.sum(axis=0), llref["recv_count"].reshape(w.E))
        before = np.cumsum(llcounts, axis=0) - llcounts                      # [R, E]
        lr = llref["layout_range"].reshape(w.E, w.R, 2)
        np.testing.assert_array_equal(before.T, lr[:, :, 0])
        np.testing.assert_array_equal(llcounts.T, lr[:, :, 1])
        np.testing.assert_array_equal(counts, full["num_tokens_per_rank"])
        np.testing.assert_array_equal(np.cumsum(counts, axis=0), pre["rank_prefix_matrix"])
        np.testing.assert_array_equal(np.cumsum(counts, axis=0)[-1], pre["recv_count"])
        np.testing.assert_array_equal(ecounts, full["num_tokens_per_expert"])
        for d in range(world):
            np.testing.assert_array_equal(ecounts[:, d * El:(d + 1) * El].sum(axis=0), nrte[d])
        assert handles == [bytes([r + 1]) * 64 for r in range(world)]
        layouts.add(repr(sorted(lay.items())))
    assert len(layouts) == 1


def _dying_worker(rank, world, port, q):
    sys.path.insert(0, ROOT)
    import time

    import torch.distributed as dist

    from combine_get_dispatch_06_b200.shard import allgather_rows

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=5))
    if rank == 1:
        os._exit(3)  # this rank fails between steps, before the notify exchange
    t0 = time.monotonic()
    try:
        allgather_rows(torch.zeros(world, dtype=torch.int32))
        q.put((rank, "completed", time.monotonic() - t0))
    except Exception as e:  # the survivor learns of it from its collective
        q.put((rank, type(e).__name__, time.monotonic() - t0))
    q.close()
    q.join_thread()  # the message is written out before the process ends
    os._exit(0)


def test_a_rank_that_dies_before_the_notify_exchange_is_detected():
    """Failure detection on the host: a rank exits between steps; the other
    rank's count exchange ends with an error within the process group's
    timeout instead of waiting for ever (no GPU is involved)."""
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_dying_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    rank, outcome, seconds = q.get(timeout=120)
    for p in procs:
        p.join(timeout=60)
    assert rank == 0
    assert outcome != "completed"
    assert seconds < 60
    assert procs[1].exitcode == 3
