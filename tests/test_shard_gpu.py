"""The sharded path on the GPU: two processes, each one rank of a 2-rank job,
both on the one GPU of the test machine.

Each process allocates its receive region, the processes exchange CUDA IPC
handles over a gloo group and map each other's region, and every rank
writes its tokens' rows and received metadata straight into the
destination's region and gathers them back at combine.  All cross-rank
ordering is a stream sync plus a gloo barrier between phases: no kernel
waits for the other process's kernels, so the two contexts may take turns
on the GPU in any order.  Every output is compared with the CPU oracle on
the stacked (single-GPU) problem: send positions, prefix matrix, receive
counts, per-expert counts, every received row and its metadata, the -1
padding past the receive count, and the combine of identity experts and of
expert outputs written into the shared output region; then a second step on
new inputs reuses the same buffers.
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


def _workloads(world):
    from workloads import Workload
    return [Workload("shard_a", R=world, T=300, H=264, E=8 * world, K=4, masked_frac=0.1,
                     seed=50),
            Workload("shard_b", R=world, T=300, H=264, E=8 * world, K=4, routing="zipf",
                     seed=51)]


def _expert_rows(rank, n, H):
    """Expert outputs of rank `rank`'s first n receive rows (seeded)."""
    g = np.random.default_rng(1000 + rank)
    from workloads import bf16_bits_from_f32
    return bf16_bits_from_f32(g.standard_normal((n, H), dtype=np.float32))


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
        from workloads import make

        ws = _workloads(world)
        w0 = ws[0]
        buf = ShardedBuffer(dist.group.WORLD, w0.T, w0.H, w0.K, w0.E, expert_outputs=True)
        results = []
        for step, w in enumerate(ws):
            inp = make(w)
            out = buf.dispatch(to_dev(inp["x"][rank]), to_dev(inp["topk_idx"][rank]),
                               to_dev(inp["topk_weights"][rank]))
            torch.cuda.synchronize()
            rc = int(out["recv_count"].item())
            res = {"recv_count": rc}
            for k in ("send_pos", "rank_prefix_matrix", "num_recv_tokens_per_expert",
                      "num_tokens_per_rank", "num_tokens_per_expert", "is_token_in_rank"):
                res[k] = to_host(out[k])
            for k in ("recv_x", "recv_topk_idx", "recv_topk_weights", "recv_src_idx"):
                res[k] = to_host(out[k][:rc])
            res["pad_ok"] = bool((out["recv_topk_idx"][rc:] == -1).all().item())
            cx, cw = buf.combine()                      # identity experts: recv_x back
            torch.cuda.synchronize()
            res["combined_x"], res["combined_w"] = to_host(cx), to_host(cw)
            # experts write their outputs into the shared region; combine reads them
            y = _expert_rows(rank, rc, w.H)
            buf.buffers["y"][:rc].copy_(to_dev(y))
            cy, _ = buf.combine(expert_outputs=True, with_weights=False)
            torch.cuda.synchronize()
            res["combined_y"] = to_host(cy)
            res["status"] = int(buf.status.item())
            results.append(res)
        probe = to_host(buf.notify_probe)
        buf.close()
        q.put((rank, results, probe, None))
    except Exception as e:  # report instead of hanging the parent
        import traceback
        q.put((rank, None, None, traceback.format_exc()))
        raise
    finally:
        dist.destroy_process_group()


def test_two_ranks_on_one_gpu_match_the_oracle():
    sys.path.insert(0, ROOT)
    import oracle
    from workloads import make

    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    got = {}
    for _ in procs:
        rank, results, probe, err = q.get(timeout=600)
        assert err is None, f"rank {rank}:\n{err}"
        got[rank] = (results, probe)
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0

    for step, w in enumerate(_workloads(world)):
        inp = make(w)
        ref = oracle.normal_path(inp["x"], inp["topk_idx"], inp["topk_weights"], w.E)
        El = w.E // w.R
        for r in range(world):
            res = got[r][0][step]
            assert res["status"] == 0
            np.testing.assert_array_equal(res["send_pos"], ref["send_pos"][r])
            np.testing.assert_array_equal(res["rank_prefix_matrix"], ref["rank_prefix_matrix"])
            np.testing.assert_array_equal(res["num_tokens_per_rank"],
                                          ref["num_tokens_per_rank"][r])
            np.testing.assert_array_equal(res["num_tokens_per_expert"],
                                          ref["num_tokens_per_expert"][r])
            np.testing.assert_array_equal(res["is_token_in_rank"], ref["is_token_in_rank"][r])
            n = int(ref["recv_count"][r])
            assert res["recv_count"] == n
            np.testing.assert_array_equal(res["num_recv_tokens_per_expert"],
                                          ref["num_recv_tokens_per_expert"][r])
            np.testing.assert_array_equal(res["recv_x"], ref["recv_x"][r, :n])
            np.testing.assert_array_equal(res["recv_src_idx"], ref["recv_src_idx"][r, :n])
            np.testing.assert_array_equal(res["recv_topk_idx"], ref["recv_topk_idx"][r, :n])
            np.testing.assert_array_equal(res["recv_topk_weights"],
                                          ref["recv_topk_weights"][r, :n])
            assert res["pad_ok"]
            np.testing.assert_array_equal(res["combined_x"], ref["combined_x"][r])
            np.testing.assert_array_equal(res["combined_w"], ref["combined_topk_weights"][r])
        # expert outputs written into each rank's shared region
        cap = w.R * w.T
        y = np.zeros((w.R, cap, w.H), np.uint16)
        for d in range(world):
            n = int(ref["recv_count"][d])
            y[d, :n] = _expert_rows(d, n, w.H)
        ry, _ = oracle.combine(y, ref["send_pos"])
        for r in range(world):
            np.testing.assert_array_equal(got[r][0][step]["combined_y"], ry[r])
        assert El >= 1
    for r in range(world):
        probe = got[r][1].astype(np.uint64)
        assert probe[1] == len(_workloads(world))       # one notify launch per step
        assert probe[0] > 0 and probe[3] >= probe[2]    # duration, last launch's start <= end
