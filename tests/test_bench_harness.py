"""The benchmark's rank plumbing on CPU: two gloo ranks agree on the slowest
rank's time and the whole-job throughput, and the reference arm (the CPU
oracle) prints one valid JSON line on rank 0 only."""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, out_q):
    import datetime

    import torch.distributed as dist

    sys.path.insert(0, ROOT)
    import bench

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        ms_local = 2.0 if rank == 0 else 3.0
        res = bench.aggregate(bytes_per_step_local=1e9 * (rank + 1),
                              tokens_per_step_local=1000.0, ms_local=ms_local)
        bench.barrier()
        out_q.put((rank, res, bench.dist_env()))
    finally:
        dist.destroy_process_group()


def test_aggregate_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    results = [q.get(timeout=120) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, res, env in results:
        assert env == (2, rank, rank)
        assert res["ms_per_step"] == 3.0                  # slowest rank
        assert res["gbs"] == pytest.approx(3e9 / 3e-3 / 1e9)  # all ranks' bytes
        assert res["tokens_per_s"] == pytest.approx(2000.0 / 3e-3)


def test_aggregate_single_process_is_identity():
    sys.path.insert(0, ROOT)
    import bench

    res = bench.aggregate(2e9, 100.0, 4.0)
    assert res["ms_per_step"] == 4.0
    assert res["gbs"] == pytest.approx(2e9 / 4e-3 / 1e9)


@pytest.mark.slow
def test_reference_arm_prints_one_json_line():
    env = dict(os.environ, WORLD_SIZE="1", RANK="0", LOCAL_RANK="0")
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                          "--steps", "1", "--warmup", "3"], capture_output=True, text=True,
                         env=env, cwd=ROOT, timeout=600)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [l for l in out.stdout.splitlines() if l.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["unit"] == "GB/s" and d["value"] > 0
    assert d["cpu_baseline"]["kind"] == "oracle"
    assert d["e2e"]["h2d_bytes_per_step"] == 0
    # rank 1 of a two-rank launch prints nothing and exits 0
    env1 = dict(os.environ, WORLD_SIZE="2", RANK="1", LOCAL_RANK="1")
    out1 = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                           "--steps", "1", "--warmup", "3"], capture_output=True, text=True,
                          env=env1, cwd=ROOT, timeout=600)
    assert out1.returncode == 0 and out1.stdout.strip() == ""
