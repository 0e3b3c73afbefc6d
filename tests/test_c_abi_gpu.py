"""The C ABI from C: tests/c/ep_c_example.c, compiled against include/ep.h and
libep.so, runs the hand-worked golden example through layout, dispatch and
combine, and through low-latency dispatch (bf16 slabs) and the weighted
low-latency combine; its printed outputs must equal the fixture."""
import json
import os
import subprocess

import numpy as np
import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_c_caller_reproduces_the_golden_example(tmp_path):
    import combine_get_dispatch_06_b200 as ep  # noqa: F401  (the library is built)

    libdir = os.path.join(ROOT, "combine_get_dispatch_06_b200")
    exe = tmp_path / "ep_c_example"
    cuda = "/usr/local/cuda"
    subprocess.check_call([
        "gcc", "-std=c99", "-O1", "-o", str(exe), os.path.join(ROOT, "tests", "c", "ep_c_example.c"),
        "-I", os.path.join(ROOT, "include"), "-I", os.path.join(cuda, "include"),
        "-L", libdir, "-l:libep.so", f"-Wl,-rpath,{libdir}",
        "-L", os.path.join(cuda, "lib64"), "-lcudart", f"-Wl,-rpath,{cuda}/lib64"])
    out = subprocess.run([str(exe)], capture_output=True, text=True, timeout=120)
    assert out.returncode == 0, out.stderr
    got = {}
    for line in out.stdout.splitlines():
        name, *vals = line.split()
        got[name] = [float(v) for v in vals]
    g = json.load(open(os.path.join(ROOT, "tests", "golden", "routing_tiny.json")))
    flat = lambda a: list(np.array(a, dtype=np.float64).ravel())  # noqa: E731
    assert got["status"] == [0.0]
    for key in ("num_tokens_per_rank", "num_tokens_per_expert", "is_token_in_rank",
                "rank_prefix_matrix", "recv_count", "send_pos", "combined_x",
                "combined_topk_weights"):
        assert got[key] == flat(g[key]), key
    assert got["num_recv_tokens_per_expert"] == flat(g["num_recv_tokens_per_expert_align1"])
    for d in range(g["R"]):
        assert got[f"recv_src_idx_{d}"] == flat(g["recv_src_idx"][d])
        assert got[f"recv_topk_idx_{d}"] == flat(g["recv_topk_idx"][d])
        assert got[f"recv_topk_weights_{d}"] == flat(g["recv_topk_weights"][d])
    # low latency (legacy-test analysis page: the low_latency_dispatch call,
    # its handle (recv_src_info, recv_layout_range) and per-expert counts, and
    # the low_latency_combine check against x times the masked weight sum)
    assert got["ll_status"] == [0.0]
    assert got["ll_recv_count"] == flat(g["ll_recv_count"])
    assert got["ll_layout_range"] == flat(g["ll_layout_range"])
    assert got["ll_pos"] == flat(g["ll_pos"])
    assert got["ll_combined_x"] == flat(g["ll_combined_x"])
    R, El, T = g["R"], g["E"] // g["R"], g["T"]
    x = np.array(g["x"], np.float64)
    for d in range(R):
        for j in range(El):
            assert got[f"ll_recv_src_info_{d}_{j}"] == flat(g["ll_recv_src_info"][d][j])
            # slab rows: the rows of their source tokens, source rank by source rank
            rows = []
            for s in range(R):
                begin, n = g["ll_layout_range"][d][j][s]
                for r in range(begin, begin + n):
                    rows.append(x[s, g["ll_recv_src_info"][d][j][r]])
            assert got[f"ll_slab_{d}_{j}"] == flat(rows), (d, j)
