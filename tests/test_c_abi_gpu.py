"""The C ABI from C: tests/c/ep_c_example.c, compiled against include/ep.h and
libep.so, runs the hand-worked golden example through layout, dispatch and
combine; its printed outputs must equal the fixture."""
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
