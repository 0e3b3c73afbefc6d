"""The C-ABI library loads on a CPU-only host, exports every entry point that
include/*.h declares, and rejects bad arguments on the host before launching
anything (these calls never reach the GPU)."""
import ctypes
import glob
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
LIB = os.path.join(ROOT, "combine_get_dispatch_06_b200", "libep.so")


def declared_symbols():
    names = []
    for h in glob.glob(os.path.join(ROOT, "include", "*.h")):
        text = open(h).read()
        names += re.findall(r"EP_API\s+[\w\s\*]+?\b(ep_\w+)\s*\(", text)
    return sorted(set(names))


@pytest.fixture(scope="module")
def lib():
    if not os.path.exists(LIB):
        from combine_get_dispatch_06_b200 import build as b  # noqa: F401
    import combine_get_dispatch_06_b200.build as bmod
    bmod.build()
    return ctypes.CDLL(LIB)


def test_header_declares_the_five_calls():
    names = declared_symbols()
    for n in ["ep_get_dispatch_layout", "ep_dispatch", "ep_combine", "ep_ll_dispatch",
              "ep_ll_combine", "ep_dispatch_workspace_bytes", "ep_ll_workspace_bytes",
              "ep_status_string"]:
        assert n in names


def test_library_exports_every_declared_symbol(lib):
    missing = [n for n in declared_symbols() if not hasattr(lib, n)]
    assert not missing, missing


def test_binding_covers_every_declared_symbol():
    src = open(os.path.join(ROOT, "combine_get_dispatch_06_b200", "__init__.py")).read()
    for n in declared_symbols():
        assert f'"{n}"' in src, n


def test_host_side_argument_checks(lib):
    P = ctypes.c_void_p
    lib.ep_get_dispatch_layout.restype = ctypes.c_int
    lib.ep_get_dispatch_layout.argtypes = [P, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                           ctypes.c_int, ctypes.c_int, P, P, P, P, P]
    bad = [
        (1, 8, 17, 16, 4),   # K > 16
        (1, 8, 0, 16, 4),    # K < 1
        (1, 8, 2, 18, 4),    # E % R != 0
        (1, 8, 2, 1024, 4),  # E > 512
        (1, 8, 2, 768, 768), # R > 384
        (0, 8, 2, 16, 4),    # no source rank
        (1, -1, 2, 16, 4),   # negative T
    ]
    fake = ctypes.c_void_p(16)
    for S, T, K, E, R in bad:
        rc = lib.ep_get_dispatch_layout(fake, S, T, K, E, R, fake, fake, fake, None, None)
        assert rc == 1, (S, T, K, E, R)
    # missing outputs
    assert lib.ep_get_dispatch_layout(fake, 1, 8, 2, 16, 4, None, fake, fake, None, None) == 1
    lib.ep_status_string.restype = ctypes.c_char_p
    assert lib.ep_status_string(1) == b"invalid argument"
    lib.ep_dispatch_workspace_bytes.restype = ctypes.c_size_t
    assert lib.ep_dispatch_workspace_bytes(8, 4096, 256) >= 256 * 8 * 8
    lib.ep_set_wait_timeout_ns.argtypes = [ctypes.c_longlong]
    assert lib.ep_set_wait_timeout_ns(-1) == 1
    assert lib.ep_set_wait_timeout_ns(10**9) == 0


def test_dispatch_rejects_misaligned_and_missing(lib):
    P, I, Z = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
    lib.ep_dispatch.restype = I
    lib.ep_dispatch.argtypes = [P, P, P, P, I, I, I, I, I, I, I, P, P, P, P, P, P, P, P, P, Z, P, P]
    a = ctypes.c_void_p(256)
    mis = ctypes.c_void_p(258)
    ws = 1 << 20

    def call(x=a, idx=a, inr=None, H=64, K=2, E=16, R=4, T=8, recv=a, align=1, cap=32):
        return lib.ep_dispatch(x, idx, None, inr, R, T, H, K, E, align, cap, recv, None, None, a,
                               a, a, None, a, a, ws, None, None)

    assert call(x=mis) == 1               # x not 16-byte aligned
    assert call(recv=mis) == 1            # recv_x not 16-byte aligned
    assert call(H=12) == 1                # H % 8 != 0
    assert call(idx=None) == 1            # neither topk_idx nor is_token_in_rank
    assert call(align=0) == 1
    assert call(cap=-1) == 1


def test_sharded_low_latency_argument_checks(lib):
    """The sharded low-latency entry points refuse bad arguments on the host:
    a rank outside [0, R), experts that do not divide over the ranks, FP8
    flag combinations that do not exist, a short workspace, missing tables."""
    P, I, Z = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
    lib.ep_shard_ll_counts.restype = I
    lib.ep_shard_ll_counts.argtypes = [P, P, I, I, I, I, I, P, P, P]
    lib.ep_shard_ll_workspace_bytes.restype = Z
    lib.ep_shard_ll_workspace_bytes.argtypes = [I, I, I]
    lib.ep_shard_ll_dispatch.restype = I
    lib.ep_shard_ll_dispatch.argtypes = [P, P, P, P, I, I, I, I, I, I, I, P, P, P, P, P, P, P,
                                         P, Z, P, P]
    lib.ep_shard_ll_combine.restype = I
    lib.ep_shard_ll_combine.argtypes = [P, P, P, P, P, I, I, I, I, I, I, P, P, P]
    f = ctypes.c_void_p(256)
    # counts: rank out of range, E % R != 0, K > 16
    assert lib.ep_shard_ll_counts(f, None, 2, 2, 8, 4, 16, f, None, None) == 1
    assert lib.ep_shard_ll_counts(f, None, -1, 2, 8, 4, 16, f, None, None) == 1
    assert lib.ep_shard_ll_counts(f, None, 0, 3, 8, 4, 16, f, None, None) == 1
    assert lib.ep_shard_ll_counts(f, None, 0, 2, 8, 17, 16, f, None, None) == 1
    need = lib.ep_shard_ll_workspace_bytes(2, 8, 16)
    assert need >= lib.ep_ll_workspace_bytes(1, 8, 16) + 16 * 4
    ok = dict(x=f, idx=f, mask=None, counts=f, rank=0, R=2, T=8, H=256, K=4, E=16, flags=1,
              rx=f, rs=f, rsi=f, lr=f, rc=f, pos=f, stats=None, ws=f, wsb=need)

    def disp(**kw):
        a = dict(ok, **kw)
        return lib.ep_shard_ll_dispatch(a["x"], a["idx"], a["mask"], a["counts"], a["rank"],
                                        a["R"], a["T"], a["H"], a["K"], a["E"], a["flags"],
                                        a["rx"], a["rs"], a["rsi"], a["lr"], a["rc"], a["pos"],
                                        a["stats"], a["ws"], a["wsb"], None, None)

    assert disp(rank=2) == 1                 # rank outside [0, R)
    assert disp(flags=4) == 1                # UE8M0 without round_scale
    assert disp(flags=2) == 1                # round_scale without FP8
    assert disp(H=200) == 1                  # FP8 needs H % 128 == 0
    assert disp(wsb=need - 16) == 1          # short workspace
    assert disp(rs=None) == 1                # FP8 without a scales table
    assert disp(counts=None) == 1            # no gathered counts
    assert lib.ep_shard_ll_combine(f, f, f, f, None, 2, 2, 8, 256, 4, 16, f, None, None) == 1
    assert lib.ep_shard_ll_combine(None, f, f, f, None, 0, 2, 8, 256, 4, 16, f, None, None) == 1


def test_phase_timer_switch_checks(lib):
    """ep_set_phase_timers only records a pointer: an unaligned one is
    refused, NULL turns the timers off; the binding wants a CUDA int64 tensor
    of at least 3 x 8 words and reads the mean duration of each phase."""
    lib.ep_set_phase_timers.argtypes = [ctypes.c_void_p, ctypes.c_int]
    assert lib.ep_set_phase_timers(ctypes.c_void_p(0x1004), 3) == 1  # EP_ERR_INVALID_ARG
    assert lib.ep_set_phase_timers(ctypes.c_void_p(0x1000), 0) == 1  # no phase
    assert lib.ep_set_phase_timers(ctypes.c_void_p(0x1000), 6) == 1  # past the last phase
    assert lib.ep_set_phase_timers(None, 0) == 0
    import torch

    import combine_get_dispatch_06_b200 as ep
    for bad in (torch.zeros(24), torch.zeros(24, dtype=torch.int64)):
        with pytest.raises(ValueError):
            ep.ep_set_phase_timers(bad)  # float, or not on a CUDA device
    ep.ep_set_phase_timers(None)
    v = torch.zeros(24, dtype=torch.int64)
    v[2], v[3] = 3_000_000, 2          # notify: 3 ms over 2 phases
    v[8 + 2], v[8 + 3] = 5_000, 1      # copy: 5 us once
    pt = ep.phase_timer_ms(v)
    assert pt["notify"] == {"ms": 1.5, "launches": 2}
    assert pt["copy"] == {"ms": 0.005, "launches": 1}
    assert pt["combine"] == {"ms": None, "launches": 0}
    assert pt["ll_dispatch"] == {"ms": None, "launches": 0}  # not in a 3-phase array
