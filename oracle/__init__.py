"""CPU oracle for MoE token routing -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The CUDA library never calls it, and it
shares no code with the CUDA library: the arithmetic lives in the plain C file
``ep_oracle.c`` next to this module (single-threaded, fp32, no fused
multiply-add unless written as ``fmaf``), loaded through ctypes.  The wrappers
below only allocate numpy arrays and pass pointers.

Pins (see ``tests/test_oracle_pins.py``): brute force on tiny inputs, the
layout invariants, the closed form of combine(dispatch(x)) with identity
experts, exhaustive e4m3 rounding, and hand-worked fixtures under
``tests/golden/``.  No function here is "parity unpinned".
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from typing import Optional

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "ep_oracle.c")
_LIB = os.path.join(_HERE, "libep_oracle.so")
# The mutation test (tests/test_oracle_mutations.py) points this at a build of
# a deliberately broken copy of ep_oracle.c to check that the pins fail.
_LIB_OVERRIDE = os.environ.get("EP_ORACLE_LIB")

_P = ctypes.c_void_p
_I = ctypes.c_int
_L = ctypes.c_long


def build(force: bool = False) -> str:
    """Compile ep_oracle.c into libep_oracle.so (gcc, -O2, no FP contraction)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call([
            "gcc", "-std=c99", "-O2", "-ffp-contract=off", "-fno-fast-math",
            "-fPIC", "-shared", "-Wall", "-o", tmp, _SRC, "-lm",
        ])
        os.replace(tmp, _LIB)
    return _LIB


_lib = None


def lib() -> ctypes.CDLL:
    global _lib
    if _lib is None:
        if _LIB_OVERRIDE:
            L = ctypes.CDLL(_LIB_OVERRIDE)
        else:
            build()
            L = ctypes.CDLL(_LIB)
        L.orc_bf16_to_f32.restype = ctypes.c_float
        L.orc_bf16_to_f32.argtypes = [ctypes.c_uint16]
        L.orc_f32_to_bf16.restype = ctypes.c_uint16
        L.orc_f32_to_bf16.argtypes = [ctypes.c_float]
        L.orc_e4m3_to_f32.restype = ctypes.c_float
        L.orc_e4m3_to_f32.argtypes = [ctypes.c_uint8]
        L.orc_f32_to_e4m3.restype = ctypes.c_uint8
        L.orc_f32_to_e4m3.argtypes = [ctypes.c_float]
        for nm in ("orc_f32_to_e4m3_array", "orc_e4m3_to_f32_array", "orc_f32_to_bf16_array"):
            getattr(L, nm).restype = None
            getattr(L, nm).argtypes = [_P, _L, _P]
        L.orc_layout.restype = _L
        L.orc_layout.argtypes = [_P, _I, _I, _I, _I, _I, _P, _P, _P]
        L.orc_prefix.restype = _L
        L.orc_prefix.argtypes = [_P, _I, _I, _I, _P, _P, _P, _P]
        L.orc_expert_recv_counts.restype = None
        L.orc_expert_recv_counts.argtypes = [_P, _I, _I, _I, _I, _P]
        L.orc_dispatch_rows.restype = None
        L.orc_dispatch_rows.argtypes = [_P, _P, _I, _I, _I, _I, _P, _L, _P]
        L.orc_dispatch_meta.restype = None
        L.orc_dispatch_meta.argtypes = [_P, _P, _P, _I, _I, _I, _I, _I, _P, _P]
        L.orc_combine.restype = None
        L.orc_combine.argtypes = [_P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _P, _L, _P, _P]
        L.orc_dispatch_rows_fp8.restype = None
        L.orc_dispatch_rows_fp8.argtypes = [_P, _P, _I, _P, _I, _I, _I, _I, _P, _P]
        L.orc_ll_layout.restype = _L
        L.orc_ll_layout.argtypes = [_P, _I, _I, _I, _I, _P, _P, _P, _P]
        L.orc_quantize_row_ex.restype = None
        L.orc_quantize_row_ex.argtypes = [_P, _I, _I, _P, _P, _P]
        L.orc_ll_layout_masked.restype = _L
        L.orc_ll_layout_masked.argtypes = [_P, _P, _I, _I, _I, _I, _P, _P, _P, _P]
        L.orc_ll_combine_masked.restype = None
        L.orc_ll_combine_masked.argtypes = [_P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _P, _L, _P]
        L.orc_quantize_row.restype = None
        L.orc_quantize_row.argtypes = [_P, _I, _P, _P]
        L.orc_ll_dispatch_rows.restype = None
        L.orc_ll_dispatch_rows.argtypes = [_P, _P, _P, _I, _I, _I, _I, _I, _I, _P, _L, _P, _P]
        L.orc_dequant_rows.restype = None
        L.orc_dequant_rows.argtypes = [_P, _P, _L, _I, _P]
        L.orc_ll_combine.restype = None
        L.orc_ll_combine.argtypes = [_P, _P, _P, _P, _I, _I, _I, _I, _I, _P, _L, _P]
        _lib = L
    return _lib


def _ptr(a: Optional[np.ndarray]):
    if a is None:
        return None
    assert a.flags["C_CONTIGUOUS"], "oracle arrays must be C-contiguous"
    return a.ctypes.data


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


def _tokens(tokens):
    if tokens is None:
        return None, 0
    t = _c(tokens, np.int64)
    return t, int(t.size)


# --------------------------------------------------------------------------
# scalar conversions
# --------------------------------------------------------------------------

def bf16_to_f32(bits: int) -> float:
    return lib().orc_bf16_to_f32(int(bits))


def f32_to_bf16(v: float) -> int:
    return int(lib().orc_f32_to_bf16(float(v)))


def e4m3_to_f32(code: int) -> float:
    return lib().orc_e4m3_to_f32(int(code))


def f32_to_e4m3(v: float) -> int:
    return int(lib().orc_f32_to_e4m3(float(v)))


def f32_to_e4m3_array(v: np.ndarray) -> np.ndarray:
    a = _c(v, np.float32)
    out = np.zeros(a.shape, np.uint8)
    lib().orc_f32_to_e4m3_array(_ptr(a), a.size, _ptr(out))
    return out


def e4m3_to_f32_array(c: np.ndarray) -> np.ndarray:
    a = _c(c, np.uint8)
    out = np.zeros(a.shape, np.float32)
    lib().orc_e4m3_to_f32_array(_ptr(a), a.size, _ptr(out))
    return out


def f32_to_bf16_array(v: np.ndarray) -> np.ndarray:
    a = _c(v, np.float32)
    out = np.zeros(a.shape, np.uint16)
    lib().orc_f32_to_bf16_array(_ptr(a), a.size, _ptr(out))
    return out


# --------------------------------------------------------------------------
# A1 .. A6
# --------------------------------------------------------------------------

def layout(topk_idx: np.ndarray, num_experts: int, num_ranks: int) -> dict:
    """topk_idx [S,T,K] int64 -> ntpr [S,R], ntpe [S,E], in_rank [S,T,R], bad."""
    idx = _c(topk_idx, np.int64)
    S, T, K = idx.shape
    R, E = num_ranks, num_experts
    ntpr = np.zeros((S, R), np.int32)
    ntpe = np.zeros((S, E), np.int32)
    in_rank = np.zeros((S, T, R), np.uint8)
    bad = lib().orc_layout(_ptr(idx), S, T, K, E, R, _ptr(ntpr), _ptr(ntpe), _ptr(in_rank))
    return {"num_tokens_per_rank": ntpr, "num_tokens_per_expert": ntpe,
            "is_token_in_rank": in_rank, "bad_slots": int(bad)}


def prefix(in_rank: np.ndarray, cap: Optional[int] = None) -> dict:
    """in_rank [R,T,R] -> rank_prefix_matrix, recv_count, send_pos, recv_src_idx."""
    ir = _c(in_rank, np.uint8)
    R, T, R2 = ir.shape
    assert R == R2
    cap = R * T if cap is None else cap
    P = np.zeros((R, R), np.int32)
    rc = np.zeros((R,), np.int32)
    sp = np.zeros((R, T, R), np.int32)
    rsi = np.full((R, max(cap, 0)), -1, np.int32)
    ovf = lib().orc_prefix(_ptr(ir), R, T, cap, _ptr(P), _ptr(rc), _ptr(sp), _ptr(rsi))
    return {"rank_prefix_matrix": P, "recv_count": rc, "send_pos": sp,
            "recv_src_idx": rsi, "overflow": int(ovf)}


def expert_recv_counts(ntpe: np.ndarray, num_ranks: int, alignment: int = 1) -> np.ndarray:
    n = _c(ntpe, np.int32)
    S, E = n.shape
    out = np.zeros((num_ranks, E // num_ranks), np.int32)
    lib().orc_expert_recv_counts(_ptr(n), S, E, num_ranks, alignment, _ptr(out))
    return out


def dispatch_rows(x: np.ndarray, send_pos: np.ndarray, cap: Optional[int] = None,
                  tokens=None, recv_x: Optional[np.ndarray] = None) -> np.ndarray:
    """x [R,T,H] bf16 bits -> recv_x [R,cap,H] (rows not written stay 0)."""
    xx = _c(x, np.uint16)
    R, T, H = xx.shape
    sp = _c(send_pos, np.int32)
    cap = R * T if cap is None else cap
    if recv_x is None:
        recv_x = np.zeros((R, cap, H), np.uint16)
    tk, nt = _tokens(tokens)
    lib().orc_dispatch_rows(_ptr(xx), _ptr(sp), R, T, H, cap, _ptr(tk), nt, _ptr(recv_x))
    return recv_x


def dispatch_meta(topk_idx, topk_weights, send_pos, num_experts: int,
                  cap: Optional[int] = None):
    idx = _c(topk_idx, np.int64)
    R, T, K = idx.shape
    w = _c(topk_weights, np.float32)
    sp = _c(send_pos, np.int32)
    cap = R * T if cap is None else cap
    ri = np.full((R, cap, K), -7, np.int64)
    rw = np.full((R, cap, K), np.nan, np.float32)
    lib().orc_dispatch_meta(_ptr(idx), _ptr(w), _ptr(sp), R, T, K, num_experts, cap,
                            _ptr(ri), _ptr(rw))
    return ri, rw


def combine(y: np.ndarray, send_pos: np.ndarray, recv_topk_weights=None,
            tokens=None, bias=None) -> tuple:
    """y [R,cap,H] bf16 bits, send_pos [R,T,R] -> (out [R,T,H], out_w [R,T,K]|None).
    bias: optional (bias_0, bias_1), each bf16 bits [R,T,H] or None."""
    yy = _c(y, np.uint16)
    R, cap, H = yy.shape
    sp = _c(send_pos, np.int32)
    T = sp.shape[1]
    out = np.zeros((R, T, H), np.uint16)
    rw = None
    out_w = None
    K = 0
    if recv_topk_weights is not None:
        rw = _c(recv_topk_weights, np.float32)
        K = rw.shape[2]
        out_w = np.zeros((R, T, K), np.float32)
    b0, b1 = bias if bias is not None else (None, None)
    b0 = None if b0 is None else _c(b0, np.uint16)
    b1 = None if b1 is None else _c(b1, np.uint16)
    tk, nt = _tokens(tokens)
    lib().orc_combine(_ptr(yy), _ptr(rw), _ptr(sp), _ptr(b0), _ptr(b1), R, T, H, K, cap,
                      _ptr(tk), nt, _ptr(out), _ptr(out_w))
    return out, out_w


def dispatch_rows_fp8(x_q: np.ndarray, x_scales: np.ndarray, send_pos: np.ndarray,
                      col_major: bool = False, cap: Optional[int] = None):
    """FP8 input rows: x_q uint8 [R,T,H], scales [R,T,H/128] (or [R,H/128,T])."""
    xq = _c(x_q, np.uint8)
    R, T, H = xq.shape
    xs = _c(x_scales, np.float32)
    sp = _c(send_pos, np.int32)
    cap = R * T if cap is None else cap
    rq = np.zeros((R, cap, H), np.uint8)
    rs = np.zeros((R, cap, H // 128), np.float32)
    lib().orc_dispatch_rows_fp8(_ptr(xq), _ptr(xs), 1 if col_major else 0, _ptr(sp), R, T, H,
                                cap, _ptr(rq), _ptr(rs))
    return rq, rs


def ll_layout(topk_idx: np.ndarray, num_experts: int, mask=None) -> dict:
    idx = _c(topk_idx, np.int64)
    R, T, K = idx.shape
    E = num_experts
    El = E // R
    count = np.zeros((E,), np.int32)
    lr = np.zeros((E, R, 2), np.int32)
    pos = np.zeros((R, T, K), np.int32)
    rsi = np.full((E, R * T), -1, np.int32)
    m = None if mask is None else _c(mask, np.int32)
    bad = lib().orc_ll_layout_masked(_ptr(idx), _ptr(m), R, T, K, E, _ptr(count), _ptr(lr),
                                     _ptr(pos), _ptr(rsi))
    return {"recv_count": count.reshape(R, El), "layout_range": lr.reshape(R, El, R, 2),
            "ll_pos": pos, "recv_src_info": rsi.reshape(R, El, R * T), "bad_slots": int(bad)}


def quantize_row(x_row: np.ndarray):
    xr = _c(x_row, np.uint16)
    H = xr.shape[-1]
    q = np.zeros((H,), np.uint8)
    s = np.zeros((H // 128,), np.float32)
    lib().orc_quantize_row(_ptr(xr), H, _ptr(q), _ptr(s))
    return q, s


def quantize_row_ex(x_row: np.ndarray, round_scale: bool = False):
    """-> (q uint8 [H], scales fp32 [H/128], ue8m0 uint8 [H/128] or None)."""
    xr = _c(x_row, np.uint16)
    H = xr.shape[-1]
    q = np.zeros((H,), np.uint8)
    s = np.zeros((H // 128,), np.float32)
    u = np.zeros((H // 128,), np.uint8) if round_scale else None
    lib().orc_quantize_row_ex(_ptr(xr), H, 1 if round_scale else 0, _ptr(q), _ptr(s), _ptr(u))
    return q, s, u


def ll_dispatch_rows(x, topk_idx, ll_pos, num_experts: int, use_fp8: bool = True,
                     tokens=None):
    """Returns (slab [R,El,R*T,H] u8 or u16, scales [R,El,R*T,H/128] | None)."""
    xx = _c(x, np.uint16)
    idx = _c(topk_idx, np.int64)
    pos = _c(ll_pos, np.int32)
    R, T, H = xx.shape
    K = idx.shape[2]
    E = num_experts
    El = E // R
    if use_fp8:
        q = np.zeros((R, El, R * T, H), np.uint8)
        sc = np.zeros((R, El, R * T, H // 128), np.float32)
    else:
        q = np.zeros((R, El, R * T, H), np.uint16)
        sc = None
    tk, nt = _tokens(tokens)
    lib().orc_ll_dispatch_rows(_ptr(xx), _ptr(idx), _ptr(pos), R, T, H, K, E,
                               1 if use_fp8 else 0, _ptr(tk), nt, _ptr(q), _ptr(sc))
    return q, sc


def dequant_rows(q: np.ndarray, scales: np.ndarray) -> np.ndarray:
    qq = _c(q, np.uint8)
    ss = _c(scales, np.float32)
    H = qq.shape[-1]
    rows = qq.size // H
    y = np.zeros(qq.shape, np.uint16)
    lib().orc_dequant_rows(_ptr(qq), _ptr(ss), rows, H, _ptr(y))
    return y


def ll_combine(y, topk_idx, topk_weights, ll_pos, tokens=None, mask=None) -> np.ndarray:
    """y [R,El,R*T,H] bf16 bits -> out [R,T,H] bf16 bits."""
    yy = _c(y, np.uint16)
    idx = _c(topk_idx, np.int64)
    w = _c(topk_weights, np.float32)
    pos = _c(ll_pos, np.int32)
    R, El, cap, H = yy.shape
    T = idx.shape[1]
    K = idx.shape[2]
    assert idx.shape[0] == R and cap == R * T, "y must be [R, E_l, R*T, H] for topk_idx [R, T, K]"
    out = np.zeros((R, T, H), np.uint16)
    tk, nt = _tokens(tokens)
    m = None if mask is None else _c(mask, np.int32)
    lib().orc_ll_combine_masked(_ptr(yy), _ptr(idx), _ptr(w), _ptr(pos), _ptr(m), R, T, H, K,
                                R * El, _ptr(tk), nt, _ptr(out))
    return out


# --------------------------------------------------------------------------
# the whole normal path, as one call (used by tests and the CPU baseline)
# --------------------------------------------------------------------------

def normal_path(x, topk_idx, topk_weights, num_experts: int, alignment: int = 1,
                cap: Optional[int] = None, y=None) -> dict:
    """layout -> prefix -> dispatch (rows + metadata) -> combine, all on the CPU.
    ``y`` (expert outputs, [R,cap,H]) defaults to the identity experts' recv_x."""
    R, T, _ = topk_idx.shape
    lay = layout(topk_idx, num_experts, R)
    pre = prefix(lay["is_token_in_rank"], cap)
    cap = R * T if cap is None else cap
    nrte = expert_recv_counts(lay["num_tokens_per_expert"], R, alignment)
    recv_x = dispatch_rows(x, pre["send_pos"], cap)
    ri, rw = dispatch_meta(topk_idx, topk_weights, pre["send_pos"], num_experts, cap)
    yy = recv_x if y is None else y
    out, out_w = combine(yy, pre["send_pos"], rw)
    res = dict(lay)
    res.update(pre)
    res.update({"num_recv_tokens_per_expert": nrte, "recv_x": recv_x,
                "recv_topk_idx": ri, "recv_topk_weights": rw,
                "combined_x": out, "combined_topk_weights": out_w})
    return res
