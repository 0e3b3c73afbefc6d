"""Python binding of libep.so, the B200 MoE token-routing library.

Argument marshalling only: every function below checks dtypes and shapes,
allocates missing outputs with torch (device memory is plumbing), passes raw
pointers and the current CUDA stream to the C entry point of the same name,
and raises on a non-zero return.  All computation runs in the CUDA kernels of
``csrc/``; there is no CPU fallback -- importing this package without the built
library, or calling it without a CUDA device, raises.

Layouts and semantics are those of ``include/ep.h``.
"""
from __future__ import annotations

import ctypes
import functools
import os
from typing import Optional

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libep.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(
        f"{LIB_PATH} is missing: build it with `python -c 'import __graft_entry__ as g; g.build()'` "
        "or `python combine_get_dispatch_06_b200/build.py`")

_lib = ctypes.CDLL(LIB_PATH)

_P = ctypes.c_void_p
_I = ctypes.c_int
_Z = ctypes.c_size_t

# name -> (restype, argtypes); mirrors include/ep.h
_SIGS = {
    "ep_status_string": (ctypes.c_char_p, [_I]),
    "ep_version": (_I, []),
    "ep_set_wait_timeout_ns": (_I, [ctypes.c_longlong]),
    "ep_set_debug_flags": (_I, [ctypes.c_uint]),
    "ep_set_phase_timers": (_I, [_P, ctypes.c_int]),
    "ep_get_dispatch_layout": (_I, [_P, _I, _I, _I, _I, _I, _P, _P, _P, _P, _P]),
    "ep_dispatch_workspace_bytes": (_Z, [_I, _I, _I]),
    "ep_dispatch": (_I, [_P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _I,
                         _P, _P, _P, _P, _P, _P, _P, _P, _P, _Z, _P, _P]),
    "ep_notify_dispatch": (_I, [_P, _P, _P, _I, _I, _I, _I, _I, _I,
                                _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _Z, _P, _P]),
    "ep_dispatch_cached": (_I, [_P, _P, _I, _I, _I, _I, _P, _P, _P]),
    "ep_dispatch_noalloc": (_I, [_P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _I,
                                 _P, _P, _P, _P, _P, _P, _P, _P, _P, _P]),
    "ep_dispatch_cached_fp8": (_I, [_P, _P, _I, _P, _I, _I, _I, _I, _P, _P, _P, _P]),
    "ep_combine": (_I, [_P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _P, _P, _P, _P]),
    "ep_ll_workspace_bytes": (_Z, [_I, _I, _I]),
    "ep_ll_dispatch": (_I, [_P, _P, _P, _I, _I, _I, _I, _I, _I, _P, _P, _P, _P, _P, _P,
                            _P, _P, _Z, _P, _P]),
    "ep_ll_combine": (_I, [_P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _P, _P, _P]),
    "ep_shard_alloc": (_I, [_Z, ctypes.POINTER(ctypes.c_void_p)]),
    "ep_shard_free": (_I, [_P]),
    "ep_ipc_handle": (_I, [_P, _P]),
    "ep_ipc_open": (_I, [_P, ctypes.POINTER(ctypes.c_void_p)]),
    "ep_ipc_close": (_I, [_P]),
    "ep_shard_workspace_bytes": (_Z, [_I, _I]),
    "ep_shard_notify": (_I, [_P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _P, _P, _P, _P, _P,
                             _P, _P, _P, _P, _P, _Z, _P, _P]),
    "ep_shard_dispatch": (_I, [_P, _P, _I, _I, _I, _I, _P, _P, _P]),
    "ep_shard_combine": (_I, [_P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _P, _P, _P, _P]),
    "ep_shard_ll_counts": (_I, [_P, _P, _I, _I, _I, _I, _I, _P, _P, _P]),
    "ep_shard_ll_workspace_bytes": (_Z, [_I, _I, _I]),
    "ep_shard_ll_dispatch": (_I, [_P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _P, _P, _P, _P,
                                  _P, _P, _P, _P, _Z, _P, _P]),
    "ep_shard_ll_combine": (_I, [_P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _P, _P, _P]),
}
for _name, (_res, _args) in _SIGS.items():
    _fn = getattr(_lib, _name)
    _fn.restype = _res
    _fn.argtypes = _args

EP_OK, EP_ERR_INVALID_ARG, EP_ERR_CUDA, EP_ERR_UNSUPPORTED = 0, 1, 2, 3
EP_STATUS_BAD_EXPERT = 1
EP_STATUS_CAPACITY = 2
EP_STATUS_WAIT_TIMEOUT = 4
EP_STATUS_BAD_POSITION = 8
EP_DEBUG_SUPPRESS_PUBLISH = 1
EP_LL_FP8, EP_LL_ROUND_SCALE, EP_LL_UE8M0 = 1, 2, 4


class EPError(RuntimeError):
    pass


def _check(rc: int, what: str):
    if rc != EP_OK:
        raise EPError(f"{what}: {_lib.ep_status_string(rc).decode()} ({rc})")


def _ptr(t: Optional[torch.Tensor]):
    if t is None:
        return None
    if not t.is_cuda:
        raise EPError("all tensors passed to libep must be CUDA tensors")
    if t.device.index != torch.cuda.current_device():
        raise EPError("all tensors of one call must be on the same CUDA device")
    if not t.is_contiguous():
        raise EPError("all tensors passed to libep must be contiguous")
    return t.data_ptr()


def _stream(stream) -> Optional[int]:
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream


def _on_tensor_device(fn):
    """Run a wrapper with the device of its first CUDA tensor argument
    current, so that allocations, the default stream and the library's
    per-device settings all refer to that device."""
    @functools.wraps(fn)
    def wrapper(*args, **kwargs):
        for a in list(args) + list(kwargs.values()):
            if isinstance(a, torch.Tensor) and a.is_cuda:
                with torch.cuda.device(a.device):
                    return fn(*args, **kwargs)
        return fn(*args, **kwargs)
    return wrapper


def _need(t: torch.Tensor, dtype, shape, name):
    if t.dtype != dtype or tuple(t.shape) != tuple(shape):
        raise EPError(f"{name}: expected {dtype} {tuple(shape)}, got {t.dtype} {tuple(t.shape)}")


def library_path() -> str:
    return LIB_PATH


def ep_version() -> int:
    return _lib.ep_version()


def ep_status_string(code: int) -> str:
    return _lib.ep_status_string(code).decode()


def ep_set_wait_timeout_ns(ns: int) -> None:
    _check(_lib.ep_set_wait_timeout_ns(int(ns)), "ep_set_wait_timeout_ns")


def ep_set_debug_flags(flags: int) -> None:
    _check(_lib.ep_set_debug_flags(int(flags)), "ep_set_debug_flags")


PHASES = ("notify", "copy", "combine", "ll_dispatch", "ll_combine")


def ep_set_phase_timers(timers: Optional[torch.Tensor]) -> None:
    """Turn the full-grid phase timers on (a zeroed int64 CUDA tensor of 8
    words per phase, in PHASES order; a shorter tensor times the first
    phases only) or off (None); see phase_timer_ms."""
    n = 0
    if timers is not None:
        if timers.dtype != torch.int64 or not timers.is_cuda or timers.numel() < 8 \
                or not timers.is_contiguous():
            raise ValueError("timers must be a contiguous CUDA int64 tensor of >= 8 words")
        n = min(timers.numel() // 8, len(PHASES))
    _check(_lib.ep_set_phase_timers(_ptr(timers), n), "ep_set_phase_timers")


def phase_timer_ms(timers: torch.Tensor) -> dict:
    """Mean duration in ms (and count) of each phase timed into `timers`."""
    v = timers.view(-1).cpu().tolist()
    out = {}
    for i, name in enumerate(PHASES):
        n = v[8 * i + 3] if 8 * i + 8 <= len(v) else 0
        out[name] = {"ms": (v[8 * i + 2] / n / 1e6) if n else None, "launches": n}
    return out


def new_status(device=None) -> torch.Tensor:
    return torch.zeros(1, dtype=torch.int32, device=device or "cuda")


# ---------------------------------------------------------------------------
# A1
# ---------------------------------------------------------------------------

@_on_tensor_device
def ep_get_dispatch_layout(topk_idx: torch.Tensor, num_experts: int, num_ranks: int, *,
                           num_tokens_per_rank=None, num_tokens_per_expert=None,
                           is_token_in_rank=None, status=None, stream=None):
    """topk_idx int64 [S, T, K] (or [T, K] for one source rank) ->
    (num_tokens_per_rank int32 [S, R], num_tokens_per_expert int32 [S, E],
    is_token_in_rank bool [S, T, R])."""
    squeeze = topk_idx.dim() == 2
    idx = topk_idx.unsqueeze(0) if squeeze else topk_idx
    S, T, K = idx.shape
    R, E = num_ranks, num_experts
    dev = idx.device
    if squeeze:  # outputs given in the single-rank shapes
        if num_tokens_per_rank is not None and num_tokens_per_rank.dim() == 1:
            num_tokens_per_rank = num_tokens_per_rank.unsqueeze(0)
        if num_tokens_per_expert is not None and num_tokens_per_expert.dim() == 1:
            num_tokens_per_expert = num_tokens_per_expert.unsqueeze(0)
        if is_token_in_rank is not None and is_token_in_rank.dim() == 2:
            is_token_in_rank = is_token_in_rank.unsqueeze(0)
    if num_tokens_per_rank is None:
        num_tokens_per_rank = torch.empty((S, R), dtype=torch.int32, device=dev)
    if num_tokens_per_expert is None:
        num_tokens_per_expert = torch.empty((S, E), dtype=torch.int32, device=dev)
    if is_token_in_rank is None:
        is_token_in_rank = torch.empty((S, T, R), dtype=torch.bool, device=dev)
    _need(idx, torch.int64, (S, T, K), "topk_idx")
    _need(num_tokens_per_rank, torch.int32, (S, R), "num_tokens_per_rank")
    _need(num_tokens_per_expert, torch.int32, (S, E), "num_tokens_per_expert")
    _need(is_token_in_rank, torch.bool, (S, T, R), "is_token_in_rank")
    rc = _lib.ep_get_dispatch_layout(
        _ptr(idx), S, T, K, E, R, _ptr(num_tokens_per_rank), _ptr(num_tokens_per_expert),
        _ptr(is_token_in_rank), _ptr(status), _stream(stream))
    _check(rc, "ep_get_dispatch_layout")
    if squeeze:
        return num_tokens_per_rank[0], num_tokens_per_expert[0], is_token_in_rank[0]
    return num_tokens_per_rank, num_tokens_per_expert, is_token_in_rank


# ---------------------------------------------------------------------------
# A2 + A3
# ---------------------------------------------------------------------------

def ep_dispatch_workspace_bytes(num_ranks: int, num_tokens: int, num_experts: int) -> int:
    return int(_lib.ep_dispatch_workspace_bytes(num_ranks, num_tokens, num_experts))


@_on_tensor_device
def ep_dispatch(x: torch.Tensor, topk_idx: Optional[torch.Tensor],
                topk_weights: Optional[torch.Tensor], num_experts: int, *,
                is_token_in_rank: Optional[torch.Tensor] = None, expert_alignment: int = 1,
                capacity: Optional[int] = None, out: Optional[dict] = None,
                with_metadata: bool = True, workspace: Optional[torch.Tensor] = None,
                status=None, stream=None) -> dict:
    """x bf16 [R, T, H] -> dict of recv_x, recv_topk_idx, recv_topk_weights,
    recv_src_idx, rank_prefix_matrix, recv_count, num_recv_tokens_per_expert,
    send_pos (see ep.h).  Outputs given in ``out`` are reused."""
    R, T, H = x.shape
    dev = x.device
    _need(x, torch.bfloat16, (R, T, H), "x")
    K = topk_idx.shape[2] if topk_idx is not None else 0
    E = num_experts
    cap = R * T if capacity is None else int(capacity)
    o = dict(out or {})

    def get(name, shape, dtype):
        if o.get(name) is None:
            o[name] = torch.empty(shape, dtype=dtype, device=dev)
        _need(o[name], dtype, shape, name)
        return o[name]

    get("recv_x", (R, cap, H), torch.bfloat16)
    get("recv_src_idx", (R, cap), torch.int32)
    get("rank_prefix_matrix", (R, R), torch.int32)
    get("recv_count", (R,), torch.int32)
    get("send_pos", (R, T, R), torch.int32)
    meta = with_metadata and topk_idx is not None
    if meta:
        get("recv_topk_idx", (R, cap, K), torch.int64)
        get("num_recv_tokens_per_expert", (R, E // R), torch.int32)
        if topk_weights is not None:
            get("recv_topk_weights", (R, cap, K), torch.float32)
    if topk_idx is not None:
        _need(topk_idx, torch.int64, (R, T, K), "topk_idx")
    if topk_weights is not None:
        _need(topk_weights, torch.float32, (R, T, K), "topk_weights")
    if is_token_in_rank is not None:
        _need(is_token_in_rank, torch.bool, (R, T, R), "is_token_in_rank")
    need = ep_dispatch_workspace_bytes(R, T, E if topk_idx is not None else 0)
    if workspace is None:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=dev)
    rc = _lib.ep_dispatch(
        _ptr(x), _ptr(topk_idx), _ptr(topk_weights), _ptr(is_token_in_rank), R, T, H, K, E,
        int(expert_alignment), cap, _ptr(o["recv_x"]), _ptr(o.get("recv_topk_idx") if meta else None),
        _ptr(o.get("recv_topk_weights") if meta else None), _ptr(o["recv_src_idx"]),
        _ptr(o["rank_prefix_matrix"]), _ptr(o["recv_count"]),
        _ptr(o.get("num_recv_tokens_per_expert") if meta else None), _ptr(o["send_pos"]),
        _ptr(workspace), workspace.numel(), _ptr(status), _stream(stream))
    _check(rc, "ep_dispatch")
    return o


@_on_tensor_device
def ep_notify_dispatch(topk_idx: Optional[torch.Tensor], topk_weights: Optional[torch.Tensor],
                       num_tokens: int, num_ranks: int, num_experts: int, *,
                       is_token_in_rank: Optional[torch.Tensor] = None,
                       expert_alignment: int = 1, capacity: Optional[int] = None,
                       out: Optional[dict] = None, with_metadata: bool = True,
                       with_layout: bool = False,
                       workspace: Optional[torch.Tensor] = None, status=None,
                       stream=None) -> dict:
    """The first half of ep_dispatch: handle + received metadata (no rows).
    with_layout (routing from topk_idx only): also return the layout,
    num_tokens_per_rank [R, R], num_tokens_per_expert [R, E],
    is_token_in_rank bool [R, T, R], from the same kernel."""
    R, T = num_ranks, num_tokens
    src = topk_idx if topk_idx is not None else is_token_in_rank
    dev = src.device
    K = topk_idx.shape[2] if topk_idx is not None else 0
    E = num_experts
    cap = R * T if capacity is None else int(capacity)
    o = dict(out or {})

    def get(name, shape, dtype):
        if o.get(name) is None:
            o[name] = torch.empty(shape, dtype=dtype, device=dev)
        _need(o[name], dtype, shape, name)
        return o[name]

    get("recv_src_idx", (R, cap), torch.int32)
    get("rank_prefix_matrix", (R, R), torch.int32)
    get("recv_count", (R,), torch.int32)
    get("send_pos", (R, T, R), torch.int32)
    meta = with_metadata and topk_idx is not None
    if meta:
        get("recv_topk_idx", (R, cap, K), torch.int64)
        get("num_recv_tokens_per_expert", (R, E // R), torch.int32)
        if topk_weights is not None:
            get("recv_topk_weights", (R, cap, K), torch.float32)
    if with_layout:
        get("num_tokens_per_rank", (R, R), torch.int32)
        get("num_tokens_per_expert", (R, E), torch.int32)
        get("is_token_in_rank", (R, T, R), torch.bool)
    if topk_idx is not None:
        _need(topk_idx, torch.int64, (R, T, K), "topk_idx")
    if topk_weights is not None:
        _need(topk_weights, torch.float32, (R, T, K), "topk_weights")
    if is_token_in_rank is not None:
        _need(is_token_in_rank, torch.bool, (R, T, R), "is_token_in_rank")
    need = ep_dispatch_workspace_bytes(R, T, E if topk_idx is not None else 0)
    if workspace is None:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=dev)
    rc = _lib.ep_notify_dispatch(
        _ptr(topk_idx), _ptr(topk_weights), _ptr(is_token_in_rank), R, T, K, E,
        int(expert_alignment), cap, _ptr(o.get("recv_topk_idx") if meta else None),
        _ptr(o.get("recv_topk_weights") if meta else None), _ptr(o["recv_src_idx"]),
        _ptr(o["rank_prefix_matrix"]), _ptr(o["recv_count"]),
        _ptr(o.get("num_recv_tokens_per_expert") if meta else None), _ptr(o["send_pos"]),
        _ptr(o.get("num_tokens_per_rank") if with_layout else None),
        _ptr(o.get("num_tokens_per_expert") if with_layout else None),
        _ptr(o.get("is_token_in_rank") if with_layout else None),
        _ptr(workspace), workspace.numel(), _ptr(status), _stream(stream))
    _check(rc, "ep_notify_dispatch")
    return o


@_on_tensor_device
def ep_dispatch_cached(x: torch.Tensor, send_pos: torch.Tensor, *, capacity: Optional[int] = None,
                       recv_x: Optional[torch.Tensor] = None, status=None,
                       stream=None) -> torch.Tensor:
    """Cached-mode dispatch: rows of x to the rows send_pos names."""
    R, T, H = x.shape
    _need(x, torch.bfloat16, (R, T, H), "x")
    _need(send_pos, torch.int32, (R, T, R), "send_pos")
    cap = R * T if capacity is None else int(capacity)
    if recv_x is None:
        recv_x = torch.empty((R, cap, H), dtype=torch.bfloat16, device=x.device)
    _need(recv_x, torch.bfloat16, (R, cap, H), "recv_x")
    rc = _lib.ep_dispatch_cached(_ptr(x), _ptr(send_pos), R, T, H, cap, _ptr(recv_x),
                                 _ptr(status), _stream(stream))
    _check(rc, "ep_dispatch_cached")
    return recv_x


@_on_tensor_device
def ep_dispatch_cached_fp8(x_e4m3: torch.Tensor, x_scales: torch.Tensor, send_pos: torch.Tensor,
                           *, scales_col_major: bool = False, capacity: Optional[int] = None,
                           recv_x: Optional[torch.Tensor] = None,
                           recv_scales: Optional[torch.Tensor] = None, status=None,
                           stream=None):
    """FP8 rows (uint8 e4m3 [R, T, H]) and their scales ([R, T, H/128], or
    [R, H/128, T] when scales_col_major) to the rows send_pos names.  Returns
    (recv_x uint8 [R, cap, H], recv_scales fp32 [R, cap, H/128])."""
    R, T, H = x_e4m3.shape
    nb = H // 128
    _need(x_e4m3, torch.uint8, (R, T, H), "x_e4m3")
    _need(x_scales, torch.float32, (R, nb, T) if scales_col_major else (R, T, nb), "x_scales")
    _need(send_pos, torch.int32, (R, T, R), "send_pos")
    cap = R * T if capacity is None else int(capacity)
    if recv_x is None:
        recv_x = torch.empty((R, cap, H), dtype=torch.uint8, device=x_e4m3.device)
    if recv_scales is None:
        recv_scales = torch.empty((R, cap, nb), dtype=torch.float32, device=x_e4m3.device)
    _need(recv_x, torch.uint8, (R, cap, H), "recv_x")
    _need(recv_scales, torch.float32, (R, cap, nb), "recv_scales")
    rc = _lib.ep_dispatch_cached_fp8(_ptr(x_e4m3), _ptr(x_scales), 1 if scales_col_major else 0,
                                     _ptr(send_pos), R, T, H, cap, _ptr(recv_x),
                                     _ptr(recv_scales), _ptr(status), _stream(stream))
    _check(rc, "ep_dispatch_cached_fp8")
    return recv_x, recv_scales


@_on_tensor_device
def ep_dispatch_noalloc(x: torch.Tensor, topk_idx: Optional[torch.Tensor],
                        topk_weights: Optional[torch.Tensor], num_experts: int, *,
                        is_token_in_rank: Optional[torch.Tensor] = None,
                        expert_alignment: int = 1, capacity: Optional[int] = None,
                        out: Optional[dict] = None, status=None, stream=None) -> dict:
    """ep_dispatch for callers that cannot allocate device memory when they call
    (their memory belongs to another allocator, or cudaMalloc is too slow for
    their loop): the scratch is a static 2 MiB array inside the library.  All
    outputs must be passed in ``out``; nothing is allocated here.  Calls that
    overlap on the GPU share that array and race."""
    R, T, H = x.shape
    _need(x, torch.bfloat16, (R, T, H), "x")
    K = topk_idx.shape[2] if topk_idx is not None else 0
    E = num_experts
    cap = R * T if capacity is None else int(capacity)
    o = dict(out or {})
    shapes = {"recv_x": ((R, cap, H), torch.bfloat16), "recv_src_idx": ((R, cap), torch.int32),
              "rank_prefix_matrix": ((R, R), torch.int32), "recv_count": ((R,), torch.int32),
              "send_pos": ((R, T, R), torch.int32)}
    if topk_idx is not None:
        shapes["recv_topk_idx"] = ((R, cap, K), torch.int64)
        shapes["num_recv_tokens_per_expert"] = ((R, E // R), torch.int32)
        if topk_weights is not None:
            shapes["recv_topk_weights"] = ((R, cap, K), torch.float32)
    for name, (shape, dtype) in shapes.items():
        if o.get(name) is None:
            raise EPError(f"ep_dispatch_noalloc allocates nothing: pass out[{name!r}]")
        _need(o[name], dtype, shape, name)
    rc = _lib.ep_dispatch_noalloc(
        _ptr(x), _ptr(topk_idx), _ptr(topk_weights), _ptr(is_token_in_rank), R, T, H, K, E,
        int(expert_alignment), cap, _ptr(o["recv_x"]), _ptr(o.get("recv_topk_idx")),
        _ptr(o.get("recv_topk_weights")), _ptr(o["recv_src_idx"]),
        _ptr(o["rank_prefix_matrix"]), _ptr(o["recv_count"]),
        _ptr(o.get("num_recv_tokens_per_expert")), _ptr(o["send_pos"]), _ptr(status),
        _stream(stream))
    _check(rc, "ep_dispatch_noalloc")
    return o


# ---------------------------------------------------------------------------
# A4
# ---------------------------------------------------------------------------

@_on_tensor_device
def ep_combine(y: torch.Tensor, send_pos: torch.Tensor,
               recv_topk_weights: Optional[torch.Tensor] = None, *,
               bias: Optional[tuple] = None,
               combined_x: Optional[torch.Tensor] = None,
               combined_topk_weights: Optional[torch.Tensor] = None,
               status=None, stream=None):
    """y bf16 [R, cap, H], send_pos int32 [R, T, R] ->
    (combined_x bf16 [R, T, H], combined_topk_weights fp32 [R, T, K] or None)."""
    R, cap, H = y.shape
    T = send_pos.shape[1]
    dev = y.device
    _need(y, torch.bfloat16, (R, cap, H), "y")
    _need(send_pos, torch.int32, (R, T, R), "send_pos")
    K = 0
    if recv_topk_weights is not None:
        K = recv_topk_weights.shape[2]
        _need(recv_topk_weights, torch.float32, (R, cap, K), "recv_topk_weights")
        if combined_topk_weights is None:
            combined_topk_weights = torch.empty((R, T, K), dtype=torch.float32, device=dev)
    if combined_x is None:
        combined_x = torch.empty((R, T, H), dtype=torch.bfloat16, device=dev)
    _need(combined_x, torch.bfloat16, (R, T, H), "combined_x")
    b0, b1 = (bias if bias is not None else (None, None))
    for b, nm in ((b0, "bias_0"), (b1, "bias_1")):
        if b is not None:
            _need(b, torch.bfloat16, (R, T, H), nm)
    rc = _lib.ep_combine(
        _ptr(y), _ptr(recv_topk_weights), _ptr(send_pos), _ptr(b0), _ptr(b1), R, T, H, K, cap,
        _ptr(combined_x),
        _ptr(combined_topk_weights if recv_topk_weights is not None else None), _ptr(status),
        _stream(stream))
    _check(rc, "ep_combine")
    return combined_x, (combined_topk_weights if recv_topk_weights is not None else None)


# ---------------------------------------------------------------------------
# A5 + A6
# ---------------------------------------------------------------------------

def ep_ll_workspace_bytes(num_ranks: int, num_tokens: int, num_experts: int) -> int:
    return int(_lib.ep_ll_workspace_bytes(num_ranks, num_tokens, num_experts))


@_on_tensor_device
def ep_ll_dispatch(x: torch.Tensor, topk_idx: torch.Tensor, num_experts: int, *,
                   use_fp8: bool = True, round_scale: bool = False, use_ue8m0: bool = False,
                   rank_mask: Optional[torch.Tensor] = None,
                   cumulative_local_expert_recv_stats: Optional[torch.Tensor] = None,
                   out: Optional[dict] = None, workspace: Optional[torch.Tensor] = None,
                   status=None, stream=None) -> dict:
    """x bf16 [R, T, H] -> dict of recv_x (uint8 e4m3 or bf16 [R, E_l, R*T, H]),
    recv_scales (fp32, or uint8 UE8M0, [R, E_l, R*T, H/128]; None for bf16),
    recv_count, recv_src_info, layout_range, ll_pos."""
    R, T, H = x.shape
    K = topk_idx.shape[2]
    E = num_experts
    El = E // R
    dev = x.device
    _need(x, torch.bfloat16, (R, T, H), "x")
    _need(topk_idx, torch.int64, (R, T, K), "topk_idx")
    if rank_mask is not None:
        _need(rank_mask, torch.int32, (R,), "rank_mask")
    if cumulative_local_expert_recv_stats is not None:
        _need(cumulative_local_expert_recv_stats, torch.int32, (R, El),
              "cumulative_local_expert_recv_stats")
    flags = (EP_LL_FP8 if use_fp8 else 0) | (EP_LL_ROUND_SCALE if round_scale else 0) | \
        (EP_LL_UE8M0 if use_ue8m0 else 0)
    o = dict(out or {})

    def get(name, shape, dtype):
        if o.get(name) is None:
            o[name] = torch.empty(shape, dtype=dtype, device=dev)
        _need(o[name], dtype, shape, name)
        return o[name]

    get("recv_x", (R, El, R * T, H), torch.uint8 if use_fp8 else torch.bfloat16)
    if use_fp8:
        get("recv_scales", (R, El, R * T, H // 128), torch.uint8 if use_ue8m0 else torch.float32)
    else:
        o["recv_scales"] = None
    get("recv_count", (R, El), torch.int32)
    get("recv_src_info", (R, El, R * T), torch.int32)
    get("layout_range", (R, El, R, 2), torch.int32)
    get("ll_pos", (R, T, K), torch.int32)
    need = ep_ll_workspace_bytes(R, T, E)
    if workspace is None:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=dev)
    rc = _lib.ep_ll_dispatch(
        _ptr(x), _ptr(topk_idx), _ptr(rank_mask), R, T, H, K, E, flags, _ptr(o["recv_x"]),
        _ptr(o["recv_scales"]), _ptr(o["recv_count"]), _ptr(o["recv_src_info"]),
        _ptr(o["layout_range"]), _ptr(o["ll_pos"]), _ptr(cumulative_local_expert_recv_stats),
        _ptr(workspace), workspace.numel(), _ptr(status), _stream(stream))
    _check(rc, "ep_ll_dispatch")
    return o


@_on_tensor_device
def ep_ll_combine(y: torch.Tensor, topk_idx: torch.Tensor, topk_weights: torch.Tensor,
                  ll_pos: torch.Tensor, *, rank_mask: Optional[torch.Tensor] = None,
                  out: Optional[torch.Tensor] = None, status=None,
                  stream=None) -> torch.Tensor:
    """y bf16 [R, E_l, R*T, H] -> out bf16 [R, T, H]."""
    R, El, cap, H = y.shape
    T = topk_idx.shape[1]
    K = topk_idx.shape[2]
    E = R * El
    _need(y, torch.bfloat16, (R, El, R * T, H), "y")
    _need(topk_idx, torch.int64, (R, T, K), "topk_idx")
    _need(topk_weights, torch.float32, (R, T, K), "topk_weights")
    _need(ll_pos, torch.int32, (R, T, K), "ll_pos")
    if out is None:
        out = torch.empty((R, T, H), dtype=torch.bfloat16, device=y.device)
    _need(out, torch.bfloat16, (R, T, H), "out")
    if rank_mask is not None:
        _need(rank_mask, torch.int32, (R,), "rank_mask")
    rc = _lib.ep_ll_combine(_ptr(y), _ptr(topk_idx), _ptr(topk_weights), _ptr(ll_pos),
                            _ptr(rank_mask), R, T, H, K, E, _ptr(out), _ptr(status),
                            _stream(stream))
    _check(rc, "ep_ll_combine")
    return out
