"""One rank per GPU: the sharded form of the routing path.

The DeepEP "Python 接口" page's Buffer, for one rank of R: each rank allocates
its receive buffers, the ranks all-gather IPC handles over a
torch.distributed group ("Distributed / ProcessGroup"), and every rank then
writes its tokens' rows and metadata straight into the destinations'
buffers and, at combine, reads its tokens' rows back from them.  The notify
step all-gathers each rank's per-destination and per-expert counts (DeepEP
PR #720 page, non-cached dispatch notify); every rank turns the gathered
counts into the same rank prefix matrix.

This module is argument marshalling and the control plane only -- the layout,
prefix matrix, positions, row moves and reduction run in the library's
kernels (``ep_get_dispatch_layout``, ``ep_shard_notify``,
``ep_shard_dispatch``, ``ep_shard_combine``; for the low-latency pair
``ep_shard_ll_counts``, ``ep_shard_ll_dispatch``, ``ep_shard_ll_combine``,
whose per-expert counts are all-gathered the same way).  The process group carries the
IPC handles, the count rows and the synchronisation between phases: with an
NCCL group the counts are gathered on the device and the synchronisation is
a one-element all-reduce on the current stream (no host round trip); with a
gloo group (CPU tests, or several processes sharing one GPU) the counts go
through the host and the synchronisation is a stream sync plus a barrier.
No kernel ever waits for another rank's kernel.

Results are bit-identical to the single-GPU path on the stacked inputs:
rank r's send positions are row r of the single-GPU send_pos, destination
d's receive rows are the single-GPU rows of d, and combine reduces in the
same ascending-destination fp32 order.
"""
from __future__ import annotations

import ctypes
from typing import Optional

import torch
import torch.distributed as dist

from . import (EP_LL_FP8, EP_LL_ROUND_SCALE, EP_LL_UE8M0, EPError, _check, _lib, _need, _ptr,
               ep_get_dispatch_layout, new_status)

IPC_HANDLE_BYTES = 64
_ALIGN = 256


def _round(n: int, a: int = _ALIGN) -> int:
    return (n + a - 1) // a * a


def region_layout(capacity: int, hidden: int, num_topk: int, expert_outputs: bool) -> dict:
    """Byte offsets and sizes of one rank's shared region (the same on every
    rank): name -> (offset, shape, dtype)."""
    cap, H, K = capacity, hidden, num_topk
    parts = [("recv_x", (cap, H), torch.bfloat16, 2),
             ("recv_topk_idx", (cap, K), torch.int64, 8),
             ("recv_topk_weights", (cap, K), torch.float32, 4),
             ("recv_src_idx", (cap,), torch.int32, 4)]
    if expert_outputs:
        parts.append(("y", (cap, H), torch.bfloat16, 2))
    return _pack(parts)


def ll_region_layout(num_ranks: int, num_tokens: int, hidden: int, local_experts: int,
                     use_fp8: bool = True, ue8m0: bool = False) -> dict:
    """The low-latency region of one rank (destination of its E_l experts):
    slabs [E_l, R*T, H] (e4m3 bytes or bf16), FP8 scales [E_l, R*T, H/128]
    (fp32, or UE8M0 bytes), recv_src_info [E_l, R*T], layout_range
    [E_l, R, 2] and the experts' output slabs ``ll_y`` [E_l, R*T, H] bf16
    that combine reads (legacy-test page, low_latency_dispatch outputs and
    low_latency_combine input)."""
    cap, H, El = num_ranks * num_tokens, hidden, local_experts
    parts = [("ll_recv_x", (El, cap, H), torch.uint8 if use_fp8 else torch.bfloat16,
              1 if use_fp8 else 2)]
    if use_fp8:
        parts.append(("ll_recv_scales", (El, cap, H // 128),
                      torch.uint8 if ue8m0 else torch.float32, 1 if ue8m0 else 4))
    parts += [("ll_recv_src_info", (El, cap), torch.int32, 4),
              ("ll_layout_range", (El, num_ranks, 2), torch.int32, 4),
              ("ll_y", (El, cap, H), torch.bfloat16, 2)]
    return _pack(parts)


def _pack(parts) -> dict:
    """Consecutive 256-byte-aligned parts: name -> (offset, shape, dtype)."""
    out, off = {}, 0
    for name, shape, dtype, size in parts:
        n = size
        for dim in shape:
            n *= dim
        out[name] = (off, shape, dtype)
        off += _round(max(n, 1))
    out["_bytes"] = off
    return out


# numpy type strings of __cuda_array_interface__; bf16 travels as int16
_TYPESTR = {torch.bfloat16: "<i2", torch.int64: "<i8", torch.float32: "<f4", torch.int32: "<i4",
            torch.uint8: "|u1"}


def _view(ptr: int, shape, dtype, device) -> torch.Tensor:
    """A tensor over device memory the library allocated (no copy, not owned)."""
    class _Mem:
        pass
    m = _Mem()
    m.__cuda_array_interface__ = {"shape": tuple(shape), "typestr": _TYPESTR[dtype],
                                  "data": (int(ptr), False), "version": 3, "strides": None}
    t = torch.as_tensor(m, device=device)
    if dtype == torch.bfloat16:
        t = t.view(torch.bfloat16)
    return t


def allgather_rows(row: torch.Tensor, group=None) -> torch.Tensor:
    """Every rank's `row` stacked in rank order, on row's device.  NCCL: on
    the device, ordered on the current stream; other backends: through the
    host."""
    ws = dist.get_world_size(group)
    if dist.get_backend(group) == "nccl":
        out = torch.empty((ws,) + tuple(row.shape), dtype=row.dtype, device=row.device)
        dist.all_gather_into_tensor(out, row.contiguous(), group=group)
        return out
    host = row.detach().cpu().contiguous()
    parts = [torch.empty_like(host) for _ in range(ws)]
    dist.all_gather(parts, host, group=group)
    return torch.stack(parts).to(row.device)


def exchange_handles(handle: bytes, group=None) -> list:
    """Every rank's IPC handle, in rank order."""
    out = [None] * dist.get_world_size(group)
    dist.all_gather_object(out, handle, group=group)
    return out


class ShardedBuffer:
    """This rank's receive buffers, mapped by every other rank, and the
    per-rank state of the sharded dispatch / combine.

    num_tokens (T) tokens per rank, hidden (H), num_topk (K), num_experts (E,
    E % R == 0); capacity rows per destination (default R*T, which never
    overflows).  expert_outputs: also share a [cap, H] buffer ``y`` that the
    experts write and combine reads (without it combine reads recv_x back:
    identity experts)."""

    def __init__(self, group, num_tokens: int, hidden: int, num_topk: int, num_experts: int,
                 capacity: Optional[int] = None, expert_outputs: bool = False, device=None):
        self.group = group
        self.R = dist.get_world_size(group)
        self.rank = dist.get_rank(group)
        self.T, self.H, self.K, self.E = num_tokens, hidden, num_topk, num_experts
        if self.E % self.R != 0:
            raise EPError("num_experts must be a multiple of the number of ranks")
        self.El = self.E // self.R
        self.cap = self.R * self.T if capacity is None else int(capacity)
        self.device = torch.device("cuda", torch.cuda.current_device()) if device is None \
            else torch.device(device)
        self.nccl = dist.get_backend(group) == "nccl"
        self.layout = region_layout(self.cap, self.H, self.K, expert_outputs)
        self._bases = []   # this rank's regions (freed at close)
        self._peers = []   # peers' regions mapped here (unmapped at close)
        self.tables, self.buffers = {}, {}
        self._ll = None
        with torch.cuda.device(self.device):
            self._share(self.layout)
            R, T, E = self.R, self.T, self.E
            dev = self.device
            self.send_pos = torch.empty((T, R), dtype=torch.int32, device=dev)
            self.rank_prefix_matrix = torch.empty((R, R), dtype=torch.int32, device=dev)
            self.recv_count = torch.empty((1,), dtype=torch.int32, device=dev)
            self.num_recv_tokens_per_expert = torch.empty((self.El,), dtype=torch.int32,
                                                          device=dev)
            self.ntpr = torch.empty((1, R), dtype=torch.int32, device=dev)
            self.ntpe = torch.empty((1, E), dtype=torch.int32, device=dev)
            self.in_rank = torch.empty((1, T, R), dtype=torch.bool, device=dev)
            self.workspace = torch.empty(max(int(_lib.ep_shard_workspace_bytes(R, T)), 16),
                                         dtype=torch.uint8, device=dev)
            self.notify_probe = torch.zeros((4,), dtype=torch.int64, device=dev)
            self.status = new_status(dev)
            self._one = torch.ones((1,), dtype=torch.int32, device=dev)
        self.sync()

    def _share(self, layout: dict) -> None:
        """Allocate this rank's region of `layout`, exchange IPC handles over
        the group (collective) and map every peer's region; adds one peer
        table and one local tensor per part."""
        p = ctypes.c_void_p()
        _check(_lib.ep_shard_alloc(layout["_bytes"], ctypes.byref(p)), "ep_shard_alloc")
        base = p.value
        self._bases.append(base)
        h = ctypes.create_string_buffer(IPC_HANDLE_BYTES)
        _check(_lib.ep_ipc_handle(base, h), "ep_ipc_handle")
        handles = exchange_handles(h.raw, self.group)
        bases = []
        for r, hr in enumerate(handles):
            if r == self.rank:
                bases.append(base)
                continue
            q = ctypes.c_void_p()
            _check(_lib.ep_ipc_open(ctypes.create_string_buffer(hr, IPC_HANDLE_BYTES),
                                    ctypes.byref(q)), "ep_ipc_open")
            self._peers.append(q.value)
            bases.append(q.value)
        parts = {k: v for k, v in layout.items() if not k.startswith("_")}
        # peer tables: entry d = rank d's buffer of each kind, in this process
        self.tables.update({name: torch.tensor([b + off for b in bases], dtype=torch.int64,
                                               device=self.device)
                            for name, (off, _, _) in parts.items()})
        # this rank's buffers, as tensors
        self.buffers.update({name: _view(base + off, shape, dtype, self.device)
                             for name, (off, shape, dtype) in parts.items()})

    # ---- cross-rank ordering -------------------------------------------------

    def sync(self) -> None:
        """All ranks' work issued so far (on the current stream) is complete
        and visible before any rank's later work runs."""
        if self.nccl:
            dist.all_reduce(self._one, group=self.group)   # stream-ordered
        else:
            torch.cuda.current_stream(self.device).synchronize()
            dist.barrier(group=self.group)

    # ---- dispatch / combine ----------------------------------------------------

    def dispatch(self, x: torch.Tensor, topk_idx: torch.Tensor,
                 topk_weights: Optional[torch.Tensor], expert_alignment: int = 1) -> dict:
        """x bf16 [T, H], topk_idx int64 [T, K], topk_weights fp32 [T, K] ->
        this rank's receive buffers (rows below recv_count are valid once
        every rank has dispatched; this call synchronises the ranks at its
        end) and the handle."""
        R, T, H, K, E, cap = self.R, self.T, self.H, self.K, self.E, self.cap
        _need(x, torch.bfloat16, (T, H), "x")
        _need(topk_idx, torch.int64, (T, K), "topk_idx")
        if topk_weights is not None:
            _need(topk_weights, torch.float32, (T, K), "topk_weights")
        stream = torch.cuda.current_stream(self.device).cuda_stream
        with torch.cuda.device(self.device):
            ep_get_dispatch_layout(topk_idx.view(1, T, K), E, R, num_tokens_per_rank=self.ntpr,
                                   num_tokens_per_expert=self.ntpe, is_token_in_rank=self.in_rank,
                                   status=self.status)
            counts = allgather_rows(self.ntpr[0], self.group)       # [R, R]
            ecounts = allgather_rows(self.ntpe[0], self.group)      # [R, E]
            t = self.tables
            rc = _lib.ep_shard_notify(
                _ptr(topk_idx), _ptr(topk_weights), _ptr(counts), _ptr(ecounts), self.rank, R, T,
                K, E, int(expert_alignment), cap, _ptr(t["recv_src_idx"]),
                _ptr(t["recv_topk_idx"]),
                _ptr(t["recv_topk_weights"]) if topk_weights is not None else None,
                _ptr(self.buffers["recv_topk_idx"]), _ptr(self.rank_prefix_matrix),
                _ptr(self.recv_count), _ptr(self.num_recv_tokens_per_expert),
                _ptr(self.send_pos), _ptr(self.notify_probe), _ptr(self.workspace),
                self.workspace.numel(), _ptr(self.status), stream)
            _check(rc, "ep_shard_notify")
            rc = _lib.ep_shard_dispatch(_ptr(x), _ptr(self.send_pos), R, T, H, cap,
                                        _ptr(t["recv_x"]), _ptr(self.status), stream)
            _check(rc, "ep_shard_dispatch")
        self.sync()
        out = {k: self.buffers[k] for k in ("recv_x", "recv_topk_idx", "recv_topk_weights",
                                            "recv_src_idx")}
        out.update(recv_count=self.recv_count, rank_prefix_matrix=self.rank_prefix_matrix,
                   num_recv_tokens_per_expert=self.num_recv_tokens_per_expert,
                   send_pos=self.send_pos, num_tokens_per_rank=self.ntpr[0],
                   num_tokens_per_expert=self.ntpe[0], is_token_in_rank=self.in_rank[0])
        return out

    def combine(self, expert_outputs: bool = False, bias: Optional[tuple] = None,
                combined_x: Optional[torch.Tensor] = None,
                combined_topk_weights: Optional[torch.Tensor] = None,
                with_weights: bool = True) -> tuple:
        """Gather this rank's tokens back from every destination and reduce
        them: from the shared ``y`` buffers (expert_outputs) or from recv_x
        (identity experts).  Synchronises the ranks before (every rank's
        experts are done) and after (no rank overwrites buffers still read)."""
        R, T, H, K, cap = self.R, self.T, self.H, self.K, self.cap
        if expert_outputs and "y" not in self.tables:
            raise EPError("this buffer has no shared expert-output region")
        if combined_x is None:
            combined_x = torch.empty((T, H), dtype=torch.bfloat16, device=self.device)
        _need(combined_x, torch.bfloat16, (T, H), "combined_x")
        if with_weights and combined_topk_weights is None:
            combined_topk_weights = torch.empty((T, K), dtype=torch.float32, device=self.device)
        b0, b1 = bias if bias is not None else (None, None)
        for b, nm in ((b0, "bias_0"), (b1, "bias_1")):
            if b is not None:
                _need(b, torch.bfloat16, (T, H), nm)
        stream = torch.cuda.current_stream(self.device).cuda_stream
        self.sync()
        with torch.cuda.device(self.device):
            rc = _lib.ep_shard_combine(
                _ptr(self.tables["y" if expert_outputs else "recv_x"]),
                _ptr(self.tables["recv_topk_weights"]) if with_weights else None,
                _ptr(self.send_pos), _ptr(b0), _ptr(b1), R, T, H, K, cap, _ptr(combined_x),
                _ptr(combined_topk_weights) if with_weights else None, _ptr(self.status), stream)
            _check(rc, "ep_shard_combine")
        self.sync()
        return combined_x, (combined_topk_weights if with_weights else None)

    # ---- the low-latency pair ------------------------------------------------

    def enable_low_latency(self, use_fp8: bool = True, use_ue8m0: bool = False) -> None:
        """Allocate and map this rank's low-latency region (collective: every
        rank calls it): the slabs of its E_l experts for every source rank's
        T tokens, their scales and handle, and the experts' output slabs."""
        if self._ll is not None:
            return
        if use_ue8m0 and not use_fp8:
            raise EPError("UE8M0 scales need the FP8 payload")
        R, T, E, El = self.R, self.T, self.E, self.El
        dev = self.device
        with torch.cuda.device(dev):
            self._share(ll_region_layout(R, T, self.H, El, use_fp8, use_ue8m0))
            self._ll = {
                "use_fp8": use_fp8, "ue8m0": use_ue8m0,
                "counts": torch.empty((E,), dtype=torch.int32, device=dev),
                "recv_count": torch.empty((El,), dtype=torch.int32, device=dev),
                "ll_pos": torch.empty((T, self.K), dtype=torch.int32, device=dev),
                "workspace": torch.empty(
                    max(int(_lib.ep_shard_ll_workspace_bytes(R, T, E)), 16), dtype=torch.uint8,
                    device=dev),
            }
        self.sync()

    def ll_dispatch(self, x: torch.Tensor, topk_idx: torch.Tensor, round_scale: bool = False,
                    rank_mask: Optional[torch.Tensor] = None,
                    cumulative_local_expert_recv_stats: Optional[torch.Tensor] = None) -> dict:
        """x bf16 [T, H], topk_idx int64 [T, K] -> this rank's slabs (as the
        destination of its E_l experts: rows below recv_count[j] are valid once
        every rank has dispatched; this call synchronises the ranks at its end)
        and ll_pos of its own tokens.  The per-expert counts travel by an
        all-gather (the notify exchange of the low-latency pair)."""
        if self._ll is None:
            raise EPError("call enable_low_latency() first")
        L = self._ll
        R, T, H, K, E, El = self.R, self.T, self.H, self.K, self.E, self.El
        _need(x, torch.bfloat16, (T, H), "x")
        _need(topk_idx, torch.int64, (T, K), "topk_idx")
        if rank_mask is not None:
            _need(rank_mask, torch.int32, (R,), "rank_mask")
        if cumulative_local_expert_recv_stats is not None:
            _need(cumulative_local_expert_recv_stats, torch.int32, (El,),
                  "cumulative_local_expert_recv_stats")
        if round_scale and not L["use_fp8"]:
            raise EPError("round_scale needs the FP8 payload")
        flags = (EP_LL_FP8 if L["use_fp8"] else 0) | \
            (EP_LL_ROUND_SCALE if round_scale or L["ue8m0"] else 0) | \
            (EP_LL_UE8M0 if L["ue8m0"] else 0)
        stream = torch.cuda.current_stream(self.device).cuda_stream
        t = self.tables
        with torch.cuda.device(self.device):
            rc = _lib.ep_shard_ll_counts(_ptr(topk_idx), _ptr(rank_mask), self.rank, R, T, K, E,
                                         _ptr(L["counts"]), _ptr(self.status), stream)
            _check(rc, "ep_shard_ll_counts")
            counts = allgather_rows(L["counts"], self.group)     # [R, E]
            rc = _lib.ep_shard_ll_dispatch(
                _ptr(x), _ptr(topk_idx), _ptr(rank_mask), _ptr(counts), self.rank, R, T, H, K, E,
                flags, _ptr(t["ll_recv_x"]),
                _ptr(t["ll_recv_scales"]) if L["use_fp8"] else None,
                _ptr(t["ll_recv_src_info"]), _ptr(t["ll_layout_range"]), _ptr(L["recv_count"]),
                _ptr(L["ll_pos"]), _ptr(cumulative_local_expert_recv_stats),
                _ptr(L["workspace"]), L["workspace"].numel(), _ptr(self.status), stream)
            _check(rc, "ep_shard_ll_dispatch")
        self.sync()
        b = self.buffers
        return {"recv_x": b["ll_recv_x"], "recv_scales": b.get("ll_recv_scales"),
                "recv_src_info": b["ll_recv_src_info"], "layout_range": b["ll_layout_range"],
                "recv_count": L["recv_count"], "ll_pos": L["ll_pos"],
                "expert_outputs": b["ll_y"]}

    def ll_combine(self, topk_idx: torch.Tensor, topk_weights: torch.Tensor,
                   rank_mask: Optional[torch.Tensor] = None,
                   out: Optional[torch.Tensor] = None) -> torch.Tensor:
        """Gather this rank's tokens' rows back from the destinations' expert
        output slabs (``ll_y``, written by the experts after ll_dispatch) and
        take their top-k weighted sum.  Synchronises the ranks before and
        after."""
        if self._ll is None:
            raise EPError("call enable_low_latency() first")
        R, T, H, K, E = self.R, self.T, self.H, self.K, self.E
        _need(topk_idx, torch.int64, (T, K), "topk_idx")
        _need(topk_weights, torch.float32, (T, K), "topk_weights")
        if rank_mask is not None:
            _need(rank_mask, torch.int32, (R,), "rank_mask")
        if out is None:
            out = torch.empty((T, H), dtype=torch.bfloat16, device=self.device)
        _need(out, torch.bfloat16, (T, H), "out")
        stream = torch.cuda.current_stream(self.device).cuda_stream
        self.sync()
        with torch.cuda.device(self.device):
            rc = _lib.ep_shard_ll_combine(_ptr(self.tables["ll_y"]), _ptr(topk_idx),
                                          _ptr(topk_weights), _ptr(self._ll["ll_pos"]),
                                          _ptr(rank_mask), self.rank, R, T, H, K, E, _ptr(out),
                                          _ptr(self.status), stream)
            _check(rc, "ep_shard_ll_combine")
        self.sync()
        return out

    def close(self) -> None:
        """Unmap the peers' buffers and free this rank's (after a final
        synchronisation, so no peer still reads or writes it)."""
        if not self._bases:
            return
        self.sync()
        torch.cuda.synchronize(self.device)
        with torch.cuda.device(self.device):
            for q in self._peers:
                _check(_lib.ep_ipc_close(q), "ep_ipc_close")
            self._peers = []
            self.buffers = {}
            self.tables = {}
        dist.barrier(group=self.group)   # every rank has unmapped this rank's buffers
        with torch.cuda.device(self.device):
            for b in self._bases:
                _check(_lib.ep_shard_free(b), "ep_shard_free")
        self._bases = []
