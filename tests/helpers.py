"""Conversions and sampled-oracle helpers shared by the GPU tests."""
import numpy as np
import torch

import oracle


def to_dev(a: np.ndarray, dtype=None) -> torch.Tensor:
    """numpy -> CUDA tensor; uint16 arrays are bf16 bit patterns."""
    if a.dtype == np.uint16:
        return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).cuda()
    t = torch.from_numpy(np.ascontiguousarray(a)).cuda()
    return t if dtype is None else t.to(dtype)


def to_host(t: torch.Tensor) -> np.ndarray:
    t = t.detach().cpu()
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).numpy().view(np.uint16)
    if t.dtype == torch.bool:
        return t.numpy().astype(np.uint8)
    return t.numpy()


def b2f(bits):
    return (np.asarray(bits, np.uint16).astype(np.uint32) << 16).view(np.float32)


def sampled_combine_oracle(y_dev: torch.Tensor, send_pos: np.ndarray, tokens: np.ndarray,
                           recv_w_dev=None):
    """Oracle combine of the flat tokens `tokens` only.  Pulls just the rows
    those tokens need from the device buffer y [R, cap, H] into a compact
    array and remaps send_pos to it."""
    R, cap, H = y_dev.shape
    T = send_pos.shape[1]
    flat = send_pos.reshape(R * T, R)[tokens]           # [n, R]
    n = len(tokens)
    sp_small = np.full((R, n, R), -1, np.int32)          # pretend R sources of n tokens
    rows_d, rows_p, slots = [], [], []
    for i in range(n):
        for d in range(R):
            p = flat[i, d]
            if 0 <= p < cap:
                rows_d.append(d)
                rows_p.append(p)
                slots.append((i, d))
    m = len(rows_d)
    ys = np.zeros((R, max(m, 1), H), np.uint16)
    if m:
        idx_d = torch.tensor(rows_d, device=y_dev.device)
        idx_p = torch.tensor(rows_p, device=y_dev.device)
        rows = to_host(y_dev[idx_d, idx_p])              # [m, H]
    rw_small = None
    if recv_w_dev is not None:
        K = recv_w_dev.shape[2]
        rw_small = np.zeros((R, max(m, 1), K), np.float32)
        if m:
            rws = to_host(recv_w_dev[idx_d, idx_p])
    for j, (i, d) in enumerate(slots):
        ys[d, j] = rows[j]
        sp_small[0, i, d] = j
        if rw_small is not None:
            rw_small[d, j] = rws[j]
    # put every sampled token under source 0 of a [R, n, R] problem
    sp_small = sp_small[:1].repeat(R, axis=0)
    sp_small[1:] = -1
    out, out_w = oracle.combine(ys, sp_small, rw_small, tokens=np.arange(n))
    return out[0], (out_w[0] if out_w is not None else None)
