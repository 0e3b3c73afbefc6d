"""Conversions shared by the GPU tests."""
import numpy as np
import torch


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
