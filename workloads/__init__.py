"""Seeded synthetic inputs for MoE token routing (layout, dispatch, combine, LL).

This module only draws random inputs.  It holds none of the routing
arithmetic: no expert-to-rank mapping, no prefix sums, no copies, no
quantisation.  Both the CPU oracle (``oracle/``) and the CUDA path consume
what it returns, so that the two sides see byte-identical inputs.

Shapes follow the DeepEP pages (``Buffer.dispatch`` / ``low_latency_dispatch``
argument descriptions, "Python 接口" page, Dispatch API section; test-data
setup in the legacy-test analysis page, "Random data" / "Data prep"):

* ``x``            bf16 ``[R, T, H]`` (stored here as raw ``uint16`` bits)
* ``topk_idx``     int64 ``[R, T, K]``, ``-1`` marks an unselected slot
* ``topk_weights`` fp32 ``[R, T, K]``

Recipe (every config, seed 0 unless stated):

* bf16 ``x`` is N(0,1) drawn in fp32 and rounded to bf16 (round to nearest,
  ties to even) by ``torch.Tensor.to(torch.bfloat16)``.
* "top-k distinct uniform": per token, draw E independent U(0,1) keys and take
  the K experts with the smallest keys, in ascending key order.  This is
  sampling without replacement in draw order.
* "Zipf(s) popularity": Gumbel-top-K over ``log p_e + Gumbel(0,1)`` with
  ``p_e ~ (e+1)^-s``, taking the K largest keys in descending order, which is
  sequential sampling without replacement from ``p``.
* masked slots: exactly ``round(frac * T * K)`` slots per source rank, chosen
  uniformly without replacement, are set to ``-1``.
* weights: ``softmax(N(0,1)[K])`` in fp32 per token; a masked slot keeps its
  weight (the routing ignores it).
* per-rank streams: ``numpy.random.SeedSequence(seed).spawn(R)``, each wrapped
  in ``Generator(PCG64(.))``; rank r draws keys, then weights, then x.
"""
from __future__ import annotations

import dataclasses
from typing import Optional

import numpy as np

__all__ = ["Workload", "CONFIGS", "make", "bf16_bits_from_f32", "softmax_f32"]


@dataclasses.dataclass(frozen=True)
class Workload:
    """Sizes and distribution of one synthetic routing problem."""

    name: str
    R: int                 # simulated ranks (each one is a source and a destination)
    T: int                 # tokens per source rank
    H: int                 # hidden size (bf16 channels per token); 0 = no payload
    E: int                 # experts in total (E % R == 0)
    K: int                 # top-k slots per token
    routing: str = "uniform"   # "uniform" | "zipf"
    zipf_s: float = 1.2
    masked_frac: float = 0.0   # fraction of slots set to -1 (exact count per rank)
    num_src: Optional[int] = None  # source ranks holding tokens (default R)
    seed: int = 0

    @property
    def S(self) -> int:
        return self.R if self.num_src is None else self.num_src


# The five workloads of the hot path (sizes from the routing pages' own
# workloads).  "layout" has a single source rank.
CONFIGS = {
    "pr1": Workload("pr1", R=4, T=64, H=256, E=16, K=2),
    "layout": Workload("layout", R=8, T=4096, H=0, E=256, K=8, num_src=1),
    "normal": Workload("normal", R=8, T=4096, H=7168, E=256, K=8),
    "skewed": Workload("skewed", R=16, T=2048, H=4096, E=128, K=6,
                       routing="zipf", zipf_s=1.2, masked_frac=0.1),
    "ll": Workload("ll", R=32, T=128, H=7168, E=256, K=8),
}


def bf16_bits_from_f32(a: np.ndarray) -> np.ndarray:
    """fp32 -> bf16 bit patterns (uint16), round to nearest even, via torch."""
    import torch

    t = torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32))
    return t.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def softmax_f32(z: np.ndarray) -> np.ndarray:
    """Row softmax of an fp32 array, computed in fp32 (input synthesis only)."""
    z = z.astype(np.float32)
    m = z.max(axis=-1, keepdims=True)
    e = np.exp(z - m, dtype=np.float32)
    return (e / e.sum(axis=-1, keepdims=True, dtype=np.float32)).astype(np.float32)


def _draw_topk(rng: np.random.Generator, T: int, E: int, K: int, routing: str,
               zipf_s: float) -> np.ndarray:
    if routing == "uniform":
        keys = rng.random((T, E))
        order = np.argsort(keys, axis=1, kind="stable")
        return order[:, :K].astype(np.int64)
    if routing == "zipf":
        logp = -zipf_s * np.log(np.arange(1, E + 1, dtype=np.float64))
        g = rng.gumbel(size=(T, E))
        keys = logp[None, :] + g
        order = np.argsort(-keys, axis=1, kind="stable")
        return order[:, :K].astype(np.int64)
    raise ValueError(f"unknown routing {routing!r}")


def make(w: Workload, *, with_x: bool = True, ranks=None) -> dict:
    """Draw the inputs of workload ``w``.

    Returns a dict with ``topk_idx`` int64 [S,T,K], ``topk_weights`` fp32
    [S,T,K] and (if ``with_x`` and H > 0) ``x`` uint16 bf16 bits [S,T,H].
    ``ranks``: draw only these source ranks (same values as in the full draw,
    stacked in the order given), e.g. one process's own rank.
    """
    S, T, H, E, K = w.S, w.T, w.H, w.E, w.K
    if K > E:
        raise ValueError("K must not exceed E")
    children = np.random.SeedSequence(w.seed).spawn(S)
    which = list(range(S)) if ranks is None else [int(r) for r in ranks]
    n = len(which)
    idx = np.empty((n, T, K), dtype=np.int64)
    wts = np.empty((n, T, K), dtype=np.float32)
    x = np.empty((n, T, H), dtype=np.uint16) if (with_x and H > 0) else None
    for i, r in enumerate(which):
        rng = np.random.Generator(np.random.PCG64(children[r]))
        idx[i] = _draw_topk(rng, T, E, K, w.routing, w.zipf_s)
        if w.masked_frac > 0.0:
            n_mask = int(round(w.masked_frac * T * K))
            flat = rng.choice(T * K, size=n_mask, replace=False)
            v = idx[i].reshape(-1)
            v[flat] = -1
        wts[i] = softmax_f32(rng.standard_normal((T, K), dtype=np.float32))
        if x is not None:
            x[i] = bf16_bits_from_f32(rng.standard_normal((T, H), dtype=np.float32))
    out = {"topk_idx": idx, "topk_weights": wts}
    if x is not None:
        out["x"] = x
    return out
