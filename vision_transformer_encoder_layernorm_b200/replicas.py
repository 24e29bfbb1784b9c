"""Multi-GPU use of the encoder: replicas.

The encoder of one image has no step that exchanges data across GPUs, and
packed images (cu_seqlens segments) never attend to each other, so N GPUs run
N independent replicas: each rank holds the full weights and encodes its own
images.  Nothing on the data path is a collective; the process group only
carries the barrier and the max-over-ranks step time of the benchmark.

``partition_images`` balances a packed batch over ranks longest-processing-
time first, with an image's cost modelled as its GEMM work (linear in its
tokens n) plus its attention work (quadratic in n).
"""
from __future__ import annotations

from typing import List, Sequence, Tuple


def image_cost(n_tokens: int, hidden: int, mlp: int) -> float:
    """Per-layer FLOP of one image of n tokens: projections 2n(4C^2 + 2CF)
    plus attention 4n^2 C."""
    n, C, F = float(n_tokens), float(hidden), float(mlp)
    return 2.0 * n * (4 * C * C + 2 * C * F) + 4.0 * n * n * C


def partition_images(grids: Sequence[Tuple[int, int]], world: int, hidden: int = 1152,
                     mlp: int = 4304) -> List[List[int]]:
    """Image indices per rank (each list in packing order).  Greedy LPT:
    images sorted by cost, each given to the currently least-loaded rank
    (ties to the lower rank).  Deterministic, so every rank computes the same
    answer without communicating."""
    if world < 1:
        raise ValueError("world must be >= 1")
    order = sorted(range(len(grids)),
                   key=lambda i: (-image_cost(grids[i][0] * grids[i][1], hidden, mlp), i))
    load = [0.0] * world
    parts: List[List[int]] = [[] for _ in range(world)]
    for i in order:
        r = min(range(world), key=lambda k: (load[k], k))
        parts[r].append(i)
        load[r] += image_cost(grids[i][0] * grids[i][1], hidden, mlp)
    return [sorted(p) for p in parts]


def max_over_ranks(value: float, device=None) -> float:
    """The maximum of a per-rank float over the default process group (the
    value itself without one)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()):
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64,
                     device=device if device is not None else "cpu")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())
