"""Host-side sharding of independent sequences across ranks (one process per GPU).

Window scoring, selection and compaction of one sequence never read another
sequence, so a ragged batch shards by whole sequences with no exchange on the
data path: each rank runs the varlen entry points on its own packed subset.
The only collective is outside the data path (the max over ranks of the
measured time, or gathering the per-rank results for a caller that wants
them on one rank).

assign_sequences() balances the token count per rank with the classic
longest-processing-time rule (sort by length, give each sequence to the
least-loaded rank; ties -> lower rank), which is deterministic, so every
rank computes the same assignment from the same lengths without talking to
the others.
"""
from __future__ import annotations

from typing import List, Sequence, Tuple

import numpy as np


def assign_sequences(lengths: Sequence[int], world: int) -> List[List[int]]:
    """Sequence ids per rank (each list ascending)."""
    if world < 1:
        raise ValueError("world must be >= 1")
    lengths = [int(x) for x in lengths]
    order = sorted(range(len(lengths)), key=lambda i: (-lengths[i], i))
    load = [0] * world
    out: List[List[int]] = [[] for _ in range(world)]
    for i in order:
        r = min(range(world), key=lambda q: (load[q], q))
        out[r].append(i)
        load[r] += lengths[i]
    return [sorted(x) for x in out]


def local_batch(cu_seqlens: np.ndarray, seq_ids: Sequence[int]) -> Tuple[np.ndarray, np.ndarray]:
    """For the sequences `seq_ids` of a packed batch: the local cu_seqlens
    (int32 [b+1]) and the packed source token of every local token (int64)."""
    cu = np.asarray(cu_seqlens, dtype=np.int64)
    lens = [int(cu[i + 1] - cu[i]) for i in seq_ids]
    local = np.zeros(len(seq_ids) + 1, dtype=np.int64)
    local[1:] = np.cumsum(lens)
    src = np.concatenate([np.arange(cu[i], cu[i + 1]) for i in seq_ids]) if seq_ids else np.zeros(0, np.int64)
    return local.astype(np.int32), src


def max_over_ranks(value: float, dist=None, device=None) -> float:
    """Max of a per-rank measurement (no-op without an initialised group)."""
    if dist is None or not dist.is_available() or not dist.is_initialized():
        return float(value)
    import torch
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())
