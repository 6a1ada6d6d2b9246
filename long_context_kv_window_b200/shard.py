"""Host-side sharding across ranks (one process per GPU).

Two splits:

* independent sequences (below): a ragged batch shards by whole sequences;
* one layer split by KV head (HeadSplitLayer, further below): every rank
  scores, selects and gathers the K/V of its own KV heads; the only exchange
  is the all-head TSP row, summed over ranks before the TSP selection, after
  which every rank ranks the same row and gathers its column slice of the
  hidden states.

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

from typing import Callable, List, Optional, Sequence, Tuple

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


# --------------------------------------------------------------------------- #
# one layer split by KV head
# --------------------------------------------------------------------------- #
def head_ranges(num_kv_heads: int, world: int) -> List[Tuple[int, int]]:
    """Contiguous KV-head ranges [g0, g1) per rank, sizes differing by at most one."""
    if world < 1 or world > num_kv_heads:
        raise ValueError(f"world must be in 1..{num_kv_heads}")
    base, extra = divmod(num_kv_heads, world)
    out, g = [], 0
    for r in range(world):
        n = base + (1 if r < extra else 0)
        out.append((g, g + n))
        g += n
    return out


def column_ranges(hidden: int, world: int, align: int = 8) -> List[Tuple[int, int]]:
    """Column ranges [c0, c1) of the hidden states per rank, in units of
    `align` columns (16 bytes of bf16), sizes differing by at most one unit."""
    if hidden % align:
        raise ValueError(f"hidden must be a multiple of {align}")
    units = hidden // align
    if world < 1 or world > units:
        raise ValueError(f"world must be in 1..{units}")
    base, extra = divmod(units, world)
    out, u = [], 0
    for r in range(world):
        n = base + (1 if r < extra else 0)
        out.append((u * align, (u + n) * align))
        u += n
    return out


class HeadSplitLayer:
    """The share of one layer that rank `rank` of `world` computes when the
    layer is split by KV head (FastKV 2.A / 2.B on a tensor-parallel layer):

      1. window scores of its KV heads [g0, g1) (their query heads
         [g0*G, g1*G)) over all n keys, and their partial all-head row;
      2. the partial rows summed over ranks (`reduce_sum`: an all-reduce, e.g.
         NCCL over NVLink, 4 bytes per key);
      3. the TSP selection of the summed row -- the same set on every rank --
         and the gather of its hidden-state columns [c0, c1);
      4. per-KV-head selection and K/V gather of its own heads (no exchange).

    Inputs are the full-layer tensors (q_win [w][H][d], k, v [n][Hkv][d],
    x [n][D]); the rank reads only its slices.  Outputs: idx_kv / k_c / v_c of
    its heads, idx_tsp, and x_c [k_tsp][c1 - c0]."""

    def __init__(self, rank: int, world: int, n: int, H: int, Hkv: int, d: int, w: int, k_kv: int, k_tsp: int,
                 hidden: int, device, pool_kernel: int = 1):
        import torch

        from long_context_kv_window_b200 import (_workspace, score_params, score_workspace_size,
                                                 select_workspace_size)
        if H % Hkv:
            raise ValueError("H must be a multiple of Hkv")
        self.rank, self.world = rank, world
        self.n, self.H, self.Hkv, self.d, self.w = n, H, Hkv, d, w
        self.G = H // Hkv
        self.k_kv, self.k_tsp, self.hidden, self.pool = k_kv, k_tsp, hidden, pool_kernel
        self.g0, self.g1 = head_ranges(Hkv, world)[rank]
        self.c0, self.c1 = column_ranges(hidden, world)[rank]
        hl = self.g1 - self.g0
        f32, i32, bf = torch.float32, torch.int32, torch.bfloat16
        self.params = score_params(hl * self.G, hl, d, w)
        self.scores = torch.empty((hl, n), dtype=f32, device=device)
        self.tsp = torch.empty((1, n), dtype=f32, device=device)
        self.ws_score = _workspace(score_workspace_size(self.params, 1, n), device)
        self.ws_sel_kv = _workspace(select_workspace_size(hl, 1, n), device)
        self.ws_sel_tsp = _workspace(select_workspace_size(1, 1, n), device)
        self.idx_kv = torch.empty((hl, min(k_kv, n)), dtype=i32, device=device)
        self.k_c = torch.empty((hl, min(k_kv, n), d), dtype=bf, device=device)
        self.v_c = torch.empty_like(self.k_c)
        self.idx_tsp = torch.empty((1, min(k_tsp, n)), dtype=i32, device=device)
        self.x_c = torch.empty((min(k_tsp, n), self.c1 - self.c0), dtype=bf, device=device)
        self.dev_err = torch.zeros(1, dtype=i32, device=device)

    def score_local(self, q_win, k, stream=None):
        """Step 1: this rank's window scores and its partial all-head row."""
        from long_context_kv_window_b200 import kvc_score
        qs = q_win[:, self.g0 * self.G:self.g1 * self.G, :]
        ks = k[:, self.g0:self.g1, :]
        kvc_score(qs, ks, scores=self.scores, tsp=self.tsp, ws=self.ws_score, dev_err=self.dev_err, stream=stream)
        return self.tsp

    def finish(self, k, v, x, stream=None):
        """Steps 3 and 4, once self.tsp holds the summed row."""
        from long_context_kv_window_b200 import kvc_gather_hidden, kvc_gather_kv, kvc_select_topk
        kvc_select_topk(self.tsp, self.w, self.pool, self.k_tsp, idx=self.idx_tsp, ws=self.ws_sel_tsp, stream=stream)
        kvc_gather_hidden(x[:, self.c0:self.c1], self.idx_tsp.view(-1), out=self.x_c, dev_err=self.dev_err,
                          stream=stream)
        kvc_select_topk(self.scores, self.w, self.pool, self.k_kv, idx=self.idx_kv, ws=self.ws_sel_kv, stream=stream)
        kvc_gather_kv(k[:, self.g0:self.g1, :], v[:, self.g0:self.g1, :], self.idx_kv, k_out=self.k_c,
                      v_out=self.v_c, dev_err=self.dev_err, stream=stream)

    def run(self, q_win, k, v, x, reduce_sum: Optional[Callable] = None, stream=None):
        """All steps; reduce_sum(tensor) sums the partial rows over the ranks in
        place (None with one rank), e.g. torch.distributed.all_reduce."""
        self.score_local(q_win, k, stream=stream)
        if reduce_sum is not None:
            reduce_sum(self.tsp)
        self.finish(k, v, x, stream=stream)
