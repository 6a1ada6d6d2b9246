"""Helpers shared by the GPU parity tests (device transfer, oracle runs)."""
from __future__ import annotations

import numpy as np
import torch

import oracle
import workloads
from tests import parity


def dev_bf16(bits: np.ndarray, device="cuda") -> torch.Tensor:
    """uint16 bf16 bit patterns -> CUDA bfloat16 tensor (same bits)."""
    return workloads.torch_bf16(bits, device)


def host_bits(t: torch.Tensor) -> np.ndarray:
    return t.detach().view(torch.int16).cpu().numpy().view(np.uint16)


def check_layer(lay, cfg, gpu_scores, gpu_idx, orc_res=None, pool=None, k=None, what=""):
    """Scores within tolerance and per-KV-head selections per the band rule."""
    pool = cfg.pool if pool is None else pool
    k = cfg.k_kv if k is None else k
    N = lay.k.shape[0]
    res = orc_res or oracle.layer(lay.q, lay.k, cfg.H, cfg.Hkv, cfg.w, cfg.scale, pool, k)
    err = parity.assert_scores_close(gpu_scores, res.A, what=f"{what} scores")
    kinds = []
    for g in range(cfg.Hkv):
        kinds.append(parity.assert_selection_matches(gpu_idx[g], res.idx_kv[g], res.pooled[g], N, cfg.w, k,
                                                     what=f"{what} head {g}"))
    return res, err, kinds
