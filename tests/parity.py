"""Comparison rules between the CUDA path and the float64 oracle.

Scores: elementwise |gpu - oracle| <= 1e-3 * |oracle| (bf16 inputs, fp32
accumulation).  Every aggregated score is a sum of positive terms, so there is
no cancellation and no absolute floor is needed.

Index sets: let s_k be the oracle's (k-w)-th largest ranking score and s_k1
the next one.  If s_k - s_k1 >= 1e-5 * s_k the sets must be identical.
Otherwise positions whose oracle score lies outside the band
|S - s_k| <= 1e-5 * s_k must agree, and inside the band both sides must keep
the same number of positions.  The GPU set must in any case be ascending,
unique, of the right size and contain the window.

Gathers: bit-exact.

Residual VQ codes: where the oracle's best and second-best distances of a
stage differ by more than 1e-4 of the best (float64 against the kernel's fp32
residual and distances), the codes must be identical; at a closer call the
kernel's codeword must be within that band of the best along the same
residual, and the row is not followed further (the residuals part ways).

Decode attention over the compacted cache: per query head,
max |gpu - oracle| <= 1e-3 * max |oracle| over the head's output row (the
outputs are signed sums that can cancel, so the row's largest magnitude sets
the scale; fp32 arithmetic keeps the error about 1e-6 of the weighted sum of
|v|, i.e. well inside this bound).
"""
from __future__ import annotations

import numpy as np

SCORE_RTOL = 1e-3
TIE_RTOL = 1e-5


def score_rel_err(gpu: np.ndarray, ref: np.ndarray) -> float:
    gpu = np.asarray(gpu, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    den = np.abs(ref)
    bad_zero = (den == 0) & (gpu != 0)
    if np.any(bad_zero):
        return float("inf")
    with np.errstate(divide="ignore", invalid="ignore"):
        r = np.where(den > 0, np.abs(gpu - ref) / den, 0.0)
    return float(r.max()) if r.size else 0.0


def assert_scores_close(gpu, ref, rtol: float = SCORE_RTOL, what: str = "scores"):
    err = score_rel_err(gpu, ref)
    assert err <= rtol, f"{what}: max relative error {err:.3e} > {rtol:.0e}"
    return err


def check_structure(idx: np.ndarray, n: int, w: int, k: int) -> None:
    idx = np.asarray(idx)
    if k >= n:
        assert np.array_equal(idx, np.arange(n)), "k >= n must keep every position"
        return
    assert idx.shape[0] == k, f"|set| {idx.shape[0]} != k {k}"
    assert np.all(np.diff(idx) > 0), "indices not strictly increasing"
    assert idx[0] >= 0 and idx[-1] < n, "index out of range"
    assert np.array_equal(idx[k - w:], np.arange(n - w, n)), "window not kept"


def assert_selection_matches(gpu_idx, orc_idx, orc_S, n: int, w: int, k: int, what: str = "selection"):
    """orc_S: the oracle's ranking scores of the n - w prefix positions."""
    gpu_idx = np.asarray(gpu_idx)
    check_structure(gpu_idx, n, w, k)
    if k >= n:
        return "all"
    kk = k - w
    S = np.asarray(orc_S, dtype=np.float64)
    L = n - w
    if kk == 0:
        assert np.array_equal(gpu_idx, np.asarray(orc_idx)), what
        return "exact"
    srt = np.sort(S)[::-1]
    s_k = srt[kk - 1]
    s_k1 = srt[kk] if kk < L else -np.inf
    if s_k - s_k1 >= TIE_RTOL * s_k:
        if not np.array_equal(gpu_idx, np.asarray(orc_idx)):
            g = set(gpu_idx[:kk].tolist())
            o = set(np.asarray(orc_idx)[:kk].tolist())
            raise AssertionError(f"{what}: sets differ (only gpu: {sorted(g - o)[:8]}, only oracle: "
                                 f"{sorted(o - g)[:8]})")
        return "exact"
    band = np.abs(S - s_k) <= TIE_RTOL * abs(s_k)
    g = np.zeros(L, bool)
    g[gpu_idx[:kk]] = True
    o = np.zeros(L, bool)
    o[np.asarray(orc_idx)[:kk]] = True
    assert np.array_equal(g[~band], o[~band]), f"{what}: sets differ outside the near-tie band"
    assert g[band].sum() == o[band].sum(), f"{what}: different counts inside the near-tie band"
    return "band"


def assert_decode_close(gpu, ref, rtol: float = SCORE_RTOL, what: str = "decode"):
    gpu = np.asarray(gpu, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    worst = 0.0
    for h in range(ref.shape[0]):
        scale = np.max(np.abs(ref[h]))
        err = np.max(np.abs(gpu[h] - ref[h])) / scale if scale > 0 else np.max(np.abs(gpu[h]))
        worst = max(worst, err)
        assert err <= rtol, f"{what}: head {h} error {err:.3e} of the row's largest magnitude > {rtol:.0e}"
    return worst


RVQ_BAND = 1e-4


def check_rvq_codes(gpu_codes, orc_codes, orc_gap, x_bits, C, what: str = "rvq"):
    """Returns the number of rows decided inside the near-tie band."""
    gpu_codes = np.asarray(gpu_codes)
    orc_codes = np.asarray(orc_codes)
    n, S = orc_codes.shape
    near = 0
    x = x_bits.astype(np.uint32) << 16
    xf = x.view(np.float32).astype(np.float64)
    for t in range(n):
        for s in range(S):
            if gpu_codes[t, s] == orc_codes[t, s]:
                continue
            # the residual the oracle ranked at this stage (earlier codes agree)
            r = xf[t] - sum(C[u][orc_codes[t, u]].astype(np.float64) for u in range(s))
            dist = np.sum((r[None, :] - C[s].astype(np.float64)) ** 2, axis=1)
            best = dist.min()
            assert orc_gap[t, s] <= RVQ_BAND * max(best, 1e-12), (
                f"{what}: row {t} stage {s}: code {gpu_codes[t, s]} != {orc_codes[t, s]} with a gap of "
                f"{orc_gap[t, s]:.3e} (best {best:.6e})")
            assert dist[gpu_codes[t, s]] - best <= RVQ_BAND * max(best, 1e-12), (
                f"{what}: row {t} stage {s}: code {gpu_codes[t, s]} is not a near-argmin")
            near += 1
            break
    return near
