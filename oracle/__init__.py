"""Float64 CPU oracle for window-attention token scoring, selection and compaction.

TEST INFRASTRUCTURE ONLY: the tests, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` use it; the product library never does.  It
shares no code with the CUDA path.

The arithmetic lives in ``kvc_oracle.c`` (plain loops, float64).  This module
compiles it with gcc on first use (``build()``), loads it with ctypes and
composes its steps into the per-layer pipelines the method runs:

  FastKV (gist.science 2502.01068) section 2.A -- window-attention scores at
  the TSP layer; the window tokens are always kept;
  FastKV section 2.B -- two independent budgets (TSP rate, KV retention
  rate) over the same scores;
  FastKV abstract (2502.01068) -- GQA-aware retention, one set per KV head;
  StructKV (gist.science 2604.06746) section 2.A -- C_global is the sum of
  the per-layer contributions; section 2.B -- entropy / sparsity / variance.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from dataclasses import dataclass
from typing import Optional

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "kvc_oracle.c")
_LIB = os.path.join(_HERE, "_build", "libkvc_oracle.so")


def build(mutant: int = 0, out: Optional[str] = None, force: bool = False) -> str:
    """Compile the C oracle (gcc, float64, no fast-math, no FMA contraction)."""
    out = out or (_LIB if mutant == 0 else os.path.join(_HERE, "_build", f"libkvc_oracle_m{mutant}.so"))
    if not force and os.path.exists(out) and os.path.getmtime(out) >= os.path.getmtime(_SRC):
        return out
    os.makedirs(os.path.dirname(out), exist_ok=True)
    tmp = out + f".tmp{os.getpid()}"
    cmd = ["gcc", "-O2", "-std=c11", "-fopenmp", "-ffp-contract=off", "-fno-fast-math",
           "-shared", "-fPIC", f"-DORACLE_MUTANT={int(mutant)}", _SRC, "-o", tmp, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, out)
    return out


_P = ctypes.c_void_p
_I64 = ctypes.c_int64
_I32 = ctypes.c_int


class Oracle:
    """ctypes view of one compiled oracle library (the real one or a mutant)."""

    def __init__(self, path: str):
        lib = ctypes.CDLL(path)
        lib.oracle_window_scores.argtypes = [_P, _I64, _I64, _P, _I64, _I64, _I64,
                                             _I32, _I32, _I32, _I32, ctypes.c_double, _P]
        lib.oracle_window_scores.restype = _I32
        lib.oracle_window_scores_lse.argtypes = [_P, _I64, _I64, _P, _I64, _I64, _I64, _I32, _I32, _I32, _I32,
                                                 ctypes.c_double, _P, _I64, _I64, _P]
        lib.oracle_window_scores_lse.restype = _I32
        lib.oracle_sum_rows.argtypes = [_P, _I32, _I64, _I64, _P]
        lib.oracle_sum_rows.restype = None
        lib.oracle_avg_pool.argtypes = [_P, _I64, _I32, _P]
        lib.oracle_avg_pool.restype = _I32
        lib.oracle_select_topk.argtypes = [_P, _I64, _I32, _I64, _P]
        lib.oracle_select_topk.restype = _I64
        lib.oracle_gather_rows.argtypes = [_P, _I64, _I64, _I64, _P, _I64, _P]
        lib.oracle_gather_rows.restype = _I64
        lib.oracle_layer_stats.argtypes = [_P, _I64, ctypes.c_double, _P]
        lib.oracle_layer_stats.restype = _I32
        lib.oracle_pivot_layer.argtypes = [_P, _I32, _I32, ctypes.c_double, _I32, _I32]
        lib.oracle_pivot_layer.restype = _I32
        lib.oracle_decode_attention.argtypes = [_P, _P, _P, _I32, _I32, _I64, _I32, ctypes.c_double, _P]
        lib.oracle_decode_attention.restype = _I32
        lib.oracle_prefill_attention.argtypes = [_P, _P, _P, _I64, _I32, _I32, _I32, ctypes.c_double, _P, _P]
        lib.oracle_prefill_attention.restype = _I32
        lib.oracle_rvq_encode.argtypes = [_P, _I64, _I64, _I32, _P, _I32, _I32, _P, _P]
        lib.oracle_rvq_encode.restype = _I32
        lib.oracle_max_threads.restype = _I32
        lib.oracle_mutant.restype = _I32
        self.lib = lib

    # -- single steps ------------------------------------------------------ #
    def window_scores(self, q: np.ndarray, k: np.ndarray, H: int, Hkv: int, w: int,
                      scale: float) -> np.ndarray:
        """A[g, j] (float64 [Hkv][N]) from bf16-bit Q_win [w][H][d] and K [N][Hkv][d]."""
        assert q.dtype == np.uint16 and k.dtype == np.uint16
        assert q.strides[2] == 2 and k.strides[2] == 2
        N, Hk, d = k.shape
        assert Hk == Hkv and q.shape[0] == w and q.shape[1] == H and q.shape[2] == d
        A = np.empty((Hkv, N), dtype=np.float64)
        rc = self.lib.oracle_window_scores(q.ctypes.data, q.strides[0] // 2, q.strides[1] // 2,
                                           k.ctypes.data, k.strides[0] // 2, k.strides[1] // 2,
                                           N, H, Hkv, d, w, float(scale), A.ctypes.data)
        if rc != 0:
            raise ValueError("oracle_window_scores: bad arguments")
        return A

    def window_scores_lse(self, q: np.ndarray, k: np.ndarray, lse: np.ndarray, H: int, Hkv: int, w: int,
                          scale: float) -> np.ndarray:
        """A[g, j] (float64 [Hkv][N]) with each window row's log-sum-exp given:
        lse [w][H] (any strides), lse[i, h] = ln sum over the keys row i of head
        h sees of exp(scale * q . k)."""
        assert q.dtype == np.uint16 and k.dtype == np.uint16
        assert q.strides[2] == 2 and k.strides[2] == 2
        N, Hk, d = k.shape
        assert Hk == Hkv and q.shape == (w, H, d)
        lse = np.asarray(lse, dtype=np.float64)
        assert lse.shape == (w, H)
        A = np.empty((Hkv, N), dtype=np.float64)
        rc = self.lib.oracle_window_scores_lse(q.ctypes.data, q.strides[0] // 2, q.strides[1] // 2,
                                               k.ctypes.data, k.strides[0] // 2, k.strides[1] // 2,
                                               N, H, Hkv, d, w, float(scale), lse.ctypes.data,
                                               lse.strides[0] // 8, lse.strides[1] // 8, A.ctypes.data)
        if rc != 0:
            raise ValueError("oracle_window_scores_lse: bad arguments")
        return A

    def sum_rows(self, rows: np.ndarray) -> np.ndarray:
        rows = np.ascontiguousarray(rows, dtype=np.float64)
        out = np.empty(rows.shape[1], dtype=np.float64)
        self.lib.oracle_sum_rows(rows.ctypes.data, rows.shape[0], rows.shape[1], rows.shape[1],
                                 out.ctypes.data)
        return out

    def avg_pool(self, x: np.ndarray, p: int) -> np.ndarray:
        x = np.ascontiguousarray(x, dtype=np.float64)
        y = np.empty_like(x)
        if self.lib.oracle_avg_pool(x.ctypes.data, x.shape[0], p, y.ctypes.data) != 0:
            raise ValueError("pool kernel must be odd and >= 1")
        return y

    def select_topk(self, S_prefix: np.ndarray, N: int, w: int, k: int) -> np.ndarray:
        S = np.ascontiguousarray(S_prefix, dtype=np.float64)
        assert S.shape[0] == N - w
        idx = np.empty(max(min(k, N), 1), dtype=np.int32)
        n = self.lib.oracle_select_topk(S.ctypes.data, N, w, k, idx.ctypes.data)
        if n < 0:
            raise ValueError("oracle_select_topk: bad arguments")
        return idx[:n].copy()

    def gather_rows(self, src: np.ndarray, idx: np.ndarray, nsrc: Optional[int] = None):
        """src: 2-D uint16 view [rows][row_elems] (row stride may exceed row_elems)."""
        assert src.dtype == np.uint16 and src.strides[1] == 2
        idx = np.ascontiguousarray(idx, dtype=np.int32)
        out = np.empty((idx.shape[0], src.shape[1]), dtype=np.uint16)
        bad = self.lib.oracle_gather_rows(src.ctypes.data, src.strides[0] // 2,
                                          src.shape[0] if nsrc is None else nsrc, src.shape[1],
                                          idx.ctypes.data, idx.shape[0], out.ctypes.data)
        return out, int(bad)

    def layer_stats(self, A_row: np.ndarray, mass_norm: float) -> np.ndarray:
        a = np.ascontiguousarray(A_row, dtype=np.float64)
        out = np.empty(3, dtype=np.float64)
        if self.lib.oracle_layer_stats(a.ctypes.data, a.shape[0], float(mass_norm),
                                       out.ctypes.data) != 0:
            raise ValueError("oracle_layer_stats: bad arguments")
        return out

    def pivot_layer(self, stats: np.ndarray, tau: float, l_min: int, l_max: int) -> int:
        """Pivot layer (1-based) from per-layer, per-KV-head statistics
        stats [L][Hkv][3] float32 (entropy, top-1% mass, variance)."""
        st = np.ascontiguousarray(stats, dtype=np.float32)
        assert st.ndim == 3 and st.shape[2] == 3
        r = int(self.lib.oracle_pivot_layer(st.ctypes.data, st.shape[0], st.shape[1], float(tau), int(l_min),
                                            int(l_max)))
        if r < 0:
            raise ValueError("oracle_pivot_layer: bad arguments")
        return r

    def decode_attention(self, q: np.ndarray, kc: np.ndarray, vc: np.ndarray, H: int, Hkv: int,
                         scale: float) -> np.ndarray:
        """out [H][d] float64: one decode query per head over the compacted
        cache kc, vc [Hkv][kk][d] (bf16 bits)."""
        q, kc, vc = (np.ascontiguousarray(a, dtype=np.uint16) for a in (q, kc, vc))
        Hk, kk, d = kc.shape
        assert Hk == Hkv and vc.shape == kc.shape and q.shape == (H, d)
        out = np.empty((H, d), dtype=np.float64)
        if self.lib.oracle_decode_attention(q.ctypes.data, kc.ctypes.data, vc.ctypes.data, H, Hkv, kk, d,
                                            float(scale), out.ctypes.data) != 0:
            raise ValueError("oracle_decode_attention: bad arguments")
        return out

    def prefill_attention(self, q: np.ndarray, k: np.ndarray, v: np.ndarray, H: int, Hkv: int,
                          scale: float):
        """Causal attention of one sequence: (out [N][H][d], lse [N][H]) in
        float64 from bf16 bits q [N][H][d], k and v [N][Hkv][d]."""
        q, k, v = (np.ascontiguousarray(a, dtype=np.uint16) for a in (q, k, v))
        N, Hq, d = q.shape
        assert Hq == H and k.shape == (N, Hkv, d) and v.shape == k.shape
        out = np.empty((N, H, d), dtype=np.float64)
        lse = np.empty((N, H), dtype=np.float64)
        if self.lib.oracle_prefill_attention(q.ctypes.data, k.ctypes.data, v.ctypes.data, N, H, Hkv, d,
                                             float(scale), out.ctypes.data, lse.ctypes.data) != 0:
            raise ValueError("oracle_prefill_attention: bad arguments")
        return out, lse

    def rvq_encode(self, x: np.ndarray, C: np.ndarray):
        """Residual VQ codes [n][S] int32 and per-stage gaps [n][S] float64 of
        bf16-bit rows x [n][d] against float32 codebooks C [S][M][d]."""
        x = np.ascontiguousarray(x, dtype=np.uint16)
        C = np.ascontiguousarray(C, dtype=np.float32)
        n, d = x.shape
        S, M, dc = C.shape
        assert dc == d
        codes = np.empty((n, S), dtype=np.int32)
        gap = np.empty((n, S), dtype=np.float64)
        if self.lib.oracle_rvq_encode(x.ctypes.data, d, n, d, C.ctypes.data, S, M, codes.ctypes.data,
                                      gap.ctypes.data) != 0:
            raise ValueError("oracle_rvq_encode: bad arguments")
        return codes, gap

    def max_threads(self) -> int:
        return int(self.lib.oracle_max_threads())

    # -- composed steps ---------------------------------------------------- #
    def rank_scores(self, A_row: np.ndarray, N: int, w: int, pool: int) -> np.ndarray:
        """Ranking scores of the prefix positions: pooled A[0 : N-w]."""
        prefix = np.ascontiguousarray(A_row[: N - w])
        return self.avg_pool(prefix, pool) if pool > 1 else prefix.copy()

    def select_rows(self, A: np.ndarray, N: int, w: int, pool: int, k: int):
        """Per-row selection; returns (idx [rows][min(k,N)], pooled [rows][N-w])."""
        pooled = np.stack([self.rank_scores(A[r], N, w, pool) for r in range(A.shape[0])])
        idx = np.stack([self.select_topk(pooled[r], N, w, k) for r in range(A.shape[0])])
        return idx, pooled

    def gather_kv(self, kv: np.ndarray, idx: np.ndarray):
        """kv [N][Hkv][d] bf16 bits, idx [Hkv][kk] -> out [Hkv][kk][d]."""
        N, Hkv, d = kv.shape
        outs, bad = [], 0
        for g in range(Hkv):
            o, b = self.gather_rows(kv[:, g, :], idx[g], nsrc=N)
            outs.append(o)
            bad += b
        return np.stack(outs), bad


_default: Optional[Oracle] = None


def get() -> Oracle:
    """The real (non-mutant) oracle, compiled on first use."""
    global _default
    if _default is None:
        _default = Oracle(build())
    return _default


def mutant(n: int) -> Oracle:
    return Oracle(build(mutant=n))


@dataclass
class LayerResult:
    A: np.ndarray                      # [Hkv][N] float64
    pooled: np.ndarray                 # [Hkv][N-w]
    idx_kv: np.ndarray                 # [Hkv][min(k_kv, N)] int32
    T: Optional[np.ndarray] = None     # [N] TSP aggregate
    pooled_tsp: Optional[np.ndarray] = None
    idx_tsp: Optional[np.ndarray] = None


def layer(q: np.ndarray, k: np.ndarray, H: int, Hkv: int, w: int, scale: float, pool: int,
          k_kv: int, k_tsp: Optional[int] = None, orc: Optional[Oracle] = None) -> LayerResult:
    """One sequence: scores -> per-KV-head retention (+ TSP set when k_tsp)."""
    orc = orc or get()
    N = k.shape[0]
    A = orc.window_scores(q, k, H, Hkv, w, scale)
    idx_kv, pooled = orc.select_rows(A, N, w, pool, k_kv)
    res = LayerResult(A=A, pooled=pooled, idx_kv=idx_kv)
    if k_tsp is not None:
        T = orc.sum_rows(A)
        pt = orc.rank_scores(T, N, w, pool)
        res.T, res.pooled_tsp = T, pt
        res.idx_tsp = orc.select_topk(pt, N, w, k_tsp)
    return res
