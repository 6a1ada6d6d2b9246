"""Seeded synthetic inputs for window-attention scoring and KV compaction.

This module holds ONLY input generation: shapes, random draws, the bf16
rounding of those draws and the planting of attention sinks / heavy-hitter
keys.  It contains none of the scoring, selection or gather arithmetic, so
both the float64 oracle (``oracle/``) and the CUDA path can take their inputs
from here without sharing any of the method.

Workload shapes follow the five configurations the method is measured on
(FastKV, "Token-Selective Propagation" and GQA-aware retention; StructKV,
"Global In-Degree Centrality"): a tiny GQA layer, a Llama-3-8B-shaped layer
at 32K and 128K tokens (the latter with TSP and a hidden-state gather), a
ragged batch passed as ``cu_seqlens``, and a 16-layer cross-layer
accumulation.

bf16 tensors are returned as ``numpy.uint16`` arrays holding the raw bf16
bit patterns (numpy has no bf16 dtype).  Draws are float32 N(0, 1) from
numpy's PCG64, rounded to bf16 with round-to-nearest-even.

Planting (the configurations say planted keys "must be selected" but give no
norm convention): a planted key of KV head g is
    K[j, g, :] = alpha * sqrt(d) * u_g + 0.1 * eps,    eps ~ N(0, I)
where u_g is the mean of the group's window queries (all query heads of the
group, all window rows), divided by its Euclidean norm.  The sqrt(d) factor
makes the planted logit alpha * (u_g . q) independent of the 1/sqrt(d)
softmax scale.
"""
from __future__ import annotations

import math
from concurrent.futures import ThreadPoolExecutor
from dataclasses import dataclass, field, replace
from typing import List, Optional

import numpy as np

_CHUNK = 1 << 22          # values per independent PCG64 stream
_THREADS = 8


# --------------------------------------------------------------------------- #
# configurations
# --------------------------------------------------------------------------- #
@dataclass(frozen=True)
class LayerConfig:
    name: str
    N: int                  # context tokens (per sequence for varlen: see lengths)
    H: int                  # query heads
    Hkv: int                # KV heads
    d: int                  # head dim
    w: int                  # observation window
    pool: int               # 1-D average-pool kernel along keys (1 = none)
    k_kv: int               # retained tokens per KV head (window included)
    k_tsp: Optional[int]    # TSP / propagation budget (window included) or None
    hidden: Optional[int]   # hidden size D of the hidden states, or None
    n_sinks: int
    sink_alpha: float
    n_hitters: int
    hitter_alpha: float
    seed: int
    with_v: bool = True
    batch: int = 1                      # >1: ragged batch
    len_range: Optional[tuple] = None   # (lo, hi) inclusive, ragged batch only
    layers: int = 1                     # >1: cross-layer accumulation
    layer_seed_base: int = 0            # per-layer Q/K seed = base + layer (1-based)

    @property
    def G(self) -> int:
        return self.H // self.Hkv

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.d)

    @property
    def rows(self) -> int:
        """Window query rows that feed one KV head's aggregate (G * w)."""
        return self.G * self.w


C1 = LayerConfig("tiny_n512_h8_kv2_d64", N=512, H=8, Hkv=2, d=64, w=8, pool=1,
                 k_kv=64, k_tsp=None, hidden=None, n_sinks=0, sink_alpha=0.0,
                 n_hitters=4, hitter_alpha=3.0, seed=1)
C2 = LayerConfig("llama3_8b_n32k", N=32768, H=32, Hkv=8, d=128, w=32, pool=7,
                 k_kv=2048, k_tsp=None, hidden=None, n_sinks=4, sink_alpha=4.0,
                 n_hitters=64, hitter_alpha=2.0, seed=2)
C3 = LayerConfig("llama3_8b_n128k_tsp", N=131072, H=32, Hkv=8, d=128, w=32, pool=7,
                 k_kv=int(0.1 * 131072), k_tsp=int(0.2 * 131072), hidden=4096,
                 n_sinks=4, sink_alpha=4.0, n_hitters=256, hitter_alpha=2.0, seed=3)
C4 = LayerConfig("varlen_b8_4k_64k", N=65536, H=32, Hkv=8, d=128, w=32, pool=7,
                 k_kv=1024, k_tsp=None, hidden=None, n_sinks=0, sink_alpha=0.0,
                 n_hitters=16, hitter_alpha=2.0, seed=4, batch=8,
                 len_range=(4096, 65536))
C5 = LayerConfig("structkv_16l_n64k_h40", N=65536, H=40, Hkv=8, d=128, w=32, pool=1,
                 k_kv=4096, k_tsp=int(0.15 * 65536), hidden=None, n_sinks=0,
                 sink_alpha=0.0, n_hitters=128, hitter_alpha=2.0, seed=5,
                 with_v=False, layers=16, layer_seed_base=5000)

CONFIGS = {1: C1, 2: C2, 3: C3, 4: C4, 5: C5}


def shrink(cfg: LayerConfig, **kw) -> LayerConfig:
    """A smaller variant of a configuration (same structure, new sizes)."""
    return replace(cfg, **kw)


# --------------------------------------------------------------------------- #
# random draws
# --------------------------------------------------------------------------- #
def _normal_f32(seedseq: np.random.SeedSequence, n: int) -> np.ndarray:
    """n float32 N(0,1) draws; chunk c uses the c-th child stream of seedseq,
    so the result does not depend on the thread count."""
    out = np.empty(n, dtype=np.float32)
    nch = (n + _CHUNK - 1) // _CHUNK
    kids = seedseq.spawn(nch)

    def work(c: int) -> None:
        g = np.random.Generator(np.random.PCG64(kids[c]))
        s = c * _CHUNK
        e = min(n, s + _CHUNK)
        g.standard_normal(e - s, dtype=np.float32, out=out[s:e])

    if nch == 1:
        work(0)
    else:
        with ThreadPoolExecutor(_THREADS) as ex:
            list(ex.map(work, range(nch)))
    return out


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 to bf16 (round-to-nearest-even); returns uint16 bits."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    if x.size >= (1 << 20):
        import torch  # multithreaded conversion for large tensors (same RNE rule)
        t = torch.from_numpy(x.reshape(-1)).to(torch.bfloat16)
        return t.view(torch.int16).numpy().view(np.uint16).reshape(x.shape)
    b = x.view(np.uint32).astype(np.uint64)
    b = (b + 0x7FFF + ((b >> 16) & 1)) >> 16
    return b.astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    """Exact widening of bf16 bit patterns to float32."""
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def torch_bf16(bits: np.ndarray, device=None):
    """uint16 bf16 bit patterns -> torch.bfloat16 tensor with the same bits
    (on `device` when given)."""
    import torch
    t = torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16)
    return t if device is None else t.to(device)


def normal_bf16(seedseq: np.random.SeedSequence, shape) -> np.ndarray:
    n = int(np.prod(shape))
    return f32_to_bf16_bits(_normal_f32(seedseq, n)).reshape(shape)


# --------------------------------------------------------------------------- #
# planting
# --------------------------------------------------------------------------- #
def group_directions(q_bits: np.ndarray, Hkv: int) -> np.ndarray:
    """u_g: mean window query of each KV head's query-head group, unit norm.
    q_bits: [w][H][d] bf16 bits.  Returns float64 [Hkv][d]."""
    q = bf16_bits_to_f32(q_bits).astype(np.float64)
    w, H, d = q.shape
    G = H // Hkv
    u = q.reshape(w, Hkv, G, d).mean(axis=(0, 2))
    return u / np.linalg.norm(u, axis=1, keepdims=True)


def plant(k_bits: np.ndarray, q_bits: np.ndarray, positions: np.ndarray,
          alphas: np.ndarray, noise_seed: np.random.SeedSequence) -> None:
    """Overwrite K rows at `positions` (in place) with alpha*sqrt(d)*u_g + 0.1*eps."""
    if len(positions) == 0:
        return
    N, Hkv, d = k_bits.shape
    u = group_directions(q_bits, Hkv)
    eps = _normal_f32(noise_seed, len(positions) * Hkv * d).reshape(len(positions), Hkv, d)
    vals = (alphas[:, None, None] * math.sqrt(d) * u[None, :, :] + 0.1 * eps.astype(np.float64))
    k_bits[positions] = f32_to_bf16_bits(vals.astype(np.float32))


def planted_positions(rng: np.random.Generator, n: int, w: int, n_sinks: int,
                      n_hitters: int) -> np.ndarray:
    """Heavy-hitter positions: uniform without replacement over the prefix
    [n_sinks, n - w); sorted."""
    lo, hi = n_sinks, n - w
    if n_hitters > hi - lo:
        raise ValueError("too many heavy hitters for the prefix")
    return np.sort(rng.choice(np.arange(lo, hi), size=n_hitters, replace=False))


# --------------------------------------------------------------------------- #
# layer / batch generation
# --------------------------------------------------------------------------- #
@dataclass
class Layer:
    cfg: LayerConfig
    q: np.ndarray                 # [B*w][H][d] bf16 bits (B = 1 unless ragged)
    k: np.ndarray                 # [total][Hkv][d] bf16 bits
    v: Optional[np.ndarray]       # same as k, or None
    x: Optional[np.ndarray]       # [total][D] bf16 bits, or None
    cu_seqlens: np.ndarray        # int32 [B+1]
    sinks: List[np.ndarray] = field(default_factory=list)    # per sequence, local
    hitters: List[np.ndarray] = field(default_factory=list)  # per sequence, local

    @property
    def batch(self) -> int:
        return len(self.cu_seqlens) - 1

    @property
    def total(self) -> int:
        return int(self.cu_seqlens[-1])

    def lengths(self) -> np.ndarray:
        return np.diff(self.cu_seqlens)


def _streams(seed: int):
    ss = np.random.SeedSequence(seed)
    return dict(zip(("q", "k", "v", "x", "pos", "noise"), ss.spawn(6)))


def ragged_lengths(cfg: LayerConfig) -> np.ndarray:
    st = _streams(cfg.seed)
    rng = np.random.Generator(np.random.PCG64(st["pos"]))
    lo, hi = cfg.len_range
    return rng.integers(lo, hi, size=cfg.batch, endpoint=True).astype(np.int64)


def make_layer(cfg: LayerConfig, with_x: Optional[bool] = None, seed: Optional[int] = None,
               layer: int = 0) -> Layer:
    """Generate one layer's inputs.

    Single sequence: Q_win [w][H][d], K/V [N][Hkv][d], X [N][D].
    Ragged batch (cfg.batch > 1): Q_win [B*w][H][d] (sequence-major), K/V/X
    packed along tokens, offsets in cu_seqlens.
    Cross-layer (cfg.layers > 1): `layer` in 1..L selects Q/K seed
    cfg.layer_seed_base + layer; planted positions come from cfg.seed and are
    the same in every layer.
    """
    if with_x is None:
        with_x = cfg.hidden is not None
    if cfg.layers > 1:
        if not 1 <= layer <= cfg.layers:
            raise ValueError("layer must be in 1..layers")
        st = _streams(cfg.layer_seed_base + layer)
        pos_st = _streams(cfg.seed)["pos"]
    else:
        st = _streams(cfg.seed if seed is None else seed)
        pos_st = st["pos"]

    pos_rng = np.random.Generator(np.random.PCG64(pos_st))
    if cfg.batch > 1:
        lo, hi = cfg.len_range
        lens = pos_rng.integers(lo, hi, size=cfg.batch, endpoint=True).astype(np.int64)
    else:
        lens = np.array([cfg.N], dtype=np.int64)
    cu = np.zeros(len(lens) + 1, dtype=np.int64)
    cu[1:] = np.cumsum(lens)
    total = int(cu[-1])
    B = len(lens)

    q = normal_bf16(st["q"], (B * cfg.w, cfg.H, cfg.d))
    k = normal_bf16(st["k"], (total, cfg.Hkv, cfg.d))
    v = normal_bf16(st["v"], (total, cfg.Hkv, cfg.d)) if cfg.with_v else None
    x = normal_bf16(st["x"], (total, cfg.hidden)) if (with_x and cfg.hidden) else None

    noise_kids = st["noise"].spawn(B)
    sinks, hitters = [], []
    for b in range(B):
        n = int(lens[b])
        s = np.arange(min(cfg.n_sinks, n - cfg.w), dtype=np.int64)
        hpos = planted_positions(pos_rng, n, cfg.w, cfg.n_sinks, cfg.n_hitters)
        pos = np.concatenate([s, hpos]).astype(np.int64)
        alphas = np.concatenate([np.full(len(s), cfg.sink_alpha),
                                 np.full(len(hpos), cfg.hitter_alpha)])
        kb = k[cu[b]:cu[b + 1]]
        plant(kb, q[b * cfg.w:(b + 1) * cfg.w], pos, alphas, noise_kids[b])
        sinks.append(s)
        hitters.append(hpos)
    return Layer(cfg, q, k, v, x, cu.astype(np.int32), sinks, hitters)


def make_codebooks(stages: int, size: int, d: int, seed: int) -> np.ndarray:
    """Random residual-VQ codebooks float32 [stages][size][d]: stage s draws
    N(0, 1) * 2^-s (each later stage refines a smaller residual).  Stand-ins
    for trained codebooks, which need training data."""
    g = np.random.Generator(np.random.PCG64(np.random.SeedSequence(seed)))
    scale = (2.0 ** -np.arange(stages, dtype=np.float64))[:, None, None]
    return (g.standard_normal((stages, size, d)) * scale).astype(np.float32)
