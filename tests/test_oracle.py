"""CPU tests of the float64 oracle against its pins (no GPU)."""
import math

import numpy as np
import pytest

import oracle
import workloads
from tests import oracle_pins as pins


@pytest.mark.parametrize("pin", pins.ALL_PINS, ids=lambda f: f.__name__)
def test_pin_holds(orc, pin):
    assert pin(orc) is None


@pytest.mark.parametrize("mutant", [1, 2, 3, 4, 5, 6, 7, 8, 9])
def test_each_planted_mistake_is_caught(mutant):
    """Every deliberately broken oracle build violates at least one pin."""
    bad = oracle.mutant(mutant)
    assert bad.lib.oracle_mutant() == mutant
    failures = [p.__name__ for p in pins.ALL_PINS if p(bad) is not None]
    assert failures, f"mutant {mutant} passed every pin"


def test_tsp_aggregate_mass(orc):
    """T = sum over KV heads of A; its total mass is w * H."""
    rng = np.random.default_rng(41)
    N, H, Hkv, d, w = 200, 8, 4, 64, 7
    q = workloads.f32_to_bf16_bits(rng.standard_normal((w, H, d)).astype(np.float32))
    k = workloads.f32_to_bf16_bits(rng.standard_normal((N, Hkv, d)).astype(np.float32))
    res = oracle.layer(q, k, H, Hkv, w, 1 / math.sqrt(d), pool=3, k_kv=20, k_tsp=40)
    assert np.allclose(res.T, res.A.sum(axis=0), rtol=0, atol=1e-15)
    assert abs(res.T.sum() - w * H) < 1e-9
    assert pins.check_selection(res.pooled_tsp, N, w, 40, res.idx_tsp) is None


def test_c1_planted_hitters_selected(orc):
    """Tiny GQA config: the 4 planted heavy-hitter keys are kept by every KV head."""
    cfg = workloads.C1
    lay = workloads.make_layer(cfg)
    res = oracle.layer(lay.q, lay.k, cfg.H, cfg.Hkv, cfg.w, cfg.scale, cfg.pool, cfg.k_kv)
    assert np.allclose(res.A.sum(axis=1), cfg.rows, atol=1e-9)
    for g in range(cfg.Hkv):
        assert pins.check_selection(res.pooled[g], cfg.N, cfg.w, cfg.k_kv, res.idx_kv[g]) is None
        assert np.all(np.isin(lay.hitters[0], res.idx_kv[g]))


def test_reduced_llama_shape_sinks_and_hitters_selected(orc):
    """Llama-3-8B head shapes at a reduced length: sinks (positions 0-3) and
    planted heavy hitters survive pooling and selection in every KV head."""
    cfg = workloads.shrink(workloads.C2, N=2048, k_kv=256, n_hitters=16, seed=102)
    lay = workloads.make_layer(cfg)
    res = oracle.layer(lay.q, lay.k, cfg.H, cfg.Hkv, cfg.w, cfg.scale, cfg.pool, cfg.k_kv)
    for g in range(cfg.Hkv):
        kept = res.idx_kv[g]
        assert np.all(np.isin(lay.sinks[0], kept))
        assert np.all(np.isin(lay.hitters[0], kept))


def test_cross_layer_accumulation(orc):
    """C_global after L layers is the sum of the per-layer aggregates (StructKV 2.A)."""
    cfg = workloads.shrink(workloads.C5, N=256, H=10, Hkv=2, w=8, k_kv=32, k_tsp=38,
                           n_hitters=4, layers=3)
    C = np.zeros((cfg.Hkv, cfg.N))
    per = []
    for ell in range(1, cfg.layers + 1):
        lay = workloads.make_layer(cfg, layer=ell)
        A = orc.window_scores(lay.q, lay.k, cfg.H, cfg.Hkv, cfg.w, cfg.scale)
        per.append(A)
        C += A
        assert np.array_equal(lay.hitters[0], workloads.make_layer(cfg, layer=1).hitters[0])
    assert abs(C.sum() - cfg.layers * cfg.w * cfg.H) < 1e-9
    assert np.allclose(C, np.sum(per, axis=0), rtol=0, atol=0)
