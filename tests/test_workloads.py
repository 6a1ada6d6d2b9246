"""CPU tests of the seeded input generator (no method arithmetic lives there)."""
import numpy as np

import workloads


def test_bf16_rounding_paths_agree():
    """The small-array (bit formula) and large-array (torch) RNE paths agree,
    including exact ties."""
    rng = np.random.default_rng(0)
    x = rng.standard_normal(1 << 20).astype(np.float32)
    ties = ((np.arange(1 << 12, dtype=np.uint32) + 0x3C00) << 16 | 0x8000).view(np.float32)
    x[: ties.size] = ties
    big = workloads.f32_to_bf16_bits(x)
    small = np.concatenate([workloads.f32_to_bf16_bits(c) for c in np.split(x, 64)])
    assert np.array_equal(big, small)
    back = workloads.bf16_bits_to_f32(big)
    assert np.all(np.abs(back - x) <= np.abs(x) * 2.0 ** -8)


def test_generation_is_deterministic_and_shaped():
    cfg = workloads.C1
    a = workloads.make_layer(cfg)
    b = workloads.make_layer(cfg)
    assert a.q.shape == (cfg.w, cfg.H, cfg.d) and a.k.shape == (cfg.N, cfg.Hkv, cfg.d)
    assert np.array_equal(a.q, b.q) and np.array_equal(a.k, b.k) and np.array_equal(a.v, b.v)
    assert len(a.hitters[0]) == cfg.n_hitters
    assert np.all(a.hitters[0] < cfg.N - cfg.w) and np.all(np.diff(a.hitters[0]) > 0)


def test_ragged_batch_layout():
    cfg = workloads.shrink(workloads.C4, len_range=(100, 300), n_hitters=4)
    lay = workloads.make_layer(cfg)
    lens = lay.lengths()
    assert lay.batch == cfg.batch and np.all((lens >= 100) & (lens <= 300))
    assert lay.k.shape[0] == lay.total and lay.q.shape[0] == cfg.batch * cfg.w
    for b in range(cfg.batch):
        assert np.all(lay.hitters[b] < lens[b] - cfg.w)


def test_planted_keys_point_along_group_direction():
    cfg = workloads.C1
    lay = workloads.make_layer(cfg)
    u = workloads.group_directions(lay.q, cfg.Hkv)
    for j in lay.hitters[0]:
        kj = workloads.bf16_bits_to_f32(lay.k[j]).astype(np.float64)
        for g in range(cfg.Hkv):
            cos = kj[g] @ u[g] / np.linalg.norm(kj[g])
            assert cos > 0.99
