"""Multi-rank host logic on CPU (gloo, world size 2): sequence sharding of a
ragged batch, the max-over-ranks timing used by bench.py, and one layer
split by KV head (partition, all-reduced TSP row, column slices of the hidden
states) on the float64 oracle's scores."""
import os
import socket

import numpy as np
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from long_context_kv_window_b200 import shard


def test_assignment_covers_every_sequence_once_and_balances():
    rng = np.random.default_rng(0)
    lens = rng.integers(4096, 65537, size=8)
    for world in (1, 2, 3, 4, 8):
        parts = shard.assign_sequences(lens, world)
        flat = sorted(i for p in parts for i in p)
        assert flat == list(range(len(lens)))
        loads = [int(lens[p].sum()) for p in parts]
        # LPT bound: max load <= average + longest sequence
        assert max(loads) <= lens.sum() / world + lens.max()
    assert shard.assign_sequences([5, 5, 5, 5], 2) == [[0, 2], [1, 3]]


def test_local_batch_offsets():
    cu = np.array([0, 3, 10, 12, 20])
    local, src = shard.local_batch(cu, [1, 3])
    assert local.tolist() == [0, 7, 15]
    assert src.tolist() == list(range(3, 10)) + list(range(12, 20))


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, lens, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        parts = shard.assign_sequences(lens, world)   # computed independently on every rank
        mine = parts[rank]
        got = [None] * world
        dist.all_gather_object(got, mine)
        measured = 1.0 + rank * 0.5                   # a per-rank "elapsed time"
        mx = shard.max_over_ranks(measured, dist)
        q.put((rank, got, mx))
    finally:
        dist.destroy_process_group()


def test_two_ranks_agree_on_the_shards_and_the_max_time():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    lens = [40000, 5000, 65536, 4096, 30000, 12000, 64000, 8000]
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, lens, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    expect = shard.assign_sequences(lens, 2)
    for rank, got, mx in res:
        assert got == expect
        assert mx == 1.5
    assert sorted(i for p in expect for i in p) == list(range(len(lens)))


def test_head_and_column_ranges_partition_everything():
    for Hkv in (1, 2, 8):
        for world in range(1, Hkv + 1):
            r = shard.head_ranges(Hkv, world)
            assert r[0][0] == 0 and r[-1][1] == Hkv
            assert all(a[1] == b[0] for a, b in zip(r, r[1:]))
            assert max(b - a for a, b in r) - min(b - a for a, b in r) <= 1
    for world in (1, 2, 3, 8):
        c = shard.column_ranges(4096, world)
        assert c[0][0] == 0 and c[-1][1] == 4096 and all(a % 8 == 0 for a, _ in c)
        assert all(a[1] == b[0] for a, b in zip(c, c[1:]))


def _split_worker(rank, world, port, q):
    """One rank of a KV-head split of a small layer, on the oracle: its heads'
    scores, its partial all-head row, the row summed over ranks (gloo), the
    TSP set and its column slice of the hidden gather, its heads' K sets."""
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import oracle
        import workloads
        cfg = workloads.shrink(workloads.C3, N=4096, k_kv=410, k_tsp=819, hidden=512, n_hitters=16, seed=77)
        lay = workloads.make_layer(cfg)
        orc = oracle.get()
        g0, g1 = shard.head_ranges(cfg.Hkv, world)[rank]
        c0, c1 = shard.column_ranges(cfg.hidden, world)[rank]
        A = orc.window_scores(lay.q[:, g0 * cfg.G:g1 * cfg.G, :], lay.k[:, g0:g1, :], (g1 - g0) * cfg.G, g1 - g0,
                              cfg.w, cfg.scale)
        T = torch.from_numpy(orc.sum_rows(A))
        dist.all_reduce(T, op=dist.ReduceOp.SUM)
        pt = orc.rank_scores(T.numpy(), cfg.N, cfg.w, cfg.pool)
        idx_tsp = orc.select_topk(pt, cfg.N, cfg.w, cfg.k_tsp)
        x_c, _ = orc.gather_rows(lay.x[:, c0:c1], idx_tsp)
        idx_kv, _ = orc.select_rows(A, cfg.N, cfg.w, cfg.pool, cfg.k_kv)
        q.put((rank, (g0, g1), (c0, c1), idx_tsp, pt, x_c, idx_kv))
    finally:
        dist.destroy_process_group()


def test_two_ranks_split_one_layer_by_kv_head():
    """The KV-head split reproduces the single-rank layer: the summed row
    ranks to the single-rank TSP set (near-tie band: the float64 sum runs in
    another order), each rank's K sets are the single-rank sets of its heads,
    and the column slices of the hidden gather concatenate to the full one."""
    import oracle
    import workloads
    from tests import parity
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_split_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=300) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    cfg = workloads.shrink(workloads.C3, N=4096, k_kv=410, k_tsp=819, hidden=512, n_hitters=16, seed=77)
    lay = workloads.make_layer(cfg)
    full = oracle.layer(lay.q, lay.k, cfg.H, cfg.Hkv, cfg.w, cfg.scale, cfg.pool, cfg.k_kv, cfg.k_tsp)
    assert [r[1] for r in res] == [(0, 4), (4, 8)] and [r[2] for r in res] == [(0, 256), (256, 512)]
    for rank, (g0, g1), _, idx_tsp, pt, _, idx_kv in res:
        parity.assert_selection_matches(idx_tsp, full.idx_tsp, full.pooled_tsp, cfg.N, cfg.w, cfg.k_tsp,
                                        what=f"TSP set on rank {rank}")
        np.testing.assert_allclose(pt, full.pooled_tsp, rtol=1e-12)
        assert np.array_equal(idx_kv, full.idx_kv[g0:g1])
    assert np.array_equal(res[0][3], res[1][3]), "the ranks must select the same TSP set"
    x_full, _ = oracle.get().gather_rows(lay.x, res[0][3])
    assert np.array_equal(np.concatenate([res[0][5], res[1][5]], axis=1), x_full)
