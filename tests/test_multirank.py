"""Multi-rank host logic on CPU (gloo, world size 2): sequence sharding of a
ragged batch and the max-over-ranks timing used by bench.py."""
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
