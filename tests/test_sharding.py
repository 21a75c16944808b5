"""Multi-rank host logic on CPU: shards are disjoint and cover the batch, and
the timing reduction returns the slowest rank's time (gloo, world size 2)."""
import os
import socket

import pytest
import torch.multiprocessing as mp

from bit_kv_cache_15_b200.sharding import max_over_ranks, rank_seed, shard_range


def test_shard_range_covers_disjointly():
    for units in (0, 1, 7, 8, 64, 101):
        for world in (1, 2, 3, 8):
            got = [shard_range(units, r, world) for r in range(world)]
            assert got[0][0] == 0 and got[-1][1] == units
            for (a, b), (c, d) in zip(got, got[1:]):
                assert b == c and b >= a
            sizes = [b - a for a, b in got]
            assert max(sizes) - min(sizes) <= 1
    with pytest.raises(ValueError):
        shard_range(8, 2, 2)
    assert len({rank_seed(5, r) for r in range(8)}) == 8


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    import torch.distributed as dist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        start, end = shard_range(16, rank, world)
        slowest = max_over_ranks(10.0 + rank)      # rank 1 is the slow one
        out[rank] = (start, end, slowest)
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_ranks_gloo():
    world = 2
    port = _free_port()
    with mp.Manager() as m:
        out = m.dict()
        mp.spawn(_worker, args=(world, port, out), nprocs=world, join=True)
        res = dict(out)
    assert res[0][:2] == (0, 8) and res[1][:2] == (8, 16)
    assert res[0][2] == res[1][2] == 11.0
