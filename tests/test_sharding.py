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


def _tp_worker(rank, world, port, out):
    """One rank of tensor parallelism over KV heads: it quantises and decodes
    only its KV heads (and their query heads) of a shared workload, with the
    oracle standing in for its GPU; the slices are gathered afterwards."""
    import numpy as np
    import torch
    import torch.distributed as dist
    from oracle import kvarn_oracle as O
    from bit_kv_cache_15_b200 import inputs
    from bit_kv_cache_15_b200.sharding import kv_head_shard
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        w = inputs.make_decode_workload("tp", [300, 129, 77], 8, 4, seed=91)
        kvh, qh = kv_head_shard(4, 8, rank, world)
        k = np.ascontiguousarray(w.k_full[:, kvh.start:kvh.stop])
        v = np.ascontiguousarray(w.v_full[:, kvh.start:kvh.stop])
        packed, scales = O.quantize_tiles(k, v, w.slot_mapping, len(kvh), w.num_blocks, 4, 2)
        tail = np.ascontiguousarray(w.tail[:, :, kvh.start:kvh.stop])
        q = np.ascontiguousarray(w.q[:, qh.start:qh.stop])
        mine = O.decode(q, packed, scales, tail, w.block_table, w.seq_lens, len(kvh), 4, 2)
        parts = [torch.zeros_like(torch.from_numpy(mine.astype(np.float32))) for _ in range(world)]
        dist.all_gather(parts, torch.from_numpy(mine.astype(np.float32)))
        out[rank] = np.concatenate([p.numpy() for p in parts], axis=1)
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_tensor_parallel_over_kv_heads_gloo():
    """Two ranks each take half the KV heads; their gathered outputs equal the
    whole problem decoded on one device."""
    import numpy as np
    from oracle import kvarn_oracle as O
    from bit_kv_cache_15_b200 import inputs
    from bit_kv_cache_15_b200.sharding import kv_head_shard
    world = 2
    port = _free_port()
    with mp.Manager() as m:
        out = m.dict()
        mp.spawn(_tp_worker, args=(world, port, out), nprocs=world, join=True)
        res = dict(out)
    w = inputs.make_decode_workload("tp", [300, 129, 77], 8, 4, seed=91)
    packed, scales = O.quantize_tiles(w.k_full, w.v_full, w.slot_mapping, 4, w.num_blocks, 4, 2)
    full = O.decode(w.q, packed, scales, w.tail, w.block_table, w.seq_lens, 4, 4, 2).astype(np.float32)
    assert np.array_equal(res[0], full) and np.array_equal(res[1], full)
    assert [tuple(r) for r in kv_head_shard(8, 64, 1, 2)] == [tuple(range(4, 8)), tuple(range(32, 64))]
    with pytest.raises(ValueError):
        kv_head_shard(8, 64, 0, 3)
