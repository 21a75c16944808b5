"""Sharding of the hot path over ranks (one process per GPU).

The path splits into independent units -- quantisation tiles and decode
(sequence, KV head) problems -- with no exchange step between them.  N GPUs
either take their own sequences (data parallel) or their own KV heads with
the query heads that read them (tensor parallel over heads, the pages' TP
setting), and never communicate on the data path.  Only the benchmark's
timing uses a collective (the max of the per-rank elapsed times).
"""
from __future__ import annotations


def shard_range(global_units: int, rank: int, world: int) -> tuple[int, int]:
    """Contiguous block of units owned by `rank`: sizes differ by at most one."""
    if world <= 0 or not 0 <= rank < world:
        raise ValueError("bad rank / world")
    base, extra = divmod(global_units, world)
    start = rank * base + min(rank, extra)
    return start, start + base + (1 if rank < extra else 0)


def kv_head_shard(num_kv_heads: int, num_q_heads: int, rank: int, world: int) -> tuple[range, range]:
    """KV heads of `rank` and the query heads that read them.  Query head j
    reads KV head j // (Hq / Hkv), so a contiguous block of KV heads owns the
    matching contiguous block of query heads; world must divide Hkv."""
    if world <= 0 or not 0 <= rank < world or num_kv_heads % world or num_q_heads % num_kv_heads:
        raise ValueError("KV heads must split evenly over the ranks")
    per = num_kv_heads // world
    g = num_q_heads // num_kv_heads
    return range(rank * per, (rank + 1) * per), range(rank * per * g, (rank + 1) * per * g)


def rank_seed(seed: int, rank: int) -> int:
    """Seed of a rank's synthetic batch: distinct per rank, reproducible."""
    return int(seed) * 1000 + int(rank)


def max_over_ranks(value: float, group=None) -> float:
    """Largest per-rank value (the job's elapsed time), via all_reduce(MAX)."""
    import torch
    import torch.distributed as dist
    if not dist.is_available() or not dist.is_initialized():
        return float(value)
    backend = dist.get_backend(group)
    dev = torch.device("cuda", torch.cuda.current_device()) if backend == "nccl" else torch.device("cpu")
    t = torch.tensor([float(value)], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX, group=group)
    return float(t.item())
