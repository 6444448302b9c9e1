"""Multi-process plumbing: one process per GPU over torch.distributed.

The same-step KV path shards without any exchange: generation streams (one
per prompt) are independent, and so are heads, so each rank serves its own
streams with its own KV store.  The only collective is the maximum over
ranks of a measured time, which the benchmark reports.
"""
from __future__ import annotations

import torch
import torch.distributed as dist


def rank_world() -> tuple[int, int]:
    if dist.is_available() and dist.is_initialized():
        return dist.get_rank(), dist.get_world_size()
    return 0, 1


def shard(n_items: int, rank: int, world: int) -> list[int]:
    """Items (streams) of one rank, round-robin: each item on exactly one rank."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError("rank outside 0..world-1")
    return list(range(rank, n_items, world))


def max_over_ranks(x: float) -> float:
    """Maximum of x over all ranks (x itself without a process group)."""
    _, world = rank_world()
    if world == 1:
        return float(x)
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([float(x)], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())
