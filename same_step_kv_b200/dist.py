"""Multi-process plumbing: one process per GPU over torch.distributed.

Two ways to spread the same-step KV path over ranks:

* by stream: generation streams (one per prompt) are independent, so each
  rank serves its own streams with its own KV store and no exchange
  (`shard`); the only collective is the maximum over ranks of a measured
  time (`max_over_ranks`).
* by head (`HeadShard`): one stream's chunk is split the way the blog
  "Learning Video Generation from the Wan2.2 Source Code" describes for
  Ulysses sequence parallelism (chapter 8, the "dimension exchange"): before
  and after the attention each rank holds a slice of the chunk's tokens with
  every head; during it, every token of the chunk for a slice of the heads.
  Each rank keeps the KV rings of its own heads only (a store configured for
  heads / world heads).  Two all-to-alls per layer over NCCL move q, k, v in
  and the attention output back.
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


# ------------------------------------------------------------------ heads
def head_groups(x: torch.Tensor, world: int) -> torch.Tensor:
    """Token-major [tokens][heads][d] -> head-group-major [world][tokens][heads/world][d]
    (a copy).  On the sequence side of HeadShard each rank's tokens are kept in
    this layout, so that the block bound for rank g is contiguous; a projection
    that feeds HeadShard writes it directly."""
    t, h, d = x.shape
    if h % world:
        raise ValueError("heads not divisible by the number of ranks")
    return x.view(t, world, h // world, d).permute(1, 0, 2, 3).contiguous()


class HeadShard:
    """One rank of the head-sharded chunk attention of one stream.

    world ranks; rank r serves heads [r * hl, (r + 1) * hl) with hl =
    heads / world for every token of the chunk, and holds tokens [r * n / world,
    (r + 1) * n / world) of an n-token chunk for every head before and after
    the attention.

    layer(layer, step, q, k, v): q, k, v are this rank's tokens in head-group-
    major layout [world][n / world][hl][d] (block g = heads of rank g), from
    the projection.  One all_to_all each brings every token of this rank's
    heads, token-major [n][hl][d], which is what the compute step takes; its
    output [n][hl][d] goes back by one more all_to_all, to this rank's tokens
    for every head, head-group-major [world][n / world][hl][d].

    compute(layer, step, q, k, v) -> out does RoPE, append and attention of
    this rank's heads on its own store: `PvHeads` is the CUDA one.  With a
    single rank the exchanges are the identity and no process group is used.
    """

    def __init__(self, heads: int, head_dim: int, compute, rank: int | None = None,
                 world: int | None = None):
        r, w = rank_world()
        self.rank = r if rank is None else rank
        self.world = w if world is None else world
        if heads % self.world:
            raise ValueError("heads not divisible by the number of ranks")
        self.heads, self.head_dim = heads, head_dim
        self.hl = heads // self.world
        self.compute = compute

    def head_range(self) -> tuple[int, int]:
        return self.rank * self.hl, (self.rank + 1) * self.hl

    def _to_heads(self, x: torch.Tensor) -> torch.Tensor:
        # [world][n/world][hl][d] of this rank's tokens -> [n][hl][d] of its heads
        if self.world == 1:
            return x.reshape(-1, self.hl, self.head_dim)
        out = torch.empty_like(x)
        dist.all_to_all_single(out, x.contiguous())
        return out.view(-1, self.hl, self.head_dim)

    def _to_tokens(self, o: torch.Tensor) -> torch.Tensor:
        # [n][hl][d] of this rank's heads -> [world][n/world][hl][d] of its tokens
        n = o.shape[0]
        if n % self.world:
            raise ValueError("chunk tokens not divisible by the number of ranks")
        o = o.reshape(self.world, n // self.world, self.hl, self.head_dim)
        if self.world == 1:
            return o
        out = torch.empty_like(o)
        dist.all_to_all_single(out, o.contiguous())
        return out

    def layer(self, layer: int, step: int, q: torch.Tensor, k: torch.Tensor, v: torch.Tensor):
        for t in (q, k, v):
            if t.dim() != 4 or t.shape[0] != self.world or t.shape[2] != self.hl:
                raise ValueError("q, k, v must be [world][tokens / world][heads / world][d]")
        out = self.compute(layer, step, self._to_heads(q), self._to_heads(k), self._to_heads(v))
        return self._to_tokens(out)


class PvHeads:
    """HeadShard's compute step on the GPU: pv_rope_append and pv_chunk_attn of
    one stream on this rank's store (configured for heads / world heads)."""

    def __init__(self, store, stream: int = 0, cuda_stream=None):
        from . import pv
        self.pv = pv
        self.store, self.stream, self.cuda_stream = store, stream, cuda_stream

    def __call__(self, layer, step, q, k, v):
        pv, c = self.pv, self.store.cfg
        n = q.shape[0]
        q_rot = torch.empty(c.heads * n * c.head_dim, dtype=torch.bfloat16, device=q.device)
        out = torch.empty(n, c.heads, c.head_dim, dtype=torch.bfloat16, device=q.device)
        pv.pv_rope_append(self.store.handle, [self.stream], layer, step, q, k, v, q_rot,
                          self.cuda_stream)
        pv.pv_chunk_attn(self.store.handle, [self.stream], layer, step, q_rot, out, None,
                         self.cuda_stream)
        return out
