"""The multi-rank helpers with two gloo ranks on the CPU: every stream lands
on exactly one rank, ranks that run their own streams of the schedule agree
with one process that runs all of them, and times reduce to their maximum."""
import os
import socket

import pytest
import torch.distributed as dist
import torch.multiprocessing as mp

from same_step_kv_b200.dist import max_over_ranks, shard


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        from oracle.schedule import Geometry, RingModel
        mine = shard(8, rank, world)
        # each rank runs the bookkeeping of its own streams
        states = {}
        for sid in mine:
            ring = RingModel(Geometry(8, 4, 2, 64, ring_slots=3))
            ring.begin_chunk(3)
            ring.bootstrap()
            for _ in range(sid + 1):
                ring.begin_chunk(1)
            states[sid] = (ring.chunk, ring.current_slot(), ring.n_keys())
        gathered = [None] * world
        dist.all_gather_object(gathered, states)
        t = max_over_ranks(1.5 + rank)
        out.put((rank, gathered, t))
    finally:
        dist.destroy_process_group()


def test_shard_covers_every_stream_once():
    for n in (1, 7, 8, 9):
        for world in (1, 2, 3, 8):
            got = sorted(i for r in range(world) for i in shard(n, r, world))
            assert got == list(range(n))
    with pytest.raises(ValueError):
        shard(4, 2, 2)


def test_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    # single-process reference for all 8 streams
    from oracle.schedule import Geometry, RingModel
    ref = {}
    for sid in range(8):
        ring = RingModel(Geometry(8, 4, 2, 64, ring_slots=3))
        ring.begin_chunk(3)
        ring.bootstrap()
        for _ in range(sid + 1):
            ring.begin_chunk(1)
        ref[sid] = (ring.chunk, ring.current_slot(), ring.n_keys())
    for rank, gathered, t in res:
        merged = {}
        for d in gathered:
            assert not set(d) & set(merged)
            merged.update(d)
        assert merged == ref
        assert t == 2.5


# ---------------------------------------------------------------- heads
# Head-sharded (Ulysses-style) execution of one stream: two gloo ranks, each
# computing its heads with the fp64 oracle, against one process that computes
# every head.  Small geometry: 8 x 4 tokens per frame, 4 heads x 64, ring 2,
# the first chunk (3 frames, 2 steps), the sink pass, then chunks 1 and 2.
HS_W, HS_H, HS_HEADS, HS_D, HS_R = 8, 4, 4, 64, 2
HS_CALLS = [(0, 3, 0), (0, 3, 1), (0, 3, "sink"), (1, 1, 0), (1, 1, 1), (2, 1, 0), (2, 1, 1)]


def _hs_inputs(chunk, step, n):
    import numpy as np
    rng = np.random.default_rng([chunk, 7 if step == "sink" else step])
    return [rng.standard_normal((n, HS_HEADS, HS_D)) for _ in range(3)]


class _OracleHeads:
    """The compute step of HeadShard on the CPU: the oracle session of this
    rank's heads (test stand-in for the CUDA PvHeads)."""

    def __init__(self, heads):
        from oracle.schedule import Geometry
        from oracle.session import StreamSession
        self.ses = StreamSession(Geometry(HS_W, HS_H, heads, HS_D, ring_slots=HS_R))

    def __call__(self, layer, step, q, k, v):
        import torch
        qr = self.ses.rope_append(layer, step, q.numpy(), k.numpy(), v.numpy())
        o, _ = self.ses.chunk_attn(layer, step, qr)
        return torch.from_numpy(o)


def _hs_worker(rank, world, port, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import torch
        from oracle.session import SINK_STEP
        from same_step_kv_b200.dist import HeadShard, head_groups
        comp = _OracleHeads(HS_HEADS // world)
        hs = HeadShard(HS_HEADS, HS_D, comp)
        assert hs.head_range() == (rank * HS_HEADS // world, (rank + 1) * HS_HEADS // world)
        results = []
        for chunk, frames, step in HS_CALLS:
            n = frames * HS_W * HS_H
            if step == 0:
                comp.ses.begin_chunk(frames)
            ostep = SINK_STEP if step == "sink" else step
            a, b = rank * n // world, (rank + 1) * n // world
            q, k, v = (head_groups(torch.from_numpy(t[a:b]), world) for t in _hs_inputs(chunk, step, n))
            o = hs.layer(0, ostep, q, k, v)            # [world][n/world][hl][d]
            mine = o.permute(1, 0, 2, 3).reshape(b - a, HS_HEADS, HS_D)   # this rank's tokens
            results.append(mine.numpy())
        gathered = [None] * world
        dist.all_gather_object(gathered, results)
        out.put((rank, gathered))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 4])
def test_head_sharded_gloo_ranks_match_one_process(world):
    # 2 ranks of 2 heads, 4 ranks of 1 head
    import numpy as np
    from oracle.schedule import Geometry
    from oracle.session import SINK_STEP, StreamSession
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_hs_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = [q.get(timeout=180) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    ses = StreamSession(Geometry(HS_W, HS_H, HS_HEADS, HS_D, ring_slots=HS_R))
    gathered = res[0][1]
    for i, (chunk, frames, step) in enumerate(HS_CALLS):
        n = frames * HS_W * HS_H
        if step == 0:
            ses.begin_chunk(frames)
        ostep = SINK_STEP if step == "sink" else step
        qq, kk, vv = _hs_inputs(chunk, step, n)
        ref, _ = ses.chunk_attn(0, ostep, ses.rope_append(0, ostep, qq, kk, vv))
        got = np.concatenate([gathered[r][i] for r in range(world)], axis=0)
        # each head is computed by the same fp64 arithmetic on one rank or the other
        assert np.array_equal(got, ref), (chunk, step)


def test_head_groups_layout():
    import torch
    from same_step_kv_b200.dist import head_groups
    x = torch.arange(6 * 4 * 3).view(6, 4, 3)
    g = head_groups(x, 2)
    assert g.shape == (2, 6, 2, 3)
    assert torch.equal(g[1, 5], x[5, 2:4])
    with pytest.raises(ValueError):
        head_groups(x, 3)
