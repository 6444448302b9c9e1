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
