"""The head-sharded driver (same_step_kv_b200.dist.HeadShard) with its CUDA
compute step on one GPU: with a single rank the exchanges are the identity,
so this runs the product path of every rank (head-group-major input, the
rank's store of heads / world heads, RoPE + append + chunk attention) and
checks it against the oracle session through a short schedule.  The
exchanges themselves are checked on the CPU with two gloo ranks
(test_dist_gloo.py)."""
import numpy as np
import pytest
import torch

from gpu_common import assert_attn_close, f64
from oracle.schedule import Geometry
from oracle.session import SINK_STEP, StreamSession
from same_step_kv_b200 import synth

pytestmark = pytest.mark.gpu


def test_head_shard_one_rank_matches_oracle():
    from same_step_kv_b200 import pv
    from same_step_kv_b200.dist import HeadShard, PvHeads, head_groups
    W, HH, H, D, R = 8, 4, 4, 128, 2
    T = W * HH
    cfg = pv.make_config(1, H, D, W, HH, ring_slots=R, max_frames=64)
    store = pv.KVStore(cfg)
    h = store.handle
    hs = HeadShard(H, D, PvHeads(store), rank=0, world=1)
    ses = StreamSession(Geometry(W, HH, H, D, ring_slots=R))
    calls = [(0, 3, 0), (0, 3, 1), (0, 3, "sink"), (1, 1, 0), (1, 1, 1), (2, 1, 0), (2, 1, 1),
             (3, 1, 0), (3, 1, 1)]
    for chunk, frames, step in calls:
        n = frames * T
        if step == 0:
            pv.pv_kv_begin_chunk(h, 0, frames)
            ses.begin_chunk(frames)
        if step == "sink":
            pv.pv_kv_begin_sink(h, 0)
        sarg = pv.PV_STEP_SINK if step == "sink" else step
        ostep = SINK_STEP if step == "sink" else step
        q, k, v = synth.chunk_qkv(0, chunk, 9 if step == "sink" else step, 0, n, H, D, "cuda")
        o = hs.layer(0, sarg, *(head_groups(t, 1) for t in (q, k, v)))
        torch.cuda.synchronize()
        assert o.shape == (1, n, H, D)
        ref, _ = ses.chunk_attn(0, ostep, ses.rope_append(0, ostep, f64(q), f64(k), f64(v)))
        assert_attn_close(f64(o[0]), ref, f"chunk {chunk} step {step}")
    assert pv.pv_kv_poll_device_error(h) == 0
    store.close()
