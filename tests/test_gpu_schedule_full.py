"""The whole generation schedule at the profile's sizes on the GPU: 880-token
frames (40 x 22), 24 heads x 128, a ring of 18, the 3-frame first chunk with
its 4 steps, the sigma = 0 sink pass, then 28 one-frame chunks of 4 steps
(the ring fills at chunk 18 and wraps after it).  Two layers run on the GPU;
the oracle session follows layer 1 for two of the heads through every call
(RoPE, append, ring) and checks sampled query rows at sampled calls, so the
bookkeeping of all 117 calls and the key sets up to 18,480 keys are
compared against the plain definition.  The checked calls cover every phase
and every edge of the ring's fill: the first chunk's first and last steps,
the sink pass, chunks 1 and 2 (one and two ring slots), 17 and 18 (the ring
filling), 19 and 20 (the first wraps) and 28 (the last chunk); the rows sit
at query-tile edges and in the one-tile last block of each frame."""
import numpy as np
import pytest
import torch

from gpu_common import assert_attn_close, assert_lse_close, f64
from oracle.schedule import Geometry
from oracle.session import SINK_STEP, StreamSession
from same_step_kv_b200 import synth

pytestmark = pytest.mark.gpu

W, HH, H, D, R, L = 40, 22, 24, 128, 18, 2
T = W * HH
LAYER = 1                      # the layer the oracle follows
HEADS = [0, 9, 17, 23]         # the heads the oracle follows
ROWS = [0, 39, 127, 128, 440, 767, 768, 879]   # query rows checked (of each 880-token frame)
CHECK = {(0, 0), (0, 3), (0, "sink"), (1, 0), (2, 1), (17, 2), (18, 1), (18, 3), (19, 3),
         (20, 0), (28, 2), (28, 3)}


@pytest.fixture(scope="module")
def pv():
    from same_step_kv_b200 import pv as m
    return m


def test_whole_schedule_profile_sizes(pv):
    cfg = pv.make_config(L, H, D, W, HH, ring_slots=R, max_streams=1, max_frames=64)
    store = pv.KVStore(cfg)
    h = store.handle
    ses = StreamSession(Geometry(W, HH, len(HEADS), D, ring_slots=R))
    q_rot = torch.empty(H * 3 * T * D, dtype=torch.bfloat16, device="cuda")
    out = torch.empty(3 * T, H, D, dtype=torch.bfloat16, device="cuda")
    lse = torch.empty(3 * T, H, dtype=torch.float32, device="cuda")
    checked = []

    def call(chunk, step, n):
        step_arg = pv.PV_STEP_SINK if step == "sink" else step
        seed_step = 99 if step == "sink" else step
        for layer in range(L):
            q, k, v = synth.chunk_qkv(0, chunk, seed_step, layer, n, H, D, "cuda")
            pv.pv_rope_append(h, [0], layer, step_arg, q, k, v, q_rot)
            pv.pv_chunk_attn(h, [0], layer, step_arg, q_rot, out[:n], lse[:n])
            if layer != LAYER:
                continue
            ostep = SINK_STEP if step == "sink" else step
            qr = ses.rope_append(LAYER, ostep, f64(q)[:, HEADS], f64(k)[:, HEADS],
                                 f64(v)[:, HEADS])
            if (chunk, step) not in CHECK:
                continue
            rows = [r + f * T for f in range(n // T) for r in ROWS]
            o_ref, lse_ref = ses.chunk_attn(LAYER, ostep, qr[rows])
            torch.cuda.synchronize()
            got = f64(out[:n])[rows][:, HEADS]
            what = f"chunk {chunk} step {step}"
            assert_attn_close(got, o_ref, what)
            assert_lse_close(f64(lse[:n])[rows][:, HEADS], lse_ref, what)
            checked.append((chunk, step, int(pv.pv_kv_get_state(h, 0).n_keys)))

    pv.pv_kv_begin_chunk(h, 0, 3)
    ses.begin_chunk(3)
    for s in range(4):
        call(0, s, 3 * T)
    pv.pv_kv_begin_sink(h, 0)
    call(0, "sink", 3 * T)
    for j in range(1, 29):
        pv.pv_kv_begin_chunk(h, 0, 1)
        ses.begin_chunk(1)
        st = pv.pv_kv_get_state(h, 0)
        assert (st.slot, st.fill, st.n_keys) == (ses.ring.current_slot(), ses.ring.fill(),
                                                  ses.ring.n_keys())
        for s in range(4):
            call(j, s, T)
    torch.cuda.synchronize()
    assert pv.pv_kv_poll_device_error(h) == 0
    assert len(checked) == len(CHECK)
    # the ring filled at chunk 18 and stayed full: 2,640 sink keys + 18 frames
    assert dict(((c, s), n) for c, s, n in checked)[(28, 2)] == 3 * T + R * T
    store.close()
