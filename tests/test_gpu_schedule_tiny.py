"""The tiny chunk schedule end to end on the GPU against the oracle session:
first chunk (3 frames, 4 steps), the sigma = 0 sink pass, then 5 one-frame
chunks with a ring of 2, two layers; every attention output, LSE and Euler
state is compared.  Head dims 64 (12/10/10 pairs) and 128 (22/21/21)."""
import numpy as np
import pytest
import torch

from gpu_common import assert_attn_close, assert_lse_close, f64, rel_l2
from oracle import euler
from oracle.schedule import Geometry
from oracle.session import SINK_STEP, StreamSession
from same_step_kv_b200 import synth

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def pv():
    from same_step_kv_b200 import pv as m
    return m


@pytest.mark.parametrize("D,R,n_chunks", [(64, 2, 5), (128, 2, 5), (64, 1, 3), (128, 3, 4)])
def test_tiny_schedule(pv, D, R, n_chunks):
    W, Hh, H, L = 8, 4, 2, 2
    T = W * Hh
    cfg = pv.make_config(L, H, D, W, Hh, ring_slots=R, max_streams=1, max_frames=64)
    store = pv.KVStore(cfg)
    h = store.handle
    ses = StreamSession(Geometry(W, Hh, H, D, ring_slots=R))
    lat_shape = (4, Hh, W)  # a 4-channel stand-in latent per frame
    worst = [0.0, 0.0]

    def one(chunk, step, layer, n):
        q, k, v = synth.chunk_qkv(0, chunk, step if step != pv.PV_STEP_SINK else 99, layer, n,
                                  H, D, "cuda")
        q_rot = torch.empty(H * n * D, dtype=torch.bfloat16, device="cuda")
        out = torch.empty(n, H, D, dtype=torch.bfloat16, device="cuda")
        lse = torch.empty(n, H, dtype=torch.float32, device="cuda")
        pv.pv_rope_append(h, [0], layer, step, q, k, v, q_rot)
        pv.pv_chunk_attn(h, [0], layer, step, q_rot, out, lse)
        torch.cuda.synchronize()
        ostep = SINK_STEP if step == pv.PV_STEP_SINK else step
        qr = ses.rope_append(layer, ostep, f64(q), f64(k), f64(v))
        o_ref, lse_ref = ses.chunk_attn(layer, ostep, qr)
        mx, rl = assert_attn_close(f64(out), o_ref, f"chunk {chunk} step {step} layer {layer}")
        assert_lse_close(f64(lse), lse_ref, f"chunk {chunk} step {step} layer {layer}")
        worst[0] = max(worst[0], mx)
        worst[1] = max(worst[1], rl)

    def denoise(chunk, nframes):
        x = synth.latent(0, nframes, *lat_shape, device="cuda").reshape(-1)
        x_ref = f64(x)
        for s in range(4):
            for layer in range(L):
                one(chunk, s, layer, nframes * T)
            vel = synth.velocity(0, chunk, s, x.numel(), "cuda")
            ds = euler.SIGMAS_4[s + 1] - euler.SIGMAS_4[s]
            pv.pv_euler_step(x, vel, x.numel(), float(ds))
            x_ref = euler.euler_step(x_ref, f64(vel), euler.SIGMAS_4[s], euler.SIGMAS_4[s + 1])
            torch.cuda.synchronize()
            assert rel_l2(f64(x), x_ref) <= 1e-5

    pv.pv_kv_begin_chunk(h, 0, 3)
    ses.begin_chunk(3)
    denoise(0, 3)
    pv.pv_kv_begin_sink(h, 0)
    for layer in range(L):
        one(0, pv.PV_STEP_SINK, layer, 3 * T)
    for j in range(1, n_chunks + 1):
        pv.pv_kv_begin_chunk(h, 0, 1)
        ses.begin_chunk(1)
        st = pv.pv_kv_get_state(h, 0)
        assert (st.slot, st.fill, st.n_keys) == (ses.ring.current_slot(), ses.ring.fill(),
                                                  ses.ring.n_keys())
        denoise(j, 1)
    print(f"D={D} R={R}: worst max-abs {worst[0]:.3g}, rel-L2 {worst[1]:.3g}")
    store.close()
