"""One pv_rope_append and one pv_chunk_attn call over streams in different
phases, at the profile's sizes (880-token frames, 24 heads x 128, ring 18):
stream 0 denoises its 3-frame first chunk (FIRST: 2,640 queries over its own
2,640 keys of the step), stream 1 is at the steady state (chunk 28: sink +
18 slots = 18,480 keys) and stream 2 early in its ring (chunk 5: sink + 5
slots = 7,040 keys).  Stream 0 is followed by an oracle session from its
first call; streams 1 and 2 start from pre-filled history, so their oracle
reads the store's earlier rows plus its own rotation of the new chunk.  The
appended K/V rows are checked too (sink rows of the step buffer for stream
0, the ring slot for the others)."""
import numpy as np
import pytest
import torch

from gpu_common import assert_attn_close, assert_lse_close, assert_rope_close, f64
from oracle import attention, rope
from oracle.schedule import Geometry
from oracle.session import StreamSession
from same_step_kv_b200 import synth

pytestmark = pytest.mark.gpu

W, HH, H, D, R = 40, 22, 24, 128, 18
T = W * HH
HEADS = [0, 13, 23]


@pytest.fixture(scope="module")
def pv():
    from same_step_kv_b200 import pv as m
    return m


def test_first_and_steady_streams_in_one_call(pv):
    layer, step = 0, 1
    chunks = [0, 28, 5]
    n = [3 * T, T, T]
    cfg = pv.make_config(1, H, D, W, HH, ring_slots=R, max_streams=3, max_frames=64)
    store = pv.KVStore(cfg)
    h = store.handle
    Kr, Vr = store.k_region(), store.v_region()
    pv.pv_kv_begin_chunk(h, 0, 3)                   # stream 0: FIRST, frames 0..2
    info = {}
    for i in (1, 2):
        st = pv.pv_kv_state()
        st.phase, st.chunk = pv.PV_PHASE_STEADY, chunks[i]
        pv.pv_kv_set_state(h, i, st)
        st = pv.pv_kv_get_state(h, i)
        kf, vf = synth.store_fill(i, layer, step, H, st.n_keys, D, "cuda")
        Kr[layer, step, i, :, :st.n_keys] = kf
        Vr[layer, step, i, :, :st.n_keys] = vf
        info[i] = (st.slot, st.n_keys, st.frame0)
    qkv = [synth.chunk_qkv(i, chunks[i], step, layer, n[i], H, D, "cuda") for i in range(3)]
    q, k, v = (torch.cat([t[j] for t in qkv]) for j in range(3))
    q_rot = torch.empty(H * sum(n) * D, dtype=torch.bfloat16, device="cuda")
    out = torch.empty(sum(n), H, D, dtype=torch.bfloat16, device="cuda")
    lse = torch.empty(sum(n), H, dtype=torch.float32, device="cuda")
    pv.pv_rope_append(h, [0, 1, 2], layer, step, q, k, v, q_rot)
    pv.pv_chunk_attn(h, [0, 1, 2], layer, step, q_rot, out, lse)
    torch.cuda.synchronize()
    assert pv.pv_kv_poll_device_error(h) == 0
    st0 = pv.pv_kv_get_state(h, 0)
    assert (st0.phase, st0.n_queries, st0.n_keys) == (pv.PV_PHASE_FIRST, 3 * T, 3 * T)

    # stream 0 against an oracle session that saw the same first call
    ses = StreamSession(Geometry(W, HH, len(HEADS), D, ring_slots=R))
    ses.begin_chunk(3)
    q0, k0, v0 = (f64(t)[:, HEADS] for t in qkv[0])
    qr0 = ses.rope_append(layer, step, q0, k0, v0)
    rows0 = np.array([0, 127, 128, 255, 256, 879, 880, 1759, 1760, 2559, 2560, 2639])
    o_ref, lse_ref = ses.chunk_attn(layer, step, qr0[rows0])
    assert_attn_close(f64(out[rows0])[:, HEADS], o_ref, "FIRST stream")
    assert_lse_close(f64(lse[rows0])[:, HEADS], lse_ref, "FIRST stream")
    k_sink, v_sink = ses.key_set(layer, step)
    for c, hd in enumerate(HEADS):
        assert_rope_close(f64(Kr[layer, step, 0, hd, :3 * T]), k_sink[:, c], f"FIRST k rows, head {hd}")
        assert torch.equal(Vr[layer, step, 0, hd, :3 * T], qkv[0][2][:, hd])
    # the q_rot block of stream 0 is head-major [H][2640][D]
    qr_gpu = q_rot[: H * 3 * T * D].view(H, 3 * T, D)
    for c, hd in enumerate(HEADS):
        assert_rope_close(f64(qr_gpu[hd]), qr0[:, c], f"FIRST q_rot, head {hd}")

    # streams 1 and 2: the store's history plus the oracle's rotation of the chunk
    rows = np.array([0, 127, 128, 255, 256, 767, 768, 879])
    tok0 = {1: 3 * T, 2: 4 * T}
    for i in (1, 2):
        slot, n_keys, frame0 = info[i]
        f, hh, ww = rope.token_coords(T, W, HH, frame0)
        k_cur = rope.rotate(f64(qkv[i][1]), f, hh, ww)
        qr = rope.rotate(f64(qkv[i][0])[rows], f[rows], hh[rows], ww[rows])
        r0 = 3 * T + slot * T
        for hd in HEADS:
            K = f64(Kr[layer, step, i, hd, :n_keys]).copy()
            V = f64(Vr[layer, step, i, hd, :n_keys]).copy()
            assert_rope_close(K[r0:r0 + T], k_cur[:, hd], f"stream {i} slot k rows, head {hd}")
            assert np.array_equal(V[r0:r0 + T], f64(qkv[i][2][:, hd]))
            K[r0:r0 + T] = k_cur[:, hd]
            o_ref, lse_ref = attention.attend(qr[:, hd], K, V)
            assert_attn_close(f64(out[tok0[i] + rows, hd]), o_ref, f"stream {i} head {hd}")
            assert_lse_close(f64(lse[tok0[i] + rows, hd]), lse_ref, f"stream {i} head {hd}")
    store.close()


def test_most_streams_one_call(pv):
    # the most streams a store holds (PV_MAX_STREAMS = 64), each in its first
    # chunk (3 frames of 8 x 4 tokens), in one pv_rope_append and one
    # pv_chunk_attn call; every row of both heads of every eighth stream
    # against the oracle's rotation and attention
    from same_step_kv_b200 import synth as sy
    Wt, Ht, Hs, Ds, S = 8, 4, 2, 64, 64
    Tt = Wt * Ht
    n = 3 * Tt
    cfg = pv.make_config(1, Hs, Ds, Wt, Ht, ring_slots=2, max_streams=S, max_frames=64)
    store = pv.KVStore(cfg)
    h = store.handle
    for i in range(S):
        pv.pv_kv_begin_chunk(h, i, 3)
    qkv = [sy.chunk_qkv(i, 0, 1, 0, n, Hs, Ds, "cuda") for i in range(S)]
    q, k, v = (torch.cat([t[j] for t in qkv]) for j in range(3))
    q_rot = torch.empty(Hs * S * n * Ds, dtype=torch.bfloat16, device="cuda")
    out = torch.empty(S * n, Hs, Ds, dtype=torch.bfloat16, device="cuda")
    lse = torch.empty(S * n, Hs, dtype=torch.float32, device="cuda")
    streams = list(range(S))
    pv.pv_rope_append(h, streams, 0, 1, q, k, v, q_rot)
    pv.pv_chunk_attn(h, streams, 0, 1, q_rot, out, lse)
    torch.cuda.synchronize()
    assert pv.pv_kv_poll_device_error(h) == 0
    f, hh, ww = rope.token_coords(n, Wt, Ht, 0)
    pairs = rope.axis_pairs(Ds)
    for i in range(0, S, 8):
        qr = rope.rotate(f64(qkv[i][0]), f, hh, ww, pairs=pairs)
        kr = rope.rotate(f64(qkv[i][1]), f, hh, ww, pairs=pairs)
        for hd in range(Hs):
            o_ref, lse_ref = attention.attend(qr[:, hd], kr[:, hd], f64(qkv[i][2][:, hd]))
            assert_attn_close(f64(out[i * n:(i + 1) * n, hd]), o_ref, f"stream {i} head {hd}")
            assert_lse_close(f64(lse[i * n:(i + 1) * n, hd]), lse_ref, f"stream {i} head {hd}")
    store.close()
