"""3D RoPE + same-step append on the GPU against the oracle: rotated values
within the bf16 bound, K/V rows placed exactly where the schedule puts them
(V copied bit for bit), and no other row of the store touched."""
import numpy as np
import pytest
import torch

from gpu_common import assert_rope_close, f64
from oracle import rope
from same_step_kv_b200 import synth

pytestmark = pytest.mark.gpu

GEOMS = {
    "tiny_d64": dict(W=8, Hh=4, H=2, D=64, R=2),
    "tiny_d128": dict(W=8, Hh=4, H=2, D=128, R=2),
    "profile_40x22_24x128": dict(W=40, Hh=22, H=24, D=128, R=18),
}


@pytest.fixture(scope="module")
def pv():
    from same_step_kv_b200 import pv as m
    return m


def pairs_of(D):
    return rope.axis_pairs(D)


@pytest.mark.parametrize("name", list(GEOMS))
def test_rope_append_places_rows(pv, name):
    g = GEOMS[name]
    W, Hh, H, D, R = g["W"], g["Hh"], g["H"], g["D"], g["R"]
    T = W * Hh
    L, S = 2, 2
    cfg = pv.make_config(L, H, D, W, Hh, ring_slots=R, max_streams=S, max_frames=64)
    st = pv.KVStore(cfg)
    h = st.handle
    Kr, Vr = st.k_region(), st.v_region()
    expect_written = torch.zeros(Kr.shape[:5], dtype=torch.bool, device="cuda")
    stream, layer = 1, 1

    def check(chunk, step, frame0, n, rows_by_step):
        q, k, v = synth.chunk_qkv(stream, chunk, step if step >= 0 else 99, layer, n, H, D, "cuda")
        q_rot = torch.empty(H * n * D, dtype=torch.bfloat16, device="cuda")
        pv.pv_rope_append(h, [stream], layer, step, q, k, v, q_rot)
        torch.cuda.synchronize()
        f, hh, ww = rope.token_coords(n, W, Hh, frame0)
        qr = rope.rotate(f64(q), f, hh, ww, pairs=pairs_of(D))
        kr = rope.rotate(f64(k), f, hh, ww, pairs=pairs_of(D))
        assert_rope_close(f64(q_rot.view(H, n, D)), qr.transpose(1, 0, 2), f"{name} q_rot")
        for s_, r0 in rows_by_step:
            got_k = Kr[layer, s_, stream, :, r0:r0 + n]
            got_v = Vr[layer, s_, stream, :, r0:r0 + n]
            assert_rope_close(f64(got_k), kr.transpose(1, 0, 2), f"{name} K step {s_}")
            assert torch.equal(got_v, v.permute(1, 0, 2)), f"{name} V step {s_} not bit-exact"
            expect_written[layer, s_, stream, :, r0:r0 + n] = True

    pv.pv_kv_begin_chunk(h, stream, 3)
    for s_ in range(4):
        check(0, s_, 0, 3 * T, [(s_, 0)])
    pv.pv_kv_begin_sink(h, stream)
    check(0, pv.PV_STEP_SINK, 0, 3 * T, [(s_, 0) for s_ in range(4)])
    for j in range(1, R + 3):
        pv.pv_kv_begin_chunk(h, stream, 1)
        slot = (j - 1) % R
        for s_ in (0, 3):
            check(j, s_, 2 + j, T, [(s_, 3 * T + slot * T)])
    # nothing outside the written rows changed (the store starts zeroed)
    untouched = ~expect_written
    assert int(torch.count_nonzero(Kr[untouched])) == 0
    assert int(torch.count_nonzero(Vr[untouched])) == 0
    st.close()


def test_rope_dense_matches_oracle(pv):
    W, Hh, H, D = 8, 4, 3, 128
    T = W * Hh
    cfg = pv.make_config(1, H, D, W, Hh, ring_slots=2, max_frames=64)
    st = pv.KVStore(cfg)
    n, frame0 = 5 * T, 7
    q, k, v = synth.chunk_qkv(9, 9, 9, 9, n, H, D, "cuda")
    q_rot = torch.empty(H, n, D, dtype=torch.bfloat16, device="cuda")
    k_rot = torch.empty_like(q_rot)
    v_hm = torch.empty_like(q_rot)
    pv.pv_rope_dense(st.handle, n, frame0, q, k, v, q_rot, k_rot, v_hm)
    torch.cuda.synchronize()
    f, hh, ww = rope.token_coords(n, W, Hh, frame0)
    assert_rope_close(f64(q_rot), rope.rotate(f64(q), f, hh, ww).transpose(1, 0, 2), "dense q")
    assert_rope_close(f64(k_rot), rope.rotate(f64(k), f, hh, ww).transpose(1, 0, 2), "dense k")
    assert torch.equal(v_hm, v.permute(1, 0, 2))
    with pytest.raises(pv.PVError):
        pv.pv_rope_dense(st.handle, n + 1, 0, q, k, v, q_rot, k_rot, v_hm)
    with pytest.raises(pv.PVError):
        pv.pv_rope_dense(st.handle, n, 62, q, k, v, q_rot, k_rot, v_hm)  # past max_frames
    st.close()


def test_generator_is_device_independent():
    a = synth.normal_bf16(1234, (3, 1000, 7), "cuda").cpu()
    b = synth.normal_bf16(1234, (3, 1000, 7), "cpu")
    assert torch.equal(a, b)
