"""q, k, v projection with QK-Norm, RoPE and the append (pv_qkv_rope_append)
on the GPU against the fp64 oracle (oracle/projection.py, oracle/rope.py):
q_rot and the K rows within the bf16 RoPE bound, V rows within half a bf16
ulp plus the f32 accumulation, rows placed where the schedule puts them, for
the three GEMM tile widths (dim a multiple of 256, 128 and 64 only) and two
streams in one call; the one-launch path (every GEMM tile resident, the norm
and RoPE in the GEMM epilogue) for the small cases and the steady chunk, the
two-launch path for the profile's first chunk."""
import numpy as np
import pytest
import torch

from gpu_common import assert_rope_close, f64
from oracle import projection, rope
from same_step_kv_b200 import synth

pytestmark = pytest.mark.gpu
EPS = 1e-6


@pytest.fixture(scope="module")
def pv():
    from same_step_kv_b200 import pv as m
    return m


def _weights(heads, d, seed):
    dim = heads * d
    w = (synth.normal_f32(synth.seed_of(0x0A1, seed), (3 * dim, dim)) / dim ** 0.5).to(torch.bfloat16)
    b = 0.1 * synth.normal_f32(synth.seed_of(0x0A2, seed), (3 * dim,))
    g_q = 1.0 + 0.1 * synth.normal_f32(synth.seed_of(0x0A3, seed), (dim,))
    g_k = 1.0 + 0.1 * synth.normal_f32(synth.seed_of(0x0A4, seed), (dim,))
    return w.cuda(), b.cuda(), g_q.cuda(), g_k.cuda()


def _assert_v_close(got, ref, what):
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    tol = 2.0 ** -8 * np.abs(ref) + 1e-5 * np.sqrt(np.mean(ref * ref))
    bad = np.abs(got - ref) > tol
    assert not bad.any(), f"{what}: {int(bad.sum())} values outside the bound"


def _oracle(x, w, b, g_q, g_k, heads, W, Hh, frame0, D, rows=None):
    x64 = f64(x) if rows is None else f64(x)[rows]
    q, k, v = projection.qkv(x64, f64(w), f64(b), f64(g_q), f64(g_k), heads, EPS)
    n = x.shape[0]
    f, hh, ww = rope.token_coords(n, W, Hh, frame0)
    if rows is not None:
        f, hh, ww = f[rows], hh[rows], ww[rows]
    pairs = rope.axis_pairs(D)
    return rope.rotate(q, f, hh, ww, pairs=pairs), rope.rotate(k, f, hh, ww, pairs=pairs), v


@pytest.mark.parametrize("heads,d", [(2, 64), (2, 128), (3, 64)])
def test_first_chunk_tiny(pv, heads, d):
    # dim 128, 256 and 192: GEMM tiles of 128, 256 and 64 features
    W, Hh, R = 8, 4, 2
    T = W * Hh
    cfg = pv.make_config(2, heads, d, W, Hh, ring_slots=R, max_streams=2, max_frames=64)
    st = pv.KVStore(cfg)
    h = st.handle
    Kr, Vr = st.k_region(), st.v_region()
    n, layer, step, stream = 3 * T, 1, 2, 1
    pv.pv_kv_begin_chunk(h, stream, 3)
    dim = heads * d
    x = synth.normal_bf16(synth.seed_of(0x0B1, heads, d), (n, dim), "cuda")
    w, b, g_q, g_k = _weights(heads, d, heads * 1000 + d)
    q_rot = torch.empty(heads * n * d, dtype=torch.bfloat16, device="cuda")
    wsb = pv.pv_qkv_ws_bytes(n, dim)
    ws = torch.empty(wsb, dtype=torch.uint8, device="cuda")
    pv.pv_qkv_rope_append(h, [stream], layer, step, x, w, b, g_q, g_k, EPS, q_rot, ws, wsb)
    torch.cuda.synchronize()
    assert pv.pv_kv_poll_device_error(h) == 0
    qr, kr, v = _oracle(x, w, b, g_q, g_k, heads, W, Hh, 0, d)
    assert_rope_close(f64(q_rot.view(heads, n, d)), qr.transpose(1, 0, 2), "q_rot")
    assert_rope_close(f64(Kr[layer, step, stream, :, :n]), kr.transpose(1, 0, 2), "K rows")
    _assert_v_close(f64(Vr[layer, step, stream, :, :n]), v.transpose(1, 0, 2), "V rows")
    # nothing else of the store was written (it starts zeroed)
    assert int(torch.count_nonzero(Kr[layer, step, stream, :, n:])) == 0
    assert int(torch.count_nonzero(Kr[layer, step, 0])) == 0
    st.close()


@pytest.mark.parametrize("heads,d", [(2, 64), (3, 64), (1, 128), (4, 64)])
def test_one_launch_several_token_blocks(pv, heads, d):
    # 3 frames of 13 x 17 = 663 tokens: 3 token blocks of 256 (the last
    # ragged) x 3 dim / BN feature tiles (dim 128, 192, 128, 256: BN = 128,
    # 64, 128, 256 with 64-dim heads), all resident at once, so the norm's
    # wait spans several blocks
    W, Hh, R = 13, 17, 2
    T = W * Hh
    n = 3 * T
    cfg = pv.make_config(1, heads, d, W, Hh, ring_slots=R, max_frames=64)
    st = pv.KVStore(cfg)
    h = st.handle
    pv.pv_kv_begin_chunk(h, 0, 3)
    dim = heads * d
    x = synth.normal_bf16(synth.seed_of(0x0B6, heads, d), (n, dim), "cuda")
    w, b, g_q, g_k = _weights(heads, d, 23 + heads * d)
    q_rot = torch.empty(heads * n * d, dtype=torch.bfloat16, device="cuda")
    wsb = pv.pv_qkv_ws_bytes(n, dim)
    ws = torch.empty(wsb, dtype=torch.uint8, device="cuda")
    for rep in range(2):  # the second call's flags hold the next epoch
        q_rot.zero_()
        pv.pv_qkv_rope_append(h, [0], 0, 3, x, w, b, g_q, g_k, EPS, q_rot, ws, wsb)
        torch.cuda.synchronize()
        assert pv.pv_kv_poll_device_error(h) == 0
        qr, kr, v = _oracle(x, w, b, g_q, g_k, heads, W, Hh, 0, d)
        Kr, Vr = st.k_region(), st.v_region()
        assert_rope_close(f64(q_rot.view(heads, n, d)), qr.transpose(1, 0, 2), f"q_rot call {rep}")
        assert_rope_close(f64(Kr[0, 3, 0, :, :n]), kr.transpose(1, 0, 2), f"K rows call {rep}")
        _assert_v_close(f64(Vr[0, 3, 0, :, :n]), v.transpose(1, 0, 2), f"V rows call {rep}")
    st.close()


def test_one_launch_more_than_sixteen_feature_tiles(pv):
    # 17 heads x 64 = 1,088 features: 64-feature tiles, 17 of them per token
    # for q and for k, so a token's factor adds 17 partial sums (16 loaded
    # together, the 17th after); 96 tokens: 51 CTAs, one launch
    W, Hh, heads, d, R = 8, 4, 17, 64, 2
    T = W * Hh
    n = 3 * T
    cfg = pv.make_config(1, heads, d, W, Hh, ring_slots=R, max_frames=64)
    st = pv.KVStore(cfg)
    h = st.handle
    pv.pv_kv_begin_chunk(h, 0, 3)
    dim = heads * d
    x = synth.normal_bf16(synth.seed_of(0x0B7, 0), (n, dim), "cuda")
    w, b, g_q, g_k = _weights(heads, d, 29)
    q_rot = torch.empty(heads * n * d, dtype=torch.bfloat16, device="cuda")
    wsb = pv.pv_qkv_ws_bytes(n, dim)
    ws = torch.empty(wsb, dtype=torch.uint8, device="cuda")
    pv.pv_qkv_rope_append(h, [0], 0, 0, x, w, b, g_q, g_k, EPS, q_rot, ws, wsb)
    torch.cuda.synchronize()
    assert pv.pv_kv_poll_device_error(h) == 0
    qr, kr, v = _oracle(x, w, b, g_q, g_k, heads, W, Hh, 0, d)
    Kr, Vr = st.k_region(), st.v_region()
    assert_rope_close(f64(q_rot.view(heads, n, d)), qr.transpose(1, 0, 2), "q_rot")
    assert_rope_close(f64(Kr[0, 0, 0, :, :n]), kr.transpose(1, 0, 2), "K rows")
    _assert_v_close(f64(Vr[0, 0, 0, :, :n]), v.transpose(1, 0, 2), "V rows")
    st.close()


def test_steady_chunk_profile(pv):
    # the profile's steady chunk: 880 tokens of dim 3072 (24 x 128) into ring slot 9
    W, Hh, heads, d, R = 40, 22, 24, 128, 18
    T = W * Hh
    cfg = pv.make_config(1, heads, d, W, Hh, ring_slots=R, max_frames=64)
    st = pv.KVStore(cfg)
    h = st.handle
    s = pv.pv_kv_state()
    s.phase, s.chunk = pv.PV_PHASE_STEADY, 28
    pv.pv_kv_set_state(h, 0, s)
    s = pv.pv_kv_get_state(h, 0)
    dim = heads * d
    x = synth.normal_bf16(synth.seed_of(0x0B2, 0), (T, dim), "cuda")
    w, b, g_q, g_k = _weights(heads, d, 7)
    q_rot = torch.empty(heads * T * d, dtype=torch.bfloat16, device="cuda")
    wsb = pv.pv_qkv_ws_bytes(T, dim)
    ws = torch.empty(wsb, dtype=torch.uint8, device="cuda")
    pv.pv_qkv_rope_append(h, [0], 0, 2, x, w, b, g_q, g_k, EPS, q_rot, ws, wsb)
    torch.cuda.synchronize()
    assert pv.pv_kv_poll_device_error(h) == 0
    rows = np.array([0, 1, 127, 128, 255, 256, 500, 767, 768, 879])
    qr, kr, v = _oracle(x, w, b, g_q, g_k, heads, W, Hh, s.frame0, d, rows)
    r0 = 3 * T + s.slot * T
    Kr, Vr = st.k_region(), st.v_region()
    assert_rope_close(f64(q_rot.view(heads, T, d)[:, rows]), qr.transpose(1, 0, 2), "q_rot")
    assert_rope_close(f64(Kr[0, 2, 0, :, r0 + rows]), kr.transpose(1, 0, 2), "K rows")
    _assert_v_close(f64(Vr[0, 2, 0, :, r0 + rows]), v.transpose(1, 0, 2), "V rows")
    st.close()


def test_first_chunk_profile_two_launch_path(pv):
    # the profile's first chunk: 2,640 tokens of dim 3072 need 396 GEMM tiles,
    # more than can be resident at once, so the call takes the two-launch path
    # (GEMM writing y and the sums of squares, then the RoPE / append kernel)
    W, Hh, heads, d, R = 40, 22, 24, 128, 18
    T = W * Hh
    n = 3 * T
    cfg = pv.make_config(1, heads, d, W, Hh, ring_slots=R, max_frames=64)
    st = pv.KVStore(cfg)
    h = st.handle
    pv.pv_kv_begin_chunk(h, 0, 3)
    dim = heads * d
    x = synth.normal_bf16(synth.seed_of(0x0B4, 0), (n, dim), "cuda")
    w, b, g_q, g_k = _weights(heads, d, 13)
    q_rot = torch.empty(heads * n * d, dtype=torch.bfloat16, device="cuda")
    wsb = pv.pv_qkv_ws_bytes(n, dim)
    ws = torch.empty(wsb, dtype=torch.uint8, device="cuda")
    pv.pv_qkv_rope_append(h, [0], 0, 1, x, w, b, g_q, g_k, EPS, q_rot, ws, wsb)
    torch.cuda.synchronize()
    assert pv.pv_kv_poll_device_error(h) == 0
    rows = np.array([0, 127, 128, 879, 880, 1759, 1760, 2559, 2560, 2639])
    qr, kr, v = _oracle(x, w, b, g_q, g_k, heads, W, Hh, 0, d, rows)
    Kr, Vr = st.k_region(), st.v_region()
    assert_rope_close(f64(q_rot.view(heads, n, d)[:, rows]), qr.transpose(1, 0, 2), "q_rot")
    assert_rope_close(f64(Kr[0, 1, 0, :, rows]), kr.transpose(1, 0, 2), "K rows")
    _assert_v_close(f64(Vr[0, 1, 0, :, rows]), v.transpose(1, 0, 2), "V rows")
    st.close()


def test_fused_and_two_launch_calls_share_a_handle(pv):
    # one handle and one workspace: the steady chunk (one launch), then a
    # 2,640-token first chunk of another stream (two launches, atomics into
    # the sums after a memset), then the steady chunk again with other
    # inputs (one launch, the next flag epoch); the last call is checked
    W, Hh, heads, d, R = 40, 22, 24, 128, 18
    T = W * Hh
    cfg = pv.make_config(1, heads, d, W, Hh, ring_slots=R, max_streams=2, max_frames=64)
    st = pv.KVStore(cfg)
    h = st.handle
    s = pv.pv_kv_state()
    s.phase, s.chunk = pv.PV_PHASE_STEADY, 28
    pv.pv_kv_set_state(h, 0, s)
    s = pv.pv_kv_get_state(h, 0)
    pv.pv_kv_begin_chunk(h, 1, 3)
    dim = heads * d
    w, b, g_q, g_k = _weights(heads, d, 31)
    wsb = pv.pv_qkv_ws_bytes(3 * T, dim)
    ws = torch.empty(wsb, dtype=torch.uint8, device="cuda")
    q_rot = torch.empty(heads * 3 * T * d, dtype=torch.bfloat16, device="cuda")
    x0 = synth.normal_bf16(synth.seed_of(0x0B8, 0), (T, dim), "cuda")
    x1 = synth.normal_bf16(synth.seed_of(0x0B8, 1), (3 * T, dim), "cuda")
    x2 = synth.normal_bf16(synth.seed_of(0x0B8, 2), (T, dim), "cuda")
    pv.pv_qkv_rope_append(h, [0], 0, 2, x0, w, b, g_q, g_k, EPS, q_rot, ws, wsb)
    pv.pv_qkv_rope_append(h, [1], 0, 2, x1, w, b, g_q, g_k, EPS, q_rot, ws, wsb)
    pv.pv_qkv_rope_append(h, [0], 0, 2, x2, w, b, g_q, g_k, EPS, q_rot, ws, wsb)
    torch.cuda.synchronize()
    assert pv.pv_kv_poll_device_error(h) == 0
    rows = np.array([0, 1, 255, 256, 511, 700, 879])
    qr, kr, v = _oracle(x2, w, b, g_q, g_k, heads, W, Hh, s.frame0, d, rows)
    r0 = 3 * T + s.slot * T
    Kr, Vr = st.k_region(), st.v_region()
    assert_rope_close(f64(q_rot[:heads * T * d].view(heads, T, d)[:, rows]), qr.transpose(1, 0, 2),
                      "q_rot")
    assert_rope_close(f64(Kr[0, 2, 0, :, r0 + rows]), kr.transpose(1, 0, 2), "K rows")
    _assert_v_close(f64(Vr[0, 2, 0, :, r0 + rows]), v.transpose(1, 0, 2), "V rows")
    # and the first chunk's rows of stream 1 from the two-launch call
    rows1 = np.array([0, 879, 880, 1759, 2639])
    qr1, kr1, _ = _oracle(x1, w, b, g_q, g_k, heads, W, Hh, 0, d, rows1)
    assert_rope_close(f64(Kr[0, 2, 1, :, rows1]), kr1.transpose(1, 0, 2), "stream 1 K rows")
    st.close()


def test_two_streams_one_call(pv):
    # a stream in its first chunk (96 tokens) and one at a steady chunk (32)
    W, Hh, heads, d, R = 8, 4, 2, 128, 2
    T = W * Hh
    cfg = pv.make_config(1, heads, d, W, Hh, ring_slots=R, max_streams=2, max_frames=64)
    st = pv.KVStore(cfg)
    h = st.handle
    pv.pv_kv_begin_chunk(h, 0, 3)
    s = pv.pv_kv_state()
    s.phase, s.chunk = pv.PV_PHASE_STEADY, 5
    pv.pv_kv_set_state(h, 1, s)
    s = pv.pv_kv_get_state(h, 1)
    dim = heads * d
    n0, n1 = 3 * T, T
    x = synth.normal_bf16(synth.seed_of(0x0B3, 0), (n0 + n1, dim), "cuda")
    w, b, g_q, g_k = _weights(heads, d, 11)
    q_rot = torch.empty(heads * (n0 + n1) * d, dtype=torch.bfloat16, device="cuda")
    wsb = pv.pv_qkv_ws_bytes(n0 + n1, dim)
    ws = torch.empty(wsb, dtype=torch.uint8, device="cuda")
    pv.pv_qkv_rope_append(h, [0, 1], 0, 1, x, w, b, g_q, g_k, EPS, q_rot, ws, wsb)
    torch.cuda.synchronize()
    Kr, Vr = st.k_region(), st.v_region()
    # stream 0: tokens 0..95 at frames 0..2, sink rows of step 1
    qr, kr, v = _oracle(x[:n0], w, b, g_q, g_k, heads, W, Hh, 0, d)
    assert_rope_close(f64(q_rot[: heads * n0 * d].view(heads, n0, d)), qr.transpose(1, 0, 2), "q0")
    assert_rope_close(f64(Kr[0, 1, 0, :, :n0]), kr.transpose(1, 0, 2), "K0")
    # stream 1: tokens 96..127 at its chunk's frame, in its ring slot
    qr, kr, v = _oracle(x[n0:], w, b, g_q, g_k, heads, W, Hh, s.frame0, d)
    q1 = q_rot[heads * n0 * d:].view(heads, n1, d)
    assert_rope_close(f64(q1), qr.transpose(1, 0, 2), "q1")
    r0 = 3 * T + s.slot * T
    assert_rope_close(f64(Kr[0, 1, 1, :, r0:r0 + n1]), kr.transpose(1, 0, 2), "K1")
    _assert_v_close(f64(Vr[0, 1, 1, :, r0:r0 + n1]), v.transpose(1, 0, 2), "V1")
    st.close()


def test_sink_pass_two_streams_boundary_inside_a_warp(pv):
    # the bootstrap pass of two streams (K/V rows to the sink of all 4 step
    # buffers) with 60 tokens each: the stream boundary falls inside the
    # second group of 32 tokens, whose rows are written lane by lane, the
    # other groups by whole-box stores, each to every step buffer
    W, Hh, heads, d, R = 5, 4, 2, 128, 2
    T = W * Hh
    n = 3 * T
    cfg = pv.make_config(1, heads, d, W, Hh, ring_slots=R, max_streams=2, max_frames=64)
    st = pv.KVStore(cfg)
    h = st.handle
    for i in (0, 1):
        pv.pv_kv_begin_chunk(h, i, 3)
        pv.pv_kv_begin_sink(h, i)
    dim = heads * d
    x = synth.normal_bf16(synth.seed_of(0x0B5, 0), (2 * n, dim), "cuda")
    w, b, g_q, g_k = _weights(heads, d, 17)
    q_rot = torch.empty(heads * 2 * n * d, dtype=torch.bfloat16, device="cuda")
    wsb = pv.pv_qkv_ws_bytes(2 * n, dim)
    ws = torch.empty(wsb, dtype=torch.uint8, device="cuda")
    pv.pv_qkv_rope_append(h, [0, 1], 0, pv.PV_STEP_SINK, x, w, b, g_q, g_k, EPS, q_rot, ws, wsb)
    torch.cuda.synchronize()
    assert pv.pv_kv_poll_device_error(h) == 0
    Kr, Vr = st.k_region(), st.v_region()
    for i in (0, 1):
        qr, kr, v = _oracle(x[i * n:(i + 1) * n], w, b, g_q, g_k, heads, W, Hh, 0, d)
        qi = q_rot[heads * i * n * d:heads * (i + 1) * n * d].view(heads, n, d)
        assert_rope_close(f64(qi), qr.transpose(1, 0, 2), f"q_rot stream {i}")
        for s_ in range(4):
            assert_rope_close(f64(Kr[0, s_, i, :, :n]), kr.transpose(1, 0, 2), f"K stream {i} step {s_}")
            _assert_v_close(f64(Vr[0, s_, i, :, :n]), v.transpose(1, 0, 2), f"V stream {i} step {s_}")
            assert int(torch.count_nonzero(Kr[0, s_, i, :, n:])) == 0
    st.close()


def test_qkv_rejects_bad_arguments(pv):
    cfg = pv.make_config(1, 2, 64, 8, 4, ring_slots=2, max_frames=64)
    st = pv.KVStore(cfg)
    h = st.handle
    pv.pv_kv_begin_chunk(h, 0, 3)
    x = torch.zeros(96, 128, dtype=torch.bfloat16, device="cuda")
    w = torch.zeros(384, 128, dtype=torch.bfloat16, device="cuda")
    f = torch.zeros(384, device="cuda")
    q_rot = torch.empty(2 * 96 * 64, dtype=torch.bfloat16, device="cuda")
    wsb = pv.pv_qkv_ws_bytes(96, 128)
    ws = torch.empty(wsb, dtype=torch.uint8, device="cuda")
    with pytest.raises(pv.PVError) as e:
        pv.pv_qkv_rope_append(h, [0], 0, 0, x, w, f, f, f, 1e-6, q_rot, ws, wsb - 256)
    assert e.value.status == pv.PV_ERR_CAPACITY
    with pytest.raises(pv.PVError):
        pv.pv_qkv_rope_append(h, [0], 0, 0, x, w, f, f, f, 0.0, q_rot, ws, wsb)
    with pytest.raises(pv.PVError):
        pv.pv_qkv_rope_append(h, [0], 0, 0, x, 0, f, f, f, 1e-6, q_rot, ws, wsb)
    # the gains are read as 16-byte vectors: a 4-byte offset is rejected
    g_off = torch.zeros(385, device="cuda")[1:]
    with pytest.raises(pv.PVError) as e:
        pv.pv_qkv_rope_append(h, [0], 0, 0, x, w, f, g_off, f, 1e-6, q_rot, ws, wsb)
    assert e.value.status == pv.PV_ERR_INVALID_ARG
    st.close()
