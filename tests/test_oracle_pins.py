"""Pins the fp64 oracle to facts that do not come from the oracle itself:
values the pages print, closed forms, invariants, library routines and brute
force.  CPU only."""
import math

import numpy as np
import pytest
import torch

from golden_io import load
from oracle import attention, euler, rope, schedule
from oracle.schedule import Geometry, RingModel
from oracle.session import SINK_STEP, StreamSession
from same_step_kv_b200 import synth

# ---------------------------------------------------------------- schedule


def test_profile_geometry_from_printed_values():
    g = load("profile_geometry.txt")
    tok_w = g["resolution_width"] // g["compression_space"]
    tok_h = g["resolution_height"] // g["compression_space"]
    assert (tok_w, tok_h) == (40, 22)
    per_frame = tok_w * tok_h
    assert per_frame == 880
    geom = Geometry(tok_w, tok_h, 24, 128, first_frames=g["first_chunk_latent_frames"],
                    ring_slots=g["recent_chunks_in_history"])
    assert geom.sink_tokens == 2640
    # 29 chunks: one of 3 frames then 28 of 1 frame -> 31 latent frames -> 121 frames
    lat = schedule.latent_frames_of_schedule(g["chunks_per_generation"], g["first_chunk_latent_frames"])
    assert lat == 31
    frames = schedule.video_frames_of_latent(lat, g["compression_time"])
    assert frames == 121 and (frames - 1) % 4 == 0
    assert abs(frames / g["output_fps"] - 5.0) < 0.05       # "5 s" at 24 fps
    # the blog's own example of the 4n+1 rule: 81 frames <-> 21 latent frames
    assert schedule.video_frames_of_latent(g["blog_frames_81_latent"]) == 81
    assert g["blog_tokens_per_frame"] * g["blog_frames_81_latent"] == g["blog_total_tokens"]
    # steady state: sink + 18 slots (the ring includes the current chunk)
    ring = RingModel(geom)
    ring.begin_chunk(3)
    ring.bootstrap()
    for _ in range(g["chunks_per_generation"] - 1):
        ring.begin_chunk(1)
    assert ring.chunk == 28
    assert ring.n_keys() == 18480


@pytest.mark.parametrize("R", [1, 2, 3, 18, 19])
def test_ring_closed_forms(R):
    geom = Geometry(8, 4, 2, 64, ring_slots=R)
    ring = RingModel(geom)
    ring.begin_chunk(3)
    assert ring.n_keys() == geom.sink_tokens and ring.current_slot() == -1
    ring.bootstrap()
    for j in range(1, 41):
        ring.begin_chunk(1)
        assert ring.current_slot() == (j - 1) % R
        assert ring.fill() == min(j, R)
        assert ring.n_keys() == geom.sink_tokens + min(j, R) * geom.tokens_per_frame
        assert ring.slot_frames()[(j - 1) % R] == 2 + j
        # history = chunks max(1, j-R+1)..j, each once, no sink duplicate
        assert sorted(ring.chunks_in_history()) == list(range(max(1, j - R + 1), j + 1))


def test_phase_machine_rejects_misuse():
    geom = Geometry(8, 4, 2, 64, ring_slots=2)
    ring = RingModel(geom)
    with pytest.raises(ValueError):
        ring.begin_chunk(1)                 # first chunk has 3 frames
    ring.begin_chunk(3)
    with pytest.raises(ValueError):
        ring.begin_chunk(1)                 # sink bootstrap missing
    ring.bootstrap()
    with pytest.raises(ValueError):
        ring.begin_chunk(3)                 # later chunks have 1 frame
    ring.begin_chunk(1)
    with pytest.raises(ValueError):
        ring.bootstrap()


def test_flop_count_reproduces_printed_value():
    g = load("attention_flops.txt")
    f = schedule.attention_flops(g["seq_len"], g["seq_len"], g["heads"], g["head_dim"])
    digits = g["printed_digits"]
    mant = f / 10 ** math.floor(math.log10(f))
    printed = g["printed_flops"] / 10 ** math.floor(math.log10(g["printed_flops"]))
    assert round(mant, digits - 1) == printed
    assert math.floor(math.log10(f)) == math.floor(math.log10(g["printed_flops"]))


# -------------------------------------------------------------------- RoPE


def test_axis_split_matches_printed_44_42_42():
    assert rope.axis_dims(128) == (44, 42, 42)        # blog chapter 4, 3D RoPE
    assert rope.axis_pairs(128) == (22, 21, 21)
    assert rope.axis_pairs(64) == (12, 10, 10)
    for d in (64, 96, 128, 256):
        assert sum(rope.axis_dims(d)) == d


def test_rope_angle_zero_is_identity():
    x = synth.normal_f32(11, (40, 3, 128)).double().numpy()
    z = np.zeros(40, dtype=int)
    assert np.array_equal(rope.rotate(x, z, z, z), x)


def test_rope_preserves_pair_norms():
    x = synth.normal_f32(12, (64, 2, 128)).double().numpy()
    f, h, w = rope.token_coords(64, 8, 4, 5)
    y = rope.rotate(x, f, h, w)
    nx = x[..., 0::2] ** 2 + x[..., 1::2] ** 2
    ny = y[..., 0::2] ** 2 + y[..., 1::2] ** 2
    np.testing.assert_allclose(ny, nx, rtol=1e-13, atol=1e-13)


def test_rope_counter_clockwise_unit_turn():
    # pair 0 of each axis block turns by exactly the coordinate, in the positive
    # sense of the complex multiplication (x + iy) e^{i phi}
    d = 128
    pt, ph, _ = rope.axis_pairs(d)
    for pair, coord in ((0, (1, 0, 0)), (pt, (0, 1, 0)), (pt + ph, (0, 0, 1))):
        x = np.zeros((1, 1, d))
        x[0, 0, 2 * pair] = 1.0
        y = rope.rotate(x, [coord[0]], [coord[1]], [coord[2]])
        assert y[0, 0, 2 * pair] == pytest.approx(math.cos(1.0), abs=1e-15)
        assert y[0, 0, 2 * pair + 1] == pytest.approx(math.sin(1.0), abs=1e-15)


def test_rope_axis_blocks_move_independently():
    d = 128
    pt, ph, pw = rope.axis_pairs(d)
    a0 = rope.pair_angles([3], [4], [5], d)
    for axis, lo, hi in ((0, 0, pt), (1, pt, pt + ph), (2, pt + ph, pt + ph + pw)):
        c = [[3], [4], [5]]
        c[axis] = [c[axis][0] + 7]
        a1 = rope.pair_angles(*c, d)
        changed = np.nonzero(a1[0] != a0[0])[0]
        assert changed.min() == lo and changed.max() == hi - 1 and len(changed) == hi - lo


def test_rope_composition_and_frequency_decay():
    # rotating by a then by b equals rotating by a+b (a group action), and within an
    # axis block the frequencies fall strictly with the pair index
    x = synth.normal_f32(13, (10, 2, 128)).double().numpy()
    f1, h1, w1 = np.arange(10), np.arange(10) % 3, np.arange(10) % 5
    f2, h2, w2 = np.full(10, 2), np.full(10, 7), np.full(10, 1)
    y = rope.rotate(rope.rotate(x, f1, h1, w1), f2, h2, w2)
    z = rope.rotate(x, f1 + f2, h1 + h2, w1 + w2)
    np.testing.assert_allclose(y, z, atol=1e-12)
    ang = rope.pair_angles([1], [1], [1], 128)[0]
    for lo, hi in ((0, 22), (22, 43), (43, 64)):
        assert ang[lo] == 1.0 and np.all(np.diff(ang[lo:hi]) < 0)


def test_rope_relative_invariance_of_logits():
    # q.k after rotation depends only on the coordinate difference (blog chapter 4)
    q = synth.normal_f32(14, (32, 2, 128)).double().numpy()
    k = synth.normal_f32(15, (32, 2, 128)).double().numpy()
    fq, hq, wq = rope.token_coords(32, 8, 4, 3)
    fk, hk, wk = rope.token_coords(32, 8, 4, 0)
    base = np.einsum("qhd,khd->hqk", rope.rotate(q, fq, hq, wq), rope.rotate(k, fk, hk, wk))
    for s in ((5, 0, 0), (0, 9, 0), (0, 0, 11), (100, 20, 40)):
        qs = rope.rotate(q, fq + s[0], hq + s[1], wq + s[2])
        ks = rope.rotate(k, fk + s[0], hk + s[1], wk + s[2])
        np.testing.assert_allclose(np.einsum("qhd,khd->hqk", qs, ks), base, atol=1e-12)


# --------------------------------------------------------------- attention


def _tiny_session(R=2, n_chunks=5, layers=1, pairs=None, d=64, seed_stream=0):
    geom = Geometry(8, 4, 2, d, ring_slots=R)
    ses = StreamSession(geom, pairs)
    T = geom.tokens_per_frame
    rec = {}

    def qkv(chunk, step, layer, n):
        return [t.double().numpy() for t in synth.chunk_qkv(seed_stream, chunk, step, layer, n, 2, d)]

    ses.begin_chunk(3)
    for s in range(4):
        for l in range(layers):
            q, k, v = qkv(0, s, l, 3 * T)
            qr = ses.rope_append(l, s, q, k, v)
            rec[(0, s, l)] = (qr, ses.chunk_attn(l, s, qr))
    for l in range(layers):
        q, k, v = qkv(0, 99, l, 3 * T)
        qr = ses.rope_append(l, SINK_STEP, q, k, v)
        rec[(0, SINK_STEP, l)] = (qr, ses.chunk_attn(l, SINK_STEP, qr))
    for j in range(1, n_chunks + 1):
        ses.begin_chunk(1)
        for s in range(4):
            for l in range(layers):
                q, k, v = qkv(j, s, l, T)
                qr = ses.rope_append(l, s, q, k, v)
                rec[(j, s, l)] = (qr, ses.chunk_attn(l, s, qr))
    return ses, rec


def test_session_matches_brute_force_masked_world():
    """Assemble every step-s token of the run (sink + all chunks) into one matrix,
    mask by the history rule, and compare dense masked softmax with the session."""
    R, J, d = 2, 5, 64
    geom = Geometry(8, 4, 2, d, ring_slots=R)
    T = geom.tokens_per_frame
    ses, rec = _tiny_session(R, J, d=d)
    # rebuild the world independently from the generator and RoPE
    def rot(x, frame0, n):
        f, h, w = rope.token_coords(n, 8, 4, frame0)
        return rope.rotate(x, f, h, w)
    _, ks, vs = [t.double().numpy() for t in synth.chunk_qkv(0, 0, 99, 0, 3 * T, 2, d)]
    sink_k, sink_v = rot(ks, 0, 3 * T), vs
    for s in range(4):
        wk = [sink_k]
        wv = [sink_v]
        owner = [0] * (3 * T)
        for j in range(1, J + 1):
            _, kj, vj = [t.double().numpy() for t in synth.chunk_qkv(0, j, s, 0, T, 2, d)]
            wk.append(rot(kj, 2 + j, T))
            wv.append(vj)
            owner += [j] * T
        Kw = np.concatenate(wk)
        Vw = np.concatenate(wv)
        owner = np.array(owner)
        for j in range(1, J + 1):
            qr, (o, lse) = rec[(j, s, 0)]
            vis = (owner == 0) | ((owner > j - R) & (owner <= j))
            mask = np.broadcast_to(vis, (T, len(owner)))
            assert vis.sum() == 3 * T + min(j, R) * T
            for hh in range(2):
                ob, lb = attention.masked_dense(qr[:, hh], Kw[:, hh], Vw[:, hh], mask)
                np.testing.assert_allclose(o[:, hh], ob, atol=1e-12, rtol=0)
                np.testing.assert_allclose(lse[:, hh], lb, atol=1e-12, rtol=0)


def test_first_chunk_is_plain_self_attention_library():
    """With an empty history the chunk reduces to plain self-attention; checked against
    torch's fp64 scaled_dot_product_attention (a library routine)."""
    ses, rec = _tiny_session(R=2, n_chunks=0)
    geom = ses.geom
    for s in range(4):
        qr, (o, _) = rec[(0, s, 0)]
        K, V = ses.first[(0, s)]
        ref = torch.nn.functional.scaled_dot_product_attention(
            torch.from_numpy(qr).permute(1, 0, 2), torch.from_numpy(K).permute(1, 0, 2),
            torch.from_numpy(V).permute(1, 0, 2)).permute(1, 0, 2).numpy()
        np.testing.assert_allclose(o, ref, atol=1e-12)
        assert K.shape[0] == geom.sink_tokens


def test_softmax_rows_sum_to_one_and_single_key():
    q = synth.normal_f32(21, (17, 64)).double().numpy()
    k = synth.normal_f32(22, (50, 64)).double().numpy()
    P = attention.softmax_weights(q, k)
    np.testing.assert_allclose(P.sum(axis=1), 1.0, atol=1e-14)
    v = synth.normal_f32(23, (1, 64)).double().numpy()
    o, lse = attention.attend(q, k[:1], v)
    np.testing.assert_allclose(o, np.broadcast_to(v, o.shape), atol=1e-15)
    np.testing.assert_allclose(lse, (q @ k[0]) / 8.0, atol=1e-13)


def test_identical_keys_average_values():
    q = synth.normal_f32(24, (9, 64)).double().numpy()
    k = np.repeat(synth.normal_f32(25, (1, 64)).double().numpy(), 40, axis=0)
    v = synth.normal_f32(26, (40, 64)).double().numpy()
    o, lse = attention.attend(q, k, v)
    np.testing.assert_allclose(o, np.broadcast_to(v.mean(axis=0), o.shape), atol=1e-14)
    np.testing.assert_allclose(lse, q @ k[0] / 8.0 + np.log(40), atol=1e-13)


def test_sink_counted_once():
    ses, rec = _tiny_session(R=2, n_chunks=3)
    K, V = ses.key_set(0, 1)
    assert K.shape[0] == ses.geom.sink_tokens + 2 * ses.geom.tokens_per_frame
    qr, (o, _) = rec[(3, 1, 0)]
    sk, sv = ses.sink[0]
    K2, V2 = np.concatenate([sk, K]), np.concatenate([sv, V])
    o2, _ = attention.attend_heads(qr, K2, V2)
    assert np.abs(o2 - o).max() > 1e-3          # a duplicated sink changes the result


def test_key_order_permutation_invariance_at_angle_zero():
    # at RoPE angle 0 (all coordinates 0) permuting the raw token order of the keys
    # does not change the output
    d = 64
    q = synth.normal_f32(27, (32, 2, d)).double().numpy()
    k = synth.normal_f32(28, (96, 2, d)).double().numpy()
    v = synth.normal_f32(29, (96, 2, d)).double().numpy()
    z32, z96 = np.zeros(32, int), np.zeros(96, int)
    perm = np.random.default_rng(0).permutation(96)
    qr = rope.rotate(q, z32, z32, z32)
    o1, _ = attention.attend_heads(qr, rope.rotate(k, z96, z96, z96), v)
    o2, _ = attention.attend_heads(qr, rope.rotate(k[perm], z96, z96, z96), v[perm])
    np.testing.assert_allclose(o1, o2, atol=1e-13)


# ------------------------------------------------------------------- Euler


def test_euler_straight_line_lands_on_data():
    # x_sigma = (1-sigma) x0 + sigma x1 with v = x1 - x0 (blog chapter 1): four
    # Euler steps from pure noise reach x0, and x - sigma v = x0 at every stop
    x0 = synth.normal_f32(31, (4, 4, 8)).double().numpy()
    x1 = synth.normal_f32(32, (4, 4, 8)).double().numpy()
    v = x1 - x0
    x = x1.copy()
    sig = euler.SIGMAS_4
    for i in range(4):
        np.testing.assert_allclose(euler.x0_prediction(x, v, sig[i]), x0, atol=1e-14)
        x = euler.euler_step(x, v, sig[i], sig[i + 1])
        np.testing.assert_allclose(x, (1 - sig[i + 1]) * x0 + sig[i + 1] * x1, atol=1e-14)
    np.testing.assert_allclose(x, x0, atol=1e-14)


# --------------------------------------------------------- sampler variants


def test_shift_schedule_reproduces_printed_timesteps():
    g = load("shift_schedule.txt")
    sig = euler.shifted_schedule(g["steps"], g["shift"])
    t = euler.timesteps(sig[:-1])
    assert list(t[:6]) == [g[f"t{i}"] for i in range(6)]
    assert int((t >= g["high_noise_boundary"]).sum()) == g["steps_at_or_above_boundary"]
    assert int((t < g["high_noise_boundary"]).sum()) == g["steps_below_boundary"]
    # "half of the sampling points fall in the t > 926 interval"
    assert int((1000 * sig[:-1] > g["median_boundary"]).sum()) == g["steps"] // 2
    assert sig[-1] == 0.0 and np.all(np.diff(sig) < 0)


def test_shift_transform_properties():
    # identity at shift 1, fixed ends 0 and 1, and shift > 1 pushes every interior
    # point toward the noise end (chapter 5)
    s = np.linspace(0.0, 1.0, 101)
    np.testing.assert_allclose(euler.shift_sigma(s, 1.0), s, atol=0)
    for k in (3.0, 5.0, 12.0):
        y = euler.shift_sigma(s, k)
        assert y[0] == 0.0 and y[-1] == 1.0
        assert np.all(y[1:-1] > s[1:-1])
        # the inverse map is the same transform with 1/shift
        np.testing.assert_allclose(euler.shift_sigma(y, 1.0 / k), s, atol=1e-15)


def test_cfg_combine_special_cases():
    u = synth.normal_f32(41, (1000,)).double().numpy()
    c = synth.normal_f32(42, (1000,)).double().numpy()
    np.testing.assert_array_equal(euler.cfg_combine(u, c, 0.0), u)          # w = 0: unconditional
    np.testing.assert_allclose(euler.cfg_combine(u, c, 1.0), c, atol=1e-15)  # w = 1: conditional
    np.testing.assert_allclose(euler.cfg_combine(u, u, 7.5), u, atol=0)      # no difference
    # linear in w
    a, b = euler.cfg_combine(u, c, 2.0), euler.cfg_combine(u, c, 4.0)
    np.testing.assert_allclose(b - a, 2.0 * (c - u), atol=1e-13)


# --------------------------------------------------------- projection + QK-Norm
from oracle import projection  # noqa: E402


def test_linear_index_order():
    # identity weights return x; zero weights return the bias; one weight
    # w[i][j] moves input feature j to output feature i (not j to i transposed)
    rng = np.random.default_rng(7)
    x = rng.standard_normal((5, 6))
    np.testing.assert_array_equal(projection.linear(x, np.eye(6)), x)
    b = rng.standard_normal(4)
    np.testing.assert_array_equal(projection.linear(x, np.zeros((4, 6)), b), np.tile(b, (5, 1)))
    w = np.zeros((4, 6))
    w[1, 3] = 2.5
    y = projection.linear(x, w)
    np.testing.assert_array_equal(y[:, 1], 2.5 * x[:, 3])
    assert np.count_nonzero(y[:, [0, 2, 3]]) == 0


def test_rms_norm_closed_forms():
    rng = np.random.default_rng(8)
    y = rng.standard_normal((7, 48))
    g1 = np.ones(48)
    eps = projection.EPS
    out = projection.rms_norm(y, g1)
    ms = np.mean(y * y, axis=1)
    # mean of the squared output is ms / (ms + eps)
    np.testing.assert_allclose(np.mean(out * out, axis=1), ms / (ms + eps), rtol=1e-13)
    # a constant row a gives a / sqrt(a^2 + eps) times the gain
    g = rng.standard_normal(48)
    c = projection.rms_norm(np.full((1, 48), -3.0), g)
    np.testing.assert_allclose(c[0], -3.0 / math.sqrt(9.0 + eps) * g, rtol=1e-14)
    # without eps the norm is scale invariant (positive scales)
    np.testing.assert_allclose(projection.rms_norm(5.0 * y, g, 0.0), projection.rms_norm(y, g, 0.0),
                               rtol=1e-13)
    # the gain multiplies feature by feature, after the normalisation
    np.testing.assert_allclose(projection.rms_norm(y, g), out * g, rtol=1e-14)


def test_qkv_split_and_norm_only_on_q_and_k():
    rng = np.random.default_rng(9)
    heads, d = 2, 8
    dim = heads * d
    x = rng.standard_normal((3, dim))
    w = rng.standard_normal((3 * dim, dim))
    b = rng.standard_normal(3 * dim)
    g_q, g_k = rng.standard_normal(dim), rng.standard_normal(dim)
    q, k, v = projection.qkv(x, w, b, g_q, g_k, heads)
    assert q.shape == k.shape == v.shape == (3, heads, d)
    # v is the plain linear layer, feature f at head f // d, dimension f % d
    yv = x @ w[2 * dim:].T + b[2 * dim:]
    for f in range(dim):
        np.testing.assert_allclose(v[:, f // d, f % d], yv[:, f], rtol=1e-13)
    # q and k rows have unit RMS over all heads once the gain is divided out
    for t, gg in ((q, g_q), (k, g_k)):
        z = t.reshape(3, dim) / gg
        np.testing.assert_allclose(np.mean(z * z, axis=1), 1.0, rtol=1e-4)
    # scaling a token scales its v, leaves its q and k (nearly) unchanged
    q2, k2, v2 = projection.qkv(4.0 * x, w, 4.0 * b, g_q, g_k, heads)
    np.testing.assert_allclose(v2, 4.0 * v, rtol=1e-13)
    np.testing.assert_allclose(q2, q, rtol=1e-5)
