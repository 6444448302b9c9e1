"""Chunk attention on the GPU against the fp64 oracle at the profile's sizes
(sampled rows, all keys) and on small dense shapes (every row), including
ragged tails, single keys and the split-KV merge."""
import numpy as np
import pytest
import torch

from gpu_common import assert_attn_close, assert_lse_close, f64
from oracle import attention, rope
from same_step_kv_b200 import synth

pytestmark = pytest.mark.gpu

W, HH, H, D, R = 40, 22, 24, 128, 18
T = W * HH


@pytest.fixture(scope="module")
def pv():
    from same_step_kv_b200 import pv as m
    return m


def _steady_run(pv, chunks, layer=0, step=2, lse_too=True):
    """Streams at the given chunk indices (>= 1) of a steady schedule; earlier
    history comes from the generator.  Returns what the oracle needs."""
    S = len(chunks)
    cfg = pv.make_config(1, H, D, W, HH, ring_slots=R, max_streams=S, max_frames=64)
    store = pv.KVStore(cfg)
    h = store.handle
    Kr, Vr = store.k_region(), store.v_region()
    qs, ks, vs, info = [], [], [], []
    for i, j in enumerate(chunks):
        st = pv.pv_kv_state()
        st.phase, st.chunk = pv.PV_PHASE_STEADY, j
        pv.pv_kv_set_state(h, i, st)
        st = pv.pv_kv_get_state(h, i)
        n_keys = st.n_keys
        kf, vf = synth.store_fill(i, layer, step, H, n_keys, D, "cuda")
        Kr[layer, step, i, :, :n_keys] = kf
        Vr[layer, step, i, :, :n_keys] = vf
        q, k, v = synth.chunk_qkv(i, j, step, layer, T, H, D, "cuda")
        qs.append(q), ks.append(k), vs.append(v)
        info.append((j, st.slot, n_keys, st.frame0))
    q, k, v = torch.cat(qs), torch.cat(ks), torch.cat(vs)
    q_rot = torch.empty(H * S * T * D, dtype=torch.bfloat16, device="cuda")
    out = torch.empty(S * T, H, D, dtype=torch.bfloat16, device="cuda")
    lse = torch.empty(S * T, H, dtype=torch.float32, device="cuda") if lse_too else None
    pv.pv_rope_append(h, list(range(S)), layer, step, q, k, v, q_rot)
    pv.pv_chunk_attn(h, list(range(S)), layer, step, q_rot, out, lse)
    torch.cuda.synchronize()
    return store, Kr, Vr, qs, ks, vs, info, out, lse


def _check_sampled(pv, chunks, rows, heads, layer=0, step=2):
    store, Kr, Vr, qs, ks, vs, info, out, lse = _steady_run(pv, chunks, layer, step)
    for i, (j, slot, n_keys, frame0) in enumerate(info):
        f, hh, ww = rope.token_coords(T, W, HH, frame0)
        q_all = f64(qs[i])
        k_cur = rope.rotate(f64(ks[i]), f, hh, ww)
        for hd in heads:
            K = f64(Kr[layer, step, i, hd, :n_keys]).copy()
            V = f64(Vr[layer, step, i, hd, :n_keys]).copy()
            # the current chunk's slot: the oracle's own rotation of k, the input v
            r0 = 3 * T + slot * T
            K[r0:r0 + T] = k_cur[:, hd]
            V[r0:r0 + T] = f64(vs[i][:, hd])
            qr = rope.rotate(q_all[rows], f[rows], hh[rows], ww[rows])[:, hd]
            o_ref, lse_ref = attention.attend(qr, K, V)
            tok = np.array(rows) + i * T
            assert_attn_close(f64(out[tok, hd]), o_ref, f"stream {i} head {hd}")
            assert_lse_close(f64(lse[tok, hd]), lse_ref, f"stream {i} head {hd}")
    store.close()


ROWS = [0, 1, 63, 127, 128, 255, 256, 400, 511, 512, 767, 768, 800, 879]


def test_steady_chunk_880x18480(pv):
    """One 880-token chunk at chunk 28: sink + 18 slots = 18,480 keys."""
    _check_sampled(pv, [28], ROWS, [0, 7, 23])


@pytest.mark.parametrize("j", [1, 2, 17, 18, 19])
def test_steady_chunk_ring_fill_edges(pv, j):
    _check_sampled(pv, [j], [0, 127, 128, 879], [5])


def test_multistream_ragged_fills(pv):
    """8 streams, each with 0..18 earlier chunks (seeded), one launch."""
    fills = synth.ragged_fills(8, R)
    _check_sampled(pv, [1 + f for f in fills], [0, 129, 500, 879], [0, 11, 23])


def _dense_case(pv, n_q, n_k, heads, dim, rows=None, seed=0):
    q = synth.normal_bf16(synth.seed_of(31, seed, n_q), (heads, n_q, dim), "cuda")
    k = synth.normal_bf16(synth.seed_of(32, seed, n_k), (heads, n_k, dim), "cuda")
    v = synth.normal_bf16(synth.seed_of(33, seed, n_k), (heads, n_k, dim), "cuda")
    out = torch.empty(n_q, heads, dim, dtype=torch.bfloat16, device="cuda")
    lse = torch.empty(n_q, heads, dtype=torch.float32, device="cuda")
    wsb = pv.pv_attn_dense_ws_bytes(n_q, n_k, heads, dim)
    ws = torch.zeros(wsb, dtype=torch.uint8, device="cuda")
    pv.pv_attn_dense(q, k, v, n_q, n_k, heads, dim, out, lse, ws, wsb)
    torch.cuda.synchronize()
    rows = np.arange(n_q) if rows is None else np.asarray(rows)
    for hd in range(heads):
        o_ref, lse_ref = attention.attend(f64(q[hd])[rows], f64(k[hd]), f64(v[hd]))
        assert_attn_close(f64(out[rows, hd]), o_ref, f"dense {n_q}x{n_k} h{hd}")
        assert_lse_close(f64(lse[rows, hd]), lse_ref, f"dense {n_q}x{n_k} h{hd}")
    return q, k, v, out, ws


@pytest.mark.parametrize("n_q,n_k,heads,dim", [
    (1, 1, 1, 64), (1, 200, 2, 128), (129, 1, 2, 128), (96, 96, 2, 64), (256, 256, 1, 128),
    (257, 385, 3, 128), (300, 1000, 2, 64), (880, 3520, 2, 128), (128, 8192, 2, 128),
    (5, 20000, 1, 64)])
def test_dense_small_shapes_every_row(pv, n_q, n_k, heads, dim):
    _dense_case(pv, n_q, n_k, heads, dim)


def test_dense_split_merge_is_repeatable(pv):
    """Split-KV units merge through arrival counters that reset themselves:
    two launches on the same workspace give identical results."""
    q, k, v, out, ws = _dense_case(pv, 200, 9000, 2, 128)
    out2 = torch.empty_like(out)
    pv.pv_attn_dense(q, k, v, 200, 9000, 2, 128, out2, None, ws, ws.numel())
    torch.cuda.synchronize()
    assert torch.equal(out, out2)
    assert int(torch.count_nonzero(ws[256:256 + 4 * 2 * 2])) == 0  # counters back to zero


def test_dense_video_18480(pv):
    """Full bidirectional attention over 21 latent frames (18,480 tokens), 24 x 128,
    3D RoPE at frames 0..20; sampled rows of three heads."""
    n = 21 * T
    cfg = pv.make_config(1, H, D, W, HH, ring_slots=R, max_frames=64)
    store = pv.KVStore(cfg)
    q, k, v = synth.chunk_qkv(0, 0, 0, 0, n, H, D, "cuda")
    q_rot = torch.empty(H, n, D, dtype=torch.bfloat16, device="cuda")
    k_rot, v_hm = torch.empty_like(q_rot), torch.empty_like(q_rot)
    pv.pv_rope_dense(store.handle, n, 0, q, k, v, q_rot, k_rot, v_hm)
    out = torch.empty(n, H, D, dtype=torch.bfloat16, device="cuda")
    wsb = pv.pv_attn_dense_ws_bytes(n, n, H, D)
    ws = torch.zeros(wsb, dtype=torch.uint8, device="cuda")
    pv.pv_attn_dense(q_rot, k_rot, v_hm, n, n, H, D, out, None, ws, wsb)
    torch.cuda.synchronize()
    f, hh, ww = rope.token_coords(n, W, HH, 0)
    rows = np.array([0, 1, 879, 880, 9000, 18000, 18479])
    for hd in (0, 12, 23):
        qr = rope.rotate(f64(q[rows]), f[rows], hh[rows], ww[rows])[:, hd]
        kr = rope.rotate(f64(k[:, hd:hd + 1]), f, hh, ww)[:, 0]
        o_ref, _ = attention.attend(qr, kr, f64(v[:, hd]))
        assert_attn_close(f64(out[rows, hd]), o_ref, f"dense video head {hd}")
    store.close()


@pytest.mark.parametrize("n_q", [256, 100, 300])
def test_dense_score_spikes_force_rescale(pv, n_q):
    """A later key tile whose scores exceed the running maximum by far more
    than the lazy-rescale threshold (log2 units): the running maximum moves
    and O and l are rescaled inside a segment.  Half the heads get such
    spikes: keys of 5.0 against queries near 2.0 lift the score by ~112 over
    the first tile's maximum, ~161 in log2 units, and a key of 10.0 further
    on lifts it by as much again.  Without the rescale those exponentials
    overflow to inf.  The spikes sit in odd and even key tiles that are not
    the first of their segment (24 heads x 32 key tiles over 148 SMs:
    stream-K segments of ~5 tiles).  256 queries: two query tiles per
    segment; 100: one (S of the next key tile computed ahead, in the other S
    buffer, and O rescaled after the previous P V has completed); 300: both
    kinds in one launch (a 44-row last query block)."""
    n_k, heads, dim = 4096, 24, 128
    g = torch.Generator().manual_seed(5)
    q = (2.0 + 0.01 * torch.randn(heads, n_q, dim, generator=g)).to(torch.bfloat16)
    k = (0.3 * torch.randn(heads, n_k, dim, generator=g)).to(torch.bfloat16)
    v = torch.randn(heads, n_k, dim, generator=g).to(torch.bfloat16)
    q[heads // 2:] = torch.randn(heads - heads // 2, n_q, dim, generator=g).to(torch.bfloat16)
    for pos in (1 * 128 + 3, 3 * 128 + 5, 9 * 128 + 77, 17 * 128, 22 * 128 + 64, 25 * 128 + 127,
                30 * 128 + 40):
        k[: heads // 2, pos] = 5.0
    k[: heads // 2, 31 * 128 + 9] = 10.0
    q, k, v = q.cuda(), k.cuda(), v.cuda()
    out = torch.empty(n_q, heads, dim, dtype=torch.bfloat16, device="cuda")
    lse = torch.empty(n_q, heads, dtype=torch.float32, device="cuda")
    wsb = pv.pv_attn_dense_ws_bytes(n_q, n_k, heads, dim)
    ws = torch.zeros(wsb, dtype=torch.uint8, device="cuda")
    pv.pv_attn_dense(q, k, v, n_q, n_k, heads, dim, out, lse, ws, wsb)
    torch.cuda.synchronize()
    assert int(ws[:4].view(torch.int32)[0]) == 0   # no wait gave up
    for hd in (0, 5, 11, 12, 23):
        o_ref, lse_ref = attention.attend(f64(q[hd]), f64(k[hd]), f64(v[hd]))
        assert_attn_close(f64(out[:, hd]), o_ref, f"spiky head {hd}")
        assert_lse_close(f64(lse[:, hd]), lse_ref, f"spiky head {hd}")
    # with spikes the output is (nearly) the value row of the largest one
    assert torch.allclose(out[:, 0].float(), v[0, 31 * 128 + 9].float().expand(n_q, dim), atol=2e-2)
