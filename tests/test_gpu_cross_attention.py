"""Cross-attention (video tokens query the prompt's text context) through
pv_attn_varlen and pv_attn_dense against the fp64 oracle: one prompt at the
profile's sizes, a batch of prompts with ragged text lengths in one launch,
the degenerate single-key context and a skipped sequence."""
import numpy as np
import pytest
import torch

from gpu_common import assert_attn_close, assert_lse_close, f64
from oracle import attention
from same_step_kv_b200 import synth

pytestmark = pytest.mark.gpu

H, D, T = 24, 128, 880      # heads, head dim, tokens of one latent frame (40 x 22)
MAX_TEXT = 512              # longest text context


@pytest.fixture(scope="module")
def pv():
    from same_step_kv_b200 import pv as m
    return m


def _packed(seed, lengths, heads, head_dim):
    """Head-major blocks [heads][n][head_dim] of each sequence, back to back."""
    parts = [synth.normal_bf16(synth.seed_of(seed, i), (heads, n, head_dim), "cuda")
             for i, n in enumerate(lengths)]
    flat = torch.cat([p.reshape(-1) for p in parts]) if parts else torch.empty(0)
    return flat, parts


def _run_varlen(pv, n_q, n_k, heads=H, head_dim=D):
    q, qs = _packed(0x51, n_q, heads, head_dim)
    k, ks = _packed(0x52, n_k, heads, head_dim)
    v, vs = _packed(0x53, n_k, heads, head_dim)
    tot = sum(n_q)
    out = torch.full((tot, heads, head_dim), float("nan"), dtype=torch.bfloat16, device="cuda")
    lse = torch.full((tot, heads), float("nan"), dtype=torch.float32, device="cuda")
    wsb = pv.pv_attn_varlen_ws_bytes(n_q, n_k, heads, head_dim)
    ws = torch.zeros(wsb, dtype=torch.uint8, device="cuda")
    pv.pv_attn_varlen(q, k, v, n_q, n_k, heads, head_dim, out, lse, ws, wsb)
    torch.cuda.synchronize()
    return qs, ks, vs, out, lse, ws


def _check(qs, ks, vs, out, lse, n_q, heads_to_check, rows=None):
    t0 = 0
    for i, nq in enumerate(n_q):
        if nq == 0:
            continue
        sel = np.arange(nq) if rows is None else rows[rows < nq]
        for h in heads_to_check:
            q = f64(qs[i][h])[sel]
            o_ref, lse_ref = attention.attend(q, f64(ks[i][h]), f64(vs[i][h]))
            assert_attn_close(f64(out[t0 + sel, h]), o_ref, f"seq {i} head {h}")
            assert_lse_close(f64(lse[t0 + sel, h]), lse_ref, f"seq {i} head {h}")
        t0 += nq


def test_one_prompt_full_text(pv):
    # one latent frame of queries against a 512-token context, every head
    n_q, n_k = [T], [MAX_TEXT]
    qs, ks, vs, out, lse, ws = _run_varlen(pv, n_q, n_k)
    _check(qs, ks, vs, out, lse, n_q, range(H))
    # the workspace is left zeroed for the next call (error word and counters)
    assert int(ws[:256].view(torch.int32)[0]) == 0


def test_prompt_batch_ragged_text(pv):
    # eight prompts in one launch: the first chunk's three frames, single
    # frames, a skipped sequence, a one-token context and the longest one
    n_k = synth.text_lengths(8)
    n_k[1], n_k[6] = 1, MAX_TEXT
    n_q = [3 * T, T, T, 0, T, T, T, T]
    qs, ks, vs, out, lse, _ = _run_varlen(pv, n_q, n_k)
    rows = np.unique(np.concatenate([np.arange(0, 3 * T, 97), [T - 1, 2 * T - 1, 3 * T - 1]]))
    _check(qs, ks, vs, out, lse, n_q, (0, 7, 13, 23), rows)
    # single key: the output is that key's value row
    t1 = n_q[0]
    got = out[t1:t1 + T].float()
    want = vs[1][:, 0, :].float().unsqueeze(0).expand(T, H, D)
    assert torch.equal(got, want)


@pytest.mark.parametrize("head_dim", [64, 128])
def test_most_sequences_one_launch(pv, head_dim):
    # the most sequences one launch takes (PV_MAX_STREAMS = 64), ragged:
    # queries 0..300 (some sequences skipped), keys 1..700; every row of
    # both heads against the oracle
    rng = np.random.default_rng(64 + head_dim)
    n_q = [int(x) for x in rng.integers(0, 301, size=64)]
    n_k = [int(x) for x in rng.integers(1, 701, size=64)]
    n_q[5], n_q[40] = 0, 0
    n_k[7] = 1
    qs, ks, vs, out, lse, _ = _run_varlen(pv, n_q, n_k, heads=2, head_dim=head_dim)
    _check(qs, ks, vs, out, lse, n_q, (0, 1))


def test_run_time_hand_out_is_repeatable(pv):
    # short items are handed out at run time from a counter in the workspace
    # (which CTA takes which item depends on timing); the last CTA returns the
    # counter to zero, so repeated launches on one workspace give the same
    # output bit for bit and leave the counters at zero
    n_k = synth.text_lengths(8, seed=3)
    n_q = [T] * 8
    assert pv.pv_attn_plan(n_q, n_k, H)[1] == 1
    qs, ks, vs, out, lse, ws = _run_varlen(pv, n_q, n_k)
    q = torch.cat([p.reshape(-1) for p in qs])
    k = torch.cat([p.reshape(-1) for p in ks])
    v = torch.cat([p.reshape(-1) for p in vs])
    out2 = torch.empty_like(out)
    for _ in range(3):
        pv.pv_attn_varlen(q, k, v, n_q, n_k, H, D, out2, None, ws, ws.numel())
        torch.cuda.synchronize()
        assert torch.equal(out, out2)
        assert int(torch.count_nonzero(ws[:256 + 8])) == 0  # error word, both counters


def test_run_time_one_tile_items_rescale(pv):
    # 64 sequences of 100 queries (one query tile per item) against 512 keys:
    # 1,536 items of 4 key tiles, handed out at run time.  In half the heads
    # keys of 5.0 and 10.0 in key tiles 1, 2 and 3 move the running maximum
    # far past the lazy-rescale threshold, so O is rescaled after the P V of
    # the previous key tile, with S of the next one already computed
    n, nq, nk, heads = 64, 100, 512, 8
    assert pv.pv_attn_plan([nq] * n, [nk] * n, heads)[1] == 1
    g = torch.Generator().manual_seed(11)
    q = (2.0 + 0.01 * torch.randn(n, heads, nq, D, generator=g)).to(torch.bfloat16)
    k = (0.3 * torch.randn(n, heads, nk, D, generator=g)).to(torch.bfloat16)
    v = torch.randn(n, heads, nk, D, generator=g).to(torch.bfloat16)
    for pos, val in ((128 + 3, 5.0), (2 * 128 + 100, 5.0), (3 * 128 + 9, 10.0)):
        k[:, : heads // 2, pos] = val
    q, k, v = q.cuda(), k.cuda(), v.cuda()
    out = torch.empty(n * nq, heads, D, dtype=torch.bfloat16, device="cuda")
    lse = torch.empty(n * nq, heads, dtype=torch.float32, device="cuda")
    wsb = pv.pv_attn_varlen_ws_bytes([nq] * n, [nk] * n, heads, D)
    ws = torch.zeros(wsb, dtype=torch.uint8, device="cuda")
    pv.pv_attn_varlen(q, k, v, [nq] * n, [nk] * n, heads, D, out, lse, ws, wsb)
    torch.cuda.synchronize()
    assert int(torch.count_nonzero(ws[:256 + 8])) == 0  # no wait gave up; counters reset
    for i in (0, 17, 63):
        for h in (0, 3, 4, 7):
            rows = slice(i * nq, (i + 1) * nq)
            o_ref, lse_ref = attention.attend(f64(q[i, h]), f64(k[i, h]), f64(v[i, h]))
            assert_attn_close(f64(out[rows, h]), o_ref, f"seq {i} head {h}")
            assert_lse_close(f64(lse[rows, h]), lse_ref, f"seq {i} head {h}")


def test_small_head_dim_and_tails(pv):
    # D = 64, query and key counts that leave ragged 128-row tiles
    n_q, n_k = [1, 129, 300], [7, 130, 385]
    qs, ks, vs, out, lse, _ = _run_varlen(pv, n_q, n_k, heads=3, head_dim=64)
    _check(qs, ks, vs, out, lse, n_q, range(3))


def test_dense_entry_on_cross_attention_shape(pv):
    # the single-sequence entry point on the same shape
    q = synth.normal_bf16(0x61, (H, T, D), "cuda")
    k = synth.normal_bf16(0x62, (H, 200, D), "cuda")
    v = synth.normal_bf16(0x63, (H, 200, D), "cuda")
    out = torch.empty(T, H, D, dtype=torch.bfloat16, device="cuda")
    wsb = pv.pv_attn_dense_ws_bytes(T, 200, H, D)
    ws = torch.zeros(wsb, dtype=torch.uint8, device="cuda")
    pv.pv_attn_dense(q, k, v, T, 200, H, D, out, None, ws, wsb)
    torch.cuda.synchronize()
    for h in (0, 11, 23):
        o_ref, _ = attention.attend(f64(q[h]), f64(k[h]), f64(v[h]))
        assert_attn_close(f64(out[:, h]), o_ref, f"head {h}")


def test_varlen_rejects_bad_arguments(pv):
    x = torch.zeros(4096, dtype=torch.bfloat16, device="cuda")
    ws = torch.zeros(1 << 20, dtype=torch.uint8, device="cuda")
    for n_q, n_k in (([5], [0]), ([-1], [3]), ([1] * 65, [1] * 65)):
        with pytest.raises(pv.PVError) as e:
            pv.pv_attn_varlen(x, x, x, n_q, n_k, 2, 64, x, None, ws, ws.numel())
        assert e.value.status == pv.PV_ERR_SHAPE
    with pytest.raises(pv.PVError) as e:
        pv.pv_attn_varlen(x, x, x, [4], [4], 2, 64, x, None, ws, 64)
    assert e.value.status == pv.PV_ERR_CAPACITY
    # no queries at all: nothing to do
    pv.pv_attn_varlen(x, x, x, [0, 0], [3, 0], 2, 64, x, None, ws, ws.numel())


@pytest.mark.parametrize("head_dim", [128, 64])
def test_ragged_one_tile_blocks_stream_k_every_row(pv, head_dim):
    # ragged sequences whose last query block holds a single tile (112, 100,
    # 44 and 1 rows over a multiple of 256) beside ones whose blocks all hold
    # two (1024, 129 queries), cut stream-K into split parts that the last CTA
    # to arrive merges; every row of every head
    n_q = [880, 100, 1024, 300, 129, 1]
    n_k = [3000, 2500, 1200, 4100, 700, 3333]
    heads = 3
    assert pv.pv_attn_plan(n_q, n_k, heads)[1] == 0   # stream-K
    qs, ks, vs, out, lse, ws = _run_varlen(pv, n_q, n_k, heads, head_dim)
    _check(qs, ks, vs, out, lse, n_q, range(heads))
    assert int(ws[:256].view(torch.int32)[0]) == 0
    # the arrival counters are back at zero: a second launch is bit-identical
    out2 = torch.empty_like(out)
    pv.pv_attn_varlen(torch.cat([t.reshape(-1) for t in qs]), torch.cat([t.reshape(-1) for t in ks]),
                      torch.cat([t.reshape(-1) for t in vs]), n_q, n_k, heads, head_dim, out2, None,
                      ws, ws.numel())
    torch.cuda.synchronize()
    assert torch.equal(out, out2)
