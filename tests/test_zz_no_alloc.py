"""pv_attn_dense_noalloc: the dense attention entry point for callers that
cannot allocate device memory where they call it (allocator callbacks,
plugins whose host owns every allocation, paths that must not touch the
allocator).  It keeps its split-KV scratch in a fixed array inside the
library; this test checks, through the C ABI, that two calls in a row give
the same result as pv_attn_dense with a caller workspace, within the
attention tolerance the other tests use, that both match the fp64 oracle on
sampled rows, that a timed-out device wait is reported through the scratch's
error word, and that an oversized problem is refused on the host.  The file
sorts last so that it runs after every other test, and it also passes on its
own in a fresh process."""
import numpy as np
import pytest
import torch

from gpu_common import assert_attn_close, assert_lse_close, f64
from oracle import attention
from same_step_kv_b200 import synth

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def pv():
    from same_step_kv_b200 import pv as m
    return m


# Split-KV partial slots of the fixed scratch at head_dim 128: the 8 MiB array
# minus the error block and 16,384 counters, over 128 x 128 + 256 floats a slot.
SCRATCH_SLOTS_D128 = ((8 << 20) - 256 - 16384 * 4) // ((128 * 128 + 256) * 4)


@pytest.mark.parametrize("n_q,n_k,heads,dim", [
    (200, 9000, 2, 128),      # 142 key tiles: whole items handed out at run time
    (256, 3000, 1, 128),      # 24 key tiles: stream-K, the merge runs through the scratch
    (257, 385, 3, 64),        # stream-K with a split merge at head_dim 64
    (1, 1, 1, 64),
    (880, 18480, 24, 128),    # the profile's steady chunk as a dense call
])
def test_noalloc_matches_workspace_entry_point(pv, n_q, n_k, heads, dim):
    q = synth.normal_bf16(synth.seed_of(41, n_q, n_k), (heads, n_q, dim), "cuda")
    k = synth.normal_bf16(synth.seed_of(42, n_q, n_k), (heads, n_k, dim), "cuda")
    v = synth.normal_bf16(synth.seed_of(43, n_q, n_k), (heads, n_k, dim), "cuda")
    ref = torch.empty(n_q, heads, dim, dtype=torch.bfloat16, device="cuda")
    ref_lse = torch.empty(n_q, heads, dtype=torch.float32, device="cuda")
    wsb = pv.pv_attn_dense_ws_bytes(n_q, n_k, heads, dim)
    ws = torch.zeros(wsb, dtype=torch.uint8, device="cuda")
    pv.pv_attn_dense(q, k, v, n_q, n_k, heads, dim, ref, ref_lse, ws, wsb)
    outs = []
    for _ in range(2):
        out = torch.full((n_q, heads, dim), float("nan"), dtype=torch.bfloat16, device="cuda")
        lse = torch.full((n_q, heads), float("nan"), dtype=torch.float32, device="cuda")
        pv.pv_attn_dense_noalloc(q, k, v, n_q, n_k, heads, dim, out, lse)
        torch.cuda.synchronize()
        assert_attn_close(f64(out), f64(ref), f"noalloc {n_q}x{n_k}")
        assert_lse_close(f64(lse), f64(ref_lse), f"noalloc {n_q}x{n_k}")
        outs.append(out)
    assert torch.equal(outs[0], outs[1])
    # both against the fp64 oracle: every row of small cases, sampled rows of
    # the others (tile edges, the ragged last tile, a seeded draw)
    if n_q * n_k <= 4_000_000:
        rows = np.arange(n_q)
    else:
        rng = np.random.default_rng(n_q)
        rows = np.unique(np.concatenate([[0, 127, 128, 255, 256, n_q - 1],
                                         rng.integers(0, n_q, 24)]))
        rows = rows[rows < n_q]
    for hd in sorted({0, heads - 1}):
        o_ref, lse_ref = attention.attend(f64(q[hd, rows]), f64(k[hd]), f64(v[hd]))
        assert_attn_close(f64(outs[1][rows, hd]), o_ref, f"noalloc vs oracle, head {hd}")
        assert_lse_close(f64(lse[rows, hd]), lse_ref, f"noalloc lse vs oracle, head {hd}")


def test_noalloc_split_case_runs_stream_k(pv):
    # the (256, 3000, 1, 128) case above cuts its one item across CTAs, so
    # the merge of the parts goes through the fixed scratch
    grid, mode, _ = pv.pv_attn_plan([256], [3000], 1, n_sm=148, partial_slots=SCRATCH_SLOTS_D128)
    assert mode == 0 and grid > 1


def test_noalloc_timeout_is_reported_through_the_scratch(pv):
    assert pv.pv_attn_poll_device_error(None) == 0
    pv.pv_attn_selftest_wait_timeout(None)   # a bounded wait that runs out (~1 s)
    with pytest.raises(pv.PVError) as e:
        pv.pv_attn_poll_device_error(None)
    assert e.value.status == pv.PV_ERR_TIMEOUT
    assert pv.pv_attn_poll_device_error(None) == 0   # cleared
    # the next call still computes the right thing
    n, H, Dh = 300, 2, 128
    q = synth.normal_bf16(81, (H, n, Dh), "cuda")
    k = synth.normal_bf16(82, (H, n, Dh), "cuda")
    v = synth.normal_bf16(83, (H, n, Dh), "cuda")
    out = torch.empty(n, H, Dh, dtype=torch.bfloat16, device="cuda")
    pv.pv_attn_dense_noalloc(q, k, v, n, n, H, Dh, out)
    assert pv.pv_attn_poll_device_error(None) == 0
    for hd in range(H):
        o_ref, _ = attention.attend(f64(q[hd]), f64(k[hd]), f64(v[hd]))
        assert_attn_close(f64(out[:, hd]), o_ref, f"noalloc after timeout, head {hd}")


def test_noalloc_refuses_sizes_beyond_its_scratch(pv):
    t = torch.zeros(64, dtype=torch.bfloat16, device="cuda")
    # 64 heads x ceil(33024 / 256) blocks x 2 tiles = 16512 query tiles > 16384
    with pytest.raises(pv.PVError) as e:
        pv.pv_attn_dense_noalloc(t, t, t, 33024, 128, 64, 128, t)
    assert e.value.status == pv.PV_ERR_CAPACITY
    assert "scratch" in str(e.value)
