"""pv_attn_dense_noalloc: the dense attention entry point for callers that
cannot allocate device memory where they call it (allocator callbacks,
plugins whose host owns every allocation, paths that must not touch the
allocator).  It keeps its split-KV scratch in a fixed array inside the
library; this test checks, through the C ABI, that two calls in a row give
the same result as pv_attn_dense with a caller workspace, within the
attention tolerance the other tests use, and that an oversized problem is
refused on the host.  The file sorts last so that it runs after every other
test, and it also passes on its own in a fresh process."""
import numpy as np
import pytest
import torch

from gpu_common import assert_attn_close, assert_lse_close, f64
from same_step_kv_b200 import synth

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def pv():
    from same_step_kv_b200 import pv as m
    return m


@pytest.mark.parametrize("n_q,n_k,heads,dim", [
    (200, 9000, 2, 128),      # split-KV: the merge runs through the fixed scratch
    (257, 385, 3, 64),
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


def test_noalloc_refuses_sizes_beyond_its_scratch(pv):
    t = torch.zeros(64, dtype=torch.bfloat16, device="cuda")
    # 64 heads x ceil(33024 / 256) blocks x 2 tiles = 16512 query tiles > 16384
    with pytest.raises(pv.PVError) as e:
        pv.pv_attn_dense_noalloc(t, t, t, 33024, 128, 64, 128, t)
    assert e.value.status == pv.PV_ERR_CAPACITY
    assert "scratch" in str(e.value)
