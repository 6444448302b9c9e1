"""Failure detection on the GPU without a fault: a device-side wait that runs
out (an mbarrier that nothing arrives on) gives up after its bound, records
a timeout in the handle's error word and returns; the host reads
PV_ERR_TIMEOUT, the word is cleared, and the context keeps working."""
import numpy as np
import pytest
import torch

from gpu_common import assert_attn_close, f64
from oracle import attention
from same_step_kv_b200 import synth

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def pv():
    from same_step_kv_b200 import pv as m
    return m


def test_wait_timeout_reports_status_and_context_survives(pv):
    cfg = pv.make_config(1, 2, 64, 8, 4, ring_slots=2, max_frames=64)
    store = pv.KVStore(cfg)
    h = store.handle
    assert pv.pv_kv_poll_device_error(h) == 0
    pv.pv_kv_selftest_wait_timeout(h)
    torch.cuda.synchronize()          # the bounded wait takes about a second
    with pytest.raises(pv.PVError) as e:
        pv.pv_kv_poll_device_error(h)
    assert e.value.status == pv.PV_ERR_TIMEOUT
    assert pv.pv_kv_poll_device_error(h) == 0   # cleared
    # the context is still usable: a dense attention call matches the oracle
    n, H, Dh = 200, 2, 64
    q = synth.normal_bf16(71, (H, n, Dh), "cuda")
    k = synth.normal_bf16(72, (H, n, Dh), "cuda")
    v = synth.normal_bf16(73, (H, n, Dh), "cuda")
    out = torch.empty(n, H, Dh, dtype=torch.bfloat16, device="cuda")
    wsb = pv.pv_attn_dense_ws_bytes(n, n, H, Dh)
    ws = torch.zeros(wsb, dtype=torch.uint8, device="cuda")
    pv.pv_attn_dense(q, k, v, n, n, H, Dh, out, None, ws, wsb)
    torch.cuda.synchronize()
    for hd in range(H):
        o_ref, _ = attention.attend(f64(q[hd]), f64(k[hd]), f64(v[hd]))
        assert_attn_close(f64(out[:, hd]), o_ref, f"after timeout, head {hd}")
    store.close()


def test_workspace_error_word_reports_timeout(pv):
    # the caller-workspace entry points: word 0 of ws is the device error word
    n, H, Dh = 200, 2, 64
    wsb = pv.pv_attn_dense_ws_bytes(n, n, H, Dh)
    ws = torch.zeros(wsb, dtype=torch.uint8, device="cuda")
    assert pv.pv_attn_poll_device_error(ws, wsb) == 0
    pv.pv_attn_selftest_wait_timeout(ws)
    with pytest.raises(pv.PVError) as e:
        pv.pv_attn_poll_device_error(ws, wsb)
    assert e.value.status == pv.PV_ERR_TIMEOUT
    assert pv.pv_attn_poll_device_error(ws, wsb) == 0
    assert int(ws.sum().item()) == 0          # the workspace is zeroed again
    q = synth.normal_bf16(74, (H, n, Dh), "cuda")
    k = synth.normal_bf16(75, (H, n, Dh), "cuda")
    v = synth.normal_bf16(76, (H, n, Dh), "cuda")
    out = torch.empty(n, H, Dh, dtype=torch.bfloat16, device="cuda")
    pv.pv_attn_dense(q, k, v, n, n, H, Dh, out, None, ws, wsb)
    assert pv.pv_attn_poll_device_error(ws, wsb) == 0
    for hd in range(H):
        o_ref, _ = attention.attend(f64(q[hd]), f64(k[hd]), f64(v[hd]))
        assert_attn_close(f64(out[:, hd]), o_ref, f"workspace after timeout, head {hd}")
