"""The C-ABI library on the host: it loads, exports every symbol that
include/pv.h declares, and its chunk bookkeeping matches the oracle bit for
bit.  No CUDA device is used (bookkeeping-only handles)."""
import os
import re

import pytest

from oracle.schedule import Geometry, RingModel
from same_step_kv_b200 import pv

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_symbols():
    text = open(os.path.join(ROOT, "include", "pv.h")).read()
    return sorted(set(re.findall(r"^PV_API\s+[\w\s\*]+?\b(pv_\w+)\s*\(", text, flags=re.M)))


def test_library_exports_every_declared_symbol():
    names = declared_symbols()
    assert len(names) >= 17
    for n in names:
        assert hasattr(pv.lib, n), n
    assert "sm_100a" in pv.pv_version()


def _cfg(R, D=64, W=8, Hh=4, H=2, layers=2, streams=2):
    return pv.make_config(layers, H, D, W, Hh, ring_slots=R, max_streams=streams, max_frames=64)


PHASE = {"NEW": pv.PV_PHASE_NEW, "FIRST": pv.PV_PHASE_FIRST, "BOOT": pv.PV_PHASE_BOOT,
         "STEADY": pv.PV_PHASE_STEADY}


def _compare(st, ring: RingModel, R):
    assert st.phase == PHASE[ring.phase]
    assert st.chunk == ring.chunk
    if ring.phase == "STEADY":
        assert st.slot == ring.current_slot()
        assert st.fill == ring.fill()
        assert list(st.slot_frame[:R]) == ring.slot_frames()
        assert st.frame0 == ring.current_frames()[0]
        assert st.nframes == len(ring.current_frames())
    assert st.n_keys == ring.n_keys()
    assert st.n_queries == len(ring.current_frames()) * ring.geom.tokens_per_frame


@pytest.mark.parametrize("R", [1, 2, 3, 18, 19])
def test_bookkeeping_bit_exact_against_oracle(R):
    h = pv.pv_kv_init(_cfg(R))
    geom = Geometry(8, 4, 2, 64, ring_slots=R)
    ring = RingModel(geom)
    pv.pv_kv_begin_chunk(h, 1, 3)
    ring.begin_chunk(3)
    _compare(pv.pv_kv_get_state(h, 1), ring, R)
    pv.pv_kv_begin_sink(h, 1)
    ring.bootstrap()
    _compare(pv.pv_kv_get_state(h, 1), ring, R)
    for _ in range(40):
        pv.pv_kv_begin_chunk(h, 1, 1)
        ring.begin_chunk(1)
        _compare(pv.pv_kv_get_state(h, 1), ring, R)
    # stream 0 was never touched
    assert pv.pv_kv_get_state(h, 0).phase == pv.PV_PHASE_NEW
    pv.pv_kv_destroy(h)


def test_production_profile_reaches_18480_keys():
    h = pv.pv_kv_init(pv.make_config(30, 24, 128, 40, 22, ring_slots=18))
    pv.pv_kv_begin_chunk(h, 0, 3)
    assert pv.pv_kv_get_state(h, 0).n_keys == 2640
    pv.pv_kv_begin_sink(h, 0)
    for j in range(1, 29):
        pv.pv_kv_begin_chunk(h, 0, 1)
    st = pv.pv_kv_get_state(h, 0)
    assert (st.chunk, st.fill, st.slot, st.n_keys, st.n_queries, st.frame0) == \
        (28, 18, 9, 18480, 880, 30)
    pv.pv_kv_destroy(h)


def test_schedule_misuse_is_rejected_and_leaves_state():
    h = pv.pv_kv_init(_cfg(2))
    with pytest.raises(pv.PVError) as e:
        pv.pv_kv_begin_chunk(h, 0, 1)
    assert e.value.status == pv.PV_ERR_STATE
    with pytest.raises(pv.PVError):
        pv.pv_kv_begin_sink(h, 0)
    pv.pv_kv_begin_chunk(h, 0, 3)
    with pytest.raises(pv.PVError):
        pv.pv_kv_begin_chunk(h, 0, 1)             # sink pass first
    pv.pv_kv_begin_sink(h, 0)
    with pytest.raises(pv.PVError):
        pv.pv_kv_begin_chunk(h, 0, 3)             # later chunks have one frame
    with pytest.raises(pv.PVError):
        pv.pv_kv_begin_sink(h, 0)
    assert pv.pv_kv_get_state(h, 0).phase == pv.PV_PHASE_BOOT
    with pytest.raises(pv.PVError) as e:
        pv.pv_kv_begin_chunk(h, 5, 1)
    assert e.value.status == pv.PV_ERR_INVALID_ARG
    # kernels need device buffers
    with pytest.raises(pv.PVError) as e:
        pv.pv_rope_append(h, [0], 0, pv.PV_STEP_SINK, 16, 16, 16, 16)
    assert e.value.status == pv.PV_ERR_STATE
    with pytest.raises(pv.PVError) as e:
        pv.pv_chunk_attn(h, [0], 0, 0, 16, 16)
    assert e.value.status == pv.PV_ERR_STATE
    pv.pv_kv_destroy(h)


def test_max_frames_bounds_the_schedule():
    h = pv.pv_kv_init(pv.make_config(1, 2, 64, 8, 4, ring_slots=2, max_frames=5))
    pv.pv_kv_begin_chunk(h, 0, 3)
    pv.pv_kv_begin_sink(h, 0)
    pv.pv_kv_begin_chunk(h, 0, 1)   # frame 3
    pv.pv_kv_begin_chunk(h, 0, 1)   # frame 4
    with pytest.raises(pv.PVError) as e:
        pv.pv_kv_begin_chunk(h, 0, 1)
    assert e.value.status == pv.PV_ERR_CAPACITY
    pv.pv_kv_destroy(h)


@pytest.mark.parametrize("bad", [
    dict(head_dim=96), dict(ring_slots=0), dict(ring_slots=65), dict(steps=9),
    dict(rope_pairs=(10, 10, 10)), dict(max_streams=65), dict(rope_theta=1.0),
    # sizes whose int products would overflow: rejected before they are formed
    dict(frame_w=65536, frame_h=65536), dict(frame_w=4097, frame_h=4096),
    dict(max_frames=(1 << 20) + 1), dict(max_frames=(1 << 31) - 1)])
def test_bad_configs_are_rejected(bad):
    kw = dict(layers=1, heads=2, head_dim=64, frame_w=8, frame_h=4)
    kw.update({k: v for k, v in bad.items() if k in kw})
    extra = {k: v for k, v in bad.items() if k not in kw}
    cfg = pv.make_config(**kw, **extra)
    with pytest.raises(pv.PVError) as e:
        pv.pv_kv_required_bytes(cfg)
    assert e.value.status == pv.PV_ERR_SHAPE


def test_required_bytes_closed_form():
    cfg = pv.make_config(30, 24, 128, 40, 22, ring_slots=18)
    kv, ws = pv.pv_kv_required_bytes(cfg)
    assert kv == 2 * 30 * 4 * 1 * 24 * (3 + 18) * 880 * 128 * 2
    assert ws > 0 and ws % 256 == 0


def test_state_checkpoint_restore():
    for R in (2, 18):
        a = pv.pv_kv_init(_cfg(R))
        pv.pv_kv_begin_chunk(a, 0, 3)
        pv.pv_kv_begin_sink(a, 0)
        for _ in range(25):
            pv.pv_kv_begin_chunk(a, 0, 1)
        snap = pv.pv_kv_get_state(a, 0)
        b = pv.pv_kv_init(_cfg(R))
        pv.pv_kv_set_state(b, 1, snap)
        got = pv.pv_kv_get_state(b, 1)
        for f in ("phase", "chunk", "fill", "slot", "frame0", "nframes", "n_queries", "n_keys"):
            assert getattr(got, f) == getattr(snap, f), f
        assert list(got.slot_frame) == list(snap.slot_frame)
        # both continue identically
        pv.pv_kv_begin_chunk(a, 0, 1)
        pv.pv_kv_begin_chunk(b, 1, 1)
        assert list(pv.pv_kv_get_state(a, 0).slot_frame) == list(pv.pv_kv_get_state(b, 1).slot_frame)
        bad = pv.pv_kv_state()
        bad.phase = 7
        with pytest.raises(pv.PVError):
            pv.pv_kv_set_state(b, 0, bad)
        pv.pv_kv_destroy(a)
        pv.pv_kv_destroy(b)


def test_row_offsets_follow_the_documented_layout():
    cfg = _cfg(2)
    h = pv.pv_kv_init(cfg)
    T, ltot = 32, (3 + 2) * 32
    k0, v0 = pv.pv_kv_row_offset(h, 1, 2, 1, 1, 7)
    row = (((1 * 4 + 2) * 2 + 1) * 2 + 1) * ltot + 7
    assert k0 == row * 64
    assert v0 == (2 * 4 * 2 * 2 * ltot + row) * 64
    with pytest.raises(pv.PVError):
        pv.pv_kv_row_offset(h, 2, 0, 0, 0, 0)
    pv.pv_kv_destroy(h)


# ------------------------------------------------------------------ sampler schedule (host)
from oracle import euler  # noqa: E402
from golden_io import load as read_golden  # noqa: E402


@pytest.mark.parametrize("n,shift", [(1, 1.0), (4, 1.0), (4, 5.0), (40, 12.0), (50, 3.0),
                                     (1000, 12.0)])
def test_sigma_schedule_matches_oracle(n, shift):
    sig, ts = pv.pv_sigma_schedule(n, shift)
    ref = euler.shifted_schedule(n, shift)
    assert len(sig) == n + 1 and sig[-1] == 0.0
    for a, b in zip(sig, ref):
        assert abs(a - b) <= 4e-16 * max(1.0, abs(b))
    assert ts == list(euler.timesteps(ref[:-1]))


def test_sigma_schedule_printed_timesteps():
    g = read_golden("shift_schedule.txt")
    sig, ts = pv.pv_sigma_schedule(int(g["steps"]), float(g["shift"]))
    assert ts[:6] == [int(g[f"t{i}"]) for i in range(6)]
    assert sum(t >= int(g["high_noise_boundary"]) for t in ts) == int(g["steps_at_or_above_boundary"])


def test_sigma_schedule_explicit_top_and_errors():
    sig, ts = pv.pv_sigma_schedule(4, 1.0, 1.0)
    assert sig == [1.0, 0.75, 0.5, 0.25, 0.0]      # the plain four-step grid
    assert ts == [1000, 750, 500, 250]
    for args in [(0, 1.0), (4, 0.0), (4, -2.0), (4, float("nan")), (4, 1.0, 1.5)]:
        with pytest.raises(pv.PVError) as e:
            pv.pv_sigma_schedule(*args)
        assert e.value.status == pv.PV_ERR_INVALID_ARG


# ------------------------------------------------------------------ varlen attention (host checks)
def test_varlen_workspace_and_shape_checks():
    one = pv.pv_attn_varlen_ws_bytes([880], [512], 24, 128)
    dense = pv.pv_attn_dense_ws_bytes(880, 512, 24, 128)
    assert one == dense and one % 256 == 0
    batch = pv.pv_attn_varlen_ws_bytes([2640, 880, 0, 880], [77, 512, 0, 1], 24, 128)
    assert batch > one
    for n_q, n_k, D in (([5], [0], 128), ([-1], [3], 128), ([1] * 65, [1] * 65, 128),
                        ([4], [4], 96)):
        with pytest.raises(pv.PVError) as e:
            pv.pv_attn_varlen_ws_bytes(n_q, n_k, 2, D)
        assert e.value.status == pv.PV_ERR_SHAPE
    # no queries anywhere: a no-op that touches no device
    pv.pv_attn_varlen(0, 0, 0, [0, 0], [3, 0], 2, 64, 0, None, 0, 0)


def test_lengths_above_two_to_the_30_are_rejected():
    # a length near 2^31 would overflow the int tile counts (n + 255) / 256;
    # every entry point rejects lengths above 2^30 before forming them
    big, ok = (1 << 30) + 1, 1 << 30
    assert pv.pv_attn_dense_ws_bytes(ok, 1, 1, 64) > 0
    calls = [
        lambda: pv.pv_attn_dense_ws_bytes(big, 1, 1, 64),
        lambda: pv.pv_attn_dense_ws_bytes(1, (1 << 31) - 1, 1, 64),
        lambda: pv.pv_attn_varlen_ws_bytes([big], [1], 1, 64),
        lambda: pv.pv_attn_varlen_ws_bytes([1], [(1 << 31) - 1], 1, 64),
        lambda: pv.pv_attn_plan([(1 << 31) - 1], [1], 1),
        # pointers are checked for NULL only before the shapes, never touched
        lambda: pv.pv_attn_dense(256, 256, 256, (1 << 31) - 1, 1, 1, 64, 256, None, 256, 0),
        lambda: pv.pv_attn_dense_noalloc(256, 256, 256, 1, big, 1, 64, 256),
    ]
    for call in calls:
        with pytest.raises(pv.PVError) as e:
            call()
        assert e.value.status == pv.PV_ERR_SHAPE


# ------------------------------------------------------------------ q/k/v projection (host checks)
def test_qkv_workspace_and_host_checks():
    # y in f32 for 3 * dim features per token, two sums of squares per token,
    # then two arrival counters per block of 256 tokens (the fused launch)
    ws = pv.pv_qkv_ws_bytes(880, 3072)
    y = 880 * 3 * 3072 * 4
    r = lambda n: ((n + 255) // 256) * 256
    # y, then one partial sum of squares per token, q / k and 256-feature tile
    assert ws == r(y) + r(880 * 2 * 12 * 4)
    for args in ((0, 3072), (880, 100), (880, 0)):
        with pytest.raises(pv.PVError) as e:
            pv.pv_qkv_ws_bytes(*args)
        assert e.value.status == pv.PV_ERR_SHAPE
    # a bookkeeping-only handle has no store to append into
    h = pv.pv_kv_init(_cfg(2))
    pv.pv_kv_begin_chunk(h, 0, 3)
    with pytest.raises(pv.PVError) as e:
        pv.pv_qkv_rope_append(h, [0], 0, 0, 16, 16, 16, 16, 16, 1e-6, 16, 256, 1 << 20)
    assert e.value.status == pv.PV_ERR_STATE
    pv.pv_kv_destroy(h)
