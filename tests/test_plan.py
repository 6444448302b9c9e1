"""The attention work planner on the host (pv_attn_plan: no device needed).

An item is (sequence, head, 256-query block), a run of ceil(n_k / 128) key
tiles; items are laid out query-block-major and end to end.  Long items run
stream-K: CTA c takes the key tiles [ranges[c], ranges[c + 1]), and these
tests check the partition (non-empty, equal shares) and the alignment of the
four query blocks of a head that lets them share K/V in L2.  Short items, or
a workspace without room for split-KV partials, are handed out whole at run
time (mode 1): only the ends of the range table are defined then.
"""
import pytest

from same_step_kv_b200 import pv, synth

HEADS, T = 24, 880


def _items(n_q, n_k, heads=HEADS):
    """(start, tiles) of every item, in launch order (query-block-major per sequence)."""
    out, pos = [], 0
    for q, k in zip(n_q, n_k):
        if q == 0:
            continue
        kt = (k + 127) // 128
        for _ in range((q + 255) // 256 * heads):
            out.append((pos, kt))
            pos += kt
    return out, pos


def _check_partition(ranges, total):
    assert ranges[0] == 0 and ranges[-1] == total
    assert all(b > a for a, b in zip(ranges, ranges[1:])), "every CTA gets work"


def test_steady_chunk_is_stream_k_with_aligned_query_blocks():
    grid, mode, ranges = pv.pv_attn_plan([T], [18480], HEADS)
    items, total = _items([T], [18480])
    assert (grid, mode, total) == (148, 0, 24 * 4 * 145)
    _check_partition(ranges, total)
    assert ranges == [c * total // grid for c in range(grid + 1)]
    # 148 = 4 x 37 CTAs over 4 query-block layers of 3,480 tiles: CTA c and
    # CTA c + 37 start at the same key tile of the same head, one layer apart
    layer = total // 4
    for c in range(grid - 37):
        assert ranges[c + 37] - ranges[c] == layer


def _check_run_time(grid, mode, ranges, total):
    assert mode == 1
    assert ranges[0] == 0 and ranges[grid] == total
    assert all(r == -1 for r in ranges[1:grid])


def test_short_items_are_handed_out_whole():
    n_k = synth.text_lengths(8)
    n_q = [T] * 8
    grid, mode, ranges = pv.pv_attn_plan(n_q, n_k, HEADS)
    items, total = _items(n_q, n_k)
    assert grid == 148
    _check_run_time(grid, mode, ranges, total)


def test_long_items_fall_back_to_whole_items_without_partial_room():
    grid, mode, ranges = pv.pv_attn_plan([T], [18480], HEADS, partial_slots=100)
    items, total = _items([T], [18480])
    assert grid == min(148, len(items))
    _check_run_time(grid, mode, ranges, total)


def test_small_launch_uses_fewer_ctas():
    # one item of 3 key tiles: split over 3 CTAs (merged by the last to arrive)
    grid, mode, ranges = pv.pv_attn_plan([5], [300], 1)
    assert (grid, mode, ranges) == (3, 0, [0, 1, 2, 3])
    grid, mode, ranges = pv.pv_attn_plan([300], [20000], 2)  # 4 items of 157 tiles
    items, total = _items([300], [20000], 2)
    assert mode == 0 and grid == 148
    _check_partition(ranges, total)


def test_many_short_items():
    # 65,536+ items of one key tile each: handed out whole at run time
    n_q, n_k = [256 * 1100], [64]
    grid, mode, ranges = pv.pv_attn_plan(n_q, n_k, 64)
    items, total = _items(n_q, n_k, 64)
    assert len(items) > 0xFFFF and grid == 148
    _check_run_time(grid, mode, ranges, total)


def test_plan_rejects_bad_arguments():
    with pytest.raises(pv.PVError) as e:
        pv.pv_attn_plan([0, 0], [5, 5], HEADS)
    assert e.value.status == pv.PV_ERR_SHAPE
    with pytest.raises(pv.PVError) as e:
        pv.pv_attn_plan([5], [0], HEADS)
    assert e.value.status == pv.PV_ERR_SHAPE
    with pytest.raises(pv.PVError):
        pv.pv_attn_plan([5], [5], HEADS, n_sm=0)
