"""Host logic of the attention work schedule (gqa_prefill_schedule; no device needed).

The persistent attention kernel walks per-CTA lists of work items, each a pair of 128-row query tiles of
one (batch row, KV group).  These tests check the lists the library builds against the item enumeration
(causal key-tile counts computed here from the shapes), not against its own code.
"""
import ctypes

import numpy as np
import pytest
from hypothesis import given, settings, strategies as st

import grouped_query_attention_gqa_b200 as G
from grouped_query_attention_gqa_b200 import _lib


def item_tiles(B, L, h_q, h_kv):
    """Key tiles of every item: the group's query tiles listed by tile descending, head ascending, paired."""
    nq = (L + 127) // 128
    g = h_q // h_kv
    tpg = nq * g
    total = (tpg + 1) // 2 * B * h_kv
    out = []
    for w in range(total):
        pair = w // (B * h_kv)
        i0, i1 = 2 * pair, 2 * pair + 1
        out.append((nq - i0 // g if i0 < tpg else 0) + (nq - i1 // g if i1 < tpg else 0))
    return np.array(out)


def snake_loads(tiles, grid):
    load = np.zeros(grid, dtype=np.int64)
    for w, t in enumerate(tiles):
        r, c = divmod(w, grid)
        load[grid - 1 - c if r & 1 else c] += t
    return load


SHAPES = [(1, 4096, 28, 4), (2, 4096, 28, 4), (1, 700, 28, 4), (1, 128, 14, 2), (3, 1000, 7, 1),
          (1, 8192, 28, 4), (4, 4096, 64, 8), (2, 300, 8, 8)]


@pytest.mark.parametrize("B,L,h_q,h_kv", SHAPES)
def test_every_item_exactly_once_heaviest_first(B, L, h_q, h_kv):
    tiles = item_tiles(B, L, h_q, h_kv)
    lists, _ = G.prefill_schedule(B, L, h_q, h_kv, 148)
    assert len(lists) == min(148, len(tiles))
    flat = np.concatenate([np.array(l, dtype=np.int64) for l in lists])
    assert np.array_equal(np.sort(flat), np.arange(len(tiles)))
    _, grouped = G.prefill_schedule(B, L, h_q, h_kv, 148)
    if not grouped:
        for l in lists:
            assert np.all(np.diff(tiles[l]) <= 0)   # each CTA takes its heaviest item first


def test_packing_balances_the_headline_shape():
    """Qwen2-7B at L=4096: 448 items over 148 CTAs.  Round-robin leaves the busiest CTA ~10 % above the
    mean number of key tiles; the packing is used there and its busiest CTA carries fewer key tiles."""
    B, L, h_q, h_kv = 1, 4096, 28, 4
    tiles = item_tiles(B, L, h_q, h_kv)
    lists, grouped = G.prefill_schedule(B, L, h_q, h_kv, 148)
    assert not grouped
    packed = np.array([tiles[l].sum() for l in lists])
    rr = snake_loads(tiles, 148)
    assert rr.max() > 1.09 * tiles.sum() / 148
    assert packed.max() < rr.max()
    assert packed.sum() == tiles.sum()


def group_planes(B, L, h_kv):
    """Planes dealt together: K' and V of d = 128 within 16 MB, at least one, at most all."""
    return max(1, min(B * h_kv, (16 << 20) // (2 * L * 128 * 2)))


@pytest.mark.parametrize("B,L,h_q,h_kv", [(1, 16384, 28, 4), (2, 8192, 28, 4)])
def test_many_items_round_robin_where_all_planes_fit_l2(B, L, h_q, h_kv):
    """K' and V of all planes within 48 MB: the snake order, as lists."""
    tiles = item_tiles(B, L, h_q, h_kv)
    lists, grouped = G.prefill_schedule(B, L, h_q, h_kv, 148)
    assert not grouped
    for c, l in enumerate(lists):
        expect = [w for w in range(len(tiles)) if (147 - w % 148 if (w // 148) & 1 else w % 148) == c]
        assert l == expect


@pytest.mark.parametrize("B,L,h_q,h_kv", [(1, 32768, 28, 4), (4, 8192, 64, 8)])
def test_many_items_dealt_by_plane_group_and_balanced(B, L, h_q, h_kv):
    """Where round-robin would already balance (many items per CTA), the items are dealt plane group by
    plane group for L2 reuse: every CTA's list runs through the groups in order, and the busiest CTA stays
    within one item of the mean load (costs: key tiles + 4 per item)."""
    tiles = item_tiles(B, L, h_q, h_kv)
    lists, grouped = G.prefill_schedule(B, L, h_q, h_kv, 148)
    assert grouped
    rr = snake_loads(tiles, 148)
    assert rr.max() <= 1.01 * tiles.sum() / 148 + tiles.max()   # the round-robin order was balanced too
    planes, gp = B * h_kv, group_planes(B, L, h_kv)
    cost = tiles + 4
    loads = np.array([cost[l].sum() for l in lists])
    assert loads.max() <= loads.mean() + cost.max()
    for l in lists:
        grp = (np.array(l) % planes) // gp
        assert np.all(np.diff(grp) >= 0)                       # groups in order
        for g in np.unique(grp):                                # heaviest first within a group
            assert np.all(np.diff(tiles[np.array(l)[grp == g]]) <= 0)


def test_fewer_items_than_ctas():
    lists, _ = G.prefill_schedule(1, 128, 14, 2, 148)   # 8 items (2 groups x 4 pairs): one per CTA
    assert all(len(l) == 1 for l in lists)


@pytest.mark.parametrize("args", [(0, 16, 28, 4, 148), (1, 0, 28, 4, 148), (1, 16, 28, 5, 148), (1, 16, 28, 4, 0),
                                  (1, 16, 0, 4, 148), (1, 16, 28, -4, 148)])
def test_schedule_validation(args):
    lib = _lib.load()
    assert lib.gqa_prefill_schedule(*args, None, None, 0, None) == -2   # GQA_ERR_DIMS


def test_small_capacity_leaves_arrays_untouched():
    lib = _lib.load()
    starts = (ctypes.c_int * 149)(*([-7] * 149))
    items = (ctypes.c_int * 4)(*([-7] * 4))
    n = lib.gqa_prefill_schedule(1, 4096, 28, 4, 148, starts, items, 4, None)
    assert n == 448
    assert list(starts) == [-7] * 149 and list(items) == [-7] * 4


@settings(max_examples=60, deadline=None)
@given(B=st.integers(1, 6), L=st.integers(1, 9000), h_kv=st.sampled_from([1, 2, 4, 8]),
       g=st.sampled_from([1, 2, 3, 7, 8, 16]), grid=st.sampled_from([1, 7, 132, 148]))
def test_schedule_properties_on_random_shapes(B, L, h_kv, g, grid):
    """Any shape and CTA count: every item exactly once, no more lists than CTAs or items, each list
    heaviest first where the items are packed or dealt round-robin, and plane groups in order where they
    are dealt by group."""
    h_q = g * h_kv
    tiles = item_tiles(B, L, h_q, h_kv)
    lists, grouped = G.prefill_schedule(B, L, h_q, h_kv, grid)
    assert len(lists) == min(grid, len(tiles))
    flat = np.concatenate([np.array(l, dtype=np.int64) for l in lists]) if lists else np.array([], np.int64)
    assert np.array_equal(np.sort(flat), np.arange(len(tiles)))
    planes = B * h_kv
    for l in lists:
        l = np.array(l, dtype=np.int64)
        if grouped:
            gp = group_planes(B, L, h_kv)
            grp = (l % planes) // gp
            assert np.all(np.diff(grp) >= 0)
            for gg in np.unique(grp):
                assert np.all(np.diff(tiles[l[grp == gg]]) <= 0)
        elif len(l) > 1:
            # packed lists are heaviest first; round-robin lists follow the item order, which is heaviest first too
            assert np.all(np.diff(tiles[l]) <= 0)
