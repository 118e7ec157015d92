"""The metadata checks of ``metadata_check.py`` accept a list written in the
documented order and reject the plausible device mistakes planted here on the
CPU: a duplicated item, a dropped item, an altered cost, a run out of key
order, a swapped dense pair, a launch order that is not longest first.  The GPU
tests then apply the same checks to what the kernels wrote."""
import numpy as np
import pytest

import metadata_check as mc

LQ = np.array([300, 45, 0, 513, 1, 128, 128], dtype=np.int64)
LKV = np.array([300, 45, 7, 513, 1, 128, 4000], dtype=np.int64)
HQ, HKV = 8, 2


def _device_like_list(lq, lkv, causal, order=None):
    keys = [mc.sequence_key(int(a), int(b), causal) for a, b in zip(lq, lkv)]
    if order is None:
        order = sorted(range(len(lq)), key=lambda b: -keys[b])
    items = []
    for b in order:
        items += mc.sequence_block(b, int(lq[b]), int(lkv[b]), HQ, HKV, causal)
    return np.array(items, dtype=np.int64).reshape(-1, 4)


@pytest.mark.parametrize("causal", [True, False])
def test_valid_list_passes(causal):
    items = _device_like_list(LQ, LKV, causal)
    mc.check_sequence_list(items, len(items), LQ, LKV, HQ, HKV, causal)


def test_bottom_right_tile_counts():
    # 1 query over 300 keys sees all 3 tiles; the first tile of a 513 x 513 causal sequence sees 1 tile
    assert mc.kv_tiles_visited(0, 1, 300, True) == 3
    assert mc.kv_tiles_visited(0, 513, 513, True) == 1
    assert mc.kv_tiles_visited(4, 513, 513, True) == 5
    # more queries than keys: the first rows see nothing
    assert mc.kv_tiles_visited(0, 300, 40, True) == 0
    assert mc.kv_tiles_visited(2, 300, 40, True) == 1
    assert mc.kv_tiles_visited(0, 10, 0, False) == 0


def test_duplicated_item_fails():
    items = _device_like_list(LQ, LKV, True)
    bad = items.copy()
    bad[3] = bad[2]
    with pytest.raises(AssertionError):
        mc.check_sequence_list(bad, len(bad), LQ, LKV, HQ, HKV, True)


def test_dropped_item_fails():
    items = _device_like_list(LQ, LKV, True)
    bad = np.delete(items, 5, axis=0)
    with pytest.raises(AssertionError):
        mc.check_sequence_list(bad, len(bad), LQ, LKV, HQ, HKV, True)
    # the same list claimed to be complete with the right count still fails (a run is short)
    with pytest.raises(AssertionError):
        mc.check_sequence_list(np.vstack([bad, bad[-1:]]), len(items), LQ, LKV, HQ, HKV, True)


def test_altered_cost_fails():
    bad = _device_like_list(LQ, LKV, True)
    bad[0, 3] += 1
    with pytest.raises(AssertionError):
        mc.check_sequence_list(bad, len(bad), LQ, LKV, HQ, HKV, True)


def test_runs_out_of_key_order_fail():
    keys = [mc.sequence_key(int(a), int(b), True) for a, b in zip(LQ, LKV)]
    order = sorted(range(len(LQ)), key=lambda b: keys[b])  # shortest first
    bad = _device_like_list(LQ, LKV, True, order=[b for b in order if LQ[b] > 0])
    with pytest.raises(AssertionError):
        mc.check_sequence_list(bad, len(bad), LQ, LKV, HQ, HKV, True)


def test_dense_list_swap_fails():
    want = np.array(mc.dense_list(2, 1100, 1100, 8, 2, True), dtype=np.int64)
    mc.check_dense_list(want, len(want), 2, 1100, 1100, 8, 2, True)
    bad = want.copy()
    bad[[0, 1]] = bad[[1, 0]]
    with pytest.raises(AssertionError):
        mc.check_dense_list(bad, len(bad), 2, 1100, 1100, 8, 2, True)


def test_decode_order_checks():
    lens = np.array([5, 70000, 3, 70000, 4096], dtype=np.int64)
    mc.check_decode_order([1, 3, 4, 0, 2], lens, 70000)
    with pytest.raises(AssertionError):
        mc.check_decode_order([1, 3, 0, 4, 2], lens, 70000)
    with pytest.raises(AssertionError):
        mc.check_decode_order([1, 1, 4, 0, 2], lens, 70000)


def test_page_coords_rule():
    table = np.array([[7, 2, -1], [0, 9, 1]], dtype=np.int32)
    got = mc.page_coords(table, [0, 0, 1, 0, 1], [0, 70, 65, 130, 127], 64, 9, 8)
    assert got.tolist() == [[7, 0, 56], [2, 6, 16], [-1, 1, -1], [-1, 2, -1], [-1, 63, -1]]


def test_routed_short_sequences_have_no_items():
    lq = np.array([1, 4, 5, 0, 300], dtype=np.int64)
    lkv = np.array([900, 100, 5, 3, 300], dtype=np.int64)
    assert mc.routed_qmax(4, 300) == 4 and mc.routed_qmax(32, 300) == 2 and mc.routed_qmax(128, 300) == 0
    assert mc.sequence_block(0, 1, 900, 8, 2, True, short_q=4) == []
    keys = [mc.sequence_key(int(a), int(b), True, 4) for a, b in zip(lq, lkv)]
    order = sorted(range(len(lq)), key=lambda b: -keys[b])
    items = [it for b in order for it in mc.sequence_block(b, int(lq[b]), int(lkv[b]), 8, 2, True, 4)]
    mc.check_sequence_list(np.array(items), len(items), lq, lkv, 8, 2, True, short_q=4)
    # a list that still holds the 1-query sequence's items is rejected
    extra = mc.sequence_block(0, 1, 900, 8, 2, True)
    with pytest.raises(AssertionError):
        mc.check_sequence_list(np.array(items + extra), len(items) + len(extra), lq, lkv, 8, 2, True, short_q=4)


def _pieces(L, Hkv, S, maxL, cu_q=None, qmax=1):
    seq = mc.decode_units(L, maxL, cu_q, qmax)
    shift = mc.decode_sort_shift(maxL)
    order = sorted(range(len(L)), key=lambda b: -min(mc.SORT_CAP, seq[b][0] >> shift))
    rows = mc.decode_pieces(seq, order, Hkv, S)
    full = np.array(rows + [(-1, 0, 0, 0, 0, 0, 0, 0)] * (S * len(L) * Hkv - len(rows)), dtype=np.int64)
    return order, full


@pytest.mark.parametrize("cu", [False, True])
def test_split_pieces_rule_passes(cu):
    L = [5000, 0, 64, 65, 1, 3000, 129, 7]
    cu_q, qmax = (np.array([0, 1, 4, 704, 706, 706, 707, 836, 840]), 4) if cu else (None, 1)
    order, rows = _pieces(L, 2, 3, 5000, cu_q, qmax)
    mc.check_decode_pieces(order, rows, L, 2, 3, 5000, cu_q, qmax)
    # pieces of one pair differ by at most one unit
    for r in rows[rows[:, 0] >= 0]:
        n = mc.decode_units(L, 5000, cu_q, qmax)[r[0] // 2][0]
        assert (r[2] - r[1]) in (n // r[4], -(-n // r[4]))


def test_split_pieces_out_of_order_fails():
    L = [5000, 64, 3000]
    order, rows = _pieces(L, 2, 3, 5000)
    with pytest.raises(AssertionError):
        mc.check_decode_pieces([order[1], order[0], order[2]], rows, L, 2, 3, 5000)


@pytest.mark.parametrize("field,delta", [(1, 1), (2, -1), (3, 1), (4, 1)])
def test_split_pieces_altered_record_fails(field, delta):
    """A piece that starts or ends one unit off (a gap or an overlap), or points at
    the wrong slots or piece count, is rejected."""
    L = [5000, 64, 3000]
    order, rows = _pieces(L, 2, 3, 5000)
    bad = rows.copy()
    bad[1, field] += delta
    with pytest.raises(AssertionError):
        mc.check_decode_pieces(order, bad, L, 2, 3, 5000)
