"""Host-side checks of the metadata the library builds on the device: the
prefill work lists (ragged, paged-prefill and dense), the split-decode launch
order and the page-table coordinates.  Each expected value is computed here
from the rule the header and the design state, with plain Python, not with the
library.  Used by ``test_gpu_metadata.py`` (device lists) and
``test_metadata_check_cpu.py`` (the checks themselves reject planted mistakes).

Work-list rules (one item = (sequence b, 128-row query tile qt, first query
head h0 of the pair, KV tiles the item visits)):
  * a query tile visits every 128-key tile that holds a key some row of the
    tile may see (bottom-right causal: row i of Lq sees keys j <= i + Lkv - Lq);
  * ragged / paged: sequences of 1..short_q queries have no items (ragged
    queries over a paged cache send them to the split-KV decode kernel,
    short_q = min(4, 64 / G, max_seqlen_q)); a sequence's items form one contiguous run ordered
    (kv head, query tile longest first, head pair); runs are ordered by the
    sequence's total tile steps (capped at 4095), most first, ties in any order;
  * dense: groups of 16 query tiles, the group of longest tiles first, inside a
    group (batch, kv head, query tile longest first, head pair);
  * header[0] = item count; after the prefill ran, header[1] = item count +
    number of persistent CTAs (each CTA makes one claim past the end).

Split decode (GQA, num_splits = S > 1):
  * sequence b owns n_b = max(1, ceil(L_b / 64)) 64-key units when the decode
    kernel takes its rows (always without cu_q; 1 <= Lq <= qmax with it), else 0;
  * the order lists the sequences longest first by key min(4095, n_b >> shift),
    shift the smallest with (max_kv_len // 64 + 1) >> shift < 4096, ties in any order;
  * in that order each of a sequence's Hkv pairs p = b * Hkv + g takes k = min(S, n_b)
    consecutive blocks slot0 .. slot0 + k - 1; block slot0 + s runs units
    [s n_b // k, (s+1) n_b // k): record (p, j0, j1, slot0, k, L, q0, Lq); blocks past
    the last piece have p = -1.
"""
from __future__ import annotations

import numpy as np

SORT_CAP = 4095
DENSE_GROUP = 16


def heads_per_item(Hq, Hkv):
    """Query heads per work item: the two heads of a pair that share a KV head (one when G is odd)."""
    return 2 if (Hq // Hkv) % 2 == 0 else 1


def kv_tiles_visited(qt, Lq, Lkv, causal):
    """128-key tiles holding at least one key visible to a row of query tile qt."""
    if Lkv <= 0:
        return 0
    if not causal:
        return (Lkv + 127) // 128
    last_row = min(Lq, (qt + 1) * 128) - 1
    max_key = min(Lkv - 1, last_row + Lkv - Lq)
    return 0 if max_key < 0 else max_key // 128 + 1


def routed_qmax(G, max_seqlen_q):
    """Query count up to which ragged queries over a paged cache take the decode kernel."""
    return 0 if G > 64 else min(4, 64 // G, max_seqlen_q)


def sequence_block(b, Lq, Lkv, Hq, Hkv, causal, short_q=0):
    """The run of items of sequence b, in its documented order."""
    G = Hq // Hkv
    hpi = heads_per_item(Hq, Hkv)
    nqt = 0 if Lq <= short_q else (Lq + 127) // 128
    out = []
    for g in range(Hkv):
        for t in range(nqt):
            qt = nqt - 1 - t
            for pr in range(G // hpi):
                out.append((b, qt, g * G + pr * hpi, kv_tiles_visited(qt, Lq, Lkv, causal)))
    return out


def sequence_key(Lq, Lkv, causal, short_q=0):
    nqt = 0 if Lq <= short_q else (Lq + 127) // 128
    return min(SORT_CAP, sum(kv_tiles_visited(qt, Lq, Lkv, causal) for qt in range(nqt)))


def check_sequence_list(items, count, lq, lkv, Hq, Hkv, causal, short_q=0):
    """items: int array [n, 4] as the device wrote them; count: header[0].
    Raises AssertionError on any deviation: a dropped, duplicated or altered
    item, a run out of its internal order, or runs out of key order."""
    items = np.asarray(items, dtype=np.int64).reshape(-1, 4)
    blocks = {b: sequence_block(b, int(lq[b]), int(lkv[b]), Hq, Hkv, causal, short_q) for b in range(len(lq))}
    want = sum(len(v) for v in blocks.values())
    assert count == want, f"item count {count}, expected {want}"
    assert len(items) >= count
    seen = set()
    pos = 0
    prev_key = None
    while pos < count:
        b = int(items[pos, 0])
        assert 0 <= b < len(lq), f"item {pos}: sequence {b} out of range"
        assert b not in seen, f"sequence {b} appears in two runs"
        blk = blocks[b]
        assert len(blk) > 0, f"sequence {b} has no queries but has items"
        got = [tuple(int(x) for x in r) for r in items[pos:pos + len(blk)]]
        assert got == blk, f"run of sequence {b} at {pos} differs from its expected items"
        key = sequence_key(int(lq[b]), int(lkv[b]), causal, short_q)
        assert prev_key is None or key <= prev_key, f"sequence {b} (key {key}) after key {prev_key}"
        prev_key = key
        seen.add(b)
        pos += len(blk)
    missing = [b for b, v in blocks.items() if v and b not in seen]
    assert not missing, f"sequences without their run: {missing}"


def dense_list(B, Sq, Skv, Hq, Hkv, causal):
    """The dense list in its documented order."""
    G = Hq // Hkv
    hpi = heads_per_item(Hq, Hkv)
    nqt = (Sq + 127) // 128
    out = []
    for t0 in range(0, nqt, DENSE_GROUP):
        ts = range(t0, min(nqt, t0 + DENSE_GROUP))
        for b in range(B):
            for g in range(Hkv):
                for t in ts:
                    qt = nqt - 1 - t if causal else t
                    for pr in range(G // hpi):
                        out.append((b, qt, g * G + pr * hpi, kv_tiles_visited(qt, Sq, Skv, causal)))
    return out


def check_dense_list(items, count, B, Sq, Skv, Hq, Hkv, causal):
    want = dense_list(B, Sq, Skv, Hq, Hkv, causal)
    assert count == len(want), f"item count {count}, expected {len(want)}"
    got = [tuple(int(x) for x in r) for r in np.asarray(items, dtype=np.int64).reshape(-1, 4)[:count]]
    assert got == want, "dense list differs from its expected order"


def ragged_max_tiles(B, max_sq, total_q):
    """Query tiles the declared capacities allow (the launch is sized by them)."""
    return min(total_q // 128 + B, B * ((max_sq + 127) // 128))


def decode_order_shift(max_kv_len):
    shift = 0
    while (max_kv_len >> shift) >= 4096:
        shift += 1
    return shift


def check_decode_order(order, kv_lens, max_kv_len):
    """A permutation of the sequences, longest first by bucket min(4095, L >> shift)."""
    order = [int(x) for x in order]
    assert sorted(order) == list(range(len(kv_lens))), "launch order is not a permutation"
    shift = decode_order_shift(max_kv_len)
    keys = [min(4095, max(0, min(int(kv_lens[b]), max_kv_len)) >> shift) for b in order]
    assert all(a >= b for a, b in zip(keys, keys[1:])), "launch order is not longest first"


def page_coords(table, b_idx, t_idx, page_size, num_pages, groups_per_page):
    """(page or -1, row, 8-row group or -1) of logical keys (b, t) by the page-table rule."""
    out = []
    for b, t in zip(b_idx, t_idx):
        page = int(table[int(b), int(t) // page_size])
        row = int(t) % page_size
        if page < 0 or page >= num_pages:
            out.append((-1, row, -1))
        else:
            out.append((page, row, page * groups_per_page + row // 8))
    return np.array(out, dtype=np.int64).reshape(-1, 3)


def decode_units(kv_lens, max_kv_len, cu_q=None, qmax=1):
    """Per sequence (units, L, q0, Lq) by the rule above."""
    out = []
    for b in range(len(kv_lens)):
        L = max(0, min(int(kv_lens[b]), max_kv_len))
        q0, lq, mine = b, 1, True
        if cu_q is not None:
            a0, a1 = int(cu_q[b]), int(cu_q[b + 1])
            q0, lq = a0, a1 - a0
            mine = 1 <= lq <= qmax
        out.append((max(1, -(-L // 64)) if mine else 0, L, q0, lq))
    return out


def decode_sort_shift(max_kv_len):
    shift = 0
    while ((max_kv_len // 64 + 1) >> shift) >= 4096:
        shift += 1
    return shift


def decode_pieces(seq, order, Hkv, S):
    """Expected piece records, one row per block, in the given sequence order."""
    rows = []
    for b in order:
        n, L, q0, lq = seq[b]
        k = min(S, n)
        for g in range(Hkv):
            slot0 = len(rows)
            for s_ in range(k):
                rows.append((b * Hkv + g, s_ * n // k, (s_ + 1) * n // k, slot0, k, L, q0, lq))
    return rows


def check_decode_pieces(order, seg_rows, kv_lens, Hkv, S, max_kv_len, cu_q=None, qmax=1):
    """Device schedule (order [B], one record per block [S * B * Hkv, 8]) against the
    rule: the order is a permutation, longest first by bucket; the records are the ones
    the rule gives for that order, bit for bit; every unit of every pair is in one block."""
    seq = decode_units(kv_lens, max_kv_len, cu_q, qmax)
    order = [int(x) for x in order]
    assert sorted(order) == list(range(len(seq))), "order is not a permutation"
    shift = decode_sort_shift(max_kv_len)
    keys = [min(SORT_CAP, seq[b][0] >> shift) for b in order]
    assert all(a >= c for a, c in zip(keys, keys[1:])), "order is not longest first"
    want = decode_pieces(seq, order, Hkv, S)
    rows = np.asarray(seg_rows, dtype=np.int64).reshape(-1, 8)
    assert len(rows) == S * len(seq) * Hkv, "one record per block of the launch"
    for c, w in enumerate(want):
        assert tuple(int(x) for x in rows[c]) == w, f"block {c}: {tuple(rows[c])} != {w}"
    assert np.all(rows[len(want):, 0] == -1), "blocks past the last piece must be empty"
    covered = set()
    for p_, j0, j1, *_ in want:
        for u in range(j0, j1):
            assert (p_, u) not in covered, "unit in two blocks"
            covered.add((p_, u))
    assert len(covered) == Hkv * sum(s[0] for s in seq), "a unit is in no block"
