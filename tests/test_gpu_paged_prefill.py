"""Ragged queries over a paged K/V cache (chunked prefill, multi-token decode)
on the GPU vs the fp64 oracle.  The oracle sees the same keys gathered out of
the pool into contiguous per-sequence K/V by this test (numpy indexing), and
the ragged oracle's bottom-right causal rule.  Also: bit-identical to the
ragged kernel over that gathered K/V, NaN in the unused slots of a last page,
empty caches and queries without keys."""
import numpy as np
import pytest
import torch

import ragged_scaled_dot_b200 as rsd
import synth
from gpu_util import (LOG2E, LSE_ATOL, assert_lse_close, assert_o_close, bits, gather_ragged, lse_alloc, orc,
                      ragged_gpu, ragged_rows_all)

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _inputs(lens_q, lens_kv, Hq, Hkv, D, ps, seed, layout="HND"):
    table, total = synth.page_table(lens_kv, ps, seed)
    P = total + 2
    cu_q = np.concatenate([[0], np.cumsum(lens_q)]).astype(np.int32)
    q = synth.normal_bf16((int(cu_q[-1]), Hq, D), seed + 1, "cpu").to(DEV)
    shape = (P, Hkv, ps, D) if layout == "HND" else (P, ps, Hkv, D)
    k = synth.normal_bf16(shape, seed + 2, "cpu").to(DEV)
    v = synth.normal_bf16(shape, seed + 3, "cpu").to(DEV)
    return q, k, v, table, np.asarray(lens_kv, dtype=np.int32), cu_q


def _gather(pool, table, lens_kv, ps, layout):
    """Contiguous THD [sum kv, Hkv, D] copy of each sequence's keys, by page table."""
    parts = []
    for b, L in enumerate(lens_kv):
        j = np.arange(int(L))
        pages = torch.as_tensor(table[b, j // ps].astype(np.int64), device=pool.device)
        slots = torch.as_tensor(j % ps, device=pool.device)
        parts.append(pool[pages, :, slots] if layout == "HND" else pool[pages, slots])
    Hkv, D = (pool.shape[1], pool.shape[3]) if layout == "HND" else (pool.shape[2], pool.shape[3])
    if not parts:
        return torch.zeros((0, Hkv, D), dtype=pool.dtype, device=pool.device)
    return torch.cat(parts, 0).contiguous()


def _run(q, k, v, table, kl, cu_q, ps, scale, causal, layout="HND", lse_layout=rsd.ATTN_LSE_PADDED_BSH,
         num_splits=1):
    B = len(cu_q) - 1
    max_sq = max(1, int(np.max(np.diff(cu_q))))
    Hq, D = q.shape[1], q.shape[2]
    o = torch.full((q.shape[0], Hq, v.shape[-1]), float("nan"), dtype=torch.bfloat16, device=DEV)
    lse = lse_alloc(lse_layout, B, max_sq, q.shape[0], Hq, float("nan"), DEV)
    Hkv = k.shape[1] if layout == "HND" else k.shape[2]
    ws = torch.full((rsd.attn_fwd_paged_prefill_workspace_size(B, max_sq, q.shape[0], Hq, Hkv, D, num_splits),),
                    0xFF, dtype=torch.uint8, device=DEV)  # stale partials must be overwritten
    rsd.attn_fwd_paged_prefill(
        q, k, v, o, lse, torch.as_tensor(cu_q, device=DEV), torch.as_tensor(table, device=DEV),
        torch.as_tensor(kl, device=DEV), max_seqlen_q=max_sq, page_size=ps,
        max_kv_len=max(1, int(np.max(kl))), scale=scale, causal=causal, workspace=ws,
        lse_layout=lse_layout, kv_layout=layout, num_splits=num_splits)
    torch.cuda.synchronize()
    assert rsd.attn_get_device_error() == rsd.ATTN_OK
    return o, lse


CASES = [
    # (lens_q, lens_kv, Hq, Hkv, D, ps, layout, causal)
    ([1, 2, 4, 100, 129], [1000, 64, 300, 100, 2000], 16, 4, 128, 64, "HND", True),   # MTP + chunks
    ([37, 256, 5], [300, 700, 77], 8, 1, 64, 16, "NHD", False),
    ([512, 300], [4096, 1024], 8, 2, 128, 128, "HND", True),                          # chunked prefill
    ([9, 130], [40, 333], 4, 4, 128, 8, "NHD", True),                                   # 8-row pages
    ([64, 200], [1500, 999], 16, 2, 64, 256, "HND", True),                              # 128-row boxes
    ([100, 3], [40, 0], 4, 1, 128, 32, "HND", True),                                    # Lq > Lkv, empty cache
]


@pytest.mark.parametrize("lens_q,lens_kv,Hq,Hkv,D,ps,layout,causal", CASES)
def test_paged_prefill_vs_oracle(lens_q, lens_kv, Hq, Hkv, D, ps, layout, causal):
    q, k, v, table, kl, cu_q = _inputs(lens_q, lens_kv, Hq, Hkv, D, ps, seed=ps + Hq + len(lens_q), layout=layout)
    scale = 1.0 / np.sqrt(D)
    o, lse = _run(q, k, v, table, kl, cu_q, ps, scale, causal, layout)
    kc, vc = _gather(k, table, kl, ps, layout), _gather(v, table, kl, ps, layout)
    cu_kv = np.concatenate([[0], np.cumsum(kl)]).astype(np.int32)
    rows = ragged_rows_all(cu_q, Hq)
    o_ref, l_ref = orc().attn_ragged_rows(bits(q), bits(kc), bits(vc), cu_q, cu_kv, Hq, Hkv, scale, causal, rows)
    og, lg = gather_ragged(o, lse, cu_q, rows, rsd.ATTN_LSE_PADDED_BSH)
    where = f"paged prefill {lens_q}/{lens_kv} ps{ps} {layout} causal={causal}"
    assert_o_close(og, o_ref, where)
    assert_lse_close(lg, l_ref, where)


def test_paged_prefill_matches_ragged_over_gathered_kv_bitwise():
    """The sequences on prefill tiles give exactly what the ragged kernel gives
    over their gathered K/V (the 1-query sequence takes the decode kernel and is
    checked against the oracle elsewhere)."""
    lens_q, lens_kv, ps = [128, 300, 1], [1024, 300, 777], 64
    q, k, v, table, kl, cu_q = _inputs(lens_q, lens_kv, 16, 4, 128, ps, seed=5)
    o1, l1 = _run(q, k, v, table, kl, cu_q, ps, 0.09, True, lse_layout=rsd.ATTN_LSE_PACKED_TH)
    kc, vc = _gather(k, table, kl, ps, "HND"), _gather(v, table, kl, ps, "HND")
    cu_kv = np.concatenate([[0], np.cumsum(kl)]).astype(np.int32)
    o2, l2 = ragged_gpu(q, kc, vc, cu_q, cu_kv, int(max(lens_q)), int(max(lens_kv)), 0.09, True,
                        lse_layout=rsd.ATTN_LSE_PACKED_TH)
    long_tok = int(cu_q[2])  # tokens of the two prefill sequences
    assert torch.equal(o1[:long_tok], o2[:long_tok]) and torch.equal(l1[:long_tok], l2[:long_tok])


@pytest.mark.parametrize("ps", [16, 64])
def test_paged_prefill_nan_past_kv_len_is_never_used(ps):
    lens_q, lens_kv = [50, 7], [170, 90]
    q, k, v, table, kl, cu_q = _inputs(lens_q, lens_kv, 8, 2, 128, ps, seed=11)
    kn, vn = k.clone(), v.clone()
    for b, L in enumerate(lens_kv):
        last = table[b, (L - 1) // ps]
        kn[last, :, L % ps:] = float("nan")
        vn[last, :, L % ps:] = float("nan")
    o1, l1 = _run(q, k, v, table, kl, cu_q, ps, 0.1, True)
    o2, l2 = _run(q, kn, vn, table, kl, cu_q, ps, 0.1, True)
    assert torch.isfinite(o2.float()).all()
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


def test_paged_prefill_head_major_base2_lse():
    """Head-major [Hq, total_q] LSE in base 2 (stats_use_log2) over a paged
    cache: the oracle's natural LSE times log2(e)."""
    lens_q, lens_kv, ps = [3, 130, 1], [700, 130, 64], 64
    q, k, v, table, kl, cu_q = _inputs(lens_q, lens_kv, 8, 2, 128, ps, seed=21)
    lay = rsd.ATTN_LSE_PACKED_HT | rsd.ATTN_LSE_LOG2
    o, lse = _run(q, k, v, table, kl, cu_q, ps, 0.09, True, lse_layout=lay)
    kc, vc = _gather(k, table, kl, ps, "HND"), _gather(v, table, kl, ps, "HND")
    cu_kv = np.concatenate([[0], np.cumsum(kl)]).astype(np.int32)
    rows = ragged_rows_all(cu_q, 8)
    o_ref, l_ref = orc().attn_ragged_rows(bits(q), bits(kc), bits(vc), cu_q, cu_kv, 8, 2, 0.09, True, rows)
    og, lg = gather_ragged(o, lse, cu_q, rows, lay)
    assert_o_close(og, o_ref, "paged prefill, head-major base-2 LSE")
    assert_lse_close(lg, l_ref * LOG2E, "paged prefill, head-major base-2 LSE", atol=LSE_ATOL * LOG2E)


@pytest.mark.parametrize("ps", [64, 16])
def test_paged_prefill_independent_kv_tables(ps):
    """Chunked prefill with V in its own pool and page table: the oracle's
    result, and bit-identical to one shared table over the original pool.
    Page 16 puts 8 page boxes in each K or V tile (one producer lane each, V
    lanes reading V's table)."""
    lens_q, lens_kv = [3, 130, 64], [700, 130, 300]
    q, k, v, table, kl, cu_q = _inputs(lens_q, lens_kv, 8, 2, 128, ps, seed=71 + ps)
    n_pages = [(L + ps - 1) // ps for L in lens_kv]
    table_v, total = synth.page_table(lens_kv, ps, 73 + ps)
    v2 = torch.full((total + 4,) + tuple(v.shape[1:]), float("nan"), dtype=v.dtype, device=DEV)
    src = np.concatenate([table[b, :n] for b, n in enumerate(n_pages)]).astype(np.int64)
    dst = np.concatenate([table_v[b, :n] for b, n in enumerate(n_pages)]).astype(np.int64)
    v2[torch.as_tensor(dst, device=DEV)] = v[torch.as_tensor(src, device=DEV)]
    B, Hq = len(lens_q), 8
    o = torch.full((q.shape[0], Hq, 128), float("nan"), dtype=torch.bfloat16, device=DEV)
    lse = lse_alloc(rsd.ATTN_LSE_PACKED_TH, B, max(lens_q), q.shape[0], Hq, float("nan"), DEV)
    ws = torch.empty(rsd.attn_fwd_paged_prefill_workspace_size(B, max(lens_q), q.shape[0], Hq, 2),
                     dtype=torch.uint8, device=DEV)
    rsd.attn_fwd_paged_prefill_kv_tables(
        q, k, v2, o, lse, torch.as_tensor(cu_q, device=DEV), torch.as_tensor(table, device=DEV),
        torch.as_tensor(table_v, device=DEV), torch.as_tensor(kl, device=DEV), max_seqlen_q=max(lens_q),
        page_size=ps, max_kv_len=max(lens_kv), scale=0.09, causal=True, workspace=ws,
        lse_layout=rsd.ATTN_LSE_PACKED_TH)
    torch.cuda.synchronize()
    assert rsd.attn_get_device_error() == rsd.ATTN_OK
    o1, l1 = _run(q, k, v, table, kl, cu_q, ps, 0.09, True, lse_layout=rsd.ATTN_LSE_PACKED_TH)
    assert torch.equal(o, o1) and torch.equal(lse, l1)
    kc, vc = _gather(k, table, kl, ps, "HND"), _gather(v, table, kl, ps, "HND")
    cu_kv = np.concatenate([[0], np.cumsum(kl)]).astype(np.int32)
    rows = ragged_rows_all(cu_q, Hq)
    o_ref, l_ref = orc().attn_ragged_rows(bits(q), bits(kc), bits(vc), cu_q, cu_kv, Hq, 2, 0.09, True, rows)
    og, lg = gather_ragged(o, lse, cu_q, rows, rsd.ATTN_LSE_PACKED_TH)
    assert_o_close(og, o_ref, "paged prefill, independent tables")
    assert_lse_close(lg, l_ref, "paged prefill, independent tables")


# --------------------------------------------------------------------------------------------
# Mixed batches: sequences of at most qmax = min(4, 64 / G) queries run on the split-KV decode
# kernel (G heads x Lq tokens as the tile rows), the others on prefill tiles, in one call.
MIXED = [
    # (lens_q, lens_kv, Hq, Hkv, D, ps, splits, causal, lse_layout)
    ([1, 2, 4, 1000, 3], [32768, 20000, 32000, 32768, 5], 8, 2, 128, 64, 1, True, rsd.ATTN_LSE_PADDED_BSH),
    ([1, 2, 4, 1000, 3], [32768, 20000, 32000, 32768, 5], 8, 2, 128, 64, 4, True,
     rsd.ATTN_LSE_PACKED_TH | rsd.ATTN_LSE_LOG2),
    ([1, 2, 4, 500], [9000, 4100, 7000, 3000], 16, 2, 128, 64, 3, True, rsd.ATTN_LSE_PACKED_HT),    # 32 rows
    ([1, 4, 3, 200], [3000, 5000, 2, 1000], 32, 2, 64, 16, 2, True, rsd.ATTN_LSE_PADDED_BSH),      # 64 rows
    ([1, 2, 2, 300], [4000, 1000, 64, 2000], 32, 1, 128, 32, 5, True, rsd.ATTN_LSE_PACKED_TH),     # G 32
    ([1, 3, 4, 130], [1000, 999, 4097, 130], 6, 2, 64, 128, 2, False, rsd.ATTN_LSE_PADDED_BSH),    # G 3
    ([1] * 8 + [4] * 8, [100 * i + 1 for i in range(16)], 8, 2, 128, 64, 3, True, rsd.ATTN_LSE_PACKED_TH),
    # short rows over an empty cache and a 1-key cache (the first query of the 2 sees no key)
    ([1, 2, 300, 4], [0, 1, 500, 70], 8, 2, 128, 64, 2, True, rsd.ATTN_LSE_PADDED_BSH),
    # 64-row (4-query, G 16) pieces of a 60000-key cache merged over two levels of groups of 8
    ([4, 2, 700], [60000, 30000, 2000], 32, 2, 64, 16, 64, True, rsd.ATTN_LSE_PACKED_TH),
]


@pytest.mark.parametrize("lens_q,lens_kv,Hq,Hkv,D,ps,splits,causal,lse_layout", MIXED)
def test_mixed_batch_every_row_vs_oracle(lens_q, lens_kv, Hq, Hkv, D, ps, splits, causal, lse_layout):
    q, k, v, table, kl, cu_q = _inputs(lens_q, lens_kv, Hq, Hkv, D, ps, seed=Hq + splits + len(lens_q))
    scale = 1.0 / np.sqrt(D)
    o, lse = _run(q, k, v, table, kl, cu_q, ps, scale, causal, lse_layout=lse_layout, num_splits=splits)
    kc, vc = _gather(k, table, kl, ps, "HND"), _gather(v, table, kl, ps, "HND")
    cu_kv = np.concatenate([[0], np.cumsum(kl)]).astype(np.int32)
    rows = ragged_rows_all(cu_q, Hq)
    o_ref, l_ref = orc().attn_ragged_rows(bits(q), bits(kc), bits(vc), cu_q, cu_kv, Hq, Hkv, scale, causal, rows)
    og, lg = gather_ragged(o, lse, cu_q, rows, lse_layout)
    where = f"mixed batch {lens_q} G={Hq // Hkv} splits={splits}"
    assert_o_close(og, o_ref, where)
    if lse_layout & rsd.ATTN_LSE_LOG2:
        assert_lse_close(lg, l_ref * LOG2E, where, atol=LSE_ATOL * LOG2E)
    else:
        assert_lse_close(lg, l_ref, where)
    if (lse_layout & ~rsd.ATTN_LSE_LOG2) == rsd.ATTN_LSE_PADDED_BSH:
        for b, n in enumerate(lens_q):  # padded rows past each length stay -inf
            assert torch.all(lse[b, n:] == -float("inf"))


@pytest.mark.parametrize("splits", [1, 3])
def test_single_query_rows_equal_paged_decode_bitwise(splits):
    """A 1-query sequence in a mixed batch (G = 4: one m16 tile) is computed
    exactly as attn_fwd_paged computes a decode row with the same splits."""
    lens_q, lens_kv, ps, Hq, Hkv, D = [1, 1, 1, 700], [5000, 64, 1, 3000], 64, 8, 2, 128
    q, k, v, table, kl, cu_q = _inputs(lens_q, lens_kv, Hq, Hkv, D, ps, seed=31)
    o, lse = _run(q, k, v, table, kl, cu_q, ps, 0.088, True, lse_layout=rsd.ATTN_LSE_PACKED_TH,
                  num_splits=splits)
    n = 3
    qd = q[:n].contiguous()
    od = torch.full((n, Hq, D), float("nan"), dtype=torch.bfloat16, device=DEV)
    ld = torch.full((n, Hq), float("nan"), dtype=torch.float32, device=DEV)
    wsn = rsd.attn_fwd_paged_workspace_size(n, Hq, D, splits)
    ws = torch.empty(max(wsn, 1), dtype=torch.uint8, device=DEV) if wsn else None
    rsd.attn_fwd_paged(qd, k, v, od, ld, torch.as_tensor(table[:n], device=DEV), torch.as_tensor(kl[:n], device=DEV),
                       page_size=ps, max_kv_len=int(max(lens_kv)), scale=0.088, num_splits=splits, workspace=ws)
    torch.cuda.synchronize()
    assert rsd.attn_get_device_error() == rsd.ATTN_OK
    assert torch.equal(o[:n], od) and torch.equal(lse[:n], ld)


def test_mixed_batch_nan_past_kv_len_in_short_rows():
    """NaN in the unused slots of the last page of short (decode-kernel) sequences never reaches O."""
    lens_q, lens_kv, ps = [1, 3, 200], [170, 90, 333], 64
    q, k, v, table, kl, cu_q = _inputs(lens_q, lens_kv, 8, 2, 128, ps, seed=41)
    kn, vn = k.clone(), v.clone()
    for b, L in enumerate(lens_kv):
        last = table[b, (L - 1) // ps]
        kn[last, :, L % ps:] = float("nan")
        vn[last, :, L % ps:] = float("nan")
    for splits in (1, 2):
        o1, l1 = _run(q, k, v, table, kl, cu_q, ps, 0.1, True, num_splits=splits)
        o2, l2 = _run(q, kn, vn, table, kl, cu_q, ps, 0.1, True, num_splits=splits)
        assert torch.isfinite(o2.float()).all()
        assert torch.equal(o1, o2) and torch.equal(l1, l2)
