"""The measured workloads at full size, in the launch configuration the
bench times (same seeds, same split counts), checked against the fp64 oracle on
sampled rows: the first and last query row of every sequence, rows on both
sides of every 128-row tile boundary of a few sequences, and random rows."""
import numpy as np
import pytest
import torch

import ragged_scaled_dot_b200 as rsd
import synth
from gpu_util import assert_lse_close, assert_o_close, bits, orc, pool_strides_np

pytestmark = [pytest.mark.gpu, pytest.mark.slow]
DEV = "cuda"


def test_dense_prefill_full_size():
    w = synth.WORKLOADS["dense_prefill"]
    q, k, v = synth.make_dense(w, DEV)
    o = torch.full_like(q, float("nan"))
    lse = torch.full((w.B, w.Hq, w.S), float("nan"), dtype=torch.float32, device=DEV)
    ws = torch.full((rsd.attn_fwd_dense_workspace_size(w.B, w.S, w.Hq, w.Hkv),), 0xFF, dtype=torch.uint8,
                    device=DEV)
    rsd.attn_fwd_dense(q, k, v, o, lse, scale=w.scale, causal=True, workspace=ws)
    torch.cuda.synchronize()
    assert not torch.isnan(o).any() and not torch.isnan(lse).any()
    rng = np.random.default_rng(0)
    rows = [(b, int(rng.integers(w.Hq)), i) for b in range(w.B) for i in (0, 127, 128, w.S - 1)]
    rows += [(int(rng.integers(w.B)), int(rng.integers(w.Hq)), int(rng.integers(w.S))) for _ in range(512)]
    rows = np.array(rows, dtype=np.int32)
    o_ref, l_ref = orc().attn_dense_rows(bits(q), bits(k), bits(v), w.S, w.S, w.Hq, w.Hkv, w.Dqk, w.Dv,
                                         w.scale, True, rows)
    r = torch.as_tensor(rows.astype(np.int64), device=DEV)
    assert_o_close(o[r[:, 0], r[:, 2], r[:, 1]], o_ref, "dense full")
    assert_lse_close(lse[r[:, 0], r[:, 1], r[:, 2]], l_ref, "dense full")


def test_ragged_prefill_full_size():
    w = synth.WORKLOADS["ragged_prefill"]
    L = w.seq_lengths()
    q, k, v, cu = synth.make_ragged(w, DEV, lengths=L)
    T, smax = q.shape[0], int(L.max())
    o = torch.full_like(q, float("nan"))
    lse = torch.full((w.B, smax, w.Hq), float("nan"), dtype=torch.float32, device=DEV)
    ws = torch.empty(rsd.attn_fwd_ragged_workspace_size(w.B, smax, T, w.Hq, w.Hkv), dtype=torch.uint8,
                     device=DEV)
    cud = torch.as_tensor(cu, device=DEV)
    rsd.attn_fwd_ragged(q, k, v, o, lse, cud, cud, max_seqlen_q=smax, max_seqlen_kv=smax, scale=w.scale,
                        causal=True, workspace=ws)
    torch.cuda.synchronize()
    assert rsd.attn_get_device_error() == rsd.ATTN_OK
    assert not torch.isnan(o).any(), "every output row must be written"
    for b in range(w.B):  # padded LSE: -inf past each length, finite inside
        assert torch.all(lse[b, int(L[b]):] == -float("inf"))
        assert torch.isfinite(lse[b, :int(L[b])]).all()
    rng = np.random.default_rng(1)
    rows = [(b, int(rng.integers(w.Hq)), i) for b in range(w.B) for i in (0, int(L[b]) - 1)]
    for b in range(0, w.B, 8):
        for t in range(128, int(L[b]), 128):
            rows += [(b, int(rng.integers(w.Hq)), t - 1), (b, int(rng.integers(w.Hq)), t)]
    for _ in range(512):
        b = int(rng.integers(w.B))
        rows.append((b, int(rng.integers(w.Hq)), int(rng.integers(L[b]))))
    rows = np.array(rows, dtype=np.int32)
    o_ref, l_ref = orc().attn_ragged_rows(bits(q), bits(k), bits(v), cu, cu, w.Hq, w.Hkv, w.scale, True,
                                          rows)
    tok = torch.as_tensor(cu[rows[:, 0]].astype(np.int64) + rows[:, 2], device=DEV)
    h = torch.as_tensor(rows[:, 1].astype(np.int64), device=DEV)
    assert_o_close(o[tok, h], o_ref, "ragged full")
    assert_lse_close(lse[torch.as_tensor(rows[:, 0].astype(np.int64), device=DEV),
                         torch.as_tensor(rows[:, 2].astype(np.int64), device=DEV), h], l_ref, "ragged full")


@pytest.mark.parametrize("name", ["paged_decode", "mla_decode", "decode_small_batch"])
def test_paged_decode_full_size(name):
    w = synth.WORKLOADS[name]
    L = w.seq_lengths()
    q, kp, vp, table, kl = synth.make_paged(w, DEV, kv_lens=L)
    maxL = int(L.max())
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    S = rsd.attn_paged_suggest_splits(w.B, w.Hq, w.Hkv, w.Dqk, w.Dv, maxL, w.page_size, sms)
    o = torch.full((w.B, w.Hq, w.Dv), float("nan"), dtype=torch.bfloat16, device=DEV)
    lse = torch.full((w.B, w.Hq), float("nan"), dtype=torch.float32, device=DEV)
    n = rsd.attn_fwd_paged_workspace_size(w.B, w.Hq, w.Dv, S)
    ws = torch.empty(max(n, 1), dtype=torch.uint8, device=DEV)
    rsd.attn_fwd_paged(q, kp, vp, o, lse, torch.as_tensor(table, device=DEV), torch.as_tensor(kl, device=DEV),
                       page_size=w.page_size, max_kv_len=maxL, scale=w.scale, num_splits=S, workspace=ws)
    torch.cuda.synchronize()
    assert rsd.attn_get_device_error() == rsd.ATTN_OK
    assert not torch.isnan(o).any()
    rng = np.random.default_rng(2)
    if name in ("paged_decode", "decode_small_batch"):
        bs = rng.choice(w.B, 24, replace=False)
        rows = np.array([(b, h) for b in bs for h in range(w.Hq)], dtype=np.int32)
    else:
        rows = np.array([(int(rng.integers(w.B)), int(rng.integers(w.Hq))) for _ in range(192)],
                        dtype=np.int32)
    kb = bits(kp)
    vb = kb if w.v_aliases_k else bits(vp)
    o_ref, l_ref = orc().attn_paged_rows(bits(q), kb, vb, table, kl, w.page_size, w.Hq, w.Hkv, w.Dqk, w.Dv,
                                         pool_strides_np(kp, "HND"), pool_strides_np(vp, "HND"), w.scale, rows)
    r = torch.as_tensor(rows.astype(np.int64), device=DEV)
    assert_o_close(o[r[:, 0], r[:, 1]], o_ref, f"{name} full (splits {S})")
    assert_lse_close(lse[r[:, 0], r[:, 1]], l_ref, f"{name} full (splits {S})")


def test_paged_prefill_full_size():
    """Chunked prefill at full size: 16 x 1024 queries over paged caches of up to
    64k keys, vs the oracle over each sampled sequence's keys gathered from the pool."""
    w = synth.WORKLOADS["paged_prefill"]
    q, kp, vp, table, kl, cu_q, lq = synth.make_paged_prefill(w, DEV)
    T, smax = q.shape[0], int(lq.max())
    o = torch.full_like(q, float("nan"))
    lse = torch.full((w.B, smax, w.Hq), float("nan"), dtype=torch.float32, device=DEV)
    ws = torch.empty(rsd.attn_fwd_paged_prefill_workspace_size(w.B, smax, T, w.Hq, w.Hkv, w.Dqk, 1), dtype=torch.uint8,
                     device=DEV)
    rsd.attn_fwd_paged_prefill(q, kp, vp, o, lse, torch.as_tensor(cu_q, device=DEV),
                               torch.as_tensor(table, device=DEV), torch.as_tensor(kl, device=DEV),
                               max_seqlen_q=smax, page_size=w.page_size, max_kv_len=int(kl.max()),
                               scale=w.scale, causal=True, workspace=ws)
    torch.cuda.synchronize()
    assert rsd.attn_get_device_error() == rsd.ATTN_OK
    assert not torch.isnan(o).any()
    rng = np.random.default_rng(2)
    # every sequence: first and last query row, rows on both sides of each 128-row query tile
    # boundary and of each page boundary of the query chunk (query i sits at cache position
    # L - n + i), plus 512 random rows spread over the sequences
    extra = {b: [] for b in range(w.B)}
    for _ in range(512):
        b = int(rng.integers(w.B))
        extra[b].append(int(rng.integers(int(lq[b]))))
    n_checked = 0
    for b in range(w.B):
        L, n = int(kl[b]), int(lq[b])
        idx = {0, n - 1}
        for t in range(128, n, 128):
            idx |= {t - 1, t}
        first_pos = L - n
        for pos in range((first_pos // w.page_size + 1) * w.page_size, L, w.page_size):
            idx |= {pos - 1 - first_pos, pos - first_pos}
        idx = sorted(i for i in idx | set(extra[b]) if 0 <= i < n)
        j = np.arange(L)
        pages = torch.as_tensor(table[b, j // w.page_size].astype(np.int64), device=DEV)
        slots = torch.as_tensor(j % w.page_size, device=DEV)
        kc, vc = kp[pages, :, slots].contiguous(), vp[pages, :, slots].contiguous()
        rows = np.array([(0, int(rng.integers(w.Hq)), i) for i in idx], dtype=np.int32)
        q_b = q[int(cu_q[b]):int(cu_q[b + 1])]
        o_ref, l_ref = orc().attn_ragged_rows(bits(q_b), bits(kc), bits(vc), np.array([0, n]),
                                              np.array([0, L]), w.Hq, w.Hkv, w.scale, True, rows)
        tok = torch.as_tensor(rows[:, 2].astype(np.int64) + int(cu_q[b]), device=DEV)
        hh = torch.as_tensor(rows[:, 1].astype(np.int64), device=DEV)
        assert_o_close(o[tok, hh], o_ref, f"paged prefill full b={b}")
        assert_lse_close(lse[b, tok - int(cu_q[b]), hh], l_ref, f"paged prefill full b={b}")
        n_checked += len(rows)
    assert n_checked >= 512 + 16 * 2


def test_mixed_batch_full_size():
    """The mixed batch at full size, in the bench's launch configuration (its
    suggested split count for the short rows, token-major LSE): every row of the
    48 short sequences for every head, and on the 16 chunk sequences the first
    and last rows, both sides of each 128-row tile boundary and of each page
    boundary, plus 512 random rows, against the oracle over each sequence's keys
    gathered from the pool."""
    w = synth.WORKLOADS["mixed_batch"]
    q, kp, vp, table, kl, cu_q, lq = synth.make_mixed_batch(w, DEV)
    T, smax = int(cu_q[-1]), int(lq.max())
    L = kl.astype(np.int64)
    n_short = int(np.sum((lq >= 1) & (lq <= 4)))
    num_sms = torch.cuda.get_device_properties(0).multi_processor_count
    S = rsd.attn_paged_suggest_splits(max(1, n_short), w.Hq, w.Hkv, w.Dqk, w.Dv, int(L.max()), w.page_size, num_sms)
    o = torch.full_like(q, float("nan"))
    lse = torch.full((T, w.Hq), float("nan"), dtype=torch.float32, device=DEV)
    ws = torch.full((rsd.attn_fwd_paged_prefill_workspace_size(w.B, smax, T, w.Hq, w.Hkv, w.Dqk, S),), 0xFF,
                    dtype=torch.uint8, device=DEV)
    rsd.attn_fwd_paged_prefill(q, kp, vp, o, lse, torch.as_tensor(cu_q, device=DEV),
                               torch.as_tensor(table, device=DEV), torch.as_tensor(kl, device=DEV),
                               max_seqlen_q=smax, page_size=w.page_size, max_kv_len=int(L.max()),
                               scale=w.scale, causal=True, workspace=ws, num_splits=S,
                               lse_layout=rsd.ATTN_LSE_PACKED_TH)
    torch.cuda.synchronize()
    assert rsd.attn_get_device_error() == rsd.ATTN_OK
    assert not torch.isnan(o).any() and not torch.isnan(lse).any()
    rng = np.random.default_rng(5)
    extra = {b: [] for b in range(w.B)}
    chunks = [b for b in range(w.B) if lq[b] > 4]
    for _ in range(512):
        b = chunks[int(rng.integers(len(chunks)))]
        extra[b].append(int(rng.integers(int(lq[b]))))
    n_checked = 0
    for b in range(w.B):
        Lb, n = int(L[b]), int(lq[b])
        if n == 0:
            continue
        if n <= 4:
            rows = np.array([(0, h, i) for i in range(n) for h in range(w.Hq)], dtype=np.int32)
        else:
            idx = {0, n - 1}
            for t in range(128, n, 128):
                idx |= {t - 1, t}
            first_pos = Lb - n
            for pos in range((first_pos // w.page_size + 1) * w.page_size, Lb, w.page_size):
                idx |= {pos - 1 - first_pos, pos - first_pos}
            idx = sorted(i for i in idx | set(extra[b]) if 0 <= i < n)
            rows = np.array([(0, int(rng.integers(w.Hq)), i) for i in idx], dtype=np.int32)
        j = np.arange(Lb)
        pages = torch.as_tensor(table[b, j // w.page_size].astype(np.int64), device=DEV)
        slots = torch.as_tensor(j % w.page_size, device=DEV)
        kc, vc = kp[pages, :, slots].contiguous(), vp[pages, :, slots].contiguous()
        q_b = q[int(cu_q[b]):int(cu_q[b + 1])]
        o_ref, l_ref = orc().attn_ragged_rows(bits(q_b), bits(kc), bits(vc), np.array([0, n]),
                                              np.array([0, Lb]), w.Hq, w.Hkv, w.scale, True, rows)
        tok = torch.as_tensor(rows[:, 2].astype(np.int64) + int(cu_q[b]), device=DEV)
        hh = torch.as_tensor(rows[:, 1].astype(np.int64), device=DEV)
        assert_o_close(o[tok, hh], o_ref, f"mixed batch full b={b}")
        assert_lse_close(lse[tok, hh], l_ref, f"mixed batch full b={b}")
        n_checked += len(rows)
    assert n_checked >= 512 + 48 * w.Hq
