"""GPU pins that need no tolerance against the oracle.

* Guard bands: every output (O and LSE) is written through a view inside a
  larger buffer filled with a canary pattern (rows before and after, and a gap
  at the end of each row); after the call the canaries are intact and the
  values inside the view equal those of a run on plain buffers, bit for bit.
* Single visible key: softmax weight 1 exactly, so the output row is that
  key's value row, bit for bit (any bf16 value survives the fp32 round trip).
* Uniform scores (scale = 0): every visible key has weight 1, the row sum is
  the count of visible keys (exact in fp32), so round(exp(LSE)) equals that
  count exactly.  This pins the causal mask, the ragged tails and the split
  ranges row by row on the GPU.
"""
import numpy as np
import pytest
import torch

import ragged_scaled_dot_b200 as rsd
import synth
from gpu_util import assert_o_close

pytestmark = pytest.mark.gpu
DEV = "cuda"
CANARY_BF16 = 0x7BAD          # a finite bf16 (about 1.8e36)
CANARY_F32 = 0x7BAD7BAD       # a finite fp32
PAD_ROWS, PAD_COLS = 3, 16


def guarded_bf16(shape):
    """(view, big, mask): a bf16 view of `shape` inside `big`, which has PAD_ROWS
    extra leading rows on each side and PAD_COLS extra last-dim elements."""
    bshape = (shape[0] + 2 * PAD_ROWS,) + tuple(shape[1:-1]) + (shape[-1] + PAD_COLS,)
    big = torch.full(bshape, CANARY_BF16, dtype=torch.int16, device=DEV).view(torch.bfloat16)
    idx = (slice(PAD_ROWS, PAD_ROWS + shape[0]),) + (slice(None),) * (len(shape) - 2) + (slice(0, shape[-1]),)
    mask = torch.zeros(bshape, dtype=torch.bool, device=DEV)
    mask[idx] = True
    return big[idx], big, mask


def guarded_f32(shape):
    """(view, big, mask): a contiguous fp32 view of `shape` inside a flat buffer
    with PAD_ROWS * 64 canary elements on each side."""
    n = int(np.prod(shape))
    pad = PAD_ROWS * 64
    big = torch.full((n + 2 * pad,), CANARY_F32, dtype=torch.int32, device=DEV).view(torch.float32)
    mask = torch.zeros(n + 2 * pad, dtype=torch.bool, device=DEV)
    mask[pad:pad + n] = True
    return big[pad:pad + n].view(shape), big, mask


def assert_canaries(big, mask, where):
    raw = big.view(torch.int16) if big.dtype == torch.bfloat16 else big.view(torch.int32)
    want = CANARY_BF16 if big.dtype == torch.bfloat16 else CANARY_F32
    outside = raw[~mask]
    bad = int((outside != want).sum())
    assert bad == 0, f"{where}: {bad} guard elements overwritten"


def same_bits(a, b, where):
    assert torch.equal(a.view(torch.int16) if a.dtype == torch.bfloat16 else a.view(torch.int32),
                       b.view(torch.int16) if b.dtype == torch.bfloat16 else b.view(torch.int32)), where


def _ragged(lq, lkv, Hq, Hkv, D, seed):
    cu_q, cu_kv = synth.cu_seqlens(lq), synth.cu_seqlens(lkv)
    q = synth.normal_bf16((int(cu_q[-1]), Hq, D), seed, "cpu").to(DEV)
    k = synth.normal_bf16((int(cu_kv[-1]), Hkv, D), seed + 1, "cpu").to(DEV)
    v = synth.normal_bf16((int(cu_kv[-1]), Hkv, D), seed + 2, "cpu").to(DEV)
    return q, k, v, cu_q, cu_kv


def _run_ragged(q, k, v, cu_q, cu_kv, scale, causal, o, lse, lse_layout):
    B = len(cu_q) - 1
    smax = int(np.max(np.diff(cu_q)))
    kmax = int(np.max(np.diff(cu_kv)))
    ws = torch.empty(rsd.attn_fwd_ragged_workspace_size(B, smax, q.shape[0], q.shape[1], k.shape[1]),
                     dtype=torch.uint8, device=DEV)
    rsd.attn_fwd_ragged(q, k, v, o, lse, torch.as_tensor(cu_q, device=DEV), torch.as_tensor(cu_kv, device=DEV),
                        max_seqlen_q=smax, max_seqlen_kv=kmax, scale=scale, causal=causal, workspace=ws,
                        lse_layout=lse_layout)
    torch.cuda.synchronize()


def _ragged_lse_shape(layout, B, smax, T, Hq):
    return {rsd.ATTN_LSE_PADDED_BSH: (B, smax, Hq), rsd.ATTN_LSE_PACKED_TH: (T, Hq),
            rsd.ATTN_LSE_PACKED_HT: (Hq, T)}[layout]


def _paged(lens, Hq, Hkv, D, ps, seed, Dv=None, alias=False):
    table, total = synth.page_table(lens, ps, seed)
    q = synth.normal_bf16((len(lens), Hq, D), seed + 1, "cpu").to(DEV)
    k = synth.normal_bf16((total + 2, Hkv, ps, D), seed + 2, "cpu").to(DEV)
    v = k if alias else synth.normal_bf16((total + 2, Hkv, ps, Dv or D), seed + 3, "cpu").to(DEV)
    return q, k, v, table


def _run_paged(q, k, v, table, lens, ps, scale, splits, o, lse):
    B, Hq, _ = q.shape
    Dv = o.shape[-1]
    n = rsd.attn_fwd_paged_workspace_size(B, Hq, Dv, splits)
    ws = torch.full((max(n, 1),), 0xFF, dtype=torch.uint8, device=DEV) if n else None
    rsd.attn_fwd_paged(q, k, v, o, lse, torch.as_tensor(table, device=DEV),
                       torch.as_tensor(np.asarray(lens, dtype=np.int32), device=DEV), page_size=ps,
                       max_kv_len=max(1, int(max(lens))), scale=scale, num_splits=splits, workspace=ws)
    torch.cuda.synchronize()


def _mixed(lens_q, lens_kv, Hq, Hkv, D, ps, seed):
    table, total = synth.page_table(lens_kv, ps, seed)
    cu_q = synth.cu_seqlens(lens_q)
    q = synth.normal_bf16((int(cu_q[-1]), Hq, D), seed + 1, "cpu").to(DEV)
    k = synth.normal_bf16((total + 2, Hkv, ps, D), seed + 2, "cpu").to(DEV)
    v = synth.normal_bf16((total + 2, Hkv, ps, D), seed + 3, "cpu").to(DEV)
    return q, k, v, cu_q, table


def _run_mixed(q, k, v, cu_q, table, lens_kv, ps, scale, splits, o, lse, lse_layout):
    B = len(cu_q) - 1
    smax = int(np.max(np.diff(cu_q)))
    T, Hq, D = q.shape
    Hkv = k.shape[1]
    ws = torch.empty(rsd.attn_fwd_paged_prefill_workspace_size(B, smax, T, Hq, Hkv, D, splits),
                     dtype=torch.uint8, device=DEV)
    rsd.attn_fwd_paged_prefill(q, k, v, o, lse, torch.as_tensor(cu_q, device=DEV), torch.as_tensor(table, device=DEV),
                               torch.as_tensor(np.asarray(lens_kv, dtype=np.int32), device=DEV), max_seqlen_q=smax,
                               page_size=ps, max_kv_len=int(max(lens_kv)), scale=scale, causal=True, workspace=ws,
                               num_splits=splits, lse_layout=lse_layout)
    torch.cuda.synchronize()


# ------------------------------------------------------------------ guard bands
@pytest.mark.parametrize("layout", [rsd.ATTN_LSE_PADDED_BSH, rsd.ATTN_LSE_PACKED_TH, rsd.ATTN_LSE_PACKED_HT])
def test_guard_bands_ragged(layout):
    lq, lkv = [37, 300, 1, 129], [37, 400, 5, 129]
    q, k, v, cu_q, cu_kv = _ragged(lq, lkv, 8, 2, 128, seed=101)
    T, Hq = q.shape[0], q.shape[1]
    lshape = _ragged_lse_shape(layout, len(lq), max(lq), T, Hq)
    o, ob, om = guarded_bf16((T, Hq, 128))
    lse, lb, lm = guarded_f32(lshape)
    _run_ragged(q, k, v, cu_q, cu_kv, 0.09, True, o, lse, layout)
    assert_canaries(ob, om, "ragged O")
    assert_canaries(lb, lm, "ragged LSE")
    o2 = torch.empty((T, Hq, 128), dtype=torch.bfloat16, device=DEV)
    lse2 = torch.empty(lshape, dtype=torch.float32, device=DEV)
    _run_ragged(q, k, v, cu_q, cu_kv, 0.09, True, o2, lse2, layout)
    same_bits(o.contiguous(), o2, "ragged O vs plain buffers")
    same_bits(lse, lse2, "ragged LSE vs plain buffers")


def test_guard_bands_dense():
    B, S, Hq, Hkv, D = 2, 200, 4, 2, 64
    q = synth.normal_bf16((B, S, Hq, D), 111, "cpu").to(DEV)
    k = synth.normal_bf16((B, S, Hkv, D), 112, "cpu").to(DEV)
    v = synth.normal_bf16((B, S, Hkv, D), 113, "cpu").to(DEV)
    o, ob, om = guarded_bf16((B, S, Hq, D))
    lse, lb, lm = guarded_f32((B, Hq, S))
    ws = torch.empty(rsd.attn_fwd_dense_workspace_size(B, S, Hq, Hkv), dtype=torch.uint8, device=DEV)
    rsd.attn_fwd_dense(q, k, v, o, lse, scale=0.1, causal=True, workspace=ws)
    torch.cuda.synchronize()
    assert_canaries(ob, om, "dense O")
    assert_canaries(lb, lm, "dense LSE")
    o2 = torch.empty((B, S, Hq, D), dtype=torch.bfloat16, device=DEV)
    lse2 = torch.empty((B, Hq, S), dtype=torch.float32, device=DEV)
    rsd.attn_fwd_dense(q, k, v, o2, lse2, scale=0.1, causal=True, workspace=ws)
    torch.cuda.synchronize()
    same_bits(o.contiguous(), o2, "dense O vs plain buffers")
    same_bits(lse, lse2, "dense LSE vs plain buffers")


@pytest.mark.parametrize("mla,splits", [(False, 1), (False, 3), (True, 1), (True, 3)])
def test_guard_bands_paged_decode(mla, splits):
    lens = [0, 1, 100, 700]
    if mla:
        q, k, v, table = _paged(lens, 128, 1, 576, 64, seed=121, alias=True)
        Dv = 512
    else:
        q, k, v, table = _paged(lens, 16, 2, 128, 64, seed=131)
        Dv = 128
    B, Hq = q.shape[0], q.shape[1]
    o, ob, om = guarded_bf16((B, Hq, Dv))
    lse, lb, lm = guarded_f32((B, Hq))
    _run_paged(q, k, v, table, lens, 64, 0.06, splits, o, lse)
    assert_canaries(ob, om, "paged O")
    assert_canaries(lb, lm, "paged LSE")
    o2 = torch.empty((B, Hq, Dv), dtype=torch.bfloat16, device=DEV)
    lse2 = torch.empty((B, Hq), dtype=torch.float32, device=DEV)
    _run_paged(q, k, v, table, lens, 64, 0.06, splits, o2, lse2)
    same_bits(o.contiguous(), o2, "paged O vs plain buffers")
    same_bits(lse, lse2, "paged LSE vs plain buffers")


@pytest.mark.parametrize("layout", [rsd.ATTN_LSE_PADDED_BSH, rsd.ATTN_LSE_PACKED_TH])
def test_guard_bands_mixed_batch(layout):
    lens_q, lens_kv = [3, 200, 1, 4], [50, 700, 64, 4]
    q, k, v, cu_q, table = _mixed(lens_q, lens_kv, 8, 2, 128, 64, seed=141)
    T, Hq = q.shape[0], q.shape[1]
    lshape = _ragged_lse_shape(layout, len(lens_q), max(lens_q), T, Hq)
    o, ob, om = guarded_bf16((T, Hq, 128))
    lse, lb, lm = guarded_f32(lshape)
    _run_mixed(q, k, v, cu_q, table, lens_kv, 64, 0.08, 2, o, lse, layout)
    assert_canaries(ob, om, "mixed O")
    assert_canaries(lb, lm, "mixed LSE")
    o2 = torch.empty((T, Hq, 128), dtype=torch.bfloat16, device=DEV)
    lse2 = torch.empty(lshape, dtype=torch.float32, device=DEV)
    _run_mixed(q, k, v, cu_q, table, lens_kv, 64, 0.08, 2, o2, lse2, layout)
    same_bits(o.contiguous(), o2, "mixed O vs plain buffers")
    same_bits(lse, lse2, "mixed LSE vs plain buffers")


# ------------------------------------------------------------------ single visible key
def test_single_key_rows_return_v_exactly():
    """Ragged and dense causal rows 0 (S_q = S_kv) and ragged rows over one-key
    sequences see exactly one key: O is that key's V row, bit for bit, and LSE is
    scale * q.k (fp64 reference)."""
    scale = 0.11
    lq, lkv = [1, 1, 300, 129], [1, 1, 300, 129]
    q, k, v, cu_q, cu_kv = _ragged(lq, lkv, 8, 2, 128, seed=151)
    T, Hq = q.shape[0], q.shape[1]
    o = torch.empty((T, Hq, 128), dtype=torch.bfloat16, device=DEV)
    lse = torch.empty((len(lq), max(lq), Hq), dtype=torch.float32, device=DEV)
    _run_ragged(q, k, v, cu_q, cu_kv, scale, True, o, lse, rsd.ATTN_LSE_PADDED_BSH)
    G = Hq // k.shape[1]
    for b in range(len(lq)):
        t, j = int(cu_q[b]), int(cu_kv[b])  # row 0 of sequence b sees only key 0
        for h in range(Hq):
            assert torch.equal(o[t, h].view(torch.int16), v[j, h // G].view(torch.int16)), (b, h)
            want = scale * float((q[t, h].double() * k[j, h // G].double()).sum())
            assert abs(float(lse[b, 0, h]) - want) < 1e-4, (b, h)
    # dense, causal: query row 0 of every batch sees key 0 only
    B, S, Hkv = 2, 130, 2
    qd = synth.normal_bf16((B, S, Hq, 64), 161, "cpu").to(DEV)
    kd = synth.normal_bf16((B, S, Hkv, 64), 162, "cpu").to(DEV)
    vd = synth.normal_bf16((B, S, Hkv, 64), 163, "cpu").to(DEV)
    od = torch.empty((B, S, Hq, 64), dtype=torch.bfloat16, device=DEV)
    ws = torch.empty(rsd.attn_fwd_dense_workspace_size(B, S, Hq, Hkv), dtype=torch.uint8, device=DEV)
    rsd.attn_fwd_dense(qd, kd, vd, od, None, scale=scale, causal=True, workspace=ws)
    torch.cuda.synchronize()
    for b in range(B):
        for h in range(Hq):
            assert torch.equal(od[b, 0, h].view(torch.int16), vd[b, 0, h // (Hq // Hkv)].view(torch.int16))


@pytest.mark.parametrize("mla,splits", [(False, 1), (False, 4), (True, 1), (True, 4)])
def test_single_key_decode_returns_v_exactly(mla, splits):
    lens = [1, 1, 1]
    if mla:
        q, k, v, table = _paged(lens, 128, 1, 576, 64, seed=171, alias=True)
        Dv = 512
    else:
        q, k, v, table = _paged(lens, 16, 2, 128, 64, seed=181)
        Dv = 128
    B, Hq = q.shape[0], q.shape[1]
    G = Hq // k.shape[1]
    o = torch.empty((B, Hq, Dv), dtype=torch.bfloat16, device=DEV)
    lse = torch.empty((B, Hq), dtype=torch.float32, device=DEV)
    _run_paged(q, k, v, table, lens, 64, 0.07, splits, o, lse)
    for b in range(B):
        page = int(table[b, 0])
        for h in range(Hq):
            vrow = v[page, h // G, 0, :Dv]
            assert torch.equal(o[b, h].view(torch.int16), vrow.contiguous().view(torch.int16)), (b, h)


# ------------------------------------------------------------------ uniform scores
def _counts(lq, lkv, causal):
    out = []
    for Lq, Lk in zip(lq, lkv):
        i = np.arange(Lq)
        c = np.minimum(Lk, i + 1 + Lk - Lq) if causal else np.full(Lq, Lk)
        out.append(np.maximum(c, 0))
    return out


def _assert_counts(lse_rows, counts, where):
    lse_rows = np.asarray(lse_rows, dtype=np.float64)
    empty = counts == 0
    assert np.all(lse_rows[empty] == -np.inf), f"{where}: rows without keys need LSE = -inf"
    got = np.rint(np.exp(lse_rows[~empty]))
    bad = got != counts[~empty]
    assert not bad.any(), f"{where}: {int(bad.sum())} rows count the wrong number of keys"


@pytest.mark.parametrize("causal", [True, False])
def test_uniform_scores_count_keys_ragged_and_dense(causal):
    lq, lkv = [1, 77, 300, 130, 5], [9, 77, 450, 129, 2]
    q, k, v, cu_q, cu_kv = _ragged(lq, lkv, 4, 1, 64, seed=191)
    T, Hq = q.shape[0], q.shape[1]
    o = torch.empty((T, Hq, 64), dtype=torch.bfloat16, device=DEV)
    lse = torch.empty((len(lq), max(lq), Hq), dtype=torch.float32, device=DEV)
    _run_ragged(q, k, v, cu_q, cu_kv, 0.0, causal, o, lse, rsd.ATTN_LSE_PADDED_BSH)
    counts = _counts(lq, lkv, causal)
    vd = v.double().cpu().numpy()
    for b in range(len(lq)):
        for h in range(Hq):
            _assert_counts(lse[b, :lq[b], h].cpu().numpy(), counts[b], f"ragged b={b} h={h}")
        # O = mean of the visible V rows
        c = counts[b]
        pre = np.cumsum(np.concatenate([np.zeros((1, 64)), vd[cu_kv[b]:cu_kv[b + 1], 0]]), axis=0)
        ref = np.where(c[:, None] > 0, pre[c] / np.maximum(c, 1)[:, None], 0.0)
        for h in range(Hq):
            assert_o_close(o[cu_q[b]:cu_q[b + 1], h], ref, f"ragged mean b={b} h={h}")
    B, S, Hq2, Hkv = 2, 260, 4, 2
    qd = synth.normal_bf16((B, S, Hq2, 128), 201, "cpu").to(DEV)
    kd = synth.normal_bf16((B, S, Hkv, 128), 202, "cpu").to(DEV)
    od = torch.empty((B, S, Hq2, 128), dtype=torch.bfloat16, device=DEV)
    ld = torch.empty((B, Hq2, S), dtype=torch.float32, device=DEV)
    ws = torch.empty(rsd.attn_fwd_dense_workspace_size(B, S, Hq2, Hkv), dtype=torch.uint8, device=DEV)
    rsd.attn_fwd_dense(qd, kd, kd, od, ld, scale=0.0, causal=causal, workspace=ws)
    torch.cuda.synchronize()
    cd = _counts([S], [S], causal)[0]
    for b in range(B):
        for h in range(Hq2):
            _assert_counts(ld[b, h].cpu().numpy(), cd, f"dense b={b} h={h}")


@pytest.mark.parametrize("splits", [1, 3])
def test_uniform_scores_count_keys_mixed_batch(splits):
    lens_q, lens_kv = [1, 2, 4, 200, 3, 130], [1, 70, 64, 700, 300, 130]
    q, k, v, cu_q, table = _mixed(lens_q, lens_kv, 8, 2, 128, 64, seed=211)
    T, Hq = q.shape[0], q.shape[1]
    o = torch.empty((T, Hq, 128), dtype=torch.bfloat16, device=DEV)
    lse = torch.empty((len(lens_q), max(lens_q), Hq), dtype=torch.float32, device=DEV)
    _run_mixed(q, k, v, cu_q, table, lens_kv, 64, 0.0, splits, o, lse, rsd.ATTN_LSE_PADDED_BSH)
    counts = _counts(lens_q, lens_kv, True)
    for b in range(len(lens_q)):
        for h in range(Hq):
            _assert_counts(lse[b, :lens_q[b], h].cpu().numpy(), counts[b], f"mixed b={b} h={h}")


@pytest.mark.parametrize("mla,splits", [(False, 1), (False, 5), (True, 1), (True, 5)])
def test_uniform_scores_count_keys_decode(mla, splits):
    lens = [1, 63, 64, 65, 1000]
    if mla:
        q, k, v, table = _paged(lens, 128, 1, 576, 64, seed=221, alias=True)
        Dv = 512
    else:
        q, k, v, table = _paged(lens, 16, 2, 128, 64, seed=231)
        Dv = 128
    B, Hq = q.shape[0], q.shape[1]
    o = torch.empty((B, Hq, Dv), dtype=torch.bfloat16, device=DEV)
    lse = torch.empty((B, Hq), dtype=torch.float32, device=DEV)
    _run_paged(q, k, v, table, lens, 64, 0.0, splits, o, lse)
    for b in range(B):
        _assert_counts(lse[b].cpu().numpy(), np.full(Hq, lens[b]), f"decode b={b}")
