"""Bit-exact checks of the metadata the device builds ("cuDNN Frontend v1.28.0
release notes", "Ragged / THD, with zero host reads": the THD metadata is built
on the device; "cuDNN Frontend v1.31.0 Release Notes", "SDPA: paged KV,
split-KV, and engine selection": page-table addressing).

After a real call, the caller-owned workspace holds the work list the device
built ({count, claim counter} header, then {b, qtile, h0, cost} items); the
test copies it out and compares it with the list ``metadata_check`` derives on
the host from the documented order: every item exactly once, each sequence's
run in order, runs most work first, and a claim counter that shows every item
was handed out once.  The split-decode schedule, the split MLA decode's
launch order and the page-table coordinates (through the diagnostic
entry point that runs the producers' own address functions) are checked the
same way."""
import numpy as np
import pytest
import torch

import metadata_check as mc
import ragged_scaled_dot_b200 as rsd
import synth

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _sms():
    return torch.cuda.get_device_properties(0).multi_processor_count


def _header_items(ws, n_max):
    h = ws[:256].cpu().view(torch.int32).numpy()
    count = int(h[0])
    assert 0 <= count <= n_max
    items = ws[256:256 + 16 * count].cpu().view(torch.int32).numpy().reshape(-1, 4)
    return count, int(h[1]), items


def _ragged_call(lq, lkv, Hq, Hkv, D, causal, seed):
    cu_q, cu_k = synth.cu_seqlens(lq), synth.cu_seqlens(lkv)
    Tq, Tk = int(cu_q[-1]), int(cu_k[-1])
    q = synth.normal_bf16((max(Tq, 1), Hq, D), seed, DEV)
    k = synth.normal_bf16((max(Tk, 1), Hkv, D), seed + 1, DEV)
    v = synth.normal_bf16((max(Tk, 1), Hkv, D), seed + 2, DEV)
    o = torch.empty_like(q)
    B, smax, kmax = len(lq), max(1, int(max(lq))), max(1, int(max(lkv)))
    n = rsd.attn_fwd_ragged_workspace_size(B, smax, Tq, Hq, Hkv)
    ws = torch.full((n,), 0xA5, dtype=torch.uint8, device=DEV)  # stale bytes must not leak into the list
    rsd.attn_fwd_ragged(q, k, v, o, None, torch.as_tensor(cu_q, device=DEV), torch.as_tensor(cu_k, device=DEV),
                        max_seqlen_q=smax, max_seqlen_kv=kmax, scale=0.1, causal=causal, workspace=ws,
                        total_q=Tq, total_kv=Tk)
    torch.cuda.synchronize()
    assert rsd.attn_get_device_error() == rsd.ATTN_OK
    n_pairs = Hq // mc.heads_per_item(Hq, Hkv)
    grid = min(mc.ragged_max_tiles(B, smax, Tq) * n_pairs, _sms())
    return ws, (n - 256) // 16, grid


RAGGED_CASES = [
    ("tiny", [37, 64], [37, 64], 4, 1, 64, True),
    ("ties_zeros_causal", [0, 128, 129, 1, 0, 300, 128, 4000], [0, 128, 129, 1, 9, 300, 128, 4000], 8, 2, 64, True),
    ("ties_zeros_full", [0, 128, 129, 1, 0, 300, 128, 4000], [5, 128, 1000, 1, 0, 300, 128, 77], 8, 2, 64, False),
    ("odd_group", [513, 200, 64], [513, 700, 64], 6, 2, 128, True),
]


@pytest.mark.parametrize("name,lq,lkv,Hq,Hkv,D,causal", RAGGED_CASES, ids=[c[0] for c in RAGGED_CASES])
def test_ragged_work_list_bit_exact(name, lq, lkv, Hq, Hkv, D, causal):
    ws, n_max, grid = _ragged_call(lq, lkv, Hq, Hkv, D, causal, seed=len(lq) + Hq)
    count, claims, items = _header_items(ws, n_max)
    mc.check_sequence_list(items, count, np.array(lq), np.array(lkv), Hq, Hkv, causal)
    assert claims == count + grid, f"claim counter {claims}, expected {count} items + {grid} CTAs"


def test_ragged_work_list_config3_lengths():
    """The ragged workload's own 64 lengths U[128, 8192] and heads 32 / 8 (head dim 64 to keep it small)."""
    L = synth.WORKLOADS["ragged_prefill"].seq_lengths()
    ws, n_max, grid = _ragged_call(L.tolist(), L.tolist(), 32, 8, 64, True, seed=3)
    count, claims, items = _header_items(ws, n_max)
    mc.check_sequence_list(items, count, L, L, 32, 8, True)
    assert claims == count + grid


@pytest.mark.parametrize("B,S,Hq,Hkv,D,causal", [(2, 1100, 8, 2, 64, True), (8, 4096, 32, 8, 128, True),
                                                 (3, 300, 6, 2, 64, False)])
def test_dense_work_list_bit_exact(B, S, Hq, Hkv, D, causal):
    q = synth.normal_bf16((B, S, Hq, D), 1, DEV)
    k = synth.normal_bf16((B, S, Hkv, D), 2, DEV)
    o = torch.empty_like(q)
    n = rsd.attn_fwd_dense_workspace_size(B, S, Hq, Hkv)
    ws = torch.full((n,), 0xA5, dtype=torch.uint8, device=DEV)
    rsd.attn_fwd_dense(q, k, k, o, None, scale=0.1, causal=causal, workspace=ws)
    torch.cuda.synchronize()
    assert rsd.attn_get_device_error() == rsd.ATTN_OK
    count, claims, items = _header_items(ws, (n - 256) // 16)
    mc.check_dense_list(items, count, B, S, S, Hq, Hkv, causal)
    assert claims == count + min(count, _sms())


def test_paged_prefill_work_list_bit_exact():
    lq = [1, 2, 4, 100, 129, 0, 1024]
    lkv = [1000, 64, 300, 100, 2000, 50, 1024]
    Hq, Hkv, D, ps = 16, 4, 128, 64
    table, total = synth.page_table(lkv, ps, 9)
    cu_q = synth.cu_seqlens(lq)
    T = int(cu_q[-1])
    q = synth.normal_bf16((T, Hq, D), 1, DEV)
    kp = synth.normal_bf16((total, Hkv, ps, D), 2, DEV)
    o = torch.empty_like(q)
    n = rsd.attn_fwd_paged_prefill_workspace_size(len(lq), max(lq), T, Hq, Hkv)
    ws = torch.full((n,), 0xA5, dtype=torch.uint8, device=DEV)
    rsd.attn_fwd_paged_prefill(q, kp, kp, o, None, torch.as_tensor(cu_q, device=DEV),
                               torch.as_tensor(table, device=DEV),
                               torch.as_tensor(np.array(lkv, dtype=np.int32), device=DEV), max_seqlen_q=max(lq),
                               page_size=ps, max_kv_len=max(lkv), scale=0.1, causal=True, workspace=ws)
    torch.cuda.synchronize()
    assert rsd.attn_get_device_error() == rsd.ATTN_OK
    count, claims, items = _header_items(ws, (n - 256) // 16)
    # the 1-, 2- and 4-query sequences go to the split-KV decode kernel: no prefill items
    short_q = mc.routed_qmax(Hq // Hkv, max(lq))
    assert short_q == 4
    mc.check_sequence_list(items, count, np.array(lq), np.array(lkv), Hq, Hkv, True, short_q)
    n_pairs = Hq // mc.heads_per_item(Hq, Hkv)
    assert claims == count + min(mc.ragged_max_tiles(len(lq), max(lq), T) * n_pairs, _sms())


@pytest.mark.parametrize("lens_kind", ["mla_workload", "ties"])
def test_split_mla_decode_launch_order(lens_kind):
    """The split MLA decode's clusters take the sequences longest first."""
    if lens_kind == "mla_workload":
        L = synth.WORKLOADS["mla_decode"].seq_lengths()
    else:
        L = np.array([64, 4096, 64, 1, 4096, 4097, 63, 64] * 4, dtype=np.int64)
    B, Hq, ps, S = len(L), 128, 64, 3
    table, total = synth.page_table(L, ps, 4)
    q = synth.normal_bf16((B, Hq, 576), 1, DEV)
    kp = synth.normal_bf16((total, 1, ps, 576), 2, DEV)
    o = torch.empty((B, Hq, 512), dtype=torch.bfloat16, device=DEV)
    n = rsd.attn_fwd_paged_workspace_size(B, Hq, 512, S)
    ws = torch.full((n,), 0xA5, dtype=torch.uint8, device=DEV)
    maxL = int(L.max())
    rsd.attn_fwd_paged(q, kp, kp, o, None, torch.as_tensor(table, device=DEV),
                       torch.as_tensor(L.astype(np.int32), device=DEV), page_size=ps, max_kv_len=maxL, scale=0.04,
                       num_splits=S, workspace=ws)
    torch.cuda.synchronize()
    assert rsd.attn_get_device_error() == rsd.ATTN_OK
    R = B * Hq

    def up(x):
        return (x + 255) // 256 * 256
    off = up(R * S * 512 * 4) + up(R * S * 4)
    order = ws[off:off + 4 * B].cpu().view(torch.int32).numpy()
    mc.check_decode_order(order, L, maxL)


def _up(x):
    return (x + 255) // 256 * 256


def _split_offsets(base, B):
    """Byte offsets of the split workspace's order and piece records, as the layout
    states: per-sequence data [B] x 16 B, order [B], then one 32-byte record per block."""
    order = _up(base + B * 16)
    return order, _up(order + B * 4)


def _pieces_from_ws(ws, order_off, segs_off, B, n_blocks):
    order = ws[order_off:order_off + 4 * B].cpu().view(torch.int32).numpy()
    rows = ws[segs_off:segs_off + 32 * n_blocks].cpu().view(torch.int32).numpy().reshape(n_blocks, 8)
    return order, rows


@pytest.mark.parametrize("lens_kind,S", [("config4", 2), ("ties_and_zeros", 3), ("one_long", 64)])
def test_split_decode_schedule(lens_kind, S):
    """The split-decode schedule the device writes (order and one piece per block)
    equals the host rule, bit for bit: longest first, each pair cut into min(S, units)
    near-equal pieces, every unit of every (sequence, KV head) in one block."""
    if lens_kind == "config4":
        L = synth.WORKLOADS["paged_decode"].seq_lengths()
    elif lens_kind == "ties_and_zeros":
        L = np.array([64, 4096, 0, 1, 4096, 4097, 63, 0, 65] * 3, dtype=np.int64)
    else:
        L = np.array([50000, 3], dtype=np.int64)
    B, Hq, Hkv, D, ps = len(L), 16, 2, 128, 64
    table, total = synth.page_table(L, ps, 4)
    q = synth.normal_bf16((B, Hq, D), 1, DEV)
    kp = synth.normal_bf16((total, Hkv, ps, D), 2, DEV)
    o = torch.empty((B, Hq, D), dtype=torch.bfloat16, device=DEV)
    n = rsd.attn_fwd_paged_workspace_size(B, Hq, D, S)
    ws = torch.full((n,), 0xA5, dtype=torch.uint8, device=DEV)
    maxL = int(L.max())
    rsd.attn_fwd_paged(q, kp, kp, o, None, torch.as_tensor(table, device=DEV),
                       torch.as_tensor(L.astype(np.int32), device=DEV), page_size=ps, max_kv_len=maxL, scale=0.1,
                       num_splits=S, workspace=ws)
    torch.cuda.synchronize()
    assert rsd.attn_get_device_error() == rsd.ATTN_OK
    order_off, segs_off = _split_offsets(0, B)
    order, rows = _pieces_from_ws(ws, order_off, segs_off, B, S * B * Hkv)
    mc.check_decode_pieces(order, rows, L, Hkv, S, maxL)


def test_split_decode_schedule_ragged_queries():
    """The mixed batch's short rows: sequences of 1..qmax queries own units, the
    chunk sequences (prefill kernel) none; the schedule follows the same rule."""
    lens_q = [1, 3, 700, 2, 0, 1, 129, 4]
    lens_kv = [5000, 90, 3000, 1, 64, 0, 800, 4100]
    B, Hq, Hkv, D, ps, S = len(lens_q), 16, 2, 128, 64, 3
    G = Hq // Hkv
    qmax = min(4, 64 // G, max(lens_q))
    cu_q = synth.cu_seqlens(lens_q)
    T = int(cu_q[-1])
    L = np.asarray(lens_kv, dtype=np.int64)
    table, total = synth.page_table(L, ps, 5)
    q = synth.normal_bf16((T, Hq, D), 1, DEV)
    kp = synth.normal_bf16((total, Hkv, ps, D), 2, DEV)
    o = torch.empty((T, Hq, D), dtype=torch.bfloat16, device=DEV)
    lse = torch.empty((B, max(lens_q), Hq), dtype=torch.float32, device=DEV)
    n = rsd.attn_fwd_paged_prefill_workspace_size(B, max(lens_q), T, Hq, Hkv, D, S)
    ws = torch.full((n,), 0xA5, dtype=torch.uint8, device=DEV)
    rsd.attn_fwd_paged_prefill(q, kp, kp, o, lse, torch.as_tensor(cu_q, device=DEV), torch.as_tensor(table, device=DEV),
                               torch.as_tensor(L.astype(np.int32), device=DEV), max_seqlen_q=max(lens_q),
                               page_size=ps, max_kv_len=int(L.max()), scale=0.1, causal=True, workspace=ws,
                               num_splits=S)
    torch.cuda.synchronize()
    assert rsd.attn_get_device_error() == rsd.ATTN_OK
    base = rsd.attn_fwd_ragged_workspace_size(B, max(lens_q), T, Hq, Hkv)
    order_off, segs_off = _split_offsets(base, B)
    order, rows = _pieces_from_ws(ws, order_off, segs_off, B, S * B * Hkv)
    mc.check_decode_pieces(order, rows, L, Hkv, S, int(L.max()), cu_q=cu_q, qmax=qmax)


@pytest.mark.parametrize("ps", [64, 16])
def test_page_coordinates_bit_exact(ps):
    L = synth.WORKLOADS["paged_decode"].seq_lengths()
    table, total = synth.page_table(L, ps, 4)
    gpp = ps // 8
    rng = np.random.default_rng(7)
    b_idx, t_idx = [], []
    for b in rng.choice(len(L), 8, replace=False):  # both sides of every page boundary of 8 sequences
        for t in range(ps, int(L[b]), ps):
            b_idx += [b, b]
            t_idx += [t - 1, t]
    for _ in range(4096):
        b = int(rng.integers(len(L)))
        b_idx.append(b)
        t_idx.append(int(rng.integers(L[b])))
    b_idx, t_idx = np.array(b_idx, dtype=np.int32), np.array(t_idx, dtype=np.int32)

    def run(tab):
        out = torch.full((len(b_idx), 3), -7, dtype=torch.int64, device=DEV)
        rsd.attn_selftest_page_coords(torch.as_tensor(tab, device=DEV), torch.as_tensor(b_idx, device=DEV),
                                      torch.as_tensor(t_idx, device=DEV), out, page_size=ps, num_pages=total,
                                      groups_per_page=gpp)
        torch.cuda.synchronize()
        return out.cpu().numpy()

    got = run(table)
    assert np.array_equal(got, mc.page_coords(table, b_idx, t_idx, ps, total, gpp))
    assert rsd.attn_get_device_error() == rsd.ATTN_OK
    # out-of-range ids read as page -1 and are reported
    bad = table.copy()
    bad[int(b_idx[0]), int(t_idx[0]) // ps] = -1
    bad[int(b_idx[-1]), int(t_idx[-1]) // ps] = total
    got = run(bad)
    assert np.array_equal(got, mc.page_coords(bad, b_idx, t_idx, ps, total, gpp))
    assert got[0, 0] == -1 and got[-1, 0] == -1
    assert rsd.attn_get_device_error() == rsd.ATTN_ERR_DEVICE_INPUT
