"""Helpers shared by the GPU parity tests: run the CUDA path through the
binding, run the fp64 oracle on the same bf16 bytes, and compare with the
tolerance the benchmark spec fixes for bf16 attention:

    |O_gpu - O_ref| <= 1e-2 + 1e-2 * |O_ref|   (per element)
    |LSE_gpu - LSE_ref| <= 1e-3                 (both -inf where the row has no keys)
"""
from __future__ import annotations

import numpy as np
import torch

import oracle
import ragged_scaled_dot_b200 as rsd
import synth

O_ATOL = 1e-2
O_RTOL = 1e-2
LSE_ATOL = 1e-3
LOG2E = 1.4426950408889634


def lse_base(lse_layout):
    """The layout part of an lse_layout value (without the base-2 flag)."""
    return lse_layout & ~rsd.ATTN_LSE_LOG2


def lse_alloc(lse_layout, B, max_sq, Tq, Hq, fill, dev):
    base = lse_base(lse_layout)
    if base == rsd.ATTN_LSE_PADDED_BSH:
        shape = (B, max_sq, Hq)
    elif base == rsd.ATTN_LSE_PACKED_TH:
        shape = (Tq, Hq)
    else:
        shape = (Hq, Tq)
    return torch.full(shape, fill, dtype=torch.float32, device=dev)


def assert_o_close(o_gpu, o_ref, where=""):
    og = o_gpu.detach().float().cpu().numpy().astype(np.float64).reshape(o_ref.shape)
    assert np.all(np.isfinite(og)), f"{where}: non-finite outputs"
    err = np.abs(og - o_ref)
    bad = err > (O_ATOL + O_RTOL * np.abs(o_ref))
    assert not bad.any(), (f"{where}: {int(bad.sum())}/{bad.size} O elements out of tolerance, "
                           f"max abs err {err.max():.3e}")
    return float(err.max())


def assert_lse_close(lse_gpu, lse_ref, where="", atol=LSE_ATOL):
    lg = np.asarray(lse_gpu.detach().cpu().numpy() if torch.is_tensor(lse_gpu) else lse_gpu,
                    dtype=np.float64).reshape(lse_ref.shape)
    ninf = lse_ref == -np.inf
    assert np.all(lg[ninf] == -np.inf), f"{where}: rows without keys must have LSE = -inf"
    fin = ~ninf
    assert np.all(np.isfinite(lg[fin])), f"{where}: non-finite LSE"
    err = np.abs(lg[fin] - lse_ref[fin]) if fin.any() else np.zeros(1)
    assert err.max() <= atol, f"{where}: LSE max abs err {err.max():.3e}"
    return float(err.max())


def bits(t):
    return synth.bf16_bits(t)


def orc():
    return oracle.default()


# ------------------------------------------------------------------ ragged
def ragged_gpu(q, k, v, cu_q, cu_kv, max_sq, max_skv, scale, causal, lse_layout=rsd.ATTN_LSE_PADDED_BSH,
               total_q=None, total_kv=None, o_fill=float("nan"), lse_fill=float("nan")):
    dev = q.device
    B = len(cu_q) - 1
    Tq = q.shape[0]
    o = torch.full((Tq, q.shape[1], v.shape[2]), o_fill, dtype=torch.bfloat16, device=dev)
    tq = Tq if total_q is None else total_q
    lse = lse_alloc(lse_layout, B, max_sq, tq, q.shape[1], lse_fill, dev)
    ws = torch.empty(rsd.attn_fwd_ragged_workspace_size(B, max_sq, tq, q.shape[1], k.shape[1]),
                     dtype=torch.uint8, device=dev)
    cq = torch.as_tensor(np.asarray(cu_q, dtype=np.int32), device=dev)
    ck = torch.as_tensor(np.asarray(cu_kv, dtype=np.int32), device=dev)
    rsd.attn_fwd_ragged(q, k, v, o, lse, cq, ck, max_seqlen_q=max_sq, max_seqlen_kv=max_skv,
                        scale=scale, causal=causal, workspace=ws, lse_layout=lse_layout,
                        total_q=total_q, total_kv=total_kv)
    torch.cuda.synchronize()
    return o, lse


def ragged_rows_all(cu_q, Hq):
    rows = []
    for b in range(len(cu_q) - 1):
        for h in range(Hq):
            for i in range(int(cu_q[b + 1] - cu_q[b])):
                rows.append((b, h, i))
    return np.array(rows, dtype=np.int32).reshape(-1, 3)


def gather_ragged(o, lse, cu_q, rows, lse_layout=rsd.ATTN_LSE_PADDED_BSH):
    """Pick GPU outputs at oracle rows (b, h, i)."""
    rows = np.asarray(rows)
    tok = np.asarray(cu_q, dtype=np.int64)[rows[:, 0]] + rows[:, 2]
    t_tok = torch.as_tensor(tok, device=o.device)
    t_h = torch.as_tensor(rows[:, 1].astype(np.int64), device=o.device)
    og = o[t_tok, t_h]
    base = lse_base(lse_layout)
    if base == rsd.ATTN_LSE_PADDED_BSH:
        lg = lse[torch.as_tensor(rows[:, 0].astype(np.int64), device=o.device),
                 torch.as_tensor(rows[:, 2].astype(np.int64), device=o.device), t_h]
    elif base == rsd.ATTN_LSE_PACKED_TH:
        lg = lse[t_tok, t_h]
    else:
        lg = lse[t_h, t_tok]
    return og, lg


def check_ragged(q, k, v, cu_q, cu_kv, scale, causal, rows=None, where="", **kw):
    max_sq = int(np.max(np.diff(cu_q))) if len(cu_q) > 1 else 0
    max_skv = int(np.max(np.diff(cu_kv))) if len(cu_kv) > 1 else 0
    max_sq = kw.pop("max_sq", max(max_sq, 1))
    max_skv = kw.pop("max_skv", max(max_skv, 1))
    o, lse = ragged_gpu(q, k, v, cu_q, cu_kv, max_sq, max_skv, scale, causal, **kw)
    if rows is None:
        rows = ragged_rows_all(cu_q, q.shape[1])
    o_ref, l_ref = orc().attn_ragged_rows(bits(q), bits(k), bits(v), cu_q, cu_kv, q.shape[1], k.shape[1],
                                          scale, causal, rows)
    layout = kw.get("lse_layout", rsd.ATTN_LSE_PADDED_BSH)
    og, lg = gather_ragged(o, lse, cu_q, rows, layout)
    e_o = assert_o_close(og, o_ref, where)
    if layout & rsd.ATTN_LSE_LOG2:
        # base-2 LSE = natural LSE * log2(e); the tolerance scales with it
        e_l = assert_lse_close(lg, l_ref * LOG2E, where, atol=LSE_ATOL * LOG2E)
    else:
        e_l = assert_lse_close(lg, l_ref, where)
    return o, lse, (e_o, e_l)


# ------------------------------------------------------------------- dense
def dense_gpu(q, k, v, scale, causal, o=None, lse=None):
    B, Sq, Hq, _ = q.shape
    if o is None:
        o = torch.full((B, Sq, Hq, v.shape[-1]), float("nan"), dtype=torch.bfloat16, device=q.device)
    if lse is None:
        lse = torch.full((B, Hq, Sq), float("nan"), dtype=torch.float32, device=q.device)
    ws = torch.empty(rsd.attn_fwd_dense_workspace_size(B, Sq, Hq, k.shape[2]), dtype=torch.uint8, device=q.device)
    ws.fill_(0xFF)  # the call must build its list and reset its counter itself
    rsd.attn_fwd_dense(q, k, v, o, lse, scale=scale, causal=causal, workspace=ws)
    torch.cuda.synchronize()
    return o, lse


def check_dense(q, k, v, scale, causal, rows=None, where=""):
    B, Sq, Hq, Dqk = q.shape
    Skv, Hkv, Dv = k.shape[1], k.shape[2], v.shape[-1]
    o, lse = dense_gpu(q, k, v, scale, causal)
    if rows is None:
        rows = np.array([(b, h, i) for b in range(B) for h in range(Hq) for i in range(Sq)],
                        dtype=np.int32)
    qs = tuple(q.stride()[:3])
    ks = tuple(k.stride()[:3])
    vs = tuple(v.stride()[:3])
    o_ref, l_ref = orc().attn_dense_rows(
        _flat_bits(q), _flat_bits(k), _flat_bits(v), Sq, Skv, Hq, Hkv, Dqk, Dv, scale, causal, rows,
        q_strides=qs, k_strides=ks, v_strides=vs)
    r = torch.as_tensor(rows.astype(np.int64), device=q.device)
    og = o[r[:, 0], r[:, 2], r[:, 1]]
    lg = lse[r[:, 0], r[:, 1], r[:, 2]]
    return o, lse, (assert_o_close(og, o_ref, where), assert_lse_close(lg, l_ref, where))


def _flat_bits(t):
    """bf16 bits of the whole storage a (possibly strided) view addresses, from its origin."""
    base = t
    n = 1 + sum((s - 1) * st for s, st in zip(t.shape, t.stride()))
    flat = torch.as_strided(base, (n,), (1,))
    return bits(flat)


# ------------------------------------------------------------------- paged
def paged_gpu(q, k_pool, v_pool, table, kv_lens, page_size, scale, num_splits, kv_layout="HND",
              max_kv_len=None, o_dv=None):
    dev = q.device
    B, Hq, _ = q.shape
    Dv = o_dv or (v_pool.shape[-1] if v_pool is not k_pool else q.shape[-1])
    o = torch.full((B, Hq, Dv), float("nan"), dtype=torch.bfloat16, device=dev)
    lse = torch.full((B, Hq), float("nan"), dtype=torch.float32, device=dev)
    ws_n = rsd.attn_fwd_paged_workspace_size(B, Hq, Dv, num_splits)
    ws = torch.empty(max(ws_n, 1), dtype=torch.uint8, device=dev) if ws_n else None
    if ws is not None:
        ws.fill_(0xFF)  # garbage partials must be overwritten
    pt = torch.as_tensor(np.asarray(table, dtype=np.int32), device=dev)
    kl = torch.as_tensor(np.asarray(kv_lens, dtype=np.int32), device=dev)
    mk = int(max_kv_len if max_kv_len is not None else max(1, int(np.max(kv_lens))))
    rsd.attn_fwd_paged(q, k_pool, v_pool, o, lse, pt, kl, page_size=page_size, max_kv_len=mk,
                       scale=scale, num_splits=num_splits, workspace=ws, kv_layout=kv_layout)
    torch.cuda.synchronize()
    return o, lse


def pool_strides_np(pool, kv_layout):
    if kv_layout == "HND":
        return (pool.stride(0), pool.stride(2), pool.stride(1))
    return (pool.stride(0), pool.stride(1), pool.stride(2))


def check_paged(q, k_pool, v_pool, table, kv_lens, page_size, scale, num_splits, kv_layout="HND",
                rows=None, where="", Dv=None, host_pools=None):
    B, Hq, Dqk = q.shape
    Hkv = k_pool.shape[1] if kv_layout == "HND" else k_pool.shape[2]
    Dv = Dv or (v_pool.shape[-1] if v_pool is not k_pool else Dqk)
    o, lse = paged_gpu(q, k_pool, v_pool, table, kv_lens, page_size, scale, num_splits, kv_layout,
                       o_dv=Dv)
    if rows is None:
        rows = np.array([(b, h) for b in range(B) for h in range(Hq)], dtype=np.int32)
    kb, vb = host_pools if host_pools is not None else (bits(k_pool), bits(v_pool))
    o_ref, l_ref = orc().attn_paged_rows(
        bits(q), kb, vb, table, kv_lens, page_size, Hq, Hkv, Dqk, Dv,
        pool_strides_np(k_pool, kv_layout), pool_strides_np(v_pool, kv_layout), scale, rows)
    r = torch.as_tensor(np.asarray(rows, dtype=np.int64), device=q.device)
    og = o[r[:, 0], r[:, 1]]
    lg = lse[r[:, 0], r[:, 1]]
    return o, lse, (assert_o_close(og, o_ref, where), assert_lse_close(lg, l_ref, where))
