"""The entry points in a CUDA graph: no call reads device memory back or
allocates, so a captured call replays with new input values in the same
buffers ("cuDNN Frontend v1.28.0 release notes", "Ragged / THD, with zero
host reads": the THD path is CUDA-graph capturable).  Each replay must give
exactly what an eager call on the same new values gives."""
import numpy as np
import pytest
import torch

import ragged_scaled_dot_b200 as rsd
import synth

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _fill(t, seed):
    t.copy_(synth.normal_bf16(tuple(t.shape), seed, "cpu").to(DEV))


def test_ragged_prefill_replays_in_a_graph():
    lens = [100, 300, 1, 257]
    Hq, Hkv, D = 8, 2, 128
    cu = torch.as_tensor(synth.cu_seqlens(lens), device=DEV)
    T, B, smax = sum(lens), len(lens), max(lens)
    q = torch.empty((T, Hq, D), dtype=torch.bfloat16, device=DEV)
    k = torch.empty((T, Hkv, D), dtype=torch.bfloat16, device=DEV)
    v = torch.empty_like(k)
    o = torch.empty_like(q)
    lse = torch.empty((B, smax, Hq), dtype=torch.float32, device=DEV)
    ws = torch.empty(rsd.attn_fwd_ragged_workspace_size(B, smax, T, Hq, Hkv), dtype=torch.uint8, device=DEV)

    def call():
        rsd.attn_fwd_ragged(q, k, v, o, lse, cu, cu, max_seqlen_q=smax, max_seqlen_kv=smax, scale=0.09,
                            causal=True, workspace=ws)

    for t, s in ((q, 1), (k, 2), (v, 3)):
        _fill(t, s)
    call()  # eager first: per-device setup happens outside the capture
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        call()
    for rep in range(2):
        for t, s in ((q, 10 + rep), (k, 20 + rep), (v, 30 + rep)):
            _fill(t, s)
        o.fill_(float("nan"))
        lse.fill_(float("nan"))
        g.replay()
        torch.cuda.synchronize()
        o_g, l_g = o.clone(), lse.clone()
        call()
        torch.cuda.synchronize()
        assert torch.isfinite(o_g.float()).all()
        assert torch.equal(o_g, o) and torch.equal(l_g, lse)
    assert rsd.attn_get_device_error() == rsd.ATTN_OK
    del g


def test_paged_decode_with_splits_replays_in_a_graph():
    """Decode + split partials in the workspace + merge, all captured."""
    lens = [1000, 64, 3000]
    Hq, Hkv, D, ps, S = 16, 2, 128, 64, 3
    table, total = synth.page_table(lens, ps, 5)
    P = total + 2
    q = torch.empty((len(lens), Hq, D), dtype=torch.bfloat16, device=DEV)
    kp = torch.empty((P, Hkv, ps, D), dtype=torch.bfloat16, device=DEV)
    vp = torch.empty_like(kp)
    o = torch.empty((len(lens), Hq, D), dtype=torch.bfloat16, device=DEV)
    lse = torch.empty((len(lens), Hq), dtype=torch.float32, device=DEV)
    pt = torch.as_tensor(table, device=DEV)
    kl = torch.as_tensor(np.asarray(lens, dtype=np.int32), device=DEV)
    ws = torch.empty(rsd.attn_fwd_paged_workspace_size(len(lens), Hq, D, S), dtype=torch.uint8, device=DEV)

    def call():
        rsd.attn_fwd_paged(q, kp, vp, o, lse, pt, kl, page_size=ps, max_kv_len=max(lens), scale=0.088,
                           num_splits=S, workspace=ws)

    for t, s in ((q, 1), (kp, 2), (vp, 3)):
        _fill(t, s)
    call()
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        call()
    for rep in range(2):
        for t, s in ((q, 40 + rep), (kp, 50 + rep), (vp, 60 + rep)):
            _fill(t, s)
        o.fill_(float("nan"))
        g.replay()
        torch.cuda.synchronize()
        o_g, l_g = o.clone(), lse.clone()
        call()
        torch.cuda.synchronize()
        assert torch.isfinite(o_g.float()).all()
        assert torch.equal(o_g, o) and torch.equal(l_g, lse)
    assert rsd.attn_get_device_error() == rsd.ATTN_OK
    del g


def test_dense_prefill_replays_in_a_graph():
    """Dense: the device-built work list and its claim counter in the workspace
    are rebuilt by every replay."""
    B, S, Hq, Hkv, D = 2, 700, 8, 2, 128
    q = torch.empty((B, S, Hq, D), dtype=torch.bfloat16, device=DEV)
    k = torch.empty((B, S, Hkv, D), dtype=torch.bfloat16, device=DEV)
    v = torch.empty_like(k)
    o = torch.empty_like(q)
    lse = torch.empty((B, Hq, S), dtype=torch.float32, device=DEV)
    ws = torch.empty(rsd.attn_fwd_dense_workspace_size(B, S, Hq, Hkv), dtype=torch.uint8, device=DEV)

    def call():
        rsd.attn_fwd_dense(q, k, v, o, lse, scale=0.09, causal=True, workspace=ws)

    for t, s in ((q, 1), (k, 2), (v, 3)):
        _fill(t, s)
    call()
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        call()
    for rep in range(2):
        for t, s in ((q, 70 + rep), (k, 80 + rep), (v, 90 + rep)):
            _fill(t, s)
        o.fill_(float("nan"))
        g.replay()
        torch.cuda.synchronize()
        o_g, l_g = o.clone(), lse.clone()
        call()
        torch.cuda.synchronize()
        assert torch.isfinite(o_g.float()).all()
        assert torch.equal(o_g, o) and torch.equal(l_g, lse)
    assert rsd.attn_get_device_error() == rsd.ATTN_OK
    del g


def test_mixed_batch_with_splits_replays_in_a_graph():
    """Ragged queries over a paged cache with short rows on the split-KV decode
    kernel: work list, decode, THD merge and prefill all captured, with new
    query lengths written into the same offset table between replays (the
    short / long split is decided on the device)."""
    lens_kv = [3000, 700, 64, 2000]
    Hq, Hkv, D, ps, S = 8, 2, 128, 64, 3
    table, total = synth.page_table(lens_kv, ps, 9)
    T = 600
    q = torch.empty((T, Hq, D), dtype=torch.bfloat16, device=DEV)
    kp = torch.empty((total + 2, Hkv, ps, D), dtype=torch.bfloat16, device=DEV)
    vp = torch.empty_like(kp)
    o = torch.empty((T, Hq, D), dtype=torch.bfloat16, device=DEV)
    lse = torch.empty((T, Hq), dtype=torch.float32, device=DEV)
    cu = torch.zeros(len(lens_kv) + 1, dtype=torch.int32, device=DEV)
    pt = torch.as_tensor(table, device=DEV)
    kl = torch.as_tensor(np.asarray(lens_kv, dtype=np.int32), device=DEV)
    max_sq = 400
    ws = torch.empty(rsd.attn_fwd_paged_prefill_workspace_size(len(lens_kv), max_sq, T, Hq, Hkv, D, S),
                     dtype=torch.uint8, device=DEV)

    def call():
        rsd.attn_fwd_paged_prefill(q, kp, vp, o, lse, cu, pt, kl, max_seqlen_q=max_sq, page_size=ps,
                                   max_kv_len=max(lens_kv), scale=0.088, causal=True, workspace=ws,
                                   num_splits=S, lse_layout=rsd.ATTN_LSE_PACKED_TH)

    def set_lengths(lq):
        cu.copy_(torch.as_tensor(synth.cu_seqlens(lq), device=DEV))

    for t, s in ((q, 1), (kp, 2), (vp, 3)):
        _fill(t, s)
    set_lengths([1, 300, 4, 2])
    call()
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        call()
    for rep, lq in enumerate(([1, 300, 4, 2], [200, 1, 3, 390], [4, 4, 4, 4])):
        set_lengths(lq)
        for t, s in ((q, 110 + rep), (kp, 120 + rep), (vp, 130 + rep)):
            _fill(t, s)
        o.fill_(float("nan"))
        lse.fill_(float("nan"))
        g.replay()
        torch.cuda.synchronize()
        n = sum(lq)
        o_g, l_g = o[:n].clone(), lse[:n].clone()
        call()
        torch.cuda.synchronize()
        assert torch.isfinite(o_g.float()).all()
        assert torch.equal(o_g, o[:n]) and torch.equal(l_g, lse[:n])
    assert rsd.attn_get_device_error() == rsd.ATTN_OK
    del g
