"""Prefill (dense BSHD and ragged THD) on the GPU vs the fp64 oracle, plus the
invariants that pin the kernel: causality, determinism, ragged == dense,
GQA == replicated MHA, strided and gapped views, NaN tails, every LSE layout
in both bases."""
import numpy as np
import pytest
import torch

import ragged_scaled_dot_b200 as rsd
import synth
from gpu_util import (LOG2E, assert_lse_close, assert_o_close, bits, check_dense, check_ragged,
                      dense_gpu, gather_ragged, orc, ragged_gpu, ragged_rows_all)

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _ragged_inputs(lq, lkv, Hq, Hkv, D, seed, dev=DEV, pad_q=0, pad_kv=0):
    cu_q = synth.cu_seqlens(lq)
    cu_kv = synth.cu_seqlens(lkv)
    Tq, Tk = int(cu_q[-1]), int(cu_kv[-1])
    q = synth.normal_bf16((Tq + pad_q, Hq, D), seed, "cpu").to(dev)
    k = synth.normal_bf16((Tk + pad_kv, Hkv, D), seed + 1, "cpu").to(dev)
    v = synth.normal_bf16((Tk + pad_kv, Hkv, D), seed + 2, "cpu").to(dev)
    return q, k, v, cu_q, cu_kv


def test_tiny_ragged_workload_full_oracle():
    """The tiny ragged workload (lengths {37, 64}, GQA 4/1, D 64, causal,
    scale 1/8): every row against the oracle; padded LSE rows past each
    sequence stay -inf."""
    w = synth.WORKLOADS["tiny_ragged"]
    q, k, v, cu = synth.make_ragged(w, "cpu")
    q, k, v = q.to(DEV), k.to(DEV), v.to(DEV)
    o, lse, errs = check_ragged(q, k, v, cu, cu, w.scale, True, where="tiny_ragged")
    for b, L in enumerate(w.lengths):
        assert torch.all(lse[b, L:] == -float("inf"))


RAGGED_CASES = [
    # (lq, lkv, Hq, Hkv, D, causal)
    ([1, 130, 300, 0, 257], None, 8, 2, 128, True),
    ([128, 129, 255, 256, 7], None, 4, 1, 128, False),
    ([5, 200, 64], [300, 200, 1000], 4, 2, 128, True),     # Lq < Lkv: bottom-right diagonal
    ([40, 3], [10, 0], 2, 1, 128, True),                    # Lq > Lkv and an empty KV
    ([37, 64, 1, 500], None, 6, 2, 64, True),               # D = 64, G = 3 (odd: one head per item)
    ([300, 2], None, 3, 3, 128, True),                      # MHA
]


@pytest.mark.parametrize("lq,lkv,Hq,Hkv,D,causal", RAGGED_CASES)
def test_ragged_small_cases(lq, lkv, Hq, Hkv, D, causal):
    lkv = lq if lkv is None else lkv
    q, k, v, cu_q, cu_kv = _ragged_inputs(lq, lkv, Hq, Hkv, D, seed=len(lq) * 7 + D)
    check_ragged(q, k, v, cu_q, cu_kv, 1.0 / np.sqrt(D), causal, where=f"ragged {lq} {lkv}")


def test_ragged_packed_lse_layout():
    lq = [100, 3, 260]
    q, k, v, cu_q, cu_kv = _ragged_inputs(lq, lq, 4, 2, 128, seed=5)
    check_ragged(q, k, v, cu_q, cu_kv, 0.1, True, lse_layout=rsd.ATTN_LSE_PACKED_TH,
                 where="packed LSE")


@pytest.mark.parametrize("layout", ["PADDED_BSH", "PACKED_TH", "PACKED_HT"])
@pytest.mark.parametrize("log2", [False, True])
def test_ragged_lse_layouts_and_base(layout, log2):
    """Every LSE layout (padded per batch, token-major, head-major [Hq, total_q])
    in natural log and in base 2 (stats_use_log2): base 2 is the natural LSE
    times log2(e), -inf rows stay -inf, padded rows past a sequence stay -inf."""
    lq, lkv = [100, 3, 260, 0, 40], [100, 500, 260, 7, 0]
    q, k, v, cu_q, cu_kv = _ragged_inputs(lq, lkv, 4, 2, 128, seed=9)
    flag = rsd.ATTN_LSE_LOG2 if log2 else 0
    lay = getattr(rsd, "ATTN_LSE_" + layout) | flag
    o, lse, _ = check_ragged(q, k, v, cu_q, cu_kv, 0.1, True, lse_layout=lay, where=f"LSE {layout} log2={log2}")
    if layout == "PADDED_BSH":
        for b, L in enumerate(lq):
            assert torch.all(lse[b, L:] == -float("inf"))
    # the same call in the other base: same O bits, LSE related by log2(e) up to fp32 rounding
    o2, lse2 = ragged_gpu(q, k, v, cu_q, cu_kv, max(lq), max(lkv), 0.1, True,
                          lse_layout=getattr(rsd, "ATTN_LSE_" + layout) | (flag ^ rsd.ATTN_LSE_LOG2))
    assert torch.equal(o, o2)
    nat, b2 = (lse2, lse) if log2 else (lse, lse2)
    fin = torch.isfinite(nat)
    assert torch.equal(fin, torch.isfinite(b2)) and torch.all(b2[~fin] == nat[~fin])
    assert torch.allclose(b2[fin].double(), nat[fin].double() * LOG2E, rtol=2e-6, atol=2e-6)


def test_ragged_gapped_token_and_head_strides():
    """Q, K, V and O as views with gaps on both THD axes (token stride larger
    than heads x D, head stride larger than D, a nonzero base offset) are read
    and written in place; the gaps are never touched."""
    lq, lkv = [130, 5, 257], [200, 5, 257]
    Hq, Hkv, D = 4, 2, 128
    cu_q = np.concatenate([[0], np.cumsum(lq)]).astype(np.int32)
    cu_kv = np.concatenate([[0], np.cumsum(lkv)]).astype(np.int32)
    Tq, Tk = int(cu_q[-1]), int(cu_kv[-1])
    qb = synth.normal_bf16((Tq, Hq + 3, D), 31, "cpu").to(DEV)
    kb = synth.normal_bf16((Tk, 2 * Hkv, D), 32, "cpu").to(DEV)
    vb = synth.normal_bf16((Tk, Hkv, 2 * D), 33, "cpu").to(DEV)
    q = qb[:, 1:Hq + 1, :]              # token gap 3 heads, base offset one head
    k = kb[:, ::2, :]                   # head stride 2 D
    v = vb[:, :, D:]                    # head stride 2 D, base offset D
    ob = torch.full((Tq, Hq, 2 * D), 7.0, dtype=torch.bfloat16, device=DEV)
    o = ob[:, :, :D]
    lse = torch.full((len(lq), max(lq), Hq), float("nan"), dtype=torch.float32, device=DEV)
    ws = torch.empty(rsd.attn_fwd_ragged_workspace_size(len(lq), max(lq), Tq, Hq, Hkv), dtype=torch.uint8,
                     device=DEV)
    rsd.attn_fwd_ragged(q, k, v, o, lse, torch.as_tensor(cu_q, device=DEV), torch.as_tensor(cu_kv, device=DEV),
                        max_seqlen_q=max(lq), max_seqlen_kv=max(lkv), scale=0.1, causal=True, workspace=ws)
    torch.cuda.synchronize()
    assert rsd.attn_get_device_error() == rsd.ATTN_OK
    assert torch.all(ob[:, :, D:] == 7.0)  # the gaps of O are left alone
    rows = ragged_rows_all(cu_q, Hq)
    o_ref, l_ref = orc().attn_ragged_rows(bits(q), bits(k), bits(v), cu_q, cu_kv, Hq, Hkv, 0.1, True, rows)
    og, lg = gather_ragged(o, lse, cu_q, rows)
    assert_o_close(og, o_ref, "gapped strides")
    assert_lse_close(lg, l_ref, "gapped strides")


def test_ragged_scale_zero_and_negative():
    """scale = 0 is honoured (uniform weights: O = mean of visible V, LSE =
    ln(count)); a negative scale is a valid input."""
    lq = [70, 190]
    q, k, v, cu_q, cu_kv = _ragged_inputs(lq, lq, 4, 1, 128, seed=9)
    o, lse, _ = check_ragged(q, k, v, cu_q, cu_kv, 0.0, True, where="scale 0")
    # LSE = ln(i + 1) exactly up to fp32 rounding for the causal diagonal
    for b, L in enumerate(lq):
        want = np.log(np.arange(1, L + 1))
        got = lse[b, :L, 0].cpu().numpy()
        assert np.max(np.abs(got - want)) < 1e-5
    check_ragged(q, k, v, cu_q, cu_kv, -0.09, True, where="negative scale")


def test_ragged_nan_tail_past_total():
    """Values past total_q / total_kv (here NaN) are never read: outputs are
    finite and identical to a run on clean buffers."""
    lq = [77, 129]
    q, k, v, cu_q, cu_kv = _ragged_inputs(lq, lq, 4, 2, 128, seed=13, pad_q=64, pad_kv=200)
    T = int(cu_q[-1])
    qn, kn, vn = q.clone(), k.clone(), v.clone()
    qn[T:] = float("nan")
    kn[T:] = float("nan")
    vn[T:] = float("nan")
    o1, l1, _ = check_ragged(q, k, v, cu_q, cu_kv, 0.08, True, total_q=T, total_kv=T, where="clean")
    o2, l2, _ = check_ragged(qn, kn, vn, cu_q, cu_kv, 0.08, True, total_q=T, total_kv=T, where="nan tail")
    assert torch.equal(o1[:T], o2[:T]) and torch.equal(l1, l2)


def test_ragged_equals_dense_bitwise():
    """A ragged batch of equal lengths equals the dense layout bit for bit."""
    B, S, Hq, Hkv, D = 3, 300, 8, 2, 128
    qd = synth.normal_bf16((B, S, Hq, D), 21, "cpu").to(DEV)
    kd = synth.normal_bf16((B, S, Hkv, D), 22, "cpu").to(DEV)
    vd = synth.normal_bf16((B, S, Hkv, D), 23, "cpu").to(DEV)
    od, ld = dense_gpu(qd, kd, vd, 0.09, True)
    cu = synth.cu_seqlens([S] * B)
    orr, lr = ragged_gpu(qd.reshape(B * S, Hq, D), kd.reshape(B * S, Hkv, D), vd.reshape(B * S, Hkv, D),
                         cu, cu, S, S, 0.09, True)
    assert torch.equal(od.reshape(B * S, Hq, D), orr)
    assert torch.equal(ld.permute(0, 2, 1), lr)


def test_ragged_determinism_and_sequence_permutation():
    lq = [300, 45, 513]
    q, k, v, cu_q, cu_kv = _ragged_inputs(lq, lq, 8, 2, 128, seed=31)
    o1, l1 = ragged_gpu(q, k, v, cu_q, cu_kv, 513, 513, 0.1, True)
    o2, l2 = ragged_gpu(q, k, v, cu_q, cu_kv, 513, 513, 0.1, True)
    assert torch.equal(o1, o2) and torch.equal(l1, l2)
    # reversing the sequence order permutes the outputs and changes nothing else
    perm = [2, 1, 0]
    pieces = lambda t, cu: [t[cu[b]:cu[b + 1]] for b in range(len(lq))]  # noqa: E731
    qp = torch.cat([pieces(q, cu_q)[b] for b in perm])
    kp = torch.cat([pieces(k, cu_kv)[b] for b in perm])
    vp = torch.cat([pieces(v, cu_kv)[b] for b in perm])
    cu_p = synth.cu_seqlens([lq[b] for b in perm])
    o3, l3 = ragged_gpu(qp, kp, vp, cu_p, cu_p, 513, 513, 0.1, True)
    for new_b, b in enumerate(perm):
        assert torch.equal(o3[cu_p[new_b]:cu_p[new_b + 1]], o1[cu_q[b]:cu_q[b + 1]])
        assert torch.equal(l3[new_b], l1[b])


def test_causality_perturbation():
    """Changing keys/values after position j leaves rows i < j bit-identical."""
    lq = [400]
    q, k, v, cu_q, cu_kv = _ragged_inputs(lq, lq, 4, 2, 128, seed=41)
    o1, l1 = ragged_gpu(q, k, v, cu_q, cu_kv, 400, 400, 0.1, True)
    j = 250
    k2, v2 = k.clone(), v.clone()
    k2[j:] = synth.normal_bf16(k2[j:].shape, 99, "cpu").to(DEV)
    v2[j:] = synth.normal_bf16(v2[j:].shape, 98, "cpu").to(DEV)
    o2, l2 = ragged_gpu(q, k2, v2, cu_q, cu_kv, 400, 400, 0.1, True)
    assert torch.equal(o1[:j], o2[:j]) and torch.equal(l1[:, :j], l2[:, :j])
    assert not torch.equal(o1[j:], o2[j:])


def test_gqa_equals_replicated_mha_bitwise():
    lq = [200, 77]
    q, k, v, cu_q, cu_kv = _ragged_inputs(lq, lq, 8, 2, 128, seed=51)
    o1, l1 = ragged_gpu(q, k, v, cu_q, cu_kv, 200, 200, 0.1, True)
    o2, l2 = ragged_gpu(q, k.repeat_interleave(4, dim=1), v.repeat_interleave(4, dim=1), cu_q, cu_kv,
                        200, 200, 0.1, True)
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


DENSE_CASES = [
    # (B, Sq, Skv, Hq, Hkv, D, causal)
    (2, 257, 257, 8, 2, 128, True),
    (2, 257, 257, 8, 2, 128, False),
    (1, 100, 333, 4, 4, 128, True),
    (3, 64, 64, 4, 1, 64, True),
    (1, 1, 700, 16, 2, 128, True),
]


@pytest.mark.parametrize("B,Sq,Skv,Hq,Hkv,D,causal", DENSE_CASES)
def test_dense_small_cases(B, Sq, Skv, Hq, Hkv, D, causal):
    q = synth.normal_bf16((B, Sq, Hq, D), 61, "cpu").to(DEV)
    k = synth.normal_bf16((B, Skv, Hkv, D), 62, "cpu").to(DEV)
    v = synth.normal_bf16((B, Skv, Hkv, D), 63, "cpu").to(DEV)
    check_dense(q, k, v, 1.0 / np.sqrt(D), causal, where=f"dense {B} {Sq} {Skv}")


def test_dense_strided_views_of_fused_qkv():
    """Q, K, V as zero-copy slices of one fused projection [B, S, Hq+2Hkv, D]."""
    B, S, Hq, Hkv, D = 2, 190, 8, 2, 128
    qkv = synth.normal_bf16((B, S, Hq + 2 * Hkv, D), 71, "cpu").to(DEV)
    q, k, v = qkv[:, :, :Hq], qkv[:, :, Hq:Hq + Hkv], qkv[:, :, Hq + Hkv:]
    check_dense(q, k, v, 0.1, True, where="fused qkv views")


@pytest.mark.parametrize("scale", [0.3, -0.3])
@pytest.mark.parametrize("causal", [True, False])
def test_ragged_running_max_jumps(scale, causal):
    """Key rows scaled by 1 + 3 t / L along each sequence make the scores grow
    (or, with a negative scale, fall) from tile to tile, so the running row
    maximum moves by more than 2^8 many times: the O rescale and the recompute
    of a tile against a new maximum both run.  V stays N(0,1)."""
    lens = [1500, 700, 130]
    Hq, Hkv, D = 4, 2, 128
    q, k, v, cu_q, cu_kv = _ragged_inputs(lens, lens, Hq, Hkv, D, seed=89)
    f = torch.cat([1.0 + 3.0 * torch.arange(L, dtype=torch.float32) / L for L in lens]).to(DEV)
    k = (k.float() * f[:, None, None]).to(torch.bfloat16)
    check_ragged(q, k, v, cu_q, cu_kv, scale, causal, where=f"running max jumps scale={scale} causal={causal}")
