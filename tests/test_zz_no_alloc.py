"""attn_fwd_ragged_noalloc: the ragged prefill for callers that cannot
allocate device memory when they call (a host framework that owns every device
allocation, or a serving loop that sizes all its buffers at start-up).  Its
work list lives in a fixed-size array built into the library instead of a
caller workspace.

Checked through the C ABI against the regular attn_fwd_ragged on two calls in
a row (two different problems, so the second call must not see the first
call's leftovers in the shared array), with the tolerance the other tests use,
and directly against the fp64 oracle; the device's free memory and torch's
allocator must not move across a call.  This file is collected last and needs
nothing from the other test files.
"""
import numpy as np
import pytest
import torch

import oracle
import ragged_scaled_dot_b200 as rsd
import synth
from gpu_util import LSE_ATOL, O_ATOL, O_RTOL

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _problem(lengths, Hq, Hkv, D, seed):
    cu = synth.cu_seqlens(lengths)
    T = int(cu[-1])
    q = synth.normal_bf16((T, Hq, D), seed, "cpu").to(DEV)
    k = synth.normal_bf16((T, Hkv, D), seed + 1, "cpu").to(DEV)
    v = synth.normal_bf16((T, Hkv, D), seed + 2, "cpu").to(DEV)
    return q, k, v, torch.as_tensor(cu, device=DEV), int(max(lengths))


def _outputs(q, B, smax):
    o = torch.full_like(q, float("nan"))
    lse = torch.full((B, smax, q.shape[1]), float("nan"), dtype=torch.float32, device=DEV)
    return o, lse


def _regular(q, k, v, cu, smax, scale):
    B = cu.numel() - 1
    o, lse = _outputs(q, B, smax)
    ws = torch.empty(rsd.attn_fwd_ragged_workspace_size(B, smax, q.shape[0], q.shape[1], k.shape[1]),
                     dtype=torch.uint8, device=DEV)
    rsd.attn_fwd_ragged(q, k, v, o, lse, cu, cu, max_seqlen_q=smax, max_seqlen_kv=smax, scale=scale,
                        causal=True, workspace=ws)
    return o, lse


def _noalloc(q, k, v, cu, smax, scale, o, lse):
    rsd.attn_fwd_ragged_noalloc(q, k, v, o, lse, cu, cu, max_seqlen_q=smax, max_seqlen_kv=smax,
                                scale=scale, causal=True)


def _close_o(o, o_ref, where):
    err = (o.float() - o_ref.float()).abs()
    assert torch.isfinite(o.float()).all(), where
    assert bool((err <= O_ATOL + O_RTOL * o_ref.float().abs()).all()), f"{where}: O max err {err.max().item()}"


def test_noalloc_matches_regular_entry_point_on_two_calls_in_a_row():
    assert rsd.attn_fwd_ragged_noalloc_max_scratch() == 4 << 20
    problems = [
        ([300, 45, 513, 1, 128], 8, 2, 128, 11, 0.09),   # first call
        ([37, 64, 700], 4, 1, 64, 23, 0.125),            # second call: other shapes, fewer items
    ]
    refs = [(_regular(*_problem(L, Hq, Hkv, D, s)[:4], max(L), sc)) for L, Hq, Hkv, D, s, sc in problems]
    torch.cuda.synchronize()
    orc = oracle.default()
    for (L, Hq, Hkv, D, s, sc), (o_ref, l_ref) in zip(problems, refs):
        q, k, v, cu, smax = _problem(L, Hq, Hkv, D, s)
        o, lse = _outputs(q, cu.numel() - 1, smax)
        torch.cuda.synchronize()
        free0, used0 = torch.cuda.mem_get_info()[0], torch.cuda.memory_allocated()
        _noalloc(q, k, v, cu, smax, sc, o, lse)
        torch.cuda.synchronize()
        # the call allocated nothing: the device's free bytes and torch's allocator are unchanged
        assert torch.cuda.mem_get_info()[0] == free0 and torch.cuda.memory_allocated() == used0
        _close_o(o, o_ref, f"noalloc {L}")
        fin = torch.isfinite(l_ref)
        assert torch.equal(torch.isfinite(lse), fin)
        assert (lse[fin] - l_ref[fin]).abs().max().item() <= LSE_ATOL
        assert torch.all(lse[~fin] == -float("inf"))
        # and on its own against the fp64 oracle, every row of every head
        cu_h = cu.cpu().numpy()
        rows = np.array([(b, h, i) for b, n in enumerate(L) for h in range(Hq) for i in range(n)], dtype=np.int32)
        oo, lo = orc.attn_ragged_rows(synth.bf16_bits(q), synth.bf16_bits(k), synth.bf16_bits(v), cu_h, cu_h,
                                      Hq, Hkv, sc, True, rows)
        tok = torch.as_tensor(cu_h[rows[:, 0]].astype(np.int64) + rows[:, 2], device=DEV)
        hh = torch.as_tensor(rows[:, 1].astype(np.int64), device=DEV)
        og = o[tok, hh].double().cpu().numpy()
        assert np.all(np.abs(og - oo) <= O_ATOL + O_RTOL * np.abs(oo)), f"noalloc {L} vs oracle"
        lg = lse[torch.as_tensor(rows[:, 0].astype(np.int64), device=DEV),
                 torch.as_tensor(rows[:, 2].astype(np.int64), device=DEV), hh].double().cpu().numpy()
        assert np.max(np.abs(lg - lo)) <= LSE_ATOL, f"noalloc {L} LSE vs oracle"
    assert rsd.attn_get_device_error() == rsd.ATTN_OK


def test_noalloc_rejects_capacities_beyond_its_scratch():
    # 64 sequences of up to 2^20 tokens, 64 query heads: the work list would
    # need far more than 4 MiB, so the call is refused before any launch.
    B, smax, T, Hq, Hkv = 64, 1 << 20, 64 << 20, 64, 8
    assert rsd.attn_fwd_ragged_workspace_size(B, smax, T, Hq, Hkv) > rsd.attn_fwd_ragged_noalloc_max_scratch()
    q = torch.empty((8, Hq, 128), dtype=torch.bfloat16, device=DEV)
    k = torch.empty((8, Hkv, 128), dtype=torch.bfloat16, device=DEV)
    cu = torch.zeros(B + 1, dtype=torch.int32, device=DEV)
    with pytest.raises(rsd.AttnError) as e:
        rsd.attn_fwd_ragged_noalloc(q, k, k, q, None, cu, cu, max_seqlen_q=smax, max_seqlen_kv=smax,
                                    scale=0.1, causal=True, total_q=T, total_kv=T)
    assert e.value.status == rsd.ATTN_ERR_WORKSPACE
