"""Failure detection without a GPU fault: bounded waits that run out record a
status and return, invalid device-side tables are reported and skipped, and
the context stays usable afterwards."""
import numpy as np
import pytest
import torch

import ragged_scaled_dot_b200 as rsd
import synth
from gpu_util import check_ragged, paged_gpu, ragged_gpu

pytestmark = pytest.mark.gpu
DEV = "cuda"


def test_bounded_wait_times_out_and_context_survives():
    assert rsd.attn_get_device_error() == rsd.ATTN_OK
    rsd.attn_selftest_bounded_wait(50_000_000)  # 50 ms on a barrier nothing signals
    assert rsd.attn_get_device_error() == rsd.ATTN_ERR_DEVICE_TIMEOUT
    assert rsd.attn_get_device_error() == rsd.ATTN_OK  # reading clears it
    # the context still computes correctly
    lq = [100, 37]
    cu = synth.cu_seqlens(lq)
    q = synth.normal_bf16((137, 4, 128), 1, "cpu").to(DEV)
    k = synth.normal_bf16((137, 1, 128), 2, "cpu").to(DEV)
    v = synth.normal_bf16((137, 1, 128), 3, "cpu").to(DEV)
    check_ragged(q, k, v, cu, cu, 0.1, True, where="after timeout")
    assert rsd.attn_get_device_error() == rsd.ATTN_OK


def test_inconsistent_offsets_are_reported_not_faulted():
    lq = [100, 37]
    q = synth.normal_bf16((137, 4, 128), 1, "cpu").to(DEV)
    k = synth.normal_bf16((137, 1, 128), 2, "cpu").to(DEV)
    v = synth.normal_bf16((137, 1, 128), 3, "cpu").to(DEV)
    bad = np.array([0, 100, 90], dtype=np.int32)  # decreasing: second sequence invalid
    rsd.attn_get_device_error()
    o, lse = ragged_gpu(q, k, v, bad, bad, 100, 100, 0.1, True, o_fill=0.0)
    assert rsd.attn_get_device_error() == rsd.ATTN_ERR_DEVICE_INPUT
    # the valid first sequence is still computed, the invalid one is skipped
    assert torch.isfinite(o[:100].float()).all()
    # a length beyond the declared maximum is reported too
    cu = synth.cu_seqlens(lq)
    ragged_gpu(q, k, v, cu, cu, 64, 64, 0.1, True)
    assert rsd.attn_get_device_error() == rsd.ATTN_ERR_DEVICE_INPUT


def test_out_of_range_page_id_is_reported():
    lens = [130]
    ps = 64
    table, total = synth.page_table(lens, ps, 5)
    q = synth.normal_bf16((1, 8, 128), 1, "cpu").to(DEV)
    k = synth.normal_bf16((total, 1, ps, 128), 2, "cpu").to(DEV)
    table = table.copy()
    table[0, 1] = total + 1000  # past the pool: TMA reads zeros, status records it
    rsd.attn_get_device_error()
    o, lse = paged_gpu(q, k, k, table, np.array(lens, np.int32), ps, 0.1, 1)
    assert rsd.attn_get_device_error() == rsd.ATTN_ERR_DEVICE_INPUT
    assert torch.isfinite(o.float()).all()


def test_fma_pipe_exp2_error_bound():
    """The softmax's FMA-pipe exponential against 2^t in float64: relative error
    <= 1.1e-4 on the range the softmax uses ([-125, 8]), exact at integers
    (so a constant score row sums to an exact count), monotone input clamp."""
    t = torch.cat([torch.linspace(-125.0, 8.0, 1_000_001), torch.arange(-125, 9, dtype=torch.float32),
                   torch.tensor([-200.0, -1e30])]).to(DEV)
    y = torch.empty_like(t)
    rsd.attn_selftest_exp2(t, y)
    torch.cuda.synchronize()
    tt = t.double().cpu().numpy()
    yy = y.double().cpu().numpy()
    ref = np.exp2(np.maximum(tt, -125.0))
    rel = np.abs(yy - ref) / ref
    assert rel.max() <= 1.1e-4, rel.max()
    ints = np.arange(-125, 9)
    n0 = 1_000_001
    assert np.array_equal(yy[n0:n0 + len(ints)], np.exp2(ints.astype(np.float64)))
