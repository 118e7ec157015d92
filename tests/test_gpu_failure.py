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
