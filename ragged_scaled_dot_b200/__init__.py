"""Python binding of libb2attn.so (forward attention for B200, sm_100a).

Argument marshalling only: every step of the computation runs in the CUDA
kernels behind the C ABI declared in ``include/b2attn.h``.  PyTorch supplies
device memory and streams.  There is no fallback: if the shared library is
missing, importing the binding's entry points raises.

Entry points keep the C names.  Tensors are torch CUDA tensors; the caller
allocates outputs and workspaces (``*_workspace_size`` tells how much).
"""
from __future__ import annotations

import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libb2attn.so")

ATTN_OK = 0
ATTN_ERR_INVALID_ARG = 1
ATTN_ERR_UNSUPPORTED = 2
ATTN_ERR_WORKSPACE = 3
ATTN_ERR_LAUNCH = 4
ATTN_ERR_DEVICE_TIMEOUT = 5
ATTN_ERR_DEVICE_INPUT = 6
ATTN_ERR_CUDA = 7
ATTN_LSE_PADDED_BSH = 0
ATTN_LSE_PACKED_TH = 1
ATTN_LSE_PACKED_HT = 2
ATTN_LSE_LOG2 = 0x100

# every symbol include/b2attn.h declares: name -> (restype, argtypes)
_I, _L, _F, _P, _Z, _U64 = (ctypes.c_int, ctypes.c_int64, ctypes.c_float, ctypes.c_void_p,
                            ctypes.c_size_t, ctypes.c_uint64)
_L2 = ctypes.c_int64 * 2
_L3 = ctypes.c_int64 * 3
SIGNATURES = {
    "attn_status_string": (ctypes.c_char_p, [_I]),
    "attn_fwd_dense": (_I, [_P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _I,
                            _L3, _L3, _L3, _L3, _F, _I, _P, _Z, _P]),
    "attn_fwd_dense_workspace_size": (_Z, [_I, _I, _I, _I]),
    "attn_fwd_ragged": (_I, [_P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _L, _L, _I, _I, _I, _I,
                             _L2, _L2, _L2, _L2, _I, _F, _I, _P, _Z, _P]),
    "attn_fwd_ragged_workspace_size": (_Z, [_I, _I, _L, _I, _I]),
    "attn_fwd_ragged_noalloc": (_I, [_P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _L, _L, _I, _I, _I, _I,
                                     _L2, _L2, _L2, _L2, _I, _F, _I, _P]),
    "attn_fwd_ragged_noalloc_max_scratch": (_Z, []),
    "attn_fwd_paged": (_I, [_P, _P, _P, _P, _P, _P, _L, _P, _I, _I, _I, _I, _I, _I, _L, _I,
                            _L2, _L2, _L3, _L3, _F, _I, _P, _Z, _P]),
    "attn_fwd_paged_kv_tables": (_I, [_P, _P, _P, _P, _P, _P, _L, _P, _L, _P, _I, _I, _I, _I, _I, _I, _L, _I,
                                      _L2, _L2, _L3, _L3, _F, _I, _P, _Z, _P]),
    "attn_fwd_paged_workspace_size": (_Z, [_I, _I, _I, _I]),
    "attn_fwd_paged_prefill": (_I, [_P, _P, _P, _P, _P, _P, _P, _L, _P, _I, _I, _L, _I, _I, _I, _I, _L, _I,
                                    _L2, _L2, _L3, _L3, _I, _F, _I, _I, _P, _Z, _P]),
    "attn_fwd_paged_prefill_kv_tables": (_I, [_P, _P, _P, _P, _P, _P, _P, _L, _P, _L, _P, _I, _I, _L, _I, _I,
                                              _I, _I, _L, _I, _L2, _L2, _L3, _L3, _I, _F, _I, _I, _P, _Z, _P]),
    "attn_fwd_paged_prefill_workspace_size": (_Z, [_I, _I, _L, _I, _I, _I, _I]),
    "attn_paged_suggest_splits": (_I, [_I, _I, _I, _I, _I, _I, _I, _I]),
    "attn_split_merge": (_I, [_P, _P, _I, _L, _I, _P, _L, _P, _P]),
    "attn_get_device_error": (_I, [_P]),
    "attn_selftest_bounded_wait": (_I, [_U64, _P]),
    "attn_selftest_exp2": (_I, [_P, _P, _L, _P]),
    "attn_selftest_page_coords": (_I, [_P, _L, _I, _L, _I, _P, _P, _L, _P, _P]),
}

_lib = None


class AttnError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {status_string(status)}")


def lib() -> ctypes.CDLL:
    """The loaded libb2attn.so.  Raises if it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(
                f"{LIB_PATH} is missing: build it with `python -m ragged_scaled_dot_b200.build` "
                "(there is no fallback implementation)")
        handle = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(handle, name)
            fn.restype = res
            fn.argtypes = args
        _lib = handle
    return _lib


def status_string(status: int) -> str:
    return lib().attn_status_string(int(status)).decode()


def _check(status: int, where: str):
    if status != ATTN_OK:
        raise AttnError(status, where)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    import torch
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _bf16(t, name):
    import torch
    if t.dtype != torch.bfloat16 or not t.is_cuda or t.stride(-1) != 1:
        raise ValueError(f"{name} must be a CUDA bf16 tensor with a contiguous last dim")


# --------------------------------------------------------------------- dense
def attn_fwd_dense_workspace_size(B, Sq, Hq, Hkv) -> int:
    return int(lib().attn_fwd_dense_workspace_size(B, Sq, Hq, Hkv))


def attn_fwd_dense(q, k, v, o, lse=None, *, scale: float, causal: bool, workspace, stream=None):
    """Dense BSHD: q [B,Sq,Hq,Dqk], k [B,Skv,Hkv,Dqk], v [B,Skv,Hkv,Dv],
    o [B,Sq,Hq,Dv] (strided views allowed), lse fp32 [B,Hq,Sq] contiguous or None.
    workspace: uint8 CUDA tensor of attn_fwd_dense_workspace_size(...) bytes."""
    for t, n in ((q, "q"), (k, "k"), (v, "v"), (o, "o")):
        _bf16(t, n)
    B, Sq, Hq, Dqk = q.shape
    _, Skv, Hkv, _ = k.shape
    Dv = v.shape[-1]
    st = lambda t: _L3(t.stride(0), t.stride(1), t.stride(2))  # noqa: E731
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(lib().attn_fwd_dense(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), B, Sq, Skv, Hq,
                                Hkv, Dqk, Dv, st(q), st(k), st(v), st(o), float(scale),
                                int(causal), _ptr(workspace), ws_bytes, _stream(stream)),
           "attn_fwd_dense")


# -------------------------------------------------------------------- ragged
def attn_fwd_ragged_workspace_size(B, max_seqlen_q, total_q, Hq, Hkv) -> int:
    return int(lib().attn_fwd_ragged_workspace_size(B, max_seqlen_q, total_q, Hq, Hkv))


def attn_fwd_ragged(q, k, v, o, lse, cu_seqlens_q, cu_seqlens_kv, *, max_seqlen_q: int,
                    max_seqlen_kv: int, scale: float, causal: bool, workspace,
                    lse_layout: int = ATTN_LSE_PADDED_BSH, total_q=None, total_kv=None,
                    stream=None):
    """Packed THD: q [T,Hq,Dqk], k/v [Tkv,Hkv,D] (token/head strides honoured),
    cu_seqlens_* int32 CUDA [B+1].  lse: fp32 [B,max_seqlen_q,Hq] (padded) or
    [T,Hq] (packed) or None.  workspace: uint8 CUDA tensor."""
    for t, n in ((q, "q"), (k, "k"), (v, "v"), (o, "o")):
        _bf16(t, n)
    B = cu_seqlens_q.numel() - 1
    Hq, Dqk = q.shape[1], q.shape[2]
    Hkv, Dv = k.shape[1], v.shape[2]
    total_q = q.shape[0] if total_q is None else total_q
    total_kv = k.shape[0] if total_kv is None else total_kv
    st = lambda t: _L2(t.stride(0), t.stride(1))  # noqa: E731
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(lib().attn_fwd_ragged(
        _ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), _ptr(cu_seqlens_q), _ptr(cu_seqlens_kv),
        B, int(max_seqlen_q), int(max_seqlen_kv), int(total_q), int(total_kv), Hq, Hkv, Dqk, Dv,
        st(q), st(k), st(v), st(o), int(lse_layout), float(scale), int(causal),
        _ptr(workspace), ws_bytes, _stream(stream)), "attn_fwd_ragged")


def attn_fwd_ragged_noalloc(q, k, v, o, lse, cu_seqlens_q, cu_seqlens_kv, *, max_seqlen_q: int,
                            max_seqlen_kv: int, scale: float, causal: bool,
                            lse_layout: int = ATTN_LSE_PADDED_BSH, total_q=None, total_kv=None,
                            stream=None):
    """attn_fwd_ragged for callers that cannot allocate device memory at call
    time (a host framework that owns every device allocation, or a serving
    loop that sizes all its buffers at start-up): the work list goes to a
    4 MiB scratch array built into the library.  Calls share that array, so
    calls that overlap on the GPU race; the first call on a device should
    come before any stream capture."""
    for t, n in ((q, "q"), (k, "k"), (v, "v"), (o, "o")):
        _bf16(t, n)
    B = cu_seqlens_q.numel() - 1
    Hq, Dqk = q.shape[1], q.shape[2]
    Hkv, Dv = k.shape[1], v.shape[2]
    total_q = q.shape[0] if total_q is None else total_q
    total_kv = k.shape[0] if total_kv is None else total_kv
    st = lambda t: _L2(t.stride(0), t.stride(1))  # noqa: E731
    _check(lib().attn_fwd_ragged_noalloc(
        _ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), _ptr(cu_seqlens_q), _ptr(cu_seqlens_kv),
        B, int(max_seqlen_q), int(max_seqlen_kv), int(total_q), int(total_kv), Hq, Hkv, Dqk, Dv,
        st(q), st(k), st(v), st(o), int(lse_layout), float(scale), int(causal), _stream(stream)),
        "attn_fwd_ragged_noalloc")


def attn_fwd_ragged_noalloc_max_scratch() -> int:
    return int(lib().attn_fwd_ragged_noalloc_max_scratch())


# --------------------------------------------------------------------- paged
def attn_fwd_paged_workspace_size(B, Hq, Dv, num_splits) -> int:
    return int(lib().attn_fwd_paged_workspace_size(B, Hq, Dv, num_splits))


def attn_paged_suggest_splits(B, Hq, Hkv, Dqk, Dv, max_kv_len, page_size, num_sms) -> int:
    return int(lib().attn_paged_suggest_splits(B, Hq, Hkv, Dqk, Dv, max_kv_len, page_size,
                                               num_sms))


def pool_strides(pool, kv_layout: str):
    """(page, slot, head) element strides of a 4D pool in HND [P,H,ps,D] or NHD [P,ps,H,D]."""
    if kv_layout == "HND":
        return _L3(pool.stride(0), pool.stride(2), pool.stride(1))
    if kv_layout == "NHD":
        return _L3(pool.stride(0), pool.stride(1), pool.stride(2))
    raise ValueError(kv_layout)


def attn_fwd_paged(q, k_pool, v_pool, o, lse, page_table, kv_lens, *, page_size: int,
                   max_kv_len: int, scale: float, num_splits: int, workspace=None,
                   kv_layout: str = "HND", stream=None):
    """Paged decode: q [B,Hq,Dqk], pools 4D in kv_layout, page_table int32 CUDA
    [B,max_pages], kv_lens int32 CUDA [B], o [B,Hq,Dv], lse fp32 [B,Hq] or None."""
    for t, n in ((q, "q"), (k_pool, "k_pool"), (v_pool, "v_pool"), (o, "o")):
        _bf16(t, n)
    B, Hq, Dqk = q.shape
    Dv = o.shape[-1]
    Hkv = k_pool.shape[1] if kv_layout == "HND" else k_pool.shape[2]
    num_pages = k_pool.shape[0]
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(lib().attn_fwd_paged(
        _ptr(q), _ptr(k_pool), _ptr(v_pool), _ptr(o), _ptr(lse), _ptr(page_table),
        int(page_table.stride(0)), _ptr(kv_lens), B, Hq, Hkv, Dqk, Dv, int(page_size),
        int(num_pages), int(max_kv_len), _L2(q.stride(0), q.stride(1)),
        _L2(o.stride(0), o.stride(1)), pool_strides(k_pool, kv_layout),
        pool_strides(v_pool, kv_layout), float(scale), int(num_splits), _ptr(workspace),
        ws_bytes, _stream(stream)), "attn_fwd_paged")


def attn_fwd_paged_kv_tables(q, k_pool, v_pool, o, lse, k_page_table, v_page_table, kv_lens, *,
                             page_size: int, max_kv_len: int, scale: float, num_splits: int,
                             workspace=None, kv_layout: str = "HND", stream=None):
    """attn_fwd_paged with independent K and V page tables (int32 CUDA
    [B, max_pages] each): key rows through k_page_table, value rows through
    v_page_table."""
    for t, n in ((q, "q"), (k_pool, "k_pool"), (v_pool, "v_pool"), (o, "o")):
        _bf16(t, n)
    B, Hq, Dqk = q.shape
    Dv = o.shape[-1]
    Hkv = k_pool.shape[1] if kv_layout == "HND" else k_pool.shape[2]
    num_pages = min(k_pool.shape[0], v_pool.shape[0])
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(lib().attn_fwd_paged_kv_tables(
        _ptr(q), _ptr(k_pool), _ptr(v_pool), _ptr(o), _ptr(lse), _ptr(k_page_table),
        int(k_page_table.stride(0)), _ptr(v_page_table), int(v_page_table.stride(0)), _ptr(kv_lens),
        B, Hq, Hkv, Dqk, Dv, int(page_size), int(num_pages), int(max_kv_len), _L2(q.stride(0), q.stride(1)),
        _L2(o.stride(0), o.stride(1)), pool_strides(k_pool, kv_layout), pool_strides(v_pool, kv_layout),
        float(scale), int(num_splits), _ptr(workspace), ws_bytes, _stream(stream)), "attn_fwd_paged_kv_tables")


def attn_fwd_paged_prefill_workspace_size(B, max_seqlen_q, total_q, Hq, Hkv, D=128, num_splits=1) -> int:
    return int(lib().attn_fwd_paged_prefill_workspace_size(B, max_seqlen_q, total_q, Hq, Hkv, D, num_splits))


def attn_fwd_paged_prefill(q, k_pool, v_pool, o, lse, cu_seqlens_q, page_table, kv_lens, *,
                           max_seqlen_q: int, page_size: int, max_kv_len: int, scale: float,
                           causal: bool, workspace, num_splits: int = 1,
                           lse_layout: int = ATTN_LSE_PADDED_BSH, kv_layout: str = "HND", total_q=None,
                           stream=None):
    """Ragged queries over a paged cache (chunked prefill, decode and multi-token
    decode rows): q [T,Hq,D] packed by cu_seqlens_q (int32 CUDA [B+1]); sequence b's
    queries are the last Lq_b positions of its kv_lens[b] keys (bottom-right causal).
    Pools 4D in kv_layout, page_table int32 CUDA [B,max_pages], o [T,Hq,D], lse as in
    attn_fwd_ragged.  Sequences of at most 4 queries run split-KV with num_splits
    splits.  workspace: uint8 CUDA tensor of attn_fwd_paged_prefill_workspace_size(...)."""
    for t, n in ((q, "q"), (k_pool, "k_pool"), (v_pool, "v_pool"), (o, "o")):
        _bf16(t, n)
    B = cu_seqlens_q.numel() - 1
    Hq, D = q.shape[1], q.shape[2]
    Hkv = k_pool.shape[1] if kv_layout == "HND" else k_pool.shape[2]
    num_pages = k_pool.shape[0]
    total_q = q.shape[0] if total_q is None else total_q
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(lib().attn_fwd_paged_prefill(
        _ptr(q), _ptr(k_pool), _ptr(v_pool), _ptr(o), _ptr(lse), _ptr(cu_seqlens_q), _ptr(page_table),
        int(page_table.stride(0)), _ptr(kv_lens), B, int(max_seqlen_q), int(total_q), Hq, Hkv, D,
        int(page_size), int(num_pages), int(max_kv_len), _L2(q.stride(0), q.stride(1)),
        _L2(o.stride(0), o.stride(1)), pool_strides(k_pool, kv_layout), pool_strides(v_pool, kv_layout),
        int(lse_layout), float(scale), int(causal), int(num_splits), _ptr(workspace), ws_bytes,
        _stream(stream)), "attn_fwd_paged_prefill")


def attn_fwd_paged_prefill_kv_tables(q, k_pool, v_pool, o, lse, cu_seqlens_q, k_page_table, v_page_table,
                                     kv_lens, *, max_seqlen_q: int, page_size: int, max_kv_len: int,
                                     scale: float, causal: bool, workspace, num_splits: int = 1,
                                     lse_layout: int = ATTN_LSE_PADDED_BSH, kv_layout: str = "HND",
                                     total_q=None, stream=None):
    """attn_fwd_paged_prefill with independent K and V page tables."""
    for t, n in ((q, "q"), (k_pool, "k_pool"), (v_pool, "v_pool"), (o, "o")):
        _bf16(t, n)
    B = cu_seqlens_q.numel() - 1
    Hq, D = q.shape[1], q.shape[2]
    Hkv = k_pool.shape[1] if kv_layout == "HND" else k_pool.shape[2]
    num_pages = min(k_pool.shape[0], v_pool.shape[0])
    total_q = q.shape[0] if total_q is None else total_q
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(lib().attn_fwd_paged_prefill_kv_tables(
        _ptr(q), _ptr(k_pool), _ptr(v_pool), _ptr(o), _ptr(lse), _ptr(cu_seqlens_q), _ptr(k_page_table),
        int(k_page_table.stride(0)), _ptr(v_page_table), int(v_page_table.stride(0)), _ptr(kv_lens), B,
        int(max_seqlen_q), int(total_q), Hq, Hkv, D, int(page_size), int(num_pages), int(max_kv_len),
        _L2(q.stride(0), q.stride(1)), _L2(o.stride(0), o.stride(1)), pool_strides(k_pool, kv_layout),
        pool_strides(v_pool, kv_layout), int(lse_layout), float(scale), int(causal), int(num_splits),
        _ptr(workspace), ws_bytes, _stream(stream)), "attn_fwd_paged_prefill_kv_tables")


# --------------------------------------------------------------------- merge
def attn_split_merge(o_part, lse_part, o, lse=None, *, stream=None):
    """o_part fp32 [S,R,Dv], lse_part fp32 [S,R] (contiguous), o bf16 [R,Dv]
    (row stride honoured), lse fp32 [R] or None."""
    S, R, Dv = o_part.shape
    _check(lib().attn_split_merge(_ptr(o_part), _ptr(lse_part), S, R, Dv, _ptr(o),
                                  int(o.stride(0)), _ptr(lse), _stream(stream)),
           "attn_split_merge")


# --------------------------------------------------------------- diagnostics
def attn_get_device_error(stream=None) -> int:
    return int(lib().attn_get_device_error(_stream(stream)))


def attn_selftest_bounded_wait(timeout_ns: int, stream=None):
    _check(lib().attn_selftest_bounded_wait(int(timeout_ns), _stream(stream)),
           "attn_selftest_bounded_wait")


def attn_selftest_exp2(t, y, stream=None):
    """y = 2**t through the prefill softmax's FMA-pipe exponential (fp32 CUDA tensors)."""
    _check(lib().attn_selftest_exp2(_ptr(t), _ptr(y), int(t.numel()), _stream(stream)),
           "attn_selftest_exp2")


def attn_selftest_page_coords(page_table, b_idx, t_idx, out, *, page_size: int, num_pages: int,
                              groups_per_page: int, stream=None):
    """(page, row, 8-row group) of sampled logical keys, as the paged producers
    compute them: page_table int32 CUDA [B, max_pages], b_idx / t_idx int32 CUDA [n],
    out int64 CUDA [n, 3]."""
    _check(lib().attn_selftest_page_coords(_ptr(page_table), int(page_table.stride(0)), int(page_size),
                                           int(num_pages), int(groups_per_page), _ptr(b_idx), _ptr(t_idx),
                                           int(b_idx.numel()), _ptr(out), _stream(stream)),
           "attn_selftest_page_coords")
