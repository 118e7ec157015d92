"""fp64 CPU oracle for forward scaled-dot-product attention.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this package.  The CUDA library never
calls it and shares no code with it; the only thing both sides consume is the
seeded input from ``synth``.

The arithmetic lives in ``attn_oracle.c`` (plain C, fp64, OpenMP over rows);
this module only marshals numpy arrays to it.  Every function takes bf16 inputs
as ``numpy.uint16`` bit patterns and returns float64 results.

Parity status: every entry point here is pinned by ``tests/test_oracle_pins.py``
(closed forms, brute force on tiny inputs, a library routine, and invariants of
the mathematics), and ``tests/test_oracle_mutants.py`` shows that plausible
mistakes planted in a copy of the C source fail those pins.  No entry point is
"parity unpinned".
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
SOURCE = os.path.join(_HERE, "attn_oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")


def compile_source(src: str, out: str) -> str:
    """Compile an oracle C source with gcc (fp64, no fast-math) into a shared object."""
    tmp = out + f".tmp{os.getpid()}"
    subprocess.check_call(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared",
                           "-std=c11", "-o", tmp, src, "-lm"])
    os.replace(tmp, out)
    return out


def build(force: bool = False) -> str:
    """Build liboracle.so next to its source if it is missing or stale."""
    stale = (not os.path.exists(_LIB_PATH)) or (
        os.path.getmtime(_LIB_PATH) < os.path.getmtime(SOURCE))
    if force or stale:
        compile_source(SOURCE, _LIB_PATH)
    return _LIB_PATH


def _p(a):
    return a.ctypes.data_as(ctypes.c_void_p)


def _u16(a):
    a = np.ascontiguousarray(a)
    assert a.dtype == np.uint16, a.dtype
    return a


def _i32(a):
    return np.ascontiguousarray(np.asarray(a, dtype=np.int32))


def _i64(a):
    return np.ascontiguousarray(np.asarray(a, dtype=np.int64))


def split_ranges(kv_len: int, page_size: int, num_splits: int):
    """Key range [lo, hi) of every split of one sequence.

    Reading taken where the pages are silent: the partition is page-granular,
    each split takes ceil(n_pages / num_splits) consecutive pages, trailing
    splits may be empty.
    """
    n_pages = -(-kv_len // page_size)
    pps = -(-n_pages // num_splits) if n_pages > 0 else 0
    out = []
    for s in range(num_splits):
        lo = min(s * pps * page_size, kv_len)
        hi = min((s + 1) * pps * page_size, kv_len)
        out.append((lo, hi))
    return out


class Oracle:
    """The oracle bound to one compiled library (the default build, or a test build)."""

    def __init__(self, lib_path: str):
        self._lib = ctypes.CDLL(lib_path)
        self._lib.oracle_num_threads.restype = ctypes.c_int

    def num_threads(self) -> int:
        return int(self._lib.oracle_num_threads())

    def set_num_threads(self, n: int) -> None:
        """Threads the oracle's OpenMP loops use from now on (threading only)."""
        self._lib.oracle_set_num_threads(ctypes.c_int(int(n)))

    def attn_ragged_rows(self, q, k, v, cu_q, cu_kv, Hq, Hkv, scale, causal, rows,
                         q_strides=None, k_strides=None, v_strides=None):
        """Rows (b, h, i) of ragged/THD attention, i the query index in its sequence.

        q, k, v: uint16 bf16 bits, [T, H, D] arrays (or flat buffers with explicit
        (token, head) element strides).  Returns (o [n, Dv], lse [n]) float64.
        """
        q, k, v = _u16(q), _u16(k), _u16(v)
        Dqk, Dv = q.shape[-1], v.shape[-1]
        qs = q_strides or (Hq * Dqk, Dqk)
        ks = k_strides or (Hkv * Dqk, Dqk)
        vs = v_strides or (Hkv * Dv, Dv)
        rows = np.asarray(rows, dtype=np.int32).reshape(-1, 3)
        n = rows.shape[0]
        rb, rh, ri = _i32(rows[:, 0]), _i32(rows[:, 1]), _i32(rows[:, 2])
        o = np.zeros((n, Dv), dtype=np.float64)
        lse = np.zeros((n,), dtype=np.float64)
        cq, ck = _i32(cu_q), _i32(cu_kv)
        self._lib.oracle_attn_ragged_rows(
            _p(q), _p(k), _p(v), _p(cq), _p(ck),
            ctypes.c_int(Hq), ctypes.c_int(Hkv), ctypes.c_int(Dqk), ctypes.c_int(Dv),
            ctypes.c_int64(qs[0]), ctypes.c_int64(qs[1]), ctypes.c_int64(ks[0]),
            ctypes.c_int64(ks[1]), ctypes.c_int64(vs[0]), ctypes.c_int64(vs[1]),
            ctypes.c_double(scale), ctypes.c_int(int(causal)),
            ctypes.c_int64(n), _p(rb), _p(rh), _p(ri), _p(o), _p(lse))
        return o, lse

    def attn_dense_rows(self, q, k, v, Sq, Skv, Hq, Hkv, Dqk, Dv, scale, causal, rows,
                        q_strides=None, k_strides=None, v_strides=None):
        """Rows (b, h, i) of dense BSHD attention.

        q, k, v: bf16 bits addressed by (b, s, h) element strides; defaults are
        the compact [B, S, H, D] strides.  Returns (o [n, Dv], lse [n]).
        """
        q, k, v = _u16(q), _u16(k), _u16(v)
        qs = _i64(q_strides or (Sq * Hq * Dqk, Hq * Dqk, Dqk))
        ks = _i64(k_strides or (Skv * Hkv * Dqk, Hkv * Dqk, Dqk))
        vs = _i64(v_strides or (Skv * Hkv * Dv, Hkv * Dv, Dv))
        rows = np.asarray(rows, dtype=np.int32).reshape(-1, 3)
        n = rows.shape[0]
        rb, rh, ri = _i32(rows[:, 0]), _i32(rows[:, 1]), _i32(rows[:, 2])
        o = np.zeros((n, Dv), dtype=np.float64)
        lse = np.zeros((n,), dtype=np.float64)
        self._lib.oracle_attn_dense_rows(
            _p(q), _p(k), _p(v), ctypes.c_int(Sq), ctypes.c_int(Skv),
            ctypes.c_int(Hq), ctypes.c_int(Hkv), ctypes.c_int(Dqk), ctypes.c_int(Dv),
            _p(qs), _p(ks), _p(vs), ctypes.c_double(scale), ctypes.c_int(int(causal)),
            ctypes.c_int64(n), _p(rb), _p(rh), _p(ri), _p(o), _p(lse))
        return o, lse

    def attn_paged_rows(self, q, k_pool, v_pool, page_table, kv_lens, page_size, Hq,
                        Hkv, Dqk, Dv, k_pool_strides, v_pool_strides, scale, rows,
                        key_lo=None, key_hi=None, q_strides=None):
        """Rows (b, h) of paged decode attention (one query token per sequence).

        q: [B, Hq, Dqk] bf16 bits.  k_pool / v_pool: bf16 bits addressed by
        (page, slot, head) element strides.  page_table: [B, max_pages] int32.
        key_lo/key_hi (optional, per row) restrict the attended key range, as one
        split of split-KV does.  Returns (o [n, Dv], lse [n]).
        """
        q, k_pool, v_pool = _u16(q), _u16(k_pool), _u16(v_pool)
        pt = _i32(page_table)
        kl = _i32(kv_lens)
        qs = q_strides or (Hq * Dqk, Dqk)
        rows = np.asarray(rows, dtype=np.int32).reshape(-1, 2)
        n = rows.shape[0]
        rb, rh = _i32(rows[:, 0]), _i32(rows[:, 1])
        lo = _i64(np.zeros(n) if key_lo is None else key_lo)
        hi = _i64(np.full(n, np.iinfo(np.int64).max) if key_hi is None else key_hi)
        o = np.zeros((n, Dv), dtype=np.float64)
        lse = np.zeros((n,), dtype=np.float64)
        self._lib.oracle_attn_paged_rows(
            _p(q), ctypes.c_int64(qs[0]), ctypes.c_int64(qs[1]), _p(k_pool), _p(v_pool),
            _p(pt), ctypes.c_int64(pt.shape[1]), _p(kl), ctypes.c_int(page_size),
            ctypes.c_int(Hq), ctypes.c_int(Hkv), ctypes.c_int(Dqk), ctypes.c_int(Dv),
            _p(_i64(k_pool_strides)), _p(_i64(v_pool_strides)), ctypes.c_double(scale),
            ctypes.c_int64(n), _p(rb), _p(rh), _p(lo), _p(hi), _p(o), _p(lse))
        return o, lse

    def split_merge(self, o_part, lse_part):
        """Merge split-KV partials by their LSE.  o_part [S, R, Dv], lse_part [S, R]
        (any float dtype, widened exactly to float64).  Returns (o [R, Dv], lse [R])."""
        o_part = np.ascontiguousarray(o_part, dtype=np.float64)
        lse_part = np.ascontiguousarray(lse_part, dtype=np.float64)
        S, R, Dv = o_part.shape
        o = np.zeros((R, Dv), dtype=np.float64)
        lse = np.zeros((R,), dtype=np.float64)
        self._lib.oracle_split_merge(_p(o_part), _p(lse_part), ctypes.c_int(S),
                                     ctypes.c_int64(R), ctypes.c_int(Dv), _p(o), _p(lse))
        return o, lse


_default = None


def default() -> Oracle:
    """The oracle built from ``attn_oracle.c`` (compiled on first use)."""
    global _default
    if _default is None:
        _default = Oracle(build())
    return _default
