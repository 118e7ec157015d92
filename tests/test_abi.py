"""C-ABI checks that need no GPU: the library loads, exports every function
include/b2attn.h declares, and rejects bad arguments on the host before any
CUDA call."""
import ctypes
import os
import re

import pytest

import ragged_scaled_dot_b200 as rsd
from ragged_scaled_dot_b200 import build as rsd_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "b2attn.h")


@pytest.fixture(scope="module")
def lib():
    rsd_build.build()
    return rsd.lib()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(attn_[a-z0-9_]+)\s*\(", text)))


def test_header_declares_expected_entry_points():
    names = declared_functions()
    for n in ("attn_fwd_dense", "attn_fwd_ragged", "attn_fwd_paged", "attn_split_merge"):
        assert n in names


def test_every_declared_symbol_is_exported(lib):
    names = declared_functions()
    assert names
    for n in names:
        assert hasattr(lib, n), n
        assert n in rsd.SIGNATURES, f"binding lacks {n}"


def test_status_strings(lib):
    for code in range(8):
        assert rsd.status_string(code).startswith("ATTN_")
    assert rsd.status_string(99) == "unknown status"


def test_workspace_sizes(lib):
    # ragged: header + one 16-byte item per (query tile, head pair) + two ints per sequence
    n = rsd.attn_fwd_ragged_workspace_size(2, 64, 101, 4, 1)
    tiles = min(101 // 128 + 2, 2 * 1)
    assert n >= 256 + tiles * 2 * 16 + 2 * 2 * 4 and n % 256 == 0
    assert rsd.attn_fwd_ragged_workspace_size(0, 64, 101, 4, 1) == 0
    # paged: none for one split; partial O (fp32) + partial LSE otherwise
    assert rsd.attn_fwd_paged_workspace_size(128, 64, 128, 1) == 0
    n = rsd.attn_fwd_paged_workspace_size(128, 64, 128, 3)
    assert n >= 3 * 128 * 64 * 128 * 4 + 3 * 128 * 64 * 4 and n % 256 == 0


def test_suggest_splits_range(lib):
    for args in [(128, 64, 8, 128, 128, 32768, 64, 148), (64, 128, 1, 576, 512, 65536, 64, 148),
                 (1, 8, 1, 128, 128, 64, 16, 148), (4096, 32, 8, 128, 128, 1024, 64, 148)]:
        s = rsd.attn_paged_suggest_splits(*args)
        assert 1 <= s <= 64


L2 = ctypes.c_int64 * 2
L3 = ctypes.c_int64 * 3


def test_dense_rejects_bad_args_on_host(lib):
    st = L3(8 * 4 * 64, 4 * 64, 64)
    f = lib.attn_fwd_dense
    fake = ctypes.c_void_p(0x100000)   # never dereferenced: rejected before launch
    ws = ctypes.c_void_p(0x100100)     # 256-byte aligned
    # Hq not a multiple of Hkv
    assert f(None, None, None, None, None, 1, 8, 8, 3, 2, 64, 64, st, st, st, st, 1.0, 1, None, 0, None) == rsd.ATTN_ERR_INVALID_ARG
    # unsupported head dim
    assert f(None, None, None, None, None, 1, 8, 8, 4, 1, 96, 96, st, st, st, st, 1.0, 1, None, 0, None) == rsd.ATTN_ERR_UNSUPPORTED
    # non-finite scale
    assert f(None, None, None, None, None, 1, 8, 8, 4, 1, 64, 64, st, st, st, st, float("nan"), 1, None, 0, None) == rsd.ATTN_ERR_INVALID_ARG
    # empty problem is a no-op, workspace or not
    assert f(None, None, None, None, None, 0, 8, 8, 4, 1, 64, 64, st, st, st, st, 1.0, 1, None, 0, None) == rsd.ATTN_OK
    # null pointers with a real shape
    assert f(None, None, None, None, None, 1, 8, 8, 4, 1, 64, 64, st, st, st, st, 1.0, 1, None, 0, None) == rsd.ATTN_ERR_INVALID_ARG
    # the work list needs a workspace: missing, too small or misaligned is refused before launch
    need = rsd.attn_fwd_dense_workspace_size(1, 8, 4, 1)
    assert f(fake, fake, fake, fake, None, 1, 8, 8, 4, 1, 64, 64, st, st, st, st, 1.0, 1, None, 0, None) == rsd.ATTN_ERR_WORKSPACE
    assert f(fake, fake, fake, fake, None, 1, 8, 8, 4, 1, 64, 64, st, st, st, st, 1.0, 1, ws, need - 1, None) == rsd.ATTN_ERR_WORKSPACE
    assert f(fake, fake, fake, fake, None, 1, 8, 8, 4, 1, 64, 64, st, st, st, st, 1.0, 1,
             ctypes.c_void_p(0x100010), need, None) == rsd.ATTN_ERR_WORKSPACE


def test_dense_workspace_size(lib):
    # header + one 16-byte item per (batch, 128-row query tile, head pair)
    n = rsd.attn_fwd_dense_workspace_size(8, 4096, 32, 8)
    assert n == 256 + 8 * 32 * 16 * 16 and n % 256 == 0
    assert rsd.attn_fwd_dense_workspace_size(2, 100, 3, 1) == 256 + 256   # G odd: one head per item, 2*1*3 items
    assert rsd.attn_fwd_dense_workspace_size(0, 100, 4, 1) == 0
    assert rsd.attn_fwd_dense_workspace_size(1, 100, 3, 2) == 0             # Hq % Hkv != 0


def test_ragged_requires_workspace(lib):
    s2 = L2(4 * 64, 64)
    f = lib.attn_fwd_ragged
    fake = ctypes.c_void_p(0x100000)  # never dereferenced: rejected before launch
    rc = f(fake, fake, fake, fake, None, fake, fake, 2, 64, 64, 101, 101, 4, 1, 64, 64,
           s2, s2, s2, s2, 0, 0.125, 1, None, 0, None)
    assert rc == rsd.ATTN_ERR_WORKSPACE
    rc = f(fake, fake, fake, fake, None, fake, fake, 2, 64, 64, 101, 101, 4, 1, 64, 64,
           s2, s2, s2, s2, 0, 0.125, 1, ctypes.c_void_p(0x100100), 8, None)
    assert rc == rsd.ATTN_ERR_WORKSPACE
    # bad LSE layout codes; the valid ones (any base layout, with or without the
    # base-2 flag) get as far as the workspace check
    for bad in (7, 3, rsd.ATTN_LSE_LOG2 | 3, 0x200):
        rc = f(fake, fake, fake, fake, None, fake, fake, 2, 64, 64, 101, 101, 4, 1, 64, 64,
               s2, s2, s2, s2, bad, 0.125, 1, None, 0, None)
        assert rc == rsd.ATTN_ERR_INVALID_ARG, bad
    for good in (rsd.ATTN_LSE_PADDED_BSH, rsd.ATTN_LSE_PACKED_TH, rsd.ATTN_LSE_PACKED_HT):
        for flag in (0, rsd.ATTN_LSE_LOG2):
            rc = f(fake, fake, fake, fake, None, fake, fake, 2, 64, 64, 101, 101, 4, 1, 64, 64,
                   s2, s2, s2, s2, good | flag, 0.125, 1, None, 0, None)
            assert rc == rsd.ATTN_ERR_WORKSPACE, (good, flag)


def test_kv_table_entry_points_validate_both_tables(lib):
    """The independent-table calls check the V table like the K table: a null
    V table or a V row shorter than max_kv_len pages is rejected on the host."""
    fake = ctypes.c_void_p(0x100000)
    q2 = L2(64 * 128, 128)
    kp = L3(8 * 64 * 128, 128, 64 * 128)
    f = lib.attn_fwd_paged_kv_tables

    def dec(vt, vstride):
        return f(fake, fake, fake, fake, None, fake, 64, vt, vstride, fake, 4, 64, 8, 128, 128, 64, 100, 4096,
                 q2, q2, kp, kp, 0.088, 3, None, 0, None)

    assert dec(fake, 64) == rsd.ATTN_ERR_WORKSPACE        # both tables fine: next check is the workspace
    assert dec(None, 64) == rsd.ATTN_ERR_INVALID_ARG
    assert dec(fake, 63) == rsd.ATTN_ERR_INVALID_ARG      # 63 pages < 4096 / 64
    g = lib.attn_fwd_paged_prefill_kv_tables
    q3 = L2(32 * 128, 128)
    kp3 = L3(4 * 64 * 128, 128, 64 * 128)

    def pre(vt, vstride):
        return g(fake, fake, fake, fake, None, fake, fake, 64, vt, vstride, fake, 2, 512, 600, 32, 4, 128, 64,
                 100, 4096, q3, q3, kp3, kp3, rsd.ATTN_LSE_PADDED_BSH, 0.088, 1, 1, None, 0, None)

    assert pre(fake, 64) == rsd.ATTN_ERR_WORKSPACE
    assert pre(None, 64) == rsd.ATTN_ERR_INVALID_ARG
    assert pre(fake, 10) == rsd.ATTN_ERR_INVALID_ARG


def test_paged_rejects_bad_args_on_host(lib):
    f = lib.attn_fwd_paged
    fake = ctypes.c_void_p(0x100000)
    q2 = L2(64 * 128, 128)
    kp = L3(8 * 64 * 128, 128, 64 * 128)
    args = dict(B=4, Hq=64, Hkv=8, Dqk=128, Dv=128, ps=64, P=100, maxkv=4096, splits=3)

    def call(**kw):
        a = dict(args, **kw)
        return f(fake, fake, fake, fake, None, fake, 64, fake, a["B"], a["Hq"], a["Hkv"], a["Dqk"],
                 a["Dv"], a["ps"], a["P"], a["maxkv"], q2, q2, kp, kp, 0.088, a["splits"], None, 0,
                 None)

    assert call() == rsd.ATTN_ERR_WORKSPACE              # 3 splits need a workspace
    # split MLA outputs go through the merge kernel, which needs batch-major O rows: refused
    # on the host, before the workspace is even looked at; the GQA blocks write rows by
    # their (batch, head) strides, so there only the missing workspace is reported
    kp_mla = L3(64 * 576, 576, 64 * 576)
    assert f(fake, fake, fake, fake, None, fake, 64, fake, 4, 128, 1, 576, 512, 64, 100, 4096,
             L2(128 * 576, 576), L2(128 * 512 + 8, 512), kp_mla, kp_mla, 0.04, 3, None, 0,
             None) == rsd.ATTN_ERR_UNSUPPORTED
    assert f(fake, fake, fake, fake, None, fake, 64, fake, 4, 64, 8, 128, 128, 64, 100, 4096,
             q2, L2(64 * 128 + 8, 128), kp, kp, 0.088, 3, None, 0, None) == rsd.ATTN_ERR_WORKSPACE
    assert call(Dqk=96, Dv=96) == rsd.ATTN_ERR_UNSUPPORTED
    assert call(ps=48) == rsd.ATTN_ERR_UNSUPPORTED        # neither divides nor is divided by 64
    assert call(Hkv=7) == rsd.ATTN_ERR_INVALID_ARG        # 64 % 7 != 0
    assert call(Hq=256, Hkv=8) == rsd.ATTN_ERR_UNSUPPORTED  # G = 32 > 16
    assert call(Dqk=576, Dv=512, Hq=128, Hkv=2) == rsd.ATTN_ERR_UNSUPPORTED  # MLA needs one KV head
    assert call(Dqk=576, Dv=512, Hq=128, Hkv=1, ps=8) == rsd.ATTN_ERR_UNSUPPORTED  # MLA page box N >= 16
    assert call(splits=0) == rsd.ATTN_ERR_INVALID_ARG


def test_merge_rejects_bad_args_on_host(lib):
    f = lib.attn_split_merge
    fake = ctypes.c_void_p(0x100000)
    assert f(fake, fake, 0, 10, 128, fake, 128, None, None) == rsd.ATTN_ERR_INVALID_ARG
    assert f(fake, fake, 2, 10, 96, fake, 96, None, None) == rsd.ATTN_ERR_UNSUPPORTED
    assert f(fake, fake, 2, 10, 128, fake, 64, None, None) == rsd.ATTN_ERR_INVALID_ARG
    assert f(None, None, 2, 0, 128, None, 128, None, None) == rsd.ATTN_OK


def test_binding_fails_loudly_without_library(monkeypatch, tmp_path):
    monkeypatch.setattr(rsd, "_lib", None)
    monkeypatch.setattr(rsd, "LIB_PATH", str(tmp_path / "missing.so"))
    with pytest.raises(ImportError):
        rsd.lib()


def test_paged_prefill_rejects_bad_args_on_host(lib):
    f = lib.attn_fwd_paged_prefill
    fake = ctypes.c_void_p(0x100000)
    q2 = L2(32 * 128, 128)
    kp = L3(4 * 64 * 128, 128, 64 * 128)          # HND [pages, 4 heads, 64 rows, 128]
    args = dict(B=2, Hq=32, Hkv=4, D=128, ps=64, P=100, maxkv=4096, maxsq=512, Tq=600, ks=kp, ws=None, splits=1)

    def call(**kw):
        a = dict(args, **kw)
        return f(fake, fake, fake, fake, None, fake, fake, 64, fake, a["B"], a["maxsq"], a["Tq"], a["Hq"],
                 a["Hkv"], a["D"], a["ps"], a["P"], a["maxkv"], q2, q2, a["ks"], a["ks"],
                 rsd.ATTN_LSE_PADDED_BSH, 0.088, 1, a["splits"], a["ws"], 1 << 30 if a["ws"] else 0, None)

    assert call() == rsd.ATTN_ERR_WORKSPACE                 # the work list needs a workspace
    assert call(D=96) == rsd.ATTN_ERR_UNSUPPORTED
    assert call(ps=48) == rsd.ATTN_ERR_UNSUPPORTED          # neither divides nor is divided by 128
    assert call(ps=4) == rsd.ATTN_ERR_UNSUPPORTED           # fewer rows than one 8-row group
    assert call(Hkv=5) == rsd.ATTN_ERR_INVALID_ARG          # 32 % 5 != 0
    # a page stride that is not a whole number of 8-row groups
    assert call(ks=L3(4 * 64 * 128 + 8, 128, 64 * 128)) == rsd.ATTN_ERR_UNSUPPORTED
    assert call(B=0) == rsd.ATTN_OK                          # nothing to do
    assert call(splits=0) == rsd.ATTN_ERR_INVALID_ARG
    assert call(splits=5000) == rsd.ATTN_ERR_INVALID_ARG
    # without splits the workspace is the prefill work list; with splits it adds the short rows'
    # partials: B * qmax * Hq rows of D floats and an LSE per split, qmax = min(4, 64 / G, max_seqlen_q)
    assert rsd.attn_fwd_paged_prefill_workspace_size(2, 512, 600, 32, 4, 128, 1) == \
        rsd.attn_fwd_ragged_workspace_size(2, 512, 600, 32, 4)
    base = rsd.attn_fwd_ragged_workspace_size(2, 512, 600, 32, 4)
    rows = 2 * 4 * 32          # G = 8: qmax = min(4, 8, 512) = 4
    n3 = rsd.attn_fwd_paged_prefill_workspace_size(2, 512, 600, 32, 4, 128, 3)
    assert n3 >= base + 3 * rows * 128 * 4 + 3 * rows * 4 + 2 * 4 and n3 % 256 == 0
    rows = 2 * 1 * 64          # G = 64: qmax = 1
    assert rsd.attn_fwd_paged_prefill_workspace_size(2, 512, 600, 64, 1, 64, 2) >= \
        rsd.attn_fwd_ragged_workspace_size(2, 512, 600, 64, 1) + 2 * rows * 64 * 4
    # G > 64: no routing, no partials
    assert rsd.attn_fwd_paged_prefill_workspace_size(2, 512, 600, 128, 1, 64, 2) == \
        rsd.attn_fwd_ragged_workspace_size(2, 512, 600, 128, 1)


def test_sizes_past_the_32_bit_token_range_are_declined(lib):
    """Token counts of 2^31 or more (32-bit token coordinates of the tensor
    maps and the work list) and grids past the launch limits are declined
    with ATTN_ERR_UNSUPPORTED on the host, never computed wrongly."""
    fake = ctypes.c_void_p(0x100000)
    s2 = L2(4 * 64, 64)
    big = 1 << 31
    f = lib.attn_fwd_ragged
    assert f(fake, fake, fake, fake, None, fake, fake, 2, 64, 64, big, 101, 4, 1, 64, 64,
             s2, s2, s2, s2, 0, 0.125, 1, None, 0, None) == rsd.ATTN_ERR_UNSUPPORTED
    assert f(fake, fake, fake, fake, None, fake, fake, 2, 64, 64, 101, big, 4, 1, 64, 64,
             s2, s2, s2, s2, 0, 0.125, 1, None, 0, None) == rsd.ATTN_ERR_UNSUPPORTED
    assert f(fake, fake, fake, fake, None, fake, fake, 2, 64, 64, big - 1, 101, 4, 1, 64, 64,
             s2, s2, s2, s2, 0, 0.125, 1, None, 0, None) == rsd.ATTN_ERR_WORKSPACE
    g = lib.attn_fwd_paged
    q2 = L2(64 * 128, 128)
    kp = L3(8 * 64 * 128, 128, 64 * 128)
    assert g(fake, fake, fake, fake, None, fake, 64, fake, 65536, 64, 8, 128, 128, 64, 100, 4096,
             q2, q2, kp, kp, 0.088, 1, None, 0, None) == rsd.ATTN_ERR_UNSUPPORTED   # B > 65535


def test_page_coords_diagnostic_rejects_bad_args_on_host(lib):
    f = lib.attn_selftest_page_coords
    fake = ctypes.c_void_p(0x100000)
    assert f(fake, 64, 64, 100, 8, fake, fake, 0, fake, None) == rsd.ATTN_OK          # nothing to do
    assert f(fake, 64, 0, 100, 8, fake, fake, 5, fake, None) == rsd.ATTN_ERR_INVALID_ARG   # page size 0
    assert f(fake, 64, 64, 0, 8, fake, fake, 5, fake, None) == rsd.ATTN_ERR_INVALID_ARG    # no pages
    assert f(None, 64, 64, 100, 8, fake, fake, 5, fake, None) == rsd.ATTN_ERR_INVALID_ARG  # no table
    assert f(fake, 64, 64, 1 << 30, 8, fake, fake, 5, fake, None) == rsd.ATTN_ERR_UNSUPPORTED  # groups >= 2^31
