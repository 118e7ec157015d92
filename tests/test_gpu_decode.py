"""Paged decode (GQA and absorbed MLA) with split-KV on the GPU vs the fp64
oracle, plus paged == contiguous (bit-exact), split == unsplit, NaN in the
unused tail of the last page, independent K and V page tables, and the
standalone LSE merge."""
import numpy as np
import pytest
import torch

import gpu_util
import oracle
import ragged_scaled_dot_b200 as rsd
import synth
from gpu_util import assert_lse_close, assert_o_close, bits, check_paged, orc, paged_gpu

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _paged_inputs(lens, Hq, Hkv, D, ps, seed, layout="HND", Dv=None, alias=False, extra_pages=3):
    table, total = synth.page_table(lens, ps, seed)
    P = total + extra_pages
    q = synth.normal_bf16((len(lens), Hq, D), seed + 1, "cpu").to(DEV)
    shape_k = (P, Hkv, ps, D) if layout == "HND" else (P, ps, Hkv, D)
    k = synth.normal_bf16(shape_k, seed + 2, "cpu").to(DEV)
    if alias:
        v = k
    else:
        Dv = Dv or D
        shape_v = (P, Hkv, ps, Dv) if layout == "HND" else (P, ps, Hkv, Dv)
        v = synth.normal_bf16(shape_v, seed + 3, "cpu").to(DEV)
    return q, k, v, table, np.asarray(lens, dtype=np.int32)


GQA_CASES = [
    # (lens, Hq, Hkv, D, ps, layout, splits)
    ([0, 1, 63, 64, 1000], 16, 2, 128, 64, "HND", 1),
    ([0, 1, 63, 64, 1000], 16, 2, 128, 64, "HND", 3),
    ([65, 700, 2049], 64, 8, 128, 64, "HND", 7),
    ([5, 300, 129], 8, 1, 128, 16, "NHD", 2),
    ([100, 1, 777], 32, 4, 64, 32, "HND", 4),
    ([1000, 20], 4, 4, 128, 128, "NHD", 2),
    ([3000], 12, 1, 128, 64, "HND", 16),   # more splits than some sequences have pages
    ([7, 64, 1000, 333], 16, 2, 128, 8, "HND", 1),   # 8-row pages: 16 lanes issue a chunk's boxes
    ([300, 45, 2000], 8, 1, 128, 16, "HND", 1),      # page 16 unsplit (the deep ring)
]


@pytest.mark.parametrize("lens,Hq,Hkv,D,ps,layout,splits", GQA_CASES)
def test_gqa_decode_cases(lens, Hq, Hkv, D, ps, layout, splits):
    q, k, v, table, kl = _paged_inputs(lens, Hq, Hkv, D, ps, seed=len(lens) * 11 + ps, layout=layout)
    check_paged(q, k, v, table, kl, ps, 1.0 / np.sqrt(D), splits, kv_layout=layout,
                where=f"gqa {lens} ps{ps} S{splits}")


def test_paged_equals_contiguous_bitwise():
    """A random page permutation gives bit-identical results to the identity
    table over a pool pre-permuted so both see the same logical K/V."""
    lens = [500, 64, 1100]
    Hq, Hkv, D, ps = 16, 2, 128, 64
    q, k, v, table, kl = _paged_inputs(lens, Hq, Hkv, D, ps, seed=3)
    o1, l1 = paged_gpu(q, k, v, table, kl, ps, 0.09, 1)
    # identity layout: logical page i of the batch stored at physical i
    n_pages = [(L + ps - 1) // ps for L in lens]
    phys = np.concatenate([table[b, :n] for b, n in enumerate(n_pages)]).astype(np.int64)
    k2 = k[torch.as_tensor(phys, device=DEV)].contiguous()
    v2 = v[torch.as_tensor(phys, device=DEV)].contiguous()
    t2 = np.full_like(table, -1)
    pos = 0
    for b, n in enumerate(n_pages):
        t2[b, :n] = np.arange(pos, pos + n)
        pos += n
    o2, l2 = paged_gpu(q, k2, v2, t2, kl, ps, 0.09, 1)
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


def test_split_equals_unsplit():
    lens = [4000, 129, 64, 1]
    q, k, v, table, kl = _paged_inputs(lens, 16, 2, 128, 64, seed=7)
    o1, l1 = paged_gpu(q, k, v, table, kl, 64, 0.09, 1)
    for S in (2, 7, 63):
        o2, l2 = paged_gpu(q, k, v, table, kl, 64, 0.09, S)
        assert_o_close(o2, o1.float().cpu().numpy().astype(np.float64), f"split {S}")
        assert np.max(np.abs(l2.cpu().numpy() - l1.cpu().numpy())) < 1e-4


def test_nan_inside_last_page_is_never_used():
    """Slots past kv_len inside a sequence's last page hold NaN: outputs stay
    finite and equal to a run with clean slots."""
    lens = [70, 200]
    ps = 64
    q, k, v, table, kl = _paged_inputs(lens, 8, 1, 128, ps, seed=17)
    kn, vn = k.clone(), v.clone()
    for b, L in enumerate(lens):
        last = table[b, (L - 1) // ps]
        kn[last, :, L % ps:] = float("nan")
        vn[last, :, L % ps:] = float("nan")
    for S in (1, 3):
        o1, l1 = paged_gpu(q, k, v, table, kl, ps, 0.1, S)
        o2, l2 = paged_gpu(q, kn, vn, table, kl, ps, 0.1, S)
        assert torch.isfinite(o2.float()).all()
        assert torch.equal(o1, o2) and torch.equal(l1, l2)


@pytest.mark.parametrize("splits", [1, 3])
@pytest.mark.parametrize("alias", [True, False])
def test_mla_decode(splits, alias):
    lens = [0, 100, 700, 33]
    Hq, D, Dv, ps = 128, 576, 512, 64
    q, k, v, table, kl = _paged_inputs(lens, Hq, 1, D, ps, seed=23, Dv=Dv, alias=alias)
    check_paged(q, k, v, table, kl, ps, 1.0 / np.sqrt(D), splits, Dv=Dv,
                where=f"mla alias={alias} S={splits}")


def test_mla_nan_past_kv_len_aliased():
    lens = [90]
    ps = 64
    q, k, _, table, kl = _paged_inputs(lens, 128, 1, 576, ps, seed=29, alias=True)
    kn = k.clone()
    kn[table[0, 1], :, 90 - 64:] = float("nan")
    o1, l1 = paged_gpu(q, k, k, table, kl, ps, 0.04, 1, o_dv=512)
    o2, l2 = paged_gpu(q, kn, kn, table, kl, ps, 0.04, 1, o_dv=512)
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


MLA_CASES = [
    # (lens, Hq, ps, splits, alias): chunk edges, padded head groups, page sizes
    ([1, 127, 128, 129, 300], 64, 64, 1, True),
    ([257, 1000], 192, 64, 2, True),
    ([500, 77], 128, 16, 1, False),
    ([600, 130], 128, 128, 3, True),
    ([3000], 16, 32, 5, True),
    ([2, 64, 65, 200], 128, 16, 2, False),
]


@pytest.mark.parametrize("lens,Hq,ps,splits,alias", MLA_CASES)
def test_mla_decode_shapes(lens, Hq, ps, splits, alias):
    q, k, v, table, kl = _paged_inputs(lens, Hq, 1, 576, ps, seed=31 + ps + Hq, Dv=512, alias=alias)
    check_paged(q, k, v, table, kl, ps, 1.0 / np.sqrt(576), splits, Dv=512,
                where=f"mla {lens} Hq{Hq} ps{ps} S{splits} alias={alias}")


def _ramp_keys(k, table, lens, ps, gain):
    """Scale the K row of logical key j by 1 + gain*j/L, so every sequence's
    scores keep growing and the running maximum moves many times."""
    k = k.clone()
    for b, L in enumerate(lens):
        j = np.arange(L)
        pages = torch.as_tensor(table[b, j // ps].astype(np.int64), device=DEV)
        slots = torch.as_tensor(j % ps, device=DEV)
        f = torch.as_tensor(1.0 + gain * j / max(L, 1), dtype=torch.float32, device=DEV)
        rows = k[pages, 0, slots].float() * f[:, None]
        k[pages, 0, slots] = rows.to(k.dtype)
    return k


@pytest.mark.parametrize("scale", [0.3, -0.3])
def test_mla_rescale_path(scale):
    """Scores that grow along the sequence force O rescales in the value CTA
    (the running max rises by more than 2^8 many times); result vs the oracle.
    V is a separate N(0,1) pool: with V aliasing the ramped K, |V| reaches ~16
    and the bf16 rounding of P alone (2^-8 relative) exceeds the tolerance."""
    lens = [1500, 700]
    ps = 64
    q, k, v, table, kl = _paged_inputs(lens, 128, 1, 576, ps, seed=37, Dv=512)
    k = _ramp_keys(k, table, lens, ps, 3.0)
    for S in (1, 2):
        check_paged(q, k, v, table, kl, ps, scale, S, Dv=512, where=f"mla rescale scale={scale} S={S}")


def test_mla_nan_past_kv_len_separate_v():
    """Separate V pool, small pages (partial TMA box at the end), splits."""
    lens = [90, 37]
    ps = 16
    q, k, v, table, kl = _paged_inputs(lens, 128, 1, 576, ps, seed=41, Dv=512)
    kn, vn = k.clone(), v.clone()
    for b, L in enumerate(lens):
        last = table[b, (L - 1) // ps]
        kn[last, :, L % ps:] = float("nan")
        vn[last, :, L % ps:] = float("nan")
    for S in (1, 3):
        o1, l1 = paged_gpu(q, k, v, table, kl, ps, 0.04, S, o_dv=512)
        o2, l2 = paged_gpu(q, kn, vn, table, kl, ps, 0.04, S, o_dv=512)
        assert torch.isfinite(o2.float()).all()
        assert torch.equal(o1, o2) and torch.equal(l1, l2)


def test_mla_paged_equals_contiguous_bitwise():
    lens = [300, 64, 1000]
    ps = 64
    q, k, _, table, kl = _paged_inputs(lens, 128, 1, 576, ps, seed=43, alias=True)
    o1, l1 = paged_gpu(q, k, k, table, kl, ps, 0.05, 1, o_dv=512)
    n_pages = [(L + ps - 1) // ps for L in lens]
    phys = np.concatenate([table[b, :n] for b, n in enumerate(n_pages)]).astype(np.int64)
    k2 = k[torch.as_tensor(phys, device=DEV)].contiguous()
    t2 = np.full_like(table, -1)
    pos = 0
    for b, n in enumerate(n_pages):
        t2[b, :n] = np.arange(pos, pos + n)
        pos += n
    o2, l2 = paged_gpu(q, k2, k2, t2, kl, ps, 0.05, 1, o_dv=512)
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


def test_mla_split_equals_unsplit():
    lens = [5000, 129, 1]
    q, k, _, table, kl = _paged_inputs(lens, 128, 1, 576, 64, seed=47, alias=True)
    o1, l1 = paged_gpu(q, k, k, table, kl, 64, 0.05, 1, o_dv=512)
    for S in (2, 7, 79):
        o2, l2 = paged_gpu(q, k, k, table, kl, 64, 0.05, S, o_dv=512)
        assert_o_close(o2, o1.float().cpu().numpy().astype(np.float64), f"mla split {S}")
        assert np.max(np.abs(l2.cpu().numpy() - l1.cpu().numpy())) < 1e-4


@pytest.mark.parametrize("Dv", [64, 128, 512])
def test_split_merge_kernel_vs_oracle(Dv):
    S, R = 5, 300
    g = torch.Generator().manual_seed(Dv)
    o_part = torch.randn((S, R, Dv), generator=g)
    lse_part = torch.randn((S, R), generator=g) * 3
    lse_part[torch.rand((S, R), generator=g) < 0.3] = -float("inf")
    lse_part[:, :7] = -float("inf")              # rows with no keys at all
    o_part[lse_part == -float("inf")] = float("nan")  # empty partials must be ignored
    o_ref, l_ref = orc().split_merge(o_part.numpy(), lse_part.numpy())
    o = torch.full((R, Dv), float("nan"), dtype=torch.bfloat16, device=DEV)
    lse = torch.empty((R,), dtype=torch.float32, device=DEV)
    rsd.attn_split_merge(o_part.to(DEV), lse_part.to(DEV), o, lse)
    torch.cuda.synchronize()
    assert_o_close(o, o_ref, "merge")
    assert_lse_close(lse, l_ref, "merge")


# ------------------------------------------------ independent K and V tables
def _independent_v(v_pool, table_k, lens, ps, seed, layout="HND"):
    """A second V pool that holds the same logical value rows as v_pool (read
    through table_k), laid out by its own page permutation table_v.  Pages no
    table entry names are NaN, so a read outside the table would show."""
    lens = np.asarray(lens, dtype=np.int64)
    n_pages = (lens + ps - 1) // ps
    table_v, total = synth.page_table(lens, ps, seed)
    v2 = torch.full((total + 5,) + tuple(v_pool.shape[1:]), float("nan"), dtype=v_pool.dtype, device=DEV)
    src = np.concatenate([table_k[b, :n] for b, n in enumerate(n_pages)] + [np.zeros(0, np.int32)])
    dst = np.concatenate([table_v[b, :n] for b, n in enumerate(n_pages)] + [np.zeros(0, np.int32)])
    v2[torch.as_tensor(dst.astype(np.int64), device=DEV)] = v_pool[torch.as_tensor(src.astype(np.int64),
                                                                                    device=DEV)]
    return v2, table_v


def _paged_kv_tables_gpu(q, k_pool, v_pool, table_k, table_v, kl, ps, scale, splits, Dv, layout="HND"):
    B, Hq, _ = q.shape
    o = torch.full((B, Hq, Dv), float("nan"), dtype=torch.bfloat16, device=DEV)
    lse = torch.full((B, Hq), float("nan"), dtype=torch.float32, device=DEV)
    ws_n = rsd.attn_fwd_paged_workspace_size(B, Hq, Dv, splits)
    ws = torch.full((ws_n,), 0xFF, dtype=torch.uint8, device=DEV) if ws_n else None
    rsd.attn_fwd_paged_kv_tables(q, k_pool, v_pool, o, lse, torch.as_tensor(table_k, device=DEV),
                                 torch.as_tensor(table_v, device=DEV), torch.as_tensor(kl, device=DEV),
                                 page_size=ps, max_kv_len=max(1, int(np.max(kl))), scale=scale,
                                 num_splits=splits, workspace=ws, kv_layout=layout)
    torch.cuda.synchronize()
    assert rsd.attn_get_device_error() == rsd.ATTN_OK
    return o, lse


@pytest.mark.parametrize("lens,Hq,Hkv,D,ps,layout,splits", [
    ([0, 1, 700, 130], 16, 2, 128, 64, "HND", 1),
    ([0, 1, 700, 130], 16, 2, 128, 64, "HND", 3),
    ([300, 45], 8, 1, 64, 16, "NHD", 2),
])
def test_gqa_decode_independent_kv_tables(lens, Hq, Hkv, D, ps, layout, splits):
    """K through one page table, V through another over a different pool: the
    oracle's result for the same logical K/V, and bit-identical to one shared
    table over a pool that stores V where K's table points."""
    q, k, v, table, kl = _paged_inputs(lens, Hq, Hkv, D, ps, seed=53 + ps, layout=layout)
    v2, table_v = _independent_v(v, table, lens, ps, seed=59 + ps, layout=layout)
    assert not np.array_equal(table, table_v)
    o, lse = _paged_kv_tables_gpu(q, k, v2, table, table_v, kl, ps, 1.0 / np.sqrt(D), splits, D, layout)
    o1, l1 = paged_gpu(q, k, v, table, kl, ps, 1.0 / np.sqrt(D), splits, kv_layout=layout)
    assert torch.equal(o, o1) and torch.equal(lse, l1)
    rows = np.array([(b, h) for b in range(len(lens)) for h in range(Hq)], dtype=np.int32)
    o_ref, l_ref = orc().attn_paged_rows(bits(q), bits(k), bits(v), table, kl, ps, Hq, Hkv, D, D,
                                         gpu_util.pool_strides_np(k, layout), gpu_util.pool_strides_np(v, layout),
                                         1.0 / np.sqrt(D), rows)
    assert_o_close(o.reshape(-1, D), o_ref, "independent tables")
    assert_lse_close(lse.reshape(-1), l_ref, "independent tables")


@pytest.mark.parametrize("splits", [1, 2])
def test_mla_decode_independent_kv_tables(splits):
    """Absorbed-MLA shapes (Q/K 576, V 512) with V in its own pool and page table."""
    lens, ps = [100, 700, 64], 64
    q, k, v, table, kl = _paged_inputs(lens, 128, 1, 576, ps, seed=61, Dv=512)
    v2, table_v = _independent_v(v, table, lens, ps, seed=67)
    o, lse = _paged_kv_tables_gpu(q, k, v2, table, table_v, kl, ps, 1.0 / np.sqrt(576), splits, 512)
    o1, l1 = paged_gpu(q, k, v, table, kl, ps, 1.0 / np.sqrt(576), splits, o_dv=512)
    assert torch.equal(o, o1) and torch.equal(lse, l1)
    check_paged(q, k, v, table, kl, ps, 1.0 / np.sqrt(576), splits, Dv=512, where="mla independent tables")


@pytest.mark.parametrize("mla", [False, True])
def test_decode_batch_permutation_bitwise(mla):
    """With splits the blocks take the sequences longest first (a device-side
    sort): permuting the batch permutes the outputs bit for bit, so every split
    lands on its own sequence whatever block runs it (GQA: a pair's pieces and
    their merge depend on its own length only)."""
    lens = [3000, 10, 700, 700, 1, 2049, 64]
    if mla:
        q, k, v, table, kl = _paged_inputs(lens, 128, 1, 576, 64, seed=79, Dv=512)
        Dv, S = 512, 4
    else:
        q, k, v, table, kl = _paged_inputs(lens, 16, 2, 128, 64, seed=83)
        Dv, S = 128, 3
    o1, l1 = paged_gpu(q, k, v, table, kl, 64, 0.07, S, o_dv=Dv)
    perm = np.array([4, 0, 6, 2, 5, 3, 1])
    o2, l2 = paged_gpu(q[torch.as_tensor(perm, device=DEV)].contiguous(), k, v, table[perm], kl[perm], 64, 0.07, S,
                       o_dv=Dv)
    assert torch.equal(o2, o1[torch.as_tensor(perm, device=DEV)])
    assert torch.equal(l2, l1[torch.as_tensor(perm, device=DEV)])


SPLIT_CASES = [
    # (lens, Hq, Hkv, D, ps, splits): a long pair cut into 64 pieces (two merge levels)
    ([50000, 3], 16, 1, 128, 64, 64),
    # one pair cut into 938 one-unit pieces (four merge levels)
    ([60000], 8, 1, 64, 16, 4096),
    # many short sequences per block, empty ones among them
    ([(i * 37) % 300 for i in range(200)], 8, 2, 128, 64, 2),
    # lengths across three orders of magnitude, page 32
    ([1, 70000, 64, 65, 0, 9000, 128, 3000], 32, 4, 128, 32, 3),
]


@pytest.mark.parametrize("lens,Hq,Hkv,D,ps,splits", SPLIT_CASES)
def test_split_decode_merge_tree_vs_oracle(lens, Hq, Hkv, D, ps, splits):
    """Split-KV with many pieces per pair (partials merged in groups of 8 by the
    last block to finish each group, level after level), many short sequences
    and empty ones, against the fp64 oracle (sampled rows for the 200-sequence
    batch)."""
    q, k, v, table, kl = _paged_inputs(lens, Hq, Hkv, D, ps, seed=len(lens) + ps + splits)
    rows = None
    if len(lens) > 100:
        rng = np.random.default_rng(5)
        rows = np.array([(b, h) for b in rng.choice(len(lens), 40, replace=False) for h in range(Hq)],
                        dtype=np.int32)
    o, lse, _ = check_paged(q, k, v, table, kl, ps, 1.0 / np.sqrt(D), splits, rows=rows,
                            where=f"split {len(lens)} seqs S{splits}")
    assert torch.isfinite(o.float()).all()
    empty = np.asarray(lens) == 0
    if empty.any():
        e = torch.as_tensor(np.nonzero(empty)[0], device=DEV)
        assert torch.all(o[e] == 0) and torch.all(lse[e] == -float("inf"))
    assert rsd.attn_get_device_error() == rsd.ATTN_OK
