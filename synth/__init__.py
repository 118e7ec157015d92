"""Seeded synthetic inputs shared by the tests, the bench and the oracle checks.

This module holds none of the attention arithmetic.  It only draws seeded
random tensors, sequence lengths and page tables, and it names the workloads
with their sizes.  Both the CUDA path and the oracle consume the same bf16 bytes
made here, so no random-number parity between the two sides is needed.

Recipe:
  * values: i.i.d. N(0, 1) drawn in fp32 by torch's seeded generator (on the
    device the tensor lives on), rounded to bf16 (round-to-nearest-even);
  * lengths: ``numpy.random.default_rng(seed).integers(lo, hi + 1, B)``;
  * page tables: the physical pages of all sequences are a seeded random
    permutation (``numpy.random.default_rng(seed + 1000).permutation``) of
    ``range(total_pages)``, handed out to sequences in order; unused table
    entries hold -1.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import numpy as np
import torch


def normal_bf16(shape, seed: int, device="cpu") -> torch.Tensor:
    """N(0, 1) values rounded to bf16, reproducible from ``seed`` on one device type."""
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    x = torch.randn(tuple(shape), generator=g, dtype=torch.float32, device=device)
    return x.to(torch.bfloat16)


def bf16_bits(t: torch.Tensor) -> np.ndarray:
    """Host copy of a bf16 tensor as its uint16 bit patterns (what the oracle reads)."""
    return t.detach().contiguous().cpu().view(torch.int16).numpy().view(np.uint16)


def uniform_lengths(B: int, lo: int, hi: int, seed: int) -> np.ndarray:
    """B lengths drawn uniformly from [lo, hi] inclusive."""
    return np.random.default_rng(seed).integers(lo, hi + 1, B).astype(np.int64)


def cu_seqlens(lengths) -> np.ndarray:
    """Prefix sums [0, L0, L0+L1, ...] as int32 (the offset table of the THD layout)."""
    out = np.zeros(len(lengths) + 1, dtype=np.int64)
    out[1:] = np.cumsum(np.asarray(lengths, dtype=np.int64))
    assert out[-1] < 2**31
    return out.astype(np.int32)


def page_table(kv_lens, page_size: int, seed: int, max_pages: int | None = None):
    """A page table over a pool holding exactly the pages the sequences need.

    Returns (table [B, max_pages] int32, total_pages).  Pages are a seeded random
    permutation of the pool, handed out to sequences in order.
    """
    kv_lens = np.asarray(kv_lens, dtype=np.int64)
    n_pages = (kv_lens + page_size - 1) // page_size
    total = int(n_pages.sum())
    mp = int(max_pages if max_pages is not None else max(1, int(n_pages.max(initial=0))))
    perm = np.random.default_rng(seed + 1000).permutation(total).astype(np.int32)
    table = np.full((len(kv_lens), mp), -1, dtype=np.int32)
    pos = 0
    for b, n in enumerate(n_pages):
        table[b, :n] = perm[pos:pos + n]
        pos += n
    return table, total


@dataclass
class Workload:
    """One named synthetic workload (sizes only; tensors are made on demand)."""
    name: str
    kind: str                      # "dense" | "ragged" | "paged"
    seed: int
    B: int
    Hq: int
    Hkv: int
    Dqk: int
    Dv: int
    causal: bool = True
    S: int = 0                     # dense: Sq = Skv = S
    lengths: tuple = ()            # ragged: q_len = kv_len per sequence
    len_range: tuple = ()          # ragged / paged: (lo, hi) of the uniform draw
    page_size: int = 64
    v_aliases_k: bool = False      # paged: V = first Dv columns of the K rows
    scale: float = 0.0
    notes: str = field(default="")

    def __post_init__(self):
        if self.scale == 0.0:
            self.scale = 1.0 / math.sqrt(self.Dqk)

    def seq_lengths(self) -> np.ndarray:
        if self.lengths:
            return np.asarray(self.lengths, dtype=np.int64)
        return uniform_lengths(self.B, self.len_range[0], self.len_range[1], self.seed)


WORKLOADS = {
    "tiny_ragged": Workload(
        "tiny_ragged", "ragged", seed=1, B=2, Hq=4, Hkv=1, Dqk=64, Dv=64,
        lengths=(37, 64), scale=1.0 / 8.0,
        notes="2 sequences q_len=kv_len {37, 64}, causal GQA 4/1, D=64"),
    "dense_prefill": Workload(
        "dense_prefill", "dense", seed=2, B=8, Hq=32, Hkv=8, Dqk=128, Dv=128, S=4096,
        notes="dense causal BSHD B=8 S=4096 H=32/8 D=128"),
    "ragged_prefill": Workload(
        "ragged_prefill", "ragged", seed=3, B=64, Hq=32, Hkv=8, Dqk=128, Dv=128,
        len_range=(128, 8192),
        notes="THD causal, 64 sequences U[128, 8192], H=32/8 D=128, padded LSE"),
    "paged_decode": Workload(
        "paged_decode", "paged", seed=4, B=128, Hq=64, Hkv=8, Dqk=128, Dv=128,
        len_range=(1024, 32768), page_size=64, causal=False,
        notes="paged decode B=128 kv U[1024, 32768] page 64, H=64/8 D=128"),
    "decode_small_batch": Workload(
        "decode_small_batch", "paged", seed=8, B=32, Hq=64, Hkv=4, Dqk=128, Dv=128,
        len_range=(4096, 4096), page_size=16, causal=False,
        notes="paged decode b=32, 4096 cached keys each, page 16, H=64/4 D=128 (the shape of the "
              "decode latencies in 'cuDNN Frontend v1.30.0 Release Notes', 'New: decode tiles')"),
    "paged_prefill": Workload(
        "paged_prefill", "paged", seed=6, B=16, Hq=32, Hkv=8, Dqk=128, Dv=128,
        lengths=(1024,), len_range=(8192, 65536), page_size=64, causal=True,
        notes="chunked prefill: 16 sequences, a 1024-token chunk at the end of a paged cache of "
              "U[8192, 65536] keys, page 64, H=32/8 D=128, bottom-right causal"),
    "mixed_batch": Workload(
        "mixed_batch", "paged", seed=7, B=64, Hq=32, Hkv=8, Dqk=128, Dv=128,
        lengths=(1024, 1, 2, 4), len_range=(4096, 32768), page_size=64, causal=True,
        notes="mixed decode / chunked-prefill batch over a paged cache: 64 sequences with cached "
              "lengths U[4096, 32768]; sequences 0-15 a 1024-query chunk, the other 48 decode rows "
              "of 1, 2, 4 queries in turn; page 64, H=32/8 D=128, bottom-right causal"),
    "mla_decode": Workload(
        "mla_decode", "paged", seed=5, B=64, Hq=128, Hkv=1, Dqk=576, Dv=512,
        len_range=(4096, 65536), page_size=64, causal=False, v_aliases_k=True,
        notes="absorbed-MLA paged decode B=64 kv U[4096, 65536] page 64, "
              "H=128/1, Dqk=576, Dv=512 (V = first 512 columns of K)"),
}


def make_ragged(w: Workload, device="cpu", lengths=None):
    """Packed THD tensors q [T, Hq, Dqk], k [T, Hkv, Dqk], v [T, Hkv, Dv] and
    the host offset table (q_len = kv_len per sequence)."""
    L = np.asarray(lengths if lengths is not None else w.seq_lengths(), dtype=np.int64)
    cu = cu_seqlens(L)
    T = int(cu[-1])
    q = normal_bf16((T, w.Hq, w.Dqk), w.seed * 10 + 1, device)
    k = normal_bf16((T, w.Hkv, w.Dqk), w.seed * 10 + 2, device)
    v = normal_bf16((T, w.Hkv, w.Dv), w.seed * 10 + 3, device)
    return q, k, v, cu


def make_dense(w: Workload, device="cpu", S=None, B=None):
    S = S or w.S
    B = B or w.B
    q = normal_bf16((B, S, w.Hq, w.Dqk), w.seed * 10 + 1, device)
    k = normal_bf16((B, S, w.Hkv, w.Dqk), w.seed * 10 + 2, device)
    v = normal_bf16((B, S, w.Hkv, w.Dv), w.seed * 10 + 3, device)
    return q, k, v


def make_paged_prefill(w: Workload, device="cpu", kv_lens=None):
    """Chunked-prefill inputs: q [B * chunk, Hq, D] packed (chunk = w.lengths[0]
    queries per sequence), HND pools, page table (host), kv_lens (host), cu_q."""
    L = np.asarray(kv_lens if kv_lens is not None else
                   uniform_lengths(w.B, w.len_range[0], w.len_range[1], w.seed), dtype=np.int64)
    chunk = int(w.lengths[0])
    lq = np.minimum(L, chunk)
    cu_q = cu_seqlens(lq)
    table, total = page_table(L, w.page_size, w.seed)
    q = normal_bf16((int(cu_q[-1]), w.Hq, w.Dqk), w.seed * 10 + 1, device)
    k_pool = normal_bf16((total, w.Hkv, w.page_size, w.Dqk), w.seed * 10 + 2, device)
    v_pool = normal_bf16((total, w.Hkv, w.page_size, w.Dv), w.seed * 10 + 3, device)
    return q, k_pool, v_pool, table, L.astype(np.int32), cu_q, lq


def make_paged(w: Workload, device="cpu", kv_lens=None, extra_pages: int = 0):
    """Paged decode inputs: q [B, Hq, Dqk], pools [P, Hkv, page, D] (HND order),
    page table [B, max_pages] int32 (host) and kv_lens (host).  With
    ``v_aliases_k`` the V pool is the K pool itself (V reads its first Dv columns)."""
    L = np.asarray(kv_lens if kv_lens is not None else w.seq_lengths(), dtype=np.int64)
    table, total = page_table(L, w.page_size, w.seed)
    P = total + extra_pages
    q = normal_bf16((len(L), w.Hq, w.Dqk), w.seed * 10 + 1, device)
    k_pool = normal_bf16((P, w.Hkv, w.page_size, w.Dqk), w.seed * 10 + 2, device)
    if w.v_aliases_k:
        v_pool = k_pool
    else:
        v_pool = normal_bf16((P, w.Hkv, w.page_size, w.Dv), w.seed * 10 + 3, device)
    return q, k_pool, v_pool, table, L.astype(np.int32)


def mixed_query_lengths(w: Workload, kv_lens, subset: str = "all"):
    """Query lengths of the mixed batch: sequences 0..B/4-1 take a chunk of
    w.lengths[0] queries, the others the short lengths w.lengths[1:] in turn
    (capped by each cached length).  subset: "all", "short" (chunks set to 0)
    or "chunks" (short rows set to 0)."""
    kv_lens = np.asarray(kv_lens, dtype=np.int64)
    n_chunk = w.B // 4
    short = list(w.lengths[1:])
    lq = np.array([w.lengths[0] if b < n_chunk else short[(b - n_chunk) % len(short)] for b in range(w.B)],
                  dtype=np.int64)
    if subset == "short":
        lq[:n_chunk] = 0
    elif subset == "chunks":
        lq[n_chunk:] = 0
    return np.minimum(lq, kv_lens)


def make_mixed_batch(w: Workload, device="cpu", subset: str = "all"):
    """Mixed-batch inputs: q [sum Lq, Hq, D] packed, HND pools, page table and
    kv_lens (host), cu_q and the query lengths (host).  Sequences a subset
    leaves out keep their cache but have no queries."""
    L = uniform_lengths(w.B, w.len_range[0], w.len_range[1], w.seed)
    lq = mixed_query_lengths(w, L, subset)
    cu_q = cu_seqlens(lq)
    table, total = page_table(L, w.page_size, w.seed)
    q = normal_bf16((max(1, int(cu_q[-1])), w.Hq, w.Dqk), w.seed * 10 + 1, device)
    k_pool = normal_bf16((total, w.Hkv, w.page_size, w.Dqk), w.seed * 10 + 2, device)
    v_pool = normal_bf16((total, w.Hkv, w.page_size, w.Dv), w.seed * 10 + 3, device)
    return q, k_pool, v_pool, table, L.astype(np.int32), cu_q, lq
