"""Pins for the fp64 oracle: checks against facts fixed by the mathematics, not
by the oracle's own formulas.

Each ``pin_*`` function takes an ``oracle.Oracle`` and raises AssertionError on a
mismatch.  ``tests/test_oracle_pins.py`` runs them on the real oracle;
``tests/test_oracle_mutants.py`` runs them on copies of the oracle with planted
mistakes and requires every mutant to fail at least one pin.

What pins what:
  * closed form "uniform scores" (scale = 0): O is the plain mean of the visible
    V rows and LSE = ln(#visible keys) -> pins the mask, the softmax
    normalisation, the PV sum and the natural-log LSE;
  * closed form "single key": O = V[0] exactly, LSE = scale * q.k0;
  * brute force on tiny integer inputs: LSE = ln(sum exp s_j) evaluated with
    Python's decimal module, no max shift;
  * library routine: torch's CPU attention kernel in float64 (output and natural
    log LSE), with K/V heads expanded by ``repeat_interleave`` for GQA;
  * invariants: ragged == per-sequence dense, paged == contiguous gather done with
    numpy indexing, split-merge == unsplit, GQA == MHA with replicated heads,
    decode rows under the bottom-right causal mask see every key.
"""
from __future__ import annotations

import math
from decimal import Decimal, getcontext

import numpy as np
import torch

import oracle as _oracle_mod


def _bits(x: torch.Tensor) -> np.ndarray:
    return x.to(torch.bfloat16).contiguous().view(torch.int16).numpy().view(np.uint16)


def _f64(bits: np.ndarray) -> np.ndarray:
    return (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def _rand_bf16(shape, seed):
    g = torch.Generator().manual_seed(seed)
    return torch.randn(shape, generator=g).to(torch.bfloat16)


def _torch_attn(q, k, v, scale, causal):
    """torch CPU attention kernel, float64, BHSD in/out.  Returns (O, LSE)."""
    out = torch.ops.aten._scaled_dot_product_flash_attention_for_cpu(
        q, k, v, 0.0, causal, scale=scale)
    return out[0], out[1]


def _all_ragged_rows(lengths, Hq):
    rows = []
    for b, L in enumerate(lengths):
        for h in range(Hq):
            for i in range(L):
                rows.append((b, h, i))
    return np.array(rows, dtype=np.int32).reshape(-1, 3)


# --------------------------------------------------------------------------- #
def pin_uniform_scores_mean(orc):
    """scale = 0: every visible key has the same score, so O = mean(V_visible)
    and LSE = ln(count).  Ragged, GQA 4/2, mixed Lq/Lkv incl. Lq > Lkv and 0."""
    Hq, Hkv, D = 4, 2, 16
    lq = [5, 9, 3, 4, 0]
    lkv = [5, 12, 1, 0, 3]
    cu_q = np.concatenate([[0], np.cumsum(lq)]).astype(np.int32)
    cu_k = np.concatenate([[0], np.cumsum(lkv)]).astype(np.int32)
    q = _bits(_rand_bf16((cu_q[-1], Hq, D), 11))
    k = _bits(_rand_bf16((max(cu_k[-1], 1), Hkv, D), 12))
    v = _bits(_rand_bf16((max(cu_k[-1], 1), Hkv, D), 13))
    vf = _f64(v)
    for causal in (False, True):
        rows = []
        for b in range(len(lq)):
            for h in range(Hq):
                for i in range(lq[b]):
                    rows.append((b, h, i))
        o, lse = orc.attn_ragged_rows(q, k, v, cu_q, cu_k, Hq, Hkv, 0.0, causal, rows)
        for r, (b, h, i) in enumerate(rows):
            g = h // (Hq // Hkv)
            if causal:
                # bottom-right: the diagonal ends at the last key for the last query
                n = int(np.clip(i + lkv[b] - lq[b] + 1, 0, lkv[b]))
            else:
                n = lkv[b]
            if n == 0:
                assert lse[r] == -math.inf and np.all(o[r] == 0.0), (b, h, i)
                continue
            mean = vf[cu_k[b]:cu_k[b] + n, g, :].mean(axis=0)
            assert np.allclose(o[r], mean, rtol=0, atol=1e-12), (causal, b, h, i)
            assert abs(lse[r] - math.log(n)) < 1e-12, (causal, b, h, i, lse[r], n)


def pin_single_key(orc):
    """One key: softmax weight 1, so O = V[0] bit-for-bit and LSE = scale q.k0."""
    D, scale = 32, 0.37
    q = _bits(_rand_bf16((1, 1, D), 21))
    k = _bits(_rand_bf16((1, 1, D), 22))
    v = _bits(_rand_bf16((1, 1, D), 23))
    cu = np.array([0, 1], dtype=np.int32)
    for causal in (False, True):
        o, lse = orc.attn_ragged_rows(q, k, v, cu, cu, 1, 1, scale, causal, [(0, 0, 0)])
        assert np.array_equal(o[0], _f64(v)[0, 0])
        want = scale * float(np.dot(_f64(q)[0, 0], _f64(k)[0, 0]))
        assert abs(lse[0] - want) < 1e-12


def pin_lse_brute_force(orc):
    """Tiny integer-valued inputs; LSE = ln(sum_j exp(s_j)) in 50-digit decimal."""
    getcontext().prec = 50
    rng = np.random.default_rng(7)
    Lq, Lkv, D, scale = 4, 6, 3, 0.5
    qi = rng.integers(-2, 3, (Lq, 1, D)).astype(np.float32)
    ki = rng.integers(-2, 3, (Lkv, 1, D)).astype(np.float32)
    vi = rng.integers(-3, 4, (Lkv, 1, D)).astype(np.float32)
    q, k, v = (_bits(torch.from_numpy(x)) for x in (qi, ki, vi))
    cu_q = np.array([0, Lq], dtype=np.int32)
    cu_k = np.array([0, Lkv], dtype=np.int32)
    rows = [(0, 0, i) for i in range(Lq)]
    for causal in (False, True):
        o, lse = orc.attn_ragged_rows(q, k, v, cu_q, cu_k, 1, 1, scale, causal, rows)
        for i in range(Lq):
            n = min(Lkv, i + Lkv - Lq + 1) if causal else Lkv
            s = [Decimal(scale) * sum(Decimal(int(qi[i, 0, d])) * Decimal(int(ki[j, 0, d]))
                                      for d in range(D)) for j in range(n)]
            e = [x.exp() for x in s]
            tot = sum(e)
            want_lse = float(tot.ln())
            want_o = [float(sum(e[j] * Decimal(int(vi[j, 0, d])) for j in range(n)) / tot)
                      for d in range(D)]
            assert abs(lse[i] - want_lse) < 1e-12, (causal, i, lse[i], want_lse)
            assert np.allclose(o[i], want_o, rtol=0, atol=1e-12), (causal, i)


def pin_torch_dense(orc):
    """Dense BSHD vs torch's CPU attention in float64 (GQA expanded by
    repeat_interleave, i.e. q head h uses kv head h // G)."""
    B, S, Hq, Hkv, D = 2, 37, 4, 2, 16
    q = _rand_bf16((B, S, Hq, D), 31)
    k = _rand_bf16((B, S, Hkv, D), 32)
    v = _rand_bf16((B, S, Hkv, D), 33)
    scale = 0.3
    rows = [(b, h, i) for b in range(B) for h in range(Hq) for i in range(S)]
    G = Hq // Hkv
    qt = q.double().permute(0, 2, 1, 3)
    kt = k.double().permute(0, 2, 1, 3).repeat_interleave(G, dim=1)
    vt = v.double().permute(0, 2, 1, 3).repeat_interleave(G, dim=1)
    for causal in (False, True):
        o, lse = orc.attn_dense_rows(_bits(q), _bits(k), _bits(v), S, S, Hq, Hkv, D, D,
                                     scale, causal, rows)
        to, tl = _torch_attn(qt, kt, vt, scale, causal)
        o_ref = to.permute(0, 2, 1, 3).reshape(-1)  # [B, S, Hq, D]
        o_got = np.zeros((B, S, Hq, D))
        l_got = np.zeros((B, Hq, S))
        for r, (b, h, i) in enumerate(rows):
            o_got[b, i, h] = o[r]
            l_got[b, h, i] = lse[r]
        assert np.allclose(o_got.reshape(-1), o_ref.numpy(), rtol=1e-12, atol=1e-12)
        assert np.allclose(l_got, tl.numpy(), rtol=1e-12, atol=1e-12)


def pin_bottom_right_rows(orc):
    """Sq != Skv, causal: row i of a bottom-right mask is plain (non-causal)
    attention over the first i + Skv - Sq + 1 keys; checked per row against
    torch's kernel on the truncated key set.  The last query row sees all keys."""
    Sq, Skv, H, D, scale = 7, 19, 2, 8, 0.4
    q = _rand_bf16((1, Sq, H, D), 41)
    k = _rand_bf16((1, Skv, H, D), 42)
    v = _rand_bf16((1, Skv, H, D), 43)
    rows = [(0, h, i) for h in range(H) for i in range(Sq)]
    o, lse = orc.attn_dense_rows(_bits(q), _bits(k), _bits(v), Sq, Skv, H, H, D, D,
                                 scale, True, rows)
    for r, (b, h, i) in enumerate(rows):
        n = i + Skv - Sq + 1
        qt = q[:, i:i + 1, h:h + 1].double().permute(0, 2, 1, 3)
        kt = k[:, :n, h:h + 1].double().permute(0, 2, 1, 3)
        vt = v[:, :n, h:h + 1].double().permute(0, 2, 1, 3)
        to, tl = _torch_attn(qt, kt, vt, scale, False)
        assert np.allclose(o[r], to.reshape(-1).numpy(), rtol=1e-12, atol=1e-12)
        assert abs(lse[r] - float(tl.reshape(-1)[0])) < 1e-12
    # the last row equals the non-causal result
    o_nc, lse_nc = orc.attn_dense_rows(_bits(q), _bits(k), _bits(v), Sq, Skv, H, H, D, D,
                                       scale, False, [(0, 0, Sq - 1)])
    assert np.array_equal(o_nc[0], o[Sq - 1]) and lse_nc[0] == lse[Sq - 1]


def pin_ragged_equals_dense(orc):
    """A ragged batch equals each sequence run on its own as a dense B=1 problem,
    and both equal torch's kernel (equal q/kv lengths, causal, GQA 4/1)."""
    lens = [37, 64, 1, 5]
    Hq, Hkv, D, scale = 4, 1, 16, 0.125
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    T = int(cu[-1])
    q = _rand_bf16((T, Hq, D), 51)
    k = _rand_bf16((T, Hkv, D), 52)
    v = _rand_bf16((T, Hkv, D), 53)
    rows = _all_ragged_rows(lens, Hq)
    o, lse = orc.attn_ragged_rows(_bits(q), _bits(k), _bits(v), cu, cu, Hq, Hkv,
                                  scale, True, rows)
    r = 0
    for b, L in enumerate(lens):
        sl = slice(int(cu[b]), int(cu[b + 1]))
        qb, kb, vb = q[sl], k[sl], v[sl]
        rws = [(0, h, i) for h in range(Hq) for i in range(L)]
        od, ld = orc.attn_dense_rows(_bits(qb), _bits(kb), _bits(vb), L, L, Hq, Hkv,
                                     D, D, scale, True, rws)
        n = len(rws)
        assert np.array_equal(o[r:r + n], od) and np.array_equal(lse[r:r + n], ld)
        qt = qb.double().unsqueeze(0).permute(0, 2, 1, 3)
        kt = kb.double().unsqueeze(0).permute(0, 2, 1, 3).repeat_interleave(Hq // Hkv, 1)
        vt = vb.double().unsqueeze(0).permute(0, 2, 1, 3).repeat_interleave(Hq // Hkv, 1)
        to, tl = _torch_attn(qt, kt, vt, scale, True)
        assert np.allclose(od, to[0].reshape(-1, D).numpy(), rtol=1e-12, atol=1e-12)
        assert np.allclose(ld, tl[0].reshape(-1).numpy(), rtol=1e-12, atol=1e-12)
        r += n


def _paged_case(seed, Hkv=2, G=3, D=16, Dv=16, ps=4, lens=(0, 1, 4, 9, 13)):
    rng = np.random.default_rng(seed)
    B = len(lens)
    n_pages = [-(-L // ps) for L in lens]
    P = sum(n_pages) + 3
    perm = rng.permutation(P)
    mp = max(max(n_pages), 1)
    table = np.full((B, mp), -1, dtype=np.int32)
    pos = 0
    for b, n in enumerate(n_pages):
        table[b, :n] = perm[pos:pos + n]
        pos += n
    Hq = Hkv * G
    q = _rand_bf16((B, Hq, D), seed + 1)
    kp = _rand_bf16((P, ps, Hkv, D), seed + 2)     # NHD pool: (page, slot, head)
    vp = _rand_bf16((P, ps, Hkv, Dv), seed + 3)
    ks = (ps * Hkv * D, Hkv * D, D)
    vs = (ps * Hkv * Dv, Hkv * Dv, Dv)
    return dict(q=q, kp=kp, vp=vp, table=table, lens=np.array(lens, dtype=np.int32),
                ps=ps, Hq=Hq, Hkv=Hkv, D=D, Dv=Dv, ks=ks, vs=vs)


def pin_paged_equals_gathered(orc):
    """Paged decode equals contiguous attention over the K/V rows gathered with
    numpy indexing (page = table[b, t // ps], slot = t % ps), bit-for-bit."""
    c = _paged_case(61)
    scale = 0.25
    Hq, Hkv, D, Dv, ps = c["Hq"], c["Hkv"], c["D"], c["Dv"], c["ps"]
    rows = [(b, h) for b in range(len(c["lens"])) for h in range(Hq)]
    o, lse = orc.attn_paged_rows(_bits(c["q"]), _bits(c["kp"]), _bits(c["vp"]),
                                 c["table"], c["lens"], ps, Hq, Hkv, D, Dv,
                                 c["ks"], c["vs"], scale, rows)
    for r, (b, h) in enumerate(rows):
        L = int(c["lens"][b])
        t = np.arange(L)
        pages = c["table"][b, t // ps]
        kg = c["kp"][torch.from_numpy(pages.astype(np.int64)), torch.from_numpy(t % ps)]
        vg = c["vp"][torch.from_numpy(pages.astype(np.int64)), torch.from_numpy(t % ps)]
        cu = np.array([0, L], dtype=np.int32)
        cq = np.array([0, 1], dtype=np.int32)
        og, lg = orc.attn_ragged_rows(_bits(c["q"][b:b + 1]), _bits(kg), _bits(vg),
                                      cq, cu, Hq, Hkv, scale, False, [(0, h, 0)])
        assert np.array_equal(o[r], og[0]) and (lse[r] == lg[0]), (b, h)


def pin_decode_sees_all_keys(orc):
    """One query row with the bottom-right causal mask sees every key: equal to
    the non-causal result (the decode reading of the mask)."""
    L, H, D = 23, 2, 8
    q = _bits(_rand_bf16((1, H, D), 71))
    k = _bits(_rand_bf16((L, H, D), 72))
    v = _bits(_rand_bf16((L, H, D), 73))
    cq = np.array([0, 1], dtype=np.int32)
    ck = np.array([0, L], dtype=np.int32)
    rows = [(0, h, 0) for h in range(H)]
    a = orc.attn_ragged_rows(q, k, v, cq, ck, H, H, 0.3, True, rows)
    b = orc.attn_ragged_rows(q, k, v, cq, ck, H, H, 0.3, False, rows)
    assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1])


def pin_split_merge(orc):
    """Merging split-KV partials reproduces attention over the whole sequence,
    for several split counts incl. more splits than pages (empty splits, -inf).
    Closed forms: two equal partials -> LSE + ln 2 and the average of the O's;
    all partials empty -> O = 0, LSE = -inf."""
    c = _paged_case(81, lens=(0, 3, 8, 17, 33))
    scale = 0.2
    Hq, Hkv, D, Dv, ps = c["Hq"], c["Hkv"], c["D"], c["Dv"], c["ps"]
    B = len(c["lens"])
    rows = [(b, h) for b in range(B) for h in range(Hq)]
    args = (_bits(c["q"]), _bits(c["kp"]), _bits(c["vp"]), c["table"], c["lens"], ps,
            Hq, Hkv, D, Dv, c["ks"], c["vs"], scale)
    o_full, lse_full = orc.attn_paged_rows(*args, rows)
    for S in (1, 2, 3, 7, 12):
        o_part = np.zeros((S, len(rows), Dv))
        l_part = np.zeros((S, len(rows)))
        for s in range(S):
            lo = [_oracle_mod.split_ranges(int(c["lens"][b]), ps, S)[s][0] for b, _ in rows]
            hi = [_oracle_mod.split_ranges(int(c["lens"][b]), ps, S)[s][1] for b, _ in rows]
            o_part[s], l_part[s] = orc.attn_paged_rows(*args, rows, key_lo=lo, key_hi=hi)
        om, lm = orc.split_merge(o_part, l_part)
        fin = np.isfinite(lse_full)
        assert np.array_equal(np.isfinite(lm), fin)
        assert np.allclose(om, o_full, rtol=1e-12, atol=1e-13), S
        assert np.allclose(lm[fin], lse_full[fin], rtol=1e-12, atol=1e-12), S
        assert np.all(om[~fin] == 0.0)
    rng = np.random.default_rng(5)
    oa = rng.standard_normal((1, 3, 4))
    ob = rng.standard_normal((1, 3, 4))
    la = np.array([[0.3, -2.0, 5.0]])
    om, lm = orc.split_merge(np.concatenate([oa, ob]), np.concatenate([la, la]))
    assert np.allclose(lm, la[0] + math.log(2.0), atol=1e-14)
    assert np.allclose(om, (oa[0] + ob[0]) / 2, atol=1e-14)
    om, lm = orc.split_merge(np.full((3, 2, 4), np.nan), np.full((3, 2), -np.inf))
    assert np.all(om == 0.0) and np.all(lm == -np.inf)


def pin_gqa_equals_replicated_mha(orc):
    """GQA (Hq = 6, Hkv = 2) equals MHA with each kv head repeated G = 3 times
    consecutively (query head h reads kv head h // G)."""
    lens = [6, 11]
    Hq, Hkv, D, scale = 6, 2, 8, 0.5
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    T = int(cu[-1])
    q = _rand_bf16((T, Hq, D), 91)
    k = _rand_bf16((T, Hkv, D), 92)
    v = _rand_bf16((T, Hkv, D), 93)
    rows = _all_ragged_rows(lens, Hq)
    o, lse = orc.attn_ragged_rows(_bits(q), _bits(k), _bits(v), cu, cu, Hq, Hkv,
                                  scale, True, rows)
    k_rep = k.repeat_interleave(Hq // Hkv, dim=1)
    v_rep = v.repeat_interleave(Hq // Hkv, dim=1)
    o2, lse2 = orc.attn_ragged_rows(_bits(q), _bits(k_rep), _bits(v_rep), cu, cu, Hq, Hq,
                                    scale, True, rows)
    assert np.array_equal(o, o2) and np.array_equal(lse, lse2)


def pin_strided_views(orc):
    """Strided THD views (gaps between tokens and between heads) give the same
    result as the compact copy of the same values."""
    lens = [5, 7]
    Hq, Hkv, D = 2, 1, 8
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    T = int(cu[-1])
    big_q = _rand_bf16((T, Hq + 1, D + 8), 101)
    big_k = _rand_bf16((T, Hkv + 2, D + 4), 102)
    big_v = _rand_bf16((T, Hkv + 2, D + 4), 103)
    q = big_q[:, :Hq, :D]
    k = big_k[:, 1:1 + Hkv, :D]
    v = big_v[:, 1:1 + Hkv, :D]
    rows = _all_ragged_rows(lens, Hq)
    o1, l1 = orc.attn_ragged_rows(_bits(q.contiguous()), _bits(k.contiguous()),
                                  _bits(v.contiguous()), cu, cu, Hq, Hkv, 0.3, True, rows)
    qb, kb, vb = _bits(big_q), _bits(big_k), _bits(big_v)
    # Flat-buffer form: the oracle reads element (t, h, d) at base + t*ts + h*hs + d.
    o3, l3 = _strided_ragged(orc, qb, kb, vb, cu, Hq, Hkv, D, 0.3, rows,
                             ((Hq + 1) * (D + 8), D + 8, 0),
                             ((Hkv + 2) * (D + 4), D + 4, D + 4),
                             ((Hkv + 2) * (D + 4), D + 4, D + 4))
    assert np.array_equal(o1, o3) and np.array_equal(l1, l3)


def _strided_ragged(orc, qb, kb, vb, cu, Hq, Hkv, D, scale, rows, qs, ks, vs):
    """Call the ragged oracle on flat buffers with (token, head) strides and a
    base offset (third entry) into each buffer."""
    qf = np.ascontiguousarray(qb.reshape(-1)[qs[2]:])
    kf = np.ascontiguousarray(kb.reshape(-1)[ks[2]:])
    vf = np.ascontiguousarray(vb.reshape(-1)[vs[2]:])
    # the wrapper reads Dqk / Dv from the last axis
    pad = (-len(qf)) % D
    qf = np.concatenate([qf, np.zeros(pad, np.uint16)]).reshape(-1, D)
    pad = (-len(kf)) % D
    kf = np.concatenate([kf, np.zeros(pad, np.uint16)]).reshape(-1, D)
    pad = (-len(vf)) % D
    vf = np.concatenate([vf, np.zeros(pad, np.uint16)]).reshape(-1, D)
    return orc.attn_ragged_rows(qf, kf, vf, cu, cu, Hq, Hkv, scale, True, rows,
                                q_strides=qs[:2], k_strides=ks[:2], v_strides=vs[:2])


ALL_PINS = [
    pin_uniform_scores_mean,
    pin_single_key,
    pin_lse_brute_force,
    pin_torch_dense,
    pin_bottom_right_rows,
    pin_ragged_equals_dense,
    pin_paged_equals_gathered,
    pin_decode_sees_all_keys,
    pin_split_merge,
    pin_gqa_equals_replicated_mha,
    pin_strided_views,
]
