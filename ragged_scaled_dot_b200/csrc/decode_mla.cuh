// decode_mla.cuh -- absorbed-MLA paged decode on tcgen05 tensor cores.
//
// Shape: Dqk = 576 (512 latent + 64 rope columns), Dv = 512, every query head
// reads the single latent KV head, and V is the first 512 columns of the K rows
// (or comes from a pool of its own) ("cuDNN Frontend v1.32.0 Release Notes",
// "SDPA: wider native forward support").  With 128 query heads per KV byte the
// contraction does about 240 flop per byte, so the query heads are the M = 128
// rows of tcgen05 MMAs and the tensor core, not HBM alone, sets the pace.
//
// The accumulator O (128 heads x 512 fp32) fills one SM's tensor memory and
// leaves no room for scores, so a work unit (sequence b, split s, group of up
// to 128 heads) runs on a cluster of two CTAs:
//
//   rank 0, the score CTA: S = Q K^T per chunk of 128 keys (N = 128, K = 576;
//     the latent part of Q sits in TMEM as the A operand, the rope part in
//     shared memory), then the online softmax.  P (bf16, 128 x 128), the
//     per-row rescale factors and, with the last chunk, 1/l go to rank 1 as
//     one message: a bulk copy from a staging buffer into rank 1's shared
//     memory that completes on rank 1's mbarrier.
//   rank 1, the value CTA: O += P V in four 128-column quarters (N = 128,
//     K = 128 keys per chunk), O in TMEM; rescales O rows when a message asks
//     for it; writes O / 1/l (or the fp32 split partial).
//
// Per chunk the score CTA issues 36 MMAs and the value CTA 32, so the two
// tensor pipes are nearly balanced.  Both CTAs stream the same pages through
// TMA (box = min(page_size, 64) rows x 64 columns; the second read of a page
// hits L2).  Keys past the split's range read zeros (an out-of-range page
// coordinate); the value rows of the one partially valid box are zeroed in
// shared memory, so 0 * NaN from stale cache slots can not reach O.
//
// Split-KV, partial layout and the merge are those of decode.cuh.
#pragma once

#include "decode.cuh"

namespace b2 {

struct MlaTcCfg {
    static constexpr uint32_t SUB = 128u * 128u;         // 128 rows x 64 bf16 columns, 128B swizzle
    static constexpr int RK = 8;                         // score CTA: ring of K sub-tiles
    static constexpr int RV = 4;                         // value CTA: ring of V quarters (2 sub-tiles)
    static constexpr uint32_t MSG_ALPHA = 2 * SUB;       // float[128] rescale factor per row
    static constexpr uint32_t MSG_INVL = MSG_ALPHA + 512;  // float[128] 1/l (last chunk)
    static constexpr uint32_t MSG_HDR = MSG_INVL + 512;    // int[4]: flags (1 rescale, 2 last), chunk
    static constexpr uint32_t MSG_BYTES = MSG_HDR + 16;
    static constexpr uint32_t PSLOT = 34u * 1024u;       // one message slot, 1024-aligned
    // score CTA
    static constexpr uint32_t S_RING = 0;
    static constexpr uint32_t S_QR = RK * SUB;           // rope columns of Q
    static constexpr uint32_t S_STAGE = S_QR + SUB;      // two outgoing message buffers
    static constexpr uint32_t S_END = S_STAGE + 2 * PSLOT;
    // value CTA
    static constexpr uint32_t V_RING = 0;
    static constexpr uint32_t V_P = RV * 2 * SUB;        // two incoming message slots
    static constexpr uint32_t V_END = V_P + 2 * PSLOT;
    static constexpr uint32_t BAR_OFF = (S_END > V_END) ? S_END : V_END;
    static constexpr uint32_t SMEM = BAR_OFF + 256 + 1024;
    static constexpr int THREADS = 192;  // warp 0 TMA, warp 1 MMA, warps 2-5 softmax / O rescale + epilogue
    // barrier offsets from BAR_OFF
    // score CTA: kfull[RK] kempty[RK] sfull[2] sfree[2] pfree[2] qready drain
    static constexpr uint32_t B_KFULL = 0, B_KEMPTY = 64, B_SFULL = 128, B_SFREE = 144, B_PFREE = 160,
                              B_QREADY = 176, B_SDRAIN = 184;
    // value CTA: vfull[RV] vempty[RV] pfull[2] pvdone[2] rescaled vtail[4] drain.  Each vtail[q]
    // completes at most once (quarter q of the last chunk), so the producer can run
    // ahead of the MMA thread without two phases of one barrier completing unseen.
    static constexpr uint32_t B_VFULL = 0, B_VEMPTY = 32, B_PFULL = 64, B_PVDONE = 80, B_RESCALED = 96,
                              B_VTAIL = 104, B_VDRAIN = 136;
    static constexpr uint32_t MISC = 192;  // tmem address, abort flag
};
static_assert(MlaTcCfg::MSG_BYTES <= MlaTcCfg::PSLOT, "message slot");
static_assert(MlaTcCfg::SMEM <= 232448, "shared memory");

// TMA loads of the 128 rows (keys t0 .. t0+127) of one 64-column block; rows
// of keys at or past `hi` come from an out-of-range page and read as zeros.
__device__ __forceinline__ void mla_issue_rows(const DecodeParams& p, const CUtensorMap* map, uint32_t dst,
                                               uint32_t bar, int b, int col, int t0, int hi) {
    for (int r = 0; r < 128; r += p.box_rows) {
        const int t = t0 + r;
        int page = -1, slot = 0;
        if (t < hi) {
            page = __ldg(p.page_table + (int64_t)b * p.pt_stride + t / p.page_size);
            if (page < 0 || (int64_t)page >= p.num_pages) {
                record_status(ATTN_ERR_DEVICE_INPUT);
                page = -1;
            }
            slot = t % p.page_size;
        }
        tma_load_4d(dst + (uint32_t)r * 128u, map, bar, col, slot, 0, page);
    }
}

__global__ void __launch_bounds__(192, 1) decode_mla_tc_kernel(const __grid_constant__ DecodeParams p) {
    using C = MlaTcCfg;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t sb = (raw + 1023u) & ~1023u;
    uint8_t* sgen = smem_raw + (sb - raw);
    const uint32_t sBar = sb + C::BAR_OFF;
    volatile uint32_t* tmem_slot = reinterpret_cast<volatile uint32_t*>(sgen + C::BAR_OFF + C::MISC);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(sgen + C::BAR_OFF + C::MISC + 4);
    const uint32_t rank = cluster_ctarank();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    // work unit: (b, s, head group), consecutive units share b
    const int n_hg = (p.Hq + 127) >> 7;
    const int unit = (int)(blockIdx.x >> 1);
    const int hg = unit % n_hg;
    const int bs = unit / n_hg;
    const int s = bs % p.num_splits;
    const int b = bs / p.num_splits;
    const int nh = min(128, p.Hq - hg * 128);
    int L, lo, hi;
    decode_split_range(p, b, s, L, lo, hi);
    const int n_chunks = (hi > lo) ? (hi - lo + 127) / 128 : 0;
    const int nvalid_last = n_chunks ? hi - (lo + (n_chunks - 1) * 128) : 0;
    const bool tail = n_chunks > 0 && (nvalid_last % p.box_rows) != 0;

    if (threadIdx.x == 0) {
        if (rank == 0) {
            for (int i = 0; i < C::RK; ++i) {
                mbar_init(sBar + C::B_KFULL + 8 * i, 1);
                mbar_init(sBar + C::B_KEMPTY + 8 * i, 1);
            }
            for (int i = 0; i < 2; ++i) {
                mbar_init(sBar + C::B_SFULL + 8 * i, 1);
                mbar_init(sBar + C::B_SFREE + 8 * i, 4);
                mbar_init(sBar + C::B_PFREE + 8 * i, 1);
            }
            mbar_init(sBar + C::B_QREADY, 4);
            mbar_init(sBar + C::B_SDRAIN, 1);
        } else {
            for (int i = 0; i < C::RV; ++i) {
                mbar_init(sBar + C::B_VFULL + 8 * i, 1);
                mbar_init(sBar + C::B_VEMPTY + 8 * i, 1);
            }
            for (int i = 0; i < 2; ++i) {
                mbar_init(sBar + C::B_PFULL + 8 * i, 1);
                mbar_init(sBar + C::B_PVDONE + 8 * i, 1);
            }
            mbar_init(sBar + C::B_RESCALED, 4);
            for (int q = 0; q < 4; ++q) mbar_init(sBar + C::B_VTAIL + 8 * q, 1);
            mbar_init(sBar + C::B_VDRAIN, 1);
        }
        *abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == 1) {
        tmem_alloc(smem_u32((const void*)tmem_slot), 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncwarp();
    cluster_sync();  // both CTAs' barriers exist before any cross-CTA arrival or copy
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const float sl2 = p.scale_log2;

    if (rank == 0) {
        // ================================================================ score CTA
        if (warp == 0 && lane == 0) {
            prefetch_tmap(&p.tm_k);
            int ki = 0;
            bool ok = true;
            for (int j = 0; ok && j < n_chunks; ++j) {
                const int t0 = lo + j * 128;
                for (int c = 0; c < 9; ++c) {
                    const int st = ki % C::RK;
                    if (!mbar_wait(sBar + C::B_KEMPTY + 8 * st, ((ki / C::RK) & 1) ^ 1, abort_flag)) {
                        ok = false;
                        break;
                    }
                    mbar_arrive_expect_tx(sBar + C::B_KFULL + 8 * st, C::SUB);
                    mla_issue_rows(p, &p.tm_k, sb + C::S_RING + st * C::SUB, sBar + C::B_KFULL + 8 * st, b,
                                   c * 64, t0, hi);
                    ++ki;
                }
            }
            // every load issued lands before the block exits
            for (int kk = max(0, ki - C::RK); kk < ki; ++kk)
                mbar_wait(sBar + C::B_KFULL + 8 * (kk % C::RK), (kk / C::RK) & 1, nullptr, 100000000ull);
        } else if (warp == 1 && lane == 0) {
            constexpr uint32_t IDESC = idesc_bf16_f32(128, 128, false);
            const SmemDesc dK = smem_desc_sw128_split(sb + C::S_RING, 16, 1024);
            const SmemDesc dQr = smem_desc_sw128_split(sb + C::S_QR, 16, 1024);
            int ki = 0;
            bool ok = n_chunks > 0 && mbar_wait(sBar + C::B_QREADY, 0, abort_flag);
            tc_fence_after();
            for (int j = 0; ok && j < n_chunks; ++j) {
                const int ps = j & 1;
                if (!mbar_wait(sBar + C::B_SFREE + 8 * ps, ((j >> 1) & 1) ^ 1, abort_flag)) break;
                tc_fence_after();
                const uint32_t d = tmem + 128u * (uint32_t)ps;
                for (int c = 0; c < 9; ++c) {
                    const int st = ki % C::RK;
                    if (!mbar_wait(sBar + C::B_KFULL + 8 * st, (ki / C::RK) & 1, abort_flag)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const SmemDesc bk{dK.lo + ((st * C::SUB) >> 4), dK.hi};
                    if (c < 8) {
#pragma unroll
                        for (int kk = 0; kk < 4; ++kk)
                            tc_mma_ts(d, tmem + 256u + 32u * c + 8u * kk, desc_at(bk, kk * 32u), IDESC,
                                      (c | kk) ? 1u : 0u);
                    } else {
#pragma unroll
                        for (int kk = 0; kk < 4; ++kk)
                            tc_mma_ss(d, desc_at(dQr, kk * 32u), desc_at(bk, kk * 32u), IDESC, 1u);
                    }
                    tc_commit(sBar + C::B_KEMPTY + 8 * st);
                    ++ki;
                }
                if (!ok) break;
                tc_commit(sBar + C::B_SFULL + 8 * ps);
            }
            tc_commit(sBar + C::B_SDRAIN);
            mbar_wait(sBar + C::B_SDRAIN, 0, nullptr, 100000000ull);
        } else if (warp >= 2) {
            // -------------------------------------------------- Q load + softmax
            const int quad = warp & 3;
            const int r = quad * 32 + lane;
            const int tid = threadIdx.x - 64;
            const uint32_t lane_off = (uint32_t)(quad * 32) << 16;
            const int h = hg * 128 + r;
            const bool hv = r < nh;
            if (n_chunks > 0) {
                const __nv_bfloat16* qrow = p.q + (int64_t)b * p.q_bs + (int64_t)(hv ? h : 0) * p.q_hs;
                const uint4 z = make_uint4(0, 0, 0, 0);
#pragma unroll 1
                for (int c = 0; c < 8; ++c) {
                    uint32_t u[32];
#pragma unroll
                    for (int v = 0; v < 8; ++v) {
                        const uint4 w = hv ? __ldg(reinterpret_cast<const uint4*>(qrow + 64 * c + 8 * v)) : z;
                        u[4 * v + 0] = w.x;
                        u[4 * v + 1] = w.y;
                        u[4 * v + 2] = w.z;
                        u[4 * v + 3] = w.w;
                    }
                    tmem_st32(tmem + lane_off + 256u + 32u * c, u);
                }
                uint8_t* qr = sgen + C::S_QR + r * 128;
#pragma unroll
                for (int v = 0; v < 8; ++v) {
                    const uint4 w = hv ? __ldg(reinterpret_cast<const uint4*>(qrow + 512 + 8 * v)) : z;
                    *reinterpret_cast<uint4*>(qr + ((v ^ (r & 7)) << 4)) = w;
                }
                tc_wait_st();
                fence_proxy_async_smem();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(sBar + C::B_QREADY);
            }
            const bool pos = sl2 >= 0.f;
            const float NEG = pos ? -INFINITY : INFINITY;
            const uint32_t peer_slot0 = peer_smem(sb + C::V_P, 1);
            const uint32_t peer_pfull0 = peer_smem(sBar + C::B_PFULL, 1);
            float m_use = -INFINITY, l = 0.f;
            for (int j = 0; j < n_chunks; ++j) {
                const int ps = j & 1;
                bool okt = mbar_wait(sBar + C::B_SFULL + 8 * ps, (j >> 1) & 1, abort_flag);
                tc_fence_after();
                float x[128];
                {
                    uint32_t u0[32], u1[32], u2[32], u3[32];
                    const uint32_t tS = tmem + lane_off + 128u * (uint32_t)ps;
                    tmem_ld32(tS, u0);
                    tmem_ld32(tS + 32u, u1);
                    tmem_ld32(tS + 64u, u2);
                    tmem_ld32(tS + 96u, u3);
                    tc_wait_ld();
#pragma unroll
                    for (int e = 0; e < 32; ++e) {
                        x[e] = __uint_as_float(u0[e]);
                        x[32 + e] = __uint_as_float(u1[e]);
                        x[64 + e] = __uint_as_float(u2[e]);
                        x[96 + e] = __uint_as_float(u3[e]);
                    }
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(sBar + C::B_SFREE + 8 * ps);
                // the staging buffer of this parity is free once the value CTA released chunk j-2
                if (tid == 0)
                    okt = mbar_wait<true>(sBar + C::B_PFREE + 8 * ps, ((j >> 1) & 1) ^ 1, abort_flag) && okt;
                if (!bar_and(1, 128, okt)) break;

                const int nvalid = min(128, hi - (lo + j * 128));
                const bool masked = nvalid < 128;
                if (masked) {
#pragma unroll
                    for (int c = 0; c < 128; ++c) x[c] = (c < nvalid) ? x[c] : NEG;
                }
                float a0 = NEG, a1 = NEG, a2 = NEG, a3 = NEG;
                if (pos) {
#pragma unroll
                    for (int c = 0; c < 128; c += 8) {
                        a0 = fmax3(a0, x[c], x[c + 1]);
                        a1 = fmax3(a1, x[c + 2], x[c + 3]);
                        a2 = fmax3(a2, x[c + 4], x[c + 5]);
                        a3 = fmax3(a3, x[c + 6], x[c + 7]);
                    }
                    a0 = fmax3(a0, a1, fmaxf(a2, a3));
                } else {
#pragma unroll
                    for (int c = 0; c < 128; c += 8) {
                        a0 = fmin3(a0, x[c], x[c + 1]);
                        a1 = fmin3(a1, x[c + 2], x[c + 3]);
                        a2 = fmin3(a2, x[c + 4], x[c + 5]);
                        a3 = fmin3(a3, x[c + 6], x[c + 7]);
                    }
                    a0 = fmin3(a0, a1, fminf(a2, a3));
                }
                const float mx = (a0 == NEG) ? -INFINITY : a0 * sl2;
                const float m_new = fmaxf(m_use, mx);
                float alpha = 1.f;
                const bool old_finite = (m_use != -INFINITY);
                if (m_new > m_use + 8.f) {
                    alpha = ex2(m_use - m_new);
                    m_use = m_new;
                }
                const bool need = (j > 0) && old_finite && (alpha != 1.f);
                uint8_t* stg = sgen + C::S_STAGE + ps * C::PSLOT;
                *reinterpret_cast<float*>(stg + C::MSG_ALPHA + 4 * r) = alpha;
                const float mref = (m_use == -INFINITY) ? 0.f : m_use;
                const float2 sc2 = make_float2(sl2, sl2);
                const float2 nm2 = make_float2(-mref, -mref);
                float2 sum0 = make_float2(0.f, 0.f), sum1 = make_float2(0.f, 0.f);
#pragma unroll
                for (int g = 0; g < 4; ++g) {
                    uint32_t pk[16];
#pragma unroll
                    for (int e = 0; e < 16; ++e) {
                        const int col = 32 * g + 2 * e;
                        const float2 t = ffma2(make_float2(x[col], x[col + 1]), sc2, nm2);
                        float2 pv;
                        pv.x = ex2(t.x);
                        pv.y = ex2(t.y);
                        if (masked) {
                            pv.x = (col < nvalid) ? pv.x : 0.f;
                            pv.y = (col + 1 < nvalid) ? pv.y : 0.f;
                        }
                        if (e & 1) sum1 = fadd2(sum1, pv);
                        else sum0 = fadd2(sum0, pv);
                        pk[e] = pack_bf16(pv.x, pv.y);
                    }
                    // keys 32g .. 32g+31: half g/2, 16-byte chunks 4(g%2) .. 4(g%2)+3 of row r
                    uint8_t* rowp = stg + (g >> 1) * C::SUB + r * 128;
#pragma unroll
                    for (int v = 0; v < 4; ++v) {
                        const int chunk = (g & 1) * 4 + v;
                        *reinterpret_cast<uint4*>(rowp + ((chunk ^ (r & 7)) << 4)) =
                            make_uint4(pk[4 * v], pk[4 * v + 1], pk[4 * v + 2], pk[4 * v + 3]);
                    }
                }
                l = l * alpha + ((sum0.x + sum0.y) + (sum1.x + sum1.y));
                const bool last = (j == n_chunks - 1);
                if (last) *reinterpret_cast<float*>(stg + C::MSG_INVL + 4 * r) = (l > 0.f) ? 1.f / l : 0.f;
                fence_proxy_async_smem();
                const bool any = bar_or(1, 128, need);
                if (tid == 0) {
                    volatile int* hdr = reinterpret_cast<volatile int*>(stg + C::MSG_HDR);
                    hdr[0] = (any ? 1 : 0) | (last ? 2 : 0);
                    hdr[1] = j;
                    fence_proxy_async_smem();
                    const uint32_t bar = peer_pfull0 + 8u * (uint32_t)ps;
                    mbar_arrive_expect_tx_peer(bar, C::MSG_BYTES);
                    bulk_copy_to_peer(peer_slot0 + (uint32_t)ps * C::PSLOT, sb + C::S_STAGE + ps * C::PSLOT,
                                      C::MSG_BYTES, bar);
                }
            }
            if (hv) {
                const float lse = (l > 0.f) ? (m_use + log2f(l)) * 0.6931471805599453f : -INFINITY;
                if (p.num_splits == 1) {
                    if (p.lse != nullptr) p.lse[(int64_t)b * p.Hq + h] = lse;
                } else {
                    p.lse_part[(int64_t)s * p.B * p.Hq + (int64_t)b * p.Hq + h] = lse;
                }
            }
        }
    } else {
        // ================================================================ value CTA
        if (warp == 0 && lane == 0) {
            prefetch_tmap(&p.tm_v);
            int vi = 0;
            bool ok = true;
            for (int j = 0; ok && j < n_chunks; ++j) {
                const int t0 = lo + j * 128;
                for (int q = 0; q < 4; ++q) {
                    const int st = vi % C::RV;
                    const uint32_t full = sBar + C::B_VFULL + 8 * st;
                    if (!mbar_wait(sBar + C::B_VEMPTY + 8 * st, ((vi / C::RV) & 1) ^ 1, abort_flag)) {
                        ok = false;
                        break;
                    }
                    mbar_arrive_expect_tx(full, 2 * C::SUB);
                    const uint32_t dst = sb + C::V_RING + st * 2 * C::SUB;
                    mla_issue_rows(p, &p.tm_v, dst, full, b, 128 * q, t0, hi);
                    mla_issue_rows(p, &p.tm_v, dst + C::SUB, full, b, 128 * q + 64, t0, hi);
                    ++vi;
                    if (tail && j == n_chunks - 1) {
                        // zero the rows of the partially valid box that lie past the sequence
                        if (!mbar_wait(full, ((vi - 1) / C::RV) & 1, abort_flag)) {
                            ok = false;
                            break;
                        }
                        const int r1 = (nvalid_last + p.box_rows - 1) / p.box_rows * p.box_rows;
                        uint8_t* vq = sgen + C::V_RING + st * 2 * C::SUB;
                        for (int rr = nvalid_last; rr < r1; ++rr)
                            for (int i = 0; i < 16; ++i)
                                *reinterpret_cast<uint4*>(vq + (i >> 3) * C::SUB + rr * 128 + (i & 7) * 16) =
                                    make_uint4(0, 0, 0, 0);
                        fence_proxy_async_smem();
                        mbar_arrive(sBar + C::B_VTAIL + 8 * q);
                    }
                }
            }
            for (int kk = max(0, vi - C::RV); kk < vi; ++kk)
                mbar_wait(sBar + C::B_VFULL + 8 * (kk % C::RV), (kk / C::RV) & 1, nullptr, 100000000ull);
        } else if (warp == 1 && lane == 0) {
            constexpr uint32_t IDESC = idesc_bf16_f32(128, 128, true);
            const SmemDesc dP = smem_desc_sw128_split(sb + C::V_P, 16, 1024);
            const SmemDesc dV = smem_desc_sw128_split(sb + C::V_RING, 16384, 1024);
            int vi = 0, rs = 0;
            bool ok = true;
            for (int j = 0; ok && j < n_chunks; ++j) {
                const int ps = j & 1;
                if (!mbar_wait<true>(sBar + C::B_PFULL + 8 * ps, (j >> 1) & 1, abort_flag)) break;
                const int flags = *reinterpret_cast<volatile int*>(sgen + C::V_P + ps * C::PSLOT + C::MSG_HDR);
                if (j > 0 && (flags & 1)) {
                    if (!mbar_wait(sBar + C::B_RESCALED, rs & 1, abort_flag)) break;
                    ++rs;
                }
                tc_fence_after();
                const SmemDesc a0{dP.lo + ((ps * C::PSLOT) >> 4), dP.hi};
                for (int q = 0; q < 4; ++q) {
                    const int st = vi % C::RV;
                    if (!mbar_wait(sBar + C::B_VFULL + 8 * st, (vi / C::RV) & 1, abort_flag)) {
                        ok = false;
                        break;
                    }
                    if (tail && j == n_chunks - 1) {
                        if (!mbar_wait(sBar + C::B_VTAIL + 8 * q, 0, abort_flag)) {
                            ok = false;
                            break;
                        }
                    }
                    tc_fence_after();
                    const SmemDesc b0{dV.lo + ((st * 2 * C::SUB) >> 4), dV.hi};
                    const uint32_t d = tmem + 128u * (uint32_t)q;
#pragma unroll
                    for (int kk = 0; kk < 8; ++kk)
                        tc_mma_ss(d, desc_at(a0, (kk >> 2) * C::SUB + (kk & 3) * 32u), desc_at(b0, kk * 2048u),
                                  IDESC, (j > 0 || kk > 0) ? 1u : 0u);
                    tc_commit(sBar + C::B_VEMPTY + 8 * st);
                    ++vi;
                }
                if (!ok) break;
                tc_commit(sBar + C::B_PVDONE + 8 * ps);
            }
            tc_commit(sBar + C::B_VDRAIN);
            mbar_wait(sBar + C::B_VDRAIN, 0, nullptr, 100000000ull);
        } else if (warp >= 2) {
            // ------------------------------------------ O rescale, slot release, epilogue
            const int quad = warp & 3;
            const int r = quad * 32 + lane;
            const int tid = threadIdx.x - 64;
            const uint32_t lane_off = (uint32_t)(quad * 32) << 16;
            const uint32_t tO = tmem + lane_off;
            const int h = hg * 128 + r;
            const bool hv = r < nh;
            const uint32_t peer_pfree0 = peer_smem(sBar + C::B_PFREE, 0);
            float inv_l = 0.f;
            bool ok = true;
            for (int j = 0; j < n_chunks; ++j) {
                const int ps = j & 1;
                bool okt = true;
                if (tid == 0) okt = mbar_wait<true>(sBar + C::B_PFULL + 8 * ps, (j >> 1) & 1, abort_flag);
                if (!bar_and(1, 128, okt)) { ok = false; break; }
                const uint8_t* slot = sgen + C::V_P + ps * C::PSLOT;
                const int flags = *reinterpret_cast<const volatile int*>(slot + C::MSG_HDR);
                if (j > 0 && (flags & 1)) {
                    // O must hold every chunk before j when it is rescaled
                    okt = true;
                    if (tid == 0)
                        okt = mbar_wait(sBar + C::B_PVDONE + 8 * ((j - 1) & 1), ((j - 1) >> 1) & 1, abort_flag);
                    const bool ok2 = bar_and(1, 128, okt);
                    tc_fence_after();
                    const float a = *reinterpret_cast<const volatile float*>(slot + C::MSG_ALPHA + 4 * r);
                    if (ok2 && __any_sync(0xffffffffu, a != 1.f)) {
#pragma unroll 1
                        for (int c = 0; c < 16; ++c) {
                            uint32_t u[32];
                            tmem_ld32(tO + 32u * c, u);
                            tc_wait_ld();
#pragma unroll
                            for (int e = 0; e < 32; ++e) u[e] = __float_as_uint(__uint_as_float(u[e]) * a);
                            tmem_st32(tO + 32u * c, u);
                        }
                        tc_wait_st();
                    }
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(sBar + C::B_RESCALED);
                    if (!ok2) { ok = false; break; }
                }
                if (flags & 2) inv_l = *reinterpret_cast<const volatile float*>(slot + C::MSG_INVL + 4 * r);
                // hand the slot back once PV(j) has read it
                okt = true;
                if (tid == 0) okt = mbar_wait(sBar + C::B_PVDONE + 8 * ps, (j >> 1) & 1, abort_flag);
                if (!bar_and(1, 128, okt)) { ok = false; break; }
                if (tid == 0) mbar_arrive_peer(peer_pfree0 + 8u * (uint32_t)ps);
            }
            tc_fence_after();
            const int64_t row = (int64_t)s * p.B * p.Hq + (int64_t)b * p.Hq + h;
#pragma unroll 1
            for (int c = 0; c < 16; ++c) {
                uint32_t u[32];
                if (n_chunks > 0) {
                    tmem_ld32(tO + 32u * c, u);
                    tc_wait_ld();
                } else {
#pragma unroll
                    for (int e = 0; e < 32; ++e) u[e] = 0u;
                }
                if (!hv || !ok) continue;
                if (p.num_splits == 1) {
                    uint4* dst = reinterpret_cast<uint4*>(p.o + (int64_t)b * p.o_bs + (int64_t)h * p.o_hs + 32 * c);
#pragma unroll
                    for (int v4 = 0; v4 < 4; ++v4) {
                        uint4 w;
                        w.x = pack_bf16(__uint_as_float(u[8 * v4 + 0]) * inv_l, __uint_as_float(u[8 * v4 + 1]) * inv_l);
                        w.y = pack_bf16(__uint_as_float(u[8 * v4 + 2]) * inv_l, __uint_as_float(u[8 * v4 + 3]) * inv_l);
                        w.z = pack_bf16(__uint_as_float(u[8 * v4 + 4]) * inv_l, __uint_as_float(u[8 * v4 + 5]) * inv_l);
                        w.w = pack_bf16(__uint_as_float(u[8 * v4 + 6]) * inv_l, __uint_as_float(u[8 * v4 + 7]) * inv_l);
                        dst[v4] = w;
                    }
                } else {
                    float4* dst = reinterpret_cast<float4*>(p.o_part + row * 512 + 32 * c);
#pragma unroll
                    for (int v4 = 0; v4 < 8; ++v4)
                        dst[v4] = make_float4(__uint_as_float(u[4 * v4 + 0]) * inv_l, __uint_as_float(u[4 * v4 + 1]) * inv_l,
                                              __uint_as_float(u[4 * v4 + 2]) * inv_l, __uint_as_float(u[4 * v4 + 3]) * inv_l);
                }
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
    __syncwarp();
    cluster_sync();  // neither CTA exits while its peer may still arrive on its barriers
}

}  // namespace b2
