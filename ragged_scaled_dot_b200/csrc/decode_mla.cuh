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
// to 128 heads) runs on a cluster of two CTAs, one 64-key chunk at a time:
//
//   rank 0, the score CTA: S = Q K^T (N = R keys per page box, K = 576; all of
//     Q sits in TMEM as the A operand), then the online softmax.  P (bf16,
//     128 x 64), the per-row rescale factors and 1/l (read with the last
//     chunk) go to rank 1 as one message: the softmax threads store it
//     straight into rank 1's shared memory with st.async, every store
//     counting its bytes on rank 1's mbarrier.
//   rank 1, the value CTA: O += P V in four 128-column quarters (N = 128,
//     K = 64 keys), O in TMEM; rescales O rows when a message asks for it;
//     writes O / 1/l (or the fp32 split partial).
//
// Loads: a page box covers R = min(page_size, 64) rows and several adjacent
// 64-column blocks of each row: all 9 blocks of a page's K rows per score-CTA
// load and the 8 value blocks per value-CTA load, so each TMA request reads a
// whole cache row.  The K boxes land group-major ([8-row group][column block]
// [8 rows][128 B]), so every ring slot is one uniform N = 64 MMA operand and
// two adjacent slots one N = 128 operand.  Measured on B200, one SM streams about 220 GB/s with such boxes but
// only 60 GB/s with boxes of one 64-column block (128-byte pieces of 1152-byte
// rows) and 80 GB/s with three; the smaller boxes left the kernel load-bound.
// Both CTAs stream the same pages (the second read hits L2); page ids are
// fetched a chunk ahead of the loads that use them.  Keys past the split's range read
// zeros (an out-of-range page coordinate); the value rows of the one
// partially valid box are zeroed in shared memory, so 0 * NaN from stale
// cache slots can not reach O.
//
// Split-KV, partial layout and the merge are those of decode.cuh.
#pragma once

#include "decode.cuh"

namespace b2 {

struct MlaTcCfg {
    // A 64-key chunk; R = min(page_size, 64) rows per page box, 64 / R pages per chunk.
    static constexpr uint32_t BLK = 64u * 128u;          // 64 rows x 64 bf16 columns (R = 64)
    static constexpr int KB = 9;                         // K column blocks per score-CTA load (9 per row)
    static constexpr int VB = 8;                         // V column blocks per value-CTA load (8 per row)
    static constexpr int KLOADS = 9 / KB, VLOADS = 8 / VB;  // loads per chunk (K: one, group-major)
    static constexpr uint32_t KSLOT = KB * BLK;          // 64 K rows group-major: [8 groups][9 blocks][8 rows][128 B]
    static constexpr uint32_t VSLOT = VB * BLK;          // [page][VB blocks][R rows][128 B]
    static constexpr int RK = 3;                         // score CTA ring (loads in flight)
    static constexpr int RV = 2;                         // value CTA ring
    static constexpr uint32_t P_TILE = 128u * 128u;      // P: 128 heads x 64 keys bf16, 128B swizzle
    static constexpr uint32_t MSG_ALPHA = P_TILE;        // float[128] rescale factor per row
    static constexpr uint32_t MSG_INVL = MSG_ALPHA + 512;  // float[128] 1/l (last chunk)
    static constexpr uint32_t MSG_HDR = MSG_INVL + 512;    // int[4]: flags (1 rescale, 2 last), chunk
    static constexpr uint32_t MSG_BYTES = MSG_HDR + 16;
    static constexpr uint32_t PSLOT = 18u * 1024u;       // one message slot, 1024-aligned
    // score CTA: the K ring only (messages are stored straight into the value CTA's slots)
    static constexpr uint32_t S_RING = 0;
    static constexpr uint32_t S_END = RK * KSLOT;
    // value CTA
    static constexpr uint32_t V_RING = 0;
    static constexpr uint32_t V_P = RV * VSLOT;          // two incoming message slots
    static constexpr uint32_t V_END = V_P + 2 * PSLOT;
    static constexpr uint32_t BAR_OFF = (S_END > V_END) ? S_END : V_END;
    static constexpr uint32_t XCH_OFF = BAR_OFF + 256;   // float[2][128] per-half row maxima, then sums
    static constexpr uint32_t SMEM = XCH_OFF + 2048 + 1024;
    // warp 0 TMA, warp 1 MMA, warps 2-9 softmax (score CTA) or O rescale + epilogue (value CTA):
    // two warps per TMEM lane quadrant, each on half of the columns
    static constexpr int THREADS = 320;
    static constexpr int NW = 256;  // threads of the softmax / epilogue warps
    // score CTA TMEM: S0 [0,64) S1 [64,128) Q [128,416) (576 bf16 per row, packed in pairs)
    static constexpr uint32_t T_Q = 128;
    // barrier offsets from BAR_OFF
    // score CTA: kfull[RK] kempty[RK] sfull[2] sfree[2] pfree[2] qready drain
    static constexpr uint32_t B_KFULL = 0, B_KEMPTY = 64, B_SFULL = 128, B_SFREE = 144, B_PFREE = 160,
                              B_QREADY = 176, B_SDRAIN = 184;
    // value CTA: vfull[RV] vempty[RV] pfull[2] pvdone[2] rescaled vtail[2] drain.  Each vtail[h]
    // completes at most once (half h of the last chunk), so the producer can run ahead of
    // the MMA thread without two phases of one barrier completing unseen.
    static constexpr uint32_t B_VFULL = 0, B_VEMPTY = 64, B_PFULL = 128, B_PVDONE = 144, B_RESCALED = 160,
                              B_VTAIL = 168, B_VDRAIN = 184;
    static constexpr uint32_t MISC = 192;  // tmem address, abort flag
};
static_assert(MlaTcCfg::MSG_BYTES <= MlaTcCfg::PSLOT, "message slot");
static_assert(MlaTcCfg::SMEM <= 232448, "shared memory");
static_assert(MlaTcCfg::RK <= 8 && MlaTcCfg::RV <= 8, "barrier area");
static_assert(MlaTcCfg::KB == 9 && MlaTcCfg::KLOADS == 1, "one group-major K load per chunk");
static_assert(9 % MlaTcCfg::KB == 0 && 8 % MlaTcCfg::VB == 0 && MlaTcCfg::VB % 2 == 0 && MlaTcCfg::VLOADS <= 2, "blocks");

// Page ids of the np = 64 / R page boxes of the chunk starting at key t0.  The
// loads are only issued here; the producer fetches the next chunk's ids while
// it issues the current chunk's boxes.  Bit i of the result: box i holds keys
// of the split.
__device__ __forceinline__ uint32_t mla_fetch_pages(const DecodeParams& p, const int32_t* table, int64_t table_stride,
                                                    int b, int t0, int hi, int np, int (&pg)[4]) {
    uint32_t live = 0;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int t = t0 + i * p.box_rows;
        pg[i] = -1;
        if (i < np && t < hi) {
            pg[i] = page_lookup(table, table_stride, b, t, p.page_size);
            live |= 1u << i;
        }
    }
    return live;
}

// The score CTA's K load of a chunk: box i (R rows, all 9 column blocks) lands
// at dst + i * R * 1152 group-major, [8-row group][column block][8 rows][128 B],
// so a slot's 64 rows are 8 groups 9 KB apart whatever the page size.  Boxes
// past the split, or with an out-of-range page id (recorded as an input
// error), start at a negative group coordinate and read as zeros.
__device__ __forceinline__ void mla_issue_k(const DecodeParams& p, uint32_t dst, uint32_t bar, int t0, int np,
                                            const int (&pg)[4], uint32_t live) {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        if (i < np) {
            int grp = -(p.box_rows / 8);
            if ((live >> i) & 1u) {
                const int page = page_checked(pg[i], p.num_pages);
                if (page >= 0) grp = page_group(page, page_slot(t0 + i * p.box_rows, p.page_size), p.groups_per_page);
            }
            tma_load_5d(dst + (uint32_t)(i * p.box_rows) * 1152u, &p.tm_k, bar, 0, 0, 0, grp, 0);
        }
    }
}

// One load of `nblk` column blocks starting at block blk0 for every page box
// of the chunk: box i lands at dst + i * nblk * R * 128.  Boxes past the split,
// or with an out-of-range page id (recorded as an input error), use page
// coordinate -1 and read as zeros.
__device__ __forceinline__ void mla_issue(const DecodeParams& p, const CUtensorMap* map, uint32_t dst, uint32_t bar,
                                          int blk0, int nblk, int t0, int np, const int (&pg)[4], uint32_t live) {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        if (i < np) {
            int page = -1, tok = 0;
            if ((live >> i) & 1u) {
                page = page_checked(pg[i], p.num_pages);
                if (page >= 0) tok = page_slot(t0 + i * p.box_rows, p.page_size);
            }
            tma_load_5d(dst + (uint32_t)(i * nblk * p.box_rows) * 128u, map, bar, 0, tok, blk0, 0, page);
        }
    }
}

__global__ void __launch_bounds__(320, 1) decode_mla_tc_kernel(const __grid_constant__ DecodeParams p) {
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
    const int b = p.order ? __ldg(p.order + bs / p.num_splits) : bs / p.num_splits;
    const int nh = min(128, p.Hq - hg * 128);
    int L, lo, hi;
    decode_split_range(p, b, s, L, lo, hi);
    const int R = p.box_rows;  // rows per page box: 16, 32 or 64
    const int np = 64 / R;     // page boxes per 64-key chunk
    const int n_chunks = (hi > lo) ? (hi - lo + 63) / 64 : 0;
    const int nvalid_last = n_chunks ? hi - (lo + (n_chunks - 1) * 64) : 0;
    const bool tail = n_chunks > 0 && (nvalid_last % R) != 0;

    if (threadIdx.x == 0) {
        if (rank == 0) {
            for (int i = 0; i < C::RK; ++i) {
                mbar_init(sBar + C::B_KFULL + 8 * i, 1);
                mbar_init(sBar + C::B_KEMPTY + 8 * i, 1);
            }
            for (int i = 0; i < 2; ++i) {
                mbar_init(sBar + C::B_SFULL + 8 * i, 1);
                mbar_init(sBar + C::B_SFREE + 8 * i, 8);
                mbar_init(sBar + C::B_PFREE + 8 * i, 1);
            }
            mbar_init(sBar + C::B_QREADY, 8);
            mbar_init(sBar + C::B_SDRAIN, 1);
        } else {
            for (int i = 0; i < C::RV; ++i) {
                mbar_init(sBar + C::B_VFULL + 8 * i, 1);
                mbar_init(sBar + C::B_VEMPTY + 8 * i, 1);
            }
            for (int i = 0; i < 2; ++i) {
                mbar_init(sBar + C::B_PFULL + 8 * i, 1);
                mbar_init(sBar + C::B_PVDONE + 8 * i, 1);
                mbar_init(sBar + C::B_VTAIL + 8 * i, 1);
            }
            mbar_init(sBar + C::B_RESCALED, 8);
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
            int pc[4], pn[4];
            uint32_t lc = 0;
            uint32_t ln = (n_chunks > 0) ? mla_fetch_pages(p, p.page_table, p.pt_stride, b, lo, hi, np, pn) : 0u;
            int ki = 0;
            bool ok = true;
            for (int j = 0; ok && j < n_chunks; ++j) {
                const int t0 = lo + j * 64;
#pragma unroll
                for (int i = 0; i < 4; ++i) pc[i] = pn[i];
                lc = ln;
                if (j + 1 < n_chunks) ln = mla_fetch_pages(p, p.page_table, p.pt_stride, b, t0 + 64, hi, np, pn);
                for (int t = 0; t < C::KLOADS; ++t) {
                    const int st = ki % C::RK;
                    if (!mbar_wait(sBar + C::B_KEMPTY + 8 * st, ((ki / C::RK) & 1) ^ 1, abort_flag)) {
                        ok = false;
                        break;
                    }
                    mbar_arrive_expect_tx(sBar + C::B_KFULL + 8 * st, C::KSLOT);
                    mla_issue_k(p, sb + C::S_RING + st * C::KSLOT, sBar + C::B_KFULL + 8 * st, t0, np, pc, lc);
                    ++ki;
                }
            }
            // every load issued lands before the block exits
            for (int kk = max(0, ki - C::RK); kk < ki; ++kk)
                mbar_wait(sBar + C::B_KFULL + 8 * (kk % C::RK), (kk / C::RK) & 1, nullptr, 100000000ull);
        } else if (warp == 1 && lane == 0) {
            // K slots are group-major: 8-row groups 9 KB apart, column blocks 1 KB apart.  A
            // chunk is one N = 64 operand at any page size, and an even chunk whose successor
            // sits in the next slot forms with it one N = 128 operand (16 groups 9 KB apart)
            // whose scores fill both S buffers: half the MMAs for two of every three pairs.
            const uint32_t IDESC64 = idesc_bf16_f32(128, 64, false);
            const uint32_t IDESC128 = idesc_bf16_f32(128, 128, false);
            const SmemDesc dK = smem_desc_sw128_split(sb + C::S_RING, 16, 9u * 1024u);
            bool ok = n_chunks > 0 && mbar_wait(sBar + C::B_QREADY, 0, abort_flag);
            tc_fence_after();
            for (int j = 0; ok && j < n_chunks;) {
                const int st = j % C::RK;  // one K load per chunk: load index = chunk index
                const bool pair = (j & 1) == 0 && j + 1 < n_chunks && st + 1 < C::RK;
                const int nc = pair ? 2 : 1;
                for (int q = 0; ok && q < nc; ++q) {
                    const int jj = j + q;
                    ok = mbar_wait(sBar + C::B_SFREE + 8 * (jj & 1), ((jj >> 1) & 1) ^ 1, abort_flag) &&
                         mbar_wait(sBar + C::B_KFULL + 8 * (jj % C::RK), (jj / C::RK) & 1, abort_flag);
                }
                if (!ok) break;
                tc_fence_after();
                const uint32_t d = tmem + 64u * (uint32_t)(j & 1);
                const uint32_t base = (uint32_t)st * C::KSLOT;
                for (int c = 0; c < 9; ++c) {
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)
                        tc_mma_ts(d, tmem + C::T_Q + 32u * c + 8u * kk, desc_at(dK, base + (uint32_t)c * 1024u + kk * 32u),
                                  pair ? IDESC128 : IDESC64, (c | kk) ? 1u : 0u);
                }
                for (int q = 0; q < nc; ++q) {
                    tc_commit(sBar + C::B_KEMPTY + 8 * ((j + q) % C::RK));
                    tc_commit(sBar + C::B_SFULL + 8 * ((j + q) & 1));
                }
                j += nc;
            }
            tc_commit(sBar + C::B_SDRAIN);
            mbar_wait(sBar + C::B_SDRAIN, 0, nullptr, 100000000ull);
        } else if (warp >= 2) {
            // -------------------------------------------------- Q load + softmax
            // thread = (row r, column half hf): columns [32 hf, 32 hf + 32) of the 64-key chunk
            const int quad = warp & 3;
            const int hf = (warp - 2) >> 2;
            const int r = quad * 32 + lane;
            const int tid = threadIdx.x - 64;
            const uint32_t lane_off = (uint32_t)(quad * 32) << 16;
            const int h = hg * 128 + r;
            const bool hv = r < nh;
            volatile float* xmax = reinterpret_cast<volatile float*>(sgen + C::XCH_OFF);         // [2][128]
            volatile float* xsum = reinterpret_cast<volatile float*>(sgen + C::XCH_OFF + 1024);  // [2][128]
            if (n_chunks > 0) {
                // Q row (576 bf16) into TMEM columns [T_Q, T_Q + 288), two values per column;
                // half 0 writes column blocks 0-4, half 1 blocks 5-8
                const __nv_bfloat16* qrow = p.q + (int64_t)b * p.q_bs + (int64_t)(hv ? h : 0) * p.q_hs;
                const uint4 z = make_uint4(0, 0, 0, 0);
#pragma unroll 1
                for (int c = hf ? 5 : 0; c < (hf ? 9 : 5); ++c) {
                    uint32_t u[32];
#pragma unroll
                    for (int v = 0; v < 8; ++v) {
                        const uint4 w = hv ? __ldg(reinterpret_cast<const uint4*>(qrow + 64 * c + 8 * v)) : z;
                        u[4 * v + 0] = w.x;
                        u[4 * v + 1] = w.y;
                        u[4 * v + 2] = w.z;
                        u[4 * v + 3] = w.w;
                    }
                    tmem_st32(tmem + lane_off + C::T_Q + 32u * c, u);
                }
                tc_wait_st();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(sBar + C::B_QREADY);
            }
            const bool pos = sl2 >= 0.f;
            const float NEG = pos ? -INFINITY : INFINITY;
            const uint32_t peer_slot0 = peer_smem(sb + C::V_P, 1);
            const uint32_t peer_pfull0 = peer_smem(sBar + C::B_PFULL, 1);
            float m_use = -INFINITY, l = 0.f;  // l: this half's partial row sum
            for (int j = 0; j < n_chunks; ++j) {
                const int ps = j & 1;
                bool okt = mbar_wait(sBar + C::B_SFULL + 8 * ps, (j >> 1) & 1, abort_flag);
                tc_fence_after();
                float x[32];
                {
                    uint32_t u0[32];
                    tmem_ld32(tmem + lane_off + 64u * (uint32_t)ps + 32u * (uint32_t)hf, u0);
                    tc_wait_ld();
#pragma unroll
                    for (int e = 0; e < 32; ++e) x[e] = __uint_as_float(u0[e]);
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(sBar + C::B_SFREE + 8 * ps);
                const int nvalid = min(64, hi - (lo + j * 64)) - 32 * hf;  // valid columns of this half
                const bool masked = nvalid < 32;
                if (masked) {
#pragma unroll
                    for (int c = 0; c < 32; ++c) x[c] = (c < nvalid) ? x[c] : NEG;
                }
                float a0 = NEG, a1 = NEG, a2 = NEG, a3 = NEG;
                if (pos) {
#pragma unroll
                    for (int c = 0; c < 32; c += 8) {
                        a0 = fmax3(a0, x[c], x[c + 1]);
                        a1 = fmax3(a1, x[c + 2], x[c + 3]);
                        a2 = fmax3(a2, x[c + 4], x[c + 5]);
                        a3 = fmax3(a3, x[c + 6], x[c + 7]);
                    }
                    a0 = fmax3(a0, a1, fmaxf(a2, a3));
                } else {
#pragma unroll
                    for (int c = 0; c < 32; c += 8) {
                        a0 = fmin3(a0, x[c], x[c + 1]);
                        a1 = fmin3(a1, x[c + 2], x[c + 3]);
                        a2 = fmin3(a2, x[c + 4], x[c + 5]);
                        a3 = fmin3(a3, x[c + 6], x[c + 7]);
                    }
                    a0 = fmin3(a0, a1, fminf(a2, a3));
                }
                xmax[hf * 128 + r] = a0;
                // the value CTA's message slot of this parity is free once it released chunk j-2
                if (tid == 0)
                    okt = mbar_wait<true>(sBar + C::B_PFREE + 8 * ps, ((j >> 1) & 1) ^ 1, abort_flag) && okt;
                if (!bar_and(1, C::NW, okt)) break;
                const float ao = xmax[(hf ^ 1) * 128 + r];
                a0 = pos ? fmaxf(a0, ao) : fminf(a0, ao);
                const float mx = (a0 == NEG) ? -INFINITY : a0 * sl2;
                const float m_new = fmaxf(m_use, mx);
                float alpha = 1.f;
                const bool old_finite = (m_use != -INFINITY);
                if (m_new > m_use + 8.f) {
                    alpha = ex2(m_use - m_new);
                    m_use = m_new;
                }
                const bool need = (j > 0) && old_finite && (alpha != 1.f);
                // the message goes straight into the value CTA's slot ps: every store counts its
                // bytes on that CTA's barrier (17424 bytes per message, 1/l included every time)
                const uint32_t slot = peer_slot0 + (uint32_t)ps * C::PSLOT;
                const uint32_t pbar = peer_pfull0 + 8u * (uint32_t)ps;
                if (hf == 0) st_async_peer_b32(slot + C::MSG_ALPHA + 4u * r, __float_as_uint(alpha), pbar);
                const float mref = (m_use == -INFINITY) ? 0.f : m_use;
                const float2 sc2 = make_float2(sl2, sl2);
                const float2 nm2 = make_float2(-mref, -mref);
                float2 sum0 = make_float2(0.f, 0.f), sum1 = make_float2(0.f, 0.f);
                uint32_t pk[16];
#pragma unroll
                for (int e = 0; e < 16; ++e) {
                    const int col = 2 * e;
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
                // keys 32hf .. 32hf+31: 16-byte chunks 4hf .. 4hf+3 of row r (128B swizzle)
                const uint32_t rowp = slot + (uint32_t)r * 128u;
#pragma unroll
                for (int v = 0; v < 4; ++v) {
                    const int chunk = 4 * hf + v;
                    st_async_peer_v4(rowp + (uint32_t)((chunk ^ (r & 7)) << 4),
                                     make_uint4(pk[4 * v], pk[4 * v + 1], pk[4 * v + 2], pk[4 * v + 3]), pbar);
                }
                l = l * alpha + ((sum0.x + sum0.y) + (sum1.x + sum1.y));
                const bool last = (j == n_chunks - 1);
                float invl = 0.f;  // read by the value CTA with the last message only
                if (last) {
                    // 1/l of the whole row: the two halves exchange their partial sums
                    xsum[hf * 128 + r] = l;
                    bar_and(1, C::NW, true);
                    const float lt = l + xsum[(hf ^ 1) * 128 + r];
                    invl = (lt > 0.f) ? 1.f / lt : 0.f;
                    l = lt;
                }
                if (hf == 0) st_async_peer_b32(slot + C::MSG_INVL + 4u * r, __float_as_uint(invl), pbar);
                const bool any = bar_or(1, C::NW, need);
                if (tid == 0) {
                    mbar_arrive_expect_tx_peer_relaxed(pbar, C::MSG_BYTES);
                    st_async_peer_v4(slot + C::MSG_HDR, make_uint4((any ? 1u : 0u) | (last ? 2u : 0u), (uint32_t)j, 0u, 0u),
                                     pbar);
                }
            }
            if (hv && hf == 0) {
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
            int pc[4], pn[4];
            uint32_t lc = 0;
            uint32_t ln = (n_chunks > 0) ? mla_fetch_pages(p, p.v_page_table, p.v_pt_stride, b, lo, hi, np, pn) : 0u;
            int vi = 0;
            bool ok = true;
            for (int j = 0; ok && j < n_chunks; ++j) {
                const int t0 = lo + j * 64;
#pragma unroll
                for (int i = 0; i < 4; ++i) pc[i] = pn[i];
                lc = ln;
                if (j + 1 < n_chunks) ln = mla_fetch_pages(p, p.v_page_table, p.v_pt_stride, b, t0 + 64, hi, np, pn);
                for (int hf = 0; hf < C::VLOADS; ++hf) {
                    const int st = vi % C::RV;
                    const uint32_t full = sBar + C::B_VFULL + 8 * st;
                    if (!mbar_wait(sBar + C::B_VEMPTY + 8 * st, ((vi / C::RV) & 1) ^ 1, abort_flag)) {
                        ok = false;
                        break;
                    }
                    mbar_arrive_expect_tx(full, C::VSLOT);
                    mla_issue(p, &p.tm_v, sb + C::V_RING + st * C::VSLOT, full, C::VB * hf, C::VB, t0, np, pc, lc);
                    ++vi;
                    if (tail && j == n_chunks - 1) {
                        // zero the value rows of the partially valid box that lie past the sequence
                        if (!mbar_wait(full, ((vi - 1) / C::RV) & 1, abort_flag)) {
                            ok = false;
                            break;
                        }
                        const int pp = (nvalid_last - 1) / R;
                        const int r0 = nvalid_last - pp * R;
                        uint8_t* vq = sgen + C::V_RING + st * C::VSLOT + pp * C::VB * R * 128;
                        for (int blk = 0; blk < C::VB; ++blk)
                            for (int rr = r0; rr < R; ++rr)
                                for (int i = 0; i < 8; ++i)
                                    *reinterpret_cast<uint4*>(vq + (blk * R + rr) * 128 + i * 16) = make_uint4(0, 0, 0, 0);
                        fence_proxy_async_smem();
                        mbar_arrive(sBar + C::B_VTAIL + 8 * hf);
                    }
                }
            }
            for (int kk = max(0, vi - C::RV); kk < vi; ++kk)
                mbar_wait(sBar + C::B_VFULL + 8 * (kk % C::RV), (kk / C::RV) & 1, nullptr, 100000000ull);
        } else if (warp == 1 && lane == 0) {
            constexpr uint32_t IDESC = idesc_bf16_f32(128, 128, true);
            const SmemDesc dP = smem_desc_sw128_split(sb + C::V_P, 16, 1024);
            const SmemDesc dV = smem_desc_sw128_split(sb + C::V_RING, (uint32_t)R * 128u, 1024);
            const uint32_t blk_bytes = (uint32_t)R * 128u;
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
                for (int hf = 0; hf < C::VLOADS; ++hf) {
                    const int st = vi % C::RV;
                    if (!mbar_wait(sBar + C::B_VFULL + 8 * st, (vi / C::RV) & 1, abort_flag)) {
                        ok = false;
                        break;
                    }
                    if (tail && j == n_chunks - 1) {
                        if (!mbar_wait(sBar + C::B_VTAIL + 8 * hf, 0, abort_flag)) {
                            ok = false;
                            break;
                        }
                    }
                    tc_fence_after();
                    const SmemDesc b0{dV.lo + ((st * C::VSLOT) >> 4), dV.hi};
                    for (int qq = 0; qq < C::VB / 2; ++qq) {
                        const uint32_t d = tmem + 128u * (uint32_t)(hf * (C::VB / 2) + qq);
#pragma unroll
                        for (int kk = 0; kk < 4; ++kk) {
                            // keys 16kk .. 16kk+15: page box pp, rows from row0
                            const int pp = (16 * kk) / R, row0 = (16 * kk) % R;
                            const uint32_t boff = (uint32_t)(pp * C::VB + 2 * qq) * blk_bytes + (uint32_t)row0 * 128u;
                            tc_mma_ss(d, desc_at(a0, kk * 32u), desc_at(b0, boff), IDESC, (j > 0 || kk > 0) ? 1u : 0u);
                        }
                    }
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
            // thread = (row r, column half hf): O columns [256 hf, 256 hf + 256)
            const int quad = warp & 3;
            const int hf = (warp - 2) >> 2;
            const int r = quad * 32 + lane;
            const int tid = threadIdx.x - 64;
            const uint32_t lane_off = (uint32_t)(quad * 32) << 16;
            const uint32_t tO = tmem + lane_off + 256u * (uint32_t)hf;
            const int h = hg * 128 + r;
            const bool hv = r < nh;
            const uint32_t peer_pfree0 = peer_smem(sBar + C::B_PFREE, 0);
            float inv_l = 0.f;
            bool ok = true;
            for (int j = 0; j < n_chunks; ++j) {
                const int ps = j & 1;
                bool okt = true;
                if (tid == 0) okt = mbar_wait<true>(sBar + C::B_PFULL + 8 * ps, (j >> 1) & 1, abort_flag);
                if (!bar_and(1, C::NW, okt)) { ok = false; break; }
                const uint8_t* slot = sgen + C::V_P + ps * C::PSLOT;
                const int flags = *reinterpret_cast<const volatile int*>(slot + C::MSG_HDR);
                if (j > 0 && (flags & 1)) {
                    // O must hold every chunk before j when it is rescaled
                    okt = true;
                    if (tid == 0)
                        okt = mbar_wait(sBar + C::B_PVDONE + 8 * ((j - 1) & 1), ((j - 1) >> 1) & 1, abort_flag);
                    const bool ok2 = bar_and(1, C::NW, okt);
                    tc_fence_after();
                    const float a = *reinterpret_cast<const volatile float*>(slot + C::MSG_ALPHA + 4 * r);
                    if (ok2 && __any_sync(0xffffffffu, a != 1.f)) {
#pragma unroll 1
                        for (int c = 0; c < 8; ++c) {
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
                if (!bar_and(1, C::NW, okt)) { ok = false; break; }
                if (tid == 0) mbar_arrive_peer_relaxed(peer_pfree0 + 8u * (uint32_t)ps);
            }
            tc_fence_after();
            const int64_t row = (int64_t)s * p.B * p.Hq + (int64_t)b * p.Hq + h;
#pragma unroll 1
            for (int c = 0; c < 8; ++c) {
                uint32_t u[32];
                if (n_chunks > 0) {
                    tmem_ld32(tO + 32u * c, u);
                    tc_wait_ld();
                } else {
#pragma unroll
                    for (int e = 0; e < 32; ++e) u[e] = 0u;
                }
                if (!hv || !ok) continue;
                const int col = 256 * hf + 32 * c;
                if (p.num_splits == 1) {
                    uint4* dst = reinterpret_cast<uint4*>(p.o + (int64_t)b * p.o_bs + (int64_t)h * p.o_hs + col);
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
                    float4* dst = reinterpret_cast<float4*>(p.o_part + row * 512 + col);
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
