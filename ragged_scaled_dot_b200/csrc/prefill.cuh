// prefill.cuh -- forward attention prefill on tcgen05 tensor cores (sm_100a).
//
// One persistent CTA per SM claims work items one at a time from a list built
// on the device (a claim counter in the caller's workspace).  A work item is
// (sequence b, query tile of 128 rows, up to two query heads of one GQA group):
// the two heads share every K/V tile, so each K/V byte brought on chip feeds
// two 128x128 score tiles ("cuDNN Frontend v1.30.0 Release Notes", "New:
// decode tiles", GQA packing; the grouping here is our own).  Ragged and paged
// items are ordered (sequence longest first, kv head, query tile longest
// first, head pair), dense items (group of query tiles longest first, batch,
// kv head, query tile, head pair), so the CTAs working at the same time share
// few sequence-heads' K/V in L2 and the long items start first.
//
// Warp roles (320 threads):
//   warp 0      claims items, publishes them to the other roles through a
//               small shared-memory ring, and issues the TMA loads: Q tiles of
//               the item, then K(j), V(j) into a ring of NST stages (one thread).
//               Over a paged cache the whole warp runs this loop: each lane
//               reads one page id of a tile and issues its page box, so the
//               id reads and box issues of a tile overlap.
//   warp 1      owns TMEM; one thread issues every tcgen05.mma and commit
//               (descriptor bases are precomputed: this thread shares its SM
//               sub-partition with two busy softmax warps, so every instruction
//               it issues is expensive).
//   warps 2-5   softmax for slot 0 (query head h0), one TMEM lane (row) each:
//               any four consecutive warps cover the four TMEM lane quadrants.
//   warps 6-9   softmax for slot 1 (query head h0 + 1).
// Ten warps put three on two of the SM's four sub-partitions, so a thread may
// hold 168 registers (16384 per sub-partition / 96); the kernel uses 165, enough
// for a 128-column score row without spilling, and little room for more.
// TMEM (512 columns): S0 [0,128) S1 [128,256) O0 [256,256+D) O1 [256+D,256+2D);
// P (bf16) overwrites the first 64 columns of its S tile and feeds the PV MMA
// straight from TMEM.
//
// MMA order per KV tile j (ping-pong between the two slots):
//   PV0(j) QK0(j+1) PV1(j) QK1(j+1)
// so the tensor core computes one slot's MMAs while the other slot's softmax
// runs.  The softmax keeps the running maximum m in the log2 domain with the
// scale folded in ("cuDNN Frontend v1.30.0 Release Notes", stats_use_log2
// section: the prefill kernels keep the softmax in the log2 domain), only
// rescales O when the maximum grows by more than 8 (P stays <= 2^8).  An
// FMA-pipe exponential ("cuDNN Frontend v1.30.0 Release Notes", "SDPA: more
// kernels and numerics": exp2 on the FMA pipe) is available through
// kEmuPer32 but measured slower here, so it is off: with one softmax warp per
// sub-partition the exponential loop is latency-bound, not MUFU-bound.
//
// Masking: bottom-right causal per sequence and ragged tails are applied by
// select, never by multiplication, so values past a sequence's end can not
// poison a row through 0 * NaN ("cuDNN Frontend v1.28.0 release notes",
// "Updates to Graph API / SDPA", max_total_seq_len).  Fully masked KV tiles
// past the causal diagonal are never loaded.
#pragma once

#include "paging.cuh"
#include "ptx.cuh"

namespace b2 {

struct PrefillParams {
    CUtensorMap tm_q;  // 5D (d in block, token, 64-column block, head, batch), 128B swizzle,
                       // box (64, 128, D/64, 1, 1): one request per tile reads whole rows
    CUtensorMap tm_k;
    CUtensorMap tm_v;
    int mode;  // 0 dense, 1 ragged
    int B, Hq, Hkv, G;
    int heads_per_item;   // 2 when G is even, else 1
    int pairs_per_group;  // G / heads_per_item
    int Sq, Skv;          // dense
    const int32_t* cu_q;
    const int32_t* cu_kv;
    const int4* items;  // work list {b, qtile, h0, cost}, built on the device
    int* header;        // [0] item count, [1] claim counter
    __nv_bfloat16* o;
    int64_t o_bs, o_ts, o_hs;  // element strides (batch, token, head)
    float* lse;
    int lse_layout;  // 0 dense [B,Hq,Sq], 1 padded [B,smax,Hq], 2 packed [T,Hq], 3 packed [Hq,T]
    int lse_smax;
    int64_t lse_hs;  // layout 3: row stride (declared total_q)
    int lse_log2;    // 1: LSE in base 2
    float scale_log2;
    int causal;
    // mode 2 (queries of a ragged batch over a paged K/V cache): key t of
    // sequence b is row t % page_size of page page_table[b * pt_stride + t / page_size];
    // the pool maps address 8-row groups: group = page * groups_per_page + row / 8
    const int32_t* kv_lens;
    const int32_t* page_table;  // K pages
    int64_t pt_stride;
    const int32_t* v_page_table;  // V pages (the K table unless the caller gives its own)
    int64_t v_pt_stride;
    int page_size, box_rows;  // box_rows = min(page_size, 128) rows per page box
    int64_t num_pages;
    int groups_per_page;      // page stride / (8 x row stride) of the pool
    int n_groups;             // extent of the pool maps' group dimension (the zero-fill coordinate)
    int max_kv_len;
};

struct PrefillItem {
    int b, qt, h0, nh;
    int q_tok0;   // token coordinate of row 0 (dense: inside the batch)
    int kv_tok0;  // token coordinate of key 0
    int batch;    // batch coordinate (dense) or 0
    int Lq, Lkv;
    int n_kv;     // KV tiles to visit
};

__device__ __forceinline__ int prefill_n_kv(int qt, int Lq, int Lkv, int causal) {
    const int total = (Lkv + 127) >> 7;
    if (!causal) return total;
    const int rows = min(128, Lq - qt * 128);
    const long long kmax = (long long)qt * 128 + rows - 1 + (long long)(Lkv - Lq);
    if (kmax < 0) return 0;
    return (int)min((long long)total, (kmax >> 7) + 1);
}

__device__ __forceinline__ void prefill_get_item(const PrefillParams& p, int idx, PrefillItem& it) {
    const int4 w = p.items[idx];
    it.b = w.x;
    it.qt = w.y;
    it.h0 = w.z;
    if (p.mode == 0) {
        // dense: sequence b is batch b of the 5D maps, every sequence Sq x Skv
        it.q_tok0 = it.qt * 128;
        it.kv_tok0 = 0;
        it.batch = it.b;
        it.Lq = p.Sq;
        it.Lkv = p.Skv;
    } else {
        const int q0 = __ldg(p.cu_q + it.b), q1 = __ldg(p.cu_q + it.b + 1);
        it.Lq = q1 - q0;
        it.q_tok0 = q0 + it.qt * 128;
        it.batch = 0;
        if (p.mode == 2) {
            // validated by the work-list kernel: items exist only for sequences with 0 <= kv_len <= max
            it.Lkv = __ldg(p.kv_lens + it.b);
            it.kv_tok0 = 0;
        } else {
            const int k0 = __ldg(p.cu_kv + it.b), k1 = __ldg(p.cu_kv + it.b + 1);
            it.Lkv = k1 - k0;
            it.kv_tok0 = k0;
        }
    }
    it.nh = p.heads_per_item;
    it.n_kv = prefill_n_kv(it.qt, it.Lq, it.Lkv, p.causal);
}

// Mode 2: does the K/V tile from t0 end inside a page box that runs past Lkv
// (rows past the sequence that can hold stale values, possibly NaN)?
__device__ __forceinline__ bool paged_tile_has_tail(const PrefillParams& p, int t0, int Lkv) {
    return t0 < Lkv && Lkv <= t0 + 128 && (Lkv % p.box_rows) != 0;
}

// Mode 2 scheduler and producer, run by the whole producer warp.  Lane 0 claims
// items, publishes them, loads Q and handles the stage barriers; after a warp
// shuffle, lane i < 128 / box_rows issues page box i of each K and V tile, reading
// its own page id, so a tile's id reads and box issues overlap.  A box is (64
// columns, 8 rows, D/64 blocks, box_rows/8 groups, 1 head) and lands as
// [group][block][8 rows][128 B]; boxes placed back to back keep one uniform
// 8-row-group stride, so the tile is a single MMA operand across pages.  Boxes at
// or past Lkv (or with a bad page id, recorded) read zeros.  One thread issuing
// the boxes one by one, each TMA issue ordered after its id read, could not keep
// the MMAs fed: with it, 4 chunks of 1024 queries ran at 313, 525, 1033 and 1035
// TFLOP/s with pages of 16, 32, 64 and 128 keys, and with the warp at 962, 1089,
// 1090 and 1094.  Kept out of line (the kernel's other roles keep their code).
// kv_it and q_it return the K/V and Q loads issued (every lane holds the same
// counts).
template <int D, int NST, int NRING>
__device__ __noinline__ void prefill_produce_paged(const PrefillParams& p, uint32_t sQ, uint32_t sKV, uint32_t sBar,
                                                   uint32_t b_qfull, uint32_t b_qempty, uint32_t b_ifull0,
                                                   uint32_t b_iempty0, uint32_t b_vtail0, volatile int* item_ring,
                                                   volatile int* abort_flag, uint8_t* kv_gen, int lane, int& kv_it,
                                                   int& q_it) {
    constexpr uint32_t TILE = (D / 64) * 16384u;
    constexpr unsigned FULL = 0xffffffffu;
    const int R = p.box_rows;
    const int nb = 128 / R;  // page boxes per K or V tile
    const uint32_t box_bytes = (uint32_t)R * (D / 64) * 128u;
    const int n_items = p.header[0];
    bool ok = true;
    for (int k = 0; ok; ++k) {
        const int r = k % NRING;
        int idx = -1;
        bool w_ok = true;
        if (lane == 0) {
            w_ok = mbar_wait(b_iempty0 + 8 * r, ((k / NRING) & 1) ^ 1, abort_flag);
            if (w_ok) {
                idx = atomicAdd(p.header + 1, 1);
                if (idx >= n_items) idx = -1;
                item_ring[r] = idx;
                mbar_arrive(b_ifull0 + 8 * r);
            }
        }
        w_ok = __shfl_sync(FULL, w_ok ? 1 : 0, 0) != 0;
        idx = __shfl_sync(FULL, idx, 0);
        if (!w_ok || idx < 0) break;
        PrefillItem it;
        prefill_get_item(p, idx, it);
        if (it.n_kv == 0) continue;
        if (lane == 0) {
            w_ok = mbar_wait(b_qempty, (q_it & 1) ^ 1, abort_flag);
            if (w_ok) {
                mbar_arrive_expect_tx(b_qfull, it.nh * TILE);
                for (int s = 0; s < it.nh; ++s)
                    tma_load_5d(sQ + s * TILE, &p.tm_q, b_qfull, 0, it.q_tok0, 0, it.h0 + s, it.batch);
            }
        }
        if (!__shfl_sync(FULL, w_ok ? 1 : 0, 0)) break;
        ++q_it;
        const int g = it.h0 / p.G;
        for (int j = 0; ok && j < it.n_kv; ++j) {
            for (int t = 0; t < 2; ++t) {
                const int st = kv_it % NST;
                const uint32_t full = sBar + 8u * st, empty = sBar + 8u * (NST + st);
                if (lane == 0) {
                    w_ok = mbar_wait(empty, ((kv_it / NST) & 1) ^ 1, abort_flag);
                    if (w_ok) mbar_arrive_expect_tx(full, TILE);
                }
                // the stage is free and its byte count set before any lane issues a box
                if (!__shfl_sync(FULL, w_ok ? 1 : 0, 0)) { ok = false; break; }
                if (lane < nb) {
                    // boxes at or past Lkv (or with a bad page id, recorded) read zeros
                    const int tk = j * 128 + lane * R;
                    int gg = p.n_groups;
                    if (tk < it.Lkv) {
                        const int32_t* table = t ? p.v_page_table : p.page_table;
                        const int64_t stride = t ? p.v_pt_stride : p.pt_stride;
                        const int page = page_checked(page_lookup(table, stride, it.b, tk, p.page_size), p.num_pages);
                        if (page >= 0) gg = page_group(page, page_slot(tk, p.page_size), p.groups_per_page);
                    }
                    tma_load_5d(sKV + st * TILE + (uint32_t)lane * box_bytes, t ? &p.tm_v : &p.tm_k, full, 0, 0, 0,
                                gg, g);
                }
                if (t == 1 && paged_tile_has_tail(p, j * 128, it.Lkv)) {
                    // value rows past the sequence: zeroed once the tile lands, then the
                    // tile goes to the MMA thread through this stage's tail barrier
                    if (lane == 0) {
                        w_ok = mbar_wait(full, (kv_it / NST) & 1, abort_flag);
                        if (w_ok) {
                            uint8_t* vt = kv_gen + st * TILE;
                            const int r0 = it.Lkv - j * 128;  // rows of the partially valid box past Lkv
                            const int r1 = min(128, (r0 + R - 1) / R * R);
                            for (int rr = r0; rr < r1; ++rr)
                                for (int c = 0; c < (D / 64) * 8; ++c)
                                    *reinterpret_cast<uint4*>(vt + (rr >> 3) * (D / 64) * 1024 + (c >> 3) * 1024 +
                                                              (rr & 7) * 128 + (c & 7) * 16) = make_uint4(0, 0, 0, 0);
                            fence_proxy_async_smem();
                            mbar_arrive(b_vtail0 + 8 * st);
                        }
                    }
                    if (!__shfl_sync(FULL, w_ok ? 1 : 0, 0)) { ok = false; break; }
                }
                ++kv_it;
            }
        }
    }
}

template <int D>
struct PrefillCfg {
    static constexpr int HALVES = D / 64;
    static constexpr uint32_t TILE = HALVES * 16384u;  // one 128-row bf16 tile
    static constexpr int NST = (D == 128) ? 5 : 8;     // K/V ring depth
    static constexpr int NRING = 2;                    // published work items in flight
    static constexpr uint32_t BAR_OFF = (2 + NST) * TILE;
    // + barriers, tmem address, abort flag, item ring (up to 264 bytes at D = 64) + alignment slack
    static constexpr uint32_t SMEM = BAR_OFF + 512 + 1024;
};

// Exponentials per 32-column chunk evaluated on the FMA pipe (the rest on MUFU).
constexpr int kEmuPer32 = 0;

template <int D, bool PAGED>
__global__ void __launch_bounds__(320, 1) prefill_kernel(const __grid_constant__ PrefillParams p) {
    using C = PrefillCfg<D>;
    constexpr int NST = C::NST;
    constexpr int NRING = C::NRING;
    constexpr uint32_t TILE = C::TILE;
    constexpr uint32_t IDESC_QK = idesc_bf16_f32(128, 128, false);
    constexpr uint32_t IDESC_PV = idesc_bf16_f32(128, D, true);

    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t sb = (raw + 1023u) & ~1023u;
    uint8_t* sgen = smem_raw + (sb - raw);
    const uint32_t sQ = sb;
    const uint32_t sKV = sb + 2 * TILE;
    const uint32_t sBar = sb + C::BAR_OFF;
    auto full_bar = [&](int i) { return sBar + 8u * i; };
    auto empty_bar = [&](int i) { return sBar + 8u * (NST + i); };
    const uint32_t b_qfull = sBar + 16u * NST;
    const uint32_t b_qempty = b_qfull + 8;
    const uint32_t b_sfull0 = b_qfull + 16;   // + 8*slot
    const uint32_t b_pready0 = b_qfull + 32;  // + 8*slot
    const uint32_t b_odone0 = b_qfull + 48;   // + 8*slot
    const uint32_t b_oempty0 = b_qfull + 64;  // + 8*slot
    const uint32_t b_drain = b_qfull + 80;
    const uint32_t b_ifull0 = b_qfull + 88;              // + 8*ring slot
    const uint32_t b_iempty0 = b_ifull0 + 8 * NRING;     // + 8*ring slot
    const uint32_t b_vtail0 = b_iempty0 + 8 * NRING;     // + 8*stage: tail rows of a V tile zeroed
    const uint32_t misc = 16u * NST + 88 + 16 * NRING + 8 * NST;  // byte offset past the barriers
    volatile uint32_t* tmem_slot = reinterpret_cast<volatile uint32_t*>(sgen + C::BAR_OFF + misc);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(sgen + C::BAR_OFF + misc + 4);
    volatile int* item_ring = reinterpret_cast<volatile int*>(sgen + C::BAR_OFF + misc + 8);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int i = 0; i < NST; ++i) {
            mbar_init(full_bar(i), 1);
            mbar_init(empty_bar(i), 1);
        }
        mbar_init(b_qfull, 1);
        mbar_init(b_qempty, 1);
        for (int s = 0; s < 2; ++s) {
            mbar_init(b_sfull0 + 8 * s, 1);
            mbar_init(b_pready0 + 8 * s, 128);
            mbar_init(b_odone0 + 8 * s, 1);
            mbar_init(b_oempty0 + 8 * s, 128);
        }
        mbar_init(b_drain, 1);
        for (int i = 0; i < NST; ++i) mbar_init(b_vtail0 + 8 * i, 1);
        for (int r = 0; r < NRING; ++r) {
            mbar_init(b_ifull0 + 8 * r, 1);
            mbar_init(b_iempty0 + 8 * r, 9);  // MMA thread + one lane of each softmax warp
        }
        *abort_flag = 0;
        fence_barrier_init();
        prefetch_tmap(&p.tm_q);
        prefetch_tmap(&p.tm_k);
        prefetch_tmap(&p.tm_v);
    }
    if (warp == 1) {
        tmem_alloc(smem_u32((const void*)tmem_slot), 512);
        tmem_relinquish();
    }
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;


    // Consumers read the next published item (-1 ends the loop).
    auto next_item = [&](int k, bool arrive_lane) -> int {
        const int r = k % NRING;
        if (!mbar_wait(b_ifull0 + 8 * r, (k / NRING) & 1, abort_flag)) return -1;
        const int idx = item_ring[r];
        if (arrive_lane) mbar_arrive(b_iempty0 + 8 * r);
        return idx;
    };

    if (PAGED && warp == 0) {
        // ------------------------------------ scheduler + producer over a paged cache
        int kv_it = 0, q_it = 0;
        prefill_produce_paged<D, NST, NRING>(p, sQ, sKV, sBar, b_qfull, b_qempty, b_ifull0, b_iempty0, b_vtail0,
                                             item_ring, abort_flag, sgen + (sKV - sb), lane, kv_it, q_it);
        // Let every load the warp issued land before the block exits.
        if (lane == 0) {
            const int n_last = min(kv_it, NST);
            for (int kk = kv_it - n_last; kk < kv_it; ++kk)
                mbar_wait(full_bar(kk % NST), (kk / NST) & 1, nullptr, 100000000ull);
            if (q_it > 0) mbar_wait(b_qfull, (q_it - 1) & 1, nullptr, 100000000ull);
        }
    } else if (warp == 0 && lane == 0) {
        // ------------------------------------------- scheduler + producer (dense, ragged)
        const int n_items = p.header[0];
        int kv_it = 0, q_it = 0;
        bool ok = true;
        for (int k = 0; ok; ++k) {
            const int r = k % NRING;
            if (!mbar_wait(b_iempty0 + 8 * r, ((k / NRING) & 1) ^ 1, abort_flag)) break;
            int idx = atomicAdd(p.header + 1, 1);
            if (idx >= n_items) idx = -1;
            item_ring[r] = idx;
            mbar_arrive(b_ifull0 + 8 * r);
            if (idx < 0) break;
            PrefillItem it;
            prefill_get_item(p, idx, it);
            if (it.n_kv == 0) continue;
            if (!mbar_wait(b_qempty, (q_it & 1) ^ 1, abort_flag)) { ok = false; break; }
            mbar_arrive_expect_tx(b_qfull, it.nh * TILE);
            for (int s = 0; s < it.nh; ++s)
                tma_load_5d(sQ + s * TILE, &p.tm_q, b_qfull, 0, it.q_tok0, 0, it.h0 + s, it.batch);
            ++q_it;
            const int g = it.h0 / p.G;
            for (int j = 0; ok && j < it.n_kv; ++j) {
                for (int t = 0; t < 2; ++t) {
                    const int st = kv_it % NST;
                    if (!mbar_wait(empty_bar(st), ((kv_it / NST) & 1) ^ 1, abort_flag)) { ok = false; break; }
                    mbar_arrive_expect_tx(full_bar(st), TILE);
                    tma_load_5d(sKV + st * TILE, t ? &p.tm_v : &p.tm_k, full_bar(st), 0, it.kv_tok0 + j * 128, 0, g,
                                it.batch);
                    ++kv_it;
                }
            }
        }
        // Let every load this thread issued land before the block exits.
        const int n_last = min(kv_it, NST);
        for (int kk = kv_it - n_last; kk < kv_it; ++kk)
            mbar_wait(full_bar(kk % NST), (kk / NST) & 1, nullptr, 100000000ull);
        if (q_it > 0) mbar_wait(b_qfull, (q_it - 1) & 1, nullptr, 100000000ull);
    } else if (warp == 1 && lane == 0) {
        // --------------------------------------------------------- MMA issuer
        int kv_it = 0, q_it = 0;
        int pr_cnt0 = 0, pr_cnt1 = 0, oe_cnt0 = 0, oe_cnt1 = 0;
        bool ok = true;
        const SmemDesc dQ = smem_desc_sw128_split(sQ, 16, 1024);
        // K/V tiles: [64-column block][128 rows] (8-row groups 1 KB apart), or in mode 2
        // [8-row group][block][8 rows] (groups (D/64) KB apart, blocks 1 KB apart)
        constexpr uint32_t NBK = D / 64;
        const SmemDesc dK = smem_desc_sw128_split(sKV, 16, PAGED ? NBK * 1024 : 1024);
        const SmemDesc dV = smem_desc_sw128_split(sKV, PAGED ? 1024 : 16384, PAGED ? NBK * 1024 : 1024);
        uint32_t tail_par = 0;  // mode 2: per-stage parity of the tail barriers
        auto issue_qk = [&](int s, int st) {
            const uint32_t d_tmem = tmem + 128u * s;
            const SmemDesc a0{dQ.lo + ((s * TILE) >> 4), dQ.hi};
            const SmemDesc b0{dK.lo + ((st * TILE) >> 4), dK.hi};
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
                const uint32_t off = (kk >> 2) * 16384u + (kk & 3) * 32u;
                const uint32_t offk = PAGED ? (kk >> 2) * 1024u + (kk & 3) * 32u : off;
                tc_mma_ss(d_tmem, desc_at(a0, off), desc_at(b0, offk), IDESC_QK, kk > 0 ? 1u : 0u);
            }
        };
        auto issue_pv = [&](int s, int st, bool acc) {
            const uint32_t d_tmem = tmem + 256u + (uint32_t)(D * s);
            const uint32_t a_tmem = tmem + 128u * s;
            const SmemDesc b0{dV.lo + ((st * TILE) >> 4), dV.hi};
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
                const uint32_t offv = PAGED ? kk * (2u * NBK * 1024u) : kk * 2048u;
                tc_mma_ts(d_tmem, a_tmem + kk * 8u, desc_at(b0, offv), IDESC_PV, (acc || kk > 0) ? 1u : 0u);
            }
        };
        for (int k = 0; ok; ++k) {
            const int idx = next_item(k, true);
            if (idx < 0) break;
            PrefillItem it;
            prefill_get_item(p, idx, it);
            if (it.n_kv == 0) continue;
            if (!mbar_wait(b_qfull, q_it & 1, abort_flag)) { ok = false; break; }
            ++q_it;
            // prologue: S = Q K(0)^T for both slots
            const int stK = kv_it % NST;
            if (!mbar_wait(full_bar(stK), (kv_it / NST) & 1, abort_flag)) { ok = false; break; }
            ++kv_it;
            tc_fence_after();
            for (int s = 0; s < it.nh; ++s) {
                issue_qk(s, stK);
                tc_commit(b_sfull0 + 8 * s);
            }
            tc_commit(empty_bar(stK));
            if (it.n_kv == 1) tc_commit(b_qempty);
            for (int j = 0; ok && j < it.n_kv; ++j) {
                const int stV = kv_it % NST;
                if (!mbar_wait(full_bar(stV), (kv_it / NST) & 1, abort_flag)) { ok = false; break; }
                if (PAGED && paged_tile_has_tail(p, j * 128, it.Lkv)) {
                    if (!mbar_wait(b_vtail0 + 8 * stV, (tail_par >> stV) & 1u, abort_flag)) { ok = false; break; }
                    tail_par ^= 1u << stV;
                }
                ++kv_it;
                const bool more = (j + 1 < it.n_kv);
                const int stK1 = kv_it % NST;
                const uint32_t parK1 = (kv_it / NST) & 1;
                for (int s = 0; ok && s < it.nh; ++s) {
                    int& pr_cnt = s ? pr_cnt1 : pr_cnt0;
                    int& oe_cnt = s ? oe_cnt1 : oe_cnt0;
                    if (!mbar_wait(b_pready0 + 8 * s, pr_cnt & 1, abort_flag)) { ok = false; break; }
                    ++pr_cnt;
                    if (j == 0) {
                        if (!mbar_wait(b_oempty0 + 8 * s, (oe_cnt & 1) ^ 1, abort_flag)) { ok = false; break; }
                        ++oe_cnt;
                    }
                    tc_fence_after();
                    issue_pv(s, stV, j > 0);
                    tc_commit(b_odone0 + 8 * s);
                    if (more) {
                        if (s == 0) {
                            if (!mbar_wait(full_bar(stK1), parK1, abort_flag)) { ok = false; break; }
                            tc_fence_after();
                        }
                        issue_qk(s, stK1);
                        tc_commit(b_sfull0 + 8 * s);
                    }
                }
                if (!ok) break;
                tc_commit(empty_bar(stV));
                if (more) {
                    ++kv_it;
                    tc_commit(empty_bar(stK1));
                    if (j + 2 == it.n_kv) tc_commit(b_qempty);
                }
            }
        }
        // Wait for every MMA this thread issued before TMEM is released.
        tc_commit(b_drain);
        mbar_wait(b_drain, 0, nullptr, 100000000ull);
    } else if (warp >= 2) {
        // ------------------------------------------------------------ softmax
        const int slot = (warp - 2) >> 2;
        const int quad = warp & 3;
        const int r = quad * 32 + lane;
        const uint32_t lane_off = (uint32_t)(quad * 32) << 16;
        const uint32_t tS = tmem + lane_off + 128u * slot;
        const uint32_t tO = tmem + lane_off + 256u + (uint32_t)(D * slot);
        const uint32_t b_sfull = b_sfull0 + 8 * slot, b_pready = b_pready0 + 8 * slot;
        const uint32_t b_odone = b_odone0 + 8 * slot, b_oempty = b_oempty0 + 8 * slot;
        const float sl2 = p.scale_log2;
        const bool pos = sl2 >= 0.f;  // sign of the scale decides max vs min of raw scores
        const float NEG = pos ? -INFINITY : INFINITY;
        int sf_cnt = 0, od_base = 0;
        bool ok = true;
        for (int k = 0; ok; ++k) {
            int idx = next_item(k, false);
            __syncwarp();
            if (lane == 0 && idx >= -1) mbar_arrive(b_iempty0 + 8 * (k % NRING));
            if (idx < 0) break;
            PrefillItem it;
            prefill_get_item(p, idx, it);
            if (slot >= it.nh) continue;
            const int h = it.h0 + slot;
            const int row = it.qt * 128 + r;
            const bool valid = row < it.Lq;
            const int tok = it.q_tok0 + r;
            __nv_bfloat16* orow = p.o + (int64_t)it.batch * p.o_bs + (int64_t)tok * p.o_ts + (int64_t)h * p.o_hs;
            float m_use = -INFINITY, l = 0.f;
            if (it.n_kv > 0) {
                const int lim = p.causal ? min(it.Lkv, row + it.Lkv - it.Lq + 1) : it.Lkv;
                for (int j = 0; j < it.n_kv; ++j) {
                    if (!mbar_wait(b_sfull, sf_cnt & 1, abort_flag)) { ok = false; break; }
                    ++sf_cnt;
                    tc_fence_after();
                    float x[128];
                    {
                        uint32_t u[128];
                        tmem_ld128(tS, u);
                        tc_wait_ld();
#pragma unroll
                        for (int e = 0; e < 128; ++e) x[e] = __uint_as_float(u[e]);
                    }
                    const int kb = j * 128;
                    const bool masked = (kb + 128 > lim);
                    if (masked) {
#pragma unroll
                        for (int c = 0; c < 128; ++c) x[c] = (kb + c < lim) ? x[c] : NEG;
                    }
                    // row maximum of the scaled scores (min of raw scores when scale < 0)
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
                    const float mref = (m_use == -INFINITY) ? 0.f : m_use;
                    const float2 sc2 = make_float2(sl2, sl2);
                    const float2 nm2 = make_float2(-mref, -mref);
                    float2 sum0 = make_float2(0.f, 0.f), sum1 = make_float2(0.f, 0.f);
                    uint32_t pk64[64];
#pragma unroll
                    for (int c = 0; c < 4; ++c) {
                        uint32_t* pk = pk64 + 16 * c;
#pragma unroll
                        for (int e = 0; e < 16; ++e) {
                            const int col = 32 * c + 2 * e;
                            const float2 t = ffma2(make_float2(x[col], x[col + 1]), sc2, nm2);
                            float2 pv;
                            if (2 * e >= 32 - kEmuPer32) {
                                pv = exp2_poly_pair(t);
                            } else {
                                pv.x = ex2(t.x);
                                pv.y = ex2(t.y);
                            }
                            if (masked) {
                                pv.x = (kb + col < lim) ? pv.x : 0.f;
                                pv.y = (kb + col + 1 < lim) ? pv.y : 0.f;
                            }
                            if (e & 1) sum1 = fadd2(sum1, pv);
                            else sum0 = fadd2(sum0, pv);
                            pk[e] = pack_bf16(pv.x, pv.y);
                        }
                    }
                    tmem_st64(tS, pk64);
                    l = l * alpha + ((sum0.x + sum0.y) + (sum1.x + sum1.y));
                    const bool need_o = (j > 0) && old_finite && (alpha != 1.f);
                    if (__any_sync(0xffffffffu, need_o)) {
                        // PV(j-1) must have landed in O before it is rescaled.
                        if (!mbar_wait(b_odone, (od_base + j - 1) & 1, abort_flag)) { ok = false; }
                        tc_fence_after();
                        const float f = need_o ? alpha : 1.f;
#pragma unroll 1
                        for (int c = 0; c < D / 32; ++c) {
                            uint32_t u[32];
                            tmem_ld32(tO + 32u * c, u);
                            tc_wait_ld();
#pragma unroll
                            for (int e = 0; e < 32; ++e) u[e] = __float_as_uint(__uint_as_float(u[e]) * f);
                            tmem_st32(tO + 32u * c, u);
                        }
                    }
                    tc_wait_st();
                    tc_fence_before();
                    mbar_arrive(b_pready);
                    if (!ok) break;
                }
                if (!ok) break;
                // epilogue: O / l -> bf16
                if (!mbar_wait(b_odone, (od_base + it.n_kv - 1) & 1, abort_flag)) { ok = false; break; }
                od_base += it.n_kv;
                tc_fence_after();
                const float inv_l = (l > 0.f) ? 1.f / l : 0.f;
#pragma unroll 1
                for (int c = 0; c < D / 32; ++c) {
                    uint32_t u[32];
                    tmem_ld32(tO + 32u * c, u);
                    tc_wait_ld();
                    if (valid) {
                        uint4* dst = reinterpret_cast<uint4*>(orow + 32 * c);
#pragma unroll
                        for (int v4 = 0; v4 < 4; ++v4) {
                            uint4 w;
                            w.x = pack_bf16(__uint_as_float(u[8 * v4 + 0]) * inv_l, __uint_as_float(u[8 * v4 + 1]) * inv_l);
                            w.y = pack_bf16(__uint_as_float(u[8 * v4 + 2]) * inv_l, __uint_as_float(u[8 * v4 + 3]) * inv_l);
                            w.z = pack_bf16(__uint_as_float(u[8 * v4 + 4]) * inv_l, __uint_as_float(u[8 * v4 + 5]) * inv_l);
                            w.w = pack_bf16(__uint_as_float(u[8 * v4 + 6]) * inv_l, __uint_as_float(u[8 * v4 + 7]) * inv_l);
                            dst[v4] = w;
                        }
                    }
                }
                tc_fence_before();
                mbar_arrive(b_oempty);
            } else if (valid) {
                uint4* dst = reinterpret_cast<uint4*>(orow);
                for (int v4 = 0; v4 < D / 8; ++v4) dst[v4] = make_uint4(0, 0, 0, 0);
            }
            if (valid && p.lse != nullptr) {
                // m is kept in the log2 domain, so m + log2(l) is the base-2 LSE
                const float lse2 = (l > 0.f) ? (m_use + log2f(l)) : -INFINITY;
                const float lse = p.lse_log2 ? lse2 : lse2 * 0.6931471805599453f;
                int64_t li;
                if (p.lse_layout == 0) li = ((int64_t)it.b * p.Hq + h) * p.Sq + row;
                else if (p.lse_layout == 1) li = ((int64_t)it.b * p.lse_smax + row) * p.Hq + h;
                else if (p.lse_layout == 2) li = (int64_t)tok * p.Hq + h;
                else li = (int64_t)h * p.lse_hs + tok;
                p.lse[li] = lse;
            }
        }
    }

    __syncthreads();
    if (warp == 1) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

}  // namespace b2
