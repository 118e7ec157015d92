// decode.cuh -- paged-KV decode (one query token per sequence) with split-KV.
//
// Pages are gathered with TMA, one box per (page, 64-wide column block): the
// page table gives the physical page of each logical page ("cuDNN Frontend
// v1.31.0 Release Notes", "SDPA: paged KV, split-KV, and engine selection").
// Decode is HBM-bound (8 flop per KV byte at Hq/Hkv = 8), so the small
// contractions run on warp-level MMAs while the memory system streams pages;
// the G query heads of one KV head are the MMA rows, so every K/V byte is read
// once per KV head ("cuDNN Frontend v1.30.0 Release Notes", "New: decode
// tiles", PackGQA).
//
// Split-KV: split s of a sequence with n_pages pages covers pages
// [s*pps, min((s+1)*pps, n_pages)), pps = ceil(n_pages / num_splits).
// With one split the kernel writes O (bf16) and LSE directly; otherwise it
// writes the normalised fp32 partial O_s and its natural-log lse_s, and
// split_merge_kernel combines them.  With splits, blocks take the sequences in
// the order seq_order_kernel leaves in the workspace (longest first), so the
// longest splits start first and the short ones fill the tail.
#pragma once

#include "aux_kernels.cuh"
#include "paging.cuh"
#include "ptx.cuh"

namespace b2 {

struct DecodeParams {
    CUtensorMap tm_k;  // 4D (d, slot, head, page), 128B swizzle, box (64, min(ps,64), 1, 1)
    CUtensorMap tm_v;
    const __nv_bfloat16* q;
    int64_t q_bs, q_hs;  // (batch, head) element strides; with cu_q: (token, head)
    const int32_t* page_table;  // K pages
    int64_t pt_stride;
    const int32_t* v_page_table;  // V pages (the K table unless the caller gives its own)
    int64_t v_pt_stride;
    const int32_t* kv_lens;
    const int32_t* order;  // launch order (sequences longest first) or null: block z runs sequence order[z]
    // Ragged queries over the cache (null: one query per sequence).  Sequence b
    // owns query tokens [cu_q[b], cu_q[b+1]); the GQA decode kernel takes the
    // sequences with 1..qmax of them (the prefill kernel takes the others), the
    // last Lq of the cached positions, bottom-right causal when `causal`.
    const int32_t* cu_q;
    int64_t total_q;  // declared token capacity of q / o (with cu_q)
    int qmax;         // query rows per sequence in the partial layout (1 without cu_q)
    int causal;
    int B, Hq, Hkv, G;
    int page_size, box_rows;  // rows per TMA box: min(page_size, chunk keys)
    int64_t num_pages;
    int max_kv_len;
    int num_splits;
    float scale_log2;
    // outputs (num_splits == 1)
    __nv_bfloat16* o;
    int64_t o_bs, o_hs;  // (batch, head) element strides; with cu_q: (token, head)
    float* lse;          // layout per lse_layout, or null
    int lse_layout;      // 0 [B, Hq]; with cu_q, the THD layouts: 1 padded [B, smax, Hq], 2 [T, Hq], 3 [Hq, T]
    int lse_smax;        // layout 1: max_seqlen_q
    int64_t lse_hs;      // layout 3: row stride (declared total_q)
    int lse_log2;        // 1: LSE in base 2
    // partials (num_splits > 1): [S][B*qmax*Hq][Dv], [S][B*qmax*Hq], row (b*qmax + qi)*Hq + h
    float* o_part;
    float* lse_part;
};

// Index of the LSE of (sequence b, query qi = token tok, head h) in the layouts
// above.
__device__ __forceinline__ int64_t decode_lse_index(int layout, int b, int qi, int64_t tok, int h, int Hq, int smax,
                                                    int64_t hs) {
    if (layout == 0) return (int64_t)b * Hq + h;
    if (layout == 1) return ((int64_t)b * smax + qi) * Hq + h;
    if (layout == 2) return tok * Hq + h;
    return (int64_t)h * hs + tok;
}

// Key range [lo, hi) of split s of sequence b (page-granular partition).
__device__ __forceinline__ void decode_split_range(const DecodeParams& p, int b, int s, int& L,
                                                   int& lo, int& hi) {
    L = __ldg(p.kv_lens + b);
    if (L < 0 || L > p.max_kv_len) {
        record_status(ATTN_ERR_DEVICE_INPUT);
        L = max(0, min(L, p.max_kv_len));
    }
    const int n_pages = (L + p.page_size - 1) / p.page_size;
    const int pps = (n_pages + p.num_splits - 1) / p.num_splits;
    lo = min(s * pps * p.page_size, L);
    hi = min((s + 1) * pps * p.page_size, L);
}

// Bytes one 64-key chunk starting at logical key t0 brings in (for expect_tx):
// whole boxes of box_rows rows, 128 bytes per row and column block.
__device__ __forceinline__ uint32_t decode_chunk_bytes(const DecodeParams& p, int t0, int hi,
                                                       int ncol_blocks, int tensors) {
    const int nkeys = min(64, hi - t0);
    const int nboxes = (nkeys + p.box_rows - 1) / p.box_rows;
    return (uint32_t)nboxes * (uint32_t)p.box_rows * 128u * (uint32_t)ncol_blocks * (uint32_t)tensors;
}

// Issues the K and V TMA loads of the chunk from t0 for kv head g of sequence b:
// rows [r, r + box_rows) come from one page (NB = 64 / box_rows boxes).  All
// page ids of the chunk are read before any box is issued, so their latencies
// overlap (each TMA issue is ordered after the reads before it; one thread
// reading them box by box could not keep a small batch's few blocks streaming),
// and with one page table for K and V the V boxes reuse the K boxes' ids.
template <int NB>
__device__ __forceinline__ void decode_issue_kv(const DecodeParams& p, uint32_t dst_k, uint32_t dst_v, uint32_t bar,
                                                int b, int g, int t0, int hi, int ncol_blocks, uint32_t block_bytes,
                                                const volatile int* ids_k, const volatile int* ids_v, int p0, int nids) {
    const int R = p.box_rows;
    const bool shared_table = p.v_page_table == p.page_table && p.v_pt_stride == p.pt_stride;
    int idk[NB], idv[NB];
#pragma unroll
    for (int i = 0; i < NB; ++i) {
        const int t = t0 + i * R;
        const int w = t / p.page_size - p0;  // position in the window of shared-memory ids
        idk[i] = (t >= hi) ? -1 : (w < nids ? ids_k[w] : page_lookup(p.page_table, p.pt_stride, b, t, p.page_size));
    }
#pragma unroll
    for (int i = 0; i < NB; ++i) {
        const int t = t0 + i * R;
        const int w = t / p.page_size - p0;
        idv[i] = shared_table ? idk[i]
                              : ((t >= hi) ? -1
                                           : (w < nids ? ids_v[w]
                                                       : page_lookup(p.v_page_table, p.v_pt_stride, b, t,
                                                                     p.page_size)));
    }
#pragma unroll
    for (int i = 0; i < NB; ++i) {
        const int t = t0 + i * R;
        if (t < hi) {
            // out of range: page -1, and TMA fills the box with zeros
            const int pk = page_checked(idk[i], p.num_pages);
            const int pv = shared_table ? pk : page_checked(idv[i], p.num_pages);
            const int slot = page_slot(t, p.page_size);
            for (int cb = 0; cb < ncol_blocks; ++cb) {
                tma_load_4d(dst_k + cb * block_bytes + (uint32_t)(i * R) * 128u, &p.tm_k, bar, cb * 64, slot, g, pk);
                tma_load_4d(dst_v + cb * block_bytes + (uint32_t)(i * R) * 128u, &p.tm_v, bar, cb * 64, slot, g, pv);
            }
        }
    }
}

// ===========================================================================
// GQA decode, Dqk = Dv = D in {64, 128}, grid (num_splits, Hkv, B), 160
// threads: warps 0-3 compute, warp 4 loads.  The MMA rows are the query rows of
// one KV head: row r = qi * G + gh is query token qi of the sequence (one
// token for decode; up to qmax with cu_q: multi-token decode, speculative
// tokens) and query head g * G + gh, 16 * RT rows in RT m16 tiles
// ("cuDNN Frontend v1.30.0 Release Notes", "New: decode tiles": G query heads
// x small query counts as the tile rows; "cuDNN Frontend v1.31.0 Release
// Notes", "SDPA: paged KV, split-KV, and engine selection": paged THD
// split-KV).  Warp w computes m-tile w % RT over keys
// [(w / RT) * 16 RT, (w / RT + 1) * 16 RT) of every 64-key chunk and keeps its
// own online-softmax state; the states of the warps of one m-tile are merged
// at the end.  RT = 1 without cu_q is plain decode.
// ===========================================================================
template <int D>
struct DecodeCfg {
    static constexpr int NCB = D / 64;                  // 64-wide column blocks
    static constexpr uint32_t BLK = 64 * 128;           // one column block of a chunk
    static constexpr uint32_t CHUNK = NCB * BLK;        // K (or V) bytes of a chunk
    static constexpr int NST = 3;
    static constexpr uint32_t STAGE = 2 * CHUNK;        // K then V
    static constexpr uint32_t BAR_OFF = NST * STAGE;
    // the block's page ids (K table, then V table when it has its own), read once at the
    // start by every thread: the producer thread then finds them in shared memory
    static constexpr int IDW = 1024;                  // page ids per table in the window
    static constexpr uint32_t IDS_OFF = BAR_OFF + 128;
    static constexpr uint32_t SMEM = IDS_OFF + 2 * IDW * 4 + 1024;
};

template <int D, int RT>
__global__ void __launch_bounds__(160) decode_gqa_kernel(const __grid_constant__ DecodeParams p) {
    using C = DecodeCfg<D>;
    constexpr int NST = C::NST;
    constexpr int KW = 16 * RT;  // keys of every chunk one compute warp owns
    static_assert(RT == 1 || RT == 2 || RT == 4, "m-tiles");
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t sb = (raw + 1023u) & ~1023u;
    uint8_t* sgen = smem_raw + (sb - raw);
    const uint32_t sBar = sb + C::BAR_OFF;
    auto full_bar = [&](int i) { return sBar + 8u * i; };
    auto empty_bar = [&](int i) { return sBar + 8u * (NST + i); };
    volatile int* abort_flag = reinterpret_cast<volatile int*>(sgen + C::BAR_OFF + 16u * NST);

    const int s = blockIdx.x, g = blockIdx.y;
    const int b = p.order ? __ldg(p.order + blockIdx.z) : (int)blockIdx.z;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    // this block's query rows: token b of q (decode), or the Lq <= qmax tokens of sequence b
    int Lq = 1, tok0 = b;
    if (p.cu_q != nullptr) {
        const int q0 = __ldg(p.cu_q + b), q1 = __ldg(p.cu_q + b + 1);
        if (q0 < 0 || q1 < q0 || (int64_t)q1 > p.total_q) {
            if (threadIdx.x == 0) record_status(ATTN_ERR_DEVICE_INPUT);
            return;  // the whole block leaves before any barrier exists
        }
        Lq = q1 - q0;
        tok0 = q0;
        if (Lq < 1 || Lq > p.qmax) return;  // no queries, or a sequence of the prefill kernel
    }
    int L, lo, hi;
    decode_split_range(p, b, s, L, lo, hi);
    const int n_chunks = (hi > lo) ? (hi - lo + 63) / 64 : 0;

    if (threadIdx.x == 0) {
        for (int i = 0; i < NST; ++i) {
            mbar_init(full_bar(i), 1);
            mbar_init(empty_bar(i), 4);
        }
        *abort_flag = 0;
        fence_barrier_init();
    }
    // the page ids of keys [lo, hi) (up to IDW per table), read once by every thread
    volatile int* ids_k = reinterpret_cast<volatile int*>(sgen + C::IDS_OFF);
    volatile int* ids_v = ids_k + C::IDW;
    const int p0 = lo / p.page_size;
    const int nids = (hi > lo) ? min(C::IDW, (hi - 1) / p.page_size - p0 + 1) : 0;
    {
        const bool own_v = !(p.v_page_table == p.page_table && p.v_pt_stride == p.pt_stride);
        const int32_t* rk = p.page_table + (int64_t)b * p.pt_stride + p0;
        const int32_t* rv = p.v_page_table + (int64_t)b * p.v_pt_stride + p0;
        for (int i = threadIdx.x; i < nids; i += blockDim.x) {
            ids_k[i] = __ldg(rk + i);
            if (own_v) ids_v[i] = __ldg(rv + i);
        }
    }
    __syncthreads();

    if (warp == 4) {
        if (lane == 0) {
            prefetch_tmap(&p.tm_k);
            prefetch_tmap(&p.tm_v);
            for (int c = 0; c < n_chunks; ++c) {
                const int st = c % NST;
                if (!mbar_wait(empty_bar(st), ((c / NST) & 1) ^ 1, abort_flag)) break;
                const int t0 = lo + c * 64;
                mbar_arrive_expect_tx(full_bar(st), decode_chunk_bytes(p, t0, hi, C::NCB, 2));
                const uint32_t dst = sb + st * C::STAGE;
                switch (64 / p.box_rows) {
                    case 1:
                        decode_issue_kv<1>(p, dst, dst + C::CHUNK, full_bar(st), b, g, t0, hi, C::NCB, C::BLK, ids_k,
                                           ids_v, p0, nids);
                        break;
                    case 2:
                        decode_issue_kv<2>(p, dst, dst + C::CHUNK, full_bar(st), b, g, t0, hi, C::NCB, C::BLK, ids_k,
                                           ids_v, p0, nids);
                        break;
                    case 4:
                        decode_issue_kv<4>(p, dst, dst + C::CHUNK, full_bar(st), b, g, t0, hi, C::NCB, C::BLK, ids_k,
                                           ids_v, p0, nids);
                        break;
                    default:
                        decode_issue_kv<8>(p, dst, dst + C::CHUNK, full_bar(st), b, g, t0, hi, C::NCB, C::BLK, ids_k,
                                           ids_v, p0, nids);
                        break;
                }
            }
            // drain: every issued load lands before the block leaves
            for (int c = max(0, n_chunks - NST); c < n_chunks; ++c)
                mbar_wait(full_bar(c % NST), (c / NST) & 1, nullptr, 100000000ull);
        }
        __syncthreads();  // matches the compute warps' final barrier
        return;
    }

    // ---------------------------------------------------------------- compute
    const float sl2 = p.scale_log2;
    const int G = p.G;
    const int n_rows = G * Lq;
    const int mt = warp % RT;            // this warp's m-tile (rows 16 mt .. 16 mt + 15)
    const int kbase = (warp / RT) * KW;  // its keys inside every chunk
    const bool active = mt * 16 < n_rows;
    const int qrow = lane >> 2;          // rows qrow and qrow + 8 of the m-tile
    // Q as A fragments (zero past the last row)
    uint32_t qa[D / 16][4];
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk) {
        const int col = kk * 16 + 2 * (lane & 3);
#pragma unroll
        for (int part = 0; part < 4; ++part) {
            const int row = mt * 16 + qrow + ((part & 1) ? 8 : 0);
            const int cc = col + ((part & 2) ? 8 : 0);
            uint32_t v = 0u;
            if (row < n_rows) {
                const int qi = row / G, gh = row - qi * G;
                v = *reinterpret_cast<const uint32_t*>(p.q + (int64_t)(tok0 + qi) * p.q_bs +
                                                       (int64_t)(g * G + gh) * p.q_hs + cc);
            }
            qa[kk][part] = v;
        }
    }
    // keys [lo, rlim) each of this thread's two rows may see (bottom-right causal:
    // query qi of Lq sees keys j <= L - Lq + qi); rows past the last see none
    int rlim[2];
#pragma unroll
    for (int hh = 0; hh < 2; ++hh) {
        const int row = mt * 16 + qrow + 8 * hh;
        if (row < n_rows) {
            const int qi = row / G;
            rlim[hh] = p.causal ? min(hi, L - Lq + qi + 1) : hi;
        } else {
            rlim[hh] = lo;
        }
    }
    float m[2] = {-INFINITY, -INFINITY};
    float l[2] = {0.f, 0.f};
    float oacc[D / 8][4];
#pragma unroll
    for (int i = 0; i < D / 8; ++i) oacc[i][0] = oacc[i][1] = oacc[i][2] = oacc[i][3] = 0.f;

    for (int c = 0; c < n_chunks; ++c) {
        const int st = c % NST;
        if (!mbar_wait(full_bar(st), (c / NST) & 1, abort_flag)) break;
        const uint32_t sK = sb + st * C::STAGE;
        const uint32_t sV = sK + C::CHUNK;
        const int t0 = lo + c * 64;
        const int nvalid = min(64, hi - t0);
        bool zeroed = false;
        if (active) {
            if (kbase + KW > nvalid) {
                zeroed = true;
                // V rows past the split (or never loaded) must be finite: zero them.
                uint8_t* vg = sgen + (sV - sb);
                for (int i = lane; i < KW * C::NCB * 8; i += 32) {
                    const int rr = kbase + i / (C::NCB * 8);
                    const int rem = i % (C::NCB * 8);
                    const int cb = rem / 8, ch = rem % 8;
                    if (rr >= nvalid)
                        *reinterpret_cast<uint4*>(vg + cb * C::BLK + rr * 128 + ch * 16) = make_uint4(0, 0, 0, 0);
                }
                __syncwarp();
            }
            // S = Q K^T over this warp's keys (n-tiles of 8 keys)
            // with RT <= 2, two accumulators per n-tile (even and odd k-steps), so each chain
            // of dependent MMAs is half as long (RT = 4 has enough independent chains and
            // no registers to spare)
            constexpr bool kTwoChains = RT <= 2;
            float sacc[2 * RT][4], sacc2[2 * RT][4];
#pragma unroll
            for (int nt = 0; nt < 2 * RT; ++nt)
#pragma unroll
                for (int e = 0; e < 4; ++e) sacc[nt][e] = sacc2[nt][e] = 0.f;
            {
                const int mat = lane >> 3, rr = lane & 7;
#pragma unroll
                for (int kg = 0; kg < RT; ++kg) {
                    const int key = kbase + 16 * kg + ((mat >> 1) << 3) + rr;
#pragma unroll
                    for (int kk = 0; kk < D / 16; ++kk) {
                        const int cb = kk >> 2;
                        const int dcol = (kk & 3) * 16 + ((mat & 1) << 3);
                        uint32_t b0, b1, b2, b3;
                        ldsm_x4(sK + cb * C::BLK + sw128_offset(key, dcol), b0, b1, b2, b3);
                        float (&a0)[4] = (kTwoChains && (kk & 1)) ? sacc2[2 * kg] : sacc[2 * kg];
                        float (&a1)[4] = (kTwoChains && (kk & 1)) ? sacc2[2 * kg + 1] : sacc[2 * kg + 1];
                        mma_bf16_16816(a0, qa[kk], b0, b1);
                        mma_bf16_16816(a1, qa[kk], b2, b3);
                    }
                }
                if constexpr (kTwoChains) {
#pragma unroll
                    for (int nt = 0; nt < 2 * RT; ++nt)
#pragma unroll
                        for (int e = 0; e < 4; ++e) sacc[nt][e] += sacc2[nt][e];
                }
            }
            // online softmax (log2 domain, scale folded in); keys outside a row's range masked
            float mx[2] = {-INFINITY, -INFINITY};
#pragma unroll
            for (int nt = 0; nt < 2 * RT; ++nt)
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int key = t0 + kbase + nt * 8 + 2 * (lane & 3) + (e & 1);
                    const float x = (key < rlim[e >> 1]) ? sacc[nt][e] * sl2 : -INFINITY;
                    sacc[nt][e] = x;
                    mx[e >> 1] = fmaxf(mx[e >> 1], x);
                }
            float alpha[2], mref[2];
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
                mx[hh] = fmaxf(mx[hh], __shfl_xor_sync(0xffffffffu, mx[hh], 1));
                mx[hh] = fmaxf(mx[hh], __shfl_xor_sync(0xffffffffu, mx[hh], 2));
                // the reference maximum moves only when a score exceeds it by more than 8
                // (P stays <= 2^8), so most chunks leave O and l as they are
                const float mn = fmaxf(m[hh], mx[hh]);
                alpha[hh] = 1.f;
                if (mn > m[hh] + 8.f) {
                    alpha[hh] = (m[hh] == -INFINITY) ? 0.f : ex2(m[hh] - mn);
                    m[hh] = mn;
                }
                mref[hh] = (m[hh] == -INFINITY) ? 0.f : m[hh];
            }
            float psum[2] = {0.f, 0.f};
#pragma unroll
            for (int nt = 0; nt < 2 * RT; ++nt)
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const float pv = ex2(sacc[nt][e] - mref[e >> 1]);
                    sacc[nt][e] = pv;
                    psum[e >> 1] += pv;
                }
            l[0] = l[0] * alpha[0] + psum[0];
            l[1] = l[1] * alpha[1] + psum[1];
            if (alpha[0] != 1.f || alpha[1] != 1.f) {
#pragma unroll
                for (int i = 0; i < D / 8; ++i) {
                    oacc[i][0] *= alpha[0];
                    oacc[i][1] *= alpha[0];
                    oacc[i][2] *= alpha[1];
                    oacc[i][3] *= alpha[1];
                }
            }
            // O += P V over this warp's keys, 16 keys per k-step
            const int mat = lane >> 3, rr = lane & 7;
#pragma unroll
            for (int kg = 0; kg < RT; ++kg) {
                uint32_t pa[4];
                pa[0] = pack_bf16(sacc[2 * kg][0], sacc[2 * kg][1]);
                pa[1] = pack_bf16(sacc[2 * kg][2], sacc[2 * kg][3]);
                pa[2] = pack_bf16(sacc[2 * kg + 1][0], sacc[2 * kg + 1][1]);
                pa[3] = pack_bf16(sacc[2 * kg + 1][2], sacc[2 * kg + 1][3]);
                const int key = kbase + 16 * kg + ((mat & 1) << 3) + rr;
#pragma unroll
                for (int nd = 0; nd < D / 16; ++nd) {
                    const int cb = nd >> 2;
                    const int dcol = (nd & 3) * 16 + ((mat >> 1) << 3);
                    uint32_t v0, v1, v2, v3;
                    ldsm_x4_t(sV + cb * C::BLK + sw128_offset(key, dcol), v0, v1, v2, v3);
                    mma_bf16_16816(oacc[2 * nd], pa, v0, v1);
                    mma_bf16_16816(oacc[2 * nd + 1], pa, v2, v3);
                }
            }
        }
        // generic writes to the stage (the zeroed V rows) are ordered before the next TMA
        // writes into it; reads need only the barrier
        if (zeroed) fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(empty_bar(st));
    }

    // ------------------------------------------- combine the warps' states
    // quad-reduce the row sums
#pragma unroll
    for (int hh = 0; hh < 2; ++hh) {
        l[hh] += __shfl_xor_sync(0xffffffffu, l[hh], 1);
        l[hh] += __shfl_xor_sync(0xffffffffu, l[hh], 2);
    }
    // wait for the last chunk of every warp before reusing the ring as scratch
    asm volatile("bar.sync 1, 128;" ::: "memory");
    float* sm_m = reinterpret_cast<float*>(sgen);              // [4 warps][16 rows of the warp's m-tile]
    float* sm_l = sm_m + 64;                                    // [4][16]
    float* sm_o = sm_m + 128;                                   // [4][16][D]
    if ((lane & 3) == 0) {
        sm_m[warp * 16 + qrow] = m[0];
        sm_m[warp * 16 + qrow + 8] = m[1];
        sm_l[warp * 16 + qrow] = l[0];
        sm_l[warp * 16 + qrow + 8] = l[1];
    }
#pragma unroll
    for (int i = 0; i < D / 8; ++i) {
        const int col = i * 8 + 2 * (lane & 3);
        float* o0 = sm_o + (warp * 16 + qrow) * D + col;
        float* o1 = sm_o + (warp * 16 + qrow + 8) * D + col;
        o0[0] = oacc[i][0];
        o0[1] = oacc[i][1];
        o1[0] = oacc[i][2];
        o1[1] = oacc[i][3];
    }
    asm volatile("bar.sync 1, 128;" ::: "memory");
    const int tid = threadIdx.x;  // 0..127
    for (int idx = tid; idx < n_rows * D; idx += 128) {
        const int row = idx / D, col = idx % D;
        const int rmt = row >> 4, rr = row & 15;  // m-tile, row inside it: warps rmt, rmt + RT, ...
        float M = -INFINITY;
#pragma unroll
        for (int w = rmt; w < 4; w += RT) M = fmaxf(M, sm_m[w * 16 + rr]);
        float Lsum = 0.f, acc = 0.f;
        if (M != -INFINITY) {
#pragma unroll
            for (int w = rmt; w < 4; w += RT) {
                const float mw = sm_m[w * 16 + rr];
                const float f = (mw == -INFINITY) ? 0.f : ex2(mw - M);
                Lsum += f * sm_l[w * 16 + rr];
                acc += f * sm_o[(w * 16 + rr) * D + col];
            }
        }
        const float outv = (Lsum > 0.f) ? acc / Lsum : 0.f;
        const float lse2 = (Lsum > 0.f) ? (M + log2f(Lsum)) : -INFINITY;  // base 2
        const int qi = row / G, gh = row - qi * G;
        const int h = g * G + gh;
        const int64_t tok = (int64_t)tok0 + qi;
        if (p.num_splits == 1) {
            p.o[tok * p.o_bs + (int64_t)h * p.o_hs + col] = __float2bfloat16_rn(outv);
            if (col == 0 && p.lse != nullptr)
                p.lse[decode_lse_index(p.lse_layout, b, qi, tok, h, p.Hq, p.lse_smax, p.lse_hs)] =
                    p.lse_log2 ? lse2 : lse2 * 0.6931471805599453f;
        } else {
            // partials: natural-log lse_s, row (b * qmax + qi) * Hq + h of split s
            const int64_t rr_glob = ((int64_t)s * p.B * p.qmax + (int64_t)b * p.qmax + qi) * p.Hq + h;
            p.o_part[rr_glob * D + col] = outv;
            if (col == 0) p.lse_part[rr_glob] = lse2 * 0.6931471805599453f;
        }
    }
    __syncthreads();
}

// Merge of the split partials of the ragged-query decode rows: row
// r = (b * qmax + qi) * Hq + h of every split is merged as split_merge_kernel
// does and written to query token cu_q[b] + qi, head h of o (token / head
// strides) and to the LSE in the call's layout (base 2 on request).  Rows of
// sequences the decode kernel skipped, and rows qi >= Lq_b, are left alone.
// One warp per row.
template <int DV>
__global__ void __launch_bounds__(256) split_merge_thd_kernel(const float* __restrict__ o_part,
                                                              const float* __restrict__ lse_part, int S,
                                                              const int32_t* __restrict__ cu_q, int B, int qmax,
                                                              int Hq, int64_t total_q, __nv_bfloat16* __restrict__ o,
                                                              int64_t o_ts, int64_t o_hs, float* __restrict__ lse,
                                                              int lse_layout, int lse_smax, int64_t lse_hs,
                                                              int lse_log2) {
    constexpr float LOG2E = 1.4426950408889634f;
    const int64_t R = (int64_t)B * qmax * Hq;
    const int64_t r = blockIdx.x * 8 + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (r >= R) return;
    const int b = (int)(r / ((int64_t)qmax * Hq));
    const int rem = (int)(r - (int64_t)b * qmax * Hq);
    const int qi = rem / Hq, h = rem - qi * Hq;
    const int q0 = __ldg(cu_q + b), q1 = __ldg(cu_q + b + 1);
    const int Lq = q1 - q0;
    if (q0 < 0 || q1 < q0 || (int64_t)q1 > total_q || Lq < 1 || Lq > qmax || qi >= Lq) return;
    float acc[MergeVec<DV>::NV][MergeVec<DV>::VEC];
    const float L = merge_row<DV>(o_part, lse_part, S, R, r, lane, acc);
    const int64_t tok = (int64_t)q0 + qi;
    store_row_bf16<DV>(o + tok * o_ts + (int64_t)h * o_hs, lane, acc);
    if (lse != nullptr && lane == 0)
        lse[decode_lse_index(lse_layout, b, qi, tok, h, Hq, lse_smax, lse_hs)] = lse_log2 ? L * LOG2E : L;
}

}  // namespace b2
