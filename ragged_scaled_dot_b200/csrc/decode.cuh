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
// split_merge_kernel combines them.
#pragma once

#include "ptx.cuh"

namespace b2 {

struct DecodeParams {
    CUtensorMap tm_k;  // 4D (d, slot, head, page), 128B swizzle, box (64, min(ps,64), 1, 1)
    CUtensorMap tm_v;
    CUtensorMap tm_q;  // MLA only: 3D (d, head, batch), box (64, 64, 1)
    const __nv_bfloat16* q;
    int64_t q_bs, q_hs;
    const int32_t* page_table;
    int64_t pt_stride;
    const int32_t* kv_lens;
    int B, Hq, Hkv, G;
    int page_size, box_rows;  // rows per TMA box: min(page_size, chunk keys)
    int64_t num_pages;
    int max_kv_len;
    int num_splits;
    float scale_log2;
    // outputs (num_splits == 1)
    __nv_bfloat16* o;
    int64_t o_bs, o_hs;
    float* lse;  // [B, Hq] or null
    // partials (num_splits > 1): [S][B*Hq][Dv], [S][B*Hq]
    float* o_part;
    float* lse_part;
};

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

// Issues the TMA loads of that chunk for kv head g of sequence b: rows
// [r, r + box_rows) of the chunk come from one page (page-table lookup).
__device__ __forceinline__ void decode_issue_chunk(const DecodeParams& p, const CUtensorMap* map,
                                                   uint32_t dst, uint32_t bar, int b, int g, int t0,
                                                   int hi, int ncol_blocks, uint32_t block_bytes) {
    const int nkeys = min(64, hi - t0);
    for (int r = 0; r < nkeys; r += p.box_rows) {
        const int t = t0 + r;
        int page = __ldg(p.page_table + (int64_t)b * p.pt_stride + t / p.page_size);
        if (page < 0 || (int64_t)page >= p.num_pages) {
            record_status(ATTN_ERR_DEVICE_INPUT);
            page = -1;  // out of range: TMA fills the box with zeros
        }
        const int slot = t % p.page_size;
        for (int cb = 0; cb < ncol_blocks; ++cb)
            tma_load_4d(dst + cb * block_bytes + (uint32_t)r * 128u, map, bar, cb * 64, slot, g, page);
    }
}

// ===========================================================================
// GQA decode, Dqk = Dv = D in {64, 128}, G <= 16 query heads per KV head.
// grid (num_splits, Hkv, B), 160 threads: warps 0-3 compute, warp 4 loads.
// Warp w owns keys [16w, 16w + 16) of every 64-key chunk and keeps its own
// online-softmax state; the four states are merged at the end.
// ===========================================================================
template <int D>
struct DecodeCfg {
    static constexpr int NCB = D / 64;                  // 64-wide column blocks
    static constexpr uint32_t BLK = 64 * 128;           // one column block of a chunk
    static constexpr uint32_t CHUNK = NCB * BLK;        // K (or V) bytes of a chunk
    static constexpr int NST = 3;
    static constexpr uint32_t STAGE = 2 * CHUNK;        // K then V
    static constexpr uint32_t BAR_OFF = NST * STAGE;
    static constexpr uint32_t SMEM = BAR_OFF + 128 + 1024;
};

template <int D>
__global__ void __launch_bounds__(160) decode_gqa_kernel(const __grid_constant__ DecodeParams p) {
    using C = DecodeCfg<D>;
    constexpr int NST = C::NST;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t sb = (raw + 1023u) & ~1023u;
    uint8_t* sgen = smem_raw + (sb - raw);
    const uint32_t sBar = sb + C::BAR_OFF;
    auto full_bar = [&](int i) { return sBar + 8u * i; };
    auto empty_bar = [&](int i) { return sBar + 8u * (NST + i); };
    volatile int* abort_flag = reinterpret_cast<volatile int*>(sgen + C::BAR_OFF + 16u * NST);

    const int s = blockIdx.x, g = blockIdx.y, b = blockIdx.z;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
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
                decode_issue_chunk(p, &p.tm_k, dst, full_bar(st), b, g, t0, hi, C::NCB, C::BLK);
                decode_issue_chunk(p, &p.tm_v, dst + C::CHUNK, full_bar(st), b, g, t0, hi, C::NCB, C::BLK);
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
    const int qrow = lane >> 2;  // rows qrow and qrow + 8 of the MMA tile
    // Q as A fragments (rows = query heads of this KV head, zero past G)
    uint32_t qa[D / 16][4];
    {
        const __nv_bfloat16* qb = p.q + (int64_t)b * p.q_bs + (int64_t)(g * G) * p.q_hs;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
            const int col = kk * 16 + 2 * (lane & 3);
#pragma unroll
            for (int part = 0; part < 4; ++part) {
                const int row = qrow + ((part & 1) ? 8 : 0);
                const int cc = col + ((part & 2) ? 8 : 0);
                qa[kk][part] = (row < G) ? *reinterpret_cast<const uint32_t*>(qb + (int64_t)row * p.q_hs + cc) : 0u;
            }
        }
    }
    float m[2] = {-INFINITY, -INFINITY};
    float l[2] = {0.f, 0.f};
    float oacc[D / 8][4];
#pragma unroll
    for (int i = 0; i < D / 8; ++i) oacc[i][0] = oacc[i][1] = oacc[i][2] = oacc[i][3] = 0.f;

    const int r0 = warp * 16;
    bool ok = true;
    for (int c = 0; c < n_chunks; ++c) {
        const int st = c % NST;
        if (!mbar_wait(full_bar(st), (c / NST) & 1, abort_flag)) { ok = false; break; }
        const uint32_t sK = sb + st * C::STAGE;
        const uint32_t sV = sK + C::CHUNK;
        const int nvalid = min(64, hi - (lo + c * 64));
        if (r0 + 16 > nvalid) {
            // V rows past the sequence (or never loaded) must be finite: zero them.
            uint8_t* vg = sgen + (sV - sb);
            for (int i = lane; i < 16 * C::NCB * 8; i += 32) {
                const int rr = r0 + i / (C::NCB * 8);
                const int rem = i % (C::NCB * 8);
                const int cb = rem / 8, ch = rem % 8;
                if (rr >= nvalid)
                    *reinterpret_cast<uint4*>(vg + cb * C::BLK + rr * 128 + ch * 16) = make_uint4(0, 0, 0, 0);
            }
            __syncwarp();
        }
        // S = Q K^T over this warp's 16 keys (two n-tiles of 8 keys)
        float sacc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
        {
            const int mat = lane >> 3, rr = lane & 7;
            const int key = r0 + ((mat >> 1) << 3) + rr;
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
                const int cb = kk >> 2;
                const int dcol = (kk & 3) * 16 + ((mat & 1) << 3);
                uint32_t b0, b1, b2, b3;
                ldsm_x4(sK + cb * C::BLK + sw128_offset(key, dcol), b0, b1, b2, b3);
                mma_bf16_16816(sacc[0], qa[kk], b0, b1);
                mma_bf16_16816(sacc[1], qa[kk], b2, b3);
            }
        }
        // online softmax (log2 domain, scale folded in); mask keys >= nvalid
        float mx[2] = {-INFINITY, -INFINITY};
#pragma unroll
        for (int nt = 0; nt < 2; ++nt)
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int key = r0 + nt * 8 + 2 * (lane & 3) + (e & 1);
                const float x = (key < nvalid) ? sacc[nt][e] * sl2 : -INFINITY;
                sacc[nt][e] = x;
                mx[e >> 1] = fmaxf(mx[e >> 1], x);
            }
        float alpha[2], mref[2];
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            mx[h] = fmaxf(mx[h], __shfl_xor_sync(0xffffffffu, mx[h], 1));
            mx[h] = fmaxf(mx[h], __shfl_xor_sync(0xffffffffu, mx[h], 2));
            const float mn = fmaxf(m[h], mx[h]);
            alpha[h] = (m[h] == -INFINITY) ? 0.f : ex2(m[h] - mn);
            m[h] = mn;
            mref[h] = (mn == -INFINITY) ? 0.f : mn;
        }
        float psum[2] = {0.f, 0.f};
#pragma unroll
        for (int nt = 0; nt < 2; ++nt)
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const float pv = ex2(sacc[nt][e] - mref[e >> 1]);
                sacc[nt][e] = pv;
                psum[e >> 1] += pv;
            }
        l[0] = l[0] * alpha[0] + psum[0];
        l[1] = l[1] * alpha[1] + psum[1];
#pragma unroll
        for (int i = 0; i < D / 8; ++i) {
            oacc[i][0] *= alpha[0];
            oacc[i][1] *= alpha[0];
            oacc[i][2] *= alpha[1];
            oacc[i][3] *= alpha[1];
        }
        uint32_t pa[4];
        pa[0] = pack_bf16(sacc[0][0], sacc[0][1]);
        pa[1] = pack_bf16(sacc[0][2], sacc[0][3]);
        pa[2] = pack_bf16(sacc[1][0], sacc[1][1]);
        pa[3] = pack_bf16(sacc[1][2], sacc[1][3]);
        // O += P V over this warp's 16 keys
        {
            const int mat = lane >> 3, rr = lane & 7;
            const int key = r0 + ((mat & 1) << 3) + rr;
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
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(empty_bar(st));
    }

    // ------------------------------------------- combine the four warps' states
    // quad-reduce the row sums
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        l[h] += __shfl_xor_sync(0xffffffffu, l[h], 1);
        l[h] += __shfl_xor_sync(0xffffffffu, l[h], 2);
    }
    // wait for the last chunk of every warp before reusing the ring as scratch
    asm volatile("bar.sync 1, 128;" ::: "memory");
    float* sm_m = reinterpret_cast<float*>(sgen);              // [4][16]
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
    for (int idx = tid; idx < G * D; idx += 128) {
        const int row = idx / D, col = idx % D;
        float M = -INFINITY;
#pragma unroll
        for (int w = 0; w < 4; ++w) M = fmaxf(M, sm_m[w * 16 + row]);
        float Lsum = 0.f, acc = 0.f;
        if (M != -INFINITY) {
#pragma unroll
            for (int w = 0; w < 4; ++w) {
                const float mw = sm_m[w * 16 + row];
                const float f = (mw == -INFINITY) ? 0.f : ex2(mw - M);
                Lsum += f * sm_l[w * 16 + row];
                acc += f * sm_o[(w * 16 + row) * D + col];
            }
        }
        const float outv = (Lsum > 0.f) ? acc / Lsum : 0.f;
        const float lse = (Lsum > 0.f) ? (M + log2f(Lsum)) * 0.6931471805599453f : -INFINITY;
        const int h = g * G + row;
        if (p.num_splits == 1) {
            p.o[(int64_t)b * p.o_bs + (int64_t)h * p.o_hs + col] = __float2bfloat16_rn(outv);
            if (col == 0 && p.lse != nullptr) p.lse[(int64_t)b * p.Hq + h] = lse;
        } else {
            const int64_t rr = (int64_t)s * p.B * p.Hq + (int64_t)b * p.Hq + h;
            p.o_part[rr * D + col] = outv;
            if (col == 0) p.lse_part[rr] = lse;
        }
    }
    (void)ok;
    __syncthreads();
}

// ===========================================================================
// Absorbed-MLA decode: Dqk = 576, Dv = 512, every query head shares one KV
// head ("cuDNN Frontend v1.32.0 Release Notes", "SDPA: wider native forward
// support").  grid (num_splits, Hq / 64, B); 288 threads: warps 0-7 compute,
// warp 8 loads.  Warp w covers query heads [16*(w/2), +16) of the block's 64
// and value columns [256*(w%2), +256); both warps of a pair compute the same
// scores.  With V aliasing K, V is read from the K tile already in shared
// memory.  Chunks are 32 keys.
// ===========================================================================
template <bool ALIAS>
struct MlaCfg {
    static constexpr int DQK = 576, DV = 512;
    static constexpr int KEYS = 32;
    static constexpr uint32_t KBLK = KEYS * 128;         // 32 rows x 128 B
    static constexpr uint32_t KCHUNK = 9 * KBLK;         // 36 KB
    static constexpr uint32_t VCHUNK = ALIAS ? 0 : 8 * KBLK;
    static constexpr uint32_t STAGE = KCHUNK + VCHUNK;
    static constexpr int NST = ALIAS ? 3 : 2;
    static constexpr uint32_t QBLK = 64 * 128;           // 64 heads x 128 B
    static constexpr uint32_t QBYTES = 9 * QBLK;         // 72 KB
    static constexpr uint32_t RING_OFF = QBYTES;
    static constexpr uint32_t BAR_OFF = RING_OFF + NST * STAGE;
    static constexpr uint32_t SMEM = BAR_OFF + 128 + 1024;
};

template <bool ALIAS>
__global__ void __launch_bounds__(288, 1) decode_mla_kernel(const __grid_constant__ DecodeParams p) {
    using C = MlaCfg<ALIAS>;
    constexpr int NST = C::NST;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t sb = (raw + 1023u) & ~1023u;
    uint8_t* sgen = smem_raw + (sb - raw);
    const uint32_t sQ = sb;
    const uint32_t sRing = sb + C::RING_OFF;
    const uint32_t sBar = sb + C::BAR_OFF;
    auto full_bar = [&](int i) { return sBar + 8u * i; };
    auto empty_bar = [&](int i) { return sBar + 8u * (NST + i); };
    const uint32_t b_q = sBar + 16u * NST;
    const uint32_t b_tail = b_q + 8;
    volatile int* abort_flag = reinterpret_cast<volatile int*>(sgen + C::BAR_OFF + 16u * NST + 16);

    const int s = blockIdx.x, hg = blockIdx.y, b = blockIdx.z;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    int L, lo, hi;
    decode_split_range(p, b, s, L, lo, hi);
    const int n_chunks = (hi > lo) ? (hi - lo + C::KEYS - 1) / C::KEYS : 0;

    if (threadIdx.x == 0) {
        for (int i = 0; i < NST; ++i) {
            mbar_init(full_bar(i), 1);
            mbar_init(empty_bar(i), 8);
        }
        mbar_init(b_q, 1);
        mbar_init(b_tail, 1);
        *abort_flag = 0;
        fence_barrier_init();
    }
    __syncthreads();

    if (warp == 8) {
        if (lane == 0) {
            prefetch_tmap(&p.tm_k);
            prefetch_tmap(&p.tm_q);
            mbar_arrive_expect_tx(b_q, C::QBYTES);
            for (int cb = 0; cb < 9; ++cb) tma_load_4d(sQ + cb * C::QBLK, &p.tm_q, b_q, cb * 64, hg * 64, b, 0);
            for (int c = 0; c < n_chunks; ++c) {
                const int st = c % NST;
                if (!mbar_wait(empty_bar(st), ((c / NST) & 1) ^ 1, abort_flag)) break;
                const int t0 = lo + c * C::KEYS;
                const int nkeys = min(C::KEYS, hi - t0);
                const int nboxes = (nkeys + p.box_rows - 1) / p.box_rows;
                const uint32_t kbytes = (uint32_t)nboxes * p.box_rows * 128u * 9u;
                const uint32_t vbytes = ALIAS ? 0u : (uint32_t)nboxes * p.box_rows * 128u * 8u;
                mbar_arrive_expect_tx(full_bar(st), kbytes + vbytes);
                const uint32_t dst = sRing + st * C::STAGE;
                for (int r = 0; r < nkeys; r += p.box_rows) {
                    const int t = t0 + r;
                    int page = __ldg(p.page_table + (int64_t)b * p.pt_stride + t / p.page_size);
                    if (page < 0 || (int64_t)page >= p.num_pages) {
                        record_status(ATTN_ERR_DEVICE_INPUT);
                        page = -1;
                    }
                    const int slot = t % p.page_size;
                    for (int cb = 0; cb < 9; ++cb)
                        tma_load_4d(dst + cb * C::KBLK + r * 128u, &p.tm_k, full_bar(st), cb * 64, slot, 0, page);
                    if (!ALIAS)
                        for (int cb = 0; cb < 8; ++cb)
                            tma_load_4d(dst + C::KCHUNK + cb * C::KBLK + r * 128u, &p.tm_v, full_bar(st),
                                        cb * 64, slot, 0, page);
                }
                if (nkeys < C::KEYS) {
                    // The one partial chunk: once it lands, zero the value rows past the
                    // sequence (aliased: the K rows) so 0 * (stale or NaN) never reaches O,
                    // then release it to the compute warps through b_tail.
                    if (!mbar_wait(full_bar(st), (c / NST) & 1, abort_flag)) break;
                    uint8_t* vg = sgen + ((ALIAS ? dst : dst + C::KCHUNK) - sb);
                    for (int rr = nkeys; rr < C::KEYS; ++rr)
                        for (int i = 0; i < 8 * 8; ++i)
                            *reinterpret_cast<uint4*>(vg + (i >> 3) * C::KBLK + rr * 128 + (i & 7) * 16) =
                                make_uint4(0, 0, 0, 0);
                    mbar_arrive(b_tail);
                }
            }
            for (int c = max(0, n_chunks - NST); c < n_chunks; ++c)
                mbar_wait(full_bar(c % NST), (c / NST) & 1, nullptr, 100000000ull);
            mbar_wait(b_q, 0, nullptr, 100000000ull);
        }
        __syncthreads();
        return;
    }

    const float sl2 = p.scale_log2;
    const int mt = warp >> 1, dh = warp & 1;
    const int hrow0 = mt * 16;  // first head row (within the block's 64) of this warp
    const int qrow = lane >> 2;
    float m[2] = {-INFINITY, -INFINITY};
    float l[2] = {0.f, 0.f};
    float oacc[32][4];  // 16 heads x 256 value columns
#pragma unroll
    for (int i = 0; i < 32; ++i) oacc[i][0] = oacc[i][1] = oacc[i][2] = oacc[i][3] = 0.f;
    bool ok = mbar_wait(b_q, 0, abort_flag);

    for (int c = 0; ok && c < n_chunks; ++c) {
        const int st = c % NST;
        if (!mbar_wait(full_bar(st), (c / NST) & 1, abort_flag)) { ok = false; break; }
        const uint32_t sK = sRing + st * C::STAGE;
        const uint32_t sV = ALIAS ? sK : sK + C::KCHUNK;
        const int nvalid = min(C::KEYS, hi - (lo + c * C::KEYS));
        if (nvalid < C::KEYS && !mbar_wait(b_tail, 0, abort_flag)) { ok = false; break; }
        // S = Q K^T: 16 heads x 32 keys (4 n-tiles), full 576 depth
        float sacc[4][4];
#pragma unroll
        for (int nt = 0; nt < 4; ++nt) sacc[nt][0] = sacc[nt][1] = sacc[nt][2] = sacc[nt][3] = 0.f;
        {
            const int mat = lane >> 3, rr = lane & 7;
#pragma unroll 4
            for (int kk = 0; kk < 36; ++kk) {
                const int cb = kk >> 2;
                uint32_t a[4];
                {
                    // A (16 x 16) from Q: matrices (rows 0-7,k0-7) (rows 8-15,k0-7) (rows 0-7,k8-15) (rows 8-15,k8-15)
                    const int row = hrow0 + ((mat & 1) << 3) + rr;
                    const int dcol = (kk & 3) * 16 + ((mat >> 1) << 3);
                    ldsm_x4(sQ + cb * C::QBLK + sw128_offset(row, dcol), a[0], a[1], a[2], a[3]);
                }
#pragma unroll
                for (int np = 0; np < 2; ++np) {
                    const int key = np * 16 + ((mat >> 1) << 3) + rr;
                    const int dcol = (kk & 3) * 16 + ((mat & 1) << 3);
                    uint32_t b0, b1, b2, b3;
                    ldsm_x4(sK + cb * C::KBLK + sw128_offset(key, dcol), b0, b1, b2, b3);
                    mma_bf16_16816(sacc[2 * np], a, b0, b1);
                    mma_bf16_16816(sacc[2 * np + 1], a, b2, b3);
                }
            }
        }
        float mx[2] = {-INFINITY, -INFINITY};
#pragma unroll
        for (int nt = 0; nt < 4; ++nt)
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int key = nt * 8 + 2 * (lane & 3) + (e & 1);
                const float x = (key < nvalid) ? sacc[nt][e] * sl2 : -INFINITY;
                sacc[nt][e] = x;
                mx[e >> 1] = fmaxf(mx[e >> 1], x);
            }
        float alpha[2], mref[2];
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            mx[h] = fmaxf(mx[h], __shfl_xor_sync(0xffffffffu, mx[h], 1));
            mx[h] = fmaxf(mx[h], __shfl_xor_sync(0xffffffffu, mx[h], 2));
            const float mn = fmaxf(m[h], mx[h]);
            alpha[h] = (m[h] == -INFINITY) ? 0.f : ex2(m[h] - mn);
            m[h] = mn;
            mref[h] = (mn == -INFINITY) ? 0.f : mn;
        }
        float psum[2] = {0.f, 0.f};
#pragma unroll
        for (int nt = 0; nt < 4; ++nt)
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const float pv = ex2(sacc[nt][e] - mref[e >> 1]);
                sacc[nt][e] = pv;
                psum[e >> 1] += pv;
            }
        l[0] = l[0] * alpha[0] + psum[0];
        l[1] = l[1] * alpha[1] + psum[1];
#pragma unroll
        for (int i = 0; i < 32; ++i) {
            oacc[i][0] *= alpha[0];
            oacc[i][1] *= alpha[0];
            oacc[i][2] *= alpha[1];
            oacc[i][3] *= alpha[1];
        }
        // O += P V: k = 32 keys (2 k-steps), n = 256 value columns (32 n-tiles)
#pragma unroll
        for (int ks = 0; ks < 2; ++ks) {
            uint32_t pa[4];
            pa[0] = pack_bf16(sacc[2 * ks][0], sacc[2 * ks][1]);
            pa[1] = pack_bf16(sacc[2 * ks][2], sacc[2 * ks][3]);
            pa[2] = pack_bf16(sacc[2 * ks + 1][0], sacc[2 * ks + 1][1]);
            pa[3] = pack_bf16(sacc[2 * ks + 1][2], sacc[2 * ks + 1][3]);
            const int mat = lane >> 3, rr = lane & 7;
            const int key = ks * 16 + ((mat & 1) << 3) + rr;
#pragma unroll
            for (int nd = 0; nd < 16; ++nd) {
                const int vcol = dh * 256 + nd * 16;
                const int cb = vcol >> 6;
                const int dcol = (vcol & 63) + ((mat >> 1) << 3);
                uint32_t v0, v1, v2, v3;
                ldsm_x4_t(sV + cb * C::KBLK + sw128_offset(key, dcol), v0, v1, v2, v3);
                mma_bf16_16816(oacc[2 * nd], pa, v0, v1);
                mma_bf16_16816(oacc[2 * nd + 1], pa, v2, v3);
            }
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(empty_bar(st));
    }

    // epilogue: each warp owns complete rows for its 256 value columns
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        l[h] += __shfl_xor_sync(0xffffffffu, l[h], 1);
        l[h] += __shfl_xor_sync(0xffffffffu, l[h], 2);
    }
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        const int head = hg * 64 + hrow0 + qrow + 8 * h;
        const float inv = (l[h] > 0.f) ? 1.f / l[h] : 0.f;
        const float lse = (l[h] > 0.f) ? (m[h] + log2f(l[h])) * 0.6931471805599453f : -INFINITY;
        if (p.num_splits == 1) {
            __nv_bfloat16* orow = p.o + (int64_t)b * p.o_bs + (int64_t)head * p.o_hs;
#pragma unroll
            for (int i = 0; i < 32; ++i) {
                const int col = dh * 256 + i * 8 + 2 * (lane & 3);
                *reinterpret_cast<uint32_t*>(orow + col) = pack_bf16(oacc[i][2 * h] * inv, oacc[i][2 * h + 1] * inv);
            }
            if (dh == 0 && (lane & 3) == 0 && p.lse != nullptr) p.lse[(int64_t)b * p.Hq + head] = lse;
        } else {
            const int64_t rr = (int64_t)s * p.B * p.Hq + (int64_t)b * p.Hq + head;
            float* orow = p.o_part + rr * C::DV;
#pragma unroll
            for (int i = 0; i < 32; ++i) {
                const int col = dh * 256 + i * 8 + 2 * (lane & 3);
                *reinterpret_cast<float2*>(orow + col) = make_float2(oacc[i][2 * h] * inv, oacc[i][2 * h + 1] * inv);
            }
            if (dh == 0 && (lane & 3) == 0) p.lse_part[rr] = lse;
        }
    }
    __syncthreads();
}

}  // namespace b2
