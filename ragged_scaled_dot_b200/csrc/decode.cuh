// decode.cuh -- paged-KV decode (one query token per sequence) with split-KV.
//
// Pages are gathered with TMA, one box per page covering every column block
// (min(page size, 64) rows): the page table gives the physical page of each
// logical page ("cuDNN Frontend v1.31.0 Release Notes", "SDPA: paged KV,
// split-KV, and engine selection").  One producer thread issues a chunk's boxes
// for pages of 64 keys or more; for smaller pages the producer warp issues them
// together, one lane per box.
// Decode is HBM-bound (8 flop per KV byte at Hq/Hkv = 8), so the small
// contractions run on warp-level MMAs while the memory system streams pages;
// the G query heads of one KV head are the MMA rows, so every K/V byte is read
// once per KV head ("cuDNN Frontend v1.30.0 Release Notes", "New: decode
// tiles", PackGQA).
//
// Split-KV (num_splits > 1).  The keys of every (sequence, KV head) pair are
// cut into 64-key units, and a pair with n units into k = min(num_splits, n)
// pieces of n/k units (to within one), one decode block per piece
// ("cuDNN Frontend v1.31.0 Release Notes", "SDPA: paged KV, split-KV, and
// engine selection").  decode_schedule_kernel writes the pieces before the
// decode launch, the sequences longest first, so the blocks of the longest
// pieces start first and the short ones fill the end of the last wave.  A
// piece that is the whole pair is written directly; otherwise each piece
// writes one fp32 partial (normalised O, base-2 LSE), and the last block to
// finish a group of up to 8 of a pair's partials merges the group by LSE --
// the arrival counters tell it so without any wait -- until one result
// remains.  No separate merge launch.
#pragma once

#include "aux_kernels.cuh"
#include "paging.cuh"
#include "ptx.cuh"

namespace b2 {

// The piece a decode block runs: units [j0, j1) (keys [64 j0, min(64 j1, L)))
// of pair = b * Hkv + g (-1: no piece for this block).  The pair's nseg pieces
// run in blocks slot0 .. slot0 + nseg - 1, whose indices are also the slots of
// their partials.  An empty sequence is one unit without keys.
struct DecodeSeg {
    int pair, j0, j1;
    int slot0, nseg;
    int L;       // cached keys of the sequence
    int q0, Lq;  // first query token and query count (decode: b, 1)
};
static_assert(sizeof(DecodeSeg) == 32, "two 16-byte loads per piece");

constexpr int kMergeFan = 8;     // partials merged by one block
constexpr int kMergeLevels = 4;  // up to kMergeFan^4 pieces per pair

struct DecodeParams {
    // GQA: 5D (column in block, slot, 64-column block, head, page), 128B swizzle, box
    // (64, min(ps, 64), D / 64, 1, 1); MLA: K (column in block, row in 8-row group,
    // column block, 8-row group, head), box (64, 8, 9, min(ps, 64) / 8, 1), and V as for GQA
    // with 8 column blocks
    CUtensorMap tm_k;
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
    int groups_per_page;      // MLA K map: 8-row groups per page stride (group-major boxes)
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
    // partials (num_splits > 1).  GQA: by block, [n_slots][G*qmax][Dv] normalised O and
    // [n_slots][G*qmax] base-2 LSE, row qi*G + gh.  MLA: [S][B*Hq][Dv] and natural-log
    // [S][B*Hq], row b*Hq + h.
    float* o_part;
    float* lse_part;
    // GQA split (null without splits): the piece of every block and kMergeLevels rows of
    // n_slots arrival counters
    const DecodeSeg* segs;
    int* ctr;
    int n_slots;  // blocks of the launch: num_splits * pairs
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
// rows [r, r + box_rows) come from one page (NB = 64 / box_rows boxes), each box
// all column blocks of those rows, landing at dst + i * (ncol_blocks * box_rows *
// 128) as [column block][rows][128 B] (for box_rows 64: the [column block][64
// rows] tile).  All page ids of the chunk are read before any box is issued, so
// their latencies overlap (each TMA issue is ordered after the reads before it),
// and with one page table for K and V the V boxes reuse the K boxes' ids.  One
// thread issues them; the kernel uses this for pages of 64 keys or more (NB = 1),
// and decode_produce_small_pages below for smaller pages.
template <int NB>
__device__ __forceinline__ void decode_issue_kv(const DecodeParams& p, uint32_t dst_k, uint32_t dst_v, uint32_t bar,
                                                int b, int g, int t0, int hi, int ncol_blocks,
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
    const uint32_t box_bytes = (uint32_t)(ncol_blocks * R) * 128u;
#pragma unroll
    for (int i = 0; i < NB; ++i) {
        const int t = t0 + i * R;
        if (t < hi) {
            // out of range: page -1, and TMA fills the box with zeros
            const int pk = page_checked(idk[i], p.num_pages);
            const int pv = shared_table ? pk : page_checked(idv[i], p.num_pages);
            const int slot = page_slot(t, p.page_size);
            tma_load_5d(dst_k + i * box_bytes, &p.tm_k, bar, 0, slot, 0, g, pk);
            tma_load_5d(dst_v + i * box_bytes, &p.tm_v, bar, 0, slot, 0, g, pv);
        }
    }
}

// Pages of fewer than 64 keys: the producer warp issues a chunk's boxes together,
// lane i < NB K box i and lane NB + i V box i (NB = 64 / box_rows), each lane reading
// its own page id (from the piece's window, else the table; V boxes read the K ids
// when K and V share a table).  One thread issuing the 8 boxes of a page-16 chunk
// one after another spent ~275 cycles a box, longer than the compute warps take to
// consume the chunk.  Kept out of line so the whole-page loop stays as it was (the
// warp-wide loop made that one slower).  Returns the chunks issued.
template <int NST>
__device__ __noinline__ int decode_produce_small_pages(const DecodeParams& p, uint32_t sBar, volatile int* abort_flag,
                                                       uint32_t sb, uint32_t stage_bytes, uint32_t chunk_bytes,
                                                       int ncb, int b, int g, int lo, int hi, int n_chunks,
                                                       const volatile int* ids_k, const volatile int* ids_v, int p0,
                                                       int nids, int lane) {
    const int R = p.box_rows;
    const int NB = 64 / R;
    const bool is_v = lane >= NB;
    const int i = is_v ? lane - NB : lane;
    const bool v_table = is_v && !(p.v_page_table == p.page_table && p.v_pt_stride == p.pt_stride);
    const uint32_t box_bytes = (uint32_t)(ncb * R) * 128u;
    int cc = 0;
    for (; cc < n_chunks; ++cc) {
        const int st = cc % NST;
        const uint32_t full = sBar + 8u * st, empty = sBar + 8u * (NST + st);
        const int t0 = lo + cc * 64;  // t0 >= hi only for the keyless unit of an empty sequence
        bool w_ok = true;
        if (lane == 0) {
            w_ok = mbar_wait(empty, ((cc / NST) & 1) ^ 1, abort_flag);
            if (w_ok) mbar_arrive_expect_tx(full, t0 < hi ? decode_chunk_bytes(p, t0, hi, ncb, 2) : 0u);
        }
        // the stage is free and its byte count set before any lane issues a box
        if (!__shfl_sync(0xffffffffu, w_ok ? 1 : 0, 0)) break;
        const int t = t0 + i * R;
        if (lane < 2 * NB && t < hi) {
            const int w = t / p.page_size - p0;  // position in the window of shared-memory ids
            int id;
            if (w < nids) id = v_table ? ids_v[w] : ids_k[w];
            else if (v_table) id = page_lookup(p.v_page_table, p.v_pt_stride, b, t, p.page_size);
            else id = page_lookup(p.page_table, p.pt_stride, b, t, p.page_size);
            // out of range: page -1, and TMA fills the box with zeros
            const int page = page_checked(id, p.num_pages);
            const uint32_t dst = sb + st * stage_bytes + (is_v ? chunk_bytes : 0u) + i * box_bytes;
            tma_load_5d(dst, is_v ? &p.tm_v : &p.tm_k, full, 0, page_slot(t, p.page_size), 0, g, page);
        }
    }
    return cc;
}

// Byte offset of key row k of a chunk's K (or V) tile, column block 0: page box
// k / R of NCB column blocks of R rows (R = 2^lR, at least 8), row k % R.  The
// 128-byte swizzle of the row is (k & 7), as each box starts on 1 KB.
__device__ __forceinline__ uint32_t decode_row_off(int k, int lR, int ncb) {
    return ((uint32_t)((k >> lR) * ncb) << (lR + 7)) + ((uint32_t)(k & ((1 << lR) - 1)) << 7);
}

// ===========================================================================
// Split schedule of the GQA decode (one block of 1024 threads, before the
// decode launch).  Units of sequence b: max(1, ceil(L_b / 64)) when its rows
// belong to the decode kernel (every sequence without cu_q; 1 <= Lq <= qmax
// with it), else none.  The sequences are sorted longest first (counting sort
// of n >> shift over kSortBuckets buckets, the host choosing shift so that
// every key fits; ties in any order).  In that order, each of the Hkv pairs
// of a sequence with n units takes k = min(num_splits, n) consecutive blocks,
// block s of them the units [s n / k, (s+1) n / k).  Writes per sequence
// (units, L, q0, Lq) into `seq`, the order into `order`, every block's piece
// into `segs` (pair -1 past the last piece) and zeroes the merge counters.
// Kernel arguments out of range (L outside [0, max_kv_len], inconsistent
// cu_q) are recorded as ATTN_ERR_DEVICE_INPUT; such a sequence is clamped or
// skipped, as without splits.
// ===========================================================================
__global__ void __launch_bounds__(1024) decode_schedule_kernel(const __grid_constant__ DecodeParams p, int shift,
                                                               int4* __restrict__ seq, int32_t* __restrict__ order,
                                                               DecodeSeg* __restrict__ segs, int* __restrict__ ctr) {
    __shared__ int hist[kSortBuckets];
    __shared__ int warp_sums[32];
    const int tid = threadIdx.x;
    const int Hkv = p.Hkv, S = p.num_splits;
    auto bucket = [&](int n) { return kSortBuckets - 1 - min(kSortBuckets - 1, n >> shift); };
    for (int i = tid; i < kSortBuckets; i += blockDim.x) hist[i] = 0;
    __syncthreads();
    for (int b = tid; b < p.B; b += blockDim.x) {
        int L = p.kv_lens[b];
        if (L < 0 || L > p.max_kv_len) {
            record_status(ATTN_ERR_DEVICE_INPUT);
            L = max(0, min(L, p.max_kv_len));
        }
        int q0 = b, Lq = 1;
        bool mine = true;
        if (p.cu_q != nullptr) {
            const int a0 = p.cu_q[b], a1 = p.cu_q[b + 1];
            if (a0 < 0 || a1 < a0 || (int64_t)a1 > p.total_q) {
                record_status(ATTN_ERR_DEVICE_INPUT);
                mine = false;
            } else {
                q0 = a0;
                Lq = a1 - a0;
                mine = Lq >= 1 && Lq <= p.qmax;
            }
        }
        const int n = mine ? max(1, (L + 63) / 64) : 0;
        seq[b] = make_int4(n, L, q0, Lq);
        atomicAdd(&hist[bucket(n)], 1);
    }
    __syncthreads();
    bucket_exclusive_scan(hist, warp_sums);
    for (int b = tid; b < p.B; b += blockDim.x) order[atomicAdd(&hist[bucket(seq[b].x)], 1)] = b;
    __syncthreads();
    // the pieces, sequence after sequence in that order
    int carry = 0;
    for (int base = 0; base < p.B; base += blockDim.x) {
        const int i = base + tid;
        int4 sq = make_int4(0, 0, 0, 0);
        int b = 0, k = 0;
        if (i < p.B) {
            b = order[i];
            sq = seq[b];
            k = min(S, sq.x);
        }
        int total;
        const int first = carry + block_exclusive_scan(Hkv * k, warp_sums, &total);
        for (int g = 0; g < Hkv && k > 0; ++g) {
            const int slot0 = first + g * k;
            for (int s = 0; s < k; ++s) {
                int4* rec = reinterpret_cast<int4*>(segs + slot0 + s);
                rec[0] = make_int4(b * Hkv + g, (int)((int64_t)s * sq.x / k), (int)((int64_t)(s + 1) * sq.x / k),
                                   slot0);
                rec[1] = make_int4(k, sq.y, sq.z, sq.w);
            }
        }
        carry += total;
    }
    for (int c = carry + tid; c < p.n_slots; c += blockDim.x)
        reinterpret_cast<int4*>(segs + c)[0] = make_int4(-1, 0, 0, 0);
    for (int i = tid; i < kMergeLevels * p.n_slots; i += blockDim.x) ctr[i] = 0;
}

// ===========================================================================
// GQA decode, Dqk = Dv = D in {64, 128}, 160 threads: warps 0-3 compute, warp
// 4 loads.  Grid (1, Hkv, B) without splits (a block per pair, all its keys),
// else one block per scheduled piece.  The MMA rows are the query rows of one
// KV head: row r = qi * G + gh is query token qi of the sequence (one token for
// decode; up to qmax with cu_q: multi-token decode, speculative tokens) and
// query head g * G + gh, 16 * RT rows in RT m16 tiles ("cuDNN Frontend v1.30.0
// Release Notes", "New: decode tiles": G query heads x small query counts as
// the tile rows; "cuDNN Frontend v1.31.0 Release Notes", "SDPA: paged KV,
// split-KV, and engine selection": paged THD split-KV).  Warp w computes
// m-tile w % RT over keys [(w / RT) * 16 RT, (w / RT + 1) * 16 RT) of every
// 64-key chunk and keeps its own online-softmax state; at the end the states
// of the warps of one m-tile are combined through the stage of the last chunk,
// each row's weights computed once.  RT = 1 without cu_q is plain decode.
// ===========================================================================
// NST stages of K/V: 3 lets two blocks share an SM; 6 is for launches with at most
// one block per SM, which then keep twice the bytes in flight.
template <int D, int NST_ = 3>
struct DecodeCfg {
    static constexpr int NCB = D / 64;                  // 64-wide column blocks
    static constexpr uint32_t BLK = 64 * 128;           // one column block of a chunk (64 rows of 128 B)
    static constexpr uint32_t CHUNK = NCB * BLK;        // K (or V) bytes of a chunk
    static constexpr int NST = NST_;
    static_assert(NST >= 2 && 16 * NST + 4 <= 128, "full and empty barriers and the abort flag fit the barrier area");
    static constexpr uint32_t STAGE = 2 * CHUNK;        // K then V
    static constexpr uint32_t BAR_OFF = NST * STAGE;
    // the page ids of the piece (K table, then V table when it has its own), read by the
    // loading warp before its first load
    static constexpr int IDW = 1024;                  // page ids per table in the window
    static constexpr uint32_t IDS_OFF = BAR_OFF + 128;
    static constexpr uint32_t ML_OFF = IDS_OFF + 2 * IDW * 4;  // float [2][4 warps][16 rows]: m, l
    static constexpr uint32_t W_OFF = ML_OFF + 512;             // float [kMergeFan][64 rows]: merge weights
    static constexpr uint32_t SMEM = W_OFF + kMergeFan * 64 * 4 + 1024;
    static_assert(4 * 16 * D * 4 <= STAGE, "one stage holds the four warps' O");
};

// Merges group after group of the pair's partials (slots slot0 .. slot0 +
// nseg - 1) as long as this block is the last of its group to arrive, by the
// 128 compute threads: weights w_e = 2^(lse_e - M) /
// sum_e 2^(lse_e - M), O = sum_e w_e O_e, LSE = M + log2(sum).  A group's
// result replaces its first element; the top group's is the output.
template <int D>
__device__ __forceinline__ void decode_merge_up(const DecodeParams& p, const DecodeSeg& sg, int id, int b, int g,
                                                int tok0, int n_rows, float* sm_w) {
    const int tid = threadIdx.x;
    const int rps = p.G * p.qmax;
    int idx = id - sg.slot0;  // this block's element at the current level
    int n = sg.nseg;          // elements at the current level
    int stride = 1;           // pieces per element
    for (int lvl = 0; lvl < kMergeLevels && n > 1; ++lvl) {
        const int first = (idx / kMergeFan) * kMergeFan;
        const int cnt = min(kMergeFan, n - first);
        const int slot0 = sg.slot0 + first * stride;
        // this block's partial before its arrival; the group's last block sees all of them
        __threadfence();
        asm volatile("bar.sync 1, 128;" ::: "memory");
        bool last = false;
        if (tid == 0) last = atomicAdd(p.ctr + (int64_t)lvl * p.n_slots + slot0, 1) == cnt - 1;
        if (!bar_or(1, 128, last)) return;
        __threadfence();
        const bool top = n <= kMergeFan;
        if (cnt > 1) {
            if (tid < n_rows) {
                float w[kMergeFan];
                float M = -INFINITY;
#pragma unroll
                for (int e = 0; e < kMergeFan; ++e) {
                    w[e] = (e < cnt) ? __ldcg(p.lse_part + (int64_t)(slot0 + e * stride) * rps + tid) : -INFINITY;
                    M = fmaxf(M, w[e]);
                }
                float sum = 0.f;
#pragma unroll
                for (int e = 0; e < kMergeFan; ++e) {
                    w[e] = (M == -INFINITY) ? 0.f : ex2(w[e] - M);
                    sum += w[e];
                }
                const float inv = sum > 0.f ? 1.f / sum : 0.f;
#pragma unroll
                for (int e = 0; e < kMergeFan; ++e) sm_w[e * 64 + tid] = w[e] * inv;
                const float lse2 = sum > 0.f ? M + log2f(sum) : -INFINITY;
                if (!top) {
                    p.lse_part[(int64_t)slot0 * rps + tid] = lse2;
                } else if (p.lse != nullptr) {
                    const int qi = tid / p.G, h = g * p.G + (tid - qi * p.G);
                    p.lse[decode_lse_index(p.lse_layout, b, qi, (int64_t)tok0 + qi, h, p.Hq, p.lse_smax, p.lse_hs)] =
                        p.lse_log2 ? lse2 : lse2 * 0.6931471805599453f;
                }
            }
            asm volatile("bar.sync 1, 128;" ::: "memory");
            for (int e4 = tid; e4 < n_rows * (D / 4); e4 += 128) {
                const int row = e4 / (D / 4), col = (e4 - row * (D / 4)) * 4;
                float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
                for (int e = 0; e < kMergeFan; ++e) {
                    if (e < cnt) {
                        const float we = sm_w[e * 64 + row];
                        const float4 v = __ldcg(reinterpret_cast<const float4*>(
                            p.o_part + ((int64_t)(slot0 + e * stride) * rps + row) * D + col));
                        acc.x += we * v.x;
                        acc.y += we * v.y;
                        acc.z += we * v.z;
                        acc.w += we * v.w;
                    }
                }
                if (!top) {
                    *reinterpret_cast<float4*>(p.o_part + ((int64_t)slot0 * rps + row) * D + col) = acc;
                } else {
                    const int qi = row / p.G, h = g * p.G + (row - qi * p.G);
                    uint2 packed;
                    packed.x = pack_bf16(acc.x, acc.y);
                    packed.y = pack_bf16(acc.z, acc.w);
                    *reinterpret_cast<uint2*>(p.o + ((int64_t)tok0 + qi) * p.o_bs + (int64_t)h * p.o_hs + col) = packed;
                }
            }
            asm volatile("bar.sync 1, 128;" ::: "memory");  // sm_w is reused
        }
        if (top) return;
        idx = first / kMergeFan;
        n = (n + kMergeFan - 1) / kMergeFan;
        stride *= kMergeFan;
    }
}

template <int D, int RT, int NST_ = 3>
__global__ void __launch_bounds__(160, NST_ <= 3 ? 2 : 1) decode_gqa_kernel(const __grid_constant__ DecodeParams p) {
    using C = DecodeCfg<D, NST_>;
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
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    // the piece this block runs: from the split schedule, or without splits KV head
    // blockIdx.y of sequence blockIdx.z, all of its keys
    DecodeSeg sg;
    if (p.segs != nullptr) {
        const int4* r = reinterpret_cast<const int4*>(p.segs + blockIdx.x);
        const int4 a = __ldg(r);
        if (a.x < 0) return;  // no piece for this block, before any barrier exists
        const int4 c = __ldg(r + 1);
        sg.pair = a.x;
        sg.j0 = a.y;
        sg.j1 = a.z;
        sg.slot0 = a.w;
        sg.nseg = c.x;
        sg.L = c.y;
        sg.q0 = c.z;
        sg.Lq = c.w;
    } else {
        const int b = blockIdx.z;
        sg.pair = b * p.Hkv + (int)blockIdx.y;
        sg.q0 = b;
        sg.Lq = 1;
        if (p.cu_q != nullptr) {
            const int q0 = __ldg(p.cu_q + b), q1 = __ldg(p.cu_q + b + 1);
            if (q0 < 0 || q1 < q0 || (int64_t)q1 > p.total_q) {
                if (threadIdx.x == 0) record_status(ATTN_ERR_DEVICE_INPUT);
                return;  // the whole block leaves before any barrier exists
            }
            sg.q0 = q0;
            sg.Lq = q1 - q0;
            if (sg.Lq < 1 || sg.Lq > p.qmax) return;  // no queries, or a sequence of the prefill kernel
        }
        int L = __ldg(p.kv_lens + b);
        if (L < 0 || L > p.max_kv_len) {
            record_status(ATTN_ERR_DEVICE_INPUT);
            L = max(0, min(L, p.max_kv_len));
        }
        sg.L = L;
        sg.j0 = 0;
        sg.j1 = max(1, (L + 63) / 64);
        sg.slot0 = 0;
        sg.nseg = 1;
    }
    const int b = sg.pair / p.Hkv, g = sg.pair - b * p.Hkv;
    const int lo = sg.j0 * 64, hi = min(sg.j1 * 64, sg.L);
    const int n_chunks = sg.j1 - sg.j0;  // at least 1

    if (threadIdx.x == 0) {
        for (int i = 0; i < NST; ++i) {
            mbar_init(full_bar(i), 1);
            mbar_init(empty_bar(i), 4);
        }
        *abort_flag = 0;
        fence_barrier_init();
    }
    __syncthreads();
    volatile int* ids_k = reinterpret_cast<volatile int*>(sgen + C::IDS_OFF);
    volatile int* ids_v = ids_k + C::IDW;

    if (warp == 4) {
        // ---------------------------------------------------------- loads
        if (lane == 0) {
            prefetch_tmap(&p.tm_k);
            prefetch_tmap(&p.tm_v);
        }
        const bool own_v = !(p.v_page_table == p.page_table && p.v_pt_stride == p.pt_stride);
        // the piece's page ids (up to IDW per table), read by the whole warp at once
        const int p0 = lo / p.page_size;
        const int nids = (hi > lo) ? min(C::IDW, (hi - 1) / p.page_size - p0 + 1) : 0;
        {
            const int32_t* rk = p.page_table + (int64_t)b * p.pt_stride + p0;
            const int32_t* rv = p.v_page_table + (int64_t)b * p.v_pt_stride + p0;
            for (int i = lane; i < nids; i += 32) {
                ids_k[i] = __ldg(rk + i);
                if (own_v) ids_v[i] = __ldg(rv + i);
            }
        }
        __syncwarp();
        int cc = 0;  // chunks issued
        if (p.box_rows < 64) {
            cc = decode_produce_small_pages<NST>(p, sBar, abort_flag, sb, C::STAGE, C::CHUNK, C::NCB, b, g, lo, hi,
                                                 n_chunks, ids_k, ids_v, p0, nids, lane);
        } else if (lane == 0) {
            for (; cc < n_chunks; ++cc) {
                const int st = cc % NST;
                if (!mbar_wait(empty_bar(st), ((cc / NST) & 1) ^ 1, abort_flag)) break;
                const int t0 = lo + cc * 64;  // t0 >= hi only for the keyless unit of an empty sequence
                mbar_arrive_expect_tx(full_bar(st), t0 < hi ? decode_chunk_bytes(p, t0, hi, C::NCB, 2) : 0u);
                const uint32_t dst = sb + st * C::STAGE;
                decode_issue_kv<1>(p, dst, dst + C::CHUNK, full_bar(st), b, g, t0, hi, C::NCB, ids_k, ids_v, p0, nids);
            }
        }
        // drain: every issued load lands before the block leaves
        if (lane == 0)
            for (int c = max(0, cc - NST); c < cc; ++c)
                mbar_wait(full_bar(c % NST), (c / NST) & 1, nullptr, 100000000ull);
        __syncthreads();  // matches the compute warps' final barrier
        return;
    }

    // ---------------------------------------------------------------- compute
    const float sl2 = p.scale_log2;
    const int G = p.G;
    const int rps = G * p.qmax;          // partial rows per slot
    const int mt = warp % RT;            // this warp's m-tile (rows 16 mt .. 16 mt + 15)
    const int kbase = (warp / RT) * KW;  // its keys inside every chunk
    const int qrow = lane >> 2;          // rows qrow and qrow + 8 of the m-tile
    const int tid = threadIdx.x;         // 0..127
    float* sm_m = reinterpret_cast<float*>(sgen + C::ML_OFF);  // [4 warps][16 rows of the warp's m-tile]
    float* sm_l = sm_m + 64;                                    // [4][16]
    float* sm_w = reinterpret_cast<float*>(sgen + C::W_OFF);
    bool ok = true;
    {
        const int L = sg.L, Lq = sg.Lq;
        const int tok0 = p.cu_q != nullptr ? sg.q0 : b;
        const int n_rows = G * Lq;
        const bool active = mt * 16 < n_rows;
        // Q as A fragments (zero past the last row)
        uint32_t qa[D / 16][4];
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
            const int col = kk * 16 + 2 * (lane & 3);
#pragma unroll
            for (int part = 0; part < 4; ++part) {
                const int row = mt * 16 + qrow + ((part & 1) ? 8 : 0);
                const int cc2 = col + ((part & 2) ? 8 : 0);
                uint32_t v = 0u;
                if (row < n_rows) {
                    const int qi = row / G, gh = row - qi * G;
                    v = *reinterpret_cast<const uint32_t*>(p.q + (int64_t)(tok0 + qi) * p.q_bs +
                                                           (int64_t)(g * G + gh) * p.q_hs + cc2);
                }
                qa[kk][part] = v;
            }
        }
        // keys each of this thread's two rows may see: below rlim (bottom-right causal:
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
        // this lane's ldmatrix rows in every chunk: keys kbase + 16 kg + (0 or 8) + lane % 8
        // of the QK (K) and PV (V) fragments, as offsets into the page-box layout; their
        // 128-byte swizzle is lane % 8
        const int lR = 31 - __clz(p.box_rows);
        const uint32_t cbs = 128u << lR;  // bytes per column block of a page box
        uint32_t row_k[RT], row_v[RT];
#pragma unroll
        for (int kg = 0; kg < RT; ++kg) {
            row_k[kg] = decode_row_off(kbase + 16 * kg + (((lane >> 3) >> 1) << 3) + (lane & 7), lR, C::NCB);
            row_v[kg] = decode_row_off(kbase + 16 * kg + (((lane >> 3) & 1) << 3) + (lane & 7), lR, C::NCB);
        }

        for (int k = 0; k < n_chunks; ++k) {
            const int st = k % NST;
            if (ok && !mbar_wait(full_bar(st), (k / NST) & 1, abort_flag)) ok = false;
            const uint32_t sK = sb + st * C::STAGE;
            const uint32_t sV = sK + C::CHUNK;
            const int t0 = lo + k * 64;
            const int nvalid = min(64, hi - t0);  // <= 0 only for the keyless unit
            bool zeroed = false;
            if (ok && active) {
                if (kbase + KW > nvalid) {
                    zeroed = true;
                    // V rows past the piece (or never loaded) must be finite: zero them.
                    uint8_t* vg = sgen + (sV - sb);
                    for (int i = lane; i < KW * C::NCB * 8; i += 32) {
                        const int rr = kbase + i / (C::NCB * 8);
                        const int rem = i % (C::NCB * 8);
                        const int cb = rem / 8, ch = rem % 8;
                        if (rr >= nvalid)
                            *reinterpret_cast<uint4*>(vg + decode_row_off(rr, lR, C::NCB) + cb * cbs + ch * 16) =
                                make_uint4(0, 0, 0, 0);
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
                    const int mat = lane >> 3, sw = lane & 7;
#pragma unroll
                    for (int kg = 0; kg < RT; ++kg) {
#pragma unroll
                        for (int kk = 0; kk < D / 16; ++kk) {
                            const int cb = kk >> 2;
                            const uint32_t chunk16 = (uint32_t)((((kk & 3) << 1) | (mat & 1)) ^ sw);
                            uint32_t b0, b1, b2, b3;
                            ldsm_x4(sK + row_k[kg] + cb * cbs + (chunk16 << 4), b0, b1, b2, b3);
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
                const int mat = lane >> 3, sw = lane & 7;
#pragma unroll
                for (int kg = 0; kg < RT; ++kg) {
                    uint32_t pa[4];
                    pa[0] = pack_bf16(sacc[2 * kg][0], sacc[2 * kg][1]);
                    pa[1] = pack_bf16(sacc[2 * kg][2], sacc[2 * kg][3]);
                    pa[2] = pack_bf16(sacc[2 * kg + 1][0], sacc[2 * kg + 1][1]);
                    pa[3] = pack_bf16(sacc[2 * kg + 1][2], sacc[2 * kg + 1][3]);
#pragma unroll
                    for (int nd = 0; nd < D / 16; ++nd) {
                        const int cb = nd >> 2;
                        const uint32_t chunk16 = (uint32_t)((((nd & 3) << 1) | (mat >> 1)) ^ sw);
                        uint32_t v0, v1, v2, v3;
                        ldsm_x4_t(sV + row_v[kg] + cb * cbs + (chunk16 << 4), v0, v1, v2, v3);
                        mma_bf16_16816(oacc[2 * nd], pa, v0, v1);
                        mma_bf16_16816(oacc[2 * nd + 1], pa, v2, v3);
                    }
                }
            }
            // the piece's last stage stays held: it is the scratch of the combine below
            if (k + 1 < n_chunks) {
                // generic writes to the stage (the zeroed V rows) are ordered before the next
                // TMA writes into it; reads need only the barrier
                if (zeroed) fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) mbar_arrive(empty_bar(st));
            }
        }

        // --------------------------------------- combine the warps' states
        // quad-reduce the row sums
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
            l[hh] += __shfl_xor_sync(0xffffffffu, l[hh], 1);
            l[hh] += __shfl_xor_sync(0xffffffffu, l[hh], 2);
        }
        const int st_last = (n_chunks - 1) % NST;
        float* sm_o = reinterpret_cast<float*>(sgen + st_last * C::STAGE);  // [4 warps][16 rows][D]
        // every warp is done with the last chunk before its stage is overwritten
        asm volatile("bar.sync 1, 128;" ::: "memory");
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
        const bool whole = sg.nseg == 1;  // the piece is the whole pair
        const int id = blockIdx.x;        // with splits, this block's partial slot
        // per row (one thread each): the weight of every warp's state, 2^(m_w - M) / Lsum,
        // and the row's LSE (base 2) -- computed once, not per element
        float* sm_f = sm_w;  // [4 warps][64 rows]
        if (tid < n_rows) {
            const int rmt = tid >> 4, rr = tid & 15;  // m-tile, row inside it: warps rmt, rmt + RT, ...
            float M = -INFINITY;
#pragma unroll
            for (int w = 0; w < 4; ++w)
                if (w % RT == rmt) M = fmaxf(M, sm_m[w * 16 + rr]);
            float f[4] = {0.f, 0.f, 0.f, 0.f};
            float Lsum = 0.f;
            if (M != -INFINITY) {
#pragma unroll
                for (int w = 0; w < 4; ++w) {
                    if (w % RT != rmt) continue;
                    const float mw = sm_m[w * 16 + rr];
                    f[w] = (mw == -INFINITY) ? 0.f : ex2(mw - M);
                    Lsum += f[w] * sm_l[w * 16 + rr];
                }
            }
            const float inv = (Lsum > 0.f) ? 1.f / Lsum : 0.f;
#pragma unroll
            for (int w = 0; w < 4; ++w)
                if (w % RT == rmt) sm_f[w * 64 + tid] = f[w] * inv;
            const float lse2 = (Lsum > 0.f) ? (M + log2f(Lsum)) : -INFINITY;
            if (!whole) {
                p.lse_part[(int64_t)id * rps + tid] = lse2;
            } else if (p.lse != nullptr) {
                const int qi = tid / G, h = g * G + (tid - qi * G);
                p.lse[decode_lse_index(p.lse_layout, b, qi, (int64_t)tok0 + qi, h, p.Hq, p.lse_smax, p.lse_hs)] =
                    p.lse_log2 ? lse2 : lse2 * 0.6931471805599453f;
            }
        }
        asm volatile("bar.sync 1, 128;" ::: "memory");
        // per element, four columns at a time: O = sum_w weight_w O_w
        for (int e4 = tid; e4 < n_rows * (D / 4); e4 += 128) {
            const int row = e4 / (D / 4), col = (e4 - row * (D / 4)) * 4;
            const int rmt = row >> 4, rr = row & 15;
            float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
            for (int w = rmt; w < 4; w += RT) {
                const float fw = sm_f[w * 64 + row];
                const float4 v = *reinterpret_cast<const float4*>(sm_o + (w * 16 + rr) * D + col);
                acc.x += fw * v.x;
                acc.y += fw * v.y;
                acc.z += fw * v.z;
                acc.w += fw * v.w;
            }
            if (whole) {
                const int qi = row / G, h = g * G + (row - qi * G);
                uint2 packed;
                packed.x = pack_bf16(acc.x, acc.y);
                packed.y = pack_bf16(acc.z, acc.w);
                *reinterpret_cast<uint2*>(p.o + ((int64_t)tok0 + qi) * p.o_bs + (int64_t)h * p.o_hs + col) = packed;
            } else {
                *reinterpret_cast<float4*>(p.o_part + ((int64_t)id * rps + row) * D + col) = acc;
            }
        }
        // the last stage is free again: the scratch (and any zeroed V rows) are generic
        // writes, ordered before the next TMA writes into it
        asm volatile("bar.sync 1, 128;" ::: "memory");
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(empty_bar(st_last));
        if (!whole) decode_merge_up<D>(p, sg, id, b, g, tok0, n_rows, sm_w);
    }
    __syncthreads();
}

}  // namespace b2
