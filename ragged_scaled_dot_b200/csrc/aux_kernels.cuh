// aux_kernels.cuh -- device-side metadata for the ragged layout, the padded
// LSE fill, the split-KV LSE merge and the bounded-wait self-test.
#pragma once

#include "prefill.cuh"
#include "ptx.cuh"

namespace b2 {

// ---------------------------------------------------------------------------
// Ragged work list, built on the device from the offset tables so the host
// never reads them back ("cuDNN Frontend v1.28.0 release notes", "Ragged /
// THD, with zero host reads"; "cuDNN Frontend v1.32.0 Release Notes", native
// THD metadata setup fused on the device, work prefixes).  One block:
//   1. validate each sequence against the host-declared capacities;
//   2. order sequences most work first (counting sort on the number of
//      (query tile, kv tile) steps, which with a paged cache of unequal
//      lengths differs between sequences of equal query length);
//   3. give each sequence a contiguous run of items, ordered
//      (kv head, query tile longest first, head pair), so that the CTAs that
//      take consecutive items read the same sequence-head's K/V from L2.
// Workspace: int header[64] (header[0] = item count, header[1] = the
// scheduler's claim counter, zeroed here), then int4 items[max_items], then
// two int arrays of B entries (sorted tile counts and ranks).
// ---------------------------------------------------------------------------
constexpr int kSortBuckets = 4096;

// Key lengths come from cu_kv (ragged K/V) or, when kv_lens is given, from
// kv_lens (K/V in a paged cache).
__device__ __forceinline__ int seq_kv_len(const int32_t* cu_kv, const int32_t* kv_lens, int b) {
    return kv_lens ? kv_lens[b] : cu_kv[b + 1] - cu_kv[b];
}

__device__ __forceinline__ bool ragged_seq_ok(const int32_t* cu_q, const int32_t* cu_kv, const int32_t* kv_lens,
                                              int b, int max_sq, int max_skv, int64_t total_q,
                                              int64_t total_kv) {
    const int q0 = cu_q[b], q1 = cu_q[b + 1];
    const int lq = q1 - q0, lk = seq_kv_len(cu_kv, kv_lens, b);
    const bool kv_ok = kv_lens ? true : (cu_kv[b] >= 0 && (int64_t)cu_kv[b + 1] <= total_kv);
    return q0 >= 0 && kv_ok && lq >= 0 && lk >= 0 && lq <= max_sq && lk <= max_skv && (int64_t)q1 <= total_q;
}

// Sort key: (query tile, kv tile) steps of all query tiles of a sequence, capped.
__device__ __forceinline__ int seq_cost_key(int lq, int lk, int causal) {
    const int nqt = (lq + 127) >> 7;
    int cost = 0;
    for (int qt = 0; qt < nqt && cost < kSortBuckets - 1; ++qt) cost += prefill_n_kv(qt, lq, lk, causal);
    return min(cost, kSortBuckets - 1);
}

// Query tiles a sequence of lq queries gives the prefill kernel: none for the
// sequences of 1..short_q queries that the split-KV decode kernel takes
// (short_q = 0: the prefill kernel takes every sequence).
__device__ __forceinline__ int prefill_qtiles(int lq, int short_q) { return lq <= short_q ? 0 : (lq + 127) >> 7; }

// Exclusive prefix sum of v over the block (blockDim.x a multiple of 32, at
// most 1024); *total gets the block's sum.  warp_sums: 32 ints of shared memory.
__device__ __forceinline__ int block_exclusive_scan(int v, int* warp_sums, int* total) {
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
    int incl = v;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const int u = __shfl_up_sync(0xffffffffu, incl, off);
        if (lane >= off) incl += u;
    }
    if (lane == 31) warp_sums[wid] = incl;
    __syncthreads();
    if (wid == 0) {
        int w = (lane < (int)(blockDim.x >> 5)) ? warp_sums[lane] : 0;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const int u = __shfl_up_sync(0xffffffffu, w, off);
            if (lane >= off) w += u;
        }
        warp_sums[lane] = w;  // inclusive prefix over warps
    }
    __syncthreads();
    const int out = incl - v + (wid > 0 ? warp_sums[wid - 1] : 0);
    *total = warp_sums[(blockDim.x >> 5) - 1];
    __syncthreads();  // warp_sums may be reused after this
    return out;
}

// Padded (b, s_max, h) LSE: rows at or past a sequence's length are -inf
// ("cuDNN Frontend v1.30.0 Release Notes", "New: the FlashInfer serving path
// runs on FROST": the padded Stats buffer is seeded with -inf on the launch
// stream).  Rows inside a sequence are written by the attention kernels.
__device__ __forceinline__ void lse_padded_fill(const int32_t* __restrict__ cu_q, int B, int smax, int Hq,
                                                float* __restrict__ lse, int64_t warp_id, int64_t n_warps) {
    // warp w takes rows [w * per, (w + 1) * per) of the B * smax rows; within one
    // sequence the padded rows are contiguous, so the lanes write that span flat
    const int lane = threadIdx.x & 31;
    const int64_t rows = (int64_t)B * smax;
    const int64_t per = (rows + n_warps - 1) / n_warps;
    int64_t r = warp_id * per;
    const int64_t r_end = min(rows, r + per);
    if (r >= r_end) return;
    int b = (int)(r / smax);
    int64_t row0 = (int64_t)b * smax;  // first row of sequence b
    while (r < r_end) {
        int lq = cu_q[b + 1] - cu_q[b];
        lq = max(0, min(lq, smax));
        const int64_t seg_end = min(r_end, row0 + smax);
        for (int64_t i = max(r, row0 + lq) * Hq + lane; i < seg_end * Hq; i += 32) lse[i] = -INFINITY;
        r = seg_end;
        row0 += smax;
        ++b;
    }
}

// Block 0 builds the list (1024 threads).  Blocks 1.. (when lse is given) write
// the padded LSE rows past each sequence's length, which the prefill kernel
// never touches, so the two parts need no ordering.
__global__ void __launch_bounds__(1024) ragged_worklist_kernel(
    const int32_t* __restrict__ cu_q, const int32_t* __restrict__ cu_kv,
    const int32_t* __restrict__ kv_lens, int B, int max_sq,
    int max_skv, int64_t total_q, int64_t total_kv, int causal, int Hkv, int pairs_per_group,
    int heads_per_item, int G, int* __restrict__ header, int4* __restrict__ items,
    int* __restrict__ sorted_nqt, int* __restrict__ rank_of, int max_tiles, int short_q,
    float* __restrict__ lse, int lse_smax, int Hq) {
    if (blockIdx.x > 0) {
        if (lse != nullptr)
            lse_padded_fill(cu_q, B, lse_smax, Hq, lse, ((int64_t)(blockIdx.x - 1) * blockDim.x + threadIdx.x) >> 5,
                            ((int64_t)(gridDim.x - 1) * blockDim.x) >> 5);
        return;
    }
    __shared__ int hist[kSortBuckets];
    __shared__ int warp_sums[32];
    __shared__ int n_tiles_sh;
    const int tid = threadIdx.x;
    for (int i = tid; i < kSortBuckets; i += blockDim.x) hist[i] = 0;
    if (tid == 0) {
        n_tiles_sh = 0;
        if (cu_q[0] != 0 || (kv_lens == nullptr && cu_kv[0] != 0)) record_status(ATTN_ERR_DEVICE_INPUT);
    }
    __syncthreads();
    // 1. validate, histogram of the sort keys
    for (int b = tid; b < B; b += blockDim.x) {
        int nqt = 0, key = 0;
        if (ragged_seq_ok(cu_q, cu_kv, kv_lens, b, max_sq, max_skv, total_q, total_kv)) {
            const int lq = cu_q[b + 1] - cu_q[b];
            nqt = prefill_qtiles(lq, short_q);
            key = nqt ? seq_cost_key(lq, seq_kv_len(cu_kv, kv_lens, b), causal) : 0;
        } else {
            record_status(ATTN_ERR_DEVICE_INPUT);
        }
        atomicAdd(&hist[key], 1);
        atomicAdd(&n_tiles_sh, nqt);
    }
    __syncthreads();
    // 2. bucket starts, largest key first: thread t owns positions
    //    [t * per, (t + 1) * per) of the buckets in descending key order
    {
        const int per = (kSortBuckets + blockDim.x - 1) / blockDim.x;
        const int p0 = min(kSortBuckets, tid * per), p1 = min(kSortBuckets, p0 + per);
        int local = 0;
        for (int pos = p0; pos < p1; ++pos) local += hist[kSortBuckets - 1 - pos];
        int total;
        int run = block_exclusive_scan(local, warp_sums, &total);
        for (int pos = p0; pos < p1; ++pos) {
            const int c = kSortBuckets - 1 - pos;
            const int h = hist[c];
            hist[c] = run;
            run += h;
        }
    }
    __syncthreads();
    for (int b = tid; b < B; b += blockDim.x) {
        int nqt = 0, key = 0;
        if (ragged_seq_ok(cu_q, cu_kv, kv_lens, b, max_sq, max_skv, total_q, total_kv)) {
            const int lq = cu_q[b + 1] - cu_q[b];
            nqt = prefill_qtiles(lq, short_q);
            key = nqt ? seq_cost_key(lq, seq_kv_len(cu_kv, kv_lens, b), causal) : 0;
        }
        const int r = atomicAdd(&hist[key], 1);
        rank_of[b] = r;
        sorted_nqt[r] = nqt;
    }
    __syncthreads();
    // exclusive scan of sorted_nqt (in place), chunked over the block
    {
        const int per = (B + blockDim.x - 1) / blockDim.x;
        const int lo = min(B, tid * per), hi = min(B, lo + per);
        int local = 0;
        for (int i = lo; i < hi; ++i) local += sorted_nqt[i];
        int total;
        int run = block_exclusive_scan(local, warp_sums, &total);
        for (int i = lo; i < hi; ++i) {
            const int v = sorted_nqt[i];
            sorted_nqt[i] = run;
            run += v;
        }
    }
    __syncthreads();
    const int n_tiles = min(n_tiles_sh, max_tiles);
    if (tid == 0) {
        if (n_tiles_sh > max_tiles) record_status(ATTN_ERR_DEVICE_INPUT);
        header[0] = n_tiles * (Hkv * pairs_per_group);
        header[1] = 0;
    }
    // 3. items of each sequence, one warp per sequence: (kv head, query tile
    //    longest first, head pair)
    const int n_pairs = Hkv * pairs_per_group;
    const int lane = tid & 31, nwarps = blockDim.x >> 5;
    for (int b = tid >> 5; b < B; b += nwarps) {
        if (!ragged_seq_ok(cu_q, cu_kv, kv_lens, b, max_sq, max_skv, total_q, total_kv)) continue;
        const int lq = cu_q[b + 1] - cu_q[b], lk = seq_kv_len(cu_kv, kv_lens, b);
        const int nqt = prefill_qtiles(lq, short_q);
        if (nqt == 0) continue;
        const int tile0 = sorted_nqt[rank_of[b]];  // first tile slot of this sequence
        if (tile0 + nqt > max_tiles) continue;
        const int64_t base = (int64_t)tile0 * n_pairs;
        const int per_g = nqt * pairs_per_group;
        for (int i = lane; i < Hkv * per_g; i += 32) {
            const int g = i / per_g;
            const int rem = i - g * per_g;
            const int t = rem / pairs_per_group;
            const int pr = rem - t * pairs_per_group;
            const int qt = nqt - 1 - t;
            items[base + i] = make_int4(b, qt, g * G + pr * heads_per_item, prefill_n_kv(qt, lq, lk, causal));
        }
    }
}

// ---------------------------------------------------------------------------
// Dense BSHD work list, built on the device into the caller's workspace (the
// same {b, qtile, h0, cost} items and {count, claim counter} header as the
// ragged list, so the prefill kernel claims dense items the same way).  All
// sequences have one length, so the order is set by the query tile: groups of
// kDenseQtGroup query tiles, the group of longest tiles first (longest
// processing time first: the last items claimed are the cheapest), and inside
// a group (batch, kv head, query tile longest first, head pair), so the CTAs
// working at the same time read few (batch, kv head) K/V streams and each
// stream's causal prefix is brought from HBM once per group.  On the dense
// workload (B 8, S 4096) groups of 16 read K/V 1.5 times from HBM (1.05x the
// algorithmic bytes in all) against 2.5 times with groups of 8, at the same
// speed.  Grid-stride over the
// items; block 0 writes the header.
// ---------------------------------------------------------------------------
constexpr int kDenseQtGroup = 16;

__global__ void __launch_bounds__(256) dense_worklist_kernel(int B, int Sq, int Skv, int causal, int Hkv,
                                                             int pairs_per_group, int heads_per_item, int G,
                                                             int n_qtiles, int n_items, int* __restrict__ header,
                                                             int4* __restrict__ items) {
    if (blockIdx.x == 0 && threadIdx.x == 0) {
        header[0] = n_items;
        header[1] = 0;
    }
    const int per_t = B * Hkv * pairs_per_group;  // items per query tile
    for (int idx = blockIdx.x * blockDim.x + threadIdx.x; idx < n_items; idx += gridDim.x * blockDim.x) {
        const int grp = idx / (kDenseQtGroup * per_t);
        const int t0 = grp * kDenseQtGroup;
        const int nt = min(kDenseQtGroup, n_qtiles - t0);  // tiles in this (maybe last) group
        int rem = idx - t0 * per_t;
        const int per_bg = nt * pairs_per_group;           // items per (batch, kv head) in the group
        const int bg = rem / per_bg;
        rem -= bg * per_bg;
        const int b = bg / Hkv;
        const int g = bg - b * Hkv;
        const int ti = rem / pairs_per_group;
        const int pr = rem - ti * pairs_per_group;
        const int t = t0 + ti;
        const int qt = causal ? (n_qtiles - 1 - t) : t;
        items[idx] = make_int4(b, qt, g * G + pr * heads_per_item, prefill_n_kv(qt, Sq, Skv, causal));
    }
}

// In-place exclusive prefix of the kSortBuckets counts in hist, by a block of
// 1024 threads (thread t owns buckets [t*per, (t+1)*per)); ends synchronised.
__device__ __forceinline__ void bucket_exclusive_scan(int* hist, int* warp_sums) {
    constexpr int per = kSortBuckets / 1024;
    const int tid = threadIdx.x;
    int local = 0;
#pragma unroll
    for (int i = 0; i < per; ++i) local += hist[tid * per + i];
    int total;
    int run = block_exclusive_scan(local, warp_sums, &total);
#pragma unroll
    for (int i = 0; i < per; ++i) {
        const int h = hist[tid * per + i];
        hist[tid * per + i] = run;
        run += h;
    }
    __syncthreads();
}

// Launch order of a split MLA decode: sequence indices by cached length, longest
// first, so the clusters of the longest splits start first and the short ones
// fill in at the end (list scheduling in longest-processing-time order; the
// splits of one sequence are equal to within a page).  Counting sort over
// 4096 buckets of key = min(4095, L >> shift), the host choosing shift so that
// max_kv_len >> shift < 4096.  Ties land in any order: the order only decides
// which block runs a (sequence, split), never what it computes.  One block of
// 1024 threads.
__global__ void __launch_bounds__(1024) seq_order_kernel(const int32_t* __restrict__ kv_lens, int B, int max_kv_len,
                                                         int shift, int32_t* __restrict__ order) {
    __shared__ int hist[kSortBuckets];
    __shared__ int warp_sums[32];
    const int tid = threadIdx.x;
    // bucket 0 holds the longest sequences
    auto bucket = [&](int b) {
        const int L = max(0, min(__ldg(kv_lens + b), max_kv_len));
        return kSortBuckets - 1 - min(kSortBuckets - 1, L >> shift);
    };
    for (int i = tid; i < kSortBuckets; i += blockDim.x) hist[i] = 0;
    __syncthreads();
    for (int b = tid; b < B; b += blockDim.x) atomicAdd(&hist[bucket(b)], 1);
    __syncthreads();
    bucket_exclusive_scan(hist, warp_sums);
    for (int b = tid; b < B; b += blockDim.x) order[atomicAdd(&hist[bucket(b)], 1)] = b;
}

// ---------------------------------------------------------------------------
// Split-KV merge by LSE.  One warp per row r:
//   M = max_s lse_s;  w_s = exp(lse_s - LSE) with LSE = M + ln sum_s exp(lse_s - M)
//   O = sum_s w_s O_s.   All partials -inf -> O = 0, LSE = -inf.
// Computed in the log2 domain: exp(x) = 2^(x log2 e).
// ---------------------------------------------------------------------------
template <int DV>
struct MergeVec {
    static constexpr int VEC = (DV % 128 == 0) ? 4 : 2;  // floats per vector access
    static constexpr int NV = DV / (32 * VEC);           // vector accesses per lane
    static_assert(NV >= 1 && DV % (32 * VEC) == 0, "unsupported Dv");
};

// The merge of row r by one warp: lane holds columns VEC * (lane + 32 i) + e in
// acc[i][e]; returns the natural-log LSE of the row (-inf when every partial is).
template <int DV>
__device__ __forceinline__ float merge_row(const float* __restrict__ o_part, const float* __restrict__ lse_part,
                                           int S, int64_t R, int64_t r, int lane,
                                           float (&acc)[MergeVec<DV>::NV][MergeVec<DV>::VEC]) {
    constexpr float LOG2E = 1.4426950408889634f;
    constexpr int VEC = MergeVec<DV>::VEC, NV = MergeVec<DV>::NV;
    float M = -INFINITY;
    for (int s = lane; s < S; s += 32) M = fmaxf(M, lse_part[(int64_t)s * R + r]);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, off));
#pragma unroll
    for (int i = 0; i < NV; ++i)
#pragma unroll
        for (int e = 0; e < VEC; ++e) acc[i][e] = 0.f;
    float L = -INFINITY;
    if (M != -INFINITY) {
        float sum = 0.f;
        for (int s = lane; s < S; s += 32) sum += ex2((lse_part[(int64_t)s * R + r] - M) * LOG2E);
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, off);
        L = M + logf(sum);
        for (int s = 0; s < S; ++s) {
            const float ls = lse_part[(int64_t)s * R + r];
            if (ls == -INFINITY) continue;
            const float w = ex2((ls - L) * LOG2E);
            const float* src = o_part + ((int64_t)s * R + r) * DV;
#pragma unroll
            for (int i = 0; i < NV; ++i) {
                const int e0 = VEC * (lane + 32 * i);
                if constexpr (VEC == 4) {
                    const float4 v = __ldg(reinterpret_cast<const float4*>(src + e0));
                    acc[i][0] += w * v.x; acc[i][1] += w * v.y;
                    acc[i][2] += w * v.z; acc[i][3] += w * v.w;
                } else {
                    const float2 v = __ldg(reinterpret_cast<const float2*>(src + e0));
                    acc[i][0] += w * v.x; acc[i][1] += w * v.y;
                }
            }
        }
    }
    return L;
}

// One merged row as bf16 at dst (8-byte aligned), the lane's columns as in merge_row.
template <int DV>
__device__ __forceinline__ void store_row_bf16(__nv_bfloat16* dst, int lane,
                                               const float (&acc)[MergeVec<DV>::NV][MergeVec<DV>::VEC]) {
    constexpr int VEC = MergeVec<DV>::VEC, NV = MergeVec<DV>::NV;
#pragma unroll
    for (int i = 0; i < NV; ++i) {
        const int e0 = VEC * (lane + 32 * i);
        if constexpr (VEC == 4) {
            uint2 w;
            w.x = pack_bf16(acc[i][0], acc[i][1]);
            w.y = pack_bf16(acc[i][2], acc[i][3]);
            *reinterpret_cast<uint2*>(dst + e0) = w;
        } else {
            *reinterpret_cast<uint32_t*>(dst + e0) = pack_bf16(acc[i][0], acc[i][1]);
        }
    }
}

template <int DV>
__global__ void __launch_bounds__(256) split_merge_kernel(const float* __restrict__ o_part,
                                                          const float* __restrict__ lse_part,
                                                          int S, int64_t R,
                                                          __nv_bfloat16* __restrict__ o,
                                                          int64_t o_row_stride,
                                                          float* __restrict__ lse) {
    const int64_t r = blockIdx.x * 8 + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (r >= R) return;
    float acc[MergeVec<DV>::NV][MergeVec<DV>::VEC];
    const float L = merge_row<DV>(o_part, lse_part, S, R, r, lane, acc);
    store_row_bf16<DV>(o + r * o_row_stride, lane, acc);
    if (lse != nullptr && lane == 0) lse[r] = L;
}

// FMA-pipe exp2 self-test: y[i] = exp2_poly_pair applied to t[i].
__global__ void selftest_exp2_kernel(const float* __restrict__ t, float* __restrict__ y, int64_t n) {
    const int64_t i = 2 * (blockIdx.x * (int64_t)blockDim.x + threadIdx.x);
    if (i >= n) return;
    const float2 a = make_float2(t[i], (i + 1 < n) ? t[i + 1] : 0.f);
    const float2 r = exp2_poly_pair(a);
    y[i] = r.x;
    if (i + 1 < n) y[i + 1] = r.y;
}

// Bounded-wait self-test: waits on a barrier that nothing signals.
__global__ void selftest_wait_kernel(unsigned long long limit_ns) {
    __shared__ __align__(8) uint64_t bar;
    __shared__ int abort_flag;
    if (threadIdx.x == 0) {
        mbar_init(smem_u32(&bar), 1);
        abort_flag = 0;
        fence_barrier_init();
    }
    __syncthreads();
    if (threadIdx.x == 0) mbar_wait(smem_u32(&bar), 0, (volatile int*)&abort_flag, limit_ns);
    __syncthreads();
}

}  // namespace b2
