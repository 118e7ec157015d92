// paging.cuh -- page-table address generation shared by every paged producer
// (GQA decode, absorbed-MLA decode, prefill over a paged cache) and by the
// diagnostic that copies the coordinates out for a bit-exact host check.
//
// Logical key t of sequence b lives in physical page
// table[b * table_stride + t / page_size], at row (slot) t % page_size of that
// page ("cuDNN Frontend v1.31.0 Release Notes", "SDPA: paged KV, split-KV, and
// engine selection": a per-sequence page table over a pool of fixed-size
// pages).  A page id outside [0, num_pages) is an input error: it is recorded
// in the device status word and the key is read as zeros (a coordinate the
// tensor maps fill with zeros), never from outside the pool.
#pragma once

#include "ptx.cuh"

namespace b2 {

// Page id the table holds for logical key t of sequence b (not yet checked).
__device__ __forceinline__ int page_lookup(const int32_t* table, int64_t table_stride, int b, int t, int page_size) {
    return __ldg(table + (int64_t)b * table_stride + t / page_size);
}

// A looked-up page id checked against the pool: the id itself, or -1 (and a
// recorded ATTN_ERR_DEVICE_INPUT) when it lies outside [0, num_pages).
__device__ __forceinline__ int page_checked(int page, int64_t num_pages) {
    if (page < 0 || (int64_t)page >= num_pages) {
        record_status(ATTN_ERR_DEVICE_INPUT);
        return -1;
    }
    return page;
}

// Row of its page that logical key t occupies.
__device__ __forceinline__ int page_slot(int t, int page_size) { return t % page_size; }

// 8-row group coordinate of the prefill pool maps, which address a pool as
// consecutive groups of 8 rows: groups_per_page groups per page stride.
__device__ __forceinline__ int page_group(int page, int slot, int groups_per_page) {
    return page * groups_per_page + slot / 8;
}

// Diagnostic: for n sampled logical keys (b[i], t[i]) writes
// out[3i .. 3i+2] = (checked page or -1, slot, 8-row group or -1), computed by
// the functions above, the ones the producers use.
__global__ void page_coords_kernel(const int32_t* __restrict__ table, int64_t table_stride, int page_size,
                                   int64_t num_pages, int groups_per_page, const int32_t* __restrict__ b_idx,
                                   const int32_t* __restrict__ t_idx, int64_t n, int64_t* __restrict__ out) {
    for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x) {
        const int t = t_idx[i];
        const int page = page_checked(page_lookup(table, table_stride, b_idx[i], t, page_size), num_pages);
        const int slot = page_slot(t, page_size);
        out[3 * i + 0] = page;
        out[3 * i + 1] = slot;
        out[3 * i + 2] = page >= 0 ? page_group(page, slot, groups_per_page) : -1;
    }
}

}  // namespace b2
