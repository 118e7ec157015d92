// b2attn.cu -- the C ABI of libb2attn.so (see include/b2attn.h): host-side
// validation, TMA descriptor encoding and kernel launches.  Nothing here
// allocates device memory, reads device memory back or synchronizes, except
// attn_get_device_error(), which is a diagnostic.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>

#include "b2attn.h"
#include "ptx.cuh"
#include "prefill.cuh"
#include "aux_kernels.cuh"
#include "decode.cuh"
#include "decode_mla.cuh"
#include "paging.cuh"

namespace {

using b2::DecodeParams;
using b2::PrefillParams;

constexpr float kLog2e = 1.4426950408889634f;
constexpr int kMaxDevices = 64;

// ---------------------------------------------------------------------------
// Per-device one-time set-up: SM count and kernel shared-memory opt-ins.
// ---------------------------------------------------------------------------
struct DeviceState {
    bool ready = false;
    int num_sms = 0;
};
DeviceState g_dev[kMaxDevices];
std::mutex g_dev_mu;

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
EncodeTiledFn g_encode = nullptr;

int setup_device(int* dev_out, int* sms_out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return ATTN_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_dev_mu);
    DeviceState& st = g_dev[dev];
    if (!st.ready) {
        if (g_encode == nullptr) {
            void* fn = nullptr;
            cudaDriverEntryPointQueryResult q;
            if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) != cudaSuccess ||
                fn == nullptr)
                return ATTN_ERR_CUDA;
            g_encode = reinterpret_cast<EncodeTiledFn>(fn);
        }
        int sms = 0;
        if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return ATTN_ERR_CUDA;
        cudaError_t e = cudaSuccess;
        e = cudaFuncSetAttribute(b2::prefill_kernel<64, false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 b2::PrefillCfg<64>::SMEM);
        if (e == cudaSuccess)
            e = cudaFuncSetAttribute(b2::prefill_kernel<128, false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     b2::PrefillCfg<128>::SMEM);
        if (e == cudaSuccess)
            e = cudaFuncSetAttribute(b2::prefill_kernel<64, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     b2::PrefillCfg<64>::SMEM);
        if (e == cudaSuccess)
            e = cudaFuncSetAttribute(b2::prefill_kernel<128, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     b2::PrefillCfg<128>::SMEM);
        const void* decode_kernels[8] = {(const void*)b2::decode_gqa_kernel<64, 1>, (const void*)b2::decode_gqa_kernel<64, 2>,
                                         (const void*)b2::decode_gqa_kernel<64, 4>, (const void*)b2::decode_gqa_kernel<128, 1>,
                                         (const void*)b2::decode_gqa_kernel<128, 2>, (const void*)b2::decode_gqa_kernel<128, 4>,
                                         (const void*)b2::decode_gqa_kernel<64, 1, 6>,
                                         (const void*)b2::decode_gqa_kernel<128, 1, 6>};
        const int decode_smem[8] = {b2::DecodeCfg<64>::SMEM,     b2::DecodeCfg<64>::SMEM,  b2::DecodeCfg<64>::SMEM,
                                    b2::DecodeCfg<128>::SMEM,    b2::DecodeCfg<128>::SMEM, b2::DecodeCfg<128>::SMEM,
                                    b2::DecodeCfg<64, 6>::SMEM, b2::DecodeCfg<128, 6>::SMEM};
        for (int i = 0; i < 8 && e == cudaSuccess; ++i)
            e = cudaFuncSetAttribute(decode_kernels[i], cudaFuncAttributeMaxDynamicSharedMemorySize, decode_smem[i]);
        if (e == cudaSuccess)
            e = cudaFuncSetAttribute(b2::decode_mla_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     b2::MlaTcCfg::SMEM);
        if (e != cudaSuccess) return ATTN_ERR_CUDA;
        st.num_sms = sms;
        st.ready = true;
    }
    *dev_out = dev;
    *sms_out = st.num_sms;
    return ATTN_OK;
}

// 5D bf16 tensor map with 128-byte swizzle; strides in BYTES for dims 1..4.
int encode_5d(CUtensorMap* map, const void* base, const uint64_t dims[5], const int64_t strides_b[4],
              const uint32_t box[5]) {
    cuuint64_t gdim[5], gstr[4];
    cuuint32_t bdim[5], estr[5] = {1, 1, 1, 1, 1};
    for (int i = 0; i < 5; ++i) {
        if (dims[i] == 0 || dims[i] > (1ull << 32)) return ATTN_ERR_INVALID_ARG;
        gdim[i] = dims[i];
        bdim[i] = box[i];
    }
    for (int i = 0; i < 4; ++i) {
        if (strides_b[i] <= 0 || (strides_b[i] % 16) != 0 || strides_b[i] >= (int64_t(1) << 40)) return ATTN_ERR_INVALID_ARG;
        gstr[i] = (cuuint64_t)strides_b[i];
    }
    CUresult r = g_encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 5, const_cast<void*>(base), gdim, gstr, bdim,
                          estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                          CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? ATTN_OK : ATTN_ERR_INVALID_ARG;
}

// Token-tile map for prefill: (column in block, token, 64-column block, head, batch),
// strides in elements for token / head / batch; box = 128 tokens x all D/64 blocks.
int encode_tok_tiles(CUtensorMap* map, const void* base, int D, int64_t H, int64_t T, int64_t Bn, int64_t ts,
                     int64_t hs, int64_t bs) {
    const uint64_t dims[5] = {64, (uint64_t)(T > 0 ? T : 1), (uint64_t)(D / 64), (uint64_t)H, (uint64_t)Bn};
    const int64_t strides[4] = {ts * 2, 128, hs * 2, bs * 2};
    const uint32_t box[5] = {64, 128, (uint32_t)(D / 64), 1, 1};
    return encode_5d(map, base, dims, strides, box);
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool stride_ok(int64_t s) { return s > 0 && (s % 8) == 0; }
int64_t round_up(int64_t x, int64_t a) { return (x + a - 1) / a * a; }
int launch_status() { return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_LAUNCH; }

// Extra blocks of the work-list launch that write the padded LSE rows past
// each sequence's length: 0 unless the LSE is in the padded (b, s_max, h)
// layout; at most two 1024-thread blocks per SM.
int lse_fill_blocks(const float* lse, int lse_base, int B, int smax, int Hq, int sms) {
    if (lse == nullptr || lse_base != ATTN_LSE_PADDED_BSH) return 0;
    const int64_t want = ((int64_t)B * smax * Hq + 1023) / 1024;
    return (int)(want < (int64_t)sms * 2 ? want : (int64_t)sms * 2);
}

// A stride for a tensor-map dimension of extent 1 (never stepped along).
int64_t unit_dim_stride(int64_t a, int64_t b) { return round_up(a > b ? a : b, 8); }

int ragged_max_tiles(int B, int max_sq, int64_t total_q) {
    const int64_t by_total = total_q / 128 + B;
    const int64_t by_max = (int64_t)B * ((max_sq + 127) / 128);
    int64_t t = by_total < by_max ? by_total : by_max;
    if (t > (int64_t)1 << 30) t = (int64_t)1 << 30;
    return (int)t;
}

void pair_shape(int Hq, int Hkv, int* hpi, int* n_pairs) {
    const int G = Hq / Hkv;
    *hpi = (G % 2 == 0) ? 2 : 1;
    *n_pairs = Hq / *hpi;
}

// Ragged workspace layout: int header[64] | int4 items[max_items] | int sorted_nqt[B] | int rank_of[B]
struct RaggedWs {
    int64_t items_off, sorted_off, rank_off, total;
};
RaggedWs ragged_ws_layout(int B, int max_sq, int64_t total_q, int Hq, int Hkv) {
    int hpi, n_pairs;
    pair_shape(Hq, Hkv, &hpi, &n_pairs);
    const int64_t tiles = ragged_max_tiles(B, max_sq, total_q);
    RaggedWs w;
    w.items_off = 256;
    w.sorted_off = round_up(w.items_off + tiles * n_pairs * 16, 256);
    w.rank_off = round_up(w.sorted_off + (int64_t)B * 4, 256);
    w.total = round_up(w.rank_off + (int64_t)B * 4, 256);
    return w;
}

// ---------------------------------------------------------------------------
// Built-in scratch for attn_fwd_ragged_noalloc: holds the ragged work list for
// callers that may not allocate device memory.  Every GPU that loads this
// library keeps these bytes reserved until the process exits.
// ---------------------------------------------------------------------------
constexpr size_t kNoAllocScratchBytes = (size_t)4 << 20;  // 4 MiB
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];
void* g_noalloc_ptr[kMaxDevices] = {};
std::mutex g_noalloc_mu;

// Device address of g_noalloc_scratch on the current device, looked up once
// per device.  In host code the symbol is only a host-side stand-in, so the
// kernel must be given the address cudaGetSymbolAddress returns.
int noalloc_scratch(void** out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return ATTN_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_noalloc_mu);
    if (g_noalloc_ptr[dev] == nullptr) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) return ATTN_ERR_CUDA;
        g_noalloc_ptr[dev] = p;
    }
    *out = g_noalloc_ptr[dev];
    return ATTN_OK;
}

// Split workspace of the GQA decode, from byte `base`: per-sequence {units, L,
// q0, Lq} [B], the longest-first order [B], every block's piece [n_slots],
// arrival counters [kMergeLevels][n_slots], partial O fp32 [n_slots][rps][Dv]
// and base-2 LSE [n_slots][rps], each 256-byte aligned; n_slots = num_splits *
// pairs, the blocks of the launch.
struct SplitWs {
    int64_t seq_off, order_off, segs_off, ctr_off, part_off, lse_off, total;
};
SplitWs split_ws_layout(int64_t base, int B, int64_t pairs, int64_t rps, int Dv, int num_splits) {
    const int64_t slots = (int64_t)num_splits * pairs;
    SplitWs w;
    w.seq_off = base;
    w.order_off = round_up(w.seq_off + (int64_t)B * 16, 256);
    w.segs_off = round_up(w.order_off + (int64_t)B * 4, 256);
    w.ctr_off = round_up(w.segs_off + slots * (int64_t)sizeof(b2::DecodeSeg), 256);
    w.part_off = round_up(w.ctr_off + (int64_t)b2::kMergeLevels * slots * 4, 256);
    w.lse_off = round_up(w.part_off + slots * rps * Dv * 4, 256);
    w.total = round_up(w.lse_off + slots * rps * 4, 256);
    return w;
}

// Blocks of a split GQA decode launch (num_splits per pair), or 0 when the grid
// or the schedule's 32-bit arithmetic would overflow (the call is then
// unsupported).
int64_t split_blocks(int64_t pairs, int max_kv_len, int num_splits) {
    const int64_t n = (int64_t)num_splits * pairs;
    if (n >= ((int64_t)1 << 30) || pairs * ((int64_t)max_kv_len / 64 + 2) >= ((int64_t)1 << 30)) return 0;
    return n;
}

// Points the decode parameters at a split workspace and enqueues its schedule.
int launch_decode_schedule(DecodeParams& dp, char* wsb, const SplitWs& w, int64_t n_blocks, int max_kv_len,
                           cudaStream_t st) {
    dp.segs = reinterpret_cast<const b2::DecodeSeg*>(wsb + w.segs_off);
    dp.ctr = reinterpret_cast<int*>(wsb + w.ctr_off);
    dp.n_slots = (int)n_blocks;
    dp.o_part = reinterpret_cast<float*>(wsb + w.part_off);
    dp.lse_part = reinterpret_cast<float*>(wsb + w.lse_off);
    // sort keys: units >> shift below the bucket count
    int shift = 0;
    while (((max_kv_len / 64 + 1) >> shift) >= b2::kSortBuckets) ++shift;
    b2::decode_schedule_kernel<<<1, 1024, 0, st>>>(dp, shift, reinterpret_cast<int4*>(wsb + w.seq_off),
                                                  reinterpret_cast<int32_t*>(wsb + w.order_off),
                                                  reinterpret_cast<b2::DecodeSeg*>(wsb + w.segs_off), dp.ctr);
    return launch_status();
}

// Launches the GQA decode kernel with RT 16-row m-tiles (1, 2 or 4): grid
// (1, Hkv, B) without splits, one block per scheduled piece with them.  A
// launch of at most one block per SM gets the 6-stage ring (RT 1).
int launch_decode_gqa(const DecodeParams& dp, int D, int RT, dim3 grid, int sms, cudaStream_t st) {
    const int64_t blocks = (int64_t)grid.x * grid.y * grid.z;
    if (RT == 1 && blocks <= sms) {
        if (D == 128) b2::decode_gqa_kernel<128, 1, 6><<<grid, 160, b2::DecodeCfg<128, 6>::SMEM, st>>>(dp);
        else b2::decode_gqa_kernel<64, 1, 6><<<grid, 160, b2::DecodeCfg<64, 6>::SMEM, st>>>(dp);
        return launch_status();
    }
    if (D == 128) {
        if (RT == 1) b2::decode_gqa_kernel<128, 1><<<grid, 160, b2::DecodeCfg<128>::SMEM, st>>>(dp);
        else if (RT == 2) b2::decode_gqa_kernel<128, 2><<<grid, 160, b2::DecodeCfg<128>::SMEM, st>>>(dp);
        else b2::decode_gqa_kernel<128, 4><<<grid, 160, b2::DecodeCfg<128>::SMEM, st>>>(dp);
    } else {
        if (RT == 1) b2::decode_gqa_kernel<64, 1><<<grid, 160, b2::DecodeCfg<64>::SMEM, st>>>(dp);
        else if (RT == 2) b2::decode_gqa_kernel<64, 2><<<grid, 160, b2::DecodeCfg<64>::SMEM, st>>>(dp);
        else b2::decode_gqa_kernel<64, 4><<<grid, 160, b2::DecodeCfg<64>::SMEM, st>>>(dp);
    }
    return launch_status();
}

// GQA decode maps over a pool: (column in block, slot, 64-column block, head,
// page), one box per page: its min(page_size, 64) rows in every column block,
// landing in shared memory as [column block][rows][128 B].
int encode_decode_pool_maps(DecodeParams& dp, const void* k_pool, const void* v_pool, int Dqk, int Dv, int page_size,
                            int Hkv, int64_t num_pages, const int64_t k_pool_strides[3],
                            const int64_t v_pool_strides[3]) {
    const int box_rows = page_size < 64 ? page_size : 64;
    const uint32_t bk[5] = {64, (uint32_t)box_rows, (uint32_t)(Dqk / 64), 1, 1};
    const uint64_t dk[5] = {64, (uint64_t)page_size, (uint64_t)(Dqk / 64), (uint64_t)Hkv, (uint64_t)num_pages};
    const int64_t sk[4] = {k_pool_strides[1] * 2, 128, k_pool_strides[2] * 2, k_pool_strides[0] * 2};
    if (encode_5d(&dp.tm_k, k_pool, dk, sk, bk)) return ATTN_ERR_INVALID_ARG;
    const uint32_t bv[5] = {64, (uint32_t)box_rows, (uint32_t)(Dv / 64), 1, 1};
    const uint64_t dv[5] = {64, (uint64_t)page_size, (uint64_t)(Dv / 64), (uint64_t)Hkv, (uint64_t)num_pages};
    const int64_t sv[4] = {v_pool_strides[1] * 2, 128, v_pool_strides[2] * 2, v_pool_strides[0] * 2};
    if (encode_5d(&dp.tm_v, v_pool, dv, sv, bv)) return ATTN_ERR_INVALID_ARG;
    dp.box_rows = box_rows;
    return ATTN_OK;
}

// Ragged queries over a paged cache: the sequences of 1..qmax queries go to
// the split-KV decode kernel (G query heads x qmax tokens as the MMA rows, at
// most 64), the others to the prefill kernel.  0 when G > 64 (no routing).
int routed_qmax(int G, int max_seqlen_q) {
    if (G > 64) return 0;
    int q = 64 / G;
    if (q > 4) q = 4;
    if (q > max_seqlen_q) q = max_seqlen_q;
    return q;
}

// Launches the prefill kernel for an already-filled PrefillParams.
int launch_prefill(PrefillParams& pp, int D, int grid, cudaStream_t st) {
    if (grid <= 0) return ATTN_OK;
    const bool paged = (pp.mode == 2);
    if (D == 128) {
        if (paged)
            b2::prefill_kernel<128, true><<<grid, 320, b2::PrefillCfg<128>::SMEM, st>>>(pp);
        else
            b2::prefill_kernel<128, false><<<grid, 320, b2::PrefillCfg<128>::SMEM, st>>>(pp);
    } else {
        if (paged)
            b2::prefill_kernel<64, true><<<grid, 320, b2::PrefillCfg<64>::SMEM, st>>>(pp);
        else
            b2::prefill_kernel<64, false><<<grid, 320, b2::PrefillCfg<64>::SMEM, st>>>(pp);
    }
    return launch_status();
}

}  // namespace

extern "C" {

const char* attn_status_string(int status) {
    switch (status) {
        case ATTN_OK: return "ATTN_OK";
        case ATTN_ERR_INVALID_ARG: return "ATTN_ERR_INVALID_ARG: invalid pointer, size, stride or alignment";
        case ATTN_ERR_UNSUPPORTED: return "ATTN_ERR_UNSUPPORTED: shape declined by this library";
        case ATTN_ERR_WORKSPACE: return "ATTN_ERR_WORKSPACE: workspace missing or too small";
        case ATTN_ERR_LAUNCH: return "ATTN_ERR_LAUNCH: kernel launch failed";
        case ATTN_ERR_DEVICE_TIMEOUT: return "ATTN_ERR_DEVICE_TIMEOUT: a bounded device wait ran out";
        case ATTN_ERR_DEVICE_INPUT: return "ATTN_ERR_DEVICE_INPUT: device offsets, lengths or page ids invalid";
        case ATTN_ERR_CUDA: return "ATTN_ERR_CUDA: CUDA runtime or driver call failed";
        default: return "unknown status";
    }
}

// ------------------------------------------------------------------ dense
size_t attn_fwd_dense_workspace_size(int B, int Sq, int Hq, int Hkv) {
    if (B <= 0 || Sq < 0 || Hq <= 0 || Hkv <= 0 || Hq % Hkv != 0) return 0;
    int hpi, n_pairs;
    pair_shape(Hq, Hkv, &hpi, &n_pairs);
    // header (item count, claim counter) + one 16-byte item per (batch, query tile, head pair)
    return (size_t)round_up(256 + (int64_t)B * n_pairs * ((Sq + 127) / 128) * 16, 256);
}

int attn_fwd_dense(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Sq, int Skv,
                   int Hq, int Hkv, int Dqk, int Dv, const int64_t q_strides[3], const int64_t k_strides[3],
                   const int64_t v_strides[3], const int64_t o_strides[3], float scale, int causal,
                   void* workspace, size_t workspace_bytes, void* stream) {
    if (B < 0 || Sq < 0 || Skv < 0 || Hq <= 0 || Hkv <= 0 || Hq % Hkv != 0) return ATTN_ERR_INVALID_ARG;
    if (!std::isfinite(scale) || (causal != 0 && causal != 1)) return ATTN_ERR_INVALID_ARG;
    if (!q_strides || !k_strides || !v_strides || !o_strides) return ATTN_ERR_INVALID_ARG;
    if (Dqk != Dv || (Dqk != 64 && Dqk != 128)) return ATTN_ERR_UNSUPPORTED;
    if (B == 0 || Sq == 0) return ATTN_OK;
    if (!q || !k || !v || !o) return ATTN_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o)) return ATTN_ERR_INVALID_ARG;
    for (int i = 0; i < 3; ++i)
        if (!stride_ok(q_strides[i]) || !stride_ok(k_strides[i]) || !stride_ok(v_strides[i]) ||
            !stride_ok(o_strides[i]))
            return ATTN_ERR_INVALID_ARG;
    int hpi, n_pairs;
    pair_shape(Hq, Hkv, &hpi, &n_pairs);
    const int n_qtiles = (Sq + 127) / 128;
    const int64_t n_items = (int64_t)B * n_pairs * n_qtiles;
    if (n_items >= (int64_t)1 << 31) return ATTN_ERR_UNSUPPORTED;
    const size_t need = attn_fwd_dense_workspace_size(B, Sq, Hq, Hkv);
    if (workspace == nullptr || workspace_bytes < need) return ATTN_ERR_WORKSPACE;
    if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return ATTN_ERR_WORKSPACE;
    int dev, sms;
    if (int e = setup_device(&dev, &sms)) return e;
    const int D = Dqk;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    PrefillParams pp;
    std::memset(&pp, 0, sizeof(pp));
    if (encode_tok_tiles(&pp.tm_q, q, D, Hq, Sq, B, q_strides[1], q_strides[2], q_strides[0]) ||
        encode_tok_tiles(&pp.tm_k, k, D, Hkv, Skv, B, k_strides[1], k_strides[2], k_strides[0]) ||
        encode_tok_tiles(&pp.tm_v, v, D, Hkv, Skv, B, v_strides[1], v_strides[2], v_strides[0]))
        return ATTN_ERR_INVALID_ARG;
    const int G = Hq / Hkv;
    char* wsb = static_cast<char*>(workspace);
    int* header = reinterpret_cast<int*>(wsb);
    int4* items = reinterpret_cast<int4*>(wsb + 256);
    {
        const int64_t want = (n_items + 255) / 256;
        const int blocks = (int)(want < (int64_t)sms * 4 ? want : (int64_t)sms * 4);
        b2::dense_worklist_kernel<<<blocks, 256, 0, st>>>(B, Sq, Skv, causal, Hkv, G / hpi, hpi, G, n_qtiles,
                                                          (int)n_items, header, items);
        if (int e = launch_status()) return e;
    }
    pp.mode = 0;
    pp.B = B;
    pp.Hq = Hq;
    pp.Hkv = Hkv;
    pp.G = G;
    pp.heads_per_item = hpi;
    pp.pairs_per_group = G / hpi;
    pp.Sq = Sq;
    pp.Skv = Skv;
    pp.items = items;
    pp.header = header;
    pp.o = static_cast<__nv_bfloat16*>(o);
    pp.o_bs = o_strides[0];
    pp.o_ts = o_strides[1];
    pp.o_hs = o_strides[2];
    pp.lse = lse;
    pp.lse_layout = 0;
    pp.scale_log2 = scale * kLog2e;
    pp.causal = causal;
    const int grid = (int)(n_items < sms ? n_items : sms);
    return launch_prefill(pp, D, grid, st);
}

// ----------------------------------------------------------------- ragged
size_t attn_fwd_ragged_workspace_size(int B, int max_seqlen_q, int64_t total_q, int Hq, int Hkv) {
    if (B <= 0 || Hq <= 0 || Hkv <= 0 || Hq % Hkv != 0 || max_seqlen_q < 0 || total_q < 0) return 0;
    return (size_t)ragged_ws_layout(B, max_seqlen_q, total_q, Hq, Hkv).total;
}

}  // extern "C"

namespace {
// Host checks of attn_fwd_ragged's arguments, before anything touches the
// device.  Returns an error status, or ATTN_OK with *empty set when the call
// has nothing to compute.
int ragged_check_args(const void* q, const void* k, const void* v, const void* o, const int32_t* cu_seqlens_q,
                      const int32_t* cu_seqlens_kv, int B, int max_seqlen_q, int max_seqlen_kv, int64_t total_q,
                      int64_t total_kv, int Hq, int Hkv, int Dqk, int Dv, const int64_t q_strides[2],
                      const int64_t k_strides[2], const int64_t v_strides[2], const int64_t o_strides[2],
                      int lse_layout, float scale, int causal, bool* empty) {
    *empty = false;
    if (B < 0 || max_seqlen_q < 0 || max_seqlen_kv < 0 || total_q < 0 || total_kv < 0) return ATTN_ERR_INVALID_ARG;
    if (Hq <= 0 || Hkv <= 0 || Hq % Hkv != 0) return ATTN_ERR_INVALID_ARG;
    if (!std::isfinite(scale) || (causal != 0 && causal != 1)) return ATTN_ERR_INVALID_ARG;
    const int lse_base = lse_layout & ~ATTN_LSE_LOG2;
    if (lse_base != ATTN_LSE_PADDED_BSH && lse_base != ATTN_LSE_PACKED_TH && lse_base != ATTN_LSE_PACKED_HT)
        return ATTN_ERR_INVALID_ARG;
    if (!q_strides || !k_strides || !v_strides || !o_strides) return ATTN_ERR_INVALID_ARG;
    if (Dqk != Dv || (Dqk != 64 && Dqk != 128)) return ATTN_ERR_UNSUPPORTED;
    if (total_q >= ((int64_t)1 << 31) || total_kv >= ((int64_t)1 << 31)) return ATTN_ERR_UNSUPPORTED;
    if (B == 0 || total_q == 0 || max_seqlen_q == 0) {
        *empty = true;
        return ATTN_OK;
    }
    if (!q || !k || !v || !o || !cu_seqlens_q || !cu_seqlens_kv) return ATTN_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o)) return ATTN_ERR_INVALID_ARG;
    for (int i = 0; i < 2; ++i)
        if (!stride_ok(q_strides[i]) || !stride_ok(k_strides[i]) || !stride_ok(v_strides[i]) ||
            !stride_ok(o_strides[i]))
            return ATTN_ERR_INVALID_ARG;
    return ATTN_OK;
}
}  // namespace

extern "C" {

int attn_fwd_ragged(const void* q, const void* k, const void* v, void* o, float* lse, const int32_t* cu_seqlens_q,
                    const int32_t* cu_seqlens_kv, int B, int max_seqlen_q, int max_seqlen_kv, int64_t total_q,
                    int64_t total_kv, int Hq, int Hkv, int Dqk, int Dv, const int64_t q_strides[2],
                    const int64_t k_strides[2], const int64_t v_strides[2], const int64_t o_strides[2],
                    int lse_layout, float scale, int causal, void* workspace, size_t workspace_bytes,
                    void* stream) {
    bool empty = false;
    if (int e = ragged_check_args(q, k, v, o, cu_seqlens_q, cu_seqlens_kv, B, max_seqlen_q, max_seqlen_kv, total_q,
                                  total_kv, Hq, Hkv, Dqk, Dv, q_strides, k_strides, v_strides, o_strides, lse_layout,
                                  scale, causal, &empty))
        return e;
    if (empty) return ATTN_OK;
    const int lse_base = lse_layout & ~ATTN_LSE_LOG2;
    const size_t need = attn_fwd_ragged_workspace_size(B, max_seqlen_q, total_q, Hq, Hkv);
    if (workspace == nullptr || workspace_bytes < need) return ATTN_ERR_WORKSPACE;
    if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return ATTN_ERR_WORKSPACE;
    int dev, sms;
    if (int e = setup_device(&dev, &sms)) return e;
    const int D = Dqk;
    cudaStream_t st = static_cast<cudaStream_t>(stream);

    PrefillParams pp;
    std::memset(&pp, 0, sizeof(pp));
    if (encode_tok_tiles(&pp.tm_q, q, D, Hq, total_q, 1, q_strides[0], q_strides[1],
                         unit_dim_stride(q_strides[0] * total_q, 8)) ||
        encode_tok_tiles(&pp.tm_k, k, D, Hkv, total_kv, 1, k_strides[0], k_strides[1],
                         unit_dim_stride(k_strides[0] * total_kv, 8)) ||
        encode_tok_tiles(&pp.tm_v, v, D, Hkv, total_kv, 1, v_strides[0], v_strides[1],
                         unit_dim_stride(v_strides[0] * total_kv, 8)))
        return ATTN_ERR_INVALID_ARG;
    int hpi, n_pairs;
    pair_shape(Hq, Hkv, &hpi, &n_pairs);
    const int G = Hq / Hkv;
    const int max_tiles = ragged_max_tiles(B, max_seqlen_q, total_q);
    const RaggedWs wl = ragged_ws_layout(B, max_seqlen_q, total_q, Hq, Hkv);
    char* wsb = static_cast<char*>(workspace);
    int* header = reinterpret_cast<int*>(wsb);
    int4* items = reinterpret_cast<int4*>(wsb + wl.items_off);

    const int fill = lse_fill_blocks(lse, lse_base, B, max_seqlen_q, Hq, sms);
    b2::ragged_worklist_kernel<<<1 + fill, 1024, 0, st>>>(
        cu_seqlens_q, cu_seqlens_kv, nullptr, B, max_seqlen_q, max_seqlen_kv, total_q, total_kv, causal, Hkv, G / hpi,
        hpi, G, header, items, reinterpret_cast<int*>(wsb + wl.sorted_off), reinterpret_cast<int*>(wsb + wl.rank_off),
        max_tiles, 0, fill ? lse : nullptr, max_seqlen_q, Hq);
    if (int e = launch_status()) return e;
    pp.mode = 1;
    pp.B = B;
    pp.Hq = Hq;
    pp.Hkv = Hkv;
    pp.G = Hq / Hkv;
    pp.heads_per_item = hpi;
    pp.pairs_per_group = G / hpi;
    pp.cu_q = cu_seqlens_q;
    pp.cu_kv = cu_seqlens_kv;
    pp.items = items;
    pp.header = header;
    pp.o = static_cast<__nv_bfloat16*>(o);
    pp.o_bs = 0;
    pp.o_ts = o_strides[0];
    pp.o_hs = o_strides[1];
    pp.lse = lse;
    pp.lse_layout = (lse_base == ATTN_LSE_PADDED_BSH) ? 1 : (lse_base == ATTN_LSE_PACKED_TH) ? 2 : 3;
    pp.lse_smax = max_seqlen_q;
    pp.lse_hs = total_q;
    pp.lse_log2 = (lse_layout & ATTN_LSE_LOG2) ? 1 : 0;
    pp.scale_log2 = scale * kLog2e;
    pp.causal = causal;
    const int64_t items_max = (int64_t)max_tiles * n_pairs;
    const int grid = (int)(items_max < sms ? items_max : sms);
    return launch_prefill(pp, D, grid, st);
}

// --------------------------------------------------- ragged, no allocation
int attn_fwd_ragged_noalloc(const void* q, const void* k, const void* v, void* o, float* lse,
                            const int32_t* cu_seqlens_q, const int32_t* cu_seqlens_kv, int B, int max_seqlen_q,
                            int max_seqlen_kv, int64_t total_q, int64_t total_kv, int Hq, int Hkv, int Dqk,
                            int Dv, const int64_t q_strides[2], const int64_t k_strides[2],
                            const int64_t v_strides[2], const int64_t o_strides[2], int lse_layout, float scale,
                            int causal, void* stream) {
    // every host check and the empty-problem return come before the first
    // device call (the scratch address lookup), so an invalid or empty call
    // never does that lookup
    bool empty = false;
    if (int e = ragged_check_args(q, k, v, o, cu_seqlens_q, cu_seqlens_kv, B, max_seqlen_q, max_seqlen_kv, total_q,
                                  total_kv, Hq, Hkv, Dqk, Dv, q_strides, k_strides, v_strides, o_strides, lse_layout,
                                  scale, causal, &empty))
        return e;
    if (empty) return ATTN_OK;
    const size_t need = attn_fwd_ragged_workspace_size(B, max_seqlen_q, total_q, Hq, Hkv);
    if (need > kNoAllocScratchBytes) return ATTN_ERR_WORKSPACE;  // work list would not fit 4 MiB
    void* scratch = nullptr;
    if (int e = noalloc_scratch(&scratch)) return e;
    return attn_fwd_ragged(q, k, v, o, lse, cu_seqlens_q, cu_seqlens_kv, B, max_seqlen_q, max_seqlen_kv, total_q,
                           total_kv, Hq, Hkv, Dqk, Dv, q_strides, k_strides, v_strides, o_strides, lse_layout,
                           scale, causal, scratch, kNoAllocScratchBytes, stream);
}

size_t attn_fwd_ragged_noalloc_max_scratch(void) { return kNoAllocScratchBytes; }

// ------------------------------------------------ paged prefill (chunked)
}  // extern "C"

namespace {
// Paged-prefill workspace: the ragged work list, then (routed short rows with
// splits) the split workspace of their decode kernel.
struct PagedPrefillWs {
    RaggedWs rw;
    int qmax;
    SplitWs sw;
    int64_t total;
};
PagedPrefillWs paged_prefill_ws_layout(int B, int max_sq, int64_t total_q, int Hq, int Hkv, int D, int num_splits) {
    PagedPrefillWs w;
    w.rw = ragged_ws_layout(B, max_sq, total_q, Hq, Hkv);
    w.qmax = routed_qmax(Hq / Hkv, max_sq);
    w.sw = SplitWs{};
    w.total = w.rw.total;
    if (w.qmax > 0 && num_splits > 1) {
        w.sw = split_ws_layout(w.rw.total, B, (int64_t)B * Hkv, (int64_t)(Hq / Hkv) * w.qmax, D, num_splits);
        w.total = w.sw.total;
    }
    return w;
}
}  // namespace

extern "C" {

size_t attn_fwd_paged_prefill_workspace_size(int B, int max_seqlen_q, int64_t total_q, int Hq, int Hkv, int D,
                                             int num_splits) {
    if (B <= 0 || Hq <= 0 || Hkv <= 0 || Hq % Hkv != 0 || max_seqlen_q < 0 || total_q < 0 || D <= 0 ||
        num_splits < 1)
        return 0;
    return (size_t)paged_prefill_ws_layout(B, max_seqlen_q, total_q, Hq, Hkv, D, num_splits).total;
}

int attn_fwd_paged_prefill(const void* q, const void* k_pool, const void* v_pool, void* o, float* lse,
                           const int32_t* cu_seqlens_q, const int32_t* page_table, int64_t page_table_stride,
                           const int32_t* kv_lens, int B, int max_seqlen_q, int64_t total_q, int Hq, int Hkv,
                           int D, int page_size, int64_t num_pages, int max_kv_len, const int64_t q_strides[2],
                           const int64_t o_strides[2], const int64_t k_pool_strides[3],
                           const int64_t v_pool_strides[3], int lse_layout, float scale, int causal, int num_splits,
                           void* workspace, size_t workspace_bytes, void* stream) {
    return attn_fwd_paged_prefill_kv_tables(q, k_pool, v_pool, o, lse, cu_seqlens_q, page_table, page_table_stride,
                                            page_table, page_table_stride, kv_lens, B, max_seqlen_q, total_q, Hq,
                                            Hkv, D, page_size, num_pages, max_kv_len, q_strides, o_strides,
                                            k_pool_strides, v_pool_strides, lse_layout, scale, causal, num_splits,
                                            workspace, workspace_bytes, stream);
}

int attn_fwd_paged_prefill_kv_tables(const void* q, const void* k_pool, const void* v_pool, void* o, float* lse,
                                     const int32_t* cu_seqlens_q, const int32_t* k_page_table,
                                     int64_t k_page_table_stride, const int32_t* v_page_table,
                                     int64_t v_page_table_stride, const int32_t* kv_lens, int B, int max_seqlen_q,
                                     int64_t total_q, int Hq, int Hkv, int D, int page_size, int64_t num_pages,
                                     int max_kv_len, const int64_t q_strides[2], const int64_t o_strides[2],
                                     const int64_t k_pool_strides[3], const int64_t v_pool_strides[3],
                                     int lse_layout, float scale, int causal, int num_splits, void* workspace,
                                     size_t workspace_bytes, void* stream) {
    if (B < 0 || max_seqlen_q < 0 || total_q < 0 || max_kv_len < 0 || num_pages < 0) return ATTN_ERR_INVALID_ARG;
    if (Hq <= 0 || Hkv <= 0 || Hq % Hkv != 0) return ATTN_ERR_INVALID_ARG;
    if (!std::isfinite(scale) || (causal != 0 && causal != 1)) return ATTN_ERR_INVALID_ARG;
    if (num_splits < 1 || num_splits > 4096) return ATTN_ERR_INVALID_ARG;
    const int lse_base = lse_layout & ~ATTN_LSE_LOG2;
    if (lse_base != ATTN_LSE_PADDED_BSH && lse_base != ATTN_LSE_PACKED_TH && lse_base != ATTN_LSE_PACKED_HT)
        return ATTN_ERR_INVALID_ARG;
    if (!q_strides || !o_strides || !k_pool_strides || !v_pool_strides) return ATTN_ERR_INVALID_ARG;
    if (page_size <= 0 || k_page_table_stride < 0 || v_page_table_stride < 0) return ATTN_ERR_INVALID_ARG;
    if (D != 64 && D != 128) return ATTN_ERR_UNSUPPORTED;
    // a page box of min(page_size, 128) rows: whole 8-row groups that tile a 128-key tile
    if (!(page_size % 128 == 0 || (128 % page_size == 0 && page_size >= 8))) return ATTN_ERR_UNSUPPORTED;
    if (total_q >= ((int64_t)1 << 31)) return ATTN_ERR_UNSUPPORTED;
    if (B > 65535 || Hkv > 65535) return ATTN_ERR_UNSUPPORTED;
    if (B == 0 || total_q == 0 || max_seqlen_q == 0) return ATTN_OK;
    if (!q || !k_pool || !v_pool || !o || !cu_seqlens_q || !k_page_table || !v_page_table || !kv_lens)
        return ATTN_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k_pool) || !aligned16(v_pool) || !aligned16(o)) return ATTN_ERR_INVALID_ARG;
    if (num_pages == 0) return ATTN_ERR_INVALID_ARG;
    const int64_t row_pages = ((int64_t)max_kv_len + page_size - 1) / page_size;
    if (B > 1 && (k_page_table_stride < row_pages || v_page_table_stride < row_pages)) return ATTN_ERR_INVALID_ARG;
    for (int i = 0; i < 2; ++i)
        if (!stride_ok(q_strides[i]) || !stride_ok(o_strides[i])) return ATTN_ERR_INVALID_ARG;
    for (int i = 0; i < 3; ++i)
        if (!stride_ok(k_pool_strides[i]) || !stride_ok(v_pool_strides[i])) return ATTN_ERR_INVALID_ARG;
    // the maps address a page as whole 8-row groups: page stride = groups_per_page x 8 rows,
    // the same for K and V
    const int64_t gk = k_pool_strides[0] / (8 * k_pool_strides[1]);
    const int64_t gv = v_pool_strides[0] / (8 * v_pool_strides[1]);
    if (k_pool_strides[0] % (8 * k_pool_strides[1]) != 0 || v_pool_strides[0] % (8 * v_pool_strides[1]) != 0 ||
        gk != gv || gk < page_size / 8)
        return ATTN_ERR_UNSUPPORTED;
    if ((int64_t)num_pages * gk >= ((int64_t)1 << 31)) return ATTN_ERR_UNSUPPORTED;
    const PagedPrefillWs wl = paged_prefill_ws_layout(B, max_seqlen_q, total_q, Hq, Hkv, D, num_splits);
    if (workspace == nullptr || workspace_bytes < (size_t)wl.total) return ATTN_ERR_WORKSPACE;
    if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return ATTN_ERR_WORKSPACE;
    int dev, sms;
    if (int e = setup_device(&dev, &sms)) return e;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const int R = page_size < 128 ? page_size : 128;
    const int G = Hq / Hkv;
    const int qmax = wl.qmax;
    char* wsb = static_cast<char*>(workspace);

    const int dev_lse_layout = (lse_base == ATTN_LSE_PADDED_BSH) ? 1 : (lse_base == ATTN_LSE_PACKED_TH) ? 2 : 3;

    // every tensor map is encoded (and may fail) before the first launch, so a host-side
    // error leaves nothing enqueued
    PrefillParams pp;
    std::memset(&pp, 0, sizeof(pp));
    if (encode_tok_tiles(&pp.tm_q, q, D, Hq, total_q, 1, q_strides[0], q_strides[1],
                         unit_dim_stride(q_strides[0] * total_q, 8)))
        return ATTN_ERR_INVALID_ARG;
    {
        // (column in block, row in 8-row group, 64-column block, 8-row group of the pool, head)
        const uint64_t dims[5] = {64, 8, (uint64_t)(D / 64), (uint64_t)(num_pages * gk), (uint64_t)Hkv};
        const uint32_t box[5] = {64, 8, (uint32_t)(D / 64), (uint32_t)(R / 8), 1};
        const int64_t sk[4] = {k_pool_strides[1] * 2, 128, 8 * k_pool_strides[1] * 2, k_pool_strides[2] * 2};
        const int64_t sv[4] = {v_pool_strides[1] * 2, 128, 8 * v_pool_strides[1] * 2, v_pool_strides[2] * 2};
        if (encode_5d(&pp.tm_k, k_pool, dims, sk, box) || encode_5d(&pp.tm_v, v_pool, dims, sv, box))
            return ATTN_ERR_INVALID_ARG;
    }
    DecodeParams dp;
    std::memset(&dp, 0, sizeof(dp));
    // short rows: G * qmax query rows in RT m16 tiles; with splits, one block per piece
    int RT = 1;
    int64_t n_split_blocks = 0;
    const int64_t dec_pairs = (int64_t)B * Hkv;
    if (qmax > 0) {
        if (int e = encode_decode_pool_maps(dp, k_pool, v_pool, D, D, page_size, Hkv, num_pages, k_pool_strides,
                                            v_pool_strides))
            return e;
        RT = (G * qmax + 15) / 16;
        if (RT == 3) RT = 4;
        if (num_splits > 1) {
            n_split_blocks = split_blocks(dec_pairs, max_kv_len, num_splits);
            if (n_split_blocks == 0) return ATTN_ERR_UNSUPPORTED;
        }
    }

    // ---- sequences of 1..qmax queries (decode, multi-token decode): split-KV decode kernel
    if (qmax > 0) {
        dp.q = static_cast<const __nv_bfloat16*>(q);
        dp.q_bs = q_strides[0];
        dp.q_hs = q_strides[1];
        dp.page_table = k_page_table;
        dp.pt_stride = k_page_table_stride;
        dp.v_page_table = v_page_table;
        dp.v_pt_stride = v_page_table_stride;
        dp.kv_lens = kv_lens;
        dp.cu_q = cu_seqlens_q;
        dp.total_q = total_q;
        dp.qmax = qmax;
        dp.causal = causal;
        dp.B = B;
        dp.Hq = Hq;
        dp.Hkv = Hkv;
        dp.G = G;
        dp.page_size = page_size;
        dp.num_pages = num_pages;
        dp.max_kv_len = max_kv_len;
        dp.num_splits = num_splits;
        dp.scale_log2 = scale * kLog2e;
        dp.o = static_cast<__nv_bfloat16*>(o);
        dp.o_bs = o_strides[0];
        dp.o_hs = o_strides[1];
        dp.lse = lse;
        dp.lse_layout = dev_lse_layout;
        dp.lse_smax = max_seqlen_q;
        dp.lse_hs = total_q;
        dp.lse_log2 = (lse_layout & ATTN_LSE_LOG2) ? 1 : 0;
        if (num_splits > 1) {
            if (int e = launch_decode_schedule(dp, wsb, wl.sw, n_split_blocks, max_kv_len, st)) return e;
            if (int e = launch_decode_gqa(dp, D, RT, dim3((unsigned)n_split_blocks, 1, 1), sms, st)) return e;
        } else {
            if (int e = launch_decode_gqa(dp, D, RT, dim3(1, Hkv, B), sms, st)) return e;
        }
    }

    // ---- the other sequences: tcgen05 prefill kernel over page boxes (tensor maps
    // encoded above, before anything was enqueued)
    int hpi, n_pairs;
    pair_shape(Hq, Hkv, &hpi, &n_pairs);
    const int max_tiles = ragged_max_tiles(B, max_seqlen_q, total_q);
    int* header = reinterpret_cast<int*>(wsb);
    int4* items = reinterpret_cast<int4*>(wsb + wl.rw.items_off);
    // blocks 1.. also write the padded LSE rows past each length (the short rows'
    // merge and the prefill kernel write the rows inside)
    const int fill = lse_fill_blocks(lse, lse_base, B, max_seqlen_q, Hq, sms);
    b2::ragged_worklist_kernel<<<1 + fill, 1024, 0, st>>>(
        cu_seqlens_q, nullptr, kv_lens, B, max_seqlen_q, max_kv_len, total_q, 0, causal, Hkv, G / hpi, hpi, G,
        header, items, reinterpret_cast<int*>(wsb + wl.rw.sorted_off), reinterpret_cast<int*>(wsb + wl.rw.rank_off),
        max_tiles, qmax, fill ? lse : nullptr, max_seqlen_q, Hq);
    if (int e = launch_status()) return e;
    // the work-list kernel also validates every sequence; with all of them short
    // (max_seqlen_q <= qmax) its list is empty and the prefill kernel has nothing to do
    if (qmax > 0 && max_seqlen_q <= qmax) return ATTN_OK;
    pp.mode = 2;
    pp.B = B;
    pp.Hq = Hq;
    pp.Hkv = Hkv;
    pp.G = G;
    pp.heads_per_item = hpi;
    pp.pairs_per_group = G / hpi;
    pp.cu_q = cu_seqlens_q;
    pp.items = items;
    pp.header = header;
    pp.o = static_cast<__nv_bfloat16*>(o);
    pp.o_ts = o_strides[0];
    pp.o_hs = o_strides[1];
    pp.lse = lse;
    pp.lse_layout = (lse_base == ATTN_LSE_PADDED_BSH) ? 1 : (lse_base == ATTN_LSE_PACKED_TH) ? 2 : 3;
    pp.lse_smax = max_seqlen_q;
    pp.lse_hs = total_q;
    pp.lse_log2 = (lse_layout & ATTN_LSE_LOG2) ? 1 : 0;
    pp.scale_log2 = scale * kLog2e;
    pp.causal = causal;
    pp.kv_lens = kv_lens;
    pp.page_table = k_page_table;
    pp.pt_stride = k_page_table_stride;
    pp.v_page_table = v_page_table;
    pp.v_pt_stride = v_page_table_stride;
    pp.page_size = page_size;
    pp.box_rows = R;
    pp.num_pages = num_pages;
    pp.groups_per_page = (int)gk;
    pp.n_groups = (int)(num_pages * gk);
    pp.max_kv_len = max_kv_len;
    const int64_t items_max = (int64_t)max_tiles * n_pairs;
    const int grid = (int)(items_max < sms ? items_max : sms);
    return launch_prefill(pp, D, grid, st);
}

// ------------------------------------------------------------------ paged
size_t attn_fwd_paged_workspace_size(int B, int Hq, int Dv, int num_splits) {
    if (B <= 0 || Hq <= 0 || Dv <= 0 || num_splits <= 1) return 0;
    const int64_t R = (int64_t)B * Hq;
    if (Dv == 512) {
        // MLA: partial O, partial LSE, launch order of the sequences
        return (size_t)(round_up(R * num_splits * Dv * 4, 256) + round_up(R * num_splits * 4, 256) +
                        round_up((int64_t)B * 4, 256));
    }
    // GQA: sized with B * Hq pairs of one row, it covers every Hkv (pairs * G rows = B * Hq)
    return (size_t)split_ws_layout(0, B, R, 1, Dv, num_splits).total;
}

int attn_paged_suggest_splits(int B, int Hq, int Hkv, int Dqk, int Dv, int max_kv_len, int page_size,
                              int num_sms) {
    if (B <= 0 || Hq <= 0 || Hkv <= 0 || max_kv_len <= 0 || page_size <= 0 || num_sms <= 0) return 1;
    const bool mla = (Dqk == 576);
    int64_t s_balance;
    double max_overhead;
    if (mla) {
        // a cluster of two CTAs (one per SM) per (sequence, split, 128-head group): about two and
        // a half waves of work units over the SM pairs (the launch order puts the longest
        // sequences first, so few waves suffice; on the 64-sequence MLA workload 3 splits measured
        // 2716 GB/s against 2650-2690 with 4 and 2678 with 2), partial traffic up to ~10% of the
        // KV bytes
        const int64_t units_per_split = (int64_t)B * ((Hq + 127) / 128);
        const int64_t pairs = num_sms / 2 > 0 ? num_sms / 2 : 1;
        s_balance = (5 * pairs + 2 * units_per_split - 1) / (2 * units_per_split);
        max_overhead = 0.10;
    } else {
        const int64_t ctas_per_split = (int64_t)Hkv * B;
        const int64_t slots = (int64_t)num_sms * 2;
        if (ctas_per_split <= slots) {
            // the batch fits one wave of blocks (two per SM) without splits: the count that
            // gives the most blocks still in one wave (b 32 / Hkv 4 / 4096 keys, page 16:
            // 2 splits 58.4 us against 85.1 with 1 and 81.9 with 3; b 8: 8 splits 29.3 us
            // against 41.5 with 3; b 64: 1 split 91.7 us against 112 with 2). With whole-page
            // boxes of 64 rows and short caches, one block per SM with the deep ring wins
            // instead (b 32, page 64: 1 split 49.7 us against 55.7 with 2; at 16384 keys 2
            // splits win, 167 against 176 us)
            int64_t s = slots / ctas_per_split;
            if (page_size >= 64 && max_kv_len <= 8192 && ctas_per_split <= num_sms) s = num_sms / ctas_per_split;
            const int64_t units = ((int64_t)max_kv_len + 63) / 64;
            if (s > units) s = units;
            if (s > 512) s = 512;
            return (int)(s < 1 ? 1 : s);
        }
        // about four waves of CTAs over the two resident CTAs per SM (longest sequences
        // first; measured best on the 128-sequence GQA workload against 8 and 16)
        s_balance = (4 * slots + ctas_per_split - 1) / ctas_per_split;
        max_overhead = 0.05;
    }
    // the fp32 partials (written + read) stay under max_overhead of the KV bytes streamed
    const double kv_bytes = 0.5 * (double)max_kv_len * Hkv * (double)(mla ? Dqk : Dqk + Dv) * 2.0;
    const double part_bytes_per_split = (double)Hq * Dv * 8.0;
    int64_t s_traffic = (int64_t)(max_overhead * kv_bytes / part_bytes_per_split);
    int64_t s = s_balance < s_traffic ? s_balance : s_traffic;
    const int64_t max_pages = (max_kv_len + page_size - 1) / page_size;
    if (s > max_pages) s = max_pages;
    if (s > 64) s = 64;
    if (s < 1) s = 1;
    return (int)s;
}

int attn_fwd_paged(const void* q, const void* k_pool, const void* v_pool, void* o, float* lse,
                   const int32_t* page_table, int64_t page_table_stride, const int32_t* kv_lens, int B, int Hq,
                   int Hkv, int Dqk, int Dv, int page_size, int64_t num_pages, int max_kv_len,
                   const int64_t q_strides[2], const int64_t o_strides[2], const int64_t k_pool_strides[3],
                   const int64_t v_pool_strides[3], float scale, int num_splits, void* workspace,
                   size_t workspace_bytes, void* stream) {
    return attn_fwd_paged_kv_tables(q, k_pool, v_pool, o, lse, page_table, page_table_stride, page_table,
                                    page_table_stride, kv_lens, B, Hq, Hkv, Dqk, Dv, page_size, num_pages,
                                    max_kv_len, q_strides, o_strides, k_pool_strides, v_pool_strides, scale,
                                    num_splits, workspace, workspace_bytes, stream);
}

int attn_fwd_paged_kv_tables(const void* q, const void* k_pool, const void* v_pool, void* o, float* lse,
                             const int32_t* k_page_table, int64_t k_page_table_stride,
                             const int32_t* v_page_table, int64_t v_page_table_stride, const int32_t* kv_lens,
                             int B, int Hq, int Hkv, int Dqk, int Dv, int page_size, int64_t num_pages,
                             int max_kv_len, const int64_t q_strides[2], const int64_t o_strides[2],
                             const int64_t k_pool_strides[3], const int64_t v_pool_strides[3], float scale,
                             int num_splits, void* workspace, size_t workspace_bytes, void* stream) {
    if (B < 0 || Hq <= 0 || Hkv <= 0 || Hq % Hkv != 0 || max_kv_len < 0 || num_pages < 0) return ATTN_ERR_INVALID_ARG;
    if (!std::isfinite(scale) || num_splits < 1 || num_splits > 4096) return ATTN_ERR_INVALID_ARG;
    if (!q_strides || !o_strides || !k_pool_strides || !v_pool_strides) return ATTN_ERR_INVALID_ARG;
    if (page_size <= 0 || k_page_table_stride < 0 || v_page_table_stride < 0) return ATTN_ERR_INVALID_ARG;
    const int G = Hq / Hkv;
    const bool mla = (Dqk == 576 && Dv == 512);
    const bool gqa = (Dqk == Dv && (Dqk == 64 || Dqk == 128) && G <= 16);
    if (!mla && !gqa) return ATTN_ERR_UNSUPPORTED;
    if (mla && Hkv != 1) return ATTN_ERR_UNSUPPORTED;
    // MLA: a page box of min(page_size, 64) rows is the N of the score MMAs (16, 32 or 64)
    if (mla && !(page_size % 64 == 0 || page_size == 32 || page_size == 16)) return ATTN_ERR_UNSUPPORTED;
    // a 64-key box is whole pages, or a page is whole boxes
    if (!(page_size % 64 == 0 || (64 % page_size == 0 && page_size >= 8))) return ATTN_ERR_UNSUPPORTED;
    if (B > 65535 || Hkv > 65535 || num_splits > 65535) return ATTN_ERR_UNSUPPORTED;
    if (B == 0) return ATTN_OK;
    if (!q || !k_pool || !v_pool || !o || !k_page_table || !v_page_table || !kv_lens) return ATTN_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k_pool) || !aligned16(v_pool) || !aligned16(o)) return ATTN_ERR_INVALID_ARG;
    if (num_pages == 0) return ATTN_ERR_INVALID_ARG;
    // every row of each page table must cover max_kv_len keys
    const int64_t row_pages = ((int64_t)max_kv_len + page_size - 1) / page_size;
    if (B > 1 && (k_page_table_stride < row_pages || v_page_table_stride < row_pages)) return ATTN_ERR_INVALID_ARG;
    for (int i = 0; i < 2; ++i)
        if (!stride_ok(q_strides[i]) || !stride_ok(o_strides[i])) return ATTN_ERR_INVALID_ARG;
    for (int i = 0; i < 3; ++i)
        if (!stride_ok(k_pool_strides[i]) || !stride_ok(v_pool_strides[i])) return ATTN_ERR_INVALID_ARG;
    if (num_splits > 1) {
        // the MLA merge writes O row r = b*Hq + h at o + r*o_strides[1]: batch-major rows
        if (mla && o_strides[0] != (int64_t)Hq * o_strides[1]) return ATTN_ERR_UNSUPPORTED;
        const size_t need = attn_fwd_paged_workspace_size(B, Hq, Dv, num_splits);
        if (workspace == nullptr || workspace_bytes < need) return ATTN_ERR_WORKSPACE;
        if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return ATTN_ERR_WORKSPACE;
    }
    int dev, sms;
    if (int e = setup_device(&dev, &sms)) return e;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    // MLA: one cluster of two CTAs (score CTA, value CTA) per (b, split, group of 128 heads)
    const int64_t mla_units = (int64_t)B * num_splits * ((Hq + 127) / 128);
    if (mla && 2 * mla_units > 0x7fffffff) return ATTN_ERR_UNSUPPORTED;
    // GQA with splits: one block per scheduled piece
    int64_t n_split_blocks = 0;
    if (!mla && num_splits > 1) {
        n_split_blocks = split_blocks((int64_t)B * Hkv, max_kv_len, num_splits);
        if (n_split_blocks == 0) return ATTN_ERR_UNSUPPORTED;
    }

    DecodeParams dp;
    std::memset(&dp, 0, sizeof(dp));
    // rows per TMA box: one page, at most 64 keys
    const int box_rows = page_size < 64 ? page_size : 64;
    if (mla) {
        // K: (column in block, row in 8-row group, 64-column block, 8-row group of the pool, head),
        // one box per page box of R rows and all 9 column blocks, landing group-major; the pool's
        // page stride must be a whole number of 8-row groups
        const int64_t gk = k_pool_strides[0] / (8 * k_pool_strides[1]);
        if (k_pool_strides[0] % (8 * k_pool_strides[1]) != 0 || gk < page_size / 8 ||
            (int64_t)num_pages * gk >= ((int64_t)1 << 31))
            return ATTN_ERR_UNSUPPORTED;
        const uint64_t dk[5] = {64, 8, 9, (uint64_t)(num_pages * gk), (uint64_t)Hkv};
        const int64_t sk[4] = {k_pool_strides[1] * 2, 128, 8 * k_pool_strides[1] * 2, k_pool_strides[2] * 2};
        const uint32_t bk[5] = {64, 8, 9, (uint32_t)(box_rows / 8), 1};
        if (encode_5d(&dp.tm_k, k_pool, dk, sk, bk)) return ATTN_ERR_INVALID_ARG;
        dp.groups_per_page = (int)gk;
        // V: (column in block, row in page, 64-column block, head, page), 8 value blocks per load
        const uint64_t dv[5] = {64, (uint64_t)page_size, 8, (uint64_t)Hkv, (uint64_t)num_pages};
        const int64_t sv[4] = {v_pool_strides[1] * 2, 128, v_pool_strides[2] * 2, v_pool_strides[0] * 2};
        const uint32_t bv[5] = {64, (uint32_t)box_rows, (uint32_t)b2::MlaTcCfg::VB, 1, 1};
        if (encode_5d(&dp.tm_v, v_pool, dv, sv, bv)) return ATTN_ERR_INVALID_ARG;
    } else {
        if (int e = encode_decode_pool_maps(dp, k_pool, v_pool, Dqk, Dv, page_size, Hkv, num_pages, k_pool_strides,
                                            v_pool_strides))
            return e;
    }
    dp.q = static_cast<const __nv_bfloat16*>(q);
    dp.q_bs = q_strides[0];
    dp.q_hs = q_strides[1];
    dp.page_table = k_page_table;
    dp.pt_stride = k_page_table_stride;
    dp.v_page_table = v_page_table;
    dp.v_pt_stride = v_page_table_stride;
    dp.kv_lens = kv_lens;
    dp.qmax = 1;  // one query token per sequence (cu_q stays null)
    dp.B = B;
    dp.Hq = Hq;
    dp.Hkv = Hkv;
    dp.G = G;
    dp.page_size = page_size;
    dp.box_rows = box_rows;
    dp.num_pages = num_pages;
    dp.max_kv_len = max_kv_len;
    dp.num_splits = num_splits;
    dp.scale_log2 = scale * kLog2e;
    dp.o = static_cast<__nv_bfloat16*>(o);
    dp.o_bs = o_strides[0];
    dp.o_hs = o_strides[1];
    dp.lse = lse;
    const int64_t R = (int64_t)B * Hq;
    char* wsb = static_cast<char*>(workspace);
    if (mla) {
        if (num_splits > 1) {
            dp.o_part = reinterpret_cast<float*>(wsb);
            dp.lse_part = reinterpret_cast<float*>(wsb + round_up(R * num_splits * Dv * 4, 256));
            // sequences longest first: the clusters of the longest splits start first
            int32_t* order = reinterpret_cast<int32_t*>(wsb + round_up(R * num_splits * Dv * 4, 256) +
                                                        round_up(R * num_splits * 4, 256));
            int shift = 0;
            while ((max_kv_len >> shift) >= 4096) ++shift;
            b2::seq_order_kernel<<<1, 1024, 0, st>>>(kv_lens, B, max_kv_len, shift, order);
            if (int e = launch_status()) return e;
            dp.order = order;
        }
        cudaLaunchConfig_t cfg;
        std::memset(&cfg, 0, sizeof(cfg));
        cfg.gridDim = dim3((unsigned)(2 * mla_units), 1, 1);
        cfg.blockDim = dim3(b2::MlaTcCfg::THREADS, 1, 1);
        cfg.dynamicSmemBytes = b2::MlaTcCfg::SMEM;
        cfg.stream = st;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = 2;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        if (cudaLaunchKernelEx(&cfg, b2::decode_mla_tc_kernel, dp) != cudaSuccess) return ATTN_ERR_LAUNCH;
        if (int e = launch_status()) return e;
        if (num_splits > 1)
            return attn_split_merge(dp.o_part, dp.lse_part, num_splits, R, Dv, o, o_strides[1], lse, stream);
        return ATTN_OK;
    }
    // GQA: the G <= 16 query heads of a KV head fill one m16 tile
    if (num_splits > 1) {
        const SplitWs sw = split_ws_layout(0, B, R, 1, Dv, num_splits);
        if (int e = launch_decode_schedule(dp, wsb, sw, n_split_blocks, max_kv_len, st)) return e;
        return launch_decode_gqa(dp, Dqk, 1, dim3((unsigned)n_split_blocks, 1, 1), sms, st);
    }
    return launch_decode_gqa(dp, Dqk, 1, dim3(1, Hkv, B), sms, st);
}

// ------------------------------------------------------------------ merge
int attn_split_merge(const float* o_part, const float* lse_part, int num_splits, int64_t R, int Dv, void* o,
                     int64_t o_row_stride, float* lse, void* stream) {
    if (num_splits < 1 || R < 0 || o_row_stride < Dv) return ATTN_ERR_INVALID_ARG;
    if (Dv != 64 && Dv != 128 && Dv != 512) return ATTN_ERR_UNSUPPORTED;
    if (R == 0) return ATTN_OK;
    if (!o_part || !lse_part || !o) return ATTN_ERR_INVALID_ARG;
    if (!aligned16(o_part) || (reinterpret_cast<uintptr_t>(o) & 7u) || (o_row_stride % 4) != 0)
        return ATTN_ERR_INVALID_ARG;
    int dev, sms;
    if (int e = setup_device(&dev, &sms)) return e;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const int64_t blocks = (R + 7) / 8;
    if (blocks > 0x7fffffff) return ATTN_ERR_UNSUPPORTED;
    __nv_bfloat16* ob = static_cast<__nv_bfloat16*>(o);
    if (Dv == 64)
        b2::split_merge_kernel<64><<<(unsigned)blocks, 256, 0, st>>>(o_part, lse_part, num_splits, R, ob, o_row_stride, lse);
    else if (Dv == 128)
        b2::split_merge_kernel<128><<<(unsigned)blocks, 256, 0, st>>>(o_part, lse_part, num_splits, R, ob, o_row_stride, lse);
    else
        b2::split_merge_kernel<512><<<(unsigned)blocks, 256, 0, st>>>(o_part, lse_part, num_splits, R, ob, o_row_stride, lse);
    return launch_status();
}

// ------------------------------------------------------------- diagnostics
int attn_get_device_error(void* stream) {
    if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return ATTN_ERR_CUDA;
    int v = 0;
    if (cudaMemcpyFromSymbol(&v, b2::g_device_status, sizeof(int)) != cudaSuccess) return ATTN_ERR_CUDA;
    const int zero = 0;
    if (cudaMemcpyToSymbol(b2::g_device_status, &zero, sizeof(int)) != cudaSuccess) return ATTN_ERR_CUDA;
    return v;
}

int attn_selftest_exp2(const float* t, float* y, int64_t n, void* stream) {
    if (n < 0 || (n > 0 && (!t || !y))) return ATTN_ERR_INVALID_ARG;
    if (n == 0) return ATTN_OK;
    const int64_t blocks = (n / 2 + 255) / 256 + 1;
    if (blocks > 0x7fffffff) return ATTN_ERR_UNSUPPORTED;
    b2::selftest_exp2_kernel<<<(unsigned)blocks, 256, 0, static_cast<cudaStream_t>(stream)>>>(t, y, n);
    return launch_status();
}

int attn_selftest_page_coords(const int32_t* page_table, int64_t page_table_stride, int page_size,
                              int64_t num_pages, int groups_per_page, const int32_t* b_idx, const int32_t* t_idx,
                              int64_t n, int64_t* out, void* stream) {
    if (n < 0 || page_size <= 0 || num_pages <= 0 || groups_per_page <= 0 || page_table_stride < 0)
        return ATTN_ERR_INVALID_ARG;
    if (num_pages * groups_per_page >= ((int64_t)1 << 31)) return ATTN_ERR_UNSUPPORTED;
    if (n == 0) return ATTN_OK;
    if (!page_table || !b_idx || !t_idx || !out) return ATTN_ERR_INVALID_ARG;
    const int64_t want = (n + 255) / 256;
    const unsigned blocks = (unsigned)(want < 1024 ? want : 1024);
    b2::page_coords_kernel<<<blocks, 256, 0, static_cast<cudaStream_t>(stream)>>>(
        page_table, page_table_stride, page_size, num_pages, groups_per_page, b_idx, t_idx, n, out);
    return launch_status();
}

int attn_selftest_bounded_wait(uint64_t timeout_ns, void* stream) {
    b2::selftest_wait_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(timeout_ns);
    return launch_status();
}

}  // extern "C"
