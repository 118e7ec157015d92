/*
 * b2attn.h -- C ABI of libb2attn.so: forward scaled-dot-product attention on
 * NVIDIA B200 (sm_100a).
 *
 *   O = softmax(scale * Q K^T + mask) V,   LSE = rowmax + ln(rowsum)   (fp32)
 *
 * in three layouts: dense BSHD, ragged/packed THD addressed through offset
 * tables, and paged KV with split-KV partials merged by their LSE.
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 *  - All tensor pointers are DEVICE pointers owned by the caller.  Q, K, V and
 *    O are bf16 (passed as void*); LSE and split partials are fp32.  Stats are
 *    FP32 only ("cuDNN Frontend v1.28.0 release notes", "Updates to Graph API /
 *    SDPA": Stats must be FP32).
 *  - LSE is the natural log: rowmax + ln(rowsum) ("cuDNN Frontend v1.30.0
 *    Release Notes", "New: stats_use_log2 -- LSE in base 2").  A query row that
 *    sees no key gets O = 0 and LSE = -inf ("cuDNN Frontend v1.32.0 Release
 *    Notes", "New: Rubin triangle operations").
 *  - Strides are int64 ELEMENT counts, and the head dimension is always
 *    contiguous (stride 1).  Every stride and the base pointer of Q, K, V and O
 *    must be 16-byte aligned (a multiple of 8 elements); 64-bit addressing
 *    throughout ("cuDNN Frontend v1.30.0 Release Notes", "New: prepared
 *    launches", int64 stride leaves).
 *  - `scale` is taken as given, 0 and negative values included ("cuDNN Frontend
 *    v1.31.0 Release Notes", "Compatibility and numerical behavior": an explicit
 *    zero is preserved).  It must be finite.
 *  - GQA/MQA: query head h reads key/value head h / (Hq / Hkv); Hq must be a
 *    multiple of Hkv ("cuDNN Frontend v1.30.0 Release Notes", "New: decode
 *    tiles").
 *  - Causal masking is bottom-right aligned per sequence: key j is visible to
 *    query i of a sequence with Lq queries and Lkv keys iff j <= i + Lkv - Lq
 *    ("cuDNN Frontend v1.28.0 release notes", "Masking, splitting, and
 *    heuristics").
 *  - The library owns no device memory, allocates none, and never blocks the
 *    host: every entry point validates its arguments on the host, enqueues its
 *    kernels on `stream` (a cudaStream_t passed as void*, NULL = legacy default
 *    stream) and returns ("cuDNN Frontend v1.30.0 Release Notes", "Graph API,
 *    Python API, and other operations": the graph API owns no device memory
 *    and never blocks the host).  No entry point reads device memory back to
 *    the host, so every call can be captured in a CUDA graph ("cuDNN Frontend
 *    v1.28.0 release notes", "Ragged / THD, with zero host reads").
 *  - Scratch space is caller-provided; a missing or undersized workspace is
 *    rejected before launch ("cuDNN Frontend v1.31.0 Release Notes",
 *    "Compatibility and numerical behavior": split-attention calls require
 *    caller workspace).
 *  - Return value: ATTN_OK or an error status.  Errors found on the host are
 *    returned before anything is enqueued.  Conditions only the device can see
 *    (inconsistent offset tables or lengths, out-of-range page ids, a bounded
 *    wait that ran out) are recorded in a device-side status word that
 *    attn_get_device_error() reads; the kernels never trap.
 *  - Inputs are supported for Dqk, Dv in {64, 128} (prefill and decode) and
 *    Dqk = 576, Dv = 512 (absorbed-MLA decode); other shapes are declined with
 *    ATTN_ERR_UNSUPPORTED, never computed wrongly.
 */
#ifndef B2ATTN_H
#define B2ATTN_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Status codes. */
#define ATTN_OK                  0
#define ATTN_ERR_INVALID_ARG     1  /* a pointer, size, stride or alignment is invalid */
#define ATTN_ERR_UNSUPPORTED     2  /* valid, but a shape this library declines      */
#define ATTN_ERR_WORKSPACE       3  /* workspace missing or smaller than required     */
#define ATTN_ERR_LAUNCH          4  /* a kernel launch failed (cudaGetLastError)      */
#define ATTN_ERR_DEVICE_TIMEOUT  5  /* device: a bounded wait ran out                 */
#define ATTN_ERR_DEVICE_INPUT    6  /* device: offsets / lengths / page ids invalid   */
#define ATTN_ERR_CUDA            7  /* a CUDA runtime or driver call failed           */

/* LSE layouts of attn_fwd_ragged. */
#define ATTN_LSE_PADDED_BSH  0  /* [B, max_seqlen_q, Hq]; rows past a sequence's
                                   length are set to -inf by the library on the
                                   launch stream ("cuDNN Frontend v1.30.0 Release
                                   Notes", "New: the FlashInfer serving path runs
                                   on FROST": per-batch padded Stats seeded -inf) */
#define ATTN_LSE_PACKED_TH   1  /* token-major [total_q, Hq]                    */
#define ATTN_LSE_PACKED_HT   2  /* head-major [Hq, total_q] (row stride total_q),
                                   FlashAttention's and PyTorch varlen's
                                   softmax_lse ("cuDNN Frontend v1.30.0 Release
                                   Notes", head-major [h, total_q] Stats)       */
/* Flag OR-ed into lse_layout: write the LSE in base 2,
 * log2(sum_j exp(s_j)) = LSE * log2(e), the convention of flash-attention-style
 * consumers, instead of the natural log ("cuDNN Frontend v1.30.0 Release
 * Notes", "New: stats_use_log2 -- LSE in base 2").  -inf stays -inf. */
#define ATTN_LSE_LOG2        0x100

/* Human-readable name of a status code (static string, never NULL). */
const char *attn_status_string(int status);

/*
 * Dense BSHD forward.
 *   q: [B, Sq, Hq, Dqk]   k: [B, Skv, Hkv, Dqk]   v: [B, Skv, Hkv, Dv]
 *   o: [B, Sq, Hq, Dv]    lse (nullable): fp32 [B, Hq, Sq], contiguous.
 * x_strides[3] are the (batch, seq, head) element strides of each tensor, so
 * strided views (e.g. slices of a fused QKV projection) are read in place
 * ("cuDNN Frontend v1.30.0 Release Notes", "New: prepared launches": dense
 * forward reads strided Q/K/V/O zero-copy).  With Sq != Skv the causal mask
 * is bottom-right aligned.
 * workspace: device scratch of at least attn_fwd_dense_workspace_size(...)
 * bytes, 256-byte aligned, owned by the caller ("cuDNN Frontend v1.31.0
 * Release Notes", "Compatibility and numerical behavior": caller workspace,
 * rejected before launch when missing); it holds the work list the device
 * builds for the call and the persistent CTAs' claim counter.  Its contents
 * need no initialisation and are rewritten by every call, so calls that
 * overlap on the GPU need workspaces of their own.
 */
int attn_fwd_dense(const void *q, const void *k, const void *v, void *o, float *lse,
                   int B, int Sq, int Skv, int Hq, int Hkv, int Dqk, int Dv,
                   const int64_t q_strides[3], const int64_t k_strides[3],
                   const int64_t v_strides[3], const int64_t o_strides[3],
                   float scale, int causal, void *workspace, size_t workspace_bytes,
                   void *stream);

/* Workspace bytes attn_fwd_dense needs: a 256-byte header plus 16 bytes per
 * (batch, 128-row query tile, pair of query heads sharing a KV head) work item
 * (same caller-workspace contract as above).  Host-only arithmetic; 0 for
 * invalid arguments. */
size_t attn_fwd_dense_workspace_size(int B, int Sq, int Hq, int Hkv);

/*
 * Ragged / packed THD forward.
 * Sequence b owns query tokens [cu_seqlens_q[b], cu_seqlens_q[b+1]) and key /
 * value tokens [cu_seqlens_kv[b], cu_seqlens_kv[b+1]); both tables are DEVICE
 * int32 arrays of B+1 nondecreasing prefix sums starting at 0 ("cuDNN Frontend
 * v1.28.0 release notes", "Ragged / THD, with zero host reads"; "cuDNN
 * Frontend v1.30.0 Release Notes": the THD gate is over (H, S, D), the batch
 * stride is never read).
 *   q: element (t, h, d) at q[t*q_strides[0] + h*q_strides[1] + d]; same for
 *   k, v, o with their own (token, head) strides.
 * max_seqlen_q / max_seqlen_kv bound every sequence's length and total_q /
 * total_kv bound the packed token counts; these host-declared capacities size
 * the launch and the TMA bounds, so no token past total_q / total_kv is ever
 * read or written ("cuDNN Frontend v1.28.0 release notes", "Updates to Graph
 * API / SDPA": max_total_seq_len_q / _kv).  A device table that breaks them
 * sets ATTN_ERR_DEVICE_INPUT and the offending sequences are skipped.
 * lse (nullable): layout per lse_layout (ATTN_LSE_PADDED_BSH, _PACKED_TH or
 * _PACKED_HT, optionally | ATTN_LSE_LOG2).
 * workspace: device scratch of at least attn_fwd_ragged_workspace_size(...)
 * bytes, 256-byte aligned; it holds the device-built work list.
 */
int attn_fwd_ragged(const void *q, const void *k, const void *v, void *o, float *lse,
                    const int32_t *cu_seqlens_q, const int32_t *cu_seqlens_kv,
                    int B, int max_seqlen_q, int max_seqlen_kv,
                    int64_t total_q, int64_t total_kv,
                    int Hq, int Hkv, int Dqk, int Dv,
                    const int64_t q_strides[2], const int64_t k_strides[2],
                    const int64_t v_strides[2], const int64_t o_strides[2],
                    int lse_layout, float scale, int causal,
                    void *workspace, size_t workspace_bytes, void *stream);

/* Workspace bytes attn_fwd_ragged needs for these declared capacities: the
 * caller sizes and owns the scratch, and passes it with the call ("cuDNN
 * Frontend v1.31.0 Release Notes", "Compatibility and numerical behavior":
 * direct callers ask for the scratch workspace size, allocate it and pass it;
 * a missing workspace is rejected before launch).  Host-only arithmetic; 0 for
 * invalid arguments. */
size_t attn_fwd_ragged_workspace_size(int B, int max_seqlen_q, int64_t total_q,
                                      int Hq, int Hkv);

/*
 * attn_fwd_ragged without a workspace argument, for callers that cannot
 * allocate device memory when they call (the release pages have no
 * counterpart; this entry point is specific to this library).  Typical
 * callers: plugins and runtimes whose host framework owns every device
 * allocation and gives a kernel library none while it executes, and serving
 * loops that size all their device buffers at start-up and may not call
 * cudaMalloc afterwards (an allocation there can synchronize the device and
 * stall the streams already in flight).
 * The work list lives in a 4 MiB array built into the library instead
 * (attn_fwd_ragged_noalloc_max_scratch() returns the size); every GPU that
 * loads the library holds it until the process exits.  Arguments, layouts
 * and results are those of attn_fwd_ragged.
 *  - Capacities whose work list needs more than 4 MiB
 *    (attn_fwd_ragged_workspace_size(...) > 4 MiB) return ATTN_ERR_WORKSPACE.
 *  - The first call on a device that passes the argument checks looks up
 *    the array's device address (cudaGetSymbolAddress, once per device);
 *    make that first call before any stream capture.
 *  - All calls share the one array, and each call rewrites it before use.
 *    Calls that overlap on the GPU (e.g. issued on two streams without an
 *    ordering between them) race on it: order them on one stream.
 *  - It allocates nothing: no cudaMalloc, no cudaFree, no allocating library call.
 */
int attn_fwd_ragged_noalloc(const void *q, const void *k, const void *v, void *o, float *lse,
                            const int32_t *cu_seqlens_q, const int32_t *cu_seqlens_kv,
                            int B, int max_seqlen_q, int max_seqlen_kv,
                            int64_t total_q, int64_t total_kv,
                            int Hq, int Hkv, int Dqk, int Dv,
                            const int64_t q_strides[2], const int64_t k_strides[2],
                            const int64_t v_strides[2], const int64_t o_strides[2],
                            int lse_layout, float scale, int causal, void *stream);

/* Bytes of the built-in scratch attn_fwd_ragged_noalloc uses (4 MiB). */
size_t attn_fwd_ragged_noalloc_max_scratch(void);

/*
 * Paged-KV decode forward: one query token per sequence, attending to all of
 * its kv_lens[b] cached keys ("cuDNN Frontend v1.31.0 Release Notes", "SDPA:
 * paged KV, split-KV, and engine selection").
 *   q: [B, Hq, Dqk] with (batch, head) element strides q_strides[2].
 *   o: [B, Hq, Dv]  with (batch, head) element strides o_strides[2]; for MLA
 *   with num_splits > 1 the rows must be batch-major (o_strides[0] == Hq *
 *   o_strides[1]), else ATTN_ERR_UNSUPPORTED before anything is enqueued.
 *   lse (nullable): fp32 [B, Hq] contiguous.
 *   k_pool / v_pool: pools of num_pages fixed-size pages; element
 *   (page, slot, head, d) at pool[page*s[0] + slot*s[1] + head*s[2] + d] with
 *   s = k_pool_strides / v_pool_strides, so K and V may have different
 *   layouts.  Logical key t of sequence b is slot t % page_size of page
 *   page_table[b*page_table_stride + t / page_size] (DEVICE int32).
 *   Absorbed MLA: pass v_pool == k_pool with Dv < Dqk; V is then the first Dv
 *   columns of each K row ("cuDNN Frontend v1.32.0 Release Notes", "SDPA:
 *   wider native forward support": Q/K576, V512, absorbed-MLA cache layouts).
 *   MLA (Dqk 576, Dv 512) needs Hkv == 1, page_size 16, 32 or a multiple of
 *   64, and a K pool whose page stride is a whole number of 8-row groups
 *   (k_pool_strides[0] % (8 * k_pool_strides[1]) == 0; dense pools qualify)
 *   (ATTN_ERR_UNSUPPORTED otherwise); any Hq (groups of 128 heads).
 *   GQA needs page_size dividing or divisible by 64 (at least 8) and
 *   Hq / Hkv <= 16.
 *   Each page-table row holds at least ceil(max_kv_len / page_size) entries.
 *   kv_lens: DEVICE int32 [B], each in [0, max_kv_len]; page ids must lie in
 *   [0, num_pages).  Violations set ATTN_ERR_DEVICE_INPUT on the device.
 * Split-KV (num_splits > 1), GQA: the keys of each (sequence, KV head) are
 * cut into 64-key units, and its n units into min(num_splits, n) pieces of
 * n / pieces units (to within one), one block per piece, the sequences
 * longest first (a device-side schedule in the workspace).  A piece that is
 * the whole sequence writes O directly; the others write fp32 partial O and
 * LSE, merged by LSE (as attn_split_merge does) inside the same launch by the
 * last block to finish each group of up to 8 of a sequence's partials.  MLA:
 * each sequence's pages are cut into num_splits ranges of ceil(n_pages /
 * num_splits) pages, the clusters take the sequences longest first and a
 * second launch merges the partials.  The schedule changes which block
 * computes a piece, never the result.  workspace: >=
 * attn_fwd_paged_workspace_size(...) bytes, 256-byte aligned (may be NULL
 * when num_splits == 1).
 */
int attn_fwd_paged(const void *q, const void *k_pool, const void *v_pool, void *o,
                   float *lse, const int32_t *page_table, int64_t page_table_stride,
                   const int32_t *kv_lens, int B, int Hq, int Hkv, int Dqk, int Dv,
                   int page_size, int64_t num_pages, int max_kv_len,
                   const int64_t q_strides[2], const int64_t o_strides[2],
                   const int64_t k_pool_strides[3], const int64_t v_pool_strides[3],
                   float scale, int num_splits,
                   void *workspace, size_t workspace_bytes, void *stream);

/*
 * attn_fwd_paged with independent K and V page tables: logical key t of
 * sequence b reads its key row from page k_page_table[b*k_page_table_stride +
 * t / page_size] of k_pool and its value row from page
 * v_page_table[b*v_page_table_stride + t / page_size] of v_pool ("cuDNN
 * Frontend v1.32.0 Release Notes", "SDPA: wider native forward support":
 * independent K/V tables and layouts).  Both are DEVICE int32 tables whose
 * rows cover max_kv_len keys; page ids of both lie in [0, num_pages) (each
 * pool holds at least num_pages pages).  Everything else, including the MLA
 * and GQA rules and the split-KV workspace, is as for attn_fwd_paged, which
 * is this call with both tables the same.
 */
int attn_fwd_paged_kv_tables(const void *q, const void *k_pool, const void *v_pool, void *o,
                             float *lse, const int32_t *k_page_table, int64_t k_page_table_stride,
                             const int32_t *v_page_table, int64_t v_page_table_stride,
                             const int32_t *kv_lens, int B, int Hq, int Hkv, int Dqk, int Dv,
                             int page_size, int64_t num_pages, int max_kv_len,
                             const int64_t q_strides[2], const int64_t o_strides[2],
                             const int64_t k_pool_strides[3], const int64_t v_pool_strides[3],
                             float scale, int num_splits,
                             void *workspace, size_t workspace_bytes, void *stream);

/*
 * Ragged queries over a paged K/V cache: chunked prefill, decode and
 * multi-token decode rows in one batch ("cuDNN Frontend v1.31.0 Release
 * Notes", "SDPA: paged KV, split-KV, and engine selection": paged K/V for
 * prefill, prepared paged D128 THD split-KV; "cuDNN Frontend v1.28.0 release
 * notes", ragged / THD queries).  Sequence b has
 * Lq_b = cu_seqlens_q[b+1] - cu_seqlens_q[b] queries, the LAST Lq_b positions
 * of its kv_lens[b] cached keys: with causal, query i sees keys
 * j <= i + kv_lens[b] - Lq_b (bottom-right); Lq_b > kv_lens[b] leaves the
 * first rows without keys (O = 0, LSE = -inf).
 *   q, o: packed THD [total_q, Hq, D], (token, head) element strides.
 *   k_pool / v_pool, page_table, kv_lens: as for attn_fwd_paged (DEVICE).
 *   lse / lse_layout: as for attn_fwd_ragged.
 * Short rows: the sequences with 1 <= Lq_b <= qmax queries, qmax =
 * min(4, 64 / (Hq / Hkv), max_seqlen_q) (none when Hq / Hkv > 64), run on the
 * split-KV decode kernel, which streams their keys once per KV head with the
 * G query heads x Lq_b tokens as the rows of its tiles; the others run on the
 * tensor-core prefill kernel in 128-row query tiles.  The split is decided on
 * the device from cu_seqlens_q (no host read); results do not depend on it.
 * num_splits (>= 1) splits the keys of each short sequence as attn_fwd_paged
 * does for GQA (pieces of 64-key units, fp32 partials in the workspace merged
 * by LSE in the same launch); it does not affect the other sequences.  attn_paged_suggest_splits gives a count.
 * Supported: D = Dqk = Dv in {64, 128}, Hq % Hkv == 0, page_size dividing 128
 * (at least 8) or a multiple of 128, and pools whose page stride is a whole
 * number of 8-row groups (page stride % (8 * row stride) == 0, the same for K
 * and V; dense HND and NHD pools qualify); else ATTN_ERR_UNSUPPORTED.
 * workspace: >= attn_fwd_paged_prefill_workspace_size(...) bytes, 256-byte
 * aligned.  Row slots past kv_len inside a sequence's last page are never
 * read into O (stale or NaN values are zeroed on chip).
 */
int attn_fwd_paged_prefill(const void *q, const void *k_pool, const void *v_pool, void *o,
                           float *lse, const int32_t *cu_seqlens_q, const int32_t *page_table,
                           int64_t page_table_stride, const int32_t *kv_lens, int B,
                           int max_seqlen_q, int64_t total_q, int Hq, int Hkv, int D,
                           int page_size, int64_t num_pages, int max_kv_len,
                           const int64_t q_strides[2], const int64_t o_strides[2],
                           const int64_t k_pool_strides[3], const int64_t v_pool_strides[3],
                           int lse_layout, float scale, int causal, int num_splits,
                           void *workspace, size_t workspace_bytes, void *stream);

/*
 * attn_fwd_paged_prefill with independent K and V page tables (K rows through
 * k_page_table, V rows through v_page_table, as for attn_fwd_paged_kv_tables);
 * otherwise identical, and attn_fwd_paged_prefill is this call with both
 * tables the same.
 */
int attn_fwd_paged_prefill_kv_tables(const void *q, const void *k_pool, const void *v_pool, void *o,
                                     float *lse, const int32_t *cu_seqlens_q,
                                     const int32_t *k_page_table, int64_t k_page_table_stride,
                                     const int32_t *v_page_table, int64_t v_page_table_stride,
                                     const int32_t *kv_lens, int B, int max_seqlen_q, int64_t total_q,
                                     int Hq, int Hkv, int D, int page_size, int64_t num_pages,
                                     int max_kv_len, const int64_t q_strides[2],
                                     const int64_t o_strides[2], const int64_t k_pool_strides[3],
                                     const int64_t v_pool_strides[3], int lse_layout, float scale,
                                     int causal, int num_splits, void *workspace, size_t workspace_bytes,
                                     void *stream);

/* Workspace bytes attn_fwd_paged_prefill needs: the prefill work list (as for
 * attn_fwd_ragged) and, with num_splits > 1, the short rows' split schedule,
 * merge counters and fp32 partials (num_splits * B * Hkv pieces of
 * Hq / Hkv * qmax rows of D floats) (caller workspace as in "cuDNN Frontend
 * v1.31.0 Release Notes", "Compatibility and numerical behavior").  Host-only
 * arithmetic; 0 for invalid arguments. */
size_t attn_fwd_paged_prefill_workspace_size(int B, int max_seqlen_q, int64_t total_q, int Hq, int Hkv,
                                             int D, int num_splits);

/* Workspace bytes attn_fwd_paged needs (0 when num_splits == 1): the split
 * schedule, the merge counters and the fp32 partials (MLA: the partials and the
 * launch order) live in caller-owned scratch ("cuDNN
 * Frontend v1.31.0 Release Notes", "Compatibility and numerical behavior":
 * split-attention calls require caller workspace, sized by a query). */
size_t attn_fwd_paged_workspace_size(int B, int Hq, int Dv, int num_splits);

/*
 * A split count for attn_fwd_paged: enough (batch, head, split) blocks to keep
 * num_sms SMs busy through the tail of uneven lengths, while the fp32 partials
 * stay a small fraction of the KV bytes streamed ("cuDNN Frontend v1.31.0
 * Release Notes", "SDPA: paged KV, split-KV, and engine selection": split
 * selection from the physical launch capacity and the ragged work, not from a
 * dense envelope).  GQA batches that fit one wave of blocks (two per SM)
 * get the count that fills that wave, or one block per SM for whole-page
 * boxes of 64 rows over caches of at most 8192 keys.  Host-only arithmetic;
 * the choice never changes results beyond rounding.
 */
int attn_paged_suggest_splits(int B, int Hq, int Hkv, int Dqk, int Dv, int max_kv_len,
                              int page_size, int num_sms);

/*
 * Split-KV merge by LSE, over R rows (R = B * Hq for decode):
 *   LSE_r = ln sum_s exp(lse_part[s][r]),   O_r = sum_s exp(lse_part[s][r] - LSE_r) * o_part[s][r][:]
 * Partials with lse = -inf (splits without keys) are ignored; a row whose
 * partials are all -inf gets O = 0, LSE = -inf ("cuDNN Frontend v1.28.0 release
 * notes", "Masking, splitting, and heuristics"; "cuDNN Frontend v1.30.0
 * Release Notes", stats_use_log2 section on split partials).
 *   o_part: fp32 [num_splits][R][Dv], lse_part: fp32 [num_splits][R] (contiguous)
 *   o: bf16, row r at o + r*o_row_stride (elements);  lse (nullable): fp32 [R].
 */
int attn_split_merge(const float *o_part, const float *lse_part, int num_splits,
                     int64_t R, int Dv, void *o, int64_t o_row_stride, float *lse,
                     void *stream);

/*
 * Synchronizes `stream`, returns the device-side status word (ATTN_OK,
 * ATTN_ERR_DEVICE_TIMEOUT or ATTN_ERR_DEVICE_INPUT; the first error recorded
 * since the last call) for the current device, and clears it.  This is the one
 * entry point that blocks the host; it is a diagnostic, not part of the
 * compute path.
 */
int attn_get_device_error(void *stream);

/*
 * Fault-free check of the bounded-wait machinery: launches one block that
 * waits, with the library's bounded wait and a limit of timeout_ns
 * nanoseconds, on a barrier nothing ever signals.  The wait runs out, the
 * kernel records ATTN_ERR_DEVICE_TIMEOUT and returns; the context stays
 * usable.  Returns the launch status.
 */
int attn_selftest_bounded_wait(uint64_t timeout_ns, void *stream);

/*
 * Diagnostic: y[i] = 2^t[i] evaluated the way the prefill softmax evaluates
 * the share of its exponentials it moves off the MUFU unit onto the FMA pipe
 * (base-2 range reduction n = round(t), f = t - n, a degree-3 polynomial for
 * 2^f, n added to the exponent; "cuDNN Frontend v1.30.0 Release Notes", "SDPA:
 * more kernels and numerics": exp2 on the FMA pipe).  Inputs below -125 give
 * 2^-125.  t and y are device arrays of n floats.
 */
int attn_selftest_exp2(const float *t, float *y, int64_t n, void *stream);

/*
 * Diagnostic of the page-table address generation: for n sampled logical keys
 * (b_idx[i], t_idx[i]) writes out[3i], out[3i+1], out[3i+2] = (physical page,
 * row in the page, 8-row group of the pool) computed by the same device
 * functions the paged producers use, so a test can check them against the
 * definition bit for bit ("cuDNN Frontend v1.31.0 Release Notes", "SDPA:
 * paged KV, split-KV, and engine selection": key t of sequence b is row
 * t % page_size of page page_table[b * page_table_stride + t / page_size]; the
 * group is page * groups_per_page + row / 8).  A table entry outside
 * [0, num_pages) gives page = group = -1 and records ATTN_ERR_DEVICE_INPUT,
 * as it does in the producers.  Every (b_idx[i], t_idx[i]) must address an
 * entry of the table (t_idx >= 0).  All arrays are DEVICE memory; out holds
 * 3n int64.  num_pages * groups_per_page must stay below 2^31
 * (ATTN_ERR_UNSUPPORTED otherwise).
 */
int attn_selftest_page_coords(const int32_t *page_table, int64_t page_table_stride, int page_size,
                              int64_t num_pages, int groups_per_page, const int32_t *b_idx,
                              const int32_t *t_idx, int64_t n, int64_t *out, void *stream);

#ifdef __cplusplus
}
#endif

#endif /* B2ATTN_H */
