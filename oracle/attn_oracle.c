/*
 * attn_oracle.c -- plain, slow, fp64 CPU oracle for forward scaled-dot-product
 * attention.  TEST INFRASTRUCTURE ONLY: tests/, __graft_entry__.smoke() and the
 * cpu_baseline leg of bench.py may call it; the library never does.  It shares
 * no code, header, table or helper with the CUDA path.
 *
 * What it computes (the plain definition, no blocking, no online softmax):
 *
 *   for a query row q and the set A of keys it may see,
 *     s_j   = scale * sum_d q[d] * k_j[d]                     (fp64)
 *     m     = max_{j in A} s_j
 *     l     = sum_{j in A} exp(s_j - m)
 *     LSE   = m + ln(l)                                       (natural log)
 *     O[:]  = sum_{j in A} exp(s_j - m) / l * v_j[:]
 *     A empty  ->  O = 0, LSE = -inf
 *
 * Sources (page title + section):
 *  - softmax(Q K^T * scale + mask) V with a natural-log Stats output:
 *    "cuDNN Frontend v1.30.0 Release Notes", section "New: stats_use_log2 -- LSE
 *    in base 2" (cuDNN returns max + ln(sum_exp)); Stats is FP32 on the library
 *    side: "cuDNN Frontend v1.28.0 release notes", "Updates to Graph API / SDPA".
 *  - rows with no live keys give a zero output and a negative-infinity LSE:
 *    "cuDNN Frontend v1.32.0 Release Notes", "New: Rubin triangle operations".
 *  - causal mask is bottom-right aligned per sequence: "cuDNN Frontend v1.28.0
 *    release notes", "Masking, splitting, and heuristics" (per-sequence THD
 *    bottom-right diagonals).  Key j is visible to query i of a sequence with
 *    Lq queries and Lkv keys iff j <= i + (Lkv - Lq).
 *  - GQA: query head h reads key/value head h / (Hq / Hkv): "cuDNN Frontend
 *    v1.30.0 Release Notes", "New: decode tiles" (G = H_q / H_kv).
 *  - packed THD addressing (head dim innermost, then heads, then tokens; a
 *    sequence's base comes from the offset table, the batch stride is never
 *    read): "cuDNN Frontend v1.30.0 Release Notes", "New: the FlashInfer
 *    serving path runs on FROST".
 *  - paged KV with a per-sequence page table and split-KV partials merged by
 *    their LSE: "cuDNN Frontend v1.31.0 Release Notes", "SDPA: paged KV,
 *    split-KV, and engine selection"; "cuDNN Frontend v1.28.0 release notes",
 *    "Masking, splitting, and heuristics".
 *
 * Inputs are bf16 bit patterns (uint16), widened exactly to double.  Strides
 * are int64 element counts.  Outputs are double.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

static double bf16_to_double(uint16_t bits)
{
    uint32_t u = ((uint32_t)bits) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/*
 * The definition for one query row.  q points at Dqk elements (unit stride);
 * key j is k_base[k_off[j] + d], value j is v_base[v_off[j] + d].
 */
static void attend_one_row(const uint16_t *q, int Dqk,
                           const uint16_t *k_base, const int64_t *k_off,
                           const uint16_t *v_base, const int64_t *v_off,
                           int64_t nkeys, int Dv, double scale,
                           double *o, double *lse)
{
    if (nkeys <= 0) {
        for (int d = 0; d < Dv; ++d) o[d] = 0.0;
        *lse = -INFINITY;
        return;
    }
    double *qd = (double *)malloc(sizeof(double) * (size_t)Dqk);
    double *s = (double *)malloc(sizeof(double) * (size_t)nkeys);
    for (int d = 0; d < Dqk; ++d) qd[d] = bf16_to_double(q[d]);

    double m = -INFINITY;
    for (int64_t j = 0; j < nkeys; ++j) {
        const uint16_t *kj = k_base + k_off[j];
        double dot = 0.0;
        for (int d = 0; d < Dqk; ++d) dot += qd[d] * bf16_to_double(kj[d]);
        s[j] = scale * dot;
        if (s[j] > m) m = s[j];
    }
    double l = 0.0;
    for (int64_t j = 0; j < nkeys; ++j) l += exp(s[j] - m);

    for (int d = 0; d < Dv; ++d) o[d] = 0.0;
    for (int64_t j = 0; j < nkeys; ++j) {
        double p = exp(s[j] - m) / l;
        const uint16_t *vj = v_base + v_off[j];
        for (int d = 0; d < Dv; ++d) o[d] += p * bf16_to_double(vj[d]);
    }
    *lse = m + log(l);
    free(qd);
    free(s);
}

/* Number of keys a query row sees under the (optional) bottom-right causal mask:
 * keys 0 .. min(Lkv-1, i + Lkv - Lq). */
static int64_t visible_keys(int64_t i, int64_t Lq, int64_t Lkv, int causal)
{
    if (!causal) return Lkv;
    int64_t last = i + (Lkv - Lq);          /* largest visible key index */
    if (last < 0) return 0;
    return (last + 1 < Lkv) ? last + 1 : Lkv;
}

/*
 * Ragged / packed THD layout.  Sequence b holds query tokens
 * [cu_q[b], cu_q[b+1]) and key/value tokens [cu_kv[b], cu_kv[b+1]).  Element
 * (t, h, d) of Q sits at q[t*q_ts + h*q_hs + d]; likewise K, V.
 * Each requested row r is (row_b[r], row_h[r], row_i[r]) with row_i the query
 * index inside its sequence.  Results: o[r*Dv + d], lse[r].
 */
void oracle_attn_ragged_rows(const uint16_t *q, const uint16_t *k, const uint16_t *v,
                             const int32_t *cu_q, const int32_t *cu_kv,
                             int Hq, int Hkv, int Dqk, int Dv,
                             int64_t q_ts, int64_t q_hs, int64_t k_ts, int64_t k_hs,
                             int64_t v_ts, int64_t v_hs,
                             double scale, int causal,
                             int64_t nrows, const int32_t *row_b, const int32_t *row_h,
                             const int32_t *row_i, double *o, double *lse)
{
    const int G = Hq / Hkv;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t r = 0; r < nrows; ++r) {
        int b = row_b[r], h = row_h[r], g = h / G;
        int64_t i = row_i[r];
        int64_t Lq = cu_q[b + 1] - cu_q[b];
        int64_t Lkv = cu_kv[b + 1] - cu_kv[b];
        int64_t n = visible_keys(i, Lq, Lkv, causal);
        int64_t *ko = (int64_t *)malloc(sizeof(int64_t) * (size_t)(n > 0 ? n : 1));
        int64_t *vo = (int64_t *)malloc(sizeof(int64_t) * (size_t)(n > 0 ? n : 1));
        for (int64_t j = 0; j < n; ++j) {
            int64_t t = (int64_t)cu_kv[b] + j;
            ko[j] = t * k_ts + (int64_t)g * k_hs;
            vo[j] = t * v_ts + (int64_t)g * v_hs;
        }
        const uint16_t *qrow = q + ((int64_t)cu_q[b] + i) * q_ts + (int64_t)h * q_hs;
        attend_one_row(qrow, Dqk, k, ko, v, vo, n, Dv, scale, o + r * Dv, lse + r);
        free(ko);
        free(vo);
    }
}

/*
 * Dense BSHD layout: element (b, s, h, d) of Q at q[b*qs[0] + s*qs[1] + h*qs[2] + d].
 * Each requested row r is (row_b[r], row_h[r], row_i[r]) with row_i in [0, Sq).
 */
void oracle_attn_dense_rows(const uint16_t *q, const uint16_t *k, const uint16_t *v,
                            int Sq, int Skv, int Hq, int Hkv, int Dqk, int Dv,
                            const int64_t *qs, const int64_t *ks, const int64_t *vs,
                            double scale, int causal,
                            int64_t nrows, const int32_t *row_b, const int32_t *row_h,
                            const int32_t *row_i, double *o, double *lse)
{
    const int G = Hq / Hkv;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t r = 0; r < nrows; ++r) {
        int b = row_b[r], h = row_h[r], g = h / G;
        int64_t i = row_i[r];
        int64_t n = visible_keys(i, Sq, Skv, causal);
        int64_t *ko = (int64_t *)malloc(sizeof(int64_t) * (size_t)(n > 0 ? n : 1));
        int64_t *vo = (int64_t *)malloc(sizeof(int64_t) * (size_t)(n > 0 ? n : 1));
        for (int64_t j = 0; j < n; ++j) {
            ko[j] = (int64_t)b * ks[0] + j * ks[1] + (int64_t)g * ks[2];
            vo[j] = (int64_t)b * vs[0] + j * vs[1] + (int64_t)g * vs[2];
        }
        const uint16_t *qrow = q + (int64_t)b * qs[0] + i * qs[1] + (int64_t)h * qs[2];
        attend_one_row(qrow, Dqk, k, ko, v, vo, n, Dv, scale, o + r * Dv, lse + r);
        free(ko);
        free(vo);
    }
}

/*
 * Paged KV, one query token per sequence (decode).  Logical key token t of
 * sequence b lives in physical page page_table[b*pt_stride + t/page_size] at
 * slot t % page_size; element (page, slot, head, d) of the K pool is at
 * k_pool[page*kps[0] + slot*kps[1] + head*kps[2] + d] (likewise V with vps).
 * Q is [B, Hq, Dqk] with element (b, h, d) at q[b*q_bs + h*q_hs + d].
 *
 * Keys [key_lo, key_hi) of the sequence are attended, clipped to [0, kv_len).
 * Passing key_lo = 0 and key_hi >= kv_len gives the whole sequence; a split of
 * split-KV passes its own key range.  Rows r are (row_b[r], row_h[r]).
 */
void oracle_attn_paged_rows(const uint16_t *q, int64_t q_bs, int64_t q_hs,
                            const uint16_t *k_pool, const uint16_t *v_pool,
                            const int32_t *page_table, int64_t pt_stride,
                            const int32_t *kv_lens, int page_size,
                            int Hq, int Hkv, int Dqk, int Dv,
                            const int64_t *kps, const int64_t *vps,
                            double scale,
                            int64_t nrows, const int32_t *row_b, const int32_t *row_h,
                            const int64_t *key_lo, const int64_t *key_hi,
                            double *o, double *lse)
{
    const int G = Hq / Hkv;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t r = 0; r < nrows; ++r) {
        int b = row_b[r], h = row_h[r], g = h / G;
        int64_t L = kv_lens[b];
        int64_t lo = key_lo[r] < 0 ? 0 : key_lo[r];
        int64_t hi = key_hi[r] > L ? L : key_hi[r];
        int64_t n = hi > lo ? hi - lo : 0;
        int64_t *ko = (int64_t *)malloc(sizeof(int64_t) * (size_t)(n > 0 ? n : 1));
        int64_t *vo = (int64_t *)malloc(sizeof(int64_t) * (size_t)(n > 0 ? n : 1));
        for (int64_t j = 0; j < n; ++j) {
            int64_t t = lo + j;
            int64_t page = page_table[(int64_t)b * pt_stride + t / page_size];
            int64_t slot = t % page_size;
            ko[j] = page * kps[0] + slot * kps[1] + (int64_t)g * kps[2];
            vo[j] = page * vps[0] + slot * vps[1] + (int64_t)g * vps[2];
        }
        const uint16_t *qrow = q + (int64_t)b * q_bs + (int64_t)h * q_hs;
        attend_one_row(qrow, Dqk, k_pool, ko, v_pool, vo, n, Dv, scale, o + r * Dv, lse + r);
        free(ko);
        free(vo);
    }
}

/*
 * Split-KV merge by LSE ("cuDNN Frontend v1.28.0 release notes", "Masking,
 * splitting, and heuristics"; "cuDNN Frontend v1.30.0 Release Notes",
 * stats_use_log2 section on split partials).  For each of the R = B*Hq rows:
 *   LSE = ln sum_s exp(lse_s)          (written with the max factored out)
 *   O   = sum_s exp(lse_s - LSE) * O_s
 * Partials with lse_s = -inf carry no keys and contribute nothing; if every
 * partial is -inf the row has no keys: O = 0, LSE = -inf.
 * o_part is [S][R][Dv], lse_part is [S][R].
 */
void oracle_split_merge(const double *o_part, const double *lse_part,
                        int num_splits, int64_t R, int Dv,
                        double *o, double *lse)
{
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < R; ++r) {
        double M = -INFINITY;
        for (int s = 0; s < num_splits; ++s)
            if (lse_part[(int64_t)s * R + r] > M) M = lse_part[(int64_t)s * R + r];
        for (int d = 0; d < Dv; ++d) o[r * Dv + d] = 0.0;
        if (M == -INFINITY) {
            lse[r] = -INFINITY;
            continue;
        }
        double sum = 0.0;
        for (int s = 0; s < num_splits; ++s) sum += exp(lse_part[(int64_t)s * R + r] - M);
        double L = M + log(sum);
        for (int s = 0; s < num_splits; ++s) {
            double w = exp(lse_part[(int64_t)s * R + r] - L);
            if (w == 0.0) continue;
            const double *os = o_part + ((int64_t)s * R + r) * Dv;
            for (int d = 0; d < Dv; ++d) o[r * Dv + d] += w * os[d];
        }
        lse[r] = L;
    }
}

/* Threads OpenMP will use (reported by the CPU baseline). */
int oracle_num_threads(void)
{
#ifdef _OPENMP
    extern int omp_get_max_threads(void);
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* Sets the threads OpenMP uses from now on (the CPU baseline times the oracle
 * on all cores and on one).  Threading only: the arithmetic is unchanged. */
void oracle_set_num_threads(int n)
{
#ifdef _OPENMP
    extern void omp_set_num_threads(int);
    omp_set_num_threads(n > 0 ? n : 1);
#else
    (void)n;
#endif
}
