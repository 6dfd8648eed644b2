/*
 * dsa_oracle.c -- plain, slow fp64 CPU oracle for the DeepSeek Sparse Attention
 * (DSA) decode path: lightning-indexer scores, per-query TopK, and sparse
 * MQA-mode MLA attention over the selected latent rows.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test suite, the package smoke check and
 * the benchmark's CPU-baseline leg may load this library.  The GPU library
 * shares no code with it and never calls it.
 *
 * Every function is the plain definition of one step, written in the pages'
 * notation, with no blocking, fusion or reordering beyond what the definition
 * states.  Loops over independent outputs may run in parallel (OpenMP); every
 * single output is summed in a fixed sequential order.
 *
 * Sources (web pages on DeepSeek-V3.2 DSA):
 *   [marsggbo]  "arXiv'25 | DSA lets DeepSeek-V3.2's long-context attention read
 *               less KV" (marsggbo.github.io), section 2 (toy example),
 *               section 3 (index score, TopK and attention equations),
 *               section 4 (MQA and MHA modes of MLA), sections 5.1 and 5.2
 *               (the indexer's distillation loss), section 6 (masked MHA
 *               for short prefill).
 *   [yuyanqi]   "DeepSeekV3.2之DSA" (yuyanqi.com), section 3.1 (symbol table),
 *               section 3.3 (TopK and the short-history rule), section 4.3
 *               (FP8 kernel comment: fp8 q.k -> relu * weights -> head sum ->
 *               * k_s), section 4.4 (topk(min(topk, end_pos)) returns indices),
 *               section 4.5 (skip scoring when the history fits in k),
 *               section 5.1 (softmax(q.[c_kv; k_pe]^T).c_kv).
 *   [aicoding]  "从稠密到稀疏：DeepSeek-V3.2的DSA机制如何重塑Transformer效率边界"
 *               (aicoding.csdn.net), section 4.3 (masked MHA below 8K tokens).
 *
 * Where the pages leave a step open, the reading taken is stated at the
 * function.  Parity is pinned by the tests under tests/ (toy example, brute
 * force, closed forms, library routines), not by this file.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* ------------------------------------------------------------------------- */
/* Number formats                                                              */
/* ------------------------------------------------------------------------- */

/* FP8 E4M3 as used by the indexer ("FP8" in [marsggbo] section 3 and the
 * e4m3 operands of the kernel comment in [yuyanqi] section 4.3).  Decoded from
 * the OCP 8-bit floating point definition of E4M3: 1 sign bit, 4 exponent bits
 * with bias 7, 3 mantissa bits; exponent field 0 is subnormal
 * (value = mantissa * 2^-9); exponent 15 with mantissa 7 is NaN; there are no
 * infinities, so the largest finite magnitude is 1.75 * 2^8 = 448. */
double dsa_oracle_e4m3_to_f64(uint8_t code)
{
    int sign = (code >> 7) & 1;
    int e = (code >> 3) & 0xF;
    int m = code & 0x7;
    double v;
    if (e == 0xF && m == 0x7) return NAN;
    if (e == 0)
        v = ldexp((double)m, -9);               /* m/8 * 2^(1-7) */
    else
        v = ldexp(1.0 + (double)m / 8.0, e - 7);
    return sign ? -v : v;
}

/* E4M3 encoding of a real number: the nearest finite E4M3 value after
 * clamping to [-448, 448], ties to the code with an even mantissa; NaN maps
 * to the NaN code.  Found by trying all 127 non-negative finite codes
 * (plain rather than clever).  Used by the q^I / k^I producer below. */
uint8_t dsa_oracle_f64_to_e4m3(double x)
{
    if (isnan(x)) return 0x7F;
    int sign = signbit(x) ? 1 : 0;
    double a = fabs(x);
    if (a > 448.0) a = 448.0;
    int best = 0;
    double best_d = INFINITY;
    for (int c = 0; c < 0x7F; ++c) {
        double d = fabs(dsa_oracle_e4m3_to_f64((uint8_t)c) - a);
        if (d < best_d || (d == best_d && (c & 1) == 0)) {
            best = c;
            best_d = d;
        }
    }
    return (uint8_t)(best | (sign << 7));
}

/* bfloat16: the upper 16 bits of an IEEE-754 binary32.  Widening is exact. */
double dsa_oracle_bf16_to_f64(uint16_t bits)
{
    uint32_t u = (uint32_t)bits << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* ------------------------------------------------------------------------- */
/* Where logical position s of a query's history lives in a cache              */
/* ------------------------------------------------------------------------- */

/* Both caches (the FP8 index-K cache and the bf16 latent cache) are indexed by
 * the same token positions ([yuyanqi] section 5.2, item 3).  A query q belongs
 * to sequence q_seq[q]; position s of that sequence is
 *   contiguous layout: row seq_row0[seq] + s
 *   paged layout:      row page_table[seq][s / page_size] * page_size
 *                          + s % page_size
 * (paged KV as named in [yuyanqi] section 4.4, "_get_topk_paged"). */
static int64_t cache_row(int32_t seq, int64_t s, const int64_t *seq_row0,
                         const int32_t *page_table, int32_t max_pages,
                         int32_t page_size)
{
    if (page_table != NULL) {
        int64_t page = page_table[(int64_t)seq * max_pages + s / page_size];
        return page * page_size + s % page_size;
    }
    return seq_row0[seq] + s;
}

static void set_threads(int32_t nthreads)
{
#ifdef _OPENMP
    if (nthreads > 0) omp_set_num_threads(nthreads);
#else
    (void)nthreads;
#endif
}

int32_t dsa_oracle_max_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* ------------------------------------------------------------------------- */
/* Step 1: lightning-indexer score                                             */
/* ------------------------------------------------------------------------- */

/* I[t,s] = sum_{j=1..H_I} w[t,j] * ReLU(q^I[t,j] . k^I[s])
 *   -- the index-score equation of [marsggbo] section 3, with the symbol
 *      table of [yuyanqi] section 3.1 (k^I has one head shared by all H_I
 *      indexer heads; w comes from the query token).
 * The FP8 kernel of [yuyanqi] section 4.3 multiplies the head sum by a
 * per-key dequantisation scale k_s; k_scale[row] plays that role here
 * (NULL means 1).
 * Reading taken: w is used exactly as given (every constant factor of
 * [yuyanqi] section 4.3 -- n_heads^-1/2, q scale, d_I^-1/2 -- is already folded
 * into it by the caller); no further scale is applied.
 *
 * Output: scores[q*ld + s] for s < q_n[q]; entries q_n[q] <= s < ld are -inf.
 * abs_scores (optional) receives sum_j |w| * ReLU(q.k) * |k_s|, the magnitude
 * against which a rounding error of the sum is measured. */
int dsa_oracle_indexer_scores(int32_t nq, int32_t h_idx, int32_t d_idx,
                              const uint8_t *q_idx, const uint16_t *w,
                              const uint8_t *kidx, const float *k_scale,
                              const int32_t *q_seq, const int32_t *q_n,
                              const int64_t *seq_row0,
                              const int32_t *page_table, int32_t max_pages,
                              int32_t page_size, double *scores,
                              double *abs_scores, int64_t ld, int32_t nthreads)
{
    if (nq < 0 || h_idx <= 0 || d_idx <= 0 || ld < 0) return -1;
    for (int32_t q = 0; q < nq; ++q)
        if (q_n[q] < 0 || q_n[q] > ld) return -1;
    set_threads(nthreads);

#pragma omp parallel for collapse(2) schedule(static)
    for (int32_t q = 0; q < nq; ++q) {
        for (int64_t s = 0; s < ld; ++s) {
            double *out = &scores[(int64_t)q * ld + s];
            double *aout = abs_scores ? &abs_scores[(int64_t)q * ld + s] : NULL;
            if (s >= q_n[q]) {
                *out = -INFINITY;
                if (aout) *aout = 0.0;
                continue;
            }
            int64_t row = cache_row(q_seq[q], s, seq_row0, page_table,
                                    max_pages, page_size);
            const uint8_t *k = kidx + row * (int64_t)d_idx;
            double ks = k_scale ? (double)k_scale[row] : 1.0;
            double total = 0.0, total_abs = 0.0;
            for (int32_t j = 0; j < h_idx; ++j) {
                const uint8_t *qj = q_idx + ((int64_t)q * h_idx + j) * d_idx;
                double dot = 0.0;
                for (int32_t d = 0; d < d_idx; ++d)
                    dot += dsa_oracle_e4m3_to_f64(qj[d]) *
                           dsa_oracle_e4m3_to_f64(k[d]);
                double relu = dot > 0.0 ? dot : 0.0;
                double wj = dsa_oracle_bf16_to_f64(w[(int64_t)q * h_idx + j]);
                total += wj * relu;
                total_abs += fabs(wj) * relu;
            }
            *out = total * ks;
            if (aout) *aout = total_abs * fabs(ks);
        }
    }
    return 0;
}

/* ------------------------------------------------------------------------- */
/* Step 2: TopK with the short-history rule                                    */
/* ------------------------------------------------------------------------- */

typedef struct {
    double score;
    int64_t pos;
} scored_pos;

/* Larger score first; among equal scores the lower position first
 * (the tie rule: lower index wins). -0.0 and +0.0 compare equal. */
static int by_score_then_pos(const void *a, const void *b)
{
    const scored_pos *x = (const scored_pos *)a, *y = (const scored_pos *)b;
    if (x->score > y->score) return -1;
    if (x->score < y->score) return 1;
    if (x->pos < y->pos) return -1;
    if (x->pos > y->pos) return 1;
    return 0;
}

/* I_t = TopK(I[t, s] over the visible history) -- [marsggbo] section 3; the
 * positions, not the scores, are the result ([yuyanqi] section 4.4,
 * "topk(...)[1]").  When the history has at most k positions every position
 * is kept ([yuyanqi] section 3.3 and section 4.5; topk(min(topk, end_pos))).
 *
 * n positions 0..n-1 with scores[0..n-1]; writes idx[0..k-1]: the min(k, n)
 * selected positions in rank order (score descending, position ascending),
 * then -1.  *nsel (optional) = min(k, n).  A full sort is used. */
int dsa_oracle_topk(int64_t n, const double *scores, int32_t k, int32_t *idx,
                    int32_t *nsel)
{
    if (n < 0 || k <= 0) return -1;
    int64_t keep = n < k ? n : k;
    if (n <= k) {
        for (int64_t i = 0; i < n; ++i) idx[i] = (int32_t)i;
    } else {
        scored_pos *all = (scored_pos *)malloc((size_t)n * sizeof(scored_pos));
        if (!all) return -2;
        for (int64_t s = 0; s < n; ++s) {
            all[s].score = scores[s];
            all[s].pos = s;
        }
        qsort(all, (size_t)n, sizeof(scored_pos), by_score_then_pos);
        for (int64_t i = 0; i < keep; ++i) idx[i] = (int32_t)all[i].pos;
        free(all);
    }
    for (int64_t i = keep; i < k; ++i) idx[i] = -1;
    if (nsel) *nsel = (int32_t)keep;
    return 0;
}

/* ------------------------------------------------------------------------- */
/* Step 3: sparse MQA-mode MLA attention over the selected latent rows          */
/* ------------------------------------------------------------------------- */

/* u_t = Attn(h_t, {c_s : s in I_t})            -- [marsggbo] section 3
 * In MQA mode every query head shares the one latent row c_s
 * ([marsggbo] section 4).  With weight absorption the attention is
 * softmax(q . [c_kv; k_pe]^T) . c_kv ([yuyanqi] section 5.1): the key is the
 * whole d_qk-wide row (512 latent + 64 rope), the value its first d_v columns.
 *
 * For every query q and head h, with the valid entries s_i of idx[q, :]
 * (entries that are -1 or >= q_n[q] are skipped; a position listed twice is
 * counted twice):
 *   S_i   = scale * sum_{d < d_qk} q[q,h,d] * c[s_i, d]
 *   m     = max_i S_i
 *   out   = sum_i exp(S_i - m) * c[s_i, 0:d_v] / sum_i exp(S_i - m)
 *   lse   = m + ln sum_i exp(S_i - m)
 * With no valid entry: out = 0 and lse = -inf.
 * kv row r starts at kv + r * kv_row_stride (elements). */
int dsa_oracle_sparse_mla(int32_t nq, int32_t h, int32_t d_qk, int32_t d_v,
                          double scale, const uint16_t *q, const uint16_t *kv,
                          int64_t kv_row_stride, const int32_t *q_seq,
                          const int32_t *q_n, const int64_t *seq_row0,
                          const int32_t *page_table, int32_t max_pages,
                          int32_t page_size, const int32_t *idx, int32_t k,
                          double *out, double *lse, int32_t nthreads)
{
    if (nq < 0 || h <= 0 || d_qk <= 0 || d_v <= 0 || d_v > d_qk || k < 0)
        return -1;
    set_threads(nthreads);
    int bad = 0;

#pragma omp parallel for collapse(2) schedule(dynamic, 1) reduction(| : bad)
    for (int32_t qi = 0; qi < nq; ++qi) {
        for (int32_t hh = 0; hh < h; ++hh) {
            const uint16_t *qv = q + ((int64_t)qi * h + hh) * d_qk;
            double *o = out + ((int64_t)qi * h + hh) * d_v;
            double *S = (double *)malloc((size_t)(k > 0 ? k : 1) * sizeof(double));
            int64_t *rows = (int64_t *)malloc((size_t)(k > 0 ? k : 1) * sizeof(int64_t));
            if (!S || !rows) { bad |= 1; free(S); free(rows); continue; }
            int32_t cnt = 0;
            for (int32_t i = 0; i < k; ++i) {
                int32_t s = idx[(int64_t)qi * k + i];
                if (s < 0 || s >= q_n[qi]) continue;
                rows[cnt++] = cache_row(q_seq[qi], s, seq_row0, page_table,
                                        max_pages, page_size);
            }
            for (int32_t d = 0; d < d_v; ++d) o[d] = 0.0;
            if (cnt == 0) {
                lse[(int64_t)qi * h + hh] = -INFINITY;
                free(S); free(rows);
                continue;
            }
            double m = -INFINITY;
            for (int32_t i = 0; i < cnt; ++i) {
                const uint16_t *c = kv + rows[i] * kv_row_stride;
                double dot = 0.0;
                for (int32_t d = 0; d < d_qk; ++d)
                    dot += dsa_oracle_bf16_to_f64(qv[d]) * dsa_oracle_bf16_to_f64(c[d]);
                S[i] = scale * dot;
                if (S[i] > m) m = S[i];
            }
            double denom = 0.0;
            for (int32_t i = 0; i < cnt; ++i) {
                double p = exp(S[i] - m);
                const uint16_t *c = kv + rows[i] * kv_row_stride;
                denom += p;
                for (int32_t d = 0; d < d_v; ++d) o[d] += p * dsa_oracle_bf16_to_f64(c[d]);
            }
            for (int32_t d = 0; d < d_v; ++d) o[d] /= denom;
            lse[(int64_t)qi * h + hh] = m + log(denom);
            free(S);
            free(rows);
        }
    }
    return bad ? -2 : 0;
}

/* The same attention over an FP8 latent cache.  Reading (the pages give FP8
 * only for the indexer's keys, [marsggbo] section 3 and [yuyanqi] section
 * 4.3): each latent row is stored in that same format, d_qk e4m3 codes and
 * one power-of-two scale per row (the pages' e8m0 k_s), and stands for
 *   c[s, d] = e4m3(code[s, d]) * kv_scale[row of s]
 * Everything else is dsa_oracle_sparse_mla's definition.  kv8 row r starts
 * at kv8 + r * kv8_row_bytes. */
int dsa_oracle_sparse_mla_fp8(int32_t nq, int32_t h, int32_t d_qk, int32_t d_v,
                              double scale, const uint16_t *q, const uint8_t *kv8,
                              int64_t kv8_row_bytes, const float *kv_scale,
                              const int32_t *q_seq, const int32_t *q_n,
                              const int64_t *seq_row0, const int32_t *page_table,
                              int32_t max_pages, int32_t page_size, const int32_t *idx,
                              int32_t k, double *out, double *lse, int32_t nthreads)
{
    if (nq < 0 || h <= 0 || d_qk <= 0 || d_v <= 0 || d_v > d_qk || k < 0)
        return -1;
    set_threads(nthreads);
    int bad = 0;

#pragma omp parallel for collapse(2) schedule(dynamic, 1) reduction(| : bad)
    for (int32_t qi = 0; qi < nq; ++qi) {
        for (int32_t hh = 0; hh < h; ++hh) {
            const uint16_t *qv = q + ((int64_t)qi * h + hh) * d_qk;
            double *o = out + ((int64_t)qi * h + hh) * d_v;
            double *S = (double *)malloc((size_t)(k > 0 ? k : 1) * sizeof(double));
            int64_t *rows = (int64_t *)malloc((size_t)(k > 0 ? k : 1) * sizeof(int64_t));
            if (!S || !rows) { bad |= 1; free(S); free(rows); continue; }
            int32_t cnt = 0;
            for (int32_t i = 0; i < k; ++i) {
                int32_t s = idx[(int64_t)qi * k + i];
                if (s < 0 || s >= q_n[qi]) continue;
                rows[cnt++] = cache_row(q_seq[qi], s, seq_row0, page_table,
                                        max_pages, page_size);
            }
            for (int32_t d = 0; d < d_v; ++d) o[d] = 0.0;
            if (cnt == 0) {
                lse[(int64_t)qi * h + hh] = -INFINITY;
                free(S); free(rows);
                continue;
            }
            double m = -INFINITY;
            for (int32_t i = 0; i < cnt; ++i) {
                const uint8_t *c = kv8 + rows[i] * kv8_row_bytes;
                const double sc = (double)kv_scale[rows[i]];
                double dot = 0.0;
                for (int32_t d = 0; d < d_qk; ++d)
                    dot += dsa_oracle_bf16_to_f64(qv[d]) * (dsa_oracle_e4m3_to_f64(c[d]) * sc);
                S[i] = scale * dot;
                if (S[i] > m) m = S[i];
            }
            double denom = 0.0;
            for (int32_t i = 0; i < cnt; ++i) {
                double p = exp(S[i] - m);
                const uint8_t *c = kv8 + rows[i] * kv8_row_bytes;
                const double sc = (double)kv_scale[rows[i]];
                denom += p;
                for (int32_t d = 0; d < d_v; ++d) o[d] += p * (dsa_oracle_e4m3_to_f64(c[d]) * sc);
            }
            for (int32_t d = 0; d < d_v; ++d) o[d] /= denom;
            lse[(int64_t)qi * h + hh] = m + log(denom);
            free(S);
            free(rows);
        }
    }
    return bad ? -2 : 0;
}

/* Dense attention over the whole visible history 0..q_n-1, with no index
 * list: the textbook MQA softmax attention.  When the history has at most k
 * positions DSA keeps all of them ([yuyanqi] section 3.3), so the sparse path
 * must reproduce this. */
int dsa_oracle_dense_mla(int32_t nq, int32_t h, int32_t d_qk, int32_t d_v,
                         double scale, const uint16_t *q, const uint16_t *kv,
                         int64_t kv_row_stride, const int32_t *q_seq,
                         const int32_t *q_n, const int64_t *seq_row0,
                         const int32_t *page_table, int32_t max_pages,
                         int32_t page_size, double *out, double *lse,
                         int32_t nthreads)
{
    if (nq < 0 || h <= 0 || d_qk <= 0 || d_v <= 0 || d_v > d_qk) return -1;
    set_threads(nthreads);
    int bad = 0;
#pragma omp parallel for collapse(2) schedule(dynamic, 1) reduction(| : bad)
    for (int32_t qi = 0; qi < nq; ++qi) {
        for (int32_t hh = 0; hh < h; ++hh) {
            int64_t n = q_n[qi];
            const uint16_t *qv = q + ((int64_t)qi * h + hh) * d_qk;
            double *o = out + ((int64_t)qi * h + hh) * d_v;
            for (int32_t d = 0; d < d_v; ++d) o[d] = 0.0;
            if (n <= 0) { lse[(int64_t)qi * h + hh] = -INFINITY; continue; }
            double *logit = (double *)malloc((size_t)n * sizeof(double));
            if (!logit) { bad |= 1; continue; }
            for (int64_t s = 0; s < n; ++s) {
                const uint16_t *c = kv + cache_row(q_seq[qi], s, seq_row0, page_table,
                                                   max_pages, page_size) * kv_row_stride;
                double dot = 0.0;
                for (int32_t d = 0; d < d_qk; ++d)
                    dot += dsa_oracle_bf16_to_f64(qv[d]) * dsa_oracle_bf16_to_f64(c[d]);
                logit[s] = scale * dot;
            }
            double m = logit[0];
            for (int64_t s = 1; s < n; ++s) if (logit[s] > m) m = logit[s];
            double z = 0.0;
            for (int64_t s = 0; s < n; ++s) {
                const uint16_t *c = kv + cache_row(q_seq[qi], s, seq_row0, page_table,
                                                   max_pages, page_size) * kv_row_stride;
                double p = exp(logit[s] - m);
                z += p;
                for (int32_t d = 0; d < d_v; ++d) o[d] += p * dsa_oracle_bf16_to_f64(c[d]);
            }
            for (int32_t d = 0; d < d_v; ++d) o[d] /= z;
            lse[(int64_t)qi * h + hh] = m + log(z);
            free(logit);
        }
    }
    return bad ? -2 : 0;
}

/* ------------------------------------------------------------------------- */
/* The three steps composed (one decode step of the attention layer)           */
/* ------------------------------------------------------------------------- */

/* Score -> TopK -> sparse attention, in the order of the decode data flow of
 * [yuyanqi] section 5.1.  A query whose history fits in k skips scoring and
 * keeps every position ([yuyanqi] section 4.5).  idx_out: [nq, k]. */
int dsa_oracle_forward(int32_t nq, int32_t h_idx, int32_t d_idx, int32_t h,
                       int32_t d_qk, int32_t d_v, int32_t k, double scale,
                       const uint8_t *q_idx, const uint16_t *w,
                       const uint8_t *kidx, const float *k_scale,
                       const uint16_t *q, const uint16_t *kv,
                       int64_t kv_row_stride, const int32_t *q_seq,
                       const int32_t *q_n, const int64_t *seq_row0,
                       const int32_t *page_table, int32_t max_pages,
                       int32_t page_size, int32_t *idx_out, double *out,
                       double *lse, int32_t nthreads)
{
    if (nq < 0 || k <= 0) return -1;
    for (int32_t qi = 0; qi < nq; ++qi) {
        int64_t n = q_n[qi];
        int32_t *row_idx = idx_out + (int64_t)qi * k;
        if (n <= k) {
            if (dsa_oracle_topk(n, NULL, k, row_idx, NULL) != 0) return -1;
            continue;
        }
        double *sc = (double *)malloc((size_t)n * sizeof(double));
        if (!sc) return -2;
        int rc = dsa_oracle_indexer_scores(1, h_idx, d_idx,
                                           q_idx + (int64_t)qi * h_idx * d_idx,
                                           w + (int64_t)qi * h_idx, kidx, k_scale,
                                           q_seq + qi, q_n + qi, seq_row0,
                                           page_table, max_pages, page_size, sc,
                                           NULL, n, nthreads);
        if (rc == 0) rc = dsa_oracle_topk(n, sc, k, row_idx, NULL);
        free(sc);
        if (rc != 0) return rc;
    }
    return dsa_oracle_sparse_mla(nq, h, d_qk, d_v, scale, q, kv, kv_row_stride,
                                 q_seq, q_n, seq_row0, page_table, max_pages,
                                 page_size, idx_out, k, out, lse, nthreads);
}

/* ------------------------------------------------------------------------- */
/* The indexer's training signal, forward only                                 */
/* ------------------------------------------------------------------------- */

/* Indexer distillation loss of each query t ([marsggbo] section 5.1 and 5.2):
 * over a set of positions T_t (the dense stage: every visible s < q_n[t],
 * when idx is NULL; the sparse stage: the valid entries of idx[t, :], a
 * position listed twice counting twice),
 *   A_h[s] = exp(S_h[s]) / sum_{s' in T_t} exp(S_h[s']),
 *            S_h[s] = scale * q[t, h] . c[s]        (each head's attention)
 *   p[s]   = sum_h A_h[s] / sum_{s' in T_t} sum_h A_h[s']
 *            (the heads' scores summed over the head dimension, then L1-
 *            normalised along the sequence)
 *   r[s]   = exp(I[t, s]) / sum_{s' in T_t} exp(I[t, s'])   (softmax of the
 *            index scores over the same set)
 *   kl[t]  = sum_{s in T_t} p[s] * (ln p[s] - ln r[s])      (0 ln 0 = 0)
 * Reading where the page is silent: in the sparse stage the main model
 * attends to T_t only, so each head's distribution is normalised over T_t.
 * index_scores [nq, ld] holds I[t, s] at column s (fp64); p_out, when not
 * NULL, receives p[s] at column s ([nq, ld]; other columns 0).  A query with
 * an empty set gets kl = 0. */
int dsa_oracle_index_kl(int32_t nq, int32_t h, int32_t d_qk, double scale, const uint16_t *q,
                        const uint16_t *kv, int64_t kv_row_stride, const int32_t *q_seq,
                        const int32_t *q_n, const int64_t *seq_row0, const int32_t *page_table,
                        int32_t max_pages, int32_t page_size, const double *index_scores,
                        int64_t ld, const int32_t *idx, int32_t k, double *kl, double *p_out,
                        int32_t nthreads)
{
    if (nq < 0 || h <= 0 || d_qk <= 0 || ld < 0 || (idx && k < 0)) return -1;
    set_threads(nthreads);
    int bad = 0;
#pragma omp parallel for schedule(dynamic, 1) reduction(| : bad)
    for (int32_t qi = 0; qi < nq; ++qi) {
        int64_t n = q_n[qi];
        int64_t cap = idx ? k : n;
        int64_t *pos = (int64_t *)malloc((size_t)(cap > 0 ? cap : 1) * sizeof(int64_t));
        double *S = (double *)malloc((size_t)(cap > 0 ? cap : 1) * sizeof(double));
        double *a = (double *)malloc((size_t)(cap > 0 ? cap : 1) * sizeof(double));
        if (!pos || !S || !a) { bad |= 1; free(pos); free(S); free(a); continue; }
        int64_t cnt = 0;
        if (idx) {
            for (int32_t i = 0; i < k; ++i) {
                int32_t sv = idx[(int64_t)qi * k + i];
                if (sv >= 0 && sv < n && sv < ld) pos[cnt++] = sv;
            }
        } else {
            for (int64_t sv = 0; sv < n && sv < ld; ++sv) pos[cnt++] = sv;
        }
        if (p_out)
            for (int64_t c = 0; c < ld; ++c) p_out[(int64_t)qi * ld + c] = 0.0;
        if (cnt == 0) {
            kl[qi] = 0.0;
            free(pos); free(S); free(a);
            continue;
        }
        for (int64_t i = 0; i < cnt; ++i) a[i] = 0.0;
        /* each head's distribution over the set, summed over heads */
        for (int32_t hh = 0; hh < h; ++hh) {
            const uint16_t *qv = q + ((int64_t)qi * h + hh) * d_qk;
            double m = -INFINITY;
            for (int64_t i = 0; i < cnt; ++i) {
                const uint16_t *c = kv + cache_row(q_seq[qi], pos[i], seq_row0, page_table,
                                                   max_pages, page_size) * kv_row_stride;
                double dot = 0.0;
                for (int32_t d = 0; d < d_qk; ++d)
                    dot += dsa_oracle_bf16_to_f64(qv[d]) * dsa_oracle_bf16_to_f64(c[d]);
                S[i] = scale * dot;
                if (S[i] > m) m = S[i];
            }
            double z = 0.0;
            for (int64_t i = 0; i < cnt; ++i) z += exp(S[i] - m);
            for (int64_t i = 0; i < cnt; ++i) a[i] += exp(S[i] - m) / z;
        }
        /* L1 normalisation along the sequence */
        double asum = 0.0;
        for (int64_t i = 0; i < cnt; ++i) asum += a[i];
        /* softmax of the index scores over the same set */
        const double *I = index_scores + (int64_t)qi * ld;
        double mi = -INFINITY;
        for (int64_t i = 0; i < cnt; ++i)
            if (I[pos[i]] > mi) mi = I[pos[i]];
        double zi = 0.0;
        for (int64_t i = 0; i < cnt; ++i) zi += exp(I[pos[i]] - mi);
        const double lse_i = mi + log(zi);
        double acc = 0.0;
        for (int64_t i = 0; i < cnt; ++i) {
            double p = a[i] / asum;
            if (p_out) p_out[(int64_t)qi * ld + pos[i]] += p;
            if (p > 0.0) acc += p * (log(p) - (I[pos[i]] - lse_i));
        }
        kl[qi] = acc;
        free(pos); free(S); free(a);
    }
    return bad ? -2 : 0;
}

/* ------------------------------------------------------------------------- */
/* Short prefill: the selection applied as a mask to dense MHA attention       */
/* ------------------------------------------------------------------------- */

/* For short prompts the DSA prefill runs as multi-head attention (each head
 * with its own key and value: the MHA form of MLA used for prefill,
 * [marsggbo] section 4) over every visible position, with a mask that keeps
 * only what the indexer selected ([marsggbo] section 6: masked MHA emulates
 * DSA for short-sequence prefill; [aicoding] section 4.3: masked MHA below
 * 8K tokens).  For query t and head h:
 *   keep[s] = s < q_n[t] and s is listed in idx[t, :]   (idx NULL: s < q_n[t])
 *   S[s]    = scale * sum_{d < d_qk} q[t,h,d] * k[s,h,d]
 *   out     = sum_{s kept} exp(S[s] - m) v[s,h,:] / sum_{s kept} exp(S[s] - m)
 *   lse     = m + ln sum_{s kept} exp(S[s] - m),   m = max_{s kept} S[s]
 * A mask holds membership, so a position listed twice is kept once; entries
 * < 0 or >= q_n[t] are ignored.  Nothing kept: out = 0, lse = -inf.
 * k [rows, h, d_qk] and v [rows, h, d_v] bf16; position s of sequence b is
 * row seq_row0[b] + s. */
int dsa_oracle_masked_mha(int32_t nq, int32_t h, int32_t d_qk, int32_t d_v, double scale,
                          const uint16_t *q, const uint16_t *k, const uint16_t *v,
                          const int32_t *q_seq, const int32_t *q_n, const int64_t *seq_row0,
                          const int32_t *idx, int32_t topk, double *out, double *lse,
                          int32_t nthreads)
{
    if (nq < 0 || h <= 0 || d_qk <= 0 || d_v <= 0 || (idx && topk < 0)) return -1;
    set_threads(nthreads);
    int bad = 0;
#pragma omp parallel for schedule(dynamic, 1) reduction(| : bad)
    for (int32_t t = 0; t < nq; ++t) {
        const int64_t n = q_n[t];
        unsigned char *keep = (unsigned char *)calloc((size_t)(n > 0 ? n : 1), 1);
        double *S = (double *)malloc((size_t)(n > 0 ? n : 1) * sizeof(double));
        if (!keep || !S) { bad |= 1; free(keep); free(S); continue; }
        if (idx) {
            for (int32_t i = 0; i < topk; ++i) {
                const int32_t sv = idx[(int64_t)t * topk + i];
                if (sv >= 0 && sv < n) keep[sv] = 1;
            }
        } else {
            for (int64_t sv = 0; sv < n; ++sv) keep[sv] = 1;
        }
        const int64_t row0 = seq_row0[q_seq[t]];
        for (int32_t hh = 0; hh < h; ++hh) {
            const uint16_t *qv = q + ((int64_t)t * h + hh) * d_qk;
            double m = -INFINITY;
            for (int64_t sv = 0; sv < n; ++sv) {
                if (!keep[sv]) continue;
                const uint16_t *kr = k + ((row0 + sv) * h + hh) * d_qk;
                double dot = 0.0;
                for (int32_t d = 0; d < d_qk; ++d)
                    dot += dsa_oracle_bf16_to_f64(qv[d]) * dsa_oracle_bf16_to_f64(kr[d]);
                S[sv] = scale * dot;
                if (S[sv] > m) m = S[sv];
            }
            double *o = out + ((int64_t)t * h + hh) * d_v;
            for (int32_t d = 0; d < d_v; ++d) o[d] = 0.0;
            if (m == -INFINITY) {
                lse[(int64_t)t * h + hh] = -INFINITY;
                continue;
            }
            double z = 0.0;
            for (int64_t sv = 0; sv < n; ++sv) {
                if (!keep[sv]) continue;
                const double e = exp(S[sv] - m);
                const uint16_t *vr = v + ((row0 + sv) * h + hh) * d_v;
                z += e;
                for (int32_t d = 0; d < d_v; ++d) o[d] += e * dsa_oracle_bf16_to_f64(vr[d]);
            }
            for (int32_t d = 0; d < d_v; ++d) o[d] /= z;
            lse[(int64_t)t * h + hh] = m + log(z);
        }
        free(keep);
        free(S);
    }
    return bad ? -2 : 0;
}

/* ------------------------------------------------------------------------- */
/* Next step on the path: the indexer's q^I / k^I / w producer                 */
/* ------------------------------------------------------------------------- */

/* The indexer's own projections, per token t ([yuyanqi] sections 4.1-4.3):
 *   q^I[t]   = W_qb . q_lora[t], reshaped to [H_I, d_I]        (wq_b)
 *   k^I[t]   = LayerNorm(W_k . x[t])                            (wk, k_norm)
 *   the first rope_dim dims of every q^I head and of k^I get the indexer's
 *   own RoPE at the token's position (split [rope_head_dim, ...], then
 *   rotary_emb(positions, q_rope, k_rope))
 *   w[t]     = (W_proj . x[t]) * H_I^-1/2 * d_I^-1/2 * q_scale   (weights_proj,
 *              the n_heads^-0.5 and softmax_scale factors, the q scale)
 * then q^I and k^I go to FP8 with a scale ("q_scale" folded into w; "k_s",
 * e8m0, multiplying the score).
 *
 * Readings where the pages are silent: linear layers are y = W x with W
 * stored [out, in] (bf16), x bf16; LayerNorm is (k - mean) / sqrt(var + eps)
 * * gamma + beta with the biased variance; RoPE rotates the pairs (2i, 2i+1)
 * of the rope dims by pos * theta^(-2i / rope_dim) (the rotary embedding's
 * own definition); both scales are powers of two (the e8m0 of k_s, and the
 * same for q so that folding it into w is exact): s = 2^ceil(log2(amax /
 * 448)), 1 when amax = 0, one per (token, head) for q and one per token for
 * k; codes = e4m3(value / s).  w is then rounded to bf16.
 *
 * Outputs (any may be NULL): q_f [nt, H_I, d_I] and k_f [nt, d_I] (fp64,
 * after RoPE, before quantisation), w_f [nt, H_I] (fp64, folded), q_code /
 * q_scale, k_code / k_scale (the FP8 codes and their scales), w_bf16. */
static double bf(const uint16_t *p, int64_t i) { return dsa_oracle_bf16_to_f64(p[i]); }

/* The power-of-two quantisation scale of a vector whose largest magnitude is
 * amax: the smallest 2^e with amax / 2^e <= 448 (the E4M3 maximum), 1 for an
 * all-zero vector. */
double dsa_oracle_pow2_scale(double amax)
{
    if (!(amax > 0.0)) return 1.0;
    return ldexp(1.0, (int)ceil(log2(amax / 448.0)));
}

/* bfloat16 nearest to v (ties to even), rounded once from fp64: 8
 * significant bits, spacing 2^(e-7) for |v| in [2^e, 2^(e+1)), 2^-133 below
 * the smallest normal; beyond the largest finite value -> infinity. */
uint16_t dsa_oracle_f64_to_bf16(double v)
{
    if (isnan(v)) return 0x7FC0;
    double a = fabs(v);
    double r = 0.0;
    if (a > 0.0) {
        int e;
        frexp(a, &e);        /* a = f * 2^e, f in [0.5, 1): a in [2^(e-1), 2^e) */
        int lo = e - 1 - 7;  /* spacing exponent of the 8-significant-bit grid */
        if (lo < -133) lo = -133;
        r = ldexp(rint(ldexp(a, -lo)), lo);  /* rint: ties to even */
        if (r > ldexp(255.0, 120)) r = INFINITY;  /* largest finite: (2 - 2^-7) * 2^127 */
    }
    float f = (float)(signbit(v) ? -r : r);  /* exact: r has at most 8 significant bits */
    uint32_t u;
    memcpy(&u, &f, sizeof u);
    return (uint16_t)(u >> 16);
}

/* FP8 quantisation of `rows` vectors of d values each (row-major v): one
 * power-of-two scale per row from its largest magnitude, codes =
 * e4m3(v / scale) ([yuyanqi] section 4.3: q and k in FP8 with a scale; the
 * e8m0 k_s).  scales[r] = the row's scale; codes [rows, d]. */
int dsa_oracle_quantize_rows(int64_t rows, int32_t d, const double *v, uint8_t *codes, float *scales)
{
    if (rows < 0 || d <= 0) return -1;
    for (int64_t r = 0; r < rows; ++r) {
        const double *x = v + r * d;
        double amax = 0.0;
        for (int32_t o = 0; o < d; ++o) amax = fmax(amax, fabs(x[o]));
        double s = dsa_oracle_pow2_scale(amax);
        if (scales) scales[r] = (float)s;
        if (codes)
            for (int32_t o = 0; o < d; ++o) codes[r * d + o] = dsa_oracle_f64_to_e4m3(x[o] / s);
    }
    return 0;
}

/* The indexer's head weights with every constant folded in ([yuyanqi]
 * section 4.3: weights_proj * n_heads^-1/2 * softmax_scale * q_scale), for
 * n tokens: w[t, j] = wp[t, j] / sqrt(H_I) / sqrt(d_I) * q_scale[t, j],
 * then rounded to bf16 (ties to even).  Either output may be NULL. */
int dsa_oracle_fold_weights(int64_t n, int32_t h_idx, int32_t d_idx, const double *wp,
                            const float *q_scale, double *w_f, uint16_t *w_bf16)
{
    if (n < 0 || h_idx <= 0 || d_idx <= 0) return -1;
    for (int64_t i = 0; i < n * h_idx; ++i) {
        double wv = wp[i] / sqrt((double)h_idx) / sqrt((double)d_idx) * (double)q_scale[i];
        if (w_f) w_f[i] = wv;
        if (w_bf16) w_bf16[i] = dsa_oracle_f64_to_bf16(wv);
    }
    return 0;
}

static void rope_rotate(double *v, int32_t rope_dim, int32_t pos, double theta)
{
    for (int32_t i = 0; i < rope_dim / 2; ++i) {
        double ang = (double)pos * pow(theta, -2.0 * (double)i / (double)rope_dim);
        double c = cos(ang), sn = sin(ang);
        double x0 = v[2 * i], x1 = v[2 * i + 1];
        v[2 * i] = x0 * c - x1 * sn;
        v[2 * i + 1] = x0 * sn + x1 * c;
    }
}

int dsa_oracle_indexer_project(int32_t nt, int32_t hidden, int32_t q_lora_rank,
                               int32_t h_idx, int32_t d_idx, int32_t rope_dim,
                               const uint16_t *x, const uint16_t *q_lora,
                               const uint16_t *w_qb, const uint16_t *w_k,
                               const uint16_t *w_proj, const float *ln_gamma,
                               const float *ln_beta, double ln_eps,
                               const int32_t *positions, double rope_theta,
                               double *q_f, double *k_f, double *w_f,
                               uint8_t *q_code, float *q_scale,
                               uint8_t *k_code, float *k_scale,
                               uint16_t *w_bf16, int32_t nthreads)
{
    if (nt < 0 || hidden <= 0 || q_lora_rank <= 0 || h_idx <= 0 || d_idx <= 0) return -1;
    if (h_idx > 256 || d_idx > 256) return -1;
    if (rope_dim < 0 || rope_dim > d_idx || (rope_dim & 1)) return -1;
    set_threads(nthreads);
    int rc = 0;
#pragma omp parallel for schedule(dynamic, 1)
    for (int32_t t = 0; t < nt; ++t) {
        double *qv = (double *)malloc((size_t)h_idx * d_idx * sizeof(double));
        double *kv = (double *)malloc((size_t)d_idx * sizeof(double));
        if (!qv || !kv) {
            free(qv);
            free(kv);
            rc = -2;
            continue;
        }
        /* q^I = W_qb . q_lora, one output row at a time */
        for (int64_t o = 0; o < (int64_t)h_idx * d_idx; ++o) {
            double acc = 0.0;
            for (int32_t r = 0; r < q_lora_rank; ++r)
                acc += bf(w_qb, o * q_lora_rank + r) * bf(q_lora, (int64_t)t * q_lora_rank + r);
            qv[o] = acc;
        }
        /* k^I = LayerNorm(W_k . x) */
        for (int32_t o = 0; o < d_idx; ++o) {
            double acc = 0.0;
            for (int32_t i = 0; i < hidden; ++i)
                acc += bf(w_k, (int64_t)o * hidden + i) * bf(x, (int64_t)t * hidden + i);
            kv[o] = acc;
        }
        double mean = 0.0, var = 0.0;
        for (int32_t o = 0; o < d_idx; ++o) mean += kv[o];
        mean /= d_idx;
        for (int32_t o = 0; o < d_idx; ++o) var += (kv[o] - mean) * (kv[o] - mean);
        var /= d_idx;
        for (int32_t o = 0; o < d_idx; ++o)
            kv[o] = (kv[o] - mean) / sqrt(var + ln_eps) * (double)ln_gamma[o] + (double)ln_beta[o];
        /* RoPE on the first rope_dim dims of every q head and of k */
        for (int32_t j = 0; j < h_idx; ++j) rope_rotate(qv + (int64_t)j * d_idx, rope_dim, positions[t], rope_theta);
        rope_rotate(kv, rope_dim, positions[t], rope_theta);
        /* k: one power-of-two scale per token */
        uint8_t kc[256];
        float ks;
        dsa_oracle_quantize_rows(1, d_idx, kv, kc, &ks);
        for (int32_t o = 0; o < d_idx; ++o) {
            if (k_f) k_f[(int64_t)t * d_idx + o] = kv[o];
            if (k_code) k_code[(int64_t)t * d_idx + o] = kc[o];
        }
        if (k_scale) k_scale[t] = ks;
        /* q: one power-of-two scale per (token, head); w folds it */
        double wps[256], wfs[256];
        float qss[256];
        uint16_t wbs[256];
        for (int32_t j = 0; j < h_idx; ++j) {
            const double *qh = qv + (int64_t)j * d_idx;
            uint8_t qc[256];
            dsa_oracle_quantize_rows(1, d_idx, qh, qc, &qss[j]);
            double wp = 0.0;
            for (int32_t i = 0; i < hidden; ++i)
                wp += bf(w_proj, (int64_t)j * hidden + i) * bf(x, (int64_t)t * hidden + i);
            wps[j] = wp;
            int64_t tj = (int64_t)t * h_idx + j;
            if (q_scale) q_scale[tj] = qss[j];
            for (int32_t o = 0; o < d_idx; ++o) {
                if (q_f) q_f[tj * d_idx + o] = qh[o];
                if (q_code) q_code[tj * d_idx + o] = qc[o];
            }
        }
        dsa_oracle_fold_weights(1, h_idx, d_idx, wps, qss, wfs, wbs);
        for (int32_t j = 0; j < h_idx; ++j) {
            int64_t tj = (int64_t)t * h_idx + j;
            if (w_f) w_f[tj] = wfs[j];
            if (w_bf16) w_bf16[tj] = wbs[j];
        }
        free(qv);
        free(kv);
    }
    return rc;
}
