/*
 * dsa.h -- C ABI of the B200 (sm_100a) DeepSeek Sparse Attention decode path.
 *
 * The path has three steps (DSA blog by marsggbo, section 3; "DeepSeekV3.2之DSA"
 * by yuyanqi, sections 3-5):
 *   1. lightning-indexer score  I[t,s] = sum_j w[t,j] * ReLU(q^I[t,j] . k^I[s])
 *   2. per-query TopK of I[t, 0..n-1]; every position when n <= k
 *   3. MQA-mode MLA attention of all query heads over the selected latent rows,
 *      softmax(q . [c_kv; k_pe]^T) . c_kv
 *
 * Conventions shared by every call
 *   - Pointers.  Every tensor argument is a DEVICE pointer owned by the caller.
 *     The library allocates no device memory; scratch comes from the caller's
 *     `ws` buffer of at least dsa_workspace_size() bytes, 256-byte aligned and
 *     zero-filled before its first use (its first word is the status word;
 *     every call leaves the rest of ws ready for the next call).
 *     `dsa_params` and `dsa_kv` themselves are host structs (their pointer
 *     members are device pointers).
 *   - Streams.  `stream` is a cudaStream_t passed as void* (NULL = legacy
 *     default stream).  Calls only enqueue work and return; nothing
 *     synchronises implicitly.
 *   - Errors.  Every call returns a dsa_status.  Host-side validation failures
 *     launch nothing.  Problems only the device can see (an index >= n, a
 *     bounded wait that expired) are recorded in a status word inside `ws`;
 *     dsa_check_status() synchronises the stream and returns (then clears) it.
 *     dsa_last_error() gives a thread-local message for the last failure.
 *   - Threads.  Calls are stateless and re-entrant; concurrent calls must use
 *     distinct workspaces.
 *   - Layouts.  Row-major, innermost dimension last, densely packed unless a
 *     stride argument says otherwise.  FP8 is OCP E4M3 ("fn": max 448, no inf),
 *     bf16 is the upper half of binary32.
 */
#ifndef DSA_B200_H
#define DSA_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    DSA_OK = 0,
    DSA_ERR_INVALID_ARG = -1,  /* a pointer, size or shape is invalid; nothing launched */
    DSA_ERR_UNSUPPORTED = -2,  /* valid but outside what this build implements */
    DSA_ERR_CUDA = -3,         /* a CUDA runtime/driver call failed */
    DSA_ERR_WORKSPACE = -4,    /* ws is NULL, misaligned or smaller than required */
    DSA_ERR_TIMEOUT = -5,      /* device: a bounded wait expired (the work was abandoned) */
    DSA_ERR_DEVICE_CHECK = -6  /* device: an input failed a check (e.g. index >= n) */
} dsa_status;

/* Problem shape.
 *   nq         query tokens in the batch (>= 0)
 *   h_idx      indexer heads H_I, 1..64 ("index_n_heads", yuyanqi section 3.1)
 *   d_idx      indexer head dim d_I: 64 or 128
 *   h          attention heads, 1..128 (all share one latent row: MQA mode,
 *              marsggbo section 4)
 *   d_qk       key width: 576 (512 latent + 64 rope, yuyanqi section 5.1)
 *   d_v        value width: 512 (the first d_v columns of the same row)
 *   topk       k, 1..2048 (DeepSeek-V3.2 uses 2048, marsggbo section 3)
 *   max_n      an upper bound of every q_n (host-known; sizes the launch grid
 *              and the workspace); 0 <= q_n[i] <= max_n <= 2^27
 *   q_per_seq  queries are in blocks of q_per_seq consecutive queries that
 *              read the same sequence (1 for plain decode, 2 for next token +
 *              one speculative token, L for a prefill of L tokens); the
 *              indexer shares each k^I tile among the queries of a block
 *   scale      softmax scale applied to q . c (576^-0.5 in the workloads)
 */
typedef struct {
    int32_t nq;
    int32_t h_idx;
    int32_t d_idx;
    int32_t h;
    int32_t d_qk;
    int32_t d_v;
    int32_t topk;
    int32_t max_n;
    int32_t q_per_seq;
    float scale;
} dsa_params;

/* Where each query's history lives.  The FP8 index-K cache and the bf16
 * latent cache are indexed by the same token positions (yuyanqi section 5.2,
 * item 3): logical position s of sequence b is cache row
 *   contiguous (page_table == NULL):  seq_row0[b] + s
 *   paged      (page_table != NULL):  page_table[b * max_pages + s / page_size]
 *                                        * page_size + s % page_size
 *   q_seq      [nq] int32, device: sequence of each query
 *   q_n        [nq] int32, device: visible positions n of each query; the
 *              query sees positions 0..n-1 (s < t of marsggbo section 3 when
 *              the caller sets n = t)
 *   seq_row0   [nseq] int64, device (contiguous layout) or NULL
 *   page_table [nseq, max_pages] int32, device (paged layout) or NULL
 *   max_pages  columns of page_table
 *   page_size  tokens per page: 64 or 128 (paged layout); ignored otherwise
 *   cache_rows rows in each cache (bounds every cache access)
 */
typedef struct {
    const int32_t *q_seq;
    const int32_t *q_n;
    const int64_t *seq_row0;
    const int32_t *page_table;
    int32_t max_pages;
    int32_t page_size;
    int64_t cache_rows;
} dsa_kv;

/* Operation selector for dsa_workspace_size(). */
typedef enum {
    DSA_OP_INDEXER_SCORES = 0,
    DSA_OP_TOPK = 1,
    DSA_OP_INDEXER_TOPK = 2,
    DSA_OP_SPARSE_MLA_DECODE = 3,
    DSA_OP_SPARSE_MLA_PREFILL = 4,
    DSA_OP_FORWARD = 5,
    DSA_OP_INDEX_KL_SPARSE = 6, /* dsa_index_kl with idx (topk entries per query) */
    DSA_OP_INDEX_KL_DENSE = 7,  /* dsa_index_kl without idx (every visible position) */
    DSA_OP_MASKED_MHA = 8       /* dsa_masked_mha_prefill */
} dsa_op;

/* Bytes of scratch `ws` the given operation needs for this shape (host only,
 * no CUDA call).  `kv` may be NULL for DSA_OP_TOPK.  Returns
 * DSA_ERR_INVALID_ARG for a shape the operation rejects. */
int dsa_workspace_size(const dsa_params *p, const dsa_kv *kv, int op, size_t *bytes);

/* Step 1 alone: the lightning-indexer score of every visible position,
 * written to HBM (index-score equation, marsggbo section 3; FP8 kernel
 * comment of yuyanqi section 4.3: fp8 q.k -> fp32 logits, ReLU, * weights,
 * sum over heads, * k_s).
 *   q_idx      [nq, h_idx, d_idx] e4m3
 *   w          [nq, h_idx] bf16; every constant factor (H_I^-1/2, the q
 *              quantisation scale, d_I^-1/2; yuyanqi section 4.3) must already
 *              be folded in: the library applies none
 *   kidx_cache [cache_rows, d_idx] e4m3 index-K cache (one head shared by all
 *              indexer heads), rows 16-byte aligned
 *   k_scale    [cache_rows] fp32 per-row dequantisation scale, or NULL (= 1)
 *   scores     [nq, ld_scores] fp32 output: scores[i, s] for s < q_n[i];
 *              -inf for q_n[i] <= s < ld_scores.  ld_scores >= max_n.
 * Arithmetic: FP8 products are exact; the d_I-term dot products are
 * accumulated in fp32 by the tensor cores; ReLU, * w and the head sum in fp32. */
int dsa_indexer_scores(const dsa_params *p, const dsa_kv *kv, const void *q_idx,
                       const void *w, const void *kidx_cache, const float *k_scale,
                       float *scores, int64_t ld_scores, void *ws, size_t ws_bytes,
                       void *stream);

/* Step 2 alone: per-query TopK of scores already in HBM (marsggbo section 3;
 * indices, not values, as in yuyanqi section 4.4).  For query i with n = q_n[i]:
 * if n <= topk the result is every position 0..n-1 (yuyanqi section 3.3);
 * otherwise the topk positions with the largest score, ties broken toward
 * the lower position.  -0.0 and +0.0 are equal.  Scores must not be NaN.
 *   scores  [nq, ld_scores] fp32 (entries s >= q_n[i] are not read)
 *   q_n     [nq] int32 device
 *   idx     [nq, topk] int32 output: the min(topk, n) selected positions in
 *           ascending order, then -1 (the same output every run)
 *   nsel    [nq] int32 output min(topk, n), or NULL
 * The result is exact: identical scores give identical sets. */
int dsa_topk(const dsa_params *p, const float *scores, int64_t ld_scores,
             const int32_t *q_n, int32_t *idx, int32_t *nsel, void *ws,
             size_t ws_bytes, void *stream);

/* Steps 1 + 2 fused: the scores of a query never leave on-chip memory; only
 * the selected positions reach HBM (the fused logits + TopK path of yuyanqi
 * section 4.4).  Queries with q_n <= topk skip scoring (yuyanqi section 4.5).
 * Arguments as dsa_indexer_scores and dsa_topk.  The selected set is the one
 * dsa_topk returns on the scores dsa_indexer_scores writes, bit for bit. */
int dsa_indexer_topk(const dsa_params *p, const dsa_kv *kv, const void *q_idx,
                     const void *w, const void *kidx_cache, const float *k_scale,
                     int32_t *idx, int32_t *nsel, void *ws, size_t ws_bytes,
                     void *stream);

/* Step 3: sparse MQA-mode MLA attention (u_t = Attn(h_t, {c_s : s in I_t}),
 * marsggbo section 3; softmax(q . [c_kv; k_pe]^T) . c_kv, yuyanqi section 5.1).
 * For every query i and head h, over the valid entries s of idx[i, :]:
 *   S_s = scale * q[i,h,:] . c[s, 0:d_qk];   P = softmax(S)
 *   out[i,h,:] = sum_s P_s c[s, 0:d_v];      lse[i,h] = ln sum_s exp(S_s)
 *   q            [nq, h, d_qk] bf16
 *   kv_cache     latent cache, bf16 rows of d_qk values, row r at element
 *                offset r * kv_row_stride (kv_row_stride >= d_qk, multiple of 8)
 *   idx          [nq, topk] int32 logical positions; -1 entries are skipped;
 *                entries >= q_n[i] are skipped and flag DSA_ERR_DEVICE_CHECK;
 *                a position listed twice counts twice
 *   out          [nq, h, d_v] bf16;  lse [nq, h] fp32 (natural log)
 * A query with no valid entry gets out = 0 and lse = -inf.
 * Arithmetic: bf16 tensor-core products with fp32 accumulation; softmax in
 * fp32; P enters the P.V product as a pair of bf16 tiles (P_hi + P_lo,
 * together exact to about 2^-16).  When a query's rows are split over
 * several CTAs, each split's normalised output is kept in ws as fp16 times
 * a power-of-two scale per 256 value columns (so a finite bf16 latent of any
 * magnitude neither overflows fp16 nor falls under its normal range relative
 * to its half row's largest value) and the splits are merged by their
 * log-sum-exp. */
int dsa_sparse_mla_decode(const dsa_params *p, const dsa_kv *kv, const void *q,
                          const void *kv_cache, int64_t kv_row_stride,
                          const int32_t *idx, void *out, float *lse, void *ws,
                          size_t ws_bytes, void *stream);

/* Step 3 over an FP8 latent cache (half the bytes of every gathered row).
 * The pages give FP8 only for the indexer's keys (e4m3 with a per-row e8m0
 * scale, yuyanqi section 4.3); the latent cache here uses that same format,
 * a reading of ours: row r holds d_qk e4m3 codes and stands for
 *   c[r, d] = e4m3(kv8_cache[r * kv8_row_bytes + d]) * kv_scale[r]
 * with kv_scale[r] a power of two (then every c is exact in bf16 and the
 * result is that of dsa_sparse_mla_decode on the bf16 cache of those values).
 *   kv8_cache     [cache_rows, kv8_row_bytes] e4m3 codes, 16-byte aligned;
 *                 kv8_row_bytes >= 576 and a multiple of 16
 *   kv_scale      [cache_rows] fp32
 * Everything else (arguments, ws, errors, arithmetic) as for
 * dsa_sparse_mla_decode. */
int dsa_sparse_mla_decode_fp8(const dsa_params *p, const dsa_kv *kv, const void *q,
                              const void *kv8_cache, int64_t kv8_row_bytes,
                              const float *kv_scale, const int32_t *idx, void *out,
                              float *lse, void *ws, size_t ws_bytes, void *stream);

/* Step 3 scheduled for many queries of one sequence (causal prefill, where
 * token t sees n = t positions).  Same arguments and results as
 * dsa_sparse_mla_decode. */
int dsa_sparse_mla_prefill(const dsa_params *p, const dsa_kv *kv, const void *q,
                           const void *kv_cache, int64_t kv_row_stride,
                           const int32_t *idx, void *out, float *lse, void *ws,
                           size_t ws_bytes, void *stream);

/* Short prefill as masked MHA: dense multi-head attention over every visible
 * position with the index set applied as a mask, the form the pages give
 * DSA for short prompts (DSA blog by marsggbo, section 6; aicoding.csdn.net
 * DSA article, section 4.3: below 8K tokens).  MHA form of MLA (marsggbo,
 * section 4): every head has its own key and value rows.  For query t, head h:
 *   keep[s] = s < q_n[t] and s listed in idx[t, :]  (idx NULL: every s < q_n[t])
 *   out[t,h] = sum_{s kept} softmax(scale * q[t,h] . k[s,h]) v[s,h]
 *   lse[t,h] = ln sum_{s kept} exp(scale * q[t,h] . k[s,h])
 * A position listed twice is kept once (a mask holds membership); nothing
 * kept gives out = 0 and lse = -inf.
 *   p      d_qk = per-head q/k width (64, 128 or 192), d_v = per-head v width
 *          (64 or 128), h heads, topk = idx columns, max_n >= every q_n
 *          (<= 2^20), q_per_seq: queries come in blocks of q_per_seq
 *          consecutive queries of one sequence (a prefill of L tokens: L);
 *          h_idx / d_idx are not read
 *   kv     q_seq, q_n, seq_row0 (contiguous layout only); cache_rows = rows
 *          of k and v; position s of sequence b is row seq_row0[b] + s (rows
 *          past cache_rows read as zero)
 *   q      [nq, h, d_qk] bf16;  k [cache_rows, h, d_qk] bf16;
 *   v      [cache_rows, h, d_v] bf16 (all 16-byte aligned)
 *   idx    [nq, topk] int32 (e.g. dsa_indexer_topk's output) or NULL;
 *          entries < 0 are skipped, entries >= q_n[t] flag DSA_ERR_DEVICE_CHECK
 *   out    [nq, h, d_v] bf16;  lse [nq, h] fp32
 *   ws     dsa_workspace_size(DSA_OP_MASKED_MHA): the membership bitmap
 * Arithmetic as in dsa_sparse_mla_decode: bf16 products, fp32 accumulation,
 * softmax in fp32 with P as a bf16 pair (P_hi + P_lo). */
int dsa_masked_mha_prefill(const dsa_params *p, const dsa_kv *kv, const void *q, const void *k,
                           const void *v, const int32_t *idx, void *out, float *lse, void *ws,
                           size_t ws_bytes, void *stream);

/* The indexer's training signal, forward only: the distillation loss of each
 * query t (DSA blog by marsggbo, section 5.1 for the dense warm-up, 5.2 for
 * the sparse stage).  Over the set T_t (idx == NULL: every visible position
 * s < q_n[t]; else the valid entries of idx[t, :], a position listed twice
 * counting twice):
 *   A_h[s] = softmax over T_t of scale * q[t, h] . c[s]   (each head's
 *            attention distribution, MQA form as in dsa_sparse_mla_decode)
 *   p[s]   = sum_h A_h[s] / sum_{s' in T_t} sum_h A_h[s']  (summed over
 *            heads, L1-normalised along the sequence)
 *   kl[t]  = sum_{s in T_t} p[s] * (ln p[s] - ln softmax_{T_t}(I[t, .])[s])
 * A query whose set is empty gets kl = 0.  In the sparse stage each head is
 * normalised over T_t, the set the main model attends to (the page does not
 * say; this is the plain reading).
 *   q, kv_cache, kv_row_stride, kv  as for dsa_sparse_mla_decode
 *   index_scores [nq, ld_scores] fp32 (e.g. dsa_indexer_scores' output);
 *                max_n <= ld_scores <= 2^27
 *   idx          [nq, topk] int32 or NULL (the dense stage); entries < 0 are
 *                skipped, entries >= q_n[t] flag DSA_ERR_DEVICE_CHECK
 *   kl           [nq] fp32 output
 *   p_out        [nq, ld_scores] fp32 output or NULL: p[s] at column s,
 *                0 elsewhere (every column of the query's row is written)
 *   ws           dsa_workspace_size(DSA_OP_INDEX_KL_SPARSE, or _DENSE when
 *                idx is NULL)
 * Arithmetic: the attention scores as in dsa_sparse_mla_decode (bf16
 * products, fp32 accumulation, exp in fp32); each head's log-sum-exp is
 * merged over the splits of the set, then the scores are recomputed and
 * exp(S - lse) summed over heads in fp32; the normalisation, the index
 * scores' softmax and the KL sum in fp64. */
int dsa_index_kl(const dsa_params *p, const dsa_kv *kv, const void *q, const void *kv_cache,
                 int64_t kv_row_stride, const float *index_scores, int64_t ld_scores,
                 const int32_t *idx, float *kl, float *p_out, void *ws, size_t ws_bytes,
                 void *stream);

/* Steps 1-3 in one call: fused indexer + TopK, then sparse attention, as in
 * the decode data flow of yuyanqi section 5.1.  idx_out [nq, topk] receives
 * the selected positions (or NULL: they stay in ws).  Arguments as above;
 * page_table may be set (paged caches) or NULL (contiguous caches). */
int dsa_forward(const dsa_params *p, const dsa_kv *kv, const void *q_idx,
                const void *w, const void *kidx_cache, const float *k_scale,
                const void *q, const void *kv_cache, int64_t kv_row_stride,
                void *out, float *lse, int32_t *idx_out, void *ws,
                size_t ws_bytes, void *stream);

/* dsa_forward over paged caches (sglang's paged TopK path named in yuyanqi
 * section 4.4): kv->page_table must be non-NULL. */
int dsa_forward_paged(const dsa_params *p, const dsa_kv *kv, const void *q_idx,
                      const void *w, const void *kidx_cache, const float *k_scale,
                      const void *q, const void *kv_cache, int64_t kv_row_stride,
                      void *out, float *lse, int32_t *idx_out, void *ws,
                      size_t ws_bytes, void *stream);

/* The indexer's own inputs, produced from the hidden state and the low-rank
 * query ("DeepSeekV3.2之DSA" by yuyanqi, sections 4.1-4.3), with k^I
 * appended to the index-K cache (the decode data flow of its section 5.1).
 * For every token t:
 *   q^I[t] = W_qb . q_lora[t] as [h_idx, d_idx]             (wq_b)
 *   k^I[t] = LayerNorm(W_k . x[t]) * ln_gamma + ln_beta      (wk, k_norm;
 *            biased variance, epsilon ln_eps)
 *   RoPE on the first rope_dim dims of every q^I head and of k^I: the pair
 *            (2i, 2i+1) rotated by positions[t] * rope_theta^(-2i / rope_dim)
 *   q_scale[t, j] / k_scale = the smallest power of two s with amax / s <= 448
 *            (the e8m0 k_s of section 4.3; per (token, head) for q, per
 *            token for k), codes = e4m3(value / s) (ties to even, saturating)
 *   w[t, j] = (W_proj . x[t])_j / sqrt(h_idx) / sqrt(d_idx) * q_scale[t, j],
 *            rounded to bf16 (weights_proj with n_heads^-1/2, the softmax
 *            scale d_I^-1/2 and the q scale folded in: the form the indexer
 *            score takes, with no factor of its own)
 * Shapes: nt tokens; hidden = width of x, q_lora_rank = width of q_lora (both
 * multiples of 8); h_idx 1..64; d_idx 64 or 128; rope_dim even, <= d_idx. */
typedef struct {
    int32_t nt;
    int32_t hidden;
    int32_t q_lora_rank;
    int32_t h_idx;
    int32_t d_idx;
    int32_t rope_dim;
    float ln_eps;
    float rope_theta;
} dsa_project_params;

/* Bytes of `ws` dsa_indexer_project needs (host only). */
int dsa_project_workspace_size(const dsa_project_params *pp, size_t *bytes);

/* Produce q^I, w and k^I of nt tokens and append k^I to the cache.
 *   kv         where each token's k^I row goes: kv->q_seq [nt] is the token's
 *              sequence and positions[t] its position; the row follows
 *              kv->seq_row0 / kv->page_table as for the score (kv->q_n is not
 *              read).  A row outside [0, cache_rows) flags DSA_ERR_DEVICE_CHECK
 *              and is not written.
 *   x          [nt, hidden] bf16;  q_lora [nt, q_lora_rank] bf16
 *   w_qb       [h_idx * d_idx, q_lora_rank] bf16; w_k [d_idx, hidden] bf16;
 *   w_proj     [h_idx, hidden] bf16  (all [out, in], 16-byte aligned)
 *   ln_gamma, ln_beta [d_idx] fp32;  positions [nt] int32
 *   q_idx      [nt, h_idx, d_idx] e4m3 output (the indexer's q_idx input)
 *   q_scale    [nt, h_idx] fp32 output, or NULL
 *   w          [nt, h_idx] bf16 output (the indexer's w input)
 *   kidx_cache [cache_rows, d_idx] e4m3: row of token t overwritten
 *   k_scale    [cache_rows] fp32: entry of token t's row overwritten (pass the
 *              same array to the score as its k_scale)
 *   q_f32, k_f32, w_f32: [nt, h_idx, d_idx], [nt, d_idx], [nt, h_idx] fp32
 *              outputs of the values before rounding (after RoPE; w before
 *              folding), or NULL
 * Arithmetic: bf16 tensor-core products with fp32 accumulation (a split of
 * the K dimension is summed in a fixed order); LayerNorm and the rounding
 * decisions in fp32, RoPE angles and the weight folding in fp64. */
int dsa_indexer_project(const dsa_project_params *pp, const dsa_kv *kv, const void *x,
                        const void *q_lora, const void *w_qb, const void *w_k, const void *w_proj,
                        const float *ln_gamma, const float *ln_beta, const int32_t *positions,
                        void *q_idx, float *q_scale, void *w, void *kidx_cache, float *k_scale,
                        float *q_f32, float *k_f32, float *w_f32, void *ws, size_t ws_bytes,
                        void *stream);

/* dsa_indexer_topk without a workspace, for callers that cannot allocate
 * device memory (their allocator owns the device, they run under a fixed
 * memory budget, or they must not enter the driver's allocator on this
 * path).  The pages have no counterpart: this is a deployment variant of
 * steps 1 + 2, same arguments and same results as dsa_indexer_topk.
 *   - Scratch lives in one fixed 8 MiB device array inside the library;
 *     every GPU that loads the library holds it until the process exits.
 *     A shape needing more scratch is rejected with DSA_ERR_UNSUPPORTED
 *     before anything is launched.  On a 148-SM B200 a decode batch of
 *     up to 78 queries at 128K context (204 at 32K) fits;
 *     dsa_workspace_size(DSA_OP_INDEXER_TOPK) gives a shape's need.
 *   - The call allocates nothing (no cudaMalloc, no allocating library
 *     call).  The first call on each device resolves the array's device
 *     address (cudaGetSymbolAddress) and keeps it for the life of the
 *     process; make that first call outside any stream capture.  Do not use
 *     this entry point after cudaDeviceReset (or anything else that tears
 *     down the device's primary context): the kept address would be stale.
 *   - All calls share the array and it keeps the last call's contents: the
 *     call clears what must start at zero itself, but calls whose work
 *     overlaps on the GPU (other streams, other threads) race; serialise them.
 *   - status (device int32, nullable) receives the device status word of
 *     this call (DSA_OK, DSA_ERR_TIMEOUT or DSA_ERR_DEVICE_CHECK) in stream
 *     order; dsa_check_status does not apply (there is no ws). */
int dsa_indexer_topk_static(const dsa_params *p, const dsa_kv *kv, const void *q_idx,
                            const void *w, const void *kidx_cache, const float *k_scale,
                            int32_t *idx, int32_t *nsel, int32_t *status, void *stream);

/* Synchronise `stream`, return the device status word stored in `ws`
 * (DSA_OK, DSA_ERR_TIMEOUT or DSA_ERR_DEVICE_CHECK) and clear it. */
int dsa_check_status(void *ws, void *stream);

/* Message describing the last failure on this thread ("" if none). */
const char *dsa_last_error(void);

#ifdef __cplusplus
}
#endif

#endif /* DSA_B200_H */
