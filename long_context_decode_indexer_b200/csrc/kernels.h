// kernels.h -- launch parameters and shared-memory layouts of the kernels,
// shared by the host-side API (dsa_api.cu) and the device code.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace dsa {

// Budget of a bounded wait, in SM clock cycles (about one second at 1.9 GHz).
// A wait that runs out records DSA_ERR_TIMEOUT and abandons the work instead
// of hanging the GPU.
constexpr long long kWaitBudgetCycles = 2000000000LL;
// A merge-mode chunk waits at most this long (about 50 us) for the other
// chunks' histograms; a shorter wait only weakens its candidate bound.
constexpr long long kHistWaitCycles = 100000;

// ---------------------------------------------------------------- indexer
constexpr int kModeFused = 0;   // scores stay on chip, TopK indices written
constexpr int kModeScores = 1;  // scores written to HBM
constexpr int kModeTopk = 2;    // TopK of scores read from HBM

// Indexer stream tuning: whether the SMs a batch of equal chunk counts
// leaves idle give some groups one more chunk (parallel selection only).
#ifndef DSA_K1_FILL_SMS
#define DSA_K1_FILL_SMS 1
#endif
constexpr int kK1MaxStages = 12;     // TMA ring barriers
constexpr int kK1MaxAcc = 4;         // TMEM accumulator buffers (even: one parity per epilogue group)
constexpr int kK1Threads = 352;      // warp 0 TMA, warps 1 and 10 MMA (even / odd tiles), warps 2-5 and 6-9: epilogue
constexpr int kK2Threads = 256;
constexpr int kMaxGroupQueries = 2;  // queries sharing one k^I tile (N <= 2 * 64)
constexpr int kMaxChunks = 32;       // chunks per query group (merge bookkeeping)
constexpr int kKeysBudget = 96 * 1024;  // bytes of on-chip scores per CTA
constexpr int kSelBinsHost = 2048;
constexpr int kK1MiscBytes = 2048;    // barriers, flags and selection scratch of k1 / k2

// Shared words an ordered emission over n elements by `nwarps` warps needs:
// one uint4 of ballots per 128-element step of each warp's slice, then 32
// words of step prefixes per warp (see emit_ordered).
__host__ __device__ constexpr int emit_ballot_words(int n, int nwarps) {
    return 4 * nwarps * ((((n + nwarps - 1) / nwarps + 127) & ~127) / 128) + 32 * nwarps;
}

struct K1Params {
    // inputs
    const uint8_t *q_idx;   // [nq, h_idx, d_idx] e4m3
    const uint16_t *w;      // [nq, h_idx] bf16
    const float *k_scale;   // [cache_rows] or null
    const int32_t *q_seq;
    const int32_t *q_n;
    const int64_t *seq_row0;
    const int32_t *page_table;
    int32_t max_pages;
    int32_t page_size;
    int64_t cache_rows;
    int32_t nq, h_idx, d_idx, topk;
    // work split
    int32_t q_per_seq, qg, groups_per_block, n_groups;
    int32_t P;      // chunks per group: groups [0, n_big) have P, the others P - 1
    int32_t n_big;
    int32_t chunk;  // positions per chunk (multiple of 128)
    int32_t stages; // TMA ring depth (stages of 256 rows)
    int32_t acc_bufs;  // TMEM accumulator buffers of qg*hp columns (2 or 4)
    uint32_t tmem_cols;
    // outputs
    float *scores;  // kModeScores output / kModeTopk input
    int64_t ld;
    int32_t *idx;
    int32_t *nsel;
    // workspace
    uint32_t *ghist;      // [nq, 2048] global top-digit histograms
    uint32_t *gtot;       // [nq] positions counted into ghist so far
    int32_t parallel;     // every CTA is co-resident: each chunk selects its own part exactly
    int32_t wait_hist;    // merge selection with every CTA co-resident: wait (briefly) for the full histogram
    uint64_t *cand;       // [nq, P, cand_stride] candidate composites
    int32_t cand_stride;  // topk rounded up to a multiple of 4 (32-byte aligned chunk lists)
    int32_t *cand_cnt;    // [nq, P]
    int32_t *cand_above;  // [nq, P] (parallel) keys of each chunk above the threshold bin
    uint32_t *published;  // [nq] (parallel) chunks that published their threshold-bin lists
    uint32_t *done;       // [n_groups] chunks finished
    int *status;
    // bounded waits: budget in SM cycles; `inject` (tests only) makes one
    // arrival the first CTA's MMA issuer waits for never happen
    long long wait_budget;
    int32_t inject;
};

struct K1Layout {
    uint32_t stages, qtile, keys, hist, wts, misc, total;
};

__host__ __device__ inline uint32_t align_up(uint32_t x, uint32_t a) { return (x + a - 1) / a * a; }

// Offsets from a 1024-byte aligned base; `total` includes the alignment slack.
// `merge`: the last CTA of a group stages every chunk's candidates (the
// selection used when the grid is not resident at once).
__host__ __device__ inline K1Layout k1_layout(int mode, int di, int qg, int hp, int chunk, int P,
                                              int topk, int stages, bool merge) {
    K1Layout L;
    uint32_t off = 0;
    L.stages = off;
    if (mode != kModeTopk) off += static_cast<uint32_t>(stages) * 128u * static_cast<uint32_t>(di);
    L.qtile = off;
    if (mode != kModeTopk) off += align_up(static_cast<uint32_t>(qg * hp * di), 1024);
    L.keys = off;
    if (mode != kModeScores) off += static_cast<uint32_t>(qg) * static_cast<uint32_t>(chunk) * 4u;
    // the last CTA of a group stages the threshold-bin candidates in the
    // area below the histogram
    if (mode != kModeScores && P > 1 && merge) {
        const uint32_t need = static_cast<uint32_t>(P) * static_cast<uint32_t>(topk + 1) * 8u;
        if (off < need) off = need;
    }
    off = align_up(off, 128);
    L.hist = off;  // radix scratch histogram, then one local histogram per query
    off += (mode != kModeScores) ? static_cast<uint32_t>(qg + 1) * kSelBinsHost * 4u : 0u;
    L.wts = off;
    off += align_up(static_cast<uint32_t>(qg * hp * 4), 16);
    off = align_up(off, 128);
    L.misc = off;
    off += kK1MiscBytes;
    L.total = off + 1024;
    return L;
}

// Dynamic shared memory to request so that no SM can host more CTAs than
// its 512 TMEM columns serve at `tmem_cols` each (tcgen05.alloc then never
// has to wait for another CTA to free columns).
inline size_t smem_for_tmem(size_t want, uint32_t tmem_cols) {
    const size_t kSmemPerSm = 233472, kReserved = 1024;
    const size_t max_ctas = tmem_cols ? 512 / tmem_cols : 32;
    const size_t floor_bytes = kSmemPerSm / (max_ctas + 1) - kReserved + 1;
    return want > floor_bytes ? want : floor_bytes;
}

// pdl: launched as the programmatic dependent of launch_clear (which must
// directly precede it in the stream)
cudaError_t launch_indexer(int mode, int hp, int di, const CUtensorMap &kmap, const K1Params &a,
                           cudaStream_t st, bool pdl);
// zero `bytes` (a multiple of 16, 16-byte aligned) at p with a kernel that
// lets its programmatic dependent start at once
cudaError_t launch_clear(void *p, size_t bytes, cudaStream_t st);
cudaError_t launch_topk(const K1Params &a, cudaStream_t st);

// ------------------------------------------------------ sparse MLA attention
constexpr int kDqk = 576;           // key width (512 latent + 64 rope)
constexpr int kDv = 512;            // value width
constexpr int kMlaHeads = 128;      // MMA M: heads per CTA (zero-padded)
constexpr int kMlaMaxRows = 256;    // KV rows per CTA (split size limit)
constexpr int kMlaStages = 4;       // pass-1 ring depth (Q chunk + K chunk)
constexpr int kMlaVRows = 32;       // rows per pass-2 V tile
constexpr int kMlaVStages = 3;      // pass-2 ring depth
constexpr int kMlaMaxSplits = 32;   // splits per query (the combine kernel's warp reads one LSE per lane)
constexpr int kMlaScaleBlocks = 2;  // power-of-two scales per partial row (one per 256 value columns)
constexpr int kMlaThreads = 320;    // warps 0-3 softmax/epilogue, 4 Q TMA, 5 MMA, 6-9 row gathers (0-3 help in pass 1)

struct MlaParams {
    const int32_t *q_seq;
    const int32_t *q_n;
    const int64_t *seq_row0;
    const int32_t *page_table;
    int32_t max_pages, page_size;
    int64_t cache_rows;
    const int32_t *idx;  // [nq, topk]
    const uint16_t *kv;  // latent cache (bf16 bits)
    int64_t kv_row_stride;  // elements between cache rows
    const uint8_t *kv8;     // FP8 latent cache (e4m3 codes), when the cache is stored in FP8
    const float *kv_scale;  // [cache_rows] power-of-two scale of each FP8 row
    int64_t kv8_row_bytes;  // bytes between FP8 cache rows
    int32_t nq, h, topk;
    int32_t splits;      // CTAs per query along the index list
    int32_t rows_per_split;
    int32_t q0;          // first query of this launch (wave)
    float scale_log2;    // scale * log2(e)
    float scale;
    // outputs
    uint16_t *out;       // [nq, h, d_v] bf16
    float *lse;          // [nq, h]
    uint16_t *part_o;    // [wave_q, splits, 128, d_v] normalised partial outputs / part_scale (fp16 bits)
    float *part_lse;     // [wave_q, splits, 128]
    float *part_scale;   // [wave_q, splits, 128, 2] power of two of each half row of part_o
    int *status;
    long long wait_budget;  // bounded waits, SM cycles
    int32_t inject;         // tests only: the first CTA's gathers skip one arrival
    // indexer distillation loss (the attention's first pass reused)
    int32_t dense;          // entries are positions e (every visible one) instead of idx[q, e]
    int64_t ld;             // columns of iscores / p_out
    float *kl_lse;          // [nq, 128] each head's log-sum-exp over the whole set
    float *kl_a;            // [nq, topk] head-summed attention probability of each entry
    const float *iscores;   // [nq, ld] index scores
    float *kl;              // [nq] the loss
    float *p_out;           // [nq, ld] the target distribution, or null
};

// What the attention kernel computes: the attention itself, or one of the
// two passes of the indexer distillation loss over the same rows.
constexpr int kMlaAttn = 0;
constexpr int kMlaKlStats = 1;  // each (split, head)'s log-sum-exp of the scaled scores
constexpr int kMlaKlSum = 2;    // each entry's attention probability summed over heads

struct MlaLayout {
    uint32_t ring, p_tile, p_lo, v_ring, misc, total;
};

__host__ __device__ inline MlaLayout mla_layout() {
    MlaLayout L;
    // pass 1: kMlaStages x (Q chunk 128x64 bf16 = 16 KB + K chunk 256x64 bf16 = 32 KB)
    const uint32_t stage = 128u * 128u + kMlaMaxRows * 128u;
    const uint32_t pass1 = kMlaStages * stage;
    // pass 2: P as a hi + lo pair of bf16 tiles (128 x 256 each, 64 KB each)
    // + kMlaVStages V tiles (32 rows x 512 bf16 = 32 KB each)
    const uint32_t ptile = 128u * kMlaMaxRows * 2u;
    const uint32_t vtile = kMlaVRows * kDv * 2u;
    L.ring = 0;
    L.p_tile = 0;
    L.p_lo = ptile;
    L.v_ring = 2 * ptile;
    const uint32_t pass2 = 2 * ptile + kMlaVStages * vtile;
    uint32_t end = pass1 > pass2 ? pass1 : pass2;
    L.misc = align_up(end, 128);
    L.total = L.misc + 2048 + 1024;  // barriers and row table, alignment slack
    return L;
}

cudaError_t launch_sparse_mla(const CUtensorMap &qmap, const MlaParams &a, int nq_wave, cudaStream_t st,
                              bool kv8 = false);
cudaError_t launch_mla_combine(const MlaParams &a, int nq_wave, cudaStream_t st);
cudaError_t launch_kl_pass(int mode, const CUtensorMap &qmap, const MlaParams &a, cudaStream_t st);
cudaError_t launch_kl_lse(const MlaParams &a, cudaStream_t st);
cudaError_t launch_kl_reduce(const MlaParams &a, cudaStream_t st);

// --------------------------------------------- masked MHA (short prefill)
// Dense multi-head attention of 128-query tiles over 128-key tiles, the
// index set applied as a membership mask.  One CTA per (query tile, head).
constexpr int kMhaTile = 128;      // queries per CTA (MMA M) and keys per tile (MMA N)
constexpr int kMhaThreads = 320;   // warp 0 TMA, warp 1 MMA, warps 2-9 softmax + epilogue (two per row)
constexpr int kMhaMaxStages = 3;   // K ring depth limit (the V ring has 2 slots)
constexpr int kMhaVStages = 2;

struct MhaParams {
    const int32_t *q_seq;
    const int32_t *q_n;
    const int64_t *seq_row0;
    const uint32_t *mask;   // [nq, mask_words] bit s of row t: s is in t's index set; null: every s < q_n
    int32_t mask_words;     // 4 * ceil(max_n / 128)
    int32_t nq, h, d_qk, d_v;
    int32_t max_n;          // q_n above this flags DSA_ERR_DEVICE_CHECK and is clamped
    int32_t q_per_seq;      // queries are in blocks of q_per_seq of one sequence; a tile stays in its block
    int32_t tiles_per_block;
    float scale_log2;
    uint16_t *out;          // [nq, h, d_v] bf16
    float *lse;             // [nq, h]
    int *status;
    long long wait_budget;
    int32_t stages;         // K ring depth
};

// Q, then a K ring (released as soon as S(j) is computed) and a V ring
// (released after P(j) . V(j)), in 128-row x 64-column swizzled chunks.
struct MhaLayout {
    uint32_t q, k_ring, k_stage, v_ring, v_stage, misc, total;
};

__host__ __device__ inline MhaLayout mha_layout(int d_qk, int d_v, int stages) {
    MhaLayout L;
    const uint32_t chunk = kMhaTile * 128u;  // 128 rows x 64 bf16 columns, 128B-swizzled
    L.q = 0;
    L.k_stage = static_cast<uint32_t>(d_qk / 64) * chunk;
    L.v_stage = static_cast<uint32_t>(d_v / 64) * chunk;
    L.k_ring = L.k_stage;
    L.v_ring = L.k_ring + static_cast<uint32_t>(stages) * L.k_stage;
    L.misc = L.v_ring + kMhaVStages * L.v_stage;
    L.total = L.misc + 4096 + 1024;  // barriers and the softmax exchange, alignment slack
    return L;
}

cudaError_t launch_mha_mask(const int32_t *idx, int topk, const int32_t *q_n, uint32_t *mask, int words, int nq,
                            int *status, cudaStream_t st);
cudaError_t launch_masked_mha(const CUtensorMap &qmap, const CUtensorMap &kmap, const CUtensorMap &vmap,
                              const MhaParams &a, int grid, cudaStream_t st);

// ------------------------------------------------ indexer producer (q^I, k^I, w)
constexpr int kProjMaxStages = 12;  // TMA ring depth limit of the projection GEMM

// Split-K GEMM of both projections: problem 0 = x . [W_k; W_proj]^T
// (N = d_I + H_I), problem 1 = q_lora . W_qb^T (N tiles of 128 rows).
struct ProjGemmParams {
    int32_t nt;              // tokens
    int32_t n_tok;           // tokens per tile (MMA N, a multiple of 16, <= 256)
    int32_t t_tiles;         // token tiles
    int32_t m_tiles[2];      // 128-output tiles per problem (MMA M: weight rows)
    int32_t k_steps[2];      // 64-wide K steps per problem
    int32_t splits[2];       // K slices per problem
    int32_t items0;          // work items of problem 0 (they come first in the grid)
    int32_t d_idx, h_idx;
    int32_t stages;          // TMA ring depth
    uint32_t stage_bytes;    // one stage: 128 weight rows + n_tok token rows, 64 K each
    float *part[2];          // [splits, nt, ld] fp32 partial sums per K slice
    int32_t ld[2];           // row lengths of part
    int *status;
    long long wait_budget;
};

struct ProjEpiParams {
    const float *part0, *part1;
    int32_t splits0, splits1, ld0, ld1;
    int32_t nt, d_idx, h_idx, rope_dim;
    float ln_eps, rope_theta;
    const float *ln_gamma, *ln_beta;  // [d_idx]
    const int32_t *positions;         // [nt]
    const int32_t *q_seq;             // [nt]
    const int64_t *seq_row0;
    const int32_t *page_table;
    int32_t max_pages, page_size;
    int64_t cache_rows;
    uint8_t *kidx_cache;              // [cache_rows, d_idx] e4m3
    float *k_scale;                   // [cache_rows]
    uint8_t *q_idx;                   // [nt, h_idx, d_idx] e4m3
    float *q_scale;                   // [nt, h_idx] or null
    uint16_t *w;                      // [nt, h_idx] bf16
    float *q_f32, *k_f32, *w_f32;     // values before rounding, or null
    int *status;
};

cudaError_t launch_project(const CUtensorMap &x_map, const CUtensorMap &ql_map, const CUtensorMap &wk_map,
                           const CUtensorMap &wp_map, const CUtensorMap &wq_map, const ProjGemmParams &g,
                           const ProjEpiParams &e, cudaStream_t st);

}  // namespace dsa
