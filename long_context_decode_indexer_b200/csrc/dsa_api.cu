// dsa_api.cu -- the C ABI declared in include/dsa.h: argument validation,
// work planning, workspace carving, TMA descriptor encoding and launches.
// Every step of the computation runs in the kernels of indexer.cu and
// sparse_mla.cu; this file only decides shapes and enqueues them.
#include <cuda.h>
#include <cuda_runtime.h>
#include <math.h>
#include <stdarg.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include <mutex>

#include "dsa.h"
#include "kernels.h"

namespace {

thread_local char g_err[512] = "";

int fail(int code, const char *fmt, ...) {
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_err, sizeof g_err, fmt, ap);
    va_end(ap);
    return code;
}

int cuda_fail(cudaError_t e, const char *what) {
    return fail(DSA_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

bool aligned(const void *p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// Test hook for the bounded waits.  DSA_TEST_INJECT_TIMEOUT=indexer (or
// =attention) makes the calls that launch that kernel run it with a short
// wait budget (1e5 SM cycles, ~50 us) and with one arrival its first CTA's
// MMA issuer waits for never made, so the wait runs out: the kernel records
// DSA_ERR_TIMEOUT in the status word, lets its other waits run out the same
// way, waits for its own copies in flight and returns.  Unset, every wait
// has the ~1 s budget and nothing is skipped.
constexpr long long kTestWaitBudget = 100000;

bool inject_timeout(const char *kernel) {
    const char *v = getenv("DSA_TEST_INJECT_TIMEOUT");
    return v != nullptr && strcmp(v, kernel) == 0;
}

// Test hook for callers' error handling: DSA_TEST_INJECT_HOST_ERROR=<step>
// (indexer, attention, index_kl, masked_mha, project, or all) makes that
// step fail on the host with DSA_ERR_CUDA after its arguments were
// validated, before anything is enqueued.  Unset, it does nothing.
int host_fault(const char *step) {
    const char *v = getenv("DSA_TEST_INJECT_HOST_ERROR");
    if (v == nullptr || (strcmp(v, step) != 0 && strcmp(v, "all") != 0)) return DSA_OK;
    return fail(DSA_ERR_CUDA, "injected host failure in %s (DSA_TEST_INJECT_HOST_ERROR)", step);
}

size_t up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// ---------------------------------------------------------------- TMA maps
typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                  const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                  const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    });
    return fn;
}

int make_map_2d(CUtensorMap *m, CUtensorMapDataType dt, const void *ptr, uint64_t inner,
                uint64_t rows, uint64_t row_bytes, uint32_t box_inner, uint32_t box_rows,
                CUtensorMapSwizzle swz) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return fail(DSA_ERR_CUDA, "cuTensorMapEncodeTiled is not available");
    cuuint64_t dims[2] = {inner, rows};
    cuuint64_t strides[1] = {row_bytes};
    cuuint32_t box[2] = {box_inner, box_rows};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = fn(m, dt, 2, const_cast<void *>(ptr), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(DSA_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", static_cast<int>(r));
    return DSA_OK;
}

int make_map_3d(CUtensorMap *m, CUtensorMapDataType dt, const void *ptr, const uint64_t (&dims)[3],
                const uint64_t (&stride_bytes)[2], const uint32_t (&box)[3], CUtensorMapSwizzle swz) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return fail(DSA_ERR_CUDA, "cuTensorMapEncodeTiled is not available");
    cuuint64_t d[3] = {dims[0], dims[1], dims[2]};
    cuuint64_t st[2] = {stride_bytes[0], stride_bytes[1]};
    cuuint32_t bx[3] = {box[0], box[1], box[2]};
    cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = fn(m, dt, 3, const_cast<void *>(ptr), d, st, bx, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, swz,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(DSA_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", static_cast<int>(r));
    return DSA_OK;
}

int num_sms() {
    static int sms = 0;
    static std::once_flag once;
    std::call_once(once, [] {
        int dev = 0;
        if (cudaGetDevice(&dev) == cudaSuccess)
            cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
        if (sms <= 0) sms = 148;
    });
    return sms;
}

// --------------------------------------------------------------- validation
int check_params(const dsa_params *p) {
    if (!p) return fail(DSA_ERR_INVALID_ARG, "params is NULL");
    if (p->nq < 0) return fail(DSA_ERR_INVALID_ARG, "nq < 0");
    if (p->h_idx < 1 || p->h_idx > 64) return fail(DSA_ERR_INVALID_ARG, "h_idx must be in [1, 64]");
    if (p->d_idx != 64 && p->d_idx != 128) return fail(DSA_ERR_INVALID_ARG, "d_idx must be 64 or 128");
    if (p->h < 1 || p->h > 128) return fail(DSA_ERR_INVALID_ARG, "h must be in [1, 128]");
    if (p->d_qk != 576 || p->d_v != 512)
        return fail(DSA_ERR_UNSUPPORTED, "only d_qk = 576 and d_v = 512 are implemented");
    if (p->topk < 1 || p->topk > 2048) return fail(DSA_ERR_INVALID_ARG, "topk must be in [1, 2048]");
    if (p->max_n < 0 || p->max_n > (1 << 27)) return fail(DSA_ERR_INVALID_ARG, "max_n must be in [0, 2^27]");
    if (p->q_per_seq < 1) return fail(DSA_ERR_INVALID_ARG, "q_per_seq must be >= 1");
    if (!isfinite(p->scale)) return fail(DSA_ERR_INVALID_ARG, "scale must be finite");
    return DSA_OK;
}

// The masked-MHA prefill reads d_qk / d_v as the per-head MHA widths.
int check_params_mha(const dsa_params *p) {
    if (!p) return fail(DSA_ERR_INVALID_ARG, "params is NULL");
    if (p->nq < 0) return fail(DSA_ERR_INVALID_ARG, "nq < 0");
    if (p->h < 1 || p->h > (1 << 16)) return fail(DSA_ERR_INVALID_ARG, "h must be in [1, 65536]");
    if (p->d_qk != 64 && p->d_qk != 128 && p->d_qk != 192)
        return fail(DSA_ERR_UNSUPPORTED, "masked MHA: d_qk must be 64, 128 or 192");
    if (p->d_v != 64 && p->d_v != 128) return fail(DSA_ERR_UNSUPPORTED, "masked MHA: d_v must be 64 or 128");
    if (p->topk < 1 || p->topk > 2048) return fail(DSA_ERR_INVALID_ARG, "topk must be in [1, 2048]");
    if (p->max_n < 0 || p->max_n > (1 << 20)) return fail(DSA_ERR_INVALID_ARG, "masked MHA: max_n must be in [0, 2^20]");
    if (p->q_per_seq < 1) return fail(DSA_ERR_INVALID_ARG, "q_per_seq must be >= 1");
    if (!isfinite(p->scale)) return fail(DSA_ERR_INVALID_ARG, "scale must be finite");
    return DSA_OK;
}

int mha_mask_words(const dsa_params *p) { return 4 * ((p->max_n + dsa::kMhaTile - 1) / dsa::kMhaTile); }

int check_kv(const dsa_params *p, const dsa_kv *kv) {
    if (!kv) return fail(DSA_ERR_INVALID_ARG, "kv is NULL");
    if (p->nq > 0 && (!kv->q_seq || !kv->q_n)) return fail(DSA_ERR_INVALID_ARG, "q_seq / q_n are NULL");
    if ((kv->seq_row0 == nullptr) == (kv->page_table == nullptr))
        return fail(DSA_ERR_INVALID_ARG, "exactly one of seq_row0 and page_table must be set");
    if (kv->page_table) {
        if (kv->page_size != 64 && kv->page_size != 128)
            return fail(DSA_ERR_UNSUPPORTED, "page_size must be 64 or 128");
        if (kv->max_pages < 1 || static_cast<int64_t>(kv->max_pages) * kv->page_size < p->max_n)
            return fail(DSA_ERR_INVALID_ARG, "max_pages * page_size < max_n");
    }
    if (kv->cache_rows < 1 || kv->cache_rows >= (int64_t(1) << 31))
        return fail(DSA_ERR_INVALID_ARG, "cache_rows must be in [1, 2^31)");
    return DSA_OK;
}

// ----------------------------------------------------------------- planning
struct IndexerPlan {
    int hp, qg, gpb, n_groups, P, n_big, chunk, stages, acc_bufs;
    bool parallel;  // fused, several chunks, every CTA resident: each chunk selects its own part
    uint32_t tmem_cols;
    size_t smem;
};

int plan_indexer(const dsa_params *p, int mode, int64_t span, IndexerPlan &pl) {
    pl.hp = p->h_idx <= 16 ? 16 : 64;
    if (mode == dsa::kModeTopk) {
        pl.qg = 1;
        pl.gpb = 1;
        pl.n_groups = p->nq;
    } else {
        pl.qg = p->q_per_seq < dsa::kMaxGroupQueries ? p->q_per_seq : dsa::kMaxGroupQueries;
        pl.gpb = (p->q_per_seq + pl.qg - 1) / pl.qg;
        const int nblocks = (p->nq + p->q_per_seq - 1) / p->q_per_seq;
        const int64_t ng = static_cast<int64_t>(nblocks) * pl.gpb;
        if (ng > (int64_t(1) << 24)) return fail(DSA_ERR_UNSUPPORTED, "too many query groups");
        pl.n_groups = static_cast<int>(ng);
    }
    const int64_t sp = span > 0 ? span : 1;
    int64_t chunk_max;
    if (mode == dsa::kModeScores)
        chunk_max = 1 << 20;
    else
        chunk_max = (dsa::kKeysBudget / (4 * pl.qg)) / 128 * 128;
    const int64_t p_min = (sp + chunk_max - 1) / chunk_max;
    const int64_t p_fill = pl.n_groups > 0 ? (num_sms() / pl.n_groups > 1 ? num_sms() / pl.n_groups : 1) : 1;
    const int64_t p_small = (sp + 1023) / 1024;  // no chunk below 1024 positions
    int64_t P = p_fill < p_small ? p_fill : p_small;
    if (P < p_min) P = p_min;
    if (P < 1) P = 1;
    pl.parallel = false;
    pl.n_big = pl.n_groups;
    int64_t p_cut = 0;  // chunk count the chunk size is planned for (0: P)
    if (mode != dsa::kModeScores) {
        // Parallel selection (fused, the grid resident at once) keeps no
        // merge list in one CTA: up to kMaxChunks chunks, and the SMs left
        // over give some groups one chunk more (every SM streams).
        // Otherwise the last CTA's merge list (P * topk composites) must
        // fit on chip.
        const int64_t p_par = P < dsa::kMaxChunks ? P : dsa::kMaxChunks;
        const int64_t sms = num_sms();
        int64_t p_cap_merge = (200 * 1024) / (8 * static_cast<int64_t>(p->topk));
        if (p_cap_merge > dsa::kMaxChunks) p_cap_merge = dsa::kMaxChunks;
        const int64_t p_merge = P < p_cap_merge ? P : p_cap_merge;
        // the merge (one CTA per group finishes the selection, the others
        // exit) measured faster whenever it keeps nine tenths of the SMs
        // streaming; the parallel selection serves the batches it cannot
        // fill (a few long queries: it allows more chunks)
        const bool merge_fills = p_merge >= p_min && 10 * static_cast<int64_t>(pl.n_groups) * p_merge >= 9 * sms;
        if (mode == dsa::kModeFused && !merge_fills && p_par > 1 && p_par >= p_min &&
            static_cast<int64_t>(pl.n_groups) * p_par <= sms) {
            int64_t extra = 0;
            if (DSA_K1_FILL_SMS && p_par < dsa::kMaxChunks && p_par < p_small) {
                extra = sms - static_cast<int64_t>(pl.n_groups) * p_par;
                if (extra > pl.n_groups) extra = pl.n_groups;
            }
            P = extra > 0 ? p_par + 1 : p_par;
            pl.n_big = extra > 0 ? static_cast<int>(extra) : pl.n_groups;
            p_cut = p_par;
            pl.parallel = true;
        } else {
            int64_t p_cap = (200 * 1024) / (8 * static_cast<int64_t>(p->topk));
            if (p_cap > dsa::kMaxChunks) p_cap = dsa::kMaxChunks;
            if (P > p_cap) {
                if (p_min > p_cap) return fail(DSA_ERR_UNSUPPORTED, "history too long for topk=%d (max_n=%d)", p->topk, p->max_n);
                P = p_cap;
            }
        }
    }
    // chunks are whole ring stages; each group cuts its own span the same
    // way on the device (no larger than this)
    const int64_t srows = 128;
    chunk_max = chunk_max / srows * srows;
    const int64_t pc = p_cut > 0 ? p_cut : P;
    int64_t chunk = (sp + pc - 1) / pc;
    chunk = (chunk + srows - 1) / srows * srows;
    if (chunk > chunk_max) chunk = chunk_max;
    if (p_cut == 0) {
        P = (sp + chunk - 1) / chunk;
        pl.n_big = pl.n_groups;
    }
    if (P <= 1) pl.parallel = false;
    pl.P = static_cast<int>(P);
    pl.chunk = static_cast<int>(chunk);
    if (mode != dsa::kModeScores) {
        // the ordered emissions record their ballots in the 2048-word radix
        // scratch (chunk lists) and in the whole histogram area (the merge)
        const int nw = (mode == dsa::kModeTopk ? dsa::kK2Threads : dsa::kK1Threads) / 32;
        const int merge_n = pl.P * (p->topk + 2);
        if (dsa::emit_ballot_words(pl.chunk, nw) > dsa::kSelBinsHost ||
            (!pl.parallel && dsa::emit_ballot_words(merge_n, nw) > (pl.qg + 1) * dsa::kSelBinsHost))
            return fail(DSA_ERR_UNSUPPORTED, "selection scratch too small for this plan");
    }
    pl.acc_bufs = (dsa::kK1MaxAcc * pl.qg * pl.hp <= 512) ? dsa::kK1MaxAcc : 2;
    uint32_t cols = 32;
    while (cols < static_cast<uint32_t>(pl.acc_bufs * pl.qg * pl.hp)) cols <<= 1;
    pl.tmem_cols = cols;
    // TMA ring: as many 128-row tiles as the shared memory left by the keys holds
    // (the merge area reuses the ring once streaming is over)
    pl.stages = 0;
    if (mode != dsa::kModeTopk) {
        int st = dsa::kK1MaxStages;
        while (st >= 2 &&
               dsa::k1_layout(mode, p->d_idx, pl.qg, pl.hp, pl.chunk, pl.P, p->topk, st, !pl.parallel).total > 232448)
            --st;
        // the two MMA threads take alternate tiles: an even ring, at least
        // as deep as the accumulator ring (the epilogue's wait on a stage's
        // commit relies on it)
        st &= ~1;
        if (st < 2) return fail(DSA_ERR_UNSUPPORTED, "indexer shared memory plan too large");
        pl.stages = st;
        if (pl.stages < pl.acc_bufs) {
            pl.acc_bufs = 2;
            pl.tmem_cols = 32;
            while (pl.tmem_cols < static_cast<uint32_t>(pl.acc_bufs * pl.qg * pl.hp)) pl.tmem_cols <<= 1;
        }
    }
    const dsa::K1Layout L = dsa::k1_layout(mode, p->d_idx, pl.qg, pl.hp, pl.chunk, pl.P, p->topk, pl.stages,
                                           !pl.parallel);
    pl.smem = L.total;
    if (pl.smem > 232448) return fail(DSA_ERR_UNSUPPORTED, "indexer shared memory plan too large");
    return DSA_OK;
}

struct MlaPlan {
    int splits, rows_per_split, wave;
};

constexpr size_t kPartialBudget = size_t(1) << 30;  // bytes of split partials per wave

MlaPlan plan_mla(const dsa_params *p) {
    MlaPlan m;
    const int k = p->topk;
    const int s_min = (k + dsa::kMlaMaxRows - 1) / dsa::kMlaMaxRows;
    int s_fill = p->nq > 0 ? num_sms() / p->nq : 1;
    const int s_small = (k + 63) / 64;
    int s = s_fill < s_small ? s_fill : s_small;
    if (s < s_min) s = s_min;
    if (s < 1) s = 1;
    int rps = (k + s - 1) / s;
    rps = (rps + 15) / 16 * 16;
    if (rps > dsa::kMlaMaxRows) rps = dsa::kMlaMaxRows;
    m.rows_per_split = rps;
    m.splits = (k + rps - 1) / rps;  // <= ceil(2048 / 64) = kMlaMaxSplits: rps >= 64 unless s_min binds
    if (m.splits == 1) {
        m.wave = p->nq;
    } else {
        const size_t per_q = static_cast<size_t>(m.splits) * 128 * (dsa::kDv * 2 + 4 + 4 * dsa::kMlaScaleBlocks);
        size_t w = kPartialBudget / per_q;
        if (w < 1) w = 1;
        m.wave = p->nq < static_cast<int>(w) ? p->nq : static_cast<int>(w);
    }
    return m;
}

// The distillation loss's set per query: topk entries of idx (sparse), or
// every visible position (dense, up to max_n).  Splits of at most 256 rows,
// as many as fill the SMs; no cap on their number (no output combine).
MlaPlan plan_kl(const dsa_params *p, bool dense) {
    MlaPlan m;
    const int k = dense ? p->max_n : p->topk;
    if (k <= 0) {
        m.splits = 1;
        m.rows_per_split = 16;
        m.wave = p->nq;
        return m;
    }
    const int s_min = (k + dsa::kMlaMaxRows - 1) / dsa::kMlaMaxRows;
    const int s_fill = p->nq > 0 ? num_sms() / p->nq : 1;
    const int s_small = (k + 63) / 64;
    int s = s_fill < s_small ? s_fill : s_small;
    if (s < s_min) s = s_min;
    if (s < 1) s = 1;
    int rps = (k + s - 1) / s;
    rps = (rps + 15) / 16 * 16;
    if (rps > dsa::kMlaMaxRows) rps = dsa::kMlaMaxRows;
    m.rows_per_split = rps;
    m.splits = (k + rps - 1) / rps;
    m.wave = p->nq;
    return m;
}

// -------------------------------------------------------------- workspace
struct WsLayout {
    size_t status, ghist, gtot, published, cand, cand_cnt, cand_above, done, idx, part_o, part_lse,
        part_scale, kl_lse, kl_a, total;
    size_t zero_begin, zero_end;  // cleared at the start of every call
};

int cand_stride(const dsa_params *p) { return (p->topk + 3) & ~3; }

size_t indexer_ws(const dsa_params *p, const IndexerPlan &pl, int mode, size_t off, WsLayout &w) {
    w.ghist = w.gtot = w.published = w.cand = w.cand_cnt = w.cand_above = w.done = off;
    if (mode == dsa::kModeScores || pl.P <= 1) return off;
    w.zero_begin = off;
    w.ghist = off;
    off = up(off + static_cast<size_t>(p->nq) * 2048 * 4, 256);
    w.gtot = off;
    off = up(off + static_cast<size_t>(p->nq) * 4, 256);
    w.published = off;
    off = up(off + static_cast<size_t>(p->nq) * 4, 256);
    w.done = off;
    off = up(off + static_cast<size_t>(pl.n_groups) * 4, 256);
    w.zero_end = off;
    w.cand = off;
    off = up(off + static_cast<size_t>(p->nq) * pl.P * cand_stride(p) * 8, 256);
    w.cand_cnt = off;
    off = up(off + static_cast<size_t>(p->nq) * pl.P * 4, 256);
    w.cand_above = off;
    off = up(off + static_cast<size_t>(p->nq) * pl.P * 4, 256);
    return off;
}

size_t mla_ws(const dsa_params *p, const MlaPlan &m, size_t off, WsLayout &w) {
    w.part_o = w.part_lse = w.part_scale = off;
    if (m.splits <= 1) return off;
    w.part_o = off;
    off = up(off + static_cast<size_t>(m.wave) * m.splits * 128 * dsa::kDv * 2, 256);  // fp16
    w.part_lse = off;
    off = up(off + static_cast<size_t>(m.wave) * m.splits * 128 * 4, 256);
    w.part_scale = off;
    off = up(off + static_cast<size_t>(m.wave) * m.splits * 128 * dsa::kMlaScaleBlocks * 4, 256);
    return off;
}

int layout_for(const dsa_params *p, int op, WsLayout &w, IndexerPlan *ipl, MlaPlan *mpl,
               int64_t ld_scores) {
    memset(&w, 0, sizeof w);
    size_t off = 256;  // status word
    w.status = 0;
    IndexerPlan pl{};
    MlaPlan m{};
    int rc;
    switch (op) {
    case DSA_OP_INDEXER_SCORES:
        rc = plan_indexer(p, dsa::kModeScores, ld_scores > p->max_n ? ld_scores : p->max_n, pl);
        if (rc) return rc;
        off = indexer_ws(p, pl, dsa::kModeScores, off, w);
        break;
    case DSA_OP_TOPK:
        rc = plan_indexer(p, dsa::kModeTopk, p->max_n, pl);
        if (rc) return rc;
        off = indexer_ws(p, pl, dsa::kModeTopk, off, w);
        break;
    case DSA_OP_INDEXER_TOPK:
        rc = plan_indexer(p, dsa::kModeFused, p->max_n, pl);
        if (rc) return rc;
        off = indexer_ws(p, pl, dsa::kModeFused, off, w);
        break;
    case DSA_OP_SPARSE_MLA_DECODE:
    case DSA_OP_SPARSE_MLA_PREFILL:
        m = plan_mla(p);
        off = mla_ws(p, m, off, w);
        break;
    case DSA_OP_INDEX_KL_SPARSE:
    case DSA_OP_INDEX_KL_DENSE: {
        const bool dense = op == DSA_OP_INDEX_KL_DENSE;
        const MlaPlan k = plan_kl(p, dense);
        const int64_t entries = dense ? p->max_n : p->topk;
        w.part_lse = off;
        off = up(off + static_cast<size_t>(p->nq) * k.splits * 128 * 4, 256);
        w.kl_lse = off;
        off = up(off + static_cast<size_t>(p->nq) * 128 * 4, 256);
        w.kl_a = off;
        off = up(off + static_cast<size_t>(p->nq) * static_cast<size_t>(entries) * 4, 256);
        w.total = off;
        if (mpl) *mpl = k;
        return DSA_OK;
    }
    case DSA_OP_MASKED_MHA:
        w.idx = off;  // the membership bitmap
        off = up(off + static_cast<size_t>(p->nq) * mha_mask_words(p) * 4, 256);
        w.total = off;
        return DSA_OK;
    case DSA_OP_FORWARD:
        rc = plan_indexer(p, dsa::kModeFused, p->max_n, pl);
        if (rc) return rc;
        off = indexer_ws(p, pl, dsa::kModeFused, off, w);
        w.idx = off;
        off = up(off + static_cast<size_t>(p->nq) * p->topk * 4, 256);
        m = plan_mla(p);
        off = mla_ws(p, m, off, w);
        break;
    default:
        return fail(DSA_ERR_INVALID_ARG, "unknown op %d", op);
    }
    if (m.splits > dsa::kMlaMaxSplits) return fail(DSA_ERR_UNSUPPORTED, "too many attention splits (%d)", m.splits);
    w.total = off;
    if (ipl) *ipl = pl;
    if (mpl) *mpl = m;
    return DSA_OK;
}

int check_ws(void *ws, size_t ws_bytes, const WsLayout &w) {
    if (!ws) return fail(DSA_ERR_WORKSPACE, "ws is NULL");
    if (!aligned(ws, 256)) return fail(DSA_ERR_WORKSPACE, "ws must be 256-byte aligned");
    if (ws_bytes < w.total) return fail(DSA_ERR_WORKSPACE, "ws_bytes %zu < required %zu", ws_bytes, w.total);
    return DSA_OK;
}

template <class T>
T *at(void *ws, size_t off) {
    return reinterpret_cast<T *>(static_cast<uint8_t *>(ws) + off);
}

// ------------------------------------------------------------ enqueue steps
int run_indexer(const dsa_params *p, const dsa_kv *kv, int mode, const void *q_idx, const void *w,
                const void *kidx_cache, const float *k_scale, float *scores, int64_t ld,
                int32_t *idx, int32_t *nsel, void *ws, const WsLayout &wl, const IndexerPlan &pl,
                cudaStream_t st) {
    dsa::K1Params a;
    memset(&a, 0, sizeof a);
    a.q_idx = static_cast<const uint8_t *>(q_idx);
    a.w = static_cast<const uint16_t *>(w);
    a.k_scale = k_scale;
    a.nq = p->nq;
    a.h_idx = p->h_idx;
    a.d_idx = p->d_idx;
    a.topk = p->topk;
    a.q_per_seq = p->q_per_seq;
    a.qg = pl.qg;
    a.groups_per_block = pl.gpb;
    a.n_groups = pl.n_groups;
    a.P = pl.P;
    a.n_big = pl.n_big;
    a.chunk = pl.chunk;
    a.stages = pl.stages;
    a.acc_bufs = pl.acc_bufs;
    a.tmem_cols = pl.tmem_cols;
    a.scores = scores;
    a.ld = ld;
    a.idx = idx;
    a.nsel = nsel;
    a.status = at<int>(ws, wl.status);
    a.wait_budget = dsa::kWaitBudgetCycles;
    if (int rc = host_fault("indexer")) return rc;
    if (mode != dsa::kModeTopk && inject_timeout("indexer")) {
        a.wait_budget = kTestWaitBudget;
        a.inject = 1;
    }
    if (mode != dsa::kModeScores && pl.P > 1) {
        a.ghist = at<uint32_t>(ws, wl.ghist);
        a.gtot = at<uint32_t>(ws, wl.gtot);
        a.published = at<uint32_t>(ws, wl.published);
        a.done = at<uint32_t>(ws, wl.done);
        // every CTA of the launch is resident at once (at most one per SM
        // is needed): each chunk selects its own part of the output
        a.parallel = pl.parallel ? 1 : 0;
        const int64_t grid = static_cast<int64_t>(pl.n_big) * pl.P + static_cast<int64_t>(pl.n_groups - pl.n_big) * (pl.P - 1);
        a.wait_hist = (!pl.parallel && grid <= num_sms()) ? 1 : 0;
        a.cand = at<uint64_t>(ws, wl.cand);
        a.cand_stride = cand_stride(p);
        a.cand_cnt = at<int32_t>(ws, wl.cand_cnt);
        a.cand_above = at<int32_t>(ws, wl.cand_above);
    }
    if (p->nq == 0) return DSA_OK;
    // the cross-chunk counters start at zero: a clearing kernel right before
    // the indexer, which starts as its programmatic dependent and waits for
    // it only after streaming (not the TopK-only kernel, which reads scores
    // a preceding kernel may still be writing)
    bool pdl = false;
    if (mode != dsa::kModeScores && pl.P > 1 && wl.zero_end > wl.zero_begin) {
        cudaError_t e = dsa::launch_clear(static_cast<uint8_t *>(ws) + wl.zero_begin, wl.zero_end - wl.zero_begin, st);
        if (e != cudaSuccess) return cuda_fail(e, "counter clear launch");
        pdl = mode != dsa::kModeTopk;
    }
    cudaError_t e;
    if (mode == dsa::kModeTopk) {
        a.q_n = kv ? kv->q_n : nullptr;
        e = dsa::launch_topk(a, st);
        if (e != cudaSuccess) return cuda_fail(e, "TopK launch");
        return DSA_OK;
    }
    a.q_seq = kv->q_seq;
    a.q_n = kv->q_n;
    a.seq_row0 = kv->seq_row0;
    a.page_table = kv->page_table;
    a.max_pages = kv->max_pages;
    a.page_size = kv->page_table ? kv->page_size : 0;
    a.cache_rows = kv->cache_rows;
    CUtensorMap kmap;
    // one box per 128-row tile, or one per page
    const uint32_t box_rows = kv->page_table ? static_cast<uint32_t>(kv->page_size) : 128u;
    int rc = make_map_2d(&kmap, CU_TENSOR_MAP_DATA_TYPE_UINT8, kidx_cache, p->d_idx, kv->cache_rows,
                         p->d_idx, p->d_idx, box_rows,
                         p->d_idx == 128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B);
    if (rc) return rc;
    e = dsa::launch_indexer(mode, pl.hp, p->d_idx, kmap, a, st, pdl);
    if (e != cudaSuccess) return cuda_fail(e, "indexer launch");
    return DSA_OK;
}

int run_mla(const dsa_params *p, const dsa_kv *kv, const void *q, const void *kv_cache,
            int64_t kv_row_stride, const int32_t *idx, void *out, float *lse, void *ws,
            const WsLayout &wl, const MlaPlan &m, cudaStream_t st, const float *kv_scale = nullptr) {
    if (p->nq == 0) return DSA_OK;
    if (int rc = host_fault("attention")) return rc;
    CUtensorMap qmap;
    const uint32_t hbox = p->h < 128 ? static_cast<uint32_t>(p->h) : 128u;
    int rc = make_map_2d(&qmap, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, q, dsa::kDqk,
                         static_cast<uint64_t>(p->nq) * p->h, dsa::kDqk * 2, 64, hbox,
                         CU_TENSOR_MAP_SWIZZLE_128B);
    if (rc) return rc;
    dsa::MlaParams a;
    memset(&a, 0, sizeof a);
    a.q_seq = kv->q_seq;
    a.q_n = kv->q_n;
    a.seq_row0 = kv->seq_row0;
    a.page_table = kv->page_table;
    a.max_pages = kv->max_pages;
    a.page_size = kv->page_table ? kv->page_size : 0;
    a.cache_rows = kv->cache_rows;
    a.idx = idx;
    // an FP8 cache (kv_scale set): kv_cache holds e4m3 codes, kv_row_stride bytes apart
    const bool kv8 = kv_scale != nullptr;
    if (kv8) {
        a.kv8 = static_cast<const uint8_t *>(kv_cache);
        a.kv8_row_bytes = kv_row_stride;
        a.kv_scale = kv_scale;
    } else {
        a.kv = static_cast<const uint16_t *>(kv_cache);
        a.kv_row_stride = kv_row_stride;
    }
    a.nq = p->nq;
    a.h = p->h;
    a.topk = p->topk;
    a.splits = m.splits;
    a.rows_per_split = m.rows_per_split;
    a.scale = p->scale;
    a.scale_log2 = p->scale * 1.4426950408889634f;
    a.out = static_cast<uint16_t *>(out);
    a.lse = lse;
    a.part_o = m.splits > 1 ? at<uint16_t>(ws, wl.part_o) : nullptr;
    a.part_lse = m.splits > 1 ? at<float>(ws, wl.part_lse) : nullptr;
    a.part_scale = m.splits > 1 ? at<float>(ws, wl.part_scale) : nullptr;
    a.status = at<int>(ws, wl.status);
    a.wait_budget = dsa::kWaitBudgetCycles;
    if (inject_timeout("attention")) {
        a.wait_budget = kTestWaitBudget;
        a.inject = 1;
    }
    for (int q0 = 0; q0 < p->nq; q0 += m.wave) {
        const int nw = (p->nq - q0) < m.wave ? (p->nq - q0) : m.wave;
        a.q0 = q0;
        cudaError_t e = dsa::launch_sparse_mla(qmap, a, nw, st, kv8);
        if (e != cudaSuccess) return cuda_fail(e, "sparse MLA launch");
        e = dsa::launch_mla_combine(a, nw, st);
        if (e != cudaSuccess) return cuda_fail(e, "split combine launch");
    }
    return DSA_OK;
}

int check_indexer_inputs(const dsa_params *p, const void *q_idx, const void *w, const void *kidx) {
    if (p->nq == 0) return DSA_OK;
    if (!q_idx || !w || !kidx) return fail(DSA_ERR_INVALID_ARG, "q_idx / w / kidx_cache is NULL");
    if (!aligned(q_idx, 16) || !aligned(kidx, 16)) return fail(DSA_ERR_INVALID_ARG, "q_idx / kidx_cache must be 16-byte aligned");
    if (!aligned(w, 2)) return fail(DSA_ERR_INVALID_ARG, "w must be 2-byte aligned");
    return DSA_OK;
}

int check_mla_inputs(const dsa_params *p, const void *q, const void *kv_cache, int64_t stride,
                     const void *idx, const void *out, const void *lse) {
    if (p->nq == 0) return DSA_OK;
    if (!q || !kv_cache || !idx || !out || !lse) return fail(DSA_ERR_INVALID_ARG, "q / kv_cache / idx / out / lse is NULL");
    if (!aligned(q, 16) || !aligned(kv_cache, 16) || !aligned(out, 16))
        return fail(DSA_ERR_INVALID_ARG, "q / kv_cache / out must be 16-byte aligned");
    if (stride < 576 || stride % 8 != 0) return fail(DSA_ERR_INVALID_ARG, "kv_row_stride must be >= 576 and a multiple of 8");
    return DSA_OK;
}

// ------------------------------------------------------- indexer producer
struct ProjPlan {
    int n_tok, t_tiles, m_tiles[2], k_steps[2], splits[2], ld[2], stages;
    uint32_t stage_bytes;
    size_t part_off[2], total;
};

int check_project(const dsa_project_params *pp) {
    if (!pp) return fail(DSA_ERR_INVALID_ARG, "params is NULL");
    if (pp->nt < 0) return fail(DSA_ERR_INVALID_ARG, "nt < 0");
    if (pp->h_idx < 1 || pp->h_idx > 64) return fail(DSA_ERR_INVALID_ARG, "h_idx must be in [1, 64]");
    if (pp->d_idx != 64 && pp->d_idx != 128) return fail(DSA_ERR_INVALID_ARG, "d_idx must be 64 or 128");
    if (pp->rope_dim < 0 || pp->rope_dim > pp->d_idx || (pp->rope_dim & 1))
        return fail(DSA_ERR_INVALID_ARG, "rope_dim must be even and in [0, d_idx]");
    if (pp->hidden < 8 || pp->hidden % 8 || pp->q_lora_rank < 8 || pp->q_lora_rank % 8)
        return fail(DSA_ERR_INVALID_ARG, "hidden and q_lora_rank must be positive multiples of 8");
    if (!(pp->ln_eps >= 0.f) || !isfinite(pp->rope_theta) || !(pp->rope_theta > 0.f))
        return fail(DSA_ERR_INVALID_ARG, "ln_eps must be >= 0 and rope_theta > 0");
    return DSA_OK;
}

// K slices so that the grid fills the SMs when few token tiles exist, in
// proportion to each problem's weight bytes (decode streams the weights).
ProjPlan plan_project(const dsa_project_params *pp) {
    ProjPlan pl;
    // token tiles of up to 256 (the MMA N), a multiple of 16
    int nt16 = (pp->nt + 15) / 16 * 16;
    pl.n_tok = nt16 < 16 ? 16 : (nt16 > 256 ? 256 : nt16);
    pl.t_tiles = (pp->nt + pl.n_tok - 1) / pl.n_tok;
    pl.m_tiles[0] = (pp->d_idx + pp->h_idx + 127) / 128;
    pl.m_tiles[1] = (pp->h_idx * pp->d_idx + 127) / 128;
    pl.k_steps[0] = (pp->hidden + 63) / 64;
    pl.k_steps[1] = (pp->q_lora_rank + 63) / 64;
    pl.ld[0] = (pp->d_idx + pp->h_idx + 3) & ~3;
    pl.ld[1] = pp->h_idx * pp->d_idx;
    // K slices fill the SMs in proportion to each problem's weight bytes
    const double b0 = static_cast<double>(pp->d_idx + pp->h_idx) * pp->hidden;
    const double b1 = static_cast<double>(pp->h_idx) * pp->d_idx * pp->q_lora_rank;
    const int sms = num_sms();
    const int base0 = pl.m_tiles[0] * pl.t_tiles, base1 = pl.m_tiles[1] * pl.t_tiles;
    int s0 = 1, s1 = 1;
    if (pl.t_tiles > 0 && base0 + base1 < sms) {
        s0 = static_cast<int>(sms * b0 / (b0 + b1) / base0);
        s1 = static_cast<int>(sms * b1 / (b0 + b1) / base1);
    }
    pl.splits[0] = s0 < 1 ? 1 : (s0 > pl.k_steps[0] ? pl.k_steps[0] : s0);
    pl.splits[1] = s1 < 1 ? 1 : (s1 > pl.k_steps[1] ? pl.k_steps[1] : s1);
    // ring: 16 KB of weights + n_tok x 128 B of activations per stage
    pl.stage_bytes = (16384u + static_cast<uint32_t>(pl.n_tok) * 128u + 1023u) & ~1023u;
    int st = dsa::kProjMaxStages;
    while (st > 2 && static_cast<size_t>(st) * pl.stage_bytes + 1024 + 1024 > 232448) --st;
    pl.stages = st;
    size_t off = 256;  // status word
    for (int q = 0; q < 2; ++q) {
        pl.part_off[q] = off;
        off = up(off + static_cast<size_t>(pl.splits[q]) * pp->nt * pl.ld[q] * 4, 256);
    }
    pl.total = off;
    return pl;
}

}  // namespace

extern "C" {

int dsa_workspace_size(const dsa_params *p, const dsa_kv *kv, int op, size_t *bytes) {
    int rc = op == DSA_OP_MASKED_MHA ? check_params_mha(p) : check_params(p);
    if (rc) return rc;
    if (!bytes) return fail(DSA_ERR_INVALID_ARG, "bytes is NULL");
    if (op != DSA_OP_TOPK) {
        rc = check_kv(p, kv);
        if (rc) return rc;
    }
    WsLayout w;
    rc = layout_for(p, op, w, nullptr, nullptr, p->max_n);
    if (rc) return rc;
    *bytes = w.total;
    return DSA_OK;
}

int dsa_indexer_scores(const dsa_params *p, const dsa_kv *kv, const void *q_idx, const void *w,
                       const void *kidx_cache, const float *k_scale, float *scores, int64_t ld_scores,
                       void *ws, size_t ws_bytes, void *stream) {
    int rc = check_params(p);
    if (!rc) rc = check_kv(p, kv);
    if (!rc) rc = check_indexer_inputs(p, q_idx, w, kidx_cache);
    if (rc) return rc;
    if (ld_scores < p->max_n || ld_scores > (int64_t(1) << 27)) return fail(DSA_ERR_INVALID_ARG, "ld_scores must be in [max_n, 2^27]");
    if (p->nq > 0 && !scores) return fail(DSA_ERR_INVALID_ARG, "scores is NULL");
    WsLayout wl;
    IndexerPlan pl;
    rc = layout_for(p, DSA_OP_INDEXER_SCORES, wl, &pl, nullptr, ld_scores);
    if (!rc) rc = check_ws(ws, ws_bytes, wl);
    if (rc) return rc;
    // the score plan covers ld_scores positions
    rc = plan_indexer(p, dsa::kModeScores, ld_scores > 0 ? ld_scores : 1, pl);
    if (rc) return rc;
    return run_indexer(p, kv, dsa::kModeScores, q_idx, w, kidx_cache, k_scale, scores, ld_scores,
                       nullptr, nullptr, ws, wl, pl, static_cast<cudaStream_t>(stream));
}

int dsa_topk(const dsa_params *p, const float *scores, int64_t ld_scores, const int32_t *q_n,
             int32_t *idx, int32_t *nsel, void *ws, size_t ws_bytes, void *stream) {
    int rc = check_params(p);
    if (rc) return rc;
    if (p->nq > 0 && (!scores || !q_n || !idx)) return fail(DSA_ERR_INVALID_ARG, "scores / q_n / idx is NULL");
    if (ld_scores < p->max_n) return fail(DSA_ERR_INVALID_ARG, "ld_scores < max_n");
    WsLayout wl;
    IndexerPlan pl;
    rc = layout_for(p, DSA_OP_TOPK, wl, &pl, nullptr, ld_scores);
    if (!rc) rc = check_ws(ws, ws_bytes, wl);
    if (rc) return rc;
    dsa_kv kv;
    memset(&kv, 0, sizeof kv);
    kv.q_n = q_n;
    return run_indexer(p, &kv, dsa::kModeTopk, nullptr, nullptr, nullptr, nullptr,
                       const_cast<float *>(scores), ld_scores, idx, nsel, ws, wl, pl,
                       static_cast<cudaStream_t>(stream));
}

int dsa_indexer_topk(const dsa_params *p, const dsa_kv *kv, const void *q_idx, const void *w,
                     const void *kidx_cache, const float *k_scale, int32_t *idx, int32_t *nsel,
                     void *ws, size_t ws_bytes, void *stream) {
    int rc = check_params(p);
    if (!rc) rc = check_kv(p, kv);
    if (!rc) rc = check_indexer_inputs(p, q_idx, w, kidx_cache);
    if (rc) return rc;
    if (p->nq > 0 && !idx) return fail(DSA_ERR_INVALID_ARG, "idx is NULL");
    WsLayout wl;
    IndexerPlan pl;
    rc = layout_for(p, DSA_OP_INDEXER_TOPK, wl, &pl, nullptr, p->max_n);
    if (!rc) rc = check_ws(ws, ws_bytes, wl);
    if (rc) return rc;
    return run_indexer(p, kv, dsa::kModeFused, q_idx, w, kidx_cache, k_scale, nullptr, 0, idx, nsel,
                       ws, wl, pl, static_cast<cudaStream_t>(stream));
}

static int mla_common(int op, const dsa_params *p, const dsa_kv *kv, const void *q,
                      const void *kv_cache, int64_t kv_row_stride, const int32_t *idx, void *out,
                      float *lse, void *ws, size_t ws_bytes, void *stream) {
    int rc = check_params(p);
    if (!rc) rc = check_kv(p, kv);
    if (!rc) rc = check_mla_inputs(p, q, kv_cache, kv_row_stride, idx, out, lse);
    if (rc) return rc;
    WsLayout wl;
    MlaPlan m;
    rc = layout_for(p, op, wl, nullptr, &m, p->max_n);
    if (!rc) rc = check_ws(ws, ws_bytes, wl);
    if (rc) return rc;
    return run_mla(p, kv, q, kv_cache, kv_row_stride, idx, out, lse, ws, wl, m,
                   static_cast<cudaStream_t>(stream));
}

int dsa_sparse_mla_decode(const dsa_params *p, const dsa_kv *kv, const void *q, const void *kv_cache,
                          int64_t kv_row_stride, const int32_t *idx, void *out, float *lse, void *ws,
                          size_t ws_bytes, void *stream) {
    return mla_common(DSA_OP_SPARSE_MLA_DECODE, p, kv, q, kv_cache, kv_row_stride, idx, out, lse, ws,
                      ws_bytes, stream);
}

int dsa_sparse_mla_prefill(const dsa_params *p, const dsa_kv *kv, const void *q, const void *kv_cache,
                           int64_t kv_row_stride, const int32_t *idx, void *out, float *lse, void *ws,
                           size_t ws_bytes, void *stream) {
    return mla_common(DSA_OP_SPARSE_MLA_PREFILL, p, kv, q, kv_cache, kv_row_stride, idx, out, lse, ws,
                      ws_bytes, stream);
}

int dsa_index_kl(const dsa_params *p, const dsa_kv *kv, const void *q, const void *kv_cache,
                 int64_t kv_row_stride, const float *index_scores, int64_t ld_scores, const int32_t *idx,
                 float *kl, float *p_out, void *ws, size_t ws_bytes, void *stream) {
    int rc = check_params(p);
    if (!rc) rc = check_kv(p, kv);
    if (rc) return rc;
    if (p->nq > 0) {
        if (!q || !kv_cache || !index_scores || !kl)
            return fail(DSA_ERR_INVALID_ARG, "q / kv_cache / index_scores / kl is NULL");
        if (!aligned(q, 16) || !aligned(kv_cache, 16)) return fail(DSA_ERR_INVALID_ARG, "q / kv_cache must be 16-byte aligned");
        if (kv_row_stride < 576 || kv_row_stride % 8 != 0)
            return fail(DSA_ERR_INVALID_ARG, "kv_row_stride must be >= 576 and a multiple of 8");
    }
    if (ld_scores < p->max_n || ld_scores > (int64_t(1) << 27)) return fail(DSA_ERR_INVALID_ARG, "ld_scores must be in [max_n, 2^27]");
    const bool dense = idx == nullptr;
    WsLayout wl;
    MlaPlan m;
    rc = layout_for(p, dense ? DSA_OP_INDEX_KL_DENSE : DSA_OP_INDEX_KL_SPARSE, wl, nullptr, &m, p->max_n);
    if (!rc) rc = check_ws(ws, ws_bytes, wl);
    if (rc) return rc;
    if (p->nq == 0) return DSA_OK;
    if (int frc = host_fault("index_kl")) return frc;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    CUtensorMap qmap;
    const uint32_t hbox = p->h < 128 ? static_cast<uint32_t>(p->h) : 128u;
    rc = make_map_2d(&qmap, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, q, dsa::kDqk, static_cast<uint64_t>(p->nq) * p->h,
                     dsa::kDqk * 2, 64, hbox, CU_TENSOR_MAP_SWIZZLE_128B);
    if (rc) return rc;
    dsa::MlaParams a;
    memset(&a, 0, sizeof a);
    a.q_seq = kv->q_seq;
    a.q_n = kv->q_n;
    a.seq_row0 = kv->seq_row0;
    a.page_table = kv->page_table;
    a.max_pages = kv->max_pages;
    a.page_size = kv->page_table ? kv->page_size : 0;
    a.cache_rows = kv->cache_rows;
    a.idx = idx;
    a.dense = dense ? 1 : 0;
    a.kv = static_cast<const uint16_t *>(kv_cache);
    a.kv_row_stride = kv_row_stride;
    a.nq = p->nq;
    a.h = p->h;
    a.topk = dense ? p->max_n : p->topk;
    a.splits = m.splits;
    a.rows_per_split = m.rows_per_split;
    a.scale = p->scale;
    a.scale_log2 = p->scale * 1.4426950408889634f;
    a.part_lse = at<float>(ws, wl.part_lse);
    a.kl_lse = at<float>(ws, wl.kl_lse);
    a.kl_a = at<float>(ws, wl.kl_a);
    a.iscores = index_scores;
    a.ld = ld_scores;
    a.kl = kl;
    a.p_out = p_out;
    a.status = at<int>(ws, wl.status);
    a.wait_budget = dsa::kWaitBudgetCycles;
    cudaError_t e = dsa::launch_kl_pass(dsa::kMlaKlStats, qmap, a, st);
    if (e == cudaSuccess) e = dsa::launch_kl_lse(a, st);
    if (e == cudaSuccess) e = dsa::launch_kl_pass(dsa::kMlaKlSum, qmap, a, st);
    if (e == cudaSuccess) e = dsa::launch_kl_reduce(a, st);
    if (e != cudaSuccess) return cuda_fail(e, "distillation loss launch");
    return DSA_OK;
}

int dsa_masked_mha_prefill(const dsa_params *p, const dsa_kv *kv, const void *q, const void *k, const void *v,
                           const int32_t *idx, void *out, float *lse, void *ws, size_t ws_bytes, void *stream) {
    int rc = check_params_mha(p);
    if (!rc) rc = check_kv(p, kv);
    if (rc) return rc;
    if (kv->page_table) return fail(DSA_ERR_UNSUPPORTED, "masked MHA: k / v are contiguous (seq_row0), not paged");
    if (p->nq > 0) {
        if (!q || !k || !v || !out || !lse) return fail(DSA_ERR_INVALID_ARG, "q / k / v / out / lse is NULL");
        if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(out, 16))
            return fail(DSA_ERR_INVALID_ARG, "q / k / v / out must be 16-byte aligned");
        if (static_cast<int64_t>(p->nq) + dsa::kMhaTile >= (int64_t(1) << 31))
            return fail(DSA_ERR_INVALID_ARG, "nq too large");
    }
    WsLayout wl;
    rc = layout_for(p, DSA_OP_MASKED_MHA, wl, nullptr, nullptr, p->max_n);
    if (!rc) rc = check_ws(ws, ws_bytes, wl);
    if (rc) return rc;
    if (p->nq == 0) return DSA_OK;
    if (int frc = host_fault("masked_mha")) return frc;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const uint64_t H = static_cast<uint64_t>(p->h);
    CUtensorMap qmap, kmap, vmap;
    rc = make_map_3d(&qmap, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, q, {static_cast<uint64_t>(p->d_qk), H, static_cast<uint64_t>(p->nq)},
                     {static_cast<uint64_t>(p->d_qk) * 2, H * p->d_qk * 2}, {64, 1, dsa::kMhaTile},
                     CU_TENSOR_MAP_SWIZZLE_128B);
    if (!rc)
        rc = make_map_3d(&kmap, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, k,
                         {static_cast<uint64_t>(p->d_qk), H, static_cast<uint64_t>(kv->cache_rows)},
                         {static_cast<uint64_t>(p->d_qk) * 2, H * p->d_qk * 2}, {64, 1, dsa::kMhaTile},
                         CU_TENSOR_MAP_SWIZZLE_128B);
    if (!rc)
        rc = make_map_3d(&vmap, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, v,
                         {static_cast<uint64_t>(p->d_v), H, static_cast<uint64_t>(kv->cache_rows)},
                         {static_cast<uint64_t>(p->d_v) * 2, H * p->d_v * 2}, {64, 1, dsa::kMhaTile},
                         CU_TENSOR_MAP_SWIZZLE_128B);
    if (rc) return rc;
    dsa::MhaParams a;
    memset(&a, 0, sizeof a);
    a.q_seq = kv->q_seq;
    a.q_n = kv->q_n;
    a.seq_row0 = kv->seq_row0;
    a.mask_words = mha_mask_words(p);
    uint32_t *mask = idx ? at<uint32_t>(ws, wl.idx) : nullptr;
    a.mask = mask;
    a.nq = p->nq;
    a.h = p->h;
    a.d_qk = p->d_qk;
    a.d_v = p->d_v;
    a.max_n = p->max_n;
    a.q_per_seq = p->q_per_seq;
    a.tiles_per_block = (p->q_per_seq + dsa::kMhaTile - 1) / dsa::kMhaTile;
    a.scale_log2 = p->scale * 1.4426950408889634f;
    a.out = static_cast<uint16_t *>(out);
    a.lse = lse;
    a.status = at<int>(ws, wl.status);
    a.wait_budget = dsa::kWaitBudgetCycles;
    int stages = dsa::kMhaMaxStages;
    while (stages > 1 && dsa::mha_layout(p->d_qk, p->d_v, stages).total > 232448) --stages;
    a.stages = stages;
    const int64_t blocks = (static_cast<int64_t>(p->nq) + p->q_per_seq - 1) / p->q_per_seq;
    const int64_t grid = blocks * a.tiles_per_block * p->h;
    if (grid >= (int64_t(1) << 31)) return fail(DSA_ERR_UNSUPPORTED, "masked MHA: grid too large");
    cudaError_t e = cudaSuccess;
    if (idx) e = dsa::launch_mha_mask(idx, p->topk, kv->q_n, mask, a.mask_words, p->nq, a.status, st);
    if (e == cudaSuccess) e = dsa::launch_masked_mha(qmap, kmap, vmap, a, static_cast<int>(grid), st);
    if (e != cudaSuccess) return cuda_fail(e, "masked MHA launch");
    return DSA_OK;
}

int dsa_sparse_mla_decode_fp8(const dsa_params *p, const dsa_kv *kv, const void *q, const void *kv8_cache,
                              int64_t kv8_row_bytes, const float *kv_scale, const int32_t *idx, void *out,
                              float *lse, void *ws, size_t ws_bytes, void *stream) {
    int rc = check_params(p);
    if (!rc) rc = check_kv(p, kv);
    if (rc) return rc;
    if (p->nq > 0) {
        if (!q || !kv8_cache || !kv_scale || !idx || !out || !lse)
            return fail(DSA_ERR_INVALID_ARG, "q / kv8_cache / kv_scale / idx / out / lse is NULL");
        if (!aligned(q, 16) || !aligned(kv8_cache, 16) || !aligned(out, 16))
            return fail(DSA_ERR_INVALID_ARG, "q / kv8_cache / out must be 16-byte aligned");
        if (kv8_row_bytes < 576 || kv8_row_bytes % 16 != 0)
            return fail(DSA_ERR_INVALID_ARG, "kv8_row_bytes must be >= 576 and a multiple of 16");
    }
    WsLayout wl;
    MlaPlan m;
    rc = layout_for(p, DSA_OP_SPARSE_MLA_DECODE, wl, nullptr, &m, p->max_n);
    if (!rc) rc = check_ws(ws, ws_bytes, wl);
    if (rc) return rc;
    return run_mla(p, kv, q, kv8_cache, kv8_row_bytes, idx, out, lse, ws, wl, m, static_cast<cudaStream_t>(stream),
                   kv_scale);
}

int dsa_forward(const dsa_params *p, const dsa_kv *kv, const void *q_idx, const void *w,
                const void *kidx_cache, const float *k_scale, const void *q, const void *kv_cache,
                int64_t kv_row_stride, void *out, float *lse, int32_t *idx_out, void *ws,
                size_t ws_bytes, void *stream) {
    int rc = check_params(p);
    if (!rc) rc = check_kv(p, kv);
    if (!rc) rc = check_indexer_inputs(p, q_idx, w, kidx_cache);
    if (!rc) rc = check_mla_inputs(p, q, kv_cache, kv_row_stride, q, out, lse);
    if (rc) return rc;
    WsLayout wl;
    IndexerPlan pl;
    MlaPlan m;
    rc = layout_for(p, DSA_OP_FORWARD, wl, &pl, &m, p->max_n);
    if (!rc) rc = check_ws(ws, ws_bytes, wl);
    if (rc) return rc;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    int32_t *idx = idx_out ? idx_out : at<int32_t>(ws, wl.idx);
    rc = run_indexer(p, kv, dsa::kModeFused, q_idx, w, kidx_cache, k_scale, nullptr, 0, idx, nullptr,
                     ws, wl, pl, st);
    if (rc) return rc;
    return run_mla(p, kv, q, kv_cache, kv_row_stride, idx, out, lse, ws, wl, m, st);
}

int dsa_forward_paged(const dsa_params *p, const dsa_kv *kv, const void *q_idx, const void *w,
                      const void *kidx_cache, const float *k_scale, const void *q,
                      const void *kv_cache, int64_t kv_row_stride, void *out, float *lse,
                      int32_t *idx_out, void *ws, size_t ws_bytes, void *stream) {
    if (!kv || !kv->page_table) return fail(DSA_ERR_INVALID_ARG, "dsa_forward_paged needs kv->page_table");
    return dsa_forward(p, kv, q_idx, w, kidx_cache, k_scale, q, kv_cache, kv_row_stride, out, lse,
                       idx_out, ws, ws_bytes, stream);
}

int dsa_project_workspace_size(const dsa_project_params *pp, size_t *bytes) {
    int rc = check_project(pp);
    if (rc) return rc;
    if (!bytes) return fail(DSA_ERR_INVALID_ARG, "bytes is NULL");
    *bytes = plan_project(pp).total;
    return DSA_OK;
}

int dsa_indexer_project(const dsa_project_params *pp, const dsa_kv *kv, const void *x,
                        const void *q_lora, const void *w_qb, const void *w_k, const void *w_proj,
                        const float *ln_gamma, const float *ln_beta, const int32_t *positions,
                        void *q_idx, float *q_scale, void *w, void *kidx_cache, float *k_scale,
                        float *q_f32, float *k_f32, float *w_f32, void *ws, size_t ws_bytes,
                        void *stream) {
    int rc = check_project(pp);
    if (rc) return rc;
    if (!kv) return fail(DSA_ERR_INVALID_ARG, "kv is NULL");
    if ((kv->seq_row0 == nullptr) == (kv->page_table == nullptr))
        return fail(DSA_ERR_INVALID_ARG, "exactly one of seq_row0 and page_table must be set");
    if (kv->page_table && kv->page_size != 64 && kv->page_size != 128)
        return fail(DSA_ERR_UNSUPPORTED, "page_size must be 64 or 128");
    if (kv->page_table && kv->max_pages < 1) return fail(DSA_ERR_INVALID_ARG, "max_pages < 1");
    if (kv->cache_rows < 1 || kv->cache_rows >= (int64_t(1) << 31))
        return fail(DSA_ERR_INVALID_ARG, "cache_rows must be in [1, 2^31)");
    const ProjPlan pl = plan_project(pp);
    if (!ws) return fail(DSA_ERR_WORKSPACE, "ws is NULL");
    if (!aligned(ws, 256)) return fail(DSA_ERR_WORKSPACE, "ws must be 256-byte aligned");
    if (ws_bytes < pl.total) return fail(DSA_ERR_WORKSPACE, "ws_bytes %zu < required %zu", ws_bytes, pl.total);
    if (pp->nt == 0) return DSA_OK;
    if (!x || !q_lora || !w_qb || !w_k || !w_proj || !ln_gamma || !ln_beta || !positions || !q_idx || !w ||
        !kidx_cache || !k_scale || !kv->q_seq)
        return fail(DSA_ERR_INVALID_ARG, "a required pointer is NULL");
    if (!aligned(x, 16) || !aligned(q_lora, 16) || !aligned(w_qb, 16) || !aligned(w_k, 16) ||
        !aligned(w_proj, 16) || !aligned(q_idx, 4) || !aligned(kidx_cache, 4))
        return fail(DSA_ERR_INVALID_ARG, "x, q_lora and the weights must be 16-byte aligned, q_idx and "
                                         "kidx_cache 4-byte aligned");
    if (int frc = host_fault("project")) return frc;
    CUtensorMap xm, qm, km, pm, wm;
    const CUtensorMapDataType bf = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
    const CUtensorMapSwizzle sw = CU_TENSOR_MAP_SWIZZLE_128B;
    // weights as 64-row (W_k, W_proj) / 128-row (W_qb) boxes, activations as
    // boxes of one token tile
    const uint32_t ntok = static_cast<uint32_t>(pl.n_tok);
    rc = make_map_2d(&xm, bf, x, pp->hidden, pp->nt, pp->hidden * 2ull, 64, ntok, sw);
    if (!rc) rc = make_map_2d(&qm, bf, q_lora, pp->q_lora_rank, pp->nt, pp->q_lora_rank * 2ull, 64, ntok, sw);
    if (!rc) rc = make_map_2d(&km, bf, w_k, pp->hidden, pp->d_idx, pp->hidden * 2ull, 64, 64, sw);
    if (!rc) rc = make_map_2d(&pm, bf, w_proj, pp->hidden, pp->h_idx, pp->hidden * 2ull, 64, pp->h_idx, sw);
    if (!rc) rc = make_map_2d(&wm, bf, w_qb, pp->q_lora_rank, static_cast<uint64_t>(pp->h_idx) * pp->d_idx,
                              pp->q_lora_rank * 2ull, 64, 128, sw);
    if (rc) return rc;
    dsa::ProjGemmParams g;
    memset(&g, 0, sizeof g);
    g.nt = pp->nt;
    g.n_tok = pl.n_tok;
    g.t_tiles = pl.t_tiles;
    for (int q = 0; q < 2; ++q) {
        g.m_tiles[q] = pl.m_tiles[q];
        g.k_steps[q] = pl.k_steps[q];
        g.splits[q] = pl.splits[q];
        g.part[q] = at<float>(ws, pl.part_off[q]);
        g.ld[q] = pl.ld[q];
    }
    g.items0 = pl.m_tiles[0] * pl.t_tiles * pl.splits[0];
    g.stages = pl.stages;
    g.stage_bytes = pl.stage_bytes;
    g.d_idx = pp->d_idx;
    g.h_idx = pp->h_idx;
    g.status = at<int>(ws, 0);
    g.wait_budget = dsa::kWaitBudgetCycles;
    dsa::ProjEpiParams e;
    memset(&e, 0, sizeof e);
    e.part0 = g.part[0];
    e.part1 = g.part[1];
    e.splits0 = pl.splits[0];
    e.splits1 = pl.splits[1];
    e.ld0 = pl.ld[0];
    e.ld1 = pl.ld[1];
    e.nt = pp->nt;
    e.d_idx = pp->d_idx;
    e.h_idx = pp->h_idx;
    e.rope_dim = pp->rope_dim;
    e.ln_eps = pp->ln_eps;
    e.rope_theta = pp->rope_theta;
    e.ln_gamma = ln_gamma;
    e.ln_beta = ln_beta;
    e.positions = positions;
    e.q_seq = kv->q_seq;
    e.seq_row0 = kv->seq_row0;
    e.page_table = kv->page_table;
    e.max_pages = kv->max_pages;
    e.page_size = kv->page_table ? kv->page_size : 1;
    e.cache_rows = kv->cache_rows;
    e.kidx_cache = static_cast<uint8_t *>(kidx_cache);
    e.k_scale = k_scale;
    e.q_idx = static_cast<uint8_t *>(q_idx);
    e.q_scale = q_scale;
    e.w = static_cast<uint16_t *>(w);
    e.q_f32 = q_f32;
    e.k_f32 = k_f32;
    e.w_f32 = w_f32;
    e.status = g.status;
    cudaError_t err = dsa::launch_project(xm, qm, km, pm, wm, g, e, static_cast<cudaStream_t>(stream));
    if (err != cudaSuccess) return cuda_fail(err, "indexer producer launch");
    return DSA_OK;
}

int dsa_check_status(void *ws, void *stream) {
    if (!ws) return fail(DSA_ERR_WORKSPACE, "ws is NULL");
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    cudaError_t e = cudaStreamSynchronize(st);
    if (e != cudaSuccess) return cuda_fail(e, "cudaStreamSynchronize");
    int v = 0;
    e = cudaMemcpy(&v, ws, sizeof v, cudaMemcpyDeviceToHost);
    if (e != cudaSuccess) return cuda_fail(e, "cudaMemcpy(status)");
    if (v != 0) {
        const int zero = 0;
        e = cudaMemcpy(ws, &zero, sizeof zero, cudaMemcpyHostToDevice);
        if (e != cudaSuccess) return cuda_fail(e, "cudaMemcpy(clear status)");
        fail(v, "device reported status %d", v);
    }
    return v;
}

const char *dsa_last_error(void) { return g_err; }

}  // extern "C"

// ---------------------------------------------------------------------------
// Fused indexer + TopK with scratch in a fixed device array.
//
// For callers that cannot call cudaMalloc -- code running where allocation is
// off limits (inside a framework whose allocator owns all device memory, a
// runtime with a fixed memory budget, a real-time path that must not enter
// the driver's allocator) -- the scratch this operation needs lives in one
// file-scope device array instead of a caller-provided workspace.  Every GPU
// that loads this library holds the array until the process exits.
// ---------------------------------------------------------------------------
namespace {

constexpr size_t kStaticScratchBytes = size_t(8) << 20;  // 8 MiB
static __device__ __align__(256) uint8_t g_static_scratch[kStaticScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_static_mu;
void *g_static_ptr[kMaxDevices] = {};

// Device address of the array for the current device, resolved once per
// device (cudaGetSymbolAddress, with that device current).  In host code the
// array's name is only a host-side stand-in, never a device address.
int static_scratch(void **out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
    if (dev < 0 || dev >= kMaxDevices) return fail(DSA_ERR_UNSUPPORTED, "device ordinal %d out of range", dev);
    std::lock_guard<std::mutex> lock(g_static_mu);
    if (!g_static_ptr[dev]) {
        void *ptr = nullptr;
        e = cudaGetSymbolAddress(&ptr, g_static_scratch);
        if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress");
        g_static_ptr[dev] = ptr;
    }
    *out = g_static_ptr[dev];
    return DSA_OK;
}

}  // namespace

extern "C" {

int dsa_indexer_topk_static(const dsa_params *p, const dsa_kv *kv, const void *q_idx, const void *w,
                            const void *kidx_cache, const float *k_scale, int32_t *idx,
                            int32_t *nsel, int32_t *status, void *stream) {
    int rc = check_params(p);
    if (!rc) rc = check_kv(p, kv);
    if (!rc) rc = check_indexer_inputs(p, q_idx, w, kidx_cache);
    if (rc) return rc;
    if (p->nq > 0 && !idx) return fail(DSA_ERR_INVALID_ARG, "idx is NULL");
    WsLayout wl;
    IndexerPlan pl;
    rc = layout_for(p, DSA_OP_INDEXER_TOPK, wl, &pl, nullptr, p->max_n);
    if (rc) return rc;
    if (wl.total > kStaticScratchBytes)
        return fail(DSA_ERR_UNSUPPORTED,
                    "dsa_indexer_topk_static: this shape needs %zu bytes of scratch, the fixed "
                    "array holds %zu (use dsa_indexer_topk with a workspace)",
                    wl.total, kStaticScratchBytes);
    void *ws = nullptr;
    rc = static_scratch(&ws);
    if (rc) return rc;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    // the array keeps the previous call's contents: start from a clear status
    // word (the per-call counters and histograms are cleared by run_indexer)
    cudaError_t e = cudaMemsetAsync(ws, 0, sizeof(int), st);
    if (e != cudaSuccess) return cuda_fail(e, "cudaMemsetAsync");
    rc = run_indexer(p, kv, dsa::kModeFused, q_idx, w, kidx_cache, k_scale, nullptr, 0, idx, nsel,
                     ws, wl, pl, st);
    if (rc) return rc;
    if (status) {
        e = cudaMemcpyAsync(status, ws, sizeof(int32_t), cudaMemcpyDeviceToDevice, st);
        if (e != cudaSuccess) return cuda_fail(e, "cudaMemcpyAsync(status)");
    }
    return DSA_OK;
}

}  // extern "C"
