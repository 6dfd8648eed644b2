// sparse_mla.cu -- sparse MQA-mode MLA attention on sm_100a.
//
// u_t = Attn(h_t, {c_s : s in I_t}) (DSA blog by marsggbo, section 3) in the
// MQA form of weight-absorbed MLA: every head attends to the same latent row,
// softmax(q . [c_kv; k_pe]^T) . c_kv ("DeepSeekV3.2之DSA" by yuyanqi,
// section 5.1).  Key = the whole 576-wide row, value = its first 512 columns.
//
// One CTA owns one query and a slice of at most 256 of its selected rows
// ("split"); all 128 heads form the MMA's M dimension.
//   pass 1  S[128 x R] = Q . K^T over 9 chunks of 64 key columns.  Each ring
//           stage holds a Q chunk (TMA tile, 16 KB) and the R rows' matching
//           128-byte pieces, gathered by eight warps (the softmax warps help:
//           they have nothing else to do yet) with 16-byte cp.async into the
//           128B-swizzled layout (the rows were first prefetched whole into
//           L2).  A gather thread owns one 16-byte piece of a fixed set of
//           rows, so its addresses are computed once for all nine chunks.
//           S accumulates in TMEM.
//   softmax one thread per head reads its S row from TMEM, takes the exact
//           max over the split, writes P = exp(S - max) into shared memory
//           as a pair of bf16 tiles P_hi = bf16(P), P_lo = bf16(P - P_hi)
//           (the A operands of pass 2) and keeps the row sum.  A single bf16
//           P would add ~1e-3 relative error on top of the ~1.7e-3 that the
//           bf16 output itself carries; the pair makes P exact to ~2^-16.
//   pass 2  O[128 x 512] = P_hi . V + P_lo . V, V re-gathered by warps 6-9
//           (32-row tiles, L2 hits) into an MN-major swizzled layout; O
//           takes all 512 TMEM columns, which is why S and O are not live at
//           the same time.
// The gather threads publish each staged chunk or tile as soon as the
// following one is requested (a lag of two chunks / one tile): publishing
// later kept the tensor cores waiting on data that had already landed.
// Epilogue: the softmax warps write columns 0..255 of O / l, the gather warps
// columns 256..511; each thread moves its head's row from TMEM to a staging
// row in shared memory and issues one 512-byte bulk store.  A split writes
// O / l as fp16 values times a power-of-two scale per (split, head, half
// row), chosen from that half row's largest magnitude: the values keep
// fp16's precision (2^-12 relative, far below the bf16 output's rounding)
// over the whole bf16 range of the latent cache, which plain fp16 (max
// 65504, subnormal below 6e-5) would not.  Each split also writes its
// log-sum-exp; the combine kernel merges splits by their log-sum-exp.  With
// one split the CTA writes the final output.
//
// The same kernel, with pass 1 only, computes the indexer distillation loss
// (DSA blog by marsggbo, sections 5.1 and 5.2): the loss's target is each
// head's attention distribution over the set, summed over heads and
// L1-normalised.  kMlaKlStats writes each (split, head)'s log-sum-exp;
// k9_kl_lse merges them into each head's log-sum-exp over the whole set;
// kMlaKlSum recomputes S and writes sum_h exp(S_h - lse_h) of every entry
// (a column sum over the 128 TMEM lanes); k10_kl_reduce takes the KL
// divergence against the softmax of the index scores.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp8.h>
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

#include "kernels.h"
#include "ptx.cuh"

namespace dsa {

namespace {

constexpr int kQChunkBytes = 128 * 128;             // 128 heads x 64 bf16
constexpr int kStageBytes = kQChunkBytes + kMlaMaxRows * 128;
constexpr int kNumKChunks = kDqk / 64;              // 9
constexpr int kVTileBytes = kMlaVRows * kDv * 2;    // 32 KB
constexpr int kVBlockBytes = kMlaVRows * 128;       // one 64-column block of a V tile
constexpr int kPBlockBytes = 128 * 128;             // 128 heads x 64 rows bf16
constexpr int kGatherWarp0 = 6;                     // warps 6..9 gather rows (and 0..3 in pass 1)
constexpr int kGatherThreads = 128;
constexpr int kPass1Threads = 256;                  // pass-1 gather threads (warps 0-3, 6-9)
constexpr int kPass1Rows = kMlaMaxRows / (kPass1Threads / 8);  // rows per pass-1 gather thread
constexpr int kEpiPitch = 512 + 16;                 // epilogue staging row pitch (bytes)
constexpr int kEpiGroupBytes = 128 * kEpiPitch;     // one epilogue group's staging rows
constexpr int kGatherLag = 2;                       // pass-1 chunks a gather thread publishes behind its newest
constexpr int kVLag = 1;                            // pass-2 tiles a gather thread publishes behind its newest

struct MlaSmem {
    uint64_t full[kMlaStages];
    uint64_t empty[kMlaStages];
    uint64_t s_full;
    uint64_t p_full;
    uint64_t v_full[kMlaVStages];
    uint64_t v_empty[kMlaVStages];
    uint64_t o_full;
    uint32_t tmem_base;
    volatile int32_t abort;
    int32_t nvalid;
    int32_t rows[kMlaMaxRows];
    uint8_t valid[kMlaMaxRows];
    uint32_t vmask[kMlaMaxRows / 32];  // bit j of word w: entry 32w + j is valid
    float inv_l[128];                  // 1 / row sum per head (softmax -> second epilogue group)
};

static_assert(sizeof(MlaSmem) <= 2048, "MlaSmem must fit the reserve in mla_layout()");
static_assert(2 * kEpiGroupBytes <= 2 * 128 * kMlaMaxRows * 2 + kMlaVStages * kVTileBytes,
              "epilogue staging must fit the pass-2 area (free once O is complete)");

__device__ __forceinline__ uint8_t *align1024(uint8_t *p) {
    return reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}

// Named barrier `id` over `count` threads that also ANDs `pred` across them.
__device__ __forceinline__ bool bar_and(int id, int count, bool pred) {
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\tsetp.ne.u32 q, %1, 0;\n\t"
        "bar.red.and.pred p, %2, %3, q;\n\tselp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(r)
        : "r"(static_cast<uint32_t>(pred)), "r"(id), "r"(count)
        : "memory");
    return r != 0;
}

__device__ __forceinline__ uint32_t pack_half2(float lo, float hi) {
    const uint32_t a = __half_as_ushort(__float2half_rn(lo));
    const uint32_t b = __half_as_ushort(__float2half_rn(hi));
    return a | (b << 16);
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    const uint32_t a = __bfloat16_as_ushort(__float2bfloat16_rn(lo));
    const uint32_t b = __bfloat16_as_ushort(__float2bfloat16_rn(hi));
    return a | (b << 16);
}

// Sixteen e4m3 codes (one 16-byte load) times a power-of-two row scale as
// sixteen bf16 values (two 16-byte shared-memory pieces).  e4m3 -> f16 is
// exact, the power-of-two product is exact in fp32 and a value with 4
// significant bits is exact in bf16: the pieces equal the cache's values.
__device__ __forceinline__ void fp8x16_to_bf16x16(uint4 codes, float sc, uint4 &lo, uint4 &hi) {
    const uint32_t w[4] = {codes.x, codes.y, codes.z, codes.w};
    uint32_t o[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const __nv_fp8x2_storage_t pair = static_cast<__nv_fp8x2_storage_t>((w[i >> 1] >> (16 * (i & 1))) & 0xFFFFu);
        const __half2 h = __half2(__nv_cvt_fp8x2_to_halfraw2(pair, __NV_E4M3));
        const float2 f = __half22float2(h);
        o[i] = pack_bf16x2(f.x * sc, f.y * sc);
    }
    lo = make_uint4(o[0], o[1], o[2], o[3]);
    hi = make_uint4(o[4], o[5], o[6], o[7]);
}

__device__ __forceinline__ uint4 ldg_u4(const uint8_t *p) {
    return __ldg(reinterpret_cast<const uint4 *>(p));
}

constexpr int kFp8Rows = kMlaMaxRows / (kPass1Threads / 4);  // pass-1 rows per gather thread (FP8)

// Pass-1 gathers from an FP8 cache.  Gather thread gt owns the 16-byte code
// piece j4 = gt % 4 (codes 16 j4 .. 16 j4 + 15 of each 64-column chunk, two
// bf16 pieces of the swizzled stage) of rows gt / 4 + 64 k; its loads run
// two chunks ahead in registers; a chunk is published once this thread's
// stores of it are done.
__device__ bool gather_pass1_fp8(const MlaParams &a, MlaSmem &sm, uint8_t *ring, int gt, int Rp) {
    const int j4 = gt & 3, r0 = gt >> 2, lane = threadIdx.x & 31;
    const uint8_t *src[kFp8Rows];
    uint32_t dst0[kFp8Rows], dst1[kFp8Rows];
    float sc[kFp8Rows];
#pragma unroll
    for (int k = 0; k < kFp8Rows; ++k) {
        const int r = r0 + 64 * k;
        src[k] = a.kv8 + static_cast<int64_t>(sm.rows[r]) * a.kv8_row_bytes + j4 * 16;
        dst0[k] = static_cast<uint32_t>(r * 128 + (((2 * j4) ^ (r & 7)) << 4));
        dst1[k] = static_cast<uint32_t>(r * 128 + (((2 * j4 + 1) ^ (r & 7)) << 4));
        sc[k] = sm.valid[r] ? a.kv_scale[sm.rows[r]] : 0.f;
    }
    // registers two chunks ahead, shifted down each chunk (a rolled loop:
    // the unrolled one stalled on instruction fetch)
    uint4 b0[kFp8Rows], b1[kFp8Rows], b2[kFp8Rows];
    auto load = [&](int c, uint4 (&b)[kFp8Rows]) {
#pragma unroll
        for (int k = 0; k < kFp8Rows; ++k)
            b[k] = (r0 + 64 * k < Rp) ? ldg_u4(src[k] + c * 64) : make_uint4(0u, 0u, 0u, 0u);
    };
    load(0, b0);
    load(1, b1);
    bool ok = true;
#pragma unroll 1
    for (int c = 0; c < kNumKChunks; ++c) {
        if (c + 2 < kNumKChunks) load(c + 2, b2);
        const int s = c % kMlaStages;
        const uint32_t ph = (c / kMlaStages) & 1;
        ok = ok && __all_sync(0xffffffffu, mbar_wait(&sm.empty[s], ph ^ 1, a.wait_budget) && !sm.abort);
        if (ok) {
            uint8_t *kst = ring + s * kStageBytes + kQChunkBytes;
#pragma unroll
            for (int k = 0; k < kFp8Rows; ++k)
                if (r0 + 64 * k < Rp) {
                    uint4 lo, hi;
                    fp8x16_to_bf16x16(b0[k], sc[k], lo, hi);
                    *reinterpret_cast<uint4 *>(kst + dst0[k]) = lo;
                    *reinterpret_cast<uint4 *>(kst + dst1[k]) = hi;
                }
        }
        fence_proxy_async_smem();
        __syncwarp();
        // tests only: the first CTA never publishes chunk 0
        const bool skip = a.inject != 0 && blockIdx.x == 0 && c == 0;
        if (lane == 0 && !skip) mbar_arrive(&sm.full[s]);
#pragma unroll
        for (int k = 0; k < kFp8Rows; ++k) {
            b0[k] = b1[k];
            b1[k] = b2[k];
        }
    }
    return ok;
}

// Pass-1 row gathers by one of the kPass1Threads gather threads (gt): it
// owns the 16-byte piece j = gt % 8 of rows gt / 8 + 32 k, and copies that
// piece of chunk c (key columns 64c .. 64c+63) of each of its rows into the
// stage's K area, 128B-swizzled.  Chunk c - kGatherLag is published (the
// warp arrives on its full barrier) once this thread's copies of it landed.
// Returns false if a wait timed out.
__device__ bool gather_pass1(const MlaParams &a, MlaSmem &sm, uint8_t *ring, int gt, int Rp) {
    const int j = gt & 7, r0 = gt >> 3, lane = threadIdx.x & 31;
    const uint16_t *src[kPass1Rows];
    uint32_t dst[kPass1Rows];
#pragma unroll
    for (int k = 0; k < kPass1Rows; ++k) {
        const int r = r0 + 32 * k;
        src[k] = a.kv + static_cast<int64_t>(sm.rows[r]) * a.kv_row_stride + j * 8;
        dst[k] = static_cast<uint32_t>(r * 128 + ((j ^ (r & 7)) << 4));
    }
    bool ok = true;
    for (int c = 0; c < kNumKChunks + kGatherLag; ++c) {
        if (c < kNumKChunks) {
            const int s = c % kMlaStages;
            const uint32_t ph = (c / kMlaStages) & 1;
            ok = ok && __all_sync(0xffffffffu, mbar_wait(&sm.empty[s], ph ^ 1, a.wait_budget) && !sm.abort);
            if (ok) {
                uint8_t *kst = ring + s * kStageBytes + kQChunkBytes;
#pragma unroll
                for (int k = 0; k < kPass1Rows; ++k)
                    if (r0 + 32 * k < Rp) cp_async16(kst + dst[k], src[k] + c * 64);
            }
            cp_async_commit();
        }
        if (c >= kGatherLag) {
            // chunk c - lag is complete for this thread: publish it
            if (c < kNumKChunks) cp_async_wait<kGatherLag>();
            else cp_async_wait<0>();
            fence_proxy_async_smem();
            __syncwarp();
            // tests only: the first CTA never publishes chunk 0
            const bool skip = a.inject != 0 && blockIdx.x == 0 && c == kGatherLag;
            if (lane == 0 && !skip) mbar_arrive(&sm.full[(c - kGatherLag) % kMlaStages]);
        }
    }
    return ok;
}

// O / l of this thread's head row, columns [c_begin, c_begin + 256): TMEM ->
// registers -> this thread's staging row in shared memory (`srow`, 512 bytes,
// rows kEpiPitch apart so that the 16-byte writes of a warp spread over the
// banks) -> one 512-byte bulk store into the row of the output (bf16) or of
// the split partials (fp16 times 2^e, e from the half row's largest
// magnitude m: m * 2^-e lies in [2^14, 2^15), below fp16's 65504).  The TMEM
// loads are warp-collective: every lane runs them; only the stores are
// skipped for padding heads (hrow >= h).  The caller waits for the bulk
// store (bulk_wait_read) before the CTA exits.
__device__ void store_output(const MlaParams &a, uint32_t lane_addr, int hrow, int q, int wq, int sp,
                             float inv_l, int c_begin, uint8_t *srow) {
    const bool partial = a.splits > 1;
    float mul = inv_l;
    if (partial) {
        float mx = 0.f;
        for (int c1 = c_begin; c1 < c_begin + 256; c1 += 64) {
            uint32_t v2[2][32];
            tmem_ld32(lane_addr + c1, v2[0]);
            tmem_ld32(lane_addr + c1 + 32, v2[1]);
            tmem_wait_ld();
#pragma unroll
            for (int j = 0; j < 32; ++j)
                mx = fmaxf(mx, fmaxf(fabsf(__uint_as_float(v2[0][j])), fabsf(__uint_as_float(v2[1][j]))));
        }
        mx *= inv_l;
        // exponent of mx minus 14 (0 for an all-zero row); a subnormal or
        // tiny mx is clamped (its values then stay below 2^14, still exact
        // enough), so that both 2^-e and 2^e are normal floats
        int e = mx > 0.f ? static_cast<int>((__float_as_uint(mx) >> 23) & 0xFFu) - 127 - 14 : 0;
        e = min(max(e, -100), 113);
        mul = inv_l * __int_as_float((127 - e) << 23);
        if (hrow < a.h)
            a.part_scale[((static_cast<int64_t>(wq) * a.splits + sp) * 128 + hrow) * 2 + (c_begin >> 8)] =
                __int_as_float((127 + e) << 23);
    }
    for (int c1 = c_begin; c1 < c_begin + 256; c1 += 64) {
        uint32_t v2[2][32];
        tmem_ld32(lane_addr + c1, v2[0]);
        tmem_ld32(lane_addr + c1 + 32, v2[1]);
        tmem_wait_ld();
#pragma unroll
        for (int g = 0; g < 8; ++g) {
            const uint32_t *u = &v2[g >> 2][(g & 3) * 8];
            uint32_t w[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const float x0 = __uint_as_float(u[2 * e]) * mul, x1 = __uint_as_float(u[2 * e + 1]) * mul;
                w[e] = partial ? pack_half2(x0, x1) : pack_bf16x2(x0, x1);
            }
            *reinterpret_cast<uint4 *>(srow + (c1 - c_begin) * 2 + g * 16) = make_uint4(w[0], w[1], w[2], w[3]);
        }
    }
    fence_proxy_async_smem();  // the staging row is read by the bulk copy
    if (hrow < a.h) {
        uint16_t *dst = !partial
                            ? a.out + (static_cast<int64_t>(q) * a.h + hrow) * kDv
                            : a.part_o + ((static_cast<int64_t>(wq) * a.splits + sp) * 128 + hrow) * kDv;
        bulk_store(dst + c_begin, srow, 512);
        bulk_commit();
    }
}

// Column sums of a warp's 32 x 32 block: lane l holds row l (v[0..31]);
// afterwards v[0] of lane j is the sum of column j over the 32 rows.  Each
// step halves the columns a lane keeps and adds its partner's half (31
// shuffles in all).
__device__ __forceinline__ float warp_column_sum(float (&v)[32]) {
    const int lane = threadIdx.x & 31;
#pragma unroll
    for (int w = 16; w >= 1; w >>= 1) {
        const bool upper = (lane & w) != 0;
#pragma unroll
        for (int j = 0; j < w; ++j) {
            const float send = upper ? v[j] : v[j + w];
            const float keep = upper ? v[j + w] : v[j];
            v[j] = keep + __shfl_xor_sync(0xffffffffu, send, w);
        }
    }
    return v[0];
}

}  // namespace

template <int MODE, bool KV8>
__global__ void __launch_bounds__(kMlaThreads, 1)
    k3_sparse_mla(const __grid_constant__ CUtensorMap qmap, const MlaParams a) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *base = align1024(smem_raw);
    const MlaLayout L = mla_layout();
    MlaSmem &sm = *reinterpret_cast<MlaSmem *>(base + L.misc);
    uint8_t *ring = base + L.ring;
    uint8_t *ptile = base + L.p_tile;
    uint8_t *plo = base + L.p_lo;
    uint8_t *vring = base + L.v_ring;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int wq = blockIdx.x / a.splits;  // query within this wave
    const int sp = blockIdx.x % a.splits;
    const int q = a.q0 + wq;
    const int e0 = sp * a.rows_per_split;
    // the entries of this split (dense: positions e0.., up to the query's n,
    // which is read after the dependency wait below)
    int R = max(min(a.rows_per_split, a.topk - e0), 0);
    const int hbox = a.h < 128 ? a.h : 128;

    if (tid == 0) {
        sm.abort = 0;
        sm.nvalid = 0;
        for (int s = 0; s < kMlaStages; ++s) {
            mbar_init(&sm.full[s], 1 + kPass1Threads / 32);  // Q TMA (with its bytes) + eight gather warps
            mbar_init(&sm.empty[s], 1);
        }
        mbar_init(&sm.s_full, 1);
        mbar_init(&sm.p_full, 4);
        for (int v = 0; v < kMlaVStages; ++v) {
            mbar_init(&sm.v_full[v], 4);     // four gather warps
            mbar_init(&sm.v_empty[v], 1);
        }
        mbar_init(&sm.o_full, 1);
        fence_mbar_init();
    }
    // rows h..127 of every Q chunk are never written by TMA: zero them once
    if (hbox < 128) {
        for (int s = 0; s < kMlaStages; ++s)
            for (int i = tid; i < (128 - hbox) * 8; i += blockDim.x)
                *reinterpret_cast<uint4 *>(ring + s * kStageBytes + hbox * 128 + i * 16) = make_uint4(0, 0, 0, 0);
    }
    if (warp == 5) {
        tmem_alloc(&sm.tmem_base, 512);
        tmem_relinquish();
    }
    // everything above touches no input: with programmatic dependent launch
    // it overlaps the end of the kernel that produced the indices
    grid_dependency_wait();
    // cache rows of this split's entries (invalid entries read row 0 and are
    // masked; P = 0 there)
    const int n = a.q_n[q];
    const int seq = a.q_seq[q];
    if (a.dense) R = max(min(R, min(n, a.topk) - e0), 0);
    const int Rp = (R + 15) & ~15;  // MMA N (multiple of 16)
    __syncthreads();
    for (int i = tid; i < kMlaMaxRows; i += blockDim.x) {
        int32_t row = 0;
        uint8_t ok = 0;
        if (i < R) {
            const int s = a.dense ? e0 + i : a.idx[static_cast<int64_t>(q) * a.topk + e0 + i];
            if (s >= n) record_status(a.status, DSA_ERR_DEVICE_CHECK);
            if (s >= 0 && s < n) {
                int64_t r;
                if (a.page_table)
                    r = static_cast<int64_t>(a.page_table[static_cast<int64_t>(seq) * a.max_pages + s / a.page_size]) * a.page_size + s % a.page_size;
                else
                    r = a.seq_row0[seq] + s;
                if (r >= 0 && r < a.cache_rows) {
                    row = static_cast<int32_t>(r);
                    ok = 1;
                } else {
                    record_status(a.status, DSA_ERR_DEVICE_CHECK);
                }
            }
        }
        sm.rows[i] = row;
        sm.valid[i] = ok;
        const unsigned bits = __ballot_sync(0xffffffffu, ok != 0);
        if ((i & 31) == 0) sm.vmask[i >> 5] = bits;
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = sm.tmem_base;

    if (Rp > 0) {
        if (warp == 4) {
            // ------------------------------------------ Q chunks by TMA
            const uint32_t qbytes = static_cast<uint32_t>(hbox) * 128u;
            if (lane == 0) {
                int c_end = 0;  // chunks whose Q tile was requested
                for (int c = 0; c < kNumKChunks; ++c) {
                    const int s = c % kMlaStages;
                    const uint32_t ph = (c / kMlaStages) & 1;
                    if (sm.abort || !mbar_wait(&sm.empty[s], ph ^ 1, a.wait_budget)) {
                        record_status(a.status, DSA_ERR_TIMEOUT);
                        sm.abort = 1;
                        break;
                    }
                    mbar_arrive_expect_tx(&sm.full[s], qbytes);
                    tma_load_2d(ring + s * kStageBytes, &qmap, &sm.full[s], c * 64, q * a.h);
                    c_end = c + 1;
                }
                // the requested tiles land before the CTA may exit: wait
                // (bounded) for the newest phase of each stage; a stage whose
                // row pieces were never published runs out the budget, which
                // happens only after a wait elsewhere already failed
                for (int c = max(c_end - kMlaStages, 0); c < c_end; ++c)
                    mbar_wait(&sm.full[c % kMlaStages], static_cast<uint32_t>(c / kMlaStages) & 1u, a.wait_budget);
            }
        } else if (warp >= kGatherWarp0) {
            // ------------------------------------------ row gathers (cp.async)
            const int gt = tid - kGatherWarp0 * 32;  // 0..127
            for (int i = gt; i < R; i += kGatherThreads)
                if (sm.valid[i]) {
                    if constexpr (KV8)
                        prefetch_l2_bulk(a.kv8 + static_cast<int64_t>(sm.rows[i]) * a.kv8_row_bytes, kDqk);
                    else
                        prefetch_l2_bulk(a.kv + static_cast<int64_t>(sm.rows[i]) * a.kv_row_stride, kDqk * 2);
                }
            bool ok = KV8 ? gather_pass1_fp8(a, sm, ring, kPass1Threads / 2 + gt, Rp)
                          : gather_pass1(a, sm, ring, kPass1Threads / 2 + gt, Rp);
            if constexpr (MODE != kMlaAttn) {
                if (!ok && lane == 0) {
                    record_status(a.status, DSA_ERR_TIMEOUT);
                    sm.abort = 1;
                }
            } else {
                // pass 2: V tiles reuse the pass-1 area once every pass-1 MMA is
                // done.  Thread gt owns row r = gt / 4 of every tile and its
                // pieces u, u + 4, ..., u + 60 (u = gt % 4): one row lookup per tile.
                ok = ok && __all_sync(0xffffffffu, mbar_wait(&sm.s_full, 0, a.wait_budget) && !sm.abort);
                const int vr = gt >> 2, vu = gt & 3;
                const int nvt = (Rp + kMlaVRows - 1) / kMlaVRows;
                if constexpr (KV8) {
                    // FP8 rows: this thread's 8 code pieces of 16 bytes
                    // (u = vu + 4 m: value columns 16 u .. 16 u + 15, the bf16
                    // pieces 2u and 2u + 1) of row vr of a tile, loaded into
                    // registers one tile ahead and converted
                    uint4 cur[8], nxt[8];
                    float csc = 0.f, nsc = 0.f;
                    auto vload = [&](int vt, uint4 (&b)[8], float &sc) {
                        const int rr = vt * kMlaVRows + vr;
                        const uint8_t *vsrc = a.kv8 + static_cast<int64_t>(sm.rows[rr]) * a.kv8_row_bytes;
                        sc = sm.valid[rr] ? a.kv_scale[sm.rows[rr]] : 0.f;
#pragma unroll
                        for (int m = 0; m < 8; ++m) b[m] = ldg_u4(vsrc + (vu + 4 * m) * 16);
                    };
                    if (nvt > 0) vload(0, cur, csc);
                    for (int vt = 0; vt < nvt; ++vt) {
                        if (vt + 1 < nvt) vload(vt + 1, nxt, nsc);
                        const int v = vt % kMlaVStages;
                        const uint32_t ph = (vt / kMlaVStages) & 1;
                        ok = ok && __all_sync(0xffffffffu, mbar_wait(&sm.v_empty[v], ph ^ 1, a.wait_budget) && !sm.abort);
                        if (ok) {
                            uint8_t *vdst = vring + v * kVTileBytes + vr * 128;
#pragma unroll
                            for (int m = 0; m < 8; ++m) {
                                const int u = vu + 4 * m;
                                const int pc0 = 2 * u, pc1 = 2 * u + 1;  // bf16 pieces (8 columns each)
                                uint4 lo, hi;
                                fp8x16_to_bf16x16(cur[m], csc, lo, hi);
                                *reinterpret_cast<uint4 *>(vdst + (pc0 >> 3) * kVBlockBytes + (((pc0 & 7) ^ (vr & 7)) << 4)) = lo;
                                *reinterpret_cast<uint4 *>(vdst + (pc1 >> 3) * kVBlockBytes + (((pc1 & 7) ^ (vr & 7)) << 4)) = hi;
                            }
                        }
                        fence_proxy_async_smem();
                        __syncwarp();
                        if (lane == 0) mbar_arrive(&sm.v_full[v]);
#pragma unroll
                        for (int m = 0; m < 8; ++m) cur[m] = nxt[m];
                        csc = nsc;
                    }
                } else {
                    for (int vt = 0; vt < nvt + kVLag; ++vt) {
                        if (vt < nvt) {
                            const int v = vt % kMlaVStages;
                            const uint32_t ph = (vt / kMlaVStages) & 1;
                            ok = ok && __all_sync(0xffffffffu, mbar_wait(&sm.v_empty[v], ph ^ 1, a.wait_budget) && !sm.abort);
                            if (ok) {
                                uint8_t *vdst = vring + v * kVTileBytes + vr * 128;
                                const uint16_t *vsrc = a.kv + static_cast<int64_t>(sm.rows[vt * kMlaVRows + vr]) * a.kv_row_stride;
#pragma unroll
                                for (int m = 0; m < 16; ++m) {
                                    const int pc = vu + 4 * m;  // 16-byte piece of the 512 value columns
                                    const int blk = pc >> 3, j = pc & 7;
                                    cp_async16(vdst + blk * kVBlockBytes + ((j ^ (vr & 7)) << 4), vsrc + pc * 8);
                                }
                            }
                            cp_async_commit();
                        }
                        if (vt >= kVLag && vt - kVLag < nvt) {
                            if (vt < nvt) cp_async_wait<kVLag>();
                            else cp_async_wait<0>();
                            fence_proxy_async_smem();
                            __syncwarp();
                            if (lane == 0) mbar_arrive(&sm.v_full[(vt - kVLag) % kMlaVStages]);
                        }
                    }
                }
                if (!ok && lane == 0) {
                    record_status(a.status, DSA_ERR_TIMEOUT);
                    sm.abort = 1;
                }
                // second epilogue group: value columns 256..511
                const int hrow = (warp & 3) * 32 + lane;
                const uint32_t lane_addr = tmem + (static_cast<uint32_t>((warp & 3) * 32) << 16);
                ok = __all_sync(0xffffffffu, mbar_wait(&sm.o_full, 0, a.wait_budget) && !sm.abort);
                // inv_l of every head is in shared memory; both groups agree on ok
                // (the epilogue's named barriers need all 128 threads of a group)
                ok = bar_and(3, 256, ok);
                if (ok) {
                    tc_fence_after();
                    store_output(a, lane_addr, hrow, q, wq, sp, sm.inv_l[hrow], 256,
                                 ptile + kEpiGroupBytes + hrow * kEpiPitch);
                }
            }
        } else if (warp == 5) {
            // ------------------------------------------------ MMA issuer
            if (lane == 0) {
                bool ok = true;
                const uint32_t idesc1 = make_idesc(1, 1, 0, 0, 128, static_cast<uint32_t>(Rp));
                for (int c = 0; c < kNumKChunks; ++c) {
                    const int s = c % kMlaStages;
                    const uint32_t ph = (c / kMlaStages) & 1;
                    if (sm.abort || !mbar_wait(&sm.full[s], ph, a.wait_budget)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t qa = smem_u32(ring + s * kStageBytes);
                    const uint32_t ka = qa + kQChunkBytes;
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk) {
                        const uint64_t ad = make_sdesc(qa + kk * 32, 16, 1024, kSwizzle128B);
                        const uint64_t bd = make_sdesc(ka + kk * 32, 16, 1024, kSwizzle128B);
                        mma_bf16_ss(tmem, ad, bd, idesc1, (c > 0 || kk > 0) ? 1u : 0u);
                    }
                    tc_commit(&sm.empty[s]);
                }
                tc_commit(&sm.s_full);
                if constexpr (MODE != kMlaAttn) {
                    if (!ok) {
                        record_status(a.status, DSA_ERR_TIMEOUT);
                        sm.abort = 1;
                    }
                    // every MMA issued completes before TMEM is freed
                    if (!mbar_wait(&sm.s_full, 0, a.wait_budget)) record_status(a.status, DSA_ERR_TIMEOUT);
                } else {
                    if (ok && mbar_wait(&sm.p_full, 0, a.wait_budget) && !sm.abort) {
                        tc_fence_after();
                        // B = V tile, MN-major: LBO = distance between 64-column
                        // blocks, SBO = 1 KB between 8-row groups.  A = P_hi, P_lo:
                        // K-major, 64-row blocks of 16 KB, 16-row k-steps 32 B apart.
                        const uint32_t idesc2 = make_idesc(1, 1, 0, 1, 128, 256);
                        const int nvt = (Rp + kMlaVRows - 1) / kMlaVRows;
                        for (int vt = 0; vt < nvt; ++vt) {
                            const int v = vt % kMlaVStages;
                            const uint32_t ph = (vt / kMlaVStages) & 1;
                            if (sm.abort || !mbar_wait(&sm.v_full[v], ph, a.wait_budget)) {
                                ok = false;
                                break;
                            }
                            tc_fence_after();
                            const int row0 = vt * kMlaVRows;
                            const uint32_t poff = (row0 >> 6) * kPBlockBytes + ((row0 & 63) >> 4) * 32;
                            const uint32_t pa_hi = smem_u32(ptile) + poff;
                            const uint32_t pa_lo = smem_u32(plo) + poff;
                            const uint32_t va = smem_u32(vring + v * kVTileBytes);
                            const int ksteps = min(kMlaVRows / 16, (Rp - row0) / 16);
                            for (int ks = 0; ks < ksteps; ++ks) {
                                const uint64_t ad_hi = make_sdesc(pa_hi + ks * 32, 16, 1024, kSwizzle128B);
                                const uint64_t ad_lo = make_sdesc(pa_lo + ks * 32, 16, 1024, kSwizzle128B);
#pragma unroll
                                for (int nh = 0; nh < 2; ++nh) {
                                    const uint64_t bd = make_sdesc(va + nh * 4 * kVBlockBytes + ks * 2048,
                                                                   kVBlockBytes, 1024, kSwizzle128B);
                                    mma_bf16_ss(tmem + nh * 256, ad_hi, bd, idesc2, (vt > 0 || ks > 0) ? 1u : 0u);
                                    mma_bf16_ss(tmem + nh * 256, ad_lo, bd, idesc2, 1u);
                                }
                            }
                            tc_commit(&sm.v_empty[v]);
                        }
                    }
                    tc_commit(&sm.o_full);
                    if (!ok) {
                        record_status(a.status, DSA_ERR_TIMEOUT);
                        sm.abort = 1;
                    }
                    // every MMA issued completes (o_full's phase) before TMEM is freed
                    if (!mbar_wait(&sm.o_full, 0, a.wait_budget)) record_status(a.status, DSA_ERR_TIMEOUT);
                }
            }
        } else if (warp < 4) {
            // ------------------- pass-1 gathers, softmax, then epilogue
            bool ok = KV8 ? gather_pass1_fp8(a, sm, ring, tid, Rp) : gather_pass1(a, sm, ring, tid, Rp);
            const int hrow = warp * 32 + lane;  // head = TMEM lane
            const uint32_t lane_addr = tmem + (static_cast<uint32_t>(warp * 32) << 16);
            ok = __all_sync(0xffffffffu, ok && mbar_wait(&sm.s_full, 0, a.wait_budget) && !sm.abort);
            if constexpr (MODE == kMlaKlSum) {
                // sum over heads of exp(S_h - lse_h), entry by entry: this
                // warp's 32 heads per block of 32 columns, then the four
                // warps' sums (the ring is free once pass 1 is complete)
                float *colsum = reinterpret_cast<float *>(ptile);  // [4][kMlaMaxRows]
                const float lse_h = hrow < a.h ? a.kl_lse[static_cast<int64_t>(q) * 128 + hrow] : -INFINITY;
                const bool live = lse_h > -INFINITY && lse_h < INFINITY;
                const float off = live ? lse_h * 1.4426950408889634f : 0.f;
                if (ok) {
                    tc_fence_after();
                    for (int c0 = 0; c0 < Rp; c0 += 32) {
                        uint32_t v[32];
                        tmem_ld32(lane_addr + c0, v);
                        const uint32_t vm = sm.vmask[c0 >> 5];
                        tmem_wait_ld();
                        float e[32];
#pragma unroll
                        for (int j = 0; j < 32; ++j)
                            e[j] = (live && ((vm >> j) & 1u))
                                       ? fast_exp2(fmaf(__uint_as_float(v[j]), a.scale_log2, -off))
                                       : 0.f;
                        colsum[warp * kMlaMaxRows + c0 + lane] = warp_column_sum(e);
                    }
                }
                ok = bar_and(1, 128, ok);
                if (ok) {
                    float *dst = a.kl_a + static_cast<int64_t>(q) * a.topk + e0;
                    for (int i = tid; i < R; i += 128)
                        dst[i] = (colsum[i] + colsum[kMlaMaxRows + i]) +
                                 (colsum[2 * kMlaMaxRows + i] + colsum[3 * kMlaMaxRows + i]);
                } else if (lane == 0) {
                    record_status(a.status, DSA_ERR_TIMEOUT);
                }
            } else {
                float m = -INFINITY, l = 0.f;
                if (ok) {
                    tc_fence_after();
                    // row max: four independent partial maxima, 32 columns per TMEM load
                    float m4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
                    for (int c0 = 0; c0 < Rp; c0 += 32) {
                        uint32_t v[32];
                        tmem_ld32(lane_addr + c0, v);
                        const uint32_t vm = sm.vmask[c0 >> 5];
                        tmem_wait_ld();
#pragma unroll
                        for (int j = 0; j < 32; ++j)
                            m4[j & 3] = fmaxf(m4[j & 3], ((vm >> j) & 1u) ? __uint_as_float(v[j]) : -INFINITY);
                    }
                    m = fmaxf(fmaxf(m4[0], m4[1]), fmaxf(m4[2], m4[3]));
                    const float mlog = (m == -INFINITY) ? 0.f : m * a.scale_log2;
                    float l4[4] = {0.f, 0.f, 0.f, 0.f};
                    for (int c0 = 0; c0 < Rp; c0 += 32) {
                        uint32_t v[32];
                        tmem_ld32(lane_addr + c0, v);
                        const uint32_t vm = sm.vmask[c0 >> 5];
                        tmem_wait_ld();
                        float p[32];
#pragma unroll
                        for (int j = 0; j < 32; ++j) {
                            p[j] = ((vm >> j) & 1u) ? fast_exp2(fmaf(__uint_as_float(v[j]), a.scale_log2, -mlog)) : 0.f;
                            l4[j & 3] += p[j];
                        }
                        if constexpr (MODE == kMlaAttn) {
                            // P row `hrow`, columns c0..c0+31: K-major 128B-swizzled blocks of 64
                            const uint32_t rowoff = (c0 >> 6) * kPBlockBytes + hrow * 128;
#pragma unroll
                            for (int g8 = 0; g8 < 4; ++g8) {
                                const int ch = ((c0 & 63) >> 3) + g8;  // 16-byte chunk within the 128B row
                                uint32_t hi[4], lo[4];
#pragma unroll
                                for (int e = 0; e < 4; ++e) {
                                    // one paired conversion each for P_hi and P_lo
                                    const float a0 = p[g8 * 8 + 2 * e], a1 = p[g8 * 8 + 2 * e + 1];
                                    const __nv_bfloat162 h2 = __floats2bfloat162_rn(a0, a1);
                                    const float2 hf = __bfloat1622float2(h2);
                                    const __nv_bfloat162 l2 = __floats2bfloat162_rn(a0 - hf.x, a1 - hf.y);
                                    hi[e] = *reinterpret_cast<const uint32_t *>(&h2);
                                    lo[e] = *reinterpret_cast<const uint32_t *>(&l2);
                                }
                                const uint32_t off = rowoff + ((ch ^ (hrow & 7)) << 4);
                                *reinterpret_cast<uint4 *>(ptile + off) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
                                *reinterpret_cast<uint4 *>(plo + off) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
                            }
                        }
                    }
                    l = (l4[0] + l4[1]) + (l4[2] + l4[3]);
                }
                if constexpr (MODE == kMlaKlStats) {
                    if (ok) {
                        if (hrow < a.h)
                            a.part_lse[(static_cast<int64_t>(wq) * a.splits + sp) * 128 + hrow] =
                                l > 0.f ? m * a.scale + logf(l) : -INFINITY;
                    } else if (lane == 0) {
                        record_status(a.status, DSA_ERR_TIMEOUT);
                    }
                } else {
                    fence_proxy_async_smem();
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&sm.p_full);
                    const bool has = l > 0.f;
                    const float inv_l = has ? 1.f / l : 0.f;
                    sm.inv_l[hrow] = inv_l;
                    ok = ok && __all_sync(0xffffffffu, mbar_wait(&sm.o_full, 0, a.wait_budget) && !sm.abort);
                    ok = bar_and(3, 256, ok);  // hand inv_l to the second group; agree on ok
                    if (ok) {
                        tc_fence_after();
                        const float lse_v = has ? (m * a.scale + logf(l)) : -INFINITY;
                        if (hrow < a.h) {
                            if (a.splits == 1) a.lse[static_cast<int64_t>(q) * a.h + hrow] = lse_v;
                            else a.part_lse[(static_cast<int64_t>(wq) * a.splits + sp) * 128 + hrow] = lse_v;
                        }
                        store_output(a, lane_addr, hrow, q, wq, sp, inv_l, 0, ptile + hrow * kEpiPitch);
                    } else if (lane == 0) {
                        record_status(a.status, DSA_ERR_TIMEOUT);
                    }
                }
            }
        }
    } else if (warp < 4) {
        // empty split: no rows at all
        const int hrow = warp * 32 + lane;
        if constexpr (MODE == kMlaKlStats) {
            if (hrow < a.h) a.part_lse[(static_cast<int64_t>(wq) * a.splits + sp) * 128 + hrow] = -INFINITY;
        } else if (MODE == kMlaAttn && hrow < a.h) {
            if (a.splits == 1) {
                uint16_t *o = a.out + (static_cast<int64_t>(q) * a.h + hrow) * kDv;
                for (int c0 = 0; c0 < kDv; c0 += 8) *reinterpret_cast<uint4 *>(o + c0) = make_uint4(0, 0, 0, 0);
                a.lse[static_cast<int64_t>(q) * a.h + hrow] = -INFINITY;
            } else {
                const int64_t row = (static_cast<int64_t>(wq) * a.splits + sp) * 128 + hrow;
                uint16_t *o = a.part_o + row * kDv;
                for (int c0 = 0; c0 < kDv; c0 += 8) *reinterpret_cast<uint4 *>(o + c0) = make_uint4(0, 0, 0, 0);
                a.part_lse[row] = -INFINITY;
                a.part_scale[row * 2] = 1.f;
                a.part_scale[row * 2 + 1] = 1.f;
            }
        }
    }

    bulk_wait_read();  // the epilogue's bulk stores have read their staging rows
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 5) tmem_dealloc(tmem, 512);

}

// Merge the splits of one (query, head), value columns [256 half, 256 half +
// 256), by one warp: out = sum_s w_s o_s / sum_s w_s with w_s = exp(lse_s -
// max lse); lse = max + ln sum_s w_s.  A split's stored half row is
// o_s * 2^-e_s (fp16), so it enters with the weight w_s * 2^e_s.  Lane s
// reads split s's log-sum-exp (splits <= 32) and the weights are shuffled
// from it; 8 columns per lane, 16-byte loads and stores, the partial loads
// of 8 splits issued before any is used.
__device__ void combine_half_head(const MlaParams &a, int wq, int hh, int half) {
    const int lane = threadIdx.x & 31;
    const int q = a.q0 + wq;
    const int64_t row0 = static_cast<int64_t>(wq) * a.splits * 128 + hh;  // split s: row0 + 128 s
    const int d = half * 256 + lane * 8;
    const float ls = lane < a.splits ? __ldcg(&a.part_lse[row0 + 128 * lane]) : -INFINITY;
    const float sc = lane < a.splits ? __ldcg(&a.part_scale[(row0 + 128 * lane) * 2 + half]) : 0.f;
    // the first kFirst splits' partial rows are loaded together with the
    // statistics (one L2 round trip for the usual split counts)
    constexpr int kFirst = 16;
    uint4 raw0[kFirst];
#pragma unroll
    for (int u = 0; u < kFirst; ++u)
        raw0[u] = u < a.splits ? __ldcg(reinterpret_cast<const uint4 *>(a.part_o + (row0 + 128 * u) * kDv + d))
                               : make_uint4(0, 0, 0, 0);
    float mx = ls;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    const float w = (mx == -INFINITY || ls == -INFINITY) ? 0.f : __expf(ls - mx);
    const float wsc = w > 0.f ? w * sc : 0.f;  // weight of the stored (scaled) values
    float tot = w;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) tot += __shfl_xor_sync(0xffffffffu, tot, o);
    uint16_t *o = a.out + (static_cast<int64_t>(q) * a.h + hh) * kDv + d;
    if (mx == -INFINITY) {
        *reinterpret_cast<uint4 *>(o) = make_uint4(0, 0, 0, 0);
        if (lane == 0 && half == 0) a.lse[static_cast<int64_t>(q) * a.h + hh] = -INFINITY;
        return;
    }
    float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int u = 0; u < kFirst; ++u) {
        const float wgt = __shfl_sync(0xffffffffu, wsc, u);
        const uint32_t r4[4] = {raw0[u].x, raw0[u].y, raw0[u].z, raw0[u].w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const float2 f = __half22float2(*reinterpret_cast<const __half2 *>(&r4[e]));
            acc[2 * e] = fmaf(wgt, f.x, acc[2 * e]);
            acc[2 * e + 1] = fmaf(wgt, f.y, acc[2 * e + 1]);
        }
    }
    for (int s0 = kFirst; s0 < a.splits; s0 += 8) {
        uint4 raw[8];
#pragma unroll
        for (int u = 0; u < 8; ++u)
            raw[u] = s0 + u < a.splits
                         ? __ldcg(reinterpret_cast<const uint4 *>(a.part_o + (row0 + 128 * (s0 + u)) * kDv + d))
                         : make_uint4(0, 0, 0, 0);
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            const float wgt = __shfl_sync(0xffffffffu, wsc, (s0 + u) & 31);
            const uint32_t r4[4] = {raw[u].x, raw[u].y, raw[u].z, raw[u].w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const float2 f = __half22float2(*reinterpret_cast<const __half2 *>(&r4[e]));
                acc[2 * e] = fmaf(wgt, f.x, acc[2 * e]);
                acc[2 * e + 1] = fmaf(wgt, f.y, acc[2 * e + 1]);
            }
        }
    }
    const float inv = 1.f / tot;
    uint4 res;
    res.x = pack_bf16x2(acc[0] * inv, acc[1] * inv);
    res.y = pack_bf16x2(acc[2] * inv, acc[3] * inv);
    res.z = pack_bf16x2(acc[4] * inv, acc[5] * inv);
    res.w = pack_bf16x2(acc[6] * inv, acc[7] * inv);
    *reinterpret_cast<uint4 *>(o) = res;
    if (lane == 0 && half == 0) a.lse[static_cast<int64_t>(q) * a.h + hh] = mx + logf(tot);
}

// The split combine as its own kernel: one warp per half head, two heads per
// 128-thread CTA, no shared memory, no CTA barrier.
__global__ void __launch_bounds__(128) k4_mla_combine(const MlaParams a, int n_slots) {
    grid_dependency_wait();  // the partials come from the preceding attention kernel
    const int warp = threadIdx.x >> 5;
    const int head_slot = blockIdx.x * 2 + (warp >> 1);  // (query in wave) * h + head
    if (head_slot >= n_slots) return;                     // whole warp: odd head count
    combine_half_head(a, head_slot / a.h, head_slot % a.h, warp & 1);
}

// Each head's log-sum-exp over the whole set from its splits' (one warp per
// (query, head); lane s reads split s, s + 32, ...).
__global__ void __launch_bounds__(128) k9_kl_lse(const MlaParams a) {
    grid_dependency_wait();  // the split statistics come from the preceding pass
    const int lane = threadIdx.x & 31;
    const int slot = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;  // query * h + head
    if (slot >= a.nq * a.h) return;
    const int q = slot / a.h, hh = slot % a.h;
    const float *pl = a.part_lse + static_cast<int64_t>(q) * a.splits * 128 + hh;
    float mx = -INFINITY;
    for (int s = lane; s < a.splits; s += 32) mx = fmaxf(mx, pl[static_cast<int64_t>(s) * 128]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    float sum = 0.f;
    if (mx > -INFINITY)
        for (int s = lane; s < a.splits; s += 32) sum += expf(pl[static_cast<int64_t>(s) * 128] - mx);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
    if (lane == 0) a.kl_lse[static_cast<int64_t>(q) * 128 + hh] = mx > -INFINITY ? mx + logf(sum) : -INFINITY;
}

constexpr int kKlThreads = 256;

// Block-wide sum and max of doubles (every thread gets the result).
__device__ double block_sum_d(double v, double *red) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    __syncthreads();
    if (lane == 0) red[warp] = v;
    __syncthreads();
    double t = 0.0;
    for (int w = 0; w < kKlThreads / 32; ++w) t += red[w];
    return t;
}

__device__ double block_max_d(double v, double *red) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmax(v, __shfl_xor_sync(0xffffffffu, v, o));
    __syncthreads();
    if (lane == 0) red[warp] = v;
    __syncthreads();
    double t = -INFINITY;
    for (int w = 0; w < kKlThreads / 32; ++w) t = fmax(t, red[w]);
    return t;
}

// The loss of one query (one CTA): p[e] = a[e] / sum a over the set's valid
// entries, r = softmax of the index scores over the same entries, and
// kl = sum_e p[e] (ln p[e] - ln r[e]) (0 ln 0 = 0), in double.  With p_out,
// the query's row of p_out is cleared and p added at each entry's position
// (a position listed twice gets both shares).
__global__ void __launch_bounds__(kKlThreads) k10_kl_reduce(const MlaParams a) {
    __shared__ double red[kKlThreads / 32];
    grid_dependency_wait();  // the head sums come from the preceding pass
    const int q = blockIdx.x, tid = threadIdx.x;
    const int n = a.q_n[q];
    const int cnt = a.dense ? min(n, a.topk) : a.topk;
    const float *I = a.iscores + static_cast<int64_t>(q) * a.ld;
    const float *A = a.kl_a + static_cast<int64_t>(q) * a.topk;
    const int32_t *ix = a.dense ? nullptr : a.idx + static_cast<int64_t>(q) * a.topk;
    float *po = a.p_out ? a.p_out + static_cast<int64_t>(q) * a.ld : nullptr;
    if (po)
        for (int64_t c = tid; c < a.ld; c += kKlThreads) po[c] = 0.f;
    auto pos_of = [&](int e) -> int {
        if (!ix) return e;
        const int s = ix[e];
        return (s >= 0 && s < n) ? s : -1;
    };
    double asum = 0.0, imax = -INFINITY;
    for (int e = tid; e < cnt; e += kKlThreads) {
        const int s = pos_of(e);
        if (s < 0) continue;
        asum += static_cast<double>(A[e]);
        imax = fmax(imax, static_cast<double>(I[s]));
    }
    asum = block_sum_d(asum, red);
    imax = block_max_d(imax, red);
    if (!(asum > 0.0) || imax == -INFINITY) {  // no valid entry
        if (tid == 0) a.kl[q] = 0.f;
        return;
    }
    double z = 0.0;
    for (int e = tid; e < cnt; e += kKlThreads) {
        const int s = pos_of(e);
        if (s >= 0) z += exp(static_cast<double>(I[s]) - imax);
    }
    const double lse_i = imax + log(block_sum_d(z, red));
    double acc = 0.0;
    for (int e = tid; e < cnt; e += kKlThreads) {
        const int s = pos_of(e);
        if (s < 0) continue;
        const double pe = static_cast<double>(A[e]) / asum;
        if (po) atomicAdd(po + s, static_cast<float>(pe));
        if (pe > 0.0) acc += pe * (log(pe) - (static_cast<double>(I[s]) - lse_i));
    }
    acc = block_sum_d(acc, red);
    if (tid == 0) a.kl[q] = static_cast<float>(acc);
}

// Launch with programmatic stream serialization: the kernel may begin while
// the previous kernel in the stream finishes; it calls grid_dependency_wait()
// before reading anything.
template <class... KArgs, class... Args>
static cudaError_t launch_pdl(void (*kern)(KArgs...), int grid, int block, size_t smem, cudaStream_t st,
                              const Args &...args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(block);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cudaError_t e = cudaLaunchKernelEx(&cfg, kern, args...);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

cudaError_t launch_sparse_mla(const CUtensorMap &qmap, const MlaParams &a, int nq_wave, cudaStream_t st,
                              bool kv8) {
    const MlaLayout L = mla_layout();
    const size_t smem = smem_for_tmem(L.total, 512);
    auto kern = kv8 ? k3_sparse_mla<kMlaAttn, true> : k3_sparse_mla<kMlaAttn, false>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    const int grid = nq_wave * a.splits;
    if (grid == 0) return cudaSuccess;
    return launch_pdl(kern, grid, kMlaThreads, smem, st, qmap, a);
}

cudaError_t launch_mla_combine(const MlaParams &a, int nq_wave, cudaStream_t st) {
    const int grid = (nq_wave * a.h + 1) / 2;  // two heads per CTA
    if (grid == 0 || a.splits <= 1) return cudaSuccess;
    return launch_pdl(k4_mla_combine, grid, 128, 0, st, a, nq_wave * a.h);
}

cudaError_t launch_kl_pass(int mode, const CUtensorMap &qmap, const MlaParams &a, cudaStream_t st) {
    const MlaLayout L = mla_layout();
    const size_t smem = smem_for_tmem(L.total, 512);
    auto kern = mode == kMlaKlStats ? k3_sparse_mla<kMlaKlStats, false> : k3_sparse_mla<kMlaKlSum, false>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    const int64_t grid = static_cast<int64_t>(a.nq) * a.splits;
    if (grid == 0) return cudaSuccess;
    return launch_pdl(kern, static_cast<int>(grid), kMlaThreads, smem, st, qmap, a);
}

cudaError_t launch_kl_lse(const MlaParams &a, cudaStream_t st) {
    const int64_t warps = static_cast<int64_t>(a.nq) * a.h;
    if (warps == 0) return cudaSuccess;
    return launch_pdl(k9_kl_lse, static_cast<int>((warps + 3) / 4), 128, 0, st, a);
}

cudaError_t launch_kl_reduce(const MlaParams &a, cudaStream_t st) {
    if (a.nq == 0) return cudaSuccess;
    return launch_pdl(k10_kl_reduce, a.nq, kKlThreads, 0, st, a);
}

}  // namespace dsa
