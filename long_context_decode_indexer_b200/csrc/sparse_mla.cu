// sparse_mla.cu -- sparse MQA-mode MLA attention on sm_100a.
//
// u_t = Attn(h_t, {c_s : s in I_t}) (DSA blog by marsggbo, section 3) in the
// MQA form of weight-absorbed MLA: every head attends to the same latent row,
// softmax(q . [c_kv; k_pe]^T) . c_kv ("DeepSeekV3.2之DSA" by yuyanqi,
// section 5.1).  Key = the whole 576-wide row, value = its first 512 columns.
//
// One CTA owns one query and a slice of at most 256 of its selected rows
// ("split"); all 128 heads form the MMA's M dimension.  Tensor memory (512
// columns) is planned so that no phase waits for space:
//   pass 1  S[128 x R] = Q . K^T.  Q's columns 0..511 sit in TMEM columns
//           256..511 (the A operand of tcgen05.mma read from tensor memory),
//           its 64 rope columns in shared memory; the selected rows stream
//           whole (1152 bytes each) in blocks of 32 through a ring, gathered
//           with 16-byte cp.async into the 128B-swizzled K-major layout, and
//           each block gives S columns [32b, 32b + 32) (N = 32): a block's
//           MMAs start as soon as its own rows land.
//   softmax two groups of four warps split S's columns; one thread per head
//           (TMEM lane); the exact max over the split, P = exp(S - max)
//           written back into TMEM columns 256..511 (Q is dead by then) as a
//           pair of bf16 tiles P_hi = bf16(P), P_lo = bf16(P - P_hi): a single
//           bf16 P would add ~1e-3 relative error on top of the ~1.7e-3 the
//           bf16 output itself carries; the pair makes P exact to ~2^-16.
//   pass 2  O = P_hi . V + P_lo . V in four quarters of 128 value columns,
//           ping-ponging between TMEM columns 0..127 and 128..255 (S is dead):
//           while the tensor cores accumulate quarter j + 1 from a fresh value
//           quarter (gathered, MN-major, by a third group of warps), the first
//           two groups drain quarter j.  A reads P from TMEM.
// A split writes O / l as fp16 values times a power-of-two scale per (split,
// head, 64 value columns), chosen from that block's largest magnitude: the
// values keep fp16's precision (2^-12 relative, far below the bf16 output's
// rounding) over the whole bf16 range of the latent cache, which plain fp16
// (max 65504, subnormal below 6e-5) would not.  Each split also writes its
// log-sum-exp; the combine kernel merges splits by their log-sum-exp.  With
// one split the CTA writes the final output.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

#include "kernels.h"
#include "ptx.cuh"

namespace dsa {

namespace {

constexpr int kRB = kMlaBlockRows;                 // rows per pass-1 block (MMA N)
constexpr int kNumKChunks = kDqk / 64;             // 9 chunks of 64 key columns
constexpr int kChunkBytes = kRB * 128;             // one chunk of a block: 4 KB
constexpr int kBlockBytes = kNumKChunks * kChunkBytes;
constexpr int kVColBlockBytes = kMlaMaxRows * 128; // 64 value columns of 256 rows: 32 KB
constexpr int kVQuarterBytes = 2 * kVColBlockBytes;
constexpr uint32_t kColS = 0;                      // S: columns 0..R-1
constexpr uint32_t kColQ = 256;                    // Q (dims 0..511): columns 256..511
constexpr uint32_t kColPhi = 256, kColPlo = 384;   // P_hi / P_lo after pass 1
constexpr int kGroupThreads = 128;
constexpr int kGatherThreads = 256;                // groups B and C stream pass 1
constexpr int kPiecesPerRow = kDqk * 2 / 16;       // 72 pieces of 16 bytes
constexpr int kPass1Pieces = kRB * kPiecesPerRow / kGatherThreads;  // 9 per thread per block
constexpr int kGatherLag = 2;                      // blocks a gather thread publishes behind its newest
constexpr int kWarpMma = 12, kWarpRope = 13;
constexpr int kBarAB = 1;                          // named barrier: groups A + B (256 threads)

struct MlaSmem {
    uint64_t full[kMlaRing];
    uint64_t empty[kMlaRing];
    uint64_t q_ready;      // group A stored Q into TMEM
    uint64_t rope_full;    // rope columns of Q landed (TMA)
    uint64_t s_full;       // every pass-1 MMA completed
    uint64_t p_full;       // P_hi / P_lo in TMEM (groups A + B)
    uint64_t vq_full[2];   // value quarter gathered (group C)
    uint64_t vq_empty[2];  // value quarter consumed (MMA)
    uint64_t o_full[2];    // O quarter accumulated (MMA)
    uint64_t o_empty[2];   // O quarter drained (groups A + B)
    uint64_t mma_done;     // every MMA issued has completed
    uint32_t tmem_base;
    volatile int32_t abort;
    int32_t rows[kMlaMaxRows];
    uint32_t vmask[kMlaMaxRows / 32];  // bit j of word w: entry 32w + j is valid
    float pmax[2][128];                // softmax: each group's partial max per head
    float psum[2][128];                // and partial sum
};

static_assert(sizeof(MlaSmem) <= 4096, "MlaSmem must fit the reserve in mla_layout()");
static_assert(kMlaRing * kBlockBytes >= 2 * kVQuarterBytes, "the value quarters reuse the pass-1 ring");
static_assert(kRB * kPiecesPerRow % kGatherThreads == 0, "pass-1 pieces split evenly");

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

// The 64 value columns [c0, c0 + 64) of this thread's head row of O (TMEM
// address `taddr`: its lane, the block's first column) -> the output row.
// Final output: bf16 of O / l.  Split partial: fp16 of O / l * 2^-e with e
// from the block's largest magnitude m (m * 2^-e in [2^14, 2^15), below
// fp16's 65504); 2^e goes to part_scale.  The TMEM loads are
// warp-collective: every lane runs them; only the stores are skipped for
// padding heads (hrow >= h).
__device__ void store_block(const MlaParams &a, uint32_t taddr, int hrow, int q, int wq, int sp,
                            float inv_l, int c0) {
    uint32_t v[2][32];
    tmem_ld32(taddr, v[0]);
    tmem_ld32(taddr + 32, v[1]);
    tmem_wait_ld();
    const bool partial = a.splits > 1;
    float mul = inv_l;
    if (partial) {
        float mx = 0.f;
#pragma unroll
        for (int j = 0; j < 32; ++j)
            mx = fmaxf(mx, fmaxf(fabsf(__uint_as_float(v[0][j])), fabsf(__uint_as_float(v[1][j]))));
        mx *= inv_l;
        // exponent of mx minus 14 (0 for an all-zero block); a subnormal or
        // tiny mx is clamped (its values then stay below 2^14, still exact
        // enough), so that both 2^-e and 2^e are normal floats
        int e = mx > 0.f ? static_cast<int>((__float_as_uint(mx) >> 23) & 0xFFu) - 127 - 14 : 0;
        e = min(max(e, -100), 113);
        mul = inv_l * __int_as_float((127 - e) << 23);
        if (hrow < a.h)
            a.part_scale[((static_cast<int64_t>(wq) * a.splits + sp) * 128 + hrow) * kMlaScaleBlocks + (c0 >> 6)] =
                __int_as_float((127 + e) << 23);
    }
    if (hrow >= a.h) return;
    uint16_t *dst = !partial ? a.out + (static_cast<int64_t>(q) * a.h + hrow) * kDv + c0
                             : a.part_o + ((static_cast<int64_t>(wq) * a.splits + sp) * 128 + hrow) * kDv + c0;
#pragma unroll
    for (int g = 0; g < 8; ++g) {
        const uint32_t *u = &v[g >> 2][(g & 3) * 8];
        uint32_t w[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const float x0 = __uint_as_float(u[2 * e]) * mul, x1 = __uint_as_float(u[2 * e + 1]) * mul;
            w[e] = partial ? pack_half2(x0, x1) : pack_bf16x2(x0, x1);
        }
        *reinterpret_cast<uint4 *>(dst + g * 8) = make_uint4(w[0], w[1], w[2], w[3]);
    }
}

}  // namespace

__global__ void __launch_bounds__(kMlaThreads, 1)
    k3_sparse_mla(const __grid_constant__ CUtensorMap qmap, const MlaParams a) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *base = align1024(smem_raw);
    const MlaLayout L = mla_layout();
    MlaSmem &sm = *reinterpret_cast<MlaSmem *>(base + L.misc);
    uint8_t *ring = base + L.ring;
    uint8_t *vq = base + L.vq;
    uint8_t *rope = base + L.rope;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int wq = blockIdx.x / a.splits;  // query within this wave
    const int sp = blockIdx.x % a.splits;
    const int q = a.q0 + wq;
    const int e0 = sp * a.rows_per_split;
    const int R = max(min(a.rows_per_split, a.topk - e0), 0);
    const int nb = (R + kRB - 1) / kRB;       // pass-1 blocks
    const int Rp = (R + 15) & ~15;            // pass-2 rows (16-row k-steps)
    const int hbox = a.h < 128 ? a.h : 128;

    if (tid == 0) {
        sm.abort = 0;
        for (int s = 0; s < kMlaRing; ++s) {
            mbar_init(&sm.full[s], kGatherThreads / 32);  // the eight gather warps
            mbar_init(&sm.empty[s], 1);
        }
        mbar_init(&sm.q_ready, 4);
        mbar_init(&sm.rope_full, 1);
        mbar_init(&sm.s_full, 1);
        mbar_init(&sm.p_full, 8);
        for (int v = 0; v < 2; ++v) {
            mbar_init(&sm.vq_full[v], 4);
            mbar_init(&sm.vq_empty[v], 1);
            mbar_init(&sm.o_full[v], 1);
            mbar_init(&sm.o_empty[v], 8);
        }
        mbar_init(&sm.mma_done, 1);
        fence_mbar_init();
    }
    // rope rows h..127 are never written by TMA: zero them once
    if (hbox < 128)
        for (int i = tid; i < (128 - hbox) * 8; i += blockDim.x)
            *reinterpret_cast<uint4 *>(rope + hbox * 128 + i * 16) = make_uint4(0, 0, 0, 0);
    if (warp == kWarpMma) {
        tmem_alloc(&sm.tmem_base, 512);
        tmem_relinquish();
    }
    // everything above touches no input: with programmatic dependent launch
    // it overlaps the end of the kernel that produced the indices
    grid_dependency_wait();
    const int n = a.q_n[q];
    const int seq = a.q_seq[q];
    __syncthreads();
    // cache rows of this split's entries (invalid entries, and rows past R,
    // read row 0 and are masked: P = 0 there)
    for (int i = tid; i < kMlaMaxRows; i += blockDim.x) {
        int32_t row = 0;
        bool ok = false;
        if (i < R) {
            const int s = a.idx[static_cast<int64_t>(q) * a.topk + e0 + i];
            if (s >= n) record_status(a.status, DSA_ERR_DEVICE_CHECK);
            if (s >= 0 && s < n) {
                int64_t r;
                if (a.page_table)
                    r = static_cast<int64_t>(a.page_table[static_cast<int64_t>(seq) * a.max_pages + s / a.page_size]) * a.page_size + s % a.page_size;
                else
                    r = a.seq_row0[seq] + s;
                if (r >= 0 && r < a.cache_rows) {
                    row = static_cast<int32_t>(r);
                    ok = true;
                } else {
                    record_status(a.status, DSA_ERR_DEVICE_CHECK);
                }
            }
        }
        sm.rows[i] = row;
        const unsigned bits = __ballot_sync(0xffffffffu, ok);
        if ((i & 31) == 0) sm.vmask[i >> 5] = bits;
    }
    fence_proxy_async_smem();  // zeroed rope rows, read by the tensor cores
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = sm.tmem_base;

    if (R > 0) {
        if (warp < 4) {
            // ---- group A: Q columns 0..511 of this head -> TMEM columns 256..511
            const int hrow = warp * 32 + lane;  // head = TMEM lane
            const uint32_t lane_base = tmem + (static_cast<uint32_t>(warp * 32) << 16);
            const uint16_t *qrow = a.q + (static_cast<int64_t>(q) * a.h + (hrow < a.h ? hrow : 0)) * kDqk;
            for (int c0 = 0; c0 < 512; c0 += 64) {  // 64 dims = 32 columns per store
                uint32_t r[32];
#pragma unroll
                for (int g = 0; g < 8; ++g) {
                    const uint4 v = hrow < a.h ? __ldg(reinterpret_cast<const uint4 *>(qrow + c0 + g * 8))
                                               : make_uint4(0, 0, 0, 0);
                    r[4 * g] = v.x;
                    r[4 * g + 1] = v.y;
                    r[4 * g + 2] = v.z;
                    r[4 * g + 3] = v.w;
                }
                tmem_st32(lane_base + kColQ + c0 / 2, r);
            }
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&sm.q_ready);
        } else if (warp < 12) {
            // ---- groups B and C: pass-1 row blocks (whole rows, 128B-swizzled
            // K-major: chunk c of the block holds key columns 64c..64c+63)
            const int gt = tid - kGroupThreads;  // 0..255
            const int r = gt >> 3;               // row within the block
            const int pbase = (gt & 7) * kPass1Pieces;
            bool ok = true;
            for (int b = 0; b < nb + kGatherLag; ++b) {
                if (b < nb) {
                    const int s = b % kMlaRing;
                    const uint32_t ph = (b / kMlaRing) & 1;
                    ok = ok && __all_sync(0xffffffffu, mbar_wait(&sm.empty[s], ph ^ 1, a.wait_budget) && !sm.abort);
                    if (ok) {
                        uint8_t *blk = ring + s * kBlockBytes;
                        const uint16_t *src = a.kv + static_cast<int64_t>(sm.rows[b * kRB + r]) * a.kv_row_stride;
#pragma unroll
                        for (int k = 0; k < kPass1Pieces; ++k) {
                            const int p = pbase + k, c = p >> 3, j = p & 7;
                            cp_async16(blk + c * kChunkBytes + r * 128 + ((j ^ (r & 7)) << 4), src + p * 8);
                        }
                    }
                    cp_async_commit();
                }
                if (b >= kGatherLag) {
                    // block b - lag is complete for this thread: publish it
                    if (b < nb) cp_async_wait<kGatherLag>();
                    else cp_async_wait<0>();
                    fence_proxy_async_smem();
                    __syncwarp();
                    // tests only: the first CTA never publishes block 0
                    const bool skip = a.inject != 0 && blockIdx.x == 0 && b == kGatherLag;
                    if (lane == 0 && !skip) mbar_arrive(&sm.full[(b - kGatherLag) % kMlaRing]);
                }
            }
            if (!ok && lane == 0) {
                record_status(a.status, DSA_ERR_TIMEOUT);
                sm.abort = 1;
            }
        } else if (warp == kWarpRope) {
            if (lane == 0) {
                mbar_arrive_expect_tx(&sm.rope_full, static_cast<uint32_t>(hbox) * 128u);
                tma_load_2d(rope, &qmap, &sm.rope_full, 512, q * a.h);
                // the load lands before the CTA may exit
                if (!mbar_wait(&sm.rope_full, 0, a.wait_budget)) record_status(a.status, DSA_ERR_TIMEOUT);
            }
        } else {
            // ---- MMA issuer (warp 12, one lane)
            if (lane == 0) {
                bool ok = mbar_wait(&sm.q_ready, 0, a.wait_budget) && mbar_wait(&sm.rope_full, 0, a.wait_budget);
                const uint32_t idesc1 = make_idesc(1, 1, 0, 0, 128, kRB);
                const uint32_t rope_a = smem_u32(rope);
                for (int b = 0; b < nb && ok; ++b) {
                    const int s = b % kMlaRing;
                    const uint32_t ph = (b / kMlaRing) & 1;
                    if (sm.abort || !mbar_wait(&sm.full[s], ph, a.wait_budget)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t blk = smem_u32(ring + s * kBlockBytes);
                    const uint32_t d = tmem + kColS + static_cast<uint32_t>(b * kRB);
#pragma unroll
                    for (int c = 0; c < kNumKChunks; ++c) {
#pragma unroll
                        for (int kk = 0; kk < 4; ++kk) {
                            const uint64_t bd = make_sdesc(blk + c * kChunkBytes + kk * 32, 16, 1024, kSwizzle128B);
                            if (c < kNumKChunks - 1)
                                mma_bf16_ts(d, tmem + kColQ + static_cast<uint32_t>(c * 32 + kk * 8), bd, idesc1,
                                            (c > 0 || kk > 0) ? 1u : 0u);
                            else
                                mma_bf16_ss(d, make_sdesc(rope_a + kk * 32, 16, 1024, kSwizzle128B), bd, idesc1, 1u);
                        }
                    }
                    tc_commit(&sm.empty[s]);
                }
                tc_commit(&sm.s_full);
                // pass 2: four value quarters, O ping-ponging in TMEM columns
                // 0..127 / 128..255; A = P_hi, P_lo from TMEM, B = the quarter's
                // rows, MN-major (LBO = distance between its two 64-column
                // blocks, SBO = 1 KB between 8-row groups along K)
                ok = ok && mbar_wait(&sm.p_full, 0, a.wait_budget) && !sm.abort;
                const uint32_t idesc2 = make_idesc(1, 1, 0, 1, 128, 128);
                for (int qq = 0; qq < 4 && ok; ++qq) {
                    const int buf = qq & 1;
                    const uint32_t ph = (qq >> 1) & 1;
                    if (sm.abort || !mbar_wait(&sm.vq_full[buf], ph, a.wait_budget) ||
                        !mbar_wait(&sm.o_empty[buf], ph ^ 1, a.wait_budget)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t va = smem_u32(vq + buf * kVQuarterBytes);
                    const uint32_t d = tmem + static_cast<uint32_t>(buf * 128);
                    for (int kk = 0; kk < Rp / 16; ++kk) {
                        const uint64_t bd = make_sdesc(va + kk * 2048, kVColBlockBytes, 1024, kSwizzle128B);
                        mma_bf16_ts(d, tmem + kColPhi + static_cast<uint32_t>(kk * 8), bd, idesc2, kk > 0 ? 1u : 0u);
                        mma_bf16_ts(d, tmem + kColPlo + static_cast<uint32_t>(kk * 8), bd, idesc2, 1u);
                    }
                    tc_commit(&sm.vq_empty[buf]);
                    tc_commit(&sm.o_full[buf]);
                }
                if (!ok) {
                    record_status(a.status, DSA_ERR_TIMEOUT);
                    sm.abort = 1;
                }
                // every MMA issued completes before the CTA may free TMEM
                tc_commit(&sm.mma_done);
                if (!mbar_wait(&sm.mma_done, 0, a.wait_budget)) record_status(a.status, DSA_ERR_TIMEOUT);
            }
        }

        if (warp < 8) {
            // ---- softmax (groups A + B split S's blocks), then the epilogue
            const int grp = warp >> 2;  // 0: A, 1: B
            const int quarter = warp & 3;
            const int hrow = quarter * 32 + lane;
            const uint32_t lane_base = tmem + (static_cast<uint32_t>(quarter * 32) << 16);
            bool ok = __all_sync(0xffffffffu, mbar_wait(&sm.s_full, 0, a.wait_budget) && !sm.abort);
            const int nbh = (nb + 1) / 2;  // blocks of S per group
            const int b_lo = grp * nbh, b_hi = min(nb, b_lo + nbh);
            float mpart = -INFINITY;
            if (ok) {
                tc_fence_after();
                for (int b = b_lo; b < b_hi; ++b) {
                    uint32_t v[32];
                    tmem_ld32(lane_base + kColS + b * 32, v);
                    const uint32_t vm = sm.vmask[b];
                    tmem_wait_ld();
#pragma unroll
                    for (int j = 0; j < 32; ++j)
                        mpart = fmaxf(mpart, ((vm >> j) & 1u) ? __uint_as_float(v[j]) : -INFINITY);
                }
            }
            sm.pmax[grp][hrow] = mpart;
            ok = bar_and(kBarAB, 2 * kGroupThreads, ok);
            const float m = fmaxf(sm.pmax[0][hrow], sm.pmax[1][hrow]);
            const float mlog = (m == -INFINITY) ? 0.f : m * a.scale_log2;
            float lpart = 0.f;
            if (ok) {
                for (int b = b_lo; b < b_hi; ++b) {
                    uint32_t v[32];
                    tmem_ld32(lane_base + kColS + b * 32, v);
                    const uint32_t vm = sm.vmask[b];
                    tmem_wait_ld();
                    uint32_t hi[16], lo[16];
#pragma unroll
                    for (int e = 0; e < 16; ++e) {
                        const float p0 = ((vm >> (2 * e)) & 1u) ? fast_exp2(fmaf(__uint_as_float(v[2 * e]), a.scale_log2, -mlog)) : 0.f;
                        const float p1 = ((vm >> (2 * e + 1)) & 1u) ? fast_exp2(fmaf(__uint_as_float(v[2 * e + 1]), a.scale_log2, -mlog)) : 0.f;
                        lpart += p0 + p1;
                        // one paired conversion each for P_hi and P_lo
                        const __nv_bfloat162 h2 = __floats2bfloat162_rn(p0, p1);
                        const float2 hf = __bfloat1622float2(h2);
                        const __nv_bfloat162 l2 = __floats2bfloat162_rn(p0 - hf.x, p1 - hf.y);
                        hi[e] = *reinterpret_cast<const uint32_t *>(&h2);
                        lo[e] = *reinterpret_cast<const uint32_t *>(&l2);
                    }
                    tmem_st16(lane_base + kColPhi + b * 16, hi);
                    tmem_st16(lane_base + kColPlo + b * 16, lo);
                }
                tmem_wait_st();
            }
            sm.psum[grp][hrow] = lpart;
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&sm.p_full);
            ok = bar_and(kBarAB, 2 * kGroupThreads, ok);
            const float l = sm.psum[0][hrow] + sm.psum[1][hrow];
            const bool has = l > 0.f;
            const float inv_l = has ? 1.f / l : 0.f;
            if (grp == 0 && ok && hrow < a.h) {
                const float lse_v = has ? (m * a.scale + logf(l)) : -INFINITY;
                if (a.splits == 1) a.lse[static_cast<int64_t>(q) * a.h + hrow] = lse_v;
                else a.part_lse[(static_cast<int64_t>(wq) * a.splits + sp) * 128 + hrow] = lse_v;
            }
            // drain the four O quarters, 64 columns per group
            for (int qq = 0; qq < 4; ++qq) {
                const int buf = qq & 1;
                const uint32_t ph = (qq >> 1) & 1;
                ok = ok && __all_sync(0xffffffffu, mbar_wait(&sm.o_full[buf], ph, a.wait_budget) && !sm.abort);
                if (ok) {
                    tc_fence_after();
                    store_block(a, lane_base + static_cast<uint32_t>(buf * 128 + grp * 64), hrow, q, wq, sp, inv_l,
                                qq * 128 + grp * 64);
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&sm.o_empty[buf]);
            }
            if (!ok && lane == 0) record_status(a.status, DSA_ERR_TIMEOUT);
        } else if (warp < 12) {
            // ---- group C: the four value quarters (rows x 128 columns),
            // MN-major 128B-swizzled: two 64-column blocks of 256-row stride
            const int gt = tid - 2 * kGroupThreads;  // 0..127
            const int j16 = gt & 15;                 // 16-byte piece of the quarter's 256 bytes of a row
            const int vblk = j16 >> 3, j = j16 & 7;
            bool ok = __all_sync(0xffffffffu, mbar_wait(&sm.s_full, 0, a.wait_budget) && !sm.abort);
            for (int qq = 0; qq < 4; ++qq) {
                const int buf = qq & 1;
                const uint32_t ph = (qq >> 1) & 1;
                ok = ok && __all_sync(0xffffffffu, mbar_wait(&sm.vq_empty[buf], ph ^ 1, a.wait_budget) && !sm.abort);
                if (ok) {
                    uint8_t *dstq = vq + buf * kVQuarterBytes + vblk * kVColBlockBytes;
                    for (int i = gt >> 4; i < Rp; i += kGroupThreads / 16) {
                        const uint16_t *src = a.kv + static_cast<int64_t>(sm.rows[i]) * a.kv_row_stride + qq * 128 + j16 * 8;
                        cp_async16(dstq + i * 128 + ((j ^ (i & 7)) << 4), src);
                    }
                }
                cp_async_commit();
                cp_async_wait<0>();
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) mbar_arrive(&sm.vq_full[buf]);
            }
            if (!ok && lane == 0) {
                record_status(a.status, DSA_ERR_TIMEOUT);
                sm.abort = 1;
            }
        }
    } else if (warp < 4) {
        // empty split: no rows at all
        const int hrow = warp * 32 + lane;
        if (hrow < a.h) {
            if (a.splits == 1) {
                uint16_t *o = a.out + (static_cast<int64_t>(q) * a.h + hrow) * kDv;
                for (int c0 = 0; c0 < kDv; c0 += 8) *reinterpret_cast<uint4 *>(o + c0) = make_uint4(0, 0, 0, 0);
                a.lse[static_cast<int64_t>(q) * a.h + hrow] = -INFINITY;
            } else {
                const int64_t row = (static_cast<int64_t>(wq) * a.splits + sp) * 128 + hrow;
                uint16_t *o = a.part_o + row * kDv;
                for (int c0 = 0; c0 < kDv; c0 += 8) *reinterpret_cast<uint4 *>(o + c0) = make_uint4(0, 0, 0, 0);
                a.part_lse[row] = -INFINITY;
                for (int k = 0; k < kMlaScaleBlocks; ++k) a.part_scale[row * kMlaScaleBlocks + k] = 1.f;
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == kWarpMma) tmem_dealloc(tmem, 512);
}

// Merge the splits of one (query, head): out = sum_s w_s o_s / sum_s w_s with
// w_s = exp(lse_s - max lse); lse = max + ln sum_s w_s.  A split's stored
// 64-column block is o_s * 2^-e (fp16), so it enters with the weight
// w_s * 2^e.  One warp covers 256 value columns of one head (8 per lane,
// 16-byte loads and stores), so a head takes two warps and a 128-thread CTA
// two heads.  Every warp reads the head's split log-sum-exps itself (lane s
// holds split s; splits <= 32) and gets the weights by shuffles: no shared
// memory, no CTA barrier.  The partial loads of all splits are issued before
// any is used.
__global__ void __launch_bounds__(128) k4_mla_combine(const MlaParams a, int n_slots) {
    grid_dependency_wait();  // the partials come from the preceding attention kernel
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int head_slot = blockIdx.x * 2 + (warp >> 1);  // (query in wave) * h + head
    if (head_slot >= n_slots) return;                     // whole warp: odd head count
    const int wq = head_slot / a.h, hh = head_slot % a.h;
    const int q = a.q0 + wq;
    const int64_t row0 = static_cast<int64_t>(wq) * a.splits * 128 + hh;  // split s: row0 + 128 s
    const int d = (warp & 1) * 256 + lane * 8;
    const int sblk = d >> 6;  // this lane's 64-column scale block
    const float ls = lane < a.splits ? a.part_lse[row0 + 128 * lane] : -INFINITY;
    float mx = ls;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    const float w = (mx == -INFINITY || ls == -INFINITY) ? 0.f : __expf(ls - mx);
    float tot = w;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) tot += __shfl_xor_sync(0xffffffffu, tot, o);
    uint16_t *o = a.out + (static_cast<int64_t>(q) * a.h + hh) * kDv + d;
    if (mx == -INFINITY) {
        *reinterpret_cast<uint4 *>(o) = make_uint4(0, 0, 0, 0);
        if (lane == 0 && (warp & 1) == 0) a.lse[static_cast<int64_t>(q) * a.h + hh] = -INFINITY;
        return;
    }
    float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    for (int s0 = 0; s0 < a.splits; s0 += 8) {
        uint4 raw[8];
        float sc[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            const bool in = s0 + u < a.splits;
            raw[u] = in ? *reinterpret_cast<const uint4 *>(a.part_o + (row0 + 128 * (s0 + u)) * kDv + d)
                        : make_uint4(0, 0, 0, 0);
            sc[u] = in ? a.part_scale[(row0 + 128 * (s0 + u)) * kMlaScaleBlocks + sblk] : 0.f;
        }
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            const float wu = __shfl_sync(0xffffffffu, w, (s0 + u) & 31);
            const float wgt = wu > 0.f ? wu * sc[u] : 0.f;  // weight of the stored (scaled) values
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
    if (lane == 0 && (warp & 1) == 0) a.lse[static_cast<int64_t>(q) * a.h + hh] = mx + logf(tot);
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

cudaError_t launch_sparse_mla(const CUtensorMap &qmap, const MlaParams &a, int nq_wave, cudaStream_t st) {
    const MlaLayout L = mla_layout();
    const size_t smem = smem_for_tmem(L.total, 512);
    cudaError_t e = cudaFuncSetAttribute(k3_sparse_mla, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    const int grid = nq_wave * a.splits;
    if (grid == 0) return cudaSuccess;
    return launch_pdl(k3_sparse_mla, grid, kMlaThreads, smem, st, qmap, a);
}

cudaError_t launch_mla_combine(const MlaParams &a, int nq_wave, cudaStream_t st) {
    const int grid = (nq_wave * a.h + 1) / 2;  // two heads per CTA
    if (grid == 0 || a.splits <= 1) return cudaSuccess;
    return launch_pdl(k4_mla_combine, grid, 128, 0, st, a, nq_wave * a.h);
}

}  // namespace dsa
