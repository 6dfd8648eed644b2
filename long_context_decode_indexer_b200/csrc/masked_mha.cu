// masked_mha.cu -- the short-prefill path: dense multi-head attention under
// the index set's mask, on sm_100a.
//
// For short prompts DSA's prefill runs as MHA (each head with its own key and
// value, the MHA form of MLA used for prefill; DSA blog by marsggbo, section
// 4) over every visible position, and the indexer's selection enters as a
// mask (the same blog, section 6: masked MHA emulates DSA where dense matrix
// work suits the GPU better than gathers; the aicoding.csdn.net DSA article,
// section 4.3: masked MHA below 8K tokens).  Query t, head h:
//   keep[s] = s < q_n[t] and s in the index set of t
//   out     = softmax over kept s of scale * q[t,h] . k[s,h], applied to v[s,h]
//
// One CTA per (128-query tile, head), the tiles of a head consecutive so
// that the CTAs running together share their K / V in L2.  Warp 0 streams Q
// once and K / V tiles of 128 positions through a TMA ring (3-D tensor maps
// over [row, head, dim], 128B swizzle); warp 1 issues the tcgen05 MMAs;
// warps 2-9 run the softmax, two warps per query row (= TMEM lane), each on
// half of a tile's keys.
//   S(j) = Q . K(j)^T      M = 128 queries, N = 128 keys, K = d_qk; one TMEM
//                           buffer, which the softmax reads first thing, so
//                           S(j+1) is computed during softmax(j)
//   P(j) = 2^(S' - m)      S' = S * scale * log2(e), masked keys -inf; P goes
//                           to TMEM (two buffers) as a pair of bf16 tiles
//                           P_hi + P_lo (together exact to ~2^-16, as in the
//                           decode attention) and is the A operand of
//   O   += P(j) . V(j)      V(j) MN-major from shared memory, O in TMEM; with
//                           two P buffers P(j+1) is written while P(j) . V(j)
//                           runs.
// The running max m is raised only when a tile's max exceeds it by more than
// 2^8 (then O and the row sum are rescaled once); otherwise P <= 2^8 and
// nothing is rescaled.  O / l and the log-sum-exp are exact either way.
// The membership mask is a bitmap [query, position] built from the index
// list by k12_mha_mask (a list entry counts once: a mask holds membership).
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

#include "kernels.h"
#include "ptx.cuh"

namespace dsa {

namespace {

constexpr uint32_t kChunkBytes = kMhaTile * 128u;  // 128 rows x 64 bf16 columns
constexpr uint32_t kColS = 0;                       // S: 128 columns
constexpr uint32_t kColO = 128;                     // O: d_v <= 128 columns
constexpr uint32_t kColP = 256;                     // two P buffers of 128 columns: P_hi (128 keys as 64
                                                    // columns of bf16 pairs), then P_lo
constexpr float kRaiseLog2 = 8.f;                   // raise the running max only past 2^8

struct MhaSmem {
    uint64_t q_full;
    uint64_t k_full[kMhaMaxStages];
    uint64_t k_empty[kMhaMaxStages];
    uint64_t v_full[kMhaVStages];
    uint64_t v_empty[kMhaVStages];
    uint64_t s_full;
    uint64_t s_free;
    uint64_t p_full[2];
    uint64_t pv_done[2];
    uint64_t mma_done;
    uint32_t tmem_base;
    volatile int32_t abort;
    int32_t n_max;
    float half_max[2][2][kMhaTile];  // [tile parity][column half][row]
    float half_sum[2][kMhaTile];     // [column half][row]
};
static_assert(sizeof(MhaSmem) <= 4096, "MhaSmem must fit the reserve in mha_layout()");

__device__ __forceinline__ uint8_t *align1024(uint8_t *p) {
    return reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}

__device__ __forceinline__ uint32_t bf16x2_bits(__nv_bfloat162 v) { return *reinterpret_cast<uint32_t *>(&v); }

// Named barrier `id` over `count` threads.
__device__ __forceinline__ void bar_sync(int id, int count) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(count) : "memory");
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

}  // namespace

__global__ void __launch_bounds__(kMhaThreads, 1)
    k11_masked_mha(const __grid_constant__ CUtensorMap qmap, const __grid_constant__ CUtensorMap kmap,
                   const __grid_constant__ CUtensorMap vmap, const MhaParams a) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *base = align1024(smem_raw);
    const MhaLayout L = mha_layout(a.d_qk, a.d_v, a.stages);
    MhaSmem &sm = *reinterpret_cast<MhaSmem *>(base + L.misc);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    // consecutive CTAs take the query tiles of one head (they read the same
    // K / V, which then stays in L2), the latest (longest) tiles first
    const int tile = a.tiles_per_block - 1 - static_cast<int>(blockIdx.x % a.tiles_per_block);
    const int rest = static_cast<int>(blockIdx.x / a.tiles_per_block);
    const int head = rest % a.h;
    const int blk = rest / a.h;
    const int t0 = blk * a.q_per_seq + tile * kMhaTile;
    const int t_end = min(blk * a.q_per_seq + a.q_per_seq, a.nq);
    const int nrows = max(min(kMhaTile, t_end - t0), 0);
    const int QC = a.d_qk / 64, VC = a.d_v / 64;

    if (tid == 0) {
        sm.abort = 0;
        sm.n_max = 0;
        mbar_init(&sm.q_full, 1);
        for (int s = 0; s < a.stages; ++s) {
            mbar_init(&sm.k_full[s], 1);
            mbar_init(&sm.k_empty[s], 1);
        }
        for (int s = 0; s < kMhaVStages; ++s) {
            mbar_init(&sm.v_full[s], 1);
            mbar_init(&sm.v_empty[s], 1);
        }
        mbar_init(&sm.s_full, 1);
        mbar_init(&sm.s_free, 8);  // the eight softmax warps
        for (int b = 0; b < 2; ++b) {
            mbar_init(&sm.p_full[b], 8);
            mbar_init(&sm.pv_done[b], 1);
        }
        mbar_init(&sm.mma_done, 1);
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc(&sm.tmem_base, 512);
        tmem_relinquish();
    }
    // nothing above reads an input: with programmatic dependent launch it
    // overlaps the end of the kernel that built the mask
    grid_dependency_wait();
    __syncthreads();
    // the positions this tile needs: the longest history among its queries
    if (warp >= 2) {
        const int r = (warp & 3) * 32 + lane;
        int n = r < nrows ? a.q_n[t0 + r] : 0;
        if (n > a.max_n) {
            record_status(a.status, DSA_ERR_DEVICE_CHECK);
            n = a.max_n;
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) n = max(n, __shfl_xor_sync(0xffffffffu, n, o));
        if (lane == 0 && n > 0) atomicMax(&sm.n_max, n);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = sm.tmem_base;
    const int nkt = (sm.n_max + kMhaTile - 1) / kMhaTile;  // key tiles
    const int64_t row0 = nrows > 0 ? a.seq_row0[a.q_seq[t0]] : 0;

    if (warp == 0) {
        // ------------------------------------------------ TMA producer
        if (lane == 0 && nkt > 0) {
            mbar_arrive_expect_tx(&sm.q_full, static_cast<uint32_t>(QC) * kChunkBytes);
            for (int c = 0; c < QC; ++c)
                tma_load_3d(base + L.q + c * kChunkBytes, &qmap, &sm.q_full, c * 64, head, t0);
            // K(j) and V(j) in order; a K slot frees once S(j) is computed,
            // a V slot once P(j) . V(j) is, so K runs ahead of V
            int k_end = 0, v_end = 0;  // tiles whose K / V loads were issued
            for (int j = 0; j < nkt; ++j) {
                const int ks = j % a.stages, vs = j % kMhaVStages;
                const int r = static_cast<int>(row0) + j * kMhaTile;
                if (sm.abort ||
                    !mbar_wait(&sm.k_empty[ks], static_cast<uint32_t>(j / a.stages) & 1u ^ 1u, a.wait_budget)) {
                    record_status(a.status, DSA_ERR_TIMEOUT);
                    sm.abort = 1;
                    break;
                }
                mbar_arrive_expect_tx(&sm.k_full[ks], L.k_stage);
                for (int c = 0; c < QC; ++c)
                    tma_load_3d(base + L.k_ring + ks * L.k_stage + c * kChunkBytes, &kmap, &sm.k_full[ks], c * 64,
                                head, r);
                k_end = j + 1;
                if (sm.abort ||
                    !mbar_wait(&sm.v_empty[vs], static_cast<uint32_t>(j / kMhaVStages) & 1u ^ 1u, a.wait_budget)) {
                    record_status(a.status, DSA_ERR_TIMEOUT);
                    sm.abort = 1;
                    break;
                }
                mbar_arrive_expect_tx(&sm.v_full[vs], L.v_stage);
                for (int c = 0; c < VC; ++c)
                    tma_load_3d(base + L.v_ring + vs * L.v_stage + c * kChunkBytes, &vmap, &sm.v_full[vs], c * 64,
                                head, r);
                v_end = j + 1;
            }
            // every load issued lands before the CTA may exit (a no-op when
            // the MMAs consumed them all)
            mbar_wait(&sm.q_full, 0, a.wait_budget);
            for (int j = max(k_end - a.stages, 0); j < k_end; ++j)
                mbar_wait(&sm.k_full[j % a.stages], static_cast<uint32_t>(j / a.stages) & 1u, a.wait_budget);
            for (int j = max(v_end - kMhaVStages, 0); j < v_end; ++j)
                mbar_wait(&sm.v_full[j % kMhaVStages], static_cast<uint32_t>(j / kMhaVStages) & 1u, a.wait_budget);
        }
    } else if (warp == 1) {
        // ------------------------------------------------ MMA issuer
        if (lane == 0 && nkt > 0) {
            const uint32_t idesc_s = make_idesc(1, 1, 0, 0, 128, 128);
            const uint32_t idesc_pv = make_idesc(1, 1, 0, 1, 128, static_cast<uint32_t>(a.d_v));
            const uint32_t qa = smem_u32(base + L.q);
            // S(j) once the softmax has read S(j - 1) (it does so first thing)
            auto issue_s = [&](int j) -> bool {
                const int st = j % a.stages;
                if (!mbar_wait(&sm.k_full[st], static_cast<uint32_t>(j / a.stages) & 1u, a.wait_budget) || sm.abort)
                    return false;
                if (j >= 1 && !mbar_wait(&sm.s_free, static_cast<uint32_t>(j - 1) & 1u, a.wait_budget))
                    return false;
                tc_fence_after();
                const uint32_t ka = smem_u32(base + L.k_ring + st * L.k_stage);
                for (int c = 0; c < QC; ++c)
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk) {
                        const uint64_t ad = make_sdesc(qa + c * kChunkBytes + kk * 32, 16, 1024, kSwizzle128B);
                        const uint64_t bd = make_sdesc(ka + c * kChunkBytes + kk * 32, 16, 1024, kSwizzle128B);
                        mma_bf16_ss(tmem + kColS, ad, bd, idesc_s, (c > 0 || kk > 0) ? 1u : 0u);
                    }
                tc_commit(&sm.k_empty[st]);
                tc_commit(&sm.s_full);
                return true;
            };
            bool ok = mbar_wait(&sm.q_full, 0, a.wait_budget) && !sm.abort;
            if (ok) ok = issue_s(0);
            for (int j = 0; j < nkt && ok; ++j) {
                if (j + 1 < nkt && !(ok = issue_s(j + 1))) break;
                if (!mbar_wait(&sm.p_full[j & 1], static_cast<uint32_t>(j >> 1) & 1u, a.wait_budget) ||
                    !mbar_wait(&sm.v_full[j % kMhaVStages], static_cast<uint32_t>(j / kMhaVStages) & 1u,
                               a.wait_budget) ||
                    sm.abort) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                // B = V(j): MN-major, 64-column blocks of 128 rows (LBO = the
                // block stride), 8-row groups 1 KB apart; a 16-key step is 2 KB.
                // A = P_hi, P_lo from TMEM: 16 keys = 8 columns per step.
                const uint32_t va = smem_u32(base + L.v_ring + (j % kMhaVStages) * L.v_stage);
#pragma unroll
                for (int ks = 0; ks < kMhaTile / 16; ++ks) {
                    const uint64_t bd = make_sdesc(va + ks * 2048, kChunkBytes, 1024, kSwizzle128B);
                    const uint32_t pcol = kColP + (j & 1) * 128 + ks * 8;
                    mma_bf16_ts(tmem + kColO, tmem + pcol, bd, idesc_pv, (j > 0 || ks > 0) ? 1u : 0u);
                    mma_bf16_ts(tmem + kColO, tmem + pcol + 64, bd, idesc_pv, 1u);
                }
                tc_commit(&sm.v_empty[j % kMhaVStages]);
                tc_commit(&sm.pv_done[j & 1]);
            }
            if (!ok) {
                record_status(a.status, DSA_ERR_TIMEOUT);
                sm.abort = 1;
            }
            // every MMA issued completes before TMEM is freed
            tc_commit(&sm.mma_done);
            if (!mbar_wait(&sm.mma_done, 0, a.wait_budget)) record_status(a.status, DSA_ERR_TIMEOUT);
        }
    } else {
        // ------------------------------------- softmax: two warps per row
        // A row (query) is TMEM lane r; warps w and w + 4 share the lane
        // quarter w % 4 and take the key columns [0, 64) and [64, 128) of
        // each tile (and halves of O's columns), exchanging their half-row
        // maxima (and, at the end, row sums) through shared memory under a
        // named barrier of the pair.
        const int qr = warp & 3;              // this warp's quarter of the TMEM lanes
        const int hf = (warp - 2) >> 2;       // which half of the columns
        const int bar_id = 1 + ((warp - 2) & 3);
        const int r = qr * 32 + lane;
        const int t = t0 + r;
        const bool valid = r < nrows;
        const int n_t = valid ? min(a.q_n[t], a.max_n) : 0;
        const uint32_t lane_addr = tmem + (static_cast<uint32_t>(qr * 32) << 16);
        const uint32_t *mrow = (a.mask != nullptr && valid) ? a.mask + static_cast<int64_t>(t) * a.mask_words : nullptr;
        const int oc0 = hf * (a.d_v / 2), oc1 = oc0 + a.d_v / 2;  // this warp's O columns
        float m_used = -INFINITY, l = 0.f;  // l: this half's share of the row sum
        bool ok = true;
        for (int j = 0; j < nkt; ++j) {
            const int b = j & 1;  // P buffer; also the slot of the half-max exchange
            ok = __all_sync(0xffffffffu, mbar_wait(&sm.s_full, static_cast<uint32_t>(j) & 1u, a.wait_budget) &&
                                             !sm.abort);
            ok = bar_and(bar_id, 64, ok);
            if (!ok) break;
            tc_fence_after();
            uint32_t u[64];
            tmem_ld32(lane_addr + kColS + hf * 64, *reinterpret_cast<uint32_t(*)[32]>(u));
            tmem_ld32(lane_addr + kColS + hf * 64 + 32, *reinterpret_cast<uint32_t(*)[32]>(u + 32));
            tmem_wait_ld();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&sm.s_free);
            // keys j*128 + hf*64 + c kept: below n_t and in the index set
            uint32_t mw[2];
#pragma unroll
            for (int w = 0; w < 2; ++w) {
                const int s0 = j * kMhaTile + hf * 64 + w * 32;
                uint32_t bits = s0 >= n_t ? 0u : (n_t - s0 >= 32 ? 0xffffffffu : ((1u << (n_t - s0)) - 1u));
                if (mrow != nullptr && bits != 0u) bits &= mrow[j * 4 + hf * 2 + w];
                mw[w] = bits;
            }
            float x[64];
            float mh = -INFINITY;
#pragma unroll
            for (int c = 0; c < 64; ++c) {
                x[c] = ((mw[c >> 5] >> (c & 31)) & 1u) ? __uint_as_float(u[c]) * a.scale_log2 : -INFINITY;
                mh = fmaxf(mh, x[c]);
            }
            // the tile's row max from both halves (double-buffered slots: the
            // partner reads slot b of tile j before either writes it again at
            // tile j + 2, two barriers later)
            sm.half_max[b][hf][r] = mh;
            bar_sync(bar_id, 64);
            const float mt = fmaxf(sm.half_max[b][0][r], sm.half_max[b][1][r]);
            float alpha = 1.f;
            bool rescale = false;  // O holds earlier tiles' products to scale by alpha
            if (mt > m_used + kRaiseLog2) {
                alpha = m_used == -INFINITY ? 0.f : fast_exp2(m_used - mt);
                rescale = m_used != -INFINITY;
                m_used = mt;
                l *= alpha;
            }
            // P(j) goes to buffer j % 2, which P(j - 2) . V(j - 2) must be done
            // reading; a rescale of O needs every tile before j in O.  (The
            // two warps of a pair hold the same rows: same decisions, same
            // waits.)
            const bool need_o = __any_sync(0xffffffffu, rescale) && j >= 1;
            if (j >= 2 || need_o) {
                bool w = true;
                if (need_o)
                    w = mbar_wait(&sm.pv_done[(j - 1) & 1], static_cast<uint32_t>((j - 1) >> 1) & 1u, a.wait_budget);
                if (w && j >= 2)
                    w = mbar_wait(&sm.pv_done[b], static_cast<uint32_t>((j - 2) >> 1) & 1u, a.wait_budget);
                ok = __all_sync(0xffffffffu, w && !sm.abort);
                ok = bar_and(bar_id, 64, ok);  // both warps of the pair leave together
                if (!ok) break;
                tc_fence_after();
            }
            if (need_o) {
                const float f = rescale ? alpha : 1.f;
                for (int c = oc0; c < oc1; c += 32) {
                    uint32_t o[32];
                    tmem_ld32(lane_addr + kColO + c, o);
                    tmem_wait_ld();
#pragma unroll
                    for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * f);
                    tmem_st32(lane_addr + kColO + c, o);
                }
            }
            float lsum = 0.f;
#pragma unroll
            for (int c0 = 0; c0 < 64; c0 += 32) {
                uint32_t hi[16], lo[16];
#pragma unroll
                for (int e = 0; e < 16; ++e) {
                    const float x0 = x[c0 + 2 * e], x1 = x[c0 + 2 * e + 1];
                    const float p0 = x0 == -INFINITY ? 0.f : fast_exp2(x0 - m_used);
                    const float p1 = x1 == -INFINITY ? 0.f : fast_exp2(x1 - m_used);
                    lsum += p0 + p1;
                    const __nv_bfloat162 h2 = __floats2bfloat162_rn(p0, p1);
                    const float2 hfl = __bfloat1622float2(h2);
                    hi[e] = bf16x2_bits(h2);
                    lo[e] = bf16x2_bits(__floats2bfloat162_rn(p0 - hfl.x, p1 - hfl.y));
                }
                tmem_st16(lane_addr + kColP + b * 128 + hf * 32 + c0 / 2, hi);
                tmem_st16(lane_addr + kColP + b * 128 + 64 + hf * 32 + c0 / 2, lo);
            }
            l += lsum;
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&sm.p_full[b]);
        }
        // epilogue: O / l as bf16 (this warp's columns), and the log-sum-exp
        if (ok && nkt > 0)
            ok = __all_sync(0xffffffffu,
                            mbar_wait(&sm.pv_done[(nkt - 1) & 1], static_cast<uint32_t>((nkt - 1) >> 1) & 1u,
                                      a.wait_budget) &&
                                !sm.abort);
        sm.half_sum[hf][r] = l;
        ok = bar_and(bar_id, 64, ok);
        if (ok) {
            tc_fence_after();
            const float lrow = sm.half_sum[0][r] + sm.half_sum[1][r];
            const float inv_l = lrow > 0.f ? 1.f / lrow : 0.f;
            uint16_t *dst = a.out + (static_cast<int64_t>(t) * a.h + head) * a.d_v;
            for (int c = oc0; c < oc1; c += 32) {
                uint32_t o[32];
                if (nkt > 0) {
                    tmem_ld32(lane_addr + kColO + c, o);
                    tmem_wait_ld();
                } else {
#pragma unroll
                    for (int i = 0; i < 32; ++i) o[i] = 0u;
                }
                uint32_t w[16];
#pragma unroll
                for (int e = 0; e < 16; ++e)
                    w[e] = bf16x2_bits(__floats2bfloat162_rn(__uint_as_float(o[2 * e]) * inv_l,
                                                             __uint_as_float(o[2 * e + 1]) * inv_l));
                if (valid) {
                    uint4 *d4 = reinterpret_cast<uint4 *>(dst + c);
#pragma unroll
                    for (int g = 0; g < 4; ++g) d4[g] = make_uint4(w[4 * g], w[4 * g + 1], w[4 * g + 2], w[4 * g + 3]);
                }
            }
            if (valid && hf == 0)
                a.lse[static_cast<int64_t>(t) * a.h + head] =
                    lrow > 0.f ? (m_used + log2f(lrow)) * 0.6931471805599453f : -INFINITY;
        } else if (lane == 0) {
            record_status(a.status, DSA_ERR_TIMEOUT);
        }
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) tmem_dealloc(tmem, 512);
}

// The membership bitmap of each query's index set: bit s of row t set iff s
// is listed in idx[t, :] and s < q_n[t].  An entry >= q_n[t] is skipped and
// flags DSA_ERR_DEVICE_CHECK.
__global__ void __launch_bounds__(256) k12_mha_mask(const int32_t *idx, int topk, const int32_t *q_n,
                                                    uint32_t *mask, int words, int *status) {
    grid_dependency_wait();
    const int t = blockIdx.x;
    uint32_t *row = mask + static_cast<int64_t>(t) * words;
    for (int w = threadIdx.x; w < words; w += blockDim.x) row[w] = 0u;
    __syncthreads();
    const int n = min(q_n[t], words * 32);
    const int32_t *ix = idx + static_cast<int64_t>(t) * topk;
    for (int e = threadIdx.x; e < topk; e += blockDim.x) {
        const int s = ix[e];
        if (s >= n) record_status(status, DSA_ERR_DEVICE_CHECK);
        else if (s >= 0) atomicOr(row + (s >> 5), 1u << (s & 31));
    }
}

namespace {
template <class... KArgs, class... Args>
cudaError_t launch_pdl(void (*kern)(KArgs...), int grid, int block, size_t smem, cudaStream_t st,
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
}  // namespace

cudaError_t launch_mha_mask(const int32_t *idx, int topk, const int32_t *q_n, uint32_t *mask, int words, int nq,
                            int *status, cudaStream_t st) {
    if (nq == 0) return cudaSuccess;
    return launch_pdl(k12_mha_mask, nq, 256, 0, st, idx, topk, q_n, mask, words, status);
}

cudaError_t launch_masked_mha(const CUtensorMap &qmap, const CUtensorMap &kmap, const CUtensorMap &vmap,
                              const MhaParams &a, int grid, cudaStream_t st) {
    const MhaLayout L = mha_layout(a.d_qk, a.d_v, a.stages);
    const size_t smem = smem_for_tmem(L.total, 512);
    cudaError_t e = cudaFuncSetAttribute(k11_masked_mha, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    if (grid == 0) return cudaSuccess;
    return launch_pdl(k11_masked_mha, grid, kMhaThreads, smem, st, qmap, kmap, vmap, a);
}

}  // namespace dsa
