// project.cu -- the lightning indexer's own projections on sm_100a: the step
// that produces q^I, k^I and the head weights the indexer score consumes
// ("DeepSeekV3.2之DSA" by yuyanqi, sections 4.1-4.3), with k^I appended to
// the index-K cache (its decode data flow, section 5.1):
//   q^I[t] = W_qb . q_lora[t]                 -> [H_I, d_I], RoPE, FP8 + scale
//   k^I[t] = LayerNorm(W_k . x[t])            -> RoPE, FP8 + scale -> cache row
//   w[t]   = (W_proj . x[t]) * H_I^-1/2 * d_I^-1/2 * q_scale[t]   -> bf16
// RoPE rotates the pairs (2i, 2i+1) of the first rope_dim dims by
// pos * theta^(-2i / rope_dim); the FP8 scales are powers of two (the e8m0
// k_s of section 4.3; the same for q, so folding it into w is exact).
//
// k5_proj_gemm: both contractions in one launch, on the tensor cores, with
// the weights as the MMA's M operand (128 output rows per tile) and the
// tokens as N (16 to 256 per tile): at decode a tile then streams 16 KB of
// weights and only N x 128 bytes of activations per 64-wide K step, so a
// deep TMA ring keeps many weight bytes in flight.  A work item is
// (problem, 128-output tile, token tile, K slice); K is split into slices
// until the grid fills the SMs, in proportion to each problem's weight
// bytes; the epilogue writes the slice's fp32 partial sums.
// k6_proj_epilogue: one CTA per token sums the slices in a fixed order and
// applies LayerNorm, RoPE, the quantisation, the weight folding and the
// cache append.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp8.h>
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

#include "kernels.h"
#include "ptx.cuh"

namespace dsa {

namespace {

constexpr int kPBm = 128;                 // weight rows per tile (MMA M)
constexpr int kPBk = 64;                  // K per stage (128 bytes of bf16: one swizzle span)
constexpr int kPABytes = kPBm * kPBk * 2; // 16 KB of weights per stage

struct ProjSmem {
    uint64_t full[kProjMaxStages];
    uint64_t empty[kProjMaxStages];
    uint64_t acc_full;
    uint32_t tmem_base;
    volatile int32_t abort;
};

__device__ __forceinline__ uint8_t *align1024(uint8_t *p) {
    return reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}

__device__ __forceinline__ float warp_sum_f(float x) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
    return x;
}
__device__ __forceinline__ float warp_max_f(float x) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, o));
    return x;
}

// The smallest power of two 2^e with amax / 2^e <= 448 (the E4M3 maximum);
// 1 when amax is 0.  frexp makes the test exact: amax / 448 = f * 2^e with f
// in [0.5, 1) is at most 2^e, and equals 2^(e-1) when f = 0.5.
__device__ __forceinline__ float pow2_scale(float amax) {
    if (!(amax > 0.f)) return 1.f;
    int e;
    const double f = frexp(static_cast<double>(amax) / 448.0, &e);
    return static_cast<float>(ldexp(1.0, f == 0.5 ? e - 1 : e));
}

__device__ __forceinline__ uint32_t e4m3(float x) {
    return static_cast<uint32_t>(__nv_cvt_float_to_fp8(x, __NV_SATFINITE, __NV_E4M3));
}

// The rotation of pair i (dims 2i, 2i+1) at position pos: angle
// pos * theta^(-2i/rope_dim) in double (positions reach 2^27; an fp32 angle
// would lose the fraction).  A token's pairs are the same for its k^I and
// every q^I head, so each CTA computes them once (rope_table).
__device__ __forceinline__ void rope_angle(int i, int rope_dim, int pos, float theta, double &s, double &c) {
    const double inv = pow(static_cast<double>(theta), -2.0 * static_cast<double>(i) / static_cast<double>(rope_dim));
    sincos(static_cast<double>(pos) * inv, &s, &c);
}

__device__ __forceinline__ void rope_pair(float &v0, float &v1, const double2 &sc) {
    const double x0 = v0, x1 = v1;
    v0 = static_cast<float>(x0 * sc.y - x1 * sc.x);
    v1 = static_cast<float>(x0 * sc.x + x1 * sc.y);
}

}  // namespace

// ---------------------------------------------------------------------------
// k5: split-K tcgen05 GEMM of both projections, D[output, token].  192
// threads: warp 0 TMA, warp 1 MMA, warps 2-5 epilogue (TMEM lane quarter =
// warp % 4; a lane is an output row, a column a token).
// Problem 0 stacks W_k (rows 0..d_I-1) and W_proj (rows d_I..d_I+H_I-1), in
// 64-row pieces; problem 1 is W_qb.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(192, 1)
    k5_proj_gemm(const __grid_constant__ CUtensorMap x_map, const __grid_constant__ CUtensorMap ql_map,
                 const __grid_constant__ CUtensorMap wk_map, const __grid_constant__ CUtensorMap wp_map,
                 const __grid_constant__ CUtensorMap wq_map, const ProjGemmParams a) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *base = align1024(smem_raw);
    ProjSmem &sm = *reinterpret_cast<ProjSmem *>(base + static_cast<uint32_t>(a.stages) * a.stage_bytes);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

    const int prob = static_cast<int>(blockIdx.x) < a.items0 ? 0 : 1;
    const int it = prob ? static_cast<int>(blockIdx.x) - a.items0 : static_cast<int>(blockIdx.x);
    const int split = it % a.splits[prob];
    const int rest = it / a.splits[prob];
    const int t_tile = rest % a.t_tiles;
    const int m_tile = rest / a.t_tiles;
    const int k_begin = static_cast<int>(static_cast<int64_t>(split) * a.k_steps[prob] / a.splits[prob]);
    const int k_end = static_cast<int>(static_cast<int64_t>(split + 1) * a.k_steps[prob] / a.splits[prob]);
    const int nk = k_end - k_begin;
    const int N = a.n_tok;
    const uint32_t tmem_cols = N <= 32 ? 32u : (N <= 64 ? 64u : (N <= 128 ? 128u : 256u));
    // problem 0: the two 64-row pieces of this tile come from W_k or W_proj
    const int n_out = prob == 0 ? a.d_idx + a.h_idx : a.h_idx * a.d_idx;
    uint32_t piece_bytes[2] = {0u, 0u};
    if (prob == 0) {
        for (int pc = 0; pc < 2; ++pc) {
            const int r0 = m_tile * kPBm + 64 * pc;
            if (r0 < a.d_idx) piece_bytes[pc] = 64u * kPBk * 2u;
            else if (r0 < a.d_idx + a.h_idx) piece_bytes[pc] = static_cast<uint32_t>(a.h_idx) * kPBk * 2u;
        }
    }
    const uint32_t a_bytes = prob == 0 ? piece_bytes[0] + piece_bytes[1] : static_cast<uint32_t>(kPABytes);
    const uint32_t b_bytes = static_cast<uint32_t>(N) * kPBk * 2u;

    if (tid == 0) {
        sm.abort = 0;
        for (int s = 0; s < a.stages; ++s) {
            mbar_init(&sm.full[s], 1);
            mbar_init(&sm.empty[s], 1);
        }
        mbar_init(&sm.acc_full, 1);
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc(&sm.tmem_base, tmem_cols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = sm.tmem_base;

    if (warp == 0) {
        if (lane == 0) {
            int s = 0;
            uint32_t ph = 0;
            int t_end = 0;
            for (int t = 0; t < nk; ++t) {
                if (!mbar_wait(&sm.empty[s], ph ^ 1, a.wait_budget) || sm.abort) {
                    record_status(a.status, DSA_ERR_TIMEOUT);
                    sm.abort = 1;
                    break;
                }
                uint8_t *st = base + static_cast<uint32_t>(s) * a.stage_bytes;
                const int k0 = (k_begin + t) * kPBk;
                mbar_arrive_expect_tx(&sm.full[s], a_bytes + b_bytes);
                if (prob == 0) {
                    for (int pc = 0; pc < 2; ++pc) {
                        const int r0 = m_tile * kPBm + 64 * pc;
                        if (r0 < a.d_idx) tma_load_2d(st + pc * 64 * 128, &wk_map, &sm.full[s], k0, r0);
                        else if (r0 < a.d_idx + a.h_idx)
                            tma_load_2d(st + pc * 64 * 128, &wp_map, &sm.full[s], k0, r0 - a.d_idx);
                    }
                    tma_load_2d(st + kPABytes, &x_map, &sm.full[s], k0, t_tile * N);
                } else {
                    tma_load_2d(st, &wq_map, &sm.full[s], k0, m_tile * kPBm);
                    tma_load_2d(st + kPABytes, &ql_map, &sm.full[s], k0, t_tile * N);
                }
                t_end = t + 1;
                if (++s == a.stages) { s = 0; ph ^= 1; }
            }
            // every load issued lands before the CTA may exit
            for (int t = max(t_end - a.stages, 0); t < t_end; ++t)
                mbar_wait(&sm.full[t % a.stages], static_cast<uint32_t>(t / a.stages) & 1u, a.wait_budget);
        }
    } else if (warp == 1) {
        if (lane == 0) {
            const uint32_t idesc = make_idesc(1, 1, 0, 0, kPBm, static_cast<uint32_t>(N));
            int s = 0;
            uint32_t ph = 0;
            for (int t = 0; t < nk; ++t) {
                if (!mbar_wait(&sm.full[s], ph, a.wait_budget) || sm.abort) {
                    record_status(a.status, DSA_ERR_TIMEOUT);
                    sm.abort = 1;
                    break;
                }
                tc_fence_after();
                const uint32_t aa = smem_u32(base + static_cast<uint32_t>(s) * a.stage_bytes);
                const uint32_t ba = aa + kPABytes;
#pragma unroll
                for (int kk = 0; kk < kPBk / 16; ++kk) {
                    const uint64_t ad = make_sdesc(aa + kk * 32, 16, 1024, kSwizzle128B);
                    const uint64_t bd = make_sdesc(ba + kk * 32, 16, 1024, kSwizzle128B);
                    mma_bf16_ss(tmem, ad, bd, idesc, (t > 0 || kk > 0) ? 1u : 0u);
                }
                tc_commit(&sm.empty[s]);
                if (++s == a.stages) { s = 0; ph ^= 1; }
            }
            // completes once every MMA issued above has (also when none was)
            tc_commit(&sm.acc_full);
        }
    } else {
        // epilogue: TMEM lane = output row, column = token of the tile
        const int quarter = warp & 3;
        const int col = m_tile * kPBm + quarter * 32 + lane;  // output index (column of part)
        const bool ok = warp_wait(&sm.acc_full, 0, &sm.abort, a.wait_budget);
        if (ok) {
            tc_fence_after();
            const uint32_t lane_addr = tmem + (static_cast<uint32_t>(quarter * 32) << 16);
            float *p = a.part[prob] + static_cast<int64_t>(split) * a.nt * a.ld[prob] + col;
            for (int c0 = 0; c0 < N; c0 += 32) {
                uint32_t v[32];
                tmem_ld32(lane_addr + c0, v);
                tmem_wait_ld();
                if (col < n_out) {
#pragma unroll
                    for (int j = 0; j < 32; ++j) {
                        const int token = t_tile * N + c0 + j;
                        if (c0 + j < N && token < a.nt) p[static_cast<int64_t>(token) * a.ld[prob]] = __uint_as_float(v[j]);
                    }
                }
            }
        } else if (lane == 0) {
            record_status(a.status, DSA_ERR_TIMEOUT);
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) tmem_dealloc(tmem, tmem_cols);
}

// ---------------------------------------------------------------------------
// k6: sum the K slices (in slice order) and finish the producer.  Grid
// (token, 1 + H_I / 8): block y = 0 produces the token's k^I (warp 0) and
// the raw head weights (warp 1); block y >= 1 produces q^I heads
// 8 (y - 1) .. 8 (y - 1) + 7, one per warp, each warp summing its own head
// weight.  Lane l of a warp holds dims [l * per, (l + 1) * per) of a
// d_I-wide vector (per = d_I / 32: 4 or 2), so every RoPE pair is in-lane.
// Spreading a token over several CTAs keeps the dependent chains (partial
// loads, reductions, quantisation) short: one CTA per token ran them head
// after head.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) k6_proj_epilogue(const ProjEpiParams a) {
    __shared__ double2 rope_table[64];  // (sin, cos) of each rotated pair at this token's position
    const int t = blockIdx.x;
    const int hgroup = static_cast<int>(blockIdx.y) - 1;  // -1: the k^I block
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int d = a.d_idx, H = a.h_idx, per = a.d_idx / 32;
    const int pos = a.positions[t];
    for (int i = threadIdx.x; i < a.rope_dim / 2; i += blockDim.x) {
        double sn, cs;
        rope_angle(i, a.rope_dim, pos, a.rope_theta, sn, cs);
        rope_table[i] = make_double2(sn, cs);
    }
    __syncthreads();

    if (hgroup < 0 && warp == 0) {
        // ---- k^I: LayerNorm, RoPE, FP8 with a power-of-two scale, cache append
        float v[4];
        for (int i = 0; i < per; ++i) {
            const int o = lane * per + i;
            float acc = 0.f;
            for (int s = 0; s < a.splits0; ++s) acc += a.part0[(static_cast<int64_t>(s) * a.nt + t) * a.ld0 + o];
            v[i] = acc;
        }
        float sum = 0.f;
        for (int i = 0; i < per; ++i) sum += v[i];
        const float mean = warp_sum_f(sum) / static_cast<float>(d);
        float sq = 0.f;
        for (int i = 0; i < per; ++i) sq += (v[i] - mean) * (v[i] - mean);
        const float var = warp_sum_f(sq) / static_cast<float>(d);
        const float inv_std = 1.f / sqrtf(var + a.ln_eps);
        for (int i = 0; i < per; ++i) {
            const int o = lane * per + i;
            v[i] = (v[i] - mean) * inv_std * a.ln_gamma[o] + a.ln_beta[o];
        }
        for (int i = 0; i < per; i += 2) {
            const int o = lane * per + i;
            if (o < a.rope_dim) rope_pair(v[i], v[i + 1], rope_table[o / 2]);
        }
        float amax = 0.f;
        for (int i = 0; i < per; ++i) amax = fmaxf(amax, fabsf(v[i]));
        const float scale = pow2_scale(warp_max_f(amax));
        const float inv = 1.f / scale;  // exact: a power of two
        // cache row of (sequence, position)
        const int seq = a.q_seq[t];
        int64_t row;
        if (a.page_table)
            row = static_cast<int64_t>(a.page_table[static_cast<int64_t>(seq) * a.max_pages + pos / a.page_size]) *
                      a.page_size + pos % a.page_size;
        else
            row = a.seq_row0[seq] + pos;
        const bool in_range = pos >= 0 && row >= 0 && row < a.cache_rows &&
                              (a.page_table == nullptr || static_cast<int64_t>(pos) / a.page_size < a.max_pages);
        if (!in_range) {
            if (lane == 0) record_status(a.status, DSA_ERR_DEVICE_CHECK);
        } else {
            uint32_t packed = 0;
            for (int i = 0; i < per; ++i) packed |= e4m3(v[i] * inv) << (8 * i);
            uint8_t *dst = a.kidx_cache + row * d + lane * per;
            if (per == 4) *reinterpret_cast<uint32_t *>(dst) = packed;
            else *reinterpret_cast<uint16_t *>(dst) = static_cast<uint16_t>(packed);
            if (lane == 0) a.k_scale[row] = scale;
        }
        if (a.k_f32)
            for (int i = 0; i < per; ++i) a.k_f32[static_cast<int64_t>(t) * d + lane * per + i] = v[i];
    } else if (hgroup < 0 && warp == 1) {
        // ---- the raw head weights W_proj . x (optional fp32 output)
        if (a.w_f32)
            for (int j = lane; j < H; j += 32) {
                float acc = 0.f;
                for (int s = 0; s < a.splits0; ++s) acc += a.part0[(static_cast<int64_t>(s) * a.nt + t) * a.ld0 + d + j];
                a.w_f32[static_cast<int64_t>(t) * H + j] = acc;
            }
    }
    // ---- q^I head h of this block: RoPE, FP8 with a power-of-two scale; w
    // folds the scale
    const int h = hgroup * 8 + warp;
    if (hgroup >= 0 && h < H) {
        float v[4];
        const int64_t col0 = static_cast<int64_t>(h) * d + lane * per;
        for (int i = 0; i < per; ++i) {
            float acc = 0.f;
            for (int s = 0; s < a.splits1; ++s) acc += a.part1[(static_cast<int64_t>(s) * a.nt + t) * a.ld1 + col0 + i];
            v[i] = acc;
        }
        for (int i = 0; i < per; i += 2) {
            const int o = lane * per + i;
            if (o < a.rope_dim) rope_pair(v[i], v[i + 1], rope_table[o / 2]);
        }
        float amax = 0.f;
        for (int i = 0; i < per; ++i) amax = fmaxf(amax, fabsf(v[i]));
        const float scale = pow2_scale(warp_max_f(amax));
        const float inv = 1.f / scale;
        uint32_t packed = 0;
        for (int i = 0; i < per; ++i) packed |= e4m3(v[i] * inv) << (8 * i);
        uint8_t *dst = a.q_idx + (static_cast<int64_t>(t) * H + h) * d + lane * per;
        if (per == 4) *reinterpret_cast<uint32_t *>(dst) = packed;
        else *reinterpret_cast<uint16_t *>(dst) = static_cast<uint16_t>(packed);
        if (a.q_f32)
            for (int i = 0; i < per; ++i) a.q_f32[(static_cast<int64_t>(t) * H + h) * d + lane * per + i] = v[i];
        if (lane == 0) {
            const int64_t th = static_cast<int64_t>(t) * H + h;
            if (a.q_scale) a.q_scale[th] = scale;
            float wraw = 0.f;  // W_proj . x for head h, slices summed in order
            for (int s = 0; s < a.splits0; ++s) wraw += a.part0[(static_cast<int64_t>(s) * a.nt + t) * a.ld0 + d + h];
            // the same operations, in the same order, as the definition:
            // w / sqrt(H_I) / sqrt(d_I) * q_scale, then bf16 (ties to even)
            const double wv = static_cast<double>(wraw) / sqrt(static_cast<double>(H)) /
                              sqrt(static_cast<double>(d)) * static_cast<double>(scale);
            a.w[th] = __bfloat16_as_ushort(__double2bfloat16(wv));
        }
    }
}

cudaError_t launch_project(const CUtensorMap &x_map, const CUtensorMap &ql_map, const CUtensorMap &wk_map,
                           const CUtensorMap &wp_map, const CUtensorMap &wq_map, const ProjGemmParams &g,
                           const ProjEpiParams &e, cudaStream_t st) {
    const size_t smem = static_cast<size_t>(g.stages) * g.stage_bytes + sizeof(ProjSmem) + 1024;
    cudaError_t err = cudaFuncSetAttribute(k5_proj_gemm, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                           static_cast<int>(smem));
    if (err != cudaSuccess) return err;
    const int grid = g.items0 + g.m_tiles[1] * g.t_tiles * g.splits[1];
    if (grid == 0 || g.nt == 0) return cudaSuccess;
    k5_proj_gemm<<<grid, 192, smem, st>>>(x_map, ql_map, wk_map, wp_map, wq_map, g);
    err = cudaGetLastError();
    if (err != cudaSuccess) return err;
    k6_proj_epilogue<<<dim3(g.nt, 1 + (g.h_idx + 7) / 8), 256, 0, st>>>(e);
    return cudaGetLastError();
}

}  // namespace dsa
