// select.cuh -- exact block-wide TopK on order-preserving keys.
//
// An element is the 64-bit composite V = key << 32 | ~pos, where key is the
// order-preserving image of its fp32 score and pos its position.  Larger V
// means a larger score, and among equal scores a lower position, so the TopK
// set with ties broken toward the lower position is exactly the K largest
// composites, and all composites are distinct.  The K-th largest composite
// is found by a most-significant-digit radix search (digits of 11, 11, 10,
// 11, 11, 10 bits) over shared-memory histograms; the set is then
// {V >= threshold}.
#pragma once

#include "kernels.h"
#include "ptx.cuh"

namespace dsa {

constexpr int kSelBins = 2048;  // widest digit: 11 bits
// Digit p of the composite covers bits [shift, shift + width).
__device__ __forceinline__ int digit_shift(int p) {
    return p == 0 ? 53 : p == 1 ? 42 : p == 2 ? 32 : p == 3 ? 21 : p == 4 ? 10 : 0;
}
__device__ __forceinline__ int digit_width(int p) { return (p == 2 || p == 5) ? 10 : 11; }

struct SelectScratch {
    uint32_t csum[64];     // per-32-bin chunk sums
    uint32_t res[4];       // digit, count above the digit's bucket, bucket size
    uint32_t counter[4];   // emission slots
    uint32_t wsum[32];     // per-warp counts of an ordered compaction
};

__device__ __forceinline__ uint64_t make_composite(uint32_t key, uint32_t pos) {
    return (static_cast<uint64_t>(key) << 32) | static_cast<uint32_t>(~pos);
}
__device__ __forceinline__ uint32_t composite_pos(uint64_t v) {
    return ~static_cast<uint32_t>(v);
}
__device__ __forceinline__ uint32_t top_digit(uint32_t key) { return key >> 21; }

__device__ __forceinline__ uint32_t warp_incl_scan(uint32_t x) {
    const int lane = threadIdx.x & 31;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        uint32_t y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
    }
    return x;
}
__device__ __forceinline__ uint32_t warp_sum(uint32_t x) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
    return x;
}

// Scanning `hist` (nbins bins) from the highest bin down, find the bin where
// the running count first reaches `need` (1 <= need <= total).  Writes
// res[0] = bin, res[1] = count in higher bins, res[2] = count in the bin.
// Block-wide: every thread must call it; ends with __syncthreads().
__device__ void find_digit(const uint32_t *hist, int nbins, uint32_t need, SelectScratch &sc) {
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, nwarps = blockDim.x >> 5;
    const int nch = nbins >> 5;
    // chunk sums: eight threads per 32-bin chunk, four bins per 16-byte load
    for (int t = tid; t < nbins / 4; t += blockDim.x) {
        const uint4 h4 = reinterpret_cast<const uint4 *>(hist)[t];
        uint32_t x = (h4.x + h4.y) + (h4.z + h4.w);
        x += __shfl_xor_sync(0xffffffffu, x, 1);
        x += __shfl_xor_sync(0xffffffffu, x, 2);
        x += __shfl_xor_sync(0xffffffffu, x, 4);
        if ((t & 7) == 0) sc.csum[t >> 3] = x;
    }
    (void)nwarps;
    __syncthreads();
    if (warp == 0) {
        // chunks in descending order: lane l holds chunk nch-1-l and nch-33-l
        uint32_t a = (lane < nch) ? sc.csum[nch - 1 - lane] : 0u;
        uint32_t b = (lane + 32 < nch) ? sc.csum[nch - 33 - lane] : 0u;
        uint32_t ia = warp_incl_scan(a);
        uint32_t tot_a = __shfl_sync(0xffffffffu, ia, 31);
        uint32_t ib = warp_incl_scan(b) + tot_a;
        unsigned ba = __ballot_sync(0xffffffffu, ia >= need);
        unsigned bb = __ballot_sync(0xffffffffu, ib >= need);
        int pos;
        uint32_t incl, own;
        if (ba) {
            pos = __ffs(ba) - 1;
            incl = __shfl_sync(0xffffffffu, ia, pos);
            own = __shfl_sync(0xffffffffu, a, pos);
        } else {
            int p2 = bb ? __ffs(bb) - 1 : 31;  // need <= total guarantees bb != 0
            pos = 32 + p2;
            incl = __shfl_sync(0xffffffffu, ib, p2);
            own = __shfl_sync(0xffffffffu, b, p2);
        }
        const int chunk = max(nch - 1 - pos, 0);  // need > total only on malformed input
        const uint32_t above_chunk = incl - own;
        // bins of the chunk in descending order
        uint32_t v = hist[chunk * 32 + 31 - lane];
        uint32_t iv = warp_incl_scan(v) + above_chunk;
        unsigned bv = __ballot_sync(0xffffffffu, iv >= need);
        int p3 = bv ? __ffs(bv) - 1 : 31;
        uint32_t incl3 = __shfl_sync(0xffffffffu, iv, p3);
        uint32_t own3 = __shfl_sync(0xffffffffu, v, p3);
        if (lane == 0) {
            sc.res[0] = static_cast<uint32_t>(chunk * 32 + 31 - p3);
            sc.res[1] = incl3 - own3;
            sc.res[2] = own3;
        }
    }
    __syncthreads();
}

// Refine the K-th largest composite among elements of `src` whose digits
// above pass `pass0` equal `prefix` (prefix holds the top digits, already
// decided), needing the `need`-th largest of them (1 <= need <= their count).
// `src.load4(i, v)` fills v with elements i..i+3 (i a multiple of 4; the
// source is readable up to the next multiple of 4 past n).
// Returns the threshold T: the wanted set is {V >= T} among the elements
// with that prefix (plus everything with a larger prefix, decided earlier).
template <class Src>
__device__ uint64_t radix_refine(const Src &src, int n, uint64_t prefix, int pass0, uint32_t need,
                                 uint32_t *hist, SelectScratch &sc) {
    const int tid = threadIdx.x, nt = blockDim.x;
    for (int pass = pass0; pass < 6; ++pass) {
        const int shift = digit_shift(pass), width = digit_width(pass);
        const int nbins = 1 << width;
        const int hi = shift + width;
        for (int b = tid; b < nbins; b += nt) hist[b] = 0;
        __syncthreads();
        for (int i0 = 4 * tid; i0 < n; i0 += 4 * nt) {
            uint64_t v[4];
            src.load4(i0, v);
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                // refinement passes see few, spread-out elements: plain atomics
                if (i0 + e < n && (pass == 0 || (v[e] >> hi) == prefix))
                    atomicAdd(&hist[static_cast<uint32_t>(v[e] >> shift) & static_cast<uint32_t>(nbins - 1)], 1u);
            }
        }
        __syncthreads();
        find_digit(hist, nbins, need, sc);
        const uint32_t digit = sc.res[0], above = sc.res[1], bucket = sc.res[2];
        __syncthreads();
        need -= above;
        prefix = (prefix << width) | digit;
        if (bucket == need) return prefix << shift;
    }
    return prefix;
}

// Ordered block-wide compaction: the elements i in [0, n) with pred(v) true
// are handed to out(slot, v) with consecutive slots base, base + 1, ... in
// increasing i.  Warp w owns a contiguous slice (a multiple of 128
// elements) in steps of 128: each lane tests four consecutive elements per
// step (one src.load4), giving a 4-bit match mask; four ballots (one per
// element of the lanes' quads) record the step's matches for the warp.
//
// Pass 1 keeps each lane's masks in registers (up to 32 steps: two 64-bit
// words) and the step ballots in `bal`; a warp scan of the steps' match
// counts gives every step its first slot within the warp, and one
// block-wide scan of the warps' totals gives every warp its first slot.
// Pass 2 is per lane: a lane visits only the steps where it has a match
// (usually none or one), reads that step's ballots and prefix, reloads its
// quad and emits.  No loop in either pass branches on data while the warp
// must stay converged.  Slices longer than 32 steps (never planned) take a
// slower path that re-tests every step.
// Returns the next free slot.  `wsum`: 32 shared words; `bal`: shared, at
// least emit_ballot_words(n, warps) / 4 uint4, plus one word per step for the
// step prefixes when a slice has at most 32 steps (emit_ballot_words covers it).
template <class Src, class Pred, class Out>
__device__ uint32_t emit_ordered(const Src &src, int n, const Pred &pred, const Out &out,
                                 uint32_t base, uint32_t *wsum, uint4 *bal) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
    const int per = ((n + nw - 1) / nw + 127) & ~127;
    const int lo = min(warp * per, n), hi = min(lo + per, n);
    const int steps = (hi - lo + 127) / 128;
    const int wsteps = per / 128;  // steps of every full slice (same for all warps)
    uint4 *wb = bal + warp * wsteps;
    const uint32_t lt = (1u << lane) - 1u;  // lanes below this one
    uint32_t before = 0, total = 0;

    if (wsteps <= 32) {
        // ---- pass 1: masks in registers, ballots and step prefixes in shared
        uint64_t mask01 = 0, mask23 = 0;  // 4 bits per step: steps 0-15, 16-31
        uint4 mine = make_uint4(0, 0, 0, 0);
        for (int t = 0; t < steps; ++t) {
            const int i0 = lo + 128 * t + 4 * lane;
            uint64_t v[4];
            src.load4(i0 < hi ? i0 : lo, v);  // clamped: no branch around the load
            uint32_t m = 0;
#pragma unroll
            for (int e = 0; e < 4; ++e) m |= ((i0 + e < hi) & pred(v[e])) ? (1u << e) : 0u;
            if (t < 16) mask01 |= static_cast<uint64_t>(m) << (4 * t);
            else mask23 |= static_cast<uint64_t>(m) << (4 * (t - 16));
            const uint32_t q0 = __ballot_sync(0xffffffffu, m & 1u);
            const uint32_t q1 = __ballot_sync(0xffffffffu, m & 2u);
            const uint32_t q2 = __ballot_sync(0xffffffffu, m & 4u);
            const uint32_t q3 = __ballot_sync(0xffffffffu, m & 8u);
            mine = lane == t ? make_uint4(q0, q1, q2, q3) : mine;
        }
        // lane t: matches of step t -> exclusive prefix over steps
        const uint32_t tot_t = __popc(mine.x) + __popc(mine.y) + __popc(mine.z) + __popc(mine.w);
        const uint32_t incl = warp_incl_scan(tot_t);
        uint32_t *wpre = reinterpret_cast<uint32_t *>(bal + nw * wsteps) + warp * 32;
        if (lane < steps) {
            wb[lane] = mine;
            wpre[lane] = incl - tot_t;
        }
        if (lane == 31) wsum[warp] = incl;
        __syncthreads();
        for (int w = 0; w < nw; ++w) {
            const uint32_t c = wsum[w];
            before += (w < warp) ? c : 0u;
            total += c;
        }
        // ---- pass 2: each lane visits only its own matching steps
        const uint32_t wbase = base + before;
#pragma unroll
        for (int half = 0; half < 2; ++half) {
            uint64_t mm = half == 0 ? mask01 : mask23;
            while (mm != 0) {
                const int bit = __ffsll(static_cast<long long>(mm)) - 1;
                const int t = (bit >> 2) + 16 * half;
                const uint32_t own = static_cast<uint32_t>(mm >> (bit & ~3)) & 0xFu;
                mm &= ~(static_cast<uint64_t>(0xFu) << (bit & ~3));
                const uint4 q = wb[t];
                const uint32_t s0 = wbase + wpre[t] + __popc(q.x & lt) + __popc(q.y & lt) +
                                    __popc(q.z & lt) + __popc(q.w & lt);
                uint64_t v[4];
                src.load4(lo + 128 * t + 4 * lane, v);
                const uint32_t o0 = own & 1u, o1 = (own >> 1) & 1u, o2 = (own >> 2) & 1u;
                const uint32_t s1 = s0 + o0, s2 = s1 + o1, s3 = s2 + o2;
                if (own & 1u) out(s0, v[0]);
                if (own & 2u) out(s1, v[1]);
                if (own & 4u) out(s2, v[2]);
                if (own & 8u) out(s3, v[3]);
            }
        }
        __syncthreads();
        return base + total;
    }

    // ---- slices of more than 32 steps: count, scan, then re-test every step
    uint32_t cnt = 0;  // warp-uniform
    for (int t = 0; t < steps; ++t) {
        const int i0 = lo + 128 * t + 4 * lane;
        uint64_t v[4];
        src.load4(i0 < hi ? i0 : lo, v);
        uint32_t m = 0;
#pragma unroll
        for (int e = 0; e < 4; ++e) m |= ((i0 + e < hi) & pred(v[e])) ? (1u << e) : 0u;
        cnt += __popc(__ballot_sync(0xffffffffu, m & 1u)) + __popc(__ballot_sync(0xffffffffu, m & 2u)) +
               __popc(__ballot_sync(0xffffffffu, m & 4u)) + __popc(__ballot_sync(0xffffffffu, m & 8u));
    }
    if (lane == 0) wsum[warp] = cnt;
    __syncthreads();
    for (int w = 0; w < nw; ++w) {
        const uint32_t c = wsum[w];
        before += (w < warp) ? c : 0u;
        total += c;
    }
    uint32_t slot = base + before;
    for (int t = 0; t < steps; ++t) {
        const int i0 = lo + 128 * t + 4 * lane;
        uint64_t v[4];
        src.load4(i0 < hi ? i0 : lo, v);
        uint32_t m = 0;
#pragma unroll
        for (int e = 0; e < 4; ++e) m |= ((i0 + e < hi) & pred(v[e])) ? (1u << e) : 0u;
        const uint32_t q0 = __ballot_sync(0xffffffffu, m & 1u);
        const uint32_t q1 = __ballot_sync(0xffffffffu, m & 2u);
        const uint32_t q2 = __ballot_sync(0xffffffffu, m & 4u);
        const uint32_t q3 = __ballot_sync(0xffffffffu, m & 8u);
        const uint32_t s0 = slot + __popc(q0 & lt) + __popc(q1 & lt) + __popc(q2 & lt) + __popc(q3 & lt);
        const uint32_t s1 = s0 + (m & 1u), s2 = s1 + ((m >> 1) & 1u), s3 = s2 + ((m >> 2) & 1u);
        if (m & 1u) out(s0, v[0]);
        if (m & 2u) out(s1, v[1]);
        if (m & 4u) out(s2, v[2]);
        if (m & 8u) out(s3, v[3]);
        slot += __popc(q0) + __popc(q1) + __popc(q2) + __popc(q3);
    }
    __syncthreads();
    return base + total;
}

// Ordered block-wide compaction for large n with few matches: thread t owns
// the contiguous elements [t * seg, (t + 1) * seg), counts its matches, one
// block-wide scan gives each thread its first slot, and a second pass over
// its own elements writes them.  `seg` is a multiple of 4 whose quarter is
// odd, so the 16-byte loads of a warp start in eight different bank groups.
// Elements i with pred(v) true go to out(slot, v), slots base, base + 1, ...
// in increasing i.  `src.load4(i, v)` as for emit_ordered (readable up to the
// next multiple of 4 past n).  `wsum`: 32 shared words.  Returns the next
// free slot; ends with __syncthreads().
template <class Src, class Pred, class Out>
__device__ uint32_t compact_ordered(const Src &src, int n, const Pred &pred, const Out &out, uint32_t base,
                                    uint32_t *wsum) {
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, nw = blockDim.x >> 5;
    int seg = ((n + static_cast<int>(blockDim.x) - 1) / static_cast<int>(blockDim.x) + 3) & ~3;
    if (((seg >> 2) & 1) == 0) seg += 4;
    const int lo = min(tid * seg, n), hi = min(lo + seg, n);
    uint32_t cnt = 0;
    for (int i = lo; i < hi; i += 4) {
        uint64_t v[4];
        src.load4(i, v);
#pragma unroll
        for (int e = 0; e < 4; ++e) cnt += (i + e < hi && pred(v[e])) ? 1u : 0u;
    }
    const uint32_t incl = warp_incl_scan(cnt);
    if (lane == 31) wsum[warp] = incl;
    __syncthreads();
    uint32_t before = 0, total = 0;
    for (int w = 0; w < nw; ++w) {
        const uint32_t c = wsum[w];
        before += (w < warp) ? c : 0u;
        total += c;
    }
    uint32_t slot = base + before + incl - cnt;
    if (cnt) {
        for (int i = lo; i < hi; i += 4) {
            uint64_t v[4];
            src.load4(i, v);
#pragma unroll
            for (int e = 0; e < 4; ++e)
                if (i + e < hi && pred(v[e])) out(slot++, v[e]);
        }
    }
    __syncthreads();
    return base + total;
}

}  // namespace dsa
