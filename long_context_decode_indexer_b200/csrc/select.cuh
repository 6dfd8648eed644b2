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

// Warp-aggregated histogram increment (lanes with the same bin add once).
__device__ __forceinline__ void hist_add(uint32_t *hist, bool active, uint32_t bin) {
    const unsigned m = __ballot_sync(0xffffffffu, active);
    if (active) {
        const unsigned peers = __match_any_sync(m, bin);
        if ((threadIdx.x & 31) == static_cast<unsigned>(__ffs(peers) - 1))
            atomicAdd(&hist[bin], static_cast<uint32_t>(__popc(peers)));
    }
}

// Scanning `hist` (nbins bins) from the highest bin down, find the bin where
// the running count first reaches `need` (1 <= need <= total).  Writes
// res[0] = bin, res[1] = count in higher bins, res[2] = count in the bin.
// Block-wide: every thread must call it; ends with __syncthreads().
__device__ void find_digit(const uint32_t *hist, int nbins, uint32_t need, SelectScratch &sc) {
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, nwarps = blockDim.x >> 5;
    const int nch = nbins >> 5;
    for (int c = warp; c < nch; c += nwarps) {
        uint32_t x = warp_sum(hist[c * 32 + lane]);
        if (lane == 0) sc.csum[c] = x;
    }
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
// `src(i, v)` returns true and sets v for a present element i in [0, n).
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
        for (int i0 = 0; i0 < n; i0 += nt) {
            const int i = i0 + tid;
            bool act = false;
            uint32_t d = 0;
            uint64_t v;
            if (i < n && src(i, v)) {
                if (pass == 0 || (v >> hi) == prefix) {
                    act = true;
                    d = static_cast<uint32_t>(v >> shift) & static_cast<uint32_t>(nbins - 1);
                }
            }
            hist_add(hist, act, d);
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
// increasing i.  Each thread owns 8 consecutive elements per round (fetched
// with src.get8(i0, v[8]), i0 a multiple of 8; entries past n are ignored);
// a block scan of the per-thread counts gives every thread its first slot.
// Returns the next free slot.  `wsum` is shared scratch of 32 words.
template <class Src, class Pred, class Out>
__device__ uint32_t emit_ordered(const Src &src, int n, const Pred &pred, const Out &out,
                                 uint32_t base, uint32_t *wsum) {
    constexpr int kPer = 8;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, nw = blockDim.x >> 5;
    const int round = blockDim.x * kPer;
    for (int r0 = 0; r0 < n; r0 += round) {
        uint64_t vals[kPer];
        uint32_t mask = 0;
        const int i0 = r0 + tid * kPer;
        if (i0 < n) src.get8(i0, vals);
#pragma unroll
        for (int e = 0; e < kPer; ++e)
            if (i0 + e < n && pred(vals[e])) mask |= 1u << e;
        const uint32_t cnt = static_cast<uint32_t>(__popc(mask));
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
#pragma unroll
        for (int e = 0; e < kPer; ++e)
            if ((mask >> e) & 1u) out(slot++, vals[e]);
        base += total;
        __syncthreads();
    }
    return base;
}

// Block-wide compaction: every element with pred(i, v) true is handed to
// out(slot, v) with a unique slot from counter[which] (order unspecified).
template <class Src, class Pred, class Out>
__device__ void emit_selected(const Src &src, int n, const Pred &pred, const Out &out,
                              SelectScratch &sc, int which) {
    const int tid = threadIdx.x, nt = blockDim.x, lane = tid & 31;
    for (int i0 = 0; i0 < n; i0 += nt) {
        const int i = i0 + tid;
        uint64_t v = 0;
        bool sel = (i < n) && src(i, v) && pred(v);
        const unsigned m = __ballot_sync(0xffffffffu, sel);
        if (m) {
            uint32_t base = 0;
            if (lane == 0) base = atomicAdd(&sc.counter[which], static_cast<uint32_t>(__popc(m)));
            base = __shfl_sync(0xffffffffu, base, 0);
            if (sel) out(base + __popc(m & ((1u << lane) - 1u)), v);
        }
    }
}

}  // namespace dsa
