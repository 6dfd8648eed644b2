// indexer.cu -- lightning indexer and TopK on sm_100a.
//
// Index score (DSA blog by marsggbo, section 3; FP8 kernel comment in
// "DeepSeekV3.2之DSA" by yuyanqi, section 4.3):
//   I[t,s] = k_s[s] * sum_j w[t,j] * ReLU(q^I[t,j] . k^I[s])
// TopK with the short-history rule (marsggbo section 3; yuyanqi sections
// 3.3, 4.4, 4.5): the min(k, n) largest positions, ties toward the lower one.
//
// Work split.  Queries come in groups of up to `qg` that read the same
// sequence; a group's history [0, span) is cut into P chunks, one CTA each.
// A CTA streams its chunk of the FP8 index-K cache through a TMA ring, and
// the tensor cores compute D[128 positions x qg*hp heads] = K_tile . Q^T
// (tcgen05 kind::f8f6f4, M = 128, N = qg*hp, K = d_I) into a ring of two or
// four TMEM accumulators.  Two groups of four epilogue warps (even and odd
// tiles) read D back (one TMEM lane = one position per thread) and apply
// ReLU, * w, the head sum and * k_s.  With four accumulators the tensor cores
// run two tiles ahead of each group, so the round trip epilogue -> MMA issue
// -> MMA completion no longer paces the stream.
//
// Fused mode keeps the chunk's scores in shared memory as order-preserving
// keys; scores never leave the SM.  With one chunk per group the CTA selects
// directly.  With several chunks, each adds the histogram of its keys' top
// 11 bits to the query's global histogram G.  Then:
//
// Parallel (every CTA of the launch is resident at once, the usual decode
// case): each chunk waits (bounded) until every chunk has added its
// histogram, so its snapshot of G is final and gives the threshold bin d*
// and the number of keys above it.  Each chunk publishes its keys of bin d*
// (at most the `need` largest) and its count of keys above d*; after a
// second bounded wait for every chunk's list, each chunk finds the exact
// threshold among the bin-d* lists itself, derives every chunk's selected
// count (hence its own offset in the ascending output) and writes its own
// selected positions.  No CTA waits for another to finish its chunk.
//
// Otherwise (more CTAs than can be resident):
//   1. any snapshot of G is a lower bound of the final one bin by bin, so
//      the bin where G's count from the top reaches k is at most the final
//      threshold bin -- keys in lower bins can never win;
//   2. each chunk publishes its keys at or above that bin (capped by an
//      exact local TopK of size k), then bumps the group's done counter;
//   3. the last CTA of the group takes everything above the final threshold
//      bin and radix-refines the threshold bin among the candidates.
#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "kernels.h"
#include "ptx.cuh"
#include "select.cuh"

namespace dsa {

namespace {

constexpr int kTileRows = 128;  // positions per ring stage, MMA (M) and epilogue tile

struct K1Smem {
    uint64_t full[kK1MaxStages];
    uint64_t empty[kK1MaxStages];        // also the epilogue's "accumulator ready": one commit per tile
    uint64_t acc_empty[kK1MaxAcc];
    uint32_t tmem_base;
    volatile int32_t abort;
    int32_t is_last;
    int32_t n_q[kMaxGroupQueries];
    uint32_t g_digit[kMaxGroupQueries];  // final threshold bin (when the snapshot was complete)
    uint32_t g_above[kMaxGroupQueries];  // positions in higher bins
    int32_t g_complete[kMaxGroupQueries];
    uint32_t g_seen;                     // positions counted into G before the snapshot
    int32_t cand_off[kMaxChunks + 1];    // merge: prefix of the chunks' (padded) candidate counts
    int32_t cand_n[kMaxChunks];
    int32_t cand_above[kMaxChunks];      // parallel: keys of each chunk above the threshold bin
    int32_t sel_cnt[kMaxChunks];         // parallel: positions each chunk selects
    int32_t sel_ok;                      // parallel: the bounded waits succeeded
    int32_t chunk_c, chunk_P;            // this CTA's chunk and its group's chunk count
    unsigned long long t_exact;          // parallel: the need-th largest listed composite
    uint64_t merge_bar;                  // merge: bulk copies of the candidate lists
    uint32_t merge_phase;
    uint64_t mma_done[2];                // every MMA issued by MMA thread i has completed
    SelectScratch sel;
};

static_assert(sizeof(K1Smem) <= kK1MiscBytes, "K1Smem must fit the misc area of k1_layout");

__device__ __forceinline__ uint8_t *align1024(uint8_t *p) {
    return reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}

// first query and query count of group g
__device__ __forceinline__ void group_queries(const K1Params &a, int g, int &q0, int &cnt) {
    const int blk = g / a.groups_per_block, sub = g % a.groups_per_block;
    q0 = blk * a.q_per_seq + sub * a.qg;
    int c = a.qg;
    c = min(c, a.q_per_seq - sub * a.qg);
    c = min(c, a.nq - q0);
    cnt = max(c, 0);
}

// Key of position p's score in the local chunk buffer -> composite.
// (the key buffer is padded to a multiple of 128 entries)
struct LocalSrc {
    const uint32_t *keys;
    int base;
    __device__ void load4(int i, uint64_t (&v)[4]) const {
        const uint4 k = *reinterpret_cast<const uint4 *>(keys + i);
        const uint32_t p = static_cast<uint32_t>(base + i);
        v[0] = make_composite(k.x, p);
        v[1] = make_composite(k.y, p + 1);
        v[2] = make_composite(k.z, p + 2);
        v[3] = make_composite(k.w, p + 3);
    }
};
// Candidates staged in shared memory (already composites; the staging area
// has room past the last entry).
struct ListSrc {
    const uint64_t *list;
    __device__ void load4(int i, uint64_t (&v)[4]) const {
        const uint4 a = *reinterpret_cast<const uint4 *>(list + i);
        const uint4 b = *reinterpret_cast<const uint4 *>(list + i + 2);
        v[0] = (static_cast<uint64_t>(a.y) << 32) | a.x;
        v[1] = (static_cast<uint64_t>(a.w) << 32) | a.z;
        v[2] = (static_cast<uint64_t>(b.y) << 32) | b.x;
        v[3] = (static_cast<uint64_t>(b.w) << 32) | b.z;
    }
};

// The chunks' candidate lists read in place from global memory (L2), as one
// list whose chunk segments start at the virtual offsets off[c] (each a
// multiple of 4; the entries past a chunk's count are zero composites).
struct GlobalSegSrc {
    const uint64_t *cand;  // [P, stride]
    int stride, P;
    const int32_t *off;    // shared: P + 1 virtual offsets
    __device__ void load4(int i, uint64_t (&v)[4]) const {
        int c = 0;
        while (c + 1 < P && off[c + 1] <= i) ++c;
        const uint64_t *p = cand + static_cast<int64_t>(c) * stride + (i - off[c]);
        const uint4 a = __ldcg(reinterpret_cast<const uint4 *>(p));
        const uint4 b = __ldcg(reinterpret_cast<const uint4 *>(p + 2));
        v[0] = (static_cast<uint64_t>(a.y) << 32) | a.x;
        v[1] = (static_cast<uint64_t>(a.w) << 32) | a.z;
        v[2] = (static_cast<uint64_t>(b.y) << 32) | b.x;
        v[3] = (static_cast<uint64_t>(b.w) << 32) | b.z;
    }
};

// Copy a query's global histogram (2048 words, L2) to shared memory.  All
// of a thread's loads are issued before any store, so the copy costs one L2
// round trip instead of one per loop iteration.  Needs blockDim >= 256.
__device__ __forceinline__ void load_global_hist(uint32_t *dst, const uint32_t *G) {
    constexpr int kVec = kSelBins / 4;  // 512 uint4
    const uint4 *src = reinterpret_cast<const uint4 *>(G);
    const int i0 = threadIdx.x, i1 = threadIdx.x + blockDim.x;
    const uint4 zero = make_uint4(0, 0, 0, 0);
    const uint4 v0 = i0 < kVec ? __ldcg(src + i0) : zero;
    const uint4 v1 = i1 < kVec ? __ldcg(src + i1) : zero;
    if (i0 < kVec) reinterpret_cast<uint4 *>(dst)[i0] = v0;
    if (i1 < kVec) reinterpret_cast<uint4 *>(dst)[i1] = v1;
}

// Sum of hist[b] for b >= lo (block-wide; every thread gets the result).
__device__ uint32_t hist_sum_from(const uint32_t *hist, uint32_t lo, SelectScratch &sc) {
    if (threadIdx.x == 0) sc.counter[2] = 0;
    __syncthreads();
    uint32_t c = 0;
    for (int b = threadIdx.x; b < kSelBins; b += blockDim.x) c += (static_cast<uint32_t>(b) >= lo) ? hist[b] : 0u;
    c = warp_sum(c);
    if ((threadIdx.x & 31) == 0) atomicAdd(&sc.counter[2], c);
    __syncthreads();
    const uint32_t r = sc.counter[2];
    __syncthreads();
    return r;
}

// The chunk's candidates: 16-bit offsets into its keys (position - start), in
// position order, read as composites four at a time (the list is padded with
// offset 0 to the next multiple of 4).
struct CandSrc {
    const uint16_t *off;
    const uint32_t *keys;
    int base;
    __device__ void load4(int i, uint64_t (&v)[4]) const {
        const uint2 o = *reinterpret_cast<const uint2 *>(off + i);
        const uint32_t o0 = o.x & 0xFFFFu, o1 = o.x >> 16, o2 = o.y & 0xFFFFu, o3 = o.y >> 16;
        v[0] = make_composite(keys[o0], static_cast<uint32_t>(base) + o0);
        v[1] = make_composite(keys[o1], static_cast<uint32_t>(base) + o1);
        v[2] = make_composite(keys[o2], static_cast<uint32_t>(base) + o2);
        v[3] = make_composite(keys[o3], static_cast<uint32_t>(base) + o3);
    }
};

constexpr int kSlotLog2 = 9;  // parallel selection: staged entries per chunk list, at most 2^9

// The chunks' lists staged in slots of 2^slot_log2 entries (slot c holds
// chunk c's first n[c] entries; the rest of a slot reads as zero composites).
struct SlotSrc {
    const uint64_t *list;
    const int32_t *n;
    int slot_log2;
    __device__ void load4(int i, uint64_t (&v)[4]) const {
        const uint4 a = *reinterpret_cast<const uint4 *>(list + i);
        const uint4 b = *reinterpret_cast<const uint4 *>(list + i + 2);
        const int m = n[i >> slot_log2];
        const int j = i & ((1 << slot_log2) - 1);
        v[0] = j < m ? (static_cast<uint64_t>(a.y) << 32) | a.x : 0ull;
        v[1] = j + 1 < m ? (static_cast<uint64_t>(a.w) << 32) | a.z : 0ull;
        v[2] = j + 2 < m ? (static_cast<uint64_t>(b.y) << 32) | b.x : 0ull;
        v[3] = j + 3 < m ? (static_cast<uint64_t>(b.w) << 32) | b.z : 0ull;
    }
};

// Parallel exact selection of query q by chunk c = blockIdx.x % P, once the
// snapshot of G taken in chunk_select is final (every chunk's histogram in
// it): d* is the threshold bin, `above` the query's keys in higher bins,
// need = K - above the keys to take from bin d*.
//   1. one pass over the chunk's keys lists its candidates C (keys of bin d*
//      or above) in position order;
//   2. publish C's keys of bin d* (its `need` largest at most: a key beaten
//      by `need` keys of the bin in its own chunk never wins) and the
//      chunk's count of keys above d*; bump the query's `published` counter;
//   3. wait (bounded) until every chunk has published; one round trip
//      brings every chunk's list (its first 2^kSlotLog2 entries) and counts on
//      chip; the exact threshold Te is the need-th largest listed composite
//      (read in place from L2 when a list is longer than that);
//   4. every chunk's selected count is its keys above d* plus its listed
//      keys >= Te; the chunks before this one give its offset, and it writes
//      its candidates >= Te there, in ascending position order.
// `list` / `list_cap`: shared memory below the chunk's keys (the TMA ring and
// the q tile, free once streaming is over), in composites: the staged lists
// at its start, C (16-bit) at its end.
__device__ void parallel_select(const K1Params &a, K1Smem &sm, int q, int qi, const uint32_t *keys,
                                int start, int len, const uint32_t *lhist, uint32_t *scratch,
                                uint64_t *list, int list_cap) {
    const int K = a.topk, P = sm.chunk_P, c = sm.chunk_c;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, nwarps = blockDim.x >> 5;
    const bool complete = sm.sel_ok && sm.g_complete[qi];
    const uint32_t d = sm.g_digit[qi];
    const uint32_t need = static_cast<uint32_t>(K) - sm.g_above[qi];
    uint64_t *cand = a.cand + (static_cast<int64_t>(q) * a.P + c) * a.cand_stride;
    const int c_cap = (len + 4 + 7) & ~7;  // 16-bit entries, room for the padding
    uint16_t *cands = reinterpret_cast<uint16_t *>(reinterpret_cast<uint8_t *>(list) +
                                                   static_cast<size_t>(list_cap) * 8 - static_cast<size_t>(c_cap) * 2);
    // slots of a power of two entries (at most 2^kSlotLog2, and the cand stride)
    int slot_log2 = kSlotLog2;
    while (slot_log2 >= 2 && ((1 << slot_log2) * P > list_cap - c_cap / 4 || (1 << slot_log2) > a.cand_stride))
        --slot_log2;
    const int stage_cap = slot_log2 >= 2 ? (1 << slot_log2) : 0;  // 0: no room, the lists are read in place
    CandSrc csrc{cands, keys, start};
    int32_t m = 0, above_c = 0;
    uint32_t nC = 0;
    if (complete) {
        above_c = static_cast<int32_t>(hist_sum_from(lhist, d + 1, sm.sel));
        const uint32_t bucket_c = lhist[d];
        nC = compact_ordered(
            LocalSrc{keys, start}, len, [d](uint64_t v) { return static_cast<uint32_t>(v >> 53) >= d; },
            [cands, start](uint32_t slot, uint64_t v) {
                cands[slot] = static_cast<uint16_t>(composite_pos(v) - static_cast<uint32_t>(start));
            },
            0u, sm.sel.wsum);
        if (tid < 4) cands[nC + tid] = 0;
        __syncthreads();
        uint64_t thr = static_cast<uint64_t>(d) << 53;
        if (bucket_c > need) thr = radix_refine(csrc, static_cast<int>(nC), d, 1, need, scratch, sm.sel);
        m = static_cast<int32_t>(compact_ordered(
            csrc, static_cast<int>(nC), [thr, d](uint64_t v) { return (v >> 53) == d && v >= thr; },
            [cand, K](uint32_t slot, uint64_t v) {
                if (slot < static_cast<uint32_t>(K)) cand[slot] = v;
            },
            0u, sm.sel.wsum));
        if (m > K) m = K;  // cannot happen: at most `need` <= K keys pass
    }
    // zero composites pad the list to a multiple of 4 (below every key)
    if (tid < 4 && m + tid < ((m + 3) & ~3)) cand[m + tid] = 0ull;
    if (tid == 0) {
        a.cand_cnt[static_cast<int64_t>(q) * a.P + c] = m;
        a.cand_above[static_cast<int64_t>(q) * a.P + c] = above_c;
    }
    __threadfence();
    __syncthreads();
    if (tid == 0) {
        atomicAdd(&a.published[q], 1u);
        sm.sel_ok = complete && wait_count(&a.published[q], static_cast<uint32_t>(P), a.wait_budget);
        if (!sm.sel_ok) record_status(a.status, DSA_ERR_TIMEOUT);
    }
    __syncthreads();
    if (!sm.sel_ok) return;
    // one round trip: each chunk's list into its slot of stage_cap entries,
    // the counts and above-counts alongside
    const uint64_t *cand_q = a.cand + static_cast<int64_t>(q) * a.P * a.cand_stride;
    if (tid == 0) mbar_arrive_expect_tx(&sm.merge_bar, static_cast<uint32_t>(P * stage_cap) * 8u);
    if (tid < P && stage_cap > 0) {
        fence_proxy_async_global();
        bulk_load(list + tid * stage_cap, cand_q + static_cast<int64_t>(tid) * a.cand_stride,
                  static_cast<uint32_t>(stage_cap) * 8u, &sm.merge_bar);
    }
    if (warp == 1) {
        const int32_t *cnt = a.cand_cnt + static_cast<int64_t>(q) * a.P;
        const int32_t *abv = a.cand_above + static_cast<int64_t>(q) * a.P;
        const int m_l = lane < P ? min(__ldcg(&cnt[lane]), K) : 0;
        const int padded = (m_l + 3) & ~3;
        const int incl = static_cast<int>(warp_incl_scan(static_cast<uint32_t>(padded)));
        if (lane < P) {
            sm.cand_off[lane] = incl - padded;  // virtual offsets of the lists read in place
            sm.cand_n[lane] = m_l;
            sm.cand_above[lane] = __ldcg(&abv[lane]);
        }
        const int tot = __shfl_sync(0xffffffffu, incl, 31);
        const uint32_t listed = warp_sum(static_cast<uint32_t>(m_l));
        const bool fits = stage_cap > 0 && __all_sync(0xffffffffu, m_l <= stage_cap);
        if (lane == 0) {
            sm.cand_off[P] = tot;
            sm.sel.res[3] = listed;
            sm.sel.res[2] = fits ? 1u : 0u;
        }
    }
    const bool landed = __syncthreads_and(mbar_wait(&sm.merge_bar, sm.merge_phase, a.wait_budget));
    if (tid == 0) sm.merge_phase ^= 1u;
    if (!landed) {
        if (tid == 0) record_status(a.status, DSA_ERR_TIMEOUT);
        return;
    }
    const bool staged = sm.sel.res[2] != 0;
    const uint32_t listed = sm.sel.res[3];
    // the threshold: the need-th largest listed composite (listed >= need:
    // a chunk whose bin-d* keys exceed `need` lists `need` of them, else all).
    // radix_refine gives a bound T with exactly `need` listed composites >= T;
    // the smallest of them, Te, is the threshold itself.  Selecting own keys
    // >= Te (not >= T) matters: a chunk's unlisted bin-d* keys lie below its
    // smallest listed one, which is <= Te, but may lie above T.
    uint64_t T = static_cast<uint64_t>(d) << 53;
    if (listed != need) {
        if (staged) T = radix_refine(SlotSrc{list, sm.cand_n, slot_log2}, P * stage_cap, d, 1, need, scratch, sm.sel);
        else T = radix_refine(GlobalSegSrc{cand_q, a.cand_stride, P, sm.cand_off}, sm.cand_off[P], d, 1, need,
                              scratch, sm.sel);
    }
    if (tid == 0) sm.t_exact = ~0ull;
    __syncthreads();
    // selected count of every chunk: keys above d* + listed keys >= T
    for (int cc = warp; cc < P; cc += nwarps) {
        const int mm = sm.cand_n[cc];
        const uint64_t *seg = staged ? list + cc * stage_cap : cand_q + static_cast<int64_t>(cc) * a.cand_stride;
        uint32_t k = 0;
        unsigned long long lo = ~0ull;
        for (int j = lane; j < mm; j += 32) {
            const uint64_t v = staged ? seg[j] : __ldcg(&seg[j]);
            if (v >= T) {
                ++k;
                lo = v < lo ? v : lo;
            }
        }
        k = warp_sum(k);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            const unsigned long long y = __shfl_xor_sync(0xffffffffu, lo, o);
            lo = y < lo ? y : lo;
        }
        if (lane == 0) {
            sm.sel_cnt[cc] = sm.cand_above[cc] + static_cast<int32_t>(k);
            if (k) atomicMin(&sm.t_exact, lo);
        }
    }
    __syncthreads();
    const uint64_t Te = sm.t_exact;
    int off = 0, all = 0;
    for (int cc = 0; cc < P; ++cc) {
        off += cc < c ? sm.sel_cnt[cc] : 0;
        all += sm.sel_cnt[cc];
    }
    int32_t *out = a.idx + static_cast<int64_t>(q) * K;
    const uint32_t got = compact_ordered(
        csrc, static_cast<int>(nC), [Te](uint64_t v) { return v >= Te; },
        [out, K](uint32_t slot, uint64_t v) {
            if (slot < static_cast<uint32_t>(K)) out[slot] = static_cast<int32_t>(composite_pos(v));
        },
        static_cast<uint32_t>(off), sm.sel.wsum);
    if (tid == 0) {
        if (got != static_cast<uint32_t>(off + sm.sel_cnt[c]) || all != K)
            record_status(a.status, DSA_ERR_DEVICE_CHECK);
        if (c == 0 && a.nsel) a.nsel[q] = K;
    }
    __syncthreads();
}

// Everything one query of a chunk does after its keys are in shared memory:
// direct selection (one chunk), or publishing candidates (several chunks).
// `keys` holds the chunk's keys for positions [start, start + len) and
// `lhist` the histogram of their top digits.  Every emission is an ordered
// compaction, so results come out in ascending position order and are the
// same from run to run.
__device__ void chunk_select(const K1Params &a, K1Smem &sm, int q, int qi, int n,
                             const uint32_t *keys, int start, int len, const uint32_t *lhist,
                             uint32_t *scratch, uint64_t *list, int list_cap) {
    const int K = a.topk;
    LocalSrc src{keys, start};
    if (sm.chunk_P == 1) {
        // the whole history is here: len == n > K
        find_digit(lhist, kSelBins, static_cast<uint32_t>(K), sm.sel);
        const uint32_t d = sm.sel.res[0], above = sm.sel.res[1], bucket = sm.sel.res[2];
        __syncthreads();
        const uint32_t need = static_cast<uint32_t>(K) - above;
        uint64_t thr = static_cast<uint64_t>(d) << 53;
        if (bucket != need) thr = radix_refine(src, len, d, 1, need, scratch, sm.sel);
        int32_t *out = a.idx + static_cast<int64_t>(q) * K;
        const uint32_t cnt = emit_ordered(
            src, len, [thr](uint64_t v) { return v >= thr; },
            [out, K](uint32_t slot, uint64_t v) {
                if (slot < static_cast<uint32_t>(K)) out[slot] = static_cast<int32_t>(composite_pos(v));
            },
            0u, sm.sel.wsum, reinterpret_cast<uint4 *>(scratch));
        if (threadIdx.x == 0) {
            if (cnt != static_cast<uint32_t>(K)) record_status(a.status, DSA_ERR_DEVICE_CHECK);
            if (a.nsel) a.nsel[q] = K;
        }
        __syncthreads();
        return;
    }

    // ---- several chunks: publish this chunk's histogram, then read G back
    uint32_t *G = a.ghist + static_cast<int64_t>(q) * kSelBins;
    const int c = sm.chunk_c;
    for (int b = threadIdx.x; b < kSelBins; b += blockDim.x)
        if (lhist[b]) atomicAdd(&G[b], lhist[b]);
    __threadfence();
    __syncthreads();
    if (threadIdx.x == 0) {
        atomicAdd(&a.gtot[q], static_cast<uint32_t>(len));
        // When every chunk runs at the same time, wait (bounded) until all of
        // them have added their histograms: parallel selection needs the
        // final threshold bin; the merge only gets a tighter candidate bound
        // (any earlier snapshot is a valid, weaker one), so its wait is short
        // and running out of it is no error.  Read the count BEFORE the
        // snapshot: every chunk adds its histogram to G before its count to
        // gtot, so a count that covers all n positions here proves the
        // snapshot below complete.  (Read after the snapshot, it could cover
        // chunks the snapshot missed.)
        if (a.parallel) {
            sm.sel_ok = wait_count(&a.gtot[q], static_cast<uint32_t>(n), a.wait_budget);
        } else {
            sm.sel_ok = 1;
            if (a.wait_hist) wait_count(&a.gtot[q], static_cast<uint32_t>(n), kHistWaitCycles);
        }
        sm.g_seen = ld_acquire_u32(&a.gtot[q]);
    }
    __syncthreads();
    load_global_hist(scratch, G);
    __syncthreads();
    find_digit(scratch, kSelBins, static_cast<uint32_t>(K), sm.sel);
    const uint32_t dlow = sm.sel.res[0];
    if (threadIdx.x == 0) {
        // complete if every position of the query was counted before the snapshot
        sm.g_complete[qi] = sm.g_seen >= static_cast<uint32_t>(n) &&
                            sm.sel.res[1] + sm.sel.res[2] >= static_cast<uint32_t>(K);
        sm.g_digit[qi] = dlow;
        sm.g_above[qi] = sm.sel.res[1];
    }
    __syncthreads();
    if (a.parallel) {
        parallel_select(a, sm, q, qi, keys, start, len, lhist, scratch, list, list_cap);
        return;
    }
    uint64_t *cand = a.cand + (static_cast<int64_t>(q) * a.P + c) * a.cand_stride;
    const uint32_t at_or_above = hist_sum_from(lhist, dlow, sm.sel);
    uint64_t thr = static_cast<uint64_t>(dlow) << 53;
    if (at_or_above > static_cast<uint32_t>(K)) {
        // cap at the exact local TopK: a key beaten by k keys of its own
        // chunk can never be selected; keep the intersection of both sets
        find_digit(lhist, kSelBins, static_cast<uint32_t>(K), sm.sel);
        const uint32_t d = sm.sel.res[0], above = sm.sel.res[1], bucket = sm.sel.res[2];
        __syncthreads();
        const uint32_t need = static_cast<uint32_t>(K) - above;
        uint64_t lthr = static_cast<uint64_t>(d) << 53;
        if (bucket != need) lthr = radix_refine(src, len, d, 1, need, scratch, sm.sel);
        thr = lthr > thr ? lthr : thr;
    }
    uint32_t m = emit_ordered(
        src, len, [thr](uint64_t v) { return v >= thr; },
        [cand, K](uint32_t slot, uint64_t v) {
            if (slot < static_cast<uint32_t>(K)) cand[slot] = v;
        },
        0u, sm.sel.wsum, reinterpret_cast<uint4 *>(scratch));
    if (threadIdx.x == 0) {
        if (m > static_cast<uint32_t>(K)) {
            record_status(a.status, DSA_ERR_DEVICE_CHECK);
            m = K;
        }
        a.cand_cnt[static_cast<int64_t>(q) * a.P + c] = static_cast<int32_t>(m);
    }
    __syncthreads();
}

// The last CTA of a group: final selection of query q from all candidates.
// Chunks publish their candidates in ascending position order and chunk c
// covers positions below chunk c + 1, so staging the lists chunk by chunk
// keeps the whole candidate list in ascending position order.
__device__ void group_merge(const K1Params &a, K1Smem &sm, int q, int qi, uint32_t *hist,
                            uint64_t *list, int list_cap) {
    const int K = a.topk;
    const int P = sm.chunk_P;  // this group's chunks (the lists' layout keeps a.P slots)
    uint32_t dstar, above;
    if (sm.g_complete[qi]) {
        // this CTA's snapshot already held every chunk's histogram
        dstar = sm.g_digit[qi];
        above = sm.g_above[qi];
    } else {
        const uint32_t *G = a.ghist + static_cast<int64_t>(q) * kSelBins;
        load_global_hist(hist, G);
        __syncthreads();
        find_digit(hist, kSelBins, static_cast<uint32_t>(K), sm.sel);
        dstar = sm.sel.res[0];
        above = sm.sel.res[1];
        __syncthreads();
    }
    // stage all candidates (ordered) in shared memory: one bulk copy per
    // chunk list, each padded to an even length (16-byte units); the pad
    // entries are set to 0, a composite no valid score reaches
    const uint64_t *cand = a.cand + static_cast<int64_t>(q) * a.P * a.cand_stride;
    const int32_t *cnt = a.cand_cnt + static_cast<int64_t>(q) * a.P;
    if (threadIdx.x < 32) {
        // one lane per chunk (P <= 32): the counts are loaded in parallel,
        // the offsets are a warp scan of the padded counts
        const int c = threadIdx.x;
        const int m = c < P ? min(__ldcg(&cnt[c]), K) : 0;
        const int padded = (m + 1) & ~1;
        const int incl = static_cast<int>(warp_incl_scan(static_cast<uint32_t>(padded)));
        if (c < P) {
            sm.cand_off[c] = incl - padded;
            sm.cand_n[c] = m;
        }
        const int off = __shfl_sync(0xffffffffu, incl, 31);
        if (c == 0) {
            sm.cand_off[P] = off;
            if (off <= list_cap) mbar_arrive_expect_tx(&sm.merge_bar, static_cast<uint32_t>(off) * 8u);
        }
    }
    __syncthreads();
    const int total = sm.cand_off[P];
    if (total > list_cap) {
        if (threadIdx.x == 0) record_status(a.status, DSA_ERR_DEVICE_CHECK);
        __syncthreads();
        return;
    }
    if (threadIdx.x < P) {
        const int c = threadIdx.x, m = sm.cand_n[c];
        if (m > 0)
            bulk_load(list + sm.cand_off[c], cand + static_cast<int64_t>(c) * a.cand_stride,
                      static_cast<uint32_t>((m + 1) & ~1) * 8u, &sm.merge_bar);
    }
    const bool staged = __syncthreads_and(mbar_wait(&sm.merge_bar, sm.merge_phase, a.wait_budget));
    if (threadIdx.x < P && (sm.cand_n[threadIdx.x] & 1)) list[sm.cand_off[threadIdx.x] + sm.cand_n[threadIdx.x]] = 0ull;
    if (threadIdx.x == 0) sm.merge_phase ^= 1u;
    __syncthreads();
    if (!staged) {
        if (threadIdx.x == 0) record_status(a.status, DSA_ERR_TIMEOUT);
        __syncthreads();
        return;
    }
    // the need-th largest candidate of bucket d* is the threshold (if the
    // candidates held fewer than `need` of the bucket, the emission count
    // below comes out short and flags it)
    const uint32_t need = static_cast<uint32_t>(K) - above;
    int32_t *out = a.idx + static_cast<int64_t>(q) * K;
    ListSrc src{list};
    const uint64_t thr = radix_refine(src, total, dstar, 1, need, hist, sm.sel);
    const uint32_t got = emit_ordered(
        src, total, [thr](uint64_t v) { return v >= thr; },
        [out, K](uint32_t slot, uint64_t v) {
            if (slot < static_cast<uint32_t>(K)) out[slot] = static_cast<int32_t>(composite_pos(v));
        },
        0u, sm.sel.wsum, reinterpret_cast<uint4 *>(hist));
    if (threadIdx.x == 0) {
        if (got != static_cast<uint32_t>(K)) record_status(a.status, DSA_ERR_DEVICE_CHECK);
        if (a.nsel) a.nsel[q] = K;
    }
    __syncthreads();
}

// Queries whose history fits in k keep every position (no scoring).
__device__ void write_fallback(const K1Params &a, int q, int n) {
    const int K = a.topk;
    int32_t *out = a.idx + static_cast<int64_t>(q) * K;
    for (int i = threadIdx.x; i < K; i += blockDim.x) out[i] = i < n ? i : -1;
    if (threadIdx.x == 0 && a.nsel) a.nsel[q] = n;
}

// After all chunks of a group published: is this CTA the last one?
__device__ bool arrive_group(const K1Params &a, K1Smem &sm, int g) {
    __threadfence();
    __syncthreads();
    if (threadIdx.x == 0) {
        const uint32_t prev = atomicAdd(&a.done[g], 1u);
        sm.is_last = (prev == static_cast<uint32_t>(sm.chunk_P - 1));
    }
    __syncthreads();
    if (sm.is_last) __threadfence();
    return sm.is_last != 0;
}

}  // namespace

// ---------------------------------------------------------------------------
// K1: streaming indexer.  MODE_FUSED (scores stay on chip, TopK written) or
// MODE_SCORES (scores written to HBM).
// ---------------------------------------------------------------------------
template <int MODE, int HP, int DI>
__global__ void __launch_bounds__(kK1Threads, 1)
    k1_indexer(const __grid_constant__ CUtensorMap kmap, const K1Params a) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *base = align1024(smem_raw);
    const K1Layout L = k1_layout(MODE, DI, a.qg, HP, a.chunk, a.P, a.topk, a.stages, !a.parallel);
    uint8_t *stages = base + L.stages;
    uint8_t *qtile = base + L.qtile;
    uint32_t *keys = reinterpret_cast<uint32_t *>(base + L.keys);
    uint32_t *hist = reinterpret_cast<uint32_t *>(base + L.hist);  // radix scratch
    uint32_t *lhist = hist + kSelBins;                                  // [qg][2048]
    float *wts = reinterpret_cast<float *>(base + L.wts);
    K1Smem &sm = *reinterpret_cast<K1Smem *>(base + L.misc);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    // group and chunk of this CTA: groups [0, n_big) have P chunks, the rest
    // P - 1 (a batch then fills every SM); each group cuts its own span
    int g, c, Pg;
    {
        const int b = blockIdx.x, big = a.n_big * a.P;
        if (b < big) {
            g = b / a.P;
            c = b % a.P;
            Pg = a.P;
        } else {
            const int r = b - big;
            g = a.n_big + r / (a.P - 1);
            c = r % (a.P - 1);
            Pg = a.P - 1;
        }
    }
    int q0, nqg;
    group_queries(a, g, q0, nqg);
    constexpr int kTileBytes = kTileRows * DI;
    const int N = a.qg * HP;  // MMA N (columns per accumulator buffer)

    // ---- set-up
    // The q^I tile and the weights are loaded first, into registers: issued
    // before the TMA ring fills, they do not queue behind it.
    constexpr int kQPieces = (kMaxGroupQueries * HP * (DI / 16) + kK1Threads - 1) / kK1Threads;
    static_assert(kMaxGroupQueries * HP <= kK1Threads, "one weight per thread");
    uint4 qv[kQPieces];
#pragma unroll
    for (int u = 0; u < kQPieces; ++u) {
        const int i = tid + u * kK1Threads;
        const int r = i / (DI / 16), ch = i % (DI / 16);
        const int qi = r / HP, j = r % HP;
        qv[u] = make_uint4(0, 0, 0, 0);
        if (r < N && qi < nqg && j < a.h_idx)
            qv[u] = *reinterpret_cast<const uint4 *>(a.q_idx + (static_cast<int64_t>(q0 + qi) * a.h_idx + j) * DI + ch * 16);
    }
    float wv = 0.f;
    if (tid < N) {
        const int qi = tid / HP, j = tid % HP;
        if (qi < nqg && j < a.h_idx) wv = bf16_bits_to_float(a.w[static_cast<int64_t>(q0 + qi) * a.h_idx + j]);
    }

    // ---- span of positions this CTA covers (every thread, from global q_n)
    int nmax = 0, nscored = 0;
    for (int i = 0; i < nqg; ++i) {
        const int n_i = a.q_n[q0 + i];
        nmax = max(nmax, n_i);
        if (MODE == kModeScores || n_i > a.topk) nscored = max(nscored, n_i);
    }
    const int seq = nqg > 0 ? a.q_seq[q0] : 0;
    const int span = (MODE == kModeScores) ? static_cast<int>(a.ld) : nscored;
    // With the merge selection a group uses only the chunks its own span
    // needs (a.chunk positions at most, the plan's size for the longest
    // span): the launch has a.P per group, and a batch of short and long
    // histories would otherwise pay a.P chunks' fixed costs (set-up,
    // histogram exchange, arrival) for every short one.  The CTAs past a
    // group's count leave before touching anything shared.
    if (MODE == kModeFused && !a.parallel) {
        const int need = max(1, (span + a.chunk - 1) / a.chunk);
        if (need < Pg) Pg = need;
        if (c >= Pg) return;
    }
    const int chunk = min(a.chunk, ((span + Pg - 1) / Pg + kTileRows - 1) / kTileRows * kTileRows);
    const int start = c * chunk;
    const int end = min(start + chunk, span);
    const int len = max(end - start, 0);
    const int ntiles = (len + kTileRows - 1) / kTileRows;

    // The producer (thread 0) fills the TMA ring as soon as its barriers
    // exist, so the first tiles are in flight during the rest of the set-up.
    const int64_t row0 = (a.page_table == nullptr && nqg > 0) ? a.seq_row0[seq] : 0;
    // tests only: the first CTA never loads its first tile, so the MMA
    // issuer's wait for it runs out
    const bool skip_first = a.inject != 0 && blockIdx.x == 0;
    // tile t: one 128-row box (contiguous cache; a box past the end of the
    // cache reads zeros), or one box per page
    // k^I is read once per call: its lines go first when L2 needs room
    const uint64_t stream_policy = l2_policy_evict_first();
    auto issue_tile = [&](int t, int s) {
        if (skip_first && t == 0) return;
        const int p0 = start + t * kTileRows;
        uint8_t *dst = stages + s * kTileBytes;
        if (a.page_table == nullptr) {
            mbar_arrive_expect_tx(&sm.full[s], kTileBytes);
            tma_load_2d_hint(dst, &kmap, &sm.full[s], 0, static_cast<int32_t>(row0 + p0), stream_policy);
        } else {
            const int box = a.page_size;
            const int32_t *pt = a.page_table + static_cast<int64_t>(seq) * a.max_pages + p0 / box;
            int n_box = 0;
            for (int h = 0; h < kTileRows / box; ++h) n_box += (p0 + h * box < nmax);
            mbar_arrive_expect_tx(&sm.full[s], static_cast<uint32_t>(n_box * box * DI));
            for (int h = 0; h < n_box; ++h, dst += box * DI)
                tma_load_2d_hint(dst, &kmap, &sm.full[s], 0, pt[h] * box, stream_policy);
        }
    };
    const int n_pro = min(ntiles, a.stages);  // tiles issued before the set-up barrier

    if (tid == 0) {
        sm.abort = 0;
        sm.is_last = 0;
        for (int i = 0; i < kMaxGroupQueries; ++i) sm.g_complete[i] = 0;
        mbar_init(&sm.merge_bar, 1);
        mbar_init(&sm.mma_done[0], 1);
        mbar_init(&sm.mma_done[1], 1);
        sm.merge_phase = 0;
        for (int s = 0; s < a.stages; ++s) {
            mbar_init(&sm.full[s], 1);
            mbar_init(&sm.empty[s], 1);
        }
        for (int b = 0; b < a.acc_bufs; ++b) {
            mbar_init(&sm.acc_empty[b], 4);  // the four warps of epilogue group b % 2
        }
        fence_mbar_init();
        for (int t = 0; t < n_pro; ++t) issue_tile(t, t);
        sm.chunk_c = c;
        sm.chunk_P = Pg;
    }
    if (tid < kMaxGroupQueries) sm.n_q[tid] = tid < nqg ? a.q_n[q0 + tid] : 0;
    // q^I tile (B operand, K-major, swizzled like the TMA tiles) and weights
#pragma unroll
    for (int u = 0; u < kQPieces; ++u) {
        const int i = tid + u * kK1Threads;
        const int r = i / (DI / 16), ch = i % (DI / 16);
        const int sw = (DI == 128) ? (ch ^ (r & 7)) : (ch ^ ((r >> 1) & 3));
        if (r < N) *reinterpret_cast<uint4 *>(qtile + r * DI + sw * 16) = qv[u];
    }
    if (tid < N) wts[tid] = wv;
    if (MODE == kModeFused)
        for (int i = tid; i < a.qg * kSelBins; i += blockDim.x) lhist[i] = 0;
    if (warp == 1) {
        tmem_alloc(&sm.tmem_base, a.tmem_cols);
        tmem_relinquish();
    }
    fence_proxy_async_smem();  // q tile written by threads, read by the tensor cores
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = sm.tmem_base;

    // a query group must read one sequence
    if (tid < nqg && a.q_seq[q0 + tid] != seq) record_status(a.status, DSA_ERR_DEVICE_CHECK);

    if (MODE == kModeFused && c == 0)
        for (int i = 0; i < nqg; ++i)
            if (sm.n_q[i] <= a.topk) write_fallback(a, q0 + i, sm.n_q[i]);

    // ---- streaming pipeline
    if (ntiles > 0) {
        if (warp == 0) {
            if (lane == 0) {
                // ring position (s, ph) advances by one per tile: no divisions
                // in this single-thread loop, which paces the whole stream
                int s = n_pro == a.stages ? 0 : n_pro;
                uint32_t ph = n_pro == a.stages ? 1u : 0u;
                int t_end = n_pro;  // tiles issued (or skipped) so far
                for (int t = n_pro; t < ntiles; ++t) {
                    if (!mbar_wait(&sm.empty[s], ph ^ 1, a.wait_budget) || sm.abort) {
                        record_status(a.status, DSA_ERR_TIMEOUT);
                        sm.abort = 1;
                        break;
                    }
                    issue_tile(t, s);
                    t_end = t + 1;
                    if (++s == a.stages) { s = 0; ph ^= 1; }
                }
                // before the CTA may exit, every load issued must have landed:
                // wait (bounded) for the newest phase of each stage (a no-op
                // when the MMA consumed them all)
                for (int t = max(t_end - a.stages, 0); t < t_end; ++t)
                    if (!(skip_first && t == 0) &&
                        !mbar_wait(&sm.full[t % a.stages], static_cast<uint32_t>(t / a.stages) & 1u, a.wait_budget))
                        record_status(a.status, DSA_ERR_TIMEOUT);
            }
        } else if (warp == 1 || warp == 10) {
            // two MMA threads: warp 1 issues the even tiles, warp 10 the odd
            // ones (each tcgen05 instruction holds its issuing thread for
            // tens of cycles; one thread issuing every tile paced the
            // stream).  One commit per tile: empty[s] frees the ring stage
            // and tells the epilogue that buffer b holds tile t.
            if (lane == 0) {
                const int r0 = warp == 1 ? 0 : 1;
                const uint32_t idesc = make_idesc(0, 0, 0, 0, kTileRows, N);
                constexpr uint32_t kSbo = 8 * DI;
                constexpr uint32_t kLayout = (DI == 128) ? kSwizzle128B : kSwizzle64B;
                // descriptors of stage 0 and of the q tile; a stage (or a 32-byte
                // K step) is a fixed offset in the 16-byte address field
                const uint64_t ad0 = make_sdesc(smem_u32(stages), 16, kSbo, kLayout);
                const uint64_t bd0 = make_sdesc(smem_u32(qtile), 16, kSbo, kLayout);
                // ring stage and accumulator of tile t = r0, r0 + 2, ...: both
                // advance by two per tile (a.stages even, a.acc_bufs even).
                // The parity waits below cannot alias an older phase because
                // tiles t - a.acc_bufs and t - a.stages (same parity) went
                // through this same thread first: a third issuer breaks that
                // (tried: it let a tile into a buffer still in use).
                int s = r0, b = r0;
                uint32_t ph = 0, aph = 0;
                for (int t = r0; t < ntiles; t += 2) {
                    if (!mbar_wait(&sm.acc_empty[b], aph ^ 1, a.wait_budget) ||
                        !mbar_wait(&sm.full[s], ph, a.wait_budget) || sm.abort) {
                        record_status(a.status, DSA_ERR_TIMEOUT);
                        sm.abort = 1;
                        // the MMAs already issued complete before TMEM is
                        // freed (on success the epilogue waits for each)
                        tc_commit(&sm.mma_done[r0]);
                        if (!mbar_wait(&sm.mma_done[r0], 0, a.wait_budget)) record_status(a.status, DSA_ERR_TIMEOUT);
                        break;
                    }
                    tc_fence_after();
                    const uint64_t ad = ad0 + static_cast<uint64_t>(s * (kTileBytes >> 4));
#pragma unroll
                    for (int kk = 0; kk < DI / 32; ++kk)
                        mma_f8_ss(tmem + b * N, ad + 2 * kk, bd0 + 2 * kk, idesc, kk > 0 ? 1u : 0u);
                    tc_commit(&sm.empty[s]);
                    s += 2;
                    if (s >= a.stages) { s -= a.stages; ph ^= 1; }
                    b += 2;
                    if (b >= a.acc_bufs) { b -= a.acc_bufs; aph ^= 1; }
                }
            }
        } else {
            // epilogue: group 0 = warps 2..5 takes even tiles (buffer 0),
            // group 1 = warps 6..9 odd tiles (buffer 1); TMEM lane quarter = warp % 4
            const int quarter = warp & 3;
            const int grp = (warp - 2) >> 2;
            const int r = quarter * 32 + lane;
            // this group's tiles t = grp, grp + 2, ... use buffers grp, grp + 2, ...
            // and ring stages grp, grp + 2, ... (whose commit marks the tile's
            // MMAs complete)
            int b = grp, se = grp;
            uint32_t eph = 0;
            for (int t = grp; t < ntiles; t += 2) {
                // lane 0 polls (eight warps polling with every lane would
                // steal issue slots from the producer and MMA threads); then
                // every lane observes the completed phase itself -- its own
                // acquire, which cannot fail: the stage's next phase is the
                // commit of tile t + a.stages, which the same MMA thread
                // issues after tile t + a.acc_bufs, whose buffer needs this
                // warp's release below.  The warp proceeds only if all lanes
                // saw it (tcgen05.ld below is warp-collective).
                const bool ok = warp_wait(&sm.empty[se], eph, &sm.abort, a.wait_budget);
                if (!ok) {
                    if (lane == 0) {
                        record_status(a.status, DSA_ERR_TIMEOUT);
                        sm.abort = 1;
                    }
                    break;
                }
                tc_fence_after();
                const int p = start + t * kTileRows + r;
                float ks = 1.f;
                if (a.k_scale && p < nmax) {
                    int64_t row;
                    if (a.page_table)
                        row = static_cast<int64_t>(a.page_table[static_cast<int64_t>(seq) * a.max_pages + p / a.page_size]) * a.page_size + p % a.page_size;
                    else
                        row = a.seq_row0[seq] + p;
                    ks = (row >= 0 && row < a.cache_rows) ? a.k_scale[row] : 0.f;
                }
                for (int qi = 0; qi < nqg; ++qi) {
                    const uint32_t taddr = tmem + (static_cast<uint32_t>(quarter * 32) << 16) +
                                           static_cast<uint32_t>(b * N + qi * HP);
                    // four running sums (heads j mod 4), kept as two pairs
                    float2 acc01 = make_float2(0.f, 0.f), acc23 = make_float2(0.f, 0.f);
                    const float4 *wq = reinterpret_cast<const float4 *>(wts + qi * HP);
                    uint32_t v[HP];
                    // issue every load of the row, then wait once
#pragma unroll
                    for (int c0 = 0; c0 < HP; c0 += 16)
                        tmem_ld16(taddr + c0, *reinterpret_cast<uint32_t(*)[16]>(&v[c0]));
                    tmem_wait_ld();
#pragma unroll
                    for (int j = 0; j < HP; j += 4) {
                        const float4 w4 = wq[j / 4];
                        acc01 = fma2(make_float2(w4.x, w4.y),
                                     make_float2(fmaxf(__uint_as_float(v[j + 0]), 0.f),
                                                 fmaxf(__uint_as_float(v[j + 1]), 0.f)),
                                     acc01);
                        acc23 = fma2(make_float2(w4.z, w4.w),
                                     make_float2(fmaxf(__uint_as_float(v[j + 2]), 0.f),
                                                 fmaxf(__uint_as_float(v[j + 3]), 0.f)),
                                     acc23);
                    }
                    const float score = ((acc01.x + acc01.y) + (acc23.x + acc23.y)) * ks;
                    if (MODE == kModeScores) {
                        if (p < end)
                            a.scores[static_cast<int64_t>(q0 + qi) * a.ld + p] =
                                p < sm.n_q[qi] ? score : -__int_as_float(0x7f800000);
                    } else {
                        const uint32_t key = float_to_key(score);
                        if (p < end) keys[qi * a.chunk + (p - start)] = key;
                        if (p < end && p < sm.n_q[qi]) atomicAdd(&lhist[qi * kSelBins + top_digit(key)], 1u);
                    }
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&sm.acc_empty[b]);
                b += 2;
                if (b >= a.acc_bufs) b -= a.acc_bufs;
                se += 2;
                if (se >= a.stages) { se -= a.stages; eph ^= 1; }
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    // The cross-chunk counters below were cleared by k0_clear, which may
    // still have been running while this grid streamed (launched as its
    // programmatic dependent); long finished by now, this waits for nothing.
    grid_dependency_wait();
    // the attention kernel may start launching on SMs this grid frees up
    // (it waits for this grid's completion before reading the indices)
    if (tid == 0) grid_launch_dependents();

    // ---- selection (fused mode)
    if (MODE == kModeFused && !sm.abort) {
        // parallel selection stages the chunks' lists below the keys (the
        // TMA ring and the q tile, free now)
        uint64_t *below_keys = reinterpret_cast<uint64_t *>(base);
        const int below_cap = static_cast<int>(L.keys / sizeof(uint64_t));
        for (int qi = 0; qi < nqg; ++qi) {
            const int n = sm.n_q[qi];
            if (n <= a.topk) continue;
            const int qlen = max(min(end, n) - start, 0);
            chunk_select(a, sm, q0 + qi, qi, n, keys + qi * a.chunk, start, qlen,
                         lhist + qi * kSelBins, hist, below_keys, below_cap);
            __syncthreads();
        }
        if (sm.chunk_P > 1 && !a.parallel) {
            bool any = false;
            for (int qi = 0; qi < nqg; ++qi) any |= sm.n_q[qi] > a.topk;
            if (any && arrive_group(a, sm, g)) {
                // candidate list of the threshold bin lives in the (now free)
                // streaming area: stages + q tile + keys
                uint64_t *list = reinterpret_cast<uint64_t *>(base);
                const int list_cap = static_cast<int>(L.hist / sizeof(uint64_t));
                for (int qi = 0; qi < nqg; ++qi)
                    if (sm.n_q[qi] > a.topk) group_merge(a, sm, q0 + qi, qi, hist, list, list_cap);
            }
        }
    }

    // ---- teardown
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) tmem_dealloc(tmem, a.tmem_cols);
}

// ---------------------------------------------------------------------------
// K2: TopK of scores already in HBM (same chunking and merge as K1).
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(kK2Threads, 1) k2_topk(const K1Params a) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *base = align1024(smem_raw);
    const K1Layout L = k1_layout(kModeTopk, 0, 1, 0, a.chunk, a.P, a.topk, 0, true);
    uint32_t *keys = reinterpret_cast<uint32_t *>(base + L.keys);
    uint32_t *hist = reinterpret_cast<uint32_t *>(base + L.hist);
    K1Smem &sm = *reinterpret_cast<K1Smem *>(base + L.misc);
    const int q = blockIdx.x / a.P, c = blockIdx.x % a.P;
    if (threadIdx.x == 0) {
        sm.abort = 0;
        sm.is_last = 0;
        sm.chunk_c = c;
        sm.chunk_P = a.P;
        sm.n_q[0] = a.q_n[q];
        sm.g_complete[0] = 0;
        mbar_init(&sm.merge_bar, 1);
        sm.merge_phase = 0;
        fence_mbar_init();
    }
    __syncthreads();
    const int n = sm.n_q[0];
    if (n <= a.topk) {
        if (c == 0) write_fallback(a, q, n);
        return;
    }
    const int start = c * a.chunk;
    const int end = min(start + a.chunk, n);
    const int len = max(end - start, 0);
    const float *src = a.scores + static_cast<int64_t>(q) * a.ld;
    uint32_t *lhist = hist + kSelBins;
    for (int i = threadIdx.x; i < kSelBins; i += blockDim.x) lhist[i] = 0;
    __syncthreads();
    for (int i0 = 0; i0 < len; i0 += blockDim.x) {
        const int i = i0 + threadIdx.x;
        const uint32_t key = i < len ? float_to_key(__ldg(&src[start + i])) : 0u;
        if (i < len) {
            keys[i] = key;
            atomicAdd(&lhist[top_digit(key)], 1u);
        }
    }
    __syncthreads();
    chunk_select(a, sm, q, 0, n, keys, start, len, lhist, hist, nullptr, 0);
    __syncthreads();
    if (a.P > 1 && arrive_group(a, sm, q)) {
        uint64_t *list = reinterpret_cast<uint64_t *>(base);
        const int list_cap = static_cast<int>(L.hist / sizeof(uint64_t));
        group_merge(a, sm, q, 0, hist, list, list_cap);
    }
}

// ---------------------------------------------------------------------------
// host-side launchers
// ---------------------------------------------------------------------------
// Clears the indexer's cross-chunk counters of one call (16-byte units).
// It lets the next kernel in the stream (k1, launched as its programmatic
// dependent) start at once: k1 streams its keys meanwhile and waits for this
// grid only before it touches the counters.
__global__ void __launch_bounds__(256) k0_clear(uint4 *p, long long n16) {
    grid_launch_dependents();
    const long long stride = static_cast<long long>(gridDim.x) * blockDim.x;
    for (long long i = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; i < n16; i += stride)
        p[i] = make_uint4(0, 0, 0, 0);
}

template <int MODE, int HP, int DI>
static cudaError_t launch_k1_t(const CUtensorMap &kmap, const K1Params &a, cudaStream_t st, bool pdl) {
    const K1Layout L = k1_layout(MODE, DI, a.qg, HP, a.chunk, a.P, a.topk, a.stages, !a.parallel);
    const size_t smem = smem_for_tmem(L.total, a.tmem_cols);
    auto kern = k1_indexer<MODE, HP, DI>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    const int grid = a.n_big * a.P + (a.n_groups - a.n_big) * (a.P - 1);
    if (grid == 0) return cudaSuccess;
    if (!pdl) {
        kern<<<grid, kK1Threads, smem, st>>>(kmap, a);
        return cudaGetLastError();
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(kK1Threads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    e = cudaLaunchKernelEx(&cfg, kern, kmap, a);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

cudaError_t launch_clear(void *p, size_t bytes, cudaStream_t st) {
    const long long n16 = static_cast<long long>(bytes / 16);
    if (n16 == 0) return cudaSuccess;
    long long grid = (n16 + 255) / 256;
    if (grid > 1184) grid = 1184;
    k0_clear<<<static_cast<int>(grid), 256, 0, st>>>(static_cast<uint4 *>(p), n16);
    return cudaGetLastError();
}

cudaError_t launch_indexer(int mode, int hp, int di, const CUtensorMap &kmap, const K1Params &a,
                           cudaStream_t st, bool pdl) {
#define DSA_K1_CASE(M, H, D) \
    if (mode == M && hp == H && di == D) return launch_k1_t<M, H, D>(kmap, a, st, pdl);
    DSA_K1_CASE(kModeFused, 64, 128)
    DSA_K1_CASE(kModeFused, 16, 128)
    DSA_K1_CASE(kModeFused, 64, 64)
    DSA_K1_CASE(kModeFused, 16, 64)
    DSA_K1_CASE(kModeScores, 64, 128)
    DSA_K1_CASE(kModeScores, 16, 128)
    DSA_K1_CASE(kModeScores, 64, 64)
    DSA_K1_CASE(kModeScores, 16, 64)
#undef DSA_K1_CASE
    return cudaErrorInvalidValue;
}

cudaError_t launch_topk(const K1Params &a, cudaStream_t st) {
    const K1Layout L = k1_layout(kModeTopk, 0, 1, 0, a.chunk, a.P, a.topk, 0, true);
    cudaError_t e = cudaFuncSetAttribute(k2_topk, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(L.total));
    if (e != cudaSuccess) return e;
    const int grid = a.nq * a.P;
    if (grid == 0) return cudaSuccess;
    k2_topk<<<grid, kK2Threads, L.total, st>>>(a);
    return cudaGetLastError();
}

}  // namespace dsa
