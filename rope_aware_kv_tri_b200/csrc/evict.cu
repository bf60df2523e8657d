// evict.cu - top-B selection with a recent window, and Forward-Packing
// Compaction of the kept K/V rows.
//
// Pages: "TriAttention: Trigonometric KV Compression for Efficient Long
// Reasoning" - "Core Mechanism" (rank keys and keep only the top-scoring
// subset; top-K selection in the data-flow figure); "TriAttention: How a
// Geometric Trick Cuts LLM Memory Use by 10x Without Losing Accuracy" -
// "Solving the Memory Fragmentation Problem" (survivors move forward so tail
// blocks empty out) and "Why Existing KV Cache Compression Breaks in
// Production" (a paged block is reclaimed only when empty).
//
// One CTA of 512 threads per unit (sequence, layer, KV head).
//
// Selection of len slots, budget B, window W (len > B): the last W slots are
// kept; among the first cand = len - W the take = B - W best by (score desc,
// slot asc).  Scores become 32-bit keys whose unsigned order is the score
// order (order_key: -0 == +0, NaN == -inf).  The exact key thr of the
// take-th best candidate and the number need_eq of candidates equal to it
// that are kept are found with three streaming passes over the unit's
// scores (vectorised, several loads in flight per thread):
//   1. a shared-memory histogram of the top 12 key bits -> the bucket that
//      holds the cut, and the cut's rank inside it;
//   2. a walk that collects that bucket's (key, slot) pairs into shared
//      memory and counts, per warp segment, the keys above the bucket;
//      two radix passes over the collected pairs (10 + 10 bits) then give
//      thr and need_eq, and the per-segment counts of keys > thr and == thr;
//   3. the emission walk: each warp owns a contiguous segment of slots, and
//      with ballots and the per-segment offsets writes the kept slots in
//      ascending order (ties go to the lower slot, so the result is unique).
// If the cut's bucket holds more keys than the shared list (e.g. many equal
// scores) the remaining 20 bits are resolved with streaming radix passes
// instead, followed by a counting walk.
//
// Compaction, in place: row j of K and V takes row idx_j (idx ascending, so
// idx_j >= j).  Rows j < m0 have idx_j == j and stay.  Only rows that are
// both a destination and a not-yet-read source can be clobbered, and every
// such source is an idx_j < kept, i.e. one of the first J entries of idx.
//   Phase 1 moves rows [m0, J) in ascending chunks of 64: the whole chunk is
//   loaded into registers, the CTA synchronises, then the chunk is stored.
//   A chunk's stores land on rows [a, b) that no later chunk reads (its
//   sources are >= b) and whose readers in this or earlier chunks have
//   loaded before the barrier.
//   Phase 2 moves rows [J, kept) in a separate kernel (move_kernel): their
//   sources are >= kept, where no store ever lands, and every earlier reader
//   of their destination rows loaded in phase 1, which the kernel boundary
//   completes; so all rows of all units move independently, many in flight.
// With a budget of a few percent of the cache, J - m0 is typically small and
// almost all rows move in phase 2.
#include <climits>

#include "tri_device.cuh"
#include "tri_internal.h"

namespace tri {

namespace {

constexpr int kEvictThreads = 512;
constexpr int kEvictWarps = kEvictThreads / 32;
constexpr int kTopShift = 20;                     // first pass: key bits [20, 32)
constexpr int kTopBins = 1 << (32 - kTopShift);   // 4096
constexpr int kListCap = 4096;                    // boundary-bucket pairs kept in shared memory
constexpr int kBitmapWords = 4096;                // bitmaps of up to 131072 candidate slots
constexpr int kLinBins = 4096;                    // linear buckets over a unit's score range
constexpr int kRankListMax = 1024;                // lists up to this size are ranked directly
constexpr int kCodeSlots = 32768;                 // candidates whose buckets fit in shared memory
constexpr int kOneListCap = 1024;                 // cut-bucket entries in the one-pass layout
constexpr int kUnroll = 8;                        // 16-byte loads in flight per thread in a walk
constexpr int kStep = 128;                        // slots per warp step (4 per lane)
constexpr int kRowBytes = kHeadDim * 2;           // 256
constexpr int kSlicesPerRowHalf = kRowBytes / 16;  // 16-byte slices of a K (or V) row: 16
constexpr int kSlicesPerRow = 2 * kSlicesPerRowHalf;   // K and V: 32
constexpr int kModeInPlace = 0, kModeScratch = 1;  // how a unit's rows [m0, J) are handled
constexpr int kMoveThreads = 256;
constexpr int kMoveRows = 8;                      // rows in flight per warp in move_kernel

// Shared scratch of the selection, in one of two layouts.  "two" serves
// units with more candidates than `code` holds (two streaming passes);
// "one" keeps every candidate's linear bucket in shared memory so the
// scores are streamed once.  Both start with the histogram.
struct TwoPassScratch {
    int hist[kTopBins];
    uint32_t list_key[kListCap];
    int list_slot[kListCap];
    uint32_t gt_bits[kBitmapWords];   // candidates kept for a score above the cut
    uint32_t eq_bits[kBitmapWords];   // candidates whose score equals the cut
};
struct OnePassScratch {
    int hist[kLinBins];
    uint32_t gt_bits[kCodeSlots / 32];
    uint32_t eq_bits[kCodeSlots / 32];
    uint32_t list_key[kOneListCap];
    int list_slot[kOneListCap];
    uint16_t code[kCodeSlots];        // linear bucket of every candidate
};
union SelectScratch {
    TwoPassScratch two;
    OnePassScratch one;
    int hist[kTopBins];
};
struct EvictSmem {
    union {
        SelectScratch sel;
    } u;
    static_assert(sizeof(OnePassScratch) <= 100 * 1024, "one-pass scratch too large");
    int warp_a[kEvictWarps];      // keys > thr in the segment (part 1)
    int warp_b[kEvictWarps];      // keys == thr in the segment
    int warp_c[kEvictWarps];      // keys > thr in the segment (part 2)
    int eq_before[kEvictWarps];
    int keep_before[kEvictWarps];
    int scan_tmp[kEvictWarps];    // scratch of block scans
    int bcast[4];
    int n_list;
};

static_assert(sizeof(SelectScratch) >= TRI_MAX_BUDGET * sizeof(int), "position staging does not fit");

// rows per ordered compaction round, staged in the selection scratch
constexpr int kStageRows = (int)(sizeof(SelectScratch) / (2 * kRowBytes));
// With many units per launch (several waves of CTAs), units whose at-risk
// prefix is longer than a few ordered rounds compact it in place: the
// scratch path moves those rows twice (out to the scratch and back), the
// ordered rounds once, and the other units' CTAs hide the rounds' latency.
// With one wave of units the longest in-place unit would set the kernel's
// time, so every prefix that fits takes the scratch.
constexpr int kScratchMaxRows = 4 * kStageRows;

__device__ __forceinline__ int block_sum(int v, EvictSmem& sm) {
    int total;
    block_exclusive_scan<kEvictThreads>(v, sm.scan_tmp, total);
    return total;
}

// The bin of `hist` (nb bins, nb >= 512, higher bin = higher value) that
// holds the rem-th largest counted element; rem becomes its rank in the bin.
__device__ int pick_bin(const int* hist, int nb, int& rem, EvictSmem& sm) {
    const int per = nb / kEvictThreads;
    const int b0 = threadIdx.x * per;
    int local = 0;
    for (int j = 0; j < per; ++j) local += hist[b0 + j];
    int total;
    const int ex = block_exclusive_scan<kEvictThreads>(local, sm.scan_tmp, total);
    int run = total - ex - local;      // elements in bins above this thread's bins
    for (int j = per - 1; j >= 0; --j) {
        const int h = hist[b0 + j];
        if (run < rem && rem <= run + h) {
            sm.bcast[0] = b0 + j;
            sm.bcast[1] = rem - run;
        }
        run += h;
    }
    __syncthreads();
    const int bin = sm.bcast[0];
    rem = sm.bcast[1];
    __syncthreads();
    return bin;
}

// Pick the digit of the histogram `hist` (nb bins) in which the rem-th
// largest counted key lies; update (prefix, mask, rem).
__device__ void pick_digit(const int* hist, int nb, int shift, uint32_t& prefix, uint32_t& mask, int& rem,
                           EvictSmem& sm) {
    const int d = pick_bin(hist, nb, rem, sm);
    prefix |= (uint32_t)d << shift;
    mask |= (uint32_t)(nb - 1) << shift;
}

// Pass 1: histogram of the top key bits of candidates [lo, cand).  Returns
// whether a NaN score was seen.
__device__ bool top_histogram(const float* __restrict__ sc, int cand, int lo, int* hist) {
    for (int i = threadIdx.x; i < kTopBins; i += kEvictThreads) hist[i] = 0;
    __syncthreads();
    bool nan_seen = false;
    const int nvec = cand >> 2;
    const float4* v4 = reinterpret_cast<const float4*>(sc);
    for (int v0 = threadIdx.x; v0 < nvec; v0 += kEvictThreads * kUnroll) {
        float4 x[kUnroll];
#pragma unroll
        for (int k = 0; k < kUnroll; ++k) {
            const int v = v0 + k * kEvictThreads;
            x[k] = v < nvec ? v4[v] : make_float4(0.f, 0.f, 0.f, 0.f);
        }
#pragma unroll
        for (int k = 0; k < kUnroll; ++k) {
            if (v0 + k * kEvictThreads < nvec) {
                const float e[4] = {x[k].x, x[k].y, x[k].z, x[k].w};
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    if (4 * (v0 + k * kEvictThreads) + c >= lo) {
                        nan_seen |= isnan(e[c]);
                        atomicAdd(&hist[order_key(e[c]) >> kTopShift], 1);
                    }
                }
            }
        }
    }
    for (int t = max(4 * nvec, lo) + threadIdx.x; t < cand; t += kEvictThreads) {
        const float e = sc[t];
        nan_seen |= isnan(e);
        atomicAdd(&hist[order_key(e) >> kTopShift], 1);
    }
    return __syncthreads_or(nan_seen) != 0;
}

// Load the 4 scores of slots t..t+3 of a warp step (those >= end invalid).
__device__ __forceinline__ void load4(const float* __restrict__ sc, int t, int end, float (&x)[4]) {
    if (t + 3 < end) {
        const float4 v = *reinterpret_cast<const float4*>(sc + t);
        x[0] = v.x; x[1] = v.y; x[2] = v.z; x[3] = v.w;
    } else {
#pragma unroll
        for (int c = 0; c < 4; ++c) x[c] = (t + c < end) ? sc[t + c] : 0.f;
    }
}

// Streaming radix pass over all candidates (fallback when the cut's bucket
// does not fit the shared list).
__device__ void stream_radix_pass(const float* __restrict__ sc, int cand, int lo, uint32_t& prefix, uint32_t& mask,
                                  int& rem, int shift, int bits, int* hist, EvictSmem& sm) {
    const int nb = 1 << bits;
    const uint32_t dmask = (uint32_t)nb - 1u;
    for (int i = threadIdx.x; i < nb; i += kEvictThreads) hist[i] = 0;
    __syncthreads();
    for (int t = lo + threadIdx.x; t < cand; t += kEvictThreads) {
        const uint32_t key = order_key(sc[t]);
        if ((key & mask) == prefix) atomicAdd(&hist[(key >> shift) & dmask], 1);
    }
    __syncthreads();
    pick_digit(hist, nb, shift, prefix, mask, rem, sm);
}

// Radix pass over the shared list of boundary-bucket keys.
__device__ void list_radix_pass(const uint32_t* keys, int n, uint32_t& prefix, uint32_t& mask, int& rem,
                                int shift, int bits, int* hist, EvictSmem& sm) {
    const int nb = 1 << bits;
    const uint32_t dmask = (uint32_t)nb - 1u;
    for (int i = threadIdx.x; i < nb; i += kEvictThreads) hist[i] = 0;
    __syncthreads();
    for (int i = threadIdx.x; i < n; i += kEvictThreads) {
        const uint32_t key = keys[i];
        if ((key & mask) == prefix) atomicAdd(&hist[(key >> shift) & dmask], 1);
    }
    __syncthreads();
    pick_digit(hist, nb, shift, prefix, mask, rem, sm);
}

// Spread the 8 low bits of x to bit positions 0, 4, 8, ..., 28.
__device__ __forceinline__ uint32_t spread4(uint32_t x) {
    x &= 0xffu;
    x = (x | (x << 12)) & 0x000f000fu;
    x = (x | (x << 6)) & 0x03030303u;
    x = (x | (x << 3)) & 0x11111111u;
    return x;
}

// A warp step covers 128 slots, lane L holding slots 4L..4L+3; c[k] is the
// ballot of component k.  Returns the 32-slot word w (slots 32w..32w+31 of
// the step) in slot order.
__device__ __forceinline__ uint32_t step_word(const uint32_t (&c)[4], int w) {
    return spread4(c[0] >> (8 * w)) | (spread4(c[1] >> (8 * w)) << 1) | (spread4(c[2] >> (8 * w)) << 2) |
           (spread4(c[3] >> (8 * w)) << 3);
}

// Inverse of order_key for keys of non-NaN scores.
__device__ __forceinline__ float key_value(uint32_t key) {
    return __uint_as_float((key & 0x80000000u) ? (key & 0x7fffffffu) : ~key);
}

// Linear bucket of score x in [lo, lo + (kLinBins-1)/scale]; monotone in x.
__device__ __forceinline__ int lin_bucket(float x, float lo, float scale) {
    const int b = (int)((x - lo) * scale);
    return b < 0 ? 0 : (b > kLinBins - 1 ? kLinBins - 1 : b);
}

// Emit the set bits of `bits` (nwords words, slot 32w + b) into sidx in
// ascending order, at most `take` of them.  Each warp takes a contiguous run
// of words; lane i tests bit i of the warp's current word, so the warp writes
// a whole word per step whatever its population.
__device__ void emit_kept(const uint32_t* bits, int nwords, int take, int* sidx, EvictSmem& sm) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int per = (nwords + kEvictWarps - 1) / kEvictWarps;
    const int w0 = min(warp * per, nwords), w1 = min(w0 + per, nwords);
    int cnt = 0;
    for (int w = w0 + lane; w < w1; w += 32) cnt += __popc(bits[w]);
    cnt = __reduce_add_sync(0xffffffffu, cnt);
    if (lane == 0) sm.warp_a[warp] = cnt;
    __syncthreads();
    int base = 0;
    for (int k = 0; k < warp; ++k) base += sm.warp_a[k];
    const uint32_t lt = lanemask_lt();
    for (int w = w0; w < w1; ++w) {
        const uint32_t kw = bits[w];
        const int pos = base + __popc(kw & lt);
        if (((kw >> lane) & 1u) && pos < take) sidx[pos] = w * 32 + lane;
        base += __popc(kw);
    }
    __syncthreads();
}

// The cut from the list of the cut bucket's keys (rem = the cut's rank in
// the bucket), then the kept candidates from the bitmaps: gt_bits holds the
// candidates above the bucket; the list's keys above the cut join them, the
// ones equal to it go to eq_bits, of which the first need_eq in slot order
// are kept.  Emits the take kept slots ascending into sidx.
__device__ void finish_from_list(const uint32_t* list_key, const int* list_slot, int n, int rem, uint32_t* gt_bits,
                                 uint32_t* eq_bits, int nwords, int take, int* sidx, int* hist, EvictSmem& sm) {
    uint32_t thr;
    int need_eq;
    if (n <= kRankListMax) {
        // the cut key is the list key with (#greater) < rem <= (#greater-or-equal)
        for (int i = threadIdx.x; i < n; i += kEvictThreads) {
            const uint32_t key = list_key[i];
            int gt = 0, ge = 0;
            for (int k = 0; k < n; ++k) {
                const uint32_t o = list_key[k];
                gt += o > key ? 1 : 0;
                ge += o >= key ? 1 : 0;
            }
            if (gt < rem && rem <= ge) {         // every thread that finds it writes the same values
                sm.bcast[2] = (int)key;
                sm.bcast[3] = rem - gt;
            }
        }
        __syncthreads();
        thr = (uint32_t)sm.bcast[2];
        need_eq = sm.bcast[3];
    } else {
        uint32_t prefix = 0, mask = 0;
        list_radix_pass(list_key, n, prefix, mask, rem, 21, 11, hist, sm);
        list_radix_pass(list_key, n, prefix, mask, rem, 10, 11, hist, sm);
        list_radix_pass(list_key, n, prefix, mask, rem, 0, 10, hist, sm);
        thr = prefix;
        need_eq = rem;
    }
    for (int i = threadIdx.x; i < n; i += kEvictThreads) {
        const uint32_t key = list_key[i];
        const int t = list_slot[i];
        if (key > thr) atomicOr(&gt_bits[t >> 5], 1u << (t & 31));
        else if (key == thr) atomicOr(&eq_bits[t >> 5], 1u << (t & 31));
    }
    __syncthreads();
    // Emission: each thread owns a run of words; the first need_eq tied
    // candidates in slot order are kept.
    const int wpt = (nwords + kEvictThreads - 1) / kEvictThreads;
    const int w0 = min(threadIdx.x * wpt, nwords), w1 = min(w0 + wpt, nwords);
    int my_eq = 0;
    for (int w = w0; w < w1; ++w) my_eq += __popc(eq_bits[w]);
    int tot;
    int eq_before = block_exclusive_scan<kEvictThreads>(my_eq, sm.scan_tmp, tot);
    for (int w = w0; w < w1; ++w) {
        uint32_t e = eq_bits[w];
        int allow = need_eq - eq_before;
        eq_before += __popc(e);
        uint32_t keep_e = 0u;
        while (e && allow > 0) {
            const uint32_t low = e & (0u - e);
            keep_e |= low;
            e ^= low;
            --allow;
        }
        gt_bits[w] |= keep_e;
    }
    __syncthreads();
    emit_kept(gt_bits, nwords, take, sidx, sm);
}

// One streaming pass (cand <= kCodeSlots): the histogram pass also keeps
// every candidate's linear bucket in shared memory; the bitmap of buckets
// above the cut's and the cut bucket's slots then come from shared memory,
// and only the (few) cut-bucket scores are read again.
__device__ bool select_one_pass(const float* __restrict__ sc, int cand, int first, int take, float lo, float scale,
                                int* sidx, EvictSmem& sm) {
    OnePassScratch& o = sm.u.sel.one;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    for (int i = threadIdx.x; i < kLinBins; i += kEvictThreads) o.hist[i] = 0;
    __syncthreads();
    const int nvec = cand >> 2;
    const float4* v4 = reinterpret_cast<const float4*>(sc);
    for (int v0 = threadIdx.x; v0 < nvec; v0 += kEvictThreads * kUnroll) {
        float4 x[kUnroll];
#pragma unroll
        for (int k = 0; k < kUnroll; ++k) {
            const int v = v0 + k * kEvictThreads;
            x[k] = v < nvec ? v4[v] : make_float4(0.f, 0.f, 0.f, 0.f);
        }
#pragma unroll
        for (int k = 0; k < kUnroll; ++k) {
            const int v = v0 + k * kEvictThreads;
            if (v < nvec) {
                const int b0 = lin_bucket(x[k].x, lo, scale), b1 = lin_bucket(x[k].y, lo, scale);
                const int b2 = lin_bucket(x[k].z, lo, scale), b3 = lin_bucket(x[k].w, lo, scale);
                *reinterpret_cast<uint2*>(&o.code[4 * v]) =
                    make_uint2((uint32_t)b0 | ((uint32_t)b1 << 16), (uint32_t)b2 | ((uint32_t)b3 << 16));
                if (4 * v >= first) {
                    atomicAdd(&o.hist[b0], 1);
                    atomicAdd(&o.hist[b1], 1);
                    atomicAdd(&o.hist[b2], 1);
                    atomicAdd(&o.hist[b3], 1);
                } else {
                    // the first vector holds excluded leading slots
                    if (4 * v + 0 >= first) atomicAdd(&o.hist[b0], 1);
                    if (4 * v + 1 >= first) atomicAdd(&o.hist[b1], 1);
                    if (4 * v + 2 >= first) atomicAdd(&o.hist[b2], 1);
                    if (4 * v + 3 >= first) atomicAdd(&o.hist[b3], 1);
                }
            }
        }
    }
    for (int t = 4 * nvec + threadIdx.x; t < cand; t += kEvictThreads) {
        const int b = lin_bucket(sc[t], lo, scale);
        o.code[t] = (uint16_t)b;
        if (t >= first) atomicAdd(&o.hist[b], 1);
    }
    __syncthreads();
    int rem = take;
    const int bstar = pick_bin(o.hist, kLinBins, rem, sm);
    if (o.hist[bstar] > kOneListCap) return false;
    const int nwords = (cand + 31) / 32;
    for (int w = threadIdx.x; w < nwords; w += kEvictThreads) o.eq_bits[w] = 0u;
    if (threadIdx.x == 0) sm.n_list = 0;
    __syncthreads();
    // 8 buckets per 16-byte load; 4 lanes make one 32-slot word
    const int nq = (cand + 7) / 8;
    for (int q0 = warp * 32; q0 < nq; q0 += kEvictWarps * 32) {
        const int q = q0 + lane;
        uint32_t m = 0u;
        if (q < nq) {
            const uint4 c4 = *reinterpret_cast<const uint4*>(&o.code[8 * q]);
            const uint32_t cw[4] = {c4.x, c4.y, c4.z, c4.w};
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const int t = 8 * q + i;
                const int b = (int)((cw[i >> 1] >> (16 * (i & 1))) & 0xffffu);
                if (t < cand && t >= first) {
                    if (b > bstar) m |= 1u << i;
                    else if (b == bstar) {
                        const int pos = atomicAdd(&sm.n_list, 1);
                        if (pos < kOneListCap) o.list_slot[pos] = t;
                    }
                }
            }
        }
        uint32_t word = m << (8 * (lane & 3));
        word |= __shfl_xor_sync(0xffffffffu, word, 1);
        word |= __shfl_xor_sync(0xffffffffu, word, 2);
        if ((lane & 3) == 0 && q < nq) o.gt_bits[q >> 2] = word;
    }
    __syncthreads();
    const int n = min(sm.n_list, kOneListCap);
    for (int i = threadIdx.x; i < n; i += kEvictThreads) o.list_key[i] = order_key(sc[o.list_slot[i]]);
    __syncthreads();
    finish_from_list(o.list_key, o.list_slot, n, rem, o.gt_bits, o.eq_bits, nwords, take, sidx, o.hist, sm);
    return true;
}

// Selection over a known score range [kmin, kmax] (order keys): a linear
// histogram finds the bucket of the cut; the candidates above that bucket go
// to a bitmap and the bucket's (key, slot) pairs to a list; the exact cut
// key and its tie count come from the list; the kept slots are then emitted
// from the bitmaps in slot order.  Returns false, with nothing kept, when the
// range is not finite, the candidates exceed the bitmap, or the cut's
// bucket exceeds the list.
__device__ bool select_linear(const float* __restrict__ sc, int cand, int first, int take, uint32_t kmin,
                              uint32_t kmax, int* sidx, EvictSmem& sm) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const float lo = key_value(kmin), hi = key_value(kmax);
    if (kmin > kmax || !isfinite(lo) || !isfinite(hi) || cand > kBitmapWords * 32) return false;
    const float span = hi - lo;
    if (!isfinite(span)) return false;
    if (span == 0.f) {
        // every score of the unit is equal: the lowest slots win every tie
        for (int j = threadIdx.x; j < take; j += kEvictThreads) sidx[j] = first + j;
        return true;
    }
    const float scale = (float)(kLinBins - 1) / span;
    if (cand <= kCodeSlots) return select_one_pass(sc, cand, first, take, lo, scale, sidx, sm);
    int* hist = sm.u.sel.hist;
    // warp segments of whole 128-slot steps
    const int seg = ((cand + kEvictWarps - 1) / kEvictWarps + kStep - 1) / kStep * kStep;
    const int beg = min(warp * seg, cand);
    const int end = min(beg + seg, cand);

    // Pass 1: linear histogram (16-byte loads, kUnroll per thread in flight).
    for (int i = threadIdx.x; i < kLinBins; i += kEvictThreads) hist[i] = 0;
    __syncthreads();
    {
        const int nvec = cand >> 2;
        const float4* v4 = reinterpret_cast<const float4*>(sc);
        for (int v0 = threadIdx.x; v0 < nvec; v0 += kEvictThreads * kUnroll) {
            float4 x[kUnroll];
#pragma unroll
            for (int k = 0; k < kUnroll; ++k) {
                const int v = v0 + k * kEvictThreads;
                x[k] = v < nvec ? v4[v] : make_float4(0.f, 0.f, 0.f, 0.f);
            }
#pragma unroll
            for (int k = 0; k < kUnroll; ++k) {
                const int t = 4 * (v0 + k * kEvictThreads);
                if (v0 + k * kEvictThreads < nvec) {
                    if (t + 0 >= first) atomicAdd(&hist[lin_bucket(x[k].x, lo, scale)], 1);
                    if (t + 1 >= first) atomicAdd(&hist[lin_bucket(x[k].y, lo, scale)], 1);
                    if (t + 2 >= first) atomicAdd(&hist[lin_bucket(x[k].z, lo, scale)], 1);
                    if (t + 3 >= first) atomicAdd(&hist[lin_bucket(x[k].w, lo, scale)], 1);
                }
            }
        }
        for (int t = max(4 * nvec, first) + threadIdx.x; t < cand; t += kEvictThreads)
            atomicAdd(&hist[lin_bucket(sc[t], lo, scale)], 1);
    }
    __syncthreads();
    int rem = take;
    const int bstar = pick_bin(hist, kLinBins, rem, sm);
    if (hist[bstar] > kListCap) return false;

    // Pass 2: bitmap of candidates above the cut's bucket; list of the bucket.
    const int nwords = (cand + 31) / 32;
    for (int w = threadIdx.x; w < nwords; w += kEvictThreads) sm.u.sel.two.eq_bits[w] = 0u;
    if (threadIdx.x == 0) sm.n_list = 0;
    __syncthreads();
    const uint32_t lt = lanemask_lt();
    for (int t0 = beg; t0 < end; t0 += kStep * kUnroll) {
        float x[kUnroll][4];
#pragma unroll
        for (int k = 0; k < kUnroll; ++k) load4(sc, t0 + k * kStep + 4 * lane, end, x[k]);
#pragma unroll
        for (int k = 0; k < kUnroll; ++k) {
            const int base = t0 + k * kStep;
            if (base < end) {
                const int t = base + 4 * lane;
                uint32_t above[4], inb[4];
                int n_in = 0;
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    const bool valid = t + c < end && t + c >= first;
                    const int b = lin_bucket(x[k][c], lo, scale);
                    above[c] = __ballot_sync(0xffffffffu, valid && b > bstar);
                    inb[c] = __ballot_sync(0xffffffffu, valid && b == bstar);
                    n_in += __popc(inb[c]);
                }
                if (lane < 4 && base + 32 * lane < end) sm.u.sel.two.gt_bits[(base >> 5) + lane] = step_word(above, lane);
                if (n_in) {
                    int at = 0;
                    if (lane == 0) at = atomicAdd(&sm.n_list, n_in);
                    at = __shfl_sync(0xffffffffu, at, 0);
#pragma unroll
                    for (int c = 0; c < 4; ++c) {
                        if (inb[c] & (1u << lane)) {
                            const int pos = at + __popc(inb[c] & lt);
                            if (pos < kListCap) {
                                sm.u.sel.two.list_key[pos] = order_key(x[k][c]);
                                sm.u.sel.two.list_slot[pos] = t + c;
                            }
                        }
                        at += __popc(inb[c]);
                    }
                }
            }
        }
    }
    __syncthreads();
    const int n = min(sm.n_list, kListCap);
    finish_from_list(sm.u.sel.two.list_key, sm.u.sel.two.list_slot, n, rem, sm.u.sel.two.gt_bits,
                     sm.u.sel.two.eq_bits, nwords, take, sidx, hist, sm);
    return true;
}

// Smallest and largest order key among the candidates (block reduction).
__device__ void candidate_key_range(const float* __restrict__ sc, int cand, int first, uint32_t& kmin,
                                    uint32_t& kmax, EvictSmem& sm) {
    uint32_t lo = 0xffffffffu, hi = 0u;
    const int nvec = cand >> 2;
    const float4* v4 = reinterpret_cast<const float4*>(sc);
    for (int v0 = threadIdx.x; v0 < nvec; v0 += kEvictThreads * kUnroll) {
        float4 x[kUnroll];
#pragma unroll
        for (int k = 0; k < kUnroll; ++k) {
            const int v = v0 + k * kEvictThreads;
            x[k] = v < nvec ? v4[v] : make_float4(0.f, 0.f, 0.f, 0.f);
        }
#pragma unroll
        for (int k = 0; k < kUnroll; ++k) {
            const int t = 4 * (v0 + k * kEvictThreads);
            if (v0 + k * kEvictThreads < nvec) {
                // an excluded leading slot takes a neutral key (the range's own bounds)
                const uint32_t a = order_key(x[k].x), b = order_key(x[k].y);
                const uint32_t c = order_key(x[k].z), d = order_key(x[k].w);
                lo = min(lo, min(min(t + 0 >= first ? a : 0xffffffffu, t + 1 >= first ? b : 0xffffffffu),
                                 min(t + 2 >= first ? c : 0xffffffffu, t + 3 >= first ? d : 0xffffffffu)));
                hi = max(hi, max(max(t + 0 >= first ? a : 0u, t + 1 >= first ? b : 0u),
                                 max(t + 2 >= first ? c : 0u, t + 3 >= first ? d : 0u)));
            }
        }
    }
    for (int t = max(4 * nvec, first) + threadIdx.x; t < cand; t += kEvictThreads) {
        const uint32_t k = order_key(sc[t]);
        lo = min(lo, k);
        hi = max(hi, k);
    }
    lo = __reduce_min_sync(0xffffffffu, lo);
    hi = __reduce_max_sync(0xffffffffu, hi);
    __shared__ uint32_t wlo[kEvictWarps], whi[kEvictWarps];
    if ((threadIdx.x & 31) == 0) {
        wlo[threadIdx.x >> 5] = lo;
        whi[threadIdx.x >> 5] = hi;
    }
    __syncthreads();
    kmin = 0xffffffffu;
    kmax = 0u;
    for (int w = 0; w < kEvictWarps; ++w) {
        kmin = min(kmin, wlo[w]);
        kmax = max(kmax, whi[w]);
    }
    __syncthreads();
}

// Kept slots of a unit of len > budget slots: [0, sinks), the best
// budget - window - sinks of [sinks, len - window), and the last window.
// The ranking passes run on a 16-byte aligned view that starts at slot
// a = sinks rounded down to a multiple of 4; the first (sinks - a) slots of
// the view are excluded, and the view's slot numbers are shifted back by a.
// kmin_in: whether (kmin, kmax) already bound the unit's score keys.
__device__ void select_unit(const float* __restrict__ sc_unit, int len, int budget, int window, int sinks,
                            int* sidx_unit, EvictSmem& sm, int32_t* status, bool kmin_in, uint32_t kmin,
                            uint32_t kmax) {
    const int a = sinks & ~3;
    const int first = sinks - a;
    const float* __restrict__ sc = sc_unit + a;
    int* sidx = sidx_unit + sinks;
    const int cand = len - window - a;
    const int take = budget - window - sinks;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    bool done = take == 0;
    if (!done) {
        // A NaN score has the key of -infinity, so it always leaves the range
        // non-finite and takes the streaming path, which flags it.
        if (!kmin_in) candidate_key_range(sc, cand, first, kmin, kmax, sm);
        done = select_linear(sc, cand, first, take, kmin, kmax, sidx, sm);
    }
    if (!done) {
        int* hist = sm.u.sel.hist;
        // warp segments: multiples of 128 slots so every step is float4-aligned
        const int seg = ((cand + kEvictWarps - 1) / kEvictWarps + kStep - 1) / kStep * kStep;
        const int beg = min(warp * seg, cand);
        const int end = min(beg + seg, cand);

        if (top_histogram(sc, cand, first, hist) && threadIdx.x == 0) raise_flag(status, TRI_DEVFLAG_NONFINITE);
        uint32_t prefix = 0, mask = 0;
        int rem = take;
        pick_digit(hist, kTopBins, kTopShift, prefix, mask, rem, sm);
        const uint32_t top = prefix >> kTopShift;
        const int in_bucket = hist[top];
        if (threadIdx.x == 0) sm.n_list = 0;
        __syncthreads();

        if (in_bucket <= kListCap) {
            // Pass 2: collect the bucket, count keys above it per segment.
            int above = 0;
            for (int t0 = beg; t0 < end; t0 += kStep * kUnroll) {
                float x[kUnroll][4];
#pragma unroll
                for (int k = 0; k < kUnroll; ++k) load4(sc, t0 + k * kStep + 4 * lane, end, x[k]);
#pragma unroll
                for (int k = 0; k < kUnroll; ++k) {
#pragma unroll
                    for (int c = 0; c < 4; ++c) {
                        const int t = t0 + k * kStep + 4 * lane + c;
                        if (t < end && t >= first) {
                            const uint32_t key = order_key(x[k][c]);
                            const uint32_t d = key >> kTopShift;
                            above += d > top ? 1 : 0;
                            if (d == top) {
                                const int pos = atomicAdd(&sm.n_list, 1);
                                if (pos < kListCap) {
                                    sm.u.sel.two.list_key[pos] = key;
                                    sm.u.sel.two.list_slot[pos] = t;
                                }
                            }
                        }
                    }
                }
            }
            above = __reduce_add_sync(0xffffffffu, above);
            if (lane == 0) sm.warp_a[warp] = above;
            __syncthreads();
            const int n = min(sm.n_list, kListCap);
            list_radix_pass(sm.u.sel.two.list_key, n, prefix, mask, rem, 10, 10, hist, sm);
            list_radix_pass(sm.u.sel.two.list_key, n, prefix, mask, rem, 0, 10, hist, sm);
            if (threadIdx.x < kEvictWarps) {
                sm.warp_b[threadIdx.x] = 0;
                sm.warp_c[threadIdx.x] = 0;
            }
            __syncthreads();
            for (int i = threadIdx.x; i < n; i += kEvictThreads) {
                const uint32_t key = sm.u.sel.two.list_key[i];
                const int w = sm.u.sel.two.list_slot[i] / seg;
                if (key > prefix) atomicAdd(&sm.warp_c[w], 1);
                else if (key == prefix) atomicAdd(&sm.warp_b[w], 1);
            }
        } else {
            // Fallback: stream the remaining bits, then count per segment.
            stream_radix_pass(sc, cand, first, prefix, mask, rem, 10, 10, hist, sm);
            stream_radix_pass(sc, cand, first, prefix, mask, rem, 0, 10, hist, sm);
            int gt = 0, eq = 0;
            for (int t0 = beg; t0 < end; t0 += kStep) {
                float x[4];
                load4(sc, t0 + 4 * lane, end, x);
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    const int t = t0 + 4 * lane + c;
                    const uint32_t key = order_key(x[c]);
                    const bool in = t < end && t >= first;
                    gt += (in && key > prefix) ? 1 : 0;
                    eq += (in && key == prefix) ? 1 : 0;
                }
            }
            gt = __reduce_add_sync(0xffffffffu, gt);
            eq = __reduce_add_sync(0xffffffffu, eq);
            if (lane == 0) {
                sm.warp_a[warp] = gt;
                sm.warp_b[warp] = eq;
                sm.warp_c[warp] = 0;
            }
        }
        __syncthreads();
        const uint32_t thr = prefix;
        const int need_eq = rem;
        if (threadIdx.x == 0) {
            int eb = 0, kb = 0;
            for (int w = 0; w < kEvictWarps; ++w) {
                const int gt_w = sm.warp_a[w] + sm.warp_c[w], eq_w = sm.warp_b[w];
                sm.eq_before[w] = eb;
                sm.keep_before[w] = kb;
                const int left = need_eq - eb;
                kb += gt_w + (left <= 0 ? 0 : (left < eq_w ? left : eq_w));
                eb += eq_w;
            }
        }
        __syncthreads();
        // Pass 3: emit the kept candidates in ascending slot order.
        int run_eq = sm.eq_before[warp], run_keep = sm.keep_before[warp];
        const uint32_t lt = lanemask_lt();
        for (int t0 = beg; t0 < end; t0 += kStep * kUnroll) {
            float x[kUnroll][4];
#pragma unroll
            for (int k = 0; k < kUnroll; ++k) load4(sc, t0 + k * kStep + 4 * lane, end, x[k]);
#pragma unroll
            for (int k = 0; k < kUnroll; ++k) {
                const int t = t0 + k * kStep + 4 * lane;
                bool g[4], e[4];
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    const uint32_t key = order_key(x[k][c]);
                    const bool in = t + c < end && t + c >= first;
                    g[c] = in && key > thr;
                    e[c] = in && key == thr;
                }
                uint32_t eb[4];
                int eq_lanes = 0, eq_all = 0;
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    eb[c] = __ballot_sync(0xffffffffu, e[c]);
                    eq_lanes += __popc(eb[c] & lt);
                    eq_all += __popc(eb[c]);
                }
                bool keep[4];
                int mine = 0;
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    keep[c] = g[c] || (e[c] && run_eq + eq_lanes + mine < need_eq);
                    mine += e[c] ? 1 : 0;
                }
                int kp_lanes = 0, kp_all = 0;
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    const uint32_t kb = __ballot_sync(0xffffffffu, keep[c]);
                    kp_lanes += __popc(kb & lt);
                    kp_all += __popc(kb);
                }
                int off = run_keep + kp_lanes;
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    if (keep[c]) {
                        if (off < take) sidx[off] = t + c;
                        ++off;
                    }
                }
                run_eq += eq_all;
                run_keep += kp_all;
            }
        }
    }
    __syncthreads();
    if (a > 0)
        for (int j = threadIdx.x; j < take; j += kEvictThreads) sidx[j] += a;
    for (int j = threadIdx.x; j < sinks; j += kEvictThreads) sidx_unit[j] = j;
    for (int j = threadIdx.x; j < window; j += kEvictThreads) sidx[take + j] = a + cand + j;
    __syncthreads();
}

// Byte offset of row `row` of (layer, head) in a pool, through the table;
// false if its block id is out of range.
__device__ __forceinline__ bool row_offset(const int32_t* bt, int row, int64_t layer_tiles, int Hkv, int h,
                                           int num_blocks, int64_t& off) {
    const int b = bt[row / kBlockRows];
    if (b < 0 || b >= num_blocks) return false;
    off = (((layer_tiles + b) * Hkv + h) * kBlockRows + (row % kBlockRows)) * kRowBytes;
    return true;
}

// Move the 16-byte slice `part` (0..31: K then V) of row j <- row sidx[j].
struct SliceMove {
    const uint8_t* src;
    uint8_t* dst;
};

__device__ __forceinline__ bool slice_move(const int* sidx, int j, int part, const int32_t* bt, int64_t layer_tiles,
                                           const EvictParams& p, int h, SliceMove& m) {
    int64_t so, dof;
    if (!row_offset(bt, sidx[j], layer_tiles, p.Hkv, h, p.num_blocks, so) ||
        !row_offset(bt, j, layer_tiles, p.Hkv, h, p.num_blocks, dof))
        return false;
    const int64_t in_row = (int64_t)(part % kSlicesPerRowHalf) * 16;
    uint8_t* pool = part < kSlicesPerRowHalf ? p.k_pool : p.v_pool;
    m.src = pool + so + in_row;
    m.dst = pool + dof + in_row;
    return true;
}

// Phase 1 of the forward-packing of one unit (see the file comment): rows
// [m0, J), whose sources may still be overwritten, in ascending rounds.  A
// round stages up to kStageRows rows in the (now unused) selection scratch
// with asynchronous 16-byte copies, all in flight at once, waits for all of
// them, and only then stores the round.  Returns true if a row referenced a
// block id out of range (skipped).
__device__ bool pack_ordered_prefix(const int* sidx, int m0, int J, int s, int l, int h, const EvictParams& p,
                                    EvictSmem& sm) {
    const int32_t* bt = p.block_table + (int64_t)s * p.max_blocks;
    const int64_t layer_tiles = (int64_t)l * p.num_blocks;
    uint4* stage = reinterpret_cast<uint4*>(&sm.u);
    bool bad = false;
    for (int base = m0; base < J; base += kStageRows) {
        const int nsl = min(kStageRows, J - base) * kSlicesPerRow;
        for (int i = threadIdx.x; i < nsl; i += kEvictThreads) {
            SliceMove m;
            if (slice_move(sidx, base + i / kSlicesPerRow, i % kSlicesPerRow, bt, layer_tiles, p, h, m))
                cp_async16(stage + i, m.src);
            else
                bad = true;
        }
        cp_async_wait_all();
        __syncthreads();
        for (int i = threadIdx.x; i < nsl; i += kEvictThreads) {
            SliceMove m;
            if (slice_move(sidx, base + i / kSlicesPerRow, i % kSlicesPerRow, bt, layer_tiles, p, h, m))
                *reinterpret_cast<uint4*>(m.dst) = stage[i];
        }
        __syncthreads();
    }
    return bad;
}

__global__ void __launch_bounds__(kEvictThreads, 2) evict_kernel(const EvictParams p) {
    extern __shared__ __align__(128) uint8_t smem[];
    EvictSmem& sm = *reinterpret_cast<EvictSmem*>(smem);
    int* sidx = reinterpret_cast<int*>(smem + sizeof(EvictSmem));
    const int u = blockIdx.x;
    const int LH = p.L * p.Hkv;
    const int s = u / LH, rem = u % LH, l = rem / p.Hkv, h = rem % p.Hkv;
    const bool head0 = (l == 0 && h == 0);
    wait_prior_grid();
    if (p.abort_word && __ldcg(p.abort_word) != 0) return;    // vetoed step: change nothing
    int len = p.lens[s];
    if (len < 0 || (int64_t)len > (int64_t)p.max_blocks * kBlockRows) {
        if (threadIdx.x == 0) raise_flag(p.status, TRI_DEVFLAG_BOUNDS);
        return;
    }
    int kept;
    if (p.do_select) {
        if (len <= p.trigger) {
            // Nothing to evict.  A standalone selection reports every slot.
            if (!p.do_compact) {
                for (int j = threadIdx.x; j < p.budget; j += kEvictThreads)
                    p.idx_out[(int64_t)u * p.budget + j] = j < len ? j : -1;
                // kept = len; past the budget (a trigger above it) idx only
                // has room for the first budget slots
                if (head0 && threadIdx.x == 0) p.kept_out[s] = len;
            }
            return;
        }
        const float* sc = p.scores + (int64_t)u * p.score_stride;
        const bool have_range = p.unit_kmin != nullptr;
        select_unit(sc, len, p.budget, p.window, p.sinks, sidx, sm, p.status, have_range,
                    have_range ? p.unit_kmin[u] : 0u, have_range ? p.unit_kmax[u] : 0u);
        kept = p.budget;
        if (p.idx_out)
            for (int j = threadIdx.x; j < p.budget; j += kEvictThreads)
                p.idx_out[(int64_t)u * p.budget + j] = sidx[j];
        if (p.idx_copy)
            for (int j = threadIdx.x; j < p.budget; j += kEvictThreads)
                p.idx_copy[(int64_t)u * p.budget + j] = sidx[j];
        if (p.kept_out && head0 && threadIdx.x == 0) p.kept_out[s] = kept;
    } else {
        kept = p.kept_in[s];
        if (kept == len) return;     // every slot kept: nothing moves (also past the budget)
        if (kept < 0 || kept > len || kept > p.budget) {
            if (threadIdx.x == 0) raise_flag(p.status, TRI_DEVFLAG_BOUNDS);
            return;
        }
        bool bad = false;
        for (int j = threadIdx.x; j < kept; j += kEvictThreads) {
            const int v = p.idx_in[(int64_t)u * p.budget + j];
            sidx[j] = v;
            bad |= (v < 0 || v >= len);
        }
        __syncthreads();
        for (int j = threadIdx.x + 1; j < kept; j += kEvictThreads) bad |= (sidx[j] <= sidx[j - 1]);
        if (__syncthreads_or(bad)) {
            if (threadIdx.x == 0) raise_flag(p.status, TRI_DEVFLAG_BOUNDS);
            return;
        }
    }
    if (p.do_compact) {
        if (p.slot_pos) {
            // Positions travel with their rows: every kept position is read
            // into the (now idle) selection scratch before any is stored.
            int32_t* pos = p.slot_pos + (int64_t)u * p.pos_stride;
            int* stage = reinterpret_cast<int*>(&sm.u);
            for (int j = threadIdx.x; j < kept; j += kEvictThreads) stage[j] = pos[sidx[j]];
            __syncthreads();
            for (int j = threadIdx.x; j < kept; j += kEvictThreads) pos[j] = stage[j];
            __syncthreads();
        }
        int fixed = 0, low = 0;
        for (int j = threadIdx.x; j < kept; j += kEvictThreads) {
            fixed += (sidx[j] == j) ? 1 : 0;
            low += (sidx[j] < kept) ? 1 : 0;
        }
        const int m0 = block_sum(fixed, sm);     // idx_j == j exactly for j < m0
        const int J = block_sum(low, sm);        // idx_j < kept exactly for j < J
        // Rows [m0, J) read sources that compaction overwrites.  With a
        // scratch area and a short prefix they are copied out first
        // (copy-out kernel) and all rows then move independently (move
        // kernel); otherwise (a long prefix, or the scratch is full) this CTA
        // moves them in place in ordered rounds and the move kernel moves
        // only rows [J, kept).
        int mode = kModeInPlace, off = 0;
        const bool reserved = p.unit_info && J > m0 && (!p.many_units || J - m0 <= kScratchMaxRows);
        if (reserved) {
            if (threadIdx.x == 0) sm.bcast[0] = atomicAdd(p.scratch_used, J - m0);
            __syncthreads();
            off = sm.bcast[0];
            if (off + (J - m0) <= p.scratch_rows) mode = kModeScratch;
        }
        if (mode == kModeInPlace &&
            __syncthreads_or(pack_ordered_prefix(sidx, m0, J, s, l, h, p, sm)) && threadIdx.x == 0)
            raise_flag(p.status, TRI_DEVFLAG_BOUNDS);
        if (mode == kModeScratch) {
            for (int r = threadIdx.x; r < J - m0; r += kEvictThreads) {
                p.scratch_owner[off + r] = u;
                p.scratch_owner[p.scratch_rows + off + r] = sidx[m0 + r];
            }
        } else if (reserved) {
            // the reservation overflowed: its rows inside the scratch stay unowned
            for (int r = off + threadIdx.x; r < min(off + (J - m0), p.scratch_rows); r += kEvictThreads)
                p.scratch_owner[r] = -1;
        }
        if (p.unit_info && threadIdx.x == 0) {
            p.unit_info[4 * u + 0] = m0;
            p.unit_info[4 * u + 1] = J;
            p.unit_info[4 * u + 2] = mode;
            p.unit_info[4 * u + 3] = off;
        }
    }
    if (head0 && p.seq_len_out) {
        // Step bookkeeping: the sequence's new length and its freed blocks.
        const int32_t* bt = p.block_table + (int64_t)s * p.max_blocks;
        const int lo = (kept + kBlockRows - 1) / kBlockRows;
        const int hi = (len + kBlockRows - 1) / kBlockRows;
        const int off = p.freed_off[s];
        if (p.freed_ids)
            for (int e = threadIdx.x; e < hi - lo; e += kEvictThreads) p.freed_ids[off + e] = bt[lo + e];
        if (p.fl_ids) {
            const int base = __ldcg(p.fl_base);
            if (base >= 0)
                for (int e = threadIdx.x; e < hi - lo; e += kEvictThreads) p.fl_ids[base + off + e] = bt[lo + e];
        }
        if (threadIdx.x == 0) p.seq_len_out[s] = kept;
    }
}

// Phase 2 of the forward-packing, for every unit at once, in one of two
// roles (MoveParams::copy_out):
//   move:     rows j >= J take pool row idx_j (>= kept, a row no store of
//             this step touches); with per-unit plans, rows [m0, J) of units
//             in scratch mode take their copied-out source from the scratch;
//   copy-out: rows [m0, J) of units in scratch mode copy pool row idx_j to
//             scratch row (off + j - m0).
// A warp takes a tile of 32 consecutive rows of one unit: lane i resolves
// row i (its index, block ids, source and destination addresses of its K
// and V halves) with coalesced loads; the warp then moves the tile
// kMoveRows rows at a time, lanes 0-15 carrying the K half and 16-31 the V
// half, 16 bytes each, all loads of a batch before its stores.
// Copy-out role: warps take tiles of kMoveRows scratch rows; lane i < kMoveRows
// resolves scratch row t + i (its unit and source row, recorded by the
// selection), then the warp copies the tile in one batch.
__device__ void copy_out_rows(const MoveParams& p) {
    const int lane = threadIdx.x & 31;
    const int LH = p.L * p.Hkv;
    const int used = min(__ldcg(p.scratch_used), p.scratch_rows);
    const int warp0 = (int)(((int64_t)blockIdx.x * kMoveThreads + threadIdx.x) >> 5);
    const int nwarps = (int)(((int64_t)gridDim.x * kMoveThreads) >> 5);
    const int in_row = (lane & 15) * 16;
    bool bad = false;
    for (int t0 = warp0 * kMoveRows; t0 < used; t0 += nwarps * kMoveRows) {
        const int R = lane < kMoveRows ? t0 + lane : used;
        const uint8_t* sk = nullptr;
        const uint8_t* sv = nullptr;
        const int u = R < used ? __ldcg(p.scratch_owner + R) : -1;
        if (u >= 0) {
            const int src = __ldcg(p.scratch_owner + p.scratch_rows + R);
            const int s = u / LH, l = (u % LH) / p.Hkv, h = u % p.Hkv;
            int64_t so;
            if (src >= 0 && (int64_t)src < (int64_t)p.max_blocks * kBlockRows &&
                row_offset(p.block_table + (int64_t)s * p.max_blocks, src, (int64_t)l * p.num_blocks, p.Hkv, h,
                           p.num_blocks, so)) {
                sk = p.k_pool + so;
                sv = p.v_pool + so;
            } else {
                bad = true;
            }
        }
        uint32_t todo = __ballot_sync(0xffffffffu, sk != nullptr);
        while (todo) {
            uint4 buf[kMoveRows];
            int rows[kMoveRows];
#pragma unroll
            for (int k = 0; k < kMoveRows; ++k) {
                const int r = todo ? __ffs(todo) - 1 : -1;
                if (todo) todo &= todo - 1u;
                const int rr = r < 0 ? 0 : r;
                const unsigned long long s_k = __shfl_sync(0xffffffffu, (unsigned long long)sk, rr);
                const unsigned long long s_v = __shfl_sync(0xffffffffu, (unsigned long long)sv, rr);
                rows[k] = r;
                if (r >= 0)
                    buf[k] = __ldcg(reinterpret_cast<const uint4*>(
                        reinterpret_cast<const uint8_t*>(lane < 16 ? s_k : s_v) + in_row));
            }
#pragma unroll
            for (int k = 0; k < kMoveRows; ++k)
                if (rows[k] >= 0)
                    *reinterpret_cast<uint4*>(p.scratch + (int64_t)(t0 + rows[k]) * 2 * kRowBytes +
                                              (lane < 16 ? 0 : kRowBytes) + in_row) = buf[k];
        }
    }
    if (__any_sync(0xffffffffu, bad) && lane == 0) raise_flag(p.status, TRI_DEVFLAG_BOUNDS);
}

__global__ void __launch_bounds__(kMoveThreads, 3) move_kernel(const MoveParams p) {
    wait_prior_grid();
    if (p.abort_word && __ldcg(p.abort_word) != 0) return;    // vetoed step: move nothing
    if (p.copy_out) {
        copy_out_rows(p);
        return;
    }
    const int lane = threadIdx.x & 31;
    const int LH = p.L * p.Hkv;
    const int tiles_per_unit = (p.budget + 31) / 32;
    const int ntiles = p.S * LH * tiles_per_unit;
    const int warp0 = (int)(((int64_t)blockIdx.x * kMoveThreads + threadIdx.x) >> 5);
    const int nwarps = (int)(((int64_t)gridDim.x * kMoveThreads) >> 5);
    const int64_t max_len = (int64_t)p.max_blocks * kBlockRows;
    const int in_row = (lane & 15) * 16;
    bool bad = false;
    for (int tile = warp0; tile < ntiles; tile += nwarps) {
        const int u = tile / tiles_per_unit;
        const int j = (tile % tiles_per_unit) * 32 + lane;      // this lane's row
        const int s = u / LH, l = (u % LH) / p.Hkv, h = u % p.Hkv;
        const int len = p.lens[s];
        int kept = -1;
        if (len >= 0 && (int64_t)len <= max_len) {
            kept = p.kept ? p.kept[s] : (len > p.trigger ? p.budget : -1);
            if (kept > len || kept > p.budget) kept = -1;
        }
        const uint8_t* sk = nullptr;
        const uint8_t* sv = nullptr;
        uint8_t* dk = nullptr;
        uint8_t* dv = nullptr;
        if (kept > 0 && j < kept) {
            int m0 = 0, J = 0, mode = kModeInPlace, off = 0;
            if (p.unit_info) {
                m0 = __ldcg(p.unit_info + 4 * u + 0);
                J = __ldcg(p.unit_info + 4 * u + 1);
                mode = __ldcg(p.unit_info + 4 * u + 2);
                off = __ldcg(p.unit_info + 4 * u + 3);
            }
            const int32_t* bt = p.block_table + (int64_t)s * p.max_blocks;
            const int64_t lt = (int64_t)l * p.num_blocks;
            const int32_t* ui = p.idx + (int64_t)u * p.budget;
            const bool scratch_row = p.unit_info && mode == kModeScratch && j >= m0 && j < J;
            {
                const int src = __ldcg(ui + j);
                const bool pool_row = src >= kept && src < len && (j == 0 || __ldcg(ui + j - 1) < src);
                if (scratch_row || pool_row) {
                    int64_t dof;
                    if (row_offset(bt, j, lt, p.Hkv, h, p.num_blocks, dof)) {
                        if (scratch_row) {
                            sk = p.scratch + (int64_t)(off + j - m0) * 2 * kRowBytes;
                            sv = sk + kRowBytes;
                        } else {
                            int64_t so;
                            if (row_offset(bt, src, lt, p.Hkv, h, p.num_blocks, so)) {
                                sk = p.k_pool + so;
                                sv = p.v_pool + so;
                            } else {
                                bad = true;
                            }
                        }
                        if (sk) {
                            dk = p.k_pool + dof;
                            dv = p.v_pool + dof;
                        }
                    } else {
                        bad = true;
                    }
                }
            }
        }
        uint32_t todo = __ballot_sync(0xffffffffu, sk != nullptr);
        while (todo) {
            uint4 buf[kMoveRows];
            uint8_t* dst[kMoveRows];
#pragma unroll
            for (int k = 0; k < kMoveRows; ++k) {
                const int r = todo ? __ffs(todo) - 1 : -1;
                if (todo) todo &= todo - 1u;
                const int rr = r < 0 ? 0 : r;
                const unsigned long long s_k = __shfl_sync(0xffffffffu, (unsigned long long)sk, rr);
                const unsigned long long s_v = __shfl_sync(0xffffffffu, (unsigned long long)sv, rr);
                const unsigned long long d_k = __shfl_sync(0xffffffffu, (unsigned long long)dk, rr);
                const unsigned long long d_v = __shfl_sync(0xffffffffu, (unsigned long long)dv, rr);
                dst[k] = nullptr;
                if (r >= 0) {
                    const uint8_t* src = reinterpret_cast<const uint8_t*>(lane < 16 ? s_k : s_v);
                    buf[k] = __ldcg(reinterpret_cast<const uint4*>(src + in_row));
                    dst[k] = reinterpret_cast<uint8_t*>(lane < 16 ? d_k : d_v) + in_row;
                }
            }
#pragma unroll
            for (int k = 0; k < kMoveRows; ++k)
                if (dst[k]) *reinterpret_cast<uint4*>(dst[k]) = buf[k];
        }
    }
    if (__any_sync(0xffffffffu, bad) && lane == 0) raise_flag(p.status, TRI_DEVFLAG_BOUNDS);
}

constexpr int kFinalizeThreads = 256;

__global__ void __launch_bounds__(kFinalizeThreads) finalize_kernel(const FinalizeParams p) {
    __shared__ int warp_tmp[kFinalizeThreads / 32];
    __shared__ int c_off[kFinalizeThreads], c_cnt[kFinalizeThreads], c_lo[kFinalizeThreads];
    const int64_t max_len = (int64_t)p.max_blocks * kBlockRows;
    int carry = 0;
    for (int c0 = 0; c0 < p.S; c0 += kFinalizeThreads) {
        const int s = c0 + threadIdx.x;
        int nf = 0, lo = 0, kept = 0;
        bool valid = false;
        if (s < p.S) {
            const int len = p.seq_len[s];
            kept = p.kept[s];
            if (len < 0 || (int64_t)len > max_len || kept < 0 || kept > len) {
                raise_flag(p.status, TRI_DEVFLAG_BOUNDS);
            } else {
                valid = true;
                lo = (kept + kBlockRows - 1) / kBlockRows;
                nf = (len + kBlockRows - 1) / kBlockRows - lo;
            }
        }
        int tot;
        const int ex = block_exclusive_scan<kFinalizeThreads>(nf, warp_tmp, tot);
        c_off[threadIdx.x] = carry + ex;
        c_cnt[threadIdx.x] = nf;
        c_lo[threadIdx.x] = lo;
        __syncthreads();
        const int n_here = min(kFinalizeThreads, p.S - c0);
        for (int k = 0; k < n_here; ++k) {
            const int32_t* bt = p.block_table + (int64_t)(c0 + k) * p.max_blocks + c_lo[k];
            for (int e = threadIdx.x; e < c_cnt[k]; e += kFinalizeThreads) p.freed_ids[c_off[k] + e] = bt[e];
        }
        if (valid) p.seq_len[s] = kept;
        carry += tot;
        __syncthreads();
    }
    if (threadIdx.x == 0) *p.freed_count = carry;
}

// Blocks newly needed by sequence s to grow by n slots (0 if invalid).
__device__ __forceinline__ int blocks_needed(int len, int n, int64_t max_len, bool& bad) {
    if (len < 0 || n < 0 || (int64_t)len + n > max_len) {
        bad = true;
        return 0;
    }
    return (int)(((int64_t)len + n + kBlockRows - 1) / kBlockRows - ((int64_t)len + kBlockRows - 1) / kBlockRows);
}

// One CTA: pop the blocks all sequences need from the top of the free list
// (all or nothing) and write them into the block table.
__global__ void __launch_bounds__(kFinalizeThreads) reserve_kernel(const ReserveParams p) {
    __shared__ int warp_tmp[kFinalizeThreads / 32];
    const int64_t max_len = (int64_t)p.max_blocks * kBlockRows;
    bool bad = false;
    int total = 0;
    for (int c0 = 0; c0 < p.S; c0 += kFinalizeThreads) {
        const int s = c0 + threadIdx.x;
        const int need = s < p.S ? blocks_needed(p.seq_len[s], p.n_new[s], max_len, bad) : 0;
        int tot;
        block_exclusive_scan<kFinalizeThreads>(need, warp_tmp, tot);
        total += tot;
    }
    if (__syncthreads_or(bad)) {
        if (threadIdx.x == 0) raise_flag(p.status, TRI_DEVFLAG_BOUNDS);
        return;
    }
    const int have = *p.fl_count;
    if (have > p.fl_capacity) {
        if (threadIdx.x == 0) raise_flag(p.status, TRI_DEVFLAG_BOUNDS);
        return;
    }
    if (have < 0 || total > have) {
        if (threadIdx.x == 0) raise_flag(p.status, TRI_DEVFLAG_FREELIST);
        return;
    }
    const int base = have - total;
    bool bad_id = false;
    for (int e = base + threadIdx.x; e < have; e += kFinalizeThreads) {
        const int b = p.fl_ids[e];
        bad_id |= (b < 0 || b >= p.num_blocks);
    }
    if (__syncthreads_or(bad_id)) {
        if (threadIdx.x == 0) raise_flag(p.status, TRI_DEVFLAG_BOUNDS);
        return;
    }
    int carry = 0;
    for (int c0 = 0; c0 < p.S; c0 += kFinalizeThreads) {
        const int s = c0 + threadIdx.x;
        bool unused = false;
        int need = 0, lo = 0;
        if (s < p.S) {
            const int len = p.seq_len[s];
            need = blocks_needed(len, p.n_new[s], max_len, unused);
            lo = (len + kBlockRows - 1) / kBlockRows;
        }
        int tot;
        const int ex = block_exclusive_scan<kFinalizeThreads>(need, warp_tmp, tot);
        for (int e = 0; e < need; ++e)
            p.block_table[(int64_t)s * p.max_blocks + lo + e] = p.fl_ids[base + carry + ex + e];
        carry += tot;
    }
    __syncthreads();
    if (threadIdx.x == 0) *p.fl_count = base;
}

}  // namespace

cudaError_t launch_reserve(const ReserveParams& p, cudaStream_t stream) {
    reserve_kernel<<<1, kFinalizeThreads, 0, stream>>>(p);
    return cudaGetLastError();
}

cudaError_t launch_evict(const EvictParams& p, cudaStream_t stream, bool pdl) {
    const int U = p.S * p.L * p.Hkv;
    if (U == 0) return cudaSuccess;
    const size_t smem = sizeof(EvictSmem) + (size_t)p.budget * sizeof(int);
    cudaError_t e = cudaFuncSetAttribute(evict_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    return launch_kernel(evict_kernel, dim3(U), dim3(kEvictThreads), smem, stream, pdl, p);
}

cudaError_t launch_move(const MoveParams& p, int num_sms, cudaStream_t stream, bool pdl) {
    const int64_t tiles = p.copy_out ? ((int64_t)p.scratch_rows + kMoveRows - 1) / kMoveRows
                                     : (int64_t)p.S * p.L * p.Hkv * ((p.budget + 31) / 32);
    if (tiles == 0) return cudaSuccess;
    if (tiles > INT_MAX) return cudaErrorInvalidValue;
    int64_t grid = (tiles + kMoveThreads / 32 - 1) / (kMoveThreads / 32);
    if (grid > (int64_t)num_sms * 3) grid = (int64_t)num_sms * 3;
    return launch_kernel(move_kernel, dim3((unsigned)grid), dim3(kMoveThreads), 0, stream, pdl, p);
}

cudaError_t launch_finalize(const FinalizeParams& p, cudaStream_t stream) {
    finalize_kernel<<<1, kFinalizeThreads, 0, stream>>>(p);
    return cudaGetLastError();
}

}  // namespace tri
