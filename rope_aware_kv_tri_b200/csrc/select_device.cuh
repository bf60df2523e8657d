// select_device.cuh - the per-unit top-B selection and the ordered in-place
// packing of a unit's at-risk rows, for a CTA (or a named group of NT
// threads of a CTA, threadIdx.x < NT) working on one unit.
//
// Pages: "TriAttention: Trigonometric KV Compression for Efficient Long
// Reasoning" - "Core Mechanism" (rank keys and keep only the top-scoring
// subset); "TriAttention: How a Geometric Trick Cuts LLM Memory Use by 10x
// Without Losing Accuracy" - "Solving the Memory Fragmentation Problem"
// (survivors move forward so tail blocks empty out).
//
// Selection of len slots, budget B, window W (len > B): the last W slots are
// kept; among the first cand = len - W the take = B - W best by (score desc,
// slot asc).  Scores become 32-bit keys whose unsigned order is the score
// order (order_key: -0 == +0, NaN == -inf).  With the unit's score range
// known, a linear histogram over that range finds the bucket of the cut;
// the candidates above that bucket go to a bitmap and the bucket's (key,
// slot) pairs to a shared list; the exact cut key and its tie count come
// from the list, and the kept slots are emitted from the bitmaps in slot
// order.  Without a usable range (NaN, or a cut bucket too full) the exact
// cut is found with radix passes over the top 12 and then 10 + 10 key bits,
// and the kept slots are emitted by a ballot walk.  Either way the result is
// unique: ties go to the lower slot.
//
// Every barrier is the named barrier kSelBarrier over NT threads, so the
// same code serves a whole CTA (the selection kernel, NT = its size) and the
// NT consumer threads of the fused step kernel while its producer warp
// waits elsewhere.  Scores are read through L2 (ld.global.cg): in the fused
// kernel they were written by other SMs during the same launch.
#pragma once

#include "tri_device.cuh"
#include "tri_internal.h"

namespace tri {

namespace {

constexpr int kSelBarrier = 1;     // named barrier of the selection group

template <int NT>
__device__ __forceinline__ void sel_sync() {
    asm volatile("bar.sync %0, %1;" ::"n"(kSelBarrier), "n"(NT) : "memory");
}

// Barrier of the selection group that also ORs a predicate over it.
template <int NT>
__device__ __forceinline__ int sel_sync_or(int pred) {
    int r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t"
        "setp.ne.s32 p, %1, 0;\n\t"
        "bar.red.or.pred q, %2, %3, p;\n\t"
        "selp.s32 %0, 1, 0, q;\n\t}"
        : "=r"(r)
        : "r"(pred), "n"(kSelBarrier), "n"(NT)
        : "memory");
    return r;
}

// Exclusive prefix sum over the selection group (two barriers).
template <int NT>
__device__ __forceinline__ int sel_scan(int v, int* warp_tmp, int& total) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    int x = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
    }
    if (lane == 31) warp_tmp[warp] = x;
    sel_sync<NT>();
    int before = 0, tot = 0;
#pragma unroll
    for (int w = 0; w < NT / 32; ++w) {
        const int c = warp_tmp[w];
        before += (w < warp) ? c : 0;
        tot += c;
    }
    sel_sync<NT>();
    total = tot;
    return before + x - v;
}

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
template <int NT>
struct EvictSmem {
    static constexpr int kWarps = NT / 32;
    union {
        SelectScratch sel;
    } u;
    static_assert(sizeof(OnePassScratch) <= 100 * 1024, "one-pass scratch too large");
    int warp_a[kWarps];      // keys > thr in the segment (part 1)
    int warp_b[kWarps];      // keys == thr in the segment
    int warp_c[kWarps];      // keys > thr in the segment (part 2)
    int eq_before[kWarps];
    int keep_before[kWarps];
    int scan_tmp[kWarps];    // scratch of block scans
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

template <int NT>
__device__ __forceinline__ int block_sum(int v, EvictSmem<NT>& sm) {
    int total;
    sel_scan<NT>(v, sm.scan_tmp, total);
    return total;
}

// The bin of `hist` (nb bins, nb >= 512, higher bin = higher value) that
// holds the rem-th largest counted element; rem becomes its rank in the bin.
template <int NT>
__device__ int pick_bin(const int* hist, int nb, int& rem, EvictSmem<NT>& sm) {
    const int per = nb / NT;
    const int b0 = threadIdx.x * per;
    int local = 0;
    for (int j = 0; j < per; ++j) local += hist[b0 + j];
    int total;
    const int ex = sel_scan<NT>(local, sm.scan_tmp, total);
    int run = total - ex - local;      // elements in bins above this thread's bins
    for (int j = per - 1; j >= 0; --j) {
        const int h = hist[b0 + j];
        if (run < rem && rem <= run + h) {
            sm.bcast[0] = b0 + j;
            sm.bcast[1] = rem - run;
        }
        run += h;
    }
    sel_sync<NT>();
    const int bin = sm.bcast[0];
    rem = sm.bcast[1];
    sel_sync<NT>();
    return bin;
}

// Pick the digit of the histogram `hist` (nb bins) in which the rem-th
// largest counted key lies; update (prefix, mask, rem).
template <int NT>
__device__ void pick_digit(const int* hist, int nb, int shift, uint32_t& prefix, uint32_t& mask, int& rem,
                           EvictSmem<NT>& sm) {
    const int d = pick_bin<NT>(hist, nb, rem, sm);
    prefix |= (uint32_t)d << shift;
    mask |= (uint32_t)(nb - 1) << shift;
}

// Pass 1: histogram of the top key bits of candidates [lo, cand).  Returns
// whether a NaN score was seen.
template <int NT>
__device__ bool top_histogram(const float* __restrict__ sc, int cand, int lo, int* hist) {
    for (int i = threadIdx.x; i < kTopBins; i += NT) hist[i] = 0;
    sel_sync<NT>();
    bool nan_seen = false;
    const int nvec = cand >> 2;
    const float4* v4 = reinterpret_cast<const float4*>(sc);
    for (int v0 = threadIdx.x; v0 < nvec; v0 += NT * kUnroll) {
        float4 x[kUnroll];
#pragma unroll
        for (int k = 0; k < kUnroll; ++k) {
            const int v = v0 + k * NT;
            x[k] = v < nvec ? __ldcg(v4 + v) : make_float4(0.f, 0.f, 0.f, 0.f);
        }
#pragma unroll
        for (int k = 0; k < kUnroll; ++k) {
            if (v0 + k * NT < nvec) {
                const float e[4] = {x[k].x, x[k].y, x[k].z, x[k].w};
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    if (4 * (v0 + k * NT) + c >= lo) {
                        nan_seen |= isnan(e[c]);
                        atomicAdd(&hist[order_key(e[c]) >> kTopShift], 1);
                    }
                }
            }
        }
    }
    for (int t = max(4 * nvec, lo) + threadIdx.x; t < cand; t += NT) {
        const float e = __ldcg(sc + t);
        nan_seen |= isnan(e);
        atomicAdd(&hist[order_key(e) >> kTopShift], 1);
    }
    return sel_sync_or<NT>(nan_seen) != 0;
}

// Load the 4 scores of slots t..t+3 of a warp step (those >= end invalid).
__device__ __forceinline__ void load4(const float* __restrict__ sc, int t, int end, float (&x)[4]) {
    if (t + 3 < end) {
        const float4 v = __ldcg(reinterpret_cast<const float4*>(sc + t));
        x[0] = v.x; x[1] = v.y; x[2] = v.z; x[3] = v.w;
    } else {
#pragma unroll
        for (int c = 0; c < 4; ++c) x[c] = (t + c < end) ? __ldcg(sc + t + c) : 0.f;
    }
}

// Streaming radix pass over all candidates (fallback when the cut's bucket
// does not fit the shared list).
template <int NT>
__device__ void stream_radix_pass(const float* __restrict__ sc, int cand, int lo, uint32_t& prefix, uint32_t& mask,
                                  int& rem, int shift, int bits, int* hist, EvictSmem<NT>& sm) {
    const int nb = 1 << bits;
    const uint32_t dmask = (uint32_t)nb - 1u;
    for (int i = threadIdx.x; i < nb; i += NT) hist[i] = 0;
    sel_sync<NT>();
    for (int t = lo + threadIdx.x; t < cand; t += NT) {
        const uint32_t key = order_key(__ldcg(sc + t));
        if ((key & mask) == prefix) atomicAdd(&hist[(key >> shift) & dmask], 1);
    }
    sel_sync<NT>();
    pick_digit<NT>(hist, nb, shift, prefix, mask, rem, sm);
}

// Radix pass over the shared list of boundary-bucket keys.
template <int NT>
__device__ void list_radix_pass(const uint32_t* keys, int n, uint32_t& prefix, uint32_t& mask, int& rem,
                                int shift, int bits, int* hist, EvictSmem<NT>& sm) {
    const int nb = 1 << bits;
    const uint32_t dmask = (uint32_t)nb - 1u;
    for (int i = threadIdx.x; i < nb; i += NT) hist[i] = 0;
    sel_sync<NT>();
    for (int i = threadIdx.x; i < n; i += NT) {
        const uint32_t key = keys[i];
        if ((key & mask) == prefix) atomicAdd(&hist[(key >> shift) & dmask], 1);
    }
    sel_sync<NT>();
    pick_digit<NT>(hist, nb, shift, prefix, mask, rem, sm);
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

// Linear bucket of score x in [lo, lo + (nb-1)/scale] (nb buckets); monotone in x.
__device__ __forceinline__ int lin_bucket(float x, float lo, float scale, int nb = kLinBins) {
    const int b = (int)((x - lo) * scale);
    return b < 0 ? 0 : (b > nb - 1 ? nb - 1 : b);
}

// Emit the set bits of `bits` (nwords words, slot 32w + b) into sidx in
// ascending order, at most `take` of them.  Each warp takes a contiguous run
// of words.  A dense run (more than a quarter of its bits set) is walked
// four words per step, lane i testing bit i, so every lane stores at once; a
// sparse run is walked 64 words per step, lane i owning words 2i and 2i + 1:
// a warp scan of their bit counts gives each lane its first output slot and
// the lane stores its own set bits in order.
template <int NT>
__device__ void emit_kept(const uint32_t* bits, int nwords, int take, int* sidx, EvictSmem<NT>& sm) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int per = (nwords + (NT / 32) - 1) / (NT / 32);
    const int w0 = min(warp * per, nwords), w1 = min(w0 + per, nwords);
    int cnt = 0;
    for (int w = w0 + lane; w < w1; w += 32) cnt += __popc(bits[w]);
    cnt = __reduce_add_sync(0xffffffffu, cnt);
    if (lane == 0) sm.warp_a[warp] = cnt;
    sel_sync<NT>();
    int base = 0;
    for (int k = 0; k < warp; ++k) base += sm.warp_a[k];
    if (4 * cnt > 32 * (w1 - w0)) {
        // four words per step: their loads do not wait on the running count
        const uint32_t lt = lanemask_lt();
        for (int w = w0; w < w1; w += 4) {
            uint32_t kw[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) kw[i] = w + i < w1 ? bits[w + i] : 0u;
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int pos = base + __popc(kw[i] & lt);
                if (((kw[i] >> lane) & 1u) && pos < take) sidx[pos] = (w + i) * 32 + lane;
                base += __popc(kw[i]);
            }
        }
    } else {
        for (int c0 = w0; c0 < w1; c0 += 64) {
            const int wa = c0 + 2 * lane;
            uint32_t a = wa < w1 ? bits[wa] : 0u;
            uint32_t b = wa + 1 < w1 ? bits[wa + 1] : 0u;
            const int n = __popc(a) + __popc(b);
            int incl = n;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int y = __shfl_up_sync(0xffffffffu, incl, o);
                if (lane >= o) incl += y;
            }
            int pos = base + incl - n;
            for (; a; a &= a - 1u, ++pos)
                if (pos < take) sidx[pos] = wa * 32 + (__ffs(a) - 1);
            for (; b; b &= b - 1u, ++pos)
                if (pos < take) sidx[pos] = (wa + 1) * 32 + (__ffs(b) - 1);
            base += __shfl_sync(0xffffffffu, incl, 31);
        }
    }
    sel_sync<NT>();
}

// The cut from the list of the cut bucket's keys (rem = the cut's rank in
// the bucket), then the kept candidates from the bitmaps: gt_bits holds the
// candidates above the bucket; the list's keys above the cut join them, the
// ones equal to it go to eq_bits, of which the first need_eq in slot order
// are kept.  Emits the take kept slots ascending into sidx.
template <int NT>
__device__ void finish_from_list(const uint32_t* list_key, const int* list_slot, int n, int rem, uint32_t* gt_bits,
                                 uint32_t* eq_bits, int nwords, int take, int* sidx, int* hist, EvictSmem<NT>& sm) {
    uint32_t thr;
    int need_eq;
    if (n <= kRankListMax) {
        // the cut key is the list key with (#greater) < rem <= (#greater-or-equal)
        for (int i = threadIdx.x; i < n; i += NT) {
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
        sel_sync<NT>();
        thr = (uint32_t)sm.bcast[2];
        need_eq = sm.bcast[3];
    } else {
        uint32_t prefix = 0, mask = 0;
        list_radix_pass<NT>(list_key, n, prefix, mask, rem, 21, 11, hist, sm);
        list_radix_pass<NT>(list_key, n, prefix, mask, rem, 10, 11, hist, sm);
        list_radix_pass<NT>(list_key, n, prefix, mask, rem, 0, 10, hist, sm);
        thr = prefix;
        need_eq = rem;
    }
    for (int i = threadIdx.x; i < n; i += NT) {
        const uint32_t key = list_key[i];
        const int t = list_slot[i];
        if (key > thr) atomicOr(&gt_bits[t >> 5], 1u << (t & 31));
        else if (key == thr) atomicOr(&eq_bits[t >> 5], 1u << (t & 31));
    }
    sel_sync<NT>();
    // Emission: each thread owns a run of words; the first need_eq tied
    // candidates in slot order are kept.
    const int wpt = (nwords + NT - 1) / NT;
    const int w0 = min(threadIdx.x * wpt, nwords), w1 = min(w0 + wpt, nwords);
    int my_eq = 0;
    for (int w = w0; w < w1; ++w) my_eq += __popc(eq_bits[w]);
    int tot;
    int eq_before = sel_scan<NT>(my_eq, sm.scan_tmp, tot);
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
    sel_sync<NT>();
    emit_kept<NT>(gt_bits, nwords, take, sidx, sm);
}

// One streaming pass (cand <= kCodeSlots): the histogram pass also keeps
// every candidate's linear bucket in shared memory; the bitmap of buckets
// above the cut's and the cut bucket's slots then come from shared memory,
// and only the (few) cut-bucket scores are read again.
template <int NT>
__device__ bool select_one_pass(const float* __restrict__ sc, int cand, int first, int take, float lo, float span,
                                int* sidx, EvictSmem<NT>& sm) {
    // about 4 candidates per bucket at most, 512 to kLinBins buckets: a short
    // unit zeroes and scans fewer buckets
    int nb = 512;
    while (nb < kLinBins && 4 * nb < cand) nb <<= 1;
    const float scale = (float)(nb - 1) / span;
    OnePassScratch& o = sm.u.sel.one;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    for (int i = threadIdx.x; i < nb; i += NT) o.hist[i] = 0;
    sel_sync<NT>();
    const int nvec = cand >> 2;
    const float4* v4 = reinterpret_cast<const float4*>(sc);
    for (int v0 = threadIdx.x; v0 < nvec; v0 += NT * kUnroll) {
        float4 x[kUnroll];
#pragma unroll
        for (int k = 0; k < kUnroll; ++k) {
            const int v = v0 + k * NT;
            x[k] = v < nvec ? __ldcg(v4 + v) : make_float4(0.f, 0.f, 0.f, 0.f);
        }
#pragma unroll
        for (int k = 0; k < kUnroll; ++k) {
            const int v = v0 + k * NT;
            if (v < nvec) {
                const int b0 = lin_bucket(x[k].x, lo, scale, nb), b1 = lin_bucket(x[k].y, lo, scale, nb);
                const int b2 = lin_bucket(x[k].z, lo, scale, nb), b3 = lin_bucket(x[k].w, lo, scale, nb);
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
    for (int t = 4 * nvec + threadIdx.x; t < cand; t += NT) {
        const int b = lin_bucket(__ldcg(sc + t), lo, scale, nb);
        o.code[t] = (uint16_t)b;
        if (t >= first) atomicAdd(&o.hist[b], 1);
    }
    sel_sync<NT>();
    int rem = take;
    const int bstar = pick_bin<NT>(o.hist, nb, rem, sm);
    if (o.hist[bstar] > kOneListCap) return false;
    const int nwords = (cand + 31) / 32;
    for (int w = threadIdx.x; w < nwords; w += NT) o.eq_bits[w] = 0u;
    if (threadIdx.x == 0) sm.n_list = 0;
    sel_sync<NT>();
    // 8 buckets per 16-byte load; 4 lanes make one 32-slot word.  Two codes
    // (< 2^15) are compared per 32-bit add: code + (0x8000 - bstar - 1) has
    // bit 15 of its halfword set exactly when code > bstar, and no carry
    // reaches the other halfword.  The vectors holding slots outside
    // [first, cand) (at most the first and the last) are tested one slot at
    // a time, since codes past the last candidate were never written.
    const int nq = (cand + 7) / 8;
    const uint32_t k_gt = (uint32_t)(0x8000 - bstar - 1) * 0x00010001u;
    const uint32_t k_ge = (uint32_t)(0x8000 - bstar) * 0x00010001u;
    for (int q0 = warp * 32; q0 < nq; q0 += (NT / 32) * 32) {
        const int q = q0 + lane;
        uint32_t m = 0u;
        if (q < nq) {
            const uint4 c4 = *reinterpret_cast<const uint4*>(&o.code[8 * q]);
            const uint32_t cw[4] = {c4.x, c4.y, c4.z, c4.w};
            uint32_t eq = 0u;
            if (8 * q >= first && 8 * q + 8 <= cand) {
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const uint32_t g = (cw[j] + k_gt) & 0x80008000u;
                    const uint32_t e = ((cw[j] + k_ge) & 0x80008000u) & ~g;
                    m |= ((g >> 15) & 1u) << (2 * j) | (g >> 31) << (2 * j + 1);
                    eq |= ((e >> 15) & 1u) << (2 * j) | (e >> 31) << (2 * j + 1);
                }
            } else {
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const int t = 8 * q + i;
                    const int b = (int)((cw[i >> 1] >> (16 * (i & 1))) & 0xffffu);
                    if (t < cand && t >= first) {
                        if (b > bstar) m |= 1u << i;
                        else if (b == bstar) eq |= 1u << i;
                    }
                }
            }
            for (; eq; eq &= eq - 1u) {
                const int pos = atomicAdd(&sm.n_list, 1);
                if (pos < kOneListCap) o.list_slot[pos] = 8 * q + (__ffs(eq) - 1);
            }
        }
        uint32_t word = m << (8 * (lane & 3));
        word |= __shfl_xor_sync(0xffffffffu, word, 1);
        word |= __shfl_xor_sync(0xffffffffu, word, 2);
        if ((lane & 3) == 0 && q < nq) o.gt_bits[q >> 2] = word;
    }
    sel_sync<NT>();
    const int n = min(sm.n_list, kOneListCap);
    for (int i = threadIdx.x; i < n; i += NT) o.list_key[i] = order_key(__ldcg(sc + o.list_slot[i]));
    sel_sync<NT>();
    finish_from_list<NT>(o.list_key, o.list_slot, n, rem, o.gt_bits, o.eq_bits, nwords, take, sidx, o.hist, sm);
    return true;
}

// Selection over a known score range [kmin, kmax] (order keys): a linear
// histogram finds the bucket of the cut; the candidates above that bucket go
// to a bitmap and the bucket's (key, slot) pairs to a list; the exact cut
// key and its tie count come from the list; the kept slots are then emitted
// from the bitmaps in slot order.  Returns false, with nothing kept, when the
// range is not finite, the candidates exceed the bitmap, or the cut's
// bucket exceeds the list.
template <int NT>
__device__ bool select_linear(const float* __restrict__ sc, int cand, int first, int take, uint32_t kmin,
                              uint32_t kmax, int* sidx, EvictSmem<NT>& sm) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const float lo = key_value(kmin), hi = key_value(kmax);
    if (kmin > kmax || !isfinite(lo) || !isfinite(hi) || cand > kBitmapWords * 32) return false;
    const float span = hi - lo;
    if (!isfinite(span)) return false;
    if (span == 0.f) {
        // every score of the unit is equal: the lowest slots win every tie
        for (int j = threadIdx.x; j < take; j += NT) sidx[j] = first + j;
        return true;
    }
    if (cand <= kCodeSlots) return select_one_pass<NT>(sc, cand, first, take, lo, span, sidx, sm);
    const float scale = (float)(kLinBins - 1) / span;
    int* hist = sm.u.sel.hist;
    // warp segments of whole 128-slot steps
    const int seg = ((cand + (NT / 32) - 1) / (NT / 32) + kStep - 1) / kStep * kStep;
    const int beg = min(warp * seg, cand);
    const int end = min(beg + seg, cand);

    // Pass 1: linear histogram (16-byte loads, kUnroll per thread in flight).
    for (int i = threadIdx.x; i < kLinBins; i += NT) hist[i] = 0;
    sel_sync<NT>();
    {
        const int nvec = cand >> 2;
        const float4* v4 = reinterpret_cast<const float4*>(sc);
        for (int v0 = threadIdx.x; v0 < nvec; v0 += NT * kUnroll) {
            float4 x[kUnroll];
#pragma unroll
            for (int k = 0; k < kUnroll; ++k) {
                const int v = v0 + k * NT;
                x[k] = v < nvec ? __ldcg(v4 + v) : make_float4(0.f, 0.f, 0.f, 0.f);
            }
#pragma unroll
            for (int k = 0; k < kUnroll; ++k) {
                const int t = 4 * (v0 + k * NT);
                if (v0 + k * NT < nvec) {
                    if (t + 0 >= first) atomicAdd(&hist[lin_bucket(x[k].x, lo, scale)], 1);
                    if (t + 1 >= first) atomicAdd(&hist[lin_bucket(x[k].y, lo, scale)], 1);
                    if (t + 2 >= first) atomicAdd(&hist[lin_bucket(x[k].z, lo, scale)], 1);
                    if (t + 3 >= first) atomicAdd(&hist[lin_bucket(x[k].w, lo, scale)], 1);
                }
            }
        }
        for (int t = max(4 * nvec, first) + threadIdx.x; t < cand; t += NT)
            atomicAdd(&hist[lin_bucket(__ldcg(sc + t), lo, scale)], 1);
    }
    sel_sync<NT>();
    int rem = take;
    const int bstar = pick_bin<NT>(hist, kLinBins, rem, sm);
    if (hist[bstar] > kListCap) return false;

    // Pass 2: bitmap of candidates above the cut's bucket; list of the bucket.
    const int nwords = (cand + 31) / 32;
    for (int w = threadIdx.x; w < nwords; w += NT) sm.u.sel.two.eq_bits[w] = 0u;
    if (threadIdx.x == 0) sm.n_list = 0;
    sel_sync<NT>();
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
    sel_sync<NT>();
    const int n = min(sm.n_list, kListCap);
    finish_from_list<NT>(sm.u.sel.two.list_key, sm.u.sel.two.list_slot, n, rem, sm.u.sel.two.gt_bits,
                     sm.u.sel.two.eq_bits, nwords, take, sidx, hist, sm);
    return true;
}

// Smallest and largest order key among the candidates (block reduction).
template <int NT>
__device__ void candidate_key_range(const float* __restrict__ sc, int cand, int first, uint32_t& kmin,
                                    uint32_t& kmax, EvictSmem<NT>& sm) {
    uint32_t lo = 0xffffffffu, hi = 0u;
    const int nvec = cand >> 2;
    const float4* v4 = reinterpret_cast<const float4*>(sc);
    for (int v0 = threadIdx.x; v0 < nvec; v0 += NT * kUnroll) {
        float4 x[kUnroll];
#pragma unroll
        for (int k = 0; k < kUnroll; ++k) {
            const int v = v0 + k * NT;
            x[k] = v < nvec ? __ldcg(v4 + v) : make_float4(0.f, 0.f, 0.f, 0.f);
        }
#pragma unroll
        for (int k = 0; k < kUnroll; ++k) {
            const int t = 4 * (v0 + k * NT);
            if (v0 + k * NT < nvec) {
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
    for (int t = max(4 * nvec, first) + threadIdx.x; t < cand; t += NT) {
        const uint32_t k = order_key(__ldcg(sc + t));
        lo = min(lo, k);
        hi = max(hi, k);
    }
    lo = __reduce_min_sync(0xffffffffu, lo);
    hi = __reduce_max_sync(0xffffffffu, hi);
    __shared__ uint32_t wlo[(NT / 32)], whi[(NT / 32)];
    if ((threadIdx.x & 31) == 0) {
        wlo[threadIdx.x >> 5] = lo;
        whi[threadIdx.x >> 5] = hi;
    }
    sel_sync<NT>();
    kmin = 0xffffffffu;
    kmax = 0u;
    for (int w = 0; w < (NT / 32); ++w) {
        kmin = min(kmin, wlo[w]);
        kmax = max(kmax, whi[w]);
    }
    sel_sync<NT>();
}

// Kept slots of a unit of len > budget slots: [0, sinks), the best
// budget - window - sinks of [sinks, len - window), and the last window.
// The ranking passes run on a 16-byte aligned view that starts at slot
// a = sinks rounded down to a multiple of 4; the first (sinks - a) slots of
// the view are excluded, and the view's slot numbers are shifted back by a.
// kmin_in: whether (kmin, kmax) already bound the unit's score keys.
template <int NT>
__device__ void select_unit(const float* __restrict__ sc_unit, int len, int budget, int window, int sinks,
                            int* sidx_unit, EvictSmem<NT>& sm, int32_t* status, bool kmin_in, uint32_t kmin,
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
        if (!kmin_in) candidate_key_range<NT>(sc, cand, first, kmin, kmax, sm);
        done = select_linear<NT>(sc, cand, first, take, kmin, kmax, sidx, sm);
    }
    if (!done) {
        int* hist = sm.u.sel.hist;
        // warp segments: multiples of 128 slots so every step is float4-aligned
        const int seg = ((cand + (NT / 32) - 1) / (NT / 32) + kStep - 1) / kStep * kStep;
        const int beg = min(warp * seg, cand);
        const int end = min(beg + seg, cand);

        if (top_histogram<NT>(sc, cand, first, hist) && threadIdx.x == 0) raise_flag(status, TRI_DEVFLAG_NONFINITE);
        uint32_t prefix = 0, mask = 0;
        int rem = take;
        pick_digit<NT>(hist, kTopBins, kTopShift, prefix, mask, rem, sm);
        const uint32_t top = prefix >> kTopShift;
        const int in_bucket = hist[top];
        if (threadIdx.x == 0) sm.n_list = 0;
        sel_sync<NT>();

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
            sel_sync<NT>();
            const int n = min(sm.n_list, kListCap);
            list_radix_pass<NT>(sm.u.sel.two.list_key, n, prefix, mask, rem, 10, 10, hist, sm);
            list_radix_pass<NT>(sm.u.sel.two.list_key, n, prefix, mask, rem, 0, 10, hist, sm);
            if (threadIdx.x < (NT / 32)) {
                sm.warp_b[threadIdx.x] = 0;
                sm.warp_c[threadIdx.x] = 0;
            }
            sel_sync<NT>();
            for (int i = threadIdx.x; i < n; i += NT) {
                const uint32_t key = sm.u.sel.two.list_key[i];
                const int w = sm.u.sel.two.list_slot[i] / seg;
                if (key > prefix) atomicAdd(&sm.warp_c[w], 1);
                else if (key == prefix) atomicAdd(&sm.warp_b[w], 1);
            }
        } else {
            // Fallback: stream the remaining bits, then count per segment.
            stream_radix_pass<NT>(sc, cand, first, prefix, mask, rem, 10, 10, hist, sm);
            stream_radix_pass<NT>(sc, cand, first, prefix, mask, rem, 0, 10, hist, sm);
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
        sel_sync<NT>();
        const uint32_t thr = prefix;
        const int need_eq = rem;
        if (threadIdx.x == 0) {
            int eb = 0, kb = 0;
            for (int w = 0; w < (NT / 32); ++w) {
                const int gt_w = sm.warp_a[w] + sm.warp_c[w], eq_w = sm.warp_b[w];
                sm.eq_before[w] = eb;
                sm.keep_before[w] = kb;
                const int left = need_eq - eb;
                kb += gt_w + (left <= 0 ? 0 : (left < eq_w ? left : eq_w));
                eb += eq_w;
            }
        }
        sel_sync<NT>();
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
    sel_sync<NT>();
    if (a > 0)
        for (int j = threadIdx.x; j < take; j += NT) sidx[j] += a;
    for (int j = threadIdx.x; j < sinks; j += NT) sidx_unit[j] = j;
    for (int j = threadIdx.x; j < window; j += NT) sidx[take + j] = a + cand + j;
    sel_sync<NT>();
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

template <int NT, typename P>
__device__ __forceinline__ bool slice_move(const int* sidx, int j, int part, const int32_t* bt, int64_t layer_tiles,
                                           const P& p, int h, SliceMove& m) {
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

// The ordered in-place packing of a unit's at-risk prefix: rows [m0, J),
// whose sources may still be overwritten, in ascending rounds.  A round
// stages up to kStageRows rows in the (now unused) selection scratch with
// asynchronous 16-byte copies, all in flight at once, waits for all of them,
// and only then stores the round.  Round r reads rows >= its own first row,
// which no earlier round writes, and its stores land on rows that only
// rounds <= r read.  (Issuing round r + 1's copies before round r's stores
// is also correct, but at half the round size it doubles the number of
// latency-bound rounds and measured slower.)  Returns true if a row
// referenced a block id out of range (skipped).
template <int NT, typename P>
__device__ bool pack_ordered_prefix(const int* sidx, int m0, int J, int s, int l, int h, const P& p,
                                    EvictSmem<NT>& sm) {
    const int32_t* bt = p.block_table + (int64_t)s * p.max_blocks;
    const int64_t layer_tiles = (int64_t)l * p.num_blocks;
    uint4* stage = reinterpret_cast<uint4*>(&sm.u);
    bool bad = false;
    for (int base = m0; base < J; base += kStageRows) {
        const int nsl = min(kStageRows, J - base) * kSlicesPerRow;
        for (int i = threadIdx.x; i < nsl; i += NT) {
            SliceMove m;
            if (slice_move<NT>(sidx, base + i / kSlicesPerRow, i % kSlicesPerRow, bt, layer_tiles, p, h, m))
                cp_async16(stage + i, m.src);
            else
                bad = true;
        }
        cp_async_wait_all();
        sel_sync<NT>();
        for (int i = threadIdx.x; i < nsl; i += NT) {
            SliceMove m;
            if (slice_move<NT>(sidx, base + i / kSlicesPerRow, i % kSlicesPerRow, bt, layer_tiles, p, h, m))
                *reinterpret_cast<uint4*>(m.dst) = stage[i];
        }
        sel_sync<NT>();
    }
    return bad;
}

}  // namespace

}  // namespace tri
