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
// kept; among the first len - W the B - W best by (score desc, slot asc).
// Scores become 32-bit keys whose unsigned order is the score order
// (order_key: -0 == +0, NaN == -inf).  Three radix passes (12 + 10 + 10
// bits) over the unit's scores, each a shared-memory histogram of the keys
// that match the prefix found so far, find the exact key of the (B-W)-th
// best candidate and how many of the candidates equal to it are taken.  Two
// more passes emit the kept slots in ascending order: each warp owns a
// contiguous segment of slots, counts its "greater" and "equal" keys with
// ballots, a 16-entry scan gives every warp its output offset and its rank
// among equal keys, and a second walk writes the slots.  The result is
// unique: ties go to the lower slot.
//
// Compaction, in place: row j of K and V takes row idx_j (idx ascending, so
// idx_j >= j).  Rows j < first_move have idx_j == j and stay.  The rest move
// in ascending chunks of 64 rows: the whole chunk is loaded into registers,
// the CTA synchronises, then the chunk is stored.  A chunk's stores land on
// rows [a, b) that no later chunk reads (their sources are >= b) and whose
// readers in this or earlier chunks have all loaded before the barrier, so
// the in-place move is race-free with one barrier per chunk.
#include "tri_device.cuh"
#include "tri_internal.h"

namespace tri {

namespace {

constexpr int kEvictThreads = 512;
constexpr int kEvictWarps = kEvictThreads / 32;
constexpr int kHistBins = 4096;
constexpr int kCompactRows = 64;                              // rows per chunk
constexpr int kSlicesPerRow = 2 * kHeadDim * 2 / 16;          // 16 B slices of K and V: 32
constexpr int kSlicesPerThread = kCompactRows * kSlicesPerRow / kEvictThreads;   // 4

struct EvictSmem {
    int hist[kHistBins];
    int warp_a[kEvictWarps];
    int warp_b[kEvictWarps];
    int eq_before[kEvictWarps];
    int keep_before[kEvictWarps];
    int bcast[4];
};

// One radix pass: narrows (prefix, mask) by `bits` bits at `shift` so that
// the rem-th largest key among the candidates matching the prefix keeps
// matching; rem becomes its rank among the keys matching the new prefix.
// Returns whether any candidate score is NaN.
__device__ bool radix_pass(const float* __restrict__ sc, int cand, uint32_t& prefix, uint32_t& mask, int& rem,
                           int shift, int bits, EvictSmem& sm) {
    const int nb = 1 << bits;
    const uint32_t dmask = (uint32_t)nb - 1u;
    for (int i = threadIdx.x; i < nb; i += kEvictThreads) sm.hist[i] = 0;
    __syncthreads();
    bool nan_seen = false;
    for (int t = threadIdx.x; t < cand; t += kEvictThreads) {
        const float x = sc[t];
        nan_seen |= isnan(x);
        const uint32_t key = order_key(x);
        if ((key & mask) == prefix) atomicAdd(&sm.hist[(key >> shift) & dmask], 1);
    }
    const bool any_nan = __syncthreads_or(nan_seen) != 0;
    const int per = nb / kEvictThreads;
    const int b0 = threadIdx.x * per;
    int local = 0;
    for (int j = 0; j < per; ++j) local += sm.hist[b0 + j];
    int total;
    const int ex = block_exclusive_scan<kEvictThreads>(local, sm.warp_a, total);
    int run = total - ex - local;      // keys in bins above this thread's bins
    for (int j = per - 1; j >= 0; --j) {
        const int h = sm.hist[b0 + j];
        if (run < rem && rem <= run + h) {
            sm.bcast[0] = b0 + j;
            sm.bcast[1] = rem - run;
        }
        run += h;
    }
    __syncthreads();
    prefix |= (uint32_t)sm.bcast[0] << shift;
    mask |= dmask << shift;
    rem = sm.bcast[1];
    __syncthreads();
    return any_nan;
}

// Kept slots of one unit into sidx[0 .. kept), ascending.  Returns kept.
__device__ int select_unit(const float* __restrict__ sc, int len, int budget, int window, int* sidx,
                           EvictSmem& sm, int32_t* status) {
    const int cand = len - window;
    const int take = budget - window;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (take > 0) {
        uint32_t prefix = 0, mask = 0;
        int rem = take;
        if (radix_pass(sc, cand, prefix, mask, rem, 20, 12, sm) && threadIdx.x == 0)
            raise_flag(status, TRI_DEVFLAG_NONFINITE);
        radix_pass(sc, cand, prefix, mask, rem, 10, 10, sm);
        radix_pass(sc, cand, prefix, mask, rem, 0, 10, sm);
        const uint32_t thr = prefix;
        const int need_eq = rem;
        const int seg = (((cand + kEvictWarps - 1) / kEvictWarps) + 31) & ~31;
        const int beg = warp * seg;
        const int end = min(beg + seg, cand);
        int gt = 0, eq = 0;
        for (int t0 = beg; t0 < end; t0 += 32) {
            const int t = t0 + lane;
            const uint32_t key = t < end ? order_key(sc[t]) : 0u;
            gt += __popc(__ballot_sync(0xffffffffu, t < end && key > thr));
            eq += __popc(__ballot_sync(0xffffffffu, t < end && key == thr));
        }
        if (lane == 0) {
            sm.warp_a[warp] = gt;
            sm.warp_b[warp] = eq;
        }
        __syncthreads();
        if (threadIdx.x == 0) {
            int eb = 0, kb = 0;
            for (int w = 0; w < kEvictWarps; ++w) {
                sm.eq_before[w] = eb;
                sm.keep_before[w] = kb;
                const int left = need_eq - eb;
                const int from_eq = left <= 0 ? 0 : (left < sm.warp_b[w] ? left : sm.warp_b[w]);
                kb += sm.warp_a[w] + from_eq;
                eb += sm.warp_b[w];
            }
        }
        __syncthreads();
        int run_eq = sm.eq_before[warp], run_keep = sm.keep_before[warp];
        const uint32_t lt = lanemask_lt();
        for (int t0 = beg; t0 < end; t0 += 32) {
            const int t = t0 + lane;
            const bool valid = t < end;
            const uint32_t key = valid ? order_key(sc[t]) : 0u;
            const bool g = valid && key > thr;
            const bool e = valid && key == thr;
            const uint32_t eqb = __ballot_sync(0xffffffffu, e);
            const bool keep = g || (e && run_eq + __popc(eqb & lt) < need_eq);
            const uint32_t kb = __ballot_sync(0xffffffffu, keep);
            const int pos = run_keep + __popc(kb & lt);
            if (keep && pos < take) sidx[pos] = t;
            run_eq += __popc(eqb);
            run_keep += __popc(kb);
        }
    }
    for (int j = threadIdx.x; j < window; j += kEvictThreads) sidx[take + j] = cand + j;
    __syncthreads();
    return budget;
}

__device__ __forceinline__ int block_sum(int v, EvictSmem& sm) {
    int total;
    block_exclusive_scan<kEvictThreads>(v, sm.warp_a, total);
    return total;
}

// Forward-packing of one unit's K and V rows (see the file comment).
__device__ void compact_unit(const int* sidx, int kept, int s, int l, int h, const EvictParams& p,
                             EvictSmem& sm) {
    int fixed = 0;
    for (int j = threadIdx.x; j < kept; j += kEvictThreads) fixed += (sidx[j] == j) ? 1 : 0;
    const int m0 = block_sum(fixed, sm);     // idx_j == j exactly for j < m0
    const int32_t* bt = p.block_table + (int64_t)s * p.max_blocks;
    const int64_t layer_tiles = (int64_t)l * p.num_blocks;
    bool bad = false;
    for (int base = m0; base < kept; base += kCompactRows) {
        uint4 buf[kSlicesPerThread];
        int64_t dst[kSlicesPerThread];
#pragma unroll
        for (int u = 0; u < kSlicesPerThread; ++u) {
            const int sl = u * kEvictThreads + threadIdx.x;
            const int r = sl / kSlicesPerRow, part = sl % kSlicesPerRow;
            const int j = base + r;
            dst[u] = -1;
            if (j < kept) {
                const int src = sidx[j];
                const int bsrc = bt[src / kBlockRows], bdst = bt[j / kBlockRows];
                if (bsrc >= 0 && bsrc < p.num_blocks && bdst >= 0 && bdst < p.num_blocks) {
                    const uint8_t* pool = part < 16 ? p.k_pool : p.v_pool;
                    const int64_t so = (((layer_tiles + bsrc) * p.Hkv + h) * kBlockRows + (src % kBlockRows)) * 256 +
                                       (part % 16) * 16;
                    dst[u] = (((layer_tiles + bdst) * p.Hkv + h) * kBlockRows + (j % kBlockRows)) * 256 +
                             (part % 16) * 16;
                    buf[u] = *reinterpret_cast<const uint4*>(pool + so);
                } else {
                    bad = true;
                }
            }
        }
        __syncthreads();
#pragma unroll
        for (int u = 0; u < kSlicesPerThread; ++u) {
            if (dst[u] >= 0) {
                const int part = (u * kEvictThreads + threadIdx.x) % kSlicesPerRow;
                uint8_t* pool = part < 16 ? p.k_pool : p.v_pool;
                *reinterpret_cast<uint4*>(pool + dst[u]) = buf[u];
            }
        }
    }
    if (bad) raise_flag(p.status, TRI_DEVFLAG_BOUNDS);
}

__global__ void __launch_bounds__(kEvictThreads, 2) evict_kernel(const EvictParams p) {
    extern __shared__ __align__(16) uint8_t smem[];
    EvictSmem& sm = *reinterpret_cast<EvictSmem*>(smem);
    int* sidx = reinterpret_cast<int*>(smem + sizeof(EvictSmem));
    const int u = blockIdx.x;
    const int LH = p.L * p.Hkv;
    const int s = u / LH, rem = u % LH, l = rem / p.Hkv, h = rem % p.Hkv;
    const bool head0 = (l == 0 && h == 0);
    int len = p.lens[s];
    if (len < 0 || (int64_t)len > (int64_t)p.max_blocks * kBlockRows) {
        if (threadIdx.x == 0) raise_flag(p.status, TRI_DEVFLAG_BOUNDS);
        return;
    }
    int kept;
    if (p.do_select) {
        if (len <= p.budget) {
            // Nothing to evict.  A standalone selection reports every slot.
            if (!p.do_compact) {
                for (int j = threadIdx.x; j < p.budget; j += kEvictThreads)
                    p.idx_out[(int64_t)u * p.budget + j] = j < len ? j : -1;
                if (head0 && threadIdx.x == 0) p.kept_out[s] = len;
            }
            return;
        }
        const float* sc = p.scores + (int64_t)u * p.score_stride;
        kept = select_unit(sc, len, p.budget, p.window, sidx, sm, p.status);
        if (p.idx_out)
            for (int j = threadIdx.x; j < p.budget; j += kEvictThreads)
                p.idx_out[(int64_t)u * p.budget + j] = j < kept ? sidx[j] : -1;
        if (p.kept_out && head0 && threadIdx.x == 0) p.kept_out[s] = kept;
    } else {
        kept = p.kept_in[s];
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
    if (p.do_compact) compact_unit(sidx, kept, s, l, h, p, sm);
    if (head0 && p.seq_len_out) {
        // Step bookkeeping: the sequence's new length and its freed blocks.
        const int32_t* bt = p.block_table + (int64_t)s * p.max_blocks;
        const int lo = (kept + kBlockRows - 1) / kBlockRows;
        const int hi = (len + kBlockRows - 1) / kBlockRows;
        const int off = p.freed_off[s];
        for (int e = threadIdx.x; e < hi - lo; e += kEvictThreads) p.freed_ids[off + e] = bt[lo + e];
        if (threadIdx.x == 0) p.seq_len_out[s] = kept;
    }
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

}  // namespace

cudaError_t launch_evict(const EvictParams& p, cudaStream_t stream) {
    const int U = p.S * p.L * p.Hkv;
    if (U == 0) return cudaSuccess;
    const size_t smem = sizeof(EvictSmem) + (size_t)p.budget * sizeof(int);
    cudaError_t e = cudaFuncSetAttribute(evict_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    evict_kernel<<<U, kEvictThreads, smem, stream>>>(p);
    return cudaGetLastError();
}

cudaError_t launch_finalize(const FinalizeParams& p, cudaStream_t stream) {
    finalize_kernel<<<1, kFinalizeThreads, 0, stream>>>(p);
    return cudaGetLastError();
}

}  // namespace tri
