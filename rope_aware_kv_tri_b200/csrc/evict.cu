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
// One CTA of 512 threads per unit (sequence, layer, KV head).  The
// selection itself (select_device.cuh) finds the exact cut key and its tie
// count and emits the kept slots ascending.
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

#include "select_device.cuh"
#include "tri_device.cuh"
#include "tri_internal.h"

namespace tri {

namespace {

constexpr int kEvictThreads = 512;
constexpr int kMoveThreads = 256;
constexpr int kMoveRows = 8;                      // rows in flight per warp in move_kernel
constexpr int kMoveWarps = kMoveThreads / 32;
constexpr size_t kMoveStageBytes = (size_t)kMoveWarps * kMoveRows * 2 * kRowBytes;   // 32 KiB
using EvictSmemT = EvictSmem<kEvictThreads>;

__global__ void __launch_bounds__(kEvictThreads, 2) evict_kernel(const EvictParams p) {
    extern __shared__ __align__(128) uint8_t smem[];
    EvictSmemT& sm = *reinterpret_cast<EvictSmemT*>(smem);
    int* sidx = reinterpret_cast<int*>(smem + sizeof(EvictSmemT));
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
        select_unit<kEvictThreads>(sc, len, p.budget, p.window, p.sinks, sidx, sm, p.status, have_range,
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
        const int m0 = block_sum<kEvictThreads>(fixed, sm);     // idx_j == j exactly for j < m0
        const int J = block_sum<kEvictThreads>(low, sm);        // idx_j < kept exactly for j < J
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
            __syncthreads_or(pack_ordered_prefix<kEvictThreads>(sidx, m0, J, s, l, h, p, sm)) && threadIdx.x == 0)
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
    extern __shared__ __align__(128) uint8_t move_smem[];
    uint64_t* bars = reinterpret_cast<uint64_t*>(move_smem + kMoveStageBytes);   // one mbarrier per warp
    if (threadIdx.x < kMoveWarps) {
        mbar_init(&bars[threadIdx.x], 1);
        fence_mbar_init();
    }
    __syncthreads();
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
    const int wl = threadIdx.x >> 5;
    uint8_t* stage = move_smem + (size_t)wl * kMoveRows * 2 * kRowBytes;
    uint64_t* bar = &bars[wl];
    uint32_t phase = 0;
    const uint64_t pol = l2_policy_evict_first();
    bool bad = false, gave_up = false;
    for (int tile = warp0; tile < ntiles && !gave_up; tile += nwarps) {
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
        // kMoveRows rows at a time: each row's lane has the TMA engine copy
        // its K and V rows into the warp's staging (counted on the warp's
        // mbarrier), then store them with bulk stores
        uint32_t todo = __ballot_sync(0xffffffffu, sk != nullptr);
        while (todo) {
            uint32_t batch = todo;
            if (__popc(todo) > kMoveRows) batch = todo & ((1u << __fns(todo, 0, kMoveRows + 1)) - 1u);
            todo &= ~batch;
            const bool in_batch = (batch >> lane) & 1u;
            uint8_t* st = stage + (size_t)__popc(batch & ((1u << lane) - 1u)) * 2 * kRowBytes;
            if (lane == 0) mbar_arrive_expect_tx(bar, (uint32_t)__popc(batch) * 2 * kRowBytes);
            if (in_batch) {
                bulk_copy_g2s(st, sk, kRowBytes, bar, pol);
                bulk_copy_g2s(st + kRowBytes, sv, kRowBytes, bar, pol);
            }
            const bool landed = mbar_wait_bounded(bar, phase);
            if (!landed) mbar_wait_bounded(bar, phase);   // copies still in flight land before the staging is reused
            phase ^= 1u;
            if (!__all_sync(0xffffffffu, landed)) {
                if (lane == 0) raise_flag(p.status, TRI_DEVFLAG_TIMEOUT);
                gave_up = true;
                break;
            }
            if (in_batch) {
                bulk_copy_s2g(dk, st, kRowBytes);
                bulk_copy_s2g(dv, st + kRowBytes, kRowBytes);
                bulk_commit_group();
                bulk_wait_group_read<0>();
            }
            __syncwarp();
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
    const size_t smem = sizeof(EvictSmemT) + (size_t)p.budget * sizeof(int);
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
    const size_t smem = kMoveStageBytes + kMoveWarps * sizeof(uint64_t);
    return launch_kernel(move_kernel, dim3((unsigned)grid), dim3(kMoveThreads), smem, stream, pdl, p);
}

cudaError_t launch_finalize(const FinalizeParams& p, cudaStream_t stream) {
    finalize_kernel<<<1, kFinalizeThreads, 0, stream>>>(p);
    return cudaGetLastError();
}

}  // namespace tri
