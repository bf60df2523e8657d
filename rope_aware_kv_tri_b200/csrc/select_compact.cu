// select_compact.cu - the selection and the Forward-Packing Compaction of a
// step, for every unit, in one persistent kernel.
//
// Pages: "TriAttention: Trigonometric KV Compression for Efficient Long
// Reasoning" - "Core Mechanism" (rank keys and keep only the top-scoring
// subset); "TriAttention: How a Geometric Trick Cuts LLM Memory Use by 10x
// Without Losing Accuracy" - "Solving the Memory Fragmentation Problem"
// (survivors move forward so tail blocks empty out).
//
// After the score pass the step has two kinds of work of very different
// shape: each unit's selection is a chain of dependent on-chip passes over
// its scores (latency-bound, ~20 us per unit at 512 threads, the scores come
// from L2), and the row moves are HBM-bound.  Run as a selection kernel
// followed by copy-out and move kernels, HBM idles during the selection wave
// and the at-risk rows cross HBM twice.  Here a persistent grid (two
// 512-thread CTAs per SM) takes units from a device counter, and the CTA
// that takes a unit does all of its work:
//
//  * selects its kept slots (select_device.cuh), writes its indices, and
//    carries slot positions with the rows when asked (distance-table step);
//  * packs the at-risk prefix [m0, J) in place in ordered rounds (rows whose
//    sources a later store overwrites): each round has the TMA engine copy
//    up to 192 rows (one row's K and V per thread, 256-byte bulk copies
//    counted on one mbarrier) into the (now idle) selection scratch, then
//    stores them with bulk stores;
//  * moves rows [J, kept): their sources idx_j >= kept are never written in
//    the step, and the prefix pass has read every destination row it needed.
//    Each warp takes rows J + w, J + w + 16, ... and moves them 12 at a time
//    through its own 6 KiB of the scratch, with bulk copies counted on its
//    own mbarrier: 96 KiB in flight per CTA.
//    Bulk copies move a row with two instructions where 16-byte copies take
//    32 loads and 32 stores: the rounds and moves run closer to the copy
//    bandwidth (one 32-layer x 8-head step of 32768 keys per unit keeping
//    2048: 127 -> 117 us; a decode round of 16 sequences keeping 2048 of
//    2176 slots: 1.93 -> 1.76 ms);
//  * does its sequence's bookkeeping (new length, freed blocks; first head
//    of layer 0).
//
// Units' moves start as soon as each unit is selected, so HBM is busy while
// slower units are still being selected; no at-risk row is copied out to a
// scratch and back.
//
// Every CTA follows its own task sequence: thread 0 takes a unit and
// __syncthreads broadcasts it, so every barrier is met by all; no CTA waits
// for another.
#include "select_device.cuh"
#include "tri_device.cuh"
#include "tri_internal.h"

namespace tri {

namespace {

constexpr int kScThreads = 512;
constexpr int kScWarps = kScThreads / 32;
constexpr int kScMoveRows = 12;                    // rows in flight per warp (6 KiB staged)
constexpr int kRowPairBytes = 2 * kHeadDim * 2;    // a K row and a V row: 512 bytes

using ScSmem = EvictSmem<kScThreads>;

__host__ __device__ inline size_t sc_sidx_offset() { return (sizeof(ScSmem) + 15) / 16 * 16; }
// the mbarriers after the kept indices: one for the prefix rounds, one per warp for the moves
__host__ __device__ inline size_t sc_bar_offset(int budget) {
    return (sc_sidx_offset() + (size_t)budget * 4 + 7) / 8 * 8;
}
__host__ __device__ inline size_t sc_smem_bytes(int budget) { return sc_bar_offset(budget) + 8 * (1 + kScWarps); }

static_assert(sizeof(SelectScratch) >= (size_t)kScWarps * kScMoveRows * kRowPairBytes,
              "move staging must fit in the selection scratch");

__device__ __forceinline__ bool compressed(const SelectCompactParams& p, int u) {
    return __ldcg(p.len_ws + u / (p.L * p.Hkv)) > p.trigger;
}

// Rows [J, kept) of unit u take their sources idx_j (>= kept), which no store
// of the step touches, so they move in any order: warp w takes rows J + w,
// J + w + 16, ..., kScMoveRows at a time; lane i of a batch has the TMA engine
// copy its row's K and V (256 bytes each) into the warp's 6 KiB of the idle
// selection scratch, counted on the warp's mbarrier, then stores them with
// bulk stores and waits until those have read the staging.  Returns true
// (for the whole warp) when a batch's copies did not land in time: the
// warp then stores nothing more and the status word says so.
__device__ bool move_rows(const SelectCompactParams& p, int u, int s, int l, int h, int len, int J, const int* sidx,
                          uint8_t* stage, uint64_t* wbar, uint32_t& wphase) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int B = p.budget;
    const int32_t* bt = p.block_table + (int64_t)s * p.max_blocks;
    const int64_t lt = (int64_t)l * p.num_blocks;
    uint8_t* mine = stage + ((size_t)warp * kScMoveRows + lane) * kRowPairBytes;
    uint64_t* bar = wbar + warp;
    const uint64_t pol = l2_policy_evict_first();
    bool bad = false, gave_up = false;
    for (int j0 = J + warp; j0 < B; j0 += kScWarps * kScMoveRows) {
        const int j = j0 + lane * kScWarps;
        int64_t so = 0, dof = 0;
        bool valid = false;
        if (lane < kScMoveRows && j < B) {
            const int src = sidx[j];
            if (src >= B && src < len) {
                if (row_offset(bt, src, lt, p.Hkv, h, p.num_blocks, so) &&
                    row_offset(bt, j, lt, p.Hkv, h, p.num_blocks, dof))
                    valid = true;
                else
                    bad = true;
            }
        }
        const uint32_t nvalid = __popc(__ballot_sync(0xffffffffu, valid));
        if (lane == 0) mbar_arrive_expect_tx(bar, nvalid * kRowPairBytes);
        if (valid) {
            bulk_copy_g2s(mine, p.k_pool + so, kRowPairBytes / 2, bar, pol);
            bulk_copy_g2s(mine + kRowPairBytes / 2, p.v_pool + so, kRowPairBytes / 2, bar, pol);
        }
        const bool landed = mbar_wait_bounded(bar, wphase);
        if (!landed) mbar_wait_bounded(bar, wphase);   // copies still in flight land before the staging is reused
        wphase ^= 1u;
        if (!__all_sync(0xffffffffu, landed)) {
            if (lane == 0) raise_flag(p.status, TRI_DEVFLAG_TIMEOUT);
            gave_up = true;
            break;
        }
        if (valid) {
            bulk_copy_s2g(p.k_pool + dof, mine, kRowPairBytes / 2);
            bulk_copy_s2g(p.v_pool + dof, mine + kRowPairBytes / 2, kRowPairBytes / 2);
            bulk_commit_group();
            bulk_wait_group_read<0>();
        }
        __syncwarp();
    }
    if (__any_sync(0xffffffffu, bad) && lane == 0) raise_flag(p.status, TRI_DEVFLAG_BOUNDS);
    return gave_up;
}

// The at-risk prefix [m0, J) in ascending rounds of kStageRows rows staged in
// the idle selection scratch: thread i of a round has the TMA engine copy row
// base + i's source (its K and V rows, 256 bytes each) into shared memory,
// every copy of the round counted on one mbarrier; then each thread has the
// staged rows stored to their destinations with bulk stores and waits until
// those have read the staging.  A later round reads only slots >= its first
// row, which no earlier round writes.  gave_up (the same in every thread)
// says a round's copies did not land in time; that round stores only the
// rows that did land, no later round runs, and the status word says so.
__device__ bool pack_prefix_bulk(const SelectCompactParams& p, const int* sidx, int m0, int J, int s, int l, int h,
                                 uint8_t* stage, uint64_t* bar, uint32_t& phase, bool& gave_up) {
    const int tid = threadIdx.x;
    const int32_t* bt = p.block_table + (int64_t)s * p.max_blocks;
    const int64_t lt = (int64_t)l * p.num_blocks;
    const uint64_t pol = l2_policy_evict_first();
    bool bad = false;
    fence_proxy_async_smem();           // the selection's stores to the scratch precede the copies into it
    sel_sync<kScThreads>();
    for (int base = m0; base < J; base += kStageRows) {
        const int n = min(kStageRows, J - base);
        int64_t so = 0, dof = 0;
        bool valid = false;
        if (tid < n) {
            const int j = base + tid;
            if (row_offset(bt, sidx[j], lt, p.Hkv, h, p.num_blocks, so) &&
                row_offset(bt, j, lt, p.Hkv, h, p.num_blocks, dof))
                valid = true;
            else
                bad = true;
        }
        const int nvalid = __syncthreads_count(valid);
        if (tid == 0) mbar_arrive_expect_tx(bar, (uint32_t)nvalid * kRowPairBytes);
        uint8_t* mine = stage + (size_t)tid * kRowPairBytes;
        if (valid) {
            bulk_copy_g2s(mine, p.k_pool + so, kRowPairBytes / 2, bar, pol);
            bulk_copy_g2s(mine + kRowPairBytes / 2, p.v_pool + so, kRowPairBytes / 2, bar, pol);
        }
        const bool landed = mbar_wait_bounded(bar, phase);
        if (!landed) {
            raise_flag(p.status, TRI_DEVFLAG_TIMEOUT);
            mbar_wait_bounded(bar, phase);  // copies still in flight land before the staging is reused
        }
        phase ^= 1u;
        if (valid && landed) {
            bulk_copy_s2g(p.k_pool + dof, mine, kRowPairBytes / 2);
            bulk_copy_s2g(p.v_pool + dof, mine + kRowPairBytes / 2, kRowPairBytes / 2);
            bulk_commit_group();
            bulk_wait_group_read<0>();
        }
        if (sel_sync_or<kScThreads>(!landed)) {   // the staging is free for the next round
            gave_up = true;
            break;
        }
    }
    return bad;
}

// Select unit u, pack its at-risk prefix in place, move its other kept rows.
// Returns true (in every thread) when a wait for copies gave up: the CTA then
// takes no further unit.
__device__ bool select_task(const SelectCompactParams& p, int u, ScSmem& sm, int* sidx, uint64_t* bar,
                            uint32_t& phase, uint32_t& wphase) {
    const int tid = threadIdx.x;
    const int LH = p.L * p.Hkv;
    const int s = u / LH, rem = u % LH, l = rem / p.Hkv, h = rem % p.Hkv;
    const int len = __ldcg(p.len_ws + s);
    const int B = p.budget;
    const float* sc = p.scores + (int64_t)u * p.score_stride;
    select_unit<kScThreads>(sc, len, B, p.window, p.sinks, sidx, sm, p.status, true, __ldcg(p.unit_kmin + u),
                            __ldcg(p.unit_kmax + u));
    if (p.idx_copy)
        for (int j = tid; j < B; j += kScThreads) p.idx_copy[(int64_t)u * B + j] = sidx[j];
    if (p.slot_pos) {
        // positions travel with their rows: every kept position is read into
        // the (idle) selection scratch before any is stored
        int32_t* pos = p.slot_pos + (int64_t)u * p.pos_stride;
        int* stage = reinterpret_cast<int*>(&sm.u);
        for (int j = tid; j < B; j += kScThreads) stage[j] = pos[sidx[j]];
        sel_sync<kScThreads>();
        for (int j = tid; j < B; j += kScThreads) pos[j] = stage[j];
        sel_sync<kScThreads>();
    }
    int fixed = 0, low = 0;
    for (int j = tid; j < B; j += kScThreads) {
        fixed += (sidx[j] == j) ? 1 : 0;
        low += (sidx[j] < B) ? 1 : 0;
    }
    const int m0 = block_sum<kScThreads>(fixed, sm);   // idx_j == j exactly for j < m0
    const int J = block_sum<kScThreads>(low, sm);      // idx_j < kept exactly for j < J
    bool gave_up = false;
    if (J > m0 &&
        sel_sync_or<kScThreads>(pack_prefix_bulk(p, sidx, m0, J, s, l, h, reinterpret_cast<uint8_t*>(&sm.u), bar,
                                                 phase, gave_up)) &&
        tid == 0)
        raise_flag(p.status, TRI_DEVFLAG_BOUNDS);
    fence_proxy_async_smem();           // the selection's stores to the scratch precede the copies into it
    sel_sync<kScThreads>();
    if (!gave_up) gave_up = move_rows(p, u, s, l, h, len, J, sidx, reinterpret_cast<uint8_t*>(&sm.u), bar + 1, wphase);
    if (l == 0 && h == 0) {
        // the sequence's new length and its freed blocks
        const int32_t* bt = p.block_table + (int64_t)s * p.max_blocks;
        const int lo = (B + kBlockRows - 1) / kBlockRows;
        const int hi = (len + kBlockRows - 1) / kBlockRows;
        const int off = __ldcg(p.freed_off + s);
        if (p.freed_ids)
            for (int e = tid; e < hi - lo; e += kScThreads) p.freed_ids[off + e] = bt[lo + e];
        if (p.fl_ids) {
            const int base = __ldcg(p.fl_base);
            if (base >= 0)
                for (int e = tid; e < hi - lo; e += kScThreads) p.fl_ids[base + off + e] = bt[lo + e];
        }
        if (tid == 0) p.seq_len_out[s] = B;
    }
    return sel_sync_or<kScThreads>(gave_up);    // the scratch is free for the next unit
}

__global__ void __launch_bounds__(kScThreads, 2) select_compact_kernel(const __grid_constant__ SelectCompactParams p) {
    extern __shared__ __align__(128) uint8_t smem[];
    ScSmem& sm = *reinterpret_cast<ScSmem*>(smem);
    int* sidx = reinterpret_cast<int*>(smem + sc_sidx_offset());
    __shared__ int s_task;
    uint64_t* bar = reinterpret_cast<uint64_t*>(smem + sc_bar_offset(p.budget));
    if (threadIdx.x == 0) {
        for (int i = 0; i <= kScWarps; ++i) mbar_init(&bar[i], 1);
        fence_mbar_init();
    }
    __syncthreads();
    uint32_t phase = 0, wphase = 0;
    wait_prior_grid();          // scores, key ranges, plan and the zeroed unit counter
    if (p.abort_word && __ldcg(p.abort_word) != 0) return;    // vetoed step: change nothing
    const int U = p.S * p.L * p.Hkv;
    for (;;) {
        if (threadIdx.x == 0) {
            int u = atomicAdd(p.qwords + kQwClaim, 1);
            while (u < U && !compressed(p, u)) u = atomicAdd(p.qwords + kQwClaim, 1);
            s_task = u;
        }
        __syncthreads();
        const int u = s_task;
        __syncthreads();
        if (u >= U) break;
        if (select_task(p, u, sm, sidx, bar, phase, wphase)) break;
    }
}

}  // namespace

bool select_compact_supported(int budget) { return budget >= 1 && sc_smem_bytes(budget) + 64 <= 227 * 1024; }

cudaError_t launch_select_compact(const SelectCompactParams& p, int num_sms, cudaStream_t stream, bool pdl) {
    const size_t smem = sc_smem_bytes(p.budget);
    cudaError_t e =
        cudaFuncSetAttribute(select_compact_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(select_compact_kernel, cudaFuncAttributePreferredSharedMemoryCarveout,
                             (int)cudaSharedmemCarveoutMaxShared);
    if (e != cudaSuccess) return e;
    int per_sm = 0;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, select_compact_kernel, kScThreads, smem);
    if (e != cudaSuccess) return e;
    if (per_sm < 1) per_sm = 1;
    const int U = p.S * p.L * p.Hkv;
    int grid = per_sm * num_sms;
    if (U < grid) grid = U;
    return launch_kernel(select_compact_kernel, dim3(grid), dim3(kScThreads), smem, stream, pdl, p);
}

}  // namespace tri
