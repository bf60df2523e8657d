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
//    sources a later store overwrites);
//  * moves rows [J, kept): their sources idx_j >= kept are never written in
//    the step, and the prefix pass has read every destination row it needed.
//    Each warp takes rows J + 32w, J + 32(w + 16), ... and moves them 12 at
//    a time through its own slice of the (now idle) selection scratch with
//    16-byte asynchronous copies (lanes 0-15 the K half of a row, 16-31 the V
//    half): 96 KiB in flight per CTA;
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
__host__ __device__ inline size_t sc_smem_bytes(int budget) { return sc_sidx_offset() + (size_t)budget * 4; }

static_assert(sizeof(SelectScratch) >= (size_t)kScWarps * kScMoveRows * kRowPairBytes,
              "move staging must fit in the selection scratch");

__device__ __forceinline__ bool compressed(const SelectCompactParams& p, int u) {
    return __ldcg(p.len_ws + u / (p.L * p.Hkv)) > p.trigger;
}

// Rows [J, kept) of unit u take their sources idx_j (>= kept).  Warp w
// takes rows J + 32w + 512k; lane i resolves one row of the 32, then the
// warp copies its rows kScMoveRows at a time through its 6 KiB staging slice.
__device__ void move_rows(const SelectCompactParams& p, int u, int s, int l, int h, int len, int J, const int* sidx,
                          uint8_t* stage) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int B = p.budget;
    const int32_t* bt = p.block_table + (int64_t)s * p.max_blocks;
    const int64_t lt = (int64_t)l * p.num_blocks;
    uint8_t* wbuf = stage + (size_t)warp * kScMoveRows * kRowPairBytes;
    const int half = lane < 16 ? 0 : kHeadDim * 2;     // K or V half of the staged row pair
    const int in_row = (lane & 15) * 16;
    uint8_t* pool = lane < 16 ? p.k_pool : p.v_pool;
    bool bad = false;
    for (int j0 = J + warp * 32; j0 < B; j0 += kScThreads) {
        const int j = j0 + lane;
        int64_t so = 0, dof = 0;
        bool valid = false;
        if (j < B) {
            const int src = sidx[j];
            if (src >= B && src < len) {
                if (row_offset(bt, src, lt, p.Hkv, h, p.num_blocks, so) &&
                    row_offset(bt, j, lt, p.Hkv, h, p.num_blocks, dof))
                    valid = true;
                else
                    bad = true;
            }
        }
        uint32_t todo = __ballot_sync(0xffffffffu, valid);
        while (todo) {
            uint32_t batch = todo;
            if (__popc(todo) > kScMoveRows) batch = todo & ((1u << __fns(todo, 0, kScMoveRows + 1)) - 1u);
            int n = 0;
            for (uint32_t b = batch; b; b &= b - 1u, ++n) {
                const long long src_off = __shfl_sync(0xffffffffu, (long long)so, __ffs(b) - 1);
                cp_async16(wbuf + n * kRowPairBytes + half + in_row, pool + src_off + in_row);
            }
            cp_async_wait_all();
            n = 0;
            for (uint32_t b = batch; b; b &= b - 1u, ++n) {
                const long long dst_off = __shfl_sync(0xffffffffu, (long long)dof, __ffs(b) - 1);
                *reinterpret_cast<uint4*>(pool + dst_off + in_row) =
                    *reinterpret_cast<const uint4*>(wbuf + n * kRowPairBytes + half + in_row);
            }
            todo &= ~batch;
        }
    }
    if (__any_sync(0xffffffffu, bad) && lane == 0) raise_flag(p.status, TRI_DEVFLAG_BOUNDS);
}

// Select unit u, pack its at-risk prefix in place, move its other kept rows.
__device__ void select_task(const SelectCompactParams& p, int u, ScSmem& sm, int* sidx) {
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
    if (J > m0 && sel_sync_or<kScThreads>(pack_ordered_prefix<kScThreads>(sidx, m0, J, s, l, h, p, sm)) && tid == 0)
        raise_flag(p.status, TRI_DEVFLAG_BOUNDS);
    move_rows(p, u, s, l, h, len, J, sidx, reinterpret_cast<uint8_t*>(&sm.u));
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
    sel_sync<kScThreads>();                // the scratch is free for the next unit
}

__global__ void __launch_bounds__(kScThreads, 2) select_compact_kernel(const __grid_constant__ SelectCompactParams p) {
    extern __shared__ __align__(128) uint8_t smem[];
    ScSmem& sm = *reinterpret_cast<ScSmem*>(smem);
    int* sidx = reinterpret_cast<int*>(smem + sc_sidx_offset());
    __shared__ int s_task;
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
        select_task(p, u, sm, sidx);
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
