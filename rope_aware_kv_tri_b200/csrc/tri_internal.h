// tri_internal.h - parameter blocks and launchers shared between the C ABI
// (tri_abi.cu) and the kernel translation units.  Not installed; not ABI.
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

#include "tri_attention.h"

namespace tri {

// Launch `kernel` with the programmatic-serialization attribute when `pdl`
// is set (the kernel must call wait_prior_grid before reading what earlier
// work in the stream wrote), else as a plain launch.
template <typename Kernel, typename Params>
cudaError_t launch_kernel(Kernel kernel, dim3 grid, dim3 block, size_t smem, cudaStream_t stream, bool pdl,
                          const Params& params) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = pdl ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, kernel, params);
}

constexpr int kHeadDim = TRI_HEAD_DIM;          // D
constexpr int kBands = TRI_HEAD_DIM / 2;        // n
constexpr int kBlockRows = TRI_BLOCK_SIZE;      // rows per paged block
constexpr int kTileBytes = kBlockRows * kHeadDim * 2;   // one (block, head) tile: 4 KiB
constexpr int kChunkBlocks = 16;                // paged blocks per score work item

// --------------------------------------------------------------- queries
struct QueryParams {
    const float* qbar;        // [L][Hq][D]
    const float* qabs;        // [L][Hq][D/2]
    const float* R;           // [L][Hq]
    const int64_t* cur_pos;   // [S]
    double base;
    int n_deltas;
    int32_t deltas[TRI_MAX_DELTAS];
    float* qeff;              // [U][D], or [U][G][D] per head (aggregate == max)
    float* wts;               // [U][D/2], or [U][G][D/2]
    int L, Hkv, G, S;
    int per_head;             // 1: per-head coefficients (max over the group), 0: group mean
    // plan (last block of the grid when do_plan != 0)
    int do_plan;
    const int32_t* seq_len;   // [S]
    int max_blocks;
    int budget;               // 0: plan every sequence (score only)
    int trigger;              // compress sequences with len > trigger (>= budget)
    int heads_per_tile;       // HG
    int32_t* len_ws;          // [S]
    int32_t* item_off;        // [S+1]
    int32_t* freed_off;       // [S+1]
    int32_t* freed_count;     // [1] or null
    uint32_t* unit_kmin;      // [U] set to the largest key (min accumulator) or null
    uint32_t* unit_kmax;      // [U] set to 0 (max accumulator) or null
    int32_t* zero_words;      // [2] set to 0 by the plan CTA, or null
    int plan_only;            // 1: the plan CTA alone (no effective queries)
    int32_t* fl_count;        // free list to push the freed ids on, or null
    int fl_capacity;
    int32_t* fl_base;         // [1] out: first list entry of this step's ids, -1 if no room
    const int32_t* abort_word; // non-zero: the statistics check vetoed the step (plan nothing), or null
    int32_t* fq_words;         // select + compact: queue words to zero (kQwWords), or null
    int32_t* status;
};
cudaError_t launch_query(const QueryParams& p, cudaStream_t stream);

// ----------------------------------------------------------------- score
struct ScoreParams {
    const uint8_t* k_pool;
    const int32_t* block_table;
    const int32_t* len_ws;
    const int32_t* item_off;
    const float* qeff;
    const float* wts;
    float* scores;
    int64_t score_stride;     // floats between units in `scores`
    uint32_t* unit_kmin;      // [U] smallest order key of each unit's scores
    uint32_t* unit_kmax;      // [U] largest order key of each unit's scores
    int32_t* status;
    int L, Hkv, num_blocks, S, max_blocks;
    int heads_per_tile;       // HG, divides 8 and Hkv
    int agg_heads;            // 0: folded group mean; G: max over G per-head scores
    int cuda_cores_only;      // 1: never the tensor-core max kernel
    int stages;
    // The CUDA-core kernel's producer plans its own work items from these,
    // by the plan's rule, so that it can stream keys before the plan ends.
    const int32_t* seq_len_in; // [S] the caller's lengths
    int budget;                // > 0: only sequences longer than `trigger` are scored
    int trigger;
    const int32_t* abort_word; // non-zero: the step was vetoed (nothing scored), or null
};
int score_heads_per_tile(int Hkv);
cudaError_t launch_score(const ScoreParams& p, int max_items, int num_sms, cudaStream_t stream, bool pdl = false);

// Max over the group with the dot products on the tensor cores (score_mma.cu):
// G in {2, 4, 8}, Hkv a multiple of 8.  The K pool is read through a TMA
// tensor map (2-D: 128 dims x all rows, 128-byte swizzle).
struct MmaScoreParams {
    ScoreParams base;
    CUtensorMap tmap;
};
bool score_mma_supported(const ScoreParams& p);
cudaError_t launch_score_mma(const ScoreParams& p, int max_items, int num_sms, cudaStream_t stream, bool pdl);

// --------------------------------------------------- select + compaction
struct EvictParams {
    const float* scores;
    int64_t score_stride;
    const uint32_t* unit_kmin; // [U] score-key range of each unit, or null
    const uint32_t* unit_kmax;
    const int32_t* lens;       // lengths the unit works from
    int budget, window;
    int sinks;                 // leading slots always kept
    int trigger;               // units with len <= trigger keep every slot (>= budget)
    int32_t* idx_out;          // [U][budget] or null
    int32_t* idx_copy;         // [U][budget] second copy of the kept slots, or null
    int32_t* kept_out;         // [S] or null
    const int32_t* idx_in;     // [U][budget] (compaction from given indices) or null
    const int32_t* kept_in;    // [S] or null
    int do_select, do_compact;
    uint8_t* k_pool;
    uint8_t* v_pool;
    const int32_t* block_table;
    int L, Hkv, num_blocks, S, max_blocks;
    // step bookkeeping: CTA (s, 0, 0) writes seq_len[s] and the freed ids
    int32_t* seq_len_out;      // or null
    const int32_t* freed_off;  // [S+1] or null
    int32_t* freed_ids;        // or null
    int32_t* fl_ids;           // free list entries, or null
    const int32_t* fl_base;    // [1] where this step's ids start in fl_ids (-1: none)
    int32_t* slot_pos;         // [U][pos_stride] cached position of every slot, compacted with the rows, or null
    int64_t pos_stride;
    int32_t* status;
    // step plans (null outside tri_compress_step)
    int32_t* scratch_used;     // [1] rows of the scratch handed out, 0 at launch
    int32_t* unit_info;        // [U][4]: m0, J, mode, scratch row
    int32_t* scratch_owner;    // [2][scratch_rows]: unit and source row of each scratch row
    int scratch_rows;          // capacity of the scratch in rows
    int many_units;            // several waves of unit CTAs: long at-risk prefixes compact in place
    const int32_t* abort_word; // non-zero: the step was vetoed, touch nothing; or null
};
cudaError_t launch_evict(const EvictParams& p, cudaStream_t stream, bool pdl = false);

// ------------------------------ select + compact (select_compact.cu)
// Selection and compaction of a step's units in one persistent kernel,
// after the score pass; used by every step variant whose budget fits.
// Queue words (workspace, zeroed by the plan CTA):
constexpr int kQwClaim = 0;     // next unit to take
constexpr int kQwWords = 8;

struct SelectCompactParams {
    uint8_t* k_pool;
    uint8_t* v_pool;
    const int32_t* block_table;
    const int32_t* len_ws;     // [S] lengths the step works from
    const float* scores;
    int64_t score_stride;
    const uint32_t* unit_kmin; // [U] score-key range of each unit
    const uint32_t* unit_kmax;
    int32_t* status;
    int L, Hkv, num_blocks, S, max_blocks;
    int budget, window, sinks, trigger;
    int32_t* idx_copy;         // [U][budget] kept slots out, or null
    int32_t* seq_len_out;
    const int32_t* freed_off;
    int32_t* freed_ids;        // or null
    int32_t* fl_ids;           // free list entries, or null
    const int32_t* fl_base;
    int32_t* slot_pos;         // [U][pos_stride] positions compacted with the rows, or null
    int64_t pos_stride;
    const int32_t* abort_word; // non-zero: the step was vetoed; or null
    int32_t* qwords;           // [kQwWords]
};
bool select_compact_supported(int budget);
cudaError_t launch_select_compact(const SelectCompactParams& p, int num_sms, cudaStream_t stream, bool pdl);

// Phase 2 of the compaction for all units (after launch_evict's phase 1).
struct MoveParams {
    const int32_t* idx;        // [U][budget] kept slots, ascending
    int budget;
    const int32_t* lens;       // [S] lengths before the step
    const int32_t* kept;       // [S], or null: budget for len > trigger, else untouched
    int trigger;               // (>= budget) used when kept is null
    uint8_t* k_pool;
    uint8_t* v_pool;
    const int32_t* block_table;
    int L, Hkv, num_blocks, S, max_blocks;
    int32_t* status;
    const int32_t* unit_info;  // [U][4] m0, J, mode, scratch row (step plans) or null
    uint8_t* scratch;          // rows of K then V (512 bytes each) or null
    const int32_t* scratch_owner;  // [2][scratch_rows] unit and source row of each scratch row
    const int32_t* scratch_used;   // [1] scratch rows handed out
    int scratch_rows;
    int copy_out;              // 1: copy at-risk sources to the scratch; 0: move rows
    const int32_t* abort_word; // non-zero: the step was vetoed, move nothing; or null
};
cudaError_t launch_move(const MoveParams& p, int num_sms, cudaStream_t stream, bool pdl = false);

// Freed-block list + new lengths after a standalone compaction.
struct FinalizeParams {
    int32_t* seq_len;
    const int32_t* kept;
    const int32_t* block_table;
    int S, max_blocks;
    int32_t* freed_ids;
    int32_t* freed_count;
    int32_t* status;
};
cudaError_t launch_finalize(const FinalizeParams& p, cudaStream_t stream);

// ------------------------------------------------------ distance variant
struct DistTableParams {
    const float* qbar;        // [L][Hq][D]
    const float* kbar;        // [L][Hkv][D]
    double base;
    int n_deltas;
    int32_t deltas[TRI_MAX_DELTAS];
    int L, Hkv, G;
    int per_head;             // 1: max over the group, 0: mean (folded)
    int max_dist;
    float* table;             // [L][Hkv][max_dist + 1]
};
cudaError_t launch_distance_table(const DistTableParams& p, cudaStream_t stream);

struct DistScoreParams {
    const float* table;
    int max_dist;
    const int32_t* slot_pos;  // [U][pos_stride]
    int64_t pos_stride;       // max_blocks * 16
    const int64_t* cur_pos;
    const int32_t* lens;      // [S] lengths the step works from (the plan's validated copy)
    const int32_t* seq_len_in; // [S] the caller's lengths (read before the plan completes; bounds prefetches only)
    int trigger;              // units of sequences with len <= trigger are skipped (-1: none)
    float* scores;
    int64_t score_stride;
    uint32_t* unit_kmin;      // [U] or null (initialised by the plan)
    uint32_t* unit_kmax;
    int L, Hkv, S;
    int32_t* status;
};
cudaError_t launch_distance_score(const DistScoreParams& p, cudaStream_t stream, bool pdl = false);

// Pop blocks for n_new[s] more slots per sequence from a device free list.
struct ReserveParams {
    const int32_t* seq_len;
    const int32_t* n_new;
    int32_t* block_table;
    int S, max_blocks, num_blocks;
    int32_t* fl_ids;
    int32_t* fl_count;
    int fl_capacity;
    int32_t* status;
};
cudaError_t launch_reserve(const ReserveParams& p, cudaStream_t stream);

// ---------------------------------------------------------- stats check
struct StatsCheckParams {
    const float* qbar;        // [n_heads][D]
    const float* qabs;        // [n_heads][D/2]
    const float* R;           // [n_heads]
    int64_t n_heads;
    int32_t* head_flags;      // [n_heads] TRI_STATS_* bits, or null
    int32_t* status;          // TRI_DEVFLAG_STATS raised here on a failure
    int32_t* abort_word;      // set to non-zero on a failure (a step's veto), or null
};
cudaError_t launch_check_stats(const StatsCheckParams& p, cudaStream_t stream);

// ------------------------------------------------------------- calibrate
cudaError_t launch_calibrate(const float* q, int N, int L, int Hq, float* qbar, float* qabs, float* R,
                             cudaStream_t stream);

}  // namespace tri
