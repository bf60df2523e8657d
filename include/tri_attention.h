/*
 * tri_attention.h - C ABI of the B200 (sm_100a) TriAttention key-importance
 * and eviction path.
 *
 * The library scores every cached post-rotary key of every (sequence, layer,
 * KV head) unit from calibrated pre-rotary query statistics, keeps the
 * top-B keys of each unit together with a recent window, and packs the kept
 * K/V rows forward inside the sequence's paged blocks so that whole blocks
 * become empty and can be returned to the caller's allocator.
 *
 * Pages cited (title, then section):
 *   [Digest]   "TriAttention: Trigonometric KV Compression for Efficient Long
 *               Reasoning" - "Core Mechanism", "Key Concepts"
 *   [Abstract] "TriAttention: Efficient Long Reasoning with Trigonometric KV
 *               Compression" - "English"
 *   [GeoTrick] "TriAttention: How a Geometric Trick Cuts LLM Memory Use by 10x
 *               Without Losing Accuracy" - "The Core Idea: Q/K Concentration
 *               in Pre-RoPE Space", "Solving the Memory Fragmentation
 *               Problem", "Why Existing KV Cache Compression Breaks in
 *               Production"
 *
 * Notation: D = 128 (head dimension), n = D/2 = 64 rotary bands; band i pairs
 * dimensions (i, i+64) (rotate-half) and turns by theta_i * position with
 * theta_i = base^(-2i/D).  Query head hq = h*G + g belongs to KV head h.
 *
 * Conventions shared by every entry point:
 *  - All array pointers are DEVICE memory owned by the caller, except where an
 *    argument says "host".  The library allocates no device memory: scratch
 *    comes from a caller-provided workspace sized by tri_workspace_size()
 *    (tri_compress_step_static_scratch uses a fixed array instead).
 *  - Every call is asynchronous on the cudaStream_t it is given (0 = the
 *    legacy default stream).  Host-side argument checks run before any
 *    launch; a rejected call launches nothing and changes nothing.
 *  - Errors a kernel can only see on the device (a block id out of range, a
 *    sequence length larger than its table, a NaN score, a bounded wait that
 *    gave up) are OR-ed as TRI_DEVFLAG_* bits into the caller's device status
 *    word (tri_kv_desc.status).  tri_sync_status() reads and clears it.
 *    After a device error the cache contents of the affected sequences are
 *    unspecified; nothing outside the arrays named in the call is touched.
 *  - Return value: TRI_OK, or the first error the host detected.
 *  - Calls that share a descriptor, workspace or output buffers must not run
 *    concurrently on different streams.
 */
#ifndef TRI_ATTENTION_H
#define TRI_ATTENTION_H

#include <stddef.h>
#include <stdint.h>
#include <cuda_runtime_api.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef int tri_status;

#define TRI_OK                 0
#define TRI_ERR_INVALID        1  /* argument rejected on the host            */
#define TRI_ERR_UNSUPPORTED    2  /* valid, but outside this build (D != 128) */
#define TRI_ERR_CUDA           3  /* a CUDA runtime call or launch failed     */
#define TRI_ERR_DEVICE_BOUNDS  4  /* device saw an out-of-range id or length  */
#define TRI_ERR_TIMEOUT        5  /* a bounded device wait gave up            */
#define TRI_ERR_NONFINITE      6  /* a NaN score was seen                     */
#define TRI_ERR_WORKSPACE      7  /* workspace missing, small or misaligned   */
/* TRI_ERR_FREELIST (8): a device free list was too short or full (see the
 * free-list calls below). */

/* Bits of the device status word. */
#define TRI_DEVFLAG_BOUNDS     1
#define TRI_DEVFLAG_TIMEOUT    2
#define TRI_DEVFLAG_NONFINITE  4

#define TRI_HEAD_DIM        128
#define TRI_BLOCK_SIZE      16
#define TRI_MAX_DELTAS      64
#define TRI_MAX_BUDGET      16384

/*
 * The paged KV cache ([GeoTrick] "Why Existing KV Cache Compression Breaks
 * in Production": fixed-size physical blocks handed out by a paged
 * allocator).
 *
 *   k_pool, v_pool : bf16 [L][num_blocks][Hkv][block_size][D], 16-byte
 *                    aligned; one (block, head) tile of 16 rows x 128 is
 *                    4 KiB and contiguous.  Post-rotary keys; values.
 *   block_table    : int32 [S][max_blocks]; entry b of sequence s is the pool
 *                    block holding its slots 16b .. 16b+15, for every layer
 *                    and head.  Only the first ceil(seq_len[s]/16) entries
 *                    are read; each must lie in [0, num_blocks) and no block
 *                    may appear twice among the entries in use.
 *   seq_len        : int32 [S]; cached slots per (layer, head) of each
 *                    sequence, in [0, max_blocks*16].  Compaction rewrites it.
 *   cur_pos        : int64 [S]; position p of each sequence's next query.
 *   status         : int32 [1]; device status word (TRI_DEVFLAG_* bits).
 *   L, Hkv, G      : layers, KV heads per layer, query heads per KV head.
 *   D, block_size  : must be 128 and 16 (TRI_ERR_UNSUPPORTED otherwise).
 */
typedef struct {
    int L, Hkv, G, D, block_size;
    void *k_pool;
    void *v_pool;
    int num_blocks;
    const int32_t *block_table;
    int S, max_blocks;
    int32_t *seq_len;
    const int64_t *cur_pos;
    int32_t *status;
} tri_kv_desc;

/* Optional phase timing: events recorded on the call's stream before the
 * first launch and after each phase of tri_compress_step.  Any member may be
 * NULL.  The events must have been created by the caller. */
typedef struct {
    cudaEvent_t start;          /* before the query build                   */
    cudaEvent_t after_query;    /* after the effective-query build          */
    cudaEvent_t after_score;    /* after the score pass over all keys       */
    cudaEvent_t after_evict;    /* after selection and compaction           */
} tri_phase_events;

/*
 * tri_calibrate_centers - reduce pre-rotary query samples to head statistics
 * ([Digest] "Core Mechanism", one-time centre calibration; "Key Concepts",
 * Q/K Concentration; [GeoTrick] "The Core Idea", measured concentration).
 *
 *   q_pre : f32 [N][L][Hq][D] samples of the pre-rotary query (any N >= 1)
 *   qbar  : f32 [L][Hq][D] out, the centre: mean sample (bands as dims i, i+64)
 *   qabs  : f32 [L][Hq][D/2] out, A_i = mean over samples of |band i|
 *   R     : f32 [L][Hq] out, concentration sum_i |qbar_i| / sum_i A_i in
 *           [0, 1]; 1 when every sample is zero
 * Accumulates in float64.  Works for keys too (pass key samples).
 * Errors: TRI_ERR_INVALID (null pointer, N/L/Hq < 1, size overflow),
 * TRI_ERR_UNSUPPORTED (D != 128), TRI_ERR_CUDA.
 */
tri_status tri_calibrate_centers(const float *q_pre, int N, int L, int Hq, int D,
                                 float *qbar, float *qabs, float *R,
                                 cudaStream_t stream);

/*
 * tri_build_query - the effective query of every unit, folded over its GQA
 * group ([Digest] "Key Concepts", Trigonometric Distance Preference; future
 * query positions p + delta averaged over the offset list):
 *
 *   m_i      = mean_delta exp(j theta_i (cur_pos[s] + delta))   (float64)
 *   qeff     = real dims of mean_g qbar_{g,i} * m_i              [S][L][Hkv][D]
 *   w_i      = mean_g (1 - R_g) (qabs_{g,i} - |qbar_{g,i}|)      [S][L][Hkv][D/2]
 *
 * so that the group score of a key K is qeff . K + sum_i w_i |K band i|.
 *   qbar, qabs, R : statistics as produced by tri_calibrate_centers, for
 *                   Hq = Hkv*G query heads
 *   rope_base     : rotary base (> 0)
 *   deltas        : HOST int32 [n_deltas], 1 <= n_deltas <= TRI_MAX_DELTAS;
 *                   read during the call only
 *   qeff, w       : f32 outputs, layouts above
 * Errors: TRI_ERR_INVALID, TRI_ERR_UNSUPPORTED, TRI_ERR_CUDA.
 */
tri_status tri_build_query(const tri_kv_desc *desc, const float *qbar, const float *qabs,
                           const float *R, double rope_base, const int32_t *deltas,
                           int n_deltas, float *qeff, float *w, cudaStream_t stream);

/*
 * tri_workspace_size - bytes of device workspace that tri_score and
 * tri_compress_step need for this descriptor's shape.  The workspace must be
 * 256-byte aligned.  Depends on S, L, Hkv and max_blocks only.
 * Returns 0 for an invalid descriptor.
 */
size_t tri_workspace_size(const tri_kv_desc *desc, int budget);

/*
 * tri_score - score every cached key of every unit ([Digest] "Key
 * Concepts"; [Abstract] "English"; [GeoTrick] "The Core Idea"):
 *
 *   s(t) = qeff . K_t + sum_i w_i sqrt(K_{t,i}^2 + K_{t,i+64}^2)
 *
 * which equals the mean over the G query heads of
 *   sum_i Re(qbar_i m_i conj(K_t band i)) + (1 - R)(qabs_i - |qbar_i|)|K_t band i|.
 * bf16 keys, fp32 arithmetic, streamed once from HBM.
 *   scores : f32 [S][L][Hkv][max_blocks*16]; entry t of unit (s, l, h) is
 *            written for t < seq_len[s]; the rest is left untouched.
 *   workspace, ws_bytes : >= tri_workspace_size(desc, 1) bytes.
 * Errors: as tri_build_query, plus TRI_ERR_WORKSPACE.  Device flags: BOUNDS
 * (seq_len or a block id out of range: those keys are skipped), TIMEOUT.
 */
tri_status tri_score(const tri_kv_desc *desc, const float *qbar, const float *qabs,
                     const float *R, double rope_base, const int32_t *deltas, int n_deltas,
                     float *scores, void *workspace, size_t ws_bytes, cudaStream_t stream);

/*
 * tri_select_topk - the kept slots of every unit ([Digest] "Core Mechanism":
 * keep only the top-scoring subset).  For a unit of len = seq_len[s] slots:
 *   len <= budget : every slot is kept;
 *   otherwise     : the last `window` slots, plus the (budget - window) best of
 *                   the other slots by (score descending, slot ascending).
 * -0 equals +0; a NaN score ranks as -infinity and sets TRI_DEVFLAG_NONFINITE.
 *   scores : f32 [S][L][Hkv][max_blocks*16] (as written by tri_score),
 *            16-byte aligned
 *   budget : B >= 1, at most TRI_MAX_BUDGET; window: 0 <= W <= B
 *   idx    : int32 [S][L][Hkv][budget] out; the kept slots ascending in the
 *            first kept[s] entries, -1 after them
 *   kept   : int32 [S] out; min(seq_len[s], budget)
 * Errors: TRI_ERR_INVALID, TRI_ERR_UNSUPPORTED, TRI_ERR_CUDA.
 */
tri_status tri_select_topk(const tri_kv_desc *desc, const float *scores, int budget,
                           int window, int32_t *idx, int32_t *kept, cudaStream_t stream);

/*
 * tri_compact_kv - Forward-Packing Compaction ([GeoTrick] "Solving the
 * Memory Fragmentation Problem"): for every unit and j < kept[s], row j of K
 * and of V takes old row idx[j], in place across the sequence's blocks, in
 * order.  Then seq_len[s] = kept[s], and the blocks
 * block_table[s][ceil(kept/16) .. ceil(old_len/16)) are appended to
 * freed_ids (sequence order, table order); *freed_count = their number.
 *   idx   : int32 [S][L][Hkv][budget], each unit's first kept[s] entries
 *           strictly ascending and < seq_len[s] (as from tri_select_topk)
 *   kept  : int32 [S], 0 <= kept[s] <= seq_len[s], and kept[s] <= budget
 *           unless kept[s] == seq_len[s] (the sequence is left as it is)
 *   freed_ids   : int32 [S*max_blocks] out;  freed_count : int32 [1] out
 * The block table is not modified; the caller truncates it.
 * Errors: TRI_ERR_INVALID, TRI_ERR_UNSUPPORTED, TRI_ERR_CUDA.  Device flags:
 * BOUNDS (an index, kept count or block id out of range: skipped).
 */
tri_status tri_compact_kv(tri_kv_desc *desc, const int32_t *idx, const int32_t *kept,
                          int budget, int32_t *freed_ids, int32_t *freed_count,
                          cudaStream_t stream);

/*
 * tri_compress_step - the whole step: effective query, score, select and
 * compact for every unit of every sequence whose seq_len exceeds `budget`;
 * shorter sequences are left untouched.  Same results as tri_score ->
 * tri_select_topk -> tri_compact_kv, without materialising scores outside the
 * workspace.
 *   idx_out : optional int32 [S][L][Hkv][budget]; when not NULL receives the
 *             kept slots of every compressed unit (entries of sequences left
 *             untouched are not written)
 *   events  : optional phase timing (see tri_phase_events)
 *   workspace, ws_bytes : >= tri_workspace_size(desc, budget) bytes
 * Errors and flags: union of the three calls above.
 */
tri_status tri_compress_step(tri_kv_desc *desc, const float *qbar, const float *qabs,
                             const float *R, double rope_base, const int32_t *deltas,
                             int n_deltas, int budget, int window, int32_t *freed_ids,
                             int32_t *freed_count, int32_t *idx_out, void *workspace,
                             size_t ws_bytes, const tri_phase_events *events,
                             cudaStream_t stream);

/*
 * tri_compress_step_static_scratch - tri_compress_step without a workspace
 * argument, for callers that cannot allocate device memory.  (The pages
 * describe nothing like it: it exists only for how this library is called.)
 *
 * Who needs it: callers that have no way to obtain device scratch, such as
 * a serving engine that hands nearly all HBM to its paged KV block pool at
 * start-up and forbids allocation on the decode path, or a plain-C plugin
 * loaded into such an engine without an allocator of its own.
 *
 * Instead of a caller workspace it uses one fixed array of
 * TRI_STATIC_SCRATCH_BYTES of device memory built into the library; every
 * GPU that loads the library holds that array until the process exits.
 *   - Shapes whose tri_workspace_size(desc, budget) exceeds
 *     TRI_STATIC_SCRATCH_BYTES are rejected with TRI_ERR_UNSUPPORTED before
 *     anything is launched (use tri_compress_step with a workspace instead).
 *   - The first call in a CUDA context looks up the array's device address
 *     (cudaGetSymbolAddress) with that context current and caches it, keyed
 *     by the context's unique id; make that first call before capturing the
 *     stream into a CUDA graph.  The array belongs to the context: after
 *     cudaDeviceReset (or anything else that destroys the device's context)
 *     the next call runs in a new context, holding a new copy of the array,
 *     and looks the address up again, so no call ever uses an address of a
 *     destroyed context.  Nothing of an earlier context's scratch survives.
 *   - All calls share the one array and it keeps the last call's contents.
 *     Every call rewrites all of the scratch it reads, so nothing in it needs
 *     to start at zero; but two calls whose work overlaps on the GPU (other
 *     streams, other host threads) race on it and must not be issued.
 *   - It allocates nothing: no cudaMalloc, cudaFree or allocating library
 *     routine is called.
 * Arguments, results, errors and device flags: as tri_compress_step (no
 * phase events).
 */
#define TRI_STATIC_SCRATCH_BYTES (16u << 20)
/* The size of that array as built into this library (TRI_STATIC_SCRATCH_BYTES
 * of the header it was compiled with); a host-only query, no CUDA call. */
size_t tri_static_scratch_bytes(void);
tri_status tri_compress_step_static_scratch(tri_kv_desc *desc, const float *qbar, const float *qabs,
                                            const float *R, double rope_base, const int32_t *deltas,
                                            int n_deltas, int budget, int window, int32_t *freed_ids,
                                            int32_t *freed_count, int32_t *idx_out, cudaStream_t stream);

/* ------------------------------------------------------------------------
 * Variants of the step.
 *
 * tri_step_options gathers the knobs of the selection and of the GQA
 * aggregation; the plain entry points above are the defaults
 * {budget, window, 0, 0, TRI_AGG_MEAN}.
 *
 *   budget    : B, slots kept per unit, 1 <= B <= TRI_MAX_BUDGET.
 *   window    : W, the last W slots are always kept (inside B).
 *   sinks     : the first `sinks` slots (the oldest tokens of the sequence)
 *               are always kept, also inside B: sinks + W <= B.  With
 *               sinks > 0 the selection ranks only slots [sinks, len - W)
 *               and keeps the best B - W - sinks of them.  ([Digest] "Key
 *               Concepts" and [GeoTrick] "The Core Idea" note that attention
 *               mass concentrates on a few early positions; keeping them is
 *               an option of this library, not a step of the method.)
 *   trigger   : a sequence is compressed only when seq_len > max(trigger, B);
 *               shorter sequences are left untouched.  0 means B.  A caller
 *               that appends chunks of C tokens between steps and sets
 *               trigger = B + C compresses once per chunk instead of after
 *               every token ([GeoTrick] "Why Existing KV Cache Compression
 *               Breaks in Production": eviction in whole chunks).
 *   aggregate : how the G query heads of a KV head combine into one key
 *               score.  TRI_AGG_MEAN: their mean, folded into one effective
 *               query (what tri_build_query computes).  TRI_AGG_MAX: their
 *               maximum, each head scored on its own; G must be 1, 2, 4 or 8
 *               (TRI_ERR_UNSUPPORTED otherwise).
 *   check_stats : non-zero: tri_compress_step_ex first runs the checks of
 *               tri_check_stats on the statistics it is given; if any head
 *               fails them (NONFINITE, R_RANGE or NORM_WEIGHT below), it
 *               raises TRI_DEVFLAG_STATS and changes nothing: no row moves,
 *               seq_len, the free list and idx_out are left as they are and
 *               *freed_count = 0.  Costs one small extra launch.  Ignored by
 *               the selection-only and distance-table entry points.
 * ---------------------------------------------------------------------- */
#define TRI_AGG_MEAN 0
#define TRI_AGG_MAX  1

typedef struct {
    int budget;
    int window;
    int sinks;
    int trigger;
    int aggregate;
    int check_stats;
} tri_step_options;

/*
 * A device-resident stack of free paged-block ids, so that a decode loop can
 * compress and grow its sequences without the host reading freed ids back.
 *   ids      : int32 [capacity]; entries [0, *count) are free block ids
 *   count    : int32 [1], device; the number of valid entries
 *   capacity : entries ids can hold
 * The library pushes freed blocks on top (tri_compress_step_ex) and pops
 * from the top (tri_reserve_blocks).  Only the calls it is passed to touch it.
 */
typedef struct {
    int32_t *ids;
    int32_t *count;
    int capacity;
} tri_free_list;

/* Device status bit: a free list had too few entries (pop) or too little
 * room (push); that call changed neither the list nor the block table. */
#define TRI_DEVFLAG_FREELIST   8
#define TRI_ERR_FREELIST       8  /* tri_sync_status: TRI_DEVFLAG_FREELIST */

/*
 * tri_check_stats - check head statistics before a step uses them ([Review]
 * "Calibration statistics are tied to a specific model": statistics of
 * another model, or a damaged statistics file, raise no error by
 * themselves; the step only keeps the wrong keys).  For every one of the
 * n = L*Hq heads (qbar [L][Hq][D], qabs [L][Hq][D/2], R [L][Hq], as for
 * tri_build_query) it checks what any valid statistics satisfy:
 *   TRI_STATS_NONFINITE   a NaN or infinity in the head's qbar, qabs or R;
 *   TRI_STATS_R_RANGE     R outside [0, 1];
 *   TRI_STATS_NORM_WEIGHT qabs_i < |qbar_i| for some band beyond a relative
 *                         1e-5 (a mean of magnitudes is never below the
 *                         magnitude of the mean; a negative norm weight
 *                         (1 - R)(qabs_i - |qbar_i|) inverts the ranking);
 * and reports, without treating it as a failure,
 *   TRI_STATS_R_MISMATCH  R differs from sum_i |qbar_i| / sum_i qabs_i (the
 *                         concentration tri_calibrate_centers computes) by
 *                         more than 1e-3 relative.
 *   head_flags : NULL, or int32 [L][Hq] out: the bits above per head
 *   status     : device status word; TRI_DEVFLAG_STATS is OR-ed into it if
 *                any head has NONFINITE, R_RANGE or NORM_WEIGHT
 * Errors: TRI_ERR_INVALID (null or misaligned pointer, L or Hq < 1, size
 * overflow), TRI_ERR_UNSUPPORTED (D != 128), TRI_ERR_CUDA.  Asynchronous:
 * tri_sync_status() returns TRI_ERR_STATS when the flag was raised.
 */
#define TRI_STATS_NONFINITE    1
#define TRI_STATS_R_RANGE      2
#define TRI_STATS_NORM_WEIGHT  4
#define TRI_STATS_R_MISMATCH   8
/* Device status bit: statistics failed the check (tri_check_stats, or a step
 * run with check_stats, which then changed nothing). */
#define TRI_DEVFLAG_STATS      16
#define TRI_ERR_STATS          9  /* tri_sync_status: TRI_DEVFLAG_STATS */
tri_status tri_check_stats(const float *qbar, const float *qabs, const float *R, int L, int Hq, int D,
                           int32_t *head_flags, int32_t *status, cudaStream_t stream);

/* Workspace bytes of tri_score_ex / tri_compress_step_ex with these options
 * (TRI_AGG_MAX keeps G coefficient sets per unit).  0 if invalid. */
size_t tri_workspace_size_ex(const tri_kv_desc *desc, const tri_step_options *opt);

/*
 * tri_score_ex - tri_score with a choice of aggregation.  TRI_AGG_MEAN is
 * tri_score.  TRI_AGG_MAX writes, for every key,
 *   max_g [ sum_i Re(qbar_{g,i} m_i conj(K band i))
 *           + (1 - R_g)(qabs_{g,i} - |qbar_{g,i}|)|K band i| ].
 *   workspace : >= tri_workspace_size_ex(desc, {1, 0, 0, 0, aggregate}).
 * Errors and flags: as tri_score; TRI_ERR_UNSUPPORTED for TRI_AGG_MAX with
 * G not in {1, 2, 4, 8}; TRI_ERR_INVALID for an unknown aggregate.
 */
tri_status tri_score_ex(const tri_kv_desc *desc, const float *qbar, const float *qabs,
                        const float *R, double rope_base, const int32_t *deltas, int n_deltas,
                        int aggregate, float *scores, void *workspace, size_t ws_bytes,
                        cudaStream_t stream);

/*
 * tri_select_topk_ex - tri_select_topk with sinks and a trigger: a unit of
 * len <= max(trigger, budget) keeps every slot (kept = len; when len > B the
 * idx entries are 0 .. B-1, as there is room for no more); otherwise it
 * keeps slots [0, sinks), the last W slots and the best B - W - sinks of the
 * slots between (score descending, slot ascending), kept = B.  tri_compact_kv
 * leaves a sequence with kept == seq_len untouched, so the two chain.
 * opt->aggregate is ignored.  Errors: as tri_select_topk, and
 * TRI_ERR_INVALID for sinks < 0, sinks + W > B or trigger < 0.
 */
tri_status tri_select_topk_ex(const tri_kv_desc *desc, const float *scores,
                              const tri_step_options *opt, int32_t *idx, int32_t *kept,
                              cudaStream_t stream);

/*
 * tri_compress_step_ex - tri_compress_step with options and an optional
 * device free list.
 *   opt        : the options above (not NULL).
 *   free_list  : NULL, or a free list that receives the freed block ids: they
 *                are pushed on top in the order tri_compress_step reports
 *                them, and *free_list->count grows by their number.  If the
 *                list lacks room, nothing is pushed and TRI_DEVFLAG_FREELIST
 *                is raised (the cache is still compacted and freed_ids, when
 *                given, still lists the blocks).
 *   freed_ids, freed_count : as tri_compress_step; may both be NULL when a
 *                free list is given.
 *   workspace  : >= tri_workspace_size_ex(desc, opt) bytes.
 * Sequences with seq_len <= max(trigger, budget) are left untouched.
 * Errors and flags: as tri_compress_step, plus TRI_DEVFLAG_FREELIST.
 */
tri_status tri_compress_step_ex(tri_kv_desc *desc, const float *qbar, const float *qabs,
                                const float *R, double rope_base, const int32_t *deltas,
                                int n_deltas, const tri_step_options *opt,
                                const tri_free_list *free_list, int32_t *freed_ids,
                                int32_t *freed_count, int32_t *idx_out, void *workspace,
                                size_t ws_bytes, const tri_phase_events *events,
                                cudaStream_t stream);

/*
 * tri_step_is_fused - 1 if a step with these options (tri_compress_step,
 * tri_compress_step_ex, tri_compress_step_distance) selects and compacts
 * in one persistent kernel after its score pass, 0 if it runs selection,
 * copy-out and move as separate kernels, -1 for an invalid descriptor or
 * options.  The results are the same either way; only the launch sequence
 * differs.  The persistent kernel serves every step (two CTAs per SM up to
 * budget 4096, one above) unless the environment sets TRI_UNFUSED_STEP=1.
 * Host-only, no CUDA work is queued.
 */
int tri_step_is_fused(const tri_kv_desc *desc, const tri_step_options *opt);

/*
 * tri_reserve_blocks - grow sequences by n_new[s] slots each, taking the
 * paged blocks they newly need from the top of a device free list
 * ([GeoTrick] "Why Existing KV Cache Compression Breaks in Production": the
 * paged allocator hands out whole blocks).
 *   block_table : int32 [S][max_blocks], the descriptor's table, writable;
 *                 entries ceil(seq_len/16) .. ceil((seq_len+n_new)/16) - 1 of
 *                 sequence s are set.  Sequences take the popped ids in
 *                 sequence order, each sequence in table order, from the
 *                 lowest of the popped entries up.
 *   n_new       : int32 [S], device, >= 0.
 * seq_len is NOT changed: the caller writes the new rows and then raises it.
 * All or nothing: if the list holds fewer ids than needed, or a sequence
 * would exceed max_blocks*16 slots, nothing changes and the device flags
 * FREELIST or BOUNDS are raised.
 * Errors: TRI_ERR_INVALID, TRI_ERR_UNSUPPORTED, TRI_ERR_CUDA.
 */
tri_status tri_reserve_blocks(const tri_kv_desc *desc, int32_t *block_table, const int32_t *n_new,
                              const tri_free_list *free_list, cudaStream_t stream);

/* ------------------------------------------------------------------------
 * Variant: distance-only scores ([Digest] "Core Mechanism": the
 * trigonometric series of the distance evaluated as lookups indexed by
 * relative position; "Key Concepts", Trigonometric Distance Preference: the
 * rotated centres' dot product depends on the query-key distance only).
 *
 * The key is replaced by its head's key centre kbar (the pre-rotary mean of
 * that head's keys, e.g. tri_calibrate_centers run on key samples), so a
 * key's score depends on its distance d = p - pos to the query alone and
 * comes from a table built once.  The centres' norm term is the same for
 * every key of a unit and is left out (it cannot change a ranking).
 * ---------------------------------------------------------------------- */

/*
 * tri_distance_table - f(d) for d = 0 .. max_dist of every (layer, KV head):
 *   f(d) = agg_g mean_delta sum_i Re( qbar_{g,i} conj(kbar_i) exp(j theta_i (d + delta)) )
 * agg = mean (TRI_AGG_MEAN) or max (TRI_AGG_MAX) over the G query heads of
 * the KV head.  Float64 arithmetic, stored fp32.
 *   L, Hkv, G, D : shapes (Hq = Hkv*G; D must be 128)
 *   qbar   : f32 [L][Hq][D] query centres;  kbar : f32 [L][Hkv][D] key centres
 *   deltas : HOST int32 [n_deltas], 1 <= n_deltas <= TRI_MAX_DELTAS
 *   max_dist : 1 <= max_dist < 2^24
 *   table  : f32 [L][Hkv][max_dist + 1] out
 * Errors: TRI_ERR_INVALID, TRI_ERR_UNSUPPORTED (D != 128; TRI_AGG_MAX with
 * G > 64), TRI_ERR_CUDA.
 */
tri_status tri_distance_table(int L, int Hkv, int G, int D, const float *qbar, const float *kbar,
                              double rope_base, const int32_t *deltas, int n_deltas, int aggregate,
                              int max_dist, float *table, cudaStream_t stream);

/*
 * tri_score_distance - scores[s][l][h][t] = table[l][h][cur_pos[s] - pos] with
 * pos = slot_pos[s][l][h][t], for t < seq_len[s]; the rest is not written.
 *   slot_pos : int32 [S][L][Hkv][max_blocks*16], 16-byte aligned: the position
 *              each slot's key was cached at (slot_pos[...][t] = t for a cache
 *              never compacted)
 *   table, max_dist : as built by tri_distance_table for this cache's L, Hkv
 *   scores   : f32 [S][L][Hkv][max_blocks*16], 16-byte aligned
 * A distance outside [0, max_dist] raises TRI_DEVFLAG_BOUNDS (the nearest
 * table entry is used).  Errors: TRI_ERR_INVALID, TRI_ERR_UNSUPPORTED,
 * TRI_ERR_CUDA.
 */
tri_status tri_score_distance(const tri_kv_desc *desc, const float *table, int max_dist,
                              const int32_t *slot_pos, float *scores, cudaStream_t stream);

/*
 * tri_compress_step_distance - tri_compress_step_ex with the table's scores:
 * no pass over the cached keys.  slot_pos (layout as above) is compacted with
 * the rows: slot j of a compressed unit takes the position of old slot
 * idx[j].  opt->aggregate is ignored (the table fixes it).
 *   workspace : >= tri_workspace_size(desc, opt->budget) bytes.
 * Other arguments, results, errors and flags: as tri_compress_step_ex.
 */
tri_status tri_compress_step_distance(tri_kv_desc *desc, const float *table, int max_dist,
                                      int32_t *slot_pos, const tri_step_options *opt,
                                      const tri_free_list *free_list, int32_t *freed_ids,
                                      int32_t *freed_count, int32_t *idx_out, void *workspace,
                                      size_t ws_bytes, const tri_phase_events *events,
                                      cudaStream_t stream);

/*
 * tri_sync_status - wait for `stream`, read the device status word, clear it,
 * and return TRI_OK or the error its bits name (BOUNDS before TIMEOUT before
 * FREELIST before STATS before NONFINITE).  TRI_ERR_CUDA if the stream itself
 * reports an error.
 */
tri_status tri_sync_status(int32_t *status, cudaStream_t stream);

/* Static, human-readable name of a status code. */
const char *tri_status_string(tri_status s);

/*
 * tri_selftest_bounded_wait - test aid for the device error contract: one
 * thread runs a device wait that nothing completes, under the same rule as
 * every wait of the library's kernels (it gives up after 2 s), then ORs
 * TRI_DEVFLAG_TIMEOUT into *status; tri_sync_status() then returns
 * TRI_ERR_TIMEOUT and the context stays usable.
 *   status : device int32 status word (caller-owned, 4-byte aligned).
 *   flag   : null - wait on a shared-memory barrier that never completes;
 *            else a device int32 the wait polls (acquire, GPU scope) and
 *            that ends the wait as soon as it is non-zero (no timeout then).
 * Returns TRI_ERR_INVALID for a null or misaligned status or flag,
 * TRI_ERR_CUDA if the launch fails, else TRI_OK (asynchronous on `stream`).
 */
tri_status tri_selftest_bounded_wait(int32_t *status, const int32_t *flag, cudaStream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* TRI_ATTENTION_H */
