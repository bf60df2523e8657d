// tri_abi.cu - the extern "C" entry points declared in tri_attention.h.
//
// Host side only: argument checks (before any launch), workspace carving,
// and the launch sequence of each call on the caller's stream.  Every
// arithmetic step of the path runs in the kernels of calibrate.cu, query.cu,
// score.cu and evict.cu.
#include <climits>
#include <cmath>
#include <cstdint>
#include <cstdlib>
#include <mutex>

#include "tri_attention.h"
#include "tri_internal.h"

using namespace tri;

namespace {

constexpr size_t kWsAlign = 256;

size_t align_up(size_t x) { return (x + kWsAlign - 1) & ~(kWsAlign - 1); }

struct WsLayout {
    size_t qeff, wts, len_ws, item_off, freed_off, kmin, kmax, scores, idx, words, info, owner, scratch, fq, total;
    int scratch_rows;
};

// Rows of the compaction scratch: a quarter of the kept rows of all units
// (units that do not fit compact their at-risk prefix in place instead).
int scratch_rows_for(const tri_kv_desc* d, int budget) {
    const int64_t rows = (int64_t)d->S * d->L * d->Hkv * (budget > 0 ? budget : 0) / 4;
    if (budget <= 0) return 0;
    return (int)(rows < 64 ? 64 : (rows > (1 << 24) ? (1 << 24) : rows));
}

// Workspace of a step with budget `budget` (0: the score-only part);
// per_head: G coefficient sets per unit (max over the group).
WsLayout ws_layout(const tri_kv_desc* d, int budget, bool per_head = false) {
    const size_t U = (size_t)d->S * d->L * d->Hkv;
    const size_t sets = U * (per_head ? (size_t)d->G : 1);
    const size_t max_len = (size_t)d->max_blocks * kBlockRows;
    WsLayout w;
    size_t off = 0;
    w.qeff = off;      off = align_up(off + sets * kHeadDim * sizeof(float));
    w.wts = off;       off = align_up(off + sets * kBands * sizeof(float));
    w.len_ws = off;    off = align_up(off + (size_t)d->S * sizeof(int32_t));
    w.item_off = off;  off = align_up(off + ((size_t)d->S + 1) * sizeof(int32_t));
    w.freed_off = off; off = align_up(off + ((size_t)d->S + 1) * sizeof(int32_t));
    w.kmin = off;      off = align_up(off + U * sizeof(uint32_t));
    w.kmax = off;      off = align_up(off + U * sizeof(uint32_t));
    w.scores = off;    off = align_up(off + U * max_len * sizeof(float));
    w.idx = off;       off = align_up(off + U * (size_t)(budget > 0 ? budget : 0) * sizeof(int32_t));
    w.scratch_rows = scratch_rows_for(d, budget);
    const size_t per_unit = budget > 0 ? 1 : 0;
    w.words = off;     off = align_up(off + 4 * sizeof(int32_t) * per_unit);   // scratch rows used, 0, free-list base, statistics veto
    w.info = off;      off = align_up(off + U * 4 * sizeof(int32_t) * per_unit);
    w.owner = off;     off = align_up(off + (size_t)w.scratch_rows * 2 * sizeof(int32_t));
    w.scratch = off;   off = align_up(off + (size_t)w.scratch_rows * 2 * kHeadDim * 2);
    // select + compact kernel: its unit counter
    w.fq = off;        off = align_up(off + (size_t)kQwWords * sizeof(int32_t) * per_unit);
    w.total = off;
    return w;
}

template <typename T>
bool aligned(const T* p, size_t a) { return ((uintptr_t)p % a) == 0; }

tri_status check_desc(const tri_kv_desc* d) {
    if (d == nullptr) return TRI_ERR_INVALID;
    if (d->L < 1 || d->Hkv < 1 || d->G < 1 || d->S < 0 || d->num_blocks < 1 || d->max_blocks < 1)
        return TRI_ERR_INVALID;
    if (d->D != TRI_HEAD_DIM || d->block_size != TRI_BLOCK_SIZE) return TRI_ERR_UNSUPPORTED;
    if (!d->k_pool || !d->v_pool || !d->block_table || !d->seq_len || !d->cur_pos || !d->status)
        return TRI_ERR_INVALID;
    if (!aligned(d->k_pool, 16) || !aligned(d->v_pool, 16) || !aligned(d->block_table, 4) ||
        !aligned(d->seq_len, 4) || !aligned(d->cur_pos, 8) || !aligned(d->status, 4))
        return TRI_ERR_INVALID;
    const int64_t U = (int64_t)d->S * d->L * d->Hkv;
    const int64_t Hq = (int64_t)d->Hkv * d->G;
    const int64_t max_len = (int64_t)d->max_blocks * kBlockRows;
    const int64_t items = (int64_t)d->S * d->L * d->Hkv * ((d->max_blocks + kChunkBlocks - 1) / kChunkBlocks);
    if (U > INT_MAX || Hq > INT_MAX || max_len > INT_MAX || items > INT_MAX) return TRI_ERR_INVALID;
    if ((int64_t)d->L * d->num_blocks * d->Hkv > INT64_MAX / kTileBytes) return TRI_ERR_INVALID;
    return TRI_OK;
}

tri_status check_stats(const float* qbar, const float* qabs, const float* R) {
    if (!qbar || !qabs || !R) return TRI_ERR_INVALID;
    if (!aligned(qbar, 4) || !aligned(qabs, 4) || !aligned(R, 4)) return TRI_ERR_INVALID;
    return TRI_OK;
}

tri_status check_query_args(double base, const int32_t* deltas, int n_deltas) {
    if (!(base > 0.0) || !std::isfinite(base)) return TRI_ERR_INVALID;
    if (deltas == nullptr || n_deltas < 1 || n_deltas > TRI_MAX_DELTAS) return TRI_ERR_INVALID;
    return TRI_OK;
}

tri_status check_budget(int budget, int window) {
    if (budget < 1 || window < 0 || window > budget) return TRI_ERR_INVALID;
    if (budget > TRI_MAX_BUDGET) return TRI_ERR_UNSUPPORTED;
    return TRI_OK;
}

tri_status check_workspace(const tri_kv_desc* d, const void* ws, size_t ws_bytes, int budget,
                           bool per_head = false) {
    if (ws == nullptr || ((uintptr_t)ws % kWsAlign) != 0) return TRI_ERR_WORKSPACE;
    if (ws_bytes < ws_layout(d, budget, per_head).total) return TRI_ERR_WORKSPACE;
    return TRI_OK;
}

tri_status check_aggregate(int aggregate, int G) {
    if (aggregate == TRI_AGG_MEAN) return TRI_OK;
    if (aggregate != TRI_AGG_MAX) return TRI_ERR_INVALID;
    return (G == 1 || G == 2 || G == 4 || G == 8) ? TRI_OK : TRI_ERR_UNSUPPORTED;
}

// Options of a selection / step; G for the aggregate check (0: not checked).
tri_status check_options(const tri_step_options* o, int G) {
    if (o == nullptr) return TRI_ERR_INVALID;
    tri_status st = check_budget(o->budget, o->window);
    if (st != TRI_OK) return st;
    if (o->sinks < 0 || o->trigger < 0 || (int64_t)o->sinks + o->window > o->budget) return TRI_ERR_INVALID;
    return G > 0 ? check_aggregate(o->aggregate, G) : TRI_OK;
}

int effective_trigger(const tri_step_options& o) { return o.trigger > o.budget ? o.trigger : o.budget; }

// TRI_UNFUSED_STEP=1 in the environment makes a step run its selection and
// compaction as separate kernels (selection, copy-out, move) even where the
// persistent select + compact kernel applies; both give the same results.
// Read once.
bool unfused_step_forced() {
    static const bool forced = [] {
        const char* v = std::getenv("TRI_UNFUSED_STEP");
        return v != nullptr && v[0] == '1';
    }();
    return forced;
}

tri_status check_free_list(const tri_free_list* fl) {
    if (fl == nullptr) return TRI_OK;
    if (!fl->ids || !fl->count || fl->capacity < 0 || !aligned(fl->ids, 4) || !aligned(fl->count, 4))
        return TRI_ERR_INVALID;
    return TRI_OK;
}

tri_status cuda_status(cudaError_t e) { return e == cudaSuccess ? TRI_OK : TRI_ERR_CUDA; }

// Whether a step with this budget selects and compacts in the persistent
// select + compact kernel (select_compact.cu).
bool persistent_compaction(int budget) { return !unfused_step_forced() && select_compact_supported(budget); }

int device_sm_count() {
    static std::mutex mu;
    static int cache[128] = {0};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 128) return 148;
    std::lock_guard<std::mutex> lock(mu);
    if (cache[dev] == 0) {
        int n = 0;
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n < 1) n = 148;
        cache[dev] = n;
    }
    return cache[dev];
}

QueryParams make_query_params(const tri_kv_desc* d, const float* qbar, const float* qabs, const float* R,
                              double base, const int32_t* deltas, int n_deltas, float* qeff, float* wts) {
    QueryParams q{};
    q.qbar = qbar;
    q.qabs = qabs;
    q.R = R;
    q.cur_pos = d->cur_pos;
    q.base = base;
    q.n_deltas = n_deltas;
    for (int i = 0; i < n_deltas; ++i) q.deltas[i] = deltas[i];
    q.qeff = qeff;
    q.wts = wts;
    q.L = d->L;
    q.Hkv = d->Hkv;
    q.G = d->G;
    q.S = d->S;
    q.seq_len = d->seq_len;
    q.max_blocks = d->max_blocks;
    q.heads_per_tile = score_heads_per_tile(d->Hkv);
    q.status = d->status;
    return q;
}

ScoreParams make_score_params(const tri_kv_desc* d, const uint8_t* ws, const WsLayout& w, float* scores,
                              int64_t stride) {
    ScoreParams s{};
    s.k_pool = static_cast<const uint8_t*>(d->k_pool);
    s.block_table = d->block_table;
    s.len_ws = reinterpret_cast<const int32_t*>(ws + w.len_ws);
    s.item_off = reinterpret_cast<const int32_t*>(ws + w.item_off);
    s.qeff = reinterpret_cast<const float*>(ws + w.qeff);
    s.wts = reinterpret_cast<const float*>(ws + w.wts);
    s.scores = scores;
    s.score_stride = stride;
    s.unit_kmin = reinterpret_cast<uint32_t*>(const_cast<uint8_t*>(ws) + w.kmin);
    s.unit_kmax = reinterpret_cast<uint32_t*>(const_cast<uint8_t*>(ws) + w.kmax);
    s.status = d->status;
    s.L = d->L;
    s.Hkv = d->Hkv;
    s.num_blocks = d->num_blocks;
    s.S = d->S;
    s.max_blocks = d->max_blocks;
    s.heads_per_tile = score_heads_per_tile(d->Hkv);
    s.agg_heads = 0;
    s.seq_len_in = d->seq_len;
    return s;
}

int max_score_items(const tri_kv_desc* d) {
    const int hg = score_heads_per_tile(d->Hkv);
    const int64_t n = (int64_t)d->S * d->L * (d->Hkv / hg) * ((d->max_blocks + kChunkBlocks - 1) / kChunkBlocks);
    return n > INT_MAX ? INT_MAX : (int)n;
}

EvictParams make_evict_params(const tri_kv_desc* d) {
    EvictParams e{};
    e.k_pool = static_cast<uint8_t*>(d->k_pool);
    e.v_pool = static_cast<uint8_t*>(d->v_pool);
    e.block_table = d->block_table;
    e.L = d->L;
    e.Hkv = d->Hkv;
    e.num_blocks = d->num_blocks;
    e.S = d->S;
    e.max_blocks = d->max_blocks;
    e.score_stride = (int64_t)d->max_blocks * kBlockRows;
    e.status = d->status;
    return e;
}

MoveParams make_move_params(const tri_kv_desc* d, const int32_t* idx, int budget) {
    MoveParams m{};
    m.idx = idx;
    m.budget = budget;
    m.k_pool = static_cast<uint8_t*>(d->k_pool);
    m.v_pool = static_cast<uint8_t*>(d->v_pool);
    m.block_table = d->block_table;
    m.L = d->L;
    m.Hkv = d->Hkv;
    m.num_blocks = d->num_blocks;
    m.S = d->S;
    m.max_blocks = d->max_blocks;
    m.status = d->status;
    return m;
}

void record(cudaEvent_t ev, cudaStream_t stream) {
    if (ev) cudaEventRecord(ev, stream);
}

// The plan CTA's part of a step's query launch: lengths, work-item and
// freed-list offsets, key ranges, scratch counters, the free-list reservation.
void set_step_plan(QueryParams& q, const tri_kv_desc* desc, uint8_t* ws, const WsLayout& w, int budget, int trigger,
                   int32_t* freed_count, const tri_free_list* free_list) {
    q.L = desc->L;
    q.Hkv = desc->Hkv;
    q.G = desc->G;
    q.S = desc->S;
    q.seq_len = desc->seq_len;
    q.max_blocks = desc->max_blocks;
    q.heads_per_tile = score_heads_per_tile(desc->Hkv);
    q.status = desc->status;
    q.do_plan = 1;
    q.budget = budget;
    q.trigger = trigger;
    q.len_ws = reinterpret_cast<int32_t*>(ws + w.len_ws);
    q.item_off = reinterpret_cast<int32_t*>(ws + w.item_off);
    q.freed_off = reinterpret_cast<int32_t*>(ws + w.freed_off);
    q.freed_count = freed_count;
    q.unit_kmin = reinterpret_cast<uint32_t*>(ws + w.kmin);
    q.unit_kmax = reinterpret_cast<uint32_t*>(ws + w.kmax);
    q.zero_words = reinterpret_cast<int32_t*>(ws + w.words);
    if (free_list) {
        q.fl_count = free_list->count;
        q.fl_capacity = free_list->capacity;
        q.fl_base = reinterpret_cast<int32_t*>(ws + w.words) + 2;
    }
    if (persistent_compaction(budget)) q.fq_words = reinterpret_cast<int32_t*>(ws + w.fq);
}

// The selection and compaction launches of a step, after its scores are in
// the workspace (evict: select + plan + at-risk rows; copy-out; move).
tri_status select_and_compact(const tri_kv_desc* desc, uint8_t* ws, const WsLayout& w, const tri_step_options& opt,
                              int trigger, const tri_free_list* free_list, int32_t* freed_ids, int32_t* idx_out,
                              int32_t* slot_pos, bool pdl, cudaStream_t stream, const int32_t* veto = nullptr) {
    const int budget = opt.budget;
    if (persistent_compaction(budget)) {
        SelectCompactParams c{};
        c.k_pool = static_cast<uint8_t*>(desc->k_pool);
        c.v_pool = static_cast<uint8_t*>(desc->v_pool);
        c.block_table = desc->block_table;
        c.len_ws = reinterpret_cast<const int32_t*>(ws + w.len_ws);
        c.scores = reinterpret_cast<const float*>(ws + w.scores);
        c.score_stride = (int64_t)desc->max_blocks * kBlockRows;
        c.unit_kmin = reinterpret_cast<const uint32_t*>(ws + w.kmin);
        c.unit_kmax = reinterpret_cast<const uint32_t*>(ws + w.kmax);
        c.status = desc->status;
        c.L = desc->L;
        c.Hkv = desc->Hkv;
        c.num_blocks = desc->num_blocks;
        c.S = desc->S;
        c.max_blocks = desc->max_blocks;
        c.budget = budget;
        c.window = opt.window;
        c.sinks = opt.sinks;
        c.trigger = trigger;
        c.idx_copy = idx_out;
        c.seq_len_out = desc->seq_len;
        c.freed_off = reinterpret_cast<const int32_t*>(ws + w.freed_off);
        c.freed_ids = freed_ids;
        if (free_list) {
            c.fl_ids = free_list->ids;
            c.fl_base = reinterpret_cast<const int32_t*>(ws + w.words) + 2;
        }
        c.slot_pos = slot_pos;
        c.pos_stride = (int64_t)desc->max_blocks * kBlockRows;
        c.abort_word = veto;
        c.qwords = reinterpret_cast<int32_t*>(ws + w.fq);
        return cuda_status(launch_select_compact(c, device_sm_count(), stream, pdl));
    }
    EvictParams e = make_evict_params(desc);
    e.scores = reinterpret_cast<const float*>(ws + w.scores);
    e.unit_kmin = reinterpret_cast<const uint32_t*>(ws + w.kmin);
    e.unit_kmax = reinterpret_cast<const uint32_t*>(ws + w.kmax);
    e.lens = reinterpret_cast<const int32_t*>(ws + w.len_ws);
    e.budget = budget;
    e.window = opt.window;
    e.sinks = opt.sinks;
    e.trigger = trigger;
    e.idx_out = reinterpret_cast<int32_t*>(ws + w.idx);
    e.idx_copy = idx_out;
    e.do_select = 1;
    e.do_compact = 1;
    e.seq_len_out = desc->seq_len;
    e.freed_off = reinterpret_cast<const int32_t*>(ws + w.freed_off);
    e.freed_ids = freed_ids;
    if (free_list) {
        e.fl_ids = free_list->ids;
        e.fl_base = reinterpret_cast<const int32_t*>(ws + w.words) + 2;
    }
    e.slot_pos = slot_pos;
    e.pos_stride = (int64_t)desc->max_blocks * kBlockRows;
    e.scratch_used = reinterpret_cast<int32_t*>(ws + w.words);
    e.unit_info = reinterpret_cast<int32_t*>(ws + w.info);
    e.scratch_owner = reinterpret_cast<int32_t*>(ws + w.owner);
    e.scratch_rows = w.scratch_rows;
    // the evict kernel keeps two 512-thread CTAs per SM resident
    e.many_units = (int64_t)desc->S * desc->L * desc->Hkv > (int64_t)4 * device_sm_count() ? 1 : 0;
    e.abort_word = veto;
    tri_status st;
    if ((st = cuda_status(launch_evict(e, stream, pdl))) != TRI_OK) return st;
    MoveParams mv = make_move_params(desc, reinterpret_cast<const int32_t*>(ws + w.idx), budget);
    mv.lens = reinterpret_cast<const int32_t*>(ws + w.len_ws);
    mv.kept = nullptr;
    mv.trigger = trigger;
    mv.unit_info = reinterpret_cast<const int32_t*>(ws + w.info);
    mv.scratch = ws + w.scratch;
    mv.scratch_owner = reinterpret_cast<const int32_t*>(ws + w.owner);
    mv.scratch_used = reinterpret_cast<const int32_t*>(ws + w.words);
    mv.scratch_rows = w.scratch_rows;
    mv.abort_word = veto;
    mv.copy_out = 1;
    if ((st = cuda_status(launch_move(mv, device_sm_count(), stream, pdl))) != TRI_OK) return st;
    mv.copy_out = 0;
    return cuda_status(launch_move(mv, device_sm_count(), stream, pdl));
}

// Step outputs: freed ids + count (both or neither), a free list, idx.
tri_status check_step_outputs(const tri_free_list* free_list, const int32_t* freed_ids, const int32_t* freed_count,
                              const int32_t* idx_out) {
    tri_status st = check_free_list(free_list);
    if (st != TRI_OK) return st;
    if ((freed_ids == nullptr) != (freed_count == nullptr)) return TRI_ERR_INVALID;
    if (!freed_ids && !free_list) return TRI_ERR_INVALID;
    if ((freed_ids && !aligned(freed_ids, 4)) || (freed_count && !aligned(freed_count, 4))) return TRI_ERR_INVALID;
    if (idx_out && !aligned(idx_out, 4)) return TRI_ERR_INVALID;
    return TRI_OK;
}

DistScoreParams make_distance_params(const tri_kv_desc* desc, const float* table, int max_dist,
                                     const int32_t* slot_pos, float* scores) {
    DistScoreParams d{};
    d.table = table;
    d.max_dist = max_dist;
    d.slot_pos = slot_pos;
    d.pos_stride = (int64_t)desc->max_blocks * kBlockRows;
    d.cur_pos = desc->cur_pos;
    d.lens = desc->seq_len;
    d.seq_len_in = desc->seq_len;
    d.trigger = -1;
    d.scores = scores;
    d.score_stride = (int64_t)desc->max_blocks * kBlockRows;
    d.L = desc->L;
    d.Hkv = desc->Hkv;
    d.S = desc->S;
    d.status = desc->status;
    return d;
}

tri_status check_distance_args(const float* table, int max_dist, const int32_t* slot_pos) {
    if (!table || !slot_pos || !aligned(table, 4) || !aligned(slot_pos, 16)) return TRI_ERR_INVALID;
    if (max_dist < 1 || max_dist >= (1 << 24)) return TRI_ERR_INVALID;
    return TRI_OK;
}

}  // namespace

extern "C" {

tri_status tri_calibrate_centers(const float* q_pre, int N, int L, int Hq, int D, float* qbar, float* qabs,
                                 float* R, cudaStream_t stream) {
    if (!q_pre || N < 1 || L < 1 || Hq < 1) return TRI_ERR_INVALID;
    if (D != TRI_HEAD_DIM) return TRI_ERR_UNSUPPORTED;
    if (check_stats(qbar, qabs, R) != TRI_OK || !aligned(q_pre, 4)) return TRI_ERR_INVALID;
    if ((int64_t)L * Hq > INT_MAX) return TRI_ERR_INVALID;
    return cuda_status(launch_calibrate(q_pre, N, L, Hq, qbar, qabs, R, stream));
}

tri_status tri_build_query(const tri_kv_desc* desc, const float* qbar, const float* qabs, const float* R,
                           double rope_base, const int32_t* deltas, int n_deltas, float* qeff, float* w,
                           cudaStream_t stream) {
    tri_status st = check_desc(desc);
    if (st != TRI_OK) return st;
    if ((st = check_stats(qbar, qabs, R)) != TRI_OK) return st;
    if ((st = check_query_args(rope_base, deltas, n_deltas)) != TRI_OK) return st;
    if (!qeff || !w || !aligned(qeff, 16) || !aligned(w, 16)) return TRI_ERR_INVALID;
    if (desc->S == 0) return TRI_OK;
    QueryParams q = make_query_params(desc, qbar, qabs, R, rope_base, deltas, n_deltas, qeff, w);
    q.do_plan = 0;
    return cuda_status(launch_query(q, stream));
}

size_t tri_workspace_size(const tri_kv_desc* desc, int budget) {
    if (check_desc(desc) != TRI_OK || budget < 0 || budget > TRI_MAX_BUDGET) return 0;
    return ws_layout(desc, budget).total;
}

size_t tri_workspace_size_ex(const tri_kv_desc* desc, const tri_step_options* opt) {
    if (check_desc(desc) != TRI_OK || check_options(opt, desc->G) != TRI_OK) return 0;
    return ws_layout(desc, opt->budget, opt->aggregate == TRI_AGG_MAX).total;
}

tri_status tri_score(const tri_kv_desc* desc, const float* qbar, const float* qabs, const float* R,
                     double rope_base, const int32_t* deltas, int n_deltas, float* scores, void* workspace,
                     size_t ws_bytes, cudaStream_t stream) {
    return tri_score_ex(desc, qbar, qabs, R, rope_base, deltas, n_deltas, TRI_AGG_MEAN, scores, workspace,
                        ws_bytes, stream);
}

tri_status tri_score_ex(const tri_kv_desc* desc, const float* qbar, const float* qabs, const float* R,
                        double rope_base, const int32_t* deltas, int n_deltas, int aggregate, float* scores,
                        void* workspace, size_t ws_bytes, cudaStream_t stream) {
    tri_status st = check_desc(desc);
    if (st != TRI_OK) return st;
    if ((st = check_stats(qbar, qabs, R)) != TRI_OK) return st;
    if ((st = check_query_args(rope_base, deltas, n_deltas)) != TRI_OK) return st;
    if ((st = check_aggregate(aggregate, desc->G)) != TRI_OK) return st;
    if (!scores || !aligned(scores, 4)) return TRI_ERR_INVALID;
    const bool per_head = aggregate == TRI_AGG_MAX;
    if ((st = check_workspace(desc, workspace, ws_bytes, 0, per_head)) != TRI_OK) return st;
    if (desc->S == 0) return TRI_OK;
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    const WsLayout w = ws_layout(desc, 0, per_head);
    QueryParams q = make_query_params(desc, qbar, qabs, R, rope_base, deltas, n_deltas,
                                      reinterpret_cast<float*>(ws + w.qeff), reinterpret_cast<float*>(ws + w.wts));
    q.per_head = per_head ? 1 : 0;
    q.do_plan = 1;
    q.budget = 0;
    q.len_ws = reinterpret_cast<int32_t*>(ws + w.len_ws);
    q.item_off = reinterpret_cast<int32_t*>(ws + w.item_off);
    q.freed_off = reinterpret_cast<int32_t*>(ws + w.freed_off);
    q.freed_count = nullptr;
    q.unit_kmin = reinterpret_cast<uint32_t*>(ws + w.kmin);
    q.unit_kmax = reinterpret_cast<uint32_t*>(ws + w.kmax);
    if ((st = cuda_status(launch_query(q, stream))) != TRI_OK) return st;
    ScoreParams sp = make_score_params(desc, ws, w, scores, (int64_t)desc->max_blocks * kBlockRows);
    sp.agg_heads = per_head ? desc->G : 0;
    return cuda_status(launch_score(sp, max_score_items(desc), device_sm_count(), stream));
}

tri_status tri_select_topk(const tri_kv_desc* desc, const float* scores, int budget, int window, int32_t* idx,
                           int32_t* kept, cudaStream_t stream) {
    const tri_step_options o = {budget, window, 0, 0, TRI_AGG_MEAN, 0};
    return tri_select_topk_ex(desc, scores, &o, idx, kept, stream);
}

tri_status tri_select_topk_ex(const tri_kv_desc* desc, const float* scores, const tri_step_options* opt,
                              int32_t* idx, int32_t* kept, cudaStream_t stream) {
    tri_status st = check_desc(desc);
    if (st != TRI_OK) return st;
    if ((st = check_options(opt, 0)) != TRI_OK) return st;
    if (!scores || !idx || !kept || !aligned(scores, 16) || !aligned(idx, 4) || !aligned(kept, 4))
        return TRI_ERR_INVALID;
    if (desc->S == 0) return TRI_OK;
    EvictParams e = make_evict_params(desc);
    e.scores = scores;
    e.lens = desc->seq_len;
    e.budget = opt->budget;
    e.window = opt->window;
    e.sinks = opt->sinks;
    e.trigger = effective_trigger(*opt);
    e.idx_out = idx;
    e.kept_out = kept;
    e.do_select = 1;
    e.do_compact = 0;
    return cuda_status(launch_evict(e, stream));
}

tri_status tri_compact_kv(tri_kv_desc* desc, const int32_t* idx, const int32_t* kept, int budget,
                          int32_t* freed_ids, int32_t* freed_count, cudaStream_t stream) {
    tri_status st = check_desc(desc);
    if (st != TRI_OK) return st;
    if (budget < 1) return TRI_ERR_INVALID;
    if (budget > TRI_MAX_BUDGET) return TRI_ERR_UNSUPPORTED;
    if (!idx || !kept || !freed_ids || !freed_count || !aligned(idx, 4) || !aligned(kept, 4) ||
        !aligned(freed_ids, 4) || !aligned(freed_count, 4))
        return TRI_ERR_INVALID;
    if (desc->S == 0) return cuda_status(cudaMemsetAsync(freed_count, 0, sizeof(int32_t), stream));
    EvictParams e = make_evict_params(desc);
    e.lens = desc->seq_len;
    e.budget = budget;
    e.trigger = budget;
    e.idx_in = idx;
    e.kept_in = kept;
    e.do_select = 0;
    e.do_compact = 1;
    if ((st = cuda_status(launch_evict(e, stream))) != TRI_OK) return st;
    MoveParams mv = make_move_params(desc, idx, budget);
    mv.lens = desc->seq_len;
    mv.kept = kept;
    mv.trigger = budget;
    if ((st = cuda_status(launch_move(mv, device_sm_count(), stream))) != TRI_OK) return st;
    FinalizeParams f{};
    f.seq_len = desc->seq_len;
    f.kept = kept;
    f.block_table = desc->block_table;
    f.S = desc->S;
    f.max_blocks = desc->max_blocks;
    f.freed_ids = freed_ids;
    f.freed_count = freed_count;
    f.status = desc->status;
    return cuda_status(launch_finalize(f, stream));
}

tri_status tri_compress_step(tri_kv_desc* desc, const float* qbar, const float* qabs, const float* R,
                             double rope_base, const int32_t* deltas, int n_deltas, int budget, int window,
                             int32_t* freed_ids, int32_t* freed_count, int32_t* idx_out, void* workspace,
                             size_t ws_bytes, const tri_phase_events* events, cudaStream_t stream) {
    if (!freed_ids || !freed_count) return TRI_ERR_INVALID;
    const tri_step_options o = {budget, window, 0, 0, TRI_AGG_MEAN, 0};
    return tri_compress_step_ex(desc, qbar, qabs, R, rope_base, deltas, n_deltas, &o, nullptr, freed_ids,
                                freed_count, idx_out, workspace, ws_bytes, events, stream);
}

tri_status tri_compress_step_ex(tri_kv_desc* desc, const float* qbar, const float* qabs, const float* R,
                                double rope_base, const int32_t* deltas, int n_deltas, const tri_step_options* opt,
                                const tri_free_list* free_list, int32_t* freed_ids, int32_t* freed_count,
                                int32_t* idx_out, void* workspace, size_t ws_bytes, const tri_phase_events* events,
                                cudaStream_t stream) {
    tri_status st = check_desc(desc);
    if (st != TRI_OK) return st;
    if ((st = check_stats(qbar, qabs, R)) != TRI_OK) return st;
    if ((st = check_query_args(rope_base, deltas, n_deltas)) != TRI_OK) return st;
    if ((st = check_options(opt, desc->G)) != TRI_OK) return st;
    if ((st = check_step_outputs(free_list, freed_ids, freed_count, idx_out)) != TRI_OK) return st;
    const int budget = opt->budget;
    const bool per_head = opt->aggregate == TRI_AGG_MAX;
    if ((st = check_workspace(desc, workspace, ws_bytes, budget, per_head)) != TRI_OK) return st;
    if (events) record(events->start, stream);
    if (desc->S == 0) {
        st = freed_count ? cuda_status(cudaMemsetAsync(freed_count, 0, sizeof(int32_t), stream)) : TRI_OK;
        if (events) {
            record(events->after_query, stream);
            record(events->after_score, stream);
            record(events->after_evict, stream);
        }
        return st;
    }
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    const WsLayout w = ws_layout(desc, budget, per_head);
    const int trigger = effective_trigger(*opt);
    // The statistics check runs first and can veto the step (the word is
    // read by the plan, the selection and the move kernels).
    int32_t* veto = opt->check_stats ? reinterpret_cast<int32_t*>(ws + w.words) + 3 : nullptr;
    if (veto) {
        if ((st = cuda_status(cudaMemsetAsync(veto, 0, sizeof(int32_t), stream))) != TRI_OK) return st;
        StatsCheckParams c{};
        c.qbar = qbar;
        c.qabs = qabs;
        c.R = R;
        c.n_heads = (int64_t)desc->L * desc->Hkv * desc->G;
        c.status = desc->status;
        c.abort_word = veto;
        if ((st = cuda_status(launch_check_stats(c, stream))) != TRI_OK) return st;
    }
    QueryParams q = make_query_params(desc, qbar, qabs, R, rope_base, deltas, n_deltas,
                                      reinterpret_cast<float*>(ws + w.qeff), reinterpret_cast<float*>(ws + w.wts));
    q.per_head = per_head ? 1 : 0;
    set_step_plan(q, desc, ws, w, budget, trigger, freed_count, free_list);
    q.abort_word = veto;
    if ((st = cuda_status(launch_query(q, stream))) != TRI_OK) return st;
    if (events) record(events->after_query, stream);

    // Later kernels overlap their launch with the previous one's tail unless
    // phase events sit between them.
    const bool pdl = events == nullptr;
    float* scores = reinterpret_cast<float*>(ws + w.scores);
    ScoreParams sp = make_score_params(desc, ws, w, scores, (int64_t)desc->max_blocks * kBlockRows);
    sp.agg_heads = per_head ? desc->G : 0;
    sp.budget = budget;
    sp.trigger = trigger;
    sp.abort_word = veto;
    if ((st = cuda_status(launch_score(sp, max_score_items(desc), device_sm_count(), stream, pdl))) != TRI_OK)
        return st;
    if (events) record(events->after_score, stream);

    if ((st = select_and_compact(desc, ws, w, *opt, trigger, free_list, freed_ids, idx_out, nullptr, pdl, stream,
                                 veto)) != TRI_OK)
        return st;
    if (events) record(events->after_evict, stream);
    return TRI_OK;
}

int tri_step_is_fused(const tri_kv_desc* desc, const tri_step_options* opt) {
    if (check_desc(desc) != TRI_OK || check_options(opt, desc->G) != TRI_OK) return -1;
    return persistent_compaction(opt->budget) ? 1 : 0;
}

tri_status tri_check_stats(const float* qbar, const float* qabs, const float* R, int L, int Hq, int D,
                           int32_t* head_flags, int32_t* status, cudaStream_t stream) {
    if (L < 1 || Hq < 1 || (int64_t)L * Hq > INT_MAX) return TRI_ERR_INVALID;
    if (D != TRI_HEAD_DIM) return TRI_ERR_UNSUPPORTED;
    if (check_stats(qbar, qabs, R) != TRI_OK || !status || !aligned(status, 4) ||
        (head_flags && !aligned(head_flags, 4)))
        return TRI_ERR_INVALID;
    StatsCheckParams c{};
    c.qbar = qbar;
    c.qabs = qabs;
    c.R = R;
    c.n_heads = (int64_t)L * Hq;
    c.head_flags = head_flags;
    c.status = status;
    return cuda_status(launch_check_stats(c, stream));
}

tri_status tri_distance_table(int L, int Hkv, int G, int D, const float* qbar, const float* kbar, double rope_base,
                              const int32_t* deltas, int n_deltas, int aggregate, int max_dist, float* table,
                              cudaStream_t stream) {
    if (L < 1 || Hkv < 1 || G < 1 || (int64_t)L * Hkv > INT_MAX || (int64_t)Hkv * G > INT_MAX) return TRI_ERR_INVALID;
    if (D != TRI_HEAD_DIM) return TRI_ERR_UNSUPPORTED;
    if (!qbar || !kbar || !table || !aligned(qbar, 4) || !aligned(kbar, 4) || !aligned(table, 4))
        return TRI_ERR_INVALID;
    tri_status st = check_query_args(rope_base, deltas, n_deltas);
    if (st != TRI_OK) return st;
    if (aggregate != TRI_AGG_MEAN && aggregate != TRI_AGG_MAX) return TRI_ERR_INVALID;
    if (aggregate == TRI_AGG_MAX && G > 64) return TRI_ERR_UNSUPPORTED;
    if (max_dist < 1 || max_dist >= (1 << 24)) return TRI_ERR_INVALID;
    DistTableParams t{};
    t.qbar = qbar;
    t.kbar = kbar;
    t.base = rope_base;
    t.n_deltas = n_deltas;
    for (int i = 0; i < n_deltas; ++i) t.deltas[i] = deltas[i];
    t.L = L;
    t.Hkv = Hkv;
    t.G = G;
    t.per_head = aggregate == TRI_AGG_MAX ? 1 : 0;
    t.max_dist = max_dist;
    t.table = table;
    return cuda_status(launch_distance_table(t, stream));
}

tri_status tri_score_distance(const tri_kv_desc* desc, const float* table, int max_dist, const int32_t* slot_pos,
                              float* scores, cudaStream_t stream) {
    tri_status st = check_desc(desc);
    if (st != TRI_OK) return st;
    if ((st = check_distance_args(table, max_dist, slot_pos)) != TRI_OK) return st;
    if (!scores || !aligned(scores, 16)) return TRI_ERR_INVALID;
    if (desc->S == 0) return TRI_OK;
    return cuda_status(launch_distance_score(make_distance_params(desc, table, max_dist, slot_pos, scores), stream));
}

tri_status tri_compress_step_distance(tri_kv_desc* desc, const float* table, int max_dist, int32_t* slot_pos,
                                      const tri_step_options* opt, const tri_free_list* free_list, int32_t* freed_ids,
                                      int32_t* freed_count, int32_t* idx_out, void* workspace, size_t ws_bytes,
                                      const tri_phase_events* events, cudaStream_t stream) {
    tri_status st = check_desc(desc);
    if (st != TRI_OK) return st;
    if ((st = check_distance_args(table, max_dist, slot_pos)) != TRI_OK) return st;
    if ((st = check_options(opt, 0)) != TRI_OK) return st;
    if ((st = check_step_outputs(free_list, freed_ids, freed_count, idx_out)) != TRI_OK) return st;
    const int budget = opt->budget;
    if ((st = check_workspace(desc, workspace, ws_bytes, budget)) != TRI_OK) return st;
    if (events) record(events->start, stream);
    if (desc->S == 0) {
        st = freed_count ? cuda_status(cudaMemsetAsync(freed_count, 0, sizeof(int32_t), stream)) : TRI_OK;
        if (events) {
            record(events->after_query, stream);
            record(events->after_score, stream);
            record(events->after_evict, stream);
        }
        return st;
    }
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    const WsLayout w = ws_layout(desc, budget);
    const int trigger = effective_trigger(*opt);
    QueryParams q{};
    q.plan_only = 1;       // the distance table replaces the effective queries
    set_step_plan(q, desc, ws, w, budget, trigger, freed_count, free_list);
    if ((st = cuda_status(launch_query(q, stream))) != TRI_OK) return st;
    if (events) record(events->after_query, stream);
    const bool pdl = events == nullptr;
    DistScoreParams d = make_distance_params(desc, table, max_dist, slot_pos, reinterpret_cast<float*>(ws + w.scores));
    d.lens = reinterpret_cast<const int32_t*>(ws + w.len_ws);
    d.trigger = trigger;
    d.unit_kmin = reinterpret_cast<uint32_t*>(ws + w.kmin);
    d.unit_kmax = reinterpret_cast<uint32_t*>(ws + w.kmax);
    if ((st = cuda_status(launch_distance_score(d, stream, pdl))) != TRI_OK) return st;
    if (events) record(events->after_score, stream);
    if ((st = select_and_compact(desc, ws, w, *opt, trigger, free_list, freed_ids, idx_out, slot_pos, pdl, stream)) !=
        TRI_OK)
        return st;
    if (events) record(events->after_evict, stream);
    return TRI_OK;
}

tri_status tri_reserve_blocks(const tri_kv_desc* desc, int32_t* block_table, const int32_t* n_new,
                              const tri_free_list* free_list, cudaStream_t stream) {
    tri_status st = check_desc(desc);
    if (st != TRI_OK) return st;
    if (!block_table || block_table != desc->block_table || !n_new || !aligned(n_new, 4) || !free_list)
        return TRI_ERR_INVALID;
    if ((st = check_free_list(free_list)) != TRI_OK) return st;
    if ((int64_t)desc->S * desc->max_blocks > INT_MAX) return TRI_ERR_INVALID;
    if (desc->S == 0) return TRI_OK;
    ReserveParams r{};
    r.seq_len = desc->seq_len;
    r.n_new = n_new;
    r.block_table = block_table;
    r.S = desc->S;
    r.max_blocks = desc->max_blocks;
    r.num_blocks = desc->num_blocks;
    r.fl_ids = free_list->ids;
    r.fl_count = free_list->count;
    r.fl_capacity = free_list->capacity;
    r.status = desc->status;
    return cuda_status(launch_reserve(r, stream));
}

tri_status tri_sync_status(int32_t* status, cudaStream_t stream) {
    if (!status || !aligned(status, 4)) return TRI_ERR_INVALID;
    int32_t h = 0;
    if (cudaStreamSynchronize(stream) != cudaSuccess) return TRI_ERR_CUDA;
    if (cudaMemcpyAsync(&h, status, sizeof(h), cudaMemcpyDeviceToHost, stream) != cudaSuccess) return TRI_ERR_CUDA;
    if (cudaStreamSynchronize(stream) != cudaSuccess) return TRI_ERR_CUDA;
    if (h != 0) {
        if (cudaMemsetAsync(status, 0, sizeof(int32_t), stream) != cudaSuccess) return TRI_ERR_CUDA;
        if (cudaStreamSynchronize(stream) != cudaSuccess) return TRI_ERR_CUDA;
    }
    if (h & TRI_DEVFLAG_BOUNDS) return TRI_ERR_DEVICE_BOUNDS;
    if (h & TRI_DEVFLAG_TIMEOUT) return TRI_ERR_TIMEOUT;
    if (h & TRI_DEVFLAG_FREELIST) return TRI_ERR_FREELIST;
    if (h & TRI_DEVFLAG_STATS) return TRI_ERR_STATS;
    if (h & TRI_DEVFLAG_NONFINITE) return TRI_ERR_NONFINITE;
    return TRI_OK;
}

const char* tri_status_string(tri_status s) {
    switch (s) {
        case TRI_OK: return "ok";
        case TRI_ERR_INVALID: return "invalid argument";
        case TRI_ERR_UNSUPPORTED: return "unsupported shape or size";
        case TRI_ERR_CUDA: return "CUDA runtime error";
        case TRI_ERR_DEVICE_BOUNDS: return "device saw an out-of-range index, length or block id";
        case TRI_ERR_TIMEOUT: return "bounded device wait timed out";
        case TRI_ERR_NONFINITE: return "NaN score";
        case TRI_ERR_WORKSPACE: return "workspace missing, too small or misaligned";
        case TRI_ERR_FREELIST: return "device free list had too few entries or too little room";
        case TRI_ERR_STATS: return "head statistics failed the sanity check";
        default: return "unknown status";
    }
}

}  // extern "C"
