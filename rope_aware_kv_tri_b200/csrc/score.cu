// score.cu - one streaming pass over every cached key.
//
// Pages: "TriAttention: Trigonometric KV Compression for Efficient Long
// Reasoning" - "Key Concepts", Trigonometric Distance Preference and Norm as
// Importance Signal; "TriAttention: Efficient Long Reasoning with
// Trigonometric KV Compression" - "English" (centres score keys through a
// trigonometric series, with Q/K norms as an additional signal);
// "TriAttention: How a Geometric Trick Cuts LLM Memory Use by 10x Without
// Losing Accuracy" - "The Core Idea" (norm signal weighted by measured
// concentration).
//
// Score of a cached post-rotary key K (bf16, D = 128), from the folded
// effective query of its unit (query.cu):
//     s = sum_d qeff_d K_d + sum_i w_i sqrt(K_i^2 + K_{i+64}^2)
//
// Design (HBM-bound: 256 bytes and ~1.5 flop per byte):
//  * Persistent CTAs, two per SM.  A work item is (sequence, layer, group of
//    HG KV heads, run of 16 paged blocks); items are dealt round-robin.
//  * Warp 8 is the producer: one lane issues one bulk copy (TMA engine, no
//    multicast) per paged block, moving the HG contiguous 4 KiB (block, head)
//    tiles of that block into a ring of shared-memory stages, with an
//    evict-first L2 policy (scores are stored evict-last, so the selection
//    finds them in L2).  Full/empty mbarriers hand stages over.
//  * Warps 0..7 consume: HG heads per stage, each warp owns one head (or a
//    quarter of one), so its 24 coefficients stay in registers for the whole
//    item.  8 lanes share a key: lane `sub` reads 16 bytes of the real half
//    (dims 8sub..8sub+7) and the matching 16 bytes of the imaginary half
//    (dims 64+8sub..), i.e. 8 whole bands; fp32 FMA on packed pairs of
//    adjacent bands (fma.rn.f32x2); 3 xor-shuffles reduce.
//  * Each warp also tracks the smallest and largest order key of the scores
//    it writes for a unit and folds them into the unit's key range with one
//    atomicMin/atomicMax per item; the selection buckets scores linearly over
//    that range.
//  * Every wait is bounded; on a timeout the CTA records TRI_DEVFLAG_TIMEOUT,
//    lets its in-flight copies land and returns.
//
// Max over the GQA group (agg_heads = G): the G heads of a unit are scored
// separately, s = max_g (qeff_g . K + sum_i w_{g,i} |K band i|).  A key is
// shared by 64/BPL lanes with BPL bands each (BPL = 8, 8, 4, 2 for G = 1, 2,
// 4, 8), so the 3*BPL*G coefficients of a lane stay within 48 registers; the
// band magnitudes are computed once per key and reused by every head.  The
// G partial sums are reduced with a butterfly that halves the live heads at
// each step (a reduce-scatter over the key's lanes), then the lanes holding
// different heads' totals exchange their maximum.
#include "score_device.cuh"
#include "tri_device.cuh"
#include "tri_internal.h"

namespace tri {

namespace {

constexpr int kConsumerWarps = 8;
constexpr int kScoreThreads = (kConsumerWarps + 1) * 32;
constexpr int kStageBudgetBytes = 96 * 1024;
constexpr int kMaxStages = 16;

struct StageMeta {
    int unit0;   // unit of the stage's first head
    int t0;      // slot of the stage's first row
    int nrows;   // valid rows (< 16 only in a sequence's last block)
    int kind;    // 0: nothing to score, 1: keys, 2: end of work
};

__device__ __forceinline__ bool wait_or_abort(uint64_t* bar, uint32_t parity, volatile int* abort_flag) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = global_timer_ns();
    for (uint32_t it = 1; it < kWaitLimitIters; ++it) {
        if (mbar_try_wait(bar, parity)) return true;
        if ((it & 31u) == 0) {
            if (*abort_flag) return false;
            if (global_timer_ns() - t0 > kWaitLimitNs) return false;
        }
    }
    return false;
}

// ---- max over the group -------------------------------------------------

template <int G> struct MaxLayout;
template <> struct MaxLayout<1> { static constexpr int kBpl = 8; };
template <> struct MaxLayout<2> { static constexpr int kBpl = 8; };
template <> struct MaxLayout<4> { static constexpr int kBpl = 4; };
template <> struct MaxLayout<8> { static constexpr int kBpl = 2; };

// BPL bf16 values of the real half (dims sub*BPL..) and of the imaginary
// half (dims 64 + sub*BPL..) of a 256-byte key row, as pairs of adjacent
// bands (element j of a pair array holds bands 2j and 2j+1 of the lane).
template <int BPL>
__device__ __forceinline__ void load_bands(const uint8_t* row, int sub, float2 (&re)[BPL / 2],
                                           float2 (&im)[BPL / 2]) {
    constexpr int W = BPL / 2;                 // 32-bit words per half
    uint32_t a[W], b[W];
    if constexpr (W == 4) {
        const uint4 x = *reinterpret_cast<const uint4*>(row + sub * 16);
        const uint4 y = *reinterpret_cast<const uint4*>(row + 128 + sub * 16);
        a[0] = x.x; a[1] = x.y; a[2] = x.z; a[3] = x.w;
        b[0] = y.x; b[1] = y.y; b[2] = y.z; b[3] = y.w;
    } else if constexpr (W == 2) {
        const uint2 x = *reinterpret_cast<const uint2*>(row + sub * 8);
        const uint2 y = *reinterpret_cast<const uint2*>(row + 128 + sub * 8);
        a[0] = x.x; a[1] = x.y;
        b[0] = y.x; b[1] = y.y;
    } else {
        a[0] = *reinterpret_cast<const uint32_t*>(row + sub * 4);
        b[0] = *reinterpret_cast<const uint32_t*>(row + 128 + sub * 4);
    }
#pragma unroll
    for (int j = 0; j < W; ++j) {
        re[j] = make_float2(bf16_lo(a[j]), bf16_hi(a[j]));
        im[j] = make_float2(bf16_lo(b[j]), bf16_hi(b[j]));
    }
}

// Butterfly over lane bit M and below: N live partial sums per lane; at each
// step a lane keeps half of them (by its bit M) and adds its partner's copy of
// that half.  Ends with v[0] = a full sum of one head.
template <int N, int M, int G>
__device__ __forceinline__ void scatter_heads(float (&v)[G], int lane) {
    if constexpr (M >= 1) {
        if constexpr (N > 1) {
            constexpr int H = N / 2;
            const bool upper = (lane & M) != 0;
#pragma unroll
            for (int j = 0; j < H; ++j) {
                const float send = upper ? v[j] : v[j + H];
                const float keep = upper ? v[j + H] : v[j];
                v[j] = keep + __shfl_xor_sync(0xffffffffu, send, M);
            }
            scatter_heads<H, M / 2, G>(v, lane);
        } else {
            v[0] += __shfl_xor_sync(0xffffffffu, v[0], M);
            scatter_heads<1, M / 2, G>(v, lane);
        }
    }
}

// Largest of the G head scores of the key shared by lanes of width LPK.
template <int G, int LPK>
__device__ __forceinline__ float group_max(float (&v)[G], int lane) {
    scatter_heads<G, LPK / 2, G>(v, lane);
    float r = v[0];
#pragma unroll
    for (int m = LPK / 2; m >= LPK / G; m >>= 1) r = fmaxf(r, __shfl_xor_sync(0xffffffffu, r, m));
    return r;
}

__device__ void produce(const ScoreParams& p, uint8_t* tiles, uint64_t* full, uint64_t* empty, StageMeta* meta,
                        volatile int* abort_flag) {
    const int HG = p.heads_per_tile;
    const uint32_t stages = (uint32_t)p.stages;
    const uint32_t stage_bytes = (uint32_t)HG * kTileBytes;
    const int n_hg = p.Hkv / HG;
    const uint64_t pol = l2_policy_evict_first();
    // The work items, by the plan's rule, from inputs the plan does not
    // write (the caller's lengths, the trigger, the statistics veto): the
    // producer needs nothing from the plan, so it streams keys while the
    // plan and the effective queries are still being built.  A length out
    // of range counts as empty (the plan flags it).
    const int64_t max_len = (int64_t)p.max_blocks * kBlockRows;
    const bool vetoed = p.abort_word != nullptr && *reinterpret_cast<const volatile int32_t*>(p.abort_word) != 0;
    auto seq_items = [&](int s, int& len) -> int {
        int n = __ldg(p.seq_len_in + s);
        if (n < 0 || (int64_t)n > max_len) n = 0;
        len = n;
        const bool scored = !vetoed && (p.budget <= 0 || n > p.trigger);
        const int nblk = (n + kBlockRows - 1) / kBlockRows;
        return scored ? p.L * n_hg * ((nblk + kChunkBlocks - 1) / kChunkBlocks) : 0;
    };
    int cs = 0, base = 0, len = 0;               // sequence cs holds items [base, base + cnt)
    int cnt = p.S > 0 ? seq_items(0, len) : 0;
    uint32_t k = 0;
    bool ok = true;
    for (int item = blockIdx.x; ok; item += gridDim.x) {
        while (cs < p.S && item >= base + cnt) {
            base += cnt;
            ++cs;
            cnt = cs < p.S ? seq_items(cs, len) : 0;
        }
        if (cs >= p.S) break;
        const int s = cs;
        const int nblk = (len + kBlockRows - 1) / kBlockRows;
        const int nch = (nblk + kChunkBlocks - 1) / kChunkBlocks;
        const int r = item - base;
        const int chunk = r % nch, lhg = r / nch;
        const int hg = lhg % n_hg, l = lhg / n_hg;
        const int unit0 = (s * p.L + l) * p.Hkv + hg * HG;
        const int b0 = chunk * kChunkBlocks;
        const int b1 = min(b0 + kChunkBlocks, nblk);
        for (int b = b0; b < b1; ++b) {
            const uint32_t slot = k % stages;
            if (k >= stages && !wait_or_abort(&empty[slot], ((k / stages) - 1) & 1u, abort_flag)) {
                ok = false;
                break;
            }
            if (*abort_flag) {
                ok = false;
                break;
            }
            const int blk = p.block_table[(int64_t)s * p.max_blocks + b];
            StageMeta m;
            m.unit0 = unit0;
            m.t0 = b * kBlockRows;
            m.nrows = min(kBlockRows, len - b * kBlockRows);
            if (blk >= 0 && blk < p.num_blocks) {
                m.kind = 1;
                meta[slot] = m;
                mbar_arrive_expect_tx(&full[slot], stage_bytes);
                const uint8_t* src =
                    p.k_pool + ((((int64_t)l * p.num_blocks + blk) * p.Hkv + (int64_t)hg * HG) * kTileBytes);
                bulk_copy_g2s(tiles + (size_t)slot * stage_bytes, src, stage_bytes, &full[slot], pol);
            } else {
                raise_flag(p.status, TRI_DEVFLAG_BOUNDS);
                m.kind = 0;
                meta[slot] = m;
                mbar_arrive(&full[slot]);
            }
            ++k;
        }
    }
    if (ok) {
        const uint32_t slot = k % stages;
        if (k >= stages && !wait_or_abort(&empty[slot], ((k / stages) - 1) & 1u, abort_flag)) {
            ok = false;
        } else {
            StageMeta m;
            m.unit0 = 0;
            m.t0 = 0;
            m.nrows = 0;
            m.kind = 2;
            meta[slot] = m;
            mbar_arrive(&full[slot]);
        }
    }
    if (!ok) {
        if (!*abort_flag) raise_flag(p.status, TRI_DEVFLAG_TIMEOUT);
        *abort_flag = 1;
        // No copy may still be landing in this CTA's shared memory when it exits.
        const uint32_t first = k > stages ? k - stages : 0u;
        for (uint32_t j = first; j < k; ++j) mbar_wait_bounded(&full[j % stages], (j / stages) & 1u);
    }
}

__device__ void consume(const ScoreParams& p, int warp, int lane, const uint8_t* tiles, uint64_t* full,
                        uint64_t* empty, const StageMeta* meta, volatile int* abort_flag) {
    const int HG = p.heads_per_tile;
    const uint32_t stages = (uint32_t)p.stages;
    const uint32_t stage_bytes = (uint32_t)HG * kTileBytes;
    const int wph = kConsumerWarps / HG;       // warps per head
    const int hig = warp / wph;                // head of the tile group
    const int q0 = warp % wph;                 // first quad of keys
    const int sub = lane & 7, kq = lane >> 3;
    float2 qr[4], qi[4], ww[4];
    int cur_unit = -1;
    const uint64_t keep_pol = l2_policy_evict_last();   // scores are re-read by the selection
    // order-key range of the scores this warp wrote for cur_unit
    uint32_t kmin = 0xffffffffu, kmax = 0u;
    auto flush_range = [&]() {
        const uint32_t lo = __reduce_min_sync(0xffffffffu, kmin);
        const uint32_t hi = __reduce_max_sync(0xffffffffu, kmax);
        if (lane == 0 && cur_unit >= 0 && lo <= hi) {
            atomicMin(&p.unit_kmin[cur_unit], lo);
            atomicMax(&p.unit_kmax[cur_unit], hi);
        }
        kmin = 0xffffffffu;
        kmax = 0u;
    };
    for (uint32_t k = 0;; ++k) {
        const uint32_t slot = k % stages;
        if (!wait_or_abort(&full[slot], (k / stages) & 1u, abort_flag)) {
            if (!*abort_flag) raise_flag(p.status, TRI_DEVFLAG_TIMEOUT);
            *abort_flag = 1;
            return;
        }
        const StageMeta m = meta[slot];
        if (m.kind == 2) {
            flush_range();
            return;
        }
        if (m.kind == 1) {
            const int unit = m.unit0 + hig;
            if (unit != cur_unit) {
                flush_range();
                load_key_coefficients(p.qeff, p.wts, unit, sub, qr, qi, ww);
                cur_unit = unit;
            }
            const uint8_t* tile = tiles + (size_t)slot * stage_bytes + (size_t)hig * kTileBytes;
            float* out = p.scores + (int64_t)unit * p.score_stride + m.t0;
            for (int q = q0; q < 4; q += wph) {
                const int row = q * 4 + kq;
                const uint4 a = *reinterpret_cast<const uint4*>(tile + row * 256 + sub * 16);
                const uint4 b = *reinterpret_cast<const uint4*>(tile + row * 256 + 128 + sub * 16);
                float acc = key_score(a, b, qr, qi, ww);
                acc += __shfl_xor_sync(0xffffffffu, acc, 1);
                acc += __shfl_xor_sync(0xffffffffu, acc, 2);
                acc += __shfl_xor_sync(0xffffffffu, acc, 4);
                if (sub == 0 && row < m.nrows) {
                    store_with_policy(out + row, acc, keep_pol);
                    const uint32_t key = order_key(acc);
                    kmin = min(kmin, key);
                    kmax = max(kmax, key);
                }
            }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[slot]);
    }
}

template <int G>
__device__ void consume_max(const ScoreParams& p, int warp, int lane, const uint8_t* tiles, uint64_t* full,
                            uint64_t* empty, const StageMeta* meta, volatile int* abort_flag) {
    constexpr int BPL = MaxLayout<G>::kBpl;
    constexpr int LPK = kBands / BPL;          // lanes per key
    constexpr int KPI = 32 / LPK;              // keys per warp step
    const int HG = p.heads_per_tile;
    const uint32_t stages = (uint32_t)p.stages;
    const uint32_t stage_bytes = (uint32_t)HG * kTileBytes;
    const int wph = kConsumerWarps / HG;
    const int hig = warp / wph;
    const int q0 = warp % wph;
    constexpr int NP = BPL / 2;                // band pairs per lane
    const int sub = lane % LPK, kq = lane / LPK;
    float2 qr[G][NP], qi[G][NP], ww[G][NP];
    int cur_unit = -1;
    const uint64_t keep_pol = l2_policy_evict_last();
    uint32_t kmin = 0xffffffffu, kmax = 0u;
    auto flush_range = [&]() {
        const uint32_t lo = __reduce_min_sync(0xffffffffu, kmin);
        const uint32_t hi = __reduce_max_sync(0xffffffffu, kmax);
        if (lane == 0 && cur_unit >= 0 && lo <= hi) {
            atomicMin(&p.unit_kmin[cur_unit], lo);
            atomicMax(&p.unit_kmax[cur_unit], hi);
        }
        kmin = 0xffffffffu;
        kmax = 0u;
    };
    for (uint32_t k = 0;; ++k) {
        const uint32_t slot = k % stages;
        if (!wait_or_abort(&full[slot], (k / stages) & 1u, abort_flag)) {
            if (!*abort_flag) raise_flag(p.status, TRI_DEVFLAG_TIMEOUT);
            *abort_flag = 1;
            return;
        }
        const StageMeta m = meta[slot];
        if (m.kind == 2) {
            flush_range();
            return;
        }
        if (m.kind == 1) {
            const int unit = m.unit0 + hig;
            if (unit != cur_unit) {
                flush_range();
#pragma unroll
                for (int g = 0; g < G; ++g) {
                    const float2* qe = reinterpret_cast<const float2*>(p.qeff + ((int64_t)unit * G + g) * kHeadDim);
                    const float2* we = reinterpret_cast<const float2*>(p.wts + ((int64_t)unit * G + g) * kBands);
#pragma unroll
                    for (int j = 0; j < NP; ++j) {
                        qr[g][j] = __ldg(qe + sub * NP + j);
                        qi[g][j] = __ldg(qe + kBands / 2 + sub * NP + j);
                        ww[g][j] = __ldg(we + sub * NP + j);
                    }
                }
                cur_unit = unit;
            }
            const uint8_t* tile = tiles + (size_t)slot * stage_bytes + (size_t)hig * kTileBytes;
            float* out = p.scores + (int64_t)unit * p.score_stride + m.t0;
            for (int q = q0; q < kBlockRows / KPI; q += wph) {
                const int row = q * KPI + kq;
                float2 re[NP], im[NP], nrm[NP];
                load_bands<BPL>(tile + row * 256, sub, re, im);
#pragma unroll
                for (int j = 0; j < NP; ++j) {
                    const float2 sq = ffma2(re[j], re[j], fmul2(im[j], im[j]));
                    nrm[j] = make_float2(sqrt_fast(sq.x), sqrt_fast(sq.y));
                }
                float v[G];
#pragma unroll
                for (int g = 0; g < G; ++g) {
                    float2 d0 = make_float2(0.f, 0.f), d1 = make_float2(0.f, 0.f);
#pragma unroll
                    for (int j = 0; j < NP; ++j) {
                        d0 = ffma2(qr[g][j], re[j], d0);
                        d1 = ffma2(qi[g][j], im[j], d1);
                        d0 = ffma2(ww[g][j], nrm[j], d0);
                    }
                    v[g] = (d0.x + d0.y) + (d1.x + d1.y);
                }
                const float acc = group_max<G, LPK>(v, lane);
                if (sub == 0 && row < m.nrows) {
                    store_with_policy(out + row, acc, keep_pol);
                    const uint32_t key = order_key(acc);
                    kmin = min(kmin, key);
                    kmax = max(kmax, key);
                }
            }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[slot]);
    }
}

// AGG = 0: folded group mean; AGG = G: max over the G heads of the group.
template <int AGG>
__global__ void __launch_bounds__(kScoreThreads, 2) score_kernel(const ScoreParams p) {
    extern __shared__ __align__(1024) uint8_t smem[];
    const uint32_t stages = (uint32_t)p.stages;
    const uint32_t stage_bytes = (uint32_t)p.heads_per_tile * kTileBytes;
    uint8_t* tiles = smem;
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + (size_t)stages * stage_bytes);
    uint64_t* empty = full + stages;
    StageMeta* meta = reinterpret_cast<StageMeta*>(empty + stages);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(meta + stages);
    if (threadIdx.x == 0) {
        for (uint32_t i = 0; i < stages; ++i) {
            mbar_init(&full[i], 1);
            mbar_init(&empty[i], kConsumerWarps);
        }
        *abort_flag = 0;
        fence_mbar_init();
    }
    __syncthreads();
    allow_next_grid();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (warp == kConsumerWarps) {
        // plans its own work items: starts streaming before query_kernel ends
        if (lane == 0) produce(p, tiles, full, empty, meta, abort_flag);
        return;
    }
    wait_prior_grid();          // the folded queries come from query_kernel
    if constexpr (AGG == 0)
        consume(p, warp, lane, tiles, full, empty, meta, abort_flag);
    else
        consume_max<AGG>(p, warp, lane, tiles, full, empty, meta, abort_flag);
}

size_t score_smem_bytes(int HG, int stages) {
    return (size_t)stages * HG * kTileBytes + (size_t)stages * 2 * sizeof(uint64_t) +
           (size_t)stages * sizeof(StageMeta) + 16;
}

}  // namespace

int score_heads_per_tile(int Hkv) {
    for (int hg = 8; hg > 1; hg >>= 1)
        if (Hkv % hg == 0) return hg;
    return 1;
}

cudaError_t launch_score(const ScoreParams& p_in, int max_items, int num_sms, cudaStream_t stream, bool pdl) {
    if (p_in.agg_heads > 1 && !p_in.cuda_cores_only && score_mma_supported(p_in))
        return launch_score_mma(p_in, max_items, num_sms, stream, pdl);
    ScoreParams p = p_in;
    int stages = kStageBudgetBytes / (p.heads_per_tile * kTileBytes);
    if (stages > kMaxStages) stages = kMaxStages;
    if (stages < 2) stages = 2;
    p.stages = stages;
    const size_t smem = score_smem_bytes(p.heads_per_tile, stages);
    void (*kernel)(const ScoreParams);
    switch (p.agg_heads) {
        case 0: kernel = score_kernel<0>; break;
        case 1: kernel = score_kernel<1>; break;
        case 2: kernel = score_kernel<2>; break;
        case 4: kernel = score_kernel<4>; break;
        case 8: kernel = score_kernel<8>; break;
        default: return cudaErrorInvalidValue;
    }
    cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    int grid = num_sms * 2;
    if (max_items < grid) grid = max_items;
    if (grid < 1) grid = 1;
    return launch_kernel(kernel, dim3(grid), dim3(kScoreThreads), smem, stream, pdl, p);
}

}  // namespace tri
