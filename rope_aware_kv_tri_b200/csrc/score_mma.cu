// score_mma.cu - max-over-group key scores with the G-column contraction on
// the tensor cores (tcgen05, accumulators in tensor memory).
//
// Pages: "TriAttention: Trigonometric KV Compression for Efficient Long
// Reasoning" - "Key Concepts", Trigonometric Distance Preference and Norm as
// Importance Signal; "TriAttention: How a Geometric Trick Cuts LLM Memory Use
// by 10x Without Losing Accuracy" - "The Core Idea".
//
// Score of a cached post-rotary key K under the max aggregation:
//     s = max_g [ qeff_g . K + sum_i w_{g,i} sqrt(K_i^2 + K_{i+64}^2) ]
// For the 8 KV heads of one (layer, block) the dot products of all their
// keys with all their heads' effective queries are one small matrix product
//     D[128 keys][8 heads x G x 2] = K[128][128] . C[128][8 x G x 2]
// where C holds every qeff_g split into bf16 hi + lo parts (so the product
// of bf16 keys with the fp32 query keeps ~16 significant bits).
//
// Design (one persistent CTA per SM, 14 warps):
//  * warp 12, producer: two TMA tensor loads per (layer, block) - dims 0..63
//    and 64..127 of its 128 rows (8 heads x 16 keys), 128-byte swizzle,
//    L2 evict-first, no multicast - into a ring of 32 KiB stages.
//  * warp 13, MMA issuer: at each new (layer, head group) writes C (and the norm
//    weights W) for its 8 units into shared memory (double-buffered by item),
//    then issues 8 tcgen05.mma (M=128, N=16G, K=16 each) per stage into one of
//    three tensor-memory accumulators, and commits their completion to the
//    epilogue's and the stage's mbarriers.
//  * warps 0..11, epilogue: three groups of four warps take the stages in
//    turn (stage j -> group j mod 3, accumulator j mod 3); warp q (mod 4)
//    owns tensor-memory lanes 32q..32q+31 = keys of heads 2q, 2q+1.
//    Each thread owns ONE key: it reads its 4G accumulator columns
//    (tcgen05.ld), reads its key row from the swizzled stage for the band
//    magnitudes (computed once, used by every head), adds the weighted norm
//    per head and keeps the maximum.  No cross-lane reduction per key.
//  * Every wait is bounded; on a timeout the CTA records TRI_DEVFLAG_TIMEOUT,
//    every role leaves its loop, in-flight copies and products are drained
//    and the tensor memory is freed before the CTA exits.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_bf16.h>

#include <mutex>

#include "tri_device.cuh"
#include "tri_internal.h"

namespace tri {

namespace {

constexpr int kGroups = 3;                             // epilogue groups = accumulators in flight
constexpr int kEpiWarps = 4 * kGroups;
constexpr int kProducerWarp = kEpiWarps;
constexpr int kMmaWarp = kEpiWarps + 1;
constexpr int kMmaThreads = (kEpiWarps + 2) * 32;
constexpr int kStageRows = 128;                        // 8 heads x 16 keys
constexpr uint32_t kHalfBytes = kStageRows * 128;      // 128 rows x 64 dims bf16
constexpr uint32_t kStageBytes = 2 * kHalfBytes;       // 32 KiB
constexpr uint32_t kSmemLimit = 227 * 1024;

struct MmaMeta {
    int unit0;   // unit of the stage's first head
    int t0;      // slot of the stage's first row
    int nrows;   // valid rows per head
    int kind;    // 0: nothing to score, 1: keys, 2: end of work
    int ord;     // ordinal of the work item within this CTA
};

template <int G>
struct MmaShape {
    static constexpr int N = 8 * 2 * G;                       // accumulator columns
    static constexpr uint32_t kCBytes = N * 256;              // C: two halves of N rows x 128 B
    static constexpr int kWHead = G * 64 + 4;                 // floats per unit: padded by 16 bytes so that
                                                              // the two units a warp reads sit in other banks
    static constexpr uint32_t kWBytes = 8 * kWHead * 4;       // norm weights of 8 units
    static constexpr uint32_t kAccCols = kGroups * N;         // one accumulator per epilogue group
    static constexpr uint32_t kTmemCols = kAccCols <= 32 ? 32 : kAccCols <= 64 ? 64 : kAccCols <= 128 ? 128
                                        : kAccCols <= 256 ? 256 : 512;
    static constexpr uint32_t kFixed = 2 * kCBytes + 2 * kWBytes + 1024 /*barriers, meta*/ + 1024 /*align*/;
    static constexpr int kStages = (int)((kSmemLimit - kFixed) / kStageBytes) > 5
                                       ? 5 : (int)((kSmemLimit - kFixed) / kStageBytes);
    static constexpr uint32_t kSmemBytes = kStages * kStageBytes + kFixed;
    static_assert(kStages >= 2, "not enough shared memory for two stages");
    static_assert(kAccCols <= 512, "TMEM columns");
};

// ------------------------------------------------ TMA tensor and tcgen05

__device__ __forceinline__ void tma_load_2d(void* smem_dst, const CUtensorMap* map, int x, int y, uint64_t* bar,
                                            uint64_t l2_policy) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
        " [%0], [%1, {%3, %4}], [%2], %5;" ::"r"(smem_u32(smem_dst)),
        "l"(map), "r"(smem_u32(bar)), "r"(x), "r"(y), "l"(l2_policy)
        : "memory");
}

__device__ __forceinline__ void tmem_alloc(uint32_t* smem_dst, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(smem_dst)),
                 "r"(ncols)
                 : "memory");
}

__device__ __forceinline__ void tmem_relinquish() {
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}

__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// D[tmem] (+)= A[smem] . B[smem]^T, bf16 inputs, fp32 accumulation.
__device__ __forceinline__ void mma_bf16(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                         uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// Arrive on `bar` once every tcgen05 operation this thread issued so far has completed.
__device__ __forceinline__ void mma_commit(uint64_t* bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
                 : "memory");
}

__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

// 32 lanes x R consecutive 32-bit columns: thread t gets lane (base lane + t).
__device__ __forceinline__ void tmem_ld8(uint32_t taddr, uint32_t (&r)[8]) {
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7])
                 : "r"(taddr)
                 : "memory");
}

__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&r)[16]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
        "%15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr)
        : "memory");
}

template <int R>
__device__ __forceinline__ void tmem_ld(uint32_t taddr, uint32_t (&r)[R]) {
    if constexpr (R == 8) {
        tmem_ld8(taddr, r);
    } else {
        static_assert(R % 16 == 0, "column count");
#pragma unroll
        for (int c = 0; c < R / 16; ++c) {
            uint32_t part[16];
            tmem_ld16(taddr + 16 * c, part);
#pragma unroll
            for (int i = 0; i < 16; ++i) r[16 * c + i] = part[i];
        }
    }
}

// Shared-memory matrix descriptor of a K-major operand in the 128-byte
// swizzled layout (rows of 128 B, 8-row atoms of 1024 B, atom-aligned base).
__device__ __forceinline__ uint64_t sw128_desc(uint32_t smem_addr) {
    uint64_t d = 0;
    d |= (uint64_t)((smem_addr & 0x3FFFFu) >> 4);      // start address
    d |= (uint64_t)1 << 16;                              // leading byte offset (unused when swizzled)
    d |= (uint64_t)(1024 >> 4) << 32;                    // stride byte offset: next 8-row atom
    d |= (uint64_t)1 << 46;                              // descriptor version
    d |= (uint64_t)2 << 61;                              // 128-byte swizzle
    return d;
}

// Instruction descriptor: bf16 A and B (both K-major), fp32 D, M = 128, N.
template <int N>
__device__ __forceinline__ constexpr uint32_t idesc_bf16_m128() {
    return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(128 >> 4) << 24);
}

// Byte offset of 16-byte chunk `c` of row `row` in a 128-byte swizzled half.
__device__ __forceinline__ uint32_t sw128_offset(int row, int c) {
    return (uint32_t)row * 128u + ((uint32_t)(c ^ (row & 7)) << 4);
}

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

// The same wait for a whole warp: lane 0 polls, the outcome is shared, and
// __syncwarp orders the other lanes' later reads after lane 0's acquire.
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, volatile int* abort_flag, int lane) {
    bool ok = true;
    if (lane == 0) ok = wait_or_abort(bar, parity, abort_flag);
    ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
    __syncwarp();
    return ok;
}

__device__ __forceinline__ void give_up(const ScoreParams& p, volatile int* abort_flag) {
    if (!*abort_flag) raise_flag(p.status, TRI_DEVFLAG_TIMEOUT);
    *abort_flag = 1;
}

struct Smem {
    uint8_t* stages;
    uint8_t* cbuf;
    float* wbuf;
    uint64_t* full;
    uint64_t* empty;
    uint64_t* tfull;
    uint64_t* tempty;
    uint64_t* wready;
    uint64_t* drain;
    MmaMeta* meta;
    volatile int* ctl;      // [0] abort, [1] stage index of the end marker
    uint32_t* tmem_slot;
};

template <int G>
__device__ Smem carve(uint8_t* base) {
    using Sh = MmaShape<G>;
    Smem s;
    s.stages = base;
    s.cbuf = base + Sh::kStages * kStageBytes;
    s.wbuf = reinterpret_cast<float*>(s.cbuf + 2 * Sh::kCBytes);
    s.full = reinterpret_cast<uint64_t*>(reinterpret_cast<uint8_t*>(s.wbuf) + 2 * Sh::kWBytes);
    s.empty = s.full + Sh::kStages;
    s.tfull = s.empty + Sh::kStages;
    s.tempty = s.tfull + kGroups;
    s.wready = s.tempty + kGroups;
    s.drain = s.wready + 2;
    s.meta = reinterpret_cast<MmaMeta*>(s.drain + 1);
    s.ctl = reinterpret_cast<volatile int*>(s.meta + Sh::kStages);
    s.tmem_slot = reinterpret_cast<uint32_t*>(const_cast<int*>(s.ctl + 2));
    return s;
}

// ------------------------------------------------------------- producer

template <int G>
__device__ void mma_produce(const MmaScoreParams& P, const Smem& sm) {
    using Sh = MmaShape<G>;
    const ScoreParams& p = P.base;
    constexpr uint32_t S_N = Sh::kStages;
    volatile int* abort_flag = sm.ctl;
    const int n_hg = p.Hkv / 8;
    const int total = p.item_off[p.S];
    const uint64_t pol = l2_policy_evict_first();
    uint32_t k = 0;
    int ord = -1, prev_group = -1;
    bool ok = true;
    // A contiguous range of work items per CTA, so that its coefficients
    // change only where the (sequence, layer, head group) changes.
    const int per = total / (int)gridDim.x, extra = total % (int)gridDim.x;
    const int first = (int)blockIdx.x * per + min((int)blockIdx.x, extra);
    const int last = first + per + ((int)blockIdx.x < extra ? 1 : 0);
    for (int item = first; ok && item < last; ++item) {
        int lo = 0, hi = p.S;
        while (hi - lo > 1) {
            const int mid = (lo + hi) >> 1;
            if (p.item_off[mid] <= item) lo = mid; else hi = mid;
        }
        const int s = lo;
        const int len = p.len_ws[s];
        const int nblk = (len + kBlockRows - 1) / kBlockRows;
        const int nch = (nblk + kChunkBlocks - 1) / kChunkBlocks;
        const int r = item - p.item_off[s];
        const int chunk = r % nch, lhg = r / nch;
        const int hg = lhg % n_hg, l = lhg / n_hg;
        const int unit0 = (s * p.L + l) * p.Hkv + hg * 8;
        const int b0 = chunk * kChunkBlocks;
        const int b1 = min(b0 + kChunkBlocks, nblk);
        if (unit0 != prev_group) {
            ++ord;
            prev_group = unit0;
        }
        for (int b = b0; b < b1; ++b) {
            const uint32_t slot = k % S_N;
            if (k >= S_N && !wait_or_abort(&sm.empty[slot], ((k / S_N) - 1) & 1u, abort_flag)) {
                ok = false;
                break;
            }
            if (*abort_flag) {
                ok = false;
                break;
            }
            const int blk = p.block_table[(int64_t)s * p.max_blocks + b];
            MmaMeta m;
            m.unit0 = unit0;
            m.t0 = b * kBlockRows;
            m.nrows = min(kBlockRows, len - b * kBlockRows);
            m.ord = ord;
            if (blk >= 0 && blk < p.num_blocks) {
                m.kind = 1;
                sm.meta[slot] = m;
                mbar_arrive_expect_tx(&sm.full[slot], kStageBytes);
                const int row0 = (int)((((int64_t)l * p.num_blocks + blk) * p.Hkv + hg * 8) * kBlockRows);
                uint8_t* dst = sm.stages + (size_t)slot * kStageBytes;
                tma_load_2d(dst, &P.tmap, 0, row0, &sm.full[slot], pol);
                tma_load_2d(dst + kHalfBytes, &P.tmap, 64, row0, &sm.full[slot], pol);
            } else {
                raise_flag(p.status, TRI_DEVFLAG_BOUNDS);
                m.kind = 0;
                sm.meta[slot] = m;
                mbar_arrive(&sm.full[slot]);
            }
            ++k;
        }
    }
    if (ok) {
        const uint32_t slot = k % S_N;
        if (k >= S_N && !wait_or_abort(&sm.empty[slot], ((k / S_N) - 1) & 1u, abort_flag)) {
            ok = false;
        } else {
            MmaMeta m;
            m.unit0 = 0;
            m.t0 = 0;
            m.nrows = 0;
            m.kind = 2;
            m.ord = ord + 1;
            sm.meta[slot] = m;
            mbar_arrive(&sm.full[slot]);
        }
    }
    if (!ok) {
        give_up(p, abort_flag);
        // No copy may still be landing in shared memory when the CTA exits.
        const uint32_t first = k > S_N ? k - S_N : 0u;
        for (uint32_t j = first; j < k; ++j) mbar_wait_bounded(&sm.full[j % S_N], (j / S_N) & 1u);
    }
}

// ------------------------------------------------------------ MMA issuer

// C (bf16 hi/lo of the 8 units' G effective queries, 128-byte swizzled, K-major)
// and W (their norm weights) for the units unit0 .. unit0+7.
template <int G>
__device__ void write_coefficients(const ScoreParams& p, int unit0, uint8_t* C, float* W, int lane) {
    constexpr int N = MmaShape<G>::N;
    constexpr int kTasks = 8 * G * 16 / 32;       // (head, query head, 8-dim chunk) tasks per lane
    constexpr int kBatch = 4;                     // tasks whose loads are in flight together
    static_assert(kTasks % kBatch == 0, "task batching");
    for (int t0 = 0; t0 < kTasks; t0 += kBatch) {
      float4 xa[kBatch], xb[kBatch];
#pragma unroll
      for (int i = 0; i < kBatch; ++i) {
        const int t = lane + 32 * (t0 + i);
        const int hh = t / (G * 16), g = (t / 16) % G, c = t % 16;
        const float4* src = reinterpret_cast<const float4*>(p.qeff + ((int64_t)(unit0 + hh) * G + g) * kHeadDim + c * 8);
        xa[i] = __ldg(src);
        xb[i] = __ldg(src + 1);
      }
#pragma unroll
      for (int i = 0; i < kBatch; ++i) {
        const int t = lane + 32 * (t0 + i);
        const int hh = t / (G * 16), g = (t / 16) % G, c = t % 16;
        const float x[8] = {xa[i].x, xa[i].y, xa[i].z, xa[i].w, xb[i].x, xb[i].y, xb[i].z, xb[i].w};
        uint32_t hi[4], lo[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const __nv_bfloat16 h0 = __float2bfloat16_rn(x[2 * j]), h1 = __float2bfloat16_rn(x[2 * j + 1]);
            const __nv_bfloat16 l0 = __float2bfloat16_rn(x[2 * j] - __bfloat162float(h0));
            const __nv_bfloat16 l1 = __float2bfloat16_rn(x[2 * j + 1] - __bfloat162float(h1));
            hi[j] = (uint32_t)__bfloat16_as_ushort(h0) | ((uint32_t)__bfloat16_as_ushort(h1) << 16);
            lo[j] = (uint32_t)__bfloat16_as_ushort(l0) | ((uint32_t)__bfloat16_as_ushort(l1) << 16);
        }
        const int n_hi = hh * 2 * G + 2 * g;
        const int half = c / 8, cin = c % 8;
        uint8_t* base = C + (size_t)half * (N * 128);
        *reinterpret_cast<uint4*>(base + sw128_offset(n_hi, cin)) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
        *reinterpret_cast<uint4*>(base + sw128_offset(n_hi + 1, cin)) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
      }
    }
    const float4* wsrc = reinterpret_cast<const float4*>(p.wts + (int64_t)unit0 * G * kBands);
    float4* wdst = reinterpret_cast<float4*>(W);
    constexpr int kW = 8 * G * kBands / 4 / 32;   // float4 per lane
    constexpr int kWBatch = kW < 8 ? kW : 8;
    for (int i0 = 0; i0 < kW; i0 += kWBatch) {
        float4 wv[kWBatch];
#pragma unroll
        for (int i = 0; i < kWBatch; ++i) wv[i] = __ldg(wsrc + lane + 32 * (i0 + i));
#pragma unroll
        for (int i = 0; i < kWBatch; ++i) {
            const int f = lane + 32 * (i0 + i);                 // float4 of unit f / (G * 16)
            wdst[f + f / (G * 16)] = wv[i];
        }
    }
}

template <int G>
__device__ void mma_issue(const ScoreParams& p, const Smem& sm, uint32_t tmem_base, int lane) {
    using Sh = MmaShape<G>;
    constexpr int N = Sh::N;
    constexpr uint32_t S_N = Sh::kStages;
    constexpr uint32_t idesc = idesc_bf16_m128<N>();
    volatile int* abort_flag = sm.ctl;
    int cur_ord = -1;
    for (uint32_t k = 0;; ++k) {
        const uint32_t slot = k % S_N, b = k % kGroups;
        if (!warp_wait(&sm.full[slot], (k / S_N) & 1u, abort_flag, lane)) {
            give_up(p, abort_flag);
            return;
        }
        const MmaMeta m = sm.meta[slot];
        // accumulator b is free once its group's epilogue of stage k - kGroups has read it
        if (k >= kGroups && !warp_wait(&sm.tempty[b], ((k / kGroups) - 1) & 1u, abort_flag, lane)) {
            give_up(p, abort_flag);
            return;
        }
        if (m.kind == 2) {
            // every product issued so far has been read: end every epilogue group
            for (uint32_t d = 1; d < kGroups && d <= k; ++d) {
                if (!warp_wait(&sm.tempty[(k - d) % kGroups], ((k - d) / kGroups) & 1u, abort_flag, lane)) {
                    give_up(p, abort_flag);
                    return;
                }
            }
            __syncwarp();
            if (lane == 0) {
                sm.ctl[1] = (int)k;
                for (int g = 0; g < kGroups; ++g) mbar_arrive(&sm.tfull[g]);
            }
            return;
        }
        tc_fence_after();
        if (m.ord != cur_ord) {
            // The buffers of set m.ord were last used by set m.ord - 2, whose
            // stages may be as recent as k - 2: wait until every stage before
            // k has been read by its epilogue (so its products are done too).
            for (uint32_t d = 1; cur_ord >= 0 && d < kGroups && d <= k; ++d) {
                if (!warp_wait(&sm.tempty[(k - d) % kGroups], ((k - d) / kGroups) & 1u, abort_flag, lane)) {
                    give_up(p, abort_flag);
                    return;
                }
            }
            tc_fence_after();
            write_coefficients<G>(p, m.unit0, sm.cbuf + (size_t)(m.ord & 1) * Sh::kCBytes,
                                  sm.wbuf + (size_t)(m.ord & 1) * (Sh::kWBytes / 4), lane);
            fence_proxy_async_smem();      // the products read C through the async proxy
            __syncwarp();
            if (lane == 0) mbar_arrive(&sm.wready[m.ord & 1]);
            cur_ord = m.ord;
        }
        __syncwarp();
        if (lane == 0) {
            if (m.kind == 1) {
                const uint32_t a0 = smem_u32(sm.stages + (size_t)slot * kStageBytes);
                const uint32_t c0 = smem_u32(sm.cbuf + (size_t)(m.ord & 1) * Sh::kCBytes);
                const uint32_t d = tmem_base + b * N;
#pragma unroll
                for (int kk = 0; kk < kHeadDim / 16; ++kk) {
                    const uint32_t koff = (uint32_t)(kk & 3) * 32u;
                    const uint64_t adesc = sw128_desc(a0 + (uint32_t)(kk >> 2) * kHalfBytes + koff);
                    const uint64_t bdesc = sw128_desc(c0 + (uint32_t)(kk >> 2) * (N * 128) + koff);
                    mma_bf16(d, adesc, bdesc, idesc, kk > 0 ? 1u : 0u);
                }
                mma_commit(&sm.tfull[b]);
                mma_commit(&sm.empty[slot]);
            } else {
                mbar_arrive(&sm.tfull[b]);
                mbar_arrive(&sm.empty[slot]);
            }
        }
        __syncwarp();
    }
}

// -------------------------------------------------------------- epilogue

template <int G>
__device__ void mma_epilogue(const ScoreParams& p, const Smem& sm, uint32_t tmem_base, int warp, int lane) {
    using Sh = MmaShape<G>;
    constexpr int N = Sh::N;
    constexpr uint32_t S_N = Sh::kStages;
    volatile int* abort_flag = sm.ctl;
    const uint32_t group = (uint32_t)warp >> 2;      // stages j with j mod kGroups == group
    const int quad = warp & 3;                        // tensor-memory lanes 32q .. 32q+31
    const int hh = 2 * quad + (lane >> 4);            // head of this thread's key within the 8
    const int r = lane & 15;                          // key row within the block
    const int row = 32 * quad + lane;                 // row of the stage = accumulator lane
    const uint64_t keep_pol = l2_policy_evict_last();
    int cur_ord = -1, cur_unit = -1;
    uint32_t kmin = 0xffffffffu, kmax = 0u;
    auto flush_range = [&]() {
#pragma unroll
        for (int o = 8; o >= 1; o >>= 1) {
            kmin = min(kmin, __shfl_xor_sync(0xffffffffu, kmin, o));
            kmax = max(kmax, __shfl_xor_sync(0xffffffffu, kmax, o));
        }
        if (r == 0 && cur_unit >= 0 && kmin <= kmax) {
            atomicMin(&p.unit_kmin[cur_unit], kmin);
            atomicMax(&p.unit_kmax[cur_unit], kmax);
        }
        kmin = 0xffffffffu;
        kmax = 0u;
    };
    for (uint32_t j = group;; j += kGroups) {
        const uint32_t slot = j % S_N;
        if (!warp_wait(&sm.tfull[group], (j / kGroups) & 1u, abort_flag, lane)) {
            give_up(p, abort_flag);
            break;
        }
        tc_fence_after();
        if ((int)j >= sm.ctl[1]) break;               // end of work
        const MmaMeta m = sm.meta[slot];
        if (m.kind == 1) {
            if (m.ord != cur_ord) {
                flush_range();
                if (!warp_wait(&sm.wready[m.ord & 1], ((uint32_t)m.ord >> 1) & 1u, abort_flag, lane)) {
                    give_up(p, abort_flag);
                    break;
                }
                cur_ord = m.ord;
                cur_unit = m.unit0 + hh;
            }
            // dot products of this key with its head's G queries (hi + lo columns)
            uint32_t dacc[4 * G];
            tmem_ld<4 * G>(tmem_base + ((uint32_t)(32 * quad) << 16) + group * N + (uint32_t)quad * 4 * G, dacc);
            tmem_wait_ld();
            const bool upper = (lane >> 4) != 0;     // lanes 16..31 hold the second head's key
            float acc[G];
#pragma unroll
            for (int g = 0; g < G; ++g) {
                const float a = __uint_as_float(dacc[2 * g]) + __uint_as_float(dacc[2 * g + 1]);
                const float b = __uint_as_float(dacc[2 * G + 2 * g]) + __uint_as_float(dacc[2 * G + 2 * g + 1]);
                acc[g] = upper ? b : a;
            }
            // band magnitudes of the key, weighted per head
            const uint8_t* st = sm.stages + (size_t)slot * kStageBytes;
            const float* W = sm.wbuf + (size_t)(m.ord & 1) * (Sh::kWBytes / 4) + (size_t)hh * Sh::kWHead;
            float2 wn[G];
#pragma unroll
            for (int g = 0; g < G; ++g) wn[g] = make_float2(0.f, 0.f);
#pragma unroll 2
            for (int c = 0; c < 8; ++c) {
                const uint4 a = *reinterpret_cast<const uint4*>(st + sw128_offset(row, c));
                const uint4 q = *reinterpret_cast<const uint4*>(st + kHalfBytes + sw128_offset(row, c));
                const uint32_t av[4] = {a.x, a.y, a.z, a.w};
                const uint32_t qv[4] = {q.x, q.y, q.z, q.w};
                float2 nrm[4];
#pragma unroll
                for (int jj = 0; jj < 4; ++jj) {
                    const float2 re = make_float2(bf16_lo(av[jj]), bf16_hi(av[jj]));
                    const float2 im = make_float2(bf16_lo(qv[jj]), bf16_hi(qv[jj]));
                    const float2 sq = ffma2(re, re, fmul2(im, im));
                    nrm[jj] = make_float2(sqrt_fast(sq.x), sqrt_fast(sq.y));
                }
#pragma unroll
                for (int g = 0; g < G; ++g) {
                    const float4 w0 = *reinterpret_cast<const float4*>(W + g * kBands + 8 * c);
                    const float4 w1 = *reinterpret_cast<const float4*>(W + g * kBands + 8 * c + 4);
                    wn[g] = ffma2(make_float2(w0.x, w0.y), nrm[0], wn[g]);
                    wn[g] = ffma2(make_float2(w0.z, w0.w), nrm[1], wn[g]);
                    wn[g] = ffma2(make_float2(w1.x, w1.y), nrm[2], wn[g]);
                    wn[g] = ffma2(make_float2(w1.z, w1.w), nrm[3], wn[g]);
                }
            }
            float best = acc[0] + (wn[0].x + wn[0].y);
#pragma unroll
            for (int g = 1; g < G; ++g) best = fmaxf(best, acc[g] + (wn[g].x + wn[g].y));
            if (r < m.nrows) {
                store_with_policy(p.scores + (int64_t)cur_unit * p.score_stride + m.t0 + r, best, keep_pol);
                const uint32_t key = order_key(best);
                kmin = min(kmin, key);
                kmax = max(kmax, key);
            }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) {
            mbar_arrive(&sm.tempty[group]);
            mbar_arrive(&sm.empty[slot]);
        }
    }
    flush_range();
}

template <int G>
__global__ void __launch_bounds__(kMmaThreads, 1) score_mma_kernel(const __grid_constant__ MmaScoreParams P) {
    using Sh = MmaShape<G>;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t pad = (1024u - (smem_u32(smem_raw) & 1023u)) & 1023u;
    const Smem sm = carve<G>(smem_raw + pad);
    const ScoreParams& p = P.base;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        for (int i = 0; i < Sh::kStages; ++i) {
            mbar_init(&sm.full[i], 1);
            mbar_init(&sm.empty[i], 1 + 4);       // the products' commit + 4 epilogue warps
        }
        for (int b = 0; b < kGroups; ++b) {
            mbar_init(&sm.tfull[b], 1);
            mbar_init(&sm.tempty[b], 4);
        }
        for (int b = 0; b < 2; ++b) mbar_init(&sm.wready[b], 1);
        mbar_init(sm.drain, 1);
        sm.ctl[0] = 0;
        sm.ctl[1] = 0x7fffffff;
        fence_mbar_init();
    }
    if (warp == kMmaWarp) {
        tmem_alloc(sm.tmem_slot, Sh::kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *sm.tmem_slot;
    allow_next_grid();
    wait_prior_grid();          // effective queries and the plan come from query_kernel

    if (warp == kProducerWarp) {
        if (lane == 0) mma_produce<G>(P, sm);
    } else if (warp == kMmaWarp) {
        mma_issue<G>(p, sm, tmem_base, lane);
    } else {
        mma_epilogue<G>(p, sm, tmem_base, warp, lane);
    }

    tc_fence_before();
    __syncthreads();
    if (warp == kMmaWarp) {
        tc_fence_after();
        // every product must have completed before the accumulators are freed
        if (lane == 0) {
            mma_commit(sm.drain);
            mbar_wait_bounded(sm.drain, 0);
        }
        __syncwarp();
        tmem_dealloc(tmem_base, Sh::kTmemCols);
    }
}

// ------------------------------------------------------------------ host

PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
    static std::mutex mu;
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static bool tried = false;
    std::lock_guard<std::mutex> lock(mu);
    if (!tried) {
        tried = true;
        void* ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
    }
    return fn;
}

template <int G>
cudaError_t launch_g(const MmaScoreParams& P, int max_items, int num_sms, cudaStream_t stream, bool pdl) {
    using Sh = MmaShape<G>;
    const size_t smem = Sh::kSmemBytes;
    cudaError_t e = cudaFuncSetAttribute(score_mma_kernel<G>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    int grid = num_sms;
    if (max_items < grid) grid = max_items;
    if (grid < 1) grid = 1;
    return launch_kernel(score_mma_kernel<G>, dim3(grid), dim3(kMmaThreads), smem, stream, pdl, P);
}

}  // namespace

bool score_mma_supported(const ScoreParams& p) {
    const int G = p.agg_heads;
    if (!(G == 2 || G == 4 || G == 8) || p.Hkv % 8 != 0) return false;
    const int64_t rows = (int64_t)p.L * p.num_blocks * p.Hkv * kBlockRows;
    if (rows >= ((int64_t)1 << 31)) return false;
    if ((reinterpret_cast<uintptr_t>(p.k_pool) & 15u) != 0) return false;
    return tensor_map_encoder() != nullptr;
}

cudaError_t launch_score_mma(const ScoreParams& p, int max_items, int num_sms, cudaStream_t stream, bool pdl) {
    MmaScoreParams P{};
    P.base = p;
    P.base.heads_per_tile = 8;
    const cuuint64_t dims[2] = {(cuuint64_t)kHeadDim, (cuuint64_t)p.L * p.num_blocks * p.Hkv * kBlockRows};
    const cuuint64_t strides[1] = {(cuuint64_t)kHeadDim * 2};
    const cuuint32_t box[2] = {64, (cuuint32_t)kStageRows};
    const cuuint32_t estr[2] = {1, 1};
    PFN_cuTensorMapEncodeTiled_v12000 encode = tensor_map_encoder();
    if (!encode) return cudaErrorNotSupported;
    const CUresult r = encode(&P.tmap, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<uint8_t*>(p.k_pool), dims,
                              strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return cudaErrorInvalidValue;
    switch (p.agg_heads) {
        case 2: return launch_g<2>(P, max_items, num_sms, stream, pdl);
        case 4: return launch_g<4>(P, max_items, num_sms, stream, pdl);
        case 8: return launch_g<8>(P, max_items, num_sms, stream, pdl);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace tri
