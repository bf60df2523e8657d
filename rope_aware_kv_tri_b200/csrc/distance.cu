// distance.cu - the distance-only variant: scores from the query and key
// centres alone, as a table over the query-key distance.
//
// Pages: "TriAttention: Trigonometric KV Compression for Efficient Long
// Reasoning" - "Core Mechanism" (the trigonometric series of the distance,
// evaluated as lookups indexed by relative position) and "Key Concepts",
// Trigonometric Distance Preference (after rotation the centres' dot product
// depends on the distance only).
//
// For query head g of KV head h (layer l) and the key centre kbar_h:
//   c_{g,i}  = qbar_{g,i} conj(kbar_i) * mean_delta exp(j theta_i delta)
//   f_g(d)   = sum_i Re( c_{g,i} exp(j theta_i d) ),    d = p - pos
// and the table holds mean_g f_g (folded: c_i = mean_g c_{g,i}) or max_g f_g,
// for d = 0 .. max_dist, built once in float64 and stored in fp32.
//
// A step then scores slot t of unit (s, l, h) as table[l][h][p_s - pos_t]
// with no pass over the keys: 4 bytes of position and 4 of table per key.
#include "tri_device.cuh"
#include "tri_internal.h"

namespace tri {

namespace {

constexpr int kTableThreads = 256;
constexpr int kDistThreads = 256;
constexpr int kDistChunk = 4096;        // slots per score CTA
constexpr int kDistVecs = 4;            // 4-slot vectors per thread whose reads are in flight together

// Block (lh, chunk): coefficients of (l, h) in shared memory, then one table
// entry per thread.
__global__ void __launch_bounds__(kTableThreads) distance_table_kernel(const DistTableParams p) {
    extern __shared__ double coef[];    // [n_sets][kBands][2]
    __shared__ double s_theta[kBands];
    const int lh = blockIdx.x;
    const int l = lh / p.Hkv, h = lh % p.Hkv;
    const int Hq = p.Hkv * p.G;
    const int n_sets = p.per_head ? p.G : 1;
    for (int i = threadIdx.x; i < kBands; i += blockDim.x)
        s_theta[i] = pow(p.base, -2.0 * (double)i / (double)kHeadDim);
    __syncthreads();
    for (int k = threadIdx.x; k < n_sets * kBands; k += blockDim.x) {
        const int set = k / kBands, i = k % kBands;
        const double theta = s_theta[i];
        double mr = 0.0, mi = 0.0;
        for (int d = 0; d < p.n_deltas; ++d) {
            double sn, cs;
            sincos(theta * (double)p.deltas[d], &sn, &cs);
            mr += cs;
            mi += sn;
        }
        mr /= p.n_deltas;
        mi /= p.n_deltas;
        const double kr = p.kbar[((int64_t)l * p.Hkv + h) * kHeadDim + i];
        const double ki = p.kbar[((int64_t)l * p.Hkv + h) * kHeadDim + i + kBands];
        double ar = 0.0, ai = 0.0;
        const int g0 = p.per_head ? set : 0, g1 = p.per_head ? set + 1 : p.G;
        for (int g = g0; g < g1; ++g) {
            const int64_t row = (int64_t)l * Hq + (int64_t)h * p.G + g;
            const double qr = p.qbar[row * kHeadDim + i];
            const double qi = p.qbar[row * kHeadDim + i + kBands];
            // qbar conj(kbar)
            ar += qr * kr + qi * ki;
            ai += qi * kr - qr * ki;
        }
        if (!p.per_head) {
            ar /= p.G;
            ai /= p.G;
        }
        coef[2 * k] = ar * mr - ai * mi;
        coef[2 * k + 1] = ar * mi + ai * mr;
    }
    __syncthreads();
    const int64_t d = (int64_t)blockIdx.y * blockDim.x + threadIdx.x;
    if (d > p.max_dist) return;
    // one-time build: exp(j theta_i d) is recomputed per coefficient set
    double best = 0.0;
    for (int set = 0; set < n_sets; ++set) {
        double acc = 0.0;
        for (int i = 0; i < kBands; ++i) {
            double sn, cs;
            sincos(s_theta[i] * (double)d, &sn, &cs);
            acc += coef[2 * (set * kBands + i)] * cs - coef[2 * (set * kBands + i) + 1] * sn;
        }
        best = (set == 0 || acc > best) ? acc : best;
    }
    p.table[(int64_t)lh * (p.max_dist + 1) + d] = (float)best;
}

// Block (u, chunk): slots [chunk*kDistChunk, ...) of unit u.
__global__ void __launch_bounds__(kDistThreads) distance_score_kernel(const DistScoreParams p) {
    static_assert(kDistChunk == kDistThreads * kDistVecs * 4, "one batch of position loads per CTA");
    __shared__ uint32_t wlo[kDistThreads / 32], whi[kDistThreads / 32];
    allow_next_grid();
    const int u = blockIdx.x;
    const int LH = p.L * p.Hkv;
    const int s = u / LH, lh = u % LH;
    const int t0 = blockIdx.y * kDistChunk;
    // The query position and this chunk's slot positions are inputs the plan
    // does not write (the previous step's compaction wrote them before the
    // plan began), so they are requested before waiting for the plan, up to
    // the caller's length of the sequence (the plan validates it after).
    const int64_t P = p.cur_pos[s];
    const int32_t* pos = p.slot_pos + (int64_t)u * p.pos_stride;
    const int4* pos4 = reinterpret_cast<const int4*>(pos + t0);
    int n4_pre = 0;
    if (p.seq_len_in) {
        const int64_t n_in = min((int64_t)__ldg(p.seq_len_in + s), p.pos_stride) - t0;
        n4_pre = n_in > 0 ? (int)(min(n_in, (int64_t)kDistChunk) >> 2) : 0;
    }
    int4 q[kDistVecs];
#pragma unroll
    for (int k = 0; k < kDistVecs; ++k) {
        const int i = threadIdx.x + k * kDistThreads;
        q[k] = i < n4_pre ? __ldcs(pos4 + i) : make_int4(0, 0, 0, 0);
    }
    wait_prior_grid();
    const int len = p.lens[s];
    if (len < 0 || (int64_t)len > p.pos_stride) {
        if (threadIdx.x == 0 && blockIdx.y == 0) raise_flag(p.status, TRI_DEVFLAG_BOUNDS);
        return;
    }
    if (len <= p.trigger) return;            // a sequence the step leaves alone
    if (t0 >= len) return;
    const int t1 = min(t0 + kDistChunk, len);
    const float* tab = p.table + (int64_t)lh * (p.max_dist + 1);
    float* out = p.scores + (int64_t)u * p.score_stride;
    uint32_t lo = 0xffffffffu, hi = 0u;
    bool bad = false;
    auto score_one = [&](int32_t position) -> float {
        int64_t d = P - (int64_t)position;
        if (d < 0 || d > p.max_dist) {
            bad = true;
            d = d < 0 ? 0 : p.max_dist;
        }
        const float v = __ldg(tab + d);
        const uint32_t key = order_key(v);
        lo = min(lo, key);
        hi = max(hi, key);
        return v;
    };
    // 16-byte position loads and score stores (t0 and the unit rows are
    // multiples of 4 slots, so both are aligned).
    const int n4 = (t1 - t0) >> 2;
    float4* out4 = reinterpret_cast<float4*>(out + t0);
    if (P >= 0 && P <= 0x7fffffff) {
        // The usual case.  The lookup is two dependent reads per slot, so a
        // thread has all its position loads (kDistVecs x 4 slots) in flight,
        // then all their table reads, and the distance is formed in 32 bits:
        // P - pos as an unsigned number is in range exactly when 0 <= d <=
        // max_dist (a position after P wraps to a large value).
        const uint32_t Pu = (uint32_t)P, maxd = (uint32_t)p.max_dist;
        {
            const int i0 = threadIdx.x;
#pragma unroll
            for (int k = 0; k < kDistVecs; ++k) {
                const int i = i0 + k * kDistThreads;
                if (i >= n4) q[k] = make_int4((int)Pu, (int)Pu, (int)Pu, (int)Pu);
                else if (i >= n4_pre) q[k] = __ldcs(pos4 + i);    // past the caller's length: not prefetched
            }
            float v[kDistVecs][4];
#pragma unroll
            for (int k = 0; k < kDistVecs; ++k) {
                const int32_t qc[4] = {q[k].x, q[k].y, q[k].z, q[k].w};
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    const uint32_t d = Pu - (uint32_t)qc[c];
                    bad |= d > maxd;
                    v[k][c] = __ldg(tab + min(d, maxd));
                }
            }
#pragma unroll
            for (int k = 0; k < kDistVecs; ++k) {
                const int i = i0 + k * kDistThreads;
                if (i < n4) {
#pragma unroll
                    for (int c = 0; c < 4; ++c) {
                        const uint32_t key = order_key(v[k][c]);
                        lo = min(lo, key);
                        hi = max(hi, key);
                    }
                    out4[i] = make_float4(v[k][0], v[k][1], v[k][2], v[k][3]);
                }
            }
        }
    } else {
        for (int i = threadIdx.x; i < n4; i += kDistThreads) {
            const int4 q = pos4[i];
            float4 v;
            v.x = score_one(q.x);
            v.y = score_one(q.y);
            v.z = score_one(q.z);
            v.w = score_one(q.w);
            out4[i] = v;
        }
    }
    for (int t = t0 + 4 * n4 + threadIdx.x; t < t1; t += kDistThreads) out[t] = score_one(pos[t]);
    if (__syncthreads_or(bad) && threadIdx.x == 0) raise_flag(p.status, TRI_DEVFLAG_BOUNDS);
    if (!p.unit_kmin) return;
    lo = __reduce_min_sync(0xffffffffu, lo);
    hi = __reduce_max_sync(0xffffffffu, hi);
    if ((threadIdx.x & 31) == 0) {
        wlo[threadIdx.x >> 5] = lo;
        whi[threadIdx.x >> 5] = hi;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        for (int w = 1; w < kDistThreads / 32; ++w) {
            lo = min(lo, wlo[w]);
            hi = max(hi, whi[w]);
        }
        atomicMin(&p.unit_kmin[u], lo);
        atomicMax(&p.unit_kmax[u], hi);
    }
}

}  // namespace

cudaError_t launch_distance_table(const DistTableParams& p, cudaStream_t stream) {
    const int n_sets = p.per_head ? p.G : 1;
    const size_t smem = (size_t)n_sets * kBands * 2 * sizeof(double);
    const int64_t chunks = ((int64_t)p.max_dist + 1 + kTableThreads - 1) / kTableThreads;
    if (chunks > 65535) return cudaErrorInvalidValue;
    cudaError_t e = cudaFuncSetAttribute(distance_table_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (e != cudaSuccess) return e;
    distance_table_kernel<<<dim3(p.L * p.Hkv, (unsigned)chunks), kTableThreads, smem, stream>>>(p);
    return cudaGetLastError();
}

cudaError_t launch_distance_score(const DistScoreParams& p, cudaStream_t stream, bool pdl) {
    const int U = p.S * p.L * p.Hkv;
    if (U == 0) return cudaSuccess;
    const int64_t chunks = (p.pos_stride + kDistChunk - 1) / kDistChunk;
    if (chunks > 65535) return cudaErrorInvalidValue;
    return launch_kernel(distance_score_kernel, dim3(U, (unsigned)chunks), dim3(kDistThreads), 0, stream, pdl, p);
}

}  // namespace tri
