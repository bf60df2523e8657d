// query.cu - the effective query of every unit, and the per-sequence plan of
// a step.
//
// Pages: "TriAttention: Trigonometric KV Compression for Efficient Long
// Reasoning" - "Key Concepts", Trigonometric Distance Preference (after
// rotation the centre dot product is a cosine series in the distance);
// "TriAttention: How a Geometric Trick Cuts LLM Memory Use by 10x Without
// Losing Accuracy" - "The Core Idea" (norm signal weighted by the measured
// concentration).
//
// For unit (s, l, h) and band i (one thread each):
//   m_i  = mean_delta exp(j theta_i (p_s + delta)),  theta_i = base^(-2i/D)
//   qeff = real dims of mean_g qbar_{g,i} m_i          (bands i -> dims i, i+64)
//   w_i  = mean_g (1 - R_g)(qabs_{g,i} - |qbar_{g,i}|)
// all in float64 (the phase reaches ~1.4e5 rad), rounded to fp32 at the end.
// The score of key K is then qeff . K + sum_i w_i |K band i|: the mean over
// the GQA group of the per-head trigonometric + weighted-norm score, because
// both terms are linear in their coefficients.
//
// The last CTA of the grid (when planning) validates the sequence lengths,
// copies them to the workspace, and writes the prefix offsets of the score
// work items and of the freed-block list.
#include "tri_device.cuh"
#include "tri_internal.h"

namespace tri {

namespace {

constexpr int kQueryThreads = 256;
constexpr int kUnitsPerCta = kQueryThreads / kBands;   // 4

__device__ void build_unit_query(const QueryParams& p, int u) {
    const int i = threadIdx.x % kBands;
    const int LH = p.L * p.Hkv;
    const int s = u / LH, rem = u % LH, l = rem / p.Hkv, h = rem % p.Hkv;
    const int Hq = p.Hkv * p.G;
    const int64_t pos = p.cur_pos[s];
    const double theta = pow(p.base, -2.0 * (double)i / (double)kHeadDim);
    double mr = 0.0, mi = 0.0;
    for (int d = 0; d < p.n_deltas; ++d) {
        double sn, cs;
        sincos(theta * (double)(pos + (int64_t)p.deltas[d]), &sn, &cs);
        mr += cs;
        mi += sn;
    }
    mr /= p.n_deltas;
    mi /= p.n_deltas;
    double cr = 0.0, ci = 0.0, wa = 0.0;
    for (int g = 0; g < p.G; ++g) {
        const int64_t row = (int64_t)l * Hq + (int64_t)h * p.G + g;
        const double xr = p.qbar[row * kHeadDim + i];
        const double xi = p.qbar[row * kHeadDim + i + kBands];
        cr += xr * mr - xi * mi;
        ci += xr * mi + xi * mr;
        wa += (1.0 - (double)p.R[row]) * ((double)p.qabs[row * kBands + i] - sqrt(xr * xr + xi * xi));
    }
    const double invG = 1.0 / p.G;
    p.qeff[(int64_t)u * kHeadDim + i] = (float)(cr * invG);
    p.qeff[(int64_t)u * kHeadDim + i + kBands] = (float)(ci * invG);
    p.wts[(int64_t)u * kBands + i] = (float)(wa * invG);
}

__device__ void plan_sequences(const QueryParams& p) {
    __shared__ int warp_tmp[kQueryThreads / 32];
    const int n_hg = p.Hkv / p.heads_per_tile;
    const int64_t max_len = (int64_t)p.max_blocks * kBlockRows;
    int carry_items = 0, carry_freed = 0;
    for (int c0 = 0; c0 < p.S; c0 += kQueryThreads) {
        const int s = c0 + threadIdx.x;
        int items = 0, nf = 0;
        if (s < p.S) {
            int len = p.seq_len[s];
            if (len < 0 || (int64_t)len > max_len) {
                raise_flag(p.status, TRI_DEVFLAG_BOUNDS);
                len = 0;
            }
            p.len_ws[s] = len;
            const int nblk = (len + kBlockRows - 1) / kBlockRows;
            const bool compress = p.budget > 0;
            const int scored = (compress && len <= p.budget) ? 0 : nblk;
            items = p.L * n_hg * ((scored + kChunkBlocks - 1) / kChunkBlocks);
            if (compress) {
                const int kept = len < p.budget ? len : p.budget;
                nf = nblk - (kept + kBlockRows - 1) / kBlockRows;
            }
        }
        int tot_i, tot_f;
        const int ex_i = block_exclusive_scan<kQueryThreads>(items, warp_tmp, tot_i);
        const int ex_f = block_exclusive_scan<kQueryThreads>(nf, warp_tmp, tot_f);
        if (s < p.S) {
            p.item_off[s] = carry_items + ex_i;
            p.freed_off[s] = carry_freed + ex_f;
        }
        carry_items += tot_i;
        carry_freed += tot_f;
    }
    if (threadIdx.x == 0) {
        p.item_off[p.S] = carry_items;
        p.freed_off[p.S] = carry_freed;
        if (p.freed_count) *p.freed_count = carry_freed;
    }
}

__global__ void __launch_bounds__(kQueryThreads) query_kernel(const QueryParams p, int n_query_ctas) {
    if ((int)blockIdx.x == n_query_ctas) {
        plan_sequences(p);
        return;
    }
    const int U = p.S * p.L * p.Hkv;
    const int u = blockIdx.x * kUnitsPerCta + threadIdx.x / kBands;
    if (u < U) build_unit_query(p, u);
}

}  // namespace

cudaError_t launch_query(const QueryParams& p, cudaStream_t stream) {
    const int U = p.S * p.L * p.Hkv;
    const int nq = (U + kUnitsPerCta - 1) / kUnitsPerCta;
    query_kernel<<<nq + (p.do_plan ? 1 : 0), kQueryThreads, 0, stream>>>(p, nq);
    return cudaGetLastError();
}

}  // namespace tri
