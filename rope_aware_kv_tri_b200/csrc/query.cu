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
// For unit (s, l, h) and band i:
//   m_i  = mean_delta exp(j theta_i (p_s + delta)),  theta_i = base^(-2i/D)
//   qeff = real dims of mean_g qbar_{g,i} m_i          (bands i -> dims i, i+64)
//   w_i  = mean_g (1 - R_g)(qabs_{g,i} - |qbar_{g,i}|)
// all in float64 (the phase reaches ~1.4e5 rad), rounded to fp32 at the end.
// The score of key K is then qeff . K + sum_i w_i |K band i|: the mean over
// the GQA group of the per-head trigonometric + weighted-norm score, because
// both terms are linear in their coefficients.
//
// With the max-over-group aggregation the G heads are not folded: head g of
// unit u gets its own qbar_g m (real dims) and (1 - R_g)(qabs_g - |qbar_g|)
// at [u][g], and the score kernel takes the largest of the G head scores.
//
// The last CTA of the grid (when planning) validates the sequence lengths,
// copies them to the workspace, and writes the prefix offsets of the score
// work items and of the freed-block list.  A sequence is compressed when its
// length exceeds the trigger (at least the budget); when a device free list
// is given it also reserves the list entries the freed ids will fill.  When
// the step's statistics check (stats_check.cu) vetoed the step, nothing is
// planned: no work items, no freed blocks, no free-list entries.
#include "tri_device.cuh"
#include "tri_internal.h"

namespace tri {

namespace {

constexpr int kQueryThreads = 256;
constexpr int kUnitsPerCta = kQueryThreads / kBands;   // 4

// CTA b builds units [4k, 4k + 4) of sequence s (k = b mod ctas_per_seq):
// the phase mean m_i of the sequence is shared, its offsets split over the
// four 64-thread groups; then group g folds unit 4k + g.
__device__ void build_unit_queries(const QueryParams& p, int b, int ctas_per_seq) {
    __shared__ double s_mr[kUnitsPerCta][kBands], s_mi[kUnitsPerCta][kBands];
    const int i = threadIdx.x % kBands;
    const int grp = threadIdx.x / kBands;
    const int LH = p.L * p.Hkv;
    const int s = b / ctas_per_seq;
    const int64_t pos = p.cur_pos[s];
    const double theta = pow(p.base, -2.0 * (double)i / (double)kHeadDim);
    double mr = 0.0, mi = 0.0;
    for (int d = grp; d < p.n_deltas; d += kUnitsPerCta) {
        double sn, cs;
        sincos(theta * (double)(pos + (int64_t)p.deltas[d]), &sn, &cs);
        mr += cs;
        mi += sn;
    }
    s_mr[grp][i] = mr;
    s_mi[grp][i] = mi;
    __syncthreads();
    mr = (s_mr[0][i] + s_mr[1][i]) + (s_mr[2][i] + s_mr[3][i]);
    mi = (s_mi[0][i] + s_mi[1][i]) + (s_mi[2][i] + s_mi[3][i]);
    mr /= p.n_deltas;
    mi /= p.n_deltas;
    const int k = (b % ctas_per_seq) * kUnitsPerCta + grp;     // unit within the sequence
    if (k >= LH) return;
    const int u = s * LH + k;
    const int l = k / p.Hkv, h = k % p.Hkv;
    const int Hq = p.Hkv * p.G;
    if (p.per_head) {
        for (int g = 0; g < p.G; ++g) {
            const int64_t row = (int64_t)l * Hq + (int64_t)h * p.G + g;
            const double xr = p.qbar[row * kHeadDim + i];
            const double xi = p.qbar[row * kHeadDim + i + kBands];
            const int64_t o = (int64_t)u * p.G + g;
            p.qeff[o * kHeadDim + i] = (float)(xr * mr - xi * mi);
            p.qeff[o * kHeadDim + i + kBands] = (float)(xr * mi + xi * mr);
            p.wts[o * kBands + i] =
                (float)((1.0 - (double)p.R[row]) * ((double)p.qabs[row * kBands + i] - sqrt(xr * xr + xi * xi)));
        }
        if (i == 0 && p.unit_kmin) {
            p.unit_kmin[u] = 0xffffffffu;
            p.unit_kmax[u] = 0u;
        }
        return;
    }
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
    if (i == 0 && p.unit_kmin) {
        p.unit_kmin[u] = 0xffffffffu;
        p.unit_kmax[u] = 0u;
    }
}

__device__ void plan_sequences(const QueryParams& p) {
    __shared__ int warp_tmp[kQueryThreads / 32];
    const int n_hg = p.Hkv / p.heads_per_tile;
    const int64_t max_len = (int64_t)p.max_blocks * kBlockRows;
    // a step vetoed by the statistics check scores, selects and frees nothing
    const bool vetoed = p.abort_word != nullptr && *p.abort_word != 0;
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
            const bool touched = !vetoed && (!compress || len > p.trigger);
            const int scored = touched ? nblk : 0;
            items = p.L * n_hg * ((scored + kChunkBlocks - 1) / kChunkBlocks);
            if (compress && touched) nf = nblk - (p.budget + kBlockRows - 1) / kBlockRows;
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
    if (p.fq_words && threadIdx.x < kQwWords) p.fq_words[threadIdx.x] = 0;   // select + compact unit counter
    if (p.plan_only && p.unit_kmin) {
        const int U = p.S * p.L * p.Hkv;
        for (int u = threadIdx.x; u < U; u += kQueryThreads) {
            p.unit_kmin[u] = 0xffffffffu;
            p.unit_kmax[u] = 0u;
        }
    }
    if (threadIdx.x == 0) {
        p.item_off[p.S] = carry_items;
        p.freed_off[p.S] = carry_freed;
        if (p.freed_count) *p.freed_count = carry_freed;
        if (p.fl_count) {
            const int have = *p.fl_count;
            if (have >= 0 && (int64_t)have + carry_freed <= (int64_t)p.fl_capacity) {
                *p.fl_count = have + carry_freed;
                *p.fl_base = have;
            } else {
                *p.fl_base = -1;
                raise_flag(p.status, TRI_DEVFLAG_FREELIST);
            }
        }
        if (p.zero_words) {
            p.zero_words[0] = 0;
            p.zero_words[1] = 0;
        }
    }
}

__global__ void __launch_bounds__(kQueryThreads) query_kernel(const QueryParams p, int ctas_per_seq) {
    allow_next_grid();
    const int n_query_ctas = p.S * ctas_per_seq;
    if ((int)blockIdx.x == n_query_ctas) {
        plan_sequences(p);
        return;
    }
    build_unit_queries(p, blockIdx.x, ctas_per_seq);
}

}  // namespace

cudaError_t launch_query(const QueryParams& p, cudaStream_t stream) {
    if (p.plan_only) {
        query_kernel<<<1, kQueryThreads, 0, stream>>>(p, 0);
        return cudaGetLastError();
    }
    const int per_seq = (p.L * p.Hkv + kUnitsPerCta - 1) / kUnitsPerCta;
    query_kernel<<<p.S * per_seq + (p.do_plan ? 1 : 0), kQueryThreads, 0, stream>>>(p, per_seq);
    return cudaGetLastError();
}

}  // namespace tri
