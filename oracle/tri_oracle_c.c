/*
 * tri_oracle_c.c - plain C float64 restatement of the oracle's per-unit
 * step (score, select, compact), used to time the CPU baseline on every
 * host core.
 *
 * TEST INFRASTRUCTURE.  Only the tests, __graft_entry__ and the CPU legs of
 * bench.py load it; the CUDA library never does, and it shares no code,
 * header, table or constant with that library.  It follows tri_oracle.py
 * definition by definition (and tests/test_oracle_c.py checks that the two
 * agree), with no blocking, folding or reordering beyond what the
 * definitions state.
 *
 * Pages (title, then section):
 *   "TriAttention: Trigonometric KV Compression for Efficient Long
 *   Reasoning" - "Core Mechanism" (keep the top-scoring keys), "Key
 *   Concepts" (Trigonometric Distance Preference, Norm as Importance Signal);
 *   "TriAttention: How a Geometric Trick Cuts LLM Memory Use by 10x Without
 *   Losing Accuracy" - "The Core Idea" (norm signal weighted by measured
 *   concentration), "Solving the Memory Fragmentation Problem"
 *   (forward-packing compaction).
 *
 * Band i of a D-dimensional vector x is the complex number x_i + j x_{i+D/2}
 * (rotate-half); theta_i = base^(-2i/D).  For a unit with G query heads:
 *   m_i    = mean_delta exp(j theta_i (p + delta))
 *   c_g,i  = qbar_g,i * m_i
 *   s_g(t) = sum_i Re(c_g,i conj(k_t,i)) + (1 - R_g) sum_i (A_g,i - |qbar_g,i|) |k_t,i|
 *   s(t)   = mean_g s_g(t)   (or max_g s_g(t), the max-over-group variant)
 * Selection: len <= B keeps every slot; otherwise the first S slots (attention
 * sinks, a variant; S = 0 for the method), the last W slots and the
 * B - W - S best of the slots between them by (score descending, slot
 * ascending), output ascending.  Compaction: row j takes row idx_j.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

static double bf16_to_double(uint16_t b) {
    uint32_t w = (uint32_t)b << 16;
    float f;
    memcpy(&f, &w, sizeof f);
    return (double)f;
}

typedef struct {
    double score;
    int slot;
} ranked;

/* score descending, slot ascending; NaN ranks as -infinity */
static int by_score_then_slot(const void *a, const void *b) {
    const ranked *x = (const ranked *)a, *y = (const ranked *)b;
    const double sx = isnan(x->score) ? -INFINITY : x->score;
    const double sy = isnan(y->score) ? -INFINITY : y->score;
    if (sx > sy) return -1;
    if (sx < sy) return 1;
    return (x->slot > y->slot) - (x->slot < y->slot);
}

static int ascending(const void *a, const void *b) {
    const int x = *(const int *)a, y = *(const int *)b;
    return (x > y) - (x < y);
}

/*
 * One unit.  keys, vals: bf16 bit patterns [T][D]; qbar [G][D], qabs [G][D/2],
 * R [G] in float64; sinks: leading slots always kept; agg_max: 0 for the
 * group mean, 1 for the group maximum.  Outputs: scores [T], idx [min(T, B)]
 * (returns its length), keys_out / vals_out [T][D] (rows past the kept count
 * unchanged).  Returns -1 on a bad argument or allocation failure.
 */
int tri_oracle_unit(const uint16_t *keys, const uint16_t *vals, int T, int D, const double *qbar,
                    const double *qabs, const double *R, int G, int64_t p, const int32_t *deltas, int nd,
                    double base, int budget, int window, int sinks, int agg_max, double *scores, int32_t *idx,
                    uint16_t *keys_out, uint16_t *vals_out) {
    if (T < 0 || D < 2 || D % 2 || G < 1 || nd < 1 || budget < 1 || window < 0 || sinks < 0 ||
        window + sinks > budget || (agg_max != 0 && agg_max != 1))
        return -1;
    const int n = D / 2;
    double *mr = (double *)malloc(sizeof(double) * n * (2 + 3 * G));
    if (!mr) return -1;
    double *mi = mr + n, *cr = mi + n, *ci = cr + n * G, *wt = ci + n * G;

    /* phase mean over the future offsets */
    for (int i = 0; i < n; ++i) {
        const double theta = pow(base, -2.0 * (double)i / (double)D);
        double re = 0.0, im = 0.0;
        for (int d = 0; d < nd; ++d) {
            const double a = theta * (double)(p + (int64_t)deltas[d]);
            re += cos(a);
            im += sin(a);
        }
        mr[i] = re / nd;
        mi[i] = im / nd;
    }
    /* per head: effective query bands and norm weights */
    for (int g = 0; g < G; ++g) {
        for (int i = 0; i < n; ++i) {
            const double xr = qbar[g * D + i], xi = qbar[g * D + i + n];
            cr[g * n + i] = xr * mr[i] - xi * mi[i];
            ci[g * n + i] = xr * mi[i] + xi * mr[i];
            wt[g * n + i] = (1.0 - R[g]) * (qabs[g * n + i] - sqrt(xr * xr + xi * xi));
        }
    }
    /* scores: mean (or maximum) over the heads of trig + weighted norm */
    for (int t = 0; t < T; ++t) {
        double total = 0.0, best = 0.0;
        for (int g = 0; g < G; ++g) {
            double trig = 0.0, norm = 0.0;
            for (int i = 0; i < n; ++i) {
                const double kr = bf16_to_double(keys[(size_t)t * D + i]);
                const double ki = bf16_to_double(keys[(size_t)t * D + i + n]);
                /* Re(c * conj(k)) */
                trig += cr[g * n + i] * kr + ci[g * n + i] * ki;
                norm += wt[g * n + i] * sqrt(kr * kr + ki * ki);
            }
            const double sg = trig + norm;
            total += sg;
            best = (g == 0 || sg > best) ? sg : best;
        }
        scores[t] = agg_max ? best : total / G;
    }
    free(mr);

    /* selection */
    int kept;
    if (T <= budget) {
        kept = T;
        for (int t = 0; t < T; ++t) idx[t] = t;
    } else {
        const int cand = T - window, take = budget - window - sinks, nr = cand - sinks;
        ranked *r = (ranked *)malloc(sizeof(ranked) * (nr > 0 ? nr : 1));
        if (!r) return -1;
        for (int t = sinks; t < cand; ++t) {
            r[t - sinks].score = scores[t];
            r[t - sinks].slot = t;
        }
        qsort(r, nr, sizeof(ranked), by_score_then_slot);
        for (int j = 0; j < sinks; ++j) idx[j] = j;
        for (int j = 0; j < take; ++j) idx[sinks + j] = r[j].slot;
        free(r);
        qsort(idx + sinks, take, sizeof(int32_t), ascending);
        for (int j = 0; j < window; ++j) idx[sinks + take + j] = cand + j;
        kept = budget;
    }

    /* compaction: row j takes row idx_j */
    memcpy(keys_out, keys, sizeof(uint16_t) * (size_t)T * D);
    memcpy(vals_out, vals, sizeof(uint16_t) * (size_t)T * D);
    for (int j = 0; j < kept; ++j) {
        memcpy(keys_out + (size_t)j * D, keys + (size_t)idx[j] * D, sizeof(uint16_t) * D);
        memcpy(vals_out + (size_t)j * D, vals + (size_t)idx[j] * D, sizeof(uint16_t) * D);
    }
    return kept;
}
