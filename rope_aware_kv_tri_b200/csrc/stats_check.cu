// stats_check.cu - sanity check of the head statistics a step is given.
//
// Page: "TriAttention: trigonometric KV cache compression for long
// reasoning" - "Calibration statistics are tied to a specific model":
// statistics from another model, or a damaged statistics file, raise no
// error of their own; the step simply keeps the wrong keys.  This kernel
// checks what the method's definitions imply about any valid statistics:
//   * every centre dimension, band magnitude mean and concentration is finite;
//   * the concentration R lies in [0, 1];
//   * E|q_i| >= |qbar_i| for every band (the mean of magnitudes is at least
//     the magnitude of the mean), so every norm weight (1 - R)(E|q_i| -
//     |qbar_i|) is >= 0.  A negative weight inverts the norm ranking.
//     Checked with a relative slack of 1e-5 for the fp32 rounding of both.
// and reports, without failing on it, whether R equals its definition
// sum_i |qbar_i| / sum_i E|q_i| to 1e-3 relative.
//
// One 64-thread group per head (thread i: band i), four heads per CTA; the
// band sums are reduced in float64.
#include "tri_device.cuh"
#include "tri_internal.h"

namespace tri {

namespace {

constexpr int kCheckThreads = 256;
constexpr int kHeadsPerCta = kCheckThreads / kBands;   // 4
constexpr double kNormSlack = 1e-5;
constexpr double kRTolerance = 1e-3;

__global__ void __launch_bounds__(kCheckThreads) check_stats_kernel(const StatsCheckParams p) {
    __shared__ double s_mag[kHeadsPerCta][2], s_abs[kHeadsPerCta][2];
    __shared__ int s_bits[kHeadsPerCta][2];
    const int i = threadIdx.x % kBands;
    const int grp = threadIdx.x / kBands;
    const int half = i / 32;                     // warp of the head's group
    const int64_t head = (int64_t)blockIdx.x * kHeadsPerCta + grp;
    const bool live = head < p.n_heads;
    int bits = 0;
    double mag = 0.0, a = 0.0;
    if (live) {
        const float xr = p.qbar[head * kHeadDim + i];
        const float xi = p.qbar[head * kHeadDim + i + kBands];
        const float qa = p.qabs[head * kBands + i];
        if (!isfinite(xr) || !isfinite(xi) || !isfinite(qa)) {
            bits |= TRI_STATS_NONFINITE;
        } else {
            mag = sqrt((double)xr * xr + (double)xi * xi);
            a = qa;
            if (a < mag * (1.0 - kNormSlack)) bits |= TRI_STATS_NORM_WEIGHT;
        }
    }
    mag = warp_sum_f64(mag);
    a = warp_sum_f64(a);
    bits = __reduce_or_sync(0xffffffffu, bits);
    if ((threadIdx.x & 31) == 0) {
        s_mag[grp][half] = mag;
        s_abs[grp][half] = a;
        s_bits[grp][half] = bits;
    }
    __syncthreads();
    if (!live || i != 0) return;
    bits = s_bits[grp][0] | s_bits[grp][1];
    const double sum_mag = s_mag[grp][0] + s_mag[grp][1];
    const double sum_abs = s_abs[grp][0] + s_abs[grp][1];
    const float r = p.R[head];
    if (!isfinite(r)) {
        bits |= TRI_STATS_NONFINITE;
    } else {
        if (r < 0.f || r > 1.f) bits |= TRI_STATS_R_RANGE;
        if (!(bits & TRI_STATS_NONFINITE)) {
            const double ref = sum_abs > 0.0 ? sum_mag / sum_abs : 1.0;
            if (fabs((double)r - ref) > kRTolerance * ref + 1e-6) bits |= TRI_STATS_R_MISMATCH;
        }
    }
    if (p.head_flags) p.head_flags[head] = bits;
    if (bits & (TRI_STATS_NONFINITE | TRI_STATS_R_RANGE | TRI_STATS_NORM_WEIGHT)) {
        raise_flag(p.status, TRI_DEVFLAG_STATS);
        if (p.abort_word) atomicOr(p.abort_word, 1);
    }
}

}  // namespace

cudaError_t launch_check_stats(const StatsCheckParams& p, cudaStream_t stream) {
    if (p.n_heads <= 0) return cudaSuccess;
    const int64_t grid = (p.n_heads + kHeadsPerCta - 1) / kHeadsPerCta;
    check_stats_kernel<<<(unsigned)grid, kCheckThreads, 0, stream>>>(p);
    return cudaGetLastError();
}

}  // namespace tri
