// calibrate.cu - reduction of pre-rotary query samples to head statistics.
//
// Pages: "TriAttention: Trigonometric KV Compression for Efficient Long
// Reasoning" - "Core Mechanism" (one-time centre calibration in the data-flow
// figure) and "Key Concepts", Q/K Concentration (the centre is the mean
// pre-rotary query); "TriAttention: How a Geometric Trick Cuts LLM Memory Use
// by 10x Without Losing Accuracy" - "The Core Idea" (a measured concentration
// per head).
//
// One CTA per (layer, query head).  256 threads = 64 bands x 4 sample
// stripes; each thread accumulates, in float64, the real and imaginary parts
// and the magnitude of its band over its stripe of samples.  A sample's 128
// floats are contiguous, so each stripe reads two coalesced 256-byte runs per
// sample.  Untimed: it runs once per model.
#include "tri_device.cuh"
#include "tri_internal.h"

namespace tri {

namespace {

constexpr int kCalThreads = 256;
constexpr int kStripes = kCalThreads / kBands;

__global__ void __launch_bounds__(kCalThreads) calibrate_kernel(const float* __restrict__ q, int N, int LHq,
                                                                float* __restrict__ qbar,
                                                                float* __restrict__ qabs,
                                                                float* __restrict__ R) {
    __shared__ double s_re[kStripes][kBands];
    __shared__ double s_im[kStripes][kBands];
    __shared__ double s_ab[kStripes][kBands];
    __shared__ double s_num[kBands / 32], s_den[kBands / 32];

    const int head = blockIdx.x;            // l * Hq + hq
    const int i = threadIdx.x % kBands;
    const int stripe = threadIdx.x / kBands;
    double re = 0.0, im = 0.0, ab = 0.0;
    const int64_t stride = (int64_t)LHq * kHeadDim;
    const float* base = q + (int64_t)head * kHeadDim;
    for (int n = stripe; n < N; n += kStripes) {
        const float* row = base + (int64_t)n * stride;
        const double x = row[i], y = row[i + kBands];
        re += x;
        im += y;
        ab += sqrt(x * x + y * y);
    }
    s_re[stripe][i] = re;
    s_im[stripe][i] = im;
    s_ab[stripe][i] = ab;
    __syncthreads();
    if (threadIdx.x < kBands) {
        double tr = 0.0, ti = 0.0, ta = 0.0;
        for (int s = 0; s < kStripes; ++s) {
            tr += s_re[s][i];
            ti += s_im[s][i];
            ta += s_ab[s][i];
        }
        const double mr = tr / N, mi = ti / N, ma = ta / N;
        qbar[(int64_t)head * kHeadDim + i] = (float)mr;
        qbar[(int64_t)head * kHeadDim + i + kBands] = (float)mi;
        qabs[(int64_t)head * kBands + i] = (float)ma;
        double num = sqrt(mr * mr + mi * mi), den = ma;
        for (int o = 16; o > 0; o >>= 1) {
            num += __shfl_xor_sync(0xffffffffu, num, o);
            den += __shfl_xor_sync(0xffffffffu, den, o);
        }
        if ((threadIdx.x & 31) == 0) {
            s_num[threadIdx.x >> 5] = num;
            s_den[threadIdx.x >> 5] = den;
        }
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        double num = 0.0, den = 0.0;
        for (int w = 0; w < kBands / 32; ++w) {
            num += s_num[w];
            den += s_den[w];
        }
        R[head] = den > 0.0 ? (float)(num / den) : 1.0f;
    }
}

}  // namespace

cudaError_t launch_calibrate(const float* q, int N, int L, int Hq, float* qbar, float* qabs, float* R,
                             cudaStream_t stream) {
    calibrate_kernel<<<L * Hq, kCalThreads, 0, stream>>>(q, N, L * Hq, qbar, qabs, R);
    return cudaGetLastError();
}

}  // namespace tri
