// score_device.cuh - the per-key score of the mean-aggregated path and the
// coefficient loads it needs (used by the score kernel, score.cu).
//
// Pages: "TriAttention: Trigonometric KV Compression for Efficient Long
// Reasoning" - "Key Concepts", Trigonometric Distance Preference and Norm as
// Importance Signal.
//
// A key K (bf16, D = 128) is split over 8 lanes: lane `sub` holds 16 bytes of
// the real half (dims 8sub..8sub+7) and the matching 16 bytes of the
// imaginary half (dims 64+8sub..), i.e. whole bands 8sub..8sub+7.  Its part
// of s = qeff . K + sum_i w_i sqrt(K_i^2 + K_{i+64}^2) is formed on packed
// pairs of adjacent bands (fma.rn.f32x2); the 8 parts are summed by the
// caller with three xor-shuffles.
#pragma once

#include "tri_device.cuh"

namespace tri {

__device__ __forceinline__ float key_score(const uint4 a, const uint4 b, const float2 (&qr)[4],
                                           const float2 (&qi)[4], const float2 (&ww)[4]) {
    const uint32_t av[4] = {a.x, a.y, a.z, a.w};
    const uint32_t bv[4] = {b.x, b.y, b.z, b.w};
    float2 dot = make_float2(0.f, 0.f), nrm = make_float2(0.f, 0.f);
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const float2 r = make_float2(bf16_lo(av[j]), bf16_hi(av[j]));
        const float2 i = make_float2(bf16_lo(bv[j]), bf16_hi(bv[j]));
        dot = ffma2(qr[j], r, dot);
        dot = ffma2(qi[j], i, dot);
        const float2 sq = ffma2(r, r, fmul2(i, i));
        nrm = ffma2(ww[j], make_float2(sqrt_fast(sq.x), sqrt_fast(sq.y)), nrm);
    }
    return (dot.x + dot.y) + (nrm.x + nrm.y);
}

// The coefficients a lane needs for its 8 bands of unit `unit`: qeff real and
// imaginary dims and the norm weights, as adjacent-band pairs.
__device__ __forceinline__ void load_key_coefficients(const float* qeff, const float* wts, int64_t unit, int sub,
                                                      float2 (&qr)[4], float2 (&qi)[4], float2 (&ww)[4]) {
    const float4* qe = reinterpret_cast<const float4*>(qeff + unit * TRI_HEAD_DIM);
    const float4* we = reinterpret_cast<const float4*>(wts + unit * (TRI_HEAD_DIM / 2));
    const float4 x0 = qe[2 * sub], x1 = qe[2 * sub + 1];
    const float4 y0 = qe[16 + 2 * sub], y1 = qe[16 + 2 * sub + 1];
    const float4 z0 = we[2 * sub], z1 = we[2 * sub + 1];
    qr[0] = make_float2(x0.x, x0.y); qr[1] = make_float2(x0.z, x0.w);
    qr[2] = make_float2(x1.x, x1.y); qr[3] = make_float2(x1.z, x1.w);
    qi[0] = make_float2(y0.x, y0.y); qi[1] = make_float2(y0.z, y0.w);
    qi[2] = make_float2(y1.x, y1.y); qi[3] = make_float2(y1.z, y1.w);
    ww[0] = make_float2(z0.x, z0.y); ww[1] = make_float2(z0.z, z0.w);
    ww[2] = make_float2(z1.x, z1.y); ww[3] = make_float2(z1.z, z1.w);
}

}  // namespace tri
