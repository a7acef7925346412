// band_f32.cuh -- K3: fp32 rows that are not global, on CUDA cores.
//
// One warp per query row i of (b, h).  The lanes split the row's key set
// K(i) = dilated window {i + dil*t : |t| <= r} (clipped to [0, T), padded
// keys dropped) plus the global keys that are not already in the window
// (each key once; "Longformer" note, sections "Sliding-Window Attention"
// and "Global Attention").  Each lane keeps an online softmax
// (running max, sum, weighted value sum) in fp32 over its keys; the warp
// then merges the 32 partial states with shuffles.  FFMA dot products and
// exp2f keep the result within 1e-5 of the fp64 definition for unit-scale
// inputs.  Global rows are written by the global-row kernel.
#pragma once
#include "lf_common.cuh"

namespace lf {

constexpr int kBandF32Warps = 4;

template <int DP>
__global__ void __launch_bounds__(kBandF32Warps * 32) band_f32_kernel(const __grid_constant__ BandF32Params p) {
    const int lane = threadIdx.x & 31;
    const long row_id = static_cast<long>(blockIdx.x) * kBandF32Warps + (threadIdx.x >> 5);
    const int T = p.T, d = p.d;
    if (row_id >= static_cast<long>(p.B) * p.H * T) return;
    const int i = static_cast<int>(row_id % T);
    const long bh = row_id / T;
    const int h = static_cast<int>(bh % p.H);
    const int b = static_cast<int>(bh / p.H);
    if ((p.ws.gbit[static_cast<size_t>(b) * p.W + (i >> 5)] >> (i & 31)) & 1u) return;  // global row

    const int dil = p.dil[h];
    const float* qi = p.q + (bh * T + i) * d;
    const float* kb = p.k + bh * T * d;
    const float* vb = p.v + bh * T * d;
    const uint8_t* pad_b = p.pad ? p.pad + static_cast<size_t>(b) * T : nullptr;

    float q[DP];
#pragma unroll
    for (int c = 0; c < DP; ++c) q[c] = c < d ? qi[c] : 0.f;
    float acc[DP];
#pragma unroll
    for (int c = 0; c < DP; ++c) acc[c] = 0.f;
    float m = -INFINITY, l = 0.f;

    auto visit = [&](int j) {
        const float* kj = kb + static_cast<size_t>(j) * d;
        float s = 0.f;
#pragma unroll
        for (int c = 0; c < DP; ++c)
            if (c < d) s = fmaf(q[c], kj[c], s);
        s *= p.sl2;
        if (s > m) {
            float f = exp2f(m - s);
            l *= f;
#pragma unroll
            for (int c = 0; c < DP; ++c) acc[c] *= f;
            m = s;
        }
        float pj = exp2f(s - m);
        l += pj;
        const float* vj = vb + static_cast<size_t>(j) * d;
#pragma unroll
        for (int c = 0; c < DP; ++c)
            if (c < d) acc[c] = fmaf(pj, vj[c], acc[c]);
    };

    // window keys
    for (long t = -static_cast<long>(p.r) + lane; t <= p.r; t += 32) {
        long j = static_cast<long>(i) + static_cast<long>(dil) * t;
        if (j < 0) continue;
        if (j >= T) break;
        if (pad_b && pad_b[j]) continue;
        visit(static_cast<int>(j));
    }
    // global keys outside the window (padded ones were dropped by prep)
    const int ngk = p.ws.n_gk[b];
    const int32_t* gk = p.ws.gk_list + static_cast<size_t>(b) * p.gstride;
    const long reach = static_cast<long>(dil) * p.r;
    for (int a = lane; a < ngk; a += 32) {
        int g = gk[a];
        long diff = static_cast<long>(g) - i;
        bool in_window = (diff % dil == 0) && (diff <= reach) && (diff >= -reach);
        if (!in_window) visit(g);
    }

    // merge the 32 lane states
    float M = m;
#pragma unroll
    for (int o = 16; o; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
    float f = (m == -INFINITY) ? 0.f : exp2f(m - M);
    float L = l * f;
#pragma unroll
    for (int o = 16; o; o >>= 1) L += __shfl_xor_sync(0xffffffffu, L, o);
    float inv = L > 0.f ? 1.f / L : 0.f;
    float* orow = p.out + (bh * T + i) * d;
#pragma unroll
    for (int c = 0; c < DP; ++c) {
        float a = acc[c] * f;
#pragma unroll
        for (int o = 16; o; o >>= 1) a += __shfl_xor_sync(0xffffffffu, a, o);
        if (c < d && lane == (c & 31)) orow[c] = a * inv;
    }
}

}  // namespace lf
