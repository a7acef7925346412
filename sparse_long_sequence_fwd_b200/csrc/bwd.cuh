// bwd.cuh -- the backward pass (dQ, dK, dV) of Longformer sparse attention,
// on the CUDA cores, one warp per row or per key.
//
// The pages train and fine-tune with this attention (Longformer wiki,
// sections 3.1 and 3.2; the aiqz.cc page, gradient checkpointing), so the
// gradients of y_i = sum_{j in K(i)} p_ij v_j, p_ij = softmax_j(s_ij),
// s_ij = scale q_i . k_j, with the key sets of the forward, are:
//   dv_j = sum_{i : j in K(i)} p_ij dy_i
//   ds_ij = p_ij (dy_i . v_j - D_i),  D_i = dy_i . y_i
//   dq_i = scale sum_{j in K(i)} ds_ij k_j
//   dk_j = scale sum_{i : j in K(i)} ds_ij q_i
// K(i) (the prep kernel's lists): for an ordinary row, the dilated window
// {i + dil t : |t| <= r} in [0, T) and the global keys, padded keys removed;
// for a global row, every non-padded key.  Three kernels: the row
// statistics (max and sum of the softmax, in the log2 domain, and D_i),
// dq by rows, and dk, dv by keys, which visits the rows whose key set holds
// key j: the window rows of j that are not global, and every global row;
// every row when j is a global key.
#pragma once
#include "global_rows.cuh"
#include "lf_common.cuh"
#include "ptx.cuh"

namespace lf {

constexpr int kBwdWarps = 4;  // warps per CTA: one row (or key) each

struct BwdParams {
    const void* q;
    const void* k;
    const void* v;
    const void* y;    // the forward's output
    const void* dy;   // the output gradient
    float* dq;        // [B,H,T,d] fp32
    float* dk;
    float* dv;
    float* stats;     // [B*H*T][3]: m (log2 domain), l, D
    const uint8_t* pad;
    Workspace ws;
    int B, H, T, d, r, gstride, W;
    int dil[kMaxHeads];
    float sl2;        // scale * log2(e)
    float scale;
};

// One lane's slice of a d-wide row (lane, lane + 32, ...; d <= 128).
template <typename Tin>
__device__ __forceinline__ void load_row(const Tin* row, int d, float* x) {
    const int lane = threadIdx.x & 31;
#pragma unroll
    for (int u = 0; u < 4; ++u) x[u] = lane + 32 * u < d ? load_as_float(row + lane + 32 * u) : 0.f;
}
__device__ __forceinline__ float warp_dot(const float* a, const float* b) {
    float s = a[0] * b[0];
#pragma unroll
    for (int u = 1; u < 4; ++u) s = fmaf(a[u], b[u], s);
#pragma unroll
    for (int o = 16; o; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
    return s;
}
__device__ __forceinline__ bool bwd_is_global(const BwdParams& p, int b, int i) {
    return (p.ws.gbit[static_cast<size_t>(b) * p.W + (i >> 5)] >> (i & 31)) & 1u;
}
__device__ __forceinline__ bool bwd_padded(const BwdParams& p, int b, int j) {
    return p.pad && p.pad[static_cast<size_t>(b) * p.T + j] != 0;
}

// Calls f(j) for every key j of row i's key set K(i), each once.
template <typename F>
__device__ __forceinline__ void for_each_key(const BwdParams& p, int b, int dil, int i, F f) {
    if (bwd_is_global(p, b, i)) {
        for (int j = 0; j < p.T; ++j)
            if (!bwd_padded(p, b, j)) f(j);
        return;
    }
    for (int t = -p.r; t <= p.r; ++t) {
        const long long j = static_cast<long long>(i) + static_cast<long long>(dil) * t;
        if (j >= 0 && j < p.T && !bwd_padded(p, b, static_cast<int>(j))) f(static_cast<int>(j));
    }
    const int ngk = p.ws.n_gk[b];  // global keys: not padded, sorted
    const int32_t* gk = p.ws.gk_list + static_cast<size_t>(b) * p.gstride;
    for (int a = 0; a < ngk; ++a) {
        const int j = gk[a], diff = j - i;
        const bool in_window = diff >= -dil * p.r && diff <= dil * p.r && diff % dil == 0;
        if (!in_window) f(j);
    }
}

// Row statistics: m_i (log2 domain), l_i and D_i = dy_i . y_i.
template <typename Tin>
__global__ void __launch_bounds__(kBwdWarps * 32) bwd_stats_kernel(const __grid_constant__ BwdParams p) {
    const size_t row = static_cast<size_t>(blockIdx.x) * kBwdWarps + (threadIdx.x >> 5);
    if (row >= static_cast<size_t>(p.B) * p.H * p.T) return;
    const int i = static_cast<int>(row % p.T), bh = static_cast<int>(row / p.T), b = bh / p.H, h = bh % p.H;
    const size_t base = static_cast<size_t>(bh) * p.T * p.d;
    const Tin* q = reinterpret_cast<const Tin*>(p.q) + base;
    const Tin* k = reinterpret_cast<const Tin*>(p.k) + base;
    float qi[4], a[4], c[4];
    load_row(q + static_cast<size_t>(i) * p.d, p.d, qi);
    load_row(reinterpret_cast<const Tin*>(p.dy) + base + static_cast<size_t>(i) * p.d, p.d, a);
    load_row(reinterpret_cast<const Tin*>(p.y) + base + static_cast<size_t>(i) * p.d, p.d, c);
    const float D = warp_dot(a, c);
    float m = -INFINITY, l = 0.f;
    for_each_key(p, b, p.dil[h], i, [&](int j) {
        float kj[4];
        load_row(k + static_cast<size_t>(j) * p.d, p.d, kj);
        const float s = warp_dot(qi, kj) * p.sl2;
        if (s > m) {
            l = l * exp2f(m - s) + 1.f;  // (m = -inf: l = 0, exp2f(-inf) = 0)
            m = s;
        } else {
            l += exp2f(s - m);
        }
    });
    if ((threadIdx.x & 31) == 0) {
        p.stats[3 * row] = m;
        p.stats[3 * row + 1] = l;
        p.stats[3 * row + 2] = D;
    }
}

// dq_i = scale sum_j ds_ij k_j.
template <typename Tin>
__global__ void __launch_bounds__(kBwdWarps * 32) bwd_dq_kernel(const __grid_constant__ BwdParams p) {
    const size_t row = static_cast<size_t>(blockIdx.x) * kBwdWarps + (threadIdx.x >> 5);
    if (row >= static_cast<size_t>(p.B) * p.H * p.T) return;
    const int lane = threadIdx.x & 31;
    const int i = static_cast<int>(row % p.T), bh = static_cast<int>(row / p.T), b = bh / p.H, h = bh % p.H;
    const size_t base = static_cast<size_t>(bh) * p.T * p.d;
    const Tin* k = reinterpret_cast<const Tin*>(p.k) + base;
    const Tin* v = reinterpret_cast<const Tin*>(p.v) + base;
    float qi[4], dyi[4], acc[4] = {0.f, 0.f, 0.f, 0.f};
    load_row(reinterpret_cast<const Tin*>(p.q) + base + static_cast<size_t>(i) * p.d, p.d, qi);
    load_row(reinterpret_cast<const Tin*>(p.dy) + base + static_cast<size_t>(i) * p.d, p.d, dyi);
    const float m = p.stats[3 * row], l = p.stats[3 * row + 1], D = p.stats[3 * row + 2];
    if (l > 0.f) {
        const float inv = 1.f / l;
        for_each_key(p, b, p.dil[h], i, [&](int j) {
            float kj[4], vj[4];
            load_row(k + static_cast<size_t>(j) * p.d, p.d, kj);
            load_row(v + static_cast<size_t>(j) * p.d, p.d, vj);
            const float pij = exp2f(warp_dot(qi, kj) * p.sl2 - m) * inv;
            const float ds = pij * (warp_dot(dyi, vj) - D);
#pragma unroll
            for (int u = 0; u < 4; ++u) acc[u] = fmaf(ds, kj[u], acc[u]);
        });
    }
    float* out = p.dq + base + static_cast<size_t>(i) * p.d;
#pragma unroll
    for (int u = 0; u < 4; ++u)
        if (lane + 32 * u < p.d) out[lane + 32 * u] = acc[u] * p.scale;
}

// dk_j, dv_j over the rows whose key set holds j.
template <typename Tin>
__global__ void __launch_bounds__(kBwdWarps * 32) bwd_dkv_kernel(const __grid_constant__ BwdParams p) {
    const size_t key = static_cast<size_t>(blockIdx.x) * kBwdWarps + (threadIdx.x >> 5);
    if (key >= static_cast<size_t>(p.B) * p.H * p.T) return;
    const int lane = threadIdx.x & 31;
    const int j = static_cast<int>(key % p.T), bh = static_cast<int>(key / p.T), b = bh / p.H, h = bh % p.H;
    const int dil = p.dil[h];
    const size_t base = static_cast<size_t>(bh) * p.T * p.d;
    const Tin* q = reinterpret_cast<const Tin*>(p.q) + base;
    const Tin* dy = reinterpret_cast<const Tin*>(p.dy) + base;
    float kj[4], vj[4], gk[4] = {0.f, 0.f, 0.f, 0.f}, gv[4] = {0.f, 0.f, 0.f, 0.f};
    load_row(reinterpret_cast<const Tin*>(p.k) + base + static_cast<size_t>(j) * p.d, p.d, kj);
    load_row(reinterpret_cast<const Tin*>(p.v) + base + static_cast<size_t>(j) * p.d, p.d, vj);
    const float* st = p.stats + static_cast<size_t>(bh) * p.T * 3;
    auto visit = [&](int i) {
        const float m = st[3 * i], l = st[3 * i + 1], D = st[3 * i + 2];
        if (!(l > 0.f)) return;
        float qi[4], dyi[4];
        load_row(q + static_cast<size_t>(i) * p.d, p.d, qi);
        load_row(dy + static_cast<size_t>(i) * p.d, p.d, dyi);
        const float pij = exp2f(warp_dot(qi, kj) * p.sl2 - m) / l;
        const float ds = pij * (warp_dot(dyi, vj) - D);
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            gv[u] = fmaf(pij, dyi[u], gv[u]);
            gk[u] = fmaf(ds, qi[u], gk[u]);
        }
    };
    if (!bwd_padded(p, b, j)) {
        if (bwd_is_global(p, b, j)) {
            for (int i = 0; i < p.T; ++i) visit(i);  // every row's key set holds a global key
        } else {
            // the rows whose window holds j (the window is symmetric), not global ...
            for (int t = -p.r; t <= p.r; ++t) {
                const long long i = static_cast<long long>(j) + static_cast<long long>(dil) * t;
                if (i >= 0 && i < p.T && !bwd_is_global(p, b, static_cast<int>(i))) visit(static_cast<int>(i));
            }
            // ... and every global row
            const int ngq = p.ws.n_gq[b];
            const int32_t* gq = p.ws.gq_list + static_cast<size_t>(b) * p.gstride;
            for (int a = 0; a < ngq; ++a) visit(gq[a]);
        }
    }
    float* odk = p.dk + base + static_cast<size_t>(j) * p.d;
    float* odv = p.dv + base + static_cast<size_t>(j) * p.d;
#pragma unroll
    for (int u = 0; u < 4; ++u)
        if (lane + 32 * u < p.d) {
            odk[lane + 32 * u] = gk[u] * p.scale;
            odv[lane + 32 * u] = gv[u];
        }
}

}  // namespace lf
