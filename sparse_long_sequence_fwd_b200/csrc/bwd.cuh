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
//
// A warp takes its row's (or key's) partners 32 at a time, one per lane:
// each lane forms its dot products over the whole head dimension (the warp's
// own row staged in shared memory, the partner's row read with 16-byte
// loads, all 32 in flight together), then the lanes sum their contributions
// into the warp's row one output column per lane.
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

__device__ __forceinline__ bool bwd_is_global(const BwdParams& p, int b, int i) {
    return (p.ws.gbit[static_cast<size_t>(b) * p.W + (i >> 5)] >> (i & 31)) & 1u;
}
__device__ __forceinline__ bool bwd_padded(const BwdParams& p, int b, int j) {
    return p.pad && p.pad[static_cast<size_t>(b) * p.T + j] != 0;
}

// x (shared memory, d floats) . row (d elements of Tin), by one lane.
template <typename Tin>
__device__ __forceinline__ float dot_row(const float* x, const Tin* row, int d) {
    float s = 0.f;
    if ((d * static_cast<int>(sizeof(Tin))) % 16 == 0) {
        constexpr int kVec = 16 / sizeof(Tin);
        for (int c0 = 0; c0 < d; c0 += kVec) {
            const uint4 u = *reinterpret_cast<const uint4*>(row + c0);
            const Tin* e = reinterpret_cast<const Tin*>(&u);
#pragma unroll
            for (int t = 0; t < kVec; ++t) s = fmaf(x[c0 + t], load_as_float(e + t), s);
        }
    } else {
        for (int c = 0; c < d; ++c) s = fmaf(x[c], load_as_float(row + c), s);
    }
    return s;
}

// The e-th entry of row i's key list (e in [0, n)): the window positions
// first, then the global keys; -1 where the entry is not a key.
struct KeyList {
    int n, glob, dil, r;
    __device__ int key(const BwdParams& p, int b, int i, int e) const {
        if (glob) return bwd_padded(p, b, e) ? -1 : e;
        const int nw = 2 * r + 1;
        if (e < nw) {
            const long long j = static_cast<long long>(i) + static_cast<long long>(dil) * (e - r);
            return (j >= 0 && j < p.T && !bwd_padded(p, b, static_cast<int>(j))) ? static_cast<int>(j) : -1;
        }
        const int j = p.ws.gk_list[static_cast<size_t>(b) * p.gstride + (e - nw)], diff = j - i;
        const bool in_window = diff >= -dil * r && diff <= dil * r && diff % dil == 0;
        return in_window ? -1 : j;
    }
};
__device__ __forceinline__ KeyList key_list(const BwdParams& p, int b, int dil, int i) {
    KeyList kl;
    kl.glob = bwd_is_global(p, b, i) ? 1 : 0;
    kl.dil = dil;
    kl.r = p.r;
    kl.n = kl.glob ? p.T : 2 * p.r + 1 + p.ws.n_gk[b];
    return kl;
}

// The warp's row of a [B*H*T][d] tensor into shared memory as floats.
template <typename Tin>
__device__ __forceinline__ void stage_row(float* dst, const Tin* row, int d) {
    for (int c = threadIdx.x & 31; c < d; c += 32) dst[c] = load_as_float(row + c);
    __syncwarp();
}

// Row statistics: m_i (log2 domain), l_i and D_i = dy_i . y_i.
template <typename Tin>
__global__ void __launch_bounds__(kBwdWarps * 32) bwd_stats_kernel(const __grid_constant__ BwdParams p) {
    __shared__ float xs[kBwdWarps][128];
    const int wib = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const size_t row = static_cast<size_t>(blockIdx.x) * kBwdWarps + wib;
    if (row >= static_cast<size_t>(p.B) * p.H * p.T) return;
    const int i = static_cast<int>(row % p.T), bh = static_cast<int>(row / p.T), b = bh / p.H, h = bh % p.H;
    const int d = p.d;
    const size_t base = static_cast<size_t>(bh) * p.T * d;
    const Tin* k = reinterpret_cast<const Tin*>(p.k) + base;
    float D = 0.f;
    for (int c = lane; c < d; c += 32)
        D = fmaf(load_as_float(reinterpret_cast<const Tin*>(p.dy) + base + static_cast<size_t>(i) * d + c),
                 load_as_float(reinterpret_cast<const Tin*>(p.y) + base + static_cast<size_t>(i) * d + c), D);
#pragma unroll
    for (int o = 16; o; o >>= 1) D += __shfl_xor_sync(0xffffffffu, D, o);
    float* qs = xs[wib];
    stage_row(qs, reinterpret_cast<const Tin*>(p.q) + base + static_cast<size_t>(i) * d, d);
    const KeyList kl = key_list(p, b, p.dil[h], i);
    float m = -INFINITY, l = 0.f;  // the warp's running max and sum (the same in every lane)
    for (int e0 = 0; e0 < kl.n; e0 += 32) {
        const int j = e0 + lane < kl.n ? kl.key(p, b, i, e0 + lane) : -1;
        const float s = j >= 0 ? dot_row(qs, k + static_cast<size_t>(j) * d, d) * p.sl2 : -INFINITY;
        float cm = s;
#pragma unroll
        for (int o = 16; o; o >>= 1) cm = fmaxf(cm, __shfl_xor_sync(0xffffffffu, cm, o));
        if (cm == -INFINITY) continue;  // no key in these 32 entries
        const float mn = fmaxf(m, cm);
        float cs = j >= 0 ? exp2f(s - mn) : 0.f;
#pragma unroll
        for (int o = 16; o; o >>= 1) cs += __shfl_xor_sync(0xffffffffu, cs, o);
        l = l * exp2f(m - mn) + cs;  // (m = -inf: exp2f gives 0, l = 0 anyway)
        m = mn;
    }
    if (lane == 0) {
        p.stats[3 * row] = m;
        p.stats[3 * row + 1] = l;
        p.stats[3 * row + 2] = D;
    }
}

// dq_i = scale sum_j ds_ij k_j.
template <typename Tin>
__global__ void __launch_bounds__(kBwdWarps * 32) bwd_dq_kernel(const __grid_constant__ BwdParams p) {
    __shared__ float xs[kBwdWarps][2][128];
    const int wib = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const size_t row = static_cast<size_t>(blockIdx.x) * kBwdWarps + wib;
    if (row >= static_cast<size_t>(p.B) * p.H * p.T) return;
    const int i = static_cast<int>(row % p.T), bh = static_cast<int>(row / p.T), b = bh / p.H, h = bh % p.H;
    const int d = p.d;
    const size_t base = static_cast<size_t>(bh) * p.T * d;
    const Tin* k = reinterpret_cast<const Tin*>(p.k) + base;
    const Tin* v = reinterpret_cast<const Tin*>(p.v) + base;
    float* qs = xs[wib][0];
    float* dys = xs[wib][1];
    stage_row(qs, reinterpret_cast<const Tin*>(p.q) + base + static_cast<size_t>(i) * d, d);
    stage_row(dys, reinterpret_cast<const Tin*>(p.dy) + base + static_cast<size_t>(i) * d, d);
    const float m = p.stats[3 * row], l = p.stats[3 * row + 1], D = p.stats[3 * row + 2];
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
    if (l > 0.f) {
        const float inv = 1.f / l;
        const KeyList kl = key_list(p, b, p.dil[h], i);
        for (int e0 = 0; e0 < kl.n; e0 += 32) {
            const int j = e0 + lane < kl.n ? kl.key(p, b, i, e0 + lane) : -1;
            float ds = 0.f;
            if (j >= 0) {
                const float pij = exp2f(dot_row(qs, k + static_cast<size_t>(j) * d, d) * p.sl2 - m) * inv;
                ds = pij * (dot_row(dys, v + static_cast<size_t>(j) * d, d) - D);
            }
            // lane c sums column c over the 32 keys
            for (int t = 0; t < 32; ++t) {
                const float w = __shfl_sync(0xffffffffu, ds, t);
                const int jt = __shfl_sync(0xffffffffu, j, t);
                if (jt < 0) continue;
                const Tin* kr = k + static_cast<size_t>(jt) * d;
#pragma unroll
                for (int u = 0; u < 4; ++u)
                    if (lane + 32 * u < d) acc[u] = fmaf(w, load_as_float(kr + lane + 32 * u), acc[u]);
            }
        }
    }
    float* out = p.dq + base + static_cast<size_t>(i) * d;
#pragma unroll
    for (int u = 0; u < 4; ++u)
        if (lane + 32 * u < d) out[lane + 32 * u] = acc[u] * p.scale;
}

// dk_j, dv_j over the rows whose key set holds j.
template <typename Tin>
__global__ void __launch_bounds__(kBwdWarps * 32) bwd_dkv_kernel(const __grid_constant__ BwdParams p) {
    __shared__ float xs[kBwdWarps][2][128];
    const int wib = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const size_t key = static_cast<size_t>(blockIdx.x) * kBwdWarps + wib;
    if (key >= static_cast<size_t>(p.B) * p.H * p.T) return;
    const int j = static_cast<int>(key % p.T), bh = static_cast<int>(key / p.T), b = bh / p.H, h = bh % p.H;
    const int dil = p.dil[h], d = p.d;
    const size_t base = static_cast<size_t>(bh) * p.T * d;
    const Tin* q = reinterpret_cast<const Tin*>(p.q) + base;
    const Tin* dy = reinterpret_cast<const Tin*>(p.dy) + base;
    float* ks = xs[wib][0];
    float* vs = xs[wib][1];
    stage_row(ks, reinterpret_cast<const Tin*>(p.k) + base + static_cast<size_t>(j) * d, d);
    stage_row(vs, reinterpret_cast<const Tin*>(p.v) + base + static_cast<size_t>(j) * d, d);
    const float* st = p.stats + static_cast<size_t>(bh) * p.T * 3;
    float gk[4] = {0.f, 0.f, 0.f, 0.f}, gv[4] = {0.f, 0.f, 0.f, 0.f};
    if (!bwd_padded(p, b, j)) {
        // the rows: every row for a global key; else the window rows of j that are
        // not global (the window is symmetric), then every global row
        const bool gkey = bwd_is_global(p, b, j);
        const int nw = 2 * p.r + 1, ngq = p.ws.n_gq[b];
        const int n = gkey ? p.T : nw + ngq;
        const int32_t* gq = p.ws.gq_list + static_cast<size_t>(b) * p.gstride;
        for (int e0 = 0; e0 < n; e0 += 32) {
            const int e = e0 + lane;
            int i = -1;
            if (e < n) {
                if (gkey) {
                    i = e;
                } else if (e < nw) {
                    const long long x = static_cast<long long>(j) + static_cast<long long>(dil) * (e - p.r);
                    i = (x >= 0 && x < p.T && !bwd_is_global(p, b, static_cast<int>(x))) ? static_cast<int>(x) : -1;
                } else {
                    i = gq[e - nw];
                }
            }
            float pw = 0.f, ds = 0.f;
            if (i >= 0) {
                const float m = st[3 * i], l = st[3 * i + 1], D = st[3 * i + 2];
                if (l > 0.f) {
                    pw = exp2f(dot_row(ks, q + static_cast<size_t>(i) * d, d) * p.sl2 - m) / l;
                    ds = pw * (dot_row(vs, dy + static_cast<size_t>(i) * d, d) - D);
                } else {
                    i = -1;
                }
            }
            for (int t = 0; t < 32; ++t) {
                const int it = __shfl_sync(0xffffffffu, i, t);
                const float wp = __shfl_sync(0xffffffffu, pw, t), wd = __shfl_sync(0xffffffffu, ds, t);
                if (it < 0) continue;
                const Tin* qr = q + static_cast<size_t>(it) * d;
                const Tin* dr = dy + static_cast<size_t>(it) * d;
#pragma unroll
                for (int u = 0; u < 4; ++u)
                    if (lane + 32 * u < d) {
                        gv[u] = fmaf(wp, load_as_float(dr + lane + 32 * u), gv[u]);
                        gk[u] = fmaf(wd, load_as_float(qr + lane + 32 * u), gk[u]);
                    }
            }
        }
    }
    float* odk = p.dk + base + static_cast<size_t>(j) * d;
    float* odv = p.dv + base + static_cast<size_t>(j) * d;
#pragma unroll
    for (int u = 0; u < 4; ++u)
        if (lane + 32 * u < d) {
            odk[lane + 32 * u] = gk[u] * p.scale;
            odv[lane + 32 * u] = gv[u];
        }
}

}  // namespace lf
