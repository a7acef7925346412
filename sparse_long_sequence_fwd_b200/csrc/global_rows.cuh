// global_rows.cuh -- K2: the rows of the global queries.
//
// A global query attends every non-padded key ("Longformer" note, section
// "Global Attention": N(i) = {1..T} for i in G).  The key axis of each (b, h)
// is split into chunks of kChunk keys, one CTA per (chunk, b*h).  Each CTA
// streams its chunk of K and V once from HBM (K rows in registers, V in
// shared memory) and, for every global query of sample b, forms the partial
// softmax state (m, l, acc[d]) of that chunk, combining the warps' partial
// maxima and sums with shuffles and shared memory.  Partial states go to the
// workspace; the last CTA of a (b, h) to finish (arrival ticket) merges the
// chunks with log-sum-exp rescaling and writes out[b, h, g, :].
// Scores use log2-domain scaling (scale * log2 e) and exp2.
#pragma once
#include "lf_common.cuh"
#include "ptx.cuh"

namespace lf {

constexpr int kGrThreads = kChunk;  // one key per thread

template <typename Tin>
__device__ __forceinline__ float load_as_float(const Tin* p);
template <>
__device__ __forceinline__ float load_as_float<float>(const float* p) { return *p; }
template <>
__device__ __forceinline__ float load_as_float<__nv_bfloat16>(const __nv_bfloat16* p) {
    return __bfloat162float(*p);
}

template <typename Tin>
__device__ __forceinline__ void store_from_float(Tin* p, float x);
template <>
__device__ __forceinline__ void store_from_float<float>(float* p, float x) { *p = x; }
template <>
__device__ __forceinline__ void store_from_float<__nv_bfloat16>(__nv_bfloat16* p, float x) {
    *p = __float2bfloat16_rn(x);
}

__device__ __forceinline__ float block_reduce_max(float v, float* red) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
    for (int o = 16; o; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    if (lane == 0) red[warp] = v;
    __syncthreads();
    float r = red[0];
#pragma unroll
    for (int w = 1; w < kGrThreads / 32; ++w) r = fmaxf(r, red[w]);
    __syncthreads();
    return r;
}
__device__ __forceinline__ float block_reduce_sum(float v, float* red) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
    for (int o = 16; o; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    if (lane == 0) red[warp] = v;
    __syncthreads();
    float r = 0.f;
#pragma unroll
    for (int w = 0; w < kGrThreads / 32; ++w) r += red[w];
    __syncthreads();
    return r;
}

// Merge of the per-chunk partial states of every global query of one (b, h)
// by the last CTA to arrive: M = max_c m_c, w_c = 2^(m_c - M),
// y = sum_c w_c acc_c / sum_c w_c l_c.  Every load is independent of the
// values loaded before it, so the partials stream in parallel.
template <typename Tout>
__device__ __forceinline__ void merge_partials(const GlobalRowParams& p, int bh, int nq, const int32_t* gq, int d) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int stride = d + 2;
    for (int a = warp; a < nq; a += kGrThreads / 32) {
        const float* src = p.ws.partial + (static_cast<size_t>(bh) * p.gstride + a) * p.nchunk * stride;
        float M = -INFINITY;
        for (int c = lane; c < p.nchunk; c += 32) M = fmaxf(M, __ldcg(src + static_cast<size_t>(c) * stride));
#pragma unroll
        for (int o = 16; o; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
        const float Mu = (M == -INFINITY) ? 0.f : M;  // every chunk empty: all weights 0
        float L = 0.f;
        for (int c = lane; c < p.nchunk; c += 32)
            L = fmaf(exp2f(__ldcg(src + static_cast<size_t>(c) * stride) - Mu),
                     __ldcg(src + static_cast<size_t>(c) * stride + 1), L);
#pragma unroll
        for (int o = 16; o; o >>= 1) L += __shfl_xor_sync(0xffffffffu, L, o);
        const float inv = L > 0.f ? 1.f / L : 0.f;
        Tout* orow = reinterpret_cast<Tout*>(p.out) + (static_cast<size_t>(bh) * p.T + gq[a]) * d;
        for (int col = lane; col < d; col += 32) {
            float acc0 = 0.f, acc1 = 0.f;
            int c = 0;
            for (; c + 1 < p.nchunk; c += 2) {
                const float* p0 = src + static_cast<size_t>(c) * stride;
                const float* p1 = p0 + stride;
                acc0 = fmaf(exp2f(__ldcg(p0) - Mu), __ldcg(p0 + 2 + col), acc0);
                acc1 = fmaf(exp2f(__ldcg(p1) - Mu), __ldcg(p1 + 2 + col), acc1);
            }
            if (c < p.nchunk) {
                const float* p0 = src + static_cast<size_t>(c) * stride;
                acc0 = fmaf(exp2f(__ldcg(p0) - Mu), __ldcg(p0 + 2 + col), acc0);
            }
            store_from_float(orow + col, (acc0 + acc1) * inv);
        }
    }
}

// DP: head dim rounded up to a multiple of 32 (32, 64 or 128).
template <typename Tin, int DP>
__global__ void __launch_bounds__(kGrThreads) global_rows_kernel(GlobalRowParams p) {
    extern __shared__ __align__(16) float gr_smem[];
    float* vs = gr_smem;                  // [kChunk][DP]
    float* qs = vs + kChunk * DP;         // [DP]
    float* ps = qs + DP;                  // [kChunk]
    float* red = ps + kChunk;             // [kGrThreads/32]
    float* accp = red + 32;               // [kGrThreads/DP][DP]
    __shared__ int is_last;

    const int tid = threadIdx.x;
    const int bh = blockIdx.y;
    const int b = bh / p.H;
    const int chunk = blockIdx.x;
    const int T = p.T, d = p.d;
    const int nq = p.ws.n_gq[b];
    if (nq == 0) return;

    const Tin* kb = reinterpret_cast<const Tin*>(p.k) + static_cast<size_t>(bh) * T * d;
    const Tin* vb = reinterpret_cast<const Tin*>(p.v) + static_cast<size_t>(bh) * T * d;
    const Tin* qb = reinterpret_cast<const Tin*>(p.q) + static_cast<size_t>(bh) * T * d;
    const int j = chunk * kChunk + tid;
    const bool valid = j < T && !(p.pad && p.pad[static_cast<size_t>(b) * T + j]);

    float kr[DP];
#pragma unroll
    for (int c = 0; c < DP; ++c) kr[c] = (valid && c < d) ? load_as_float(kb + static_cast<size_t>(j) * d + c) : 0.f;
    // V chunk into shared memory (coalesced), zero for invalid keys
    for (int idx = tid; idx < kChunk * DP; idx += kGrThreads) {
        int jj = idx / DP, c = idx - jj * DP;
        int jg = chunk * kChunk + jj;
        float x = 0.f;
        if (jg < T && c < d) x = load_as_float(vb + static_cast<size_t>(jg) * d + c);
        vs[idx] = x;
    }

    const int groups = kGrThreads / DP;  // key groups for the p*v sum
    const int col = tid % DP, grp = tid / DP;
    const int32_t* gq = p.ws.gq_list + static_cast<size_t>(b) * p.gstride;
    for (int a = 0; a < nq; ++a) {
        const int g = gq[a];
        __syncthreads();
        if (tid < DP) qs[tid] = tid < d ? load_as_float(qb + static_cast<size_t>(g) * d + tid) : 0.f;
        __syncthreads();
        float s = 0.f;
#pragma unroll
        for (int c = 0; c < DP; ++c) s = fmaf(qs[c], kr[c], s);
        s = valid ? s * p.sl2 : -INFINITY;
        const float m = block_reduce_max(s, red);
        const float m_use = (m == -INFINITY) ? 0.f : m;
        const float pj = valid ? exp2f(s - m_use) : 0.f;
        ps[tid] = pj;
        const float l = block_reduce_sum(pj, red);  // also orders the ps[] writes
        float acc = 0.f;
        const int per = kChunk / groups;
        for (int jj = grp * per; jj < (grp + 1) * per; ++jj) acc = fmaf(ps[jj], vs[jj * DP + col], acc);
        accp[grp * DP + col] = acc;
        __syncthreads();
        if (tid < DP) {
            float t = 0.f;
            for (int gi = 0; gi < groups; ++gi) t += accp[gi * DP + tid];
            float* dst = p.ws.partial + ((static_cast<size_t>(bh) * p.gstride + a) * p.nchunk + chunk) * (d + 2);
            if (tid < d) dst[2 + tid] = t;
            if (tid == 0) {
                dst[0] = m;
                dst[1] = l;
            }
        }
    }

    // arrival ticket: the last chunk of this (b, h) merges
    __threadfence();
    __syncthreads();
    if (tid == 0) {
        int ticket = atomicAdd(&p.ws.counters[bh], 1);
        is_last = (ticket == p.nchunk - 1);
    }
    __syncthreads();
    if (!is_last) return;
    __threadfence();
    merge_partials<Tin>(p, bh, nq, gq, d);
    if (tid == 0) p.ws.counters[bh] = 0;  // ready for the next call
}


// bf16, d = 64: the chunk of K and V is staged in shared memory with
// coalesced 16-byte loads (K rows padded to 144 bytes so that one thread per
// key reads its row without bank conflicts); one thread per key forms the
// scores, and the p*v sums run with 32 column pairs x 8 key groups.
constexpr int kKsStride = 72;  // bf16 elements per staged K row (64 + 8 pad)

__global__ void __launch_bounds__(kGrThreads) global_rows_bf16_kernel(const __grid_constant__ GlobalRowParams p) {
    extern __shared__ __align__(16) uint8_t grb_smem[];
    __nv_bfloat16* Ks = reinterpret_cast<__nv_bfloat16*>(grb_smem);             // [kChunk][72]
    __nv_bfloat16* Vs = Ks + kChunk * kKsStride;                                // [kChunk][64]
    float* qs = reinterpret_cast<float*>(Vs + kChunk * 64);                     // [64]
    float* ps = qs + 64;                                                         // [kChunk]
    float* red = ps + kChunk;                                                    // [32]
    float* accp = red + 32;                                                      // [8][64]
    __shared__ int is_last;

    const int tid = threadIdx.x;
    const int bh = blockIdx.y;
    const int b = bh / p.H;
    const int chunk = blockIdx.x;
    const int T = p.T;
    const int nq = p.ws.n_gq[b];
    if (nq == 0) return;
    const size_t base = static_cast<size_t>(bh) * T * 64;
    const uint4* k4 = reinterpret_cast<const uint4*>(reinterpret_cast<const __nv_bfloat16*>(p.k) + base);
    const uint4* v4 = reinterpret_cast<const uint4*>(reinterpret_cast<const __nv_bfloat16*>(p.v) + base);
    const int j0 = chunk * kChunk;
    // stage the chunk (8 x 16 B per key and tensor)
    uint4 kreg[8], vreg[8];
#pragma unroll
    for (int it = 0; it < 8; ++it) {
        const int u = it * kGrThreads + tid;  // 16-byte unit inside the chunk
        const int key = u >> 3;
        const bool in = j0 + key < T;
        kreg[it] = in ? __ldg(k4 + static_cast<size_t>(j0) * 8 + u) : make_uint4(0u, 0u, 0u, 0u);
        vreg[it] = in ? __ldg(v4 + static_cast<size_t>(j0) * 8 + u) : make_uint4(0u, 0u, 0u, 0u);
    }
#pragma unroll
    for (int it = 0; it < 8; ++it) {
        const int u = it * kGrThreads + tid;
        const int key = u >> 3, part = u & 7;
        *reinterpret_cast<uint4*>(Ks + key * kKsStride + part * 8) = kreg[it];
        *reinterpret_cast<uint4*>(Vs + key * 64 + part * 8) = vreg[it];
    }
    const int j = j0 + tid;
    const bool valid = j < T && !(p.pad && p.pad[static_cast<size_t>(b) * T + j]);
    const int cp = tid & 31, grp = tid >> 5;  // column pair, key group of 32
    const int32_t* gq = p.ws.gq_list + static_cast<size_t>(b) * p.gstride;
    const __nv_bfloat16* qb = reinterpret_cast<const __nv_bfloat16*>(p.q) + base;

    for (int a = 0; a < nq; ++a) {
        __syncthreads();  // staged chunk visible; previous query's buffers free
        if (tid < 64) qs[tid] = __bfloat162float(qb[static_cast<size_t>(gq[a]) * 64 + tid]);
        __syncthreads();
        float s0 = 0.f, s1 = 0.f, s2 = 0.f, s3 = 0.f;
        const uint4* krow = reinterpret_cast<const uint4*>(Ks + tid * kKsStride);
#pragma unroll
        for (int part = 0; part < 8; ++part) {
            const uint4 kv = krow[part];
            const __nv_bfloat162* k2 = reinterpret_cast<const __nv_bfloat162*>(&kv);
            const float2 f0 = __bfloat1622float2(k2[0]), f1 = __bfloat1622float2(k2[1]);
            const float2 f2 = __bfloat1622float2(k2[2]), f3 = __bfloat1622float2(k2[3]);
            const float* qq = qs + part * 8;
            s0 = fmaf(qq[0], f0.x, s0);
            s1 = fmaf(qq[1], f0.y, s1);
            s2 = fmaf(qq[2], f1.x, s2);
            s3 = fmaf(qq[3], f1.y, s3);
            s0 = fmaf(qq[4], f2.x, s0);
            s1 = fmaf(qq[5], f2.y, s1);
            s2 = fmaf(qq[6], f3.x, s2);
            s3 = fmaf(qq[7], f3.y, s3);
        }
        const float s = valid ? ((s0 + s1) + (s2 + s3)) * p.sl2 : -INFINITY;
        const float m = block_reduce_max(s, red);
        const float m_use = (m == -INFINITY) ? 0.f : m;
        const float pj = valid ? exp2f(s - m_use) : 0.f;
        ps[tid] = pj;
        const float l = block_reduce_sum(pj, red);  // its barriers also publish ps[]
        float ax = 0.f, ay = 0.f;
#pragma unroll 8
        for (int jj = grp * 32; jj < grp * 32 + 32; ++jj) {
            const float2 vv = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(Vs + jj * 64 + 2 * cp));
            ax = fmaf(ps[jj], vv.x, ax);
            ay = fmaf(ps[jj], vv.y, ay);
        }
        accp[grp * 64 + 2 * cp] = ax;
        accp[grp * 64 + 2 * cp + 1] = ay;
        __syncthreads();
        if (tid < 64) {
            float t = 0.f;
#pragma unroll
            for (int gi = 0; gi < 8; ++gi) t += accp[gi * 64 + tid];
            float* dst = p.ws.partial + ((static_cast<size_t>(bh) * p.gstride + a) * p.nchunk + chunk) * 66;
            dst[2 + tid] = t;
            if (tid == 0) {
                dst[0] = m;
                dst[1] = l;
            }
        }
    }

    __threadfence();
    __syncthreads();
    if (tid == 0) is_last = (atomicAdd(&p.ws.counters[bh], 1) == p.nchunk - 1);
    __syncthreads();
    if (!is_last) return;
    __threadfence();
    merge_partials<__nv_bfloat16>(p, bh, nq, gq, 64);
    if (tid == 0) p.ws.counters[bh] = 0;
}

constexpr int kGrBf16Smem = kChunk * kKsStride * 2 + kChunk * 64 * 2 + (64 + kChunk + 32 + 8 * 64) * 4;

}  // namespace lf
