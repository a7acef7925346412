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
template <>
__device__ __forceinline__ float load_as_float<__half>(const __half* p) {
    return __half2float(*p);
}

template <typename Tin>
__device__ __forceinline__ void store_from_float(Tin* p, float x);
template <>
__device__ __forceinline__ void store_from_float<float>(float* p, float x) { *p = x; }
template <>
__device__ __forceinline__ void store_from_float<__nv_bfloat16>(__nv_bfloat16* p, float x) {
    *p = __float2bfloat16_rn(x);
}
template <>
__device__ __forceinline__ void store_from_float<__half>(__half* p, float x) {
    *p = __float2half_rn(x);
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

// The kChunk rows [chunk * kChunk, +kChunk) of a 16-bit [T][DP] matrix into
// shared memory as fp32 (rows past T are zero): 16-byte loads, all of a
// thread's loads issued before any is used, so the copy costs one round trip
// to memory.  kSkew: element c of row jj goes to column (c + jj) mod DP.
template <typename Tin, int DP, bool kSkew>
__device__ __forceinline__ void stage_chunk16(float* dst, const Tin* src, int chunk, int T) {
    constexpr int kVec = 8;                                  // elements per 16-byte word
    constexpr int kRowWords = DP / kVec;
    constexpr int kPer = kChunk * kRowWords / kGrThreads;    // words per thread
    static_assert(kPer * kGrThreads == kChunk * kRowWords, "whole words per thread");
    const int tid = threadIdx.x;
    uint4 u[kPer];
#pragma unroll
    for (int it = 0; it < kPer; ++it) {
        const int w = tid + it * kGrThreads, jj = w / kRowWords, c0 = (w - jj * kRowWords) * kVec;
        const int jg = chunk * kChunk + jj;
        u[it] = jg < T ? *reinterpret_cast<const uint4*>(src + static_cast<size_t>(jg) * DP + c0)
                       : make_uint4(0u, 0u, 0u, 0u);
    }
#pragma unroll
    for (int it = 0; it < kPer; ++it) {
        const int w = tid + it * kGrThreads, jj = w / kRowWords, c0 = (w - jj * kRowWords) * kVec;
        const Tin* e = reinterpret_cast<const Tin*>(&u[it]);
#pragma unroll
        for (int t = 0; t < kVec; ++t) {
            const int c = c0 + t;
            dst[jj * DP + (kSkew ? ((c + jj) & (DP - 1)) : c)] = load_as_float(e + t);
        }
    }
}

// Rows mode: the partial state (M, L, acc) of each of the n_rows query rows
// over this call's keys, from the chunks' partial states (same weights as
// merge_partials, without the division).
__device__ __forceinline__ void merge_partials_rows(const GlobalRowParams& p, int bh, int nq, int d) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int stride = d + 2;
    for (int a = warp; a < nq; a += kGrThreads / 32) {
        const float* src = p.ws.partial + (static_cast<size_t>(bh) * p.gstride + a) * p.nchunk * stride;
        float M = -INFINITY;
        for (int c = lane; c < p.nchunk; c += 32) M = fmaxf(M, __ldcg(src + static_cast<size_t>(c) * stride));
#pragma unroll
        for (int o = 16; o; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
        const float Mu = (M == -INFINITY) ? 0.f : M;
        float L = 0.f;
        for (int c = lane; c < p.nchunk; c += 32)
            L = fmaf(exp2f(__ldcg(src + static_cast<size_t>(c) * stride) - Mu),
                     __ldcg(src + static_cast<size_t>(c) * stride + 1), L);
#pragma unroll
        for (int o = 16; o; o >>= 1) L += __shfl_xor_sync(0xffffffffu, L, o);
        const size_t row = static_cast<size_t>(bh) * p.n_rows + a;
        if (lane == 0) {
            p.out_ml[2 * row] = M;
            p.out_ml[2 * row + 1] = L;
        }
        for (int col = lane; col < d; col += 32) {
            float acc = 0.f;
            for (int c = 0; c < p.nchunk; ++c) {
                const float* pc = src + static_cast<size_t>(c) * stride;
                acc = fmaf(exp2f(__ldcg(pc) - Mu), __ldcg(pc + 2 + col), acc);
            }
            p.out_acc[row * d + col] = acc;
        }
    }
}

// DP: head dim rounded up to a multiple of 32 (32, 64 or 128).  kRows: rows
// mode (GlobalRowParams).
template <typename Tin, int DP, bool kRows = false>
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
    const int nq = kRows ? p.n_rows : p.ws.n_gq[b];
    if (nq == 0) return;

    const Tin* kb = reinterpret_cast<const Tin*>(p.k) + static_cast<size_t>(bh) * T * d;
    const Tin* vb = reinterpret_cast<const Tin*>(p.v) + static_cast<size_t>(bh) * T * d;
    const Tin* qb = reinterpret_cast<const Tin*>(p.q) + static_cast<size_t>(bh) * T * d;
    const int j = chunk * kChunk + tid;
    const bool valid = j < T && !(p.pad && p.pad[static_cast<size_t>(b) * T + j]);

    // the chunk's K rows, read coalesced into shared memory first (the V area;
    // element c of row jj at column (c + jj) mod DP, so the row reads below
    // hit 32 different banks), then each thread's row into registers
    if constexpr (sizeof(Tin) == 2) {
        stage_chunk16<Tin, DP, true>(vs, kb, chunk, T);  // (16-bit inputs: d == DP)
    } else {
        for (int idx = tid; idx < kChunk * DP; idx += kGrThreads) {
            const int jj = idx / DP, c = idx - jj * DP;
            const int jg = chunk * kChunk + jj;
            vs[jj * DP + ((c + jj) & (DP - 1))] =
                (jg < T && c < d) ? load_as_float(kb + static_cast<size_t>(jg) * d + c) : 0.f;
        }
    }
    __syncthreads();
    float kr[DP];
#pragma unroll
    for (int c = 0; c < DP; ++c) kr[c] = valid ? vs[tid * DP + ((c + tid) & (DP - 1))] : 0.f;
    __syncthreads();
    // V chunk into shared memory (coalesced), zero for invalid keys
    if constexpr (sizeof(Tin) == 2) {
        stage_chunk16<Tin, DP, false>(vs, vb, chunk, T);
    } else {
        for (int idx = tid; idx < kChunk * DP; idx += kGrThreads) {
            int jj = idx / DP, c = idx - jj * DP;
            int jg = chunk * kChunk + jj;
            float x = 0.f;
            if (jg < T && c < d) x = load_as_float(vb + static_cast<size_t>(jg) * d + c);
            vs[idx] = x;
        }
    }

    const int groups = kGrThreads / DP;  // key groups for the p*v sum
    const int col = tid % DP, grp = tid / DP;
    const int32_t* gq = p.ws.gq_list + static_cast<size_t>(b) * p.gstride;
    for (int a = 0; a < nq; ++a) {
        const Tin* qrow = kRows ? reinterpret_cast<const Tin*>(p.q_rows) + (static_cast<size_t>(bh) * p.n_rows + a) * d
                                : qb + static_cast<size_t>(gq[a]) * d;
        __syncthreads();
        if (tid < DP) qs[tid] = tid < d ? load_as_float(qrow + tid) : 0.f;
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
    if constexpr (kRows)
        merge_partials_rows(p, bh, nq, d);
    else
        merge_partials<Tin>(p, bh, nq, gq, d);
    if (tid == 0) p.ws.counters[bh] = 0;  // ready for the next call
}

// Sequence-sharded forward: the partial states of a row from every key
// shard combine as M = max_p M_p, w_p = 2^(M_p - M),
// y = sum_p w_p acc_p / sum_p w_p L_p (as merge_partials does for chunks).
// One CTA per (row a, b*h), one thread per output column.
template <typename Tout>
__global__ void __launch_bounds__(128) merge_rows_kernel(const __grid_constant__ MergeRowsParams p) {
    const int a = blockIdx.x, bh = blockIdx.y, b = bh / p.H, col = threadIdx.x;
    const int pos = p.pos[static_cast<size_t>(b) * p.n_rows + a];
    if (pos < 0 || col >= p.d) return;
    const size_t row = static_cast<size_t>(bh) * p.n_rows + a, per_part = static_cast<size_t>(p.BH) * p.n_rows;
    float M = -INFINITY;
    for (int q = 0; q < p.n_parts; ++q) M = fmaxf(M, p.ml[2 * (q * per_part + row)]);
    const float Mu = M == -INFINITY ? 0.f : M;
    float L = 0.f, acc = 0.f;
    for (int q = 0; q < p.n_parts; ++q) {
        const float w = exp2f(p.ml[2 * (q * per_part + row)] - Mu);
        L = fmaf(w, p.ml[2 * (q * per_part + row) + 1], L);
        acc = fmaf(w, p.acc[(q * per_part + row) * p.d + col], acc);
    }
    store_from_float(reinterpret_cast<Tout*>(p.out) + (static_cast<size_t>(bh) * p.T_out + pos) * p.d + col,
                     L > 0.f ? acc / L : 0.f);
}


// bf16, d = 64: tensor-core global rows.  CTA (split, b*h, row group) takes
// up to KPW / 2 global queries of sample b and cpc consecutive 128-key
// chunks of the key axis.  Its 4 warps form an RG x KP grid: RG row tiles of
// 16 queries (one m16n8k16 row tile each) times KP key slices of KPW keys,
// warp (rg, kp) taking keys [kp KPW, (kp + 1) KPW) of every chunk for the
// queries of row tile rg.  With few global queries the warps split the keys
// instead of idling, so all four SM sub-partitions run the warp-level MMA.
// The chunks of K and V stream through a two-stage ring in padded shared
// memory (cp.async, zero-filled past T); the first two are requested before
// anything that depends on the prep kernel (the global-query count and the
// query rows, which prep packs in list order), so the HBM latency overlaps
// those reads.  Every warp forms S = Q K^T (16 x KPW, fp32 in registers),
// applies the key padding mask, runs the online softmax (log2 domain, exp2)
// and accumulates O += P V with P re-packed from the S registers as bf16 A
// fragments and V fragments from ldmatrix.trans.  At the end the KP slices of
// a row tile combine their states (m, l, O) through shared memory in slice
// order, and the result goes to the workspace as this split's partial state;
// global_rows_merge_kernel combines the splits.  Every K/V row of a (b, h) is
// read once per row group; the warp-level MMA (a quarter of the tcgen05
// rate) keeps up with that as long as every sub-partition issues it.
constexpr int kGrKeys = 128;       // keys per chunk
constexpr int kGrWarps = 4;        // row tiles x key slices
constexpr int kGrXchFloats = 36;   // per lane when slices combine: m_a, m_b, l_a, l_b, O[8][4]
// Keys per warp slice of a chunk for a global-query capacity: every warp
// gets work whatever the count (16 queries or fewer: 4 slices of 32 keys;
// 32 or fewer: 2 row tiles x 2 slices of 64; more: 4 row tiles x 128 keys).
// A CTA then holds KPW / 2 global-query slots.  (The host takes 128, no
// slices, when every CTA has a single chunk: the combine would cost more
// than the slices save.)
__host__ __device__ constexpr int gr_kpw(int gstride) { return gstride <= 16 ? 32 : (gstride <= 32 ? 64 : 128); }
constexpr int kGrStride = 72;      // bf16 per staged row: 64 + 8 (conflict-free fragments and ldmatrix)
constexpr int kGrStages = 2;
constexpr int kGrChunkElems = kGrKeys * kGrStride;          // bf16 per K (or V) chunk
constexpr int kGrSmem = kGrStages * 2 * kGrChunkElems * 2;  // bytes of the ring
constexpr int kMaxSplits = 64;                              // key splits per (b, h): the merge holds them in registers
static_assert(kGrWarps * kGrXchFloats * 32 * 4 <= kGrSmem, "slice states fit in the ring");

// D += A B, m16n8k16, fp32 accumulators; A and B bf16 (kHalf: f16).
template <bool kHalf>
__device__ __forceinline__ void mma_16816(float* d, const uint32_t* a, uint32_t b0, uint32_t b1) {
    if constexpr (kHalf)
        asm volatile(
            "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
            "{%0, %1, %2, %3};"
            : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
            : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
    else
        asm volatile(
            "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
            "{%0, %1, %2, %3};"
            : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
            : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
__device__ __forceinline__ void ldmatrix_x4_trans(uint32_t* r, const void* smem_row) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(smem_u32(smem_row)));
}
// 16-byte global -> shared copy; src_bytes = 0 fills zeros
__device__ __forceinline__ void cp_async16(void* dst, const void* src, uint32_t src_bytes) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem_u32(dst)), "l"(src), "r"(src_bytes)
                 : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
// wait until at most N committed groups of this thread are still in flight
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

template <int KPW, bool kHalf>
__global__ void __launch_bounds__(kGrWarps * 32, 3) global_rows_mma_kernel(const __grid_constant__ GlobalRowParams p) {
    constexpr int KP = kGrKeys / KPW;    // key slices of a chunk
    constexpr int RG = kGrWarps / KP;    // row tiles of 16 queries
    constexpr int ROWS = 16 * RG;        // global-query slots per CTA
    constexpr int NT = KPW / 8;          // 8-key tiles of a slice (S columns)
    constexpr int KK = KPW / 16;         // 16-key steps of a slice (P V)
    static_assert(KP * RG == kGrWarps, "the warps cover row tiles x slices");
    extern __shared__ __align__(16) __nv_bfloat16 gr_ring[];  // [stage][K, V][kGrKeys][kGrStride]
    __shared__ uint32_t valid_bits[kGrStages][kGrKeys / 32];

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int g8 = lane >> 2, t4 = lane & 3;  // fragment row group and column pair
    const int rg = warp % RG, kp = warp / RG;
    const int k0 = kp * KPW;                  // this warp's first key in every chunk
    const int split = blockIdx.x, bh = blockIdx.y, b = bh / p.H;
    const int T = p.T;
    const size_t base = static_cast<size_t>(bh) * T * 64;
    const __nv_bfloat16* kb = reinterpret_cast<const __nv_bfloat16*>(p.k) + base;
    const __nv_bfloat16* vb = reinterpret_cast<const __nv_bfloat16*>(p.v) + base;
    const int nblk = (T + kGrKeys - 1) / kGrKeys;
    const int c_lo = split * p.cpc, c_hi = min(nblk, c_lo + p.cpc);

    // one commit group per chunk: its K and V into ring stage st
    auto issue = [&](int ch, int st) {
        const int j0 = ch * kGrKeys;
        __nv_bfloat16* Ks = gr_ring + st * 2 * kGrChunkElems;
        __nv_bfloat16* Vs = Ks + kGrChunkElems;
        for (int u = tid; u < kGrKeys * 8; u += kGrWarps * 32) {
            const int key = u >> 3, part = u & 7;
            const bool in = j0 + key < T;
            const size_t src = static_cast<size_t>(in ? j0 + key : 0) * 64 + part * 8;
            cp_async16(Ks + key * kGrStride + part * 8, kb + src, in ? 16u : 0u);
            cp_async16(Vs + key * kGrStride + part * 8, vb + src, in ? 16u : 0u);
        }
    };
    issue(c_lo, 0);
    cp_async_commit();
    if (c_lo + 1 < c_hi) issue(c_lo + 1, 1);
    cp_async_commit();

    // Q fragments of rows row0 + g8 and row0 + g8 + 8 from the packed global
    // queries (prep's output: zero past the sample's count, so no count or list
    // is needed first), loaded alongside the count
    const int row0 = blockIdx.z * ROWS + rg * 16;  // this warp's first global-row slot
    uint32_t qa[4][4];
    {
        const __nv_bfloat16* qgb = p.ws.qg + static_cast<size_t>(bh) * p.ngp * 64;
        const int ra = row0 + g8, rb = row0 + g8 + 8;
        const __nv_bfloat16* qra = ra < p.ngp ? qgb + static_cast<size_t>(ra) * 64 : nullptr;
        const __nv_bfloat16* qrb = rb < p.ngp ? qgb + static_cast<size_t>(rb) * 64 : nullptr;
#pragma unroll
        for (int ks = 0; ks < 4; ++ks) {
            const int c0 = 16 * ks + 2 * t4;
            qa[ks][0] = qra ? *reinterpret_cast<const uint32_t*>(qra + c0) : 0u;
            qa[ks][1] = qrb ? *reinterpret_cast<const uint32_t*>(qrb + c0) : 0u;
            qa[ks][2] = qra ? *reinterpret_cast<const uint32_t*>(qra + c0 + 8) : 0u;
            qa[ks][3] = qrb ? *reinterpret_cast<const uint32_t*>(qrb + c0 + 8) : 0u;
        }
    }
    const int nq = p.ws.n_gq[b];
    if (blockIdx.z * ROWS >= nq) {
        cp_async_wait<0>();  // no copy may still target this CTA's shared memory
        return;
    }
    const bool active = row0 < nq;
    float o[8][4];
#pragma unroll
    for (int nd = 0; nd < 8; ++nd) o[nd][0] = o[nd][1] = o[nd][2] = o[nd][3] = 0.f;
    float m_a = -INFINITY, m_b = -INFINITY, l_a = 0.f, l_b = 0.f;  // rows g8, g8 + 8
    const float sl2 = p.sl2;

    for (int ch = c_lo; ch < c_hi; ++ch) {
        // the merge kernel may launch once every CTA is on its last chunk (it
        // waits for this whole grid before reading): its launch overlaps that
        // chunk without its CTAs sitting resident through the earlier ones
        if (ch == c_hi - 1) grid_dep_launch();
        const int st = (ch - c_lo) & 1;
        const __nv_bfloat16* Ks = gr_ring + st * 2 * kGrChunkElems;
        const __nv_bfloat16* Vs = Ks + kGrChunkElems;
        if (tid < kGrKeys) {  // valid keys of this chunk (inside T, not padded)
            const int j = ch * kGrKeys + tid;
            const bool ok = j < T && !(p.pad && p.pad[static_cast<size_t>(b) * T + j]);
            const uint32_t w = __ballot_sync(0xffffffffu, ok);
            if (lane == 0) valid_bits[st][tid >> 5] = w;
        }
        cp_async_wait<1>();  // this chunk has landed (the next one may still be in flight)
        __syncthreads();
        if (active) {
            // S = Q K^T over this warp's slice: NT key tiles of 8
            float s[NT][4];
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
                s[nt][0] = s[nt][1] = s[nt][2] = s[nt][3] = 0.f;
                const __nv_bfloat16* kr = Ks + (k0 + 8 * nt + g8) * kGrStride + 2 * t4;
#pragma unroll
                for (int ks = 0; ks < 4; ++ks) {
                    const uint32_t b0 = *reinterpret_cast<const uint32_t*>(kr + 16 * ks);
                    const uint32_t b1 = *reinterpret_cast<const uint32_t*>(kr + 16 * ks + 8);
                    mma_16816<kHalf>(s[nt], qa[ks], b0, b1);
                }
            }
            // mask, scale, row maxima (each row's scores live in the 4 lanes of its quad)
            float mx_a = -INFINITY, mx_b = -INFINITY;
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
                const int key = k0 + 8 * nt;  // first key of the tile; this lane has key + 2 t4, + 1
                const uint32_t vw = valid_bits[st][key >> 5] >> ((key & 31) + 2 * t4);
                const bool v0 = vw & 1u, v1 = (vw >> 1) & 1u;
                s[nt][0] = v0 ? s[nt][0] * sl2 : -INFINITY;
                s[nt][1] = v1 ? s[nt][1] * sl2 : -INFINITY;
                s[nt][2] = v0 ? s[nt][2] * sl2 : -INFINITY;
                s[nt][3] = v1 ? s[nt][3] * sl2 : -INFINITY;
                mx_a = fmaxf(mx_a, fmaxf(s[nt][0], s[nt][1]));
                mx_b = fmaxf(mx_b, fmaxf(s[nt][2], s[nt][3]));
            }
#pragma unroll
            for (int off = 1; off <= 2; off <<= 1) {
                mx_a = fmaxf(mx_a, __shfl_xor_sync(0xffffffffu, mx_a, off));
                mx_b = fmaxf(mx_b, __shfl_xor_sync(0xffffffffu, mx_b, off));
            }
            const float mn_a = fmaxf(m_a, mx_a), mn_b = fmaxf(m_b, mx_b);
            const float al_a = m_a == -INFINITY ? 0.f : exp2f(m_a - mn_a);
            const float al_b = m_b == -INFINITY ? 0.f : exp2f(m_b - mn_b);
            m_a = mn_a;
            m_b = mn_b;
            const float bs_a = mn_a == -INFINITY ? 0.f : mn_a, bs_b = mn_b == -INFINITY ? 0.f : mn_b;
            l_a *= al_a;
            l_b *= al_b;
#pragma unroll
            for (int nd = 0; nd < 8; ++nd) {
                o[nd][0] *= al_a;
                o[nd][1] *= al_a;
                o[nd][2] *= al_b;
                o[nd][3] *= al_b;
            }
            // P (bf16 A fragments) and row sums
            uint32_t pa[KK][4];
#pragma unroll
            for (int kk = 0; kk < KK; ++kk) {
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    float* sv = s[2 * kk + h];
                    const float e0 = exp2f(sv[0] - bs_a), e1 = exp2f(sv[1] - bs_a);
                    const float e2 = exp2f(sv[2] - bs_b), e3 = exp2f(sv[3] - bs_b);
                    l_a += e0 + e1;
                    l_b += e2 + e3;
                    pa[kk][2 * h] = pack16x2<kHalf>(e0, e1);
                    pa[kk][2 * h + 1] = pack16x2<kHalf>(e2, e3);
                }
            }
            // O += P V: for each 16-key step, two 8-column tiles of V per ldmatrix
#pragma unroll
            for (int kk = 0; kk < KK; ++kk) {
                const uint32_t a4[4] = {pa[kk][0], pa[kk][1], pa[kk][2], pa[kk][3]};
#pragma unroll
                for (int nd = 0; nd < 8; nd += 2) {
                    uint32_t vf[4];
                    ldmatrix_x4_trans(vf, Vs + (k0 + 16 * kk + (lane & 7) + 8 * ((lane >> 3) & 1)) * kGrStride +
                                              8 * (nd + (lane >> 4)));
                    mma_16816<kHalf>(o[nd], a4, vf[0], vf[1]);
                    mma_16816<kHalf>(o[nd + 1], a4, vf[2], vf[3]);
                }
            }
        }
        __syncthreads();  // this stage is consumed: the chunk two ahead may overwrite it
        if (ch + 2 < c_hi) issue(ch + 2, st);
        cp_async_commit();  // (empty past the last chunk, so every wait above counts the same)
    }
    cp_async_wait<0>();
    // full row sums over the quad
#pragma unroll
    for (int off = 1; off <= 2; off <<= 1) {
        l_a += __shfl_xor_sync(0xffffffffu, l_a, off);
        l_b += __shfl_xor_sync(0xffffffffu, l_b, off);
    }
    if (KP > 1) {
        // the slices' states through shared memory (the ring is free: every copy
        // has landed and been consumed), then the first slice of each row tile
        // combines them in slice order: M = max m_k, w_k = 2^(m_k - M),
        // L = sum w_k l_k, O = sum w_k O_k
        __syncthreads();
        float* xs = reinterpret_cast<float*>(gr_ring);  // [warp][kGrXchFloats][32 lanes]
        {
            float* mine = xs + warp * kGrXchFloats * 32 + lane;
            mine[0] = m_a;
            mine[32] = m_b;
            mine[64] = l_a;
            mine[96] = l_b;
#pragma unroll
            for (int nd = 0; nd < 8; ++nd)
#pragma unroll
                for (int j = 0; j < 4; ++j) mine[(4 + 4 * nd + j) * 32] = o[nd][j];
        }
        __syncthreads();
        if (kp != 0 || !active) return;
        float Ma = -INFINITY, Mb = -INFINITY;
#pragma unroll
        for (int q = 0; q < KP; ++q) {
            const float* src = xs + (q * RG + rg) * kGrXchFloats * 32 + lane;
            Ma = fmaxf(Ma, src[0]);
            Mb = fmaxf(Mb, src[32]);
        }
        const float Mua = Ma == -INFINITY ? 0.f : Ma, Mub = Mb == -INFINITY ? 0.f : Mb;
        l_a = l_b = 0.f;
#pragma unroll
        for (int nd = 0; nd < 8; ++nd) o[nd][0] = o[nd][1] = o[nd][2] = o[nd][3] = 0.f;
#pragma unroll
        for (int q = 0; q < KP; ++q) {
            const float* src = xs + (q * RG + rg) * kGrXchFloats * 32 + lane;
            const float wa = src[0] == -INFINITY ? 0.f : ex2_approx(src[0] - Mua);
            const float wb = src[32] == -INFINITY ? 0.f : ex2_approx(src[32] - Mub);
            l_a = fmaf(wa, src[64], l_a);
            l_b = fmaf(wb, src[96], l_b);
#pragma unroll
            for (int nd = 0; nd < 8; ++nd) {
                o[nd][0] = fmaf(wa, src[(4 + 4 * nd) * 32], o[nd][0]);
                o[nd][1] = fmaf(wa, src[(5 + 4 * nd) * 32], o[nd][1]);
                o[nd][2] = fmaf(wb, src[(6 + 4 * nd) * 32], o[nd][2]);
                o[nd][3] = fmaf(wb, src[(7 + 4 * nd) * 32], o[nd][3]);
            }
        }
        m_a = Ma;
        m_b = Mb;
    } else if (!active) {
        return;
    }
    // the partial state of each row of this split
    const int nsplit = p.nchunk;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        const int row = row0 + g8 + 8 * h;
        if (row >= nq) continue;
        float* dst = p.ws.partial + ((static_cast<size_t>(bh) * p.gstride + row) * nsplit + split) * 66;
        if (t4 == 0) {
            dst[0] = h ? m_b : m_a;
            dst[1] = h ? l_b : l_a;
        }
#pragma unroll
        for (int nd = 0; nd < 8; ++nd) {
            const int col = 8 * nd + 2 * t4;
            dst[2 + col] = o[nd][2 * h];
            dst[3 + col] = o[nd][2 * h + 1];
        }
    }
}

// One CTA per (global-row slot, b*h), one thread per output column: the
// splits' partial states combine as M = max_c m_c, w_c = 2^(m_c - M),
// y = sum_c w_c acc_c / sum_c w_c l_c.  Launched as the split kernel's
// programmatic dependent: the split kernel lets it launch once every split
// CTA is on its last chunk, so only griddepcontrol.wait separates the two.  All
// its loads are issued before any value is used (one round trip to L2).
template <bool kHalf>
__global__ void __launch_bounds__(64) global_rows_merge_kernel(const __grid_constant__ GlobalRowParams p) {
    __shared__ float wsh[kMaxSplits];
    __shared__ float red[2];
    grid_dep_wait();  // the split kernel's partial states are complete and visible
    const int a = blockIdx.x, bh = blockIdx.y, b = bh / p.H;
    if (a >= p.ws.n_gq[b]) return;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int nsplit = p.nchunk;
    const float* src = p.ws.partial + (static_cast<size_t>(bh) * p.gstride + a) * nsplit * 66;
    const int32_t g = p.ws.gq_list[static_cast<size_t>(b) * p.gstride + a];

    // every load first, so the whole merge costs one round trip to L2: split
    // c's (m, l) in thread c (nsplit <= 64), and column tid of every split
    const float mc = tid < nsplit ? __ldcg(src + static_cast<size_t>(tid) * 66) : -INFINITY;
    const float lc = tid < nsplit ? __ldcg(src + static_cast<size_t>(tid) * 66 + 1) : 0.f;
    float v[kMaxSplits];
    const float* col = src + 2 + tid;
#pragma unroll
    for (int c = 0; c < kMaxSplits; ++c) v[c] = c < nsplit ? __ldcg(col + static_cast<size_t>(c) * 66) : 0.f;
    float M = mc;
#pragma unroll
    for (int o = 16; o; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
    if (lane == 0) red[warp] = M;
    __syncthreads();
    M = fmaxf(red[0], red[1]);
    const float Mu = M == -INFINITY ? 0.f : M;  // every split empty: all weights 0
    const float wc = exp2f(mc - Mu);            // m = -inf gives 0
    if (tid < nsplit) wsh[tid] = wc;
    float L = wc * lc;
#pragma unroll
    for (int o = 16; o; o >>= 1) L += __shfl_xor_sync(0xffffffffu, L, o);
    __syncthreads();
    if (lane == 0) red[warp] = L;
    __syncthreads();
    L = red[0] + red[1];

    // the weighted sum of the splits' columns
    float acc0 = 0.f, acc1 = 0.f;
#pragma unroll
    for (int c = 0; c < kMaxSplits; c += 2) {
        if (c < nsplit) acc0 = fmaf(wsh[c], v[c], acc0);
        if (c + 1 < nsplit) acc1 = fmaf(wsh[c + 1], v[c + 1], acc1);
    }
    const float y = L > 0.f ? (acc0 + acc1) / L : 0.f;
    if constexpr (kHalf)
        reinterpret_cast<__half*>(p.out)[(static_cast<size_t>(bh) * p.T + g) * 64 + tid] = __float2half_rn(y);
    else
        reinterpret_cast<__nv_bfloat16*>(p.out)[(static_cast<size_t>(bh) * p.T + g) * 64 + tid] = __float2bfloat16_rn(y);
}

}  // namespace lf
