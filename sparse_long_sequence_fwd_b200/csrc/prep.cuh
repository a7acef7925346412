// prep.cuh -- K0: global-token and padding preparation.
//
// One CTA per (b, h).  From global_idx[b, :] it builds the set G_b (in-range
// entries, duplicates collapsed) as a bitmap in shared memory, then the
// sorted lists
//   gq_list[b] = G_b                       (global queries: full rows)
//   gk_list[b] = G_b minus padded keys     (global keys: extra columns)
// and the global-query bitmap gbit[b].  Set semantics follow the "Longformer"
// note, section "Global Attention" (N(i) = N_local(i) U G); a padded position
// is removed as a key ("Implementation Reading": padding must be masked) but
// is still a global query.  Entries outside [0, T) are ignored and raise the
// status bit.  It also zeroes the arrival counters the global-row kernel
// uses for its (b, h), and (all CTAs together) the band kernel's merge
// tickets.  On the bf16 path every CTA also packs the rows of k and v
// named by gk_list into contiguous [ngp][64] blocks for its (b, h), zero
// beyond the list, so the band kernel can stage them with one TMA box, and
// the rows of q named by gq_list the same way, so the global-row kernel
// reads its queries without first reading the list.
#pragma once
#include "lf_common.cuh"
#include "ptx.cuh"

namespace lf {

constexpr int kPrepThreads = 256;

// Exclusive prefix sum of v over the CTA (warp shuffles, then the warps'
// totals); sbuf holds at least kPrepThreads / 32 ints.
__device__ __forceinline__ int block_exclusive_scan(int v, int* sbuf) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    int x = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
    }
    if (lane == 31) sbuf[warp] = x;
    __syncthreads();
    if (warp == 0) {
        int t = lane < kPrepThreads / 32 ? sbuf[lane] : 0;
#pragma unroll
        for (int o = 1; o < kPrepThreads / 32; o <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, t, o);
            if (lane >= o) t += y;
        }
        if (lane < kPrepThreads / 32) sbuf[lane] = t;
    }
    __syncthreads();
    return (warp ? sbuf[warp - 1] : 0) + x - v;
}

// Padding bits of the 32 keys of word w (independent byte loads, no chain of
// dependent ones: the whole word costs one round trip).
__device__ __forceinline__ uint32_t pad_word(const uint8_t* pad_b, int w, int T) {
    uint32_t m = 0u;
#pragma unroll
    for (int k = 0; k < 32; ++k) {
        const int j = (w << 5) + k;
        m |= (j < T && pad_b[j] != 0) ? (1u << k) : 0u;
    }
    return m;
}

__global__ void __launch_bounds__(kPrepThreads) prep_kernel(PrepParams p) {
    extern __shared__ __align__(16) uint32_t prep_smem[];
    uint32_t* bits = prep_smem;                                      // [W]
    int* scan_q = reinterpret_cast<int*>(bits + p.W);                // [256]
    int* scan_k = scan_q + kPrepThreads;                             // [256]
    int* gk_s = scan_k + kPrepThreads;                               // [gstride]
    int* gq_s = gk_s + p.gstride;                                    // [gstride]
    __shared__ int n_k_total, n_q_total;

    grid_dep_launch();  // the band kernel may set itself up meanwhile; it waits for this grid before reading
    const int tid = threadIdx.x;
    const int b = blockIdx.x / p.H;
    const int h = blockIdx.x - b * p.H;
    const int T = p.T;
    const uint8_t* pad_b = p.pad ? p.pad + static_cast<size_t>(b) * T : nullptr;

    for (int w = tid; w < p.W; w += kPrepThreads) bits[w] = 0u;
    if (tid == 0) p.ws.counters[blockIdx.x] = 0;  // arrival tickets of the global-row kernel
    for (int a = blockIdx.x * kPrepThreads + tid; a < p.n_band_cnt; a += gridDim.x * kPrepThreads)
        p.band_cnt[a] = 0;  // the band kernel's merge tickets (its mergers also reset what they use)
    __syncthreads();
    for (int a = tid; a < p.n_global; a += kPrepThreads) {
        int g = p.gidx[static_cast<size_t>(b) * p.n_global + a];
        if (g < 0 || g >= T) {
            if (h == 0) atomicOr(p.status, kStatusBadGlobal);
        } else {
            atomicOr(&bits[g >> 5], 1u << (g & 31));
        }
    }
    __syncthreads();

    // contiguous word range per thread
    const int per = (p.W + kPrepThreads - 1) / kPrepThreads;
    const int w0 = min(p.W, tid * per), w1 = min(p.W, w0 + per);
    int cq = 0, ck = 0;
    // padding words of this thread's words that hold global tokens, kept for the
    // second pass (each costs 32 byte loads); two cover T <= 16384
    int pw_w[2] = {-1, -1};
    uint32_t pw_v[2] = {0u, 0u};
    for (int w = w0; w < w1; ++w) {
        uint32_t qb = bits[w];
        cq += __popc(qb);
        uint32_t pw = 0u;
        if (pad_b && qb) {
            pw = pad_word(pad_b, w, T);
            if (pw_w[0] < 0) {
                pw_w[0] = w;
                pw_v[0] = pw;
            } else if (pw_w[1] < 0) {
                pw_w[1] = w;
                pw_v[1] = pw;
            }
        }
        ck += __popc(qb & ~pw);
    }
    int oq = block_exclusive_scan(cq, scan_q);
    int ok = block_exclusive_scan(ck, scan_k);
    if (tid == kPrepThreads - 1) {
        n_k_total = ok + ck;
        n_q_total = oq + cq;
    }
    const bool writer = (h == 0);
    int32_t* gq_out = p.ws.gq_list + static_cast<size_t>(b) * p.gstride;
    int32_t* gk_out = p.ws.gk_list + static_cast<size_t>(b) * p.gstride;
    for (int w = w0; w < w1; ++w) {
        uint32_t qb = bits[w];
        if (writer) p.ws.gbit[static_cast<size_t>(b) * p.W + w] = qb;
        const uint32_t pw = !(pad_b && qb) ? 0u
                            : w == pw_w[0]   ? pw_v[0]
                            : w == pw_w[1]   ? pw_v[1]
                                             : pad_word(pad_b, w, T);
        for (uint32_t t = qb; t; t &= t - 1) {
            int j = (w << 5) + __ffs(t) - 1;
            gq_s[oq] = j;
            if (writer) gq_out[oq] = j;
            ++oq;
            if (!((pw >> (j & 31)) & 1u)) {
                gk_s[ok] = j;
                if (writer) gk_out[ok] = j;
                ++ok;
            }
        }
    }
    if (writer && tid == kPrepThreads - 1) {
        p.ws.n_gq[b] = oq;
        p.ws.n_gk[b] = ok;
    }
    __syncthreads();

    if (p.pack) {
        const int nk = n_k_total, nq = n_q_total;
        const size_t bh = static_cast<size_t>(b) * p.H + h;
        // 16-byte words per row: 8 (d = 64) or 16 (d = 128)
        const int wsh = p.d == 128 ? 4 : 3, rw = 1 << wsh;
        const uint4* q4 = reinterpret_cast<const uint4*>(p.q) + bh * T * rw;
        const uint4* k4 = reinterpret_cast<const uint4*>(p.k) + bh * T * rw;
        const uint4* v4 = reinterpret_cast<const uint4*>(p.v) + bh * T * rw;
        uint4* qg4 = reinterpret_cast<uint4*>(p.ws.qg) + bh * p.ngp * rw;
        uint4* kg4 = reinterpret_cast<uint4*>(p.ws.kg) + bh * p.ngp * rw;
        uint4* vg4 = reinterpret_cast<uint4*>(p.ws.vg) + bh * p.ngp * rw;
#pragma unroll 4
        for (int idx = tid; idx < p.ngp * rw; idx += kPrepThreads) {  // (unrolled: the loads of several rows in flight)
            int a = idx >> wsh, c = idx & (rw - 1);
            uint4 kv = make_uint4(0u, 0u, 0u, 0u), vv = kv, qv = kv;
            if (a < nk) {
                size_t row = static_cast<size_t>(gk_s[a]);
                kv = k4[row * rw + c];
                vv = v4[row * rw + c];
            }
            if (a < nq) qv = q4[static_cast<size_t>(gq_s[a]) * rw + c];
            kg4[idx] = kv;
            vg4[idx] = vv;
            qg4[idx] = qv;
        }
    }
}

}  // namespace lf
