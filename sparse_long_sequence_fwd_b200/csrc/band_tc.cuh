// band_tc.cuh -- K1: fused band kernel for bf16, d = 64, on the 5th-generation
// tensor cores (tcgen05) with TMA staging and TMEM accumulators.
//
// Work item = 128 consecutive queries of one residue class c of one (b, h):
// rows i = c + dil*(q0 + x), x in [0, 128).  Inside a class the dilated
// window {i + dil*t : |t| <= r} ("Longformer" wiki, section 2.2.3; the
// "Longformer" note, section "Sliding-Window Attention") is a dense window
// of radius r over the class's own positions, so the item needs the key
// rows of its diagonal band only: decimated keys [q0 - r, q0 + 127 + r],
// fetched in blocks of 128 with TMA boxes whose row traversal stride is dil.
// After the band blocks come ceil(n_gk / 128) blocks of packed global keys
// (built by the prep kernel), masked where a global key already lies in the
// row's window so each key counts once ("Global Attention": N(i) = N_local(i)
// U G).
//
// Per key block:   S = Q K^T        tcgen05.mma, M=128, N=128 (or the global
//                                   count rounded to 16), K=64 -> TMEM (fp32),
//                                   double-buffered so the next block's S is
//                                   computed during this block's softmax
//                  online softmax   two threads per query row, one per half
//                                   of the block's 128 key columns; each
//                                   keeps its own running max and exponent
//                                   base (fp32, log2 domain)
//                  O_h += P_h V_h   P (bf16) through 128B-swizzled shared
//                                   memory (double-buffered); the PV
//                                   product's first 4 k-steps (keys 0..63)
//                                   accumulate into O_0, the last 4 into
//                                   O_1, so each half's exponent base
//                                   stays private; M=128, N=64, in TMEM
//                  L_h += P_h 1     row sums from the tensor core too (N=16
//                                   against a tile of ones)
// At the end of a tile the two halves swap bases once and each writes half
// of the output row: y = (2^m0 O_0 + 2^m1 O_1) / (2^m0 L_0 + 2^m1 L_1).
// The exponent base of a row is only moved (and O, l rescaled in place) when
// the running max exceeds it by more than 2^8; otherwise p = 2^(s - base)
// stays below 256, which fp32 accumulation and bf16 P absorb exactly as well.
// The mask view of the note ("Mask View": A = QK^T/sqrt(d) + M, M = -inf off
// the pattern) is applied inline: band limits and sequence ends as a per-row
// column interval, padded keys from the key padding mask, the global-key
// dedup test per column.  Nothing of size T x T is built.
//
// Warp roles (320 threads): warp 0 lane 0 TMA producer, warp 1 lane 0 MMA
// issuer (warp 1 also owns the TMEM allocation), warps 2..5 softmax of key
// columns 0..63, warps 6..9 softmax of columns 64..127 of the same rows (warp
// w serves TMEM lanes 32*(w%4)..+31).  Every hand-off is an mbarrier and
// every wait is bounded (ptx.cuh).  In steady state the softmax warps never
// wait on a round trip through the MMA warp: S is double-buffered, and P(k)
// only needs the product of block k-2 to have finished.
#pragma once
#include "lf_common.cuh"
#include "ptx.cuh"

namespace lf {

constexpr int kBM = 128;
constexpr int kBN = 128;
constexpr int kHD = 64;
constexpr int kStages = 4;
constexpr int kTileBytes = kBM * kHD * 2;  // 16 KB: 128 rows x 128 bytes
constexpr int kBandThreads = 320;
constexpr int kSoftmaxWarp0 = 2;           // warps 2..9
constexpr float kRescaleLog2 = 8.f;        // move the exponent base only past 2^8

constexpr int kOffQ = 0;
constexpr int kOffK = kOffQ + kTileBytes;                  // kStages x 16 KB
constexpr int kOffV = kOffK + kStages * kTileBytes;        // kStages x 16 KB
constexpr int kOffP = kOffV + kStages * kTileBytes;        // 2 buffers x (keys 0..63 | 64..127) x 16 KB
constexpr int kOffOnes = kOffP + 2 * 2 * kTileBytes;       // 16 x 128 bf16 ones (row-sum operand), 4 KB
constexpr int kOffX = kOffOnes + 4096;                     // per-tile exchange of bases: [2 parity][2 half][128] f32
constexpr int kOffBar = kOffX + 2 * 2 * kBM * 4;
// barrier slots
constexpr int kBarQFull = 0, kBarQEmpty = 1, kBarKvFull = 2, kBarKvEmpty = kBarKvFull + kStages,
              kBarSFull = kBarKvEmpty + kStages, kBarSFree = kBarSFull + 2, kBarPFull = kBarSFree + 2,
              kBarOFull = kBarPFull + 2, kBarXchg = kBarOFull + 2, kBarDrain = kBarXchg + 4,
              kNumBars = kBarDrain + 1;
constexpr int kOffMisc = kOffBar + ((kNumBars * 8 + 15) / 16) * 16;
constexpr int kMiscBytes = 16;
constexpr int kBandSmem = kOffMisc + kMiscBytes + 1024;  // + alignment slack
static_assert(kBandSmem <= 232448, "shared memory budget");

constexpr uint32_t kTmemCols = 512;
// TMEM columns: S buffers at 0 and 128 (fp32, 128 wide); per key half h
// (keys 0..63 / 64..127 of every block) an output accumulator O_h at
// 256 + 64 h (fp32, 64 wide) and a row-sum accumulator L_h at 384 + 16 h
// (fp32, 16 identical columns: P times a ones tile).
__device__ __forceinline__ uint32_t col_s(uint32_t buf) { return buf * 128u; }
__device__ __forceinline__ uint32_t col_o(uint32_t h) { return 256u + 64u * h; }
__device__ __forceinline__ uint32_t col_l(uint32_t h) { return 384u + 16u * h; }

struct BandTile {
    int b, bh, c, dil, dk, R;
    int Tc, q0, kbase, kb_lo, nbb, ngk, ngb;
};

__device__ __forceinline__ BandTile band_decode(const BandTcParams& p, int item) {
    BandTile t;
    t.b = item / p.items_per_b;
    int rem = item - t.b * p.items_per_b;
    int h = 0;
    while (p.head_start[h + 1] <= rem) ++h;
    rem -= p.head_start[h];
    t.bh = t.b * p.H + h;
    t.dk = p.head_dk[h];
    t.dil = p.dk_dil[t.dk];
    t.R = p.dk_rows[t.dk];
    int c = 0, Tc = 0;
    for (c = 0; c < t.dil; ++c) {
        Tc = (p.T - c + t.dil - 1) / t.dil;
        const int nt = (Tc + kBM - 1) / kBM;
        if (rem < nt) break;
        rem -= nt;
    }
    t.c = c;
    t.Tc = Tc;
    t.q0 = rem * kBM;
    t.kbase = t.q0 - p.r;
    const int lo = max(0, t.kbase);
    const int hi = min(Tc - 1, t.q0 + kBM - 1 + p.r);
    t.kb_lo = (lo - t.kbase) / kBN;
    t.nbb = (hi - t.kbase) / kBN + 1 - t.kb_lo;
    t.ngk = p.n_gk[t.b];
    t.ngb = (t.ngk + kBN - 1) / kBN;
    return t;
}

// Columns of global block gb that the MMA computes (multiple of 16).
__device__ __forceinline__ int global_block_cols(int ngk, int gb) {
    const int rem = min(kBN, ngk - gb * kBN);
    return (rem + 15) & ~15;
}

// Bits [lo, hi) of a 32-bit word (lo, hi clamped to [0, 32]).
__device__ __forceinline__ uint32_t range_bits(int lo, int hi) {
    lo = max(0, min(32, lo));
    hi = max(0, min(32, hi));
    if (hi <= lo) return 0u;
    const uint32_t upto_hi = hi >= 32 ? 0xffffffffu : ((1u << hi) - 1u);
    const uint32_t upto_lo = (1u << lo) - 1u;
    return upto_hi & ~upto_lo;
}

// ------------------------------------------------------------ softmax role
// Thread (row x, half hf) owns key columns [64 hf, 64 hf + 64) of row x but
// reads all 128 for the row max.  POS: scale > 0, so maxima are taken on raw
// scores and the scale is folded into the exp2 argument.
template <bool POS, bool KEEP = true>
__device__ __forceinline__ float masked_max32(uint32_t* v, uint32_t mk, bool full, float sl2) {
    float mxp[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) mxp[u] = -INFINITY;
    if (full) {
#pragma unroll
        for (int j = 0; j < 32; ++j) {
            float f = __uint_as_float(v[j]);
            if (!POS) f *= sl2;
            if (KEEP) v[j] = __float_as_uint(f);
            mxp[j & 7] = fmaxf(mxp[j & 7], f);
        }
    } else {
#pragma unroll
        for (int j = 0; j < 32; ++j) {
            float f = __uint_as_float(v[j]);
            if (!POS) f *= sl2;
            f = ((mk >> j) & 1u) ? f : -INFINITY;
            if (KEEP) v[j] = __float_as_uint(f);
            mxp[j & 7] = fmaxf(mxp[j & 7], f);
        }
    }
    return fmaxf(fmaxf(fmaxf(mxp[0], mxp[1]), fmaxf(mxp[2], mxp[3])),
                 fmaxf(fmaxf(mxp[4], mxp[5]), fmaxf(mxp[6], mxp[7])));
}

template <bool POS>
__device__ __forceinline__ void softmax_role(const BandTcParams& p, uint8_t* smem, uint64_t* bars,
                                             volatile int* abort_flag, uint32_t tmem_base) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int wq = warp & 3;
    const int hf = (warp - kSoftmaxWarp0) >> 2;  // column half
    const int x = wq * 32 + lane;                // query row inside the tile = TMEM lane
    const uint32_t lane_off = static_cast<uint32_t>(wq * 32) << 16;
    const uint32_t tO = tmem_base + lane_off + col_o(hf);  // this key half's output accumulator
    const uint32_t tL = tmem_base + lane_off + col_l(hf);  // ... and row-sum accumulator
    float* xm = reinterpret_cast<float*>(smem + kOffX);    // [2 parity][2 half][128]
    uint64_t* xbar = &bars[kBarXchg + wq];
    uint32_t x_cnt = 0;
    const int rowoff = (x >> 3) * 1024 + (x & 7) * 128;
    const float sl2 = p.sl2;
    uint32_t blk_it = 0;  // key blocks processed by this CTA (all tiles)

    auto wait_warp = [&](uint64_t* bar, uint32_t parity) -> bool {
        int ok = 1;
        if (lane == 0) ok = mbar_wait(bar, parity, abort_flag) ? 1 : 0;
        ok = __shfl_sync(0xffffffffu, ok, 0);
        __syncwarp();  // memory order for the other lanes
        return ok != 0;
    };
    // block j's product O += P V has completed (barrier of P buffer j % 2)
    auto wait_pv = [&](uint32_t j) -> bool { return wait_warp(&bars[kBarOFull + (j & 1u)], (j >> 1) & 1u); };
    // swap one float per row with the other half's thread of the same row
    auto exchange = [&](float mine, float* other) -> bool {
        float* slot = xm + (x_cnt & 1u) * (2 * kBM);
        slot[hf * kBM + x] = mine;
        __syncwarp();
        if (lane == 0) mbar_arrive(xbar);
        if (!wait_warp(xbar, x_cnt & 1u)) return false;
        *other = slot[(hf ^ 1) * kBM + x];
        ++x_cnt;
        return true;
    };

    for (int item = blockIdx.x; item < p.n_items; item += gridDim.x) {
        const BandTile t = band_decode(p, item);
        const int ip = t.q0 + x;         // decimated row index
        const int i = t.c + t.dil * ip;  // position in the sequence
        bool row_ok = ip < t.Tc;
        if (row_ok && ((p.gbit[static_cast<size_t>(t.b) * p.W + (i >> 5)] >> (i & 31)) & 1u)) row_ok = false;
        const int32_t* gk = p.gk_list + static_cast<size_t>(t.b) * p.gstride;
        const long reach = static_cast<long>(t.dil) * p.r;

        float m_run = -INFINITY;  // running row max (scaled, log2 domain)
        float m_ref = -INFINITY;  // exponent base in use (-inf: nothing valid yet)
        const int nb = t.nbb + t.ngb;
        for (int blk = 0; blk < nb; ++blk, ++blk_it) {
            const uint32_t sb = blk_it & 1u;
            const bool band = blk < t.nbb;
            uint32_t mk[2];  // valid-key bits of this half's two 32-column chunks
            uint32_t need = 0;
            int ncols = kBN;
            if (band) {
                const int kb = t.kb_lo + blk;
                const int j0 = t.kbase + kBN * kb;
                uint32_t padw[2] = {0u, 0u};
                if (p.pad) {
#pragma unroll
                    for (int u = 0; u < 2; ++u) {
                        const int jd = j0 + 64 * hf + 32 * u + lane;
                        bool padded = false;
                        if (jd >= 0 && jd < t.Tc)
                            padded = p.pad[static_cast<size_t>(t.b) * p.T + t.c + static_cast<size_t>(t.dil) * jd] != 0;
                        padw[u] = __ballot_sync(0xffffffffu, padded);
                    }
                }
                const int ylo = max(max(0, x - kBN * kb), -j0);
                const int yhi = min(min(kBN, x + 2 * p.r + 1 - kBN * kb), t.Tc - j0);
#pragma unroll
                for (int u = 0; u < 2; ++u) {
                    const int c0 = 64 * hf + 32 * u;
                    mk[u] = range_bits(ylo - c0, yhi - c0) & ~padw[u];
                    const bool any = max(ylo, c0) < min(yhi, c0 + 32);
                    if (__any_sync(0xffffffffu, any)) need |= 1u << u;
                }
            } else {
                const int gb = blk - t.nbb;
                ncols = global_block_cols(t.ngk, gb);
                const int nvalid = min(kBN, t.ngk - gb * kBN);
#pragma unroll
                for (int u = 0; u < 2; ++u) {
                    const int c0 = 64 * hf + 32 * u;
                    mk[u] = 0u;
                    if (c0 < nvalid) {
                        need |= 1u << u;
                        for (int a = 0; a < 32 && c0 + a < nvalid; ++a) {
                            const long diff = static_cast<long>(__ldg(gk + gb * kBN + c0 + a)) - i;
                            const bool in_window = (diff % t.dil == 0) && diff <= reach && diff >= -reach;
                            if (!in_window) mk[u] |= 1u << a;
                        }
                    }
                }
            }
            bool full[2];
#pragma unroll
            for (int u = 0; u < 2; ++u) full[u] = __all_sync(0xffffffffu, mk[u] == 0xffffffffu);

            // ---- this half's 64 columns of the S block
            if (!wait_warp(&bars[kBarSFull + sb], (blk_it >> 1) & 1u)) return;
            tc_fence_after();
            const uint32_t tS = tmem_base + lane_off + col_s(sb) + 64u * hf;
            uint32_t sr[64];
            if (need & 1u) tmem_ld32(tS, sr);
            if (need & 2u) tmem_ld32(tS + 32, sr + 32);
            tmem_ld_wait(sr);
            reg_fence32(sr + 32);
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars[kBarSFree + sb]);

            float mx = -INFINITY;
            if (need & 1u) mx = masked_max32<POS>(sr, mk[0], full[0], sl2);
            if (need & 2u) mx = fmaxf(mx, masked_max32<POS>(sr + 32, mk[1], full[1], sl2));
            if (POS) mx *= sl2;  // -inf stays -inf
            m_run = fmaxf(m_run, mx);

            // ---- move this half's exponent base if its max ran past it (rare): rescale O_h and L_h
            float alpha = 1.f;
            bool move = (m_run != -INFINITY) && (m_ref == -INFINITY || m_run > m_ref + kRescaleLog2);
            if (blk == 0) {
                m_ref = m_run;  // the first product of the tile overwrites O_h and L_h
                move = false;
            } else if (move) {
                alpha = (m_ref == -INFINITY) ? 0.f : ex2_approx(m_ref - m_run);
                m_ref = m_run;
            }
            if (__any_sync(0xffffffffu, move)) {
                if (!wait_pv(blk_it - 1)) return;  // O_h and L_h hold every earlier product
                tc_fence_after();
                uint32_t orr[32];
#pragma unroll 1
                for (int part = 0; part < 2; ++part) {  // O_h, 32 columns at a time
                    tmem_ld32(tO + 32u * part, orr);
                    tmem_ld_wait(orr);
#pragma unroll
                    for (int c = 0; c < 32; ++c) orr[c] = __float_as_uint(__uint_as_float(orr[c]) * alpha);
                    tmem_st32(tO + 32u * part, orr);
                }
                tmem_ld16(tL, orr);  // L_h: exactly its 16 columns
                tmem_ld_wait16(orr);
#pragma unroll
                for (int c = 0; c < 16; ++c) orr[c] = __float_as_uint(__uint_as_float(orr[c]) * alpha);
                tmem_st16(tL, orr);
                tmem_st_wait();
            }
            const float base = (m_ref == -INFINITY) ? 0.f : m_ref;

            // ---- p = 2^(s - base) on this half, as bf16 into P buffer sb once the
            //      product of block blk_it - 2 has read that buffer
            if (blk_it >= 2 && !wait_pv(blk_it - 2)) return;
            uint8_t* pbuf = smem + kOffP + sb * (2 * kTileBytes) + hf * kTileBytes;
#pragma unroll
            for (int ch = 0; ch < 8; ++ch) {
                if (64 * hf + 8 * ch < ncols) {
                    uint4 val = make_uint4(0u, 0u, 0u, 0u);
                    if (need & (1u << (ch >> 2))) {
                        float e[8];
#pragma unroll
                        for (int j = 0; j < 8; ++j) {
                            const float v = __uint_as_float(sr[8 * ch + j]);
                            e[j] = POS ? ex2_approx(fmaf(v, sl2, -base)) : ex2_approx(v - base);
                        }
                        val.x = pack_bf16x2(e[0], e[1]);
                        val.y = pack_bf16x2(e[2], e[3]);
                        val.z = pack_bf16x2(e[4], e[5]);
                        val.w = pack_bf16x2(e[6], e[7]);
                    }
                    *reinterpret_cast<uint4*>(pbuf + rowoff + ((ch ^ (x & 7)) << 4)) = val;
                }
            }
            fence_proxy_async_smem();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars[kBarPFull + sb]);
        }

        // ---- epilogue: output columns [32 hf, 32 hf + 32) of this row from both key
        //      halves, y = (2^m0 O_0 + 2^m1 O_1) / (2^m0 L_0 + 2^m1 L_1)
        //      (global rows are written by K2)
        float m_other;
        if (!exchange(m_ref, &m_other)) return;
        if (!wait_pv(blk_it - 1)) return;
        tc_fence_after();
        const float m0 = hf == 0 ? m_ref : m_other, m1 = hf == 0 ? m_other : m_ref;
        const float mm = fmaxf(m0, m1);
        const float f0 = (m0 == -INFINITY) ? 0.f : ex2_approx(m0 - mm);
        const float f1 = (m1 == -INFINITY) ? 0.f : ex2_approx(m1 - mm);
        float l0, l1;
        {
            uint32_t lr[16];
            tmem_ld16(tmem_base + lane_off + col_l(0), lr);
            tmem_ld_wait16(lr);
            l0 = __uint_as_float(lr[0]);
            tmem_ld16(tmem_base + lane_off + col_l(1), lr);
            tmem_ld_wait16(lr);
            l1 = __uint_as_float(lr[0]);
        }
        const float l = f0 * l0 + f1 * l1;
        const float inv = l > 0.f ? 1.f / l : 0.f;
        uint4* dst = reinterpret_cast<uint4*>(p.out + (static_cast<size_t>(t.bh) * p.T + i) * kHD + 32 * hf);
#pragma unroll 1
        for (int q16 = 0; q16 < 2; ++q16) {  // 16 output columns at a time
            uint32_t a0[16], a1[16];
            tmem_ld16(tmem_base + lane_off + col_o(0) + 32u * hf + 16u * q16, a0);
            tmem_ld16(tmem_base + lane_off + col_o(1) + 32u * hf + 16u * q16, a1);
            tmem_ld_wait16(a0);
            reg_fence16(a1);
            float y[16];
#pragma unroll
            for (int c = 0; c < 16; ++c) y[c] = (f0 * __uint_as_float(a0[c]) + f1 * __uint_as_float(a1[c])) * inv;
            if (row_ok) {
#pragma unroll
                for (int v8 = 0; v8 < 2; ++v8) {
                    uint4 val;
                    val.x = pack_bf16x2(y[8 * v8 + 0], y[8 * v8 + 1]);
                    val.y = pack_bf16x2(y[8 * v8 + 2], y[8 * v8 + 3]);
                    val.z = pack_bf16x2(y[8 * v8 + 4], y[8 * v8 + 5]);
                    val.w = pack_bf16x2(y[8 * v8 + 6], y[8 * v8 + 7]);
                    dst[2 * q16 + v8] = val;
                }
            }
        }
        tc_fence_before();
    }
}

__global__ void __launch_bounds__(kBandThreads, 1) band_tc_kernel(const __grid_constant__ BandTcParams p) {
    extern __shared__ uint8_t band_smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(band_smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kOffBar);
    uint32_t* misc = reinterpret_cast<uint32_t*>(smem + kOffMisc);
    uint32_t* tmem_slot = misc;
    volatile int* abort_flag = reinterpret_cast<volatile int*>(misc + 1);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        mbar_init(&bars[kBarQFull], 1);
        mbar_init(&bars[kBarQEmpty], 1);
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&bars[kBarKvFull + s], 1);
            mbar_init(&bars[kBarKvEmpty + s], 1);
        }
        for (int s = 0; s < 2; ++s) {
            mbar_init(&bars[kBarSFull + s], 1);
            mbar_init(&bars[kBarSFree + s], 8);
        }
        for (int s = 0; s < 2; ++s) {
            mbar_init(&bars[kBarPFull + s], 8);
            mbar_init(&bars[kBarOFull + s], 1);
        }
        for (int w = 0; w < 4; ++w) mbar_init(&bars[kBarXchg + w], 2);
        mbar_init(&bars[kBarDrain], 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 0 && lane == 0) {
        for (int k = 0; k < kMaxDilKinds; ++k) {
            prefetch_tmap(&p.tm_q[k]);
            prefetch_tmap(&p.tm_k[k]);
            prefetch_tmap(&p.tm_v[k]);
        }
        prefetch_tmap(&p.tm_kg);
        prefetch_tmap(&p.tm_vg);
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, kTmemCols);
        tmem_relinquish();
    }
    {  // the ones tile (bf16 1.0) read by the row-sum MMA
        uint32_t* ones = reinterpret_cast<uint32_t*>(smem + kOffOnes);
        for (int u = threadIdx.x; u < 1024; u += kBandThreads) ones[u] = 0x3F803F80u;
        fence_proxy_async_smem();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;

    if (warp == 0) {
        // ------------------------------------------------------ TMA producer
        if (lane == 0) {
            uint32_t kv_it = 0, q_it = 0;
            bool alive = true;
            for (int item = blockIdx.x; item < p.n_items && alive; item += gridDim.x) {
                const BandTile t = band_decode(p, item);
                if (!mbar_wait(&bars[kBarQEmpty], (q_it & 1u) ^ 1u, abort_flag)) break;
                ++q_it;
                mbar_arrive_expect_tx(&bars[kBarQFull], kTileBytes);
                for (int u = 0; u < kBM; u += t.R)
                    tma_load_3d(smem + kOffQ + u * 128, &p.tm_q[t.dk], &bars[kBarQFull], 0,
                                t.c + t.dil * (t.q0 + u), t.bh);
                const int nb = t.nbb + t.ngb;
                for (int blk = 0; blk < nb; ++blk) {
                    const uint32_t s = kv_it % kStages, ph = (kv_it / kStages) & 1u;
                    if (!mbar_wait(&bars[kBarKvEmpty + s], ph ^ 1u, abort_flag)) {
                        alive = false;
                        break;
                    }
                    mbar_arrive_expect_tx(&bars[kBarKvFull + s], 2 * kTileBytes);
                    uint8_t* dK = smem + kOffK + s * kTileBytes;
                    uint8_t* dV = smem + kOffV + s * kTileBytes;
                    if (blk < t.nbb) {
                        const int j0 = t.kbase + kBN * (t.kb_lo + blk);
                        for (int u = 0; u < kBN; u += t.R) {
                            const int y = t.c + t.dil * (j0 + u);
                            tma_load_3d(dK + u * 128, &p.tm_k[t.dk], &bars[kBarKvFull + s], 0, y, t.bh);
                            tma_load_3d(dV + u * 128, &p.tm_v[t.dk], &bars[kBarKvFull + s], 0, y, t.bh);
                        }
                    } else {
                        const int gb = blk - t.nbb;
                        tma_load_3d(dK, &p.tm_kg, &bars[kBarKvFull + s], 0, gb * kBN, t.bh);
                        tma_load_3d(dV, &p.tm_vg, &bars[kBarKvFull + s], 0, gb * kBN, t.bh);
                    }
                    ++kv_it;
                }
            }
            if (*abort_flag) {  // let issued copies land before the CTA can exit
                for (uint32_t s = 0; s < kStages && kv_it > s; ++s)
                    (void)mbar_wait_drain(&bars[kBarKvFull + s], ((kv_it - 1 - s) / kStages) & 1u);
                if (q_it) (void)mbar_wait_drain(&bars[kBarQFull], (q_it - 1) & 1u);
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------- MMA issuer
        if (lane == 0) {
            const uint32_t idesc_pv = idesc_bf16(kBM, kHD, 0, 1);
            const uint32_t sQ = smem_u32(smem + kOffQ);
            const uint32_t sK0 = smem_u32(smem + kOffK);
            const uint32_t sV0 = smem_u32(smem + kOffV);
            const uint32_t sP = smem_u32(smem + kOffP);
            const uint32_t idesc_l = idesc_bf16(kBM, 16, 0, 0);
            const uint32_t sOnes = smem_u32(smem + kOffOnes);
            uint32_t kv_it = 0, q_it = 0, blk_it = 0;
            bool alive = true;
            // O += P V and l += P 1 for block j (P buffer j % 2)
            auto issue_pv = [&](uint32_t j, uint32_t stage, int nk, bool first) -> bool {
                const uint32_t pb = j & 1u;
                if (!mbar_wait(&bars[kBarPFull + pb], (j >> 1) & 1u, abort_flag)) return false;
                tc_fence_after();
                const uint32_t aP = sP + pb * (2 * kTileBytes);
                const uint32_t bV = sV0 + stage * kTileBytes;
                for (int ks = 0; ks < nk / 16; ++ks) {
                    // k-steps 0..3 cover keys 0..63 (accumulators of half 0), 4..7 keys 64..127 (half 1)
                    const uint32_t h = static_cast<uint32_t>(ks >> 2);
                    const uint64_t ad = sdesc_k_sw128(aP + h * kTileBytes + (ks & 3) * 32);
                    const uint32_t acc = ((ks & 3) > 0 || !first) ? 1u : 0u;
                    tc_mma_ss(tmem_base + col_o(h), ad, sdesc_mn_sw128(bV + ks * 2048), idesc_pv, acc);
                    tc_mma_ss(tmem_base + col_l(h), ad, sdesc_k_sw128(sOnes + h * 2048 + (ks & 3) * 32), idesc_l, acc);
                }
                tc_commit(&bars[kBarOFull + pb]);
                tc_commit(&bars[kBarKvEmpty + stage]);
                return true;
            };
            for (int item = blockIdx.x; item < p.n_items && alive; item += gridDim.x) {
                const BandTile t = band_decode(p, item);
                if (!mbar_wait(&bars[kBarQFull], q_it & 1u, abort_flag)) break;
                ++q_it;
                tc_fence_after();
                const int nb = t.nbb + t.ngb;
                uint32_t prev_stage = 0;
                int prev_nk = 0;
                for (int blk = 0; blk < nb; ++blk) {
                    const uint32_t s = kv_it % kStages, ph = (kv_it / kStages) & 1u;
                    const uint32_t sb = blk_it & 1u;
                    if (!mbar_wait(&bars[kBarKvFull + s], ph, abort_flag) ||
                        !mbar_wait(&bars[kBarSFree + sb], ((blk_it >> 1) & 1u) ^ 1u, abort_flag)) {
                        alive = false;
                        break;
                    }
                    tc_fence_after();
                    const int ncols = blk < t.nbb ? kBN : global_block_cols(t.ngk, blk - t.nbb);
                    const uint32_t idesc_s = idesc_bf16(kBM, ncols, 0, 0);
                    const uint32_t bK = sK0 + s * kTileBytes;
#pragma unroll
                    for (int ks = 0; ks < kHD / 16; ++ks)
                        tc_mma_ss(tmem_base + col_s(sb), sdesc_k_sw128(sQ + ks * 32), sdesc_k_sw128(bK + ks * 32),
                                  idesc_s, ks > 0 ? 1u : 0u);
                    tc_commit(&bars[kBarSFull + sb]);
                    if (blk == nb - 1) tc_commit(&bars[kBarQEmpty]);
                    if (blk > 0 && !issue_pv(blk_it - 1, prev_stage, prev_nk, blk == 1)) {
                        alive = false;
                        break;
                    }
                    prev_stage = s;
                    prev_nk = ncols;
                    ++blk_it;
                    ++kv_it;
                }
                if (alive && !issue_pv(blk_it - 1, prev_stage, prev_nk, nb == 1)) alive = false;
            }
            // all MMAs issued by this thread complete before TMEM is released
            tc_commit(&bars[kBarDrain]);
            (void)mbar_wait_drain(&bars[kBarDrain], 0u);
        }
    } else {
        // ------------------------------------------- softmax and epilogue
        if (p.sl2 > 0.f)
            softmax_role<true>(p, smem, bars, abort_flag, tmem_base);
        else
            softmax_role<false>(p, smem, bars, abort_flag, tmem_base);
    }

    tc_fence_before();
    __syncthreads();
    if (threadIdx.x == 0 && *abort_flag) atomicOr(p.status, kStatusTimeout);
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, kTmemCols);
    }
}

}  // namespace lf
