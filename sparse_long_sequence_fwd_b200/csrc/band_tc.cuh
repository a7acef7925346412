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
//                  online softmax   four threads per query row, one per
//                                   quarter (32 keys) of the block; each
//                                   keeps its own running max, exponent base
//                                   and row sum (fp32, log2 domain)
//                  O_q += P_q V_q   P (bf16) through 128B-swizzled shared
//                                   memory (double-buffered); k-steps 2q and
//                                   2q+1 of the PV product (keys 32q..32q+31)
//                                   accumulate into O_q, so each quarter's
//                                   exponent base stays private; M=128, N=64
// A quarter's base only moves (O_q and its sum rescaled in place) when its
// running max exceeds the base by more than 2^8; otherwise p = 2^(s - base)
// stays below 256, which fp32 accumulation and bf16 P absorb.  At the end of
// a tile the quarters swap (base, sum) once and each writes 16 output
// columns: y = sum_q 2^(m_q - M) O_q / sum_q 2^(m_q - M) l_q.
// The mask view of the note ("Mask View": A = QK^T/sqrt(d) + M, M = -inf off
// the pattern) is applied inline: band limits and sequence ends as a per-row
// column interval, padded keys from the key padding mask, the global-key
// dedup test per column.  Nothing of size T x T is built.
//
// Warp roles (640 threads): warp 0 lane 0 TMA producer, warp 1 lane 0 issues
// S = Q K^T (warp 1 also owns the TMEM allocation), warps 2 and 3 lane 0
// issue the two halves of the PV product, warps 4..19 softmax: quarter (w - 4) / 4 of TMEM lanes 32*(w%4)..+31, so every SM
// sub-partition runs four softmax warps.  Every hand-off is an mbarrier and
// every wait is bounded (ptx.cuh).  In steady state no softmax warp waits on
// a round trip through the MMA warp: S is double-buffered, and P(k) only
// needs the product of block k-2 to have finished.
#pragma once
#include "lf_common.cuh"
#include "ptx.cuh"

namespace lf {

constexpr int kBM = 128;
constexpr int kBN = 128;
constexpr int kHD = 64;
constexpr int kStages = 4;
constexpr int kTileBytes = kBM * kHD * 2;  // 16 KB: 128 rows x 128 bytes
constexpr int kBandThreads = 640;
constexpr int kSoftmaxWarp0 = 4;           // warps 4..19
constexpr int kSoftmaxWarps = 16;
constexpr float kRescaleLog2 = 8.f;        // move the exponent base only past 2^8

constexpr int kOffQ = 0;
constexpr int kOffK = kOffQ + kTileBytes;                  // kStages x 16 KB
constexpr int kOffV = kOffK + kStages * kTileBytes;        // kStages x 16 KB
constexpr int kOffP = kOffV + kStages * kTileBytes;        // 2 buffers x (keys 0..63 | 64..127) x 16 KB
constexpr int kOffX = kOffP + 2 * 2 * kTileBytes;          // per-tile exchange: [2 parity][2 (m, l)][4 q][128] f32
constexpr int kOffBar = kOffX + 2 * 2 * 4 * kBM * 4;
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
// TMEM columns: S buffers at 0 and 128 (fp32, 128 wide); output accumulator
// O_q of key quarter q at 256 + 64 q (fp32, 64 wide).
__device__ __forceinline__ uint32_t col_s(uint32_t buf) { return buf * 128u; }
__device__ __forceinline__ uint32_t col_o(uint32_t q) { return 256u + 64u * q; }

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
// Thread (row x, quarter q) owns key columns [32 q, 32 q + 32) of every block
// of row x.  POS: scale > 0, so maxima are taken on raw scores and the scale
// is folded into the exp2 argument.
template <bool POS>
__device__ __forceinline__ void softmax_role(const BandTcParams& p, uint8_t* smem, uint64_t* bars,
                                             volatile int* abort_flag, uint32_t tmem_base) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int wq = warp & 3;
    const int qi = (warp - kSoftmaxWarp0) >> 2;  // key quarter
    const int x = wq * 32 + lane;                // query row inside the tile = TMEM lane
    const uint32_t lane_off = static_cast<uint32_t>(wq * 32) << 16;
    const uint32_t tOq = tmem_base + lane_off + col_o(qi);
    const int rowoff = (x >> 3) * 1024 + (x & 7) * 128;
    const float sl2 = p.sl2;
    float* xm = reinterpret_cast<float*>(smem + kOffX);  // [2 parity][2][4][128]
    uint64_t* xbar = &bars[kBarXchg + wq];
    uint32_t blk_it = 0, x_cnt = 0;

    // every lane polls (each lane's own acquire), then the warp agrees on the outcome
    auto wait_warp = [&](uint64_t* bar, uint32_t parity) -> bool {
        const bool ok = mbar_wait(bar, parity, abort_flag);
        return __all_sync(0xffffffffu, ok);
    };
    // block j's product O += P V has completed (barrier of P buffer j % 2)
    auto wait_pv = [&](uint32_t j) -> bool { return wait_warp(&bars[kBarOFull + (j & 1u)], (j >> 1) & 1u); };

    for (int item = blockIdx.x; item < p.n_items; item += gridDim.x) {
        const BandTile t = band_decode(p, item);
        const int ip = t.q0 + x;         // decimated row index
        const int i = t.c + t.dil * ip;  // position in the sequence
        bool row_ok = ip < t.Tc;
        if (row_ok && ((p.gbit[static_cast<size_t>(t.b) * p.W + (i >> 5)] >> (i & 31)) & 1u)) row_ok = false;
        const int32_t* gk = p.gk_list + static_cast<size_t>(t.b) * p.gstride;
        const int reach = t.dil * p.r;

        float m_run = -INFINITY;  // running max of this quarter (scaled, log2 domain)
        float m_ref = -INFINITY;  // its exponent base (-inf: nothing valid yet)
        float l_q = 0.f;          // its row sum, relative to m_ref
        const int nb = t.nbb + t.ngb;
        for (int blk = 0; blk < nb; ++blk, ++blk_it) {
            const uint32_t sb = blk_it & 1u;
            const int c0 = 32 * qi;
            uint32_t mk = 0u;
            bool need;
            int ncols = kBN;
            if (blk < t.nbb) {
                const int kb = t.kb_lo + blk;
                const int j0 = t.kbase + kBN * kb;
                // block inside the band for every row and inside [0, Tc): no per-column test
                // (128 kb + y - x lies in [0, 2r] for all x, y in [0, 128))
                const bool interior = !p.pad && kb >= 1 && kBN * kb + kBN - 1 <= 2 * p.r && j0 >= 0 &&
                                      j0 + kBN <= t.Tc;
                if (interior) {
                    mk = 0xffffffffu;
                    need = true;
                } else {
                    uint32_t padw = 0u;
                    if (p.pad) {
                        const int jd = j0 + c0 + lane;
                        bool padded = false;
                        if (jd >= 0 && jd < t.Tc)
                            padded = p.pad[static_cast<size_t>(t.b) * p.T + t.c + static_cast<size_t>(t.dil) * jd] != 0;
                        padw = __ballot_sync(0xffffffffu, padded);
                    }
                    const int ylo = max(max(0, x - kBN * kb), -j0);
                    const int yhi = min(min(kBN, x + 2 * p.r + 1 - kBN * kb), t.Tc - j0);
                    mk = range_bits(ylo - c0, yhi - c0) & ~padw;
                    need = __any_sync(0xffffffffu, max(ylo, c0) < min(yhi, c0 + 32));
                }
            } else {
                const int gb = blk - t.nbb;
                ncols = global_block_cols(t.ngk, gb);
                const int nvalid = min(kBN, t.ngk - gb * kBN);
                need = c0 < nvalid;
                if (need) {
                    for (int a = 0; a < 32 && c0 + a < nvalid; ++a) {
                        const int diff = __ldg(gk + gb * kBN + c0 + a) - i;
                        const bool in_window = (diff % t.dil == 0) && diff <= reach && diff >= -reach;
                        if (!in_window) mk |= 1u << a;
                    }
                }
            }
            const bool full = __all_sync(0xffffffffu, mk == 0xffffffffu);

            // ---- this quarter of the S block
            if (!wait_warp(&bars[kBarSFull + sb], (blk_it >> 1) & 1u)) return;
            tc_fence_after();
            uint32_t sr[32];
            if (need) tmem_ld32(tmem_base + lane_off + col_s(sb) + 32u * qi, sr);
            tmem_ld_wait(sr);
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars[kBarSFree + sb]);

            float mx = -INFINITY;
            if (need) {
                float mxp[8];
#pragma unroll
                for (int u = 0; u < 8; ++u) mxp[u] = -INFINITY;
                if (full) {
#pragma unroll
                    for (int j = 0; j < 32; ++j) {
                        float f = __uint_as_float(sr[j]);
                        if (!POS) f *= sl2;
                        sr[j] = __float_as_uint(f);
                        mxp[j & 7] = fmaxf(mxp[j & 7], f);
                    }
                } else {
#pragma unroll
                    for (int j = 0; j < 32; ++j) {
                        float f = __uint_as_float(sr[j]);
                        if (!POS) f *= sl2;
                        f = ((mk >> j) & 1u) ? f : -INFINITY;
                        sr[j] = __float_as_uint(f);
                        mxp[j & 7] = fmaxf(mxp[j & 7], f);
                    }
                }
                mx = fmaxf(fmaxf(fmaxf(mxp[0], mxp[1]), fmaxf(mxp[2], mxp[3])),
                           fmaxf(fmaxf(mxp[4], mxp[5]), fmaxf(mxp[6], mxp[7])));
                if (POS) mx *= sl2;  // -inf stays -inf
            }
            m_run = fmaxf(m_run, mx);

            // ---- move this quarter's exponent base if its max ran past it (rare)
            float alpha = 1.f;
            bool move = (m_run != -INFINITY) && (m_ref == -INFINITY || m_run > m_ref + kRescaleLog2);
            if (blk == 0) {
                m_ref = m_run;  // the first product of the tile overwrites O_q
                move = false;
            } else if (move) {
                alpha = (m_ref == -INFINITY) ? 0.f : ex2_approx(m_ref - m_run);
                m_ref = m_run;
                l_q *= alpha;
            }
            if (__any_sync(0xffffffffu, move)) {
                if (!wait_pv(blk_it - 1)) return;  // O_q holds every earlier product
                tc_fence_after();
                uint32_t orr[32];
#pragma unroll 1
                for (int part = 0; part < 2; ++part) {
                    tmem_ld32(tOq + 32u * part, orr);
                    tmem_ld_wait(orr);
#pragma unroll
                    for (int c = 0; c < 32; ++c) orr[c] = __float_as_uint(__uint_as_float(orr[c]) * alpha);
                    tmem_st32(tOq + 32u * part, orr);
                }
                tmem_st_wait();
            }
            const float base = (m_ref == -INFINITY) ? 0.f : m_ref;

            // ---- p = 2^(s - base) as bf16 into P buffer sb (free once block blk_it - 2's product is done)
            uint32_t pk[16];
            float lsum[4] = {0.f, 0.f, 0.f, 0.f};
            if (need) {
#pragma unroll
                for (int j = 0; j < 32; j += 2) {
                    const float v0 = __uint_as_float(sr[j]), v1 = __uint_as_float(sr[j + 1]);
                    const float e0 = POS ? ex2_approx(fmaf(v0, sl2, -base)) : ex2_approx(v0 - base);
                    const float e1 = POS ? ex2_approx(fmaf(v1, sl2, -base)) : ex2_approx(v1 - base);
                    lsum[(j >> 1) & 3] += e0 + e1;
                    pk[j >> 1] = pack_bf16x2(e0, e1);
                }
            } else {
#pragma unroll
                for (int u = 0; u < 16; ++u) pk[u] = 0u;
            }
            l_q += (lsum[0] + lsum[1]) + (lsum[2] + lsum[3]);
            if (blk_it >= 2 && !wait_pv(blk_it - 2)) return;
            uint8_t* psub = smem + kOffP + sb * (2 * kTileBytes) + (qi >> 1) * kTileBytes + rowoff;
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                if (c0 + 8 * u < ncols) {
                    const int ch = ((qi & 1) << 2) + u;  // 16-byte chunk inside the 128-byte row
                    *reinterpret_cast<uint4*>(psub + ((ch ^ (x & 7)) << 4)) =
                        make_uint4(pk[4 * u], pk[4 * u + 1], pk[4 * u + 2], pk[4 * u + 3]);
                }
            }
            fence_proxy_async_smem();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars[kBarPFull + sb]);
        }

        // ---- epilogue: the four quarters swap (base, sum); this thread writes output
        //      columns [16 q, 16 q + 16) of its row (global rows are written by K2)
        float* slot = xm + (x_cnt & 1u) * (2 * 4 * kBM);
        slot[qi * kBM + x] = m_ref;
        slot[4 * kBM + qi * kBM + x] = l_q;
        __syncwarp();
        if (lane == 0) mbar_arrive(xbar);
        if (!wait_warp(xbar, x_cnt & 1u)) return;
        ++x_cnt;
        float mq[4], lq[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            mq[u] = slot[u * kBM + x];
            lq[u] = slot[4 * kBM + u * kBM + x];
        }
        const float M = fmaxf(fmaxf(mq[0], mq[1]), fmaxf(mq[2], mq[3]));
        float wgt[4], L = 0.f;
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            wgt[u] = (mq[u] == -INFINITY) ? 0.f : ex2_approx(mq[u] - M);
            L = fmaf(wgt[u], lq[u], L);
        }
        const float inv = L > 0.f ? 1.f / L : 0.f;
        if (!wait_pv(blk_it - 1)) return;
        tc_fence_after();
        float y[16];
#pragma unroll
        for (int c = 0; c < 16; ++c) y[c] = 0.f;
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            uint32_t a[16];
            tmem_ld16(tmem_base + lane_off + col_o(u) + 16u * qi, a);
            tmem_ld_wait16(a);
#pragma unroll
            for (int c = 0; c < 16; ++c) y[c] = fmaf(wgt[u], __uint_as_float(a[c]), y[c]);
        }
        tc_fence_before();
        if (row_ok) {
            uint4* dst = reinterpret_cast<uint4*>(p.out + (static_cast<size_t>(t.bh) * p.T + i) * kHD + 16 * qi);
#pragma unroll
            for (int v8 = 0; v8 < 2; ++v8) {
                uint4 val;
                val.x = pack_bf16x2(y[8 * v8 + 0] * inv, y[8 * v8 + 1] * inv);
                val.y = pack_bf16x2(y[8 * v8 + 2] * inv, y[8 * v8 + 3] * inv);
                val.z = pack_bf16x2(y[8 * v8 + 4] * inv, y[8 * v8 + 5] * inv);
                val.w = pack_bf16x2(y[8 * v8 + 6] * inv, y[8 * v8 + 7] * inv);
                dst[v8] = val;
            }
        }
    }
}

// --------------------------------------------------------------- MMA roles
// The MMA pipe accepts one tcgen05.mma every ~54 cycles at best, and an
// issuing thread shares its SM sub-partition with four softmax warps, so the
// work is split over three threads on three sub-partitions (S, and the two
// halves of the PV product), and the issue path is kept free of arithmetic:
// shared-memory descriptors are built once per stage / buffer and advanced
// by constants (the start-address field counts 16-byte units), k-loops are
// unrolled and the accumulate flags are literals.
constexpr uint64_t kTile16 = kTileBytes >> 4;  // one 16 KB tile in descriptor units

// S = Q K^T for every key block, in order.  The stage's K half is released
// by this thread's commit (one of three arrivals on the stage's empty
// barrier); V is released by the two product issuers.
__device__ __forceinline__ void mma_s_role(const BandTcParams& p, uint8_t* smem, uint64_t* bars,
                                           volatile int* abort_flag, uint32_t tmem_base) {
    const uint32_t idesc_s = idesc_bf16(kBM, kBN, 0, 0);
    const uint64_t dQ = sdesc_k_sw128(smem_u32(smem + kOffQ));
    uint64_t dK[kStages];
#pragma unroll
    for (int s = 0; s < kStages; ++s) dK[s] = sdesc_k_sw128(smem_u32(smem + kOffK + s * kTileBytes));
    uint32_t kv_it = 0, q_it = 0, blk_it = 0;
    bool alive = true;
    for (int item = blockIdx.x; item < p.n_items && alive; item += gridDim.x) {
        const BandTile t = band_decode(p, item);
        if (!mbar_wait(&bars[kBarQFull], q_it & 1u, abort_flag)) break;
        ++q_it;
        tc_fence_after();
        const int nb = t.nbb + t.ngb;
        for (int blk = 0; blk < nb; ++blk, ++blk_it, ++kv_it) {
            const uint32_t s = kv_it % kStages, ph = (kv_it / kStages) & 1u;
            const uint32_t sb = blk_it & 1u;
            if (!mbar_wait(&bars[kBarKvFull + s], ph, abort_flag) ||
                !mbar_wait(&bars[kBarSFree + sb], ((blk_it >> 1) & 1u) ^ 1u, abort_flag)) {
                alive = false;
                break;
            }
            tc_fence_after();
            const int ncols = blk < t.nbb ? kBN : global_block_cols(t.ngk, blk - t.nbb);
            const uint32_t ids = ncols == kBN ? idesc_s : idesc_bf16(kBM, ncols, 0, 0);
            uint64_t dKs = dK[0];
#pragma unroll
            for (int u = 1; u < kStages; ++u)
                if (s == static_cast<uint32_t>(u)) dKs = dK[u];
            const uint32_t dS = tmem_base + col_s(sb);
            tc_mma<false>(dS, dQ + 0, dKs + 0, ids);  // K-steps of 16 (32 bytes = 2 units)
            tc_mma<true>(dS, dQ + 2, dKs + 2, ids);
            tc_mma<true>(dS, dQ + 4, dKs + 4, ids);
            tc_mma<true>(dS, dQ + 6, dKs + 6, ids);
            tc_commit(&bars[kBarSFull + sb]);
            tc_commit(&bars[kBarKvEmpty + s]);
            if (blk == nb - 1) tc_commit(&bars[kBarQEmpty]);
        }
    }
    tc_commit(&bars[kBarDrain]);
}

// O_q += P V for every key block, k-steps 4*half .. 4*half+3 (accumulators
// O_{2 half}, O_{2 half + 1}).  Two of these threads run, one per half.
__device__ __forceinline__ void mma_pv_role(const BandTcParams& p, uint8_t* smem, uint64_t* bars,
                                            volatile int* abort_flag, uint32_t tmem_base, int half) {
    const uint32_t idesc_pv = idesc_bf16(kBM, kHD, 0, 1);
    uint64_t dV[kStages];
#pragma unroll
    for (int s = 0; s < kStages; ++s) dV[s] = sdesc_mn_sw128(smem_u32(smem + kOffV + s * kTileBytes));
    // P sub-tile `half` holds keys 64 half .. 64 half + 63
    const uint64_t dP0 = sdesc_k_sw128(smem_u32(smem + kOffP)) + half * kTile16;
    const uint32_t t_o = tmem_base + col_o(2 * half);
    const int ks0 = 4 * half;
    uint32_t kv_it = 0, blk_it = 0;
    bool alive = true;
    for (int item = blockIdx.x; item < p.n_items && alive; item += gridDim.x) {
        const BandTile t = band_decode(p, item);
        const int nb = t.nbb + t.ngb;
        for (int blk = 0; blk < nb; ++blk, ++blk_it, ++kv_it) {
            const uint32_t s = kv_it % kStages;
            const uint32_t pb = blk_it & 1u;
            if (!mbar_wait(&bars[kBarPFull + pb], (blk_it >> 1) & 1u, abort_flag)) {
                alive = false;
                break;
            }
            tc_fence_after();
            const int nk = blk < t.nbb ? kBN : global_block_cols(t.ngk, blk - t.nbb);
            const uint64_t dP = dP0 + pb * (2 * kTile16);
            uint64_t dVs = dV[0];
#pragma unroll
            for (int u = 1; u < kStages; ++u)
                if (s == static_cast<uint32_t>(u)) dVs = dV[u];
            dVs += ks0 * 128;  // 16 keys x 128 bytes per k-step
            if (nk == kBN) {
                if (blk == 0) {  // the first product of a tile overwrites the accumulators
                    tc_mma<false>(t_o, dP + 0, dVs + 0, idesc_pv);
                    tc_mma<true>(t_o, dP + 2, dVs + 128, idesc_pv);
                    tc_mma<false>(t_o + 64u, dP + 4, dVs + 256, idesc_pv);
                    tc_mma<true>(t_o + 64u, dP + 6, dVs + 384, idesc_pv);
                } else {
                    tc_mma<true>(t_o, dP + 0, dVs + 0, idesc_pv);
                    tc_mma<true>(t_o, dP + 2, dVs + 128, idesc_pv);
                    tc_mma<true>(t_o + 64u, dP + 4, dVs + 256, idesc_pv);
                    tc_mma<true>(t_o + 64u, dP + 6, dVs + 384, idesc_pv);
                }
            } else {  // a partial block of global keys (never the first block of a tile)
                for (int k = 0; k < 4 && ks0 + k < nk / 16; ++k)
                    tc_mma<true>(t_o + 64u * (k >> 1), dP + 2 * k, dVs + 128 * k, idesc_pv);
            }
            tc_commit(&bars[kBarOFull + pb]);
            tc_commit(&bars[kBarKvEmpty + s]);
        }
    }
    tc_commit(&bars[kBarDrain]);
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
            mbar_init(&bars[kBarKvEmpty + s], 3);  // S issuer + two PV issuers
        }
        for (int s = 0; s < 2; ++s) {
            mbar_init(&bars[kBarSFull + s], 1);
            mbar_init(&bars[kBarSFree + s], kSoftmaxWarps);
            mbar_init(&bars[kBarPFull + s], kSoftmaxWarps);
            mbar_init(&bars[kBarOFull + s], 2);  // two PV issuers
        }
        for (int w = 0; w < 4; ++w) mbar_init(&bars[kBarXchg + w], 4);
        mbar_init(&bars[kBarDrain], 3);
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
        if (lane == 0) mma_s_role(p, smem, bars, abort_flag, tmem_base);
    } else if (warp < kSoftmaxWarp0) {
        if (lane == 0) mma_pv_role(p, smem, bars, abort_flag, tmem_base, warp - 2);
    } else {
        if (p.sl2 > 0.f)
            softmax_role<true>(p, smem, bars, abort_flag, tmem_base);
        else
            softmax_role<false>(p, smem, bars, abort_flag, tmem_base);
    }

    tc_fence_before();
    __syncthreads();
    // every MMA of the three issuers has completed before TMEM is released
    if (threadIdx.x == 32) (void)mbar_wait_drain(&bars[kBarDrain], 0u);
    __syncthreads();
    if (threadIdx.x == 0 && *abort_flag) atomicOr(p.status, kStatusTimeout);
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, kTmemCols);
    }
}

}  // namespace lf
