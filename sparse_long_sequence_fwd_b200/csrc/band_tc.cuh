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
//                                   count rounded to 16), K=64, operands in
//                                   shared memory -> S in TMEM (fp32)
//                  online softmax   one thread per query row (TMEM lane),
//                                   the block read in four 32-column chunks;
//                                   running max, exponent base and row sum
//                                   in fp32, log2 domain
//                  O += P V         P (bf16) written back to TMEM by the
//                                   softmax threads and read from there as
//                                   the A operand; V from shared memory;
//                                   M=128, N=64, K=128
// The exponent base only moves (O and the row sum rescaled in place) between
// blocks, when the max seen exceeds it by more than 2^8; otherwise
// p = 2^(s - base) stays below 256, which fp32 accumulation and bf16 P absorb
// (a jump of more than 2^64 inside a block is handled at once, see the
// softmax role).
// The mask view of the note ("Mask View": A = QK^T/sqrt(d) + M, M = -inf off
// the pattern) is applied inline: band limits and sequence ends as a per-row
// column interval, padded keys from the key padding mask, the global-key
// dedup test per column.  Blocks that lie inside every row's window need no
// test at all.  Nothing of size T x T is built.
//
// Two CTAs share an SM (96 KB of shared memory and 256 TMEM columns each):
// while one CTA's softmax warps wait on a barrier or a TMEM load, the
// other's keep the exponent unit busy.  Warp roles (192 threads): warp 0
// lane 0 TMA producer, warp 1 TMEM owner and lane 0 MMA issuer, warps 2..5
// softmax (TMEM lanes 32*(w%4)..+31).  Every hand-off is an mbarrier and
// every wait is bounded (ptx.cuh).
#pragma once
#include "lf_common.cuh"
#include "ptx.cuh"

namespace lf {

constexpr int kBM = 128;
constexpr int kBN = 128;
constexpr int kHD = 64;
constexpr int kStages = 2;                 // Q, K and V rings
constexpr int kTileBytes = kBM * kHD * 2;  // 16 KB: 128 rows x 128 bytes
constexpr int kBandThreads = 192;
constexpr int kBandCtasPerSm = 2;
constexpr int kSoftmaxWarp0 = 2;  // warps 2..5
constexpr int kSoftmaxWarps = 4;
constexpr float kRescaleLog2 = 8.f;  // move the exponent base only past 2^8

constexpr int kOffQ = 0;
constexpr int kOffK = kOffQ + kStages * kTileBytes;
constexpr int kOffV = kOffK + kStages * kTileBytes;
constexpr int kOffBar = kOffV + kStages * kTileBytes;
// barrier slots
constexpr int kBarQFull = 0, kBarQEmpty = kBarQFull + kStages, kBarKFull = kBarQEmpty + kStages,
              kBarKEmpty = kBarKFull + kStages, kBarVFull = kBarKEmpty + kStages, kBarVEmpty = kBarVFull + kStages,
              kBarSFull = kBarVEmpty + kStages, kBarSFree = kBarSFull + 1, kBarPFull = kBarSFree + 1,
              kBarOFull = kBarPFull + 1, kBarDrain = kBarOFull + 1, kNumBars = kBarDrain + 1;
// Tile descriptors (BandTile), one per Q slot: written by the producer before
// it arrives on the slot's Q-full barrier, read by the MMA and softmax roles
// after waiting on it, so only the producer decodes work items.
constexpr int kOffDesc = kOffBar + ((kNumBars * 8 + 15) / 16) * 16;
constexpr int kDescBytes = 64;
constexpr int kOffMisc = kOffDesc + kStages * kDescBytes;
constexpr int kMiscBytes = 16;
constexpr int kBandSmem = kOffMisc + kMiscBytes + 1024;  // + alignment slack
static_assert(kBandCtasPerSm * (kBandSmem + 1024) <= 233472, "shared memory budget for two CTAs per SM");

// TMEM columns (256 per CTA): S (fp32, 128 wide) at 0, P (bf16 pairs, 64
// wide) at 128, O (fp32, 64 wide) at 192.
constexpr uint32_t kTmemCols = 256;
constexpr uint32_t kColS = 0, kColP = 128, kColO = 192;

struct BandTile {
    int b, bh, c, dil, dk, R;
    int Tc, q0, kbase, kb_lo, nbb, ngk, ngb;
};
static_assert(sizeof(BandTile) <= kDescBytes, "tile descriptor slot");

// Out of line: every role walks the same tiles, and one copy of this code
// (integer divisions included) keeps the kernel small.
__device__ __noinline__ BandTile band_decode(const BandTcParams& p, int item) {
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

__device__ __forceinline__ float fmin3(float a, float b, float c) {
    float d;
    asm("min.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
    return d;
}
__device__ __forceinline__ float fmax3(float a, float b, float c) {
    float d;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
    return d;
}

// Work item of a slot: the CTA with blockIdx b takes slots b, b + grid, ...;
// the host may order the items so the longest tiles come first.
__device__ __forceinline__ int slot_item(const BandTcParams& p, int slot) {
    return p.item_order ? __ldg(p.item_order + slot) : slot;
}

// Walks the (slot, block) sequence of this CTA in the order every role uses.
struct BlockCursor {
    int item, blk, nb;
    BandTile t;
    __device__ __forceinline__ void start(const BandTcParams& p) {
        item = blockIdx.x;
        blk = 0;
        if (item < p.n_items) {
            t = band_decode(p, slot_item(p, item));
            nb = t.nbb + t.ngb;
        } else {
            nb = 0;
        }
    }
    __device__ __forceinline__ bool valid(const BandTcParams& p) const { return item < p.n_items; }
    __device__ __forceinline__ void next(const BandTcParams& p) {
        if (++blk < nb) return;
        blk = 0;
        item += gridDim.x;
        if (item < p.n_items) {
            t = band_decode(p, slot_item(p, item));
            nb = t.nbb + t.ngb;
        }
    }
};

// ------------------------------------------------------------- TMA producer
// K runs one block ahead of V: K(g + 1) is needed as soon as the softmax has
// read S(g), V(g) only once P(g) is written.
__device__ __forceinline__ void producer_role(const BandTcParams& p, uint8_t* smem, uint64_t* bars,
                                              volatile int* abort_flag) {
    BlockCursor kc, vc;
    kc.start(p);
    vc.start(p);
    uint32_t gk = 0, gv = 0, qt = 0;
    auto issue_k = [&]() -> bool {
        const BandTile& t = kc.t;
        if (kc.blk == 0) {
            const uint32_t qs = qt & 1u;
            if (!mbar_wait(&bars[kBarQEmpty + qs], ((qt >> 1) & 1u) ^ 1u, abort_flag)) return false;
            *reinterpret_cast<BandTile*>(smem + kOffDesc + qs * kDescBytes) = t;  // released by the arrive
            mbar_arrive_expect_tx(&bars[kBarQFull + qs], kTileBytes);
            uint8_t* dQ = smem + kOffQ + qs * kTileBytes;
            for (int u = 0; u < kBM; u += t.R)
                tma_load_3d(dQ + u * 128, &p.tm_q[t.dk], &bars[kBarQFull + qs], 0, t.c + t.dil * (t.q0 + u), t.bh);
            ++qt;
        }
        const uint32_t s = gk & 1u;
        if (!mbar_wait(&bars[kBarKEmpty + s], ((gk >> 1) & 1u) ^ 1u, abort_flag)) return false;
        mbar_arrive_expect_tx(&bars[kBarKFull + s], kTileBytes);
        uint8_t* dK = smem + kOffK + s * kTileBytes;
        if (kc.blk < t.nbb) {
            const int j0 = t.kbase + kBN * (t.kb_lo + kc.blk);
            for (int u = 0; u < kBN; u += t.R)
                tma_load_3d(dK + u * 128, &p.tm_k[t.dk], &bars[kBarKFull + s], 0, t.c + t.dil * (j0 + u), t.bh);
        } else {
            tma_load_3d(dK, &p.tm_kg, &bars[kBarKFull + s], 0, (kc.blk - t.nbb) * kBN, t.bh);
        }
        ++gk;
        return true;
    };
    auto issue_v = [&]() -> bool {
        const BandTile& t = vc.t;
        const uint32_t s = gv & 1u;
        if (!mbar_wait(&bars[kBarVEmpty + s], ((gv >> 1) & 1u) ^ 1u, abort_flag)) return false;
        mbar_arrive_expect_tx(&bars[kBarVFull + s], kTileBytes);
        uint8_t* dV = smem + kOffV + s * kTileBytes;
        if (vc.blk < t.nbb) {
            const int j0 = t.kbase + kBN * (t.kb_lo + vc.blk);
            for (int u = 0; u < kBN; u += t.R)
                tma_load_3d(dV + u * 128, &p.tm_v[t.dk], &bars[kBarVFull + s], 0, t.c + t.dil * (j0 + u), t.bh);
        } else {
            tma_load_3d(dV, &p.tm_vg, &bars[kBarVFull + s], 0, (vc.blk - t.nbb) * kBN, t.bh);
        }
        ++gv;
        return true;
    };
    bool first = true;
    while (vc.valid(p)) {  // K(0); then K(g + 1), V(g) for g = 0, 1, ...
        if (kc.valid(p)) {
            if (!issue_k()) break;
            kc.next(p);
            if (first) {
                first = false;
                continue;
            }
        }
        if (!issue_v()) break;
        vc.next(p);
    }
    if (*abort_flag) {  // let issued copies land before the CTA can exit
        for (uint32_t s = 0; s < kStages; ++s) {
            if (gk > s) (void)mbar_wait_drain(&bars[kBarKFull + s], ((gk - 1 - s) >> 1) & 1u);
            if (gv > s) (void)mbar_wait_drain(&bars[kBarVFull + s], ((gv - 1 - s) >> 1) & 1u);
            if (qt > s) (void)mbar_wait_drain(&bars[kBarQFull + s], ((qt - 1 - s) >> 1) & 1u);
        }
    }
}

// --------------------------------------------------------------- MMA issuer
// S(g) = Q K(g)^T as soon as K(g) has landed and the softmax has read S(g-1);
// then O += P(g-1) V(g-1) once P(g-1) is in TMEM.  The MMA pipe accepts one
// tcgen05.mma every ~54-64 cycles, 12 per block: well inside the exponent
// unit's ~1000 cycles per block, so one issuing thread is enough.
__device__ __forceinline__ void mma_role(const BandTcParams& p, uint8_t* smem, uint64_t* bars,
                                         volatile int* abort_flag, uint32_t tmem_base) {
    const uint32_t idesc_s = idesc_bf16(kBM, kBN, 0, 0);
    const uint32_t idesc_pv = idesc_bf16(kBM, kHD, 0, 1);
    uint64_t dQ[kStages], dK[kStages], dV[kStages];
#pragma unroll
    for (int s = 0; s < kStages; ++s) {
        dQ[s] = sdesc_k_sw128(smem_u32(smem + kOffQ + s * kTileBytes));
        dK[s] = sdesc_k_sw128(smem_u32(smem + kOffK + s * kTileBytes));
        dV[s] = sdesc_mn_sw128(smem_u32(smem + kOffV + s * kTileBytes));
    }
    const uint32_t tS = tmem_base + kColS, tP = tmem_base + kColP, tO = tmem_base + kColO;

    // O += P(g) V(g) over nk keys; the first block of a tile overwrites O
    auto issue_pv = [&](uint32_t g, int nk, bool first) -> bool {
        const uint32_t s = g & 1u;
        if (!mbar_wait(&bars[kBarPFull], g & 1u, abort_flag) ||
            !mbar_wait(&bars[kBarVFull + s], (g >> 1) & 1u, abort_flag))
            return false;
        tc_fence_after();
        const uint64_t dv = dV[s];
        if (nk == kBN) {
            if (first)
                tc_mma_ts<false>(tO, tP + 0, dv + 0, idesc_pv);
            else
                tc_mma_ts<true>(tO, tP + 0, dv + 0, idesc_pv);
#pragma unroll
            for (int k = 1; k < 8; ++k) tc_mma_ts<true>(tO, tP + 8u * k, dv + 128u * k, idesc_pv);
        } else {  // a partial block of global keys (never the first block of a tile)
            for (int k = 0; k < nk / 16; ++k) tc_mma_ts<true>(tO, tP + 8u * k, dv + 128u * k, idesc_pv);
        }
        tc_commit(&bars[kBarOFull]);
        tc_commit(&bars[kBarVEmpty + s]);
        return true;
    };

    uint32_t g = 0, qt = 0, qs = 0;
    int item = blockIdx.x, blk = 0, nb = 0, nbb = 0, ngk = 0;
    int prev_nk = 0;
    bool prev_first = false;
    for (;;) {  // S(g), then the product of block g - 1
        const bool have = item < p.n_items;
        int cur_nk = 0;
        bool cur_first = false;
        if (have) {
            if (blk == 0) {  // the tile's Q has landed and its descriptor is visible
                qs = qt & 1u;
                if (!mbar_wait(&bars[kBarQFull + qs], (qt >> 1) & 1u, abort_flag)) break;
                ++qt;
                const BandTile* d = reinterpret_cast<const BandTile*>(smem + kOffDesc + qs * kDescBytes);
                nbb = d->nbb;
                ngk = d->ngk;
                nb = nbb + d->ngb;
            }
            const uint32_t s = g & 1u;
            if (!mbar_wait(&bars[kBarKFull + s], (g >> 1) & 1u, abort_flag) ||
                (g > 0 && !mbar_wait(&bars[kBarSFree], (g - 1) & 1u, abort_flag)))
                break;
            tc_fence_after();
            const int ncols = blk < nbb ? kBN : global_block_cols(ngk, blk - nbb);
            const uint32_t ids = ncols == kBN ? idesc_s : idesc_bf16(kBM, ncols, 0, 0);
            const uint64_t dq = dQ[qs], dk = dK[s];
            tc_mma<false>(tS, dq + 0, dk + 0, ids);  // K-steps of 16 (32 bytes = 2 units)
            tc_mma<true>(tS, dq + 2, dk + 2, ids);
            tc_mma<true>(tS, dq + 4, dk + 4, ids);
            tc_mma<true>(tS, dq + 6, dk + 6, ids);
            tc_commit(&bars[kBarSFull]);
            tc_commit(&bars[kBarKEmpty + s]);
            if (blk == nb - 1) tc_commit(&bars[kBarQEmpty + qs]);
            cur_nk = ncols;
            cur_first = blk == 0;
        }
        if (g > 0 && !issue_pv(g - 1, prev_nk, prev_first)) break;
        if (!have) break;
        prev_nk = cur_nk;
        prev_first = cur_first;
        ++g;
        if (++blk == nb) {
            blk = 0;
            item += gridDim.x;
        }
    }
    tc_commit(&bars[kBarDrain]);
}

// ------------------------------------------------------------ softmax role
// Thread x owns query row x of the tile (TMEM lane x) and walks each S block
// in four chunks of 32 columns, one loop body for all of them: TMEM load,
// mask, max, exponentials, P (16 columns of bf16 pairs) back to TMEM, so
// only one chunk of S is held in registers.
//
// Exponent base.  p = 2^(s*sl2 - base) with base = m_ref.  The base moves
// between blocks, to the largest scaled score seen so far, once that exceeds
// it by more than 2^8 (O and the row sum are rescaled then; the O rescale
// needs the previous product to have finished, which the P store waits for
// anyway).  Inside a block the base stays put unless a chunk's max exceeds
// it by more than 2^64, so p < 2^64 and fp32 sums stay finite; that rare
// jump rescales O and the P chunks already stored.
constexpr float kBigJumpLog2 = 64.f;

// Multiplies the first nchunks P chunks (16 columns of bf16 pairs each) of
// this thread's row by alpha, in TMEM.
__device__ __forceinline__ void rescale_p_chunks(uint32_t tP, int nchunks, float alpha) {
    tmem_st_wait();  // this thread's own stores have landed
#pragma unroll 1
    for (int c = 0; c < nchunks; ++c) {
        uint32_t pr[16];
        tmem_ld16(tP + 16u * c, pr);
        tmem_ld_wait16(pr);
#pragma unroll
        for (int u = 0; u < 16; ++u) {
            __nv_bfloat162 h = *reinterpret_cast<__nv_bfloat162*>(&pr[u]);
            const float2 f = __bfloat1622float2(h);
            pr[u] = pack_bf16x2(f.x * alpha, f.y * alpha);
        }
        tmem_st16(tP + 16u * c, pr);
    }
}

// Multiplies this thread's row of O (64 fp32 columns) by alpha, in TMEM.
__device__ __noinline__ void rescale_o(uint32_t tO, float alpha) {
#pragma unroll 1
    for (int part = 0; part < 4; ++part) {
        uint32_t orr[16];
        tmem_ld16(tO + 16u * part, orr);
        tmem_ld_wait16(orr);
#pragma unroll
        for (int c = 0; c < 16; ++c) orr[c] = __float_as_uint(__uint_as_float(orr[c]) * alpha);
        tmem_st16(tO + 16u * part, orr);
    }
}

// Writes this thread's output row, y = O * inv as bf16 (dst null: row not
// written), from TMEM.  Once per tile, out of line.
__device__ __noinline__ void write_rows(uint32_t tO, uint4* dst, float inv) {
#pragma unroll 1
    for (int part = 0; part < 4; ++part) {
        uint32_t o[16];
        tmem_ld16(tO + 16u * part, o);
        tmem_ld_wait16(o);
        if (dst) {
            uint4 v0, v1;
            v0.x = pack_bf16x2(__uint_as_float(o[0]) * inv, __uint_as_float(o[1]) * inv);
            v0.y = pack_bf16x2(__uint_as_float(o[2]) * inv, __uint_as_float(o[3]) * inv);
            v0.z = pack_bf16x2(__uint_as_float(o[4]) * inv, __uint_as_float(o[5]) * inv);
            v0.w = pack_bf16x2(__uint_as_float(o[6]) * inv, __uint_as_float(o[7]) * inv);
            v1.x = pack_bf16x2(__uint_as_float(o[8]) * inv, __uint_as_float(o[9]) * inv);
            v1.y = pack_bf16x2(__uint_as_float(o[10]) * inv, __uint_as_float(o[11]) * inv);
            v1.z = pack_bf16x2(__uint_as_float(o[12]) * inv, __uint_as_float(o[13]) * inv);
            v1.w = pack_bf16x2(__uint_as_float(o[14]) * inv, __uint_as_float(o[15]) * inv);
            dst[2 * part] = v0;
            dst[2 * part + 1] = v1;
        }
    }
}

// Rare path of a score jump inside a block: multiplies the first nchunks P
// chunks of this thread's row, and (with_o) its row of O, by alpha, in TMEM.
__device__ __noinline__ void rescale_held(uint32_t tP, int nchunks, uint32_t tO, bool with_o, float alpha) {
    rescale_p_chunks(tP, nchunks, alpha);
    if (with_o) rescale_o(tO, alpha);
}

__device__ __forceinline__ uint32_t pick4(const uint32_t* v, int c) {
    return c == 0 ? v[0] : (c == 1 ? v[1] : (c == 2 ? v[2] : v[3]));
}

__device__ __forceinline__ void softmax_role(const BandTcParams& p, uint8_t* smem, uint64_t* bars,
                                             volatile int* abort_flag, uint32_t tmem_base) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int wq = warp & 3;
    const int x = wq * 32 + lane;  // query row inside the tile = TMEM lane
    const uint32_t lane_off = static_cast<uint32_t>(wq * 32) << 16;
    const uint32_t tS = tmem_base + lane_off + kColS;
    const uint32_t tP = tmem_base + lane_off + kColP;
    const uint32_t tO = tmem_base + lane_off + kColO;
    // scale >= 0: maxima on raw scores (masked columns -inf); scale < 0: minima
    // (masked columns +inf); either way the scale is folded into the exp2 FMA
    const bool pos = p.sl2 >= 0.f;
    const float kmul = p.sl2 == 0.f ? 1e-30f : p.sl2;
    const uint32_t fill = __float_as_uint(pos ? -INFINITY : INFINITY);
    uint32_t g = 0;

    // every lane polls (each lane's own acquire), then the warp agrees on the outcome
    auto wait_warp = [&](uint64_t* bar, uint32_t parity) -> bool {
        const bool ok = mbar_wait(bar, parity, abort_flag);
        return __all_sync(0xffffffffu, ok);
    };

    // The output row of a finished tile is written once the product that
    // completes its O is done, which the first P store of the next tile (or
    // the end of the role) waits for anyway.
    bool pend = false, pend_ok = false;
    float pend_inv = 0.f;
    uint4* pend_dst = nullptr;
    auto flush = [&]() {
        if (!pend) return;
        pend = false;
        write_rows(tO, pend_ok ? pend_dst : nullptr, pend_inv);
    };

    uint32_t qt = 0;
    for (int item = blockIdx.x; item < p.n_items; item += gridDim.x) {
        // the tile's descriptor, published by the producer with its Q tile
        const uint32_t qs = qt & 1u;
        if (!wait_warp(&bars[kBarQFull + qs], (qt >> 1) & 1u)) return;
        ++qt;
        const BandTile t = *reinterpret_cast<const BandTile*>(smem + kOffDesc + qs * kDescBytes);
        const int ip = t.q0 + x;         // decimated row index
        const int i = t.c + t.dil * ip;  // position in the sequence
        // global-row bitmap word of this row; consumed only when the tile's rows are written
        const uint32_t gbw = ip < t.Tc ? __ldg(p.gbit + static_cast<size_t>(t.b) * p.W + (i >> 5)) : 0u;
        const int32_t* gk = p.gk_list + static_cast<size_t>(t.b) * p.gstride;
        const int reach = t.dil * p.r;
        // the first block of global keys, one key per lane and chunk, fetched early
        uint32_t kreg[4] = {0u, 0u, 0u, 0u};
        if (t.ngb > 0) {
#pragma unroll
            for (int w = 0; w < 4; ++w)
                if (32 * w + lane < t.ngk) kreg[w] = static_cast<uint32_t>(__ldg(gk + 32 * w + lane));
        }

        float m_ref = -INFINITY;   // exponent base (scaled, log2 domain; -inf: nothing valid yet)
        float m_seen = -INFINITY;  // largest scaled score seen so far
        float l_row = 0.f;         // row sum relative to m_ref
        const int nb = t.nbb + t.ngb;
        for (int blk = 0; blk < nb; ++blk, ++g) {
            // ---- which columns this row keeps: band blocks inside every row's window and
            //      inside [0, Tc) need no test (128 kb + y - x lies in [0, 2r] for all x, y)
            const bool band = blk < t.nbb;
            const int kb = t.kb_lo + blk;
            const int j0 = t.kbase + kBN * kb;
            const bool interior =
                band && !p.pad && kb >= 1 && kBN * kb + kBN - 1 <= 2 * p.r && j0 >= 0 && j0 + kBN <= t.Tc;
            const int ylo = max(max(0, x - kBN * kb), -j0);  // band: kept columns [ylo, yhi)
            const int yhi = min(min(kBN, x + 2 * p.r + 1 - kBN * kb), t.Tc - j0);
            uint32_t padv[4] = {0u, 0u, 0u, 0u};  // band: key padding of column 32 w + lane
            int nch = 4, nvalid = kBN;
            if (band) {
                if (p.pad) {
#pragma unroll
                    for (int w = 0; w < 4; ++w) {
                        const int jd = j0 + 32 * w + lane;
                        if (jd >= 0 && jd < t.Tc)
                            padv[w] = p.pad[static_cast<size_t>(t.b) * p.T + t.c + static_cast<size_t>(t.dil) * jd];
                    }
                }
            } else {
                const int gb = blk - t.nbb;
                nvalid = min(kBN, t.ngk - gb * kBN);
                nch = (nvalid + 31) >> 5;
                if (gb > 0) {
#pragma unroll
                    for (int w = 0; w < 4; ++w)
                        kreg[w] = 32 * w + lane < nvalid ? static_cast<uint32_t>(__ldg(gk + gb * kBN + 32 * w + lane)) : 0u;
                }
            }

            // ---- deferred base move (decided on the blocks before this one)
            float alpha_o = 1.f;
            const bool o_move = m_ref != -INFINITY && m_seen > m_ref + kRescaleLog2;
            if (o_move) {
                alpha_o = ex2_approx(m_ref - m_seen);
                m_ref = m_seen;
                l_row *= alpha_o;
            }
            const bool warp_o_move = __any_sync(0xffffffffu, o_move);
            // P may be overwritten (and O touched) once the previous product is done
            bool p_ready = false;
            auto ensure_p_ready = [&]() -> bool {
                if (p_ready) return true;
                if (g > 0) {
                    if (!wait_warp(&bars[kBarOFull], (g - 1) & 1u)) return false;
                    tc_fence_after();
                }
                flush();
                if (warp_o_move) rescale_o(tO, alpha_o);
                p_ready = true;
                return true;
            };

            if (!wait_warp(&bars[kBarSFull], g & 1u)) return;
            tc_fence_after();
            float lsum[4] = {0.f, 0.f, 0.f, 0.f};
            // one body for every chunk: a second copy (for a load in flight during the
            // previous chunk) costs more in instruction fetch than it hides
#pragma unroll 1
            for (int c = 0; c < nch; ++c) {
                uint32_t cur[32];
                tmem_ld32(tS + 32u * c, cur);
                tmem_ld_wait(cur);
                if (c + 1 == nch) {  // the whole S block has been read: the MMA may overwrite it
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&bars[kBarSFree]);
                }
                if (!interior) {
                    uint32_t m;
                    if (band) {
                        m = range_bits(ylo - 32 * c, yhi - 32 * c);
                        if (p.pad) m &= ~__ballot_sync(0xffffffffu, pick4(padv, c) != 0u);
                    } else {  // global keys not already in the row's window
                        m = 0u;
                        const uint32_t kc = pick4(kreg, c);
                        const int na = min(32, nvalid - 32 * c);
#pragma unroll 1
                        for (int a = 0; a < na; ++a) {
                            const int diff = static_cast<int>(__shfl_sync(0xffffffffu, kc, a)) - i;
                            const bool in_window =
                                diff <= reach && diff >= -reach && (t.dil == 1 || diff % t.dil == 0);
                            m |= in_window ? 0u : (1u << a);
                        }
                    }
                    if (!__all_sync(0xffffffffu, m == 0xffffffffu)) {  // only chunks some row masks
#pragma unroll
                        for (int j = 0; j < 32; ++j)
                            if (!((m >> j) & 1u)) cur[j] = fill;
                    }
                }
                float mx;
                if (pos) {
                    float mxp[4];
#pragma unroll
                    for (int u = 0; u < 4; ++u) mxp[u] = fmaxf(__uint_as_float(cur[2 * u]), __uint_as_float(cur[2 * u + 1]));
#pragma unroll
                    for (int j = 8; j < 32; j += 8)
#pragma unroll
                        for (int u = 0; u < 4; ++u)
                            mxp[u] = fmax3(mxp[u], __uint_as_float(cur[j + 2 * u]), __uint_as_float(cur[j + 2 * u + 1]));
                    mx = fmaxf(fmaxf(mxp[0], mxp[1]), fmaxf(mxp[2], mxp[3]));
                } else {
                    float mnp[4];
#pragma unroll
                    for (int u = 0; u < 4; ++u) mnp[u] = fminf(__uint_as_float(cur[2 * u]), __uint_as_float(cur[2 * u + 1]));
#pragma unroll
                    for (int j = 8; j < 32; j += 8)
#pragma unroll
                        for (int u = 0; u < 4; ++u)
                            mnp[u] = fmin3(mnp[u], __uint_as_float(cur[j + 2 * u]), __uint_as_float(cur[j + 2 * u + 1]));
                    mx = fminf(fminf(mnp[0], mnp[1]), fminf(mnp[2], mnp[3]));
                }
                mx *= kmul;  // the largest scaled score of the chunk (-inf if none is kept)
                m_seen = fmaxf(m_seen, mx);
                if (m_ref == -INFINITY) m_ref = mx;  // everything so far had zero weight
                const bool big = mx > m_ref + kBigJumpLog2;
                if (__any_sync(0xffffffffu, big)) {  // rare: rescale what this block already holds
                    const float alpha = big ? ex2_approx(m_ref - mx) : 1.f;
                    if (big) {
                        m_ref = mx;
                        l_row *= alpha;
                        lsum[0] *= alpha;
                        lsum[1] *= alpha;
                        lsum[2] *= alpha;
                        lsum[3] *= alpha;
                    }
                    if (c > 0 || blk > 0) {
                        if (!ensure_p_ready()) return;
                        rescale_held(tP, c, tO, blk > 0, alpha);
                    }
                }
                const float nb2 = (m_ref == -INFINITY) ? 0.f : -m_ref;
                uint32_t pk[16];
#pragma unroll
                for (int j = 0; j < 32; j += 2) {
                    const float e0 = ex2_approx(fmaf(__uint_as_float(cur[j]), kmul, nb2));
                    const float e1 = ex2_approx(fmaf(__uint_as_float(cur[j + 1]), kmul, nb2));
                    lsum[(j >> 1) & 3] += e0 + e1;
                    pk[j >> 1] = pack_bf16x2(e0, e1);
                }
                // the previous product is waited for only here, after chunk 0's work
                if (c == 0 && !ensure_p_ready()) return;
                tmem_st16(tP + 16u * c, pk);
            }
            l_row += (lsum[0] + lsum[1]) + (lsum[2] + lsum[3]);
            tmem_st_wait();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars[kBarPFull]);
        }
        // ---- this tile's rows: y = O / l, written once its last product is done
        pend = true;
        pend_ok = ip < t.Tc && !((gbw >> (i & 31)) & 1u);
        pend_inv = l_row > 0.f ? 1.f / l_row : 0.f;
        pend_dst = reinterpret_cast<uint4*>(p.out + (static_cast<size_t>(t.bh) * p.T + i) * kHD);
    }
    if (g > 0) {
        if (!wait_warp(&bars[kBarOFull], (g - 1) & 1u)) return;
        tc_fence_after();
        flush();
    }
}

__global__ void __launch_bounds__(kBandThreads, kBandCtasPerSm) band_tc_kernel(const __grid_constant__ BandTcParams p) {
    extern __shared__ uint8_t band_smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(band_smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kOffBar);
    uint32_t* misc = reinterpret_cast<uint32_t*>(smem + kOffMisc);
    uint32_t* tmem_slot = misc;
    volatile int* abort_flag = reinterpret_cast<volatile int*>(misc + 1);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&bars[kBarQFull + s], 1);
            mbar_init(&bars[kBarQEmpty + s], 1);
            mbar_init(&bars[kBarKFull + s], 1);
            mbar_init(&bars[kBarKEmpty + s], 1);
            mbar_init(&bars[kBarVFull + s], 1);
            mbar_init(&bars[kBarVEmpty + s], 1);
        }
        mbar_init(&bars[kBarSFull], 1);
        mbar_init(&bars[kBarSFree], kSoftmaxWarps);
        mbar_init(&bars[kBarPFull], kSoftmaxWarps);
        mbar_init(&bars[kBarOFull], 1);
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
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    // the set-up above may overlap the prep kernel; its lists and packed keys are read below
    grid_dep_wait();

    if (warp == 0) {
        if (lane == 0) producer_role(p, smem, bars, abort_flag);
    } else if (warp == 1) {
        if (lane == 0) mma_role(p, smem, bars, abort_flag, tmem_base);
    } else {
        softmax_role(p, smem, bars, abort_flag, tmem_base);
    }

    tc_fence_before();
    __syncthreads();
    // every MMA has completed before TMEM is released
    if (threadIdx.x == 32) (void)mbar_wait_drain(&bars[kBarDrain], 0u);
    __syncthreads();
    if (threadIdx.x == 0 && *abort_flag) atomicOr(p.status, kStatusTimeout);
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, kTmemCols);
    }
}

}  // namespace lf
