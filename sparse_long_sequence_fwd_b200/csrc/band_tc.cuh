// band_tc.cuh -- K1: fused band kernel for bf16, d = 64, on the 5th-generation
// tensor cores (tcgen05) with TMA staging and TMEM accumulators.
//
// Tile = 128 consecutive queries of one residue class c of one (b, h): rows
// i = c + dil*(q0 + x), x in [0, 128).  Inside a class the dilated window
// {i + dil*t : |t| <= r} ("Longformer" wiki, section 2.2.3; the "Longformer"
// note, section "Sliding-Window Attention") is a dense window of radius r
// over the class's own positions, so a tile needs the key rows of its
// diagonal band only: decimated keys [q0 - r, q0 + 127 + r], fetched in
// blocks of 64 with TMA boxes whose row traversal stride is dil.  After the
// band blocks come ngb blocks of packed global keys (built by the prep
// kernel), masked where a global key already lies in the row's window so
// each key counts once ("Global Attention": N(i) = N_local(i) U G).
//
// Per key block:   S = Q K^T        tcgen05.mma, M=128, N=64 (or the global
//                                   count rounded to 16), K=64, operands in
//                                   shared memory -> S in TMEM (fp32)
//                  online softmax   one thread per query row (TMEM lane): the
//                                   row's 64 scores in registers, masked,
//                                   block max, exponent base, exp2, row sum
//                  O += P V         P (bf16) written over the S block it came
//                                   from and read from TMEM as the A operand;
//                                   V from shared memory; M=128, N=64, K=64
// S lives in a ring of three TMEM buffers, so the products of the next blocks
// are ready while the softmax threads work on this one: in steady state the
// softmax threads wait for nothing but S.  The exponent base moves (O and the
// row sum rescaled in place) only when a block's max exceeds it by more than
// 2^8; otherwise p = 2^(s - base) stays below 256, which fp32 accumulation
// and bf16 P absorb.
// The mask view of the note ("Mask View": A = QK^T/sqrt(d) + M, M = -inf off
// the pattern) is applied inline: band limits and sequence ends as a per-row
// column interval, padded keys from the key padding mask, the global-key
// dedup test per column.  Blocks inside every row's window need no test, and
// 32-column chunks that no row of a warp keeps skip their exponentials.
// Nothing of size T x T is built.
//
// Work split ("stream-K").  The tiles' key blocks, in the order (b, h, c,
// tile, block), form one sequence; CTA s takes the contiguous range
// [s*N/G, (s+1)*N/G) of it, so every CTA gets the same number of blocks
// whatever the tile count.  A range boundary that cuts a tile leaves pieces
// of it in neighbouring CTAs; each piece ends with its partial softmax state
// (m, l, O) per row.  Per 32-row quarter, each piece takes a ticket (atomic)
// as it starts its last block; the last to arrive merges the partial states,
// which the others write to the workspace without waiting for anything, in
// CTA order (so the result does not depend on who arrives last), and stores
// the rows.  A piece only ever waits for pieces that have already arrived.
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

constexpr int kBM = 128;  // queries per tile
constexpr int kBN = 64;   // keys per block
constexpr int kQStages = 2;
constexpr int kKVStages = 4;
constexpr int kSBufs = 3;                // S / P buffers in TMEM
constexpr int kBandThreads = 192;
constexpr int kSoftmaxWarps = 4;
constexpr float kRescaleLog2 = 8.f;  // move the exponent base only past 2^8

// barrier slots
constexpr int kBarQFull = 0, kBarQEmpty = kBarQFull + kQStages, kBarKFull = kBarQEmpty + kQStages,
              kBarKEmpty = kBarKFull + kKVStages, kBarVFull = kBarKEmpty + kKVStages,
              kBarVEmpty = kBarVFull + kKVStages, kBarSFull = kBarVEmpty + kKVStages, kBarPFull = kBarSFull + kSBufs,
              kBarBufFree = kBarPFull + kSBufs, kBarOFull = kBarBufFree + kSBufs, kBarDrain = kBarOFull + 2,
              kNumBars = kBarDrain + 1;
constexpr int kDescBytes = 128;
constexpr int kMaxRand = 4;  // random key blocks per 64-row query block (the BigBird variant)
constexpr int kMiscBytes = 16;
constexpr uint32_t kColO = 192;

// What depends on the head dimension HD (64 or 128).  Rows of q, k and v are
// staged as HD / 64 sub-tiles of 64 columns (128 bytes, one 128-byte swizzle
// atom per row), each a separate TMA box and MMA operand.
//   Shared memory: Q tiles (kQStages), then the K and V rings (kKVStages),
//   the barriers, the piece descriptors (one per Q slot: written by the
//   producer before it arrives on the slot's Q-full barrier, read by the MMA
//   and softmax roles after waiting on it, so only the producer walks the
//   work sequence; a slot is free again once the piece's last product has
//   been issued and its rows have been written), then the TMEM slot and the
//   abort flag.
//   TMEM: three S buffers of 64 fp32 columns at 0, 64, 128 (P, 16-bit pairs,
//   over the first 32 columns of its own buffer), O (fp32, HD wide) at 192:
//   256 columns, two CTAs per SM, for HD = 64; 320 (a 512-column
//   allocation), one CTA per SM, for HD = 128.
//   Partial state of one piece (128 rows): O as [HD / 4][128][4] fp32 (four
//   columns of every row per 16-byte group, so a warp's stores and loads are
//   contiguous), then m[128] and l[128].
template <int HD>
struct BandCfg {
    static_assert(HD == 64 || HD == 128, "head dimension");
    static constexpr int kHD = HD;
    static constexpr int kSub = HD / 64;            // 64-column sub-tiles per row
    static constexpr int kQBytes = kBM * HD * 2;    // 16 KB per 64 columns: 128 rows x 128 bytes
    static constexpr int kQSubBytes = kBM * 128;
    static constexpr int kKVBytes = kBN * HD * 2;   // 8 KB per 64 columns
    static constexpr int kKVSubBytes = kBN * 128;
    static constexpr int kOffQ = 0;
    static constexpr int kOffK = kOffQ + kQStages * kQBytes;
    static constexpr int kOffV = kOffK + kKVStages * kKVBytes;
    static constexpr int kOffBar = kOffV + kKVStages * kKVBytes;
    static constexpr int kOffDesc = kOffBar + ((kNumBars * 8 + 15) / 16) * 16;
    static constexpr int kOffMisc = kOffDesc + kQStages * kDescBytes;
    static constexpr int kSmem = kOffMisc + kMiscBytes + 1024;  // + alignment slack
    static constexpr int kCtasPerSm = HD == 64 ? 2 : 1;
    static constexpr uint32_t kTmemCols = HD == 64 ? 256 : 512;
    static constexpr int kPartFloats = kBM * HD + 2 * kBM;
    static_assert(kCtasPerSm * (kSmem + 1024) <= 233472, "shared memory budget per SM");
    static_assert(kColO + HD <= kTmemCols, "TMEM budget");
};

// One piece: blocks [blk_lo, blk_hi) of one tile's nbb band blocks and ngb
// global blocks.
struct BandPiece {
    int b, bh, c, dil, dk, R;
    int Tc, q0, kbase, kb_lo, nbb, ngb;
    int blk_lo, blk_hi;
    int tile;          // tile index (its merge tickets)
    int s0, s1;        // the CTAs whose ranges hold the tile's blocks
    int last;          // 1: the last piece this CTA processes
    int tstart;        // position of the tile's first block in the sequence
    int rb[2 * kMaxRand];  // random variant: the tile's random key blocks (-1: none), query block 0's then 1's
};
static_assert(sizeof(BandPiece) <= kDescBytes, "piece descriptor slot");

// Band blocks of tile t of a class with Tc decimated rows: the decimated keys
// [q0 - r, q0 + 127 + r] clipped to [0, Tc), in kBN-key blocks counted from
// kbase = q0 - r.
__host__ __device__ __forceinline__ void tile_band(int Tc, int r, int t, int& kbase, int& kb_lo, int& nbb) {
    const int q0 = t * kBM;
    kbase = q0 - r;
    const int lo = kbase > 0 ? kbase : 0;
    const int hi = (q0 + kBM - 1 + r) < (Tc - 1) ? (q0 + kBM - 1 + r) : (Tc - 1);
    kb_lo = (lo - kbase) / kBN;
    nbb = (hi - kbase) / kBN + 1 - kb_lo;
}

// First block of CTA s's range, floor(s * N / G), from N = q * G + rm
// (32-bit arithmetic: N < 2^31, G <= 296).
__host__ __device__ __forceinline__ int range_start(const BandTcParams& p, int s) {
    return p.blk_q * s + (p.blk_rm * s) / p.grid_ctas;
}
// The CTA whose range holds block x (every range has q or q + 1 blocks).
__host__ __device__ __forceinline__ int cta_of(const BandTcParams& p, int x) {
    int s = static_cast<int>(static_cast<double>(x) * p.grid_ctas / p.n_blocks);
    while (s + 1 < p.grid_ctas && range_start(p, s + 1) <= x) ++s;
    while (s > 0 && range_start(p, s) > x) --s;
    return s;
}

// Walks the tiles in sequence order.
struct TileWalker {
    int b, h, c, t, tile;
    int dk, dil, Tc, nt;
    int kbase, kb_lo, nbb;
    int start;  // position of the tile's first block

    __host__ __device__ void set_class(const BandTcParams& p) {
        dk = p.head_dk[h];
        dil = p.dk_dil[dk];
        Tc = (p.T - c + dil - 1) / dil;
        nt = (Tc + kBM - 1) / kBM;
    }
    __host__ __device__ void shape(const BandTcParams& p) { tile_band(Tc, p.r, t, kbase, kb_lo, nbb); }
    __host__ __device__ int nb(const BandTcParams& p) const { return nbb + p.ngb; }

    // The tile that holds block x of the sequence.
    __host__ __device__ void locate(const BandTcParams& p, int x) {
        b = x / p.blocks_per_b;
        int rem = x - b * p.blocks_per_b;
        h = 0;
        while (h + 1 < p.H && p.head_blk[h + 1] <= rem) ++h;
        rem -= p.head_blk[h];
        c = 0;
        dk = p.head_dk[h];
        while (c + 1 < p.dk_dil[dk] && p.dk_class_blk[dk][c + 1] <= rem) ++c;
        rem -= p.dk_class_blk[dk][c];
        set_class(p);
        tile = b * p.tiles_per_b + p.head_tile[h] + p.dk_class_tile[dk][c];
        start = x - rem;
        // interior tiles (whole band inside [0, Tc)) all have the same block count
        const int t_a = (p.r + kBM - 1) / kBM;
        const int t_b = Tc - kBM - p.r >= 0 ? (Tc - kBM - p.r) / kBM + 1 : 0;
        t = 0;
        for (;;) {
            shape(p);
            const int n = nb(p);
            if (t == t_a && t_b > t_a) {
                const int span = (t_b - t_a) * n;
                if (rem >= span) {
                    rem -= span;
                    start += span;
                    tile += t_b - t_a;
                    t = t_b;
                    continue;
                }
                const int k = rem / n;
                rem -= k * n;
                start += k * n;
                tile += k;
                t += k;
                shape(p);
                break;
            }
            if (rem < n) break;
            rem -= n;
            start += n;
            ++tile;
            ++t;
        }
    }
    // The next tile (residue classes with no rows, T < dil, are skipped).
    __host__ __device__ void next(const BandTcParams& p) {
        start += nb(p);
        ++tile;
        if (++t >= nt) {
            t = 0;
            do {
                if (++c >= dil) {
                    c = 0;
                    if (++h == p.H) {
                        h = 0;
                        ++b;
                    }
                }
                set_class(p);
            } while (nt == 0);
        }
        shape(p);
    }
};

// Columns of global block gb that the MMA computes (a multiple of 16, at
// least 16 even where the block holds no key of this sample).
__device__ __forceinline__ int global_block_cols(int ngk, int gb) {
    int rem = ngk - gb * kBN;
    rem = rem < 16 ? 16 : (rem > kBN ? kBN : rem);
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
// Largest / smallest of 32 consecutive scores (four independent chains).
__device__ __forceinline__ float max32(const uint32_t* v) {
    float m[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) m[u] = fmaxf(__uint_as_float(v[2 * u]), __uint_as_float(v[2 * u + 1]));
#pragma unroll
    for (int j = 8; j < 32; j += 8)
#pragma unroll
        for (int u = 0; u < 4; ++u) m[u] = fmax3(m[u], __uint_as_float(v[j + 2 * u]), __uint_as_float(v[j + 2 * u + 1]));
    return fmaxf(fmaxf(m[0], m[1]), fmaxf(m[2], m[3]));
}
__device__ __forceinline__ float min32(const uint32_t* v) {
    float m[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) m[u] = fminf(__uint_as_float(v[2 * u]), __uint_as_float(v[2 * u + 1]));
#pragma unroll
    for (int j = 8; j < 32; j += 8)
#pragma unroll
        for (int u = 0; u < 4; ++u) m[u] = fmin3(m[u], __uint_as_float(v[j + 2 * u]), __uint_as_float(v[j + 2 * u + 1]));
    return fminf(fminf(m[0], m[1]), fminf(m[2], m[3]));
}

// ------------------------------------------------------------- TMA producer
// Walks this CTA's range once: for each piece it publishes the descriptor and
// loads the tile's Q, then the K and V blocks; K runs one block ahead of V
// (K(g + 1) is needed for the next product, V(g) only once P(g) is written).
// Processing order: when the range ends inside a tile (its head; the rest of
// that tile is the first piece of the next CTA), that piece goes first, then
// the range from its start.  Both pieces of every split tile are then done
// early in their CTAs, so the merges that join them overlap other work
// instead of ending the kernel.
// Only the global-key blocks read the prep kernel's output (packed keys), so
// the wait for prep comes just before the first of them: the band blocks of
// the first tile overlap prep.
template <int HD, bool kRand>
__device__ __forceinline__ void producer_role(const BandTcParams& p, uint8_t* smem, uint64_t* bars,
                                              volatile int* abort_flag) {
    using C = BandCfg<HD>;
    const int nrb = kRand ? p.nrb : 0;  // random key blocks per tile (dilation 1 only)
    const int s = blockIdx.x;
    const int x0 = range_start(p, s);
    const int x1 = range_start(p, s + 1);
    TileWalker w;
    w.locate(p, x0);
    TileWalker wz = w;  // the tile that holds the range's last block: a few tiles on at most
    while (wz.start + wz.nb(p) < x1) wz.next(p);
    if (p.test_stall) return;  // test hook: nothing is published, so the other roles' waits run out
    const bool front = wz.tile != w.tile && wz.start + wz.nb(p) > x1;  // the split last tile goes first
    const int x_main_end = front ? wz.start : x1;
    bool prep_done = false;

    uint32_t gk = 0, gv = 0, qt = 0;
    auto issue_kv = [&](const BandPiece& d, int blk, bool is_v, uint32_t g) -> bool {
        const uint32_t st = g % kKVStages;
        const uint32_t ph = (g / kKVStages) & 1u;
        uint64_t* empty = &bars[(is_v ? kBarVEmpty : kBarKEmpty) + st];
        uint64_t* full = &bars[(is_v ? kBarVFull : kBarKFull) + st];
        if (!mbar_wait(empty, ph ^ 1u, abort_flag, p.wait_ns)) return false;
        uint8_t* dst = smem + (is_v ? C::kOffV : C::kOffK) + st * C::kKVBytes;
        if (blk < d.nbb) {
            mbar_arrive_expect_tx(full, C::kKVBytes);
            const int j0 = d.kbase + kBN * (d.kb_lo + blk);
            const CUtensorMap* tm = is_v ? &p.tm_v[d.dk] : &p.tm_k[d.dk];
#pragma unroll
            for (int sub = 0; sub < C::kSub; ++sub)
                for (int u = 0; u < kBN; u += d.R)
                    tma_load_3d(dst + sub * C::kKVSubBytes + u * 128, tm, full, 64 * sub, d.c + d.dil * (j0 + u), d.bh);
        } else if (kRand && blk < d.nbb + nrb) {  // a random key block (none: rows past T, zero-filled)
            mbar_arrive_expect_tx(full, C::kKVBytes);
            const int rb = d.rb[blk - d.nbb];
            const int j0 = rb >= 0 ? kBN * rb : p.T;
            const CUtensorMap* tm = is_v ? &p.tm_v[d.dk] : &p.tm_k[d.dk];
#pragma unroll
            for (int sub = 0; sub < C::kSub; ++sub)
                for (int u = 0; u < kBN; u += d.R)
                    tma_load_3d(dst + sub * C::kKVSubBytes + u * 128, tm, full, 64 * sub, j0 + u, d.bh);
        } else {
            if (!prep_done) {  // packed global keys from here on
                grid_dep_wait();
                prep_done = true;
            }
            mbar_arrive_expect_tx(full, C::kKVBytes);
#pragma unroll
            for (int sub = 0; sub < C::kSub; ++sub)
                tma_load_3d(dst + sub * C::kKVSubBytes, is_v ? &p.tm_vg : &p.tm_kg, full, 64 * sub,
                            (blk - d.nbb - nrb) * kBN, d.bh);
        }
        return true;
    };

    // current position: block x of tile cw, inside the segment that ends at x_stop
    bool in_front = front;
    TileWalker* cw = in_front ? &wz : &w;
    int x = in_front ? wz.start : x0;
    int x_stop = in_front ? x1 : x_main_end;
    bool piece_start = true;
    bool have_prev = false;
    int prev_slot = 0, prev_blk = 0;
    bool ok = true;
    while (ok) {
        const bool have_cur = x < x_stop;
        int cur_slot = 0, cur_blk = 0;
        if (have_cur) {
            const int tend = cw->start + cw->nb(p);
            const int blk = x - cw->start;
            const uint32_t qs = qt & 1u;
            if (piece_start) {  // a new piece: descriptor and Q
                piece_start = false;
                if (!mbar_wait(&bars[kBarQEmpty + qs], ((qt >> 1) & 1u) ^ 1u, abort_flag, p.wait_ns)) break;
                BandPiece d;
                d.b = cw->b;
                d.bh = cw->b * p.H + cw->h;
                d.c = cw->c;
                d.dil = cw->dil;
                d.dk = cw->dk;
                d.R = p.dk_rows[cw->dk];
                d.Tc = cw->Tc;
                d.q0 = cw->t * kBM;
                d.kbase = cw->kbase;
                d.kb_lo = cw->kb_lo;
                d.nbb = cw->nbb;
                d.ngb = p.ngb;
                d.blk_lo = blk;
                const int pend = tend < x_stop ? tend : x_stop;
                d.blk_hi = pend - cw->start;
                d.tile = cw->tile;
                // the CTAs whose ranges hold the tile's blocks, found from this one
                int s0 = s, s1 = s;
                while (s0 > 0 && range_start(p, s0) > cw->start) --s0;
                while (s1 + 1 < p.grid_ctas && range_start(p, s1 + 1) <= tend - 1) ++s1;
                d.s0 = s0;
                d.s1 = s1;
                d.last = (!in_front && pend == x_main_end) ? 1 : 0;
                d.tstart = cw->start;
                if constexpr (kRand) {  // the draws of the tile's two query blocks (q0 / 64 and the next)
                    const int nr = p.n_rand;
#pragma unroll
                    for (int k = 0; k < 2 * kMaxRand; ++k) {
                        int rb = -1;
                        if (k < 2 * nr) {
                            const int qb = d.q0 / kBN + k / nr;
                            if (qb < p.nqb) rb = p.rnd[(static_cast<size_t>(d.bh) * p.nqb + qb) * nr + k % nr];
                            if (rb < 0 || rb >= p.nqb) rb = -1;  // outside the sequence: ignored
                        }
                        d.rb[k] = rb;
                    }
                }
                *reinterpret_cast<BandPiece*>(smem + C::kOffDesc + qs * kDescBytes) = d;  // released by the arrive
                mbar_arrive_expect_tx(&bars[kBarQFull + qs], C::kQBytes);
                uint8_t* dQ = smem + C::kOffQ + qs * C::kQBytes;
#pragma unroll
                for (int sub = 0; sub < C::kSub; ++sub)
                    for (int u = 0; u < kBM; u += d.R)
                        tma_load_3d(dQ + sub * C::kQSubBytes + u * 128, &p.tm_q[d.dk], &bars[kBarQFull + qs], 64 * sub,
                                    d.c + d.dil * (d.q0 + u), d.bh);
                ++qt;
            }
            cur_slot = (qt - 1) & 1u;
            cur_blk = blk;
            const BandPiece& d = *reinterpret_cast<const BandPiece*>(smem + C::kOffDesc + cur_slot * kDescBytes);
            if (!issue_kv(d, blk, false, gk)) break;
            ++gk;
            ++x;
            if (x == x_stop || x == tend) {  // the piece ends here
                piece_start = true;
                if (x == x_stop && in_front) {  // on to the range from its start
                    in_front = false;
                    cw = &w;
                    x = x0;
                    x_stop = x_main_end;
                } else if (x < x_stop) {
                    cw->next(p);
                }
            }
        }
        if (have_prev) {
            const BandPiece& d = *reinterpret_cast<const BandPiece*>(smem + C::kOffDesc + prev_slot * kDescBytes);
            if (!issue_kv(d, prev_blk, true, gv)) break;
            ++gv;
        }
        have_prev = have_cur;
        prev_slot = cur_slot;
        prev_blk = cur_blk;
        ok = have_cur || have_prev;
    }
    if (*abort_flag) {  // let issued copies land before the CTA can exit
        for (uint32_t k = 0; k < kKVStages; ++k) {
            if (gk > k) (void)mbar_wait_drain(&bars[kBarKFull + (gk - 1 - k) % kKVStages], ((gk - 1 - k) / kKVStages) & 1u);
            if (gv > k) (void)mbar_wait_drain(&bars[kBarVFull + (gv - 1 - k) % kKVStages], ((gv - 1 - k) / kKVStages) & 1u);
        }
        for (uint32_t k = 0; k < kQStages; ++k)
            if (qt > k) (void)mbar_wait_drain(&bars[kBarQFull + ((qt - 1 - k) & 1u)], ((qt - 1 - k) >> 1) & 1u);
    }
}

// --------------------------------------------------------------- MMA issuer
// S(g) = Q K(g)^T into TMEM buffer g % 3 once K(g) has landed and the
// product that last read that buffer, P(g - 3) V(g - 3), has finished; then
// O += P(g-1) V(g-1) once P(g-1) is in TMEM.  Every product commits to the
// O-complete barrier of its parity (two barriers, so a softmax thread that
// only sometimes waits for a product can still tell the phases apart).
// kHalf: q, k, v (and so P) are f16 instead of bf16.
// With HD = 128, S sums the products of the two 64-column sub-tiles of Q and
// K, and O's two 64-column halves each take the product with their own
// sub-tile of V.
template <bool kHalf, int HD, bool kRand>
__device__ __forceinline__ void mma_role(const BandTcParams& p, uint8_t* smem, uint64_t* bars,
                                         volatile int* abort_flag, uint32_t tmem_base) {
    using C = BandCfg<HD>;
    const int nrb = kRand ? p.nrb : 0;  // random key blocks per tile, after the band blocks
    const uint32_t idesc_pv = kHalf ? idesc_f16(kBM, 64, 0, 1) : idesc_bf16(kBM, 64, 0, 1);
    uint64_t dQ[kQStages];
#pragma unroll
    for (int st = 0; st < kQStages; ++st) dQ[st] = sdesc_k_sw128(smem_u32(smem + C::kOffQ + st * C::kQBytes));
    const uint64_t dK0 = sdesc_k_sw128(smem_u32(smem + C::kOffK));
    const uint64_t dV0 = sdesc_mn_sw128(smem_u32(smem + C::kOffV));
    constexpr uint64_t kKVDescStep = C::kKVBytes >> 4;  // start-address units per ring stage
    constexpr uint64_t kQSubStep = C::kQSubBytes >> 4, kKVSubStep = C::kKVSubBytes >> 4;
    const uint32_t tO = tmem_base + kColO;

    // O += P(g) V(g) over nk keys; the first block of a piece overwrites O
    auto issue_pv = [&](uint32_t g, int nk, bool first) -> bool {
        const uint32_t b = g % kSBufs, st = g % kKVStages;
        if (!mbar_wait(&bars[kBarPFull + b], (g / kSBufs) & 1u, abort_flag, p.wait_ns) ||
            !mbar_wait(&bars[kBarVFull + st], (g / kKVStages) & 1u, abort_flag, p.wait_ns))
            return false;
        tc_fence_after();
        const uint32_t tP = tmem_base + 64u * b;
#pragma unroll
        for (int sub = 0; sub < C::kSub; ++sub) {
            const uint64_t dv = dV0 + kKVDescStep * st + kKVSubStep * sub;
            const uint32_t to = tO + 64u * sub;
            if (first)
                tc_mma_ts<false>(to, tP, dv, idesc_pv);
            else
                tc_mma_ts<true>(to, tP, dv, idesc_pv);
            for (int k = 1; k < nk / 16; ++k) tc_mma_ts<true>(to, tP + 8u * k, dv + 128u * k, idesc_pv);
        }
        tc_commit(&bars[kBarBufFree + b]);
        tc_commit(&bars[kBarOFull + (g & 1u)]);
        tc_commit(&bars[kBarVEmpty + st]);
        return true;
    };

    uint32_t g = 0, qt = 0;
    int prev_nk = 0;
    bool prev_first = false, done = false;
    while (!done) {
        const uint32_t qs = qt & 1u;
        if (!mbar_wait(&bars[kBarQFull + qs], (qt >> 1) & 1u, abort_flag, p.wait_ns)) break;
        ++qt;
        const BandPiece* d = reinterpret_cast<const BandPiece*>(smem + C::kOffDesc + qs * kDescBytes);
        const int blk_lo = d->blk_lo, blk_hi = d->blk_hi, nbb = d->nbb, bsm = d->b;
        int ngk = -1;  // global keys of this sample (prep's output), read at the first global block
        done = d->last != 0;
        bool ok = true;
        for (int blk = blk_lo; blk < blk_hi; ++blk, ++g) {
            const uint32_t b = g % kSBufs, st = g % kKVStages;
            if (!mbar_wait(&bars[kBarKFull + st], (g / kKVStages) & 1u, abort_flag, p.wait_ns) ||
                (g >= kSBufs && !mbar_wait(&bars[kBarBufFree + b], ((g / kSBufs) & 1u) ^ 1u, abort_flag, p.wait_ns))) {
                ok = false;
                break;
            }
            tc_fence_after();
            if (blk >= nbb + nrb && ngk < 0) {
                grid_dep_wait();
                ngk = *reinterpret_cast<const volatile int*>(p.n_gk + bsm);
            }
            const int ncols = blk < nbb + nrb ? kBN : global_block_cols(ngk, blk - nbb - nrb);
            const uint32_t ids = kHalf ? idesc_f16(kBM, ncols, 0, 0) : idesc_bf16(kBM, ncols, 0, 0);
            const uint64_t dq = dQ[qs], dk = dK0 + kKVDescStep * st;
            const uint32_t tS = tmem_base + 64u * b;
            tc_mma<false>(tS, dq + 0, dk + 0, ids);  // K-steps of 16 (32 bytes = 2 units)
            tc_mma<true>(tS, dq + 2, dk + 2, ids);
            tc_mma<true>(tS, dq + 4, dk + 4, ids);
            tc_mma<true>(tS, dq + 6, dk + 6, ids);
#pragma unroll
            for (int sub = 1; sub < C::kSub; ++sub) {  // the next 64 columns of q and k
                const uint64_t dqs = dq + kQSubStep * sub, dks = dk + kKVSubStep * sub;
                tc_mma<true>(tS, dqs + 0, dks + 0, ids);
                tc_mma<true>(tS, dqs + 2, dks + 2, ids);
                tc_mma<true>(tS, dqs + 4, dks + 4, ids);
                tc_mma<true>(tS, dqs + 6, dks + 6, ids);
            }
            tc_commit(&bars[kBarSFull + b]);
            tc_commit(&bars[kBarKEmpty + st]);
            if (blk == blk_hi - 1) tc_commit(&bars[kBarQEmpty + qs]);
            if (g > 0 && !issue_pv(g - 1, prev_nk, prev_first)) {
                ok = false;
                break;
            }
            prev_nk = ncols;
            prev_first = blk == blk_lo;
        }
        if (!ok) break;
        if (done && g > 0) (void)issue_pv(g - 1, prev_nk, prev_first);
    }
    tc_commit(&bars[kBarDrain]);
}

// ------------------------------------------------------------ softmax role
// Thread x owns query row x of the tile (TMEM lane x).  Per block: wait for
// S, load the row's 64 scores, mask, take the block max, move the exponent
// base if needed, exponentiate, store P over S.  The output (or partial
// state) of a piece is written when the next piece starts, or at the end,
// once the piece's last product has finished.

// Multiplies this thread's row of O (HD fp32 columns) by alpha, in TMEM,
// 16 columns at a time (few registers: it runs inside the block loop).
template <int HD>
__device__ __forceinline__ void rescale_o(uint32_t tO, float alpha) {
#pragma unroll 1
    for (int part = 0; part < HD / 16; ++part) {
        uint32_t o[16];
        tmem_ld16(tO + 16u * part, o);
        tmem_ld_wait16(o);
#pragma unroll
        for (int c = 0; c < 16; ++c) o[c] = __float_as_uint(__uint_as_float(o[c]) * alpha);
        tmem_st16(tO + 16u * part, o);
    }
}

// Writes output dimensions [32 hd, 32 hd + 32) of the warp's 32 rows as
// bf16: y = o * inv for this lane's row (32 values) to row_ptr + 32 hd when
// `write`.  Every store instruction writes whole 64-byte row halves, eight of
// them: each group of 4 lanes transposes its 4 x 4 block of 16-byte chunks
// with two rounds of xor shuffles, after which store e of lane 4g + j writes
// chunk j of row 4g + e.  (One lane per row would make every store touch 32
// lines.)  Warp-wide: every lane calls it.
template <bool kHalf>
__device__ __forceinline__ void store_half_rows(__nv_bfloat16* row_ptr, bool write, int hd, const float* o,
                                                float inv) {
    const int lane = threadIdx.x & 31;
    uint32_t x[4][4];
#pragma unroll
    for (int c = 0; c < 4; ++c)
#pragma unroll
        for (int w = 0; w < 4; ++w) x[c][w] = pack16x2<kHalf>(o[8 * c + 2 * w] * inv, o[8 * c + 2 * w + 1] * inv);
#pragma unroll
    for (int sh = 2; sh >= 1; sh >>= 1) {
        const bool upper = (lane & sh) != 0;
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            if (e & sh) continue;
#pragma unroll
            for (int w = 0; w < 4; ++w) {
                const uint32_t send = upper ? x[e][w] : x[e + sh][w];
                const uint32_t recv = __shfl_xor_sync(0xffffffffu, send, sh);
                if (upper)
                    x[e][w] = recv;
                else
                    x[e + sh][w] = recv;
            }
        }
    }
    const int g0 = lane & ~3, j = lane & 3;
    const unsigned long long rp = reinterpret_cast<unsigned long long>(row_ptr + 32 * hd);
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        const unsigned long long dst = __shfl_sync(0xffffffffu, rp, g0 + e);
        const int wr = __shfl_sync(0xffffffffu, write ? 1 : 0, g0 + e);
        if (wr) *reinterpret_cast<uint4*>(dst + 16ull * j) = make_uint4(x[e][0], x[e][1], x[e][2], x[e][3]);
    }
}

// Partial slot of CTA s's piece of a tile that starts at tstart: 2s for the
// piece at the start of s's range, 2s + 1 for the one at its end.
template <int HD>
__device__ __forceinline__ float* part_slot(const BandTcParams& p, int s, int tstart) {
    const int k = 2 * s + (tstart > range_start(p, s) ? 1 : 0);
    return p.part + static_cast<size_t>(k) * BandCfg<HD>::kPartFloats;
}

// Output of a finished piece (warp-wide: every lane calls it): its
// descriptor d stays in shared memory until this is done; m and l are this
// thread's row's exponent base and sum.  The row is handled 32 output
// dimensions at a time (registers: this runs with the next piece's state live).
template <bool kHalf, int HD>
__device__ __forceinline__ void flush_rows(const BandTcParams& p, const BandPiece* d, float m, float l, uint32_t tO,
                                          int wq, int ticket, volatile int* abort_flag) {
    constexpr int kHD = HD, kHalves = HD / 32;  // 32-column groups of a row
    const int lane = threadIdx.x & 31;
    const int x = wq * 32 + lane;
    const int self = static_cast<int>(blockIdx.x);
    const int ip = d->q0 + x, Tc = d->Tc;
    const int i = d->c + d->dil * ip;
    bool write = ip < Tc;
    if (write) write = !((p.gbit[static_cast<size_t>(d->b) * p.W + (i >> 5)] >> (i & 31)) & 1u);
    __nv_bfloat16* dst = p.out + (static_cast<size_t>(d->bh) * p.T + (write ? i : 0)) * kHD;
    // 32 columns of this row's O (dimensions [32 hd, 32 hd + 32))
    auto load_o = [&](int hd, float* o) {
        uint32_t r[32];
        tmem_ld32(tO + 32u * hd, r);
        tmem_ld_wait(r);
#pragma unroll
        for (int c = 0; c < 32; ++c) o[c] = __uint_as_float(r[c]);
    };
    if (d->blk_lo == 0 && d->blk_hi == d->nbb + d->ngb) {  // the whole tile
        const float inv = l > 0.f ? 1.f / l : 0.f;
#pragma unroll 1
        for (int hd = 0; hd < kHalves; ++hd) {
            float o[32];
            load_o(hd, o);
            store_half_rows<kHalf>(dst, write, hd, o, inv);
        }
        return;
    }
    const int s0 = d->s0, s1 = d->s1;
    const int tstart = d->tstart;
    int* cnt = p.cnt + (static_cast<size_t>(d->tile) * 4 + wq) * 2;  // [0] arrivals, [1] lanes done writing
    const int npieces = s1 - s0 + 1;
    if (ticket < npieces - 1) {  // not the last to arrive: leave the partial state for the last
        float* slot = part_slot<HD>(p, self, tstart);
        float4* o4 = reinterpret_cast<float4*>(slot);
#pragma unroll 1
        for (int hd = 0; hd < kHalves; ++hd) {
            float o[32];
            load_o(hd, o);
#pragma unroll
            for (int u = 0; u < 8; ++u)
                o4[(8 * hd + u) * kBM + x] = make_float4(o[4 * u], o[4 * u + 1], o[4 * u + 2], o[4 * u + 3]);
        }
        slot[kBM * kHD + x] = m;
        slot[kBM * kHD + kBM + x] = l;
        red_release_add(cnt + 1, 1);  // each lane: its stores, then its count (no wait)
        return;
    }
    // the last to arrive: the others arrived earlier and write without waiting
    // for anything; every lane acquires their count, so their partial states
    // are visible to it
    bool ok = true;
    {
        const int want = 32 * (npieces - 1);
        const uint64_t t0 = globaltimer_ns();
        for (uint32_t it = 0; __any_sync(0xffffffffu, ld_acquire(cnt + 1) < want); ++it) {
            if ((it & 63u) == 63u && globaltimer_ns() - t0 > p.wait_ns) {
                if (lane == 0) *abort_flag = 1;
                ok = false;
                break;
            }
        }
    }
    // M = max of the pieces' bases; y = sum_s w_s O_s / sum_s w_s l_s with w_s = 2^(m_s - M),
    // summed in CTA order whichever piece merges (the same operations either way)
    if (npieces == 2 && ok) {  // the common case: one other piece
        const int so = self == s0 ? s1 : s0;
        const float* slot = part_slot<HD>(p, so, tstart);
        const float4* o4 = reinterpret_cast<const float4*>(slot);
        const float mo = __ldcg(slot + kBM * kHD + x);
        const float lo = __ldcg(slot + kBM * kHD + kBM + x);
        const float M = fmaxf(m, mo);
        const float Mu = M == -INFINITY ? 0.f : M;
        const float ws = m == -INFINITY ? 0.f : ex2_approx(m - Mu);
        const float wo = mo == -INFINITY ? 0.f : ex2_approx(mo - Mu);
        const bool self_first = self == s0;
        const float w1 = self_first ? ws : wo, w2 = self_first ? wo : ws;
        const float L = fmaf(w2, self_first ? lo : l, w1 * (self_first ? l : lo));
        const float inv = L > 0.f ? 1.f / L : 0.f;
#pragma unroll 1
        for (int hd = 0; hd < kHalves; ++hd) {
            float4 v[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) v[u] = __ldcg(o4 + (8 * hd + u) * kBM + x);
            float o[32];
            load_o(hd, o);
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const float a[4] = {v[u].x, v[u].y, v[u].z, v[u].w};
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    const float b = o[4 * u + k];
                    o[4 * u + k] = fmaf(w2, self_first ? a[k] : b, w1 * (self_first ? b : a[k]));
                }
            }
            store_half_rows<kHalf>(dst, write, hd, o, inv);
        }
    } else {
        float M = m;
        for (int s = s0; s <= s1; ++s)
            if (s != self && ok) M = fmaxf(M, __ldcg(part_slot<HD>(p, s, tstart) + kBM * kHD + x));
        const float Mu = M == -INFINITY ? 0.f : M;
        float L = 0.f;
        for (int s = s0; s <= s1; ++s) {
            if (s == self) {
                L = fmaf(m == -INFINITY ? 0.f : ex2_approx(m - Mu), l, L);
            } else if (ok) {
                const float* slot = part_slot<HD>(p, s, tstart);
                const float ms = __ldcg(slot + kBM * kHD + x);
                L = fmaf(ms == -INFINITY ? 0.f : ex2_approx(ms - Mu), __ldcg(slot + kBM * kHD + kBM + x), L);
            }
        }
        const float inv = L > 0.f ? 1.f / L : 0.f;
#pragma unroll 1
        for (int hd = 0; hd < kHalves; ++hd) {
            float acc[32];
#pragma unroll
            for (int c = 0; c < 32; ++c) acc[c] = 0.f;
            for (int s = s0; s <= s1; ++s) {
                if (s == self) {
                    const float wv = m == -INFINITY ? 0.f : ex2_approx(m - Mu);
                    float o[32];
                    load_o(hd, o);
#pragma unroll
                    for (int c = 0; c < 32; ++c) acc[c] = fmaf(wv, o[c], acc[c]);
                    continue;
                }
                if (!ok) continue;
                const float* slot = part_slot<HD>(p, s, tstart);
                const float ms = __ldcg(slot + kBM * kHD + x);
                const float wv = ms == -INFINITY ? 0.f : ex2_approx(ms - Mu);
                const float4* o4 = reinterpret_cast<const float4*>(slot);
#pragma unroll
                for (int u = 0; u < 8; ++u) {
                    const float4 v = __ldcg(o4 + (8 * hd + u) * kBM + x);
                    acc[4 * u] = fmaf(wv, v.x, acc[4 * u]);
                    acc[4 * u + 1] = fmaf(wv, v.y, acc[4 * u + 1]);
                    acc[4 * u + 2] = fmaf(wv, v.z, acc[4 * u + 2]);
                    acc[4 * u + 3] = fmaf(wv, v.w, acc[4 * u + 3]);
                }
            }
            store_half_rows<kHalf>(dst, write, hd, acc, inv);
        }
    }
    __syncwarp();
    if (lane == 0) {  // ready for the next call
        cnt[0] = 0;
        cnt[1] = 0;
    }
}

// kSearch: the sample may have more than 32 global keys; the global-key block's
// dedup then finds the keys in a row's window by binary search (below).
template <bool kSearch, bool kHalf, int HD, bool kRand>
__device__ __forceinline__ void softmax_role(const BandTcParams& p, uint8_t* smem, uint64_t* bars,
                                             volatile int* abort_flag, uint32_t tmem_base) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int wq = warp & 3;
    const int x = wq * 32 + lane;  // query row inside the tile = TMEM lane
    const uint32_t lane_off = static_cast<uint32_t>(wq * 32) << 16;
    const uint32_t tO = tmem_base + lane_off + kColO;
    // scale >= 0: maxima on raw scores (masked columns -inf); scale < 0: minima
    // (masked columns +inf); either way the scale is folded into the exp2 FMA
    const bool pos = p.sl2 >= 0.f;
    const float kmul = p.sl2 == 0.f ? 1e-30f : p.sl2;
    const uint32_t fill = __float_as_uint(pos ? -INFINITY : INFINITY);
    // prep's output (global-key lists and counts, the global-row bitmap, the
    // zeroed merge tickets) is needed only from the first global-key block or
    // the first rows written; the band blocks before that overlap prep
    bool prep_done = false;
    auto need_prep = [&]() {
        if (!prep_done) {
            grid_dep_wait();
            prep_done = true;
        }
    };

    // every lane polls (each lane's own acquire), then the warp agrees on the outcome
    auto wait_warp = [&](uint64_t* bar, uint32_t parity) -> bool {
        const bool ok = mbar_wait(bar, parity, abort_flag, p.wait_ns);
        return __all_sync(0xffffffffu, ok);
    };
    // the product of block gp has finished (the O-complete barrier of its parity)
    auto wait_product = [&](uint32_t gp) -> bool {
        if (!wait_warp(&bars[kBarOFull + (gp & 1u)], (gp >> 1) & 1u)) return false;
        tc_fence_after();
        return true;
    };

    // this CTA's current sample's global keys: count and the first 64 (lane a
    // holds keys a and 32 + a), loaded at the first global block of a sample
    int gk_b = -1, ngk = 0;
    uint32_t gk_reg[2] = {0u, 0u};

    uint32_t g = 0, qt = 0;
    bool done = false;
    // The previous piece, until its last product is done and its rows are
    // written; its descriptor slot is released (Q-empty) only then.
    int prev_slot = -1;
    float m_prev = 0.f, l_prev = 0.f;
    int ticket = 0;       // merge ticket of the current piece (split pieces), taken at its last block
    int ticket_prev = 0;  // the previous piece's, kept until its rows are written
    auto finish_prev = [&]() {
        const BandPiece* dq = reinterpret_cast<const BandPiece*>(smem + BandCfg<HD>::kOffDesc + prev_slot * kDescBytes);
        flush_rows<kHalf, HD>(p, dq, m_prev, l_prev, tO, wq, __shfl_sync(0xffffffffu, ticket_prev, 0), abort_flag);
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars[kBarQEmpty + prev_slot]);
        prev_slot = -1;
    };
    for (;;) {
        // After the last piece, one more pass with no piece (one empty block)
        // writes that piece's rows.
        const bool have = !done;
        const uint32_t qs = qt & 1u;
        if (have) {  // the piece's descriptor, published by the producer with its Q tile
            if (!wait_warp(&bars[kBarQFull + qs], (qt >> 1) & 1u)) return;
            ++qt;
        }
        const BandPiece* dp = reinterpret_cast<const BandPiece*>(smem + BandCfg<HD>::kOffDesc + qs * kDescBytes);
        if (have) done = dp->last != 0;
        const int blk_lo = have ? dp->blk_lo : 0, blk_hi = have ? dp->blk_hi : 1, nbb = dp->nbb;
        const int i = dp->c + dp->dil * (dp->q0 + x);  // this row's position in the sequence
        // Band blocks inside every row's window and inside [0, Tc) need no mask:
        // 0 <= 64 kb + y - x <= 2r for all x < 128, y < 64, and 0 <= j0, j0 + 64 <= Tc.
        int ib_lo = nbb, ib_hi = nbb;
        if (!p.pad) {
            const int kb_a = max(2, (-dp->kbase + kBN - 1) / kBN);
            const int kb_b = min((2 * p.r - kBN + 1) / kBN, (dp->Tc - kBN - dp->kbase) >= 0 ? (dp->Tc - kBN - dp->kbase) / kBN : -1);
            if (kb_b >= kb_a) {
                ib_lo = max(0, kb_a - dp->kb_lo);
                ib_hi = min(nbb, kb_b + 1 - dp->kb_lo);
            }
        }
        const bool split = blk_lo > 0 || blk_hi < nbb + dp->ngb;

        float m_ref = -INFINITY;  // exponent base (scaled, log2 domain; -inf: nothing kept yet)
        float l_row = 0.f;        // row sum relative to m_ref
#pragma unroll 1
        for (int blk = blk_lo; blk < blk_hi; ++blk) {
            const uint32_t b = g % kSBufs;
            const uint32_t tS = tmem_base + lane_off + 64u * b;
            float alpha = 1.f;
            bool o_move = false;
            if (have) {
                // ---- which columns this row keeps (bit j of mk[c]: column 32 c + j)
                uint32_t mk[2] = {0xffffffffu, 0xffffffffu};
                bool live0 = true, live1 = true, full0 = true, full1 = true;
                if (blk < ib_lo || blk >= ib_hi) {
                    if (blk < nbb) {
                        const int kb = dp->kb_lo + blk;
                        const int Tc = dp->Tc;
                        const int j0 = dp->kbase + kBN * kb;
                        // kept columns [ylo, yhi): the window and [0, Tc)
                        const int ylo = max(max(0, x - kBN * kb), -j0);
                        const int yhi = min(min(kBN, x + 2 * p.r + 1 - kBN * kb), Tc - j0);
#pragma unroll
                        for (int c = 0; c < 2; ++c) {
                            uint32_t m = range_bits(ylo - 32 * c, yhi - 32 * c);
                            if (p.pad) {
                                const int jd = j0 + 32 * c + lane;
                                const bool padded =
                                    jd >= 0 && jd < Tc &&
                                    p.pad[static_cast<size_t>(dp->b) * p.T + dp->c + static_cast<size_t>(dp->dil) * jd] != 0;
                                m &= ~__ballot_sync(0xffffffffu, padded);
                            }
                            mk[c] = m;
                        }
                    } else if (kRand && blk < nbb + p.nrb) {
                        // a random key block of one of the tile's two query blocks: kept for the
                        // rows of that query block, minus keys past T, in the row's window, global
                        // (the global block has them) or padded, and minus a block its query
                        // block drew before (a set: counted once)
                        need_prep();  // the global-position bitmap
                        const int k = blk - nbb, nr = p.n_rand, half = k / nr;
                        const int rbk = dp->rb[k];
                        bool dup = false;
                        for (int kk = half * nr; kk < k; ++kk) dup |= dp->rb[kk] == rbk;
                        const bool use = rbk >= 0 && !dup && (x >> 6) == half;  // the same for the whole warp
#pragma unroll
                        for (int c = 0; c < 2; ++c) {
                            uint32_t m = 0u;
                            const int j0 = kBN * rbk + 32 * c;
                            if (use && j0 < p.T) {
                                m = range_bits(0, p.T - j0) & ~range_bits(i - p.r - j0, i + p.r + 1 - j0);
                                m &= ~p.gbit[static_cast<size_t>(dp->b) * p.W + (j0 >> 5)];
                                if (p.pad) {
                                    const int jd = j0 + lane;
                                    const bool padded = jd < p.T && p.pad[static_cast<size_t>(dp->b) * p.T + jd] != 0;
                                    m &= ~__ballot_sync(0xffffffffu, padded);
                                }
                            }
                            mk[c] = m;
                        }
                    } else {  // global keys not already in the row's window
                        const int bs = dp->b;
                        if (bs != gk_b) {
                            need_prep();
                            gk_b = bs;
                            ngk = *reinterpret_cast<const volatile int*>(p.n_gk + bs);
                            const int32_t* gl = p.gk_list + static_cast<size_t>(bs) * p.gstride;
                            gk_reg[0] = lane < ngk ? static_cast<uint32_t>(gl[lane]) : 0u;
                            gk_reg[1] = 32 + lane < ngk ? static_cast<uint32_t>(gl[32 + lane]) : 0u;
                        }
                        const int gb = blk - nbb - (kRand ? p.nrb : 0);
                        const int nvalid = min(kBN, ngk - gb * kBN);
                        bool searched = false;
                        if constexpr (kSearch) {
                            if (ngk <= kBN) {
                                // all the keys are in registers, sorted and unique: the ones in
                                // this row's window are the index range [lo, hi) of the keys in
                                // [i - dil r, i + dil r] (two binary searches), within the row's
                                // residue class (the same for every row of the tile)
                                const int reach_s = dp->dil * p.r;
                                auto count_below = [&](int t) -> int {  // keys < t
                                    int pos = 0;
#pragma unroll
                                    for (int step = 64; step >= 1; step >>= 1) {
                                        const int probe = min(pos + step - 1, kBN - 1);
                                        const int k0 = static_cast<int>(__shfl_sync(0xffffffffu, gk_reg[0], probe & 31));
                                        const int k1 = static_cast<int>(__shfl_sync(0xffffffffu, gk_reg[1], probe & 31));
                                        if (pos + step - 1 < ngk && (probe < 32 ? k0 : k1) < t) pos += step;
                                    }
                                    return pos;
                                };
                                const int lo = count_below(i - reach_s), hi = count_below(i + reach_s + 1);
#pragma unroll
                                for (int c = 0; c < 2; ++c) {
                                    uint32_t in_win = range_bits(lo - 32 * c, hi - 32 * c);
                                    if (dp->dil > 1)
                                        in_win &= __ballot_sync(0xffffffffu,
                                                                static_cast<int>(gk_reg[c]) % dp->dil == dp->c);
                                    mk[c] = range_bits(0, nvalid - 32 * c) & ~in_win;
                                }
                                searched = true;
                            }
                        }
                        if (!searched) {
                        const int32_t* gkl = p.gk_list + static_cast<size_t>(bs) * p.gstride + gb * kBN;
                        const int dil = dp->dil, reach = dil * p.r;
#pragma unroll
                        for (int c = 0; c < 2; ++c) {
                            uint32_t m = 0u;
                            const int na = min(32, nvalid - 32 * c);
                            if (na > 0) {
                                const uint32_t kc = gb == 0 ? gk_reg[c] : (lane < na ? static_cast<uint32_t>(gkl[32 * c + lane]) : 0u);
#pragma unroll 1
                                for (int a = 0; a < na; ++a) {
                                    const int diff = static_cast<int>(__shfl_sync(0xffffffffu, kc, a)) - i;
                                    const bool in_window = diff <= reach && diff >= -reach && (dil == 1 || diff % dil == 0);
                                    m |= in_window ? 0u : (1u << a);
                                }
                            }
                            mk[c] = m;
                        }
                        }
                    }
                    live0 = __any_sync(0xffffffffu, mk[0] != 0u);
                    live1 = __any_sync(0xffffffffu, mk[1] != 0u);
                    full0 = __all_sync(0xffffffffu, mk[0] == 0xffffffffu);
                    full1 = __all_sync(0xffffffffu, mk[1] == 0xffffffffu);
                }

                if (split && blk == blk_hi - 1) {  // the merge ticket, while this last block is computed
                    need_prep();                     // (prep zeroes the tickets)
                    if (lane == 0) ticket = atomicAdd(p.cnt + (static_cast<size_t>(dp->tile) * 4 + wq) * 2, 1);
                }

                // ---- the row's 64 scores
                if (!wait_warp(&bars[kBarSFull + b], (g / kSBufs) & 1u)) return;
                tc_fence_after();
                uint32_t s[64];
                tmem_ld64(tS, s);
                tmem_ld_wait(s);
                reg_fence32(s + 32);

                // ---- mask and block max (scaled: the largest kept s * kmul)
                float mx0 = -INFINITY, mx1 = -INFINITY;
                if (live0) {
                    if (!full0) {
#pragma unroll
                        for (int j = 0; j < 32; ++j)
                            if (!((mk[0] >> j) & 1u)) s[j] = fill;
                    }
                    mx0 = (pos ? max32(s) : min32(s)) * kmul;
                }
                if (live1) {
                    if (!full1) {
#pragma unroll
                        for (int j = 0; j < 32; ++j)
                            if (!((mk[1] >> j) & 1u)) s[32 + j] = fill;
                    }
                    mx1 = (pos ? max32(s + 32) : min32(s + 32)) * kmul;
                }
                const float mxs = fmaxf(mx0, mx1);
                // ---- exponent base
                if (m_ref == -INFINITY) {
                    m_ref = mxs;  // nothing held so far (the row's O and l are 0)
                } else if (mxs > m_ref + kRescaleLog2) {
                    alpha = ex2_approx(m_ref - mxs);
                    l_row *= alpha;
                    m_ref = mxs;
                    o_move = true;
                }
                const float nb2 = m_ref == -INFINITY ? 0.f : -m_ref;

                // ---- p = 2^(s * kmul - base), row sums, bf16 pairs
                uint32_t pk[32];
                float2 acc0 = make_float2(0.f, 0.f), acc1 = acc0;
                const float2 k2 = make_float2(kmul, kmul), b2 = make_float2(nb2, nb2);
#pragma unroll
                for (int c = 0; c < 2; ++c) {
                    if (c == 0 ? live0 : live1) {
#pragma unroll
                        for (int j = 0; j < 32; j += 4) {
                            const float2 t0 = ffma2(make_float2(__uint_as_float(s[32 * c + j]), __uint_as_float(s[32 * c + j + 1])), k2, b2);
                            const float2 t1 = ffma2(make_float2(__uint_as_float(s[32 * c + j + 2]), __uint_as_float(s[32 * c + j + 3])), k2, b2);
                            const float2 e0 = make_float2(ex2_approx(t0.x), ex2_approx(t0.y));
                            const float2 e1 = make_float2(ex2_approx(t1.x), ex2_approx(t1.y));
                            acc0 = fadd2(acc0, e0);
                            acc1 = fadd2(acc1, e1);
                            pk[16 * c + j / 2] = pack16x2<kHalf>(e0.x, e0.y);
                            pk[16 * c + j / 2 + 1] = pack16x2<kHalf>(e1.x, e1.y);
                        }
                    } else {
#pragma unroll
                        for (int j = 0; j < 16; ++j) pk[16 * c + j] = 0u;
                    }
                }
                l_row += (acc0.x + acc0.y) + (acc1.x + acc1.y);

                // ---- P over S (released to the MMA below)
                tmem_st32(tS, pk);
            }
            // ---- the previous piece's rows, once its last product is done.  This
            // block's P is held back until they are written (the first product
            // of a piece overwrites O), so the wait overlaps this block's work.
            if (prev_slot >= 0) {
                if (!wait_product(g - 1)) return;
                need_prep();
                finish_prev();
            }
            if (!have) break;
            // ---- O is rescaled only once the previous product is done
            if (__any_sync(0xffffffffu, o_move)) {
                if (!wait_product(g - 1)) return;
                rescale_o<HD>(tO, alpha);
            }
            tmem_st_wait();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars[kBarPFull + b]);
            ++g;
        }
        if (!have) break;
        // ---- this piece's rows are written during the next piece's first block
        prev_slot = static_cast<int>(qs);
        m_prev = m_ref;
        l_prev = l_row;
        ticket_prev = ticket;
    }
}

// Instantiations from one source: kSearch = true for calls with more than 32
// global tokens (see softmax_role), false otherwise, so each keeps its own
// code for the block loop; kHalf = true for f16 inputs, false for bf16; HD =
// the head dimension (64: two CTAs per SM; 128: one); kRand: the BigBird
// variant's random key blocks follow each tile's band blocks.
template <bool kSearch, bool kHalf, int HD, bool kRand = false>
__global__ void __launch_bounds__(kBandThreads, BandCfg<HD>::kCtasPerSm)
    band_tc_kernel(const __grid_constant__ BandTcParams p) {
    using C = BandCfg<HD>;
    extern __shared__ uint8_t band_smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(band_smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kOffBar);
    uint32_t* misc = reinterpret_cast<uint32_t*>(smem + C::kOffMisc);
    uint32_t* tmem_slot = misc;
    volatile int* abort_flag = reinterpret_cast<volatile int*>(misc + 1);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kQStages; ++s) {
            mbar_init(&bars[kBarQFull + s], 1);
            mbar_init(&bars[kBarQEmpty + s], 1 + kSoftmaxWarps);  // last product of the piece + its rows written
        }
        for (int s = 0; s < kKVStages; ++s) {
            mbar_init(&bars[kBarKFull + s], 1);
            mbar_init(&bars[kBarKEmpty + s], 1);
            mbar_init(&bars[kBarVFull + s], 1);
            mbar_init(&bars[kBarVEmpty + s], 1);
        }
        for (int s = 0; s < kSBufs; ++s) {
            mbar_init(&bars[kBarSFull + s], 1);
            mbar_init(&bars[kBarPFull + s], kSoftmaxWarps);
            mbar_init(&bars[kBarBufFree + s], 1);
        }
        mbar_init(&bars[kBarOFull], 1);
        mbar_init(&bars[kBarOFull + 1], 1);
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
        tmem_alloc(tmem_slot, C::kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;

    // The set-up above may overlap the prep kernel; each role waits for it
    // (griddepcontrol.wait) before it reads prep's output.
    if (warp == 0) {
        if (lane == 0) producer_role<HD, kRand>(p, smem, bars, abort_flag);
    } else if (warp == 1) {
        if (lane == 0) mma_role<kHalf, HD, kRand>(p, smem, bars, abort_flag, tmem_base);
    } else {
        {  // touch every 64-byte line of the parameters once, so the producer's walk hits in cache
            const int t = threadIdx.x - 64;
            constexpr int kLines = (sizeof(BandTcParams) + 63) / 64;
            if (t < kLines) {
                int v;
                memcpy(&v, reinterpret_cast<const char*>(&p) + 64 * t, sizeof(int));
                asm volatile("" ::"r"(v));
            }
        }
        softmax_role<kSearch, kHalf, HD, kRand>(p, smem, bars, abort_flag, tmem_base);
    }

    tc_fence_before();
    __syncthreads();
    // every MMA has completed before TMEM is released
    if (threadIdx.x == 32) (void)mbar_wait_drain(&bars[kBarDrain], 0u);
    __syncthreads();
    if (threadIdx.x == 0 && *abort_flag) atomicOr(p.status, kStatusTimeout);
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, C::kTmemCols);
    }
}

}  // namespace lf
