// lf_common.cuh -- limits, device status bits and kernel parameter blocks
// shared by the host launcher and the kernels.
#pragma once
#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>

namespace lf {

constexpr int kMaxHeads = 128;      // H limit (per-head tables travel in the kernel parameters)
constexpr int kMaxDilKinds = 4;     // distinct dilation values per call (tensor-core path)
constexpr int kMaxDilTma = 8;       // TMA element stride limit
constexpr int kMaxT = 1 << 20;      // sequence length limit (prep bitmap lives in shared memory)
constexpr int kMaxGlobal = 4096;    // n_global limit
constexpr int kChunk = 256;         // keys per CTA in the global-row kernel

// device status word bits
constexpr uint32_t kStatusBadGlobal = 1u;  // a global_idx entry outside [0, T)
constexpr uint32_t kStatusTimeout = 2u;    // a pipeline wait gave up

// Workspace carved by the host (all offsets 256-byte aligned).
struct Workspace {
    int32_t* n_gq;      // [B]      in-range unique global queries
    int32_t* n_gk;      // [B]      ... of which not padded (global keys)
    int32_t* gq_list;   // [B][gstride] sorted
    int32_t* gk_list;   // [B][gstride] sorted
    uint32_t* gbit;     // [B][W]   bit i = position i is a global query
    int32_t* counters;  // [B*H]    arrival tickets of the global-row kernel (kept at 0 between calls)
    float* partial;     // [B*H][gstride][nchunk][d + 2] partial (m, l, acc) of each global row
    __nv_bfloat16* kg;  // [B*H][ngp][64] packed global keys (bf16 path)
    __nv_bfloat16* vg;  // [B*H][ngp][64] packed global values
    __nv_bfloat16* qg;  // [B*H][ngp][64] packed global queries, in gq_list order, zero past n_gq
};

struct PrepParams {
    const int32_t* gidx;  // [B][n_global] or null
    int32_t* band_cnt;    // band kernel merge tickets, zeroed here (n_band_cnt entries)
    int n_band_cnt;
    const uint8_t* pad;   // [B][T] or null
    const void* q;        // [B,H,T,d] (bf16 path: global query rows packed into qg)
    const void* k;        // [B,H,T,d] (bf16 path: packed into kg)
    const void* v;
    Workspace ws;
    uint32_t* status;
    int B, H, T, d, n_global, gstride, ngp, W;
    int pack;             // 1: write kg/vg/qg (bf16, d == 64)
};

struct GlobalRowParams {
    const void* q;
    const void* k;
    const void* v;
    void* out;
    const uint8_t* pad;
    Workspace ws;
    int B, H, T, d, gstride, nchunk;  // nchunk: partial states per global row
    int cpc;                          // bf16: 128-key chunks per CTA
    int ngp;                          // bf16: rows per (b, h) of the packed global queries
    float sl2;  // scale * log2(e)
    // Rows mode (sequence-sharded forward): the query rows come from q_rows
    // ([B*H][n_rows][d]) instead of q at the global positions, and the merge
    // of the chunks writes each row's partial state over these keys,
    // out_ml [B*H][n_rows][2] = (M, L) and out_acc [B*H][n_rows][d] =
    // sum_j 2^(s_j - M) v_j (s_j = scale * log2(e) * q . k_j), instead of y.
    const void* q_rows;
    float* out_ml;
    float* out_acc;
    int n_rows;
};

// Merge of partial row states from several key shards (sequence-sharded
// forward): parts p = 0..n_parts-1 of ml [p][B*H][n_rows][2] and acc
// [p][B*H][n_rows][d]; row a of sample b goes to out row pos[b][a] of
// [B*H][T_out][d] (pos < 0: not written).
struct MergeRowsParams {
    const float* ml;
    const float* acc;
    const int32_t* pos;
    void* out;
    int n_parts, BH, H, n_rows, d, T_out;
};

struct BandF32Params {
    const float* q;
    const float* k;
    const float* v;
    float* out;
    const uint8_t* pad;
    Workspace ws;
    int B, H, T, d, r, gstride, W;
    float sl2;
    int dil[kMaxHeads];  // per-head dilation
};

struct BandTcParams {
    CUtensorMap tm_q[kMaxDilKinds];
    CUtensorMap tm_k[kMaxDilKinds];
    CUtensorMap tm_v[kMaxDilKinds];
    CUtensorMap tm_kg;
    CUtensorMap tm_vg;
    __nv_bfloat16* out;
    const uint8_t* pad;
    const int32_t* gk_list;
    const int32_t* n_gk;
    const uint32_t* gbit;
    uint32_t* status;
    int32_t* cnt;  // [tiles][4][2] merge tickets and lanes done writing (zero between calls)
    float* part;   // [2 * grid_ctas] partial states of split tiles
    int B, H, T, r, W, gstride;
    float sl2;
    unsigned long long wait_ns;  // limit of every pipeline wait (drains keep their own)
    int test_stall;              // test hook: the producers publish nothing
    // The work sequence: per sample, heads in order; per head, residue
    // classes; per class, 128-query tiles; per tile, nbb band blocks then ngb
    // global blocks.  CTA s takes blocks [s*N/G, (s+1)*N/G).
    int n_blocks;        // N (< 2^31)
    int grid_ctas;       // G
    int blk_q, blk_rm;   // N = blk_q * G + blk_rm
    int blocks_per_b, tiles_per_b, ngb;  // ngb: blocks after the band blocks (random, then global keys)
    // The BigBird variant (random key blocks): rnd [B*H][nqb][n_rand] key
    // blocks of every 64-row query block; each tile's first nrb = 2 * n_rand
    // blocks after its band blocks are its two query blocks' draws (0: none).
    const int32_t* rnd;
    int n_rand, nrb, nqb;
    int dk_dil[kMaxDilKinds];
    int dk_rows[kMaxDilKinds];                          // rows per TMA box for that dilation
    int dk_class_blk[kMaxDilKinds][kMaxDilTma + 1];     // block offset of class c in a head of that kind
    int dk_class_tile[kMaxDilKinds][kMaxDilTma + 1];    // tile offset of class c
    int head_blk[kMaxHeads + 1];                        // block offset of head h in a sample
    int head_tile[kMaxHeads + 1];                       // tile offset of head h in a sample
    uint8_t head_dk[kMaxHeads];
};

}  // namespace lf
