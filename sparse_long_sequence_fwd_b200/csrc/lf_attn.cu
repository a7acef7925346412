// lf_attn.cu -- host side of liblfattn: argument checks, per-device
// workspace, TMA tensor maps and the launch sequence
//   K0 prep  ->  K1 band (bf16, tensor cores) | K3 band (fp32, CUDA cores)
//            ->  K2 global rows (only when n_global > 0)
// all on the caller's stream, nothing synchronised.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <atomic>
#include <mutex>
#include <vector>

#include "lf_attn.h"
#include "band_f32.cuh"
#include "band_tc.cuh"
#include "bwd.cuh"
#include "global_rows.cuh"
#include "lf_common.cuh"
#include "prep.cuh"

namespace {

using namespace lf;

constexpr int kMaxDevices = 64;
constexpr double kLog2e = 1.4426950408889634;

struct DeviceState {
    bool init = false;
    int sm_count = 0;
    uint32_t* status = nullptr;  // persistent device status word
    void* ws = nullptr;
    size_t ws_bytes = 0;
    void* io = nullptr;  // staging for lf_attn_fwd_host
    size_t io_bytes = 0;
    // The global-row kernels run on a low-priority side stream forked after
    // prep, so their CTAs fill the SMs the band kernel's CTAs leave as they
    // finish; null: everything runs in order on the caller's stream.
    cudaStream_t aux = nullptr;
    cudaEvent_t ev_fork = nullptr, ev_join = nullptr;
    // lf_attn_fwd_host: copy-in / copy-out streams and per-slice events, so the
    // copies of one slice overlap the kernels of another.  Four slices: every copy
    // costs a fixed set-up on top of its bytes, which more, smaller slices pay
    // more often than their overlap saves (measured on the bench workloads).
    static constexpr int kMaxSlices = 4;
    cudaStream_t cin = nullptr, cout = nullptr;
    cudaEvent_t ev_in[kMaxSlices] = {}, ev_done[kMaxSlices] = {};
};

std::mutex g_mu;
DeviceState g_dev[kMaxDevices];
PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
thread_local int t_last_launches = 0;
// Test hooks (lf_attn_test_hooks): the band kernel's pipeline-wait limit
// (0: LF_WAIT_NS) and whether its producers stop before their first load.
std::atomic<unsigned long long> g_test_wait_ns{0};
std::atomic<int> g_test_stall{0};

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

// Band kernel: at most this many CTAs (two per SM of a 148-SM B200; larger
// GPUs run it on 296 CTAs too), so its partial-state region has a size
// known without a device.
constexpr int kMaxBandCtas = 296;
// ... for a head dimension (one CTA per SM at HD = 128)
constexpr int max_band_ctas(int d) { return d == 64 ? kMaxBandCtas : kMaxBandCtas / 2; }
constexpr int kFewGlobals = 4;        // global tokens up to which ...
constexpr int kFewGlobalsSlots = 24;  // ... the band kernel leaves this many CTA slots free

struct Layout {
    size_t off_ngq, off_ngk, off_gq, off_gk, off_gbit, off_cnt, off_part, off_kg, off_vg, off_qg, off_bcnt, off_bpart,
        total;
    int W, gstride, nchunk, ngp, cpc;  // nchunk: partial states per global row
    int gr_kpw;                        // bf16 global rows: keys per warp slice of a chunk
    long long band_tiles;             // upper bound on the band kernel's tiles (its merge tickets)
};

Layout make_layout(int B, int H, int T, int d, int n_global, lf_dtype dtype) {
    Layout L{};
    L.W = (T + 31) / 32;
    L.gstride = std::max(1, std::min(n_global, T));
    if (dtype != LF_F32 && d == 64) {
        // tensor-core global rows: 128-key chunks, cpc per CTA, about three CTAs
        // per SM of a 148-SM B200 (each holds a two-stage ring of 72 KB)
        const int nblk = (T + kGrKeys - 1) / kGrKeys;
        // Warps split each chunk's keys when there are few global queries, but
        // combining the slices only pays off when a CTA takes two chunks or more.
        // With few global tokens the band kernel leaves CTA slots free (launch_all),
        // and fewer, longer global-row CTAs (about two per SM) finish sooner in them.
        const long budget = n_global <= kFewGlobals ? 296 : 444;
        auto chunks_per_cta = [&](int kpw) {
            const int rows = kpw / 2;  // global-query slots per CTA
            const long units = long(nblk) * B * H * ((L.gstride + rows - 1) / rows);
            return static_cast<int>(std::max(1L, std::min<long>(nblk, (units + budget - 1) / budget)));
        };
        L.gr_kpw = gr_kpw(L.gstride);
        L.cpc = chunks_per_cta(L.gr_kpw);
        if (L.cpc == 1 && L.gr_kpw != kGrKeys) {
            L.gr_kpw = kGrKeys;
            L.cpc = chunks_per_cta(L.gr_kpw);
        }
        L.nchunk = (nblk + L.cpc - 1) / L.cpc;
        while (L.nchunk > kMaxSplits) L.nchunk = (nblk + ++L.cpc - 1) / L.cpc;
    } else {
        L.cpc = 1;
        L.nchunk = (T + kChunk - 1) / kChunk;
    }
    L.ngp = (L.gstride + 15) & ~15;
    size_t o = 0;
    L.off_ngq = o; o = align256(o + sizeof(int32_t) * B);
    L.off_ngk = o; o = align256(o + sizeof(int32_t) * B);
    L.off_gq = o; o = align256(o + sizeof(int32_t) * size_t(B) * L.gstride);
    L.off_gk = o; o = align256(o + sizeof(int32_t) * size_t(B) * L.gstride);
    L.off_gbit = o; o = align256(o + sizeof(uint32_t) * size_t(B) * L.W);
    L.off_cnt = o; o = align256(o + sizeof(int32_t) * size_t(B) * H);
    L.off_part = o;
    if (n_global > 0) o = align256(o + sizeof(float) * size_t(B) * H * L.gstride * L.nchunk * (d + 2));
    L.off_kg = o;
    L.off_vg = o;
    L.off_qg = o;
    if (dtype != LF_F32 && n_global > 0) {
        const size_t kgb = sizeof(__nv_bfloat16) * size_t(B) * H * L.ngp * d;
        L.off_vg = align256(o + kgb);
        L.off_qg = align256(L.off_vg + kgb);
        o = align256(L.off_qg + kgb);
    }
    L.off_bcnt = o;
    L.off_bpart = o;
    L.band_tiles = 0;
    if (dtype != LF_F32) {
        // every head has at most ceil(T / 128) + kMaxDilTma - 1 tiles (one per residue class more)
        L.band_tiles = (long long)B * H * ((T + kBM - 1) / kBM + kMaxDilTma - 1);
        L.off_bpart = align256(o + sizeof(int32_t) * size_t(L.band_tiles) * 8);
        const size_t part_floats = d == 64 ? BandCfg<64>::kPartFloats : BandCfg<128>::kPartFloats;
        o = align256(L.off_bpart + sizeof(float) * size_t(2 * max_band_ctas(d)) * part_floats);
    }
    L.total = std::max<size_t>(o, 256);
    return L;
}

bool is_capturing(cudaStream_t s) {
    cudaStreamCaptureStatus st = cudaStreamCaptureStatusNone;
    if (cudaStreamIsCapturing(s, &st) != cudaSuccess) return false;
    return st != cudaStreamCaptureStatusNone;
}

// Shared-memory limits of every kernel, and the carveout that lets two band
// CTAs share an SM.
lf_status set_kernel_attributes() {
    const int prep_max = (kMaxT / 32 + 2 * kPrepThreads + 2 * kMaxGlobal) * 4;
    const int gr_max = (kChunk * 128 + 128 + kChunk + 32 + kGrThreads) * 4;
    for (auto kern : {band_tc_kernel<false, false, 64>, band_tc_kernel<true, false, 64>,
                      band_tc_kernel<false, true, 64>, band_tc_kernel<true, true, 64>,
                      band_tc_kernel<false, false, 64, true>, band_tc_kernel<true, false, 64, true>,
                      band_tc_kernel<false, true, 64, true>, band_tc_kernel<true, true, 64, true>})
        if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, BandCfg<64>::kSmem) !=
                cudaSuccess ||
            cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout,
                                 cudaSharedmemCarveoutMaxShared) != cudaSuccess)
            return LF_ERR_CUDA;
    for (auto kern : {band_tc_kernel<false, false, 128>, band_tc_kernel<true, false, 128>,
                      band_tc_kernel<false, true, 128>, band_tc_kernel<true, true, 128>})
        if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, BandCfg<128>::kSmem) !=
                cudaSuccess ||
            cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout,
                                 cudaSharedmemCarveoutMaxShared) != cudaSuccess)
            return LF_ERR_CUDA;
    for (auto kern : {global_rows_mma_kernel<32, false>, global_rows_mma_kernel<64, false>,
                      global_rows_mma_kernel<128, false>, global_rows_mma_kernel<32, true>,
                      global_rows_mma_kernel<64, true>, global_rows_mma_kernel<128, true>})
        if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kGrSmem) != cudaSuccess)
            return LF_ERR_CUDA;
    for (auto kern : {global_rows_kernel<float, 32, true>, global_rows_kernel<float, 64, true>,
                      global_rows_kernel<float, 128, true>, global_rows_kernel<__nv_bfloat16, 32, true>,
                      global_rows_kernel<__nv_bfloat16, 64, true>, global_rows_kernel<__nv_bfloat16, 128, true>,
                      global_rows_kernel<__half, 32, true>, global_rows_kernel<__half, 64, true>,
                      global_rows_kernel<__half, 128, true>})
        if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, gr_max) != cudaSuccess)
            return LF_ERR_CUDA;
    if (cudaFuncSetAttribute(prep_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, prep_max) != cudaSuccess ||
        cudaFuncSetAttribute(global_rows_kernel<float, 128>, cudaFuncAttributeMaxDynamicSharedMemorySize, gr_max) !=
            cudaSuccess ||
        cudaFuncSetAttribute(global_rows_kernel<float, 64>, cudaFuncAttributeMaxDynamicSharedMemorySize, gr_max) !=
            cudaSuccess ||
        cudaFuncSetAttribute(global_rows_kernel<float, 32>, cudaFuncAttributeMaxDynamicSharedMemorySize, gr_max) !=
            cudaSuccess ||
        cudaFuncSetAttribute(global_rows_kernel<__nv_bfloat16, 128>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             gr_max) != cudaSuccess ||
        cudaFuncSetAttribute(global_rows_kernel<__half, 128>, cudaFuncAttributeMaxDynamicSharedMemorySize, gr_max) !=
            cudaSuccess)
        return LF_ERR_CUDA;
    return LF_OK;
}

lf_status device_state(DeviceState** out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return LF_ERR_CUDA;
    DeviceState& s = g_dev[dev];
    if (!s.init) {
        cudaDeviceProp prop;
        if (cudaGetDeviceProperties(&prop, dev) != cudaSuccess) return LF_ERR_CUDA;
        if (prop.major < 10) return LF_ERR_UNSUPPORTED;
        s.sm_count = prop.multiProcessorCount;
        if (cudaMalloc(&s.status, 256) != cudaSuccess) return LF_ERR_NO_MEMORY;
        if (cudaMemset(s.status, 0, 256) != cudaSuccess) return LF_ERR_CUDA;
        if (set_kernel_attributes() != LF_OK) return LF_ERR_CUDA;
        int least = 0, greatest = 0;
        if (cudaDeviceGetStreamPriorityRange(&least, &greatest) != cudaSuccess ||
            cudaStreamCreateWithPriority(&s.aux, cudaStreamNonBlocking, least) != cudaSuccess ||
            cudaEventCreateWithFlags(&s.ev_fork, cudaEventDisableTiming) != cudaSuccess ||
            cudaEventCreateWithFlags(&s.ev_join, cudaEventDisableTiming) != cudaSuccess ||
            cudaStreamCreateWithFlags(&s.cin, cudaStreamNonBlocking) != cudaSuccess ||
            cudaStreamCreateWithFlags(&s.cout, cudaStreamNonBlocking) != cudaSuccess)
            return LF_ERR_CUDA;
        for (int a = 0; a < DeviceState::kMaxSlices; ++a)
            if (cudaEventCreateWithFlags(&s.ev_in[a], cudaEventDisableTiming) != cudaSuccess ||
                cudaEventCreateWithFlags(&s.ev_done[a], cudaEventDisableTiming) != cudaSuccess)
                return LF_ERR_CUDA;
        s.init = true;
    }
    *out = &s;
    return LF_OK;
}

lf_status grow(void** buf, size_t* have, size_t need, cudaStream_t stream) {
    if (*have >= need) return LF_OK;
    if (is_capturing(stream)) return LF_ERR_NO_MEMORY;
    if (*buf) {
        cudaFree(*buf);  // synchronises the device: no kernel still uses it
        *buf = nullptr;
        *have = 0;
    }
    if (cudaMalloc(buf, need) != cudaSuccess) {
        *buf = nullptr;
        return LF_ERR_NO_MEMORY;
    }
    if (cudaMemset(*buf, 0, need) != cudaSuccess) return LF_ERR_CUDA;
    *have = need;
    return LF_OK;
}

lf_status get_encoder() {
    if (g_encode) return LF_OK;
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess || !fn)
        return LF_ERR_CUDA;
    g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
    return LF_OK;
}

// 3-D map of 16-bit elements (bf16, or f16 when half) over [d, rows, B*H]
// (d = 64 or 128) with a 128-byte swizzle; box = 64 x (rows_per_box *
// stride) x 1 (one 64-column sub-tile; with d = 128 two boxes per row, at
// x = 0 and 64), element stride `stride` along the rows.
lf_status encode_rows_map(CUtensorMap* tm, const void* base, uint64_t rows, uint64_t bh, uint32_t rows_per_box,
                          uint32_t stride, bool half, int d) {
    cuuint64_t gdim[3] = {static_cast<cuuint64_t>(d), rows, bh};
    cuuint64_t gstr[2] = {static_cast<cuuint64_t>(d) * 2, rows * d * 2};
    cuuint32_t box[3] = {64, rows_per_box * stride, 1};
    cuuint32_t estr[3] = {1, stride, 1};
    CUresult r = g_encode(tm, half ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), gdim, gstr, box, estr,
                          CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                          CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? LF_OK : LF_ERR_CUDA;
}

lf_status check_args(const void* q, const void* k, const void* v, void* out, int B, int H, int T, int d, int r,
                     const int32_t* dil, const int32_t* gidx, int n_global, float scale, lf_dtype dtype) {
    if (!q || !k || !v || !out) return LF_ERR_INVALID_ARG;
    if (B <= 0 || H <= 0 || T <= 0 || d <= 0 || r < 0 || n_global < 0) return LF_ERR_INVALID_ARG;
    if (n_global > 0 && !gidx) return LF_ERR_INVALID_ARG;
    if (n_global == 0 && gidx) return LF_ERR_INVALID_ARG;
    if (!std::isfinite(scale)) return LF_ERR_INVALID_ARG;
    if (dtype != LF_F32 && dtype != LF_BF16 && dtype != LF_F16) return LF_ERR_INVALID_ARG;
    if (dil)
        for (int h = 0; h < H; ++h)
            if (dil[h] < 1) return LF_ERR_INVALID_ARG;
    const uint64_t n = uint64_t(B) * uint64_t(H) * uint64_t(T) * uint64_t(d);
    if (n / uint64_t(d) / uint64_t(T) / uint64_t(H) != uint64_t(B) || n > (uint64_t(1) << 40))
        return LF_ERR_INVALID_ARG;
    for (const void* p : {q, k, v, static_cast<const void*>(out)})
        if (reinterpret_cast<uintptr_t>(p) & 15u) return LF_ERR_INVALID_ARG;
    if (T > kMaxT || n_global > kMaxGlobal) return LF_ERR_UNSUPPORTED;
    if (uint64_t(B) * H > 0x7fffffffull || uint64_t(B) * H * T > (uint64_t(1) << 31) * 64) return LF_ERR_UNSUPPORTED;
    if (dtype == LF_F32 && d > 128) return LF_ERR_UNSUPPORTED;
    if (n_global > 0 && uint64_t(B) * H > 65535u) return LF_ERR_UNSUPPORTED;  // global-row grid.y
    if (dtype != LF_F32) {  // the tensor-core path, bf16 or f16
        if ((d != 64 && d != 128) || H > kMaxHeads) return LF_ERR_UNSUPPORTED;
        int kinds[kMaxDilKinds];
        int nk = 0;
        for (int h = 0; h < H; ++h) {
            const int dl = dil ? dil[h] : 1;
            if (dl > kMaxDilTma) return LF_ERR_UNSUPPORTED;
            bool seen = false;
            for (int a = 0; a < nk; ++a) seen |= kinds[a] == dl;
            if (!seen) {
                if (nk == kMaxDilKinds) return LF_ERR_UNSUPPORTED;
                kinds[nk++] = dl;
            }
        }
    }
    return LF_OK;
}

// Groups the heads by dilation (one set of tensor maps per distinct value).
int assign_kinds(BandTcParams& bp, int H, const int32_t* dil, int* kind_of_head) {
    int nk = 0;
    for (int h = 0; h < H; ++h) {
        const int dl = dil ? dil[h] : 1;
        int kidx = -1;
        for (int a = 0; a < nk; ++a)
            if (bp.dk_dil[a] == dl) kidx = a;
        if (kidx < 0) {
            kidx = nk++;
            bp.dk_dil[kidx] = dl;
            bp.dk_rows[kidx] = dl <= 4 ? 64 : 32;  // TMA box rows x stride <= 256
        }
        kind_of_head[h] = kidx;
    }
    for (int a = nk; a < kMaxDilKinds; ++a) {
        bp.dk_dil[a] = 1;
        bp.dk_rows[a] = 64;
    }
    return nk;
}

// The band kernel's work sequence and its split over at most max_ctas CTAs:
// per (kind, class) and per head, block and tile offsets (band_tc.cuh).
lf_status band_schedule(BandTcParams& bp, int B, int H, int T, int r_eff, int ngb, const int* kind_of_head,
                        int max_ctas, long long tile_cap) {
    bp.ngb = ngb;
    for (int kd = 0; kd < kMaxDilKinds; ++kd) {
        const int dl = bp.dk_dil[kd];
        bp.dk_class_blk[kd][0] = 0;
        bp.dk_class_tile[kd][0] = 0;
        long long blk = 0, tiles = 0;
        for (int c = 0; c < kMaxDilTma; ++c) {
            if (c < dl) {
                const int Tc = (T - c + dl - 1) / dl;
                const int nt = (Tc + kBM - 1) / kBM;
                for (int t = 0; t < nt; ++t) {
                    int kbase = 0, kb_lo = 0, nbb = 0;
                    tile_band(Tc, r_eff, t, kbase, kb_lo, nbb);
                    blk += nbb + ngb;
                }
                tiles += nt;
            }
            if (blk > INT32_MAX) return LF_ERR_UNSUPPORTED;
            bp.dk_class_blk[kd][c + 1] = static_cast<int>(blk);
            bp.dk_class_tile[kd][c + 1] = static_cast<int>(tiles);
        }
    }
    long long hb = 0, ht = 0;
    for (int h = 0; h < H; ++h) {
        const int kd = kind_of_head[h];
        bp.head_blk[h] = static_cast<int>(hb);
        bp.head_tile[h] = static_cast<int>(ht);
        bp.head_dk[h] = static_cast<uint8_t>(kd);
        hb += bp.dk_class_blk[kd][bp.dk_dil[kd]];
        ht += bp.dk_class_tile[kd][bp.dk_dil[kd]];
        if (hb > INT32_MAX) return LF_ERR_UNSUPPORTED;
    }
    for (int h = H; h <= kMaxHeads; ++h) {
        bp.head_blk[h] = static_cast<int>(hb);
        bp.head_tile[h] = static_cast<int>(ht);
    }
    bp.H = H;
    bp.T = T;
    bp.r = r_eff;
    bp.blocks_per_b = static_cast<int>(hb);
    bp.tiles_per_b = static_cast<int>(ht);
    const long long nblk = static_cast<long long>(B) * hb;
    if (nblk >= INT32_MAX || static_cast<long long>(B) * ht > tile_cap) return LF_ERR_UNSUPPORTED;
    bp.n_blocks = static_cast<int>(nblk);
    bp.grid_ctas = static_cast<int>(std::min<long long>(nblk, max_ctas));
    bp.blk_q = bp.n_blocks / bp.grid_ctas;
    bp.blk_rm = bp.n_blocks % bp.grid_ctas;
    return LF_OK;
}

lf_status launch_all(const void* q, const void* k, const void* v, void* out, int B, int H, int T, int d, int r,
                     const int32_t* dil, const int32_t* gidx, int n_global, const uint8_t* pad, float scale,
                     lf_dtype dtype, cudaStream_t stream, DeviceState* ds, uint32_t stages = 7u,
                     const int32_t* rnd = nullptr, int n_rand = 0) {
    const Layout L = make_layout(B, H, T, d, n_global, dtype);
    lf_status st = grow(&ds->ws, &ds->ws_bytes, L.total, stream);
    if (st != LF_OK) return st;
    uint8_t* base = static_cast<uint8_t*>(ds->ws);
    Workspace ws;
    ws.n_gq = reinterpret_cast<int32_t*>(base + L.off_ngq);
    ws.n_gk = reinterpret_cast<int32_t*>(base + L.off_ngk);
    ws.gq_list = reinterpret_cast<int32_t*>(base + L.off_gq);
    ws.gk_list = reinterpret_cast<int32_t*>(base + L.off_gk);
    ws.gbit = reinterpret_cast<uint32_t*>(base + L.off_gbit);
    ws.counters = reinterpret_cast<int32_t*>(base + L.off_cnt);
    ws.partial = reinterpret_cast<float*>(base + L.off_part);
    ws.kg = reinterpret_cast<__nv_bfloat16*>(base + L.off_kg);
    ws.vg = reinterpret_cast<__nv_bfloat16*>(base + L.off_vg);
    ws.qg = reinterpret_cast<__nv_bfloat16*>(base + L.off_qg);
    const int r_eff = std::min(r, T);  // a window wider than the sequence changes nothing
    const bool half = dtype == LF_F16;
    const float sl2 = static_cast<float>(double(scale) * kLog2e);
    int launches = 0;

    // K0
    PrepParams pp;
    pp.gidx = gidx;
    pp.pad = pad;
    pp.q = q;
    pp.k = k;
    pp.v = v;
    pp.ws = ws;
    pp.status = ds->status;
    pp.B = B; pp.H = H; pp.T = T; pp.d = d;
    pp.n_global = n_global;
    pp.gstride = L.gstride;
    pp.ngp = L.ngp;
    pp.W = L.W;
    pp.pack = (dtype != LF_F32 && n_global > 0) ? 1 : 0;
    pp.band_cnt = reinterpret_cast<int32_t*>(base + L.off_bcnt);
    pp.n_band_cnt = static_cast<int>(L.band_tiles * 8);
    const size_t prep_smem = size_t(L.W + 2 * kPrepThreads + 2 * L.gstride) * 4;
    if (stages & 1u) {
        prep_kernel<<<B * H, kPrepThreads, prep_smem, stream>>>(pp);
        ++launches;
    }
    // The global rows depend on prep only: with a side stream they are forked
    // here and joined after the band kernel, which is launched first and so
    // takes the SMs first.
    const bool global_stage = n_global > 0 && (stages & 4u);
    const bool fork = global_stage && (stages & 2u) && dtype != LF_F32 && ds->aux != nullptr;
    if (fork && cudaEventRecord(ds->ev_fork, stream) != cudaSuccess) return LF_ERR_CUDA;

    if (!(stages & 2u)) {
        // band stage skipped
    } else if (dtype == LF_F32) {
        // K3: fp32 band rows on CUDA cores
        BandF32Params bp;
        bp.q = static_cast<const float*>(q);
        bp.k = static_cast<const float*>(k);
        bp.v = static_cast<const float*>(v);
        bp.out = static_cast<float*>(out);
        bp.pad = pad;
        bp.ws = ws;
        bp.B = B; bp.H = H; bp.T = T; bp.d = d; bp.r = r_eff;
        bp.gstride = L.gstride;
        bp.W = L.W;
        bp.sl2 = sl2;
        for (int h = 0; h < kMaxHeads; ++h) bp.dil[h] = (h < H && dil) ? dil[h] : 1;
        const long rows = long(B) * H * T;
        const unsigned grid = static_cast<unsigned>((rows + kBandF32Warps - 1) / kBandF32Warps);
        if (d <= 16) band_f32_kernel<16><<<grid, kBandF32Warps * 32, 0, stream>>>(bp);
        else if (d <= 32) band_f32_kernel<32><<<grid, kBandF32Warps * 32, 0, stream>>>(bp);
        else if (d <= 64) band_f32_kernel<64><<<grid, kBandF32Warps * 32, 0, stream>>>(bp);
        else band_f32_kernel<128><<<grid, kBandF32Warps * 32, 0, stream>>>(bp);
        ++launches;
    } else {
        // K1: bf16 or f16 band rows on the tensor cores
        st = get_encoder();
        if (st != LF_OK) return st;
        static thread_local BandTcParams bp;  // large (tensor maps); filled per call
        std::memset(&bp, 0, sizeof(bp));
        int kind_of_head[kMaxHeads];
        const int nk = assign_kinds(bp, H, dil, kind_of_head);
        for (int kd = 0; kd < nk; ++kd) {
            const int dl = bp.dk_dil[kd];
            const uint32_t R = static_cast<uint32_t>(bp.dk_rows[kd]);
            if ((st = encode_rows_map(&bp.tm_q[kd], q, T, uint64_t(B) * H, R, dl, half, d)) != LF_OK ||
                (st = encode_rows_map(&bp.tm_k[kd], k, T, uint64_t(B) * H, R, dl, half, d)) != LF_OK ||
                (st = encode_rows_map(&bp.tm_v[kd], v, T, uint64_t(B) * H, R, dl, half, d)) != LF_OK)
                return st;
        }
        for (int a = nk; a < kMaxDilKinds; ++a) {  // unused slots: valid maps, never read
            bp.tm_q[a] = bp.tm_q[0];
            bp.tm_k[a] = bp.tm_k[0];
            bp.tm_v[a] = bp.tm_v[0];
        }
        if (n_global > 0) {
            if ((st = encode_rows_map(&bp.tm_kg, ws.kg, L.ngp, uint64_t(B) * H, kBN, 1, half, d)) != LF_OK ||
                (st = encode_rows_map(&bp.tm_vg, ws.vg, L.ngp, uint64_t(B) * H, kBN, 1, half, d)) != LF_OK)
                return st;
        } else {
            bp.tm_kg = bp.tm_k[0];
            bp.tm_vg = bp.tm_v[0];
        }
        // after each tile's band blocks: 2 * n_rand random key blocks (the BigBird variant), then
        // the global-key blocks
        const int nrb = 2 * n_rand;
        bp.rnd = rnd;
        bp.n_rand = n_rand;
        bp.nrb = nrb;
        bp.nqb = (T + kBN - 1) / kBN;
        // With a few global rows (their stage is short), some SM slots are left to the
        // global-row kernel from the start instead of only in the band kernel's tail.  (The
        // same launch shape whichever stages or entry point run, so a band-only call times
        // the same kernel and every entry point gives the same bits.)
        int band_ctas = std::min((d == 64 ? BandCfg<64>::kCtasPerSm : BandCfg<128>::kCtasPerSm) * ds->sm_count,
                                 max_band_ctas(d));
        if (d == 64 && n_global > 0 && n_global <= kFewGlobals) band_ctas -= kFewGlobalsSlots;
        if ((st = band_schedule(bp, B, H, T, r_eff, nrb + (n_global > 0 ? (L.gstride + kBN - 1) / kBN : 0), kind_of_head,
                                band_ctas, L.band_tiles)) != LF_OK)
            return st;
        bp.cnt = reinterpret_cast<int32_t*>(base + L.off_bcnt);
        bp.part = reinterpret_cast<float*>(base + L.off_bpart);
        bp.out = static_cast<__nv_bfloat16*>(out);
        bp.pad = pad;
        bp.gk_list = ws.gk_list;
        bp.n_gk = ws.n_gk;
        bp.gbit = ws.gbit;
        bp.status = ds->status;
        bp.B = B; bp.H = H; bp.T = T; bp.r = r_eff;
        bp.W = L.W;
        bp.gstride = L.gstride;
        bp.sl2 = sl2;
        const unsigned long long wl = g_test_wait_ns.load();
        bp.wait_ns = wl ? wl : LF_WAIT_NS;
        bp.test_stall = g_test_stall.load();
        const int grid = bp.grid_ctas;  // persistent: two CTAs per SM (one at d = 128)
        // right after prep on the same stream, launched as its programmatic dependent: the
        // band kernel's set-up (barriers, TMEM, tensor-map prefetch) overlaps prep
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(static_cast<unsigned>(grid));
        cfg.blockDim = dim3(kBandThreads);
        cfg.dynamicSmemBytes = d == 64 ? BandCfg<64>::kSmem : BandCfg<128>::kSmem;
        cfg.stream = stream;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[0].val.programmaticStreamSerializationAllowed = (stages & 1u) ? 1 : 0;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        // more than 32 global tokens: the instantiation whose global-key dedup searches
        void (*kern)(BandTcParams) =
            n_rand > 0  // (d == 64 only)
                ? (n_global > 32 ? (half ? band_tc_kernel<true, true, 64, true> : band_tc_kernel<true, false, 64, true>)
                                 : (half ? band_tc_kernel<false, true, 64, true> : band_tc_kernel<false, false, 64, true>))
            : d == 64 ? (n_global > 32 ? (half ? band_tc_kernel<true, true, 64> : band_tc_kernel<true, false, 64>)
                                       : (half ? band_tc_kernel<false, true, 64> : band_tc_kernel<false, false, 64>))
                      : (n_global > 32 ? (half ? band_tc_kernel<true, true, 128> : band_tc_kernel<true, false, 128>)
                                       : (half ? band_tc_kernel<false, true, 128> : band_tc_kernel<false, false, 128>));
        if (cudaLaunchKernelEx(&cfg, kern, bp) != cudaSuccess) return LF_ERR_CUDA;
        ++launches;
    }

    if (global_stage) {
        cudaStream_t gs = stream;
        if (fork) {
            if (cudaStreamWaitEvent(ds->aux, ds->ev_fork, 0) != cudaSuccess) return LF_ERR_CUDA;
            gs = ds->aux;
        }
        // K2: rows of the global queries
        GlobalRowParams gp;
        gp.q = q;
        gp.k = k;
        gp.v = v;
        gp.out = out;
        gp.pad = pad;
        gp.ws = ws;
        gp.B = B; gp.H = H; gp.T = T; gp.d = d;
        gp.gstride = L.gstride;
        gp.nchunk = L.nchunk;
        gp.sl2 = sl2;
        gp.cpc = L.cpc;
        gp.ngp = L.ngp;
        if (dtype != LF_F32 && d == 128) {
            // 16-bit inputs with d = 128: the CUDA-core global-row kernel (chunks of keys, the
            // last chunk of a (b, h) merges)
            const dim3 grid(L.nchunk, B * H);
            const size_t smem = size_t(kChunk * 128 + 128 + kChunk + 32 + kGrThreads) * 4;
            if (half) global_rows_kernel<__half, 128><<<grid, kGrThreads, smem, gs>>>(gp);
            else global_rows_kernel<__nv_bfloat16, 128><<<grid, kGrThreads, smem, gs>>>(gp);
            ++launches;
        } else if (dtype != LF_F32) {
            // key splits x (b, h) x groups of kpw / 2 global rows, then the merge of the splits
            const int kpw = L.gr_kpw, rows = kpw / 2;
            const dim3 grid(L.nchunk, B * H, (L.gstride + rows - 1) / rows);
            void (*grk)(GlobalRowParams) =
                kpw == 32 ? (half ? global_rows_mma_kernel<32, true> : global_rows_mma_kernel<32, false>)
                : kpw == 64 ? (half ? global_rows_mma_kernel<64, true> : global_rows_mma_kernel<64, false>)
                            : (half ? global_rows_mma_kernel<128, true> : global_rows_mma_kernel<128, false>);
            grk<<<grid, kGrWarps * 32, kGrSmem, gs>>>(gp);
            // the merge is the split kernel's programmatic dependent: it launches while the
            // splits finish and waits for them (griddepcontrol.wait) before reading
            cudaLaunchConfig_t mc = {};
            mc.gridDim = dim3(static_cast<unsigned>(L.gstride), static_cast<unsigned>(B * H));
            mc.blockDim = dim3(64);
            mc.stream = gs;
            cudaLaunchAttribute mattr[1];
            mattr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
            mattr[0].val.programmaticStreamSerializationAllowed = 1;
            mc.attrs = mattr;
            mc.numAttrs = 1;
            if (cudaLaunchKernelEx(&mc, half ? global_rows_merge_kernel<true> : global_rows_merge_kernel<false>, gp) !=
                cudaSuccess)
                return LF_ERR_CUDA;
            launches += 2;
        } else {
            const dim3 grid(L.nchunk, B * H);
            const int DP = d <= 32 ? 32 : (d <= 64 ? 64 : 128);
            const size_t smem = size_t(kChunk * DP + DP + kChunk + 32 + kGrThreads) * 4;
            if (DP == 32) global_rows_kernel<float, 32><<<grid, kGrThreads, smem, stream>>>(gp);
            else if (DP == 64) global_rows_kernel<float, 64><<<grid, kGrThreads, smem, stream>>>(gp);
            else global_rows_kernel<float, 128><<<grid, kGrThreads, smem, stream>>>(gp);
            ++launches;
        }
        if (fork && (cudaEventRecord(ds->ev_join, ds->aux) != cudaSuccess ||
                     cudaStreamWaitEvent(stream, ds->ev_join, 0) != cudaSuccess))
            return LF_ERR_CUDA;
    }
    if (cudaGetLastError() != cudaSuccess) return LF_ERR_CUDA;
    t_last_launches = launches;
    return LF_OK;
}

// ------------------------------------------------------------------------
// Allocation-free variant.  Some callers cannot call cudaMalloc at all: code
// that runs while a CUDA graph is being captured in global mode, processes
// under a strict memory budget or a custom pool that forbids the runtime's
// allocator, or embedded runtimes that reserve all device memory up front.
// For them lf_attn_fwd_static runs the same kernels on a fixed scratch area
// that the module image carries: one file-scope __device__ array per GPU that
// loads this library, held until the process exits.  Its first 256 bytes
// take the device-side flags of this variant; the rest is the workspace.
constexpr size_t kStaticScratchBytes = size_t(32) << 20;  // 32 MiB
static __device__ __align__(256) uint8_t g_static_scratch[kStaticScratchBytes];

struct StaticState {
    bool init = false;
    int sm_count = 0;
    uint8_t* scratch = nullptr;  // device address of g_static_scratch on this device
};
StaticState g_static[kMaxDevices];

// Once per device, with that device current: kernel attributes and the
// device address of the scratch array (the host-side symbol is only a
// stand-in and must never reach a kernel).  Allocates nothing.
lf_status static_state(StaticState** out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return LF_ERR_CUDA;
    StaticState& s = g_static[dev];
    if (!s.init) {
        cudaDeviceProp prop;
        if (cudaGetDeviceProperties(&prop, dev) != cudaSuccess) return LF_ERR_CUDA;
        if (prop.major < 10) return LF_ERR_UNSUPPORTED;
        void* ptr = nullptr;
        if (cudaGetSymbolAddress(&ptr, g_static_scratch) != cudaSuccess || !ptr) return LF_ERR_CUDA;
        if (set_kernel_attributes() != LF_OK) return LF_ERR_CUDA;
        s.sm_count = prop.multiProcessorCount;
        s.scratch = static_cast<uint8_t*>(ptr);
        s.init = true;
    }
    *out = &s;
    return LF_OK;
}

}  // namespace

extern "C" {

lf_status lf_attn_fwd(const void* q, const void* k, const void* v, void* out, int B, int H, int T, int d, int r,
                      const int32_t* dil, const int32_t* global_idx, int n_global, const uint8_t* key_pad_mask,
                      float scale, lf_dtype dtype, void* stream) {
    lf_status st = check_args(q, k, v, out, B, H, T, d, r, dil, global_idx, n_global, scale, dtype);
    if (st != LF_OK) return st;
    std::lock_guard<std::mutex> lock(g_mu);
    DeviceState* ds = nullptr;
    if ((st = device_state(&ds)) != LF_OK) return st;
    return launch_all(q, k, v, out, B, H, T, d, r, dil, global_idx, n_global, key_pad_mask, scale, dtype,
                      static_cast<cudaStream_t>(stream), ds);
}

lf_status lf_attn_fwd_rand(const void* q, const void* k, const void* v, void* out, int B, int H, int T, int d,
                           int r, const int32_t* dil, const int32_t* global_idx, int n_global,
                           const uint8_t* key_pad_mask, float scale, lf_dtype dtype, const int32_t* rand_blocks,
                           int n_rand, void* stream) {
    lf_status st = check_args(q, k, v, out, B, H, T, d, r, dil, global_idx, n_global, scale, dtype);
    if (st != LF_OK) return st;
    if (n_rand < 0 || n_rand > kMaxRand || (n_rand > 0) != (rand_blocks != nullptr) ||
        (reinterpret_cast<uintptr_t>(rand_blocks) & 3u))
        return LF_ERR_INVALID_ARG;
    if (n_rand > 0) {
        if (dtype == LF_F32 || d != 64) return LF_ERR_UNSUPPORTED;
        if (dil)
            for (int h = 0; h < H; ++h)
                if (dil[h] != 1) return LF_ERR_UNSUPPORTED;
    }
    std::lock_guard<std::mutex> lock(g_mu);
    DeviceState* ds = nullptr;
    if ((st = device_state(&ds)) != LF_OK) return st;
    return launch_all(q, k, v, out, B, H, T, d, r, dil, global_idx, n_global, key_pad_mask, scale, dtype,
                      static_cast<cudaStream_t>(stream), ds, 7u, rand_blocks, n_rand);
}

lf_status lf_attn_bwd(const void* q, const void* k, const void* v, const void* y, const void* dy, float* dq,
                       float* dk, float* dv, int B, int H, int T, int d, int r, const int32_t* dil,
                       const int32_t* global_idx, int n_global, const uint8_t* key_pad_mask, float scale,
                       lf_dtype dtype, void* stream) {
    if (!q || !k || !v || !y || !dy || !dq || !dk || !dv) return LF_ERR_INVALID_ARG;
    if (B <= 0 || H <= 0 || T <= 0 || d <= 0 || r < 0 || n_global < 0 || !std::isfinite(scale))
        return LF_ERR_INVALID_ARG;
    if ((n_global > 0) != (global_idx != nullptr)) return LF_ERR_INVALID_ARG;
    if (dtype != LF_F32 && dtype != LF_BF16 && dtype != LF_F16) return LF_ERR_INVALID_ARG;
    if (dil)
        for (int h = 0; h < H; ++h)
            if (dil[h] < 1) return LF_ERR_INVALID_ARG;
    for (const void* p : {q, k, v, y, dy, static_cast<const void*>(dq), static_cast<const void*>(dk),
                          static_cast<const void*>(dv)})
        if (reinterpret_cast<uintptr_t>(p) & 15u) return LF_ERR_INVALID_ARG;
    const uint64_t n = uint64_t(B) * uint64_t(H) * uint64_t(T) * uint64_t(d);
    if (n / uint64_t(d) / uint64_t(T) / uint64_t(H) != uint64_t(B) || n > (uint64_t(1) << 40)) return LF_ERR_INVALID_ARG;
    if (d > 128 || T > kMaxT || n_global > kMaxGlobal || H > kMaxHeads) return LF_ERR_UNSUPPORTED;
    if (uint64_t(B) * H * T > (uint64_t(1) << 31) - 1) return LF_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lock(g_mu);
    DeviceState* ds = nullptr;
    lf_status st = device_state(&ds);
    if (st != LF_OK) return st;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const Layout L = make_layout(B, H, T, d, n_global, LF_F32);  // prep's lists and bitmap
    const size_t off_stats = align256(L.total);
    const size_t total = off_stats + sizeof(float) * 3 * size_t(B) * H * T;
    if ((st = grow(&ds->ws, &ds->ws_bytes, total, s)) != LF_OK) return st;
    uint8_t* base = static_cast<uint8_t*>(ds->ws);
    Workspace ws{};
    ws.n_gq = reinterpret_cast<int32_t*>(base + L.off_ngq);
    ws.n_gk = reinterpret_cast<int32_t*>(base + L.off_ngk);
    ws.gq_list = reinterpret_cast<int32_t*>(base + L.off_gq);
    ws.gk_list = reinterpret_cast<int32_t*>(base + L.off_gk);
    ws.gbit = reinterpret_cast<uint32_t*>(base + L.off_gbit);
    ws.counters = reinterpret_cast<int32_t*>(base + L.off_cnt);
    PrepParams pp{};
    pp.gidx = global_idx;
    pp.pad = key_pad_mask;
    pp.q = q;
    pp.k = k;
    pp.v = v;
    pp.ws = ws;
    pp.status = ds->status;
    pp.B = B; pp.H = H; pp.T = T; pp.d = d;
    pp.n_global = n_global;
    pp.gstride = L.gstride;
    pp.ngp = L.ngp;
    pp.W = L.W;
    pp.pack = 0;
    const size_t prep_smem = size_t(L.W + 2 * kPrepThreads + 2 * L.gstride) * 4;
    prep_kernel<<<B * H, kPrepThreads, prep_smem, s>>>(pp);
    static thread_local BwdParams bp;
    std::memset(&bp, 0, sizeof(bp));
    bp.q = q; bp.k = k; bp.v = v; bp.y = y; bp.dy = dy;
    bp.dq = dq; bp.dk = dk; bp.dv = dv;
    bp.stats = reinterpret_cast<float*>(base + off_stats);
    bp.pad = key_pad_mask;
    bp.ws = ws;
    bp.B = B; bp.H = H; bp.T = T; bp.d = d; bp.r = std::min(r, T);
    bp.gstride = L.gstride;
    bp.W = L.W;
    for (int h = 0; h < kMaxHeads; ++h) bp.dil[h] = (h < H && dil) ? dil[h] : 1;
    bp.sl2 = static_cast<float>(double(scale) * kLog2e);
    bp.scale = scale;
    const unsigned grid = static_cast<unsigned>((uint64_t(B) * H * T + kBwdWarps - 1) / kBwdWarps);
    if (dtype == LF_F32) {
        bwd_stats_kernel<float><<<grid, kBwdWarps * 32, 0, s>>>(bp);
        bwd_dq_kernel<float><<<grid, kBwdWarps * 32, 0, s>>>(bp);
        bwd_dkv_kernel<float><<<grid, kBwdWarps * 32, 0, s>>>(bp);
    } else if (dtype == LF_F16) {
        bwd_stats_kernel<__half><<<grid, kBwdWarps * 32, 0, s>>>(bp);
        bwd_dq_kernel<__half><<<grid, kBwdWarps * 32, 0, s>>>(bp);
        bwd_dkv_kernel<__half><<<grid, kBwdWarps * 32, 0, s>>>(bp);
    } else {
        bwd_stats_kernel<__nv_bfloat16><<<grid, kBwdWarps * 32, 0, s>>>(bp);
        bwd_dq_kernel<__nv_bfloat16><<<grid, kBwdWarps * 32, 0, s>>>(bp);
        bwd_dkv_kernel<__nv_bfloat16><<<grid, kBwdWarps * 32, 0, s>>>(bp);
    }
    return cudaGetLastError() == cudaSuccess ? LF_OK : LF_ERR_CUDA;
}

lf_status lf_attn_rows_partial(const void* q_rows, const void* k, const void* v, int B, int H, int n_rows, int T,
                               int d, const uint8_t* key_pad_mask, float scale, lf_dtype dtype, float* out_ml,
                               float* out_acc, void* stream) {
    if (!q_rows || !k || !v || !out_ml || !out_acc) return LF_ERR_INVALID_ARG;
    if (B <= 0 || H <= 0 || n_rows < 0 || T <= 0 || d <= 0 || !std::isfinite(scale)) return LF_ERR_INVALID_ARG;
    if (dtype != LF_F32 && dtype != LF_BF16 && dtype != LF_F16) return LF_ERR_INVALID_ARG;
    for (const void* p : {q_rows, k, v}) if (reinterpret_cast<uintptr_t>(p) & 15u) return LF_ERR_INVALID_ARG;
    if ((reinterpret_cast<uintptr_t>(out_ml) | reinterpret_cast<uintptr_t>(out_acc)) & 3u) return LF_ERR_INVALID_ARG;
    if (d > 128 || (dtype != LF_F32 && d != 32 && d != 64 && d != 128)) return LF_ERR_UNSUPPORTED;
    if (uint64_t(B) * H > 65535u || T > kMaxT || uint64_t(B) * H * T > (uint64_t(1) << 31)) return LF_ERR_UNSUPPORTED;
    if (n_rows == 0) return LF_OK;
    std::lock_guard<std::mutex> lock(g_mu);
    DeviceState* ds = nullptr;
    lf_status st = device_state(&ds);
    if (st != LF_OK) return st;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const int nchunk = (T + kChunk - 1) / kChunk;
    const size_t off_part = align256(sizeof(int32_t) * size_t(B) * H);
    const size_t total = off_part + sizeof(float) * size_t(B) * H * n_rows * nchunk * (d + 2);
    if ((st = grow(&ds->ws, &ds->ws_bytes, total, s)) != LF_OK) return st;
    uint8_t* base = static_cast<uint8_t*>(ds->ws);
    GlobalRowParams gp{};
    gp.k = k;
    gp.v = v;
    gp.pad = key_pad_mask;
    gp.ws.counters = reinterpret_cast<int32_t*>(base);
    gp.ws.partial = reinterpret_cast<float*>(base + off_part);
    gp.B = B; gp.H = H; gp.T = T; gp.d = d;
    gp.gstride = n_rows;
    gp.nchunk = nchunk;
    gp.sl2 = static_cast<float>(double(scale) * kLog2e);
    gp.q_rows = q_rows;
    gp.out_ml = out_ml;
    gp.out_acc = out_acc;
    gp.n_rows = n_rows;
    if (cudaMemsetAsync(gp.ws.counters, 0, sizeof(int32_t) * size_t(B) * H, s) != cudaSuccess) return LF_ERR_CUDA;
    const dim3 grid(nchunk, B * H);
    const int DP = d <= 32 ? 32 : (d <= 64 ? 64 : 128);
    const size_t smem = size_t(kChunk * DP + DP + kChunk + 32 + kGrThreads) * 4;
    void (*kern)(GlobalRowParams) =
        dtype == LF_F32  ? (DP == 32 ? global_rows_kernel<float, 32, true>
                            : DP == 64 ? global_rows_kernel<float, 64, true> : global_rows_kernel<float, 128, true>)
        : dtype == LF_F16 ? (DP == 32 ? global_rows_kernel<__half, 32, true>
                             : DP == 64 ? global_rows_kernel<__half, 64, true> : global_rows_kernel<__half, 128, true>)
                          : (DP == 32 ? global_rows_kernel<__nv_bfloat16, 32, true>
                             : DP == 64 ? global_rows_kernel<__nv_bfloat16, 64, true>
                                        : global_rows_kernel<__nv_bfloat16, 128, true>);
    kern<<<grid, kGrThreads, smem, s>>>(gp);
    return cudaGetLastError() == cudaSuccess ? LF_OK : LF_ERR_CUDA;
}

lf_status lf_attn_merge_rows(const float* ml, const float* acc, int n_parts, int B, int H, int n_rows, int d,
                             const int32_t* out_pos, void* out, int T_out, lf_dtype dtype, void* stream) {
    if (!ml || !acc || !out_pos || !out) return LF_ERR_INVALID_ARG;
    if (n_parts <= 0 || B <= 0 || H <= 0 || n_rows < 0 || d <= 0 || T_out <= 0) return LF_ERR_INVALID_ARG;
    if (dtype != LF_F32 && dtype != LF_BF16 && dtype != LF_F16) return LF_ERR_INVALID_ARG;
    if (d > 128 || uint64_t(B) * H > 65535u) return LF_ERR_UNSUPPORTED;
    if (n_rows == 0) return LF_OK;
    MergeRowsParams mp;
    mp.ml = ml;
    mp.acc = acc;
    mp.pos = out_pos;
    mp.out = out;
    mp.n_parts = n_parts;
    mp.BH = B * H;
    mp.H = H;
    mp.n_rows = n_rows;
    mp.d = d;
    mp.T_out = T_out;
    const dim3 grid(n_rows, B * H);
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (dtype == LF_F32) merge_rows_kernel<float><<<grid, 128, 0, s>>>(mp);
    else if (dtype == LF_F16) merge_rows_kernel<__half><<<grid, 128, 0, s>>>(mp);
    else merge_rows_kernel<__nv_bfloat16><<<grid, 128, 0, s>>>(mp);
    return cudaGetLastError() == cudaSuccess ? LF_OK : LF_ERR_CUDA;
}

lf_status lf_attn_fwd_stages(const void* q, const void* k, const void* v, void* out, int B, int H, int T, int d,
                             int r, const int32_t* dil, const int32_t* global_idx, int n_global,
                             const uint8_t* key_pad_mask, float scale, lf_dtype dtype, void* stream,
                             uint32_t stage_mask) {
    lf_status st = check_args(q, k, v, out, B, H, T, d, r, dil, global_idx, n_global, scale, dtype);
    if (st != LF_OK) return st;
    if (stage_mask == 0u || stage_mask > 7u) return LF_ERR_INVALID_ARG;
    std::lock_guard<std::mutex> lock(g_mu);
    DeviceState* ds = nullptr;
    if ((st = device_state(&ds)) != LF_OK) return st;
    return launch_all(q, k, v, out, B, H, T, d, r, dil, global_idx, n_global, key_pad_mask, scale, dtype,
                      static_cast<cudaStream_t>(stream), ds, stage_mask);
}

lf_status lf_attn_fwd_host(const void* q, const void* k, const void* v, void* out, int B, int H, int T, int d,
                           int r, const int32_t* dil, const int32_t* global_idx, int n_global,
                           const uint8_t* key_pad_mask, float scale, lf_dtype dtype, void* stream) {
    lf_status st = check_args(q, k, v, out, B, H, T, d, r, dil, global_idx, n_global, scale, dtype);
    if (st != LF_OK) return st;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    std::lock_guard<std::mutex> lock(g_mu);
    DeviceState* ds = nullptr;
    if ((st = device_state(&ds)) != LF_OK) return st;
    const size_t es = dtype == LF_F32 ? 4 : 2;
    const size_t nb = size_t(B) * H * T * d * es;
    const size_t o_q = 0, o_k = align256(nb), o_v = 2 * align256(nb), o_o = 3 * align256(nb);
    const size_t o_g = 4 * align256(nb);
    const size_t o_p = o_g + align256(sizeof(int32_t) * size_t(B) * std::max(n_global, 1));
    const size_t total = o_p + align256(size_t(B) * T);
    if ((st = grow(&ds->io, &ds->io_bytes, total, s)) != LF_OK) return st;
    uint8_t* io = static_cast<uint8_t*>(ds->io);
    // The copies stay ordered after the work already queued on `s`.
    if (cudaEventRecord(ds->ev_fork, s) != cudaSuccess || cudaStreamWaitEvent(ds->cin, ds->ev_fork, 0) != cudaSuccess)
        return LF_ERR_CUDA;
    // Small inputs first (global lists and padding of every sample), on the copy-in stream.
    if (n_global > 0 &&
        cudaMemcpyAsync(io + o_g, global_idx, sizeof(int32_t) * size_t(B) * n_global, cudaMemcpyHostToDevice,
                        ds->cin) != cudaSuccess)
        return LF_ERR_CUDA;
    if (key_pad_mask && cudaMemcpyAsync(io + o_p, key_pad_mask, size_t(B) * T, cudaMemcpyHostToDevice, ds->cin) !=
                            cudaSuccess)
        return LF_ERR_CUDA;
    // Slices of (sample, group of heads), each an independent problem: its q, k, v go in
    // on the copy-in stream, its kernels run on `s` once they have landed, and its
    // output goes back on the copy-out stream, so the copies of one slice overlap the
    // kernels and copies of the others.  The kernels of the slices share the workspace
    // in stream order on `s`.
    const int groups = std::max(1, std::min(H, (DeviceState::kMaxSlices + B - 1) / B));
    const int hg = (H + groups - 1) / groups;
    const int nslices = B * ((H + hg - 1) / hg);
    const bool sliced = nslices > 1 && nslices <= DeviceState::kMaxSlices;
    const int slice_h = sliced ? hg : H;
    const size_t per_head = size_t(T) * d * es;
    int a = 0;
    for (int b = 0; b < (sliced ? B : 1) && st == LF_OK; ++b)
        for (int h0 = 0; h0 < H && st == LF_OK; h0 += slice_h, ++a) {
            const int nh = sliced ? std::min(slice_h, H - h0) : H;
            const int bb = sliced ? 1 : B;
            const size_t off = (size_t(b) * H + h0) * per_head, bytes = size_t(bb) * nh * per_head;
            cudaEvent_t ev_in = ds->ev_in[a], ev_done = ds->ev_done[a];
            if (cudaMemcpyAsync(io + o_q + off, static_cast<const uint8_t*>(q) + off, bytes, cudaMemcpyHostToDevice,
                                ds->cin) != cudaSuccess ||
                cudaMemcpyAsync(io + o_k + off, static_cast<const uint8_t*>(k) + off, bytes, cudaMemcpyHostToDevice,
                                ds->cin) != cudaSuccess ||
                cudaMemcpyAsync(io + o_v + off, static_cast<const uint8_t*>(v) + off, bytes, cudaMemcpyHostToDevice,
                                ds->cin) != cudaSuccess ||
                cudaEventRecord(ev_in, ds->cin) != cudaSuccess || cudaStreamWaitEvent(s, ev_in, 0) != cudaSuccess) {
                st = LF_ERR_CUDA;
                break;
            }
            const int32_t* gdev = n_global > 0 ? reinterpret_cast<const int32_t*>(io + o_g) + size_t(b) * n_global
                                               : nullptr;
            const uint8_t* pdev = key_pad_mask ? io + o_p + size_t(b) * T : nullptr;
            st = launch_all(io + o_q + off, io + o_k + off, io + o_v + off, io + o_o + off, bb, nh, T, d, r,
                            dil ? dil + h0 : nullptr, gdev, n_global, pdev, scale, dtype, s, ds);
            if (st != LF_OK) break;
            if (cudaEventRecord(ev_done, s) != cudaSuccess || cudaStreamWaitEvent(ds->cout, ev_done, 0) != cudaSuccess ||
                cudaMemcpyAsync(static_cast<uint8_t*>(out) + off, io + o_o + off, bytes, cudaMemcpyDeviceToHost,
                                ds->cout) != cudaSuccess)
                st = LF_ERR_CUDA;
        }
    // everything queued so far must finish before the staging area is reused or `out` is read
    const bool synced = cudaStreamSynchronize(ds->cin) == cudaSuccess &&
                        cudaStreamSynchronize(s) == cudaSuccess && cudaStreamSynchronize(ds->cout) == cudaSuccess;
    if (st != LF_OK) return st;
    if (!synced) return LF_ERR_CUDA;
    return LF_OK;
}

lf_status lf_attn_device_status(void* stream, uint32_t* flags) {
    if (flags) *flags = 0;
    if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return LF_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_mu);
    DeviceState* ds = nullptr;
    lf_status st = device_state(&ds);
    if (st != LF_OK) return st;
    uint32_t h = 0;
    if (cudaMemcpy(&h, ds->status, sizeof(h), cudaMemcpyDeviceToHost) != cudaSuccess) return LF_ERR_CUDA;
    if (cudaMemset(ds->status, 0, sizeof(h)) != cudaSuccess) return LF_ERR_CUDA;
    if (flags) *flags = h;
    return h ? LF_ERR_DEVICE_CHECK : LF_OK;
}

const char* lf_attn_strerror(lf_status s) {
    switch (s) {
        case LF_OK: return "ok";
        case LF_ERR_INVALID_ARG: return "invalid argument";
        case LF_ERR_UNSUPPORTED: return "unsupported shape or option";
        case LF_ERR_CUDA: return "CUDA error";
        case LF_ERR_NO_MEMORY: return "workspace allocation failed (or attempted during stream capture)";
        case LF_ERR_DEVICE_CHECK: return "device-side check failed";
        case LF_ERR_SCRATCH_TOO_SMALL:
            return "the workspace these sizes need exceeds the static scratch of lf_attn_fwd_static (32 MiB)";
    }
    return "unknown status";
}

void lf_attn_release(void) {
    std::lock_guard<std::mutex> lock(g_mu);
    int cur = 0;
    cudaGetDevice(&cur);
    for (int dev = 0; dev < kMaxDevices; ++dev) {
        DeviceState& s = g_dev[dev];
        if (!s.init) continue;
        cudaSetDevice(dev);
        if (s.ws) cudaFree(s.ws);
        if (s.io) cudaFree(s.io);
        if (s.status) cudaFree(s.status);
        if (s.ev_fork) cudaEventDestroy(s.ev_fork);
        if (s.ev_join) cudaEventDestroy(s.ev_join);
        if (s.aux) cudaStreamDestroy(s.aux);
        if (s.cin) cudaStreamDestroy(s.cin);
        if (s.cout) cudaStreamDestroy(s.cout);
        for (int a = 0; a < DeviceState::kMaxSlices; ++a) {
            if (s.ev_in[a]) cudaEventDestroy(s.ev_in[a]);
            if (s.ev_done[a]) cudaEventDestroy(s.ev_done[a]);
        }
        s = DeviceState();
    }
    cudaSetDevice(cur);
}

uint64_t lf_attn_workspace_bytes(int B, int H, int T, int d, int n_global, lf_dtype dtype) {
    if (B <= 0 || H <= 0 || T <= 0 || d <= 0 || n_global < 0) return 0;
    return make_layout(B, H, T, d, n_global, dtype).total;
}

int lf_attn_last_launch_count(void) { return t_last_launches; }

void lf_attn_test_hooks(uint32_t flags, uint64_t wait_ns) {
    g_test_stall.store((flags & 1u) ? 1 : 0);
    g_test_wait_ns.store(wait_ns);
}

int lf_attn_band_plan(int B, int H, int T, int r, const int32_t* dil, int n_global, int max_ctas, int32_t* pieces,
                      int capacity) {
    if (B <= 0 || H <= 0 || H > kMaxHeads || T <= 0 || r < 0 || n_global < 0 || max_ctas <= 0) return -1;
    for (int h = 0; h < H; ++h)
        if (dil && (dil[h] < 1 || dil[h] > kMaxDilTma)) return -1;
    static thread_local BandTcParams bp;
    std::memset(&bp, 0, sizeof(bp));
    int kind_of_head[kMaxHeads];
    if (assign_kinds(bp, H, dil, kind_of_head) > kMaxDilKinds) return -1;
    const int r_eff = std::min(r, T);
    const int gstride = std::max(1, std::min(n_global, T));
    const Layout L = make_layout(B, H, T, 64, n_global, LF_BF16);
    if (band_schedule(bp, B, H, T, r_eff, n_global > 0 ? (gstride + kBN - 1) / kBN : 0, kind_of_head,
                      std::min(max_ctas, kMaxBandCtas), L.band_tiles) != LF_OK)
        return -1;
    bp.B = B;
    // the walk each CTA's producer makes (band_tc.cuh), on the host
    int n = 0;
    for (int s = 0; s < bp.grid_ctas; ++s) {
        const int x0 = range_start(bp, s), x1 = range_start(bp, s + 1);
        TileWalker w;
        w.locate(bp, x0);
        for (int x = x0; x < x1;) {
            const int tend = w.start + w.nb(bp);
            const int pend = std::min(tend, x1);
            if (pieces && n < capacity) {
                int32_t* e = pieces + size_t(n) * 10;
                e[0] = s;
                e[1] = w.tile;
                e[2] = static_cast<int32_t>(x - w.start);
                e[3] = static_cast<int32_t>(pend - w.start);
                e[4] = w.nb(bp);
                e[5] = cta_of(bp, w.start);
                e[6] = cta_of(bp, tend - 1);
                e[7] = 2 * s + (w.start > x0 ? 1 : 0);  // partial slot (band_tc.cuh part_slot)
                e[8] = w.b * H + w.h;
                e[9] = w.c * 65536 + w.t;
            }
            ++n;
            x = pend;
            if (x < x1) w.next(bp);
        }
    }
    return n;
}


lf_status lf_attn_fwd_static(const void* q, const void* k, const void* v, void* out, int B, int H, int T, int d,
                             int r, const int32_t* dil, const int32_t* global_idx, int n_global,
                             const uint8_t* key_pad_mask, float scale, lf_dtype dtype, void* stream) {
    lf_status st = check_args(q, k, v, out, B, H, T, d, r, dil, global_idx, n_global, scale, dtype);
    if (st != LF_OK) return st;
    const size_t cap = kStaticScratchBytes - 256;
    if (make_layout(B, H, T, d, n_global, dtype).total > cap) return LF_ERR_SCRATCH_TOO_SMALL;
    std::lock_guard<std::mutex> lock(g_mu);
    StaticState* ss = nullptr;
    if ((st = static_state(&ss)) != LF_OK) return st;
    // The workspace already has the capacity the layout needs, so launch_all
    // never grows (allocates) it.  Prep zeroes what must start at zero.
    DeviceState view;
    view.init = true;
    view.sm_count = ss->sm_count;
    view.status = reinterpret_cast<uint32_t*>(ss->scratch);
    view.ws = ss->scratch + 256;
    view.ws_bytes = cap;
    return launch_all(q, k, v, out, B, H, T, d, r, dil, global_idx, n_global, key_pad_mask, scale, dtype,
                      static_cast<cudaStream_t>(stream), &view);
}



}  // extern "C"
