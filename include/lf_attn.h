/*
 * lf_attn.h -- C ABI of liblfattn: Longformer sparse self-attention, forward,
 * on NVIDIA B200 (sm_100a).
 *
 * Operation (the "Longformer" note, eightmm.github.io/papers/architectures/
 * longformer, sections "Sliding-Window Attention", "Global Attention" and
 * "Mask View"; dilation as in the Longformer wiki, ciallo.wiki, section
 * 2.2.3):
 *
 *   y[b,h,i] = sum_{j in N(i)} softmax_j( scale * q[b,h,i] . k[b,h,j] ) v[b,h,j]
 *
 *   N(i) = ( {i + dil[h]*t : |t| <= r} clipped to [0,T)  U  G_b ) \ padded keys
 *          for i not in G_b;
 *   N(i) = all non-padded keys, for i in G_b.
 *
 * G_b is the set of in-range entries of global_idx[b, :] (duplicates
 * collapse; a global key inside the window is counted once).  A padded
 * position is never a key; if it is also global it is still a global query.
 * Rows whose key set is empty produce 0.  Every output row is written,
 * padded query rows included.
 *
 * Conventions for every entry point:
 *   - Tensors q, k, v, out are contiguous [B, H, T, d], row-major (d
 *     innermost), all of the dtype given by `dtype`; they must be 16-byte
 *     aligned.
 *   - "device" pointers are CUDA device (or managed) memory of the current
 *     device; "host" pointers are ordinary CPU memory.
 *   - The caller owns every pointer; the library keeps none after return.
 *     It owns one workspace per device (grown on demand with cudaMalloc,
 *     freed by lf_attn_release).  Calls that use the same device share that
 *     workspace, so calls on different streams of one device must not
 *     overlap in time.  The first call that needs a larger workspace must
 *     not be made while `stream` is being captured into a CUDA graph.
 *   - Errors in arguments are reported before anything is launched.  No
 *     entry point traps or aborts.
 */
#ifndef LF_ATTN_H
#define LF_ATTN_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum { LF_F32 = 0, LF_BF16 = 1, LF_F16 = 2 } lf_dtype;

typedef enum {
    LF_OK = 0,
    LF_ERR_INVALID_ARG = 1,  /* null pointer, bad size, misalignment, bad dil/r/n_global */
    LF_ERR_UNSUPPORTED = 2,  /* valid but outside what this build implements (see lf_attn_fwd) */
    LF_ERR_CUDA = 3,         /* a CUDA runtime call or a launch failed */
    LF_ERR_NO_MEMORY = 4,    /* workspace could not be allocated (or not during capture) */
    LF_ERR_DEVICE_CHECK = 5, /* a device-side check fired (see lf_attn_device_status) */
    LF_ERR_SCRATCH_TOO_SMALL = 6 /* lf_attn_fwd_static: sizes need more than its fixed scratch */
} lf_status;

/*
 * lf_attn_fwd -- the forward pass, asynchronous on `stream`.
 *
 *   q, k, v     device, [B,H,T,d], dtype `dtype`
 *   out         device, [B,H,T,d], dtype `dtype`; fully overwritten
 *   B, H, T, d  sizes (all >= 1)
 *   r           one-sided window radius, w = 2r + 1, r >= 0
 *   dil         HOST int32 [H], per-head dilation, each >= 1; NULL = all 1
 *   global_idx  DEVICE int32 [B, n_global]: global positions per sample, any
 *               order, duplicates allowed; NULL iff n_global == 0.  Entries
 *               outside [0, T) are ignored and flagged in the device status.
 *   n_global    >= 0
 *   key_pad_mask DEVICE uint8 [B, T], nonzero = padded key; NULL = none
 *   scale       softmax scale (usually 1/sqrt(d))
 *   dtype       LF_F32: CUDA-core fp32 path, d <= 128.
 *               LF_BF16: tensor-core path (tcgen05 + TMA), d == 64 or 128,
 *               fp32 accumulation and softmax, every dil[h] <= 8, at most 4
 *               distinct dilation values, H <= 128.  (d == 128 runs one band
 *               CTA per SM, and its global rows on the CUDA cores.)
 *               LF_F16: the same tensor-core path with fp16 q, k, v and out
 *               (fp16 MMA operands, the probabilities rounded to fp16 for the
 *               P V product), with the same limits.  The pages train with
 *               fp16 mixed precision (Longformer wiki, section 6.3).
 *   stream      a cudaStream_t (NULL = legacy default stream)
 *
 * Returns LF_OK once the kernels are queued; nothing is synchronised.
 * On the bf16 path with global tokens, the global-row kernels are queued on
 * a library-owned low-priority stream that waits for the earlier work of
 * `stream` and that `stream` waits for in turn, so the call stays ordered
 * on `stream` (also under stream capture).  Calls on different streams
 * share that side stream, so their global-row kernels run in call order.
 */
lf_status lf_attn_fwd(const void* q, const void* k, const void* v, void* out,
                      int B, int H, int T, int d, int r, const int32_t* dil,
                      const int32_t* global_idx, int n_global,
                      const uint8_t* key_pad_mask, float scale, lf_dtype dtype,
                      void* stream);

/*
 * lf_attn_fwd_host -- the same forward on HOST buffers.
 *
 * q, k, v, out, global_idx and key_pad_mask are host pointers with the
 * layouts above (page-locked memory gives full copy bandwidth).  The call
 * copies the inputs into a library-owned device staging area, runs the
 * forward and copies `out` back, ordered after the work already queued on
 * `stream`, and returns when `out` is ready.  It works on up to 4 slices
 * of (sample, group of heads): the inputs of a slice are copied on a
 * library-owned copy-in stream, its kernels run on `stream`, and its output
 * is copied back on a copy-out stream, so the copies of one slice overlap
 * the kernels and copies of the others.
 */
lf_status lf_attn_fwd_host(const void* q, const void* k, const void* v, void* out,
                           int B, int H, int T, int d, int r, const int32_t* dil,
                           const int32_t* global_idx, int n_global,
                           const uint8_t* key_pad_mask, float scale, lf_dtype dtype,
                           void* stream);

/*
 * lf_attn_fwd_rand -- the BigBird variant: window + global tokens + random
 * key blocks (the mhpn.cn page, sections 2.2.1 and 2.2.2: random attention
 * beside the window and the global tokens, in blocks of 64; the aiqz.cc
 * page's BigBird comparison).  Arguments as lf_attn_fwd, plus
 *
 *   rand_blocks DEVICE int32 [B, H, ceil(T / 64), n_rand]: the key blocks
 *               drawn for each 64-row query block (key block c = keys
 *               [64 c, 64 c + 64) clipped to T).  The caller draws them (for
 *               instance from a seeded generator); entries outside
 *               [0, ceil(T / 64)) are ignored.  NULL iff n_rand == 0.
 *   n_rand      0..4 draws per query block.
 *
 *   An ordinary row i keeps K(i) of lf_attn_fwd together with the keys of
 *   the blocks drawn for its query block i / 64, as a set (duplicate draws,
 *   and keys already in the window or global, count once), padded keys
 *   removed.  Global rows are unchanged.  n_rand == 0 is lf_attn_fwd.
 *   With n_rand > 0: LF_BF16 or LF_F16, d == 64, every dil[h] == 1 (else
 *   LF_ERR_UNSUPPORTED).
 */
lf_status lf_attn_fwd_rand(const void* q, const void* k, const void* v, void* out,
                           int B, int H, int T, int d, int r, const int32_t* dil,
                           const int32_t* global_idx, int n_global,
                           const uint8_t* key_pad_mask, float scale, lf_dtype dtype,
                           const int32_t* rand_blocks, int n_rand, void* stream);

/*
 * lf_attn_bwd -- the backward pass: gradients of the forward's output with
 * respect to q, k and v (the pages train and fine-tune with this attention:
 * Longformer wiki, sections 3.1 and 3.2; aiqz.cc page, gradient
 * checkpointing), asynchronous on `stream`.  With the forward's key sets
 * K(i), p_ij = softmax over K(i) of scale q_i . k_j, D_i = dy_i . y_i:
 *   dv_j = sum_{i: j in K(i)} p_ij dy_i,  ds_ij = p_ij (dy_i . v_j - D_i),
 *   dq_i = scale sum_{j in K(i)} ds_ij k_j,  dk_j = scale sum_{i: j in K(i)} ds_ij q_i.
 *
 *   q, k, v, y, dy  DEVICE [B,H,T,d], dtype `dtype` (y: lf_attn_fwd's output
 *                   for these inputs; dy: the gradient of the loss w.r.t. y)
 *   dq, dk, dv      DEVICE fp32 [B,H,T,d], fully overwritten
 *   other arguments as lf_attn_fwd; any dtype with d <= 128 (CUDA cores).
 *   Pointers 16-byte aligned.  Uses the device workspace of lf_attn_fwd.
 */
lf_status lf_attn_bwd(const void* q, const void* k, const void* v, const void* y, const void* dy,
                      float* dq, float* dk, float* dv, int B, int H, int T, int d, int r,
                      const int32_t* dil, const int32_t* global_idx, int n_global,
                      const uint8_t* key_pad_mask, float scale, lf_dtype dtype, void* stream);

/*
 * Sequence-sharded forward (several GPUs, each holding a contiguous range
 * of the sequence; the orchestration, with its halo and global-row
 * exchanges, is sharded.py in the Python package).  A global row attends
 * every key ("Longformer" note, section "Global Attention"), so its softmax
 * is split over the key shards and merged: each shard contributes the
 * partial state (M, L, acc) of the row over its own keys, and
 * y = sum_p 2^(M_p - M) acc_p / sum_p 2^(M_p - M) L_p with M = max_p M_p.
 *
 * lf_attn_rows_partial -- partial states of n_rows query rows over every
 * non-padded key of [B, H, T, d] k and v, asynchronous on `stream`.
 *   q_rows   DEVICE [B, H, n_rows, d], dtype `dtype` (16-byte aligned)
 *   k, v     DEVICE [B, H, T, d] (16-byte aligned); key_pad_mask DEVICE
 *            uint8 [B, T] or NULL
 *   out_ml   DEVICE fp32 [B, H, n_rows, 2]: M (the largest scale * log2(e) *
 *            q . k over the kept keys; -inf when none) and L = sum 2^(s - M)
 *   out_acc  DEVICE fp32 [B, H, n_rows, d]: sum 2^(s - M) v
 *   d <= 128; for LF_BF16 / LF_F16, d is 32, 64 or 128.  Uses the device
 *   workspace of lf_attn_fwd (same rules).
 *
 * lf_attn_merge_rows -- merges n_parts partial states per row and writes
 * the rows: ml [n_parts][B][H][n_rows][2], acc [n_parts][B][H][n_rows][d]
 * (DEVICE fp32); row a of sample b goes to out row out_pos[b * n_rows + a]
 * of the DEVICE [B, H, T_out, d] tensor `out` (dtype `dtype`), or nowhere
 * when that entry is negative.  d <= 128.
 */
lf_status lf_attn_rows_partial(const void* q_rows, const void* k, const void* v, int B, int H, int n_rows,
                               int T, int d, const uint8_t* key_pad_mask, float scale, lf_dtype dtype,
                               float* out_ml, float* out_acc, void* stream);
lf_status lf_attn_merge_rows(const float* ml, const float* acc, int n_parts, int B, int H, int n_rows, int d,
                             const int32_t* out_pos, void* out, int T_out, lf_dtype dtype, void* stream);

/*
 * lf_attn_fwd_stages -- runs a subset of the kernels lf_attn_fwd queues, for
 * timing one kernel at a time.  Same arguments as lf_attn_fwd, plus
 * stage_mask: bit 0 = prep (global lists, padding, packed global keys),
 * bit 1 = band rows, bit 2 = global rows.  The band and global-row stages
 * read what the prep stage of an earlier call with the same sizes,
 * global_idx, key_pad_mask and k/v values left in the workspace; results
 * are only defined when that holds.  stage_mask == 7 is lf_attn_fwd.
 */
lf_status lf_attn_fwd_stages(const void* q, const void* k, const void* v, void* out,
                             int B, int H, int T, int d, int r, const int32_t* dil,
                             const int32_t* global_idx, int n_global,
                             const uint8_t* key_pad_mask, float scale, lf_dtype dtype,
                             void* stream, uint32_t stage_mask);

/*
 * lf_attn_device_status -- synchronises `stream`, then reads and clears the
 * current device's status word.  Returns LF_ERR_DEVICE_CHECK if a kernel
 * since the last read flagged a data error (a global_idx entry outside
 * [0, T)) or gave up waiting on one of its own pipeline barriers; `flags`
 * (may be NULL) receives the raw bits:
 *   bit 0  global_idx entry out of range (ignored by the computation)
 *   bit 1  a pipeline wait timed out; that call's output is incomplete
 */
lf_status lf_attn_device_status(void* stream, uint32_t* flags);

/* Text for a status code (static storage). */
const char* lf_attn_strerror(lf_status status);

/* Frees the workspaces of every device this process used. */
void lf_attn_release(void);

/* Bytes of device workspace lf_attn_fwd needs for these sizes. */
uint64_t lf_attn_workspace_bytes(int B, int H, int T, int d, int n_global, lf_dtype dtype);

/* Kernels launched by the last successful lf_attn_fwd on this host thread. */
int lf_attn_last_launch_count(void);

/*
 * lf_attn_test_hooks -- test hook for the device-side failure path (no
 * counterpart in the pages).  wait_ns sets the limit of every pipeline wait
 * of the bf16 band kernel in later calls (0 restores the default, 1 s);
 * flags bit 0 makes the band kernel's producers stop before their first
 * load, so the other roles' waits run out, the kernel ends early with
 * status bit 1 set (lf_attn_device_status reports LF_ERR_DEVICE_CHECK) and
 * that call's output is not written.  Nothing faults or hangs; a later call
 * with lf_attn_test_hooks(0, 0) computes normally.  Process-wide setting.
 */
void lf_attn_test_hooks(uint32_t flags, uint64_t wait_ns);

/*
 * lf_attn_band_plan -- diagnostic: how the bf16 band kernel splits its work
 * for these sizes over at most max_ctas CTAs, computed on the host by the
 * same code the kernel's producer runs (no device is touched).  The tiles'
 * key blocks form one sequence (per sample, heads; per head, residue
 * classes of the dilation; per class, 128-query tiles; per tile, its band
 * blocks then its global-key blocks), and CTA s takes an equal contiguous
 * share of it, cutting tiles into pieces where needed.
 *   pieces: host array of capacity x 10 int32 (may be NULL); piece k gets
 *     {cta, tile, first block, end block, blocks of the tile, first CTA of
 *      the tile, last CTA of the tile, partial-state slot, b*H + h,
 *      class * 65536 + tile within the class}.
 * Returns the number of pieces (which may exceed capacity), or -1 for
 * invalid or unsupported sizes.
 */
int lf_attn_band_plan(int B, int H, int T, int r, const int32_t* dil, int n_global, int max_ctas,
                      int32_t* pieces, int capacity);

/*
 * lf_attn_fwd_static -- lf_attn_fwd for callers that cannot allocate device
 * memory (the pages describe no counterpart; this is a deployment variant).
 *
 * Some callers cannot call cudaMalloc: code running while a CUDA graph is
 * captured in global mode, processes confined to a fixed memory budget or
 * to their own pool allocator, runtimes that reserve all device memory at
 * start-up.  This entry point allocates nothing, neither itself nor through
 * any library: its workspace is a fixed scratch array compiled into this
 * library (one per GPU that loads the library, 32 MiB minus a 256-byte
 * status word, held until the process exits).
 *
 *   Arguments, layouts, ownership and the result are those of lf_attn_fwd;
 *   the caller still provides q, k, v, out, global_idx and key_pad_mask.
 *   Returns LF_ERR_SCRATCH_TOO_SMALL, before launching anything, when these
 *   sizes need more than 32 MiB - 256 bytes of workspace (the
 *   lf_attn_workspace_bytes figure).  bf16 sizes need about 19 MiB for
 *   the band kernel's fixed partial-state slots (two per CTA, 296 CTAs)
 *   plus what grows with B, H, T and n_global: 19 to 26 MiB for the sizes
 *   the tests use (up to B = 2, H = 16, T = 16384, 64 global tokens).
 *   The first call on a device sets that device up (kernel attributes and
 *   the scratch array's device address); make that first call before any
 *   stream capture.
 *   Every call on a device shares the one scratch array, which keeps the
 *   last call's contents (the prep kernel clears what must start at zero).
 *   Calls whose kernels overlap on the GPU -- on different streams, or
 *   concurrently with another host thread -- race on that array.
 *   Device-side flags of this variant (out-of-range global_idx entries,
 *   which are ignored as in lf_attn_fwd; a pipeline wait that gave up) stay
 *   in its scratch area and are not reported: check global_idx on the host.
 */
lf_status lf_attn_fwd_static(const void* q, const void* k, const void* v, void* out,
                             int B, int H, int T, int d, int r, const int32_t* dil,
                             const int32_t* global_idx, int n_global,
                             const uint8_t* key_pad_mask, float scale, lf_dtype dtype,
                             void* stream);

#ifdef __cplusplus
}
#endif

#endif /* LF_ATTN_H */
