/*
 * lf_oracle.c -- CPU oracle for Longformer sparse self-attention (forward).
 *
 * TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the
 * benchmark's CPU-baseline leg may load this file's library.  The CUDA
 * library never calls it and shares no code with it.
 *
 * What it computes, with the passage each step follows:
 *
 *   For every sample b, head h and query row i in [0, T):
 *     * Ordinary row (i not in G):
 *         K(i) = ( { i + dil_h * t : -r <= t <= r, 0 <= i + dil_h*t < T }  U  G_b )
 *                minus the padded keys.
 *       - window N_local(i) = { j : |i - j| <= r }, w = 2r + 1:
 *         "Longformer" note (eightmm.github.io), section "Sliding-Window
 *         Attention", the N_local and w equations;
 *       - dilation samples every dil-th position inside the window, so the
 *         reach grows to dil*r at the same key count: "Longformer" wiki
 *         (ciallo.wiki) section 2.2.3, and the aiqz.cc engineering page,
 *         section on dilated windows (distances d, 2d, 3d ...);
 *       - out-of-range positions are dropped (aiqz.cc page, Python demo,
 *         step 3 of its walk-through);
 *       - N(i) = N_local(i) U G for i not in G: "Longformer" note, section
 *         "Global Attention"; a set, so a global key inside the window is
 *         counted once.
 *     * Global row (i in G):  K(i) = all non-padded keys
 *       ("Longformer" note, section "Global Attention": N(i) = {1..T}).
 *     * Padding: padded keys are masked everywhere ("Longformer" note,
 *       section "Implementation Reading": padding must be masked).
 *     * s_j = scale * q_i . k_j   (fp64),  y_i = sum_j softmax_j(s) v_j
 *       ("Longformer" note, the y_i equation and the "Mask View" section).
 *     * K(i) empty -> y_i = 0 (the pages are silent; this is the reading
 *       taken).
 *     * Random blocks (the BigBird variant, lf_oracle_fwd_rand): an
 *       ordinary row also keeps the keys of the random key blocks drawn for
 *       its query block, K(i) U R(i), before padding is removed.  BigBird
 *       adds random attention to the window and the global tokens, each
 *       token attending a few randomly chosen others (mhpn.cn page, section
 *       2.2.1), in blocks of block_size = 64 (same page, section 2.2.2; the
 *       aiqz.cc page's BigBird comparison: neighbours + front desk + random
 *       picks).  Reading taken: query block i / 64 draws n_rand key blocks
 *       (passed in, since the draws are random); key block c holds keys
 *       [64 c, 64 c + 64) clipped to T; blocks outside [0, ceil(T / 64))
 *       are ignored; a set again, so duplicates and keys already in K(i)
 *       count once.  Global rows are unchanged.
 *
 * Readings of points the pages leave open: 0-based indices; r is the
 * one-sided radius; the dilated window is {i + dil*t : |t| <= r} (the
 * aiqz.cc demo code that adds every dil-th key out to both sequence ends
 * contradicts that page's own prose and the other pages, and is not
 * followed); the same q/k/v serve local and global attention; global
 * entries outside [0, T) are ignored; duplicates collapse; a padded global
 * position still acts as a global *query* but is removed as a key.
 *
 * Inputs are fp32 arrays (fp32 workloads, or bf16 values, which fp32
 * represents exactly); every operation after loading is done in double.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#ifdef _OPENMP
#include <omp.h>
#endif

#define OR_OK 0
#define OR_RAND_BLOCK 64  /* BigBird block_size */
#define OR_BAD_ARG 1
#define OR_NO_MEM 4

/* Is position i one of the (in-range) global positions of this sample? */
static int is_global(int i, int T, const int32_t* G, int nG)
{
    for (int a = 0; a < nG; a++)
        if (G[a] >= 0 && G[a] < T && G[a] == i) return 1;
    return 0;
}

/*
 * Key set K(i) of one row, in ascending order, written to keys[]; returns
 * its size.  `marker` is caller scratch of T bytes.
 */
static int key_set(int T, int r, int dil, int i, const int32_t* G, int nG,
                   const uint8_t* pad_b, const int32_t* rnd, int n_rand, uint8_t* marker, int* keys)
{
    memset(marker, 0, (size_t)T);
    if (is_global(i, T, G, nG)) {
        for (int j = 0; j < T; j++) marker[j] = 1;
    } else {
        for (long t = -(long)r; t <= (long)r; t++) {
            long j = (long)i + (long)dil * t;
            if (j >= 0 && j < T) marker[j] = 1;
        }
        for (int a = 0; a < nG; a++)
            if (G[a] >= 0 && G[a] < T) marker[G[a]] = 1;
        if (rnd) {  /* rnd: [ceil(T / 64)][n_rand] key blocks of each query block of this (b, h) */
            const int32_t* ri = rnd + (size_t)(i / OR_RAND_BLOCK) * n_rand;
            for (int a = 0; a < n_rand; a++) {
                long j0 = (long)ri[a] * OR_RAND_BLOCK;
                if (ri[a] < 0 || j0 >= T) continue;
                for (long j = j0; j < j0 + OR_RAND_BLOCK && j < T; j++) marker[j] = 1;
            }
        }
    }
    if (pad_b)
        for (int j = 0; j < T; j++)
            if (pad_b[j]) marker[j] = 0;
    int n = 0;
    for (int j = 0; j < T; j++)
        if (marker[j]) keys[n++] = j;
    return n;
}

/* One output row: y_i over K(i).  probs (optional, T doubles) receives the
 * softmax weights p_j / l at the key positions and 0 elsewhere. */
static void one_row(const float* q, const float* k, const float* v, double* y,
                    int T, int d, int r, int dil, int i, const int32_t* G, int nG,
                    const uint8_t* pad_b, const int32_t* rnd, int n_rand, double scale,
                    uint8_t* marker, int* keys, double* s, double* probs)
{
    int n = key_set(T, r, dil, i, G, nG, pad_b, rnd, n_rand, marker, keys);
    if (probs)
        for (int j = 0; j < T; j++) probs[j] = 0.0;
    if (n == 0) {
        for (int c = 0; c < d; c++) y[c] = 0.0;
        return;
    }
    const float* qi = q + (size_t)i * d;
    double m = -INFINITY;
    for (int a = 0; a < n; a++) {
        const float* kj = k + (size_t)keys[a] * d;
        double dot = 0.0;
        for (int c = 0; c < d; c++) dot += (double)qi[c] * (double)kj[c];
        s[a] = scale * dot;
        if (s[a] > m) m = s[a];
    }
    double l = 0.0;
    for (int a = 0; a < n; a++) {
        s[a] = exp(s[a] - m);           /* s now holds p_j */
        l += s[a];
    }
    for (int c = 0; c < d; c++) {
        double acc = 0.0;
        for (int a = 0; a < n; a++) acc += s[a] * (double)v[(size_t)keys[a] * d + c];
        y[c] = acc / l;
    }
    if (probs)
        for (int a = 0; a < n; a++) probs[keys[a]] = s[a] / l;
}

static int check_args(int B, int H, int T, int d, int r, const int32_t* dil, int nG)
{
    if (B <= 0 || H <= 0 || T <= 0 || d <= 0 || r < 0 || nG < 0) return OR_BAD_ARG;
    for (int h = 0; h < H; h++)
        if (!dil || dil[h] < 1) return OR_BAD_ARG;
    return OR_OK;
}

/*
 * Sampled rows.  rows[3*n + 0..2] = (b, h, i); out_rows[n*d + c] receives
 * y.  q, k, v: fp32 [B, H, T, d].  global_idx: [B, n_global] (may be NULL
 * when n_global == 0).  key_pad: uint8 [B, T] or NULL.  nthreads <= 0 uses
 * the OpenMP default.
 */
int lf_oracle_rows_rand(const float* q, const float* k, const float* v,
                        int B, int H, int T, int d, int r, const int32_t* dil,
                        const int32_t* global_idx, int n_global, const uint8_t* key_pad,
                        double scale, const int32_t* rows, long n_rows, double* out_rows,
                        int nthreads, const int32_t* rand_blocks, int n_rand)
{
    int st = check_args(B, H, T, d, r, dil, n_global);
    if (st) return st;
    if (n_rand < 0 || (n_rand > 0 && !rand_blocks)) return OR_BAD_ARG;
    const long nqb = (T + OR_RAND_BLOCK - 1) / OR_RAND_BLOCK;
    for (long n = 0; n < n_rows; n++) {
        int b = rows[3 * n], h = rows[3 * n + 1], i = rows[3 * n + 2];
        if (b < 0 || b >= B || h < 0 || h >= H || i < 0 || i >= T) return OR_BAD_ARG;
    }
    int err = 0;
#ifdef _OPENMP
    if (nthreads > 0) omp_set_num_threads(nthreads);
#else
    (void)nthreads;
#endif
#pragma omp parallel
    {
        uint8_t* marker = (uint8_t*)malloc((size_t)T);
        int* keys = (int*)malloc(sizeof(int) * (size_t)T);
        double* s = (double*)malloc(sizeof(double) * (size_t)T);
        if (!marker || !keys || !s) {
#pragma omp atomic write
            err = 1;
        } else {
#pragma omp for schedule(dynamic, 16)
            for (long n = 0; n < n_rows; n++) {
                int b = rows[3 * n], h = rows[3 * n + 1], i = rows[3 * n + 2];
                size_t bh = (size_t)b * H + h;
                const int32_t* G = n_global > 0 ? global_idx + (size_t)b * n_global : NULL;
                const uint8_t* pad_b = key_pad ? key_pad + (size_t)b * T : NULL;
                const int32_t* rnd = n_rand > 0 ? rand_blocks + bh * (size_t)nqb * n_rand : NULL;
                one_row(q + bh * T * d, k + bh * T * d, v + bh * T * d, out_rows + (size_t)n * d,
                        T, d, r, dil[h], i, G, n_global, pad_b, rnd, n_rand, scale, marker, keys, s, NULL);
            }
        }
        free(marker);
        free(keys);
        free(s);
    }
    return err ? OR_NO_MEM : OR_OK;
}

int lf_oracle_rows(const float* q, const float* k, const float* v,
                   int B, int H, int T, int d, int r, const int32_t* dil,
                   const int32_t* global_idx, int n_global, const uint8_t* key_pad,
                   double scale, const int32_t* rows, long n_rows, double* out_rows,
                   int nthreads)
{
    return lf_oracle_rows_rand(q, k, v, B, H, T, d, r, dil, global_idx, n_global, key_pad, scale,
                               rows, n_rows, out_rows, nthreads, NULL, 0);
}

/* Every row: out is double [B, H, T, d].  rand_blocks: int32
 * [B, H, ceil(T / 64), n_rand] (NULL when n_rand == 0). */
int lf_oracle_fwd_rand(const float* q, const float* k, const float* v, double* out,
                       int B, int H, int T, int d, int r, const int32_t* dil,
                       const int32_t* global_idx, int n_global, const uint8_t* key_pad,
                       double scale, int nthreads, const int32_t* rand_blocks, int n_rand)
{
    int st = check_args(B, H, T, d, r, dil, n_global);
    if (st) return st;
    long n_rows = (long)B * H * T;
    int32_t* rows = (int32_t*)malloc(sizeof(int32_t) * 3 * (size_t)n_rows);
    if (!rows) return OR_NO_MEM;
    long n = 0;
    for (int b = 0; b < B; b++)
        for (int h = 0; h < H; h++)
            for (int i = 0; i < T; i++) {
                rows[3 * n] = b;
                rows[3 * n + 1] = h;
                rows[3 * n + 2] = i;
                n++;
            }
    st = lf_oracle_rows_rand(q, k, v, B, H, T, d, r, dil, global_idx, n_global, key_pad, scale,
                             rows, n_rows, out, nthreads, rand_blocks, n_rand);
    free(rows);
    return st;
}

int lf_oracle_fwd(const float* q, const float* k, const float* v, double* out,
                  int B, int H, int T, int d, int r, const int32_t* dil,
                  const int32_t* global_idx, int n_global, const uint8_t* key_pad,
                  double scale, int nthreads)
{
    return lf_oracle_fwd_rand(q, k, v, out, B, H, T, d, r, dil, global_idx, n_global, key_pad, scale,
                              nthreads, NULL, 0);
}

/* K(i) of one row of sample b (head dilation `dil`): writes the sorted keys,
 * returns |K(i)| (or -1 on bad arguments). */
int lf_oracle_key_set(int T, int r, int dil, int i, const int32_t* G, int nG,
                      const uint8_t* pad_b, int32_t* keys_out)
{
    if (T <= 0 || r < 0 || dil < 1 || i < 0 || i >= T || nG < 0) return -1;
    uint8_t* marker = (uint8_t*)malloc((size_t)T);
    int* keys = (int*)malloc(sizeof(int) * (size_t)T);
    if (!marker || !keys) {
        free(marker);
        free(keys);
        return -1;
    }
    int n = key_set(T, r, dil, i, G, nG, pad_b, NULL, 0, marker, keys);
    if (keys_out)
        for (int a = 0; a < n; a++) keys_out[a] = keys[a];
    free(marker);
    free(keys);
    return n;
}

/* Sum over rows of |K(i)| for one sample and one head dilation. */
long lf_oracle_key_total(int T, int r, int dil, const int32_t* G, int nG, const uint8_t* pad_b)
{
    if (T <= 0 || r < 0 || dil < 1 || nG < 0) return -1;
    uint8_t* marker = (uint8_t*)malloc((size_t)T);
    int* keys = (int*)malloc(sizeof(int) * (size_t)T);
    if (!marker || !keys) {
        free(marker);
        free(keys);
        return -1;
    }
    long total = 0;
    for (int i = 0; i < T; i++) total += key_set(T, r, dil, i, G, nG, pad_b, NULL, 0, marker, keys);
    free(marker);
    free(keys);
    return total;
}

/* Softmax weights of one row (b, h, i): probs is double [T], p_j/l at the
 * keys of K(i) and 0 elsewhere; y (double [d]) receives the output. */
int lf_oracle_row_probs(const float* q, const float* k, const float* v,
                        int B, int H, int T, int d, int r, const int32_t* dil,
                        const int32_t* global_idx, int n_global, const uint8_t* key_pad,
                        double scale, int b, int h, int i, double* probs, double* y)
{
    int st = check_args(B, H, T, d, r, dil, n_global);
    if (st) return st;
    if (b < 0 || b >= B || h < 0 || h >= H || i < 0 || i >= T || !probs || !y) return OR_BAD_ARG;
    uint8_t* marker = (uint8_t*)malloc((size_t)T);
    int* keys = (int*)malloc(sizeof(int) * (size_t)T);
    double* s = (double*)malloc(sizeof(double) * (size_t)T);
    if (!marker || !keys || !s) {
        free(marker);
        free(keys);
        free(s);
        return OR_NO_MEM;
    }
    size_t bh = (size_t)b * H + h;
    const int32_t* G = n_global > 0 ? global_idx + (size_t)b * n_global : NULL;
    const uint8_t* pad_b = key_pad ? key_pad + (size_t)b * T : NULL;
    one_row(q + bh * T * d, k + bh * T * d, v + bh * T * d, y, T, d, r, dil[h], i, G, n_global,
            pad_b, NULL, 0, scale, marker, keys, s, probs);
    free(marker);
    free(keys);
    free(s);
    return OR_OK;
}

int lf_oracle_max_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
