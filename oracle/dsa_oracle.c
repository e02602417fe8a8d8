/*
 * dsa_oracle.c -- plain, slow fp64 CPU oracle for DeepSeek Sparse Attention.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path may link, load or
 * call this file; only the tests, __graft_entry__.smoke() and the benchmark's
 * CPU-baseline leg do.  It shares no code, header, table or constant with the
 * CUDA library.
 *
 * What it computes, stage by stage (the plain definition, no blocking, no
 * fusion, no reordering):
 *
 *  1. Lightning indexer ("DeepSeek-V3.2-Exp DSA 技术深度解析", section 1: a
 *     light indexer with few heads, low-dimensional FP8 query/key and ReLU
 *     scores every history token of a query):
 *        I[t,s] = sum_h w[t,h] * max(0, sum_j qhat[t,h,j] * khat[s,j]),  0 <= s <= t
 *     with qhat = e4m3(q8) * sq[t], khat = e4m3(k8) * sk[s] (per-token fp32
 *     scales; fp32 inputs are used as they are).
 *  2. Top-k selector (same section; the "fine-grained selector" of the hotdry
 *     page): the min(k, t+1) positions s <= t with the largest I[t,s], ties
 *     to the lower s, emitted in ascending s and padded with -1.
 *  3. Main attention over the selected set only (same section; O(L^2) ->
 *     O(L k)):  z_j = sm * q[t,h] . K[j],  p = softmax(z),  o = sum_j p_j V[j],
 *     lse = max z + log sum exp(z - max z), natural log.
 *  4. Decode: stages 1-3 for one query per sequence whose context (already
 *     holding the current token) lives in paged caches.
 *  5. Sliding window with top-k ("DeepSeek-V4 百万 token 上下文的工程实现",
 *     section on the sliding-window KV cache and the hybrid strategy: the most
 *     recent 4K-16K tokens keep their full KV, older tokens are kept only as
 *     far as an importance score retains them): the W most recent positions
 *     of a query are always attended, and stage 2 selects min(k, t+1-W) of
 *     the older positions 0..t-W by indexer score.  Output: the top-k part in
 *     ascending position, then the window positions, then -1 up to k + W.
 *  7. FP8 K/V for the main attention (the hotdry page's FP8 decoding
 *     section: the KV cache moves from 16-bit to FP8): the decode caches hold
 *     E4M3 codes with one fp32 scale per cached token for K and for V, and the
 *     attention of stage 3 uses Khat[j] = e4m3(k8[j]) * ks[j],
 *     Vhat[j] = e4m3(v8[j]) * vs[j].
 *  6. FP8 quantisation of the indexer's query and key ("DeepSeek-V3.2-Exp
 *     DSA 技术深度解析", section 1: FP8 indexer; the hotdry page's section on
 *     FP8 decoding) and the append of a new token to the paged caches: one
 *     fp32 scale per token, scale = amax / 448 (1 when that is 0), code =
 *     the E4M3 value nearest to x / scale, ties to an even code, magnitudes
 *     past 448 saturating to 448.  The scale and the quotient are fp32
 *     operations (the precision the library computes them in), so that the
 *     integer codes are decided the same way on both sides.
 *
 * Number formats are decoded from their published definitions:
 *   E4M3 (OCP 8-bit floating point, "E4M3FN"): 1 sign, 4 exponent (bias 7),
 *   3 mantissa bits, subnormals when the exponent field is 0, no infinities,
 *   S.1111.111 is NaN; largest finite magnitude 448.
 *   bfloat16: the upper 16 bits of an IEEE-754 binary32.
 *
 * Build: gcc -O2 -fopenmp -shared -fPIC (no fast-math: every sum is taken in
 * the order written here, in double precision).
 */
#include <float.h>
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

enum { OR_F32 = 0, OR_BF16 = 1, OR_E4M3 = 2 };

/* Stage 6's fp32 operations must round once, in single precision. */
#if FLT_EVAL_METHOD != 0
#error "the quantiser needs FLT_EVAL_METHOD == 0 (single-precision float arithmetic)"
#endif

/* ---------------- number formats ---------------- */

double dsa_or_e4m3(uint8_t code)
{
    int sign = (code >> 7) & 1;
    int e = (code >> 3) & 0xF;
    int m = code & 0x7;
    double mag;
    if (e == 0xF && m == 0x7) return NAN;             /* the only NaN pattern */
    if (e == 0) mag = ldexp((double)m / 8.0, 1 - 7);   /* subnormal: 0.m * 2^(1-bias) */
    else mag = ldexp(1.0 + (double)m / 8.0, e - 7);    /* normal: 1.m * 2^(e-bias) */
    return sign ? -mag : mag;
}

double dsa_or_bf16(uint16_t bits)
{
    uint32_t u = (uint32_t)bits << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

static double load_elem(const void *p, int dtype, int64_t i)
{
    switch (dtype) {
    case OR_F32: return (double)((const float *)p)[i];
    case OR_BF16: return dsa_or_bf16(((const uint16_t *)p)[i]);
    case OR_E4M3: return dsa_or_e4m3(((const uint8_t *)p)[i]);
    }
    return NAN;
}

/* ---------------- stage 1: indexer scores ---------------- */

/* One score I[t,s].  q_row: the H*D dequantised query values of token t;
 * k_row: the D dequantised key values of token s; w_row: H weights. */
static double index_score(const double *q_row, const double *k_row, const double *w_row,
                          int H, int D)
{
    double total = 0.0;
    for (int h = 0; h < H; ++h) {
        double dot = 0.0;
        for (int j = 0; j < D; ++j) dot += q_row[(int64_t)h * D + j] * k_row[j];
        double relu = dot > 0.0 ? dot : 0.0;
        total += w_row[h] * relu;
    }
    return total;
}

/* Dequantise the whole key matrix once: khat[s,j] = value(k[s,j]) * sk[s]. */
static double *dequant_keys(const void *k_idx, const float *k_scale, int kdt, int64_t T, int D)
{
    double *khat = (double *)malloc(sizeof(double) * (size_t)T * D);
    if (!khat) return NULL;
#pragma omp parallel for schedule(static)
    for (int64_t s = 0; s < T; ++s) {
        double sc = k_scale ? (double)k_scale[s] : 1.0;
        for (int j = 0; j < D; ++j) khat[s * D + j] = load_elem(k_idx, kdt, s * D + j) * sc;
    }
    return khat;
}

/* qhat / w of the r-th listed query row (arrays hold only the listed rows). */
static void dequant_query(const void *q_idx, const float *q_scale, int qdt, const void *w, int wdt,
                          int64_t r, int H, int D, double *q_row, double *w_row)
{
    double sc = q_scale ? (double)q_scale[r] : 1.0;
    for (int64_t i = 0; i < (int64_t)H * D; ++i)
        q_row[i] = load_elem(q_idx, qdt, r * H * D + i) * sc;
    for (int h = 0; h < H; ++h) w_row[h] = load_elem(w, wdt, r * H + h);
}

/*
 * Scores of the query rows at positions rows[0..nrows) against every key
 * 0..T-1: out[r*T + s] = I[rows[r], s] for s <= rows[r], -inf for s > rows[r].
 * q_idx [nrows,H,D], q_scale [nrows], w [nrows,H] hold the listed rows only;
 * k_idx [T,D], k_scale [T] hold every key.
 * idx_dtype: OR_F32 (q/k fp32, no scales) or OR_E4M3 (q/k bytes + scales);
 * w_dtype: OR_F32 or OR_BF16.  Returns 0, or -1 on allocation failure.
 */
int dsa_or_index_scores(const void *q_idx, const float *q_scale, const void *k_idx,
                        const float *k_scale, const void *w, int idx_dtype, int w_dtype,
                        int64_t T, int H, int D, const int64_t *rows, int64_t nrows, double *out)
{
    double *khat = dequant_keys(k_idx, k_scale, idx_dtype, T, D);
    if (!khat) return -1;
    int err = 0;
#pragma omp parallel
    {
        double *q_row = (double *)malloc(sizeof(double) * (size_t)H * D);
        double *w_row = (double *)malloc(sizeof(double) * (size_t)H);
        if (!q_row || !w_row) {
#pragma omp atomic write
            err = -1;
        } else {
#pragma omp for schedule(dynamic, 1)
            for (int64_t r = 0; r < nrows; ++r) {
                int64_t t = rows[r];
                dequant_query(q_idx, q_scale, idx_dtype, w, w_dtype, r, H, D, q_row, w_row);
                for (int64_t s = 0; s < T; ++s)
                    out[r * T + s] = (s <= t) ? index_score(q_row, khat + s * D, w_row, H, D)
                                              : -INFINITY;
            }
        }
        free(q_row);
        free(w_row);
    }
    free(khat);
    return err;
}

/* ---------------- stage 2: top-k ---------------- */

typedef struct { double score; int64_t pos; } cand_t;

/* (score descending, position ascending): the selector's total order. */
static int cand_cmp(const void *a, const void *b)
{
    const cand_t *x = (const cand_t *)a, *y = (const cand_t *)b;
    if (x->score > y->score) return -1;
    if (x->score < y->score) return 1;
    return (x->pos < y->pos) ? -1 : (x->pos > y->pos);
}

static int pos_cmp(const void *a, const void *b)
{
    int32_t x = *(const int32_t *)a, y = *(const int32_t *)b;
    return (x > y) - (x < y);
}

/* Select from scores[0..n) (n = t+1 candidates) the min(k,n) best positions. */
static int select_row(const double *scores, int64_t n, int k, int32_t *out, cand_t *buf)
{
    for (int64_t s = 0; s < n; ++s) { buf[s].score = scores[s]; buf[s].pos = s; }
    qsort(buf, (size_t)n, sizeof(cand_t), cand_cmp);
    int64_t m = n < k ? n : k;
    for (int64_t i = 0; i < m; ++i) out[i] = (int32_t)buf[i].pos;
    qsort(out, (size_t)m, sizeof(int32_t), pos_cmp);
    for (int64_t i = m; i < k; ++i) out[i] = -1;
    return 0;
}

/*
 * Top-k of each score row: row r holds the scores of query position rows[r]
 * (entries 0..rows[r] are candidates, the rest is ignored), with leading
 * dimension ld.  idx_out[r*k + i]: selected positions ascending, -1 padded.
 */
int dsa_or_topk(const double *scores, int64_t ld, const int64_t *rows, int64_t nrows, int k,
                int32_t *idx_out)
{
    int err = 0;
#pragma omp parallel
    {
        int64_t maxn = 0;
        for (int64_t r = 0; r < nrows; ++r) if (rows[r] + 1 > maxn) maxn = rows[r] + 1;
        cand_t *buf = (cand_t *)malloc(sizeof(cand_t) * (size_t)(maxn > 0 ? maxn : 1));
        if (!buf) {
#pragma omp atomic write
            err = -1;
        } else {
#pragma omp for schedule(dynamic, 4)
            for (int64_t r = 0; r < nrows; ++r)
                select_row(scores + r * ld, rows[r] + 1, k, idx_out + r * k, buf);
        }
        free(buf);
    }
    return err;
}

/* Stage 5 for one row of n = t+1 candidates: positions before the window
 * (0..n-1-window) compete by score for k slots, the last `window` positions
 * are taken as they are.  out[k + window]: the selected older positions
 * ascending, the window positions ascending, then -1. */
static void select_row_window(const double *scores, int64_t n, int k, int window, int32_t *out,
                              cand_t *buf)
{
    int64_t older = n > window ? n - window : 0;
    int64_t m = older < k ? older : k;
    if (older > 0) select_row(scores, older, k, out, buf);
    int64_t i = m;
    for (int64_t s = older; s < n; ++s) out[i++] = (int32_t)s;
    for (; i < (int64_t)k + window; ++i) out[i] = -1;
}

/*
 * Window-plus-top-k selection of each score row (stage 5): row r belongs to
 * query position rows[r]; idx_out[r*(k+window) + i] as select_row_window.
 */
int dsa_or_topk_window(const double *scores, int64_t ld, const int64_t *rows, int64_t nrows, int k,
                       int window, int32_t *idx_out)
{
    int err = 0;
    const int64_t width = (int64_t)k + window;
#pragma omp parallel
    {
        int64_t maxn = 0;
        for (int64_t r = 0; r < nrows; ++r) if (rows[r] + 1 > maxn) maxn = rows[r] + 1;
        cand_t *buf = (cand_t *)malloc(sizeof(cand_t) * (size_t)(maxn > 0 ? maxn : 1));
        if (!buf) {
#pragma omp atomic write
            err = -1;
        } else {
#pragma omp for schedule(dynamic, 4)
            for (int64_t r = 0; r < nrows; ++r)
                select_row_window(scores + r * ld, rows[r] + 1, k, window, idx_out + r * width, buf);
        }
        free(buf);
    }
    return err;
}

/* ---------------- stage 3: attention over the selected set ---------------- */

/* Attention of one query token (H heads of dimension D) over the rows listed
 * in sel[0..k) (-1 = unused).  krow(j)/vrow(j) give the key / value element
 * offsets of cache row j.  Writes o[H*D] and lse[H] (lse = -inf, o = 0 when
 * nothing is selected). */
static void attend_one_kv(const void *q, int64_t q_off, int qdt, const void *K, const void *V, int kvdt,
                          const float *ks, const float *vs, const int64_t *koff, int64_t nsel, int H,
                          int D, double sm, double *o, double *lse, double *z)
{
    for (int h = 0; h < H; ++h) {
        double zmax = -INFINITY;
        for (int64_t j = 0; j < nsel; ++j) {
            double kscale = ks ? (double)ks[koff[j] / D] : 1.0;
            double dot = 0.0;
            for (int c = 0; c < D; ++c)
                dot += load_elem(q, qdt, q_off + (int64_t)h * D + c) * (load_elem(K, kvdt, koff[j] + c) * kscale);
            z[j] = sm * dot;
            if (z[j] > zmax) zmax = z[j];
        }
        double l = 0.0;
        for (int64_t j = 0; j < nsel; ++j) { z[j] = exp(z[j] - zmax); l += z[j]; }
        for (int c = 0; c < D; ++c) {
            double acc = 0.0;
            for (int64_t j = 0; j < nsel; ++j) {
                double vscale = vs ? (double)vs[koff[j] / D] : 1.0;
                acc += z[j] * (load_elem(V, kvdt, koff[j] + c) * vscale);
            }
            o[(int64_t)h * D + c] = nsel > 0 ? acc / l : 0.0;
        }
        lse[h] = nsel > 0 ? zmax + log(l) : -INFINITY;
    }
}

/* Stage 3 with Q, K and V of one dtype and no scales. */
static void attend_one(const void *q, int64_t q_off, const void *K, const void *V, int dtype,
                       const int64_t *koff, int64_t nsel, int H, int D, double sm,
                       double *o, double *lse, double *z)
{
    attend_one_kv(q, q_off, dtype, K, V, dtype, NULL, NULL, koff, nsel, H, D, sm, o, lse, z);
}

/*
 * Sparse attention of nrows query rows: q [nrows,H,D] (the listed rows only),
 * K/V [*,D] of dtype OR_F32 or OR_BF16; idx [nrows, k] lists the K/V rows
 * each query attends to, entries -1 ignored.  out [nrows, H, D], lse
 * [nrows, H] (nullable).
 */
int dsa_or_sparse_attn(const void *q, const void *K, const void *V, int dtype, const int32_t *idx,
                       int64_t nrows, int k, int H, int D, double sm, double *out, double *lse)
{
    int err = 0;
#pragma omp parallel
    {
        int64_t *koff = (int64_t *)malloc(sizeof(int64_t) * (size_t)k);
        double *z = (double *)malloc(sizeof(double) * (size_t)k);
        double *l = (double *)malloc(sizeof(double) * (size_t)H);
        if (!koff || !z || !l) {
#pragma omp atomic write
            err = -1;
        } else {
#pragma omp for schedule(dynamic, 1)
            for (int64_t r = 0; r < nrows; ++r) {
                int64_t n = 0;
                for (int i = 0; i < k; ++i) {
                    int32_t j = idx[r * k + i];
                    if (j >= 0) koff[n++] = (int64_t)j * D;
                }
                attend_one(q, r * H * D, K, V, dtype, koff, n, H, D, sm,
                           out + r * H * D, l, z);
                if (lse) for (int h = 0; h < H; ++h) lse[r * H + h] = l[h];
            }
        }
        free(koff); free(z); free(l);
    }
    return err;
}

/* ---------------- stage 4: decode over paged caches ---------------- */

/*
 * One decode step for B sequences.  Sequence b has n = ctx[b] cached tokens
 * (the current token included) at positions 0..n-1; position s lives in
 * physical page bt[b*max_pages + s/ps], slot s%ps.
 *   q_idx  e4m3 [B,H_I,D_I], q_scale [B], w bf16 [B,H_I], q bf16 [B,H_q,D]
 *   kidx   e4m3 [P,ps,D_I], kscale f32 [P,ps], kc/vc bf16 [P,ps,D], or (stage
 *   7, when kcs and vcs are given) e4m3 [P,ps,D] with scales kcs/vcs f32 [P,ps]
 * window > 0 applies stage 5: the last `window` positions are always
 * attended and the top-k runs over the positions before them.
 * Outputs: scores_out [B, ld] (nullable; entries s < n), idx_out
 * [B, k+window] (positions, ascending, -1 padded), out [B,H_q,D], lse [B,H_q]
 * (nullable).
 */
int dsa_or_decode(const uint8_t *q_idx, const float *q_scale, const uint16_t *w,
                  const uint16_t *q, const uint8_t *kidx, const float *kscale,
                  const void *kc, const void *vc, const float *kcs, const float *vcs,
                  const int32_t *bt, const int32_t *ctx, int B, int max_pages, int ps, int H_I,
                  int D_I, int H_q, int D, int k, int window, double sm, double *scores_out,
                  int64_t ld, int32_t *idx_out, double *out, double *lse)
{
    int err = 0;
    for (int b = 0; b < B && !err; ++b) {
        int64_t n = ctx[b];
        double *sc = (double *)malloc(sizeof(double) * (size_t)(n > 0 ? n : 1));
        double *q_row = (double *)malloc(sizeof(double) * (size_t)H_I * D_I);
        double *w_row = (double *)malloc(sizeof(double) * (size_t)H_I);
        cand_t *buf = (cand_t *)malloc(sizeof(cand_t) * (size_t)(n > 0 ? n : 1));
        const int width = k + window;
        int64_t *koff = (int64_t *)malloc(sizeof(int64_t) * (size_t)width);
        double *z = (double *)malloc(sizeof(double) * (size_t)width);
        if (!sc || !q_row || !w_row || !buf || !koff || !z) err = -1;
        if (!err) {
            double sq = q_scale[b];
            for (int64_t i = 0; i < (int64_t)H_I * D_I; ++i)
                q_row[i] = dsa_or_e4m3(q_idx[(int64_t)b * H_I * D_I + i]) * sq;
            for (int h = 0; h < H_I; ++h) w_row[h] = dsa_or_bf16(w[(int64_t)b * H_I + h]);
#pragma omp parallel
            {
                double k_row[1024];
#pragma omp for schedule(static)
                for (int64_t s = 0; s < n; ++s) {
                    int64_t page = bt[(int64_t)b * max_pages + s / ps];
                    int64_t slot = page * ps + s % ps;
                    double sk = kscale[slot];
                    for (int j = 0; j < D_I; ++j) k_row[j] = dsa_or_e4m3(kidx[slot * D_I + j]) * sk;
                    sc[s] = index_score(q_row, k_row, w_row, H_I, D_I);
                }
            }
            if (scores_out) for (int64_t s = 0; s < n; ++s) scores_out[(int64_t)b * ld + s] = sc[s];
            int32_t *sel = idx_out + (int64_t)b * width;
            if (window > 0) select_row_window(sc, n, k, window, sel, buf);
            else select_row(sc, n, k, sel, buf);
            int64_t m = 0;
            for (int i = 0; i < width; ++i) {
                if (sel[i] < 0) continue;
                int64_t page = bt[(int64_t)b * max_pages + sel[i] / ps];
                koff[m++] = (page * ps + sel[i] % ps) * D;
            }
            double l[1024];
            attend_one_kv(q, (int64_t)b * H_q * D, OR_BF16, kc, vc, kcs ? OR_E4M3 : OR_BF16, kcs, vcs,
                          koff, m, H_q, D, sm, out + (int64_t)b * H_q * D, l, z);
            if (lse) for (int h = 0; h < H_q; ++h) lse[(int64_t)b * H_q + h] = l[h];
        }
        free(sc); free(q_row); free(w_row); free(buf); free(koff); free(z);
    }
    return err;
}

/* ---------------- stage 6: FP8 quantisation and cache append ---------------- */

/* The E4M3 code nearest to y: codes 0x00..0x7E are the non-negative finite
 * values in increasing order, so the two neighbours of |y| are found by a
 * scan; a tie goes to the even code (last mantissa bit 0); magnitudes past
 * the largest finite value (448) saturate to it.  The sign bit follows y's
 * sign (so -0 and negatives that round to zero give 0x80).  y must not be
 * NaN. */
uint8_t dsa_or_e4m3_encode(float y)
{
    double a = fabs((double)y);
    int lo = 0;
    for (int c = 0; c <= 0x7E; ++c)
        if (dsa_or_e4m3((uint8_t)c) <= a) lo = c;
    int mag;
    if (lo == 0x7E || dsa_or_e4m3((uint8_t)lo) == a) {
        mag = lo;
    } else {
        double below = a - dsa_or_e4m3((uint8_t)lo), above = dsa_or_e4m3((uint8_t)(lo + 1)) - a;
        if (below < above) mag = lo;
        else if (above < below) mag = lo + 1;
        else mag = (lo % 2 == 0) ? lo : lo + 1;
    }
    return (uint8_t)((signbit(y) ? 0x80 : 0x00) | mag);
}

/* Per-token scale and codes of one row of `cols` values. */
static void quantize_row(const void *x, int dtype, int64_t off, int64_t cols, uint8_t *codes,
                         float *scale)
{
    float amax = 0.0f;
    for (int64_t j = 0; j < cols; ++j) {
        float m = fabsf((float)load_elem(x, dtype, off + j));
        if (m > amax) amax = m;
    }
    float s = amax / 448.0f;
    if (!(s > 0.0f)) s = 1.0f;
    *scale = s;
    for (int64_t j = 0; j < cols; ++j) {
        float v = (float)load_elem(x, dtype, off + j);
        float y = v / s;
        codes[j] = dsa_or_e4m3_encode(y);
    }
}

/*
 * FP8 E4M3 quantisation with one scale per row: x [rows, cols] of dtype
 * OR_F32 or OR_BF16 (finite values) -> codes uint8 [rows, cols], scale f32
 * [rows].  Returns 0.
 */
int dsa_or_quantize_e4m3(const void *x, int dtype, int64_t rows, int64_t cols, uint8_t *codes,
                         float *scale)
{
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < rows; ++r) quantize_row(x, dtype, r * cols, cols, codes + r * cols, scale + r);
    return 0;
}

/*
 * Append N new tokens to the paged caches.  Token i goes to sequence seq[i]
 * at position pos[i], i.e. physical page bt[seq[i]*max_pages + pos[i]/ps],
 * slot pos[i]%ps: its index key kidx_new[i, 0..D_I) (OR_F32 or OR_BF16) is
 * quantised into kidx_cache/kscale_cache (stage 6), and its bf16 K and V rows
 * are copied into k_cache/v_cache -- or, when kcs/vcs are given (stage 7),
 * quantised into E4M3 k_cache/v_cache with scales kcs/vcs [P,ps].  bt is [B, max_pages].  Returns 0, or -2
 * (and stops) at the first token whose sequence, position or page id is out
 * of range.
 */
int dsa_or_cache_append(const void *kidx_new, int kdt, const uint16_t *k_new, const uint16_t *v_new,
                        const int32_t *seq, const int32_t *pos, int64_t N, int B, const int32_t *bt,
                        int max_pages, int64_t num_pages, int ps, int D_I, int D,
                        uint8_t *kidx_cache, float *kscale_cache, void *k_cache,
                        void *v_cache, float *kcs, float *vcs)
{
    for (int64_t i = 0; i < N; ++i) {
        int64_t p = pos[i];
        if (seq[i] < 0 || seq[i] >= B || p < 0 || p >= (int64_t)max_pages * ps) return -2;
        int64_t page = bt[(int64_t)seq[i] * max_pages + p / ps];
        if (page < 0 || page >= num_pages) return -2;
        int64_t slot = page * ps + p % ps;
        quantize_row(kidx_new, kdt, i * D_I, D_I, kidx_cache + slot * D_I, kscale_cache + slot);
        if (kcs) {                                  /* stage 7: FP8 K/V rows, one scale each */
            quantize_row(k_new, OR_BF16, i * D, D, (uint8_t *)k_cache + slot * D, kcs + slot);
            quantize_row(v_new, OR_BF16, i * D, D, (uint8_t *)v_cache + slot * D, vcs + slot);
        } else {
            for (int c = 0; c < D; ++c) {
                ((uint16_t *)k_cache)[slot * D + c] = k_new[i * D + c];
                ((uint16_t *)v_cache)[slot * D + c] = v_new[i * D + c];
            }
        }
    }
    return 0;
}
