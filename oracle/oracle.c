/*
 * oracle.c -- plain, slow, obviously-correct CPU reference for
 *   (1) the lightning-indexer score and exact top-k of FlashTopK, and
 *   (2) DeepSelect's row top-k.
 *
 * TEST INFRASTRUCTURE ONLY.  The tests, the smoke check and the CPU-baseline
 * leg of the benchmark load this library; the product library never links,
 * loads or calls it, and the two share no code (no headers, no tables).
 *
 * Everything is computed in IEEE double.  Every FP8-e4m3 / BF16 / FP32 input
 * value converts to double exactly, every product of two FP8 or two BF16
 * values is exact in double, so the only rounding here is in the sums.
 *
 * Sources (web pages; cited by page title and section):
 *   [FTK-QS]  FlashTopK README, "Quick start": the score
 *             I[t,s] = sigma_s * sum_{h=1..H} w[t,h] * ReLU(q[t,h] . k[s]),
 *             H = 32 heads of dimension 128, window [ks[t], ke[t]),
 *             sigma = kv_scales, 1 for BF16 keys; output int32 indices
 *             [T, topk].
 *   [FTK-RM]  FlashTopK README, "Roadmap": indexers with other head counts,
 *             such as 64 heads.  The head count H is an argument here
 *             (the sum runs over every head of q[t]).
 *   [FTK-HL]  FlashTopK README, "Highlights": exact top-k; ties at the k-th
 *             score keep the smallest key indices.
 *   [FTK-SUP] FlashTopK README, "Support": 32 heads x 128, FP8 or BF16,
 *             topk up to 4096.
 *   [DS-USE]  DeepSelect README, "Usage" / "Variable-length rows": row top-k
 *             of a [batch, vocab] bf16/fp32 matrix, values of x's dtype,
 *             short rows padded with fill values.
 *   [DS-NAN]  DeepSelect README, "NaN handling".
 *
 * Readings where the pages are silent:
 *   - padding of a window shorter than topk: index -1, value -inf;
 *   - -0.0 and +0.0 are the same score (compared by value);
 *   - a NaN anywhere in a row's scores makes that row's result unspecified
 *     and sets the row's flag (the pages' library aborts instead);
 *   - the FP8 format is e4m3fn: bias 7, no infinities, S.1111.111 is NaN.
 *
 * Parity status: every function here is pinned by tests/test_oracle.py
 * against torch's dtype conversions, numpy matmul special cases, brute-force
 * subset enumeration and closed-form cases.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

enum { ORC_E4M3 = 1, ORC_BF16 = 2, ORC_F32 = 3 };
enum { ORC_DIM = 128 };  /* head dimension; the head count H is an argument */

/* ---------------------------------------------------------------------- */
/* Value decoding                                                           */
/* ---------------------------------------------------------------------- */

/* FP8 e4m3fn code -> double.  1 sign bit, 4 exponent bits (bias 7), 3
 * mantissa bits; exponent field 0 is subnormal (m/8 * 2^-6); exponent 15
 * with mantissa 7 is NaN; there is no infinity. */
double orc_e4m3_value(unsigned code)
{
    unsigned sign = (code >> 7) & 1u;
    unsigned e = (code >> 3) & 15u;
    unsigned m = code & 7u;
    double mag;
    if (e == 15u && m == 7u)
        return NAN;
    if (e == 0u)
        mag = ldexp((double)m / 8.0, -6);
    else
        mag = ldexp(1.0 + (double)m / 8.0, (int)e - 7);
    return sign ? -mag : mag;
}

/* BF16 bits -> double: the bf16 pattern is the top half of an IEEE binary32. */
double orc_bf16_value(unsigned bits)
{
    uint32_t w = (uint32_t)(bits & 0xFFFFu) << 16;
    float f;
    memcpy(&f, &w, sizeof f);
    return (double)f;
}

static double f32_value(const void *p, int64_t i)
{
    float f;
    memcpy(&f, (const char *)p + 4 * i, sizeof f);
    return (double)f;
}

/* Element i of a buffer of the given dtype, as a double. */
static double element(int dtype, const void *p, int64_t i)
{
    if (dtype == ORC_E4M3)
        return orc_e4m3_value(((const uint8_t *)p)[i]);
    if (dtype == ORC_BF16)
        return orc_bf16_value(((const uint16_t *)p)[i]);
    return f32_value(p, i);
}

/* Decode n elements into doubles (exposed for the dtype pins). */
void orc_decode(int dtype, const void *src, int64_t n, double *dst)
{
    for (int64_t i = 0; i < n; ++i)
        dst[i] = element(dtype, src, i);
}

/* ---------------------------------------------------------------------- */
/* Score  [FTK-QS]                                                          */
/* ---------------------------------------------------------------------- */

/* Score of one (t, s) pair and its rounding-error scale
 *   E = sigma_s * sum_h |w[t,h]| * sum_d |q[t,h,d] * k[s,d]|.
 * qd: the heads x 128 decoded heads of q[t]; wt: the heads weights of row t. */
static void score_pair(int heads, const double *qd, const double *wt, const double *kd,
                       double sigma, double *I_out, double *E_out)
{
    double acc = 0.0, err = 0.0;
    for (int h = 0; h < heads; ++h) {
        double dot = 0.0, absdot = 0.0;
        for (int d = 0; d < ORC_DIM; ++d) {
            double p = qd[h * ORC_DIM + d] * kd[d];
            dot += p;
            absdot += fabs(p);
        }
        double relu = dot > 0.0 ? dot : 0.0;
        acc += wt[h] * relu;
        err += fabs(wt[h]) * absdot;
    }
    *I_out = sigma * acc;
    *E_out = fabs(sigma) * err;
}

static int window_ok(int32_t ks, int32_t ke, int64_t S)
{
    return ks >= 0 && ks <= ke && (int64_t)ke <= S;
}

/*
 * Scores of the windows of the listed rows.
 *   heads    H >= 1, the head count of the indexer
 *   q        [T, H, 128] of dtype, row-major
 *   kv       [S, 128] of dtype
 *   kv_scales [S] float32, or NULL for all-ones
 *   weights  [T, H] float32
 *   rows     the nrows query indices to score
 *   out_I, out_E  [nrows, ld]: entry (r, s - ks[t]) for s in [ks[t], ke[t])
 * Returns the number of listed rows with an invalid window (those rows are
 * left untouched).
 */
int64_t orc_index_scores(int dtype, int heads, const void *q, const void *kv,
                         const float *kv_scales, const float *weights,
                         int64_t T, int64_t S, const int32_t *ks,
                         const int32_t *ke, const int64_t *rows,
                         int64_t nrows, int64_t ld, double *out_I,
                         double *out_E)
{
    int64_t bad = 0;
#pragma omp parallel for schedule(dynamic, 1) reduction(+ : bad)
    for (int64_t r = 0; r < nrows; ++r) {
        int64_t t = rows[r];
        if (t < 0 || t >= T || !window_ok(ks[t], ke[t], S)) {
            bad += 1;
            continue;
        }
        double *qd = (double *)malloc(sizeof(double) * heads * ORC_DIM);
        double *wt = (double *)malloc(sizeof(double) * heads);
        double kd[ORC_DIM];
        for (int64_t i = 0; i < (int64_t)heads * ORC_DIM; ++i)
            qd[i] = element(dtype, q, t * heads * ORC_DIM + i);
        for (int h = 0; h < heads; ++h)
            wt[h] = (double)weights[t * heads + h];
        for (int64_t s = ks[t]; s < ke[t]; ++s) {
            for (int d = 0; d < ORC_DIM; ++d)
                kd[d] = element(dtype, kv, s * ORC_DIM + d);
            double sigma = kv_scales ? (double)kv_scales[s] : 1.0;
            double I, E;
            score_pair(heads, qd, wt, kd, sigma, &I, &E);
            out_I[r * ld + (s - ks[t])] = I;
            if (out_E)
                out_E[r * ld + (s - ks[t])] = E;
        }
        free(qd);
        free(wt);
    }
    return bad;
}

/* ---------------------------------------------------------------------- */
/* Score bound of a key block  [FTK-HL]                                     */
/* ---------------------------------------------------------------------- */

/*
 * Upper bound on the score of row t over a block of keys [FTK-HL: adaptive
 * key pruning skips keys by a score bound.  The pages give the bound no
 * formula; this is the plain per-dimension box bound].
 * For the keys s of block b, i.e. [b*block, min((b+1)*block, S)):
 *   hi[d] = max_s sigma_s * k[s,d],  lo[d] = min_s sigma_s * k[s,d]
 *   U_h = sum_d max(q[t,h,d] * hi[d], q[t,h,d] * lo[d])   (>= q_h . sigma_s k_s)
 *   L_h = sum_d min(q[t,h,d] * hi[d], q[t,h,d] * lo[d])   (<= q_h . sigma_s k_s)
 *   UB  = sum_h (w[t,h] >= 0 ? w[t,h] * ReLU(U_h) : w[t,h] * ReLU(L_h))
 * For sigma_s > 0, sigma_s * sum_h w_h ReLU(x_h) = sum_h w_h ReLU(sigma_s x_h),
 * so UB >= I[t,s] for every key of the block.
 *   out_ub    [nrows, nblocks]: UB of (rows[r], b); NaN for a listed row
 *             outside [0, T)
 *   out_scale [nrows, nblocks] or NULL: sum_h |w| sum_d |q| max(|hi|, |lo|),
 *             the size of the terms UB is summed from
 */
void orc_block_bound(int dtype, int heads, const void *q, const void *kv, const float *kv_scales,
                     const float *weights, int64_t T, int64_t S, int64_t block,
                     const int64_t *rows, int64_t nrows, double *out_ub, double *out_scale)
{
    int64_t nb = (S + block - 1) / block;
    double *hi = malloc(sizeof(double) * nb * ORC_DIM);
    double *lo = malloc(sizeof(double) * nb * ORC_DIM);
    for (int64_t b = 0; b < nb; ++b) {
        for (int d = 0; d < ORC_DIM; ++d) {
            hi[b * ORC_DIM + d] = -INFINITY;
            lo[b * ORC_DIM + d] = INFINITY;
        }
        for (int64_t s = b * block; s < S && s < (b + 1) * block; ++s) {
            double sigma = kv_scales ? (double)kv_scales[s] : 1.0;
            for (int d = 0; d < ORC_DIM; ++d) {
                double v = sigma * element(dtype, kv, s * ORC_DIM + d);
                if (v > hi[b * ORC_DIM + d]) hi[b * ORC_DIM + d] = v;
                if (v < lo[b * ORC_DIM + d]) lo[b * ORC_DIM + d] = v;
            }
        }
    }
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t r = 0; r < nrows; ++r) {
        int64_t t = rows[r];
        if (t < 0 || t >= T) {
            for (int64_t b = 0; b < nb; ++b) {
                out_ub[r * nb + b] = NAN;
                if (out_scale)
                    out_scale[r * nb + b] = NAN;
            }
            continue;
        }
        double *qd = (double *)malloc(sizeof(double) * heads * ORC_DIM);
        double *wt = (double *)malloc(sizeof(double) * heads);
        for (int64_t i = 0; i < (int64_t)heads * ORC_DIM; ++i)
            qd[i] = element(dtype, q, t * heads * ORC_DIM + i);
        for (int h = 0; h < heads; ++h)
            wt[h] = weights[(int64_t)t * heads + h];
        for (int64_t b = 0; b < nb; ++b) {
            const double *bh = hi + b * ORC_DIM, *bl = lo + b * ORC_DIM;
            double ub = 0.0, scale = 0.0;
            for (int h = 0; h < heads; ++h) {
                double U = 0.0, L = 0.0, mag = 0.0;
                for (int d = 0; d < ORC_DIM; ++d) {
                    double x = qd[h * ORC_DIM + d] * bh[d];
                    double y = qd[h * ORC_DIM + d] * bl[d];
                    U += x > y ? x : y;
                    L += x < y ? x : y;
                    mag += fabs(qd[h * ORC_DIM + d]) * (fabs(bh[d]) > fabs(bl[d]) ? fabs(bh[d]) : fabs(bl[d]));
                }
                if (wt[h] >= 0.0)
                    ub += wt[h] * (U > 0.0 ? U : 0.0);
                else
                    ub += wt[h] * (L > 0.0 ? L : 0.0);
                scale += fabs(wt[h]) * mag;
            }
            out_ub[r * nb + b] = ub;
            if (out_scale)
                out_scale[r * nb + b] = scale;
        }
        free(qd);
        free(wt);
    }
    free(hi);
    free(lo);
}

/* ---------------------------------------------------------------------- */
/* Selection  [FTK-HL], [DS-USE]                                            */
/* ---------------------------------------------------------------------- */

typedef struct {
    double v;
    int64_t i;
} keyed;

/* Order: larger value first; equal values by smaller index first.  NaN is
 * placed after every number so that the sort stays a total order (rows with
 * NaN are flagged and their result is unspecified). */
static int keyed_cmp(const void *a, const void *b)
{
    const keyed *x = (const keyed *)a, *y = (const keyed *)b;
    int xn = isnan(x->v), yn = isnan(y->v);
    if (xn != yn)
        return xn ? 1 : -1;
    if (!xn) {
        if (x->v > y->v)
            return -1;
        if (x->v < y->v)
            return 1;
    }
    return (x->i < y->i) ? -1 : (x->i > y->i) ? 1 : 0;
}

/*
 * Exact top-k of one window of values.
 *   vals[j] is the score of key (first_index + j), j < L.
 * Writes min(k, L) entries in (value desc, index asc) order, then pads with
 * index -1 / value -inf up to k.  Returns 1 if a NaN was seen, else 0.
 */
int orc_select_f64(const double *vals, int64_t L, int64_t first_index, int k,
                   int64_t *out_idx, double *out_val)
{
    int nan_seen = 0;
    keyed *buf = (keyed *)malloc((size_t)(L > 0 ? L : 1) * sizeof(keyed));
    for (int64_t j = 0; j < L; ++j) {
        buf[j].v = vals[j];
        buf[j].i = first_index + j;
        if (isnan(vals[j]))
            nan_seen = 1;
    }
    qsort(buf, (size_t)L, sizeof(keyed), keyed_cmp);
    int64_t n = L < k ? L : k;
    for (int64_t j = 0; j < k; ++j) {
        out_idx[j] = j < n ? buf[j].i : -1;
        out_val[j] = j < n ? buf[j].v : -INFINITY;
    }
    free(buf);
    return nan_seen;
}

/* Same selection on float32 values (each widened exactly to double), one
 * call per row: scores [rows, ld], row r holds the window of query
 * (row_ids ? row_ids[r] : r) starting at column 0.  Returns the number of
 * rows with a NaN or an invalid window. */
int64_t orc_select_f32_rows(const float *scores, int64_t rows, int64_t ld,
                            const int32_t *ks, const int32_t *ke, int64_t S,
                            const int64_t *row_ids, int k, int64_t *out_idx,
                            double *out_val)
{
    int64_t flagged = 0;
#pragma omp parallel for schedule(dynamic, 1) reduction(+ : flagged)
    for (int64_t r = 0; r < rows; ++r) {
        int64_t t = row_ids ? row_ids[r] : r;
        if (!window_ok(ks[t], ke[t], S)) {
            flagged += 1;
            for (int j = 0; j < k; ++j) {
                out_idx[r * k + j] = -1;
                out_val[r * k + j] = -INFINITY;
            }
            continue;
        }
        int64_t L = (int64_t)ke[t] - ks[t];
        double *v = (double *)malloc((size_t)(L > 0 ? L : 1) * sizeof(double));
        for (int64_t j = 0; j < L; ++j)
            v[j] = (double)scores[r * ld + j];
        flagged += orc_select_f64(v, L, ks[t], k, out_idx + r * k,
                                  out_val + r * k);
        free(v);
    }
    return flagged;
}

/*
 * Fused score + exact top-k for the listed rows [FTK-QS], [FTK-HL]:
 * the definition written out -- score every key of the window in double,
 * then sort.  out_idx / out_val are [nrows, k].  row_flags (optional,
 * [nrows]) gets 1 for a NaN score, 2 for an invalid window.
 * Returns the number of flagged rows.
 */
int64_t orc_fused_select(int dtype, int heads, const void *q, const void *kv,
                         const float *kv_scales, const float *weights,
                         int64_t T, int64_t S, const int32_t *ks,
                         const int32_t *ke, const int64_t *rows, int64_t nrows,
                         int k, int64_t *out_idx, double *out_val,
                         int32_t *row_flags)
{
    int64_t flagged = 0;
#pragma omp parallel for schedule(dynamic, 1) reduction(+ : flagged)
    for (int64_t r = 0; r < nrows; ++r) {
        int64_t t = rows[r];
        int32_t flag = 0;
        if (t < 0 || t >= T || !window_ok(ks[t], ke[t], S)) {
            flag = 2;
            for (int j = 0; j < k; ++j) {
                out_idx[r * k + j] = -1;
                out_val[r * k + j] = -INFINITY;
            }
        } else {
            int64_t L = (int64_t)ke[t] - ks[t];
            double *I = (double *)malloc((size_t)(L > 0 ? L : 1) * sizeof(double));
            int64_t one = t;
            orc_index_scores(dtype, heads, q, kv, kv_scales, weights, T, S, ks, ke,
                             &one, 1, L > 0 ? L : 1, I, NULL);
            if (orc_select_f64(I, L, ks[t], k, out_idx + r * k,
                               out_val + r * k))
                flag = 1;
            free(I);
        }
        if (row_flags)
            row_flags[r] = flag;
        flagged += flag != 0;
    }
    return flagged;
}

/*
 * Row top-k [DS-USE]: x is [rows, cols] (row stride ld elements) of bf16 or
 * float32.  Keeps the k largest values of each row, ties to the smaller
 * column index; rows shorter than k are padded with (-1, -inf).
 * out_val holds the selected values widened to double.  row_flags
 * (optional) gets 1 for a row containing NaN [DS-NAN].  Returns the number of
 * flagged rows.
 */
int64_t orc_topk_rows(int dtype, const void *x, int64_t rows, int64_t cols,
                      int64_t ld, int k, int64_t *out_idx, double *out_val,
                      int32_t *row_flags)
{
    int64_t flagged = 0;
#pragma omp parallel for schedule(dynamic, 1) reduction(+ : flagged)
    for (int64_t r = 0; r < rows; ++r) {
        double *v = (double *)malloc((size_t)(cols > 0 ? cols : 1) * sizeof(double));
        for (int64_t c = 0; c < cols; ++c)
            v[c] = element(dtype, x, r * ld + c);
        int f = orc_select_f64(v, cols, 0, k, out_idx + r * k, out_val + r * k);
        if (row_flags)
            row_flags[r] = f;
        flagged += f;
        free(v);
    }
    return flagged;
}

/* Threads the OpenMP loops above use (the benchmark reports it). */
int orc_num_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
