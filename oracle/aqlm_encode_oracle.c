/*
 * aqlm_encode_oracle.c -- plain, slow CPU oracle for the step before AQLM
 * inference: turning a weight matrix into scales, codebooks and codes.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path may link, load or
 * call this file: only the tests and the benchmark's CPU baseline leg use it.
 * It shares no code, header, table or helper with the CUDA library.
 *
 * Source: "The AQLM Quantization Algorithm, Explained" (Towards Data Science
 * repost), section "AQLM quantization process": for every linear layer the
 * codes are learned first with the codebooks and scales fixed, the codebooks
 * being "initialized with a residual k-means approach"; the loss, the search
 * and the later codebook updates are not given (their formulas were lost or
 * never stated).  Section "What is Multi-Codebook Quantization (MCQ)?": each
 * output channel is scaled, then cut into groups of g = 8 inputs, and each
 * group is approximated by the sum of M codewords, one per codebook of 2^B.
 *
 * Readings where the pages are silent (each listed in the design notes):
 *   E1 scale of row i: the root mean square of the row, rounded to binary16
 *      (1.0 if that rounds to zero); the sum of squares is a plain
 *      left-to-right sum in double of the exact squares (double holds the
 *      square of every binary32 value exactly);
 *   E2 the groups to encode are the row's inputs divided by the scale
 *      (binary32 division, correctly rounded);
 *   E3 nearest codeword: the one of least squared Euclidean distance
 *      |v - c|^2 = sum_t (v_t - c_t)^2, evaluated here in double for every
 *      codeword, ties to the lowest index.  Any evaluation of the distance
 *      carries rounding error, so another implementation (in binary32, in
 *      any order) may pick a different codeword only where two distances
 *      lie within its error bound of each other; the tests check exactly
 *      that, with the bound stated there;
 *   E4 k-means update (Lloyd): a centroid becomes the mean of the groups
 *      assigned to it (sums in double, one rounding to binary32); a centroid
 *      with no group keeps its value;
 *   E5 residual k-means: codebook m is k-means (with `iters` updates) of the
 *      residuals left by codebooks 0..m-1, started from the K residuals named
 *      by init_idx[m] (the random draw, passed in); the residual then loses
 *      the nearest centroid of the final codebook;
 *   E6 codes, with the codebooks fixed: greedy, codebook by codebook, each
 *      code the nearest codeword of the current residual (binary32
 *      subtraction of the chosen codeword).
 */
#include <stdint.h>
#include <string.h>
#include <math.h>
#include <stdlib.h>

#ifdef _OPENMP
#include <omp.h>
#endif

/* ---- real number -> binary16, round to nearest, ties to even ------------- */
/* From the IEEE 754 definition: 1 sign bit, 5 exponent bits (bias 15), 10
 * fraction bits; subnormals are the multiples of 2^-24 below 2^-14; values
 * from 65520 up round to infinity.  The input is a double, which holds every
 * binary32 value exactly, so this serves both the binary32 codebooks and the
 * double scales without a second rounding.  rint() rounds half to even in
 * the default rounding mode; the divisions by powers of two are exact. */
uint16_t aqlm_oracle_double_to_half(double x)
{
    const uint16_t sign = signbit(x) ? 0x8000u : 0u;
    const double a = fabs(x);
    if (isnan(x)) return (uint16_t)(sign | 0x7e00u);
    if (a >= 65520.0) return (uint16_t)(sign | 0x7c00u);
    if (a < ldexp(1.0, -14)) {                   /* subnormal: q * 2^-24 */
        return (uint16_t)(sign | (uint16_t)rint(ldexp(a, 24)));
    }
    int e;
    frexp(a, &e);                                /* a in [2^(e-1), 2^e) */
    double q = rint(ldexp(a, 11 - e));           /* a / 2^(e-11), in [1024, 2048] */
    if (q == 2048.0) {
        q = 1024.0;
        e += 1;
    }
    const int hexp = e - 1 + 15;
    if (hexp >= 31) return (uint16_t)(sign | 0x7c00u);
    return (uint16_t)(sign | (uint16_t)(hexp << 10) | (uint16_t)((int)q - 1024));
}

static float half_to_float(uint16_t h)
{
    const int sign = (h >> 15) & 1;
    const int expo = (h >> 10) & 0x1f;
    const int frac = h & 0x3ff;
    double v;
    if (expo == 0) {
        v = ldexp((double)frac, -24);
    } else if (expo == 31) {
        v = frac ? NAN : INFINITY;
    } else {
        v = ldexp((double)(frac | 0x400), expo - 25);
    }
    return (float)(sign ? -v : v);
}

/* ---- E1, E2: row scales and the groups to encode ------------------------ */

/* Sum of squares of one row, left to right, in double. */
static double row_sum_squares(const float *row, int64_t n)
{
    double acc = 0.0;
    for (int64_t k = 0; k < n; ++k) acc += (double)row[k] * (double)row[k];
    return acc;
}

int aqlm_oracle_encode_scales(const float *W, int64_t d_out, int64_t d_in, uint16_t *scales, float *V)
{
    if (d_out < 1 || d_in < 8 || d_in % 8) return 1;
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < d_out; ++i) {
        const float *row = W + i * d_in;
        const double rms = sqrt(row_sum_squares(row, d_in) / (double)d_in);
        uint16_t h = aqlm_oracle_double_to_half(rms);
        if ((h & 0x7fffu) == 0) h = 0x3c00u;       /* 1.0 */
        scales[i] = h;
        const float s = half_to_float(h);
        for (int64_t k = 0; k < d_in; ++k) V[i * d_in + k] = row[k] / s;
    }
    return 0;
}

/* ---- E3: nearest codeword ------------------------------------------------ */

/* Squared Euclidean distance of two groups, in double. */
static double distance(const float *v, const float *c)
{
    double d = 0.0;
    for (int t = 0; t < 8; ++t) {
        const double e = (double)v[t] - (double)c[t];
        d += e * e;
    }
    return d;
}

/* The nearest codeword of v (least distance, ties to the lowest index);
 * *best_d receives its distance and *second_d the least distance over the
 * other codewords (+inf when K = 1). */
static int64_t nearest_one(const float *v, const float *C, int64_t K, double *best_d, double *second_d)
{
    int64_t best = 0;
    double bd = distance(v, C), sd = INFINITY;
    for (int64_t k = 1; k < K; ++k) {
        const double dk = distance(v, C + k * 8);
        if (dk < bd) {
            sd = bd;
            bd = dk;
            best = k;
        } else if (dk < sd) {
            sd = dk;
        }
    }
    if (best_d) *best_d = bd;
    if (second_d) *second_d = sd;
    return best;
}

/* idx[n], dist[n] (its distance) and second[n] (the runner-up's distance) of
 * each of the N groups of V; dist and second may be NULL. */
int aqlm_oracle_nearest(const float *V, int64_t N, const float *C, int64_t K, int32_t *idx, double *dist,
                        double *second)
{
    if (N < 0 || K < 1) return 1;
#pragma omp parallel for schedule(static)
    for (int64_t n = 0; n < N; ++n) {
        double bd, sd;
        idx[n] = (int32_t)nearest_one(V + n * 8, C, K, &bd, &sd);
        if (dist) dist[n] = bd;
        if (second) second[n] = sd;
    }
    return 0;
}

/* ---- E4: k-means update -------------------------------------------------- */

int aqlm_oracle_kmeans_update(const float *V, const int32_t *idx, int64_t N, int64_t K, const float *C_prev,
                              float *C_out, int64_t *counts)
{
    if (N < 0 || K < 1) return 1;
    double *sums = (double *)calloc((size_t)K * 8, sizeof(double));
    if (!sums) return 2;
    for (int64_t k = 0; k < K; ++k) counts[k] = 0;
    for (int64_t n = 0; n < N; ++n) {
        const int64_t k = idx[n];
        if (k < 0 || k >= K) {
            free(sums);
            return 1;
        }
        counts[k] += 1;
        for (int t = 0; t < 8; ++t) sums[k * 8 + t] += (double)V[n * 8 + t];
    }
    for (int64_t k = 0; k < K; ++k) {
        for (int t = 0; t < 8; ++t)
            C_out[k * 8 + t] = counts[k] ? (float)(sums[k * 8 + t] / (double)counts[k]) : C_prev[k * 8 + t];
    }
    free(sums);
    return 0;
}

/* ---- E5: residual k-means ------------------------------------------------ */

int aqlm_oracle_residual_kmeans(const float *V, int64_t N, int M, int64_t K, const int32_t *init_idx, int iters,
                                float *C_out)
{
    if (N < 1 || M < 1 || K < 1 || iters < 0) return 1;
    float *R = (float *)malloc((size_t)N * 8 * sizeof(float));
    int32_t *idx = (int32_t *)malloc((size_t)N * sizeof(int32_t));
    float *tmp = (float *)malloc((size_t)K * 8 * sizeof(float));
    int64_t *counts = (int64_t *)malloc((size_t)K * sizeof(int64_t));
    if (!R || !idx || !tmp || !counts) {
        free(R); free(idx); free(tmp); free(counts);
        return 2;
    }
    memcpy(R, V, (size_t)N * 8 * sizeof(float));
    int rc = 0;
    for (int m = 0; m < M && !rc; ++m) {
        float *C = C_out + (int64_t)m * K * 8;
        for (int64_t k = 0; k < K; ++k) {
            const int64_t n = init_idx[(int64_t)m * K + k];
            if (n < 0 || n >= N) { rc = 1; break; }
            memcpy(C + k * 8, R + n * 8, 8 * sizeof(float));
        }
        for (int it = 0; it < iters && !rc; ++it) {
            aqlm_oracle_nearest(R, N, C, K, idx, NULL, NULL);
            rc = aqlm_oracle_kmeans_update(R, idx, N, K, C, tmp, counts);
            memcpy(C, tmp, (size_t)K * 8 * sizeof(float));
        }
        if (rc) break;
        aqlm_oracle_nearest(R, N, C, K, idx, NULL, NULL);
        for (int64_t n = 0; n < N; ++n)
            for (int t = 0; t < 8; ++t) R[n * 8 + t] = R[n * 8 + t] - C[(int64_t)idx[n] * 8 + t];
    }
    free(R); free(idx); free(tmp); free(counts);
    return rc;
}

/* ---- E6: greedy codes with fixed binary16 codebooks ---------------------- */

/* codebooks [M][K][8] binary16; codes [N][M] as uint16 (the code value). */
int aqlm_oracle_encode_greedy(const float *V, int64_t N, const uint16_t *codebooks, int M, int64_t K,
                              uint16_t *codes)
{
    if (N < 0 || M < 1 || K < 1 || K > 65536) return 1;
    float *C = (float *)malloc((size_t)M * K * 8 * sizeof(float));
    if (!C) return 2;
    for (int64_t i = 0; i < (int64_t)M * K * 8; ++i) C[i] = half_to_float(codebooks[i]);
#pragma omp parallel for schedule(static)
    for (int64_t n = 0; n < N; ++n) {
        float r[8];
        memcpy(r, V + n * 8, sizeof(r));
        for (int m = 0; m < M; ++m) {
            const float *Cm = C + (int64_t)m * K * 8;
            const int64_t best = nearest_one(r, Cm, K, NULL, NULL);
            codes[n * M + m] = (uint16_t)best;
            for (int t = 0; t < 8; ++t) r[t] = r[t] - Cm[best * 8 + t];
        }
    }
    free(C);
    return 0;
}
