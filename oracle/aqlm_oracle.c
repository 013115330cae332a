/*
 * aqlm_oracle.c -- plain, slow CPU oracle for AQLM inference.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path may link, load or
 * call this file: only the tests, the package's smoke() check and the CPU
 * baseline leg of the benchmark use it.  It shares no code, header, table or
 * helper with the CUDA library.
 *
 * Source of every definition below: the blog post "The AQLM Quantization
 * Algorithm, Explained" (Towards Data Science repost), sections
 *   - "What is Multi-Codebook Quantization (MCQ)?": each row of W (d_out x
 *     d_in) is cut into groups of g consecutive inputs; a group is the sum of
 *     M codewords, one from each of M codebooks of 2^B codewords; the stored
 *     code of a codeword is its B-bit index; after decoding, the summed
 *     codewords are scaled per output channel and the product W.X is taken in
 *     native precision;
 *   - "Memory footprint of AQLM-quantized models": the three stored terms
 *     (codebooks at 16 bit, d_out 16-bit scales, M B-bit codes per group),
 *     whose sum per parameter is the average bit rate of one layer;
 * and the abstract of "Extreme Compression of Large Language Models via
 * Additive Quantization" (ICML 2024 record): additive quantization of weight
 * matrices.
 *
 * Readings where the pages are silent (each listed in the design notes):
 *   - codes are stored [d_out][d_in/g][M], m fastest; B = 8 codes are uint8,
 *     B = 16 codes are 16-bit words whose index is the unsigned value;
 *   - codebooks are [M][2^B][g] IEEE binary16, scales [d_out] binary16;
 *   - the scale multiplies the sum of the M codewords.
 *
 * Precision: everything is evaluated in double from the exact values of the
 * 16-bit inputs, except aqlm_oracle_dequant_bf16, which restates the
 * dequantisation as an explicit sequence of IEEE binary32 operations so that
 * a bf16 result can be compared bit for bit.
 *
 * Parity pins for each function are in tests/test_oracle.py.
 */
#include <stdint.h>
#include <string.h>
#include <math.h>

#ifdef _OPENMP
#include <omp.h>
#endif

/* ---- number formats, written from the IEEE 754 definitions ------------- */

/* binary16: 1 sign bit, 5 exponent bits (bias 15), 10 fraction bits. */
static double half_bits_to_double(uint16_t h)
{
    int sign = (h >> 15) & 1;
    int expo = (h >> 10) & 0x1f;
    int frac = h & 0x3ff;
    double v;
    if (expo == 0) {
        v = ldexp((double)frac, -24);                 /* subnormal: frac * 2^-24 */
    } else if (expo == 31) {
        v = frac ? NAN : INFINITY;
    } else {
        v = ldexp((double)(frac | 0x400), expo - 25);  /* 1.frac * 2^(e-15) */
    }
    return sign ? -v : v;
}

/* bfloat16 is the upper half of a binary32. */
static float bf16_bits_to_float(uint16_t b)
{
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, 4);
    return f;
}

/* binary32 -> bfloat16, round to nearest, ties to even; NaN stays NaN. */
static uint16_t float_to_bf16_bits_rne(float f)
{
    uint32_t u;
    memcpy(&u, &f, 4);
    if ((u & 0x7f800000u) == 0x7f800000u && (u & 0x007fffffu)) {
        return (uint16_t)((u >> 16) | 0x0040u);       /* quiet NaN, sign kept */
    }
    uint32_t lower = u & 0xffffu;
    uint32_t upper = u >> 16;
    if (lower > 0x8000u || (lower == 0x8000u && (upper & 1u))) {
        upper += 1u;                                   /* may carry into inf */
    }
    return (uint16_t)upper;
}

/* ---- code access ------------------------------------------------------- */

/* Index of the codeword that codebook m contributes to group j of row i.
 * B = 8: one byte per code; B = 16: one 16-bit word, read as unsigned. */
static uint32_t code_at(const void *codes, int64_t i, int64_t j, int m,
                        int64_t groups, int M, int B)
{
    int64_t pos = (i * groups + j) * M + m;
    if (B == 8) {
        return ((const uint8_t *)codes)[pos];
    }
    return ((const uint16_t *)codes)[pos];
}

static int shape_ok(int64_t d_out, int64_t d_in, int g, int M, int B)
{
    if (d_out < 0 || d_in < 0 || g <= 0 || M <= 0) return 0;
    if (B != 8 && B != 16) return 0;
    if (d_in % g) return 0;
    return 1;
}

/* ---- exported oracle functions ----------------------------------------- */

/* Unpacked codeword indices, idx[(i*G + j)*M + m] = index of codebook m for
 * group j of row i (G = d_in/g).  Storing an index of B bits per codebook per
 * group is the MCQ section's code representation. */
int aqlm_oracle_decode_indices(const void *codes, int64_t d_out, int64_t d_in,
                               int g, int M, int B, uint16_t *idx)
{
    if (!shape_ok(d_out, d_in, g, M, B)) return 1;
    int64_t groups = d_in / g;
    for (int64_t i = 0; i < d_out; ++i)
        for (int64_t j = 0; j < groups; ++j)
            for (int m = 0; m < M; ++m)
                idx[(i * groups + j) * M + m] =
                    (uint16_t)code_at(codes, i, j, m, groups, M, B);
    return 0;
}

/* Dense dequantised weight, in double:
 *   W[i][g*j + t] = s_i * sum_{m<M} C_m[b(i,j,m)][t].
 * codebooks: binary16 bits [M][2^B][g]; scales: binary16 bits [d_out]. */
int aqlm_oracle_dequant_f64(const void *codes, const uint16_t *codebooks,
                            const uint16_t *scales, int64_t d_out, int64_t d_in,
                            int g, int M, int B, double *W)
{
    if (!shape_ok(d_out, d_in, g, M, B)) return 1;
    int64_t groups = d_in / g;
    int64_t K = (int64_t)1 << B;
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < d_out; ++i) {
        double s = half_bits_to_double(scales[i]);
        for (int64_t j = 0; j < groups; ++j) {
            for (int t = 0; t < g; ++t) {
                double sum = 0.0;
                for (int m = 0; m < M; ++m) {
                    uint32_t k = code_at(codes, i, j, m, groups, M, B);
                    sum += half_bits_to_double(codebooks[((int64_t)m * K + k) * g + t]);
                }
                W[i * d_in + j * g + t] = s * sum;
            }
        }
    }
    return 0;
}

/* Activations of T tokens, [T][d_in], as 16-bit patterns: is_bf16 = 0 for
 * binary16, 1 for bfloat16.  Converted to double exactly. */
static double act_value(const uint16_t *x, int64_t pos, int is_bf16)
{
    return is_bf16 ? (double)bf16_bits_to_float(x[pos]) : half_bits_to_double(x[pos]);
}

/* The layer product, following the MCQ section's inference description step
 * by step for every row i: take each group's M codes, fetch the codewords,
 * sum them, scale the sum by s_i, and accumulate its dot product with the
 * matching g inputs of every token.  All in double.
 *   y[tau][i] = sum_j < s_i * sum_m C_m[b(i,j,m)], x[tau][g*j : g*j+g] >   */
int aqlm_oracle_gemv_f64(const void *codes, const uint16_t *codebooks,
                         const uint16_t *scales, const uint16_t *x, int is_bf16,
                         int64_t tokens, int64_t d_out, int64_t d_in, int g,
                         int M, int B, double *y)
{
    if (!shape_ok(d_out, d_in, g, M, B) || tokens < 0 || g > 64) return 1;
    int64_t groups = d_in / g;
    int64_t K = (int64_t)1 << B;
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < d_out; ++i) {
        double s = half_bits_to_double(scales[i]);
        for (int64_t tau = 0; tau < tokens; ++tau) {
            double acc = 0.0;
            for (int64_t j = 0; j < groups; ++j) {
                double w[64];
                for (int t = 0; t < g; ++t) w[t] = 0.0;
                for (int m = 0; m < M; ++m) {
                    uint32_t k = code_at(codes, i, j, m, groups, M, B);
                    const uint16_t *cw = codebooks + ((int64_t)m * K + k) * g;
                    for (int t = 0; t < g; ++t) w[t] += half_bits_to_double(cw[t]);
                }
                for (int t = 0; t < g; ++t) {
                    acc += (s * w[t]) * act_value(x, tau * d_in + j * g + t, is_bf16);
                }
            }
            y[tau * d_out + i] = acc;
        }
    }
    return 0;
}

/* Plain double matmul Y[tau][i] = sum_k W[i][k] * X[tau][k] (W.X convention of
 * the MCQ section's note: rows of W are output channels). */
int aqlm_oracle_matmul_f64(const double *W, int64_t d_out, int64_t d_in,
                           const double *X, int64_t tokens, double *Y)
{
    if (d_out < 0 || d_in < 0 || tokens < 0) return 1;
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < d_out; ++i) {
        for (int64_t tau = 0; tau < tokens; ++tau) {
            double acc = 0.0;
            for (int64_t k = 0; k < d_in; ++k) acc += W[i * d_in + k] * X[tau * d_in + k];
            Y[tau * d_out + i] = acc;
        }
    }
    return 0;
}

/* Dequantisation to bfloat16 restated as separate IEEE binary32 steps, one
 * rounding each, no fused multiply-add:
 *   f = C_0[b0][t];  f = f + C_m[b_m][t] for m = 1..M-1;  w = f * s_i;
 *   W[i][g*j+t] = bf16_rne(w).
 * binary16 -> binary32 is exact.  The `volatile` stores keep the compiler from
 * contracting or reassociating the two operations. */
int aqlm_oracle_dequant_bf16(const void *codes, const uint16_t *codebooks,
                             const uint16_t *scales, int64_t d_out, int64_t d_in,
                             int g, int M, int B, uint16_t *Wbf16)
{
    if (!shape_ok(d_out, d_in, g, M, B)) return 1;
    int64_t groups = d_in / g;
    int64_t K = (int64_t)1 << B;
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < d_out; ++i) {
        float s = (float)half_bits_to_double(scales[i]);
        for (int64_t j = 0; j < groups; ++j) {
            for (int t = 0; t < g; ++t) {
                volatile float f = (float)half_bits_to_double(
                    codebooks[((int64_t)0 * K + code_at(codes, i, j, 0, groups, M, B)) * g + t]);
                for (int m = 1; m < M; ++m) {
                    uint32_t k = code_at(codes, i, j, m, groups, M, B);
                    float c = (float)half_bits_to_double(codebooks[((int64_t)m * K + k) * g + t]);
                    f = f + c;
                }
                volatile float w = f * s;
                Wbf16[i * d_in + j * g + t] = float_to_bf16_bits_rne(w);
            }
        }
    }
    return 0;
}

/* Average bits per parameter of one layer, the sum of the three storage terms
 * listed in "Memory footprint of AQLM-quantized models", divided by the
 * d_out*d_in parameters:
 *   codebooks  M * 2^B * g * 16 bits
 *   scales     d_out * 16 bits
 *   codes      (d_out * d_in / g) * M * B bits                              */
double aqlm_oracle_bits_per_param(int64_t d_out, int64_t d_in, int g, int M, int B)
{
    double codebook_bits = (double)M * ldexp(1.0, B) * g * 16.0;
    double scale_bits = (double)d_out * 16.0;
    double code_bits = ((double)d_out * (double)d_in / g) * M * B;
    return (codebook_bits + scale_bits + code_bits) / ((double)d_out * (double)d_in);
}

/* Exposed so that the tests can pin the number-format helpers on their own. */
double aqlm_oracle_half_to_double(uint16_t h) { return half_bits_to_double(h); }
uint16_t aqlm_oracle_float_to_bf16(float f) { return float_to_bf16_bits_rne(f); }

int aqlm_oracle_num_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
