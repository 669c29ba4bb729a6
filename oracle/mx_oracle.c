/*
 * mx_oracle.c -- plain, slow CPU oracle for MXFP8 quantisation and GEMM.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the
 * bench's CPU-baseline / reference arm may load this library.  The CUDA
 * path never calls it and shares no code, header or table with it.
 *
 * What it computes, and where each step comes from:
 *  - MXFP8 = 8-bit floating-point elements that share one power-of-two
 *    exponent per block of 32 consecutive elements along K
 *    ("PyTorch and Nebius ... DeepSeek-V3 MoE training on B200", glossary
 *    entry on microscaling FP8, and its pointer to the OCP Microscaling
 *    specification).  Elements are E4M3 (bias 7, no infinities, S.1111.111
 *    is NaN, largest finite 448); the shared scale is UE8M0, value
 *    2^(code-127), code 0xFF = NaN.
 *  - Scale choice: X = floor(log2(amax)) - 8 (8 = exponent of the largest
 *    E4M3 power of two, 256), clamped to [-127, 127]; elements are v*2^-X
 *    rounded to nearest-even and saturated to +-448.
 *  - The pipeline "BF16 -> MXFP8 -> grouped GEMM -> BF16" (same page,
 *    diagram description of the MXFP8 flow from router input to all-to-all
 *    combine).  The GEMM here is the exact sum of products of the
 *    dequantised operands, accumulated in double, k ascending.
 *  - Grouped GEMMs in contiguous and masked layouts ("DeepGEMM" summary
 *    page, list of MoE grouped GEMM layouts; the DeepGEMM release page,
 *    section 4 "MoE optimisation").  Both are defined as a dense GEMM per
 *    group.
 *
 * Readings where the pages are silent (each one is listed in the design
 * notes of the repository):
 *  - an all-zero block gets scale code 0x00 (X = -127);
 *  - a block holding any NaN or +-Inf gets scale 0xFF and every element 0x7F;
 *  - a result that rounds to zero keeps the sign of its input (0x80 for -0);
 *  - the scale bytes are stored in 128-row x 4-column tiles of 512 bytes,
 *    byte (r%32)*16 + ((r%128)/32)*4 + (c%4), tiles ordered row-block major.
 *
 * Plain C99 + OpenMP across independent output rows only.  Build:
 *   gcc -O2 -fopenmp -shared -fPIC -o libmx_oracle.so mx_oracle.c -lm
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#include "mx_oracle.h"

#ifdef _OPENMP
#include <omp.h>
#endif

/* ---------------------------------------------------------------- E4M3 */

/* Value of one E4M3 code, by the format's definition: sign s, 4 exponent
 * bits e (bias 7), 3 mantissa bits m.  e == 0 is subnormal (m/8 * 2^-6);
 * S.1111.111 is NaN; there is no infinity. */
double mxo_e4m3_decode(uint8_t code)
{
    int s = (code >> 7) & 1;
    int e = (code >> 3) & 0xF;
    int m = code & 0x7;
    double mag;
    if (e == 15 && m == 7)
        return NAN;
    if (e == 0)
        mag = ldexp((double)m / 8.0, -6);
    else
        mag = ldexp(1.0 + (double)m / 8.0, e - 7);
    return s ? -mag : mag;
}

void mxo_e4m3_table(double out[256])
{
    for (int c = 0; c < 256; ++c)
        out[c] = mxo_e4m3_decode((uint8_t)c);
}

/* Encode an already-scaled value v' as E4M3, round to nearest with ties to
 * the even code, saturating: |v'| >= 448 gives +-448.  The search runs over
 * the 127 finite non-negative codes 0x00..0x7E, whose values increase
 * strictly with the code, so "even code" is "even mantissa LSB". */
static double e4m3_mag[127]; /* values of codes 0x00..0x7E, filled at load */

__attribute__((constructor)) static void fill_e4m3_mag(void)
{
    for (int c = 0; c < 127; ++c)
        e4m3_mag[c] = mxo_e4m3_decode((uint8_t)c);
}

uint8_t mxo_e4m3_encode(double v)
{
    const double *mag = e4m3_mag;
    if (isnan(v))
        return 0x7F;
    uint8_t sign = signbit(v) ? 0x80 : 0x00;
    double a = fabs(v);
    if (a >= 448.0)
        return sign | 0x7E;
    /* largest lo with mag[lo] <= a (binary search; mag[0] = 0 <= a) */
    int lo = 0, hi = 126;
    while (lo < hi) {
        int mid = (lo + hi + 1) / 2;
        if (mag[mid] <= a)
            lo = mid;
        else
            hi = mid - 1;
    }
    int code;
    if (mag[lo] == a) {
        code = lo;
    } else {
        /* a lies strictly between mag[lo] and mag[lo+1] (a < 448 = mag[126]) */
        double dlo = a - mag[lo];
        double dhi = mag[lo + 1] - a;
        if (dlo < dhi)
            code = lo;
        else if (dhi < dlo)
            code = lo + 1;
        else
            code = (lo % 2 == 0) ? lo : lo + 1;
    }
    return sign | (uint8_t)code;
}

/* ---------------------------------------------------------------- UE8M0 */

double mxo_ue8m0_decode(uint8_t code)
{
    if (code == 0xFF)
        return NAN;
    return ldexp(1.0, (int)code - 127);
}

/* floor(log2(a)) for finite a > 0, from the C library's exact frexp:
 * a = f * 2^e with f in [0.5, 1), so floor(log2 a) = e - 1. */
int mxo_floor_log2(double a)
{
    int e;
    (void)frexp(a, &e);
    return e - 1;
}

/* ---------------------------------------------------------------- BF16 */

double mxo_bf16_to_double(uint16_t bits)
{
    uint32_t u = (uint32_t)bits << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* ------------------------------------------------------- block quantiser */

/* Quantise one block of 32 values (each exactly representable in double):
 * scale selection, then each element scaled by 2^-X (exact in double) and
 * encoded. */
static void quantize_values(const double *v, uint8_t *q, uint8_t *scale)
{
    double amax = 0.0;
    int nonfinite = 0;
    for (int i = 0; i < 32; ++i) {
        if (!isfinite(v[i]))
            nonfinite = 1;
        else if (fabs(v[i]) > amax)
            amax = fabs(v[i]);
    }
    if (nonfinite) {
        *scale = 0xFF;
        for (int i = 0; i < 32; ++i)
            q[i] = 0x7F;
        return;
    }
    int X;
    if (amax == 0.0)
        X = -127;
    else
        X = mxo_floor_log2(amax) - 8;
    if (X < -127)
        X = -127;
    if (X > 127)
        X = 127;
    *scale = (uint8_t)(X + 127);
    for (int i = 0; i < 32; ++i)
        q[i] = mxo_e4m3_encode(ldexp(v[i], -X));
}

/* Quantise one block of 32 BF16 values. */
void mxo_quantize_block(const uint16_t *x, uint8_t *q, uint8_t *scale)
{
    double v[32];
    for (int i = 0; i < 32; ++i)
        v[i] = mxo_bf16_to_double(x[i]);
    quantize_values(v, q, scale);
}

/* Quantise one block of 32 FP32 values (the same scale and rounding rule;
 * FP32 is the precision of a GEMM epilogue that requantises its result). */
void mxo_quantize_block_f32(const float *x, uint8_t *q, uint8_t *scale)
{
    double v[32];
    for (int i = 0; i < 32; ++i)
        v[i] = (double)x[i];
    quantize_values(v, q, scale);
}

/* Quantise a row-major [rows, k] BF16 matrix (k % 32 == 0) along k.
 * q is [rows, k] bytes; sf is the PLAIN row-major [rows, k/32] scale matrix. */
void mxo_quantize(const uint16_t *x, int64_t rows, int64_t k, uint8_t *q, uint8_t *sf)
{
    int64_t kb = k / 32;
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < rows; ++r)
        for (int64_t c = 0; c < kb; ++c)
            mxo_quantize_block(x + r * k + c * 32, q + r * k + c * 32, sf + r * kb + c);
}

/* Quantise a row-major [rows, k] FP32 matrix (k % 32 == 0) along k; q and
 * the plain row-major sf as in mxo_quantize. */
void mxo_quantize_f32(const float *x, int64_t rows, int64_t k, uint8_t *q, uint8_t *sf)
{
    int64_t kb = k / 32;
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < rows; ++r)
        for (int64_t c = 0; c < kb; ++c)
            mxo_quantize_block_f32(x + r * k + c * 32, q + r * k + c * 32, sf + r * kb + c);
}

/* ------------------------------------------------------ SwiGLU */

/* SiLU (the "swish" gate of SwiGLU): x * sigmoid(x) = x / (1 + e^-x). */
double mxo_silu(double x)
{
    return x / (1.0 + exp(-x));
}

/* h = silu(g) * u elementwise over n values (the expert activation between
 * the gate/up and the down GEMM of a DeepSeek-V3 MoE expert). */
void mxo_swiglu(const double *g, const double *u, int64_t n, double *h)
{
    for (int64_t i = 0; i < n; ++i)
        h[i] = mxo_silu(g[i]) * u[i];
}

/* ------------------------------------------------------ scale tile layout */

int64_t mxo_scale_bytes(int64_t rows, int64_t k)
{
    int64_t kb = k / 32;
    int64_t rpad = (rows + 127) / 128 * 128;
    int64_t kbpad = (kb + 3) / 4 * 4;
    return rpad * kbpad;
}

/* Byte offset of scale (r, c) -- row r, K-block c -- in the tiled layout. */
int64_t mxo_sf_offset(int64_t r, int64_t c, int64_t k)
{
    int64_t kb = k / 32;
    int64_t kbpad = (kb + 3) / 4 * 4;
    int64_t tile = (r / 128) * (kbpad / 4) + c / 4;
    return tile * 512 + (r % 32) * 16 + ((r % 128) / 32) * 4 + (c % 4);
}

void mxo_sf_tile(const uint8_t *sf_rm, int64_t rows, int64_t k, uint8_t *tiled)
{
    int64_t kb = k / 32;
    memset(tiled, 0, (size_t)mxo_scale_bytes(rows, k));
    for (int64_t r = 0; r < rows; ++r)
        for (int64_t c = 0; c < kb; ++c)
            tiled[mxo_sf_offset(r, c, k)] = sf_rm[r * kb + c];
}

void mxo_sf_untile(const uint8_t *tiled, int64_t rows, int64_t k, uint8_t *sf_rm)
{
    int64_t kb = k / 32;
    for (int64_t r = 0; r < rows; ++r)
        for (int64_t c = 0; c < kb; ++c)
            sf_rm[r * kb + c] = tiled[mxo_sf_offset(r, c, k)];
}

/* ------------------------------------------------------------------ GEMM */

/* Value tables: the 256 E4M3 codes and the 256 UE8M0 codes (2^(c-127),
 * 0xFF = NaN).  A dequantised element is tab[q] * stab[sf]. */
struct mxo_tables {
    double tab[256];
    double stab[256];
};

static void fill_tables(struct mxo_tables *t)
{
    mxo_e4m3_table(t->tab);
    for (int c = 0; c < 256; ++c)
        t->stab[c] = mxo_ue8m0_decode((uint8_t)c);
}

/* One output row: d[j] = sum_k deq(a[i,k]) * deq(b[j,k]) for j < n, k
 * ascending, in double; abssum[j] = sum_k |deq(a) * deq(b)|. */
static void gemm_row(const struct mxo_tables *t, const uint8_t *qa_row, const uint8_t *sfa_row,
                     const uint8_t *qb, const uint8_t *sfb, int64_t n, int64_t k,
                     double *d_row, double *abs_row)
{
    int64_t kb = k / 32;
    for (int64_t j = 0; j < n; ++j) {
        const uint8_t *qb_row = qb + j * k;
        const uint8_t *sfb_row = sfb + j * kb;
        double acc = 0.0, aacc = 0.0;
        for (int64_t kk = 0; kk < k; ++kk) {
            double a = t->tab[qa_row[kk]] * t->stab[sfa_row[kk / 32]];
            double b = t->tab[qb_row[kk]] * t->stab[sfb_row[kk / 32]];
            double p = a * b;
            acc += p;
            aacc += fabs(p);
        }
        d_row[j] = acc;
        if (abs_row)
            abs_row[j] = aacc;
    }
}

/* D = A * B^T for the listed rows of A (all rows when row_ids is NULL).
 * qa [m, k], sfa row-major [m, k/32], qb [n, k], sfb row-major [n, k/32].
 * d and abssum are [nrows, n] (row t holds A-row row_ids[t]). */
void mxo_gemm(const uint8_t *qa, const uint8_t *sfa, const uint8_t *qb, const uint8_t *sfb,
              int64_t m, int64_t n, int64_t k, const int64_t *row_ids, int64_t nrows,
              double *d, double *abssum)
{
    struct mxo_tables t;
    fill_tables(&t);
    int64_t kb = k / 32;
    if (!row_ids)
        nrows = m;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t r = 0; r < nrows; ++r) {
        int64_t i = row_ids ? row_ids[r] : r;
        gemm_row(&t, qa + i * k, sfa + i * kb, qb, sfb, n, k, d + r * n,
                 abssum ? abssum + r * n : NULL);
    }
}

/* Contiguous grouped GEMM: rows [off[e], off[e+1]) of A use expert e's B.
 * qb is [groups, n, k], sfb row-major [groups, n, k/32].  Only listed rows
 * (or all rows 0..nrows-1 when row_ids is NULL) are computed; a row outside
 * every group gives NaN (such rows are never written on the device). */
void mxo_grouped_contiguous(const uint8_t *qa, const uint8_t *sfa, const uint8_t *qb,
                            const uint8_t *sfb, const int32_t *offsets, int32_t groups,
                            int64_t n, int64_t k, const int64_t *row_ids, int64_t nrows,
                            double *d, double *abssum)
{
    struct mxo_tables t;
    fill_tables(&t);
    int64_t kb = k / 32;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t r = 0; r < nrows; ++r) {
        int64_t i = row_ids ? row_ids[r] : r;
        int e = -1;
        for (int g = 0; g < groups; ++g)
            if (i >= offsets[g] && i < offsets[g + 1])
                e = g;
        if (e < 0) {
            for (int64_t j = 0; j < n; ++j) {
                d[r * n + j] = NAN;
                if (abssum)
                    abssum[r * n + j] = NAN;
            }
            continue;
        }
        gemm_row(&t, qa + i * k, sfa + i * kb, qb + (int64_t)e * n * k, sfb + (int64_t)e * n * kb, n, k,
                 d + r * n, abssum ? abssum + r * n : NULL);
    }
}

/* Masked grouped GEMM: A is [groups, max_m, k]; for expert e only rows
 * r < masked_m[e] are products (d[e, r, :] = A[e, r, :] * B[e]^T).  Rows are
 * addressed by flat index e*max_m + r: the listed ones, or all of them when
 * row_ids is NULL (nrows = groups*max_m).  Rows at or beyond masked_m[e] give
 * NaN here; on the device they must stay untouched. */
void mxo_grouped_masked(const uint8_t *qa, const uint8_t *sfa, const uint8_t *qb,
                        const uint8_t *sfb, const int32_t *masked_m, int32_t groups,
                        int64_t max_m, int64_t n, int64_t k, const int64_t *row_ids,
                        int64_t nrows, double *d, double *abssum)
{
    struct mxo_tables t;
    fill_tables(&t);
    int64_t kb = k / 32;
    if (!row_ids)
        nrows = (int64_t)groups * max_m;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t r = 0; r < nrows; ++r) {
        int64_t flat = row_ids ? row_ids[r] : r;
        int64_t e = flat / max_m, i = flat % max_m;
        if (i >= masked_m[e]) {
            for (int64_t j = 0; j < n; ++j) {
                d[r * n + j] = NAN;
                if (abssum)
                    abssum[r * n + j] = NAN;
            }
            continue;
        }
        gemm_row(&t, qa + flat * k, sfa + flat * kb, qb + e * n * k, sfb + e * n * kb, n, k,
                 d + r * n, abssum ? abssum + r * n : NULL);
    }
}

/* K-grouped GEMM (the weight gradient of an MoE expert layer: the
 * reduction runs over tokens, and each expert owns a range of them).  For
 * expert e and k ranging over [off[e], off[e+1]):
 *   d[e, i, j] = sum_k deq(a[i, k]) * deq(b[j, k]),  k ascending, in double.
 * qa [m, k_total], qb [n, k_total], scales row-major [., k_total/32]
 * (blocks of 32 along the token dimension).  An expert with no tokens gives
 * zeros.  Only the listed flat indices e*m + i are computed when row_ids is
 * given; d and abssum are [nrows, n]. */
void mxo_grouped_kgrouped(const uint8_t *qa, const uint8_t *sfa, const uint8_t *qb,
                          const uint8_t *sfb, const int32_t *offsets, int32_t groups,
                          int64_t m, int64_t n, int64_t k_total, const int64_t *row_ids,
                          int64_t nrows, double *d, double *abssum)
{
    struct mxo_tables t;
    fill_tables(&t);
    int64_t kb = k_total / 32;
    if (!row_ids)
        nrows = (int64_t)groups * m;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t r = 0; r < nrows; ++r) {
        int64_t flat = row_ids ? row_ids[r] : r;
        int64_t e = flat / m, i = flat % m;
        const uint8_t *qa_row = qa + i * k_total;
        const uint8_t *sfa_row = sfa + i * kb;
        for (int64_t j = 0; j < n; ++j) {
            const uint8_t *qb_row = qb + j * k_total;
            const uint8_t *sfb_row = sfb + j * kb;
            double acc = 0.0, aacc = 0.0;
            for (int64_t kk = offsets[e]; kk < offsets[e + 1]; ++kk) {
                double a = t.tab[qa_row[kk]] * t.stab[sfa_row[kk / 32]];
                double b = t.tab[qb_row[kk]] * t.stab[sfb_row[kk / 32]];
                double p = a * b;
                acc += p;
                aacc += fabs(p);
            }
            d[r * n + j] = acc;
            if (abssum)
                abssum[r * n + j] = aacc;
        }
    }
}

/* ------------------------------------------------- tile-wise FP32-scaled FP8 */

/* The FP8 format with fine-grained FP32 scales that DeepGEMM's GEMMs take
 * (the pages: "tile-wise" scaling of the FP8 mixed-precision recipe, and
 * DeepGEMM's FP32 two-level accumulation).  One FP32 scale per tile of
 * elements: s = amax / 448 in FP32 (448 = largest E4M3 value), each element
 * x / s in FP32 (IEEE division, round to nearest) encoded as E4M3 with
 * round-to-nearest-even and saturation.  An all-zero tile gets s = 1; a tile
 * holding NaN or +-Inf gets s = NaN and every element 0x7F.  FP32 arithmetic
 * is done in float on purpose: the device quantiser computes the same
 * correctly rounded FP32 quotients. */
static void tw_quantize_tile(const uint16_t *x, int64_t stride, int rows, int cols, uint8_t *q,
                             int64_t qstride, float *scale)
{
    float amax = 0.0f;
    int nonfinite = 0;
    for (int r = 0; r < rows; ++r)
        for (int c = 0; c < cols; ++c) {
            float v = (float)mxo_bf16_to_double(x[r * stride + c]);
            if (!isfinite(v))
                nonfinite = 1;
            else if (fabsf(v) > amax)
                amax = fabsf(v);
        }
    if (nonfinite) {
        *scale = NAN;
        for (int r = 0; r < rows; ++r)
            for (int c = 0; c < cols; ++c)
                q[r * qstride + c] = 0x7F;
        return;
    }
    volatile float s = amax == 0.0f ? 1.0f : amax / 448.0f;
    *scale = s;
    for (int r = 0; r < rows; ++r)
        for (int c = 0; c < cols; ++c) {
            volatile float v = (float)mxo_bf16_to_double(x[r * stride + c]) / s;
            q[r * qstride + c] = mxo_e4m3_encode((double)v);
        }
}

/* Activations: one scale per row and 128-element K tile ("1 x 128").
 * x [rows, k] BF16, k % 128 == 0; q [rows, k]; s [k/128, rows] (K-tile major). */
void mxo_tw_quantize_rows(const uint16_t *x, int64_t rows, int64_t k, uint8_t *q, float *s)
{
    int64_t kt = k / 128;
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < rows; ++r)
        for (int64_t t = 0; t < kt; ++t)
            tw_quantize_tile(x + r * k + t * 128, k, 1, 128, q + r * k + t * 128, k, s + t * rows + r);
}

/* Weights: one scale per 128 x 128 block ("128 x 128"; a last block of
 * fewer than 128 rows covers what there is).  x [rows, k] BF16, k % 128 == 0;
 * q [rows, k]; s [ceil(rows/128), k/128]. */
void mxo_tw_quantize_blocks(const uint16_t *x, int64_t rows, int64_t k, uint8_t *q, float *s)
{
    int64_t kt = k / 128, rb = (rows + 127) / 128;
#pragma omp parallel for schedule(static)
    for (int64_t b = 0; b < rb; ++b) {
        int nr = (int)(rows - b * 128 < 128 ? rows - b * 128 : 128);
        for (int64_t t = 0; t < kt; ++t)
            tw_quantize_tile(x + b * 128 * k + t * 128, k, nr, 128, q + b * 128 * k + t * 128, k,
                             s + b * kt + t);
    }
}

/* D = deq(A) * deq(B)^T in double, k ascending, for the listed rows (all when
 * row_ids is NULL): deq(a[i, kk]) = e4m3(qa[i, kk]) * sa[kk/128, i],
 * deq(b[j, kk]) = e4m3(qb[j, kk]) * sb[j/128, kk/128].  d, abssum [nrows, n]. */
void mxo_tw_gemm(const uint8_t *qa, const float *sa, const uint8_t *qb, const float *sb, int64_t m,
                 int64_t n, int64_t k, const int64_t *row_ids, int64_t nrows, double *d,
                 double *abssum)
{
    double tab[256];
    mxo_e4m3_table(tab);
    int64_t kt = k / 128;
    if (!row_ids)
        nrows = m;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t r = 0; r < nrows; ++r) {
        int64_t i = row_ids ? row_ids[r] : r;
        for (int64_t j = 0; j < n; ++j) {
            double acc = 0.0, aacc = 0.0;
            for (int64_t kk = 0; kk < k; ++kk) {
                double a = tab[qa[i * k + kk]] * (double)sa[(kk / 128) * m + i];
                double b = tab[qb[j * k + kk]] * (double)sb[(j / 128) * kt + kk / 128];
                double p = a * b;
                acc += p;
                aacc += fabs(p);
            }
            d[r * n + j] = acc;
            if (abssum)
                abssum[r * n + j] = aacc;
        }
    }
}

/* ------------------------------------------------------------------ MoE expert layer
 *
 * The data movement around the grouped GEMM in a mixture-of-experts layer:
 * the B200 MoE-training page's diagram of the MXFP8 expert layer (router
 * output -> BF16 -> MXFP8 -> grouped GEMM -> BF16 -> all-to-all combine) and
 * its glossary entry on all-to-all (tokens are sent to the experts that
 * process them and the results are gathered back); the DeepGEMM release
 * page, section 4 (the contiguous layout: each expert's tokens grouped, one
 * group after another).  The router itself is not part of the path: ids and
 * gate weights are inputs.
 */

/* Routing plan.  ids [n] holds the expert of each entry (t, j) of a [T, topk]
 * routing table in token-major order (n = T*topk).  Expert e's rows are its
 * entries in that order, starting at offsets[e]; each group is padded to a
 * multiple of `pad` rows: offsets[e+1] = offsets[e] + ceil(counts[e]/pad)*pad.
 * row[i] is the row of entry i, or -1 when ids[i] is outside [0, E) (such an
 * entry is dropped).  Returns the number of dropped entries. */
int64_t mxo_moe_route(const int32_t *ids, int64_t n, int32_t E, int32_t pad, int32_t *counts,
                      int32_t *offsets, int32_t *row)
{
    int64_t bad = 0;
    for (int32_t e = 0; e < E; ++e)
        counts[e] = 0;
    for (int64_t i = 0; i < n; ++i)
        if (ids[i] >= 0 && ids[i] < E)
            counts[ids[i]] += 1;
    offsets[0] = 0;
    for (int32_t e = 0; e < E; ++e)
        offsets[e + 1] = offsets[e] + (counts[e] + pad - 1) / pad * pad;
    int32_t *next = (int32_t *)malloc(sizeof(int32_t) * (size_t)(E > 0 ? E : 1));
    for (int32_t e = 0; e < E; ++e)
        next[e] = offsets[e];
    for (int64_t i = 0; i < n; ++i) {
        if (ids[i] >= 0 && ids[i] < E) {
            row[i] = next[ids[i]];
            next[ids[i]] += 1;
        } else {
            row[i] = -1;
            ++bad;
        }
    }
    free(next);
    return bad;
}

/* Expert-parallel placement (the B200 MoE-training page, its DeepEP section
 * and glossary entry on all-to-all: each token goes to the rank that holds
 * its expert).  `ranks` ranks each hold E/ranks experts (rank o owns experts
 * [o*E/ranks, (o+1)*E/ranks)) and their own entries: ids holds rank r's n_of[r]
 * entries after those of ranks 0..r-1.  On the owner of expert e, e's rows
 * are its entries of rank 0 in entry order, then those of rank 1, and so on;
 * the owner's experts are placed one after another, each group padded to a
 * multiple of `pad` rows.  Entry i (in ids order) goes to rank dst_rank[i],
 * row dst_row[i]; an id outside [0, E) is dropped (-1, -1).  Owner o's plan:
 * counts_local[o*el + l] entries of its expert l (el = E/ranks) and
 * offsets_local[o*(el+1) + l] its padded group starts, el + 1 values. */
void mxo_moe_peer_plan(const int32_t *ids, const int64_t *n_of, int32_t ranks, int32_t E, int32_t pad,
                       int32_t *dst_rank, int32_t *dst_row, int32_t *counts_local, int32_t *offsets_local)
{
    int32_t el = E / ranks;
    int64_t n = 0;
    for (int32_t r = 0; r < ranks; ++r)
        n += n_of[r];
    int64_t *tot = (int64_t *)calloc((size_t)(E > 0 ? E : 1), sizeof(int64_t));
    int64_t *next = (int64_t *)calloc((size_t)(E > 0 ? E : 1), sizeof(int64_t));
    for (int64_t i = 0; i < n; ++i)
        if (ids[i] >= 0 && ids[i] < E)
            tot[ids[i]] += 1;
    for (int32_t o = 0; o < ranks; ++o) {
        int64_t start = 0;
        for (int32_t l = 0; l < el; ++l) {
            int32_t e = o * el + l;
            next[e] = start;
            counts_local[o * el + l] = (int32_t)tot[e];
            offsets_local[o * (el + 1) + l] = (int32_t)start;
            start += (tot[e] + pad - 1) / pad * pad;
        }
        offsets_local[o * (el + 1) + el] = (int32_t)start;
    }
    for (int64_t i = 0; i < n; ++i) {   /* rank by rank, each rank's entries in order */
        int32_t e = ids[i];
        if (e >= 0 && e < E) {
            dst_rank[i] = e / el;
            dst_row[i] = (int32_t)next[e];
            next[e] += 1;
        } else {
            dst_rank[i] = -1;
            dst_row[i] = -1;
        }
    }
    free(tot);
    free(next);
}

/* Dispatch into the contiguous layout: the E4M3 row and scales of token t
 * (quantised as by mxo_quantize) are written to row[t*topk + j] for every j
 * with row >= 0.  q [m_rows, k] and sf_rm [m_rows, k/32] are first set to
 * zero, so every row no entry maps to (the group padding) is the quantisation
 * of a zero row: E4M3 0x00 elements, scale code 0x00. */
void mxo_moe_dispatch(const uint16_t *x, int64_t T, int64_t k, const int32_t *row, int64_t topk,
                      int64_t m_rows, uint8_t *q, uint8_t *sf_rm)
{
    int64_t kb = k / 32;
    memset(q, 0, (size_t)(m_rows * k));
    memset(sf_rm, 0, (size_t)(m_rows * kb));
    uint8_t *tq = (uint8_t *)malloc((size_t)(k > 0 ? k : 1));
    uint8_t *ts = (uint8_t *)malloc((size_t)(kb > 0 ? kb : 1));
    for (int64_t t = 0; t < T; ++t) {
        mxo_quantize(x + t * k, 1, k, tq, ts);
        for (int64_t j = 0; j < topk; ++j) {
            int32_t r = row[t * topk + j];
            if (r < 0)
                continue;
            memcpy(q + (int64_t)r * k, tq, (size_t)k);
            memcpy(sf_rm + (int64_t)r * kb, ts, (size_t)kb);
        }
    }
    free(tq);
    free(ts);
}

/* Combine: out[t, :] = sum_j w[t, j] * y[row[t*topk + j], :] in fp64, j
 * ascending, over the entries with row >= 0; y holds BF16 bit patterns
 * [*, n].  abssum (optional) = sum_j |w * y|, the scale of the rounding
 * error a reduced-precision sum may make. */
void mxo_moe_combine(const uint16_t *y, int64_t n, const int32_t *row, const float *w, int64_t T,
                     int64_t topk, double *out, double *abssum)
{
#pragma omp parallel for schedule(static)
    for (int64_t t = 0; t < T; ++t) {
        for (int64_t c = 0; c < n; ++c) {
            double acc = 0.0, aacc = 0.0;
            for (int64_t j = 0; j < topk; ++j) {
                int32_t r = row[t * topk + j];
                if (r < 0)
                    continue;
                double p = (double)w[t * topk + j] * mxo_bf16_to_double(y[(int64_t)r * n + c]);
                acc += p;
                aacc += fabs(p);
            }
            out[t * n + c] = acc;
            if (abssum)
                abssum[t * n + c] = aacc;
        }
    }
}

int mxo_num_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
