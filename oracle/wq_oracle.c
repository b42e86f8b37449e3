/*
 * wq_oracle.c -- plain, slow CPU reference for the weight-only quantized
 * linear layer y = x . dequant(Wq)^T.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product library calls, links or
 * loads this file.  Only the tests, the package's smoke() check and the
 * benchmark's CPU-baseline leg use it.  It shares no code, header, table or
 * constant with the CUDA path.
 *
 * What it computes (restated from the pages, see the citation on each
 * function):
 *   - W8A16: int8 weight q[n][k] with one bf16 scale s[n] per output channel
 *     ("Per-channel W8A16 quantization", tileInfer README, Features table);
 *     w[n][k] = s[n] * q[n][k].
 *   - W4A16: unsigned 4-bit weight q[n][k] in [0,15] with a bf16 scale and a
 *     4-bit zero point per (group of 128 along K, output column) (the
 *     scale / zero-point / group-size triple named in "Toward a Cleaner
 *     Quantization Stack in SGLang", review of Figure 4);
 *     w[n][k] = s[n][g] * (q[n][k] - z[n][g]),  g = floor(k / G).
 *   - y[m][n] = sum_k x[m][k] * w[n][k], evaluated in fp64 with k ascending
 *     (the dense "linear" that the GEMV and the GEMM of the tileInfer README,
 *     Features table, both compute).
 *
 * Every fp operation is IEEE binary64 with round-to-nearest-even; the file
 * must be compiled without fast-math and with -ffp-contract=off so that no
 * fused multiply-add changes a rounding.  Each dot product is one sequential
 * loop, so the result does not depend on the number of OpenMP threads.
 *
 * Packed-word conventions of the canonical (unpacked-layout) inputs:
 *   - INT4 weights: uint32 words [N][K/8]; nibble j (bits 4j..4j+3) of word
 *     (n, c) is q[n][8c + j]  (low nibble first).
 *   - INT4 zero points: uint32 words [N][ceil((K/G)/8)]; nibble j of word
 *     (n, c) is z[n][8c + j], the zero of group 8c + j.
 *   - INT4 scales: bf16 [N][K/G].   INT8: q int8 [N][K], scales bf16 [N].
 *   - G (INT4) is the group: 32, 64, 128, or K for one scale and zero point
 *     per output channel ("per-channel and groups 32/64/128" in the
 *     validation matrix of the Marlin register and launch scheduling
 *     benchmark, "Validation and limits").
 *   - Activations x are bf16, or IEEE binary16 in the *_fmt entry points.
 *
 * Parity pins: every function here is pinned by the tests in
 * tests/test_oracle_pins.py against closed forms, brute force in exact
 * rational arithmetic, library routines (torch's fp32->bf16 conversion,
 * numpy's fp64 matmul) and invariants.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

double wqo_f16_to_f64(uint16_t h);
void wqo_linear_int8_fmt(const uint16_t *x, int fmt, int64_t M, int64_t K, const int8_t *q, const uint16_t *s,
                         int64_t N, const int64_t *rows, int64_t n_rows, double *y);
void wqo_linear_int4_fmt(const uint16_t *x, int fmt, int64_t M, int64_t K, const uint32_t *q_words,
                         const uint16_t *s, const uint32_t *z_words, int64_t G, int64_t N, const int64_t *rows,
                         int64_t n_rows, double *y);

/* ------------------------------------------------------------------ */
/* bf16 <-> binary64                                                   */
/* ------------------------------------------------------------------ */

/* A bf16 value is the upper 16 bits of an IEEE binary32 value, so the
 * conversion to binary64 is exact. */
double wqo_bf16_to_f64(uint16_t b)
{
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

static uint16_t upper_half_of_f32(float f)
{
    uint32_t u;
    memcpy(&u, &f, sizeof u);
    return (uint16_t)(u >> 16);
}

/* Round a binary64 value to bf16 (8 significant bits, exponent range of
 * binary32, subnormal quantum 2^-133).
 *   mode 0: round to nearest, ties to even
 *   mode 1: round toward +infinity
 * Written from the IEEE-754 definition: find the quantum of the binade that
 * holds |v|, scale |v| to an integer count of quanta (exact: a power-of-two
 * scaling), round that count, scale back. */
static uint16_t round_to_bf16(double v, int mode)
{
    if (isnan(v))
        return 0x7FC0;
    const int neg = signbit(v) ? 1 : 0;
    if (isinf(v))
        return neg ? 0xFF80 : 0x7F80;
    if (v == 0.0)
        return neg ? 0x8000 : 0x0000;

    const double a = fabs(v);
    int e;
    (void)frexp(a, &e); /* a in [2^(e-1), 2^e) */
    const int qexp = (e - 1 >= -126) ? (e - 1 - 7) : -133;
    const double count = ldexp(a, -qexp); /* exact */
    double r;
    if (mode == 0)
        r = nearbyint(count); /* default rounding mode: ties to even */
    else
        r = neg ? floor(count) : ceil(count); /* toward +inf on v */

    double res = ldexp(r, qexp);
    if (res >= 0x1p128) { /* beyond the largest finite bf16 */
        if (mode == 1 && neg)
            return 0xFF7F; /* toward +inf never reaches -inf */
        return neg ? 0xFF80 : 0x7F80;
    }
    /* res has at most 8 significant bits inside the binary32 range, so the
     * conversion to float is exact. */
    uint16_t h = upper_half_of_f32((float)res);
    if (neg)
        h |= 0x8000;
    return h;
}

uint16_t wqo_f64_to_bf16_rne(double v) { return round_to_bf16(v, 0); }
uint16_t wqo_f64_to_bf16_up(double v) { return round_to_bf16(v, 1); }

/* Array forms, used by the tests. */
void wqo_bf16_round_array(const double *v, int64_t n, int mode, uint16_t *out)
{
    for (int64_t i = 0; i < n; ++i)
        out[i] = round_to_bf16(v[i], mode);
}

/* ------------------------------------------------------------------ */
/* IEEE binary16 (fp16) <-> binary64: the FP16 activations of the      */
/* validation matrix (Marlin register and launch scheduling benchmark,  */
/* "Validation and limits").                                            */
/* ------------------------------------------------------------------ */

/* binary16: sign, 5 exponent bits (bias 15), 10 fraction bits.  Normal:
 * (1024 + f) 2^(e - 25); subnormal (e = 0): f 2^-24; e = 31: inf / NaN.
 * Exact in binary64. */
double wqo_f16_to_f64(uint16_t h)
{
    const int sign = h >> 15, e = (h >> 10) & 0x1F, f = h & 0x3FF;
    double v;
    if (e == 0)
        v = ldexp((double)f, -24);
    else if (e == 31)
        v = f ? NAN : INFINITY;
    else
        v = ldexp((double)(1024 + f), e - 25);
    return sign ? -v : v;
}

/* binary64 -> binary16, round to nearest, ties to even: the quantum of the
 * binade of |v| (11 significant bits; 2^-24 below the smallest normal
 * 2^-14), the exact count of quanta rounded, overflow to infinity at
 * 65520 = 65504 + half a quantum. */
uint16_t wqo_f64_to_f16_rne(double v)
{
    const int neg = signbit(v) ? 1 : 0;
    const double a = fabs(v);
    if (a == 0.0)
        return neg ? 0x8000 : 0;
    int e2;
    frexp(a, &e2); /* a = m 2^e2, m in [0.5, 1): binade 2^(e2 - 1) */
    const int qe = (e2 - 1 >= -14) ? (e2 - 1) - 10 : -24;
    const double r = nearbyint(ldexp(a, -qe)); /* default rounding: to nearest even */
    const double res = ldexp(r, qe);
    if (res >= 65520.0 || res > 65504.0)
        return (uint16_t)(neg ? 0xFC00 : 0x7C00);
    uint16_t out;
    if (res < ldexp(1.0, -14)) {
        out = (uint16_t)r; /* subnormal (or the smallest normal when r = 1024) */
    } else {
        int e3;
        const double m = frexp(res, &e3); /* res = m 2^e3 */
        const int biased = (e3 - 1) + 15;
        const int frac = (int)(ldexp(m, 11) - 1024.0);
        out = (uint16_t)((biased << 10) | frac);
    }
    return (uint16_t)(out | (neg ? 0x8000 : 0));
}

void wqo_f16_to_f64_array(const uint16_t *h, int64_t n, double *out)
{
    for (int64_t i = 0; i < n; ++i)
        out[i] = wqo_f16_to_f64(h[i]);
}

void wqo_f16_round_array(const double *v, int64_t n, uint16_t *out)
{
    for (int64_t i = 0; i < n; ++i)
        out[i] = wqo_f64_to_f16_rne(v[i]);
}

void wqo_bf16_to_f64_array(const uint16_t *b, int64_t n, double *out)
{
    for (int64_t i = 0; i < n; ++i)
        out[i] = wqo_bf16_to_f64(b[i]);
}

/* ------------------------------------------------------------------ */
/* Threads                                                             */
/* ------------------------------------------------------------------ */

void wqo_set_threads(int n)
{
#ifdef _OPENMP
    if (n > 0)
        omp_set_num_threads(n);
#else
    (void)n;
#endif
}

int wqo_get_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* ------------------------------------------------------------------ */
/* Unpack                                                              */
/* ------------------------------------------------------------------ */

/* INT4: nibble j of word i becomes element 8i + j, as an integer 0..15. */
void wqo_unpack_int4(const uint32_t *words, int64_t n_words, uint8_t *q_out)
{
    for (int64_t i = 0; i < n_words; ++i)
        for (int j = 0; j < 8; ++j)
            q_out[8 * i + j] = (uint8_t)((words[i] >> (4 * j)) & 0xFu);
}

/* INT8: a byte is a two's-complement integer -128..127. */
void wqo_unpack_int8(const uint8_t *bytes, int64_t n, int32_t *q_out)
{
    for (int64_t i = 0; i < n; ++i)
        q_out[i] = (int32_t)(int8_t)bytes[i];
}

/* ------------------------------------------------------------------ */
/* Dequantize one output row to binary64                               */
/* ------------------------------------------------------------------ */

/* W8A16 per output channel: w[k] = s * q[k].  The product of an 8-bit
 * scale significand and a 7-bit integer is exact in binary64. */
static void dequant_row_int8(const int8_t *q_row, uint16_t s_bf16, int64_t K, double *w)
{
    const double s = wqo_bf16_to_f64(s_bf16);
    for (int64_t k = 0; k < K; ++k)
        w[k] = s * (double)q_row[k];
}

/* W4A16, group G along K: w[k] = s[g] * (q[k] - z[g]), g = k / G.
 * Unpacks the row's weight nibbles and zero nibbles first. */
static void dequant_row_int4(const uint32_t *q_words_row, const uint16_t *s_row,
                             const uint32_t *z_words_row, int64_t K, int64_t G, double *w)
{
    const int64_t n_groups = K / G;
    for (int64_t k = 0; k < K; ++k) {
        const int64_t g = k / G;
        const uint32_t q = (q_words_row[k / 8] >> (4 * (k % 8))) & 0xFu;
        const uint32_t z = (z_words_row[g / 8] >> (4 * (g % 8))) & 0xFu;
        const double s = wqo_bf16_to_f64(s_row[g]);
        w[k] = s * ((double)q - (double)z);
    }
    (void)n_groups;
}

static int64_t zero_words_per_row(int64_t K, int64_t G) { return (K / G + 7) / 8; }

/* Dequantize selected rows (rows == NULL: all N rows in order) into
 * out[i][K] for the i-th selected row. */
void wqo_dequant_int8(const int8_t *q, const uint16_t *s, int64_t K, int64_t N,
                      const int64_t *rows, int64_t n_rows, double *out)
{
    if (!rows)
        n_rows = N;
#pragma omp parallel for schedule(dynamic, 16)
    for (int64_t i = 0; i < n_rows; ++i) {
        const int64_t n = rows ? rows[i] : i;
        dequant_row_int8(q + n * K, s[n], K, out + i * K);
    }
}

void wqo_dequant_int4(const uint32_t *q_words, const uint16_t *s, const uint32_t *z_words,
                      int64_t K, int64_t N, int64_t G, const int64_t *rows, int64_t n_rows,
                      double *out)
{
    if (!rows)
        n_rows = N;
    const int64_t zw = zero_words_per_row(K, G);
#pragma omp parallel for schedule(dynamic, 16)
    for (int64_t i = 0; i < n_rows; ++i) {
        const int64_t n = rows ? rows[i] : i;
        dequant_row_int4(q_words + n * (K / 8), s + n * (K / G), z_words + n * zw, K, G,
                         out + i * K);
    }
}

/* ------------------------------------------------------------------ */
/* Linear: unpack, dequantize to binary64, then the plain dot products */
/* ------------------------------------------------------------------ */

/* x: bf16 [M][K].  y: binary64 [M][n_rows], column i is output channel
 * rows[i] (rows == NULL: all N channels, n_rows = N). */
static void linear_rows(const double *xd, int64_t M, int64_t K, int64_t n_rows, double *y,
                        void (*row_fn)(const void *ctx, int64_t i, double *w), const void *ctx)
{
#pragma omp parallel
    {
        double *w = (double *)malloc((size_t)K * sizeof(double));
#pragma omp for schedule(dynamic, 8)
        for (int64_t i = 0; i < n_rows; ++i) {
            row_fn(ctx, i, w);
            for (int64_t m = 0; m < M; ++m) {
                const double *xr = xd + m * K;
                double acc = 0.0;
                for (int64_t k = 0; k < K; ++k)
                    acc += xr[k] * w[k];
                y[m * n_rows + i] = acc;
            }
        }
        free(w);
    }
}

/* x as binary64: bf16 (fmt 0) or IEEE binary16 (fmt 1) bit patterns. */
static double *act_matrix_to_f64(const uint16_t *x, int64_t n, int fmt)
{
    double *xd = (double *)malloc((size_t)(n > 0 ? n : 1) * sizeof(double));
    for (int64_t i = 0; i < n; ++i)
        xd[i] = fmt ? wqo_f16_to_f64(x[i]) : wqo_bf16_to_f64(x[i]);
    return xd;
}

struct int8_ctx {
    const int8_t *q;
    const uint16_t *s;
    int64_t K;
    const int64_t *rows;
};

static void int8_row(const void *vctx, int64_t i, double *w)
{
    const struct int8_ctx *c = (const struct int8_ctx *)vctx;
    const int64_t n = c->rows ? c->rows[i] : i;
    dequant_row_int8(c->q + n * c->K, c->s[n], c->K, w);
}

struct int4_ctx {
    const uint32_t *q_words;
    const uint16_t *s;
    const uint32_t *z_words;
    int64_t K, G;
    const int64_t *rows;
};

static void int4_row(const void *vctx, int64_t i, double *w)
{
    const struct int4_ctx *c = (const struct int4_ctx *)vctx;
    const int64_t n = c->rows ? c->rows[i] : i;
    const int64_t zw = zero_words_per_row(c->K, c->G);
    dequant_row_int4(c->q_words + n * (c->K / 8), c->s + n * (c->K / c->G),
                     c->z_words + n * zw, c->K, c->G, w);
}

void wqo_linear_int8(const uint16_t *x, int64_t M, int64_t K, const int8_t *q,
                     const uint16_t *s, int64_t N, const int64_t *rows, int64_t n_rows,
                     double *y)
{
    wqo_linear_int8_fmt(x, 0, M, K, q, s, N, rows, n_rows, y);
}

/* As wqo_linear_int8, x in activation format fmt (0 bf16, 1 fp16). */
void wqo_linear_int8_fmt(const uint16_t *x, int fmt, int64_t M, int64_t K, const int8_t *q,
                         const uint16_t *s, int64_t N, const int64_t *rows, int64_t n_rows,
                         double *y)
{
    if (!rows)
        n_rows = N;
    double *xd = act_matrix_to_f64(x, M * K, fmt);
    struct int8_ctx ctx = {q, s, K, rows};
    linear_rows(xd, M, K, n_rows, y, int8_row, &ctx);
    free(xd);
}

void wqo_linear_int4(const uint16_t *x, int64_t M, int64_t K, const uint32_t *q_words,
                     const uint16_t *s, const uint32_t *z_words, int64_t G, int64_t N,
                     const int64_t *rows, int64_t n_rows, double *y)
{
    wqo_linear_int4_fmt(x, 0, M, K, q_words, s, z_words, G, N, rows, n_rows, y);
}

/* As wqo_linear_int4, x in activation format fmt (0 bf16, 1 fp16). */
void wqo_linear_int4_fmt(const uint16_t *x, int fmt, int64_t M, int64_t K, const uint32_t *q_words,
                         const uint16_t *s, const uint32_t *z_words, int64_t G, int64_t N,
                         const int64_t *rows, int64_t n_rows, double *y)
{
    if (!rows)
        n_rows = N;
    double *xd = act_matrix_to_f64(x, M * K, fmt);
    struct int4_ctx ctx = {q_words, s, z_words, K, G, rows};
    linear_rows(xd, M, K, n_rows, y, int4_row, &ctx);
    free(xd);
}

/* ------------------------------------------------------------------ */
/* Quantizers (how the synthetic weights of the workloads are made)    */
/* ------------------------------------------------------------------ */

/* Symmetric per-output-channel INT8 ("Per-channel W8A16 quantization",
 * tileInfer README, Features table).  For row n:
 *   s = bf16_rne(max_k |W[n][k]| / 127)     (binary64 division)
 *   q = clamp(rint(W / s), -127, 127)        (binary64 division, ties to even)
 * A row whose scale is zero gets q = 0. */
void wqo_quant_int8(const float *W, int64_t K, int64_t N, int8_t *q, uint16_t *s)
{
#pragma omp parallel for schedule(dynamic, 16)
    for (int64_t n = 0; n < N; ++n) {
        const float *wr = W + n * K;
        double amax = 0.0;
        for (int64_t k = 0; k < K; ++k) {
            const double a = fabs((double)wr[k]);
            if (a > amax)
                amax = a;
        }
        const uint16_t sb = wqo_f64_to_bf16_rne(amax / 127.0);
        s[n] = sb;
        const double sd = wqo_bf16_to_f64(sb);
        for (int64_t k = 0; k < K; ++k) {
            double v = 0.0;
            if (sd != 0.0) {
                v = nearbyint((double)wr[k] / sd);
                if (v > 127.0)
                    v = 127.0;
                if (v < -127.0)
                    v = -127.0;
            }
            q[n * K + k] = (int8_t)v;
        }
    }
}

/* Asymmetric INT4 with group G along K, a bf16 scale and a 4-bit zero point
 * per (output channel, group).  For group (n, g):
 *   lo = min(min W, 0), hi = max(max W, 0)
 *   s  = bf16 rounded toward +inf of (hi - lo) / 15   (binary64 arithmetic)
 *   z  = clamp(rint(-lo / s), 0, 15)
 *   q  = clamp(rint(W / s) + z, 0, 15)
 * A group with hi == lo (all zero) gets s = 0, z = 0, q = 0.
 * Outputs use the canonical packed-word conventions in the file header;
 * z_words must be zero-initialised by the caller for unused nibbles. */
void wqo_quant_int4(const float *W, int64_t K, int64_t N, int64_t G, uint32_t *q_words,
                    uint16_t *s, uint32_t *z_words)
{
    const int64_t n_groups = K / G;
    const int64_t zw = zero_words_per_row(K, G);
#pragma omp parallel for schedule(dynamic, 16)
    for (int64_t n = 0; n < N; ++n) {
        const float *wr = W + n * K;
        for (int64_t c = 0; c < zw; ++c)
            z_words[n * zw + c] = 0u;
        for (int64_t c = 0; c < K / 8; ++c)
            q_words[n * (K / 8) + c] = 0u;
        for (int64_t g = 0; g < n_groups; ++g) {
            double lo = 0.0, hi = 0.0;
            for (int64_t k = g * G; k < (g + 1) * G; ++k) {
                const double v = (double)wr[k];
                if (v < lo)
                    lo = v;
                if (v > hi)
                    hi = v;
            }
            uint16_t sb = 0;
            uint32_t z = 0;
            double sd = 0.0;
            if (hi - lo > 0.0) {
                sb = wqo_f64_to_bf16_up((hi - lo) / 15.0);
                sd = wqo_bf16_to_f64(sb);
                double zf = nearbyint(-lo / sd);
                if (zf < 0.0)
                    zf = 0.0;
                if (zf > 15.0)
                    zf = 15.0;
                z = (uint32_t)zf;
            }
            s[n * n_groups + g] = sb;
            z_words[n * zw + g / 8] |= z << (4 * (g % 8));
            for (int64_t k = g * G; k < (g + 1) * G; ++k) {
                uint32_t qv = 0;
                if (sd != 0.0) {
                    double v = nearbyint((double)wr[k] / sd) + (double)z;
                    if (v < 0.0)
                        v = 0.0;
                    if (v > 15.0)
                        v = 15.0;
                    qv = (uint32_t)v;
                }
                q_words[n * (K / 8) + k / 8] |= qv << (4 * (k % 8));
            }
        }
    }
}
