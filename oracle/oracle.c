/*
 * oracle.c -- plain fp64 CPU reference of the LoRA linear layer.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path may call, link or load
 * this file; it is used by the tests, by the package's smoke check and by the
 * benchmark's CPU-baseline leg.  It shares no code with the CUDA library.
 *
 * Every input arrives exactly as the GPU receives it (bf16 bit patterns; for a frozen
 * weight also the 4-bit blockwise code plus bf16 scales, or 8-bit e4m3 codes plus a
 * bf16 scale per row) and is widened to fp64 without rounding.  Every sum runs in fp64, in increasing index order, with
 * no blocking or reordering beyond what the definition states.
 *
 * Notation (row-major, tokens are rows):
 *   x [M, d_in], W [d_out, d_in] (frozen), A [r, d_in], B [d_out, r], s = alpha / r,
 *   h [M, d_out], dY = dL/dh [M, d_out], dX [M, d_in], dA [r, d_in], dB [d_out, r].
 *
 * The forward is the low-rank update of a frozen weight, h = W x + B (A x)
 * (page "UnSloth加速库集成：编译级优化带来的性能飞跃", section 为什么标准LoRA会慢？),
 * written here for row vectors with the scale s = alpha / r on the update.
 * The backward is the chain rule of that forward for L = sum(dY * h).  The page
 * "ms-swift高效微调组合：LoRA+UnSloth提速实践", section 1.2 (梯度计算绕过Autograd),
 * prints the weight gradients in a shortened form without x or s; the complete
 * chain-rule forms are used here.  The input-gradient keeps the rank-r product in
 * the order A.(B.dY), never forming the d_out x d_in update (page
 * "Unsloth — 微调 2-5x 加速", section 核心要点, 数学化简反向公式).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define Q4_BLOCK 64

static double bf16_to_f64(uint16_t b) {
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

int oracle_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

void oracle_set_threads(int n) {
#ifdef _OPENMP
    if (n > 0) omp_set_num_threads(n);
#else
    (void)n;
#endif
}

/*
 * FP8 E4M3 value of an 8-bit code, as the OCP 8-bit floating point specification
 * defines the format: sign bit, 4 exponent bits with bias 7, 3 mantissa bits; exponent
 * field 0 is subnormal, m/8 * 2^-6; otherwise (1 + m/8) * 2^(e - 7); no infinities,
 * and S.1111.111 is NaN (so the largest value is 1.75 * 2^8 = 448).
 */
static double e4m3_to_f64(uint8_t c) {
    const int e = (c >> 3) & 0xF, m = c & 0x7;
    const double sign = (c & 0x80) ? -1.0 : 1.0;
    if (e == 0xF && m == 0x7) return NAN;
    if (e == 0) return sign * ldexp((double)m, -9);
    return sign * ldexp(1.0 + m / 8.0, e - 7);
}

/*
 * Frozen weight W[n, k] as fp64.  wfmt 0: bf16 [d_out, d_in].  wfmt 1: 4-bit code,
 * w'[n, k] = (q[n, k] - 8) * scale[n, k / 64] / 7 with the stored bf16 scale; two
 * codes per byte along d_in, low nibble = even k (page "Unsloth — 微调 2-5x 加速",
 * section 核心要点: 4-bit weights dequantised inside the matmul; page
 * "ms-swift框架下UnSloth与Liger-Kernel优化实战", section UnSloth：让LoRA真正“低秩”起来:
 * int4 storage restored on the fly).  wfmt 2: 8-bit FP8 E4M3 codes [d_out, d_in], one
 * per byte, with a bf16 scale per row: w'[n, k] = e4m3(q[n, k]) * scale[n] (page
 * "ms-swift高效微调组合：LoRA+UnSloth提速实践", section 3.2: weights stored in FP8,
 * computed in BF16).  wfmt 3: 4-bit codebook code (the BNB-style 4-bit format of page
 * "ms-swift框架下UnSloth与Liger-Kernel优化实战", section UnSloth：让LoRA真正“低秩”起来),
 * codes and scales laid out as wfmt 1, w'[n, k] = codebook[q[n, k]] * scale[n, k / 64]
 * with the 16 codebook values set by oracle_set_codebook (NF4: the NormalFloat values).
 */
static double g_codebook[16];

void oracle_set_codebook(const double *cb) {
    for (int i = 0; i < 16; ++i) g_codebook[i] = cb[i];
}
typedef struct {
    int wfmt;
    const uint16_t *w;
    const uint8_t *q;
    const uint16_t *scale;
    int64_t d_out, d_in;
} wsrc_t;

static void w_row(const wsrc_t *W, int64_t n, double *row) {
    if (W->wfmt == 0) {
        const uint16_t *p = W->w + n * W->d_in;
        for (int64_t k = 0; k < W->d_in; ++k) row[k] = bf16_to_f64(p[k]);
        return;
    }
    if (W->wfmt == 2) {
        const uint8_t *p = W->q + n * W->d_in;
        const double sc = bf16_to_f64(W->scale[n]);
        for (int64_t k = 0; k < W->d_in; ++k) row[k] = e4m3_to_f64(p[k]) * sc;
        return;
    }
    const uint8_t *p = W->q + n * (W->d_in / 2);
    const uint16_t *sc = W->scale + n * (W->d_in / Q4_BLOCK);
    for (int64_t k = 0; k < W->d_in; ++k) {
        uint8_t byte = p[k / 2];
        int code = (k % 2 == 0) ? (byte & 0x0F) : (byte >> 4);
        if (W->wfmt == 3)
            row[k] = g_codebook[code] * bf16_to_f64(sc[k / Q4_BLOCK]);
        else
            row[k] = (double)(code - 8) * bf16_to_f64(sc[k / Q4_BLOCK]) / 7.0;
    }
}

static wsrc_t make_w(int wfmt, const uint16_t *w, const uint8_t *q, const uint16_t *scale,
                     int64_t d_out, int64_t d_in) {
    wsrc_t W = {wfmt, w, q, scale, d_out, d_in};
    return W;
}

/* Dequantised weight as fp64 (wfmt as above); small shapes only. */
void oracle_weight(int wfmt, const uint16_t *w, const uint8_t *q, const uint16_t *scale,
                   int64_t d_out, int64_t d_in, double *out) {
    wsrc_t W = make_w(wfmt, w, q, scale, d_out, d_in);
    for (int64_t n = 0; n < d_out; ++n) w_row(&W, n, out + n * d_in);
}

/* Step 1: xa[m, j] = sum_k x[m, k] * A[j, k]   (the rank-r product A x). */
void oracle_xa(const uint16_t *x, const uint16_t *A, int64_t M, int64_t d_in, int64_t r,
               double *xa) {
#pragma omp parallel for schedule(dynamic, 4)
    for (int64_t m = 0; m < M; ++m) {
        for (int64_t j = 0; j < r; ++j) {
            double acc = 0.0;
            for (int64_t k = 0; k < d_in; ++k)
                acc += bf16_to_f64(x[m * d_in + k]) * bf16_to_f64(A[j * d_in + k]);
            xa[m * r + j] = acc;
        }
    }
}

/*
 * Step 2: h[m, n] = sum_k x[m, k] * W[n, k] + s * sum_j xa[m, j] * B[n, j].
 * rows == NULL computes every row (n_rows must equal M); otherwise only the listed
 * token rows, written densely to h[i, :] for i < n_rows.  xa is the full [M, r]
 * product of step 1.
 */
void oracle_h(const uint16_t *x, int wfmt, const uint16_t *w, const uint8_t *q,
              const uint16_t *scale, const uint16_t *B, const double *xa, double s,
              int64_t M, int64_t d_in, int64_t d_out, int64_t r, const int64_t *rows,
              int64_t n_rows, double *h) {
    wsrc_t W = make_w(wfmt, w, q, scale, d_out, d_in);
    (void)M;
#pragma omp parallel
    {
        double *xrow = (double *)malloc(sizeof(double) * (size_t)d_in);
        double *wrow = (double *)malloc(sizeof(double) * (size_t)d_in);
#pragma omp for schedule(dynamic, 1)
        for (int64_t i = 0; i < n_rows; ++i) {
            int64_t m = rows ? rows[i] : i;
            for (int64_t k = 0; k < d_in; ++k) xrow[k] = bf16_to_f64(x[m * d_in + k]);
            for (int64_t n = 0; n < d_out; ++n) {
                w_row(&W, n, wrow);
                double base = 0.0;
                for (int64_t k = 0; k < d_in; ++k) base += xrow[k] * wrow[k];
                double lora = 0.0;
                for (int64_t j = 0; j < r; ++j) lora += xa[m * r + j] * bf16_to_f64(B[n * r + j]);
                h[i * d_out + n] = base + s * lora;
            }
        }
        free(xrow);
        free(wrow);
    }
}

/* Step 3: g[m, j] = sum_n dY[m, n] * B[n, j]   (B^T applied to the upstream gradient). */
void oracle_g(const uint16_t *dY, const uint16_t *B, int64_t M, int64_t d_out, int64_t r,
              double *g) {
#pragma omp parallel for schedule(dynamic, 4)
    for (int64_t m = 0; m < M; ++m) {
        for (int64_t j = 0; j < r; ++j) {
            double acc = 0.0;
            for (int64_t n = 0; n < d_out; ++n)
                acc += bf16_to_f64(dY[m * d_out + n]) * bf16_to_f64(B[n * r + j]);
            g[m * r + j] = acc;
        }
    }
}

/*
 * Step 4: dX[m, k] = sum_n dY[m, n] * W[n, k] + s * sum_j g[m, j] * A[j, k].
 * Row selection as in oracle_h; g is the full [M, r] product of step 3.
 */
void oracle_dx(const uint16_t *dY, int wfmt, const uint16_t *w, const uint8_t *q,
               const uint16_t *scale, const uint16_t *A, const double *g, double s,
               int64_t M, int64_t d_in, int64_t d_out, int64_t r, const int64_t *rows,
               int64_t n_rows, double *dX) {
    wsrc_t W = make_w(wfmt, w, q, scale, d_out, d_in);
    (void)M;
#pragma omp parallel
    {
        double *wrow = (double *)malloc(sizeof(double) * (size_t)d_in);
        double *base = (double *)malloc(sizeof(double) * (size_t)d_in);
#pragma omp for schedule(dynamic, 1)
        for (int64_t i = 0; i < n_rows; ++i) {
            int64_t m = rows ? rows[i] : i;
            for (int64_t k = 0; k < d_in; ++k) base[k] = 0.0;
            /* each base[k] accumulates over n in increasing order */
            for (int64_t n = 0; n < d_out; ++n) {
                double c = bf16_to_f64(dY[m * d_out + n]);
                w_row(&W, n, wrow);
                for (int64_t k = 0; k < d_in; ++k) base[k] += c * wrow[k];
            }
            for (int64_t k = 0; k < d_in; ++k) {
                double lora = 0.0;
                for (int64_t j = 0; j < r; ++j) lora += g[m * r + j] * bf16_to_f64(A[j * d_in + k]);
                dX[i * d_in + k] = base[k] + s * lora;
            }
        }
        free(wrow);
        free(base);
    }
}

/*
 * Step 5: dB[n, j] = s * sum_m dY[m, n] * xa[m, j]   (sum over every token).
 * The token loop is outermost so dY is read row by row; each dB[n, j] still sums
 * its terms in increasing m, exactly as the definition reads.
 */
void oracle_db(const uint16_t *dY, const double *xa, double s, int64_t M, int64_t d_out,
               int64_t r, double *dB) {
    const int64_t NB = 256;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t n0 = 0; n0 < d_out; n0 += NB) {
        int64_t n1 = n0 + NB < d_out ? n0 + NB : d_out;
        double *acc = (double *)calloc((size_t)((n1 - n0) * r), sizeof(double));
        for (int64_t m = 0; m < M; ++m)
            for (int64_t n = n0; n < n1; ++n) {
                double c = bf16_to_f64(dY[m * d_out + n]);
                for (int64_t j = 0; j < r; ++j) acc[(n - n0) * r + j] += c * xa[m * r + j];
            }
        for (int64_t n = n0; n < n1; ++n)
            for (int64_t j = 0; j < r; ++j) dB[n * r + j] = s * acc[(n - n0) * r + j];
        free(acc);
    }
}

/*
 * Step 6: dA[j, k] = s * sum_m g[m, j] * x[m, k]   (sum over every token).
 * Token loop outermost as in step 5; each dA[j, k] sums in increasing m.
 */
void oracle_da(const uint16_t *x, const double *g, double s, int64_t M, int64_t d_in,
               int64_t r, double *dA) {
    const int64_t KB = 256;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t k0 = 0; k0 < d_in; k0 += KB) {
        int64_t k1 = k0 + KB < d_in ? k0 + KB : d_in;
        double *acc = (double *)calloc((size_t)((k1 - k0) * r), sizeof(double));
        for (int64_t m = 0; m < M; ++m)
            for (int64_t k = k0; k < k1; ++k) {
                double c = bf16_to_f64(x[m * d_in + k]);
                for (int64_t j = 0; j < r; ++j) acc[(k - k0) * r + j] += g[m * r + j] * c;
            }
        for (int64_t k = k0; k < k1; ++k)
            for (int64_t j = 0; j < r; ++j) dA[j * d_in + k] = s * acc[(k - k0) * r + j];
        free(acc);
    }
}
