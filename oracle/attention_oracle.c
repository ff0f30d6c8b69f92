/*
 * attention_oracle.c -- the fp64 CPU oracle for non-causal multi-head attention.
 *
 * TEST INFRASTRUCTURE, NOT PRODUCT CODE.  Only the test suite, the smoke check
 * and the CPU-baseline leg of the benchmark may load this library.  The CUDA
 * path never links, includes or calls anything here, and nothing here knows
 * about the CUDA path: the two share no code, tables or headers.
 *
 * What it computes (plain definition, no blocking, no fusion):
 *   for every batch b and head h, with Q_bh[i,:] = q[b,i,h,:] (likewise K, V),
 *     s_ij   = scale * sum_d Q[i,d] * K[j,d]
 *     p_ij   = exp(s_ij - max_j s_ij) / sum_j exp(s_ij - max_j s_ij)
 *     O[i,:] = sum_j p_ij * V[j,:]
 *   written back token-major as out[b,i,h,:].
 * Sources:
 *   - "hf2q -- src/inference/vision/vit_gpu.rs", doc of `vit_attention_gpu`
 *     ("Full GPU scaled-dot-product attention for ViT"): inputs are seq-major
 *     [batch, num_heads, head_dim], output has the same shape, no mask because
 *     a ViT is bidirectional; softmax of the scaled scores times V.
 *   - same page, doc of `vit_attention_scores_gpu`: scores = (Q K^T) * scale
 *     per head, the scale is the caller's and is applied as given (no implicit
 *     1/sqrt(head_dim)).
 *   - same page, `vit_softmax_last_dim_gpu`: numerically stable row softmax,
 *     i.e. the row maximum is subtracted before exponentiating.
 *   - "inferencelayer 0.2.1 -- src/vision_gpu.rs", `vis_attn_coop_src` doc
 *     ("Shape"): one head's queries are rows of the token-major [rows, nh*hd]
 *     activation, element (r, h, d) at r*nh*hd + h*hd + d.
 * Inputs are the bf16 / f16 bit patterns that the GPU path also receives; they
 * are widened exactly to double here (bf16 and f16 are subsets of double).
 *
 * Every floating-point step is in double (mode 0 and 1) or long double
 * (mode 2).  Mode 1 (log-sum-exp normalisation) and mode 2 (no max shift,
 * long double) are alternative formulations of the same definition, kept as
 * an internal cross-check on tiny inputs; mode 0 is the oracle proper.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ORACLE_BF16 0
#define ORACLE_F16 1
#define ORACLE_F64 2

/* bf16 is the upper half of an IEEE binary32: shift it back into place. */
static double widen_bf16(uint16_t bits) {
    uint32_t u = (uint32_t)bits << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* IEEE binary16: 1 sign bit, 5 exponent bits (bias 15), 10 mantissa bits. */
static double widen_f16(uint16_t bits) {
    int sign = (bits >> 15) & 1;
    int e = (bits >> 10) & 0x1f;
    int m = bits & 0x3ff;
    double mag;
    if (e == 0) {
        mag = ldexp((double)m, -24); /* subnormal: m * 2^-14 * 2^-10 */
    } else if (e == 31) {
        mag = m ? NAN : INFINITY;
    } else {
        mag = ldexp((double)(1024 + m), e - 25); /* (1 + m/1024) * 2^(e-15) */
    }
    return sign ? -mag : mag;
}

static double fetch(const void* src, int64_t idx, int dtype) {
    if (dtype == ORACLE_F64) return ((const double*)src)[idx];
    uint16_t b = ((const uint16_t*)src)[idx];
    return dtype == ORACLE_BF16 ? widen_bf16(b) : widen_f16(b);
}

int oracle_widen(const uint16_t* bits, int64_t n, int dtype, double* out) {
    if (!bits || !out || n < 0) return -1;
    if (dtype != ORACLE_BF16 && dtype != ORACLE_F16) return -4;
    for (int64_t i = 0; i < n; ++i)
        out[i] = dtype == ORACLE_BF16 ? widen_bf16(bits[i]) : widen_f16(bits[i]);
    return 0;
}

/* Offset of element (b, i, h, d) in a dense token-major [B, N, H, D] tensor. */
static int64_t at(int64_t b, int64_t i, int64_t h, int64_t d, int64_t N, int64_t H, int64_t D) {
    return ((b * N + i) * H + h) * D + d;
}

/* One output row: the three lines of the definition above, in order. */
static void attend_row(const double* qrow, const double* Kbh, const double* Vbh, int64_t N,
                       int64_t D, double scale, int mode, double* s, double* orow) {
    for (int64_t j = 0; j < N; ++j) {
        double dot = 0.0;
        for (int64_t d = 0; d < D; ++d) dot += qrow[d] * Kbh[j * D + d];
        s[j] = scale * dot;
    }
    for (int64_t d = 0; d < D; ++d) orow[d] = 0.0;
    if (mode == 2) {
        /* brute force: exp without the max shift, long double sums */
        long double z = 0.0L;
        for (int64_t j = 0; j < N; ++j) z += expl((long double)s[j]);
        for (int64_t d = 0; d < D; ++d) {
            long double acc = 0.0L;
            for (int64_t j = 0; j < N; ++j) acc += expl((long double)s[j]) / z * Vbh[j * D + d];
            orow[d] = (double)acc;
        }
        return;
    }
    double m = -INFINITY;
    for (int64_t j = 0; j < N; ++j)
        if (s[j] > m) m = s[j];
    double z = 0.0;
    for (int64_t j = 0; j < N; ++j) z += exp(s[j] - m);
    if (mode == 1) {
        double lse = m + log(z); /* log sum_j exp(s_j) */
        for (int64_t j = 0; j < N; ++j) {
            double p = exp(s[j] - lse);
            for (int64_t d = 0; d < D; ++d) orow[d] += p * Vbh[j * D + d];
        }
    } else {
        for (int64_t j = 0; j < N; ++j) {
            double p = exp(s[j] - m) / z;
            for (int64_t d = 0; d < D; ++d) orow[d] += p * Vbh[j * D + d];
        }
    }
}

static int check_dims(int64_t B, int64_t N, int64_t H, int64_t D) {
    if (B <= 0 || N <= 0 || H <= 0 || D <= 0) return -2;
    if (N > (int64_t)1 << 26 || D > 4096) return -2;
    return 0;
}

/*
 * Attention for a list of output rows.  rows[r] is the flat token-head index
 * (b*N + i)*H + h of the r-th requested row; out is nrows x D doubles.
 * dtype: 0 = bf16 bits, 1 = f16 bits, 2 = double.  mode: see the file header.
 * Rows may come in any order; each (b, h) slice is widened once.
 */
int oracle_attention_rows(const void* q, const void* k, const void* v, int64_t B, int64_t N,
                          int64_t H, int64_t D, double scale, int dtype, int mode,
                          const int64_t* rows, int64_t nrows, double* out) {
    if (!q || !k || !v || !out || (nrows > 0 && !rows)) return -1;
    int rc = check_dims(B, N, H, D);
    if (rc) return rc;
    if (dtype < 0 || dtype > 2) return -4;
    if (mode < 0 || mode > 2) return -4;
    for (int64_t r = 0; r < nrows; ++r)
        if (rows[r] < 0 || rows[r] >= B * N * H) return -2;
    if (nrows == 0) return 0;

    /* bucket the requested rows by (b, h) */
    int64_t nbh = B * H;
    int64_t* count = (int64_t*)calloc((size_t)nbh + 1, sizeof(int64_t));
    int64_t* order = (int64_t*)malloc((size_t)nrows * sizeof(int64_t));
    double* Kbh = (double*)malloc((size_t)(N * D) * sizeof(double));
    double* Vbh = (double*)malloc((size_t)(N * D) * sizeof(double));
    if (!count || !order || !Kbh || !Vbh) {
        free(count); free(order); free(Kbh); free(Vbh);
        return -10;
    }
    for (int64_t r = 0; r < nrows; ++r) {
        int64_t tok = rows[r] / H, h = rows[r] % H, b = tok / N;
        count[b * H + h + 1]++;
    }
    for (int64_t g = 0; g < nbh; ++g) count[g + 1] += count[g];
    {
        int64_t* fill = (int64_t*)malloc((size_t)nbh * sizeof(int64_t));
        if (!fill) {
            free(count); free(order); free(Kbh); free(Vbh);
            return -10;
        }
        memcpy(fill, count, (size_t)nbh * sizeof(int64_t));
        for (int64_t r = 0; r < nrows; ++r) {
            int64_t tok = rows[r] / H, h = rows[r] % H, b = tok / N;
            order[fill[b * H + h]++] = r;
        }
        free(fill);
    }

    int failed = 0;
    for (int64_t g = 0; g < nbh && !failed; ++g) {
        int64_t lo = count[g], hi = count[g + 1];
        if (lo == hi) continue;
        int64_t b = g / H, h = g % H;
#pragma omp parallel for schedule(static)
        for (int64_t j = 0; j < N; ++j)
            for (int64_t d = 0; d < D; ++d) {
                Kbh[j * D + d] = fetch(k, at(b, j, h, d, N, H, D), dtype);
                Vbh[j * D + d] = fetch(v, at(b, j, h, d, N, H, D), dtype);
            }
#pragma omp parallel
        {
            double* s = (double*)malloc((size_t)N * sizeof(double));
            double* qrow = (double*)malloc((size_t)D * sizeof(double));
            if (!s || !qrow) {
#pragma omp atomic write
                failed = 1;
            }
#pragma omp for schedule(dynamic, 4)
            for (int64_t t = lo; t < hi; ++t) {
                if (!s || !qrow) continue;
                int64_t r = order[t];
                int64_t i = (rows[r] / H) % N;
                for (int64_t d = 0; d < D; ++d) qrow[d] = fetch(q, at(b, i, h, d, N, H, D), dtype);
                attend_row(qrow, Kbh, Vbh, N, D, scale, mode, s, out + r * D);
            }
            free(s);
            free(qrow);
        }
    }
    free(count); free(order); free(Kbh); free(Vbh);
    return failed ? -10 : 0;
}

/* The whole output, token-major [B, N, H, D] doubles. */
int oracle_attention(const void* q, const void* k, const void* v, int64_t B, int64_t N, int64_t H,
                     int64_t D, double scale, int dtype, int mode, double* out) {
    int rc = check_dims(B, N, H, D);
    if (rc) return rc;
    int64_t nrows = B * N * H;
    int64_t* rows = (int64_t*)malloc((size_t)nrows * sizeof(int64_t));
    if (!rows) return -10;
    for (int64_t r = 0; r < nrows; ++r) rows[r] = r; /* row r of out is token-head r */
    rc = oracle_attention_rows(q, k, v, B, N, H, D, scale, dtype, mode, rows, nrows, out);
    free(rows);
    return rc;
}

/*
 * The N x N probability matrix p_ij of one (b, h) slice, row-major, from the
 * same definition (mode 0 normalisation).  Used to check that rows sum to 1.
 */
int oracle_attention_probs(const void* q, const void* k, int64_t B, int64_t N, int64_t H,
                           int64_t D, double scale, int dtype, int64_t b, int64_t h, double* P) {
    if (!q || !k || !P) return -1;
    int rc = check_dims(B, N, H, D);
    if (rc) return rc;
    if (b < 0 || b >= B || h < 0 || h >= H) return -2;
    if (dtype < 0 || dtype > 2) return -4;
    for (int64_t i = 0; i < N; ++i) {
        double* s = P + i * N;
        for (int64_t j = 0; j < N; ++j) {
            double dot = 0.0;
            for (int64_t d = 0; d < D; ++d)
                dot += fetch(q, at(b, i, h, d, N, H, D), dtype) * fetch(k, at(b, j, h, d, N, H, D), dtype);
            s[j] = scale * dot;
        }
        double m = -INFINITY, z = 0.0;
        for (int64_t j = 0; j < N; ++j)
            if (s[j] > m) m = s[j];
        for (int64_t j = 0; j < N; ++j) z += exp(s[j] - m);
        for (int64_t j = 0; j < N; ++j) s[j] = exp(s[j] - m) / z;
    }
    return 0;
}

int oracle_num_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
