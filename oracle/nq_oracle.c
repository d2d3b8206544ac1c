/*
 * nq_oracle.c -- plain, slow, single-threaded CPU oracle for the low-rank binary (LRB)
 * matmul of NanoQuant.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path may call, link or load this
 * file: only the tests, the package smoke check and the CPU-baseline leg of bench.py use
 * it.  It shares no code, header, table or helper with the CUDA library.
 *
 * What it computes, and where each piece comes from
 * (page "NanoQuant: Efficient Sub-1-Bit Quantization of Large Language Models",
 *  research.samsung.com blog, unless stated otherwise):
 *
 *   - Section 2, "Low-Rank Binary Factorization", first display equation:
 *         W ~= s1 (.) (U V^T) (.) s2^T,   U in {-1,+1}^{d_out x r},  V in {-1,+1}^{d_in x r},
 *         s1 in R^{d_out},  s2 in R^{d_in}.
 *     Read elementwise: W_ij = s1_i * (sum_k U_ik V_jk) * s2_j.  The oracle materialises
 *     W in fp64 and returns y[b][i] = sum_j W_ij x[b][j], plus
 *     S[b][i] = sum_j |W_ij x[b][j]| (the magnitude of the terms of that sum).
 *   - Same section, the sentence after the equation: the representation holds
 *     r (d_out + d_in) binary values plus (d_out + d_in) floating-point values.
 *   - Section 3, "Step 3: Factorized Component Refinement", objective: binary factors are
 *     sign(U), sign(V) of latent real matrices.  sign(0) is not stated; the reading taken
 *     is +1 iff latent >= 0 (so +0, -0 -> +1; NaN -> -1).
 *   - Section 3, "Phase 3: Scale-Only Model Reconstruction": frozen binary factors are
 *     "packed into efficient integer formats"; no layout is given.  The reading taken:
 *     32 signs per uint32 along r, element k of a row in word k/32 at bit k%32
 *     (least significant bit first), bit = 1 for +1.  Words of a row beyond r/32 (row
 *     padding up to the leading dimension) are written as 0 and never read as data.
 *
 * Precision: fp16 scales and bf16 activations convert exactly to fp64; the integer Gram
 * entry G_ij = sum_k U_ik V_jk is exact; W_ij = s1_i G_ij s2_j needs 11+11+13 significant
 * bits and each product W_ij x_j another 8, all below fp64's 53, so only the final sums
 * round.  The oracle is therefore the exact result up to one fp64 summation.
 *
 * Two evaluation orders are provided on purpose:
 *   nq_oracle_dense_*     materialise W (the definition);
 *   nq_oracle_factored_*  y = s1 (.) (U (V^T (s2 (.) x))) in fp64 (the same product, with
 *                         the associativity the factorisation exists for).
 * Tests pin each against closed forms, invariants, brute force and integer matmul.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORACLE_API __attribute__((visibility("default")))

/* ---------------------------------------------------------------------------------
 * Number formats, written from the IEEE 754 binary16 definition and from bfloat16 being
 * the upper half of an IEEE binary32.
 * --------------------------------------------------------------------------------- */

/* binary16: 1 sign bit, 5 exponent bits (bias 15), 10 fraction bits. */
ORACLE_API double nq_oracle_f16_to_double(uint16_t h) {
    int sign = (h >> 15) & 1;
    int e = (h >> 10) & 0x1F;
    int f = h & 0x3FF;
    double v;
    if (e == 0) {
        v = ldexp((double)f, -24); /* subnormal: f * 2^-24 */
    } else if (e == 31) {
        v = (f == 0) ? INFINITY : NAN;
    } else {
        v = ldexp((double)(1024 + f), e - 25); /* (1 + f/1024) * 2^(e-15) */
    }
    return sign ? -v : v;
}

/* bfloat16: the 16 most significant bits of an IEEE binary32. */
ORACLE_API double nq_oracle_bf16_to_double(uint16_t b) {
    uint32_t u = ((uint32_t)b) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* fp64 -> bfloat16, round to nearest, ties to even, directly from the real value (no
 * intermediate binary32 rounding).  bfloat16 keeps 8 significant bits; its smallest normal
 * is 2^-126 and its quantum below that is 2^-133. */
/* fp64 -> IEEE binary16 (1 sign, 5 exponent bits with bias 15, 10 fraction bits), round to
 * nearest, ties to even: keep 11 significant bits (quantum 2^(e-11) for a in [2^(e-1), 2^e)),
 * never finer than the subnormal quantum 2^-24; results of 65536 and above overflow to inf. */
ORACLE_API uint16_t nq_oracle_double_to_f16(double v) {
    if (isnan(v)) return 0x7E00;
    uint16_t sign = signbit(v) ? 0x8000 : 0;
    double a = fabs(v);
    if (isinf(a)) return sign | 0x7C00;
    if (a == 0.0) return sign;
    int e;
    frexp(a, &e); /* a = m * 2^e, 0.5 <= m < 1 */
    int qexp = e - 11;
    if (qexp < -24) qexp = -24;
    double q = nearbyint(ldexp(a, -qexp)); /* default rounding mode: to nearest, ties even */
    double rv = ldexp(q, qexp);
    if (rv >= 65536.0) return sign | 0x7C00;
    if (rv < ldexp(1.0, -14)) return sign | (uint16_t)ldexp(rv, 24); /* subnormal (1024 -> 0x0400) */
    int e2;
    double m2 = frexp(rv, &e2); /* rv = m2 * 2^e2, 0.5 <= m2 < 1: exponent field e2 - 1 + 15 */
    uint16_t frac = (uint16_t)(ldexp(m2, 11) - 1024.0);
    return sign | (uint16_t)((e2 + 14) << 10) | frac;
}

ORACLE_API uint16_t nq_oracle_double_to_bf16(double v) {
    if (isnan(v)) return 0x7FC0;
    uint16_t sign = signbit(v) ? 0x8000 : 0;
    double a = fabs(v);
    if (isinf(a)) return sign | 0x7F80;
    if (a == 0.0) return sign;
    int e;
    frexp(a, &e); /* a = m * 2^e, 0.5 <= m < 1 */
    int qexp = e - 8;
    if (qexp < -133) qexp = -133;
    double q = nearbyint(ldexp(a, -qexp)); /* default rounding mode: to nearest, ties even */
    double rv = ldexp(q, qexp);
    if (rv >= ldexp(1.0, 128)) return sign | 0x7F80;
    float f = (float)rv; /* exact: rv has at most 8 significant bits and is in range */
    uint32_t u;
    memcpy(&u, &f, sizeof u);
    return sign | (uint16_t)(u >> 16);
}

/* Array forms of the two conversions above. */
ORACLE_API void nq_oracle_f16_array_to_double(const uint16_t* h, int64_t n, double* out) {
    for (int64_t e = 0; e < n; ++e) out[e] = nq_oracle_f16_to_double(h[e]);
}

ORACLE_API void nq_oracle_bf16_array_to_double(const uint16_t* b, int64_t n, double* out) {
    for (int64_t e = 0; e < n; ++e) out[e] = nq_oracle_bf16_to_double(b[e]);
}

/* ---------------------------------------------------------------------------------
 * sign() and packing.
 * --------------------------------------------------------------------------------- */

/* Packs sign(latent) of a [rows][ld_latent] fp32 matrix (first r columns) into
 * [rows][ld_words] uint32 words.  Returns 0, or -1 on bad sizes. */
ORACLE_API int nq_oracle_pack(const float* latent, int64_t rows, int64_t r, int64_t ld_latent,
                              uint32_t* packed, int64_t ld_words) {
    if (rows < 0 || r < 0 || r % 32 != 0 || ld_latent < r || ld_words < r / 32) return -1;
    for (int64_t i = 0; i < rows; ++i) {
        uint32_t* row = packed + i * ld_words;
        for (int64_t w = 0; w < ld_words; ++w) row[w] = 0u;
        for (int64_t k = 0; k < r; ++k) {
            float v = latent[i * ld_latent + k];
            if (v >= 0.0f) row[k / 32] |= 1u << (k % 32);
        }
    }
    return 0;
}

/* Unpacks [rows][ld_words] words to int8 signs [rows][r] (+1 for bit 1, -1 for bit 0). */
ORACLE_API int nq_oracle_unpack(const uint32_t* packed, int64_t rows, int64_t r, int64_t ld_words,
                                int8_t* signs) {
    if (rows < 0 || r < 0 || r % 32 != 0 || ld_words < r / 32) return -1;
    for (int64_t i = 0; i < rows; ++i)
        for (int64_t k = 0; k < r; ++k) {
            uint32_t bit = (packed[i * ld_words + k / 32] >> (k % 32)) & 1u;
            signs[i * r + k] = bit ? (int8_t)1 : (int8_t)-1;
        }
    return 0;
}

/* ---------------------------------------------------------------------------------
 * Gram matrix G = U V^T of the sign factors (exact integers).
 * --------------------------------------------------------------------------------- */

/* Literal triple loop on unpacked signs: G[i][j] = sum_k U[i][k] V[j][k]. */
ORACLE_API void nq_oracle_gram_signs(const int8_t* U, const int8_t* V, int64_t d_out, int64_t d_in,
                                     int64_t r, int32_t* G) {
    for (int64_t i = 0; i < d_out; ++i)
        for (int64_t j = 0; j < d_in; ++j) {
            int32_t acc = 0;
            for (int64_t k = 0; k < r; ++k) acc += (int32_t)U[i * r + k] * (int32_t)V[j * r + k];
            G[i * d_in + j] = acc;
        }
}

/* One Gram entry from packed rows: matching bits contribute +1, differing bits -1, so
 * G_ij = r - 2 * (number of differing bits). */
static int32_t gram_entry_packed(const uint32_t* u_row, const uint32_t* v_row, int64_t r) {
    int64_t differ = 0;
    for (int64_t w = 0; w < r / 32; ++w) differ += __builtin_popcount(u_row[w] ^ v_row[w]);
    return (int32_t)(r - 2 * differ);
}

ORACLE_API void nq_oracle_gram_packed(const uint32_t* U, int64_t ldu, const uint32_t* V, int64_t ldv,
                                      int64_t d_out, int64_t d_in, int64_t r, int32_t* G) {
    for (int64_t i = 0; i < d_out; ++i)
        for (int64_t j = 0; j < d_in; ++j)
            G[i * d_in + j] = gram_entry_packed(U + i * ldu, V + j * ldv, r);
}

/* ---------------------------------------------------------------------------------
 * Forward products.
 * --------------------------------------------------------------------------------- */

/* The definition on unpacked signs and fp64 values:
 *   W_ij = s1_i * G_ij * s2_j,  y[b][i] = sum_j W_ij x[b][j],  S[b][i] = sum_j |W_ij x[b][j]|.
 * U int8 [d_out][r], V int8 [d_in][r], x [B][d_in]; y, S [B][d_out].  S may be NULL. */
ORACLE_API void nq_oracle_dense_signs(const int8_t* U, const int8_t* V, const double* s1,
                                      const double* s2, int64_t d_out, int64_t d_in, int64_t r,
                                      const double* x, int64_t B, double* y, double* S) {
    for (int64_t b = 0; b < B; ++b)
        for (int64_t i = 0; i < d_out; ++i) {
            y[b * d_out + i] = 0.0;
            if (S) S[b * d_out + i] = 0.0;
        }
    for (int64_t i = 0; i < d_out; ++i)
        for (int64_t j = 0; j < d_in; ++j) {
            int64_t g = 0;
            for (int64_t k = 0; k < r; ++k) g += (int64_t)U[i * r + k] * (int64_t)V[j * r + k];
            double w = s1[i] * (double)g * s2[j];
            for (int64_t b = 0; b < B; ++b) {
                double term = w * x[b * d_in + j];
                y[b * d_out + i] += term;
                if (S) S[b * d_out + i] += fabs(term);
            }
        }
}

/* The definition on the packed layout with fp16 scales and bf16 activations given as raw
 * bit patterns, for a chosen subset of output rows (rows == NULL means all d_out rows, in
 * order).  y and S are [B][n_rows]. */
ORACLE_API int nq_oracle_dense_packed(const uint32_t* U, int64_t ldu, const uint32_t* V, int64_t ldv,
                                      const uint16_t* s1_f16, const uint16_t* s2_f16, int64_t d_out,
                                      int64_t d_in, int64_t r, const uint16_t* x_bf16, int64_t B,
                                      const int64_t* rows, int64_t n_rows, double* y, double* S) {
    if (r % 32 != 0 || ldu < r / 32 || ldv < r / 32) return -1;
    if (rows == NULL) n_rows = d_out;
    double* s2 = (double*)malloc(sizeof(double) * (size_t)(d_in > 0 ? d_in : 1));
    double* x = (double*)malloc(sizeof(double) * (size_t)(B * d_in > 0 ? B * d_in : 1));
    if (!s2 || !x) {
        free(s2);
        free(x);
        return -2;
    }
    for (int64_t j = 0; j < d_in; ++j) s2[j] = nq_oracle_f16_to_double(s2_f16[j]);
    for (int64_t e = 0; e < B * d_in; ++e) x[e] = nq_oracle_bf16_to_double(x_bf16[e]);
    for (int64_t n = 0; n < n_rows; ++n) {
        int64_t i = rows ? rows[n] : n;
        if (i < 0 || i >= d_out) {
            free(s2);
            free(x);
            return -1;
        }
        double s1 = nq_oracle_f16_to_double(s1_f16[i]);
        for (int64_t b = 0; b < B; ++b) {
            y[b * n_rows + n] = 0.0;
            if (S) S[b * n_rows + n] = 0.0;
        }
        for (int64_t j = 0; j < d_in; ++j) {
            double w = s1 * (double)gram_entry_packed(U + i * ldu, V + j * ldv, r) * s2[j];
            for (int64_t b = 0; b < B; ++b) {
                double term = w * x[b * d_in + j];
                y[b * n_rows + n] += term;
                if (S) S[b * n_rows + n] += fabs(term);
            }
        }
    }
    free(s2);
    free(x);
    return 0;
}

/* The factored evaluation order, in fp64, on the packed layout:
 *   z[b][j] = s2_j x[b][j];  t[b][k] = sum_j V_jk z[b][j];  y[b][i] = s1_i sum_k U_ik t[b][k].
 * y is [B][d_out]. */
ORACLE_API int nq_oracle_factored_packed(const uint32_t* U, int64_t ldu, const uint32_t* V, int64_t ldv,
                                         const uint16_t* s1_f16, const uint16_t* s2_f16, int64_t d_out,
                                         int64_t d_in, int64_t r, const uint16_t* x_bf16, int64_t B,
                                         double* y) {
    if (r % 32 != 0 || ldu < r / 32 || ldv < r / 32) return -1;
    double* t = (double*)malloc(sizeof(double) * (size_t)(r > 0 ? r : 1));
    if (!t) return -2;
    for (int64_t b = 0; b < B; ++b) {
        for (int64_t k = 0; k < r; ++k) t[k] = 0.0;
        for (int64_t j = 0; j < d_in; ++j) {
            double z = nq_oracle_f16_to_double(s2_f16[j]) * nq_oracle_bf16_to_double(x_bf16[b * d_in + j]);
            const uint32_t* vrow = V + j * ldv;
            for (int64_t k = 0; k < r; ++k) {
                uint32_t bit = (vrow[k / 32] >> (k % 32)) & 1u;
                t[k] += bit ? z : -z;
            }
        }
        for (int64_t i = 0; i < d_out; ++i) {
            const uint32_t* urow = U + i * ldu;
            double acc = 0.0;
            for (int64_t k = 0; k < r; ++k) {
                uint32_t bit = (urow[k / 32] >> (k % 32)) & 1u;
                acc += bit ? t[k] : -t[k];
            }
            y[b * d_out + i] = nq_oracle_f16_to_double(s1_f16[i]) * acc;
        }
    }
    free(t);
    return 0;
}

/* ---------------------------------------------------------------------------------
 * Products through the frozen factors for scale-only calibration (section 3, "Phase 3:
 * Scale-Only Model Reconstruction": U and V stay fixed while s1 and s2 are optimised, so
 * the training step needs the layer's transpose and the derivatives of its output with
 * respect to the two scale vectors).  Both follow from the section 2 equation read
 * elementwise, W_ij = s1_i G_ij s2_j, y[b][i] = sum_j W_ij x[b][j]:
 *
 *   transpose:   xbar[b][j] = sum_i W_ij ybar[b][i]
 *   scale grads: for L = sum_b sum_i ybar[b][i] y[b][i] (ybar the cotangent of y),
 *                dL/ds1_i = sum_b ybar[b][i] sum_j G_ij s2_j x[b][j]
 *                dL/ds2_j = sum_b x[b][j]    sum_i G_ij s1_i ybar[b][i]
 * --------------------------------------------------------------------------------- */

/* The transpose on the packed layout, for a chosen subset of output columns j (cols ==
 * NULL means all d_in, in order).  ybar [B][d_out] bf16 bits; xbar, S [B][n_cols], with
 * S[b][n] = sum_i |W_ij ybar[b][i]|. */
ORACLE_API int nq_oracle_transposed_packed(const uint32_t* U, int64_t ldu, const uint32_t* V, int64_t ldv,
                                           const uint16_t* s1_f16, const uint16_t* s2_f16, int64_t d_out,
                                           int64_t d_in, int64_t r, const uint16_t* ybar_bf16, int64_t B,
                                           const int64_t* cols, int64_t n_cols, double* xbar, double* S) {
    if (r % 32 != 0 || ldu < r / 32 || ldv < r / 32) return -1;
    if (cols == NULL) n_cols = d_in;
    double* s1 = (double*)malloc(sizeof(double) * (size_t)(d_out > 0 ? d_out : 1));
    double* yb = (double*)malloc(sizeof(double) * (size_t)(B * d_out > 0 ? B * d_out : 1));
    if (!s1 || !yb) {
        free(s1);
        free(yb);
        return -2;
    }
    for (int64_t i = 0; i < d_out; ++i) s1[i] = nq_oracle_f16_to_double(s1_f16[i]);
    for (int64_t e = 0; e < B * d_out; ++e) yb[e] = nq_oracle_bf16_to_double(ybar_bf16[e]);
    for (int64_t n = 0; n < n_cols; ++n) {
        int64_t j = cols ? cols[n] : n;
        if (j < 0 || j >= d_in) {
            free(s1);
            free(yb);
            return -1;
        }
        double s2 = nq_oracle_f16_to_double(s2_f16[j]);
        for (int64_t b = 0; b < B; ++b) {
            xbar[b * n_cols + n] = 0.0;
            if (S) S[b * n_cols + n] = 0.0;
        }
        for (int64_t i = 0; i < d_out; ++i) {
            double w = s1[i] * (double)gram_entry_packed(U + i * ldu, V + j * ldv, r) * s2;
            for (int64_t b = 0; b < B; ++b) {
                double term = w * yb[b * d_out + i];
                xbar[b * n_cols + n] += term;
                if (S) S[b * n_cols + n] += fabs(term);
            }
        }
    }
    free(s1);
    free(yb);
    return 0;
}

/* Both scale gradients on the packed layout, with the magnitudes of their terms:
 * g1, S1 [d_out]; g2, S2 [d_in].  x [B][d_in], ybar [B][d_out] bf16 bits. */
ORACLE_API int nq_oracle_scale_grads_packed(const uint32_t* U, int64_t ldu, const uint32_t* V, int64_t ldv,
                                            const uint16_t* s1_f16, const uint16_t* s2_f16, int64_t d_out,
                                            int64_t d_in, int64_t r, const uint16_t* x_bf16,
                                            const uint16_t* ybar_bf16, int64_t B, double* g1, double* S1,
                                            double* g2, double* S2) {
    if (r % 32 != 0 || ldu < r / 32 || ldv < r / 32) return -1;
    double* x = (double*)malloc(sizeof(double) * (size_t)(B * d_in > 0 ? B * d_in : 1));
    double* yb = (double*)malloc(sizeof(double) * (size_t)(B * d_out > 0 ? B * d_out : 1));
    if (!x || !yb) {
        free(x);
        free(yb);
        return -2;
    }
    for (int64_t e = 0; e < B * d_in; ++e) x[e] = nq_oracle_bf16_to_double(x_bf16[e]);
    for (int64_t e = 0; e < B * d_out; ++e) yb[e] = nq_oracle_bf16_to_double(ybar_bf16[e]);
    for (int64_t i = 0; i < d_out; ++i) g1[i] = S1[i] = 0.0;
    for (int64_t j = 0; j < d_in; ++j) g2[j] = S2[j] = 0.0;
    for (int64_t i = 0; i < d_out; ++i) {
        double s1 = nq_oracle_f16_to_double(s1_f16[i]);
        for (int64_t j = 0; j < d_in; ++j) {
            double g = (double)gram_entry_packed(U + i * ldu, V + j * ldv, r);
            double s2 = nq_oracle_f16_to_double(s2_f16[j]);
            for (int64_t b = 0; b < B; ++b) {
                double t1 = yb[b * d_out + i] * g * s2 * x[b * d_in + j];
                double t2 = x[b * d_in + j] * g * s1 * yb[b * d_out + i];
                g1[i] += t1;
                S1[i] += fabs(t1);
                g2[j] += t2;
                S2[j] += fabs(t2);
            }
        }
    }
    free(x);
    free(yb);
    return 0;
}

/* ---------------------------------------------------------------------------------
 * Gradients with respect to the two sign factors (section 3, "Step 3: Factorized Component
 * Refinement": the latent factors are refined through sign() with straight-through
 * estimators).  For L = sum_b sum_i ybar[b][i] y[b][i] the section 2 equation, read
 * elementwise, gives
 *     dL/dU_ik = sum_b sum_j ybar[b][i] s1_i V_jk s2_j x[b][j]
 *     dL/dV_jk = sum_b sum_i x[b][j] s2_j U_ik s1_i ybar[b][i]
 * and the straight-through estimator passes them to the latent entries unchanged (the pages
 * name no variant; the reading taken is the identity estimator).  Every term is an exact
 * fp64 product (8 + 11 + 1 + 11 + 8 significant bits), so only the sums round.
 *
 * Entries (rows_u[a], ks[c]) of dL/dU and (rows_v[a], ks[c]) of dL/dV are evaluated (a NULL
 * list means every row, or every k, in order), with the magnitudes of their terms:
 * gU, SU [n_rows_u][n_ks]; gV, SV [n_rows_v][n_ks].  x [B][d_in], ybar [B][d_out] bf16 bits.
 * --------------------------------------------------------------------------------- */
static int sign_of_packed(const uint32_t* row, int64_t k) { return ((row[k / 32] >> (k % 32)) & 1u) ? 1 : -1; }

ORACLE_API int nq_oracle_sign_grads_packed(const uint32_t* U, int64_t ldu, const uint32_t* V, int64_t ldv,
                                           const uint16_t* s1_f16, const uint16_t* s2_f16, int64_t d_out,
                                           int64_t d_in, int64_t r, const uint16_t* x_bf16,
                                           const uint16_t* ybar_bf16, int64_t B, const int64_t* rows_u,
                                           int64_t n_rows_u, const int64_t* rows_v, int64_t n_rows_v,
                                           const int64_t* ks, int64_t n_ks, double* gU, double* SU, double* gV,
                                           double* SV) {
    if (r % 32 != 0 || ldu < r / 32 || ldv < r / 32) return -1;
    if (rows_u == NULL) n_rows_u = d_out;
    if (rows_v == NULL) n_rows_v = d_in;
    if (ks == NULL) n_ks = r;
    double* x = (double*)malloc(sizeof(double) * (size_t)(B * d_in > 0 ? B * d_in : 1));
    double* yb = (double*)malloc(sizeof(double) * (size_t)(B * d_out > 0 ? B * d_out : 1));
    if (!x || !yb) {
        free(x);
        free(yb);
        return -2;
    }
    for (int64_t e = 0; e < B * d_in; ++e) x[e] = nq_oracle_bf16_to_double(x_bf16[e]);
    for (int64_t e = 0; e < B * d_out; ++e) yb[e] = nq_oracle_bf16_to_double(ybar_bf16[e]);
    int rc = 0;
    for (int64_t a = 0; a < n_rows_u && rc == 0; ++a) {
        const int64_t i = rows_u ? rows_u[a] : a;
        if (i < 0 || i >= d_out) {
            rc = -1;
            break;
        }
        const double s1 = nq_oracle_f16_to_double(s1_f16[i]);
        for (int64_t c = 0; c < n_ks; ++c) {
            const int64_t k = ks ? ks[c] : c;
            if (k < 0 || k >= r) {
                rc = -1;
                break;
            }
            double g = 0.0, S = 0.0;
            for (int64_t b = 0; b < B; ++b) {
                for (int64_t j = 0; j < d_in; ++j) {
                    double term = yb[b * d_out + i] * s1 * (double)sign_of_packed(V + j * ldv, k) *
                                  nq_oracle_f16_to_double(s2_f16[j]) * x[b * d_in + j];
                    g += term;
                    S += fabs(term);
                }
            }
            if (gU) gU[a * n_ks + c] = g;
            if (SU) SU[a * n_ks + c] = S;
        }
    }
    for (int64_t a = 0; a < n_rows_v && rc == 0; ++a) {
        const int64_t j = rows_v ? rows_v[a] : a;
        if (j < 0 || j >= d_in) {
            rc = -1;
            break;
        }
        const double s2 = nq_oracle_f16_to_double(s2_f16[j]);
        for (int64_t c = 0; c < n_ks; ++c) {
            const int64_t k = ks ? ks[c] : c;
            if (k < 0 || k >= r) {
                rc = -1;
                break;
            }
            double g = 0.0, S = 0.0;
            for (int64_t b = 0; b < B; ++b) {
                for (int64_t i = 0; i < d_out; ++i) {
                    double term = x[b * d_in + j] * s2 * (double)sign_of_packed(U + i * ldu, k) *
                                  nq_oracle_f16_to_double(s1_f16[i]) * yb[b * d_out + i];
                    g += term;
                    S += fabs(term);
                }
            }
            if (gV) gV[a * n_ks + c] = g;
            if (SV) SV[a * n_ks + c] = S;
        }
    }
    free(x);
    free(yb);
    return rc;
}

/* ---------------------------------------------------------------------------------
 * From latent factors to a packed layer (section 3, "Step 2", "Magnitude Balancing and Scale
 * Extraction", then "Phase 3" packing): for the continuous proxies Uh [d_out][r] and
 * Vh [d_in][r],
 *     eta = sqrt( ||Vh||_F / ||Uh||_F ),   U := eta Uh,   V := Vh / eta,
 *     s1_i = mean over k of |U_ik|,        s2_j = mean over k of |V_jk|,
 * and the binary factors are sign(U), sign(V), packed as nq_oracle_pack does.  Readings:
 * the mean runs over the r entries of a row; eta = 1 when either norm is zero; s1, s2 are
 * stored as fp16 (round to nearest even).  Outputs: packed U, V; s1, s2 as fp16 bits and,
 * when the pointers are not NULL, eta and the fp64 scales before rounding.
 * --------------------------------------------------------------------------------- */
ORACLE_API int nq_oracle_from_latent(const float* Uh, int64_t ld_uh, const float* Vh, int64_t ld_vh, int64_t d_out,
                                     int64_t d_in, int64_t r, uint32_t* U, int64_t ldu, uint32_t* V, int64_t ldv,
                                     uint16_t* s1_f16, uint16_t* s2_f16, double* eta_out, double* s1_out,
                                     double* s2_out) {
    if (d_out < 0 || d_in < 0 || r <= 0 || r % 32 != 0 || ld_uh < r || ld_vh < r || ldu < r / 32 || ldv < r / 32)
        return -1;
    double su = 0.0, sv = 0.0;
    for (int64_t i = 0; i < d_out; ++i)
        for (int64_t k = 0; k < r; ++k) su += (double)Uh[i * ld_uh + k] * (double)Uh[i * ld_uh + k];
    for (int64_t j = 0; j < d_in; ++j)
        for (int64_t k = 0; k < r; ++k) sv += (double)Vh[j * ld_vh + k] * (double)Vh[j * ld_vh + k];
    const double nu = sqrt(su), nv = sqrt(sv);
    const double eta = (nu > 0.0 && nv > 0.0) ? sqrt(nv / nu) : 1.0;
    if (eta_out) *eta_out = eta;
    for (int64_t i = 0; i < d_out; ++i) {
        double acc = 0.0;
        for (int64_t w = 0; w < ldu; ++w) U[i * ldu + w] = 0u;
        for (int64_t k = 0; k < r; ++k) {
            double b = eta * (double)Uh[i * ld_uh + k];
            acc += fabs(b);
            if (b >= 0.0) U[i * ldu + k / 32] |= 1u << (k % 32);
        }
        if (s1_out) s1_out[i] = acc / (double)r;
        s1_f16[i] = nq_oracle_double_to_f16(acc / (double)r);
    }
    for (int64_t j = 0; j < d_in; ++j) {
        double acc = 0.0;
        for (int64_t w = 0; w < ldv; ++w) V[j * ldv + w] = 0u;
        for (int64_t k = 0; k < r; ++k) {
            double b = (double)Vh[j * ld_vh + k] / eta;
            acc += fabs(b);
            if (b >= 0.0) V[j * ldv + k / 32] |= 1u << (k % 32);
        }
        if (s2_out) s2_out[j] = acc / (double)r;
        s2_f16[j] = nq_oracle_double_to_f16(acc / (double)r);
    }
    return 0;
}

/* ---------------------------------------------------------------------------------
 * SiLU-gated product between the gate/up and down projections of a Llama MLP block.  This
 * is not on the pages; it is the MLP composition of the 7B/70B workloads:
 *   h = bf16( silu(g) * u ),  silu(g) = g / (1 + exp(-g)),  in fp64 before the rounding.
 * g, u given as fp64; h returned as bf16 bit patterns.
 * --------------------------------------------------------------------------------- */
ORACLE_API void nq_oracle_silu_mul(const double* g, const double* u, int64_t n, uint16_t* h_bf16) {
    for (int64_t e = 0; e < n; ++e) {
        double s = g[e] / (1.0 + exp(-g[e]));
        h_bf16[e] = nq_oracle_double_to_bf16(s * u[e]);
    }
}

/* Rounds n fp64 values to bf16 bit patterns (round to nearest, ties to even). */
ORACLE_API void nq_oracle_round_bf16(const double* v, int64_t n, uint16_t* out) {
    for (int64_t e = 0; e < n; ++e) out[e] = nq_oracle_double_to_bf16(v[e]);
}
