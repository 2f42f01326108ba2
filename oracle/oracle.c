/*
 * oracle.c -- plain, slow, obviously correct fp64 CPU reference for the
 * LUT binary GEMV of the FluxBin page ("FluxBin: Flexible LUT-based
 * Ultra-low-bit LLM Inference by Algorithm-Kernel Synergy").
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the library calls this code: only
 * tests/, __graft_entry__.smoke() and the cpu_baseline leg of bench.py may load
 * it.  It shares no code, header, table or constant with the CUDA path.
 *
 * What is computed (all in double precision, loops in the order written):
 *
 *  1. Dense dequantisation (FluxBin page, Methodology, "1. Algorithm
 *     innovation": decoupled row-column binary decomposition, the equation
 *     W^(k) = (alpha_r^(k) alpha_c^(k)^T) (.) B^(k), summed over the bases k;
 *     plus "Hessian-guided saliency-aware hybrid bases": the final weight is
 *     the global binary approximation PLUS the refinement on the salient
 *     columns).
 *        W[i][j]     = sum_k alpha_r[k][i] * alpha_c[k][j] * B[k][i][j]
 *        W[i][S[t]] += sum_k' s_alpha_r[k'][i] * s_alpha_c[k'][t] * Bs[k'][i][t]
 *  2. The matvec y[i] = sum_j W[i][j] * x[j], j ascending, together with
 *     d[i] = sum_j |W[i][j] x[j]| (the tolerance denominator) and
 *     e[i] = sum over every base of sum_j |alpha_r alpha_c x_j| (the same
 *     magnitude before bases cancel one another).
 *  3. The LUT formulation (FluxBin page, Methodology, "2. Kernel innovation":
 *     LUT-BSF fuses alpha_c into the table entries at build time; the kernel
 *     extracts pattern indices from the packed weights, fetches the
 *     precomputed partial sums, and applies alpha_r in the reduction):
 *        T_k[q][p] = sum_{t<g} (bit t of p ? +1 : -1) * alpha_c[k][qg+t] * x[qg+t]
 *        y'[i]     = sum_k alpha_r[k][i] * sum_q T_k[q][ pattern of B[k][i][qg..qg+g-1] ]
 *     plus the same over the salient columns gathered into a dense compact
 *     vector (virtual columnar mapping, same section).
 *
 * Sign bits use the canonical interchange format: bit t (LSB first) of byte j
 * of a row is column 8j+t; a set bit is +1, a clear bit is -1.  Bit t of a
 * LUT pattern index p is column qg+t of its group (same convention).
 */
#include <math.h>
#include <omp.h>
#include <stddef.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

typedef struct {
    int64_t M, N;
    int32_t K, Ks;
    int64_t nS;
    const uint8_t *sign_bits;   /* [K][M][N/8] */
    const float *alpha_r;       /* [K][M] */
    const float *alpha_c;       /* [K][N], or NULL for all ones */
    const uint32_t *s_idx;      /* [nS] salient columns */
    const uint8_t *s_sign_bits; /* [Ks][M][s_row_bytes] over compact columns */
    int64_t s_row_bytes;
    const float *s_alpha_r;     /* [Ks][M] */
    const float *s_alpha_c;     /* [Ks][nS] */
} oracle_weights;

enum { ORACLE_OK = 0, ORACLE_EINVAL = -1, ORACLE_ENOMEM = -2 };

int oracle_num_threads(void) { return omp_get_max_threads(); }

/* Threads the parallel loops use from now on (n >= 1); for timing the oracle
 * on one core beside all cores.  Changes no arithmetic: rows are independent
 * and each row's sums run in the order written whatever the thread count. */
void oracle_set_num_threads(int n) {
    if (n >= 1) omp_set_num_threads(n);
}

/* ---- activations: stored dtype -> double, exactly ------------------------ */

static double f16_to_f64(uint16_t h) {
    int sign = h >> 15, e = (h >> 10) & 31, m = h & 1023;
    double v;
    if (e == 0)
        v = ldexp((double)m, -24);               /* subnormal: m * 2^-24 */
    else if (e == 31)
        v = m ? NAN : INFINITY;
    else
        v = ldexp((double)(m + 1024), e - 25);   /* (1 + m/1024) * 2^(e-15) */
    return sign ? -v : v;
}

static double bf16_to_f64(uint16_t b) {
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* dtype: 0 = float32, 1 = float16, 2 = bfloat16 (bit patterns). */
int oracle_x_to_f64(int dtype, const void *x, int64_t n, double *out) {
    if (!x || !out || n < 0) return ORACLE_EINVAL;
    for (int64_t i = 0; i < n; ++i) {
        if (dtype == 0)
            out[i] = (double)((const float *)x)[i];
        else if (dtype == 1)
            out[i] = f16_to_f64(((const uint16_t *)x)[i]);
        else if (dtype == 2)
            out[i] = bf16_to_f64(((const uint16_t *)x)[i]);
        else
            return ORACLE_EINVAL;
    }
    return ORACLE_OK;
}

/* ---- weights ------------------------------------------------------------- */

static int sign_at(const uint8_t *row_bits, int64_t j) {
    return ((row_bits[j >> 3] >> (j & 7)) & 1) ? +1 : -1;
}

static int check_weights(const oracle_weights *w) {
    if (!w || w->M < 1 || w->N < 1 || w->N % 8 || w->K < 1 || !w->sign_bits ||
        !w->alpha_r)
        return ORACLE_EINVAL;
    if (w->nS < 0 || w->nS > w->N) return ORACLE_EINVAL;
    if (w->nS > 0) {
        if (w->Ks < 1 || !w->s_idx || !w->s_sign_bits || !w->s_alpha_r ||
            !w->s_alpha_c || w->s_row_bytes * 8 < w->nS)
            return ORACLE_EINVAL;
        for (int64_t t = 0; t < w->nS; ++t)
            if ((int64_t)w->s_idx[t] >= w->N) return ORACLE_EINVAL;
    }
    return ORACLE_OK;
}

/* One row of the dense weight, straight from the definition. */
static void dequant_row(const oracle_weights *w, int64_t i, double *Wrow) {
    const int64_t M = w->M, N = w->N;
    for (int64_t j = 0; j < N; ++j) Wrow[j] = 0.0;
    for (int k = 0; k < w->K; ++k) {
        const uint8_t *bits = w->sign_bits + ((size_t)k * M + i) * (size_t)(N / 8);
        const double ar = w->alpha_r[(size_t)k * M + i];
        for (int64_t j = 0; j < N; ++j) {
            const double ac = w->alpha_c ? w->alpha_c[(size_t)k * N + j] : 1.0;
            Wrow[j] += ar * ac * sign_at(bits, j);
        }
    }
    for (int k = 0; k < (w->nS > 0 ? w->Ks : 0); ++k) {
        const uint8_t *bits = w->s_sign_bits + ((size_t)k * M + i) * (size_t)w->s_row_bytes;
        const double ar = w->s_alpha_r[(size_t)k * M + i];
        for (int64_t t = 0; t < w->nS; ++t) {
            const double ac = w->s_alpha_c[(size_t)k * w->nS + t];
            Wrow[w->s_idx[t]] += ar * ac * sign_at(bits, t);
        }
    }
}

/* Dense rows of W.  rows == NULL means rows 0..nrows-1. */
int oracle_dequant_rows(const oracle_weights *w, int64_t nrows, const int64_t *rows,
                        double *Wout /* [nrows][N] */) {
    int rc = check_weights(w);
    if (rc) return rc;
    if (!Wout || nrows < 0) return ORACLE_EINVAL;
    for (int64_t r = 0; r < nrows; ++r) {
        const int64_t i = rows ? rows[r] : r;
        if (i < 0 || i >= w->M) return ORACLE_EINVAL;
        dequant_row(w, i, Wout + (size_t)r * w->N);
    }
    return ORACLE_OK;
}

/* y[b][r] = sum_j W[i][j] x[b][j] for i = rows[r]; also d and e (see top). */
int oracle_gemv(const oracle_weights *w, const double *x /* [batch][N] */, int batch,
                int64_t nrows, const int64_t *rows, double *y, double *d, double *e) {
    int rc = check_weights(w);
    if (rc) return rc;
    if (!x || !y || batch < 1 || nrows < 0) return ORACLE_EINVAL;
    for (int64_t r = 0; r < nrows; ++r) {
        const int64_t i = rows ? rows[r] : r;
        if (i < 0 || i >= w->M) return ORACLE_EINVAL;
    }
    const int64_t M = w->M, N = w->N;
    int failed = 0;
#pragma omp parallel
    {
        double *Wrow = (double *)malloc(sizeof(double) * (size_t)N);
        if (!Wrow) {
#pragma omp atomic write
            failed = 1;
        }
#pragma omp for schedule(dynamic, 4)
        for (int64_t r = 0; r < nrows; ++r) {
            if (!Wrow) continue;
            const int64_t i = rows ? rows[r] : r;
            dequant_row(w, i, Wrow);
            for (int b = 0; b < batch; ++b) {
                const double *xb = x + (size_t)b * N;
                double acc = 0.0, mag = 0.0;
                for (int64_t j = 0; j < N; ++j) {
                    acc += Wrow[j] * xb[j];
                    mag += fabs(Wrow[j] * xb[j]);
                }
                y[(size_t)b * nrows + r] = acc;
                if (d) d[(size_t)b * nrows + r] = mag;
                if (e) {
                    double m2 = 0.0;
                    for (int k = 0; k < w->K; ++k) {
                        const double ar = fabs((double)w->alpha_r[(size_t)k * M + i]);
                        for (int64_t j = 0; j < N; ++j) {
                            const double ac = w->alpha_c ? w->alpha_c[(size_t)k * N + j] : 1.0;
                            m2 += fabs(ar * ac * xb[j]);
                        }
                    }
                    for (int k = 0; k < (w->nS > 0 ? w->Ks : 0); ++k) {
                        const double ar = fabs((double)w->s_alpha_r[(size_t)k * M + i]);
                        for (int64_t t = 0; t < w->nS; ++t)
                            m2 += fabs(ar * w->s_alpha_c[(size_t)k * w->nS + t] * xb[w->s_idx[t]]);
                    }
                    e[(size_t)b * nrows + r] = m2;
                }
            }
        }
        free(Wrow);
    }
    return failed ? ORACLE_ENOMEM : ORACLE_OK;
}

/* ---- LUT formulation ----------------------------------------------------- */

/* LUT-BSF tables with alpha_c fused at build time:
 * T[k][q][p] = sum_{t<g} (bit t of p ? +1 : -1) * alpha_c[k][q*g+t] * x[q*g+t].
 * ncols must be a multiple of g; alpha_c may be NULL (all ones); ld_ac is the
 * row stride of alpha_c and n_ac the number of columns it covers (columns at or
 * past n_ac take alpha_c = 0, which is how compact salient padding is zeroed). */
static void lut_tables(int64_t ncols, int K, int g, const double *x, const float *alpha_c,
                       int64_t ld_ac, int64_t n_ac, double *T) {
    const int64_t Q = ncols / g, P = (int64_t)1 << g;
    for (int k = 0; k < K; ++k)
        for (int64_t q = 0; q < Q; ++q)
            for (int64_t p = 0; p < P; ++p) {
                double s = 0.0;
                for (int t = 0; t < g; ++t) {
                    const int64_t col = q * g + t;
                    double ac = 1.0;
                    if (alpha_c) ac = col < n_ac ? alpha_c[(size_t)k * ld_ac + col] : 0.0;
                    const double z = ac * x[col];
                    s += ((p >> t) & 1) ? z : -z;
                }
                T[((size_t)k * Q + q) * P + p] = s;
            }
}

int oracle_lut_tables(int64_t N, int K, int g, const double *x, const float *alpha_c,
                      double *T /* [K][N/g][2^g] */) {
    if (N < 1 || K < 1 || !x || !T || !(g == 1 || g == 2 || g == 4 || g == 8) || N % g)
        return ORACLE_EINVAL;
    lut_tables(N, K, g, x, alpha_c, N, N, T);
    return ORACLE_OK;
}

/* Virtual columnar mapping: x_S[t] = x[S[t]] for t < nS, 0 up to nS_pad. */
int oracle_vcm_gather(const double *x, int64_t N, const uint32_t *s_idx, int64_t nS,
                      int64_t nS_pad, double *x_S) {
    if (!x || !x_S || nS < 0 || nS_pad < nS || (nS && !s_idx)) return ORACLE_EINVAL;
    for (int64_t t = 0; t < nS_pad; ++t) {
        if (t < nS) {
            if ((int64_t)s_idx[t] >= N) return ORACLE_EINVAL;
            x_S[t] = x[s_idx[t]];
        } else {
            x_S[t] = 0.0;
        }
    }
    return ORACLE_OK;
}

/* Pattern index of group q (g columns) in one row of sign bits. */
static int64_t pattern_at(const uint8_t *row_bits, int64_t q, int g, int64_t ncols) {
    int64_t p = 0;
    for (int t = 0; t < g; ++t) {
        const int64_t col = q * g + t;
        const int bit = col < ncols ? ((row_bits[col >> 3] >> (col & 7)) & 1) : 0;
        p |= (int64_t)bit << t;
    }
    return p;
}

int oracle_gemv_lut(const oracle_weights *w, int g, const double *x /* [batch][N] */,
                    int batch, int64_t nrows, const int64_t *rows, double *y) {
    int rc = check_weights(w);
    if (rc) return rc;
    if (!x || !y || batch < 1 || nrows < 0 || !(g == 1 || g == 2 || g == 4 || g == 8) ||
        w->N % g)
        return ORACLE_EINVAL;
    for (int64_t r = 0; r < nrows; ++r) {
        const int64_t i = rows ? rows[r] : r;
        if (i < 0 || i >= w->M) return ORACLE_EINVAL;
    }
    const int64_t M = w->M, N = w->N, P = (int64_t)1 << g;
    const int64_t Q = N / g;
    const int64_t nS = w->nS;
    const int Ks = nS > 0 ? w->Ks : 0;
    const int64_t nSg = nS > 0 ? (nS + g - 1) / g * g : 0; /* compact width, whole groups */
    const int64_t Qs = nSg / g;
    double *T = (double *)malloc(sizeof(double) * (size_t)(w->K * Q * P + 1));
    double *Ts = (double *)malloc(sizeof(double) * (size_t)(Ks * Qs * P + 1));
    double *xS = (double *)malloc(sizeof(double) * (size_t)(nSg + 1));
    if (!T || !Ts || !xS) {
        free(T); free(Ts); free(xS);
        return ORACLE_ENOMEM;
    }
    for (int b = 0; b < batch; ++b) {
        const double *xb = x + (size_t)b * N;
        lut_tables(N, w->K, g, xb, w->alpha_c, N, N, T);
        if (nS > 0) {
            oracle_vcm_gather(xb, N, w->s_idx, nS, nSg, xS);
            lut_tables(nSg, Ks, g, xS, w->s_alpha_c, nS, nS, Ts);
        }
#pragma omp parallel for schedule(dynamic, 16)
        for (int64_t r = 0; r < nrows; ++r) {
            const int64_t i = rows ? rows[r] : r;
            double acc = 0.0;
            for (int k = 0; k < w->K; ++k) {
                const uint8_t *bits = w->sign_bits + ((size_t)k * M + i) * (size_t)(N / 8);
                double s = 0.0;
                for (int64_t q = 0; q < Q; ++q)
                    s += T[((size_t)k * Q + q) * P + pattern_at(bits, q, g, N)];
                acc += w->alpha_r[(size_t)k * M + i] * s;
            }
            for (int k = 0; k < Ks; ++k) {
                const uint8_t *bits = w->s_sign_bits + ((size_t)k * M + i) * (size_t)w->s_row_bytes;
                double s = 0.0;
                for (int64_t q = 0; q < Qs; ++q)
                    s += Ts[((size_t)k * Qs + q) * P + pattern_at(bits, q, g, nS)];
                acc += w->s_alpha_r[(size_t)k * M + i] * s;
            }
            y[(size_t)b * nrows + r] = acc;
        }
    }
    free(T); free(Ts); free(xS);
    return ORACLE_OK;
}
