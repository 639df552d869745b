/*
 * mHC CPU oracle in fp64. TEST INFRASTRUCTURE ONLY: loaded by tests/, the smoke check and
 * bench.py's cpu_baseline leg; never by the library. Plain loops in the order the pages state the
 * steps; the only parallelism is an OpenMP loop over independent tokens. See mhc_oracle.h for the
 * sources and layouts.
 */
#include "mhc_oracle.h"

#include <fenv.h>
#include <math.h>
#include <stdlib.h>
#include <string.h>

#ifdef _OPENMP
#include <omp.h>
#endif

enum { HC = 4, MIX = 24 };

int mhc_oracle_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

void mhc_oracle_set_threads(int n) {
#ifdef _OPENMP
    if (n >= 1) omp_set_num_threads(n);
#else
    (void)n;
#endif
}

double mhc_oracle_bf16_to_double(uint16_t bits) {
    uint32_t u = (uint32_t)bits << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* bf16: 8 significant bits, exponent range of fp32. A finite x is rounded to a multiple of its
 * bf16 spacing 2^(max(e,-126) - 7), where e = floor(log2 |x|); the quotient is an exact double, and
 * nearbyint in the default rounding mode breaks ties to even. */
static double round_one_bf16(double x) {
    if (x == 0.0 || !isfinite(x)) return x;
    int e = ilogb(x);
    if (e < -126) e = -126;
    double spacing = ldexp(1.0, e - 7);
    double q = nearbyint(x / spacing) * spacing;
    /* Largest finite bf16 is (2 - 2^-7) * 2^127; anything that rounds past it is infinite. */
    if (fabs(q) >= ldexp(1.0, 128)) return x > 0 ? INFINITY : -INFINITY;
    return q;
}

void mhc_oracle_round_bf16(const double* in, int64_t n, double* out) {
    fesetround(FE_TONEAREST);
    for (int64_t i = 0; i < n; ++i) out[i] = round_one_bf16(in[i]);
}

void mhc_oracle_norm_project(const uint16_t* R, const float* hc_fn, int64_t T, int64_t H,
                             double rms_eps, double* ss_out, double* rstd_out, double* raw_out) {
    const int64_t K = HC * H;
#pragma omp parallel for schedule(static)
    for (int64_t t = 0; t < T; ++t) {
        const uint16_t* row = R + t * K; /* flattened [4][H] row: k = i*H + h */
        double ss = 0.0;
        double raw[MIX] = {0};
        for (int64_t k = 0; k < K; ++k) {
            double v = mhc_oracle_bf16_to_double(row[k]);
            ss += v * v;
            for (int j = 0; j < MIX; ++j) raw[j] += v * (double)hc_fn[k * MIX + j];
        }
        double rstd = 1.0 / sqrt(ss / (double)K + rms_eps);
        if (ss_out) ss_out[t] = ss;
        if (rstd_out) rstd_out[t] = rstd;
        if (raw_out)
            for (int j = 0; j < MIX; ++j) raw_out[t * MIX + j] = raw[j];
    }
}

/* Start of the Sinkhorn step for one token ([FI] §5.2 test reference, §3.4 kernel phase 2): a
 * softmax over each row of the 4x4 logits, computed with the row maximum subtracted first, and eps
 * added to every entry of the result. */
static void softmax_plus_eps(const double* l, double eps, double* A) {
    for (int o = 0; o < HC; ++o) {
        double m = l[o * HC];
        for (int n = 1; n < HC; ++n)
            if (l[o * HC + n] > m) m = l[o * HC + n];
        double e[HC], s = 0.0;
        for (int n = 0; n < HC; ++n) {
            e[n] = exp(l[o * HC + n] - m);
            s += e[n];
        }
        for (int n = 0; n < HC; ++n) A[o * HC + n] = e[n] / s + eps;
    }
}

/* One Sinkhorn round ([FI] §5.2): every row divided by its sum, then every column by its sum. */
static void row_then_column(double* A) {
    for (int o = 0; o < HC; ++o) {
        double s = 0.0;
        for (int n = 0; n < HC; ++n) s += A[o * HC + n];
        for (int n = 0; n < HC; ++n) A[o * HC + n] /= s;
    }
    for (int n = 0; n < HC; ++n) {
        double s = 0.0;
        for (int o = 0; o < HC; ++o) s += A[o * HC + n];
        for (int o = 0; o < HC; ++o) A[o * HC + n] /= s;
    }
}

static void sinkhorn_one(const double* l, int iters, double eps, double* A) {
    softmax_plus_eps(l, eps, A);
    for (int it = 0; it < iters; ++it) row_then_column(A);
}

void mhc_oracle_sinkhorn(const double* logits, int64_t T, int iters, double eps, double* comb) {
#pragma omp parallel for schedule(static)
    for (int64_t t = 0; t < T; ++t) sinkhorn_one(logits + t * 16, iters, eps, comb + t * 16);
}

int mhc_oracle_sinkhorn_converge(const double* logits, int64_t T, double eps, double tol,
                                 int max_iters, double* comb) {
    int used = 0;
    for (int64_t t = 0; t < T; ++t) {
        double A[16], prev[16];
        softmax_plus_eps(logits + t * 16, eps, A);
        int it = 0;
        for (; it < max_iters; ++it) {
            memcpy(prev, A, sizeof A);
            row_then_column(A);
            double d = 0.0;
            for (int i = 0; i < 16; ++i) d = fmax(d, fabs(A[i] - prev[i]));
            if (d < tol) {
                ++it;
                break;
            }
        }
        memcpy(comb + t * 16, A, sizeof A);
        used = it;
    }
    return used;
}

/* Other readings of the Sinkhorn step, kept only so that a test can report how far each sits from
 * mhc_oracle_sinkhorn:
 *   variant 1 (rwkv-ops sinkhorn_knopp, whose eps guards the divisions): A = exp(l - rowmax),
 *             nothing added to the entries, eps added to every row and column sum instead;
 *   variant 2 ([FI] §3.4 read as three phases): softmax + eps, one column normalisation, then
 *             `iters` full (row, column) rounds. */
void mhc_oracle_sinkhorn_variant(const double* logits, int64_t T, int iters, double eps,
                                 int variant, double* comb) {
    for (int64_t t = 0; t < T; ++t) {
        const double* l = logits + t * 16;
        double* A = comb + t * 16;
        if (variant == 1) {
            for (int o = 0; o < HC; ++o) {
                double m = l[o * HC];
                for (int n = 1; n < HC; ++n)
                    if (l[o * HC + n] > m) m = l[o * HC + n];
                for (int n = 0; n < HC; ++n) A[o * HC + n] = exp(l[o * HC + n] - m);
            }
            for (int it = 0; it < iters; ++it) {
                for (int o = 0; o < HC; ++o) {
                    double s = 0.0;
                    for (int n = 0; n < HC; ++n) s += A[o * HC + n];
                    for (int n = 0; n < HC; ++n) A[o * HC + n] /= (s + eps);
                }
                for (int n = 0; n < HC; ++n) {
                    double s = 0.0;
                    for (int o = 0; o < HC; ++o) s += A[o * HC + n];
                    for (int o = 0; o < HC; ++o) A[o * HC + n] /= (s + eps);
                }
            }
        } else {
            softmax_plus_eps(l, eps, A);
            for (int n = 0; n < HC; ++n) {
                double s = 0.0;
                for (int o = 0; o < HC; ++o) s += A[o * HC + n];
                for (int o = 0; o < HC; ++o) A[o * HC + n] /= s;
            }
            for (int it = 0; it < iters; ++it) row_then_column(A);
        }
    }
}

static double sigmoid(double v) { return 1.0 / (1.0 + exp(-v)); }

void mhc_oracle_coefficients(const double* raw, const double* rstd, const float* scale,
                             const float* base, int64_t T, double pre_eps, double post_mult,
                             int iters, double sinkhorn_eps, double* logits, double* pre,
                             double* post, double* comb) {
#pragma omp parallel for schedule(static)
    for (int64_t t = 0; t < T; ++t) {
        double l[MIX];
        for (int j = 0; j < MIX; ++j) {
            int g = j < 4 ? 0 : (j < 8 ? 1 : 2);
            double m = raw[t * MIX + j] * rstd[t];
            l[j] = m * (double)scale[g] + (double)base[j];
        }
        if (logits)
            for (int j = 0; j < MIX; ++j) logits[t * MIX + j] = l[j];
        for (int i = 0; i < HC; ++i) {
            if (pre) pre[t * HC + i] = sigmoid(l[i]) + pre_eps;
            if (post) post[t * HC + i] = post_mult * sigmoid(l[4 + i]);
        }
        if (comb) sinkhorn_one(l + 8, iters, sinkhorn_eps, comb + t * 16);
    }
}

void mhc_oracle_aggregate(const uint16_t* R, const double* pre, int64_t T, int64_t H, double* y) {
#pragma omp parallel for schedule(static)
    for (int64_t t = 0; t < T; ++t) {
        for (int64_t h = 0; h < H; ++h) {
            double s = 0.0;
            for (int i = 0; i < HC; ++i)
                s += pre[t * HC + i] * mhc_oracle_bf16_to_double(R[(t * HC + i) * H + h]);
            y[t * H + h] = s;
        }
    }
}

void mhc_oracle_pre(const uint16_t* R, const float* hc_fn, const float* scale, const float* base,
                    int64_t T, int64_t H, double rms_eps, double pre_eps, double post_mult,
                    int iters, double sinkhorn_eps, double* rstd, double* logits, double* pre,
                    double* post, double* comb, double* y) {
    double* raw = (double*)malloc(sizeof(double) * (size_t)(T > 0 ? T : 1) * MIX);
    double* own_rstd = rstd ? NULL : (double*)malloc(sizeof(double) * (size_t)(T > 0 ? T : 1));
    double* own_pre = pre ? NULL : (double*)malloc(sizeof(double) * (size_t)(T > 0 ? T : 1) * HC);
    double* r = rstd ? rstd : own_rstd;
    double* p = pre ? pre : own_pre;
    mhc_oracle_norm_project(R, hc_fn, T, H, rms_eps, NULL, r, raw);
    mhc_oracle_coefficients(raw, r, scale, base, T, pre_eps, post_mult, iters, sinkhorn_eps, logits,
                            p, post, comb);
    if (y) mhc_oracle_aggregate(R, p, T, H, y);
    free(raw);
    free(own_rstd);
    free(own_pre);
}

void mhc_oracle_post(const uint16_t* x, const uint16_t* R, const float* post, const float* comb,
                     int64_t T, int64_t H, double* out) {
#pragma omp parallel for schedule(static)
    for (int64_t t = 0; t < T; ++t) {
        for (int n = 0; n < HC; ++n) {
            for (int64_t h = 0; h < H; ++h) {
                double v = mhc_oracle_bf16_to_double(x[t * H + h]) * (double)post[t * HC + n];
                for (int o = 0; o < HC; ++o)
                    v += mhc_oracle_bf16_to_double(R[(t * HC + o) * H + h]) *
                         (double)comb[t * 16 + o * HC + n];
                out[(t * HC + n) * H + h] = v;
            }
        }
    }
}
