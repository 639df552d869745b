/*
 * mHC (manifold-constrained hyper-connection, HC = 4 streams) CPU oracle, fp64.
 *
 * TEST INFRASTRUCTURE ONLY. This is the plain, slow, obviously-correct restatement of what the
 * pre-map and post-map compute. It shares no code with the CUDA library; only tests/, the package's
 * smoke check and bench.py's cpu_baseline leg load it. Nothing in the product path calls it.
 *
 * Sources (page title, then section):
 *  [FI]  "FlashInfer mHC module deep dive" (www.pwwt.cn/news/5432433): §2.1 post-map formula,
 *        §3.1-3.2 pre-map parameters and defaults, §3.4 kernel phases, §4 prenorm variant (RMS
 *        denominator 4*H), §5.2 test reference math.
 *  [RW]  "rwkv-ops 0.6.1 wheel, rwkv_ops/mhc_kernel/jax_kernel/mhu_jax.py": docstrings of
 *        sinkhorn_knopp, stream_aggregate and mhc_pre_op (H_pre = sigmoid, H_post = 2*sigmoid).
 *  [GLM] "metrale_model_arch/glm5next_mhc.rs": glm_hc_post doc comment (post formula,
 *        comb[i][j] = weight of old stream i into new stream j), mix_hc layout.
 *
 * Layouts (all dense, row-major):
 *   R      [T][4][H]  bf16 bit patterns (uint16)     residual streams
 *   x      [T][H]     bf16 bit patterns              layer output fed to the post-map
 *   hc_fn  [4H][24]   fp32                            projection, row index k = i*H + h
 *   scale  [3]        fp32 (pre, post, comb)          base [24] fp32
 *   logits [T][24]    pre(4) | post(4) | comb(16, row-major 4x4, [old][new])
 *
 * Parity status: every function below is pinned by tests/test_oracle_pins.py against closed
 * forms, invariants and brute force; none is "parity unpinned".
 */
#ifndef MHC_ORACLE_H
#define MHC_ORACLE_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Exact widening of a bf16 bit pattern. */
double mhc_oracle_bf16_to_double(uint16_t bits);

/* Round each double to the nearest bf16 value (ties to even, subnormals and overflow to inf
 * handled), written back as a double holding that exact bf16 value. */
void mhc_oracle_round_bf16(const double* in, int64_t n, double* out);

/* Steps a1-a2: per token, ss = sum of squares of the flattened 4H row, rstd = 1/sqrt(ss/(4H) + rms_eps),
 * raw[j] = sum_k R_flat[k] * hc_fn[k][j]. [FI] §3.4 phase 1 and §5.2 (rstd, mixes = dot_mix * rstd). */
void mhc_oracle_norm_project(const uint16_t* R, const float* hc_fn, int64_t T, int64_t H,
                             double rms_eps, double* ss, double* rstd, double* raw);

/* Step a4 on already-formed logits, as [FI] §5.2's test reference states it: each row of the 4x4
 * goes through a softmax (row maximum subtracted first, [FI] §3.4), eps is added to every entry,
 * then `iters` rounds of (every row divided by its sum; every column divided by its sum), the sums
 * taken plainly. logits and comb are [T][16], [old][new]. */
void mhc_oracle_sinkhorn(const double* logits, int64_t T, int iters, double eps, double* comb);

/* The same normalisation run until the largest change in a round drops below tol or max_iters
 * rounds have run; returns the rounds used for the last token. Used only for invariants. */
int mhc_oracle_sinkhorn_converge(const double* logits, int64_t T, double eps, double tol,
                                 int max_iters, double* comb);

/* Other readings of the pages' Sinkhorn, kept only so a test can report how far each sits from
 * mhc_oracle_sinkhorn: variant 1 = rwkv-ops sinkhorn_knopp's (exp after the row-max shift, eps
 * added to each row and column sum, nothing added to the entries); variant 2 = [FI] §3.4 read as
 * three phases (softmax + eps, one column normalisation, then `iters` full rounds). */
void mhc_oracle_sinkhorn_variant(const double* logits, int64_t T, int iters, double eps,
                                 int variant, double* comb);

/* Step a3 + a4: logits l = raw*rstd*scale[g(j)] + base[j] (g = 0,1,2 for pre, post, comb),
 * pre = sigmoid(l[0:4]) + pre_eps, post = post_mult*sigmoid(l[4:8]), comb = Sinkhorn(l[8:24]). */
void mhc_oracle_coefficients(const double* raw, const double* rstd, const float* scale,
                             const float* base, int64_t T, double pre_eps, double post_mult,
                             int iters, double sinkhorn_eps, double* logits, double* pre,
                             double* post, double* comb);

/* Step a5: y[t][h] = sum_i pre[t][i] * R[t][i][h] (fp64, unrounded). */
void mhc_oracle_aggregate(const uint16_t* R, const double* pre, int64_t T, int64_t H, double* y);

/* Whole pre-map (a1-a5). Any output pointer may be NULL except those the later steps need
 * internally (they are allocated here when NULL). */
void mhc_oracle_pre(const uint16_t* R, const float* hc_fn, const float* scale, const float* base,
                    int64_t T, int64_t H, double rms_eps, double pre_eps, double post_mult,
                    int iters, double sinkhorn_eps, double* rstd, double* logits, double* pre,
                    double* post, double* comb, double* y);

/* Step a6: out[t][n][h] = x[t][h]*post[t][n] + sum_o R[t][o][h]*comb[t][o][n], with post/comb
 * taken as the fp32 values given. [FI] §2.1, [GLM] glm_hc_post. */
void mhc_oracle_post(const uint16_t* x, const uint16_t* R, const float* post, const float* comb,
                     int64_t T, int64_t H, double* out);

/* Number of OpenMP threads the oracle runs with (1 when built without OpenMP). */
int mhc_oracle_threads(void);

/* Sets the number of OpenMP threads later calls use (n >= 1; no effect without OpenMP). */
void mhc_oracle_set_threads(int n);

#ifdef __cplusplus
}
#endif
#endif
