/*
 * falcon_oracle.c -- TEST INFRASTRUCTURE ONLY. Not part of the product path.
 *
 * A plain, slow, fp64 CPU oracle for the forward pass of the Falcon fast-weight
 * memory ("Fast Weight Attention for Continual Learning"). Only the test suite,
 * the package smoke check and the CPU-baseline leg of the benchmark call it.
 * It shares no code, header, table or helper with the CUDA library; the two
 * meet only through the seeded input generator, which holds none of the
 * method's arithmetic.
 *
 * What the method computes, as stated in the authors' abstract (Hugging Face
 * paper page, ai.info and hotpaper.ai pages for "Fast Weight Attention for
 * Continual Learning"):
 *   - each head keeps a fixed-size state S (d_v x d_k) and the state transition
 *     is an online learning rule;
 *   - under read-after-write semantics the example written at step t is the
 *     prefix-aligned pair (x_t, y_t) = (phi(k_{t-1}), v_t);
 *   - normalised first-order updates of a squared-error regression objective
 *     give Falcon-1 (scalar NLMS) and Falcon-3 (sliding-window mini-batch); the
 *     negative inner-product objective gives the "A" variants;
 *   - recurrent, masked-parallel and chunk-parallel forms exist, with a
 *     numerically stable positive-decay renormalisation.
 * The normalised step size is the Kaczmarz/NLMS one, written out explicitly in
 * the Kaczmarz Linear Attention abstract on the thelatestinai.com page
 * "Fast Weight Attention for Continual Learning": beta = eta / (||key||^2 + eps).
 *
 * Readings taken where the pages are silent (each is also listed in the
 * design notes):
 *   R1 read after write: o_t = S_t q_t.
 *   R2 decay before the step, residual at the decayed state:
 *        Sbar = alpha_t S_{t-1};   Falcon-1: S_t = Sbar - beta_t (Sbar x_t - y_t) x_t^T.
 *   R3 alpha_t, eta_t belong to write step t.
 *   R4 phi = identity; q is not mapped.
 *   R5 beta_t = eta_t / (||x_t||^2 + eps); Falcon-3 uses the window's summed
 *      squared key norms; if the denominator is 0 (zero key and eps = 0) the
 *      step is a no-op (beta = 0).
 *   R6 x_1 = k_prev when a cache is given, else 0 (no write at the first step).
 *   R7 Falcon-3 window W_t = {max(1, t-w+1) .. t}; all residuals of one step use
 *      the same decayed state (a simultaneous mini-batch gradient step).
 *   R8 Falcon-1A / Falcon-3A: gradient step of -y^T S x with the same beta:
 *        S_t = alpha_t S_{t-1} + beta_t sum_{j in W_t} y_j x_j^T.
 *   R9 positive-decay renormalisation: only decay factors exp(g_i - g_j) with
 *      i >= j are ever formed, so each factor lies in (0, 1]; nothing is divided
 *      by a cumulative product of alphas.
 *   R11 Falcon-2 / Falcon-2A: see f2_head below.
 *   R10 same-step association (flag OR_SAME_STEP in `rule`): the pair written at
 *      step t is (phi(k_t), v_t), the association of Kaczmarz Linear Attention
 *      (thelatestinai.com page, KLA abstract), which the authors' abstract names
 *      as the alternative to the prefix-aligned pair. k_prev is then not used as
 *      a key; k_last is still the last key.
 *
 * Indices below are 0-based: pair j has x_j = k_{j-1} (j >= 1), x_0 = k_prev
 * or 0 (same-step association: x_j = k_j), and y_j = v_j.
 *
 * Layout: q, k (B,H,T,dk); v, o (B,H,T,dv); alpha, eta (B,H,T);
 *         S0, S_out (B,H,dv,dk) with S[i][c] the weight from key coordinate c
 *         to value coordinate i; k_prev, k_last (B,H,dk). All row-major fp64.
 */
#include <math.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define OR_RULE_1 1
#define OR_RULE_1A 2
#define OR_RULE_3 3
#define OR_RULE_3A 4
#define OR_RULE_2 5
#define OR_RULE_2A 6
#define OR_SAME_STEP 0x100 /* flag bit in `rule`: reading R10 */

#define OR_OK 0
#define OR_EINVAL -1
#define OR_ENOMEM -2

static int base_rule(int rule) { return rule & ~OR_SAME_STEP; }
static int same_step(int rule) { return (rule & OR_SAME_STEP) != 0; }

static int rule_ok(int rule) {
    const int b = base_rule(rule);
    return b == OR_RULE_1 || b == OR_RULE_1A || b == OR_RULE_3 || b == OR_RULE_3A;
}

/* The regression family (Falcon-1, Falcon-3) versus the inner-product family. */
static int is_regression(int rule) { return base_rule(rule) == OR_RULE_1 || base_rule(rule) == OR_RULE_3; }

/* Falcon-1 and Falcon-1A write one pair per step; Falcon-3 and -3A a window. */
static int eff_window(int rule, int window) {
    return (base_rule(rule) == OR_RULE_3 || base_rule(rule) == OR_RULE_3A) ? window : 1;
}

static double dotd(const double *a, const double *b, int n) {
    double s = 0.0;
    for (int i = 0; i < n; ++i) s += a[i] * b[i];
    return s;
}

/* x_j: the key half of pair j (prefix-aligned pair of the abstract, reading R6; same-step
 * association k_j when `same` is set, reading R10). */
static void pair_key(double *x, const double *kh, const double *kprev_h, long j, int dk, int same) {
    if (same) {
        if (j >= 0)
            memcpy(x, kh + (size_t)j * dk, sizeof(double) * dk);
        else
            memset(x, 0, sizeof(double) * dk);
    } else if (j >= 1)
        memcpy(x, kh + (size_t)(j - 1) * dk, sizeof(double) * dk);
    else if (j == 0 && kprev_h)
        memcpy(x, kprev_h, sizeof(double) * dk);
    else
        memset(x, 0, sizeof(double) * dk);
}

/* Normalised step size (Kaczmarz Linear Attention abstract; reading R5). */
static double step_size(double eta, double norm_sum, double eps) {
    double den = norm_sum + eps;
    return den > 0.0 ? eta / den : 0.0;
}

static int check_args(int rule, int B, int H, int T, int dk, int dv, int window,
                      const double *q, const double *k, const double *v,
                      const double *alpha, const double *eta) {
    if (!rule_ok(rule) || B < 0 || H < 0 || T < 0 || dk <= 0 || dv <= 0) return 0;
    if ((base_rule(rule) == OR_RULE_3 || base_rule(rule) == OR_RULE_3A) && window < 1) return 0;
    if ((size_t)B * H * T > 0 && (!q || !k || !v || !alpha || !eta)) return 0;
    return 1;
}

/* ------------------------------------------------------------------------
 * Recurrent form, one head (authors' abstract; ai.info overview, section
 * Methodology in Plain English; update rules of the abstract).
 * Literally per token:
 *   Sbar = alpha_t S
 *   beta = eta_t / (sum_{j in W_t} ||x_j||^2 + eps)
 *   regression:     S = Sbar - beta * sum_j (Sbar x_j - y_j) x_j^T
 *   inner product:  S = Sbar + beta * sum_j y_j x_j^T
 *   o_t = S q_t
 * ------------------------------------------------------------------------ */
static int recurrent_head(int rule, int T, int dk, int dv, const double *q, const double *k,
                          const double *v, const double *alpha, const double *eta, double eps,
                          int w, const double *S0, const double *kprev, double *o,
                          double *S_out, double *k_last) {
    double *S = (double *)calloc((size_t)dv * dk, sizeof(double));
    double *X = (double *)malloc(sizeof(double) * (size_t)w * dk);
    double *R = (double *)malloc(sizeof(double) * (size_t)w * dv);
    if (!S || !X || !R) {
        free(S); free(X); free(R);
        return OR_ENOMEM;
    }
    if (S0) memcpy(S, S0, sizeof(double) * (size_t)dv * dk);
    const int regression = is_regression(rule);

    for (long t = 0; t < T; ++t) {
        const double a = alpha[t];
        for (size_t i = 0; i < (size_t)dv * dk; ++i) S[i] *= a; /* Sbar = alpha_t S */

        double nsum = 0.0;
        for (int m = 0; m < w; ++m) {
            pair_key(X + (size_t)m * dk, k, kprev, t - m, dk, same_step(rule));
            nsum += dotd(X + (size_t)m * dk, X + (size_t)m * dk, dk);
        }
        const double beta = step_size(eta[t], nsum, eps);

        if (regression) {
            /* all residuals at the same decayed state (reading R7) */
            for (int m = 0; m < w; ++m) {
                const long j = t - m;
                for (int i = 0; i < dv; ++i) {
                    const double yi = (j >= 0) ? v[(size_t)j * dv + i] : 0.0;
                    R[(size_t)m * dv + i] = dotd(S + (size_t)i * dk, X + (size_t)m * dk, dk) - yi;
                }
            }
            for (int m = 0; m < w; ++m)
                for (int i = 0; i < dv; ++i) {
                    const double ri = beta * R[(size_t)m * dv + i];
                    for (int c = 0; c < dk; ++c) S[(size_t)i * dk + c] -= ri * X[(size_t)m * dk + c];
                }
        } else {
            for (int m = 0; m < w; ++m) {
                const long j = t - m;
                if (j < 0) continue;
                for (int i = 0; i < dv; ++i) {
                    const double yi = beta * v[(size_t)j * dv + i];
                    for (int c = 0; c < dk; ++c) S[(size_t)i * dk + c] += yi * X[(size_t)m * dk + c];
                }
            }
        }
        /* read after write (reading R1) */
        for (int i = 0; i < dv; ++i) o[(size_t)t * dv + i] = dotd(S + (size_t)i * dk, q + (size_t)t * dk, dk);
    }
    if (S_out) memcpy(S_out, S, sizeof(double) * (size_t)dv * dk);
    if (k_last) {
        if (T > 0) memcpy(k_last, k + (size_t)(T - 1) * dk, sizeof(double) * dk);
        else if (kprev) memcpy(k_last, kprev, sizeof(double) * dk);
        else memset(k_last, 0, sizeof(double) * dk);
    }
    free(S); free(X); free(R);
    return OR_OK;
}

/* ------------------------------------------------------------------------
 * Chunk-parallel form, one head (chunk-parallel and masked-parallel forms of
 * the abstract, with positive-decay renormalisation; reading R9).
 *
 * Unrolling the recurrence over one block of steps s = 0..n-1 that starts from
 * state S_c: every step writes pseudo-values u_{s,m} (one per window slot m,
 * pair j = c0 + s - m):
 *   S_after_s = exp(g_s) S_c + sum_{s' <= s} sum_m exp(g_s - g_s') u_{s',m} x_{s'-m}^T
 * where g_s = sum_{s'' <= s} log alpha is the block-local cumulative log decay.
 * Substituting into the step rule gives, for the regression family, the unit
 * lower-triangular system
 *   u_{s,m} + beta_s sum_{s' < s} sum_m' exp(g_s - g_s') (x_{s-m} . x_{s'-m'}) u_{s',m'}
 *       = beta_s (y_{s-m} - exp(g_s) S_c x_{s-m}),
 * and u_{s,m} = beta_s y_{s-m} for the inner-product family. Then
 *   o_{c0+i} = exp(g_i) S_c q_i + sum_{s' <= i} sum_m exp(g_i - g_s') (q_i . x_{s'-m}) u_{s',m}
 *   S_{c+1}  = exp(g_{n-1}) S_c + sum_{s'} sum_m exp(g_{n-1} - g_s') u_{s',m} x_{s'-m}^T.
 * Every decay factor formed has a non-positive exponent. With block = T this is
 * the masked-parallel form (one T-step block, global cumulative log decay).
 * ------------------------------------------------------------------------ */
static int blocked_head(int rule, int T, int dk, int dv, const double *q, const double *k,
                        const double *v, const double *alpha, const double *eta, double eps,
                        int w, int C, const double *S0, const double *kprev, double *o,
                        double *S_out, double *k_last) {
    const size_t Emax = (size_t)C * w;
    double *S = (double *)calloc((size_t)dv * dk, sizeof(double));
    double *Xe = (double *)malloc(sizeof(double) * Emax * dk);
    double *Ye = (double *)malloc(sizeof(double) * Emax * dv);
    double *U = (double *)malloc(sizeof(double) * Emax * dv);
    double *beta = (double *)malloc(sizeof(double) * (size_t)C);
    double *g = (double *)malloc(sizeof(double) * (size_t)C);
    if (!S || !Xe || !Ye || !U || !beta || !g) {
        free(S); free(Xe); free(Ye); free(U); free(beta); free(g);
        return OR_ENOMEM;
    }
    if (S0) memcpy(S, S0, sizeof(double) * (size_t)dv * dk);
    const int regression = is_regression(rule);

    for (long c0 = 0; c0 < T; c0 += C) {
        const int n = (int)((T - c0) < C ? (T - c0) : C);
        const int E = n * w;
        /* expanded rows e = s*w + m hold pair j = c0 + s - m */
        for (int s = 0; s < n; ++s)
            for (int m = 0; m < w; ++m) {
                const int e = s * w + m;
                const long j = c0 + s - m;
                pair_key(Xe + (size_t)e * dk, k, kprev, j, dk, same_step(rule));
                if (j >= 0) memcpy(Ye + (size_t)e * dv, v + (size_t)j * dv, sizeof(double) * dv);
                else memset(Ye + (size_t)e * dv, 0, sizeof(double) * dv);
            }
        double acc = 0.0;
        for (int s = 0; s < n; ++s) {
            double nsum = 0.0;
            for (int m = 0; m < w; ++m) {
                const double *xe = Xe + (size_t)(s * w + m) * dk;
                nsum += dotd(xe, xe, dk);
            }
            beta[s] = step_size(eta[c0 + s], nsum, eps);
            acc += log(alpha[c0 + s]);
            g[s] = acc;
        }
        /* pseudo-values */
        for (int e = 0; e < E; ++e) {
            const int s = e / w;
            const double *xe = Xe + (size_t)e * dk;
            double *ue = U + (size_t)e * dv;
            if (regression) {
                const double gs = exp(g[s]);
                for (int i = 0; i < dv; ++i)
                    ue[i] = beta[s] * (Ye[(size_t)e * dv + i] - gs * dotd(S + (size_t)i * dk, xe, dk));
                /* forward substitution through the strictly lower block part */
                for (int e2 = 0; e2 < s * w; ++e2) {
                    const int s2 = e2 / w;
                    const double l = beta[s] * exp(g[s] - g[s2]) * dotd(xe, Xe + (size_t)e2 * dk, dk);
                    const double *u2 = U + (size_t)e2 * dv;
                    for (int i = 0; i < dv; ++i) ue[i] -= l * u2[i];
                }
            } else {
                for (int i = 0; i < dv; ++i) ue[i] = beta[s] * Ye[(size_t)e * dv + i];
            }
        }
        /* outputs, read after write: the inclusive (s' <= i) sum */
        for (int i = 0; i < n; ++i) {
            const long t = c0 + i;
            const double *qt = q + (size_t)t * dk;
            double *ot = o + (size_t)t * dv;
            const double gi = exp(g[i]);
            for (int r = 0; r < dv; ++r) ot[r] = gi * dotd(S + (size_t)r * dk, qt, dk);
            for (int e2 = 0; e2 < (i + 1) * w; ++e2) {
                const int s2 = e2 / w;
                const double p = exp(g[i] - g[s2]) * dotd(qt, Xe + (size_t)e2 * dk, dk);
                const double *u2 = U + (size_t)e2 * dv;
                for (int r = 0; r < dv; ++r) ot[r] += p * u2[r];
            }
        }
        /* state passing */
        const double gl = g[n - 1];
        const double dl = exp(gl);
        for (size_t idx = 0; idx < (size_t)dv * dk; ++idx) S[idx] *= dl;
        for (int e2 = 0; e2 < E; ++e2) {
            const int s2 = e2 / w;
            const double f = exp(gl - g[s2]);
            const double *u2 = U + (size_t)e2 * dv;
            const double *x2 = Xe + (size_t)e2 * dk;
            for (int r = 0; r < dv; ++r) {
                const double fr = f * u2[r];
                for (int c = 0; c < dk; ++c) S[(size_t)r * dk + c] += fr * x2[c];
            }
        }
    }
    if (S_out) memcpy(S_out, S, sizeof(double) * (size_t)dv * dk);
    if (k_last) {
        if (T > 0) memcpy(k_last, k + (size_t)(T - 1) * dk, sizeof(double) * dk);
        else if (kprev) memcpy(k_last, kprev, sizeof(double) * dk);
        else memset(k_last, 0, sizeof(double) * dk);
    }
    free(S); free(Xe); free(Ye); free(U); free(beta); free(g);
    return OR_OK;
}

typedef struct {
    int rule, B, H, T, dk, dv, w, C;
    const double *q, *k, *v, *alpha, *eta, *S0, *k_prev;
    double eps;
    double *o, *S_out, *k_last;
} job_t;

static int run_heads(const job_t *J, int blocked, int threads) {
    const long BH = (long)J->B * J->H;
    int status = OR_OK;
    if (threads < 1) threads = 1;
#ifdef _OPENMP
#pragma omp parallel for schedule(dynamic, 1) num_threads(threads)
#endif
    for (long bh = 0; bh < BH; ++bh) {
        const size_t T = (size_t)J->T;
        const double *S0h = J->S0 ? J->S0 + (size_t)bh * J->dv * J->dk : NULL;
        const double *kph = J->k_prev ? J->k_prev + (size_t)bh * J->dk : NULL;
        double *Soh = J->S_out ? J->S_out + (size_t)bh * J->dv * J->dk : NULL;
        double *klh = J->k_last ? J->k_last + (size_t)bh * J->dk : NULL;
        int rc;
        if (blocked)
            rc = blocked_head(J->rule, J->T, J->dk, J->dv, J->q + bh * T * J->dk, J->k + bh * T * J->dk,
                              J->v + bh * T * J->dv, J->alpha + bh * T, J->eta + bh * T, J->eps, J->w,
                              J->C, S0h, kph, J->o + bh * T * J->dv, Soh, klh);
        else
            rc = recurrent_head(J->rule, J->T, J->dk, J->dv, J->q + bh * T * J->dk, J->k + bh * T * J->dk,
                                J->v + bh * T * J->dv, J->alpha + bh * T, J->eta + bh * T, J->eps, J->w,
                                S0h, kph, J->o + bh * T * J->dv, Soh, klh);
        if (rc != OR_OK) {
#ifdef _OPENMP
#pragma omp atomic write
#endif
            status = rc;
        }
    }
    return status;
}

/* Exported entry points (fp64 host arrays; threads = OpenMP threads over (b,h)). */

int falcon_oracle_recurrent(int rule, int B, int H, int T, int dk, int dv, const double *q,
                            const double *k, const double *v, const double *alpha,
                            const double *eta, double eps, int window, const double *S0,
                            const double *k_prev, double *o, double *S_out, double *k_last,
                            int threads) {
    if (!check_args(rule, B, H, T, dk, dv, window, q, k, v, alpha, eta)) return OR_EINVAL;
    if ((size_t)B * H * T > 0 && !o) return OR_EINVAL;
    job_t J = {rule, B, H, T, dk, dv, eff_window(rule, window), 1, q, k, v, alpha, eta, S0, k_prev,
               eps, o, S_out, k_last};
    return run_heads(&J, 0, threads);
}

int falcon_oracle_chunk(int rule, int B, int H, int T, int dk, int dv, const double *q,
                        const double *k, const double *v, const double *alpha, const double *eta,
                        double eps, int window, int chunk, const double *S0, const double *k_prev,
                        double *o, double *S_out, double *k_last, int threads) {
    if (!check_args(rule, B, H, T, dk, dv, window, q, k, v, alpha, eta) || chunk < 1) return OR_EINVAL;
    if ((size_t)B * H * T > 0 && !o) return OR_EINVAL;
    job_t J = {rule, B, H, T, dk, dv, eff_window(rule, window), chunk, q, k, v, alpha, eta, S0,
               k_prev, eps, o, S_out, k_last};
    return run_heads(&J, 1, threads);
}

/* Masked-parallel form: the whole sequence as one block (global cumulative log decay). */
int falcon_oracle_masked(int rule, int B, int H, int T, int dk, int dv, const double *q,
                         const double *k, const double *v, const double *alpha, const double *eta,
                         double eps, int window, const double *S0, const double *k_prev, double *o,
                         double *S_out, double *k_last, int threads) {
    return falcon_oracle_chunk(rule, B, H, T, dk, dv, q, k, v, alpha, eta, eps, window,
                               T > 0 ? T : 1, S0, k_prev, o, S_out, k_last, threads);
}

/* ------------------------------------------------------------------------
 * Falcon-2 / Falcon-2A (reading R11 below; the pages name Falcon-2 only as the
 * per-column extension of the scalar NLMS update, "a version that keeps a
 * separate normalization per column", ai.info overview, sections Key
 * Contributions and Methodology in Plain English).
 *   R11 Column c of S multiplies key coordinate c, so each column keeps its own
 *       normaliser: the running energy of its key coordinate,
 *         n_{t,c} = alpha_t n_{t-1,c} + x_{t,c}^2      (n_0 = n0 or 0),
 *       decayed with the state's gate. The step is the NLMS step in the metric
 *       D_t = diag(1 / (n_{t,c} + eps)): with the write key
 *         z_t = eta_t D_t x_t / (x_t^T D_t x_t + eps)   (0 where a denominator is 0),
 *       Falcon-2:  S_t = Sbar - (Sbar x_t - y_t) z_t^T,
 *       Falcon-2A: S_t = Sbar + y_t z_t^T,   o_t = S_t q_t.
 *       The step is the gradient of 1/2 ||Sbar x - y||^2 (resp. -y^T Sbar x) with
 *       column c scaled by its own step eta D_cc / (x^T D x + eps). With eps = 0 it
 *       interpolates exactly (S_t x_t = y_t for eta = 1), and with equal column
 *       energies (D a multiple of I) it is Falcon-1. The reading that divides each
 *       column by the instantaneous x_{t,c}^2 alone (no running energy) was tried
 *       and rejected: its write key has entries up to 1/|x_c|, and on normalised
 *       random keys the state grows without bound within a few thousand steps.
 * ------------------------------------------------------------------------ */
static void f2_write_key(double *z, const double *x, double *nrun, double alpha, double eta, double eps, int dk) {
    double N = 0.0;
    for (int c = 0; c < dk; ++c) {
        nrun[c] = alpha * nrun[c] + x[c] * x[c];
        const double den = nrun[c] + eps;
        z[c] = den > 0.0 ? x[c] / den : 0.0;
        N += z[c] * x[c];
    }
    const double den = N + eps;
    const double coef = den > 0.0 ? eta / den : 0.0;
    for (int c = 0; c < dk; ++c) z[c] *= coef;
}

/* Falcon-2 / 2A, one head: recurrent form (C == 0) or blocked form with C-step blocks (the
 * chunk-parallel form of a delta rule whose write key z_t differs from its read key x_t):
 *   u_s = y_s - exp(g_s) S_c x_s - sum_{s' < s} exp(g_s - g_s') (x_s . z_s') u_s'   (Falcon-2)
 *   u_s = y_s                                                                      (Falcon-2A)
 *   o_i = exp(g_i) S_c q_i + sum_{s' <= i} exp(g_i - g_s') (q_i . z_s') u_s'
 *   S_{c+1} = exp(g_last) S_c + sum_s exp(g_last - g_s) u_s z_s^T
 * Every decay factor has a non-positive exponent (reading R9). */
static int f2_head(int rule, int T, int dk, int dv, const double *q, const double *k, const double *v,
                   const double *alpha, const double *eta, double eps, int C, const double *S0,
                   const double *kprev, const double *n0, double *o, double *S_out, double *k_last,
                   double *n_out) {
    const int regression = base_rule(rule) == OR_RULE_2;
    const int B = C > 0 ? C : 1;
    double *S = (double *)calloc((size_t)dv * dk, sizeof(double));
    double *nrun = (double *)calloc((size_t)dk, sizeof(double));
    double *X = (double *)malloc(sizeof(double) * (size_t)B * dk);
    double *Z = (double *)malloc(sizeof(double) * (size_t)B * dk);
    double *U = (double *)malloc(sizeof(double) * (size_t)B * dv);
    double *g = (double *)malloc(sizeof(double) * (size_t)B);
    if (!S || !nrun || !X || !Z || !U || !g) {
        free(S); free(nrun); free(X); free(Z); free(U); free(g);
        return OR_ENOMEM;
    }
    if (S0) memcpy(S, S0, sizeof(double) * (size_t)dv * dk);
    if (n0) memcpy(nrun, n0, sizeof(double) * dk);
    if (C <= 0) {
        for (long t = 0; t < T; ++t) {
            pair_key(X, k, kprev, t, dk, same_step(rule));
            f2_write_key(Z, X, nrun, alpha[t], eta[t], eps, dk);
            for (size_t i = 0; i < (size_t)dv * dk; ++i) S[i] *= alpha[t];   /* Sbar */
            for (int i = 0; i < dv; ++i) {
                const double y = v[(size_t)t * dv + i];
                const double coef = regression ? dotd(S + (size_t)i * dk, X, dk) - y : -y;
                for (int c = 0; c < dk; ++c) S[(size_t)i * dk + c] -= coef * Z[c];
            }
            for (int i = 0; i < dv; ++i) o[(size_t)t * dv + i] = dotd(S + (size_t)i * dk, q + (size_t)t * dk, dk);
        }
    } else {
        for (long c0 = 0; c0 < T; c0 += C) {
            const int n = (int)((T - c0) < C ? (T - c0) : C);
            double acc = 0.0;
            for (int s2 = 0; s2 < n; ++s2) {
                pair_key(X + (size_t)s2 * dk, k, kprev, c0 + s2, dk, same_step(rule));
                f2_write_key(Z + (size_t)s2 * dk, X + (size_t)s2 * dk, nrun, alpha[c0 + s2], eta[c0 + s2], eps, dk);
                acc += log(alpha[c0 + s2]);
                g[s2] = acc;
            }
            for (int s2 = 0; s2 < n; ++s2) {
                double *us = U + (size_t)s2 * dv;
                const double *xs = X + (size_t)s2 * dk;
                for (int i = 0; i < dv; ++i) {
                    us[i] = v[(size_t)(c0 + s2) * dv + i];
                    if (regression) us[i] -= exp(g[s2]) * dotd(S + (size_t)i * dk, xs, dk);
                }
                if (regression)
                    for (int s3 = 0; s3 < s2; ++s3) {
                        const double l = exp(g[s2] - g[s3]) * dotd(xs, Z + (size_t)s3 * dk, dk);
                        for (int i = 0; i < dv; ++i) us[i] -= l * U[(size_t)s3 * dv + i];
                    }
            }
            for (int i2 = 0; i2 < n; ++i2) {
                const double *qt = q + (size_t)(c0 + i2) * dk;
                double *ot = o + (size_t)(c0 + i2) * dv;
                for (int r = 0; r < dv; ++r) ot[r] = exp(g[i2]) * dotd(S + (size_t)r * dk, qt, dk);
                for (int s3 = 0; s3 <= i2; ++s3) {
                    const double pz = exp(g[i2] - g[s3]) * dotd(qt, Z + (size_t)s3 * dk, dk);
                    for (int r = 0; r < dv; ++r) ot[r] += pz * U[(size_t)s3 * dv + r];
                }
            }
            const double gl = g[n - 1];
            for (size_t idx = 0; idx < (size_t)dv * dk; ++idx) S[idx] *= exp(gl);
            for (int s3 = 0; s3 < n; ++s3) {
                const double f = exp(gl - g[s3]);
                for (int r = 0; r < dv; ++r)
                    for (int c = 0; c < dk; ++c) S[(size_t)r * dk + c] += f * U[(size_t)s3 * dv + r] * Z[(size_t)s3 * dk + c];
            }
        }
    }
    if (S_out) memcpy(S_out, S, sizeof(double) * (size_t)dv * dk);
    if (n_out) memcpy(n_out, nrun, sizeof(double) * dk);
    if (k_last) {
        if (T > 0) memcpy(k_last, k + (size_t)(T - 1) * dk, sizeof(double) * dk);
        else if (kprev) memcpy(k_last, kprev, sizeof(double) * dk);
        else memset(k_last, 0, sizeof(double) * dk);
    }
    free(S); free(nrun); free(X); free(Z); free(U); free(g);
    return OR_OK;
}

/* Falcon-2 / 2A for every head: chunk = 0 runs the recurrent form, chunk >= 1 the blocked form
 * (chunk >= T is the masked-parallel form). n0 / n_out: (B,H,dk) running column energies, or NULL. */
int falcon_oracle_f2(int rule, int B, int H, int T, int dk, int dv, const double *q, const double *k,
                     const double *v, const double *alpha, const double *eta, double eps, int chunk,
                     const double *S0, const double *k_prev, const double *n0, double *o, double *S_out,
                     double *k_last, double *n_out, int threads) {
    const int b = base_rule(rule);
    if ((b != OR_RULE_2 && b != OR_RULE_2A) || B < 0 || H < 0 || T < 0 || dk <= 0 || dv <= 0 || chunk < 0)
        return OR_EINVAL;
    if ((size_t)B * H * T > 0 && (!q || !k || !v || !alpha || !eta || !o)) return OR_EINVAL;
    const long BH = (long)B * H;
    int status = OR_OK;
    if (threads < 1) threads = 1;
#ifdef _OPENMP
#pragma omp parallel for schedule(dynamic, 1) num_threads(threads)
#endif
    for (long bh = 0; bh < BH; ++bh) {
        const size_t TT = (size_t)T, DD = (size_t)dv * dk;
        const int rc = f2_head(rule, T, dk, dv, q + bh * TT * dk, k + bh * TT * dk, v + bh * TT * dv,
                               alpha + bh * TT, eta + bh * TT, eps, chunk, S0 ? S0 + bh * DD : NULL,
                               k_prev ? k_prev + bh * dk : NULL, n0 ? n0 + bh * dk : NULL, o + bh * TT * dv,
                               S_out ? S_out + bh * DD : NULL, k_last ? k_last + bh * dk : NULL,
                               n_out ? n_out + bh * dk : NULL);
        if (rc != OR_OK) {
#ifdef _OPENMP
#pragma omp atomic write
#endif
            status = rc;
        }
    }
    return status;
}

/* ------------------------------------------------------------------------
 * Gradients of the recurrent form, one head: reverse mode through the literal
 * per-token recurrence above. The pages give the forward rules only (authors'
 * abstract); these are their derivatives, written out step by step, to check a
 * backward pass. For a loss L with upstream gradients dO = dL/do (T x dv) and
 * dST = dL/dS_T (dv x dk, NULL = 0), with U = dL/dS_after at step t:
 *   o_t = S_t q_t:            U += dO_t q_t^T,  dq_t = S_t^T dO_t
 *   regression, r_j = Sbar x_j - y_j, S_t = Sbar - beta sum_j r_j x_j^T:
 *     dbeta = -sum_j r_j^T U x_j;  dr_j = -beta U x_j;
 *     dx_j += -beta U^T r_j + Sbar^T dr_j;  dy_j = -dr_j;  dSbar = U + sum_j dr_j x_j^T
 *   inner product, S_t = Sbar + beta sum_j y_j x_j^T:
 *     dbeta = sum_j y_j^T U x_j;  dy_j = beta U x_j;  dx_j += beta U^T y_j;  dSbar = U
 *   beta = eta / (N + eps), N = sum_j ||x_j||^2 (no gradient when N + eps = 0):
 *     deta_t = dbeta / (N + eps);  dx_j += 2 (-dbeta beta / (N + eps)) x_j
 *   Sbar = alpha_t S_{t-1}:  dalpha_t = <dSbar, S_{t-1}>,  U <- alpha_t dSbar
 * then dk and dk_prev collect dx through the pairing of reading R6 / R10, dv
 * collects dy, and dS0 is the final U. Every state S_0..S_T is kept (small
 * problems only).
 * ------------------------------------------------------------------------ */
static int backward_head(int rule, int T, int dk, int dv, const double *q, const double *k,
                         const double *v, const double *alpha, const double *eta, double eps, int w,
                         const double *S0, const double *kprev, const double *dO, const double *dST,
                         double *dq, double *dkk, double *dvv, double *dal, double *det, double *dS0,
                         double *dkp) {
    const size_t DD = (size_t)dv * dk;
    double *St = (double *)calloc((size_t)(T + 1) * DD, sizeof(double));   /* St[t] = state before step t */
    double *U = (double *)calloc(DD, sizeof(double));
    double *Sb = (double *)malloc(sizeof(double) * DD);
    double *dSb = (double *)malloc(sizeof(double) * DD);
    double *X = (double *)malloc(sizeof(double) * (size_t)w * dk);
    double *Y = (double *)malloc(sizeof(double) * (size_t)w * dv);
    double *Rr = (double *)malloc(sizeof(double) * (size_t)w * dv);
    double *dX = (double *)malloc(sizeof(double) * (size_t)w * dk);
    double *dY = (double *)malloc(sizeof(double) * (size_t)w * dv);
    double *Ux = (double *)malloc(sizeof(double) * dv);
    if (!St || !U || !Sb || !dSb || !X || !Y || !Rr || !dX || !dY || !Ux) {
        free(St); free(U); free(Sb); free(dSb); free(X); free(Y); free(Rr); free(dX); free(dY); free(Ux);
        return OR_ENOMEM;
    }
    const int regression = is_regression(rule), same = same_step(rule);
    /* forward, keeping every state: the same literal recurrence, one step at a time */
    if (S0) memcpy(St, S0, sizeof(double) * DD);
    for (long t = 0; t < T; ++t) {
        const double a = alpha[t];
        double *Sn = St + (size_t)(t + 1) * DD;
        for (size_t i = 0; i < DD; ++i) Sn[i] = a * St[(size_t)t * DD + i];
        double nsum = 0.0;
        for (int m = 0; m < w; ++m) {
            pair_key(X + (size_t)m * dk, k, kprev, t - m, dk, same);
            nsum += dotd(X + (size_t)m * dk, X + (size_t)m * dk, dk);
            for (int i = 0; i < dv; ++i) Y[(size_t)m * dv + i] = (t - m >= 0) ? v[(size_t)(t - m) * dv + i] : 0.0;
        }
        const double beta = step_size(eta[t], nsum, eps);
        if (regression) {
            for (int m = 0; m < w; ++m)
                for (int i = 0; i < dv; ++i)
                    Rr[(size_t)m * dv + i] = dotd(Sn + (size_t)i * dk, X + (size_t)m * dk, dk) - Y[(size_t)m * dv + i];
            for (int m = 0; m < w; ++m)
                for (int i = 0; i < dv; ++i)
                    for (int c = 0; c < dk; ++c)
                        Sn[(size_t)i * dk + c] -= beta * Rr[(size_t)m * dv + i] * X[(size_t)m * dk + c];
        } else {
            for (int m = 0; m < w; ++m)
                for (int i = 0; i < dv; ++i)
                    for (int c = 0; c < dk; ++c)
                        Sn[(size_t)i * dk + c] += beta * Y[(size_t)m * dv + i] * X[(size_t)m * dk + c];
        }
    }
    /* reverse sweep */
    memset(dq, 0, sizeof(double) * (size_t)T * dk);
    memset(dkk, 0, sizeof(double) * (size_t)T * dk);
    memset(dvv, 0, sizeof(double) * (size_t)T * dv);
    if (dkp) memset(dkp, 0, sizeof(double) * dk);
    if (dST) memcpy(U, dST, sizeof(double) * DD);
    for (long t = T - 1; t >= 0; --t) {
        const double *Sa = St + (size_t)(t + 1) * DD;   /* state after step t */
        const double *Sp = St + (size_t)t * DD;         /* state before step t */
        const double *g = dO + (size_t)t * dv;
        for (int i = 0; i < dv; ++i)
            for (int c = 0; c < dk; ++c) U[(size_t)i * dk + c] += g[i] * q[(size_t)t * dk + c];
        for (int c = 0; c < dk; ++c) {
            double acc = 0.0;
            for (int i = 0; i < dv; ++i) acc += Sa[(size_t)i * dk + c] * g[i];
            dq[(size_t)t * dk + c] = acc;
        }
        const double a = alpha[t];
        for (size_t i = 0; i < DD; ++i) Sb[i] = a * Sp[i];
        double nsum = 0.0;
        for (int m = 0; m < w; ++m) {
            pair_key(X + (size_t)m * dk, k, kprev, t - m, dk, same);
            nsum += dotd(X + (size_t)m * dk, X + (size_t)m * dk, dk);
            for (int i = 0; i < dv; ++i) Y[(size_t)m * dv + i] = (t - m >= 0) ? v[(size_t)(t - m) * dv + i] : 0.0;
        }
        const double den = nsum + eps;
        const double beta = step_size(eta[t], nsum, eps);
        memset(dX, 0, sizeof(double) * (size_t)w * dk);
        memset(dY, 0, sizeof(double) * (size_t)w * dv);
        memcpy(dSb, U, sizeof(double) * DD);
        double dbeta = 0.0;
        for (int m = 0; m < w; ++m) {
            const double *x = X + (size_t)m * dk, *y = Y + (size_t)m * dv;
            for (int i = 0; i < dv; ++i) Ux[i] = dotd(U + (size_t)i * dk, x, dk);   /* U x_j */
            if (regression) {
                double *r = Rr + (size_t)m * dv;
                for (int i = 0; i < dv; ++i) r[i] = dotd(Sb + (size_t)i * dk, x, dk) - y[i];
                for (int i = 0; i < dv; ++i) dbeta -= r[i] * Ux[i];
                for (int i = 0; i < dv; ++i) {
                    const double dr = -beta * Ux[i];
                    dY[(size_t)m * dv + i] = -dr;
                    for (int c = 0; c < dk; ++c) {
                        dSb[(size_t)i * dk + c] += dr * x[c];
                        dX[(size_t)m * dk + c] += -beta * U[(size_t)i * dk + c] * r[i] + Sb[(size_t)i * dk + c] * dr;
                    }
                }
            } else {
                for (int i = 0; i < dv; ++i) dbeta += y[i] * Ux[i];
                for (int i = 0; i < dv; ++i) {
                    dY[(size_t)m * dv + i] = beta * Ux[i];
                    for (int c = 0; c < dk; ++c) dX[(size_t)m * dk + c] += beta * U[(size_t)i * dk + c] * y[i];
                }
            }
        }
        if (den > 0.0) {
            det[t] = dbeta / den;
            const double dN = -dbeta * beta / den;
            for (int m = 0; m < w; ++m)
                for (int c = 0; c < dk; ++c) dX[(size_t)m * dk + c] += 2.0 * dN * X[(size_t)m * dk + c];
        } else {
            det[t] = 0.0;
        }
        double da = 0.0;
        for (size_t i = 0; i < DD; ++i) da += dSb[i] * Sp[i];
        dal[t] = da;
        for (size_t i = 0; i < DD; ++i) U[i] = a * dSb[i];
        /* scatter through the pairing: x_j = k_{j-1} (k_prev for j = 0), or k_j with the flag */
        for (int m = 0; m < w; ++m) {
            const long j = t - m;
            if (j < 0) continue;
            for (int i = 0; i < dv; ++i) dvv[(size_t)j * dv + i] += dY[(size_t)m * dv + i];
            double *dst = NULL;
            if (same) dst = dkk + (size_t)j * dk;
            else if (j >= 1) dst = dkk + (size_t)(j - 1) * dk;
            else if (kprev && dkp) dst = dkp;
            if (dst)
                for (int c = 0; c < dk; ++c) dst[c] += dX[(size_t)m * dk + c];
        }
    }
    if (dS0) memcpy(dS0, U, sizeof(double) * DD);
    free(St); free(U); free(Sb); free(dSb); free(X); free(Y); free(Rr); free(dX); free(dY); free(Ux);
    return OR_OK;
}

/* Gradients of the recurrent form for every head (threads = OpenMP threads over (b,h)). dO must be
 * given; dST, S0, k_prev, dS0 and dkprev may be NULL. */
int falcon_oracle_backward(int rule, int B, int H, int T, int dk, int dv, const double *q,
                           const double *k, const double *v, const double *alpha, const double *eta,
                           double eps, int window, const double *S0, const double *k_prev,
                           const double *dO, const double *dST, double *dq, double *dk_out,
                           double *dv_out, double *dalpha, double *deta, double *dS0, double *dkprev,
                           int threads) {
    if (!check_args(rule, B, H, T, dk, dv, window, q, k, v, alpha, eta)) return OR_EINVAL;
    if ((size_t)B * H * T > 0 && (!dO || !dq || !dk_out || !dv_out || !dalpha || !deta)) return OR_EINVAL;
    const long BH = (long)B * H;
    const int w = eff_window(rule, window);
    int status = OR_OK;
    if (threads < 1) threads = 1;
#ifdef _OPENMP
#pragma omp parallel for schedule(dynamic, 1) num_threads(threads)
#endif
    for (long bh = 0; bh < BH; ++bh) {
        const size_t TT = (size_t)T, DD = (size_t)dv * dk;
        const int rc = backward_head(rule, T, dk, dv, q + bh * TT * dk, k + bh * TT * dk, v + bh * TT * dv,
                                     alpha + bh * TT, eta + bh * TT, eps, w, S0 ? S0 + bh * DD : NULL,
                                     k_prev ? k_prev + bh * dk : NULL, dO + bh * TT * dv,
                                     dST ? dST + bh * DD : NULL, dq + bh * TT * dk, dk_out + bh * TT * dk,
                                     dv_out + bh * TT * dv, dalpha + bh * TT, deta + bh * TT,
                                     dS0 ? dS0 + bh * DD : NULL, dkprev ? dkprev + bh * dk : NULL);
        if (rc != OR_OK) {
#ifdef _OPENMP
#pragma omp atomic write
#endif
            status = rc;
        }
    }
    return status;
}

int falcon_oracle_max_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
