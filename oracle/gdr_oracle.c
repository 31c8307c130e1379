/*
 * Gated delta-rule oracle: a plain, slow, fp64, token-by-token CPU recurrence.
 *
 * TEST INFRASTRUCTURE ONLY.  This file is the arithmetic that the CUDA path is
 * checked against.  It shares no code, header, constant or helper with the
 * CUDA library; only tests, the package's smoke check and the benchmark's CPU
 * baseline load it.  Nothing on the product path may call it.
 *
 * What it computes, per (batch, head), starting from S_0 (zeros or given):
 *
 *   for t = 0 .. T-1:
 *     S~   = Diag(g_t) S_{t-1}                        decay of the previous state
 *     x_t  = S~^T k_t                                 readout at the key
 *     S_t  = S~ - a_t x_t^T + c_t v_t^T               erase, then write
 *     o_t  = S_t^T (scale * q_t)                      readout after the update
 *
 * with, per variant,
 *   DeltaNet       g_t = 1,                   a_t = c_t = beta_t k_t
 *   Gated DeltaNet g_t = alpha_t (scalar),    a_t = c_t = beta_t k_t
 *   KDA            g_t in R^{d_k},            a_t = c_t = beta_t k_t
 *   KLA            g_t = alpha_t (scalar),    a_t = c_t = beta_t k_t,
 *                  beta_t = eta_t / (||k_t||^2 + eps)
 *   GDN-2          g_t in R^{d_k},            a_t = b_t (.) k_t,  c_t = w_t (.) k_t
 *
 * Sources:
 *  - "Kaczmarz Linear Attention" (gist.science/ja/paper/2605.08587), sections
 *    "problem definition", "theoretical derivation" and "KLA update rule": the
 *    decayed state S~, the residual e_t = v_t - S~^T k_t, the update
 *    S_t = S~ + beta_t k_t e_t^T and beta_t = eta_t / (||k_t||_2^2 + eps).
 *    For a_t = c_t the form above is exactly that update, and the a = c
 *    variants are written in that residual form below.
 *  - "Gated DeltaNet-2: Decoupling Erase and Write in Linear Attention"
 *    (ai-auto-bdv.pages.dev/blog/arxiv-260522791/), sections "what is new"
 *    and "technical core": the delta rule subtracts the current readout
 *    before writing; KDA makes the decay channel-wise; GDN-2 gives the erase
 *    (key side) and the write separate channel-wise gates b_t and w_t, and
 *    reduces to KDA when both gates are the same scalar.  Reading used here
 *    (that page prints only a garbled paraphrase): S_t = (I - (b_t.k_t) k_t^T)
 *    Diag(g_t) S_{t-1} + (w_t.k_t) v_t^T.
 *  - The decay acts on the d_k rows of S and the readout uses the state after
 *    the update at t; the pages leave both open and these are the readings.
 *
 * Layouts (row-major, contiguous):
 *   q, k   [B, T, H, dk]      v, o  [B, T, H, dv]
 *   beta   [B, T, H]  (beta_t, or eta_t for KLA; unused by GDN-2)
 *   log_g  [B, T, H]  for GDN / KLA,  [B, T, H, dk] for KDA / GDN-2,
 *          unused by DeltaNet.  g_t = exp(log_g).
 *   erase_b, write_w  [B, T, H, dk]   (GDN-2 only)
 *   state  [B, H, dk, dv]
 *
 * oracle_backward gives the gradients of the same recurrence with respect to
 * every input (reverse mode, the forward's steps taken backwards); it is pinned
 * by finite differences of oracle_forward.
 *
 * Mutants: building with -DORACLE_MUTANT=n plants one plausible mistake so
 * that the CPU tests can show that their pins catch it (1-7 in the forward,
 * 8-10 in the backward).  The default build (no define) is the oracle.
 */
#include <math.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#ifndef ORACLE_MUTANT
#define ORACLE_MUTANT 0
#endif

/* Variant names are passed as small integers by the Python wrapper. */
enum { OR_DELTANET = 0, OR_GDN = 1, OR_KDA = 2, OR_GDN2 = 3, OR_KLA = 4 };

static int scalar_decay(int variant) { return variant == OR_GDN || variant == OR_KLA; }
static int channel_decay(int variant) { return variant == OR_KDA || variant == OR_GDN2; }

static void oracle_decay(int variant, int dk, int dv, double *S, const double *log_g)
{
    int i, j;
    if (scalar_decay(variant)) {
        double g = exp(log_g[0]);
        for (i = 0; i < dk * dv; ++i) S[i] *= g;
    } else if (channel_decay(variant)) {
        for (i = 0; i < dk; ++i) {
            double g = exp(log_g[i]);
            for (j = 0; j < dv; ++j) S[i * dv + j] *= g;
        }
    }
}

static void oracle_readout(int dk, int dv, const double *S, const double *k, double *x)
{
    int i, j;
    for (j = 0; j < dv; ++j) {
        double acc = 0.0;
        for (i = 0; i < dk; ++i) {
#if ORACLE_MUTANT == 3
            acc += S[j * dv + i] * k[i];          /* mutant: transposed state */
#else
            acc += S[i * dv + j] * k[i];
#endif
        }
        x[j] = acc;
    }
}

/*
 * One token of the recurrence on one (batch, head) state S [dk][dv], in place.
 * q, k: dk values; v: dv values; beta: one value; log_g: 1 or dk values (or
 * NULL); b, w: dk values (GDN-2).  Writes o (dv values).  x and work are
 * scratch of dv and dk doubles.
 */
static void oracle_token(int variant, int dk, int dv, double *S,
                         const double *q, const double *k, const double *v,
                         double beta, const double *log_g,
                         const double *b, const double *w,
                         double eps, double scale, double *o,
                         double *x, double *work)
{
    int i, j;

#if ORACLE_MUTANT == 2
    /* mutant: readout taken before the decay */
    oracle_readout(dk, dv, S, k, x);
#endif
#if ORACLE_MUTANT != 7
    /* 1. decay: S~ = Diag(g_t) S_{t-1} */
    oracle_decay(variant, dk, dv, S, log_g);
#endif
#if ORACLE_MUTANT != 2
    /* 2. readout at the key: x = S~^T k */
    oracle_readout(dk, dv, S, k, x);
#endif
#if ORACLE_MUTANT == 4
    /* mutant: readout of the state before the write (o = S~^T q) */
    for (j = 0; j < dv; ++j) {
        double acc = 0.0;
        for (i = 0; i < dk; ++i) acc += S[i * dv + j] * q[i];
        o[j] = scale * acc;
    }
#endif
    if (variant == OR_GDN2) {
        /* 3'. separate erase and write: S = S~ - (b.k) x^T + (w.k) v^T */
        for (i = 0; i < dk; ++i) {
            double ai = b[i] * k[i];
            double ci = w[i] * k[i];
#if ORACLE_MUTANT == 6
            ai = w[i] * k[i];                      /* mutant: gates swapped */
            ci = b[i] * k[i];
#endif
            for (j = 0; j < dv; ++j)
                S[i * dv + j] += -ai * x[j] + ci * v[j];
        }
    } else {
        /* 3. step size: beta_t, or the Kaczmarz step eta_t / (||k||^2 + eps) */
        double step = beta;
        if (variant == OR_KLA) {
            double nk = 0.0;
            for (i = 0; i < dk; ++i) nk += k[i] * k[i];
#if ORACLE_MUTANT == 5
            step = beta / (sqrt(nk) + eps);        /* mutant: norm, not squared norm */
#else
            step = beta / (nk + eps);
#endif
        }
        /* 4. residual and rank-one write: S = S~ + step * k (v - x)^T */
        for (j = 0; j < dv; ++j) {
#if ORACLE_MUTANT == 1
            work[j] = v[j] + x[j];                 /* mutant: wrong sign of the readout */
#else
            work[j] = v[j] - x[j];
#endif
        }
        for (i = 0; i < dk; ++i) {
            double ai = step * k[i];
            for (j = 0; j < dv; ++j) S[i * dv + j] += ai * work[j];
        }
    }

#if ORACLE_MUTANT == 7
    /* mutant: decay applied after the write instead of before the readout */
    oracle_decay(variant, dk, dv, S, log_g);
#endif
#if ORACLE_MUTANT != 4
    /* 5. readout after the update: o = S_t^T (scale q) */
    for (j = 0; j < dv; ++j) {
        double acc = 0.0;
        for (i = 0; i < dk; ++i) acc += S[i * dv + j] * q[i];
        o[j] = scale * acc;
    }
#endif
}

static const double *gate_ptr(int variant, const double *log_g, long tok_head, int dk)
{
    if (scalar_decay(variant)) return log_g + tok_head;
    if (channel_decay(variant)) return log_g + tok_head * dk;
    return NULL;
}

/*
 * Whole-sequence forward.  Returns 0 on success, -1 on a bad argument.
 * initial_state may be NULL (zeros); final_state may be NULL.
 */
int oracle_forward(int variant, int B, int T, int H, int dk, int dv,
                   const double *q, const double *k, const double *v,
                   const double *beta, const double *log_g,
                   const double *erase_b, const double *write_w,
                   const double *initial_state, double *o, double *final_state,
                   double eps, double scale, int nthreads)
{
    long bh;
    if (B < 0 || T < 0 || H < 0 || dk <= 0 || dv <= 0) return -1;
    if (variant < OR_DELTANET || variant > OR_KLA) return -1;
    if ((scalar_decay(variant) || channel_decay(variant)) && !log_g) return -1;
    if (variant == OR_GDN2 && (!erase_b || !write_w)) return -1;
    if (variant != OR_GDN2 && !beta) return -1;
#ifdef _OPENMP
    if (nthreads > 0) omp_set_num_threads(nthreads);
#else
    (void)nthreads;
#endif

#pragma omp parallel for schedule(dynamic, 1)
    for (bh = 0; bh < (long)B * H; ++bh) {
        int b_ = (int)(bh / H), h = (int)(bh % H), t;
        double *S = (double *)malloc(sizeof(double) * (size_t)dk * dv);
        double *x = (double *)malloc(sizeof(double) * (size_t)dv);
        double *work = (double *)malloc(sizeof(double) * (size_t)(dk > dv ? dk : dv));
        if (initial_state)
            memcpy(S, initial_state + bh * (long)dk * dv, sizeof(double) * (size_t)dk * dv);
        else
            memset(S, 0, sizeof(double) * (size_t)dk * dv);
        for (t = 0; t < T; ++t) {
            long th = ((long)b_ * T + t) * H + h;          /* token-head index */
            oracle_token(variant, dk, dv, S, q + th * dk, k + th * dk, v + th * dv,
                         beta ? beta[th] : 0.0, gate_ptr(variant, log_g, th, dk),
                         erase_b ? erase_b + th * dk : NULL,
                         write_w ? write_w + th * dk : NULL,
                         eps, scale, o + th * dv, x, work);
        }
        if (final_state)
            memcpy(final_state + bh * (long)dk * dv, S, sizeof(double) * (size_t)dk * dv);
        free(S); free(x); free(work);
    }
    return 0;
}

/*
 * One decode step for N independent sequences: q, k [N, H, dk], v, o [N, H, dv],
 * beta [N, H], log_g [N, H] or [N, H, dk], erase_b / write_w [N, H, dk],
 * state [N, H, dk, dv] updated in place.
 */
int oracle_decode_step(int variant, int N, int H, int dk, int dv,
                       const double *q, const double *k, const double *v,
                       const double *beta, const double *log_g,
                       const double *erase_b, const double *write_w,
                       double *state, double *o, double eps, double scale, int nthreads)
{
    long nh;
    if (N < 0 || H < 0 || dk <= 0 || dv <= 0 || !state) return -1;
    if (variant < OR_DELTANET || variant > OR_KLA) return -1;
    if ((scalar_decay(variant) || channel_decay(variant)) && !log_g) return -1;
    if (variant == OR_GDN2 && (!erase_b || !write_w)) return -1;
    if (variant != OR_GDN2 && !beta) return -1;
#ifdef _OPENMP
    if (nthreads > 0) omp_set_num_threads(nthreads);
#else
    (void)nthreads;
#endif

#pragma omp parallel for schedule(static)
    for (nh = 0; nh < (long)N * H; ++nh) {
        double *x = (double *)malloc(sizeof(double) * (size_t)dv);
        double *work = (double *)malloc(sizeof(double) * (size_t)(dk > dv ? dk : dv));
        oracle_token(variant, dk, dv, state + nh * (long)dk * dv,
                     q + nh * dk, k + nh * dk, v + nh * dv,
                     beta ? beta[nh] : 0.0, gate_ptr(variant, log_g, nh, dk),
                     erase_b ? erase_b + nh * dk : NULL,
                     write_w ? write_w + nh * dk : NULL,
                     eps, scale, o + nh * dv, x, work);
        free(x); free(work);
    }
    return 0;
}

/*
 * Backward of the whole-sequence forward (reverse mode through the token
 * recurrence, in the forward's own steps taken backwards).  Given the
 * gradient of a loss with respect to the outputs, d_o [B,T,H,dv], and to the
 * final state, d_final [B,H,dk,dv] (NULL: zero), it writes the gradient with
 * respect to every input of oracle_forward:
 *   dq, dk [B,T,H,dk]; dv [B,T,H,dv];
 *   dbeta [B,T,H] (d/d beta_t, or d/d eta_t for KLA; not for GDN-2);
 *   dlog_g [B,T,H] or [B,T,H,dk] (not for DeltaNet);
 *   derase_b, dwrite_w [B,T,H,dk] (GDN-2 only);
 *   dinitial_state [B,H,dk,dv] (may be NULL).
 * Outputs a variant does not use may be NULL.  The states S_0 .. S_T of each
 * (batch, head) are kept (T + 1 matrices of dk x dv doubles).
 *
 * Per token t, with dS the gradient with respect to S_t on entry:
 *   o_t = S_t^T (scale q_t)    dS += scale q_t d_o_t^T,  dq_t = scale S_t d_o_t
 *   S_t = S~ - a x^T + c v^T   da = -dS x,  dc = dS v,  dv_t = dS^T c,
 *                              dx = -dS^T a,  dS~ = dS
 *   x = S~^T k                 dS~ += k dx^T,  dk_t += S~ dx
 *   S~ = Diag(g) S_{t-1}       d log g_i = g_i sum_j dS~_ij (S_{t-1})_ij (summed
 *                              over i for a scalar decay),  dS_{t-1} = Diag(g) dS~
 * then a, c back to their inputs: a = c = beta k (dbeta = k.(da + dc),
 * dk += beta (da + dc)); for KLA beta = eta / (||k||^2 + eps) adds
 * d eta = dbeta / (||k||^2 + eps) and dk -= 2 dbeta eta k / (||k||^2 + eps)^2;
 * for GDN-2 a = b.k, c = w.k (db = da.k, dw = dc.k, dk += b.da + w.dc).
 * Mutants 8-10 plant mistakes in these steps for the finite-difference pins.
 */
int oracle_backward(int variant, int B, int T, int H, int dk, int dv,
                    const double *q, const double *k, const double *v,
                    const double *beta, const double *log_g,
                    const double *erase_b, const double *write_w,
                    const double *initial_state, const double *d_o, const double *d_final,
                    double *dq, double *dkey, double *dval, double *dbeta, double *dlog_g,
                    double *derase_b, double *dwrite_w, double *dinitial_state,
                    double eps, double scale, int nthreads)
{
    long bh;
    if (B < 0 || T < 0 || H < 0 || dk <= 0 || dv <= 0 || !d_o) return -1;
    if (variant < OR_DELTANET || variant > OR_KLA) return -1;
    if ((scalar_decay(variant) || channel_decay(variant)) && !log_g) return -1;
    if (variant == OR_GDN2 && (!erase_b || !write_w)) return -1;
    if (variant != OR_GDN2 && !beta) return -1;
    if (!dq || !dkey || !dval) return -1;
#ifdef _OPENMP
    if (nthreads > 0) omp_set_num_threads(nthreads);
#else
    (void)nthreads;
#endif

#pragma omp parallel for schedule(dynamic, 1)
    for (bh = 0; bh < (long)B * H; ++bh) {
        int b_ = (int)(bh / H), h = (int)(bh % H), t, i, j;
        const size_t mat = (size_t)dk * dv;
        double *Sall = (double *)malloc(sizeof(double) * mat * (size_t)(T + 1));
        double *dS = (double *)malloc(sizeof(double) * mat);
        double *St = (double *)malloc(sizeof(double) * mat);     /* S~ of token t */
        double *x = (double *)malloc(sizeof(double) * (size_t)dv);
        double *work = (double *)malloc(sizeof(double) * (size_t)(dk > dv ? dk : dv));
        double *obuf = (double *)malloc(sizeof(double) * (size_t)dv);
        double *a = (double *)malloc(sizeof(double) * (size_t)dk);
        double *c = (double *)malloc(sizeof(double) * (size_t)dk);
        double *da = (double *)malloc(sizeof(double) * (size_t)dk);
        double *dc = (double *)malloc(sizeof(double) * (size_t)dk);
        double *dx = (double *)malloc(sizeof(double) * (size_t)dv);
        double *g = (double *)malloc(sizeof(double) * (size_t)dk);

        /* forward, keeping S_0 .. S_T */
        if (initial_state)
            memcpy(Sall, initial_state + bh * (long)mat, sizeof(double) * mat);
        else
            memset(Sall, 0, sizeof(double) * mat);
        for (t = 0; t < T; ++t) {
            long th = ((long)b_ * T + t) * H + h;
            memcpy(Sall + (size_t)(t + 1) * mat, Sall + (size_t)t * mat, sizeof(double) * mat);
            oracle_token(variant, dk, dv, Sall + (size_t)(t + 1) * mat, q + th * dk, k + th * dk, v + th * dv,
                         beta ? beta[th] : 0.0, gate_ptr(variant, log_g, th, dk),
                         erase_b ? erase_b + th * dk : NULL, write_w ? write_w + th * dk : NULL,
                         eps, scale, obuf, x, work);
        }

        /* backward */
        if (d_final)
            memcpy(dS, d_final + bh * (long)mat, sizeof(double) * mat);
        else
            memset(dS, 0, sizeof(double) * mat);
        for (t = T - 1; t >= 0; --t) {
            long th = ((long)b_ * T + t) * H + h;
            const double *qt = q + th * dk, *kt = k + th * dk, *vt = v + th * dv;
            const double *dot = d_o + th * dv;
            const double *Snew = Sall + (size_t)(t + 1) * mat, *Sprev = Sall + (size_t)t * mat;
            const double *lg = gate_ptr(variant, log_g, th, dk);
            double *dqt = dq + th * dk, *dkt = dkey + th * dk, *dvt = dval + th * dv;
            double step = 0.0, nk = 0.0, dstep = 0.0;

            /* readout o_t = S_t^T (scale q_t) */
            for (i = 0; i < dk; ++i) {
                double acc = 0.0;
                for (j = 0; j < dv; ++j) {
                    acc += Snew[i * dv + j] * dot[j];
                    dS[i * dv + j] += scale * qt[i] * dot[j];
                }
                dqt[i] = scale * acc;
            }

            /* recompute S~, x and the erase / write vectors a, c */
            for (i = 0; i < dk; ++i)
                g[i] = scalar_decay(variant) ? exp(lg[0]) : channel_decay(variant) ? exp(lg[i]) : 1.0;
            for (i = 0; i < dk; ++i)
                for (j = 0; j < dv; ++j) St[i * dv + j] = g[i] * Sprev[i * dv + j];
            oracle_readout(dk, dv, St, kt, x);
            if (variant == OR_GDN2) {
                for (i = 0; i < dk; ++i) {
                    a[i] = erase_b[th * dk + i] * kt[i];
                    c[i] = write_w[th * dk + i] * kt[i];
                }
            } else {
                step = beta[th];
                if (variant == OR_KLA) {
                    for (i = 0; i < dk; ++i) nk += kt[i] * kt[i];
                    step = beta[th] / (nk + eps);
                }
                for (i = 0; i < dk; ++i) a[i] = c[i] = step * kt[i];
            }

            /* S_t = S~ - a x^T + c v^T */
            for (i = 0; i < dk; ++i) {
                double sa = 0.0, sc = 0.0;
                for (j = 0; j < dv; ++j) {
                    sa += dS[i * dv + j] * x[j];
                    sc += dS[i * dv + j] * vt[j];
                }
                da[i] = -sa;
                dc[i] = sc;
            }
            for (j = 0; j < dv; ++j) {
                double sa = 0.0, sc = 0.0;
                for (i = 0; i < dk; ++i) {
                    sa += dS[i * dv + j] * a[i];
                    sc += dS[i * dv + j] * c[i];
                }
#if ORACLE_MUTANT == 8
                dx[j] = sa;                               /* mutant: sign of the erase term */
#else
                dx[j] = -sa;
#endif
                dvt[j] = sc;
            }
            /* dS now holds dS~; x = S~^T k adds k dx^T and gives dk its readout term */
            for (i = 0; i < dk; ++i) {
                double acc = 0.0;
                for (j = 0; j < dv; ++j) {
                    acc += St[i * dv + j] * dx[j];
                    dS[i * dv + j] += kt[i] * dx[j];
                }
#if ORACLE_MUTANT == 10
                dkt[i] = 0.0;                             /* mutant: readout term of dk dropped */
#else
                dkt[i] = acc;
#endif
            }
            /* S~ = Diag(g) S_{t-1} */
            if (scalar_decay(variant) || channel_decay(variant)) {
                double tot = 0.0;
                for (i = 0; i < dk; ++i) {
                    double acc = 0.0;
                    for (j = 0; j < dv; ++j) acc += dS[i * dv + j] * Sprev[i * dv + j];
                    if (channel_decay(variant)) {
                        if (dlog_g) dlog_g[th * dk + i] = g[i] * acc;
                    } else {
                        tot += g[i] * acc;
                    }
                }
                if (scalar_decay(variant) && dlog_g) dlog_g[th] = tot;
            }
            for (i = 0; i < dk; ++i)
                for (j = 0; j < dv; ++j) {
#if ORACLE_MUTANT == 9
                    (void)0;                              /* mutant: decay not applied to dS */
#else
                    dS[i * dv + j] *= g[i];
#endif
                }

            /* a, c back to k and the gates */
            if (variant == OR_GDN2) {
                for (i = 0; i < dk; ++i) {
                    if (derase_b) derase_b[th * dk + i] = da[i] * kt[i];
                    if (dwrite_w) dwrite_w[th * dk + i] = dc[i] * kt[i];
                    dkt[i] += erase_b[th * dk + i] * da[i] + write_w[th * dk + i] * dc[i];
                }
            } else {
                for (i = 0; i < dk; ++i) {
                    dstep += kt[i] * (da[i] + dc[i]);
                    dkt[i] += step * (da[i] + dc[i]);
                }
                if (variant == OR_KLA) {
                    double den = nk + eps;
                    if (dbeta) dbeta[th] = dstep / den;
                    for (i = 0; i < dk; ++i) dkt[i] -= 2.0 * dstep * beta[th] * kt[i] / (den * den);
                } else if (dbeta) {
                    dbeta[th] = dstep;
                }
            }
        }
        if (dinitial_state) memcpy(dinitial_state + bh * (long)mat, dS, sizeof(double) * mat);
        free(Sall); free(dS); free(St); free(x); free(work); free(obuf);
        free(a); free(c); free(da); free(dc); free(dx); free(g);
    }
    return 0;
}

/* Threads an OpenMP region would use (1 when built without OpenMP). */
int oracle_max_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
