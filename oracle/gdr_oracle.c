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
 * Mutants: building with -DORACLE_MUTANT=n plants one plausible mistake so
 * that the CPU tests can show that their pins catch it.  The default build
 * (no define) is the oracle.
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

/* Threads an OpenMP region would use (1 when built without OpenMP). */
int oracle_max_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
