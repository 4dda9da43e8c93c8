/*
 * Plain, slow fp64 CPU oracle of the gated delta-rule decode step.
 *
 * TEST INFRASTRUCTURE ONLY. Nothing in the product path may call this; only
 * the tests, the smoke check and the benchmark's CPU-baseline leg load it.
 * It shares no code, header or constant with the CUDA library.
 *
 * What it computes (the method of "DeltaLog: Deferred Materialization of
 * Recurrent States for Linear Attention Decoding", Technical Summary):
 *
 *   Per (sequence, head) the recurrent state S is a d_v x d_k matrix (stored
 *   row-major, the key index contiguous). One decode step with inputs
 *   q, k in R^{d_k}, v in R^{d_v}, scalar beta, and decay a (one scalar per
 *   head for Gated DeltaNet, one value per key channel for Kimi Delta
 *   Attention; section "Kernel Implementation", operator list) is
 *
 *       S_t = S_{t-1} Diag(a_t) (I - beta_t k_t k_t^T) + beta_t v_t k_t^T
 *       o_t = S_t q_t
 *
 *   i.e. decay, then the delta-rule correction that subtracts the current
 *   read S k before writing the new value v.
 *
 *   RWKV6, the page's third model (per-key decay, "raw-value updates" with
 *   no delta-rule correction, "Kernel Implementation"), is read as
 *
 *       S_t = S_{t-1} Diag(a_t) + v_t k_t^T,    o_t = S_t q_t
 *
 *   (no beta; RWKV6's "bonus" term is not given by the pages and is left out).
 *   `kind` selects the rule: 0 head-wise decay (GDN), 1 channel-wise decay
 *   (KDA), 2 RWKV6.
 *
 * Three forms:
 *   oracle_eager     -- the definition, one step at a time (the "eager"
 *                       schedule of section "Problem: The State-Update Tax").
 *   oracle_deferred  -- the DeltaLog schedule (section "Methodology", "Core
 *                       Mechanism: Base + Log"): a dense base S_bar that is
 *                       not written between merges, a bounded log of the raw
 *                       per-step factors, outputs read from base + log, and a
 *                       merge of the whole log into the base when the log
 *                       holds L entries and once more at the end.
 *   (the third form, dense brute-force matrix products, is in oracle/__init__.py)
 *
 * Heads are independent; OpenMP runs one head per thread with the time loop
 * inside, so a head's state stays in the thread's cache.
 *
 * Array layouts (fp64, row-major): NH = number of heads (a flattened [B, H]).
 *   S     [NH, d_v, d_k]          in: S_0, out: S_T (deferred: after the final merge)
 *   q, k  [T, NH, d_k]
 *   v     [T, NH, d_v]
 *   beta  [T, NH]
 *   a     [T, NH]  (head-wise decay)  or  [T, NH, d_k]  (channel-wise decay, RWKV6)
 *   beta  is not read for RWKV6
 *   o     [T, NH, d_v]             out
 */
#include <math.h>
#include <stdlib.h>
#include <string.h>

/* decay value of channel j at step t for head h */
static double decay_at(const double *a, int kind, long NH, int dk,
                       int t, long h, int j)
{
    if (kind != 0)
        return a[((long)t * NH + h) * dk + j];
    return a[(long)t * NH + h];
}

/* ------------------------------------------------------------------ eager */

/* One eager step on one head's state (the definition, expanded):
 *   1. S'[i][j] = S[i][j] * a_j                      (S_{t-1} Diag(a))
 *   2. u_i      = sum_j S'[i][j] k_j                   (S' k)
 *   3. S[i][j]  = S'[i][j] + beta (v_i - u_i) k_j      (S'(I - beta k k^T) + beta v k^T)
 *   4. o_i      = sum_j S[i][j] q_j                    (S_t q), from the updated S
 * RWKV6 (delta = 0) replaces step 3 by S[i][j] = S'[i][j] + v_i k_j.
 */
static void eager_head_step(double *S, int dk, int dv, int delta,
                            const double *q, const double *k, const double *v,
                            double beta, const double *avec, double *o)
{
    for (int i = 0; i < dv; ++i) {
        double *row = S + (long)i * dk;
        for (int j = 0; j < dk; ++j)
            row[j] = row[j] * avec[j];
        double u = 0.0;
        for (int j = 0; j < dk; ++j)
            u += row[j] * k[j];
        double coef = delta ? beta * (v[i] - u) : v[i];
        for (int j = 0; j < dk; ++j)
            row[j] = row[j] + coef * k[j];
        double acc = 0.0;
        for (int j = 0; j < dk; ++j)
            acc += row[j] * q[j];
        o[i] = acc;
    }
}

void oracle_eager(long NH, int T, int dk, int dv, int kind,
                  double *S, const double *q, const double *k, const double *v,
                  const double *beta, const double *a, double *o)
{
    const int delta = kind != 2;
#pragma omp parallel for schedule(dynamic, 1)
    for (long h = 0; h < NH; ++h) {
        double *Sh = S + h * (long)dv * dk;
        double *avec = (double *)malloc(sizeof(double) * (size_t)dk);
        for (int t = 0; t < T; ++t) {
            for (int j = 0; j < dk; ++j)
                avec[j] = decay_at(a, kind, NH, dk, t, h, j);
            eager_head_step(Sh, dk, dv, delta,
                            q + ((long)t * NH + h) * dk,
                            k + ((long)t * NH + h) * dk,
                            v + ((long)t * NH + h) * dv,
                            delta ? beta[(long)t * NH + h] : 0.0, avec,
                            o + ((long)t * NH + h) * dv);
        }
        free(avec);
    }
}

/* --------------------------------------------------------------- deferred */

/* One head's bounded log: n entries of the raw step factors (k, v, beta, a),
 * the decay always held as a d_k vector (a head-wise decay is repeated). */
typedef struct {
    int cap, n, dk, dv;
    int delta;    /* 1: delta rule (GDN, KDA); 0: RWKV6 */
    double *k;    /* [cap, dk] */
    double *v;    /* [cap, dv] */
    double *beta; /* [cap]     */
    double *a;    /* [cap, dk] */
} head_log;

/* Deferred read of o = S_n q without forming S_n (the log holds entries
 * 1..n, stored at 0..n-1). With A_i = Diag(a_i)(I - beta_i k_i k_i^T),
 *
 *   S_n = S_bar A_1 ... A_n + sum_i beta_i v_i k_i^T A_{i+1} ... A_n,
 *
 * so  o = S_bar x_0 + sum_i s_i v_i  where x_n = q and, for i = n..1,
 *   c_i = k_i . x_i,  s_i = beta_i c_i,  x_{i-1} = A_i x_i = a_i o (x_i - s_i k_i).
 * (A product of Householder-like factors applied to q from the right end.)
 * RWKV6 has A_i = Diag(a_i) and adds v_i k_i^T unscaled: s_i = c_i and
 * x_{i-1} = a_i o x_i.
 */
static void deferred_read(const double *Sbar, const head_log *lg,
                          const double *q, double *o, double *x, double *s)
{
    const int dk = lg->dk, dv = lg->dv;
    for (int j = 0; j < dk; ++j)
        x[j] = q[j];
    for (int i = lg->n - 1; i >= 0; --i) {
        const double *ki = lg->k + (long)i * dk;
        const double *ai = lg->a + (long)i * dk;
        double c = 0.0;
        for (int j = 0; j < dk; ++j)
            c += ki[j] * x[j];
        if (lg->delta) {
            s[i] = lg->beta[i] * c;
            for (int j = 0; j < dk; ++j)
                x[j] = ai[j] * (x[j] - s[i] * ki[j]);
        } else {
            s[i] = c;
            for (int j = 0; j < dk; ++j)
                x[j] = ai[j] * x[j];
        }
    }
    for (int r = 0; r < dv; ++r) {
        const double *row = Sbar + (long)r * dk;
        double acc = 0.0;
        for (int j = 0; j < dk; ++j)
            acc += row[j] * x[j];
        for (int i = 0; i < lg->n; ++i)
            acc += s[i] * lg->v[(long)i * dv + r];
        o[r] = acc;
    }
}

/* Merge of the n log entries into the base, in the log-decay form (the
 * page's "log-decay metadata": Lambda_i = sum_{m<=i} log a_m per channel).
 * Write D(i, j) = exp(Lambda_i - Lambda_j) = prod_{m=j+1..i} a_m (computed as
 * that product, so a zero decay needs no logarithm), gamma_i = D(i, 0).
 * For each row s_bar of the base, the rows s_i of the replayed states are
 *
 *   s_i = s_bar o gamma_i + sum_{j<=i} delta_j (k_j o D(i, j)),
 *
 * with the per-row scalars delta_i = beta_i (v_i[r] - u_i) and the read
 *   u_i = s_{i-1} . (a_i o k_i) = G_i + sum_{j<i} C(i, j) delta_j,
 *   G_i = s_bar . (gamma_i o k_i),  C(i, j) = sum_c k_j[c] D(i, j)[c] k_i[c],
 *
 * found by forward substitution in i; then s_bar <- s_n. The log empties.
 * RWKV6 adds each value unscaled and uncorrected: delta_i = v_i[r].
 */
static void deferred_merge(double *Sbar, head_log *lg)
{
    const int dk = lg->dk, dv = lg->dv, n = lg->n;
    if (n == 0)
        return;
    /* D(i, j) for 0 <= j <= i <= n, as vectors; index i, j are 1-based entries,
     * j = 0 means "from the base" (gamma). Stored densely [n+1][n+1][dk]. */
    double *D = (double *)calloc((size_t)(n + 1) * (n + 1) * dk, sizeof(double));
    for (int j = 0; j <= n; ++j) {
        double *Djj = D + ((long)j * (n + 1) + j) * dk;
        for (int c = 0; c < dk; ++c)
            Djj[c] = 1.0;
        for (int i = j + 1; i <= n; ++i) {
            const double *prev = D + ((long)(i - 1) * (n + 1) + j) * dk;
            double *cur = D + ((long)i * (n + 1) + j) * dk;
            const double *ai = lg->a + (long)(i - 1) * dk; /* entry i is stored at i-1 */
            for (int c = 0; c < dk; ++c)
                cur[c] = prev[c] * ai[c];
        }
    }
#define DV(i, j) (D + ((long)(i) * (n + 1) + (j)) * dk)
#define KE(i) (lg->k + (long)((i) - 1) * dk)
    /* C(i, j) for 1 <= j < i <= n */
    double *C = (double *)calloc((size_t)(n + 1) * (n + 1), sizeof(double));
    for (int i = 1; i <= n; ++i)
        for (int j = 1; j < i; ++j) {
            double acc = 0.0;
            const double *dij = DV(i, j), *ki = KE(i), *kj = KE(j);
            for (int c = 0; c < dk; ++c)
                acc += kj[c] * dij[c] * ki[c];
            C[i * (n + 1) + j] = acc;
        }
    double *delta = (double *)malloc(sizeof(double) * (size_t)(n + 1));
    double *newrow = (double *)malloc(sizeof(double) * (size_t)dk);
    for (int r = 0; r < dv; ++r) {
        double *row = Sbar + (long)r * dk;
        for (int i = 1; i <= n; ++i) {
            if (!lg->delta) {
                delta[i] = lg->v[(long)(i - 1) * dv + r];
                continue;
            }
            const double *gi = DV(i, 0), *ki = KE(i);
            double G = 0.0;
            for (int c = 0; c < dk; ++c)
                G += row[c] * gi[c] * ki[c];
            double u = G;
            for (int j = 1; j < i; ++j)
                u += C[i * (n + 1) + j] * delta[j];
            delta[i] = lg->beta[i - 1] * (lg->v[(long)(i - 1) * dv + r] - u);
        }
        const double *gn = DV(n, 0);
        for (int c = 0; c < dk; ++c)
            newrow[c] = row[c] * gn[c];
        for (int j = 1; j <= n; ++j) {
            const double *dnj = DV(n, j), *kj = KE(j);
            for (int c = 0; c < dk; ++c)
                newrow[c] += delta[j] * kj[c] * dnj[c];
        }
        memcpy(row, newrow, sizeof(double) * (size_t)dk);
    }
#undef DV
#undef KE
    free(newrow);
    free(delta);
    free(C);
    free(D);
    lg->n = 0;
}

/* The DeltaLog schedule with log capacity L. Per step: append (k, v, beta, a)
 * as entry n+1 (the base is not written), read o from base + log; when the
 * log holds L entries, merge it into the base and empty it. After the last
 * step any remaining entries are merged, so S returns S_T. */
void oracle_deferred(long NH, int T, int dk, int dv, int kind, int L,
                     double *S, const double *q, const double *k, const double *v,
                     const double *beta, const double *a, double *o)
{
#pragma omp parallel for schedule(dynamic, 1)
    for (long h = 0; h < NH; ++h) {
        double *Sbar = S + h * (long)dv * dk;
        head_log lg;
        lg.cap = L; lg.n = 0; lg.dk = dk; lg.dv = dv; lg.delta = kind != 2;
        lg.k = (double *)malloc(sizeof(double) * (size_t)L * dk);
        lg.v = (double *)malloc(sizeof(double) * (size_t)L * dv);
        lg.beta = (double *)malloc(sizeof(double) * (size_t)L);
        lg.a = (double *)malloc(sizeof(double) * (size_t)L * dk);
        double *x = (double *)malloc(sizeof(double) * (size_t)dk);
        double *s = (double *)malloc(sizeof(double) * (size_t)L);
        for (int t = 0; t < T; ++t) {
            int e = lg.n;
            memcpy(lg.k + (long)e * dk, k + ((long)t * NH + h) * dk, sizeof(double) * (size_t)dk);
            memcpy(lg.v + (long)e * dv, v + ((long)t * NH + h) * dv, sizeof(double) * (size_t)dv);
            lg.beta[e] = lg.delta ? beta[(long)t * NH + h] : 0.0;
            for (int j = 0; j < dk; ++j)
                lg.a[(long)e * dk + j] = decay_at(a, kind, NH, dk, t, h, j);
            lg.n = e + 1;
            deferred_read(Sbar, &lg, q + ((long)t * NH + h) * dk,
                          o + ((long)t * NH + h) * dv, x, s);
            if (lg.n == L)
                deferred_merge(Sbar, &lg);
        }
        deferred_merge(Sbar, &lg);
        free(s); free(x);
        free(lg.a); free(lg.beta); free(lg.v); free(lg.k);
    }
}

/* ----------------------------------------------------- int8 deferred base */

/* Quantisation of a base held in int8 with one scale per state row (a value
 * channel): scale = max_c |row_c| / 127 and code_c = the nearest integer to
 * row_c / scale (ties to even, clamped to [-127, 127]), so that row_c becomes
 * code_c * scale; a row whose largest magnitude is zero becomes zero. (The
 * low-precision base of the DAMP abstract, "Decay-Aware Mixed-Precision
 * Recurrent-State Quantization", which stores recurrent states in INT8: with
 * the deferred schedule the base is written, and so rounded, only when a merge
 * writes it.)
 *
 * The pages fix no precision for this rounding, so it is taken in fp32, the
 * precision of the kernel that stores the base: the row is first taken to fp32,
 * and the maximum, the scale, each quotient and each code * scale are single
 * correctly rounded fp32 operations (this file is built with -ffp-contract=off,
 * so none is fused). A value then takes the same code on both sides whenever
 * both hold the same fp32 value. */
static void quantize_rows_i8(double *S, int dv, int dk)
{
    for (int r = 0; r < dv; ++r) {
        double *row = S + (long)r * dk;
        float m = 0.0f;
        for (int c = 0; c < dk; ++c)
            if (fabsf((float)row[c]) > m)
                m = fabsf((float)row[c]);
        const float scale = m / 127.0f;
        for (int c = 0; c < dk; ++c) {
            float code = 0.0f;
            if (scale != 0.0f) {
                code = nearbyintf((float)row[c] / scale);
                if (code > 127.0f) code = 127.0f;
                if (code < -127.0f) code = -127.0f;
            }
            row[c] = (double)(code * scale);
        }
    }
}

/* oracle_deferred with an int8 base: the initial base is quantised, and so is
 * the base after every merge (the final one included); reads use the base as
 * stored plus the exact log. */
void oracle_deferred_i8(long NH, int T, int dk, int dv, int kind, int L,
                        double *S, const double *q, const double *k, const double *v,
                        const double *beta, const double *a, double *o)
{
#pragma omp parallel for schedule(dynamic, 1)
    for (long h = 0; h < NH; ++h) {
        double *Sbar = S + h * (long)dv * dk;
        head_log lg;
        lg.cap = L; lg.n = 0; lg.dk = dk; lg.dv = dv; lg.delta = kind != 2;
        lg.k = (double *)malloc(sizeof(double) * (size_t)L * dk);
        lg.v = (double *)malloc(sizeof(double) * (size_t)L * dv);
        lg.beta = (double *)malloc(sizeof(double) * (size_t)L);
        lg.a = (double *)malloc(sizeof(double) * (size_t)L * dk);
        double *x = (double *)malloc(sizeof(double) * (size_t)dk);
        double *s = (double *)malloc(sizeof(double) * (size_t)L);
        quantize_rows_i8(Sbar, dv, dk);
        for (int t = 0; t < T; ++t) {
            int e = lg.n;
            memcpy(lg.k + (long)e * dk, k + ((long)t * NH + h) * dk, sizeof(double) * (size_t)dk);
            memcpy(lg.v + (long)e * dv, v + ((long)t * NH + h) * dv, sizeof(double) * (size_t)dv);
            lg.beta[e] = lg.delta ? beta[(long)t * NH + h] : 0.0;
            for (int j = 0; j < dk; ++j)
                lg.a[(long)e * dk + j] = decay_at(a, kind, NH, dk, t, h, j);
            lg.n = e + 1;
            deferred_read(Sbar, &lg, q + ((long)t * NH + h) * dk,
                          o + ((long)t * NH + h) * dv, x, s);
            if (lg.n == L) {
                deferred_merge(Sbar, &lg);
                quantize_rows_i8(Sbar, dv, dk);
            }
        }
        if (lg.n) {
            deferred_merge(Sbar, &lg);
            quantize_rows_i8(Sbar, dv, dk);
        }
        free(s); free(x);
        free(lg.a); free(lg.beta); free(lg.v); free(lg.k);
    }
}

/* The quantisation alone, for the tests: NH heads of d_v x d_k in place. */
void oracle_quantize_i8(long NH, int dk, int dv, double *S)
{
    for (long h = 0; h < NH; ++h)
        quantize_rows_i8(S + h * (long)dv * dk, dv, dk);
}

/* Version tag so the Python side can tell a stale build. */
int oracle_abi_version(void) { return 3; }
