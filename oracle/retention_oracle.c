/*
 * retention_oracle.c -- plain, slow fp64 CPU oracle for multi-scale retention.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path may include, link,
 * load or call this file.  Only the test suite, the smoke check of the entry
 * module and the CPU-baseline leg of the benchmark use it.  It shares no code
 * with the CUDA library: it has its own rotation, decay and normalisation, all
 * in double precision with the C library's cos, sin and pow.
 *
 * Sources (cited by page title and section):
 *   [RetNet summary]  "Retentive Network: A Successor to Transformer for Large
 *                     Language Models" paper summary (blog.csdn.net article
 *                     132817411), section 2.1 "Retention" and 2.2 "Gated
 *                     Multi-Scale Retention".
 *   [Dual-mode manual] "RetNet dual-mode hands-on manual" (lanjinlin.com.cn
 *                     news 2041318), section 3.1 (parallel/recurrent
 *                     equivalence) and 3.2 (recurrent inference wrapper).
 *
 * Layouts (all contiguous, row-major, double):
 *   Q, K   [B][H][L][dk]      V, O   [B][H][L][dv]
 *   G, Y   [B][L][H*dv]       state  [B][H][dk][dv]
 * Row t of a (b,h) slice sits at absolute position pos_offset + t.  The
 * state passed in is S after absorbing every token before pos_offset.
 */
#include <math.h>
#include <pthread.h>
#include <stdlib.h>
#include <string.h>
#include <unistd.h>

typedef struct {
    int B, H, L, dk, dv;
    const double *gamma;   /* [H] decay per head                          */
    int rotate;            /* 1: apply the xPos rotation e^{i n theta}      */
    double theta_base;     /* theta_j = theta_base^(-2j/dk)                */
    long long pos_offset;  /* absolute position of row 0                   */
    int nthreads;          /* 0: one thread per online core                */
} oracle_problem;

/* ------------------------------------------------------------------ */
/* [RetNet summary] 2.2: gamma = 1 - 2^(-5-arange(0,h)), one per head. */
void oracle_msr_gammas(int H, double *gamma)
{
    for (int h = 0; h < H; ++h)
        gamma[h] = 1.0 - pow(2.0, -5.0 - (double)h);
}

/* [RetNet summary] 2.1, the scalar-gamma form o_n = sum gamma^{n-m}
 * (Q_n e^{in theta})(K_m e^{im theta})^dagger v_m.  A real row of even
 * width d is read as d/2 complex numbers z_j = x[2j] + i x[2j+1]; the factor
 * e^{i pos theta_j} multiplies z_j, theta_j = base^(-2j/d).  Both Q and K are
 * turned by their own position with the same sign, so the real part of
 * q^ conj(k^) -- the dot product of the rotated real rows -- depends only on
 * n - m. */
void oracle_xpos_rotate(const double *x, int d, double pos, double theta_base,
                        double *out)
{
    for (int j = 0; j < d / 2; ++j) {
        double theta = pow(theta_base, -2.0 * (double)j / (double)d);
        double c = cos(pos * theta), s = sin(pos * theta);
        double re = x[2 * j], im = x[2 * j + 1];
        out[2 * j] = re * c - im * s;
        out[2 * j + 1] = re * s + im * c;
    }
    if (d & 1) out[d - 1] = x[d - 1];
}

static double *rotated_copy(const oracle_problem *p, const double *x, int d)
{
    double *r = (double *)malloc(sizeof(double) * (size_t)p->L * (size_t)d);
    if (!r) return NULL;
    for (int t = 0; t < p->L; ++t) {
        if (p->rotate)
            oracle_xpos_rotate(x + (size_t)t * d, d,
                               (double)(p->pos_offset + t), p->theta_base,
                               r + (size_t)t * d);
        else
            memcpy(r + (size_t)t * d, x + (size_t)t * d, sizeof(double) * d);
    }
    return r;
}

static double dot(const double *a, const double *b, int n)
{
    double s = 0.0;
    for (int i = 0; i < n; ++i) s += a[i] * b[i];
    return s;
}

/* ------------------------------------------------------------------ */
/* A tiny work queue over the independent (b, h) slices.               */
typedef struct {
    const oracle_problem *p;
    int chunk;
    const double *Q, *K, *V, *state_in;
    double *state_out, *O;
    int (*fn)(const oracle_problem *, int, int, int, const double *,
              const double *, const double *, const double *, double *,
              double *);
    int next, err;
    pthread_mutex_t mu;
} pool;

static void *pool_worker(void *arg)
{
    pool *w = (pool *)arg;
    const oracle_problem *p = w->p;
    for (;;) {
        pthread_mutex_lock(&w->mu);
        int i = w->next++;
        pthread_mutex_unlock(&w->mu);
        if (i >= p->B * p->H) break;
        size_t qk = (size_t)i * p->L * p->dk, vo = (size_t)i * p->L * p->dv;
        size_t st = (size_t)i * p->dk * p->dv;
        int rc = w->fn(p, i % p->H, i, w->chunk, w->Q + qk, w->K + qk,
                       w->V + vo, w->state_in ? w->state_in + st : NULL,
                       w->state_out ? w->state_out + st : NULL, w->O + vo);
        if (rc) {
            pthread_mutex_lock(&w->mu);
            w->err = rc;
            pthread_mutex_unlock(&w->mu);
        }
    }
    return NULL;
}

static int run_pool(pool *w)
{
    const oracle_problem *p = w->p;
    int n = p->nthreads > 0 ? p->nthreads : (int)sysconf(_SC_NPROCESSORS_ONLN);
    if (n < 1) n = 1;
    if (n > p->B * p->H) n = p->B * p->H;
    if (n < 1) return 0;
    pthread_t *th = (pthread_t *)malloc(sizeof(pthread_t) * n);
    if (!th) return 2;
    w->next = 0;
    w->err = 0;
    pthread_mutex_init(&w->mu, NULL);
    int started = 0;
    for (int i = 1; i < n; ++i)
        if (pthread_create(&th[started], NULL, pool_worker, w) == 0) ++started;
    /* the calling thread works too */
    pool_worker(w);
    for (int i = 0; i < started; ++i) pthread_join(th[i], NULL);
    pthread_mutex_destroy(&w->mu);
    free(th);
    return w->err;
}

static int check_problem(const oracle_problem *p)
{
    if (!p || !p->gamma) return 1;
    if (p->B < 0 || p->H < 0 || p->L < 0 || p->dk < 1 || p->dv < 1) return 1;
    if (p->rotate && (p->dk & 1)) return 1;
    return 0;
}

/* ------------------------------------------------------------------ */
/* Parallel representation, [RetNet summary] 2.1 (1): with D_nm =
 * gamma^{n-m} for n >= m and 0 otherwise, Retention(X) = (Q K^T (.) D) V.
 * Written out element by element: o_t = sum_{m<=t} gamma^{t-m} (q^_t.k^_m) v_m.
 * gamma^0 is 1 for every gamma, gamma = 0 included (C's pow(0,0) = 1). */
static int parallel_bh(const oracle_problem *p, int h, int bh, int chunk,
                       const double *Q, const double *K, const double *V,
                       const double *state_in, double *state_out, double *O)
{
    (void)bh; (void)chunk; (void)state_in; (void)state_out;
    const int L = p->L, dk = p->dk, dv = p->dv;
    const double g = p->gamma[h];
    double *q = rotated_copy(p, Q, dk), *k = rotated_copy(p, K, dk);
    if (!q || !k) { free(q); free(k); return 2; }
    for (int t = 0; t < L; ++t) {
        double *o = O + (size_t)t * dv;
        for (int j = 0; j < dv; ++j) o[j] = 0.0;
        for (int m = 0; m <= t; ++m) {
            double w = pow(g, (double)(t - m)) *
                       dot(q + (size_t)t * dk, k + (size_t)m * dk, dk);
            const double *v = V + (size_t)m * dv;
            for (int j = 0; j < dv; ++j) o[j] += w * v[j];
        }
    }
    free(q);
    free(k);
    return 0;
}

/* Recurrent representation, [RetNet summary] 2.1 (2):
 * S_n = gamma S_{n-1} + K_n^T V_n, Retention(X_n) = Q_n S_n, n = 1..|x|.
 * The state is updated with token n before it is read for token n, the
 * order the [Dual-mode manual] 3.2 inference wrapper also uses. */
static int recurrent_bh(const oracle_problem *p, int h, int bh, int chunk,
                        const double *Q, const double *K, const double *V,
                        const double *state_in, double *state_out, double *O)
{
    (void)bh; (void)chunk;
    const int L = p->L, dk = p->dk, dv = p->dv;
    const double g = p->gamma[h];
    double *S = (double *)calloc((size_t)dk * dv, sizeof(double));
    double *q = (double *)malloc(sizeof(double) * dk);
    double *k = (double *)malloc(sizeof(double) * dk);
    if (!S || !q || !k) { free(S); free(q); free(k); return 2; }
    if (state_in) memcpy(S, state_in, sizeof(double) * (size_t)dk * dv);
    for (int t = 0; t < L; ++t) {
        double pos = (double)(p->pos_offset + t);
        if (p->rotate) {
            oracle_xpos_rotate(Q + (size_t)t * dk, dk, pos, p->theta_base, q);
            oracle_xpos_rotate(K + (size_t)t * dk, dk, pos, p->theta_base, k);
        } else {
            memcpy(q, Q + (size_t)t * dk, sizeof(double) * dk);
            memcpy(k, K + (size_t)t * dk, sizeof(double) * dk);
        }
        const double *v = V + (size_t)t * dv;
        for (int i = 0; i < dk; ++i)
            for (int j = 0; j < dv; ++j)
                S[(size_t)i * dv + j] = g * S[(size_t)i * dv + j] + k[i] * v[j];
        double *o = O + (size_t)t * dv;
        for (int j = 0; j < dv; ++j) {
            double s = 0.0;
            for (int i = 0; i < dk; ++i) s += q[i] * S[(size_t)i * dv + j];
            o[j] = s;
        }
    }
    if (state_out) memcpy(state_out, S, sizeof(double) * (size_t)dk * dv);
    free(S); free(q); free(k);
    return 0;
}

/* Chunkwise recurrent representation, [RetNet summary] 2.1 (3): the pages
 * give it in words only -- parallel inside a chunk, recurrent between chunks.
 * Unrolling the recurrent form over the rows j = 0..n-1 of a chunk that
 * starts after state R gives S_j = gamma^{j+1} R + sum_{j'<=j} gamma^{j-j'}
 * k^_{j'}^T v_{j'}, hence
 *   o_j  = sum_{j'<=j} gamma^{j-j'} (q^_j.k^_{j'}) v_{j'}   (inside, parallel)
 *        + gamma^{j+1} q^_j R                               (carried state)
 *   R'   = gamma^n R + sum_{j'} gamma^{n-1-j'} k^_{j'}^T v_{j'}.
 * n is the chunk's own length, so a ragged last chunk decays by gamma^n. */
static int chunkwise_bh(const oracle_problem *p, int h, int bh, int chunk,
                        const double *Q, const double *K, const double *V,
                        const double *state_in, double *state_out, double *O)
{
    (void)bh;
    const int L = p->L, dk = p->dk, dv = p->dv;
    const double g = p->gamma[h];
    double *R = (double *)calloc((size_t)dk * dv, sizeof(double));
    double *Rn = (double *)malloc(sizeof(double) * (size_t)dk * dv);
    double *q = rotated_copy(p, Q, dk), *k = rotated_copy(p, K, dk);
    if (!R || !Rn || !q || !k) { free(R); free(Rn); free(q); free(k); return 2; }
    if (state_in) memcpy(R, state_in, sizeof(double) * (size_t)dk * dv);
    for (int c0 = 0; c0 < L; c0 += chunk) {
        int n = (L - c0 < chunk) ? L - c0 : chunk;
        for (int j = 0; j < n; ++j) {
            const double *qj = q + (size_t)(c0 + j) * dk;
            double *o = O + (size_t)(c0 + j) * dv;
            for (int c = 0; c < dv; ++c) o[c] = 0.0;
            for (int jj = 0; jj <= j; ++jj) {
                double w = pow(g, (double)(j - jj)) *
                           dot(qj, k + (size_t)(c0 + jj) * dk, dk);
                const double *v = V + (size_t)(c0 + jj) * dv;
                for (int c = 0; c < dv; ++c) o[c] += w * v[c];
            }
            double xi = pow(g, (double)(j + 1));
            for (int c = 0; c < dv; ++c) {
                double s = 0.0;
                for (int i = 0; i < dk; ++i) s += qj[i] * R[(size_t)i * dv + c];
                o[c] += xi * s;
            }
        }
        double gn = pow(g, (double)n);
        for (size_t e = 0; e < (size_t)dk * dv; ++e) Rn[e] = gn * R[e];
        for (int jj = 0; jj < n; ++jj) {
            double zeta = pow(g, (double)(n - 1 - jj));
            const double *kj = k + (size_t)(c0 + jj) * dk;
            const double *v = V + (size_t)(c0 + jj) * dv;
            for (int i = 0; i < dk; ++i)
                for (int c = 0; c < dv; ++c)
                    Rn[(size_t)i * dv + c] += zeta * kj[i] * v[c];
        }
        memcpy(R, Rn, sizeof(double) * (size_t)dk * dv);
    }
    if (state_out) memcpy(state_out, R, sizeof(double) * (size_t)dk * dv);
    free(R); free(Rn); free(q); free(k);
    return 0;
}

int oracle_retention_parallel(const oracle_problem *p, const double *Q,
                              const double *K, const double *V, double *O)
{
    if (check_problem(p) || (p->L && (!Q || !K || !V || !O))) return 1;
    pool w = {0};
    w.p = p; w.Q = Q; w.K = K; w.V = V; w.O = O; w.fn = parallel_bh;
    return run_pool(&w);
}

int oracle_retention_recurrent(const oracle_problem *p, const double *Q,
                               const double *K, const double *V,
                               const double *state_in, double *state_out,
                               double *O)
{
    if (check_problem(p) || (p->L && (!Q || !K || !V || !O))) return 1;
    pool w = {0};
    w.p = p; w.Q = Q; w.K = K; w.V = V; w.O = O; w.state_in = state_in;
    w.state_out = state_out; w.fn = recurrent_bh;
    return run_pool(&w);
}

int oracle_retention_chunkwise(const oracle_problem *p, int chunk,
                               const double *Q, const double *K,
                               const double *V, const double *state_in,
                               double *state_out, double *O)
{
    if (check_problem(p) || chunk < 1 || (p->L && (!Q || !K || !V || !O)))
        return 1;
    pool w = {0};
    w.p = p; w.chunk = chunk; w.Q = Q; w.K = K; w.V = V; w.O = O;
    w.state_in = state_in; w.state_out = state_out; w.fn = chunkwise_bh;
    return run_pool(&w);
}

/* Selected rows of one (b,h) slice straight from the parallel definition:
 * o_t = sum_{m<=t} gamma^{t-m} (q^_t.k^_m) v_m (+ gamma^{t+1} q^_t S0 when a
 * starting state S0 -- the state before row 0 -- is given, which is the
 * recurrent form unrolled to row 0).  Q, K are [L][dk], V is [L][dv], out is
 * [nrows][dv].  Used to check single outputs of full-size runs. */
int oracle_retention_rows(int L, int dk, int dv, const double *Q,
                          const double *K, const double *V, double gamma,
                          int rotate, double theta_base, long long pos_offset,
                          const double *state0, int nrows,
                          const long long *rows, double *out)
{
    if (L < 0 || dk < 1 || dv < 1 || (rotate && (dk & 1))) return 1;
    double *q = (double *)malloc(sizeof(double) * dk);
    double *k = (double *)malloc(sizeof(double) * dk);
    if (!q || !k) { free(q); free(k); return 2; }
    for (int r = 0; r < nrows; ++r) {
        long long t = rows[r];
        if (t < 0 || t >= L) { free(q); free(k); return 1; }
        double *o = out + (size_t)r * dv;
        for (int c = 0; c < dv; ++c) o[c] = 0.0;
        if (rotate)
            oracle_xpos_rotate(Q + (size_t)t * dk, dk,
                               (double)(pos_offset + t), theta_base, q);
        else
            memcpy(q, Q + (size_t)t * dk, sizeof(double) * dk);
        for (long long m = 0; m <= t; ++m) {
            if (rotate)
                oracle_xpos_rotate(K + (size_t)m * dk, dk,
                                   (double)(pos_offset + m), theta_base, k);
            else
                memcpy(k, K + (size_t)m * dk, sizeof(double) * dk);
            double w = pow(gamma, (double)(t - m)) * dot(q, k, dk);
            const double *v = V + (size_t)m * dv;
            for (int c = 0; c < dv; ++c) o[c] += w * v[c];
        }
        if (state0) {
            double xi = pow(gamma, (double)(t + 1));
            for (int c = 0; c < dv; ++c) {
                double s = 0.0;
                for (int i = 0; i < dk; ++i) s += q[i] * state0[(size_t)i * dv + c];
                o[c] += xi * s;
            }
        }
    }
    free(q); free(k);
    return 0;
}

/* [RetNet summary] 2.2: Y = GroupNorm_h(Concat(head_1..head_h)) and the
 * gate swish(X W_G) (.) Y, with X W_G given as G.  One group per head, taken
 * per token over that head's dv channels; population (biased) variance; no
 * affine weight or bias; swish(x) = x * sigmoid(x).
 * O is [B][H][L][dv]; G and Y are [B][L][H*dv]. */
int oracle_gate_groupnorm(int B, int L, int H, int dv, const double *O,
                          const double *G, double eps, double *Y)
{
    if (B < 0 || L < 0 || H < 0 || dv < 1 || eps < 0.0) return 1;
    for (int b = 0; b < B; ++b)
        for (int t = 0; t < L; ++t)
            for (int h = 0; h < H; ++h) {
                const double *o = O + (((size_t)b * H + h) * L + t) * dv;
                size_t gy = ((size_t)b * L + t) * (size_t)H * dv + (size_t)h * dv;
                double mu = 0.0, var = 0.0;
                for (int c = 0; c < dv; ++c) mu += o[c];
                mu /= dv;
                for (int c = 0; c < dv; ++c) var += (o[c] - mu) * (o[c] - mu);
                var /= dv;
                double inv = 1.0 / sqrt(var + eps);
                for (int c = 0; c < dv; ++c) {
                    double gv = G[gy + c];
                    double sw = gv / (1.0 + exp(-gv));
                    Y[gy + c] = sw * (o[c] - mu) * inv;
                }
            }
    return 0;
}

/* Gradients of the section 2.2 output Y = swish(G) (.) GroupNorm_h(O) above,
 * for a given dY, by the chain rule through its three steps, per (b, t, h)
 * row of dv channels, fp64:
 *   n_c = (o_c - mu) r with r = 1 / sqrt(var + eps)   (the normalised row)
 *   Y_c = s(g_c) n_c, s(g) = g sigmoid(g)
 *   dG_c = dY_c n_c s'(g_c), s'(g) = sigmoid(g) (1 + g (1 - sigmoid(g)))
 *   dn_c = dY_c s(g_c)
 *   dO_c = r (dn_c - mean_j dn_j - n_c mean_j (dn_j n_j))
 * The last line is the derivative of the normalisation: mu and var both
 * depend on every o_j of the row (d mu / d o_j = 1/dv, d var / d o_j =
 * 2 (o_j - mu) / dv).  Layouts as in oracle_gate_groupnorm; dY and dG share
 * G's, dO shares O's. */
int oracle_gate_groupnorm_backward(int B, int L, int H, int dv, const double *O,
                                   const double *G, const double *dY, double eps,
                                   double *dO, double *dG)
{
    if (B < 0 || L < 0 || H < 0 || dv < 1 || eps < 0.0) return 1;
    double *n = (double *)malloc(sizeof(double) * (size_t)dv);
    double *dn = (double *)malloc(sizeof(double) * (size_t)dv);
    if (!n || !dn) { free(n); free(dn); return 2; }
    for (int b = 0; b < B; ++b)
        for (int t = 0; t < L; ++t)
            for (int h = 0; h < H; ++h) {
                size_t orow = (((size_t)b * H + h) * L + t) * dv;
                size_t gy = ((size_t)b * L + t) * (size_t)H * dv + (size_t)h * dv;
                const double *o = O + orow;
                double mu = 0.0, var = 0.0;
                for (int c = 0; c < dv; ++c) mu += o[c];
                mu /= (double)dv;
                for (int c = 0; c < dv; ++c) var += (o[c] - mu) * (o[c] - mu);
                var /= (double)dv;
                double r = 1.0 / sqrt(var + eps);
                double mean_dn = 0.0, mean_dnn = 0.0;
                for (int c = 0; c < dv; ++c) {
                    double gv = G[gy + c];
                    double sig = 1.0 / (1.0 + exp(-gv));
                    n[c] = (o[c] - mu) * r;
                    dn[c] = dY[gy + c] * gv * sig;
                    dG[gy + c] = dY[gy + c] * n[c] * sig * (1.0 + gv * (1.0 - sig));
                    mean_dn += dn[c];
                    mean_dnn += dn[c] * n[c];
                }
                mean_dn /= dv;
                mean_dnn /= dv;
                for (int c = 0; c < dv; ++c)
                    dO[orow + c] = r * (dn[c] - mean_dn - n[c] * mean_dnn);
            }
    free(n); free(dn);
    return 0;
}
