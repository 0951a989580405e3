/*
 * efla_oracle.c -- plain fp64 CPU oracle for the Exact Flow Linear Attention
 * (EFLA) forward pass.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test suite, the smoke check and the
 * benchmark's CPU-baseline leg may load this library.  The CUDA library never
 * links, calls or includes anything from this directory, and this file shares
 * no code, header, table or helper with it.
 *
 * What it computes (source: "Exact Flow Linear Attention: Exact Solution from
 * Continuous-Time Dynamics", technical summary, Methodology 2 and 3):
 *
 *   lambda_t = ||k_t||^2                                   (Methodology 2)
 *   alpha_t  = (1 - exp(-beta_t lambda_t)) / lambda_t      (Methodology 3)
 *   S_t      = (I - alpha_t k_t k_t^T) S_{t-1} + alpha_t k_t v_t^T
 *                                                          (Methodology 3)
 *   o_t      = S_t^T q_t      (the standard delta-rule readout, taken after
 *                              the update; the summary prints no readout)
 *
 * and, for comparison, the delta rule that the summary identifies as the
 * explicit Euler step of the same ODE, dS/dtau = -k k^T S + k v^T over an
 * interval beta_t (Methodology 1; Key Contributions): S + beta_t (k v^T -
 * k k^T S), i.e. the same update with alpha_t = beta_t ("rule" 1 below).
 *
 * Gated form (a per-token decay g_t in (0, 1] on the carried state): the summary
 * names Gated DeltaNet among its baselines (Experimental Results) but prints no
 * equations for it.  The reading taken here is Gated DeltaNet's placement of the
 * gate, on the previous state's transition, with EFLA's coefficient:
 *
 *   S_t = g_t (I - alpha_t k_t k_t^T) S_{t-1} + alpha_t k_t v_t^T
 *
 * so that g_t = 1 is EFLA itself and k_t = 0 is a pure decay S_t = g_t S_{t-1}.
 *
 * Readings where the pages are silent:
 *   - alpha is evaluated as -expm1(-beta*lambda)/lambda, which is the same
 *     number without the cancellation of 1 - exp(x) for small x; at
 *     lambda == 0 the 0/0 form is replaced by its limit alpha = beta.
 *   - (I - alpha k k^T) S is evaluated as S - alpha k (k^T S): the same
 *     matrix product grouped so that it costs O(dk*dv) instead of O(dk^2*dv).
 *   - the state is dk x dv (k v^T is dk x dv), row-major, per (b, h) head.
 *   - no scaling or normalisation is applied to q or k.
 *
 * Heads (b, h) are independent; fwd() runs them on a pool of POSIX threads.
 * Within a head every token is processed in order, one at a time.  Nothing is
 * blocked, fused or reordered.
 *
 * Parity status: every function here is pinned by the CPU tests against
 * closed forms, an ODE integration, limits and invariants (see the oracle
 * tests); the pages print no worked numeric example.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* alpha_t from lambda_t and beta_t (Methodology 3), with the lambda -> 0 limit. */
double efla_oracle_alpha(double lambda, double beta)
{
    if (lambda == 0.0)
        return beta;
    return -expm1(-beta * lambda) / lambda;
}

/* The coefficient of the rank-1 update under a rule: 0 = exact flow, 1 = Euler step. */
double efla_oracle_coeff(double lambda, double beta, int rule)
{
    return rule == 1 ? beta : efla_oracle_alpha(lambda, beta);
}

/*
 * One token of the recurrence on one head, in place.
 *   S  : dk x dv, row-major (S[i*dv + j]), updated to S_t
 *   q,k: dk ; v: dv ; o: dv (may be NULL)
 *   x  : scratch of length dv supplied by the caller
 */
static void step_one(int dk, int dv, double *S, const double *q, const double *k,
                     const double *v, double beta, double *o, double *x, int rule, double g)
{
    double lambda = 0.0;
    for (int i = 0; i < dk; ++i)
        lambda += k[i] * k[i];
    const double alpha = efla_oracle_coeff(lambda, beta, rule);

    /* x = S^T k  (so that (I - alpha k k^T) S = S - alpha k x^T) */
    for (int j = 0; j < dv; ++j)
        x[j] = 0.0;
    for (int i = 0; i < dk; ++i)
        for (int j = 0; j < dv; ++j)
            x[j] += S[(size_t)i * dv + j] * k[i];

    /* S_t = g (S - alpha k x^T) + alpha k v^T; without a gate (g = 1) this is
       S + alpha k (v - x)^T, evaluated exactly so */
    if (g == 1.0) {
        for (int i = 0; i < dk; ++i) {
            const double ak = alpha * k[i];
            for (int j = 0; j < dv; ++j)
                S[(size_t)i * dv + j] += ak * (v[j] - x[j]);
        }
    } else {
        for (int i = 0; i < dk; ++i) {
            const double ak = alpha * k[i];
            for (int j = 0; j < dv; ++j)
                S[(size_t)i * dv + j] = g * (S[(size_t)i * dv + j] - ak * x[j]) + ak * v[j];
        }
    }

    /* o_t = S_t^T q */
    if (o) {
        for (int j = 0; j < dv; ++j)
            o[j] = 0.0;
        for (int i = 0; i < dk; ++i)
            for (int j = 0; j < dv; ++j)
                o[j] += S[(size_t)i * dv + j] * q[i];
    }
}

/*
 * Single token on a single head (the decode form) under a rule.  S is updated
 * in place.  Returns the coefficient used.
 */
double efla_oracle_step_rule(int dk, int dv, double *S, const double *q, const double *k,
                             const double *v, double beta, double *o, int rule)
{
    double *x = (double *)malloc(sizeof(double) * (size_t)(dv > 0 ? dv : 1));
    if (!x)
        return NAN;
    double lambda = 0.0;
    for (int i = 0; i < dk; ++i)
        lambda += k[i] * k[i];
    step_one(dk, dv, S, q, k, v, beta, o, x, rule, 1.0);
    free(x);
    return efla_oracle_coeff(lambda, beta, rule);
}

/* One token of the gated form (decay g on the previous state's transition). */
double efla_oracle_step_gated(int dk, int dv, double *S, const double *q, const double *k,
                              const double *v, double beta, double g, double *o, int rule)
{
    double *x = (double *)malloc(sizeof(double) * (size_t)(dv > 0 ? dv : 1));
    if (!x)
        return NAN;
    double lambda = 0.0;
    for (int i = 0; i < dk; ++i)
        lambda += k[i] * k[i];
    step_one(dk, dv, S, q, k, v, beta, o, x, rule, g);
    free(x);
    return efla_oracle_coeff(lambda, beta, rule);
}

/* The exact-flow step (rule 0).  Returns alpha_t. */
double efla_oracle_step(int dk, int dv, double *S, const double *q, const double *k,
                        const double *v, double beta, double *o)
{
    return efla_oracle_step_rule(dk, dv, S, q, k, v, beta, o, 0);
}

/* ---- whole forward pass over [B, H, L, d] tensors ---------------------- */

typedef struct {
    int B, H, L, dk, dv;
    const double *q, *k, *v, *beta, *gate, *S0;  /* gate: NULL = no decay */
    double *o, *S_final;
    int rule;
    int next_head; /* shared work counter */
    pthread_mutex_t lock;
    int failed;
} fwd_job;

static void run_head(fwd_job *J, int bh)
{
    const int L = J->L, dk = J->dk, dv = J->dv;
    const size_t sz = (size_t)dk * dv;
    double *S = J->S_final + (size_t)bh * sz; /* state lives in the output */
    double *x = (double *)malloc(sizeof(double) * (size_t)(dv > 0 ? dv : 1));
    if (!x) {
        J->failed = 1;
        return;
    }
    if (J->S0)
        memcpy(S, J->S0 + (size_t)bh * sz, sizeof(double) * sz);
    else
        memset(S, 0, sizeof(double) * sz);
    for (int t = 0; t < L; ++t) {
        const size_t tok = (size_t)bh * L + t;
        step_one(dk, dv, S, J->q + tok * dk, J->k + tok * dk, J->v + tok * dv,
                 J->beta[tok], J->o ? J->o + tok * dv : NULL, x, J->rule,
                 J->gate ? J->gate[tok] : 1.0);
    }
    free(x);
}

static void *worker(void *arg)
{
    fwd_job *J = (fwd_job *)arg;
    for (;;) {
        pthread_mutex_lock(&J->lock);
        int bh = J->next_head++;
        pthread_mutex_unlock(&J->lock);
        if (bh >= J->B * J->H)
            break;
        run_head(J, bh);
    }
    return NULL;
}

/*
 * Full forward pass.
 *   q,k    : [B,H,L,dk]   v, o : [B,H,L,dv]   beta, gate : [B,H,L] (gate NULL: none)
 *   S0     : [B,H,dk,dv] or NULL (zeros)      S_final : [B,H,dk,dv]
 *   o may be NULL (state only).  nthreads <= 0 means one thread.
 * Returns 0 on success, -1 on allocation failure.
 */
int efla_oracle_fwd_gated(int B, int H, int L, int dk, int dv, const double *q, const double *k,
                          const double *v, const double *beta, const double *gate,
                          const double *S0, double *o, double *S_final, int nthreads, int rule)
{
    fwd_job J;
    J.B = B; J.H = H; J.L = L; J.dk = dk; J.dv = dv;
    J.rule = rule;
    J.q = q; J.k = k; J.v = v; J.beta = beta; J.gate = gate; J.S0 = S0;
    J.o = o; J.S_final = S_final;
    J.next_head = 0;
    J.failed = 0;
    pthread_mutex_init(&J.lock, NULL);
    if (nthreads < 1)
        nthreads = 1;
    if (nthreads > B * H)
        nthreads = B * H > 0 ? B * H : 1;
    pthread_t *th = (pthread_t *)malloc(sizeof(pthread_t) * (size_t)nthreads);
    int started = 0;
    if (th) {
        for (int i = 0; i < nthreads; ++i)
            if (pthread_create(&th[started], NULL, worker, &J) == 0)
                ++started;
    }
    if (started == 0)
        worker(&J); /* run inline */
    for (int i = 0; i < started; ++i)
        pthread_join(th[i], NULL);
    free(th);
    pthread_mutex_destroy(&J.lock);
    return J.failed ? -1 : 0;
}

/* Forward pass without a gate under a rule. */
int efla_oracle_fwd_rule(int B, int H, int L, int dk, int dv, const double *q, const double *k,
                         const double *v, const double *beta, const double *S0, double *o,
                         double *S_final, int nthreads, int rule)
{
    return efla_oracle_fwd_gated(B, H, L, dk, dv, q, k, v, beta, NULL, S0, o, S_final, nthreads,
                                 rule);
}

/* The exact-flow forward pass (rule 0). */
int efla_oracle_fwd(int B, int H, int L, int dk, int dv, const double *q, const double *k,
                    const double *v, const double *beta, const double *S0, double *o,
                    double *S_final, int nthreads)
{
    return efla_oracle_fwd_rule(B, H, L, dk, dv, q, k, v, beta, S0, o, S_final, nthreads, 0);
}

/* ---- backward pass (reverse mode through the token recurrence) --------------------------
 *
 * Gradients of a loss through the forward above, given do (dL/do_t) and dS_final (dL/dS_L,
 * may be NULL = 0): dq, dk, dv, dbeta and dS0 (dL/dS0).  Per token the forward is
 *   lambda = k.k, a = f(lambda, beta), x = S^T k, r = v - x, u = a r, S' = S + k u^T,
 *   o = S'^T q,
 * and the reverse step, with G = dL/dS' gathered from the later tokens, is
 *   G += q do^T;  dq = S' do;  du = G^T k;  dk = G u;  da = du.r;  dv = a du;  dx = -a du;
 *   dS = G + k dx^T;  dk += S dx;  dbeta = da df/dbeta;  dk += 2 da df/dlambda k;  G = dS.
 * For the exact rule df/dbeta = e^{-beta lambda} and df/dlambda = (beta e^{-beta lambda} - a) /
 * lambda (its series in x = beta lambda near 0); for the Euler rule df/dbeta = 1 and
 * df/dlambda = 0.  The states S_t come from a forward sweep kept in full (the oracle has memory
 * to spare).  Pinned in the tests by central finite differences of the forward.
 */
static void coeff_grads(double lambda, double beta, int rule, double *dfdb, double *dfdl)
{
    if (rule == 1) {
        *dfdb = 1.0;
        *dfdl = 0.0;
        return;
    }
    const double x = beta * lambda;
    *dfdb = exp(-x);
    if (fabs(x) < 1e-4) {  /* beta^2 (-1/2 + x/3 - x^2/8 + x^3/30) */
        *dfdl = beta * beta * (-0.5 + x / 3.0 - x * x / 8.0 + x * x * x / 30.0);
    } else {
        const double a = efla_oracle_alpha(lambda, beta);
        *dfdl = (beta * exp(-x) - a) / lambda;
    }
}

static void bwd_head(int L, int dk, int dv, const double *q, const double *k, const double *v,
                     const double *beta, const double *S0, const double *dO, const double *dSL,
                     double *dq, double *dkk, double *dvv, double *db, double *dS0, int rule)
{
    const size_t sz = (size_t)dk * dv;
    double *Ss = (double *)malloc(sizeof(double) * sz * (size_t)(L + 1)); /* S_0 .. S_L */
    double *G = (double *)malloc(sizeof(double) * sz);
    double *x = (double *)malloc(sizeof(double) * (size_t)dv);
    double *du = (double *)malloc(sizeof(double) * (size_t)dv);
    double *u = (double *)malloc(sizeof(double) * (size_t)dv);
    if (!Ss || !G || !x || !du || !u) {
        free(Ss); free(G); free(x); free(du); free(u);
        return;
    }
    if (S0) memcpy(Ss, S0, sizeof(double) * sz);
    else memset(Ss, 0, sizeof(double) * sz);
    for (int t = 0; t < L; ++t) {
        memcpy(Ss + sz * (size_t)(t + 1), Ss + sz * (size_t)t, sizeof(double) * sz);
        step_one(dk, dv, Ss + sz * (size_t)(t + 1), q + (size_t)t * dk, k + (size_t)t * dk,
                 v + (size_t)t * dv, beta[t], NULL, x, rule, 1.0);
    }
    if (dSL) memcpy(G, dSL, sizeof(double) * sz);
    else memset(G, 0, sizeof(double) * sz);
    for (int t = L - 1; t >= 0; --t) {
        const double *S = Ss + sz * (size_t)t, *Sp = Ss + sz * (size_t)(t + 1);
        const double *qt = q + (size_t)t * dk, *kt = k + (size_t)t * dk, *vt = v + (size_t)t * dv;
        const double *dot = dO + (size_t)t * dv;
        double lambda = 0.0;
        for (int i = 0; i < dk; ++i) lambda += kt[i] * kt[i];
        const double a = efla_oracle_coeff(lambda, beta[t], rule);
        for (int j = 0; j < dv; ++j) {  /* x = S^T k, u = a (v - x) */
            double s = 0.0;
            for (int i = 0; i < dk; ++i) s += S[(size_t)i * dv + j] * kt[i];
            x[j] = s;
            u[j] = a * (vt[j] - s);
        }
        for (int i = 0; i < dk; ++i)  /* G += q do^T */
            for (int j = 0; j < dv; ++j) G[(size_t)i * dv + j] += qt[i] * dot[j];
        for (int i = 0; i < dk; ++i) {  /* dq = S' do */
            double s = 0.0;
            for (int j = 0; j < dv; ++j) s += Sp[(size_t)i * dv + j] * dot[j];
            dq[(size_t)t * dk + i] = s;
        }
        double da = 0.0;
        for (int j = 0; j < dv; ++j) {  /* du = G^T k, da = du.r, dv = a du */
            double s = 0.0;
            for (int i = 0; i < dk; ++i) s += G[(size_t)i * dv + j] * kt[i];
            du[j] = s;
            da += s * (vt[j] - x[j]);
            dvv[(size_t)t * dv + j] = a * s;
        }
        for (int i = 0; i < dk; ++i) {  /* dk = G u + S dx with dx = -a du */
            double s1 = 0.0, s2 = 0.0;
            for (int j = 0; j < dv; ++j) {
                s1 += G[(size_t)i * dv + j] * u[j];
                s2 += S[(size_t)i * dv + j] * (-a * du[j]);
            }
            dkk[(size_t)t * dk + i] = s1 + s2;
        }
        double dfdb, dfdl;
        coeff_grads(lambda, beta[t], rule, &dfdb, &dfdl);
        db[t] = da * dfdb;
        for (int i = 0; i < dk; ++i) dkk[(size_t)t * dk + i] += 2.0 * da * dfdl * kt[i];
        for (int i = 0; i < dk; ++i)  /* G = G + k dx^T */
            for (int j = 0; j < dv; ++j) G[(size_t)i * dv + j] += kt[i] * (-a * du[j]);
    }
    if (dS0) memcpy(dS0, G, sizeof(double) * sz);
    free(Ss); free(G); free(x); free(du); free(u);
}

/*
 * Backward pass over [B,H,L,d] tensors (heads in sequence):
 *   dO : [B,H,L,dv]   dS_final : [B,H,dk,dv] or NULL
 *   dq, dk : [B,H,L,dk]   dv : [B,H,L,dv]   dbeta : [B,H,L]   dS0 : [B,H,dk,dv] or NULL
 */
void efla_oracle_bwd(int B, int H, int L, int dk, int dv, const double *q, const double *k,
                     const double *v, const double *beta, const double *S0, const double *dO,
                     const double *dS_final, double *dq, double *dkk, double *dvv, double *dbeta,
                     double *dS0, int rule)
{
    const size_t sz = (size_t)dk * dv;
    for (int bh = 0; bh < B * H; ++bh) {
        const size_t tk = (size_t)bh * L * dk, tv = (size_t)bh * L * dv, tb = (size_t)bh * L;
        bwd_head(L, dk, dv, q + tk, k + tk, v + tv, beta + tb, S0 ? S0 + sz * bh : NULL, dO + tv,
                 dS_final ? dS_final + sz * bh : NULL, dq + tk, dkk + tk, dvv + tv, dbeta + tb,
                 dS0 ? dS0 + sz * bh : NULL, rule);
    }
}
