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
                     const double *v, double beta, double *o, double *x, int rule)
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

    /* S_t = S - alpha k x^T + alpha k v^T */
    for (int i = 0; i < dk; ++i) {
        const double ak = alpha * k[i];
        for (int j = 0; j < dv; ++j)
            S[(size_t)i * dv + j] += ak * (v[j] - x[j]);
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
    step_one(dk, dv, S, q, k, v, beta, o, x, rule);
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
    const double *q, *k, *v, *beta, *S0;
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
                 J->beta[tok], J->o ? J->o + tok * dv : NULL, x, J->rule);
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
 *   q,k    : [B,H,L,dk]   v, o : [B,H,L,dv]   beta : [B,H,L]
 *   S0     : [B,H,dk,dv] or NULL (zeros)      S_final : [B,H,dk,dv]
 *   o may be NULL (state only).  nthreads <= 0 means one thread.
 * Returns 0 on success, -1 on allocation failure.
 */
int efla_oracle_fwd_rule(int B, int H, int L, int dk, int dv, const double *q, const double *k,
                         const double *v, const double *beta, const double *S0, double *o,
                         double *S_final, int nthreads, int rule)
{
    fwd_job J;
    J.B = B; J.H = H; J.L = L; J.dk = dk; J.dv = dv;
    J.rule = rule;
    J.q = q; J.k = k; J.v = v; J.beta = beta; J.S0 = S0;
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

/* The exact-flow forward pass (rule 0). */
int efla_oracle_fwd(int B, int H, int L, int dk, int dv, const double *q, const double *k,
                    const double *v, const double *beta, const double *S0, double *o,
                    double *S_final, int nthreads)
{
    return efla_oracle_fwd_rule(B, H, L, dk, dv, q, k, v, beta, S0, o, S_final, nthreads, 0);
}
