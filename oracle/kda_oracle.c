/*
 * kda_oracle.c -- plain fp64 CPU oracle for the Kimi Delta Attention forward pass.
 *
 * TEST INFRASTRUCTURE ONLY. Nothing in the product path links, loads or calls
 * this file; only the tests, the package's smoke check and the CPU-baseline
 * leg of the benchmark do. It shares no code, header, table or helper with the
 * CUDA library.
 *
 * What it computes (Kimi Linear feature page, chapter 4 "innovation 2",
 * state-update equation; chapter 3 delta-rule equation):
 *
 *   S_t = (Diag(alpha_t) - beta_t k_t (k_t (.) alpha_t)^T) S_{t-1} + beta_t k_t v_t^T
 *   o_t = scale * S_t^T q_t
 *
 * token by token, in double precision, with alpha_t = exp(g_t) per key
 * channel (g is the raw per-token log-decay, never cumulative), S a Dk x Dv
 * matrix whose rows are indexed by key channels. The rank-one term is applied
 * as k_t times the row vector (k_t (.) alpha_t)^T S_{t-1}; no Dk x Dk matrix is
 * formed. The output of token t reads the state after token t's update.
 * Sequences of a packed batch are independent: each starts from its own
 * initial state (or zero) and its final state is written out.
 *
 * No chunking, no blocking, no reordering: one token after another.
 * Work is spread over (sequence, head) pairs with POSIX threads; the
 * arithmetic of each pair is sequential and identical whatever the thread
 * count.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* Planted mistakes for the mutation tests (tests/test_oracle_pins.py builds
 * this file with -DKDA_ORACLE_MUTANT=n to check that the pins catch them).
 * The default build (0) is the oracle. */
#ifndef KDA_ORACLE_MUTANT
#define KDA_ORACLE_MUTANT 0
#endif

typedef struct {
    const float *q, *k, *v, *g, *beta;
    double scale;
    const int64_t *cu_seqlens;
    int64_t num_seqs, H, Dk, Dv;
    const double *h0;
    double *out, *hT;
    int64_t next_unit; /* shared work counter, guarded by mu */
    pthread_mutex_t mu;
} job_t;

/* One (sequence, head) pair, tokens in order. */
static void run_unit(job_t *J, int64_t unit, double *S, double *u) {
    const int64_t s = unit / J->H, h = unit % J->H;
    const int64_t H = J->H, Dk = J->Dk, Dv = J->Dv;
    const int64_t bos = J->cu_seqlens[s], eos = J->cu_seqlens[s + 1];
    const size_t state_off = (size_t)((s * H + h) * Dk * Dv);

    if (J->h0) memcpy(S, J->h0 + state_off, sizeof(double) * (size_t)(Dk * Dv));
    else memset(S, 0, sizeof(double) * (size_t)(Dk * Dv));

    for (int64_t t = bos; t < eos; ++t) {
        const float *qt = J->q + (size_t)((t * H + h) * Dk);
        const float *kt = J->k + (size_t)((t * H + h) * Dk);
        const float *vt = J->v + (size_t)((t * H + h) * Dv);
        const float *gt = J->g + (size_t)((t * H + h) * Dk);
        const double bt = (double)J->beta[t * H + h];
        double *ot = J->out + (size_t)((t * H + h) * Dv);

        /* u = (k (.) alpha)^T S_{t-1}  (a row vector of length Dv) */
        for (int64_t j = 0; j < Dv; ++j) u[j] = 0.0;
        for (int64_t i = 0; i < Dk; ++i) {
#if KDA_ORACLE_MUTANT == 1 /* rank-one term forgets the decay */
            const double ka = (double)kt[i];
#else
            const double ka = (double)kt[i] * exp((double)gt[i]);
#endif
            const double *Si = S + i * Dv;
            for (int64_t j = 0; j < Dv; ++j) u[j] += ka * Si[j];
        }
        /* S_t = Diag(alpha) S_{t-1} - beta k u + beta k v^T */
        for (int64_t i = 0; i < Dk; ++i) {
#if KDA_ORACLE_MUTANT == 2 /* decay applied with the wrong sign */
            const double a = exp(-(double)gt[i]);
#else
            const double a = exp((double)gt[i]);
#endif
            const double bk = bt * (double)kt[i];
            double *Si = S + i * Dv;
#if KDA_ORACLE_MUTANT == 3 /* retrieval error term dropped (plain gated linear attention) */
            for (int64_t j = 0; j < Dv; ++j) Si[j] = a * Si[j] + bk * (double)vt[j];
#elif KDA_ORACLE_MUTANT == 4 /* beta applied to the value only */
            for (int64_t j = 0; j < Dv; ++j) Si[j] = a * Si[j] - (double)kt[i] * u[j] + bk * (double)vt[j];
#else
            for (int64_t j = 0; j < Dv; ++j) Si[j] = a * Si[j] - bk * u[j] + bk * (double)vt[j];
#endif
        }
        /* o_t = scale * S_t^T q_t */
        for (int64_t j = 0; j < Dv; ++j) ot[j] = 0.0;
        for (int64_t i = 0; i < Dk; ++i) {
            const double qi = (double)qt[i];
            const double *Si = S + i * Dv;
#if KDA_ORACLE_MUTANT == 5 /* transposed read-out: uses the key row index for the value */
            for (int64_t j = 0; j < Dv; ++j) ot[j] += qi * S[j * Dv + i];
#else
            for (int64_t j = 0; j < Dv; ++j) ot[j] += qi * Si[j];
#endif
        }
        for (int64_t j = 0; j < Dv; ++j) ot[j] *= J->scale;
    }
    if (J->hT) memcpy(J->hT + state_off, S, sizeof(double) * (size_t)(Dk * Dv));
}

static void *worker(void *arg) {
    job_t *J = (job_t *)arg;
    double *S = (double *)malloc(sizeof(double) * (size_t)(J->Dk * J->Dv));
    double *u = (double *)malloc(sizeof(double) * (size_t)J->Dv);
    const int64_t units = J->num_seqs * J->H;
    for (;;) {
        pthread_mutex_lock(&J->mu);
        const int64_t unit = J->next_unit++;
        pthread_mutex_unlock(&J->mu);
        if (unit >= units) break;
        run_unit(J, unit, S, u);
    }
    free(S);
    free(u);
    return NULL;
}

/*
 * kda_oracle_fwd -- run the recurrence over a packed batch.
 *
 *   q, k, g   : [Ttot, H, Dk] float32 (bf16 inputs are widened exactly by the caller)
 *   v         : [Ttot, H, Dv] float32
 *   beta      : [Ttot, H]     float32
 *   cu_seqlens: [num_seqs + 1] host int64, cu_seqlens[0] = 0, non-decreasing
 *   h0        : [num_seqs, H, Dk, Dv] float64, or NULL for zero initial states
 *   out       : [Ttot, H, Dv] float64 (written)
 *   hT        : [num_seqs, H, Dk, Dv] float64 (written), or NULL
 *   nthreads  : worker threads (>= 1)
 *
 * Returns 0 on success, -1 on a malformed argument (nothing is written then).
 */
int kda_oracle_fwd(const float *q, const float *k, const float *v, const float *g,
                   const float *beta, double scale, const int64_t *cu_seqlens,
                   int64_t num_seqs, int64_t H, int64_t Dk, int64_t Dv, const double *h0,
                   double *out, double *hT, int nthreads) {
    if (!q || !k || !v || !g || !beta || !cu_seqlens || !out) return -1;
    if (num_seqs < 0 || H < 1 || Dk < 1 || Dv < 1 || nthreads < 1) return -1;
    if (cu_seqlens[0] != 0) return -1;
    for (int64_t s = 0; s < num_seqs; ++s)
        if (cu_seqlens[s + 1] < cu_seqlens[s]) return -1;

    job_t J;
    J.q = q; J.k = k; J.v = v; J.g = g; J.beta = beta; J.scale = scale;
    J.cu_seqlens = cu_seqlens; J.num_seqs = num_seqs; J.H = H; J.Dk = Dk; J.Dv = Dv;
    J.h0 = h0; J.out = out; J.hT = hT; J.next_unit = 0;
    pthread_mutex_init(&J.mu, NULL);

    const int64_t units = num_seqs * H;
    int nt = nthreads;
    if ((int64_t)nt > units) nt = units > 0 ? (int)units : 1;
    pthread_t *th = (pthread_t *)malloc(sizeof(pthread_t) * (size_t)nt);
    for (int i = 0; i < nt; ++i) pthread_create(&th[i], NULL, worker, &J);
    for (int i = 0; i < nt; ++i) pthread_join(th[i], NULL);
    free(th);
    pthread_mutex_destroy(&J.mu);
    return 0;
}
