/*
 * kda_oracle.c -- plain fp64 CPU oracle for the Kimi Delta Attention forward pass, and (at the
 * end of the file) its reverse-mode gradients for the tests of a backward kernel.
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

/* ------------------------------------------------------------------------------------------
 * Backward pass of the same recurrence (reverse mode, fp64), for the gradient tests of a
 * backward kernel. Per token, in the delta-rule form of the state-update equation:
 *
 *   S' = Diag(alpha) S_prev,  e = v - S'^T k,  S = S' + beta k e^T,  o = scale S^T q
 *
 * and, walking the tokens backwards with dS the gradient of the loss with respect to S:
 *
 *   dq = scale S do,                 dS += scale q do^T
 *   dbeta = k^T dS e,  dk += beta dS e,  de = beta dS^T k,  dS' = dS
 *   dv = de,  dS' -= k de^T,  dk -= S' de
 *   dS_prev = Diag(alpha) dS',  dg_i = alpha_i sum_j dS'_ij S_prev_ij
 *
 * The states of a sequence are recomputed from checkpoints taken every BWD_BLOCK tokens.
 * Inputs are double here, so that finite differences of the forward can pin this code.
 */
#define BWD_BLOCK 64

typedef struct {
    const double *q, *k, *v, *g, *beta;
    double scale;
    const int64_t *cu_seqlens;
    int64_t num_seqs, H, Dk, Dv;
    const double *h0, *dout, *dhT;
    double *dq, *dk, *dv, *dg, *dbeta, *dh0;
    int64_t next_unit;
    pthread_mutex_t mu;
} bjob_t;

/* S <- the state after token t, given the state before it (S_prev in S on entry) */
static void bwd_step_forward(const bjob_t *J, int64_t t, int64_t h, double *S, double *u) {
    const int64_t H = J->H, Dk = J->Dk, Dv = J->Dv;
    const double *kt = J->k + (size_t)((t * H + h) * Dk), *gt = J->g + (size_t)((t * H + h) * Dk);
    const double *vt = J->v + (size_t)((t * H + h) * Dv);
    const double bt = J->beta[t * H + h];
    for (int64_t i = 0; i < Dk; ++i) {
        const double a = exp(gt[i]);
        for (int64_t j = 0; j < Dv; ++j) S[i * Dv + j] *= a;
    }
    for (int64_t j = 0; j < Dv; ++j) {
        double s = 0.0;
        for (int64_t i = 0; i < Dk; ++i) s += S[i * Dv + j] * kt[i];
        u[j] = vt[j] - s; /* e */
    }
    for (int64_t i = 0; i < Dk; ++i)
        for (int64_t j = 0; j < Dv; ++j) S[i * Dv + j] += bt * kt[i] * u[j];
}

static void bwd_unit(bjob_t *J, int64_t unit, double *blk, double *dS, double *dSp, double *w) {
    const int64_t s = unit / J->H, h = unit % J->H;
    const int64_t H = J->H, Dk = J->Dk, Dv = J->Dv, DD = Dk * Dv;
    const int64_t bos = J->cu_seqlens[s], eos = J->cu_seqlens[s + 1], L = eos - bos;
    const size_t state_off = (size_t)((s * H + h) * DD);
    const int64_t nblk = (L + BWD_BLOCK - 1) / BWD_BLOCK;
    /* checkpoints: the state before each block */
    double *ck = (double *)malloc(sizeof(double) * (size_t)((nblk > 0 ? nblk : 1) * DD));
    double *S = w, *u = w + DD, *de = u + Dv;
    if (J->h0) memcpy(S, J->h0 + state_off, sizeof(double) * (size_t)DD);
    else memset(S, 0, sizeof(double) * (size_t)DD);
    for (int64_t b = 0; b < nblk; ++b) {
        memcpy(ck + b * DD, S, sizeof(double) * (size_t)DD);
        const int64_t t1 = bos + (b + 1) * BWD_BLOCK < eos ? bos + (b + 1) * BWD_BLOCK : eos;
        for (int64_t t = bos + b * BWD_BLOCK; t < t1; ++t) bwd_step_forward(J, t, h, S, u);
    }
    if (J->dhT) memcpy(dS, J->dhT + state_off, sizeof(double) * (size_t)DD);
    else memset(dS, 0, sizeof(double) * (size_t)DD);

    for (int64_t b = nblk - 1; b >= 0; --b) {
        const int64_t t0 = bos + b * BWD_BLOCK, t1 = t0 + BWD_BLOCK < eos ? t0 + BWD_BLOCK : eos;
        /* blk[i] = the state before token t0 + i */
        memcpy(blk, ck + b * DD, sizeof(double) * (size_t)DD);
        for (int64_t t = t0; t + 1 < t1; ++t) {
            memcpy(blk + (t - t0 + 1) * DD, blk + (t - t0) * DD, sizeof(double) * (size_t)DD);
            bwd_step_forward(J, t, h, blk + (t - t0 + 1) * DD, u);
        }
        for (int64_t t = t1 - 1; t >= t0; --t) {
            const double *Sprev = blk + (t - t0) * DD;
            const double *qt = J->q + (size_t)((t * H + h) * Dk), *kt = J->k + (size_t)((t * H + h) * Dk);
            const double *vt = J->v + (size_t)((t * H + h) * Dv), *gt = J->g + (size_t)((t * H + h) * Dk);
            const double *dot = J->dout + (size_t)((t * H + h) * Dv);
            const double bt = J->beta[t * H + h];
            double *dqt = J->dq + (size_t)((t * H + h) * Dk), *dkt = J->dk + (size_t)((t * H + h) * Dk);
            double *dvt = J->dv + (size_t)((t * H + h) * Dv), *dgt = J->dg + (size_t)((t * H + h) * Dk);
            /* S' (into S) and e (into u), then S_t (into dSp as scratch) */
            for (int64_t i = 0; i < Dk; ++i) {
                const double a = exp(gt[i]);
                for (int64_t j = 0; j < Dv; ++j) S[i * Dv + j] = a * Sprev[i * Dv + j];
            }
            for (int64_t j = 0; j < Dv; ++j) {
                double x = 0.0;
                for (int64_t i = 0; i < Dk; ++i) x += S[i * Dv + j] * kt[i];
                u[j] = vt[j] - x;
            }
            /* o = scale S_t^T q:  dq = scale S_t do,  dS += scale q do^T */
            for (int64_t i = 0; i < Dk; ++i) {
                double x = 0.0;
                for (int64_t j = 0; j < Dv; ++j) x += (S[i * Dv + j] + bt * kt[i] * u[j]) * dot[j];
                dqt[i] = J->scale * x;
                for (int64_t j = 0; j < Dv; ++j) dS[i * Dv + j] += J->scale * qt[i] * dot[j];
            }
            /* S_t = S' + beta k e^T */
            double db = 0.0;
            for (int64_t i = 0; i < Dk; ++i) {
                double x = 0.0;
                for (int64_t j = 0; j < Dv; ++j) x += dS[i * Dv + j] * u[j];
                db += kt[i] * x;
                dkt[i] = bt * x;
            }
            J->dbeta[t * H + h] = db;
            for (int64_t j = 0; j < Dv; ++j) {
                double x = 0.0;
                for (int64_t i = 0; i < Dk; ++i) x += dS[i * Dv + j] * kt[i];
                de[j] = bt * x;
                dvt[j] = de[j]; /* e = v - S'^T k */
            }
            /* dS' = dS - k de^T;  dk -= S' de */
            for (int64_t i = 0; i < Dk; ++i) {
                double x = 0.0;
                for (int64_t j = 0; j < Dv; ++j) {
                    dSp[i * Dv + j] = dS[i * Dv + j] - kt[i] * de[j];
                    x += S[i * Dv + j] * de[j];
                }
                dkt[i] -= x;
            }
            /* S' = Diag(alpha) S_prev */
            for (int64_t i = 0; i < Dk; ++i) {
                const double a = exp(gt[i]);
                double x = 0.0;
                for (int64_t j = 0; j < Dv; ++j) {
                    x += dSp[i * Dv + j] * Sprev[i * Dv + j];
                    dS[i * Dv + j] = a * dSp[i * Dv + j];
                }
                dgt[i] = a * x;
            }
        }
    }
    if (J->dh0) memcpy(J->dh0 + state_off, dS, sizeof(double) * (size_t)DD);
    free(ck);
}

static void *bwd_worker(void *arg) {
    bjob_t *J = (bjob_t *)arg;
    const int64_t DD = J->Dk * J->Dv;
    double *blk = (double *)malloc(sizeof(double) * (size_t)(BWD_BLOCK * DD));
    double *dS = (double *)malloc(sizeof(double) * (size_t)DD);
    double *dSp = (double *)malloc(sizeof(double) * (size_t)DD);
    double *w = (double *)malloc(sizeof(double) * (size_t)(DD + 2 * J->Dv));
    const int64_t units = J->num_seqs * J->H;
    for (;;) {
        pthread_mutex_lock(&J->mu);
        const int64_t unit = J->next_unit++;
        pthread_mutex_unlock(&J->mu);
        if (unit >= units) break;
        bwd_unit(J, unit, blk, dS, dSp, w);
    }
    free(blk);
    free(dS);
    free(dSp);
    free(w);
    return NULL;
}

/*
 * kda_oracle_bwd -- gradients of  L = sum(dout * out) + sum(dhT * hT)  with respect to the
 * inputs of kda_oracle_fwd, for the same packed batch (all arrays double, same layouts):
 *
 *   dout : [Ttot, H, Dv];  dhT : [num_seqs, H, Dk, Dv] or NULL (no loss on the final states)
 *   dq, dk, dg : [Ttot, H, Dk];  dv : [Ttot, H, Dv];  dbeta : [Ttot, H]   (written)
 *   dh0  : [num_seqs, H, Dk, Dv] or NULL                                   (written)
 *
 * Tokens outside every sequence are left untouched. Returns 0, or -1 on a malformed argument.
 */
int kda_oracle_bwd(const double *q, const double *k, const double *v, const double *g,
                   const double *beta, double scale, const int64_t *cu_seqlens, int64_t num_seqs,
                   int64_t H, int64_t Dk, int64_t Dv, const double *h0, const double *dout,
                   const double *dhT, double *dq, double *dk, double *dv, double *dg, double *dbeta,
                   double *dh0, int nthreads) {
    if (!q || !k || !v || !g || !beta || !cu_seqlens || !dout || !dq || !dk || !dv || !dg || !dbeta)
        return -1;
    if (num_seqs < 0 || H < 1 || Dk < 1 || Dv < 1 || nthreads < 1) return -1;
    if (cu_seqlens[0] != 0) return -1;
    for (int64_t s = 0; s < num_seqs; ++s)
        if (cu_seqlens[s + 1] < cu_seqlens[s]) return -1;
    bjob_t J;
    J.q = q; J.k = k; J.v = v; J.g = g; J.beta = beta; J.scale = scale;
    J.cu_seqlens = cu_seqlens; J.num_seqs = num_seqs; J.H = H; J.Dk = Dk; J.Dv = Dv;
    J.h0 = h0; J.dout = dout; J.dhT = dhT;
    J.dq = dq; J.dk = dk; J.dv = dv; J.dg = dg; J.dbeta = dbeta; J.dh0 = dh0; J.next_unit = 0;
    pthread_mutex_init(&J.mu, NULL);
    const int64_t units = num_seqs * H;
    int nt = nthreads;
    if ((int64_t)nt > units) nt = units > 0 ? (int)units : 1;
    pthread_t *th = (pthread_t *)malloc(sizeof(pthread_t) * (size_t)nt);
    for (int i = 0; i < nt; ++i) pthread_create(&th[i], NULL, bwd_worker, &J);
    for (int i = 0; i < nt; ++i) pthread_join(th[i], NULL);
    free(th);
    pthread_mutex_destroy(&J.mu);
    return 0;
}
