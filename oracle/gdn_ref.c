/*
 * Gated DeltaNet token-by-token oracle, fp64, plain C.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path may link, load or
 * call this file; only the tests, the smoke check and the benchmark's CPU
 * baseline leg do.  It shares no code, header or constant with the CUDA
 * library.
 *
 * What it computes (per unit = one (document, head) pair of L tokens):
 *
 *   S_0   = h0^T                         (h0 is stored K x V, i.e. S^T)
 *   S_t   = a_t * S_{t-1} * (I - b_t k_t k_t^T) + b_t v_t k_t^T,
 *           a_t = exp(g_t)               (g is the log-decay, b the write
 *                                         strength: jax-linear-attention 0.1.0,
 *                                         "Quick start")
 *   o_t   = scale * S_t q_t
 *   hT    = S_L^T
 *
 * S is V x K (row index = value dim, column index = key dim).  The state is
 * carried in fp64 (the pages ask for fp32 states; the oracle keeps more).
 * The token-by-token form is the reference the pages hold every kernel to
 * (jax-linear-attention 0.1.0, "How it works": a token-by-token reference
 * is the oracle, tested on dense inputs, packed documents, initial and final
 * states and every gradient).
 *
 * Backward: reverse-mode of the same recurrence, one token at a time, with
 * the state recomputed from fp64 checkpoints taken every CKPT tokens.  With
 * X = dLoss/dS_t accumulated from the later tokens (X starts at dhT^T):
 *
 *   X    += scale * do_t q_t^T           (from o_t = scale S_t q_t)
 *   dq_t  = scale * S_t^T do_t
 *   y     = X k_t ;  delta = v_t - a_t S_{t-1} k_t
 *   dv_t  = b_t y
 *   db_t  = y . delta
 *   dk_t  = b_t X^T delta - a_t b_t S_{t-1}^T y
 *   da_t  = <X, S_{t-1}> - b_t (X k_t).(S_{t-1} k_t);   dg_t = a_t da_t
 *   X     = a_t (X - b_t (X k_t) k_t^T)  (= dLoss/dS_{t-1})
 *   dh0   = X^T after the first token.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define CKPT 64

typedef struct {
    int64_t L;
    const double *q, *k, *v, *g, *beta; /* q,k: L x K ; v: L x V ; g, beta: L */
    const double *h0;                   /* K x V, may be NULL (zero state) */
    double *o;                          /* L x V (forward output, may be NULL in bwd) */
    double *hT;                         /* K x V, may be NULL */
    const double *do_;                  /* L x V (bwd) */
    const double *dhT;                  /* K x V, may be NULL (zero) */
    double *dq, *dk, *dv, *dg, *dbeta;  /* bwd outputs */
    double *dh0;                        /* K x V, may be NULL */
} gdn_ref_unit;

/* S <- a S (I - b k k^T) + b v k^T, written out elementwise; Sk is scratch (V). */
static void step(double *S, double *Sk, int64_t K, int64_t V, double a, double b,
                 const double *k, const double *v) {
    for (int64_t i = 0; i < V; ++i) {
        double s = 0.0;
        for (int64_t j = 0; j < K; ++j) s += S[i * K + j] * k[j];
        Sk[i] = s;
    }
    for (int64_t i = 0; i < V; ++i)
        for (int64_t j = 0; j < K; ++j)
            S[i * K + j] = a * (S[i * K + j] - b * Sk[i] * k[j]) + b * v[i] * k[j];
}

static void load_state(double *S, const double *h, int64_t K, int64_t V) {
    if (!h) {
        memset(S, 0, sizeof(double) * K * V);
        return;
    }
    for (int64_t j = 0; j < K; ++j)
        for (int64_t i = 0; i < V; ++i) S[i * K + j] = h[j * V + i];
}

static void store_state(double *h, const double *S, int64_t K, int64_t V) {
    for (int64_t j = 0; j < K; ++j)
        for (int64_t i = 0; i < V; ++i) h[j * V + i] = S[i * K + j];
}

static int fwd_unit(const gdn_ref_unit *u, int64_t K, int64_t V, double scale) {
    double *S = malloc(sizeof(double) * K * V);
    double *Sk = malloc(sizeof(double) * V);
    if (!S || !Sk) { free(S); free(Sk); return 1; }
    load_state(S, u->h0, K, V);
    for (int64_t t = 0; t < u->L; ++t) {
        step(S, Sk, K, V, exp(u->g[t]), u->beta[t], u->k + t * K, u->v + t * V);
        if (u->o) {
            for (int64_t i = 0; i < V; ++i) {
                double s = 0.0;
                for (int64_t j = 0; j < K; ++j) s += S[i * K + j] * u->q[t * K + j];
                u->o[t * V + i] = scale * s;
            }
        }
    }
    if (u->hT) store_state(u->hT, S, K, V);
    free(S);
    free(Sk);
    return 0;
}

static int bwd_unit(const gdn_ref_unit *u, int64_t K, int64_t V, double scale) {
    const int64_t L = u->L, KV = K * V;
    const int64_t nck = (L + CKPT - 1) / CKPT + 1;
    double *ck = malloc(sizeof(double) * KV * nck);          /* state before token c*CKPT */
    double *blk = malloc(sizeof(double) * KV * (CKPT + 1));  /* states inside one block */
    double *X = malloc(sizeof(double) * KV);
    double *Sk = malloc(sizeof(double) * V);
    double *y = malloc(sizeof(double) * V);
    double *delta = malloc(sizeof(double) * V);
    if (!ck || !blk || !X || !Sk || !y || !delta) {
        free(ck); free(blk); free(X); free(Sk); free(y); free(delta);
        return 1;
    }
    /* forward sweep: checkpoints */
    load_state(ck, u->h0, K, V);
    {
        double *S = blk; /* reuse as running state */
        memcpy(S, ck, sizeof(double) * KV);
        for (int64_t t = 0; t < L; ++t) {
            step(S, Sk, K, V, exp(u->g[t]), u->beta[t], u->k + t * K, u->v + t * V);
            if ((t + 1) % CKPT == 0) memcpy(ck + ((t + 1) / CKPT) * KV, S, sizeof(double) * KV);
        }
    }
    load_state(X, u->dhT, K, V);
    for (int64_t c = (L + CKPT - 1) / CKPT - 1; c >= 0; --c) {
        const int64_t t0 = c * CKPT;
        const int64_t n = (L - t0 < CKPT) ? (L - t0) : CKPT;
        /* blk[i] = state before token t0+i, i = 0..n */
        memcpy(blk, ck + c * KV, sizeof(double) * KV);
        for (int64_t i = 0; i < n; ++i) {
            memcpy(blk + (i + 1) * KV, blk + i * KV, sizeof(double) * KV);
            step(blk + (i + 1) * KV, Sk, K, V, exp(u->g[t0 + i]), u->beta[t0 + i],
                 u->k + (t0 + i) * K, u->v + (t0 + i) * V);
        }
        for (int64_t i = n - 1; i >= 0; --i) {
            const int64_t t = t0 + i;
            const double *Sp = blk + i * KV;       /* S_{t-1} */
            const double *St = blk + (i + 1) * KV; /* S_t */
            const double *qt = u->q + t * K, *kt = u->k + t * K, *vt = u->v + t * V;
            const double *dot = u->do_ + t * V;
            const double a = exp(u->g[t]), b = u->beta[t];
            /* X += scale do_t q_t^T ; dq_t = scale S_t^T do_t */
            for (int64_t r = 0; r < V; ++r)
                for (int64_t j = 0; j < K; ++j) X[r * K + j] += scale * dot[r] * qt[j];
            for (int64_t j = 0; j < K; ++j) {
                double s = 0.0;
                for (int64_t r = 0; r < V; ++r) s += St[r * K + j] * dot[r];
                u->dq[t * K + j] = scale * s;
            }
            /* y = X k ; Sk = S_{t-1} k ; delta = v - a Sk */
            for (int64_t r = 0; r < V; ++r) {
                double s1 = 0.0, s2 = 0.0;
                for (int64_t j = 0; j < K; ++j) {
                    s1 += X[r * K + j] * kt[j];
                    s2 += Sp[r * K + j] * kt[j];
                }
                y[r] = s1;
                Sk[r] = s2;
                delta[r] = vt[r] - a * s2;
            }
            double db = 0.0, xs = 0.0, ysk = 0.0;
            for (int64_t r = 0; r < V; ++r) {
                u->dv[t * V + r] = b * y[r];
                db += y[r] * delta[r];
                ysk += y[r] * Sk[r];
            }
            for (int64_t e = 0; e < KV; ++e) xs += X[e] * Sp[e];
            u->dbeta[t] = db;
            u->dg[t] = a * (xs - b * ysk);
            for (int64_t j = 0; j < K; ++j) {
                double s1 = 0.0, s2 = 0.0;
                for (int64_t r = 0; r < V; ++r) {
                    s1 += X[r * K + j] * delta[r];
                    s2 += Sp[r * K + j] * y[r];
                }
                u->dk[t * K + j] = b * s1 - a * b * s2;
            }
            /* X <- a (X - b y k^T) */
            for (int64_t r = 0; r < V; ++r)
                for (int64_t j = 0; j < K; ++j) X[r * K + j] = a * (X[r * K + j] - b * y[r] * kt[j]);
        }
    }
    if (u->dh0) store_state(u->dh0, X, K, V);
    free(ck); free(blk); free(X); free(Sk); free(y); free(delta);
    return 0;
}

typedef struct {
    gdn_ref_unit *units;
    int n_units, stride, first, bwd;
    int64_t K, V;
    double scale;
    int err;
} job;

static void *worker(void *p) {
    job *j = (job *)p;
    for (int i = j->first; i < j->n_units; i += j->stride) {
        int e = j->bwd ? bwd_unit(&j->units[i], j->K, j->V, j->scale)
                       : fwd_unit(&j->units[i], j->K, j->V, j->scale);
        if (e) j->err = e;
    }
    return NULL;
}

static int run(gdn_ref_unit *units, int n_units, int64_t K, int64_t V, double scale,
               int nthreads, int bwd) {
    if (n_units <= 0) return 0;
    if (nthreads < 1) nthreads = 1;
    if (nthreads > n_units) nthreads = n_units;
    pthread_t *th = malloc(sizeof(pthread_t) * nthreads);
    job *jobs = malloc(sizeof(job) * nthreads);
    if (!th || !jobs) { free(th); free(jobs); return 1; }
    for (int i = 0; i < nthreads; ++i) {
        jobs[i] = (job){units, n_units, nthreads, i, bwd, K, V, scale, 0};
        pthread_create(&th[i], NULL, worker, &jobs[i]);
    }
    int err = 0;
    for (int i = 0; i < nthreads; ++i) {
        pthread_join(th[i], NULL);
        if (jobs[i].err) err = jobs[i].err;
    }
    free(th);
    free(jobs);
    return err;
}

/* Forward over independent units, spread over nthreads threads. 0 = ok. */
int gdn_ref_fwd(gdn_ref_unit *units, int n_units, int64_t K, int64_t V, double scale, int nthreads) {
    return run(units, n_units, K, V, scale, nthreads, 0);
}

/* Backward over independent units (fills dq, dk, dv, dg, dbeta, dh0). 0 = ok. */
int gdn_ref_bwd(gdn_ref_unit *units, int n_units, int64_t K, int64_t V, double scale, int nthreads) {
    return run(units, n_units, K, V, scale, nthreads, 1);
}
