/*
 * TEST INFRASTRUCTURE — the fp64 CPU oracle for the gradient of the Kimi Delta
 * Attention recurrence (the same update and readout as kda_oracle.c, Kimi
 * Linear report section 3 Eq. 1 with o~_t = S_t^T q_t read after the update).
 * Only tests/ may load it.  It shares no code with the CUDA library.
 *
 * For one sequence, write the token step as
 *   X_t = Diag(alpha_t) S_{t-1},  p_t = X_t^T k_t,  r_t = beta_t (v_t - p_t),
 *   S_t = X_t + k_t r_t^T,        o_t = S_t^T q_t,
 * which is Eq. 1 term by term.  Given dL/do_t for every token and dL/dS_T,
 * reverse-mode differentiation of these five lines, token by token from the
 * last one (all S_t kept from a forward pass), gives
 *   dS_t <- dS_t + q_t do_t^T;                 dq_t = S_t do_t
 *   dk_t = dS_t r_t;  dr_t = dS_t^T k_t
 *   dbeta_t = dr_t . (v_t - p_t);  dv_t = beta_t dr_t;  dp_t = -beta_t dr_t
 *   dX_t = dS_t + k_t dp_t^T;  dk_t += X_t dp_t
 *   dalpha_t = rowsum(dX_t * S_{t-1});  dS_{t-1} = Diag(alpha_t) dX_t
 * and, through alpha = exp(g), g = g_min * sigmoid(z):
 *   dg_t = dalpha_t * alpha_t;  dz_t = dg_t * g_min * sigmoid(z_t) (1 - sigmoid(z_t)).
 * dL/dS_0 is the last dS.  fp64 throughout.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

typedef struct {
    int64_t S, Dk, Dv, sk, sv, sb;
    const float *q, *k, *v, *z, *log_decay, *beta, *dO, *S0, *dST;
    double g_min;
    double *dq, *dk, *dv, *dbeta, *dg, *dS0;   /* dg: d/dz when z is given, else d/dlog_decay */
} bwd_seq_t;

static double sig(double x) { return 1.0 / (1.0 + exp(-x)); }

static int run_bwd(const bwd_seq_t *a)
{
    const int64_t S = a->S, Dk = a->Dk, Dv = a->Dv, N = Dk * Dv;
    double *St = (double *)malloc(sizeof(double) * (size_t)((S + 1) * N));   /* S_{-1} .. S_{S-1} */
    double *al = (double *)malloc(sizeof(double) * (size_t)(S * Dk));
    double *u = (double *)malloc(sizeof(double) * (size_t)(S * Dv));          /* v_t - p_t */
    double *dS = (double *)malloc(sizeof(double) * (size_t)N);
    double *dX = (double *)malloc(sizeof(double) * (size_t)N);
    double *dr = (double *)malloc(sizeof(double) * (size_t)Dv);
    if (!St || !al || !u || !dS || !dX || !dr) {
        free(St); free(al); free(u); free(dS); free(dX); free(dr);
        return -2;
    }
    /* forward, keeping every state */
    for (int64_t i = 0; i < N; ++i) St[i] = a->S0 ? (double)a->S0[i] : 0.0;
    for (int64_t t = 0; t < S; ++t) {
        const float *k = a->k + t * a->sk, *v = a->v + t * a->sv;
        const double beta = (double)a->beta[t * a->sb];
        const double *Sp = St + t * N;
        double *Sc = St + (t + 1) * N;
        for (int64_t c = 0; c < Dk; ++c) {
            const double g = a->log_decay ? (double)a->log_decay[t * a->sk + c]
                                          : a->g_min * sig((double)a->z[t * a->sk + c]);
            al[t * Dk + c] = exp(g);
        }
        for (int64_t c = 0; c < Dk; ++c)
            for (int64_t j = 0; j < Dv; ++j) Sc[c * Dv + j] = al[t * Dk + c] * Sp[c * Dv + j];   /* X_t */
        for (int64_t j = 0; j < Dv; ++j) {
            double p = 0.0;
            for (int64_t c = 0; c < Dk; ++c) p += Sc[c * Dv + j] * (double)k[c];
            u[t * Dv + j] = (double)v[j] - p;
        }
        for (int64_t c = 0; c < Dk; ++c)
            for (int64_t j = 0; j < Dv; ++j) Sc[c * Dv + j] += (double)k[c] * beta * u[t * Dv + j];
    }
    /* backward */
    for (int64_t i = 0; i < N; ++i) dS[i] = a->dST ? (double)a->dST[i] : 0.0;
    for (int64_t t = S - 1; t >= 0; --t) {
        const float *q = a->q + t * a->sk, *k = a->k + t * a->sk, *dO = a->dO + t * a->sv;
        const double beta = (double)a->beta[t * a->sb];
        const double *Sp = St + t * N, *Sc = St + (t + 1) * N;
        double *dq = a->dq + t * a->sk, *dk = a->dk + t * a->sk, *dv = a->dv + t * a->sv;
        for (int64_t c = 0; c < Dk; ++c)
            for (int64_t j = 0; j < Dv; ++j) dS[c * Dv + j] += (double)q[c] * (double)dO[j];
        for (int64_t c = 0; c < Dk; ++c) {
            double s = 0.0;
            for (int64_t j = 0; j < Dv; ++j) s += Sc[c * Dv + j] * (double)dO[j];
            dq[c] = s;
        }
        for (int64_t c = 0; c < Dk; ++c) {
            double s = 0.0;
            for (int64_t j = 0; j < Dv; ++j) s += dS[c * Dv + j] * beta * u[t * Dv + j];
            dk[c] = s;
        }
        for (int64_t j = 0; j < Dv; ++j) {
            double s = 0.0;
            for (int64_t c = 0; c < Dk; ++c) s += dS[c * Dv + j] * (double)k[c];
            dr[j] = s;
        }
        double db = 0.0;
        for (int64_t j = 0; j < Dv; ++j) db += dr[j] * u[t * Dv + j];
        a->dbeta[t * a->sb] = db;
        for (int64_t j = 0; j < Dv; ++j) dv[j] = beta * dr[j];
        for (int64_t c = 0; c < Dk; ++c)
            for (int64_t j = 0; j < Dv; ++j) dX[c * Dv + j] = dS[c * Dv + j] + (double)k[c] * (-beta * dr[j]);
        for (int64_t c = 0; c < Dk; ++c) {
            const double alc = al[t * Dk + c];
            double s = 0.0, da = 0.0;
            for (int64_t j = 0; j < Dv; ++j) {
                s += alc * Sp[c * Dv + j] * (-beta * dr[j]);
                da += dX[c * Dv + j] * Sp[c * Dv + j];
            }
            dk[c] += s;
            const double dg = da * alc;
            if (a->log_decay) {
                a->dg[t * a->sk + c] = dg;
            } else {
                const double sz = sig((double)a->z[t * a->sk + c]);
                a->dg[t * a->sk + c] = dg * a->g_min * sz * (1.0 - sz);
            }
            for (int64_t j = 0; j < Dv; ++j) dS[c * Dv + j] = alc * dX[c * Dv + j];
        }
    }
    if (a->dS0) memcpy(a->dS0, dS, sizeof(double) * (size_t)N);
    free(St); free(al); free(u); free(dS); free(dX); free(dr);
    return 0;
}

typedef struct {
    bwd_seq_t *seqs;
    int64_t n, next;
    pthread_mutex_t mu;
    int failed;
} bpool_t;

static void *bworker(void *p)
{
    bpool_t *pool = (bpool_t *)p;
    for (;;) {
        pthread_mutex_lock(&pool->mu);
        const int64_t i = pool->next++;
        pthread_mutex_unlock(&pool->mu);
        if (i >= pool->n) break;
        if (run_bwd(&pool->seqs[i]) != 0) {
            pthread_mutex_lock(&pool->mu);
            pool->failed = 1;
            pthread_mutex_unlock(&pool->mu);
        }
    }
    return NULL;
}

/*
 * Gradient of the batched recurrence (layout as kda_oracle_recurrence):
 *   q, k, z, log_decay (B,S,H,Dk); v, dO (B,S,H,Dv); beta (B,S,H); S0, dST (B,H,Dk,Dv) or NULL.
 * Outputs (fp64, same layouts): dq, dk (B,S,H,Dk); dv (B,S,H,Dv); dbeta (B,S,H);
 * dg (B,S,H,Dk) = d/dz if z is given, else d/dlog_decay; dS0 (B,H,Dk,Dv) or NULL.
 * Returns 0, -1 on bad arguments, -2 on allocation failure.
 */
int kda_oracle_recurrence_bwd(int64_t B, int64_t S, int64_t H, int64_t Dk, int64_t Dv,
                              const float *q, const float *k, const float *v, const float *z,
                              const float *log_decay, const float *beta, double g_min, const float *S0,
                              const float *dO, const float *dST,
                              double *dq, double *dk, double *dv, double *dbeta, double *dg, double *dS0,
                              int nthreads)
{
    if (B < 0 || S < 0 || H <= 0 || Dk <= 0 || Dv <= 0) return -1;
    if (!q || !k || !v || !beta || !dO || !dq || !dk || !dv || !dbeta || !dg) return -1;
    if (!z && !log_decay) return -1;
    const int64_t n = B * H;
    if (n == 0) return 0;
    bwd_seq_t *seqs = (bwd_seq_t *)calloc((size_t)n, sizeof(bwd_seq_t));
    if (!seqs) return -2;
    for (int64_t b = 0; b < B; ++b)
        for (int64_t h = 0; h < H; ++h) {
            bwd_seq_t *s = &seqs[b * H + h];
            const int64_t rk = (b * S * H + h) * Dk, rv = (b * S * H + h) * Dv, rb = b * S * H + h;
            s->S = S; s->Dk = Dk; s->Dv = Dv; s->sk = H * Dk; s->sv = H * Dv; s->sb = H;
            s->q = q + rk; s->k = k + rk; s->v = v + rv;
            s->z = z ? z + rk : NULL;
            s->log_decay = log_decay ? log_decay + rk : NULL;
            s->beta = beta + rb; s->dO = dO + rv;
            s->S0 = S0 ? S0 + (b * H + h) * Dk * Dv : NULL;
            s->dST = dST ? dST + (b * H + h) * Dk * Dv : NULL;
            s->g_min = g_min;
            s->dq = dq + rk; s->dk = dk + rk; s->dv = dv + rv; s->dbeta = dbeta + rb; s->dg = dg + rk;
            s->dS0 = dS0 ? dS0 + (b * H + h) * Dk * Dv : NULL;
        }
    bpool_t pool;
    pool.seqs = seqs; pool.n = n; pool.next = 0; pool.failed = 0;
    pthread_mutex_init(&pool.mu, NULL);
    if (nthreads < 1) nthreads = 1;
    if (nthreads > n) nthreads = (int)n;
    pthread_t *th = (pthread_t *)malloc(sizeof(pthread_t) * (size_t)nthreads);
    int started = 0;
    if (th)
        for (int i = 1; i < nthreads; ++i) {
            if (pthread_create(&th[i], NULL, bworker, &pool) != 0) break;
            ++started;
        }
    bworker(&pool);
    for (int i = 1; i <= started; ++i) pthread_join(th[i], NULL);
    free(th);
    pthread_mutex_destroy(&pool.mu);
    free(seqs);
    return pool.failed ? -2 : 0;
}
