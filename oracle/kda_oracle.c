/*
 * TEST INFRASTRUCTURE — the fp64 CPU oracle for the Kimi Delta Attention (KDA)
 * recurrence.  Only tests/, __graft_entry__.smoke() and bench.py's cpu_baseline
 * leg may load this file's library.  It shares no code, header or constant with
 * the CUDA library and must never be called from the product path.
 *
 * What it computes (plain definition, token by token, fp64):
 *
 *   alpha_t   = exp(g_min * sigmoid(z_t))                      per key channel
 *               ("KDA Recurrence" problem page, decay-gate formula)
 *   S_t       = (I - beta_t k_t k_t^T) Diag(alpha_t) S_{t-1} + beta_t k_t v_t^T
 *               (Kimi Linear report, section 3, Eq. 1; the same update is
 *                restated on the "KDA Recurrence" page and as Eq. 1 of the
 *                "Diagonal-Plus-Low-Rank Matrices and Kimi Delta Attention" post)
 *   o~_t      = S_t^T q_t, read from the UPDATED state
 *               ("KDA Recurrence" page: "read from the updated state")
 *
 * S is a D_k x D_v matrix (row index = key channel, column index = value
 * channel), stored row-major.  The product (I - beta k k^T) X with
 * X = Diag(alpha) S is evaluated as X - beta k (k^T X): the same matrix product
 * written with the rank-1 factor applied by associativity, no other
 * reordering.  Parity of this form against explicitly formed D_k x D_k
 * transition matrices is one of the oracle's pins.
 *
 * Inputs are single-precision arrays whose values (fp32, or bf16 widened to
 * fp32) are promoted to fp64 before any arithmetic.  All arithmetic is fp64.
 * Compiled with IEEE semantics (no fast-math).
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* One independent sequence: a fixed batch row b and head h.  Row strides are
 * in elements and give the distance between consecutive tokens. */
typedef struct {
    int64_t S, Dk, Dv;
    const float *q, *k, *z, *log_decay; /* rows of Dk, stride sk          */
    const float *v;                     /* rows of Dv, stride sv          */
    const float *beta;                  /* one per token, stride sb       */
    int64_t sk, sv, sb;
    double g_min;
    const float *S0;                    /* Dk x Dv row-major, or NULL (=0) */
    double *S_final;                    /* Dk x Dv row-major, out         */
    double *o;                          /* n_rec rows of Dv, stride so    */
    int64_t so;
    const int64_t *t_rec;               /* sorted token indices to record, or NULL = all */
    int64_t n_rec;
} kda_seq_t;

static double sigmoid_d(double x) { return 1.0 / (1.0 + exp(-x)); }

static void run_sequence(const kda_seq_t *a, double *S, double *alpha,
                         double *ktx, double *kv)
{
    const int64_t Dk = a->Dk, Dv = a->Dv;
    if (a->S0) {
        for (int64_t i = 0; i < Dk * Dv; ++i) S[i] = (double)a->S0[i];
    } else {
        memset(S, 0, sizeof(double) * (size_t)(Dk * Dv));
    }
    int64_t rec = 0;
    for (int64_t t = 0; t < a->S; ++t) {
        const float *q = a->q + t * a->sk;
        const float *k = a->k + t * a->sk;
        const float *v = a->v + t * a->sv;
        const double beta = (double)a->beta[t * a->sb];

        /* alpha_t = exp(g_min * sigmoid(z_t)); a caller may instead supply
         * log(alpha_t) directly (used by the closed-form special cases). */
        for (int64_t c = 0; c < Dk; ++c) {
            if (a->log_decay) {
                alpha[c] = exp((double)a->log_decay[t * a->sk + c]);
            } else {
                const double zc = (double)a->z[t * a->sk + c];
                alpha[c] = exp(a->g_min * sigmoid_d(zc));
            }
        }
        /* X = Diag(alpha_t) S_{t-1} */
        for (int64_t c = 0; c < Dk; ++c)
            for (int64_t j = 0; j < Dv; ++j) S[c * Dv + j] *= alpha[c];
        /* k^T X */
        for (int64_t j = 0; j < Dv; ++j) ktx[j] = 0.0;
        for (int64_t c = 0; c < Dk; ++c) {
            const double kc = (double)k[c];
            for (int64_t j = 0; j < Dv; ++j) ktx[j] += kc * S[c * Dv + j];
        }
        /* S_t = X - beta k (k^T X) + beta k v^T */
        for (int64_t j = 0; j < Dv; ++j) kv[j] = (double)v[j];
        for (int64_t c = 0; c < Dk; ++c) {
            const double kc = (double)k[c];
            for (int64_t j = 0; j < Dv; ++j)
                S[c * Dv + j] += -beta * kc * ktx[j] + beta * kc * kv[j];
        }
        /* o~_t = S_t^T q_t (updated state) */
        int record = 0;
        if (a->o) {
            if (!a->t_rec) record = 1;
            else if (rec < a->n_rec && a->t_rec[rec] == t) record = 1;
        }
        if (record) {
            double *o = a->o + rec * a->so;
            for (int64_t j = 0; j < Dv; ++j) o[j] = 0.0;
            for (int64_t c = 0; c < Dk; ++c) {
                const double qc = (double)q[c];
                for (int64_t j = 0; j < Dv; ++j) o[j] += qc * S[c * Dv + j];
            }
            ++rec;
        }
    }
    if (a->S_final) memcpy(a->S_final, S, sizeof(double) * (size_t)(Dk * Dv));
}

typedef struct {
    const kda_seq_t *seqs;
    int64_t n;
    int64_t next;
    pthread_mutex_t mu;
    int64_t Dk, Dv;
    int failed;
} pool_t;

static void *worker(void *p)
{
    pool_t *pool = (pool_t *)p;
    double *S = (double *)malloc(sizeof(double) * (size_t)(pool->Dk * pool->Dv));
    double *alpha = (double *)malloc(sizeof(double) * (size_t)pool->Dk);
    double *ktx = (double *)malloc(sizeof(double) * (size_t)pool->Dv);
    double *kv = (double *)malloc(sizeof(double) * (size_t)pool->Dv);
    if (!S || !alpha || !ktx || !kv) {
        pthread_mutex_lock(&pool->mu);
        pool->failed = 1;
        pthread_mutex_unlock(&pool->mu);
    } else {
        for (;;) {
            pthread_mutex_lock(&pool->mu);
            const int64_t i = pool->next++;
            pthread_mutex_unlock(&pool->mu);
            if (i >= pool->n) break;
            run_sequence(&pool->seqs[i], S, alpha, ktx, kv);
        }
    }
    free(S); free(alpha); free(ktx); free(kv);
    return NULL;
}

/*
 * Batched recurrence over the "KDA Recurrence" page's layout:
 *   q, k, z, log_decay : (B, S, H, Dk)      v : (B, S, H, Dv)
 *   beta               : (B, S, H)          S0: (B, H, Dk, Dv) or NULL (zeros)
 * Outputs:
 *   S_final : (B, H, Dk, Dv) fp64
 *   o_core  : (B, n_rec, H, Dv) fp64, o~_t for the recorded tokens
 *             (t_rec sorted ascending, or NULL to record every token,
 *             n_rec = S), or NULL to skip.
 * log_decay, when non-NULL, replaces g_min*sigmoid(z) as log(alpha).
 * Sequences (b, h) run on `nthreads` POSIX threads.  Returns 0 on success,
 * -1 on bad arguments, -2 on allocation failure.
 */
int kda_oracle_recurrence(int64_t B, int64_t S, int64_t H, int64_t Dk, int64_t Dv,
                          const float *q, const float *k, const float *v,
                          const float *z, const float *log_decay, const float *beta,
                          double g_min, const float *S0,
                          const int64_t *t_rec, int64_t n_rec,
                          double *o_core, double *S_final, int nthreads)
{
    if (B < 0 || S < 0 || H <= 0 || Dk <= 0 || Dv <= 0) return -1;
    if (!q || !k || !v || !beta || !S_final) return -1;
    if (!z && !log_decay) return -1;
    if (!t_rec) n_rec = S;
    const int64_t n = B * H;
    if (n == 0) return 0;
    kda_seq_t *seqs = (kda_seq_t *)calloc((size_t)n, sizeof(kda_seq_t));
    if (!seqs) return -2;
    for (int64_t b = 0; b < B; ++b) {
        for (int64_t h = 0; h < H; ++h) {
            kda_seq_t *s = &seqs[b * H + h];
            const int64_t rowk = (b * S * H + h) * Dk;
            const int64_t rowv = (b * S * H + h) * Dv;
            s->S = S; s->Dk = Dk; s->Dv = Dv;
            s->q = q + rowk; s->k = k + rowk;
            s->z = z ? z + rowk : NULL;
            s->log_decay = log_decay ? log_decay + rowk : NULL;
            s->v = v + rowv;
            s->beta = beta + b * S * H + h;
            s->sk = H * Dk; s->sv = H * Dv; s->sb = H;
            s->g_min = g_min;
            s->S0 = S0 ? S0 + (b * H + h) * Dk * Dv : NULL;
            s->S_final = S_final + (b * H + h) * Dk * Dv;
            s->o = o_core ? o_core + (b * n_rec * H + h) * Dv : NULL;
            s->so = H * Dv;
            s->t_rec = t_rec;
            s->n_rec = n_rec;
        }
    }
    pool_t pool;
    pool.seqs = seqs; pool.n = n; pool.next = 0; pool.Dk = Dk; pool.Dv = Dv;
    pool.failed = 0;
    pthread_mutex_init(&pool.mu, NULL);
    if (nthreads < 1) nthreads = 1;
    if (nthreads > n) nthreads = (int)n;
    pthread_t *th = (pthread_t *)malloc(sizeof(pthread_t) * (size_t)nthreads);
    int started = 0;
    if (th) {
        for (int i = 1; i < nthreads; ++i) {
            if (pthread_create(&th[i], NULL, worker, &pool) != 0) break;
            ++started;
        }
    }
    worker(&pool);
    for (int i = 1; i <= started; ++i) pthread_join(th[i], NULL);
    free(th);
    pthread_mutex_destroy(&pool.mu);
    free(seqs);
    return pool.failed ? -2 : 0;
}
