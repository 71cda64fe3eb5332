/*
 * gdn2_oracle.c -- float64 token-by-token reference of the channel-wise gated
 * delta rule (GDN-2 state update with the Muir readout).
 *
 * TEST INFRASTRUCTURE.  Only the tests, the smoke check and the CPU-baseline
 * leg of the benchmark may load this library.  The CUDA product path shares no
 * code with it.
 *
 * What it computes, per head, for t = 0..T-1 (row-vector convention; S is
 * d_k x d_v; "Muir review" = the review page of arXiv:2611.08376 "Muir: Linear
 * Attention with Sensitivity-Allocated Gating and Matched-Filter Readout"):
 *
 *   alpha_t = exp(log_alpha_t)                         per key channel
 *   S_hat   = Diag(alpha_t) S                          Muir review §2.1
 *   r       = k_t S_hat                                (1 x d_v)
 *   S       = S_hat - (b_t*k_t)^T r + k_t^T (w_t*v_t)  erase along the key with
 *                                                      the erase gate, write the
 *                                                      value through the write
 *                                                      gate (Muir review §2.1;
 *                                                      the display equation is
 *                                                      lost on the page, this is
 *                                                      the form the reductions
 *                                                      to KDA / Gated DeltaNet /
 *                                                      DeltaNet fix)
 *   q_til   = q_t * gamma_stat * 2*sigmoid(z_t)        readout gain scales the
 *                                                      query only (§2.1)
 *   o_t     = q_til S                                  read after the write
 *                                                      ("Kimi3 = GPT2 x 22580"
 *                                                      §3: o = q @ S after the
 *                                                      update, no denominator)
 *   y_t     = g_t * o_t / sqrt(mean_j o_tj^2 + eps)    per-head RMSNorm, then the
 *                                                      channel-wise output gate
 *                                                      (Muir review §2.1)
 *
 * Value columns of S evolve independently (column j only ever meets column j
 * of S), so the work is split over (head, block of value columns) and run on
 * a pool of POSIX threads.  Nothing is blocked, fused or reordered inside a
 * column block beyond the loop order written above.
 *
 * Parity: pinned by the tests under tests/test_oracle_pins.py (reductions to
 * KDA, Gated DeltaNet and DeltaNet, exact retrieval, causal linear attention,
 * the pages' chunked algorithm, split runs, erase-only invariants).
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#include <unistd.h>

#define COLS_PER_TASK 16

typedef struct {
    int n_heads, T, dk, dv;
    const double *q, *k, *v, *b, *w, *z, *g, *log_alpha; /* [n][T][d] */
    const double *gamma_stat;                           /* [n][dk] */
    double *S;                                          /* [n][dk][dv] in/out */
    double *o_raw;                                      /* [n][T][dv] */
    int n_tasks;
    int next;
    pthread_mutex_t lock;
} job_t;

static int take_task(job_t *job) {
    pthread_mutex_lock(&job->lock);
    int t = job->next < job->n_tasks ? job->next++ : -1;
    pthread_mutex_unlock(&job->lock);
    return t;
}

static void run_task(job_t *job, int task) {
    const int dk = job->dk, dv = job->dv, T = job->T;
    const int blocks = (dv + COLS_PER_TASK - 1) / COLS_PER_TASK;
    const int h = task / blocks;
    const int j0 = (task % blocks) * COLS_PER_TASK;
    const int nb = (dv - j0) < COLS_PER_TASK ? (dv - j0) : COLS_PER_TASK;

    double *Sblk = (double *)malloc(sizeof(double) * (size_t)dk * COLS_PER_TASK);
    double *alpha = (double *)malloc(sizeof(double) * (size_t)dk);
    double *qt = (double *)malloc(sizeof(double) * (size_t)dk);
    double r[COLS_PER_TASK], vh[COLS_PER_TASK], o[COLS_PER_TASK];

    double *S = job->S + (size_t)h * dk * dv;
    for (int i = 0; i < dk; ++i)
        for (int j = 0; j < nb; ++j) Sblk[i * COLS_PER_TASK + j] = S[(size_t)i * dv + j0 + j];

    const double *gs = job->gamma_stat + (size_t)h * dk;
    for (int t = 0; t < T; ++t) {
        const size_t rk = ((size_t)h * T + t) * dk, rv = ((size_t)h * T + t) * dv;
        const double *q = job->q + rk, *k = job->k + rk, *b = job->b + rk;
        const double *z = job->z + rk, *la = job->log_alpha + rk;
        const double *v = job->v + rv, *w = job->w + rv;
        for (int i = 0; i < dk; ++i) {
            alpha[i] = exp(la[i]);
            qt[i] = q[i] * gs[i] * (2.0 / (1.0 + exp(-z[i])));
        }
        for (int j = 0; j < nb; ++j) vh[j] = w[j0 + j] * v[j0 + j];

        /* S_hat = Diag(alpha) S */
        for (int i = 0; i < dk; ++i)
            for (int j = 0; j < nb; ++j) Sblk[i * COLS_PER_TASK + j] *= alpha[i];
        /* r = k S_hat */
        for (int j = 0; j < nb; ++j) r[j] = 0.0;
        for (int i = 0; i < dk; ++i)
            for (int j = 0; j < nb; ++j) r[j] += k[i] * Sblk[i * COLS_PER_TASK + j];
        /* S = S_hat - (b*k)^T r + k^T (w*v) */
        for (int i = 0; i < dk; ++i) {
            const double kh = b[i] * k[i];
            for (int j = 0; j < nb; ++j)
                Sblk[i * COLS_PER_TASK + j] += -kh * r[j] + k[i] * vh[j];
        }
        /* o = q_til S */
        for (int j = 0; j < nb; ++j) o[j] = 0.0;
        for (int i = 0; i < dk; ++i)
            for (int j = 0; j < nb; ++j) o[j] += qt[i] * Sblk[i * COLS_PER_TASK + j];
        double *orow = job->o_raw + rv;
        for (int j = 0; j < nb; ++j) orow[j0 + j] = o[j];
    }

    for (int i = 0; i < dk; ++i)
        for (int j = 0; j < nb; ++j) S[(size_t)i * dv + j0 + j] = Sblk[i * COLS_PER_TASK + j];
    free(Sblk);
    free(alpha);
    free(qt);
}

static void *worker(void *arg) {
    job_t *job = (job_t *)arg;
    for (int task; (task = take_task(job)) >= 0;) run_task(job, task);
    return NULL;
}

int oracle_num_threads(void) {
    long n = sysconf(_SC_NPROCESSORS_ONLN);
    return n > 0 ? (int)n : 1;
}

/*
 * Runs the recurrence for n_heads independent heads.  Inputs are float64,
 * contiguous [n_heads][T][d]; gamma_stat is [n_heads][dk] (one profile per
 * head, the caller gathers it); S is [n_heads][dk][dv], read as S_0 and
 * overwritten with S_T; o_raw and y are [n_heads][T][dv] outputs.
 * Returns the number of threads used, or -1 on a bad argument.
 */
int oracle_gdn2_forward(int n_heads, int T, int dk, int dv, const double *q, const double *k,
                        const double *v, const double *b, const double *w, const double *z,
                        const double *g, const double *log_alpha, const double *gamma_stat,
                        double *S, double *o_raw, double *y, double eps, int n_threads) {
    if (n_heads < 0 || T < 0 || dk <= 0 || dv <= 0) return -1;
    if (n_heads == 0 || T == 0) return 0;
    job_t job;
    memset(&job, 0, sizeof(job));
    job.n_heads = n_heads; job.T = T; job.dk = dk; job.dv = dv;
    job.q = q; job.k = k; job.v = v; job.b = b; job.w = w; job.z = z; job.g = g;
    job.log_alpha = log_alpha; job.gamma_stat = gamma_stat; job.S = S; job.o_raw = o_raw;
    const int blocks = (dv + COLS_PER_TASK - 1) / COLS_PER_TASK;
    job.n_tasks = n_heads * blocks;
    job.next = 0;
    pthread_mutex_init(&job.lock, NULL);

    if (n_threads <= 0) n_threads = oracle_num_threads();
    if (n_threads > job.n_tasks) n_threads = job.n_tasks;
    pthread_t *th = (pthread_t *)malloc(sizeof(pthread_t) * (size_t)n_threads);
    for (int i = 0; i < n_threads; ++i) pthread_create(&th[i], NULL, worker, &job);
    for (int i = 0; i < n_threads; ++i) pthread_join(th[i], NULL);
    free(th);
    pthread_mutex_destroy(&job.lock);

    /* y = g * o / sqrt(mean(o^2) + eps), per head and token over d_v */
    for (size_t row = 0; row < (size_t)n_heads * T; ++row) {
        const double *o = o_raw + row * dv, *gg = g + row * dv;
        double ss = 0.0;
        for (int j = 0; j < dv; ++j) ss += o[j] * o[j];
        const double inv = 1.0 / sqrt(ss / dv + eps);
        for (int j = 0; j < dv; ++j) y[row * dv + j] = gg[j] * o[j] * inv;
    }
    return n_threads;
}
