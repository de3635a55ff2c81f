/*
 * kda_oracle.c -- fp64 CPU oracle for the Kimi Delta Attention (KDA) recurrence.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may link, load or call
 * this file: only the tests, the smoke check and the CPU-baseline leg of the
 * benchmark use it.  It shares no code, header or constant with the CUDA library.
 *
 * What it computes (the plain definition, token by token, in fp64):
 *
 *   Source: wiki page "Kimi Linear 高效注意力架构" (Kimi Linear: An Expressive,
 *   Efficient Attention Architecture), section "关键技术方法 > Kimi Delta Attention
 *   (KDA)", the state-update equation
 *
 *       S_t = (I - beta_t k_t k_t^T) Diag(alpha_t) S_{t-1} + beta_t k_t v_t^T
 *
 *   with S_t a d_k x d_v matrix per head, alpha_t in [0,1]^{d_k} one decay per key
 *   channel (same section, "Channel-wise 衰减" bullet), beta_t a scalar.
 *   The pages print no read-out equation; the one used here is the standard
 *   delta-rule read-out of the post-update state, o_t = S_t^T q_t.
 *
 * Per (sequence, head) the loop below takes the steps in the equation's order:
 *   1. alpha_t = exp(log_alpha_t)                  (decay given in log space)
 *   2. S <- Diag(alpha_t) S                        (the current token's decay
 *                                                   acts on S_{t-1})
 *   3. S <- S + beta_t k_t (v_t - S^T k_t)^T       (equal to (I - beta k k^T) S
 *                                                   + beta k v^T, multiplied out)
 *   4. o_t = S^T q_t
 * The state after a sequence's last token is its final state.
 *
 * Layouts (all row-major, packed over the sequences of a batch):
 *   q, k, log_alpha : [T_total, H, d_k]      v : [T_total, H, d_v]
 *   beta            : [T_total, H]
 *   S0, S_out       : [N, H, d_k, d_v]      (S0 may be NULL: zero initial state)
 *   o               : [T_total, H, d_v]
 *   cu_seqlens      : [N + 1], cu_seqlens[0] = 0, non-decreasing; sequence n
 *                     holds tokens cu_seqlens[n] .. cu_seqlens[n+1]-1.
 *
 * Work is split over (sequence, head) units, which never interact, with one
 * POSIX thread per worker; each unit is computed by exactly the same scalar
 * loop, so the result does not depend on the number of threads.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#include <unistd.h>

typedef struct {
    const double *q, *k, *v, *log_alpha, *beta, *S0;
    const int64_t *cu_seqlens;
    int64_t num_seqs;
    int H, dk, dv;
    double *o, *S_out;
    int64_t next_unit; /* shared work counter, guarded by lock */
    pthread_mutex_t lock;
} oracle_job;

/* One (sequence, head) unit: the token loop of the recurrence. */
static void oracle_unit(oracle_job *J, int64_t seq, int h, double *S, double *y)
{
    const int H = J->H, dk = J->dk, dv = J->dv;
    const int64_t bos = J->cu_seqlens[seq], eos = J->cu_seqlens[seq + 1];

    if (J->S0)
        memcpy(S, J->S0 + ((seq * H + h) * (int64_t)dk * dv), sizeof(double) * dk * dv);
    else
        memset(S, 0, sizeof(double) * dk * dv);

    for (int64_t t = bos; t < eos; ++t) {
        const int64_t th = t * H + h;
        const double *qt = J->q + th * dk;
        const double *kt = J->k + th * dk;
        const double *vt = J->v + th * dv;
        const double *la = J->log_alpha + th * dk;
        const double bt = J->beta[th];

        /* step 2: S <- Diag(alpha_t) S, alpha_t = exp(log_alpha_t) (step 1) */
        for (int i = 0; i < dk; ++i) {
            const double a = exp(la[i]);
            for (int j = 0; j < dv; ++j)
                S[i * dv + j] *= a;
        }
        /* step 3: y = S^T k_t ; S <- S + beta_t k_t (v_t - y)^T */
        for (int j = 0; j < dv; ++j) {
            double acc = 0.0;
            for (int i = 0; i < dk; ++i)
                acc += kt[i] * S[i * dv + j];
            y[j] = acc;
        }
        for (int i = 0; i < dk; ++i) {
            const double bk = bt * kt[i];
            for (int j = 0; j < dv; ++j)
                S[i * dv + j] += bk * (vt[j] - y[j]);
        }
        /* step 4: o_t = S_t^T q_t */
        double *ot = J->o + th * dv;
        for (int j = 0; j < dv; ++j) {
            double acc = 0.0;
            for (int i = 0; i < dk; ++i)
                acc += qt[i] * S[i * dv + j];
            ot[j] = acc;
        }
    }
    memcpy(J->S_out + ((seq * H + h) * (int64_t)dk * dv), S, sizeof(double) * dk * dv);
}

static void *oracle_worker(void *arg)
{
    oracle_job *J = (oracle_job *)arg;
    double *S = (double *)malloc(sizeof(double) * (size_t)J->dk * J->dv);
    double *y = (double *)malloc(sizeof(double) * (size_t)J->dv);
    const int64_t units = J->num_seqs * J->H;
    for (;;) {
        pthread_mutex_lock(&J->lock);
        const int64_t u = J->next_unit++;
        pthread_mutex_unlock(&J->lock);
        if (u >= units)
            break;
        oracle_unit(J, u / J->H, (int)(u % J->H), S, y);
    }
    free(y);
    free(S);
    return NULL;
}

/* Number of worker threads the oracle uses when asked for 0 (= all cores). */
int kda_oracle_default_threads(void)
{
    long n = sysconf(_SC_NPROCESSORS_ONLN);
    return n > 0 ? (int)n : 1;
}

/*
 * kda_oracle_prefill: run the recurrence over every (sequence, head) of a packed
 * batch.  Returns 0 on success, -1 on bad arguments.  nthreads <= 0 uses all
 * online cores.  All arrays are caller-owned fp64 host memory.
 */
int kda_oracle_prefill(const double *q, const double *k, const double *v,
                       const double *log_alpha, const double *beta, const double *S0,
                       const int64_t *cu_seqlens, int64_t num_seqs, int H, int dk, int dv,
                       double *o, double *S_out, int nthreads)
{
    if (!q || !k || !v || !log_alpha || !beta || !cu_seqlens || !o || !S_out)
        return -1;
    if (num_seqs < 0 || H <= 0 || dk <= 0 || dv <= 0)
        return -1;
    if (cu_seqlens[0] != 0)
        return -1;
    for (int64_t n = 0; n < num_seqs; ++n)
        if (cu_seqlens[n + 1] < cu_seqlens[n])
            return -1;

    oracle_job J;
    J.q = q; J.k = k; J.v = v; J.log_alpha = log_alpha; J.beta = beta; J.S0 = S0;
    J.cu_seqlens = cu_seqlens; J.num_seqs = num_seqs; J.H = H; J.dk = dk; J.dv = dv;
    J.o = o; J.S_out = S_out; J.next_unit = 0;
    pthread_mutex_init(&J.lock, NULL);

    if (nthreads <= 0)
        nthreads = kda_oracle_default_threads();
    const int64_t units = num_seqs * H;
    if (nthreads > units)
        nthreads = units > 0 ? (int)units : 1;

    pthread_t *tid = (pthread_t *)malloc(sizeof(pthread_t) * nthreads);
    int started = 0;
    for (int w = 1; w < nthreads; ++w)
        if (pthread_create(&tid[started], NULL, oracle_worker, &J) == 0)
            ++started;
    /* the calling thread works too; then join the helpers it started */
    oracle_worker(&J);
    for (int w = 0; w < started; ++w)
        pthread_join(tid[w], NULL);
    free(tid);
    pthread_mutex_destroy(&J.lock);
    return 0;
}
