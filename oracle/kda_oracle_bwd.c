/*
 * kda_oracle_bwd.c -- fp64 CPU oracle of the gradients of the KDA recurrence.
 *
 * TEST INFRASTRUCTURE ONLY (same rule as kda_oracle.c): only the tests may use it; it
 * shares no code, header or constant with the CUDA library.
 *
 * The forward map is the state-update equation of the wiki page "Kimi Linear
 * 高效注意力架构", section "关键技术方法 > Kimi Delta Attention (KDA)", with the
 * delta-rule read-out of the post-update state, token by token:
 *
 *   St~ = Diag(alpha_t) S_{t-1},  y_t = St~^T k_t,  u_t = beta_t (v_t - y_t),
 *   S_t = St~ + k_t u_t^T,        o_t = S_t^T q_t,   alpha_t = exp(log_alpha_t).
 *
 * Given dO = dL/do_t for every token and dS_T = dL/dS_final (NULL = 0), this file
 * runs the reverse-mode (adjoint) sweep of that map exactly, token by token, with
 * G = dL/dS_t carried backwards:
 *
 *   G += q_t do_t^T                        dq_t = S_t do_t
 *   du = G^T k_t                           dv_t = beta_t du
 *   dbeta_t = du . (v_t - y_t)             dy = -beta_t du
 *   dSt~ = G + k_t dy^T                    dk_t = G u_t + St~ dy
 *   dlog_alpha_t[i] = sum_j dSt~[i][j] St~[i][j]
 *   G <- Diag(alpha_t) dSt~                (= dL/dS_{t-1});   dS0 = G at the start.
 *
 * States are recomputed from checkpoints every 64 tokens, in fp64.  Work is split
 * over (sequence, head) units with POSIX threads, as in kda_oracle.c.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#include <unistd.h>

enum { CK = 64 };

typedef struct {
    const double *q, *k, *v, *log_alpha, *beta, *S0, *dO, *dS_final;
    const int64_t *cu_seqlens;
    int64_t num_seqs;
    int H, dk, dv;
    double *dq, *dk_, *dv_, *dlog_alpha, *dbeta, *dS0;
    int64_t next_unit;
    pthread_mutex_t lock;
} bwd_job;

typedef struct {
    double *ck;    /* checkpoints: state before tokens bos, bos + CK, ... */
    double *sbuf;  /* states after each token of one block */
    double *G, *St, *dSt, *y, *u, *du, *dy;
    int64_t ck_cap;
} bwd_scratch;

/* S <- state after token t, from the state before it (in place). Writes y and u. */
static void step_forward(const bwd_job *J, int64_t th, double *S, double *y, double *u)
{
    const int dk = J->dk, dv = J->dv;
    const double *kt = J->k + th * dk, *vt = J->v + th * dv, *la = J->log_alpha + th * dk;
    const double bt = J->beta[th];
    for (int i = 0; i < dk; ++i) {
        const double a = exp(la[i]);
        for (int j = 0; j < dv; ++j) S[i * dv + j] *= a;
    }
    for (int j = 0; j < dv; ++j) {
        double acc = 0.0;
        for (int i = 0; i < dk; ++i) acc += kt[i] * S[i * dv + j];
        y[j] = acc;
        u[j] = bt * (vt[j] - acc);
    }
    for (int i = 0; i < dk; ++i)
        for (int j = 0; j < dv; ++j) S[i * dv + j] += kt[i] * u[j];
}

static void bwd_unit(bwd_job *J, bwd_scratch *W, int64_t seq, int h)
{
    const int H = J->H, dk = J->dk, dv = J->dv;
    const int64_t bos = J->cu_seqlens[seq], eos = J->cu_seqlens[seq + 1], L = eos - bos;
    const int64_t nblk = (L + CK - 1) / CK, sz = (int64_t)dk * dv;
    double *ck = W->ck, *sb = W->sbuf, *G = W->G, *St = W->St, *dSt = W->dSt;
    double *y = W->y, *u = W->u, *du = W->du, *dy = W->dy;

    /* forward sweep: checkpoints */
    if (J->S0) memcpy(ck, J->S0 + (seq * H + h) * sz, sizeof(double) * sz);
    else memset(ck, 0, sizeof(double) * sz);
    for (int64_t b = 1; b <= nblk; ++b) {
        memcpy(ck + b * sz, ck + (b - 1) * sz, sizeof(double) * sz);
        const int64_t t1 = bos + b * CK < eos ? bos + b * CK : eos;
        for (int64_t t = bos + (b - 1) * CK; t < t1; ++t) step_forward(J, t * H + h, ck + b * sz, y, u);
    }
    /* adjoint sweep */
    if (J->dS_final) memcpy(G, J->dS_final + (seq * H + h) * sz, sizeof(double) * sz);
    else memset(G, 0, sizeof(double) * sz);
    for (int64_t b = nblk - 1; b >= 0; --b) {
        const int64_t t0 = bos + b * CK, t1 = t0 + CK < eos ? t0 + CK : eos;
        /* states after each token of the block */
        memcpy(St, ck + b * sz, sizeof(double) * sz);
        for (int64_t t = t0; t < t1; ++t) {
            step_forward(J, t * H + h, St, y, u);
            memcpy(sb + (t - t0) * sz, St, sizeof(double) * sz);
        }
        for (int64_t t = t1 - 1; t >= t0; --t) {
            const int64_t th = t * H + h;
            const double *qt = J->q + th * dk, *kt = J->k + th * dk, *vt = J->v + th * dv;
            const double *la = J->log_alpha + th * dk, *dot = J->dO + th * dv;
            const double bt = J->beta[th];
            const double *Sprev = t > t0 ? sb + (t - 1 - t0) * sz : ck + b * sz;
            const double *Snow = sb + (t - t0) * sz;
            /* St~ = Diag(alpha) S_{t-1}; y, u */
            for (int i = 0; i < dk; ++i) {
                const double a = exp(la[i]);
                for (int j = 0; j < dv; ++j) St[i * dv + j] = a * Sprev[i * dv + j];
            }
            for (int j = 0; j < dv; ++j) {
                double acc = 0.0;
                for (int i = 0; i < dk; ++i) acc += kt[i] * St[i * dv + j];
                y[j] = acc;
                u[j] = bt * (vt[j] - acc);
            }
            /* G += q do^T; dq = S_t do */
            for (int i = 0; i < dk; ++i)
                for (int j = 0; j < dv; ++j) G[i * dv + j] += qt[i] * dot[j];
            double *dqt = J->dq + th * dk;
            for (int i = 0; i < dk; ++i) {
                double acc = 0.0;
                for (int j = 0; j < dv; ++j) acc += Snow[i * dv + j] * dot[j];
                dqt[i] = acc;
            }
            /* du = G^T k; dv = beta du; dbeta = du . (v - y); dy = -beta du */
            double db = 0.0;
            double *dvt = J->dv_ + th * dv;
            for (int j = 0; j < dv; ++j) {
                double acc = 0.0;
                for (int i = 0; i < dk; ++i) acc += G[i * dv + j] * kt[i];
                du[j] = acc;
                dvt[j] = bt * acc;
                db += acc * (vt[j] - y[j]);
                dy[j] = -bt * acc;
            }
            J->dbeta[th] = db;
            /* dSt~ = G + k dy^T; dk = G u + St~ dy; dlog_alpha = rowsum(dSt~ * St~) */
            double *dkt = J->dk_ + th * dk, *dlt = J->dlog_alpha + th * dk;
            for (int i = 0; i < dk; ++i) {
                double ak = 0.0, al = 0.0;
                for (int j = 0; j < dv; ++j) {
                    const double g = G[i * dv + j] + kt[i] * dy[j];
                    dSt[i * dv + j] = g;
                    ak += G[i * dv + j] * u[j] + St[i * dv + j] * dy[j];
                    al += g * St[i * dv + j];
                }
                dkt[i] = ak;
                dlt[i] = al;
            }
            /* G <- Diag(alpha) dSt~ */
            for (int i = 0; i < dk; ++i) {
                const double a = exp(la[i]);
                for (int j = 0; j < dv; ++j) G[i * dv + j] = a * dSt[i * dv + j];
            }
        }
    }
    memcpy(J->dS0 + (seq * H + h) * sz, G, sizeof(double) * sz);
}

static void *bwd_worker(void *arg)
{
    bwd_job *J = (bwd_job *)arg;
    const int64_t sz = (int64_t)J->dk * J->dv;
    int64_t maxlen = 0;
    for (int64_t n = 0; n < J->num_seqs; ++n) {
        const int64_t L = J->cu_seqlens[n + 1] - J->cu_seqlens[n];
        if (L > maxlen) maxlen = L;
    }
    bwd_scratch W;
    W.ck_cap = (maxlen + CK - 1) / CK + 1;
    W.ck = (double *)malloc(sizeof(double) * sz * W.ck_cap);
    W.sbuf = (double *)malloc(sizeof(double) * sz * CK);
    W.G = (double *)malloc(sizeof(double) * sz);
    W.St = (double *)malloc(sizeof(double) * sz);
    W.dSt = (double *)malloc(sizeof(double) * sz);
    W.y = (double *)malloc(sizeof(double) * J->dv);
    W.u = (double *)malloc(sizeof(double) * J->dv);
    W.du = (double *)malloc(sizeof(double) * J->dv);
    W.dy = (double *)malloc(sizeof(double) * J->dv);
    const int64_t units = J->num_seqs * J->H;
    for (;;) {
        pthread_mutex_lock(&J->lock);
        const int64_t un = J->next_unit++;
        pthread_mutex_unlock(&J->lock);
        if (un >= units) break;
        bwd_unit(J, &W, un / J->H, (int)(un % J->H));
    }
    free(W.ck); free(W.sbuf); free(W.G); free(W.St); free(W.dSt);
    free(W.y); free(W.u); free(W.du); free(W.dy);
    return NULL;
}

/*
 * kda_oracle_backward: gradients of L = sum_t <dO_t, o_t> + <dS_final, S_final> with
 * respect to q, k, v, log_alpha, beta and S0.  Layouts as in kda_oracle_prefill;
 * dO [T_total, H, d_v]; dS_final and dS0 [N, H, d_k, d_v] (dS_final may be NULL).
 * Returns 0, or -1 on bad arguments.
 */
int kda_oracle_backward(const double *q, const double *k, const double *v, const double *log_alpha,
                        const double *beta, const double *S0, const double *dO, const double *dS_final,
                        const int64_t *cu_seqlens, int64_t num_seqs, int H, int dk, int dv,
                        double *dq, double *dk_, double *dv_, double *dlog_alpha, double *dbeta,
                        double *dS0, int nthreads)
{
    if (!q || !k || !v || !log_alpha || !beta || !dO || !cu_seqlens || !dq || !dk_ || !dv_ ||
        !dlog_alpha || !dbeta || !dS0)
        return -1;
    if (num_seqs < 0 || H <= 0 || dk <= 0 || dv <= 0 || cu_seqlens[0] != 0) return -1;
    for (int64_t n = 0; n < num_seqs; ++n)
        if (cu_seqlens[n + 1] < cu_seqlens[n]) return -1;
    bwd_job J;
    J.q = q; J.k = k; J.v = v; J.log_alpha = log_alpha; J.beta = beta; J.S0 = S0;
    J.dO = dO; J.dS_final = dS_final; J.cu_seqlens = cu_seqlens; J.num_seqs = num_seqs;
    J.H = H; J.dk = dk; J.dv = dv;
    J.dq = dq; J.dk_ = dk_; J.dv_ = dv_; J.dlog_alpha = dlog_alpha; J.dbeta = dbeta; J.dS0 = dS0;
    J.next_unit = 0;
    pthread_mutex_init(&J.lock, NULL);
    if (nthreads <= 0) {
        const long n = sysconf(_SC_NPROCESSORS_ONLN);
        nthreads = n > 0 ? (int)n : 1;
    }
    const int64_t units = num_seqs * H;
    if (nthreads > units) nthreads = units > 0 ? (int)units : 1;
    pthread_t *th = (pthread_t *)malloc(sizeof(pthread_t) * nthreads);
    for (int i = 0; i < nthreads; ++i) pthread_create(&th[i], NULL, bwd_worker, &J);
    for (int i = 0; i < nthreads; ++i) pthread_join(th[i], NULL);
    free(th);
    pthread_mutex_destroy(&J.lock);
    return 0;
}
