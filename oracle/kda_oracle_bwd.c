/*
 * kda_oracle_bwd.c -- fp64 CPU oracle for the gradients of Kimi Delta
 * Attention (KDA).
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path may link, load or
 * call this file; only the tests and the benchmark's CPU-baseline leg do.  It
 * shares no code, header, table or helper with the CUDA library, and none
 * with the forward oracle (kda_oracle.c) either: the forward states it needs
 * it recomputes with its own loops, so a mistake in one file cannot hide in
 * the other.
 *
 * The recurrence is that of the page "Kimi K3: Open Frontier Intelligence
 * and Implementation Framework" (section "Hybrid Attention Mechanism", KDA
 * bullet), per (sequence, head) chain, one token at a time:
 *     1. P = Diag(alpha_t) S_{t-1},   alpha_t = exp(log_alpha_t)
 *     2. e = v_t - P^T k_t
 *     3. S_t = P + beta_t k_t e^T
 *     4. o_t = S_t^T q_t
 *
 * Arithmetic: IEEE double, no fused multiply-add contraction, no fast-math,
 * plain loops; independent chains are spread over POSIX threads, one thread
 * per chain, so results do not depend on the thread count.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/*
 * Backward pass (gradients for training).
 *
 * The same page trains the model that uses KDA, so the operator needs the
 * gradients of a scalar loss L with respect to every input, given dL/do_t for
 * every token (d_out) and optionally dL/dS_final.  Nothing on the pages
 * states them; they follow from the four forward steps above by the chain
 * rule, taken in reverse order.  With G = dL/dS_t on entry to token t
 * (dS_final for the last token of a chain, zero when it is NULL):
 *     4'. o_t = S_t^T q_t         dq_t = S_t do_t;       G <- G + q_t do_t^T
 *     3'. S_t = P + beta k e^T    dP = G;  de = beta G^T k;
 *                                 dk_t = beta G e;       dbeta_t = k^T G e
 *     2'. e = v - P^T k           dv_t = de;  dP <- dP - k de^T;  dk_t <- dk_t - P de
 *     1'. P = Diag(alpha) S_{t-1} dlog_alpha_t[c] = alpha_c sum_j dP[c,j] S_{t-1}[c,j]
 *                                 G <- Diag(alpha) dP    (= dL/dS_{t-1})
 * after the chain's first token dS0 = G.  The forward states of the chain
 * are recomputed with the forward steps and kept, all of them (memory
 * (len + 1) * Dk * Dv doubles per chain: for test-sized inputs).
 *
 * Layouts as the forward; d_out [T_tot, H, Dv]; dS_final, dS0 [N, H, Dk, Dv]
 * (either may be NULL); dq, dk, dlog_alpha [T_tot, H, Dk]; dv [T_tot, H, Dv];
 * dbeta [T_tot, H].
 */
typedef struct {
    int64_t n_seqs, H, Dk, Dv;
    const int64_t *cu;
    const double *q, *k, *v, *la, *beta, *S0, *dout, *dSf;
    double *dq, *dk, *dv, *dla, *dbeta, *dS0;
    int64_t next;
    pthread_mutex_t lock;
    int failed;
} bjob_t;

static int backward_chain(bjob_t *J, int64_t n, int64_t h)
{
    const int64_t H = J->H, Dk = J->Dk, Dv = J->Dv, KV = Dk * Dv;
    const int64_t t0 = J->cu[n], t1 = J->cu[n + 1], L = t1 - t0;
    /* St[i] = state after i tokens of the chain (St[0] = S0) */
    double *St = (double *)malloc(sizeof(double) * (size_t)((L + 1) * KV));
    double *G = (double *)malloc(sizeof(double) * (size_t)KV);
    double *dP = (double *)malloc(sizeof(double) * (size_t)KV);
    double *e = (double *)malloc(sizeof(double) * (size_t)Dv);
    double *de = (double *)malloc(sizeof(double) * (size_t)Dv);
    if (!St || !G || !dP || !e || !de) {
        free(St); free(G); free(dP); free(e); free(de);
        return -2;
    }
    if (J->S0) memcpy(St, J->S0 + (n * H + h) * KV, sizeof(double) * KV);
    else memset(St, 0, sizeof(double) * KV);

    /* forward, keeping every state */
    for (int64_t i = 0; i < L; ++i) {
        const int64_t t = t0 + i;
        const double *kt = J->k + (t * H + h) * Dk, *vt = J->v + (t * H + h) * Dv;
        const double *lat = J->la + (t * H + h) * Dk;
        const double bt = J->beta[t * H + h];
        const double *Sp = St + i * KV;
        double *S = St + (i + 1) * KV;
        for (int64_t c = 0; c < Dk; ++c) {               /* 1. P = Diag(alpha) S_{t-1} */
            const double a = exp(lat[c]);
            for (int64_t j = 0; j < Dv; ++j) S[c * Dv + j] = a * Sp[c * Dv + j];
        }
        for (int64_t j = 0; j < Dv; ++j) e[j] = 0.0;     /* 2. e = v - P^T k */
        for (int64_t c = 0; c < Dk; ++c)
            for (int64_t j = 0; j < Dv; ++j) e[j] = e[j] + kt[c] * S[c * Dv + j];
        for (int64_t j = 0; j < Dv; ++j) e[j] = vt[j] - e[j];
        for (int64_t c = 0; c < Dk; ++c)                 /* 3. S = P + beta k e^T */
            for (int64_t j = 0; j < Dv; ++j) S[c * Dv + j] = S[c * Dv + j] + bt * kt[c] * e[j];
    }

    if (J->dSf) memcpy(G, J->dSf + (n * H + h) * KV, sizeof(double) * KV);
    else memset(G, 0, sizeof(double) * KV);

    for (int64_t i = L - 1; i >= 0; --i) {
        const int64_t t = t0 + i;
        const double *qt = J->q + (t * H + h) * Dk, *kt = J->k + (t * H + h) * Dk;
        const double *vt = J->v + (t * H + h) * Dv, *lat = J->la + (t * H + h) * Dk;
        const double *dot = J->dout + (t * H + h) * Dv;
        const double bt = J->beta[t * H + h];
        const double *Sp = St + i * KV, *S = St + (i + 1) * KV;
        double *dqt = J->dq + (t * H + h) * Dk, *dkt = J->dk + (t * H + h) * Dk;
        double *dvt = J->dv + (t * H + h) * Dv, *dlat = J->dla + (t * H + h) * Dk;

        /* 4'. o = S^T q */
        for (int64_t c = 0; c < Dk; ++c) {
            double acc = 0.0;
            for (int64_t j = 0; j < Dv; ++j) acc = acc + S[c * Dv + j] * dot[j];
            dqt[c] = acc;
            for (int64_t j = 0; j < Dv; ++j) G[c * Dv + j] = G[c * Dv + j] + qt[c] * dot[j];
        }
        /* recompute e = v - P^T k with P = Diag(alpha) S_{t-1} */
        for (int64_t j = 0; j < Dv; ++j) e[j] = 0.0;
        for (int64_t c = 0; c < Dk; ++c) {
            const double a = exp(lat[c]);
            for (int64_t j = 0; j < Dv; ++j) e[j] = e[j] + kt[c] * (a * Sp[c * Dv + j]);
        }
        for (int64_t j = 0; j < Dv; ++j) e[j] = vt[j] - e[j];
        /* 3'. S = P + beta k e^T */
        double db = 0.0;
        for (int64_t j = 0; j < Dv; ++j) de[j] = 0.0;
        for (int64_t c = 0; c < Dk; ++c) {
            double ge = 0.0;
            for (int64_t j = 0; j < Dv; ++j) {
                dP[c * Dv + j] = G[c * Dv + j];
                de[j] = de[j] + bt * kt[c] * G[c * Dv + j];
                ge = ge + G[c * Dv + j] * e[j];
            }
            dkt[c] = bt * ge;
            db = db + kt[c] * ge;
        }
        J->dbeta[t * H + h] = db;
        /* 2'. e = v - P^T k */
        for (int64_t j = 0; j < Dv; ++j) dvt[j] = de[j];
        for (int64_t c = 0; c < Dk; ++c) {
            const double a = exp(lat[c]);
            double pde = 0.0;
            for (int64_t j = 0; j < Dv; ++j) {
                dP[c * Dv + j] = dP[c * Dv + j] - kt[c] * de[j];
                pde = pde + (a * Sp[c * Dv + j]) * de[j];
            }
            dkt[c] = dkt[c] - pde;
        }
        /* 1'. P = Diag(alpha) S_{t-1} */
        for (int64_t c = 0; c < Dk; ++c) {
            const double a = exp(lat[c]);
            double acc = 0.0;
            for (int64_t j = 0; j < Dv; ++j) acc = acc + dP[c * Dv + j] * Sp[c * Dv + j];
            dlat[c] = a * acc;
            for (int64_t j = 0; j < Dv; ++j) G[c * Dv + j] = a * dP[c * Dv + j];
        }
    }
    if (J->dS0) memcpy(J->dS0 + (n * H + h) * KV, G, sizeof(double) * KV);
    free(St); free(G); free(dP); free(e); free(de);
    return 0;
}

static void *bworker(void *arg)
{
    bjob_t *J = (bjob_t *)arg;
    const int64_t total = J->n_seqs * J->H;
    for (;;) {
        pthread_mutex_lock(&J->lock);
        const int64_t i = J->next++;
        pthread_mutex_unlock(&J->lock);
        if (i >= total) break;
        if (backward_chain(J, i / J->H, i % J->H) != 0) {
            pthread_mutex_lock(&J->lock);
            J->failed = 1;
            pthread_mutex_unlock(&J->lock);
        }
    }
    return NULL;
}

/*
 * kda_oracle_backward: the gradients described above for every chain.
 * Returns 0 on success, -1 on bad arguments, -2 on allocation/thread failure.
 */
int kda_oracle_backward(int64_t n_seqs, const int64_t *cu_seqlens, int64_t H, int64_t Dk,
                        int64_t Dv, const double *q, const double *k, const double *v,
                        const double *log_alpha, const double *beta, const double *S0,
                        const double *d_out, const double *dS_final, double *dq, double *dk,
                        double *dv, double *dlog_alpha, double *dbeta, double *dS0,
                        int n_threads)
{
    if (n_seqs < 0 || H <= 0 || Dk <= 0 || Dv <= 0 || !cu_seqlens) return -1;
    if (cu_seqlens[0] != 0) return -1;
    for (int64_t n = 0; n < n_seqs; ++n)
        if (cu_seqlens[n + 1] < cu_seqlens[n]) return -1;
    if (cu_seqlens[n_seqs] > 0 && (!q || !k || !v || !log_alpha || !beta || !d_out || !dq ||
                                   !dk || !dv || !dlog_alpha || !dbeta))
        return -1;

    bjob_t J;
    J.n_seqs = n_seqs; J.H = H; J.Dk = Dk; J.Dv = Dv; J.cu = cu_seqlens;
    J.q = q; J.k = k; J.v = v; J.la = log_alpha; J.beta = beta; J.S0 = S0;
    J.dout = d_out; J.dSf = dS_final;
    J.dq = dq; J.dk = dk; J.dv = dv; J.dla = dlog_alpha; J.dbeta = dbeta; J.dS0 = dS0;
    J.next = 0; J.failed = 0;
    pthread_mutex_init(&J.lock, NULL);

    const int64_t total = n_seqs * H;
    if (n_threads < 1) n_threads = 1;
    if (n_threads > total) n_threads = (int)(total > 0 ? total : 1);
    pthread_t *th = (pthread_t *)malloc(sizeof(pthread_t) * (size_t)n_threads);
    if (!th) { pthread_mutex_destroy(&J.lock); return -2; }
    int started = 0, rc = 0;
    for (int i = 0; i < n_threads; ++i) {
        if (pthread_create(&th[i], NULL, bworker, &J) != 0) { rc = -2; break; }
        ++started;
    }
    for (int i = 0; i < started; ++i) pthread_join(th[i], NULL);
    free(th);
    pthread_mutex_destroy(&J.lock);
    if (J.failed) rc = -2;
    return rc;
}
