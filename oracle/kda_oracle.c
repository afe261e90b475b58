/*
 * kda_oracle.c -- fp64 CPU oracle for Kimi Delta Attention (KDA).
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path may link, load or
 * call this file; only the tests, the smoke check and the CPU-baseline leg of
 * the benchmark do.  It shares no code, header, table or helper with the CUDA
 * library.
 *
 * What it computes.  The page "Kimi K3: Open Frontier Intelligence and
 * Implementation Framework" (section "Technical Architecture and Scaling
 * Efficiency", sub-section "Hybrid Attention Mechanism", KDA bullet)
 * describes KDA as the delta-rule recurrence extended with a channel-wise
 * forget gate whose decay is bounded below.  Written out per head, with a
 * d_k x d_v state S, a per-channel decay alpha_t = exp(log_alpha_t) and a
 * scalar write strength beta_t:
 *
 *     S_t = (I - beta_t k_t k_t^T) Diag(alpha_t) S_{t-1} + beta_t k_t v_t^T
 *     o_t = S_t^T q_t
 *
 * The oracle applies that definition one token at a time, in the order the
 * definition reads:
 *     1. S <- Diag(alpha_t) S                (channel-wise forget gate)
 *     2. e <- v_t - S^T k_t                  (delta-rule prediction error)
 *     3. S <- S + beta_t k_t e^T             (rank-one write)
 *     4. o_t <- S^T q_t                      (read-out after the update)
 * Steps 2-3 equal (I - beta k k^T) S + beta k v^T with S already decayed.
 *
 * Readings where the pages are silent:
 *   - o_t uses the state after the token's own update (the formula above);
 *   - q carries no extra attention scale;
 *   - beta is one scalar per (token, head); log_alpha is given directly and
 *     alpha = exp(log_alpha) per channel;
 *   - sequences are packed along the token axis and delimited by cu_seqlens;
 *     each (sequence, head) pair is an independent chain that starts from
 *     S0[n,h] (zero when S0 is NULL) and ends in S_final[n,h];
 *     a zero-length sequence yields S_final = S0.
 *
 * Arithmetic: IEEE double, no fused multiply-add contraction, no fast-math
 * (the build passes -ffp-contract=off -fno-fast-math), plain loops.
 * Parallelism: independent chains are spread over POSIX threads; each chain
 * is computed by exactly one thread, so results do not depend on the thread
 * count.
 *
 * Layouts (row-major, packed token axis of length T_tot):
 *   q, k, log_alpha : [T_tot, H, Dk]     v, out : [T_tot, H, Dv]
 *   beta            : [T_tot, H]         S0, S_final : [N, H, Dk, Dv]
 *
 * State snapshots.  The same page, section "Inference Serving", bullet
 * "KDA-Aware Prefix Caching", keeps KDA recurrent states in a paged pool so
 * that a prefix can be resumed at 512-token boundaries.  Reading taken: a
 * snapshot is the state of a (sequence, head) chain right after token
 * number m * every of that sequence (m = 1, 2, ...; counted from the
 * sequence start), for every such m inside the sequence.  The oracle writes
 * snapshot m-1 of sequence n to snap[(snap_off[n] + m - 1), h] (layout
 * [*, H, Dk, Dv]); resuming from a snapshot is a forward pass whose S0 is
 * that snapshot.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

typedef struct {
    int64_t n_seqs, H, Dk, Dv;
    const int64_t *cu;
    const double *q, *k, *v, *la, *beta, *S0;
    double *out, *Sf;
    int64_t snap_every;      /* tokens between snapshots; 0: none */
    const int64_t *snap_off; /* [N] first snapshot index of each sequence */
    double *snap;            /* [*, H, Dk, Dv] */
    int64_t next;            /* next chain index, taken under the lock */
    pthread_mutex_t lock;
} job_t;

/* One chain: sequence n, head h.  S is scratch of Dk*Dv doubles, e of Dv. */
static void run_chain(const job_t *J, int64_t n, int64_t h, double *S, double *e)
{
    const int64_t H = J->H, Dk = J->Dk, Dv = J->Dv;
    const int64_t t0 = J->cu[n], t1 = J->cu[n + 1];

    if (J->S0)
        memcpy(S, J->S0 + (n * H + h) * Dk * Dv, sizeof(double) * Dk * Dv);
    else
        memset(S, 0, sizeof(double) * Dk * Dv);

    for (int64_t t = t0; t < t1; ++t) {
        const double *qt = J->q + (t * H + h) * Dk;
        const double *kt = J->k + (t * H + h) * Dk;
        const double *vt = J->v + (t * H + h) * Dv;
        const double *lat = J->la + (t * H + h) * Dk;
        const double bt = J->beta[t * H + h];
        double *ot = J->out + (t * H + h) * Dv;

        /* 1. channel-wise decay: row c of S scaled by alpha_c */
        for (int64_t c = 0; c < Dk; ++c) {
            const double a = exp(lat[c]);
            double *row = S + c * Dv;
            for (int64_t j = 0; j < Dv; ++j) row[j] = a * row[j];
        }
        /* 2. e = v - S^T k */
        for (int64_t j = 0; j < Dv; ++j) e[j] = 0.0;
        for (int64_t c = 0; c < Dk; ++c) {
            const double kc = kt[c];
            const double *row = S + c * Dv;
            for (int64_t j = 0; j < Dv; ++j) e[j] = e[j] + kc * row[j];
        }
        for (int64_t j = 0; j < Dv; ++j) e[j] = vt[j] - e[j];
        /* 3. S = S + beta k e^T */
        for (int64_t c = 0; c < Dk; ++c) {
            const double w = bt * kt[c];
            double *row = S + c * Dv;
            for (int64_t j = 0; j < Dv; ++j) row[j] = row[j] + w * e[j];
        }
        /* 4. o = S^T q */
        for (int64_t j = 0; j < Dv; ++j) ot[j] = 0.0;
        for (int64_t c = 0; c < Dk; ++c) {
            const double qc = qt[c];
            const double *row = S + c * Dv;
            for (int64_t j = 0; j < Dv; ++j) ot[j] = ot[j] + qc * row[j];
        }
        /* snapshot after token number (t - t0 + 1) of the sequence */
        const int64_t done = t - t0 + 1;
        if (J->snap && done % J->snap_every == 0) {
            const int64_t m = J->snap_off[n] + done / J->snap_every - 1;
            memcpy(J->snap + (m * H + h) * Dk * Dv, S, sizeof(double) * Dk * Dv);
        }
    }
    if (J->Sf)
        memcpy(J->Sf + (n * H + h) * Dk * Dv, S, sizeof(double) * Dk * Dv);
}

static void *worker(void *arg)
{
    job_t *J = (job_t *)arg;
    double *S = (double *)malloc(sizeof(double) * (size_t)(J->Dk * J->Dv));
    double *e = (double *)malloc(sizeof(double) * (size_t)J->Dv);
    if (!S || !e) { free(S); free(e); return (void *)1; }
    const int64_t total = J->n_seqs * J->H;
    for (;;) {
        pthread_mutex_lock(&J->lock);
        const int64_t i = J->next++;
        pthread_mutex_unlock(&J->lock);
        if (i >= total) break;
        run_chain(J, i / J->H, i % J->H, S, e);
    }
    free(S);
    free(e);
    return NULL;
}

/*
 * kda_oracle_forward: the recurrence over every (sequence, head) chain.
 * S0 and S_final may be NULL; S_final may equal S0 (each chain copies its
 * S0 slice before it writes the same slice of S_final).
 * Returns 0 on success, -1 on bad arguments, -2 on allocation/thread failure.
 */
int kda_oracle_forward_snapshots(int64_t n_seqs, const int64_t *cu_seqlens, int64_t H,
                                 int64_t Dk, int64_t Dv, const double *q, const double *k,
                                 const double *v, const double *log_alpha,
                                 const double *beta, const double *S0, double *out,
                                 double *S_final, int64_t snap_every,
                                 const int64_t *snap_off, double *snap, int n_threads);

int kda_oracle_forward(int64_t n_seqs, const int64_t *cu_seqlens, int64_t H,
                       int64_t Dk, int64_t Dv, const double *q, const double *k,
                       const double *v, const double *log_alpha,
                       const double *beta, const double *S0, double *out,
                       double *S_final, int n_threads)
{
    return kda_oracle_forward_snapshots(n_seqs, cu_seqlens, H, Dk, Dv, q, k, v, log_alpha,
                                        beta, S0, out, S_final, 0, NULL, NULL, n_threads);
}

/*
 * kda_oracle_forward_snapshots: kda_oracle_forward that also records the
 * state snapshots described at the top of this file.  snap_every = 0 (or
 * snap = NULL) records none.  snap_off[n] is the index of sequence n's first
 * snapshot; the caller sizes snap for sum_n floor(len_n / snap_every) of
 * them.
 */
int kda_oracle_forward_snapshots(int64_t n_seqs, const int64_t *cu_seqlens, int64_t H,
                                 int64_t Dk, int64_t Dv, const double *q, const double *k,
                                 const double *v, const double *log_alpha,
                                 const double *beta, const double *S0, double *out,
                                 double *S_final, int64_t snap_every,
                                 const int64_t *snap_off, double *snap, int n_threads)
{
    if (n_seqs < 0 || H <= 0 || Dk <= 0 || Dv <= 0 || !cu_seqlens) return -1;
    if (snap && (snap_every <= 0 || !snap_off)) return -1;
    for (int64_t n = 0; n < n_seqs; ++n)
        if (cu_seqlens[n + 1] < cu_seqlens[n]) return -1;
    if (cu_seqlens[0] != 0) return -1;
    if (cu_seqlens[n_seqs] > 0 && (!q || !k || !v || !log_alpha || !beta || !out))
        return -1;

    job_t J;
    J.n_seqs = n_seqs; J.H = H; J.Dk = Dk; J.Dv = Dv; J.cu = cu_seqlens;
    J.q = q; J.k = k; J.v = v; J.la = log_alpha; J.beta = beta; J.S0 = S0;
    J.out = out; J.Sf = S_final; J.next = 0;
    J.snap_every = snap ? snap_every : 0; J.snap_off = snap_off; J.snap = snap;
    pthread_mutex_init(&J.lock, NULL);

    const int64_t total = n_seqs * H;
    if (n_threads < 1) n_threads = 1;
    if (n_threads > total) n_threads = (int)(total > 0 ? total : 1);
    pthread_t *th = (pthread_t *)malloc(sizeof(pthread_t) * (size_t)n_threads);
    if (!th) { pthread_mutex_destroy(&J.lock); return -2; }
    int started = 0, rc = 0;
    for (int i = 0; i < n_threads; ++i) {
        if (pthread_create(&th[i], NULL, worker, &J) != 0) { rc = -2; break; }
        ++started;
    }
    for (int i = 0; i < started; ++i) {
        void *ret = NULL;
        pthread_join(th[i], &ret);
        if (ret) rc = -2;
    }
    free(th);
    pthread_mutex_destroy(&J.lock);
    return rc;
}

/*
 * kda_oracle_decode_step: one token of the recurrence for N independent
 * sequences, updating S [N,H,Dk,Dv] in place.  It is the same chain step as
 * above with every sequence one token long:
 *   q, k, log_alpha : [N, H, Dk]   v, out : [N, H, Dv]   beta : [N, H].
 */
int kda_oracle_decode_step(int64_t n_seqs, int64_t H, int64_t Dk, int64_t Dv,
                           const double *q, const double *k, const double *v,
                           const double *log_alpha, const double *beta,
                           double *S, double *out, int n_threads)
{
    if (n_seqs < 0 || !S) return -1;
    int64_t *cu = (int64_t *)malloc(sizeof(int64_t) * (size_t)(n_seqs + 1));
    if (!cu) return -2;
    for (int64_t n = 0; n <= n_seqs; ++n) cu[n] = n;
    const int rc = kda_oracle_forward(n_seqs, cu, H, Dk, Dv, q, k, v, log_alpha,
                                      beta, S, out, S, n_threads);
    free(cu);
    return rc;
}

