/*
 * gdn_oracle.c -- fp64 CPU oracle of the gated delta rule.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may link, load or call
 * this file; only the tests, the smoke check and the CPU-baseline leg of the
 * benchmark do.  It shares no code, header, table or helper with the CUDA
 * library: it is the plain definition of the recurrence, written out token by
 * token, in double precision.
 *
 * What it computes (per sequence n and head h, independently):
 *
 *   S <- initial state (d_v x d_k), or zeros
 *   for every token t of the sequence, in order:
 *     1. forget:  S~ = alpha_t * S            (scalar gate, one alpha per head)
 *                 S~ = S * Diag(alpha_t)      (per-channel gate, alpha over d_k)
 *        with alpha_t = exp(g_t), g_t being the gate passed as a logarithm.
 *     2. correct: S  = S~ + beta_t * (v_t - S~ k_t) k_t^T
 *        (the "additive" test mode writes S = S~ + beta_t * v_t k_t^T instead)
 *     3. read:    o_t = S (scale * q_t)       -- the state *after* the write.
 *     4. every `snapshot_stride` tokens of the sequence, copy S out.
 *   final state <- S
 *
 * Sources:
 *  - "Hybrid models: what Gated DeltaNet replaces in the KV cache", sections
 *    "The delta rule: write the correction, not the sum" and "Gated DeltaNet:
 *    add decay" (the update S_t = alpha_t S_{t-1}(I - beta_t k_t k_t^T)
 *    + beta_t v_t k_t^T and the d_v x d_k state), and "What a recurrent state
 *    changes for serving" item 1 (a snapshot is the state at position N).
 *  - "From Traditional Attention to hybrid ones", section 5 "From DeltaNet to
 *    Gated DeltaNet": decay first (S~ = alpha_t S_{t-1}), then the delta update
 *    on the decayed state, then the read o_t = S_t q_t; section 7: the KDA form
 *    S_t = S_{t-1} Diag(alpha_t)(I - beta_t k_t k_t^T) + beta_t v_t k_t^T in the
 *    d_v x d_k convention, i.e. alpha scales the key channels (columns).
 *  - "Attention, Part 4: Linear Attention, Gated DeltaNet and Hybrid Models",
 *    section 6 (the token loop: forget, correct, read) and "Where alpha and
 *    beta come from" (the gate is stored as g = log alpha).
 *  - "Hybrid Linear Attention Architecture Design Explained", section 3.1 item
 *    6 (KDA: first forget, then correct).
 *
 * Work is split over (sequence, head) units with POSIX threads; each unit is
 * computed by exactly one thread, so the result does not depend on the thread
 * count.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

typedef struct {
    int64_t n_seqs, H, dk, dv;
    const int64_t *seq_start; /* first packed token row of each sequence   */
    const int64_t *seq_len;   /* number of tokens of each sequence         */
    const double *q, *k, *v;  /* (rows, H, dk) / (rows, H, dk) / (rows, H, dv) */
    const double *g;          /* (rows, H) or, per channel, (rows, H, dk)  */
    const double *beta;       /* (rows, H)                                 */
    const double *h0;         /* (n_seqs, H, dv, dk) or NULL for zeros     */
    int per_channel, additive;
    double scale;
    int64_t snapshot_stride;  /* 0: no snapshots                           */
    int64_t n_snap_max;       /* second dimension of `snapshots`           */
    double *out;              /* (rows, H, dv)                             */
    double *final_state;      /* (n_seqs, H, dv, dk) or NULL               */
    double *snapshots;        /* (n_seqs, n_snap_max, H, dv, dk) or NULL   */
    /* work distribution */
    int64_t next_unit;
    pthread_mutex_t lock;
} oracle_job;

static void run_unit(const oracle_job *J, int64_t unit, double *S, double *y, double *al)
{
    const int64_t H = J->H, dk = J->dk, dv = J->dv;
    const int64_t n = unit / H, h = unit % H;
    const int64_t start = J->seq_start[n], len = J->seq_len[n];

    if (J->h0)
        memcpy(S, J->h0 + (n * H + h) * dv * dk, sizeof(double) * dv * dk);
    else
        memset(S, 0, sizeof(double) * dv * dk);

    for (int64_t t = 0; t < len; ++t) {
        const int64_t row = start + t;
        const double *qt = J->q + (row * H + h) * dk;
        const double *kt = J->k + (row * H + h) * dk;
        const double *vt = J->v + (row * H + h) * dv;
        const double bt = J->beta[row * H + h];

        /* 1. forget */
        if (J->per_channel) {
            const double *gt = J->g + (row * H + h) * dk;
            for (int64_t c = 0; c < dk; ++c)
                al[c] = exp(gt[c]);
            for (int64_t i = 0; i < dv; ++i)
                for (int64_t c = 0; c < dk; ++c)
                    S[i * dk + c] *= al[c];
        } else {
            const double a = exp(J->g[row * H + h]);
            for (int64_t i = 0; i < dv * dk; ++i)
                S[i] *= a;
        }

        /* 2. correct: what the decayed state predicts for k_t ... */
        for (int64_t i = 0; i < dv; ++i) {
            double acc = 0.0;
            for (int64_t c = 0; c < dk; ++c)
                acc += S[i * dk + c] * kt[c];
            y[i] = acc;
        }
        /* ... and the write of the error (or of v_t itself in additive mode) */
        for (int64_t i = 0; i < dv; ++i) {
            const double e = J->additive ? vt[i] : (vt[i] - y[i]);
            for (int64_t c = 0; c < dk; ++c)
                S[i * dk + c] += bt * e * kt[c];
        }

        /* 3. read the updated state */
        double *ot = J->out + (row * H + h) * dv;
        for (int64_t i = 0; i < dv; ++i) {
            double acc = 0.0;
            for (int64_t c = 0; c < dk; ++c)
                acc += S[i * dk + c] * (J->scale * qt[c]);
            ot[i] = acc;
        }

        /* 4. snapshot after every `snapshot_stride` tokens of this sequence */
        if (J->snapshots && J->snapshot_stride > 0 && (t + 1) % J->snapshot_stride == 0) {
            const int64_t s = (t + 1) / J->snapshot_stride - 1;
            if (s < J->n_snap_max)
                memcpy(J->snapshots + ((n * J->n_snap_max + s) * H + h) * dv * dk, S,
                       sizeof(double) * dv * dk);
        }
    }
    if (J->final_state)
        memcpy(J->final_state + (n * H + h) * dv * dk, S, sizeof(double) * dv * dk);
}

static void *worker(void *arg)
{
    oracle_job *J = (oracle_job *)arg;
    double *S = (double *)malloc(sizeof(double) * J->dv * J->dk);
    double *y = (double *)malloc(sizeof(double) * J->dv);
    double *al = (double *)malloc(sizeof(double) * J->dk);
    const int64_t units = J->n_seqs * J->H;
    if (S && y && al) {
        for (;;) {
            pthread_mutex_lock(&J->lock);
            const int64_t u = J->next_unit++;
            pthread_mutex_unlock(&J->lock);
            if (u >= units)
                break;
            run_unit(J, u, S, y, al);
        }
    }
    free(S);
    free(y);
    free(al);
    return NULL;
}

/* Returns 0 on success, -1 on bad arguments. */
int oracle_gdn_forward(int64_t n_seqs, const int64_t *seq_start, const int64_t *seq_len,
                       int64_t H, int64_t dk, int64_t dv,
                       const double *q, const double *k, const double *v,
                       const double *g, const double *beta, const double *h0,
                       int per_channel, int additive, double scale,
                       int64_t snapshot_stride, int64_t n_snap_max,
                       double *out, double *final_state, double *snapshots,
                       int n_threads)
{
    if (n_seqs < 0 || H <= 0 || dk <= 0 || dv <= 0 || !seq_start || !seq_len ||
        !q || !k || !v || !g || !beta || !out || snapshot_stride < 0)
        return -1;
    oracle_job J;
    memset(&J, 0, sizeof J);
    J.n_seqs = n_seqs; J.H = H; J.dk = dk; J.dv = dv;
    J.seq_start = seq_start; J.seq_len = seq_len;
    J.q = q; J.k = k; J.v = v; J.g = g; J.beta = beta; J.h0 = h0;
    J.per_channel = per_channel; J.additive = additive; J.scale = scale;
    J.snapshot_stride = snapshot_stride; J.n_snap_max = n_snap_max;
    J.out = out; J.final_state = final_state; J.snapshots = snapshots;
    J.next_unit = 0;
    pthread_mutex_init(&J.lock, NULL);

    const int64_t units = n_seqs * H;
    if (n_threads < 1)
        n_threads = 1;
    if (n_threads > units)
        n_threads = (int)(units > 0 ? units : 1);
    /* Every path below processes every unit: threads that fail to start
       leave their share to the others, or to the calling thread. */
    pthread_t *tid = (pthread_t *)malloc(sizeof(pthread_t) * (size_t)n_threads);
    int started = 0;
    if (tid) {
        for (int i = 0; i < n_threads; ++i) {
            if (pthread_create(&tid[i], NULL, worker, &J) != 0)
                break;
            ++started;
        }
        for (int i = 0; i < started; ++i)
            pthread_join(tid[i], NULL);
    }
    if (started == 0)
        worker(&J);
    free(tid);
    pthread_mutex_destroy(&J.lock);
    return 0;
}
