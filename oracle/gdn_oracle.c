/*
 * gdn_oracle.c -- fp64 CPU oracle for the gated delta rule (Gated DeltaNet).
 *
 * TEST INFRASTRUCTURE ONLY. This file is the independent checker that the
 * CUDA path is compared against. It shares no code, header or table with the
 * CUDA library; only tests, the smoke check and the bench's CPU-baseline and
 * reference legs (both time this oracle on the host cores) may load it.
 *
 * What it computes (token by token, no chunking, no reordering):
 *
 *   For each sequence n and each value head h (qk head hq = h / (Hv/Hq)),
 *   with state S in R^{V x K} starting from S_0 = transpose(h0[n,h]) (or 0):
 *
 *     S_bar_t = exp(g_t) * S_{t-1}                       (gate / decay)
 *     p_t     = S_bar_t k_t                              (prediction of v_t)
 *     d_t     = beta_t * (v_t - p_t)                     (delta-rule error)
 *     S_t     = S_bar_t + d_t k_t^T
 *     o_t     = scale * S_t q_t
 *
 *   which is S_t = exp(g_t) S_{t-1} (I - beta_t k_t k_t^T) + beta_t v_t k_t^T,
 *   o_t = scale S_t q_t: the gated delta rule stated for the GDN layers that
 *   the FlashQLA pages ("什么是 FlashQLA", page 1) serve, with the
 *   chunk_gated_delta_rule argument list of page 1's "高级 API 示例"
 *   (q,k: [B,T,Hq,K]; v: [B,T,Hv,V]; g, beta: [B,T,Hv]; scale;
 *   initial_state; output_final_state; cu_seqlens).
 *
 *   The final state is returned as h = S^T, row-major [K][V] per (n, h).
 *
 * Reverse mode (gdn_oracle_bwd) is the hand-derived adjoint of exactly the
 * five steps above, taken in reverse order per token, giving the gradients
 * (dq, dk, dv, dbeta, dg, dh0) that the low-level backward of page 1's
 * "底层 API" returns. dg is with respect to the raw per-token log-decay g_t.
 * dq and dk of a qk head sum the contributions of every value head of its
 * group. The state is checkpointed every CKPT tokens and the states inside a
 * block are recomputed during the reverse sweep.
 *
 * Layouts (all fp64, contiguous):
 *   q, k   [B, T, Hq, K]       v, o      [B, T, Hv, V]
 *   g, beta [B, T, Hv]         h0, final [N, Hv, K, V]   (N = B, or num_seqs)
 *   cu_seqlens int32 [num_seqs + 1] when num_seqs > 0 (then B must be 1).
 *
 * Work is split over (sequence, head) tasks with POSIX threads; every task
 * writes disjoint outputs, so results do not depend on the thread count.
 */
#include <math.h>
#include <pthread.h>
#include <stdatomic.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define CKPT 64

typedef struct {
    int B, T, Hq, Hv, K, V, num_seqs;
    const int32_t *cu;
    const double *q, *k, *v, *g, *beta, *h0;
    double scale;
    /* forward outputs */
    double *o, *final_state;
    /* backward inputs / outputs */
    const double *d_o, *dht;
    double *dq, *dk, *dv, *dg, *dbeta, *dh0;
    atomic_int next;
    int ntasks;
    int failed;
} job_t;

static int num_sequences(const job_t *J) { return J->num_seqs > 0 ? J->num_seqs : J->B; }

/* Token row (index into the flattened [B*T] token axis) of position t of sequence n. */
static long seq_begin(const job_t *J, int n) {
    return J->num_seqs > 0 ? (long)J->cu[n] : (long)n * J->T;
}
static long seq_len(const job_t *J, int n) {
    return J->num_seqs > 0 ? (long)(J->cu[n + 1] - J->cu[n]) : (long)J->T;
}

/* ---------------------------------------------------------------- forward */

static void fwd_task(job_t *J, int n, int h, double *S, double *p) {
    const int K = J->K, V = J->V, Hq = J->Hq, Hv = J->Hv;
    const int hq = h / (Hv / Hq);
    const long t0 = seq_begin(J, n), L = seq_len(J, n);
    /* S[i*K + j] = S_ij, i over V, j over K */
    if (J->h0) {
        const double *H = J->h0 + ((long)n * Hv + h) * K * V;
        for (int i = 0; i < V; ++i)
            for (int j = 0; j < K; ++j) S[i * K + j] = H[(long)j * V + i];
    } else {
        memset(S, 0, sizeof(double) * K * V);
    }
    for (long t = 0; t < L; ++t) {
        const long row = t0 + t;
        const double *kt = J->k + (row * Hq + hq) * K;
        const double *qt = J->q + (row * Hq + hq) * K;
        const double *vt = J->v + (row * Hv + h) * V;
        const double a = exp(J->g[row * Hv + h]);
        const double b = J->beta[row * Hv + h];
        for (int e = 0; e < V * K; ++e) S[e] *= a;
        for (int i = 0; i < V; ++i) {
            double s = 0.0;
            for (int j = 0; j < K; ++j) s += S[i * K + j] * kt[j];
            p[i] = s;
        }
        for (int i = 0; i < V; ++i) {
            const double d = b * (vt[i] - p[i]);
            for (int j = 0; j < K; ++j) S[i * K + j] += d * kt[j];
        }
        if (J->o) {
            double *ot = J->o + (row * Hv + h) * V;
            for (int i = 0; i < V; ++i) {
                double s = 0.0;
                for (int j = 0; j < K; ++j) s += S[i * K + j] * qt[j];
                ot[i] = J->scale * s;
            }
        }
    }
    if (J->final_state) {
        double *F = J->final_state + ((long)n * Hv + h) * K * V;
        for (int i = 0; i < V; ++i)
            for (int j = 0; j < K; ++j) F[(long)j * V + i] = S[i * K + j];
    }
}

static void *fwd_worker(void *arg) {
    job_t *J = (job_t *)arg;
    double *S = (double *)malloc(sizeof(double) * J->K * J->V);
    double *p = (double *)malloc(sizeof(double) * J->V);
    if (!S || !p) { J->failed = 1; free(S); free(p); return NULL; }
    for (;;) {
        const int task = atomic_fetch_add(&J->next, 1);
        if (task >= J->ntasks) break;
        fwd_task(J, task / J->Hv, task % J->Hv, S, p);
    }
    free(S); free(p);
    return NULL;
}

/* --------------------------------------------------------------- backward */

/* Adjoint of one (sequence, qk-head group) task: all value heads of the group,
 * in increasing head order, so the dq/dk sums are taken in a fixed order. */
typedef struct {
    double *S;      /* running state                         V*K   */
    double *ck;     /* checkpoints: state before each block  nblk*V*K */
    double *blk;    /* states S_{t-1} inside one block       CKPT*V*K */
    double *dS, *Sb, *p, *dd, *dp;
} bwd_scratch;

static void bwd_head(job_t *J, int n, int h, bwd_scratch *W) {
    const int K = J->K, V = J->V, Hq = J->Hq, Hv = J->Hv;
    const int hq = h / (Hv / Hq);
    const long t0 = seq_begin(J, n), L = seq_len(J, n);
    const long VK = (long)V * K;
    const long nblk = (L + CKPT - 1) / CKPT;
    double *S = W->S;

    /* forward sweep: store the state at the start of every block */
    if (J->h0) {
        const double *H = J->h0 + ((long)n * Hv + h) * VK;
        for (int i = 0; i < V; ++i)
            for (int j = 0; j < K; ++j) S[i * K + j] = H[(long)j * V + i];
    } else {
        memset(S, 0, sizeof(double) * VK);
    }
    for (long t = 0; t < L; ++t) {
        if (t % CKPT == 0) memcpy(W->ck + (t / CKPT) * VK, S, sizeof(double) * VK);
        const long row = t0 + t;
        const double *kt = J->k + (row * Hq + hq) * K;
        const double *vt = J->v + (row * Hv + h) * V;
        const double a = exp(J->g[row * Hv + h]);
        const double b = J->beta[row * Hv + h];
        for (long e = 0; e < VK; ++e) S[e] *= a;
        for (int i = 0; i < V; ++i) {
            double s = 0.0;
            for (int j = 0; j < K; ++j) s += S[i * K + j] * kt[j];
            const double d = b * (vt[i] - s);
            for (int j = 0; j < K; ++j) S[i * K + j] += d * kt[j];
        }
    }

    /* dS = dL/dS_T, seeded from dht (given as h-layout [K][V]) */
    double *dS = W->dS;
    if (J->dht) {
        const double *D = J->dht + ((long)n * Hv + h) * VK;
        for (int i = 0; i < V; ++i)
            for (int j = 0; j < K; ++j) dS[i * K + j] = D[(long)j * V + i];
    } else {
        memset(dS, 0, sizeof(double) * VK);
    }

    for (long bi = nblk - 1; bi >= 0; --bi) {
        const long tb = bi * CKPT;
        const long te = (tb + CKPT < L) ? tb + CKPT : L;
        /* recompute S_{t-1} for t in [tb, te) */
        memcpy(S, W->ck + bi * VK, sizeof(double) * VK);
        for (long t = tb; t < te; ++t) {
            memcpy(W->blk + (t - tb) * VK, S, sizeof(double) * VK);
            const long row = t0 + t;
            const double *kt = J->k + (row * Hq + hq) * K;
            const double *vt = J->v + (row * Hv + h) * V;
            const double a = exp(J->g[row * Hv + h]);
            const double b = J->beta[row * Hv + h];
            for (long e = 0; e < VK; ++e) S[e] *= a;
            for (int i = 0; i < V; ++i) {
                double s = 0.0;
                for (int j = 0; j < K; ++j) s += S[i * K + j] * kt[j];
                const double d = b * (vt[i] - s);
                for (int j = 0; j < K; ++j) S[i * K + j] += d * kt[j];
            }
        }
        for (long t = te - 1; t >= tb; --t) {
            const long row = t0 + t;
            const double *kt = J->k + (row * Hq + hq) * K;
            const double *qt = J->q + (row * Hq + hq) * K;
            const double *vt = J->v + (row * Hv + h) * V;
            const double *dot = J->d_o ? J->d_o + (row * Hv + h) * V : NULL;
            const double a = exp(J->g[row * Hv + h]);
            const double b = J->beta[row * Hv + h];
            const double *Sprev = W->blk + (t - tb) * VK;
            double *Sb = W->Sb, *p = W->p, *dd = W->dd, *dp = W->dp;
            /* re-run this token's forward steps: S_bar, p, d, S_t */
            for (long e = 0; e < VK; ++e) Sb[e] = a * Sprev[e];
            for (int i = 0; i < V; ++i) {
                double s = 0.0;
                for (int j = 0; j < K; ++j) s += Sb[i * K + j] * kt[j];
                p[i] = s;
            }
            /* S_t = S_bar + d k^T, held in S (only needed for dq) */
            for (int i = 0; i < V; ++i) {
                const double d = b * (vt[i] - p[i]);
                for (int j = 0; j < K; ++j) S[i * K + j] = Sb[i * K + j] + d * kt[j];
            }
            double *dqt = J->dq + (row * Hq + hq) * K;
            double *dkt = J->dk + (row * Hq + hq) * K;
            /* o_t = scale S_t q_t */
            if (dot) {
                for (int j = 0; j < K; ++j) {
                    double s = 0.0;
                    for (int i = 0; i < V; ++i) s += S[i * K + j] * dot[i];
                    dqt[j] += J->scale * s;
                }
                for (int i = 0; i < V; ++i)
                    for (int j = 0; j < K; ++j) dS[i * K + j] += J->scale * dot[i] * qt[j];
            }
            /* S_t = S_bar + d k^T:  dd = dS k,  dk += dS^T d,  dS_bar = dS */
            for (int i = 0; i < V; ++i) {
                double s = 0.0;
                for (int j = 0; j < K; ++j) s += dS[i * K + j] * kt[j];
                dd[i] = s;
            }
            for (int j = 0; j < K; ++j) {
                double s = 0.0;
                for (int i = 0; i < V; ++i) s += dS[i * K + j] * b * (vt[i] - p[i]);
                dkt[j] += s;
            }
            /* d = beta (v - p): dbeta, dv, dp */
            double db = 0.0;
            for (int i = 0; i < V; ++i) {
                db += dd[i] * (vt[i] - p[i]);
                J->dv[(row * Hv + h) * V + i] = b * dd[i];
                dp[i] = -b * dd[i];
            }
            J->dbeta[row * Hv + h] = db;
            /* p = S_bar k: dS_bar += dp k^T, dk += S_bar^T dp */
            for (int j = 0; j < K; ++j) {
                double s = 0.0;
                for (int i = 0; i < V; ++i) s += Sb[i * K + j] * dp[i];
                dkt[j] += s;
            }
            for (int i = 0; i < V; ++i)
                for (int j = 0; j < K; ++j) dS[i * K + j] += dp[i] * kt[j];
            /* S_bar = exp(g) S_{t-1}: dg = <dS_bar, S_bar>, dS_{t-1} = exp(g) dS_bar */
            double dga = 0.0;
            for (long e = 0; e < VK; ++e) dga += dS[e] * Sb[e];
            J->dg[row * Hv + h] = dga;
            for (long e = 0; e < VK; ++e) dS[e] *= a;
        }
    }
    if (J->dh0) {
        double *D = J->dh0 + ((long)n * Hv + h) * VK;
        for (int i = 0; i < V; ++i)
            for (int j = 0; j < K; ++j) D[(long)j * V + i] = dS[i * K + j];
    }
}

static void *bwd_worker(void *arg) {
    job_t *J = (job_t *)arg;
    const long VK = (long)J->V * J->K;
    /* longest sequence decides the checkpoint buffer */
    long Lmax = 0;
    for (int n = 0; n < num_sequences(J); ++n)
        if (seq_len(J, n) > Lmax) Lmax = seq_len(J, n);
    const long nblk = (Lmax + CKPT - 1) / CKPT;
    bwd_scratch W;
    W.S = malloc(sizeof(double) * VK);
    W.ck = malloc(sizeof(double) * VK * (nblk > 0 ? nblk : 1));
    W.blk = malloc(sizeof(double) * VK * CKPT);
    W.dS = malloc(sizeof(double) * VK);
    W.Sb = malloc(sizeof(double) * VK);
    W.p = malloc(sizeof(double) * J->V);
    W.dd = malloc(sizeof(double) * J->V);
    W.dp = malloc(sizeof(double) * J->V);
    if (!W.S || !W.ck || !W.blk || !W.dS || !W.Sb || !W.p || !W.dd || !W.dp) {
        J->failed = 1;
    } else {
        const int G = J->Hv / J->Hq;
        for (;;) {
            const int task = atomic_fetch_add(&J->next, 1);
            if (task >= J->ntasks) break;
            const int n = task / J->Hq, hq = task % J->Hq;
            for (int h = hq * G; h < (hq + 1) * G; ++h) bwd_head(J, n, h, &W);
        }
    }
    free(W.S); free(W.ck); free(W.blk); free(W.dS); free(W.Sb);
    free(W.p); free(W.dd); free(W.dp);
    return NULL;
}

/* ------------------------------------------------------------ entry points */

static int check_args(const job_t *J) {
    if (J->B <= 0 || J->T < 0 || J->Hq <= 0 || J->Hv <= 0 || J->K <= 0 || J->V <= 0) return -1;
    if (J->Hv % J->Hq) return -1;
    if (J->num_seqs < 0) return -1;
    if (J->num_seqs > 0) {
        if (J->B != 1 || !J->cu) return -1;
        if (J->cu[0] != 0 || J->cu[J->num_seqs] != J->T) return -1;
        for (int n = 0; n < J->num_seqs; ++n)
            if (J->cu[n + 1] < J->cu[n]) return -1;
    }
    return 0;
}

static int run(job_t *J, void *(*worker)(void *), int nthreads) {
    if (nthreads < 1) nthreads = 1;
    if (nthreads > J->ntasks) nthreads = J->ntasks > 0 ? J->ntasks : 1;
    atomic_store(&J->next, 0);
    J->failed = 0;
    pthread_t *th = (pthread_t *)malloc(sizeof(pthread_t) * nthreads);
    if (!th) return -2;
    int started = 0;
    for (int i = 0; i < nthreads; ++i) {
        if (pthread_create(&th[i], NULL, worker, J) != 0) break;
        ++started;
    }
    if (started == 0) worker(J);
    for (int i = 0; i < started; ++i) pthread_join(th[i], NULL);
    free(th);
    return J->failed ? -2 : 0;
}

/* Forward. o and/or final_state may be NULL. Returns 0 on success,
 * -1 on invalid arguments, -2 on allocation failure. */
int gdn_oracle_fwd(int B, int T, int Hq, int Hv, int K, int V, int num_seqs,
                   const int32_t *cu_seqlens, const double *q, const double *k,
                   const double *v, const double *g, const double *beta, double scale,
                   const double *h0, double *o, double *final_state, int nthreads) {
    job_t J;
    memset(&J, 0, sizeof(J));
    J.B = B; J.T = T; J.Hq = Hq; J.Hv = Hv; J.K = K; J.V = V; J.num_seqs = num_seqs;
    J.cu = cu_seqlens; J.q = q; J.k = k; J.v = v; J.g = g; J.beta = beta; J.h0 = h0;
    J.scale = scale; J.o = o; J.final_state = final_state;
    if (check_args(&J)) return -1;
    J.ntasks = num_sequences(&J) * Hv;
    return run(&J, fwd_worker, nthreads);
}

/* Backward. d_o, dht, h0 may be NULL (treated as zero). dq and dk are
 * overwritten (zeroed here, then accumulated over each qk head's group).
 * dh0 may be NULL. Same return codes as the forward. */
int gdn_oracle_bwd(int B, int T, int Hq, int Hv, int K, int V, int num_seqs,
                   const int32_t *cu_seqlens, const double *q, const double *k,
                   const double *v, const double *g, const double *beta, double scale,
                   const double *h0, const double *d_o, const double *dht,
                   double *dq, double *dk, double *dv, double *dg, double *dbeta,
                   double *dh0, int nthreads) {
    job_t J;
    memset(&J, 0, sizeof(J));
    J.B = B; J.T = T; J.Hq = Hq; J.Hv = Hv; J.K = K; J.V = V; J.num_seqs = num_seqs;
    J.cu = cu_seqlens; J.q = q; J.k = k; J.v = v; J.g = g; J.beta = beta; J.h0 = h0;
    J.scale = scale; J.d_o = d_o; J.dht = dht;
    J.dq = dq; J.dk = dk; J.dv = dv; J.dg = dg; J.dbeta = dbeta; J.dh0 = dh0;
    if (check_args(&J)) return -1;
    if (!dq || !dk || !dv || !dg || !dbeta) return -1;
    const long ntok = (long)B * T;
    memset(dq, 0, sizeof(double) * ntok * Hq * K);
    memset(dk, 0, sizeof(double) * ntok * Hq * K);
    memset(dv, 0, sizeof(double) * ntok * Hv * V);
    memset(dg, 0, sizeof(double) * ntok * Hv);
    memset(dbeta, 0, sizeof(double) * ntok * Hv);
    J.ntasks = num_sequences(&J) * Hq;
    return run(&J, bwd_worker, nthreads);
}
