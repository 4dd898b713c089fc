/*
 * gdn_oracle.c -- plain, slow fp64 CPU oracle of the gated delta rule.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path links, loads or calls
 * this file; only the tests, the smoke check and the benchmark's CPU-baseline
 * leg do.  It shares no code, header, table or helper with the CUDA library.
 *
 * What it computes (state orientation S in R^{d_v x d_k}, o_t = S_t q_t):
 *
 *   Gated DeltaNet, scalar decay alpha_t in (0,1) and one scalar beta_t used for
 *   both the erase and the write (FG2-GDN paper, section 1 "Introduction" and
 *   section 5 "Delta Rule and Online Learning"; the Gated Delta Networks page,
 *   the claim check on its section 3.1):
 *       S_t = alpha_t S_{t-1} (I - beta_t k_t k_t^T) + beta_t v_t k_t^T
 *       o_t = S_t q_t
 *   Kimi Delta Attention (KDA), channel-wise decay Diag(alpha_t), alpha_t in
 *   R^{d_k}, in place of the scalar (FG2-GDN paper, section 1, "tied
 *   diagonal-plus-rank-1 transition"):
 *       S_t = S_{t-1} Diag(alpha_t) (I - beta_t k_t k_t^T) + beta_t v_t k_t^T
 *
 * The unified linear-attention view of FG2-GDN section 5 writes the same map
 * transposed (S in R^{d_k x d_v}, o_t = S_t^T q_t); here S is stored as
 * [d_v][d_k], row i = output channel i.
 *
 * Two routines:
 *   oracle_gdn_recurrent  -- the plain definition, token by token.
 *   oracle_gdn_chunkwise  -- the chunkwise WY / UT-transform form of FG2-GDN
 *                            section 3.6 (split into chunks of C tokens,
 *                            triangular solve for the UT factor, inter-chunk
 *                            state propagation, intra-chunk causal product),
 *                            written out step by step with explicit matrices.
 *                            Equal to the recurrence in exact arithmetic.
 * oracle_gdn_chunk_stage exposes one chunk's intermediates (g, A, T, W, U, V',
 * O, S_out) so the steps can be pinned one by one.
 *
 * oracle_fg2_recurrent is FG2-GDN's channel-wise writing rate (FG2-GDN paper,
 * section 3.2 "FG2-GDN Update Rule", section 3.4 "FG2-GDN+ Variant", section
 * 3.6 "Chunkwise Parallel Training"; the update's equations are lost from the
 * page, and this is the reading the text supports): the key is scaled by the
 * square root of the per-channel rate, k~ = sqrt(beta^k) . k, which keeps KDA's
 * tied (symmetric) transition; the FG2-GDN+ value gate scales the value the
 * same way, v~ = sqrt(beta^v) . v (FG2-GDN: no value gate, v~ = v); then
 *       S_t = S_{t-1} Diag(alpha_t) (I - k~_t k~_t^T) + v~_t k~_t^T
 *       o_t = S_t q_t
 * which is KDA's update with unit rate on (k~, v~): uniform beta^k = beta^v = b
 * gives KDA with beta = b.
 *
 * Everything is fp64; inputs are passed in already rounded to the precision
 * the GPU path reads (bf16 or fp32), upcast to double.  Independent (sequence,
 * head) chains run on POSIX threads; the arithmetic inside one chain is
 * sequential and follows the definition's order.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#include <unistd.h>

/* ------------------------------------------------------------------------ */
/* Problem description shared by the two drivers.                            */
/* ------------------------------------------------------------------------ */
typedef struct {
    int n_seqs;                 /* number of sequences                          */
    const int64_t *seq_start;   /* n_seqs+1 token offsets into the packed axis  */
    int H, dk, dv;
    int channel_decay;          /* 0: log_alpha [tok,H]; 1: log_alpha [tok,H,dk] */
    const double *q, *k;        /* [tok, H, dk]                                 */
    const double *v;            /* [tok, H, dv]                                 */
    const double *log_alpha;    /* [tok, H] or [tok, H, dk]                     */
    const double *beta;         /* [tok, H]                                     */
    const double *S0;           /* [n_seqs, H, dv, dk] or NULL (zeros)          */
    double *o;                  /* [tok, H, dv]                                 */
    double *S_final;            /* [n_seqs, H, dv, dk] or NULL                  */
    int chunk;                  /* chunk size (chunkwise driver only)           */
    const double *beta_k;       /* FG2: [tok, H, dk] key-side rate (else NULL)   */
    const double *beta_v;       /* FG2+: [tok, H, dv] value-side rate, or NULL   */
} problem;

/* log decay of channel c for token t of head h */
static double log_decay(const problem *p, int64_t t, int h, int c) {
    if (p->channel_decay) return p->log_alpha[(t * p->H + h) * p->dk + c];
    return p->log_alpha[t * p->H + h];
}

/* ------------------------------------------------------------------------ */
/* The recurrence, token by token, for one (sequence, head).                 */
/* ------------------------------------------------------------------------ */
static void recurrent_chain(const problem *p, int n, int h, double *S, double *r) {
    const int H = p->H, dk = p->dk, dv = p->dv;
    for (int64_t t = p->seq_start[n]; t < p->seq_start[n + 1]; ++t) {
        const double *q = p->q + (t * H + h) * dk;
        const double *k = p->k + (t * H + h) * dk;
        const double *v = p->v + (t * H + h) * dv;
        if (p->beta_k) {
            /* FG2: S <- S Diag(alpha) (I - k~ k~^T) + v~ k~^T with
             * k~ = sqrt(beta^k) . k and v~ = sqrt(beta^v) . v (or v)          */
            double *kt = r + dv, *vt = r + dv + dk;
            for (int c = 0; c < dk; ++c) kt[c] = sqrt(p->beta_k[(t * H + h) * dk + c]) * k[c];
            for (int i = 0; i < dv; ++i)
                vt[i] = p->beta_v ? sqrt(p->beta_v[(t * H + h) * dv + i]) * v[i] : v[i];
            for (int c = 0; c < dk; ++c) {
                const double ac = exp(log_decay(p, t, h, c));   /* column c decays */
                for (int i = 0; i < dv; ++i) S[i * dk + c] = ac * S[i * dk + c];
            }
            for (int i = 0; i < dv; ++i) {
                double e = 0.0;
                for (int c = 0; c < dk; ++c) e += kt[c] * S[i * dk + c];
                r[i] = e;                         /* (S_{t-1} Diag(alpha) k~)_i */
            }
            for (int i = 0; i < dv; ++i)
                for (int c = 0; c < dk; ++c) S[i * dk + c] += (vt[i] - r[i]) * kt[c];
            double *ot = p->o + (t * H + h) * dv;
            for (int i = 0; i < dv; ++i) {
                double e = 0.0;
                for (int c = 0; c < dk; ++c) e += q[c] * S[i * dk + c];
                ot[i] = e;                                      /* o_t = S_t q_t */
            }
            continue;
        }
        const double b = p->beta[t * H + h];
        if (!p->channel_decay) {
            /* S <- alpha S (I - b k k^T) + b v k^T
             *    = alpha S - alpha b (S k) k^T + b v k^T                     */
            const double a = exp(log_decay(p, t, h, 0));
            for (int i = 0; i < dv; ++i) {
                double acc = 0.0;
                for (int j = 0; j < dk; ++j) acc += S[i * dk + j] * k[j];
                r[i] = acc;                                  /* (S_{t-1} k)_i */
            }
            for (int i = 0; i < dv; ++i)
                for (int j = 0; j < dk; ++j)
                    S[i * dk + j] = a * S[i * dk + j] - a * b * r[i] * k[j] + b * v[i] * k[j];
        } else {
            /* S <- S Diag(alpha) (I - b k k^T) + b v k^T: decay the key
             * columns first, then the delta-rule erase/write along k.         */
            for (int j = 0; j < dk; ++j) {
                const double a = exp(log_decay(p, t, h, j));
                for (int i = 0; i < dv; ++i) S[i * dk + j] *= a;
            }
            for (int i = 0; i < dv; ++i) {
                double acc = 0.0;
                for (int j = 0; j < dk; ++j) acc += S[i * dk + j] * k[j];
                r[i] = acc;                        /* (S_{t-1} Diag(alpha) k)_i */
            }
            for (int i = 0; i < dv; ++i)
                for (int j = 0; j < dk; ++j)
                    S[i * dk + j] = S[i * dk + j] - b * r[i] * k[j] + b * v[i] * k[j];
        }
        /* read-out with the updated state: o_t = S_t q_t */
        double *o = p->o + (t * H + h) * dv;
        for (int i = 0; i < dv; ++i) {
            double acc = 0.0;
            for (int j = 0; j < dk; ++j) acc += S[i * dk + j] * q[j];
            o[i] = acc;
        }
    }
}

/* ------------------------------------------------------------------------ */
/* One chunk of the chunkwise form.                                          */
/*                                                                           */
/* Inputs for L <= C tokens r = 0..L-1 of one head: q, k [L][dk], v [L][dv], */
/* per-channel log decay la [L][dk] (for scalar decay every channel holds    */
/* the same value), beta [L], state S [dv][dk] at the chunk start.           */
/* Outputs (each may be NULL except S_out and O):                            */
/*   G  [L][dk]  cumulative log decay  g_r = sum_{s<=r} log alpha_s          */
/*   A  [L][L]   strictly lower: A_rs = beta_r sum_c k_rc k_sc e^{g_rc-g_sc} */
/*   T  [L][L]   (I + A)^{-1}, unit lower triangular                         */
/*   W  [L][dk]  T diag(beta) (K . e^{G})                                    */
/*   U  [L][dv]  T diag(beta) V                                              */
/*   Vp [L][dv]  V' = U - W S^T                                              */
/*   O  [L][dv]  (Q . e^{G}) S^T + (causal decayed Q K^T) V'                 */
/*   S_out [dv][dk]  S Diag(e^{g_L}) + V'^T (K . e^{g_L - G})                */
/* ------------------------------------------------------------------------ */
void oracle_gdn_chunk_stage(int L, int dk, int dv,
                            const double *q, const double *k, const double *v,
                            const double *la, const double *beta, const double *S,
                            double *G_out, double *A_out, double *T_out,
                            double *W_out, double *U_out, double *Vp_out,
                            double *O, double *S_out) {
    double *G = (double *)calloc((size_t)L * dk, sizeof(double));
    double *A = (double *)calloc((size_t)L * L, sizeof(double));
    double *T = (double *)calloc((size_t)L * L, sizeof(double));
    double *W = (double *)calloc((size_t)L * dk, sizeof(double));
    double *U = (double *)calloc((size_t)L * dv, sizeof(double));
    double *Vp = (double *)calloc((size_t)L * dv, sizeof(double));

    /* step 1: cumulative log decay within the chunk */
    for (int c = 0; c < dk; ++c) {
        double acc = 0.0;
        for (int r = 0; r < L; ++r) { acc += la[r * dk + c]; G[r * dk + c] = acc; }
    }
    /* step 2: strictly lower-triangular beta-scaled, decay-scaled K K^T */
    for (int r = 0; r < L; ++r)
        for (int s = 0; s < r; ++s) {
            double acc = 0.0;
            for (int c = 0; c < dk; ++c)
                acc += k[r * dk + c] * k[s * dk + c] * exp(G[r * dk + c] - G[s * dk + c]);
            A[r * L + s] = beta[r] * acc;
        }
    /* step 3: UT factor T = (I + A)^{-1} by forward substitution:
     * (I + A) T = I  =>  T_ij = delta_ij - sum_{j <= m < i} A_im T_mj         */
    for (int i = 0; i < L; ++i) {
        T[i * L + i] = 1.0;
        for (int j = 0; j < i; ++j) {
            double acc = 0.0;
            for (int m = j; m < i; ++m) acc += A[i * L + m] * T[m * L + j];
            T[i * L + j] = -acc;
        }
    }
    /* step 4: W = T diag(beta) (K . e^{G}),  U = T diag(beta) V */
    for (int r = 0; r < L; ++r) {
        for (int c = 0; c < dk; ++c) {
            double acc = 0.0;
            for (int s = 0; s <= r; ++s)
                acc += T[r * L + s] * beta[s] * k[s * dk + c] * exp(G[s * dk + c]);
            W[r * dk + c] = acc;
        }
        for (int i = 0; i < dv; ++i) {
            double acc = 0.0;
            for (int s = 0; s <= r; ++s) acc += T[r * L + s] * beta[s] * v[s * dv + i];
            U[r * dv + i] = acc;
        }
    }
    /* step 5a: V' = U - W S^T (the pseudo-values once the chunk-start state's
     * prediction is subtracted)                                              */
    for (int r = 0; r < L; ++r)
        for (int i = 0; i < dv; ++i) {
            double acc = 0.0;
            for (int c = 0; c < dk; ++c) acc += W[r * dk + c] * S[i * dk + c];
            Vp[r * dv + i] = U[r * dv + i] - acc;
        }
    /* step 6: output = query on the chunk-start state + intra-chunk causal part */
    for (int r = 0; r < L; ++r)
        for (int i = 0; i < dv; ++i) {
            double acc = 0.0;
            for (int c = 0; c < dk; ++c) acc += q[r * dk + c] * exp(G[r * dk + c]) * S[i * dk + c];
            for (int s = 0; s <= r; ++s) {
                double qk = 0.0;
                for (int c = 0; c < dk; ++c)
                    qk += q[r * dk + c] * k[s * dk + c] * exp(G[r * dk + c] - G[s * dk + c]);
                acc += qk * Vp[s * dv + i];
            }
            O[r * dv + i] = acc;
        }
    /* step 5b: state at the chunk end */
    for (int i = 0; i < dv; ++i)
        for (int c = 0; c < dk; ++c) {
            const double gL = G[(L - 1) * dk + c];
            double acc = S[i * dk + c] * exp(gL);
            for (int s = 0; s < L; ++s) acc += Vp[s * dv + i] * k[s * dk + c] * exp(gL - G[s * dk + c]);
            S_out[i * dk + c] = acc;
        }

    if (G_out) memcpy(G_out, G, sizeof(double) * L * dk);
    if (A_out) memcpy(A_out, A, sizeof(double) * L * L);
    if (T_out) memcpy(T_out, T, sizeof(double) * L * L);
    if (W_out) memcpy(W_out, W, sizeof(double) * L * dk);
    if (U_out) memcpy(U_out, U, sizeof(double) * L * dv);
    if (Vp_out) memcpy(Vp_out, Vp, sizeof(double) * L * dv);
    free(G); free(A); free(T); free(W); free(U); free(Vp);
}

static void chunkwise_chain(const problem *p, int n, int h, double *S) {
    const int H = p->H, dk = p->dk, dv = p->dv, C = p->chunk;
    double *q = (double *)malloc(sizeof(double) * C * dk);
    double *k = (double *)malloc(sizeof(double) * C * dk);
    double *v = (double *)malloc(sizeof(double) * C * dv);
    double *la = (double *)malloc(sizeof(double) * C * dk);
    double *b = (double *)malloc(sizeof(double) * C);
    double *O = (double *)malloc(sizeof(double) * C * dv);
    double *S_next = (double *)malloc(sizeof(double) * dv * dk);
    for (int64_t t0 = p->seq_start[n]; t0 < p->seq_start[n + 1]; t0 += C) {
        int64_t rem = p->seq_start[n + 1] - t0;
        const int L = rem < C ? (int)rem : C;   /* chunks never cross sequences */
        for (int r = 0; r < L; ++r) {
            const int64_t t = t0 + r;
            memcpy(q + r * dk, p->q + (t * H + h) * dk, sizeof(double) * dk);
            memcpy(k + r * dk, p->k + (t * H + h) * dk, sizeof(double) * dk);
            memcpy(v + r * dv, p->v + (t * H + h) * dv, sizeof(double) * dv);
            for (int c = 0; c < dk; ++c) la[r * dk + c] = log_decay(p, t, h, c);
            b[r] = p->beta[t * H + h];
        }
        oracle_gdn_chunk_stage(L, dk, dv, q, k, v, la, b, S,
                               NULL, NULL, NULL, NULL, NULL, NULL, O, S_next);
        for (int r = 0; r < L; ++r)
            memcpy(p->o + ((t0 + r) * H + h) * dv, O + r * dv, sizeof(double) * dv);
        memcpy(S, S_next, sizeof(double) * dv * dk);
    }
    free(q); free(k); free(v); free(la); free(b); free(O); free(S_next);
}

/* ------------------------------------------------------------------------ */
/* Thread pool over independent (sequence, head) chains.                     */
/* ------------------------------------------------------------------------ */
typedef struct {
    const problem *p;
    int chunkwise;
    int64_t next;              /* next work item, taken under the mutex */
    pthread_mutex_t mu;
} pool;

static void *worker(void *arg) {
    pool *pl = (pool *)arg;
    const problem *p = pl->p;
    const int64_t items = (int64_t)p->n_seqs * p->H;
    double *S = (double *)malloc(sizeof(double) * p->dv * p->dk);
    double *r = (double *)malloc(sizeof(double) * (2 * p->dv + p->dk));
    for (;;) {
        pthread_mutex_lock(&pl->mu);
        const int64_t it = pl->next++;
        pthread_mutex_unlock(&pl->mu);
        if (it >= items) break;
        const int n = (int)(it / p->H), h = (int)(it % p->H);
        const size_t sd = (size_t)p->dv * p->dk;
        if (p->S0) memcpy(S, p->S0 + ((size_t)n * p->H + h) * sd, sizeof(double) * sd);
        else memset(S, 0, sizeof(double) * sd);
        if (pl->chunkwise) chunkwise_chain(p, n, h, S);
        else recurrent_chain(p, n, h, S, r);
        if (p->S_final) memcpy(p->S_final + ((size_t)n * p->H + h) * sd, S, sizeof(double) * sd);
    }
    free(S); free(r);
    return NULL;
}

static int run(const problem *p, int chunkwise, int nthreads) {
    if (nthreads <= 0) nthreads = (int)sysconf(_SC_NPROCESSORS_ONLN);
    if (nthreads < 1) nthreads = 1;
    const int64_t items = (int64_t)p->n_seqs * p->H;
    if (nthreads > items) nthreads = items > 0 ? (int)items : 1;
    pool pl;
    pl.p = p; pl.chunkwise = chunkwise; pl.next = 0;
    pthread_mutex_init(&pl.mu, NULL);
    pthread_t *th = (pthread_t *)malloc(sizeof(pthread_t) * nthreads);
    for (int i = 0; i < nthreads; ++i) pthread_create(&th[i], NULL, worker, &pl);
    for (int i = 0; i < nthreads; ++i) pthread_join(th[i], NULL);
    free(th);
    pthread_mutex_destroy(&pl.mu);
    return nthreads;
}

/* Returns the number of threads used, or -1 on invalid arguments. */
int oracle_gdn_recurrent(int n_seqs, const int64_t *seq_start, int H, int dk, int dv,
                         int channel_decay, const double *q, const double *k, const double *v,
                         const double *log_alpha, const double *beta, const double *S0,
                         double *o, double *S_final, int nthreads) {
    if (n_seqs < 0 || H <= 0 || dk <= 0 || dv <= 0 || !seq_start) return -1;
    problem p = {n_seqs, seq_start, H, dk, dv, channel_decay, q, k, v, log_alpha, beta,
                 S0, o, S_final, 0, NULL, NULL};
    return run(&p, 0, nthreads);
}

/* FG2-GDN / FG2-GDN+ (channel decay): beta_k [tok, H, dk]; beta_v [tok, H, dv]
 * or NULL for FG2-GDN.  Returns the number of threads used, or -1. */
int oracle_fg2_recurrent(int n_seqs, const int64_t *seq_start, int H, int dk, int dv,
                         const double *q, const double *k, const double *v,
                         const double *log_alpha, const double *beta_k, const double *beta_v,
                         const double *S0, double *o, double *S_final, int nthreads) {
    if (n_seqs < 0 || H <= 0 || dk <= 0 || dv <= 0 || !seq_start || !beta_k) return -1;
    problem p = {n_seqs, seq_start, H, dk, dv, 1, q, k, v, log_alpha, NULL,
                 S0, o, S_final, 0, beta_k, beta_v};
    return run(&p, 0, nthreads);
}

int oracle_gdn_chunkwise(int n_seqs, const int64_t *seq_start, int H, int dk, int dv,
                         int channel_decay, const double *q, const double *k, const double *v,
                         const double *log_alpha, const double *beta, const double *S0,
                         double *o, double *S_final, int chunk, int nthreads) {
    if (n_seqs < 0 || H <= 0 || dk <= 0 || dv <= 0 || chunk <= 0 || !seq_start) return -1;
    problem p = {n_seqs, seq_start, H, dk, dv, channel_decay, q, k, v, log_alpha, beta,
                 S0, o, S_final, chunk, NULL, NULL};
    return run(&p, 1, nthreads);
}

/* ------------------------------------------------------------------------ */
/* The input prologue of the fused entry point (FG2-GDN paper, section 3.5,  */
/* "Gate Parameterization"): queries and keys are L2-normalised per token    */
/* and head; the writing rate is a sigmoid of its projection, beta_t =       */
/* sigmoid(b_t); the decay comes from a negative softplus of its projection  */
/* plus an optional bias, log alpha_t = -softplus(a_t + bias).  A zero        */
/* vector is left at zero (its norm is clamped below at 1e-12).              */
/* ------------------------------------------------------------------------ */
static double softplus(double x) {
    /* log(1 + e^x) without overflow: x + log(1 + e^-x) for x > 0 */
    return x > 0 ? x + log1p(exp(-x)) : log1p(exp(x));
}

static double sigmoid(double x) { return 1.0 / (1.0 + exp(-x)); }

static void unit_rows(int64_t rows, int d, const double *in, double *out) {
    for (int64_t r = 0; r < rows; ++r) {
        double ss = 0.0;
        for (int c = 0; c < d; ++c) ss += in[r * d + c] * in[r * d + c];
        double nrm = sqrt(ss);
        if (nrm < 1e-12) nrm = 1e-12;
        for (int c = 0; c < d; ++c) out[r * d + c] = in[r * d + c] / nrm;
    }
}

/* ntok tokens x H heads.  channel = 0: a_logit [ntok,H], a_bias [H] or NULL;
 * channel = 1: a_logit [ntok,H,dk], a_bias [H,dk] or NULL.  b_logit [ntok,H]. */
int oracle_gdn_prologue(int64_t ntok, int H, int dk, int channel, const double *q_raw,
                        const double *k_raw, const double *a_logit, const double *a_bias,
                        const double *b_logit, double *q, double *k, double *log_alpha,
                        double *beta) {
    if (ntok < 0 || H <= 0 || dk <= 0) return -1;
    unit_rows(ntok * H, dk, q_raw, q);
    unit_rows(ntok * H, dk, k_raw, k);
    const int per = channel ? dk : 1;
    for (int64_t t = 0; t < ntok; ++t)
        for (int h = 0; h < H; ++h) {
            beta[t * H + h] = sigmoid(b_logit[t * H + h]);
            for (int c = 0; c < per; ++c) {
                const int64_t i = (t * H + h) * per + c;
                const double bias = a_bias ? a_bias[h * per + c] : 0.0;
                log_alpha[i] = -softplus(a_logit[i] + bias);
            }
        }
    return 0;
}
