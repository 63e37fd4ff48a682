/*
 * gdr_oracle.c -- plain, slow, fp64 CPU oracle for the Gated DeltaNet token mixer.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path links, loads or calls
 * this file.  Only the test suite, the smoke check and the CPU-baseline leg of
 * the benchmark use it.  It shares no code, header, table or helper with the
 * CUDA library; the two meet only through the inputs a test hands to both.
 *
 * What it computes (one value head at a time, tokens in order):
 *
 *   The pages name the mixer but never write its equations.  The Qwen3.5 Chat
 *   guide (soniqo.audio/de/guides/chat, section "Architektur"; the Arabic copy
 *   has the same section) describes these layers as linear attention driven
 *   by a gated delta rule recurrence and followed by RMSNormGated.  The Core
 *   AI model-zoo card for Qwen3.6-35B-A3B (first section) gives the head
 *   layout: 16 key/query heads, each serving two of 32 value heads (GVA).  The recurrence used here is the gated
 *   delta rule as published in "Gated Delta Networks: Improving Mamba2 with
 *   Delta Rule" (Yang, Kautz, Hatamizadeh, ICLR 2025, eq. of the gated delta
 *   rule):
 *
 *       S_t = exp(g_t) * S_{t-1} * (I - beta_t k_t k_t^T) + beta_t v_t k_t^T
 *       o_t = S_t q_t
 *
 *   with q, k L2-normalised per (token, key head), and the output gate
 *       y_t = o_t / sqrt(mean(o_t^2) + eps_n) * w * z_t * sigmoid(z_t).
 *
 *   S is d_v x d_k, row-major, so row i belongs to value dimension i.
 *   Value head h_v reads key head floor(h_v * H_k / H_v) (each key head feeds
 *   H_v/H_k consecutive value heads: the same card expands key heads by
 *   repetition, section "How to reproduce").
 *
 * Three independent forms are provided so they can be checked against each
 * other and against closed forms:
 *   orc_gdr_recurrent   -- the definition, one token at a time;
 *   orc_gdr_chunked     -- the chunkwise (WY / UT transform) form derived from
 *                          the same definition, any chunk size;
 *   orc_gdr_bruteforce  -- explicit d_k x d_k transition matrices multiplied
 *                          out for short sequences (T <= 8), no recurrence.
 * plus orc_rmsnorm_gated, the output gate on its own.
 *
 * All arithmetic is double precision.  Callers pass inputs already widened to
 * double (bf16 and fp32 values widen exactly).
 */
#include <math.h>
#include <pthread.h>
#include <stdatomic.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* One problem: packed variable-length sequences.
 *   q, k        [n_tok, H_k, d_k]
 *   v, z        [n_tok, H_v, d_v]      (z may be NULL: y is then not produced)
 *   g, beta     [n_tok, H_v]           (g is the log of the decay, exp(g) in (0,1])
 *   cu_seqlens  [n_seq + 1]            token offsets of each sequence
 *   s0          [n_seq, H_v, d_v, d_k] initial state, NULL means zeros
 *   w           [d_v]                  output-gate weight, NULL means ones
 */
typedef struct orc_problem {
    int64_t n_tok;
    int32_t n_seq, H_k, H_v, d_k, d_v;
    int32_t qk_l2norm; /* 1: normalise q and k here; 0: use them as given */
    double scale;      /* multiplies q after normalisation */
    double eps_l2;     /* q_hat = q / sqrt(|q|^2 + eps_l2) */
    double eps_norm;   /* y = o / sqrt(mean(o^2) + eps_norm) * ... */
    const double *q, *k, *v, *z, *g, *beta, *s0, *w;
    const int64_t *cu_seqlens;
} orc_problem;

/* ---------------------------------------------------------------- helpers */

static int key_head_of(const orc_problem *p, int hv) {
    return (int)(((int64_t)hv * p->H_k) / p->H_v);
}

/* x_hat = mult * x / sqrt(sum x^2 + eps), or mult * x when normalisation is off. */
static void l2_normalise(const double *x, int n, int on, double eps, double mult,
                         double *out) {
    double ss = 0.0;
    for (int i = 0; i < n; ++i) ss += x[i] * x[i];
    double f = on ? mult / sqrt(ss + eps) : mult;
    for (int i = 0; i < n; ++i) out[i] = x[i] * f;
}

static void load_q_hat(const orc_problem *p, int64_t tok, int hk, double *out) {
    l2_normalise(p->q + (tok * p->H_k + hk) * p->d_k, p->d_k, p->qk_l2norm, p->eps_l2,
                 p->scale, out);
}

static void load_k_hat(const orc_problem *p, int64_t tok, int hk, double *out) {
    l2_normalise(p->k + (tok * p->H_k + hk) * p->d_k, p->d_k, p->qk_l2norm, p->eps_l2,
                 1.0, out);
}

static void load_s0(const orc_problem *p, int seq, int hv, double *S) {
    size_t n = (size_t)p->d_v * p->d_k;
    if (p->s0)
        memcpy(S, p->s0 + ((size_t)seq * p->H_v + hv) * n, n * sizeof(double));
    else
        memset(S, 0, n * sizeof(double));
}

static void store_state(const orc_problem *p, int seq, int hv, const double *S,
                        double *s_final) {
    if (!s_final) return;
    size_t n = (size_t)p->d_v * p->d_k;
    memcpy(s_final + ((size_t)seq * p->H_v + hv) * n, S, n * sizeof(double));
}

/* ------------------------------------------------------- RMSNormGated gate */

/* y = o / sqrt(mean_i o_i^2 + eps) * w * z * sigmoid(z) over one row of n.
 * sigmoid(z) = 1 / (1 + exp(-z)); z * sigmoid(z) is SiLU(z). */
static void rmsnorm_gated_row(const double *o, const double *z, const double *w, int n,
                              double eps, double *y) {
    double ms = 0.0;
    for (int i = 0; i < n; ++i) ms += o[i] * o[i];
    ms /= n;
    double r = 1.0 / sqrt(ms + eps);
    for (int i = 0; i < n; ++i) {
        double wi = w ? w[i] : 1.0;
        double silu = z[i] / (1.0 + exp(-z[i]));
        y[i] = o[i] * r * wi * silu;
    }
}

/* Rows of n values: o, z, y are [rows, n]. */
void orc_rmsnorm_gated(const double *o, const double *z, const double *w, int64_t rows,
                       int n, double eps, double *y) {
    for (int64_t r = 0; r < rows; ++r)
        rmsnorm_gated_row(o + r * n, z + r * n, w, n, eps, y + r * n);
}

/* Gate inputs from raw projection outputs (the reading taken where the pages
 * are silent: the parameterisation of the published Gated DeltaNet and Mamba-2
 * layers, per value head h):
 *   g_t    = -exp(A_log[h]) * softplus(a_t + dt_bias[h])
 *   beta_t = sigmoid(b_t) = 1 / (1 + exp(-b_t))
 * with softplus(x) = log(1 + exp(x)), evaluated as max(x, 0) + log1p(exp(-|x|)),
 * the same number without overflow.  a, b, g, beta are [n_tok, H_v]. */
void orc_gate_from_raw(int64_t n_tok, int H_v, const double *a, const double *b,
                       const double *A_log, const double *dt_bias, double *g, double *beta) {
    for (int64_t t = 0; t < n_tok; ++t) {
        for (int h = 0; h < H_v; ++h) {
            const size_t i = (size_t)t * H_v + h;
            const double x = a[i] + dt_bias[h];
            const double softplus = fmax(x, 0.0) + log1p(exp(-fabs(x)));
            g[i] = -exp(A_log[h]) * softplus;
            beta[i] = 1.0 / (1.0 + exp(-b[i]));
        }
    }
}

/* Apply the gate to every (token, value head) row of o produced for a problem. */
static void gate_outputs(const orc_problem *p, int seq, int hv, const double *o,
                         double *y) {
    if (!y || !p->z) return;
    for (int64_t t = p->cu_seqlens[seq]; t < p->cu_seqlens[seq + 1]; ++t) {
        size_t off = ((size_t)t * p->H_v + hv) * p->d_v;
        rmsnorm_gated_row(o + off, p->z + off, p->w, p->d_v, p->eps_norm, y + off);
    }
}

/* ------------------------------------------------------ recurrent (definition) */

/* One (sequence, value head): the definition, token by token.
 *   1. q_hat, k_hat (L2 normalised, q also scaled)
 *   2. alpha = exp(g_t)
 *   3. S <- alpha * S
 *   4. u = S k_hat
 *   5. delta = beta_t (v_t - u)
 *   6. S <- S + delta k_hat^T
 *   7. o_t = S q_hat
 * Steps 3-6 equal exp(g) S (I - beta k k^T) + beta v k^T after expansion. */
static void recurrent_one(const orc_problem *p, int seq, int hv, double *o,
                          double *s_final, double *S, double *qh, double *kh, double *u) {
    const int dk = p->d_k, dv = p->d_v, hk = key_head_of(p, hv);
    load_s0(p, seq, hv, S);
    for (int64_t t = p->cu_seqlens[seq]; t < p->cu_seqlens[seq + 1]; ++t) {
        load_q_hat(p, t, hk, qh);
        load_k_hat(p, t, hk, kh);
        const double alpha = exp(p->g[t * p->H_v + hv]);
        const double beta = p->beta[t * p->H_v + hv];
        const double *vt = p->v + ((size_t)t * p->H_v + hv) * dv;
        for (int i = 0; i < dv * dk; ++i) S[i] *= alpha;
        for (int i = 0; i < dv; ++i) {
            double acc = 0.0;
            for (int j = 0; j < dk; ++j) acc += S[i * dk + j] * kh[j];
            u[i] = acc;
        }
        for (int i = 0; i < dv; ++i) {
            double delta = beta * (vt[i] - u[i]);
            for (int j = 0; j < dk; ++j) S[i * dk + j] += delta * kh[j];
        }
        double *ot = o + ((size_t)t * p->H_v + hv) * dv;
        for (int i = 0; i < dv; ++i) {
            double acc = 0.0;
            for (int j = 0; j < dk; ++j) acc += S[i * dk + j] * qh[j];
            ot[i] = acc;
        }
    }
    store_state(p, seq, hv, S, s_final);
}

/* Work is split over (sequence, value head) pairs; threads take pairs from a
 * shared counter.  Each pair is independent, so the result does not depend on
 * the thread count. */
typedef struct work_ctx {
    const orc_problem *p;
    double *o, *y, *s_final;
    int chunk;
    atomic_long next;
    int kind; /* 0 recurrent, 1 chunked */
} work_ctx;

static void chunked_one(const orc_problem *p, int seq, int hv, int C, double *o,
                        double *s_final);

static void *worker(void *arg) {
    work_ctx *c = (work_ctx *)arg;
    const orc_problem *p = c->p;
    const long total = (long)p->n_seq * p->H_v;
    double *S = malloc(sizeof(double) * (size_t)p->d_v * p->d_k);
    double *qh = malloc(sizeof(double) * p->d_k);
    double *kh = malloc(sizeof(double) * p->d_k);
    double *u = malloc(sizeof(double) * p->d_v);
    for (;;) {
        long item = atomic_fetch_add(&c->next, 1);
        if (item >= total) break;
        int seq = (int)(item / p->H_v), hv = (int)(item % p->H_v);
        if (c->kind == 0)
            recurrent_one(p, seq, hv, c->o, c->s_final, S, qh, kh, u);
        else
            chunked_one(p, seq, hv, c->chunk, c->o, c->s_final);
        gate_outputs(p, seq, hv, c->o, c->y);
    }
    free(S); free(qh); free(kh); free(u);
    return NULL;
}

static int run_pool(work_ctx *c, int n_threads) {
    if (n_threads < 1) n_threads = 1;
    atomic_init(&c->next, 0);
    if (n_threads == 1) {
        worker(c);
        return 0;
    }
    pthread_t *th = malloc(sizeof(pthread_t) * n_threads);
    int started = 0;
    for (int i = 0; i < n_threads; ++i) {
        if (pthread_create(&th[i], NULL, worker, c) != 0) break;
        ++started;
    }
    if (started == 0) worker(c);
    for (int i = 0; i < started; ++i) pthread_join(th[i], NULL);
    free(th);
    return 0;
}

/* o [n_tok, H_v, d_v] (required), y same shape or NULL, s_final
 * [n_seq, H_v, d_v, d_k] or NULL.  Returns 0. */
int orc_gdr_recurrent(const orc_problem *p, double *o, double *y, double *s_final,
                      int n_threads) {
    work_ctx c = {.p = p, .o = o, .y = y, .s_final = s_final, .chunk = 0, .kind = 0};
    return run_pool(&c, n_threads);
}

/* ------------------------------------------------------------ chunked form */

/* Decay from token s to token r inside a chunk (s <= r, chunk-local indices):
 * prod_{s < j <= r} alpha_j = exp(gamma_r - gamma_s), gamma the running sum
 * of g.  Written as a product so that g = -inf (alpha = 0) stays exact. */
static double decay_between(const double *alpha, int s, int r) {
    double d = 1.0;
    for (int j = s + 1; j <= r; ++j) d *= alpha[j];
    return d;
}

/* One (sequence, value head), chunks of C tokens (the last one may be shorter).
 * Derivation, with S_0 the state entering the chunk, r, s chunk-local token
 * indices, e^{gamma_r} = prod_{j<=r} alpha_j:
 *   S_r = e^{gamma_r} S_0 + sum_{s<=r} e^{gamma_r-gamma_s} delta_s k_s^T
 *   delta_r = beta_r (v_r - alpha_r S_{r-1} k_r)
 *     => delta_r + sum_{s<r} A_rs delta_s = beta_r v_r - beta_r e^{gamma_r} S_0 k_r,
 *        A_rs = beta_r e^{gamma_r-gamma_s} (k_r . k_s)            (s < r)
 *     => Delta = T diag(beta) V - T diag(beta e^gamma) K S_0^T = U - W S_0^T,
 *        T = (I + A)^{-1}  (unit lower triangular: forward substitution)
 *   O   = diag(e^gamma) Q S_0^T + P Delta,  P_rs = e^{gamma_r-gamma_s} (q_r . k_s), s <= r
 *   S_L = e^{gamma_L} S_0 + Delta^T diag(e^{gamma_L-gamma}) K
 */
static void chunked_one(const orc_problem *p, int seq, int hv, int C, double *o,
                        double *s_final) {
    const int dk = p->d_k, dv = p->d_v, hk = key_head_of(p, hv);
    double *S = malloc(sizeof(double) * (size_t)dv * dk);
    double *Snew = malloc(sizeof(double) * (size_t)dv * dk);
    double *Q = malloc(sizeof(double) * (size_t)C * dk);
    double *K = malloc(sizeof(double) * (size_t)C * dk);
    double *V = malloc(sizeof(double) * (size_t)C * dv);
    double *alpha = malloc(sizeof(double) * C);
    double *beta = malloc(sizeof(double) * C);
    double *eg = malloc(sizeof(double) * C); /* e^{gamma_r} */
    double *A = malloc(sizeof(double) * (size_t)C * C);
    double *T = malloc(sizeof(double) * (size_t)C * C);
    double *P = malloc(sizeof(double) * (size_t)C * C);
    double *U = malloc(sizeof(double) * (size_t)C * dv);
    double *W = malloc(sizeof(double) * (size_t)C * dk);
    double *D = malloc(sizeof(double) * (size_t)C * dv); /* Delta */

    load_s0(p, seq, hv, S);
    const int64_t t0 = p->cu_seqlens[seq], t1 = p->cu_seqlens[seq + 1];
    for (int64_t c0 = t0; c0 < t1; c0 += C) {
        const int L = (int)((t1 - c0) < C ? (t1 - c0) : C);
        for (int r = 0; r < L; ++r) {
            int64_t t = c0 + r;
            load_q_hat(p, t, hk, Q + (size_t)r * dk);
            load_k_hat(p, t, hk, K + (size_t)r * dk);
            memcpy(V + (size_t)r * dv, p->v + ((size_t)t * p->H_v + hv) * dv,
                   sizeof(double) * dv);
            alpha[r] = exp(p->g[t * p->H_v + hv]);
            beta[r] = p->beta[t * p->H_v + hv];
            eg[r] = (r == 0 ? 1.0 : eg[r - 1]) * alpha[r];
        }
        /* A (strictly lower) and P (lower, diagonal included). */
        for (int r = 0; r < L; ++r)
            for (int s = 0; s < L; ++s) {
                double kk = 0.0, qk = 0.0;
                for (int j = 0; j < dk; ++j) {
                    kk += K[(size_t)r * dk + j] * K[(size_t)s * dk + j];
                    qk += Q[(size_t)r * dk + j] * K[(size_t)s * dk + j];
                }
                A[r * C + s] = (s < r) ? beta[r] * decay_between(alpha, s, r) * kk : 0.0;
                P[r * C + s] = (s <= r) ? decay_between(alpha, s, r) * qk : 0.0;
            }
        /* T = (I + A)^{-1} by forward substitution, column by column:
         * T_rc = [r == c] - sum_{c <= s < r} A_rs T_sc. */
        for (int c = 0; c < L; ++c)
            for (int r = 0; r < L; ++r) {
                if (r < c) { T[r * C + c] = 0.0; continue; }
                double acc = (r == c) ? 1.0 : 0.0;
                for (int s = c; s < r; ++s) acc -= A[r * C + s] * T[s * C + c];
                T[r * C + c] = acc;
            }
        /* U = T diag(beta) V ; W = T diag(beta e^gamma) K */
        for (int r = 0; r < L; ++r) {
            for (int i = 0; i < dv; ++i) {
                double acc = 0.0;
                for (int s = 0; s <= r; ++s) acc += T[r * C + s] * beta[s] * V[(size_t)s * dv + i];
                U[(size_t)r * dv + i] = acc;
            }
            for (int j = 0; j < dk; ++j) {
                double acc = 0.0;
                for (int s = 0; s <= r; ++s)
                    acc += T[r * C + s] * beta[s] * eg[s] * K[(size_t)s * dk + j];
                W[(size_t)r * dk + j] = acc;
            }
        }
        /* Delta = U - W S_0^T */
        for (int r = 0; r < L; ++r)
            for (int i = 0; i < dv; ++i) {
                double acc = 0.0;
                for (int j = 0; j < dk; ++j) acc += W[(size_t)r * dk + j] * S[(size_t)i * dk + j];
                D[(size_t)r * dv + i] = U[(size_t)r * dv + i] - acc;
            }
        /* O = diag(e^gamma) Q S_0^T + P Delta */
        for (int r = 0; r < L; ++r) {
            double *ot = o + ((size_t)(c0 + r) * p->H_v + hv) * dv;
            for (int i = 0; i < dv; ++i) {
                double inter = 0.0, intra = 0.0;
                for (int j = 0; j < dk; ++j) inter += Q[(size_t)r * dk + j] * S[(size_t)i * dk + j];
                for (int s = 0; s <= r; ++s) intra += P[r * C + s] * D[(size_t)s * dv + i];
                ot[i] = eg[r] * inter + intra;
            }
        }
        /* S_L = e^{gamma_L} S_0 + Delta^T diag(e^{gamma_L - gamma}) K */
        for (int i = 0; i < dv; ++i)
            for (int j = 0; j < dk; ++j) {
                double acc = eg[L - 1] * S[(size_t)i * dk + j];
                for (int s = 0; s < L; ++s)
                    acc += D[(size_t)s * dv + i] * decay_between(alpha, s, L - 1) *
                           K[(size_t)s * dk + j];
                Snew[(size_t)i * dk + j] = acc;
            }
        memcpy(S, Snew, sizeof(double) * (size_t)dv * dk);
    }
    store_state(p, seq, hv, S, s_final);
    free(S); free(Snew); free(Q); free(K); free(V); free(alpha); free(beta); free(eg);
    free(A); free(T); free(P); free(U); free(W); free(D);
}

int orc_gdr_chunked(const orc_problem *p, int chunk, double *o, double *y,
                    double *s_final, int n_threads) {
    if (chunk < 1) return 1;
    work_ctx c = {.p = p, .o = o, .y = y, .s_final = s_final, .chunk = chunk, .kind = 1};
    return run_pool(&c, n_threads);
}

/* ------------------------------------------------------------ brute force */

/* out = a (m x n) * b (n x n), all row-major, out must not alias. */
static void matmul_sq(const double *a, const double *b, int m, int n, double *out) {
    for (int i = 0; i < m; ++i)
        for (int j = 0; j < n; ++j) {
            double acc = 0.0;
            for (int l = 0; l < n; ++l) acc += a[i * n + l] * b[l * n + j];
            out[i * n + j] = acc;
        }
}

/* Short sequences only (every sequence length <= 8).  For each t the state is
 * formed from scratch as the unrolled sum
 *   S_t = S_0 M_1 ... M_t + sum_{s<=t} beta_s v_s k_s^T M_{s+1} ... M_t,
 *   M_s = alpha_s (I - beta_s k_s k_s^T)            (d_k x d_k),
 * and o_t = S_t q_t.  No state is carried from one t to the next.
 * Returns 1 if a sequence is longer than 8. */
int orc_gdr_bruteforce(const orc_problem *p, double *o, double *y, double *s_final) {
    const int dk = p->d_k, dv = p->d_v;
    for (int seq = 0; seq < p->n_seq; ++seq)
        if (p->cu_seqlens[seq + 1] - p->cu_seqlens[seq] > 8) return 1;
    double *M = malloc(sizeof(double) * 8 * dk * dk);
    double *tmp = malloc(sizeof(double) * dk * dk);
    double *S0 = malloc(sizeof(double) * dv * dk);
    double *St = malloc(sizeof(double) * dv * dk);
    double *term = malloc(sizeof(double) * dv * dk);
    double *vk = malloc(sizeof(double) * dv * dk);
    double *qh = malloc(sizeof(double) * 8 * dk);
    double *kh = malloc(sizeof(double) * 8 * dk);
    for (int seq = 0; seq < p->n_seq; ++seq) {
        const int64_t t0 = p->cu_seqlens[seq];
        const int T = (int)(p->cu_seqlens[seq + 1] - t0);
        for (int hv = 0; hv < p->H_v; ++hv) {
            const int hk = key_head_of(p, hv);
            load_s0(p, seq, hv, S0);
            for (int s = 0; s < T; ++s) {
                load_q_hat(p, t0 + s, hk, qh + s * dk);
                load_k_hat(p, t0 + s, hk, kh + s * dk);
                double a = exp(p->g[(t0 + s) * p->H_v + hv]);
                double b = p->beta[(t0 + s) * p->H_v + hv];
                for (int i = 0; i < dk; ++i)
                    for (int j = 0; j < dk; ++j)
                        M[(size_t)s * dk * dk + i * dk + j] =
                            a * ((i == j ? 1.0 : 0.0) - b * kh[s * dk + i] * kh[s * dk + j]);
            }
            for (int t = 0; t < T; ++t) {
                /* S_0 M_1 ... M_t  (matrix indices 0..t) */
                memcpy(St, S0, sizeof(double) * dv * dk);
                for (int s = 0; s <= t; ++s) {
                    matmul_sq(St, M + (size_t)s * dk * dk, dv, dk, tmp);
                    memcpy(St, tmp, sizeof(double) * dv * dk);
                }
                for (int s = 0; s <= t; ++s) {
                    double b = p->beta[(t0 + s) * p->H_v + hv];
                    const double *vs = p->v + ((size_t)(t0 + s) * p->H_v + hv) * dv;
                    for (int i = 0; i < dv; ++i)
                        for (int j = 0; j < dk; ++j) vk[i * dk + j] = b * vs[i] * kh[s * dk + j];
                    /* vk * M_{s+1} ... M_t */
                    for (int r = s + 1; r <= t; ++r) {
                        matmul_sq(vk, M + (size_t)r * dk * dk, dv, dk, term);
                        memcpy(vk, term, sizeof(double) * dv * dk);
                    }
                    for (int i = 0; i < dv * dk; ++i) St[i] += vk[i];
                }
                double *ot = o + ((size_t)(t0 + t) * p->H_v + hv) * dv;
                for (int i = 0; i < dv; ++i) {
                    double acc = 0.0;
                    for (int j = 0; j < dk; ++j) acc += St[i * dk + j] * qh[t * dk + j];
                    ot[i] = acc;
                }
                if (t == T - 1) store_state(p, seq, hv, St, s_final);
            }
            if (T == 0) store_state(p, seq, hv, S0, s_final);
            gate_outputs(p, seq, hv, o, y);
        }
    }
    free(M); free(tmp); free(S0); free(St); free(term); free(vk); free(qh);
    free(kh);
    return 0;
}
