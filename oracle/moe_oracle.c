/*
 * moe_oracle.c -- plain, slow, fp64 CPU oracle for the routed-expert MoE
 * feed-forward block of the hybrid decoder at decode time.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path links, loads or calls
 * this file; the test suite and the benchmark's CPU leg use it.  It shares no
 * code, header, table or helper with the CUDA library.
 *
 * What it computes.  The Core AI card for the Qwen3.6-35B-A3B text decoder
 * (first section) describes every FFN as a 256-expert top-8 mixture with a
 * shared expert: a router Linear(hidden, 256), a softmax over all experts,
 * the top 8, renormalised by their sum; the experts as SwitchGLU layers
 * gathered by index; an always-on shared MLP scaled by a per-token
 * sigmoid(shared_expert_gate(x)); output = routed sum + gated shared.  Its
 * "Speed" section puts the cost in reading only the routed experts' weights.
 * Where the card stops, this oracle takes the plainest reading:
 *
 *   SwitchGLU(x) = W_down (silu(W_gate x) * (W_up x)),  silu(u) = u sigmoid(u)
 *   logits = W_router x;  p = softmax(logits);  top-k by p (ties: lower index);
 *   w_e = p_e / sum_{top-k} p;   y = sum_{e in top-k} w_e SwitchGLU_e(x)
 *       + sigmoid(w_sgate . x) SwitchGLU_shared(x)
 *
 * Layouts (row-major, fp64):
 *   x        [n_tok, hidden]
 *   w_router [n_exp, hidden]
 *   w_gate, w_up [n_exp, inter, hidden];  w_down [n_exp, hidden, inter]
 *   ws_gate, ws_up [s_inter, hidden];     ws_down [hidden, s_inter];  w_sgate [hidden]
 *   (s_inter == 0: no shared expert)
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

typedef struct orc_moe_problem {
    int32_t n_tok, hidden, n_exp, top_k, inter, s_inter;
    const double *x, *w_router;
    const double *w_gate, *w_up, *w_down;
    const double *ws_gate, *ws_up, *ws_down, *w_sgate;
} orc_moe_problem;

/* Router of every token: probabilities p [n_tok, n_exp] (softmax of the
 * logits), the top-k experts idx [n_tok, top_k] in decreasing p (ties to the
 * lower index) and their renormalised weights w [n_tok, top_k]. */
void orc_moe_route(const orc_moe_problem *p, double *probs, int32_t *idx, double *w) {
    const int H = p->hidden, E = p->n_exp, K = p->top_k;
    double *lg = malloc(sizeof(double) * E);
    char *taken = malloc((size_t)E);
    for (int t = 0; t < p->n_tok; ++t) {
        const double *xt = p->x + (size_t)t * H;
        double m = -INFINITY;
        for (int e = 0; e < E; ++e) {
            double s = 0.0;
            for (int i = 0; i < H; ++i) s += p->w_router[(size_t)e * H + i] * xt[i];
            lg[e] = s;
            if (s > m) m = s;
        }
        double z = 0.0;
        for (int e = 0; e < E; ++e) z += exp(lg[e] - m);
        double *pt = probs + (size_t)t * E;
        for (int e = 0; e < E; ++e) pt[e] = exp(lg[e] - m) / z;
        memset(taken, 0, (size_t)E);
        double sum = 0.0;
        for (int k = 0; k < K; ++k) {
            int best = -1;
            for (int e = 0; e < E; ++e)
                if (!taken[e] && (best < 0 || pt[e] > pt[best])) best = e;
            taken[best] = 1;
            idx[(size_t)t * K + k] = best;
            sum += pt[best];
        }
        for (int k = 0; k < K; ++k) w[(size_t)t * K + k] = pt[idx[(size_t)t * K + k]] / sum;
    }
    free(lg);
    free(taken);
}

static double silu(double u) { return u / (1.0 + exp(-u)); }

/* SwitchGLU of one token through one expert's (or the shared expert's)
 * weights, accumulated into y with factor f. */
static void swiglu_acc(const double *xt, const double *wg, const double *wu, const double *wd,
                       int H, int I, double f, double *h, double *y) {
    for (int j = 0; j < I; ++j) {
        double g = 0.0, u = 0.0;
        for (int i = 0; i < H; ++i) {
            g += wg[(size_t)j * H + i] * xt[i];
            u += wu[(size_t)j * H + i] * xt[i];
        }
        h[j] = silu(g) * u;
    }
    for (int i = 0; i < H; ++i) {
        double s = 0.0;
        for (int j = 0; j < I; ++j) s += wd[(size_t)i * I + j] * h[j];
        y[i] += f * s;
    }
}

/* The block's output y [n_tok, hidden] for a given routing (idx, w as from
 * orc_moe_route, or any other valid choice): the weighted routed experts plus
 * the gated shared expert.  Returns 1 for an expert index out of range. */
int orc_moe_forward(const orc_moe_problem *p, const int32_t *idx, const double *w, double *y) {
    const int H = p->hidden, I = p->inter, K = p->top_k;
    const int hmax = I > p->s_inter ? I : p->s_inter;
    double *h = malloc(sizeof(double) * (hmax > 0 ? hmax : 1));
    int rc = 0;
    for (int t = 0; t < p->n_tok && !rc; ++t) {
        const double *xt = p->x + (size_t)t * H;
        double *yt = y + (size_t)t * H;
        for (int i = 0; i < H; ++i) yt[i] = 0.0;
        for (int k = 0; k < K; ++k) {
            const int e = idx[(size_t)t * K + k];
            if (e < 0 || e >= p->n_exp) {
                rc = 1;
                break;
            }
            const size_t off = (size_t)e * I * H;
            swiglu_acc(xt, p->w_gate + off, p->w_up + off, p->w_down + off, H, I,
                       w[(size_t)t * K + k], h, yt);
        }
        if (p->s_inter > 0 && !rc) {
            double s = 0.0;
            for (int i = 0; i < H; ++i) s += p->w_sgate[i] * xt[i];
            swiglu_acc(xt, p->ws_gate, p->ws_up, p->ws_down, H, p->s_inter, 1.0 / (1.0 + exp(-s)),
                       h, yt);
        }
    }
    free(h);
    return rc;
}
