/*
 * gattn_oracle.c -- plain, slow, fp64 CPU oracle for one decode step of the
 * gated full-attention layer that sits between the Gated DeltaNet mixers.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path links, loads or calls
 * this file; the test suite and the CPU-baseline leg of the benchmark use it.
 * It shares no code, header, table or helper with the CUDA library.
 *
 * What it computes.  The Qwen3.5 Chat guide (soniqo.audio/de/guides/chat,
 * section "Architektur") names these layers GatedAttention and says they are
 * standard scaled-dot-product attention with a KV cache; the Core AI card for
 * the Qwen3.6-35B-A3B text decoder (first section) gives their shape: head_dim
 * 256, 16 query heads over 2 key/value heads (GQA), partial mRoPE with
 * theta = 1e7.  Where the pages stop, this oracle takes the plainest reading
 * (each reading is listed in the design notes):
 *
 *   - the rotary embedding turns the first rot_dim dimensions of every query
 *     and key head, pairing dimension i with i + rot_dim/2 ("rotate half"),
 *     frequency theta^(-2i/rot_dim), angle = position * frequency; the other
 *     dimensions pass through.  For text tokens the three position components
 *     of mRoPE coincide, which makes it this one-dimensional rotation;
 *   - the new token's position is the number of tokens already cached; its
 *     rotated key and its value are appended at that index;
 *   - query head h reads key/value head floor(h * H_kv / H_q) (consecutive
 *     query heads share a key/value head);
 *   - o = sum_t softmax_t(scale * q_rot . k_t) v_t over the cached tokens and
 *     the new one; the "gate" of gated attention is an output gate,
 *     y = o * sigmoid(gate), elementwise, with gate a second per-head
 *     projection of the token.
 *
 * Layouts (row-major, fp64):
 *   q, gate   [batch, H_q, d]          k, v  [batch, H_kv, d]   (the new token)
 *   k_cache, v_cache  [batch, H_kv, max_len, d]   entries t < cache_len[b] used
 *   cache_len [batch]
 *   y, o      [batch, H_q, d]          k_rot [batch, H_kv, d]  (appended key)
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

typedef struct orc_attn_problem {
    int32_t batch, H_q, H_kv, d, rot_dim, max_len;
    double theta, scale;
    const double *q, *gate, *k, *v;
    const double *k_cache, *v_cache;
    const int64_t *cache_len;
} orc_attn_problem;

/* Rotary embedding of n vectors of d values at one position: pairs
 * (i, i + rot_dim/2) for i < rot_dim/2 turned by the angle pos * theta^(-2i/rot_dim);
 * dimensions from rot_dim on are copied. */
void orc_rope_partial(const double *x, int64_t n, int d, int rot_dim, double pos, double theta,
                      double *out) {
    const int half = rot_dim / 2;
    for (int64_t r = 0; r < n; ++r) {
        const double *xr = x + r * d;
        double *yr = out + r * d;
        for (int i = 0; i < d; ++i) yr[i] = xr[i];
        for (int i = 0; i < half; ++i) {
            const double freq = pow(theta, -2.0 * i / rot_dim);
            const double ang = pos * freq;
            const double c = cos(ang), s = sin(ang);
            const double a = xr[i], b = xr[i + half];
            yr[i] = a * c - b * s;
            yr[i + half] = b * c + a * s;
        }
    }
}

/* One decode step for every sequence and query head.  Returns 0, or 1 when a
 * sequence's cache is full (cache_len[b] >= max_len) or the shape is invalid. */
int orc_gated_attn_decode(const orc_attn_problem *p, double *y, double *o, double *k_rot_out) {
    if (p->H_kv <= 0 || p->H_q % p->H_kv || p->rot_dim < 0 || p->rot_dim > p->d ||
        p->rot_dim % 2)
        return 1;
    const int d = p->d;
    double *qr = malloc(sizeof(double) * d);
    double *kr = malloc(sizeof(double) * d);
    double *acc = malloc(sizeof(double) * d);
    double *score = malloc(sizeof(double) * ((size_t)p->max_len + 1));
    int rc = 0;
    for (int b = 0; b < p->batch && !rc; ++b) {
        const int64_t L = p->cache_len[b];
        if (L < 0 || L >= p->max_len) {
            rc = 1;
            break;
        }
        const double pos = (double)L;
        for (int h = 0; h < p->H_q; ++h) {
            const int g = (int)(((int64_t)h * p->H_kv) / p->H_q);
            const double *kc = p->k_cache + ((size_t)b * p->H_kv + g) * p->max_len * d;
            const double *vc = p->v_cache + ((size_t)b * p->H_kv + g) * p->max_len * d;
            const double *vn = p->v + ((size_t)b * p->H_kv + g) * d;
            orc_rope_partial(p->q + ((size_t)b * p->H_q + h) * d, 1, d, p->rot_dim, pos, p->theta,
                             qr);
            orc_rope_partial(p->k + ((size_t)b * p->H_kv + g) * d, 1, d, p->rot_dim, pos,
                             p->theta, kr);
            if (k_rot_out && h * p->H_kv % p->H_q == 0)
                memcpy(k_rot_out + ((size_t)b * p->H_kv + g) * d, kr, sizeof(double) * d);
            /* Scores of the cached tokens, then of the new one. */
            double m = -INFINITY;
            for (int64_t t = 0; t <= L; ++t) {
                const double *kt = t < L ? kc + t * d : kr;
                double s = 0.0;
                for (int i = 0; i < d; ++i) s += qr[i] * kt[i];
                score[t] = p->scale * s;
                if (score[t] > m) m = score[t];
            }
            double l = 0.0;
            for (int i = 0; i < d; ++i) acc[i] = 0.0;
            for (int64_t t = 0; t <= L; ++t) {
                const double w = exp(score[t] - m);
                const double *vt = t < L ? vc + t * d : vn;
                l += w;
                for (int i = 0; i < d; ++i) acc[i] += w * vt[i];
            }
            const double *gt = p->gate + ((size_t)b * p->H_q + h) * d;
            double *orow = o ? o + ((size_t)b * p->H_q + h) * d : NULL;
            double *yrow = y + ((size_t)b * p->H_q + h) * d;
            for (int i = 0; i < d; ++i) {
                const double oi = acc[i] / l;
                if (orow) orow[i] = oi;
                yrow[i] = oi / (1.0 + exp(-gt[i]));
            }
        }
    }
    free(qr);
    free(kr);
    free(acc);
    free(score);
    return rc;
}
