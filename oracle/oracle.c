/*
 * oracle.c -- fp64 CPU reference for batch-1 decode (see oracle.h).
 *
 * TEST INFRASTRUCTURE ONLY: the product path never loads this file.
 *
 * Plain and slow on purpose: each function is the textbook definition written
 * out, with OpenMP only across independent output rows / heads.  Sources:
 *   - decoder forward (RMSNorm -> QKV -> RoPE -> cache append -> GQA attention
 *     -> O-proj + residual -> RMSNorm -> SiLU-gated FFN -> down + residual,
 *     then final norm -> LM head -> greedy argmax): the Llama family named in
 *     the epic-kernel README, "3B model support";
 *   - MoE FFN (router scores -> top-k experts -> softmax over the selected
 *     scores -> weighted sum of expert FFNs): epic-kernel README, "Mixtral
 *     8x7B MoE for batch-1 inference";
 *   - RoPE in the rotate-half pairing (i, i + d/2) with angle pos *
 *     theta^(-2i/d), no frequency scaling (the plain reading; the pages print
 *     no formula);
 *   - the KV cache is bf16 and the appended entry is rounded to bf16 before it
 *     is attended to (the cache format is part of the workload).
 */
#include "oracle.h"

#include <math.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

int orc_num_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* bf16 is the top half of an IEEE binary32; widening is exact. */
double orc_bf16_to_double(uint16_t b) {
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, 4);
    return (double)f;
}

/* double -> bf16 with one rounding (nearest, ties to even) at bf16's 8-bit
 * significand: round the binary64 significand at bit 45, then the result is
 * exactly representable in binary32 (for |v| in binary32's normal range). */
uint16_t orc_bf16_from_double(double v) {
    if (isnan(v)) return 0x7FC0;
    uint64_t u;
    memcpy(&u, &v, 8);
    const uint64_t lsb = (u >> 45) & 1u;
    u += ((uint64_t)1 << 44) - 1 + lsb;
    u &= ~(((uint64_t)1 << 45) - 1);
    double r;
    memcpy(&r, &u, 8);
    float f = (float)r;
    uint32_t fu;
    memcpy(&fu, &f, 4);
    return (uint16_t)(fu >> 16);
}

#define BF(x) orc_bf16_to_double(x)

/* RMSNorm: out_i = x_i / sqrt(mean(x^2) + eps) * w_i. */
void orc_rmsnorm(const double *x, const uint16_t *w, int n, double eps, double *out) {
    double ss = 0.0;
    for (int i = 0; i < n; ++i) ss += x[i] * x[i];
    const double inv = 1.0 / sqrt(ss / (double)n + eps);
    for (int i = 0; i < n; ++i) out[i] = x[i] * inv * BF(w[i]);
}

/* y = W x, W bf16 [rows, cols] row-major (the nn.Linear [out, in] layout). */
void orc_gemv(const uint16_t *W, int rows, int cols, const double *x, double *y) {
#pragma omp parallel for schedule(static)
    for (int r = 0; r < rows; ++r) {
        const uint16_t *row = W + (size_t)r * (size_t)cols;
        double acc = 0.0;
        for (int c = 0; c < cols; ++c) acc += BF(row[c]) * x[c];
        y[r] = acc;
    }
}

/* Rotary embedding, rotate-half pairing, in place on n_heads heads of
 * head_dim: for i < d/2 with a = pos * theta^(-2i/d),
 *   (v_i, v_{i+d/2}) <- (v_i cos a - v_{i+d/2} sin a, v_{i+d/2} cos a + v_i sin a). */
void orc_rope(double *v, int n_heads, int head_dim, int pos, double theta) {
    const int half = head_dim / 2;
    for (int i = 0; i < half; ++i) {
        const double freq = pow(theta, -2.0 * (double)i / (double)head_dim);
        const double a = (double)pos * freq;
        const double c = cos(a), s = sin(a);
        for (int h = 0; h < n_heads; ++h) {
            double *x = v + (size_t)h * head_dim;
            const double x1 = x[i], x2 = x[i + half];
            x[i] = x1 * c - x2 * s;
            x[i + half] = x2 * c + x1 * s;
        }
    }
}

/* p = softmax(s), shifted by max(s) for range. */
void orc_softmax(const double *s, int n, double *p) {
    double m = -INFINITY;
    for (int j = 0; j < n; ++j) m = s[j] > m ? s[j] : m;
    double z = 0.0;
    for (int j = 0; j < n; ++j) {
        p[j] = exp(s[j] - m);
        z += p[j];
    }
    for (int j = 0; j < n; ++j) p[j] /= z;
}

/* One query head over n cached positions: out = softmax(q K^T / sqrt(d)) V.
 * K, V: bf16 [n, head_dim]. */
void orc_attend(const double *q, const uint16_t *K, const uint16_t *V, int n, int head_dim, double *out) {
    double *s = (double *)malloc(sizeof(double) * (size_t)(n > 0 ? n : 1));
    double *p = (double *)malloc(sizeof(double) * (size_t)(n > 0 ? n : 1));
    const double scale = 1.0 / sqrt((double)head_dim);
    for (int j = 0; j < n; ++j) {
        double acc = 0.0;
        for (int i = 0; i < head_dim; ++i) acc += q[i] * BF(K[(size_t)j * head_dim + i]);
        s[j] = acc * scale;
    }
    orc_softmax(s, n, p);
    for (int i = 0; i < head_dim; ++i) {
        double acc = 0.0;
        for (int j = 0; j < n; ++j) acc += p[j] * BF(V[(size_t)j * head_dim + i]);
        out[i] = acc;
    }
    free(s);
    free(p);
}

/* SiLU (swish): z * sigmoid(z) = z / (1 + e^{-z}). */
double orc_silu(double z) { return z / (1.0 + exp(-z)); }

/* Top-k selection by repeated argmax (lowest index wins a tie), weights =
 * softmax over the k selected scores (equal to the full softmax renormalised
 * over the selected experts). */
void orc_topk(const double *r, int n_experts, int k, int *idx, double *w) {
    int taken[64] = {0};
    for (int t = 0; t < k; ++t) {
        int best = -1;
        for (int e = 0; e < n_experts; ++e) {
            if (taken[e]) continue;
            if (best < 0 || r[e] > r[best]) best = e;
        }
        taken[best] = 1;
        idx[t] = best;
    }
    double sel[64];
    for (int t = 0; t < k; ++t) sel[t] = r[idx[t]];
    orc_softmax(sel, k, w);
}

int orc_argmax(const double *v, int n) {
    int best = 0;
    for (int i = 1; i < n; ++i)
        if (v[i] > v[best]) best = i;
    return best;
}

/* SiLU-gated FFN of one expert (or the dense FFN): Wd (silu(Wg xn) * (Wu xn)). */
static void ffn(const uint16_t *wg, const uint16_t *wu, const uint16_t *wd, int H, int F, const double *xn,
                double *out) {
    double *g = (double *)malloc(sizeof(double) * (size_t)F);
    double *u = (double *)malloc(sizeof(double) * (size_t)F);
    orc_gemv(wg, F, H, xn, g);
    orc_gemv(wu, F, H, xn, u);
    for (int i = 0; i < F; ++i) g[i] = orc_silu(g[i]) * u[i];
    orc_gemv(wd, H, F, g, out);
    free(g);
    free(u);
}

int orc_predict_experts(const orc_shape *s, const orc_weights *w, int layer, const double *x, int *idx) {
    const int H = s->hidden, E = s->n_experts, K = s->top_k;
    if (E <= 0 || K < 1 || K > E || E > 64 || layer < 0 || layer >= s->n_layers) return -1;
    double *xn = (double *)malloc(sizeof(double) * (size_t)H);
    double r[64], wt[64];
    orc_rmsnorm(x, w->attn_norm[layer], H, s->rms_eps, xn);
    orc_gemv(w->router[layer], E, H, xn, r);
    orc_topk(r, E, K, idx, wt);
    free(xn);
    return 0;
}

int orc_decode_step(const orc_shape *s, const orc_weights *w, uint16_t *kcache, uint16_t *vcache, int token,
                    int pos, double *logits, double *hidden, int *router_idx, double *router_w) {
    const int L = s->n_layers, H = s->hidden, nq = s->n_heads, nkv = s->n_kv_heads, d = s->head_dim;
    const int F = s->ffn, V = s->vocab, E = s->n_experts, K = s->top_k;
    if (token < 0 || token >= V || pos < 0 || pos >= s->max_seq || nkv <= 0 || nq % nkv != 0) return -1;
    if (E > 0 && (K < 1 || K > E || E > 64)) return -1;
    const int group = nq / nkv;

    double *x = (double *)malloc(sizeof(double) * (size_t)H);
    double *xn = (double *)malloc(sizeof(double) * (size_t)H);
    double *q = (double *)malloc(sizeof(double) * (size_t)nq * d);
    double *k = (double *)malloc(sizeof(double) * (size_t)nkv * d);
    double *v = (double *)malloc(sizeof(double) * (size_t)nkv * d);
    double *att = (double *)malloc(sizeof(double) * (size_t)nq * d);
    double *tmp = (double *)malloc(sizeof(double) * (size_t)H);
    double *acc = (double *)malloc(sizeof(double) * (size_t)H);

    /* Embedding lookup. */
    for (int i = 0; i < H; ++i) x[i] = BF(w->embed[(size_t)token * H + i]);
    if (hidden) memcpy(hidden, x, sizeof(double) * (size_t)H);

    for (int l = 0; l < L; ++l) {
        /* Attention block. */
        orc_rmsnorm(x, w->attn_norm[l], H, s->rms_eps, xn);
        orc_gemv(w->wq[l], nq * d, H, xn, q);
        orc_gemv(w->wk[l], nkv * d, H, xn, k);
        orc_gemv(w->wv[l], nkv * d, H, xn, v);
        orc_rope(q, nq, d, pos, s->rope_theta);
        orc_rope(k, nkv, d, pos, s->rope_theta);
        for (int g = 0; g < nkv; ++g) {
            const size_t base = (((size_t)l * nkv + g) * (size_t)s->max_seq + (size_t)pos) * (size_t)d;
            for (int i = 0; i < d; ++i) {
                kcache[base + i] = orc_bf16_from_double(k[(size_t)g * d + i]);
                vcache[base + i] = orc_bf16_from_double(v[(size_t)g * d + i]);
            }
        }
        /* GQA: query head h reads kv head floor(h / (nq / nkv)), positions 0..pos. */
#pragma omp parallel for schedule(static)
        for (int h = 0; h < nq; ++h) {
            const int g = h / group;
            const size_t base = ((size_t)l * nkv + g) * (size_t)s->max_seq * (size_t)d;
            orc_attend(q + (size_t)h * d, kcache + base, vcache + base, pos + 1, d, att + (size_t)h * d);
        }
        orc_gemv(w->wo[l], H, nq * d, att, tmp);
        for (int i = 0; i < H; ++i) x[i] += tmp[i];

        /* FFN block. */
        orc_rmsnorm(x, w->ffn_norm[l], H, s->rms_eps, xn);
        if (E == 0) {
            ffn(w->w_gate[l], w->w_up[l], w->w_down[l], H, F, xn, tmp);
            for (int i = 0; i < H; ++i) x[i] += tmp[i];
        } else {
            double r[64], wt[64];
            int idx[64];
            orc_gemv(w->router[l], E, H, xn, r);
            orc_topk(r, E, K, idx, wt);
            for (int i = 0; i < H; ++i) acc[i] = 0.0;
            for (int t = 0; t < K; ++t) {
                const size_t e = (size_t)l * E + idx[t];
                ffn(w->w_gate[e], w->w_up[e], w->w_down[e], H, F, xn, tmp);
                for (int i = 0; i < H; ++i) acc[i] += wt[t] * tmp[i];
            }
            for (int i = 0; i < H; ++i) x[i] += acc[i];
            if (router_idx)
                for (int t = 0; t < K; ++t) router_idx[(size_t)l * K + t] = idx[t];
            if (router_w)
                for (int t = 0; t < K; ++t) router_w[(size_t)l * K + t] = wt[t];
        }
        if (hidden) memcpy(hidden + (size_t)(l + 1) * H, x, sizeof(double) * (size_t)H);
    }

    /* Final norm, LM head, greedy choice. */
    orc_rmsnorm(x, w->final_norm, H, s->rms_eps, xn);
    orc_gemv(w->lm_head, V, H, xn, logits);
    const int next = orc_argmax(logits, V);

    free(x);
    free(xn);
    free(q);
    free(k);
    free(v);
    free(att);
    free(tmp);
    free(acc);
    return next;
}
