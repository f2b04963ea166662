/*
 * mk_oracle.c -- plain, slow, CPU reference of one decode step of a dense
 * Llama-architecture decoder, and of the fused SwiGLU first stage.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path links, loads or
 * calls this file: only the tests, the smoke check and the benchmark's CPU
 * baseline leg use it.  It shares no code, header, table or constant with the
 * CUDA library.
 *
 * What it computes, and where the pages fix it:
 *   - "Look Ma, No Bubbles! Designing a Low-Latency Megakernel for Llama-1B"
 *     (Hazy Research), introduction: the workload is generating one sequence
 *     with Llama-3.2-1B, i.e. the next token from the previous tokens, the
 *     weights and the KV cache.
 *   - "Deep Kernel Fusion for Transformers", Key points, "Fusion scope": the MLP
 *     is two stages, stage one = Up and Gate GEMMs + SiLU + elementwise
 *     product, stage two = the Down projection.  Its reference list (Shazeer
 *     2020, "GLU variants improve transformer") is the SwiGLU definition.
 *   - The pages do not define RMSNorm, RoPE or grouped-query attention; the
 *     plain Llama definitions are used (rotate-half RoPE pairing (i, i+d/2),
 *     eps inside the square root, no RoPE frequency scaling, no biases).
 *
 * Precision: every tensor (activations, KV cache, logits) is stored as fp32,
 * as the method statement asks.  Dot products, sums of squares and softmax
 * sums are carried in double so that the oracle's own rounding is far below
 * the GPU's; bf16/fp16 weights are widened exactly.
 *
 * Parallelism: OpenMP over output rows of each matrix-vector product and
 * nothing else; the order of every sum is the plain left-to-right order.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* ---------------------------------------------------------------------- */
/* Exact widening of 16-bit storage formats.                               */
/* ---------------------------------------------------------------------- */

/* bfloat16 is the upper half of an IEEE-754 binary32: widening is a shift. */
float orc_bf16_to_f32(uint16_t h) {
    uint32_t u = (uint32_t)h << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return f;
}

/* IEEE-754 binary16 -> binary32 via the compiler's _Float16 type. */
float orc_f16_to_f32(uint16_t h) {
    _Float16 v;
    memcpy(&v, &h, sizeof v);
    return (float)v;
}

/* ---------------------------------------------------------------------- */
/* Building blocks.                                                        */
/* ---------------------------------------------------------------------- */

/* y[n] = sum_k W[n][k] * x[k]; W is bf16, row-major [N][K] (the nn.Linear
 * [out, in] layout). */
void orc_gemv_bf16(const uint16_t *W, const float *x, float *y, int64_t N, int64_t K) {
#pragma omp parallel for schedule(static)
    for (int64_t n = 0; n < N; ++n) {
        const uint16_t *w = W + n * K;
        double s = 0.0;
        for (int64_t k = 0; k < K; ++k) s += (double)orc_bf16_to_f32(w[k]) * (double)x[k];
        y[n] = (float)s;
    }
}

/* RMSNorm: out = x / sqrt(mean(x^2) + eps) * g, g stored bf16. */
void orc_rmsnorm(const float *x, const uint16_t *g, float *out, int64_t n, float eps) {
    double ss = 0.0;
    for (int64_t i = 0; i < n; ++i) ss += (double)x[i] * (double)x[i];
    double r = 1.0 / sqrt(ss / (double)n + (double)eps);
    for (int64_t i = 0; i < n; ++i) out[i] = (float)((double)x[i] * r * (double)orc_bf16_to_f32(g[i]));
}

/* Rotary position embedding, rotate-half pairing: element i is rotated with
 * element i + d/2 by the angle pos * theta^(-2i/d), i in [0, d/2). */
void orc_rope(float *v, int d, int64_t pos, double theta) {
    int h = d / 2;
    for (int i = 0; i < h; ++i) {
        double ang = (double)pos * pow(theta, -2.0 * (double)i / (double)d);
        double c = cos(ang), s = sin(ang);
        double a = v[i], b = v[i + h];
        v[i] = (float)(a * c - b * s);
        v[i + h] = (float)(b * c + a * s);
    }
}

/* SiLU(z) = z * sigmoid(z) = z / (1 + e^-z). */
double orc_silu(double z) { return z / (1.0 + exp(-z)); }

/* Softmax attention of one query over n key/value rows.  K and V rows are d
 * floats apart by `stride` floats.  scores s_j = q.k_j / sqrt(d);
 * o = sum_j softmax(s)_j v_j. */
void orc_attend(const float *q, const float *K, const float *V, int64_t stride, int64_t n, int d,
                float *o) {
    double *s = (double *)malloc(sizeof(double) * (size_t)(n > 0 ? n : 1));
    double m = -INFINITY;
    for (int64_t j = 0; j < n; ++j) {
        double dot = 0.0;
        for (int e = 0; e < d; ++e) dot += (double)q[e] * (double)K[j * stride + e];
        s[j] = dot / sqrt((double)d);
        if (s[j] > m) m = s[j];
    }
    double l = 0.0;
    for (int64_t j = 0; j < n; ++j) {
        s[j] = exp(s[j] - m);
        l += s[j];
    }
    for (int e = 0; e < d; ++e) {
        double acc = 0.0;
        for (int64_t j = 0; j < n; ++j) acc += s[j] * (double)V[j * stride + e];
        o[e] = (float)(acc / l);
    }
    free(s);
}

/* Index of the largest value, the lowest index on ties. */
int64_t orc_argmax(const float *v, int64_t n) {
    int64_t best = 0;
    for (int64_t i = 1; i < n; ++i)
        if (v[i] > v[best]) best = i;
    return best;
}

/* ---------------------------------------------------------------------- */
/* The decoder.                                                            */
/* ---------------------------------------------------------------------- */

typedef struct {
    int n_layers, hidden, n_heads, n_kv_heads, head_dim, intermediate, vocab;
    float rms_eps, rope_theta;
    int tied, qk_norm;
    int batch, max_seq;
} orc_config;

/* Host pointers to bf16 weights, nn.Linear layout [out, in].  Per-layer
 * entries are arrays of n_layers pointers.  q_norm/k_norm are read only when
 * qk_norm is set; lm_head is ignored when tied (the embedding is the head). */
typedef struct {
    const uint16_t *embed;      /* [V, H] */
    const uint16_t *final_norm; /* [H] */
    const uint16_t *lm_head;    /* [V, H] */
    const uint16_t *const *attn_norm; /* [H] */
    const uint16_t *const *wq;  /* [nq*d, H] */
    const uint16_t *const *wk;  /* [nkv*d, H] */
    const uint16_t *const *wv;  /* [nkv*d, H] */
    const uint16_t *const *wo;  /* [H, nq*d] */
    const uint16_t *const *q_norm; /* [d] */
    const uint16_t *const *k_norm; /* [d] */
    const uint16_t *const *mlp_norm; /* [H] */
    const uint16_t *const *wg;  /* [I, H] */
    const uint16_t *const *wu;  /* [I, H] */
    const uint16_t *const *wd;  /* [H, I] */
} orc_weights;

/* KV cache layout, fp32: [layer][seq][kv_head][position][head_dim]. */
static inline int64_t kv_index(const orc_config *c, int l, int b, int g, int64_t p) {
    return ((((int64_t)l * c->batch + b) * c->n_kv_heads + g) * c->max_seq + p) * c->head_dim;
}

/* One decode step for every sequence b: the token tok[b] sits at position
 * pos[b]; its K and V rows are written to the cache at that position, it
 * attends to positions 0..pos[b], and pos[b] is advanced.  logits [B][V]
 * (may be NULL) and next [B] (may be NULL) receive the output.
 * Returns 0, or -1 for a bad argument (token or position out of range). */
int orc_decode_step(const orc_config *c, const orc_weights *w, float *kc, float *vc, int32_t *pos,
                    const int32_t *tok, float *logits, int32_t *next) {
    const int H = c->hidden, nq = c->n_heads, nkv = c->n_kv_heads, d = c->head_dim;
    const int I = c->intermediate, V = c->vocab, G = nq / nkv;
    for (int b = 0; b < c->batch; ++b) {
        if (tok[b] < 0 || tok[b] >= V || pos[b] < 0 || pos[b] >= c->max_seq) return -1;
    }
    float *x = (float *)malloc(sizeof(float) * H);
    float *h = (float *)malloc(sizeof(float) * H);
    float *q = (float *)malloc(sizeof(float) * nq * d);
    float *k = (float *)malloc(sizeof(float) * nkv * d);
    float *v = (float *)malloc(sizeof(float) * nkv * d);
    float *o = (float *)malloc(sizeof(float) * nq * d);
    float *t = (float *)malloc(sizeof(float) * (I > H ? I : H));
    float *gt = (float *)malloc(sizeof(float) * I);
    float *up = (float *)malloc(sizeof(float) * I);
    float *lg = (float *)malloc(sizeof(float) * V);
    const uint16_t *head = c->tied ? w->embed : w->lm_head;

    for (int b = 0; b < c->batch; ++b) {
        const int64_t p = pos[b];
        for (int i = 0; i < H; ++i) x[i] = orc_bf16_to_f32(w->embed[(int64_t)tok[b] * H + i]);
        for (int l = 0; l < c->n_layers; ++l) {
            /* attention block */
            orc_rmsnorm(x, w->attn_norm[l], h, H, c->rms_eps);
            orc_gemv_bf16(w->wq[l], h, q, (int64_t)nq * d, H);
            orc_gemv_bf16(w->wk[l], h, k, (int64_t)nkv * d, H);
            orc_gemv_bf16(w->wv[l], h, v, (int64_t)nkv * d, H);
            if (c->qk_norm) {
                for (int hh = 0; hh < nq; ++hh) orc_rmsnorm(q + hh * d, w->q_norm[l], q + hh * d, d, c->rms_eps);
                for (int g = 0; g < nkv; ++g) orc_rmsnorm(k + g * d, w->k_norm[l], k + g * d, d, c->rms_eps);
            }
            for (int hh = 0; hh < nq; ++hh) orc_rope(q + hh * d, d, p, c->rope_theta);
            for (int g = 0; g < nkv; ++g) orc_rope(k + g * d, d, p, c->rope_theta);
            for (int g = 0; g < nkv; ++g) {
                memcpy(kc + kv_index(c, l, b, g, p), k + g * d, sizeof(float) * d);
                memcpy(vc + kv_index(c, l, b, g, p), v + g * d, sizeof(float) * d);
            }
            for (int hh = 0; hh < nq; ++hh) {
                int g = hh / G; /* query head hh reads KV head floor(hh / (nq/nkv)) */
                orc_attend(q + hh * d, kc + kv_index(c, l, b, g, 0), vc + kv_index(c, l, b, g, 0), d, p + 1,
                           d, o + hh * d);
            }
            orc_gemv_bf16(w->wo[l], o, t, H, (int64_t)nq * d);
            for (int i = 0; i < H; ++i) x[i] += t[i];
            /* MLP block: stage one (gate, up, SiLU, product), stage two (down) */
            orc_rmsnorm(x, w->mlp_norm[l], h, H, c->rms_eps);
            orc_gemv_bf16(w->wg[l], h, gt, I, H);
            orc_gemv_bf16(w->wu[l], h, up, I, H);
            for (int i = 0; i < I; ++i) t[i] = (float)(orc_silu((double)gt[i]) * (double)up[i]);
            orc_gemv_bf16(w->wd[l], t, gt, H, I);
            for (int i = 0; i < H; ++i) x[i] += gt[i];
        }
        orc_rmsnorm(x, w->final_norm, h, H, c->rms_eps);
        orc_gemv_bf16(head, h, lg, V, H);
        if (logits) memcpy(logits + (int64_t)b * V, lg, sizeof(float) * V);
        if (next) next[b] = (int32_t)orc_argmax(lg, V);
        pos[b] += 1;
    }
    free(x); free(h); free(q); free(k); free(v); free(o); free(t); free(gt); free(up); free(lg);
    return 0;
}

/* Full causal recompute for ONE sequence of T tokens, computed layer by layer
 * over all positions at once (no KV cache is kept between calls).  Writes the
 * logits [V] of the last position.  Only batch==1 semantics; c->batch and
 * c->max_seq are not used.  Used to check the incremental decode against. */
int orc_forward_full(const orc_config *c, const orc_weights *w, const int32_t *tokens, int64_t T,
                     float *logits_last) {
    const int H = c->hidden, nq = c->n_heads, nkv = c->n_kv_heads, d = c->head_dim;
    const int I = c->intermediate, V = c->vocab, G = nq / nkv;
    if (T <= 0) return -1;
    for (int64_t s = 0; s < T; ++s)
        if (tokens[s] < 0 || tokens[s] >= V) return -1;
    float *X = (float *)malloc(sizeof(float) * T * H);
    float *Q = (float *)malloc(sizeof(float) * T * nq * d);
    float *Kf = (float *)malloc(sizeof(float) * T * nkv * d);
    float *Vf = (float *)malloc(sizeof(float) * T * nkv * d);
    float *h = (float *)malloc(sizeof(float) * H);
    float *o = (float *)malloc(sizeof(float) * nq * d);
    float *t = (float *)malloc(sizeof(float) * (I > H ? I : H));
    float *gt = (float *)malloc(sizeof(float) * I);
    float *up = (float *)malloc(sizeof(float) * I);
    float *kh = (float *)malloc(sizeof(float) * T * d);
    float *vh = (float *)malloc(sizeof(float) * T * d);
    const uint16_t *head = c->tied ? w->embed : w->lm_head;
    for (int64_t s = 0; s < T; ++s)
        for (int i = 0; i < H; ++i) X[s * H + i] = orc_bf16_to_f32(w->embed[(int64_t)tokens[s] * H + i]);
    for (int l = 0; l < c->n_layers; ++l) {
        for (int64_t s = 0; s < T; ++s) {
            orc_rmsnorm(X + s * H, w->attn_norm[l], h, H, c->rms_eps);
            float *qs = Q + s * nq * d, *ks = Kf + s * nkv * d, *vs = Vf + s * nkv * d;
            orc_gemv_bf16(w->wq[l], h, qs, (int64_t)nq * d, H);
            orc_gemv_bf16(w->wk[l], h, ks, (int64_t)nkv * d, H);
            orc_gemv_bf16(w->wv[l], h, vs, (int64_t)nkv * d, H);
            if (c->qk_norm) {
                for (int hh = 0; hh < nq; ++hh) orc_rmsnorm(qs + hh * d, w->q_norm[l], qs + hh * d, d, c->rms_eps);
                for (int g = 0; g < nkv; ++g) orc_rmsnorm(ks + g * d, w->k_norm[l], ks + g * d, d, c->rms_eps);
            }
            for (int hh = 0; hh < nq; ++hh) orc_rope(qs + hh * d, d, s, c->rope_theta);
            for (int g = 0; g < nkv; ++g) orc_rope(ks + g * d, d, s, c->rope_theta);
        }
        for (int64_t s = 0; s < T; ++s) {
            for (int hh = 0; hh < nq; ++hh) {
                int g = hh / G;
                for (int64_t j = 0; j <= s; ++j) {
                    memcpy(kh + j * d, Kf + j * nkv * d + g * d, sizeof(float) * d);
                    memcpy(vh + j * d, Vf + j * nkv * d + g * d, sizeof(float) * d);
                }
                orc_attend(Q + s * nq * d + hh * d, kh, vh, d, s + 1, d, o + hh * d);
            }
            orc_gemv_bf16(w->wo[l], o, t, H, (int64_t)nq * d);
            for (int i = 0; i < H; ++i) X[s * H + i] += t[i];
        }
        for (int64_t s = 0; s < T; ++s) {
            orc_rmsnorm(X + s * H, w->mlp_norm[l], h, H, c->rms_eps);
            orc_gemv_bf16(w->wg[l], h, gt, I, H);
            orc_gemv_bf16(w->wu[l], h, up, I, H);
            for (int i = 0; i < I; ++i) t[i] = (float)(orc_silu((double)gt[i]) * (double)up[i]);
            orc_gemv_bf16(w->wd[l], t, gt, H, I);
            for (int i = 0; i < H; ++i) X[s * H + i] += gt[i];
        }
    }
    orc_rmsnorm(X + (T - 1) * H, w->final_norm, h, H, c->rms_eps);
    orc_gemv_bf16(head, h, logits_last, V, H);
    free(X); free(Q); free(Kf); free(Vf); free(h); free(o); free(t); free(gt); free(up); free(kh); free(vh);
    return 0;
}

/* ---------------------------------------------------------------------- */
/* Fused SwiGLU first stage ("Deep Kernel Fusion for Transformers", Key    */
/* points, "Fusion scope"): out[b][n] = SiLU(sum_k x[b][k] Wg[k][n]) *     */
/* sum_k x[b][k] Wu[k][n].  x [B][K], Wg/Wu [K][N] (K-major), all fp16;    */
/* out fp32 [B][N].                                                        */
/* ---------------------------------------------------------------------- */
void orc_swiglu_stage1_f16(const uint16_t *x, const uint16_t *wg, const uint16_t *wu, float *out, int64_t B,
                           int64_t K, int64_t N) {
    for (int64_t b = 0; b < B; ++b) {
#pragma omp parallel
        {
            double *sg = NULL, *su = NULL;
            int64_t cap = 0;
#pragma omp for schedule(static)
            for (int64_t n0 = 0; n0 < N; n0 += 256) {
                int64_t n1 = n0 + 256 < N ? n0 + 256 : N;
                if (cap < n1 - n0) {
                    free(sg); free(su);
                    cap = n1 - n0;
                    sg = (double *)malloc(sizeof(double) * cap);
                    su = (double *)malloc(sizeof(double) * cap);
                }
                for (int64_t n = n0; n < n1; ++n) sg[n - n0] = su[n - n0] = 0.0;
                for (int64_t k = 0; k < K; ++k) {
                    double xv = orc_f16_to_f32(x[b * K + k]);
                    const uint16_t *rg = wg + k * N, *ru = wu + k * N;
                    for (int64_t n = n0; n < n1; ++n) {
                        sg[n - n0] += xv * (double)orc_f16_to_f32(rg[n]);
                        su[n - n0] += xv * (double)orc_f16_to_f32(ru[n]);
                    }
                }
                for (int64_t n = n0; n < n1; ++n) out[b * N + n] = (float)(orc_silu(sg[n - n0]) * su[n - n0]);
            }
            free(sg); free(su);
        }
    }
}

/* Thread count of later calls (n < 1: all processors); the benchmark times
 * the oracle on one core beside the all-core figure.  No effect on results:
 * only the output rows of a matrix-vector product are divided among threads. */
void orc_set_num_threads(int n) {
#ifdef _OPENMP
    omp_set_num_threads(n > 0 ? n : omp_get_num_procs());
#else
    (void)n;
#endif
}

/* Number of OpenMP threads the oracle uses (reported with its timings). */
int orc_num_threads(void) {
    int n = 1;
#ifdef _OPENMP
#pragma omp parallel
    {
#pragma omp single
        n = omp_get_num_threads();
    }
#endif
    return n;
}
