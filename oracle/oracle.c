/*
 * CPU oracle for one decode iteration of a Qwen3-style decoder-only transformer.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the bench's CPU
 * baseline leg load this file's library.  It shares no code, header, table or
 * helper with the CUDA path.
 *
 * What it follows:
 *  - "Mirage Persistent Kernel: Fusing Multi-GPU LLM Inference into One Kernel
 *    Launch", section "How MPK Works": `step` is an integer array of decode
 *    positions, advanced by one after every decoding iteration, and
 *    tokens[num_requests, seq_length] holds the prompts and the generated tokens.
 *  - Same page, section "The API", and "Mirage Persistent Kernel kompiliert
 *    LLM-Inferenz in einen Persistent Kernel", section "Grenzen der
 *    README-Aussagen": the fused rmsnorm_linear operation (an RMSNorm feeding a
 *    linear layer).
 *  - MPK blog excerpt (gokawiil.com article 13250), Figure 1: greedy decoding,
 *    no speculative decoding.
 * The layer arithmetic itself is the public Qwen3 decoder definition (the pages
 * name Qwen3-8B as the demo model but do not restate it), written out directly:
 * RMSNorm, Q/K/V projections, per-head QK-RMSNorm, rotate-half RoPE, causal
 * grouped-query attention with softmax, output projection with residual,
 * RMSNorm, SwiGLU MLP with residual, final RMSNorm, LM head, argmax.
 *
 * Arithmetic: double throughout.  Weights and the KV cache are bf16 (the
 * stored state).  ORC_ROUND_NONE, the plain reading, keeps every activation in
 * double.  ORC_ROUND_BF16 models a deployment that also stores activations in
 * bf16: the inputs of every projection (the normed hidden state, the attention
 * output, the SiLU*up product and the final normed state) are rounded to bf16.
 * The greedy choice is taken on the logits rounded to fp32, lowest index on
 * ties.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ORC_ROUND_NONE 0
#define ORC_ROUND_BF16 1

/* ---------------------------------------------------------------- numbers */

double orc_bf16_to_f64(uint16_t b) {
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, 4);
    return (double)f;
}

/* Round a double to the nearest bf16 value (ties to even), returned as double.
 * bf16 keeps 8 significant bits with fp32's exponent range. */
double orc_round_bf16(double x) {
    if (x == 0.0 || isnan(x) || isinf(x)) return x;
    const double min_normal = ldexp(1.0, -126);
    if (fabs(x) < min_normal) {
        /* bf16 subnormals are multiples of 2^-133 */
        return ldexp(nearbyint(ldexp(x, 133)), -133);
    }
    int e;
    double m = frexp(x, &e); /* x = m * 2^e, 0.5 <= |m| < 1 */
    double q = nearbyint(ldexp(m, 8));
    double r = ldexp(q, e - 8);
    const double max_bf16 = ldexp(255.0, 120); /* (2 - 2^-7) * 2^127 */
    if (fabs(r) > max_bf16) return x > 0 ? INFINITY : -INFINITY;
    return r;
}

uint16_t orc_f64_to_bf16_bits(double x) {
    float f = (float)orc_round_bf16(x); /* exact: the value is a bf16 */
    uint32_t u;
    memcpy(&u, &f, 4);
    return (uint16_t)(u >> 16);
}

static void round_vec(double *v, int64_t n, int mode) {
    if (mode != ORC_ROUND_BF16) return;
    for (int64_t i = 0; i < n; i++) v[i] = orc_round_bf16(v[i]);
}

/* ---------------------------------------------------------------- building blocks */

/* RMSNorm: y_i = x_i / sqrt(mean_j x_j^2 + eps) * w_i  (w is bf16). */
void orc_rmsnorm(const double *x, const uint16_t *w, int64_t n, double eps, double *y) {
    double ss = 0.0;
    for (int64_t i = 0; i < n; i++) ss += x[i] * x[i];
    double r = 1.0 / sqrt(ss / (double)n + eps);
    for (int64_t i = 0; i < n; i++) y[i] = x[i] * r * orc_bf16_to_f64(w[i]);
}

/* y = W x with W bf16 [N, K] row-major (a linear layer stored [out, in]). */
void orc_gemv(const uint16_t *W, int64_t N, int64_t K, const double *x, double *y) {
#pragma omp parallel for schedule(static)
    for (int64_t n = 0; n < N; n++) {
        const uint16_t *row = W + n * K;
        double acc = 0.0;
        for (int64_t k = 0; k < K; k++) acc += orc_bf16_to_f64(row[k]) * x[k];
        y[n] = acc;
    }
}

/* Rotate-half rotary embedding at absolute position pos: for i < d/2 the pair
 * (v_i, v_{i+d/2}) turns by angle pos * theta^(-2i/d). */
void orc_rope(double *v, int d, int64_t pos, double theta) {
    int half = d / 2;
    for (int i = 0; i < half; i++) {
        double ang = (double)pos * pow(theta, -2.0 * (double)i / (double)d);
        double c = cos(ang), s = sin(ang);
        double a = v[i], b = v[i + half];
        v[i] = a * c - b * s;
        v[i + half] = b * c + a * s;
    }
}

/* SiLU(z) = z * sigmoid(z). */
double orc_silu(double z) { return z / (1.0 + exp(-z)); }

/* One query head against npos cached positions of one kv head:
 * p = softmax_t(q . K_t / sqrt(d)),  o = sum_t p_t V_t.  K, V bf16 [npos, d]. */
void orc_attend(const double *q, const uint16_t *K, const uint16_t *V, int64_t npos, int d,
                double *o) {
    double *sc = (double *)malloc(sizeof(double) * (size_t)(npos > 0 ? npos : 1));
    double scale = 1.0 / sqrt((double)d);
    double mx = -INFINITY;
    for (int64_t t = 0; t < npos; t++) {
        double acc = 0.0;
        for (int i = 0; i < d; i++) acc += q[i] * orc_bf16_to_f64(K[t * d + i]);
        sc[t] = acc * scale;
        if (sc[t] > mx) mx = sc[t];
    }
    double z = 0.0;
    for (int64_t t = 0; t < npos; t++) {
        sc[t] = exp(sc[t] - mx);
        z += sc[t];
    }
    for (int i = 0; i < d; i++) o[i] = 0.0;
    for (int64_t t = 0; t < npos; t++) {
        double p = sc[t] / z;
        for (int i = 0; i < d; i++) o[i] += p * orc_bf16_to_f64(V[t * d + i]);
    }
    free(sc);
}

/* Index of the largest fp32-rounded value, lowest index on ties. */
int64_t orc_argmax_f32(const double *z, int64_t n) {
    int64_t best = 0;
    float bv = (float)z[0];
    for (int64_t i = 1; i < n; i++) {
        float v = (float)z[i];
        if (v > bv) {
            bv = v;
            best = i;
        }
    }
    return best;
}

/* ---------------------------------------------------------------- the decoder */

typedef struct {
    int L, H, Hq, Hkv, d, I, V;
    double eps, theta;
    const uint16_t *embed;      /* [V, H] */
    const uint16_t *final_norm; /* [H] */
    const uint16_t *lm_head;    /* [V, H]; the embedding itself when tied */
    const uint16_t *const *in_norm;   /* L x [H] */
    const uint16_t *const *wq;        /* L x [Hq*d, H] */
    const uint16_t *const *wk;        /* L x [Hkv*d, H] */
    const uint16_t *const *wv;        /* L x [Hkv*d, H] */
    const uint16_t *const *q_norm;    /* L x [d] */
    const uint16_t *const *k_norm;    /* L x [d] */
    const uint16_t *const *wo;        /* L x [H, Hq*d] */
    const uint16_t *const *post_norm; /* L x [H] */
    const uint16_t *const *wg;        /* L x [I, H] */
    const uint16_t *const *wu;        /* L x [I, H] */
    const uint16_t *const *wd;        /* L x [H, I] */
} orc_model;

/* KV cache element offset of [l][r][j][s][0] in a [L][R][Hkv][S][d] array. */
static int64_t kv_off(const orc_model *m, int R, int64_t S, int l, int r, int j, int64_t s) {
    return ((((int64_t)l * R + r) * m->Hkv + j) * S + s) * m->d;
}

/* Full forward pass of one token of request r at position s.  Appends this
 * position's K/V to the cache, returns the logits in z[V]. */
static void forward_one(const orc_model *m, int R, int64_t S, uint16_t *kc, uint16_t *vc, int r,
                        int64_t s, int64_t tok, int mode, double *z, double *hidden) {
    const int H = m->H, d = m->d, Hq = m->Hq, Hkv = m->Hkv, I = m->I;
    const int qd = Hq * d, kvd = Hkv * d;
    double *x = calloc((size_t)H, sizeof(double));
    double *h = calloc((size_t)(H > I ? H : I), sizeof(double));
    double *q = calloc((size_t)qd, sizeof(double));
    double *k = calloc((size_t)kvd, sizeof(double));
    double *v = calloc((size_t)kvd, sizeof(double));
    double *o = calloc((size_t)qd, sizeof(double));
    double *t1 = calloc((size_t)(H > I ? H : I), sizeof(double));
    double *g = calloc((size_t)I, sizeof(double));
    double *u = calloc((size_t)I, sizeof(double));

    for (int i = 0; i < H; i++) x[i] = orc_bf16_to_f64(m->embed[tok * H + i]);
    if (hidden) memcpy(hidden + ((int64_t)0 * R + r) * H, x, sizeof(double) * H);

    for (int l = 0; l < m->L; l++) {
        /* attention block */
        orc_rmsnorm(x, m->in_norm[l], H, m->eps, h);
        round_vec(h, H, mode);
        orc_gemv(m->wq[l], qd, H, h, q);
        orc_gemv(m->wk[l], kvd, H, h, k);
        orc_gemv(m->wv[l], kvd, H, h, v);
        for (int j = 0; j < Hkv; j++) {
            double kn[512];
            orc_rmsnorm(k + j * d, m->k_norm[l], d, m->eps, kn);
            orc_rope(kn, d, s, m->theta);
            int64_t off = kv_off(m, R, S, l, r, j, s);
            for (int i = 0; i < d; i++) {
                kc[off + i] = orc_f64_to_bf16_bits(kn[i]);
                vc[off + i] = orc_f64_to_bf16_bits(v[j * d + i]);
            }
        }
#pragma omp parallel for schedule(static)
        for (int hh = 0; hh < Hq; hh++) {
            double qn[512];
            orc_rmsnorm(q + hh * d, m->q_norm[l], d, m->eps, qn);
            orc_rope(qn, d, s, m->theta);
            int j = (int)(((int64_t)hh * Hkv) / Hq);
            int64_t base = kv_off(m, R, S, l, r, j, 0);
            orc_attend(qn, kc + base, vc + base, s + 1, d, o + hh * d);
        }
        round_vec(o, qd, mode);
        orc_gemv(m->wo[l], H, qd, o, t1);
        for (int i = 0; i < H; i++) x[i] += t1[i];

        /* MLP block */
        orc_rmsnorm(x, m->post_norm[l], H, m->eps, h);
        round_vec(h, H, mode);
        orc_gemv(m->wg[l], I, H, h, g);
        orc_gemv(m->wu[l], I, H, h, u);
        for (int i = 0; i < I; i++) t1[i] = orc_silu(g[i]) * u[i];
        round_vec(t1, I, mode);
        orc_gemv(m->wd[l], H, I, t1, h);
        for (int i = 0; i < H; i++) x[i] += h[i];
        if (hidden) memcpy(hidden + ((int64_t)(l + 1) * R + r) * H, x, sizeof(double) * H);
    }
    orc_rmsnorm(x, m->final_norm, H, m->eps, h);
    round_vec(h, H, mode);
    orc_gemv(m->lm_head, m->V, H, h, z);

    free(x); free(h); free(q); free(k); free(v); free(o); free(t1); free(g); free(u);
}

/*
 * One decoding iteration over all requests, with the meta-tensor semantics of
 * "How MPK Works": a request r is active while step[r] < step_end[r] and
 * step[r] + 1 < S.  An active request consumes tokens[r, s] at s = step[r],
 * appends K/V at s, predicts position s+1 by greedy argmax, writes the
 * prediction into tokens[r, s+1] only if that slot holds -1 (pre-filled slots
 * are prompt or teacher-forced tokens), records it in pred[r, s+1] and advances
 * step[r].  step_end may be NULL (run to the end of the row).
 * logits [R, V] and hidden [(L+1), R, H] are optional captures (NULL = off);
 * inactive requests leave them untouched.  Returns the number of requests
 * advanced.
 */
int orc_decode_iteration(const orc_model *m, int R, int64_t S, uint16_t *kcache, uint16_t *vcache,
                         int32_t *step, int64_t *tokens, const int32_t *step_end, int round_mode,
                         double *logits, double *hidden, int64_t *pred) {
    int advanced = 0;
    double *z = malloc(sizeof(double) * (size_t)m->V);
    for (int r = 0; r < R; r++) {
        int64_t s = step[r];
        int64_t end = step_end ? step_end[r] : S - 1;
        if (end > S - 1) end = S - 1;
        if (s < 0 || s >= end) continue;
        int64_t tok = tokens[(int64_t)r * S + s];
        if (tok < 0 || tok >= m->V) continue;
        forward_one(m, R, S, kcache, vcache, r, s, tok, round_mode, z, hidden);
        if (logits) memcpy(logits + (int64_t)r * m->V, z, sizeof(double) * (size_t)m->V);
        int64_t nxt = orc_argmax_f32(z, m->V);
        if (tokens[(int64_t)r * S + s + 1] == -1) tokens[(int64_t)r * S + s + 1] = nxt;
        if (pred) pred[(int64_t)r * S + s + 1] = nxt;
        step[r] = (int32_t)(s + 1);
        advanced++;
    }
    free(z);
    return advanced;
}

int orc_num_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

void orc_set_num_threads(int n) {
#ifdef _OPENMP
    if (n > 0) omp_set_num_threads(n);
#else
    (void)n;
#endif
}
