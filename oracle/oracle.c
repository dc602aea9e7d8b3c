/*
 * CPU ORACLE for the decode step of a dense decoder-only transformer.
 *
 * TEST INFRASTRUCTURE ONLY. Only the tests, the smoke check and the CPU-baseline leg of
 * the benchmark may load this library. The engine never calls it, and it shares no
 * code, header, table or constant generator with the engine.
 *
 * What it computes. The pages ("Kog 3000 tok/s 实时推理：内存带宽优化与请求级并发的工程权衡",
 * section 内存带宽优化的三层策略) fix only that a decode step loads all model weights and the
 * KV cache for each token; the step itself is the textbook Llama-style forward pass
 * (pre-norm RMSNorm, rotary positions, grouped-query attention, SwiGLU MLP, untied LM
 * head, greedy argmax), written out here one definition at a time:
 *
 *   x      = E[token]
 *   per layer:
 *     h    = x / sqrt(mean(x^2) + eps) * g_attn
 *     q, k, v = Wq h, Wk h, Wv h
 *     q, k rotated by position p (rotate-half pairing (i, i + D/2), angle p * theta^(-2i/D))
 *     K[p], V[p] = k, v rounded to the storage dtype (the fp16/bf16 KV cache)
 *     o_h  = sum_j softmax_j(q_h . K_j / sqrt(D)) V_j, j = 0..p, kv head g = floor(h * Hkv / Hq)
 *     x   += Wo o
 *     h    = x / sqrt(mean(x^2) + eps) * g_mlp
 *     x   += Wd (silu(Wg h) * (Wu h)),  silu(z) = z / (1 + exp(-z))
 *   logits = W_lm (x / sqrt(mean(x^2) + eps) * g_final);  token = argmax (lowest index on ties)
 *
 * The sampling variant (orc_sample, at the end) replaces the argmax by temperature / top-k
 * sampling with one counter-based uniform draw per step (splitmix64 keyed by a seed and the
 * step's position).
 *
 * Arithmetic is fp64 throughout; weights are read as exact fp16/bf16 values. The only
 * rounding besides fp64's own is the one the method defines: K and V are stored in the
 * weight dtype (rounded fp64 -> fp32 -> storage, both round-to-nearest-even).
 * Summations run in plain index order; OpenMP splits only independent output rows.
 */
#include <math.h>
#include <omp.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

typedef struct {
    int32_t n_layers, d_model, n_heads, n_kv_heads, head_dim, ffn, vocab, dtype; /* 0 fp16, 1 bf16 */
    double rms_eps, rope_theta;
} orc_config;

enum { W_ATTN_NORM, W_Q, W_K, W_V, W_O, W_MLP_NORM, W_GATE, W_UP, W_DOWN, W_PER_LAYER };

typedef struct {
    const uint16_t *tok_emb;          /* [vocab][d_model]  */
    const uint16_t *final_norm;       /* [d_model]         */
    const uint16_t *lm_head;          /* [vocab][d_model]  */
    const uint16_t *const *layers;    /* [n_layers * 9], order of the enum above */
    /* Optional FP8 weights (all NULL for the 16-bit model): E4M3 codes and per-row scales of
       every matrix (entries of the norm gains unused) and of the LM head; when q8 is set, every
       matrix-vector product uses value(code) * scale[row] instead of the 16-bit weights. */
    const uint8_t *const *q8;         /* [n_layers * 9] */
    const float *const *q8_scale;     /* [n_layers * 9] */
    const uint8_t *q8_head;
    const float *q8_head_scale;
} orc_weights;

/* ---------------------------------------------------------------- storage types */

/* Exact value of a stored fp16 / bf16 element. */
double orc_value(uint16_t bits, int32_t dtype) {
    if (dtype == 1) {
        uint32_t u = (uint32_t)bits << 16;
        float f;
        memcpy(&f, &u, 4);
        return (double)f;
    }
    int sign = bits >> 15, e = (bits >> 10) & 0x1F, m = bits & 0x3FF;
    double v;
    if (e == 0) v = ldexp((double)m, -24);                       /* subnormal */
    else if (e == 31) v = m ? NAN : INFINITY;
    else v = ldexp((double)(m | 0x400), e - 25);
    return sign ? -v : v;
}

/* fp64 -> fp32 (C cast, round to nearest even) -> storage dtype (round to nearest even). */
uint16_t orc_store(double v, int32_t dtype) {
    float f = (float)v;
    uint32_t x;
    memcpy(&x, &f, 4);
    if (dtype == 1) {
        if ((x & 0x7FFFFFFFu) > 0x7F800000u) return (uint16_t)((x >> 16) | 0x40);
        uint32_t lsb = (x >> 16) & 1u;
        return (uint16_t)((x + 0x7FFFu + lsb) >> 16);
    }
    /* binary16: take the value apart and rebuild it with exact integer rounding */
    uint16_t sign = (uint16_t)((x >> 16) & 0x8000u);
    double a = fabs((double)f);
    if (isnan(a)) return sign | 0x7E00;
    if (a >= 65520.0) return sign | 0x7C00;
    if (a == 0.0) return sign;
    int e;
    frexp(a, &e);                         /* a = fr * 2^e, fr in [0.5, 1) */
    int exp16 = e - 1;                    /* a = 1.xxx * 2^exp16 */
    if (exp16 < -14) exp16 = -14;         /* subnormal range uses the fixed 2^-24 step */
    double step = ldexp(1.0, exp16 - 10); /* spacing of binary16 values at this exponent */
    double q = a / step;                  /* exact: a has 24 bits, step is a power of two */
    double fl = floor(q), rem = q - fl;
    uint32_t qi = (uint32_t)fl;
    if (rem > 0.5 || (rem == 0.5 && (qi & 1u))) qi++;
    /* qi counts steps of 2^(exp16-10); rebuild the bit pattern */
    if (exp16 == -14 && qi < 0x400) return sign | (uint16_t)qi;   /* subnormal (or zero) */
    if (qi == 0x800) { qi = 0x400; exp16++; }                    /* rounding carried */
    if (exp16 > 15) return sign | 0x7C00;
    return sign | (uint16_t)(((exp16 + 15) << 10) | (qi & 0x3FF));
}

/* ---------------------------------------------------------------- building blocks */

static double *g_table[2];  /* exact values of all 65536 patterns, per dtype */

static const double *value_table(int32_t dtype) {
    double *t = g_table[dtype ? 1 : 0];
    if (t) return t;
#pragma omp critical(orc_table)
    {
        if (!g_table[dtype ? 1 : 0]) {
            double *nt = (double *)malloc(65536 * sizeof(double));
            for (int i = 0; i < 65536; i++) nt[i] = orc_value((uint16_t)i, dtype);
            g_table[dtype ? 1 : 0] = nt;
        }
        t = g_table[dtype ? 1 : 0];
    }
    return t;
}

/* RMSNorm: out_i = x_i / sqrt(mean(x^2) + eps) * g_i. */
void orc_rmsnorm(int32_t n, const double *x, const uint16_t *g, int32_t dtype, double eps, double *out) {
    double ss = 0.0;
    for (int i = 0; i < n; i++) ss += x[i] * x[i];
    double r = 1.0 / sqrt(ss / n + eps);
    for (int i = 0; i < n; i++) out[i] = x[i] * r * orc_value(g[i], dtype);
}

/* y = W x for W stored row-major [N][K]. */
void orc_matvec(int32_t N, int32_t K, const uint16_t *W, int32_t dtype, const double *x, double *y) {
    const double *tv = value_table(dtype);
#pragma omp parallel for schedule(static)
    for (int n = 0; n < N; n++) {
        const uint16_t *row = W + (int64_t)n * K;
        double acc = 0.0;
        for (int k = 0; k < K; k++) acc += tv[row[k]] * x[k];
        y[n] = acc;
    }
}

/* ---------------------------------------------------------------- FP8 (E4M3) weights
 *
 * E4M3 (the "fn" variant of the OCP FP8 formats): 1 sign bit, 4 exponent bits with bias 7,
 * 3 fraction bits; exponent 0 holds the subnormals m/8 * 2^-6; the all-ones exponent with
 * fraction 111 is NaN and there are no infinities, so the largest finite value is
 * 1.75 * 2^8 = 448.
 */

/* Exact value of an E4M3 code. */
double orc_e4m3_value(uint8_t b) {
    const int sign = b >> 7, e = (b >> 3) & 0xF, m = b & 7;
    double v;
    if (e == 0xF && m == 7) return NAN;
    if (e == 0) v = ldexp((double)m, -9);            /* m/8 * 2^-6 */
    else v = ldexp((double)(8 + m), e - 10);          /* (1 + m/8) * 2^(e-7) */
    return sign ? -v : v;
}

/* fp32 value -> nearest E4M3 code, ties to the even code, finite results saturated at +-448
   (a value beyond the largest finite code encodes as that code); NaN -> 0x7F. */
uint8_t orc_e4m3_encode(float f) {
    if (f != f) return 0x7F;
    const uint8_t sign = signbit(f) ? 0x80 : 0;
    double a = fabs((double)f);
    if (a >= 448.0) return sign | 0x7E;
    if (a == 0.0) return sign;
    int e;
    frexp(a, &e);                        /* a = fr * 2^e, fr in [0.5, 1) */
    int exp8 = e - 1;                    /* a = 1.xxx * 2^exp8 */
    if (exp8 < -6) exp8 = -6;            /* subnormal range: fixed step 2^-9 */
    const double step = ldexp(1.0, exp8 - 3);
    const double q = a / step;           /* exact: a has 24 bits, step a power of two */
    const double fl = floor(q), rem = q - fl;
    uint32_t qi = (uint32_t)fl;
    if (rem > 0.5 || (rem == 0.5 && (qi & 1u))) qi++;
    if (exp8 == -6 && qi < 8) return sign | (uint8_t)qi;   /* subnormal (or zero) */
    if (qi == 16) { qi = 8; exp8++; }                       /* rounding carried */
    if (exp8 > 8 || (exp8 == 8 && qi > 14)) return sign | 0x7E;
    return sign | (uint8_t)(((exp8 + 7) << 3) | (qi & 7));
}

/* Per-row quantisation of a 16-bit matrix [N][K]: scale[n] = max_k |W[n][k]| / 448 (fp32; 1 for
   an all-zero row) and q[n][k] = encode(W[n][k] / scale[n]), the quotient in fp32. */
void orc_quantize_rows(int32_t N, int32_t K, const uint16_t *W, int32_t dtype, uint8_t *q, float *scale) {
#pragma omp parallel for schedule(static)
    for (int n = 0; n < N; n++) {
        const uint16_t *row = W + (int64_t)n * K;
        float amax = 0.f;
        for (int k = 0; k < K; k++) {
            const float a = (float)fabs(orc_value(row[k], dtype));
            if (a > amax) amax = a;
        }
        const float s = amax > 0.f ? amax / 448.0f : 1.0f;
        scale[n] = s;
        for (int k = 0; k < K; k++) q[(int64_t)n * K + k] = orc_e4m3_encode((float)orc_value(row[k], dtype) / s);
    }
}

/* y = (scale * Q) x for E4M3 codes Q [N][K] with per-row scales. */
void orc_matvec_q8(int32_t N, int32_t K, const uint8_t *Q, const float *scale, const double *x, double *y) {
    double tv[256];
    for (int i = 0; i < 256; i++) tv[i] = orc_e4m3_value((uint8_t)i);
#pragma omp parallel for schedule(static)
    for (int n = 0; n < N; n++) {
        const uint8_t *row = Q + (int64_t)n * K;
        double acc = 0.0;
        for (int k = 0; k < K; k++) acc += tv[row[k]] * x[k];
        y[n] = (double)scale[n] * acc;
    }
}

/* Matrix j of layer l (an enum index above) times x: the FP8 codes when the model has them. */
static void layer_matvec(const orc_config *c, const orc_weights *w, int l, int j, int32_t N, int32_t K,
                         const double *x, double *y) {
    const int64_t i = (int64_t)l * W_PER_LAYER + j;
    if (w->q8) orc_matvec_q8(N, K, w->q8[i], w->q8_scale[i], x, y);
    else orc_matvec(N, K, w->layers[i], c->dtype, x, y);
}

static void head_matvec(const orc_config *c, const orc_weights *w, const double *x, double *y) {
    if (w->q8) orc_matvec_q8(c->vocab, c->d_model, w->q8_head, w->q8_head_scale, x, y);
    else orc_matvec(c->vocab, c->d_model, w->lm_head, c->dtype, x, y);
}

/* Rotary position embedding, rotate-half form: for i < D/2 the pair (v_i, v_{i+D/2})
   turns by the angle pos * theta^(-2i/D). */
void orc_rope(int32_t D, int32_t pos, double theta, double *v) {
    int half = D / 2;
    for (int i = 0; i < half; i++) {
        double ang = (double)pos * pow(theta, -2.0 * i / D);
        double c = cos(ang), s = sin(ang);
        double a = v[i], b = v[i + half];
        v[i] = a * c - b * s;
        v[i + half] = b * c + a * s;
    }
}

/* Single-query attention over n stored keys/values (rows of D, row stride D):
   out = sum_j softmax_j(q . K_j / sqrt(D)) V_j, softmax by max subtraction. */
void orc_attention(int32_t D, int32_t n, const double *q, const uint16_t *K, const uint16_t *V,
                   int32_t dtype, double *out) {
    double *s = (double *)malloc(sizeof(double) * (n > 0 ? n : 1));
    double scale = 1.0 / sqrt((double)D), m = -INFINITY;
    for (int j = 0; j < n; j++) {
        double acc = 0.0;
        for (int i = 0; i < D; i++) acc += q[i] * orc_value(K[(int64_t)j * D + i], dtype);
        s[j] = acc * scale;
        if (s[j] > m) m = s[j];
    }
    double sum = 0.0;
    for (int j = 0; j < n; j++) { s[j] = exp(s[j] - m); sum += s[j]; }
    for (int i = 0; i < D; i++) out[i] = 0.0;
    for (int j = 0; j < n; j++)
        for (int i = 0; i < D; i++) out[i] += (s[j] / sum) * orc_value(V[(int64_t)j * D + i], dtype);
    free(s);
}

double orc_silu(double z) { return z / (1.0 + exp(-z)); }

/* Index of the largest value; the lowest index wins ties. */
int32_t orc_argmax(int32_t n, const double *v) {
    int best = 0;
    for (int i = 1; i < n; i++)
        if (v[i] > v[best]) best = i;
    return best;
}

/* ---------------------------------------------------------------- the decode step */

static int64_t kv_index(const orc_config *c, int32_t max_ctx, int l, int g, int p) {
    return (((int64_t)l * c->n_kv_heads + g) * max_ctx + p) * c->head_dim;
}

/*
 * One decode step at position `pos` (the cache already holds positions 0..pos-1).
 * kcache / vcache: [n_layers][n_kv_heads][max_ctx][head_dim] storage-dtype elements;
 * position `pos` is written. logits: [vocab] (may be NULL to skip the head).
 * Returns the argmax token, or -1 on bad arguments.
 */
int32_t orc_step(const orc_config *c, const orc_weights *w, uint16_t *kcache, uint16_t *vcache,
                 int32_t max_ctx, int32_t pos, int32_t token, double *logits) {
    if (pos < 0 || pos >= max_ctx || token < 0 || token >= c->vocab) return -1;
    const int d = c->d_model, Hq = c->n_heads, Hkv = c->n_kv_heads, D = c->head_dim, F = c->ffn;
    const int dt = c->dtype;
    double *x = calloc(d, sizeof(double)), *h = calloc(d, sizeof(double));
    double *q = calloc((size_t)Hq * D, sizeof(double)), *k = calloc((size_t)Hkv * D, sizeof(double));
    double *v = calloc((size_t)Hkv * D, sizeof(double)), *o = calloc((size_t)Hq * D, sizeof(double));
    double *y = calloc(d, sizeof(double)), *gt = calloc(F, sizeof(double)), *up = calloc(F, sizeof(double));

    for (int i = 0; i < d; i++) x[i] = orc_value(w->tok_emb[(int64_t)token * d + i], dt);

    for (int l = 0; l < c->n_layers; l++) {
        const uint16_t *const *L = w->layers + (int64_t)l * W_PER_LAYER;
        orc_rmsnorm(d, x, L[W_ATTN_NORM], dt, c->rms_eps, h);
        layer_matvec(c, w, l, W_Q, Hq * D, d, h, q);
        layer_matvec(c, w, l, W_K, Hkv * D, d, h, k);
        layer_matvec(c, w, l, W_V, Hkv * D, d, h, v);
        for (int hh = 0; hh < Hq; hh++) orc_rope(D, pos, c->rope_theta, q + hh * D);
        for (int g = 0; g < Hkv; g++) orc_rope(D, pos, c->rope_theta, k + g * D);
        for (int g = 0; g < Hkv; g++)
            for (int i = 0; i < D; i++) {
                kcache[kv_index(c, max_ctx, l, g, pos) + i] = orc_store(k[g * D + i], dt);
                vcache[kv_index(c, max_ctx, l, g, pos) + i] = orc_store(v[g * D + i], dt);
            }
        for (int hh = 0; hh < Hq; hh++) {
            int g = (int)(((int64_t)hh * Hkv) / Hq);
            orc_attention(D, pos + 1, q + hh * D, kcache + kv_index(c, max_ctx, l, g, 0),
                          vcache + kv_index(c, max_ctx, l, g, 0), dt, o + hh * D);
        }
        layer_matvec(c, w, l, W_O, d, Hq * D, o, y);
        for (int i = 0; i < d; i++) x[i] += y[i];
        orc_rmsnorm(d, x, L[W_MLP_NORM], dt, c->rms_eps, h);
        layer_matvec(c, w, l, W_GATE, F, d, h, gt);
        layer_matvec(c, w, l, W_UP, F, d, h, up);
        for (int i = 0; i < F; i++) gt[i] = orc_silu(gt[i]) * up[i];
        layer_matvec(c, w, l, W_DOWN, d, F, gt, y);
        for (int i = 0; i < d; i++) x[i] += y[i];
    }
    int32_t tok = -2;
    if (logits) {
        orc_rmsnorm(d, x, w->final_norm, dt, c->rms_eps, h);
        head_matvec(c, w, h, logits);
        tok = orc_argmax(c->vocab, logits);
    }
    free(x); free(h); free(q); free(k); free(v); free(o); free(y); free(gt); free(up);
    return tok;
}

/*
 * Full-sequence recompute: the same network applied to all n positions at once with a
 * causal mask and no carried cache (K and V are still rounded to the storage dtype,
 * as the method stores them). logits: [n][vocab]. Returns 0, or -1 on bad arguments.
 */
int32_t orc_forward_sequence(const orc_config *c, const orc_weights *w, int32_t n, const int32_t *tokens,
                             double *logits) {
    const int d = c->d_model, Hq = c->n_heads, Hkv = c->n_kv_heads, D = c->head_dim, F = c->ffn;
    const int dt = c->dtype;
    for (int t = 0; t < n; t++)
        if (tokens[t] < 0 || tokens[t] >= c->vocab) return -1;
    double *X = calloc((size_t)n * d, sizeof(double)), *H = calloc((size_t)n * d, sizeof(double));
    double *Q = calloc((size_t)n * Hq * D, sizeof(double)), *O = calloc((size_t)n * Hq * D, sizeof(double));
    double *Kf = calloc((size_t)Hkv * D, sizeof(double)), *Vf = calloc((size_t)Hkv * D, sizeof(double));
    uint16_t *Ks = calloc((size_t)Hkv * n * D, sizeof(uint16_t)), *Vs = calloc((size_t)Hkv * n * D, sizeof(uint16_t));
    double *Y = calloc(d, sizeof(double)), *G = calloc(F, sizeof(double)), *U = calloc(F, sizeof(double));

    for (int t = 0; t < n; t++)
        for (int i = 0; i < d; i++) X[(int64_t)t * d + i] = orc_value(w->tok_emb[(int64_t)tokens[t] * d + i], dt);

    for (int l = 0; l < c->n_layers; l++) {
        const uint16_t *const *L = w->layers + (int64_t)l * W_PER_LAYER;
        /* projections of every position; keys/values laid out [kv head][position][D] */
        for (int t = 0; t < n; t++) {
            orc_rmsnorm(d, X + (int64_t)t * d, L[W_ATTN_NORM], dt, c->rms_eps, H + (int64_t)t * d);
            layer_matvec(c, w, l, W_Q, Hq * D, d, H + (int64_t)t * d, Q + (int64_t)t * Hq * D);
            layer_matvec(c, w, l, W_K, Hkv * D, d, H + (int64_t)t * d, Kf);
            layer_matvec(c, w, l, W_V, Hkv * D, d, H + (int64_t)t * d, Vf);
            for (int hh = 0; hh < Hq; hh++) orc_rope(D, t, c->rope_theta, Q + ((int64_t)t * Hq + hh) * D);
            for (int g = 0; g < Hkv; g++) {
                orc_rope(D, t, c->rope_theta, Kf + g * D);
                for (int i = 0; i < D; i++) {
                    Ks[((int64_t)g * n + t) * D + i] = orc_store(Kf[g * D + i], dt);
                    Vs[((int64_t)g * n + t) * D + i] = orc_store(Vf[g * D + i], dt);
                }
            }
        }
        /* causal attention: position t sees positions 0..t */
        for (int t = 0; t < n; t++)
            for (int hh = 0; hh < Hq; hh++) {
                int g = (int)(((int64_t)hh * Hkv) / Hq);
                orc_attention(D, t + 1, Q + ((int64_t)t * Hq + hh) * D, Ks + (int64_t)g * n * D,
                              Vs + (int64_t)g * n * D, dt, O + ((int64_t)t * Hq + hh) * D);
            }
        for (int t = 0; t < n; t++) {
            double *x = X + (int64_t)t * d;
            layer_matvec(c, w, l, W_O, d, Hq * D, O + (int64_t)t * Hq * D, Y);
            for (int i = 0; i < d; i++) x[i] += Y[i];
            orc_rmsnorm(d, x, L[W_MLP_NORM], dt, c->rms_eps, H + (int64_t)t * d);
            layer_matvec(c, w, l, W_GATE, F, d, H + (int64_t)t * d, G);
            layer_matvec(c, w, l, W_UP, F, d, H + (int64_t)t * d, U);
            for (int i = 0; i < F; i++) G[i] = orc_silu(G[i]) * U[i];
            layer_matvec(c, w, l, W_DOWN, d, F, G, Y);
            for (int i = 0; i < d; i++) x[i] += Y[i];
        }
    }
    for (int t = 0; t < n; t++) {
        orc_rmsnorm(d, X + (int64_t)t * d, w->final_norm, dt, c->rms_eps, H + (int64_t)t * d);
        head_matvec(c, w, H + (int64_t)t * d, logits + (int64_t)t * c->vocab);
    }
    free(X); free(H); free(Q); free(O); free(Kf); free(Vf); free(Ks); free(Vs); free(Y); free(G); free(U);
    return 0;
}

int32_t orc_num_threads(void) { return omp_get_max_threads(); }

/* ---------------------------------------------------------------- sampling
 *
 * The variant beside greedy decoding: temperature and top-k sampling of the next token, with
 * one uniform draw per decode step taken from a counter-based generator, so a step's token is
 * a function of (logits, temperature, top_k, seed, position) alone.
 */

/* splitmix64: the state advances by the golden-ratio increment 0x9E3779B97F4A7C15 and each
   output is the new state through the finalizer below (two xor-shift-multiply rounds and a
   final xor-shift). Output n >= 1 of the generator started from state s is mix(s + n * inc). */
uint64_t orc_splitmix64(uint64_t seed, uint64_t n) {
    uint64_t z = seed + n * 0x9E3779B97F4A7C15ull;
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
    return z ^ (z >> 31);
}

/* The draw of the decode step at position pos: the top 24 bits of output pos + 1 of the
   generator started from `seed`, as a multiple of 2^-24 in [0, 1). */
double orc_uniform(uint64_t seed, int32_t pos) {
    return (double)(orc_splitmix64(seed, (uint64_t)pos + 1) >> 40) / 16777216.0;
}

/*
 * One sampled token. The candidates are the top_k largest logits, in order of value
 * (descending) and, for equal values, of index (ascending). Candidate k weighs
 * w_k = exp((z_k - z_0) / temperature); the token is the first candidate whose cumulative
 * weight exceeds u * (total weight). top_k = 1 is the greedy argmax.
 * Returns the token; -1 on bad arguments; -2 if a candidate's logit is not finite.
 * *margin (nullable) receives the distance from u * total to the nearest boundary between
 * candidates, divided by the total (1 when there is no boundary).
 */
int32_t orc_sample(int32_t n, const double *logits, double temperature, int32_t top_k, double u, double *margin) {
    if (n <= 0 || top_k < 1 || top_k > n || !(temperature > 0.0) || !(u >= 0.0 && u < 1.0)) return -1;
    int32_t *cand = (int32_t *)malloc(sizeof(int32_t) * top_k);
    char *taken = (char *)calloc(n, 1);
    /* the candidates in order: repeatedly the largest remaining value, lowest index first */
    for (int k = 0; k < top_k; k++) {
        int best = -1;
        for (int i = 0; i < n; i++) {
            if (taken[i]) continue;
            const double v = isnan(logits[i]) ? -INFINITY : logits[i];
            if (best < 0 || v > (isnan(logits[best]) ? -INFINITY : logits[best])) best = i;
        }
        cand[k] = best;
        taken[best] = 1;
    }
    int32_t tok = -2;
    int finite = 1;
    for (int k = 0; k < top_k; k++) finite &= isfinite(logits[cand[k]]) != 0;
    if (finite) {
        double *cum = (double *)malloc(sizeof(double) * top_k);
        double total = 0.0;
        for (int k = 0; k < top_k; k++) {
            total += exp((logits[cand[k]] - logits[cand[0]]) / temperature);
            cum[k] = total;
        }
        const double r = u * total;
        int pick = top_k - 1;
        for (int k = 0; k < top_k; k++)
            if (cum[k] > r) {
                pick = k;
                break;
            }
        tok = cand[pick];
        if (margin) {
            double m = 1.0;
            if (pick > 0) m = fmin(m, (r - cum[pick - 1]) / total);
            if (pick < top_k - 1) m = fmin(m, (cum[pick] - r) / total);
            *margin = m;
        }
        free(cum);
    }
    free(cand);
    free(taken);
    return tok;
}
