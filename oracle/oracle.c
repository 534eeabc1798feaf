/*
 * ORACLE - test infrastructure only.  A plain, slow, fp64 CPU statement of what
 * the padding-free varlen GPT-3 layer stack computes.  Only the tests, the
 * smoke check and the bench's CPU-baseline leg may load it; the product path
 * never does.  It shares no code, header or constant with the CUDA library.
 *
 * Sources (pages on Energon-AI):
 *  [A]  "最新大模型推理系统Energon-AI开源，来自Colossal-AI团队" (QbitAI article),
 *       section "Runtime": transpose_padding_remove / transpose_padding_rebuild
 *       serve variable-length NLP inputs by eliminating the redundant work of
 *       padding; section "易用性" (usability): the FasterTransformer excerpt with
 *       the bias+GELU and bias+residual+LayerNorm steps of a transformer MLP.
 *  [B]  EnergonAI README, section "Scaling Ability": GPT-3 layers in FP16,
 *       redundant computation elimination (EffectiveTransformer's method),
 *       sequence length half the padding length.
 * The pages give no formulas.  Where they are silent this file takes the plain
 * reading of a pre-LN GPT decoder layer; every such reading is listed at the
 * function it concerns.
 *
 * Arithmetic is IEEE double throughout.  Storage inputs (f32 / f16 / bf16) are
 * decoded exactly to double; nothing is rounded back to a narrow type.  A sum
 * is a plain loop in index order; a matrix product is the defining
 * sum over k written out for each output element.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define OR_F32 0
#define OR_F16 1
#define OR_BF16 2
#define OR_F64 3

/* ------------------------------------------------------------------ decoding */

/* IEEE binary16 bits -> exact double. */
static double dec_f16(uint16_t h) {
    int sign = (h >> 15) & 1, e = (h >> 10) & 31, m = h & 1023;
    double v;
    if (e == 0) v = ldexp((double)m, -24);
    else if (e == 31) v = m ? NAN : INFINITY;
    else v = ldexp((double)(1024 + m), e - 25);
    return sign ? -v : v;
}

/* bfloat16 bits -> exact double (bf16 is the upper half of an IEEE binary32). */
static double dec_bf16(uint16_t h) {
    uint32_t u = (uint32_t)h << 16;
    float f;
    memcpy(&f, &u, 4);
    return (double)f;
}

static double elem(const void* p, int dtype, int64_t i) {
    switch (dtype) {
    case OR_F32: return (double)((const float*)p)[i];
    case OR_F16: return dec_f16(((const uint16_t*)p)[i]);
    case OR_BF16: return dec_bf16(((const uint16_t*)p)[i]);
    default: return ((const double*)p)[i];
    }
}

/* Storage array -> double array (exact). */
int oracle_decode(const void* in, int dtype, int64_t n, double* out) {
    if (!in || !out || n < 0 || dtype < 0 || dtype > 3) return 1;
    for (int64_t i = 0; i < n; ++i) out[i] = elem(in, dtype, i);
    return 0;
}

/* ------------------------------------------------------- offsets, remove, rebuild */

/*
 * Offsets of the packed layout ([A] "Runtime": the packing behind
 * transpose_padding_remove; the offsets are the exclusive prefix sum of the
 * per-sequence lengths):  cu[0] = 0,  cu[b+1] = cu[b] + len[b].
 * Reading for invalid input (the pages are silent): a length outside
 * [0, pad_len] sets *status = 1 and the whole cu array to 0 (an empty
 * packing); otherwise *status = 0.
 */
int oracle_offsets(const int32_t* lengths, int batch, int pad_len, int32_t* cu, int32_t* status) {
    if (!lengths || !cu || !status || batch < 0) return 1;
    int ok = 1;
    for (int b = 0; b < batch; ++b)
        if (lengths[b] < 0 || lengths[b] > pad_len) ok = 0;
    if (!ok) {
        for (int b = 0; b <= batch; ++b) cu[b] = 0;
        *status = 1;
        return 0;
    }
    cu[0] = 0;
    for (int b = 0; b < batch; ++b) cu[b + 1] = cu[b] + lengths[b];
    *status = 0;
    return 0;
}

/*
 * transpose_padding_remove ([A] "Runtime"): packed row cu[b] + s is padded
 * row (b, s) for every s < len[b] = cu[b+1] - cu[b].  A byte copy of
 * `row_bytes` bytes per row; packed rows at or beyond cu[batch] are not
 * touched.
 */
int oracle_remove_padding(const void* padded, const int32_t* cu, int batch, int pad_len,
                          int64_t row_bytes, void* packed) {
    if (!padded || !cu || !packed || batch < 0 || pad_len < 0 || row_bytes < 0) return 1;
    const unsigned char* src = (const unsigned char*)padded;
    unsigned char* dst = (unsigned char*)packed;
    for (int b = 0; b < batch; ++b) {
        int len = cu[b + 1] - cu[b];
        for (int s = 0; s < len; ++s)
            for (int64_t k = 0; k < row_bytes; ++k)
                dst[((int64_t)cu[b] + s) * row_bytes + k] = src[((int64_t)b * pad_len + s) * row_bytes + k];
    }
    return 0;
}

/*
 * transpose_padding_rebuild ([A] "Runtime"): padded row (b, s) is packed row
 * cu[b] + s when s < len[b]; every other padded row is all-zero bytes (the
 * pages say the result returns to padded layout; zero pads are the reading).
 */
int oracle_rebuild_padding(const void* packed, const int32_t* cu, int batch, int pad_len,
                           int64_t row_bytes, void* padded) {
    if (!padded || !cu || !packed || batch < 0 || pad_len < 0 || row_bytes < 0) return 1;
    const unsigned char* src = (const unsigned char*)packed;
    unsigned char* dst = (unsigned char*)padded;
    for (int b = 0; b < batch; ++b) {
        int len = cu[b + 1] - cu[b];
        for (int s = 0; s < pad_len; ++s)
            for (int64_t k = 0; k < row_bytes; ++k)
                dst[((int64_t)b * pad_len + s) * row_bytes + k] =
                    s < len ? src[((int64_t)cu[b] + s) * row_bytes + k] : 0;
    }
    return 0;
}

/*
 * Head-transposing forms of the two operations.  The pages give only the names
 * transpose_padding_remove / transpose_padding_rebuild ([A] "Runtime"); the
 * reading for "transpose" is the [token, head] <-> [head, token] exchange a
 * padded attention stage needs: a packed token row holds `parts` blocks
 * (1 for an attention output, 3 for Q | K | V) of n_heads heads of
 * `head_bytes` bytes each, and the head-major padded tensor is
 * [parts][batch][n_heads][pad_len][head_bytes].
 *
 * transpose_padding_rebuild: head-major element (c, b, h, s) is packed row
 * cu[b] + s, block c, head h, for s < len[b]; all-zero bytes for s >= len[b].
 */
int oracle_transpose_padding_rebuild(const void* packed, const int32_t* cu, int batch, int pad_len, int parts,
                                     int n_heads, int64_t head_bytes, void* heads) {
    if (!packed || !cu || !heads || batch < 0 || pad_len < 0 || parts < 1 || n_heads < 1 || head_bytes < 0)
        return 1;
    const unsigned char* src = (const unsigned char*)packed;
    unsigned char* dst = (unsigned char*)heads;
    const int64_t row = (int64_t)parts * n_heads * head_bytes;
    for (int c = 0; c < parts; ++c)
        for (int b = 0; b < batch; ++b) {
            int len = cu[b + 1] - cu[b];
            for (int h = 0; h < n_heads; ++h)
                for (int s = 0; s < pad_len; ++s) {
                    int64_t o = ((((int64_t)c * batch + b) * n_heads + h) * pad_len + s) * head_bytes;
                    int64_t i = ((int64_t)cu[b] + s) * row + ((int64_t)c * n_heads + h) * head_bytes;
                    for (int64_t k = 0; k < head_bytes; ++k) dst[o + k] = s < len ? src[i + k] : 0;
                }
        }
    return 0;
}

/*
 * transpose_padding_remove: packed row cu[b] + s, block c, head h is head-major
 * element (c, b, h, s), for every s < len[b]; packed rows at or beyond
 * cu[batch] are not touched.
 */
int oracle_transpose_padding_remove(const void* heads, const int32_t* cu, int batch, int pad_len, int parts,
                                    int n_heads, int64_t head_bytes, void* packed) {
    if (!packed || !cu || !heads || batch < 0 || pad_len < 0 || parts < 1 || n_heads < 1 || head_bytes < 0)
        return 1;
    const unsigned char* src = (const unsigned char*)heads;
    unsigned char* dst = (unsigned char*)packed;
    const int64_t row = (int64_t)parts * n_heads * head_bytes;
    for (int b = 0; b < batch; ++b) {
        int len = cu[b + 1] - cu[b];
        for (int s = 0; s < len; ++s)
            for (int c = 0; c < parts; ++c)
                for (int h = 0; h < n_heads; ++h) {
                    int64_t o = ((int64_t)cu[b] + s) * row + ((int64_t)c * n_heads + h) * head_bytes;
                    int64_t i = ((((int64_t)c * batch + b) * n_heads + h) * pad_len + s) * head_bytes;
                    for (int64_t k = 0; k < head_bytes; ++k) dst[o + k] = src[i + k];
                }
    }
    return 0;
}

/* ----------------------------------------------------------- layer building blocks */

/*
 * LayerNorm over the last dimension (the normalisation of [A]'s
 * add_bias_input_layernorm step; placed before each sub-layer, the pre-LN GPT
 * reading):  y = (v - mean(v)) / sqrt(mean((v - mean(v))^2) + eps) * g + b,
 * biased variance.
 */
int oracle_layernorm(const double* x, int64_t rows, int hidden, const void* g, const void* beta,
                     int wdtype, double eps, double* y) {
    if (!x || !y || !g || !beta || hidden <= 0 || rows < 0) return 1;
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < rows; ++r) {
        const double* v = x + r * hidden;
        double mean = 0.0;
        for (int k = 0; k < hidden; ++k) mean += v[k];
        mean /= hidden;
        double var = 0.0;
        for (int k = 0; k < hidden; ++k) var += (v[k] - mean) * (v[k] - mean);
        var /= hidden;
        double inv = 1.0 / sqrt(var + eps);
        for (int k = 0; k < hidden; ++k)
            y[r * hidden + k] = (v[k] - mean) * inv * elem(g, wdtype, k) + elem(beta, wdtype, k);
    }
    return 0;
}

/*
 * Linear layer in nn.Linear layout: y[t][n] = sum_k x[t][k] * W[n][k] + bias[n]
 * (the GEMMs of [A]'s excerpt; W is [out, in]).  `bias` may be NULL.
 * Each output element is its own k-ordered sum; output columns are spread
 * over threads.
 */
int oracle_linear(const double* x, int64_t rows, int in_dim, const void* W, const void* bias,
                  int out_dim, int wdtype, double* y) {
    if (!x || !W || !y || in_dim <= 0 || out_dim <= 0 || rows < 0) return 1;
#pragma omp parallel
    {
        double* w = (double*)malloc(sizeof(double) * (size_t)in_dim);
#pragma omp for schedule(static)
        for (int n = 0; n < out_dim; ++n) {
            for (int k = 0; k < in_dim; ++k) w[k] = elem(W, wdtype, (int64_t)n * in_dim + k);
            double bn = bias ? elem(bias, wdtype, n) : 0.0;
            for (int64_t t = 0; t < rows; ++t) {
                const double* xt = x + t * in_dim;
                double acc = 0.0;
                for (int k = 0; k < in_dim; ++k) acc += xt[k] * w[k];
                y[t * out_dim + n] = acc + bn;
            }
        }
        free(w);
    }
    return 0;
}

/*
 * GELU ([A]'s add_bias_act step with ActivationType::GELU).  The pages name
 * the activation only; tanh_form = 1 is the GPT-2/GPT-3 tanh approximation
 * 0.5 x (1 + tanh(sqrt(2/pi) (x + 0.044715 x^3))), tanh_form = 0 the exact
 * 0.5 x (1 + erf(x / sqrt(2))).
 */
int oracle_gelu(const double* x, int64_t n, int tanh_form, double* y) {
    if (!x || !y || n < 0) return 1;
    const double c = sqrt(2.0 / 3.14159265358979323846);
    for (int64_t i = 0; i < n; ++i) {
        double v = x[i];
        y[i] = tanh_form ? 0.5 * v * (1.0 + tanh(c * (v + 0.044715 * v * v * v)))
                         : 0.5 * v * (1.0 + erf(v / sqrt(2.0)));
    }
    return 0;
}

/*
 * Causal self-attention of ONE sequence of L tokens.  qkv is [L, 3H] with
 * columns [Q | K | V], each H wide and head-major (head j owns columns
 * j*d .. j*d+d-1, d = H / n_heads).  For every head j and position s:
 *     o_j(s) = sum_{t <= s} softmax_t(q_j(s) . k_j(t) / sqrt(d)) v_j(t)
 * Keys come from the same sequence only (positions of other sequences and
 * padding never enter).  The softmax subtracts the row maximum before
 * exponentiating, which leaves its value unchanged.
 */
int oracle_causal_attention(const double* qkv, int L, int hidden, int n_heads, double* o) {
    if (!qkv || !o || L < 0 || hidden <= 0 || n_heads <= 0 || hidden % n_heads) return 1;
    const int d = hidden / n_heads;
    const double scale = 1.0 / sqrt((double)d);
    const int64_t ld = 3 * (int64_t)hidden;
#pragma omp parallel
    {
        double* p = (double*)malloc(sizeof(double) * (size_t)(L > 0 ? L : 1));
#pragma omp for collapse(2) schedule(static)
        for (int j = 0; j < n_heads; ++j)
            for (int s = 0; s < L; ++s) {
                const double* q = qkv + s * ld + (int64_t)j * d;
                double m = -INFINITY;
                for (int t = 0; t <= s; ++t) {
                    const double* k = qkv + t * ld + hidden + (int64_t)j * d;
                    double dot = 0.0;
                    for (int e = 0; e < d; ++e) dot += q[e] * k[e];
                    p[t] = dot * scale;
                    if (p[t] > m) m = p[t];
                }
                double z = 0.0;
                for (int t = 0; t <= s; ++t) {
                    p[t] = exp(p[t] - m);
                    z += p[t];
                }
                for (int e = 0; e < d; ++e) {
                    double acc = 0.0;
                    for (int t = 0; t <= s; ++t) acc += p[t] * qkv[t * ld + 2 * (int64_t)hidden + (int64_t)j * d + e];
                    o[(int64_t)s * hidden + (int64_t)j * d + e] = acc / z;
                }
            }
        free(p);
    }
    return 0;
}

/* ------------------------------------------------------------------- the layer */

typedef struct {
    int hidden, n_heads, ffn;
    int wdtype;     /* storage type of every weight tensor: OR_F32 / OR_F16 / OR_BF16 / OR_F64 */
    double ln_eps;
    int gelu_tanh;
} oracle_layer_cfg;

typedef struct {
    const void *ln1_g, *ln1_b, *w_qkv, *b_qkv, *w_o, *b_o, *ln2_g, *ln2_b, *w_1, *b_1, *w_2, *b_2;
} oracle_layer_weights;

/*
 * One pre-LN GPT decoder layer on the L valid tokens of one sequence
 * (x, y: [L, H]; y may not alias x):
 *     a  = LN(x; g1, b1)
 *     q|k|v = a W_qkv^T + b_qkv
 *     x1 = x + attn(q, k, v) W_o^T + b_o
 *     y  = x1 + GELU(LN(x1; g2, b2) W_1^T + b_1) W_2^T + b_2
 * The pre-LN placement, the fused [Q | K | V] projection and the absence of
 * dropout and position embeddings are readings (the pages print none of it;
 * [A]'s FasterTransformer excerpt is a post-LN variant of the same parts).
 */
int oracle_layer_sequence(const oracle_layer_cfg* c, const oracle_layer_weights* w, const double* x,
                          int L, double* y) {
    if (!c || !w || !x || !y || L < 0) return 1;
    const int H = c->hidden, F = c->ffn, dt = c->wdtype;
    if (L == 0) return 0;
    double* a = (double*)malloc(sizeof(double) * (size_t)L * H);
    double* qkv = (double*)malloc(sizeof(double) * (size_t)L * 3 * H);
    double* o = (double*)malloc(sizeof(double) * (size_t)L * H);
    double* x1 = (double*)malloc(sizeof(double) * (size_t)L * H);
    double* f = (double*)malloc(sizeof(double) * (size_t)L * F);
    int rc = 0;
    if (!a || !qkv || !o || !x1 || !f) { rc = 2; goto done; }

    rc |= oracle_layernorm(x, L, H, w->ln1_g, w->ln1_b, dt, c->ln_eps, a);
    rc |= oracle_linear(a, L, H, w->w_qkv, w->b_qkv, 3 * H, dt, qkv);
    rc |= oracle_causal_attention(qkv, L, H, c->n_heads, o);
    rc |= oracle_linear(o, L, H, w->w_o, w->b_o, H, dt, x1);
    for (int64_t i = 0; i < (int64_t)L * H; ++i) x1[i] += x[i];
    rc |= oracle_layernorm(x1, L, H, w->ln2_g, w->ln2_b, dt, c->ln_eps, a);
    rc |= oracle_linear(a, L, H, w->w_1, w->b_1, F, dt, f);
    rc |= oracle_gelu(f, (int64_t)L * F, c->gelu_tanh, f);
    rc |= oracle_linear(f, L, F, w->w_2, w->b_2, H, dt, y);
    for (int64_t i = 0; i < (int64_t)L * H; ++i) y[i] += x1[i];
done:
    free(a); free(qkv); free(o); free(x1); free(f);
    return rc;
}

/*
 * The layer on a padded batch, the way the pages frame the problem: padded
 * input [batch, pad_len, H] plus per-sequence lengths.  Valid rows (s < len[b])
 * get the layer of their own sequence; every pad row of the output is 0.
 * Returns 3 when a length lies outside [0, pad_len].
 */
int oracle_layer_padded(const oracle_layer_cfg* c, const oracle_layer_weights* w, const double* x_padded,
                        const int32_t* lengths, int batch, int pad_len, double* y_padded) {
    if (!c || !w || !x_padded || !lengths || !y_padded || batch < 0 || pad_len < 0) return 1;
    for (int b = 0; b < batch; ++b)
        if (lengths[b] < 0 || lengths[b] > pad_len) return 3;
    const int64_t H = c->hidden;
    for (int b = 0; b < batch; ++b) {
        const double* xb = x_padded + (int64_t)b * pad_len * H;
        double* yb = y_padded + (int64_t)b * pad_len * H;
        int rc = oracle_layer_sequence(c, w, xb, lengths[b], yb);
        if (rc) return rc;
        for (int64_t i = (int64_t)lengths[b] * H; i < (int64_t)pad_len * H; ++i) yb[i] = 0.0;
    }
    return 0;
}
