/*
 * oracle.c - CPU oracle of the batch-1 quantized decode step.
 *
 * TEST INFRASTRUCTURE ONLY: loaded by the tests, the smoke check and the
 * benchmark's CPU-baseline leg, never by the product path.  Plain loops in the
 * order the definitions are written, double accumulation, OpenMP over
 * independent output rows / heads only.  Shares no code with the CUDA library.
 *
 * Source of each definition: the ntransformer news summary (news.hada.io topic
 * 26894) names the formats ("Descripción general de NTransformer": Q4_0, Q8_0,
 * Q4_K_M, Q6_K), the kernels ("Arquitectura y estructura del código": GEMV,
 * RMSNorm, RoPE, SwiGLU, softmax), the Llama architecture pieces ("Funciones
 * principales": RoPE, GQA, SwiGLU, RMSNorm, KV cache) and the F16 KV cache
 * ("Hoja de ruta de desarrollo", Fase 3).  The pages print no formula or layout,
 * so each function below states the reading it implements.
 */
#include "oracle.h"

#include <math.h>
#include <stdlib.h>
#include <string.h>

#ifdef _OPENMP
#include <omp.h>
#endif

#define ORC_EXPORT __attribute__((visibility("default")))

/* ------------------------------------------------------------------ fp16 */

/* IEEE-754 binary16: 1 sign bit, 5 exponent bits (bias 15), 10 fraction bits.
 * exponent 0: subnormal, value = fraction * 2^-24; exponent 31: inf / NaN;
 * otherwise value = (1024 + fraction) * 2^(exponent - 25). */
ORC_EXPORT float orc_f16_to_f32(uint16_t h)
{
    int sign = (h >> 15) & 1;
    int e = (h >> 10) & 31;
    int f = h & 1023;
    double v;
    if (e == 0)
        v = ldexp((double)f, -24);
    else if (e == 31)
        v = f ? NAN : INFINITY;
    else
        v = ldexp((double)(1024 + f), e - 25);
    return (float)(sign ? -v : v);
}

/* Round an fp32 value to the nearest binary16 value, ties to even; overflow to
 * infinity.  The quantum (spacing of binary16 values) at |x| is
 * 2^(max(E, -14) - 10) where E = floor(log2 |x|). */
ORC_EXPORT uint16_t orc_f32_to_f16(float f)
{
    uint16_t sign = signbit(f) ? 0x8000 : 0;
    if (isnan(f)) return (uint16_t)(sign | 0x7E00);
    if (isinf(f)) return (uint16_t)(sign | 0x7C00);
    double a = fabs((double)f);
    if (a == 0.0) return sign;
    int E;
    frexp(a, &E);
    E -= 1;                                  /* a = m * 2^E, 1 <= m < 2 */
    int qe = (E < -14 ? -14 : E) - 10;       /* exponent of the quantum */
    double n = nearbyint(ldexp(a, -qe));     /* default mode: ties to even */
    if (E < -14) {
        /* subnormal range: n * 2^-24 with n in [0, 1024]; n == 1024 is the
         * smallest normal number, whose bit pattern is also 1024 */
        return (uint16_t)(sign | (uint16_t)n);
    }
    if (n >= 2048.0) { n = 1024.0; E += 1; }
    if (E > 15) return (uint16_t)(sign | 0x7C00);
    return (uint16_t)(sign | (uint16_t)((E + 15) << 10) | (uint16_t)((int)n - 1024));
}

static float f16_at(const uint8_t* p) { return orc_f16_to_f32((uint16_t)(p[0] | (p[1] << 8))); }

/* --------------------------------------------------------------- blocks */

ORC_EXPORT int orc_block_elems(int qtype)
{
    switch (qtype) {
    case ORC_Q8_0: case ORC_Q4_0: return 32;
    case ORC_Q4_K: case ORC_Q6_K: case ORC_Q5_K: return 256;
    case ORC_F16: case ORC_F32: return 1;
    default: return 0;
    }
}

ORC_EXPORT int orc_block_bytes(int qtype)
{
    switch (qtype) {
    case ORC_Q8_0: return 34;
    case ORC_Q4_0: return 18;
    case ORC_Q4_K: return 144;
    case ORC_Q6_K: return 210;
    case ORC_Q5_K: return 176;
    case ORC_F16: return 2;
    case ORC_F32: return 4;
    default: return 0;
    }
}

/* Q8_0 (34 B): fp16 d, then 32 int8 codes q; w_i = d * q_i.  (Format named in
 * "Descripción general de NTransformer"; block content as in the Q8_0 GEMV
 * workload: 32 int8 codes with one fp16 scale, w = q d.) */
static void dq_q8_0(const uint8_t* b, float* w)
{
    float d = f16_at(b);
    for (int i = 0; i < 32; ++i) w[i] = d * (float)(int8_t)b[2 + i];
}

/* Q4_0 (18 B): fp16 d, then 16 bytes; byte j holds element j in its low nibble
 * and element j+16 in its high nibble; w = (q - 8) * d. */
static void dq_q4_0(const uint8_t* b, float* w)
{
    float d = f16_at(b);
    for (int j = 0; j < 16; ++j) {
        int lo = b[2 + j] & 15, hi = b[2 + j] >> 4;
        w[j] = d * (float)(lo - 8);
        w[j + 16] = d * (float)(hi - 8);
    }
}

/* Q4_K scale/min of sub-block j (0..7) from the 12 packed bytes s:
 * sub-blocks 0..3: scale = low 6 bits of s[j], min = low 6 bits of s[j+4];
 * sub-blocks 4..7: scale = low nibble of s[j+4] plus the top 2 bits of s[j-4]
 * as bits 4..5; min = high nibble of s[j+4] plus the top 2 bits of s[j]. */
static void q4k_scale_min(const uint8_t* s, int j, int* sc, int* m)
{
    if (j < 4) {
        *sc = s[j] & 63;
        *m = s[j + 4] & 63;
    } else {
        *sc = (s[j + 4] & 15) | ((s[j - 4] >> 6) << 4);
        *m = (s[j + 4] >> 4) | ((s[j] >> 6) << 4);
    }
}

/* Q4_K (144 B / 256 weights): fp16 d, fp16 dmin, 12 bytes of scales/mins, 128
 * bytes of 4-bit codes.  Element 64c + l (c = 0..3, l = 0..31) is the low
 * nibble of code byte 32c + l, element 64c + 32 + l its high nibble; element e
 * is in sub-block e / 32.  w = d * scale_j * q - dmin * min_j. */
static void dq_q4_k(const uint8_t* b, float* w)
{
    float d = f16_at(b), dmin = f16_at(b + 2);
    const uint8_t* s = b + 4;
    const uint8_t* qs = b + 16;
    for (int e = 0; e < 256; ++e) {
        int c = e / 64, r = e % 64;
        int byte = qs[32 * c + (r % 32)];
        int q = r < 32 ? (byte & 15) : (byte >> 4);
        int sc, m;
        q4k_scale_min(s, e / 32, &sc, &m);
        float a = (d * (float)sc) * (float)q;   /* exact: at most 21 significant bits */
        float z = dmin * (float)m;              /* exact */
        w[e] = a - z;                           /* the one rounding */
    }
}

/* Q6_K (210 B / 256 weights): 128 bytes of low code bits ql, 64 bytes of high
 * code bits qh, 16 int8 sub-block scales, fp16 d.  For element e, with half
 * h = e / 128, t = e % 128, l = t % 32:
 *   low 4 bits: t <  64 -> low nibble of ql[64h + t]
 *               t >= 64 -> high nibble of ql[64h + t - 64]
 *   high 2 bits: bits 2*(t/32) .. +1 of qh[32h + l]
 * q in 0..63, sub-block j = e / 16, w = d * scale_j * (q - 32). */
static void dq_q6_k(const uint8_t* b, float* w)
{
    const uint8_t* ql = b;
    const uint8_t* qh = b + 128;
    const int8_t* sc = (const int8_t*)(b + 192);
    float d = f16_at(b + 208);
    for (int e = 0; e < 256; ++e) {
        int h = e / 128, t = e % 128, l = t % 32;
        int lo = t < 64 ? (ql[64 * h + t] & 15) : (ql[64 * h + t - 64] >> 4);
        int hi = (qh[32 * h + l] >> (2 * (t / 32))) & 3;
        int q = lo | (hi << 4);
        w[e] = (d * (float)sc[e / 16]) * (float)(q - 32);   /* exact */
    }
}

/* Q5_K (176 B / 256 weights): fp16 d, fp16 dmin, 12 bytes of scales/mins packed
 * as in Q4_K, 32 bytes qh of fifth code bits, 128 bytes qs of low 4 code bits.
 * (Format named with the K-quants in "Descripción general de NTransformer"; the
 * pages print no layout, so this is the GGUF convention as best known.)  Element
 * 64c + l (c = 0..3, l = 0..31): low 4 bits = low nibble of qs[32c + l], fifth bit =
 * bit 2c of qh[l]; element 64c + 32 + l: high nibble of qs[32c + l] and bit 2c + 1 of
 * qh[l].  q in 0..31, sub-block j = e / 32, w = d * scale_j * q - dmin * min_j. */
static void dq_q5_k(const uint8_t* b, float* w)
{
    float d = f16_at(b), dmin = f16_at(b + 2);
    const uint8_t* s = b + 4;
    const uint8_t* qh = b + 16;
    const uint8_t* qs = b + 48;
    for (int e = 0; e < 256; ++e) {
        int c = e / 64, r = e % 64, l = r % 32, upper = r >= 32;
        int lo = upper ? (qs[32 * c + l] >> 4) : (qs[32 * c + l] & 15);
        int hi = (qh[l] >> (2 * c + upper)) & 1;
        int q = lo + 16 * hi;
        int sc, m;
        q4k_scale_min(s, e / 32, &sc, &m);
        float a = (d * (float)sc) * (float)q;   /* exact: at most 22 significant bits */
        float z = dmin * (float)m;              /* exact */
        w[e] = a - z;                           /* the one rounding */
    }
}

/* F16: one IEEE binary16 value per weight (little-endian); F32: one binary32.
 * (Formats named in "Descripción general de NTransformer".) */
static void dq_f16(const uint8_t* b, float* w) { *w = f16_at(b); }

static void dq_f32(const uint8_t* b, float* w) { memcpy(w, b, 4); }

static int dequant_block(int qtype, const uint8_t* b, float* w)
{
    switch (qtype) {
    case ORC_Q8_0: dq_q8_0(b, w); return 0;
    case ORC_Q4_0: dq_q4_0(b, w); return 0;
    case ORC_Q4_K: dq_q4_k(b, w); return 0;
    case ORC_Q6_K: dq_q6_k(b, w); return 0;
    case ORC_Q5_K: dq_q5_k(b, w); return 0;
    case ORC_F16: dq_f16(b, w); return 0;
    case ORC_F32: dq_f32(b, w); return 0;
    default: return -1;
    }
}

static int dequant_row(int qtype, const uint8_t* row, int64_t cols, float* out)
{
    int be = orc_block_elems(qtype), bb = orc_block_bytes(qtype);
    for (int64_t kb = 0; kb < cols / be; ++kb)
        if (dequant_block(qtype, row + kb * bb, out + kb * be)) return -1;
    return 0;
}

static int shape_ok(int qtype, int64_t cols)
{
    int be = orc_block_elems(qtype);
    return be > 0 && cols > 0 && cols % be == 0;
}

ORC_EXPORT int orc_dequant(int qtype, const uint8_t* W, int64_t rows, int64_t cols, float* out)
{
    if (!shape_ok(qtype, cols)) return -1;
    int64_t rb = cols / orc_block_elems(qtype) * orc_block_bytes(qtype);
    #pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < rows; ++r) dequant_row(qtype, W + r * rb, cols, out + r * cols);
    return 0;
}

/* GEMV, "cuda/: kernels de GEMV": y_r = sum_k w_{r,k} x_k over the dequantized
 * row, products and sum in double, stored as fp32. */
ORC_EXPORT int orc_gemv(int qtype, const uint8_t* W, int64_t rows, int64_t cols, const float* x, float* y)
{
    if (!shape_ok(qtype, cols)) return -1;
    int64_t rb = cols / orc_block_elems(qtype) * orc_block_bytes(qtype);
    #pragma omp parallel
    {
        float* w = (float*)malloc((size_t)cols * sizeof(float));
        #pragma omp for schedule(static)
        for (int64_t r = 0; r < rows; ++r) {
            dequant_row(qtype, W + r * rb, cols, w);
            double acc = 0.0;
            for (int64_t k = 0; k < cols; ++k) acc += (double)w[k] * (double)x[k];
            y[r] = (float)acc;
        }
        free(w);
    }
    return 0;
}

/* RMSNorm: y_i = x_i / sqrt(mean(x^2) + eps) * w_i (eps inside the root, weight
 * applied after normalising). */
ORC_EXPORT void orc_rmsnorm(const float* x, const float* w, float* y, int64_t n, float eps)
{
    double ss = 0.0;
    for (int64_t i = 0; i < n; ++i) ss += (double)x[i] * (double)x[i];
    double inv = 1.0 / sqrt(ss / (double)n + (double)eps);
    for (int64_t i = 0; i < n; ++i) y[i] = (float)((double)x[i] * inv * (double)w[i]);
}

/* RoPE on adjacent pairs (2i, 2i+1) of every head of q and k: the pair is
 * rotated by the angle pos * theta^(-2i / head_dim). */
static void rope_head(float* x, int head_dim, int32_t pos, double theta)
{
    for (int i = 0; i < head_dim / 2; ++i) {
        double ang = (double)pos * pow(theta, -(2.0 * i) / (double)head_dim);
        double c = cos(ang), s = sin(ang);
        double a = x[2 * i], b = x[2 * i + 1];
        x[2 * i] = (float)(a * c - b * s);
        x[2 * i + 1] = (float)(a * s + b * c);
    }
}

ORC_EXPORT void orc_rope(float* q, float* k, int n_q_heads, int n_kv_heads, int head_dim, int32_t pos,
                         double theta)
{
    for (int h = 0; h < n_q_heads; ++h) rope_head(q + (int64_t)h * head_dim, head_dim, pos, theta);
    for (int h = 0; h < n_kv_heads; ++h) rope_head(k + (int64_t)h * head_dim, head_dim, pos, theta);
}

/* GQA decode attention for one query token: q head h reads kv head
 * g = h / (n_q_heads / n_kv_heads); s_t = q . K[g][t] / sqrt(head_dim) for
 * t = 0..n_ctx-1; p = softmax(s); out_h = sum_t p_t V[g][t].  The caches are
 * [n_kv_heads][max_ctx][head_dim] fp16. */
ORC_EXPORT void orc_attn_decode(const float* q, const uint16_t* k_cache, const uint16_t* v_cache, float* out,
                                int n_q_heads, int n_kv_heads, int head_dim, int32_t n_ctx, int32_t max_ctx)
{
    int group = n_q_heads / n_kv_heads;
    double scale = 1.0 / sqrt((double)head_dim);
    #pragma omp parallel for schedule(static)
    for (int h = 0; h < n_q_heads; ++h) {
        int g = h / group;
        const float* qh = q + (int64_t)h * head_dim;
        double* s = (double*)malloc((size_t)n_ctx * sizeof(double));
        double* o = (double*)calloc((size_t)head_dim, sizeof(double));
        double mx = -INFINITY;
        for (int32_t t = 0; t < n_ctx; ++t) {
            const uint16_t* kt = k_cache + ((int64_t)g * max_ctx + t) * head_dim;
            double dot = 0.0;
            for (int d = 0; d < head_dim; ++d) dot += (double)qh[d] * (double)orc_f16_to_f32(kt[d]);
            s[t] = dot * scale;
            if (s[t] > mx) mx = s[t];
        }
        double sum = 0.0;
        for (int32_t t = 0; t < n_ctx; ++t) { s[t] = exp(s[t] - mx); sum += s[t]; }
        for (int32_t t = 0; t < n_ctx; ++t) {
            const uint16_t* vt = v_cache + ((int64_t)g * max_ctx + t) * head_dim;
            double p = s[t] / sum;
            for (int d = 0; d < head_dim; ++d) o[d] += p * (double)orc_f16_to_f32(vt[d]);
        }
        for (int d = 0; d < head_dim; ++d) out[(int64_t)h * head_dim + d] = (float)o[d];
        free(s);
        free(o);
    }
}

/* SwiGLU: out_i = silu(gate_i) * up_i, silu(g) = g / (1 + e^-g). */
ORC_EXPORT void orc_swiglu(const float* gate, const float* up, float* out, int64_t n)
{
    for (int64_t i = 0; i < n; ++i) {
        double g = gate[i];
        out[i] = (float)(g / (1.0 + exp(-g)) * (double)up[i]);
    }
}

/* softmax: y_i = e^(x_i - max x) / sum_j e^(x_j - max x). */
ORC_EXPORT void orc_softmax(const float* x, float* y, int64_t n)
{
    double mx = -INFINITY;
    for (int64_t i = 0; i < n; ++i) if (x[i] > mx) mx = x[i];
    double sum = 0.0;
    for (int64_t i = 0; i < n; ++i) sum += exp((double)x[i] - mx);
    for (int64_t i = 0; i < n; ++i) y[i] = (float)(exp((double)x[i] - mx) / sum);
}

/* ------------------------------------------------------------ decode step */

static int64_t rbytes(int qtype, int64_t cols)
{
    return cols / orc_block_elems(qtype) * orc_block_bytes(qtype);
}

/* One Llama layer at position pos:
 *   xn = RMSNorm(h, attn_norm); [q|k|v] = W_qkv xn; RoPE(q, k, pos);
 *   K[g][pos] = fp16(k_g), V[g][pos] = fp16(v_g);
 *   a = attention(q, K, V) over positions 0..pos; h += W_o a;
 *   xn = RMSNorm(h, ffn_norm); f = silu(W_gate xn) * (W_up xn); h += W_down f. */
ORC_EXPORT int orc_decode_layer(const orc_dims* D, const orc_layer* L, float* h, int32_t pos)
{
    int64_t H = D->hidden, hd = D->head_dim, qd = (int64_t)D->n_q_heads * hd, kvd = (int64_t)D->n_kv_heads * hd;
    int64_t F = D->ffn;
    const int qt_qkv = L->qtype[0], qt_o = L->qtype[1], qt_ffn = L->qtype[2], qt_down = L->qtype[3];
    if (!shape_ok(qt_qkv, H) || !shape_ok(qt_o, qd) || !shape_ok(qt_ffn, H) || !shape_ok(qt_down, F) || pos < 0 ||
        pos >= D->max_ctx)
        return -1;
    float* xn = (float*)malloc((size_t)H * sizeof(float));
    float* qkv = (float*)malloc((size_t)(qd + 2 * kvd) * sizeof(float));
    float* att = (float*)malloc((size_t)qd * sizeof(float));
    float* o = (float*)malloc((size_t)H * sizeof(float));
    float* g = (float*)malloc((size_t)F * sizeof(float));
    float* u = (float*)malloc((size_t)F * sizeof(float));
    float* a = (float*)malloc((size_t)F * sizeof(float));

    orc_rmsnorm(h, L->attn_norm, xn, H, D->rms_eps);
    orc_gemv(qt_qkv, L->w_qkv, qd + 2 * kvd, H, xn, qkv);
    float *q = qkv, *k = qkv + qd, *v = qkv + qd + kvd;
    orc_rope(q, k, D->n_q_heads, D->n_kv_heads, D->head_dim, pos, D->rope_theta);
    for (int gi = 0; gi < D->n_kv_heads; ++gi)
        for (int64_t d = 0; d < hd; ++d) {
            int64_t at = ((int64_t)gi * D->max_ctx + pos) * hd + d;
            L->k_cache[at] = orc_f32_to_f16(k[gi * hd + d]);
            L->v_cache[at] = orc_f32_to_f16(v[gi * hd + d]);
        }
    orc_attn_decode(q, L->k_cache, L->v_cache, att, D->n_q_heads, D->n_kv_heads, D->head_dim, pos + 1, D->max_ctx);
    orc_gemv(qt_o, L->w_o, H, qd, att, o);
    for (int64_t i = 0; i < H; ++i) h[i] = h[i] + o[i];

    orc_rmsnorm(h, L->ffn_norm, xn, H, D->rms_eps);
    orc_gemv(qt_ffn, L->w_gate, F, H, xn, g);
    orc_gemv(qt_ffn, L->w_up, F, H, xn, u);
    orc_swiglu(g, u, a, F);
    orc_gemv(qt_down, L->w_down, H, F, a, o);
    for (int64_t i = 0; i < H; ++i) h[i] = h[i] + o[i];

    free(xn); free(qkv); free(att); free(o); free(g); free(u); free(a);
    return 0;
}

/* Token embedding lookup: the dequantized row `token` of E. */
ORC_EXPORT int orc_embed(int qtype, const uint8_t* E, int64_t hidden, int32_t token, float* h)
{
    if (!shape_ok(qtype, hidden) || token < 0) return -1;
    return dequant_row(qtype, E + (int64_t)token * rbytes(qtype, hidden), hidden, h);
}

ORC_EXPORT int orc_lm_head(int qtype, const float* out_norm, const uint8_t* W_out, int64_t vocab, int64_t hidden,
                           float eps, const float* h, float* logits)
{
    if (!shape_ok(qtype, hidden)) return -1;
    float* xn = (float*)malloc((size_t)hidden * sizeof(float));
    orc_rmsnorm(h, out_norm, xn, hidden, eps);
    int rc = orc_gemv(qtype, W_out, vocab, hidden, xn, logits);
    free(xn);
    return rc;
}

ORC_EXPORT void orc_set_threads(int n)
{
#ifdef _OPENMP
    if (n > 0) omp_set_num_threads(n);
#else
    (void)n;
#endif
}

ORC_EXPORT int orc_get_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
