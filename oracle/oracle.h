/*
 * oracle.h - CPU oracle of the batch-1 quantized decode step.
 *
 * TEST INFRASTRUCTURE ONLY.  This is the plain, slow, obviously-correct CPU
 * statement of what the GPU path computes; only the tests, the smoke check and
 * the CPU-baseline leg of the benchmark may load it.  It shares no code with the
 * CUDA library (own fp16 conversion, own block decoding, double accumulation).
 *
 * What it follows: the ntransformer news summary (news.hada.io topic 26894).
 *   - "Descripción general de NTransformer": GGUF model format, Q4_0, Q8_0,
 *     Q4_K_M, Q5_K, Q6_K, F16, F32 weights.
 *   - "Funciones principales": Llama architecture with RoPE, GQA, SwiGLU,
 *     RMSNorm and a KV cache.
 *   - "Arquitectura y estructura del código": GEMV, RMSNorm, RoPE, SwiGLU and
 *     softmax kernels; model/ holds attention, FFN and normalization.
 *   - "Hoja de ruta de desarrollo", Fase 3: the KV cache is stored in F16.
 * The pages define no block layout or formula; the readings taken here are the
 * plain GGUF-style ones, written out per function in oracle.c.
 *
 * Precision: every dot product, norm and softmax sum accumulates in double; each
 * op's output vector is stored as fp32 (fp16 for the KV cache), like the GPU path.
 */
#ifndef NTX_ORACLE_H
#define NTX_ORACLE_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

enum { ORC_Q8_0 = 0, ORC_Q4_0 = 1, ORC_Q4_K = 2, ORC_Q6_K = 3, ORC_Q5_K = 4, ORC_F16 = 5, ORC_F32 = 6 };

float orc_f16_to_f32(uint16_t h);
uint16_t orc_f32_to_f16(float f);

int orc_block_elems(int qtype);
int orc_block_bytes(int qtype);

/* Dequantize a [rows, cols] packed tensor to fp32 (row-major).  Returns 0, or -1
 * on a bad qtype / cols. */
int orc_dequant(int qtype, const uint8_t* W, int64_t rows, int64_t cols, float* out);

/* y[r] = sum_k w[r,k] * x[k], w dequantized, double accumulation. */
int orc_gemv(int qtype, const uint8_t* W, int64_t rows, int64_t cols, const float* x, float* y);

void orc_rmsnorm(const float* x, const float* w, float* y, int64_t n, float eps);
void orc_rope(float* q, float* k, int n_q_heads, int n_kv_heads, int head_dim, int32_t pos, double theta);
void orc_attn_decode(const float* q, const uint16_t* k_cache, const uint16_t* v_cache, float* out,
                     int n_q_heads, int n_kv_heads, int head_dim, int32_t n_ctx, int32_t max_ctx);
void orc_swiglu(const float* gate, const float* up, float* out, int64_t n);
void orc_softmax(const float* x, float* y, int64_t n);

typedef struct orc_dims {
    int32_t hidden, n_q_heads, n_kv_heads, head_dim, ffn, max_ctx;
    float rms_eps;
    double rope_theta;
} orc_dims;

typedef struct orc_layer {
    int32_t qtype[4];        /* formats of w_qkv, w_o, w_gate and w_up, w_down */
    const float* attn_norm;
    const uint8_t* w_qkv;    /* [(nq + 2 nkv) * hd, hidden]: q rows, then k rows, then v rows */
    const uint8_t* w_o;      /* [hidden, nq * hd] */
    const float* ffn_norm;
    const uint8_t* w_gate;   /* [ffn, hidden] */
    const uint8_t* w_up;     /* [ffn, hidden] */
    const uint8_t* w_down;   /* [hidden, ffn] */
    uint16_t* k_cache;       /* [nkv, max_ctx, hd] fp16 bits */
    uint16_t* v_cache;
} orc_layer;

/* One transformer layer of the decode step at position pos (attends to 0..pos).
 * Updates h (fp32[hidden]) in place and writes k, v at pos into the caches. */
int orc_decode_layer(const orc_dims* D, const orc_layer* L, float* h, int32_t pos);

/* Embedding: h = dequant(row `token` of E [vocab, hidden]). */
int orc_embed(int qtype, const uint8_t* E, int64_t hidden, int32_t token, float* h);

/* Final RMSNorm + LM head: logits = W_out . rmsnorm(h). */
int orc_lm_head(int qtype, const float* out_norm, const uint8_t* W_out, int64_t vocab, int64_t hidden,
                float eps, const float* h, float* logits);

void orc_set_threads(int n);
int orc_get_threads(void);

#ifdef __cplusplus
}
#endif

#endif
