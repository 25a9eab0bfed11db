/*
 * ntx.h - C ABI of the B200 (sm_100a) batch-1 quantized decode library (libntx.so).
 *
 * Source of the operations: the ntransformer news summary (news.hada.io topic
 * 26894).  "Descripción general de NTransformer" lists the GGUF weight formats
 * (Q4_0, Q8_0, Q4_K_M, Q6_K, ...); "Arquitectura y estructura del código" lists the
 * CUDA kernels (GEMV, RMSNorm, RoPE, SwiGLU, softmax) and the model pieces
 * (attention, FFN, normalization); "Funciones principales" names the Llama
 * architecture pieces (RoPE, GQA, SwiGLU, RMSNorm, KV cache) and the SLEP
 * double-buffered streaming; "Hoja de ruta de desarrollo" gives the F16 KV cache
 * (Fase 3) and the planned public C API (Fase 5).  The pages print no formula,
 * layout or signature; the readings used are stated per function below.
 *
 * Conventions (every function):
 *  - returns ntx_status; NTX_OK = 0.  A failing call sets a thread-local message
 *    readable with ntx_last_error().  Nothing aborts or throws across the ABI.
 *  - arguments are checked on the host before anything is launched; a rejected
 *    call launches nothing.
 *  - device pointers are owned by the caller (the library never frees them) and
 *    must stay valid until the work queued on the stream has finished.
 *  - work is queued asynchronously on the caller's stream (`stream`, a
 *    cudaStream_t passed as void*; NULL = legacy default stream).  Launch errors
 *    are returned as NTX_ECUDA; errors raised while kernels run surface at the
 *    caller's next synchronisation.  Kernels that wait on a barrier give up
 *    after a bounded time and record a code readable with ntx_device_error().
 *  - packed weights are row-major: row r occupies ntx_row_bytes(qtype, cols)
 *    bytes starting at W + r * ntx_row_bytes(qtype, cols); inside a row, blocks
 *    follow one another in the GGUF-style layouts below.
 *
 * Block layouts (little-endian; one block covers consecutive elements of a row):
 *   NTX_Q8_0  34 B / 32:  fp16 d | 32 x int8 q                w = d q
 *   NTX_Q4_0  18 B / 32:  fp16 d | 16 B; byte j: element j in the low nibble,
 *                         element j+16 in the high nibble     w = d (q - 8)
 *   NTX_Q4_K 144 B / 256: fp16 d | fp16 dmin | 12 B of 6-bit scales and mins |
 *                         128 B of 4-bit codes                w = d sc_j q - dmin m_j
 *                         (j = element / 32; code byte 32c+l holds element 64c+l in
 *                         its low nibble and 64c+32+l in its high nibble; scales /
 *                         mins of sub-blocks 0..3 in the low 6 bits of bytes 0..3 /
 *                         4..7, sub-blocks 4..7 split between bytes 8..11 (low 4
 *                         bits) and the top 2 bits of bytes 0..7)
 *   NTX_Q6_K 210 B / 256: 128 B low code bits | 64 B high code bits | 16 x int8
 *                         scales | fp16 d                     w = d sc_j (q - 32)
 *                         (j = element / 16; element e, t = e % 128, h = e / 128:
 *                         low 4 bits from ql[64h + t % 64], low nibble if t < 64
 *                         else high nibble; high 2 bits = bits 2 (t / 32) of
 *                         qh[32h + t % 32])
 */
#ifndef NTX_H
#define NTX_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum ntx_status {
    NTX_OK = 0,
    NTX_EINVAL = 1,        /* bad argument (null pointer, bad size, misalignment, range) */
    NTX_EUNSUPPORTED = 2,  /* valid but not supported (format, shape) */
    NTX_ENOMEM = 3,        /* library-owned allocation failed */
    NTX_ECUDA = 4,         /* a CUDA runtime call failed; see ntx_last_error() */
    NTX_ETIMEOUT = 5       /* a bounded wait ran out */
} ntx_status;

typedef enum ntx_qtype {
    NTX_Q8_0 = 0,
    NTX_Q4_0 = 1,
    NTX_Q4_K = 2,
    NTX_Q6_K = 3,
    /* Q5_K 176 B / 256: fp16 d | fp16 dmin | 12 B of 6-bit scales and mins packed as in
     * Q4_K | 32 B of fifth code bits | 128 B of low 4-bit codes    w = d sc_j q - dmin m_j
     * (q in 0..31, j = element / 32; element 64c + l and 64c + 32 + l, l < 32, take the
     * low and high nibble of low-code byte 32c + l and bits 2c and 2c + 1 of fifth-bit
     * byte l).  F16 / F32: one little-endian IEEE value per weight. */
    NTX_Q5_K = 4,
    NTX_F16 = 5,
    NTX_F32 = 6,
    /* Tiled layouts (flag NTX_TILED): the same information in the same bytes per
     * row, reordered for the streaming GEMV.  Produced from the GGUF-style
     * layout by ntx_repack_q, lossless.  Rows come in groups of 16 (a tiled
     * tensor has a multiple of 16 rows); a group is a run of units along the
     * row, unit u covering columns [u UK, (u + 1) UK) of the group's 16 rows in
     * 16 x the GGUF-style bytes of UK columns (UK = 32 for Q8_0 / Q4_0: one
     * block; 256 for Q4_K / Q6_K: one superblock).  Inside a unit the codes of
     * each 32-column step sit in "lane" order: lane 4 gid + tig holds rows gid
     * and gid + 8 at columns 4 tig .. 4 tig + 3 and 16 + 4 tig .. 16 + 4 tig + 3
     * (the A fragment of an m16n8k32 integer MMA; the four lanes of a gid are
     * adjacent, so one gid's two rows over the whole step are contiguous bytes),
     * followed by the unit's scales:
     *   NTX_Q8_0_T  unit 544 B: 32 lanes x 16 int8 codes | 8 x (d[r], d[r+8])
     *   NTX_Q4_0_T  unit 288 B: 32 lanes x 8 B (two 4-bit codes per byte) | 8 x (d[r], d[r+8])
     *   NTX_Q6_K_T  unit 3360 B: 8 steps x 32 lanes x 12 B (four 6-bit codes per 3
     *               bytes) | 256 B int8 sub-block scales | 8 x (d[r], d[r+8])
     *   NTX_Q4_K_T  unit 2304 B: 8 steps x 32 lanes x 8 B | 8 x 24 B of 6-bit scales
     *               and mins | 8 x (d[r], d[r+8], dmin[r], dmin[r+8])
     *   NTX_Q5_K_T  unit 2816 B: 8 steps x (32 lanes x 8 B of low 4 bits as Q4_K | 8 gids x
     *               8 B of fifth bits: word H0 row gid, H1 row gid + 8, the bit of column
     *               4 tig + j at 8 j + 2 tig, of column 16 + 4 tig + j at 8 j + 2 tig + 1) |
     *               scales, mins, d and dmin as NTX_Q4_K_T
     * A row of a tiled tensor must hold whole units.  F16 and F32 have no tiled form. */
    NTX_TILED = 16,
    NTX_Q8_0_T = 16,
    NTX_Q4_0_T = 17,
    NTX_Q4_K_T = 18,
    NTX_Q6_K_T = 19,
    NTX_Q5_K_T = 20
} ntx_qtype;

/* Message of the last failing ntx_* call on this thread ("" if none). */
const char* ntx_last_error(void);

/* Library version as major * 10000 + minor * 100 + patch. */
int ntx_version(void);

/* Bytes of one packed row of `cols` elements; 0 if qtype is unknown or cols is
 * not a positive multiple of the format's block size (32 or 256).  Tiled and
 * GGUF-style rows have the same length. */
size_t ntx_row_bytes(int qtype, int64_t cols);

/* Elements per block of qtype (32 or 256), 0 if unknown. */
int ntx_block_elems(int qtype);

/* Error code recorded by a kernel on the current device (0 = none), and reset
 * it: bit 0 a consumer's wait for a filled stage ran out, bit 1 a producer's
 * wait for a drained stage, bit 2 a producer's final drain, bit 3 shared memory
 * was not aligned as the copies need (the kernel did nothing).  Bits of several
 * kernels are OR-ed.  Synchronises the current device. */
ntx_status ntx_device_error(uint32_t* code);

/* ---------------------------------------------------------------- quantized GEMV
 * y = W x: y[r] = sum_k dequant(W)[r, k] * x[k] for r < rows, k < cols
 * (the GEMV kernel of "Arquitectura y estructura del código"; batch 1).
 *   W    device, packed [rows, cols] in `qtype`; 16-byte aligned
 *   x    device fp32 [cols];  y  device fp32 [rows] (must not overlap x or W)
 * Accumulation is fp32; results match the exact dot product to a normwise
 * relative error far below 2e-3.  rows >= 1 (a multiple of 16 for a tiled
 * qtype); cols a multiple of the block size.  Tiled layouts take integer dots
 * of the codes with x as 24-bit fixed point (relative to max |x|) by dp4a on the
 * CUDA cores (NTX_GEMV_CORE=tc selects integer MMAs instead; same results up to
 * fp32 rounding order); GGUF-style rows whose byte length is a multiple of 16
 * take the bulk-copy fp32 CUDA-core pipeline; other shapes a simpler kernel.
 * The two pipelines launch as programmatic dependents: when the previous kernel
 * on the stream is one of this library's, they start streaming W before it has
 * finished (x is read and y written only after it completed), so W must not be
 * written by that previous kernel (no kernel of this library writes weights). */
ntx_status ntx_gemv_q(int qtype, const void* W, int64_t rows, int64_t cols, const float* x, float* y,
                      void* stream);

/* Measurement helper, not part of the decode path: streams `bytes` bytes of src
 * (device, 16-byte aligned, a multiple of 16 bytes) from HBM into shared memory the
 * way the tiled GEMV streams its weights (one CTA per SM, 1-D bulk copies, L2
 * evict-first, a ring of 24 KB stages) and does nothing else; its bytes per second
 * are the practical ceiling of the GEMV's data path.  Asynchronous on `stream`. */
ntx_status ntx_stream_read_probe(const void* src, size_t bytes, void* stream);

/* Repack W [rows, cols] from the GGUF-style layout of `qtype` (NTX_Q8_0 ..
 * NTX_Q6_K) into the tiled layout qtype | NTX_TILED, device to device: W_tiled
 * receives rows * ntx_row_bytes(qtype, cols) bytes and must not overlap W.
 * rows must be a multiple of 16.  A lossless reordering of the bits. */
ntx_status ntx_repack_q(int qtype, const void* W, void* W_tiled, int64_t rows, int64_t cols, void* stream);

/* Dequantize W [rows, cols] to fp32 out [rows, cols] (row-major).  The result
 * is bit-exact: every weight is one fp32 product of exact factors (Q4_K: one
 * rounding of d sc q - dmin m). */
ntx_status ntx_dequant_q(int qtype, const void* W, int64_t rows, int64_t cols, float* out, void* stream);

/* ------------------------------------------------------------------ decode ops */

/* RMSNorm (listed in "Arquitectura y estructura del código"):
 * y_i = x_i / sqrt(mean(x^2) + eps) * w_i, fp32, n >= 1.  x, w, y device fp32 [n];
 * y may equal x. */
ntx_status ntx_rmsnorm(const float* x, const float* w, float* y, int64_t n, float eps, void* stream);

/* RoPE on adjacent pairs (2i, 2i+1) of every head of q [n_q_heads, head_dim] and
 * k [n_kv_heads, head_dim], in place: rotation by pos * theta^(-2i/head_dim),
 * the angle and its sine / cosine evaluated in double.  k may be NULL
 * (n_kv_heads ignored).  head_dim even, pos >= 0. */
ntx_status ntx_rope(float* q, float* k, int n_q_heads, int n_kv_heads, int head_dim, int32_t pos, float theta,
                    void* stream);

/* GQA decode attention of one query token (attention with GQA of "Funciones
 * principales", F16 KV cache of "Hoja de ruta de desarrollo" Fase 3):
 * q head h reads kv head g = h / (n_q_heads / n_kv_heads);
 * out_h = sum_t softmax_t(q_h . K[g][t] / sqrt(head_dim)) V[g][t], t < n_ctx.
 *   q       device fp32 [n_q_heads, head_dim]
 *   k_cache, v_cache  device fp16 [n_kv_heads, max_ctx, head_dim]
 *   out     device fp32 [n_q_heads, head_dim]
 *   workspace / workspace_bytes: device scratch of at least
 *           ntx_attn_workspace_bytes(...) bytes, 16-byte aligned, for the partial
 *           results of the context splits; it needs no initialisation.
 * Two kernels run on `stream`: the split kernel, then the merge of the splits.
 * head_dim == 128, n_q_heads a multiple of n_kv_heads with at most 8 q heads per
 * kv head, 1 <= n_ctx <= max_ctx.  Calls sharing a workspace must not overlap. */
ntx_status ntx_attn_decode(const float* q, const void* k_cache, const void* v_cache, float* out, int n_q_heads,
                           int n_kv_heads, int head_dim, int32_t n_ctx, int32_t max_ctx, void* workspace,
                           size_t workspace_bytes, void* stream);
size_t ntx_attn_workspace_bytes(int n_q_heads, int n_kv_heads, int head_dim, int32_t max_ctx);

/* The same attention as ntx_attn_decode, for callers that cannot allocate device
 * memory: code that runs under a fixed, pre-planned memory budget or inside a
 * host framework whose allocator hands out no scratch, and so has no workspace
 * to pass.  (The pages have no counterpart; this is an addition of this library.)
 * The split partials live in a device array of 512 KiB that the
 * library holds on every GPU that loads it, until the process exits.  Shapes
 * whose workspace (ntx_attn_workspace_bytes) exceeds 512 KiB are rejected with
 * NTX_EUNSUPPORTED (on a 148-SM B200: 8 q heads per kv head with 8 kv heads, as
 * in Llama-70B, needs about 600 KB; 4 per kv head, as in Llama-8B, about 300 KB).  Nothing is allocated: the first call on a device looks up
 * the array's device address (cudaGetSymbolAddress) and caches it, so make that
 * first call before any stream capture.  All calls share the one array, so calls
 * whose work overlaps on the GPU (different streams, or another thread) race:
 * serialise them.  Arguments, layouts and errors as for ntx_attn_decode. */
ntx_status ntx_attn_decode_noalloc(const float* q, const void* k_cache, const void* v_cache, float* out,
                                   int n_q_heads, int n_kv_heads, int head_dim, int32_t n_ctx, int32_t max_ctx,
                                   void* stream);

/* SwiGLU (listed in "Arquitectura y estructura del código"):
 * out_i = gate_i / (1 + e^-gate_i) * up_i, fp32 [n]. */
ntx_status ntx_swiglu(const float* gate, const float* up, float* out, int64_t n, void* stream);

/* softmax (listed in "Arquitectura y estructura del código") over one row:
 * y_i = e^(x_i - max x) / sum_j e^(x_j - max x), fp32 [n], 1 <= n <= 2^26. */
ntx_status ntx_softmax(const float* x, float* y, int64_t n, void* stream);

/* Greedy token pick: *out_index = argmax_i x_i (lowest index among ties), device
 * int32 output; n <= 2^26. */
ntx_status ntx_argmax(const float* x, int64_t n, int32_t* out_index, void* stream);

/* Embedding lookup: h = dequant(row `token` of E [vocab, hidden]); token is read
 * from device memory (`token_dev`, int32) so the call can be replayed. */
ntx_status ntx_embed(int qtype, const void* E, int64_t vocab, int64_t hidden, const int32_t* token_dev, float* h,
                     void* stream);

/* ------------------------------------------------------------------ decode step
 * A Llama-architecture model ("Funciones principales"; model/ of "Arquitectura y
 * estructura del código") with per-layer packed weights.  One call runs one
 * batch-1 decode step: embedding, then per layer
 *   xn = RMSNorm(h); [q|k|v] = W_qkv xn; RoPE(q, k, pos); K[pos] = fp16(k),
 *   V[pos] = fp16(v); a = attention over positions 0..pos; h += W_o a;
 *   xn = RMSNorm(h); h += W_down (silu(W_gate xn) * (W_up xn)),
 * then logits = W_out RMSNorm(h). */
typedef struct ntx_layer_desc {
    const float* attn_norm;   /* device fp32 [hidden] */
    const void* w_qkv;        /* packed [(n_q + 2 n_kv) * head_dim, hidden]: q rows, k rows, v rows */
    const void* w_o;          /* packed [hidden, n_q * head_dim] */
    const float* ffn_norm;    /* device fp32 [hidden] */
    const void* w_gate;       /* packed [ffn, hidden] */
    const void* w_up;         /* packed [ffn, hidden] */
    const void* w_down;       /* packed [hidden, ffn] */
    void* k_cache;            /* device fp16 [n_kv, max_ctx, head_dim] */
    void* v_cache;            /* device fp16 [n_kv, max_ctx, head_dim] */
} ntx_layer_desc;

typedef struct ntx_model_desc {
    int32_t n_layers, hidden, n_q_heads, n_kv_heads, head_dim, ffn, vocab, max_ctx;
    float rms_eps, rope_theta;
    int32_t qtype;                 /* format of every packed tensor (unless tensor_qtypes says otherwise) */
    const void* tok_embd;          /* packed [vocab, hidden], device */
    const float* out_norm;         /* device fp32 [hidden] */
    const void* output;            /* packed [vocab, hidden], device */
    const ntx_layer_desc* layers;  /* host array [n_layers], copied by ntx_model_create */
    /* Layer streaming ("Streaming SLEP" of "Funciones principales"): layers
     * [n_resident, n_layers) hold their five packed weight pointers in pinned host
     * memory and are copied each step through a two-slot HBM ring by
     * ntx_stream_layers.  Norm weights and KV caches of every layer stay in HBM.
     * n_resident == n_layers: fully resident model. */
    int32_t n_resident;
    /* Per-tensor formats, for models that mix formats (the "Q4_K_M" models of
     * "Rendimiento y estructura de caché", e.g. most matrices Q4_K and some Q6_K):
     * NULL (every tensor in qtype), or a host array of 2 + 4 n_layers formats, copied
     * by ntx_model_create: tok_embd, output, then per layer w_qkv, w_o, w_gate and w_up
     * (one format for both), w_down.  Any format of ntx_qtype; GGUF-style Q5_K rows have
     * no streaming kernel, so a Q5_K matrix is given in its tiled form NTX_Q5_K_T. */
    const int32_t* tensor_qtypes;
} ntx_model_desc;

typedef struct ntx_model ntx_model;

/* Automatic tier split ("Rendimiento y estructura de caché": as many layers as fit stay
 * in VRAM, the rest are streamed from host memory each token).  From the descriptor's
 * shapes and formats alone (no pointer is read; it may be a planning copy with null
 * pointers), the largest n_resident such that everything the model keeps in HBM fits
 * in hbm_budget bytes: the embedding and LM-head matrices, the norm weights, the KV
 * caches of every layer, the matrices of layers [0, n_resident), the two-slot ring for
 * the others (when n_resident < n_layers: each slot holds the largest of each matrix
 * over the streamed layers), and the model's own scratch.  *hbm_used receives that
 * total (may be NULL).  NTX_ENOMEM if even n_resident = 0 does not fit.  Host only: it
 * launches nothing.  Place layers [0, *n_resident) in device memory and the others in
 * host memory, and set desc.n_resident to it. */
ntx_status ntx_plan_resident(const ntx_model_desc* desc, size_t hbm_budget, int32_t* n_resident, size_t* hbm_used);

/* How the streamed layers' matrices are copied (decided by ntx_model_create, the data-path
 * selection of "Funciones principales"): page-locked host memory is copied by DMA as it
 * is; other host memory is page-locked in place (cudaHostRegister, undone by
 * ntx_model_destroy) unless the environment variable NTX_NO_HOST_REGISTER is set or the
 * system refuses, and is otherwise copied from pageable memory (the driver stages each
 * copy and the host waits for it, so copy and compute overlap less).  The model's path is
 * the slowest any streamed matrix takes.  Streamed matrices in device memory are
 * rejected by ntx_model_create. */
enum { NTX_HOST_PATH_NONE = 0, NTX_HOST_PATH_PINNED = 1, NTX_HOST_PATH_REGISTERED = 2, NTX_HOST_PATH_PAGEABLE = 3 };
ntx_status ntx_model_host_path(ntx_model* model, int32_t* path);

/* Validate the descriptor and allocate the model's scratch (activations,
 * attention partials, and the HBM ring when n_resident < n_layers).  The model
 * must be used on the device that was current at creation. */
ntx_status ntx_model_create(const ntx_model_desc* desc, ntx_model** model);
ntx_status ntx_model_destroy(ntx_model* model);

/* One decode step of a fully resident model: token at position pos (attends to
 * 0..pos, writes K/V at pos), logits device fp32 [vocab].  0 <= pos < max_ctx,
 * 0 <= token < vocab.  Queued on `stream`.  The first call on a stream records a
 * CUDA graph of the step that later calls replay. */
ntx_status ntx_decode_step(ntx_model* model, int32_t token, int32_t pos, float* logits, void* stream);

/* One decode step of a partly resident model: resident layers on `compute`,
 * streamed layers copied host -> HBM ring on `copy` (cudaMemcpyAsync, one slot
 * ahead) and computed on `compute` once their copy event has fired.  Returns
 * after queueing if timeout_ms == 0; otherwise waits up to timeout_ms for the
 * step to finish and returns NTX_ETIMEOUT if it has not (work stays queued). */
ntx_status ntx_stream_layers(ntx_model* model, int32_t token, int32_t pos, float* logits, void* compute,
                             void* copy, int64_t timeout_ms);

/* Measurement helper, not part of the decode path: enqueue `n_launches` launches of
 * one kind of the step's fused GEMVs on `stream`, exactly as ntx_decode_step issues
 * them (same kernels, prologues, epilogues and launch attributes), cycling over the
 * resident layers 0, 1, ... so consecutive launches read different weights:
 *   NTX_GEMV_QKV      RMSNorm prologue, RoPE and fp16 K/V append at the step's position
 *   NTX_GEMV_O        residual add into the hidden state
 *   NTX_GEMV_GATE_UP  RMSNorm prologue, gate and up rows streamed together, SwiGLU
 *   NTX_GEMV_DOWN     residual add into the hidden state
 *   NTX_GEMV_HEAD     final RMSNorm prologue, logits into `logits` (device fp32 [vocab];
 *                     unused by the other kinds, may be NULL there)
 * Inputs are the model's activation buffers as the last step left them; outputs
 * overwrite them (and the KV rows at the last step's position), so run a decode step
 * again before relying on its results.  The launches may be captured in a CUDA graph. */
enum { NTX_GEMV_QKV = 0, NTX_GEMV_O = 1, NTX_GEMV_GATE_UP = 2, NTX_GEMV_DOWN = 3, NTX_GEMV_HEAD = 4 };
ntx_status ntx_model_replay_gemv(ntx_model* model, int kind, int n_launches, float* logits, void* stream);

/* Layer skip ("Rendimiento y estructura de caché": layers whose hidden states barely
 * change, judged by cosine similarity, are left out; 20 of 80 on the pages' 70B run).
 *
 * ntx_model_layer_similarity runs one decode step of token at pos with every layer (the
 * skip mask ignored; the LM head is not run) and writes, for each layer l, the cosine
 * similarity of the hidden state before and after it, cos_out[l] = h_in . h_out /
 * (|h_in| |h_out|), to the host array cos_out [n_layers]; it returns once they are there.
 * Like a step, it writes the K / V rows at pos.  Streamed models need distinct compute and
 * copy streams (copy is unused otherwise).
 *
 * ntx_model_set_layer_skip sets the layers the decode step leaves out: skip is a host
 * array [n_layers], nonzero = skip (NULL clears the mask).  A skipped layer is neither
 * computed nor, if streamed, copied, and writes no K / V rows (its cache is never read
 * while it stays skipped).  The next ntx_decode_step records its CUDA graph again.  Which
 * layers to skip is the caller's choice, e.g. the k layers of highest similarity. */
ntx_status ntx_model_layer_similarity(ntx_model* model, int32_t token, int32_t pos, float* cos_out, void* compute,
                                      void* copy);
ntx_status ntx_model_set_layer_skip(ntx_model* model, const uint8_t* skip);

/* Self-speculative decoding ("Funciones principales": the layers resident in VRAM act as
 * the draft model and the full model verifies several drafted tokens in one pass, so each
 * streamed layer crosses the host link once for all of them; "Hoja de ruta de
 * desarrollo").
 *
 * ntx_verify_tokens: one pass of the model as ntx_decode_step / ntx_stream_layers run it
 * (skip mask included) over n tokens (host array, 1 <= n <= 8) at positions pos0 ..
 * pos0 + n - 1.  Token i attends to positions 0 .. pos0 + i, including the K / V rows the
 * earlier tokens of the pass write; its logits go to logits + i vocab (device fp32
 * [n, vocab]).  Every layer runs for all n tokens before the next, so a streamed layer is
 * copied once per pass, and each fused GEMV of the layer (and the LM head) runs once for up
 * to 4 tokens, streaming its weights once for all of them (tiled formats whose x vectors
 * fit in shared memory; otherwise, and with NTX_VERIFY_PER_TOKEN=1 in the environment, one
 * launch per token).  Per token the arithmetic is that of a one-token step.  On a fully
 * resident model the pass is recorded as a CUDA graph on first use (per token count and
 * logits buffer; recorded again after ntx_model_set_layer_skip) and replayed, reading the
 * tokens and positions from device memory; so are the draft steps of
 * ntx_speculative_step.  Queued on `compute` (and `copy` for a partly resident model, which
 * must differ); returns after queueing.
 *
 * ntx_speculative_step: from `token` at `pos`, drafts k - 1 tokens (2 <= k <= 8) greedily
 * with the draft model (the resident layers, minus the layers draft_skip marks: host array
 * [n_layers] or NULL), verifies token and drafts with one ntx_verify_tokens pass, and
 * accepts the drafted tokens up to the first one the full model's greedy pick disagrees
 * with, followed by the full model's own pick there.  out_tokens (host [k]) receives those
 * tokens, *n_out their number (1 .. k): exactly the tokens greedy decoding of the full model
 * gives from (token, pos).  The K / V rows at pos .. pos + *n_out - 1 hold the accepted
 * tokens' values; continue from out_tokens[*n_out - 1] at pos + *n_out.  Synchronises with
 * the work it queued (bounded by timeout_ms when > 0: NTX_ETIMEOUT leaves the work queued).
 * Drafting uses greedy picks (argmax, lowest index among ties). */
ntx_status ntx_verify_tokens(ntx_model* model, const int32_t* tokens, int32_t n, int32_t pos0, float* logits,
                             void* compute, void* copy);
ntx_status ntx_speculative_step(ntx_model* model, int32_t token, int32_t pos, int32_t k, const uint8_t* draft_skip,
                                int32_t* out_tokens, int32_t* n_out, void* compute, void* copy, int64_t timeout_ms);

/* Number of kernel launches one ntx_decode_step of this model queues (the step word,
 * the embedding, the layers' kernels, the LM head), for accounting. */
ntx_status ntx_model_step_launches(ntx_model* model, int32_t* launches);

/* Per-step counters of the last ntx_stream_layers call: bytes copied host ->
 * device, and device milliseconds of the whole step (between the step's first
 * and last event; valid once the step finished). */
ntx_status ntx_stream_stats(ntx_model* model, int64_t* h2d_bytes, float* step_ms);

#ifdef __cplusplus
}
#endif

#endif /* NTX_H */
