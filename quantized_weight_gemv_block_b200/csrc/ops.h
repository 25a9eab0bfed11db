// ops.h - internal launchers shared by the op, attention and decode-step files.
#pragma once

#include "common.cuh"
#include "gemv.cuh"

namespace ntx {

ntx_status embed_launch(int qtype, const void* E, int64_t hidden, const int32_t* token_dev, float* h, cudaStream_t s,
                        bool pdl);
// Writes the step word (token, pos) and, if rope is not null, the RoPE table of pos
// ([head_dim / 2][cos, sin] floats) for the kernels of the step; the token is read from
// device memory (token_dev) when that is not null.
ntx_status set_step_launch(int32_t* step, int32_t token, int32_t pos, float* rope, float theta, int head_dim,
                           cudaStream_t s, const int32_t* token_dev = nullptr);
ntx_status gemv_launch(int qtype, int epi, int pro, const gemv::Params& P, cudaStream_t s);
// y_v = W x_v for nx = 2..4 vectors (tiled formats; qmma_multi.cu), each weight streamed once;
// NTX_EUNSUPPORTED, with nothing launched, when the format or the shape does not allow it.
ntx_status gemv_multi_launch(int qtype, int epi, int pro, const gemv::Params& P, const gemv::Vecs& V, int nx,
                             cudaStream_t s);
// *out_index = the lowest index of the largest x (n <= 2^26), one CTA.
ntx_status argmax_launch(const float* x, int64_t n, int32_t* out_index, cudaStream_t s);
// *out = a . b / (|a| |b|) for device fp32 vectors of n <= 2^26 elements (0 if either is zero).
ntx_status cosine_launch(const float* a, const float* b, int64_t n, float* out, cudaStream_t s);
ntx_status qmma_launch(int qtype, int epi, int pro, const gemv::Params& P, cudaStream_t s);
// F16 / F32 weights (fgemv.cu): the streaming kernel needs W and x 16-byte aligned,
// rows that are 16-byte multiples and at most 32768 columns.
bool fgemv_shape_ok(int qtype, const void* W, const void* x, int64_t cols);
ntx_status fgemv_launch(int qtype, int epi, int pro, const gemv::Params& P, cudaStream_t s);
ntx_status repack_launch(int qtype, const void* W, void* W_tiled, int64_t rows, int64_t cols, cudaStream_t s);
bool gemv_fast_path_ok(int qtype, const void* W, int64_t cols);

// Split-KV decode attention (attn.cu).

// An L2 prefetch of K / V rows that a later kernel will read (a hint: it changes no result):
// rows [0, pos) of the n_kv heads of one layer's caches, K at k, V at v, head h at
// h * head_stride bytes, row_b bytes per position.
struct KvPrefetch {
    const uint8_t* k;
    const uint8_t* v;
    int64_t head_stride;
    int n_kv, row_b;
};

struct AttnArgs {
    const float* q;
    const __half* k_cache;
    const __half* v_cache;
    float* out;
    int n_q_heads, n_kv_heads, head_dim, max_ctx;
    int32_t n_ctx;              // used when n_ctx_from_pos is null
    const int32_t* pos_dev;     // if set: n_ctx = *pos_dev + 1 (read on the device)
    void* workspace;            // split partials (no initialisation needed)
    int n_split;                // CTAs per kv head
    bool pdl;
    KvPrefetch pf;              // rows of another layer to fetch into L2 once the copies are
                                // under way (the step's next layer; k null: none)
};
ntx_status attn_check(const void* q, const void* k_cache, const void* v_cache, const void* out, int n_q_heads,
                      int n_kv_heads, int head_dim, int32_t n_ctx, int32_t max_ctx, const char* who);
int attn_split_for(int n_q_heads, int n_kv_heads, int32_t max_ctx);
size_t attn_workspace_bytes_for(int n_q_heads, int n_kv_heads, int head_dim, int n_split);
ntx_status attn_launch(const AttnArgs& a, cudaStream_t s);

}  // namespace ntx
