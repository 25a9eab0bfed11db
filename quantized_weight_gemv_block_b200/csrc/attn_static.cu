// attn_static.cu - decode attention whose scratch is a fixed device array owned
// by this library, for callers that cannot allocate device memory themselves.
//
// The split partials of the attention kernel normally live in a workspace the
// caller allocates.  Here they live in g_attn_scratch, a
// file-scope device array of kStaticScratchBytes that exists on every GPU that
// loads the library, for as long as the process runs.  In host code the array's
// name only stands for the symbol; its device address is looked up once per
// device with cudaGetSymbolAddress and cached.
#include <mutex>

#include "ops.h"

namespace ntx {
namespace {

constexpr size_t kStaticScratchBytes = size_t(512) << 10;   // 512 KiB per device

static __device__ __align__(256) uint8_t g_attn_scratch[kStaticScratchBytes];

std::mutex g_scratch_mu;
void* g_scratch_ptr[64] = {};

// Device address of g_attn_scratch on the current device (looked up on first use).
ntx_status static_scratch(void** out)
{
    int dev = 0;
    NTX_CUDA_TRY(cudaGetDevice(&dev));
    if (dev < 0 || dev >= 64) return fail(NTX_EUNSUPPORTED, "ntx_attn_decode_noalloc: device index above 63");
    std::lock_guard<std::mutex> lock(g_scratch_mu);
    if (!g_scratch_ptr[dev]) {
        void* p = nullptr;
        const cudaError_t e = cudaGetSymbolAddress(&p, g_attn_scratch);
        if (e != cudaSuccess || !p)
            return fail(NTX_ECUDA, std::string("ntx_attn_decode_noalloc: scratch address lookup: ") +
                                       cudaGetErrorString(e));
        g_scratch_ptr[dev] = p;
    }
    *out = g_scratch_ptr[dev];
    return NTX_OK;
}

}  // namespace
}  // namespace ntx

using namespace ntx;

NTX_EXPORT ntx_status ntx_attn_decode_noalloc(const float* q, const void* k_cache, const void* v_cache, float* out,
                                              int n_q_heads, int n_kv_heads, int head_dim, int32_t n_ctx,
                                              int32_t max_ctx, void* stream)
{
    ntx_status st = attn_check(q, k_cache, v_cache, out, n_q_heads, n_kv_heads, head_dim, n_ctx, max_ctx,
                               "ntx_attn_decode_noalloc");
    if (st != NTX_OK) return st;
    const int n_split = attn_split_for(n_q_heads, n_kv_heads, max_ctx);
    const size_t need = attn_workspace_bytes_for(n_q_heads, n_kv_heads, head_dim, n_split);
    if (need > kStaticScratchBytes)
        return fail(NTX_EUNSUPPORTED, "ntx_attn_decode_noalloc: this shape needs " + std::to_string(need) +
                                          " bytes of scratch, more than the fixed 512 KiB; use ntx_attn_decode");
    void* ws = nullptr;
    if ((st = static_scratch(&ws)) != NTX_OK) return st;
    cudaStream_t s = (cudaStream_t)stream;
    // nothing in the scratch carries over between calls: every split's partial is
    // written before the merge reads it, so it needs no clearing
    AttnArgs a{};
    a.q = q;
    a.k_cache = (const __half*)k_cache;
    a.v_cache = (const __half*)v_cache;
    a.out = out;
    a.n_q_heads = n_q_heads;
    a.n_kv_heads = n_kv_heads;
    a.head_dim = head_dim;
    a.max_ctx = max_ctx;
    a.n_ctx = n_ctx;
    a.pos_dev = nullptr;
    a.workspace = ws;
    a.n_split = n_split;
    a.pdl = false;
    return attn_launch(a, s);
}
