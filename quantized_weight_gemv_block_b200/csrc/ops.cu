// ops.cu - the small decode ops of the ntransformer news summary's kernel list
// ("Arquitectura y estructura del código": RMSNorm, RoPE, SwiGLU, softmax) as
// standalone kernels, plus the embedding lookup and a greedy argmax.  Inside the
// decode step RMSNorm, RoPE and SwiGLU run fused into the GEMV kernels; these
// standalone forms serve callers composing their own step and the tests.
#include <algorithm>

#include "blocks.cuh"
#include "ops.h"

namespace ntx {
namespace {

constexpr int kBlock = 1024;

__device__ __forceinline__ float block_sum(float v, float* red)
{
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
    v = gemv::warp_sum(v);
    __syncthreads();
    if (lane == 0) red[warp] = v;
    __syncthreads();
    float r = 0.f;
    for (int w = 0; w < nw; ++w) r += red[w];
    return r;
}

__device__ __forceinline__ float block_max(float v, float* red)
{
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
    v = gemv::warp_max(v);
    __syncthreads();
    if (lane == 0) red[warp] = v;
    __syncthreads();
    float r = -INFINITY;
    for (int w = 0; w < nw; ++w) r = fmaxf(r, red[w]);
    return r;
}

__global__ void rmsnorm_kernel(const float* x, const float* w, float* y, int64_t n, float eps)
{
    __shared__ float red[32];
    float ss = 0.f;
    for (int64_t i = threadIdx.x; i < n; i += blockDim.x) ss = fmaf(x[i], x[i], ss);
    ss = block_sum(ss, red);
    const float inv = 1.0f / sqrtf(ss / (float)n + eps);
    __syncthreads();
    for (int64_t i = threadIdx.x; i < n; i += blockDim.x) y[i] = x[i] * inv * w[i];
}

// One thread per pair; the angle pos * theta^(-2i/d) and its sine / cosine in double.
__global__ void rope_kernel(float* q, float* k, int nq, int nkv, int hd, int32_t pos, float theta)
{
    const int half = hd / 2;
    const int total = (nq + nkv) * half;
    for (int idx = blockIdx.x * blockDim.x + threadIdx.x; idx < total; idx += gridDim.x * blockDim.x) {
        const int head = idx / half, i = idx % half;
        float* v = head < nq ? q + (int64_t)head * hd : k + (int64_t)(head - nq) * hd;
        const double ang = (double)pos * pow((double)theta, -(2.0 * i) / (double)hd);
        double s, c;
        sincos(ang, &s, &c);
        const float cf = (float)c, sf = (float)s;
        const float a = v[2 * i], b = v[2 * i + 1];
        v[2 * i] = a * cf - b * sf;
        v[2 * i + 1] = a * sf + b * cf;
    }
}

__global__ void swiglu_kernel(const float* g, const float* u, float* out, int64_t n)
{
    for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x) {
        const float gv = g[i];
        out[i] = gv / (1.0f + expf(-gv)) * u[i];
    }
}

__global__ void softmax_kernel(const float* x, float* y, int64_t n)
{
    __shared__ float red[32];
    float mx = -INFINITY;
    for (int64_t i = threadIdx.x; i < n; i += blockDim.x) mx = fmaxf(mx, x[i]);
    mx = block_max(mx, red);
    float s = 0.f;
    for (int64_t i = threadIdx.x; i < n; i += blockDim.x) s += expf(x[i] - mx);
    s = block_sum(s, red);
    const float inv = 1.0f / s;
    for (int64_t i = threadIdx.x; i < n; i += blockDim.x) y[i] = expf(x[i] - mx) * inv;
}

__global__ void argmax_kernel(const float* x, int64_t n, int32_t* out)
{
    __shared__ float bv[32];
    __shared__ int32_t bi[32];
    float best = -INFINITY;
    int32_t idx = INT32_MAX;
    for (int64_t i = threadIdx.x; i < n; i += blockDim.x) {
        const float v = x[i];
        if (v > best || (v == best && (int32_t)i < idx)) {
            best = v;
            idx = (int32_t)i;
        }
    }
    for (int o = 16; o > 0; o >>= 1) {
        const float ov = __shfl_xor_sync(0xffffffffu, best, o);
        const int32_t oi = __shfl_xor_sync(0xffffffffu, idx, o);
        if (ov > best || (ov == best && oi < idx)) {
            best = ov;
            idx = oi;
        }
    }
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    if (lane == 0) {
        bv[warp] = best;
        bi[warp] = idx;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        for (int w = 1; w < (int)(blockDim.x >> 5); ++w)
            if (bv[w] > best || (bv[w] == best && bi[w] < idx)) {
                best = bv[w];
                idx = bi[w];
            }
        *out = idx == INT32_MAX ? 0 : idx;
    }
}

template <int QT>
__global__ void embed_kernel(const uint8_t* E, int64_t rb, int64_t hidden, const int32_t* token_dev, float* h,
                             int use_pdl)
{
    if (use_pdl) {
        pdl_launch_dependents();
        pdl_wait();
    }
    const int32_t token = *token_dev;
    for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < hidden; i += (int64_t)gridDim.x * blockDim.x)
        h[i] = gemv::weight_at<QT>(E, token, i, rb);
}

// The step word (token, position) and the RoPE table of the position: rope[2i] and
// rope[2i + 1] = cos and sin of pos theta^(-2i/head_dim), computed in double, for
// i < head_dim / 2 (the rotation of "RoPE" in the ntransformer news summary's kernel
// list).  Later kernels of the step read both.
__global__ void set_step_kernel(int32_t* step, int32_t token, const int32_t* token_dev, int32_t pos, float* rope,
                                float theta, int head_dim)
{
    const int i = threadIdx.x;
    if (i == 0) {
        step[0] = token_dev ? *token_dev : token;
        step[1] = pos;
    }
    if (rope && i < head_dim / 2) {
        const double ang = (double)pos * pow((double)theta, -(2.0 * i) / (double)head_dim);
        double sn, cs;
        sincos(ang, &sn, &cs);
        rope[2 * i] = (float)cs;
        rope[2 * i + 1] = (float)sn;
    }
}

// Cosine similarity of two vectors, by one CTA (the similarity of a layer's input and
// output hidden states, the measure the layer skip of "Rendimiento y estructura de
// caché" in the ntransformer news summary ranks layers by); sums in double.
__global__ void cosine_kernel(const float* a, const float* b, int64_t n, float* out)
{
    __shared__ double red[3][32];
    double ab = 0.0, aa = 0.0, bb = 0.0;
    for (int64_t i = threadIdx.x; i < n; i += blockDim.x) {
        const double x = a[i], y = b[i];
        ab += x * y;
        aa += x * x;
        bb += y * y;
    }
    for (int o = 16; o > 0; o >>= 1) {
        ab += __shfl_xor_sync(0xffffffffu, ab, o);
        aa += __shfl_xor_sync(0xffffffffu, aa, o);
        bb += __shfl_xor_sync(0xffffffffu, bb, o);
    }
    const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (lane == 0) {
        red[0][w] = ab;
        red[1][w] = aa;
        red[2][w] = bb;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        double s0 = 0.0, s1 = 0.0, s2 = 0.0;
        for (int k = 0; k < (int)(blockDim.x >> 5); ++k) {
            s0 += red[0][k];
            s1 += red[1][k];
            s2 += red[2][k];
        }
        *out = (s1 > 0.0 && s2 > 0.0) ? (float)(s0 / sqrt(s1 * s2)) : 0.f;
    }
}

}  // namespace

ntx_status cosine_launch(const float* a, const float* b, int64_t n, float* out, cudaStream_t s)
{
    cosine_kernel<<<1, 1024, 0, s>>>(a, b, n, out);
    return check_launch("cosine similarity");
}

ntx_status embed_launch(int qtype, const void* E, int64_t hidden, const int32_t* token_dev, float* h, cudaStream_t s,
                        bool pdl)
{
    const int64_t rb = row_bytes(qtype, hidden);
    const int threads = 256;
    const int grid = (int)std::min<int64_t>((hidden + threads - 1) / threads, 1024);
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(threads);
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = pdl ? 1 : 0;
    const uint8_t* e = (const uint8_t*)E;
    const int p = pdl ? 1 : 0;
    cudaError_t err = cudaErrorInvalidValue;
    switch (qtype) {
    case NTX_Q8_0: err = cudaLaunchKernelEx(&cfg, embed_kernel<NTX_Q8_0>, e, rb, hidden, token_dev, h, p); break;
    case NTX_Q4_0: err = cudaLaunchKernelEx(&cfg, embed_kernel<NTX_Q4_0>, e, rb, hidden, token_dev, h, p); break;
    case NTX_Q4_K: err = cudaLaunchKernelEx(&cfg, embed_kernel<NTX_Q4_K>, e, rb, hidden, token_dev, h, p); break;
    case NTX_Q6_K: err = cudaLaunchKernelEx(&cfg, embed_kernel<NTX_Q6_K>, e, rb, hidden, token_dev, h, p); break;
    case NTX_Q5_K: err = cudaLaunchKernelEx(&cfg, embed_kernel<NTX_Q5_K>, e, rb, hidden, token_dev, h, p); break;
    case NTX_F16: err = cudaLaunchKernelEx(&cfg, embed_kernel<NTX_F16>, e, rb, hidden, token_dev, h, p); break;
    case NTX_F32: err = cudaLaunchKernelEx(&cfg, embed_kernel<NTX_F32>, e, rb, hidden, token_dev, h, p); break;
    case NTX_Q8_0_T: err = cudaLaunchKernelEx(&cfg, embed_kernel<NTX_Q8_0_T>, e, rb, hidden, token_dev, h, p); break;
    case NTX_Q4_0_T: err = cudaLaunchKernelEx(&cfg, embed_kernel<NTX_Q4_0_T>, e, rb, hidden, token_dev, h, p); break;
    case NTX_Q4_K_T: err = cudaLaunchKernelEx(&cfg, embed_kernel<NTX_Q4_K_T>, e, rb, hidden, token_dev, h, p); break;
    case NTX_Q6_K_T: err = cudaLaunchKernelEx(&cfg, embed_kernel<NTX_Q6_K_T>, e, rb, hidden, token_dev, h, p); break;
    case NTX_Q5_K_T: err = cudaLaunchKernelEx(&cfg, embed_kernel<NTX_Q5_K_T>, e, rb, hidden, token_dev, h, p); break;
    }
    if (err != cudaSuccess) return fail(NTX_ECUDA, std::string("embedding launch: ") + cudaGetErrorString(err));
    return NTX_OK;
}

ntx_status set_step_launch(int32_t* step, int32_t token, int32_t pos, float* rope, float theta, int head_dim,
                           cudaStream_t s, const int32_t* token_dev)
{
    set_step_kernel<<<1, std::max(32, head_dim / 2), 0, s>>>(step, token, token_dev, pos, rope, theta, head_dim);
    return check_launch("step counter");
}

}  // namespace ntx

using namespace ntx;

NTX_EXPORT ntx_status ntx_rmsnorm(const float* x, const float* w, float* y, int64_t n, float eps, void* stream)
{
    if (!x || !w || !y) return fail(NTX_EINVAL, "ntx_rmsnorm: null pointer");
    if (n < 1 || n > (1ll << 30)) return fail(NTX_EINVAL, "ntx_rmsnorm: n out of range");
    if (!(eps >= 0.f)) return fail(NTX_EINVAL, "ntx_rmsnorm: eps must be >= 0");
    rmsnorm_kernel<<<1, kBlock, 0, (cudaStream_t)stream>>>(x, w, y, n, eps);
    return check_launch("ntx_rmsnorm");
}

NTX_EXPORT ntx_status ntx_rope(float* q, float* k, int n_q_heads, int n_kv_heads, int head_dim, int32_t pos,
                               float theta, void* stream)
{
    if (!q) return fail(NTX_EINVAL, "ntx_rope: null q");
    if (!k) n_kv_heads = 0;
    if (n_q_heads < 0 || n_kv_heads < 0 || n_q_heads + n_kv_heads < 1)
        return fail(NTX_EINVAL, "ntx_rope: bad head counts");
    if (head_dim < 2 || head_dim % 2) return fail(NTX_EINVAL, "ntx_rope: head_dim must be even and >= 2");
    if (pos < 0) return fail(NTX_EINVAL, "ntx_rope: pos must be >= 0");
    if (!(theta > 0.f)) return fail(NTX_EINVAL, "ntx_rope: theta must be > 0");
    const int total = (n_q_heads + n_kv_heads) * (head_dim / 2);
    const int grid = std::min((total + 255) / 256, 1024);
    rope_kernel<<<grid, 256, 0, (cudaStream_t)stream>>>(q, k, n_q_heads, n_kv_heads, head_dim, pos, theta);
    return check_launch("ntx_rope");
}

NTX_EXPORT ntx_status ntx_swiglu(const float* gate, const float* up, float* out, int64_t n, void* stream)
{
    if (!gate || !up || !out) return fail(NTX_EINVAL, "ntx_swiglu: null pointer");
    if (n < 1) return fail(NTX_EINVAL, "ntx_swiglu: n must be >= 1");
    const int grid = (int)std::min<int64_t>((n + 255) / 256, 4096);
    swiglu_kernel<<<grid, 256, 0, (cudaStream_t)stream>>>(gate, up, out, n);
    return check_launch("ntx_swiglu");
}

NTX_EXPORT ntx_status ntx_softmax(const float* x, float* y, int64_t n, void* stream)
{
    if (!x || !y) return fail(NTX_EINVAL, "ntx_softmax: null pointer");
    if (n < 1 || n > (1ll << 26)) return fail(NTX_EINVAL, "ntx_softmax: n out of range");
    softmax_kernel<<<1, kBlock, 0, (cudaStream_t)stream>>>(x, y, n);
    return check_launch("ntx_softmax");
}

namespace ntx {
ntx_status argmax_launch(const float* x, int64_t n, int32_t* out_index, cudaStream_t s)
{
    argmax_kernel<<<1, kBlock, 0, s>>>(x, n, out_index);
    return check_launch("argmax");
}
}  // namespace ntx

NTX_EXPORT ntx_status ntx_argmax(const float* x, int64_t n, int32_t* out_index, void* stream)
{
    if (!x || !out_index) return fail(NTX_EINVAL, "ntx_argmax: null pointer");
    if (n < 1 || n > (1ll << 26)) return fail(NTX_EINVAL, "ntx_argmax: n out of range");
    return argmax_launch(x, n, out_index, (cudaStream_t)stream);
}

NTX_EXPORT ntx_status ntx_embed(int qtype, const void* E, int64_t vocab, int64_t hidden, const int32_t* token_dev,
                                float* h, void* stream)
{
    if (qtraits(qtype).block_elems == 0) return fail(NTX_EINVAL, "ntx_embed: unknown qtype");
    if (!E || !token_dev || !h) return fail(NTX_EINVAL, "ntx_embed: null pointer");
    if (vocab < 1 || row_bytes(qtype, hidden) == 0) return fail(NTX_EINVAL, "ntx_embed: bad shape");
    return embed_launch(qtype, E, hidden, token_dev, h, (cudaStream_t)stream, false);
}
