// attn.cu - GQA decode attention of one query token over the fp16 KV cache
// (attention with GQA of the ntransformer news summary, "Funciones principales";
// F16 KV cache of "Hoja de ruta de desarrollo", Fase 3), split over the context.
//
// Grid: n_kv_heads x n_split CTAs (n_split sized so two CTAs per SM cover the
// whole context).  CTA (g, s) takes positions [s P, s P + P) of kv head g and the
// G = n_q / n_kv query heads that read it, so every K / V row is fetched once:
//  * the V rows of the range go to shared memory with one bulk copy issued at
//    entry, overlapping the score phase;
//  * scores: lanes own 8 dims of a K row (16-byte loads, two rows per warp per
//    step, four steps in flight), the G dot products are reduced over 16 lanes;
//  * a local softmax (max m, sum l of e^(s - m)), then P.V from shared memory;
//  * the partial (m, l, acc[128]) per query head goes to the workspace and the
//    last CTA of kv head g (ticket counter, reset after use) merges the splits
//    with the log-sum-exp rule in a fixed order, so results are deterministic.
#include <algorithm>

#include "ops.h"

namespace ntx {
namespace {

constexpr int HD = 128;
constexpr int kThreads = 256;
constexpr int kMaxRows = 256;       // positions per CTA (V rows in shared memory)
constexpr int kCounterBytes = 256;  // ticket counters at the start of the workspace
constexpr int kPartFloats = 4 + HD;   // m, l, 2 pad, acc[128]: 528 B, 16-byte aligned records

struct KArgs {
    const float* q;
    const __half* kc;
    const __half* vc;
    float* out;
    uint32_t* cnt;
    float* part;
    int max_ctx, n_split, p_alloc, sc_len;   // sc_len = max(p_alloc, n_split)
    int32_t n_ctx;
    const int32_t* pos_dev;
    int use_pdl;
};

template <int G>
__global__ void __launch_bounds__(kThreads, 2) attn_kernel(const KArgs a)
{
    extern __shared__ __align__(128) uint8_t sm[];
    uint64_t* bar = reinterpret_cast<uint64_t*>(sm);
    int* flag = reinterpret_cast<int*>(sm + 8);
    __half* vbuf = reinterpret_cast<__half*>(sm + 128);
    float* sc = reinterpret_cast<float*>(sm + 128 + (size_t)a.p_alloc * HD * 2);   // [G][p_alloc]
    float* red = sc + G * a.sc_len;                                                 // [8][HD]
    float* stat = red + 8 * HD;                                                     // m[G], l[G]

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    if (a.use_pdl) {
        pdl_launch_dependents();
        pdl_wait();
    }
    const int g = blockIdx.x / a.n_split, sp = blockIdx.x % a.n_split;
    const int n_ctx = a.pos_dev ? (*a.pos_dev + 1) : a.n_ctx;
    const int P = (n_ctx + a.n_split - 1) / a.n_split;
    const int t0 = sp * P;
    const int np = max(0, min(n_ctx, t0 + P) - t0);

    if (tid == 0) {
        mbar_init(bar, 1);
        fence_mbar_init();
    }
    __syncthreads();
    if (tid == 0 && np > 0) {
        mbar_arrive_expect_tx(bar, (uint32_t)np * HD * 2);
        bulk_g2s(vbuf, a.vc + ((int64_t)g * a.max_ctx + t0) * HD, (uint32_t)np * HD * 2, bar, policy_evict_first());
    }

    // ---- scores s[h][t] = (q_h / sqrt(128)) . K[t]
    const int half = lane >> 4, dl = lane & 15;
    float qr[G][8];
    const float scale = 0.08838834764831845f;   // 1 / sqrt(128)
#pragma unroll
    for (int h = 0; h < G; ++h) {
        const float4* qp = reinterpret_cast<const float4*>(a.q + (int64_t)(g * G + h) * HD + 8 * dl);
        const float4 x0 = qp[0], x1 = qp[1];
        qr[h][0] = x0.x * scale; qr[h][1] = x0.y * scale; qr[h][2] = x0.z * scale; qr[h][3] = x0.w * scale;
        qr[h][4] = x1.x * scale; qr[h][5] = x1.y * scale; qr[h][6] = x1.z * scale; qr[h][7] = x1.w * scale;
    }
    const __half* kbase = a.kc + ((int64_t)g * a.max_ctx + t0) * HD + 8 * dl;
    constexpr int U = 4;
    for (int tb = 2 * warp; tb < np; tb += 16 * U) {
        uint4 kv[U];
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int t = tb + 16 * u + half;
            kv[u] = t < np ? __ldg(reinterpret_cast<const uint4*>(kbase + (int64_t)t * HD)) : make_uint4(0, 0, 0, 0);
        }
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int t = tb + 16 * u + half;
            const __half2* k2 = reinterpret_cast<const __half2*>(&kv[u]);
            float kf[8];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const float2 f = __half22float2(k2[i]);
                kf[2 * i] = f.x;
                kf[2 * i + 1] = f.y;
            }
            float part[G];
#pragma unroll
            for (int h = 0; h < G; ++h) {
                float s = 0.f;
#pragma unroll
                for (int i = 0; i < 8; ++i) s = fmaf(qr[h][i], kf[i], s);
                part[h] = s;
            }
#pragma unroll
            for (int h = 0; h < G; ++h) {
#pragma unroll
                for (int o = 8; o > 0; o >>= 1) part[h] += __shfl_xor_sync(0xffffffffu, part[h], o);
            }
            if (dl == 0 && t < np) {
#pragma unroll
                for (int h = 0; h < G; ++h) sc[h * a.p_alloc + t] = part[h];
            }
        }
    }
    __syncthreads();

    // ---- local softmax statistics per query head
    for (int h = warp; h < G; h += kThreads / 32) {
        float m = -INFINITY;
        for (int t = lane; t < np; t += 32) m = fmaxf(m, sc[h * a.p_alloc + t]);
        m = gemv::warp_max(m);
        float l = 0.f;
        for (int t = lane; t < np; t += 32) {
            const float e = expf(sc[h * a.p_alloc + t] - m);
            sc[h * a.p_alloc + t] = e;
            l += e;
        }
        l = gemv::warp_sum(l);
        if (lane == 0) {
            stat[h] = m;
            stat[G + h] = l;
        }
    }
    bool dead = false;
    if (np > 0 && !mbar_wait(bar, 0, 1u << 22)) {
        record_device_error(DEVERR_FULL_WAIT);
        dead = true;
    }
    __syncthreads();

    // ---- acc_h = sum_t e_t V[t]; warps per head WPH = 8 / G
    constexpr int WPH = (kThreads / 32) / G;
    const int h = warp / WPH, sub = warp % WPH;
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
    if (!dead) {
        for (int t = sub; t < np; t += WPH) {
            const float p = sc[h * a.p_alloc + t];
            const uint2 raw = *reinterpret_cast<const uint2*>(vbuf + (size_t)t * HD + 4 * lane);
            const float2 v0 = __half22float2(*reinterpret_cast<const __half2*>(&raw.x));
            const float2 v1 = __half22float2(*reinterpret_cast<const __half2*>(&raw.y));
            acc[0] = fmaf(p, v0.x, acc[0]);
            acc[1] = fmaf(p, v0.y, acc[1]);
            acc[2] = fmaf(p, v1.x, acc[2]);
            acc[3] = fmaf(p, v1.y, acc[3]);
        }
    }
    if (WPH > 1) {
#pragma unroll
        for (int i = 0; i < 4; ++i) red[warp * HD + 4 * lane + i] = acc[i];
    }
    __syncthreads();
    float* pp = a.part + ((size_t)(g * a.n_split + sp) * G + h) * kPartFloats;
    if (sub == 0) {
        if (WPH > 1) {
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                float s = 0.f;
                for (int w = 0; w < WPH; ++w) s += red[(warp + w) * HD + 4 * lane + i];
                acc[i] = s;
            }
        }
        *reinterpret_cast<float4*>(pp + 4 + 4 * lane) = make_float4(acc[0], acc[1], acc[2], acc[3]);
        if (lane == 0) {
            pp[0] = stat[h];
            pp[1] = stat[G + h];
        }
    }

    // ---- the last CTA of kv head g merges the splits (fixed order)
    __threadfence();
    __syncthreads();
    if (tid == 0) {
        const uint32_t ticket = atomicAdd(&a.cnt[g], 1u);
        *flag = (ticket == (uint32_t)a.n_split - 1u) ? 1 : 0;
    }
    __syncthreads();
    if (*flag) {
        __threadfence();
        // (1) all (m, l) of this kv head's splits in parallel; weights e^(m_s - M_h)
        const float* base = a.part + (size_t)g * a.n_split * G * kPartFloats;
        float* wsm = sc;                         // [n_split][G] weights (score buffer is free now)
        for (int r = tid; r < a.n_split * G; r += kThreads) {
            const float2 ml = __ldcg(reinterpret_cast<const float2*>(base + (size_t)r * kPartFloats));
            wsm[r] = ml.y > 0.f ? ml.x : -INFINITY;
            red[r] = ml.y;                       // l (red has 8 * 128 >= 64 * 8 floats)
        }
        __syncthreads();
        for (int hh = warp; hh < G; hh += kThreads / 32) {
            float M = -INFINITY;
            for (int s2 = lane; s2 < a.n_split; s2 += 32) M = fmaxf(M, wsm[s2 * G + hh]);
            M = gemv::warp_max(M);
            float L = 0.f;
            for (int s2 = lane; s2 < a.n_split; s2 += 32) {
                const int r = s2 * G + hh;
                const float w = wsm[r] == -INFINITY ? 0.f : expf(wsm[r] - M);
                L = fmaf(red[r], w, L);
                wsm[r] = w;
            }
            L = gemv::warp_sum(L);
            if (lane == 0) stat[hh] = L;
        }
        __syncthreads();
        // (2) acc: warp -> head h, lane -> 4 dims; splits interleaved over the WPH warps of
        // the head; independent 16-byte loads, eight in flight
        float o[4] = {0.f, 0.f, 0.f, 0.f};
        constexpr int UM = 8;
        for (int s0 = sub; s0 < a.n_split; s0 += WPH * UM) {
            float4 v[UM];
            float w[UM];
#pragma unroll
            for (int u = 0; u < UM; ++u) {
                const int s2 = s0 + u * WPH;
                const bool ok = s2 < a.n_split;
                w[u] = ok ? wsm[s2 * G + h] : 0.f;
                v[u] = ok ? __ldcg(reinterpret_cast<const float4*>(base + ((size_t)s2 * G + h) * kPartFloats + 4) + lane)
                          : make_float4(0.f, 0.f, 0.f, 0.f);
            }
#pragma unroll
            for (int u = 0; u < UM; ++u) {
                o[0] = fmaf(w[u], v[u].x, o[0]);
                o[1] = fmaf(w[u], v[u].y, o[1]);
                o[2] = fmaf(w[u], v[u].z, o[2]);
                o[3] = fmaf(w[u], v[u].w, o[3]);
            }
        }
        __syncthreads();
        if (WPH > 1) {
#pragma unroll
            for (int i = 0; i < 4; ++i) red[warp * HD + 4 * lane + i] = o[i];
        }
        __syncthreads();
        if (sub == 0) {
            if (WPH > 1) {
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    float s3 = 0.f;
                    for (int w2 = 0; w2 < WPH; ++w2) s3 += red[(warp + w2) * HD + 4 * lane + i];
                    o[i] = s3;
                }
            }
            const float invL = 1.0f / stat[h];
            *reinterpret_cast<float4*>(a.out + (int64_t)(g * G + h) * HD + 4 * lane) =
                make_float4(o[0] * invL, o[1] * invL, o[2] * invL, o[3] * invL);
        }
        if (tid == 0) a.cnt[g] = 0u;
    }
}

int smem_for(int G, int p_alloc, int sc_len) { return 128 + p_alloc * HD * 2 + (G * sc_len + 8 * HD + 2 * G) * 4 + 64; }

template <int G>
ntx_status launch_g(const KArgs& k, int grid, int p_alloc, cudaStream_t s, bool pdl)
{
    const int smem = smem_for(G, p_alloc, k.sc_len);
    static bool configured = false;
    if (!configured) {
        cudaFuncSetAttribute(attn_kernel<G>, cudaFuncAttributeMaxDynamicSharedMemorySize, 200 * 1024);
        configured = true;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = (size_t)smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = pdl ? 1 : 0;
    cudaError_t e = cudaLaunchKernelEx(&cfg, attn_kernel<G>, k);
    if (e != cudaSuccess) return fail(NTX_ECUDA, std::string("attention launch: ") + cudaGetErrorString(e));
    return NTX_OK;
}

}  // namespace

cudaError_t take_device_error_attn(uint32_t* out) { return take_tu_device_error(out); }

int attn_split_for(int n_kv_heads, int32_t max_ctx)
{
    const int target = (2 * num_sms() + n_kv_heads - 1) / n_kv_heads;
    const int by_rows = (max_ctx + kMaxRows - 1) / kMaxRows;
    return std::min(128, std::max(1, std::max(target, by_rows)));
}

size_t attn_workspace_bytes_for(int n_q_heads, int n_kv_heads, int head_dim, int n_split)
{
    (void)head_dim;
    const int G = n_q_heads / n_kv_heads;
    return (size_t)kCounterBytes + (size_t)n_kv_heads * n_split * G * kPartFloats * sizeof(float);
}

ntx_status attn_launch(const AttnArgs& a, cudaStream_t s)
{
    const int G = a.n_q_heads / a.n_kv_heads;
    KArgs k{};
    k.q = a.q;
    k.kc = a.k_cache;
    k.vc = a.v_cache;
    k.out = a.out;
    k.cnt = reinterpret_cast<uint32_t*>(a.workspace);
    k.part = reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(a.workspace) + kCounterBytes);
    k.max_ctx = a.max_ctx;
    k.n_split = a.n_split;
    k.p_alloc = ((a.max_ctx + a.n_split - 1) / a.n_split + 1) & ~1;
    k.sc_len = std::max(k.p_alloc, a.n_split);
    if (a.n_split * G > 8 * HD || smem_for(G, k.p_alloc, k.sc_len) > 200 * 1024)
        return fail(NTX_EUNSUPPORTED, "attention: context too long for one split pass");
    k.n_ctx = a.n_ctx;
    k.pos_dev = a.pos_dev;
    k.use_pdl = a.pdl ? 1 : 0;
    const int grid = a.n_kv_heads * a.n_split;
    switch (G) {
    case 1: return launch_g<1>(k, grid, k.p_alloc, s, a.pdl);
    case 2: return launch_g<2>(k, grid, k.p_alloc, s, a.pdl);
    case 4: return launch_g<4>(k, grid, k.p_alloc, s, a.pdl);
    case 8: return launch_g<8>(k, grid, k.p_alloc, s, a.pdl);
    default: return fail(NTX_EUNSUPPORTED, "attention: q heads per kv head must be 1, 2, 4 or 8");
    }
}

}  // namespace ntx

using namespace ntx;

NTX_EXPORT size_t ntx_attn_workspace_bytes(int n_q_heads, int n_kv_heads, int head_dim, int32_t max_ctx)
{
    if (n_kv_heads < 1 || n_q_heads < n_kv_heads || n_q_heads % n_kv_heads || max_ctx < 1) return 0;
    return attn_workspace_bytes_for(n_q_heads, n_kv_heads, head_dim, attn_split_for(n_kv_heads, max_ctx));
}

NTX_EXPORT ntx_status ntx_attn_decode(const float* q, const void* k_cache, const void* v_cache, float* out,
                                      int n_q_heads, int n_kv_heads, int head_dim, int32_t n_ctx, int32_t max_ctx,
                                      void* workspace, size_t workspace_bytes, void* stream)
{
    if (!q || !k_cache || !v_cache || !out || !workspace) return fail(NTX_EINVAL, "ntx_attn_decode: null pointer");
    if (head_dim != HD) return fail(NTX_EUNSUPPORTED, "ntx_attn_decode: head_dim must be 128");
    if (n_kv_heads < 1 || n_q_heads < n_kv_heads || n_q_heads % n_kv_heads)
        return fail(NTX_EINVAL, "ntx_attn_decode: n_q_heads must be a positive multiple of n_kv_heads");
    const int G = n_q_heads / n_kv_heads;
    if (G != 1 && G != 2 && G != 4 && G != 8)
        return fail(NTX_EUNSUPPORTED, "ntx_attn_decode: q heads per kv head must be 1, 2, 4 or 8");
    if (n_kv_heads > 64) return fail(NTX_EUNSUPPORTED, "ntx_attn_decode: at most 64 kv heads");
    if (max_ctx < 1 || n_ctx < 1 || n_ctx > max_ctx) return fail(NTX_EINVAL, "ntx_attn_decode: need 1 <= n_ctx <= max_ctx");
    if (!aligned(q, 16) || !aligned(out, 16) || !aligned(k_cache, 16) || !aligned(v_cache, 16) || !aligned(workspace, 16))
        return fail(NTX_EINVAL, "ntx_attn_decode: q, out, caches and workspace must be 16-byte aligned");
    const int n_split = attn_split_for(n_kv_heads, max_ctx);
    if (workspace_bytes < attn_workspace_bytes_for(n_q_heads, n_kv_heads, head_dim, n_split))
        return fail(NTX_EINVAL, "ntx_attn_decode: workspace smaller than ntx_attn_workspace_bytes()");
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
    a.workspace = workspace;
    a.n_split = n_split;
    a.pdl = false;
    return attn_launch(a, (cudaStream_t)stream);
}
