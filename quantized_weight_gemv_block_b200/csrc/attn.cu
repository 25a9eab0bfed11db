// attn.cu - GQA decode attention of one query token over the fp16 KV cache
// (attention with GQA of the ntransformer news summary, "Funciones principales";
// F16 KV cache of "Hoja de ruta de desarrollo", Fase 3), split over the context.
//
// Grid: n_kv_heads x n_split CTAs, one per SM.  CTA (g, s) takes positions
// [s P, s P + P) of kv head g together with the G = n_q / n_kv query heads that
// read it, so every K / V row is fetched from HBM once:
//  * a producer warp streams the range in stages of 64 positions (K rows and V
//    rows, 32 KB) with 1-D bulk copies into a ring of shared-memory stages;
//  * 16 consumer warps: scores (lanes own 4 dims of a K row, the G partial dot
//    products are reduced across the warp with a transposed butterfly), an
//    online softmax per query head (running max m and sum l), then P.V with
//    paired fp32 FMAs;
//  * the partial (m, l, acc[128]) of each query head goes to the workspace; the
//    last CTA of kv head g (ticket counter, reset after use) bulk-copies all
//    partials of its head into shared memory and merges them with the
//    log-sum-exp rule in a fixed order, so the result is deterministic.
// Every wait is bounded; a wait that runs out records an error and the CTA still
// finishes.
#include <algorithm>

#include "ops.h"

namespace ntx {
namespace {

constexpr int HD = 128;
constexpr int kConsumerWarps = 16;
constexpr int kConsumers = kConsumerWarps * 32;
constexpr int kThreads = kConsumers + 32;
constexpr int kSub = 64;                          // positions per stage
constexpr int kStageBytes = kSub * HD * 2 * 2;    // K and V rows
constexpr int kStages = 4;
constexpr int kCounterBytes = kAttnCounterBytes;  // ticket counters at the start of the workspace
constexpr int kPartFloats = 4 + HD;               // m, l, 2 pad, acc[128]: 528-byte records
constexpr int kMaxSplit = 128;
constexpr uint32_t kPolls = 1u << 22;

struct KArgs {
    const float* q;
    const __half* kc;
    const __half* vc;
    float* out;
    uint32_t* cnt;
    float* part;
    int max_ctx, n_split;
    int32_t n_ctx;
    const int32_t* pos_dev;
    int use_pdl;
};

// shared-memory layout (bytes)
constexpr int kOffBars = 0;                             // full[4], empty[4], merge barrier
constexpr int kOffFlag = 80;
constexpr int kOffStat = 128;                           // m[8], l[8], alpha[8]
constexpr int kOffScore = 256;                          // s[8][64] floats
constexpr int kOffRed = kOffScore + 8 * kSub * 4;       // [16][128] floats
constexpr int kOffRing = kOffRed + kConsumerWarps * HD * 4;
constexpr int kSmem = kOffRing + kStages * kStageBytes;

template <int G>
__global__ void __launch_bounds__(kThreads, 1) attn_kernel(const KArgs a)
{
    extern __shared__ __align__(128) uint8_t sm[];
    uint64_t* full = reinterpret_cast<uint64_t*>(sm + kOffBars);
    uint64_t* empty = full + kStages;
    uint64_t* mbar = empty + kStages;
    int* flag = reinterpret_cast<int*>(sm + kOffFlag);
    float* s_m = reinterpret_cast<float*>(sm + kOffStat);
    float* s_l = s_m + 8;
    float* s_alpha = s_l + 8;
    float* sc = reinterpret_cast<float*>(sm + kOffScore);
    float* red = reinterpret_cast<float*>(sm + kOffRed);
    uint8_t* ring = sm + kOffRing;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    if (tid == 0) {
        for (int i = 0; i < kStages; ++i) {
            mbar_init(&full[i], 1);
            mbar_init(&empty[i], kConsumerWarps);
        }
        mbar_init(mbar, 1);
        fence_mbar_init();
    }
    if (tid < 8) {
        s_m[tid] = -INFINITY;
        s_l[tid] = 0.f;
    }
    __syncthreads();
    if (a.use_pdl) {
        pdl_launch_dependents();
        pdl_wait();
    }
    const int g = blockIdx.x / a.n_split, sp = blockIdx.x % a.n_split;
    const int n_ctx = a.pos_dev ? (*a.pos_dev + 1) : a.n_ctx;
    const int P = (n_ctx + a.n_split - 1) / a.n_split;
    const int t0 = sp * P;
    const int np = max(0, min(n_ctx, t0 + P) - t0);
    const int nsub = (np + kSub - 1) / kSub;

    if (warp == kConsumerWarps) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            const uint64_t pol = policy_evict_first();
            const __half* kb = a.kc + ((int64_t)g * a.max_ctx + t0) * HD;
            const __half* vb = a.vc + ((int64_t)g * a.max_ctx + t0) * HD;
            int s = 0;
            uint32_t ph = 0;
            for (int i = 0; i < nsub; ++i) {
                if (!mbar_wait(&empty[s], ph ^ 1u, kPolls)) {
                    record_device_error(DEVERR_EMPTY_WAIT);
                    // the stages issued last must land before the CTA may exit
                    for (int k = 1; k <= kStages && k <= i; ++k) {
                        const int j = i - k;
                        mbar_wait(&full[j % kStages], (uint32_t)(j / kStages) & 1u, 1u << 20);
                    }
                    break;
                }
                const int cnt = min(kSub, np - i * kSub);
                const uint32_t bytes = (uint32_t)cnt * HD * 2;
                uint8_t* st = ring + s * kStageBytes;
                mbar_arrive_expect_tx(&full[s], 2 * bytes);
                bulk_g2s(st, kb + (int64_t)i * kSub * HD, bytes, &full[s], pol);
                bulk_g2s(st + kSub * HD * 2, vb + (int64_t)i * kSub * HD, bytes, &full[s], pol);
                if (++s == kStages) {
                    s = 0;
                    ph ^= 1u;
                }
            }
        }
    } else {
        // ----------------------------------------------------------- consumers
        // q of the G heads, pre-scaled by 1/sqrt(128); lane owns dims 4 lane .. +3
        uint64_t q2[G][2];
        const float scale = 0.08838834764831845f;
#pragma unroll
        for (int h = 0; h < G; ++h) {
            const float4 v = *reinterpret_cast<const float4*>(a.q + (int64_t)(g * G + h) * HD + 4 * lane);
            q2[h][0] = pack2(__float_as_uint(v.x * scale), __float_as_uint(v.y * scale));
            q2[h][1] = pack2(__float_as_uint(v.z * scale), __float_as_uint(v.w * scale));
        }
        // P.V ownership: WPH = 16 / G warps per head, positions interleaved over them
        constexpr int WPH = kConsumerWarps / G;
        const int pv_head = warp / WPH, pv_sub = warp % WPH;
        uint64_t acc2[2] = {0, 0};
        bool dead = false;
        int s = 0;
        uint32_t ph = 0;
        for (int i = 0; i < nsub; ++i) {
            const int cnt = min(kSub, np - i * kSub);
            if (!dead && !mbar_wait(&full[s], ph, kPolls)) {
                record_device_error(DEVERR_FULL_WAIT);
                dead = true;
            }
            const __half* Ks = reinterpret_cast<const __half*>(ring + s * kStageBytes);
            const __half* Vs = Ks + kSub * HD;
            // scores: warp w takes positions w, w + 16, ...
#pragma unroll
            for (int t = warp; t < kSub; t += kConsumerWarps) {
                float part[G];
                if (t < cnt && !dead) {
                    const uint2 raw = *reinterpret_cast<const uint2*>(Ks + t * HD + 4 * lane);
                    const float2 k01 = __half22float2(*reinterpret_cast<const __half2*>(&raw.x));
                    const float2 k23 = __half22float2(*reinterpret_cast<const __half2*>(&raw.y));
                    const uint64_t ka = pack2(__float_as_uint(k01.x), __float_as_uint(k01.y));
                    const uint64_t kb2 = pack2(__float_as_uint(k23.x), __float_as_uint(k23.y));
#pragma unroll
                    for (int h = 0; h < G; ++h) {
                        uint64_t d2 = 0;
                        fma2(d2, q2[h][0], ka);
                        fma2(d2, q2[h][1], kb2);
                        const f2 d = f2_from(d2);
                        part[h] = d.x + d.y;
                    }
                } else {
#pragma unroll
                    for (int h = 0; h < G; ++h) part[h] = 0.f;
                }
                // transposed butterfly: halving rounds leave one head per lane group
                int head = 0;
#pragma unroll
                for (int n = G, sh = 16; n > 1; n >>= 1, sh >>= 1) {
                    const bool hi = (lane & sh) != 0;
#pragma unroll
                    for (int k = 0; k < n / 2; ++k) {
                        const float send = hi ? part[k] : part[k + n / 2];
                        const float keep = hi ? part[k + n / 2] : part[k];
                        part[k] = keep + __shfl_xor_sync(0xffffffffu, send, sh);
                    }
                    head += hi ? n / 2 : 0;
                }
                float v = part[0];
#pragma unroll
                for (int sh = 16 / G; sh > 0; sh >>= 1) v += __shfl_xor_sync(0xffffffffu, v, sh);
                if ((lane & (32 / G - 1)) == 0) sc[head * kSub + t] = v;
            }
            named_bar_sync(1, kConsumers);
            // online softmax: warp h updates head h
            if (warp < G) {
                const int h = warp;
                const float x0 = lane < cnt ? sc[h * kSub + lane] : -INFINITY;
                const float x1 = lane + 32 < cnt ? sc[h * kSub + lane + 32] : -INFINITY;
                const float mx = gemv::warp_max(fmaxf(x0, x1));
                const float m_old = s_m[h];
                const float m_new = fmaxf(m_old, mx);
                const float e0 = lane < cnt ? expf(x0 - m_new) : 0.f;
                const float e1 = lane + 32 < cnt ? expf(x1 - m_new) : 0.f;
                sc[h * kSub + lane] = e0;
                sc[h * kSub + lane + 32] = e1;
                const float sum = gemv::warp_sum(e0 + e1);
                if (lane == 0) {
                    const float alpha = m_old == -INFINITY ? 0.f : expf(m_old - m_new);
                    s_alpha[h] = alpha;
                    s_m[h] = m_new;
                    s_l[h] = s_l[h] * alpha + sum;
                }
            }
            named_bar_sync(1, kConsumers);
            // P.V: this thread's 4 dims of head pv_head, positions pv_sub, pv_sub + WPH, ...
            {
                const float alpha = s_alpha[pv_head];
                const uint64_t al2 = pack2(__float_as_uint(alpha), __float_as_uint(alpha));
                acc2[0] = mul2(acc2[0], al2);
                acc2[1] = mul2(acc2[1], al2);
                if (!dead) {
#pragma unroll 4
                    for (int t = pv_sub; t < cnt; t += WPH) {
                        const float p = sc[pv_head * kSub + t];
                        const uint64_t p2 = pack2(__float_as_uint(p), __float_as_uint(p));
                        const uint2 raw = *reinterpret_cast<const uint2*>(Vs + t * HD + 4 * lane);
                        const float2 v01 = __half22float2(*reinterpret_cast<const __half2*>(&raw.x));
                        const float2 v23 = __half22float2(*reinterpret_cast<const __half2*>(&raw.y));
                        fma2(acc2[0], p2, pack2(__float_as_uint(v01.x), __float_as_uint(v01.y)));
                        fma2(acc2[1], p2, pack2(__float_as_uint(v23.x), __float_as_uint(v23.y)));
                    }
                }
            }
            // the next stage's scores overwrite sc: every consumer must be done reading it
            named_bar_sync(1, kConsumers);
            if (lane == 0) mbar_arrive(&empty[s]);
            if (++s == kStages) {
                s = 0;
                ph ^= 1u;
            }
        }
        // combine the WPH warps of each head, write this split's partial
        const f2 a01 = f2_from(acc2[0]), a23 = f2_from(acc2[1]);
        *reinterpret_cast<float4*>(red + warp * HD + 4 * lane) = make_float4(a01.x, a01.y, a23.x, a23.y);
        named_bar_sync(1, kConsumers);
        if (pv_sub == 0) {
            float4 o = *reinterpret_cast<const float4*>(red + warp * HD + 4 * lane);
            for (int w = 1; w < WPH; ++w) {
                const float4 r = *reinterpret_cast<const float4*>(red + (warp + w) * HD + 4 * lane);
                o.x += r.x;
                o.y += r.y;
                o.z += r.z;
                o.w += r.w;
            }
            float* pp = a.part + ((size_t)(g * a.n_split + sp) * G + pv_head) * kPartFloats;
            *reinterpret_cast<float4*>(pp + 4 + 4 * lane) = o;
            if (lane == 0) {
                pp[0] = s_m[pv_head];
                pp[1] = s_l[pv_head];
            }
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
        // all partials of this kv head in one bulk copy (the ring is free now)
        const float* base = a.part + (size_t)g * a.n_split * G * kPartFloats;
        const uint32_t bytes = (uint32_t)(a.n_split * G * kPartFloats * 4);
        float* pm = reinterpret_cast<float*>(ring);
        if (tid == 0) {
            asm volatile("fence.proxy.async.global;" ::: "memory");
            mbar_arrive_expect_tx(mbar, bytes);
            bulk_g2s(pm, base, bytes, mbar, policy_evict_first());
        }
        const bool ok = mbar_wait(mbar, 0, kPolls);
        if (!ok && tid == 0) record_device_error(DEVERR_FULL_WAIT);
        for (int idx = tid; ok && idx < G * HD; idx += kThreads) {
            const int hh = idx / HD, d = idx % HD;
            float M = -INFINITY;
            for (int s2 = 0; s2 < a.n_split; ++s2) {
                const float* ps = pm + ((size_t)s2 * G + hh) * kPartFloats;
                if (ps[1] > 0.f) M = fmaxf(M, ps[0]);
            }
            float L = 0.f, o = 0.f;
            for (int s2 = 0; s2 < a.n_split; ++s2) {
                const float* ps = pm + ((size_t)s2 * G + hh) * kPartFloats;
                if (ps[1] > 0.f) {
                    const float w = expf(ps[0] - M);
                    L = fmaf(ps[1], w, L);
                    o = fmaf(ps[4 + d], w, o);
                }
            }
            a.out[(int64_t)(g * G + hh) * HD + d] = o / L;
        }
        if (tid == 0) a.cnt[g] = 0u;
    }
}

template <int G>
ntx_status launch_g(const KArgs& k, int grid, cudaStream_t s, bool pdl)
{
    static bool configured = false;
    if (!configured) {
        cudaFuncSetAttribute(attn_kernel<G>, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmem);
        configured = true;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = (size_t)kSmem;
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

int attn_split_for(int n_q_heads, int n_kv_heads, int32_t max_ctx)
{
    (void)max_ctx;
    const int G = n_q_heads / n_kv_heads;
    // one CTA per SM, and every split's partial must fit the merge buffer
    const int by_merge = (kStages * kStageBytes) / (G * kPartFloats * 4);
    return std::min(std::min(kMaxSplit, by_merge), std::max(1, num_sms() / n_kv_heads));
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
    if ((size_t)a.n_split * G * kPartFloats * 4 > (size_t)kStages * kStageBytes)
        return fail(NTX_EUNSUPPORTED, "attention: too many splits for the merge buffer");
    KArgs k{};
    k.q = a.q;
    k.kc = a.k_cache;
    k.vc = a.v_cache;
    k.out = a.out;
    k.cnt = reinterpret_cast<uint32_t*>(a.workspace);
    k.part = reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(a.workspace) + kCounterBytes);
    k.max_ctx = a.max_ctx;
    k.n_split = a.n_split;
    k.n_ctx = a.n_ctx;
    k.pos_dev = a.pos_dev;
    k.use_pdl = a.pdl ? 1 : 0;
    const int grid = a.n_kv_heads * a.n_split;
    switch (G) {
    case 1: return launch_g<1>(k, grid, s, a.pdl);
    case 2: return launch_g<2>(k, grid, s, a.pdl);
    case 4: return launch_g<4>(k, grid, s, a.pdl);
    case 8: return launch_g<8>(k, grid, s, a.pdl);
    default: return fail(NTX_EUNSUPPORTED, "attention: q heads per kv head must be 1, 2, 4 or 8");
    }
}

}  // namespace ntx

using namespace ntx;

NTX_EXPORT size_t ntx_attn_workspace_bytes(int n_q_heads, int n_kv_heads, int head_dim, int32_t max_ctx)
{
    if (n_kv_heads < 1 || n_q_heads < n_kv_heads || n_q_heads % n_kv_heads || max_ctx < 1) return 0;
    return attn_workspace_bytes_for(n_q_heads, n_kv_heads, head_dim, attn_split_for(n_q_heads, n_kv_heads, max_ctx));
}

namespace ntx {

ntx_status attn_check(const void* q, const void* k_cache, const void* v_cache, const void* out, int n_q_heads,
                      int n_kv_heads, int head_dim, int32_t n_ctx, int32_t max_ctx, const char* who)
{
    const std::string w(who);
    if (!q || !k_cache || !v_cache || !out) return fail(NTX_EINVAL, w + ": null pointer");
    if (head_dim != HD) return fail(NTX_EUNSUPPORTED, w + ": head_dim must be 128");
    if (n_kv_heads < 1 || n_q_heads < n_kv_heads || n_q_heads % n_kv_heads)
        return fail(NTX_EINVAL, w + ": n_q_heads must be a positive multiple of n_kv_heads");
    const int G = n_q_heads / n_kv_heads;
    if (G != 1 && G != 2 && G != 4 && G != 8)
        return fail(NTX_EUNSUPPORTED, w + ": q heads per kv head must be 1, 2, 4 or 8");
    if (n_kv_heads > 64) return fail(NTX_EUNSUPPORTED, w + ": at most 64 kv heads");
    if (max_ctx < 1 || n_ctx < 1 || n_ctx > max_ctx) return fail(NTX_EINVAL, w + ": need 1 <= n_ctx <= max_ctx");
    if (!aligned(q, 16) || !aligned(out, 16) || !aligned(k_cache, 16) || !aligned(v_cache, 16))
        return fail(NTX_EINVAL, w + ": q, out and the caches must be 16-byte aligned");
    return NTX_OK;
}

}  // namespace ntx

NTX_EXPORT ntx_status ntx_attn_decode(const float* q, const void* k_cache, const void* v_cache, float* out,
                                      int n_q_heads, int n_kv_heads, int head_dim, int32_t n_ctx, int32_t max_ctx,
                                      void* workspace, size_t workspace_bytes, void* stream)
{
    ntx_status st = attn_check(q, k_cache, v_cache, out, n_q_heads, n_kv_heads, head_dim, n_ctx, max_ctx,
                               "ntx_attn_decode");
    if (st != NTX_OK) return st;
    if (!workspace || !aligned(workspace, 16))
        return fail(NTX_EINVAL, "ntx_attn_decode: workspace must be non-null and 16-byte aligned");
    const int n_split = attn_split_for(n_q_heads, n_kv_heads, max_ctx);
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
