// fgemv.cu - GEMV for unquantized F16 / F32 weights (batch 1), with the same fused
// prologue (RMSNorm) and epilogues (store, residual add, SwiGLU of a gate / up row
// pair, RoPE + fp16 KV-cache append) as the quantized kernels.
//
// F16 and F32 are among the weight formats of the ntransformer news summary
// ("Descripción general de NTransformer").  There are no codes to multiply as
// integers: each weight is one fp32 product with x (fp16 widens exactly), summed in
// fp32.  The kernel is a pure weight stream, built like the tiled GEMV:
//  * one CTA per SM; 8 consumer warps and a producer warp; a CTA owns a contiguous
//    range of 16-row groups;
//  * a stage is one group x one chunk of CE columns (16 row segments of 2 KB, one
//    1-D bulk copy each, L2 evict-first) in a ring of shared-memory stages guarded by
//    mbarriers; the producer starts streaming before the programmatic wait (weights
//    do not depend on the previous kernel);
//  * x (RMSNorm applied) is staged once per CTA in shared memory as fp32;
//  * consumer warp w takes rows 2w and 2w + 1 of each stage; lane i takes columns
//    4i .. 4i + 3 of every 128 (one 8- or 16-byte weight load and one float4 of x per
//    row pair), so a warp's loads are contiguous; row totals are reduced over the warp
//    and the epilogue runs once per group.
#include <algorithm>

#include "launch.h"
#include "ops.h"
#include "qmma.cuh"

namespace ntx {
namespace fgemv {

using gemv::Params;

constexpr int kWarps = 8;
constexpr int kCons = kWarps * 32;
constexpr int kThreads = kCons + 32;
constexpr int kProducer = kWarps;
constexpr int kMaxStages = 8;
constexpr int kStageBytes = 16 * 2048;            // 16 row segments of 2 KB
constexpr int kOffRed = 256;                      // [16 rows][2 mats] totals of the current group
constexpr int kOffRope = 512;                     // [64][cos, sin]
constexpr int kHeader = 1024 + 256;
constexpr int kSmemLimit = 227 * 1024;
constexpr uint32_t kWaitPolls = 1u << 22;

template <int ET>
struct Elem;
template <>
struct Elem<NTX_F16> {
    static constexpr int bytes = 2, CE = 1024;    // columns per stage
    // weights 4 lane .. 4 lane + 3 of a 128-column slice, widened to fp32
    static __device__ __forceinline__ float4 load4(const uint8_t* seg, int col)
    {
        const uint2 v = *reinterpret_cast<const uint2*>(seg + 2 * col);
        const float2 a = __half22float2(*reinterpret_cast<const __half2*>(&v.x));
        const float2 b = __half22float2(*reinterpret_cast<const __half2*>(&v.y));
        return make_float4(a.x, a.y, b.x, b.y);
    }
};
template <>
struct Elem<NTX_F32> {
    static constexpr int bytes = 4, CE = 512;
    static __device__ __forceinline__ float4 load4(const uint8_t* seg, int col)
    {
        return *reinterpret_cast<const float4*>(seg + 4 * col);
    }
};

template <int ET, int EPI, int PRO>
__global__ void __launch_bounds__(kThreads, 1) fgemv_kernel(const Params P)
{
    using E = Elem<ET>;
    constexpr int NM = EPI == gemv::EPI_SWIGLU ? 2 : 1;
    constexpr int CE = E::CE;
    extern __shared__ __align__(128) uint8_t smem[];
    uint64_t* full = reinterpret_cast<uint64_t*>(smem);
    uint64_t* empty = full + kMaxStages;
    float* red = reinterpret_cast<float*>(smem + kOffRed);
    float* rope_cs = reinterpret_cast<float*>(smem + kOffRope);
    float* xs = reinterpret_cast<float*>(smem + kHeader);
    uint8_t* stages = smem + kHeader + P.x_bytes;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int n_groups = (P.M + 15) / 16;
    const int g_begin = (int)((long long)n_groups * blockIdx.x / gridDim.x);
    const int g_end = (int)((long long)n_groups * (blockIdx.x + 1) / gridDim.x);
    const int NCH = (P.K + CE - 1) / CE;

    if (warp == kProducer) {
        if (lane == 0) {
            for (int s = 0; s < P.n_stages; ++s) {
                mbar_init(&full[s], 1);
                mbar_init(&empty[s], kWarps);
            }
            fence_mbar_init();
        }
        __syncwarp();
        qmma::named_bar_arrive(2, kThreads);
        // ------------------------------------------------------------- producer
        const uint64_t pol = policy_evict_first();
        const int NS = P.n_stages;
        int s = 0, issued = 0;
        uint32_t ph = 0;
        bool okay = true;
        for (int gi = g_begin; gi < g_end && okay; ++gi) {
            const int rows = min(16, P.M - 16 * gi);
            for (int mat = 0; mat < NM && okay; ++mat) {
                const uint8_t* base = (mat ? P.W2 : P.W) + (int64_t)16 * gi * P.row_bytes;
                for (int c = 0; c < NCH; ++c) {
                    const uint32_t seg = (uint32_t)(min(CE, P.K - c * CE) * E::bytes);
                    bool ok = true;
                    if (lane == 0) {
                        ok = mbar_wait(&empty[s], ph ^ 1u, kWaitPolls);
                        if (ok) mbar_arrive_expect_tx(&full[s], seg * (uint32_t)rows);
                        else record_device_error(DEVERR_EMPTY_WAIT);
                    }
                    ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
                    if (!ok) {
                        okay = false;
                        break;
                    }
                    __syncwarp();
                    // one row segment per lane (rows of the group past P.M are not copied)
                    if (lane < rows)
                        bulk_g2s(stages + (size_t)s * kStageBytes + (size_t)lane * 2048,
                                 base + (int64_t)lane * P.row_bytes + (int64_t)c * CE * E::bytes, seg, &full[s], pol);
                    ++issued;
                    if (++s == NS) {
                        s = 0;
                        ph ^= 1u;
                    }
                }
            }
        }
        // Drain: the stages issued last must complete before the CTA may exit.
        if (!okay && lane == 0) {
            for (int k = 1; k <= NS && k <= issued; ++k) {
                const int j = issued - k;
                mbar_wait(&full[j % NS], (uint32_t)(j / NS) & 1u, 1u << 20);
            }
        }
        return;
    }
    // ------------------------------------------------------------- consumers
    named_bar_sync(2, kThreads);
    constexpr bool RMS = PRO == gemv::PRO_RMSNORM;
    const float rope_v = (EPI == gemv::EPI_QKV && tid < P.head_dim) ? P.rope_cs[tid] : 0.f;
    if (P.use_pdl) {
        pdl_launch_dependents();
        pdl_wait();
    }
    // x (normalised) into shared memory: the sum of squares over the whole vector first
    const int K4 = P.K / 4;
    const float4* x4 = reinterpret_cast<const float4*>(P.x);
    float4* xs4 = reinterpret_cast<float4*>(xs);
    float ss = 0.f;
    for (int i = tid; i < K4; i += kCons) {
        const float4 v = x4[i];
        xs4[i] = v;
        if (RMS) ss = fmaf(v.x, v.x, fmaf(v.y, v.y, fmaf(v.z, v.z, fmaf(v.w, v.w, ss))));
    }
    if (RMS) {
        ss = gemv::warp_sum(ss);
        if (lane == 0) red[warp] = ss;
    }
    named_bar_sync(1, kCons);
    if (RMS) {
        float tot = 0.f;
#pragma unroll
        for (int w = 0; w < kWarps; ++w) tot += red[w];
        const float inv = 1.0f / sqrtf(tot / (float)P.K + P.eps);
        const float4* w4 = reinterpret_cast<const float4*>(P.norm_w);
        for (int i = tid; i < K4; i += kCons) {
            const float4 v = xs4[i], w = w4[i];
            xs4[i] = make_float4(v.x * w.x * inv, v.y * w.y * inv, v.z * w.z * inv, v.w * w.w * inv);
        }
    }
    if (EPI == gemv::EPI_QKV && tid < P.head_dim) rope_cs[tid] = rope_v;
    named_bar_sync(1, kCons);   // x and the RoPE table complete; red free again

    const int NS = P.n_stages;
    int s = 0;
    uint32_t ph = 0;
    bool dead = false;
    const int32_t pos = (EPI == gemv::EPI_QKV) ? (P.pos_dev ? *P.pos_dev : P.pos) : 0;
    for (int gi = g_begin; gi < g_end; ++gi) {
        const int rows = min(16, P.M - 16 * gi);
#pragma unroll 1
        for (int mat = 0; mat < NM; ++mat) {
            float a0 = 0.f, a1 = 0.f;   // rows 2 warp, 2 warp + 1
            for (int c = 0; c < NCH; ++c) {
                const int cols = min(CE, P.K - c * CE);
                if (!dead && !mbar_wait(&full[s], ph, kWaitPolls)) {
                    record_device_error(DEVERR_FULL_WAIT);
                    dead = true;    // keep taking part in every barrier so the CTA still finishes
                }
                if (!dead) {
                    const uint8_t* st = stages + (size_t)s * kStageBytes;
                    const uint8_t* r0 = st + (size_t)(2 * warp) * 2048;
                    const uint8_t* r1 = r0 + 2048;
                    const float* xc = xs + c * CE;
                    const bool has0 = 2 * warp < rows, has1 = 2 * warp + 1 < rows;
#pragma unroll 4
                    for (int col = 4 * lane; col < cols; col += 128) {
                        const float4 x = *reinterpret_cast<const float4*>(xc + col);
                        if (has0) {
                            const float4 w = E::load4(r0, col);
                            a0 = fmaf(w.x, x.x, fmaf(w.y, x.y, fmaf(w.z, x.z, fmaf(w.w, x.w, a0))));
                        }
                        if (has1) {
                            const float4 w = E::load4(r1, col);
                            a1 = fmaf(w.x, x.x, fmaf(w.y, x.y, fmaf(w.z, x.z, fmaf(w.w, x.w, a1))));
                        }
                    }
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(&empty[s]);
                if (++s == NS) {
                    s = 0;
                    ph ^= 1u;
                }
            }
            a0 = gemv::warp_sum(a0);
            a1 = gemv::warp_sum(a1);
            if (lane == 0) {
                red[(2 * warp) * 2 + mat] = a0;
                red[(2 * warp + 1) * 2 + mat] = a1;
            }
        }
        named_bar_sync(1, kCons);
        if (warp == 0) {
            // rows of the group in lanes 0..15; RoPE partners (2i, 2i + 1) sit in adjacent lanes
            const int r = lane & 15;
            const bool ok = lane < 16 && r < rows;
            const float t = red[r * 2], t_up = NM == 2 ? red[r * 2 + 1] : 0.f;
            qmma::epilogue<EPI>(P, 16 * gi + r, ok, t, t_up, pos, rope_cs);
        }
        named_bar_sync(1, kCons);   // red is rewritten by the next group
    }
}

template <int ET, int EPI, int PRO>
ntx_status launch_e(Params P, cudaStream_t s)
{
    using E = Elem<ET>;
    auto kern = fgemv_kernel<ET, EPI, PRO>;
    const ntx_status st = ensure_smem_limit((const void*)kern, kSmemLimit);
    if (st != NTX_OK) return st;
    P.x_bytes = (P.K * 4 + 127) / 128 * 128;
    const int avail = kSmemLimit - kHeader - P.x_bytes;
    const int ns = std::min(kMaxStages, avail / kStageBytes);
    if (ns < 2) return fail(NTX_EUNSUPPORTED, "gemv (F16 / F32): row too long for the shared-memory pipeline");
    P.n_stages = ns;
    P.chunk_elems = E::CE;
    const int groups = (P.M + 15) / 16;
    const int grid = std::max(1, std::min(num_sms(), groups));
    const int smem = kHeader + P.x_bytes + ns * kStageBytes;
    return launch_kernel(kern, dim3(grid), dim3(kThreads), smem, s, P.use_pdl != 0, P);
}

template <int EPI, int PRO>
ntx_status launch_f(int qtype, const Params& P, cudaStream_t s)
{
    return qtype == NTX_F16 ? launch_e<NTX_F16, EPI, PRO>(P, s) : launch_e<NTX_F32, EPI, PRO>(P, s);
}

}  // namespace fgemv

bool fgemv_shape_ok(int qtype, const void* W, const void* x, int64_t cols)
{
    const int64_t rb = row_bytes(qtype, cols);
    return is_float_format(qtype) && aligned(W, 16) && aligned(x, 16) && rb % 16 == 0 && cols <= 32768;
}

ntx_status fgemv_launch(int qtype, int epi, int pro, const gemv::Params& P, cudaStream_t s)
{
    using namespace gemv;
    if (!is_float_format(qtype)) return fail(NTX_EINVAL, "gemv: not an F16 / F32 format");
    if (epi == EPI_STORE && pro == PRO_X) return fgemv::launch_f<EPI_STORE, PRO_X>(qtype, P, s);
    if (epi == EPI_ADD && pro == PRO_X) return fgemv::launch_f<EPI_ADD, PRO_X>(qtype, P, s);
    if (epi == EPI_SWIGLU && pro == PRO_RMSNORM) return fgemv::launch_f<EPI_SWIGLU, PRO_RMSNORM>(qtype, P, s);
    if (epi == EPI_QKV && pro == PRO_RMSNORM) return fgemv::launch_f<EPI_QKV, PRO_RMSNORM>(qtype, P, s);
    if (epi == EPI_STORE && pro == PRO_RMSNORM) return fgemv::launch_f<EPI_STORE, PRO_RMSNORM>(qtype, P, s);
    return fail(NTX_EUNSUPPORTED, "gemv: unsupported prologue / epilogue combination");
}

cudaError_t take_device_error_fgemv(uint32_t* out) { return take_tu_device_error(out); }

}  // namespace ntx
