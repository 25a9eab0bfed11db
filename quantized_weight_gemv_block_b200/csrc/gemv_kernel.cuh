// gemv_kernel.cuh - the pipelined block-quantized GEMV kernel (see gemv.cuh).
#pragma once

#include "gemv.cuh"

namespace ntx {
namespace gemv {

// Rows [r0, r1) of output handled by CTA `cta` of `n_cta`, split in whole pairs so a
// RoPE pair (2i, 2i+1) never straddles two CTAs.
__device__ __forceinline__ void cta_rows(int M, int cta, int n_cta, int& r0, int& r1)
{
    const long long pairs = (M + 1) / 2;
    r0 = (int)(2 * (pairs * cta / n_cta));
    r1 = (int)(2 * (pairs * (cta + 1) / n_cta));
    if (r1 > M) r1 = M;
    if (r0 > M) r0 = M;
}

// Outputs per stage: 8 rows, or 4 gate/up pairs for SwiGLU.
template <int QT, int EPI>
struct Outs {
    static constexpr int value = EPI == EPI_SWIGLU ? Slots<QT>::value / 2 : Slots<QT>::value;
};

template <int QT, int EPI>
__device__ __forceinline__ const uint8_t* slot_src(const Params& P, int out_row, int slot)
{
    if (EPI == EPI_SWIGLU) {
        const int half = Slots<QT>::value / 2;
        return slot < half ? P.W + (int64_t)(out_row + slot) * P.row_bytes
                           : P.W2 + (int64_t)(out_row + slot - half) * P.row_bytes;
    }
    return P.W + (int64_t)(out_row + slot) * P.row_bytes;
}

template <int QT, int EPI>
__device__ __forceinline__ bool slot_valid(int slot, int n_out)
{
    return EPI == EPI_SWIGLU ? ((slot & (Slots<QT>::value / 2 - 1)) < n_out) : (slot < n_out);
}

// Epilogue for one finished output (thread i < outs of warp 0 after the reduction).
template <int QT, int EPI>
__device__ __forceinline__ void epilogue(const Params& P, const float* tot, int out_row, int i, int n_out,
                                         int32_t pos, const float* rope_cs)
{
    if (EPI == EPI_STORE) {
        if (i < n_out) P.y[out_row + i] = tot[i];
    } else if (EPI == EPI_ADD) {
        if (i < n_out) P.y[out_row + i] = P.y[out_row + i] + tot[i];
    } else if (EPI == EPI_SWIGLU) {
        if (i < n_out) {
            const float g = tot[i], u = tot[Slots<QT>::value / 2 + i];
            P.y[out_row + i] = g / (1.0f + expf(-g)) * u;
        }
    } else if (EPI == EPI_QKV) {
        // rows: q [0, q_rows), k [q_rows, q_rows + kv_rows), v after; RoPE on (2i, 2i+1)
        if (i < n_out && (i & 1) == 0) {
            const int r = out_row + i;
            float a = tot[i];
            float b = (i + 1 < n_out) ? tot[i + 1] : 0.f;
            const int hd = P.head_dim;
            if (r < P.q_rows + P.kv_rows) {
                const int pi = (r % hd) / 2;
                const float cf = rope_cs[2 * pi], sf = rope_cs[2 * pi + 1];
                const float ra = a * cf - b * sf, rb = a * sf + b * cf;
                a = ra;
                b = rb;
            }
            for (int k = 0; k < 2 && i + k < n_out; ++k) {
                const int rr = r + k;
                const float v = k == 0 ? a : b;
                if (rr < P.q_rows) {
                    P.q_out[rr] = v;
                } else {
                    const int kvr = rr - P.q_rows;
                    const bool is_v = kvr >= P.kv_rows;
                    const int j = is_v ? kvr - P.kv_rows : kvr;
                    const int g = j / hd, dd = j % hd;
                    __half* cache = is_v ? P.v_cache : P.k_cache;
                    cache[((int64_t)g * P.max_ctx + pos) * hd + dd] = __float2half_rn(v);
                }
            }
        }
    }
}

template <int QT, int EPI, int PRO>
__global__ void __launch_bounds__(kThreads, 1) gemv_kernel(const Params P)
{
    using F = Fmt<QT>;
    constexpr int E = F::E;
    constexpr int NP = E / 4;      // float4 pieces per thread per chunk
    constexpr int SL = Slots<QT>::value;
    constexpr int R = Slots<QT>::per_thread;
    constexpr int OUTS = Outs<QT, EPI>::value;

    extern __shared__ __align__(128) uint8_t smem[];
    uint64_t* full = reinterpret_cast<uint64_t*>(smem);
    uint64_t* empty = full + kMaxStages;
    float* red = reinterpret_cast<float*>(empty + kMaxStages);          // [2][16 warps][R]
    float* tot = red + 2 * kConsumerWarps * R;                            // [2][SL]
    float* rope_cs = reinterpret_cast<float*>(smem + kHeader - 512);       // [head_dim / 2 <= 64][cos, sin]
    float4* xs = reinterpret_cast<float4*>(smem + kHeader);               // x, P.x_bytes
    uint8_t* stages = smem + kHeader + P.x_bytes;                         // n_stages * stage_bytes

    const int tid = threadIdx.x;
    const int warp = tid >> 5, lane = tid & 31;
    int r0, r1;
    cta_rows(P.M, blockIdx.x, gridDim.x, r0, r1);

    if (tid == 0) {
        for (int s = 0; s < P.n_stages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], kConsumerWarps);
        }
        fence_mbar_init();
    }
    __syncthreads();
    if (P.use_pdl) pdl_launch_dependents();

    const int n_groups = (r1 - r0 + OUTS - 1) / OUTS;

    if (warp == kConsumerWarps) {
        // ------------------------------------------------------------- producer
        if (lane == 0) {
            const uint64_t pol = policy_evict_first();
            const int NS = P.n_stages, NCH = P.n_chunks, CE = P.chunk_elems, CB = P.chunk_bytes, K = P.K;
            const int SB = P.stage_bytes;
            int s = 0, issued = 0;
            uint32_t ph = 0;
            bool okay = true;
            for (int g = 0; g < n_groups && okay; ++g) {
                const int out_row = r0 + g * OUTS;
                const int n_out = min(OUTS, r1 - out_row);
                int n_slots = 0;
#pragma unroll
                for (int sl = 0; sl < SL; ++sl) n_slots += slot_valid<QT, EPI>(sl, n_out) ? 1 : 0;
                for (int c = 0; c < NCH; ++c) {
                    if (!mbar_wait(&empty[s], ph ^ 1u, kWaitPolls)) {
                        record_device_error(DEVERR_EMPTY_WAIT);
                        okay = false;
                        break;
                    }
                    const int c_elems = min(CE, K - c * CE);
                    const uint32_t c_bytes = (uint32_t)(c_elems / F::BE * F::BB);
                    mbar_arrive_expect_tx(&full[s], c_bytes * (uint32_t)n_slots);
                    uint8_t* st = stages + (size_t)s * SB;
                    for (int sl = 0; sl < SL; ++sl) {
                        if (!slot_valid<QT, EPI>(sl, n_out)) continue;
                        const uint8_t* src = slot_src<QT, EPI>(P, out_row, sl) + (int64_t)c * CB;
                        bulk_g2s(st + (size_t)sl * CB, src, c_bytes, &full[s], pol);
                    }
                    ++issued;
                    if (++s == NS) {
                        s = 0;
                        ph ^= 1u;
                    }
                }
            }
            // Drain: the stages issued last must complete before the CTA may exit.
            if (!okay) {
                for (int k = 1; k <= NS && k <= issued; ++k) {
                    const int j = issued - k;
                    mbar_wait(&full[j % NS], (uint32_t)(j / NS) & 1u, 1u << 20);
                }
            }
        }
        return;
    }

    // ----------------------------------------------------------------- consumers
    // 16 consumer warps in two groups of 256 threads: both groups read the same
    // input values (thread lt = tid & 255 owns E elements of each chunk); group A
    // handles row slots 0-3 of every stage, group B slots 4-7.
    const int lt = tid & (kOwners - 1);
    const int grp = tid >> 8;
    if (P.use_pdl) pdl_wait();

    // Stage the input vector.  (1) coalesced copy into shared memory in natural
    // order (RMSNorm applied, statistics gathered); (2) per chunk, in place, into
    // the per-thread layout, pre-scaled by 2^(S - p) for the code field at bit p.
    float* xn = reinterpret_cast<float*>(xs);
    const int K4 = P.K / 4;
    const float4* x4 = reinterpret_cast<const float4*>(P.x);
    float inv = 1.0f;
    if (PRO == PRO_RMSNORM) {
        float ss = 0.f;
        for (int i = tid; i < K4; i += kConsumers) {
            const float4 v = x4[i];
            xs[i] = v;
            ss = fmaf(v.x, v.x, fmaf(v.y, v.y, fmaf(v.z, v.z, fmaf(v.w, v.w, ss))));
        }
        ss = consumers_reduce(ss, red, false);
        inv = 1.0f / sqrtf(ss / (float)P.K + P.eps);
    }
    float mx = 0.f;
    {
        const float4* w4 = reinterpret_cast<const float4*>(P.norm_w);
        for (int i = tid; i < K4; i += kConsumers) {
            float4 v;
            if (PRO == PRO_RMSNORM) {
                const float4 a = xs[i], w = w4[i];
                v = make_float4(a.x * inv * w.x, a.y * inv * w.y, a.z * inv * w.z, a.w * inv * w.w);
            } else {
                v = x4[i];
            }
            xs[i] = v;
            mx = fmaxf(mx, fmaxf(fmaxf(fabsf(v.x), fabsf(v.y)), fmaxf(fabsf(v.z), fabsf(v.w))));
        }
    }
    mx = consumers_reduce(mx, red, true);      // also orders the natural copy before the swizzle
    const int S = (mx > 0.f) ? max(-100, min(250, 120 - ilogbf(mx))) : 0;

    for (int c = 0; c < P.n_chunks; ++c) {
        const int c_elems = min(P.chunk_elems, P.K - c * P.chunk_elems);
        const int act = c_elems / E;
        float* base = xn + (size_t)c * P.chunk_elems;
        float4 piece[NP];
        if (grp == 0 && lt < act) {
#pragma unroll
            for (int j = 0; j < NP; ++j) {
                int e, p;
                elem_of<QT>(lt, j, 0, e, p);
                const float4 v = *reinterpret_cast<const float4*>(base + e);
                const float vv[4] = {v.x, v.y, v.z, v.w};
                float o[4];
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    elem_of<QT>(lt, j, k, e, p);
                    o[k] = scale2(vv[k], S - p);
                }
                piece[j] = make_float4(o[0], o[1], o[2], o[3]);
            }
        }
        named_bar_sync(1, kConsumers);
        if (grp == 0 && lt < act) {
            float4* dst = reinterpret_cast<float4*>(base) + lt;
#pragma unroll
            for (int j = 0; j < NP; ++j) dst[(size_t)j * act] = piece[j];
        }
        named_bar_sync(1, kConsumers);
    }

    const int32_t pos = (EPI == EPI_QKV) ? (P.pos_dev ? *P.pos_dev : P.pos) : 0;
    if (EPI == EPI_QKV && tid < P.head_dim) rope_cs[tid] = P.rope_cs[tid];   // the step's RoPE table
    bool dead = false;
    // this thread's x pieces of a chunk, and the offset / min sums of its elements
    uint64_t xr[2 * NP];
    float offs[4] = {0.f, 0.f, 0.f, 0.f};
    auto load_x = [&](int c, int act) {
        const float4* src = xs + (size_t)c * (P.chunk_elems / 4) + lt;
        offs[0] = offs[1] = offs[2] = offs[3] = 0.f;
#pragma unroll
        for (int j = 0; j < NP; ++j) {
            const float4 v = src[(size_t)j * act];
            xr[2 * j] = pack2(__float_as_uint(v.x), __float_as_uint(v.y));
            xr[2 * j + 1] = pack2(__float_as_uint(v.z), __float_as_uint(v.w));
            const float vv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                int e, p;
                elem_of<QT>(lt, j, k, e, p);
                // offset code at bit p as an fp32 bit pattern (value code * 2^(p-149))
                constexpr int B = QT;
                const uint32_t code = B == NTX_Q8_0 ? 128u : B == NTX_Q4_0 ? 8u : B == NTX_Q6_K ? 32u : 1u;
                const float unit = __uint_as_float(code << p);
                const int og = B == NTX_Q4_K ? (j >> 2) : B == NTX_Q6_K ? (j >> 1) : 0;
                offs[og] = fmaf(unit, vv[k], offs[og]);
            }
        }
    };
    const int NS = P.n_stages, NCH = P.n_chunks, CE = P.chunk_elems, K = P.K;
    const int CB = P.chunk_bytes, SB = P.stage_bytes;
    const bool one_chunk = NCH == 1;
    if (one_chunk && lt < K / E) load_x(0, K / E);
    const uint8_t* my_stage0 = stages + (size_t)(grp * R) * CB;
    int s = 0;
    uint32_t ph = 0;
    for (int g = 0; g < n_groups; ++g) {
        const int out_row = r0 + g * OUTS;
        const int n_out = min(OUTS, r1 - out_row);
        float acc[R];
#pragma unroll
        for (int r = 0; r < R; ++r) acc[r] = 0.f;

        for (int c = 0; c < NCH; ++c) {
            const int act = one_chunk ? K / E : min(CE, K - c * CE) / E;
            const bool active = lt < act;
            if (active && !one_chunk) load_x(c, act);
            if (!dead && !mbar_wait(&full[s], ph, kWaitPolls)) {
                record_device_error(DEVERR_FULL_WAIT);
                dead = true;    // keep taking part in every barrier so the CTA still finishes
            }
            const uint8_t* b = my_stage0 + (size_t)s * SB;
            if (active && !dead) {
                // rows past the end of a partial group hold stale bytes; their sums are never stored
#pragma unroll
                for (int r = 0; r < R; ++r)
                    acc[r] += dot_row<QT>(b + (size_t)r * CB, lt, xr, offs, P);
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[s]);
            if (++s == NS) {
                s = 0;
                ph ^= 1u;
            }
        }

        // ---- reduce the R row partials of each group over its 256 threads (transposed butterfly)
        {
            // halving rounds at lane strides 16, 8, ... keep R/2, R/4, ... rows per lane; then
            // the remaining strides sum the single row each lane holds
            float v[R];
#pragma unroll
            for (int k = 0; k < R; ++k) v[k] = acc[k];
            int row = 0;
#pragma unroll
            for (int n = R, sh = 16; n > 1; n >>= 1, sh >>= 1) {
                const bool hi = (lane & sh) != 0;
#pragma unroll
                for (int k = 0; k < n / 2; ++k) {
                    const float send = hi ? v[k] : v[k + n / 2];
                    const float keep = hi ? v[k + n / 2] : v[k];
                    v[k] = keep + __shfl_xor_sync(0xffffffffu, send, sh);
                }
                row += hi ? n / 2 : 0;
            }
            float v1 = v[0];
#pragma unroll
            for (int sh = 32 / R / 2; sh > 0; sh >>= 1) v1 += __shfl_xor_sync(0xffffffffu, v1, sh);
            float* rb = red + (g & 1) * kConsumerWarps * R;
            if ((lane & (32 / R - 1)) == 0) rb[warp * R + row] = v1;
            named_bar_sync(1, kConsumers);
            if (tid < SL) {
                const int gsel = tid / R, rr = tid % R;
                float t = 0.f;
#pragma unroll
                for (int w = 0; w < kConsumerWarps / 2; ++w) t += rb[(gsel * (kConsumerWarps / 2) + w) * R + rr];
                tot[(g & 1) * SL + tid] = scale2(t, 149 - S);
            }
            if (warp == 0) {
                __syncwarp();
                const float* tg = tot + (g & 1) * SL;
                if (tid < OUTS) epilogue<QT, EPI>(P, tg, out_row, tid, n_out, pos, rope_cs);
            }
        }
    }
}

}  // namespace gemv
}  // namespace ntx
