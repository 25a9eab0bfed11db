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
template <int EPI>
struct Outs {
    static constexpr int value = EPI == EPI_SWIGLU ? kSlots / 2 : kSlots;
};

template <int QT, int EPI>
__device__ __forceinline__ const uint8_t* slot_src(const Params& P, int out_row, int slot)
{
    if (EPI == EPI_SWIGLU) {
        const int half = kSlots / 2;
        return slot < half ? P.W + (int64_t)(out_row + slot) * P.row_bytes
                           : P.W2 + (int64_t)(out_row + slot - half) * P.row_bytes;
    }
    return P.W + (int64_t)(out_row + slot) * P.row_bytes;
}

template <int EPI>
__device__ __forceinline__ bool slot_valid(int slot, int n_out)
{
    return EPI == EPI_SWIGLU ? ((slot & (kSlots / 2 - 1)) < n_out) : (slot < n_out);
}

// Epilogue for one finished output (thread i < outs of warp 0 after the reduction).
template <int EPI>
__device__ __forceinline__ void epilogue(const Params& P, const float* tot, int out_row, int i, int n_out,
                                         int32_t pos)
{
    if (EPI == EPI_STORE) {
        if (i < n_out) P.y[out_row + i] = tot[i];
    } else if (EPI == EPI_ADD) {
        if (i < n_out) P.y[out_row + i] = P.y[out_row + i] + tot[i];
    } else if (EPI == EPI_SWIGLU) {
        if (i < n_out) {
            const float g = tot[i], u = tot[kSlots / 2 + i];
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
                const double ang = (double)pos * pow((double)P.theta, -(2.0 * pi) / (double)hd);
                double s, c;
                sincos(ang, &s, &c);
                const float cf = (float)c, sf = (float)s;
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
    constexpr int OUTS = Outs<EPI>::value;

    extern __shared__ __align__(128) uint8_t smem[];
    uint64_t* full = reinterpret_cast<uint64_t*>(smem);
    uint64_t* empty = full + kMaxStages;
    float* red = reinterpret_cast<float*>(empty + kMaxStages);          // [2][8 warps][8]
    float* tot = red + 2 * kConsumerWarps * kSlots;                       // [2][8]
    float4* xs = reinterpret_cast<float4*>(smem + 1024);                  // x, P.x_bytes
    uint8_t* stages = smem + 1024 + P.x_bytes;                            // n_stages * stage_bytes

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
            int it = 0;
            bool okay = true;
            for (int g = 0; g < n_groups && okay; ++g) {
                const int out_row = r0 + g * OUTS;
                const int n_out = min(OUTS, r1 - out_row);
                for (int c = 0; c < P.n_chunks; ++c, ++it) {
                    const int s = it % P.n_stages;
                    const uint32_t round = (uint32_t)(it / P.n_stages);
                    if (!mbar_wait(&empty[s], (round & 1u) ^ 1u, kWaitPolls)) {
                        record_device_error(DEVERR_EMPTY_WAIT);
                        okay = false;
                        break;
                    }
                    const int c_elems = min(P.chunk_elems, P.K - c * P.chunk_elems);
                    const uint32_t c_bytes = (uint32_t)(c_elems / F::BE * F::BB);
                    int n_slots = 0;
#pragma unroll
                    for (int sl = 0; sl < kSlots; ++sl) n_slots += slot_valid<EPI>(sl, n_out) ? 1 : 0;
                    mbar_arrive_expect_tx(&full[s], c_bytes * (uint32_t)n_slots);
                    uint8_t* st = stages + (size_t)s * P.stage_bytes;
                    for (int sl = 0; sl < kSlots; ++sl) {
                        if (!slot_valid<EPI>(sl, n_out)) continue;
                        const uint8_t* src = slot_src<QT, EPI>(P, out_row, sl) + (int64_t)c * P.chunk_bytes;
                        bulk_g2s(st + (size_t)sl * P.chunk_bytes, src, c_bytes, &full[s], pol);
                    }
                }
            }
            // Drain: every stage the consumers have not consumed must complete before exit.
            if (!okay) {
                for (int k = 0; k < P.n_stages; ++k) {
                    const int j = it - 1 - k;
                    if (j < 0) break;
                    mbar_wait(&full[j % P.n_stages], (uint32_t)(j / P.n_stages) & 1u, 1u << 20);
                }
            }
        }
        return;
    }

    // ----------------------------------------------------------------- consumers
    if (P.use_pdl) pdl_wait();

    // Stage the input vector: x'' = x * 2^(S - p) in per-thread float4 pieces.
    float inv = 1.0f;
    if (PRO == PRO_RMSNORM) {
        float ss = 0.f;
        for (int i = tid; i < P.K; i += kConsumers) ss = fmaf(P.x[i], P.x[i], ss);
        ss = consumers_reduce(ss, red, false);
        inv = 1.0f / sqrtf(ss / (float)P.K + P.eps);
    }
    float mx = 0.f;
    for (int i = tid; i < P.K; i += kConsumers) {
        float v = P.x[i];
        if (PRO == PRO_RMSNORM) v = v * inv * P.norm_w[i];
        mx = fmaxf(mx, fabsf(v));
    }
    mx = consumers_reduce(mx, red, true);
    const int S = (mx > 0.f) ? max(-100, min(250, 120 - ilogbf(mx))) : 0;

    for (int c = 0; c < P.n_chunks; ++c) {
        const int c_elems = min(P.chunk_elems, P.K - c * P.chunk_elems);
        const int act = c_elems / E;                   // active threads of this chunk
        if (tid < act) {
            float4* dst = xs + (size_t)c * (P.chunk_elems / 4) + tid;
#pragma unroll
            for (int j = 0; j < NP; ++j) {
                float v4[4];
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    int e, p;
                    elem_of<QT>(tid, j, k, e, p);
                    const int gi = c * P.chunk_elems + e;
                    float v = P.x[gi];
                    if (PRO == PRO_RMSNORM) v = v * inv * P.norm_w[gi];
                    v4[k] = scale2(v, S - p);
                }
                dst[(size_t)j * act] = make_float4(v4[0], v4[1], v4[2], v4[3]);
            }
        }
    }
    named_bar_sync(1, kConsumers);

    const int32_t pos = (EPI == EPI_QKV) ? (P.pos_dev ? *P.pos_dev : P.pos) : 0;
    bool dead = false;
    int it = 0;
    for (int g = 0; g < n_groups; ++g) {
        const int out_row = r0 + g * OUTS;
        const int n_out = min(OUTS, r1 - out_row);
        float acc[kSlots];
#pragma unroll
        for (int sl = 0; sl < kSlots; ++sl) acc[sl] = 0.f;

        for (int c = 0; c < P.n_chunks; ++c, ++it) {
            const int s = it % P.n_stages;
            const uint32_t round = (uint32_t)(it / P.n_stages);
            const int c_elems = min(P.chunk_elems, P.K - c * P.chunk_elems);
            const int act = c_elems / E;
            const bool active = tid < act;
            // this thread's x pieces for chunk c, and the offset / min sums
            uint64_t xr[2 * NP];
            float offs[4] = {0.f, 0.f, 0.f, 0.f};
            if (active) {
                const float4* src = xs + (size_t)c * (P.chunk_elems / 4) + tid;
#pragma unroll
                for (int j = 0; j < NP; ++j) {
                    const float4 v = src[(size_t)j * act];
                    xr[2 * j] = pack2(__float_as_uint(v.x), __float_as_uint(v.y));
                    xr[2 * j + 1] = pack2(__float_as_uint(v.z), __float_as_uint(v.w));
                    const float vv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
                    for (int k = 0; k < 4; ++k) {
                        int e, p;
                        elem_of<QT>(tid, j, k, e, p);
                        // offset code at bit p as an fp32 bit pattern (value code * 2^(p-149))
                        const uint32_t code = QT == NTX_Q8_0 ? 128u : QT == NTX_Q4_0 ? 8u : QT == NTX_Q6_K ? 32u : 1u;
                        const float unit = __uint_as_float(code << p);
                        const int grp = QT == NTX_Q4_K ? (j >> 2) : QT == NTX_Q6_K ? (j >> 1) : 0;
                        offs[grp] = fmaf(unit, vv[k], offs[grp]);
                    }
                }
            }
            if (!dead && !mbar_wait(&full[s], round & 1u, kWaitPolls)) {
                record_device_error(DEVERR_FULL_WAIT);
                dead = true;    // keep taking part in every barrier so the CTA still finishes
            }
            const uint8_t* st = stages + (size_t)s * P.stage_bytes;
            if (active && !dead) {
#pragma unroll
                for (int sl = 0; sl < kSlots; ++sl) {
                    if (!slot_valid<EPI>(sl, n_out)) continue;
                    const uint8_t* rowp = st + (size_t)sl * P.chunk_bytes;
                    float v;
                    if constexpr (QT == NTX_Q8_0) {
                        v = Dot<NTX_Q8_0>::row(rowp, tid, reinterpret_cast<const uint64_t(&)[8]>(xr), offs[0]);
                    } else if constexpr (QT == NTX_Q4_0) {
                        v = Dot<NTX_Q4_0>::row(rowp, tid, reinterpret_cast<const uint64_t(&)[8]>(xr), offs[0]);
                    } else if constexpr (QT == NTX_Q4_K) {
                        v = Dot<NTX_Q4_K>::row(rowp, tid, reinterpret_cast<const uint64_t(&)[16]>(xr), offs[0],
                                               offs[1]);
                    } else {
                        v = Dot<NTX_Q6_K>::row(rowp, tid, reinterpret_cast<const uint64_t(&)[16]>(xr), offs);
                    }
                    acc[sl] += v;
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[s]);
        }

        // ---- reduce the 8 row partials over the CTA (transposed butterfly)
        {
            float v4[4], v2[2], v1;
            const bool b4 = lane & 16, b3 = lane & 8, b2 = lane & 4;
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const float send = b4 ? acc[k] : acc[k + 4];
                const float keep = b4 ? acc[k + 4] : acc[k];
                v4[k] = keep + __shfl_xor_sync(0xffffffffu, send, 16);
            }
#pragma unroll
            for (int k = 0; k < 2; ++k) {
                const float send = b3 ? v4[k] : v4[k + 2];
                const float keep = b3 ? v4[k + 2] : v4[k];
                v2[k] = keep + __shfl_xor_sync(0xffffffffu, send, 8);
            }
            {
                const float send = b2 ? v2[0] : v2[1];
                const float keep = b2 ? v2[1] : v2[0];
                v1 = keep + __shfl_xor_sync(0xffffffffu, send, 4);
            }
            v1 += __shfl_xor_sync(0xffffffffu, v1, 2);
            v1 += __shfl_xor_sync(0xffffffffu, v1, 1);
            // lane holds the row (b4 ? 4 : 0) + (b3 ? 2 : 0) + (b2 ? 1 : 0)
            float* rb = red + (g & 1) * kConsumerWarps * kSlots;
            if ((lane & 3) == 0) rb[warp * kSlots + ((lane >> 4) & 1) * 4 + ((lane >> 3) & 1) * 2 + ((lane >> 2) & 1)] = v1;
            named_bar_sync(1, kConsumers);
            if (tid < kSlots) {
                float t = 0.f;
#pragma unroll
                for (int w = 0; w < kConsumerWarps; ++w) t += rb[w * kSlots + tid];
                tot[(g & 1) * kSlots + tid] = scale2(t, 149 - S);
            }
            if (warp == 0) {
                __syncwarp();
                const float* tg = tot + (g & 1) * kSlots;
                if (tid < OUTS) epilogue<EPI>(P, tg, out_row, tid, n_out, pos);
            }
        }
    }
}

}  // namespace gemv
}  // namespace ntx
