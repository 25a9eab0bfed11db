// attn.cu - GQA decode attention of one query token over the fp16 KV cache
// (attention with GQA of the ntransformer news summary, "Funciones principales";
// F16 KV cache of "Hoja de ruta de desarrollo", Fase 3), split over the context.
//
// Grid: n_kv_heads x n_split CTAs, one per SM.  CTA (g, s) takes positions
// [s P, s P + P) of kv head g together with the G = n_q / n_kv query heads that
// read it, so every K / V row is fetched from HBM once:
//  * a producer warp streams the range in stages of 64 positions (K rows and V
//    rows, 32 KB) into a ring of shared-memory stages with TMA tensor copies of
//    64 x 64 fp16 boxes in the 128-byte swizzle, so the tensor-core operand loads
//    (ldmatrix, 8 rows of one column) hit 8 different bank groups;
//  * both contractions run on the tensor cores (mma.sync m16n8k16, fp16
//    operands, fp32 accumulation), in two warp roles that overlap across stages:
//    4 score warps form S^T = K q^T (q split into an fp16 high part and an fp16
//    remainder, two products, so q keeps ~22 bits) and run the online softmax
//    (running max m per query head, per-lane shares of the running sum l), and
//    hand P and the rescale factors of stage i through a double buffer to 8 P.V
//    warps, which form O^T = V^T P^T (P split the same way) while the score warps
//    move on to stage i + 1.  K and V are fp16 already, so every product is exact
//    and only the fp32 accumulation rounds;
//  * the partial (m, l, acc[128]) of each query head goes to the workspace, and a
//    second kernel (one CTA per query head, launched as a programmatic dependent)
//    merges the splits with the log-sum-exp rule in a fixed order, so the result
//    is deterministic.
// Every wait is bounded; a wait that runs out records an error and the CTA still
// finishes.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <mutex>

#include "ops.h"

namespace ntx {
namespace {

constexpr int HD = 128;
constexpr int kSWarps = 4;                        // score + softmax warps, 16 positions each
constexpr int kPVWarps = 8;                       // P.V warps, 16 dims each
constexpr int kProducerWarp = kSWarps + kPVWarps;
constexpr int kThreads = (kProducerWarp + 1) * 32;
constexpr int kSub = 64;                          // positions per stage
constexpr int kBoxBytes = kSub * 128;             // 64 rows x 64 dims fp16, swizzled 128 B rows
constexpr int kStageBytes = 4 * kBoxBytes;        // K dims 0-63, 64-127, then V the same
constexpr int kStages = 4;
constexpr int kPartFloats = 4 + HD;               // m, l, 2 pad, acc[128]: 528-byte records
constexpr int kMaxSplit = 128;
constexpr uint32_t kPolls = 1u << 22;

struct KArgs {
    CUtensorMap tk, tv;         // K and V caches as [n_kv][max_ctx][128] fp16, 64 x 64 boxes
    const float* q;
    float* out;
    float* part;
    int max_ctx, n_split;
    int32_t n_ctx;
    const int32_t* pos_dev;
    int use_pdl;
    KvPrefetch pf;              // the next layer's rows [0, pos), fetched into L2 (k null: none)
};

// Tensor-core helpers (mma.sync m16n8k16, fp16 in, fp32 accumulate).
__device__ __forceinline__ void mma_f16(float (&c)[4], const uint32_t (&a)[4], const uint32_t (&b)[2])
{
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b[0]), "r"(b[1]));
}

__device__ __forceinline__ void ldsm_x4(uint32_t (&r)[4], const void* p)
{
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(smem_addr(p)));
}

__device__ __forceinline__ void ldsm_x4_trans(uint32_t (&r)[4], const void* p)
{
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(smem_addr(p)));
}

// (x, y) as an fp16 pair (element x in the low half) plus the fp16 pair of what
// that rounding left out; hi + lo carries ~22 significant bits of each value.
__device__ __forceinline__ void split_f16x2(float x, float y, uint32_t& hi, uint32_t& lo)
{
    const __half2 h = __floats2half2_rn(x, y);
    const float2 hf = __half22float2(h);
    const __half2 l = __floats2half2_rn(x - hf.x, y - hf.y);
    hi = *reinterpret_cast<const uint32_t*>(&h);
    lo = *reinterpret_cast<const uint32_t*>(&l);
}

// shared-memory layout (bytes)
constexpr int kOffBars = 0;      // full[4], empty[4], pfull[2], pempty[2]
constexpr int kOffWMax = 256;    // [2][4 warps][8 heads] stage maxima of the score warps
constexpr int kOffWSum = 512;    // [4 warps][8 heads] final sums
constexpr int kOffAlpha = 640;   // [2][8] rescale factors of the running accumulators
constexpr int kScStride = kSub + 8;                     // floats per head row of P (bank spread)
constexpr int kOffP = 1024;                             // P[2][8 heads][72] floats
constexpr int kOffRing = (kOffP + 2 * 8 * kScStride * 4 + 1023) & ~1023;   // the swizzle repeats every 1024 B
constexpr int kSmem = kOffRing + kStages * kStageBytes;

// Byte offset of 16-byte chunk c (dims 8c .. 8c + 7) of row r inside a swizzled
// 64 x 64 box: chunk index XOR (row mod 8), as the 128-byte TMA swizzle stores it.
__device__ __forceinline__ uint32_t swz(int r, int c) { return (uint32_t)(r * 128 + (((c ^ r) & 7) << 4)); }

__device__ __forceinline__ void tma_box(void* dst, const CUtensorMap* map, int x, int y, int z, uint64_t* bar,
                                        uint64_t policy)
{
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint "
        "[%0], [%1, {%2, %3, %4}], [%5], %6;" ::"r"(smem_addr(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(z), "r"(smem_addr(bar)), "l"(policy)
        : "memory");
}

// This CTA's share (b of G) of the rows of p (none when p.k is null): CTA b takes head
// region r = b mod R (R = 2 n_kv: the K heads, then the V heads) and slice j = b / R of the
// CTAs that share it.  32-bit index arithmetic only (a 64-bit division would raise the
// register count of the whole kernel).
__device__ __forceinline__ void kv_prefetch_share(const KvPrefetch& p, int b, int G, int pos)
{
    const int R = 2 * p.n_kv;
    if (!p.k || pos <= 0 || R <= 0) return;
    const int r = b % R, j = b / R, k = (G - r + R - 1) / R;
    const int r0 = (int)((unsigned)pos * (unsigned)j / (unsigned)k);
    const int r1 = (int)((unsigned)pos * (unsigned)(j + 1) / (unsigned)k);
    const uint8_t* base = (r < p.n_kv ? p.k : p.v) + (int64_t)(r < p.n_kv ? r : r - p.n_kv) * p.head_stride;
    const uint8_t* q = base + (int64_t)r0 * p.row_b;
    int64_t n = (int64_t)(r1 - r0) * p.row_b;   // a multiple of 16: row_b is
    while (n > 0) {
        const uint32_t c = (uint32_t)(n < 65536 ? n : 65536);
        asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(q), "r"(c) : "memory");
        q += c;
        n -= c;
    }
}

template <int G>
__global__ void __launch_bounds__(kThreads, 1) attn_kernel(const __grid_constant__ KArgs a)
{
    extern __shared__ __align__(1024) uint8_t sm[];
    uint64_t* full = reinterpret_cast<uint64_t*>(sm + kOffBars);
    uint64_t* empty = full + kStages;
    uint64_t* pfull = empty + kStages;
    uint64_t* pempty = pfull + 2;
    float* wmax = reinterpret_cast<float*>(sm + kOffWMax);
    float* wsum = reinterpret_cast<float*>(sm + kOffWSum);
    float* s_alpha = reinterpret_cast<float*>(sm + kOffAlpha);
    float* Pbuf = reinterpret_cast<float*>(sm + kOffP);
    uint8_t* ring = sm + kOffRing;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    if (warp == kProducerWarp && lane == 0) {
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&a.tk)) : "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&a.tv)) : "memory");
    }
    if (smem_addr(ring) & 1023u) {
        // the swizzled boxes need a 1024-byte aligned ring; never issue a copy otherwise
        if (tid == 0) record_device_error(DEVERR_SMEM_ALIGN);
        return;
    }
    if (tid == 0) {
        for (int i = 0; i < kStages; ++i) {
            mbar_init(&full[i], 1);
            mbar_init(&empty[i], kSWarps + kPVWarps);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&pfull[b], kSWarps);
            mbar_init(&pempty[b], kPVWarps);
        }
        fence_mbar_init();
    }
    __syncthreads();
    // Programmatic dependent launch: the consumers wait for the previous kernel (which
    // writes q and the K / V row at the new position) before reading anything; the
    // producer waits only before the first stage that holds that row, since older rows
    // were written by earlier steps (the step word was written before the first kernel
    // that launches early).
    if (a.use_pdl) {
        pdl_launch_dependents();
        if (warp != kProducerWarp) pdl_wait();
    }
    const int g = blockIdx.x / a.n_split, sp = blockIdx.x % a.n_split;
    const int n_ctx = a.pos_dev ? (*a.pos_dev + 1) : a.n_ctx;
    const int P = (n_ctx + a.n_split - 1) / a.n_split;
    const int t0 = sp * P;
    const int np = max(0, min(n_ctx, t0 + P) - t0);
    const int nsub = (np + kSub - 1) / kSub;
    const int gid = lane >> 2, tig = lane & 3;
    float* part = a.part + (size_t)(g * a.n_split + sp) * G * kPartFloats;

    if (warp == kProducerWarp) {
        // ------------------------------------------------------------ producer
        const uint64_t pol = policy_evict_first();
        int s = 0;
        uint32_t ph = 0;
        bool waited = !a.use_pdl;
        for (int i = 0; i < nsub && lane == 0; ++i) {
            if (!waited && t0 + (i + 1) * kSub > n_ctx - 1) {
                pdl_wait();
                waited = true;
            }
            if (!mbar_wait(&empty[s], ph ^ 1u, kPolls)) {
                record_device_error(DEVERR_EMPTY_WAIT);
                // the stages issued last must land before the CTA may exit
                for (int k = 1; k <= kStages && k <= i; ++k) {
                    const int jj = i - k;
                    mbar_wait(&full[jj % kStages], (uint32_t)(jj / kStages) & 1u, 1u << 20);
                }
                break;
            }
            // whole boxes always arrive: rows past the context are zero-filled or masked later
            uint8_t* st = ring + s * kStageBytes;
            const int y = t0 + i * kSub;
            mbar_arrive_expect_tx(&full[s], (uint32_t)kStageBytes);
            tma_box(st, &a.tk, 0, y, g, &full[s], pol);
            tma_box(st + kBoxBytes, &a.tk, 64, y, g, &full[s], pol);
            tma_box(st + 2 * kBoxBytes, &a.tv, 0, y, g, &full[s], pol);
            tma_box(st + 3 * kBoxBytes, &a.tv, 64, y, g, &full[s], pol);
            if (++s == kStages) {
                s = 0;
                ph ^= 1u;
            }
        }
        // every copy of this CTA is under way: the rows the next layer's attention will read
        // at this position come from HBM into L2 now, while the GEMVs in between stream
        // their weights with the evict-first policy
        if (lane == 0) kv_prefetch_share(a.pf, blockIdx.x, gridDim.x, n_ctx - 1);
    } else if (warp < kSWarps) {
        // ------------------------------------------- score and softmax warps
        // S^T[position][head] = K q^T for positions 16 warp .. +15 of each stage.  q^T is
        // the B operand (k = dim, n = head): each head is brought to max |q| in [1, 2)
        // by a power of two (undone on the scores, exactly), then split into an fp16
        // high part and an fp16 remainder; heads >= G are zero.  The four lanes of a
        // quad (same gid) hold the 128 dims of head gid.
        uint32_t qh[8][2], ql[8][2];
        float mul0, mul1;   // score multipliers of heads 2 tig and 2 tig + 1
        {
            const float* qrow = a.q + (int64_t)(g * G + gid) * HD;
            float2 v[8][2];
            float mx = 0.f;
#pragma unroll
            for (int ks = 0; ks < 8; ++ks) {
#pragma unroll
                for (int half = 0; half < 2; ++half) {
                    v[ks][half] = make_float2(0.f, 0.f);
                    if (gid < G) v[ks][half] = *reinterpret_cast<const float2*>(qrow + 16 * ks + 8 * half + 2 * tig);
                    mx = fmaxf(mx, fmaxf(fabsf(v[ks][half].x), fabsf(v[ks][half].y)));
                }
            }
            mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
            mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
            // e = floor(log2 mx) from the bit pattern (mx normal); zero or subnormal heads keep e = 0
            int e = 0;
            if (mx >= 1.17549435e-38f && mx <= 3.4e38f) e = (int)((__float_as_uint(mx) >> 23) & 0xffu) - 127;
            e = max(-100, min(100, e));
            const float down = __uint_as_float((uint32_t)(127 - e) << 23);
            // scores carry 1/sqrt(128) = 2^-3.5: 2^-4 goes into the exponent, sqrt(2) stays a multiply
            const float up = __uint_as_float((uint32_t)(127 + e - 4) << 23) * 1.41421356237309515f;
            mul0 = __shfl_sync(0xffffffffu, up, (2 * tig) << 2);
            mul1 = __shfl_sync(0xffffffffu, up, (2 * tig + 1) << 2);
#pragma unroll
            for (int ks = 0; ks < 8; ++ks)
#pragma unroll
                for (int half = 0; half < 2; ++half)
                    split_f16x2(v[ks][half].x * down, v[ks][half].y * down, qh[ks][half], ql[ks][half]);
        }
        // running max of heads 2 tig, 2 tig + 1 (identical in every lane with this tig)
        // and this lane's share of the running sums
        float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;
        const int m0w = 16 * warp;
        const int j = lane >> 3, r = m0w + ((j & 1) << 3) + (lane & 7);
        int s = 0;
        uint32_t ph = 0;
        for (int i = 0; i < nsub; ++i) {
            const int cnt = min(kSub, np - i * kSub);
            const int b = i & 1;
            const bool ok_full = mbar_wait(&full[s], ph, kPolls);
            const bool ok_p = mbar_wait(&pempty[b], ((uint32_t)(i >> 1) & 1u) ^ 1u, kPolls);
            if (!ok_full || !ok_p) record_device_error(DEVERR_FULL_WAIT);
            const uint8_t* Ks = ring + s * kStageBytes;
            // ldmatrix: lane -> matrix j = lane / 8 (rows +8 if j odd, dims +8 if j >= 2), row lane % 8;
            // four accumulation chains (dims 0-63 / 64-127, high / low part of q)
            float c[4][4] = {};
            if (m0w < cnt) {
#pragma unroll
                for (int ks = 0; ks < 8; ++ks) {
                    uint32_t av[4];
                    ldsm_x4(av, Ks + (ks >> 2) * kBoxBytes + swz(r, 2 * ks + (j >> 1)));
                    mma_f16(c[(ks >> 2) * 2], av, qh[ks]);
                    mma_f16(c[(ks >> 2) * 2 + 1], av, ql[ks]);
                }
            }
            // K of this stage is no longer needed by this warp
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[s]);
            // sc[q]: q = 0 position gid, head 2 tig; 1 same position, head 2 tig + 1; 2, 3 position gid + 8
            const bool v0 = m0w + gid < cnt, v1 = m0w + gid + 8 < cnt;
            float sc[4];
#pragma unroll
            for (int q = 0; q < 4; ++q) sc[q] = ((c[0][q] + c[1][q]) + (c[2][q] + c[3][q])) * ((q & 1) ? mul1 : mul0);
            if (!v0) sc[0] = sc[1] = -INFINITY;
            if (!v1) sc[2] = sc[3] = -INFINITY;
            // stage maximum per head: this warp's 16 positions, then the four warps'
            float x0 = fmaxf(sc[0], sc[2]), x1 = fmaxf(sc[1], sc[3]);
#pragma unroll
            for (int o = 4; o < 32; o <<= 1) {
                x0 = fmaxf(x0, __shfl_xor_sync(0xffffffffu, x0, o));
                x1 = fmaxf(x1, __shfl_xor_sync(0xffffffffu, x1, o));
            }
            float* wm = wmax + b * (kSWarps * 8);
            if (gid == 0) {
                wm[warp * 8 + 2 * tig] = x0;
                wm[warp * 8 + 2 * tig + 1] = x1;
            }
            named_bar_sync(2, kSWarps * 32);
#pragma unroll
            for (int w = 0; w < kSWarps; ++w) {
                x0 = fmaxf(x0, wm[w * 8 + 2 * tig]);
                x1 = fmaxf(x1, wm[w * 8 + 2 * tig + 1]);
            }
            const float n0 = fmaxf(m0, x0), n1 = fmaxf(m1, x1);
            const float al0 = m0 == -INFINITY ? 0.f : expf(m0 - n0);
            const float al1 = m1 == -INFINITY ? 0.f : expf(m1 - n1);
            m0 = n0;
            m1 = n1;
            float p[4];
            p[0] = v0 ? expf(sc[0] - n0) : 0.f;
            p[1] = v0 ? expf(sc[1] - n1) : 0.f;
            p[2] = v1 ? expf(sc[2] - n0) : 0.f;
            p[3] = v1 ? expf(sc[3] - n1) : 0.f;
            l0 = l0 * al0 + (p[0] + p[2]);
            l1 = l1 * al1 + (p[1] + p[3]);
            // P[head][position] for the P.V warps (masked positions are 0)
            float* Pb = Pbuf + b * (8 * kScStride);
            if (m0w < cnt) {
                Pb[(2 * tig) * kScStride + m0w + gid] = p[0];
                Pb[(2 * tig + 1) * kScStride + m0w + gid] = p[1];
                Pb[(2 * tig) * kScStride + m0w + gid + 8] = p[2];
                Pb[(2 * tig + 1) * kScStride + m0w + gid + 8] = p[3];
            }
            if (warp == 0 && gid == 0) {
                s_alpha[b * 8 + 2 * tig] = al0;
                s_alpha[b * 8 + 2 * tig + 1] = al1;
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&pfull[b]);
            if (++s == kStages) {
                s = 0;
                ph ^= 1u;
            }
        }
        // sums over the 16 positions of each warp, then over the warps
#pragma unroll
        for (int o = 4; o < 32; o <<= 1) {
            l0 += __shfl_xor_sync(0xffffffffu, l0, o);
            l1 += __shfl_xor_sync(0xffffffffu, l1, o);
        }
        if (gid == 0) {
            wsum[warp * 8 + 2 * tig] = l0;
            wsum[warp * 8 + 2 * tig + 1] = l1;
        }
        named_bar_sync(2, kSWarps * 32);
        if (warp == 0 && gid == 0) {
            float L0 = 0.f, L1 = 0.f;
            for (int w = 0; w < kSWarps; ++w) {
                L0 += wsum[w * 8 + 2 * tig];
                L1 += wsum[w * 8 + 2 * tig + 1];
            }
            if (2 * tig < G) {
                part[(2 * tig) * kPartFloats] = m0;
                part[(2 * tig) * kPartFloats + 1] = L0;
            }
            if (2 * tig + 1 < G) {
                part[(2 * tig + 1) * kPartFloats] = m1;
                part[(2 * tig + 1) * kPartFloats + 1] = L1;
            }
        }
    } else {
        // ------------------------------------------------------ P.V warps
        // O^T[dim][head] += V^T[dim][t] P^T[t][head] for dims 16 pw .. +15; the high and
        // low fp16 parts of P accumulate in separate chains
        const int pw = warp - kSWarps;
        const int j = lane >> 3;
        float acc[2][4] = {};
        int s = 0;
        uint32_t ph = 0;
        for (int i = 0; i < nsub; ++i) {
            const int cnt = min(kSub, np - i * kSub);
            const int b = i & 1;
            const bool ok_full = mbar_wait(&full[s], ph, kPolls);
            const bool ok_p = mbar_wait(&pfull[b], (uint32_t)(i >> 1) & 1u, kPolls);
            if (!ok_full || !ok_p) record_device_error(DEVERR_FULL_WAIT);
            uint8_t* Vs = ring + s * kStageBytes + 2 * kBoxBytes + (pw >> 2) * kBoxBytes;
            const int r_end = (cnt + 15) & ~15;
            if (cnt < r_end) {
                // rows cnt .. r_end - 1 were not part of the context: zero this warp's 16 dims of
                // them (two 16-byte chunks per row) so 0 * garbage cannot reach the sums
                for (int idx = lane; idx < 2 * (r_end - cnt); idx += 32) {
                    const int rr = cnt + (idx >> 1);
                    *reinterpret_cast<uint4*>(Vs + swz(rr, 2 * pw + (idx & 1))) = make_uint4(0u, 0u, 0u, 0u);
                }
                asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
                __syncwarp();
            }
            const float* Pb = Pbuf + b * (8 * kScStride);
            const float a0 = s_alpha[b * 8 + 2 * tig], a1 = s_alpha[b * 8 + 2 * tig + 1];
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                acc[h][0] *= a0;
                acc[h][1] *= a1;
                acc[h][2] *= a0;
                acc[h][3] *= a1;
            }
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
                const int k0 = 16 * kk;
                if (k0 < cnt) {
                    // matrix j: positions +8 if j >= 2, dims +8 if j odd
                    uint32_t av[4];
                    ldsm_x4_trans(av, Vs + swz(k0 + ((j >> 1) << 3) + (lane & 7), 2 * pw + (j & 1)));
                    const float2 p0 = *reinterpret_cast<const float2*>(Pb + gid * kScStride + k0 + 2 * tig);
                    const float2 p1 = *reinterpret_cast<const float2*>(Pb + gid * kScStride + k0 + 8 + 2 * tig);
                    uint32_t bh[2], bl[2];
                    split_f16x2(p0.x, p0.y, bh[0], bl[0]);
                    split_f16x2(p1.x, p1.y, bh[1], bl[1]);
                    mma_f16(acc[0], av, bh);
                    mma_f16(acc[1], av, bl);
                }
            }
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(&pempty[b]);
                mbar_arrive(&empty[s]);
            }
            if (++s == kStages) {
                s = 0;
                ph ^= 1u;
            }
        }
        // acc[.][0]: dim 16 pw + gid, head 2 tig; [1] head 2 tig + 1; [2], [3] the same for dim + 8
        const int d0 = 16 * pw + gid;
        if (2 * tig < G) {
            part[(2 * tig) * kPartFloats + 4 + d0] = acc[0][0] + acc[1][0];
            part[(2 * tig) * kPartFloats + 4 + d0 + 8] = acc[0][2] + acc[1][2];
        }
        if (2 * tig + 1 < G) {
            part[(2 * tig + 1) * kPartFloats + 4 + d0] = acc[0][1] + acc[1][1];
            part[(2 * tig + 1) * kPartFloats + 4 + d0 + 8] = acc[0][3] + acc[1][3];
        }
    }

}

// Merge of the splits, one CTA per query head and one thread per dim: with
// M = max_s m_s over splits that saw a position, w_s = e^(m_s - M) and
// L = sum_s l_s w_s, out[d] = (sum_s w_s acc_s[d]) / L.  Each thread reads every
// split's (m, l) (the same addresses across the CTA) and its dim of every split's
// accumulator, 32 splits per round of loads, and merges the rounds online (the
// running sums rescaled when the maximum grows), so one round trip to L2 serves up
// to 32 splits and no barrier is needed.
template <int G>
__global__ void __launch_bounds__(HD) attn_merge_kernel(const float* part, float* out, int n_split, int use_pdl)
{
    constexpr int B = 32;   // splits whose records are loaded together
    if (use_pdl) {
        pdl_launch_dependents();
        pdl_wait();
    }
    const int qh = blockIdx.x, g = qh / G, h = qh % G, d = threadIdx.x;
    const size_t rec = (size_t)G * kPartFloats;   // floats from one split's record of this head to the next
    const float* base = part + ((size_t)g * n_split * G + h) * kPartFloats;
    float M = -INFINITY, L = 0.f, o = 0.f;
    for (int s0 = 0; s0 < n_split; s0 += B) {
        float2 ml[B];
        float v[B];
#pragma unroll
        for (int k = 0; k < B; ++k) {
            const bool ok = s0 + k < n_split;
            ml[k] = ok ? __ldcg(reinterpret_cast<const float2*>(base + (s0 + k) * rec)) : make_float2(0.f, 0.f);
            v[k] = ok ? __ldcg(base + (s0 + k) * rec + 4 + d) : 0.f;
        }
        float Mb = M;
#pragma unroll
        for (int k = 0; k < B; ++k)
            if (ml[k].y > 0.f) Mb = fmaxf(Mb, ml[k].x);
        if (Mb == -INFINITY) continue;   // no split of this round saw a position
        const float r = M == -INFINITY ? 0.f : expf(M - Mb);
        L *= r;
        o *= r;
#pragma unroll
        for (int k = 0; k < B; ++k) {
            const float w = ml[k].y > 0.f ? expf(ml[k].x - Mb) : 0.f;
            L = fmaf(ml[k].y, w, L);
            o = fmaf(w, v[k], o);
        }
        M = Mb;
    }
    out[(size_t)qh * HD + d] = o / L;
}

template <int G>
ntx_status launch_g(const KArgs& k, int n_q_heads, cudaStream_t s, bool pdl)
{
    const ntx_status st = ensure_smem_limit((const void*)attn_kernel<G>, kSmem);
    if (st != NTX_OK) return st;
    const int grid = (n_q_heads / G) * k.n_split;
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
    // the merge always waits for the split kernel through the programmatic dependency
    cudaLaunchConfig_t mc = {};
    mc.gridDim = dim3(n_q_heads);
    mc.blockDim = dim3(HD);
    mc.stream = s;
    mc.attrs = attr;
    mc.numAttrs = 1;
    e = cudaLaunchKernelEx(&mc, attn_merge_kernel<G>, (const float*)k.part, k.out, k.n_split, 1);
    if (e != cudaSuccess) return fail(NTX_ECUDA, std::string("attention merge launch: ") + cudaGetErrorString(e));
    return NTX_OK;
}

// cuTensorMapEncodeTiled from the driver, looked up once through the runtime.
PFN_cuTensorMapEncodeTiled_v12000 tmap_encoder()
{
    static std::once_flag once;
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q = cudaDriverEntryPointSymbolNotFound;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    });
    return fn;
}

// A KV cache [n_kv][max_ctx][128] fp16 as a 3-D tensor map read in 64 x 64 boxes
// with the 128-byte swizzle; boxes past max_ctx are zero-filled.
ntx_status encode_kv_map(CUtensorMap* m, const __half* cache, int n_kv, int max_ctx)
{
    const PFN_cuTensorMapEncodeTiled_v12000 enc = tmap_encoder();
    if (!enc) return fail(NTX_ECUDA, "attention: cuTensorMapEncodeTiled is not available from the driver");
    const cuuint64_t dims[3] = {(cuuint64_t)HD, (cuuint64_t)max_ctx, (cuuint64_t)n_kv};
    const cuuint64_t strides[2] = {(cuuint64_t)HD * 2, (cuuint64_t)max_ctx * HD * 2};
    const cuuint32_t box[3] = {64, (cuuint32_t)kSub, 1};
    const cuuint32_t estr[3] = {1, 1, 1};
    const CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 3, const_cast<__half*>(cache), dims, strides, box, estr,
                           CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                           CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(NTX_ECUDA, "attention: KV tensor map encoding failed (" + std::to_string(r) + ")");
    return NTX_OK;
}

}  // namespace

cudaError_t take_device_error_attn(uint32_t* out) { return take_tu_device_error(out); }

int attn_split_for(int n_q_heads, int n_kv_heads, int32_t max_ctx)
{
    (void)max_ctx;
    (void)n_q_heads;
    // one CTA per SM
    return std::min(kMaxSplit, std::max(1, num_sms() / n_kv_heads));
}

size_t attn_workspace_bytes_for(int n_q_heads, int n_kv_heads, int head_dim, int n_split)
{
    (void)head_dim;
    const int G = n_q_heads / n_kv_heads;
    return (size_t)n_kv_heads * n_split * G * kPartFloats * sizeof(float);
}

ntx_status attn_launch(const AttnArgs& a, cudaStream_t s)
{
    const int G = a.n_q_heads / a.n_kv_heads;
    if (a.n_split < 1 || a.n_split > kMaxSplit || G * a.n_split * 4 > 2 * 8 * kScStride * 4)
        return fail(NTX_EUNSUPPORTED, "attention: split count out of range");
    KArgs k{};
    ntx_status st = encode_kv_map(&k.tk, a.k_cache, a.n_kv_heads, a.max_ctx);
    if (st != NTX_OK) return st;
    if ((st = encode_kv_map(&k.tv, a.v_cache, a.n_kv_heads, a.max_ctx)) != NTX_OK) return st;
    k.q = a.q;
    k.out = a.out;
    k.part = reinterpret_cast<float*>(a.workspace);
    k.max_ctx = a.max_ctx;
    k.n_split = a.n_split;
    k.n_ctx = a.n_ctx;
    k.pos_dev = a.pos_dev;
    k.use_pdl = a.pdl ? 1 : 0;
    k.pf = a.pf;
    switch (G) {
    case 1: return launch_g<1>(k, a.n_q_heads, s, a.pdl);
    case 2: return launch_g<2>(k, a.n_q_heads, s, a.pdl);
    case 4: return launch_g<4>(k, a.n_q_heads, s, a.pdl);
    case 8: return launch_g<8>(k, a.n_q_heads, s, a.pdl);
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
