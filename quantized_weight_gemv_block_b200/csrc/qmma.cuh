// qmma.cuh - block-quantized GEMV for the tiled layouts (batch 1).
//
// The GEMV kernel of the ntransformer news summary ("Arquitectura y estructura
// del código": cuda/ holds the GEMV kernels) for B200.  Batch-1 GEMV streams every
// weight once, so the work per weight must stay far below the SM's issue rate to
// keep HBM busy.  Dequantizing each weight to fp32 and multiplying costs several
// instructions per weight; here the packed codes are multiplied as integers:
//  * the input vector x is turned once per CTA into 24-bit fixed point with one
//    exponent per 32-column step u: x_int = rint(x 2^(S + e_u)) with |x_int| < 2^22,
//    written as three balanced signed 8-bit limbs, x_int = l0 + 2^8 l1 + 2^16 l2.
//    S comes from max |x| over the CTA's columns; e_u >= 0 adds the bits a step whose
//    values are all small can carry (from the step's own max |x|), so every step keeps
//    23 bits relative to its own largest value and an outlier channel only costs
//    precision to the 31 columns that share its step;
//  * the codes (int8 for Q8_0, unsigned 4- or 6-bit codes for the others, unpacked
//    to bytes with a few logic ops per word) are dotted with each limb, four bytes
//    at a time, by dp4a on the CUDA cores (CORE 1, the default): every partial sum is
//    an exact integer;
//  * the format's per-block scale (fp16 d, int8 or 6-bit sub-block scales, the
//    Q4_K mins, the code offsets 8 and 32) is applied to those integers, in
//    integer arithmetic where it is exact, and in fp32 once per step together with
//    the step's 2^-e_u (exact: a power of two);
//  * the limbs are recombined (weights 1, 2^8, 2^16) and the row total is scaled
//    by 2^-S, exactly.
// The products are exact; x carries 23 bits relative to the largest value of its
// 32-column step where fp32 carries 24 per value; sums round at fp32 once per step.
// CORE 0 does the same integer dots with one m16n8k32 integer MMA per 16 x 32 block
// (codes as A, the limbs as the 8 columns of B); it is kept as a measured
// alternative (NTX_GEMV_CORE=tc): on B200 the dp4a path streams as fast or faster on
// every decode shape, so no tensor core is needed for batch 1.
//
// Structure (one CTA per SM, 8 consumer warps and a producer warp):
//  * the grid is made of clusters of 1 or 2 CTAs; a cluster owns a contiguous
//    range of 16-row groups.  For matrices with few groups per SM the two CTAs of
//    a pair split the columns in halves (so the groups spread over 74 pairs
//    instead of 148 CTAs, which evens out the last round, and each CTA stages
//    only its half of x); both CTAs add each group's partial
//    row sums into a zeroed buffer in the first CTA's shared memory (the second
//    through distributed shared memory), and after a cluster barrier the first
//    CTA runs the epilogue of all its rows (with two addends the sum does not
//    depend on their order);
//  * a stage is one group x one chunk of KC columns of the CTA's half, contiguous
//    in the tiled layout, streamed by the producer warp with one 1-D bulk copy
//    (cp.async.bulk, L2 evict-first) into a ring of shared-memory stages guarded
//    by mbarriers;
//  * each consumer warp takes every 8th unit (32 or 256 columns) of a stage; the
//    shared-memory reads of a warp are contiguous or spread over distinct banks
//    (lane units for Q8_0, row-pair units for the others, below);
//  * row totals are reduced over the threads of a warp that share rows and over the
//    8 warps through shared memory in a fixed order (a barrier of the consumer
//    warps per group: measured faster on B200 than handing the sums to a separate
//    reducer warp through mbarriers) into the pair's sums; after the cluster
//    barrier the fused epilogue runs (store, residual add, SwiGLU of a gate / up
//    group pair, RoPE + fp16 KV-cache append).
#pragma once

#include "blocks.cuh"

namespace ntx {
namespace qmma {

using gemv::Params;

constexpr int kWarps = 8;                  // consumer warps
constexpr int kCons = kWarps * 32;
constexpr int kProducer = kWarps;          // warp index of the producer
constexpr int kThreads = kCons + 32;
constexpr int kMaxStages = 8;
constexpr int kOffXBar = 128;              // mbarrier of the bulk copy of x
constexpr int kOffRed = 256;               // [2][kWarps][2 mats][16] floats
constexpr int kOffRope = kOffRed + 2 * kWarps * 32 * 4;   // [64][cos, sin]
constexpr int kHeader = kOffRope + 512 + 256;
constexpr int kSmemLimit = 227 * 1024;
constexpr uint32_t kWaitPolls = 1u << 22;
// Extra bits a step may take beyond the CTA's exponent S: a step whose largest value is
// 2^40 below the CTA's largest keeps 23 bits; smaller steps keep 23 - (their shortfall).
constexpr int kMaxStepShift = 40;

// ------------------------------------------------------------------ MMA helpers

// C = A B for A 16 x 32 int8 (row), B 32 x 8 int8 (col), int32 accumulation from 0.
__device__ __forceinline__ void mma_s8(int (&c)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1)
{
    asm volatile(
        "mma.sync.aligned.m16n8k32.row.col.s32.s8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%10,%10,%10,%10};"
        : "=r"(c[0]), "=r"(c[1]), "=r"(c[2]), "=r"(c[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1), "r"(0));
}

// The same with A unsigned 8-bit.
__device__ __forceinline__ void mma_u8(int (&c)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1)
{
    asm volatile(
        "mma.sync.aligned.m16n8k32.row.col.s32.u8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%10,%10,%10,%10};"
        : "=r"(c[0]), "=r"(c[1]), "=r"(c[2]), "=r"(c[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1), "r"(0));
}

// Byte k of w, sign-extended (prmt with the sign-replicate selector).
template <int k>
__device__ __forceinline__ int sbyte(uint32_t w)
{
    constexpr uint32_t sel = k | ((8 | k) << 4) | ((8 | k) << 8) | ((8 | k) << 12);
    uint32_t r;
    asm("prmt.b32 %0, %1, 0, %2;" : "=r"(r) : "r"(w), "n"(sel));
    return (int)r;
}

// Byte k of w, zero-extended.
template <int k>
__device__ __forceinline__ int ubyte(uint32_t w)
{
    return (int)__byte_perm(w, 0u, 0x4440u | k);
}

// ------------------------------------------------------------------ cluster helpers

__device__ __forceinline__ uint32_t cluster_rank()
{
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}

__device__ __forceinline__ uint32_t cluster_size()
{
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_nctarank;" : "=r"(r));
    return r;
}

__device__ __forceinline__ void cluster_arrive()
{
    asm volatile("barrier.cluster.arrive.release;" ::: "memory");
}

__device__ __forceinline__ void cluster_wait()
{
    asm volatile("barrier.cluster.wait.acquire;" ::: "memory");
}

// Arrive on named barrier `id` without waiting (the waiting side uses named_bar_sync).
__device__ __forceinline__ void named_bar_arrive(int id, int threads)
{
    asm volatile("bar.arrive %0, %1;" ::"r"(id), "r"(threads) : "memory");
}

// Barrier of all threads of the cluster (of the CTA alone when the cluster is one CTA).
__device__ __forceinline__ void cluster_sync(uint32_t csize)
{
    if (csize == 1)
        __syncthreads();
    else
        asm volatile("barrier.cluster.arrive.release;\n\tbarrier.cluster.wait.acquire;" ::: "memory");
}



// Address of `p` (this CTA's shared memory) in the shared memory of cluster CTA `rank`.
__device__ __forceinline__ uint32_t peer_addr(const void* p, uint32_t rank)
{
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(smem_addr(p)), "r"(rank));
    return r;
}

// Atomic add of v to the fp32 at shared::cluster address addr.
__device__ __forceinline__ void red_add_cluster(uint32_t addr, float v)
{
    asm volatile("red.relaxed.cluster.shared::cluster.add.f32 [%0], %1;" ::"r"(addr), "f"(v) : "memory");
}

// ------------------------------------------------------------------ x staging
// Step u (columns 32u .. 32u + 31) of x occupies 32 words at xq + 32u:
//  words 8l + w (l = 0..2, w = 0..7): limb l of columns 32u + 4w .. + 3, one byte each
//    (PAIRED, the CUDA-core lane units: word 8 (w mod 4) + 2l + w / 4 instead, and the
//    step's factor 2^-e_u as a float at word 8 tig + 6 for tig = 0..3, so the seven words
//    lane tig needs, limbs 0..2 of columns 4 tig.. and 16 + 4 tig.. and the factor, are
//    contiguous: two 16-byte loads);
//  words 24..31: per-column sums of the limbs over what one C column covers
//    (Q6_K: words 24 + 4h + l = sum of limb l over the 16 columns of half h, words
//    27 and 31 zero; other formats: word 24 + l = sum of limb l over the 32 columns,
//    words 27..31 zero).  Lane tig reads its two C columns' sums at 24 + 2 tig.
// For the CUDA-core row-pair units every word index i of step u is stored at
// i XOR 8 (u mod 4) (sx below): the four quarter-warps of a warp read the same words of
// four consecutive steps, and a warp converting x writes four consecutive steps, which
// then fall in four different bank groups.  The Q8_0 lane units read no sums (words
// 24..31 hold no data there); only the tensor-core units read the zero words.
// A separate array of floats holds, per step u, 2^-e_u: the factor that brings the
// step's integer dots back to the CTA's common scale 2^S (fs below).

// The limb words and column sums of the 4 columns a lane holds (lane w of the 8 lanes
// of a step); the sums are already reduced over the step's lanes (or each half's).
struct XLimbs {
    uint32_t w0, w1, w2;
    int s0, s1, s2;
};

template <bool HALVES, bool SUMS>
__device__ __forceinline__ XLimbs x_limbs(float4 v, float two_s)
{
    // z = x_int + 0x8080: bytes 0 and 1 of z are the low limbs + 128, z >> 16 the top limb
    const float mag = 12582912.0f;   // 1.5 * 2^23: fmaf rounds x 2^S to an integer in its low bits
    const int bias = 0x8080 - 0x4B400000;
    const int z0 = __float_as_int(fmaf(v.x, two_s, mag)) + bias;
    const int z1 = __float_as_int(fmaf(v.y, two_s, mag)) + bias;
    const int z2 = __float_as_int(fmaf(v.z, two_s, mag)) + bias;
    const int z3 = __float_as_int(fmaf(v.w, two_s, mag)) + bias;
    const uint32_t lo01 = __byte_perm(z0, z1, 0x5410), lo23 = __byte_perm(z2, z3, 0x5410);
    XLimbs r;
    r.w0 = __byte_perm(lo01, lo23, 0x6420) ^ 0x80808080u;
    r.w1 = __byte_perm(lo01, lo23, 0x7531) ^ 0x80808080u;
    r.w2 = __byte_perm(__byte_perm(z0, z1, 0x0062), __byte_perm(z2, z3, 0x0062), 0x5410);
    r.s0 = r.s1 = r.s2 = 0;
    if (SUMS) {
        // column sums of the four values (byte sums of the signed limbs)
        r.s0 = __dp4a((int)r.w0, 0x01010101, 0);
        r.s1 = __dp4a((int)r.w1, 0x01010101, 0);
        r.s2 = __dp4a((int)r.w2, 0x01010101, 0);
#pragma unroll
        for (int o = 1; o < (HALVES ? 4 : 8); o <<= 1) {
            r.s0 += __shfl_xor_sync(0xffffffffu, r.s0, o);
            r.s1 += __shfl_xor_sync(0xffffffffu, r.s1, o);
            r.s2 += __shfl_xor_sync(0xffffffffu, r.s2, o);
        }
    }
    return r;
}

// Store lane w's limb words of step xs and, from the lanes that hold them, the sums
// (SUMS) and the zero words (ZEROS: words 27..31, or 27 and 31 with HALVES, which the
// tensor-core units read; the CUDA-core units leave them unread).
template <bool HALVES, bool PAIRED, bool SUMS, bool ZEROS>
__device__ __forceinline__ void x_store(uint32_t* xs, int w, const XLimbs& r, int sx, float f)
{
    if (PAIRED) {
        const int b = 8 * (w & 3) + (w >> 2);
        xs[b] = r.w0;
        xs[b + 2] = r.w1;
        xs[b + 4] = r.w2;
        if (w < 4) xs[8 * w + 6] = __float_as_uint(f);
    } else {
        xs[w ^ sx] = r.w0;
        xs[(8 + w) ^ sx] = r.w1;
        xs[(16 + w) ^ sx] = r.w2;
    }
    if (!SUMS) return;
    if (HALVES) {
        if ((w & 3) == 0) {
            const int h = w >> 2;
            xs[(24 + 4 * h) ^ sx] = (uint32_t)r.s0;
            xs[(25 + 4 * h) ^ sx] = (uint32_t)r.s1;
            xs[(26 + 4 * h) ^ sx] = (uint32_t)r.s2;
            if (ZEROS) xs[(27 + 4 * h) ^ sx] = 0u;
        }
    } else {
        if (w == 0) {
            xs[24 ^ sx] = (uint32_t)r.s0;
            xs[25 ^ sx] = (uint32_t)r.s1;
            xs[26 ^ sx] = (uint32_t)r.s2;
        } else if (ZEROS && w == 1) {
            xs[27 ^ sx] = 0u;
            xs[28 ^ sx] = 0u;
            xs[29 ^ sx] = 0u;
            xs[30 ^ sx] = 0u;
            xs[31 ^ sx] = 0u;
        }
    }
}

// ------------------------------------------------------------------ lane constants

struct Lane {
    int lane, gid, tig;
    int boff;        // word of this lane's B value in a step
    bool bval;       // lane's B column is a limb column (not a zero column)
    bool b_hi;       // Q6_K: the column belongs to the second 16-column half (B word b1)
};

template <int QT>
__device__ __forceinline__ Lane make_lane(int lane)
{
    Lane L;
    L.lane = lane;
    L.gid = lane >> 2;
    L.tig = lane & 3;
    if constexpr (QT == NTX_Q6_K_T) {
        // column n = gid: half g = n / 4, limb l = n % 4 (limb 3 is a zero column)
        const int g = L.gid >> 2, l = L.gid & 3;
        L.boff = 8 * l + 4 * g + L.tig;
        L.bval = l < 3;
        L.b_hi = g == 1;
    } else {
        // column n = gid: limb n for n < 3, zero columns after
        L.boff = 8 * L.gid + L.tig;
        L.bval = L.gid < 3;
        L.b_hi = false;
    }
    return L;
}

// B operand of one step: b0 covers columns 0-15 of the step, b1 columns 16-31.
template <int QT>
__device__ __forceinline__ void b_frag(const uint32_t* xs, const Lane& L, uint32_t& b0, uint32_t& b1)
{
    if constexpr (QT == NTX_Q6_K_T) {
        const uint32_t w = L.bval ? xs[L.boff] : 0u;
        b0 = L.b_hi ? 0u : w;
        b1 = L.b_hi ? w : 0u;
    } else {
        b0 = L.bval ? xs[L.boff] : 0u;
        b1 = L.bval ? xs[L.boff + 4] : 0u;
    }
}

__device__ __forceinline__ float2 d_pair(const uint8_t* p)
{
    return __half22float2(*reinterpret_cast<const __half2*>(p));
}

// Q4_K / Q5_K: the 32 six-bit scales / mins of rows gid and gid + 8 of a unit, one word
// per step m: byte 0 scale row gid, 1 scale row gid + 8, 2 min row gid, 3 min row gid + 8
// (SOFF: byte offset of the unit's scale section).
template <int SOFF = 2048>
__device__ __forceinline__ void q4k_scale_words(const uint8_t* U, int gid, uint32_t (&S)[8])
{
    const uint8_t* v = U + SOFF + 24 * gid;    // 8-byte aligned
    const uint2 na = *reinterpret_cast<const uint2*>(v);
    const uint2 nb = *reinterpret_cast<const uint2*>(v + 8);
    const uint2 hw = *reinterpret_cast<const uint2*>(v + 16);
    const uint32_t n4[4] = {na.x, na.y, nb.x, nb.y};
#pragma unroll
    for (int m = 0; m < 8; ++m) {
        const uint32_t lo = (m & 1 ? (n4[m >> 1] >> 4) : n4[m >> 1]) & 0x0F0F0F0Fu;
        const uint32_t h = m < 4 ? hw.x : hw.y;
        const int sh = 2 * (m & 3);
        const uint32_t hi = (sh <= 4 ? (h << (4 - sh)) : (h >> (sh - 4))) & 0x30303030u;
        S[m] = lo | hi;
    }
}

// ------------------------------------------------------------------ units
// acc0 / acc1: this lane's running fp32 sums for rows gid / gid + 8, in units of
// its C columns' limb (the quad reduction applies the limb weights).

template <int QT>
struct Unit;

template <>
struct Unit<NTX_Q8_0_T> {
    static __device__ __forceinline__ void run(const uint8_t* U, const uint32_t* xs, const float* fs, const Lane& L,
                                               float& acc0, float& acc1)
    {
        const uint4 a4 = *reinterpret_cast<const uint4*>(U + 16 * L.lane);
        const uint32_t a[4] = {a4.x, a4.y, a4.z, a4.w};
        uint32_t b0, b1;
        b_frag<NTX_Q8_0_T>(xs, L, b0, b1);
        int c[4];
        mma_s8(c, a, b0, b1);
        const float2 d = d_pair(U + 512 + 4 * L.gid);
        const float f = fs[0];
        acc0 = fmaf((float)(c[0] + 256 * c[1]), d.x * f, acc0);
        acc1 = fmaf((float)(c[2] + 256 * c[3]), d.y * f, acc1);
    }
};

template <>
struct Unit<NTX_Q4_0_T> {
    static __device__ __forceinline__ void run(const uint8_t* U, const uint32_t* xs, const float* fs, const Lane& L,
                                               float& acc0, float& acc1)
    {
        const uint2 pq = *reinterpret_cast<const uint2*>(U + 8 * L.lane);
        const uint32_t M = 0x0F0F0F0Fu;
        const uint32_t a[4] = {pq.x & M, pq.y & M, (pq.x >> 4) & M, (pq.y >> 4) & M};
        uint32_t b0, b1;
        b_frag<NTX_Q4_0_T>(xs, L, b0, b1);
        int c[4];
        mma_u8(c, a, b0, b1);
        // codes carry +8: subtract 8 x (this lane's two columns' limb sums)
        const int2 X = *reinterpret_cast<const int2*>(xs + 24 + 2 * L.tig);
        const int off = -8 * (X.x + 256 * X.y);
        const float2 d = d_pair(U + 256 + 4 * L.gid);
        const float f = fs[0];
        acc0 = fmaf((float)(c[0] + 256 * c[1] + off), d.x * f, acc0);
        acc1 = fmaf((float)(c[2] + 256 * c[3] + off), d.y * f, acc1);
    }
};

template <>
struct Unit<NTX_Q6_K_T> {
    static __device__ __forceinline__ void run(const uint8_t* U, const uint32_t* xs, const float* fs, const Lane& L,
                                               float& acc0, float& acc1)
    {
        // this lane's scales: sub-blocks 2m + (tig / 2) of rows gid (bytes 0-7) and gid + 8 (8-15)
        const uint4 sv = *reinterpret_cast<const uint4*>(U + 3072 + 16 * (2 * L.gid + (L.tig >> 1)));
        const float2 d = d_pair(U + 3328 + 4 * L.gid);
        const uint32_t M6 = 0x3F3F3F3Fu;
#pragma unroll
        for (int m = 0; m < 8; ++m) {
            const uint8_t* w = U + 384 * m + 12 * L.lane;
            const uint32_t A = *reinterpret_cast<const uint32_t*>(w);
            const uint32_t B = *reinterpret_cast<const uint32_t*>(w + 4);
            const uint32_t C = *reinterpret_cast<const uint32_t*>(w + 8);
            uint32_t a[4];
            a[0] = A & M6;
            a[1] = B & M6;
            a[2] = C & M6;
            a[3] = ((A >> 6) & 0x03030303u) | ((B >> 4) & 0x0C0C0C0Cu) | ((C >> 2) & 0x30303030u);
            const uint32_t* x = xs + 32 * m;
            uint32_t b0, b1;
            b_frag<NTX_Q6_K_T>(x, L, b0, b1);
            int c[4];
            mma_u8(c, a, b0, b1);
            const int2 X = *reinterpret_cast<const int2*>(x + 24 + 2 * L.tig);
            int s0, s1;
            if (m < 4) {
                s0 = m == 0 ? sbyte<0>(sv.x) : m == 1 ? sbyte<1>(sv.x) : m == 2 ? sbyte<2>(sv.x) : sbyte<3>(sv.x);
                s1 = m == 0 ? sbyte<0>(sv.z) : m == 1 ? sbyte<1>(sv.z) : m == 2 ? sbyte<2>(sv.z) : sbyte<3>(sv.z);
            } else {
                s0 = m == 4 ? sbyte<0>(sv.y) : m == 5 ? sbyte<1>(sv.y) : m == 6 ? sbyte<2>(sv.y) : sbyte<3>(sv.y);
                s1 = m == 4 ? sbyte<0>(sv.w) : m == 5 ? sbyte<1>(sv.w) : m == 6 ? sbyte<2>(sv.w) : sbyte<3>(sv.w);
            }
            // codes carry +32; the step's column totals are exact integers before the fp32 step
            const int p0 = s0 * (c[0] - 32 * X.x), p1 = s0 * (c[1] - 32 * X.y);
            const int q0 = s1 * (c[2] - 32 * X.x), q1 = s1 * (c[3] - 32 * X.y);
            const float f = fs[m];
            acc0 = fmaf(d.x * f, fmaf(256.f, (float)p1, (float)p0), acc0);
            acc1 = fmaf(d.y * f, fmaf(256.f, (float)q1, (float)q0), acc1);
        }
    }
};

template <>
struct Unit<NTX_Q4_K_T> {
    static __device__ __forceinline__ void run(const uint8_t* U, const uint32_t* xs, const float* fs, const Lane& L,
                                               float& acc0, float& acc1)
    {
        uint32_t S[8];
        q4k_scale_words(U, L.gid, S);
        const uint2 dd = *reinterpret_cast<const uint2*>(U + 2240 + 8 * L.gid);
        const float2 d = __half22float2(*reinterpret_cast<const __half2*>(&dd.x));
        const float2 dm = __half22float2(*reinterpret_cast<const __half2*>(&dd.y));
        const uint32_t M = 0x0F0F0F0Fu;
#pragma unroll
        for (int m = 0; m < 8; ++m) {
            const uint2 pq = *reinterpret_cast<const uint2*>(U + 256 * m + 8 * L.lane);
            const uint32_t a[4] = {pq.x & M, pq.y & M, (pq.x >> 4) & M, (pq.y >> 4) & M};
            const uint32_t* x = xs + 32 * m;
            uint32_t b0, b1;
            b_frag<NTX_Q4_K_T>(x, L, b0, b1);
            int c[4];
            mma_u8(c, a, b0, b1);
            const int2 X = *reinterpret_cast<const int2*>(x + 24 + 2 * L.tig);
            const int xp = X.x + 256 * X.y;
            const int sc0 = ubyte<0>(S[m]), sc1 = ubyte<1>(S[m]), mn0 = ubyte<2>(S[m]), mn1 = ubyte<3>(S[m]);
            const float f = fs[m];
            acc0 = fmaf(d.x * f, fmaf(256.f, (float)(sc0 * c[1]), (float)(sc0 * c[0])),
                        fmaf(-dm.x * f, (float)(mn0 * xp), acc0));
            acc1 = fmaf(d.y * f, fmaf(256.f, (float)(sc1 * c[3]), (float)(sc1 * c[2])),
                        fmaf(-dm.y * f, (float)(mn1 * xp), acc1));
        }
    }
};

// Q5_K: the fifth bits of the 4 codes of group gi (columns 4 t .. + 3 for gi = 2 t, 16 + 4 t
// .. + 3 for gi = 2 t + 1) of one row, from its fifth-bit word h, at bit 4 of each byte.
template <int gi>
__device__ __forceinline__ uint32_t q5_bits(uint32_t h)
{
    return (gi <= 4 ? (h << (4 - gi)) : (h >> (gi - 4))) & 0x10101010u;
}
__device__ __forceinline__ uint32_t q5_bits_r(uint32_t h, int gi) { return ((h >> gi) & 0x01010101u) << 4; }

template <>
struct Unit<NTX_Q5_K_T> {
    static __device__ __forceinline__ void run(const uint8_t* U, const uint32_t* xs, const float* fs, const Lane& L,
                                               float& acc0, float& acc1)
    {
        uint32_t S[8];
        q4k_scale_words<2560>(U, L.gid, S);
        const uint2 dd = *reinterpret_cast<const uint2*>(U + 2752 + 8 * L.gid);
        const float2 d = __half22float2(*reinterpret_cast<const __half2*>(&dd.x));
        const float2 dm = __half22float2(*reinterpret_cast<const __half2*>(&dd.y));
        const uint32_t M = 0x0F0F0F0Fu;
#pragma unroll
        for (int m = 0; m < 8; ++m) {
            const uint2 pq = *reinterpret_cast<const uint2*>(U + 320 * m + 8 * L.lane);
            const uint2 H = *reinterpret_cast<const uint2*>(U + 320 * m + 256 + 8 * L.gid);
            const uint32_t a[4] = {(pq.x & M) | q5_bits_r(H.x, 2 * L.tig), (pq.y & M) | q5_bits_r(H.y, 2 * L.tig),
                                   ((pq.x >> 4) & M) | q5_bits_r(H.x, 2 * L.tig + 1),
                                   ((pq.y >> 4) & M) | q5_bits_r(H.y, 2 * L.tig + 1)};
            const uint32_t* x = xs + 32 * m;
            uint32_t b0, b1;
            b_frag<NTX_Q5_K_T>(x, L, b0, b1);
            int c[4];
            mma_u8(c, a, b0, b1);
            const int2 X = *reinterpret_cast<const int2*>(x + 24 + 2 * L.tig);
            const int xp = X.x + 256 * X.y;
            const int sc0 = ubyte<0>(S[m]), sc1 = ubyte<1>(S[m]), mn0 = ubyte<2>(S[m]), mn1 = ubyte<3>(S[m]);
            const float f = fs[m];
            acc0 = fmaf(d.x * f, fmaf(256.f, (float)(sc0 * c[1]), (float)(sc0 * c[0])),
                        fmaf(-dm.x * f, (float)(mn0 * xp), acc0));
            acc1 = fmaf(d.y * f, fmaf(256.f, (float)(sc1 * c[3]), (float)(sc1 * c[2])),
                        fmaf(-dm.y * f, (float)(mn1 * xp), acc1));
        }
    }
};

// ------------------------------------------------------------------ CUDA-core units
// The same tiled bytes, reduced on the CUDA cores with dp4a (four 8-bit products and
// an int32 add per instruction).  Integer partial sums (exact) are weighted by the
// sub-block scales in int32 and recombined over the limbs (1, 2^8, 2^16) in fp32 once
// per block or superblock.
//
// Lane units (Q8_0): each lane takes the 16 bytes the MMA would give it as its A
// fragment (a warp's loads are contiguous and conflict-free): row gid at columns
// 4 tig .. + 3 and 16 + 4 tig .. + 3 and the same columns of row gid + 8, dotted with
// its 8 columns of each of the three limbs.  The lane's two limb words of a step sit
// side by side (the PAIRED x layout).  acc0 / acc1 end as this lane's share of rows
// gid / gid + 8 in units of x_int, summed over the quad afterwards.

// dot of one code word with one limb word, added to c
__device__ __forceinline__ int dp4(uint32_t a, uint32_t x, int c)
{
    return __dp4a((int)a, (int)x, c);
}

// the limbs' integer sums c0 + 2^8 c1 + 2^16 c2 in fp32
__device__ __forceinline__ float limbs_f(int c0, int c1, int c2)
{
    return fmaf((float)c2, 65536.f, fmaf((float)c1, 256.f, (float)c0));
}

// The same value with the two low limbs combined in int32 first (one conversion fewer):
// c0 + 256 c1 is exact there when |c0|, |c1| < 2^22, and its single rounding to fp32
// equals that of fmaf(c1, 256, c0) on the exact operands.  Used by the 4-bit row units
// (Q4_0 sweep +1 %); on the Q8_0 lane units it measured 0.5 % slower and is not used.
__device__ __forceinline__ float limbs_f2(int c0, int c1, int c2)
{
    return fmaf((float)c2, 65536.f, (float)(c0 + 256 * c1));
}

// limb words of a step for lane tig (the PAIRED layout): X[l].x = columns 4 tig..,
// X[l].y = 16 + 4 tig..; f = the step's factor 2^-e_u
__device__ __forceinline__ void x_words(const uint32_t* xs, int tig, uint2 (&X)[3], float& f)
{
    const uint4 a = *reinterpret_cast<const uint4*>(xs + 8 * tig);
    const uint4 b = *reinterpret_cast<const uint4*>(xs + 8 * tig + 4);
    X[0] = make_uint2(a.x, a.y);
    X[1] = make_uint2(a.z, a.w);
    X[2] = make_uint2(b.x, b.y);
    f = __uint_as_float(b.z);
}

template <int QT>
struct Dot;

template <>
struct Dot<NTX_Q8_0_T> {
    static __device__ __forceinline__ void run(const uint8_t* U, const uint32_t* xs, const float* fs, const Lane& L,
                                               float& acc0, float& acc1)
    {
        const uint4 a = *reinterpret_cast<const uint4*>(U + 16 * L.lane);
        uint2 X[3];
        float f;
        x_words(xs, L.tig, X, f);
        (void)fs;
        int c0[3], c1[3];
#pragma unroll
        for (int l = 0; l < 3; ++l) {
            c0[l] = dp4(a.z, X[l].y, dp4(a.x, X[l].x, 0));
            c1[l] = dp4(a.w, X[l].y, dp4(a.y, X[l].x, 0));
        }
        const float2 d = d_pair(U + 512 + 4 * L.gid);
        acc0 = fmaf(d.x * f, limbs_f(c0[0], c0[1], c0[2]), acc0);
        acc1 = fmaf(d.y * f, limbs_f(c1[0], c1[1], c1[2]), acc1);
    }
};

// Row-pair units (Q4_0, Q4_K, Q6_K): a thread takes the bytes of the four lanes of
// one gid in one step, i.e. rows gid and gid + 8 over all 32 columns of the step, so
// each sub-block's dp4a chain runs over its 16 or 32 columns before the one scale
// multiply, and the x words of the step are shared by the whole chain.  Threads
// 8j .. 8j + 7 of a warp take gids 0..7 of the same step (their x loads are one
// broadcast; their code loads start 32 or 48 bytes apart).  g = lane mod 8,
// j = lane / 8; acc0 / acc1 end as this thread's share of rows g / g + 8 in units of
// x_int, summed over j afterwards.

// Byte `sel & 3` of w, sign-extended; sel from sbyte_sel(k).
__device__ __forceinline__ uint32_t sbyte_sel(int k)
{
    return (uint32_t)k | ((uint32_t)(8 | k) * 0x1110u);
}
__device__ __forceinline__ int sbyte_r(uint32_t w, uint32_t sel)
{
    uint32_t r;
    asm("prmt.b32 %0, %1, 0, %2;" : "=r"(r) : "r"(w), "r"(sel));
    return (int)r;
}

// limb words of a step (word i at i XOR sx): X[l][h] = limb l of columns 16h .. 16h + 15
__device__ __forceinline__ void x_step(const uint32_t* xs, int sx, uint4 (&X)[3][2])
{
#pragma unroll
    for (int l = 0; l < 3; ++l)
#pragma unroll
        for (int h = 0; h < 2; ++h) X[l][h] = *reinterpret_cast<const uint4*>(xs + ((8 * l + 4 * h) ^ sx));
}

// component t of a uint4 (t a compile-time index after unrolling)
__device__ __forceinline__ uint32_t comp(const uint4& v, int t)
{
    return t == 0 ? v.x : t == 1 ? v.y : t == 2 ? v.z : v.w;
}

template <int QT>
struct Row;

template <>
struct Row<NTX_Q4_0_T> {
    // U: the unit (one step), xs: its x words, sx: the step's x swizzle, f: the step's factor
    static __device__ __forceinline__ void run(const uint8_t* U, const uint32_t* xs, int sx, float f, int g,
                                               float& acc0, float& acc1)
    {
        const uint4* L = reinterpret_cast<const uint4*>(U + 32 * g);   // (P, Q) of lanes tig 0..3
        const uint4 u0 = L[0], u1 = L[1];
        const uint32_t Pw[4] = {u0.x, u0.z, u1.x, u1.z}, Qw[4] = {u0.y, u0.w, u1.y, u1.w};
        uint4 X[3][2];
        x_step(xs, sx, X);
        const uint4 xsum = *reinterpret_cast<const uint4*>(xs + (24 ^ sx));
        const uint32_t M = 0x0F0F0F0Fu;
        int c0[3], c1[3];
#pragma unroll
        for (int l = 0; l < 3; ++l) {
            // codes carry +8: start at -8 x (the limb's sum over the step)
            c0[l] = c1[l] = -8 * (int)comp(xsum, l);
#pragma unroll
            for (int t = 0; t < 4; ++t) {
                c0[l] = dp4((Pw[t] >> 4) & M, comp(X[l][1], t), dp4(Pw[t] & M, comp(X[l][0], t), c0[l]));
                c1[l] = dp4((Qw[t] >> 4) & M, comp(X[l][1], t), dp4(Qw[t] & M, comp(X[l][0], t), c1[l]));
            }
        }
        const float2 d = d_pair(U + 256 + 4 * g);
        // |c| <= 8 * 32 * 128 + 32 * 15 * 128 per limb
        acc0 = fmaf(d.x * f, limbs_f2(c0[0], c0[1], c0[2]), acc0);
        acc1 = fmaf(d.y * f, limbs_f2(c1[0], c1[1], c1[2]), acc1);
    }
};

template <>
struct Row<NTX_Q6_K_T> {
    // U: the superblock unit, xs: its x words, fs: its steps' factors; the thread takes
    // steps j and j + 4
    static __device__ __forceinline__ void run(const uint8_t* U, const uint32_t* xs, const float* fs, int g, int j,
                                               float& acc0, float& acc1)
    {
        // int8 scales: vector (g, parity) holds row g at bytes 0-7 and row g + 8 at bytes
        // 8-15, byte m of each = sub-block 2m + parity (se: parity 0, so: parity 1)
        const uint4 se = *reinterpret_cast<const uint4*>(U + 3072 + 32 * g);
        const uint4 so = *reinterpret_cast<const uint4*>(U + 3072 + 32 * g + 16);
        const uint32_t sel = sbyte_sel(j);   // byte m mod 4 = j
        const uint32_t M6 = 0x3F3F3F3Fu;
        const float2 d = d_pair(U + 3328 + 4 * g);
#pragma unroll
        for (int k = 0; k < 2; ++k) {
            int p0[3] = {0, 0, 0}, p1[3] = {0, 0, 0};   // per limb: rows g, g + 8
            const int m = j + 4 * k;
            // lanes tig 0..3 of gid g: words A, B, C of each
            const uint4* L = reinterpret_cast<const uint4*>(U + 384 * m + 48 * g);
            const uint4 v0 = L[0], v1 = L[1], v2 = L[2];
            const uint32_t A[4] = {v0.x, v0.w, v1.z, v2.y}, B[4] = {v0.y, v1.x, v1.w, v2.z},
                           C[4] = {v0.z, v1.y, v2.x, v2.w};
            const uint32_t* x = xs + 32 * m;
            const int sx = 8 * j;   // step m mod 4 = j (a unit starts on a multiple of 8 steps)
            uint4 X[3][2];
            x_step(x, sx, X);
            const uint4 h0 = *reinterpret_cast<const uint4*>(x + (24 ^ sx));   // limb sums of half 0
            const uint4 h1 = *reinterpret_cast<const uint4*>(x + (28 ^ sx));   // and of half 1
            // sub-blocks 2m (e) and 2m + 1 (o) of rows g (0) and g + 8 (1)
            const int s_e0 = sbyte_r(k ? se.y : se.x, sel), s_e1 = sbyte_r(k ? se.w : se.z, sel);
            const int s_o0 = sbyte_r(k ? so.y : so.x, sel), s_o1 = sbyte_r(k ? so.w : so.z, sel);
            // 6-bit codes of rows g / g + 8, sub-blocks 2m / 2m + 1, per lane tig
            uint32_t a0[4], a1[4], a2[4], a3[4];
#pragma unroll
            for (int t = 0; t < 4; ++t) {
                a0[t] = A[t] & M6;
                a1[t] = B[t] & M6;
                a2[t] = C[t] & M6;
                a3[t] = ((A[t] >> 6) & 0x03030303u) | ((B[t] >> 4) & 0x0C0C0C0Cu) | ((C[t] >> 2) & 0x30303030u);
            }
#pragma unroll
            for (int l = 0; l < 3; ++l) {
                // codes carry +32: each chain starts at -32 x (the limb's sum over its half)
                int e0 = -32 * (int)comp(h0, l), e1 = e0, o0 = -32 * (int)comp(h1, l), o1 = o0;
#pragma unroll
                for (int t = 0; t < 4; ++t) {
                    e0 = dp4(a0[t], comp(X[l][0], t), e0);
                    e1 = dp4(a1[t], comp(X[l][0], t), e1);
                    o0 = dp4(a2[t], comp(X[l][1], t), o0);
                    o1 = dp4(a3[t], comp(X[l][1], t), o1);
                }
                p0[l] += s_e0 * e0 + s_o0 * o0;
                p1[l] += s_e1 * e1 + s_o1 * o1;
            }
            const float f = fs[m];
            acc0 = fmaf(d.x * f, limbs_f(p0[0], p0[1], p0[2]), acc0);
            acc1 = fmaf(d.y * f, limbs_f(p1[0], p1[1], p1[2]), acc1);
        }
    }
};

template <>
struct Row<NTX_Q4_K_T> {
    // U: the superblock unit, xs: its x words, fs: its steps' factors; the thread takes
    // steps (= sub-blocks) j and j + 4
    static __device__ __forceinline__ void run(const uint8_t* U, const uint32_t* xs, const float* fs, int g, int j,
                                               float& acc0, float& acc1)
    {
        const uint8_t* v = U + 2048 + 24 * g;   // packed 6-bit scales / mins of rows g, g + 8
        const uint32_t M = 0x0F0F0F0Fu;
        const uint2 dd = *reinterpret_cast<const uint2*>(U + 2240 + 8 * g);
        const float2 d = __half22float2(*reinterpret_cast<const __half2*>(&dd.x));
        const float2 dm = __half22float2(*reinterpret_cast<const __half2*>(&dd.y));
#pragma unroll
        for (int k = 0; k < 2; ++k) {
            int p0[3] = {0, 0, 0}, p1[3] = {0, 0, 0};   // per limb: rows g, g + 8
            int n0[3] = {0, 0, 0}, n1[3] = {0, 0, 0};   // mins x limb sums
            const int m = j + 4 * k;
            // sub-block m: byte 0 scale row g, 1 scale row g + 8, 2 min row g, 3 min row g + 8
            const uint32_t nw = *reinterpret_cast<const uint32_t*>(v + 4 * (m >> 1));
            const uint32_t hw = *reinterpret_cast<const uint32_t*>(v + 16 + 4 * k);
            const uint32_t S = ((nw >> (4 * (m & 1))) & 0x0F0F0F0Fu) | (((hw >> (2 * j)) & 0x03030303u) << 4);
            const uint4* L = reinterpret_cast<const uint4*>(U + 256 * m + 32 * g);
            const uint4 u0 = L[0], u1 = L[1];
            const uint32_t Pw[4] = {u0.x, u0.z, u1.x, u1.z}, Qw[4] = {u0.y, u0.w, u1.y, u1.w};
            const uint32_t* x = xs + 32 * m;
            const int sx = 8 * j;   // step m mod 4 = j (a unit starts on a multiple of 8 steps)
            uint4 X[3][2];
            x_step(x, sx, X);
            const uint4 xsum = *reinterpret_cast<const uint4*>(x + (24 ^ sx));
            const int sc0 = ubyte<0>(S), sc1 = ubyte<1>(S), mn0 = ubyte<2>(S), mn1 = ubyte<3>(S);
#pragma unroll
            for (int l = 0; l < 3; ++l) {
                int c0 = 0, c1 = 0;
#pragma unroll
                for (int t = 0; t < 4; ++t) {
                    c0 = dp4((Pw[t] >> 4) & M, comp(X[l][1], t), dp4(Pw[t] & M, comp(X[l][0], t), c0));
                    c1 = dp4((Qw[t] >> 4) & M, comp(X[l][1], t), dp4(Qw[t] & M, comp(X[l][0], t), c1));
                }
                p0[l] += sc0 * c0;
                p1[l] += sc1 * c1;
                n0[l] += mn0 * (int)comp(xsum, l);
                n1[l] += mn1 * (int)comp(xsum, l);
            }
            const float f = fs[m];
            // |p| <= 63 * 32 * 15 * 128 < 2^22, |n| <= 63 * 32 * 128 per limb
            acc0 = fmaf(d.x * f, limbs_f2(p0[0], p0[1], p0[2]), fmaf(-dm.x * f, limbs_f2(n0[0], n0[1], n0[2]), acc0));
            acc1 = fmaf(d.y * f, limbs_f2(p1[0], p1[1], p1[2]), fmaf(-dm.y * f, limbs_f2(n1[0], n1[1], n1[2]), acc1));
        }
    }
};

template <>
struct Row<NTX_Q5_K_T> {
    // As Row<NTX_Q4_K_T>, with each code's fifth bit ORed in from the step's fifth-bit words
    static __device__ __forceinline__ void run(const uint8_t* U, const uint32_t* xs, const float* fs, int g, int j,
                                               float& acc0, float& acc1)
    {
        const uint8_t* v = U + 2560 + 24 * g;   // packed 6-bit scales / mins of rows g, g + 8
        const uint32_t M = 0x0F0F0F0Fu;
        const uint2 dd = *reinterpret_cast<const uint2*>(U + 2752 + 8 * g);
        const float2 d = __half22float2(*reinterpret_cast<const __half2*>(&dd.x));
        const float2 dm = __half22float2(*reinterpret_cast<const __half2*>(&dd.y));
#pragma unroll
        for (int k = 0; k < 2; ++k) {
            int p0[3] = {0, 0, 0}, p1[3] = {0, 0, 0};   // per limb: rows g, g + 8
            int n0[3] = {0, 0, 0}, n1[3] = {0, 0, 0};   // mins x limb sums
            const int m = j + 4 * k;
            const uint32_t nw = *reinterpret_cast<const uint32_t*>(v + 4 * (m >> 1));
            const uint32_t hw = *reinterpret_cast<const uint32_t*>(v + 16 + 4 * k);
            const uint32_t S = ((nw >> (4 * (m & 1))) & 0x0F0F0F0Fu) | (((hw >> (2 * j)) & 0x03030303u) << 4);
            const uint4* L = reinterpret_cast<const uint4*>(U + 320 * m + 32 * g);
            const uint4 u0 = L[0], u1 = L[1];
            const uint2 H = *reinterpret_cast<const uint2*>(U + 320 * m + 256 + 8 * g);
            const uint32_t Pw[4] = {u0.x, u0.z, u1.x, u1.z}, Qw[4] = {u0.y, u0.w, u1.y, u1.w};
            // 5-bit codes of rows g (P) and g + 8 (Q): columns 4 t .. (lo) and 16 + 4 t .. (hi) of lane t
            uint32_t Plo[4], Phi[4], Qlo[4], Qhi[4];
            Plo[0] = (Pw[0] & M) | q5_bits<0>(H.x);
            Phi[0] = ((Pw[0] >> 4) & M) | q5_bits<1>(H.x);
            Plo[1] = (Pw[1] & M) | q5_bits<2>(H.x);
            Phi[1] = ((Pw[1] >> 4) & M) | q5_bits<3>(H.x);
            Plo[2] = (Pw[2] & M) | q5_bits<4>(H.x);
            Phi[2] = ((Pw[2] >> 4) & M) | q5_bits<5>(H.x);
            Plo[3] = (Pw[3] & M) | q5_bits<6>(H.x);
            Phi[3] = ((Pw[3] >> 4) & M) | q5_bits<7>(H.x);
            Qlo[0] = (Qw[0] & M) | q5_bits<0>(H.y);
            Qhi[0] = ((Qw[0] >> 4) & M) | q5_bits<1>(H.y);
            Qlo[1] = (Qw[1] & M) | q5_bits<2>(H.y);
            Qhi[1] = ((Qw[1] >> 4) & M) | q5_bits<3>(H.y);
            Qlo[2] = (Qw[2] & M) | q5_bits<4>(H.y);
            Qhi[2] = ((Qw[2] >> 4) & M) | q5_bits<5>(H.y);
            Qlo[3] = (Qw[3] & M) | q5_bits<6>(H.y);
            Qhi[3] = ((Qw[3] >> 4) & M) | q5_bits<7>(H.y);
            const uint32_t* x = xs + 32 * m;
            const int sx = 8 * j;   // step m mod 4 = j (a unit starts on a multiple of 8 steps)
            uint4 X[3][2];
            x_step(x, sx, X);
            const uint4 xsum = *reinterpret_cast<const uint4*>(x + (24 ^ sx));
            const int sc0 = ubyte<0>(S), sc1 = ubyte<1>(S), mn0 = ubyte<2>(S), mn1 = ubyte<3>(S);
#pragma unroll
            for (int l = 0; l < 3; ++l) {
                int c0 = 0, c1 = 0;
#pragma unroll
                for (int t = 0; t < 4; ++t) {
                    c0 = dp4(Phi[t], comp(X[l][1], t), dp4(Plo[t], comp(X[l][0], t), c0));
                    c1 = dp4(Qhi[t], comp(X[l][1], t), dp4(Qlo[t], comp(X[l][0], t), c1));
                }
                p0[l] += sc0 * c0;
                p1[l] += sc1 * c1;
                n0[l] += mn0 * (int)comp(xsum, l);
                n1[l] += mn1 * (int)comp(xsum, l);
            }
            const float f = fs[m];
            // |p| may reach 63 * 32 * 31 * 128 > 2^22: three conversions; |n| <= 63 * 32 * 128
            acc0 = fmaf(d.x * f, limbs_f(p0[0], p0[1], p0[2]), fmaf(-dm.x * f, limbs_f2(n0[0], n0[1], n0[2]), acc0));
            acc1 = fmaf(d.y * f, limbs_f(p1[0], p1[1], p1[2]), fmaf(-dm.y * f, limbs_f2(n1[0], n1[1], n1[2]), acc1));
        }
    }
};

// ------------------------------------------------------------------ epilogue

// Output row `row` (t = row total, t_up the up-projection total for SwiGLU).  Called
// by whole warps; `ok` is false for lanes past the last row.
template <int EPI>
__device__ __forceinline__ void epilogue(const Params& P, int row, bool ok, float t, float t_up, int32_t pos,
                                         const float* rope_cs)
{
    using namespace gemv;
    if (EPI == EPI_STORE) {
        if (ok) P.y[row] = t;
    } else if (EPI == EPI_ADD) {
        if (ok) P.y[row] = P.y[row] + t;
    } else if (EPI == EPI_SWIGLU) {
        if (ok) P.y[row] = t / (1.0f + expf(-t)) * t_up;
    } else if (EPI == EPI_QKV) {
        // rows: q [0, q_rows), k [q_rows, q_rows + kv_rows), v after; RoPE on (2i, 2i+1)
        const float other = __shfl_xor_sync(0xffffffffu, t, 1);
        if (!ok) return;
        float v = t;
        const int hd = P.head_dim;
        if (row < P.q_rows + P.kv_rows) {
            const int pi = (row % hd) / 2;
            const float cf = rope_cs[2 * pi], sf = rope_cs[2 * pi + 1];
            v = (row & 1) ? (other * sf + t * cf) : (t * cf - other * sf);
        }
        if (row < P.q_rows) {
            P.q_out[row] = v;
        } else {
            const int kvr = row - P.q_rows;
            const bool is_v = kvr >= P.kv_rows;
            const int j = is_v ? kvr - P.kv_rows : kvr;
            const int g = j / hd, dd = j % hd;
            __half* cache = is_v ? P.v_cache : P.k_cache;
            cache[((int64_t)g * P.max_ctx + pos) * hd + dd] = __float2half_rn(v);
        }
    }
}

// ------------------------------------------------------------------ kernel

// CORE 0: the per-step sums on the tensor cores (Unit); CORE 1: on the CUDA cores (Dot, Row).
template <int QT, int EPI, int PRO, int CORE>
__global__ void __launch_bounds__(kThreads, 1) qmma_kernel(const Params P)
{
    using T = gemv::Tiled<QT>;
    constexpr int NM = EPI == gemv::EPI_SWIGLU ? 2 : 1;    // matrices per group (gate, up)
    constexpr int SPU = T::UK / 32;                         // steps per unit
    // CUDA-core path: lane units (the MMA's fragments) for Q8_0, row-pair units otherwise
    constexpr bool ROWS = CORE == 1 && QT != NTX_Q8_0_T;
    // the x limb sums are read by every unit but the Q8_0 lane units (no code offset)
    constexpr bool XSUMS = !(CORE == 1 && QT == NTX_Q8_0_T);

    extern __shared__ __align__(128) uint8_t smem[];
    uint64_t* full = reinterpret_cast<uint64_t*>(smem);
    uint64_t* empty = full + kMaxStages;
    uint64_t* xbar = reinterpret_cast<uint64_t*>(smem + kOffXBar);
    float* red = reinterpret_cast<float*>(smem + kOffRed);
    float* rope_cs = reinterpret_cast<float*>(smem + kOffRope);
    uint32_t* xq = reinterpret_cast<uint32_t*>(smem + kHeader);
    float* xsf = reinterpret_cast<float*>(smem + kHeader + P.fs_off);   // per-step factors 2^-e_u
    uint8_t* stages = smem + kHeader + P.x_bytes;
    float* sums = reinterpret_cast<float*>(stages + (size_t)P.n_stages * P.stage_bytes);   // [group][mat][16]

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    // clusters of 1 CTA (whole rows) or 2 CTAs (each takes one half of the columns)
    const uint32_t rank = cluster_rank(), csize = cluster_size();
    const int n_clusters = gridDim.x / csize, cluster = blockIdx.x / csize;
    const int n_groups = P.M / 16;
    const int g_begin = (int)((long long)n_groups * cluster / n_clusters);
    const int g_end = (int)((long long)n_groups * (cluster + 1) / n_clusters);
    const int64_t group_bytes = 16 * P.row_bytes;
    // this CTA's columns: units [u0, u1) of the row (rank 0 takes the larger half)
    const int n_units_row = P.K / T::UK, half = csize == 2 ? (n_units_row + 1) / 2 : n_units_row;
    const int u0 = rank ? half : 0, u1 = rank ? n_units_row : half;
    const int k0 = u0 * T::UK, KR = (u1 - u0) * T::UK;
    const int CE = P.chunk_elems, NCH = (KR + CE - 1) / CE;

    // Start-up: the producer warp initialises the barriers and starts streaming at once;
    // the consumers zero the pair's sums and wait for the barriers (and, in a pair, for
    // both CTAs: cluster barrier phase 0, which the producer joins without waiting).
    if (warp == kProducer) {
        if (lane == 0) {
            for (int s = 0; s < P.n_stages; ++s) {
                mbar_init(&full[s], 1);
                mbar_init(&empty[s], kWarps);
            }
            mbar_init(xbar, 1);
            fence_mbar_init();
        }
        __syncwarp();
        if (csize == 1)
            named_bar_arrive(2, kThreads);
        else
            cluster_arrive();
        // ------------------------------------------------------------- producer
        // (weights do not depend on earlier kernels, so streaming starts at once)
        if (lane == 0) {
            const uint64_t pol = policy_evict_first();
            const int NS = P.n_stages;
            int s = 0, issued = 0;
            uint32_t ph = 0;
            bool okay = true;
            for (int gi = g_begin; gi < g_end && okay; ++gi) {
                for (int mat = 0; mat < NM && okay; ++mat) {
                    const uint8_t* base = (mat ? P.W2 : P.W) + (int64_t)gi * group_bytes + (int64_t)u0 * T::UB;
                    for (int c = 0; c < NCH; ++c) {
                        if (issued == P.stall_stage) {
                            // test of the consumers' bounded wait: stop issuing (every copy issued
                            // so far lands before the consumers reach this stage)
                            okay = false;
                            break;
                        }
                        if (!mbar_wait(&empty[s], ph ^ 1u, kWaitPolls)) {
                            record_device_error(DEVERR_EMPTY_WAIT);
                            okay = false;
                            break;
                        }
                        const uint32_t bytes = (uint32_t)(min(CE, KR - c * CE) / T::UK * T::UB);
                        mbar_arrive_expect_tx(&full[s], bytes);
                        bulk_g2s(stages + (size_t)s * P.stage_bytes, base + (int64_t)c * P.chunk_bytes, bytes,
                                 &full[s], pol);
                        ++issued;
                        if (++s == NS) {
                            s = 0;
                            ph ^= 1u;
                        }
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
        __syncwarp();
        if (csize == 2) cluster_wait();   // phase 0, joined at the start
    } else {
        // ------------------------------------------------------------- consumers
        for (int i = tid; i < P.recv_bytes / 4; i += kCons) sums[i] = 0.f;
        if (csize == 1) {
            named_bar_sync(2, kThreads);
        } else {
            // both CTAs initialised before either touches the other's shared memory
            cluster_arrive();
            cluster_wait();
        }
        float* rs = red;   // scratch for the prologue reductions
        const int K4 = P.K / 4, h0 = k0 / 4, h1 = (k0 + KR) / 4, nh = h1 - h0;
        float4* xf = reinterpret_cast<float4*>(xq);
        const float4* x4 = reinterpret_cast<const float4*>(P.x);
        const float4* w4 = reinterpret_cast<const float4*>(P.norm_w) + h0;
        // (0) Before the programmatic wait, what needs nothing from the previous kernel:
        // the RMSNorm weights of this thread's first NW float4 of x (float4 i = tid + j kCons,
        // the same float4 the passes below take) into registers, and the step's RoPE table
        // (written with the position word before the first kernel of a step that launches
        // early) into shared memory for the epilogue.
        const float rope_v = (EPI == gemv::EPI_QKV && tid < P.head_dim) ? P.rope_cs[tid] : 0.f;
        constexpr bool RMS = PRO == gemv::PRO_RMSNORM;
        constexpr int NW = RMS ? 8 : 4;
        float4 wr[NW];
#pragma unroll
        for (int j = 0; j < NW; ++j) {
            const int i = tid + j * kCons;
            wr[j] = (RMS && i < nh) ? w4[i] : make_float4(1.f, 1.f, 1.f, 1.f);
        }
        if (P.use_pdl) {
            pdl_launch_dependents();
            pdl_wait();
        }
        // (1) this CTA's columns of x into shared memory with one bulk copy (x is
        // 16-byte aligned and the half starts on a 32-column step)
        if (tid == 0 && KR > 0) {
            mbar_arrive_expect_tx(xbar, (uint32_t)KR * 4u);
            bulk_g2s(xf, P.x + k0, (uint32_t)KR * 4u, xbar, policy_evict_last());
        }
        if (KR > 0 && !mbar_wait(xbar, 0, kWaitPolls) && tid == 0) record_device_error(DEVERR_FULL_WAIT);
        // (2) one pass: the sum of squares (RMSNorm; it runs over the whole vector) and max |x w|
        // (w = 1 without RMSNorm) over the CTA's columns; float4 i = tid + j kCons
        float ss = 0.f, mw = 0.f;
        const int n_steps = KR / 32, n_rounds = (n_steps + 31) / 32, wl = lane & 7;
        auto pass1 = [&](const float4& v, const float4& w) {
            if (RMS) ss = fmaf(v.x, v.x, fmaf(v.y, v.y, fmaf(v.z, v.z, fmaf(v.w, v.w, ss))));
            mw = fmaxf(mw, fmaxf(fmaxf(fabsf(v.x * w.x), fabsf(v.y * w.y)), fmaxf(fabsf(v.z * w.z), fabsf(v.w * w.w))));
        };
#pragma unroll
        for (int j = 0; j < NW; ++j) {
            const int i = tid + j * kCons;
            if (i < nh) pass1(xf[i], wr[j]);
        }
        for (int i = tid + NW * kCons; i < nh; i += kCons)
            pass1(xf[i], RMS ? w4[i] : make_float4(1.f, 1.f, 1.f, 1.f));
        if (RMS) {
            // the other CTA's columns, from global memory, 8 loads in flight per thread
            for (int j0 = tid; j0 < K4 - nh; j0 += 8 * kCons) {
                float4 v[8];
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    const int jj = j0 + j * kCons;
                    v[j] = jj < K4 - nh ? x4[jj < h0 ? jj : jj + nh] : make_float4(0.f, 0.f, 0.f, 0.f);
                }
#pragma unroll
                for (int j = 0; j < 8; ++j)
                    ss = fmaf(v[j].x, v[j].x, fmaf(v[j].y, v[j].y, fmaf(v[j].z, v[j].z, fmaf(v[j].w, v[j].w, ss))));
            }
            ss = gemv::warp_sum(ss);
        }
        mw = gemv::warp_max(mw);
        if (lane == 0) {
            rs[warp] = ss;
            rs[kWarps + warp] = mw;
        }
        named_bar_sync(1, kCons);
        float tot = 0.f, mx = 0.f;
#pragma unroll
        for (int w = 0; w < kWarps; ++w) {
            tot += rs[w];
            mx = fmaxf(mx, rs[kWarps + w]);
        }
        // the normalised value is fl(fl(x w) inv): its largest magnitude is fl(max |x w| inv)
        const float inv = RMS ? 1.0f / sqrtf(tot / (float)P.K + P.eps) : 1.f;
        if (RMS) mx *= inv;
        // |x| 2^S < 2^22 over the CTA's columns; a zero half keeps S = 0 (all limbs zero)
        const int S = (mx > 0.f && mx <= 3.4e38f) ? max(-100, min(127, 21 - ilogbf(mx))) : 0;
        const int e_cap = min(kMaxStepShift, 127 - S);
        // (3) normalised fp32 -> limbs, in place: 8 lanes per 32-column step, float4
        // i = tid + j kCons; 4 rounds at a time, all reads of a round before its stores.
        // Step u takes 2^(S + e_u) with e_u the extra bits its own largest value leaves room
        // for (|x| 2^(S + e_u) < 2^22 still holds), and records 2^-e_u.  The step's binary
        // exponent is the largest of its 8 lanes' (each lane's from the float bits of its own
        // largest normalised magnitude; a subnormal reads as 2^-127, above its true exponent,
        // which only leaves e_u smaller): the four rounds' exponent bytes travel packed in one
        // word, so one 3-shuffle chain serves them all.
        {
            auto convert4 = [&](int j0, const float4 (&w)[4]) {
                XLimbs r[4];
                float fk[4];
                float4 v[4];
                uint32_t packed = 0;
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    const int i = tid + (j0 + k) * kCons;
                    v[k] = i < nh ? xf[i] : make_float4(0.f, 0.f, 0.f, 0.f);
                    if (RMS)
                        v[k] = make_float4(v[k].x * w[k].x * inv, v[k].y * w[k].y * inv, v[k].z * w[k].z * inv,
                                           v[k].w * w[k].w * inv);
                    const float m = fmaxf(fmaxf(fabsf(v[k].x), fabsf(v[k].y)), fmaxf(fabsf(v[k].z), fabsf(v[k].w)));
                    packed |= ((__float_as_uint(m) >> 23) & 0xFFu) << (8 * k);
                }
#pragma unroll
                for (int o = 1; o < 8; o <<= 1) packed = __vmaxu4(packed, __shfl_xor_sync(0xffffffffu, packed, o));
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    const int be = (int)((packed >> (8 * k)) & 0xFFu);   // biased exponent of the step's max
                    // a zero step (be = 0) keeps e = e_cap: its limbs are zero either way
                    const int e = be < 255 ? max(0, min(e_cap, 21 - (be - 127) - S)) : 0;
                    r[k] = x_limbs<QT == NTX_Q6_K_T, XSUMS>(v[k], __uint_as_float((uint32_t)(127 + S + e) << 23));
                    fk[k] = __uint_as_float((uint32_t)(127 - e) << 23);
                }
                __syncwarp();   // every lane of a step has read its floats before any limb word lands
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    const int u = (tid + (j0 + k) * kCons) >> 3;
                    if (u < n_steps) {
                        x_store<QT == NTX_Q6_K_T, CORE == 1 && QT == NTX_Q8_0_T, XSUMS, CORE == 0>(
                            xq + 32 * u, wl, r[k], ROWS ? 8 * (u & 3) : 0, fk[k]);
                        if (wl == 0) xsf[u] = fk[k];
                    }
                }
            };
#pragma unroll
            for (int j0 = 0; j0 < NW; j0 += 4) {
                if (j0 < n_rounds) {
                    const float4 w[4] = {wr[j0], wr[j0 + 1], wr[j0 + 2], wr[j0 + 3]};
                    convert4(j0, w);
                }
            }
            for (int j0 = NW; j0 < n_rounds; j0 += 4) {
                float4 w[4];
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    const int i = tid + (j0 + k) * kCons;
                    w[k] = (RMS && i < nh) ? w4[i] : make_float4(1.f, 1.f, 1.f, 1.f);
                }
                convert4(j0, w);
            }
        }
        if (EPI == gemv::EPI_QKV && tid < P.head_dim) rope_cs[tid] = rope_v;   // read by the epilogue
        named_bar_sync(1, kCons);   // limbs and the RoPE table complete

        const Lane L = make_lane<QT>(lane);
        // CORE 0: this lane's C columns hold limbs 0, 1 or limb 2; CORE 1 sums are whole
        const float limb_w = (CORE == 0 && (L.tig & 1)) ? 65536.f : 1.f;
        const int rgid = lane & 7, rj = lane >> 3;   // row-pair units: gid, step slot
        const int NS = P.n_stages;
        int s = 0;
        uint32_t ph = 0;
        bool dead = false;
        int gl = 0;
        const uint32_t sums0 = peer_addr(sums, 0);   // the pair's sums, in the first CTA
        for (int gi = g_begin; gi < g_end; ++gi, ++gl) {
            float* rg = red + (gl & 1) * (kWarps * 32);   // [warp][mat][16]
#pragma unroll 1
            for (int mat = 0; mat < NM; ++mat) {
                float acc0 = 0.f, acc1 = 0.f;   // this lane's shares of rows gid, gid + 8
                for (int c = 0; c < NCH; ++c) {
                    const int n_units = min(CE, KR - c * CE) / T::UK;
                    if (!dead && !mbar_wait(&full[s], ph, kWaitPolls)) {
                        record_device_error(DEVERR_FULL_WAIT);
                        dead = true;    // keep taking part in every barrier so the CTA still finishes
                    }
                    const uint8_t* st = stages + (size_t)s * P.stage_bytes;
                    if (!dead) {
                        const uint32_t* xc = xq + 32 * (c * CE / 32);
                        const float* fc = xsf + c * CE / 32;
                        if (CORE == 0) {
                            for (int un = warp; un < n_units; un += kWarps)
                                Unit<QT>::run(st + (size_t)un * T::UB, xc + 32 * SPU * un, fc + SPU * un, L, acc0,
                                              acc1);
                        } else if constexpr (QT == NTX_Q8_0_T) {
#pragma unroll 4
                            for (int un = warp; un < n_units; un += kWarps)
                                Dot<QT>::run(st + (size_t)un * T::UB, xc + 32 * un, fc + un, L, acc0, acc1);
                        } else if constexpr (QT == NTX_Q4_0_T) {
                            // a warp takes 4 units (steps) at a time, one per 8 threads
                            const int sx = 8 * ((c * CE / 32 + rj) & 3);
#pragma unroll 2
                            for (int u4 = 4 * warp; u4 < n_units; u4 += 4 * kWarps) {
                                const int un = u4 + rj;
                                if (un < n_units)
                                    Row<QT>::run(st + (size_t)un * T::UB, xc + 32 * un, sx, fc[un], rgid, acc0, acc1);
                            }
                        } else {
#pragma unroll 2
                            for (int un = warp; un < n_units; un += kWarps)
                                Row<QT>::run(st + (size_t)un * T::UB, xc + 32 * SPU * un, fc + SPU * un, rgid, rj,
                                             acc0, acc1);
                        }
                    }
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&empty[s]);
                    if (++s == NS) {
                        s = 0;
                        ph ^= 1u;
                    }
                }
                if constexpr (ROWS) {
                    // sum over the 4 threads of each gid: lane g < 8 ends with rows g, g + 8
                    acc0 += __shfl_xor_sync(0xffffffffu, acc0, 8);
                    acc1 += __shfl_xor_sync(0xffffffffu, acc1, 8);
                    acc0 += __shfl_xor_sync(0xffffffffu, acc0, 16);
                    acc1 += __shfl_xor_sync(0xffffffffu, acc1, 16);
                    if (lane < 8) {
                        rg[warp * 32 + mat * 16 + lane] = acc0;
                        rg[warp * 32 + mat * 16 + lane + 8] = acc1;
                    }
                } else {
                    // quad reduction (with the limb weights of the MMA's C columns): lane tig 0
                    // ends with rows gid, gid + 8
                    acc0 *= limb_w;
                    acc1 *= limb_w;
                    acc0 += __shfl_xor_sync(0xffffffffu, acc0, 1);
                    acc1 += __shfl_xor_sync(0xffffffffu, acc1, 1);
                    acc0 += __shfl_xor_sync(0xffffffffu, acc0, 2);
                    acc1 += __shfl_xor_sync(0xffffffffu, acc1, 2);
                    if (L.tig == 0) {
                        rg[warp * 32 + mat * 16 + L.gid] = acc0;
                        rg[warp * 32 + mat * 16 + L.gid + 8] = acc1;
                    }
                }
            }
            named_bar_sync(1, kCons);
            if (tid < 16 * NM) {
                // the 8 warps' sums in warp order, scaled by 2^-S, into the pair's sums
                const int row = tid & 15, mat = tid >> 4;
                float t = 0.f;
#pragma unroll
                for (int w = 0; w < kWarps; ++w) t += rg[w * 32 + mat * 16 + row];
                t = gemv::scale2(t, -S);
                const int slot = (gl * NM + mat) * 16 + row;
                if (csize == 1)
                    sums[slot] = t;
                else
                    red_add_cluster(sums0 + 4u * slot, t);
            }
        }
        // every addend of the pair has landed once both CTAs pass the cluster barrier
        cluster_sync(csize);
        if (rank == 0) {
            // epilogue of all rows of the pair's groups; RoPE partners (2i, 2i + 1) sit in adjacent lanes
            const int32_t pos = (EPI == gemv::EPI_QKV) ? (P.pos_dev ? *P.pos_dev : P.pos) : 0;
            const int n_rows = (g_end - g_begin) * 16;
            for (int base = 0; base < n_rows; base += kCons) {
                const int r = base + tid;
                const bool ok = r < n_rows;
                const int gl2 = ok ? r >> 4 : 0, rr = r & 15;
                const float a = ok ? sums[(gl2 * NM) * 16 + rr] : 0.f;
                const float b = (ok && NM == 2) ? sums[(gl2 * NM + 1) * 16 + rr] : 0.f;
                epilogue<EPI>(P, g_begin * 16 + r, ok, a, b, pos, rope_cs);
            }
        }
        return;
    }
    // the producer warp meets the consumers at the cluster barrier
    cluster_sync(csize);
}

}  // namespace qmma
}  // namespace ntx
