// qmma_multi.cuh - the tiled GEMV over several input vectors at once: y_v = W x_v for
// v < NX (NX = 2..4), each weight streamed from HBM and unpacked once, then dotted with
// every vector.  It is the small-N GEMM of the verification pass of self-speculative
// decoding ("Funciones principales" of the ntransformer news summary: the drafted tokens
// are checked together), where one pass of the model covers NX positions.
//
// The arithmetic of each product is that of the single-vector kernel (qmma.cuh): every
// x_v becomes 24-bit fixed point with its own exponent S_v and its own per-step
// exponents, the codes are dotted with the limbs by dp4a on the CUDA cores, the block
// scales apply in integer arithmetic and in fp32 once per step.  The structure is that
// kernel's whole-row layout (one CTA per SM, 8 consumer warps and a producer warp,
// stages of one 16-row group x one chunk in a shared-memory ring), with NX x regions
// and NX row sums per group; there are no CTA pairs (the rows of every decode shape fit
// whole).
#pragma once

#include "qmma.cuh"

namespace ntx {
namespace qmma {

constexpr int kMaxNX = gemv::kMaxVecs;
using gemv::Vecs;

// Shared memory of the multi-vector kernel: mbarriers, then the per-group reduction
// scratch [2][warp][NX][mat][16], the RoPE tables [NX][64][2], the exponents S_v, then the
// NX x regions (x_bytes each), the ring and the row sums [group][NX][mat][16].
constexpr int kMOffRed = 256;
constexpr int kMOffRope = kMOffRed + 2 * kWarps * kMaxNX * 2 * 16 * 4;
constexpr int kMOffS = kMOffRope + kMaxNX * 128 * 4;
constexpr int kMHeader = kMOffS + 64;

// ------------------------------------------------------------------ units
// The unit's codes and scales are read and unpacked once; the loop over v reads the
// vector's x words (xs + v XW) and step factors (fs + v XW) and accumulates acc0[v] /
// acc1[v] (this thread's shares of rows gid / gid + 8), exactly as the single-vector unit.

template <int QT, int NX>
struct RowsN;

template <int NX>
struct RowsN<NTX_Q8_0_T, NX> {
    // lane units: xs = the step's words of vector 0 (PAIRED layout, the factor inside)
    static __device__ __forceinline__ void run(const uint8_t* U, const uint32_t* xs, int XW, const Lane& L,
                                               float (&acc0)[NX], float (&acc1)[NX])
    {
        const uint4 a = *reinterpret_cast<const uint4*>(U + 16 * L.lane);
        const float2 d = d_pair(U + 512 + 4 * L.gid);
#pragma unroll
        for (int v = 0; v < NX; ++v) {
            uint2 X[3];
            float f;
            x_words(xs + v * XW, L.tig, X, f);
            int c0[3], c1[3];
#pragma unroll
            for (int l = 0; l < 3; ++l) {
                c0[l] = dp4(a.z, X[l].y, dp4(a.x, X[l].x, 0));
                c1[l] = dp4(a.w, X[l].y, dp4(a.y, X[l].x, 0));
            }
            acc0[v] = fmaf(d.x * f, limbs_f(c0[0], c0[1], c0[2]), acc0[v]);
            acc1[v] = fmaf(d.y * f, limbs_f(c1[0], c1[1], c1[2]), acc1[v]);
        }
    }
};

template <int NX>
struct RowsN<NTX_Q4_0_T, NX> {
    // row-pair unit of one step: xs / fs of vector 0, sx the step's swizzle
    static __device__ __forceinline__ void run(const uint8_t* U, const uint32_t* xs, const float* fs, int XW, int sx,
                                               int g, float (&acc0)[NX], float (&acc1)[NX])
    {
        const uint4* Lp = reinterpret_cast<const uint4*>(U + 32 * g);
        const uint4 u0 = Lp[0], u1 = Lp[1];
        const uint32_t Pw[4] = {u0.x, u0.z, u1.x, u1.z}, Qw[4] = {u0.y, u0.w, u1.y, u1.w};
        const uint32_t M = 0x0F0F0F0Fu;
        uint32_t Plo[4], Phi[4], Qlo[4], Qhi[4];
#pragma unroll
        for (int t = 0; t < 4; ++t) {
            Plo[t] = Pw[t] & M;
            Phi[t] = (Pw[t] >> 4) & M;
            Qlo[t] = Qw[t] & M;
            Qhi[t] = (Qw[t] >> 4) & M;
        }
        const float2 d = d_pair(U + 256 + 4 * g);
#pragma unroll
        for (int v = 0; v < NX; ++v) {
            const uint32_t* x = xs + v * XW;
            uint4 X[3][2];
            x_step(x, sx, X);
            const uint4 xsum = *reinterpret_cast<const uint4*>(x + (24 ^ sx));
            int c0[3], c1[3];
#pragma unroll
            for (int l = 0; l < 3; ++l) {
                // codes carry +8: start at -8 x (the limb's sum over the step)
                c0[l] = c1[l] = -8 * (int)comp(xsum, l);
#pragma unroll
                for (int t = 0; t < 4; ++t) {
                    c0[l] = dp4(Phi[t], comp(X[l][1], t), dp4(Plo[t], comp(X[l][0], t), c0[l]));
                    c1[l] = dp4(Qhi[t], comp(X[l][1], t), dp4(Qlo[t], comp(X[l][0], t), c1[l]));
                }
            }
            const float f = fs[v * XW];
            acc0[v] = fmaf(d.x * f, limbs_f2(c0[0], c0[1], c0[2]), acc0[v]);
            acc1[v] = fmaf(d.y * f, limbs_f2(c1[0], c1[1], c1[2]), acc1[v]);
        }
    }
};

template <int NX>
struct RowsN<NTX_Q6_K_T, NX> {
    // superblock unit: xs / fs of vector 0 at the unit; the thread takes steps j and j + 4
    static __device__ __forceinline__ void run(const uint8_t* U, const uint32_t* xs, const float* fs, int XW, int g,
                                               int j, float (&acc0)[NX], float (&acc1)[NX])
    {
        const uint4 se = *reinterpret_cast<const uint4*>(U + 3072 + 32 * g);
        const uint4 so = *reinterpret_cast<const uint4*>(U + 3072 + 32 * g + 16);
        const uint32_t sel = sbyte_sel(j);
        const uint32_t M6 = 0x3F3F3F3Fu;
        const float2 d = d_pair(U + 3328 + 4 * g);
#pragma unroll
        for (int k = 0; k < 2; ++k) {
            const int m = j + 4 * k;
            const uint4* Lp = reinterpret_cast<const uint4*>(U + 384 * m + 48 * g);
            const uint4 v0 = Lp[0], v1 = Lp[1], v2 = Lp[2];
            const uint32_t A[4] = {v0.x, v0.w, v1.z, v2.y}, B[4] = {v0.y, v1.x, v1.w, v2.z},
                           C[4] = {v0.z, v1.y, v2.x, v2.w};
            const int s_e0 = sbyte_r(k ? se.y : se.x, sel), s_e1 = sbyte_r(k ? se.w : se.z, sel);
            const int s_o0 = sbyte_r(k ? so.y : so.x, sel), s_o1 = sbyte_r(k ? so.w : so.z, sel);
            uint32_t a0[4], a1[4], a2[4], a3[4];
#pragma unroll
            for (int t = 0; t < 4; ++t) {
                a0[t] = A[t] & M6;
                a1[t] = B[t] & M6;
                a2[t] = C[t] & M6;
                a3[t] = ((A[t] >> 6) & 0x03030303u) | ((B[t] >> 4) & 0x0C0C0C0Cu) | ((C[t] >> 2) & 0x30303030u);
            }
            const int sx = 8 * j;
#pragma unroll
            for (int v = 0; v < NX; ++v) {
                const uint32_t* x = xs + v * XW + 32 * m;
                uint4 X[3][2];
                x_step(x, sx, X);
                const uint4 h0 = *reinterpret_cast<const uint4*>(x + (24 ^ sx));
                const uint4 h1 = *reinterpret_cast<const uint4*>(x + (28 ^ sx));
                int p0[3] = {0, 0, 0}, p1[3] = {0, 0, 0};
#pragma unroll
                for (int l = 0; l < 3; ++l) {
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
                const float f = fs[v * XW + m];
                acc0[v] = fmaf(d.x * f, limbs_f(p0[0], p0[1], p0[2]), acc0[v]);
                acc1[v] = fmaf(d.y * f, limbs_f(p1[0], p1[1], p1[2]), acc1[v]);
            }
        }
    }
};

// Q4_K (FIVE = false) and Q5_K (FIVE = true): the 4-bit codes (with the fifth bit ORed in
// from the step's fifth-bit words for Q5_K), 6-bit scales and mins.
template <bool FIVE, int NX>
__device__ __forceinline__ void rows_k4(const uint8_t* U, const uint32_t* xs, const float* fs, int XW, int g, int j,
                                        float (&acc0)[NX], float (&acc1)[NX])
{
    constexpr int SOFF = FIVE ? 2560 : 2048, DOFF = FIVE ? 2752 : 2240, STEP = FIVE ? 320 : 256;
    const uint8_t* sv = U + SOFF + 24 * g;
    const uint32_t M = 0x0F0F0F0Fu;
    const uint2 dd = *reinterpret_cast<const uint2*>(U + DOFF + 8 * g);
    const float2 d = __half22float2(*reinterpret_cast<const __half2*>(&dd.x));
    const float2 dm = __half22float2(*reinterpret_cast<const __half2*>(&dd.y));
#pragma unroll
    for (int k = 0; k < 2; ++k) {
        const int m = j + 4 * k;
        const uint32_t nw = *reinterpret_cast<const uint32_t*>(sv + 4 * (m >> 1));
        const uint32_t hw = *reinterpret_cast<const uint32_t*>(sv + 16 + 4 * k);
        const uint32_t S = ((nw >> (4 * (m & 1))) & 0x0F0F0F0Fu) | (((hw >> (2 * j)) & 0x03030303u) << 4);
        const uint4* Lp = reinterpret_cast<const uint4*>(U + STEP * m + 32 * g);
        const uint4 u0 = Lp[0], u1 = Lp[1];
        const uint32_t Pw[4] = {u0.x, u0.z, u1.x, u1.z}, Qw[4] = {u0.y, u0.w, u1.y, u1.w};
        uint32_t Plo[4], Phi[4], Qlo[4], Qhi[4];
#pragma unroll
        for (int t = 0; t < 4; ++t) {
            Plo[t] = Pw[t] & M;
            Phi[t] = (Pw[t] >> 4) & M;
            Qlo[t] = Qw[t] & M;
            Qhi[t] = (Qw[t] >> 4) & M;
        }
        if constexpr (FIVE) {
            const uint2 H = *reinterpret_cast<const uint2*>(U + STEP * m + 256 + 8 * g);
            Plo[0] |= q5_bits<0>(H.x);
            Phi[0] |= q5_bits<1>(H.x);
            Plo[1] |= q5_bits<2>(H.x);
            Phi[1] |= q5_bits<3>(H.x);
            Plo[2] |= q5_bits<4>(H.x);
            Phi[2] |= q5_bits<5>(H.x);
            Plo[3] |= q5_bits<6>(H.x);
            Phi[3] |= q5_bits<7>(H.x);
            Qlo[0] |= q5_bits<0>(H.y);
            Qhi[0] |= q5_bits<1>(H.y);
            Qlo[1] |= q5_bits<2>(H.y);
            Qhi[1] |= q5_bits<3>(H.y);
            Qlo[2] |= q5_bits<4>(H.y);
            Qhi[2] |= q5_bits<5>(H.y);
            Qlo[3] |= q5_bits<6>(H.y);
            Qhi[3] |= q5_bits<7>(H.y);
        }
        const int sc0 = ubyte<0>(S), sc1 = ubyte<1>(S), mn0 = ubyte<2>(S), mn1 = ubyte<3>(S);
        const int sx = 8 * j;
#pragma unroll
        for (int v = 0; v < NX; ++v) {
            const uint32_t* x = xs + v * XW + 32 * m;
            uint4 X[3][2];
            x_step(x, sx, X);
            const uint4 xsum = *reinterpret_cast<const uint4*>(x + (24 ^ sx));
            int p0[3] = {0, 0, 0}, p1[3] = {0, 0, 0}, n0[3] = {0, 0, 0}, n1[3] = {0, 0, 0};
#pragma unroll
            for (int l = 0; l < 3; ++l) {
                int c0 = 0, c1 = 0;
#pragma unroll
                for (int t = 0; t < 4; ++t) {
                    c0 = dp4(Phi[t], comp(X[l][1], t), dp4(Plo[t], comp(X[l][0], t), c0));
                    c1 = dp4(Qhi[t], comp(X[l][1], t), dp4(Qlo[t], comp(X[l][0], t), c1));
                }
                p0[l] = sc0 * c0;
                p1[l] = sc1 * c1;
                n0[l] = mn0 * (int)comp(xsum, l);
                n1[l] = mn1 * (int)comp(xsum, l);
            }
            const float f = fs[v * XW + m];
            if constexpr (FIVE) {
                acc0[v] = fmaf(d.x * f, limbs_f(p0[0], p0[1], p0[2]),
                               fmaf(-dm.x * f, limbs_f2(n0[0], n0[1], n0[2]), acc0[v]));
                acc1[v] = fmaf(d.y * f, limbs_f(p1[0], p1[1], p1[2]),
                               fmaf(-dm.y * f, limbs_f2(n1[0], n1[1], n1[2]), acc1[v]));
            } else {
                acc0[v] = fmaf(d.x * f, limbs_f2(p0[0], p0[1], p0[2]),
                               fmaf(-dm.x * f, limbs_f2(n0[0], n0[1], n0[2]), acc0[v]));
                acc1[v] = fmaf(d.y * f, limbs_f2(p1[0], p1[1], p1[2]),
                               fmaf(-dm.y * f, limbs_f2(n1[0], n1[1], n1[2]), acc1[v]));
            }
        }
    }
}

template <int NX>
struct RowsN<NTX_Q4_K_T, NX> {
    static __device__ __forceinline__ void run(const uint8_t* U, const uint32_t* xs, const float* fs, int XW, int g,
                                               int j, float (&acc0)[NX], float (&acc1)[NX])
    {
        rows_k4<false, NX>(U, xs, fs, XW, g, j, acc0, acc1);
    }
};

template <int NX>
struct RowsN<NTX_Q5_K_T, NX> {
    static __device__ __forceinline__ void run(const uint8_t* U, const uint32_t* xs, const float* fs, int XW, int g,
                                               int j, float (&acc0)[NX], float (&acc1)[NX])
    {
        rows_k4<true, NX>(U, xs, fs, XW, g, j, acc0, acc1);
    }
};

// Tensor-core units (CORE 0): per step the A fragment (the codes) is built once and
// multiplied with each vector's B fragment (its limbs, columns gid < 3) by one m16n8k32
// integer MMA each; per vector the products, offsets, scales and the accumulation are
// those of the single-vector tensor-core unit (Unit<QT> in qmma.cuh), so acc0[v] / acc1[v]
// end in units of the lane's C columns' limb (the quad reduction applies the weights).

template <int QT, int NX>
struct UnitsN;

template <int NX>
struct UnitsN<NTX_Q8_0_T, NX> {
    static __device__ __forceinline__ void run(const uint8_t* U, const uint32_t* xs, const float* fs, int XW,
                                               const Lane& L, float (&acc0)[NX], float (&acc1)[NX])
    {
        const uint4 a4 = *reinterpret_cast<const uint4*>(U + 16 * L.lane);
        const uint32_t a[4] = {a4.x, a4.y, a4.z, a4.w};
        const float2 d = d_pair(U + 512 + 4 * L.gid);
#pragma unroll
        for (int v = 0; v < NX; ++v) {
            uint32_t b0, b1;
            b_frag<NTX_Q8_0_T>(xs + v * XW, L, b0, b1);
            int c[4];
            mma_s8(c, a, b0, b1);
            const float f = fs[v * XW];
            acc0[v] = fmaf((float)(c[0] + 256 * c[1]), d.x * f, acc0[v]);
            acc1[v] = fmaf((float)(c[2] + 256 * c[3]), d.y * f, acc1[v]);
        }
    }
};

template <int NX>
struct UnitsN<NTX_Q4_0_T, NX> {
    static __device__ __forceinline__ void run(const uint8_t* U, const uint32_t* xs, const float* fs, int XW,
                                               const Lane& L, float (&acc0)[NX], float (&acc1)[NX])
    {
        const uint2 pq = *reinterpret_cast<const uint2*>(U + 8 * L.lane);
        const uint32_t M = 0x0F0F0F0Fu;
        const uint32_t a[4] = {pq.x & M, pq.y & M, (pq.x >> 4) & M, (pq.y >> 4) & M};
        const float2 d = d_pair(U + 256 + 4 * L.gid);
#pragma unroll
        for (int v = 0; v < NX; ++v) {
            const uint32_t* x = xs + v * XW;
            uint32_t b0, b1;
            b_frag<NTX_Q4_0_T>(x, L, b0, b1);
            int c[4];
            mma_u8(c, a, b0, b1);
            // codes carry +8: subtract 8 x (this lane's two columns' limb sums)
            const int2 X = *reinterpret_cast<const int2*>(x + 24 + 2 * L.tig);
            const int off = -8 * (X.x + 256 * X.y);
            const float f = fs[v * XW];
            acc0[v] = fmaf((float)(c[0] + 256 * c[1] + off), d.x * f, acc0[v]);
            acc1[v] = fmaf((float)(c[2] + 256 * c[3] + off), d.y * f, acc1[v]);
        }
    }
};

template <int NX>
struct UnitsN<NTX_Q6_K_T, NX> {
    static __device__ __forceinline__ void run(const uint8_t* U, const uint32_t* xs, const float* fs, int XW,
                                               const Lane& L, float (&acc0)[NX], float (&acc1)[NX])
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
            int s0, s1;
            if (m < 4) {
                s0 = m == 0 ? sbyte<0>(sv.x) : m == 1 ? sbyte<1>(sv.x) : m == 2 ? sbyte<2>(sv.x) : sbyte<3>(sv.x);
                s1 = m == 0 ? sbyte<0>(sv.z) : m == 1 ? sbyte<1>(sv.z) : m == 2 ? sbyte<2>(sv.z) : sbyte<3>(sv.z);
            } else {
                s0 = m == 4 ? sbyte<0>(sv.y) : m == 5 ? sbyte<1>(sv.y) : m == 6 ? sbyte<2>(sv.y) : sbyte<3>(sv.y);
                s1 = m == 4 ? sbyte<0>(sv.w) : m == 5 ? sbyte<1>(sv.w) : m == 6 ? sbyte<2>(sv.w) : sbyte<3>(sv.w);
            }
#pragma unroll
            for (int v = 0; v < NX; ++v) {
                const uint32_t* x = xs + v * XW + 32 * m;
                uint32_t b0, b1;
                b_frag<NTX_Q6_K_T>(x, L, b0, b1);
                int c[4];
                mma_u8(c, a, b0, b1);
                const int2 X = *reinterpret_cast<const int2*>(x + 24 + 2 * L.tig);
                // codes carry +32; the step's column totals are exact integers before the fp32 step
                const int p0 = s0 * (c[0] - 32 * X.x), p1 = s0 * (c[1] - 32 * X.y);
                const int q0 = s1 * (c[2] - 32 * X.x), q1 = s1 * (c[3] - 32 * X.y);
                const float f = fs[v * XW + m];
                acc0[v] = fmaf(d.x * f, fmaf(256.f, (float)p1, (float)p0), acc0[v]);
                acc1[v] = fmaf(d.y * f, fmaf(256.f, (float)q1, (float)q0), acc1[v]);
            }
        }
    }
};

// Q4_K (FIVE = false) and Q5_K (FIVE = true) on the tensor cores
template <bool FIVE, int NX>
__device__ __forceinline__ void units_k4(const uint8_t* U, const uint32_t* xs, const float* fs, int XW, const Lane& L,
                                         float (&acc0)[NX], float (&acc1)[NX])
{
    constexpr int SOFF = FIVE ? 2560 : 2048, DOFF = FIVE ? 2752 : 2240, STEP = FIVE ? 320 : 256;
    uint32_t S[8];
    q4k_scale_words<SOFF>(U, L.gid, S);
    const uint2 dd = *reinterpret_cast<const uint2*>(U + DOFF + 8 * L.gid);
    const float2 d = __half22float2(*reinterpret_cast<const __half2*>(&dd.x));
    const float2 dm = __half22float2(*reinterpret_cast<const __half2*>(&dd.y));
    const uint32_t M = 0x0F0F0F0Fu;
#pragma unroll
    for (int m = 0; m < 8; ++m) {
        const uint2 pq = *reinterpret_cast<const uint2*>(U + STEP * m + 8 * L.lane);
        uint32_t a[4] = {pq.x & M, pq.y & M, (pq.x >> 4) & M, (pq.y >> 4) & M};
        if constexpr (FIVE) {
            const uint2 H = *reinterpret_cast<const uint2*>(U + STEP * m + 256 + 8 * L.gid);
            a[0] |= q5_bits_r(H.x, 2 * L.tig);
            a[1] |= q5_bits_r(H.y, 2 * L.tig);
            a[2] |= q5_bits_r(H.x, 2 * L.tig + 1);
            a[3] |= q5_bits_r(H.y, 2 * L.tig + 1);
        }
        const int sc0 = ubyte<0>(S[m]), sc1 = ubyte<1>(S[m]), mn0 = ubyte<2>(S[m]), mn1 = ubyte<3>(S[m]);
#pragma unroll
        for (int v = 0; v < NX; ++v) {
            const uint32_t* x = xs + v * XW + 32 * m;
            uint32_t b0, b1;
            b_frag<FIVE ? NTX_Q5_K_T : NTX_Q4_K_T>(x, L, b0, b1);
            int c[4];
            mma_u8(c, a, b0, b1);
            const int2 X = *reinterpret_cast<const int2*>(x + 24 + 2 * L.tig);
            const int xp = X.x + 256 * X.y;
            const float f = fs[v * XW + m];
            acc0[v] = fmaf(d.x * f, fmaf(256.f, (float)(sc0 * c[1]), (float)(sc0 * c[0])),
                           fmaf(-dm.x * f, (float)(mn0 * xp), acc0[v]));
            acc1[v] = fmaf(d.y * f, fmaf(256.f, (float)(sc1 * c[3]), (float)(sc1 * c[2])),
                           fmaf(-dm.y * f, (float)(mn1 * xp), acc1[v]));
        }
    }
}

template <int NX>
struct UnitsN<NTX_Q4_K_T, NX> {
    static __device__ __forceinline__ void run(const uint8_t* U, const uint32_t* xs, const float* fs, int XW,
                                               const Lane& L, float (&acc0)[NX], float (&acc1)[NX])
    {
        units_k4<false, NX>(U, xs, fs, XW, L, acc0, acc1);
    }
};

template <int NX>
struct UnitsN<NTX_Q5_K_T, NX> {
    static __device__ __forceinline__ void run(const uint8_t* U, const uint32_t* xs, const float* fs, int XW,
                                               const Lane& L, float (&acc0)[NX], float (&acc1)[NX])
    {
        units_k4<true, NX>(U, xs, fs, XW, L, acc0, acc1);
    }
};

// ------------------------------------------------------------------ epilogue

// Output row `row` of vector v (t = row total, t_up the up-projection total for SwiGLU).
// Called by whole warps; `ok` is false for lanes past the last row.
template <int EPI>
__device__ __forceinline__ void epilogue_v(const Params& P, const Vecs& V, int v, int row, bool ok, float t,
                                           float t_up, int32_t pos, const float* rope_cs)
{
    using namespace gemv;
    if (EPI == EPI_STORE) {
        if (ok) V.y[v][row] = t;
    } else if (EPI == EPI_ADD) {
        if (ok) V.y[v][row] = V.y[v][row] + t;
    } else if (EPI == EPI_SWIGLU) {
        if (ok) V.y[v][row] = t / (1.0f + expf(-t)) * t_up;
    } else if (EPI == EPI_QKV) {
        const float other = __shfl_xor_sync(0xffffffffu, t, 1);
        if (!ok) return;
        float val = t;
        const int hd = P.head_dim;
        if (row < P.q_rows + P.kv_rows) {
            const int pi = (row % hd) / 2;
            const float cf = rope_cs[2 * pi], sf = rope_cs[2 * pi + 1];
            val = (row & 1) ? (other * sf + t * cf) : (t * cf - other * sf);
        }
        if (row < P.q_rows) {
            V.q_out[v][row] = val;
        } else {
            const int kvr = row - P.q_rows;
            const bool is_v = kvr >= P.kv_rows;
            const int jj = is_v ? kvr - P.kv_rows : kvr;
            const int g = jj / hd, dd = jj % hd;
            __half* cache = is_v ? P.v_cache : P.k_cache;
            cache[((int64_t)g * P.max_ctx + pos) * hd + dd] = __float2half_rn(val);
        }
    }
}

// ------------------------------------------------------------------ kernel

// CORE 1: dp4a on the CUDA cores (RowsN); CORE 0: the integer tensor cores (UnitsN).
template <int QT, int EPI, int PRO, int NX, int CORE>
__global__ void __launch_bounds__(kThreads, 1) qmma_multi_kernel(const Params P, const Vecs V)
{
    using T = gemv::Tiled<QT>;
    constexpr int NM = EPI == gemv::EPI_SWIGLU ? 2 : 1;
    constexpr int SPU = T::UK / 32;
    constexpr bool ROWS = CORE == 1 && QT != NTX_Q8_0_T;           // row-pair units
    constexpr bool XSUMS = !(CORE == 1 && QT == NTX_Q8_0_T);       // the Q8_0 lane units read no limb sums
    constexpr bool RMS = PRO == gemv::PRO_RMSNORM;
    constexpr int RG = kWarps * NX * NM * 16;   // floats of one reduction buffer

    extern __shared__ __align__(128) uint8_t smem[];
    uint64_t* full = reinterpret_cast<uint64_t*>(smem);
    uint64_t* empty = full + kMaxStages;
    uint64_t* xbar = reinterpret_cast<uint64_t*>(smem + kOffXBar);
    float* red = reinterpret_cast<float*>(smem + kMOffRed);
    float* rope_sm = reinterpret_cast<float*>(smem + kMOffRope);
    int* S_sm = reinterpret_cast<int*>(smem + kMOffS);
    uint32_t* xq = reinterpret_cast<uint32_t*>(smem + kMHeader);
    const int XW = P.x_bytes / 4;                      // words per vector region
    uint8_t* stages = smem + kMHeader + (size_t)NX * P.x_bytes;
    float* sums = reinterpret_cast<float*>(stages + (size_t)P.n_stages * P.stage_bytes);   // [group][v][mat][16]

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int n_groups = P.M / 16;
    const int g_begin = (int)((long long)n_groups * blockIdx.x / gridDim.x);
    const int g_end = (int)((long long)n_groups * (blockIdx.x + 1) / gridDim.x);
    const int64_t group_bytes = 16 * P.row_bytes;
    const int K = P.K, CE = P.chunk_elems, NCH = (K + CE - 1) / CE;

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
        named_bar_arrive(2, kThreads);
        // ------------------------------------------------------------- producer
        if (lane == 0) {
            const uint64_t pol = policy_evict_first();
            const int NS = P.n_stages;
            int s = 0, issued = 0;
            uint32_t ph = 0;
            bool okay = true;
            for (int gi = g_begin; gi < g_end && okay; ++gi) {
                for (int mat = 0; mat < NM && okay; ++mat) {
                    const uint8_t* base = (mat ? P.W2 : P.W) + (int64_t)gi * group_bytes;
                    for (int c = 0; c < NCH; ++c) {
                        if (issued == P.stall_stage) {
                            // test of the consumers' bounded wait: stop issuing
                            okay = false;
                            break;
                        }
                        if (!mbar_wait(&empty[s], ph ^ 1u, kWaitPolls)) {
                            record_device_error(DEVERR_EMPTY_WAIT);
                            okay = false;
                            break;
                        }
                        const uint32_t bytes = (uint32_t)(min(CE, K - c * CE) / T::UK * T::UB);
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
            if (!okay) {
                // the stages issued last must complete before the CTA may exit
                for (int k = 1; k <= NS && k <= issued; ++k) {
                    const int jj = issued - k;
                    mbar_wait(&full[jj % NS], (uint32_t)(jj / NS) & 1u, 1u << 20);
                }
            }
        }
        return;
    }

    // ----------------------------------------------------------------- consumers
    named_bar_sync(2, kThreads);
    const int nh = K / 4, n_steps = K / 32, n_rounds = (n_steps + 31) / 32, wl = lane & 7;
    const float4* w4 = reinterpret_cast<const float4*>(P.norm_w);
    // before the programmatic wait: the RoPE tables of the vectors (written with their
    // step words before the first kernel of the pass)
    if (EPI == gemv::EPI_QKV && tid < P.head_dim)
        for (int v = 0; v < NX; ++v) rope_sm[v * 128 + tid] = V.rope_cs[v][tid];
    if (P.use_pdl) {
        pdl_launch_dependents();
        pdl_wait();
    }
    // (1) every vector into its x region, one bulk copy each (x 16-byte aligned)
    if (tid == 0) {
        mbar_arrive_expect_tx(xbar, (uint32_t)(NX * K * 4));
        for (int v = 0; v < NX; ++v)
            bulk_g2s(xq + (size_t)v * XW, V.x[v], (uint32_t)K * 4u, xbar, policy_evict_last());
    }
    if (!mbar_wait(xbar, 0, kWaitPolls) && tid == 0) record_device_error(DEVERR_FULL_WAIT);

    // (2) + (3) per vector, as the single-vector prologue: sum of squares and max |x w| in
    // one pass, then normalised fp32 -> limbs in place with each step's exponent
#pragma unroll 1
    for (int v = 0; v < NX; ++v) {
        uint32_t* xv = xq + (size_t)v * XW;
        float4* xf = reinterpret_cast<float4*>(xv);
        float* xsf = reinterpret_cast<float*>(xv) + P.fs_off / 4;
        float ss = 0.f, mw = 0.f;
        for (int i = tid; i < nh; i += kCons) {
            const float4 x = xf[i];
            const float4 w = RMS ? w4[i] : make_float4(1.f, 1.f, 1.f, 1.f);
            if (RMS) ss = fmaf(x.x, x.x, fmaf(x.y, x.y, fmaf(x.z, x.z, fmaf(x.w, x.w, ss))));
            mw = fmaxf(mw, fmaxf(fmaxf(fabsf(x.x * w.x), fabsf(x.y * w.y)), fmaxf(fabsf(x.z * w.z), fabsf(x.w * w.w))));
        }
        if (RMS) ss = gemv::warp_sum(ss);
        mw = gemv::warp_max(mw);
        if (lane == 0) {
            red[warp] = ss;
            red[kWarps + warp] = mw;
        }
        named_bar_sync(1, kCons);
        float tot = 0.f, mx = 0.f;
#pragma unroll
        for (int w = 0; w < kWarps; ++w) {
            tot += red[w];
            mx = fmaxf(mx, red[kWarps + w]);
        }
        const float inv = RMS ? 1.0f / sqrtf(tot / (float)K + P.eps) : 1.f;
        if (RMS) mx *= inv;
        const int S = (mx > 0.f && mx <= 3.4e38f) ? max(-100, min(127, 21 - ilogbf(mx))) : 0;
        const int e_cap = min(kMaxStepShift, 127 - S);
        if (tid == 0) S_sm[v] = S;
        for (int j0 = 0; j0 < n_rounds; j0 += 4) {
            XLimbs r[4];
            float fk[4];
            float4 x[4];
            uint32_t packed = 0;   // the four rounds' exponent bytes of each lane's largest value
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const int i = tid + (j0 + k) * kCons;
                x[k] = i < nh ? xf[i] : make_float4(0.f, 0.f, 0.f, 0.f);
                if (RMS) {
                    const float4 w = i < nh ? w4[i] : make_float4(1.f, 1.f, 1.f, 1.f);
                    x[k] = make_float4(x[k].x * w.x * inv, x[k].y * w.y * inv, x[k].z * w.z * inv, x[k].w * w.w * inv);
                }
                const float m = fmaxf(fmaxf(fabsf(x[k].x), fabsf(x[k].y)), fmaxf(fabsf(x[k].z), fabsf(x[k].w)));
                packed |= ((__float_as_uint(m) >> 23) & 0xFFu) << (8 * k);
            }
#pragma unroll
            for (int o = 1; o < 8; o <<= 1) packed = __vmaxu4(packed, __shfl_xor_sync(0xffffffffu, packed, o));
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const int be = (int)((packed >> (8 * k)) & 0xFFu);
                const int e = be < 255 ? max(0, min(e_cap, 21 - (be - 127) - S)) : 0;
                r[k] = x_limbs<QT == NTX_Q6_K_T, XSUMS>(x[k], __uint_as_float((uint32_t)(127 + S + e) << 23));
                fk[k] = __uint_as_float((uint32_t)(127 - e) << 23);
            }
            __syncwarp();   // every lane of a step has read its floats before any limb word lands
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const int u = (tid + (j0 + k) * kCons) >> 3;
                if (u < n_steps) {
                    x_store<QT == NTX_Q6_K_T, CORE == 1 && QT == NTX_Q8_0_T, XSUMS, CORE == 0>(
                        xv + 32 * u, wl, r[k], ROWS ? 8 * (u & 3) : 0, fk[k]);
                    if (wl == 0) xsf[u] = fk[k];
                }
            }
        }
        named_bar_sync(1, kCons);   // this vector's limbs complete; the scratch may be reused
    }

    const Lane L = make_lane<QT>(lane);
    const int rgid = lane & 7, rj = lane >> 3;
    const float* fs0 = reinterpret_cast<const float*>(xq) + P.fs_off / 4;
    const int NS = P.n_stages;
    int s = 0;
    uint32_t ph = 0;
    bool dead = false;
    int gl = 0;
    for (int gi = g_begin; gi < g_end; ++gi, ++gl) {
        float* rg = red + (gl & 1) * RG;   // [warp][v][mat][16]
#pragma unroll 1
        for (int mat = 0; mat < NM; ++mat) {
            float acc0[NX], acc1[NX];
#pragma unroll
            for (int v = 0; v < NX; ++v) acc0[v] = acc1[v] = 0.f;
            for (int c = 0; c < NCH; ++c) {
                const int n_units = min(CE, K - c * CE) / T::UK;
                if (!dead && !mbar_wait(&full[s], ph, kWaitPolls)) {
                    record_device_error(DEVERR_FULL_WAIT);
                    dead = true;    // keep taking part in every barrier so the CTA still finishes
                }
                const uint8_t* st = stages + (size_t)s * P.stage_bytes;
                if (!dead) {
                    const int u0 = c * CE / 32;   // first step of the chunk
                    if constexpr (CORE == 0) {
                        for (int un = warp; un < n_units; un += kWarps)
                            UnitsN<QT, NX>::run(st + (size_t)un * T::UB, xq + 32 * (u0 + SPU * un), fs0 + u0 + SPU * un,
                                                XW, L, acc0, acc1);
                    } else if constexpr (QT == NTX_Q8_0_T) {
                        for (int un = warp; un < n_units; un += kWarps)
                            RowsN<QT, NX>::run(st + (size_t)un * T::UB, xq + 32 * (u0 + un), XW, L, acc0, acc1);
                    } else if constexpr (QT == NTX_Q4_0_T) {
                        const int sx = 8 * ((u0 + rj) & 3);
                        for (int u4 = 4 * warp; u4 < n_units; u4 += 4 * kWarps) {
                            const int un = u4 + rj;
                            if (un < n_units)
                                RowsN<QT, NX>::run(st + (size_t)un * T::UB, xq + 32 * (u0 + un), fs0 + u0 + un, XW,
                                                   sx, rgid, acc0, acc1);
                        }
                    } else {
                        for (int un = warp; un < n_units; un += kWarps)
                            RowsN<QT, NX>::run(st + (size_t)un * T::UB, xq + 32 * (u0 + SPU * un),
                                               fs0 + u0 + SPU * un, XW, rgid, rj, acc0, acc1);
                    }
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(&empty[s]);
                if (++s == NS) {
                    s = 0;
                    ph ^= 1u;
                }
            }
            // CORE 0: this lane's C columns hold limbs 0, 1 or limb 2
            const float limb_w = (CORE == 0 && (L.tig & 1)) ? 65536.f : 1.f;
#pragma unroll
            for (int v = 0; v < NX; ++v) {
                float a0 = acc0[v], a1 = acc1[v];
                if constexpr (ROWS) {
                    // sum over the 4 threads of each gid: lane g < 8 ends with rows g, g + 8
                    a0 += __shfl_xor_sync(0xffffffffu, a0, 8);
                    a1 += __shfl_xor_sync(0xffffffffu, a1, 8);
                    a0 += __shfl_xor_sync(0xffffffffu, a0, 16);
                    a1 += __shfl_xor_sync(0xffffffffu, a1, 16);
                    if (lane < 8) {
                        rg[((warp * NX + v) * NM + mat) * 16 + lane] = a0;
                        rg[((warp * NX + v) * NM + mat) * 16 + lane + 8] = a1;
                    }
                } else {
                    // quad reduction (with the limb weights of the MMA's C columns): lane tig 0
                    // ends with rows gid, gid + 8
                    a0 *= limb_w;
                    a1 *= limb_w;
                    a0 += __shfl_xor_sync(0xffffffffu, a0, 1);
                    a1 += __shfl_xor_sync(0xffffffffu, a1, 1);
                    a0 += __shfl_xor_sync(0xffffffffu, a0, 2);
                    a1 += __shfl_xor_sync(0xffffffffu, a1, 2);
                    if (L.tig == 0) {
                        rg[((warp * NX + v) * NM + mat) * 16 + L.gid] = a0;
                        rg[((warp * NX + v) * NM + mat) * 16 + L.gid + 8] = a1;
                    }
                }
            }
        }
        named_bar_sync(1, kCons);
        for (int i = tid; i < NX * NM * 16; i += kCons) {
            // the 8 warps' sums in warp order, scaled by 2^-S_v
            const int row = i & 15, mat = (i >> 4) % NM, v = i / (16 * NM);
            float t = 0.f;
#pragma unroll
            for (int w = 0; w < kWarps; ++w) t += rg[((w * NX + v) * NM + mat) * 16 + row];
            sums[((gl * NX + v) * NM + mat) * 16 + row] = gemv::scale2(t, -S_sm[v]);
        }
    }
    named_bar_sync(1, kCons);
    // epilogue of every vector's rows; RoPE partners (2i, 2i + 1) sit in adjacent lanes
    const int n_rows = (g_end - g_begin) * 16;
#pragma unroll 1
    for (int v = 0; v < NX; ++v) {
        const int32_t pos = EPI == gemv::EPI_QKV ? *V.pos_dev[v] : 0;
        for (int base = 0; base < n_rows; base += kCons) {
            const int r = base + tid;
            const bool ok = r < n_rows;
            const int gl2 = ok ? r >> 4 : 0, rr = r & 15;
            const float a = ok ? sums[((gl2 * NX + v) * NM) * 16 + rr] : 0.f;
            const float b = (ok && NM == 2) ? sums[((gl2 * NX + v) * NM + 1) * 16 + rr] : 0.f;
            epilogue_v<EPI>(P, V, v, g_begin * 16 + r, ok, a, b, pos, rope_sm + v * 128);
        }
    }
}

}  // namespace qmma
}  // namespace ntx
