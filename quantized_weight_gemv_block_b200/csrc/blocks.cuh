// blocks.cuh - scalar decoders of one weight of each block format, in the
// GGUF-style layout and in the tiled layout (used by the dequantization,
// embedding, repack and simple GEMV kernels).  Every weight is computed as
// fp32 products of exact factors, so the result is the exactly rounded value of
// the format's formula (one rounding for Q4_K's subtraction, none otherwise).
#pragma once

#include "gemv.cuh"

namespace ntx {
namespace gemv {

__device__ __forceinline__ float ldh(const uint8_t* p) { return f16_bits_to_f32((uint16_t)(p[0] | (p[1] << 8))); }

__device__ __forceinline__ void q4k_sm(const uint8_t* s, int j, int& sc, int& m)
{
    if (j < 4) {
        sc = s[j] & 63;
        m = s[j + 4] & 63;
    } else {
        sc = (s[j + 4] & 15) | ((s[j - 4] >> 6) << 4);
        m = (s[j + 4] >> 4) | ((s[j] >> 6) << 4);
    }
}

// Weight e (0 <= e < cols) of one packed row in a GGUF-style layout QT (or F16 / F32).
template <int QT>
__device__ __forceinline__ float weight_in_row(const uint8_t* row, int64_t e)
{
    static_assert(QT >= NTX_Q8_0 && QT <= NTX_F32, "GGUF-style layouts only");
    if constexpr (QT == NTX_F16) {
        return ldh(row + 2 * e);
    } else if constexpr (QT == NTX_F32) {
        float v;
        memcpy(&v, row + 4 * e, 4);
        return v;
    } else if constexpr (QT == NTX_Q5_K) {
        // fp16 d | fp16 dmin | 12 B scales and mins | 32 B fifth bits | 128 B low nibbles
        const uint8_t* b = row + (e >> 8) * 176;
        const int r256 = (int)(e & 255);
        const float d = ldh(b), dmin = ldh(b + 2);
        const int c = r256 >> 6, r = r256 & 63, l = r & 31, up = r >> 5;
        const int byte = b[48 + 32 * c + l];
        const int q = (up ? (byte >> 4) : (byte & 15)) | (((b[16 + l] >> (2 * c + up)) & 1) << 4);
        int sc, m;
        q4k_sm(b + 4, r256 >> 5, sc, m);
        return __fsub_rn(__fmul_rn(__fmul_rn(d, (float)sc), (float)q), __fmul_rn(dmin, (float)m));
    } else if constexpr (QT == NTX_Q8_0) {
        const uint8_t* blk = row + (e >> 5) * 34;
        return ldh(blk) * (float)(int8_t)blk[2 + (e & 31)];
    } else if constexpr (QT == NTX_Q4_0) {
        const uint8_t* blk = row + (e >> 5) * 18;
        const int i = (int)(e & 31);
        const int byte = blk[2 + (i & 15)];
        const int q = i < 16 ? (byte & 15) : (byte >> 4);
        return ldh(blk) * (float)(q - 8);
    } else if constexpr (QT == NTX_Q4_K) {
        const uint8_t* b = row + (e >> 8) * 144;
        const int r256 = (int)(e & 255);
        const float d = ldh(b), dmin = ldh(b + 2);
        const int c = r256 >> 6, r = r256 & 63;
        const int byte = b[16 + 32 * c + (r & 31)];
        const int q = r < 32 ? (byte & 15) : (byte >> 4);
        int sc, m;
        q4k_sm(b + 4, r256 >> 5, sc, m);
        return __fsub_rn(__fmul_rn(__fmul_rn(d, (float)sc), (float)q), __fmul_rn(dmin, (float)m));
    } else {
        const uint8_t* b = row + (e >> 8) * 210;
        const int r256 = (int)(e & 255);
        const int h = r256 >> 7, t = r256 & 127;
        const int lo = t < 64 ? (b[64 * h + t] & 15) : (b[64 * h + t - 64] >> 4);
        const int hi = (b[128 + 32 * h + (t & 31)] >> (2 * (t >> 5))) & 3;
        const int q = lo | (hi << 4);
        return __fmul_rn(__fmul_rn(ldh(b + 208), (float)(int8_t)b[192 + (r256 >> 4)]), (float)(q - 32));
    }
}

// ------------------------------------------------------------------ tiled layouts
// Rows are taken in groups of 16; a group is a run of units along the row, each
// unit covering columns [u UK, (u + 1) UK) of the group's 16 rows in 16 x the
// GGUF-style bytes of one row's UK columns.  Inside a unit the codes sit in the
// order in which lane L = 4 gid + tig of a warp needs them as the A operand of an
// m16n8k32 integer MMA step (rows gid and gid + 8; columns 4 tig .. 4 tig + 3 and
// 16 + 4 tig .. 16 + 4 tig + 3 of the step), so a lane fetches one step's codes of
// two rows with one shared-memory load:
//  Q8_0 (UK 32, 544 B):  [0, 512) lane L at 16 L: 4 words a0..a3 of int8 codes
//                        (a0 row gid cols 4tig+j, a1 row gid+8 same cols, a2 row gid
//                        cols 16+4tig+j, a3 row gid+8 cols 16+4tig+j; byte j);
//                        [512, 544) word gid = (d[gid], d[gid+8]) fp16.
//  Q4_0 (UK 32, 288 B):  [0, 256) lane L at 8 L: word P (row gid), Q (row gid+8);
//                        byte j holds column 4tig+j in its low nibble and column
//                        16+4tig+j in its high nibble; [256, 288) d pairs as Q8_0.
//  Q6_K (UK 256, 3360 B): 8 steps of 32 columns, step m at 384 m, lane L at 12 L:
//                        words A, B, C hold the 6-bit codes of a0, a1, a2 in the low
//                        6 bits of byte j, and bits 6-7 of byte j of A, B, C hold
//                        bits 0-1, 2-3, 4-5 of the a3 code; [3072, 3328) the int8
//                        scales: 16 bytes per (gid, parity p) at 16 (2 gid + p): byte
//                        m = scale of sub-block 2m + p of row gid, byte 8 + m the same
//                        for row gid + 8; [3328, 3360) d pairs as Q8_0.
//  Q4_K (UK 256, 2304 B): 8 steps (one 32-column sub-block each), step m at 256 m,
//                        lane L at 8 L: words P, Q as Q4_0; [2048, 2240) 24 bytes per
//                        gid at 24 gid: the 6-bit values V(m, b), b = 0 scale of row
//                        gid, 1 scale of row gid+8, 2 min of row gid, 3 min of row
//                        gid+8, as 4 nibble words (word m/2, byte b, low nibble for
//                        even m) then 2 words of their top 2 bits (word m/4, byte b,
//                        bits 2 (m mod 4)); [2240, 2304) 8 bytes per gid: d[gid],
//                        d[gid+8], dmin[gid], dmin[gid+8] fp16.
//  Q5_K (UK 256, 2816 B): 8 steps (one 32-column sub-block each), step m at 320 m:
//                        [0, 256) lane L at 8 L: the low 4 bits of the codes as Q4_K's
//                        words P, Q; [256, 320) 8 bytes per gid at 256 + 8 gid: words
//                        H0 (row gid), H1 (row gid + 8) of fifth bits, the bit of column
//                        4 t + j at bit 8 j + 2 t and that of column 16 + 4 t + j at bit
//                        8 j + 2 t + 1 (t = tig); then [2560, 2752) scales and mins and
//                        [2752, 2816) d, dmin exactly as Q4_K's [2048, 2304).
template <int QT>
struct Tiled;
template <>
struct Tiled<NTX_Q8_0_T> {
    static constexpr int UK = 32, UB = 544;
};
template <>
struct Tiled<NTX_Q4_0_T> {
    static constexpr int UK = 32, UB = 288;
};
template <>
struct Tiled<NTX_Q4_K_T> {
    static constexpr int UK = 256, UB = 2304;
};
template <>
struct Tiled<NTX_Q6_K_T> {
    static constexpr int UK = 256, UB = 3360;
};
template <>
struct Tiled<NTX_Q5_K_T> {
    static constexpr int UK = 256, UB = 2816;
};

// Weight (r, e) of a tiled matrix W whose rows hold rb bytes each.
template <int QT>
__device__ __forceinline__ float weight_tiled(const uint8_t* W, int64_t r, int64_t e, int64_t rb)
{
    using T = Tiled<QT>;
    const uint8_t* U = W + (r >> 4) * 16 * rb + (e / T::UK) * T::UB;
    const int rr = (int)(r & 15), gid = rr & 7, hi = rr >> 3;
    const int c = (int)(e % T::UK), cs = c & 31;
    const int tig = (cs & 15) >> 2, j = cs & 3, kh = cs >> 4;
    const int lane = 4 * gid + tig;
    if constexpr (QT == NTX_Q8_0_T) {
        return ldh(U + 512 + 4 * gid + 2 * hi) * (float)(int8_t)U[16 * lane + 4 * (2 * kh + hi) + j];
    } else if constexpr (QT == NTX_Q4_0_T) {
        const int q = (U[8 * lane + 4 * hi + j] >> (4 * kh)) & 15;
        return ldh(U + 256 + 4 * gid + 2 * hi) * (float)(q - 8);
    } else if constexpr (QT == NTX_Q6_K_T) {
        const int m = c >> 5, reg = 2 * kh + hi;
        const uint8_t* w = U + 384 * m + 12 * lane + j;
        int q;
        if (reg < 3) {
            q = w[4 * reg] & 63;
        } else {
            q = ((w[0] >> 6) & 3) | (((w[4] >> 6) & 3) << 2) | (((w[8] >> 6) & 3) << 4);
        }
        const int sb = c >> 4;
        const int sc = (int8_t)U[3072 + 16 * (2 * gid + (sb & 1)) + 8 * hi + (sb >> 1)];
        return __fmul_rn(__fmul_rn(ldh(U + 3328 + 4 * gid + 2 * hi), (float)sc), (float)(q - 32));
    } else if constexpr (QT == NTX_Q5_K_T) {
        const int m = c >> 5;
        const int lo = (U[320 * m + 8 * lane + 4 * hi + j] >> (4 * kh)) & 15;
        const int b5 = (U[320 * m + 256 + 8 * gid + 4 * hi + j] >> (2 * tig + kh)) & 1;
        const int q = lo | (b5 << 4);
        const uint8_t* v = U + 2560 + 24 * gid;
        auto val = [&](int b) {
            const int lo4 = (v[4 * (m >> 1) + b] >> (4 * (m & 1))) & 15;
            const int hi2 = (v[16 + 4 * (m >> 2) + b] >> (2 * (m & 3))) & 3;
            return lo4 | (hi2 << 4);
        };
        const int sc = val(hi), mn = val(2 + hi);
        const uint8_t* dd = U + 2752 + 8 * gid;
        const float d = ldh(dd + 2 * hi), dmin = ldh(dd + 4 + 2 * hi);
        return __fsub_rn(__fmul_rn(__fmul_rn(d, (float)sc), (float)q), __fmul_rn(dmin, (float)mn));
    } else {
        const int m = c >> 5;
        const int q = (U[256 * m + 8 * lane + 4 * hi + j] >> (4 * kh)) & 15;
        const uint8_t* v = U + 2048 + 24 * gid;
        auto val = [&](int b) {
            const int lo4 = (v[4 * (m >> 1) + b] >> (4 * (m & 1))) & 15;
            const int hi2 = (v[16 + 4 * (m >> 2) + b] >> (2 * (m & 3))) & 3;
            return lo4 | (hi2 << 4);
        };
        const int sc = val(hi), mn = val(2 + hi);
        const uint8_t* dd = U + 2240 + 8 * gid;
        const float d = ldh(dd + 2 * hi), dmin = ldh(dd + 4 + 2 * hi);
        return __fsub_rn(__fmul_rn(__fmul_rn(d, (float)sc), (float)q), __fmul_rn(dmin, (float)mn));
    }
}

// Weight (r, e) of a matrix in any layout.
template <int QT>
__device__ __forceinline__ float weight_at(const uint8_t* W, int64_t r, int64_t e, int64_t rb)
{
    if constexpr ((QT & NTX_TILED) != 0)
        return weight_tiled<QT>(W, r, e, rb);
    else
        return weight_in_row<QT>(W + r * rb, e);
}

}  // namespace gemv
}  // namespace ntx
