// blocks.cuh - scalar decoders of one weight of each block format, in the
// GGUF-style layout and in the tiled layout (used by the dequantization,
// embedding, repack-check and simple GEMV kernels).  Every weight is computed as
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

// Weight e (0 <= e < cols) of one packed row in layout QT (GGUF-style 0..3, tiled 16..19).
template <int QT>
__device__ __forceinline__ float weight_in_row(const uint8_t* row, int64_t e)
{
    constexpr int B = QT & 3;
    constexpr bool T = (QT & NTX_TILED) != 0;
    if constexpr (B == NTX_Q8_0) {
        const int64_t b = e >> 5;
        const int i = (int)(e & 31);
        float d;
        int q;
        if constexpr (T) {
            const uint8_t* tile = row + (b >> 3) * 272;
            d = ldh(tile + 256 + 2 * (b & 7));
            q = (int8_t)tile[(e & 255)];
        } else {
            const uint8_t* blk = row + b * 34;
            d = ldh(blk);
            q = (int8_t)blk[2 + i];
        }
        return d * (float)q;
    } else if constexpr (B == NTX_Q4_0) {
        const int64_t b = e >> 5;
        const int i = (int)(e & 31);
        const uint8_t* codes;
        float d;
        if constexpr (T) {
            const uint8_t* tile = row + (b >> 3) * 144;
            codes = tile + 16 * (b & 7);
            d = ldh(tile + 128 + 2 * (b & 7));
        } else {
            codes = row + b * 18 + 2;
            d = ldh(row + b * 18);
        }
        const int byte = codes[i & 15];
        const int q = i < 16 ? (byte & 15) : (byte >> 4);
        return d * (float)(q - 8);
    } else if constexpr (B == NTX_Q4_K) {
        const uint8_t* b = row + (e >> 8) * 144;          // identical in both layouts
        const int r256 = (int)(e & 255);
        const float d = ldh(b), dmin = ldh(b + 2);
        const int c = r256 >> 6, r = r256 & 63;
        const int byte = b[16 + 32 * c + (r & 31)];
        const int q = r < 32 ? (byte & 15) : (byte >> 4);
        int sc, m;
        q4k_sm(b + 4, r256 >> 5, sc, m);
        return __fsub_rn(__fmul_rn(__fmul_rn(d, (float)sc), (float)q), __fmul_rn(dmin, (float)m));
    } else {
        const int64_t sb = e >> 8;
        const int r256 = (int)(e & 255);
        const uint8_t *ql, *qh, *sc, *dp;
        if constexpr (T) {
            const uint8_t* tile = row + (sb >> 3) * 1680;
            const int s = (int)(sb & 7);
            ql = tile + 128 * s;
            qh = tile + 1024 + 64 * s;
            sc = tile + 1536 + 16 * s;
            dp = tile + 1664 + 2 * s;
        } else {
            const uint8_t* b = row + sb * 210;
            ql = b;
            qh = b + 128;
            sc = b + 192;
            dp = b + 208;
        }
        const int h = r256 >> 7, t = r256 & 127;
        const int lo = t < 64 ? (ql[64 * h + t] & 15) : (ql[64 * h + t - 64] >> 4);
        const int hi = (qh[32 * h + (t & 31)] >> (2 * (t >> 5))) & 3;
        const int q = lo | (hi << 4);
        return __fmul_rn(__fmul_rn(ldh(dp), (float)(int8_t)sc[r256 >> 4]), (float)(q - 32));
    }
}

}  // namespace gemv
}  // namespace ntx
