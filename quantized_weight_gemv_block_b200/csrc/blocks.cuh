// blocks.cuh - scalar decoders of one weight of each block format (used by the
// dequantization, embedding and simple GEMV kernels).  Every weight is computed
// as fp32 products of exact factors, so the result is the exactly rounded value
// of the format's formula (one rounding for Q4_K's subtraction, none otherwise).
#pragma once

#include "gemv.cuh"

namespace ntx {
namespace gemv {

__device__ __forceinline__ float ldh(const uint8_t* p) { return f16_bits_to_f32((uint16_t)(p[0] | (p[1] << 8))); }

template <int QT>
__device__ __forceinline__ float weight_at(const uint8_t* b, int e);

template <>
__device__ __forceinline__ float weight_at<NTX_Q8_0>(const uint8_t* b, int e)
{
    return ldh(b) * (float)(int8_t)b[2 + e];
}

template <>
__device__ __forceinline__ float weight_at<NTX_Q4_0>(const uint8_t* b, int e)
{
    const int byte = b[2 + (e & 15)];
    const int q = e < 16 ? (byte & 15) : (byte >> 4);
    return ldh(b) * (float)(q - 8);
}

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

template <>
__device__ __forceinline__ float weight_at<NTX_Q4_K>(const uint8_t* b, int e)
{
    const float d = ldh(b), dmin = ldh(b + 2);
    const int c = e >> 6, r = e & 63;
    const int byte = b[16 + 32 * c + (r & 31)];
    const int q = r < 32 ? (byte & 15) : (byte >> 4);
    int sc, m;
    q4k_sm(b + 4, e >> 5, sc, m);
    return __fsub_rn(__fmul_rn(__fmul_rn(d, (float)sc), (float)q), __fmul_rn(dmin, (float)m));
}

template <>
__device__ __forceinline__ float weight_at<NTX_Q6_K>(const uint8_t* b, int e)
{
    const int h = e >> 7, t = e & 127;
    const int lo = t < 64 ? (b[64 * h + t] & 15) : (b[64 * h + t - 64] >> 4);
    const int hi = (b[128 + 32 * h + (t & 31)] >> (2 * (t >> 5))) & 3;
    const int q = lo | (hi << 4);
    const float d = ldh(b + 208);
    return __fmul_rn(__fmul_rn(d, (float)(int8_t)b[192 + (e >> 4)]), (float)(q - 32));
}

}  // namespace gemv
}  // namespace ntx
