/*
 * synth.h - seeded, counter-based synthetic inputs for the quantized decode path.
 *
 * This header is input infrastructure shared by the CPU oracle (compiled by gcc)
 * and by the device-side fill kernels (compiled by nvcc).  It holds none of the
 * decode arithmetic: it only produces bytes (packed quant blocks, fp16 / fp32
 * values) from (seed, tensor id, index).  Every routine is integer arithmetic, so
 * the host and the device produce identical bytes.
 *
 * Generator: SplitMix64 (Sebastiano Vigna, public domain), used counter-style.
 * The n-th output of a SplitMix64 stream whose state starts at `key` is
 * mix64(key + (n + 1) * GAMMA), so any element can be produced on its own.
 *
 * Block layouts written here (byte offsets inside one block, little-endian):
 *   Q8_0 (34 B / 32 weights):  [0,2) fp16 d | [2,34) int8 codes
 *   Q4_0 (18 B / 32 weights):  [0,2) fp16 d | [2,18) 16 bytes of 4-bit codes
 *   Q4_K (144 B / 256 weights): [0,2) fp16 d | [2,4) fp16 dmin | [4,16) packed 6-bit
 *                               scales and mins | [16,144) 4-bit codes
 *   Q6_K (210 B / 256 weights): [0,128) low 4 code bits | [128,192) high 2 code bits
 *                               | [192,208) int8 sub-block scales | [208,210) fp16 d
 *   Q5_K (176 B / 256 weights): [0,2) fp16 d | [2,4) fp16 dmin | [4,16) packed 6-bit
 *                               scales and mins (as Q4_K) | [16,48) fifth code bits |
 *                               [48,176) low 4 code bits
 * Codes are random bytes; only the scale fields are shaped (see syn_fill_block).
 */
#ifndef SYNTH_H
#define SYNTH_H

#include <stdint.h>
#include <string.h>

#ifdef __CUDACC__
#define SYN_HD __host__ __device__ __forceinline__
#else
#define SYN_HD static inline
#endif

/* Format numbering used by the generator (declared here on its own). */
#define SYN_Q8_0 0
#define SYN_Q4_0 1
#define SYN_Q4_K 2
#define SYN_Q6_K 3
#define SYN_Q5_K 4
#define SYN_F16 5
#define SYN_F32 6

/* Scale-field distribution of one tensor.
 *   d = fp16(k * 2^d_exp) with k uniform in [d_lo, d_hi]
 *   mode 0: the sweep distribution: Q4_K 6-bit scales/mins uniform in 0..63 and
 *           dmin drawn like d; Q6_K sub-scales uniform in -127..127.
 *   mode 1: the decode distribution: Q4_K scales uniform in 1..8, mins =
 *           round(7.5 * scale) (so weights are centred), dmin = d; Q5_K scales
 *           uniform in 1..4, mins = round(15.5 * scale); Q6_K sub-scales uniform in
 *           1..16.  (Q5_K uses the sweep rule of Q4_K in mode 0.)
 * Q8_0 codes are uniform in -127..127 and Q4_0 / Q4_K / Q6_K codes are uniform
 * over their full range in both modes. */
typedef struct syn_qparams {
    uint64_t d_lo;
    uint64_t d_hi;
    int32_t d_exp;
    int32_t mode;
} syn_qparams;

#define SYN_GAMMA 0x9E3779B97F4A7C15ull

SYN_HD uint64_t syn_mix64(uint64_t z)
{
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
    return z ^ (z >> 31);
}

/* n-th output of the SplitMix64 stream with starting state `key`. */
SYN_HD uint64_t syn_draw(uint64_t key, uint64_t n)
{
    return syn_mix64(key + (n + 1ull) * SYN_GAMMA);
}

/* Stream key of tensor `id` under `seed`. */
SYN_HD uint64_t syn_key(uint64_t seed, uint64_t id)
{
    return syn_mix64(syn_draw(seed, id) ^ 0x6A09E667F3BCC909ull);
}

/* Integer in [lo, hi] (hi - lo < 2^32) from 32 random bits (multiply-shift). */
SYN_HD int64_t syn_uniform_int(uint32_t r, int64_t lo, int64_t hi)
{
    uint64_t span = (uint64_t)(hi - lo) + 1ull;
    return lo + (int64_t)(((uint64_t)r * span) >> 32);
}

SYN_HD int syn_clz64(uint64_t x)
{
#ifdef __CUDA_ARCH__
    return __clzll((long long)x);
#else
    return __builtin_clzll(x);
#endif
}

/* IEEE binary16 bits of k * 2^e (k >= 0, k < 2^63), round to nearest even. */
SYN_HD uint16_t syn_f16_from_scaled(uint64_t k, int e)
{
    if (k == 0) return 0;
    int p = 63 - syn_clz64(k);     /* index of the leading one */
    int E = p + e;                  /* unbiased exponent of the value */
    if (E > 15) return 0x7C00;
    int normal = E >= -14;
    int sh = normal ? p - 10 : -(e + 24);
    uint64_t q;
    if (sh <= 0) {
        q = k << (-sh);
    } else if (sh >= 64) {
        q = 0;
    } else {
        q = k >> sh;
        uint64_t rem = k & ((1ull << sh) - 1ull);
        uint64_t half = 1ull << (sh - 1);
        if (rem > half || (rem == half && (q & 1ull))) q++;
    }
    if (normal) {
        if (q == 2048) { q = 1024; E++; if (E > 15) return 0x7C00; }
        return (uint16_t)(((uint32_t)(E + 15) << 10) | (uint32_t)(q & 0x3FFu));
    }
    return (uint16_t)q;     /* q == 1024 is the smallest normal, as the bits say */
}

SYN_HD void syn_put_u16(uint8_t* p, uint16_t v)
{
    p[0] = (uint8_t)(v & 0xFF);
    p[1] = (uint8_t)(v >> 8);
}

SYN_HD void syn_put_u64(uint8_t* p, uint64_t v)
{
    for (int i = 0; i < 8; ++i) p[i] = (uint8_t)(v >> (8 * i));
}

SYN_HD uint16_t syn_scale_bits(uint32_t r, const syn_qparams* P)
{
    return syn_f16_from_scaled((uint64_t)syn_uniform_int(r, (int64_t)P->d_lo, (int64_t)P->d_hi), P->d_exp);
}

SYN_HD int syn_block_bytes(int qtype)
{
    return qtype == SYN_Q8_0 ? 34 : qtype == SYN_Q4_0 ? 18 : qtype == SYN_Q4_K ? 144 : qtype == SYN_Q6_K ? 210
         : qtype == SYN_Q5_K ? 176 : qtype == SYN_F16 ? 2 : qtype == SYN_F32 ? 4 : 0;
}

SYN_HD int syn_block_elems(int qtype)
{
    return (qtype == SYN_Q8_0 || qtype == SYN_Q4_0) ? 32
         : (qtype == SYN_Q4_K || qtype == SYN_Q6_K || qtype == SYN_Q5_K) ? 256
         : (qtype == SYN_F16 || qtype == SYN_F32) ? 1 : 0;
}

/* Draws consumed per block (block b uses draws [b*D, b*D + D)). */
SYN_HD uint64_t syn_block_draws(int qtype)
{
    return qtype == SYN_Q8_0 ? 17 : qtype == SYN_Q4_0 ? 3 : qtype == SYN_Q4_K ? 19 : qtype == SYN_Q5_K ? 23
         : (qtype == SYN_F16 || qtype == SYN_F32) ? 3 : 33;
}

/* 6-bit scale / min packing of the K-quants: sub-blocks 0..3 whole in bytes 0..3 (scale)
 * and 4..7 (min); sub-blocks 4..7 keep their low 4 bits in bytes 8..11 (scale low nibble,
 * min high nibble) and their top 2 bits in the top bits of bytes 0..3 (scale) and 4..7
 * (min). */
SYN_HD void syn_pack_k_scales(const uint8_t* s6, const uint8_t* m6, uint8_t* sc)
{
    for (int j = 0; j < 4; ++j) {
        sc[j] = (uint8_t)(s6[j] | ((s6[j + 4] >> 4) << 6));
        sc[j + 4] = (uint8_t)(m6[j] | ((m6[j + 4] >> 4) << 6));
        sc[j + 8] = (uint8_t)((s6[j + 4] & 0xF) | ((m6[j + 4] & 0xF) << 4));
    }
}

/* Irwin-Hall(12) stand-in for N(0,1): sum of twelve 16-bit uniforms
 * U = (u + 1/2) / 65536, minus 6.  Returns the numerator n of n * 2^-16. */
SYN_HD int32_t syn_ih12(uint64_t key, uint64_t i)
{
    int32_t s = 0;
    for (int j = 0; j < 3; ++j) {
        uint64_t r = syn_draw(key, 3 * i + j);
        s += (int32_t)(r & 0xFFFF) + (int32_t)((r >> 16) & 0xFFFF) + (int32_t)((r >> 32) & 0xFFFF) + (int32_t)(r >> 48);
    }
    return s - 393210;
}

/* Write block number `b` of the tensor with stream key `key` to out[0 .. block_bytes).
 * F16 / F32 "blocks" are one weight: an Irwin-Hall(12) value times 2^d_exp (a power of
 * two, no other rounding than fp16's). */
SYN_HD void syn_fill_block(int qtype, uint64_t key, uint64_t b, const syn_qparams* P, uint8_t* out)
{
    uint64_t n0 = b * syn_block_draws(qtype);
    if (qtype == SYN_F16 || qtype == SYN_F32) {
        const int32_t n = syn_ih12(key, b);
        if (qtype == SYN_F16) {
            const uint64_t a = (uint64_t)(n < 0 ? -n : n);
            syn_put_u16(out, (uint16_t)((n < 0 ? 0x8000 : 0) | syn_f16_from_scaled(a, P->d_exp - 16)));
        } else {
            float v = (float)n;
            int e = P->d_exp - 16;
            while (e < 0) { v *= 0.5f; ++e; }
            while (e > 0) { v *= 2.0f; --e; }
            uint32_t u;
            memcpy(&u, &v, 4);
            for (int i = 0; i < 4; ++i) out[i] = (uint8_t)(u >> (8 * i));
        }
        return;
    }
    if (qtype == SYN_Q8_0) {
        syn_put_u16(out, syn_scale_bits((uint32_t)syn_draw(key, n0), P));
        for (int i = 0; i < 16; ++i) {
            uint64_t r = syn_draw(key, n0 + 1 + i);
            out[2 + 2 * i] = (uint8_t)(int8_t)syn_uniform_int((uint32_t)r, -127, 127);
            out[3 + 2 * i] = (uint8_t)(int8_t)syn_uniform_int((uint32_t)(r >> 32), -127, 127);
        }
    } else if (qtype == SYN_Q4_0) {
        syn_put_u16(out, syn_scale_bits((uint32_t)syn_draw(key, n0), P));
        syn_put_u64(out + 2, syn_draw(key, n0 + 1));
        syn_put_u64(out + 10, syn_draw(key, n0 + 2));
    } else if (qtype == SYN_Q4_K) {
        uint64_t r0 = syn_draw(key, n0);
        uint16_t d = syn_scale_bits((uint32_t)r0, P);
        syn_put_u16(out, d);
        uint8_t* sc = out + 4;
        if (P->mode == 0) {
            syn_put_u16(out + 2, syn_scale_bits((uint32_t)(r0 >> 32), P));
            uint64_t r1 = syn_draw(key, n0 + 1), r2 = syn_draw(key, n0 + 2);
            for (int i = 0; i < 8; ++i) sc[i] = (uint8_t)(r1 >> (8 * i));
            for (int i = 0; i < 4; ++i) sc[8 + i] = (uint8_t)(r2 >> (8 * i));
        } else {
            syn_put_u16(out + 2, d);
            uint64_t r1 = syn_draw(key, n0 + 1);
            uint8_t s6[8], m6[8];
            for (int j = 0; j < 8; ++j) {
                s6[j] = (uint8_t)(1 + ((r1 >> (3 * j)) & 7));
                m6[j] = (uint8_t)((15 * s6[j] + 1) / 2);
            }
            syn_pack_k_scales(s6, m6, sc);
        }
        for (int i = 0; i < 16; ++i) syn_put_u64(out + 16 + 8 * i, syn_draw(key, n0 + 3 + i));
    } else if (qtype == SYN_Q5_K) {
        uint64_t r0 = syn_draw(key, n0);
        uint16_t d = syn_scale_bits((uint32_t)r0, P);
        syn_put_u16(out, d);
        uint8_t* sc = out + 4;
        if (P->mode == 0) {
            syn_put_u16(out + 2, syn_scale_bits((uint32_t)(r0 >> 32), P));
            uint64_t r1 = syn_draw(key, n0 + 1), r2 = syn_draw(key, n0 + 2);
            for (int i = 0; i < 8; ++i) sc[i] = (uint8_t)(r1 >> (8 * i));
            for (int i = 0; i < 4; ++i) sc[8 + i] = (uint8_t)(r2 >> (8 * i));
        } else {
            syn_put_u16(out + 2, d);
            uint64_t r1 = syn_draw(key, n0 + 1);
            uint8_t s6[8], m6[8];
            for (int j = 0; j < 8; ++j) {
                s6[j] = (uint8_t)(1 + ((r1 >> (2 * j)) & 3));
                m6[j] = (uint8_t)((31 * s6[j] + 1) / 2);
            }
            syn_pack_k_scales(s6, m6, sc);
        }
        for (int i = 0; i < 4; ++i) syn_put_u64(out + 16 + 8 * i, syn_draw(key, n0 + 3 + i));
        for (int i = 0; i < 16; ++i) syn_put_u64(out + 48 + 8 * i, syn_draw(key, n0 + 7 + i));
    } else if (qtype == SYN_Q6_K) {
        for (int i = 0; i < 24; ++i) syn_put_u64(out + 8 * i, syn_draw(key, n0 + 1 + i));
        int8_t* sc = (int8_t*)(out + 192);
        if (P->mode == 0) {
            for (int i = 0; i < 8; ++i) {
                uint64_t r = syn_draw(key, n0 + 25 + i);
                sc[2 * i] = (int8_t)syn_uniform_int((uint32_t)r, -127, 127);
                sc[2 * i + 1] = (int8_t)syn_uniform_int((uint32_t)(r >> 32), -127, 127);
            }
        } else {
            uint64_t r = syn_draw(key, n0 + 25);
            for (int i = 0; i < 16; ++i) sc[i] = (int8_t)(1 + ((r >> (4 * i)) & 15));
        }
        syn_put_u16(out + 208, syn_scale_bits((uint32_t)syn_draw(key, n0), P));
    }
}

SYN_HD float syn_normal_f32(uint64_t key, uint64_t i)
{
    return (float)syn_ih12(key, i) * (1.0f / 65536.0f);
}

SYN_HD uint16_t syn_normal_f16(uint64_t key, uint64_t i)
{
    int32_t n = syn_ih12(key, i);
    uint16_t sign = n < 0 ? 0x8000 : 0;
    uint64_t a = (uint64_t)(n < 0 ? -n : n);
    return (uint16_t)(sign | syn_f16_from_scaled(a, -16));
}

/* k * 2^e with k uniform in [k_lo, k_hi]; exact in fp32 while k < 2^24. */
SYN_HD float syn_uniform_f32(uint64_t key, uint64_t i, uint64_t k_lo, uint64_t k_hi, int e)
{
    int64_t k = syn_uniform_int((uint32_t)syn_draw(key, i), (int64_t)k_lo, (int64_t)k_hi);
    float v = (float)k;
    /* scale by 2^e one power at a time keeps every step exact */
    while (e < 0) { v *= 0.5f; ++e; }
    while (e > 0) { v *= 2.0f; --e; }
    return v;
}

#endif /* SYNTH_H */
