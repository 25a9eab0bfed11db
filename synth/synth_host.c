/*
 * synth_host.c - host (CPU) side of the seeded input generator.
 * Fills host buffers from (seed, tensor id, index); see synth.h.
 */
#include "synth.h"

#include <stddef.h>

#define SYN_EXPORT __attribute__((visibility("default")))

SYN_EXPORT void syn_fill_blocks(int qtype, uint64_t seed, uint64_t id, int64_t block0, int64_t nblocks,
                                const syn_qparams* P, uint8_t* out)
{
    uint64_t key = syn_key(seed, id);
    int bb = syn_block_bytes(qtype);
    #pragma omp parallel for schedule(static)
    for (int64_t b = 0; b < nblocks; ++b)
        syn_fill_block(qtype, key, (uint64_t)(block0 + b), P, out + (size_t)b * (size_t)bb);
}

SYN_EXPORT void syn_fill_normal_f32(uint64_t seed, uint64_t id, int64_t i0, int64_t n, float* out)
{
    uint64_t key = syn_key(seed, id);
    #pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; ++i) out[i] = syn_normal_f32(key, (uint64_t)(i0 + i));
}

SYN_EXPORT void syn_fill_normal_f16(uint64_t seed, uint64_t id, int64_t i0, int64_t n, uint16_t* out)
{
    uint64_t key = syn_key(seed, id);
    #pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; ++i) out[i] = syn_normal_f16(key, (uint64_t)(i0 + i));
}

SYN_EXPORT void syn_fill_uniform_f32(uint64_t seed, uint64_t id, int64_t i0, int64_t n, uint64_t k_lo,
                                     uint64_t k_hi, int e, float* out)
{
    uint64_t key = syn_key(seed, id);
    #pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; ++i) out[i] = syn_uniform_f32(key, (uint64_t)(i0 + i), k_lo, k_hi, e);
}

SYN_EXPORT uint64_t syn_uniform_index(uint64_t seed, uint64_t id, uint64_t n_range)
{
    uint64_t key = syn_key(seed, id);
    return (uint64_t)syn_uniform_int((uint32_t)syn_draw(key, 0), 0, (int64_t)n_range - 1);
}

SYN_EXPORT uint16_t syn_f16_bits_of_scaled(uint64_t k, int e) { return syn_f16_from_scaled(k, e); }

SYN_EXPORT int syn_block_bytes_of(int qtype) { return syn_block_bytes(qtype); }
SYN_EXPORT int syn_block_elems_of(int qtype) { return syn_block_elems(qtype); }
