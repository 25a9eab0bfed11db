// synth_dev.cu - device side of the seeded input generator: fills device buffers
// with the same bytes the host generator produces (same header, integer math).
#include <cuda_runtime.h>

#include "synth.h"

#define SYN_EXPORT extern "C" __attribute__((visibility("default")))

namespace {

__global__ void fill_blocks_kernel(int qtype, uint64_t key, int64_t block0, int64_t nblocks, syn_qparams P,
                                   uint8_t* out)
{
    const int bb = syn_block_bytes(qtype);
    for (int64_t b = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; b < nblocks;
         b += (int64_t)gridDim.x * blockDim.x) {
        uint8_t tmp[210];
        syn_fill_block(qtype, key, (uint64_t)(block0 + b), &P, tmp);
        uint8_t* dst = out + b * bb;
        for (int i = 0; i < bb; ++i) dst[i] = tmp[i];
    }
}

__global__ void fill_normal_f32_kernel(uint64_t key, int64_t i0, int64_t n, float* out)
{
    for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x)
        out[i] = syn_normal_f32(key, (uint64_t)(i0 + i));
}

__global__ void fill_normal_f16_kernel(uint64_t key, int64_t i0, int64_t n, uint16_t* out)
{
    for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x)
        out[i] = syn_normal_f16(key, (uint64_t)(i0 + i));
}

__global__ void fill_uniform_f32_kernel(uint64_t key, int64_t i0, int64_t n, uint64_t k_lo, uint64_t k_hi, int e,
                                        float* out)
{
    for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x)
        out[i] = syn_uniform_f32(key, (uint64_t)(i0 + i), k_lo, k_hi, e);
}

int grid_for(int64_t n)
{
    int64_t g = (n + 255) / 256;
    return (int)(g < 148 * 64 ? (g < 1 ? 1 : g) : 148 * 64);
}

}  // namespace

SYN_EXPORT int syn_fill_blocks_dev(int qtype, uint64_t seed, uint64_t id, int64_t block0, int64_t nblocks,
                                   const syn_qparams* P, void* out, void* stream)
{
    if (nblocks <= 0) return 0;
    fill_blocks_kernel<<<grid_for(nblocks), 256, 0, (cudaStream_t)stream>>>(qtype, syn_key(seed, id), block0,
                                                                           nblocks, *P, (uint8_t*)out);
    return (int)cudaGetLastError();
}

SYN_EXPORT int syn_fill_normal_f32_dev(uint64_t seed, uint64_t id, int64_t i0, int64_t n, void* out, void* stream)
{
    if (n <= 0) return 0;
    fill_normal_f32_kernel<<<grid_for(n), 256, 0, (cudaStream_t)stream>>>(syn_key(seed, id), i0, n, (float*)out);
    return (int)cudaGetLastError();
}

SYN_EXPORT int syn_fill_normal_f16_dev(uint64_t seed, uint64_t id, int64_t i0, int64_t n, void* out, void* stream)
{
    if (n <= 0) return 0;
    fill_normal_f16_kernel<<<grid_for(n), 256, 0, (cudaStream_t)stream>>>(syn_key(seed, id), i0, n,
                                                                          (uint16_t*)out);
    return (int)cudaGetLastError();
}

SYN_EXPORT int syn_fill_uniform_f32_dev(uint64_t seed, uint64_t id, int64_t i0, int64_t n, uint64_t k_lo,
                                        uint64_t k_hi, int e, void* out, void* stream)
{
    if (n <= 0) return 0;
    fill_uniform_f32_kernel<<<grid_for(n), 256, 0, (cudaStream_t)stream>>>(syn_key(seed, id), i0, n, k_lo, k_hi,
                                                                          e, (float*)out);
    return (int)cudaGetLastError();
}
