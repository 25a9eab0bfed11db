// common.cuh - shared pieces of the ntx library: status handling, format traits,
// sm_100a PTX wrappers (mbarrier, bulk copy, paired fp32 math).
#pragma once

#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <string>

#include "ntx.h"

#define NTX_EXPORT extern "C" __attribute__((visibility("default")))

namespace ntx {

// ------------------------------------------------------------------ status

void set_error(const std::string& msg);
ntx_status fail(ntx_status code, const std::string& msg);
ntx_status check_launch(const char* what);
ntx_status ok();

#define NTX_CUDA_TRY(call)                                                                  \
    do {                                                                                    \
        cudaError_t e_ = (call);                                                            \
        if (e_ != cudaSuccess)                                                              \
            return ::ntx::fail(NTX_ECUDA, std::string(#call) + ": " + cudaGetErrorString(e_)); \
    } while (0)

// Codes a kernel records when a bounded wait gives up.
enum : uint32_t {
    DEVERR_FULL_WAIT = 1u,     // consumer waited too long for a stage to fill
    DEVERR_EMPTY_WAIT = 2u,    // producer waited too long for a stage to drain
    DEVERR_DRAIN_WAIT = 4u,    // producer gave up draining its copies on exit
    DEVERR_SMEM_ALIGN = 8u,    // shared memory not aligned as the copies need; nothing was done
};

// One flag per translation unit; ntx_device_error() collects them all.
static __device__ uint32_t g_dev_error;

__device__ __forceinline__ void record_device_error(uint32_t code) { atomicOr(&g_dev_error, code); }

// Host: read and clear this translation unit's flag.
static inline cudaError_t take_tu_device_error(uint32_t* out)
{
    uint32_t zero = 0;
    cudaError_t e = cudaMemcpyFromSymbol(out, g_dev_error, sizeof(uint32_t));
    if (e != cudaSuccess) return e;
    return cudaMemcpyToSymbol(g_dev_error, &zero, sizeof(uint32_t));
}

// Per-file collectors (each kernel file defines one).
cudaError_t take_device_error_gemv(uint32_t* out);
cudaError_t take_device_error_attn(uint32_t* out);
cudaError_t take_device_error_decode(uint32_t* out);
cudaError_t take_device_error_qmma(uint32_t* out);
cudaError_t take_device_error_probe(uint32_t* out);
cudaError_t take_device_error_fgemv(uint32_t* out);
cudaError_t take_device_error_qmma_multi(uint32_t* out);

int num_sms();

// Raise the dynamic shared-memory limit of kernel `func` to `bytes` on the current
// device, once per (device, kernel, size); thread-safe.  NTX_ECUDA if the driver refuses.
ntx_status ensure_smem_limit(const void* func, int bytes);

// ------------------------------------------------------------------ formats

struct QTraits {
    int block_elems;
    int block_bytes;
};

inline bool is_tiled(int qtype) { return (qtype & NTX_TILED) != 0; }
inline int base_qtype(int qtype) { return qtype & ~NTX_TILED; }

// Columns per unit of a tiled layout (one block, or one superblock).
inline int tile_elems(int qtype)
{
    switch (base_qtype(qtype)) {
    case NTX_Q8_0: case NTX_Q4_0: return 32;
    case NTX_Q4_K: case NTX_Q6_K: case NTX_Q5_K: return 256;
    default: return 0;
    }
}

// F16 / F32: unquantized weights (no blocks, no tiled form).
inline bool is_float_format(int qtype) { return qtype == NTX_F16 || qtype == NTX_F32; }

inline QTraits qtraits(int qtype)
{
    if (is_tiled(qtype)) {
        const int b = base_qtype(qtype);
        if (b < NTX_Q8_0 || b > NTX_Q5_K) return {0, 0};
        qtype = b;
    }
    switch (qtype) {
    case NTX_Q8_0: return {32, 34};
    case NTX_Q4_0: return {32, 18};
    case NTX_Q4_K: return {256, 144};
    case NTX_Q6_K: return {256, 210};
    case NTX_Q5_K: return {256, 176};
    case NTX_F16: return {1, 2};
    case NTX_F32: return {1, 4};
    default: return {0, 0};
    }
}

inline int64_t row_bytes(int qtype, int64_t cols)
{
    QTraits t = qtraits(qtype);
    if (t.block_elems == 0 || cols <= 0 || cols % t.block_elems) return 0;
    if (is_tiled(qtype) && cols % tile_elems(qtype)) return 0;
    return cols / t.block_elems * t.block_bytes;
}

inline bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// ------------------------------------------------------------------ PTX wrappers

__device__ __forceinline__ uint32_t smem_addr(const void* p)
{
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count)
{
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_mbar_init()
{
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes)
{
    asm volatile("mbarrier.arrive.expect_tx.release.cta.shared::cta.b64 _, [%0], %1;" ::"r"(smem_addr(bar)),
                 "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar)
{
    asm volatile("mbarrier.arrive.release.cta.shared::cta.b64 _, [%0];" ::"r"(smem_addr(bar)) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity)
{
    uint32_t done;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.acquire.cta.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(done)
        : "r"(smem_addr(bar)), "r"(parity)
        : "memory");
    return done != 0;
}

// Bounded wait: false if the phase did not complete within `limit` polls.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, uint32_t limit = (1u << 24))
{
    for (uint32_t i = 0; i < limit; ++i)
        if (mbar_try_wait(bar, parity)) return true;
    return false;
}

__device__ __forceinline__ uint64_t policy_evict_first()
{
    uint64_t p;
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
    return p;
}

// For data many CTAs read (an input vector): keep it in L2.
__device__ __forceinline__ uint64_t policy_evict_last()
{
    uint64_t p;
    asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(p));
    return p;
}

// 1-D bulk copy global -> this CTA's shared memory, completion counted on `bar`.
// dst, src 16-byte aligned; bytes a multiple of 16.
__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, uint32_t bytes, uint64_t* bar,
                                         uint64_t policy)
{
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint [%0], [%1], %2, [%3], "
        "%4;" ::"r"(smem_addr(dst)),
        "l"(src), "r"(bytes), "r"(smem_addr(bar)), "l"(policy)
        : "memory");
}

__device__ __forceinline__ void named_bar_sync(int id, int threads)
{
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(threads) : "memory");
}

// Programmatic dependent launch: allow the next kernel of the stream to launch,
// and wait for the previous kernel's results.
__device__ __forceinline__ void pdl_launch_dependents()
{
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

__device__ __forceinline__ void pdl_wait()
{
    asm volatile("griddepcontrol.wait;" ::: "memory");
}

// Paired fp32 arithmetic of sm_100 (two lanes per instruction).
struct f2 {
    float x, y;
};

__device__ __forceinline__ uint64_t f2_bits(f2 v)
{
    return (uint64_t)__float_as_uint(v.x) | ((uint64_t)__float_as_uint(v.y) << 32);
}

__device__ __forceinline__ f2 f2_from(uint64_t b)
{
    return {__uint_as_float((uint32_t)b), __uint_as_float((uint32_t)(b >> 32))};
}

// acc += a * b, lane-wise, round to nearest, subnormals kept.
__device__ __forceinline__ void fma2(uint64_t& acc, uint64_t a, uint64_t b)
{
    asm("fma.rn.f32x2 %0, %1, %2, %0;" : "+l"(acc) : "l"(a), "l"(b));
}

// Two 32-bit values as one register pair (no arithmetic).
__device__ __forceinline__ uint64_t pack2(uint32_t lo, uint32_t hi)
{
    uint64_t r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "r"(lo), "r"(hi));
    return r;
}

// a * b, lane-wise.
__device__ __forceinline__ uint64_t mul2(uint64_t a, uint64_t b)
{
    uint64_t r;
    asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
    return r;
}

// a + b, lane-wise.
__device__ __forceinline__ uint64_t add2(uint64_t a, uint64_t b)
{
    uint64_t r;
    asm("add.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
    return r;
}

__device__ __forceinline__ float f16_bits_to_f32(uint16_t h) { return __half2float(__ushort_as_half(h)); }

}  // namespace ntx
