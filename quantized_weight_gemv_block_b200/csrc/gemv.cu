// gemv.cu - host side of the quantized GEMV (launch shaping, C ABI; the tiled
// layouts go to the integer-dot kernel of qmma.cu), the simple kernel for rows
// that are not 16-byte multiples, and the dequantization kernel.
#include <algorithm>
#include <mutex>

#include "blocks.cuh"
#include "gemv_kernel.cuh"
#include "launch.h"
#include "ops.h"

namespace ntx {
namespace gemv {

template <int QT>
__global__ void dequant_kernel(const uint8_t* W, int64_t rows, int64_t cols, int64_t rb, float* out)
{
    const int64_t total = rows * cols;
    for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < total; i += (int64_t)gridDim.x * blockDim.x) {
        const int64_t r = i / cols, e = i % cols;
        out[i] = weight_at<QT>(W, r, e, rb);
    }
}

// Simple GEMV: one warp per row, lanes stride over the elements; any row length.
template <int QT>
__global__ void gemv_simple_kernel(const uint8_t* W, int rows, int cols, int64_t rb, const float* x, float* y)
{
    const int warps = blockDim.x >> 5;
    const int lane = threadIdx.x & 31;
    for (int r = blockIdx.x * warps + (threadIdx.x >> 5); r < rows; r += gridDim.x * warps) {
        float acc = 0.f;
        for (int i = lane; i < cols; i += 32) acc = fmaf(weight_at<QT>(W, r, i, rb), x[i], acc);
        acc = warp_sum(acc);
        if (lane == 0) y[r] = acc;
    }
}

// ------------------------------------------------------------------ launch shaping

template <int QT>
bool shape(Params& P, int n_sm_unused)
{
    (void)n_sm_unused;
    using F = Fmt<QT>;
    P.chunk_elems = kOwners * F::E;
    P.n_chunks = (P.K + P.chunk_elems - 1) / P.chunk_elems;
    P.chunk_bytes = P.chunk_elems / F::BE * F::BB;
    P.stage_bytes = Slots<QT>::value * P.chunk_bytes;
    P.x_bytes = ((P.K * 4 + 127) / 128) * 128;
    const int fixed = kHeader + P.x_bytes + 128;   // barriers / reduction, x, tail padding
    int ns = (kSmemLimit - fixed) / P.stage_bytes;
    ns = std::min(ns, kMaxStages);
    if (ns < 2) return false;
    P.n_stages = ns;
    return true;
}

int smem_bytes(const Params& P) { return kHeader + P.x_bytes + P.n_stages * P.stage_bytes + 128; }

template <int QT, int EPI, int PRO>
ntx_status launch_t(Params P, cudaStream_t s, int grid_cap)
{
    if (!shape<QT>(P, 0)) return fail(NTX_EUNSUPPORTED, "gemv: row too long for the shared-memory pipeline");
    auto kern = gemv_kernel<QT, EPI, PRO>;
    const int smem = smem_bytes(P);
    const ntx_status st = ensure_smem_limit((const void*)kern, kSmemLimit);
    if (st != NTX_OK) return st;
    P.m24 = 1u << 24;
    const int outs = Outs<QT, EPI>::value;
    int grid = std::min(grid_cap, (P.M + outs - 1) / outs);
    grid = std::max(grid, 1);
    return launch_kernel(kern, dim3(grid), dim3(kThreads), smem, s, P.use_pdl != 0, P);
}

template <int EPI, int PRO>
ntx_status launch_q(int qtype, const Params& P, cudaStream_t s, int grid_cap)
{
    switch (qtype) {
    case NTX_Q8_0: return launch_t<NTX_Q8_0, EPI, PRO>(P, s, grid_cap);
    case NTX_Q4_0: return launch_t<NTX_Q4_0, EPI, PRO>(P, s, grid_cap);
    case NTX_Q4_K: return launch_t<NTX_Q4_K, EPI, PRO>(P, s, grid_cap);
    case NTX_Q6_K: return launch_t<NTX_Q6_K, EPI, PRO>(P, s, grid_cap);
    default: return fail(NTX_EINVAL, "unknown qtype");
    }
}

}  // namespace gemv

ntx_status gemv_launch(int qtype, int epi, int pro, const gemv::Params& P, cudaStream_t s)
{
    using namespace gemv;
    if (epi == EPI_QKV && (!P.rope_cs || P.head_dim > 128))
        return fail(NTX_EINVAL, "gemv: the fused QKV epilogue needs the step's RoPE table (head_dim <= 128)");
    if (is_tiled(qtype)) return qmma_launch(qtype, epi, pro, P, s);
    if (is_float_format(qtype)) return fgemv_launch(qtype, epi, pro, P, s);
    if (qtype == NTX_Q5_K)
        return fail(NTX_EUNSUPPORTED, "gemv: Q5_K streams in its tiled layout only (ntx_repack_q to NTX_Q5_K_T)");
    const int cap = num_sms();
    if (epi == EPI_STORE && pro == PRO_X) return launch_q<EPI_STORE, PRO_X>(qtype, P, s, cap);
    if (epi == EPI_ADD && pro == PRO_X) return launch_q<EPI_ADD, PRO_X>(qtype, P, s, cap);
    if (epi == EPI_SWIGLU && pro == PRO_RMSNORM) return launch_q<EPI_SWIGLU, PRO_RMSNORM>(qtype, P, s, cap);
    if (epi == EPI_QKV && pro == PRO_RMSNORM) return launch_q<EPI_QKV, PRO_RMSNORM>(qtype, P, s, cap);
    if (epi == EPI_STORE && pro == PRO_RMSNORM) return launch_q<EPI_STORE, PRO_RMSNORM>(qtype, P, s, cap);
    return fail(NTX_EUNSUPPORTED, "gemv: unsupported prologue / epilogue combination");
}

cudaError_t take_device_error_gemv(uint32_t* out) { return take_tu_device_error(out); }

bool gemv_fast_path_ok(int qtype, const void* W, int64_t cols)
{
    // the tiled layouts need only a 16-byte aligned base (their 16-row groups are 16-byte multiples);
    // GGUF-style Q5_K has no streaming kernel (its tiled form has), F16 / F32 have their own
    if (qtype == NTX_Q5_K || is_float_format(qtype)) return false;
    return aligned(W, 16) && (is_tiled(qtype) || row_bytes(qtype, cols) % 16 == 0);
}

}  // namespace ntx

using namespace ntx;

NTX_EXPORT ntx_status ntx_gemv_q(int qtype, const void* W, int64_t rows, int64_t cols, const float* x, float* y,
                                 void* stream)
{
    if (qtraits(qtype).block_elems == 0) return fail(NTX_EINVAL, "ntx_gemv_q: unknown qtype");
    if (!W || !x || !y) return fail(NTX_EINVAL, "ntx_gemv_q: null pointer");
    if (rows < 1 || rows > (1 << 30)) return fail(NTX_EINVAL, "ntx_gemv_q: rows out of range");
    if (is_tiled(qtype) && rows % 16) return fail(NTX_EINVAL, "ntx_gemv_q: tiled layouts need a multiple of 16 rows");
    if (row_bytes(qtype, cols) == 0 || cols > (1 << 28))
        return fail(NTX_EINVAL, "ntx_gemv_q: cols must be a positive multiple of the block size");
    if (!aligned(x, 4) || !aligned(y, 4)) return fail(NTX_EINVAL, "ntx_gemv_q: x / y must be 4-byte aligned");
    if (!aligned(W, 2)) return fail(NTX_EINVAL, "ntx_gemv_q: W must be at least 2-byte aligned");
    cudaStream_t s = (cudaStream_t)stream;
    const int64_t rb = row_bytes(qtype, cols);
    if ((gemv_fast_path_ok(qtype, W, cols) && cols <= 32768 && aligned(x, 16)) || fgemv_shape_ok(qtype, W, x, cols)) {
        gemv::Params P{};
        P.W = (const uint8_t*)W;
        P.row_bytes = rb;
        P.M = (int)rows;
        P.K = (int)cols;
        P.x = x;
        P.y = y;
        // programmatic dependent launch: the weight stream may start while the previous
        // kernel of the stream finishes; x is read and y written only after it completed
        P.use_pdl = true;
        return gemv_launch(qtype, gemv::EPI_STORE, gemv::PRO_X, P, s);
    }
    const int threads = 256, warps = threads / 32;
    int grid = (int)std::min<int64_t>((rows + warps - 1) / warps, (int64_t)num_sms() * 8);
#define NTX_SIMPLE(Q) gemv::gemv_simple_kernel<Q><<<grid, threads, 0, s>>>((const uint8_t*)W, (int)rows, (int)cols, rb, x, y)
    switch (qtype) {
    case NTX_Q8_0: NTX_SIMPLE(NTX_Q8_0); break;
    case NTX_Q4_0: NTX_SIMPLE(NTX_Q4_0); break;
    case NTX_Q4_K: NTX_SIMPLE(NTX_Q4_K); break;
    case NTX_Q6_K: NTX_SIMPLE(NTX_Q6_K); break;
    case NTX_Q5_K: NTX_SIMPLE(NTX_Q5_K); break;
    case NTX_F16: NTX_SIMPLE(NTX_F16); break;
    case NTX_F32: NTX_SIMPLE(NTX_F32); break;
    case NTX_Q8_0_T: NTX_SIMPLE(NTX_Q8_0_T); break;
    case NTX_Q4_0_T: NTX_SIMPLE(NTX_Q4_0_T); break;
    case NTX_Q4_K_T: NTX_SIMPLE(NTX_Q4_K_T); break;
    case NTX_Q6_K_T: NTX_SIMPLE(NTX_Q6_K_T); break;
    case NTX_Q5_K_T: NTX_SIMPLE(NTX_Q5_K_T); break;
    }
#undef NTX_SIMPLE
    return check_launch("ntx_gemv_q (simple kernel)");
}

NTX_EXPORT ntx_status ntx_dequant_q(int qtype, const void* W, int64_t rows, int64_t cols, float* out, void* stream)
{
    if (qtraits(qtype).block_elems == 0) return fail(NTX_EINVAL, "ntx_dequant_q: unknown qtype");
    if (!W || !out) return fail(NTX_EINVAL, "ntx_dequant_q: null pointer");
    if (rows < 1 || row_bytes(qtype, cols) == 0) return fail(NTX_EINVAL, "ntx_dequant_q: bad shape");
    if (is_tiled(qtype) && rows % 16) return fail(NTX_EINVAL, "ntx_dequant_q: tiled layouts need a multiple of 16 rows");
    if (!aligned(out, 4)) return fail(NTX_EINVAL, "ntx_dequant_q: out must be 4-byte aligned");
    cudaStream_t s = (cudaStream_t)stream;
    const int64_t rb = row_bytes(qtype, cols);
    const int64_t n = rows * cols;
    const int threads = 256;
    const int grid = (int)std::min<int64_t>((n + threads - 1) / threads, (int64_t)num_sms() * 32);
#define NTX_DQ(Q) gemv::dequant_kernel<Q><<<grid, threads, 0, s>>>((const uint8_t*)W, rows, cols, rb, out)
    switch (qtype) {
    case NTX_Q8_0: NTX_DQ(NTX_Q8_0); break;
    case NTX_Q4_0: NTX_DQ(NTX_Q4_0); break;
    case NTX_Q4_K: NTX_DQ(NTX_Q4_K); break;
    case NTX_Q6_K: NTX_DQ(NTX_Q6_K); break;
    case NTX_Q5_K: NTX_DQ(NTX_Q5_K); break;
    case NTX_F16: NTX_DQ(NTX_F16); break;
    case NTX_F32: NTX_DQ(NTX_F32); break;
    case NTX_Q8_0_T: NTX_DQ(NTX_Q8_0_T); break;
    case NTX_Q4_0_T: NTX_DQ(NTX_Q4_0_T); break;
    case NTX_Q4_K_T: NTX_DQ(NTX_Q4_K_T); break;
    case NTX_Q6_K_T: NTX_DQ(NTX_Q6_K_T); break;
    case NTX_Q5_K_T: NTX_DQ(NTX_Q5_K_T); break;
    }
#undef NTX_DQ
    return check_launch("ntx_dequant_q");
}

NTX_EXPORT ntx_status ntx_repack_q(int qtype, const void* W, void* W_tiled, int64_t rows, int64_t cols, void* stream)
{
    if (qtype < NTX_Q8_0 || qtype > NTX_Q5_K)
        return fail(NTX_EINVAL, "ntx_repack_q: qtype must be a GGUF-style block format (F16 / F32 have no tiled form)");
    if (!W || !W_tiled) return fail(NTX_EINVAL, "ntx_repack_q: null pointer");
    if (rows < 1 || row_bytes(qtype | NTX_TILED, cols) == 0)
        return fail(NTX_EINVAL, "ntx_repack_q: cols must be a positive multiple of the tile size");
    if (rows % 16) return fail(NTX_EINVAL, "ntx_repack_q: tiled layouts need a multiple of 16 rows");
    const int64_t n = rows * row_bytes(qtype, cols);
    const char* a = (const char*)W;
    const char* b = (const char*)W_tiled;
    if (a < b + n && b < a + n) return fail(NTX_EINVAL, "ntx_repack_q: W and W_tiled overlap");
    return repack_launch(qtype, W, W_tiled, rows, cols, (cudaStream_t)stream);
}
