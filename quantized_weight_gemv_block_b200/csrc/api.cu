// api.cu - status handling and small C-ABI helpers of the ntx library.
#include <mutex>
#include <set>
#include <string>
#include <tuple>

#include "common.cuh"

namespace ntx {

static thread_local std::string t_last_error;

void set_error(const std::string& msg) { t_last_error = msg; }

ntx_status fail(ntx_status code, const std::string& msg)
{
    t_last_error = msg;
    return code;
}

ntx_status ok() { return NTX_OK; }

ntx_status check_launch(const char* what)
{
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return fail(NTX_ECUDA, std::string(what) + ": " + cudaGetErrorString(e));
    return NTX_OK;
}

ntx_status ensure_smem_limit(const void* func, int bytes)
{
    static std::mutex mu;
    static std::set<std::tuple<int, const void*, int>> done;
    int dev = 0;
    NTX_CUDA_TRY(cudaGetDevice(&dev));
    const auto key = std::make_tuple(dev, func, bytes);
    std::lock_guard<std::mutex> lock(mu);
    if (done.count(key)) return NTX_OK;
    const cudaError_t e = cudaFuncSetAttribute(func, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (e != cudaSuccess)
        return fail(NTX_ECUDA, std::string("setting a kernel's shared-memory limit: ") + cudaGetErrorString(e));
    done.insert(key);
    return NTX_OK;
}

int num_sms()
{
    static int cached[64] = {0};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
    if (cached[dev] == 0) {
        int n = 0;
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
        cached[dev] = n;
    }
    return cached[dev];
}

}  // namespace ntx

using namespace ntx;

NTX_EXPORT const char* ntx_last_error(void) { return t_last_error.c_str(); }

NTX_EXPORT int ntx_version(void) { return 100; }

NTX_EXPORT size_t ntx_row_bytes(int qtype, int64_t cols) { return (size_t)row_bytes(qtype, cols); }

NTX_EXPORT int ntx_block_elems(int qtype) { return qtraits(qtype).block_elems; }

NTX_EXPORT ntx_status ntx_device_error(uint32_t* code)
{
    if (!code) return fail(NTX_EINVAL, "ntx_device_error: null pointer");
    NTX_CUDA_TRY(cudaDeviceSynchronize());
    uint32_t a = 0, b = 0, c = 0, d = 0, e = 0, f = 0, g = 0;
    NTX_CUDA_TRY(take_device_error_gemv(&a));
    NTX_CUDA_TRY(take_device_error_attn(&b));
    NTX_CUDA_TRY(take_device_error_decode(&c));
    NTX_CUDA_TRY(take_device_error_qmma(&d));
    NTX_CUDA_TRY(take_device_error_probe(&e));
    NTX_CUDA_TRY(take_device_error_fgemv(&f));
    NTX_CUDA_TRY(take_device_error_qmma_multi(&g));
    *code = a | b | c | d | e | f | g;
    return NTX_OK;
}
