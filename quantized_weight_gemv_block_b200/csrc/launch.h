// launch.h - kernel launch with an optional programmatic-dependent-launch attribute.
#pragma once

#include "common.cuh"

namespace ntx {

template <typename... KArgs, typename... Args>
ntx_status launch_kernel(void (*kern)(KArgs...), dim3 grid, dim3 block, int smem, cudaStream_t s, bool pdl,
                         Args&&... args)
{
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = (size_t)smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = pdl ? 1 : 0;
    cudaError_t e = cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
    if (e != cudaSuccess) return fail(NTX_ECUDA, std::string("kernel launch: ") + cudaGetErrorString(e));
    return NTX_OK;
}

}  // namespace ntx
