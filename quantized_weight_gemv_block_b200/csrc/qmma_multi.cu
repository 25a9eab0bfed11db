// qmma_multi.cu - host side of the multi-vector tiled GEMV (qmma_multi.cuh): launch
// shaping and the format / epilogue dispatch.
#include <algorithm>
#include <cstdlib>

#include "launch.h"
#include "qmma_multi.cuh"

namespace ntx {
namespace qmma {
namespace {

using gemv::Params;

// x regions, ring and row sums for NX vectors of K columns; false when they do not fit
// (the caller then runs the vectors one at a time).
template <int QT>
bool shape_multi(Params& P, int nx, int n_ctas, int n_mats)
{
    using T = gemv::Tiled<QT>;
    const int K = P.K;
    P.fs_off = K * 4;
    P.x_bytes = K * 4 + (K / 32 * 4 + 15) / 16 * 16;
    const int max_groups = (P.M / 16 + n_ctas - 1) / n_ctas;
    P.recv_bytes = max_groups * nx * n_mats * 16 * 4;
    const int avail = kSmemLimit - kMHeader - nx * P.x_bytes - P.recv_bytes - 128;
    if (avail <= 0) return false;
    // chunks of 2048 columns, shrunk for a third stage only while a chunk keeps at least 8
    // units: every consumer warp then has a unit of each stage and takes the same columns, in
    // the same order, as in the single-vector kernel (whose 4096-column chunks hand each warp
    // the units of two such chunks at once), so each vector's sums are added in the same order
    int ce = std::min(K, 2048) / T::UK * T::UK;
    while (ce / T::UK > 8 && avail / (ce / T::UK * T::UB) < 3) ce = std::max(8 * T::UK, ce / 2 / T::UK * T::UK);
    P.chunk_elems = ce;
    P.n_chunks = (K + ce - 1) / ce;
    P.chunk_bytes = ce / T::UK * T::UB;
    P.stage_bytes = P.chunk_bytes;
    const int ns = std::min(kMaxStages, avail / P.stage_bytes);
    if (ns < 2) return false;
    P.n_stages = ns;
    return true;
}

template <int QT, int EPI, int PRO, int NX, int CORE>
ntx_status launch_m(Params P, const Vecs& V, cudaStream_t s)
{
    auto kern = qmma_multi_kernel<QT, EPI, PRO, NX, CORE>;
    const ntx_status st = ensure_smem_limit((const void*)kern, kSmemLimit);
    if (st != NTX_OK) return st;
    const int n_ctas = std::max(1, std::min(num_sms(), P.M / 16));
    // NTX_TEST_STALL_STAGE=k (tests of the failure path only): the producer stops before
    // stage k, so the consumers' bounded wait runs out and the kernel records an error
    const char* stall = std::getenv("NTX_TEST_STALL_STAGE");
    P.stall_stage = (stall && stall[0]) ? std::atoi(stall) : -1;
    if (!shape_multi<QT>(P, NX, n_ctas, EPI == gemv::EPI_SWIGLU ? 2 : 1))
        return fail(NTX_EUNSUPPORTED, "gemv (several vectors): the vectors do not fit in shared memory");
    const int smem = kMHeader + NX * P.x_bytes + P.n_stages * P.stage_bytes + P.recv_bytes + 128;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(n_ctas);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = (size_t)smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = P.use_pdl ? 1 : 0;
    const cudaError_t e = cudaLaunchKernelEx(&cfg, kern, P, V);
    if (e != cudaSuccess)
        return fail(NTX_ECUDA, std::string("gemv (several vectors) launch: ") + cudaGetErrorString(e));
    return NTX_OK;
}

template <int EPI, int PRO, int NX, int CORE>
ntx_status launch_c(int qtype, const Params& P, const Vecs& V, cudaStream_t s)
{
    switch (qtype) {
    case NTX_Q8_0_T: return launch_m<NTX_Q8_0_T, EPI, PRO, NX, CORE>(P, V, s);
    case NTX_Q4_0_T: return launch_m<NTX_Q4_0_T, EPI, PRO, NX, CORE>(P, V, s);
    case NTX_Q4_K_T: return launch_m<NTX_Q4_K_T, EPI, PRO, NX, CORE>(P, V, s);
    case NTX_Q6_K_T: return launch_m<NTX_Q6_K_T, EPI, PRO, NX, CORE>(P, V, s);
    case NTX_Q5_K_T: return launch_m<NTX_Q5_K_T, EPI, PRO, NX, CORE>(P, V, s);
    default: return fail(NTX_EUNSUPPORTED, "gemv (several vectors): tiled formats only");
    }
}

// Which units reduce the codes of a batch: the integer tensor cores (0) or dp4a on the CUDA
// cores (1).  NTX_VERIFY_CORE=tc / dp4a overrides the choice (a tuning override).
inline int pick_multi_core()
{
    const char* env = std::getenv("NTX_VERIFY_CORE");
    if (env && env[0] == 't') return 0;
    if (env && env[0] == 'd') return 1;
    return 1;
}

template <int EPI, int PRO, int NX>
ntx_status launch_q(int qtype, const Params& P, const Vecs& V, cudaStream_t s)
{
    return pick_multi_core() == 0 ? launch_c<EPI, PRO, NX, 0>(qtype, P, V, s) : launch_c<EPI, PRO, NX, 1>(qtype, P, V, s);
}

template <int NX>
ntx_status launch_nx(int qtype, int epi, int pro, const Params& P, const Vecs& V, cudaStream_t s)
{
    using namespace gemv;
    if (epi == EPI_QKV && pro == PRO_RMSNORM) return launch_q<EPI_QKV, PRO_RMSNORM, NX>(qtype, P, V, s);
    if (epi == EPI_ADD && pro == PRO_X) return launch_q<EPI_ADD, PRO_X, NX>(qtype, P, V, s);
    if (epi == EPI_SWIGLU && pro == PRO_RMSNORM) return launch_q<EPI_SWIGLU, PRO_RMSNORM, NX>(qtype, P, V, s);
    if (epi == EPI_STORE && pro == PRO_RMSNORM) return launch_q<EPI_STORE, PRO_RMSNORM, NX>(qtype, P, V, s);
    return fail(NTX_EUNSUPPORTED, "gemv (several vectors): unsupported prologue / epilogue");
}

}  // namespace
}  // namespace qmma

// y_v = W x_v for nx (2..4) vectors of the same fused kind, the weights streamed once.
// NTX_EUNSUPPORTED when the format is not tiled or the vectors do not fit (nothing is
// launched then).
ntx_status gemv_multi_launch(int qtype, int epi, int pro, const gemv::Params& P, const gemv::Vecs& V, int nx,
                             cudaStream_t s)
{
    if (P.K % 256 != 0 || P.M % 16 != 0) return fail(NTX_EUNSUPPORTED, "gemv (several vectors): shape");
    switch (nx) {
    case 2: return qmma::launch_nx<2>(qtype, epi, pro, P, V, s);
    case 3: return qmma::launch_nx<3>(qtype, epi, pro, P, V, s);
    case 4: return qmma::launch_nx<4>(qtype, epi, pro, P, V, s);
    default: return fail(NTX_EUNSUPPORTED, "gemv (several vectors): 2 to 4 vectors");
    }
}

cudaError_t take_device_error_qmma_multi(uint32_t* out) { return take_tu_device_error(out); }

}  // namespace ntx
