// qmma.cu - host side of the GEMV for the tiled layouts (launch shaping, the choice
// of CUDA-core or tensor-core units) and the repack kernel GGUF-style -> tiled.
#include <algorithm>
#include <cstdlib>
#include <map>
#include <mutex>

#include "qmma.cuh"

namespace ntx {
namespace qmma {

// ------------------------------------------------------------------ repack
// Readers of the GGUF-style source row (the codes as the formats store them).

__device__ __forceinline__ int src_q4_0(const uint8_t* row, int64_t e)
{
    const uint8_t* blk = row + (e >> 5) * 18 + 2;
    const int i = (int)(e & 31);
    return i < 16 ? (blk[i] & 15) : (blk[i - 16] >> 4);
}

__device__ __forceinline__ int src_q6_k(const uint8_t* row, int64_t e)
{
    const uint8_t* b = row + (e >> 8) * 210;
    const int r256 = (int)(e & 255), h = r256 >> 7, t = r256 & 127;
    const int lo = t < 64 ? (b[64 * h + t] & 15) : (b[64 * h + t - 64] >> 4);
    const int hi = (b[128 + 32 * h + (t & 31)] >> (2 * (t >> 5))) & 3;
    return lo | (hi << 4);
}

__device__ __forceinline__ int src_q4_k(const uint8_t* row, int64_t e)
{
    const uint8_t* b = row + (e >> 8) * 144;
    const int r256 = (int)(e & 255), c = r256 >> 6, r = r256 & 63;
    const int byte = b[16 + 32 * c + (r & 31)];
    return r < 32 ? (byte & 15) : (byte >> 4);
}

// Q5_K: the low 4 bits and the fifth bit of element e of a GGUF-style row.
__device__ __forceinline__ int src_q5_k_lo(const uint8_t* row, int64_t e)
{
    const uint8_t* b = row + (e >> 8) * 176;
    const int r256 = (int)(e & 255), c = r256 >> 6, r = r256 & 63;
    const int byte = b[48 + 32 * c + (r & 31)];
    return r < 32 ? (byte & 15) : (byte >> 4);
}

__device__ __forceinline__ int src_q5_k_b5(const uint8_t* row, int64_t e)
{
    const uint8_t* b = row + (e >> 8) * 176;
    const int r256 = (int)(e & 255), c = r256 >> 6, r = r256 & 63;
    return (b[16 + (r & 31)] >> (2 * c + (r >> 5))) & 1;
}

// Q4_K / Q5_K 6-bit value V(m, b) of the tiled layout for rows (gid, gid + 8) of group W16
// (BB: bytes of one GGUF-style superblock; the scales sit at byte 4 of it in both).
template <int BB>
__device__ __forceinline__ int src_k_v(const uint8_t* W16, int64_t rb, int64_t sb, int gid, int m, int b)
{
    const uint8_t* blk = W16 + (int64_t)(gid + 8 * (b & 1)) * rb + sb * BB;
    int sc, mn;
    gemv::q4k_sm(blk + 4, m, sc, mn);
    return (b & 2) ? mn : sc;
}

// Byte p (< 192) of the scale section of a Q4_K / Q5_K tiled unit.
template <int BB>
__device__ __forceinline__ uint8_t k_scale_byte(const uint8_t* W16, int64_t rb, int64_t u, int p)
{
    const int gid = p / 24, r = p % 24;
    if (r < 16) {
        const int wn = r >> 2, b = r & 3;
        return (uint8_t)((src_k_v<BB>(W16, rb, u, gid, 2 * wn, b) & 15) |
                         ((src_k_v<BB>(W16, rb, u, gid, 2 * wn + 1, b) & 15) << 4));
    }
    const int wh = (r - 16) >> 2, b = r & 3;
    int v = 0;
    for (int t = 0; t < 4; ++t) v |= ((src_k_v<BB>(W16, rb, u, gid, 4 * wh + t, b) >> 4) & 3) << (2 * t);
    return (uint8_t)v;
}

// Byte `o` of unit u of the 16-row group that starts at GGUF row pointer W16.
template <int QT>
__device__ __forceinline__ uint8_t tiled_byte(const uint8_t* W16, int64_t rb, int64_t u, int o)
{
    if constexpr (QT == NTX_Q8_0_T) {
        if (o < 512) {
            const int lane = o >> 4, reg = (o >> 2) & 3, j = o & 3;
            const int row = (lane >> 2) + 8 * (reg & 1);
            const int col = 16 * (reg >> 1) + 4 * (lane & 3) + j;
            return W16[row * rb + u * 34 + 2 + col];
        }
        const int p = o - 512, row = (p >> 2) + 8 * ((p >> 1) & 1);
        return W16[row * rb + u * 34 + (p & 1)];
    } else if constexpr (QT == NTX_Q4_0_T) {
        if (o < 256) {
            const int lane = o >> 3, hi = (o >> 2) & 1, j = o & 3;
            const uint8_t* row = W16 + (int64_t)((lane >> 2) + 8 * hi) * rb;
            const int64_t e = 32 * u + 4 * (lane & 3) + j;
            return (uint8_t)(src_q4_0(row, e) | (src_q4_0(row, e + 16) << 4));
        }
        const int p = o - 256, row = (p >> 2) + 8 * ((p >> 1) & 1);
        return W16[row * rb + u * 18 + (p & 1)];
    } else if constexpr (QT == NTX_Q6_K_T) {
        if (o < 3072) {
            const int m = o / 384, r = o % 384, lane = r / 12, wi = (r % 12) >> 2, j = r & 3;
            const int gid = lane >> 2, tig = lane & 3;
            const int64_t e0 = 256 * u + 32 * m + 4 * tig + j;
            // A: row gid col c; B: row gid+8 col c; C: row gid col c+16; a3: row gid+8 col c+16
            const uint8_t* rowA = W16 + (int64_t)(gid + (wi == 1 ? 8 : 0)) * rb;
            const int q = src_q6_k(rowA, e0 + (wi == 2 ? 16 : 0));
            const int q3 = src_q6_k(W16 + (int64_t)(gid + 8) * rb, e0 + 16);
            return (uint8_t)(q | (((q3 >> (2 * wi)) & 3) << 6));
        }
        if (o < 3328) {
            const int p = o - 3072, vec = p >> 4, bi = p & 15;
            const int gid = vec >> 1, par = vec & 1, hi = bi >> 3, mm = bi & 7;
            return W16[(int64_t)(gid + 8 * hi) * rb + u * 210 + 192 + 2 * mm + par];
        }
        const int p = o - 3328, row = (p >> 2) + 8 * ((p >> 1) & 1);
        return W16[row * rb + u * 210 + 208 + (p & 1)];
    } else {
        if (o < 2048) {
            const int m = o >> 8, r = o & 255, lane = r >> 3, hi = (r >> 2) & 1, j = r & 3;
            const uint8_t* row = W16 + (int64_t)((lane >> 2) + 8 * hi) * rb;
            const int64_t e = 256 * u + 32 * m + 4 * (lane & 3) + j;
            return (uint8_t)(src_q4_k(row, e) | (src_q4_k(row, e + 16) << 4));
        }
        if (o < 2240) return k_scale_byte<144>(W16, rb, u, o - 2048);
        const int p = o - 2240, gid = p >> 3, k = (p >> 1) & 3;
        // k: 0 d(gid), 1 d(gid+8), 2 dmin(gid), 3 dmin(gid+8)
        const int row = gid + 8 * (k & 1);
        return W16[(int64_t)row * rb + u * 144 + 2 * (k >> 1) + (p & 1)];
    }
}

// Byte `o` of Q5_K unit u of the 16-row group that starts at GGUF row pointer W16.
__device__ __forceinline__ uint8_t tiled_byte_q5_k(const uint8_t* W16, int64_t rb, int64_t u, int o)
{
    if (o < 2560) {
        const int m = o / 320, r = o % 320;
        const int64_t e0 = 256 * u + 32 * m;
        if (r < 256) {
            // low 4 bits as Q4_K: lane, word P / Q, byte j
            const int lane = r >> 3, hi = (r >> 2) & 1, j = r & 3;
            const uint8_t* row = W16 + (int64_t)((lane >> 2) + 8 * hi) * rb;
            const int64_t e = e0 + 4 * (lane & 3) + j;
            return (uint8_t)(src_q5_k_lo(row, e) | (src_q5_k_lo(row, e + 16) << 4));
        }
        // fifth bits: gid, word H0 / H1 (row gid / gid + 8), byte j holds bit 2t (column
        // 4t + j) and bit 2t + 1 (column 16 + 4t + j) for t = 0..3
        const int p = r - 256, gid = p >> 3, hi = (p >> 2) & 1, j = p & 3;
        const uint8_t* row = W16 + (int64_t)(gid + 8 * hi) * rb;
        int v = 0;
        for (int t = 0; t < 4; ++t)
            v |= (src_q5_k_b5(row, e0 + 4 * t + j) << (2 * t)) | (src_q5_k_b5(row, e0 + 16 + 4 * t + j) << (2 * t + 1));
        return (uint8_t)v;
    }
    if (o < 2752) return k_scale_byte<176>(W16, rb, u, o - 2560);
    const int p = o - 2752, gid = p >> 3, k = (p >> 1) & 3;
    const int row = gid + 8 * (k & 1);
    return W16[(int64_t)row * rb + u * 176 + 2 * (k >> 1) + (p & 1)];
}

template <int QT>
__global__ void repack_kernel(const uint8_t* in, uint8_t* out, int64_t n_bytes, int64_t rb)
{
    using T = gemv::Tiled<QT>;
    const int64_t gb = 16 * rb;
    for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n_bytes; i += (int64_t)gridDim.x * blockDim.x) {
        const int64_t grp = i / gb, o = i - grp * gb;
        const int64_t u = o / T::UB;
        if constexpr (QT == NTX_Q5_K_T)
            out[i] = tiled_byte_q5_k(in + grp * gb, rb, u, (int)(o - u * T::UB));
        else
            out[i] = tiled_byte<QT>(in + grp * gb, rb, u, (int)(o - u * T::UB));
    }
}

// ------------------------------------------------------------------ launch shaping

// Columns a CTA takes: the whole row, or the larger half when CTA pairs split it.
template <int QT>
int cta_cols(int K, int csize)
{
    using T = gemv::Tiled<QT>;
    return csize == 2 ? (K / T::UK + 1) / 2 * T::UK : K;
}

template <int QT>
bool shape(Params& P, int n_clusters, int csize, int n_mats)
{
    using T = gemv::Tiled<QT>;
    const int kh = cta_cols<QT>(P.K, csize);
    // 32 words per 32-column step of the half, then one float per step (16-byte multiple)
    P.fs_off = kh * 4;
    P.x_bytes = kh * 4 + (kh / 32 * 4 + 15) / 16 * 16;
    const int max_groups = (P.M / 16 + n_clusters - 1) / n_clusters;
    P.recv_bytes = max_groups * n_mats * 16 * 4;
    const int avail = kSmemLimit - kHeader - P.x_bytes - P.recv_bytes - 128;
    // chunks of up to 4096 columns (whole units), shrunk until at least 3 stages fit: each
    // consumer warp then takes two K-quant units (or 16 Q8_0 units) per stage, two
    // independent dot chains to interleave, and crosses half as many stage barriers.
    // Measured on B200 against 2048: Llama-70B Q6_K decode 80.6 -> 85.1 tok/s, Llama-8B
    // Q8_0 493.4 -> 503.2.  NTX_GEMV_CE overrides the first choice (a tuning override).
    const char* ce_env = std::getenv("NTX_GEMV_CE");
    const int ce_max = (ce_env && ce_env[0]) ? std::max(T::UK, std::atoi(ce_env)) : 4096;
    int ce = std::min(kh, ce_max) / T::UK * T::UK;
    while (ce > T::UK && avail / (ce / T::UK * T::UB) < 3) ce = std::max(T::UK, ce / 2 / T::UK * T::UK);
    if (ce < T::UK || avail <= 0) return false;
    P.chunk_elems = ce;
    P.n_chunks = (kh + ce - 1) / ce;
    P.chunk_bytes = ce / T::UK * T::UB;
    P.stage_bytes = P.chunk_bytes;
    const int ns = std::min(kMaxStages, avail / P.stage_bytes);
    if (ns < 2) return false;
    P.n_stages = ns;
    return true;
}

// Clusters of `csize` CTAs (one per SM) that fit on the current device at once, per
// kernel (queried once per device and cluster size).
template <int QT, int EPI, int PRO, int CORE>
int max_clusters(int csize)
{
    static std::mutex mu;
    static std::map<std::pair<int, int>, int> cache;
    int dev = 0;
    cudaGetDevice(&dev);
    std::lock_guard<std::mutex> lock(mu);
    const auto key = std::make_pair(dev, csize);
    const auto it = cache.find(key);
    if (it != cache.end()) return it->second;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(csize * 256);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = kSmemLimit;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = csize;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int c = 0;
    if (cudaOccupancyMaxActiveClusters(&c, qmma_kernel<QT, EPI, PRO, CORE>, &cfg) != cudaSuccess || c < 1) {
        cudaGetLastError();
        c = std::max(1, num_sms() / csize);
    }
    cache[key] = c;
    return c;
}

// Whether CTA pairs split the columns: when whole rows would leave the last round of
// 16-row groups unbalanced (fewer than 6 groups per SM) and the rows are long
// (16384 columns or more) so half a row still amortises a group's fixed costs.
// Measured on B200: 8192 x 28672 Q6_K 4.84 TB/s split against 4.39 whole; at 8192
// columns the two are even, at 4096 the split loses.  NTX_GEMV_SPLIT=0 / 1
// overrides the choice (a tuning override).
inline int pick_cluster_size(int M, int K)
{
    const char* env = std::getenv("NTX_GEMV_SPLIT");
    if (env && env[0] == '0') return 1;
    if (env && env[0] == '1') return 2;
    return (M / 16 < 6 * num_sms() && K >= 16384) ? 2 : 1;
}

template <int QT, int EPI, int PRO, int CORE>
ntx_status launch_t(Params P, cudaStream_t s)
{
    auto kern = qmma_kernel<QT, EPI, PRO, CORE>;
    const ntx_status st = ensure_smem_limit((const void*)kern, kSmemLimit);
    if (st != NTX_OK) return st;
    // NTX_TEST_STALL_STAGE=k (tests of the failure path only): the producer stops before
    // stage k, so the consumers' bounded wait runs out and the kernel records an error
    const char* stall = std::getenv("NTX_TEST_STALL_STAGE");
    P.stall_stage = (stall && stall[0]) ? std::atoi(stall) : -1;
    const int csize = pick_cluster_size(P.M, P.K);
    const int n_clusters = std::max(1, std::min(max_clusters<QT, EPI, PRO, CORE>(csize), P.M / 16));
    if (!shape<QT>(P, n_clusters, csize, EPI == gemv::EPI_SWIGLU ? 2 : 1))
        return fail(NTX_EUNSUPPORTED, "gemv: row too long for the shared-memory pipeline");
    const int smem = kHeader + P.x_bytes + P.n_stages * P.stage_bytes + P.recv_bytes + 128;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(csize * n_clusters);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = (size_t)smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = csize;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = P.use_pdl ? 2 : 1;
    const cudaError_t e = cudaLaunchKernelEx(&cfg, kern, P);
    if (e != cudaSuccess) return fail(NTX_ECUDA, std::string("gemv (tiled) launch: ") + cudaGetErrorString(e));
    return NTX_OK;
}

// Which units reduce the codes: dp4a on the CUDA cores (1, the default) or the integer
// tensor cores (0).  Measured on B200 (event-timed, inputs larger than L2): Q6_K
// 28672 x 8192 5.10 TB/s dp4a against 5.11 MMA, 8192 x 28672 5.11 against 5.05, Q8_0
// 32768 x 4096 5.07 against 5.18, Q4_0 57344 x 4096 3.48 against 2.87, Q4_K 3.50 against
// 3.69.  NTX_GEMV_CORE=tc / dp4a overrides the choice (a tuning override).
inline int pick_core()
{
    const char* env = std::getenv("NTX_GEMV_CORE");
    if (env && env[0] == 't') return 0;
    if (env && env[0] == 'd') return 1;
    return 1;
}

template <int QT, int EPI, int PRO>
ntx_status launch_c(const Params& P, cudaStream_t s)
{
    return pick_core() == 0 ? launch_t<QT, EPI, PRO, 0>(P, s) : launch_t<QT, EPI, PRO, 1>(P, s);
}

template <int EPI, int PRO>
ntx_status launch_q(int qtype, const Params& P, cudaStream_t s)
{
    switch (qtype) {
    case NTX_Q8_0_T: return launch_c<NTX_Q8_0_T, EPI, PRO>(P, s);
    case NTX_Q4_0_T: return launch_c<NTX_Q4_0_T, EPI, PRO>(P, s);
    case NTX_Q4_K_T: return launch_c<NTX_Q4_K_T, EPI, PRO>(P, s);
    case NTX_Q6_K_T: return launch_c<NTX_Q6_K_T, EPI, PRO>(P, s);
    case NTX_Q5_K_T: return launch_c<NTX_Q5_K_T, EPI, PRO>(P, s);
    default: return fail(NTX_EINVAL, "unknown tiled qtype");
    }
}

}  // namespace qmma

ntx_status qmma_launch(int qtype, int epi, int pro, const gemv::Params& P, cudaStream_t s)
{
    using namespace gemv;
    if (P.M % 16) return fail(NTX_EINVAL, "gemv: tiled layouts need a multiple of 16 rows");
    if (epi == EPI_STORE && pro == PRO_X) return qmma::launch_q<EPI_STORE, PRO_X>(qtype, P, s);
    if (epi == EPI_ADD && pro == PRO_X) return qmma::launch_q<EPI_ADD, PRO_X>(qtype, P, s);
    if (epi == EPI_SWIGLU && pro == PRO_RMSNORM) return qmma::launch_q<EPI_SWIGLU, PRO_RMSNORM>(qtype, P, s);
    if (epi == EPI_QKV && pro == PRO_RMSNORM) return qmma::launch_q<EPI_QKV, PRO_RMSNORM>(qtype, P, s);
    if (epi == EPI_STORE && pro == PRO_RMSNORM) return qmma::launch_q<EPI_STORE, PRO_RMSNORM>(qtype, P, s);
    return fail(NTX_EUNSUPPORTED, "gemv: unsupported prologue / epilogue combination");
}

ntx_status repack_launch(int qtype, const void* W, void* W_tiled, int64_t rows, int64_t cols, cudaStream_t s)
{
    const int64_t rb = row_bytes(qtype, cols);
    const int64_t n = rows * rb;
    const int threads = 256;
    const int grid = (int)std::min<int64_t>((n + threads - 1) / threads, (int64_t)num_sms() * 32);
    const uint8_t* in = (const uint8_t*)W;
    uint8_t* out = (uint8_t*)W_tiled;
    switch (qtype) {
    case NTX_Q8_0: qmma::repack_kernel<NTX_Q8_0_T><<<grid, threads, 0, s>>>(in, out, n, rb); break;
    case NTX_Q4_0: qmma::repack_kernel<NTX_Q4_0_T><<<grid, threads, 0, s>>>(in, out, n, rb); break;
    case NTX_Q4_K: qmma::repack_kernel<NTX_Q4_K_T><<<grid, threads, 0, s>>>(in, out, n, rb); break;
    case NTX_Q6_K: qmma::repack_kernel<NTX_Q6_K_T><<<grid, threads, 0, s>>>(in, out, n, rb); break;
    case NTX_Q5_K: qmma::repack_kernel<NTX_Q5_K_T><<<grid, threads, 0, s>>>(in, out, n, rb); break;
    default: return fail(NTX_EINVAL, "ntx_repack_q: qtype must be a GGUF-style format");
    }
    return check_launch("ntx_repack_q");
}

// The tiled GEMV's device error flag (this translation unit's).
cudaError_t take_device_error_qmma(uint32_t* out) { return take_tu_device_error(out); }

}  // namespace ntx
