// probe.cu - read-only HBM streaming probe: the practical bandwidth ceiling of the
// GEMV's data path.
//
// The tiled GEMV streams its weights with one 1-D bulk copy (cp.async.bulk, L2
// evict-first) per stage into a ring of shared-memory stages guarded by mbarriers,
// one CTA per SM.  This kernel does exactly that and nothing else: each CTA takes a
// contiguous slice of the buffer, a producer thread keeps the ring full, one consumer
// warp waits for each stage, reads one word of it and releases it.  Its bytes per
// second are what the GEMV could reach if its arithmetic were free, measured in the
// same run as the GEMV (the copy-test peak is a device-to-device copy instead).
#include "common.cuh"

namespace ntx {
namespace {

constexpr int kStages = 8;
constexpr uint32_t kStageBytes = 24 * 1024;
constexpr uint32_t kPolls = 1u << 22;

static __device__ uint32_t g_probe_sink;   // keeps the consumer's reads live

__global__ void __launch_bounds__(64, 1) stream_probe_kernel(const uint8_t* src, size_t bytes)
{
    extern __shared__ __align__(128) uint8_t smem[];
    uint64_t* full = reinterpret_cast<uint64_t*>(smem);
    uint64_t* empty = full + kStages;
    uint8_t* ring = smem + 256;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    // this CTA's slice, in 16-byte units
    const size_t units = bytes / 16, b0 = units * blockIdx.x / gridDim.x * 16, b1 = units * (blockIdx.x + 1) / gridDim.x * 16;
    const uint32_t n_chunks = (uint32_t)((b1 - b0 + kStageBytes - 1) / kStageBytes);
    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        fence_mbar_init();
    }
    __syncthreads();
    if (warp == 0) {
        if (lane == 0) {
            const uint64_t pol = policy_evict_first();
            uint32_t issued = 0, ph = 0;
            int s = 0;
            bool okay = true;
            for (uint32_t c = 0; c < n_chunks; ++c) {
                if (!mbar_wait(&empty[s], ph ^ 1u, kPolls)) {
                    record_device_error(DEVERR_EMPTY_WAIT);
                    okay = false;
                    break;
                }
                const size_t off = b0 + (size_t)c * kStageBytes;
                const uint32_t n = (uint32_t)min((size_t)kStageBytes, b1 - off);
                mbar_arrive_expect_tx(&full[s], n);
                bulk_g2s(ring + (size_t)s * kStageBytes, src + off, n, &full[s], pol);
                ++issued;
                if (++s == kStages) {
                    s = 0;
                    ph ^= 1u;
                }
            }
            if (!okay) {   // the copies in flight must land before the CTA exits
                for (uint32_t k = 1; k <= kStages && k <= issued; ++k) {
                    const uint32_t j = issued - k;
                    mbar_wait(&full[j % kStages], (j / kStages) & 1u, kPolls);
                }
            }
        }
    } else {
        uint32_t acc = 0, ph = 0;
        int s = 0;
        for (uint32_t c = 0; c < n_chunks; ++c) {
            if (!mbar_wait(&full[s], ph, kPolls)) {
                if (lane == 0) record_device_error(DEVERR_FULL_WAIT);
                break;
            }
            acc += reinterpret_cast<const uint32_t*>(ring + (size_t)s * kStageBytes)[lane];
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[s]);
            if (++s == kStages) {
                s = 0;
                ph ^= 1u;
            }
        }
        if (acc == 0x9E3779B9u) atomicAdd(&g_probe_sink, 1u);
    }
}

}  // namespace

cudaError_t take_device_error_probe(uint32_t* out) { return take_tu_device_error(out); }

}  // namespace ntx

using namespace ntx;

NTX_EXPORT ntx_status ntx_stream_read_probe(const void* src, size_t bytes, void* stream)
{
    if (!src || bytes < 16 || bytes % 16) return fail(NTX_EINVAL, "ntx_stream_read_probe: bytes must be a positive multiple of 16");
    if (!aligned(src, 16)) return fail(NTX_EINVAL, "ntx_stream_read_probe: src must be 16-byte aligned");
    const int smem = 256 + kStages * (int)kStageBytes;
    const ntx_status st = ensure_smem_limit((const void*)stream_probe_kernel, smem);
    if (st != NTX_OK) return st;
    stream_probe_kernel<<<num_sms(), 64, smem, (cudaStream_t)stream>>>((const uint8_t*)src, bytes);
    return check_launch("ntx_stream_read_probe");
}
