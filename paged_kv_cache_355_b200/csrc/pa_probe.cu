// pa_probe.cu -- HBM streaming-read probe: the read bandwidth a plain bulk
// read stream reaches on this device, the ceiling against which the decode
// kernel's K/V read rate is measured.
//
// The decode pass reads every K/V byte once and writes almost nothing, so its
// natural roofline is a read-only stream, which runs faster than the
// read-plus-write copy that a STREAM-style measurement gives.  This kernel is
// that stream and nothing else: each CTA walks a grid-strided list of
// fixed-size chunks of the buffer and moves each one into a ring of
// shared-memory stages with the TMA engine (cp.async.bulk, no multicast),
// completion counted on one mbarrier per stage; the bytes are never looked
// at.  One thread per CTA issues and waits; several CTAs per SM keep enough
// bytes in flight to cover the DRAM latency.  Every wait is bounded.
#include <cuda_runtime.h>
#include <stdint.h>

#include "pa.h"
#include "pa_device.cuh"
#include "pa_internal.h"

namespace pa {
namespace {

// 96 KB in flight per SM: a sweep of chunk size (8-64 KB), ring depth (2-8)
// and CTAs per SM (1-8) on a 4 GiB buffer peaked at 96-128 KB per SM
// (7.40-7.42 TB/s); deeper (196 KB per SM) streamed ~2-3 % slower.
constexpr int kProbeStages = 6;
constexpr uint32_t kProbeChunk = 8192;  // bytes per stage
constexpr int kProbeCtasPerSm = 2;

__global__ void __launch_bounds__(32) hbm_read_probe_kernel(const uint8_t* __restrict__ buf, uint64_t bytes,
                                                            int* err) {
    extern __shared__ __align__(128) uint8_t ring[];
    __shared__ uint64_t bar[kProbeStages];
    if (threadIdx.x != 0) return;
    for (int s = 0; s < kProbeStages; ++s) mbar_init(&bar[s], 1);
    fence_barrier_init();
    const uint64_t policy = l2_policy_evict_first();
    const uint64_t nchunks = (bytes + kProbeChunk - 1) / kProbeChunk;
    uint64_t k = 0;  // chunks issued by this CTA
    for (uint64_t c = blockIdx.x; c < nchunks; c += gridDim.x, ++k) {
        const int s = (int)(k % kProbeStages);
        if (k >= kProbeStages && !mbar_wait(&bar[s], (uint32_t)((k / kProbeStages) - 1) & 1u, err)) return;
        const uint64_t off = c * kProbeChunk;
        const uint32_t n = (uint32_t)(bytes - off < kProbeChunk ? bytes - off : kProbeChunk);
        mbar_arrive_expect_tx(&bar[s], n);
        bulk_load(ring + (size_t)s * kProbeChunk, buf + off, n, &bar[s], policy);
    }
    // drain: the last min(k, stages) copies are still in flight
    for (uint64_t j = (k > kProbeStages ? k - kProbeStages : 0); j < k; ++j) {
        const int s = (int)(j % kProbeStages);
        if (!mbar_wait(&bar[s], (uint32_t)(j / kProbeStages) & 1u, err)) return;
    }
}

}  // namespace
}  // namespace pa

extern "C" int pa_hbm_read_probe(const void* buffer, size_t bytes, void* stream) {
    PA_NVTX_RANGE("pa_hbm_read_probe");
    if (bytes == 0) return PA_OK;
    if (!buffer || !pa::aligned16(buffer) || bytes % 16 != 0) return PA_ERR_INVALID_ARG;
    int* err = pa::error_word_ptr();
    if (!err) return PA_ERR_CUDA;
    static bool configured[64] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return PA_ERR_CUDA;
    const size_t smem = (size_t)pa::kProbeStages * pa::kProbeChunk;
    if (!configured[dev]) {
        if (cudaFuncSetAttribute(pa::hbm_read_probe_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) !=
            cudaSuccess)
            return PA_ERR_CUDA;
        configured[dev] = true;
    }
    const uint64_t nchunks = (bytes + pa::kProbeChunk - 1) / pa::kProbeChunk;
    uint64_t grid = (uint64_t)pa::num_sms() * pa::kProbeCtasPerSm;
    if (grid > nchunks) grid = nchunks;
    pa::hbm_read_probe_kernel<<<(unsigned)grid, 32, smem, static_cast<cudaStream_t>(stream)>>>(
        static_cast<const uint8_t*>(buffer), (uint64_t)bytes, err);
    return pa::launch_status();
}
