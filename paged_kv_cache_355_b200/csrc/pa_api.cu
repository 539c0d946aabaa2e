// pa_api.cu -- library-wide pieces of libpa: the device error word, status
// strings, the version string and the per-device caches the entry points use.
#include <cuda_runtime.h>

#include <stdlib.h>

#include <mutex>

#include "pa.h"
#include "pa_device.cuh"
#include "pa_internal.h"

namespace pa {

// The device error word: written by kernels (first error wins, atomicCAS from
// 0), read and cleared by pa_read_error_flag.  One instance per device.
__device__ int g_error_word = 0;

namespace {
constexpr int kMaxDevices = 64;
std::mutex g_cache_mutex;
int* g_error_ptr[kMaxDevices] = {};
int g_num_sms[kMaxDevices] = {};

int current_device() {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return -1;
    return dev;
}
}  // namespace

// Cached per device: valid while the device's primary context lives (the
// library is not used across a cudaDeviceReset).
int* error_word_ptr() {
    const int dev = current_device();
    if (dev < 0) return nullptr;
    std::lock_guard<std::mutex> lock(g_cache_mutex);
    if (!g_error_ptr[dev]) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_error_word) != cudaSuccess) return nullptr;
        g_error_ptr[dev] = static_cast<int*>(p);
    }
    return g_error_ptr[dev];
}

bool nvtx_enabled() {
    static const bool on = [] {
        const char* v = getenv("PA_NVTX");
        return v && v[0] == '1' && v[1] == 0;
    }();
    return on;
}

int num_sms() {
    const int dev = current_device();
    if (dev < 0) return 148;
    std::lock_guard<std::mutex> lock(g_cache_mutex);
    if (!g_num_sms[dev]) {
        int n = 0;
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
        g_num_sms[dev] = n;
    }
    return g_num_sms[dev];
}

namespace {
// One CTA waits on an mbarrier that nothing ever arrives on: the bounded wait
// runs out after limit_ns, records PA_ERR_TIMEOUT and the kernel returns.
__global__ void wait_selftest_kernel(int* err, uint64_t limit_ns) {
    __shared__ uint64_t bar;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        fence_barrier_init();
    }
    __syncthreads();
    if (threadIdx.x == 0) mbar_wait_for(&bar, 0, err, limit_ns);
}
}  // namespace

}  // namespace pa

extern "C" int pa_selftest_wait_timeout(uint32_t limit_us, void* stream) {
    PA_NVTX_RANGE("pa_selftest_wait_timeout");
    if (limit_us == 0 || limit_us > 2000000u) return PA_ERR_INVALID_ARG;
    int* err = pa::error_word_ptr();
    if (!err) return PA_ERR_CUDA;
    pa::wait_selftest_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(err, (uint64_t)limit_us * 1000u);
    return pa::launch_status();
}

extern "C" const char* pa_status_string(int status) {
    switch (status) {
        case PA_OK: return "PA_OK";
        case PA_ERR_INVALID_ARG: return "PA_ERR_INVALID_ARG";
        case PA_ERR_UNSUPPORTED: return "PA_ERR_UNSUPPORTED";
        case PA_ERR_WORKSPACE: return "PA_ERR_WORKSPACE";
        case PA_ERR_CUDA: return "PA_ERR_CUDA";
        case PA_ERR_BAD_BLOCK_ID: return "PA_ERR_BAD_BLOCK_ID";
        case PA_ERR_TIMEOUT: return "PA_ERR_TIMEOUT";
        default: return "PA_ERR_UNKNOWN";
    }
}

extern "C" const char* pa_version(void) { return "0.1.0"; }

extern "C" int pa_read_error_flag(void* stream) {
    PA_NVTX_RANGE("pa_read_error_flag");
    int* err = pa::error_word_ptr();
    if (!err) return PA_ERR_CUDA;
    int value = 0;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (cudaMemcpyAsync(&value, err, sizeof(int), cudaMemcpyDeviceToHost, s) != cudaSuccess) return PA_ERR_CUDA;
    if (cudaMemsetAsync(err, 0, sizeof(int), s) != cudaSuccess) return PA_ERR_CUDA;
    if (cudaStreamSynchronize(s) != cudaSuccess) return PA_ERR_CUDA;
    return value;
}
