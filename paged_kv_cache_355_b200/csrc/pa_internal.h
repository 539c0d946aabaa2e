// pa_internal.h -- host-side helpers shared by the libpa translation units.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include <nvtx3/nvToolsExt.h>

#include <utility>

#include "pa.h"

namespace pa {

// NVTX ranges around the entry points that launch work, for timeline
// profilers: on when the environment has PA_NVTX=1 (read once per process),
// otherwise one predictable branch per call.
bool nvtx_enabled();

struct NvtxRange {
    bool on;
    explicit NvtxRange(const char* name) : on(nvtx_enabled()) {
        if (on) nvtxRangePushA(name);
    }
    ~NvtxRange() {
        if (on) nvtxRangePop();
    }
};

// Device address of the current device's error word (resolved once per
// device with cudaGetSymbolAddress).  NULL if the lookup failed.
int* error_word_ptr();

// Streaming multiprocessors of the current device (cached per device).
int num_sms();

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

inline size_t dtype_bytes(int dtype) { return dtype == PA_BF16 ? 2 : 4; }

inline bool valid_dtype(int dtype) { return dtype == PA_F32 || dtype == PA_BF16; }

inline bool supported_head_dim(int d) { return d == 64 || d == 128; }

inline bool supported_block_size(int bs) { return bs == 8 || bs == 16 || bs == 32; }

inline int launch_status() {
    return cudaGetLastError() == cudaSuccess ? PA_OK : PA_ERR_CUDA;
}

// Launch with programmatic stream serialisation: the kernel may be scheduled
// before the previous kernel on the stream has fully drained, and must call
// griddep_wait() before touching global memory.  Captured into CUDA graphs
// as a programmatic edge.
template <typename... KArgs, typename... Args>
inline int launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                      Args&&... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    const cudaError_t e = cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
    if (e != cudaSuccess) {
        (void)cudaGetLastError();
        return PA_ERR_CUDA;
    }
    return launch_status();
}

}  // namespace pa

#define PA_NVTX_RANGE(name) ::pa::NvtxRange pa_nvtx_range_(name)
