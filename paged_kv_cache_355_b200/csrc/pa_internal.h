// pa_internal.h -- host-side helpers shared by the libpa translation units.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "pa.h"

namespace pa {

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

}  // namespace pa
