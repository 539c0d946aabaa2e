// pa_static_scratch.cu -- decode attention for callers that cannot allocate
// device memory.
//
// pa_paged_attention_decode needs caller-provided scratch for the split-KV
// partial results.  Some callers cannot call cudaMalloc at the point where
// they run decode attention: code that runs inside a CUDA graph capture or a
// real-time serving loop that must not enter the allocator, embedders whose
// memory is owned by another framework's pool, plugin hosts that forbid
// allocation after start-up.  This entry point serves them: its scratch is a
// fixed file-scope __device__ array that the CUDA runtime places in device
// memory when the library's module is loaded on a device, so the call itself
// allocates nothing.
//
// Costs and limits (also stated in pa.h):
//  * every GPU that loads the library holds PA_STATIC_SCRATCH_BYTES of it
//    until the process exits;
//  * a call whose split-KV scratch would exceed that size is rejected with
//    PA_ERR_WORKSPACE (a larger partition_size needs less scratch);
//  * all calls share the one array, so two calls that overlap on the GPU (on
//    different streams, say) race on it; calls on one stream are ordered and
//    safe.  The array keeps the previous call's contents; nothing in it needs
//    to start at zero, because the first pass writes every partial result the
//    merge pass reads.
#include <cuda_runtime.h>

#include <mutex>

#include "pa.h"
#include "pa_internal.h"

namespace pa {
namespace {

// In host code this name is only a stand-in for the device array; its device
// address comes from cudaGetSymbolAddress, once per device.
__device__ __align__(256) unsigned char g_decode_scratch[PA_STATIC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_mutex;
void* g_scratch_addr[kMaxDevices] = {};

// Device address of the scratch array on the current device.  Resolved on the
// first call per device (with that device current) and cached; NULL if the
// lookup fails.  The cache assumes the device's primary context lives until
// the process exits: after a cudaDeviceReset the cached address is stale.
void* scratch_address() {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
    std::lock_guard<std::mutex> lock(g_mutex);
    if (!g_scratch_addr[dev]) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_decode_scratch) != cudaSuccess) return nullptr;
        g_scratch_addr[dev] = p;
    }
    return g_scratch_addr[dev];
}

}  // namespace
}  // namespace pa

extern "C" int pa_paged_attention_decode_static_scratch(
    const void* q, const void* k_pool, const void* v_pool, const int32_t* block_tables, int max_blocks_per_seq,
    const int32_t* context_lens, int max_context_len, float scale, int block_size, void* out, int out_dtype,
    int batch, int num_q_heads, int num_kv_heads, int head_dim, int64_t num_blocks, int kv_dtype, int partition_size,
    void* stream) {
    PA_NVTX_RANGE("pa_paged_attention_decode_static_scratch");
    size_t need = 0;
    int rc = pa_paged_attention_workspace_size(batch, num_q_heads, num_kv_heads, head_dim, max_context_len,
                                               block_size, partition_size, &need);
    if (rc != PA_OK) return rc;
    if (need > (size_t)PA_STATIC_SCRATCH_BYTES) return PA_ERR_WORKSPACE;
    void* scratch = nullptr;
    if (need > 0) {
        scratch = pa::scratch_address();
        if (!scratch) return PA_ERR_CUDA;
    }
    return pa_paged_attention_decode(q, k_pool, v_pool, block_tables, max_blocks_per_seq, context_lens,
                                     max_context_len, scale, block_size, out, out_dtype, batch, num_q_heads,
                                     num_kv_heads, head_dim, num_blocks, kv_dtype, partition_size, scratch, need,
                                     stream);
}
