// pa_cache.cu -- the kernels that feed the KV pool: slot mapping,
// reshape_and_cache (write a new token's K/V into its slot), copy_blocks
// (copy-on-write duplication of a shared block) and swap_blocks (whole blocks
// between a device pool and a pinned host pool, for preemption by swapping).
//
// All are bit copies or integer index work, bound by latency (tiny per-step
// sizes), by HBM bandwidth (copy_blocks) or by the host link (swap_blocks).  Each moves 16-byte
// vectors: one (token, kv head) row of head_dim elements is head_dim *
// elt / 16 vectors (8 to 32), contiguous in both source and destination.
#include <cuda_runtime.h>
#include <stdint.h>

#include "pa.h"
#include "pa_device.cuh"
#include "pa_internal.h"

namespace pa {
namespace {

constexpr int kThreads = 256;

// slot of (sequence seq_ids[i], position positions[i]); -1 if unmappable.
// "How does vLLM PagedAttention manage Virtual Memory Pages ...", "Detail":
// virtual block pos / bs -> physical block table[pos / bs], offset pos % bs.
__global__ void slot_mapping_kernel(const int32_t* __restrict__ block_tables, int max_blocks_per_seq, int batch,
                                    const int32_t* __restrict__ seq_ids, const int32_t* __restrict__ positions,
                                    int64_t num_tokens, int block_size, int64_t* __restrict__ slots, int* err) {
    for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < num_tokens;
         i += (int64_t)gridDim.x * blockDim.x) {
        const int b = seq_ids[i];
        const int pos = positions[i];
        int64_t slot = -1;
        if (b >= 0 && b < batch && pos >= 0 && pos / block_size < max_blocks_per_seq) {
            const int32_t phys = block_tables[(int64_t)b * max_blocks_per_seq + pos / block_size];
            if (phys >= 0) slot = (int64_t)phys * block_size + pos % block_size;
        }
        if (slot < 0) record_error(err, PA_ERR_BAD_BLOCK_ID);
        slots[i] = slot;
    }
}

// decode step: token b is position context_lens[b] - 1 of sequence b.
__global__ void decode_slot_mapping_kernel(const int32_t* __restrict__ block_tables, int max_blocks_per_seq,
                                           const int32_t* __restrict__ context_lens, int batch, int block_size,
                                           int64_t* __restrict__ slots, int* err) {
    for (int b = blockIdx.x * blockDim.x + threadIdx.x; b < batch; b += gridDim.x * blockDim.x) {
        const int L = context_lens[b];
        int64_t slot = -1;
        if (L > 0) {
            const int pos = L - 1;
            if (pos / block_size < max_blocks_per_seq) {
                const int32_t phys = block_tables[(int64_t)b * max_blocks_per_seq + pos / block_size];
                if (phys >= 0) slot = (int64_t)phys * block_size + pos % block_size;
            }
            if (slot < 0) record_error(err, PA_ERR_BAD_BLOCK_ID);
        } else if (L < 0) {
            record_error(err, PA_ERR_BAD_BLOCK_ID);
        }
        slots[b] = slot;
    }
}

// One thread per 16-byte vector of one (token, kv head) row, for K and V.
__global__ void reshape_and_cache_kernel(const uint4* __restrict__ key, const uint4* __restrict__ value,
                                         uint4* __restrict__ k_pool, uint4* __restrict__ v_pool,
                                         const int64_t* __restrict__ slots, int64_t num_tokens, int num_kv_heads,
                                         int row_vecs, int block_size, int64_t num_blocks, int* err) {
    const int64_t per_token = (int64_t)num_kv_heads * row_vecs;
    const int64_t total = num_tokens * per_token;
    for (int64_t idx = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; idx < total;
         idx += (int64_t)gridDim.x * blockDim.x) {
        const int64_t tok = idx / per_token;
        const int64_t rem = idx - tok * per_token;
        const int64_t slot = slots[tok];
        if (slot < 0) continue;
        const int64_t blk = slot / block_size;
        if (blk >= num_blocks) {
            if (rem == 0) record_error(err, PA_ERR_BAD_BLOCK_ID);
            continue;
        }
        const int h = (int)(rem / row_vecs);
        const int c = (int)(rem - (int64_t)h * row_vecs);
        const int64_t off = slot - blk * block_size;
        const int64_t dst = ((blk * num_kv_heads + h) * block_size + off) * row_vecs + c;
        k_pool[dst] = key[idx];
        v_pool[dst] = value[idx];
    }
}

// Decode step, slot mapping and cache write in one pass: token b is position
// context_lens[b] - 1 of sequence b; every thread of its rows derives the slot
// from the table itself, so no slot array has to round-trip through memory
// between two launches.  The thread owning vector 0 of token b stores the
// slot (if asked) and records a bad table entry.
__global__ void decode_append_kernel(const uint4* __restrict__ key, const uint4* __restrict__ value,
                                     uint4* __restrict__ k_pool, uint4* __restrict__ v_pool,
                                     const int32_t* __restrict__ block_tables, int max_blocks_per_seq,
                                     const int32_t* __restrict__ context_lens, int batch, int num_kv_heads,
                                     int row_vecs, int block_size, int64_t num_blocks, int64_t* __restrict__ slots,
                                     int* err) {
    griddep_wait();
    griddep_launch_dependents();
    const int64_t per_token = (int64_t)num_kv_heads * row_vecs;
    const int64_t total = (int64_t)batch * per_token;
    for (int64_t idx = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; idx < total;
         idx += (int64_t)gridDim.x * blockDim.x) {
        const int b = (int)(idx / per_token);
        const int64_t rem = idx - (int64_t)b * per_token;
        const int L = context_lens[b];
        int64_t blk = -1;
        int off = 0;
        if (L > 0 && (L - 1) / block_size < max_blocks_per_seq) {
            const int pos = L - 1;
            blk = block_tables[(int64_t)b * max_blocks_per_seq + pos / block_size];
            off = pos % block_size;
        }
        // the slot as pa_decode_slot_mapping gives it; the write also needs
        // the block inside the pool
        const bool ok = blk >= 0 && blk < num_blocks;
        if (rem == 0) {
            if (slots) slots[b] = blk >= 0 ? blk * block_size + off : -1;
            if (!ok && L != 0) record_error(err, PA_ERR_BAD_BLOCK_ID);
        }
        if (!ok) continue;
        const int h = (int)(rem / row_vecs);
        const int c = (int)(rem - (int64_t)h * row_vecs);
        const int64_t dst = ((blk * num_kv_heads + h) * block_size + off) * row_vecs + c;
        k_pool[dst] = key[idx];
        v_pool[dst] = value[idx];
    }
}

// blockIdx.x = pair; blockIdx.y strides over the block's 16-byte vectors.
// Source and destination pools may be the same pool (copy-on-write) or two
// pools, one of them in pinned host memory mapped into the device address
// space (swap).  Each thread keeps four 16-byte loads in flight so that a
// source across PCIe still sees enough outstanding requests.
__global__ void copy_blocks_kernel(const uint4* src_k, const uint4* src_v, uint4* dst_k, uint4* dst_v,
                                   const int64_t* __restrict__ block_mapping, int64_t src_num_blocks,
                                   int64_t dst_num_blocks, int64_t block_vecs, int* err) {
    constexpr int kUnroll = 4;
    const int64_t p = blockIdx.x;
    const int64_t src = block_mapping[2 * p];
    const int64_t dst = block_mapping[2 * p + 1];
    if (src < 0 || src >= src_num_blocks || dst < 0 || dst >= dst_num_blocks) {
        if (threadIdx.x == 0 && blockIdx.y == 0) record_error(err, PA_ERR_BAD_BLOCK_ID);
        return;
    }
    const uint4* ks = src_k + src * block_vecs;
    const uint4* vs = src_v + src * block_vecs;
    uint4* kd = dst_k + dst * block_vecs;
    uint4* vd = dst_v + dst * block_vecs;
    const int64_t step = (int64_t)gridDim.y * blockDim.x;
    for (int64_t i0 = blockIdx.y * (int64_t)blockDim.x + threadIdx.x; i0 < block_vecs; i0 += step * kUnroll) {
        uint4 a[kUnroll], b[kUnroll];
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
            const int64_t i = i0 + u * step;
            if (i < block_vecs) {
                a[u] = ks[i];
                b[u] = vs[i];
            }
        }
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
            const int64_t i = i0 + u * step;
            if (i < block_vecs) {
                kd[i] = a[u];
                vd[i] = b[u];
            }
        }
    }
}

int launch_copy(const void* src_k, const void* src_v, void* dst_k, void* dst_v, const int64_t* block_mapping,
                int64_t num_pairs, int num_kv_heads, int head_dim, int block_size, int64_t src_num_blocks,
                int64_t dst_num_blocks, int dtype, void* stream) {
    int* err = error_word_ptr();
    if (!err) return PA_ERR_CUDA;
    const int64_t block_vecs = (int64_t)num_kv_heads * block_size * head_dim * (int64_t)dtype_bytes(dtype) / 16;
    int64_t slices = (block_vecs + kThreads * 4 - 1) / (kThreads * 4);
    if (slices > 64) slices = 64;
    if (slices < 1) slices = 1;
    dim3 grid((unsigned)num_pairs, (unsigned)slices);
    copy_blocks_kernel<<<grid, kThreads, 0, (cudaStream_t)stream>>>(
        static_cast<const uint4*>(src_k), static_cast<const uint4*>(src_v), static_cast<uint4*>(dst_k),
        static_cast<uint4*>(dst_v), block_mapping, src_num_blocks, dst_num_blocks, block_vecs, err);
    return launch_status();
}

inline int grid_for(int64_t work) {
    int64_t blocks = (work + kThreads - 1) / kThreads;
    const int64_t cap = (int64_t)num_sms() * 16;
    if (blocks > cap) blocks = cap;
    return (int)(blocks < 1 ? 1 : blocks);
}

}  // namespace
}  // namespace pa

using namespace pa;

extern "C" int pa_slot_mapping(const int32_t* block_tables, int max_blocks_per_seq, int batch,
                               const int32_t* seq_ids, const int32_t* positions, int64_t num_tokens,
                               int block_size, int64_t* slot_mapping, void* stream) {
    PA_NVTX_RANGE("pa_slot_mapping");
    if (num_tokens < 0 || batch < 0 || max_blocks_per_seq < 0 || block_size <= 0) return PA_ERR_INVALID_ARG;
    if (num_tokens == 0) return PA_OK;
    if (!block_tables || !seq_ids || !positions || !slot_mapping) return PA_ERR_INVALID_ARG;
    int* err = error_word_ptr();
    if (!err) return PA_ERR_CUDA;
    slot_mapping_kernel<<<grid_for(num_tokens), kThreads, 0, (cudaStream_t)stream>>>(
        block_tables, max_blocks_per_seq, batch, seq_ids, positions, num_tokens, block_size, slot_mapping, err);
    return launch_status();
}

extern "C" int pa_decode_slot_mapping(const int32_t* block_tables, int max_blocks_per_seq,
                                      const int32_t* context_lens, int batch, int block_size,
                                      int64_t* slot_mapping, void* stream) {
    PA_NVTX_RANGE("pa_decode_slot_mapping");
    if (batch < 0 || max_blocks_per_seq < 0 || block_size <= 0) return PA_ERR_INVALID_ARG;
    if (batch == 0) return PA_OK;
    if (!block_tables || !context_lens || !slot_mapping) return PA_ERR_INVALID_ARG;
    int* err = error_word_ptr();
    if (!err) return PA_ERR_CUDA;
    decode_slot_mapping_kernel<<<grid_for(batch), kThreads, 0, (cudaStream_t)stream>>>(
        block_tables, max_blocks_per_seq, context_lens, batch, block_size, slot_mapping, err);
    return launch_status();
}

extern "C" int pa_reshape_and_cache(const void* key, const void* value, void* k_pool, void* v_pool,
                                    const int64_t* slot_mapping, int64_t num_tokens, int num_kv_heads,
                                    int head_dim, int block_size, int64_t num_blocks, int dtype,
                                    void* stream) {
    PA_NVTX_RANGE("pa_reshape_and_cache");
    if (num_tokens < 0 || num_kv_heads <= 0 || head_dim <= 0 || block_size <= 0 || num_blocks < 0 ||
        !valid_dtype(dtype))
        return PA_ERR_INVALID_ARG;
    if (!supported_head_dim(head_dim) || !supported_block_size(block_size)) return PA_ERR_UNSUPPORTED;
    if (num_tokens == 0) return PA_OK;
    if (!key || !value || !k_pool || !v_pool || !slot_mapping) return PA_ERR_INVALID_ARG;
    if (!aligned16(key) || !aligned16(value) || !aligned16(k_pool) || !aligned16(v_pool))
        return PA_ERR_INVALID_ARG;
    int* err = error_word_ptr();
    if (!err) return PA_ERR_CUDA;
    const int row_vecs = (int)(head_dim * dtype_bytes(dtype) / 16);
    reshape_and_cache_kernel<<<grid_for(num_tokens * num_kv_heads * row_vecs), kThreads, 0,
                               (cudaStream_t)stream>>>(
        static_cast<const uint4*>(key), static_cast<const uint4*>(value), static_cast<uint4*>(k_pool),
        static_cast<uint4*>(v_pool), slot_mapping, num_tokens, num_kv_heads, row_vecs, block_size, num_blocks, err);
    return launch_status();
}

extern "C" int pa_reshape_and_cache_decode(const void* key, const void* value, void* k_pool, void* v_pool,
                                           const int32_t* block_tables, int max_blocks_per_seq,
                                           const int32_t* context_lens, int batch, int num_kv_heads, int head_dim,
                                           int block_size, int64_t num_blocks, int dtype, int64_t* slot_mapping,
                                           void* stream) {
    PA_NVTX_RANGE("pa_reshape_and_cache_decode");
    if (batch < 0 || max_blocks_per_seq < 0 || num_kv_heads <= 0 || head_dim <= 0 || block_size <= 0 ||
        num_blocks < 0 || !valid_dtype(dtype))
        return PA_ERR_INVALID_ARG;
    if (!supported_head_dim(head_dim) || !supported_block_size(block_size)) return PA_ERR_UNSUPPORTED;
    if (batch == 0) return PA_OK;
    if (!key || !value || !k_pool || !v_pool || !block_tables || !context_lens) return PA_ERR_INVALID_ARG;
    if (!aligned16(key) || !aligned16(value) || !aligned16(k_pool) || !aligned16(v_pool))
        return PA_ERR_INVALID_ARG;
    int* err = error_word_ptr();
    if (!err) return PA_ERR_CUDA;
    const int row_vecs = (int)(head_dim * dtype_bytes(dtype) / 16);
    return launch_pdl(decode_append_kernel, dim3(grid_for((int64_t)batch * num_kv_heads * row_vecs)), dim3(kThreads),
                      0, (cudaStream_t)stream, static_cast<const uint4*>(key), static_cast<const uint4*>(value),
                      static_cast<uint4*>(k_pool), static_cast<uint4*>(v_pool), block_tables, max_blocks_per_seq,
                      context_lens, batch, num_kv_heads, row_vecs, block_size, num_blocks, slot_mapping, err);
}

extern "C" int pa_copy_blocks(void* k_pool, void* v_pool, const int64_t* block_mapping, int64_t num_pairs,
                              int num_kv_heads, int head_dim, int block_size, int64_t num_blocks, int dtype,
                              void* stream) {
    PA_NVTX_RANGE("pa_copy_blocks");
    if (num_pairs < 0 || num_kv_heads <= 0 || head_dim <= 0 || block_size <= 0 || num_blocks < 0 ||
        !valid_dtype(dtype))
        return PA_ERR_INVALID_ARG;
    if (!supported_head_dim(head_dim) || !supported_block_size(block_size)) return PA_ERR_UNSUPPORTED;
    if (num_pairs == 0) return PA_OK;
    if (num_pairs > 0x7fffffff) return PA_ERR_INVALID_ARG;
    if (!k_pool || !v_pool || !block_mapping || !aligned16(k_pool) || !aligned16(v_pool)) return PA_ERR_INVALID_ARG;
    return launch_copy(k_pool, v_pool, k_pool, v_pool, block_mapping, num_pairs, num_kv_heads, head_dim, block_size,
                       num_blocks, num_blocks, dtype, stream);
}

extern "C" int pa_swap_blocks(const void* src_k, const void* src_v, void* dst_k, void* dst_v,
                              const int64_t* block_mapping, int64_t num_pairs, int num_kv_heads, int head_dim,
                              int block_size, int64_t src_num_blocks, int64_t dst_num_blocks, int dtype,
                              void* stream) {
    PA_NVTX_RANGE("pa_swap_blocks");
    if (num_pairs < 0 || num_kv_heads <= 0 || head_dim <= 0 || block_size <= 0 || src_num_blocks < 0 ||
        dst_num_blocks < 0 || !valid_dtype(dtype))
        return PA_ERR_INVALID_ARG;
    if (!supported_head_dim(head_dim) || !supported_block_size(block_size)) return PA_ERR_UNSUPPORTED;
    if (num_pairs == 0) return PA_OK;
    if (num_pairs > 0x7fffffff) return PA_ERR_INVALID_ARG;
    if (!src_k || !src_v || !dst_k || !dst_v || !block_mapping) return PA_ERR_INVALID_ARG;
    if (!aligned16(src_k) || !aligned16(src_v) || !aligned16(dst_k) || !aligned16(dst_v)) return PA_ERR_INVALID_ARG;
    return launch_copy(src_k, src_v, dst_k, dst_v, block_mapping, num_pairs, num_kv_heads, head_dim, block_size,
                       src_num_blocks, dst_num_blocks, dtype, stream);
}
