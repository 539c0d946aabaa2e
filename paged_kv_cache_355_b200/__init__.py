"""Paged KV-cache decode attention for NVIDIA B200 (sm_100a).

The work happens in libpa.so (hand-written CUDA kernels behind a C ABI, see
include/pa.h); this package is its thin Python binding plus the seeded
workload generators used by the tests and the benchmark.

    from paged_kv_cache_355_b200 import pa_paged_attention_decode, decode_step

The first use of a binding function fails with ImportError if libpa.so has
not been built (build it with ``python -m paged_kv_cache_355_b200.build``);
there is no fallback implementation.
"""
_BINDING_NAMES = (
    "EXPORTED", "LIB_PATH", "PA_BF16", "PA_F32", "PAError", "pa_copy_blocks", "pa_swap_blocks",
    "pa_decode_slot_mapping",
    "pa_paged_attention_decode", "pa_paged_attention_decode_contiguous", "pa_paged_attention_partition_size",
    "pa_paged_attention_workspace_size", "pa_read_error_flag", "pa_reshape_and_cache", "pa_slot_mapping",
    "pa_status_string", "pa_version", "pa_paged_attention_decode_static_scratch", "STATIC_SCRATCH_BYTES",
    "pa_paged_attention_prefill", "pa_reshape_and_cache_decode", "pa_selftest_wait_timeout",
    "pa_paged_attention_decode_append", "pa_hbm_read_probe", "pa_paged_attention_decode_shared_prefix",
    "pa_paged_attention_shared_prefix_workspace_size",
)
__all__ = list(_BINDING_NAMES) + ["decode_step"]


def __getattr__(name):
    # The binding (and with it libpa.so) loads on first use, so that the build
    # script and the workload generators import without a built library.
    if name in _BINDING_NAMES:
        from . import _binding

        return getattr(_binding, name)
    raise AttributeError(name)


def decode_step(q, k_new, v_new, k_pool, v_pool, block_tables, context_lens, max_context_len, scale, out,
                slots, workspace=None, partition_size=0, cow_pairs=None, stream=None):
    """One decode step of one attention layer, entirely in libpa's kernels:

    1. copy_blocks for pending copy-on-write pairs (if any),
    2. the new token's slot from the block table, the write of its K and V
       there, and paged decode attention over every sequence
       (pa_paged_attention_decode_append: one launch for bf16).

    `context_lens` counts the new token; `slots` is an int64 [B] output buffer
    (or None) that receives each token's slot.
    """
    from . import _binding as b

    if cow_pairs is not None and cow_pairs.numel():
        b.pa_copy_blocks(k_pool, v_pool, cow_pairs, stream=stream)
    b.pa_paged_attention_decode_append(q, k_new, v_new, k_pool, v_pool, block_tables, context_lens, max_context_len,
                                       scale, out, partition_size=partition_size, workspace=workspace,
                                       slot_mapping=slots, stream=stream)
