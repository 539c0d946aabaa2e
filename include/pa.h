/*
 * pa.h -- C ABI of libpa.so, the paged KV-cache decode path for NVIDIA B200
 * (sm_100a).
 *
 * The pages this follows:
 *   [P1] "PagedAttention and KV memory management" (guide.dupenodi.dev)
 *   [P2] "Paged Attention: OS-Inspired Memory Management for KV Caches"
 *        (Modern AI Engineering, lesson 13.6)
 *   [P3] "How does vLLM PagedAttention manage Virtual Memory Pages to
 *        eliminate KV cache fragmentation?" (iloveeagents.com)
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 *  * Every array argument is a device pointer owned by the caller (for
 *    example the storage of a contiguous torch tensor), 16-byte aligned, and
 *    stays owned by the caller.  The library allocates no device memory and
 *    keeps no state between calls other than one device-side error word per
 *    device (see pa_read_error_flag).
 *  * `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *    stream).  Every call only enqueues work on it and returns; a returned
 *    PA_OK means the arguments passed host-side validation and the launches
 *    were accepted, not that the kernels have finished.  The decode kernels
 *    and pa_reshape_and_cache_decode are launched with programmatic stream
 *    serialisation: they may be scheduled while the previous kernel on the
 *    stream drains, but touch no global memory before it has completed, so
 *    stream order holds exactly as for ordinary launches.  Calls may be
 *    captured into CUDA graphs.
 *  * Element types: PA_F32 (IEEE fp32) or PA_BF16 (bfloat16).  Query, key
 *    and value share one element type; all arithmetic accumulates in fp32.
 *  * KV pool layout (the pages fix none; [P1] "The kernel side" only says
 *    "a pool of blocks"): k_pool and v_pool are separate arrays, each
 *    [num_blocks][num_kv_heads][block_size][head_dim] row-major, so one
 *    (block, kv head) tile is block_size * head_dim contiguous elements.
 *  * A slot is block_id * block_size + offset: token position pos of a
 *    sequence whose block table is `table` has slot
 *    table[pos / block_size] * block_size + pos % block_size ([P3] "Detail",
 *    virtual block i -> physical block table[i], one block of block_size
 *    tokens allocated at a time).
 *  * Grouped query heads: query head h reads kv head h / (Hq / Hkv).
 *  * Supported shapes: head_dim in {64, 128}; block_size in {8, 16, 32};
 *    Hq % Hkv == 0 with Hq / Hkv in {1, 2, 4, 8}, or 16 for bf16.  Anything
 *    else returns PA_ERR_UNSUPPORTED without launching.
 *  * Device-side checks: a block id outside [0, num_blocks), a negative or
 *    too-long context length, or a slot outside the pool is never
 *    dereferenced.  The kernel skips it and records the first such error in
 *    the device error word (PA_ERR_BAD_BLOCK_ID), which pa_read_error_flag
 *    returns; outputs that depended on it are unspecified.  No kernel traps.
 *  * Every wait inside a kernel is bounded in time; a wait that runs out
 *    records PA_ERR_TIMEOUT in the error word and the kernel returns.
 */
#ifndef PA_H_
#define PA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum { PA_F32 = 0, PA_BF16 = 1 } pa_dtype;

typedef enum {
    PA_OK = 0,
    PA_ERR_INVALID_ARG = 1,  /* null pointer, negative size, misaligned pointer, bad enum */
    PA_ERR_UNSUPPORTED = 2,  /* valid but unsupported head_dim / block_size / group size */
    PA_ERR_WORKSPACE = 3,    /* workspace missing or smaller than required */
    PA_ERR_CUDA = 4,         /* a CUDA runtime call or launch failed */
    PA_ERR_BAD_BLOCK_ID = 5, /* device side: block id / slot / length outside its range */
    PA_ERR_TIMEOUT = 6       /* device side: a bounded wait ran out */
} pa_status;

/* Human-readable name of a status code (static storage, never NULL). */
const char* pa_status_string(int status);

/* Library version as "major.minor.patch" (static storage). */
const char* pa_version(void);

/*
 * pa_read_error_flag -- synchronise `stream`, then return the first
 * device-side error recorded by any kernel of this library on the current
 * device since the previous call (PA_OK if none), and clear it.  Returns
 * PA_ERR_CUDA if the synchronisation itself fails.  The error word's device
 * address is looked up once per device and cached, which assumes the
 * device's primary context lives until the process exits (no
 * cudaDeviceReset between calls into the library).
 */
int pa_read_error_flag(void* stream);

/*
 * pa_selftest_wait_timeout -- exercise the bounded-wait path without a
 * fault (no counterpart in the pages; it exists so that tests can show a wait
 * that runs out is reported and leaves the context usable).  Launches one
 * CTA that waits on a shared-memory mbarrier nothing ever arrives on; after
 * limit_us microseconds (1 .. 2,000,000) the wait gives up, records
 * PA_ERR_TIMEOUT in the device error word and the kernel returns normally.
 * Read the result with pa_read_error_flag.
 */
int pa_selftest_wait_timeout(uint32_t limit_us, void* stream);

/*
 * pa_hbm_read_probe -- read `bytes` of device memory at `buffer` as one
 * stream and discard them: the HBM read ceiling against which paged decode
 * attention, itself a read stream of K/V bytes, is measured.  No counterpart in
 * the pages: a measurement aid.  Each CTA (2 per SM) moves a grid-strided
 * series of 8 KB chunks of the buffer into a 6-stage shared-memory ring with
 * bulk TMA copies and never looks at them; nothing is written to global
 * memory.  buffer: device pointer, 16-byte aligned; bytes: a multiple of 16
 * (0 does nothing); else PA_ERR_INVALID_ARG.  Waits are bounded as everywhere.
 */
int pa_hbm_read_probe(const void* buffer, size_t bytes, void* stream);

/*
 * pa_slot_mapping -- slot of each new token ([P3] "Detail": logical block
 * pos / block_size of the sequence maps to the physical block its table
 * names; the token sits at offset pos % block_size inside it).
 *   block_tables      int32 [batch][max_blocks_per_seq]
 *   seq_ids           int32 [num_tokens]  sequence of token i
 *   positions         int32 [num_tokens]  0-based position of token i
 *   slot_mapping      int64 [num_tokens]  output
 * A token whose sequence id or position is out of range, or whose table
 * entry is negative, gets slot -1 (reshape_and_cache then skips it) and
 * records PA_ERR_BAD_BLOCK_ID.
 */
int pa_slot_mapping(const int32_t* block_tables, int max_blocks_per_seq, int batch,
                    const int32_t* seq_ids, const int32_t* positions, int64_t num_tokens,
                    int block_size, int64_t* slot_mapping, void* stream);

/*
 * pa_decode_slot_mapping -- the decode-step special case of pa_slot_mapping:
 * token b is the last token (position context_lens[b] - 1) of sequence b.
 * A sequence of length 0 gets slot -1 (nothing to write).
 *   context_lens int32 [batch] (lengths INCLUDING the token being written)
 *   slot_mapping int64 [batch] output
 */
int pa_decode_slot_mapping(const int32_t* block_tables, int max_blocks_per_seq,
                           const int32_t* context_lens, int batch, int block_size,
                           int64_t* slot_mapping, void* stream);

/*
 * pa_reshape_and_cache -- write each new token's K and V into its slot:
 *   k_pool[s / bs][h][s % bs][:] = key[i][h][:]  and the same for value,
 * for every token i with s = slot_mapping[i] >= 0 ([P3] "Key Technical
 * Innovations" item 2: blocks fill one token at a time as generation
 * proceeds).  Bit-exact copy.
 *   key, value    [num_tokens][num_kv_heads][head_dim]   (dtype)
 *   k_pool,v_pool [num_blocks][num_kv_heads][block_size][head_dim] (dtype), updated in place
 *   slot_mapping  int64 [num_tokens]; negative = skip.  Slots must be
 *                 distinct within one call (caller's precondition).
 */
int pa_reshape_and_cache(const void* key, const void* value, void* k_pool, void* v_pool,
                         const int64_t* slot_mapping, int64_t num_tokens, int num_kv_heads,
                         int head_dim, int block_size, int64_t num_blocks, int dtype,
                         void* stream);

/*
 * pa_reshape_and_cache_decode -- pa_decode_slot_mapping and
 * pa_reshape_and_cache of one decode step in a single launch ([P3] "Detail"
 * for the slot, "Key Technical Innovations" item 2 for the write): token b
 * is position context_lens[b] - 1 of sequence b, its slot is
 * block_tables[b][pos / bs] * bs + pos % bs, and its K and V rows go there.
 *   key, value    [batch][num_kv_heads][head_dim]   (dtype)
 *   block_tables  int32 [batch][max_blocks_per_seq]
 *   context_lens  int32 [batch], lengths INCLUDING the token being written
 *   slot_mapping  int64 [batch] output, or NULL: the slot each token got,
 *                 exactly as pa_decode_slot_mapping computes it
 * Length 0 writes nothing (slot -1).  A negative length, an unmapped
 * position or a block outside [0, num_blocks) writes nothing and records
 * PA_ERR_BAD_BLOCK_ID.  Pool contents after the call are bit-identical to
 * the two-call sequence.  Launched with programmatic stream serialisation,
 * so a following pa_paged_attention_decode can be scheduled while it drains.
 */
int pa_reshape_and_cache_decode(const void* key, const void* value, void* k_pool, void* v_pool,
                                const int32_t* block_tables, int max_blocks_per_seq,
                                const int32_t* context_lens, int batch, int num_kv_heads,
                                int head_dim, int block_size, int64_t num_blocks, int dtype,
                                int64_t* slot_mapping, void* stream);

/*
 * pa_copy_blocks -- copy-on-write duplication of shared blocks ([P2] "Key
 * terms in this lesson", Copy-on-write: a block is shared until someone
 * writes to it, and the writer then gets a private copy; [P1] "Myths and
 * failure modes", parallel samples share their prompt this way).
 * For every pair p: block block_mapping[p][1] := block block_mapping[p][0],
 * whole K block and whole V block, bit-exact.
 *   block_mapping int64 [num_pairs][2] as (src, dst).  Destinations must be
 *                 distinct and no destination may also be a source in the
 *                 same call (caller's precondition).  An id outside
 *                 [0, num_blocks) skips the pair and records PA_ERR_BAD_BLOCK_ID.
 */
int pa_copy_blocks(void* k_pool, void* v_pool, const int64_t* block_mapping, int64_t num_pairs,
                   int num_kv_heads, int head_dim, int block_size, int64_t num_blocks, int dtype,
                   void* stream);

/*
 * pa_swap_blocks -- move whole blocks between two pools of the same shape
 * except their block counts, typically a device pool and a pinned host pool
 * (swap-out and swap-in when the scheduler preempts a sequence by swapping,
 * [P1] "Key takeaways": the scheduler preempts by swapping or recomputing,
 * and paging makes both finer-grained).
 * For every pair p: dst block block_mapping[p][1] := src block
 * block_mapping[p][0], K and V, bit-exact.
 *   src_k, src_v  [src_num_blocks][num_kv_heads][block_size][head_dim]
 *   dst_k, dst_v  [dst_num_blocks][...same...]
 * Each pool pointer is device memory or pinned host memory that the device
 * can address (cudaHostAlloc / torch pin_memory under unified addressing);
 * one kernel moves all pairs, so a host-side pool is read or written across
 * the host link without per-block copy calls.  block_mapping (int64
 * [num_pairs][2]) must be device-addressable too.  Destinations must be
 * distinct.  Ids outside their pool skip the pair and record
 * PA_ERR_BAD_BLOCK_ID.
 */
int pa_swap_blocks(const void* src_k, const void* src_v, void* dst_k, void* dst_v,
                   const int64_t* block_mapping, int64_t num_pairs, int num_kv_heads, int head_dim,
                   int block_size, int64_t src_num_blocks, int64_t dst_num_blocks, int dtype,
                   void* stream);

/*
 * pa_paged_attention_partition_size -- tokens per KV split that
 * pa_paged_attention_decode uses for these sizes when called with
 * partition_size == 0 (a multiple of 32, at most 8192).  Sequences longer
 * than it are processed as several splits merged by a second pass.
 */
int pa_paged_attention_partition_size(int batch, int num_q_heads, int num_kv_heads, int head_dim,
                                      int max_context_len, int block_size, int* partition_size);

/*
 * pa_paged_attention_workspace_size -- bytes of scratch the decode call
 * needs for the split-KV partial results (0 when no sequence can need more
 * than one split).  partition_size: 0 = automatic, else a multiple of 32 in
 * [32, 8192].
 */
int pa_paged_attention_workspace_size(int batch, int num_q_heads, int num_kv_heads, int head_dim,
                                      int max_context_len, int block_size, int partition_size,
                                      size_t* workspace_bytes);

/*
 * pa_paged_attention_decode -- single-query (decode) attention that reads
 * every sequence's K and V straight from the block pool through its block
 * table, with no gather into a contiguous buffer ([P1] "The kernel side":
 * read the block table, load each physical block's K and V tiles in turn,
 * compute scores and weighted values in place).  For each sequence b and
 * query head h, with L = context_lens[b] and kv head g = h / (Hq / Hkv):
 *   s_t = scale * <q[b][h], K_t>,  out[b][h] = sum_t softmax(s)_t * V_t,
 * over the tokens t < L; L == 0 gives a zero row.  Softmax is evaluated
 * online in fp32; sequences longer than the partition size are split and
 * merged by a log-sum-exp second pass (deterministic, no atomics).
 *   q             [batch][num_q_heads][head_dim] (kv_dtype)
 *   k_pool,v_pool [num_blocks][num_kv_heads][block_size][head_dim] (kv_dtype)
 *   block_tables  int32 [batch][max_blocks_per_seq]; only the first
 *                 ceil(L / block_size) entries of a row are read
 *   context_lens  int32 [batch]
 *   max_context_len  host-side upper bound of context_lens (sizes the grid;
 *                 must be <= max_blocks_per_seq * block_size)
 *   out           [batch][num_q_heads][head_dim], out_dtype PA_F32 or PA_BF16
 *   partition_size  0 = automatic (pa_paged_attention_partition_size)
 *   workspace     device scratch of at least the size
 *                 pa_paged_attention_workspace_size returns (NULL if 0)
 */
int pa_paged_attention_decode(const void* q, const void* k_pool, const void* v_pool,
                              const int32_t* block_tables, int max_blocks_per_seq,
                              const int32_t* context_lens, int max_context_len, float scale,
                              int block_size, void* out, int out_dtype, int batch,
                              int num_q_heads, int num_kv_heads, int head_dim,
                              int64_t num_blocks, int kv_dtype, int partition_size,
                              void* workspace, size_t workspace_bytes, void* stream);

/*
 * pa_paged_attention_decode_append -- one whole decode step: the new token's
 * slot and cache write (exactly pa_reshape_and_cache_decode: token b is
 * position context_lens[b] - 1 of sequence b) followed by
 * pa_paged_attention_decode over lengths that include it ([P3] "Key
 * Technical Innovations" item 2 for the write, [P1] "The kernel side" for the
 * attention).  Arguments are those of the two calls: key, value
 * [batch][num_kv_heads][head_dim] (kv_dtype); slot_mapping int64 [batch]
 * output or NULL.  The pools are updated in place, bit for bit as the
 * two-call sequence leaves them, and the output matches it within rounding.
 * For bf16 it is one launch (plus the merge when sequences are split): the
 * CTA that reads a sequence's last block writes the new K and V rows into
 * the pool slot and into the tile it has staged, so no separate write kernel
 * runs.  fp32 runs the two calls.  Errors as for the two calls.  As for
 * pa_reshape_and_cache, the written slots must be distinct and the block
 * holding each one must belong to its sequence alone (no other sequence of
 * the batch reads it), which copy-on-write before the step guarantees.
 */
int pa_paged_attention_decode_append(const void* q, const void* key, const void* value,
                                     void* k_pool, void* v_pool, const int32_t* block_tables,
                                     int max_blocks_per_seq, const int32_t* context_lens,
                                     int max_context_len, float scale, int block_size, void* out,
                                     int out_dtype, int batch, int num_q_heads, int num_kv_heads,
                                     int head_dim, int64_t num_blocks, int kv_dtype,
                                     int partition_size, void* workspace, size_t workspace_bytes,
                                     int64_t* slot_mapping, void* stream);

/*
 * pa_paged_attention_shared_prefix_workspace_size -- bytes of scratch that
 * pa_paged_attention_decode_shared_prefix needs for these sizes (always > 0:
 * the partial results, each sequence's prefix length and, when the prefix
 * pass runs last, one counter).
 * num_groups >= 1, max_group_size >= 1, 0 <= max_prefix_len <=
 * max_context_len; partition_size as for pa_paged_attention_decode.
 */
int pa_paged_attention_shared_prefix_workspace_size(int batch, int num_q_heads, int num_kv_heads,
                                                    int head_dim, int max_context_len,
                                                    int block_size, int num_groups,
                                                    int max_group_size, int max_prefix_len,
                                                    int partition_size, size_t* workspace_bytes);

/*
 * pa_paged_attention_decode_shared_prefix -- pa_paged_attention_decode for a
 * batch whose sequences come in groups that share a prompt: parallel samples
 * hold one copy of the prompt's blocks, shared by reference count
 * ([P1] "Key takeaways": samples share a prompt without copying it;
 * [P2] "Key terms in this lesson", Reference count and Copy-on-write).  The
 * result is the same attention as pa_paged_attention_decode over the same
 * tables and lengths (within rounding: the softmax is split at different
 * points), but each shared block is read from memory once per group instead
 * of once per member: a prefix pass attends the group's shared tokens for
 * all its members' query heads at once (tensor cores: for head_dim 128 the
 * shared tokens are the M side of tcgen05 MMAs and the query heads their N
 * side; for 64 the query heads are stacked on the M side of mma.sync), and
 * pass 1 attends each member's own tokens after the prefix.  For head_dim
 * 128, when the prefix is one split (at most the prefix partition, 4096
 * tokens by default) and the own tokens one split, a one-CTA set-up kernel
 * checks the groups and stores each sequence's prefix length, pass 1 runs
 * next and stores each own part's partial result, and the prefix pass runs
 * last -- its CTAs start as pass 1's last wave drains -- and writes every
 * shared row, its own state combined with pass 1's partial by the
 * log-sum-exp rescale.  Otherwise the prefix pass runs first, pass 1 folds
 * the prefix in, and the merge pass combines the two where a member's own
 * tokens span several splits.
 *   group_starts       int32 [num_groups + 1], device: group g is sequences
 *                      group_starts[g] .. group_starts[g + 1] - 1, with
 *                      group_starts[0] = 0, non-decreasing,
 *                      group_starts[num_groups] = batch (the groups cover the
 *                      batch; a sequence that shares nothing is a group of
 *                      one with prefix 0)
 *   group_prefix_lens  int32 [num_groups], device: tokens 0 .. P_g - 1 of
 *                      every member of group g are the same physical slots:
 *                      P_g is a multiple of block_size, the first P_g /
 *                      block_size entries of every member's table are equal,
 *                      and P_g <= context_lens[b] for every member
 *   max_group_size     host-side upper bound of the group sizes
 *   max_prefix_len     host-side upper bound of the P_g (<= max_context_len)
 *   workspace          pa_paged_attention_shared_prefix_workspace_size bytes
 * Other arguments as for pa_paged_attention_decode.  bf16 only (kv_dtype
 * PA_BF16, else PA_ERR_UNSUPPORTED).  A group whose prefix breaks these
 * rules (not whole blocks, longer than a member or than max_prefix_len) or
 * that is larger than max_group_size records PA_ERR_BAD_BLOCK_ID and is
 * attended without sharing (prefix 0), with the correct result.  Starts out
 * of order or out of range, and groups that do not cover the batch, record it
 * too; the outputs of the sequences that no well-formed group covers are then
 * unspecified (but nothing outside the arrays is read or written).  Equal
 * table entries are the caller's precondition and are not checked.
 */
int pa_paged_attention_decode_shared_prefix(const void* q, const void* k_pool, const void* v_pool,
                                            const int32_t* block_tables, int max_blocks_per_seq,
                                            const int32_t* context_lens, int max_context_len,
                                            float scale, int block_size, void* out, int out_dtype,
                                            int batch, int num_q_heads, int num_kv_heads,
                                            int head_dim, int64_t num_blocks, int kv_dtype,
                                            const int32_t* group_starts,
                                            const int32_t* group_prefix_lens, int num_groups,
                                            int max_group_size, int max_prefix_len,
                                            int partition_size, void* workspace,
                                            size_t workspace_bytes, void* stream);

/*
 * pa_paged_attention_prefill -- causal attention for several new query
 * tokens per sequence over the paged cache (chunked prefill, or speculative
 * tokens): the multi-query form of pa_paged_attention_decode, reading K and V
 * through the block table in the same way ([P1] "The kernel side").
 * Sequence b of length L = context_lens[b] (counting its new tokens, whose
 * K/V must already be in the pool) owns query rows query_start[b] ..
 * query_start[b + 1] - 1, its last n = query_start[b + 1] - query_start[b]
 * tokens; row i sits at position p = L - n + i and attends keys 0..p:
 *   out[r][h] = sum_{t <= p} softmax_t(scale * <q[r][h], K_t>) V_t.
 *   q             [num_tokens][num_q_heads][head_dim] bf16
 *   query_start   int32 [batch + 1], non-decreasing, query_start[0] = 0,
 *                 query_start[batch] = num_tokens
 *   max_query_len host-side upper bound of the n (sizes the grid)
 *   out           [num_tokens][num_q_heads][head_dim], out_dtype PA_F32 or PA_BF16
 * bf16 only (kv_dtype PA_BF16, else PA_ERR_UNSUPPORTED); head_dim 64 or 128;
 * Hq / Hkv in {1, 2, 4, 8, 16}.  Runs on the 5th-generation tensor cores
 * (tcgen05 with tensor-memory accumulators).  A sequence with n > L or a
 * length beyond its table is skipped and records PA_ERR_BAD_BLOCK_ID.
 */
int pa_paged_attention_prefill(const void* q, const void* k_pool, const void* v_pool,
                               const int32_t* block_tables, int max_blocks_per_seq,
                               const int32_t* context_lens, const int32_t* query_start,
                               int max_query_len, float scale, int block_size, void* out,
                               int out_dtype, int batch, int num_q_heads, int num_kv_heads,
                               int head_dim, int64_t num_tokens, int64_t num_blocks, int kv_dtype,
                               void* stream);

/*
 * pa_paged_attention_decode_contiguous -- the same attention over a
 * contiguous cache, the "ideal contiguous attention" [P1] "The kernel side"
 * measures the paged kernel against.  Same kernel, same tiling and staging
 * (tiles of block_size tokens), only the address of a tile differs:
 *   k_c, v_c  [batch][num_kv_heads][L_pad][head_dim] (kv_dtype), L_pad >= max_context_len
 */
int pa_paged_attention_decode_contiguous(const void* q, const void* k_c, const void* v_c,
                                         int64_t L_pad, const int32_t* context_lens,
                                         int max_context_len, float scale, int block_size,
                                         void* out, int out_dtype, int batch, int num_q_heads,
                                         int num_kv_heads, int head_dim, int kv_dtype,
                                         int partition_size, void* workspace,
                                         size_t workspace_bytes, void* stream);

/*
 * ------------------------------------------------------------------------
 * Host-side block manager.
 *
 * The allocator the pages describe: fixed-size blocks, a per-sequence block
 * table, one block taken at a time as a sequence grows ([P1] introduction;
 * [P3] "Detail", "Key Technical Innovations" 1-2), a first-in first-out free
 * list that starts as every block id in increasing order ([P3] "Example"),
 * reference counts and copy-on-write for shared blocks ([P2] "Key terms in
 * this lesson").  Unlike the kernels above it is stateful host code: the
 * handle owns host memory until pa_bm_destroy.  Not thread-safe.  Every
 * pointer argument here is a HOST pointer.
 * ------------------------------------------------------------------------
 */
typedef struct pa_block_manager pa_block_manager;

/* A manager for num_blocks blocks of block_size tokens; NULL on bad sizes or
 * out of host memory.  Block ids are 0..num_blocks-1 (num_blocks < 2^31). */
pa_block_manager* pa_bm_create(int64_t num_blocks, int block_size);
void pa_bm_destroy(pa_block_manager* bm);

/* Register an empty sequence (PA_ERR_INVALID_ARG if the id exists). */
int pa_bm_add_sequence(pa_block_manager* bm, int64_t seq_id);

/*
 * Append one token to each seq_ids[i] in order (unknown ids start empty).
 * slots[i] receives the token's slot.  A token at position pos takes a new
 * block from the head of the free list when pos % block_size == 0.  A token
 * written into a block shared with other sequences (refcount > 1) first moves
 * its sequence onto a fresh block: the pair (shared, fresh) is appended to
 * cow_pairs (int64 [2 * capacity], may be NULL to only count) and counted in
 * *num_cow_pairs; the caller runs pa_copy_blocks on those pairs before
 * writing the tokens.  Returns PA_ERR_WORKSPACE when the free list runs out;
 * the tokens before the failing one stay appended.
 */
int pa_bm_append_tokens(pa_block_manager* bm, const int64_t* seq_ids, int64_t n, int64_t* slots,
                        int64_t* cow_pairs, int64_t* num_cow_pairs);

/* child shares every block of parent (reference counts + 1). */
int pa_bm_fork(pa_block_manager* bm, int64_t parent, int64_t child);

/* Drop a sequence; blocks whose count reaches 0 return to the free list's tail. */
int pa_bm_free_sequence(pa_block_manager* bm, int64_t seq_id);

/* Free blocks, a block's reference count, a sequence's length (-1 if unknown). */
int64_t pa_bm_num_free(const pa_block_manager* bm);
int pa_bm_refcount(const pa_block_manager* bm, int64_t block);
int64_t pa_bm_length(const pa_block_manager* bm, int64_t seq_id);

/* Dense block tables int32 [n][max_blocks_per_seq] (-1 past each sequence's
 * blocks) and, if context_lens is not NULL, their lengths: the inputs of
 * pa_paged_attention_decode once copied to the device.  PA_ERR_UNSUPPORTED if
 * a table is wider than max_blocks_per_seq. */
int pa_bm_block_tables(const pa_block_manager* bm, const int64_t* seq_ids, int64_t n,
                       int max_blocks_per_seq, int32_t* tables, int32_t* context_lens);

/* The free list in hand-out order: the first min(cap, free) ids into out,
 * the number of free blocks into *n. */
int pa_bm_free_list(const pa_block_manager* bm, int64_t* out, int64_t cap, int64_t* n);

/*
 * The sharing structure of a batch as pa_paged_attention_decode_shared_prefix
 * takes it (reference-counted prompt blocks shared by parallel samples,
 * [P2] "Key terms in this lesson"; [P1] "Key takeaways").  seq_ids[0..n) in
 * batch order are cut into groups of consecutive sequences whose tables begin
 * with the same physical block; a sequence with no block, or whose first
 * block differs from its predecessor's, starts a new group.  A group's prefix
 * is the run of leading table entries that are equal in every member, cut to
 * the blocks that are full in every member, times block_size (0 when the
 * members share nothing full).
 *   group_starts   int32 [n + 1] output: group g is batch rows
 *                  group_starts[g] .. group_starts[g + 1] - 1
 *   prefix_lens    int32 [n] output: the first *num_groups entries are used
 *   num_groups, max_group_size, max_prefix_len  outputs (the host-side
 *                  bounds the decode call takes)
 * PA_ERR_INVALID_ARG for an unknown sequence id or a null output.
 */
int pa_bm_shared_prefix_groups(const pa_block_manager* bm, const int64_t* seq_ids, int64_t n,
                               int32_t* group_starts, int32_t* prefix_lens, int64_t* num_groups,
                               int32_t* max_group_size, int32_t* max_prefix_len);

/*
 * pa_paged_attention_decode_static_scratch -- pa_paged_attention_decode for
 * callers that cannot allocate device memory.  The pages have no counterpart:
 * this is a deployment convenience of this library.
 *
 * Some callers cannot call cudaMalloc (or any allocating routine) where they
 * run decode attention: code inside a CUDA graph capture or a latency-bound
 * serving loop that must not enter the allocator, or an embedder whose device
 * memory belongs to another framework's pool.  This entry point takes the
 * same arguments as pa_paged_attention_decode minus the workspace and uses
 * instead a fixed scratch array of PA_STATIC_SCRATCH_BYTES that lives in the
 * library itself (a file-scope __device__ array).  It calls no cudaMalloc,
 * cudaFree or other allocating routine.  The caller still passes q, the
 * pools, the tables and `out`, exactly as for pa_paged_attention_decode, and
 * gets bit-identical results.
 *
 *  * Memory: every GPU that loads the library holds the PA_STATIC_SCRATCH_BYTES
 *    array until the process exits, whether or not this entry point is used.
 *  * Limit: a call whose split-KV scratch (pa_paged_attention_workspace_size)
 *    exceeds PA_STATIC_SCRATCH_BYTES returns PA_ERR_WORKSPACE without
 *    launching; a larger partition_size needs less scratch.
 *  * Set-up: the first call on each device looks up the array's device
 *    address (cudaGetSymbolAddress, with that device current) and caches it;
 *    make that first call before any stream capture on the device.  The
 *    cached address assumes the device's primary CUDA context lives as long
 *    as the process: after cudaDeviceReset (or any teardown of that context)
 *    the library must not be called again in the same process, since the
 *    cached address (and the library's cached error-word address, see
 *    pa_read_error_flag) would point into the destroyed context.
 *  * Sharing: every call uses the same array, which keeps the previous call's
 *    contents (nothing in it needs to start at zero).  Calls that overlap on
 *    the GPU, for example on two streams, race on it; calls ordered on one
 *    stream are safe.
 */
#define PA_STATIC_SCRATCH_BYTES (16u << 20)

int pa_paged_attention_decode_static_scratch(const void* q, const void* k_pool, const void* v_pool,
                                             const int32_t* block_tables, int max_blocks_per_seq,
                                             const int32_t* context_lens, int max_context_len,
                                             float scale, int block_size, void* out, int out_dtype,
                                             int batch, int num_q_heads, int num_kv_heads,
                                             int head_dim, int64_t num_blocks, int kv_dtype,
                                             int partition_size, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* PA_H_ */
