// pa_decode.cu -- paged decode attention for sm_100a.
//
// What it computes ("PagedAttention and KV memory management", section "The
// kernel side"): for each sequence, read its block table, load each physical
// block's K and V tiles in turn, and compute scores and weighted values in
// place, without first gathering the sequence into one buffer.
//
// Design (one GPU, HBM-bound: every K/V byte is read exactly once):
//  * Work item = (split, kv head, sequence), one CTA each.  A split is a run
//    of `partition` tokens (a multiple of 32); sequences longer than that are
//    cut into several splits whose partial results a second kernel merges
//    with a log-sum-exp rescale.  Split boundaries depend only on logical
//    token positions, so the result is independent of where the blocks sit
//    in the pool and bit-identical from run to run (no atomics).
//  * Sequences are taken longest first: every CTA's prologue ranks the
//    batch's lengths into 64 length buckets (a counting sort) and maps its
//    blockIdx.z to the sequence of that rank, so the grid's tail holds the
//    short sequences.
//  * Warp 0 is the producer: the CTA's slice of the block table is staged
//    once into shared memory, and lane i of warp 0 copies tile i of each
//    32-token stage (one block, or block_size contiguous tokens) with the
//    TMA engine into a ring of `stages` shared-memory stages (K and V of 32
//    tokens each), so the copies of one stage are issued in parallel.  bf16
//    tiles use tiled copies (cp.async.bulk.tensor, 128-byte swizzle), fp32
//    tiles linear ones (cp.async.bulk).  A stage gathers 32 / block_size
//    physical blocks into one contiguous 32-token tile, so the math never
//    depends on block_size.  Full/empty mbarriers hand stages to the
//    consumers and back; every wait is bounded.
//  * Warps 1..2 are consumers.  Stage j goes to consumer warp j % 2, which
//    keeps its own fp32 online-softmax state (running max m, running sum l,
//    output accumulator o) for all G = Hq / Hkv query heads of the kv head:
//    every K and V element loaded from shared memory is used by all G heads.
//    bf16 runs the contractions on the tensor cores (decode_pass1_mma_kernel,
//    described there); fp32 on the CUDA cores (decode_pass1_kernel): a group
//    of TPT lanes owns one token row (16 bytes per lane), so shared-memory
//    reads are conflict-free row segments, and the q.k partial sums are
//    reduced across the TPT lanes with shuffles.
//  * At the end the warps' states are merged (shuffles, then shared memory),
//    and the CTA writes either the final row (one split) or its normalised
//    partial row plus (m, l) for the merge kernel.
//  * Scores are kept in the log2 domain (scale * log2(e) folded in) and
//    exponentials are exp2.
//  * Tokens past the sequence end are masked to -inf and their V rows are
//    never multiplied (stale shared memory may hold anything, NaN included).
//  * Pass 1 and the merge are launched with programmatic stream
//    serialisation and wait (griddepcontrol.wait) before touching global
//    memory, so they can be scheduled while the previous kernel drains.  In
//    the shared-prefix call's prefix-last order a chain of such waits lets
//    two kernels read the call's inputs earlier: a grid starts only after
//    every CTA of the kernel before it has signalled, and each signals after
//    its own wait, so pass 1 (after the set-up kernel) and the prefix pass
//    (after pass 1) find the inputs final; each waits only for its
//    predecessor's results (the prefix lengths; pass 1's partial rows).
//
// The contiguous-cache variant is the same kernel: only the producer's source
// address differs (one bulk copy per 32-token stage instead of one per block).
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>
#include <math.h>
#include <stdint.h>

#include <atomic>
#include <mutex>

#include "pa.h"
#include "pa_device.cuh"
#include "pa_internal.h"
#include "pa_tc.cuh"
#include "pa_timeline.cuh"

namespace pa {
namespace {

constexpr int kConsumerWarps = 2;
constexpr int kDecodeThreads = 32 * (1 + kConsumerWarps);
constexpr int kStageTokens = 32;
constexpr int kMaxPartition = 8192;
constexpr int kMinAutoPartition = 512;
constexpr int kMaxAutoPartition = 4096;
constexpr int kCtasPerSmEstimate = 6;  // resident pass-1 CTAs per SM (34 KB of shared memory each)
constexpr int kLongestFirstMaxBatch = 2048;  // O(batch) per CTA for the launch order
constexpr int kRingTargetBytes = 32 * 1024;
constexpr int kMaxDynamicSmem = 200 * 1024;
constexpr float kLog2e = 1.4426950408889634f;

struct DecodeParams {
    const void* q;
    const void* k;  // pool [NB, Hkv, bs, D] or contiguous cache [B, Hkv, L_pad, D]
    const void* v;
    const int32_t* block_tables;
    const int32_t* context_lens;
    void* out;
    float* part_o;   // [B, Hq, max_splits, D]
    float* part_ml;  // [B, Hq, max_splits, 2] = (m in log2 units, l)
    int* err;
    int64_t num_blocks;
    int64_t L_pad;
    int64_t max_len;  // max_context_len: longer sequences are clamped and flagged
    int max_blocks_per_seq;
    int num_q_heads;
    int num_kv_heads;
    int block_size;
    int partition;
    int max_splits;
    int stages;
    int ring_offset;
    int out_bf16;
    int contiguous;
    int batch;
    int longest_first;  // blockIdx.z is a rank in decreasing-length order
    float scale_log2;
    // decode step with the new token's cache write folded in (bf16 only):
    // token b is position context_lens[b] - 1 of sequence b; its K and V rows
    // k_new / v_new [batch][Hkv][D] go to the pool slot and into the staged
    // tile of the CTA that owns that position; slots (optional) receives the
    // slot of each token
    const void* k_new;
    const void* v_new;
    int64_t* slots;
    int append;
    // shared-prefix calls: pass 1 has room after its ring for the one prefix
    // partial it folds into a row (G rows of D floats, then their (m, l))
    int fold_prefetch;
    // bf16 paged pass 1: block-table entries of the window that CTA (split,
    // kvh, b) loads at its start, before it knows the sequence's length and
    // prefix length: entries split * partition / block_size onwards, enough
    // for any prefix up to max_prefix plus one partition (0: load the slice
    // once the length is known)
    int table_window;
    // shared-prefix calls with one prefix split and one own split, head_dim
    // 128: a set-up kernel checks the groups and writes seq_prefix, pass 1
    // runs next and stores each own part's partial in slot 1, and the
    // tensor-core prefix pass runs last, beside pass 1's tail, and finishes
    // every row (its own state folded with slot 1).  done_count counts the
    // prefix pass's finished CTAs.
    int prefix_last;
    int* done_count;
    // shared-prefix decode: sequences [group_starts[g], group_starts[g + 1])
    // share their first group_prefix[g] tokens (whole blocks, the same
    // physical ids in every member's table).  The prefix pass attends each
    // group's shared tokens once for all its members' queries and stores each
    // member's prefix length in seq_prefix; pass 1 then covers only tokens
    // [seq_prefix[b], L) of sequence b.  Partial-result slot s of a row holds
    // prefix split s for s < ceil(prefix / prefix_partition), then the
    // suffix splits.  seq_prefix == nullptr: no sharing.
    const int32_t* group_starts;
    const int32_t* group_prefix;
    int32_t* seq_prefix;
    int num_groups;
    int max_group;
    int max_prefix;
    int prefix_partition;
};

template <typename T>
struct Elt;

template <>
struct Elt<float> {
    static constexpr int VEC = 4;  // elements per 16-byte lane vector
    __device__ __forceinline__ static void unpack(const uint4& r, float* f) {
        f[0] = __uint_as_float(r.x);
        f[1] = __uint_as_float(r.y);
        f[2] = __uint_as_float(r.z);
        f[3] = __uint_as_float(r.w);
    }
};

template <>
struct Elt<__nv_bfloat16> {
    static constexpr int VEC = 8;
    __device__ __forceinline__ static void unpack(const uint4& r, float* f) {
        // bf16 -> fp32 is exact: the 16 bits become the high half of the word.
        f[0] = __uint_as_float(r.x << 16);
        f[1] = __uint_as_float(r.x & 0xffff0000u);
        f[2] = __uint_as_float(r.y << 16);
        f[3] = __uint_as_float(r.y & 0xffff0000u);
        f[4] = __uint_as_float(r.z << 16);
        f[5] = __uint_as_float(r.z & 0xffff0000u);
        f[6] = __uint_as_float(r.w << 16);
        f[7] = __uint_as_float(r.w & 0xffff0000u);
    }
};

__device__ __forceinline__ int clamp_len_value(const DecodeParams& p, int L, bool report) {
    if (L < 0 || (int64_t)L > p.max_len) {
        if (report) record_error(p.err, PA_ERR_BAD_BLOCK_ID);
        L = L < 0 ? 0 : (int)p.max_len;
    }
    return L;
}

__device__ __forceinline__ int clamp_len(const DecodeParams& p, int b, bool report) {
    int L = p.context_lens[b];
    if (L < 0 || (int64_t)L > p.max_len) {
        if (report) record_error(p.err, PA_ERR_BAD_BLOCK_ID);
        L = L < 0 ? 0 : (int)p.max_len;
    }
    return L;
}

// Leading tokens of sequence b that the prefix pass covered (0 without
// shared prefixes), clamped to [0, min(L, max_prefix)] and to whole blocks, so
// that a value left unwritten under a violated precondition can never send
// pass 1 or the merge outside the table or the partial-result slots.
__device__ __forceinline__ int clamp_prefix(const DecodeParams& p, int v, int L) {
    if (!p.seq_prefix) return 0;
    const int hi = L < p.max_prefix ? L : p.max_prefix;
    v = v < 0 ? 0 : (v > hi ? hi : v);
    return v - v % p.block_size;
}

__device__ __forceinline__ int seq_prefix_len(const DecodeParams& p, int b, int L) {
    return p.seq_prefix ? clamp_prefix(p, p.seq_prefix[b], L) : 0;
}

// Partial-result slots of sequence b (prefix splits, then suffix splits; at
// least one suffix split, empty when the prefix covers the whole sequence),
// and the number of prefix splits before the suffix's first slot.
__device__ __forceinline__ int row_splits(const DecodeParams& p, int L, int pre, int* prefix_splits) {
    const int sp = pre > 0 ? (pre + p.prefix_partition - 1) / p.prefix_partition : 0;
    const int nsuf = L > pre ? (L - pre + p.partition - 1) / p.partition : 1;
    *prefix_splits = sp;
    return sp + nsuf;
}

__device__ __forceinline__ void store_out(const DecodeParams& p, int64_t idx, float v) {
    if (p.out_bf16)
        static_cast<__nv_bfloat16*>(p.out)[idx] = __float2bfloat16_rn(v);
    else
        static_cast<float*>(p.out)[idx] = v;
}

// Output elements idx .. idx + 3 (idx a multiple of 4): one vector store when
// the output buffer is aligned for it (the caller's buffer need not be).
__device__ __forceinline__ void store_out4(const DecodeParams& p, int64_t idx, float4 v) {
    const uintptr_t base = reinterpret_cast<uintptr_t>(p.out);
    if (p.out_bf16 && (base & 7u) == 0)
        *reinterpret_cast<uint2*>(static_cast<__nv_bfloat16*>(p.out) + idx) =
            make_uint2(pack_bf16x2(v.x, v.y), pack_bf16x2(v.z, v.w));
    else if (!p.out_bf16 && (base & 15u) == 0)
        *reinterpret_cast<float4*>(static_cast<float*>(p.out) + idx) = v;
    else {
        store_out(p, idx, v.x);
        store_out(p, idx + 1, v.y);
        store_out(p, idx + 2, v.z);
        store_out(p, idx + 3, v.w);
    }
}

// Prefix splits that pass 1 folds into a row itself (more are left to the
// merge pass).
constexpr int kMaxFoldSplits = 16;

// Shared scratch of the epilogue merge, per query head: one factor per
// consumer warp's accumulator, then one per prefix split folded in.
constexpr int kCoefStride = kConsumerWarps + kMaxFoldSplits;

// Combine the consumer warps' (m, l, o) states of one work item, held in
// shared memory as o[w][h][d], m[w][h], l[w][h], and write the final row (one
// split) or the normalised partial row plus (m, l) for the merge kernel.
// First one thread per row turns the row's maxima and sums into one factor
// per warp (and per folded prefix split), then every output element is a
// short dot product of the warps' (and splits') values with those factors.
// With prefix splits and one own split (`fold`), the row is finished here:
// the prefix pass's partials (complete before this grid started) are
// combined with the CTA's own state by the log-sum-exp rescale the merge
// pass applies.  `pf` (one prefix split only): that split's partial already
// copied into shared memory as G rows of D floats followed by the rows'
// (m, l).  `coef` is shared scratch of G * kCoefStride floats.
__device__ __forceinline__ void merge_warps_and_store(const DecodeParams& p, const float* sm_o, const float* sm_m,
                                                      const float* sm_l, float* coef, int G, int D, int b, int kvh,
                                                      int split, int num_splits_b, int prefix_splits = 0,
                                                      bool fold = false, const float* pf = nullptr) {
    const int sp = (fold && prefix_splits > 0 && prefix_splits <= kMaxFoldSplits && num_splits_b == prefix_splits + 1)
                       ? prefix_splits
                       : 0;
    const bool final_row = num_splits_b == 1 || sp > 0;
    for (int h = threadIdx.x; h < G; h += blockDim.x) {
        const int64_t qrow = (int64_t)b * p.num_q_heads + (int64_t)kvh * G + h;
        float* c = coef + h * kCoefStride;
        float M = -INFINITY;
#pragma unroll
        for (int w = 0; w < kConsumerWarps; ++w) M = fmaxf(M, sm_m[w * G + h]);
        float a[kConsumerWarps], lt = 0.f;
#pragma unroll
        for (int w = 0; w < kConsumerWarps; ++w) {
            const float mw = sm_m[w * G + h];
            a[w] = mw == -INFINITY ? 0.f : exp2f(mw - M);
            lt += sm_l[w * G + h] * a[w];
        }
        if (sp == 0) {
            const float inv = lt > 0.f ? 1.f / lt : 0.f;
#pragma unroll
            for (int w = 0; w < kConsumerWarps; ++w) c[w] = a[w] * inv;
            if (!final_row) {
                const int64_t r = qrow * p.max_splits + split;
                p.part_ml[2 * r] = M;
                p.part_ml[2 * r + 1] = lt;
            }
        } else {
            const float* ml = pf ? pf + G * D + 2 * h : p.part_ml + qrow * p.max_splits * 2;
            float Mt = M;
            for (int s = 0; s < sp; ++s) Mt = fmaxf(Mt, ml[2 * s]);
            const float own = M == -INFINITY ? 0.f : exp2f(M - Mt);
            float W = lt * own;
            for (int s = 0; s < sp; ++s) {
                const float ms = ml[2 * s];
                const float ws = ms == -INFINITY ? 0.f : ml[2 * s + 1] * exp2f(ms - Mt);
                c[kConsumerWarps + s] = ws;
                W += ws;
            }
            const float inv = W > 0.f ? 1.f / W : 0.f;
#pragma unroll
            for (int w = 0; w < kConsumerWarps; ++w) c[w] = a[w] * own * inv;
            for (int s = 0; s < sp; ++s) c[kConsumerWarps + s] *= inv;
        }
    }
    __syncthreads();
    // four consecutive elements of a row per thread step (D is a multiple of
    // 4, rows start 16-byte aligned in every array)
    for (int idx = 4 * threadIdx.x; idx < G * D; idx += 4 * blockDim.x) {
        const int h = idx / D;
        const int d = idx - h * D;
        const int64_t qrow = (int64_t)b * p.num_q_heads + (int64_t)kvh * G + h;
        const float* c = coef + h * kCoefStride;
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
        for (int w = 0; w < kConsumerWarps; ++w) {
            const float4 o = *reinterpret_cast<const float4*>(sm_o + (w * G + h) * D + d);
            const float cw = c[w];
            acc.x = fmaf(o.x, cw, acc.x);
            acc.y = fmaf(o.y, cw, acc.y);
            acc.z = fmaf(o.z, cw, acc.z);
            acc.w = fmaf(o.w, cw, acc.w);
        }
        if (sp > 0) {
            const float* po = pf ? pf + h * D + d : p.part_o + qrow * p.max_splits * D + d;
            // four splits' loads in flight at a time
            for (int s0 = 0; s0 < sp; s0 += 4) {
                float4 v[4];
#pragma unroll
                for (int u = 0; u < 4; ++u)
                    v[u] = s0 + u < sp ? *reinterpret_cast<const float4*>(po + (int64_t)(s0 + u) * D)
                                       : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
                for (int u = 0; u < 4; ++u)
                    if (s0 + u < sp) {
                        const float cs = c[kConsumerWarps + s0 + u];
                        acc.x = fmaf(cs, v[u].x, acc.x);
                        acc.y = fmaf(cs, v[u].y, acc.y);
                        acc.z = fmaf(cs, v[u].z, acc.z);
                        acc.w = fmaf(cs, v[u].w, acc.w);
                    }
            }
        }
        if (final_row)
            store_out4(p, qrow * D + d, acc);
        else
            *reinterpret_cast<float4*>(p.part_o + (qrow * p.max_splits + split) * D + d) = acc;
    }
}

// Longest-first launch order.  The hardware dispatches CTAs in the order of
// their linear index, so the grid's z coordinate is used as a rank: the CTA
// works on the sequence with that rank when sequences are ordered by
// decreasing length (64 length buckets, ties by index).  This is
// longest-processing-time-first list scheduling; it keeps the tail of the
// grid short when lengths vary.  All threads read each length once into a
// shared-memory key and a bucket histogram; then one warp scans the histogram,
// finds the bucket holding the CTA's rank and the rank's position in it, and
// picks the sequence at that position among the bucket's members in index
// order with ballots, 32 keys at a time.  Only this CTA's sequence is
// selected (every CTA computes the same order, so the mapping is a
// bijection).  `scratch` is shared memory that is free at this point (at
// least 512 + batch bytes).  With longest_first == 0 the rank is the sequence
// index.
__device__ __forceinline__ int schedule_sequence(const DecodeParams& p, uint8_t* scratch) {
    const int rank = blockIdx.z;
    if (!p.longest_first) return rank;
    __shared__ int s_seq;
    int* hist = reinterpret_cast<int*>(scratch);  // [64]
    uint8_t* key = scratch + 512;                 // [batch]
    const int tid = threadIdx.x;
    for (int k = tid; k < 64; k += blockDim.x) hist[k] = 0;
    if (tid == 0) s_seq = rank;
    __syncthreads();
    // the loads of four sequences per thread are issued before any is used:
    // one memory round trip for batches up to four times the block size
    constexpr int U = 4;
    for (int b0 = tid; b0 < p.batch; b0 += U * blockDim.x) {
        int lv[U], pv[U];
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int b = b0 + u * blockDim.x;
            lv[u] = b < p.batch ? p.context_lens[b] : 0;
            pv[u] = (b < p.batch && p.seq_prefix) ? p.seq_prefix[b] : 0;
        }
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int b = b0 + u * blockDim.x;
            if (b >= p.batch) break;
            int L = lv[u];
            L = L < 0 ? 0 : ((int64_t)L > p.max_len ? (int)p.max_len : L);
            L -= clamp_prefix(p, pv[u], L);  // the tokens this pass reads
            int k = (int)(((int64_t)L * 64) / (p.max_len + 1));
            k = 63 - (k > 63 ? 63 : k);  // longer sequences get lower keys
            key[b] = (uint8_t)k;
            atomicAdd(&hist[k], 1);
        }
    }
    __syncthreads();
    if (tid < 32) {
        const int lane = tid;
        const int a0 = hist[2 * lane], a1 = hist[2 * lane + 1];
        int incl = a0 + a1;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, incl, off);
            if (lane >= off) incl += y;
        }
        const int excl = incl - a0 - a1;
        // the bucket holding this rank (the lane owning it broadcasts the
        // bucket and the rank's position inside it), then that position's
        // sequence among the bucket's members in index order, 32 at a time
        const bool in0 = rank >= excl && rank < excl + a0;
        const bool in1 = rank >= excl + a0 && rank < incl;
        const unsigned owner = __ballot_sync(0xffffffffu, in0 || in1);
        const int src = owner ? __ffs(owner) - 1 : 0;
        const int kb = __shfl_sync(0xffffffffu, in0 ? 2 * lane : 2 * lane + 1, src);
        int pos = rank - __shfl_sync(0xffffffffu, in0 ? excl : excl + a0, src);
        for (int c = 0; owner && c < p.batch; c += 32) {
            const int b = c + lane;
            const unsigned m = __ballot_sync(0xffffffffu, b < p.batch && key[b] == kb);
            const int cnt = __popc(m);
            if (pos < cnt) {
                if (((m >> lane) & 1u) && __popc(m & ((1u << lane) - 1u)) == pos) s_seq = b;
                break;
            }
            pos -= cnt;
        }
    }
    __syncthreads();
    return s_seq;
}

template <typename T, int D, int G>
__global__ void __launch_bounds__(kDecodeThreads) decode_pass1_kernel(const DecodeParams p) {
    using E = Elt<T>;
    constexpr int VEC = E::VEC;
    constexpr int TPT = D / VEC;             // lanes per token row
    constexpr int NG = 32 / TPT;             // token groups per warp
    constexpr int PASSES = kStageTokens / NG;  // rows per lane per stage
    constexpr int PCH = PASSES < 32 / G ? PASSES : 32 / G;  // rows per softmax update
    constexpr int NCH = PASSES / PCH;
    constexpr int ROW_BYTES = D * (int)sizeof(T);
    constexpr int STAGE_BYTES = kStageTokens * ROW_BYTES;  // K (or V) part of one stage
    static_assert(TPT >= 1 && TPT <= 32 && NG * TPT == 32, "lane layout");
    static_assert(PASSES % PCH == 0, "chunking");

    extern __shared__ __align__(1024) uint8_t smem[];
    uint64_t* full = reinterpret_cast<uint64_t*>(smem);
    uint64_t* empty = full + p.stages;
    int32_t* tbl = reinterpret_cast<int32_t*>(empty + p.stages);
    uint8_t* ring = smem + p.ring_offset;
    __shared__ int s_abort;

    griddep_wait();  // q, lengths, tables and the pool may come from the kernel before
    griddep_launch_dependents();
    const int split = blockIdx.x;
    const int kvh = blockIdx.y;
    const int b = schedule_sequence(p, ring);
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    const int L = clamp_len(p, b, threadIdx.x == 0 && split == 0 && kvh == 0);
    const int tok_begin = split * p.partition;
    if (split > 0 && tok_begin >= L) return;  // uniform over the CTA, before any barrier
    const int ntok = max(0, min(L, tok_begin + p.partition) - tok_begin);
    const int nstage = (ntok + kStageTokens - 1) / kStageTokens;
    const int num_splits_b = L > 0 ? (L + p.partition - 1) / p.partition : 1;

    if (threadIdx.x == 0) {
        s_abort = 0;
        for (int s = 0; s < p.stages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        fence_barrier_init();
    }
    if (!p.contiguous) {
        const int first_blk = tok_begin / p.block_size;
        const int nblk = (ntok + p.block_size - 1) / p.block_size;
        const int32_t* row = p.block_tables + (int64_t)b * p.max_blocks_per_seq + first_blk;
        for (int i = threadIdx.x; i < nblk; i += blockDim.x) tbl[i] = row[i];
    }
    __syncthreads();

    // per-consumer-lane softmax state (unused by the producer warp)
    float o[G][VEC];
    float m[G], l[G];
#pragma unroll
    for (int h = 0; h < G; ++h) {
        m[h] = -INFINITY;
        l[h] = 0.f;
#pragma unroll
        for (int v = 0; v < VEC; ++v) o[h][v] = 0.f;
    }
    const int grp = lane / TPT;
    const int sub = lane % TPT;

    if (warp == 0) {
        // ---------------- producer ----------------
        // Lane i issues the bulk copies of tile i of the stage (tile = one
        // block of block_size tokens, or the same number of tokens of the
        // contiguous cache), so the copies of a stage are issued in parallel.
        const uint64_t policy = l2_policy_evict_first();
        const char* kbase = static_cast<const char*>(p.k);
        const char* vbase = static_cast<const char*>(p.v);
        const int bs = p.block_size;
        const int tiles = kStageTokens / bs;
        for (int j = 0; j < nstage; ++j) {
            const int slot = j % p.stages;
            if (j >= p.stages) {
                int ok = 1;
                if (lane == 0) ok = mbar_wait(&empty[slot], ((j / p.stages) - 1) & 1, p.err);
                if (!__shfl_sync(0xffffffffu, ok, 0)) {
                    if (lane == 0) s_abort = 1;
                    break;
                }
            }
            uint8_t* kdst = ring + (size_t)slot * 2 * STAGE_BYTES;
            uint8_t* vdst = kdst + STAGE_BYTES;
            const int t0 = j * kStageTokens;
            const int rows = min(kStageTokens, ntok - t0);
            const int r = lane * bs;
            uint32_t nbytes = 0;
            int64_t off = 0;
            if (lane < tiles && r < rows) {
                nbytes = (uint32_t)min(bs, rows - r) * ROW_BYTES;
                if (p.contiguous) {
                    off = (((int64_t)b * p.num_kv_heads + kvh) * p.L_pad + tok_begin + t0 + r) * (int64_t)ROW_BYTES;
                } else {
                    const int32_t phys = tbl[(t0 + r) / bs];
                    if (phys < 0 || phys >= p.num_blocks) {
                        record_error(p.err, PA_ERR_BAD_BLOCK_ID);
                        nbytes = 0;
                    } else {
                        off = ((int64_t)phys * p.num_kv_heads + kvh) * bs * (int64_t)ROW_BYTES;
                    }
                }
            }
            const uint32_t total = __reduce_add_sync(0xffffffffu, nbytes);
            if (lane == 0) mbar_arrive_expect_tx(&full[slot], 2 * total);
            __syncwarp();
            if (nbytes) {
                bulk_load(kdst + r * ROW_BYTES, kbase + off, nbytes, &full[slot], policy);
                bulk_load(vdst + r * ROW_BYTES, vbase + off, nbytes, &full[slot], policy);
            }
        }
    } else {
        // ---------------- consumers ----------------
        const int cw = warp - 1;
        float qf[G][VEC];
        {
            const T* qrow = static_cast<const T*>(p.q) + ((int64_t)b * p.num_q_heads + (int64_t)kvh * G) * D;
#pragma unroll
            for (int h = 0; h < G; ++h) {
                const uint4 raw = *reinterpret_cast<const uint4*>(qrow + h * D + sub * VEC);
                E::unpack(raw, qf[h]);
#pragma unroll
                for (int v = 0; v < VEC; ++v) qf[h][v] *= p.scale_log2;
            }
        }
        for (int j = cw; j < nstage; j += kConsumerWarps) {
            const int slot = j % p.stages;
            if (!mbar_wait(&full[slot], (j / p.stages) & 1, p.err)) {
                s_abort = 1;
                break;
            }
            const T* ks = reinterpret_cast<const T*>(ring + (size_t)slot * 2 * STAGE_BYTES);
            const T* vs = ks + kStageTokens * D;
            const int valid = min(kStageTokens, ntok - j * kStageTokens);
#pragma unroll
            for (int c = 0; c < NCH; ++c) {
                float s[PCH][G];
#pragma unroll
                for (int pp = 0; pp < PCH; ++pp) {
                    const int t = (c * PCH + pp) * NG + grp;
                    const uint4 raw = *reinterpret_cast<const uint4*>(ks + t * D + sub * VEC);
                    float kf[VEC];
                    E::unpack(raw, kf);
#pragma unroll
                    for (int h = 0; h < G; ++h) {
                        float acc = 0.f;
#pragma unroll
                        for (int v = 0; v < VEC; ++v) acc = fmaf(qf[h][v], kf[v], acc);
                        s[pp][h] = acc;
                    }
                }
#pragma unroll
                for (int off = TPT / 2; off >= 1; off >>= 1) {
#pragma unroll
                    for (int pp = 0; pp < PCH; ++pp)
#pragma unroll
                        for (int h = 0; h < G; ++h) s[pp][h] += __shfl_xor_sync(0xffffffffu, s[pp][h], off);
                }
#pragma unroll
                for (int h = 0; h < G; ++h) {
                    float mx = -INFINITY;
#pragma unroll
                    for (int pp = 0; pp < PCH; ++pp) {
                        const int t = (c * PCH + pp) * NG + grp;
                        if (t >= valid) s[pp][h] = -INFINITY;
                        mx = fmaxf(mx, s[pp][h]);
                    }
                    const float m_new = fmaxf(m[h], mx);
                    if (m_new == -INFINITY) {
#pragma unroll
                        for (int pp = 0; pp < PCH; ++pp) s[pp][h] = 0.f;
                        continue;
                    }
                    const float alpha = exp2f(m[h] - m_new);
                    m[h] = m_new;
                    l[h] *= alpha;
#pragma unroll
                    for (int v = 0; v < VEC; ++v) o[h][v] *= alpha;
#pragma unroll
                    for (int pp = 0; pp < PCH; ++pp) {
                        s[pp][h] = exp2f(s[pp][h] - m_new);
                        l[h] += s[pp][h];
                    }
                }
#pragma unroll
                for (int pp = 0; pp < PCH; ++pp) {
                    const int t = (c * PCH + pp) * NG + grp;
                    if (t < valid) {
                        const uint4 raw = *reinterpret_cast<const uint4*>(vs + t * D + sub * VEC);
                        float vf[VEC];
                        E::unpack(raw, vf);
#pragma unroll
                        for (int h = 0; h < G; ++h)
#pragma unroll
                            for (int v = 0; v < VEC; ++v) o[h][v] = fmaf(s[pp][h], vf[v], o[h][v]);
                    }
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[slot]);
        }
        // merge the token groups of this warp
#pragma unroll
        for (int off = TPT; off < 32; off <<= 1) {
#pragma unroll
            for (int h = 0; h < G; ++h) {
                const float mo = __shfl_xor_sync(0xffffffffu, m[h], off);
                const float lo = __shfl_xor_sync(0xffffffffu, l[h], off);
                const float mn = fmaxf(m[h], mo);
                const float a = m[h] == -INFINITY ? 0.f : exp2f(m[h] - mn);
                const float a2 = mo == -INFINITY ? 0.f : exp2f(mo - mn);
                l[h] = l[h] * a + lo * a2;
#pragma unroll
                for (int v = 0; v < VEC; ++v) {
                    const float ov = __shfl_xor_sync(0xffffffffu, o[h][v], off);
                    o[h][v] = o[h][v] * a + ov * a2;
                }
                m[h] = mn;
            }
        }
    }
    __syncthreads();  // pipeline drained: the ring is free for the merge scratch
    if (s_abort) return;

    float* sm_o = reinterpret_cast<float*>(ring);    // [warps][G][D]
    float* sm_m = sm_o + kConsumerWarps * G * D;      // [warps][G]
    float* sm_l = sm_m + kConsumerWarps * G;          // [warps][G]
    if (warp > 0 && grp == 0) {
        const int cw = warp - 1;
#pragma unroll
        for (int h = 0; h < G; ++h) {
#pragma unroll
            for (int v = 0; v < VEC; ++v) sm_o[(cw * G + h) * D + sub * VEC + v] = o[h][v];
            if (sub == 0) {
                sm_m[cw * G + h] = m[h];
                sm_l[cw * G + h] = l[h];
            }
        }
    }
    __syncthreads();
    merge_warps_and_store(p, sm_o, sm_m, sm_l, sm_l + kConsumerWarps * G, G, D, b, kvh, split, num_splits_b);
}

// ---------------------------------------------------------------------------
// bf16 pass 1 on the tensor cores.
//
// Same work decomposition, ring and producer/consumer roles as the kernel
// above, with two differences:
//  * K/V tiles are staged by tiled TMA (cp.async.bulk.tensor, 2-D tensor map
//    over the pool viewed as [rows, head_dim]) with the 128-byte swizzle: a
//    stage holds, per 64-element column slab, 32 token rows of 128 bytes in
//    which 16-byte chunk c of row r sits at chunk c ^ (r & 7).  ldmatrix of 8
//    token rows then touches 8 different bank groups.
//  * The consumer warp does the two contractions with mma.sync m16n8k16
//    (bf16 in, fp32 accumulate), tokens on the M side and the G query heads of
//    the kv head on the N side:
//        S^T[tokens, heads] = K[tokens, D] . Q^T[D, heads]
//        O^T[D, heads]     += V^T[D, tokens] . P^T[tokens, heads]
//    P^T comes from the S^T accumulator transposed in registers (movmatrix);
//    P is split into a bf16 high part and a bf16 residual, both multiplied by
//    V, so the weights keep ~16 significant bits instead of 8.
// G <= 8 uses one 8-wide N tile (NT = 1), G == 16 two.
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t swizzled(uint32_t slab, int row, int chunk) {
    return slab + row * 128 + ((chunk ^ (row & 7)) << 4);
}

template <int D, int NT>
__global__ void __launch_bounds__(kDecodeThreads)
    decode_pass1_mma_kernel(const DecodeParams p, const __grid_constant__ CUtensorMap tmk,
                            const __grid_constant__ CUtensorMap tmv) {
    constexpr int SLABS = D / 64;
    constexpr int SLAB_BYTES = kStageTokens * 128;
    constexpr int STAGE_BYTES = SLABS * SLAB_BYTES;  // K (or V) part of one stage
    constexpr int KSTEPS = D / 16;

    extern __shared__ __align__(1024) uint8_t smem[];
    uint64_t* full = reinterpret_cast<uint64_t*>(smem);
    uint64_t* empty = full + p.stages;
    int32_t* const tbl_base = reinterpret_cast<int32_t*>(empty + p.stages);
    // the 128-byte swizzle pattern assumes 1024-byte aligned slabs: align the
    // ring at run time (the launch reserves 1 KB of slack for this)
    uint8_t* ring = smem + p.ring_offset + ((1024u - (smem_addr(smem) & 1023u)) & 1023u);
    __shared__ int s_abort;

    if (threadIdx.x == 0) {
        PA_TL(2, 0);
        prefetch_tmap(&tmk);
        prefetch_tmap(&tmv);
    }
    // q, lengths, tables and the pool may come from the kernel before.  In the
    // prefix-last order that kernel is the set-up kernel, which waited for the
    // kernels before the call before this grid could start: only its own
    // result (the prefix length) needs the wait, taken below, after the
    // prologue's other loads are in flight.
    if (!p.prefix_last) {
        griddep_wait();
        griddep_launch_dependents();
    }
    const int split = blockIdx.x;
    const int kvh = blockIdx.y;
    const int b = schedule_sequence(p, ring);
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int G = p.num_q_heads / p.num_kv_heads;

    // the length, the prefix length and the block-table window, loaded together
    const int len_raw = p.context_lens[b];
    constexpr int TW = 4;  // window entries per thread in flight
    const int win0 = (int)(((int64_t)split * p.partition) / p.block_size);
    const int nwin = (p.contiguous || !p.table_window) ? 0 : max(0, min(p.table_window, p.max_blocks_per_seq - win0));
    const int32_t* wrow = p.block_tables + (int64_t)b * p.max_blocks_per_seq + win0;
    int32_t tw[TW];
#pragma unroll
    for (int u = 0; u < TW; ++u) {
        const int i = threadIdx.x + u * kDecodeThreads;
        tw[u] = i < nwin ? wrow[i] : 0;
    }
    if (p.prefix_last) {
        griddep_wait();
        griddep_launch_dependents();  // after the wait: the prefix pass relies on the set-up kernel's counter
    }
    const int pre_raw = p.seq_prefix ? p.seq_prefix[b] : 0;
    const int L = clamp_len_value(p, len_raw, threadIdx.x == 0 && split == 0 && kvh == 0);
    // A length beyond max_context_len is clamped for the attention (and
    // flagged), but the folded write still goes to the slot of the length as
    // given, where pa_reshape_and_cache_decode puts it: split 0 writes it
    // directly, outside the (clamped) range any CTA of this launch reads.
    const bool overflow = p.append && len_raw > p.max_len;
    if (p.append && !overflow && L == 0 && split == 0 && kvh == 0 && threadIdx.x == 0 && p.slots) p.slots[b] = -1;
    // with shared prefixes this pass covers the tokens after the sequence's
    // prefix, and its splits' partial results follow the prefix splits' slots
    const int pre = clamp_prefix(p, pre_raw, L);
    const int tok_begin = pre + split * p.partition;
    if (split > 0 && tok_begin >= L) return;
    const int ntok = max(0, min(L, tok_begin + p.partition) - tok_begin);
    const int nstage = (ntok + kStageTokens - 1) / kStageTokens;
    int prefix_splits;
    const int num_splits_b = row_splits(p, L, pre, &prefix_splits);
    // one prefix split to fold in: its partial is copied to shared memory
    // (after the ring) while the last stages are consumed
    float* pf = (p.fold_prefetch && prefix_splits == 1 && num_splits_b == 2)
                    ? reinterpret_cast<float*>(ring + (size_t)p.stages * 2 * STAGE_BYTES)
                    : nullptr;

    if (threadIdx.x == 0) {
        s_abort = 0;
        for (int s = 0; s < p.stages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        fence_barrier_init();
    }
    // the block ids of the split's tokens: from the window loaded above (the
    // slice starts pre / block_size entries into it), or loaded now
    int32_t* tbl = tbl_base;
    if (nwin) {
#pragma unroll
        for (int u = 0; u < TW; ++u) {
            const int i = threadIdx.x + u * kDecodeThreads;
            if (i < nwin) tbl_base[i] = tw[u];
        }
        for (int i = threadIdx.x + TW * kDecodeThreads; i < nwin; i += kDecodeThreads) tbl_base[i] = wrow[i];
        tbl = tbl_base + (tok_begin / p.block_size - win0);
    } else if (!p.contiguous) {
        const int first_blk = tok_begin / p.block_size;
        const int nblk = (ntok + p.block_size - 1) / p.block_size;
        const int32_t* row = p.block_tables + (int64_t)b * p.max_blocks_per_seq + first_blk;
        for (int i = threadIdx.x; i < nblk; i += blockDim.x) tbl[i] = row[i];
    }
    __syncthreads();
    if (threadIdx.x == 0) PA_TL(2, 1);

    if (overflow && split == 0 && warp == 1) {
        const int pos = p.context_lens[b] - 1;
        int32_t phys = -1;
        if (pos / p.block_size < p.max_blocks_per_seq)
            phys = p.block_tables[(int64_t)b * p.max_blocks_per_seq + pos / p.block_size];
        if (phys >= 0 && phys < p.num_blocks && lane < D / 8) {
            const int64_t src = ((int64_t)b * p.num_kv_heads + kvh) * (D / 8) + lane;
            const int64_t dst =
                (((int64_t)phys * p.num_kv_heads + kvh) * p.block_size + pos % p.block_size) * (D / 8) + lane;
            static_cast<uint4*>(const_cast<void*>(p.k))[dst] = static_cast<const uint4*>(p.k_new)[src];
            static_cast<uint4*>(const_cast<void*>(p.v))[dst] = static_cast<const uint4*>(p.v_new)[src];
        }
        if (lane == 0 && kvh == 0 && p.slots)
            p.slots[b] = phys >= 0 ? (int64_t)phys * p.block_size + pos % p.block_size : -1;
    }

    const int g = lane >> 2;  // fragment row group
    const int t = lane & 3;   // fragment column pair
    float o[KSTEPS][NT][4];
    float m[NT][2], l[NT][2];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
#pragma unroll
        for (int i = 0; i < 2; ++i) {
            m[nt][i] = -INFINITY;
            l[nt][i] = 0.f;
        }
#pragma unroll
        for (int mt = 0; mt < KSTEPS; ++mt)
#pragma unroll
            for (int c = 0; c < 4; ++c) o[mt][nt][c] = 0.f;
    }

    if (warp == 0) {
        // ---------------- producer ----------------
        // Lane i loads tile i of the stage (block_size rows) for every column
        // slab of K and V; the box is always block_size full rows.
        const uint64_t policy = l2_policy_evict_first();
        const int bs = p.block_size;
        const int tiles = kStageTokens / bs;
        const uint32_t tile_bytes = (uint32_t)(SLABS * bs * 128);
        for (int j = 0; j < nstage; ++j) {
            const int slot = j % p.stages;
            if (j >= p.stages) {
                int ok = 1;
                if (lane == 0) ok = mbar_wait(&empty[slot], ((j / p.stages) - 1) & 1, p.err);
                if (!__shfl_sync(0xffffffffu, ok, 0)) {
                    if (lane == 0) s_abort = 1;
                    break;
                }
            }
            uint8_t* kdst = ring + (size_t)slot * 2 * STAGE_BYTES;
            uint8_t* vdst = kdst + STAGE_BYTES;
            const int t0 = j * kStageTokens;
            const int rows = min(kStageTokens, ntok - t0);
            const int r = lane * bs;
            int y = 0;
            uint32_t nbytes = 0;
            if (lane < tiles && r < rows) {
                nbytes = tile_bytes;
                if (p.contiguous) {
                    y = (int)(((int64_t)b * p.num_kv_heads + kvh) * p.L_pad + tok_begin + t0 + r);
                } else {
                    const int32_t phys = tbl[(t0 + r) / bs];
                    if (phys < 0 || phys >= p.num_blocks) {
                        record_error(p.err, PA_ERR_BAD_BLOCK_ID);
                        nbytes = 0;
                    } else {
                        y = (phys * p.num_kv_heads + kvh) * bs;
                    }
                }
            }
            const uint32_t total = __reduce_add_sync(0xffffffffu, nbytes);
            if (lane == 0) mbar_arrive_expect_tx(&full[slot], 2 * total);
            __syncwarp();
            if (nbytes) {
#pragma unroll
                for (int sl = 0; sl < SLABS; ++sl) {
                    tma_load_2d(kdst + sl * SLAB_BYTES + r * 128, &tmk, sl * 64, y, &full[slot], policy);
                    tma_load_2d(vdst + sl * SLAB_BYTES + r * 128, &tmv, sl * 64, y, &full[slot], policy);
                }
            }
        }
        if (pf) {
            // the prefix partial (complete before this grid started): rows of
            // the G heads, four float4 per lane in flight, then their (m, l)
            const int64_t qrow0 = (int64_t)b * p.num_q_heads + (int64_t)kvh * G;
            const int nv = G * D / 4;
            for (int i0 = lane; i0 < nv; i0 += 4 * 32) {
                float4 v[4];
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const int i = i0 + 32 * u;
                    if (i < nv)
                        v[u] = *reinterpret_cast<const float4*>(p.part_o + (qrow0 + i / (D / 4)) * p.max_splits * D +
                                                                (i % (D / 4)) * 4);
                }
#pragma unroll
                for (int u = 0; u < 4; ++u)
                    if (i0 + 32 * u < nv) reinterpret_cast<float4*>(pf)[i0 + 32 * u] = v[u];
            }
            if (lane < 2 * G) pf[G * D + lane] = p.part_ml[(qrow0 + lane / 2) * p.max_splits * 2 + (lane & 1)];
        }
    } else {
        // ---------------- consumers ----------------
        const int cw = warp - 1;
        // Q^T fragments (k = head_dim, n = query head of the group), bf16 pairs
        uint32_t qb[NT][KSTEPS][2];
        {
            const uint16_t* qbase = static_cast<const uint16_t*>(p.q) +
                                    ((int64_t)b * p.num_q_heads + (int64_t)kvh * G) * D;
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
                const int head = nt * 8 + g;
#pragma unroll
                for (int kk = 0; kk < KSTEPS; ++kk) {
                    if (head < G) {
                        qb[nt][kk][0] = *reinterpret_cast<const uint32_t*>(qbase + head * D + kk * 16 + 2 * t);
                        qb[nt][kk][1] = *reinterpret_cast<const uint32_t*>(qbase + head * D + kk * 16 + 8 + 2 * t);
                    } else {
                        qb[nt][kk][0] = qb[nt][kk][1] = 0u;
                    }
                }
            }
        }
        const int q4 = lane >> 3;  // which of the four ldmatrix matrices this lane addresses
        const int r8 = lane & 7;   // which row of it
        // a folded-in cache write: the warp that takes the last stage of the
        // sequence's last split loads the new K and V rows now, so their
        // latency is hidden behind the stream (lane c holds 16-byte chunk c)
        const bool appends = p.append && !overflow && nstage > 0 && split == num_splits_b - prefix_splits - 1 &&
                             (nstage - 1) % kConsumerWarps == cw;
        uint4 new_k = make_uint4(0u, 0u, 0u, 0u), new_v = new_k;
        if (appends && lane < D / 8) {
            const int64_t src = ((int64_t)b * p.num_kv_heads + kvh) * (D / 8) + lane;
            new_k = static_cast<const uint4*>(p.k_new)[src];
            new_v = static_cast<const uint4*>(p.v_new)[src];
        }
        for (int j = cw; j < nstage; j += kConsumerWarps) {
            const int slot = j % p.stages;
            if (!mbar_wait(&full[slot], (j / p.stages) & 1, p.err)) {
                s_abort = 1;
                break;
            }
            if (threadIdx.x == 32 && j == 0) PA_TL(2, 3);
            uint8_t* kstage = ring + (size_t)slot * 2 * STAGE_BYTES;
            uint8_t* vstage = kstage + STAGE_BYTES;
            const uint32_t kst = smem_addr(kstage);
            const uint32_t vst = smem_addr(vstage);
            const int valid = min(kStageTokens, ntok - j * kStageTokens);
            if (valid < kStageTokens) {
                // rows past the sequence end may hold anything (NaN included):
                // zero them so that 0-weight * V stays 0 in the MMA
                const int nchunks = (kStageTokens - valid) * SLABS * 8;
                for (int c = lane; c < nchunks; c += 32) {
                    const int row = valid + c / (SLABS * 8);
                    const int rem = c % (SLABS * 8);
                    *reinterpret_cast<uint4*>(vstage + (rem >> 3) * SLAB_BYTES + row * 128 + (rem & 7) * 16) =
                        make_uint4(0u, 0u, 0u, 0u);
                }
                fence_proxy_async_smem();  // the slot is refilled by TMA later
                __syncwarp();
            }
            if (appends && j == nstage - 1) {
                // the appended token is the stage's last valid row: its K and V
                // rows (loaded at the start) go into the staged tile, whatever
                // the copy brought from the slot, and into the pool slot itself
                const int r = valid - 1;
                const int pos = L - 1;
                const int32_t phys = tbl[(pos - tok_begin) / p.block_size];
                const bool in_pool = phys >= 0 && phys < p.num_blocks;
                const int64_t dst = (((int64_t)phys * p.num_kv_heads + kvh) * p.block_size + pos % p.block_size) * (D / 8);
                if (lane < D / 8) {
                    const int c = lane;
                    const int off = (c >> 3) * SLAB_BYTES + r * 128 + (((c & 7) ^ (r & 7)) << 4);
                    *reinterpret_cast<uint4*>(kstage + off) = new_k;
                    *reinterpret_cast<uint4*>(vstage + off) = new_v;
                    if (in_pool) {
                        static_cast<uint4*>(const_cast<void*>(p.k))[dst + c] = new_k;
                        static_cast<uint4*>(const_cast<void*>(p.v))[dst + c] = new_v;
                    }
                }
                if (lane == 0 && kvh == 0 && p.slots)
                    p.slots[b] = phys >= 0 ? (int64_t)phys * p.block_size + pos % p.block_size : -1;
                fence_proxy_async_smem();
                __syncwarp();
            }
            // S^T = K . Q^T : two 16-token M tiles
            float s[2][NT][4];
#pragma unroll
            for (int mt = 0; mt < 2; ++mt)
#pragma unroll
                for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                    for (int c = 0; c < 4; ++c) s[mt][nt][c] = 0.f;
#pragma unroll
            for (int kk = 0; kk < KSTEPS; ++kk) {
                const uint32_t slab = kst + (kk >> 2) * SLAB_BYTES;
                const int chunk = (kk & 3) * 2 + (q4 >> 1);
#pragma unroll
                for (int mt = 0; mt < 2; ++mt) {
                    uint32_t a[4];
                    ldmatrix_x4(swizzled(slab, 16 * mt + r8 + 8 * (q4 & 1), chunk), a[0], a[1], a[2], a[3]);
#pragma unroll
                    for (int nt = 0; nt < NT; ++nt) mma_bf16_16816(s[mt][nt], a, qb[nt][kk][0], qb[nt][kk][1]);
                }
            }
            // online softmax, one column (query head) at a time; this lane holds
            // tokens g, g + 8, 16 + g, 24 + g of columns 8 nt + 2 t + i
            bool rescale = false;
            float alpha[NT][2];
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
#pragma unroll
                for (int i = 0; i < 2; ++i) {
                    float v[4] = {s[0][nt][i], s[0][nt][2 + i], s[1][nt][i], s[1][nt][2 + i]};
                    float mx = -INFINITY;
#pragma unroll
                    for (int k = 0; k < 4; ++k) {
                        const int tok = 16 * (k >> 1) + g + 8 * (k & 1);
                        v[k] = tok < valid ? v[k] * p.scale_log2 : -INFINITY;
                        mx = fmaxf(mx, v[k]);
                    }
                    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 4));
                    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 8));
                    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 16));
                    const float m_new = fmaxf(m[nt][i], mx);
                    float a = 1.f;
                    if (m_new == -INFINITY) {
#pragma unroll
                        for (int k = 0; k < 4; ++k) v[k] = 0.f;
                    } else {
                        a = exp2f(m[nt][i] - m_new);
                        float sum = 0.f;
#pragma unroll
                        for (int k = 0; k < 4; ++k) {
                            v[k] = exp2f(v[k] - m_new);
                            sum += v[k];
                        }
                        l[nt][i] = l[nt][i] * a + sum;
                        m[nt][i] = m_new;
                    }
                    alpha[nt][i] = a;
                    rescale |= a != 1.f;
                    s[0][nt][i] = v[0];
                    s[0][nt][2 + i] = v[1];
                    s[1][nt][i] = v[2];
                    s[1][nt][2 + i] = v[3];
                }
            }
            if (__any_sync(0xffffffffu, rescale)) {
#pragma unroll
                for (int mt = 0; mt < KSTEPS; ++mt)
#pragma unroll
                    for (int nt = 0; nt < NT; ++nt) {
                        o[mt][nt][0] *= alpha[nt][0];
                        o[mt][nt][1] *= alpha[nt][1];
                        o[mt][nt][2] *= alpha[nt][0];
                        o[mt][nt][3] *= alpha[nt][1];
                    }
            }
            // O^T += V^T . P^T, one 16-token K step per S^T M tile
#pragma unroll
            for (int ks = 0; ks < 2; ++ks) {
                uint32_t bh[NT][2], bl[NT][2];
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) {
#pragma unroll
                    for (int half = 0; half < 2; ++half) {
                        const float p0 = s[ks][nt][2 * half], p1 = s[ks][nt][2 * half + 1];
                        const uint32_t hi = pack_bf16x2(p0, p1);
                        const uint32_t lo = pack_bf16x2(p0 - bf16_lo_to_f32(hi), p1 - bf16_hi_to_f32(hi));
                        bh[nt][half] = movmatrix_trans(hi);
                        bl[nt][half] = movmatrix_trans(lo);
                    }
                }
                // two row tiles at a time: both high-part MMAs, then both
                // residual ones, so no MMA waits on the one just issued into
                // the same accumulator
#pragma unroll
                for (int mp = 0; mp < KSTEPS; mp += 2) {
                    uint32_t a[2][4];
#pragma unroll
                    for (int u = 0; u < 2; ++u) {
                        const int mt = mp + u;
                        const uint32_t slab = vst + (mt >> 2) * SLAB_BYTES;
                        const int chunk = (mt & 3) * 2 + (q4 & 1);
                        ldmatrix_x4_trans(swizzled(slab, 16 * ks + r8 + 8 * (q4 >> 1), chunk), a[u][0], a[u][1],
                                          a[u][2], a[u][3]);
                    }
#pragma unroll
                    for (int nt = 0; nt < NT; ++nt) {
                        mma_bf16_16816(o[mp][nt], a[0], bh[nt][0], bh[nt][1]);
                        mma_bf16_16816(o[mp + 1][nt], a[1], bh[nt][0], bh[nt][1]);
                        mma_bf16_16816(o[mp][nt], a[0], bl[nt][0], bl[nt][1]);
                        mma_bf16_16816(o[mp + 1][nt], a[1], bl[nt][0], bl[nt][1]);
                    }
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[slot]);
        }
        // l was summed per lane over its own tokens: add the 8 lanes of a column
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int i = 0; i < 2; ++i) {
                l[nt][i] += __shfl_xor_sync(0xffffffffu, l[nt][i], 4);
                l[nt][i] += __shfl_xor_sync(0xffffffffu, l[nt][i], 8);
                l[nt][i] += __shfl_xor_sync(0xffffffffu, l[nt][i], 16);
            }
    }
    __syncthreads();  // pipeline drained: the ring is free for the merge scratch
    if (threadIdx.x == 0) PA_TL(2, 4);
    if (s_abort) return;

    float* sm_o = reinterpret_cast<float*>(ring);  // [warps][G][D]
    float* sm_m = sm_o + kConsumerWarps * G * D;    // [warps][G]
    float* sm_l = sm_m + kConsumerWarps * G;        // [warps][G]
    if (warp > 0) {
        const int cw = warp - 1;
#pragma unroll
        for (int mt = 0; mt < KSTEPS; ++mt)
#pragma unroll
            for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    const int head = nt * 8 + 2 * t + (c & 1);
                    const int dim = 16 * mt + g + 8 * (c >> 1);
                    if (head < G) sm_o[(cw * G + head) * D + dim] = o[mt][nt][c];
                }
        if (g == 0) {
#pragma unroll
            for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                for (int i = 0; i < 2; ++i) {
                    const int head = nt * 8 + 2 * t + i;
                    if (head < G) {
                        sm_m[cw * G + head] = m[nt][i];
                        sm_l[cw * G + head] = l[nt][i];
                    }
                }
        }
    }
    __syncthreads();
    merge_warps_and_store(p, sm_o, sm_m, sm_l, sm_l + kConsumerWarps * G, G, D, b, kvh, prefix_splits + split,
                          num_splits_b, prefix_splits, !p.prefix_last, pf);
    if (threadIdx.x == 0) PA_TL(2, 2);
}

// ---------------------------------------------------------------------------
// Shared-prefix pass (bf16, tensor cores).
//
// Parallel samples of one prompt share the prompt's blocks by reference count
// ("PagedAttention and KV memory management", "Key takeaways"; "Paged
// Attention: OS-Inspired Memory Management for KV Caches", "Key terms in this
// lesson", Reference count).  Per-sequence attention reads those blocks once
// per sample.  This pass reads them once per group instead: a CTA owns
// (prefix split, kv head x row chunk, group), streams the split's K/V tiles
// through the same TMA ring as pass 1, and computes them against the queries
// of every member of the group at once, so each shared K/V element in shared
// memory is used by n * G query rows.
//  * Query rows r = member * G + head are the M side of mma.sync m16n8k16:
//        S[rows, tokens] = Q[rows, D] . K^T[D, tokens]
//        O[rows, D]     += P[rows, tokens] . V[tokens, D]
//    P goes from the S accumulators straight into A fragments (the two
//    layouts coincide), split into bf16 high and residual parts as in pass 1.
//  * The CTA's 16 MT query rows are staged once in shared memory (128-byte
//    swizzle, read by ldmatrix), which keeps registers for two CTAs' worth of
//    latency hiding.  Consumer warp (tile t, parity q) owns rows 16 t ..
//    16 t + 15 and the stages j with j % PAR == q: PAR groups of MT warps
//    work on alternate stages, and at the end each group's (m, l, o) is
//    combined with the others' through shared memory (same lane layout, so
//    lane by lane).  Larger groups take several row chunks (blockIdx.y / Hkv).
//  * The first consumer group writes its rows' normalised partial and (m, l)
//    to the prefix split's slot for pass 1 (which folds them into the row) or
//    the merge pass.  CTA (0, 0, g) also checks the group's description and
//    stores each member's prefix length in seq_prefix; a description that
//    breaks the preconditions is flagged and its group falls back to prefix 0
//    (pass 1 then covers the whole sequences).
// ---------------------------------------------------------------------------
__device__ __forceinline__ void consumer_barrier(int id, int threads) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(threads) : "memory");
}

// A shared-prefix group as the prefix passes use it: first member, member
// count and the prefix length it can share (0 when it cannot).
struct PrefixGroup {
    int start;
    int n;
    int prefix;
};

// Group grp's description as given (one thread): its span, its prefix length
// if the description keeps the rules that need no member's length (else 0
// and `bad`).  A well-formed span gets its members' prefix lengths written in
// any case (0 when the group cannot share); a malformed one names no
// members, and the sequences it should have covered stay unspecified.  The
// reporter CTA flags groups that do not cover the batch.
__device__ __forceinline__ void prefix_group_describe(const DecodeParams& p, int grp, bool reporter, int& start,
                                                      int& n, int& prefix, int& bad) {
    const int s = p.group_starts[grp], e = p.group_starts[grp + 1], P = p.group_prefix[grp];
    const bool span_ok = s >= 0 && e >= s && e <= p.batch;
    const bool ok = span_ok && e - s <= p.max_group && P >= 0 && P <= p.max_prefix && P % p.block_size == 0;
    start = span_ok ? s : 0;
    n = span_ok ? e - s : 0;
    prefix = ok ? P : 0;
    bad = !ok;
    if (reporter && ((grp == 0 && s != 0) || (grp == p.num_groups - 1 && e != p.batch)))
        record_error(p.err, PA_ERR_BAD_BLOCK_ID);  // the groups do not cover the batch
}

// The outcome, once every member's length has been checked against the
// prefix (`bad` set by any member shorter than it): the reporter CTA flags a
// bad description and writes each member's prefix length to seq_prefix.
// Called by all threads, after a barrier that follows the checks.
__device__ __forceinline__ PrefixGroup prefix_group_outcome(const DecodeParams& p, bool reporter, int start, int n,
                                                            int prefix, int bad) {
    const PrefixGroup g{start, n, bad ? 0 : prefix};
    if (reporter) {
        if (threadIdx.x == 0 && bad) record_error(p.err, PA_ERR_BAD_BLOCK_ID);
        for (int m = threadIdx.x; m < g.n; m += blockDim.x) p.seq_prefix[g.start + m] = g.prefix;
    }
    return g;
}

// Check group grp's description; every CTA of the group reaches the same
// outcome.  Called by all threads.
__device__ PrefixGroup prefix_group_setup(const DecodeParams& p, int grp, bool reporter) {
    __shared__ int s_start, s_n, s_prefix, s_bad;
    if (threadIdx.x == 0) prefix_group_describe(p, grp, reporter, s_start, s_n, s_prefix, s_bad);
    __syncthreads();
    for (int m = threadIdx.x; m < s_n; m += blockDim.x)
        if (clamp_len(p, s_start + m, false) < s_prefix) s_bad = 1;  // a member shorter than the prefix
    __syncthreads();
    return prefix_group_outcome(p, reporter, s_start, s_n, s_prefix, s_bad);
}

// Prefix-last order: the groups' descriptions, checked once per call before
// pass 1 (one CTA).  Every sequence's prefix length in seq_prefix starts at 0;
// then each member of a well-formed group gets the group's prefix length.  A
// description that breaks the preconditions is flagged, and its sequences
// keep prefix 0 (attended without sharing).  The rules are those of
// prefix_group_describe and prefix_group_setup, so the prefix pass reaches
// the same outcome on its own.  Also clears the prefix pass's exit counter.
__global__ void __launch_bounds__(1024) decode_prefix_setup_kernel(const DecodeParams p) {
    if (threadIdx.x == 0) PA_TL(0, 0);
    griddep_wait();  // lengths and descriptions may come from the kernel before
    griddep_launch_dependents();
    if (threadIdx.x == 0) PA_TL(0, 1);
    for (int b = threadIdx.x; b < p.batch; b += blockDim.x) p.seq_prefix[b] = 0;
    if (threadIdx.x == 0) *p.done_count = 0;
    __syncthreads();
    for (int g = threadIdx.x; g < p.num_groups; g += blockDim.x) {
        int start, n, P, bad;
        prefix_group_describe(p, g, true, start, n, P, bad);
        for (int m0 = start; !bad && m0 < start + n; m0 += 8) {
            // a member shorter than the prefix (eight lengths in flight)
            int Lm[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) Lm[u] = m0 + u < start + n ? clamp_len(p, m0 + u, false) : P;
#pragma unroll
            for (int u = 0; u < 8; ++u) bad |= Lm[u] < P;
        }
        if (bad) {
            record_error(p.err, PA_ERR_BAD_BLOCK_ID);
            continue;
        }
        for (int m = start; m < start + n; ++m) p.seq_prefix[m] = P;
    }
    if (threadIdx.x == 0) PA_TL(0, 2);
}

template <int D, int MT, int PAR>
__global__ void __launch_bounds__(32 * (1 + MT * PAR), 3)
    decode_prefix_mma_kernel(const DecodeParams p, const __grid_constant__ CUtensorMap tmk,
                             const __grid_constant__ CUtensorMap tmv) {
    constexpr int SLABS = D / 64;
    constexpr int SLAB_BYTES = kStageTokens * 128;
    constexpr int STAGE_BYTES = SLABS * SLAB_BYTES;
    constexpr int KSTEPS = D / 16;
    constexpr int NTD = D / 8;  // 8-column tiles of the output row
    constexpr int ROWS = 16 * MT;
    constexpr int QSLAB = ROWS * 128;  // bytes of one 64-column slab of the Q tile
    constexpr int CONSUMERS = 32 * MT * PAR;

    extern __shared__ __align__(1024) uint8_t smem[];
    uint64_t* full = reinterpret_cast<uint64_t*>(smem);
    uint64_t* empty = full + p.stages;
    int32_t* tbl = reinterpret_cast<int32_t*>(empty + p.stages);
    uint8_t* ring = smem + p.ring_offset + ((1024u - (smem_addr(smem) & 1023u)) & 1023u);
    uint8_t* qtile = ring + (size_t)p.stages * 2 * STAGE_BYTES;  // [SLABS][ROWS][128 B], swizzled
    if (threadIdx.x == 0) {
        prefetch_tmap(&tmk);
        prefetch_tmap(&tmv);
    }
    griddep_wait();  // q, lengths, tables and the pool may come from the kernel before
    griddep_launch_dependents();
    const int split = blockIdx.x;
    const int kvh = blockIdx.y % p.num_kv_heads;
    const int chunk = blockIdx.y / p.num_kv_heads;
    const int grp = blockIdx.z;
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int G = p.num_q_heads / p.num_kv_heads;
    const PrefixGroup pgrp = prefix_group_setup(p, grp, split == 0 && blockIdx.y == 0);
    const int s_start = pgrp.start;
    const int n = pgrp.n;
    const int P = pgrp.prefix;
    const int tok_begin = split * p.prefix_partition;
    const int rows_total = n * G;
    const int row0 = chunk * ROWS;
    if (tok_begin >= P || row0 >= rows_total) return;  // uniform over the CTA, before any barrier
    const int ntok = min(P, tok_begin + p.prefix_partition) - tok_begin;
    const int nstage = (ntok + kStageTokens - 1) / kStageTokens;

    if (threadIdx.x == 0) {
        for (int s = 0; s < p.stages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], MT);
        }
        fence_barrier_init();
    }
    {
        // the shared blocks, from the first member's table
        const int first_blk = tok_begin / p.block_size;
        const int nblk = (ntok + p.block_size - 1) / p.block_size;
        const int32_t* row = p.block_tables + (int64_t)s_start * p.max_blocks_per_seq + first_blk;
        for (int i = threadIdx.x; i < nblk; i += blockDim.x) tbl[i] = row[i];
        // the chunk's query rows (zero past the group), 16-byte chunk c of
        // row r of a slab at chunk c ^ (r & 7)
        const uint16_t* qv = static_cast<const uint16_t*>(p.q);
        for (int i = threadIdx.x; i < ROWS * (D / 8); i += blockDim.x) {
            const int r = i / (D / 8);
            const int c = i % (D / 8);
            const int gr = row0 + r;
            uint4 v = make_uint4(0u, 0u, 0u, 0u);
            if (gr < rows_total)
                v = *reinterpret_cast<const uint4*>(
                    qv + ((int64_t)(s_start + gr / G) * p.num_q_heads + (int64_t)kvh * G + gr % G) * D + c * 8);
            *reinterpret_cast<uint4*>(qtile + (c >> 3) * QSLAB + r * 128 + (((c & 7) ^ (r & 7)) << 4)) = v;
        }
    }
    __syncthreads();

    if (warp == 0) {
        // ---------------- producer ----------------
        const uint64_t policy = l2_policy_evict_first();
        const int bs = p.block_size;
        const int tiles = kStageTokens / bs;
        const uint32_t tile_bytes = (uint32_t)(SLABS * bs * 128);
        for (int j = 0; j < nstage; ++j) {
            const int slot = j % p.stages;
            if (j >= p.stages) {
                int ok = 1;
                if (lane == 0) ok = mbar_wait(&empty[slot], ((j / p.stages) - 1) & 1, p.err);
                if (!__shfl_sync(0xffffffffu, ok, 0)) break;
            }
            uint8_t* kdst = ring + (size_t)slot * 2 * STAGE_BYTES;
            uint8_t* vdst = kdst + STAGE_BYTES;
            const int t0 = j * kStageTokens;
            const int rows = min(kStageTokens, ntok - t0);
            if (rows < kStageTokens) {
                // every consumer of this stage reads all its rows: the
                // producer zeroes the V rows past the prefix (0-weight * stale
                // NaN would be NaN)
                const int nchunks = (kStageTokens - rows) * SLABS * 8;
                for (int c = lane; c < nchunks; c += 32) {
                    const int row = rows + c / (SLABS * 8);
                    const int rem = c % (SLABS * 8);
                    *reinterpret_cast<uint4*>(vdst + (rem >> 3) * SLAB_BYTES + row * 128 + (rem & 7) * 16) =
                        make_uint4(0u, 0u, 0u, 0u);
                }
                fence_proxy_async_smem();
            }
            const int r = lane * bs;
            int y = 0;
            uint32_t nbytes = 0;
            if (lane < tiles && r < rows) {
                const int32_t phys = tbl[(t0 + r) / bs];
                if (phys < 0 || phys >= p.num_blocks) {
                    record_error(p.err, PA_ERR_BAD_BLOCK_ID);
                } else {
                    nbytes = tile_bytes;
                    y = (phys * p.num_kv_heads + kvh) * bs;
                }
            }
            const uint32_t total = __reduce_add_sync(0xffffffffu, nbytes);
            __syncwarp();
            if (lane == 0) mbar_arrive_expect_tx(&full[slot], 2 * total);
            __syncwarp();
            if (nbytes) {
#pragma unroll
                for (int sl = 0; sl < SLABS; ++sl) {
                    tma_load_2d(kdst + sl * SLAB_BYTES + r * 128, &tmk, sl * 64, y, &full[slot], policy);
                    tma_load_2d(vdst + sl * SLAB_BYTES + r * 128, &tmv, sl * 64, y, &full[slot], policy);
                }
            }
        }
        return;
    }

    // ---------------- consumers ----------------
    const int cw = warp - 1;
    const int mtile = cw % MT;  // 16-row tile of the chunk
    const int par = cw / MT;    // stages j with j % PAR == par
    const int g = lane >> 2;    // fragment row group
    const int t = lane & 3;     // fragment column pair
    const int q4 = lane >> 3;
    const int r8 = lane & 7;
    const int rbase = row0 + 16 * mtile;
    const uint32_t qbase = smem_addr(qtile);
    float o[NTD][4];
#pragma unroll
    for (int nd = 0; nd < NTD; ++nd)
#pragma unroll
        for (int c = 0; c < 4; ++c) o[nd][c] = 0.f;
    float m[2] = {-INFINITY, -INFINITY}, l[2] = {0.f, 0.f};
    bool aborted = false;
    for (int j = par; j < nstage; j += PAR) {
        const int slot = j % p.stages;
        if (!mbar_wait(&full[slot], (j / p.stages) & 1, p.err)) {
            aborted = true;
            break;
        }
        const uint32_t kst = smem_addr(ring + (size_t)slot * 2 * STAGE_BYTES);
        const uint32_t vst = kst + STAGE_BYTES;
        const int valid = min(kStageTokens, ntok - j * kStageTokens);
        // S = Q . K^T over the stage's 32 tokens: four 8-token column tiles;
        // the head dimension in two halves with their own accumulators, so
        // each MMA waits on the one eight issues back, not four
        float s[4][4], s2[4][4];
#pragma unroll
        for (int nt = 0; nt < 4; ++nt)
#pragma unroll
            for (int c = 0; c < 4; ++c) s[nt][c] = s2[nt][c] = 0.f;
#pragma unroll
        for (int kh = 0; kh < KSTEPS / 2; ++kh) {
            uint32_t a[2][4], b[2][2][4];
#pragma unroll
            for (int half = 0; half < 2; ++half) {
                const int kk = kh + half * (KSTEPS / 2);
                // Q rows 16 mtile + {0..15}, columns 16 kk .. 16 kk + 15
                ldmatrix_x4(swizzled(qbase + (kk >> 2) * QSLAB, 16 * mtile + r8 + 8 * (q4 & 1),
                                     (kk & 3) * 2 + (q4 >> 1)),
                            a[half][0], a[half][1], a[half][2], a[half][3]);
                const uint32_t slab = kst + (kk >> 2) * SLAB_BYTES;
                const int chunk16 = (kk & 3) * 2 + (q4 & 1);
#pragma unroll
                for (int pair = 0; pair < 2; ++pair)
                    ldmatrix_x4(swizzled(slab, 8 * (2 * pair + (q4 >> 1)) + r8, chunk16), b[half][pair][0],
                                b[half][pair][1], b[half][pair][2], b[half][pair][3]);
            }
#pragma unroll
            for (int pair = 0; pair < 2; ++pair) {
                mma_bf16_16816(s[2 * pair], a[0], b[0][pair][0], b[0][pair][1]);
                mma_bf16_16816(s[2 * pair + 1], a[0], b[0][pair][2], b[0][pair][3]);
                mma_bf16_16816(s2[2 * pair], a[1], b[1][pair][0], b[1][pair][1]);
                mma_bf16_16816(s2[2 * pair + 1], a[1], b[1][pair][2], b[1][pair][3]);
            }
        }
#pragma unroll
        for (int nt = 0; nt < 4; ++nt)
#pragma unroll
            for (int c = 0; c < 4; ++c) s[nt][c] += s2[nt][c];
        // online softmax per row (this lane: rows g and g + 8, tokens
        // 8 nt + 2 t and 8 nt + 2 t + 1), log2 domain, masked past the prefix
        float alpha[2];
        bool rescale = false;
#pragma unroll
        for (int i = 0; i < 2; ++i) {
            float mx = -INFINITY;
#pragma unroll
            for (int nt = 0; nt < 4; ++nt)
#pragma unroll
                for (int c = 0; c < 2; ++c) {
                    const int tok = 8 * nt + 2 * t + c;
                    const float v = tok < valid ? s[nt][2 * i + c] * p.scale_log2 : -INFINITY;
                    s[nt][2 * i + c] = v;
                    mx = fmaxf(mx, v);
                }
            mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
            mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
            const float m_new = fmaxf(m[i], mx);
            float a = 1.f;
            if (m_new == -INFINITY) {
#pragma unroll
                for (int nt = 0; nt < 4; ++nt) s[nt][2 * i] = s[nt][2 * i + 1] = 0.f;
            } else {
                a = exp2f(m[i] - m_new);
                float sum = 0.f;
#pragma unroll
                for (int nt = 0; nt < 4; ++nt)
#pragma unroll
                    for (int c = 0; c < 2; ++c) {
                        const float e = exp2f(s[nt][2 * i + c] - m_new);
                        s[nt][2 * i + c] = e;
                        sum += e;
                    }
                l[i] = l[i] * a + sum;
                m[i] = m_new;
            }
            alpha[i] = a;
            rescale |= a != 1.f;
        }
        if (__any_sync(0xffffffffu, rescale)) {
#pragma unroll
            for (int nd = 0; nd < NTD; ++nd) {
                o[nd][0] *= alpha[0];
                o[nd][1] *= alpha[0];
                o[nd][2] *= alpha[1];
                o[nd][3] *= alpha[1];
            }
        }
        // O += P . V, one 16-token K step per pair of S column tiles
#pragma unroll
        for (int ks = 0; ks < 2; ++ks) {
            uint32_t ah[4], al[4];
#pragma unroll
            for (int f = 0; f < 4; ++f) {
                // f = 0: row g, tile 2 ks; 1: row g + 8, tile 2 ks; 2, 3: tile 2 ks + 1
                const float p0 = s[2 * ks + (f >> 1)][2 * (f & 1)], p1 = s[2 * ks + (f >> 1)][2 * (f & 1) + 1];
                ah[f] = pack_bf16x2(p0, p1);
                al[f] = pack_bf16x2(p0 - bf16_lo_to_f32(ah[f]), p1 - bf16_hi_to_f32(ah[f]));
            }
            // four column-tile pairs at a time: their eight high-part MMAs,
            // then the eight residual ones, so no MMA waits on the one just
            // issued into the same accumulator
#pragma unroll
            for (int ng = 0; ng < NTD / 8; ++ng) {
                uint32_t b[4][4];
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const int nd = 2 * (4 * ng + u) + (q4 >> 1);
                    ldmatrix_x4_trans(swizzled(vst + (nd >> 3) * SLAB_BYTES, 16 * ks + 8 * (q4 & 1) + r8, nd & 7),
                                      b[u][0], b[u][1], b[u][2], b[u][3]);
                }
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    mma_bf16_16816(o[2 * (4 * ng + u)], ah, b[u][0], b[u][1]);
                    mma_bf16_16816(o[2 * (4 * ng + u) + 1], ah, b[u][2], b[u][3]);
                }
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    mma_bf16_16816(o[2 * (4 * ng + u)], al, b[u][0], b[u][1]);
                    mma_bf16_16816(o[2 * (4 * ng + u) + 1], al, b[u][2], b[u][3]);
                }
            }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[slot]);
    }
    if (PAR > 1) {
        // combine the parity groups lane by lane through the (drained) ring:
        // every consumer has finished its stages before anything is written
        consumer_barrier(1, CONSUMERS);
        constexpr int REC = NTD * 4 + 4;  // floats per lane: o, m[2], l[2]
        float* xch = reinterpret_cast<float*>(ring);
        if (par > 0) {
            float* dst = xch + ((size_t)((par - 1) * MT + mtile) * 32 + lane) * REC;
#pragma unroll
            for (int nd = 0; nd < NTD; ++nd)
#pragma unroll
                for (int c = 0; c < 4; ++c) dst[nd * 4 + c] = o[nd][c];
            dst[NTD * 4] = m[0];
            dst[NTD * 4 + 1] = m[1];
            dst[NTD * 4 + 2] = l[0];
            dst[NTD * 4 + 3] = l[1];
        }
        consumer_barrier(1, CONSUMERS);
        if (par > 0) return;
#pragma unroll
        for (int q = 1; q < PAR; ++q) {
            const float* src = xch + ((size_t)((q - 1) * MT + mtile) * 32 + lane) * REC;
            float a0[2], a1[2];
#pragma unroll
            for (int i = 0; i < 2; ++i) {
                const float mq = src[NTD * 4 + i];
                const float M = fmaxf(m[i], mq);
                a0[i] = m[i] == -INFINITY ? 0.f : exp2f(m[i] - M);
                a1[i] = mq == -INFINITY ? 0.f : exp2f(mq - M);
                l[i] = l[i] * a0[i] + src[NTD * 4 + 2 + i] * a1[i];
                m[i] = M;
            }
#pragma unroll
            for (int nd = 0; nd < NTD; ++nd)
#pragma unroll
                for (int c = 0; c < 4; ++c) o[nd][c] = o[nd][c] * a0[c >> 1] + src[nd * 4 + c] * a1[c >> 1];
        }
    }
    if (aborted) return;
    // l was summed per lane over its own columns: add the quad's four lanes
#pragma unroll
    for (int i = 0; i < 2; ++i) {
        l[i] += __shfl_xor_sync(0xffffffffu, l[i], 1);
        l[i] += __shfl_xor_sync(0xffffffffu, l[i], 2);
    }
#pragma unroll
    for (int i = 0; i < 2; ++i) {
        const int r = rbase + g + 8 * i;
        if (r >= rows_total) continue;
        const int64_t qrow = (int64_t)(s_start + r / G) * p.num_q_heads + (int64_t)kvh * G + r % G;
        const int64_t slotrow = qrow * p.max_splits + split;
        float* dst = p.part_o + slotrow * D + 2 * t;
#pragma unroll
        for (int nd = 0; nd < NTD; ++nd) {
            float2 v;
            v.x = l[i] > 0.f ? o[nd][2 * i] / l[i] : 0.f;
            v.y = l[i] > 0.f ? o[nd][2 * i + 1] / l[i] : 0.f;
            *reinterpret_cast<float2*>(dst + 8 * nd) = v;
        }
        if (t == 0) {
            p.part_ml[2 * slotrow] = m[i];
            p.part_ml[2 * slotrow + 1] = l[i];
        }
    }
}

// ---------------------------------------------------------------------------
// Shared-prefix pass on the 5th-generation tensor cores (head_dim 128).
//
// Same work item, inputs and outputs as the mma.sync pass above, with 32 query
// rows per CTA.  The shared tokens are the M side of tcgen05 MMAs, so one
// 128-token tile of K and V feeds all the rows at once:
//     S^T[tokens, rows] = K[tokens, D] . Q^T[D, rows]         (M = 128 tokens)
//     O^T[D, rows]     += V^T[D, tokens] . P^T[tokens, rows]  (M = D = 128)
// K is the A operand as it lands from TMA (K-major, 128-byte swizzle); V is the
// A operand read M-major from the same kind of tile; Q (staged once) and P are
// the B operands; S^T (double-buffered) and O^T live in tensor memory.
//  * warp 0 streams K and V tiles of 128 shared tokens (tiled TMA boxes of
//    block_size rows, one pool block per lane) into one K and one V buffer: K
//    of the next tile is requested as soon as S of this one is computed, V as
//    soon as its P.V is.  With one buffer each a CTA takes ~90 KB of shared
//    memory, so two run on an SM: one's start-up and epilogue overlap the
//    other's stream, and the GPU holds the whole grid of a typical call;
//  * warp 1 owns the tensor memory (allocated first thing: the SM starts a
//    second CTA of this kernel only once the first has given up its
//    allocation permit) and issues the MMAs from one thread: P_{j-1}.V_{j-1}
//    once the softmax has written P_{j-1}, then S_j;
//  * warps 2..5 (one per TMEM lane quarter) run the softmax: thread t holds
//    token t's scores for all 32 rows.  Every thread keeps the rows' running
//    maxima; they move only when a score exceeds them by more than 2^8
//    (found with one barrier reduction per tile), so most tiles need no
//    cross-thread max.  When they move, the tile's exact row maxima come
//    from a transposing shuffle reduction and O^T is rescaled in tensor
//    memory.  Each thread keeps partial row sums over its own tokens
//    (combined once at the end) and writes its token's row of P^T, as bf16
//    high and residual parts (M/N-major, 64-byte swizzle), for the next P.V;
//  * at the end they stage O^T through shared memory and write each row's
//    normalised partial (as float4 rows) and (m, l), as the mma.sync pass
//    does; in the prefix-last order (the pass launched after pass 1) they
//    instead wait for pass 1, fold its partial of each row's own tokens in
//    by the log-sum-exp rescale, and write the final rows.
// The group's check, the table slice and the query rows are fetched in one
// round trip before any of them is used.
// ---------------------------------------------------------------------------
// Prefix-last order: the prefix pass's grid must not complete before pass 1
// (kernels after the call wait for the prefix pass only).  CTAs with work wait
// for pass 1 before their epilogue; to cover a grid in which none has work,
// the last CTA to finish waits too.  One thread per CTA, at its exit.
__device__ __forceinline__ void prefix_last_exit(const DecodeParams& p) {
    if (!p.prefix_last) return;
    const unsigned total = gridDim.x * gridDim.y * gridDim.z;
    if (atomicAdd(reinterpret_cast<unsigned*>(p.done_count), 1u) == total - 1) griddep_wait();
}

constexpr int kTcTokens = 128;         // shared tokens per tile (M of S^T)
constexpr int kTcRows = 32;            // query rows per CTA (N of both MMAs)
constexpr int kTcThreads = 64 + 128;   // producer, MMA issuer, softmax warpgroup
constexpr float kTcRescaleLog2 = 8.f;  // lazy-rescale threshold of the running max (log2 units)
constexpr int kTcSlab = kTcTokens * 128;        // one 64-column slab of a K or V tile
constexpr int kTcTile = 2 * kTcSlab;            // a K or V tile of 128 tokens x 128 columns
constexpr int kTcQSlab = kTcRows * 128;         // one 64-column slab of the Q tile
constexpr int kTcPRow = kTcRows * 2;            // bytes of one token's row of P^T
constexpr int kTcPBytes = kTcTokens * kTcPRow;  // one part (high or residual) of P^T
constexpr uint32_t kTcTmemCols = 128;           // O^T in [0, 32), S^T buffers in [32, 96)
static_assert(kTcRows * kTcTokens * 4 <= kTcTile, "the epilogue stages O^T in the K buffer");

// Dynamic shared memory of the tensor-core prefix pass: the K and V buffers,
// P^T (high + residual), the Q tile, the reduction scratch and the split's
// block-table slice, after 1024-byte alignment.
inline size_t prefix_tc_smem_bytes(int table_entries) {
    return 1024 + 2 * (size_t)kTcTile + 2 * (size_t)kTcPBytes + 2 * (size_t)kTcQSlab + 4 * kTcRows * sizeof(float) +
           (size_t)table_entries * sizeof(int32_t);
}

// OR of a predicate over the 128 softmax threads (named barrier 1).
__device__ __forceinline__ bool softmax_any(bool v) {
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred pi, po;\n\tsetp.ne.u32 pi, %1, 0;\n\t"
        "bar.red.or.pred po, 1, 128, pi;\n\tselp.u32 %0, 1, 0, po;\n\t}"
        : "=r"(r)
        : "r"((uint32_t)v)
        : "memory");
    return r != 0;
}

// Reduce v[0..31] element-wise over the warp's 32 lanes so that lane i ends
// with the result for element i (max or sum): five exchange steps, each
// halving the elements a lane keeps, 31 shuffles in all.  Destroys v.
template <bool kMax>
__device__ __forceinline__ float warp_transpose_reduce(float (&v)[32], int lane) {
#pragma unroll
    for (int w = 16; w >= 1; w >>= 1) {
        const bool upper = (lane & w) != 0;
#pragma unroll
        for (int i = 0; i < w; ++i) {
            const float send = upper ? v[i] : v[i + w];
            const float keep = upper ? v[i + w] : v[i];
            const float recv = __shfl_xor_sync(0xffffffffu, send, w);
            v[i] = kMax ? fmaxf(keep, recv) : keep + recv;
        }
    }
    return v[0];
}

__global__ void __launch_bounds__(kTcThreads, 2)
    decode_prefix_tc_kernel(const DecodeParams p, const __grid_constant__ CUtensorMap tmk,
                            const __grid_constant__ CUtensorMap tmv) {
    constexpr int D = 128;
    constexpr int N = kTcRows;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* smem = smem_raw + ((1024u - (smem_addr(smem_raw) & 1023u)) & 1023u);
    uint8_t* sK = smem;                                        // K tile (the epilogue's O staging after)
    uint8_t* sV = sK + kTcTile;                                // V tile
    uint8_t* sP = sV + kTcTile;                                // P^T: high part, residual part
    uint8_t* sQ = sP + 2 * kTcPBytes;                          // [2 slabs][kTcQSlab]
    float* red = reinterpret_cast<float*>(sQ + 2 * kTcQSlab);  // [4 warps][N]
    int32_t* tbl = reinterpret_cast<int32_t*>(red + 4 * N);
    __shared__ uint64_t k_full, k_empty, v_full, v_empty, s_full[2], p_full, pv_done;
    __shared__ uint32_t tmem_base;
    __shared__ int64_t row_off[N];  // epilogue: element offset of row r's partial, or -1
    __shared__ float row_inv[N];    //           factor of the row's own O (1 / row sum)
    __shared__ float row_c1[N];     //           prefix-last order: factor of pass 1's partial
    __shared__ int64_t row_own[N];  //           prefix-last order: element offset of pass 1's partial

    if (threadIdx.x == 0) {
        PA_TL(1, 0);
        prefetch_tmap(&tmk);
        prefetch_tmap(&tmv);
    }
    // q, lengths, tables and the pool may come from the kernel before.  In the
    // prefix-last order that kernel is pass 1, which waited for the set-up
    // kernel (which waited for the kernels before the call) before this grid
    // could start: the inputs are final, and only pass 1's partial results,
    // read in the epilogue, need the wait, taken there.
    if (!p.prefix_last) griddep_wait();
    griddep_launch_dependents();
    const int split = blockIdx.x;
    const int kvh = blockIdx.y % p.num_kv_heads;
    const int chunk = blockIdx.y / p.num_kv_heads;
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int G = p.num_q_heads / p.num_kv_heads;
    // the set-up kernel reports (and writes seq_prefix) in the prefix-last order
    const bool reporter = !p.prefix_last && split == 0 && blockIdx.y == 0;
    // Tensor memory first: the SM schedules a second CTA of this kernel only
    // once the first has given up its allocation permit.
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_addr(&tmem_base)),
                     "r"(kTcTmemCols));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
    }
    __shared__ int d_start, d_n, d_prefix, d_bad;
    if (threadIdx.x == 0) prefix_group_describe(p, blockIdx.z, reporter, d_start, d_n, d_prefix, d_bad);
    __syncthreads();
    const int tok_begin = split * p.prefix_partition;
    const int row0 = chunk * N;
    {
        // One round trip for the rest of the prologue: the members' lengths
        // (the check of the prefix against them), and, for the group as
        // described, the split's slice of the shared blocks (from the first
        // member's table) and the chunk's query rows, staged K-major with the
        // 128-byte swizzle (16-byte chunk c of row r of a slab at c ^ (r & 7),
        // zero past the group).  All loads are issued before any is used.
        const int rows_d = d_n * G;
        const bool work = row0 < rows_d && tok_begin < d_prefix;
        const int nblk_d = work ? (min(d_prefix, tok_begin + p.prefix_partition) - tok_begin + p.block_size - 1) /
                                      p.block_size
                                : 0;
        const int32_t* row = p.block_tables + (int64_t)d_start * p.max_blocks_per_seq + tok_begin / p.block_size;
        const uint16_t* qv = static_cast<const uint16_t*>(p.q);
        constexpr int QV = (N * (D / 8) + kTcThreads - 1) / kTcThreads;  // 16-byte query chunks per thread
        uint4 qr[QV];
#pragma unroll
        for (int u = 0; u < QV; ++u) {
            const int i = threadIdx.x + u * kTcThreads;
            const int r = i / (D / 8);
            const int c = i % (D / 8);
            const int gr = row0 + r;
            qr[u] = make_uint4(0u, 0u, 0u, 0u);
            if (work && i < N * (D / 8) && gr < rows_d)
                qr[u] = *reinterpret_cast<const uint4*>(
                    qv + ((int64_t)(d_start + gr / G) * p.num_q_heads + (int64_t)kvh * G + gr % G) * D + c * 8);
        }
        int tv[2];
        for (int i0 = threadIdx.x; i0 < nblk_d; i0 += 2 * kTcThreads) {
#pragma unroll
            for (int u = 0; u < 2; ++u) tv[u] = i0 + u * kTcThreads < nblk_d ? row[i0 + u * kTcThreads] : 0;
#pragma unroll
            for (int u = 0; u < 2; ++u)
                if (i0 + u * kTcThreads < nblk_d) tbl[i0 + u * kTcThreads] = tv[u];
        }
        for (int m = threadIdx.x; m < d_n; m += kTcThreads)
            if (clamp_len(p, d_start + m, false) < d_prefix) d_bad = 1;  // a member shorter than the prefix
#pragma unroll
        for (int u = 0; u < QV; ++u) {
            const int i = threadIdx.x + u * kTcThreads;
            const int r = i / (D / 8);
            const int c = i % (D / 8);
            if (i < N * (D / 8))
                *reinterpret_cast<uint4*>(sQ + (c >> 3) * kTcQSlab + r * 128 + (((c & 7) ^ (r & 7)) << 4)) = qr[u];
        }
        fence_proxy_async_smem();  // the tensor core reads Q through the async proxy
    }
    if (threadIdx.x == 0) PA_TL(1, 1);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = tmem_base;
    const PrefixGroup grp = prefix_group_outcome(p, reporter, d_start, d_n, d_prefix, d_bad);
    const int rows_total = grp.n * G;
    if (tok_begin >= grp.prefix || row0 >= rows_total) {  // uniform over the CTA
        if (warp == 1) asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTcTmemCols));
        if (threadIdx.x == 0) prefix_last_exit(p);
        return;
    }
    const int ntok = min(grp.prefix, tok_begin + p.prefix_partition) - tok_begin;
    const int nt = (ntok + kTcTokens - 1) / kTcTokens;

    if (threadIdx.x == 0) {
        mbar_init(&k_full, 1);
        mbar_init(&k_empty, 1);
        mbar_init(&v_full, 1);
        mbar_init(&v_empty, 1);
        mbar_init(&s_full[0], 1);
        mbar_init(&s_full[1], 1);
        mbar_init(&p_full, 4);
        mbar_init(&pv_done, 1);
        fence_barrier_init();
    }
    __syncthreads();
    if (threadIdx.x == 0) PA_TL(1, 3);

    if (warp == 0) {
        // ---------------- producer ----------------
        const uint64_t policy = l2_policy_evict_first();
        const int bs = p.block_size;
        const int boxes = kTcTokens / bs;  // pool blocks per tile
        bool streamed = true;
        for (int j = 0; j < nt; ++j) {
            const int t0 = j * kTcTokens;
            const int valid = min(kTcTokens, ntok - t0);
            const int r = lane * bs;
            int y = 0;
            uint32_t nbytes = 0;
            if (lane < boxes && r < valid) {
                const int32_t phys = tbl[(t0 + r) / bs];
                if (phys < 0 || phys >= p.num_blocks) {
                    record_error(p.err, PA_ERR_BAD_BLOCK_ID);
                } else {
                    nbytes = (uint32_t)(2 * bs * 128);
                    y = (phys * p.num_kv_heads + kvh) * bs;
                }
            }
            const uint32_t total = __reduce_add_sync(0xffffffffu, nbytes);
            // K_j once S_{j-1} has read the K buffer
            if (j >= 1) {
                int ok = 1;
                if (lane == 0) ok = mbar_wait(&k_empty, (j - 1) & 1, p.err);
                if (!(streamed = __shfl_sync(0xffffffffu, ok, 0))) break;
            }
            if (lane == 0) {
                mbar_arrive_expect_tx(&k_full, total);
                PA_TT(j, 5);
            }
            __syncwarp();
            if (nbytes) {
                tma_load_2d(sK + r * 128, &tmk, 0, y, &k_full, policy);
                tma_load_2d(sK + kTcSlab + r * 128, &tmk, 64, y, &k_full, policy);
            }
            // V_j once P_{j-1}.V_{j-1} has read the V buffer
            if (j >= 1) {
                int ok = 1;
                if (lane == 0) ok = mbar_wait(&v_empty, (j - 1) & 1, p.err);
                if (!(streamed = __shfl_sync(0xffffffffu, ok, 0))) break;
            }
            if (valid < kTcTokens) {
                // the tile's tokens past the split carry weight 0, but 0 * NaN
                // is NaN in the MMA: zero those V rows (stale or never loaded)
                const int nch = (kTcTokens - valid) * 16;
                for (int c = lane; c < nch; c += 32) {
                    const int row = valid + c / 16;
                    const int rem = c % 16;
                    *reinterpret_cast<uint4*>(sV + (rem >> 3) * kTcSlab + row * 128 + (rem & 7) * 16) =
                        make_uint4(0u, 0u, 0u, 0u);
                }
                fence_proxy_async_smem();
                __syncwarp();
            }
            if (lane == 0) {
                mbar_arrive_expect_tx(&v_full, total);
                PA_TT(j, 6);
            }
            __syncwarp();
            if (nbytes) {
                tma_load_2d(sV + r * 128, &tmv, 0, y, &v_full, policy);
                tma_load_2d(sV + kTcSlab + r * 128, &tmv, 64, y, &v_full, policy);
            }
        }
        // the last tile's releases are tensor-core commits that land in this
        // CTA's shared memory: wait for them before the CTA may exit
        if (lane == 0 && streamed && mbar_wait(&k_empty, (nt - 1) & 1, p.err))
            mbar_wait(&v_empty, (nt - 1) & 1, p.err);
    } else if (warp == 1) {
        // ---------------- MMA issuer ----------------
        if (lane == 0) {
            constexpr uint32_t IDESC_S = umma_idesc(kTcTokens, N, false, false);
            constexpr uint32_t IDESC_O = umma_idesc(D, N, true, true);
            const uint32_t q_base = smem_addr(sQ);
            const uint32_t k_base = smem_addr(sK);
            const uint32_t v_base = smem_addr(sV);
            const uint32_t p_base = smem_addr(sP);
            for (int j = 0; j <= nt; ++j) {
                if (j >= 1) {
                    // O^T += V_{j-1}^T . P_{j-1}^T, high part then residual,
                    // 16 tokens per step
                    const int jp = j - 1;
                    if (!mbar_wait(&p_full, jp & 1, p.err)) break;
                    if (!mbar_wait(&v_full, jp & 1, p.err)) break;
                    tc_fence_after();
                    PA_TT(jp, 3);
#pragma unroll
                    for (int kk = 0; kk < kTcTokens / 16; ++kk) {
                        const uint64_t da = umma_desc(v_base + kk * 16 * 128, kTcSlab, 1024);
                        const uint32_t pk = p_base + kk * 16 * kTcPRow;
                        umma(tmem, da, umma_desc_sw(pk, kTcPBytes, 8 * kTcPRow, kUmmaSwizzle64), IDESC_O,
                             (jp > 0 || kk > 0) ? 1u : 0u);
                        umma(tmem, da, umma_desc_sw(pk + kTcPBytes, kTcPBytes, 8 * kTcPRow, kUmmaSwizzle64), IDESC_O,
                             1u);
                    }
                    umma_commit(&pv_done);
                    umma_commit(&v_empty);
                }
                if (j < nt) {
                    // S_j^T = K_j . Q^T into S buffer j & 1 (the softmax
                    // loaded S_{j-2} before it signalled P_{j-2})
                    if (!mbar_wait(&k_full, j & 1, p.err)) break;
                    tc_fence_after();
                    PA_TT(j, 4);
#pragma unroll
                    for (int kk = 0; kk < D / 16; ++kk) {
                        const uint32_t off = (kk >> 2) * kTcSlab + (kk & 3) * 32;
                        const uint32_t qoff = (kk >> 2) * kTcQSlab + (kk & 3) * 32;
                        umma(tmem + N + (j & 1) * N, umma_desc(k_base + off, 16, 1024),
                             umma_desc(q_base + qoff, 16, 1024), IDESC_S, kk > 0 ? 1u : 0u);
                    }
                    umma_commit(&s_full[j & 1]);
                    umma_commit(&k_empty);
                }
            }
        }
    } else {
        // ---------------- softmax: one token per thread ----------------
        const int q4 = warp & 3;         // TMEM lane quarter this warp may access
        const int tok = q4 * 32 + lane;  // token of the tile = TMEM lane
        const int st = threadIdx.x - 64; // thread index within the softmax warpgroup
        const uint32_t lane_base = tmem + ((uint32_t)(q4 * 32) << 16);
        float m[N], l[N];  // reference maxima (log2 units, scaled; the same in every thread), partial sums
#pragma unroll
        for (int r = 0; r < N; ++r) {
            m[r] = -INFINITY;
            l[r] = 0.f;
        }
        bool ok = true;
        for (int j = 0; j < nt; ++j) {
            // S_j is ready, and P.V of tile j - 1 is done: O^T holds the tiles
            // before j (for a rescale) and the P buffer is free
            bool wok = mbar_wait(&s_full[j & 1], (j >> 1) & 1, p.err);
            if (wok && j >= 1) wok = mbar_wait(&pv_done, (j - 1) & 1, p.err);
            if (softmax_any(!wok)) {
                ok = false;
                break;
            }
            tc_fence_after();
            if (threadIdx.x == 64) {
                PA_TT(j, 0);
                if (j == 0) PA_TL(1, 4);
            }
            const uint32_t s_col = lane_base + N + (j & 1) * N;
            const bool tvalid = j * kTcTokens + tok < ntok;
            float x[N];
            bool grow = false;
            tmem_ld32(s_col, x);
            tmem_wait_ld();
#pragma unroll
            for (int r = 0; r < N; ++r) grow |= tvalid && x[r] * p.scale_log2 > m[r] + kTcRescaleLog2;
            if (softmax_any(grow)) {
                // the tile's exact row maxima: over this warp's 32 tokens by
                // a transposing shuffle reduction (lane i gets row i), then
                // over the four warps through shared memory
#pragma unroll
                for (int r = 0; r < N; ++r) x[r] = tvalid ? x[r] * p.scale_log2 : -INFINITY;
                red[q4 * N + lane] = warp_transpose_reduce<true>(x, lane);
                consumer_barrier(1, 128);
                const float mt = fmaxf(fmaxf(red[lane], red[N + lane]), fmaxf(red[2 * N + lane], red[3 * N + lane]));
                // O^T (lane = output element, column = row) holds the tiles
                // before j: rescale it with the partial sums
                float ov[32];
                if (j >= 1) {
                    tmem_ld32(lane_base, ov);
                    tmem_wait_ld();
                }
#pragma unroll
                for (int r = 0; r < N; ++r) {
                    const float mn = fmaxf(m[r], __shfl_sync(0xffffffffu, mt, r));
                    const float alpha = m[r] == -INFINITY ? 0.f : ex2_approx(m[r] - mn);
                    m[r] = mn;
                    l[r] *= alpha;
                    ov[r] *= alpha;
                }
                if (j >= 1) {
                    tmem_st32(lane_base, ov);
                    tmem_wait_st();
                }
                // the reduction consumed the scores: read them again
                tmem_ld32(s_col, x);
                tmem_wait_ld();
            }
#pragma unroll
            for (int r = 0; r < N; ++r) x[r] = tvalid ? x[r] * p.scale_log2 : -INFINITY;
            // weights of this token for every row, split into bf16 high and
            // residual parts, written as token tok's row of P^T: rows
            // 8c..8c+7 form 16-byte chunk c, stored at chunk c ^ ((tok & 7) >> 1)
            // (the 64-byte swizzle)
            uint8_t* prow = sP + tok * kTcPRow;
#pragma unroll
            for (int c = 0; c < kTcPRow / 16; ++c) {
                uint32_t hi[4], lo[4];
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const int r = 8 * c + 2 * i;
                    const float e0 = m[r] == -INFINITY ? 0.f : ex2_approx(x[r] - m[r]);
                    const float e1 = m[r + 1] == -INFINITY ? 0.f : ex2_approx(x[r + 1] - m[r + 1]);
                    l[r] += e0;
                    l[r + 1] += e1;
                    hi[i] = pack_bf16x2(e0, e1);
                    lo[i] = pack_bf16x2(e0 - bf16_lo_to_f32(hi[i]), e1 - bf16_hi_to_f32(hi[i]));
                }
                const int pc = c ^ ((tok & 7) >> 1);
                *reinterpret_cast<uint4*>(prow + pc * 16) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
                *reinterpret_cast<uint4*>(prow + kTcPBytes + pc * 16) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
            }
            fence_proxy_async_smem();  // P is read by the tensor core
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&p_full);
            if (threadIdx.x == 64) PA_TT(j, 1);
        }
        // the last P.V done: O^T is complete (and every MMA has read its
        // operands, so the K buffer is free for the epilogue)
        if (ok) {
            const bool wok = mbar_wait(&pv_done, (nt - 1) & 1, p.err);
            ok = !softmax_any(!wok);
        }
        if (ok) {
            tc_fence_after();
            // row sums: each thread's over its tokens, added over the warp
            // (lane i gets row i) and then over the four warps
            float v[32];
#pragma unroll
            for (int r = 0; r < N; ++r) v[r] = l[r];
            red[q4 * N + lane] = warp_transpose_reduce<false>(v, lane);
            // O^T column tok (output element tok of every row) into the K
            // buffer as rows [N][D]
            float* so = reinterpret_cast<float*>(sK);
            float ov[32];
            tmem_ld32(lane_base, ov);
            tmem_wait_ld();
#pragma unroll
            for (int r = 0; r < N; ++r) so[r * D + tok] = ov[r];
            consumer_barrier(1, 128);
            // prefix-last order: pass 1's partial results are needed now
            if (p.prefix_last) griddep_wait();
            if (q4 == 0) {
                // row `lane`: where it goes and its factors
                const float lt = (red[lane] + red[N + lane]) + (red[2 * N + lane] + red[3 * N + lane]);
                float mr = m[0];
#pragma unroll
                for (int r = 1; r < N; ++r) mr = lane == r ? m[r] : mr;
                const int gr = row0 + lane;
                int64_t off = -1, own = -1;
                float c0 = 0.f, c1 = 0.f;
                if (gr < rows_total) {
                    const int64_t qrow = (int64_t)(grp.start + gr / G) * p.num_q_heads + (int64_t)kvh * G + gr % G;
                    if (p.prefix_last) {
                        // the final row: this split's state folded with pass
                        // 1's partial of the own tokens (slot 1) by the
                        // log-sum-exp rescale
                        const int64_t r1 = qrow * p.max_splits + 1;
                        const float m1 = __ldcg(p.part_ml + 2 * r1), l1 = __ldcg(p.part_ml + 2 * r1 + 1);
                        const float Mt = fmaxf(mr, m1);
                        const float a0 = mr == -INFINITY ? 0.f : exp2f(mr - Mt);
                        const float w1 = m1 == -INFINITY ? 0.f : l1 * exp2f(m1 - Mt);
                        const float W = lt * a0 + w1;
                        const float inv = W > 0.f ? 1.f / W : 0.f;
                        c0 = a0 * inv;
                        c1 = w1 * inv;
                        off = qrow * D;
                        own = r1 * D;
                    } else {
                        // the normalised partial and (m, l) in the split's slot
                        const int64_t slotrow = qrow * p.max_splits + split;
                        off = slotrow * D;
                        p.part_ml[2 * slotrow] = mr;
                        p.part_ml[2 * slotrow + 1] = lt;
                        c0 = lt > 0.f ? 1.f / lt : 0.f;
                    }
                }
                row_off[lane] = off;
                row_inv[lane] = c0;
                row_c1[lane] = c1;
                row_own[lane] = own;
            }
            consumer_barrier(1, 128);
            // each row's 128 elements as 32 float4, one row per warp step
            const float4* so4 = reinterpret_cast<const float4*>(so);
            for (int i = st; i < N * (D / 4); i += 128) {
                const int r = i / (D / 4);
                const int64_t off = row_off[r];
                if (off >= 0) {
                    const int c = (i % (D / 4)) * 4;
                    float4 o = so4[i];
                    const float c0 = row_inv[r];
                    o.x *= c0;
                    o.y *= c0;
                    o.z *= c0;
                    o.w *= c0;
                    if (p.prefix_last) {
                        const float c1 = row_c1[r];
                        const float4 o1 = __ldcg(reinterpret_cast<const float4*>(p.part_o + row_own[r] + c));
                        o.x = fmaf(c1, o1.x, o.x);
                        o.y = fmaf(c1, o1.y, o.y);
                        o.z = fmaf(c1, o1.z, o.z);
                        o.w = fmaf(c1, o1.w, o.w);
                        store_out4(p, off + c, o);
                    } else {
                        *reinterpret_cast<float4*>(p.part_o + off + c) = o;
                    }
                }
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTcTmemCols));
    }
    if (threadIdx.x == 0) {
        prefix_last_exit(p);
        PA_TL(1, 2);
    }
}

// Second pass: out = sum_s w_s o_s / sum_s w_s with w_s = l_s * 2^(m_s - max m),
// for sequences that were cut into more than one split.  W warps share a
// (sequence, query head) row: W = 4 with two rows per CTA, or W = 8 with one
// row per CTA when rows are few and splits many.  Warp k of a row takes
// splits k, k + W, ..., eight at a time, issuing all their (m, l) and partial-row
// loads before it needs any of them (lane i holds output elements
// [i * D / 32, (i + 1) * D / 32)), and keeps its own running max, weight sum
// and accumulator; the W warps' states are then combined through shared
// memory by the row's first warp.  The order of every sum is fixed, so the
// result is deterministic.
constexpr int kMergeWarps = 8;
constexpr int kMergeChunk = 8;  // splits per warp in flight

template <int D, int kMergeWarpsPerRow>
__global__ void __launch_bounds__(32 * kMergeWarps) decode_merge_kernel(const DecodeParams p, int64_t rows) {
    constexpr int VPL = D / 32;  // output elements per lane
    constexpr int STRIDE = kMergeWarpsPerRow * kMergeChunk;
    __shared__ float s_acc[kMergeWarps][D];
    __shared__ float s_m[kMergeWarps], s_w[kMergeWarps];
    const int lane = threadIdx.x & 31;
    const int warp = threadIdx.x >> 5;
    const int wk = warp % kMergeWarpsPerRow;
    griddep_wait();  // the partial rows come from pass 1
    const int64_t row = (int64_t)blockIdx.x * (kMergeWarps / kMergeWarpsPerRow) + warp / kMergeWarpsPerRow;
    int ns = 0;
    if (row < rows) {
        const int b = (int)(row / p.num_q_heads);
        const int L = clamp_len(p, b, false);
        int sp;
        ns = row_splits(p, L, seq_prefix_len(p, b, L), &sp);
        if (sp > 0 && sp <= kMaxFoldSplits && ns == sp + 1) ns = 1;  // pass 1 folded the prefix in and wrote the row
    }
    float m = -INFINITY, W = 0.f, acc[VPL];
#pragma unroll
    for (int i = 0; i < VPL; ++i) acc[i] = 0.f;
    if (ns > 1) {
        const float* ml = p.part_ml + row * p.max_splits * 2;
        const float* po = p.part_o + row * p.max_splits * D + lane * VPL;
        for (int s0 = wk; s0 < ns; s0 += STRIDE) {
            float mv[kMergeChunk], lv[kMergeChunk], ov[kMergeChunk][VPL];
#pragma unroll
            for (int k = 0; k < kMergeChunk; ++k) {
                const int sp = s0 + k * kMergeWarpsPerRow;
                if (sp < ns) {
                    mv[k] = ml[2 * sp];
                    lv[k] = ml[2 * sp + 1];
                    const float* src = po + (int64_t)sp * D;
                    if constexpr (VPL == 4) {
                        const float4 v = *reinterpret_cast<const float4*>(src);
                        ov[k][0] = v.x;
                        ov[k][1] = v.y;
                        ov[k][2] = v.z;
                        ov[k][3] = v.w;
                    } else {
                        const float2 v = *reinterpret_cast<const float2*>(src);
                        ov[k][0] = v.x;
                        ov[k][1] = v.y;
                    }
                } else {
                    mv[k] = -INFINITY;
                    lv[k] = 0.f;
#pragma unroll
                    for (int i = 0; i < VPL; ++i) ov[k][i] = 0.f;
                }
            }
            float cm = m;
#pragma unroll
            for (int k = 0; k < kMergeChunk; ++k) cm = fmaxf(cm, mv[k]);
            const float alpha = m == -INFINITY ? 0.f : exp2f(m - cm);
            W *= alpha;
#pragma unroll
            for (int i = 0; i < VPL; ++i) acc[i] *= alpha;
#pragma unroll
            for (int k = 0; k < kMergeChunk; ++k) {
                const float w = mv[k] == -INFINITY ? 0.f : lv[k] * exp2f(mv[k] - cm);
                W += w;
#pragma unroll
                for (int i = 0; i < VPL; ++i) acc[i] = fmaf(w, ov[k][i], acc[i]);
            }
            m = cm;
        }
    }
#pragma unroll
    for (int i = 0; i < VPL; ++i) s_acc[warp][lane * VPL + i] = acc[i];
    if (lane == 0) {
        s_m[warp] = m;
        s_w[warp] = W;
    }
    __syncthreads();
    if (wk != 0 || ns <= 1) return;
    float M = -INFINITY;
#pragma unroll
    for (int k = 0; k < kMergeWarpsPerRow; ++k) M = fmaxf(M, s_m[warp + k]);
    float scale[kMergeWarpsPerRow], Wt = 0.f;
#pragma unroll
    for (int k = 0; k < kMergeWarpsPerRow; ++k) {
        scale[k] = s_m[warp + k] == -INFINITY ? 0.f : exp2f(s_m[warp + k] - M);
        Wt += s_w[warp + k] * scale[k];
    }
#pragma unroll
    for (int i = 0; i < VPL; ++i) {
        float v = 0.f;
#pragma unroll
        for (int k = 0; k < kMergeWarpsPerRow; ++k) v = fmaf(scale[k], s_acc[warp + k][lane * VPL + i], v);
        store_out(p, row * D + lane * VPL + i, Wt > 0.f ? v / Wt : 0.f);
    }
}

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------
struct Plan {
    int partition;
    int max_splits;     // partial-result slots per row (prefix splits + suffix splits)
    int suffix_splits;  // pass 1's grid.x
    size_t part_o_bytes;
    size_t part_ml_bytes;
    size_t seq_prefix_bytes;
    size_t done_bytes;
    size_t workspace;
    // shared-prefix calls only
    int prefix_partition;
    int prefix_splits;
    int tc;      // head_dim 128: the tensor-core (tcgen05) prefix pass, 32 query rows per CTA
    int mt;      // otherwise: 16-row query tiles per prefix CTA (consumer warps)
    int chunks;  // prefix CTAs per (group, kv head) along the query rows
    // one prefix split and one own split on the tensor-core path: set-up
    // kernel, pass 1, then the prefix pass, which finishes the rows
    int prefix_last;
};

constexpr int kPrefixRingBytes = 64 * 1024;
constexpr int kMinPrefixPartition = 256;

inline size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

int auto_partition(int batch, int num_q_heads, int num_kv_heads, int max_context_len) {
    // With longest-first launch order, long work items cost nothing in the
    // tail while each split adds a CTA start-up and G partial rows to write
    // and merge; so the partition is as long as possible (4096 tokens) while
    // the grid still holds two waves of work items (counted as if every
    // sequence had max_context_len tokens), halved down to 512 otherwise.
    // Measured on the B200 over batch 1..256, groups 1..8, lengths 128..128k.
    (void)num_q_heads;
    int P = kMaxAutoPartition;
    const int64_t waves = 2ll * num_sms() * kCtasPerSmEstimate;
    const int64_t L = max_context_len > 0 ? max_context_len : 1;
    while (P > kMinAutoPartition && (int64_t)batch * num_kv_heads * ((L + P - 1) / P) < waves) P /= 2;
    return P;
}

// Tokens per prefix split: as long as possible (4096) while the prefix pass
// still has a CTA per SM to run, halved down to 256 otherwise.  Longer
// splits mean fewer CTA start-ups and fewer prefix partials for pass 1 to fold
// in: on the shared-prefix workload (256 groups x kv heads of 992 tokens) one
// split per group ran 11 % faster than four.
int auto_prefix_partition(int num_groups, int num_kv_heads, int chunks, int max_prefix_len) {
    int P = kMaxAutoPartition;
    const int64_t want = num_sms();
    const int64_t L = max_prefix_len > 0 ? max_prefix_len : 1;
    while (P > kMinPrefixPartition && (int64_t)num_groups * num_kv_heads * chunks * ((L + P - 1) / P) < want) P /= 2;
    return P;
}

// num_groups == 0: plain decode.  Otherwise the shared-prefix layout: the
// prefix pass's tiling and split size, prefix slots before suffix slots, and
// the per-sequence prefix lengths after the partial results.
int make_plan(int batch, int num_q_heads, int num_kv_heads, int head_dim, int max_context_len, int partition_size,
              Plan* plan, int num_groups = 0, int max_group = 0, int max_prefix = 0) {
    int P = partition_size;
    if (P == 0) P = auto_partition(batch, num_q_heads, num_kv_heads, max_context_len);
    if (P < kStageTokens || P > kMaxPartition || P % kStageTokens != 0) return PA_ERR_INVALID_ARG;
    const int L = max_context_len > 0 ? max_context_len : 1;
    const int splits = (L + P - 1) / P;
    *plan = Plan{};
    plan->partition = P;
    plan->suffix_splits = splits;
    plan->max_splits = splits;
    if (num_groups > 0) {
        const int rows = max_group * (num_q_heads / num_kv_heads);
        plan->tc = head_dim == 128;
        plan->mt = rows <= 16 ? 1 : (rows <= 32 ? 2 : 4);
        const int rows_per_cta = plan->tc ? kTcRows : 16 * plan->mt;
        plan->chunks = (rows + rows_per_cta - 1) / rows_per_cta;
        plan->prefix_partition = auto_prefix_partition(num_groups, num_kv_heads, plan->chunks, max_prefix);
        plan->prefix_splits = max_prefix > 0 ? (max_prefix + plan->prefix_partition - 1) / plan->prefix_partition : 0;
        plan->max_splits = plan->prefix_splits + splits;
        plan->seq_prefix_bytes = align256((size_t)batch * sizeof(int32_t));
        plan->prefix_last = plan->tc && plan->prefix_splits == 1 && plan->suffix_splits == 1;
        plan->done_bytes = plan->prefix_last ? 256 : 0;
    }
    if (plan->max_splits > 1) {
        const size_t rows = (size_t)batch * num_q_heads * plan->max_splits;
        plan->part_o_bytes = align256(rows * head_dim * sizeof(float));
        plan->part_ml_bytes = align256(rows * 2 * sizeof(float));
    }
    plan->workspace = plan->part_o_bytes + plan->part_ml_bytes + plan->seq_prefix_bytes + plan->done_bytes;
    return PA_OK;
}

using TensorMapEncodeFn = PFN_cuTensorMapEncodeTiled_v12000;

TensorMapEncodeFn tensor_map_encoder() {
    static TensorMapEncodeFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* ptr = nullptr;
        cudaDriverEntryPointQueryResult q = cudaDriverEntryPointSymbolNotFound;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<TensorMapEncodeFn>(ptr);
    });
    return fn;
}

// 2-D bf16 tensor map over `rows` rows of head_dim elements, boxes of 64
// elements (128 bytes, the swizzle span) by box_rows rows, 128-byte swizzle.
int encode_kv_map(CUtensorMap* map, const void* base, uint64_t rows, int head_dim, int box_rows) {
    TensorMapEncodeFn enc = tensor_map_encoder();
    if (!enc) return PA_ERR_CUDA;
    cuuint64_t dims[2] = {(cuuint64_t)head_dim, rows > 0 ? rows : 1};
    cuuint64_t strides[1] = {(cuuint64_t)head_dim * 2};
    cuuint32_t box[2] = {64u, (cuuint32_t)box_rows};
    cuuint32_t elem_strides[2] = {1u, 1u};
    const CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box,
                           elem_strides, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                           CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? PA_OK : PA_ERR_CUDA;
}

template <int D, int NT>
int launch_pass1_mma(const DecodeParams& p, const CUtensorMap& tmk, const CUtensorMap& tmv, dim3 grid, size_t smem,
                     cudaStream_t st) {
    static std::atomic<unsigned long long> configured{0};
    int dev = 0;
    cudaGetDevice(&dev);
    const unsigned long long bit = 1ull << (dev & 63);
    if (!(configured.load() & bit)) {
        if (cudaFuncSetAttribute(decode_pass1_mma_kernel<D, NT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 kMaxDynamicSmem) != cudaSuccess)
            return PA_ERR_CUDA;
        configured.fetch_or(bit);
    }
    return launch_pdl(decode_pass1_mma_kernel<D, NT>, grid, dim3(kDecodeThreads), smem, st, p, tmk, tmv);
}

template <int D, int MT, int PAR>
int launch_prefix_mma(const DecodeParams& p, const CUtensorMap& tmk, const CUtensorMap& tmv, dim3 grid, size_t smem,
                      cudaStream_t st) {
    static std::atomic<unsigned long long> configured{0};
    int dev = 0;
    cudaGetDevice(&dev);
    const unsigned long long bit = 1ull << (dev & 63);
    if (!(configured.load() & bit)) {
        if (cudaFuncSetAttribute(decode_prefix_mma_kernel<D, MT, PAR>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 kMaxDynamicSmem) != cudaSuccess)
            return PA_ERR_CUDA;
        configured.fetch_or(bit);
    }
    return launch_pdl(decode_prefix_mma_kernel<D, MT, PAR>, grid, dim3(32 * (1 + MT * PAR)), smem, st, p, tmk, tmv);
}

int launch_prefix_tc(const DecodeParams& p, const CUtensorMap& tmk, const CUtensorMap& tmv, dim3 grid, size_t smem,
                     cudaStream_t st) {
    static std::atomic<unsigned long long> configured{0};
    int dev = 0;
    cudaGetDevice(&dev);
    const unsigned long long bit = 1ull << (dev & 63);
    if (!(configured.load() & bit)) {
        if (cudaFuncSetAttribute(decode_prefix_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 kMaxDynamicSmem) != cudaSuccess)
            return PA_ERR_CUDA;
        configured.fetch_or(bit);
    }
    return launch_pdl(decode_prefix_tc_kernel, grid, dim3(kTcThreads), smem, st, p, tmk, tmv);
}

// Consumer groups of the prefix pass: two parity groups for 16 or 32 query
// rows per CTA, one for 64 (the block stays at five warps or fewer).
template <int D>
int launch_prefix_for_rows(int mt, const DecodeParams& p, const CUtensorMap& tmk, const CUtensorMap& tmv, dim3 grid,
                           size_t smem, cudaStream_t st) {
    return mt == 1 ? launch_prefix_mma<D, 1, 2>(p, tmk, tmv, grid, smem, st)
         : mt == 2 ? launch_prefix_mma<D, 2, 2>(p, tmk, tmv, grid, smem, st)
                   : launch_prefix_mma<D, 4, 1>(p, tmk, tmv, grid, smem, st);
}

template <typename T, int D, int G>
int launch_pass1(const DecodeParams& p, dim3 grid, size_t smem, cudaStream_t st) {
    static std::atomic<unsigned long long> configured{0};
    int dev = 0;
    cudaGetDevice(&dev);
    const unsigned long long bit = 1ull << (dev & 63);
    if (!(configured.load() & bit)) {
        if (cudaFuncSetAttribute(decode_pass1_kernel<T, D, G>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 kMaxDynamicSmem) != cudaSuccess)
            return PA_ERR_CUDA;
        configured.fetch_or(bit);
    }
    return launch_pdl(decode_pass1_kernel<T, D, G>, grid, dim3(kDecodeThreads), smem, st, p);
}

template <typename T, int D>
int dispatch_group(int G, const DecodeParams& p, dim3 grid, size_t smem, cudaStream_t st) {
    switch (G) {
        case 1: return launch_pass1<T, D, 1>(p, grid, smem, st);
        case 2: return launch_pass1<T, D, 2>(p, grid, smem, st);
        case 4: return launch_pass1<T, D, 4>(p, grid, smem, st);
        case 8: return launch_pass1<T, D, 8>(p, grid, smem, st);
        default: return PA_ERR_UNSUPPORTED;
    }
}

// p.num_groups > 0: shared-prefix decode (bf16, paged), with the prefix pass
// launched before pass 1.
int run_decode(DecodeParams p, int head_dim, int kv_dtype, int batch, void* workspace, size_t workspace_bytes,
               int max_context_len, int partition_size, cudaStream_t st) {
    const int G = p.num_q_heads / p.num_kv_heads;
    Plan plan;
    int rc = make_plan(batch, p.num_q_heads, p.num_kv_heads, head_dim, max_context_len, partition_size, &plan,
                       p.num_groups, p.max_group, p.max_prefix);
    if (rc) return rc;
    if (plan.workspace > 0) {
        if (!workspace || workspace_bytes < plan.workspace || !aligned16(workspace)) return PA_ERR_WORKSPACE;
        char* ws = static_cast<char*>(workspace);
        p.part_o = plan.part_o_bytes ? reinterpret_cast<float*>(ws) : nullptr;
        p.part_ml = plan.part_ml_bytes ? reinterpret_cast<float*>(ws + plan.part_o_bytes) : nullptr;
        p.seq_prefix = plan.seq_prefix_bytes
                           ? reinterpret_cast<int32_t*>(ws + plan.part_o_bytes + plan.part_ml_bytes)
                           : nullptr;
        p.done_count = plan.done_bytes ? reinterpret_cast<int*>(ws + plan.part_o_bytes + plan.part_ml_bytes +
                                                                plan.seq_prefix_bytes)
                                       : nullptr;
    } else {
        p.part_o = nullptr;
        p.part_ml = nullptr;
        p.seq_prefix = nullptr;
    }
    p.partition = plan.partition;
    p.max_splits = plan.max_splits;
    p.prefix_partition = plan.prefix_partition;
    p.batch = batch;
    // with shared prefixes the own parts are short and alike (generated
    // tokens): the ranking's cost outweighs its balance (6 % on the
    // shared-prefix workload), so sequences go in index order
    p.longest_first = batch <= kLongestFirstMaxBatch && p.num_groups == 0;
    p.err = error_word_ptr();
    if (!p.err) return PA_ERR_CUDA;

    const int stage_bytes = 2 * kStageTokens * head_dim * (int)dtype_bytes(kv_dtype);  // K + V
    // Stage j lives in slot j % stages and is consumed by warp j % 2.  The
    // stage count must be a multiple of the consumer-warp count: then the
    // previous user of a slot is the same warp, so a warp never waits on a
    // full-barrier phase more than one ahead of the barrier's current phase
    // (a parity wait cannot tell phase k + 2 from phase k).
    int stages = (kRingTargetBytes / stage_bytes) / kConsumerWarps * kConsumerWarps;
    stages = stages < kConsumerWarps ? kConsumerWarps : (stages > 4 * kConsumerWarps ? 4 * kConsumerWarps : stages);
    p.stages = stages;
    // bf16 pass 1 loads its block-table window speculatively (one round trip
    // fewer) while the window stays within twice a partition's blocks
    const int part_blocks = plan.partition / p.block_size;
    p.table_window = 0;
    if (!p.contiguous && kv_dtype == PA_BF16 && (p.num_groups == 0 || p.max_prefix <= plan.partition))
        p.table_window = min((p.num_groups > 0 ? p.max_prefix : 0) / p.block_size + part_blocks,
                             max(p.max_blocks_per_seq, 1));
    const int table_bytes = p.contiguous ? 0 : max(part_blocks, p.table_window) * 4;
    p.ring_offset = (int)((16 * stages + table_bytes + 127) & ~127);
    const size_t ring_bytes = (size_t)stages * stage_bytes;
    const size_t merge_bytes = ((size_t)kConsumerWarps * G * (head_dim + 2) + (size_t)G * kCoefStride) * sizeof(float);
    if (merge_bytes > ring_bytes) return PA_ERR_UNSUPPORTED;
    const size_t smem = p.ring_offset + ring_bytes;
    if (smem > (size_t)kMaxDynamicSmem) return PA_ERR_UNSUPPORTED;

    dim3 grid((unsigned)plan.suffix_splits, (unsigned)p.num_kv_heads, (unsigned)batch);
    if (kv_dtype == PA_BF16) {
        // tensor-core path: K/V tiles by tiled TMA, contractions by mma.sync
        const uint64_t rows = p.contiguous ? (uint64_t)batch * p.num_kv_heads * (uint64_t)p.L_pad
                                           : (uint64_t)p.num_blocks * p.num_kv_heads * (uint64_t)p.block_size;
        if (rows >= (1ull << 31)) return PA_ERR_UNSUPPORTED;
        CUtensorMap tmk, tmv;
        if ((rc = encode_kv_map(&tmk, p.k, rows, head_dim, p.block_size))) return rc;
        if ((rc = encode_kv_map(&tmv, p.v, rows, head_dim, p.block_size))) return rc;
        // the prefix pass on the tensor cores: 128-token tiles, its own
        // buffers and tensor memory
        p.prefix_last = p.num_groups > 0 && plan.prefix_last;
        const auto prefix_tc = [&]() -> int {
            const size_t psmem = prefix_tc_smem_bytes(plan.prefix_partition / p.block_size);
            if (psmem > (size_t)kMaxDynamicSmem) return PA_ERR_UNSUPPORTED;
            const int64_t gy = (int64_t)p.num_kv_heads * plan.chunks;
            if (gy > 65535) return PA_ERR_UNSUPPORTED;
            const dim3 pg((unsigned)(plan.prefix_splits > 0 ? plan.prefix_splits : 1), (unsigned)gy,
                          (unsigned)p.num_groups);
            return launch_prefix_tc(p, tmk, tmv, pg, psmem, st);
        };
        if (p.prefix_last) {
            // set-up kernel, pass 1, then the prefix pass (below)
            if ((rc = launch_pdl(decode_prefix_setup_kernel, dim3(1), dim3(1024), 0, st, p))) return rc;
        } else if (p.num_groups > 0 && plan.tc) {
            if ((rc = prefix_tc())) return rc;
        } else if (p.num_groups > 0) {
            // the prefix pass: a deeper ring (few, long-lived CTAs), every
            // consumer warp reads every stage
            DecodeParams pp = p;
            pp.stages = kPrefixRingBytes / stage_bytes;
            const int ptable = (plan.prefix_partition / p.block_size) * 4;
            pp.ring_offset = (int)((16 * pp.stages + ptable + 1023) & ~1023);
            // ring (a multiple of two stages: two consumer parity groups),
            // then the chunk's query rows
            const size_t qbytes = (size_t)16 * plan.mt * head_dim * 2;
            const size_t psmem = pp.ring_offset + (size_t)pp.stages * stage_bytes + qbytes + 1024;
            if (psmem > (size_t)kMaxDynamicSmem || pp.stages % 2) return PA_ERR_UNSUPPORTED;
            const int64_t gy = (int64_t)p.num_kv_heads * plan.chunks;
            if (gy > 65535) return PA_ERR_UNSUPPORTED;
            const dim3 pg((unsigned)(plan.prefix_splits > 0 ? plan.prefix_splits : 1), (unsigned)gy,
                          (unsigned)p.num_groups);
            rc = head_dim == 128 ? launch_prefix_for_rows<128>(plan.mt, pp, tmk, tmv, pg, psmem, st)
                                 : launch_prefix_for_rows<64>(plan.mt, pp, tmk, tmv, pg, psmem, st);
            if (rc) return rc;
        }
        p.ring_offset = (int)((16 * stages + table_bytes + 1023) & ~1023);
        // shared-prefix calls with the prefix pass first: room for the
        // prefix partial a row folds in
        p.fold_prefetch = p.num_groups > 0 && !p.prefix_last;
        const size_t pf_bytes = p.fold_prefetch ? ((size_t)G * (head_dim + 2) * sizeof(float) + 15) & ~(size_t)15 : 0;
        const size_t smem_mma = p.ring_offset + ring_bytes + pf_bytes + 1024;
        if (smem_mma > (size_t)kMaxDynamicSmem) return PA_ERR_UNSUPPORTED;
        if (head_dim == 128)
            rc = G <= 8 ? launch_pass1_mma<128, 1>(p, tmk, tmv, grid, smem_mma, st)
                        : launch_pass1_mma<128, 2>(p, tmk, tmv, grid, smem_mma, st);
        else
            rc = G <= 8 ? launch_pass1_mma<64, 1>(p, tmk, tmv, grid, smem_mma, st)
                        : launch_pass1_mma<64, 2>(p, tmk, tmv, grid, smem_mma, st);
        if (!rc && p.prefix_last) rc = prefix_tc();
    } else {
        rc = head_dim == 128 ? dispatch_group<float, 128>(G, p, grid, smem, st)
                             : dispatch_group<float, 64>(G, p, grid, smem, st);
    }
    if (rc) return rc;
    // with shared prefixes, rows whose suffix is one split are finished by
    // pass 1 (or, in the prefix-last order, by the prefix pass); the merge
    // pass is needed only when a suffix can be split
    if (p.num_groups > 0 ? !plan.prefix_last && (plan.suffix_splits > 1 || plan.prefix_splits > kMaxFoldSplits)
                         : plan.max_splits > 1) {
        const int64_t rows = (int64_t)batch * p.num_q_heads;
        // four warps per row, or all eight of a CTA when rows carry many splits
        // and there are too few rows to fill the GPU with four-warp groups
        const bool wide = plan.max_splits > 32 && rows < (int64_t)num_sms() * 2;
        const int rows_per_cta = wide ? 1 : kMergeWarps / 4;
        const unsigned blocks = (unsigned)((rows + rows_per_cta - 1) / rows_per_cta);
        const dim3 mg(blocks), mb(32 * kMergeWarps);
        if (head_dim == 128)
            rc = wide ? launch_pdl(decode_merge_kernel<128, 8>, mg, mb, 0, st, p, rows)
                      : launch_pdl(decode_merge_kernel<128, 4>, mg, mb, 0, st, p, rows);
        else
            rc = wide ? launch_pdl(decode_merge_kernel<64, 8>, mg, mb, 0, st, p, rows)
                      : launch_pdl(decode_merge_kernel<64, 4>, mg, mb, 0, st, p, rows);
    }
    return rc;
}

int check_shapes(int batch, int num_q_heads, int num_kv_heads, int head_dim, int block_size, int kv_dtype,
                 int out_dtype, int max_context_len) {
    if (batch < 0 || num_q_heads <= 0 || num_kv_heads <= 0 || head_dim <= 0 || block_size <= 0 ||
        max_context_len < 0 || !valid_dtype(kv_dtype) || !valid_dtype(out_dtype))
        return PA_ERR_INVALID_ARG;
    if (num_q_heads % num_kv_heads != 0) return PA_ERR_INVALID_ARG;
    if (!supported_head_dim(head_dim) || !supported_block_size(block_size)) return PA_ERR_UNSUPPORTED;
    const int G = num_q_heads / num_kv_heads;
    if (G != 1 && G != 2 && G != 4 && G != 8 && !(G == 16 && kv_dtype == PA_BF16)) return PA_ERR_UNSUPPORTED;
    if (batch > 65535 || num_kv_heads > 65535) return PA_ERR_UNSUPPORTED;
    return PA_OK;
}

}  // namespace
}  // namespace pa

using namespace pa;

extern "C" int pa_paged_attention_partition_size(int batch, int num_q_heads, int num_kv_heads, int head_dim,
                                                 int max_context_len, int block_size, int* partition_size) {
    if (!partition_size) return PA_ERR_INVALID_ARG;
    int rc = check_shapes(batch, num_q_heads, num_kv_heads, head_dim, block_size, PA_BF16, PA_F32, max_context_len);
    if (rc) return rc;
    *partition_size = auto_partition(batch, num_q_heads, num_kv_heads, max_context_len);
    return PA_OK;
}

extern "C" int pa_paged_attention_workspace_size(int batch, int num_q_heads, int num_kv_heads, int head_dim,
                                                 int max_context_len, int block_size, int partition_size,
                                                 size_t* workspace_bytes) {
    if (!workspace_bytes) return PA_ERR_INVALID_ARG;
    int rc = check_shapes(batch, num_q_heads, num_kv_heads, head_dim, block_size, PA_BF16, PA_F32, max_context_len);
    if (rc) return rc;
    Plan plan;
    rc = make_plan(batch, num_q_heads, num_kv_heads, head_dim, max_context_len, partition_size, &plan);
    if (rc) return rc;
    *workspace_bytes = plan.workspace;
    return PA_OK;
}

extern "C" int pa_paged_attention_decode(const void* q, const void* k_pool, const void* v_pool,
                                         const int32_t* block_tables, int max_blocks_per_seq,
                                         const int32_t* context_lens, int max_context_len, float scale,
                                         int block_size, void* out, int out_dtype, int batch, int num_q_heads,
                                         int num_kv_heads, int head_dim, int64_t num_blocks, int kv_dtype,
                                         int partition_size, void* workspace, size_t workspace_bytes,
                                         void* stream) {
    PA_NVTX_RANGE("pa_paged_attention_decode");
    int rc = check_shapes(batch, num_q_heads, num_kv_heads, head_dim, block_size, kv_dtype, out_dtype,
                          max_context_len);
    if (rc) return rc;
    if (max_blocks_per_seq < 0 || num_blocks < 0) return PA_ERR_INVALID_ARG;
    if ((int64_t)max_context_len > (int64_t)max_blocks_per_seq * block_size) return PA_ERR_INVALID_ARG;
    if (batch == 0) return PA_OK;
    if (!q || !k_pool || !v_pool || !block_tables || !context_lens || !out) return PA_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k_pool) || !aligned16(v_pool)) return PA_ERR_INVALID_ARG;
    DecodeParams p = {};
    p.q = q;
    p.k = k_pool;
    p.v = v_pool;
    p.block_tables = block_tables;
    p.context_lens = context_lens;
    p.out = out;
    p.num_blocks = num_blocks;
    p.L_pad = 0;
    p.max_len = max_context_len;  // validated <= max_blocks_per_seq * block_size
    p.max_blocks_per_seq = max_blocks_per_seq;
    p.num_q_heads = num_q_heads;
    p.num_kv_heads = num_kv_heads;
    p.block_size = block_size;
    p.out_bf16 = out_dtype == PA_BF16;
    p.contiguous = 0;
    p.scale_log2 = scale * kLog2e;
    return run_decode(p, head_dim, kv_dtype, batch, workspace, workspace_bytes, max_context_len, partition_size,
                      static_cast<cudaStream_t>(stream));
}

extern "C" int pa_paged_attention_decode_append(const void* q, const void* key, const void* value, void* k_pool,
                                                void* v_pool, const int32_t* block_tables, int max_blocks_per_seq,
                                                const int32_t* context_lens, int max_context_len, float scale,
                                                int block_size, void* out, int out_dtype, int batch, int num_q_heads,
                                                int num_kv_heads, int head_dim, int64_t num_blocks, int kv_dtype,
                                                int partition_size, void* workspace, size_t workspace_bytes,
                                                int64_t* slot_mapping, void* stream) {
    PA_NVTX_RANGE("pa_paged_attention_decode_append");
    int rc = check_shapes(batch, num_q_heads, num_kv_heads, head_dim, block_size, kv_dtype, out_dtype,
                          max_context_len);
    if (rc) return rc;
    if (max_blocks_per_seq < 0 || num_blocks < 0) return PA_ERR_INVALID_ARG;
    if ((int64_t)max_context_len > (int64_t)max_blocks_per_seq * block_size) return PA_ERR_INVALID_ARG;
    if (batch == 0) return PA_OK;
    if (!q || !key || !value || !k_pool || !v_pool || !block_tables || !context_lens || !out)
        return PA_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(key) || !aligned16(value) || !aligned16(k_pool) || !aligned16(v_pool))
        return PA_ERR_INVALID_ARG;
    if (kv_dtype != PA_BF16) {
        // fp32: the write and the attention as two launches
        rc = pa_reshape_and_cache_decode(key, value, k_pool, v_pool, block_tables, max_blocks_per_seq, context_lens,
                                         batch, num_kv_heads, head_dim, block_size, num_blocks, kv_dtype,
                                         slot_mapping, stream);
        if (rc) return rc;
        return pa_paged_attention_decode(q, k_pool, v_pool, block_tables, max_blocks_per_seq, context_lens,
                                         max_context_len, scale, block_size, out, out_dtype, batch, num_q_heads,
                                         num_kv_heads, head_dim, num_blocks, kv_dtype, partition_size, workspace,
                                         workspace_bytes, stream);
    }
    DecodeParams p = {};
    p.q = q;
    p.k = k_pool;
    p.v = v_pool;
    p.block_tables = block_tables;
    p.context_lens = context_lens;
    p.out = out;
    p.num_blocks = num_blocks;
    p.L_pad = 0;
    p.max_len = max_context_len;
    p.max_blocks_per_seq = max_blocks_per_seq;
    p.num_q_heads = num_q_heads;
    p.num_kv_heads = num_kv_heads;
    p.block_size = block_size;
    p.out_bf16 = out_dtype == PA_BF16;
    p.contiguous = 0;
    p.scale_log2 = scale * kLog2e;
    p.k_new = key;
    p.v_new = value;
    p.slots = slot_mapping;
    p.append = 1;
    return run_decode(p, head_dim, kv_dtype, batch, workspace, workspace_bytes, max_context_len, partition_size,
                      static_cast<cudaStream_t>(stream));
}

extern "C" int pa_paged_attention_shared_prefix_workspace_size(int batch, int num_q_heads, int num_kv_heads,
                                                              int head_dim, int max_context_len, int block_size,
                                                              int num_groups, int max_group_size, int max_prefix_len,
                                                              int partition_size, size_t* workspace_bytes) {
    if (!workspace_bytes) return PA_ERR_INVALID_ARG;
    int rc = check_shapes(batch, num_q_heads, num_kv_heads, head_dim, block_size, PA_BF16, PA_F32, max_context_len);
    if (rc) return rc;
    if (num_groups < 1 || max_group_size < 1 || max_prefix_len < 0 || max_prefix_len > max_context_len)
        return PA_ERR_INVALID_ARG;
    Plan plan;
    rc = make_plan(batch, num_q_heads, num_kv_heads, head_dim, max_context_len, partition_size, &plan, num_groups,
                   max_group_size, max_prefix_len);
    if (rc) return rc;
    *workspace_bytes = plan.workspace;
    return PA_OK;
}

extern "C" int pa_paged_attention_decode_shared_prefix(
    const void* q, const void* k_pool, const void* v_pool, const int32_t* block_tables, int max_blocks_per_seq,
    const int32_t* context_lens, int max_context_len, float scale, int block_size, void* out, int out_dtype,
    int batch, int num_q_heads, int num_kv_heads, int head_dim, int64_t num_blocks, int kv_dtype,
    const int32_t* group_starts, const int32_t* group_prefix_lens, int num_groups, int max_group_size,
    int max_prefix_len, int partition_size, void* workspace, size_t workspace_bytes, void* stream) {
    PA_NVTX_RANGE("pa_paged_attention_decode_shared_prefix");
    int rc = check_shapes(batch, num_q_heads, num_kv_heads, head_dim, block_size, kv_dtype, out_dtype,
                          max_context_len);
    if (rc) return rc;
    if (kv_dtype != PA_BF16) return PA_ERR_UNSUPPORTED;
    if (max_blocks_per_seq < 0 || num_blocks < 0) return PA_ERR_INVALID_ARG;
    if ((int64_t)max_context_len > (int64_t)max_blocks_per_seq * block_size) return PA_ERR_INVALID_ARG;
    if (batch == 0) return PA_OK;
    if (num_groups < 1 || num_groups > batch || max_group_size < 1 || max_group_size > batch ||
        max_prefix_len < 0 || max_prefix_len > max_context_len)
        return PA_ERR_INVALID_ARG;
    if (!q || !k_pool || !v_pool || !block_tables || !context_lens || !out || !group_starts || !group_prefix_lens)
        return PA_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k_pool) || !aligned16(v_pool)) return PA_ERR_INVALID_ARG;
    DecodeParams p = {};
    p.q = q;
    p.k = k_pool;
    p.v = v_pool;
    p.block_tables = block_tables;
    p.context_lens = context_lens;
    p.out = out;
    p.num_blocks = num_blocks;
    p.max_len = max_context_len;
    p.max_blocks_per_seq = max_blocks_per_seq;
    p.num_q_heads = num_q_heads;
    p.num_kv_heads = num_kv_heads;
    p.block_size = block_size;
    p.out_bf16 = out_dtype == PA_BF16;
    p.contiguous = 0;
    p.scale_log2 = scale * kLog2e;
    p.group_starts = group_starts;
    p.group_prefix = group_prefix_lens;
    p.num_groups = num_groups;
    p.max_group = max_group_size;
    p.max_prefix = max_prefix_len;
    return run_decode(p, head_dim, kv_dtype, batch, workspace, workspace_bytes, max_context_len, partition_size,
                      static_cast<cudaStream_t>(stream));
}

extern "C" int pa_paged_attention_decode_contiguous(const void* q, const void* k_c, const void* v_c, int64_t L_pad,
                                                    const int32_t* context_lens, int max_context_len, float scale,
                                                    int block_size, void* out, int out_dtype, int batch,
                                                    int num_q_heads, int num_kv_heads, int head_dim, int kv_dtype,
                                                    int partition_size, void* workspace, size_t workspace_bytes,
                                                    void* stream) {
    PA_NVTX_RANGE("pa_paged_attention_decode_contiguous");
    int rc = check_shapes(batch, num_q_heads, num_kv_heads, head_dim, block_size, kv_dtype, out_dtype,
                          max_context_len);
    if (rc) return rc;
    if (L_pad < 0 || (int64_t)max_context_len > L_pad) return PA_ERR_INVALID_ARG;
    if (batch == 0) return PA_OK;
    if (!q || !k_c || !v_c || !context_lens || !out) return PA_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k_c) || !aligned16(v_c)) return PA_ERR_INVALID_ARG;
    DecodeParams p = {};
    p.q = q;
    p.k = k_c;
    p.v = v_c;
    p.block_tables = nullptr;
    p.context_lens = context_lens;
    p.out = out;
    p.num_blocks = 0;
    p.L_pad = L_pad;
    p.max_len = max_context_len;  // validated <= L_pad
    p.max_blocks_per_seq = 0;
    p.num_q_heads = num_q_heads;
    p.num_kv_heads = num_kv_heads;
    p.block_size = block_size;
    p.out_bf16 = out_dtype == PA_BF16;
    p.contiguous = 1;
    p.scale_log2 = scale * kLog2e;
    return run_decode(p, head_dim, kv_dtype, batch, workspace, workspace_bytes, max_context_len, partition_size,
                      static_cast<cudaStream_t>(stream));
}

#ifdef PA_TIMELINE
// The timeline build's readers (include/pa_timeline.h).
extern "C" int pa_timeline_clear(void) {
    void* a = nullptr;
    void* t = nullptr;
    if (cudaGetSymbolAddress(&a, pa::g_pa_tl) != cudaSuccess || cudaGetSymbolAddress(&t, pa::g_pa_tt) != cudaSuccess)
        return PA_ERR_CUDA;
    if (cudaMemset(a, 0, sizeof(pa::g_pa_tl)) != cudaSuccess || cudaMemset(t, 0, sizeof(pa::g_pa_tt)) != cudaSuccess)
        return PA_ERR_CUDA;
    return cudaDeviceSynchronize() == cudaSuccess ? PA_OK : PA_ERR_CUDA;
}

extern "C" int pa_timeline_read(int which, void* dst, size_t bytes) {
    if (!dst || (which != 0 && which != 1)) return PA_ERR_INVALID_ARG;
    const size_t size = which == 0 ? sizeof(pa::g_pa_tl) : sizeof(pa::g_pa_tt);
    if (bytes > size) return PA_ERR_INVALID_ARG;
    const cudaError_t e = which == 0 ? cudaMemcpyFromSymbol(dst, pa::g_pa_tl, bytes)
                                     : cudaMemcpyFromSymbol(dst, pa::g_pa_tt, bytes);
    return e == cudaSuccess ? PA_OK : PA_ERR_CUDA;
}
#endif
