// pa_prefill.cu -- causal multi-query attention over the paged cache
// (several new tokens per sequence, as in chunked prefill), on the 5th-
// generation tensor cores (tcgen05, accumulators in tensor memory).
//
// What it computes: sequence b of length L has n new query tokens, its last
// n; query i sits at position p = L - n + i and attends keys 0..p.  K and V
// are read from the block pool through the block table ("PagedAttention and
// KV memory management", "The kernel side"), never gathered.
//
// Query tile = 128 query rows of one (sequence, kv head): 128 / G query
// tokens x the G query heads that share the kv head.  One CTA takes two
// neighbouring tiles, which need (almost) the same keys:
//  * warp 0 loads both Q tiles once (tiled TMA, 3-D map over q [T, Hq, D])
//    and streams K/V tiles of 64 tokens through a 4-stage ring (tiled TMA
//    boxes of block_size rows from the pool, 128-byte swizzle), each tile
//    used by both query tiles;
//  * warp 1 allocates all 512 tensor-memory columns; warps 1 and 2 each issue
//    one query tile's MMAs from one thread, so neither tile's chain waits on
//    the other's softmax:
//        S_tj = Q_t . K_j^T       (M = 128 rows, N = 64 keys, K = D)
//        O_t += P_tj . V_j        (M = 128 rows, N = D, K = 64 keys)
//    S is double-buffered in tensor memory, so S_t,j+1 runs while the
//    softmax works on S_tj, and P_tj is written back over S_tj's columns and
//    read by the P.V MMA straight from tensor memory;
//  * warps 3..6 and 7..10 are the two tiles' softmax warpgroups (one query
//    row per thread: TMEM lane = row).  Each loads S_tj, applies the causal
//    mask and scale, keeps its row's running max and sum in registers,
//    rescales O in tensor memory only when the max has grown by more than
//    2^8 (lazy rescale), and stores P as a bf16 high part plus a bf16
//    residual (both multiplied by V, so the weights keep ~16 significant
//    bits), in two halves of 32 keys, each handed to the MMA thread as soon
//    as it is written.  With two warpgroups per CTA one tile's softmax
//    overlaps the other tile's MMAs.  At the end they read O and divide by
//    the row sum; a whole tile with bf16 output goes out through its Q
//    buffer by tiled TMA stores, other rows are stored directly.
// The heaviest pairs of tiles (latest query tokens, most keys) start first,
// across windows of four (sequence, kv head) groups.
// Every wait is a bounded mbarrier wait; on expiry the CTA records
// PA_ERR_TIMEOUT and winds down (tensor memory is always released).
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

// Per-CTA timeline stamps, compiled in only for libpa_timeline.so (the
// switch PA_TIMELINE; events listed in include/pa_timeline.h).
#ifdef PA_TIMELINE
namespace pa {
constexpr int kPfTlCtas = 65536;
constexpr int kPfTlSlots = 8;
__device__ unsigned long long g_pa_prefill_tl[(size_t)kPfTlCtas * kPfTlSlots];
__device__ __forceinline__ void prefill_stamp(int slot) {
    if (blockIdx.x >= (unsigned)kPfTlCtas) return;
    unsigned smid;
    asm volatile("mov.u32 %0, %%smid;" : "=r"(smid));
    unsigned long long* row = g_pa_prefill_tl + (size_t)blockIdx.x * kPfTlSlots;
    row[slot] = global_timer_ns();
    row[kPfTlSlots - 1] = smid;
}
}  // namespace pa
#define PF_TL(slot) ::pa::prefill_stamp(slot)
#else
#define PF_TL(slot) ((void)0)
#endif

namespace pa {
namespace {

constexpr int kRows = 128;    // query rows per tile (TMEM lanes)
constexpr int kTiles = 2;     // query tiles per CTA
constexpr int kKeys = 64;     // keys per tile
constexpr int kThreads = 96 + kTiles * 128;  // producer, two MMA issuers, one softmax warpgroup per query tile
static_assert(kTiles == 2, "the softmax warpgroups select their tile's values between two");
constexpr int kStages = 4;     // K/V ring depth
// Parts of a P tile handed to the MMA thread one by one (chunked-prefill
// workload, results bit-identical: 1 part 781, 2 parts 790, 4 parts 771
// TFLOP/s; with four the extra hand-offs cost more than the overlap gives).
constexpr int kHandoffs = 2;
constexpr int kPartKeys = kKeys / kHandoffs;    // keys per part (a multiple of the MMA's 16)
static_assert(kHandoffs == 2 || kHandoffs == 4, "P hand-off parts of 32 or 16 keys");
// (sequence, kv head) groups per launch-order window: wide enough that the
// grid's tail holds light pairs, narrow enough that the window's K/V stays
// in L2 (chunked-prefill workload: 1 group 766-770, 4 groups 773-779, 8
// groups 772, 64 groups 746 TFLOP/s)
constexpr int kWindow = 4;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kRescaleLog2 = 8.f;  // lazy-rescale threshold of the running max (log2 units)
// P.V with P as a bf16 high part plus a bf16 residual (two MMAs per key
// step, ~16 significant bits of weight) or as the high part alone (one MMA,
// 8 bits).  The library is built with the split; building with
// -DPA_PREFILL_SINGLE_P gives the one-MMA form, for measuring what the split
// costs and what it buys in accuracy.
#ifdef PA_PREFILL_SINGLE_P
constexpr bool kSplitP = false;
#else
constexpr bool kSplitP = true;
#endif

struct PrefillParams {
    const void* q;
    void* out;
    const int32_t* block_tables;
    const int32_t* context_lens;
    const int32_t* query_start;
    int* err;
    int64_t num_blocks;
    int max_blocks_per_seq;
    int num_q_heads;
    int num_kv_heads;
    int block_size;
    int out_bf16;
    float scale_log2;
    int pairs;   // pairs of query tiles per (sequence, kv head)
    int groups;  // batch x kv heads
};

// ---- the kernel ------------------------------------------------------------
// Two query tiles per CTA (tiles 2x and 2x + 1 of one (sequence, kv head)),
// each with its own softmax warpgroup, S double buffer and O accumulator in
// tensor memory; the K/V tiles they both need are loaded once.  While one
// warpgroup works on its scores the tensor core runs the other tile's MMAs.
template <int D>
__global__ void __launch_bounds__(kThreads, 1)
    prefill_tc_kernel(const PrefillParams p, const __grid_constant__ CUtensorMap tmq,
                      const __grid_constant__ CUtensorMap tmk, const __grid_constant__ CUtensorMap tmv,
                      const __grid_constant__ CUtensorMap tmo) {
    constexpr int SLABS = D / 64;
    constexpr int Q_BYTES = SLABS * kRows * 128;  // 128 rows x D
    constexpr int KV_SLAB = kKeys * 128;          // 64 rows x 64 elements
    constexpr int KV_BYTES = SLABS * KV_SLAB;     // one of K or V for one tile
    constexpr int S_COLS = kKeys;                 // TMEM columns of one S buffer
    constexpr uint32_t O_COL = 2 * S_COLS;        // O after the tile's two S buffers
    constexpr uint32_t TILE_COLS = 256;           // TMEM columns per query tile
    static_assert(O_COL + D <= TILE_COLS, "tensor-memory layout");

    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* smem = smem_raw + ((1024u - (smem_addr(smem_raw) & 1023u)) & 1023u);
    uint8_t* sQ = smem;                          // [kTiles][Q_BYTES]
    uint8_t* sK = sQ + kTiles * Q_BYTES;         // [kStages][KV_BYTES]
    uint8_t* sV = sK + kStages * KV_BYTES;       // [kStages][KV_BYTES]

    __shared__ uint64_t q_full, kv_full[kStages], kv_empty[kStages];
    // p_full[t][s][h]: part h (keys kPartKeys * h ..) of P in S buffer s of tile t
    __shared__ uint64_t s_full[kTiles][2], p_full[kTiles][2][kHandoffs], pv_done[kTiles][2];
    __shared__ uint32_t tmem_base;
    __shared__ int s_abort;

    // Launch order (the hardware dispatches CTAs by index): the (sequence,
    // kv head) groups are taken kWindow at a time, and inside a window the
    // pairs go heaviest first (latest query tokens, most keys) across its
    // groups.  The grid's tail then holds light pairs, while the K/V that a
    // window's pairs share stays within L2.
    const int P = p.pairs;
    const int wi = (int)(blockIdx.x / (unsigned)(kWindow * P));
    const int r = (int)blockIdx.x - wi * kWindow * P;
    const int g0 = wi * kWindow;
    const int wn = min(kWindow, p.groups - g0);
    const int pr = r / wn;
    const int grp = g0 + (r - pr * wn);
    const int pair = P - 1 - pr;
    const int b = grp / p.num_kv_heads;
    const int kvh = grp - b * p.num_kv_heads;
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int G = p.num_q_heads / p.num_kv_heads;
    const int TQ = kRows / G;  // query tokens per tile

    const int q0 = p.query_start[b];
    const int n = p.query_start[b + 1] - q0;
    const int L = p.context_lens[b];
    if (pair * kTiles * TQ >= n) return;  // uniform over the CTA
    if (n > L || (int64_t)L > (int64_t)p.max_blocks_per_seq * p.block_size) {
        if (threadIdx.x == 0 && pair == 0 && kvh == 0) record_error(p.err, PA_ERR_BAD_BLOCK_ID);
        return;
    }
    if (threadIdx.x == 0) PF_TL(0);
    // per tile: first query token, tokens, position of the first one, key tiles
    int t0[kTiles], nq[kTiles], pos_first[kTiles], nt[kTiles];
    int n_kv = 0, nt_cta = 0;
#pragma unroll
    for (int t = 0; t < kTiles; ++t) {
        t0[t] = (pair * kTiles + t) * TQ;
        nq[t] = max(0, min(TQ, n - t0[t]));
        pos_first[t] = L - n + t0[t];
        nt[t] = nq[t] > 0 ? (pos_first[t] + nq[t] + kKeys - 1) / kKeys : 0;
        if (nq[t] > 0) n_kv = pos_first[t] + nq[t];
        nt_cta = max(nt_cta, nt[t]);
    }

    if (threadIdx.x == 0) {
        s_abort = 0;
        prefetch_tmap(&tmq);
        prefetch_tmap(&tmk);
        prefetch_tmap(&tmv);
        mbar_init(&q_full, 1);
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&kv_full[s], 1);
            mbar_init(&kv_empty[s], kTiles);
        }
        for (int t = 0; t < kTiles; ++t)
            for (int s = 0; s < 2; ++s) {
                mbar_init(&s_full[t][s], 1);
                for (int h = 0; h < kHandoffs; ++h) mbar_init(&p_full[t][s][h], 4);
                mbar_init(&pv_done[t][s], 1);
            }
        fence_barrier_init();
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_addr(&tmem_base)),
                     "r"(kTiles * TILE_COLS));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = tmem_base;
    if (threadIdx.x == 0) PF_TL(1);

    if (warp == 0) {
        // ---------------- producer ----------------
        const int bs = p.block_size;
        const int boxes = kKeys / bs;  // pool boxes per tile and slab
        if (lane == 0) {
            uint32_t qbytes = 0;
#pragma unroll
            for (int t = 0; t < kTiles; ++t) qbytes += nq[t] > 0 ? (uint32_t)Q_BYTES : 0u;
            mbar_arrive_expect_tx(&q_full, qbytes);
#pragma unroll
            for (int t = 0; t < kTiles; ++t) {
                if (nq[t] == 0) continue;
#pragma unroll
                for (int sl = 0; sl < SLABS; ++sl)
                    tma_load_3d(sQ + t * Q_BYTES + sl * kRows * 128, &tmq, sl * 64, kvh * G, q0 + t0[t], &q_full);
            }
        }
        const int32_t* table = p.block_tables + (int64_t)b * p.max_blocks_per_seq;
        const uint64_t policy = l2_policy_evict_first();
        for (int j = 0; j < nt_cta; ++j) {
            const int s = j % kStages;
            if (j >= kStages) {
                int ok = 1;
                if (lane == 0) ok = mbar_wait(&kv_empty[s], ((j / kStages) - 1) & 1, p.err);
                if (!__shfl_sync(0xffffffffu, ok, 0)) {
                    if (lane == 0) s_abort = 1;
                    break;
                }
            }
            // lane i loads pool block i of the tile (if it holds keys < n_kv)
            const int key0 = j * kKeys + lane * bs;
            uint32_t bytes = 0;
            int y = 0;
            if (lane < boxes && key0 < n_kv) {
                const int32_t phys = table[key0 / bs];
                if (phys < 0 || phys >= p.num_blocks) {
                    record_error(p.err, PA_ERR_BAD_BLOCK_ID);
                } else {
                    bytes = (uint32_t)(2 * SLABS * bs * 128);
                    y = (phys * p.num_kv_heads + kvh) * bs;
                }
            }
            const uint32_t total = __reduce_add_sync(0xffffffffu, bytes);
            if (lane == 0) mbar_arrive_expect_tx(&kv_full[s], total);
            __syncwarp();
            if (bytes) {
#pragma unroll
                for (int sl = 0; sl < SLABS; ++sl) {
                    tma_load_2d(sK + s * KV_BYTES + sl * KV_SLAB + lane * bs * 128, &tmk, sl * 64, y, &kv_full[s],
                                policy);
                    tma_load_2d(sV + s * KV_BYTES + sl * KV_SLAB + lane * bs * 128, &tmv, sl * 64, y, &kv_full[s],
                                policy);
                }
            }
        }
    } else if (warp <= kTiles) {
        // ---------------- MMA issuers: warp 1 + t for query tile t ----------------
        // Each issuer runs its tile's chain on its own: S_j = Q_t . K_j^T, then
        // O_t += P_{j-1} . V_{j-1} once the softmax has written P_{j-1}.  Its
        // tcgen05.mma ops run in issue order, so S_j may overwrite the buffer
        // that held P_{j-2}.  A K/V stage is released when both issuers have
        // arrived; a tile that needs fewer key tiles arrives for the rest once
        // they are loaded (so the arrival lands in the right phase).
        const int t = warp - 1;
        if (lane == 0) {
            constexpr uint32_t IDESC_S = umma_idesc(kRows, kKeys, false);
            constexpr uint32_t IDESC_O = umma_idesc(kRows, D, true);
            const int ntt = t ? nt[1] : nt[0];
            const uint32_t q_base = smem_addr(sQ + t * Q_BYTES);
            bool ok = ntt == 0 || mbar_wait(&q_full, 0, p.err);
            for (int j = 0; ok && j <= ntt; ++j) {
                if (j < ntt) {
                    const int ks = j % kStages;
                    if (!(ok = mbar_wait(&kv_full[ks], (j / kStages) & 1, p.err))) break;
                    tc_fence_after();
                    const uint32_t k_base = smem_addr(sK + ks * KV_BYTES);
                    const uint32_t d_s = tmem + t * TILE_COLS + (j & 1) * S_COLS;
#pragma unroll
                    for (int kk = 0; kk < D / 16; ++kk) {
                        const uint32_t off = (kk & 3) * 32;
                        const uint64_t da = umma_desc(q_base + (kk >> 2) * (kRows * 128) + off, 16, 1024);
                        const uint64_t db = umma_desc(k_base + (kk >> 2) * KV_SLAB + off, 16, 1024);
                        umma(d_s, da, db, IDESC_S, kk > 0 ? 1u : 0u);
                    }
                    umma_commit(&s_full[t][j & 1]);
                    if (t == 0 && j == 0) PF_TL(2);
                }
                if (j >= 1) {
                    const int jp = j - 1;
                    const uint32_t v_base = smem_addr(sV + (jp % kStages) * KV_BYTES);
                    const uint32_t p_col = tmem + t * TILE_COLS + (jp & 1) * S_COLS;
                    // each part of P's keys as soon as the softmax has written it
#pragma unroll
                    for (int h = 0; h < kHandoffs; ++h) {
                        if (!(ok = mbar_wait(&p_full[t][jp & 1][h], (jp >> 1) & 1, p.err))) break;
                        tc_fence_after();
#pragma unroll
                        for (int kk = h * (kPartKeys / 16); kk < (h + 1) * (kPartKeys / 16); ++kk) {
                            const uint64_t db = umma_desc(v_base + kk * 2048, KV_SLAB, 1024);
                            umma_tmem_a(tmem + t * TILE_COLS + O_COL, p_col + kk * 8, db, IDESC_O,
                                        (jp > 0 || kk > 0) ? 1u : 0u);
                            if (kSplitP)
                                umma_tmem_a(tmem + t * TILE_COLS + O_COL, p_col + S_COLS / 2 + kk * 8, db, IDESC_O,
                                            1u);
                        }
                    }
                    if (!ok) break;
                    umma_commit(&pv_done[t][jp & 1]);
                    if (jp == ntt - 1) PF_TL(3 + t);
                    umma_commit(&kv_empty[jp % kStages]);
                }
            }
            for (int j = ntt; ok && j < nt_cta; ++j) {
                const int ks = j % kStages;
                if (!(ok = mbar_wait(&kv_full[ks], (j / kStages) & 1, p.err))) break;
                mbar_arrive(&kv_empty[ks]);
            }
            if (!ok) s_abort = 1;
        }
    } else {
        // ---------------- softmax / epilogue: one query row per thread ----------------
        const int t = (warp - 1 - kTiles) >> 2;      // query tile of this warpgroup
        const int quarter = warp & 3;                // TMEM lane quarter this warp may access
        const int row = quarter * 32 + lane;         // query row of the tile = TMEM lane
        const int tq = row / G;                      // query token within the tile
        const int my_t0 = t ? t0[1] : t0[0];
        const bool valid = tq < (t ? nq[1] : nq[0]);
        const int limit = valid ? (t ? pos_first[1] : pos_first[0]) + tq : -1;  // last key this row may see
        const uint32_t lane_base = tmem + ((uint32_t)(quarter * 32) << 16) + t * TILE_COLS;
        const int ntt = t ? nt[1] : nt[0];
        float m = -INFINITY, l = 0.f;  // running max (log2 units, scaled) and sum
        bool ok = true;
        for (int j = 0; j < ntt; ++j) {
            const int s = j & 1;
            if (!(ok = mbar_wait(&s_full[t][s], (j >> 1) & 1, p.err))) break;
            tc_fence_after();
            float sv[kKeys];
            tmem_ld32(lane_base + s * S_COLS, sv);
            tmem_ld32(lane_base + s * S_COLS + 32, sv + 32);
            tmem_wait_ld();
            const int kbase = j * kKeys;
            // With a positive scale (the usual case) the row max is taken on
            // the raw scores and the scale folds into the exponent's FMA;
            // otherwise the scores are scaled first.  Masked keys are -inf
            // either way.
            const bool fold = p.scale_log2 > 0.f;
            if (!fold) {
#pragma unroll
                for (int c = 0; c < kKeys; ++c) sv[c] *= p.scale_log2;
            }
            if (!__all_sync(0xffffffffu, kbase + kKeys - 1 <= limit)) {
#pragma unroll
                for (int c = 0; c < kKeys; ++c)
                    if (kbase + c > limit) sv[c] = -INFINITY;
            }
            // row max in eight independent chains
            float mx8[8];
#pragma unroll
            for (int c = 0; c < 8; ++c) mx8[c] = sv[c];
#pragma unroll
            for (int c = 8; c < kKeys; ++c) mx8[c & 7] = fmaxf(mx8[c & 7], sv[c]);
            float mx = fmaxf(fmaxf(fmaxf(mx8[0], mx8[1]), fmaxf(mx8[2], mx8[3])),
                             fmaxf(fmaxf(mx8[4], mx8[5]), fmaxf(mx8[6], mx8[7])));
            if (fold) mx *= p.scale_log2;
            // Lazy rescale: the weights are exp2(s - m) against a reference max
            // m that only moves when the row's max exceeds it by more than
            // kRescaleLog2 (weights stay <= 2^kRescaleLog2, far inside fp32 and
            // bf16 range); the result O / l does not depend on m.  Most tiles
            // then leave O alone and need not wait for the previous P.V.
            const bool grow = mx > m + kRescaleLog2;
            float alpha = 1.f;
            if (grow) {
                alpha = m == -INFINITY ? 0.f : exp2f(m - mx);
                m = mx;
            }
            // P_j over S_j's columns: bf16 high parts of the 64 weights in the
            // first 32 columns (two per column, lower key in the low half),
            // bf16 residuals in the last 32.  It goes to the MMA thread in
            // kHandoffs parts of kPartKeys keys (kPartKeys / 2 columns of each
            // of the two): a part's P.V runs while the next part's
            // exponentials are computed.
            float sum8[8];
#pragma unroll
            for (int c = 0; c < 8; ++c) sum8[c] = 0.f;
            const float neg_m = -m;
            const float mul = fold ? p.scale_log2 : 1.f;
#pragma unroll
            for (int h = 0; h < kHandoffs; ++h) {
#pragma unroll
                for (int c = kPartKeys * h; c < kPartKeys * (h + 1); ++c) {
                    sv[c] = m != -INFINITY ? ex2_approx(fmaf(sv[c], mul, neg_m)) : 0.f;
                    sum8[c & 7] += sv[c];
                }
                if (h == 0 && j > 0 && __any_sync(0xffffffffu, grow)) {
                    // O holds P.V of tiles < j: wait for the last of them, then
                    // rescale (before any of P_j is handed over)
                    if (!(ok = mbar_wait(&pv_done[t][(j - 1) & 1], ((j - 1) >> 1) & 1, p.err))) break;
                    tc_fence_after();
#pragma unroll
                    for (int c0 = 0; c0 < D; c0 += 32) {
                        float ov[32];
                        tmem_ld32(lane_base + O_COL + c0, ov);
                        tmem_wait_ld();
#pragma unroll
                        for (int i = 0; i < 32; ++i) ov[i] *= alpha;
                        tmem_st32(lane_base + O_COL + c0, ov);
                    }
                }
                constexpr int PC = kPartKeys / 2;  // columns of one part
                uint32_t hi[PC], lo[PC];
#pragma unroll
                for (int c = 0; c < PC; ++c) {
                    const float a = sv[kPartKeys * h + 2 * c], bb = sv[kPartKeys * h + 2 * c + 1];
                    hi[c] = pack_bf16x2(a, bb);
                    if (kSplitP) lo[c] = pack_bf16x2(a - bf16_lo_to_f32(hi[c]), bb - bf16_hi_to_f32(hi[c]));
                }
                if constexpr (PC == 16) {
                    tmem_st16u(lane_base + s * S_COLS + PC * h, hi);
                    if (kSplitP) tmem_st16u(lane_base + s * S_COLS + S_COLS / 2 + PC * h, lo);
                } else {
                    tmem_st8u(lane_base + s * S_COLS + PC * h, hi);
                    if (kSplitP) tmem_st8u(lane_base + s * S_COLS + S_COLS / 2 + PC * h, lo);
                }
                // keys past the sequence end carry weight 0, but 0 * NaN is NaN
                // in the MMA: zero those V rows of the CTA's last tile (both
                // warpgroups that use it do, each before it signals its first
                // part of P)
                if (h == 0 && j == nt_cta - 1 && n_kv < nt_cta * kKeys) {
                    uint8_t* vs = sV + (j % kStages) * KV_BYTES;
                    const int first = n_kv - j * kKeys;
                    const int nch = (kKeys - first) * SLABS * 8;
                    for (int c = row; c < nch; c += 128) {
                        const int r = first + c / (SLABS * 8);
                        const int rem = c % (SLABS * 8);
                        *reinterpret_cast<uint4*>(vs + (rem >> 3) * KV_SLAB + r * 128 + (rem & 7) * 16) =
                            make_uint4(0u, 0u, 0u, 0u);
                    }
                    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
                }
                tmem_wait_st();
                // each warp signals its 32 rows' part of P (and its share of
                // the V zeroing) to the MMA thread once all its lanes are done
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&p_full[t][s][h]);
            }
            if (!ok) break;
            l = l * alpha + (((sum8[0] + sum8[1]) + (sum8[2] + sum8[3])) + ((sum8[4] + sum8[5]) + (sum8[6] + sum8[7])));
        }
        // epilogue: O / l for this row.  A whole tile with bf16 output is
        // staged in the tile's Q buffer (its S MMAs are done), laid out as a
        // Q tile is loaded (row r, 16-byte chunk c of a 64-element slab at
        // chunk c ^ (r & 7)), and written by tiled TMA stores through the
        // output map; other tiles store their rows directly.
        if (ok && ntt > 0 && (ok = mbar_wait(&pv_done[t][(ntt - 1) & 1], ((ntt - 1) >> 1) & 1, p.err))) {
            tc_fence_after();
            const float inv = l > 0.f ? 1.f / l : 0.f;
            if (p.out_bf16 && (t ? nq[1] : nq[0]) == TQ) {
                uint8_t* so = sQ + t * Q_BYTES;
#pragma unroll
                for (int c0 = 0; c0 < D; c0 += 32) {
                    float ov[32];
                    tmem_ld32(lane_base + O_COL + c0, ov);
                    tmem_wait_ld();
                    uint8_t* slab_row = so + (c0 >> 6) * (kRows * 128) + row * 128;
#pragma unroll
                    for (int q4 = 0; q4 < 4; ++q4) {
                        const int c = ((c0 & 63) >> 3) + q4;
                        const float* v = ov + 8 * q4;
                        *reinterpret_cast<uint4*>(slab_row + ((c ^ (row & 7)) << 4)) =
                            make_uint4(pack_bf16x2(v[0] * inv, v[1] * inv), pack_bf16x2(v[2] * inv, v[3] * inv),
                                       pack_bf16x2(v[4] * inv, v[5] * inv), pack_bf16x2(v[6] * inv, v[7] * inv));
                    }
                }
                fence_proxy_async_smem();  // the TMA store reads the rows through the async proxy
                asm volatile("bar.sync %0, 128;" ::"r"(1 + t) : "memory");  // the warpgroup's 128 rows
                if (quarter == 0 && lane == 0) {
#pragma unroll
                    for (int sl = 0; sl < SLABS; ++sl)
                        tma_store_3d(&tmo, sl * 64, kvh * G, q0 + my_t0, so + sl * (kRows * 128));
                    bulk_commit_group();
                    bulk_wait_group_read0();
                }
            } else {
            const int64_t orow =
                ((int64_t)(q0 + my_t0 + tq) * p.num_q_heads + (int64_t)kvh * G + (row % G)) * D;
#pragma unroll
            for (int c0 = 0; c0 < D; c0 += 32) {
                float ov[32];
                tmem_ld32(lane_base + O_COL + c0, ov);
                tmem_wait_ld();
                if (valid) {
                    if (p.out_bf16) {
                        uint4* o = reinterpret_cast<uint4*>(static_cast<uint16_t*>(p.out) + orow + c0);
#pragma unroll
                        for (int i = 0; i < 32; i += 8)
                            o[i / 8] = make_uint4(pack_bf16x2(ov[i] * inv, ov[i + 1] * inv),
                                                  pack_bf16x2(ov[i + 2] * inv, ov[i + 3] * inv),
                                                  pack_bf16x2(ov[i + 4] * inv, ov[i + 5] * inv),
                                                  pack_bf16x2(ov[i + 6] * inv, ov[i + 7] * inv));
                    } else {
                        float4* o = reinterpret_cast<float4*>(static_cast<float*>(p.out) + orow + c0);
#pragma unroll
                        for (int i = 0; i < 32; i += 4)
                            o[i / 4] = make_float4(ov[i] * inv, ov[i + 1] * inv, ov[i + 2] * inv, ov[i + 3] * inv);
                    }
                }
            }
            }
        }
        if (!ok) s_abort = 1;
    }
    tc_fence_before();
    __syncthreads();
    if (threadIdx.x == 0) PF_TL(5);
    if (warp == 1) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTiles * TILE_COLS));
    }
}

// ---- host side -------------------------------------------------------------
using TensorMapEncodeFn = PFN_cuTensorMapEncodeTiled_v12000;

TensorMapEncodeFn encoder() {
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

int encode(CUtensorMap* map, const void* base, int rank, const cuuint64_t* dims, const cuuint64_t* strides,
           const cuuint32_t* box) {
    TensorMapEncodeFn enc = encoder();
    if (!enc) return PA_ERR_CUDA;
    cuuint32_t es[3] = {1u, 1u, 1u};
    const CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, rank, const_cast<void*>(base), dims, strides, box, es,
                           CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                           CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? PA_OK : PA_ERR_CUDA;
}

template <int D>
size_t prefill_smem_bytes() {
    constexpr int SLABS = D / 64;
    // at least 120 KB so that one CTA, holding all 512 TMEM columns, is
    // alone on its SM (the head_dim 64 tiles alone would let two fit)
    const size_t need = 1024 + kTiles * SLABS * kRows * 128 + 2 * kStages * SLABS * kKeys * 128;
    return need < 120 * 1024 ? 120 * 1024 : need;
}

template <int D>
int launch_prefill(const PrefillParams& p, const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                   const CUtensorMap& to, dim3 grid, cudaStream_t st) {
    static std::atomic<unsigned long long> configured{0};
    const size_t smem = prefill_smem_bytes<D>();
    int dev = 0;
    cudaGetDevice(&dev);
    const unsigned long long bit = 1ull << (dev & 63);
    if (!(configured.load() & bit)) {
        if (cudaFuncSetAttribute(prefill_tc_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) !=
            cudaSuccess)
            return PA_ERR_CUDA;
        configured.fetch_or(bit);
    }
    prefill_tc_kernel<D><<<grid, kThreads, smem, st>>>(p, tq, tk, tv, to);
    return launch_status();
}

}  // namespace
}  // namespace pa

using namespace pa;

extern "C" int pa_paged_attention_prefill(const void* q, const void* k_pool, const void* v_pool,
                                          const int32_t* block_tables, int max_blocks_per_seq,
                                          const int32_t* context_lens, const int32_t* query_start,
                                          int max_query_len, float scale, int block_size, void* out,
                                          int out_dtype, int batch, int num_q_heads, int num_kv_heads,
                                          int head_dim, int64_t num_tokens, int64_t num_blocks, int kv_dtype,
                                          void* stream) {
    PA_NVTX_RANGE("pa_paged_attention_prefill");
    if (batch < 0 || num_q_heads <= 0 || num_kv_heads <= 0 || head_dim <= 0 || block_size <= 0 ||
        max_query_len < 0 || num_tokens < 0 || num_blocks < 0 || max_blocks_per_seq < 0 || !valid_dtype(kv_dtype) ||
        !valid_dtype(out_dtype) || num_q_heads % num_kv_heads != 0)
        return PA_ERR_INVALID_ARG;
    const int G = num_q_heads / num_kv_heads;
    if (kv_dtype != PA_BF16 || !supported_head_dim(head_dim) || !supported_block_size(block_size) ||
        (G != 1 && G != 2 && G != 4 && G != 8 && G != 16))
        return PA_ERR_UNSUPPORTED;
    if (batch == 0 || num_tokens == 0 || max_query_len == 0) return PA_OK;
    if (!q || !k_pool || !v_pool || !block_tables || !context_lens || !query_start || !out) return PA_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k_pool) || !aligned16(v_pool) || !aligned16(out)) return PA_ERR_INVALID_ARG;
    const uint64_t pool_rows = (uint64_t)num_blocks * num_kv_heads * (uint64_t)block_size;
    if (pool_rows >= (1ull << 31) || num_tokens >= (1ll << 31)) return PA_ERR_UNSUPPORTED;
    int* err = error_word_ptr();
    if (!err) return PA_ERR_CUDA;

    CUtensorMap tq, tk, tv, to;
    const int TQ = kRows / G;
    {
        // q, and bf16 out (the same [num_tokens][Hq][D] geometry) for the
        // epilogue's stores of whole tiles
        cuuint64_t dims[3] = {(cuuint64_t)head_dim, (cuuint64_t)num_q_heads, (cuuint64_t)num_tokens};
        cuuint64_t strides[2] = {(cuuint64_t)head_dim * 2, (cuuint64_t)num_q_heads * head_dim * 2};
        cuuint32_t box[3] = {64u, (cuuint32_t)G, (cuuint32_t)TQ};
        int rc = encode(&tq, q, 3, dims, strides, box);
        if (!rc) rc = out_dtype == PA_BF16 ? encode(&to, out, 3, dims, strides, box) : (to = tq, PA_OK);
        if (rc) return rc;
    }
    {
        cuuint64_t dims[2] = {(cuuint64_t)head_dim, pool_rows > 0 ? pool_rows : 1};
        cuuint64_t strides[1] = {(cuuint64_t)head_dim * 2};
        cuuint32_t box[2] = {64u, (cuuint32_t)block_size};
        int rc = encode(&tk, k_pool, 2, dims, strides, box);
        if (!rc) rc = encode(&tv, v_pool, 2, dims, strides, box);
        if (rc) return rc;
    }
    PrefillParams p = {};
    p.q = q;
    p.out = out;
    p.block_tables = block_tables;
    p.context_lens = context_lens;
    p.query_start = query_start;
    p.err = err;
    p.num_blocks = num_blocks;
    p.max_blocks_per_seq = max_blocks_per_seq;
    p.num_q_heads = num_q_heads;
    p.num_kv_heads = num_kv_heads;
    p.block_size = block_size;
    p.out_bf16 = out_dtype == PA_BF16;
    p.scale_log2 = scale * kLog2e;
    const int q_tiles = (max_query_len + TQ - 1) / TQ;
    p.pairs = (q_tiles + kTiles - 1) / kTiles;
    p.groups = batch * num_kv_heads;
    const int64_t ctas = (int64_t)p.pairs * p.groups;
    if (ctas > INT32_MAX) return PA_ERR_UNSUPPORTED;
    dim3 grid((unsigned)ctas);
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    return head_dim == 128 ? launch_prefill<128>(p, tq, tk, tv, to, grid, st)
                           : launch_prefill<64>(p, tq, tk, tv, to, grid, st);
}

#ifdef PA_TIMELINE
extern "C" int pa_timeline_clear_prefill(void) {
    void* a = nullptr;
    if (cudaGetSymbolAddress(&a, pa::g_pa_prefill_tl) != cudaSuccess ||
        cudaMemset(a, 0, sizeof(pa::g_pa_prefill_tl)) != cudaSuccess || cudaDeviceSynchronize() != cudaSuccess)
        return PA_ERR_CUDA;
    return PA_OK;
}

extern "C" int pa_timeline_read_prefill(void* dst, size_t bytes) {
    if (!dst || bytes > sizeof(pa::g_pa_prefill_tl)) return PA_ERR_INVALID_ARG;
    return cudaMemcpyFromSymbol(dst, pa::g_pa_prefill_tl, bytes) == cudaSuccess ? PA_OK : PA_ERR_CUDA;
}
#endif
