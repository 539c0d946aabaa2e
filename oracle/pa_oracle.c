/*
 * pa_oracle.c -- plain, slow, obviously correct CPU oracle for the paged
 * KV-cache decode path.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path may link, load or
 * call this file; only the tests, the smoke check and the benchmark's CPU
 * baseline leg do.  It shares no code, header, table or helper with the CUDA
 * library: it includes nothing but the C standard library and OpenMP.
 *
 * What it computes, and where the pages define it:
 *
 *  - oracle_paged_decode / oracle_paged_decode_rows
 *      "PagedAttention and KV memory management", section "The kernel side":
 *      attention over K and V that live in a pool of fixed-size blocks,
 *      reached through a per-sequence block table.  The GPU path must not
 *      gather; this oracle deliberately does: it walks the block table into
 *      contiguous fp64 K and V (logical block i of a sequence lives in
 *      physical block block_table[i], token t at offset t % block_size,
 *      as in the worked mapping of "How does vLLM PagedAttention manage
 *      Virtual Memory Pages ...", section "Detail"), then runs textbook
 *      two-pass softmax attention:
 *          s_t = scale * <q, k_t>,  m = max_t s_t,  w_t = exp(s_t - m),
 *          out = (sum_t w_t v_t) / (sum_t w_t).
 *      Query head h reads kv head h / G with G = Hq / Hkv (consecutive query
 *      heads share a kv head; the pages are silent on grouped heads).
 *      A sequence of length 0 yields a zero row.
 *
 *  - oracle_paged_prefill
 *      several new query tokens per sequence over the same paged cache
 *      (chunked prefill): a sequence of length L with n new queries has query
 *      i (0-based) at position p = L - n + i, attending keys 0..p (causal);
 *      each query row is the attention above with the first p + 1 tokens.
 *
 *  - oracle_contiguous_decode
 *      the same attention over a contiguous [B, Hkv, L_pad, D] cache, the
 *      "ideal contiguous attention" the same section compares against.
 *
 *  - oracle_slot_mapping
 *      the slot of token position pos of sequence b is
 *      block_table[b][pos / block_size] * block_size + pos % block_size
 *      (the worked virtual-to-physical mapping, section "Detail", with the
 *      in-block offset pos % block_size).
 *
 *  - oracle_reshape_and_cache
 *      writes each new token's K and V into its slot, one block allocated at
 *      a time as generation proceeds ("Key Technical Innovations", item 2).
 *
 *  - oracle_copy_blocks
 *      copy-on-write: "Paged Attention: OS-Inspired Memory Management for KV
 *      Caches", section "Key terms in this lesson" (Copy-on-write): a shared
 *      block is duplicated so that the writer gets a private copy.
 *
 *  - oracle_round_bf16
 *      rounds fp64 values once to bfloat16, round to nearest, ties to even.
 *
 * Pool layout (the pages fix none): k_pool and v_pool are each
 * [num_blocks, Hkv, block_size, D] row-major.  dtype 0 = fp32, 1 = bf16
 * (bf16 data is passed as raw 16-bit words and widened exactly).
 *
 * Return codes: 0 ok, 1 invalid argument (including a block id outside the
 * pool or a length beyond the block table), never partial silent output.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define OR_F32 0
#define OR_BF16 1

static size_t elt_size(int dtype) { return dtype == OR_BF16 ? 2u : 4u; }

/* Exact widening of one stored element to double. */
static double widen(const void* base, int64_t idx, int dtype) {
    if (dtype == OR_F32) return (double)((const float*)base)[idx];
    uint32_t bits = (uint32_t)((const uint16_t*)base)[idx] << 16;
    float f;
    memcpy(&f, &bits, sizeof f);
    return (double)f;
}

int oracle_num_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* Textbook two-pass softmax attention of one query row over L contiguous
 * fp64 keys/values.  o receives D values. */
static int attend(const double* qrow, const double* Kc, const double* Vc,
                  int64_t L, int D, double scale, double* o) {
    for (int d = 0; d < D; ++d) o[d] = 0.0;
    if (L == 0) return 0;
    double* s = (double*)malloc((size_t)L * sizeof(double));
    if (!s) return 1;
    double m = -INFINITY;
    for (int64_t t = 0; t < L; ++t) {
        double acc = 0.0;
        for (int d = 0; d < D; ++d) acc += qrow[d] * Kc[t * D + d];
        s[t] = scale * acc;
        if (s[t] > m) m = s[t];
    }
    double Z = 0.0;
    for (int64_t t = 0; t < L; ++t) {
        double w = exp(s[t] - m);
        Z += w;
        for (int d = 0; d < D; ++d) o[d] += w * Vc[t * D + d];
    }
    for (int d = 0; d < D; ++d) o[d] /= Z;
    free(s);
    return 0;
}

/* Walk one sequence's block table into contiguous fp64 K and V for kv head
 * kvh.  Returns 1 if a table entry points outside the pool. */
static int gather_paged(const void* k_pool, const void* v_pool,
                        const int32_t* table_row, int64_t L, int kvh,
                        int Hkv, int block_size, int D, int64_t num_blocks,
                        int dtype, double* Kc, double* Vc) {
    for (int64_t t = 0; t < L; ++t) {
        int64_t logical = t / block_size;
        int64_t offset = t % block_size;
        int64_t phys = table_row[logical];
        if (phys < 0 || phys >= num_blocks) return 1;
        int64_t row = ((phys * Hkv + kvh) * block_size + offset) * D;
        for (int d = 0; d < D; ++d) {
            Kc[t * D + d] = widen(k_pool, row + d, dtype);
            Vc[t * D + d] = widen(v_pool, row + d, dtype);
        }
    }
    return 0;
}

static int check_common(int batch, int Hq, int Hkv, int D, int dtype) {
    if (batch < 0 || Hq <= 0 || Hkv <= 0 || D <= 0) return 1;
    if (Hq % Hkv != 0) return 1;
    if (dtype != OR_F32 && dtype != OR_BF16) return 1;
    return 0;
}

/* Compute the output rows (rows_b[i], rows_h[i]) for i < nrows into
 * out[i * D + d].  Rows are independent; OpenMP splits them across cores. */
int oracle_paged_decode_rows(const void* q, const void* k_pool, const void* v_pool,
                             const int32_t* block_tables, int max_blocks_per_seq,
                             const int32_t* context_lens, float scale, int block_size,
                             int batch, int Hq, int Hkv, int D, int64_t num_blocks,
                             int dtype, const int32_t* rows_b, const int32_t* rows_h,
                             int64_t nrows, double* out) {
    if (check_common(batch, Hq, Hkv, D, dtype) || block_size <= 0 ||
        max_blocks_per_seq < 0 || nrows < 0)
        return 1;
    const int G = Hq / Hkv;
    for (int64_t i = 0; i < nrows; ++i) {
        if (rows_b[i] < 0 || rows_b[i] >= batch || rows_h[i] < 0 || rows_h[i] >= Hq) return 1;
        int64_t L = context_lens[rows_b[i]];
        if (L < 0 || L > (int64_t)max_blocks_per_seq * block_size) return 1;
    }
    int bad = 0;
#pragma omp parallel for schedule(dynamic, 1) reduction(| : bad)
    for (int64_t i = 0; i < nrows; ++i) {
        const int b = rows_b[i], h = rows_h[i], kvh = h / G;
        const int64_t L = context_lens[b];
        double* Kc = (double*)malloc((size_t)(L > 0 ? L : 1) * D * sizeof(double));
        double* Vc = (double*)malloc((size_t)(L > 0 ? L : 1) * D * sizeof(double));
        double* qrow = (double*)malloc((size_t)D * sizeof(double));
        if (!Kc || !Vc || !qrow) {
            bad |= 1;
        } else {
            for (int d = 0; d < D; ++d) qrow[d] = widen(q, ((int64_t)b * Hq + h) * D + d, dtype);
            if (gather_paged(k_pool, v_pool, block_tables + (int64_t)b * max_blocks_per_seq, L,
                             kvh, Hkv, block_size, D, num_blocks, dtype, Kc, Vc))
                bad |= 1;
            else
                bad |= attend(qrow, Kc, Vc, L, D, (double)scale, out + i * D);
        }
        free(Kc);
        free(Vc);
        free(qrow);
    }
    return bad;
}

/* Every output row, out[(b * Hq + h) * D + d].  One task per (b, kv head):
 * the gather is done once and shared by the G query heads of the group. */
int oracle_paged_decode(const void* q, const void* k_pool, const void* v_pool,
                        const int32_t* block_tables, int max_blocks_per_seq,
                        const int32_t* context_lens, float scale, int block_size,
                        int batch, int Hq, int Hkv, int D, int64_t num_blocks,
                        int dtype, double* out) {
    if (check_common(batch, Hq, Hkv, D, dtype) || block_size <= 0 || max_blocks_per_seq < 0)
        return 1;
    for (int b = 0; b < batch; ++b) {
        int64_t L = context_lens[b];
        if (L < 0 || L > (int64_t)max_blocks_per_seq * block_size) return 1;
    }
    const int G = Hq / Hkv;
    const int64_t tasks = (int64_t)batch * Hkv;
    int bad = 0;
#pragma omp parallel for schedule(dynamic, 1) reduction(| : bad)
    for (int64_t task = 0; task < tasks; ++task) {
        const int b = (int)(task / Hkv), kvh = (int)(task % Hkv);
        const int64_t L = context_lens[b];
        double* Kc = (double*)malloc((size_t)(L > 0 ? L : 1) * D * sizeof(double));
        double* Vc = (double*)malloc((size_t)(L > 0 ? L : 1) * D * sizeof(double));
        double* qrow = (double*)malloc((size_t)D * sizeof(double));
        if (!Kc || !Vc || !qrow) {
            bad |= 1;
        } else if (gather_paged(k_pool, v_pool, block_tables + (int64_t)b * max_blocks_per_seq,
                                L, kvh, Hkv, block_size, D, num_blocks, dtype, Kc, Vc)) {
            bad |= 1;
        } else {
            for (int g = 0; g < G; ++g) {
                const int h = kvh * G + g;
                for (int d = 0; d < D; ++d) qrow[d] = widen(q, ((int64_t)b * Hq + h) * D + d, dtype);
                bad |= attend(qrow, Kc, Vc, L, D, (double)scale, out + ((int64_t)b * Hq + h) * D);
            }
        }
        free(Kc);
        free(Vc);
        free(qrow);
    }
    return bad;
}

/* Causal multi-query attention.  q and out rows: [T, Hq, D] with sequence b
 * owning rows query_start[b] .. query_start[b + 1] - 1, its last n_b tokens. */
int oracle_paged_prefill(const void* q, const void* k_pool, const void* v_pool,
                         const int32_t* block_tables, int max_blocks_per_seq,
                         const int32_t* context_lens, const int32_t* query_start, float scale,
                         int block_size, int batch, int Hq, int Hkv, int D, int64_t num_blocks,
                         int dtype, double* out) {
    if (check_common(batch, Hq, Hkv, D, dtype) || block_size <= 0 || max_blocks_per_seq < 0)
        return 1;
    for (int b = 0; b < batch; ++b) {
        const int64_t L = context_lens[b];
        const int64_t n = (int64_t)query_start[b + 1] - query_start[b];
        if (L < 0 || L > (int64_t)max_blocks_per_seq * block_size || n < 0 || n > L) return 1;
    }
    const int G = Hq / Hkv;
    const int64_t tasks = (int64_t)batch * Hkv;
    int bad = 0;
#pragma omp parallel for schedule(dynamic, 1) reduction(| : bad)
    for (int64_t task = 0; task < tasks; ++task) {
        const int b = (int)(task / Hkv), kvh = (int)(task % Hkv);
        const int64_t L = context_lens[b];
        const int64_t n = (int64_t)query_start[b + 1] - query_start[b];
        double* Kc = (double*)malloc((size_t)(L > 0 ? L : 1) * D * sizeof(double));
        double* Vc = (double*)malloc((size_t)(L > 0 ? L : 1) * D * sizeof(double));
        double* qrow = (double*)malloc((size_t)D * sizeof(double));
        if (!Kc || !Vc || !qrow) {
            bad |= 1;
        } else if (gather_paged(k_pool, v_pool, block_tables + (int64_t)b * max_blocks_per_seq,
                                L, kvh, Hkv, block_size, D, num_blocks, dtype, Kc, Vc)) {
            bad |= 1;
        } else {
            for (int64_t i = 0; i < n; ++i) {
                const int64_t pos = L - n + i;
                const int64_t row = query_start[b] + i;
                for (int g = 0; g < G; ++g) {
                    const int h = kvh * G + g;
                    for (int d = 0; d < D; ++d) qrow[d] = widen(q, (row * Hq + h) * D + d, dtype);
                    bad |= attend(qrow, Kc, Vc, pos + 1, D, (double)scale, out + (row * Hq + h) * D);
                }
            }
        }
        free(Kc);
        free(Vc);
        free(qrow);
    }
    return bad;
}

/* Attention over a contiguous cache k_c, v_c: [B, Hkv, L_pad, D]. */
int oracle_contiguous_decode(const void* q, const void* k_c, const void* v_c, int L_pad,
                             const int32_t* context_lens, float scale, int batch, int Hq,
                             int Hkv, int D, int dtype, double* out) {
    if (check_common(batch, Hq, Hkv, D, dtype) || L_pad < 0) return 1;
    for (int b = 0; b < batch; ++b)
        if (context_lens[b] < 0 || context_lens[b] > L_pad) return 1;
    const int G = Hq / Hkv;
    const int64_t tasks = (int64_t)batch * Hkv;
    int bad = 0;
#pragma omp parallel for schedule(dynamic, 1) reduction(| : bad)
    for (int64_t task = 0; task < tasks; ++task) {
        const int b = (int)(task / Hkv), kvh = (int)(task % Hkv);
        const int64_t L = context_lens[b];
        double* Kc = (double*)malloc((size_t)(L > 0 ? L : 1) * D * sizeof(double));
        double* Vc = (double*)malloc((size_t)(L > 0 ? L : 1) * D * sizeof(double));
        double* qrow = (double*)malloc((size_t)D * sizeof(double));
        if (!Kc || !Vc || !qrow) {
            bad |= 1;
        } else {
            const int64_t base = ((int64_t)b * Hkv + kvh) * L_pad * D;
            for (int64_t t = 0; t < L; ++t)
                for (int d = 0; d < D; ++d) {
                    Kc[t * D + d] = widen(k_c, base + t * D + d, dtype);
                    Vc[t * D + d] = widen(v_c, base + t * D + d, dtype);
                }
            for (int g = 0; g < G; ++g) {
                const int h = kvh * G + g;
                for (int d = 0; d < D; ++d) qrow[d] = widen(q, ((int64_t)b * Hq + h) * D + d, dtype);
                bad |= attend(qrow, Kc, Vc, L, D, (double)scale, out + ((int64_t)b * Hq + h) * D);
            }
        }
        free(Kc);
        free(Vc);
        free(qrow);
    }
    return bad;
}

/* slots[i] for token i of sequence seq_ids[i] at position positions[i]. */
int oracle_slot_mapping(const int32_t* block_tables, int max_blocks_per_seq, int batch,
                        const int32_t* seq_ids, const int32_t* positions, int64_t num_tokens,
                        int block_size, int64_t* slots) {
    if (block_size <= 0 || max_blocks_per_seq < 0 || num_tokens < 0) return 1;
    for (int64_t i = 0; i < num_tokens; ++i) {
        const int b = seq_ids[i];
        const int64_t pos = positions[i];
        if (b < 0 || b >= batch || pos < 0 || pos / block_size >= max_blocks_per_seq) return 1;
        const int64_t phys = block_tables[(int64_t)b * max_blocks_per_seq + pos / block_size];
        if (phys < 0) return 1;
        slots[i] = phys * block_size + pos % block_size;
    }
    return 0;
}

/* k_pool[slot / bs, h, slot % bs, :] = key[i, h, :] (and the same for V);
 * a negative slot means "skip this token". */
int oracle_reshape_and_cache(const void* key, const void* value, void* k_pool, void* v_pool,
                             const int64_t* slots, int64_t num_tokens, int Hkv, int D,
                             int block_size, int64_t num_blocks, int dtype) {
    if (Hkv <= 0 || D <= 0 || block_size <= 0 || num_tokens < 0) return 1;
    if (dtype != OR_F32 && dtype != OR_BF16) return 1;
    const size_t row_bytes = (size_t)D * elt_size(dtype);
    for (int64_t i = 0; i < num_tokens; ++i) {
        const int64_t s = slots[i];
        if (s < 0) continue;
        const int64_t blk = s / block_size, off = s % block_size;
        if (blk >= num_blocks) return 1;
        for (int h = 0; h < Hkv; ++h) {
            const int64_t dst = ((blk * Hkv + h) * block_size + off);
            const int64_t src = i * Hkv + h;
            memcpy((char*)k_pool + dst * row_bytes, (const char*)key + src * row_bytes, row_bytes);
            memcpy((char*)v_pool + dst * row_bytes, (const char*)value + src * row_bytes, row_bytes);
        }
    }
    return 0;
}

/* For each pair p (in order): block mapping[p][1] := block mapping[p][0],
 * whole K block and whole V block. */
int oracle_copy_blocks(void* k_pool, void* v_pool, const int64_t* block_mapping,
                       int64_t num_pairs, int Hkv, int D, int block_size, int64_t num_blocks,
                       int dtype) {
    if (Hkv <= 0 || D <= 0 || block_size <= 0 || num_pairs < 0) return 1;
    if (dtype != OR_F32 && dtype != OR_BF16) return 1;
    const size_t block_bytes = (size_t)Hkv * block_size * D * elt_size(dtype);
    for (int64_t p = 0; p < num_pairs; ++p) {
        const int64_t src = block_mapping[2 * p], dst = block_mapping[2 * p + 1];
        if (src < 0 || src >= num_blocks || dst < 0 || dst >= num_blocks) return 1;
        memmove((char*)k_pool + dst * block_bytes, (const char*)k_pool + src * block_bytes, block_bytes);
        memmove((char*)v_pool + dst * block_bytes, (const char*)v_pool + src * block_bytes, block_bytes);
    }
    return 0;
}

/* Round each double once to bfloat16 (8 significant bits, exponent range of
 * fp32), round to nearest with ties to even; returns the 16-bit patterns. */
void oracle_round_bf16(const double* in, int64_t n, uint16_t* out) {
    for (int64_t i = 0; i < n; ++i) {
        const double x = in[i];
        uint32_t bits;
        float f;
        if (isnan(x)) {
            out[i] = 0x7fc0;
            continue;
        }
        double r;
        if (x == 0.0 || isinf(x)) {
            r = x;
        } else {
            int e;
            (void)frexp(x, &e); /* |x| = m * 2^e, m in [0.5, 1) */
            /* quantum of a bf16 with that exponent; subnormals share 2^-133 */
            int qexp = e - 8;
            if (qexp < -133) qexp = -133;
            const double quantum = ldexp(1.0, qexp);
            r = nearbyint(x / quantum) * quantum; /* default mode: ties to even */
            /* largest finite bf16 is (2 - 2^-7) * 2^127 */
            if (fabs(r) > ldexp(255.0, 120)) r = copysign(INFINITY, x);
        }
        f = (float)r; /* exact: r is representable in bf16, hence in fp32 */
        memcpy(&bits, &f, sizeof bits);
        out[i] = (uint16_t)(bits >> 16);
    }
}
