// pa_block_manager.cpp -- host-side KV block manager of libpa.
//
// What it models (the pages' allocator):
//  * fixed-size blocks of block_size tokens, a per-sequence block table that
//    maps logical block i to a physical block, one block allocated at a time
//    as the sequence grows ("PagedAttention and KV memory management",
//    introduction; "How does vLLM PagedAttention manage Virtual Memory Pages
//    ...", sections "Detail" and "Key Technical Innovations" items 1-2);
//  * a free list that starts as every block id in increasing order and is
//    used first-in first-out (same page, section "Example"); freed blocks go
//    back to its tail;
//  * reference counts and copy-on-write ("Paged Attention: OS-Inspired Memory
//    Management for KV Caches", section "Key terms in this lesson"): a fork
//    shares every block of the parent; a write into a block whose count is
//    above one first moves the writer onto a private copy (a (src, dst) pair
//    for pa_copy_blocks), the last sharer writes in place.
// A token at position pos needs a new block when pos % block_size == 0; its
// slot is table[pos / block_size] * block_size + pos % block_size.
//
// The free list is a ring buffer of block ids (pop at the head, push at the
// tail), reference counts a flat array, tables per sequence id in a hash map:
// every operation is O(1) amortised except fork and free, which are O(blocks
// of the sequence).  Not thread-safe: one manager per scheduler thread.
#include <stdint.h>

#include <new>
#include <unordered_map>
#include <vector>

#include "pa.h"

struct pa_block_manager {
    int64_t num_blocks;
    int block_size;
    std::vector<int64_t> ring;  // free block ids, FIFO
    int64_t head = 0;           // index of the next block to hand out
    int64_t count = 0;          // free blocks in the ring
    std::vector<int32_t> refcount;
    struct Seq {
        std::vector<int32_t> table;
        int64_t length = 0;
    };
    std::unordered_map<int64_t, Seq> seqs;

    pa_block_manager(int64_t nb, int bs) : num_blocks(nb), block_size(bs), ring(nb), refcount(nb, 0) {
        for (int64_t i = 0; i < nb; ++i) ring[i] = i;
        count = nb;
    }
    bool take(int32_t* blk) {
        if (count == 0) return false;
        *blk = (int32_t)ring[head];
        head = (head + 1) % num_blocks;
        --count;
        refcount[*blk] = 1;
        return true;
    }
    void release(int32_t blk) {
        if (--refcount[blk] == 0) {
            ring[(head + count) % num_blocks] = blk;
            ++count;
        }
    }
};

extern "C" pa_block_manager* pa_bm_create(int64_t num_blocks, int block_size) {
    if (num_blocks <= 0 || num_blocks > INT32_MAX || block_size <= 0) return nullptr;
    return new (std::nothrow) pa_block_manager(num_blocks, block_size);
}

extern "C" void pa_bm_destroy(pa_block_manager* bm) { delete bm; }

extern "C" int pa_bm_add_sequence(pa_block_manager* bm, int64_t seq) {
    if (!bm) return PA_ERR_INVALID_ARG;
    if (bm->seqs.count(seq)) return PA_ERR_INVALID_ARG;
    bm->seqs.emplace(seq, pa_block_manager::Seq{});
    return PA_OK;
}

extern "C" int pa_bm_append_tokens(pa_block_manager* bm, const int64_t* seq_ids, int64_t n, int64_t* slots,
                                   int64_t* cow_pairs, int64_t* num_cow_pairs) {
    if (!bm || n < 0 || (n > 0 && (!seq_ids || !slots)) || !num_cow_pairs) return PA_ERR_INVALID_ARG;
    *num_cow_pairs = 0;
    for (int64_t i = 0; i < n; ++i) {
        auto it = bm->seqs.find(seq_ids[i]);
        if (it == bm->seqs.end()) it = bm->seqs.emplace(seq_ids[i], pa_block_manager::Seq{}).first;
        auto& s = it->second;
        const int64_t pos = s.length;
        if (pos % bm->block_size == 0) {
            int32_t blk;
            if (!bm->take(&blk)) return PA_ERR_WORKSPACE;  // out of blocks: tokens before i are appended
            s.table.push_back(blk);
        } else {
            const int32_t last = s.table.back();
            if (bm->refcount[last] > 1) {
                int32_t fresh;
                if (!bm->take(&fresh)) return PA_ERR_WORKSPACE;
                bm->refcount[last] -= 1;
                s.table.back() = fresh;
                if (cow_pairs) {
                    cow_pairs[2 * *num_cow_pairs] = last;
                    cow_pairs[2 * *num_cow_pairs + 1] = fresh;
                }
                ++*num_cow_pairs;
            }
        }
        s.length = pos + 1;
        slots[i] = (int64_t)s.table[pos / bm->block_size] * bm->block_size + pos % bm->block_size;
    }
    return PA_OK;
}

extern "C" int pa_bm_fork(pa_block_manager* bm, int64_t parent, int64_t child) {
    if (!bm) return PA_ERR_INVALID_ARG;
    auto it = bm->seqs.find(parent);
    if (it == bm->seqs.end() || bm->seqs.count(child)) return PA_ERR_INVALID_ARG;
    pa_block_manager::Seq copy = it->second;
    for (int32_t blk : copy.table) bm->refcount[blk] += 1;
    bm->seqs.emplace(child, std::move(copy));
    return PA_OK;
}

extern "C" int pa_bm_free_sequence(pa_block_manager* bm, int64_t seq) {
    if (!bm) return PA_ERR_INVALID_ARG;
    auto it = bm->seqs.find(seq);
    if (it == bm->seqs.end()) return PA_ERR_INVALID_ARG;
    for (int32_t blk : it->second.table) bm->release(blk);
    bm->seqs.erase(it);
    return PA_OK;
}

extern "C" int64_t pa_bm_num_free(const pa_block_manager* bm) { return bm ? bm->count : -1; }

extern "C" int pa_bm_refcount(const pa_block_manager* bm, int64_t block) {
    if (!bm || block < 0 || block >= bm->num_blocks) return -1;
    return bm->refcount[block];
}

extern "C" int64_t pa_bm_length(const pa_block_manager* bm, int64_t seq) {
    if (!bm) return -1;
    auto it = bm->seqs.find(seq);
    return it == bm->seqs.end() ? -1 : it->second.length;
}

extern "C" int pa_bm_block_tables(const pa_block_manager* bm, const int64_t* seq_ids, int64_t n,
                                  int max_blocks_per_seq, int32_t* tables, int32_t* context_lens) {
    if (!bm || n < 0 || max_blocks_per_seq <= 0 || (n > 0 && (!seq_ids || !tables))) return PA_ERR_INVALID_ARG;
    for (int64_t i = 0; i < n; ++i) {
        auto it = bm->seqs.find(seq_ids[i]);
        if (it == bm->seqs.end()) return PA_ERR_INVALID_ARG;
        const auto& t = it->second.table;
        if ((int64_t)t.size() > max_blocks_per_seq) return PA_ERR_UNSUPPORTED;
        int32_t* row = tables + i * max_blocks_per_seq;
        for (int j = 0; j < max_blocks_per_seq; ++j) row[j] = j < (int)t.size() ? t[j] : -1;
        if (context_lens) context_lens[i] = (int32_t)it->second.length;
    }
    return PA_OK;
}

extern "C" int pa_bm_free_list(const pa_block_manager* bm, int64_t* out, int64_t cap, int64_t* n) {
    if (!bm || !n || (cap > 0 && !out)) return PA_ERR_INVALID_ARG;
    *n = bm->count;
    for (int64_t i = 0; i < bm->count && i < cap; ++i) out[i] = bm->ring[(bm->head + i) % bm->num_blocks];
    return PA_OK;
}

// The sharing structure of a batch, in the form the shared-prefix decode takes
// it: consecutive sequences (in the order given) whose tables begin with the
// same physical block form a group; the group's prefix is the run of leading
// table entries equal in every member, cut to the blocks that are full in
// every member (entry i counts only if every member has at least
// (i + 1) * block_size tokens).  A sequence with no block, or one whose first
// block differs from its predecessor's, starts a new group.
extern "C" int pa_bm_shared_prefix_groups(const pa_block_manager* bm, const int64_t* seq_ids, int64_t n,
                                          int32_t* group_starts, int32_t* prefix_lens, int64_t* num_groups,
                                          int32_t* max_group_size, int32_t* max_prefix_len) {
    if (!bm || n < 0 || !num_groups || !max_group_size || !max_prefix_len ||
        (n > 0 && (!seq_ids || !group_starts || !prefix_lens)) || n > INT32_MAX)
        return PA_ERR_INVALID_ARG;
    std::vector<const pa_block_manager::Seq*> seqs((size_t)n);
    for (int64_t i = 0; i < n; ++i) {
        auto it = bm->seqs.find(seq_ids[i]);
        if (it == bm->seqs.end()) return PA_ERR_INVALID_ARG;
        seqs[(size_t)i] = &it->second;
    }
    int64_t g = 0;
    *max_group_size = 0;
    *max_prefix_len = 0;
    for (int64_t a = 0; a < n;) {
        const auto& lead = seqs[(size_t)a]->table;
        int64_t e = a + 1;
        if (!lead.empty())
            while (e < n && !seqs[(size_t)e]->table.empty() && seqs[(size_t)e]->table[0] == lead[0]) ++e;
        // common leading entries, full in every member
        int64_t k = (int64_t)lead.size();
        for (int64_t m = a; m < e; ++m) {
            const auto& t = seqs[(size_t)m]->table;
            int64_t c = 0;
            while (c < k && c < (int64_t)t.size() && t[(size_t)c] == lead[(size_t)c]) ++c;
            k = c;
            const int64_t full = seqs[(size_t)m]->length / bm->block_size;
            if (full < k) k = full;
        }
        group_starts[g] = (int32_t)a;
        prefix_lens[g] = (int32_t)(k * bm->block_size);
        if (e - a > *max_group_size) *max_group_size = (int32_t)(e - a);
        if (prefix_lens[g] > *max_prefix_len) *max_prefix_len = prefix_lens[g];
        ++g;
        a = e;
    }
    if (n > 0) group_starts[g] = (int32_t)n;
    *num_groups = g;
    return PA_OK;
}
