// Host block allocator for the paged KV cache: a first-in-first-out free
// list, per-block reference counts, per-sequence block tables, and
// copy-on-write when a sequence writes into a block it shares.
//
// Follows "Inside vLLM: How PagedAttention Changes Python LLM Inference at
// the Systems Level", sections "PagedAttention: What the OS Figured Out
// Decades Ago" (blocks claimed on demand, released when a sequence ends, a
// block table per sequence) and "Copy-on-Write Makes Beam Search Cheap"
// (shared prefix blocks by refcount; only the written block is copied).
// The interface is documented in include/pa_alloc.h.
#include <cmath>
#include <cstdint>
#include <deque>
#include <new>
#include <unordered_map>
#include <vector>

#include "pa_alloc.h"
#include "pa_api.h"

namespace {

struct Sequence {
    std::vector<int32_t> blocks;  // logical block i -> physical block
    int32_t num_tokens = 0;
};

}  // namespace

struct pa_alloc {
    int32_t num_blocks = 0;
    int32_t block_size = 0;
    std::deque<int32_t> free_list;
    std::vector<int32_t> refcount;
    std::unordered_map<int64_t, Sequence> seqs;
    int64_t cow_copies = 0;

    int32_t claim() {
        int32_t b = free_list.front();
        free_list.pop_front();
        refcount[b] = 1;
        return b;
    }
    void release(int32_t b) {
        if (--refcount[b] == 0) free_list.push_back(b);
    }
    int64_t blocks_for(int64_t tokens) const { return (tokens + block_size - 1) / block_size; }
};

extern "C" {

pa_alloc *pa_alloc_create(int32_t num_blocks, int32_t block_size) {
    if (num_blocks <= 0 || block_size <= 0) return nullptr;
    pa_alloc *a = new (std::nothrow) pa_alloc();
    if (!a) return nullptr;
    a->num_blocks = num_blocks;
    a->block_size = block_size;
    a->refcount.assign(num_blocks, 0);
    for (int32_t b = 0; b < num_blocks; ++b) a->free_list.push_back(b);
    return a;
}

void pa_alloc_destroy(pa_alloc *a) { delete a; }

int pa_alloc_add_seq(pa_alloc *a, int64_t seq_id, int32_t num_tokens) {
    if (!a || num_tokens < 0 || a->seqs.count(seq_id)) return PA_ERR_INVALID_ARG;
    int64_t need = a->blocks_for(num_tokens);
    if (need > (int64_t)a->free_list.size()) return PA_ERR_NO_BLOCKS;
    Sequence s;
    s.num_tokens = num_tokens;
    s.blocks.reserve(need);
    for (int64_t i = 0; i < need; ++i) s.blocks.push_back(a->claim());
    a->seqs.emplace(seq_id, std::move(s));
    return PA_OK;
}

int pa_alloc_fork(pa_alloc *a, int64_t parent_id, int64_t child_id) {
    if (!a || parent_id == child_id || a->seqs.count(child_id)) return PA_ERR_INVALID_ARG;
    auto it = a->seqs.find(parent_id);
    if (it == a->seqs.end()) return PA_ERR_INVALID_ARG;
    Sequence child = it->second;
    for (int32_t b : child.blocks) ++a->refcount[b];
    a->seqs.emplace(child_id, std::move(child));
    return PA_OK;
}

int pa_alloc_append_slot(pa_alloc *a, int64_t seq_id, int64_t *slot, int32_t *cow_src,
                         int32_t *cow_dst) {
    if (!a || !slot || !cow_src || !cow_dst) return PA_ERR_INVALID_ARG;
    auto it = a->seqs.find(seq_id);
    if (it == a->seqs.end()) return PA_ERR_INVALID_ARG;
    Sequence &s = it->second;
    const int32_t p = s.num_tokens;
    const int32_t logical = p / a->block_size;
    *cow_src = -1;
    *cow_dst = -1;
    if (logical == (int32_t)s.blocks.size()) {
        // position p opens a new block
        if (a->free_list.empty()) return PA_ERR_NO_BLOCKS;
        s.blocks.push_back(a->claim());
    } else {
        int32_t last = s.blocks[logical];
        if (a->refcount[last] > 1) {
            // writing into a block others still read: copy it first
            if (a->free_list.empty()) return PA_ERR_NO_BLOCKS;
            int32_t fresh = a->claim();
            a->release(last);
            s.blocks[logical] = fresh;
            *cow_src = last;
            *cow_dst = fresh;
            ++a->cow_copies;
        }
    }
    *slot = (int64_t)s.blocks[logical] * a->block_size + p % a->block_size;
    s.num_tokens = p + 1;
    return PA_OK;
}

int pa_alloc_append_slots(pa_alloc *a, const int64_t *seq_ids, int32_t n, int64_t *slots,
                          int32_t *pairs, int32_t *num_pairs) {
    if (!a || n < 0 || (n > 0 && (!seq_ids || !slots || !pairs)) || !num_pairs)
        return PA_ERR_INVALID_ARG;
    *num_pairs = 0;
    for (int32_t i = 0; i < n; ++i) {
        int32_t src, dst;
        int rc = pa_alloc_append_slot(a, seq_ids[i], &slots[i], &src, &dst);
        if (rc != PA_OK) return rc;
        if (src >= 0) {
            pairs[2 * *num_pairs] = src;
            pairs[2 * *num_pairs + 1] = dst;
            ++*num_pairs;
        }
    }
    return PA_OK;
}

int pa_alloc_free_seq(pa_alloc *a, int64_t seq_id) {
    if (!a) return PA_ERR_INVALID_ARG;
    auto it = a->seqs.find(seq_id);
    if (it == a->seqs.end()) return PA_ERR_INVALID_ARG;
    for (int32_t b : it->second.blocks) a->release(b);
    a->seqs.erase(it);
    return PA_OK;
}

int32_t pa_alloc_num_tokens(const pa_alloc *a, int64_t seq_id) {
    if (!a) return PA_ERR_INVALID_ARG;
    auto it = a->seqs.find(seq_id);
    return it == a->seqs.end() ? PA_ERR_INVALID_ARG : it->second.num_tokens;
}

int32_t pa_alloc_block_table(const pa_alloc *a, int64_t seq_id, int32_t *out, int32_t cap) {
    if (!a || cap < 0 || (cap > 0 && !out)) return PA_ERR_INVALID_ARG;
    auto it = a->seqs.find(seq_id);
    if (it == a->seqs.end()) return PA_ERR_INVALID_ARG;
    const auto &b = it->second.blocks;
    for (int32_t i = 0; i < (int32_t)b.size() && i < cap; ++i) out[i] = b[i];
    return (int32_t)b.size();
}

int pa_alloc_build_tables(const pa_alloc *a, const int64_t *seq_ids, int32_t n, int32_t *tables,
                          int32_t max_blocks, int32_t *context_lens) {
    if (!a || n < 0 || max_blocks <= 0 || (n > 0 && (!seq_ids || !tables || !context_lens)))
        return PA_ERR_INVALID_ARG;
    for (int32_t i = 0; i < n; ++i) {
        auto it = a->seqs.find(seq_ids[i]);
        if (it == a->seqs.end() || (int32_t)it->second.blocks.size() > max_blocks)
            return PA_ERR_INVALID_ARG;
    }
    for (int32_t i = 0; i < n; ++i) {
        const Sequence &s = a->seqs.find(seq_ids[i])->second;
        int32_t *row = tables + (int64_t)i * max_blocks;
        int32_t j = 0;
        for (; j < (int32_t)s.blocks.size(); ++j) row[j] = s.blocks[j];
        for (; j < max_blocks; ++j) row[j] = -1;
        context_lens[i] = s.num_tokens;
    }
    return PA_OK;
}

int32_t pa_alloc_refcount(const pa_alloc *a, int32_t block) {
    if (!a || block < 0 || block >= a->num_blocks) return -1;
    return a->refcount[block];
}

int pa_alloc_get_stats(const pa_alloc *a, pa_alloc_stats *out) {
    if (!a || !out) return PA_ERR_INVALID_ARG;
    pa_alloc_stats st = {};
    st.num_blocks = a->num_blocks;
    st.free_blocks = (int64_t)a->free_list.size();
    std::vector<int32_t> filled(a->num_blocks, 0);
    for (const auto &kv : a->seqs) {
        const Sequence &s = kv.second;
        st.logical_tokens += s.num_tokens;
        st.logical_blocks += (int64_t)s.blocks.size();
        for (size_t i = 0; i < s.blocks.size(); ++i) {
            int64_t in_block = (int64_t)s.num_tokens - (int64_t)i * a->block_size;
            int32_t n = (int32_t)(in_block > a->block_size ? a->block_size : in_block);
            if (n > filled[s.blocks[i]]) filled[s.blocks[i]] = n;
        }
    }
    st.num_seqs = (int64_t)a->seqs.size();
    for (int32_t b = 0; b < a->num_blocks; ++b) {
        if (a->refcount[b] > 0) ++st.used_blocks;
        if (a->refcount[b] > 1) ++st.shared_blocks;
        st.filled_slots += filled[b];
    }
    st.cow_copies = a->cow_copies;
    st.usage = (double)st.used_blocks / (double)st.num_blocks;
    st.waste = st.used_blocks
                   ? 1.0 - (double)st.filled_slots / ((double)st.used_blocks * a->block_size)
                   : 0.0;
    st.sharing_saving =
        st.logical_blocks ? 1.0 - (double)st.used_blocks / (double)st.logical_blocks : 0.0;
    *out = st;
    return PA_OK;
}

int64_t pa_kv_bytes_per_token(int32_t layers, int32_t kv_heads, int32_t head_dim,
                              int32_t dtype_bytes) {
    return 2LL * layers * kv_heads * head_dim * dtype_bytes;
}

double pa_pool_bytes(double gpu_bytes, double weight_bytes, double utilization) {
    double left = gpu_bytes - weight_bytes;
    return left > 0 ? utilization * left : 0.0;
}

int64_t pa_pool_num_blocks(double pool_bytes, int32_t layers, int32_t kv_heads, int32_t head_dim,
                           int32_t block_size, int32_t dtype_bytes) {
    double per_block =
        (double)block_size * (double)pa_kv_bytes_per_token(layers, kv_heads, head_dim, dtype_bytes);
    if (per_block <= 0 || pool_bytes <= 0) return 0;
    return (int64_t)std::floor(pool_bytes / per_block);
}

}  // extern "C"
