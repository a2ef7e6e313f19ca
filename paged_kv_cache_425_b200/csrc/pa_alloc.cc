// Host block allocator for the paged KV cache: a first-in-first-out free
// list, per-block reference counts, per-sequence block tables,
// copy-on-write when a sequence writes into a block it shares, and
// automatic prefix caching of full prompt blocks.
//
// Follows "Inside vLLM: How PagedAttention Changes Python LLM Inference at
// the Systems Level", sections "PagedAttention: What the OS Figured Out
// Decades Ago" (blocks claimed on demand, released when a sequence ends, a
// block table per sequence), "Copy-on-Write Makes Beam Search Cheap" (shared
// prefix blocks by refcount; only the written block is copied) and
// "PagedAttention in a Python RAG Application" (the content of each block is
// hashed; a request whose prefix matches reuses the cached physical blocks).
// The interface is documented in include/pa_alloc.h.
#include <cmath>
#include <cstdint>
#include <cstring>
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

// 64-bit FNV-1a over a byte string, continued from `h`.
uint64_t fnv1a(uint64_t h, const void *data, size_t n) {
    const unsigned char *p = static_cast<const unsigned char *>(data);
    for (size_t i = 0; i < n; ++i) {
        h ^= p[i];
        h *= 1099511628211ull;
    }
    return h;
}
constexpr uint64_t kFnvOffset = 1469598103934665603ull;

}  // namespace

struct pa_alloc {
    int32_t num_blocks = 0;
    int32_t block_size = 0;
    // free list: intrusive doubly linked list in block order of release, so a
    // cached block can leave it from the middle in O(1)
    std::vector<int32_t> next, prev;
    std::vector<char> in_free;
    int32_t head = -1, tail = -1;
    int64_t free_count = 0;
    std::vector<int32_t> refcount;
    std::unordered_map<int64_t, Sequence> seqs;
    int64_t cow_copies = 0;
    // prefix cache: chain hash of a full block -> block; per block its hash
    // and token ids (compared on every hit, so a hash collision cannot alias)
    bool prefix_caching = false;
    std::unordered_map<uint64_t, int32_t> cached;
    std::vector<uint64_t> block_hash;
    std::vector<char> registered;
    std::vector<int32_t> block_tokens;  // [num_blocks][block_size]
    int64_t prefix_query_blocks = 0, prefix_hit_blocks = 0;

    void push_back_free(int32_t b) {
        next[b] = -1;
        prev[b] = tail;
        if (tail >= 0) next[tail] = b; else head = b;
        tail = b;
        in_free[b] = 1;
        ++free_count;
    }
    void unlink_free(int32_t b) {
        if (prev[b] >= 0) next[prev[b]] = next[b]; else head = next[b];
        if (next[b] >= 0) prev[next[b]] = prev[b]; else tail = prev[b];
        next[b] = prev[b] = -1;
        in_free[b] = 0;
        --free_count;
    }
    void unregister(int32_t b) {
        if (!registered[b]) return;
        auto it = cached.find(block_hash[b]);
        if (it != cached.end() && it->second == b) cached.erase(it);
        registered[b] = 0;
    }
    // Hand out the block at the front of the free list; a cached block that
    // comes up is evicted (its contents will be overwritten).
    int32_t claim() {
        const int32_t b = head;
        unlink_free(b);
        unregister(b);
        refcount[b] = 1;
        return b;
    }
    void release(int32_t b) {
        if (--refcount[b] == 0) push_back_free(b);
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
    a->next.assign(num_blocks, -1);
    a->prev.assign(num_blocks, -1);
    a->in_free.assign(num_blocks, 0);
    a->block_hash.assign(num_blocks, 0);
    a->registered.assign(num_blocks, 0);
    for (int32_t b = 0; b < num_blocks; ++b) a->push_back_free(b);
    return a;
}

void pa_alloc_destroy(pa_alloc *a) { delete a; }

int pa_alloc_add_seq(pa_alloc *a, int64_t seq_id, int32_t num_tokens) {
    if (!a || num_tokens < 0 || a->seqs.count(seq_id)) return PA_ERR_INVALID_ARG;
    int64_t need = a->blocks_for(num_tokens);
    if (need > a->free_count) return PA_ERR_NO_BLOCKS;
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
        if (a->free_count == 0) return PA_ERR_NO_BLOCKS;
        s.blocks.push_back(a->claim());
    } else {
        int32_t last = s.blocks[logical];
        if (a->refcount[last] > 1) {
            // writing into a block others still read: copy it first
            if (a->free_count == 0) return PA_ERR_NO_BLOCKS;
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
    st.free_blocks = a->free_count;
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
    st.cached_blocks = (int64_t)a->cached.size();
    st.prefix_query_blocks = a->prefix_query_blocks;
    st.prefix_hit_blocks = a->prefix_hit_blocks;
    st.usage = (double)st.used_blocks / (double)st.num_blocks;
    st.waste = st.used_blocks
                   ? 1.0 - (double)st.filled_slots / ((double)st.used_blocks * a->block_size)
                   : 0.0;
    st.sharing_saving =
        st.logical_blocks ? 1.0 - (double)st.used_blocks / (double)st.logical_blocks : 0.0;
    *out = st;
    return PA_OK;
}

int pa_alloc_enable_prefix_caching(pa_alloc *a, int32_t enable) {
    if (!a) return PA_ERR_INVALID_ARG;
    if (enable && a->block_tokens.empty())
        a->block_tokens.assign((size_t)a->num_blocks * a->block_size, 0);
    if (!enable) {
        for (int32_t b = 0; b < a->num_blocks; ++b) a->unregister(b);
    }
    a->prefix_caching = enable != 0;
    return PA_OK;
}

int pa_alloc_add_seq_tokens(pa_alloc *a, int64_t seq_id, const int32_t *tokens,
                            int32_t num_tokens, int32_t *num_cached_tokens) {
    if (!a || num_tokens < 0 || (num_tokens > 0 && !tokens) || !num_cached_tokens ||
        a->seqs.count(seq_id))
        return PA_ERR_INVALID_ARG;
    const int32_t bs = a->block_size;
    const int64_t need = a->blocks_for(num_tokens);
    const int32_t full = num_tokens / bs;
    // 1. leading full blocks already in the cache (chain hash + exact tokens)
    std::vector<uint64_t> hashes(full);
    std::vector<int32_t> hits;
    uint64_t h = kFnvOffset;
    for (int32_t i = 0; i < full; ++i) {
        h = fnv1a(h, tokens + (size_t)i * bs, sizeof(int32_t) * bs);
        hashes[i] = h;
    }
    if (a->prefix_caching) {
        for (int32_t i = 0; i < full; ++i) {
            auto it = a->cached.find(hashes[i]);
            if (it == a->cached.end()) break;
            const int32_t b = it->second;
            if (std::memcmp(&a->block_tokens[(size_t)b * bs], tokens + (size_t)i * bs,
                            sizeof(int32_t) * bs) != 0)
                break;
            hits.push_back(b);
        }
    }
    // 2. enough free blocks for the rest?  (a hit that sits on the free list
    // leaves it, so it cannot also be claimed)
    int64_t hits_on_free = 0;
    for (int32_t b : hits) hits_on_free += a->in_free[b];
    if (need - (int64_t)hits.size() > a->free_count - hits_on_free) return PA_ERR_NO_BLOCKS;
    // 3. commit
    Sequence s;
    s.num_tokens = num_tokens;
    s.blocks.reserve(need);
    for (int32_t b : hits) {
        if (a->in_free[b]) {
            a->unlink_free(b);
            a->refcount[b] = 1;
        } else {
            ++a->refcount[b];
        }
        s.blocks.push_back(b);
    }
    for (int64_t i = (int64_t)hits.size(); i < need; ++i) {
        const int32_t b = a->claim();
        s.blocks.push_back(b);
        if (a->prefix_caching && i < full && !a->cached.count(hashes[i])) {
            a->cached.emplace(hashes[i], b);
            a->block_hash[b] = hashes[i];
            a->registered[b] = 1;
            std::memcpy(&a->block_tokens[(size_t)b * bs], tokens + (size_t)i * bs,
                        sizeof(int32_t) * bs);
        }
    }
    if (a->prefix_caching) {
        a->prefix_query_blocks += full;
        a->prefix_hit_blocks += (int64_t)hits.size();
    }
    *num_cached_tokens = (int32_t)hits.size() * bs;
    a->seqs.emplace(seq_id, std::move(s));
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
