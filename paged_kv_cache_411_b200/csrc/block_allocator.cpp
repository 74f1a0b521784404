// Host block allocator of libpagedkv.
//
// The pool, free list and per-request block tables of the block manager on
// the page "LLM 推理引擎 Continuous Batching 与 PagedAttention" (§3.2 核心数据
// 结构), with the refcounted shared-prefix blocks of §4.1.  Semantics:
//   * the free list is a stack: every take pops its end; blocks whose refcount
//     reaches zero are pushed on the end in block-table order;
//   * allocate / append_tokens are all-or-nothing; OOM leaves every field as
//     it was and bumps oom_count;
//   * append_token takes a block iff the request's current length is a
//     multiple of block_size (current length = tokens stored before the call);
//   * fork shares whole blocks only (floor(prefix / block_size));
//   * a token's slot is table[pos / block_size] * block_size + pos % block_size
//     (the address form of the page's §3.3 kernel).
// Everything is O(1) per token except free, which is O(table length).
//
// Automatic prefix caching (§4.1 hashes the token content of blocks and keeps
// identical blocks once; §4.2 keeps recently used blocks in an LRU):
//   * a full block's content is identified exactly by a node of a prefix trie,
//     node = intern(parent node, the block's block_size token ids), so two
//     blocks match only when the whole token prefix up to their end matches;
//   * allocate_cached reuses the cached blocks of the longest cached prefix
//     (walking from the first block, stopping at the first miss), takes new
//     blocks for the rest and registers the new full blocks; the partial last
//     block stays private;
//   * a registered block whose refcount drops to zero is not freed but parked
//     in an LRU of evictable blocks (a request's blocks are parked last block
//     first, so a prefix is always at least as recent as its extensions);
//   * a take pops the free list, or, when it is empty, evicts the least
//     recently used parked block (its cache entry is dropped);
//   * a cache entry lives as long as its block: when an evicted block's node
//     has no children it is dropped, and so, walking up, is every ancestor
//     left without a block and without children (node ids are never reused),
//     so the trie stays bounded by the blocks it describes;
//   * begin_cached starts a request with only the cached blocks of the
//     longest cached prefix that leaves at least one token to compute, and a
//     request started by begin_cached or allocate_cached is tracked: its known
//     token ids (extend_tokens adds generated ones) register every block its
//     appends fill, under the node of the block before it, until a filled
//     block's ids are unknown or its content is already cached elsewhere.
#include <algorithm>
#include <cstdint>
#include <cstring>
#include <list>
#include <new>
#include <unordered_map>
#include <vector>

#include "common.h"

namespace pagedkv {

static thread_local std::string g_last_error;

pa_status fail(pa_status s, const char* fmt, ...) {
    char buf[512];
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(buf, sizeof(buf), fmt, ap);
    va_end(ap);
    g_last_error = buf;
    return s;
}

void clear_error() { g_last_error.clear(); }

const char* last_error() { return g_last_error.c_str(); }

}  // namespace pagedkv

using pagedkv::fail;

namespace {

struct PrefixKey {
    int64_t parent;
    std::vector<int32_t> tokens;
    bool operator==(const PrefixKey& o) const { return parent == o.parent && tokens == o.tokens; }
};

struct PrefixKeyHash {
    size_t operator()(const PrefixKey& k) const {
        uint64_t h = 1469598103934665603ull ^ static_cast<uint64_t>(k.parent);
        for (int32_t t : k.tokens) {
            h ^= static_cast<uint32_t>(t);
            h *= 1099511628211ull;
        }
        return static_cast<size_t>(h ^ (h >> 29));
    }
};

}  // namespace

struct pa_alloc {
    struct Request {
        std::vector<int32_t> table;
        int32_t len = 0;
        bool tracked = false;               // its filled blocks get registered
        std::vector<int32_t> tokens;        // known token ids (tracked requests)
        int64_t last_node = -1;             // node of its last registered block (-1: the root)
    };
    int32_t num_blocks = 0;
    int32_t block_size = 0;
    std::vector<int32_t> free_list;      // stack; back() is the next pop
    std::vector<int32_t> refcount;
    std::unordered_map<int64_t, Request> reqs;
    int64_t oom_count = 0;
    // prefix cache
    std::unordered_map<PrefixKey, int64_t, PrefixKeyHash> trie;   // (parent node, tokens) -> node
    std::unordered_map<int64_t, PrefixKey> node_key;               // node -> its key
    std::unordered_map<int64_t, int32_t> children;                 // node -> child nodes
    int64_t next_node = 0;
    std::unordered_map<int64_t, int32_t> cache;                    // node -> block
    std::vector<int64_t> block_node;                               // block -> node, -1 if not registered
    std::list<int32_t> lru;                                        // parked blocks, least recent first
    std::vector<std::list<int32_t>::iterator> lru_pos;
    std::vector<char> in_lru;
    int64_t hit_blocks = 0, evictions = 0;

    int64_t blocks_for(int64_t tokens) const { return (tokens + block_size - 1) / block_size; }
    int64_t available() const { return static_cast<int64_t>(free_list.size() + lru.size()); }
    void unpark(int32_t b) {
        lru.erase(lru_pos[b]);
        in_lru[b] = 0;
    }
    int32_t take() {
        int32_t b;
        if (!free_list.empty()) {
            b = free_list.back();
            free_list.pop_back();
        } else {
            b = lru.front();
            unpark(b);
            const int64_t node = block_node[b];
            cache.erase(node);
            block_node[b] = -1;
            evictions += 1;
            prune(node);
        }
        refcount[b] += 1;
        return b;
    }
    // Drops `node`, then its ancestors, while they hold no block and have no children.
    void prune(int64_t node) {
        while (node >= 0 && !cache.count(node) && children[node] == 0) {
            auto k = node_key.find(node);
            const int64_t parent = k->second.parent;
            trie.erase(k->second);
            node_key.erase(k);
            children.erase(node);
            node = parent;
            if (node >= 0) children[node] -= 1;
        }
    }
    // Drop one reference to every block of `table`; blocks reaching zero go to the free list
    // (unregistered, table order) or are parked in the LRU (registered, last block first).
    void release(const std::vector<int32_t>& table) {
        std::vector<int32_t> zero;
        for (int32_t b : table)
            if (--refcount[b] == 0) zero.push_back(b);
        for (int32_t b : zero)
            if (block_node[b] < 0) free_list.push_back(b);
        for (auto it = zero.rbegin(); it != zero.rend(); ++it) {
            const int32_t b = *it;
            if (block_node[b] >= 0) {
                lru.push_back(b);
                lru_pos[b] = std::prev(lru.end());
                in_lru[b] = 1;
            }
        }
    }
    int64_t intern(int64_t parent, const int32_t* tokens) {
        PrefixKey k{parent, std::vector<int32_t>(tokens, tokens + block_size)};
        auto it = trie.find(k);
        if (it != trie.end()) return it->second;
        const int64_t node = next_node++;
        node_key.emplace(node, k);
        trie.emplace(std::move(k), node);
        children[node] = 0;
        if (parent >= 0) children[parent] += 1;
        return node;
    }
    // Cached blocks (and their nodes) of the longest cached prefix of whole blocks, at most max_blocks.
    void lookup_prefix(const int32_t* tokens, int64_t max_blocks, std::vector<int32_t>* hits,
                       std::vector<int64_t>* nodes) const {
        int64_t parent = -1;
        for (int64_t i = 0; i < max_blocks; ++i) {
            const int64_t node = lookup(parent, tokens + i * block_size);
            if (node < 0) break;
            auto c = cache.find(node);
            if (c == cache.end()) break;
            hits->push_back(c->second);
            if (nodes) nodes->push_back(node);
            parent = node;
        }
    }
    // A tracked request just stored position len - 1: register its block if that filled it.
    void on_append(Request& r) {
        if (!r.tracked || r.len % block_size != 0) return;
        if (static_cast<int64_t>(r.tokens.size()) < r.len) {
            r.tracked = false;                       // ids unknown: the chain ends
            return;
        }
        const int64_t node = intern(r.last_node, r.tokens.data() + (r.len - block_size));
        if (cache.count(node)) {
            r.tracked = false;                       // content cached in another block: the chain ends
            return;
        }
        cache.emplace(node, r.table.back());
        block_node[r.table.back()] = node;
        r.last_node = node;
    }
    int64_t lookup(int64_t parent, const int32_t* tokens) const {
        PrefixKey k{parent, std::vector<int32_t>(tokens, tokens + block_size)};
        auto it = trie.find(k);
        return it == trie.end() ? -1 : it->second;
    }
    int64_t slot(const Request& r, int64_t pos) const {
        return static_cast<int64_t>(r.table[pos / block_size]) * block_size + pos % block_size;
    }
};

extern "C" {

pa_status pa_alloc_create(int32_t num_blocks, int32_t block_size, const int32_t* init_free_order,
                          pa_alloc** out) {
    if (!out) return fail(PA_ERR_INVALID_ARG, "pa_alloc_create: out is NULL");
    *out = nullptr;
    if (num_blocks < 0 || block_size <= 0)
        return fail(PA_ERR_INVALID_ARG, "pa_alloc_create: num_blocks=%d block_size=%d", num_blocks, block_size);
    pa_alloc* a = new (std::nothrow) pa_alloc();
    if (!a) return fail(PA_ERR_OOM, "pa_alloc_create: host allocation failed");
    a->num_blocks = num_blocks;
    a->block_size = block_size;
    a->refcount.assign(num_blocks, 0);
    a->block_node.assign(num_blocks, -1);
    a->lru_pos.resize(num_blocks);
    a->in_lru.assign(num_blocks, 0);
    a->free_list.resize(num_blocks);
    if (init_free_order) {
        std::vector<char> seen(num_blocks, 0);
        for (int32_t i = 0; i < num_blocks; ++i) {
            int32_t b = init_free_order[i];
            if (b < 0 || b >= num_blocks || seen[b]) {
                delete a;
                return fail(PA_ERR_INVALID_ARG, "pa_alloc_create: init_free_order is not a permutation (entry %d = %d)", i, b);
            }
            seen[b] = 1;
            a->free_list[i] = b;
        }
    } else {
        for (int32_t i = 0; i < num_blocks; ++i) a->free_list[i] = i;
    }
    *out = a;
    return PA_OK;
}

void pa_alloc_destroy(pa_alloc* a) { delete a; }

pa_status pa_alloc_allocate(pa_alloc* a, int64_t req, int32_t num_tokens) {
    if (!a) return fail(PA_ERR_INVALID_ARG, "pa_alloc_allocate: NULL allocator");
    if (num_tokens < 0) return fail(PA_ERR_INVALID_ARG, "pa_alloc_allocate: num_tokens=%d", num_tokens);
    if (a->reqs.count(req)) return fail(PA_ERR_EXISTS, "pa_alloc_allocate: request %lld exists", (long long)req);
    int64_t n = a->blocks_for(num_tokens);
    if (n > a->available()) {
        a->oom_count += 1;
        return fail(PA_ERR_OOM, "pa_alloc_allocate: need %lld blocks, %lld available", (long long)n,
                    (long long)a->available());
    }
    pa_alloc::Request r;
    r.table.reserve(n);
    for (int64_t i = 0; i < n; ++i) r.table.push_back(a->take());
    r.len = num_tokens;
    a->reqs.emplace(req, std::move(r));
    return PA_OK;
}

pa_status pa_alloc_append_token(pa_alloc* a, int64_t req, int64_t* slot_out) {
    if (!a) return fail(PA_ERR_INVALID_ARG, "pa_alloc_append_token: NULL allocator");
    auto it = a->reqs.find(req);
    if (it == a->reqs.end()) return fail(PA_ERR_NOT_FOUND, "pa_alloc_append_token: request %lld not found", (long long)req);
    pa_alloc::Request& r = it->second;
    if (r.len % a->block_size == 0) {
        if (a->available() == 0) {
            a->oom_count += 1;
            return fail(PA_ERR_OOM, "pa_alloc_append_token: no free block");
        }
        r.table.push_back(a->take());
    }
    if (slot_out) *slot_out = a->slot(r, r.len);
    r.len += 1;
    a->on_append(r);
    return PA_OK;
}

pa_status pa_alloc_append_tokens(pa_alloc* a, int64_t req, int32_t n, int64_t* slots_out) {
    if (!a) return fail(PA_ERR_INVALID_ARG, "pa_alloc_append_tokens: NULL allocator");
    if (n < 0) return fail(PA_ERR_INVALID_ARG, "pa_alloc_append_tokens: n=%d", n);
    auto it = a->reqs.find(req);
    if (it == a->reqs.end()) return fail(PA_ERR_NOT_FOUND, "pa_alloc_append_tokens: request %lld not found", (long long)req);
    pa_alloc::Request& r = it->second;
    int64_t extra = a->blocks_for(static_cast<int64_t>(r.len) + n) - static_cast<int64_t>(r.table.size());
    if (extra > a->available()) {
        a->oom_count += 1;
        return fail(PA_ERR_OOM, "pa_alloc_append_tokens: need %lld blocks, %lld available", (long long)extra,
                    (long long)a->available());
    }
    for (int32_t i = 0; i < n; ++i) {
        if (r.len % a->block_size == 0) r.table.push_back(a->take());
        if (slots_out) slots_out[i] = a->slot(r, r.len);
        r.len += 1;
        a->on_append(r);
    }
    return PA_OK;
}

pa_status pa_alloc_fork(pa_alloc* a, int64_t src, int64_t dst, int32_t prefix_tokens) {
    if (!a) return fail(PA_ERR_INVALID_ARG, "pa_alloc_fork: NULL allocator");
    auto it = a->reqs.find(src);
    if (it == a->reqs.end()) return fail(PA_ERR_NOT_FOUND, "pa_alloc_fork: source %lld not found", (long long)src);
    if (a->reqs.count(dst)) return fail(PA_ERR_EXISTS, "pa_alloc_fork: destination %lld exists", (long long)dst);
    if (prefix_tokens < 0 || prefix_tokens > it->second.len)
        return fail(PA_ERR_INVALID_ARG, "pa_alloc_fork: prefix_tokens=%d, source holds %d", prefix_tokens, it->second.len);
    int32_t shared = prefix_tokens / a->block_size;
    pa_alloc::Request r;
    r.table.assign(it->second.table.begin(), it->second.table.begin() + shared);
    for (int32_t b : r.table) a->refcount[b] += 1;
    r.len = shared * a->block_size;
    a->reqs.emplace(dst, std::move(r));
    return PA_OK;
}

pa_status pa_alloc_free(pa_alloc* a, int64_t req) {
    if (!a) return fail(PA_ERR_INVALID_ARG, "pa_alloc_free: NULL allocator");
    auto it = a->reqs.find(req);
    if (it == a->reqs.end()) return PA_OK;
    a->release(it->second.table);
    a->reqs.erase(it);
    return PA_OK;
}

pa_status pa_alloc_get_block_table(const pa_alloc* a, int64_t req, int32_t* out, int32_t cap, int32_t* len_out) {
    if (!a) return fail(PA_ERR_INVALID_ARG, "pa_alloc_get_block_table: NULL allocator");
    auto it = a->reqs.find(req);
    if (it == a->reqs.end()) return fail(PA_ERR_NOT_FOUND, "pa_alloc_get_block_table: request %lld not found", (long long)req);
    int32_t n = static_cast<int32_t>(it->second.table.size());
    if (len_out) *len_out = n;
    if (cap < n || (n > 0 && !out))
        return fail(PA_ERR_INVALID_ARG, "pa_alloc_get_block_table: capacity %d < table length %d", cap, n);
    if (n) std::memcpy(out, it->second.table.data(), sizeof(int32_t) * n);
    return PA_OK;
}

pa_status pa_alloc_seq_len(const pa_alloc* a, int64_t req, int32_t* out) {
    if (!a || !out) return fail(PA_ERR_INVALID_ARG, "pa_alloc_seq_len: NULL argument");
    auto it = a->reqs.find(req);
    if (it == a->reqs.end()) return fail(PA_ERR_NOT_FOUND, "pa_alloc_seq_len: request %lld not found", (long long)req);
    *out = it->second.len;
    return PA_OK;
}

pa_status pa_alloc_slots(const pa_alloc* a, int64_t req, int32_t pos_begin, int32_t n, int64_t* slots_out) {
    if (!a) return fail(PA_ERR_INVALID_ARG, "pa_alloc_slots: NULL allocator");
    auto it = a->reqs.find(req);
    if (it == a->reqs.end()) return fail(PA_ERR_NOT_FOUND, "pa_alloc_slots: request %lld not found", (long long)req);
    const pa_alloc::Request& r = it->second;
    if (pos_begin < 0 || n < 0 || static_cast<int64_t>(pos_begin) + n > r.len || (n > 0 && !slots_out))
        return fail(PA_ERR_INVALID_ARG, "pa_alloc_slots: positions [%d, %d) outside [0, %d)", pos_begin, pos_begin + n, r.len);
    for (int32_t i = 0; i < n; ++i) slots_out[i] = a->slot(r, static_cast<int64_t>(pos_begin) + i);
    return PA_OK;
}

pa_status pa_alloc_pack(const pa_alloc* a, const int64_t* reqs, int32_t n, int32_t max_blocks,
                        int32_t* tables, int32_t* seq_lens) {
    if (!a || n < 0 || max_blocks < 0 || (n > 0 && (!reqs || !tables || !seq_lens)))
        return fail(PA_ERR_INVALID_ARG, "pa_alloc_pack: bad arguments");
    std::vector<const pa_alloc::Request*> rs(n);
    for (int32_t i = 0; i < n; ++i) {
        auto it = a->reqs.find(reqs[i]);
        if (it == a->reqs.end()) return fail(PA_ERR_NOT_FOUND, "pa_alloc_pack: request %lld not found", (long long)reqs[i]);
        if (static_cast<int64_t>(it->second.table.size()) > max_blocks)
            return fail(PA_ERR_INVALID_ARG, "pa_alloc_pack: request %lld holds %zu blocks > max_blocks %d",
                        (long long)reqs[i], it->second.table.size(), max_blocks);
        rs[i] = &it->second;
    }
    for (int32_t i = 0; i < n; ++i) {
        int32_t* row = tables + static_cast<int64_t>(i) * max_blocks;
        size_t k = rs[i]->table.size();
        if (k) std::memcpy(row, rs[i]->table.data(), sizeof(int32_t) * k);
        for (int32_t j = static_cast<int32_t>(k); j < max_blocks; ++j) row[j] = -1;
        seq_lens[i] = rs[i]->len;
    }
    return PA_OK;
}

pa_status pa_alloc_stats(const pa_alloc* a, pa_alloc_stats_t* out) {
    if (!a || !out) return fail(PA_ERR_INVALID_ARG, "pa_alloc_stats: NULL argument");
    pa_alloc_stats_t s{};
    s.num_blocks = a->num_blocks;
    s.block_size = a->block_size;
    s.num_free = static_cast<int32_t>(a->free_list.size());
    for (int32_t c : a->refcount) {
        if (c > 0) s.num_used += 1;
        s.total_refs += c;
    }
    s.num_requests = static_cast<int64_t>(a->reqs.size());
    s.oom_count = a->oom_count;
    for (const auto& kv : a->reqs)
        s.waste_tokens += static_cast<int64_t>(kv.second.table.size()) * a->block_size - kv.second.len;
    *out = s;
    return PA_OK;
}

pa_status pa_alloc_available(const pa_alloc* a, int64_t* out) {
    if (!a || !out) return fail(PA_ERR_INVALID_ARG, "pa_alloc_available: NULL argument");
    *out = a->available();
    return PA_OK;
}

pa_status pa_alloc_refcount(const pa_alloc* a, int32_t block, int32_t* out) {
    if (!a || !out || block < 0 || block >= a->num_blocks)
        return fail(PA_ERR_INVALID_ARG, "pa_alloc_refcount: bad block %d", block);
    *out = a->refcount[block];
    return PA_OK;
}

pa_status pa_alloc_free_list(const pa_alloc* a, int32_t* out, int32_t cap, int32_t* len_out) {
    if (!a) return fail(PA_ERR_INVALID_ARG, "pa_alloc_free_list: NULL allocator");
    int32_t n = static_cast<int32_t>(a->free_list.size());
    if (len_out) *len_out = n;
    if (cap < n || (n > 0 && !out)) return fail(PA_ERR_INVALID_ARG, "pa_alloc_free_list: capacity %d < %d", cap, n);
    if (n) std::memcpy(out, a->free_list.data(), sizeof(int32_t) * n);
    return PA_OK;
}

pa_status pa_alloc_allocate_cached(pa_alloc* a, int64_t req, const int32_t* tokens, int32_t num_tokens,
                                   int32_t* cached_tokens_out) {
    if (!a) return fail(PA_ERR_INVALID_ARG, "pa_alloc_allocate_cached: NULL allocator");
    if (num_tokens < 0 || (num_tokens > 0 && !tokens))
        return fail(PA_ERR_INVALID_ARG, "pa_alloc_allocate_cached: num_tokens=%d", num_tokens);
    if (a->reqs.count(req)) return fail(PA_ERR_EXISTS, "pa_alloc_allocate_cached: request %lld exists", (long long)req);
    const int32_t bs = a->block_size;
    const int64_t nfull = num_tokens / bs, nblocks = a->blocks_for(num_tokens);
    // longest cached prefix of whole blocks
    std::vector<int32_t> hits;
    a->lookup_prefix(tokens, nfull, &hits, nullptr);
    int64_t parked_hits = 0;
    for (int32_t b : hits) parked_hits += a->in_lru[b] ? 1 : 0;
    const int64_t need = nblocks - static_cast<int64_t>(hits.size());
    if (need > a->available() - parked_hits) {
        a->oom_count += 1;
        return fail(PA_ERR_OOM, "pa_alloc_allocate_cached: need %lld new blocks, %lld available", (long long)need,
                    (long long)(a->available() - parked_hits));
    }
    pa_alloc::Request r;
    r.table.reserve(nblocks);
    for (int32_t b : hits) {
        if (a->in_lru[b]) a->unpark(b);
        a->refcount[b] += 1;
        r.table.push_back(b);
    }
    for (int64_t i = 0; i < need; ++i) r.table.push_back(a->take());
    // register the new full blocks under their prefix nodes
    int64_t parent = -1;
    bool chain = true;
    for (int64_t i = 0; i < nfull; ++i) {
        const int64_t node = a->intern(parent, tokens + i * bs);
        if (i >= static_cast<int64_t>(hits.size()) && !a->cache.count(node)) {
            a->cache.emplace(node, r.table[i]);
            a->block_node[r.table[i]] = node;
        }
        auto c = a->cache.find(node);
        chain = chain && c != a->cache.end() && c->second == r.table[i];
        parent = node;
    }
    if (chain) {            // every full block is its own node's block: later filled blocks register too
        r.tracked = true;
        r.tokens.assign(tokens, tokens + num_tokens);
        r.last_node = parent;
    }
    r.len = num_tokens;
    a->hit_blocks += static_cast<int64_t>(hits.size());
    a->reqs.emplace(req, std::move(r));
    if (cached_tokens_out) *cached_tokens_out = static_cast<int32_t>(hits.size()) * bs;
    return PA_OK;
}

pa_status pa_alloc_cached_prefix(const pa_alloc* a, const int32_t* tokens, int32_t num_tokens, int32_t* hit_blocks,
                                 int32_t* parked_blocks) {
    if (!a || num_tokens < 0 || (num_tokens > 0 && !tokens))
        return fail(PA_ERR_INVALID_ARG, "pa_alloc_cached_prefix: bad arguments");
    std::vector<int32_t> hits;
    a->lookup_prefix(tokens, num_tokens > 0 ? (num_tokens - 1) / a->block_size : 0, &hits, nullptr);
    int32_t parked = 0;
    for (int32_t b : hits) parked += a->in_lru[b] ? 1 : 0;
    if (hit_blocks) *hit_blocks = static_cast<int32_t>(hits.size());
    if (parked_blocks) *parked_blocks = parked;
    return PA_OK;
}

pa_status pa_alloc_begin_cached(pa_alloc* a, int64_t req, const int32_t* tokens, int32_t num_tokens,
                                int32_t* cached_tokens_out) {
    if (!a || num_tokens < 0 || (num_tokens > 0 && !tokens))
        return fail(PA_ERR_INVALID_ARG, "pa_alloc_begin_cached: bad arguments");
    if (a->reqs.count(req)) return fail(PA_ERR_EXISTS, "pa_alloc_begin_cached: request %lld exists", (long long)req);
    std::vector<int32_t> hits;
    std::vector<int64_t> nodes;
    a->lookup_prefix(tokens, num_tokens > 0 ? (num_tokens - 1) / a->block_size : 0, &hits, &nodes);
    pa_alloc::Request r;
    for (int32_t b : hits) {
        if (a->in_lru[b]) a->unpark(b);
        a->refcount[b] += 1;
    }
    r.table = hits;
    r.len = static_cast<int32_t>(hits.size()) * a->block_size;
    r.tracked = true;
    r.tokens.assign(tokens, tokens + num_tokens);
    r.last_node = nodes.empty() ? -1 : nodes.back();
    a->hit_blocks += static_cast<int64_t>(hits.size());
    a->reqs.emplace(req, std::move(r));
    if (cached_tokens_out) *cached_tokens_out = static_cast<int32_t>(hits.size()) * a->block_size;
    return PA_OK;
}

pa_status pa_alloc_extend_tokens(pa_alloc* a, int64_t req, const int32_t* ids, int32_t n) {
    if (!a || n < 0 || (n > 0 && !ids)) return fail(PA_ERR_INVALID_ARG, "pa_alloc_extend_tokens: bad arguments");
    auto it = a->reqs.find(req);
    if (it == a->reqs.end()) return fail(PA_ERR_NOT_FOUND, "pa_alloc_extend_tokens: request %lld not found", (long long)req);
    if (it->second.tracked) it->second.tokens.insert(it->second.tokens.end(), ids, ids + n);
    return PA_OK;
}

pa_status pa_alloc_cache_stats(const pa_alloc* a, pa_cache_stats_t* out) {
    if (!a || !out) return fail(PA_ERR_INVALID_ARG, "pa_alloc_cache_stats: NULL argument");
    pa_cache_stats_t s{};
    s.cached_blocks = static_cast<int64_t>(a->cache.size());
    s.evictable_blocks = static_cast<int64_t>(a->lru.size());
    s.hit_blocks = a->hit_blocks;
    s.evictions = a->evictions;
    s.prefix_nodes = static_cast<int64_t>(a->trie.size());
    *out = s;
    return PA_OK;
}

pa_status pa_alloc_evictable_list(const pa_alloc* a, int32_t* out, int32_t cap, int32_t* len_out) {
    if (!a) return fail(PA_ERR_INVALID_ARG, "pa_alloc_evictable_list: NULL allocator");
    const int32_t n = static_cast<int32_t>(a->lru.size());
    if (len_out) *len_out = n;
    if (cap < n || (n > 0 && !out)) return fail(PA_ERR_INVALID_ARG, "pa_alloc_evictable_list: capacity %d < %d", cap, n);
    int32_t i = 0;
    for (int32_t b : a->lru) out[i++] = b;
    return PA_OK;
}

}  // extern "C"

// ---- checkpoint / resume of the host state ----------------------------------------------------------
// Format (little-endian, version 1): "PKVA", u32 version, i32 num_blocks, i32 block_size, i64 oom_count,
// i64 hit_blocks, i64 evictions, i64 next_node; u64 n, i32 free_list[n] (bottom of the stack first);
// i32 refcount[num_blocks]; u64 n_requests, then per request in increasing id: i64 id, i32 len, u8 tracked,
// i64 last_node, u64 n, i32 table[n], u64 m, i32 tokens[m]; u64 n_nodes, then per trie node in increasing
// id: i64 node, i64 parent, i32 children, i32 cached block (-1: none), i32 tokens[block_size]; u64 n,
// i32 lru[n] (least recently used first).  Maps are written in key order, so equal states give equal bytes.
namespace {

constexpr uint32_t kStateVersion = 1;

struct Writer {
    uint8_t* buf;
    size_t cap, n = 0;
    template <typename T>
    void put(T v) {
        if (buf && n + sizeof(T) <= cap) std::memcpy(buf + n, &v, sizeof(T));
        n += sizeof(T);
    }
    void put_i32s(const int32_t* v, size_t count) {
        put<uint64_t>(count);
        for (size_t i = 0; i < count; ++i) put<int32_t>(v[i]);
    }
};

struct Reader {
    const uint8_t* buf;
    size_t size, n = 0;
    bool ok = true;
    template <typename T>
    T get() {
        T v{};
        if (!ok || n + sizeof(T) > size) {
            ok = false;
            return v;
        }
        std::memcpy(&v, buf + n, sizeof(T));
        n += sizeof(T);
        return v;
    }
    // a count of int32 entries that must still fit in the buffer
    uint64_t count() {
        const uint64_t c = get<uint64_t>();
        if (ok && c > (size - n) / sizeof(int32_t)) ok = false;
        return ok ? c : 0;
    }
};

}  // namespace

extern "C" {

pa_status pa_alloc_serialize(const pa_alloc* a, uint8_t* buf, size_t capacity, size_t* size) {
    if (!a || !size) return fail(PA_ERR_INVALID_ARG, "pa_alloc_serialize: NULL argument");
    auto write = [&](Writer& w) {
        w.put<uint32_t>(0x41564B50u);   // "PKVA"
        w.put<uint32_t>(kStateVersion);
        w.put<int32_t>(a->num_blocks);
        w.put<int32_t>(a->block_size);
        w.put<int64_t>(a->oom_count);
        w.put<int64_t>(a->hit_blocks);
        w.put<int64_t>(a->evictions);
        w.put<int64_t>(a->next_node);
        w.put_i32s(a->free_list.data(), a->free_list.size());
        for (int32_t b = 0; b < a->num_blocks; ++b) w.put<int32_t>(a->refcount[b]);
        std::vector<int64_t> ids;
        for (const auto& kv : a->reqs) ids.push_back(kv.first);
        std::sort(ids.begin(), ids.end());
        w.put<uint64_t>(ids.size());
        for (int64_t id : ids) {
            const auto& r = a->reqs.at(id);
            w.put<int64_t>(id);
            w.put<int32_t>(r.len);
            w.put<uint8_t>(r.tracked ? 1 : 0);
            w.put<int64_t>(r.last_node);
            w.put_i32s(r.table.data(), r.table.size());
            w.put_i32s(r.tokens.data(), r.tokens.size());
        }
        std::vector<int64_t> nodes;
        for (const auto& kv : a->node_key) nodes.push_back(kv.first);
        std::sort(nodes.begin(), nodes.end());
        w.put<uint64_t>(nodes.size());
        for (int64_t node : nodes) {
            const PrefixKey& k = a->node_key.at(node);
            auto ch = a->children.find(node);
            auto c = a->cache.find(node);
            w.put<int64_t>(node);
            w.put<int64_t>(k.parent);
            w.put<int32_t>(ch == a->children.end() ? 0 : ch->second);
            w.put<int32_t>(c == a->cache.end() ? -1 : c->second);
            for (int32_t t : k.tokens) w.put<int32_t>(t);
        }
        w.put<uint64_t>(a->lru.size());
        for (int32_t b : a->lru) w.put<int32_t>(b);
    };
    Writer probe{nullptr, 0};
    write(probe);
    *size = probe.n;
    if (!buf) return PA_OK;                                   // size query
    if (capacity < probe.n)
        return fail(PA_ERR_INVALID_ARG, "pa_alloc_serialize: capacity %zu < %zu bytes", capacity, probe.n);
    Writer w{buf, capacity};
    write(w);
    return PA_OK;
}

pa_status pa_alloc_deserialize(const uint8_t* buf, size_t size, pa_alloc** out) {
    if (!out) return fail(PA_ERR_INVALID_ARG, "pa_alloc_deserialize: out is NULL");
    *out = nullptr;
    if (!buf) return fail(PA_ERR_INVALID_ARG, "pa_alloc_deserialize: NULL buffer");
    Reader r{buf, size};
    if (r.get<uint32_t>() != 0x41564B50u || r.get<uint32_t>() != kStateVersion || !r.ok)
        return fail(PA_ERR_INVALID_ARG, "pa_alloc_deserialize: not an allocator state of version %u", kStateVersion);
    const int32_t nb = r.get<int32_t>(), bs = r.get<int32_t>();
    // every count below must be backed by bytes of the buffer before anything is sized from it
    if (!r.ok || nb < 0 || bs <= 0 || static_cast<uint64_t>(nb) > (size - r.n) / sizeof(int32_t) ||
        static_cast<uint64_t>(bs) > (size - r.n) / sizeof(int32_t))
        return fail(PA_ERR_INVALID_ARG, "pa_alloc_deserialize: bad pool shape");
    pa_alloc* a = nullptr;
    if (pa_alloc_create(nb, bs, nullptr, &a) != PA_OK) return PA_ERR_OOM;
    auto bad = [&](const char* what) {
        delete a;
        return fail(PA_ERR_INVALID_ARG, "pa_alloc_deserialize: %s", what);
    };
    auto block_ok = [&](int64_t b) { return b >= 0 && b < nb; };
    a->oom_count = r.get<int64_t>();
    a->hit_blocks = r.get<int64_t>();
    a->evictions = r.get<int64_t>();
    a->next_node = r.get<int64_t>();
    const uint64_t nf = r.count();
    if (!r.ok || nf > static_cast<uint64_t>(nb)) return bad("free list");
    a->free_list.assign(nf, 0);
    std::vector<char> seen(nb, 0);
    for (uint64_t i = 0; i < nf; ++i) {
        const int32_t b = r.get<int32_t>();
        if (!r.ok || !block_ok(b) || seen[b]) return bad("free list entry");
        seen[b] = 1;
        a->free_list[i] = b;
    }
    for (int32_t b = 0; b < nb; ++b) {
        a->refcount[b] = r.get<int32_t>();
        if (!r.ok || a->refcount[b] < 0) return bad("refcount");
    }
    const uint64_t nr = r.get<uint64_t>();
    for (uint64_t i = 0; r.ok && i < nr; ++i) {
        const int64_t id = r.get<int64_t>();
        pa_alloc::Request q;
        q.len = r.get<int32_t>();
        q.tracked = r.get<uint8_t>() != 0;
        q.last_node = r.get<int64_t>();
        const uint64_t nt = r.count();
        for (uint64_t k = 0; r.ok && k < nt; ++k) {
            const int32_t b = r.get<int32_t>();
            if (!block_ok(b)) return bad("table entry");
            q.table.push_back(b);
        }
        const uint64_t nk = r.count();
        for (uint64_t k = 0; r.ok && k < nk; ++k) q.tokens.push_back(r.get<int32_t>());
        if (!r.ok || q.len < 0 || static_cast<int64_t>(q.table.size()) != a->blocks_for(q.len) ||
            a->reqs.count(id))
            return bad("request");
        a->reqs.emplace(id, std::move(q));
    }
    const uint64_t nn = r.get<uint64_t>();
    for (uint64_t i = 0; r.ok && i < nn; ++i) {
        const int64_t node = r.get<int64_t>(), parent = r.get<int64_t>();
        const int32_t nch = r.get<int32_t>(), blk = r.get<int32_t>();
        if (!r.ok || static_cast<uint64_t>(bs) > (size - r.n) / sizeof(int32_t)) return bad("trie node");
        PrefixKey k{parent, std::vector<int32_t>(bs)};
        for (int32_t t = 0; t < bs; ++t) k.tokens[t] = r.get<int32_t>();
        if (!r.ok || node < 0 || node >= a->next_node || nch < 0 || (blk != -1 && !block_ok(blk)) ||
            a->node_key.count(node) || a->trie.count(k))
            return bad("trie node");
        a->node_key.emplace(node, k);
        a->trie.emplace(std::move(k), node);
        a->children[node] = nch;
        if (blk >= 0) {
            if (a->block_node[blk] != -1) return bad("block cached twice");
            a->cache.emplace(node, blk);
            a->block_node[blk] = node;
        }
    }
    // every parent and every request's last registered node is a node of the trie (or the root)
    for (const auto& kv : a->node_key)
        if (kv.second.parent != -1 && !a->node_key.count(kv.second.parent)) return bad("trie parent");
    for (const auto& kv : a->reqs)
        if (kv.second.last_node != -1 && !a->node_key.count(kv.second.last_node)) return bad("request node");
    const uint64_t nl = r.count();
    for (uint64_t i = 0; r.ok && i < nl; ++i) {
        const int32_t b = r.get<int32_t>();
        if (!block_ok(b) || a->in_lru[b] || a->block_node[b] < 0 || a->refcount[b] != 0) return bad("LRU entry");
        a->lru.push_back(b);
        a->lru_pos[b] = std::prev(a->lru.end());
        a->in_lru[b] = 1;
    }
    if (!r.ok || r.n != size) return bad("length");
    // Cross-checks, so that only a consistent state is accepted: a block's refcount is the number of
    // request tables holding it; every unreferenced block is either free (unregistered) or parked
    // (registered, in the LRU), and nothing else is; a node's child count is the number of nodes
    // naming it as parent.
    std::vector<int64_t> held(nb, 0);
    for (const auto& kv : a->reqs)
        for (int32_t b : kv.second.table) held[b] += 1;
    int64_t unreferenced = 0;
    for (int32_t b = 0; b < nb; ++b) {
        if (held[b] != a->refcount[b]) return bad("refcount does not match the block tables");
        unreferenced += a->refcount[b] == 0;
    }
    for (int32_t b : a->free_list)
        if (a->refcount[b] != 0 || a->block_node[b] >= 0) return bad("free block in use or registered");
    if (unreferenced != static_cast<int64_t>(a->free_list.size() + a->lru.size()))
        return bad("unreferenced block neither free nor parked");
    std::unordered_map<int64_t, int32_t> kids;
    for (const auto& kv : a->node_key)
        if (kv.second.parent != -1) kids[kv.second.parent] += 1;
    for (const auto& kv : a->node_key) {
        auto k = kids.find(kv.first);
        if (a->children[kv.first] != (k == kids.end() ? 0 : k->second)) return bad("trie child count");
    }
    *out = a;
    return PA_OK;
}

}  // extern "C"
