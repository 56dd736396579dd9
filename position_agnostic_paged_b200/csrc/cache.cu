// cache.cu -- host-side block cache for the shared paged pool.
//
// Source: gist.science, "LazyAttention: Efficient Retrieval-Augmented
// Generation with Deferred Positional Encoding", Technical Summary (the pool
// holds one physical copy per document, reusable at any position) and
// Experimental Results (hit ratios of position-agnostic caching against
// position-aware caching and prefix caching under a KV-cache byte budget).
//
// The cache maps a key to the pool blocks of one cached entry and evicts the
// least recently used entries when a new entry does not fit.  The caching
// policy is the caller's choice of key: the document alone (position-agnostic:
// one copy serves every offset), the document and its offset
// (position-aware: one copy per offset), or the whole preceding sequence of
// documents (prefix caching).  Blocks are handed out first-fit from a set of
// free extents kept coalesced, so an entry's blocks are consecutive whenever
// a large enough free extent exists (the attention kernels then load its
// tiles with one box per 8 blocks); otherwise they come from several extents.
#include <cstdint>
#include <iterator>
#include <list>
#include <map>
#include <new>
#include <unordered_map>
#include <vector>

#include "lazy_attn.h"

struct lazy_block_cache {
    struct Entry {
        std::vector<int32_t> blocks;
        std::list<uint64_t>::iterator lru;   // position in the recency list
    };
    int64_t capacity = 0, used = 0;
    std::map<int64_t, int64_t> free_extents;   // first block -> length, disjoint and coalesced
    std::list<uint64_t> lru;                   // front: least recently used
    std::unordered_map<uint64_t, Entry> entries;
    int64_t hits = 0, misses = 0, hit_blocks = 0, miss_blocks = 0, evictions = 0;

    void release(const std::vector<int32_t> &blocks) {
        for (int32_t b : blocks) {
            int64_t start = b, len = 1;
            auto next = free_extents.lower_bound(start);
            if (next != free_extents.end() && next->first == start + len) {
                len += next->second;
                next = free_extents.erase(next);
            }
            if (next != free_extents.begin()) {
                auto prev = std::prev(next);
                if (prev->first + prev->second == start) {
                    prev->second += len;
                    continue;
                }
            }
            free_extents.emplace(start, len);
        }
        used -= static_cast<int64_t>(blocks.size());
    }

    void evict_lru() {
        const uint64_t key = lru.front();
        lru.pop_front();
        auto it = entries.find(key);
        release(it->second.blocks);
        entries.erase(it);
        ++evictions;
    }

    // n blocks, consecutive from the first extent that holds them all, else lowest addresses first
    std::vector<int32_t> allocate(int64_t n) {
        std::vector<int32_t> out;
        out.reserve(static_cast<size_t>(n));
        for (auto it = free_extents.begin(); it != free_extents.end(); ++it) {
            if (it->second >= n) {
                const int64_t start = it->first, len = it->second;
                free_extents.erase(it);
                if (len > n) free_extents.emplace(start + n, len - n);
                for (int64_t b = 0; b < n; ++b) out.push_back(static_cast<int32_t>(start + b));
                used += n;
                return out;
            }
        }
        while (static_cast<int64_t>(out.size()) < n) {
            auto it = free_extents.begin();
            const int64_t take = std::min<int64_t>(it->second, n - static_cast<int64_t>(out.size()));
            const int64_t start = it->first, len = it->second;
            free_extents.erase(it);
            if (len > take) free_extents.emplace(start + take, len - take);
            for (int64_t b = 0; b < take; ++b) out.push_back(static_cast<int32_t>(start + b));
        }
        used += n;
        return out;
    }
};

extern "C" {

lazy_block_cache *lazy_cache_create(int64_t capacity_blocks) {
    if (capacity_blocks <= 0 || capacity_blocks > static_cast<int64_t>(LAZY_MAX_BLOCKS)) return nullptr;
    lazy_block_cache *c = new (std::nothrow) lazy_block_cache();
    if (!c) return nullptr;
    c->capacity = capacity_blocks;
    c->free_extents.emplace(0, capacity_blocks);
    return c;
}

void lazy_cache_destroy(lazy_block_cache *c) { delete c; }

int lazy_cache_access(lazy_block_cache *c, uint64_t key, int32_t n_blocks, int32_t *blocks) {
    if (!c || n_blocks <= 0 || !blocks) return LAZY_EINVAL;
    auto it = c->entries.find(key);
    if (it != c->entries.end()) {
        if (static_cast<int32_t>(it->second.blocks.size()) != n_blocks) return LAZY_EINVAL;
        c->lru.splice(c->lru.end(), c->lru, it->second.lru);   // most recently used
        for (int32_t i = 0; i < n_blocks; ++i) blocks[i] = it->second.blocks[i];
        ++c->hits;
        c->hit_blocks += n_blocks;
        return 1;
    }
    ++c->misses;
    c->miss_blocks += n_blocks;
    if (n_blocks > c->capacity) return LAZY_ERANGE;   // larger than the whole cache: not cached
    while (c->capacity - c->used < n_blocks) c->evict_lru();
    lazy_block_cache::Entry e;
    e.blocks = c->allocate(n_blocks);
    for (int32_t i = 0; i < n_blocks; ++i) blocks[i] = e.blocks[i];
    e.lru = c->lru.insert(c->lru.end(), key);
    c->entries.emplace(key, std::move(e));
    return 0;
}

int lazy_cache_contains(const lazy_block_cache *c, uint64_t key) {
    if (!c) return LAZY_EINVAL;
    return c->entries.count(key) ? 1 : 0;
}

int lazy_cache_stats(const lazy_block_cache *c, int64_t *stats) {
    if (!c || !stats) return LAZY_EINVAL;
    stats[0] = c->hits;
    stats[1] = c->misses;
    stats[2] = c->hit_blocks;
    stats[3] = c->miss_blocks;
    stats[4] = c->evictions;
    stats[5] = c->used;
    stats[6] = static_cast<int64_t>(c->entries.size());
    stats[7] = static_cast<int64_t>(c->free_extents.size());
    return LAZY_OK;
}

}  // extern "C"
