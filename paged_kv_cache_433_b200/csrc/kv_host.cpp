// Host side of the paged KV cache: refcounted page pool, chained-hash prefix
// index, slot bookkeeping. Plain C++17, no CUDA. See include/kvpaged.h for the
// contract of every entry point and the pages each one follows.
//
// Pages cited: [HB-07] "07｜KV Cache、FlashAttention与PagedAttention的内部过程"
// (Q028 block-table walk, shared blocks and copy-on-write); [CN-06]
// "06 KV Cache、Prefix Cache、PagedAttention 与 vLLM" (6.4 chained block hash,
// 6.5 allocation flow); [KV-04] "04. 注意力与 KV 缓存" (prefix demo, pages still
// in use are not reclaimed).
#include "kvpaged.h"

#include <cstring>
#include <memory>
#include <new>
#include <unordered_map>
#include <vector>

namespace {

constexpr int32_t kNone = -1;

}  // namespace

struct kv_prefix;

// Free list: doubly linked list threaded through per-page prev/next arrays, so
// a cached page can leave the middle of the list in O(1) when it is revived.
struct kv_pool {
    int32_t num_pages = 0;
    int32_t page_size = 0;
    std::vector<int32_t> ref;
    std::vector<int32_t> prev, next;
    std::vector<uint8_t> in_free;
    int32_t head = kNone, tail = kNone, n_free = 0;
    std::vector<kv_prefix*> indexes;  // prefix indexes bound to this pool

    void push_tail(int32_t p) {
        prev[p] = tail;
        next[p] = kNone;
        if (tail != kNone) next[tail] = p; else head = p;
        tail = p;
        in_free[p] = 1;
        ++n_free;
    }
    void unlink(int32_t p) {
        if (prev[p] != kNone) next[prev[p]] = next[p]; else head = next[p];
        if (next[p] != kNone) prev[next[p]] = prev[p]; else tail = prev[p];
        prev[p] = next[p] = kNone;
        in_free[p] = 0;
        --n_free;
    }
    bool valid(int32_t p) const { return p >= 0 && p < num_pages; }
};

// One registered full block. Entries form a tree through `parent` (the block
// before it in the same prefix); ids are never reused, so a child can check
// that it hangs under the entry matched one block earlier.
struct PrefixEntry {
    uint64_t id;
    uint64_t key;
    uint64_t parent;  // 0 = first block of a prefix
    int32_t page;
    std::vector<int32_t> tokens;
    std::vector<uint64_t> children;
};

struct kv_prefix {
    int32_t page_size = 0;
    uint64_t salt = 0;
    kv_pool* pool = nullptr;
    uint64_t next_id = 1;
    std::unordered_map<uint64_t, PrefixEntry> entries;                 // id -> entry
    std::unordered_map<uint64_t, std::vector<uint64_t>> by_key;        // chained key -> entry ids
    std::unordered_map<int32_t, uint64_t> by_page;                     // page -> entry id

    // FNV-1a 64 over the parent key (8 bytes, little-endian) and the block's
    // tokens (4 bytes each, little-endian).
    static uint64_t chain(uint64_t parent_key, const int32_t* toks, int32_t n) {
        uint64_t h = 0xcbf29ce484222325ull;
        auto mix = [&h](uint8_t byte) {
            h ^= byte;
            h *= 0x100000001b3ull;
        };
        for (int i = 0; i < 8; ++i) mix(static_cast<uint8_t>(parent_key >> (8 * i)));
        for (int32_t t = 0; t < n; ++t) {
            uint32_t v = static_cast<uint32_t>(toks[t]);
            for (int i = 0; i < 4; ++i) mix(static_cast<uint8_t>(v >> (8 * i)));
        }
        return h;
    }

    // Entry for (parent entry, block tokens) under `key`, or 0.
    uint64_t find(uint64_t key, uint64_t parent, const int32_t* toks) const {
        auto it = by_key.find(key);
        if (it == by_key.end()) return 0;
        for (uint64_t id : it->second) {
            const PrefixEntry& e = entries.at(id);
            if (e.parent == parent && std::memcmp(e.tokens.data(), toks, sizeof(int32_t) * page_size) == 0) return id;
        }
        return 0;
    }

    void erase_subtree(uint64_t id) {
        std::vector<uint64_t> stack{id};
        while (!stack.empty()) {
            uint64_t cur = stack.back();
            stack.pop_back();
            auto it = entries.find(cur);
            if (it == entries.end()) continue;
            for (uint64_t c : it->second.children) stack.push_back(c);
            auto& bucket = by_key[it->second.key];
            for (size_t i = 0; i < bucket.size(); ++i)
                if (bucket[i] == cur) { bucket.erase(bucket.begin() + i); break; }
            if (bucket.empty()) by_key.erase(it->second.key);
            by_page.erase(it->second.page);
            if (it->second.parent) {
                auto pit = entries.find(it->second.parent);
                if (pit != entries.end()) {
                    auto& ch = pit->second.children;
                    for (size_t i = 0; i < ch.size(); ++i)
                        if (ch[i] == cur) { ch.erase(ch.begin() + i); break; }
                }
            }
            entries.erase(it);
        }
    }

    void evict_page(int32_t page) {
        auto it = by_page.find(page);
        if (it != by_page.end()) erase_subtree(it->second);
    }
    bool registered(int32_t page) const { return by_page.count(page) != 0; }
};

namespace {

bool pool_page_cached(const kv_pool* pool, int32_t p) {
    for (const kv_prefix* ix : pool->indexes)
        if (ix->registered(p)) return true;
    return false;
}

void detach_index(kv_prefix* ix) {
    if (!ix->pool) return;
    auto& v = ix->pool->indexes;
    for (size_t i = 0; i < v.size(); ++i)
        if (v[i] == ix) { v.erase(v.begin() + i); break; }
    ix->pool = nullptr;
}

}  // namespace

extern "C" {

const char* kv_status_string(int status) {
    switch (status) {
        case KV_OK: return "ok";
        case KV_ERR_ARG: return "invalid argument";
        case KV_ERR_OOM: return "out of pages";
        case KV_ERR_BAD_ID: return "bad page id";
        case KV_ERR_DOUBLE_FREE: return "page freed more times than held";
        case KV_ERR_SHARED_TAIL: return "append into a shared partial page (copy-on-write needed)";
        case KV_ERR_CUDA: return "CUDA error";
        case KV_ERR_WORKSPACE: return "workspace missing or too small";
        case KV_ERR_UNSUPPORTED: return "unsupported shape";
        default: return "unknown status";
    }
}

int kv_version(void) { return 1; }

int kv_pool_create(int32_t num_pages, int32_t page_size, const int32_t* init_free_order, kv_pool_t** out) {
    if (!out || num_pages <= 0 || page_size <= 0) return KV_ERR_ARG;
    std::unique_ptr<kv_pool> p(new (std::nothrow) kv_pool());
    if (!p) return KV_ERR_OOM;
    p->num_pages = num_pages;
    p->page_size = page_size;
    p->ref.assign(num_pages, 0);
    p->prev.assign(num_pages, kNone);
    p->next.assign(num_pages, kNone);
    p->in_free.assign(num_pages, 0);
    if (init_free_order) {
        std::vector<uint8_t> seen(num_pages, 0);
        for (int32_t i = 0; i < num_pages; ++i) {
            int32_t id = init_free_order[i];
            if (id < 0 || id >= num_pages || seen[id]) return KV_ERR_ARG;
            seen[id] = 1;
        }
        for (int32_t i = 0; i < num_pages; ++i) p->push_tail(init_free_order[i]);
    } else {
        for (int32_t i = 0; i < num_pages; ++i) p->push_tail(i);
    }
    *out = p.release();
    return KV_OK;
}

int kv_pool_destroy(kv_pool_t* pool) {
    if (!pool) return KV_ERR_ARG;
    for (kv_prefix* ix : pool->indexes) ix->pool = nullptr;
    delete pool;
    return KV_OK;
}

int kv_pool_alloc(kv_pool_t* pool, int32_t n, int32_t* out_ids) {
    if (!pool || n < 0 || (n > 0 && !out_ids)) return KV_ERR_ARG;
    if (n > pool->n_free) return KV_ERR_OOM;
    for (int32_t i = 0; i < n; ++i) {
        int32_t p = pool->head;
        pool->unlink(p);
        pool->ref[p] = 1;
        for (kv_prefix* ix : pool->indexes) ix->evict_page(p);
        out_ids[i] = p;
    }
    return KV_OK;
}

int kv_pool_free(kv_pool_t* pool, int32_t n, const int32_t* ids) {
    if (!pool || n < 0 || (n > 0 && !ids)) return KV_ERR_ARG;
    std::unordered_map<int32_t, int32_t> need;
    for (int32_t i = 0; i < n; ++i) {
        if (!pool->valid(ids[i])) return KV_ERR_BAD_ID;
        ++need[ids[i]];
    }
    for (auto& kv : need)
        if (kv.second > pool->ref[kv.first]) return KV_ERR_DOUBLE_FREE;
    for (int32_t i = 0; i < n; ++i) {
        int32_t p = ids[i];
        if (--pool->ref[p] == 0) pool->push_tail(p);
    }
    return KV_OK;
}

int kv_pool_incref(kv_pool_t* pool, int32_t n, const int32_t* ids) {
    if (!pool || n < 0 || (n > 0 && !ids)) return KV_ERR_ARG;
    for (int32_t i = 0; i < n; ++i) {
        if (!pool->valid(ids[i])) return KV_ERR_BAD_ID;
        if (pool->ref[ids[i]] == 0 && !pool_page_cached(pool, ids[i])) return KV_ERR_BAD_ID;
    }
    for (int32_t i = 0; i < n; ++i) {
        int32_t p = ids[i];
        if (pool->ref[p] == 0) pool->unlink(p);
        ++pool->ref[p];
    }
    return KV_OK;
}

int kv_pool_refcount(const kv_pool_t* pool, int32_t id, int32_t* out) {
    if (!pool || !out) return KV_ERR_ARG;
    if (!pool->valid(id)) return KV_ERR_BAD_ID;
    *out = pool->ref[id];
    return KV_OK;
}

int kv_pool_num_free(const kv_pool_t* pool, int32_t* out) {
    if (!pool || !out) return KV_ERR_ARG;
    *out = pool->n_free;
    return KV_OK;
}

int kv_pool_page_size(const kv_pool_t* pool, int32_t* out) {
    if (!pool || !out) return KV_ERR_ARG;
    *out = pool->page_size;
    return KV_OK;
}

int kv_blocks_for_len(int32_t len, int32_t page_size, int32_t* pages, int32_t* slots, int32_t* wasted) {
    if (len < 0 || page_size <= 0 || !pages || !slots || !wasted) return KV_ERR_ARG;
    int32_t b = (len + page_size - 1) / page_size;
    *pages = b;
    *slots = b * page_size;
    *wasted = b * page_size - len;
    return KV_OK;
}

int kv_cache_bytes(int64_t L, int64_t B, int64_t T, int64_t H_kv, int64_t Dh, int64_t bytes_per_elem, int64_t* out) {
    if (!out || L < 0 || B < 0 || T < 0 || H_kv < 0 || Dh < 0 || bytes_per_elem < 0) return KV_ERR_ARG;
    *out = 2 * L * B * T * H_kv * Dh * bytes_per_elem;
    return KV_OK;
}

int kv_slot_for_pos(const int32_t* table_row, int32_t n_blocks, int32_t page_size, int64_t pos, int64_t* out) {
    if (!table_row || !out || page_size <= 0 || pos < 0) return KV_ERR_ARG;
    int64_t blk = pos / page_size;
    if (blk >= n_blocks) return KV_ERR_ARG;
    int32_t page = table_row[blk];
    if (page < 0) return KV_ERR_BAD_ID;
    *out = static_cast<int64_t>(page) * page_size + pos % page_size;
    return KV_OK;
}

int kv_slots_for_range(const int32_t* table_row, int32_t n_blocks, int32_t page_size, int64_t start, int64_t n,
                       int64_t* out_slots) {
    if (!table_row || page_size <= 0 || start < 0 || n < 0 || (n > 0 && !out_slots)) return KV_ERR_ARG;
    for (int64_t i = 0; i < n; ++i) {
        int rc = kv_slot_for_pos(table_row, n_blocks, page_size, start + i, &out_slots[i]);
        if (rc != KV_OK) return rc;
    }
    return KV_OK;
}

int kv_append_slots(kv_pool_t* pool, int32_t B, int32_t* block_tables, int32_t max_blocks, int32_t* seq_lens,
                    int64_t* slot_mapping) {
    if (!pool || B < 0 || max_blocks <= 0 || (B > 0 && (!block_tables || !seq_lens || !slot_mapping))) return KV_ERR_ARG;
    const int32_t P = pool->page_size;
    int32_t need = 0;
    for (int32_t b = 0; b < B; ++b) {
        int32_t L = seq_lens[b];
        if (L < 0 || L / P >= max_blocks) return KV_ERR_ARG;
        if (L % P == 0) {
            ++need;
        } else {
            int32_t tail = block_tables[static_cast<int64_t>(b) * max_blocks + L / P];
            if (!pool->valid(tail)) return KV_ERR_BAD_ID;
            if (pool->ref[tail] > 1) return KV_ERR_SHARED_TAIL;
        }
    }
    std::vector<int32_t> fresh(need);
    int rc = kv_pool_alloc(pool, need, fresh.data());
    if (rc != KV_OK) return rc;
    int32_t k = 0;
    for (int32_t b = 0; b < B; ++b) {
        int32_t L = seq_lens[b];
        int32_t* row = block_tables + static_cast<int64_t>(b) * max_blocks;
        if (L % P == 0) row[L / P] = fresh[k++];
        slot_mapping[b] = static_cast<int64_t>(row[L / P]) * P + L % P;
        seq_lens[b] = L + 1;
    }
    return KV_OK;
}

int kv_pool_cow_tails(kv_pool_t* pool, int32_t B, int32_t* block_tables, int32_t max_blocks, const int32_t* seq_lens,
                      int32_t* src_pages, int32_t* dst_pages, int32_t* n_copies) {
    if (!pool || !n_copies || B < 0 || max_blocks <= 0 ||
        (B > 0 && (!block_tables || !seq_lens || !src_pages || !dst_pages)))
        return KV_ERR_ARG;
    const int32_t P = pool->page_size;
    // First pass: which sequences copy (in order, while the tail is still shared).
    std::unordered_map<int32_t, int32_t> sim;
    std::vector<int32_t> marked;
    for (int32_t b = 0; b < B; ++b) {
        const int32_t L = seq_lens[b];
        if (L < 0 || L / P >= max_blocks) return KV_ERR_ARG;
        if (L % P == 0) continue;
        const int32_t t = block_tables[static_cast<int64_t>(b) * max_blocks + L / P];
        if (!pool->valid(t)) return KV_ERR_BAD_ID;
        auto it = sim.find(t);
        const int32_t r = it == sim.end() ? pool->ref[t] : it->second;
        if (r > 1) {
            marked.push_back(b);
            sim[t] = r - 1;
        }
    }
    std::vector<int32_t> fresh(marked.size());
    int rc = kv_pool_alloc(pool, static_cast<int32_t>(marked.size()), fresh.data());
    if (rc != KV_OK) return rc;
    for (size_t k = 0; k < marked.size(); ++k) {
        const int32_t b = marked[k];
        int32_t& slot = block_tables[static_cast<int64_t>(b) * max_blocks + seq_lens[b] / P];
        const int32_t old = slot;
        slot = fresh[k];
        if (--pool->ref[old] == 0) pool->push_tail(old);
        src_pages[k] = old;
        dst_pages[k] = fresh[k];
    }
    *n_copies = static_cast<int32_t>(marked.size());
    return KV_OK;
}

int kv_prefix_index_create(int32_t page_size, uint64_t salt, kv_prefix_t** out) {
    if (!out || page_size <= 0) return KV_ERR_ARG;
    kv_prefix* ix = new (std::nothrow) kv_prefix();
    if (!ix) return KV_ERR_OOM;
    ix->page_size = page_size;
    ix->salt = salt;
    *out = ix;
    return KV_OK;
}

int kv_prefix_index_destroy(kv_prefix_t* index) {
    if (!index) return KV_ERR_ARG;
    detach_index(index);
    delete index;
    return KV_OK;
}

int kv_prefix_register(kv_prefix_t* ix, kv_pool_t* pool, const int32_t* tokens, int32_t n, const int32_t* page_ids) {
    if (!ix || !pool || n < 0 || (n > 0 && !tokens)) return KV_ERR_ARG;
    if (pool->page_size != ix->page_size) return KV_ERR_ARG;
    if (ix->pool && ix->pool != pool) return KV_ERR_ARG;
    const int32_t P = ix->page_size;
    const int32_t nfull = n / P;
    if (nfull > 0 && !page_ids) return KV_ERR_ARG;
    // Validate everything first (all-or-nothing).
    {
        uint64_t key = ix->salt, parent = 0;
        bool chain_known = true;
        for (int32_t i = 0; i < nfull; ++i) {
            int32_t p = page_ids[i];
            if (!pool->valid(p) || pool->ref[p] == 0) return KV_ERR_BAD_ID;
            uint64_t k = kv_prefix::chain(key, tokens + static_cast<int64_t>(i) * P, P);
            uint64_t id = chain_known ? ix->find(k, parent, tokens + static_cast<int64_t>(i) * P) : 0;
            auto bp = ix->by_page.find(p);
            if (bp != ix->by_page.end() && bp->second != id) return KV_ERR_ARG;  // page holds another prefix
            if (id == 0) chain_known = false;
            parent = id;
            key = k;
        }
    }
    if (!ix->pool) {
        ix->pool = pool;
        pool->indexes.push_back(ix);
    }
    uint64_t key = ix->salt, parent = 0;
    for (int32_t i = 0; i < nfull; ++i) {
        const int32_t* blk = tokens + static_cast<int64_t>(i) * P;
        uint64_t k = kv_prefix::chain(key, blk, P);
        uint64_t id = ix->find(k, parent, blk);
        if (id == 0) {
            id = ix->next_id++;
            PrefixEntry e;
            e.id = id;
            e.key = k;
            e.parent = parent;
            e.page = page_ids[i];
            e.tokens.assign(blk, blk + P);
            ix->entries.emplace(id, std::move(e));
            ix->by_key[k].push_back(id);
            ix->by_page[page_ids[i]] = id;
            if (parent) ix->entries.at(parent).children.push_back(id);
        }
        parent = id;
        key = k;
    }
    return KV_OK;
}

int kv_prefix_match(const kv_prefix_t* ix, const int32_t* tokens, int32_t n, int32_t page_size, int32_t* out_page_ids,
                    int32_t* out_num_pages) {
    if (!ix || !out_num_pages || n < 0 || (n > 0 && !tokens)) return KV_ERR_ARG;
    if (page_size != ix->page_size) return KV_ERR_ARG;
    const int32_t P = ix->page_size;
    uint64_t key = ix->salt, parent = 0;
    int32_t hits = 0;
    for (int32_t i = 0; i < n / P; ++i) {
        const int32_t* blk = tokens + static_cast<int64_t>(i) * P;
        uint64_t k = kv_prefix::chain(key, blk, P);
        uint64_t id = ix->find(k, parent, blk);
        if (id == 0) break;
        if (out_page_ids) out_page_ids[hits] = ix->entries.at(id).page;
        ++hits;
        parent = id;
        key = k;
    }
    *out_num_pages = hits;
    return KV_OK;
}

int kv_prefix_num_entries(const kv_prefix_t* ix, int32_t* out) {
    if (!ix || !out) return KV_ERR_ARG;
    *out = static_cast<int32_t>(ix->entries.size());
    return KV_OK;
}

}  // extern "C"
