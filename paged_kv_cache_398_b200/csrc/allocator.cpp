// Host block allocator of the paged KV cache: a pool of fixed-size physical
// blocks, a free list, per-block reference counts and per-sequence block
// tables, with copy-on-write for shared partially filled blocks.
//
// Follows "PagedAttention: How vLLM Serves AI Like an Operating System":
//   "How It Works"                 -- blocks, block tables, scattered blocks
//   "The Magic: No Pre-allocation" -- one block at arrival, another at token
//                                     17, 33, ...; at most 15 slots wasted
//   "Copy-on-Write: Sharing KV Cache", "Parallel Sampling", "Prefix Caching"
//                                  -- shared blocks, copy before modifying
// and "vLLM Architecture and PagedAttention" ("Page Table Visualization":
// a finished sequence's pages are freed immediately).
//
// The policy choices the pages leave open are stated in include/paged_kv.h.
#include <algorithm>
#include <cstring>
#include <list>
#include <memory>
#include <new>
#include <unordered_map>
#include <vector>

#include "paged_kv.h"

namespace {

struct Seq {
    std::vector<int32_t> blocks;
    int64_t ntok = 0;
    bool swapped = false;  // blocks live in host memory (swap_blocks_out)
    int32_t nswap = 0;     // how many
};

// Identity of a cached full block: the block it follows (and that block's
// generation, so a reused id never matches stale children) plus its tokens.
// Equal keys mean equal prefixes, compared exactly.
struct BlockKey {
    int32_t parent;    // -1 for the first block of a prompt
    uint32_t pgen;
    std::vector<int32_t> toks;
    bool operator==(const BlockKey& o) const { return parent == o.parent && pgen == o.pgen && toks == o.toks; }
};

struct BlockKeyHash {
    size_t operator()(const BlockKey& k) const
    {
        uint64_t h = 0x9e3779b97f4a7c15ull ^ (uint64_t)(uint32_t)k.parent ^ ((uint64_t)k.pgen << 32);
        for (int32_t t : k.toks) {
            h ^= (uint64_t)(uint32_t)t + 0x9e3779b97f4a7c15ull + (h << 6) + (h >> 2);
        }
        return (size_t)h;
    }
};

using CacheMap = std::unordered_map<BlockKey, int32_t, BlockKeyHash>;

// Every C entry point that can allocate runs its body through guarded: a
// failed host allocation becomes PKV_ERR_HOST_MEMORY instead of a C++
// exception crossing the C ABI.
template <typename F>
int guarded(F&& body) noexcept
{
    try {
        return body();
    } catch (...) {  // std::bad_alloc, or std::length_error for sizes past the address space
        return PKV_ERR_HOST_MEMORY;
    }
}

}  // namespace

struct pkv_allocator {
    int32_t num_blocks = 0;
    int32_t block_size = 16;
    std::vector<int32_t> free_stack;  // back() is handed out next
    std::vector<int32_t> ref;         // reference count per block
    std::unordered_map<int64_t, Seq> seqs;
    int32_t shared = 0;               // blocks with ref > 1
    // prefix cache: full prompt blocks findable by content.  Its buckets are
    // reserved for every block of the pool at creation, so it never rehashes
    // and each cached block keeps the iterator of its entry.
    CacheMap cache;
    std::vector<CacheMap::iterator> key_it;  // per block, valid while cached[b]
    std::vector<char> cached;
    std::vector<uint32_t> gen;        // per block; +1 each time it is handed out
    std::list<int32_t> lru;           // cached blocks with ref 0, least recently released first
    std::vector<std::list<int32_t>::iterator> lru_pos;
    std::vector<char> in_lru;
    int64_t lookups = 0, hits = 0, hit_tokens = 0, evictions = 0;

    int64_t available() const { return (int64_t)free_stack.size() + (int64_t)lru.size(); }
    int32_t pop()
    {
        int32_t b;
        if (!free_stack.empty()) {
            b = free_stack.back();
            free_stack.pop_back();
        } else {  // evict the least recently released cached block
            b = lru.front();
            lru.pop_front();
            in_lru[b] = 0;
            cache.erase(key_it[b]);
            cached[b] = 0;
            ++evictions;
        }
        ++gen[b];
        ref[b] = 1;
        return b;
    }
    void incref(int32_t b)
    {
        if (ref[b] == 0 && in_lru[b]) {  // a cached block comes back into use
            lru.erase(lru_pos[b]);
            in_lru[b] = 0;
        }
        if (++ref[b] == 2) ++shared;
    }
    // returns true when the block stopped being used
    bool decref(int32_t b)
    {
        if (ref[b]-- == 2) --shared;
        if (ref[b] == 0) {
            if (cached[b]) {  // keep its contents findable until evicted
                lru_pos[b] = lru.insert(lru.end(), b);
                in_lru[b] = 1;
            } else {
                free_stack.push_back(b);
            }
            return true;
        }
        return false;
    }
    // blocks an append of n tokens takes from the free list
    int64_t needs(const Seq& s, int64_t n) const
    {
        if (n == 0) return 0;
        int64_t cow = (s.ntok % block_size != 0 && ref[s.blocks.back()] > 1) ? 1 : 0;
        int64_t total = (s.ntok + n + block_size - 1) / block_size;
        return cow + total - (int64_t)s.blocks.size();
    }
    // room in s for n more tokens' block ids; the only step of an append that
    // can fail, so it comes before any change
    void reserve_for(Seq& s, int64_t n) const { s.blocks.reserve((size_t)((s.ntok + n + block_size - 1) / block_size)); }
    // caller has checked needs() against the free list and called reserve_for
    void append(Seq& s, int64_t n, int64_t* slots, int64_t* cow_pair, int32_t* cow)
    {
        int32_t did_cow = 0;
        if (n > 0 && s.ntok % block_size != 0 && ref[s.blocks.back()] > 1) {
            int32_t src = s.blocks.back();
            int32_t dst = pop();
            decref(src);
            s.blocks.back() = dst;
            did_cow = 1;
            if (cow_pair) {
                cow_pair[0] = src;
                cow_pair[1] = dst;
            }
        }
        for (int64_t i = 0; i < n; ++i) {
            int64_t p = s.ntok + i;
            if (p % block_size == 0) s.blocks.push_back(pop());
            if (slots) slots[i] = (int64_t)s.blocks[p / block_size] * block_size + p % block_size;
        }
        s.ntok += n;
        if (cow) *cow = did_cow;
    }
    Seq* find(int64_t id)
    {
        auto it = seqs.find(id);
        return it == seqs.end() ? nullptr : &it->second;
    }
    // a sequence whose blocks are on the device
    Seq* live(int64_t id)
    {
        Seq* s = find(id);
        return (s && !s->swapped) ? s : nullptr;
    }
    const Seq* find(int64_t id) const
    {
        auto it = seqs.find(id);
        return it == seqs.end() ? nullptr : &it->second;
    }
};

extern "C" {

int pkv_alloc_create(int32_t num_blocks, int32_t block_size, const int32_t* initial_order,
                     pkv_allocator** out)
{
    if (!out || num_blocks < 0 || block_size < 1) return PKV_ERR_INVALID_ARG;
    *out = nullptr;
    return guarded([&]() -> int {
        std::unique_ptr<pkv_allocator> a(new pkv_allocator());
        a->num_blocks = num_blocks;
        a->block_size = block_size;
        a->ref.assign(num_blocks, 0);
        a->cache.reserve((size_t)num_blocks);
        a->key_it.resize(num_blocks);
        a->cached.assign(num_blocks, 0);
        a->gen.assign(num_blocks, 0);
        a->lru_pos.resize(num_blocks);
        a->in_lru.assign(num_blocks, 0);
        a->free_stack.resize(num_blocks);
        if (initial_order) {
            std::vector<char> seen(num_blocks, 0);
            for (int32_t i = 0; i < num_blocks; ++i) {
                int32_t b = initial_order[i];
                if (b < 0 || b >= num_blocks || seen[b]) return PKV_ERR_INVALID_ARG;
                seen[b] = 1;
                a->free_stack[num_blocks - 1 - i] = b;
            }
        } else {
            for (int32_t i = 0; i < num_blocks; ++i) a->free_stack[num_blocks - 1 - i] = i;
        }
        *out = a.release();
        return PKV_OK;
    });
}

void pkv_alloc_destroy(pkv_allocator* a) { delete a; }

int pkv_seq_add(pkv_allocator* a, int64_t seq)
{
    if (!a || a->find(seq)) return PKV_ERR_INVALID_ARG;
    return guarded([&]() -> int {
        a->seqs.emplace(seq, Seq{});
        return PKV_OK;
    });
}

int pkv_seq_append_tokens(pkv_allocator* a, int64_t seq, int32_t n, int64_t* slots_out,
                          int64_t* cow_pair_out, int32_t* cow_out)
{
    if (!a || n < 0) return PKV_ERR_INVALID_ARG;
    Seq* s = a->live(seq);
    if (!s) return PKV_ERR_INVALID_ARG;
    if (a->needs(*s, n) > a->available()) return PKV_ERR_OUT_OF_BLOCKS;
    return guarded([&]() -> int {
        a->reserve_for(*s, n);
        a->append(*s, n, slots_out, cow_pair_out, cow_out);
        return PKV_OK;
    });
}

int pkv_batch_append_one(pkv_allocator* a, const int64_t* seqs, int32_t n_seqs,
                         int64_t* slots_out, int64_t* cow_pairs_out, int32_t* n_cow_out)
{
    if (!a || n_seqs < 0 || (n_seqs > 0 && (!seqs || !slots_out))) return PKV_ERR_INVALID_ARG;
    return guarded([&]() -> int {
    std::vector<Seq*> recs(n_seqs);
    int64_t need = 0;
    for (int32_t i = 0; i < n_seqs; ++i) {
        recs[i] = a->live(seqs[i]);
        if (!recs[i]) return PKV_ERR_INVALID_ARG;
        need += a->needs(*recs[i], 1);
    }
    {
        std::vector<int64_t> ids(seqs, seqs + n_seqs);
        std::sort(ids.begin(), ids.end());
        if (std::adjacent_find(ids.begin(), ids.end()) != ids.end()) return PKV_ERR_INVALID_ARG;
    }
    if (need > a->available()) return PKV_ERR_OUT_OF_BLOCKS;
    for (int32_t i = 0; i < n_seqs; ++i) a->reserve_for(*recs[i], 1);  // all-or-nothing: room first
    int32_t ncow = 0;
    for (int32_t i = 0; i < n_seqs; ++i) {
        int64_t pair[2];
        int32_t cow = 0;
        a->append(*recs[i], 1, slots_out + i, pair, &cow);
        if (cow) {
            if (cow_pairs_out) {
                cow_pairs_out[2 * ncow] = pair[0];
                cow_pairs_out[2 * ncow + 1] = pair[1];
            }
            ++ncow;
        }
    }
    if (n_cow_out) *n_cow_out = ncow;
    return PKV_OK;
    });
}

int pkv_seq_free(pkv_allocator* a, int64_t seq)
{
    if (!a) return PKV_ERR_INVALID_ARG;
    Seq* s = a->find(seq);
    if (!s) return PKV_ERR_INVALID_ARG;
    return guarded([&]() -> int {
        for (auto it = s->blocks.rbegin(); it != s->blocks.rend(); ++it) a->decref(*it);
        a->seqs.erase(seq);
        return PKV_OK;
    });
}

int pkv_seq_fork(pkv_allocator* a, int64_t parent, int64_t child)
{
    if (!a) return PKV_ERR_INVALID_ARG;
    const Seq* p = a->live(parent);
    if (!p || a->find(child)) return PKV_ERR_INVALID_ARG;
    return guarded([&]() -> int {
        Seq c = *p;
        const Seq& added = a->seqs.emplace(child, std::move(c)).first->second;  // the step that can fail
        for (int32_t b : added.blocks) a->incref(b);
        return PKV_OK;
    });
}

int pkv_seq_share_prefix(pkv_allocator* a, int64_t seq, const int32_t* blocks, int32_t n_blocks,
                         int32_t n_tokens)
{
    if (!a || n_blocks < 0 || n_tokens < 0 || (n_blocks > 0 && !blocks)) return PKV_ERR_INVALID_ARG;
    Seq* s = a->live(seq);
    if (!s || !s->blocks.empty() || s->ntok != 0) return PKV_ERR_INVALID_ARG;
    if ((int64_t)(n_tokens + a->block_size - 1) / a->block_size != n_blocks) return PKV_ERR_INVALID_ARG;
    for (int32_t i = 0; i < n_blocks; ++i) {
        if (blocks[i] < 0 || blocks[i] >= a->num_blocks || a->ref[blocks[i]] < 1) return PKV_ERR_BAD_BLOCK;
    }
    return guarded([&]() -> int {
        s->blocks.assign(blocks, blocks + n_blocks);  // the step that can fail
        for (int32_t i = 0; i < n_blocks; ++i) a->incref(blocks[i]);
        s->ntok = n_tokens;
        return PKV_OK;
    });
}

int pkv_seq_block_table(const pkv_allocator* a, int64_t seq, int32_t* out, int32_t cap,
                        int32_t* n_out)
{
    if (!a) return PKV_ERR_INVALID_ARG;
    const Seq* s = a->find(seq);
    if (!s) return PKV_ERR_INVALID_ARG;
    int32_t n = (int32_t)s->blocks.size();
    if (n_out) *n_out = n;
    if (n > cap || (n > 0 && !out)) return PKV_ERR_INVALID_ARG;
    if (n > 0) std::memcpy(out, s->blocks.data(), sizeof(int32_t) * n);
    return PKV_OK;
}

int pkv_seq_num_tokens(const pkv_allocator* a, int64_t seq, int32_t* out)
{
    if (!a || !out) return PKV_ERR_INVALID_ARG;
    const Seq* s = a->find(seq);
    if (!s) return PKV_ERR_INVALID_ARG;
    *out = (int32_t)s->ntok;
    return PKV_OK;
}

int pkv_batch_tables(const pkv_allocator* a, const int64_t* seqs, int32_t n_seqs,
                     int32_t* tables_out, int32_t max_blocks_per_seq, int32_t pad,
                     int32_t* context_lens_out)
{
    if (!a || n_seqs < 0 || max_blocks_per_seq < 0 || (n_seqs > 0 && (!seqs || !tables_out)))
        return PKV_ERR_INVALID_ARG;
    for (int32_t i = 0; i < n_seqs; ++i) {
        const Seq* s = a->find(seqs[i]);
        if (!s || s->swapped || (int64_t)s->blocks.size() > max_blocks_per_seq) return PKV_ERR_INVALID_ARG;
    }
    for (int32_t i = 0; i < n_seqs; ++i) {
        const Seq* s = a->find(seqs[i]);
        int32_t* row = tables_out + (int64_t)i * max_blocks_per_seq;
        int32_t n = (int32_t)s->blocks.size();
        if (n > 0) std::memcpy(row, s->blocks.data(), sizeof(int32_t) * n);
        if (pad != PKV_TABLE_KEEP_TAIL)
            for (int32_t j = n; j < max_blocks_per_seq; ++j) row[j] = pad;
        if (context_lens_out) context_lens_out[i] = (int32_t)s->ntok;
    }
    return PKV_OK;
}

int32_t pkv_num_free(const pkv_allocator* a) { return a ? (int32_t)a->available() : -1; }

int pkv_free_list(const pkv_allocator* a, int32_t* out, int32_t cap, int32_t* n_out)
{
    if (!a) return PKV_ERR_INVALID_ARG;
    const int32_t ns = (int32_t)a->free_stack.size();
    const int32_t n = (int32_t)a->available();
    if (n_out) *n_out = n;
    if (n > cap || (n > 0 && !out)) return PKV_ERR_INVALID_ARG;
    for (int32_t i = 0; i < ns; ++i) out[i] = a->free_stack[ns - 1 - i];
    int32_t i = ns;
    for (int32_t b : a->lru) out[i++] = b;  // then the cached blocks, in eviction order
    return PKV_OK;
}

int32_t pkv_refcount(const pkv_allocator* a, int32_t block)
{
    if (!a || block < 0 || block >= a->num_blocks) return -1;
    return a->ref[block];
}

int pkv_alloc_get_stats(const pkv_allocator* a, pkv_alloc_stats* out)
{
    if (!a || !out) return PKV_ERR_INVALID_ARG;
    out->num_blocks = a->num_blocks;
    out->free_blocks = (int32_t)a->available();
    out->used_blocks = a->num_blocks - out->free_blocks;
    out->shared_blocks = a->shared;
    out->num_seqs = (int64_t)a->seqs.size();
    int64_t tok = 0, frag = 0;
    for (const auto& kv : a->seqs) {
        tok += kv.second.ntok;
        if (!kv.second.swapped) frag += (int64_t)kv.second.blocks.size() * a->block_size - kv.second.ntok;
    }
    out->num_tokens = tok;
    out->fragmentation_tokens = frag;
    return PKV_OK;
}

int pkv_seq_append_prompt(pkv_allocator* a, int64_t seq, const int32_t* token_ids, int32_t n,
                          int64_t* slots_out, int32_t* n_cached_out)
{
    if (!a || n < 0 || (n > 0 && !token_ids)) return PKV_ERR_INVALID_ARG;
    Seq* s = a->live(seq);
    if (!s || !s->blocks.empty() || s->ntok != 0) return PKV_ERR_INVALID_ARG;
    return guarded([&]() -> int {
        const int32_t B = a->block_size;
        const int32_t nfull = n / B;
        // leading full blocks already cached, walked in order with one probe key
        std::vector<int32_t> hit;
        hit.reserve((size_t)nfull);
        BlockKey probe{-1, 0, std::vector<int32_t>((size_t)B)};
        int32_t revived = 0;  // hits now resting in the LRU list (not available to others)
        for (int32_t k = 0; k < nfull; ++k) {
            std::copy(token_ids + (int64_t)k * B, token_ids + (int64_t)(k + 1) * B, probe.toks.begin());
            auto it = a->cache.find(probe);
            if (it == a->cache.end()) break;
            hit.push_back(it->second);
            if (a->ref[it->second] == 0) ++revived;
            probe.parent = it->second;
            probe.pgen = a->gen[it->second];
        }
        const int64_t fresh = (int64_t)(n + B - 1) / B - (int64_t)hit.size();
        if (fresh > a->available() - revived) return PKV_ERR_OUT_OF_BLOCKS;
        a->reserve_for(*s, n);
        a->lookups += nfull > 0 ? 1 : 0;
        a->hits += hit.empty() ? 0 : 1;
        for (int32_t b : hit) {
            a->incref(b);
            s->blocks.push_back(b);
        }
        const int32_t cached = (int32_t)hit.size() * B;
        a->hit_tokens += cached;
        s->ntok = cached;
        for (int32_t i = 0; i < cached && slots_out; ++i) slots_out[i] = -1;
        a->append(*s, n - cached, slots_out ? slots_out + cached : nullptr, nullptr, nullptr);
        // make this prompt's new full blocks findable by the next request.  The
        // first is keyed under the last hit (whose lookup just missed), the rest
        // under freshly handed-out blocks, so every key is new.  Caching is
        // best effort: if host memory runs out here, the remaining blocks stay
        // unfindable (a later miss, never a wrong hit) and the admission stands.
        try {
            for (int32_t k = (int32_t)hit.size(); k < nfull; ++k) {
                const int32_t b = s->blocks[k];
                const int32_t par = k == 0 ? -1 : s->blocks[k - 1];
                auto res = a->cache.emplace(
                    BlockKey{par, par < 0 ? 0u : a->gen[par],
                             std::vector<int32_t>(token_ids + (int64_t)k * B, token_ids + (int64_t)(k + 1) * B)},
                    b);
                if (res.second) {
                    a->key_it[b] = res.first;
                    a->cached[b] = 1;
                }
            }
        } catch (...) {
        }
        if (n_cached_out) *n_cached_out = cached;
        return PKV_OK;
    });
}

int pkv_prefix_cache_stats(const pkv_allocator* a, pkv_prefix_stats* out)
{
    if (!a || !out) return PKV_ERR_INVALID_ARG;
    out->cached_blocks = (int32_t)a->cache.size();
    out->evictable_blocks = (int32_t)a->lru.size();
    out->prompts = a->lookups;
    out->prompts_with_hits = a->hits;
    out->hit_tokens = a->hit_tokens;
    out->evictions = a->evictions;
    return PKV_OK;
}

int pkv_seq_swap_out(pkv_allocator* a, int64_t seq, int32_t* blocks_out, int32_t cap, int32_t* n_out)
{
    if (!a) return PKV_ERR_INVALID_ARG;
    Seq* s = a->live(seq);
    if (!s) return PKV_ERR_INVALID_ARG;
    const int32_t n = (int32_t)s->blocks.size();
    if (n_out) *n_out = n;
    if (n > cap || (n > 0 && !blocks_out)) return PKV_ERR_INVALID_ARG;
    if (n > 0) std::memcpy(blocks_out, s->blocks.data(), sizeof(int32_t) * n);
    return guarded([&]() -> int {
        for (auto it = s->blocks.rbegin(); it != s->blocks.rend(); ++it) a->decref(*it);
        s->blocks.clear();
        s->swapped = true;
        s->nswap = n;
        return PKV_OK;
    });
}

int pkv_seq_swap_in(pkv_allocator* a, int64_t seq, int32_t* blocks_out, int32_t cap, int32_t* n_out)
{
    if (!a) return PKV_ERR_INVALID_ARG;
    Seq* s = a->find(seq);
    if (!s || !s->swapped) return PKV_ERR_INVALID_ARG;
    const int32_t n = s->nswap;
    if (n_out) *n_out = n;
    if (n > cap || (n > 0 && !blocks_out)) return PKV_ERR_INVALID_ARG;
    if (n > a->available()) return PKV_ERR_OUT_OF_BLOCKS;
    return guarded([&]() -> int {
        s->blocks.reserve((size_t)n);  // the step that can fail, before any change
        for (int32_t i = 0; i < n; ++i) s->blocks.push_back(a->pop());
        if (n > 0) std::memcpy(blocks_out, s->blocks.data(), sizeof(int32_t) * n);
        s->swapped = false;
        s->nswap = 0;
        return PKV_OK;
    });
}

int pkv_seq_is_swapped(const pkv_allocator* a, int64_t seq, int32_t* out)
{
    if (!a || !out) return PKV_ERR_INVALID_ARG;
    const Seq* s = a->find(seq);
    if (!s) return PKV_ERR_INVALID_ARG;
    *out = s->swapped ? 1 : 0;
    return PKV_OK;
}

int pkv_slot_mapping(const int32_t* block_tables, int32_t max_blocks_per_seq,
                     const int32_t* positions, int32_t num_seqs, int32_t block_size,
                     int64_t* slots_out)
{
    if (num_seqs < 0 || block_size < 1 || max_blocks_per_seq < 0 ||
        (num_seqs > 0 && (!block_tables || !positions || !slots_out)))
        return PKV_ERR_INVALID_ARG;
    for (int32_t s = 0; s < num_seqs; ++s) {
        int32_t p = positions[s];
        if (p < 0) continue;
        if (p / block_size >= max_blocks_per_seq) return PKV_ERR_INVALID_ARG;
        if (block_tables[(int64_t)s * max_blocks_per_seq + p / block_size] < 0) return PKV_ERR_BAD_BLOCK;
    }
    for (int32_t s = 0; s < num_seqs; ++s) {
        int32_t p = positions[s];
        if (p < 0) {
            slots_out[s] = -1;
            continue;
        }
        int64_t phys = block_tables[(int64_t)s * max_blocks_per_seq + p / block_size];
        slots_out[s] = phys * block_size + p % block_size;
    }
    return PKV_OK;
}

}  // extern "C"
