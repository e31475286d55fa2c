// Host side of shared-prefix decode: find, in a batch's block tables, the
// runs of consecutive sequences that start with the same physical blocks
// (samples forked from one prompt, requests that found one cached prefix:
// "Copy-on-Write: Sharing KV Cache", "Parallel Sampling", "Prefix Caching"),
// and the length x whose blocks each such group can read once per step.
//
// Greedy, in batch order: a group starts at sequence i and takes i + 1,
// i + 2, ... while the blocks every member has in common still cover at
// least min_shared_tokens positions and the group has room.  x is those
// common blocks times the block size, kept below every member's length, so
// each member still has its own last position (where the step's new token
// lands) for its own pass.
//
// The work list names every partition of both passes for the decode launch
// (one thread block per item and kv head): (~g, p) for partition p of group
// g's shared positions, (s, p) for partition p of sequence s's own.  Items go
// longest first (ties: group items, then batch order), so the long ones
// start early and the short ones fill the end of the launch.
#include <algorithm>
#include <cstdint>
#include <cstring>
#include <numeric>
#include <vector>

#include "paged_kv.h"

namespace {

// Leading entries of rows a and b that are equal, up to n: whole chunks by
// memcmp (sibling rows agree over a whole prompt), then the differing chunk
// entry by entry.
int32_t common_entries(const int32_t* a, const int32_t* b, int32_t n)
{
    constexpr int32_t kChunk = 16;
    int32_t k = 0;
    while (k + kChunk <= n && std::memcmp(a + k, b + k, kChunk * sizeof(int32_t)) == 0) k += kChunk;
    while (k < n && a[k] == b[k]) ++k;
    return k;
}

// Leading entries of a row that name a block (non-negative), up to n.
int32_t valid_entries(const int32_t* a, int32_t n)
{
    int32_t k = 0;
    while (k < n && a[k] >= 0) ++k;
    return k;
}

}  // namespace

extern "C" int pkv_shared_prefix_plan(const int32_t* block_tables, int32_t max_blocks_per_seq,
                                      const int32_t* context_lens, int32_t num_seqs, int32_t block_size,
                                      int32_t max_group, int32_t min_shared_tokens, int32_t part_tokens,
                                      int32_t* groups_out, int32_t* num_groups_out, int32_t* shared_lens_out,
                                      int32_t* work_out, int32_t work_cap, int32_t* num_work_out,
                                      int32_t* max_shared_len_out, int32_t* max_own_len_out)
{
    if (num_seqs < 0 || max_blocks_per_seq < 1 || block_size < 1 || max_group < 1 || min_shared_tokens < 0 ||
        part_tokens < 1 || work_cap < 0 || !num_groups_out || !num_work_out || !max_shared_len_out ||
        !max_own_len_out)
        return PKV_ERR_INVALID_ARG;
    if (num_seqs > 0 && (!block_tables || !context_lens || !groups_out || !shared_lens_out))
        return PKV_ERR_INVALID_ARG;
    const int64_t cap = (int64_t)max_blocks_per_seq * block_size;
    for (int32_t s = 0; s < num_seqs; ++s)
        if (context_lens[s] < 1 || context_lens[s] > cap) return PKV_ERR_INVALID_ARG;

    auto row = [&](int32_t s) { return block_tables + (int64_t)s * max_blocks_per_seq; };
    // blocks of sequence s that lie wholly below its last position
    auto below_last = [&](int32_t s) { return (context_lens[s] - 1) / block_size; };
    const int64_t min_tokens = std::max<int64_t>(min_shared_tokens, block_size);

    int32_t ng = 0, max_shared = 0, max_own = 0;
    int32_t i = 0;
    while (i < num_seqs) {
        int32_t common = valid_entries(row(i), below_last(i));  // blocks all members hold, so far
        int32_t n = 1;
        while (i + n < num_seqs && n < max_group) {
            const int32_t j = i + n;
            const int32_t c = common_entries(row(i), row(j), std::min(common, below_last(j)));
            if ((int64_t)c * block_size < min_tokens) break;
            common = c;
            ++n;
        }
        const int32_t x = n >= 2 ? common * block_size : 0;
        if (n >= 2) {
            groups_out[2 * ng] = i;
            groups_out[2 * ng + 1] = n;
            ++ng;
        } else {
            n = 1;
        }
        for (int32_t j = i; j < i + n; ++j) {
            shared_lens_out[j] = x;
            max_own = std::max(max_own, context_lens[j] - x);
        }
        max_shared = std::max(max_shared, x);
        i += n;
    }
    *num_groups_out = ng;
    *max_shared_len_out = max_shared;
    *max_own_len_out = max_own;

    // the work list: (tokens, first, second) per item, longest first
    struct Item {
        int32_t tokens, a, p;
    };
    std::vector<Item> items;
    try {
        items.reserve((size_t)num_seqs + (size_t)ng * 4);
    } catch (...) {
        return PKV_ERR_HOST_MEMORY;  // no memory for the list: the outputs are not written
    }
    try {
        for (int32_t g = 0; g < ng; ++g) {
            const int32_t x = shared_lens_out[groups_out[2 * g]];
            for (int32_t p = 0; (int64_t)p * part_tokens < x; ++p)
                items.push_back({std::min(part_tokens, x - p * part_tokens), ~g, p});
        }
        for (int32_t s = 0; s < num_seqs; ++s) {
            const int32_t own = context_lens[s] - shared_lens_out[s];
            for (int32_t p = 0; (int64_t)p * part_tokens < own; ++p)
                items.push_back({std::min(part_tokens, own - p * part_tokens), s, p});
        }
    } catch (...) {
        return PKV_ERR_HOST_MEMORY;
    }
    std::stable_sort(items.begin(), items.end(), [](const Item& l, const Item& r) { return l.tokens > r.tokens; });
    *num_work_out = (int32_t)items.size();
    if (!work_out) return PKV_OK;  // a query of the size
    if ((int64_t)items.size() > work_cap) return PKV_ERR_INVALID_ARG;
    for (size_t k = 0; k < items.size(); ++k) {
        work_out[2 * k] = items[k].a;
        work_out[2 * k + 1] = items[k].p;
    }
    return PKV_OK;
}

// A batch order that puts sequences whose tables start with the same blocks
// next to each other: the rows' shareable blocks (valid ids wholly below the
// sequence's last position) in lexicographic order, stable, so a common
// prefix makes a contiguous run and siblings keep their batch order.
extern "C" int pkv_shared_prefix_order(const int32_t* block_tables, int32_t max_blocks_per_seq,
                                       const int32_t* context_lens, int32_t num_seqs, int32_t block_size,
                                       int64_t* order_out)
{
    if (num_seqs < 0 || max_blocks_per_seq < 1 || block_size < 1) return PKV_ERR_INVALID_ARG;
    if (num_seqs == 0) return PKV_OK;
    if (!block_tables || !context_lens || !order_out) return PKV_ERR_INVALID_ARG;
    const int64_t cap = (int64_t)max_blocks_per_seq * block_size;
    for (int32_t s = 0; s < num_seqs; ++s)
        if (context_lens[s] < 1 || context_lens[s] > cap) return PKV_ERR_INVALID_ARG;
    std::vector<int32_t> idx, len;
    try {
        idx.resize((size_t)num_seqs);
        len.resize((size_t)num_seqs);
    } catch (...) {  // no C++ exception leaves a C call
        return PKV_ERR_HOST_MEMORY;
    }
    auto row = [&](int32_t s) { return block_tables + (int64_t)s * max_blocks_per_seq; };
    for (int32_t s = 0; s < num_seqs; ++s) len[s] = valid_entries(row(s), (context_lens[s] - 1) / block_size);
    std::iota(idx.begin(), idx.end(), 0);
    std::stable_sort(idx.begin(), idx.end(), [&](int32_t a, int32_t b) {
        const int32_t n = std::min(len[a], len[b]);
        const int32_t k = common_entries(row(a), row(b), n);
        return k < n ? row(a)[k] < row(b)[k] : len[a] < len[b];  // a row that is a prefix of the other first
    });
    for (int32_t i = 0; i < num_seqs; ++i) order_out[i] = idx[i];
    return PKV_OK;
}
