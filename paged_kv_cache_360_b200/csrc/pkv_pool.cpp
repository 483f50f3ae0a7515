// pkv_pool.cpp -- host block manager of the paged KV cache.
//
// Data structures of the "PagedAttention" ops page (Concept -- What it is; How it
// works -- The mechanics) and the KV-cache lesson's analogy table: one pool of
// fixed-size blocks, a free stack, a block table and length per sequence, and a
// reference count per block.  Blocks are handed out one at a time when a
// sequence's last block is full, go back to the free stack when their count
// drops to zero, and a block that other sequences share is copied before a
// sequence writes into it.  The tie-breaks (LIFO free stack seeded by a
// caller-given order, logical-order release, ids counting up, all-or-nothing
// requests) are stated in pkv.h.
#include <cstdint>
#include <map>
#include <new>
#include <unordered_set>
#include <utility>
#include <vector>

#include "pkv.h"
#include "pkv_internal.h"

struct pkv_pool {
    int32_t num_blocks = 0;
    int32_t block_size = 0;
    std::vector<int32_t> free_stack;  // back() is the top
    std::vector<int32_t> refcount;
    struct Seq {
        bool live = false;
        bool swapped = false;       // preempted: blocks given back, length kept
        bool tokens_known = false;  // `tokens` holds every token id of the sequence
        int64_t len = 0;
        std::vector<int32_t> blocks;
        std::vector<int32_t> tokens;
    };
    std::vector<Seq> seqs;  // index = sequence id

    // Prefix cache: a full block is named by (previous block or -1, its token
    // ids).  An entry lives while its block is in use.
    using Key = std::pair<int32_t, std::vector<int32_t>>;
    std::map<Key, int32_t> cache;
    std::vector<char> registered;            // per block
    std::vector<Key> key_of;                 // per block, valid when registered
    std::vector<std::vector<Key>> children;  // per block: names registered below it, in order

    // Drop a block's entry and, depth first, every entry chained below it.
    void drop(int32_t b) {
        if (!registered[b]) return;
        registered[b] = 0;
        const Key key = key_of[b];
        cache.erase(key);
        if (key.first >= 0) {
            auto& sib = children[key.first];
            for (size_t i = 0; i < sib.size(); ++i)
                if (sib[i] == key) {
                    sib.erase(sib.begin() + static_cast<std::ptrdiff_t>(i));
                    break;
                }
        }
        std::vector<Key> below = std::move(children[b]);
        children[b].clear();
        for (const Key& k : below) {
            auto it = cache.find(k);
            if (it != cache.end()) drop(it->second);
        }
    }

    // Register logical block i of `s` (full, token ids known) unless its block is
    // already named, its predecessor is not registered, or the name is taken.
    void register_block(const Seq& s, int64_t i) {
        const int32_t b = s.blocks[i];
        if (registered[b]) return;
        const int32_t prev = i == 0 ? -1 : s.blocks[i - 1];
        if (i > 0 && !registered[prev]) return;
        Key key(prev, std::vector<int32_t>(s.tokens.begin() + i * block_size,
                                           s.tokens.begin() + (i + 1) * block_size));
        if (cache.count(key)) return;
        cache.emplace(key, b);
        registered[b] = 1;
        key_of[b] = key;
        if (prev >= 0) children[prev].push_back(std::move(key));
    }

    Seq* find(int32_t id) {
        if (id < 0 || id >= static_cast<int32_t>(seqs.size()) || !seqs[id].live) return nullptr;
        return &seqs[id];
    }
    const Seq* find(int32_t id) const {
        if (id < 0 || id >= static_cast<int32_t>(seqs.size()) || !seqs[id].live) return nullptr;
        return &seqs[id];
    }
    int32_t pop() {
        int32_t b = free_stack.back();
        free_stack.pop_back();
        refcount[b] = 1;
        return b;
    }
    Seq* resident(int32_t id) {
        Seq* s = find(id);
        return (s && !s->swapped) ? s : nullptr;
    }
    // refcount - 1; at 0 the block leaves the cache and goes on the free stack
    void decrement(int32_t b) {
        if (--refcount[b] == 0) {
            drop(b);
            free_stack.push_back(b);
        }
    }
    // decrement every block, logical order
    void release(const std::vector<int32_t>& blocks) {
        for (int32_t b : blocks) decrement(b);
    }
};

using pkv::fail;

extern "C" pkv_status pkv_pool_create(int32_t num_blocks, int32_t block_size,
                                      const int32_t* free_order, pkv_pool** out) {
    if (!out) return fail(PKV_ERR_INVALID_ARG, "pkv_pool_create: out is NULL");
    *out = nullptr;
    if (num_blocks <= 0 || block_size <= 0)
        return fail(PKV_ERR_INVALID_ARG, "pkv_pool_create: num_blocks and block_size must be > 0");
    pkv_pool* p = new (std::nothrow) pkv_pool();
    if (!p) return fail(PKV_ERR_INVALID_ARG, "pkv_pool_create: out of host memory");
    p->num_blocks = num_blocks;
    p->block_size = block_size;
    p->refcount.assign(num_blocks, 0);
    p->registered.assign(num_blocks, 0);
    p->key_of.resize(num_blocks);
    p->children.resize(num_blocks);
    p->free_stack.resize(num_blocks);
    if (free_order) {
        std::vector<char> seen(num_blocks, 0);
        for (int32_t i = 0; i < num_blocks; ++i) {
            int32_t b = free_order[i];
            if (b < 0 || b >= num_blocks || seen[b]) {
                delete p;
                return fail(PKV_ERR_INVALID_ARG,
                            "pkv_pool_create: free_order is not a permutation of the block ids");
            }
            seen[b] = 1;
        }
    }
    // free_order[0] ends on top of the stack.
    for (int32_t i = 0; i < num_blocks; ++i)
        p->free_stack[num_blocks - 1 - i] = free_order ? free_order[i] : i;
    *out = p;
    return PKV_OK;
}

extern "C" void pkv_pool_destroy(pkv_pool* pool) { delete pool; }

extern "C" pkv_status pkv_seq_new(pkv_pool* pool, int32_t* seq_id) {
    if (!pool || !seq_id) return fail(PKV_ERR_INVALID_ARG, "pkv_seq_new: NULL argument");
    pool->seqs.emplace_back();
    pool->seqs.back().live = true;
    *seq_id = static_cast<int32_t>(pool->seqs.size() - 1);
    return PKV_OK;
}

extern "C" pkv_status pkv_seq_fork(pkv_pool* pool, int32_t parent, int32_t* child) {
    if (!pool || !child) return fail(PKV_ERR_INVALID_ARG, "pkv_seq_fork: NULL argument");
    if (!pool->resident(parent))
        return fail(PKV_ERR_INVALID_ARG, "pkv_seq_fork: unknown or swapped-out parent");
    pkv_pool::Seq copy = *pool->find(parent);
    for (int32_t b : copy.blocks) pool->refcount[b] += 1;
    pool->seqs.push_back(std::move(copy));
    *child = static_cast<int32_t>(pool->seqs.size() - 1);
    return PKV_OK;
}

namespace {

// Whether writing n_tokens more tokens to s must first copy its last block: the
// first token lands in a partly filled block that other sequences share.
bool needs_copy(const pkv_pool* pool, const pkv_pool::Seq* s, int32_t n_tokens) {
    const int64_t bs = pool->block_size;
    return n_tokens > 0 && s->len % bs != 0 && pool->refcount[s->blocks[s->len / bs]] > 1;
}

pkv_status reserve_impl(pkv_pool* pool, pkv_pool::Seq* s, int32_t n_tokens, int64_t* slots_out,
                        int32_t* cow_pair_out, int32_t* n_cow_out) {
    const int64_t bs = pool->block_size;
    if (n_cow_out) *n_cow_out = 0;
    // Blocks needed: one per block boundary crossed, plus a copy if the first
    // token lands in a shared, partly filled block.
    const int64_t have = (s->len + bs - 1) / bs;
    const int64_t want = (s->len + n_tokens + bs - 1) / bs;
    int64_t need = want - have;
    const bool cow = needs_copy(pool, s, n_tokens);
    if (cow) {
        need += 1;
        if (!cow_pair_out || !n_cow_out)
            return fail(PKV_ERR_INVALID_ARG,
                        "pkv_seq_reserve: the write needs a copy but cow_pair_out is NULL");
    }
    if (need > static_cast<int64_t>(pool->free_stack.size()))
        return fail(PKV_ERR_NO_FREE_BLOCK, "pkv_seq_reserve: free pool exhausted");
    if (cow) {
        const int64_t i = s->len / bs;
        const int32_t src = s->blocks[i];
        const int32_t dst = pool->pop();
        pool->decrement(src);
        s->blocks[i] = dst;
        cow_pair_out[0] = src;
        cow_pair_out[1] = dst;
        *n_cow_out = 1;
    }
    for (int32_t k = 0; k < n_tokens; ++k) {
        const int64_t pos = s->len;
        if (pos % bs == 0) s->blocks.push_back(pool->pop());
        slots_out[k] = static_cast<int64_t>(s->blocks[pos / bs]) * bs + pos % bs;
        s->len = pos + 1;
    }
    return PKV_OK;
}

}  // namespace

extern "C" pkv_status pkv_seq_reserve(pkv_pool* pool, int32_t seq, int32_t n_tokens,
                                      int64_t* slots_out, int32_t* cow_pair_out,
                                      int32_t* n_cow_out) {
    if (!pool || n_tokens < 0 || (n_tokens > 0 && !slots_out))
        return fail(PKV_ERR_INVALID_ARG, "pkv_seq_reserve: bad argument");
    pkv_pool::Seq* s = pool->resident(seq);
    if (!s) return fail(PKV_ERR_INVALID_ARG, "pkv_seq_reserve: unknown or swapped-out sequence");
    const pkv_status st = reserve_impl(pool, s, n_tokens, slots_out, cow_pair_out, n_cow_out);
    if (st == PKV_OK && n_tokens > 0) {  // the token ids are unknown from here on
        s->tokens_known = false;
        s->tokens.clear();
    }
    return st;
}

extern "C" pkv_status pkv_pool_reserve_batch(pkv_pool* pool, const int32_t* seqs, int32_t n_seqs,
                                             const int32_t* n_tokens, int64_t* slots_out,
                                             int32_t* cow_pairs_out, int32_t cow_cap,
                                             int32_t* n_cow_out, int32_t* n_done) {
    if (n_cow_out) *n_cow_out = 0;
    if (n_done) *n_done = 0;
    if (!pool || n_seqs < 0 || (n_seqs > 0 && !seqs) || !n_cow_out || !n_done || cow_cap < 0 ||
        (cow_cap > 0 && !cow_pairs_out))
        return fail(PKV_ERR_INVALID_ARG, "pkv_pool_reserve_batch: bad argument");
    int64_t total = 0;
    for (int32_t i = 0; i < n_seqs; ++i) {
        const int32_t n = n_tokens ? n_tokens[i] : 1;
        if (n < 0) return fail(PKV_ERR_INVALID_ARG, "pkv_pool_reserve_batch: negative token count");
        total += n;
    }
    if (total > 0 && !slots_out) return fail(PKV_ERR_INVALID_ARG, "pkv_pool_reserve_batch: slots_out is NULL");
    // Sequence by sequence, exactly as pkv_seq_reserve; the first failure stops
    // the batch with the sequences before it served.
    int64_t off = 0;
    int32_t ncow = 0;
    for (int32_t i = 0; i < n_seqs; ++i) {
        const int32_t n = n_tokens ? n_tokens[i] : 1;
        pkv_pool::Seq* s = pool->resident(seqs[i]);
        if (!s)
            return fail(PKV_ERR_INVALID_ARG, "pkv_pool_reserve_batch: unknown or swapped-out sequence");
        if (ncow == cow_cap && needs_copy(pool, s, n))
            return fail(PKV_ERR_INVALID_ARG, "pkv_pool_reserve_batch: more copies than cow_cap");
        int32_t c = 0;
        const pkv_status st = reserve_impl(pool, s, n, slots_out + off,
                                           ncow < cow_cap ? cow_pairs_out + 2 * ncow : nullptr, &c);
        if (st != PKV_OK) return st;
        if (n > 0) {  // the token ids are unknown from here on
            s->tokens_known = false;
            s->tokens.clear();
        }
        off += n;
        ncow += c;
        *n_cow_out = ncow;
        *n_done = i + 1;
    }
    return PKV_OK;
}

extern "C" pkv_status pkv_seq_reserve_tokens(pkv_pool* pool, int32_t seq, const int32_t* tokens,
                                             int32_t n_tokens, int64_t* slots_out,
                                             int32_t* cow_pair_out, int32_t* n_cow_out) {
    if (!pool || n_tokens < 0 || (n_tokens > 0 && (!slots_out || !tokens)))
        return fail(PKV_ERR_INVALID_ARG, "pkv_seq_reserve_tokens: bad argument");
    pkv_pool::Seq* s = pool->resident(seq);
    if (!s) return fail(PKV_ERR_INVALID_ARG, "pkv_seq_reserve_tokens: unknown or swapped-out sequence");
    const bool known = s->tokens_known || s->len == 0;
    const pkv_status st = reserve_impl(pool, s, n_tokens, slots_out, cow_pair_out, n_cow_out);
    if (st != PKV_OK || !known) return st;
    s->tokens_known = true;
    const int64_t start = static_cast<int64_t>(s->tokens.size());
    s->tokens.insert(s->tokens.end(), tokens, tokens + n_tokens);
    const int64_t bs = pool->block_size;
    for (int64_t i = start / bs; i < s->len / bs; ++i)
        if ((i + 1) * bs > start) pool->register_block(*s, i);
    return PKV_OK;
}

extern "C" pkv_status pkv_seq_new_cached(pkv_pool* pool, const int32_t* prompt, int32_t n,
                                         int32_t* seq_id, int32_t* n_cached) {
    if (!pool || !seq_id || !n_cached || n < 0 || (n > 0 && !prompt))
        return fail(PKV_ERR_INVALID_ARG, "pkv_seq_new_cached: bad argument");
    pool->seqs.emplace_back();
    pkv_pool::Seq& s = pool->seqs.back();
    s.live = true;
    s.tokens_known = true;
    const int32_t bs = pool->block_size;
    int32_t prev = -1;
    for (int32_t i = 0; i < n / bs; ++i) {
        pkv_pool::Key key(prev, std::vector<int32_t>(prompt + i * bs, prompt + (i + 1) * bs));
        auto it = pool->cache.find(key);
        if (it == pool->cache.end()) break;
        const int32_t b = it->second;
        pool->refcount[b] += 1;
        s.blocks.push_back(b);
        s.tokens.insert(s.tokens.end(), key.second.begin(), key.second.end());
        prev = b;
    }
    s.len = static_cast<int64_t>(s.blocks.size()) * bs;
    *seq_id = static_cast<int32_t>(pool->seqs.size() - 1);
    *n_cached = static_cast<int32_t>(s.len);
    return PKV_OK;
}

extern "C" pkv_status pkv_seq_cow(pkv_pool* pool, int32_t seq, int32_t logical_block,
                                  int32_t* pair_out, int32_t* n_out) {
    if (!pool || !pair_out || !n_out) return fail(PKV_ERR_INVALID_ARG, "pkv_seq_cow: NULL argument");
    pkv_pool::Seq* s = pool->resident(seq);
    if (!s) return fail(PKV_ERR_INVALID_ARG, "pkv_seq_cow: unknown or swapped-out sequence");
    if (logical_block < 0 || logical_block >= static_cast<int32_t>(s->blocks.size()))
        return fail(PKV_ERR_INVALID_ARG, "pkv_seq_cow: logical block out of range");
    *n_out = 0;
    const int32_t src = s->blocks[logical_block];
    if (pool->refcount[src] <= 1) return PKV_OK;
    if (pool->free_stack.empty())
        return fail(PKV_ERR_NO_FREE_BLOCK, "pkv_seq_cow: free pool exhausted");
    const int32_t dst = pool->pop();
    pool->decrement(src);
    s->blocks[logical_block] = dst;  // the copy is not registered
    pair_out[0] = src;
    pair_out[1] = dst;
    *n_out = 1;
    return PKV_OK;
}

extern "C" pkv_status pkv_seq_free(pkv_pool* pool, int32_t seq) {
    if (!pool) return fail(PKV_ERR_INVALID_ARG, "pkv_seq_free: NULL pool");
    pkv_pool::Seq* s = pool->find(seq);
    if (!s) return fail(PKV_ERR_INVALID_ARG, "pkv_seq_free: unknown sequence");
    pool->release(s->blocks);
    s->blocks.clear();
    s->blocks.shrink_to_fit();
    s->tokens.clear();
    s->tokens.shrink_to_fit();
    s->len = 0;
    s->live = false;
    s->swapped = false;
    s->tokens_known = false;
    return PKV_OK;
}

extern "C" pkv_status pkv_seq_swap_out(pkv_pool* pool, int32_t seq, int32_t* blocks_out, int32_t cap,
                                       int32_t* n) {
    if (!pool || !n) return fail(PKV_ERR_INVALID_ARG, "pkv_seq_swap_out: NULL argument");
    pkv_pool::Seq* s = pool->resident(seq);
    if (!s) return fail(PKV_ERR_INVALID_ARG, "pkv_seq_swap_out: unknown or swapped-out sequence");
    const int32_t nb = static_cast<int32_t>(s->blocks.size());
    if (cap < nb || (nb > 0 && !blocks_out))
        return fail(PKV_ERR_INVALID_ARG, "pkv_seq_swap_out: blocks_out holds fewer than the sequence's blocks");
    for (int32_t i = 0; i < nb; ++i) blocks_out[i] = s->blocks[i];
    *n = nb;
    pool->release(s->blocks);
    s->blocks.clear();
    s->swapped = true;
    return PKV_OK;
}

extern "C" pkv_status pkv_seq_swap_in(pkv_pool* pool, int32_t seq, int32_t* blocks_out, int32_t cap,
                                      int32_t* n) {
    if (!pool || !n) return fail(PKV_ERR_INVALID_ARG, "pkv_seq_swap_in: NULL argument");
    pkv_pool::Seq* s = pool->find(seq);
    if (!s || !s->swapped) return fail(PKV_ERR_INVALID_ARG, "pkv_seq_swap_in: sequence is not swapped out");
    const int64_t need = (s->len + pool->block_size - 1) / pool->block_size;
    if (cap < need || (need > 0 && !blocks_out))
        return fail(PKV_ERR_INVALID_ARG, "pkv_seq_swap_in: blocks_out holds fewer than the blocks needed");
    if (need > static_cast<int64_t>(pool->free_stack.size()))
        return fail(PKV_ERR_NO_FREE_BLOCK, "pkv_seq_swap_in: free pool exhausted");
    for (int64_t i = 0; i < need; ++i) s->blocks.push_back(pool->pop());
    for (int64_t i = 0; i < need; ++i) blocks_out[i] = s->blocks[i];
    *n = static_cast<int32_t>(need);
    s->swapped = false;
    return PKV_OK;
}

extern "C" pkv_status pkv_seq_len(const pkv_pool* pool, int32_t seq, int64_t* len) {
    if (!pool || !len) return fail(PKV_ERR_INVALID_ARG, "pkv_seq_len: NULL argument");
    const pkv_pool::Seq* s = pool->find(seq);
    if (!s) return fail(PKV_ERR_INVALID_ARG, "pkv_seq_len: unknown sequence");
    *len = s->len;
    return PKV_OK;
}

extern "C" pkv_status pkv_seq_block_table(const pkv_pool* pool, int32_t seq, int32_t* row,
                                          int32_t cap, int32_t* n) {
    if (!pool || !n || (cap > 0 && !row))
        return fail(PKV_ERR_INVALID_ARG, "pkv_seq_block_table: bad argument");
    const pkv_pool::Seq* s = pool->find(seq);
    if (!s) return fail(PKV_ERR_INVALID_ARG, "pkv_seq_block_table: unknown sequence");
    *n = static_cast<int32_t>(s->blocks.size());
    for (int32_t i = 0; i < *n && i < cap; ++i) row[i] = s->blocks[i];
    return PKV_OK;
}

extern "C" pkv_status pkv_pool_block_tables(const pkv_pool* pool, const int32_t* seqs,
                                            int32_t n_seqs, int32_t* tables,
                                            int32_t max_blocks_per_seq, int32_t* context_lens,
                                            int32_t pad) {
    if (!pool || n_seqs < 0 || max_blocks_per_seq <= 0 ||
        (n_seqs > 0 && (!seqs || !tables || !context_lens)))
        return fail(PKV_ERR_INVALID_ARG, "pkv_pool_block_tables: bad argument");
    for (int32_t i = 0; i < n_seqs; ++i) {
        const pkv_pool::Seq* s = pool->find(seqs[i]);
        if (!s || s->swapped)
            return fail(PKV_ERR_INVALID_ARG, "pkv_pool_block_tables: unknown or swapped-out sequence");
        if (static_cast<int64_t>(s->blocks.size()) > max_blocks_per_seq)
            return fail(PKV_ERR_INVALID_ARG,
                        "pkv_pool_block_tables: a sequence has more blocks than max_blocks_per_seq");
        if (s->len > INT32_MAX) return fail(PKV_ERR_INVALID_ARG, "pkv_pool_block_tables: length overflow");
    }
    for (int32_t i = 0; i < n_seqs; ++i) {
        const pkv_pool::Seq* s = pool->find(seqs[i]);
        int32_t* row = tables + static_cast<int64_t>(i) * max_blocks_per_seq;
        const int32_t nb = static_cast<int32_t>(s->blocks.size());
        for (int32_t j = 0; j < max_blocks_per_seq; ++j) row[j] = j < nb ? s->blocks[j] : pad;
        context_lens[i] = static_cast<int32_t>(s->len);
    }
    return PKV_OK;
}

extern "C" pkv_status pkv_pool_refcount(const pkv_pool* pool, int32_t block, int32_t* refcount) {
    if (!pool || !refcount || block < 0 || block >= pool->num_blocks)
        return fail(PKV_ERR_INVALID_ARG, "pkv_pool_refcount: bad argument");
    *refcount = pool->refcount[block];
    return PKV_OK;
}

extern "C" pkv_status pkv_pool_free_list(const pkv_pool* pool, int32_t* out, int32_t cap,
                                         int32_t* n) {
    if (!pool || !n || (cap > 0 && !out))
        return fail(PKV_ERR_INVALID_ARG, "pkv_pool_free_list: bad argument");
    const int32_t total = static_cast<int32_t>(pool->free_stack.size());
    *n = total;
    for (int32_t i = 0; i < total && i < cap; ++i) out[i] = pool->free_stack[total - 1 - i];
    return PKV_OK;
}

extern "C" pkv_status pkv_pool_stats(const pkv_pool* pool, pkv_stats* st) {
    if (!pool || !st) return fail(PKV_ERR_INVALID_ARG, "pkv_pool_stats: NULL argument");
    const int64_t bs = pool->block_size;
    st->free_blocks = static_cast<int64_t>(pool->free_stack.size());
    st->allocated_slots = (pool->num_blocks - st->free_blocks) * bs;
    st->live_tokens = 0;
    st->num_seqs = 0;
    st->swapped_seqs = 0;
    std::unordered_set<int64_t> live;
    for (const auto& s : pool->seqs) {
        if (!s.live) continue;
        if (s.swapped) {
            st->swapped_seqs += 1;
            continue;
        }
        st->num_seqs += 1;
        st->live_tokens += s.len;
        for (int64_t t = 0; t < s.len; ++t) live.insert(static_cast<int64_t>(s.blocks[t / bs]) * bs + t % bs);
    }
    st->live_slots = static_cast<int64_t>(live.size());
    st->shared_blocks = 0;
    for (int32_t r : pool->refcount) st->shared_blocks += r > 1;
    st->cached_blocks = static_cast<int64_t>(pool->cache.size());
    return PKV_OK;
}

// Groups for paged_attention_decode_shared_prefix from host copies of a
// batch's block tables and lengths.  Walking the batch in order, a group
// starts at sequence i and takes i + 1, i + 2, ... while the first entries
// they have in common with row i (counting only blocks that are full in every
// sequence taken so far) stay at least min_shared_blocks; it is kept when it
// holds at least min_group_seqs sequences (else the walk moves on to i + 1).
// Sequences outside every group are left out of group_start: they are decoded
// as usual.  At most max_groups groups.
extern "C" pkv_status pkv_shared_prefix_groups(const int32_t* block_tables, int32_t num_seqs,
                                               int32_t max_blocks_per_seq,
                                               const int32_t* context_lens, int32_t block_size,
                                               int32_t min_group_seqs, int32_t min_shared_blocks,
                                               int32_t max_groups, int32_t* group_start,
                                               int32_t* group_shared_blocks, int32_t* num_groups) {
    if (!num_groups || num_seqs < 0 || max_blocks_per_seq <= 0 || block_size <= 0 ||
        min_group_seqs < 1 || min_shared_blocks < 1 || max_groups < 0)
        return pkv::fail(PKV_ERR_INVALID_ARG, "pkv_shared_prefix_groups: bad sizes");
    if (num_seqs > 0 && (!block_tables || !context_lens))
        return pkv::fail(PKV_ERR_INVALID_ARG, "pkv_shared_prefix_groups: NULL tables or lengths");
    if (max_groups > 0 && (!group_start || !group_shared_blocks))
        return pkv::fail(PKV_ERR_INVALID_ARG, "pkv_shared_prefix_groups: NULL outputs");
    auto full_blocks = [&](int32_t b) {
        const int64_t f = context_lens[b] > 0 ? context_lens[b] / block_size : 0;
        return static_cast<int32_t>(f < max_blocks_per_seq ? f : max_blocks_per_seq);
    };
    int32_t n = 0;
    std::vector<int32_t> starts, ends, shared;
    int32_t i = 0;
    while (i < num_seqs && n < max_groups) {
        const int32_t* row_i = block_tables + static_cast<int64_t>(i) * max_blocks_per_seq;
        int32_t common = full_blocks(i);
        int32_t j = i + 1;
        for (; j < num_seqs; ++j) {
            const int32_t* row_j = block_tables + static_cast<int64_t>(j) * max_blocks_per_seq;
            int32_t lim = common < full_blocks(j) ? common : full_blocks(j);
            int32_t k = 0;
            while (k < lim && row_j[k] == row_i[k]) ++k;
            if (k < min_shared_blocks) break;
            common = k;
        }
        if (j - i >= min_group_seqs && common >= min_shared_blocks) {
            starts.push_back(i);
            ends.push_back(j);
            shared.push_back(common);
            ++n;
            i = j;
        } else {
            ++i;
        }
    }
    // Groups must be back to back in group_start; a gap between two groups
    // becomes a group of its own that shares nothing.
    int32_t out = 0;
    for (int32_t g = 0; g < n; ++g) {
        const bool gap = g > 0 && starts[g] != ends[g - 1];
        if (out + (gap ? 2 : 1) > max_groups) break;
        if (gap) {
            group_start[out] = ends[g - 1];
            group_shared_blocks[out] = 0;
            ++out;
        }
        group_start[out] = starts[g];
        group_shared_blocks[out] = shared[g];
        ++out;
        group_start[out] = ends[g];
    }
    *num_groups = out;
    return PKV_OK;
}
