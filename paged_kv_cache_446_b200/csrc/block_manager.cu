// Host block manager: the allocation side of the paged KV cache (host code only, no CUDA call).
//
//  * 一文搞懂vLLM：为啥它能让一张GPU扛住几十倍用户？, "PagedAttention：核心思路": the cache is a pool of
//    equal blocks; a sequence receives a block when it starts and another one whenever its last block
//    is full -- any free block will do; when it finishes, all its blocks return to the pool.
//  * blog.mckayzhao.com/?p=56, "PagedAttention：操作系统课本里翻出来的灵感": N tokens occupy
//    ceil(N / block_size) blocks; the only waste is the unused part of the last block.
//  * same page, "还不止是分页：Copy-on-Write 和内存共享": several sequences may share blocks (parallel
//    sampling, beam search) under a reference count; a sequence about to write into a shared block
//    first copies it and writes the copy, leaving the original unchanged.
//  * 一文搞懂vLLM, "PagedAttention 是怎么共享内存的", and blog.mckayzhao.com/?p=56, "进阶特性：让推理再快
//    一点" (Prefix Caching): requests beginning with the same prefix reuse its blocks; a hash of the
//    prefix finds blocks computed before.
// Free blocks form a queue threaded through two index arrays (least recently released at the
// front), so a block can also leave it from the middle when a prefix lookup reuses it. A shared block
// is never written while shared (any writer copies it first), so all sharers see the same number of
// filled slots in it. Every entry point checks everything it needs before changing state, so a
// failing call leaves the manager as it was.
#include <algorithm>
#include <climits>
#include <cstring>
#include <new>
#include <unordered_map>
#include <unordered_set>
#include <vector>

#include "internal.h"
#include "pkv.h"

struct pkv_block_manager {
    struct Seq {
        std::vector<int32_t> blocks;  // logical block i -> physical block id
        int64_t tokens = 0;
        bool tracked = false;         // token ids known (prefix-caching managers only)
        std::vector<int32_t> ids;     // token ids of a tracked sequence
        int32_t keyed = 0;            // leading full blocks entered in the prefix index
        int32_t last_entry = -1;      // index entry of the prefix those blocks end (-1: empty prefix)
    };
    // Prefix index: one entry per distinct prefix of whole blocks that is or may again be cached,
    // linked to the entry of the prefix one block shorter. An entry stays while it holds a block,
    // has children, or ends the indexed part of a live sequence (refs counts all three), so the
    // chain to a cached block survives the eviction of a block before it.
    struct Entry {
        uint64_t uid;      // never reused: identifies the prefix in its children's keys
        uint64_t key;      // index key (parent uid folded with the block's token ids)
        int32_t parent;    // entry of the prefix one block shorter, -1 for the first block
        int32_t block;     // physical block holding this prefix's last block, -1 when none
        int32_t refs;
    };
    int32_t num_blocks = 0;
    int32_t block_size = 0;
    bool caching = false;
    std::vector<int32_t> refcount;    // per physical block; 0 = free
    // Free queue: doubly linked through prev/next, head = least recently released.
    std::vector<int32_t> prev, next;
    int32_t head = -1, tail = -1;
    int64_t free_count = 0;
    std::vector<Entry> entries;
    std::vector<int32_t> entry_ids;   // entries.size() x block_size token ids
    std::vector<int32_t> free_entries;
    std::vector<int32_t> entry_of;    // per physical block: the entry it caches, -1 when none
    std::unordered_map<uint64_t, int32_t> index;
    uint64_t next_uid = 1;
    std::unordered_map<int64_t, Seq> seqs;
    int64_t copies = 0, queries = 0, hits = 0, cached = 0;
};

namespace {

using BM = pkv_block_manager;
using Seq = BM::Seq;

pkv_status bm_fail(pkv_status s, const char* msg) {
    pkv::set_last_error(msg);
    return s;
}

int64_t blocks_for(int64_t tokens, int32_t bs) { return tokens <= 0 ? 0 : (tokens + bs - 1) / bs; }

// SplitMix64 output function (Steele, Lea and Flood, "Fast splittable pseudorandom number
// generators", OOPSLA 2014): a bijective 64-bit mixer.
uint64_t mix64(uint64_t z) {
    z = (z ^ (z >> 30)) * 0xbf58476d1ce4e5b9ull;
    z = (z ^ (z >> 27)) * 0x94d049bb133111ebull;
    return z ^ (z >> 31);
}

// Index key of a block: the uid of the prefix before it (0 for none) folded with its token ids.
uint64_t entry_key(uint64_t parent_uid, const int32_t* ids, int32_t n) {
    uint64_t h = mix64(parent_uid + 0x9e3779b97f4a7c15ull);
    for (int32_t i = 0; i < n; ++i) h = mix64(h ^ (uint64_t)(uint32_t)ids[i]);
    return h;
}

// ---- free queue ------------------------------------------------------------------------------
void queue_push_back(BM* bm, int32_t b) {
    bm->prev[b] = bm->tail;
    bm->next[b] = -1;
    if (bm->tail >= 0) bm->next[bm->tail] = b;
    else bm->head = b;
    bm->tail = b;
    ++bm->free_count;
}

void queue_unlink(BM* bm, int32_t b) {
    const int32_t p = bm->prev[b], n = bm->next[b];
    if (p >= 0) bm->next[p] = n;
    else bm->head = n;
    if (n >= 0) bm->prev[n] = p;
    else bm->tail = p;
    bm->prev[b] = bm->next[b] = -1;
    --bm->free_count;
}

// ---- prefix index ------------------------------------------------------------------------------
void entry_ref(BM* bm, int32_t e) {
    if (e >= 0) ++bm->entries[e].refs;
}

// Drops one reference; an entry left with none leaves the index and releases its parent.
void entry_unref(BM* bm, int32_t e) {
    while (e >= 0 && --bm->entries[e].refs == 0) {
        BM::Entry& en = bm->entries[e];
        auto it = bm->index.find(en.key);
        if (it != bm->index.end() && it->second == e) bm->index.erase(it);
        const int32_t parent = en.parent;
        bm->free_entries.push_back(e);
        e = parent;
    }
}

// The entry for prefix `parent` + ids[0, block_size), or -1. Exact: the parent and every token id
// are compared, not only the key.
int32_t entry_find(const BM* bm, int32_t parent, const int32_t* ids) {
    const uint64_t puid = parent >= 0 ? bm->entries[parent].uid : 0;
    auto it = bm->index.find(entry_key(puid, ids, bm->block_size));
    if (it == bm->index.end()) return -1;
    const int32_t e = it->second;
    if (bm->entries[e].parent != parent) return -1;
    if (std::memcmp(&bm->entry_ids[(size_t)e * bm->block_size], ids, sizeof(int32_t) * bm->block_size) != 0) return -1;
    return e;
}

// The entry for prefix `parent` + ids, created if missing; -1 only if its key is taken by another
// prefix (a 64-bit collision: that prefix is then simply not cached).
int32_t entry_get(BM* bm, int32_t parent, const int32_t* ids) {
    const int32_t found = entry_find(bm, parent, ids);
    if (found >= 0) return found;
    const int32_t bs = bm->block_size;
    const uint64_t key = entry_key(parent >= 0 ? bm->entries[parent].uid : 0, ids, bs);
    if (bm->index.count(key)) return -1;
    int32_t e;
    if (!bm->free_entries.empty()) {
        e = bm->free_entries.back();
        bm->free_entries.pop_back();
    } else {
        e = (int32_t)bm->entries.size();
        bm->entries.push_back({});
        bm->entry_ids.resize(bm->entry_ids.size() + bs);
    }
    bm->entries[e] = BM::Entry{bm->next_uid++, key, parent, -1, 0};
    std::memcpy(&bm->entry_ids[(size_t)e * bs], ids, sizeof(int32_t) * bs);
    bm->index[key] = e;
    entry_ref(bm, parent);  // a child keeps its parent
    return e;
}

// Forgets what block b caches (it is about to hold other data).
void evict(BM* bm, int32_t b) {
    const int32_t e = bm->entry_of[b];
    if (e < 0) return;
    bm->entry_of[b] = -1;
    bm->entries[e].block = -1;
    --bm->cached;
    entry_unref(bm, e);
}

// Moves a tracked sequence's indexed prefix to entry e.
void set_last_entry(BM* bm, Seq& s, int32_t e) {
    entry_ref(bm, e);
    entry_unref(bm, s.last_entry);
    s.last_entry = e;
}

void stop_tracking(BM* bm, Seq& s) {
    if (!s.tracked) return;
    s.tracked = false;
    set_last_entry(bm, s, -1);
    s.ids.clear();
    s.ids.shrink_to_fit();
}

// ---- blocks ------------------------------------------------------------------------------------
// A fresh block from the front of the queue; a cached block taken this way is evicted.
int32_t take_block(BM* bm) {
    const int32_t b = bm->head;
    queue_unlink(bm, b);
    evict(bm, b);
    bm->refcount[b] = 1;
    return b;
}

void release_block(BM* bm, int32_t b) {
    if (--bm->refcount[b] == 0) queue_push_back(bm, b);
}

// Adds one holder to a block found in the cache (it may be free, then it leaves the queue).
void hold_cached(BM* bm, int32_t b) {
    if (bm->refcount[b] == 0) queue_unlink(bm, b);
    ++bm->refcount[b];
}

// Enters the full blocks of a tracked sequence that are not indexed yet. A block whose prefix is
// cached already in another block is not entered (the index keeps one block per prefix).
void register_full_blocks(BM* bm, Seq& s) {
    const int32_t bs = bm->block_size;
    const int32_t full = (int32_t)(s.tokens / bs);
    for (; s.keyed < full; ++s.keyed) {
        const int32_t b = s.blocks[s.keyed];
        const int32_t e = entry_get(bm, s.last_entry, s.ids.data() + (size_t)s.keyed * bs);
        if (e < 0) {
            stop_tracking(bm, s);
            return;
        }
        if (bm->entries[e].block < 0 && bm->entry_of[b] < 0) {
            bm->entries[e].block = b;
            bm->entry_of[b] = e;
            entry_ref(bm, e);
            ++bm->cached;
        }
        set_last_entry(bm, s, e);
    }
}

// True when appending to `s` writes into its partially filled last block.
bool writes_into_last(const Seq& s, int32_t bs) { return s.tokens % bs != 0; }

// Blocks an append of n tokens takes from the free queue, given the last block's current count.
int64_t append_need(const Seq& s, int64_t n, int32_t bs, int32_t last_count) {
    if (n == 0) return 0;
    const int64_t grow = blocks_for(s.tokens + n, bs) - (int64_t)s.blocks.size();
    const bool cow = writes_into_last(s, bs) && last_count > 1;
    return grow + (cow ? 1 : 0);
}

// Performs an append already known to fit. ids: the new tokens' ids, or null (tracking stops).
// cow_pair receives {src, dst} or {-1, -1}.
void do_append(BM* bm, Seq& s, int64_t n, const int32_t* ids, int32_t* cow_pair) {
    cow_pair[0] = cow_pair[1] = -1;
    if (n == 0) return;
    const int32_t bs = bm->block_size;
    if (writes_into_last(s, bs) && bm->refcount[s.blocks.back()] > 1) {
        const int32_t src = s.blocks.back();
        const int32_t dst = take_block(bm);
        release_block(bm, src);  // stays allocated: another sequence still holds it
        s.blocks.back() = dst;
        cow_pair[0] = src;
        cow_pair[1] = dst;
        ++bm->copies;
    }
    const int64_t grow = blocks_for(s.tokens + n, bs) - (int64_t)s.blocks.size();
    for (int64_t i = 0; i < grow; ++i) s.blocks.push_back(take_block(bm));
    s.tokens += n;
    if (s.tracked && ids) {
        s.ids.insert(s.ids.end(), ids, ids + n);
        register_full_blocks(bm, s);
    } else {
        stop_tracking(bm, s);
    }
}

void write_row(const Seq& s, int32_t* row, int max_blocks) {
    std::copy(s.blocks.begin(), s.blocks.end(), row);
    std::fill(row + s.blocks.size(), row + max_blocks, -1);
}

pkv_status append_impl(BM* bm, int64_t seq_id, const int32_t* ids, int64_t n, int32_t* cow_pair) {
    if (!bm || n < 0 || !cow_pair) return bm_fail(PKV_ERR_INVALID_ARG, "bad arguments");
    auto it = bm->seqs.find(seq_id);
    if (it == bm->seqs.end()) return bm_fail(PKV_ERR_INVALID_ARG, "unknown sequence");
    Seq& s = it->second;
    const int32_t last_count = s.blocks.empty() ? 0 : bm->refcount[s.blocks.back()];
    if (append_need(s, n, bm->block_size, last_count) > bm->free_count)
        return bm_fail(PKV_ERR_OUT_OF_BLOCKS, "not enough free blocks");
    do_append(bm, s, n, ids, cow_pair);
    return PKV_OK;
}

}  // namespace

extern "C" {

pkv_status pkv_bm_create_ex(int num_blocks, int block_size, int flags, pkv_block_manager** out) {
    if (!out || num_blocks < 0 || block_size < 1 || (flags & ~PKV_BM_PREFIX_CACHE))
        return bm_fail(PKV_ERR_INVALID_ARG, "bad block manager arguments");
    BM* bm = new (std::nothrow) BM();
    if (!bm) return bm_fail(PKV_ERR_INVALID_ARG, "out of host memory");
    const size_t nb = (size_t)num_blocks;
    bm->num_blocks = num_blocks;
    bm->block_size = block_size;
    bm->caching = (flags & PKV_BM_PREFIX_CACHE) != 0;
    bm->refcount.assign(nb, 0);
    bm->prev.assign(nb, -1);
    bm->next.assign(nb, -1);
    bm->entry_of.assign(nb, -1);
    for (int32_t b = 0; b < num_blocks; ++b) queue_push_back(bm, b);  // id 0 at the front
    *out = bm;
    return PKV_OK;
}

pkv_status pkv_bm_create(int num_blocks, int block_size, pkv_block_manager** out) {
    return pkv_bm_create_ex(num_blocks, block_size, 0, out);
}

void pkv_bm_destroy(pkv_block_manager* bm) { delete bm; }

pkv_status pkv_bm_add_sequence(pkv_block_manager* bm, int64_t seq_id, int64_t num_tokens) {
    if (!bm || num_tokens < 0) return bm_fail(PKV_ERR_INVALID_ARG, "bad arguments");
    if (bm->seqs.count(seq_id)) return bm_fail(PKV_ERR_INVALID_ARG, "sequence id already live");
    const int64_t need = blocks_for(num_tokens, bm->block_size);
    if (need > bm->free_count) return bm_fail(PKV_ERR_OUT_OF_BLOCKS, "not enough free blocks");
    Seq s;
    s.tokens = num_tokens;
    s.blocks.reserve((size_t)need);
    for (int64_t i = 0; i < need; ++i) s.blocks.push_back(take_block(bm));
    bm->seqs.emplace(seq_id, std::move(s));
    return PKV_OK;
}

pkv_status pkv_bm_add_cached_prefix(pkv_block_manager* bm, int64_t seq_id, const int32_t* tokens, int64_t n,
                                    int64_t* num_cached_tokens) {
    if (!bm || n < 0 || !num_cached_tokens || (n > 0 && !tokens)) return bm_fail(PKV_ERR_INVALID_ARG, "bad arguments");
    if (bm->seqs.count(seq_id)) return bm_fail(PKV_ERR_INVALID_ARG, "sequence id already live");
    const int32_t bs = bm->block_size;
    Seq s;
    s.tracked = bm->caching;
    if (bm->caching) {
        // Longest run of cached blocks, leaving at least one prompt token to compute.
        const int64_t max_hits = n > 0 ? (n - 1) / bs : 0;
        int32_t e = -1;
        for (int64_t i = 0; i < max_hits; ++i) {
            ++bm->queries;
            const int32_t c = entry_find(bm, e, tokens + i * bs);
            if (c < 0 || bm->entries[c].block < 0) break;
            hold_cached(bm, bm->entries[c].block);
            s.blocks.push_back(bm->entries[c].block);
            e = c;
            ++bm->hits;
        }
        s.tokens = (int64_t)s.blocks.size() * bs;
        s.ids.assign(tokens, tokens + s.tokens);
        s.keyed = (int32_t)s.blocks.size();
        set_last_entry(bm, s, e);
    }
    *num_cached_tokens = s.tokens;
    bm->seqs.emplace(seq_id, std::move(s));
    return PKV_OK;
}

pkv_status pkv_bm_fork(pkv_block_manager* bm, int64_t parent, int64_t child) {
    if (!bm) return bm_fail(PKV_ERR_INVALID_ARG, "null manager");
    auto it = bm->seqs.find(parent);
    if (it == bm->seqs.end()) return bm_fail(PKV_ERR_INVALID_ARG, "unknown parent sequence");
    if (bm->seqs.count(child)) return bm_fail(PKV_ERR_INVALID_ARG, "child id already live");
    Seq s = it->second;  // the same physical blocks, now shared
    for (int32_t b : s.blocks) ++bm->refcount[b];
    entry_ref(bm, s.last_entry);
    bm->seqs.emplace(child, std::move(s));
    return PKV_OK;
}

pkv_status pkv_bm_append(pkv_block_manager* bm, int64_t seq_id, int64_t num_new_tokens, int32_t* cow_pair) {
    return append_impl(bm, seq_id, nullptr, num_new_tokens, cow_pair);
}

pkv_status pkv_bm_append_tokens(pkv_block_manager* bm, int64_t seq_id, const int32_t* tokens, int64_t num_new_tokens,
                                int32_t* cow_pair) {
    if (num_new_tokens > 0 && !tokens) return bm_fail(PKV_ERR_INVALID_ARG, "null token ids");
    return append_impl(bm, seq_id, tokens, num_new_tokens, cow_pair);
}

pkv_status pkv_bm_free(pkv_block_manager* bm, int64_t seq_id) {
    if (!bm) return bm_fail(PKV_ERR_INVALID_ARG, "null manager");
    auto it = bm->seqs.find(seq_id);
    if (it == bm->seqs.end()) return bm_fail(PKV_ERR_INVALID_ARG, "unknown sequence");
    const auto& b = it->second.blocks;
    for (auto p = b.rbegin(); p != b.rend(); ++p) release_block(bm, *p);  // last to first
    entry_unref(bm, it->second.last_entry);
    bm->seqs.erase(it);
    return PKV_OK;
}

pkv_status pkv_bm_sequence(const pkv_block_manager* bm, int64_t seq_id, int64_t* num_tokens, int32_t* blocks,
                           int capacity, int* num_blocks) {
    if (!bm || !num_tokens || !num_blocks) return bm_fail(PKV_ERR_INVALID_ARG, "null argument");
    auto it = bm->seqs.find(seq_id);
    if (it == bm->seqs.end()) return bm_fail(PKV_ERR_INVALID_ARG, "unknown sequence");
    const Seq& s = it->second;
    if (blocks && capacity < (int64_t)s.blocks.size()) return bm_fail(PKV_ERR_INVALID_ARG, "block array too small");
    *num_tokens = s.tokens;
    *num_blocks = (int)s.blocks.size();
    if (blocks) std::copy(s.blocks.begin(), s.blocks.end(), blocks);
    return PKV_OK;
}

pkv_status pkv_bm_block_tables(const pkv_block_manager* bm, const int64_t* seq_ids, int num_seqs, int32_t* tables,
                               int max_blocks_per_seq) {
    if (!bm || num_seqs < 0 || max_blocks_per_seq < 0 || (num_seqs > 0 && (!seq_ids || !tables)))
        return bm_fail(PKV_ERR_INVALID_ARG, "bad arguments");
    std::vector<const Seq*> rows((size_t)num_seqs);
    for (int r = 0; r < num_seqs; ++r) {
        auto it = bm->seqs.find(seq_ids[r]);
        if (it == bm->seqs.end()) return bm_fail(PKV_ERR_INVALID_ARG, "unknown sequence");
        if ((int64_t)it->second.blocks.size() > max_blocks_per_seq)
            return bm_fail(PKV_ERR_INVALID_ARG, "table row too short");
        rows[r] = &it->second;
    }
    for (int r = 0; r < num_seqs; ++r) write_row(*rows[r], tables + (size_t)r * max_blocks_per_seq, max_blocks_per_seq);
    return PKV_OK;
}

pkv_status pkv_bm_refcount(const pkv_block_manager* bm, int32_t block, int32_t* count) {
    if (!bm || !count || block < 0 || block >= bm->num_blocks) return bm_fail(PKV_ERR_INVALID_ARG, "bad block id");
    *count = bm->refcount[block];
    return PKV_OK;
}

pkv_status pkv_bm_stats(const pkv_block_manager* bm, pkv_pool_stats* st) {
    if (!bm || !st) return bm_fail(PKV_ERR_INVALID_ARG, "null argument");
    std::memset(st, 0, sizeof *st);
    const int32_t bs = bm->block_size;
    st->num_blocks = bm->num_blocks;
    st->free_blocks = bm->free_count;
    st->used_blocks = st->num_blocks - st->free_blocks;
    st->num_sequences = (int64_t)bm->seqs.size();
    st->cow_copies = bm->copies;
    st->cache_queries = bm->queries;
    st->cache_hits = bm->hits;
    st->cached_blocks = bm->cached;
    for (int32_t c : bm->refcount)
        if (c > 1) ++st->shared_blocks;
    // Filled slots per used block: every block but a sequence's last is full; sharers agree on the
    // fill of a shared block, so taking the maximum over holders counts each block once.
    std::vector<int32_t> fill((size_t)bm->num_blocks, 0);
    for (const auto& kv : bm->seqs) {
        const Seq& s = kv.second;
        st->logical_tokens += s.tokens;
        const size_t nb = s.blocks.size();
        for (size_t i = 0; i < nb; ++i) {
            const int32_t f = i + 1 < nb ? bs : (int32_t)(s.tokens - (int64_t)(nb - 1) * bs);
            fill[s.blocks[i]] = std::max(fill[s.blocks[i]], f);
        }
    }
    for (int32_t f : fill) st->stored_tokens += f;
    st->wasted_slots = st->used_blocks * bs - st->stored_tokens;
    return PKV_OK;
}

pkv_status pkv_bm_step(pkv_block_manager* bm, const int64_t* seq_ids, const int32_t* num_new_tokens, int num_seqs,
                       const int32_t* new_tokens, int32_t* block_tables, int max_blocks_per_seq,
                       int32_t* context_lens, int32_t* query_start_loc, int32_t* cow_pairs, int* num_cow_pairs) {
    if (!bm || num_seqs < 0 || max_blocks_per_seq < 0 || !query_start_loc || !num_cow_pairs ||
        (num_seqs > 0 && (!seq_ids || !num_new_tokens || !block_tables || !context_lens || !cow_pairs)))
        return bm_fail(PKV_ERR_INVALID_ARG, "bad arguments");
    const int32_t bs = bm->block_size;
    // Pass 1: resolve ids and count the blocks the whole batch takes. An append copies its last
    // block only while that block is still shared when its turn comes, so count the copies made by
    // earlier members of the batch against the shared counts as the batch proceeds.
    std::vector<Seq*> rows((size_t)num_seqs);
    std::unordered_set<int64_t> seen;
    std::unordered_map<int32_t, int32_t> released;  // block -> copies made from it so far in this batch
    int64_t need = 0, total_rows = 0;
    for (int r = 0; r < num_seqs; ++r) {
        const int64_t n = num_new_tokens[r];
        if (n < 0) return bm_fail(PKV_ERR_INVALID_ARG, "negative token count");
        if (!seen.insert(seq_ids[r]).second) return bm_fail(PKV_ERR_INVALID_ARG, "sequence repeated in the batch");
        auto it = bm->seqs.find(seq_ids[r]);
        if (it == bm->seqs.end()) return bm_fail(PKV_ERR_INVALID_ARG, "unknown sequence");
        Seq& s = it->second;
        rows[r] = &s;
        if (s.tokens + n > INT32_MAX) return bm_fail(PKV_ERR_INVALID_ARG, "sequence length over INT32_MAX");
        if (blocks_for(s.tokens + n, bs) > max_blocks_per_seq) return bm_fail(PKV_ERR_INVALID_ARG, "table row too short");
        total_rows += n;
        if (total_rows > INT32_MAX) return bm_fail(PKV_ERR_INVALID_ARG, "batch over INT32_MAX rows");
        int32_t last_count = 0;
        if (!s.blocks.empty()) {
            const int32_t last = s.blocks.back();
            auto rel = released.find(last);
            last_count = bm->refcount[last] - (rel == released.end() ? 0 : rel->second);
            if (n > 0 && writes_into_last(s, bs) && last_count > 1) ++released[last];
        }
        need += append_need(s, n, bs, last_count);
    }
    if (need > bm->free_count) return bm_fail(PKV_ERR_OUT_OF_BLOCKS, "not enough free blocks");
    // Pass 2: apply in batch order and write the step's inputs.
    int pairs = 0;
    query_start_loc[0] = 0;
    for (int r = 0; r < num_seqs; ++r) {
        Seq& s = *rows[r];
        int32_t pair[2];
        do_append(bm, s, num_new_tokens[r], new_tokens ? new_tokens + query_start_loc[r] : nullptr, pair);
        if (pair[0] >= 0) {
            cow_pairs[2 * pairs] = pair[0];
            cow_pairs[2 * pairs + 1] = pair[1];
            ++pairs;
        }
        write_row(s, block_tables + (size_t)r * max_blocks_per_seq, max_blocks_per_seq);
        context_lens[r] = (int32_t)s.tokens;
        query_start_loc[r + 1] = query_start_loc[r] + num_new_tokens[r];
    }
    *num_cow_pairs = pairs;
    return PKV_OK;
}

}  // extern "C"
