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
// Free blocks are kept on a stack (the most recently released block is handed out first). A shared
// block is never written while shared (any writer copies it first), so all sharers see the same
// number of filled slots in it. Every entry point checks everything it needs before changing state,
// so a failing call leaves the manager as it was.
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
    };
    int32_t num_blocks = 0;
    int32_t block_size = 0;
    std::vector<int32_t> refcount;    // per physical block; 0 = free
    std::vector<int32_t> free_stack;  // free block ids; back() is handed out next
    std::unordered_map<int64_t, Seq> seqs;
    int64_t copies = 0;               // copy-on-write copies requested so far
};

namespace {

using Seq = pkv_block_manager::Seq;

pkv_status bm_fail(pkv_status s, const char* msg) {
    pkv::set_last_error(msg);
    return s;
}

int64_t blocks_for(int64_t tokens, int32_t bs) { return tokens <= 0 ? 0 : (tokens + bs - 1) / bs; }

int32_t take_block(pkv_block_manager* bm) {
    const int32_t b = bm->free_stack.back();
    bm->free_stack.pop_back();
    bm->refcount[b] = 1;
    return b;
}

void release_block(pkv_block_manager* bm, int32_t b) {
    if (--bm->refcount[b] == 0) bm->free_stack.push_back(b);
}

// True when appending to `s` writes into its partially filled last block.
bool writes_into_last(const Seq& s, int32_t bs) { return s.tokens % bs != 0; }

// Blocks an append of n tokens takes from the free stack, given the last block's current count.
int64_t append_need(const Seq& s, int64_t n, int32_t bs, int32_t last_count) {
    if (n == 0) return 0;
    const int64_t grow = blocks_for(s.tokens + n, bs) - (int64_t)s.blocks.size();
    const bool cow = writes_into_last(s, bs) && last_count > 1;
    return grow + (cow ? 1 : 0);
}

// Performs an append already known to fit. cow_pair receives {src, dst} or {-1, -1}.
void do_append(pkv_block_manager* bm, Seq& s, int64_t n, int32_t* cow_pair) {
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
}

void write_row(const Seq& s, int32_t* row, int max_blocks) {
    std::copy(s.blocks.begin(), s.blocks.end(), row);
    std::fill(row + s.blocks.size(), row + max_blocks, -1);
}

}  // namespace

extern "C" {

pkv_status pkv_bm_create(int num_blocks, int block_size, pkv_block_manager** out) {
    if (!out || num_blocks < 0 || block_size < 1) return bm_fail(PKV_ERR_INVALID_ARG, "bad block manager arguments");
    pkv_block_manager* bm = new (std::nothrow) pkv_block_manager();
    if (!bm) return bm_fail(PKV_ERR_INVALID_ARG, "out of host memory");
    bm->num_blocks = num_blocks;
    bm->block_size = block_size;
    bm->refcount.assign((size_t)num_blocks, 0);
    bm->free_stack.reserve((size_t)num_blocks);
    for (int32_t b = num_blocks - 1; b >= 0; --b) bm->free_stack.push_back(b);  // id 0 on top
    *out = bm;
    return PKV_OK;
}

void pkv_bm_destroy(pkv_block_manager* bm) { delete bm; }

pkv_status pkv_bm_add_sequence(pkv_block_manager* bm, int64_t seq_id, int64_t num_tokens) {
    if (!bm || num_tokens < 0) return bm_fail(PKV_ERR_INVALID_ARG, "bad arguments");
    if (bm->seqs.count(seq_id)) return bm_fail(PKV_ERR_INVALID_ARG, "sequence id already live");
    const int64_t need = blocks_for(num_tokens, bm->block_size);
    if (need > (int64_t)bm->free_stack.size()) return bm_fail(PKV_ERR_OUT_OF_BLOCKS, "not enough free blocks");
    Seq s;
    s.tokens = num_tokens;
    s.blocks.reserve((size_t)need);
    for (int64_t i = 0; i < need; ++i) s.blocks.push_back(take_block(bm));
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
    bm->seqs.emplace(child, std::move(s));
    return PKV_OK;
}

pkv_status pkv_bm_append(pkv_block_manager* bm, int64_t seq_id, int64_t num_new_tokens, int32_t* cow_pair) {
    if (!bm || num_new_tokens < 0 || !cow_pair) return bm_fail(PKV_ERR_INVALID_ARG, "bad arguments");
    auto it = bm->seqs.find(seq_id);
    if (it == bm->seqs.end()) return bm_fail(PKV_ERR_INVALID_ARG, "unknown sequence");
    Seq& s = it->second;
    const int32_t last_count = s.blocks.empty() ? 0 : bm->refcount[s.blocks.back()];
    if (append_need(s, num_new_tokens, bm->block_size, last_count) > (int64_t)bm->free_stack.size())
        return bm_fail(PKV_ERR_OUT_OF_BLOCKS, "not enough free blocks");
    do_append(bm, s, num_new_tokens, cow_pair);
    return PKV_OK;
}

pkv_status pkv_bm_free(pkv_block_manager* bm, int64_t seq_id) {
    if (!bm) return bm_fail(PKV_ERR_INVALID_ARG, "null manager");
    auto it = bm->seqs.find(seq_id);
    if (it == bm->seqs.end()) return bm_fail(PKV_ERR_INVALID_ARG, "unknown sequence");
    const auto& b = it->second.blocks;
    for (auto p = b.rbegin(); p != b.rend(); ++p) release_block(bm, *p);  // last to first
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
    st->free_blocks = (int64_t)bm->free_stack.size();
    st->used_blocks = st->num_blocks - st->free_blocks;
    st->num_sequences = (int64_t)bm->seqs.size();
    st->cow_copies = bm->copies;
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
                       int32_t* block_tables, int max_blocks_per_seq, int32_t* context_lens, int32_t* query_start_loc,
                       int32_t* cow_pairs, int* num_cow_pairs) {
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
    if (need > (int64_t)bm->free_stack.size()) return bm_fail(PKV_ERR_OUT_OF_BLOCKS, "not enough free blocks");
    // Pass 2: apply in batch order and write the step's inputs.
    int pairs = 0;
    query_start_loc[0] = 0;
    for (int r = 0; r < num_seqs; ++r) {
        Seq& s = *rows[r];
        int32_t pair[2];
        do_append(bm, s, num_new_tokens[r], pair);
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
