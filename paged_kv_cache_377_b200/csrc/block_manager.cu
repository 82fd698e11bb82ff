// block_manager.cu -- host-side block manager of the paged KV pool (no device code).
//
// Follows the block-table scheme of "Deep Dive into vLLM" (section 2.1:
// logical blocks, physical blocks, a block table per sequence; section 2.2:
// blocks are allocated only when data is stored, and sequences of parallel
// sampling or beam search share the blocks of their prompt, copy-on-write as
// in an OS) and of runbyai post 449 (section 3: sequences whose prompts start
// alike share those blocks; section 4: finished sequences free their blocks at
// once and new ones join). "vLLM Fundamentals" ("Just a python process"): block
// management runs on the CPU and the engine packs the block tables into
// tensors for the GPU at every step -- pkv_bm_pack below.
//
// Data: a reference count per physical block, a LIFO free list, and per
// sequence its block list and length. A block is free exactly when its count
// is 0. A pending copy-on-write copy holds one reference on its source block
// until pkv_bm_take_copies hands it out, so the source cannot be reallocated
// (and overwritten) before the copy has been issued.
#include <cstdint>
#include <cstring>
#include <mutex>
#include <unordered_map>
#include <vector>

#include "pagedkv.h"

namespace {

struct Sequence {
    std::vector<int32_t> blocks;
    int64_t len = 0;
};

}  // namespace

struct pkv_block_manager {
    int num_blocks = 0;
    int block_size = 0;
    std::vector<int32_t> refs;
    std::vector<int32_t> free_list;  // stack; back() is allocated next
    std::unordered_map<int64_t, Sequence> seqs;
    std::vector<int32_t> copy_src, copy_dst;
    mutable std::mutex mu;

    int32_t take_block() {
        const int32_t b = free_list.back();
        free_list.pop_back();
        refs[b] = 1;
        return b;
    }
    void drop(int32_t b) {
        if (--refs[b] == 0) free_list.push_back(b);
    }
};

namespace {

thread_local char g_bm_err[256];

int bm_fail(int code, const char *msg) {
    std::strncpy(g_bm_err, msg, sizeof(g_bm_err) - 1);
    g_bm_err[sizeof(g_bm_err) - 1] = 0;
    return code;
}

int64_t blocks_for(int64_t tokens, int bs) { return (tokens + bs - 1) / bs; }

}  // namespace

extern "C" {

const char *pkv_bm_last_error(void) { return g_bm_err; }

pkv_block_manager *pkv_bm_create(int num_blocks, int block_size) {
    if (num_blocks <= 0 || block_size <= 0) return nullptr;
    auto *bm = new pkv_block_manager;
    bm->num_blocks = num_blocks;
    bm->block_size = block_size;
    bm->refs.assign(num_blocks, 0);
    bm->free_list.reserve(num_blocks);
    for (int b = num_blocks - 1; b >= 0; --b) bm->free_list.push_back(b);  // block 0 is allocated first
    return bm;
}

void pkv_bm_destroy(pkv_block_manager *bm) { delete bm; }

int pkv_bm_num_free(const pkv_block_manager *bm) {
    if (!bm) return PKV_ERR_INVALID_ARGUMENT;
    std::lock_guard<std::mutex> lock(bm->mu);
    return static_cast<int>(bm->free_list.size());
}

int pkv_bm_refcount(const pkv_block_manager *bm, int block) {
    if (!bm || block < 0 || block >= bm->num_blocks) return PKV_ERR_INVALID_ARGUMENT;
    std::lock_guard<std::mutex> lock(bm->mu);
    return bm->refs[block];
}

int pkv_bm_add(pkv_block_manager *bm, int64_t seq_id, int64_t num_tokens, int64_t prefix_seq,
               int64_t prefix_tokens, int64_t *slots) {
    if (!bm || num_tokens < 0 || prefix_tokens < 0) return bm_fail(PKV_ERR_INVALID_ARGUMENT, "bad argument");
    std::lock_guard<std::mutex> lock(bm->mu);
    if (bm->seqs.count(seq_id)) return bm_fail(PKV_ERR_INVALID_ARGUMENT, "sequence id already in use");
    const int bs = bm->block_size;
    std::vector<int32_t> shared;
    if (prefix_seq >= 0) {
        auto it = bm->seqs.find(prefix_seq);
        if (it == bm->seqs.end()) return bm_fail(PKV_ERR_INVALID_ARGUMENT, "unknown prefix sequence");
        if (prefix_tokens > num_tokens || prefix_tokens > it->second.len)
            return bm_fail(PKV_ERR_INVALID_ARGUMENT, "prefix longer than either sequence");
        // whole blocks only: a partly filled block would be written by both
        shared.assign(it->second.blocks.begin(), it->second.blocks.begin() + prefix_tokens / bs);
    }
    const int64_t need = blocks_for(num_tokens, bs) - static_cast<int64_t>(shared.size());
    if (need > static_cast<int64_t>(bm->free_list.size())) return bm_fail(PKV_ERR_OUT_OF_BLOCKS, "out of blocks");
    Sequence s;
    s.len = num_tokens;
    s.blocks = shared;
    for (int32_t b : shared) ++bm->refs[b];
    for (int64_t i = 0; i < need; ++i) s.blocks.push_back(bm->take_block());
    if (slots)
        for (int64_t t = 0; t < num_tokens; ++t)
            slots[t] = t / bs < static_cast<int64_t>(shared.size())
                           ? -1
                           : static_cast<int64_t>(s.blocks[t / bs]) * bs + t % bs;
    bm->seqs.emplace(seq_id, std::move(s));
    return PKV_OK;
}

int pkv_bm_fork(pkv_block_manager *bm, int64_t parent, int64_t child) {
    if (!bm) return bm_fail(PKV_ERR_INVALID_ARGUMENT, "bad argument");
    std::lock_guard<std::mutex> lock(bm->mu);
    auto it = bm->seqs.find(parent);
    if (it == bm->seqs.end()) return bm_fail(PKV_ERR_INVALID_ARGUMENT, "unknown parent sequence");
    if (bm->seqs.count(child)) return bm_fail(PKV_ERR_INVALID_ARGUMENT, "sequence id already in use");
    if (!bm->copy_src.empty())
        return bm_fail(PKV_ERR_INVALID_ARGUMENT, "copies are pending: fork between steps, after pkv_bm_take_copies");
    Sequence s = it->second;
    for (int32_t b : s.blocks) ++bm->refs[b];
    bm->seqs.emplace(child, std::move(s));
    return PKV_OK;
}

int pkv_bm_append(pkv_block_manager *bm, int64_t seq_id, int64_t *slot) {
    if (!bm || !slot) return bm_fail(PKV_ERR_INVALID_ARGUMENT, "bad argument");
    std::lock_guard<std::mutex> lock(bm->mu);
    auto it = bm->seqs.find(seq_id);
    if (it == bm->seqs.end()) return bm_fail(PKV_ERR_INVALID_ARGUMENT, "unknown sequence");
    Sequence &s = it->second;
    const int bs = bm->block_size;
    const int64_t pos = s.len;
    if (pos % bs == 0) {  // the last block is full (or there is none): a fresh block
        if (bm->free_list.empty()) return bm_fail(PKV_ERR_OUT_OF_BLOCKS, "out of blocks");
        s.blocks.push_back(bm->take_block());
    } else {
        const int32_t last = s.blocks.back();
        if (bm->refs[last] > 1) {  // shared and not full: copy it first (copy-on-write)
            if (bm->free_list.empty()) return bm_fail(PKV_ERR_OUT_OF_BLOCKS, "out of blocks");
            const int32_t fresh = bm->take_block();
            bm->copy_src.push_back(last);  // the copy keeps this sequence's reference until taken
            bm->copy_dst.push_back(fresh);
            s.blocks.back() = fresh;
        }
    }
    s.len = pos + 1;
    *slot = static_cast<int64_t>(s.blocks.back()) * bs + pos % bs;
    return PKV_OK;
}

int pkv_bm_free(pkv_block_manager *bm, int64_t seq_id) {
    if (!bm) return bm_fail(PKV_ERR_INVALID_ARGUMENT, "bad argument");
    std::lock_guard<std::mutex> lock(bm->mu);
    auto it = bm->seqs.find(seq_id);
    if (it == bm->seqs.end()) return bm_fail(PKV_ERR_INVALID_ARGUMENT, "unknown sequence");
    for (int32_t b : it->second.blocks) bm->drop(b);
    bm->seqs.erase(it);
    return PKV_OK;
}

int pkv_bm_take_copies(pkv_block_manager *bm, int32_t *src, int32_t *dst, int capacity) {
    if (!bm || capacity < 0 || (capacity > 0 && (!src || !dst))) return bm_fail(PKV_ERR_INVALID_ARGUMENT, "bad argument");
    std::lock_guard<std::mutex> lock(bm->mu);
    const int n = static_cast<int>(bm->copy_src.size());
    if (n > capacity) return bm_fail(PKV_ERR_INVALID_ARGUMENT, "capacity below the pending copies");
    for (int i = 0; i < n; ++i) {
        src[i] = bm->copy_src[i];
        dst[i] = bm->copy_dst[i];
        bm->drop(bm->copy_src[i]);  // the caller issues the copy before any later write of the pool
    }
    bm->copy_src.clear();
    bm->copy_dst.clear();
    return n;
}

int pkv_bm_pending_copies(const pkv_block_manager *bm) {
    if (!bm) return PKV_ERR_INVALID_ARGUMENT;
    std::lock_guard<std::mutex> lock(bm->mu);
    return static_cast<int>(bm->copy_src.size());
}

int pkv_bm_seq_len(const pkv_block_manager *bm, int64_t seq_id, int64_t *len) {
    if (!bm || !len) return bm_fail(PKV_ERR_INVALID_ARGUMENT, "bad argument");
    std::lock_guard<std::mutex> lock(bm->mu);
    auto it = bm->seqs.find(seq_id);
    if (it == bm->seqs.end()) return bm_fail(PKV_ERR_INVALID_ARGUMENT, "unknown sequence");
    *len = it->second.len;
    return PKV_OK;
}

int pkv_bm_pack(const pkv_block_manager *bm, const int64_t *seq_ids, int num_seqs, int max_blocks_per_seq,
                int32_t *block_tables, int32_t *context_lens) {
    if (!bm || num_seqs < 0 || max_blocks_per_seq <= 0 || (num_seqs > 0 && (!seq_ids || !block_tables || !context_lens)))
        return bm_fail(PKV_ERR_INVALID_ARGUMENT, "bad argument");
    std::lock_guard<std::mutex> lock(bm->mu);
    for (int i = 0; i < num_seqs; ++i) {
        auto it = bm->seqs.find(seq_ids[i]);
        if (it == bm->seqs.end()) return bm_fail(PKV_ERR_INVALID_ARGUMENT, "unknown sequence");
        if (static_cast<int64_t>(it->second.blocks.size()) > max_blocks_per_seq)
            return bm_fail(PKV_ERR_INVALID_ARGUMENT, "a sequence has more blocks than max_blocks_per_seq");
        if (it->second.len > 0x7fffffff) return bm_fail(PKV_ERR_INVALID_ARGUMENT, "sequence too long for int32");
    }
    for (int i = 0; i < num_seqs; ++i) {
        const Sequence &s = bm->seqs.find(seq_ids[i])->second;
        int32_t *row = block_tables + static_cast<int64_t>(i) * max_blocks_per_seq;
        const int nb = static_cast<int>(s.blocks.size());
        for (int j = 0; j < max_blocks_per_seq; ++j) row[j] = j < nb ? s.blocks[j] : -1;
        context_lens[i] = static_cast<int32_t>(s.len);
    }
    return PKV_OK;
}

}  // extern "C"

// ---------------------------------------------------------------------------
// Prefix groups of a packed batch (see pkv_find_prefix_groups in pagedkv.h):
// runs of consecutive sequences whose tables start with the same physical
// blocks, which the decode then reads once per group.
extern "C" int pkv_find_prefix_groups(const int32_t *block_tables, const int32_t *context_lens, int num_seqs,
                                      int max_blocks_per_seq, int block_size, int min_blocks, int32_t *begin,
                                      int32_t *end, int32_t *blocks, int max_groups, int *num_groups) {
    if (!num_groups || num_seqs < 0 || max_blocks_per_seq <= 0 || block_size <= 0 || min_blocks < 1 ||
        max_groups < 0 || (num_seqs > 0 && (!block_tables || !context_lens)) ||
        (max_groups > 0 && (!begin || !end || !blocks)))
        return bm_fail(PKV_ERR_INVALID_ARGUMENT, "bad argument");
    auto covered = [&](int s) {  // table entries the context of s uses
        const int64_t L = context_lens[s] < 0 ? 0 : context_lens[s];
        const int64_t n = (L + block_size - 1) / block_size;
        return static_cast<int>(n < max_blocks_per_seq ? n : max_blocks_per_seq);
    };
    auto row = [&](int s) { return block_tables + static_cast<int64_t>(s) * max_blocks_per_seq; };
    int n = 0, s = 0;
    while (s < num_seqs && n < max_groups) {
        int shared = covered(s), e = s + 1;
        while (e < num_seqs) {
            const int lim = shared < covered(e) ? shared : covered(e);
            int c = 0;
            while (c < lim && row(s)[c] == row(e)[c]) ++c;
            if (c < min_blocks) break;
            shared = c;
            ++e;
        }
        if (e - s >= 2) {
            begin[n] = s;
            end[n] = e;
            blocks[n] = shared;
            ++n;
            s = e;
        } else {
            ++s;
        }
    }
    *num_groups = n;
    return PKV_OK;
}
