// Host block manager for the paged KV cache (C ABI in include/paged_kv.h).
//
// "KV Cache 深度解析" §三: the cache is cut into fixed 16-token blocks; a block
// table maps each sequence's logical blocks to physical ones; blocks are
// allocated on demand as a sequence grows (at most one partly used block per
// sequence) and several sequences may share a physical block (beam branches,
// common prefixes).  "大模型推理为何这么慢" (PagedAttention section): a finished
// request's blocks are released at once.  "llm-inference-optimization" notes
// §二: a sequence takes a new block when it has none or its last one is full.
//
// Sharing is by reference count.  A shared block that is full is read-only
// for everyone; when a sequence appends into a shared block that still has
// free slots, it first gets a private copy (copy-on-write): a new block is
// allocated, the caller copies the old block's contents into it on the GPU
// (paged_kv_copy_blocks), and the sequence's table points at the copy.
//
// Deterministic policies (so tests can compare with a plain restatement):
// free blocks form a LIFO stack that initially pops 0, 1, 2, ...; a sequence
// id is the lowest unused one.  Host only: no device work, no CUDA calls.
#include <algorithm>
#include <cstdint>
#include <new>
#include <vector>

#include "paged_kv.h"

struct kv_block_manager {
    int32_t block_size = 16;
    int32_t max_blocks_per_seq = 0;
    std::vector<int32_t> free_stack;   // top = back
    std::vector<int32_t> refcount;     // per physical block
    struct Seq {
        bool live = false;
        int32_t len = 0;
        std::vector<int32_t> blocks;
    };
    std::vector<Seq> seqs;

    int32_t pop_block() {
        const int32_t b = free_stack.back();
        free_stack.pop_back();
        refcount[b] = 1;
        return b;
    }
    void release(int32_t b) {
        if (--refcount[b] == 0) free_stack.push_back(b);
    }
    bool valid_seq(int32_t s) const {
        return s >= 0 && s < static_cast<int32_t>(seqs.size()) && seqs[s].live;
    }
};

namespace {
constexpr int32_t kPoisonBlock = 0x7fffffff;
}

extern "C" {

kv_status kv_block_manager_create(int32_t num_blocks, int32_t max_seqs,
                                  int32_t max_blocks_per_seq, kv_block_manager** out) {
    if (out == nullptr || num_blocks <= 0 || max_seqs <= 0 || max_blocks_per_seq <= 0)
        return KV_ERR_INVALID_ARGUMENT;
    kv_block_manager* m = new (std::nothrow) kv_block_manager();
    if (m == nullptr) return KV_ERR_OUT_OF_BLOCKS;
    m->max_blocks_per_seq = max_blocks_per_seq;
    m->refcount.assign(num_blocks, 0);
    m->free_stack.reserve(num_blocks);
    for (int32_t b = num_blocks - 1; b >= 0; --b) m->free_stack.push_back(b);
    m->seqs.resize(max_seqs);
    *out = m;
    return KV_OK;
}

void kv_block_manager_destroy(kv_block_manager* m) { delete m; }

int32_t kv_block_manager_num_free_blocks(const kv_block_manager* m) {
    return m == nullptr ? -1 : static_cast<int32_t>(m->free_stack.size());
}

kv_status kv_block_manager_add_sequence(kv_block_manager* m, int32_t* seq_id) {
    if (m == nullptr || seq_id == nullptr) return KV_ERR_INVALID_ARGUMENT;
    for (size_t s = 0; s < m->seqs.size(); ++s) {
        if (!m->seqs[s].live) {
            m->seqs[s].live = true;
            m->seqs[s].len = 0;
            m->seqs[s].blocks.clear();
            *seq_id = static_cast<int32_t>(s);
            return KV_OK;
        }
    }
    return KV_ERR_OUT_OF_BLOCKS;
}

kv_status kv_block_manager_fork(kv_block_manager* m, int32_t parent, int32_t* child) {
    if (m == nullptr || child == nullptr || !m->valid_seq(parent)) return KV_ERR_INVALID_ARGUMENT;
    int32_t c = 0;
    const kv_status st = kv_block_manager_add_sequence(m, &c);
    if (st != KV_OK) return st;
    m->seqs[c].len = m->seqs[parent].len;
    m->seqs[c].blocks = m->seqs[parent].blocks;
    for (int32_t b : m->seqs[c].blocks) ++m->refcount[b];
    *child = c;
    return KV_OK;
}

kv_status kv_block_manager_free_sequence(kv_block_manager* m, int32_t seq) {
    if (m == nullptr || !m->valid_seq(seq)) return KV_ERR_INVALID_ARGUMENT;
    // release in reverse so a sequence's blocks come back in allocation order
    auto& blocks = m->seqs[seq].blocks;
    for (auto it = blocks.rbegin(); it != blocks.rend(); ++it) m->release(*it);
    blocks.clear();
    m->seqs[seq].live = false;
    m->seqs[seq].len = 0;
    return KV_OK;
}

kv_status kv_block_manager_append_slots(kv_block_manager* m, const int32_t* seq_ids,
                                        int32_t num_tokens, int64_t* slots,
                                        int32_t* copy_src, int32_t* copy_dst,
                                        int32_t* num_copies) {
    if (m == nullptr || num_tokens < 0 || num_copies == nullptr) return KV_ERR_INVALID_ARGUMENT;
    if (num_tokens > 0 && (seq_ids == nullptr || slots == nullptr || copy_src == nullptr ||
                           copy_dst == nullptr))
        return KV_ERR_INVALID_ARGUMENT;
    const int32_t bs = m->block_size;
    // dry run: validate and count the blocks this batch needs, so a batch that
    // cannot be served changes nothing
    std::vector<int32_t> len(m->seqs.size());
    std::vector<char> cow_done(m->seqs.size(), 0);
    for (size_t s = 0; s < m->seqs.size(); ++s) len[s] = m->seqs[s].len;
    int64_t need = 0;
    for (int32_t i = 0; i < num_tokens; ++i) {
        const int32_t s = seq_ids[i];
        if (!m->valid_seq(s)) return KV_ERR_INVALID_ARGUMENT;
        const int32_t pos = len[s]++;
        if (pos / bs >= m->max_blocks_per_seq) return KV_ERR_OUT_OF_BLOCKS;
        if (pos % bs == 0) {
            ++need;
            cow_done[s] = 1;  // the sequence's last block is now a fresh private one
        } else if (!cow_done[s] && m->refcount[m->seqs[s].blocks.back()] > 1) {
            ++need;
            cow_done[s] = 1;
        }
    }
    if (need > static_cast<int64_t>(m->free_stack.size())) return KV_ERR_OUT_OF_BLOCKS;
    // apply, token by token in the given order
    int32_t copies = 0;
    for (int32_t i = 0; i < num_tokens; ++i) {
        auto& sq = m->seqs[seq_ids[i]];
        const int32_t pos = sq.len;
        if (pos % bs == 0) {
            sq.blocks.push_back(m->pop_block());  // last block full (or none): a new one
        } else {
            const int32_t last = sq.blocks.back();
            if (m->refcount[last] > 1) {           // shared, partly filled: copy on write
                const int32_t fresh = m->pop_block();
                copy_src[copies] = last;
                copy_dst[copies] = fresh;
                ++copies;
                m->release(last);
                sq.blocks.back() = fresh;
            }
        }
        slots[i] = static_cast<int64_t>(sq.blocks[pos / bs]) * bs + pos % bs;
        sq.len = pos + 1;
    }
    *num_copies = copies;
    return KV_OK;
}

kv_status kv_block_manager_export(const kv_block_manager* m, int32_t* block_table,
                                  int32_t* context_lens) {
    if (m == nullptr || block_table == nullptr || context_lens == nullptr)
        return KV_ERR_INVALID_ARGUMENT;
    const int32_t mb = m->max_blocks_per_seq;
    for (size_t s = 0; s < m->seqs.size(); ++s) {
        const auto& sq = m->seqs[s];
        int32_t* row = block_table + s * mb;
        std::fill(row, row + mb, kPoisonBlock);
        std::copy(sq.blocks.begin(), sq.blocks.end(), row);
        context_lens[s] = sq.live ? sq.len : 0;
    }
    return KV_OK;
}

int32_t kv_block_manager_refcount(const kv_block_manager* m, int32_t block) {
    if (m == nullptr || block < 0 || block >= static_cast<int32_t>(m->refcount.size())) return -1;
    return m->refcount[block];
}

}  // extern "C"
