// Host-side block manager: on-demand allocation, reference-counted sharing,
// copy-on-write, and the slot mappings / copy pairs / block tables the
// kernels take.  See include/pa_block_manager.h for the contract.
//
// The pages' model ("PagedAttention" digest, sections "This is just virtual
// memory", "PagedAttention in one picture", "Copy-on-write: when two
// requests share a prefix"): a request's logical blocks map to physical
// blocks of a shared pool; a block is allocated when the last one fills;
// forks share blocks and count references; a write into a shared block first
// clones it.
#include <algorithm>
#include <cstdint>
#include <new>
#include <unordered_map>
#include <vector>

#include "pa_block_manager.h"

namespace {

struct Sequence {
    std::vector<int32_t> blocks;  // physical block of each logical block (a host block where on_host)
    std::vector<uint8_t> on_host; // while swapped out: 1 where the block lives in the host pool
    bool swapped = false;
    int64_t len = 0;              // tokens
    int64_t pending = 0;          // scratch of pa_bm_append_tokens: tokens of this call counted so far
    int64_t pending_blocks = 0;   // scratch: fresh blocks this call appends to the table
};

}  // namespace

struct pa_block_manager {
    int32_t num_blocks = 0;
    int32_t block_size = 16;
    std::vector<int32_t> ref;          // references per block (0 = free)
    std::vector<int32_t> free_stack;   // top = back: the next block handed out
    int32_t num_host_blocks = 0;
    std::vector<int32_t> host_free;    // the host pool's free blocks, handed out the same way
    std::unordered_map<int64_t, Sequence> seqs;
    // scratch of pa_bm_append_tokens, kept between calls to avoid allocations
    std::vector<Sequence*> batch;      // sequence of each token
    std::vector<int32_t> copied;       // per block: references a counted copy took off it
    std::vector<int32_t> touched;      // blocks whose `copied` entry is set

    int32_t take() {
        const int32_t b = free_stack.back();
        free_stack.pop_back();
        ref[b] = 1;
        return b;
    }
    void drop(int32_t b) {
        if (--ref[b] == 0) free_stack.push_back(b);
    }
    int64_t slot(int32_t block, int64_t offset) const { return (int64_t)block * block_size + offset; }
};

extern "C" {

pa_block_manager* pa_bm_create(int32_t num_blocks, int32_t block_size, int32_t num_host_blocks) {
    if (num_blocks <= 0 || block_size <= 0 || block_size > 1024 || num_host_blocks < 0) return nullptr;
    if ((int64_t)num_blocks * block_size > INT64_MAX / 2) return nullptr;
    pa_block_manager* bm = new (std::nothrow) pa_block_manager;
    if (!bm) return nullptr;
    try {
        bm->num_blocks = num_blocks;
        bm->block_size = block_size;
        bm->ref.assign(num_blocks, 0);
        bm->copied.assign(num_blocks, 0);
        bm->free_stack.resize(num_blocks);
        for (int32_t i = 0; i < num_blocks; ++i) bm->free_stack[i] = num_blocks - 1 - i;   // pops 0, 1, 2, ...
        bm->num_host_blocks = num_host_blocks;
        bm->host_free.resize(num_host_blocks);
        for (int32_t i = 0; i < num_host_blocks; ++i) bm->host_free[i] = num_host_blocks - 1 - i;
    } catch (...) {
        delete bm;
        return nullptr;
    }
    return bm;
}

void pa_bm_destroy(pa_block_manager* bm) { delete bm; }

int32_t pa_bm_num_blocks(const pa_block_manager* bm) { return bm ? bm->num_blocks : 0; }
int32_t pa_bm_num_free_blocks(const pa_block_manager* bm) { return bm ? (int32_t)bm->free_stack.size() : 0; }
int32_t pa_bm_num_sequences(const pa_block_manager* bm) { return bm ? (int32_t)bm->seqs.size() : 0; }
int32_t pa_bm_num_free_host_blocks(const pa_block_manager* bm) { return bm ? (int32_t)bm->host_free.size() : 0; }

int32_t pa_bm_ref_count(const pa_block_manager* bm, int32_t block) {
    if (!bm || block < 0 || block >= bm->num_blocks) return -1;
    return bm->ref[block];
}

pa_status pa_bm_add_sequence(pa_block_manager* bm, int64_t seq_id, int32_t num_tokens, int64_t* slot_mapping) {
    if (!bm || num_tokens < 0) return PA_ERR_INVALID_ARG;
    if (bm->seqs.count(seq_id)) return PA_ERR_INVALID_ARG;
    const int64_t need = ((int64_t)num_tokens + bm->block_size - 1) / bm->block_size;
    if (need > (int64_t)bm->free_stack.size()) return PA_ERR_NO_BLOCKS;
    try {
        Sequence s;
        s.blocks.reserve(need);
        for (int64_t i = 0; i < need; ++i) s.blocks.push_back(bm->take());
        s.len = num_tokens;
        if (slot_mapping)
            for (int64_t t = 0; t < num_tokens; ++t)
                slot_mapping[t] = bm->slot(s.blocks[t / bm->block_size], t % bm->block_size);
        bm->seqs.emplace(seq_id, std::move(s));
    } catch (...) {
        return PA_ERR_INVALID_ARG;
    }
    return PA_OK;
}

pa_status pa_bm_fork(pa_block_manager* bm, int64_t parent_id, int64_t child_id) {
    if (!bm) return PA_ERR_INVALID_ARG;
    auto it = bm->seqs.find(parent_id);
    if (it == bm->seqs.end() || it->second.swapped || bm->seqs.count(child_id)) return PA_ERR_INVALID_ARG;
    try {
        Sequence child = it->second;   // same table: shared blocks
        for (int32_t b : child.blocks) ++bm->ref[b];
        bm->seqs.emplace(child_id, std::move(child));
    } catch (...) {
        return PA_ERR_INVALID_ARG;
    }
    return PA_OK;
}

pa_status pa_bm_append_tokens(pa_block_manager* bm, const int64_t* seq_ids, int32_t n, int64_t* slot_mapping,
                              int64_t* copy_pairs, int32_t* num_copy_pairs) {
    if (!bm || n < 0) return PA_ERR_INVALID_ARG;
    if (n > 0 && (!seq_ids || !slot_mapping || !copy_pairs)) return PA_ERR_INVALID_ARG;
    if (num_copy_pairs) *num_copy_pairs = 0;
    // First pass: validate and count the fresh blocks the batch needs, so the
    // call either succeeds completely or changes nothing.  It replays the
    // second pass's decisions: a sequence listed k times takes its k tokens
    // in order, and only its first token can need a copy (afterwards its last
    // block is private); a copy takes one reference off the shared block, so
    // the last of the sequences sharing it writes into it in place.
    std::vector<Sequence*>& seq = bm->batch;
    int64_t need = 0;
    bool ok = true;
    try {
        seq.resize(n);
    } catch (...) {
        return PA_ERR_INVALID_ARG;
    }
    int32_t k = 0;
    for (; k < n; ++k) {
        auto it = bm->seqs.find(seq_ids[k]);
        if (it == bm->seqs.end() || it->second.swapped) {
            ok = false;
            break;
        }
        Sequence* s = &it->second;
        seq[k] = s;
        if ((s->len + s->pending) % bm->block_size == 0) {
            ++need;   // the last block is full (or there is none)
            ++s->pending_blocks;
        } else if (s->pending == 0) {
            const int32_t last = s->blocks.back();
            if (bm->ref[last] - bm->copied[last] > 1) {   // still shared when this token comes: copy-on-write
                ++need;
                if (bm->copied[last]++ == 0) bm->touched.push_back(last);
            }
        }
        ++s->pending;
    }
    // clear the scratch counters; make room in the tables that grow, so the
    // second pass cannot fail half way
    bool room = true;
    for (int32_t i = 0; i < k; ++i) {
        Sequence* s = seq[i];
        if (s->pending_blocks > 0 && ok && need <= (int64_t)bm->free_stack.size()) {
            const size_t want = s->blocks.size() + (size_t)s->pending_blocks;
            if (want > s->blocks.capacity()) {
                try {
                    s->blocks.reserve(std::max(want, 2 * s->blocks.capacity()));
                } catch (...) {
                    room = false;
                }
            }
        }
        s->pending = 0;
        s->pending_blocks = 0;
    }
    for (int32_t b : bm->touched) bm->copied[b] = 0;
    bm->touched.clear();
    if (!ok || !room) return PA_ERR_INVALID_ARG;
    if (need > (int64_t)bm->free_stack.size()) return PA_ERR_NO_BLOCKS;
    int32_t pairs = 0;
    for (k = 0; k < n; ++k) {
        Sequence& s = *seq[k];
        const int64_t off = s.len % bm->block_size;
        if (off == 0) {
            s.blocks.push_back(bm->take());
        } else {
            const int32_t last = s.blocks.back();
            if (bm->ref[last] > 1) {   // copy-on-write: this sequence gets its own copy
                const int32_t fresh = bm->take();
                copy_pairs[2 * pairs] = last;
                copy_pairs[2 * pairs + 1] = fresh;
                ++pairs;
                bm->drop(last);
                s.blocks.back() = fresh;
            }
        }
        slot_mapping[k] = bm->slot(s.blocks.back(), off);
        ++s.len;
    }
    if (num_copy_pairs) *num_copy_pairs = pairs;
    return PA_OK;
}

pa_status pa_bm_free_sequence(pa_block_manager* bm, int64_t seq_id) {
    if (!bm) return PA_ERR_INVALID_ARG;
    auto it = bm->seqs.find(seq_id);
    if (it == bm->seqs.end()) return PA_ERR_INVALID_ARG;
    // release from the last block back, so the prompt's first block is handed out first again
    const Sequence& sq = it->second;
    for (size_t j = sq.blocks.size(); j-- > 0;) {
        if (sq.swapped && sq.on_host[j]) bm->host_free.push_back(sq.blocks[j]);
        else bm->drop(sq.blocks[j]);
    }
    bm->seqs.erase(it);
    return PA_OK;
}

pa_status pa_bm_swap_out(pa_block_manager* bm, int64_t seq_id, int64_t* pairs, int32_t* num_pairs) {
    if (!bm || !pairs || !num_pairs) return PA_ERR_INVALID_ARG;
    *num_pairs = 0;
    auto it = bm->seqs.find(seq_id);
    if (it == bm->seqs.end() || it->second.swapped) return PA_ERR_INVALID_ARG;
    Sequence& s = it->second;
    int64_t need = 0;   // blocks only this sequence holds move; shared ones stay for the others
    for (int32_t b : s.blocks) need += bm->ref[b] == 1;
    if (need > (int64_t)bm->host_free.size()) return PA_ERR_NO_BLOCKS;
    try {
        s.on_host.assign(s.blocks.size(), 0);
    } catch (...) {
        return PA_ERR_INVALID_ARG;
    }
    int32_t k = 0;
    for (size_t j = 0; j < s.blocks.size(); ++j) {
        const int32_t b = s.blocks[j];
        if (bm->ref[b] != 1) continue;
        const int32_t h = bm->host_free.back();
        bm->host_free.pop_back();
        pairs[2 * k] = b;
        pairs[2 * k + 1] = h;
        ++k;
        bm->drop(b);
        s.blocks[j] = h;
        s.on_host[j] = 1;
    }
    s.swapped = true;
    *num_pairs = k;
    return PA_OK;
}

pa_status pa_bm_swap_in(pa_block_manager* bm, int64_t seq_id, int64_t* pairs, int32_t* num_pairs) {
    if (!bm || !pairs || !num_pairs) return PA_ERR_INVALID_ARG;
    *num_pairs = 0;
    auto it = bm->seqs.find(seq_id);
    if (it == bm->seqs.end() || !it->second.swapped) return PA_ERR_INVALID_ARG;
    Sequence& s = it->second;
    int64_t need = 0;
    for (uint8_t h : s.on_host) need += h;
    if (need > (int64_t)bm->free_stack.size()) return PA_ERR_NO_BLOCKS;
    int32_t k = 0;
    for (size_t j = 0; j < s.blocks.size(); ++j) {
        if (!s.on_host[j]) continue;
        const int32_t h = s.blocks[j];
        const int32_t d = bm->take();
        pairs[2 * k] = h;
        pairs[2 * k + 1] = d;
        ++k;
        bm->host_free.push_back(h);
        s.blocks[j] = d;
    }
    s.on_host.clear();
    s.swapped = false;
    *num_pairs = k;
    return PA_OK;
}

int32_t pa_bm_is_swapped(const pa_block_manager* bm, int64_t seq_id) {
    if (!bm) return -1;
    auto it = bm->seqs.find(seq_id);
    return it == bm->seqs.end() ? -1 : (it->second.swapped ? 1 : 0);
}

pa_status pa_bm_block_tables(const pa_block_manager* bm, const int64_t* seq_ids, int32_t n,
                             int32_t max_blocks_per_seq, int32_t* block_tables, int32_t* context_lens) {
    if (!bm || n < 0 || max_blocks_per_seq <= 0) return PA_ERR_INVALID_ARG;
    if (n > 0 && (!seq_ids || !block_tables || !context_lens)) return PA_ERR_INVALID_ARG;
    // validate everything before writing anything; each id is looked up once
    std::vector<const Sequence*> seq;
    try {
        seq.resize(n);
    } catch (...) {
        return PA_ERR_INVALID_ARG;
    }
    for (int32_t k = 0; k < n; ++k) {
        auto it = bm->seqs.find(seq_ids[k]);
        if (it == bm->seqs.end() || it->second.swapped || (int64_t)it->second.blocks.size() > max_blocks_per_seq ||
            it->second.len > INT32_MAX)
            return PA_ERR_INVALID_ARG;
        seq[k] = &it->second;
    }
    for (int32_t k = 0; k < n; ++k) {
        const Sequence& s = *seq[k];
        int32_t* row = block_tables + (size_t)k * max_blocks_per_seq;
        std::copy(s.blocks.begin(), s.blocks.end(), row);
        std::fill(row + s.blocks.size(), row + max_blocks_per_seq, -1);
        context_lens[k] = (int32_t)s.len;
    }
    return PA_OK;
}

int32_t pa_bm_sequence_blocks(const pa_block_manager* bm, int64_t seq_id) {
    if (!bm) return -1;
    auto it = bm->seqs.find(seq_id);
    return it == bm->seqs.end() ? -1 : (int32_t)it->second.blocks.size();
}

int64_t pa_bm_sequence_length(const pa_block_manager* bm, int64_t seq_id) {
    if (!bm) return -1;
    auto it = bm->seqs.find(seq_id);
    return it == bm->seqs.end() ? -1 : it->second.len;
}

}  // extern "C"
