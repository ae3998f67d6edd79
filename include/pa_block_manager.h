/*
 * pa_block_manager.h -- C ABI of the host-side block manager that feeds the
 * paged KV-cache kernels (include/pa.h).
 *
 * What it implements is the bookkeeping the pages describe around the pool:
 *   - the KV cache is a pool of fixed-size physical blocks; a request's
 *     logical blocks map to physical ones through its block table, and blocks
 *     are taken from the pool only when a request's last block is full
 *     ("PagedAttention" digest, sections "This is just virtual memory" and
 *     "PagedAttention in one picture"; "LLM Inference Visualizer", lesson 06,
 *     "How paging grows");
 *   - requests that share a prefix share its physical blocks, each block
 *     carrying a reference count; a request that must write into a shared
 *     block first gets a private copy of it (copy-on-write; digest, section
 *     "Copy-on-write: when two requests share a prefix"; "PagedAttention,
 *     Visualized", Part 3);
 *   - a finished request returns its blocks; a block goes back to the free
 *     pool when its last reference is gone.
 *
 * The manager produces exactly what the kernels consume: the slot of every
 * new token (pa_reshape_and_cache's slot_mapping), the (src, dst) pairs of
 * copy-on-write clones (pa_copy_blocks), and block tables plus context
 * lengths (pa_decode).  It only does host bookkeeping: it touches no device
 * memory.
 *
 * Conventions
 * -----------
 *  * A manager is an opaque handle owned by the caller (create / destroy).
 *    It is not thread-safe: one caller at a time.
 *  * Sequences are named by caller-chosen int64 ids.
 *  * All pointer arguments are HOST memory, owned by the caller.
 *  * A slot is block * block_size + offset, as in pa.h.
 *  * Free blocks are handed out from a stack: the most recently freed block
 *    first; a fresh pool hands out 0, 1, 2, ...
 *  * Every call either succeeds completely or changes nothing: a call that
 *    would need more blocks than are free returns PA_ERR_NO_BLOCKS and leaves
 *    the manager as it was (so the caller can preempt or swap and retry).
 */
#ifndef PA_BLOCK_MANAGER_H_
#define PA_BLOCK_MANAGER_H_

#include <stddef.h>
#include <stdint.h>

#include "pa.h"

#ifdef __cplusplus
extern "C" {
#endif

typedef struct pa_block_manager pa_block_manager;

/* A pool of num_blocks device blocks of block_size tokens (1 .. 1024; the
 * attention and cache kernels take 8, 16 or 32, prefill 16) and a pool of
 * num_host_blocks blocks in CPU memory that swapped-out sequences move to
 * (0: no swapping).  Returns NULL for invalid arguments or when memory runs
 * out. */
pa_block_manager* pa_bm_create(int32_t num_blocks, int32_t block_size, int32_t num_host_blocks);
void pa_bm_destroy(pa_block_manager* bm);

int32_t pa_bm_num_blocks(const pa_block_manager* bm);
int32_t pa_bm_num_free_blocks(const pa_block_manager* bm);
int32_t pa_bm_num_sequences(const pa_block_manager* bm);
int32_t pa_bm_num_free_host_blocks(const pa_block_manager* bm);

/* References to a block (0 = free), or -1 for an id outside the pool. */
int32_t pa_bm_ref_count(const pa_block_manager* bm, int32_t block);

/*
 * pa_bm_add_sequence -- a new sequence holding num_tokens >= 0 tokens (its
 * prompt): ceil(num_tokens / block_size) fresh blocks.  If slot_mapping is
 * not NULL it receives the num_tokens slots in order.  A seq_id already in
 * use is PA_ERR_INVALID_ARG.
 */
pa_status pa_bm_add_sequence(pa_block_manager* bm, int64_t seq_id, int32_t num_tokens, int64_t* slot_mapping);

/*
 * pa_bm_fork -- child_id (new) shares every block of parent_id: same block
 * table, same length, each block's reference count + 1.  No block is copied
 * until one of them writes into a shared, partly filled block.
 */
pa_status pa_bm_fork(pa_block_manager* bm, int64_t parent_id, int64_t child_id);

/*
 * pa_bm_append_tokens -- one new token for each of the n sequences (one
 * decode step), in order; a sequence may appear more than once.  For token k:
 *   - if the sequence's last block is full (or it has none), a fresh block is
 *     appended to its table;
 *   - else if its last block is shared, a fresh block replaces it in this
 *     sequence's table, the pair (old, fresh) is written to copy_pairs, and
 *     the old block loses one reference (copy-on-write);
 *   - slot_mapping[k] = the new token's slot.
 *   slot_mapping   int64 [n]
 *   copy_pairs     int64 [n][2] (capacity n pairs), the pa_copy_blocks input;
 *                  apply the copies before writing the new tokens
 *   num_copy_pairs pairs written
 */
pa_status pa_bm_append_tokens(pa_block_manager* bm, const int64_t* seq_ids, int32_t n, int64_t* slot_mapping,
                              int64_t* copy_pairs, int32_t* num_copy_pairs);

/* pa_bm_free_sequence -- drop the sequence (resident or swapped out); its
 * device blocks lose one reference each, its host blocks are free again. */
pa_status pa_bm_free_sequence(pa_block_manager* bm, int64_t seq_id);

/*
 * pa_bm_swap_out -- evict a resident sequence to the host pool under memory
 * pressure ("PagedAttention, Visualized", Part 3: swapping to disk is
 * evicting blocks to CPU memory; shared blocks stay, since others still use
 * them).  Every block only this sequence references gets a host block and is
 * freed on the device; shared blocks keep the sequence's reference.  pairs
 * (int64 [n][2], capacity = the sequence's block count) receives (device
 * block, host block) for pa_swap_blocks from the device pools to the host
 * pools; run that copy before the freed device blocks are written again.  A
 * swapped-out sequence cannot be appended to, forked or decoded.
 */
pa_status pa_bm_swap_out(pa_block_manager* bm, int64_t seq_id, int64_t* pairs, int32_t* num_pairs);

/*
 * pa_bm_swap_in -- bring a swapped-out sequence back: a fresh device block for
 * each of its host blocks; pairs receives (host block, device block) for
 * pa_swap_blocks from the host pools to the device pools.
 */
pa_status pa_bm_swap_in(pa_block_manager* bm, int64_t seq_id, int64_t* pairs, int32_t* num_pairs);

/* 1 if the sequence is swapped out, 0 if resident, -1 for an unknown id. */
int32_t pa_bm_is_swapped(const pa_block_manager* bm, int64_t seq_id);

/*
 * pa_bm_block_tables -- the pa_decode inputs for n sequences:
 *   block_tables  int32 [n][max_blocks_per_seq], rows padded with -1
 *   context_lens  int32 [n]
 * A sequence with more than max_blocks_per_seq blocks is PA_ERR_INVALID_ARG.
 */
pa_status pa_bm_block_tables(const pa_block_manager* bm, const int64_t* seq_ids, int32_t n,
                             int32_t max_blocks_per_seq, int32_t* block_tables, int32_t* context_lens);

/* Blocks and tokens of one sequence (-1 for an unknown id). */
int32_t pa_bm_sequence_blocks(const pa_block_manager* bm, int64_t seq_id);
int64_t pa_bm_sequence_length(const pa_block_manager* bm, int64_t seq_id);

#ifdef __cplusplus
}
#endif

#endif /* PA_BLOCK_MANAGER_H_ */
