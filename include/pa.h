/*
 * pa.h -- C ABI of the B200 (sm_100a) paged KV-cache decode-attention library.
 *
 * What the library implements is the hot path the pages describe:
 *   - the KV cache lives in a shared pool of fixed-size physical blocks (16
 *     tokens by default), and each request reaches its blocks through a block table that
 *     maps logical block index -> physical block index ("PagedAttention"
 *     digest, section "PagedAttention in one picture");
 *   - each decoded token appends one K/V entry inside the current logical
 *     block ("LLM Inference Visualizer", lesson 06, "How paging grows");
 *   - attention walks the block table and gathers K and V from wherever they
 *     live, computing exactly ordinary attention ("PagedAttention" digest,
 *     sections "PagedAttention in one picture", "Why the attention kernel
 *     works at all" and "Misconceptions");
 *   - a shared block that a request must write is cloned first
 *     (copy-on-write; "PagedAttention" digest, section "Copy-on-write: when
 *     two requests share a prefix").
 *
 * Conventions shared by every call
 * --------------------------------
 *  * All tensor arguments are DEVICE pointers owned by the caller.  Scalars
 *    are passed by value.  Nothing is allocated, and no state is kept between
 *    calls.
 *  * Every call is asynchronous on `stream` (a cudaStream_t; NULL = legacy
 *    default stream).  A return of PA_OK means the work was enqueued.
 *  * Arguments that can be checked on the host are checked before anything is
 *    enqueued; a failing check returns PA_ERR_INVALID_ARG or
 *    PA_ERR_UNSUPPORTED and enqueues nothing.  A failed launch returns
 *    PA_ERR_CUDA.
 *  * Values that only the device sees (block ids, slots, context lengths) are
 *    range-checked by the kernels.  A bad value is skipped -- never read or
 *    written out of bounds -- and PA_ERR_OUT_OF_RANGE is OR-ed into
 *    `*status` when `status` is not NULL.  `status` is a device int32 the
 *    caller zeroes and reads back after synchronising.  Kernels never trap.
 *  * Dtypes: q, K, V, out and the appended key/value share one element type.
 *  * Pool layout (both key_cache and value_cache), with BS = block_size:
 *        [num_blocks][num_kv_heads][BS][head_dim]   row-major,
 *    so one (block, KV head) tile of BS tokens is a contiguous run of
 *    BS * head_dim elements.  Slot s of the pool is block s / BS, offset s % BS.
 *  * GQA: query head h uses KV head h / (num_heads / num_kv_heads).
 *  * Supported: block_size 8, 16 or 32 (pa_prefill: 16); head_dim 64 or 128;
 *    float32, float16, bfloat16.  16 is the pages' default: smaller blocks
 *    waste fewer slots in a sequence's last block but need longer block
 *    tables and more, smaller reads ("PagedAttention" digest,
 *    "Misconceptions").
 *  * Slots of a block past a sequence's context may hold anything (NaN bit
 *    patterns included): the attention calls never let them reach a result.
 */
#ifndef PA_H_
#define PA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as cudaStream_t, declared here so the header needs no CUDA headers. */
typedef struct CUstream_st* pa_stream_t;

/* Host return codes; the device status word ORs the same bit values. */
typedef enum {
    PA_OK = 0,
    PA_ERR_INVALID_ARG = 1,   /* null pointer, negative size, misaligned buffer, small workspace */
    PA_ERR_UNSUPPORTED = 2,   /* valid but not implemented: block_size, head_dim, dtype */
    PA_ERR_OUT_OF_RANGE = 4,  /* device: block id, slot or context length outside its range */
    PA_ERR_CUDA = 8,          /* a CUDA launch or query failed */
    PA_ERR_TIMEOUT = 16,      /* device: a bounded wait inside a kernel gave up */
    PA_ERR_NO_BLOCKS = 32     /* block manager (pa_block_manager.h): not enough free blocks */
} pa_status;

typedef enum { PA_F32 = 0, PA_F16 = 1, PA_BF16 = 2 } pa_dtype;

/*
 * pa_reshape_and_cache -- write the K/V of newly decoded tokens into the pool.
 *
 * For every token t < num_tokens with s = slot_mapping[t] >= 0:
 *     key_cache  [s / BS][h][s % BS][:] = key  [t][h][:]   for all h < num_kv_heads
 *     value_cache[s / BS][h][s % BS][:] = value[t][h][:]
 * A negative slot is padding and writes nothing.  A slot >= num_blocks * BS
 * writes nothing and sets PA_ERR_OUT_OF_RANGE in *status.  The copy is
 * bit-exact.  Distinct tokens must name distinct slots (otherwise which one
 * lands is unspecified).
 *
 *   key, value      [num_tokens][num_kv_heads][head_dim], contiguous, 16-byte aligned
 *   key_cache,
 *   value_cache     pools, layout above, 16-byte aligned
 *   slot_mapping    int64 [num_tokens]
 *   status          nullable device int32, OR-ed with PA_ERR_* bits
 */
pa_status pa_reshape_and_cache(const void* key, const void* value, void* key_cache, void* value_cache,
                               const int64_t* slot_mapping, int64_t num_tokens, int32_t num_blocks,
                               int32_t num_kv_heads, int32_t head_dim, int32_t block_size,
                               pa_dtype dtype, int32_t* status, pa_stream_t stream);

/*
 * pa_decode_workspace_size -- bytes of device workspace pa_decode needs.
 *
 * The workspace holds the work list of (sequence, partition, KV head) items
 * and, for sequences split into several partitions, each partition's
 * (max logit, sum of exponentials, unnormalised output) in fp32.  The result
 * depends only on the arguments given here; pass the same values (including
 * partition_size, 0 = automatic) to pa_decode.  Returns 0 for invalid
 * arguments.
 */
size_t pa_decode_workspace_size(int32_t num_seqs, int32_t num_heads, int32_t num_kv_heads,
                                int32_t head_dim, int32_t max_context_len, int32_t partition_size);

/*
 * pa_decode -- one decode step of attention through the block tables.
 *
 * For every sequence b < num_seqs and query head h < num_heads, with
 * n = context_lens[b] and g = h / (num_heads / num_kv_heads):
 *     K_i = key_cache  [block_tables[b][i / BS]][g][i % BS][:]   (i < n)
 *     V_i = value_cache[block_tables[b][i / BS]][g][i % BS][:]
 *     out[b][h][:] = sum_i softmax_i(scale * q[b][h][:] . K_i) V_i
 * computed in fp32 from the stored values and rounded to the element type.
 * n = 0 gives a zero row.  The context is split into partitions of
 * partition_size tokens that run in parallel.  When no sequence spans more
 * than 8 partitions (fp16/bf16, at most 16 query heads per KV head), the
 * attention kernel merges a sequence's partitions itself: the CTA that
 * finishes its last partition combines them, and no second kernel runs.
 * Otherwise a reduce kernel merges them after the attention kernel.  The
 * merge is exact algebra, so the result does not depend on the split beyond
 * fp32 rounding, and it does not depend on where blocks live.  Scheduling
 * alternatives (kernel shape, planner, split, order) are selectable through
 * pa_decode_tuned (pa_tuning.h); this call always uses the defaults.
 *
 *   out                 [num_seqs][num_heads][head_dim], 16-byte aligned
 *   q                   [num_seqs][num_heads][head_dim], 16-byte aligned
 *   key_cache,
 *   value_cache         pools, layout above
 *   block_tables        int32 [num_seqs][max_blocks_per_seq]; only the first
 *                       ceil(n / BS) entries of row b are read, each must be
 *                       in [0, num_blocks): else PA_ERR_OUT_OF_RANGE, and the
 *                       16-token tile holding the bad block contributes
 *                       nothing (with 8-token blocks that includes the other
 *                       block of the tile; with 32-token blocks, both tiles
 *                       of the block)
 *                       (with context_lens: read-only here, and possibly read
 *                       before this call's kernels wait for kernels enqueued
 *                       earlier with programmatic dependent launch, i.e.
 *                       kernels that signal their dependents before they end;
 *                       no kernel of this library writes either array, and a
 *                       kernel without that signal has ended before this call
 *                       starts)
 *   context_lens        int32 [num_seqs]; a value outside
 *                       [0, min(max_context_len, max_blocks_per_seq * BS)] is
 *                       clamped into that range and sets PA_ERR_OUT_OF_RANGE
 *   max_context_len     host-side upper bound of context_lens (sizes the split)
 *   partition_size      tokens per partition: 0 = automatic, else a multiple
 *                       of 16 in [16, 512]
 *   workspace           device buffer of at least pa_decode_workspace_size()
 *                       bytes, 256-byte aligned, ZERO-FILLED before its first
 *                       use (cudaMemset).  It holds counters that each call
 *                       leaves at zero for the next, whatever the sizes of the
 *                       next problem, and the call's plan, which
 *                       pa_decode_planned may reuse (below); the rest is
 *                       scratch.  After a call that reported PA_ERR_TIMEOUT,
 *                       zero it again.  Calls that share a workspace must not
 *                       overlap in time.
 *
 * The call enqueues pa_decode_launch_count() kernels on `stream`.
 */
pa_status pa_decode(void* out, const void* q, const void* key_cache, const void* value_cache,
                    const int32_t* block_tables, int32_t max_blocks_per_seq,
                    const int32_t* context_lens, int32_t num_seqs, int32_t num_heads,
                    int32_t num_kv_heads, int32_t head_dim, int32_t block_size, int32_t num_blocks,
                    float scale, int32_t max_context_len, int32_t partition_size, void* workspace,
                    size_t workspace_bytes, pa_dtype dtype, int32_t* status, pa_stream_t stream);

/*
 * pa_decode_launch_count -- number of kernels pa_decode enqueues for these
 * sizes on the current device (1 to 3: an optional planning kernel, the
 * attention kernel, an optional reduce kernel).  Returns -1 for arguments
 * pa_decode would reject, or when the device cannot be queried.
 */
int32_t pa_decode_launch_count(int32_t num_seqs, int32_t num_heads, int32_t num_kv_heads, int32_t head_dim,
                               int32_t max_context_len, int32_t partition_size, pa_dtype dtype);

/*
 * pa_decode_plan, pa_decode_planned -- pa_decode split into a plan, made once
 * per step, and one planned decode per model layer.
 *
 * The work of a decode step is a list of (sequence, partition, KV head) items
 * (long contexts are split into partitions that run in parallel, see
 * pa_decode) that depends only on context_lens and the sizes; every layer of
 * a model decodes the same step over its own pools.  pa_decode_plan
 * writes that list into `workspace` (one small kernel), and every pa_decode
 * call leaves the list it worked from there too; each pa_decode_planned call
 * then decodes without making it.  pa_decode_planned computes exactly what
 * pa_decode computes (the same kernels, the same result bits) provided that:
 *   - the workspace was last planned, by pa_decode_plan or by pa_decode (or
 *     pa_decode_tuned with the default partition split), with this call's
 *     context_lens values, num_seqs, num_heads, num_kv_heads, head_dim,
 *     block_size, max_blocks_per_seq, max_context_len and partition_size;
 *   - the plan is ordered before the call: the same stream (the library's
 *     kernels complete in stream order), or an event or synchronization
 *     between streams;
 *   - no call on the workspace has since reported an error (after
 *     PA_ERR_TIMEOUT, zero the workspace and plan again).
 * A plan stays valid for any number of planned calls; the next pa_decode or
 * pa_decode_plan on the workspace replaces it.
 *
 * pa_decode_plan's arguments mean what they mean for pa_decode (status and
 * stream too: a length outside [0, min(max_context_len, max_blocks_per_seq *
 * block_size)] is clamped and reported as PA_ERR_OUT_OF_RANGE); it reads only
 * context_lens, and its validation and errors are pa_decode's for those
 * arguments.  It enqueues one kernel.  pa_decode_planned takes pa_decode's
 * arguments and enqueues pa_decode_planned_launch_count() kernels (the
 * attention kernel, and the reduce kernel when a sequence spans more
 * partitions than the attention kernel merges).
 */
pa_status pa_decode_plan(const int32_t* context_lens, int32_t num_seqs, int32_t num_heads, int32_t num_kv_heads,
                         int32_t head_dim, int32_t block_size, int32_t max_blocks_per_seq, int32_t max_context_len,
                         int32_t partition_size, void* workspace, size_t workspace_bytes, int32_t* status,
                         pa_stream_t stream);
pa_status pa_decode_planned(void* out, const void* q, const void* key_cache, const void* value_cache,
                            const int32_t* block_tables, int32_t max_blocks_per_seq,
                            const int32_t* context_lens, int32_t num_seqs, int32_t num_heads,
                            int32_t num_kv_heads, int32_t head_dim, int32_t block_size, int32_t num_blocks,
                            float scale, int32_t max_context_len, int32_t partition_size, void* workspace,
                            size_t workspace_bytes, pa_dtype dtype, int32_t* status, pa_stream_t stream);
int32_t pa_decode_planned_launch_count(int32_t num_seqs, int32_t num_heads, int32_t num_kv_heads,
                                       int32_t head_dim, int32_t max_context_len, int32_t partition_size,
                                       pa_dtype dtype);

/*
 * pa_copy_blocks -- copy-on-write clone of whole blocks, in both pools.
 *
 * For each pair k < num_pairs with (src, dst) = (block_pairs[2k], block_pairs[2k+1]):
 *     key_cache[dst] = key_cache[src];  value_cache[dst] = value_cache[src]
 * (all num_kv_heads * BS * head_dim elements; bit-exact).  A pair with an id
 * outside [0, num_blocks) is skipped and sets PA_ERR_OUT_OF_RANGE.  No dst
 * may repeat and no dst may also be a src in the same call (that would be a
 * write/write or read/write race); the result is then unspecified.
 *
 *   block_pairs   int64 [num_pairs][2], device
 */
pa_status pa_copy_blocks(void* key_cache, void* value_cache, const int64_t* block_pairs,
                         int32_t num_pairs, int32_t num_blocks, int32_t num_kv_heads,
                         int32_t head_dim, int32_t block_size, pa_dtype dtype, int32_t* status,
                         pa_stream_t stream);

/*
 * pa_prefill -- causal attention of a chunk of new query tokens per sequence
 * over everything the sequence has in the paged cache (prompt processing, and
 * chunked prefill on top of an existing context).
 *
 * Sequence b's new tokens are q rows [query_start[b], query_start[b+1]); with
 * n = context_lens[b] tokens in the cache, the new ones included (written
 * first with pa_reshape_and_cache), and L = query_start[b+1] - query_start[b],
 * query row i < L sits at position p = n - L + i and attends to positions
 * 0 .. p through the block table ("PagedAttention" digest, sections
 * "PagedAttention in one picture" and "Why the attention kernel works at
 * all"): with g = h / (num_heads / num_kv_heads),
 *     out[query_start[b] + i][h][:] = sum_{j <= p} softmax_j(scale * q . K_j) V_j
 * computed in fp32 from the stored values and rounded to the element type.
 *
 *   out, q          [query_start[num_seqs]][num_heads][head_dim], 16-byte aligned
 *   block_tables    int32 [num_seqs][max_blocks_per_seq]; entries outside
 *                   [0, num_blocks) set PA_ERR_OUT_OF_RANGE and contribute nothing
 *   query_start     int32 [num_seqs + 1], nondecreasing, device
 *   context_lens    int32 [num_seqs], device; n < L or n > max_blocks_per_seq * 16
 *                   sets PA_ERR_OUT_OF_RANGE and leaves that sequence's rows unwritten
 *   max_query_len   host-side upper bound of the L (sizes the grid)
 * Supported: block_size 16, float16 and bfloat16, head_dim 64 or 128, at most
 * 16 query heads per KV head (PA_ERR_UNSUPPORTED otherwise).  No workspace.
 */
pa_status pa_prefill(void* out, const void* q, const void* key_cache, const void* value_cache,
                     const int32_t* block_tables, int32_t max_blocks_per_seq, const int32_t* query_start,
                     const int32_t* context_lens, int32_t num_seqs, int32_t num_heads, int32_t num_kv_heads,
                     int32_t head_dim, int32_t block_size, int32_t num_blocks, float scale, int32_t max_query_len,
                     pa_dtype dtype, int32_t* status, pa_stream_t stream);

/*
 * pa_prefill_ws -- pa_prefill with a workspace, which lets the tensor-core
 * kernel balance its last wave.  That kernel runs one CTA per SM on 128-row
 * tiles; when the tiles do not fill whole waves, each tile of the last,
 * partial wave is split by key range into pieces (up to 16) that run on the
 * SMs the wave would leave idle.  Each piece writes its rows' unnormalised
 * partial output, reference max and sum to the workspace, and a second
 * kernel, chained to the first, merges them (exact algebra: out = sum_q
 * 2^(m_q - m) O_q / sum_q 2^(m_q - m) l_q).  The result is the same function
 * as pa_prefill's, up to fp32 rounding.
 *
 *   workspace        device memory of at least pa_prefill_workspace_size()
 *                    bytes for these sizes, 16-byte aligned; scratch only (no
 *                    contents carry from one call to the next).  May be NULL
 *                    when the size is 0.
 *   workspace_bytes  its size; smaller than required: PA_ERR_INVALID_ARG
 * Calls that share a workspace must not run concurrently.  Everything else is
 * as pa_prefill.
 */
pa_status pa_prefill_ws(void* out, const void* q, const void* key_cache, const void* value_cache,
                        const int32_t* block_tables, int32_t max_blocks_per_seq, const int32_t* query_start,
                        const int32_t* context_lens, int32_t num_seqs, int32_t num_heads, int32_t num_kv_heads,
                        int32_t head_dim, int32_t block_size, int32_t num_blocks, float scale, int32_t max_query_len,
                        void* workspace, size_t workspace_bytes, pa_dtype dtype, int32_t* status,
                        pa_stream_t stream);

/*
 * pa_prefill_workspace_size -- the workspace pa_prefill_ws needs for these
 * sizes on the current device (the split depends on its SM count; 0 when the
 * tiles fill whole waves or the chunk is served by the mma.sync kernel).
 * Invalid sizes: the error pa_prefill would return.
 */
pa_status pa_prefill_workspace_size(int32_t num_seqs, int32_t num_heads, int32_t num_kv_heads, int32_t head_dim,
                                    int32_t max_query_len, pa_dtype dtype, size_t* bytes);

/*
 * pa_swap_blocks -- copy whole blocks from one pool to another of the same
 * shape, for evicting blocks to CPU memory and bringing them back
 * ("PagedAttention, Visualized", Part 3: the operating-system table, where
 * swapping to disk corresponds to evicting blocks to CPU memory; an evicted
 * sequence's shared blocks stay, because others still use them).  The block
 * manager (pa_block_manager.h) produces the pairs.
 *
 * For each pair k < num_pairs with (s, d) = (block_pairs[2k], block_pairs[2k+1]):
 *     dst_key_cache[d] = src_key_cache[s];  dst_value_cache[d] = src_value_cache[s]
 * (all num_kv_heads * BS * head_dim elements; bit-exact).  Either pool may be
 * pinned host memory that the device addresses directly (cudaHostAlloc or
 * cudaMallocHost memory, which unified addressing maps at the same pointer):
 * swapping out is device -> host, swapping in host -> device.  A pair with an
 * id outside [0, src_num_blocks) or [0, dst_num_blocks) is skipped and sets
 * PA_ERR_OUT_OF_RANGE.  No dst may repeat.  The source pool must not be
 * written by other work until the call has completed on `stream`.
 *
 *   block_pairs   int64 [num_pairs][2], device-addressable (device or pinned host)
 */
pa_status pa_swap_blocks(const void* src_key_cache, const void* src_value_cache, void* dst_key_cache,
                         void* dst_value_cache, const int64_t* block_pairs, int32_t num_pairs, int32_t src_num_blocks,
                         int32_t dst_num_blocks, int32_t num_kv_heads, int32_t head_dim, int32_t block_size,
                         pa_dtype dtype, int32_t* status, pa_stream_t stream);

/*
 * pa_decode_noalloc -- pa_decode without a caller-allocated workspace.
 *
 * The pages have no counterpart to this call; it exists for callers that
 * cannot allocate device memory: code hosted by an engine that owns all
 * device memory and gives its extensions no allocator, or a latency-critical
 * loop that must not call cudaMalloc (which can synchronise the device).
 * Arguments and results are those of pa_decode minus the workspace; the
 * caller still passes every input and output buffer.
 *
 * The scratch is a fixed 32 MiB array in the library's device memory, held
 * on every GPU that loads the library until the process exits.  A problem
 * whose pa_decode_workspace_size() exceeds 32 MiB returns PA_ERR_UNSUPPORTED
 * and enqueues nothing.  The first call made with a given device current
 * looks up the array's device address (cudaGetSymbolAddress), zero-fills it
 * on `stream` and waits for that (cudaStreamSynchronize); make that first
 * call before any stream capture begins (a first call on a stream that is
 * being captured returns PA_ERR_INVALID_ARG and enqueues nothing).  No
 * cudaMalloc or cudaFree is made.
 * All calls share the one array: calls whose kernels overlap on the GPU (two
 * streams, two host threads) race on it and give wrong results.  After a call
 * that reported PA_ERR_TIMEOUT, stop using this entry point in the process.
 */
pa_status pa_decode_noalloc(void* out, const void* q, const void* key_cache, const void* value_cache,
                            const int32_t* block_tables, int32_t max_blocks_per_seq,
                            const int32_t* context_lens, int32_t num_seqs, int32_t num_heads,
                            int32_t num_kv_heads, int32_t head_dim, int32_t block_size, int32_t num_blocks,
                            float scale, int32_t max_context_len, int32_t partition_size, pa_dtype dtype,
                            int32_t* status, pa_stream_t stream);

/* Static, human-readable name of a status code (or of the lowest bit set). */
const char* pa_get_error_string(pa_status status);

/* Library version as major * 10000 + minor * 100 + patch. */
int32_t pa_version(void);

#ifdef __cplusplus
}
#endif

#endif /* PA_H_ */
