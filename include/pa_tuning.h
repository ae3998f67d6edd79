/*
 * pa_tuning.h -- explicit scheduling and test options for pa_decode.
 *
 * pa_decode (pa.h) always runs its default schedule: the one measured fastest
 * on B200 for every workload the library was tuned on.  This header exposes
 * the alternatives it was measured against, and two fault-path test hooks, as
 * an explicit argument: nothing in the library reads the environment, so its
 * behaviour depends only on the arguments of each call.
 *
 * The computed function never changes: every option below gives the same
 * attention output up to fp32 rounding order (the split of a context into
 * partitions and the merge of partitions are exact algebra), and the tests
 * run the parity suite under each of them.
 */
#ifndef PA_TUNING_H_
#define PA_TUNING_H_

#include <stddef.h>
#include <stdint.h>

#include "pa.h"

#ifdef __cplusplus
extern "C" {
#endif

/* Kernel shape of the tensor-core attention kernel (fp16/bf16, GQA group <= 8). */
typedef enum {
    PA_SHAPE_AUTO = 0,    /* default: PA_SHAPE_QUAD */
    PA_SHAPE_PAIRED = 1,  /* 2 CTAs per SM, two consumer warps, 10-stage ring; partitions merged by the reduce kernel */
    PA_SHAPE_QUAD = 2,    /* 4 CTAs per SM, one consumer warp, 6-stage ring, merger warp for <= 8 partitions */
    PA_SHAPE_TRIPLE = 3,  /* 3 CTAs per SM, one consumer warp, 8-stage ring */
    PA_SHAPE_PAIR1 = 4    /* 2 CTAs per SM, one consumer warp, 13-stage ring */
} pa_decode_shape;

typedef struct {
    int32_t shape;            /* pa_decode_shape */
    int32_t planner;          /* 0: automatic (attention CTAs plan their own items for batches of
                                    <= 256 sequences); 1: always the one-CTA planning kernel */
    int32_t split;            /* 0: a sequence's partitions are full, the remainder last;
                                 1: near-equal partition lengths */
    int32_t order;            /* 0: items of sequences split into several partitions first,
                                    each class largest first; 1: all items largest first */
    /* ---- fault-path test hooks (leave zero in production) ---- */
    int64_t wait_limit_ns;    /* bound of every wait inside the attention kernel; 0 = 2 s */
    int32_t stall_first_item; /* 1: CTA 0 of the attention kernel never publishes its first item,
                                 so the waits on it run out: the kernel reports PA_ERR_TIMEOUT in
                                 *status, drains the copies it issued and returns; the results
                                 are then incomplete and the workspace must be zeroed again */
    int32_t reserved;
} pa_decode_tuning;

/*
 * pa_decode_tuned -- pa_decode with explicit options; `tuning` NULL (or all
 * zero) is exactly pa_decode.  Arguments, workspace contract, errors and
 * results are those of pa_decode (pa.h).  Out-of-range option values return
 * PA_ERR_INVALID_ARG and enqueue nothing.
 */
pa_status pa_decode_tuned(void* out, const void* q, const void* key_cache, const void* value_cache,
                          const int32_t* block_tables, int32_t max_blocks_per_seq, const int32_t* context_lens,
                          int32_t num_seqs, int32_t num_heads, int32_t num_kv_heads, int32_t head_dim,
                          int32_t block_size, int32_t num_blocks, float scale, int32_t max_context_len,
                          int32_t partition_size, void* workspace, size_t workspace_bytes, pa_dtype dtype,
                          int32_t* status, pa_stream_t stream, const pa_decode_tuning* tuning);

/* pa_decode_launch_count for pa_decode_tuned with these options (NULL = defaults). */
int32_t pa_decode_launch_count_tuned(int32_t num_seqs, int32_t num_heads, int32_t num_kv_heads, int32_t head_dim,
                                     int32_t max_context_len, int32_t partition_size, pa_dtype dtype,
                                     const pa_decode_tuning* tuning);

#ifdef __cplusplus
}
#endif

#endif /* PA_TUNING_H_ */
