// Internal launch interface between the C ABI (pa_api.cu) and the kernels.
#pragma once

#include <cuda_runtime.h>

#include "pa_common.cuh"
#include "pa_tuning.h"

namespace pa {

// Device properties the launchers need (cached per device).
struct DeviceInfo {
    int sm_count;
    int max_smem_optin;
};
cudaError_t device_info(DeviceInfo* out);

cudaError_t launch_reshape_and_cache(const void* key, const void* value, void* key_cache, void* value_cache,
                                     const int64_t* slot_mapping, int64_t num_tokens, int32_t num_blocks,
                                     int32_t num_kv_heads, int32_t head_dim, int32_t block_size, int elt_bytes,
                                     int32_t* status,
                                     cudaStream_t stream);

cudaError_t launch_copy_blocks(void* key_cache, void* value_cache, const int64_t* block_pairs, int32_t num_pairs,
                               int32_t num_blocks, int32_t num_kv_heads, int32_t head_dim, int32_t block_size,
                               int elt_bytes, int32_t* status, cudaStream_t stream);

cudaError_t launch_swap_blocks(const void* src_key, const void* src_value, void* dst_key, void* dst_value,
                               const int64_t* block_pairs, int32_t num_pairs, int32_t src_num_blocks,
                               int32_t dst_num_blocks, int32_t num_kv_heads, int32_t head_dim, int32_t block_size,
                               int elt_bytes, int32_t* status, cudaStream_t stream);

// Causal attention of each sequence's new query tokens over its paged cache:
// the tcgen05 kernel where prefill_tc_serves() (chunks that fill its 128-row
// tiles), else the mma.sync kernel.
// With a workspace of prefill_workspace_bytes(p) bytes (scratch), the tcgen05
// kernel splits the items of its last, partial wave by key range and a second
// kernel merges the pieces.
cudaError_t launch_prefill(const PrefillParams& p, void* ws, size_t ws_bytes, pa_dtype dtype, cudaStream_t stream);
size_t prefill_workspace_bytes(const PrefillParams& p);
bool prefill_tc_serves(const PrefillParams& p);
size_t prefill_tc_workspace_bytes(const PrefillParams& p);
cudaError_t launch_prefill_tc(const PrefillParams& p, void* ws, size_t ws_bytes, pa_dtype dtype, cudaStream_t stream);

// TMA descriptor of a K or V pool viewed as 2-D: rows of head_dim elements,
// one row per (block, KV head, slot); a box is 16 rows (8 for 8-token blocks)
// x 64 elements (128 B), 128-byte swizzled in shared memory.
cudaError_t make_pool_map(CUtensorMap* map, const void* pool, pa_dtype dtype, int num_blocks, int num_kv_heads,
                          int head_dim, int block_size);

// Which main decode kernel serves a shape.
enum class DecodePath { kTensorCore, kSimt };
DecodePath decode_path(pa_dtype dtype, int head_dim, int group);

// Merge counters the workspace always reserves (at a fixed offset); problems
// with more (sequence, KV head) pairs than this use the plan kernel, which
// zeroes the counters it uses.
constexpr int kCounterSlots = 16384;

// Host-side scheduling choices of a decode call (pa_decode_tuning).
struct DecodeOptions {
    int shape = PA_SHAPE_AUTO;       // pa_decode_shape
    bool force_plan_kernel = false;  // the planning kernel even where attention CTAs could plan
    bool planned = false;            // the workspace holds this step's plan (pa_decode_plan): none is made
};

// [plan] + partition kernel + (if sequences span several partitions and the
// partition kernel does not merge them) reduce.
cudaError_t launch_decode(const DecodeParams& p, const DecodeOptions& o, pa_dtype dtype, cudaStream_t stream);

// The planning kernel alone: the work list of p's step into p's workspace
// (pa_decode_plan).  It reads context_lens and writes hdr, items and the
// zeroed merge counters.
cudaError_t launch_decode_plan(const DecodeParams& p, cudaStream_t stream);

// Number of kernels launch_decode enqueues for these sizes (p's pointers unused).
cudaError_t decode_launch_count(const DecodeParams& p, const DecodeOptions& o, pa_dtype dtype, int* launches);

// Most partitions per sequence that the attention kernel merges itself (more
// take the reduce kernel).
int decode_fused_max_parts();

// Every library kernel asks for the same (maximum) shared-memory carveout, so
// that SMs need not reconfigure L1/shared memory between chained kernels.
cudaError_t prefer_max_shared(const void* kernel);

// Launch with programmatic stream serialisation so a kernel's launch overlaps
// the tail of its predecessor; every kernel calls griddep_wait() before it
// touches memory a predecessor may write.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                       Args&&... args) {
    const cudaError_t ce = prefer_max_shared(reinterpret_cast<const void*>(kernel));
    if (ce != cudaSuccess) return ce;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

}  // namespace pa
