// Cache write (append) and copy-on-write block copy.
//
// reshape_and_cache: each decoded token appends one K/V entry inside the
// current logical block; the host picked the slot ("LLM Inference
// Visualizer", lesson 06, "How paging grows").
// copy_blocks: a shared block that a request is about to write is cloned into
// a fresh block first ("PagedAttention" digest, section "Copy-on-write: when
// two requests share a prefix").
//
// Both are pure data movement, bit-exact, in 16-byte vectors.  One thread
// moves one 16-byte chunk of K and the matching chunk of V; consecutive
// threads walk consecutive chunks of a row, so loads and stores coalesce.
#include <utility>

#include "pa_internal.h"

namespace pa {

// key/value [T, Hkv, D] -> pools [NB, Hkv, block_size, D];  chunk = 16 bytes
__global__ void __launch_bounds__(256) reshape_and_cache_kernel(
    const uint4* __restrict__ key, const uint4* __restrict__ value, uint4* __restrict__ key_cache,
    uint4* __restrict__ value_cache, const int64_t* __restrict__ slot_mapping, int64_t num_tokens,
    int num_kv_heads, int chunks_per_head, int block_size, int64_t num_slots, int32_t* status) {
    griddep_launch_dependents();
    griddep_wait();
    const int64_t chunks_per_token = (int64_t)num_kv_heads * chunks_per_head;
    const int64_t total = num_tokens * chunks_per_token;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < total;
         i += (int64_t)gridDim.x * blockDim.x) {
        const int64_t t = i / chunks_per_token;
        const int64_t r = i - t * chunks_per_token;        // = h * chunks_per_head + c
        const int64_t s = slot_mapping[t];
        if (s < 0) continue;                                // padding token
        if (s >= num_slots) {
            if (r == 0) set_status(status, PA_ERR_OUT_OF_RANGE);
            continue;
        }
        const int64_t blk = s / block_size, off = s % block_size;
        const int64_t h = r / chunks_per_head, c = r - h * chunks_per_head;
        const int64_t dst = ((blk * num_kv_heads + h) * block_size + off) * chunks_per_head + c;
        key_cache[dst] = key[i];
        value_cache[dst] = value[i];
    }
}

// one CTA per (pair, pool); the CTA moves the whole block in 16-byte chunks
__global__ void __launch_bounds__(256) copy_blocks_kernel(uint4* __restrict__ key_cache,
                                                          uint4* __restrict__ value_cache,
                                                          const int64_t* __restrict__ pairs, int num_pairs,
                                                          int64_t num_blocks, int64_t block_chunks,
                                                          int32_t* status) {
    griddep_launch_dependents();
    griddep_wait();
    const int k = blockIdx.x;
    if (k >= num_pairs) return;
    const int64_t src = pairs[2 * k], dst = pairs[2 * k + 1];
    if (src < 0 || src >= num_blocks || dst < 0 || dst >= num_blocks) {
        if (blockIdx.y == 0 && threadIdx.x == 0) set_status(status, PA_ERR_OUT_OF_RANGE);
        return;
    }
    uint4* pool = blockIdx.y == 0 ? key_cache : value_cache;
    const uint4* s = pool + src * block_chunks;
    uint4* d = pool + dst * block_chunks;
    for (int64_t i = threadIdx.x; i < block_chunks; i += blockDim.x) d[i] = s[i];
}

// Whole blocks between two pools of the same shape, either of which may be
// pinned host memory the device addresses (swap out / swap in).  Grid: (pair,
// K or V); 16-byte chunks, consecutive threads on consecutive chunks, so the
// transfers over PCIe are full 128-byte lines.
__global__ void __launch_bounds__(256) swap_blocks_kernel(const uint4* __restrict__ src_key,
                                                          const uint4* __restrict__ src_value,
                                                          uint4* __restrict__ dst_key, uint4* __restrict__ dst_value,
                                                          const int64_t* __restrict__ pairs, int num_pairs,
                                                          int64_t src_blocks, int64_t dst_blocks,
                                                          int64_t block_chunks, int32_t* status) {
    griddep_launch_dependents();
    griddep_wait();
    const int k = blockIdx.x;
    if (k >= num_pairs) return;
    const int64_t src = pairs[2 * k], dst = pairs[2 * k + 1];
    if (src < 0 || src >= src_blocks || dst < 0 || dst >= dst_blocks) {
        if (blockIdx.y == 0 && threadIdx.x == 0) set_status(status, PA_ERR_OUT_OF_RANGE);
        return;
    }
    const uint4* s = (blockIdx.y == 0 ? src_key : src_value) + src * block_chunks;
    uint4* d = (blockIdx.y == 0 ? dst_key : dst_value) + dst * block_chunks;
    for (int64_t i = threadIdx.x; i < block_chunks; i += blockDim.x) d[i] = s[i];
}

cudaError_t launch_reshape_and_cache(const void* key, const void* value, void* key_cache, void* value_cache,
                                     const int64_t* slot_mapping, int64_t num_tokens, int32_t num_blocks,
                                     int32_t num_kv_heads, int32_t head_dim, int32_t block_size, int elt_bytes,
                                     int32_t* status,
                                     cudaStream_t stream) {
    if (num_tokens == 0) return cudaSuccess;
    DeviceInfo dev;
    cudaError_t e = device_info(&dev);
    if (e != cudaSuccess) return e;
    const int chunks_per_head = head_dim * elt_bytes / 16;
    const int64_t total = num_tokens * num_kv_heads * chunks_per_head;
    const int64_t want = (total + 255) / 256;
    const int64_t cap = (int64_t)dev.sm_count * 16;
    const int grid = (int)(want < cap ? want : cap);
    return launch_pdl(reshape_and_cache_kernel, dim3(grid), dim3(256), 0, stream,
                      static_cast<const uint4*>(key), static_cast<const uint4*>(value),
                      static_cast<uint4*>(key_cache), static_cast<uint4*>(value_cache), slot_mapping, num_tokens,
                      (int)num_kv_heads, chunks_per_head, (int)block_size, (int64_t)num_blocks * block_size, status);
}

cudaError_t launch_copy_blocks(void* key_cache, void* value_cache, const int64_t* block_pairs, int32_t num_pairs,
                               int32_t num_blocks, int32_t num_kv_heads, int32_t head_dim, int32_t block_size,
                               int elt_bytes, int32_t* status, cudaStream_t stream) {
    if (num_pairs == 0) return cudaSuccess;
    const int64_t block_chunks = (int64_t)num_kv_heads * block_size * head_dim * elt_bytes / 16;
    return launch_pdl(copy_blocks_kernel, dim3(num_pairs, 2), dim3(256), 0, stream,
                      static_cast<uint4*>(key_cache), static_cast<uint4*>(value_cache), block_pairs, (int)num_pairs,
                      (int64_t)num_blocks, block_chunks, status);
}

cudaError_t launch_swap_blocks(const void* src_key, const void* src_value, void* dst_key, void* dst_value,
                               const int64_t* block_pairs, int32_t num_pairs, int32_t src_num_blocks,
                               int32_t dst_num_blocks, int32_t num_kv_heads, int32_t head_dim, int32_t block_size,
                               int elt_bytes, int32_t* status, cudaStream_t stream) {
    if (num_pairs == 0) return cudaSuccess;
    const int64_t block_chunks = (int64_t)num_kv_heads * block_size * head_dim * elt_bytes / 16;
    return launch_pdl(swap_blocks_kernel, dim3(num_pairs, 2), dim3(256), 0, stream,
                      static_cast<const uint4*>(src_key), static_cast<const uint4*>(src_value),
                      static_cast<uint4*>(dst_key), static_cast<uint4*>(dst_value), block_pairs, (int)num_pairs,
                      (int64_t)src_num_blocks, (int64_t)dst_num_blocks, block_chunks, status);
}

}  // namespace pa
