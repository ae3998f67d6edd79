// Internal launch interface between the C ABI (pa_api.cu) and the kernels.
#pragma once

#include <cuda_runtime.h>

#include "pa_common.cuh"

namespace pa {

// Device properties the launchers need (cached per device).
struct DeviceInfo {
    int sm_count;
    int max_smem_optin;
};
cudaError_t device_info(DeviceInfo* out);

cudaError_t launch_reshape_and_cache(const void* key, const void* value, void* key_cache, void* value_cache,
                                     const int64_t* slot_mapping, int64_t num_tokens, int32_t num_blocks,
                                     int32_t num_kv_heads, int32_t head_dim, int elt_bytes, int32_t* status,
                                     cudaStream_t stream);

cudaError_t launch_copy_blocks(void* key_cache, void* value_cache, const int64_t* block_pairs, int32_t num_pairs,
                               int32_t num_blocks, int32_t num_kv_heads, int32_t head_dim, int elt_bytes,
                               int32_t* status, cudaStream_t stream);

// Which main decode kernel serves a shape.
enum class DecodePath { kTensorCore, kSimt };
DecodePath decode_path(pa_dtype dtype, int head_dim, int group);

// Plan + partition kernel + (if any sequence spans several partitions) reduce.
cudaError_t launch_decode(const DecodeParams& p, pa_dtype dtype, cudaStream_t stream);

// Launch with programmatic stream serialisation so a kernel's launch overlaps
// the tail of its predecessor; every kernel calls griddep_wait() before it
// touches memory a predecessor may write.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                       Args&&... args) {
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
