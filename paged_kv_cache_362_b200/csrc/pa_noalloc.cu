// pa_decode_noalloc: pa_decode for callers that cannot allocate device memory.
//
// pa_decode needs a scratch workspace (its work list and the per-partition
// partial results) that the caller allocates.  Some callers have no way to do
// that: code hosted inside an engine that owns all device memory and gives
// its extensions no allocator, or a latency-critical loop that must not call
// cudaMalloc (which can synchronise the device).  For them this entry point
// takes its scratch from a fixed array in the library's own device memory.
//
// The array is kStaticScratchBytes (32 MiB).  Every GPU on which the library's
// module is loaded holds it until the process exits.  Problems whose
// workspace (pa_decode_workspace_size) exceeds it are rejected.
//
// All calls share the one array; calls whose kernels overlap on the GPU (two
// streams, or two host threads) race on it and give wrong results.  The first
// call on a device zero-fills it (the state pa_decode asks of a fresh
// workspace: its merge counters at zero); every call that completes leaves
// them zeroed again.
#include <mutex>

#include "pa_internal.h"

namespace {

constexpr size_t kStaticScratchBytes = size_t(32) << 20;

// Scratch in the library's device memory.  In host code this name is only a
// host-side stand-in: its device address comes from cudaGetSymbolAddress.
static __device__ __align__(256) uint8_t g_decode_scratch[kStaticScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void* g_scratch_addr[kMaxDevices] = {};

// Device address of g_decode_scratch on the current device, resolved on the
// first call made with that device current.  That first call also zero-fills
// the array on `stream` and waits for it, so the state pa_decode expects of a
// fresh workspace does not rest on how the module was loaded.  A first call
// on a stream that is being captured into a graph could neither wait nor
// leave the fill out of the graph: it is refused (PA_ERR_INVALID_ARG) before
// anything is enqueued.
pa_status scratch_address(void** out, cudaStream_t stream) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return PA_ERR_CUDA;
    if (dev < 0 || dev >= kMaxDevices) return PA_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_mu);
    if (g_scratch_addr[dev] == nullptr) {
        cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
        if (cudaStreamIsCapturing(stream, &cs) != cudaSuccess) return PA_ERR_CUDA;
        if (cs != cudaStreamCaptureStatusNone) return PA_ERR_INVALID_ARG;
        cudaError_t e;
        void* p = nullptr;
        e = cudaGetSymbolAddress(&p, g_decode_scratch);
        if (e != cudaSuccess) return PA_ERR_CUDA;
        e = cudaMemsetAsync(p, 0, kStaticScratchBytes, stream);
        if (e != cudaSuccess) return PA_ERR_CUDA;
        e = cudaStreamSynchronize(stream);
        if (e != cudaSuccess) return PA_ERR_CUDA;
        g_scratch_addr[dev] = p;
    }
    *out = g_scratch_addr[dev];
    return PA_OK;
}

}  // namespace

extern "C" pa_status pa_decode_noalloc(void* out, const void* q, const void* key_cache, const void* value_cache,
                                       const int32_t* block_tables, int32_t max_blocks_per_seq,
                                       const int32_t* context_lens, int32_t num_seqs, int32_t num_heads,
                                       int32_t num_kv_heads, int32_t head_dim, int32_t block_size,
                                       int32_t num_blocks, float scale, int32_t max_context_len,
                                       int32_t partition_size, pa_dtype dtype, int32_t* status,
                                       pa_stream_t stream) {
    const size_t need = pa_decode_workspace_size(num_seqs, num_heads, num_kv_heads, head_dim, max_context_len,
                                                 partition_size);
    if (need == 0) return PA_ERR_INVALID_ARG;
    if (need > kStaticScratchBytes) return PA_ERR_UNSUPPORTED;  // problem too large for the fixed scratch
    void* scratch = nullptr;
    const pa_status st = scratch_address(&scratch, reinterpret_cast<cudaStream_t>(stream));
    if (st != PA_OK) return st;
    return pa_decode(out, q, key_cache, value_cache, block_tables, max_blocks_per_seq, context_lens, num_seqs,
                     num_heads, num_kv_heads, head_dim, block_size, num_blocks, scale, max_context_len,
                     partition_size, scratch, kStaticScratchBytes, dtype, status, stream);
}
