// C ABI of the library: host-side argument checks, workspace layout, launches.
// See include/pa.h for the contract of every entry point.
#include <cmath>
#include <cstdint>
#include <mutex>

#include "pa_internal.h"

namespace pa {

cudaError_t device_info(DeviceInfo* out) {
    static DeviceInfo cache[64];
    static bool have[64] = {};
    static std::mutex mu;
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(mu);
    if (!have[dev]) {
        DeviceInfo d{};
        e = cudaDeviceGetAttribute(&d.sm_count, cudaDevAttrMultiProcessorCount, dev);
        if (e != cudaSuccess) return e;
        e = cudaDeviceGetAttribute(&d.max_smem_optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
        if (e != cudaSuccess) return e;
        cache[dev] = d;
        have[dev] = true;
    }
    *out = cache[dev];
    return cudaSuccess;
}

cudaError_t prefer_max_shared(const void* kernel) {
    static std::mutex mu;
    static const void* done[256];
    static int n = 0;
    std::lock_guard<std::mutex> lock(mu);
    for (int i = 0; i < n; ++i)
        if (done[i] == kernel) return cudaSuccess;
    const cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributePreferredSharedMemoryCarveout,
                                               cudaSharedmemCarveoutMaxShared);
    if (e != cudaSuccess) return e;
    if (n < 256) done[n++] = kernel;
    return cudaSuccess;
}

namespace {

int elt_bytes(pa_dtype d) { return d == PA_F32 ? 4 : 2; }
bool valid_dtype(int d) { return d == PA_F32 || d == PA_F16 || d == PA_BF16; }
bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }
int64_t ceil_div64(int64_t a, int64_t b) { return (a + b - 1) / b; }

// Partition size when the caller passes 0.  First the largest of
// 512/256/128/64 tokens that still yields enough (sequence, partition, KV
// head) items, at the batch's longest context, to keep every SM of a B200
// busy several times over (8 per SM).  If that splits the longest context
// into more partitions than the attention kernel merges itself, the smallest
// size that stays within that limit is taken instead, provided it still
// fills one wave of CTAs (4 per SM): one launch instead of an extra reduce
// kernel, measured 6% faster for 32 sequences of up to 2048 tokens.
//
// The SM count is the current device's (148 on a B200, also the value taken
// when no device can be queried); pa_decode_workspace_size and pa_decode
// therefore agree as long as they are called with the same device current.
int64_t current_sm_count() {
    DeviceInfo d;
    return device_info(&d) == cudaSuccess && d.sm_count > 0 ? d.sm_count : 148;
}

int auto_partition_size(int64_t num_seqs, int64_t num_kv_heads, int64_t max_context_len) {
    const int64_t sms = current_sm_count();
    auto items = [&](int P) { return num_seqs * num_kv_heads * ceil_div64(max_context_len, P); };
    int P = 512;
    while (P > 64 && items(P) < 8 * sms) P /= 2;
    const int64_t fused = decode_fused_max_parts();
    if (ceil_div64(max_context_len, P) > fused) {
        int Pf = P;
        while (Pf < 512 && ceil_div64(max_context_len, Pf) > fused) Pf *= 2;
        if (ceil_div64(max_context_len, Pf) <= fused && items(Pf) >= 4 * sms) P = Pf;
    }
    return P;
}

// Options of pa_decode_tuned: NULL (or all zero) gives the defaults.
bool decode_options(const pa_decode_tuning* t, DecodeOptions* o, int* equal_split, int* class_first,
                    uint64_t* wait_limit_ns, int* stall) {
    *o = DecodeOptions{};
    *equal_split = 0;
    *class_first = 1;
    *wait_limit_ns = kWaitLimitNs;
    *stall = 0;
    if (t == nullptr) return true;
    if (t->shape < PA_SHAPE_AUTO || t->shape > PA_SHAPE_PAIR1) return false;
    if ((t->planner | t->split | t->order | t->stall_first_item) & ~1) return false;
    if (t->wait_limit_ns < 0) return false;
    o->shape = t->shape;
    o->force_plan_kernel = t->planner == 1;
    *equal_split = t->split;
    *class_first = t->order == 0 ? 1 : 0;
    if (t->wait_limit_ns > 0) *wait_limit_ns = (uint64_t)t->wait_limit_ns;
    *stall = t->stall_first_item;
    return true;
}

// Workspace: a 256-byte header (the plan kernel's list length), the merge
// counters, the work list, then the partitions' (m, l, O).  The merge counters
// sit at the same place for every problem, in a region of at least
// kCounterSlots entries, so a workspace reused for problems of another shape
// still finds them zeroed: every call leaves its counters at zero, and no
// other region ever overlaps the first kCounterSlots.
struct WsLayout {
    int partition_size, max_parts;
    int64_t max_items;
    size_t off_items, off_cnt, off_m, off_l, off_o, total;
};

bool ws_layout(int64_t num_seqs, int64_t num_heads, int64_t num_kv_heads, int64_t head_dim,
               int64_t max_context_len, int64_t partition_size, WsLayout* w) {
    if (num_seqs < 0 || num_heads <= 0 || num_kv_heads <= 0 || head_dim <= 0 || max_context_len < 0) return false;
    if (partition_size == 0) partition_size = auto_partition_size(num_seqs, num_kv_heads, max_context_len);
    if (partition_size < kChunk || partition_size > kChunk * kMaxPartBlocks || partition_size % kChunk != 0)
        return false;
    const int64_t np = std::max<int64_t>(1, ceil_div64(max_context_len, partition_size));
    w->partition_size = (int)partition_size;
    w->max_parts = (int)np;
    w->max_items = num_seqs * np * num_kv_heads;
    const int64_t parts = np > 1 ? num_seqs * num_heads * np : 0;
    w->off_cnt = 256;
    const int64_t counters = std::max<int64_t>(kCounterSlots, num_seqs * num_kv_heads);
    w->off_items = round_up(w->off_cnt + (size_t)counters * sizeof(int32_t), 256);
    w->off_m = round_up(w->off_items + (size_t)w->max_items * sizeof(int4), 256);
    w->off_l = round_up(w->off_m + (size_t)parts * sizeof(float), 256);
    w->off_o = round_up(w->off_l + (size_t)parts * sizeof(float), 256);
    w->total = round_up(w->off_o + (size_t)parts * head_dim * sizeof(float), 256);
    return true;
}

}  // namespace
}  // namespace pa

using namespace pa;

extern "C" {

pa_status pa_reshape_and_cache(const void* key, const void* value, void* key_cache, void* value_cache,
                               const int64_t* slot_mapping, int64_t num_tokens, int32_t num_blocks,
                               int32_t num_kv_heads, int32_t head_dim, int32_t block_size, pa_dtype dtype,
                               int32_t* status, pa_stream_t stream) {
    if (num_tokens < 0 || num_blocks <= 0 || num_kv_heads <= 0 || head_dim <= 0) return PA_ERR_INVALID_ARG;
    if (!valid_dtype(dtype)) return PA_ERR_INVALID_ARG;
    if (!block_size_supported(block_size) || (head_dim != 64 && head_dim != 128)) return PA_ERR_UNSUPPORTED;
    if (num_tokens == 0) return PA_OK;
    if (!key || !value || !key_cache || !value_cache || !slot_mapping) return PA_ERR_INVALID_ARG;
    if (!aligned16(key) || !aligned16(value) || !aligned16(key_cache) || !aligned16(value_cache))
        return PA_ERR_INVALID_ARG;
    const cudaError_t e = launch_reshape_and_cache(key, value, key_cache, value_cache, slot_mapping, num_tokens,
                                                   num_blocks, num_kv_heads, head_dim, block_size, elt_bytes(dtype), status,
                                                   reinterpret_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? PA_OK : PA_ERR_CUDA;
}

size_t pa_decode_workspace_size(int32_t num_seqs, int32_t num_heads, int32_t num_kv_heads, int32_t head_dim,
                                int32_t max_context_len, int32_t partition_size) {
    WsLayout w;
    if (!ws_layout(num_seqs, num_heads, num_kv_heads, head_dim, max_context_len, partition_size, &w)) return 0;
    return w.total;
}

pa_status pa_decode(void* out, const void* q, const void* key_cache, const void* value_cache,
                    const int32_t* block_tables, int32_t max_blocks_per_seq, const int32_t* context_lens,
                    int32_t num_seqs, int32_t num_heads, int32_t num_kv_heads, int32_t head_dim,
                    int32_t block_size, int32_t num_blocks, float scale, int32_t max_context_len,
                    int32_t partition_size, void* workspace, size_t workspace_bytes, pa_dtype dtype,
                    int32_t* status, pa_stream_t stream) {
    return pa_decode_tuned(out, q, key_cache, value_cache, block_tables, max_blocks_per_seq, context_lens, num_seqs,
                           num_heads, num_kv_heads, head_dim, block_size, num_blocks, scale, max_context_len,
                           partition_size, workspace, workspace_bytes, dtype, status, stream, nullptr);
}

namespace {
// pa_decode_tuned and pa_decode_planned: validation, parameters, launch
// (planned: the workspace holds the step's plan, from pa_decode_plan).
pa_status decode_impl(void* out, const void* q, const void* key_cache, const void* value_cache,
                      const int32_t* block_tables, int32_t max_blocks_per_seq, const int32_t* context_lens,
                      int32_t num_seqs, int32_t num_heads, int32_t num_kv_heads, int32_t head_dim, int32_t block_size,
                      int32_t num_blocks, float scale, int32_t max_context_len, int32_t partition_size,
                      void* workspace, size_t workspace_bytes, pa_dtype dtype, int32_t* status, pa_stream_t stream,
                      const pa_decode_tuning* tuning, bool planned) {
    DecodeOptions opt;
    int equal_split = 0, class_first = 1, stall = 0;
    uint64_t wait_limit = kWaitLimitNs;
    if (!decode_options(tuning, &opt, &equal_split, &class_first, &wait_limit, &stall)) return PA_ERR_INVALID_ARG;
    opt.planned = planned;
    if (num_seqs < 0 || num_heads <= 0 || num_kv_heads <= 0 || head_dim <= 0 || num_blocks <= 0 ||
        max_blocks_per_seq <= 0 || max_context_len < 0)
        return PA_ERR_INVALID_ARG;
    if (!valid_dtype(dtype) || !std::isfinite(scale)) return PA_ERR_INVALID_ARG;
    if (num_heads % num_kv_heads != 0) return PA_ERR_INVALID_ARG;
    if (!block_size_supported(block_size) || (head_dim != 64 && head_dim != 128) || num_kv_heads > 255)
        return PA_ERR_UNSUPPORTED;
    if (partition_size != 0 &&
        (partition_size < kChunk || partition_size > kChunk * kMaxPartBlocks || partition_size % kChunk))
        return PA_ERR_INVALID_ARG;
    if ((int64_t)num_blocks * num_kv_heads * block_size > INT32_MAX) return PA_ERR_UNSUPPORTED;
    if (num_seqs == 0) return PA_OK;
    if (!out || !q || !key_cache || !value_cache || !block_tables || !context_lens || !workspace)
        return PA_ERR_INVALID_ARG;
    if (!aligned16(out) || !aligned16(q) || !aligned16(key_cache) || !aligned16(value_cache) ||
        (reinterpret_cast<uintptr_t>(workspace) & 255u))
        return PA_ERR_INVALID_ARG;
    WsLayout w;
    if (!ws_layout(num_seqs, num_heads, num_kv_heads, head_dim, max_context_len, partition_size, &w))
        return PA_ERR_INVALID_ARG;
    if (workspace_bytes < w.total) return PA_ERR_INVALID_ARG;
    if (w.max_items > INT32_MAX) return PA_ERR_UNSUPPORTED;

    DecodeParams p{};
    p.out = out;
    p.q = q;
    p.key_cache = key_cache;
    p.value_cache = value_cache;
    p.block_tables = block_tables;
    p.context_lens = context_lens;
    p.status = status;
    p.num_seqs = num_seqs;
    p.num_heads = num_heads;
    p.num_kv_heads = num_kv_heads;
    p.head_dim = head_dim;
    p.group = num_heads / num_kv_heads;
    p.max_blocks_per_seq = max_blocks_per_seq;
    p.num_blocks = num_blocks;
    p.block_size = block_size;
    p.ctx_cap = (int)std::min<int64_t>(max_context_len, (int64_t)max_blocks_per_seq * block_size);
    p.part_blocks = w.partition_size / kChunk;
    p.max_parts = w.max_parts;
    p.scale_log2 = scale * 1.4426950408889634f;  // log2(e)
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    p.hdr = reinterpret_cast<int32_t*>(ws);
    p.merge_count = reinterpret_cast<int32_t*>(ws + w.off_cnt);
    p.items = reinterpret_cast<int4*>(ws + w.off_items);
    p.part_m = reinterpret_cast<float*>(ws + w.off_m);
    p.part_l = reinterpret_cast<float*>(ws + w.off_l);
    p.part_o = reinterpret_cast<float*>(ws + w.off_o);
    p.equal_split = equal_split;
    p.class_first = class_first;
    p.wait_limit_ns = wait_limit;
    p.stall_first_item = stall;
    const cudaError_t e = launch_decode(p, opt, dtype, reinterpret_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? PA_OK : PA_ERR_CUDA;
}
}  // namespace

pa_status pa_decode_tuned(void* out, const void* q, const void* key_cache, const void* value_cache,
                          const int32_t* block_tables, int32_t max_blocks_per_seq, const int32_t* context_lens,
                          int32_t num_seqs, int32_t num_heads, int32_t num_kv_heads, int32_t head_dim,
                          int32_t block_size, int32_t num_blocks, float scale, int32_t max_context_len,
                          int32_t partition_size, void* workspace, size_t workspace_bytes, pa_dtype dtype,
                          int32_t* status, pa_stream_t stream, const pa_decode_tuning* tuning) {
    return decode_impl(out, q, key_cache, value_cache, block_tables, max_blocks_per_seq, context_lens, num_seqs,
                       num_heads, num_kv_heads, head_dim, block_size, num_blocks, scale, max_context_len,
                       partition_size, workspace, workspace_bytes, dtype, status, stream, tuning, false);
}

pa_status pa_decode_planned(void* out, const void* q, const void* key_cache, const void* value_cache,
                            const int32_t* block_tables, int32_t max_blocks_per_seq, const int32_t* context_lens,
                            int32_t num_seqs, int32_t num_heads, int32_t num_kv_heads, int32_t head_dim,
                            int32_t block_size, int32_t num_blocks, float scale, int32_t max_context_len,
                            int32_t partition_size, void* workspace, size_t workspace_bytes, pa_dtype dtype,
                            int32_t* status, pa_stream_t stream) {
    return decode_impl(out, q, key_cache, value_cache, block_tables, max_blocks_per_seq, context_lens, num_seqs,
                       num_heads, num_kv_heads, head_dim, block_size, num_blocks, scale, max_context_len,
                       partition_size, workspace, workspace_bytes, dtype, status, stream, nullptr, true);
}

pa_status pa_decode_plan(const int32_t* context_lens, int32_t num_seqs, int32_t num_heads, int32_t num_kv_heads,
                         int32_t head_dim, int32_t block_size, int32_t max_blocks_per_seq, int32_t max_context_len,
                         int32_t partition_size, void* workspace, size_t workspace_bytes, int32_t* status,
                         pa_stream_t stream) {
    if (num_seqs < 0 || num_heads <= 0 || num_kv_heads <= 0 || head_dim <= 0 || max_blocks_per_seq <= 0 ||
        max_context_len < 0)
        return PA_ERR_INVALID_ARG;
    if (num_heads % num_kv_heads != 0) return PA_ERR_INVALID_ARG;
    if (!block_size_supported(block_size) || (head_dim != 64 && head_dim != 128) || num_kv_heads > 255)
        return PA_ERR_UNSUPPORTED;
    if (partition_size != 0 &&
        (partition_size < kChunk || partition_size > kChunk * kMaxPartBlocks || partition_size % kChunk))
        return PA_ERR_INVALID_ARG;
    if (num_seqs == 0) return PA_OK;
    if (!context_lens || !workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u)) return PA_ERR_INVALID_ARG;
    WsLayout w;
    if (!ws_layout(num_seqs, num_heads, num_kv_heads, head_dim, max_context_len, partition_size, &w))
        return PA_ERR_INVALID_ARG;
    if (workspace_bytes < w.total) return PA_ERR_INVALID_ARG;
    if (w.max_items > INT32_MAX) return PA_ERR_UNSUPPORTED;
    // what the planning kernel reads and writes: the lengths, the partition
    // geometry (default split and order, as pa_decode_planned uses) and the workspace
    DecodeParams p{};
    p.context_lens = context_lens;
    p.status = status;
    p.num_seqs = num_seqs;
    p.num_heads = num_heads;
    p.num_kv_heads = num_kv_heads;
    p.head_dim = head_dim;
    p.group = num_heads / num_kv_heads;
    p.max_blocks_per_seq = max_blocks_per_seq;
    p.block_size = block_size;
    p.ctx_cap = (int)std::min<int64_t>(max_context_len, (int64_t)max_blocks_per_seq * block_size);
    p.part_blocks = w.partition_size / kChunk;
    p.max_parts = w.max_parts;
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    p.hdr = reinterpret_cast<int32_t*>(ws);
    p.merge_count = reinterpret_cast<int32_t*>(ws + w.off_cnt);
    p.items = reinterpret_cast<int4*>(ws + w.off_items);
    p.part_m = reinterpret_cast<float*>(ws + w.off_m);
    p.part_l = reinterpret_cast<float*>(ws + w.off_l);
    p.part_o = reinterpret_cast<float*>(ws + w.off_o);
    p.equal_split = 0;
    p.class_first = 1;
    const cudaError_t e = launch_decode_plan(p, reinterpret_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? PA_OK : PA_ERR_CUDA;
}

int32_t pa_decode_launch_count(int32_t num_seqs, int32_t num_heads, int32_t num_kv_heads, int32_t head_dim,
                               int32_t max_context_len, int32_t partition_size, pa_dtype dtype) {
    return pa_decode_launch_count_tuned(num_seqs, num_heads, num_kv_heads, head_dim, max_context_len, partition_size,
                                        dtype, nullptr);
}

namespace {
int32_t launch_count(int32_t num_seqs, int32_t num_heads, int32_t num_kv_heads, int32_t head_dim,
                     int32_t max_context_len, int32_t partition_size, pa_dtype dtype, const pa_decode_tuning* tuning,
                     bool planned) {
    DecodeOptions opt;
    int equal_split = 0, class_first = 1, stall = 0;
    uint64_t wait_limit = kWaitLimitNs;
    if (!decode_options(tuning, &opt, &equal_split, &class_first, &wait_limit, &stall)) return -1;
    opt.planned = planned;
    if (num_seqs <= 0 || num_heads <= 0 || num_kv_heads <= 0 || num_heads % num_kv_heads != 0) return -1;
    if (!valid_dtype(dtype) || (head_dim != 64 && head_dim != 128) || num_kv_heads > 255) return -1;
    WsLayout w;
    if (!ws_layout(num_seqs, num_heads, num_kv_heads, head_dim, max_context_len, partition_size, &w)) return -1;
    if (w.max_items > INT32_MAX) return -1;
    DecodeParams p{};
    p.num_seqs = num_seqs;
    p.num_heads = num_heads;
    p.num_kv_heads = num_kv_heads;
    p.head_dim = head_dim;
    p.group = num_heads / num_kv_heads;
    p.part_blocks = w.partition_size / kChunk;
    p.max_parts = w.max_parts;
    int n = 0;
    return decode_launch_count(p, opt, dtype, &n) == cudaSuccess ? n : -1;
}
}  // namespace

int32_t pa_decode_launch_count_tuned(int32_t num_seqs, int32_t num_heads, int32_t num_kv_heads, int32_t head_dim,
                                     int32_t max_context_len, int32_t partition_size, pa_dtype dtype,
                                     const pa_decode_tuning* tuning) {
    return launch_count(num_seqs, num_heads, num_kv_heads, head_dim, max_context_len, partition_size, dtype, tuning,
                        false);
}

int32_t pa_decode_planned_launch_count(int32_t num_seqs, int32_t num_heads, int32_t num_kv_heads, int32_t head_dim,
                                       int32_t max_context_len, int32_t partition_size, pa_dtype dtype) {
    return launch_count(num_seqs, num_heads, num_kv_heads, head_dim, max_context_len, partition_size, dtype, nullptr,
                        true);
}

pa_status pa_copy_blocks(void* key_cache, void* value_cache, const int64_t* block_pairs, int32_t num_pairs,
                         int32_t num_blocks, int32_t num_kv_heads, int32_t head_dim, int32_t block_size,
                         pa_dtype dtype, int32_t* status, pa_stream_t stream) {
    if (num_pairs < 0 || num_blocks <= 0 || num_kv_heads <= 0 || head_dim <= 0) return PA_ERR_INVALID_ARG;
    if (!valid_dtype(dtype)) return PA_ERR_INVALID_ARG;
    if (!block_size_supported(block_size) || (head_dim != 64 && head_dim != 128)) return PA_ERR_UNSUPPORTED;
    if (num_pairs == 0) return PA_OK;
    if (!key_cache || !value_cache || !block_pairs) return PA_ERR_INVALID_ARG;
    if (!aligned16(key_cache) || !aligned16(value_cache)) return PA_ERR_INVALID_ARG;
    const cudaError_t e = launch_copy_blocks(key_cache, value_cache, block_pairs, num_pairs, num_blocks,
                                             num_kv_heads, head_dim, block_size, elt_bytes(dtype), status,
                                             reinterpret_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? PA_OK : PA_ERR_CUDA;
}

namespace {
// Validates pa_prefill's sizes and fills the kernel parameters (pointers are
// checked by the callers, which know whether the call has work to do).
pa_status prefill_params(PrefillParams* p, int32_t max_blocks_per_seq, int32_t num_seqs, int32_t num_heads,
                         int32_t num_kv_heads, int32_t head_dim, int32_t block_size, int32_t num_blocks, float scale,
                         int32_t max_query_len, pa_dtype dtype) {
    if (num_seqs < 0 || num_heads <= 0 || num_kv_heads <= 0 || head_dim <= 0 || num_blocks <= 0 ||
        max_blocks_per_seq <= 0 || max_query_len < 0)
        return PA_ERR_INVALID_ARG;
    if (!valid_dtype(dtype) || !std::isfinite(scale) || num_heads % num_kv_heads != 0) return PA_ERR_INVALID_ARG;
    if (block_size != kChunk || (head_dim != 64 && head_dim != 128) || dtype == PA_F32 ||
        num_heads / num_kv_heads > 16)
        return PA_ERR_UNSUPPORTED;
    // pool rows (blocks x KV heads x 16) index the tensor copies in int32
    if ((int64_t)num_blocks * num_kv_heads * kChunk > INT32_MAX) return PA_ERR_UNSUPPORTED;
    *p = PrefillParams{};
    p->num_seqs = num_seqs;
    p->num_heads = num_heads;
    p->num_kv_heads = num_kv_heads;
    p->head_dim = head_dim;
    p->group = num_heads / num_kv_heads;
    p->max_blocks_per_seq = max_blocks_per_seq;
    p->num_blocks = num_blocks;
    p->max_query_len = max_query_len;
    p->scale_log2 = scale * 1.4426950408889634f;  // log2(e)
    return PA_OK;
}

pa_status prefill_impl(void* out, const void* q, const void* key_cache, const void* value_cache,
                       const int32_t* block_tables, int32_t max_blocks_per_seq, const int32_t* query_start,
                       const int32_t* context_lens, int32_t num_seqs, int32_t num_heads, int32_t num_kv_heads,
                       int32_t head_dim, int32_t block_size, int32_t num_blocks, float scale, int32_t max_query_len,
                       bool with_ws, void* workspace, size_t workspace_bytes, pa_dtype dtype, int32_t* status,
                       pa_stream_t stream) {
    PrefillParams p;
    const pa_status v = prefill_params(&p, max_blocks_per_seq, num_seqs, num_heads, num_kv_heads, head_dim,
                                       block_size, num_blocks, scale, max_query_len, dtype);
    if (v != PA_OK) return v;
    if (num_seqs == 0 || max_query_len == 0) return PA_OK;
    if (!out || !q || !key_cache || !value_cache || !block_tables || !query_start || !context_lens)
        return PA_ERR_INVALID_ARG;
    if (!aligned16(out) || !aligned16(q) || !aligned16(key_cache) || !aligned16(value_cache))
        return PA_ERR_INVALID_ARG;
    if (with_ws) {
        const size_t need = prefill_workspace_bytes(p);
        if (need > 0 && (!workspace || workspace_bytes < need || !aligned16(workspace))) return PA_ERR_INVALID_ARG;
    }
    p.out = out;
    p.q = q;
    p.key_cache = key_cache;
    p.value_cache = value_cache;
    p.block_tables = block_tables;
    p.query_start = query_start;
    p.context_lens = context_lens;
    p.status = status;
    const cudaError_t e = launch_prefill(p, with_ws ? workspace : nullptr, with_ws ? workspace_bytes : 0, dtype,
                                         reinterpret_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? PA_OK : PA_ERR_CUDA;
}
}  // namespace

pa_status pa_prefill(void* out, const void* q, const void* key_cache, const void* value_cache,
                     const int32_t* block_tables, int32_t max_blocks_per_seq, const int32_t* query_start,
                     const int32_t* context_lens, int32_t num_seqs, int32_t num_heads, int32_t num_kv_heads,
                     int32_t head_dim, int32_t block_size, int32_t num_blocks, float scale, int32_t max_query_len,
                     pa_dtype dtype, int32_t* status, pa_stream_t stream) {
    return prefill_impl(out, q, key_cache, value_cache, block_tables, max_blocks_per_seq, query_start, context_lens,
                        num_seqs, num_heads, num_kv_heads, head_dim, block_size, num_blocks, scale, max_query_len,
                        false, nullptr, 0, dtype, status, stream);
}

pa_status pa_prefill_workspace_size(int32_t num_seqs, int32_t num_heads, int32_t num_kv_heads, int32_t head_dim,
                                    int32_t max_query_len, pa_dtype dtype, size_t* bytes) {
    if (!bytes) return PA_ERR_INVALID_ARG;
    PrefillParams p;
    const pa_status v = prefill_params(&p, 1, num_seqs, num_heads, num_kv_heads, head_dim, kChunk, 1, 1.f,
                                       max_query_len, dtype);
    if (v != PA_OK) return v;
    *bytes = (num_seqs == 0 || max_query_len == 0) ? 0 : prefill_workspace_bytes(p);
    return PA_OK;
}

pa_status pa_prefill_ws(void* out, const void* q, const void* key_cache, const void* value_cache,
                        const int32_t* block_tables, int32_t max_blocks_per_seq, const int32_t* query_start,
                        const int32_t* context_lens, int32_t num_seqs, int32_t num_heads, int32_t num_kv_heads,
                        int32_t head_dim, int32_t block_size, int32_t num_blocks, float scale, int32_t max_query_len,
                        void* workspace, size_t workspace_bytes, pa_dtype dtype, int32_t* status,
                        pa_stream_t stream) {
    return prefill_impl(out, q, key_cache, value_cache, block_tables, max_blocks_per_seq, query_start, context_lens,
                        num_seqs, num_heads, num_kv_heads, head_dim, block_size, num_blocks, scale, max_query_len,
                        true, workspace, workspace_bytes, dtype, status, stream);
}

pa_status pa_swap_blocks(const void* src_key_cache, const void* src_value_cache, void* dst_key_cache,
                         void* dst_value_cache, const int64_t* block_pairs, int32_t num_pairs, int32_t src_num_blocks,
                         int32_t dst_num_blocks, int32_t num_kv_heads, int32_t head_dim, int32_t block_size,
                         pa_dtype dtype, int32_t* status, pa_stream_t stream) {
    if (num_pairs < 0 || src_num_blocks <= 0 || dst_num_blocks <= 0 || num_kv_heads <= 0 || head_dim <= 0)
        return PA_ERR_INVALID_ARG;
    if (!valid_dtype(dtype)) return PA_ERR_INVALID_ARG;
    if (!block_size_supported(block_size) || (head_dim != 64 && head_dim != 128)) return PA_ERR_UNSUPPORTED;
    if (num_pairs == 0) return PA_OK;
    if (!src_key_cache || !src_value_cache || !dst_key_cache || !dst_value_cache || !block_pairs)
        return PA_ERR_INVALID_ARG;
    if (!aligned16(src_key_cache) || !aligned16(src_value_cache) || !aligned16(dst_key_cache) ||
        !aligned16(dst_value_cache))
        return PA_ERR_INVALID_ARG;
    const cudaError_t e = launch_swap_blocks(src_key_cache, src_value_cache, dst_key_cache, dst_value_cache,
                                             block_pairs, num_pairs, src_num_blocks, dst_num_blocks, num_kv_heads,
                                             head_dim, block_size, elt_bytes(dtype), status,
                                             reinterpret_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? PA_OK : PA_ERR_CUDA;
}

const char* pa_get_error_string(pa_status s) {
    const int v = (int)s;
    if (v == PA_OK) return "PA_OK";
    if (v & PA_ERR_INVALID_ARG) return "PA_ERR_INVALID_ARG: invalid argument";
    if (v & PA_ERR_UNSUPPORTED) return "PA_ERR_UNSUPPORTED: configuration not supported";
    if (v & PA_ERR_OUT_OF_RANGE) return "PA_ERR_OUT_OF_RANGE: block id, slot or context length out of range";
    if (v & PA_ERR_CUDA) return "PA_ERR_CUDA: CUDA launch or query failed";
    if (v & PA_ERR_TIMEOUT) return "PA_ERR_TIMEOUT: bounded wait inside a kernel expired";
    if (v & PA_ERR_NO_BLOCKS) return "PA_ERR_NO_BLOCKS: not enough free blocks in the pool";
    return "unknown pa_status";
}

int32_t pa_version(void) { return 100; }

}  // extern "C"
