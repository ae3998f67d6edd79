// Paged prefill on sm_100a: causal attention of a chunk of new query tokens
// over everything a sequence has in the paged KV cache.
//
// What is computed (the same attention as decode, for many query positions:
// "PagedAttention" digest, sections "PagedAttention in one picture" and "Why
// the attention kernel works at all"; the cache is read block by block
// through the table): for sequence b with n = context_lens[b] tokens in the
// cache, of which the last L = query_start[b+1] - query_start[b] are the new
// ones, query row i < L sits at position p = n - L + i and attends to the
// keys at positions 0 .. p:
//     out[query_start[b] + i][h] = sum_{j <= p} softmax_j(scale * q . K_j) V_j
// with K_j, V_j of KV head h / G.  The new tokens' K/V must already be in the
// cache (pa_reshape_and_cache).
//
// Blocks of 16 tokens (the block size of the pages' default).
//
// How: one CTA per (16-query tile, KV head, sequence), one warp per query
// head of the GQA group, so each K/V block is loaded once into shared memory
// (cp.async, a ring of kStages blocks) for all G heads and 16 queries.  Per block a
// warp computes S = Q K^T (m16n8k16: 16 queries x 16 keys, two n-tiles), the
// causal mask on the diagonal blocks, an online softmax per query row in fp32
// (2^x on log2-scaled logits), and O += P V with the S accumulators reused as
// the A operand (bf16 P carried as a hi + lo pair, as in decode).
#include <type_traits>

#include "pa_internal.h"

namespace pa {

namespace {

constexpr float kNegInfP = -__builtin_huge_valf();
constexpr int kQTile = 16;
// K/V blocks in flight per CTA.  Registers hold a CTA of G <= 16 warps to
// about 2 per SM, so each CTA hides its own load latency: a block is
// requested kStages - 1 steps before it is used.
constexpr int kStages = 4;

template <int N>
__device__ __forceinline__ void cp_async_wait_pending() {
    asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

template <int D>
struct PrefillCfg {
    static constexpr int kRow = D + 8;                 // padded smem row (halves): conflict-free ldmatrix
    static constexpr int kTileBytes = kChunk * kRow * 2;
    static constexpr int kQBytes = kQTile * kRow * 2;  // one head's query tile
};

template <typename T, int D>
__global__ void __launch_bounds__(16 * 32) prefill_kernel(PrefillParams p) {
    using C = PrefillCfg<D>;
    extern __shared__ __align__(16) uint8_t smem[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nthr = blockDim.x;
    const int G = p.group, b = blockIdx.z, g = blockIdx.y, i0 = blockIdx.x * kQTile;
    griddep_launch_dependents();
    griddep_wait();
    const int qs = p.query_start[b], qlen = p.query_start[b + 1] - qs;
    if (i0 >= qlen || qlen <= 0) return;
    int n = p.context_lens[b];
    if (n < qlen || n > p.max_blocks_per_seq * kChunk) {   // a query position outside the cache
        if (threadIdx.x == 0) set_status(p.status, PA_ERR_OUT_OF_RANGE);
        return;
    }
    const int rows = min(kQTile, qlen - i0);
    const int pos0 = n - qlen + i0;                  // position of query row 0 of the tile
    const int kend = pos0 + rows;                    // keys [0, kend) are visible to some row
    const int nkb = ceil_div_i(kend, kChunk);
    uint8_t* qsm = smem;                                              // [G][16][kRow]
    uint8_t* kv = smem + G * C::kQBytes;                              // [kStages][K, V][16][kRow]
    __shared__ int bad[kStages];                                      // the stage's block id was out of range
    const T* q = static_cast<const T*>(p.q);
    const T* kc = static_cast<const T*>(p.key_cache);
    const T* vc = static_cast<const T*>(p.value_cache);
    constexpr int kChunks = D * 2 / 16;              // 16-byte chunks per row

    // Q tiles of the group's heads (rows past the chunk are zero)
    for (int c = threadIdx.x; c < G * kQTile * kChunks; c += nthr) {
        const int hh = c / (kQTile * kChunks), r = (c / kChunks) % kQTile, k = c % kChunks;
        uint4 v = make_uint4(0, 0, 0, 0);
        if (r < rows)
            v = *reinterpret_cast<const uint4*>(q + ((size_t)(qs + i0 + r) * p.num_heads + g * G + hh) * D + k * 8);
        *reinterpret_cast<uint4*>(qsm + hh * C::kQBytes + r * C::kRow * 2 + k * 16) = v;
    }
    // K and V tiles of key block kb into stage st (zeros and a status bit for a
    // bad block id).  Rows at or past kend are zero-filled, not loaded: no
    // query of the tile sees them, and the slots past the context hold
    // whatever the pool held (NaN bit patterns in a fresh allocation), which
    // a masked probability of 0 would still carry into O (0 * NaN = NaN).
    auto load_block = [&](int kb, int st) {
        const int blk = p.block_tables[(size_t)b * p.max_blocks_per_seq + kb];
        const bool good = blk >= 0 && blk < p.num_blocks;
        if (threadIdx.x == 0) {
            bad[st] = !good;   // its keys are masked: the block contributes nothing
            if (!good) set_status(p.status, PA_ERR_OUT_OF_RANGE);
        }
        const size_t base = ((size_t)blk * p.num_kv_heads + g) * kChunk * D;
        for (int c = threadIdx.x; c < 2 * kChunk * kChunks; c += nthr) {
            const int which = c / (kChunk * kChunks), r = (c / kChunks) % kChunk, k = c % kChunks;
            uint8_t* dst = kv + (st * 2 + which) * C::kTileBytes + r * C::kRow * 2 + k * 16;
            if (good && kb * kChunk + r < kend) cp_async_16(smem_u32(dst), (which ? vc : kc) + base + r * D + k * 8);
            else *reinterpret_cast<uint4*>(dst) = make_uint4(0, 0, 0, 0);
        }
    };
    for (int s = 0; s < kStages - 1; ++s) {
        if (s < nkb) load_block(s, s);
        cp_async_commit();
    }

    const int h = warp;   // this warp's query head within the group
    const bool active = h < G;
    const int gid = lane >> 2, t4 = lane & 3, mi = lane >> 3, r8 = lane & 7;
    constexpr int KS = D / 16, NT = D / 8;
    constexpr bool kSplitP = std::is_same<T, __nv_bfloat16>::value;
    float o[NT][4];
#pragma unroll
    for (int j = 0; j < NT; ++j) o[j][0] = o[j][1] = o[j][2] = o[j][3] = 0.f;
    float mrun[2] = {kNegInfP, kNegInfP}, lrun[2] = {0.f, 0.f};
    const uint32_t qbase = smem_u32(qsm + h * C::kQBytes);
    const float sl2 = p.scale_log2;

    for (int kb = 0; kb < nkb; ++kb) {
        const int st = kb % kStages;
        // the stage computed in the previous step takes block kb + kStages - 1
        if (kb + kStages - 1 < nkb) load_block(kb + kStages - 1, (kb + kStages - 1) % kStages);
        cp_async_commit();
        cp_async_wait_pending<kStages - 1>();   // block kb has landed
        __syncthreads();
        if (active) {
            const uint32_t kt = smem_u32(kv + (st * 2) * C::kTileBytes);
            const uint32_t vt = smem_u32(kv + (st * 2 + 1) * C::kTileBytes);
            // ---- S[16 queries x 16 keys] = Q K^T
            float s[2][4];
#pragma unroll
            for (int j = 0; j < 2; ++j) s[j][0] = s[j][1] = s[j][2] = s[j][3] = 0.f;
#pragma unroll
            for (int kk = 0; kk < KS; ++kk) {
                uint32_t a[4], bq[4];
                ldsm_x4(qbase + (((mi & 1) * 8 + r8) * C::kRow + kk * 16 + (mi >> 1) * 8) * 2, a[0], a[1], a[2], a[3]);
                ldsm_x4(kt + (((mi >> 1) * 8 + r8) * C::kRow + kk * 16 + (mi & 1) * 8) * 2, bq[0], bq[1], bq[2], bq[3]);
                Mma<T>::run(s[0], a, bq[0], bq[1]);
                Mma<T>::run(s[1], a, bq[2], bq[3]);
            }
            // ---- causal mask and online softmax per query row (rows gid and gid + 8)
            const int key0 = kb * kChunk;
            const bool skip = bad[st] != 0;
            float mx[2] = {kNegInfP, kNegInfP};
#pragma unroll
            for (int j = 0; j < 2; ++j)
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    const int row = gid + (c >> 1) * 8, key = key0 + j * 8 + 2 * t4 + (c & 1);
                    float v = s[j][c] * sl2;
                    if (skip || row >= rows || key > pos0 + row) v = kNegInfP;
                    s[j][c] = v;
                    mx[c >> 1] = fmaxf(mx[c >> 1], v);
                }
            float al[2], ms[2];
#pragma unroll
            for (int r = 0; r < 2; ++r) {
                mx[r] = fmaxf(mx[r], __shfl_xor_sync(0xffffffffu, mx[r], 1));
                mx[r] = fmaxf(mx[r], __shfl_xor_sync(0xffffffffu, mx[r], 2));
                const float mn = fmaxf(mrun[r], mx[r]);
                ms[r] = mn == kNegInfP ? 0.f : mn;
                al[r] = mn == mrun[r] ? 1.f : fast_exp2(mrun[r] - ms[r]);
                mrun[r] = mn;
            }
            float pv[2][4];
#pragma unroll
            for (int j = 0; j < 2; ++j)
#pragma unroll
                for (int c = 0; c < 4; ++c) pv[j][c] = fast_exp2(s[j][c] - ms[c >> 1]);
            lrun[0] = lrun[0] * al[0] + (pv[0][0] + pv[0][1] + pv[1][0] + pv[1][1]);
            lrun[1] = lrun[1] * al[1] + (pv[0][2] + pv[0][3] + pv[1][2] + pv[1][3]);
            if (al[0] != 1.f || al[1] != 1.f) {
#pragma unroll
                for (int j = 0; j < NT; ++j) {
                    o[j][0] *= al[0];
                    o[j][1] *= al[0];
                    o[j][2] *= al[1];
                    o[j][3] *= al[1];
                }
            }
            // ---- O[16 x D] += P V: the S accumulators are the A fragment of P
            uint32_t ph[4], pl[4];
            ph[0] = Elt<T>::pack2(pv[0][0], pv[0][1]);
            ph[1] = Elt<T>::pack2(pv[0][2], pv[0][3]);
            ph[2] = Elt<T>::pack2(pv[1][0], pv[1][1]);
            ph[3] = Elt<T>::pack2(pv[1][2], pv[1][3]);
            if constexpr (kSplitP) {
                // remainder of p after bf16 rounding, itself in bf16: hi + lo carries ~16 bits
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&ph[k]));
                    const float* src = &pv[k >> 1][(k & 1) * 2];
                    pl[k] = Elt<T>::pack2(src[0] - f.x, src[1] - f.y);
                }
            }
#pragma unroll
            for (int j = 0; j < NT; j += 2) {
                uint32_t bv[4];
                ldsm_x4_t(vt + (((mi & 1) * 8 + r8) * C::kRow + j * 8 + (mi >> 1) * 8) * 2, bv[0], bv[1], bv[2], bv[3]);
                Mma<T>::run(o[j], ph, bv[0], bv[1]);
                Mma<T>::run(o[j + 1], ph, bv[2], bv[3]);
                if constexpr (kSplitP) {
                    Mma<T>::run(o[j], pl, bv[0], bv[1]);
                    Mma<T>::run(o[j + 1], pl, bv[2], bv[3]);
                }
            }
        }
        __syncthreads();   // the next step refills this stage
    }
    if (!active) return;
    // ---- out = O / l for the tile's rows
#pragma unroll
    for (int r = 0; r < 2; ++r) {
        lrun[r] += __shfl_xor_sync(0xffffffffu, lrun[r], 1);
        lrun[r] += __shfl_xor_sync(0xffffffffu, lrun[r], 2);
    }
    T* out = static_cast<T*>(p.out);
#pragma unroll
    for (int r = 0; r < 2; ++r) {
        const int row = gid + r * 8;
        if (row >= rows) continue;
        const float inv = lrun[r] > 0.f ? 1.f / lrun[r] : 0.f;
        T* dst = out + ((size_t)(qs + i0 + row) * p.num_heads + g * G + h) * D;
#pragma unroll
        for (int j = 0; j < NT; ++j) {
            const uint32_t v = Elt<T>::pack2(o[j][r * 2] * inv, o[j][r * 2 + 1] * inv);
            *reinterpret_cast<uint32_t*>(dst + j * 8 + 2 * t4) = v;
        }
    }
}

template <typename T, int D>
cudaError_t launch_prefill_t(const PrefillParams& p, cudaStream_t stream) {
    using C = PrefillCfg<D>;
    auto kernel = prefill_kernel<T, D>;
    const size_t smem = (size_t)p.group * C::kQBytes + 2 * kStages * C::kTileBytes;
    // the attribute is per device: set it on every call (a cheap host-side call)
    const cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    const dim3 grid((p.max_query_len + kQTile - 1) / kQTile, p.num_kv_heads, p.num_seqs);
    return launch_pdl(kernel, grid, dim3(32 * p.group), smem, stream, p);
}

}  // namespace

size_t prefill_workspace_bytes(const PrefillParams& p) { return prefill_tc_workspace_bytes(p); }

cudaError_t launch_prefill(const PrefillParams& p, void* ws, size_t ws_bytes, pa_dtype dtype, cudaStream_t stream) {
    if (prefill_tc_serves(p)) return launch_prefill_tc(p, ws, ws_bytes, dtype, stream);
    if (dtype == PA_F16) return p.head_dim == 64 ? launch_prefill_t<__half, 64>(p, stream)
                                                 : launch_prefill_t<__half, 128>(p, stream);
    if (dtype == PA_BF16) return p.head_dim == 64 ? launch_prefill_t<__nv_bfloat16, 64>(p, stream)
                                                  : launch_prefill_t<__nv_bfloat16, 128>(p, stream);
    return cudaErrorInvalidValue;
}

}  // namespace pa
