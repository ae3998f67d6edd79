// Paged decode attention on sm_100a.
//
// What is computed (the pages: "PagedAttention" digest, sections
// "PagedAttention in one picture", "Why the attention kernel works at all",
// "Misconceptions"): for each sequence b and query head h, ordinary softmax
// attention of q[b,h] over the sequence's K/V, which the kernel reaches by
// walking the block table; the result is that of contiguous attention.
//
// How (kernels chained with programmatic dependent launch):
//
//  1. plan    -- the work list of items (sequence b, partition p, KV head g):
//                every item of the sequences that span several partitions
//                first, then the rest, each class largest first.  A sequence
//                of nblk blocks has n = ceil(nblk / PB) partitions, the first
//                n - 1 of PB blocks (see seq_parts).  For batches of up to
//                256 sequences each CTA of the partition kernel derives its
//                own items of the list from context_lens (no launch); a
//                one-CTA plan kernel writes the whole list for larger
//                batches, for many items per CTA and for the SIMT kernel.
//  2. partition kernel -- persistent CTAs (4 per SM).  CTA c takes items
//                c, 2C-1-c, 2C+c, ... (snake order over the sorted list, which
//                balances the load).  Per CTA:
//                  * a producer warp streams, for each item, the Q rows of the
//                    GQA group (1-D bulk copy) and every 16-token tile of K and
//                    of V of the KV head (one 16-token block, contiguous 4 KB at
//                    D = 128; half of a 32-token block; or two 8-token blocks)
//                    with 2-D TMA tensor copies into a ring of
//                    shared-memory stages, 128-byte swizzled, tracked by
//                    mbarriers, evict-first in L2; work-list entries and table
//                    rows are prefetched two items ahead with cp.async;
//                  * consumer warps run two blocks per step on tensor cores:
//                    S^T = K Q^T (m16n8k16, tokens x heads, the GQA group padded
//                    to 8 or 16 columns), an online softmax in fp32 (column max
//                    by warp shuffles, 2^x on log2-scaled logits), then
//                    O^T += V^T P^T with P transposed in registers (movmatrix;
//                    bf16 P carried as a hi + lo pair);
//                  * with one consumer warp, the warp writes its item's result
//                    straight from the accumulators (final row, or the
//                    partition's (m, l, O)); the CTA that finishes the last
//                    partition of a (sequence, KV head) -- a per-group counter
//                    in the workspace says which -- hands it to a merger warp
//                    that combines all partitions (when there are at most 8)
//                    and resets the counter, so no reduce kernel runs;
//                  * (tuning shape) with two consumer warps, block j goes to
//                    warp j % 2 and the warps' states are merged through a
//                    double-buffered shared-memory slot by a rotating merger.
//                A SIMT variant serves float32 and groups above 16.
//  3. reduce  -- (sequences over 8 partitions, or two-warp CTAs) rows of the
//                multi-partition sequences: M = max m_p, L = sum l_p 2^(m_p - M),
//                out = sum O_p 2^(m_p - M) / L.
#include <type_traits>
#include <utility>

#include "pa_internal.h"

namespace pa {

namespace {
constexpr float kNegInf = -__builtin_huge_valf();
}

// ===========================================================================
// 1. plan
// ===========================================================================
// Partitions.  A sequence of nblk blocks has n = max(1, ceil(nblk / PB))
// partitions: partitions 0 .. nbig-1 hold `big` blocks, the others `small`.
//  * full split (default): n - 1 partitions of PB blocks, then the remainder.
//  * equal split (pa_decode_tuning.split = 1): near-equal lengths, q + 1 blocks
//    for the first r = nblk % n partitions and q = nblk / n for the rest.  It
//    avoids small tail partitions, yet measured 1-6% slower on every workload.
struct SeqParts {
    int n, nbig, big, small;
    __device__ __forceinline__ int start(int p) const { return p < nbig ? p * big : nbig * big + (p - nbig) * small; }
    __device__ __forceinline__ int len(int p) const { return p < nbig ? big : small; }
};
__device__ __forceinline__ SeqParts seq_parts(int nblk, int PB, bool equal) {
    SeqParts s;
    s.n = max(1, ceil_div_i(nblk, PB));
    if (equal) {
        s.small = nblk / s.n;
        s.big = s.small + 1;
        s.nbig = nblk - s.small * s.n;
    } else {
        const int tail = nblk - (s.n - 1) * PB;   // 1 .. PB (0 for an empty sequence)
        s.big = PB;
        s.nbig = tail == PB ? s.n : s.n - 1;
        s.small = tail == PB ? PB : tail;
    }
    return s;
}
// the same, without a division for the common single-partition case
__device__ __forceinline__ SeqParts seq_parts_fast(int nblk, int PB, bool equal) {
    if (nblk <= PB) {
        SeqParts s;
        s.n = 1;
        s.big = equal ? nblk + 1 : PB;
        s.nbig = (!equal && nblk == PB) ? 1 : 0;
        s.small = nblk;
        return s;
    }
    return seq_parts(nblk, PB, equal);
}

// Item order.  Largest first (key = PB - blocks; empty sequences last), which
// the snake assignment of the partition kernel turns into an even load.  With
// p.class_first (the default), all items of split sequences come before the
// others, each class largest first, so that the merges of split sequences
// happen early.  Inside a key the order is free; results do not depend on it.
constexpr int kMaxKeys = 2 * (kMaxPartBlocks + 1);
constexpr int kNoKey = 0xff;

struct PlanKeys {
    int PB, KB, Hkv, cf;
    // key of an item of `blocks` blocks; single-partition class offset by KB when cf
    __device__ __forceinline__ int key_of(int blocks, bool multi) const { return ((cf && !multi) ? KB : 0) + PB - blocks; }
    __device__ __forceinline__ int nkeys() const { return cf ? 2 * KB : KB; }
};

// a sequence's items fall in at most two keys: nbig partitions of `big`
// blocks and n - nbig of `small` blocks (kNoKey where there are none)
__device__ __forceinline__ void seq_keys(const PlanKeys& K, const SeqParts& s, int& kbig, int& ksmall) {
    const bool multi = s.n > 1;
    kbig = s.nbig > 0 ? K.key_of(s.big, multi) : kNoKey;
    ksmall = s.n > s.nbig ? K.key_of(s.small, multi) : kNoKey;
}

// Bucket offsets from the key counts: warp 0 scans the (at most 66) keys, 3
// per lane, into off[0 .. nkeys] (off[nkeys] = total); returns the total on
// lane 31.
__device__ __forceinline__ int scan_keys(const int* cnt, int* off, int nkeys, int lane) {
    static_assert(kMaxKeys <= 96, "the key scan covers 3 keys per lane");
    int v[3], sum = 0;
#pragma unroll
    for (int k = 0; k < 3; ++k) {
        const int key = lane * 3 + k;
        v[k] = key < nkeys ? cnt[key] : 0;
        sum += v[k];
    }
    int incl = sum;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int u = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += u;
    }
    int acc = incl - sum;
#pragma unroll
    for (int k = 0; k < 3; ++k) {
        const int key = lane * 3 + k;
        if (key < nkeys) off[key] = acc;
        acc += v[k];
    }
    if (lane == 31) off[nkeys] = incl;
    return incl;
}

// One CTA writes the whole list (items of one key in arbitrary order) and
// zeroes the merge counters of the problem.
template <int kThreads>
__global__ void __launch_bounds__(kThreads) decode_plan_kernel(const DecodeParams p) {
    __shared__ int cnt[kMaxKeys];
    __shared__ int cursor[kMaxKeys + 1];
    // the partition kernel may launch now and set up; it waits for this grid to finish
    griddep_launch_dependents();
    griddep_wait();
    const PlanKeys K{p.part_blocks, p.part_blocks + 1, p.num_kv_heads, p.class_first};
    const int nkeys = K.nkeys(), Hkv = K.Hkv, B = p.num_seqs;
    const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
    for (int i = tid; i < nkeys; i += kThreads) cnt[i] = 0;
    for (int i = tid; i < B * Hkv; i += kThreads) p.merge_count[i] = 0;
    __syncthreads();
    // pass 1: histogram of item keys
    for (int b = tid; b < B; b += kThreads) {
        const SeqParts sp = seq_parts_fast(ceil_div_i(load_ctx(p, b, true), kChunk), K.PB, p.equal_split);
        int kb, ks;
        seq_keys(K, sp, kb, ks);
        if (kb != kNoKey) atomicAdd(&cnt[kb], sp.nbig * Hkv);
        if (ks != kNoKey) atomicAdd(&cnt[ks], (sp.n - sp.nbig) * Hkv);
    }
    __syncthreads();
    if (wid == 0) {
        const int total = scan_keys(cnt, cursor, nkeys, lane);
        if (lane == 31) p.hdr[kHdrItems] = total;
    }
    __syncthreads();
    // pass 2: every lane reserves its sequence's slots; the warp then writes
    // the items of its 32 sequences one sequence at a time
    for (int b0 = wid * 32; b0 < B; b0 += kThreads) {
        const int b = b0 + lane;
        int ctx = 0, r = 0, n = 0, ob = 0, os = 0;
        if (b < B) {
            ctx = load_ctx(p, b, false);
            const SeqParts sp = seq_parts_fast(ceil_div_i(ctx, kChunk), K.PB, p.equal_split);
            int kb, ks;
            seq_keys(K, sp, kb, ks);
            r = sp.nbig;
            n = sp.n;
            if (kb != kNoKey) ob = atomicAdd(&cursor[kb], r * Hkv);
            if (ks != kNoKey) os = atomicAdd(&cursor[ks], (n - r) * Hkv);
        }
        for (int l = 0; l < 32; ++l) {
            const int bl = b0 + l;
            if (bl >= B) break;
            const int cl = __shfl_sync(0xffffffffu, ctx, l), rl = __shfl_sync(0xffffffffu, r, l);
            const int nl = __shfl_sync(0xffffffffu, n, l);
            const int obl = __shfl_sync(0xffffffffu, ob, l), osl = __shfl_sync(0xffffffffu, os, l);
            for (int i = lane; i < rl * Hkv; i += 32) p.items[obl + i] = make_int4(bl, ((i / Hkv) << 8) | (i % Hkv), cl, 0);
            for (int i = lane; i < (nl - rl) * Hkv; i += 32)
                p.items[osl + i] = make_int4(bl, ((rl + i / Hkv) << 8) | (i % Hkv), cl, 0);
        }
    }
}

// geometry of one item, identical in every kernel
struct ItemGeom {
    int b, g, p, ctx, j0, nblk, nparts;
};
__device__ __forceinline__ ItemGeom item_geom(const DecodeParams& p, int4 it) {
    ItemGeom m;
    m.b = it.x;
    m.p = it.y >> 8;
    m.g = it.y & 255;
    m.ctx = it.z;
    const SeqParts sp = seq_parts_fast(ceil_div_i(m.ctx, kChunk), p.part_blocks, p.equal_split);
    m.j0 = sp.start(m.p);
    m.nblk = sp.len(m.p);
    m.nparts = sp.n;
    return m;
}

// ===========================================================================
// 2a. partition kernel, tensor cores (fp16 / bf16)
// ===========================================================================
// Fused merge (single-warp CTAs, at most kFusedMaxParts = 8 partitions): one
// warp combines every partition of (sequence b, KV head g) for the G query
// heads of the group, out = sum_p O_p 2^(m_p - M) / sum_p l_p 2^(m_p - M).  The
// partials were written by other CTAs: cache-global loads.  Round trips: one
// for every (head, partition)'s m and l, then one per two or four heads for O.
// (Sixteen partitions per warp were measured slower than the reduce kernel.)
constexpr int kFusedMaxParts = 8;

template <typename T, int D, int GMAX>
__device__ __forceinline__ void merge_group(const DecodeParams& p, int b, int g, int nparts, int lane,
                                            float* s_w, float* s_inv) {
    constexpr int E = D / 32;
    constexpr int MP = kFusedMaxParts;
    constexpr int kSlots = GMAX * MP / 32;
    // heads whose partial rows are in flight together (4 fits the register
    // budget of the D = 128, 8-head shape without raising it; 2 elsewhere)
    constexpr int HP = (D == 128 && GMAX == 8) ? 4 : 2;
    using VecE = typename std::conditional<E == 4, float4, float2>::type;
    const int G = p.group;
    const size_t hq0 = (size_t)b * p.num_heads + (size_t)g * G;
    // (m, l) of entry e = h * MP + q: lane e % 32, slot e / 32
    float mv[kSlots], lv[kSlots];
#pragma unroll
    for (int k = 0; k < kSlots; ++k) {
        const int e = lane + 32 * k, h = e / MP, q = e % MP;
        const bool ok = h < G && q < nparts;
        const size_t pi = (hq0 + h) * p.max_parts + q;
        mv[k] = ok ? __ldcg(p.part_m + pi) : kNegInf;
        lv[k] = ok ? __ldcg(p.part_l + pi) : 0.f;
    }
#pragma unroll
    for (int k = 0; k < kSlots; ++k) {
        // the MP lanes of one head are consecutive: reduce over them
        float M = mv[k];
#pragma unroll
        for (int off = 1; off < MP; off <<= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, off));
        const float Ms = M == kNegInf ? 0.f : M;
        const float w = mv[k] == kNegInf ? 0.f : fast_exp2(mv[k] - Ms);
        float L = w * lv[k];
#pragma unroll
        for (int off = 1; off < MP; off <<= 1) L += __shfl_xor_sync(0xffffffffu, L, off);
        const int e = lane + 32 * k;
        if (e / MP < G) {
            s_w[e] = w;
            if (e % MP == 0) s_inv[e / MP] = L > 0.f ? 1.f / L : 0.f;
        }
    }
    __syncwarp();
    // out = sum_q w_q O_q / L, lane l owning dims [l*E, l*E + E)
    T* out = static_cast<T*>(p.out);
    for (int h0 = 0; h0 < G; h0 += HP) {
        VecE v[HP][MP];
#pragma unroll
        for (int hh = 0; hh < HP; ++hh)
#pragma unroll
            for (int q = 0; q < MP; ++q)
                if (h0 + hh < G && q < nparts)
                    v[hh][q] = __ldcg(reinterpret_cast<const VecE*>(p.part_o + ((hq0 + h0 + hh) * p.max_parts + q) * D +
                                                                    lane * E));
#pragma unroll
        for (int hh = 0; hh < HP; ++hh) {
            const int h = h0 + hh;
            if (h >= G) break;
            float acc[E];
#pragma unroll
            for (int e = 0; e < E; ++e) acc[e] = 0.f;
#pragma unroll
            for (int q = 0; q < MP; ++q) {
                if (q < nparts) {
                    const float wq = s_w[h * MP + q];
                    const float* f = reinterpret_cast<const float*>(&v[hh][q]);
#pragma unroll
                    for (int e = 0; e < E; ++e) acc[e] += wq * f[e];
                }
            }
            const float inv = s_inv[h];
#pragma unroll
            for (int e = 0; e < E; ++e) out[(hq0 + h) * D + lane * E + e] = Elt<T>::from_f(acc[e] * inv);
        }
    }
    __syncwarp();
}

struct ItemMeta {
    int b, g, p, ctx, j0, nblk, nparts, pad;
};

// work-list entry and table row of one item, prefetched by the producer
struct DescSlot {
    int4 e;
    int bt[kMaxPartBlocks];    // per chunk: its block (8-token blocks: the first of its two)
    int bt2[kMaxPartBlocks];   // 8-token blocks: the chunk's second block, if the context reaches it
    int rank;      // position in the work list
    int pad[3];
};

// ---------------------------------------------------------------------------
// Self-planning: with p.self_plan set, no plan kernel runs; every CTA of the
// partition kernel derives its own items of the largest-first list from
// context_lens before its first tile copy.  The list has the plan kernel's
// keys in the same order; inside a key the items go in sequence order.  Each
// CTA reads all of context_lens (one round trip of cp.async), builds the key
// histogram and its prefix, then each warp finds items rank by rank: the key
// by binary search over the prefix, the sequence by a warp scan of the key's
// per-sequence item counts.  Scratch lives in the tile ring, which is free
// until the first copy.
//
// Scratch layout (ints): key counts, key offsets, then per sequence its
// clamped context length, nbig, partition count and keys.
constexpr int kPlanCtxOff = 2 * kMaxKeys + 2;

// First step of self-planning, issued at the very start of the kernel so that
// its latency overlaps the prologue: context_lens into the scratch, one
// cp.async group per thread (plan_own_items waits for it).
__device__ __forceinline__ void plan_load_ctx(const DecodeParams& p, int* scratch) {
    int* s_ctx = scratch + kPlanCtxOff;
    for (int b = threadIdx.x; b < p.num_seqs; b += blockDim.x) cp_async_4(smem_u32(&s_ctx[b]), p.context_lens + b);
    cp_async_commit();
}

// Fills own[0 .. n_own) with this CTA's items (ranks c, 2C-1-c, 2C+c, ...);
// s_list[0] = list length, s_list[1] = n_own.  Called by every thread of the
// CTA, after plan_load_ctx.
template <int kMaxOwn>
__device__ void plan_own_items(const DecodeParams& p, int* scratch, int4* own, int* s_list) {
    const int tid = threadIdx.x, nthr = blockDim.x, lane = tid & 31, wid = tid >> 5, nwarps = nthr >> 5;
    const int B = p.num_seqs;
    int* s_cnt = scratch;                        // [kMaxKeys]
    int* s_off = s_cnt + kMaxKeys;               // [kMaxKeys + 1]
    int* s_ctx = scratch + kPlanCtxOff;          // [B] clamped context lengths
    int* s_r = s_ctx + B;                        // [B] partitions of the longer length (nbig)
    int* s_np = s_r + B;                         // [B] partitions
    int* s_key = s_np + B;                       // [B] kbig | ksmall << 8
    const PlanKeys K{p.part_blocks, p.part_blocks + 1, p.num_kv_heads, p.class_first};
    const int nkeys = K.nkeys();
    for (int i = tid; i < nkeys; i += nthr) s_cnt[i] = 0;
    cp_async_wait_all();
    __syncthreads();
    // histogram of item keys; CTA 0 reports bad lengths
    const bool report = blockIdx.x == 0;
    for (int b = tid; b < B; b += nthr) {
        const int c = clamp_ctx(p, s_ctx[b], report);
        const SeqParts sp = seq_parts_fast(ceil_div_i(c, kChunk), K.PB, p.equal_split);
        int kb, ks;
        seq_keys(K, sp, kb, ks);
        s_ctx[b] = c;
        s_r[b] = sp.nbig;
        s_np[b] = sp.n;
        s_key[b] = kb | (ks << 8);
        if (kb != kNoKey) atomicAdd(&s_cnt[kb], sp.nbig * K.Hkv);
        if (ks != kNoKey) atomicAdd(&s_cnt[ks], (sp.n - sp.nbig) * K.Hkv);
    }
    __syncthreads();
    // bucket offsets and this CTA's share of the list
    if (wid == 0) {
        const int total = scan_keys(s_cnt, s_off, nkeys, lane);
        if (lane == 31) {
            const int C = gridDim.x, c = blockIdx.x;
            const int full = total / C, rem = total - full * C;
            int n_own = full + (((full & 1) ? C - 1 - c : c) < rem ? 1 : 0);
            s_list[0] = total;
            if (n_own > kMaxOwn) {   // excluded by the host: report it, and this CTA takes nothing
                set_status(p.status, PA_ERR_UNSUPPORTED);
                n_own = 0;
                s_list[0] = 0;
            }
            s_list[1] = n_own;
        }
    }
    __syncthreads();
    const int n_own = s_list[1];
    const int C = gridDim.x, c = blockIdx.x;
    for (int it = wid; it < n_own; it += nwarps) {
        const int r = it * C + ((it & 1) ? C - 1 - c : c);
        int lo = 0, hi = nkeys;   // last key whose offset is <= r (never an empty one)
        while (hi - lo > 1) {
            const int mid = (lo + hi) >> 1;
            if (s_off[mid] <= r) lo = mid;
            else hi = mid;
        }
        const int k = lo;
        int j = r - s_off[k];     // index inside key k
        for (int b0 = 0; b0 < B; b0 += 32) {
            const int b = b0 + lane;
            const int kk = b < B ? s_key[b] : (kNoKey | (kNoKey << 8));
            const bool big = (kk & 0xff) == k, small = (kk >> 8) == k;
            const int w = big ? s_r[b] * K.Hkv : (small ? (s_np[b] - s_r[b]) * K.Hkv : 0);
            const int tot = __reduce_add_sync(0xffffffffu, w);
            if (j >= tot) {
                j -= tot;
                continue;
            }
            int incl = w;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int u = __shfl_up_sync(0xffffffffu, incl, o);
                if (lane >= o) incl += u;
            }
            if (j >= incl - w && j < incl) {
                const int local = j - (incl - w);
                const int part = (big ? 0 : s_r[b]) + local / K.Hkv;
                own[it] = make_int4(b, (part << 8) | (local % K.Hkv), s_ctx[b], 0);
            }
            break;
        }
    }
    __syncthreads();
}

template <int D, int NT, int NCW, int STAGES>
struct TcCfg {
    static constexpr int kBoxes = D / 64;                    // 64-element (128 B) boxes per tile row
    static constexpr int kBoxBytes = kChunk * 128;           // 2 KB: 16 rows x 128 B
    static constexpr int kTileBytes = kChunk * D * 2;        // one K or V tile (16 tokens)
    static constexpr int kStageBytes = 2 * kTileBytes;
    static constexpr int kISlots = NCW == 1 ? 2 : 4;         // item metadata / Q ring
    static constexpr int kDSlots = 4;                        // descriptor prefetch ring
    static constexpr int kMSlots = NCW == 1 ? 0 : 2;         // merge buffers (double-buffered; none for one warp)
    static constexpr int kHeadsPad = 8 * NT;
    static constexpr int kQBytes = kHeadsPad * D * 2;
    static constexpr int kMergeStride = D + 4;               // floats per head row (bank-conflict pad)
    static constexpr int kMergeFloats = NCW * kHeadsPad * kMergeStride;   // one merge buffer
    static constexpr int kOffStages = 0;
    static constexpr int kOffQ = kOffStages + STAGES * kStageBytes;
    static constexpr int kOffMerge = kOffQ + kISlots * kQBytes;
    static constexpr int kOffMl = kOffMerge + kMSlots * kMergeFloats * 4;
    static constexpr int kOffDesc = kOffMl + kMSlots * NCW * kHeadsPad * 2 * 4;
    static constexpr int kOffMeta = kOffDesc + kDSlots * (int)sizeof(DescSlot);
    static constexpr int kQSlots = NCW == 1 ? 4 : 0;          // merge-task queue (single-warp CTAs)
    static constexpr int kOffTasks = kOffMeta + kISlots * (int)sizeof(ItemMeta);
    // merger's partition weights (heads x kFusedMaxParts) and 1/L (heads)
    static constexpr int kMergeW = NCW == 1 ? kHeadsPad * kFusedMaxParts + kHeadsPad : 0;
    static constexpr int kOffMW = kOffTasks + kQSlots * 16;
    static constexpr int kMaxOwn = 64;                       // items a self-planning CTA can hold
    static constexpr int kOffOwn = kOffMW + kMergeW * 4;
    static constexpr int kOffBar = kOffOwn + kMaxOwn * 16;
    static constexpr int kNumBars = 2 * STAGES + 2 * kISlots + 2 * kMSlots + 2 * kQSlots;
    static constexpr int kOffFlags = kOffBar + kNumBars * 8;
    static constexpr int kBytes = kOffFlags + 16 + STAGES * 4;
    static constexpr int kSmemBytes = kBytes + 1024;         // slack for 1024-byte alignment
    // largest batch a self-planning CTA can plan in its ring (4 ints per sequence)
    static constexpr int kPlanSeqs = (STAGES * kStageBytes / 4 - 2 * kMaxKeys - 2) / 4;
    // warps: NCW consumers, one producer, and (single-warp CTAs) one merger
    static constexpr int kWarps = NCW + 1 + (NCW == 1 ? 1 : 0);
    static constexpr int kThreads = kWarps * 32;
    // CTAs per SM the shape is sized for (shared memory at D = 128); the
    // register budget is capped to match
    static constexpr int kMinBlocks = (NCW == 2 || NT == 2 || STAGES >= 13) ? 2 : (STAGES >= 8 ? 3 : 4);
    static_assert(kOffDesc % 16 == 0 && sizeof(DescSlot) % 16 == 0, "cp.async 16-byte destinations");
    static_assert(kOffOwn % 16 == 0, "own-item list alignment");
    // the shared memory a shape is sized for: kMinBlocks CTAs per SM (228 KB,
    // 1 KB reserved per CTA)
    static_assert(kMinBlocks * (kSmemBytes + 1024) <= 228 * 1024 || D != 128, "shape no longer fits its CTAs per SM");
    // Ring stage n and stage n + STAGES reuse one slot and one parity bit, so a
    // consumer may only wait for stage n once stage n - STAGES has landed, or it
    // would take the old phase for the new one.  Stage n is consumed by warp
    // n % NCW; with STAGES a multiple of NCW both stages belong to the same
    // warp, which takes its stages in order.
    static_assert(STAGES % NCW == 0, "ring depth must be a multiple of the consumer warps");
};

template <typename T, int D, int NT, int NCW, int STAGES>
__global__ void __launch_bounds__(TcCfg<D, NT, NCW, STAGES>::kThreads, TcCfg<D, NT, NCW, STAGES>::kMinBlocks)
    decode_tc_kernel(const DecodeParams p, const __grid_constant__ CUtensorMap tmK,
                     const __grid_constant__ CUtensorMap tmV) {
    using C = TcCfg<D, NT, NCW, STAGES>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* stages = smem + C::kOffStages;
    uint8_t* qbuf = smem + C::kOffQ;
    float* merge = reinterpret_cast<float*>(smem + C::kOffMerge);
    float* ml = reinterpret_cast<float*>(smem + C::kOffMl);
    DescSlot* dsc = reinterpret_cast<DescSlot*>(smem + C::kOffDesc);
    ItemMeta* meta = reinterpret_cast<ItemMeta*>(smem + C::kOffMeta);
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::kOffBar);
    uint64_t* empty = full + STAGES;
    uint64_t* ifull = empty + STAGES;
    uint64_t* iempty = ifull + C::kISlots;
    uint64_t* mfull = iempty + C::kISlots;       // all NCW warps deposited their item state
    uint64_t* mempty = mfull + C::kMSlots;       // the item's merger has read the buffer
    uint64_t* qfull = mempty + C::kMSlots;       // a merge task is queued
    uint64_t* qempty = qfull + C::kQSlots;       // the merger took it
    int4* tasks = reinterpret_cast<int4*>(smem + C::kOffTasks);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::kOffFlags);
    volatile int* stage_bad = reinterpret_cast<volatile int*>(smem + C::kOffFlags + 16);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int G = p.group;
    if (p.self_plan) plan_load_ctx(p, reinterpret_cast<int*>(stages));
    // every wait of the kernel is bounded (p.wait_limit_ns); on expiry the
    // kernel reports PA_ERR_TIMEOUT, lets the copies it issued land and returns
    const uint64_t wait_limit = p.wait_limit_ns;
    auto wait_on = [wait_limit](uint64_t* bar, uint32_t parity) { return mbar_wait(bar, parity, wait_limit); };

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int i = 0; i < C::kISlots; ++i) {
            mbar_init(&ifull[i], 1);
            mbar_init(&iempty[i], NCW);
        }
        for (int i = 0; i < C::kMSlots; ++i) {
            mbar_init(&mfull[i], NCW);
            mbar_init(&mempty[i], 1);
        }
        for (int i = 0; i < C::kQSlots; ++i) {
            mbar_init(&qfull[i], 1);
            mbar_init(&qempty[i], 1);
        }
        *abort_flag = 0;
        mbar_fence_init();
    }
    // rows of the padded GQA group beyond G stay zero; TMA fills rows < G
    for (int i = threadIdx.x; i < C::kISlots * C::kQBytes / 16; i += blockDim.x)
        reinterpret_cast<uint4*>(qbuf)[i] = make_uint4(0, 0, 0, 0);
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    __syncthreads();

    griddep_launch_dependents();
    const int PB = p.part_blocks;
    int4* own = reinterpret_cast<int4*>(smem + C::kOffOwn);
    int* s_plan = const_cast<int*>(abort_flag) + 1;   // [0] list length, [1] own items (self-planning)
    // Self-planning reads only context_lens and block_tables, which no kernel
    // of this library writes, so it runs before the wait for the preceding
    // kernel (the append of the same step, chained by programmatic dependent
    // launch); everything that kernel may write -- the pools, q, out, the
    // workspace -- is touched only after griddep_wait() below.
    if (p.self_plan) {
        {   // warm L2 with this CTA's share of the block tables: the rows are read right after planning
            const char* bt = reinterpret_cast<const char*>(p.block_tables);
            const size_t bytes = (size_t)p.num_seqs * p.max_blocks_per_seq * sizeof(int32_t);
            const size_t share = (bytes + gridDim.x - 1) / gridDim.x;
            const size_t lo = share * blockIdx.x, hi = min(bytes, lo + share);
            for (size_t off = lo + (size_t)threadIdx.x * 128; off < hi; off += (size_t)blockDim.x * 128)
                prefetch_l2(bt + off);
        }
        plan_own_items<C::kMaxOwn>(p, reinterpret_cast<int*>(stages), own, s_plan);
        // the scratch was written through the generic proxy; tile copies (async proxy) follow
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        __syncthreads();
    }
    griddep_wait();
    if (p.self_plan) {
        // The plan stays in the workspace for pa_decode_planned: each CTA writes
        // its items at their ranks (the planning kernel's list, entry for entry)
        // and CTA 0 the length.  After the wait: the preceding kernel may be a
        // planned decode still reading the previous list.
        const int n_own = s_plan[1], Cn = (int)gridDim.x, cb = (int)blockIdx.x;
        for (int it = threadIdx.x; it < n_own; it += blockDim.x) p.items[it * Cn + ((it & 1) ? Cn - 1 - cb : cb)] = own[it];
        if (blockIdx.x == 0 && threadIdx.x == 0) p.hdr[kHdrItems] = s_plan[0];
    }

    if constexpr (NCW == 1) {
        if (warp == NCW + 1) {
            // -------------------------------------------------------- merger
            // Takes (sequence, KV head) groups whose last partition this CTA
            // finished and merges all their partitions, off the consumer's path.
            for (int t = 0;; ++t) {
                const int qs = t % C::kQSlots;
                if (!__all_sync(0xffffffffu, wait_on(&qfull[qs], (t / C::kQSlots) & 1)) || *abort_flag) {
                    *abort_flag = 1;
                    break;
                }
                const int4 task = tasks[qs];
                __syncwarp();
                if (lane == 0) mbar_arrive(&qempty[qs]);
                if (task.x < 0) break;
                __threadfence();
                float* s_w = reinterpret_cast<float*>(smem + C::kOffMW);
                merge_group<T, D, C::kHeadsPad>(p, task.x, task.y, task.z, lane, s_w,
                                                s_w + C::kHeadsPad * kFusedMaxParts);
                // every partition has arrived: the counter is free, leave it zeroed for the next call
                if (lane == 0) p.merge_count[(size_t)task.x * p.num_kv_heads + task.y] = 0;
            }
            return;
        }
    }

    if (warp == NCW) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            prefetch_tensormap(&tmK);
            prefetch_tensormap(&tmV);
        }
        const uint64_t pol = policy_evict_first();
        const size_t q_row_bytes = (size_t)D * 2;

        // Descriptor pipeline, so that no global-memory latency sits between
        // two items' tile loads: item k's rank, work-list entry and table row
        // land in slot k % kDSlots.  At the top of iteration i, entry(i),
        // row(i) and entry(i+1) are visible and the group {row(i+1),
        // entry(i+2)} is in flight.  A self-planning CTA has its entries in
        // shared memory already (own[k] is item k).
        const bool self_plan = p.self_plan != 0;
        int n_items = 0;  // set once the plan's count has been read (below)
        auto fetch_entry = [&](int it, int r) {
            if (lane == 0) {
                dsc[it % C::kDSlots].rank = r;
                if (r < n_items) {
                    if (self_plan) dsc[it % C::kDSlots].e = own[it];
                    else cp_async_16(smem_u32(&dsc[it % C::kDSlots].e), &p.items[r]);
                }
            }
        };
        auto fetch_row = [&](int it) {
            const int r = dsc[it % C::kDSlots].rank;
            if (r >= n_items) return;
            const ItemGeom m = item_geom(p, dsc[it % C::kDSlots].e);
            if (lane < m.nblk) {
                // chunk c is block c (16-token blocks), the half (c & 1) of block
                // c / 2 (32-token blocks) or blocks 2c and 2c + 1 (8-token blocks,
                // the second only where the context reaches it)
                DescSlot& ds = dsc[it % C::kDSlots];
                const int32_t* row = p.block_tables + (size_t)m.b * p.max_blocks_per_seq;
                const int c = m.j0 + lane;
                if (p.block_size == kChunk) {
                    cp_async_4(smem_u32(&ds.bt[lane]), row + c);
                } else if (p.block_size > kChunk) {
                    cp_async_4(smem_u32(&ds.bt[lane]), row + (c >> 1));
                } else {
                    cp_async_4(smem_u32(&ds.bt[lane]), row + 2 * c);
                    if (2 * c + 1 < ceil_div_i(m.ctx, p.block_size))
                        cp_async_4(smem_u32(&ds.bt2[lane]), row + 2 * c + 1);
                }
            }
        };
        // Static schedule: CTA c takes ranks c, 2C-1-c, 2C+c, ... of the
        // largest-first list (snake order), which balances the load without a
        // shared counter.  (Claiming the list's tail from a counter at run
        // time was measured slower on every workload.)
        const int ctas = gridDim.x, cta = blockIdx.x;
        auto rank_of = [&](int it) { return it * ctas + ((it & 1) ? (ctas - 1 - cta) : cta); };
        // the item count and this CTA's first work-list entry (rank = cta; the
        // list holds at least gridDim.x entries) arrive in one round trip
        if (self_plan) {
            n_items = s_plan[0];
            if (lane == 0) {
                dsc[0].rank = cta < n_items ? cta : n_items;
                if (cta < n_items) dsc[0].e = own[0];
            }
        } else {
            if (lane == 0) {
                cp_async_4(smem_u32(s_plan), &p.hdr[kHdrItems]);
                cp_async_16(smem_u32(&dsc[0].e), &p.items[cta]);
            }
            cp_async_commit();
            cp_async_wait_all();
            __syncwarp();
            n_items = s_plan[0];
            if (lane == 0) dsc[0].rank = cta < n_items ? cta : n_items;
        }
        __syncwarp();
        fetch_row(0);
        fetch_entry(1, rank_of(1));
        cp_async_commit();
        cp_async_wait_all();
        __syncwarp();
        fetch_row(1);
        fetch_entry(2, rank_of(2));
        cp_async_commit();
        __syncwarp();

        // Item k's metadata and Q rows are published (and the Q copy issued) at
        // the start of item k-1's tile stream, so they have landed by the time
        // the consumers reach item k.  publish() returns 1 if item `it` was
        // published, 0 at the end of the work list (sentinel published), -1 on
        // a wait that timed out.
        auto publish = [&](int it) -> int {
            const int islot = it % C::kISlots;
            int okw = 1;
            if (lane == 0) okw = wait_on(&iempty[islot], ((it / C::kISlots) & 1) ^ 1);
            if (!__shfl_sync(0xffffffffu, okw, 0)) return -1;
            const DescSlot& dd = dsc[it % C::kDSlots];
            if (dd.rank >= n_items) {
                if (lane == 0) {
                    meta[islot].nblk = -1;
                    mbar_arrive(&ifull[islot]);
                }
                return 0;
            }
            if (p.stall_first_item && it == 0 && blockIdx.x == 0) return 1;   // test hook: never published
            if (lane == 0) {
                const ItemGeom mm = item_geom(p, dd.e);
                meta[islot] = ItemMeta{mm.b, mm.g, mm.p, mm.ctx, mm.j0, mm.nblk, mm.nparts, 0};
                const uint32_t qbytes = (uint32_t)(G * q_row_bytes);
                mbar_arrive_expect_tx(&ifull[islot], qbytes);
                bulk_load_1d(smem_u32(qbuf + islot * C::kQBytes),
                             static_cast<const uint8_t*>(p.q) +
                                 ((size_t)mm.b * p.num_heads + (size_t)mm.g * G) * q_row_bytes,
                             qbytes, &ifull[islot]);
            }
            return 1;
        };

        // With 4 item slots, item k+1 is published while item k streams; with 2
        // (single-warp CTAs) that would hold the producer back to one item ahead
        // of the consumer, so item k is published when its tiles start.
        constexpr int kLook = C::kISlots >= 4 ? 1 : 0;
        uint32_t stage = 0;
        int npub = 0;  // items whose Q copy was issued
        bool ok = true;
        int pub = publish(0);
        if (pub < 0) ok = false;
        npub += pub > 0;
        bool more = pub > 0;   // item iter exists
        for (int iter = 0; ok && more; ++iter) {
            if (kLook) {
                pub = publish(iter + 1);
                if (pub < 0) { ok = false; break; }
                npub += pub > 0;
                more = pub > 0;
            } else if (iter > 0) {
                pub = publish(iter);
                if (pub < 0) { ok = false; break; }
                npub += pub > 0;
                if (pub == 0) break;
            }
            const DescSlot& d = dsc[iter % C::kDSlots];
            const ItemGeom m = item_geom(p, d.e);
            int okw = 1;
            if (lane == 0) {
                // each item starts on a stage that is a multiple of NCW, so block j
                // always goes to consumer warp j % NCW wherever the item runs
                // (bitwise-reproducible results); the padding stages carry no data
                for (; stage % NCW != 0; ++stage) {
                    const int s = stage % STAGES;
                    if (!wait_on(&empty[s], ((stage / STAGES) & 1) ^ 1)) { okw = 0; break; }
                    stage_bad[s] = 1;
                    mbar_arrive(&full[s]);
                }
                const int bs = p.block_size;
                const int nphys = ceil_div_i(m.ctx, bs);   // blocks the context occupies
                for (int j = 0; j < m.nblk && okw; ++j, ++stage) {
                    const int c = m.j0 + j;
                    const int blk = d.bt[j];
                    // 8-token blocks: the chunk's second block, absent past the context
                    const bool has1 = bs < kChunk && 2 * c + 1 < nphys;
                    const int blk1 = has1 ? d.bt2[j] : 0;
                    const int s = stage % STAGES;
                    if (!wait_on(&empty[s], ((stage / STAGES) & 1) ^ 1)) { okw = 0; break; }
                    if (blk >= 0 && blk < p.num_blocks && blk1 >= 0 && blk1 < p.num_blocks) {
                        stage_bad[s] = 0;
                        const uint32_t kdst = smem_u32(stages + s * C::kStageBytes);
                        if (bs >= kChunk) {
                            // one 16-row box per 64 columns: the block, or its half c & 1
                            mbar_arrive_expect_tx(&full[s], C::kStageBytes);
                            const int y = (blk * p.num_kv_heads + m.g) * bs + (bs > kChunk ? (c & 1) * kChunk : 0);
#pragma unroll
                            for (int h = 0; h < C::kBoxes; ++h)
                                tma_load_2d(kdst + h * C::kBoxBytes, &tmK, h * 64, y, &full[s], pol);
#pragma unroll
                            for (int h = 0; h < C::kBoxes; ++h)
                                tma_load_2d(kdst + C::kTileBytes + h * C::kBoxBytes, &tmV, h * 64, y, &full[s],
                                            pol);
                        } else {
                            // 8-row boxes: rows 0-7 of the tile from the first block,
                            // rows 8-15 (1 KB further, the next 128-byte swizzle atom,
                            // so the tile's layout is that of one 16-row box) from the
                            // second; past the context, rows 8-15 keep stale data that
                            // the consumer masks (K) and clears (V)
                            mbar_arrive_expect_tx(&full[s], has1 ? C::kStageBytes : C::kStageBytes / 2);
                            const int y0 = blk * p.num_kv_heads + m.g, y1 = blk1 * p.num_kv_heads + m.g;
#pragma unroll
                            for (int h = 0; h < C::kBoxes; ++h) {
                                tma_load_2d(kdst + h * C::kBoxBytes, &tmK, h * 64, y0 * bs, &full[s], pol);
                                tma_load_2d(kdst + C::kTileBytes + h * C::kBoxBytes, &tmV, h * 64, y0 * bs,
                                            &full[s], pol);
                                if (has1) {
                                    tma_load_2d(kdst + h * C::kBoxBytes + C::kBoxBytes / 2, &tmK, h * 64, y1 * bs,
                                                &full[s], pol);
                                    tma_load_2d(kdst + C::kTileBytes + h * C::kBoxBytes + C::kBoxBytes / 2, &tmV,
                                                h * 64, y1 * bs, &full[s], pol);
                                }
                            }
                        }
                    } else {
                        stage_bad[s] = 1;
                        set_status(p.status, PA_ERR_OUT_OF_RANGE);
                        mbar_arrive(&full[s]);
                    }
                }
            }
            stage = __shfl_sync(0xffffffffu, stage, 0);
            if (!__shfl_sync(0xffffffffu, okw, 0) || *abort_flag) { ok = false; break; }
            if (!kLook) more = true;
            // descriptors of items iter+2 and iter+3 start loading; item iter+1's are ready
            cp_async_wait_all();
            __syncwarp();
            fetch_row(iter + 2);
            fetch_entry(iter + 3, rank_of(iter + 3));
            cp_async_commit();
            __syncwarp();
        }
        cp_async_wait_all();
        if (!ok) {
            if (lane == 0) {
                *abort_flag = 1;
                set_status(p.status, PA_ERR_TIMEOUT);
                // let copies already issued land before the CTA's memory is released
                const uint32_t outstanding = stage < (uint32_t)STAGES ? stage : (uint32_t)STAGES;
                for (uint32_t k = 1; k <= outstanding; ++k) {
                    const uint32_t n = stage - k;
                    wait_on(&full[n % STAGES], (n / STAGES) & 1);
                }
                const int qout = npub < C::kISlots ? npub : C::kISlots;
                for (int k = 1; k <= qout; ++k) {
                    const int it = npub - k;
                    wait_on(&ifull[it % C::kISlots], (it / C::kISlots) & 1);
                }
            }
        }
        return;
    }

    // ---------------------------------------------------------------- consumers
    const int cw = warp;
    const int gid = lane >> 2, t4 = lane & 3;
    const int mi = lane >> 3, r8 = lane & 7;
    const float sl2 = p.scale_log2;
    constexpr int KS = D / 16;  // k-steps of QK^T == m-tiles of PV
    constexpr bool kSplitP = std::is_same<T, __nv_bfloat16>::value;  // P as hi + lo bf16 pair
    uint32_t stage_base = 0;
    int nq = 0;  // merge tasks queued (single-warp CTAs)
    // per-lane parts of the ldmatrix row addresses (tile-relative, bytes)
    uint32_t koff[KS], voff[KS];
#pragma unroll
    for (int kk = 0; kk < KS; ++kk) {
        const int kd0 = kk * 16 + 8 * (mi >> 1), ktok = r8 + 8 * (mi & 1);
        koff[kk] = (kd0 >> 6) * C::kBoxBytes + ktok * 128 + ((((kd0 & 63) >> 3) ^ r8) << 4);
        const int vd0 = kk * 16 + 8 * (mi & 1), vtok = r8 + 8 * (mi >> 1);
        voff[kk] = C::kTileBytes + (vd0 >> 6) * C::kBoxBytes + vtok * 128 + ((((vd0 & 63) >> 3) ^ r8) << 4);
    }

    for (int iter = 0;; ++iter) {
        const int islot = iter % C::kISlots;
        const uint32_t iph = (iter / C::kISlots) & 1;
        if (!__all_sync(0xffffffffu, wait_on(&ifull[islot], iph)) || *abort_flag) {
            *abort_flag = 1;
            break;
        }
        const ItemMeta m = meta[islot];
        if (m.nblk < 0) break;

        // B fragments of Q^T (k = dim, n = head) for this item's GQA group
        uint32_t qf[NT][KS][2];
        {
            const uint8_t* qb = qbuf + islot * C::kQBytes;
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
                const uint8_t* row = qb + (nt * 8 + gid) * D * 2;
#pragma unroll
                for (int kk = 0; kk < KS; ++kk) {
                    qf[nt][kk][0] = *reinterpret_cast<const uint32_t*>(row + (kk * 16 + 2 * t4) * 2);
                    qf[nt][kk][1] = *reinterpret_cast<const uint32_t*>(row + (kk * 16 + 8 + 2 * t4) * 2);
                }
            }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&iempty[islot]);

        float mrun[NT][2], lrun[NT][2];
        float o[NT][KS][4];
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
            mrun[nt][0] = mrun[nt][1] = kNegInf;
            lrun[nt][0] = lrun[nt][1] = 0.f;
#pragma unroll
            for (int i = 0; i < KS; ++i) o[nt][i][0] = o[nt][i][1] = o[nt][i][2] = o[nt][i][3] = 0.f;
        }

        // padding stages in front of the item (see the producer), then the
        // item's blocks: block j is stage item_base + j, owned by warp j % NCW
        const uint32_t item_base = (stage_base + NCW - 1) / NCW * NCW;
        for (uint32_t n = stage_base + (((uint32_t)cw + NCW - stage_base % NCW) % NCW); n < item_base; n += NCW) {
            const int s = n % STAGES;
            if (!__all_sync(0xffffffffu, wait_on(&full[s], (n / STAGES) & 1)) || *abort_flag) {
                *abort_flag = 1;
                break;
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[s]);
        }
        stage_base = item_base;
        const uint32_t item_end = stage_base + (uint32_t)m.nblk;

        // One step of NB blocks (tiles at tb[], valid token counts vl[]):
        // S^T = K Q^T for each block (two accumulator chains per block, the
        // blocks' chains interleaved), one online-softmax update over all NB*16
        // tokens, then O^T += V^T P^T for each block.
        auto step = [&](auto nb_tag, const uint32_t* tb, const int* vl) {
            constexpr int NB = decltype(nb_tag)::value;
            float sa[NB][NT][4], sb[NB][NT][4];
#pragma unroll
            for (int bb = 0; bb < NB; ++bb)
#pragma unroll
                for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                    for (int c = 0; c < 4; ++c) sa[bb][nt][c] = sb[bb][nt][c] = 0.f;
#pragma unroll
            for (int kk = 0; kk < KS; ++kk) {
#pragma unroll
                for (int bb = 0; bb < NB; ++bb) {
                    uint32_t a[4];
                    ldsm_x4(tb[bb] + koff[kk], a[0], a[1], a[2], a[3]);
#pragma unroll
                    for (int nt = 0; nt < NT; ++nt) {
                        if (kk & 1) Mma<T>::run(sb[bb][nt], a, qf[nt][kk][0], qf[nt][kk][1]);
                        else Mma<T>::run(sa[bb][nt], a, qf[nt][kk][0], qf[nt][kk][1]);
                    }
                }
            }

            // ---- online softmax per head column; P^T fragments for the PV product
            uint32_t pb[NB][NT][2], pl[NB][NT][2];
            bool rescale = false;
            float al[NT][2];
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
                float sv[NB][4];
                float mx0 = kNegInf, mx1 = kNegInf;
#pragma unroll
                for (int bb = 0; bb < NB; ++bb) {
#pragma unroll
                    for (int c = 0; c < 4; ++c) sv[bb][c] = (sa[bb][nt][c] + sb[bb][nt][c]) * sl2;
                    if (gid >= vl[bb]) sv[bb][0] = sv[bb][1] = kNegInf;
                    if (gid + 8 >= vl[bb]) sv[bb][2] = sv[bb][3] = kNegInf;
                    mx0 = fmaxf(mx0, fmaxf(sv[bb][0], sv[bb][2]));
                    mx1 = fmaxf(mx1, fmaxf(sv[bb][1], sv[bb][3]));
                }
#pragma unroll
                for (int off = 4; off < 32; off <<= 1) {
                    mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, off));
                    mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, off));
                }
                const float mn0 = fmaxf(mrun[nt][0], mx0), mn1 = fmaxf(mrun[nt][1], mx1);
                const float ms0 = mn0 == kNegInf ? 0.f : mn0, ms1 = mn1 == kNegInf ? 0.f : mn1;
                // alpha = 2^(m_old - m_new), exactly 1 when the running max did not move
                al[nt][0] = mn0 == mrun[nt][0] ? 1.f : fast_exp2(mrun[nt][0] - ms0);
                al[nt][1] = mn1 == mrun[nt][1] ? 1.f : fast_exp2(mrun[nt][1] - ms1);
                rescale |= (al[nt][0] != 1.f) | (al[nt][1] != 1.f);
                mrun[nt][0] = mn0;
                mrun[nt][1] = mn1;
                float l0 = 0.f, l1 = 0.f;
#pragma unroll
                for (int bb = 0; bb < NB; ++bb) {
                    const float p0 = fast_exp2(sv[bb][0] - ms0), p1 = fast_exp2(sv[bb][1] - ms1);
                    const float p2 = fast_exp2(sv[bb][2] - ms0), p3 = fast_exp2(sv[bb][3] - ms1);
                    l0 += p0 + p2;
                    l1 += p1 + p3;
                    const uint32_t h01 = Elt<T>::pack2(p0, p1), h23 = Elt<T>::pack2(p2, p3);
                    pb[bb][nt][0] = movmatrix_t(h01);
                    pb[bb][nt][1] = movmatrix_t(h23);
                    if constexpr (kSplitP) {
                        // remainder of p after bf16 rounding, itself in bf16: hi + lo carries ~16 bits
                        const float2 f01 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&h01));
                        const float2 f23 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&h23));
                        pl[bb][nt][0] = movmatrix_t(Elt<T>::pack2(p0 - f01.x, p1 - f01.y));
                        pl[bb][nt][1] = movmatrix_t(Elt<T>::pack2(p2 - f23.x, p3 - f23.y));
                    }
                }
                lrun[nt][0] = lrun[nt][0] * al[nt][0] + l0;
                lrun[nt][1] = lrun[nt][1] * al[nt][1] + l1;
            }
            if (__any_sync(0xffffffffu, rescale)) {
#pragma unroll
                for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                    for (int i = 0; i < KS; ++i) {
                        o[nt][i][0] *= al[nt][0];
                        o[nt][i][1] *= al[nt][1];
                        o[nt][i][2] *= al[nt][0];
                        o[nt][i][3] *= al[nt][1];
                    }
            }

            // ---- O^T[D x 8*NT] += V^T P^T
#pragma unroll
            for (int i = 0; i < KS; ++i) {
#pragma unroll
                for (int bb = 0; bb < NB; ++bb) {
                    uint32_t a[4];
                    ldsm_x4_t(tb[bb] + voff[i], a[0], a[1], a[2], a[3]);
#pragma unroll
                    for (int nt = 0; nt < NT; ++nt) {
                        Mma<T>::run(o[nt][i], a, pb[bb][nt][0], pb[bb][nt][1]);
                        if constexpr (kSplitP) Mma<T>::run(o[nt][i], a, pl[bb][nt][0], pl[bb][nt][1]);
                    }
                }
            }
        };
        auto tile_of = [&](uint32_t n) { return smem_u32(stages + (n % STAGES) * C::kStageBytes); };
        auto valid_of = [&](uint32_t n) { return min(kChunk, m.ctx - (m.j0 + (int)(n - stage_base)) * kChunk); };
        // The last chunk of a sequence is partly past the context.  Its rows
        // there hold whatever the pool (or an earlier stage) held: the logits
        // of those rows are masked, but a probability of 0 times a NaN in V
        // is still NaN, so the V rows past the context are zeroed first.
        // Returns whether it wrote (the stage then needs a proxy fence before
        // the tensor copies refill it).
        auto clear_v_tail = [&](uint32_t n) {
            const int vl = valid_of(n);
            if (vl >= kChunk) return false;
            const uint32_t vt = tile_of(n) + C::kTileBytes;
            const int per_box = (kChunk - vl) * 8;   // 16-byte pieces past row vl in one 128-byte-wide box
            for (int i = lane; i < C::kBoxes * per_box; i += 32) {
                const int bx = i / per_box, r = i - bx * per_box;
                st_shared_zero16(vt + bx * C::kBoxBytes + vl * 128 + r * 16);
            }
            __syncwarp();
            return true;
        };
        auto wait_full = [&](uint32_t n) {
            if (!__all_sync(0xffffffffu, wait_on(&full[n % STAGES], (n / STAGES) & 1)) || *abort_flag) {
                *abort_flag = 1;
                return false;
            }
            return true;
        };
        // Block j belongs to warp j % NCW, which takes its blocks two at a
        // time (j and j + NCW): that interleaves two blocks' dependent chains,
        // which the warp has no other warp to hide behind.  (Two n-tiles of
        // heads leave no registers for pairs.)
        constexpr bool kPairs = NT == 1;
        uint32_t n = stage_base + (uint32_t)cw;
        while (n < item_end) {
            if (kPairs && n + NCW < item_end) {
                const uint32_t n1 = n + NCW;
                if (!wait_full(n) || !wait_full(n1)) break;
                const bool bad0 = stage_bad[n % STAGES] != 0, bad1 = stage_bad[n1 % STAGES] != 0;
                const uint32_t tb[2] = {tile_of(n), tile_of(n1)};
                const int vl[2] = {valid_of(n), valid_of(n1)};
                // only the later chunk of the pair can end a sequence
                const bool cleared = !bad1 && clear_v_tail(n1);
                if (!bad0 && !bad1) {
                    step(std::integral_constant<int, 2>{}, tb, vl);
                } else {   // a block the producer skipped (bad id) holds no data
                    if (!bad0) step(std::integral_constant<int, 1>{}, tb, vl);
                    if (!bad1) step(std::integral_constant<int, 1>{}, tb + 1, vl + 1);
                }
                if (cleared) fence_proxy_async_shared();
                __syncwarp();
                if (lane == 0) {
                    mbar_arrive(&empty[n % STAGES]);
                    mbar_arrive(&empty[n1 % STAGES]);
                }
                n += 2 * NCW;
            } else {
                if (!wait_full(n)) break;
                bool cleared = false;
                if (!stage_bad[n % STAGES]) {
                    cleared = clear_v_tail(n);
                    const uint32_t tb[1] = {tile_of(n)};
                    const int vl[1] = {valid_of(n)};
                    step(std::integral_constant<int, 1>{}, tb, vl);
                }
                if (cleared) fence_proxy_async_shared();
                __syncwarp();
                if (lane == 0) mbar_arrive(&empty[n % STAGES]);
                n += NCW;
            }
        }
        stage_base = item_end;
        if (*abort_flag) break;

#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int c = 0; c < 2; ++c)
#pragma unroll
                for (int off = 4; off < 32; off <<= 1) lrun[nt][c] += __shfl_xor_sync(0xffffffffu, lrun[nt][c], off);

        if constexpr (NCW == 1) {
            // ---- a single warp owns the whole item: write the result straight from
            // the accumulator fragments (thread holds dims 16i+gid, 16i+gid+8 of heads
            // 2*t4 and 2*t4+1 of each n-tile)
            T* out = static_cast<T*>(p.out);
#pragma unroll
            for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                for (int c = 0; c < 2; ++c) {
                    const int h = nt * 8 + 2 * t4 + c;
                    if (h >= G) continue;
                    const size_t hq = (size_t)m.b * p.num_heads + (size_t)m.g * G + h;
                    if (m.nparts == 1) {
                        const float inv = lrun[nt][c] > 0.f ? 1.f / lrun[nt][c] : 0.f;
#pragma unroll
                        for (int i = 0; i < KS; ++i) {
                            out[hq * D + i * 16 + gid] = Elt<T>::from_f(o[nt][i][c] * inv);
                            out[hq * D + i * 16 + gid + 8] = Elt<T>::from_f(o[nt][i][2 + c] * inv);
                        }
                    } else {
                        const size_t pi = hq * p.max_parts + m.p;
#pragma unroll
                        for (int i = 0; i < KS; ++i) {
                            p.part_o[pi * D + i * 16 + gid] = o[nt][i][c];
                            p.part_o[pi * D + i * 16 + gid + 8] = o[nt][i][2 + c];
                        }
                        if (gid == 0) {
                            p.part_m[pi] = mrun[nt][c];
                            p.part_l[pi] = lrun[nt][c];
                        }
                    }
                }
            if (p.fused_merge && m.nparts > 1) {
                // the CTA that finishes the group's last partition queues it for its merger warp
                __threadfence();
                __syncwarp();
                int prev = 0;
                if (lane == 0) {
                    prev = atomicAdd(&p.merge_count[(size_t)m.b * p.num_kv_heads + m.g], 1);
                    __threadfence();
                }
                prev = __shfl_sync(0xffffffffu, prev, 0);
                if (prev == m.nparts - 1) {
                    const int qs = nq % C::kQSlots;
                    if (!__all_sync(0xffffffffu, wait_on(&qempty[qs], ((nq / C::kQSlots) & 1) ^ 1))) {
                        *abort_flag = 1;
                        break;
                    }
                    if (lane == 0) {
                        tasks[qs] = make_int4(m.b, m.g, m.nparts, 0);
                        mbar_arrive(&qfull[qs]);
                    }
                    ++nq;
                }
            }
            continue;
        }

        // ---- deposit this warp's state in merge buffer iter % 2 (no CTA-wide barrier)
        const int mslot = iter & 1;
        const uint32_t mph = (iter >> 1) & 1;
        if (!__all_sync(0xffffffffu, wait_on(&mempty[mslot], mph ^ 1))) {
            *abort_flag = 1;
            break;
        }
        float* mbuf = merge + mslot * C::kMergeFloats;
        float* mlb = ml + mslot * NCW * C::kHeadsPad * 2;
        {
            float* mo = mbuf + cw * C::kHeadsPad * C::kMergeStride;
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
                const int h0 = nt * 8 + 2 * t4;
#pragma unroll
                for (int i = 0; i < KS; ++i) {
                    const int d = i * 16 + gid;
                    mo[h0 * C::kMergeStride + d] = o[nt][i][0];
                    mo[(h0 + 1) * C::kMergeStride + d] = o[nt][i][1];
                    mo[h0 * C::kMergeStride + d + 8] = o[nt][i][2];
                    mo[(h0 + 1) * C::kMergeStride + d + 8] = o[nt][i][3];
                }
                if (gid == 0) {
                    mlb[(cw * C::kHeadsPad + h0) * 2 + 0] = mrun[nt][0];
                    mlb[(cw * C::kHeadsPad + h0) * 2 + 1] = lrun[nt][0];
                    mlb[(cw * C::kHeadsPad + h0 + 1) * 2 + 0] = mrun[nt][1];
                    mlb[(cw * C::kHeadsPad + h0 + 1) * 2 + 1] = lrun[nt][1];
                }
            }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&mfull[mslot]);

        // ---- the item's merger (warp iter % NCW) combines the NCW states and writes the result
        if (cw == iter % NCW) {
            if (!__all_sync(0xffffffffu, wait_on(&mfull[mslot], mph))) {
                *abort_flag = 1;
                break;
            }
            T* out = static_cast<T*>(p.out);
            for (int h = 0; h < G; ++h) {
                float mw[NCW];
                float M = kNegInf;
#pragma unroll
                for (int w = 0; w < NCW; ++w) {
                    mw[w] = mlb[(w * C::kHeadsPad + h) * 2];
                    M = fmaxf(M, mw[w]);
                }
                const float Ms = M == kNegInf ? 0.f : M;
                float L = 0.f;
#pragma unroll
                for (int w = 0; w < NCW; ++w) {
                    mw[w] = fast_exp2(mw[w] - Ms);
                    L += mw[w] * mlb[(w * C::kHeadsPad + h) * 2 + 1];
                }
                const size_t hq = (size_t)m.b * p.num_heads + (size_t)m.g * G + h;
                const float inv = L > 0.f ? 1.f / L : 0.f;
#pragma unroll
                for (int k = 0; k < D / 32; ++k) {
                    const int d = k * 32 + lane;
                    float acc = 0.f;
#pragma unroll
                    for (int w = 0; w < NCW; ++w) acc += mw[w] * mbuf[(w * C::kHeadsPad + h) * C::kMergeStride + d];
                    if (m.nparts == 1) {
                        out[hq * D + d] = Elt<T>::from_f(acc * inv);
                    } else {
                        p.part_o[(hq * p.max_parts + m.p) * D + d] = acc;
                    }
                }
                if (m.nparts > 1 && lane == 0) {
                    p.part_m[hq * p.max_parts + m.p] = M;
                    p.part_l[hq * p.max_parts + m.p] = L;
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&mempty[mslot]);
        }
    }
    if constexpr (NCW == 1) {
        // tell the merger warp there is nothing more
        const int qs = nq % C::kQSlots;
        const bool okq = __all_sync(0xffffffffu, wait_on(&qempty[qs], ((nq / C::kQSlots) & 1) ^ 1));
        if (lane == 0) {
            if (!okq) *abort_flag = 1;
            tasks[qs] = make_int4(-1, 0, 0, 0);
            mbar_arrive(&qfull[qs]);
        }
    }
    if (*abort_flag && lane == 0) set_status(p.status, PA_ERR_TIMEOUT);
}

// ===========================================================================
// 2b. partition kernel, SIMT (any dtype, any group size)
// ===========================================================================
// One warp per (item, query head of the group).  Lane l owns dims
// [l*E, l*E + E) of the head; a token's logit is a warp all-reduce.
template <typename T, int D, int NW>
__global__ void __launch_bounds__(NW * 32) decode_simt_kernel(const DecodeParams p) {
    constexpr int E = D / 32;
    griddep_wait();
    const int n_items = p.hdr[kHdrItems];
    const int G = p.group;
    const int lane = threadIdx.x & 31;
    const T* qp = static_cast<const T*>(p.q);
    const T* kc = static_cast<const T*>(p.key_cache);
    const T* vc = static_cast<const T*>(p.value_cache);
    T* out = static_cast<T*>(p.out);
    const long long units = (long long)n_items * G;
    for (long long u = (long long)blockIdx.x * NW + (threadIdx.x >> 5); u < units; u += (long long)gridDim.x * NW) {
        const int rank = (int)(u / G), h = (int)(u % G);
        const ItemGeom m = item_geom(p, p.items[rank]);
        const size_t hq = (size_t)m.b * p.num_heads + (size_t)m.g * G + h;
        float qv[E], acc[E];
#pragma unroll
        for (int e = 0; e < E; ++e) {
            qv[e] = Elt<T>::to_f(qp[hq * D + lane * E + e]);
            acc[e] = 0.f;
        }
        float mrun = kNegInf, lrun = 0.f;
        const int bs = p.block_size;
        const int32_t* row = p.block_tables + (size_t)m.b * p.max_blocks_per_seq;
        for (int j = 0; j < m.nblk; ++j) {
            // the 16-token chunk's block (8-token blocks: its two blocks); a bad
            // id drops the whole chunk, as in the tensor-core kernel
            const int pos0 = (m.j0 + j) * kChunk;
            const int ntok = min(kChunk, m.ctx - pos0);
            const int blk0 = row[pos0 / bs];
            const int blk1 = ntok > bs ? row[pos0 / bs + 1] : blk0;
            if (blk0 < 0 || blk0 >= p.num_blocks || blk1 < 0 || blk1 >= p.num_blocks) {
                if (lane == 0) set_status(p.status, PA_ERR_OUT_OF_RANGE);
                continue;
            }
            for (int t = 0; t < ntok; ++t) {
                const int pos = pos0 + t;
                const size_t tok = (((size_t)(t < bs ? blk0 : blk1) * p.num_kv_heads + m.g) * bs + pos % bs) * D;
                const T* kr = kc + tok + lane * E;
                const T* vr = vc + tok + lane * E;
                float dot = 0.f;
#pragma unroll
                for (int e = 0; e < E; ++e) dot += qv[e] * Elt<T>::to_f(kr[e]);
#pragma unroll
                for (int off = 16; off > 0; off >>= 1) dot += __shfl_xor_sync(0xffffffffu, dot, off);
                const float s = dot * p.scale_log2;
                const float mn = fmaxf(mrun, s);
                const float al = fast_exp2(mrun - mn), pe = fast_exp2(s - mn);
                lrun = lrun * al + pe;
#pragma unroll
                for (int e = 0; e < E; ++e) acc[e] = acc[e] * al + pe * Elt<T>::to_f(vr[e]);
                mrun = mn;
            }
        }
        if (m.nparts == 1) {
#pragma unroll
            for (int e = 0; e < E; ++e) out[hq * D + lane * E + e] = Elt<T>::from_f(lrun > 0.f ? acc[e] / lrun : 0.f);
        } else {
            const size_t pi = hq * p.max_parts + m.p;
#pragma unroll
            for (int e = 0; e < E; ++e) p.part_o[pi * D + lane * E + e] = acc[e];
            if (lane == 0) {
                p.part_m[pi] = mrun;
                p.part_l[pi] = lrun;
            }
        }
    }
}

// ===========================================================================
// 3. reduce
// ===========================================================================
// Rows (sequence, query head); a CTA takes rows in turn and skips those of
// sequences with one partition, which the partition kernel finished.  Its 4
// warps split a row's partitions (warp w takes partitions w, w + 4, ...; lane
// l owns D/32 consecutive dims), then add up through shared memory.  Loads
// are cache-global: the partials were written by other SMs in the previous
// kernel.
template <typename T, int D>
__global__ void __launch_bounds__(128) decode_reduce_kernel(const DecodeParams p) {
    constexpr int kW = 4, E = D / 32, U = 8;
    __shared__ float sacc[kW][D];
    __shared__ float sl[kW];
    griddep_wait();
    const int wid = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int Hq = p.num_heads;
    const long long n_rows = (long long)p.num_seqs * Hq;
    for (long long r = blockIdx.x; r < n_rows; r += gridDim.x) {
        const int b = (int)(r / Hq), h = (int)(r % Hq);
        const int ctx = load_ctx(p, b, false);
        const int nparts = max(1, ceil_div_i(ceil_div_i(ctx, kChunk), p.part_blocks));
        if (nparts == 1) continue;   // (uniform over the CTA)
        const size_t base = ((size_t)b * Hq + h) * p.max_parts;
        float M = kNegInf;
        for (int q = lane; q < nparts; q += 32) M = fmaxf(M, __ldcg(p.part_m + base + q));
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, off));
        const float Ms = M == kNegInf ? 0.f : M;
        float L = 0.f, acc[E];
#pragma unroll
        for (int e = 0; e < E; ++e) acc[e] = 0.f;
        for (int q0 = wid; q0 < nparts; q0 += kW * U) {
            float w[U], v[U][E];
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const int q = q0 + u * kW;
                w[u] = 0.f;
                if (q < nparts) {
                    w[u] = fast_exp2(__ldcg(p.part_m + base + q) - Ms);
                    L += w[u] * __ldcg(p.part_l + base + q);
                    const float* po = p.part_o + (base + q) * D + lane * E;
#pragma unroll
                    for (int e = 0; e < E; ++e) v[u][e] = __ldcg(po + e);
                } else {
#pragma unroll
                    for (int e = 0; e < E; ++e) v[u][e] = 0.f;
                }
            }
#pragma unroll
            for (int u = 0; u < U; ++u)
#pragma unroll
                for (int e = 0; e < E; ++e) acc[e] += w[u] * v[u][e];
        }
#pragma unroll
        for (int e = 0; e < E; ++e) sacc[wid][lane * E + e] = acc[e];
        if (lane == 0) sl[wid] = L;
        __syncthreads();
        if (threadIdx.x < D) {
            float a = 0.f, lt = 0.f;
#pragma unroll
            for (int w2 = 0; w2 < kW; ++w2) {
                a += sacc[w2][threadIdx.x];
                lt += sl[w2];
            }
            static_cast<T*>(p.out)[((size_t)b * Hq + h) * D + threadIdx.x] =
                Elt<T>::from_f(lt > 0.f ? a * (1.f / lt) : 0.f);
        }
        __syncthreads();
    }
}

// ===========================================================================
// host side
// ===========================================================================
static PFN_cuTensorMapEncodeTiled_v12000 get_encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = []() -> PFN_cuTensorMapEncodeTiled_v12000 {
        void* f = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) != cudaSuccess ||
            q != cudaDriverEntryPointSuccess)
            return nullptr;
        return reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(f);
    }();
    return fn;
}

// 2-D view of a pool: rows of head_dim elements, one row per (block, KV head, slot);
// a box is 16 rows (8 for 8-token blocks) x 64 elements (128 B), 128-byte
// swizzled in shared memory.
cudaError_t make_pool_map(CUtensorMap* map, const void* pool, pa_dtype dtype, int num_blocks, int num_kv_heads,
                          int head_dim, int block_size) {
    auto encode = get_encode_fn();
    if (!encode) return cudaErrorNotSupported;
    const cuuint64_t dims[2] = {(cuuint64_t)head_dim, (cuuint64_t)num_blocks * num_kv_heads * block_size};
    const cuuint64_t strides[1] = {(cuuint64_t)head_dim * 2};
    const cuuint32_t box[2] = {64, (cuuint32_t)(block_size < kChunk ? block_size : kChunk)};
    const cuuint32_t estr[2] = {1, 1};
    const CUtensorMapDataType dt =
        dtype == PA_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
    const CUresult r = encode(map, dt, 2, const_cast<void*>(pool), dims, strides, box, estr,
                              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

namespace {

// Shapes of the tensor-core partition kernel (consumer warps x ring stages; CTAs per SM
// at D = 128 and a GQA group of at most 8, as shared memory allows):
//   kPaired: 2 x 10 (80 KB ring), 2 CTAs per SM, warps merge through shared memory
//   kQuad:   1 x 6  (48 KB ring), 4 CTAs per SM, one warp per item, no merge
//   kTriple: 1 x 8  (64 KB ring), 3 CTAs per SM
//   kPair1:  1 x 13 (104 KB ring), 2 CTAs per SM
// The ring holds the bytes in flight that cover HBM latency; each consumer
// warp holds two stages while it computes.  kQuad is the automatic choice
// (measured best on every workload once consumers took two blocks per step);
// the others are selectable through DecodeOptions (pa_tuning.h) for tuning
// and for the tests.
enum class TcShape { kAuto, kPaired, kQuad, kTriple, kPair1 };
TcShape tc_shape(const DecodeOptions& o) {
    switch (o.shape) {
        case PA_SHAPE_PAIRED: return TcShape::kPaired;
        case PA_SHAPE_QUAD: return TcShape::kQuad;
        case PA_SHAPE_TRIPLE: return TcShape::kTriple;
        case PA_SHAPE_PAIR1: return TcShape::kPair1;
        default: return TcShape::kAuto;
    }
}

template <int NT_, int NCW_, int ST_>
struct TcTag {
    static constexpr int NT = NT_, NCW = NCW_, ST = ST_;
};

// calls f(TcTag<NT, NCW, STAGES>{}) for the kernel instance of a shape
template <typename F>
cudaError_t dispatch_shape(int group, TcShape sh, F&& f) {
    if (group > 8) return f(TcTag<2, 1, 6>{});
    switch (sh) {
        case TcShape::kPaired: return f(TcTag<1, 2, 10>{});
        case TcShape::kTriple: return f(TcTag<1, 1, 8>{});
        case TcShape::kPair1: return f(TcTag<1, 1, 13>{});
        default: return f(TcTag<1, 1, 6>{});
    }
}

constexpr int kSelfPlanMaxSeqs = 256;

// What launch_decode enqueues for a problem.
struct DecodeChoice {
    bool tc = false;         // tensor-core partition kernel (else SIMT)
    TcShape shape = TcShape::kAuto;
    bool fused = false;      // the partition kernel merges partitions (no reduce kernel)
    bool self_plan = false;  // CTAs plan their own items (no plan kernel)
    bool reduce = false;
    int grid = 1;            // partition-kernel CTAs
    int launches = 0;
};

// grid of a tensor-core instance (one wave of resident CTAs) and whether it can self-plan
template <typename T, int D, int NT, int NCW, int STAGES>
cudaError_t tc_choice(const DecodeParams& p, const DecodeOptions& o, long long max_items, DecodeChoice* c) {
    using Cfg = TcCfg<D, NT, NCW, STAGES>;
    auto kernel = decode_tc_kernel<T, D, NT, NCW, STAGES>;
    // the attribute is per device: set it on every call (a cheap host-side call)
    cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg::kSmemBytes);
    if (e != cudaSuccess) return e;
    e = prefer_max_shared(reinterpret_cast<const void*>(kernel));
    if (e != cudaSuccess) return e;
    DeviceInfo dev;
    e = device_info(&dev);
    if (e != cudaSuccess) return e;
    int ctas_per_sm = 1;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&ctas_per_sm, kernel, Cfg::kThreads, Cfg::kSmemBytes);
    if (e != cudaSuccess) return e;
    if (ctas_per_sm < 1) return cudaErrorInvalidConfiguration;
    long long grid = (long long)dev.sm_count * ctas_per_sm;
    if (grid > max_items) grid = max_items;
    if (grid < 1) grid = 1;
    c->grid = (int)grid;
    // Each self-planning CTA scans all of context_lens; past a few hundred
    // sequences one plan kernel is cheaper (measured: equal at 256, the plan
    // kernel 3.6% faster at 1024, self-planning 2-11% faster at 8 and 32).
    c->self_plan = !o.force_plan_kernel && !o.planned && p.num_seqs <= kSelfPlanMaxSeqs && p.num_seqs <= Cfg::kPlanSeqs &&
                   (long long)p.num_seqs * p.num_kv_heads <= kCounterSlots &&
                   (max_items + grid - 1) / grid <= Cfg::kMaxOwn;
    return cudaSuccess;
}

template <typename T, int D>
cudaError_t choose(const DecodeParams& p, const DecodeOptions& o, pa_dtype dtype, DecodeChoice* c) {
    const long long max_items = (long long)p.num_seqs * p.max_parts * p.num_kv_heads;
    *c = DecodeChoice{};
    if constexpr (!std::is_same<T, float>::value) {
        if (decode_path(dtype, D, p.group) == DecodePath::kTensorCore) {
            c->tc = true;
            TcShape sh = tc_shape(o);
            // Automatic: four single-warp CTAs per SM, which merge partitions
            // themselves when there are at most kFusedMaxParts of them.
            if (sh == TcShape::kAuto) sh = TcShape::kQuad;
            c->shape = sh;
            const bool one_warp = p.group > 8 || sh != TcShape::kPaired;
            c->fused = one_warp && p.max_parts > 1 && p.max_parts <= kFusedMaxParts;
            const cudaError_t e = dispatch_shape(p.group, sh, [&](auto tag) {
                using Tg = decltype(tag);
                return tc_choice<T, D, Tg::NT, Tg::NCW, Tg::ST>(p, o, max_items, c);
            });
            if (e != cudaSuccess) return e;
        }
    }
    c->reduce = p.max_parts > 1 && !c->fused;
    c->launches = ((c->self_plan || o.planned) ? 0 : 1) + 1 + (c->reduce ? 1 : 0);
    return cudaSuccess;
}

template <typename T, int D, int NT, int NCW, int STAGES>
cudaError_t launch_tc(const DecodeParams& p, pa_dtype dtype, cudaStream_t stream, int grid) {
    using Cfg = TcCfg<D, NT, NCW, STAGES>;
    CUtensorMap mk, mv;
    cudaError_t e = make_pool_map(&mk, p.key_cache, dtype, p.num_blocks, p.num_kv_heads, D, p.block_size);
    if (e != cudaSuccess) return e;
    e = make_pool_map(&mv, p.value_cache, dtype, p.num_blocks, p.num_kv_heads, D, p.block_size);
    if (e != cudaSuccess) return e;
    return launch_pdl(decode_tc_kernel<T, D, NT, NCW, STAGES>, dim3(grid), dim3(Cfg::kThreads), Cfg::kSmemBytes,
                      stream, p, mk, mv);
}

template <typename T, int D>
cudaError_t launch_simt(const DecodeParams& p, cudaStream_t stream, long long max_items) {
    DeviceInfo dev;
    cudaError_t e = device_info(&dev);
    if (e != cudaSuccess) return e;
    constexpr int NW = 4;
    long long want = (max_items * p.group + NW - 1) / NW;
    long long cap = (long long)dev.sm_count * 8;
    int grid = (int)(want < cap ? want : cap);
    if (grid < 1) grid = 1;
    return launch_pdl(decode_simt_kernel<T, D, NW>, dim3(grid), dim3(NW * 32), 0, stream, p);
}

// plan: one CTA; 256 threads cover typical batches in one pass, 1024 large ones
cudaError_t launch_plan(const DecodeParams& p, cudaStream_t stream) {
    return p.num_seqs <= 256 ? launch_pdl(decode_plan_kernel<256>, dim3(1), dim3(256), 0, stream, p)
                             : launch_pdl(decode_plan_kernel<1024>, dim3(1), dim3(1024), 0, stream, p);
}

template <typename T, int D>
cudaError_t launch_all(DecodeParams p, const DecodeOptions& o, pa_dtype dtype, cudaStream_t stream) {
    DecodeChoice c;
    cudaError_t e = choose<T, D>(p, o, dtype, &c);
    if (e != cudaSuccess) return e;
    p.fused_merge = c.fused ? 1 : 0;
    p.self_plan = c.self_plan ? 1 : 0;
    // a planned call reads the list an earlier pa_decode_plan left in the workspace
    if (!c.self_plan && !o.planned) {
        e = launch_plan(p, stream);
        if (e != cudaSuccess) return e;
    }
    if constexpr (std::is_same<T, float>::value) {
        e = launch_simt<T, D>(p, stream, (long long)p.num_seqs * p.max_parts * p.num_kv_heads);
    } else {
        if (c.tc) {
            e = dispatch_shape(p.group, c.shape, [&](auto tag) {
                using Tg = decltype(tag);
                return launch_tc<T, D, Tg::NT, Tg::NCW, Tg::ST>(p, dtype, stream, c.grid);
            });
        } else {
            e = launch_simt<T, D>(p, stream, (long long)p.num_seqs * p.max_parts * p.num_kv_heads);
        }
    }
    if (e != cudaSuccess) return e;
    if (c.reduce) {
        DeviceInfo dev;
        e = device_info(&dev);
        if (e != cudaSuccess) return e;
        const long long rows = (long long)p.num_seqs * p.num_heads;
        const long long cap = (long long)dev.sm_count * 8;
        e = launch_pdl(decode_reduce_kernel<T, D>, dim3((unsigned)(rows < cap ? rows : cap)), dim3(128), 0, stream, p);
    }
    return e;
}

}  // namespace

DecodePath decode_path(pa_dtype dtype, int head_dim, int group) {
    (void)head_dim;
    if (dtype == PA_F32 || group > 16) return DecodePath::kSimt;
    return DecodePath::kTensorCore;
}

cudaError_t launch_decode(const DecodeParams& p, const DecodeOptions& o, pa_dtype dtype, cudaStream_t stream) {
    switch (dtype) {
        case PA_F32: return p.head_dim == 64 ? launch_all<float, 64>(p, o, dtype, stream)
                                             : launch_all<float, 128>(p, o, dtype, stream);
        case PA_F16: return p.head_dim == 64 ? launch_all<__half, 64>(p, o, dtype, stream)
                                             : launch_all<__half, 128>(p, o, dtype, stream);
        case PA_BF16: return p.head_dim == 64 ? launch_all<__nv_bfloat16, 64>(p, o, dtype, stream)
                                              : launch_all<__nv_bfloat16, 128>(p, o, dtype, stream);
    }
    return cudaErrorInvalidValue;
}

cudaError_t decode_launch_count(const DecodeParams& p, const DecodeOptions& o, pa_dtype dtype, int* launches) {
    DecodeChoice c;
    cudaError_t e = cudaErrorInvalidValue;
    switch (dtype) {
        case PA_F32:
            e = p.head_dim == 64 ? choose<float, 64>(p, o, dtype, &c) : choose<float, 128>(p, o, dtype, &c);
            break;
        case PA_F16:
            e = p.head_dim == 64 ? choose<__half, 64>(p, o, dtype, &c) : choose<__half, 128>(p, o, dtype, &c);
            break;
        case PA_BF16:
            e = p.head_dim == 64 ? choose<__nv_bfloat16, 64>(p, o, dtype, &c)
                                 : choose<__nv_bfloat16, 128>(p, o, dtype, &c);
            break;
    }
    if (e == cudaSuccess) *launches = c.launches;
    return e;
}

int decode_fused_max_parts() { return kFusedMaxParts; }

cudaError_t launch_decode_plan(const DecodeParams& p, cudaStream_t stream) { return launch_plan(p, stream); }

}  // namespace pa
