// Paged decode attention on sm_100a.
//
// What is computed (the pages: "PagedAttention" digest, sections
// "PagedAttention in one picture", "Why the attention kernel works at all",
// "Misconceptions"): for each sequence b and query head h, ordinary softmax
// attention of q[b,h] over the sequence's K/V, which the kernel reaches by
// walking the block table; the result is that of contiguous attention.
//
// How (three kernels, chained with programmatic dependent launch):
//
//  1. plan    -- one CTA turns context_lens into a work list of items
//                (sequence b, partition p, KV head g), largest first: all full
//                partitions, then partial ones by decreasing block count,
//                then empty sequences.  Partition p of b covers logical blocks
//                [p*PB, min((p+1)*PB, ceil(ctx/16))).
//  2. partition kernel -- persistent CTAs, one or two per SM.  CTA c takes
//                items c, 2C-1-c, 2C+c, ... (snake order over the sorted list,
//                which balances the load).  Per CTA:
//                  * one producer warp streams, for each item, the Q rows of
//                    the GQA group (1-D bulk copy) and every (block, KV head)
//                    tile of K and of V (16 tokens x head_dim, contiguous
//                    4 KB at D = 128) with 2-D TMA tensor copies into a ring of
//                    shared-memory stages, 128-byte swizzled, tracked by
//                    mbarriers, evict-first in L2;
//                  * consumer warps take the item's blocks round-robin and run
//                    on tensor cores: S^T = K Q^T (m16n8k16, tokens x heads,
//                    the GQA group padded to 8 or 16 columns), an online
//                    softmax in fp32 (column max by warp shuffles, 2^x on
//                    log2-scaled logits), then O^T += V^T P^T with P
//                    transposed in registers (movmatrix);
//                  * at the end of an item the consumer warps merge their
//                    (max, sum, O) through shared memory and write either the
//                    final output (single-partition sequence) or the
//                    partition's (m, l, O) to the workspace.
//                A SIMT variant serves float32 and groups above 16.
//  3. reduce  -- one warp per (b, h) of a multi-partition sequence:
//                M = max m_p, L = sum l_p 2^(m_p - M),
//                out = sum O_p 2^(m_p - M) / L.
#include <cstdlib>
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
__global__ void __launch_bounds__(1024) decode_plan_kernel(const DecodeParams p) {
    __shared__ int cnt[kMaxPartBlocks + 1];
    __shared__ int cursor[kMaxPartBlocks + 1];
    griddep_wait();
    const int PB = p.part_blocks, Hkv = p.num_kv_heads;
    const int lane = threadIdx.x & 31;
    for (int i = threadIdx.x; i <= PB; i += blockDim.x) cnt[i] = 0;
    __syncthreads();
    // pass 1: histogram of item sizes (in blocks)
    for (int b0 = 0; b0 < p.num_seqs; b0 += blockDim.x) {
        const int b = b0 + threadIdx.x;
        int nfull = 0, tail = -1;
        if (b < p.num_seqs) {
            const int nblk = ceil_div_i(load_ctx(p, b, true), kBlockSize);
            nfull = nblk / PB;
            const int t = nblk - nfull * PB;
            if (t > 0 || nblk == 0) tail = t;
        }
        const int wsum = __reduce_add_sync(0xffffffffu, nfull);
        if (lane == 0 && wsum) atomicAdd(&cnt[PB], wsum);
        if (tail >= 0) atomicAdd(&cnt[tail], 1);
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        int acc = 0;
        for (int s = PB; s >= 0; --s) {
            cursor[s] = acc;
            acc += cnt[s] * Hkv;
        }
        *p.n_items = acc;
    }
    __syncthreads();
    // pass 2: place items (order inside a size class is irrelevant)
    for (int b0 = 0; b0 < p.num_seqs; b0 += blockDim.x) {
        const int b = b0 + threadIdx.x;
        int nfull = 0, tail = -1, ctx = 0;
        if (b < p.num_seqs) {
            ctx = load_ctx(p, b, false);
            const int nblk = ceil_div_i(ctx, kBlockSize);
            nfull = nblk / PB;
            const int t = nblk - nfull * PB;
            if (t > 0 || nblk == 0) tail = t;
        }
        // warp-aggregated reservation in the full-partition class
        const int mine = nfull * Hkv;
        int incl = mine;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int v = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += v;
        }
        int base = 0;
        if (lane == 31 && incl) base = atomicAdd(&cursor[PB], incl);
        base = __shfl_sync(0xffffffffu, base, 31) + incl - mine;
        for (int j = 0; j < nfull; ++j)
            for (int g = 0; g < Hkv; ++g) p.items[base + j * Hkv + g] = make_int4(b, (j << 8) | g, ctx, 0);
        if (tail >= 0) {
            const int tb = atomicAdd(&cursor[tail], Hkv);
            for (int g = 0; g < Hkv; ++g) p.items[tb + g] = make_int4(b, (nfull << 8) | g, ctx, 0);
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
    const int nblk_total = ceil_div_i(m.ctx, kBlockSize);
    m.j0 = m.p * p.part_blocks;
    m.nblk = max(0, min(p.part_blocks, nblk_total - m.j0));
    m.nparts = max(1, ceil_div_i(nblk_total, p.part_blocks));
    return m;
}

// snake assignment of sorted items to persistent CTAs
__device__ __forceinline__ int item_rank(int iter, int cta, int ctas) {
    return iter * ctas + ((iter & 1) ? (ctas - 1 - cta) : cta);
}

// ===========================================================================
// 2a. partition kernel, tensor cores (fp16 / bf16)
// ===========================================================================
struct ItemMeta {
    int b, g, p, ctx, j0, nblk, nparts, pad;
};

// work-list entry and table row of one item, prefetched by the producer
struct DescSlot {
    int4 e;
    int bt[kMaxPartBlocks];
};

template <int D, int NT, int NCW, int STAGES>
struct TcCfg {
    static constexpr int kBoxes = D / 64;                    // 64-element (128 B) boxes per tile row
    static constexpr int kBoxBytes = kBlockSize * 128;       // 2 KB
    static constexpr int kTileBytes = kBlockSize * D * 2;    // one K or V tile
    static constexpr int kStageBytes = 2 * kTileBytes;
    static constexpr int kISlots = 4;                        // item metadata / Q ring
    static constexpr int kDSlots = 4;                        // descriptor prefetch ring
    static constexpr int kHeadsPad = 8 * NT;
    static constexpr int kQBytes = kHeadsPad * D * 2;
    static constexpr int kMergeStride = D + 4;               // floats per head row (bank-conflict pad)
    static constexpr int kOffStages = 0;
    static constexpr int kOffQ = kOffStages + STAGES * kStageBytes;
    static constexpr int kOffMerge = kOffQ + kISlots * kQBytes;
    static constexpr int kOffMl = kOffMerge + NCW * kHeadsPad * kMergeStride * 4;
    static constexpr int kOffDesc = kOffMl + NCW * kHeadsPad * 2 * 4;
    static constexpr int kOffMeta = kOffDesc + kDSlots * (int)sizeof(DescSlot);
    static constexpr int kOffBar = kOffMeta + kISlots * (int)sizeof(ItemMeta);
    static constexpr int kOffFlags = kOffBar + (2 * STAGES + 2 * kISlots) * 8;
    static constexpr int kBytes = kOffFlags + 16 + STAGES * 4;
    static constexpr int kSmemBytes = kBytes + 1024;         // slack for 1024-byte alignment
    static constexpr int kThreads = (NCW + 1) * 32;
    static_assert(kOffDesc % 16 == 0 && sizeof(DescSlot) % 16 == 0, "cp.async 16-byte destinations");
    // Ring stage n and stage n + STAGES reuse one slot and one parity bit.  A
    // consumer may only wait for stage n once stage n - STAGES (same slot, same
    // parity) has been consumed, or it would take the old phase for the new
    // one.  Within an item, block j goes to warp j % NCW, so with STAGES a
    // multiple of NCW both stages belong to the same warp, which takes them in
    // order; across items, the merge barrier at each item's end orders them.
    static_assert(STAGES % NCW == 0, "ring depth must be a multiple of the consumer warps");
};

template <typename T, int D, int NT, int NCW, int STAGES>
__global__ void __launch_bounds__((NCW + 1) * 32, 1)
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
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::kOffFlags);
    volatile int* stage_bad = reinterpret_cast<volatile int*>(smem + C::kOffFlags + 16);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int G = p.group;

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int i = 0; i < C::kISlots; ++i) {
            mbar_init(&ifull[i], 1);
            mbar_init(&iempty[i], NCW);
        }
        *abort_flag = 0;
        mbar_fence_init();
    }
    // rows of the padded GQA group beyond G stay zero; TMA fills rows < G
    for (int i = threadIdx.x; i < C::kISlots * C::kQBytes / 16; i += blockDim.x)
        reinterpret_cast<uint4*>(qbuf)[i] = make_uint4(0, 0, 0, 0);
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    __syncthreads();

    griddep_wait();
    const int n_items = *p.n_items;
    const int ctas = gridDim.x, cta = blockIdx.x;
    const int PB = p.part_blocks;

    if (warp == NCW) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            prefetch_tensormap(&tmK);
            prefetch_tensormap(&tmV);
        }
        const uint64_t pol = policy_evict_first();
        const size_t q_row_bytes = (size_t)D * 2;

        // Descriptor pipeline, so that no global-memory latency sits between
        // two items' tile loads: item k's work-list entry and table row land
        // (cp.async) in slot k % kDSlots.  At the top of iteration i, entry(i),
        // row(i) and entry(i+1) are visible and the group {row(i+1),
        // entry(i+2)} is in flight; it completes while item i's tiles are
        // being issued.
        auto fetch_entry = [&](int it) {
            const int r = item_rank(it, cta, ctas);
            if (lane == 0 && r < n_items) cp_async_16(smem_u32(&dsc[it % C::kDSlots].e), &p.items[r]);
        };
        auto fetch_row = [&](int it) {
            const int r = item_rank(it, cta, ctas);
            if (r >= n_items) return;
            const int4 e = dsc[it % C::kDSlots].e;
            const int j0 = (e.y >> 8) * PB;
            const int nblk = min(PB, ceil_div_i(e.z, kBlockSize) - j0);
            if (lane < nblk)
                cp_async_4(smem_u32(&dsc[it % C::kDSlots].bt[lane]),
                           p.block_tables + (size_t)e.x * p.max_blocks_per_seq + j0 + lane);
        };
        fetch_entry(0);
        cp_async_commit();
        cp_async_wait_all();
        __syncwarp();
        fetch_row(0);
        fetch_entry(1);
        cp_async_commit();
        cp_async_wait_all();
        __syncwarp();
        fetch_row(1);
        fetch_entry(2);
        cp_async_commit();

        uint32_t stage = 0;
        bool ok = true;
        for (int iter = 0; ok; ++iter) {
            const int rank = item_rank(iter, cta, ctas);
            const int islot = iter % C::kISlots;
            const uint32_t iph = (iter / C::kISlots) & 1;
            int okw = 1;
            if (lane == 0) okw = mbar_wait(&iempty[islot], iph ^ 1);
            if (!__shfl_sync(0xffffffffu, okw, 0)) { ok = false; break; }
            if (rank >= n_items) {
                if (lane == 0) {
                    meta[islot].nblk = -1;
                    mbar_arrive(&ifull[islot]);
                }
                break;
            }
            const DescSlot& d = dsc[iter % C::kDSlots];
            const ItemGeom m = item_geom(p, d.e);
            if (lane == 0) {
                meta[islot] = ItemMeta{m.b, m.g, m.p, m.ctx, m.j0, m.nblk, m.nparts, 0};
                const uint32_t qbytes = (uint32_t)(G * q_row_bytes);
                mbar_arrive_expect_tx(&ifull[islot], qbytes);
                bulk_load_1d(smem_u32(qbuf + islot * C::kQBytes),
                             static_cast<const uint8_t*>(p.q) + ((size_t)m.b * p.num_heads + (size_t)m.g * G) * q_row_bytes,
                             qbytes, &ifull[islot]);
                for (int j = 0; j < m.nblk; ++j, ++stage) {
                    const int blk = d.bt[j];
                    const int s = stage % STAGES;
                    if (!mbar_wait(&empty[s], ((stage / STAGES) & 1) ^ 1)) { okw = 0; break; }
                    if (blk >= 0 && blk < p.num_blocks) {
                        stage_bad[s] = 0;
                        mbar_arrive_expect_tx(&full[s], C::kStageBytes);
                        const int y = (blk * p.num_kv_heads + m.g) * kBlockSize;
                        const uint32_t kdst = smem_u32(stages + s * C::kStageBytes);
#pragma unroll
                        for (int h = 0; h < C::kBoxes; ++h)
                            tma_load_2d(kdst + h * C::kBoxBytes, &tmK, h * 64, y, &full[s], pol);
#pragma unroll
                        for (int h = 0; h < C::kBoxes; ++h)
                            tma_load_2d(kdst + C::kTileBytes + h * C::kBoxBytes, &tmV, h * 64, y, &full[s], pol);
                    } else {
                        stage_bad[s] = 1;
                        set_status(p.status, PA_ERR_OUT_OF_RANGE);
                        mbar_arrive(&full[s]);
                    }
                }
            }
            stage = __shfl_sync(0xffffffffu, stage, 0);
            if (!__shfl_sync(0xffffffffu, okw, 0) || *abort_flag) { ok = false; break; }
            // descriptors of items iter+2 and iter+3 start loading; item iter+1's are ready
            cp_async_wait_all();
            __syncwarp();
            fetch_row(iter + 2);
            fetch_entry(iter + 3);
            cp_async_commit();
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
                    mbar_wait(&full[n % STAGES], (n / STAGES) & 1);
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
        if (!__all_sync(0xffffffffu, mbar_wait(&ifull[islot], iph)) || *abort_flag) {
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

        for (int j = cw; j < m.nblk; j += NCW) {
            const uint32_t n = stage_base + j;
            const int s = n % STAGES;
            if (!__all_sync(0xffffffffu, mbar_wait(&full[s], (n / STAGES) & 1)) || *abort_flag) {
                *abort_flag = 1;
                break;
            }
            if (!stage_bad[s]) {
                const int valid = min(kBlockSize, m.ctx - (m.j0 + j) * kBlockSize);
                const uint32_t tbase = smem_u32(stages + s * C::kStageBytes);

                // ---- S^T[16 tokens x 8*NT heads] = K Q^T, two accumulator chains
                float sa[NT][4], sb[NT][4];
#pragma unroll
                for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                    for (int c = 0; c < 4; ++c) sa[nt][c] = sb[nt][c] = 0.f;
#pragma unroll
                for (int kk = 0; kk < KS; ++kk) {
                    uint32_t a[4];
                    ldsm_x4(tbase + koff[kk], a[0], a[1], a[2], a[3]);
#pragma unroll
                    for (int nt = 0; nt < NT; ++nt) {
                        if (kk & 1) Mma<T>::run(sb[nt], a, qf[nt][kk][0], qf[nt][kk][1]);
                        else Mma<T>::run(sa[nt], a, qf[nt][kk][0], qf[nt][kk][1]);
                    }
                }

                // ---- online softmax per head column; P^T fragments for the PV product
                uint32_t pb[NT][2], pl[NT][2];
                bool rescale = false;
                float al[NT][2];
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) {
                    float s0 = (sa[nt][0] + sb[nt][0]) * sl2, s1 = (sa[nt][1] + sb[nt][1]) * sl2;
                    float s2 = (sa[nt][2] + sb[nt][2]) * sl2, s3 = (sa[nt][3] + sb[nt][3]) * sl2;
                    if (gid >= valid) s0 = s1 = kNegInf;
                    if (gid + 8 >= valid) s2 = s3 = kNegInf;
                    float mx0 = fmaxf(s0, s2), mx1 = fmaxf(s1, s3);
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
                    const float p0 = fast_exp2(s0 - ms0), p1 = fast_exp2(s1 - ms1);
                    const float p2 = fast_exp2(s2 - ms0), p3 = fast_exp2(s3 - ms1);
                    lrun[nt][0] = lrun[nt][0] * al[nt][0] + (p0 + p2);
                    lrun[nt][1] = lrun[nt][1] * al[nt][1] + (p1 + p3);
                    const uint32_t h01 = Elt<T>::pack2(p0, p1), h23 = Elt<T>::pack2(p2, p3);
                    pb[nt][0] = movmatrix_t(h01);
                    pb[nt][1] = movmatrix_t(h23);
                    if constexpr (kSplitP) {
                        // remainder of p after bf16 rounding, itself in bf16: hi + lo carries ~16 bits
                        const float2 f01 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&h01));
                        const float2 f23 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&h23));
                        pl[nt][0] = movmatrix_t(Elt<T>::pack2(p0 - f01.x, p1 - f01.y));
                        pl[nt][1] = movmatrix_t(Elt<T>::pack2(p2 - f23.x, p3 - f23.y));
                    }
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
                    uint32_t a[4];
                    ldsm_x4_t(tbase + voff[i], a[0], a[1], a[2], a[3]);
#pragma unroll
                    for (int nt = 0; nt < NT; ++nt) {
                        Mma<T>::run(o[nt][i], a, pb[nt][0], pb[nt][1]);
                        if constexpr (kSplitP) Mma<T>::run(o[nt][i], a, pl[nt][0], pl[nt][1]);
                    }
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[s]);
        }
        stage_base += (uint32_t)m.nblk;

        // ---- merge the consumer warps' states, write output or partials
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int c = 0; c < 2; ++c)
#pragma unroll
                for (int off = 4; off < 32; off <<= 1) lrun[nt][c] += __shfl_xor_sync(0xffffffffu, lrun[nt][c], off);
        {
            float* mo = merge + cw * C::kHeadsPad * C::kMergeStride;
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
                    ml[(cw * C::kHeadsPad + h0) * 2 + 0] = mrun[nt][0];
                    ml[(cw * C::kHeadsPad + h0) * 2 + 1] = lrun[nt][0];
                    ml[(cw * C::kHeadsPad + h0 + 1) * 2 + 0] = mrun[nt][1];
                    ml[(cw * C::kHeadsPad + h0 + 1) * 2 + 1] = lrun[nt][1];
                }
            }
        }
        named_bar_sync(1, NCW * 32);
        {
            const int tid = cw * 32 + lane;
            T* out = static_cast<T*>(p.out);
            for (int e = tid; e < G * D; e += NCW * 32) {
                const int h = e / D, d = e - h * D;
                float M = kNegInf;
#pragma unroll
                for (int w = 0; w < NCW; ++w) M = fmaxf(M, ml[(w * C::kHeadsPad + h) * 2]);
                const float Ms = M == kNegInf ? 0.f : M;
                float L = 0.f, acc = 0.f;
#pragma unroll
                for (int w = 0; w < NCW; ++w) {
                    const float sc = fast_exp2(ml[(w * C::kHeadsPad + h) * 2] - Ms);
                    L += sc * ml[(w * C::kHeadsPad + h) * 2 + 1];
                    acc += sc * merge[(w * C::kHeadsPad + h) * C::kMergeStride + d];
                }
                const size_t hq = (size_t)m.b * p.num_heads + (size_t)m.g * G + h;
                if (m.nparts == 1) {
                    out[hq * D + d] = Elt<T>::from_f(L > 0.f ? acc / L : 0.f);
                } else {
                    const size_t pi = hq * p.max_parts + m.p;
                    p.part_o[pi * D + d] = acc;
                    if (d == 0) {
                        p.part_m[pi] = M;
                        p.part_l[pi] = L;
                    }
                }
            }
        }
        named_bar_sync(1, NCW * 32);
        if (*abort_flag) break;
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
    const int n_items = *p.n_items;
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
        for (int j = 0; j < m.nblk; ++j) {
            const int blk = p.block_tables[(size_t)m.b * p.max_blocks_per_seq + m.j0 + j];
            if (blk < 0 || blk >= p.num_blocks) {
                if (lane == 0) set_status(p.status, PA_ERR_OUT_OF_RANGE);
                continue;
            }
            const int ntok = min(kBlockSize, m.ctx - (m.j0 + j) * kBlockSize);
            const size_t tile = ((size_t)blk * p.num_kv_heads + m.g) * kBlockSize * D;
            for (int t = 0; t < ntok; ++t) {
                const T* kr = kc + tile + (size_t)t * D + lane * E;
                const T* vr = vc + tile + (size_t)t * D + lane * E;
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
template <typename T, int D>
__global__ void __launch_bounds__(128) decode_reduce_kernel(const DecodeParams p) {
    constexpr int E = D / 32;
    griddep_wait();
    const long long wi = (long long)blockIdx.x * 4 + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (wi >= (long long)p.num_seqs * p.num_heads) return;
    const int b = (int)(wi / p.num_heads);
    const int ctx = load_ctx(p, b, false);
    const int nparts = max(1, ceil_div_i(ceil_div_i(ctx, kBlockSize), p.part_blocks));
    if (nparts <= 1) return;
    const size_t base = (size_t)wi * p.max_parts;
    float M = kNegInf;
    for (int q = lane; q < nparts; q += 32) M = fmaxf(M, p.part_m[base + q]);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, off));
    const float Ms = M == kNegInf ? 0.f : M;
    float L = 0.f, acc[E];
#pragma unroll
    for (int e = 0; e < E; ++e) acc[e] = 0.f;
    for (int q = 0; q < nparts; ++q) {
        const float sc = fast_exp2(p.part_m[base + q] - Ms);
        L += sc * p.part_l[base + q];
        const float* po = p.part_o + (base + q) * D + lane * E;
#pragma unroll
        for (int e = 0; e < E; ++e) acc[e] += sc * po[e];
    }
    T* out = static_cast<T*>(p.out) + (size_t)wi * D + lane * E;
#pragma unroll
    for (int e = 0; e < E; ++e) out[e] = Elt<T>::from_f(L > 0.f ? acc[e] / L : 0.f);
}

// ===========================================================================
// host side
// ===========================================================================
namespace {

constexpr int kStages = 16;      // shared-memory ring depth (one stage = one K and one V tile)

// consumer warps per CTA: 4 by default; PA_TC_CONSUMER_WARPS=8 selects 8 (tuning)
int tc_consumer_warps() {
    static const int n = [] {
        const char* e = getenv("PA_TC_CONSUMER_WARPS");
        return (e && atoi(e) == 8) ? 8 : 4;
    }();
    return n;
}

PFN_cuTensorMapEncodeTiled_v12000 get_encode_fn() {
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
// a box is 16 rows x 64 elements (128 B), 128-byte swizzled in shared memory.
cudaError_t make_pool_map(CUtensorMap* map, const void* pool, pa_dtype dtype, int num_blocks, int num_kv_heads,
                          int head_dim) {
    auto encode = get_encode_fn();
    if (!encode) return cudaErrorNotSupported;
    const cuuint64_t dims[2] = {(cuuint64_t)head_dim, (cuuint64_t)num_blocks * num_kv_heads * kBlockSize};
    const cuuint64_t strides[1] = {(cuuint64_t)head_dim * 2};
    const cuuint32_t box[2] = {64, (cuuint32_t)kBlockSize};
    const cuuint32_t estr[2] = {1, 1};
    const CUtensorMapDataType dt =
        dtype == PA_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
    const CUresult r = encode(map, dt, 2, const_cast<void*>(pool), dims, strides, box, estr,
                              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

template <typename T, int D, int NT, int NCW>
cudaError_t launch_tc(const DecodeParams& p, pa_dtype dtype, cudaStream_t stream, int max_items) {
    using Cfg = TcCfg<D, NT, NCW, kStages>;
    auto kernel = decode_tc_kernel<T, D, NT, NCW, kStages>;
    static bool attr_done = false;
    if (!attr_done) {
        cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg::kSmemBytes);
        if (e != cudaSuccess) return e;
        attr_done = true;
    }
    CUtensorMap mk, mv;
    cudaError_t e = make_pool_map(&mk, p.key_cache, dtype, p.num_blocks, p.num_kv_heads, D);
    if (e != cudaSuccess) return e;
    e = make_pool_map(&mv, p.value_cache, dtype, p.num_blocks, p.num_kv_heads, D);
    if (e != cudaSuccess) return e;
    DeviceInfo dev;
    e = device_info(&dev);
    if (e != cudaSuccess) return e;
    int ctas_per_sm = 1;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&ctas_per_sm, kernel, Cfg::kThreads, Cfg::kSmemBytes);
    if (e != cudaSuccess) return e;
    if (ctas_per_sm < 1) return cudaErrorInvalidConfiguration;
    int grid = dev.sm_count * ctas_per_sm;
    if (grid > max_items) grid = max_items;
    if (grid < 1) grid = 1;
    return launch_pdl(kernel, dim3(grid), dim3(Cfg::kThreads), Cfg::kSmemBytes, stream, p, mk, mv);
}

template <typename T, int D>
cudaError_t launch_simt(const DecodeParams& p, cudaStream_t stream, int max_items) {
    DeviceInfo dev;
    cudaError_t e = device_info(&dev);
    if (e != cudaSuccess) return e;
    constexpr int NW = 4;
    long long want = ((long long)max_items * p.group + NW - 1) / NW;
    long long cap = (long long)dev.sm_count * 8;
    int grid = (int)(want < cap ? want : cap);
    if (grid < 1) grid = 1;
    return launch_pdl(decode_simt_kernel<T, D, NW>, dim3(grid), dim3(NW * 32), 0, stream, p);
}

template <typename T, int D>
cudaError_t launch_all(const DecodeParams& p, pa_dtype dtype, cudaStream_t stream) {
    const int max_items = p.num_seqs * p.max_parts * p.num_kv_heads;
    cudaError_t e = launch_pdl(decode_plan_kernel, dim3(1), dim3(1024), 0, stream, p);
    if (e != cudaSuccess) return e;
    const DecodePath path = decode_path(dtype, D, p.group);
    if constexpr (std::is_same<T, float>::value) {
        e = launch_simt<T, D>(p, stream, max_items);
    } else {
        if (path == DecodePath::kTensorCore) {
            const bool w8 = tc_consumer_warps() == 8;
            if (p.group <= 8)
                e = w8 ? launch_tc<T, D, 1, 8>(p, dtype, stream, max_items)
                       : launch_tc<T, D, 1, 4>(p, dtype, stream, max_items);
            else
                e = w8 ? launch_tc<T, D, 2, 8>(p, dtype, stream, max_items)
                       : launch_tc<T, D, 2, 4>(p, dtype, stream, max_items);
        }
        else
            e = launch_simt<T, D>(p, stream, max_items);
    }
    if (e != cudaSuccess) return e;
    if (p.max_parts > 1) {
        const long long warps = (long long)p.num_seqs * p.num_heads;
        e = launch_pdl(decode_reduce_kernel<T, D>, dim3((unsigned)((warps + 3) / 4)), dim3(128), 0, stream, p);
    }
    return e;
}

}  // namespace

DecodePath decode_path(pa_dtype dtype, int head_dim, int group) {
    (void)head_dim;
    if (dtype == PA_F32 || group > 16) return DecodePath::kSimt;
    return DecodePath::kTensorCore;
}

cudaError_t launch_decode(const DecodeParams& p, pa_dtype dtype, cudaStream_t stream) {
    switch (dtype) {
        case PA_F32: return p.head_dim == 64 ? launch_all<float, 64>(p, dtype, stream)
                                             : launch_all<float, 128>(p, dtype, stream);
        case PA_F16: return p.head_dim == 64 ? launch_all<__half, 64>(p, dtype, stream)
                                             : launch_all<__half, 128>(p, dtype, stream);
        case PA_BF16: return p.head_dim == 64 ? launch_all<__nv_bfloat16, 64>(p, dtype, stream)
                                              : launch_all<__nv_bfloat16, 128>(p, dtype, stream);
    }
    return cudaErrorInvalidValue;
}

}  // namespace pa
