// Paged prefill on sm_100a tensor cores (tcgen05, accumulators in TMEM).
//
// What is computed is pa_prefill's definition (pa.h): for sequence b with
// n = context_lens[b] tokens in the cache, of which the last L are the new
// ones, query row i < L sits at position p = n - L + i and attends to the
// keys at positions 0 .. p, read block by block through the block table
// ("PagedAttention" digest, sections "PagedAttention in one picture" and "Why
// the attention kernel works at all": the tiled attention loop, with the
// cache block as the unit the tile is made of).
//
// Tiles.  A CTA owns 128 rows of (query position, GQA head) pairs of one
// (sequence, KV head), in the order position * G + head, so every K/V tile it
// loads serves the whole group and no row is left empty except at the end of
// a chunk (a tile may begin and end inside a position's group).  It walks the
// keys 128 at a time (eight 16-token blocks):
//     S = Q K^T           tcgen05.mma, M = 128 rows, N = 128 keys, K = D
//     P = 2^(S*scale*log2 e - m)   fp32 online softmax, four threads per row
//     O += P V            tcgen05.mma with P in tensor memory, M = 128, N = D,
//                         K = 128 keys (bf16: once for P's hi part, once for lo)
// S has three buffers in tensor memory; the softmax writes a tile's P over
// its scores in place (16-bit pairs: hi in the buffer's first 64 columns, lo
// in the next 64), so QK^T runs up to three tiles ahead and the softmax never
// waits for the previous PV product except to rescale O.  O also lives in
// tensor memory (columns 384..511); Q, K and V in shared memory, 128-byte
// swizzled.
//
// Warps (384 threads, one CTA per SM):
//   0-7  softmax, two warps per scheduler: warp w owns the first (w < 4) or
//        last 16 TMEM lanes of quarter w mod 4, each thread two rows (lanes
//        L and L + 8) and a quarter of each 8-key group, read and written
//        through the 16-lane tcgen05.ld/st shapes; the row max and sum are
//        combined over a row's four threads with shuffles.  The warps load Q
//        into shared memory; per key tile they read S, mask keys past each
//        row's position (and blocks whose id is out of range), update the
//        running max and sum, write P back (one tensor-memory store per
//        part); at the end they scale O by 1/l and store it.  The max used for the
//        exponentials only moves when the tile max exceeds it by more than 8
//        (log2 units), so O is rescaled rarely; the sum and O always use the
//        same reference, which keeps the result exact algebra.
//   8, 10 producers of K (warp 8) and V (warp 10): 2-D TMA of each block of
//        the key step (16-row, 128-byte boxes, one per 64 columns), two
//        stages each.  Blocks no row of the tile sees are not loaded; a block
//        id out of range is reported and not loaded (the V producer hands the
//        mask of such blocks to the PV issuer with the stage).
//   9    QK^T issuer and TMEM owner: QK^T of tile j once the PV product of
//        tile j - 3 (which reads the same buffer) has completed.
//   11   PV issuer: per tile, once its P is written, the PV product(s).  Before
//        one it zeroes the V rows that are not data (slots past the context
//        in the sequence's last block, and blocks that were not loaded),
//        since a probability of 0 times a NaN left in shared memory would
//        still be NaN.
// The issuers run their loops as whole warps (an elected lane issues), each on
// a scheduler of its own beside two softmax warps.
// Every mbarrier wait is bounded (PA_ERR_TIMEOUT); on expiry the CTA lets
// its copies and MMAs finish, frees its TMEM and returns.
#include <algorithm>

#include "pa_internal.h"

namespace pa {

namespace {

constexpr float kNegInfT = -__builtin_huge_valf();
constexpr int kRowsT = 128;       // M: rows of a tile
constexpr int kKeysT = 128;       // N of QK^T: keys per step (8 blocks)
constexpr int kBlkT = 16;         // tokens per block
// The max used for the exponentials moves only when a tile's max exceeds it
// by more than this (log2 units): p <= 2^8, well inside fp16 and bf16.
constexpr float kRescaleSlack = 8.f;
// Waiting warps sleep this long between polls of an mbarrier: the softmax warps
// and the MMA issuers share schedulers, and a tight poll takes the issue slots
// the warp being waited for needs (1.5% of the kernel's time on the bench
// workload; suspending in mbarrier.try_wait instead cost 3.5%).
constexpr uint32_t kPollNs = 20;

template <int D>
struct TcPf {
    static constexpr int kHalves = D / 64;                 // 128-byte column groups of a D-wide row
    static constexpr int kGroupBytes = kRowsT * 128;       // 128 rows x 128 B (16 KB)
    static constexpr int kQBytes = kHalves * kGroupBytes;  // Q tile (K-major, K = D)
    static constexpr int kKVBytes = kHalves * kGroupBytes; // one K or V tile of 128 keys
    static constexpr int kStages = 2;                      // K and V stages
    static constexpr int kSBufs = 3;                       // S (then P) buffers in tensor memory
    static constexpr int kOffQ = 0;
    static constexpr int kOffK = kOffQ + kQBytes;
    static constexpr int kOffV = kOffK + kStages * kKVBytes;
    static constexpr int kOffBar = kOffV + kStages * kKVBytes;
    // q_full, k_full[2], v_full[2], k_empty[2], v_empty[2], s_full[3], p_full[3], pv_done[3], qk_done, pv_all
    static constexpr int kNumBars = 1 + 4 * kStages + 3 * kSBufs + 2;
    static constexpr int kOffMisc = kOffBar + kNumBars * 8;   // TMEM base, abort flag, per-stage bad-block masks
    static constexpr int kBytes = kOffMisc + 16 + 4 * kStages;
    // one CTA per SM (the CTA holds all 512 TMEM columns): at least half of the SM's shared memory
    static constexpr int kSmemBytes = (kBytes + 1024) > 120 * 1024 ? (kBytes + 1024) : 120 * 1024;
    // softmax warps 0-7 (two per scheduler: warps w and w + 4 own the first and
    // the last 16 lanes of quarter w), then on the four schedulers the K
    // producer (8), the QK^T issuer (9), the V producer (10), the PV issuer (11)
    static constexpr int kThreads = 384;
    static constexpr uint32_t kTmemCols = 512;
    // S buffer b at columns 128b: the fp32 scores of a 128-key tile, then, in
    // place, P as 16-bit pairs: columns 0-63 (hi) and 64-127 (lo, bf16 only)
    static constexpr uint32_t kColS = 0;
    static constexpr uint32_t kColPLo = 64;                 // lo part, relative to the buffer
    static constexpr uint32_t kColO = 384;                  // O: D columns
    static_assert(kBytes + 1024 <= 227 * 1024, "shared memory");
};

// Spin with a short sleep between polls (bounded like mbar_wait): a waiting
// warp then leaves most issue slots to the warps that share its scheduler,
// and still resumes within tens of nanoseconds of the phase completing.
__device__ __forceinline__ bool mbar_sleep_wait(uint64_t* bar, uint32_t parity, uint32_t sleep_ns,
                                                uint64_t limit_ns = kWaitLimitNs) {
    if (mbar_test_wait(bar, parity)) return true;
    const uint64_t t0 = global_timer_ns();
    for (;;) {
        __nanosleep(sleep_ns);
        if (mbar_test_wait(bar, parity)) return true;
        if (global_timer_ns() - t0 > limit_ns) return false;
    }
}
// The same for a warp: lane 0 polls, then every lane observes the completed
// phase itself.  Returns false on expiry, for every lane.
__device__ __forceinline__ bool warp_sleep_wait(uint64_t* bar, uint32_t parity, int lane, uint32_t sleep_ns) {
    int ok = 1;
    if (lane == 0) ok = mbar_sleep_wait(bar, parity, sleep_ns);
    ok = __shfl_sync(0xffffffffu, ok, 0);
    if (ok) mbar_test_wait(bar, parity);
    return ok != 0;
}

// Tensor-memory loads and stores in the 16-lane shapes, for a warp that owns
// 16 of its quarter's 32 lanes (the address carries the first lane).  Thread
// t holds lanes L = first + (t >> 2) and L + 8:
//   .16x256b, repetition r: registers 4r, 4r + 1 are lane L, columns
//       8r + 2(t & 3) and 8r + 2(t & 3) + 1; 4r + 2, 4r + 3 the same for L + 8;
//   .16x128b, repetition r: registers 2r, 2r + 1 are lanes L, L + 8 at column
//       4r + (t & 3).
// (Measured: each lane's values written through the 32x32b shape and read
// back through these.)
__device__ __forceinline__ void tmem_ld_16x256b_x8(uint32_t taddr, uint32_t* r) {
    asm volatile(
        "tcgen05.ld.sync.aligned.16x256b.x8.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
        "%15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
          "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
          "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr));
}
__device__ __forceinline__ void tmem_st_16x256b_x8(uint32_t taddr, const uint32_t* r) {
    asm volatile(
        "tcgen05.st.sync.aligned.16x256b.x8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
        "%15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32};" ::"r"(taddr),
        "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]),
        "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]), "r"(r[16]), "r"(r[17]),
        "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]), "r"(r[24]), "r"(r[25]), "r"(r[26]),
        "r"(r[27]), "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31])
        : "memory");
}
__device__ __forceinline__ void tmem_st_16x128b_x16(uint32_t taddr, const uint32_t* r) {
    asm volatile(
        "tcgen05.st.sync.aligned.16x128b.x16.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
        "%15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32};" ::"r"(taddr),
        "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]),
        "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]), "r"(r[16]), "r"(r[17]),
        "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]), "r"(r[24]), "r"(r[25]), "r"(r[26]),
        "r"(r[27]), "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31])
        : "memory");
}

// byte offset of 16-byte unit u (0..7) of row r inside a 128-byte-swizzled group
__device__ __forceinline__ uint32_t sw128(int r, int u) { return (uint32_t)(r * 128 + ((u ^ (r & 7)) << 4)); }

// Block ids of key tile j: lane l < 8 reads the table entry of block 8j + l
// if some row of the tile needs it (else 0, a valid id).  Issued a tile ahead
// of its use, so no global-memory latency sits in front of an MMA issue.
__device__ __forceinline__ int tile_block_id(const int32_t* row, int j, int nkt, int kend, int lane) {
    const int blk = j * 8 + lane;
    return (j < nkt && lane < 8 && blk * kBlkT < kend) ? __ldg(row + blk) : 0;
}
// 8-bit mask of the blocks of a key tile whose ids are out of range
__device__ __forceinline__ uint32_t bad_mask(const PrefillParams& p, int id) {
    return __ballot_sync(0xffffffffu, id < 0 || id >= p.num_blocks) & 0xffu;
}

// The grid: tx tiles per (sequence, KV head); work item i is tile
// tx - 1 - i / (Hkv B) of KV head (i mod Hkv B) mod Hkv of sequence
// (i mod Hkv B) / Hkv: every (sequence, KV head)'s last tile first, then
// every one's second-last, ..., so that the grid runs longest tiles first
// (a tile's keys grow with its last query position) and each SM's share of
// whole tiles evens out.  Items 0 .. nfull - 1 are whole CTAs;
// each item after them (the grid's last, partial wave) is split by key range
// into ksplit pieces, one CTA each, whose partial results (O unnormalised,
// the reference max and the sum, per row) go to `part`; prefill_merge_kernel,
// launched next, combines them.
struct PrefillGrid {
    int tx, nfull, ksplit;
    float* part;   // [tail items][ksplit][128 rows][D + 4]: O, then m and l (and 2 floats of padding)
};
// At most this many pieces per split item: more would shorten the last wave
// further but make the merge read more partial rows.
constexpr int kMaxSplit = 16;
// floats per partial row: 16-byte aligned rows for the vector stores and loads
__host__ __device__ constexpr int part_row_floats(int d) { return d + 4; }

template <typename T, int D>
__global__ void __launch_bounds__(384, 1)
    prefill_tc_kernel(const PrefillParams p, const __grid_constant__ CUtensorMap tmK,
                      const __grid_constant__ CUtensorMap tmV, uint32_t idesc_qk, uint32_t idesc_pv,
                      const PrefillGrid pg) {
    // bf16 P (8-bit significand) would perturb the softmax weights by up to
    // 2^-8, which on rows with a few comparable keys moves the output by up
    // to ~1e-2; it is carried as hi + lo (two bf16 parts, ~16 bits) and the PV
    // product runs once per part.  fp16 P (11 bits) is used as is.
    constexpr bool kSplitP = std::is_same<T, __nv_bfloat16>::value;
    using C = TcPf<D>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kOffBar);
    uint64_t* q_full = bars;
    uint64_t* k_full = bars + 1;
    uint64_t* v_full = k_full + C::kStages;
    uint64_t* k_empty = v_full + C::kStages;
    uint64_t* v_empty = k_empty + C::kStages;
    // per S buffer b (key tiles j = b mod 3): scores written, P written, PV done.
    // One buffer's barrier completes once per three tiles and a waiter is never
    // more than one phase behind it.
    uint64_t* s_full = v_empty + C::kStages;
    uint64_t* p_full = s_full + C::kSBufs;
    uint64_t* pv_done = p_full + C::kSBufs;
    uint64_t* qk_done = pv_done + C::kSBufs;   // every QK^T product has completed
    uint64_t* pv_all = qk_done + 1;             // every PV product has completed
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::kOffMisc);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::kOffMisc + 4);
    // the V stage's blocks with an out-of-range id (written by the V producer before the stage's
    // arrival, read by the MMA issuer after it)
    volatile uint32_t* stage_bad = reinterpret_cast<volatile uint32_t*>(smem + C::kOffMisc + 16);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int G = p.group;
    int item = (int)blockIdx.x, piece = 0, npieces = 1;
    if (item >= pg.nfull) {
        const int t = item - pg.nfull;
        item = pg.nfull + t / pg.ksplit;
        piece = t % pg.ksplit;
        npieces = pg.ksplit;
    }
    const int pairs = p.num_kv_heads * p.num_seqs;
    const int g = (item % pairs) % p.num_kv_heads, b = (item % pairs) / p.num_kv_heads;
    const int tile = pg.tx - 1 - item / pairs;   // the longest tiles start first

    griddep_launch_dependents();
    // query_start, context_lens, the block table and Q may be written by the
    // preceding kernel: read only once it has completed
    griddep_wait();
    const int qs = p.query_start[b], L = p.query_start[b + 1] - qs;
    const int n = p.context_lens[b];
    // The chunk's query rows are (position i, head k of the group) pairs in
    // the order i * G + k; tile t holds rows 128t .. 128t + 127, so a tile may
    // start and end in the middle of a position's group.
    const int R0 = tile * kRowsT;                    // the tile's first row
    bool active = L > 0 && R0 < L * G;
    if (active && (n < L || n > p.max_blocks_per_seq * kBlkT)) {   // a query position outside the cache
        if (threadIdx.x == 0) set_status(p.status, PA_ERR_OUT_OF_RANGE);
        active = false;
    }
    const int nrows = active ? min(kRowsT, L * G - R0) : 1;   // rows of this tile that hold a query
    const int i0 = R0 / G;                                     // query index of the tile's first row
    const int pos0 = n - L + i0;                               // its position in the sequence
    const int kend = n - L + (R0 + nrows - 1) / G + 1;         // keys [0, kend) are visible to some row
    const int nkt = ceil_div_i(kend, kKeysT);
    // this CTA's key tiles: all of them, or its piece of the range
    const int kt_lo = (int)((long long)nkt * piece / npieces);
    const int kt_hi = (int)((long long)nkt * (piece + 1) / npieces);
    const int nloc = kt_hi - kt_lo;
    const int32_t* bt_row = p.block_tables + (size_t)b * p.max_blocks_per_seq;
    // Issued before the CTA's setup, so that their latency overlaps it: the
    // first key tile's block ids and, in the softmax warps, the thread's half
    // of a Q row (all its pieces at once: one round trip, not one per piece).
    const int id_first = active ? tile_block_id(bt_row, kt_lo, kt_hi, kend, lane) : 0;
    uint4 qv[D / 16];
    const int q_r = threadIdx.x >> 1, q_h = threadIdx.x & 1;   // Q row and half (softmax warps)
    if (active && warp < 8) {
        const bool real = q_r < nrows;
        const int rq = R0 + min(q_r, nrows - 1), qi = rq / G, qk = rq - qi * G;
        const uint4* qrow = reinterpret_cast<const uint4*>(static_cast<const T*>(p.q) +
                                                           ((size_t)(qs + qi) * p.num_heads + g * G + qk) * D) +
                            q_h * (D / 16);
#pragma unroll
        for (int cc = 0; cc < D / 16; ++cc) qv[cc] = real ? qrow[cc] : make_uint4(0, 0, 0, 0);
    }

    if (threadIdx.x == 256) {
        mbar_init(q_full, 8);
        for (int s = 0; s < C::kStages; ++s) {
            mbar_init(&k_full[s], 1);
            mbar_init(&v_full[s], 1);
            mbar_init(&k_empty[s], 1);
            mbar_init(&v_empty[s], 1);
        }
        for (int i = 0; i < C::kSBufs; ++i) {
            mbar_init(&s_full[i], 1);
            mbar_init(&p_full[i], 8);
            mbar_init(&pv_done[i], 1);
        }
        mbar_init(qk_done, 1);
        mbar_init(pv_all, 1);
        *abort_flag = 0;
        mbar_fence_init();
    }
    if (warp == 9) {
        tmem_alloc(tmem_slot, C::kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (active) {
        const uint32_t sQ = smem_u32(smem + C::kOffQ);
        const uint32_t sK = smem_u32(smem + C::kOffK);
        const uint32_t sV = smem_u32(smem + C::kOffV);
        auto fail = [&]() {
            *abort_flag = 1;
            set_status(p.status, PA_ERR_TIMEOUT);
        };

        if (warp < 8) {
            // ================================================= softmax warps
            // Warp w owns TMEM lanes 32(w mod 4) + 16(w / 4) .. + 15 (its
            // quarter's first or last 16 lanes); thread t of it holds rows
            // rA = that base + t / 4 and rB = rA + 8, and in each 8-key group of
            // a tile the keys 2(t mod 4) and 2(t mod 4) + 1.  A row's four
            // threads are lanes 4k .. 4k + 3 of the warp.
            const int cg = lane & 3;
            const int lbase = 32 * (warp & 3) + 16 * (warp >> 2);
            const int rA = lbase + (lane >> 2), rB = rA + 8;
            const int rqA = R0 + min(rA, nrows - 1), rqB = R0 + min(rB, nrows - 1);   // rows past the chunk
            const int qiA = rqA / G, qkA = rqA - qiA * G;                             // repeat its last row
            const int qiB = rqB / G, qkB = rqB - qiB * G;
            const int posA = n - L + qiA, posB = n - L + qiB;
            const uint32_t tl = tmem + ((uint32_t)lbase << 16);
            const float sl2 = p.scale_log2;                         // > 0 (a negative scale negates A)
            {   // Q: thread i stores half i mod 2 of row i / 2, loaded above (16-byte
                // pieces into the swizzled K-major layout)
#pragma unroll
                for (int cc = 0; cc < D / 16; ++cc) {
                    const int c = q_h * (D / 16) + cc;
                    const uint32_t a = sQ + (c >> 3) * C::kGroupBytes + sw128(q_r, c & 7);
                    asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(a), "r"(qv[cc].x), "r"(qv[cc].y),
                                 "r"(qv[cc].z), "r"(qv[cc].w)
                                 : "memory");
                }
                fence_proxy_async_shared();
                __syncwarp();
                if (lane == 0) mbar_arrive(q_full);
            }
            // per row: the reference max (equal in the row's four threads) and this
            // thread's share of the sum
            float mA = kNegInfT, mB = kNegInfT, lA = 0.f, lB = 0.f;
            bool ok = true;
            int id_next = id_first;
            for (int j = kt_lo; j < kt_hi && ok; ++j) {
                const int jj = j - kt_lo;                       // local index: buffers and phases
                const int id_cur = id_next;
                id_next = tile_block_id(bt_row, j + 1, kt_hi, kend, lane);
                const int sb = jj % C::kSBufs;
                const uint32_t sph = (uint32_t)(jj / C::kSBufs) & 1u;
                if (!warp_sleep_wait(&s_full[sb], sph, lane, kPollNs) || *abort_flag) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t tS = tl + C::kColS + sb * kKeysT;
                // sv[4e + 0, 1]: row A, keys 8e + 2cg, + 1; sv[4e + 2, 3]: row B, the same keys
                uint32_t sv[kKeysT / 2];
                tmem_ld_16x256b_x8(tS, sv);
                tmem_ld_16x256b_x8(tS + 64, sv + 32);
                tmem_ld_wait(sv);
                const uint32_t badm = bad_mask(p, id_cur);

                // causal mask (the tile's first row sees keys up to pos0) and bad blocks
                const int kb0 = j * kKeysT;
                if (kb0 + kKeysT - 1 > pos0 || badm != 0) {
#pragma unroll
                    for (int e = 0; e < kKeysT / 8; ++e) {
                        const bool bad = (badm >> (e >> 1)) & 1u;
                        const int key = kb0 + 8 * e + 2 * cg;
                        if (bad || key > posA) sv[4 * e] = __float_as_uint(kNegInfT);
                        if (bad || key + 1 > posA) sv[4 * e + 1] = __float_as_uint(kNegInfT);
                        if (bad || key > posB) sv[4 * e + 2] = __float_as_uint(kNegInfT);
                        if (bad || key + 1 > posB) sv[4 * e + 3] = __float_as_uint(kNegInfT);
                    }
                }
                float xa0 = kNegInfT, xa1 = kNegInfT, xb0 = kNegInfT, xb1 = kNegInfT;
#pragma unroll
                for (int e = 0; e < kKeysT / 8; e += 2) {
                    xa0 = fmax3(xa0, __uint_as_float(sv[4 * e]), __uint_as_float(sv[4 * e + 1]));
                    xb0 = fmax3(xb0, __uint_as_float(sv[4 * e + 2]), __uint_as_float(sv[4 * e + 3]));
                    xa1 = fmax3(xa1, __uint_as_float(sv[4 * e + 4]), __uint_as_float(sv[4 * e + 5]));
                    xb1 = fmax3(xb1, __uint_as_float(sv[4 * e + 6]), __uint_as_float(sv[4 * e + 7]));
                }
                // the row maxima over the row's four threads
                float mxA = fmaxf(xa0, xa1), mxB = fmaxf(xb0, xb1);
                mxA = fmaxf(mxA, __shfl_xor_sync(0xffffffffu, mxA, 1));
                mxB = fmaxf(mxB, __shfl_xor_sync(0xffffffffu, mxB, 1));
                mxA = fmaxf(mxA, __shfl_xor_sync(0xffffffffu, mxA, 2));
                mxB = fmaxf(mxB, __shfl_xor_sync(0xffffffffu, mxB, 2));
                const float mnA = mxA * sl2, mnB = mxB * sl2;
                float alphaA = 1.f, alphaB = 1.f;
                if (mnA > mA + kRescaleSlack) {
                    alphaA = mA == kNegInfT ? 0.f : fast_exp2(mA - mnA);
                    mA = mnA;
                }
                if (mnB > mB + kRescaleSlack) {
                    alphaB = mB == kNegInfT ? 0.f : fast_exp2(mB - mnB);
                    mB = mnB;
                }
                const float msA = mA == kNegInfT ? 0.f : mA, msB = mB == kNegInfT ? 0.f : mB;
                // P in the input dtype (bf16: hi + lo); the row sums add what the PV
                // products use: the rounded fp16 values, or the fp32 values hi + lo
                // carry.  The pair of keys 8e + 2cg, + 1 of a row goes to P column
                // 4e + cg of its lane (the buffer's scores are overwritten in place),
                // one store per part for the whole tile (fewer, wider tensor-memory
                // stores measured faster than a quarter at a time).  The PV product of
                // this tile is issued before the QK^T product that next writes this
                // buffer, and the QK^T issuer waits for it.  Pairs of keys go through
                // the packed fp32x2 add and fma.
                const float2 sl2v = make_float2(sl2, sl2), nmA = make_float2(-msA, -msA), nmB = make_float2(-msB, -msB);
                float2 lsA = make_float2(0.f, 0.f), lsB = make_float2(0.f, 0.f);
                {
                    // 16x128b repetition e: P column 4e + cg, rows A, B
                    uint32_t pk[kKeysT / 4];
                    uint32_t pl[kSplitP ? kKeysT / 4 : 1];
#pragma unroll
                    for (int e = 0; e < kKeysT / 8; ++e) {
#pragma unroll
                        for (int rb = 0; rb < 2; ++rb) {
                            const float2 x = __ffma2_rn(
                                make_float2(__uint_as_float(sv[4 * e + 2 * rb]), __uint_as_float(sv[4 * e + 2 * rb + 1])),
                                sl2v, rb ? nmB : nmA);
                            const float e0 = fast_exp2(x.x), e1 = fast_exp2(x.y);
                            float2& ls = rb ? lsB : lsA;
                            if constexpr (kSplitP) {
                                // hi = p truncated to bf16 (its upper 16 bits), lo = p - hi (exact
                                // in fp32) truncated likewise: hi + lo is p to within 2^-15
                                // relative.  No float -> bf16 conversion: it would run on the
                                // transcendental pipe that computes 2^x.  The pair's hi parts are
                                // one byte permute; back as floats, one is a shift of it and the
                                // other a mask, and lo is one packed fma (hi * -1 + p): the
                                // integer pipe, the busiest here after the tensor core, gets
                                // three operations per pair.
                                const uint32_t hp = __byte_perm(__float_as_uint(e0), __float_as_uint(e1), 0x7632);
                                pk[2 * e + rb] = hp;
                                const float2 rr =
                                    __ffma2_rn(make_float2(__uint_as_float(hp << 16), __uint_as_float(hp & 0xffff0000u)),
                                               make_float2(-1.f, -1.f), make_float2(e0, e1));
                                pl[2 * e + rb] = __byte_perm(__float_as_uint(rr.x), __float_as_uint(rr.y), 0x7632);
                                ls = __fadd2_rn(ls, make_float2(e0, e1));
                            } else {
                                pk[2 * e + rb] = Elt<T>::pack2(e0, e1);
                                ls = __fadd2_rn(ls, __half22float2(*reinterpret_cast<const __half2*>(&pk[2 * e + rb])));
                            }
                        }
                    }
                    tmem_st_16x128b_x16(tS, pk);
                    if constexpr (kSplitP) tmem_st_16x128b_x16(tS + C::kColPLo, pl);
                }
                lA = lA * alphaA + (lsA.x + lsA.y);
                lB = lB * alphaB + (lsB.x + lsB.y);
                // O is rescaled only when some row's reference max moved: that needs
                // the previous tiles' PV products complete.  The PV of tile j - 1
                // signals buffer (j - 1) mod 3, whose previous signal (tile j - 4)
                // preceded this tile's scores, so the parity names one phase.
                if (jj > 0 && __any_sync(0xffffffffu, alphaA != 1.f || alphaB != 1.f)) {
                    const int pb = (jj - 1) % C::kSBufs;
                    if (!warp_sleep_wait(&pv_done[pb], (uint32_t)((jj - 1) / C::kSBufs) & 1u, lane, kPollNs) ||
                        *abort_flag) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
#pragma unroll
                    for (int c = 0; c < D / 64; ++c) {
                        uint32_t ov[32];
                        tmem_ld_16x256b_x8(tl + C::kColO + c * 64, ov);
                        tmem_ld_wait(ov);
#pragma unroll
                        for (int k = 0; k < 32; ++k)
                            ov[k] = __float_as_uint(__uint_as_float(ov[k]) * ((k & 2) ? alphaB : alphaA));
                        tmem_st_16x256b_x8(tl + C::kColO + c * 64, ov);
                    }
                }
                tmem_st_wait();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&p_full[sb]);
            }
            // every PV product of this CTA has completed (a piece with no key tile has none)
            if (ok && nloc > 0)
                ok = warp_sleep_wait(&pv_done[(nloc - 1) % C::kSBufs], (uint32_t)((nloc - 1) / C::kSBufs) & 1u, lane,
                                     kPollNs) &&
                     !*abort_flag;
            if (ok) tc_fence_after();
            // the rows' sums: the four threads' shares
            lA += __shfl_xor_sync(0xffffffffu, lA, 1);
            lA += __shfl_xor_sync(0xffffffffu, lA, 2);
            lB += __shfl_xor_sync(0xffffffffu, lB, 1);
            lB += __shfl_xor_sync(0xffffffffu, lB, 2);
            if (ok && npieces == 1) {
                const float invA = lA > 0.f ? 1.f / lA : 0.f, invB = lB > 0.f ? 1.f / lB : 0.f;
                T* dA = static_cast<T*>(p.out) + ((size_t)(qs + qiA) * p.num_heads + g * G + qkA) * D + 2 * cg;
                T* dB = static_cast<T*>(p.out) + ((size_t)(qs + qiB) * p.num_heads + g * G + qkB) * D + 2 * cg;
#pragma unroll
                for (int c = 0; c < D / 64; ++c) {
                    uint32_t ov[32];
                    tmem_ld_16x256b_x8(tl + C::kColO + c * 64, ov);
                    tmem_ld_wait(ov);
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        const int col = c * 64 + 8 * e;
                        if (rA < nrows)
                            *reinterpret_cast<uint32_t*>(dA + col) =
                                Elt<T>::pack2(__uint_as_float(ov[4 * e]) * invA, __uint_as_float(ov[4 * e + 1]) * invA);
                        if (rB < nrows)
                            *reinterpret_cast<uint32_t*>(dB + col) = Elt<T>::pack2(
                                __uint_as_float(ov[4 * e + 2]) * invB, __uint_as_float(ov[4 * e + 3]) * invB);
                    }
                }
            } else if (ok) {
                // A piece of a split item: its rows' O (unnormalised, relative to the
                // reference max), the max and the sum go to the workspace for
                // prefill_merge_kernel (a piece that saw no key leaves l = 0 and an O
                // the merge ignores).
                constexpr int kRow = part_row_floats(D);
                float* base = pg.part + ((size_t)(item - pg.nfull) * npieces + piece) * kRowsT * kRow;
                float* mineA = base + (size_t)rA * kRow;
                float* mineB = base + (size_t)rB * kRow;
#pragma unroll
                for (int c = 0; c < D / 64; ++c) {
                    uint32_t ov[32];
                    tmem_ld_16x256b_x8(tl + C::kColO + c * 64, ov);
                    tmem_ld_wait(ov);
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        const int col = c * 64 + 8 * e + 2 * cg;
                        *reinterpret_cast<float2*>(mineA + col) =
                            make_float2(__uint_as_float(ov[4 * e]), __uint_as_float(ov[4 * e + 1]));
                        *reinterpret_cast<float2*>(mineB + col) =
                            make_float2(__uint_as_float(ov[4 * e + 2]), __uint_as_float(ov[4 * e + 3]));
                    }
                }
                if (cg == 0) {
                    mineA[D] = mA;
                    mineA[D + 1] = lA;
                    mineB[D] = mB;
                    mineB[D + 1] = lB;
                }
            }
            if (!ok && lane == 0) fail();
        } else if (warp == 8 || warp == 10) {
            // ============================== producers: warp 8 loads K, warp 10 loads V
            // (separately, so that a K stage is refilled as soon as its QK^T is done,
            // not after the previous tile's PV has freed a V stage)
            const bool is_k = warp == 8;
            const CUtensorMap* map = is_k ? &tmK : &tmV;
            uint64_t* fullb = is_k ? k_full : v_full;
            uint64_t* emptyb = is_k ? k_empty : v_empty;
            const uint32_t base = is_k ? sK : sV;
            if (lane == 0) prefetch_tensormap(map);
            constexpr uint32_t kBlockBytes = kBlkT * D * 2;   // one block of one KV head: K or V
            int issued = 0;
            bool ok = true;
            int id_next = id_first;
            for (int j = kt_lo; j < kt_hi && ok; ++j) {
                const int jj = j - kt_lo;                     // local index: stages and phases
                const int s = jj % C::kStages;
                const uint32_t par = ((jj / C::kStages) & 1) ^ 1;
                const int id = id_next;
                id_next = tile_block_id(bt_row, j + 1, kt_hi, kend, lane);
                const bool need = lane < 8 && (j * 8 + lane) * kBlkT < kend;
                const bool good = need && id >= 0 && id < p.num_blocks;
                if (is_k && need && !good) set_status(p.status, PA_ERR_OUT_OF_RANGE);
                const uint32_t nload = __popc(__ballot_sync(0xffffffffu, good));
                const int y = (id * p.num_kv_heads + g) * kBlkT;
                const uint32_t badm = __ballot_sync(0xffffffffu, need && !good) & 0xffu;
                int w = 1;
                if (lane == 0) {
                    w = mbar_wait(&emptyb[s], par);
                    if (w && !is_k) stage_bad[s] = badm;
                    if (w) mbar_arrive_expect_tx(&fullb[s], nload * kBlockBytes);
                }
                if (!__shfl_sync(0xffffffffu, w, 0) || *abort_flag) { ok = false; break; }
                if (good) {
#pragma unroll
                    for (int h = 0; h < C::kHalves; ++h)
                        tma_load_2d_keep(base + s * C::kKVBytes + h * C::kGroupBytes + lane * (kBlkT * 128), map,
                                         h * 64, y, &fullb[s]);
                }
                issued = jj + 1;
            }
            if (!ok && lane == 0) {
                // let the copies this warp issued land before the CTA's memory is released
                fail();
                for (int j = max(0, issued - C::kStages); j < issued; ++j)
                    mbar_wait(&fullb[j % C::kStages], (j / C::kStages) & 1);
            }
        } else {
            // ============================= MMA issuers: QK^T (warp 9), PV (warp 11)
            bool ok = true;
            // descriptors: Q, K, P K-major (8-row atoms 1024 B apart, K steps of 16
            // elements 32 B apart inside a 128-byte row, 64-element groups 16 KB
            // apart); V MN-major (64 D-columns per 128-byte row, 16 KB between
            // column groups, 16 keys = 2 atoms per K step)
            //
            // The issuing thread shares its scheduler with a softmax warp that
            // always has work, so its own instruction count between MMAs is what
            // the tensor core waits on: descriptors are built once, and a K step
            // only adds a constant to the start-address field (bits 0-13, in
            // 16-byte units) of the step-0 descriptor.
            auto kdesc = [&](uint32_t base, int k) {
                return umma_desc_sw128(base + (k >> 2) * C::kGroupBytes + (k & 3) * 32, 16, 1024);
            };
            auto vdesc = [&](uint32_t base, int k) {
                return umma_desc_sw128(base + k * (2 * 1024), C::kGroupBytes, 1024);
            };
            const uint64_t dQ = kdesc(sQ, 0);
            const uint64_t dK0 = kdesc(sK, 0), dV0 = vdesc(sV, 0);
            constexpr uint64_t kStageStep = (uint64_t)(C::kKVBytes >> 4);    // one K or V stage
            auto kstep = [](int k) { return (uint64_t)(((k >> 2) * C::kGroupBytes + (k & 3) * 32) >> 4); };
            constexpr uint64_t kVStep = (2 * 1024) >> 4;                      // 16 keys of V
            // The whole warp runs the issue loop (warp-uniform control flow: the
            // descriptors stay in uniform registers) and one elected lane issues
            // each product; waits poll with a short sleep (bounded) and end for
            // all lanes together.
            auto wait_all = [&](uint64_t* bar, uint32_t par) -> bool {
                return __all_sync(0xffffffffu, mbar_sleep_wait(bar, par, kPollNs) && !*abort_flag);
            };
            // key tile j of the item; stages, buffers and phases follow this CTA's
            // local index j - kt_lo
            auto issue_qk = [&](int j) -> bool {
                const int jj = j - kt_lo;
                const int s = jj % C::kStages;
                if (!wait_all(&k_full[s], (jj / C::kStages) & 1)) return false;
                tc_fence_after();
                const uint64_t dk = dK0 + (uint64_t)s * kStageStep;
                const int sb = jj % C::kSBufs;
                const uint32_t dS = tmem + C::kColS + sb * kKeysT;
#pragma unroll
                for (int k = 0; k < D / 16; ++k)
                    umma_f16_ss_warp(dS, dQ + kstep(k), dk + kstep(k), idesc_qk, k > 0 ? 1u : 0u);
                umma_commit_warp(&s_full[sb]);
                umma_commit_warp(&k_empty[s]);
                return true;
            };
            auto issue_pv = [&](int i) -> bool {
                const int ii = i - kt_lo;
                const int s = ii % C::kStages;
                const int sb = ii % C::kSBufs;
                if (!wait_all(&p_full[sb], (uint32_t)(ii / C::kSBufs) & 1u)) return false;
                if (!wait_all(&v_full[s], (ii / C::kStages) & 1)) return false;
                const uint32_t badm = __shfl_sync(0xffffffffu, stage_bad[s], 0);
                // keys of this tile the PV product covers: whole 16-key steps up to kend
                const int nks = min(kKeysT, kend - i * kKeysT + kBlkT - 1) / kBlkT;
                // rows of V that hold no data: blocks not loaded (bad ids) and slots
                // at or past n in the sequence's last block (only the sequence's last
                // tile has those; a tile with neither skips the scan)
                const int tail_blk = n / kBlkT - i * 8;      // the last block's index in this tile, if partial
                const int tail_from = n % kBlkT;
                if (badm != 0 || (tail_from != 0 && tail_blk < nks)) {
                    // 16-byte pieces of the rows to clear, spread over the warp
                    for (int k = 0; k < nks; ++k) {
                        const int r0 = ((badm >> k) & 1u) ? 0 : (k == tail_blk ? tail_from : kBlkT);
                        for (int u = (k * kBlkT + r0) * 8 * C::kHalves + lane; u < (k + 1) * kBlkT * 8 * C::kHalves;
                             u += 32) {
                            const int rr = u / (8 * C::kHalves), hh = (u / 8) % C::kHalves, uu = u % 8;
                            st_shared_zero16(sV + s * C::kKVBytes + hh * C::kGroupBytes + rr * 128 + (uu << 4));
                        }
                    }
                    fence_proxy_async_shared();
                    __syncwarp();
                }
                tc_fence_after();
                const uint64_t dv = dV0 + (uint64_t)s * kStageStep;
                const uint32_t tP = tmem + C::kColS + sb * kKeysT;
                const uint32_t acc0 = ii > 0 ? 1u : 0u;
#pragma unroll
                for (int k = 0; k < kKeysT / kBlkT; ++k)
                    if (k < nks)
                        umma_f16_ts_warp(tmem + C::kColO, tP + k * 8, dv + k * kVStep, idesc_pv, k > 0 ? 1u : acc0);
                if constexpr (kSplitP) {
#pragma unroll
                    for (int k = 0; k < kKeysT / kBlkT; ++k)
                        if (k < nks)
                            umma_f16_ts_warp(tmem + C::kColO, tP + C::kColPLo + k * 8, dv + k * kVStep, idesc_pv, 1u);
                }
                umma_commit_warp(&pv_done[sb]);
                umma_commit_warp(&v_empty[s]);
                return true;
            };
            if (warp == 9) {
                // QK^T runs up to three tiles ahead (one per S buffer).  Buffer
                // j mod 3 holds the P of tile j - 3, which the other issuer's PV
                // product reads: the QK^T of tile j waits for that product to
                // complete (products of different threads are not ordered).
                ok = wait_all(q_full, 0);
                for (int j = kt_lo; j < kt_hi && ok; ++j) {
                    const int jj = j - kt_lo;
                    if (jj >= C::kSBufs &&
                        !wait_all(&pv_done[(jj - C::kSBufs) % C::kSBufs], (uint32_t)((jj - C::kSBufs) / C::kSBufs) & 1u)) {
                        ok = false;
                        break;
                    }
                    ok = issue_qk(j);
                }
                // every product this warp issued has completed before TMEM and
                // shared memory are released
                umma_commit_warp(qk_done);
                mbar_wait(qk_done, 0);
            } else {
                for (int j = kt_lo; j < kt_hi && ok; ++j) ok = issue_pv(j);
                umma_commit_warp(pv_all);
                mbar_wait(pv_all, 0);
            }
            if (!ok && lane == 0) fail();
            __syncwarp();
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 9) {
        tc_fence_after();
        tmem_dealloc(tmem, C::kTmemCols);
    }
}


// The grid for one CTA per SM: tx tiles per (sequence, KV head), and the
// items of the last, partial wave split into ksplit pieces when that leaves
// at least two pieces per item.
struct SplitPlan {
    int tx = 0;
    long long items = 0;
    int tail = 0, ksplit = 1;
    size_t bytes = 0;   // workspace: the split items' partial rows
};
SplitPlan split_plan(const PrefillParams& p, int sm_count) {
    SplitPlan s;
    s.tx = (int)(((long long)p.max_query_len * p.group + kRowsT - 1) / kRowsT);
    s.items = (long long)s.tx * p.num_kv_heads * p.num_seqs;
    if (sm_count > 0 && s.items > sm_count) {
        const int tail = (int)(s.items % sm_count);
        const int k = tail > 0 ? std::min(kMaxSplit, sm_count / tail) : 1;
        if (k >= 2) {
            s.tail = tail;
            s.ksplit = k;
            s.bytes = (size_t)tail * k * kRowsT * part_row_floats(p.head_dim) * sizeof(float);
        }
    }
    return s;
}
int sm_count_now() {
    DeviceInfo d;
    return device_info(&d) == cudaSuccess && d.sm_count > 0 ? d.sm_count : 148;
}

// Combines the pieces of the split items: one warp per (item, row), lanes
// over the row's columns (4 each), the pieces' maxima and sums combined with
// warp shuffles:
//     out = sum_q 2^(m_q - m) O_q / sum_q 2^(m_q - m) l_q,  m = max_q m_q,
// over the pieces that saw a key (l_q > 0).  Runs after the attention kernel
// (programmatic dependent launch: it waits for that grid's completion).
template <typename T, int D>
__global__ void __launch_bounds__(128) prefill_merge_kernel(const PrefillParams p, const PrefillGrid pg, int tail) {
    griddep_wait();
    const int lane = threadIdx.x & 31;
    const long long gw = (long long)blockIdx.x * 4 + (threadIdx.x >> 5);
    const int ti = (int)(gw / kRowsT), r = (int)(gw % kRowsT);
    if (ti >= tail) return;
    const int G = p.group, item = pg.nfull + ti;
    const int pairs = p.num_kv_heads * p.num_seqs;
    const int g = (item % pairs) % p.num_kv_heads, b = (item % pairs) / p.num_kv_heads;
    const int tile = pg.tx - 1 - item / pairs;
    const int qs = p.query_start[b], L = p.query_start[b + 1] - qs, n = p.context_lens[b];
    const int R = tile * kRowsT + r;
    // the rows the attention kernel computed (its sequence checks, and rows that hold a query)
    if (L <= 0 || R >= L * G || n < L || n > p.max_blocks_per_seq * kBlkT) return;
    constexpr int kRow = part_row_floats(D);
    const float* rows = pg.part + ((size_t)ti * pg.ksplit * kRowsT + r) * kRow;
    const size_t pstride = (size_t)kRowsT * kRow;
    float mq = kNegInfT, lq = 0.f;
    if (lane < pg.ksplit) {
        mq = __ldcg(rows + lane * pstride + D);
        lq = __ldcg(rows + lane * pstride + D + 1);
    }
    float m = lq > 0.f ? mq : kNegInfT;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    const float w = lq > 0.f ? fast_exp2(mq - m) : 0.f;
    float lt = w * lq;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) lt += __shfl_xor_sync(0xffffffffu, lt, o);
    const float inv = lt > 0.f ? 1.f / lt : 0.f;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int q = 0; q < kMaxSplit; ++q) {
        const float f = __shfl_sync(0xffffffffu, w, q) * inv;
        if (q < pg.ksplit && f != 0.f && lane * 4 < D) {
            const float4 o = __ldcg(reinterpret_cast<const float4*>(rows + q * pstride) + lane);
            acc.x += f * o.x;
            acc.y += f * o.y;
            acc.z += f * o.z;
            acc.w += f * o.w;
        }
    }
    if (lane * 4 < D) {
        const int qi = R / G, qk = R - (R / G) * G;
        T* dst = static_cast<T*>(p.out) + ((size_t)(qs + qi) * p.num_heads + g * G + qk) * D + lane * 4;
        *reinterpret_cast<uint2*>(dst) = make_uint2(Elt<T>::pack2(acc.x, acc.y), Elt<T>::pack2(acc.z, acc.w));
    }
}

template <typename T, int D>
cudaError_t launch_prefill_tc_t(const PrefillParams& p_in, void* ws, size_t ws_bytes, cudaStream_t stream) {
    using C = TcPf<D>;
    PrefillParams p = p_in;
    const bool neg = p.scale_log2 < 0.f;   // a negative scale: negate Q inside the QK^T product
    if (neg) p.scale_log2 = -p.scale_log2;
    // a zero scale gives uniform weights; the smallest normal float gives the
    // same ones and keeps masked logits at -inf through the scaling
    if (p.scale_log2 == 0.f) p.scale_log2 = 1.17549435e-38f;
    const bool bf = std::is_same<T, __nv_bfloat16>::value;
    const uint32_t idesc_qk = umma_idesc_f16(bf, kRowsT, kKeysT, false, neg);
    const uint32_t idesc_pv = umma_idesc_f16(bf, kRowsT, D, true, false);
    const pa_dtype dt = bf ? PA_BF16 : PA_F16;
    CUtensorMap mk, mv;
    cudaError_t e = make_pool_map(&mk, p.key_cache, dt, p.num_blocks, p.num_kv_heads, D, kBlkT);
    if (e != cudaSuccess) return e;
    e = make_pool_map(&mv, p.value_cache, dt, p.num_blocks, p.num_kv_heads, D, kBlkT);
    if (e != cudaSuccess) return e;
    auto kernel = prefill_tc_kernel<T, D>;
    e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes);
    if (e != cudaSuccess) return e;
    // 128-row tiles over the (position, head) rows of the longest chunk, one
    // work item per (tile, KV head, sequence); with a workspace, the last
    // partial wave's items are split by key range
    const SplitPlan sp = split_plan(p, sm_count_now());
    PrefillGrid pg{sp.tx, (int)sp.items, 1, nullptr};
    const bool split = ws && sp.tail > 0 && ws_bytes >= sp.bytes;
    if (split) {
        pg.nfull = (int)(sp.items - sp.tail);
        pg.ksplit = sp.ksplit;
        pg.part = static_cast<float*>(ws);
    }
    const long long ctas = pg.nfull + (sp.items - pg.nfull) * pg.ksplit;
    if (ctas > INT32_MAX) return cudaErrorInvalidValue;
    e = launch_pdl(kernel, dim3((unsigned)ctas), dim3(C::kThreads), C::kSmemBytes, stream, p, mk, mv, idesc_qk,
                   idesc_pv, pg);
    if (e != cudaSuccess || !split) return e;
    // one warp per row of the split items
    return launch_pdl(prefill_merge_kernel<T, D>, dim3((unsigned)(sp.tail * kRowsT / 4)), dim3(128), 0, stream, p,
                      pg, sp.tail);
}

}  // namespace

bool prefill_tc_serves(const PrefillParams& p) {
    // tensor-core tiles hold 128 (position, head) rows; when a chunk fills
    // less than a quarter of one (a few tokens per sequence: decode-like and
    // bound by reading the cache), the 16-query mma.sync kernel wastes less
    return (long long)p.max_query_len * p.group >= 32;
}

size_t prefill_tc_workspace_bytes(const PrefillParams& p) {
    return prefill_tc_serves(p) ? split_plan(p, sm_count_now()).bytes : 0;
}

cudaError_t launch_prefill_tc(const PrefillParams& p, void* ws, size_t ws_bytes, pa_dtype dtype, cudaStream_t stream) {
    if (dtype == PA_F16) return p.head_dim == 64 ? launch_prefill_tc_t<__half, 64>(p, ws, ws_bytes, stream)
                                                 : launch_prefill_tc_t<__half, 128>(p, ws, ws_bytes, stream);
    if (dtype == PA_BF16) return p.head_dim == 64 ? launch_prefill_tc_t<__nv_bfloat16, 64>(p, ws, ws_bytes, stream)
                                                  : launch_prefill_tc_t<__nv_bfloat16, 128>(p, ws, ws_bytes, stream);
    return cudaErrorInvalidValue;
}

}  // namespace pa
