// prefill_stream.cu — the streaming heads' work items of a prefill chunk
// (DuoAttention pre-filling: streaming heads attend to the sinks and the recent
// window only), on tcgen05, in persistent CTAs.
//
// Work item = one (batch, streaming query head, 128-query tile), a few key
// tiles each. One CTA per SM takes items (heaviest first) from a counter in
// global memory until none are left, so an item costs its key tiles rather than
// a CTA start, a TMEM allocation, a Q load and an exposed epilogue: the tile
// pipeline runs on across items (the K/V rings and S buffers are indexed by the
// CTA's running tile count) and the next item's Q and first K/V tiles load
// while the previous item's last tiles and epilogue run. The kernel is launched
// behind the retrieval-item kernel (prefill.cu) with programmatic dependent
// launch and takes the SMs that kernel's CTAs leave; it reads nothing that
// kernel writes, and waits for it to complete before its own CTAs exit, so the
// pair completes as one stream-ordered step.
//
// Key tiles of 128 keys are listed per item (fully masked tiles never are): the
// streaming-cache tiles holding the sinks (and the ring when the window of the
// first query reaches below len), chunk tiles holding chunk-resident sinks, then
// the band tiles [first query - recent + 1, last query]. Keys are masked
// element-wise by absolute position only on tiles that need it.
//
// Warp roles (384 threads):
//   warps 0-7  softmax, two threads per query row: warps w and w+4 read the
//              same TMEM lanes (rows 32*(w%4) ..); warp w takes keys 0-63 of
//              every tile, warp w+4 keys 64-127. Each half keeps its own running
//              max, row sum and O accumulator, so the halves never wait for each
//              other inside the key loop; the epilogue combines them with
//              log-sum-exp weights;
//   warp 8     takes the work items and publishes them to the other roles
//              through a 4-slot queue in shared memory; TMA producer of Q and
//              the K tiles (2-stage ring);
//   warp 10    TMA producer of the V tiles (2-stage ring);
//   warp 9     TMEM allocator and MMA issuer (one thread); warp 11 idle.
// TMEM (512 columns): S in two 128-column buffers [0,128) [128,256), then O of
// key half 0 at [256, 256+D) and of key half 1 at [256+D, 256+2D).
// Key tile j (counted over the CTA's items) uses S buffer j&1, so the tensor
// core computes S(j+1) while the softmax works on S(j). Each half writes its P
// (bf16 pairs) back into the S buffer it read, at column +32 (keys 0-63) or +64
// (keys 64-127), and the PV product of that half (A operand in TMEM, four K=16
// steps) accumulates into its own O as soon as its four warps are done. MMA
// issue order per key tile j (one thread; tcgen05 MMAs run in issue order, so a
// later QK never overwrites a P before the PV that reads it): PV_0(j), PV_1(j),
// QK(j+2), where a QK of a new item waits for the last PV of the previous one.
// An item's first PV overwrites O, after the previous item's epilogue has read it.
// Softmax runs in the exp2 domain with a stale-max rule: O and the row sum are
// rescaled only when the row max grows by more than 2^8 (exact: both stay
// relative to the same stale max).
// All operand tiles in shared memory are 128-byte swizzled (TMA writes them,
// the MMA reads them through descriptors). Every mbarrier wait is time-bounded;
// on timeout the CTA records kErrPrefillWait and unwinds.
#include "prefill_common.cuh"

namespace duo {

namespace {

constexpr int kKStages = 2;  // K ring (V: 2 stages)

template <int D>
struct Layout {
    static constexpr int kColBlocks = D / 64;
    static constexpr int kTile = kColBlocks * kTileBytesPerColBlock;  // Q, K or V tile
    static constexpr int kQ = 0;
    static constexpr int kK = kQ + kTile;              // kKStages stages
    static constexpr int kV = kK + kKStages * kTile;   // 2 stages
    static constexpr int kO = kV + 2 * kTile;          // output tile staged for the tile store
    static constexpr int kBar = kO + kTile;
    // Epilogue exchange of the two halves of a row: maxima and row sums
    // [item parity][half][row].
    static constexpr int kXchg = kBar + 40 * 8;
    // Work items handed to the roles: item index [slot], the MMA issuer's tile
    // counts [slot], then the items themselves [slot].
    static constexpr int kQueue = kXchg + 2 * 2 * 2 * 128 * 4;
    static constexpr int kItems = kQueue + 16 * 4;
    static constexpr int kMisc = kItems + 4 * static_cast<int>(sizeof(Item));
    static constexpr int kBytes = kMisc + 64;
    static constexpr int kAlloc = kBytes + 1024;  // slack for 1024-byte alignment
};
static_assert(Layout<128>::kAlloc <= 227 * 1024, "shared memory of one CTA");

// mbarrier indices
constexpr int kQFull = 0;       // one phase per item
constexpr int kQEmpty = 1;      // one phase per item: every QK of the item has run
constexpr int kKFull = 2;       // + K stage (room for 3)
constexpr int kKEmpty = 5;      // + K stage (room for 3)
constexpr int kVFull = 8;       // + V stage
constexpr int kVEmpty = 10;     // + V stage
constexpr int kSFull = 12;      // + S buffer
constexpr int kP0Full = 14;     // + S buffer: P of keys 0-63 written (4 arrivals: warps 0-3)
constexpr int kP1Full = 16;     // + S buffer: P of keys 64-127 written (4 arrivals: warps 4-7)
constexpr int kODone = 18;      // one phase per key tile (both PV halves)
constexpr int kOFinal = 19;     // one phase per item, after its last PV
constexpr int kOEmpty = 20;     // one phase per item: its O read out (8 arrivals: softmax warps)
constexpr int kDrain = 21;
constexpr int kItemFull = 22;   // + queue slot: work item published (producer)
constexpr int kItemEmpty = 26;  // + queue slot: read by every consumer (kConsumers arrivals)
constexpr int kPair = 30;       // + row quarter: both halves of the rows wrote their max and sum (2 arrivals)
constexpr int kStaged = 34;     // one phase per item: the output tile is staged (8 arrivals: softmax warps)
constexpr int kOFree = 35;      // one phase per item: the previous item's tile store has read the staging tile
constexpr int kQueueSlots = 4;
constexpr int kConsumers = 10;  // V producer, MMA issuer, 8 softmax warps
// Every barrier is waited with a phase parity, so none may complete two phases
// beyond the one its waiter waits for. Tiles are counted over all items of the
// CTA (g), items in the order the CTA took them (ord): S and P barriers are per
// S buffer (S(g+2) needs both PV halves of tile g, which need P(g)); OFinal of
// item ord+1 needs OEmpty of item ord, which follows the wait on OFinal(ord);
// Q is reloaded for item ord only after QEmpty(ord-1); a queue slot is refilled
// only after its previous item was read by every consumer.

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
    prefill_stream_kernel(const __grid_constant__ PrefillParams p, const __grid_constant__ PrefillMaps maps) {
    using Lay = Layout<D>;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_addr = smem_u32(smem_raw);
    const uint32_t base = (raw_addr + 1023u) & ~1023u;
    uint8_t* const sbase = smem_raw + (base - raw_addr);
    const uint32_t sQ = base + Lay::kQ;
    const uint32_t sK = base + Lay::kK;
    const uint32_t sV = base + Lay::kV;
    auto bar = [&](int i) { return base + Lay::kBar + 8u * i; };
    volatile float* xchg = reinterpret_cast<volatile float*>(sbase + Lay::kXchg);
    volatile int* queue = reinterpret_cast<volatile int*>(sbase + Lay::kQueue);
    Item* items = reinterpret_cast<Item*>(sbase + Lay::kItems);  // written before, read after the slot's barrier
    volatile uint32_t* tmem_slot = reinterpret_cast<volatile uint32_t*>(sbase + Lay::kMisc);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(sbase + Lay::kMisc + 4);

    const int tid = threadIdx.x;
    const int warp = tid >> 5;
    const int lane = tid & 31;
    const int n_retr_items = p.B * p.n_retr_q * p.n_qt;  // the other kernel's items come first
    const int n_items = p.B * (p.Hq - p.n_retr_q) * p.n_qt;

    if (tid == 0) {
        mbar_init(bar(kQFull), 1);
        mbar_init(bar(kQEmpty), 1);
        for (int s = 0; s < kKStages; ++s) {
            mbar_init(bar(kKFull + s), 1);
            mbar_init(bar(kKEmpty + s), 1);
        }
        for (int s = 0; s < 2; ++s) {
            mbar_init(bar(kVFull + s), 1);
            mbar_init(bar(kVEmpty + s), 1);
            mbar_init(bar(kSFull + s), 1);
            mbar_init(bar(kP0Full + s), 4);
            mbar_init(bar(kP1Full + s), 4);
        }
        mbar_init(bar(kODone), 1);
        mbar_init(bar(kOFinal), 1);
        mbar_init(bar(kOEmpty), 8);
        mbar_init(bar(kDrain), 1);
        for (int s = 0; s < kQueueSlots; ++s) {
            mbar_init(bar(kItemFull + s), 1);
            mbar_init(bar(kItemEmpty + s), kConsumers);
            mbar_init(bar(kPair + s), 2);  // s = row quarter
        }
        mbar_init(bar(kStaged), 8);
        mbar_init(bar(kOFree), 1);
        *abort_flag = 0;
        fence_barrier_init();
        fence_proxy_async_smem();
    }
    if (warp == 9) {
        tmem_alloc(base + Lay::kMisc, kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    // Item `ord` of this CTA from the queue: its index (-1: no more work, -2: the
    // wait gave up) and, for an index >= 0, the item itself. Every consumer reads
    // each slot once and then frees it.
    auto take_item = [&](int ord, Item& out) -> int {
        const int slot = ord % kQueueSlots;
        if (!mbar_wait(bar(kItemFull + slot), (ord / kQueueSlots) & 1, abort_flag)) return -2;
        const int idx = queue[slot];
        if (idx >= 0) out = items[slot];
        mbar_arrive(bar(kItemEmpty + slot));
        return idx;
    };

    if (warp == 8) {
        // ------------------------------------------------------------ work items, Q and K
        // Takes the next item of the launch (heaviest first) as soon as the K tiles
        // of the previous one are issued, publishes it to the other roles, loads its
        // Q once the previous item's QKs have run, then its K tiles.
        if (lane == 0) {
            tma_prefetch_desc(&maps.q);
            // Test of the bounded waits: CTA 0 never issues its first K tile.
            const bool withhold = p.test_withhold != 0 && blockIdx.x == 0;
            int ord = 0, g = 0, issued = 0;
            while (true) {
                int idx = -1;
                Item it;
                while (*abort_flag == 0) {
                    const int i = static_cast<int>(atomicAdd(p.work, 1u));
                    if (i >= n_items) break;
                    it = make_item(p, n_retr_items + i);
                    if (it.n_tiles > 0) {
                        idx = n_retr_items + i;
                        break;
                    }
                }
                const int slot = ord % kQueueSlots;
                if (ord >= kQueueSlots &&
                    !mbar_wait(bar(kItemEmpty + slot), ((ord / kQueueSlots) - 1) & 1, abort_flag)) {
                    record_abort(p.err, abort_flag);
                    break;
                }
                queue[slot] = idx;
                if (idx >= 0) items[slot] = it;
                mbar_arrive(bar(kItemFull + slot));  // release: the consumers see queue[slot] and items[slot]
                if (idx < 0) break;
                // Q of the previous item is free once its last QK has run (the MMA
                // issuer starts this item's QKs only after that item's last PV).
                if (ord >= 1 && !mbar_wait(bar(kQEmpty), (ord - 1) & 1, abort_flag)) {
                    record_abort(p.err, abort_flag);
                    break;
                }
                mbar_arrive_expect_tx(bar(kQFull), Lay::kTile);
                for (int kb = 0; kb < Lay::kColBlocks; ++kb)
                    tma_load_4d(sQ + kb * kTileBytesPerColBlock, &maps.q, bar(kQFull), kb * 64, it.head, it.q0,
                                it.b);
                ++ord;
                bool ok = true;
                for (int j = 0; j < it.n_tiles; ++j, ++g) {
                    const int st = g % kKStages;
                    int src, row0;
                    tile_of(it, j, src, row0);
                    const CUtensorMap* m = src == 0 ? &maps.rk : (src == 1 ? &maps.sk : &maps.k);
                    if (g >= kKStages && !mbar_wait(bar(kKEmpty + st), ((g / kKStages) - 1) & 1, abort_flag)) {
                        record_abort(p.err, abort_flag);
                        ok = false;
                        break;
                    }
                    issued = g + 1;
                    if (withhold && g == 0) continue;
                    mbar_arrive_expect_tx(bar(kKFull + st), Lay::kTile);
                    const int zpool = it.pool * p.B + it.b;
                    for (int kb = 0; kb < Lay::kColBlocks; ++kb) {
                        const uint32_t dst = sK + st * Lay::kTile + kb * kTileBytesPerColBlock;
                        if (src == 2) tma_load_4d(dst, m, bar(kKFull + st), kb * 64, it.g, row0, it.b);
                        else tma_load_3d(dst, m, bar(kKFull + st), kb * 64, row0, zpool);
                    }
                }
                if (!ok) break;
            }
            // Let every load this thread issued land before the CTA can exit.
            for (int j = (issued > kKStages ? issued - kKStages : 0); j < issued; ++j)
                if (!(withhold && j == 0)) mbar_wait(bar(kKFull + j % kKStages), (j / kKStages) & 1, nullptr);
            if (ord > 0) mbar_wait(bar(kQFull), (ord - 1) & 1, nullptr);
        }
    } else if (warp == 10) {
        // ------------------------------------------------------------ V tiles
        if (lane == 0) {
            int g = 0, issued = 0;
            for (int ord = 0;; ++ord) {
                Item it;
                const int idx = take_item(ord, it);
                if (idx == -2) record_abort(p.err, abort_flag);
                if (idx < 0) break;
                bool ok = true;
                for (int j = 0; j < it.n_tiles; ++j, ++g) {
                    const int st = g & 1;
                    int src, row0;
                    tile_of(it, j, src, row0);
                    const CUtensorMap* m = src == 0 ? &maps.rv : (src == 1 ? &maps.sv : &maps.v);
                    if (g >= 2 && !mbar_wait(bar(kVEmpty + st), ((g >> 1) - 1) & 1, abort_flag)) {
                        record_abort(p.err, abort_flag);
                        ok = false;
                        break;
                    }
                    issued = g + 1;
                    mbar_arrive_expect_tx(bar(kVFull + st), Lay::kTile);
                    const int zpool = it.pool * p.B + it.b;
                    for (int kb = 0; kb < Lay::kColBlocks; ++kb) {
                        const uint32_t dst = sV + st * Lay::kTile + kb * kTileBytesPerColBlock;
                        if (src == 2) tma_load_4d(dst, m, bar(kVFull + st), kb * 64, it.g, row0, it.b);
                        else tma_load_3d(dst, m, bar(kVFull + st), kb * 64, row0, zpool);
                    }
                }
                if (!ok) break;
            }
            for (int j = (issued > 2 ? issued - 2 : 0); j < issued; ++j)
                mbar_wait(bar(kVFull + (j & 1)), (j >> 1) & 1, nullptr);
        }
    } else if (warp == 9) {
        // ------------------------------------------------------------ MMA issuer
        // Two cursors over the CTA's tiles: QK runs up to two tiles ahead of PV (it
        // takes the items from the queue; PV follows their tile counts). QK moves on
        // to a new item only once every PV of the previous one is issued: the issuer
        // blocks on the K tile of each QK, and the first K tile of an item is often
        // the slowest load (a cache tile from DRAM), which must not hold back the last
        // PV of the item before it (and with it that item's epilogue).
        if (lane == 0) {
            constexpr uint32_t idesc_qk = idesc_bf16_f32(128, kTileK, 0, 0);
            constexpr uint32_t idesc_pv = idesc_bf16_f32(128, D, 0, 1);
            volatile int* n_of = queue + 8;  // tiles of the items the QK cursor has taken [ord % slots]
            int qk_ord = 0, qk_cur = -1, qk_j = 0, qk_n = 0, qk_g = 0;
            bool qk_end = false;
            int pv_g = 0;  // PVs issued
            // S(qk_g) = Q(item) K(qk_g)^T into S buffer qk_g&1: 1 issued, 0 none to issue
            // now (no tiles left, or the next item waits for the previous one's PVs),
            // -1 failed.
            auto qk_next = [&]() -> int {
                if (qk_end) return 0;
                if (qk_j == qk_n) {
                    if (pv_g != qk_g) return 0;
                    Item it;
                    const int idx = take_item(qk_ord, it);
                    if (idx == -2) return -1;
                    if (idx < 0) {
                        qk_end = true;
                        return 0;
                    }
                    qk_cur = qk_ord++;
                    qk_n = it.n_tiles;
                    n_of[qk_cur % kQueueSlots] = qk_n;
                    qk_j = 0;
                    if (!mbar_wait(bar(kQFull), qk_cur & 1, abort_flag)) return -1;
                }
                const int st = qk_g & 1;         // S buffer
                const int kst = qk_g % kKStages;  // K stage
                const bool withheld = qk_g == 0 && p.test_withhold != 0 && blockIdx.x == 0;
                if (!mbar_wait(bar(kKFull + kst), (qk_g / kKStages) & 1, abort_flag,
                               withheld ? p.test_timeout_ns : kWaitTimeoutNs))
                    return -1;
                tc_fence_after();
                const uint32_t qt = sQ;
                const uint32_t kt = sK + kst * Lay::kTile;
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t off = (kk >> 2) * kTileBytesPerColBlock + (kk & 3) * 32;
                    tc_mma_ss(tmem + st * kTileK, smem_desc_sw128(qt + off, 16, 1024),
                              smem_desc_sw128(kt + off, 16, 1024), idesc_qk, kk > 0 ? 1u : 0u);
                }
                tc_commit(bar(kSFull + st));
                tc_commit(bar(kKEmpty + kst));
                ++qk_j;
                ++qk_g;
                if (qk_j == qk_n) tc_commit(bar(kQEmpty));
                return 1;
            };
            // Keep QK up to two tiles ahead of PV.
            auto fill = [&]() -> bool {
                while (qk_g < pv_g + 2) {
                    const int r = qk_next();
                    if (r < 0) return false;
                    if (r == 0) break;
                }
                return true;
            };
            bool ok = fill();
            int pv_ord = 0, pv_j = 0, pv_n = 0;
            for (int g = 0; ok && g < qk_g; ++g) {
                if (pv_j == pv_n) {  // the first tile of the next item
                    pv_n = n_of[pv_ord % kQueueSlots];
                    pv_j = 0;
                    // O is overwritten by this item's first PV: the previous item's
                    // epilogue must have read it.
                    if (pv_ord >= 1 && !mbar_wait(bar(kOEmpty), (pv_ord - 1) & 1, abort_flag)) {
                        ok = false;
                        break;
                    }
                    ++pv_ord;
                }
                const int st = g & 1;
                if (!mbar_wait(bar(kVFull + st), (g >> 1) & 1, abort_flag)) {
                    ok = false;
                    break;
                }
                // O_h += P_h(g) V_h(g) for the two key halves, each as soon as its
                // four softmax warps have written P_h (in TMEM at S buffer g&1 + kTmemP).
                const uint32_t vt = sV + st * Lay::kTile;
                for (int half = 0; ok && half < 2; ++half) {
                    if (!mbar_wait(bar((half ? kP1Full : kP0Full) + st), (g >> 1) & 1, abort_flag)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
#pragma unroll
                    for (int k4 = 0; k4 < 4; ++k4) {
                        const int kk = half * 4 + k4;
                        const uint64_t bd = smem_desc_sw128(vt + kk * 2048, kTileBytesPerColBlock, 1024);
                        tc_mma_ts(tmem + kTmemO + half * D, tmem + st * kTileK + kTmemP + kk * 8, bd, idesc_pv,
                                  (pv_j > 0 || k4 > 0) ? 1u : 0u);
                    }
                }
                if (!ok) break;
                tc_commit(bar(kODone));
                if (++pv_j == pv_n) tc_commit(bar(kOFinal));
                tc_commit(bar(kVEmpty + st));
                pv_g = g + 1;
                ok = fill();  // S(g+2), or the next item's first tiles
            }
            if (!ok) record_abort(p.err, abort_flag);
            // Drain: every MMA issued above completes before TMEM is released.
            tc_commit(bar(kDrain));
            mbar_wait(bar(kDrain), 0, nullptr);
        }
    } else if (warp < 8) {
        // ------------------------------------------------------------ softmax warps
        // Warps w and w+4 hold the same rows; each owns half of every key tile, its
        // own running max and sum and its own O accumulator, so the two work
        // independently until the epilogue combines them.
        const int quarter = warp & 3;  // TMEM lanes 32*quarter .. (query rows)
        const int h = warp >> 2;       // key half of every tile
        const int row = quarter * 32 + lane;
        const uint32_t lane_base = static_cast<uint32_t>(quarter * 32) << 16;
        const uint32_t tO = tmem + lane_base + kTmemO + h * D;
        const uint64_t scale2 = f2pack(p.scale_log2, p.scale_log2);
        bool ok = true;
        int g = 0;  // key tiles of this CTA so far
        // The warp's lanes read a queue slot together, then lane 0 frees it.
        auto take = [&](int ord, Item& out) -> int {
            const int slot = ord % kQueueSlots;
            if (!__all_sync(0xffffffffu, mbar_wait(bar(kItemFull + slot), (ord / kQueueSlots) & 1, abort_flag)))
                return -2;
            const int idx = queue[slot];
            if (idx >= 0) out = items[slot];
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(kItemEmpty + slot));
            return idx;
        };
        Item it{};
        int idx = take(0, it);
        RowVis vis = row_visible(it.retr, it.L, it.C, p.S, p.R, it.q0 + row);
        if (idx == -2) record_abort(p.err, abort_flag);
        for (int ord = 0; ok && idx >= 0; ++ord) {
            const int n = it.n_tiles;
            const int qrow = it.q0 + row;
            float m_run = -INFINITY;
            float l_run = 0.f;
            for (int j = 0; j < n; ++j, ++g) {
                const int buf = g & 1;
                const uint32_t tS = tmem + lane_base + buf * kTileK;
                // Waits that guard warp-collective tcgen05 instructions are warp-uniform.
                if (!__all_sync(0xffffffffu, mbar_wait(bar(kSFull + buf), (g >> 1) & 1, abort_flag))) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                float s[kHalf];
                {
                    uint32_t r[2][32];
                    tmem_ld32(tS + h * kHalf, r[0]);
                    tmem_ld32(tS + h * kHalf + 32, r[1]);
                    tc_wait_ld();
#pragma unroll
                    for (int c = 0; c < 2; ++c)
#pragma unroll
                        for (int i = 0; i < 32; ++i) s[c * 32 + i] = __uint_as_float(r[c][i]);
                }
                int src, row0;
                tile_of(it, j, src, row0);
                const bool full =
                    it.retr && ((src == 0 && row0 + kTileK <= it.L) || (src == 2 && row0 + kTileK <= it.q0));
                // Each 32-key word of this half: masked element-wise only when some lane
                // of the warp sees part of it; skipped altogether (no max, no exp2, P = 0)
                // when no lane of the warp sees any of its keys. Both tests are
                // warp-uniform, so the branches do not diverge.
                bool live[2] = {true, true};
                if (!full) {
#pragma unroll
                    for (int w = 0; w < 2; ++w) {
                        const uint32_t bits = visible_bits(vis, src, row0 + 32 * (2 * h + w));
                        live[w] = __any_sync(0xffffffffu, bits != 0u);
                        if (live[w] && !__all_sync(0xffffffffu, bits == 0xFFFFFFFFu)) {
#pragma unroll
                            for (int k = 0; k < 32; ++k)
                                if (!((bits >> k) & 1u)) s[w * 32 + k] = -INFINITY;
                        }
                    }
                }
                float m0 = -INFINITY, m1 = -INFINITY, m2 = -INFINITY, m3 = -INFINITY;
                static_assert(kHalf == 64, "two 32-key words per softmax thread and tile");
#pragma unroll
                for (int w = 0; w < 2; ++w) {
                    if (!live[w]) continue;
#pragma unroll
                    for (int i = 32 * w; i < 32 * w + 32; i += 8) {
                        m0 = fmax3(m0, s[i], s[i + 1]);
                        m1 = fmax3(m1, s[i + 2], s[i + 3]);
                        m2 = fmax3(m2, s[i + 4], s[i + 5]);
                        m3 = fmax3(m3, s[i + 6], s[i + 7]);
                    }
                }
                const float mt = fmax3(fmaxf(m0, m1), m2, m3) * p.scale_log2;
                float factor = 1.f;
                if (mt > m_run + kRescaleThreshold) {  // also taken when m_run is -inf and mt finite
                    factor = fast_exp2(m_run - mt);
                    m_run = mt;
                }
                const float m_use = (m_run == -INFINITY) ? 0.f : m_run;
                const uint64_t negm = f2pack(-m_use, -m_use);
                uint64_t acc2[2] = {f2pack(0.f, 0.f), f2pack(0.f, 0.f)};
                uint32_t pk[kHalf / 2];
#pragma unroll
                for (int w = 0; w < 2; ++w) {
                    if (!live[w]) {
#pragma unroll
                        for (int i = 16 * w; i < 16 * w + 16; ++i) pk[i] = 0u;
                        continue;
                    }
#pragma unroll
                    for (int i = 32 * w; i < 32 * w + 32; i += 2) {
                        float e0, e1;
                        f2unpack(ffma2(f2pack(s[i], s[i + 1]), scale2, negm), e0, e1);
                        const float p0 = fast_exp2(e0);
                        const float p1 = fast_exp2(e1);
                        acc2[(i / 2) & 1] = fadd2(acc2[(i / 2) & 1], f2pack(p0, p1));
                        pk[i / 2] = pack_bf16x2(p0, p1);
                    }
                }
                float a0, a1;
                f2unpack(fadd2(acc2[0], acc2[1]), a0, a1);
                l_run = l_run * factor + (a0 + a1);
                tmem_st32(tS + kTmemP + h * (kHalf / 2), pk);  // P of this half (S columns already read)
                // O_h must be complete before it is rescaled: PV(g-1) is the last MMA that
                // wrote it (kODone completes one phase per key tile; the commit behind
                // S(g) covered PV(g-2)). The item's first tile overwrites O instead.
                if (j >= 1 && __any_sync(0xffffffffu, factor != 1.f)) {
                    if (__all_sync(0xffffffffu, mbar_wait(bar(kODone), (g - 1) & 1, abort_flag))) {
                        tc_fence_after();
                        uint32_t r[32];
#pragma unroll
                        for (int c = 0; c < D / 32; ++c) {
                            tmem_ld32(tO + c * 32, r);
                            tc_wait_ld();
#pragma unroll
                            for (int i = 0; i < 32; ++i) r[i] = __float_as_uint(__uint_as_float(r[i]) * factor);
                            tmem_st32(tO + c * 32, r);
                        }
                    } else {
                        ok = false;
                        record_abort(p.err, abort_flag);
                    }
                }
                tc_wait_st();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(bar((h ? kP1Full : kP0Full) + buf));
                if (!ok) break;
            }
            if (!ok) {
                record_abort(p.err, abort_flag);
                break;
            }
            // The next item (taken and its row bounds computed while this item's last PV
            // runs, before the epilogue waits for it).
            Item nit{};
            const int nidx = take(ord + 1, nit);
            const RowVis nvis = row_visible(nit.retr, nit.L, nit.C, p.S, p.R, nit.q0 + row);
            // Combine the halves: O = (O_0 2^(m_0-m) + O_1 2^(m_1-m)) / (l_0 2^(m_0-m) + l_1 2^(m_1-m)),
            // each thread of a pair writing D/2 of the row's columns. The exchange
            // buffers alternate between items, so a fast pair member never overwrites
            // what its partner has yet to read.
            volatile float* xm = xchg + (ord & 1) * 512;  // [half][row] running max
            volatile float* xl = xm + 256;                // [half][row] row sum
            xm[h * 128 + row] = m_run;
            xl[h * 128 + row] = l_run;
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(kPair + quarter));
            if (!__all_sync(0xffffffffu, mbar_wait(bar(kPair + quarter), ord & 1, abort_flag))) {
                ok = false;
                record_abort(p.err, abort_flag);
                break;
            }
            const float m_o = xm[(1 - h) * 128 + row];
            const float l_o = xl[(1 - h) * 128 + row];
            const float m_all = fmaxf(m_run, m_o);  // finite: every row sees at least its own key
            const float f_self = (m_run == -INFINITY) ? 0.f : fast_exp2(m_run - m_all);
            const float f_o = (m_o == -INFINITY) ? 0.f : fast_exp2(m_o - m_all);
            const float inv = 1.f / (l_run * f_self + l_o * f_o);
            const float f0 = (h == 0 ? f_self : f_o) * inv;
            const float f1 = (h == 0 ? f_o : f_self) * inv;
            if (!__all_sync(0xffffffffu, mbar_wait(bar(kOFinal), ord & 1, abort_flag))) {
                ok = false;
                record_abort(p.err, abort_flag);
                break;
            }
            tc_fence_after();
            // A tile whose 128 rows are all output rows goes out as one tile store from
            // shared memory (128-byte swizzled like the operand tiles); other tiles
            // (the last rows of a sequence's chunk) are stored row by row. One
            // thread issues the stores; the staging tile is rewritten only after the
            // previous item's store has read it, and the phases of kOFree (arrived
            // after the issuer's own wait on this item's O) never run ahead of a
            // warp that has yet to wait on them.
            const bool issuer = warp == 0 && lane == 0;
            if (issuer) {
                bulk_wait_group_read0();
                mbar_arrive(bar(kOFree));
            }
            if (!__all_sync(0xffffffffu, mbar_wait(bar(kOFree), ord & 1, abort_flag))) {
                ok = false;
                record_abort(p.err, abort_flag);
                break;
            }
            const bool tile_store = it.q0 + kTileQ <= it.C;
            const uint32_t tO0 = tmem + lane_base + kTmemO + h * (D / 2);
            bf16* orow = p.out + ((static_cast<int64_t>(it.b) * p.C + qrow) * p.Hq + it.head) * D + h * (D / 2);
            uint32_t r0[32], r1[32];
#pragma unroll
            for (int c = 0; c < D / 64; ++c) {
                tmem_ld32(tO0 + c * 32, r0);
                tmem_ld32(tO0 + D + c * 32, r1);
                tc_wait_ld();
#pragma unroll
                for (int v8 = 0; v8 < 4; ++v8) {
                    uint32_t w[4];
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        const int e = v8 * 8 + 2 * i;
                        w[i] = pack_bf16x2(__uint_as_float(r0[e]) * f0 + __uint_as_float(r1[e]) * f1,
                                           __uint_as_float(r0[e + 1]) * f0 + __uint_as_float(r1[e + 1]) * f1);
                    }
                    if (tile_store) {
                        const int col = h * (D / 2) + c * 32 + v8 * 8;
                        const int off = (col >> 6) * kTileBytesPerColBlock + row * 128 +
                                        ((((col & 63) >> 3) ^ (row & 7)) << 4);
                        *reinterpret_cast<uint4*>(sbase + Lay::kO + off) = make_uint4(w[0], w[1], w[2], w[3]);
                    } else if (qrow < it.C) {
                        *reinterpret_cast<uint4*>(orow + c * 32 + v8 * 8) = make_uint4(w[0], w[1], w[2], w[3]);
                    }
                }
            }
            if (tile_store) fence_proxy_async_smem();  // generic writes -> visible to the tile store
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(kStaged));
            if (issuer) {
                if (mbar_wait(bar(kStaged), ord & 1, abort_flag)) {
                    if (tile_store) {
                        for (int kb = 0; kb < Lay::kColBlocks; ++kb)
                            tma_store_4d(&maps.out, base + Lay::kO + kb * kTileBytesPerColBlock, kb * 64, it.head,
                                         it.q0, it.b);
                        bulk_commit_group();
                    }
                } else {
                    ok = false;
                    record_abort(p.err, abort_flag);
                }
            }
            // O is read: the next item's first PV may overwrite it.
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(kOEmpty));
            if (nidx == -2) {
                ok = false;
                record_abort(p.err, abort_flag);
            }
            idx = nidx;
            it = nit;
            vis = nvis;
        }
        if (warp == 0 && lane == 0) bulk_wait_group0();  // every tile store completes before the CTA exits
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 9) tmem_dealloc(tmem, kTmemCols);
    if (tid == 0) {
        // The last CTA of the launch resets the item counters for the next launch
        // (every CTA has stopped taking items by the time it counts itself done).
        __threadfence();
        if (atomicAdd(p.work + 1, 1u) == gridDim.x - 1) {
            p.work[0] = 0u;
            p.work[1] = 0u;
            __threadfence();
        }
    }
    // Complete only after the retrieval-item kernel this one was launched behind
    // (a no-op without that dependency).
    grid_dependency_wait();
}

template <int D>
cudaError_t launch_d(const PrefillParams& p, const PrefillMaps& maps, int num_sms, bool after_retrieval,
                     cudaStream_t s) {
    // Same shared-memory request for every D (one CTA per SM); one CTA per SM,
    // each taking items until none are left.
    const int smem = Layout<128>::kAlloc;
    static SmemLimitOnce limit;
    cudaError_t e = limit.apply(reinterpret_cast<const void*>(&prefill_stream_kernel<D>), smem);
    if (e != cudaSuccess) return e;
    const int n_items = p.B * (p.Hq - p.n_retr_q) * p.n_qt;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(n_items < num_sms ? n_items : num_sms));
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = after_retrieval ? 1 : 0;  // otherwise an ordinary stream-ordered launch
    return cudaLaunchKernelEx(&cfg, prefill_stream_kernel<D>, p, maps);
}

}  // namespace

cudaError_t launch_prefill_streaming(const PrefillParams& p, const PrefillMaps& maps, int num_sms,
                                     bool after_retrieval, cudaStream_t s) {
    if (p.B * (p.Hq - p.n_retr_q) * p.n_qt == 0) return cudaSuccess;
    if (num_sms < 1) return cudaErrorInvalidValue;
    if (p.D == 128) return launch_d<128>(p, maps, num_sms, after_retrieval, s);
    if (p.D == 64) return launch_d<64>(p, maps, num_sms, after_retrieval, s);
    return cudaErrorInvalidValue;
}

}  // namespace duo
