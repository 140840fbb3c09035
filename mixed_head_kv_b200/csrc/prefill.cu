// prefill.cu — mixed-head attention of one prefill chunk (DuoAttention
// pre-filling) on tcgen05: the retrieval heads' work items, one per CTA, and
// the launch of both prefill kernels.
//
// Work item = one (batch, query head, 128-query tile). This kernel runs the
// retrieval items, one per CTA, heaviest (last query tile) first; the streaming
// items (a few key tiles each, so a CTA start, a Q load and an epilogue per item
// would weigh on them) run in prefill_stream.cu's persistent kernel, launched
// right behind this one with programmatic dependent launch: its CTAs take the
// SMs that this grid's CTAs leave.
//
// Key tiles of 128 keys are listed per item and fully masked tiles are never
// listed:
//   retrieval: cache tiles covering [0, len) of the retrieval pool, then chunk
//              tiles 0 .. (the diagonal tile);
//   streaming: the streaming-cache tiles holding the sinks (and the ring when
//              the window of the first query reaches below len), chunk tiles
//              holding chunk-resident sinks, then the band tiles
//              [first query - recent + 1, last query].
// Keys are masked element-wise by absolute position only on tiles that need it.
//
// Warp roles (384 threads):
//   warps 0-7  softmax, two threads per query row: warps w and w+4 read the
//              same TMEM lanes (rows 32*(w%4) ..); warp w takes keys 0-63 of
//              every tile, warp w+4 keys 64-127. Each half keeps its own running
//              max, row sum and O accumulator, so the halves never wait for each
//              other inside the key loop; the epilogue combines them with
//              log-sum-exp weights;
//   warp 8     TMA producer of Q and the K tiles (2-stage ring);
//   warp 10    TMA producer of the V tiles (2-stage ring);
//   warp 9     TMEM allocator and MMA issuer (one thread); warp 11 idle.
// TMEM (512 columns): S in two 128-column buffers [0,128) [128,256), then O of
// key half 0 at [256, 256+D) and of key half 1 at [256+D, 256+2D).
// Key tile j uses S buffer j&1, so the tensor core computes S(j+1) while the
// softmax works on S(j). Each half writes its P (bf16 pairs) back into the S
// buffer it read, at column +32 (keys 0-63) or +64 (keys 64-127), and the PV
// product of that half (A operand in TMEM, four K=16 steps) accumulates into
// its own O as soon as its four warps are done. MMA issue order per key tile j
// (one thread; tcgen05 MMAs run in issue order, so a later QK never overwrites
// a P before the PV that reads it): PV_0(j), PV_1(j), QK(j+2).
// Softmax runs in the exp2 domain with a stale-max rule: O and the row sum are
// rescaled only when the row max grows by more than 2^8 (exact: both stay
// relative to the same stale max).
// All operand tiles in shared memory are 128-byte swizzled (TMA writes them,
// the MMA reads them through descriptors). Every mbarrier wait is time-bounded;
// on timeout the CTA records kErrPrefillWait and unwinds.
#include "prefill_common.cuh"

namespace duo {

namespace {


template <int D>
struct Layout {
    static constexpr int kColBlocks = D / 64;
    static constexpr int kTile = kColBlocks * kTileBytesPerColBlock;  // Q, K or V tile
    static constexpr int kQ = 0;
    static constexpr int kK = kQ + kTile;       // 2 stages
    static constexpr int kV = kK + 2 * kTile;   // 2 stages
    static constexpr int kO = kV + 2 * kTile;   // output tile staged for the tile store
    static constexpr int kBar = kO + kTile;
    // Pair exchange: maxima [tile parity][half][row], ok flags [parity][half][quarter],
    // row sums [half][row].
    static constexpr int kXchg = kBar + 32 * 8;
    static constexpr int kMisc = kXchg + (2 * 2 * 128 + 2 * 2 * 4 + 2 * 128) * 4;
    static constexpr int kBytes = kMisc + 64;
    static constexpr int kAlloc = kBytes + 1024;  // slack for 1024-byte alignment
};
static_assert(Layout<128>::kAlloc <= 227 * 1024, "shared memory of one CTA");

// mbarrier indices
constexpr int kQFull = 0;
constexpr int kKFull = 1;      // + stage
constexpr int kVFull = 3;      // + stage
constexpr int kKEmpty = 5;     // + stage
constexpr int kVEmpty = 7;     // + stage
constexpr int kSFull = 9;      // + S buffer
constexpr int kP0Full = 11;    // + S buffer: P of keys 0-63 written (4 arrivals: warps 0-3)
constexpr int kP1Full = 13;    // + S buffer: P of keys 64-127 written (4 arrivals: warps 4-7)
constexpr int kODone = 15;     // one phase per key tile (both PV halves)
constexpr int kOFinal = 16;    // one phase, after the last PV
constexpr int kDrain = 17;
constexpr int kStaged = 18;    // the output tile is staged (8 arrivals: softmax warps)
// Every barrier is waited with a phase parity, so none may complete two phases
// beyond the one its waiter waits for: S and P barriers are per S buffer (P(j+2)
// needs S(j+2), which needs both PV halves of tile j to have consumed P(j)) and
// the output waits on a single-phase barrier.

// Named barrier over the two warps (64 threads) that share one row quarter.
__device__ __forceinline__ void pair_sync(int quarter) {
    asm volatile("bar.sync %0, 64;" ::"r"(1 + quarter) : "memory");
}

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
    prefill_kernel(const __grid_constant__ PrefillParams p, const __grid_constant__ PrefillMaps maps) {
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
    volatile uint32_t* tmem_slot = reinterpret_cast<volatile uint32_t*>(sbase + Lay::kMisc);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(sbase + Lay::kMisc + 4);

    // The streaming-item kernel behind this one reads nothing this grid writes: it
    // may start as soon as every CTA of this grid is resident.
    grid_launch_dependents();
    const int tid = threadIdx.x;
    const int warp = tid >> 5;
    const int lane = tid & 31;
    const Item it = make_item(p, static_cast<int>(blockIdx.x));
    if (it.n_tiles == 0) return;  // uniform over the CTA, before any barrier or TMEM use

    if (tid == 0) {
        mbar_init(bar(kQFull), 1);
        for (int s = 0; s < 2; ++s) {
            mbar_init(bar(kKFull + s), 1);
            mbar_init(bar(kVFull + s), 1);
            mbar_init(bar(kKEmpty + s), 1);
            mbar_init(bar(kVEmpty + s), 1);
            mbar_init(bar(kSFull + s), 1);
            mbar_init(bar(kP0Full + s), 4);
            mbar_init(bar(kP1Full + s), 4);
        }
        mbar_init(bar(kODone), 1);
        mbar_init(bar(kOFinal), 1);
        mbar_init(bar(kDrain), 1);
        mbar_init(bar(kStaged), 8);
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
    const int n = it.n_tiles;

    if (warp == 8 || warp == 10) {
        // ------------------------------------------------------------ TMA producers
        // Warp 8 loads Q and the K tiles, warp 10 the V tiles: K runs ahead of V,
        // gated only by the QK products that free its stages.
        if (lane == 0) {
            const bool is_k = warp == 8;
            if (is_k) {
                tma_prefetch_desc(&maps.q);
                mbar_arrive_expect_tx(bar(kQFull), Lay::kTile);
                for (int kb = 0; kb < Lay::kColBlocks; ++kb)
                    tma_load_4d(sQ + kb * kTileBytesPerColBlock, &maps.q, bar(kQFull), kb * 64, it.head, it.q0, it.b);
            }
            const uint32_t ring = is_k ? sK : sV;
            const int full = is_k ? kKFull : kVFull;
            const int empty = is_k ? kKEmpty : kVEmpty;
            // Test of the bounded waits: CTA 0 never issues its first K tile.
            const bool withhold = is_k && p.test_withhold != 0 && blockIdx.x == 0;
            int issued = 0;  // tiles whose load was issued
            for (int j = 0; j < n; ++j) {
                const int st = j & 1;
                int src, row0;
                tile_of(it, j, src, row0);
                const CUtensorMap* m =
                    is_k ? (src == 0 ? &maps.rk : (src == 1 ? &maps.sk : &maps.k))
                         : (src == 0 ? &maps.rv : (src == 1 ? &maps.sv : &maps.v));
                const int zpool = it.pool * p.B + it.b;
                if (j >= 2 && !mbar_wait(bar(empty + st), ((j >> 1) - 1) & 1, abort_flag)) {
                    record_abort(p.err, abort_flag);
                    break;
                }
                issued = j + 1;
                if (withhold && j == 0) continue;
                mbar_arrive_expect_tx(bar(full + st), Lay::kTile);
                for (int kb = 0; kb < Lay::kColBlocks; ++kb) {
                    const uint32_t dst = ring + st * Lay::kTile + kb * kTileBytesPerColBlock;
                    if (src == 2) tma_load_4d(dst, m, bar(full + st), kb * 64, it.g, row0, it.b);
                    else tma_load_3d(dst, m, bar(full + st), kb * 64, row0, zpool);
                }
            }
            // Let every load this thread issued land before the CTA can exit.
            for (int j = (issued > 2 ? issued - 2 : 0); j < issued; ++j)
                if (!(withhold && j == 0)) mbar_wait(bar(full + (j & 1)), (j >> 1) & 1, nullptr);
        }
    } else if (warp == 9) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            constexpr uint32_t idesc_qk = idesc_bf16_f32(128, kTileK, 0, 0);
            constexpr uint32_t idesc_pv = idesc_bf16_f32(128, D, 0, 1);
            // S(j) = Q K(j)^T into S buffer j&1.
            auto qk = [&](int j) -> bool {
                const int st = j & 1;
                const bool withheld = j == 0 && p.test_withhold != 0 && blockIdx.x == 0;
                if (!mbar_wait(bar(kKFull + st), (j >> 1) & 1, abort_flag,
                               withheld ? p.test_timeout_ns : kWaitTimeoutNs))
                    return false;
                tc_fence_after();
                const uint32_t kt = sK + st * Lay::kTile;
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t off = (kk >> 2) * kTileBytesPerColBlock + (kk & 3) * 32;
                    tc_mma_ss(tmem + st * kTileK, smem_desc_sw128(sQ + off, 16, 1024),
                              smem_desc_sw128(kt + off, 16, 1024), idesc_qk, kk > 0 ? 1u : 0u);
                }
                tc_commit(bar(kSFull + st));
                tc_commit(bar(kKEmpty + st));
                return true;
            };
            bool ok = mbar_wait(bar(kQFull), 0, abort_flag);
            for (int j = 0; ok && j < 2 && j < n; ++j) ok = qk(j);
            for (int j = 0; ok && j < n; ++j) {
                const int st = j & 1;
                if (!mbar_wait(bar(kVFull + st), (j >> 1) & 1, abort_flag)) {
                    ok = false;
                    break;
                }
                // O_h += P_h(j) V_h(j) for the two key halves, each as soon as its
                // four softmax warps have written P_h (in TMEM at S buffer j&1 + kTmemP).
                const uint32_t vt = sV + st * Lay::kTile;
                for (int half = 0; ok && half < 2; ++half) {
                    if (!mbar_wait(bar((half ? kP1Full : kP0Full) + st), (j >> 1) & 1, abort_flag)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
#pragma unroll
                    for (int k4 = 0; k4 < 4; ++k4) {
                        const int kk = half * 4 + k4;
                        const uint64_t bd = smem_desc_sw128(vt + kk * 2048, kTileBytesPerColBlock, 1024);
                        tc_mma_ts(tmem + kTmemO + half * D, tmem + st * kTileK + kTmemP + kk * 8, bd, idesc_pv,
                                  (j > 0 || k4 > 0) ? 1u : 0u);
                    }
                }
                if (!ok) break;
                tc_commit(bar(kODone));
                if (j + 1 == n) tc_commit(bar(kOFinal));
                tc_commit(bar(kVEmpty + st));
                if (j + 2 < n) ok = qk(j + 2);
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
        const int qrow = it.q0 + row;
        const uint32_t lane_base = static_cast<uint32_t>(quarter * 32) << 16;
        const uint32_t tO = tmem + lane_base + kTmemO + h * D;
        const RowVis vis = row_visible(it.retr, it.L, it.C, p.S, p.R, qrow);
        const uint64_t scale2 = f2pack(p.scale_log2, p.scale_log2);
        volatile float* xm = xchg;        // [half][row] running max
        volatile float* xl = xchg + 256;  // [half][row] row sum
        float m_run = -INFINITY;
        float l_run = 0.f;
        bool ok = true;
        for (int j = 0; j < n; ++j) {
            const int buf = j & 1;
            const uint32_t tS = tmem + lane_base + buf * kTileK;
            // Waits that guard warp-collective tcgen05 instructions are warp-uniform.
            if (!(ok && __all_sync(0xffffffffu, mbar_wait(bar(kSFull + buf), (j >> 1) & 1, abort_flag)))) {
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
            // O_h must be complete before it is rescaled: PV(j-1) is the last MMA that
            // wrote it (kODone completes one phase per key tile; the commit behind
            // S(j) covered PV(j-2)).
            if (j >= 1 && __any_sync(0xffffffffu, factor != 1.f)) {
                if (__all_sync(0xffffffffu, mbar_wait(bar(kODone), (j - 1) & 1, abort_flag))) {
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
        // Combine the halves: O = (O_0 2^(m_0-m) + O_1 2^(m_1-m)) / (l_0 2^(m_0-m) + l_1 2^(m_1-m)),
        // each thread of a pair writing D/2 of the row's columns.
        xm[h * 128 + row] = m_run;
        xl[h * 128 + row] = l_run;
        pair_sync(quarter);
        const float m_o = xm[(1 - h) * 128 + row];
        const float l_o = xl[(1 - h) * 128 + row];
        const float m_all = fmaxf(m_run, m_o);  // finite: every row sees at least its own key
        const float f_self = (m_run == -INFINITY) ? 0.f : fast_exp2(m_run - m_all);
        const float f_o = (m_o == -INFINITY) ? 0.f : fast_exp2(m_o - m_all);
        const float inv = 1.f / (l_run * f_self + l_o * f_o);
        const float f0 = (h == 0 ? f_self : f_o) * inv;
        const float f1 = (h == 0 ? f_o : f_self) * inv;
        if (__all_sync(0xffffffffu, ok && mbar_wait(bar(kOFinal), 0, abort_flag))) {
            tc_fence_after();
            // A tile whose 128 rows are all output rows goes out as one tile store from
            // shared memory (128-byte swizzled), issued by one thread once every
            // softmax warp has staged its part; other tiles (the last rows of a
            // sequence's chunk) are stored row by row.
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
            if (warp == 0 && lane == 0) {
                if (mbar_wait(bar(kStaged), 0, abort_flag)) {
                    if (tile_store) {
                        for (int kb = 0; kb < Lay::kColBlocks; ++kb)
                            tma_store_4d(&maps.out, base + Lay::kO + kb * kTileBytesPerColBlock, kb * 64, it.head,
                                         it.q0, it.b);
                        bulk_commit_group();
                        bulk_wait_group0();  // completes before the CTA exits
                    }
                } else {
                    record_abort(p.err, abort_flag);
                }
            }
        } else {
            record_abort(p.err, abort_flag);
        }
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 9) tmem_dealloc(tmem, kTmemCols);
}

template <int D>
cudaError_t launch_d(const PrefillParams& p, const PrefillMaps& maps, int n_items, cudaStream_t s) {
    // Same shared-memory request for every D: one CTA per SM, so a CTA never
    // waits on another for TMEM columns.
    const int smem = Layout<128>::kAlloc;
    static SmemLimitOnce limit;
    cudaError_t e = limit.apply(reinterpret_cast<const void*>(&prefill_kernel<D>), smem);
    if (e != cudaSuccess) return e;
    prefill_kernel<D><<<static_cast<unsigned>(n_items), kThreads, smem, s>>>(p, maps);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_prefill(const PrefillParams& p, const PrefillMaps& maps, int num_sms, cudaStream_t s) {
    if (p.D != 128 && p.D != 64) return cudaErrorInvalidValue;
    const int n_retr_items = p.B * p.n_retr_q * p.n_qt;
    const int n_strm_items = p.B * (p.Hq - p.n_retr_q) * p.n_qt;
    if (n_retr_items > 0) {
        const cudaError_t e = p.D == 128 ? launch_d<128>(p, maps, n_retr_items, s) : launch_d<64>(p, maps, n_retr_items, s);
        if (e != cudaSuccess) return e;
    }
    if (n_strm_items > 0) return launch_prefill_streaming(p, maps, num_sms, n_retr_items > 0, s);
    return cudaSuccess;
}

}  // namespace duo
