// prefill.cu — mixed-head attention of one prefill chunk (DuoAttention
// pre-filling), retrieval and streaming heads in one launch, on tcgen05.
//
// One CTA = one (batch, query head, pair of 128-query tiles) work item: tiles
// A = queries [256t, 256t+128) and B = [256t+128, 256t+256) of the chunk share
// every K/V tile the CTA loads. Retrieval items come first, heaviest (last
// tile pair) first; streaming items fill in behind them.
//
// Key tiles of 128 keys are listed per item and fully masked tiles are never
// listed (the list is the union of what A and B need):
//   retrieval: cache tiles covering [0, len) of the retrieval pool, then chunk
//              tiles 0 .. (B's diagonal tile);
//   streaming: the streaming-cache tiles holding the sinks (and the ring when
//              the window of A's first query reaches below len), chunk tiles
//              holding chunk-resident sinks, then the band tiles
//              [first query of A - recent + 1, last query of B].
// Keys are masked element-wise by absolute position only on tiles that need it.
//
// Warp roles (384 threads, three warpgroups):
//   warps 0-3  softmax of tile A: thread t owns query row t (TMEM lane t);
//   warps 4-7  softmax of tile B, same lanes, other TMEM columns;
//   warp 8     TMA producer: Q_A and Q_B once, then K/V tiles into 2-stage rings;
//   warp 9     TMEM allocator and MMA issuer (one thread); warps 10-11 idle.
// Registers: launched at 168 per thread; the third warpgroup gives back down
// to 72 and the softmax warpgroups take 216 (2*128*216 + 128*72 = 384*168).
// TMEM (512 columns): S_A [0,128), S_B [128,256), O_A [256,384), O_B [384,512).
// The softmax writes P (bf16 pairs) back into its S columns at +32 and the
// PV product reads it from there (A operand in TMEM). MMAs issued by one
// thread execute in order, so S_X(j+1) is written only after PV_X(j) read P_X(j).
// MMA issue order per key tile j:
//   PV_A(j), QK_A(j+1), PV_B(j), QK_B(j+1)
// so the tensor core works on one tile while the other tile's softmax runs.
// Softmax runs in the exp2 domain with a stale-max rule: O and the row sum are
// rescaled only when the row max grows by more than 2^8 (exact: both stay
// relative to the same stale max). A commit after QK_X(j+1) covers PV_X(j),
// so O_X is stable when the softmax sees S_X(j+1).
// All operand tiles in shared memory are 128-byte swizzled (TMA writes them,
// the MMA reads them through descriptors). Every mbarrier wait is time-bounded;
// on timeout the CTA records kErrPrefillWait and unwinds.
#include "duo_internal.cuh"
#include "sm100.cuh"

namespace duo {

namespace {

constexpr int kThreads = 384;
constexpr int kSoftmaxRegs = 216;
constexpr int kControlRegs = 72;
static_assert(2 * 128 * kSoftmaxRegs + 128 * kControlRegs <= kThreads * 168, "register split exceeds the launch");
constexpr int kTileBytesPerColBlock = kTileQ * 128;  // 128 rows x 64 bf16 (128 B)
constexpr float kRescaleThreshold = 8.0f;             // log2 units: rescale when max grows by > 2^8

template <int D>
struct Layout {
    static constexpr int kColBlocks = D / 64;
    static constexpr int kTile = kColBlocks * kTileBytesPerColBlock;  // Q, K or V tile
    static constexpr int kQA = 0;
    static constexpr int kQB = kQA + kTile;
    static constexpr int kK = kQB + kTile;      // 2 stages
    static constexpr int kV = kK + 2 * kTile;   // 2 stages
    static constexpr int kBar = kV + 2 * kTile;
    static constexpr int kMisc = kBar + 32 * 8;
    static constexpr int kBytes = kMisc + 64;
    static constexpr int kAlloc = kBytes + 1024;  // slack for 1024-byte alignment
};

enum Bar {
    kQFull = 0,
    kKFull = 1,    // +stage
    kVFull = 3,    // +stage
    kKEmpty = 5,   // +stage
    kVEmpty = 7,   // +stage
    kSFull = 9,    // +tile (A, B)
    kPFull = 11,   // +tile
    kOFinal = 13,  // +tile
    kDrain = 15,
};

constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kTmemP = 32;  // P of tile X at S_X + 32 (64 columns of bf16 pairs)

__device__ __forceinline__ uint32_t tmem_s(int x) { return x ? 128u : 0u; }
__device__ __forceinline__ uint32_t tmem_o(int x) { return x ? 384u : 256u; }

// What one work item attends to.
struct Item {
    int b, head, g, tp, retr, pool;
    int q0a, q0b;  // first chunk row of tile A / B (scalars: no local memory)
    int n_cache;  // cache tiles
    int src_cache;
    int a;        // streaming: chunk tiles holding chunk-resident sinks
    int b0;       // streaming: first band tile after them
    int n_tiles;
};

__device__ __forceinline__ Item make_item(const PrefillParams& p) {
    Item it;
    const int n_tp = (p.n_qt + 1) / 2;
    const int n_retr_items = p.n_retr_q * p.B * n_tp;
    int idx = blockIdx.x;
    int nh, hbase;
    if (idx < n_retr_items) {
        nh = p.n_retr_q;
        hbase = 0;
    } else {
        idx -= n_retr_items;
        nh = p.Hq - p.n_retr_q;
        hbase = p.n_retr_q;
    }
    it.tp = n_tp - 1 - idx / (nh * p.B);
    const int rem = idx % (nh * p.B);
    it.head = p.qhead[hbase + rem / p.B];
    it.b = rem % p.B;
    it.g = it.head / p.G;
    it.retr = p.heads.is_retr[it.g];
    it.pool = p.heads.pool_idx[it.g];
    it.q0a = it.tp * 2 * kTileQ;
    it.q0b = it.q0a + kTileQ;
    const int qt_last = (2 * it.tp + 1 < p.n_qt) ? 2 * it.tp + 1 : 2 * it.tp;
    const int64_t L = p.len;
    if (it.retr) {
        it.src_cache = 0;
        it.n_cache = static_cast<int>((L + kTileK - 1) / kTileK);
        it.a = 0;
        it.b0 = 0;
        it.n_tiles = it.n_cache + qt_last + 1;
    } else {
        it.src_cache = 1;
        int64_t slots = 0;
        if (L > 0) {
            const bool band_in_cache = (L > p.S) && (it.q0a < p.R - 1);
            slots = band_in_cache ? (L < p.W ? L : p.W) : (L < p.S ? L : p.S);
        }
        it.n_cache = static_cast<int>((slots + kTileK - 1) / kTileK);
        int a = 0;
        if (L < p.S) {
            const int64_t sink_rows = (p.S - L < p.C) ? (p.S - L) : p.C;
            a = static_cast<int>((sink_rows + kTileK - 1) / kTileK);
            if (a > qt_last + 1) a = qt_last + 1;
        }
        const int band_lo = it.q0a - p.R + 1 > 0 ? it.q0a - p.R + 1 : 0;
        const int tb = band_lo / kTileK;
        it.a = a;
        it.b0 = a > tb ? a : tb;
        it.n_tiles = it.n_cache + a + (qt_last + 1 - it.b0);
    }
    return it;
}

// Tile t of an item: source (0 retrieval pool, 1 streaming pool, 2 chunk) and first row.
__device__ __forceinline__ void tile_of(const Item& it, int t, int& src, int& row0) {
    if (t < it.n_cache) {
        src = it.src_cache;
        row0 = t * kTileK;
        return;
    }
    const int u = t - it.n_cache;
    src = 2;
    row0 = (it.retr || u < it.a) ? u * kTileK : (it.b0 + u - it.a) * kTileK;
}

__device__ __forceinline__ void record_abort(uint32_t* err, volatile int* abort_flag) {
    *abort_flag = 1;
    atomicOr(err, kErrPrefillWait);
}

// Bits k of a 32-bit word set for k < x (x clamped to [0, 32]).
__device__ __forceinline__ uint32_t bits_below(int64_t x) {
    if (x <= 0) return 0u;
    if (x >= 32) return 0xFFFFFFFFu;
    return (1u << static_cast<uint32_t>(x)) - 1u;
}

// Visibility of keys [32w, 32w+32) of tile (src, row0) from chunk query row
// `qrow` (absolute position len + qrow), one bit per key.
//   src 0 (retrieval cache): slot j holds position j, valid for j < len.
//   src 1 (streaming cache): sink slots j < sink hold position j; ring slot
//     sink + r holds the latest position p < len with (p - sink) mod recent == r;
//     visible when inside the query's window.
//   src 2 (chunk): row c is position len + c, valid for c < C, causal, and for
//     streaming heads a sink (len + c < sink) or inside the window.
__device__ __forceinline__ uint32_t visible_bits(const PrefillParams& p, int retr, int src, int row0, int w,
                                                 int qrow, int64_t ring_last_r) {
    const int64_t L = p.len;
    const int base = row0 + 32 * w;
    if (src == 0) return bits_below(L - base);
    if (src == 2) {
        const int hi = (qrow < p.C - 1 ? qrow : p.C - 1);
        const uint32_t causal = bits_below(static_cast<int64_t>(hi) + 1 - base);
        if (retr) return causal;
        const uint32_t sink = bits_below(static_cast<int64_t>(p.S) - L - base);
        const uint32_t band = ~bits_below(static_cast<int64_t>(qrow) - p.R + 1 - base);
        return causal & (sink | band);
    }
    const int64_t pq = L + qrow;
    const int64_t last = L - 1;
    uint32_t bits = 0;
    for (int k = 0; k < 32; ++k) {
        const int64_t slot = base + k;
        bool vis;
        if (slot < p.S) {
            vis = slot < L;
        } else if (slot < p.W && L > p.S) {
            const int64_t r = slot - p.S;
            const int64_t back = (r <= ring_last_r) ? (ring_last_r - r) : (ring_last_r - r + p.R);
            const int64_t pos = last - back;
            vis = (pos >= p.S) && (pq - pos < p.R);
        } else {
            vis = false;
        }
        bits |= static_cast<uint32_t>(vis) << k;
    }
    return bits;
}

// ---------------------------------------------------------------- packed fp32 pairs
__device__ __forceinline__ uint64_t f2pack(float lo, float hi) {
    uint64_t r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
    return r;
}
__device__ __forceinline__ void f2unpack(uint64_t v, float& lo, float& hi) {
    asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
__device__ __forceinline__ uint64_t ffma2(uint64_t a, uint64_t b, uint64_t c) {
    uint64_t d;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
    return d;
}
__device__ __forceinline__ uint64_t fadd2(uint64_t a, uint64_t b) {
    uint64_t d;
    asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}

// D[tmem] (+)= A[tmem] * B[smem], kind::f16: the PV product with P held in TMEM.
__device__ __forceinline__ void tc_mma_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                          uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
        "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
    prefill_kernel(const __grid_constant__ PrefillParams p, const __grid_constant__ PrefillMaps maps) {
    using Lay = Layout<D>;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_addr = smem_u32(smem_raw);
    const uint32_t base = (raw_addr + 1023u) & ~1023u;
    uint8_t* const sbase = smem_raw + (base - raw_addr);
    const uint32_t sK = base + Lay::kK;
    const uint32_t sV = base + Lay::kV;
    auto sQ = [&](int x) { return base + (x ? Lay::kQB : Lay::kQA); };
    auto bar = [&](int i) { return base + Lay::kBar + 8u * i; };
    volatile uint32_t* tmem_slot = reinterpret_cast<volatile uint32_t*>(sbase + Lay::kMisc);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(sbase + Lay::kMisc + 4);

    const int tid = threadIdx.x;
    const int warp = tid >> 5;
    const int lane = tid & 31;
    const Item it = make_item(p);

    if (tid == 0) {
        mbar_init(bar(kQFull), 1);
        for (int s = 0; s < 2; ++s) {
            mbar_init(bar(kKFull + s), 1);
            mbar_init(bar(kVFull + s), 1);
            mbar_init(bar(kKEmpty + s), 1);
            mbar_init(bar(kVEmpty + s), 1);
            mbar_init(bar(kSFull + s), 1);
            mbar_init(bar(kPFull + s), 4);
            mbar_init(bar(kOFinal + s), 1);
        }
        mbar_init(bar(kDrain), 1);
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

    // Each role's code stays inside the branch that sets its register budget.
    if (warp >= 8) {
        asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kControlRegs));
    if (warp == 8) {
        // ------------------------------------------------------------ TMA producer
        if (lane == 0) {
            tma_prefetch_desc(&maps.q);
            mbar_arrive_expect_tx(bar(kQFull), 2 * Lay::kTile);
            for (int x = 0; x < 2; ++x)
                for (int kb = 0; kb < Lay::kColBlocks; ++kb)
                    tma_load_4d(sQ(x) + kb * kTileBytesPerColBlock, &maps.q, bar(kQFull), kb * 64, it.head, x ? it.q0b : it.q0a,
                                it.b);
            int issued = 0;
            for (int j = 0; j < n; ++j) {
                const int st = j & 1;
                const uint32_t use = j >> 1;
                int src, row0;
                tile_of(it, j, src, row0);
                const CUtensorMap* mk = src == 0 ? &maps.rk : (src == 1 ? &maps.sk : &maps.k);
                const CUtensorMap* mv = src == 0 ? &maps.rv : (src == 1 ? &maps.sv : &maps.v);
                const int zpool = it.pool * p.B + it.b;
                if (j >= 2 && !mbar_wait(bar(kKEmpty + st), (use - 1) & 1, abort_flag)) {
                    record_abort(p.err, abort_flag);
                    break;
                }
                mbar_arrive_expect_tx(bar(kKFull + st), Lay::kTile);
                for (int kb = 0; kb < Lay::kColBlocks; ++kb) {
                    const uint32_t dst = sK + st * Lay::kTile + kb * kTileBytesPerColBlock;
                    if (src == 2) tma_load_4d(dst, mk, bar(kKFull + st), kb * 64, it.g, row0, it.b);
                    else tma_load_3d(dst, mk, bar(kKFull + st), kb * 64, row0, zpool);
                }
                if (j >= 2 && !mbar_wait(bar(kVEmpty + st), (use - 1) & 1, abort_flag)) {
                    record_abort(p.err, abort_flag);
                    issued = 2 * j + 1;
                    break;
                }
                mbar_arrive_expect_tx(bar(kVFull + st), Lay::kTile);
                for (int kb = 0; kb < Lay::kColBlocks; ++kb) {
                    const uint32_t dst = sV + st * Lay::kTile + kb * kTileBytesPerColBlock;
                    if (src == 2) tma_load_4d(dst, mv, bar(kVFull + st), kb * 64, it.g, row0, it.b);
                    else tma_load_3d(dst, mv, bar(kVFull + st), kb * 64, row0, zpool);
                }
                issued = 2 * j + 2;
            }
            // Let every load this thread issued land before the CTA can exit.
            const int nk = (issued + 1) / 2, nv = issued / 2;  // tiles with K / V issued
            for (int j = (nk > 2 ? nk - 2 : 0); j < nk; ++j)
                mbar_wait(bar(kKFull + (j & 1)), (j >> 1) & 1, nullptr);
            for (int j = (nv > 2 ? nv - 2 : 0); j < nv; ++j)
                mbar_wait(bar(kVFull + (j & 1)), (j >> 1) & 1, nullptr);
        }
    } else if (warp == 9) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            constexpr uint32_t idesc_qk = idesc_bf16_f32(128, kTileK, 0, 0);
            constexpr uint32_t idesc_pv = idesc_bf16_f32(128, D, 0, 1);
            auto qk = [&](int x, int j) {
                const uint32_t kt = sK + (j & 1) * Lay::kTile;
                const uint32_t qt = sQ(x);
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t off = (kk >> 2) * kTileBytesPerColBlock + (kk & 3) * 32;
                    tc_mma_ss(tmem + tmem_s(x), smem_desc_sw128(qt + off, 16, 1024),
                              smem_desc_sw128(kt + off, 16, 1024), idesc_qk, kk > 0 ? 1u : 0u);
                }
                tc_commit(bar(kSFull + x));
            };
            auto pv = [&](int x, int j) {
                const uint32_t vt = sV + (j & 1) * Lay::kTile;
#pragma unroll
                for (int kk = 0; kk < kTileK / 16; ++kk) {
                    const uint64_t bd = smem_desc_sw128(vt + kk * 2048, kTileBytesPerColBlock, 1024);
                    tc_mma_ts(tmem + tmem_o(x), tmem + tmem_s(x) + kTmemP + kk * 8, bd, idesc_pv,
                              (j > 0 || kk > 0) ? 1u : 0u);
                }
            };
            bool ok = mbar_wait(bar(kQFull), 0, abort_flag) && mbar_wait(bar(kKFull + 0), 0, abort_flag);
            if (ok) {
                tc_fence_after();
                qk(0, 0);
                qk(1, 0);
                tc_commit(bar(kKEmpty + 0));
            }
            for (int j = 0; ok && j < n; ++j) {
                const int st = j & 1;
                const bool more = j + 1 < n;
                if (!mbar_wait(bar(kVFull + st), (j >> 1) & 1, abort_flag) ||
                    !mbar_wait(bar(kPFull + 0), j & 1, abort_flag)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                pv(0, j);
                if (!more) tc_commit(bar(kOFinal + 0));
                if (more) {
                    if (!mbar_wait(bar(kKFull + ((j + 1) & 1)), ((j + 1) >> 1) & 1, abort_flag)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    qk(0, j + 1);
                }
                if (!mbar_wait(bar(kPFull + 1), j & 1, abort_flag)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                pv(1, j);
                tc_commit(bar(kVEmpty + st));
                if (!more) tc_commit(bar(kOFinal + 1));
                if (more) {
                    qk(1, j + 1);
                    tc_commit(bar(kKEmpty + ((j + 1) & 1)));
                }
            }
            if (!ok) record_abort(p.err, abort_flag);
            // Drain: every MMA issued above completes before TMEM is released.
            tc_commit(bar(kDrain));
            mbar_wait(bar(kDrain), 0, nullptr);
        }
    }
    } else {
        asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kSoftmaxRegs));
        // ------------------------------------------------------------ softmax warps
        const int x = warp >> 2;          // 0: tile A (warps 0-3), 1: tile B (warps 4-7)
        const int row = tid & 127;        // TMEM lane == query row of the tile
        const int q0 = x ? it.q0b : it.q0a;
        const int qrow = q0 + row;
        const uint32_t lane_base = static_cast<uint32_t>((warp & 3) * 32) << 16;
        const uint32_t tS = tmem + lane_base + tmem_s(x);
        const uint32_t tO = tmem + lane_base + tmem_o(x);
        const int64_t ring_last_r = (p.len > p.S) ? (p.len - 1 - p.S) % p.R : 0;
        const uint64_t scale2 = f2pack(p.scale_log2, p.scale_log2);
        float m_run = -INFINITY;
        float l_run = 0.f;
        bool ok = true;
        for (int j = 0; j < n; ++j) {
            // Waits that guard warp-collective tcgen05 instructions are made
            // warp-uniform, so a timeout can never split a warp at one of them.
            if (!__all_sync(0xffffffffu, mbar_wait(bar(kSFull + x), j & 1, abort_flag))) {
                ok = false;
                break;
            }
            tc_fence_after();
            float s[kTileK];
            {
                uint32_t r[32];
#pragma unroll
                for (int c = 0; c < kTileK / 32; ++c) {
                    tmem_ld32(tS + c * 32, r);
                    tc_wait_ld();
#pragma unroll
                    for (int i = 0; i < 32; ++i) s[c * 32 + i] = __uint_as_float(r[i]);
                }
            }
            int src, row0;
            tile_of(it, j, src, row0);
            const bool full =
                it.retr && ((src == 0 && row0 + kTileK <= p.len) || (src == 2 && row0 + kTileK <= q0));
            if (!full) {
#pragma unroll
                for (int w = 0; w < kTileK / 32; ++w) {
                    const uint32_t bits = visible_bits(p, it.retr, src, row0, w, qrow, ring_last_r);
#pragma unroll
                    for (int k = 0; k < 32; ++k)
                        if (!((bits >> k) & 1u)) s[w * 32 + k] = -INFINITY;
                }
            }
            float mt = fmaxf(s[0], s[1]);
#pragma unroll
            for (int i = 2; i < kTileK; ++i) mt = fmaxf(mt, s[i]);
            mt *= p.scale_log2;
            float factor = 1.f;
            if (mt > m_run + kRescaleThreshold) {  // also taken when m_run is -inf and mt finite
                factor = fast_exp2(m_run - mt);
                m_run = mt;
            }
            const float m_use = (m_run == -INFINITY) ? 0.f : m_run;
            const uint64_t negm = f2pack(-m_use, -m_use);

            // O_X is stable here: the commit behind S_X(j) covered PV_X(j-1).
            if (j >= 1 && __any_sync(0xffffffffu, factor != 1.f)) {
                uint32_t r[32];
#pragma unroll
                for (int c = 0; c < D / 32; ++c) {
                    tmem_ld32(tO + c * 32, r);
                    tc_wait_ld();
#pragma unroll
                    for (int i = 0; i < 32; ++i) r[i] = __float_as_uint(__uint_as_float(r[i]) * factor);
                    tmem_st32(tO + c * 32, r);
                }
            }
            // P = exp2(s * scale - m) as bf16 pairs, stored into TMEM 64 keys at a time.
            uint64_t acc2 = f2pack(0.f, 0.f);
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                uint32_t pk[32];
#pragma unroll
                for (int i = 0; i < 64; i += 2) {
                    float e0, e1;
                    f2unpack(ffma2(f2pack(s[h * 64 + i], s[h * 64 + i + 1]), scale2, negm), e0, e1);
                    const float p0 = fast_exp2(e0);
                    const float p1 = fast_exp2(e1);
                    acc2 = fadd2(acc2, f2pack(p0, p1));
                    pk[i / 2] = pack_bf16x2(p0, p1);
                }
                tmem_st32(tS + kTmemP + h * 32, pk);
            }
            float a0, a1;
            f2unpack(acc2, a0, a1);
            l_run = l_run * factor + (a0 + a1);
            tc_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(kPFull + x));
        }
        if (__all_sync(0xffffffffu, ok && mbar_wait(bar(kOFinal + x), 0, abort_flag))) {
            tc_fence_after();
            const float inv = 1.f / l_run;
            bf16* orow = p.out + ((static_cast<int64_t>(it.b) * p.C + qrow) * p.Hq + it.head) * D;
            uint32_t r[32];
#pragma unroll
            for (int c = 0; c < D / 32; ++c) {
                tmem_ld32(tO + c * 32, r);
                tc_wait_ld();
                if (qrow < p.C) {
#pragma unroll
                    for (int v8 = 0; v8 < 4; ++v8) {
                        uint4 o;
                        o.x = pack_bf16x2(__uint_as_float(r[v8 * 8 + 0]) * inv, __uint_as_float(r[v8 * 8 + 1]) * inv);
                        o.y = pack_bf16x2(__uint_as_float(r[v8 * 8 + 2]) * inv, __uint_as_float(r[v8 * 8 + 3]) * inv);
                        o.z = pack_bf16x2(__uint_as_float(r[v8 * 8 + 4]) * inv, __uint_as_float(r[v8 * 8 + 5]) * inv);
                        o.w = pack_bf16x2(__uint_as_float(r[v8 * 8 + 6]) * inv, __uint_as_float(r[v8 * 8 + 7]) * inv);
                        *reinterpret_cast<uint4*>(orow + c * 32 + v8 * 8) = o;
                    }
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
cudaError_t launch_d(const PrefillParams& p, const PrefillMaps& maps, cudaStream_t s) {
    // Same shared-memory request for every D: one CTA per SM, so a CTA never
    // waits on another for TMEM columns.
    const int smem = Layout<128>::kAlloc;
    cudaError_t e = cudaFuncSetAttribute(prefill_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    const unsigned grid = static_cast<unsigned>(p.B * p.Hq * ((p.n_qt + 1) / 2));
    prefill_kernel<D><<<grid, kThreads, smem, s>>>(p, maps);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_prefill(const PrefillParams& p, const PrefillMaps& maps, cudaStream_t s) {
    if (p.B * p.Hq * p.n_qt == 0) return cudaSuccess;
    if (p.D == 128) return launch_d<128>(p, maps, s);
    if (p.D == 64) return launch_d<64>(p, maps, s);
    return cudaErrorInvalidValue;
}

}  // namespace duo
