// prefill.cu — mixed-head attention of one prefill chunk (DuoAttention
// pre-filling), retrieval and streaming heads in one launch, on tcgen05.
//
// One CTA = one (batch, query head, 128-query tile) work item. Retrieval items
// come first, heaviest (last query tile) first, so the block scheduler runs the
// long ones early; streaming items fill in behind them.
//
// Key tiles of 128 keys are listed per item and fully masked tiles are never
// listed:
//   retrieval: cache tiles covering [0, len) of the retrieval pool, then chunk
//              tiles 0 .. (the diagonal tile);
//   streaming: the streaming-cache tiles that hold the sinks (and the ring, if
//              the window of the first query reaches below len), then chunk
//              tiles holding chunk-resident sinks, then the band tiles
//              [first query - recent + 1, last query].
// Keys are masked element-wise by absolute position only on tiles that need it.
//
// Warp roles (192 threads):
//   warps 0-3  softmax: thread t owns query row t (TMEM lane t); reads S from
//              TMEM, masks, online softmax in the exp2 domain with a stale-max
//              rule (rescale O only when the row max grows by more than 2^8),
//              writes P (bf16) into shared memory, and the output at the end;
//   warp 4     TMA producer: Q once, then K/V tiles into 2-stage rings;
//   warp 5     TMEM allocator and MMA issuer (one thread): S = Q K^T into one
//              of two TMEM buffers, O += P V into a TMEM accumulator.
// All operand tiles are 128-byte swizzled (TMA writes them, the MMA reads them
// through shared-memory descriptors). Every mbarrier wait is time-bounded; on
// timeout the CTA records kErrPrefillWait and unwinds.
#include "duo_internal.cuh"
#include "sm100.cuh"

namespace duo {

namespace {

constexpr int kThreads = 192;
constexpr int kTileBytesPerColBlock = kTileQ * 128;  // 128 rows x 64 bf16 (128 B)
constexpr float kRescaleThreshold = 8.0f;             // log2 units: rescale when max grows by > 2^8

template <int D>
struct Layout {
    static constexpr int kColBlocks = D / 64;
    static constexpr int kTile = kColBlocks * kTileBytesPerColBlock;  // Q, K or V tile
    static constexpr int kQ = 0;
    static constexpr int kK = kQ + kTile;        // 2 stages
    static constexpr int kV = kK + 2 * kTile;    // 2 stages
    static constexpr int kP = kV + 2 * kTile;    // 128 x 128 bf16, 2 column blocks
    static constexpr int kBar = kP + 2 * kTileBytesPerColBlock;
    static constexpr int kMisc = kBar + 16 * 8;
    static constexpr int kBytes = kMisc + 64;
    static constexpr int kAlloc = kBytes + 1024;  // slack for 1024-byte alignment
};

enum Bar {
    kQFull = 0,
    kKFull = 1,   // +stage
    kVFull = 3,   // +stage
    kKEmpty = 5,  // +stage
    kVEmpty = 7,  // +stage
    kSFull = 9,   // +buffer
    kSFree = 11,  // +buffer
    kPFull = 13,
    kODone = 14,
    kDrain = 15,
};

constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kTmemO = 256;  // S buffers at columns 0 and 128

// What one work item attends to.
struct Item {
    int b, head, g, qt, retr, pool;
    int n_cache;  // cache tiles
    int src_cache;
    int a;        // streaming: chunk tiles holding chunk-resident sinks
    int b0;       // streaming: first band tile after them
    int n_tiles;
};

__device__ __forceinline__ Item make_item(const PrefillParams& p) {
    Item it;
    const int n_retr_items = p.n_retr_q * p.B * p.n_qt;
    int idx = blockIdx.x;
    int nh, hbase;
    if (idx < n_retr_items) {
        nh = p.n_retr_q;
        hbase = 0;
        it.qt = p.n_qt - 1 - idx / (nh * p.B);
    } else {
        idx -= n_retr_items;
        nh = p.Hq - p.n_retr_q;
        hbase = p.n_retr_q;
        it.qt = p.n_qt - 1 - idx / (nh * p.B);
    }
    const int rem = idx % (nh * p.B);
    it.head = p.qhead[hbase + rem / p.B];
    it.b = rem % p.B;
    it.g = it.head / p.G;
    it.retr = p.heads.is_retr[it.g];
    it.pool = p.heads.pool_idx[it.g];
    const int64_t L = p.len;
    const int q0 = it.qt * kTileQ;
    if (it.retr) {
        it.src_cache = 0;
        it.n_cache = static_cast<int>((L + kTileK - 1) / kTileK);
        it.a = 0;
        it.b0 = 0;
        it.n_tiles = it.n_cache + it.qt + 1;
    } else {
        it.src_cache = 1;
        int64_t slots = 0;
        if (L > 0) {
            const bool band_in_cache = (L > p.S) && (q0 < p.R - 1);
            slots = band_in_cache ? (L < p.W ? L : p.W) : (L < p.S ? L : p.S);
        }
        it.n_cache = static_cast<int>((slots + kTileK - 1) / kTileK);
        int a = 0;
        if (L < p.S) {
            const int64_t sink_rows = (p.S - L < p.C) ? (p.S - L) : p.C;
            a = static_cast<int>((sink_rows + kTileK - 1) / kTileK);
            if (a > it.qt + 1) a = it.qt + 1;
        }
        const int band_lo = q0 - p.R + 1 > 0 ? q0 - p.R + 1 : 0;
        const int tb = band_lo / kTileK;
        it.a = a;
        it.b0 = a > tb ? a : tb;
        it.n_tiles = it.n_cache + a + (it.qt + 1 - it.b0);
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
    const uint32_t sP = base + Lay::kP;
    auto bar = [&](int i) { return base + Lay::kBar + 8u * i; };
    volatile uint32_t* tmem_slot = reinterpret_cast<volatile uint32_t*>(sbase + Lay::kMisc);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(sbase + Lay::kMisc + 4);

    const int tid = threadIdx.x;
    const int warp = tid >> 5;
    const int lane = tid & 31;
    const Item it = make_item(p);
    const int q0 = it.qt * kTileQ;

    if (tid == 0) {
        mbar_init(bar(kQFull), 1);
        for (int s = 0; s < 2; ++s) {
            mbar_init(bar(kKFull + s), 1);
            mbar_init(bar(kVFull + s), 1);
            mbar_init(bar(kKEmpty + s), 1);
            mbar_init(bar(kVEmpty + s), 1);
            mbar_init(bar(kSFull + s), 1);
            mbar_init(bar(kSFree + s), 4);
        }
        mbar_init(bar(kPFull), 4);
        mbar_init(bar(kODone), 1);
        mbar_init(bar(kDrain), 1);
        *abort_flag = 0;
        fence_barrier_init();
        fence_proxy_async_smem();
    }
    if (warp == 5) {
        tmem_alloc(base + Lay::kMisc, kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const int n = it.n_tiles;

    if (warp == 4) {
        // ------------------------------------------------------------ TMA producer
        if (lane == 0) {
            tma_prefetch_desc(&maps.q);
            mbar_arrive_expect_tx(bar(kQFull), Lay::kTile);
            for (int kb = 0; kb < Lay::kColBlocks; ++kb)
                tma_load_4d(sQ + kb * kTileBytesPerColBlock, &maps.q, bar(kQFull), kb * 64, it.head, q0, it.b);
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
    } else if (warp == 5) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            constexpr uint32_t idesc_qk = idesc_bf16_f32(128, kTileK, 0, 0);
            constexpr uint32_t idesc_pv = idesc_bf16_f32(128, D, 0, 1);
            bool ok = mbar_wait(bar(kQFull), 0, abort_flag);
            auto issue_pv = [&](int jj) -> bool {
                const int st = jj & 1;
                if (!mbar_wait(bar(kPFull), jj & 1, abort_flag)) return false;
                if (!mbar_wait(bar(kVFull + st), (jj >> 1) & 1, abort_flag)) return false;
                tc_fence_after();
                const uint32_t vt = sV + st * Lay::kTile;
#pragma unroll
                for (int kk = 0; kk < kTileK / 16; ++kk) {
                    const uint64_t ad = smem_desc_sw128(sP + (kk >> 2) * kTileBytesPerColBlock + (kk & 3) * 32, 16, 1024);
                    const uint64_t bd = smem_desc_sw128(vt + kk * 2048, kTileBytesPerColBlock, 1024);
                    tc_mma_ss(tmem + kTmemO, ad, bd, idesc_pv, (jj > 0 || kk > 0) ? 1u : 0u);
                }
                tc_commit(bar(kODone));
                tc_commit(bar(kVEmpty + st));
                return true;
            };
            for (int j = 0; ok && j < n; ++j) {
                const int st = j & 1;
                if (!mbar_wait(bar(kKFull + st), (j >> 1) & 1, abort_flag)) { ok = false; break; }
                if (j >= 2 && !mbar_wait(bar(kSFree + st), ((j >> 1) - 1) & 1, abort_flag)) { ok = false; break; }
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
                if (j >= 1 && !issue_pv(j - 1)) { ok = false; break; }
            }
            if (ok && n > 0) ok = issue_pv(n - 1);
            if (!ok) record_abort(p.err, abort_flag);
            // Drain: every MMA issued above completes before TMEM is released.
            tc_commit(bar(kDrain));
            mbar_wait(bar(kDrain), 0, nullptr);
        }
    } else {
        // ------------------------------------------------------------ softmax warps 0-3
        const int row = tid;  // TMEM lane == query row of the tile
        const int qrow = q0 + row;
        // Ring slot of the newest cached non-sink position (streaming heads).
        const int64_t ring_last_r = (p.len > p.S) ? (p.len - 1 - p.S) % p.R : 0;
        const uint32_t lane_base = static_cast<uint32_t>(warp * 32) << 16;
        float m_run = -INFINITY;
        float l_run = 0.f;
        bool ok = true;
        for (int j = 0; j < n; ++j) {
            const int buf = j & 1;
            if (!mbar_wait(bar(kSFull + buf), (j >> 1) & 1, abort_flag)) { ok = false; break; }
            tc_fence_after();
            float s[kTileK];
            {
                uint32_t r[32];
#pragma unroll
                for (int c = 0; c < kTileK / 32; ++c) {
                    tmem_ld32(tmem + lane_base + buf * kTileK + c * 32, r);
                    tc_wait_ld();
#pragma unroll
                    for (int i = 0; i < 32; ++i) s[c * 32 + i] = __uint_as_float(r[i]);
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(kSFree + buf));

            int src, row0;
            tile_of(it, j, src, row0);
            const bool full = it.retr && ((src == 0 && row0 + kTileK <= p.len) || (src == 2 && row0 < q0));
            if (!full) {
#pragma unroll
                for (int w = 0; w < kTileK / 32; ++w) {
                    const uint32_t bits = visible_bits(p, it.retr, src, row0, w, qrow, ring_last_r);
#pragma unroll
                    for (int k = 0; k < 32; ++k)
                        if (!((bits >> k) & 1u)) s[w * 32 + k] = -INFINITY;
                }
            }
            float mt = s[0];
#pragma unroll
            for (int i = 1; i < kTileK; ++i) mt = fmaxf(mt, s[i]);
            mt *= p.scale_log2;
            float factor = 1.f;
            if (mt > m_run + kRescaleThreshold) {  // also taken when m_run is -inf and mt finite
                factor = fast_exp2(m_run - mt);
                m_run = mt;
            }
            const float m_use = (m_run == -INFINITY) ? 0.f : m_run;
            float rs = 0.f;
            uint32_t pk[kTileK / 2];
#pragma unroll
            for (int i = 0; i < kTileK; i += 2) {
                const float p0 = fast_exp2(fmaf(s[i], p.scale_log2, -m_use));
                const float p1 = fast_exp2(fmaf(s[i + 1], p.scale_log2, -m_use));
                rs += p0 + p1;
                pk[i / 2] = pack_bf16x2(p0, p1);
            }
            l_run = l_run * factor + rs;

            // PV of the previous tile must be done: it reads the P buffer and accumulates O.
            if (j >= 1) {
                if (!mbar_wait(bar(kODone), (j - 1) & 1, abort_flag)) { ok = false; break; }
                tc_fence_after();
                if (__any_sync(0xffffffffu, factor != 1.f)) {
                    uint32_t r[32];
#pragma unroll
                    for (int c = 0; c < D / 32; ++c) {
                        const uint32_t ta = tmem + lane_base + kTmemO + c * 32;
                        tmem_ld32(ta, r);
                        tc_wait_ld();
#pragma unroll
                        for (int i = 0; i < 32; ++i) r[i] = __float_as_uint(__uint_as_float(r[i]) * factor);
                        tmem_st32(ta, r);
                    }
                    tc_wait_st();
                }
            }
            uint8_t* prow = sbase + Lay::kP + row * 128;
#pragma unroll
            for (int kb = 0; kb < 2; ++kb) {
#pragma unroll
                for (int c = 0; c < 8; ++c) {
                    const int w0 = kb * 32 + c * 4;
                    *reinterpret_cast<uint4*>(prow + kb * kTileBytesPerColBlock + ((c ^ (row & 7)) << 4)) =
                        make_uint4(pk[w0], pk[w0 + 1], pk[w0 + 2], pk[w0 + 3]);
                }
            }
            fence_proxy_async_smem();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(kPFull));
        }
        if (ok && n > 0 && mbar_wait(bar(kODone), (n - 1) & 1, abort_flag)) {
            tc_fence_after();
            const float inv = 1.f / l_run;
            bf16* orow = p.out + ((static_cast<int64_t>(it.b) * p.C + qrow) * p.Hq + it.head) * D;
            uint32_t r[32];
#pragma unroll
            for (int c = 0; c < D / 32; ++c) {
                tmem_ld32(tmem + lane_base + kTmemO + c * 32, r);
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
        } else if (n > 0) {
            record_abort(p.err, abort_flag);
        }
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 5) tmem_dealloc(tmem, kTmemCols);
}

template <int D>
cudaError_t launch_d(const PrefillParams& p, const PrefillMaps& maps, cudaStream_t s) {
    // Same shared-memory request for every D: one CTA per SM, so a CTA never
    // waits on another for TMEM columns.
    const int smem = Layout<128>::kAlloc;
    cudaError_t e = cudaFuncSetAttribute(prefill_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    const unsigned grid = static_cast<unsigned>(p.B * p.Hq * p.n_qt);
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
