// decode_tc.cu — one DuoAttention decoding step on the tensor cores, for query
// groups of G = 4 and 8 heads with head_dim 128 (the group's queries share every
// K/V row, so the per-row dot products and the P·V update form small matrix
// products), over bf16 caches or caches whose retrieval rows are E4M3 codes.
//
// Work items, one CTA each (one CTA per SM), the same items as the
// CUDA-core kernel (decode.cu):
//   retrieval (b, KV head, split): keys [s*split_rows, min((s+1)*split_rows, len+1))
//     of the full cache; partial (o, log2-sum-exp2) to scratch, merged by the
//     last CTA of the (b, KV head);
//   streaming (b, KV head): the min(len+1, sink+recent) valid slots of the sink
//     + ring cache, written straight to `out`.
// The CTA that owns position len first writes the new token into its cache
// slot (for a streaming head, the ring slot that held position len - recent,
// outside the new query's window) and then reads it back with the other rows.
//
// Roles:
//   warps 0-3  softmax: thread t owns key t of every 128-key tile (TMEM lane t);
//   warp 4     TMA producer of the K and V tiles (3-stage rings, 128-B swizzle);
//   warp 5     TMEM allocator and MMA issuer (one thread);
//   warps 6-13 (E4M3 caches only) converters: a retrieval item's K and V tiles
//              arrive as one-byte codes (staging rings of 3 K and 2 V stages)
//              and these warps write them as f16 into 128-B-swizzled operand
//              tiles (2 stages each): warps 6-9 the K tiles, warps 10-13 the V
//              tiles, each group on its own chain (a K stage is free once its
//              QK product has run, a V stage once its PV product has);
//              every E4M3 value is exact in f16, so the item's products run in
//              f16 (the queries and P too), k_scale folded into the score scale
//              and v_scale into the output. Streaming items stay bf16 and load
//              straight into the operand tiles.
// Per key tile j (keys r0 + 128j ..):
//   S^T(j) = K(j) Q^T    M = 128 keys, N = 16 (the G query heads, zero-padded),
//                        K = head_dim; A = the K tile (K-major), B = the queries
//                        (K-major, built once in shared memory);
//   P^T(j)               thread t writes the G probabilities of key t as bf16 into
//                        a 16 x 128 K-major buffer (double-buffered);
//   O^T += V(j)^T P^T(j) M = 128 output columns, N = 16, K = 128 keys; A = the V
//                        tile read MN-major, B = P^T; O^T lives in TMEM (lane = column).
// S^T is double-buffered in TMEM: QK(j+2) is issued after PV(j) (tcgen05 MMAs of
// one thread run in issue order). The running max of each head is shared by the
// CTA and raised only when a score exceeds it by more than 2^8 (one barrier
// reduction per tile decides). Every mbarrier wait is time-bounded; on timeout
// the CTA records kErrDecodeCopy, drains what it issued and unwinds.
#include <cfloat>

#include "duo_internal.cuh"
#include "sm100.cuh"
#include "decode_merge.cuh"

namespace duo {

namespace {

constexpr int kTcD = 128;
constexpr int kTcKeys = 128;                    // keys per tile
constexpr int kTcN = 16;                        // query heads padded to the MMA's N
constexpr int kTcTile = kTcKeys * kTcD * 2;     // one K or V operand tile: 32 KB
constexpr int kTcCodeTile = kTcKeys * kTcD;     // one K or V tile of E4M3 codes: 16 KB
constexpr int kTcColBlock = kTcKeys * 128;      // 128 rows x 128 B (64 two-byte elements)
constexpr int kTcQBytes = kTcN * kTcD * 2;      // 4 KB: 2 column blocks of 16 rows x 128 B
constexpr int kTcPBytes = kTcN * kTcKeys * 2;   // 4 KB: 2 key blocks of 16 rows x 128 B
constexpr float kTcRescale = 8.0f;

// Shared-memory map (offsets from a 1024-byte-aligned base). bf16 caches: 3
// operand stages. E4M3 caches: 2 operand stages and 2 stages of code staging.
template <bool Fp8>
struct TcLayout {
    static constexpr int kThreads = Fp8 ? 448 : 192;
    static constexpr int kStages = Fp8 ? 2 : 3;  // operand stages (K and V tiles)
    static constexpr int kOffK = 0;
    static constexpr int kOffV = kOffK + kStages * kTcTile;
    // E4M3 code staging: 3 stages of K codes (their loads run two tiles ahead of
    // the K conversion), 2 of V codes (the V conversion of tile j waits for PV(j-2)).
    static constexpr int kCodeStagesK = 3;
    static constexpr int kCodeStagesV = 2;
    static constexpr int kOffCK = kOffV + kStages * kTcTile;
    static constexpr int kOffCV = kOffCK + (Fp8 ? kCodeStagesK * kTcCodeTile : 0);
    static constexpr int kOffQ = kOffCV + (Fp8 ? kCodeStagesV * kTcCodeTile : 0);
    static constexpr int kOffP = kOffQ + kTcQBytes;                 // 2 buffers
    static constexpr int kOffBar = kOffP + 2 * kTcPBytes;
    static constexpr int kOffRed = kOffBar + 40 * 8;                // [2][4 warps][16 heads] floats
    static constexpr int kOffMisc = kOffRed + 2 * 4 * kTcN * 4;
    static constexpr int kSmem = kOffMisc + 64 + 1024;              // + slack for 1024-byte alignment
    static_assert(kSmem <= 227 * 1024, "shared memory of one CTA");
};

// mbarriers
constexpr int bKFull = 0;    // + stage: K operand tile loaded (TMA) or converted (4 converter warps)
constexpr int bVFull = 3;    // + stage: V operand tile, likewise
constexpr int bKEmpty = 6;   // + stage
constexpr int bVEmpty = 9;   // + stage
constexpr int bSFull = 12;   // + S buffer
constexpr int bPFull = 14;   // + P buffer (4 arrivals)
constexpr int bPEmpty = 16;  // + P buffer
constexpr int bODone = 18;   // one phase per tile
constexpr int bOFinal = 19;
constexpr int bDrain = 20;
constexpr int bCKFull = 21;   // + K staging stage (3): K codes loaded (E4M3)
constexpr int bCVFull = 24;   // + V staging stage (2): V codes loaded
constexpr int bCKEmpty = 26;  // + K staging stage: K codes converted (4 converter warps)
constexpr int bCVEmpty = 29;  // + V staging stage: V codes converted

// TMEM columns: S^T buffers [0,16) [16,32), O^T [32,48)
constexpr uint32_t kTcTmemCols = 64;
constexpr uint32_t kTcTmemO = 32;

// OR of a predicate over the 128 softmax threads (named barrier 1; every
// softmax thread executes it once per tile, whatever its state).
__device__ __forceinline__ bool softmax_any(bool pred) {
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t"
        "setp.ne.u32 p, %1, 0;\n\t"
        "bar.red.or.pred q, 1, 128, p;\n\t"
        "selp.u32 %0, 1, 0, q;\n\t}"
        : "=r"(r)
        : "r"(pred ? 1u : 0u)
        : "memory");
    return r != 0;
}

__device__ __forceinline__ void softmax_sync() { asm volatile("bar.sync 1, 128;" ::: "memory"); }

__device__ __forceinline__ void fence_proxy_async_global() { asm volatile("fence.proxy.async.global;" ::: "memory"); }

__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&r)[16]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr));
}

// Byte offset of element (row, col) of a 16-row, K-major, 128-byte-swizzled
// operand whose K extent is split into 64-element blocks of 2 KB (8-row swizzle
// atoms of 1 KB; the 16-byte chunk index is XORed with the row within the atom).
__device__ __forceinline__ uint32_t sw128_off16(int row, int col) {
    const int blk = col >> 6;
    const int chunk = (col & 63) >> 3;
    return static_cast<uint32_t>(blk * 2048 + (row >> 3) * 1024 + (row & 7) * 128 + ((chunk ^ (row & 7)) << 4) +
                                 (col & 7) * 2);
}

__device__ __forceinline__ void tc_abort(uint32_t* err, volatile int* abort_flag) {
    *abort_flag = 1;
    atomicOr(err, kErrDecodeCopy);
}

// f16 pair of two floats (lo in the low half), as one 32-bit word.
__device__ __forceinline__ uint32_t pack_f16x2(float lo, float hi) {
    const __half2 h = __floats2half2_rn(lo, hi);
    return *reinterpret_cast<const uint32_t*>(&h);
}

// f16 values of the two E4M3 codes of a 16-bit word (low byte -> low half).
__device__ __forceinline__ uint32_t f16x2_from_e4m3x2(uint32_t c) {
    uint32_t r;
    asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(r) : "h"(static_cast<unsigned short>(c)));
    return r;
}

template <int G, bool Fp8>
__global__ void __launch_bounds__(TcLayout<Fp8>::kThreads, 1)
    decode_tc_kernel(const __grid_constant__ DecodeParams p, const __grid_constant__ DecodeMaps maps) {
    static_assert(G <= kTcN, "query group larger than the MMA's N");
    using Lay = TcLayout<Fp8>;
    constexpr int D = kTcD;
    constexpr int kStages = Lay::kStages;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    uint8_t* const sb = smem_raw + (base - raw);
    auto bar = [&](int i) { return base + Lay::kOffBar + 8u * i; };
    volatile float* red = reinterpret_cast<volatile float*>(sb + Lay::kOffRed);
    volatile uint32_t* tmem_slot = reinterpret_cast<volatile uint32_t*>(sb + Lay::kOffMisc);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(sb + Lay::kOffMisc + 4);
    volatile int* last_flag = reinterpret_cast<volatile int*>(sb + Lay::kOffMisc + 8);

    const int tid = threadIdx.x;
    const int warp = tid >> 5;
    const int lane = tid & 31;

    // Work item.
    const int n_retr_items = p.B * p.n_retr * p.nsplit;
    const bool is_retr = static_cast<int>(blockIdx.x) < n_retr_items;
    int b, g, ri = 0, split = 0;
    if (is_retr) {
        split = blockIdx.x % p.nsplit;
        const int t_ = blockIdx.x / p.nsplit;
        ri = t_ % p.n_retr;
        b = t_ / p.n_retr;
        g = p.retr_list[ri];
    } else {
        const int si = blockIdx.x - n_retr_items;
        b = si / p.n_strm;
        g = p.strm_list[si % p.n_strm];
    }
    // E4M3 retrieval rows: converted to f16 operands, products in f16.
    const bool f16ops = Fp8 && is_retr;
    const int pool = p.heads.pool_idx[g];
    const int64_t L = p.ragged ? p.seq_len[b] : p.len;  // this sequence's new token position
    int64_t r0, r_end, new_slot;
    bool owns_new;
    if (is_retr) {
        r0 = static_cast<int64_t>(split) * p.split_rows;
        const int64_t s1 = r0 + p.split_rows;
        // Splits are cut for the longest sequence: in a ragged batch a shorter
        // sequence's last splits hold no rows (they still report to the merge).
        owns_new = r0 <= L && s1 >= L + 1;
        r_end = owns_new ? L + 1 : (s1 < L ? s1 : (L > r0 ? L : r0));
        new_slot = L;
    } else {
        r0 = 0;
        r_end = (L + 1 < p.W) ? (L + 1) : p.W;
        owns_new = true;
        new_slot = (L < p.S) ? L : p.S + (L - p.S) % p.R;
    }
    const int n_tiles = static_cast<int>((r_end - r0 + kTcKeys - 1) / kTcKeys);
    const int zrow = pool * p.B + b;  // the pool map's third coordinate
    const CUtensorMap* mk = f16ops ? &maps.rk8 : (is_retr ? &maps.rk : &maps.sk);
    const CUtensorMap* mv = f16ops ? &maps.rv8 : (is_retr ? &maps.rv : &maps.sv);
    float k_scale = 1.f, v_scale = 1.f, k_inv = 1.f, v_inv = 1.f;
    if (f16ops) {
        k_scale = p.kv_scale[g * 4 + 0];
        v_scale = p.kv_scale[g * 4 + 1];
        k_inv = p.kv_scale[g * 4 + 2];
        v_inv = p.kv_scale[g * 4 + 3];
    }

    if (tid == 0) {
        for (int s = 0; s < kStages; ++s) {
            // Operand tiles: filled by TMA (one arrival + bytes) or by the four converter warps.
            mbar_init(bar(bKFull + s), f16ops ? 4 : 1);
            mbar_init(bar(bVFull + s), f16ops ? 4 : 1);
            mbar_init(bar(bKEmpty + s), 1);
            mbar_init(bar(bVEmpty + s), 1);
        }
        for (int s = 0; s < 2; ++s) {
            mbar_init(bar(bSFull + s), 1);
            mbar_init(bar(bPFull + s), 4);
            mbar_init(bar(bPEmpty + s), 1);
        }
        for (int s = 0; s < Lay::kCodeStagesK; ++s) {
            mbar_init(bar(bCKFull + s), 1);
            mbar_init(bar(bCKEmpty + s), 4);
        }
        for (int s = 0; s < Lay::kCodeStagesV; ++s) {
            mbar_init(bar(bCVFull + s), 1);
            mbar_init(bar(bCVEmpty + s), 4);
        }
        mbar_init(bar(bODone), 1);
        mbar_init(bar(bOFinal), 1);
        mbar_init(bar(bDrain), 1);
        *abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == 5) {
        tmem_alloc(base + Lay::kOffMisc, kTcTmemCols);
        tmem_relinquish();
    }
    if (tid == 0) {
        tma_prefetch_desc(mk);
        tma_prefetch_desc(mv);
    }
    grid_dependency_wait();  // launched with programmatic stream serialization
    grid_launch_dependents();

    // The owner writes the new token into its slot first (E4M3 codes for an E4M3
    // retrieval head, as the append would store them); its tile reads it back
    // through TMA (generic-proxy stores made visible to the async proxy).
    if (owns_new && warp == 4) {
        const bf16* knew = p.k_new + (static_cast<int64_t>(b) * p.Hkv + g) * D;
        const bf16* vnew = p.v_new + (static_cast<int64_t>(b) * p.Hkv + g) * D;
        const int64_t slots = is_retr ? p.max_len : p.W;
        const int64_t off = (static_cast<int64_t>(zrow) * slots + new_slot) * D;  // elements
        if (f16ops) {
            uint8_t* dk = reinterpret_cast<uint8_t*>(p.pools.rk) + off;
            uint8_t* dv = reinterpret_cast<uint8_t*>(p.pools.rv) + off;
            if (lane < 16) {
                *reinterpret_cast<uint2*>(dk + lane * 8) = e4m3x8_from_bf16x8(ld_nc_v4(knew + lane * 8), k_inv);
            } else {
                *reinterpret_cast<uint2*>(dv + (lane - 16) * 8) =
                    e4m3x8_from_bf16x8(ld_nc_v4(vnew + (lane - 16) * 8), v_inv);
            }
        } else {
            bf16* dk = is_retr ? p.pools.rk : p.pools.sk;
            bf16* dv = is_retr ? p.pools.rv : p.pools.sv;
            if (lane < 16) {
                *reinterpret_cast<uint4*>(dk + off + lane * 8) = ld_nc_v4(knew + lane * 8);
            } else {
                *reinterpret_cast<uint4*>(dv + off + (lane - 16) * 8) = ld_nc_v4(vnew + (lane - 16) * 8);
            }
        }
        fence_proxy_async_global();
    }
    // Queries of the group as the B operand (rows G..15 zero); f16 for E4M3 items.
    for (int i = tid; i < kTcN * D / 8; i += Lay::kThreads) {
        const int row = i / (D / 8);
        const int c8 = (i % (D / 8)) * 8;
        uint4 v = make_uint4(0, 0, 0, 0);
        if (row < G) {
            v = ld_nc_v4(p.q + (static_cast<int64_t>(b) * p.Hq + g * G + row) * D + c8);
            if (f16ops) {
                v = make_uint4(pack_f16x2(bf16lo_to_f32(v.x), bf16hi_to_f32(v.x)),
                               pack_f16x2(bf16lo_to_f32(v.y), bf16hi_to_f32(v.y)),
                               pack_f16x2(bf16lo_to_f32(v.z), bf16hi_to_f32(v.z)),
                               pack_f16x2(bf16lo_to_f32(v.w), bf16hi_to_f32(v.w)));
            }
        }
        *reinterpret_cast<uint4*>(sb + Lay::kOffQ + sw128_off16(row, c8)) = v;
    }
    // P buffers: rows G..15 stay zero.
    for (int i = tid; i < 2 * kTcPBytes / 16; i += Lay::kThreads)
        reinterpret_cast<uint4*>(sb + Lay::kOffP)[i] = make_uint4(0, 0, 0, 0);
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == 4) {
        // ------------------------------------------------------------ producer
        if (f16ops && lane < 2 && n_tiles > 0) {
            // E4M3 items: lane 0 loads the K codes, lane 1 the V codes, each into its
            // own staging ring (a stage is free once the converters have read it).
            const bool is_k = lane == 0;
            const int ns = is_k ? Lay::kCodeStagesK : Lay::kCodeStagesV;
            const int cfull = is_k ? bCKFull : bCVFull;
            const int cempty = is_k ? bCKEmpty : bCVEmpty;
            const uint32_t ring = base + (is_k ? Lay::kOffCK : Lay::kOffCV);
            const CUtensorMap* m = is_k ? mk : mv;
            int issued = 0;
            for (int j = 0; j < n_tiles; ++j) {
                const int cs = j % ns;
                if (j >= ns && !mbar_wait(bar(cempty + cs), ((j / ns) - 1) & 1, abort_flag)) {
                    tc_abort(p.err, abort_flag);
                    break;
                }
                mbar_arrive_expect_tx(bar(cfull + cs), kTcCodeTile);
                tma_load_3d(ring + cs * kTcCodeTile, m, bar(cfull + cs), 0, static_cast<int>(r0) + j * kTcKeys, zrow);
                issued = j + 1;
            }
            // Let every load this thread issued land before the CTA can exit.
            for (int j = (issued > ns ? issued - ns : 0); j < issued; ++j)
                mbar_wait(bar(cfull + j % ns), (j / ns) & 1, nullptr);
        } else if (!f16ops && lane == 0 && n_tiles > 0) {
            // bf16 tiles straight into the operand rings.
            int issued = 0;
            for (int j = 0; j < n_tiles; ++j) {
                const int row0 = static_cast<int>(r0) + j * kTcKeys;
                const int st = j % kStages;
                if (j >= kStages) {
                    const uint32_t par = ((j / kStages) - 1) & 1;
                    if (!mbar_wait(bar(bKEmpty + st), par, abort_flag) ||
                        !mbar_wait(bar(bVEmpty + st), par, abort_flag)) {
                        tc_abort(p.err, abort_flag);
                        break;
                    }
                }
                mbar_arrive_expect_tx(bar(bKFull + st), kTcTile);
                mbar_arrive_expect_tx(bar(bVFull + st), kTcTile);
                for (int kb = 0; kb < D / 64; ++kb) {
                    tma_load_3d(base + Lay::kOffK + st * kTcTile + kb * kTcColBlock, mk, bar(bKFull + st), kb * 64,
                                row0, zrow);
                    tma_load_3d(base + Lay::kOffV + st * kTcTile + kb * kTcColBlock, mv, bar(bVFull + st), kb * 64,
                                row0, zrow);
                }
                issued = j + 1;
            }
            // Let every load this thread issued land before the CTA can exit.
            for (int j = (issued > kStages ? issued - kStages : 0); j < issued; ++j) {
                mbar_wait(bar(bKFull + j % kStages), (j / kStages) & 1, nullptr);
                mbar_wait(bar(bVFull + j % kStages), (j / kStages) & 1, nullptr);
            }
        }
    } else if (Fp8 && warp >= 6) {
        // ------------------------------------------------------------ converters (E4M3 items)
        // Warps 6-9 convert the K tiles, warps 10-13 the V tiles; warp c of a group
        // converts rows [32c, 32c+32): 16 codes per lane and step (four rows per
        // step), written as 16 f16 into the row's two 16-byte chunks of the
        // 128-byte-swizzled operand tile.
        if (f16ops && n_tiles > 0) {
            const int cw = (warp - 6) & 3;
            const int kv = warp >= 10 ? 1 : 0;
            const int ncs = kv ? Lay::kCodeStagesV : Lay::kCodeStagesK;
            bool ok = true;
            for (int j = 0; ok && j < n_tiles; ++j) {
                const int cs = j % ncs;  // staging stage
                const int os = j & 1;    // operand stage (2 stages for E4M3 caches)
                {
                    const int cfull = kv ? bCVFull : bCKFull;
                    const int cempty = kv ? bCVEmpty : bCKEmpty;
                    const int ofull = kv ? bVFull : bKFull;
                    const int oempty = kv ? bVEmpty : bKEmpty;
                    if (!__all_sync(0xffffffffu, mbar_wait(bar(cfull + cs), (j / ncs) & 1, abort_flag)) ||
                        (j >= 2 &&
                         !__all_sync(0xffffffffu, mbar_wait(bar(oempty + os), ((j >> 1) - 1) & 1, abort_flag)))) {
                        if (lane == 0) tc_abort(p.err, abort_flag);
                        ok = false;
                        break;
                    }
                    const uint8_t* src = sb + (kv ? Lay::kOffCV : Lay::kOffCK) + cs * kTcCodeTile;
                    uint8_t* dst = sb + (kv ? Lay::kOffV : Lay::kOffK) + os * kTcTile;
                    // Lane -> (row, 16-code group): each quarter-warp takes two adjacent rows,
                    // groups 0-3 of one and 4-7 of the other, so that its eight 16-byte code
                    // loads and its eight swizzled f16 stores each land on eight distinct
                    // 16-byte bank groups (one shared-memory wavefront per quarter).
                    const int qw = lane >> 3;
                    const int hr = (lane >> 2) & 1;
                    const int row_l = 2 * (qw & 1) + hr;
                    const int c16 = (lane & 3) + 4 * (hr ^ (qw >> 1));
#pragma unroll
                    for (int i = 0; i < 8; ++i) {
                        const int r = 32 * cw + 4 * i + row_l;
                        const uint4 c = *reinterpret_cast<const uint4*>(src + r * 128 + c16 * 16);
                        const uint4 lo = make_uint4(f16x2_from_e4m3x2(c.x & 0xFFFFu), f16x2_from_e4m3x2(c.x >> 16),
                                                    f16x2_from_e4m3x2(c.y & 0xFFFFu), f16x2_from_e4m3x2(c.y >> 16));
                        const uint4 hi = make_uint4(f16x2_from_e4m3x2(c.z & 0xFFFFu), f16x2_from_e4m3x2(c.z >> 16),
                                                    f16x2_from_e4m3x2(c.w & 0xFFFFu), f16x2_from_e4m3x2(c.w >> 16));
                        uint8_t* row = dst + (c16 >> 2) * kTcColBlock + r * 128;
                        const int ch = (c16 & 3) * 2;  // first 16-byte chunk (8 elements) within the block's row
                        *reinterpret_cast<uint4*>(row + (((ch) ^ (r & 7)) << 4)) = lo;
                        *reinterpret_cast<uint4*>(row + (((ch + 1) ^ (r & 7)) << 4)) = hi;
                    }
                    fence_proxy_async_smem();  // generic writes -> visible to the MMA (async proxy)
                    __syncwarp();
                    if (lane == 0) {
                        mbar_arrive(bar(cempty + cs));
                        mbar_arrive(bar(ofull + os));
                    }
                }
            }
        }
    } else if (warp == 5) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0 && n_tiles > 0) {
            const uint32_t idesc_qk = f16ops ? idesc_f16_f32(128, kTcN, 0, 0) : idesc_bf16_f32(128, kTcN, 0, 0);
            const uint32_t idesc_pv = f16ops ? idesc_f16_f32(128, kTcN, 1, 0) : idesc_bf16_f32(128, kTcN, 1, 0);
            // S^T(j) = K(j) Q^T into S buffer j&1.
            auto qk = [&](int j) -> bool {
                const int st = j % kStages;
                if (!mbar_wait(bar(bKFull + st), (j / kStages) & 1, abort_flag)) return false;
                tc_fence_after();
                const uint32_t kt = base + Lay::kOffK + st * kTcTile;
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint64_t a = smem_desc_sw128(kt + (kk >> 2) * kTcColBlock + (kk & 3) * 32, 16, 1024);
                    const uint64_t bq = smem_desc_sw128(base + Lay::kOffQ + (kk >> 2) * 2048 + (kk & 3) * 32, 16, 1024);
                    tc_mma_ss(tmem + (j & 1) * kTcN, a, bq, idesc_qk, kk > 0 ? 1u : 0u);
                }
                tc_commit(bar(bSFull + (j & 1)));
                tc_commit(bar(bKEmpty + st));  // the K stage is free
                return true;
            };
            bool ok = true;
            for (int j = 0; ok && j < 2 && j < n_tiles; ++j) ok = qk(j);
            for (int j = 0; ok && j < n_tiles; ++j) {
                const int st = j % kStages;
                const int pb = j & 1;
                if (!mbar_wait(bar(bVFull + st), (j / kStages) & 1, abort_flag) ||
                    !mbar_wait(bar(bPFull + pb), (j >> 1) & 1, abort_flag)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t vt = base + Lay::kOffV + st * kTcTile;
#pragma unroll
                for (int kk = 0; kk < kTcKeys / 16; ++kk) {
                    // A = V^T: the V tile read MN-major (16 keys per step, two 64-column blocks)
                    const uint64_t a = smem_desc_sw128(vt + kk * 2048, kTcColBlock, 1024);
                    const uint64_t bp =
                        smem_desc_sw128(base + Lay::kOffP + pb * kTcPBytes + (kk >> 2) * 2048 + (kk & 3) * 32, 16, 1024);
                    tc_mma_ss(tmem + kTcTmemO, a, bp, idesc_pv, (j > 0 || kk > 0) ? 1u : 0u);
                }
                tc_commit(bar(bODone));
                tc_commit(bar(bPEmpty + pb));
                tc_commit(bar(bVEmpty + st));  // the V stage is free
                if (j + 1 == n_tiles) tc_commit(bar(bOFinal));
                if (j + 2 < n_tiles) ok = qk(j + 2);
            }
            if (!ok) tc_abort(p.err, abort_flag);
            // Drain: every MMA issued above completes before TMEM is released.
            tc_commit(bar(bDrain));
            mbar_wait(bar(bDrain), 0, nullptr);
        }
    } else if (warp < 4) {
        // ------------------------------------------------------------ softmax: thread = key
        const uint32_t lane_base = static_cast<uint32_t>(warp * 32) << 16;
        const float score_scale = p.scale_log2 * k_scale;  // E4M3 items: the codes times k_scale
        float m[G], l[G];
#pragma unroll
        for (int h = 0; h < G; ++h) {
            m[h] = -INFINITY;
            l[h] = 0.f;
        }
        bool ok = true;
        for (int j = 0; j < n_tiles; ++j) {
            const int sbuf = j & 1;
            if (!(ok && __all_sync(0xffffffffu, mbar_wait(bar(bSFull + sbuf), (j >> 1) & 1, abort_flag)))) ok = false;
            float x[G];
            if (ok) {
                tc_fence_after();
                uint32_t r[16];
                tmem_ld16(tmem + lane_base + sbuf * kTcN, r);
                tc_wait_ld();
                const int64_t key = r0 + static_cast<int64_t>(j) * kTcKeys + tid;
                const bool valid = key < r_end;
#pragma unroll
                for (int h = 0; h < G; ++h) x[h] = valid ? __uint_as_float(r[h]) * score_scale : -INFINITY;
            } else {
#pragma unroll
                for (int h = 0; h < G; ++h) x[h] = -INFINITY;
            }
            // Raise the running maxima (and rescale O^T and l) only when a score
            // exceeds them by more than 2^8; every thread takes the same decision.
            bool need = false;
#pragma unroll
            for (int h = 0; h < G; ++h) need = need || (x[h] > m[h] + kTcRescale);
            if (softmax_any(need)) {
                volatile float* rr = red + (j & 1) * 4 * kTcN;
#pragma unroll
                for (int h = 0; h < G; ++h) {
                    float v = x[h];
#pragma unroll
                    for (int o = 16; o >= 1; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
                    if (lane == 0) rr[warp * kTcN + h] = v;
                }
                softmax_sync();
                float factor[G];
                bool any_factor = false;
#pragma unroll
                for (int h = 0; h < G; ++h) {
                    const float tmax = fmaxf(fmaxf(rr[h], rr[kTcN + h]), fmaxf(rr[2 * kTcN + h], rr[3 * kTcN + h]));
                    factor[h] = 1.f;
                    if (tmax > m[h]) {
                        factor[h] = (m[h] == -INFINITY) ? 0.f : fast_exp2(m[h] - tmax);
                        m[h] = tmax;
                    }
                    l[h] *= factor[h];
                    any_factor = any_factor || factor[h] != 1.f;
                }
                // O^T rows are output columns: thread t rescales column t of every head,
                // after PV(j-1) has written it (S(j) ready means PV(j-2) is complete, so
                // the barrier's phase for PV(j-1) is the only one outstanding).
                if (j >= 1 && __any_sync(0xffffffffu, any_factor)) {
                    if (__all_sync(0xffffffffu, ok && mbar_wait(bar(bODone), (j - 1) & 1, abort_flag))) {
                        tc_fence_after();
                        uint32_t r[16];
                        tmem_ld16(tmem + lane_base + kTcTmemO, r);
                        tc_wait_ld();
#pragma unroll
                        for (int h = 0; h < G; ++h) r[h] = __float_as_uint(__uint_as_float(r[h]) * factor[h]);
                        tmem_st16(tmem + lane_base + kTcTmemO, r);
                        tc_wait_st();
                    } else {
                        ok = false;
                    }
                }
            }
            // P^T(j): this thread's key column of every head (f16 for E4M3 items).
            const int pb = j & 1;
            if (j >= 2 && !__all_sync(0xffffffffu, ok && mbar_wait(bar(bPEmpty + pb), ((j >> 1) - 1) & 1, abort_flag)))
                ok = false;
            if (ok) {
                uint8_t* pbuf = sb + Lay::kOffP + pb * kTcPBytes;
#pragma unroll
                for (int h = 0; h < G; ++h) {
                    const float pv = (x[h] == -INFINITY) ? 0.f : fast_exp2(x[h] - m[h]);
                    l[h] += pv;
                    if (f16ops) *reinterpret_cast<__half*>(pbuf + sw128_off16(h, tid)) = __float2half_rn(pv);
                    else *reinterpret_cast<bf16*>(pbuf + sw128_off16(h, tid)) = __float2bfloat16_rn(pv);
                }
                fence_proxy_async_smem();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(bar(bPFull + pb));
            }
        }
        // Row sums over the CTA's keys, then this thread's output column.
        {
            volatile float* rr = red;  // reused: [4 warps][16]
            softmax_sync();
#pragma unroll
            for (int h = 0; h < G; ++h) {
                float v = l[h];
#pragma unroll
                for (int o = 16; o >= 1; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
                if (lane == 0) rr[warp * kTcN + h] = v;
            }
            softmax_sync();
#pragma unroll
            for (int h = 0; h < G; ++h) l[h] = rr[h] + rr[kTcN + h] + rr[2 * kTcN + h] + rr[3 * kTcN + h];
        }
        const int64_t item = (static_cast<int64_t>(b) * p.n_retr + ri) * p.nsplit + split;
        const bool final_now = !is_retr || p.nsplit == 1;
        if (n_tiles > 0 && __all_sync(0xffffffffu, ok && mbar_wait(bar(bOFinal), 0, abort_flag))) {
            tc_fence_after();
            uint32_t r[16];
            tmem_ld16(tmem + lane_base + kTcTmemO, r);
            tc_wait_ld();
#pragma unroll
            for (int h = 0; h < G; ++h) {
                const float o = l[h] > 0.f ? __uint_as_float(r[h]) * v_scale / l[h] : 0.f;
                if (final_now) {
                    p.out[(static_cast<int64_t>(b) * p.Hq + g * G + h) * D + tid] = __float2bfloat16_rn(o);
                } else {
                    p.part_o[(item * G + h) * D + tid] = o;
                    if (tid == 0) p.part_lse[item * G + h] = l[h] > 0.f ? m[h] + __log2f(l[h]) : -INFINITY;
                }
            }
        } else {
            // a split without rows (ragged batch), or an abort: an empty partial
            if (n_tiles > 0) tc_abort(p.err, abort_flag);
#pragma unroll
            for (int h = 0; h < G; ++h) {
                if (!final_now) {
                    p.part_o[(item * G + h) * D + tid] = 0.f;
                    if (tid == 0) p.part_lse[item * G + h] = -INFINITY;
                }
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 5) tmem_dealloc(tmem, kTcTmemCols);
    if (!is_retr || p.nsplit == 1) return;

    // Split-KV merge (D4): the last CTA of this (b, KV head) combines the
    // partials (decode_merge.cuh), in the shared memory of the operand rings.
    if (!split_arrive(&p.counters[b * p.Hkv + g], static_cast<uint32_t>(p.nsplit), last_flag)) return;
    merge_split_partials<G, kTcD, Lay::kThreads>(p, b, g, ri, sb);
    if (tid == 0) p.counters[b * p.Hkv + g] = 0u;  // ready for the next step (stream-ordered)
}

template <int G, bool Fp8>
cudaError_t launch_tc_g(const DecodeParams& p, const DecodeMaps& maps, unsigned grid, cudaStream_t s) {
    using Lay = TcLayout<Fp8>;
    static SmemLimitOnce limit;
    const cudaError_t e = limit.apply(reinterpret_cast<const void*>(&decode_tc_kernel<G, Fp8>), Lay::kSmem);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(Lay::kThreads);
    cfg.dynamicSmemBytes = Lay::kSmem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, decode_tc_kernel<G, Fp8>, p, maps);
}

}  // namespace

cudaError_t launch_decode_tc(const DecodeParams& p, const DecodeMaps& maps, cudaStream_t s) {
    const unsigned grid = static_cast<unsigned>(p.B * p.n_retr * p.nsplit + p.B * p.n_strm);
    if (grid == 0) return cudaSuccess;
    if (!decode_on_tensor_cores(p.G, p.D, p.fp8 != 0)) return cudaErrorInvalidValue;
    if (p.fp8) {
        if (p.G == 4) return launch_tc_g<4, true>(p, maps, grid, s);
        if (p.G == 8) return launch_tc_g<8, true>(p, maps, grid, s);
    } else {
        if (p.G == 4) return launch_tc_g<4, false>(p, maps, grid, s);
        if (p.G == 8) return launch_tc_g<8, false>(p, maps, grid, s);
    }
    return cudaErrorInvalidValue;
}

}  // namespace duo
