// decode.cu — one DuoAttention decoding step for one layer, in one launch.
//
// Work items (one CTA each):
//   retrieval (b, KV head, split): keys [s*split_rows, min((s+1)*split_rows, len+1))
//     of the full cache; partial (o, log2-sum-exp2) go to scratch and the last
//     CTA of the (b, KV head) merges them (atomic counter, no spinning);
//   streaming (b, KV head): every valid slot of the sink + ring cache, written
//     straight to `out`.
// The new token is appended inside the launch by the CTA whose key range ends
// at position len; that CTA reads the new row from the input, not the cache,
// so no CTA depends on another's cache write. Its ring slot held position
// len - recent, which is outside the new query's window.
//
// Memory path: each of the 4 warps streams a contiguous part of the item's
// rows through its own ring in shared memory (3 stages; 2 for query groups of
// 2 and 4, which run three CTAs per SM), filled by bulk async
// copies (cp.async.bulk, one K block and one V block of 4 KB per stage,
// completion on an mbarrier). Each K/V row is read from HBM exactly once and
// serves all G query heads of its group. A row of D bf16 is consumed by D/8
// lanes (16 bytes each, conflict-free); scores are reduced with warp shuffles;
// online softmax runs in the exp2 domain per lane group, and the groups, the
// warps and finally the splits are merged with log-sum-exp weights.
#include <cfloat>

#include "duo_internal.cuh"
#include "sm100.cuh"
#include "decode_merge.cuh"

namespace duo {

namespace {

constexpr int kWarps = kDecodeThreads / 32;
constexpr int kGroupRows = 4;  // row groups accumulated per register batch
// Rows per warp hinted into L2 before the wait for the previous kernel (32 KB of
// K and V at D = 128).
template <int D>
constexpr int64_t kPrefetchRows = 16384 / (D * 2);

// Ring depth and residency per group size: for G = 2 and 4 (issue-heavy rows)
// three CTAs of 2-stage rings per SM hide latency better than two of 3 stages;
// the same bytes are in flight either way.
template <int D, int G>
struct Geom {
    static constexpr int kStages = (G == 2 || G == 4) ? 2 : 3;
    static constexpr int LPR = D / 8;                 // lanes per row
    static constexpr int RPW = 32 / LPR;              // rows per warp instruction
    static constexpr int BLK = 4096 / (D * 2);        // rows per 4 KB block
    static constexpr int kBlockBytes = BLK * D * 2;   // one K (or V) block
    static constexpr int kStageBytes = 2 * kBlockBytes;
    static constexpr int kWarpBytes = kStages * kStageBytes;
    static constexpr int kRingBytes = kWarps * kWarpBytes;  // 96 KB (3 stages) or 64 KB
    static constexpr int kBarOff = kRingBytes;
    static constexpr int kSmem = kBarOff + kWarps * kStages * 8 + 16;
};

template <int G>
struct DecState {
    float m[G];       // running max (log2 domain), stale by up to kDecodeRescale
    float l[G];
    uint64_t o[G][4];  // output accumulators, packed fp32 pairs (elements 2i, 2i+1)
};

// The running max of a lane group is raised, and l and o rescaled, only when a
// score exceeds it by more than 2^8: exact (l and o stay relative to the same
// max), and the rescale is skipped for almost every row batch.
constexpr float kDecodeRescale = 8.0f;

template <int G>
__device__ __forceinline__ void init_state(DecState<G>& st) {
#pragma unroll
    for (int h = 0; h < G; ++h) {
        st.m[h] = -INFINITY;
        st.l[h] = 0.f;
#pragma unroll
        for (int i = 0; i < 4; ++i) st.o[h][i] = f2pack(0.f, 0.f);
    }
}

// Eight bf16 of a 16-byte slice as four packed fp32 pairs.
__device__ __forceinline__ void bf16x8_to_f2(const uint4& x, uint64_t (&r)[4]) {
    const uint32_t w[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) r[i] = f2pack(bf16lo_to_f32(w[i]), bf16hi_to_f32(w[i]));
}

// Fold U row groups (this lane's 16-byte slices of K and V rows) into the state.
// q2: this lane's 8 query elements of each head, pre-scaled into the exp2 domain.
template <int D, int G, int U>
__device__ __forceinline__ void accumulate(DecState<G>& st, const uint64_t (&q2)[G][4], const uint4 (&kx)[U],
                                           const uint4 (&vx)[U], const bool (&valid)[U]) {
    constexpr int LPR = D / 8;
    float s[U][G];
#pragma unroll
    for (int u = 0; u < U; ++u) {
        uint64_t k2[4];
        bf16x8_to_f2(kx[u], k2);
#pragma unroll
        for (int h = 0; h < G; ++h) {
            uint64_t acc = f2pack(0.f, 0.f);
#pragma unroll
            for (int i = 0; i < 4; ++i) acc = ffma2(q2[h][i], k2[i], acc);
            float lo, hi;
            f2unpack(acc, lo, hi);
            s[u][h] = lo + hi;
        }
    }
#pragma unroll
    for (int off = LPR / 2; off >= 1; off >>= 1) {
#pragma unroll
        for (int u = 0; u < U; ++u) {
#pragma unroll
            for (int h = 0; h < G; ++h) s[u][h] += __shfl_xor_sync(0xffffffffu, s[u][h], off);
        }
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
        if (!valid[u]) {
#pragma unroll
            for (int h = 0; h < G; ++h) s[u][h] = -INFINITY;
        }
    }
    uint64_t v2[U][4];
#pragma unroll
    for (int u = 0; u < U; ++u) bf16x8_to_f2(vx[u], v2[u]);
#pragma unroll
    for (int h = 0; h < G; ++h) {
        float mb = s[0][h];
#pragma unroll
        for (int u = 1; u < U; ++u) mb = fmaxf(mb, s[u][h]);
        if (mb > st.m[h] + kDecodeRescale) {  // also taken when m is -inf and mb finite
            const float f = fast_exp2(st.m[h] - mb);  // 0 when the old max is -inf
            st.m[h] = mb;
            st.l[h] *= f;
            const uint64_t f2 = f2pack(f, f);
            const uint64_t z2 = f2pack(0.f, 0.f);
#pragma unroll
            for (int i = 0; i < 4; ++i) st.o[h][i] = ffma2(st.o[h][i], f2, z2);
        }
        if (st.m[h] == -INFINITY) continue;  // nothing valid for this lane group yet
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const float pu = fast_exp2(s[u][h] - st.m[h]);
            st.l[h] += pu;
            const uint64_t p2 = f2pack(pu, pu);
#pragma unroll
            for (int i = 0; i < 4; ++i) st.o[h][i] = ffma2(p2, v2[u][i], st.o[h][i]);
        }
    }
}

// Merge the partial softmax state of the partner lane (xor `off`) into st.
template <int G>
__device__ __forceinline__ void merge_lanes(DecState<G>& st, int off) {
#pragma unroll
    for (int h = 0; h < G; ++h) {
        const float m2 = __shfl_xor_sync(0xffffffffu, st.m[h], off);
        const float l2 = __shfl_xor_sync(0xffffffffu, st.l[h], off);
        const float mn = fmaxf(st.m[h], m2);
        const float ms = (mn == -INFINITY) ? 0.f : mn;
        const float f1 = fast_exp2(st.m[h] - ms);
        const float f2 = fast_exp2(m2 - ms);
        st.l[h] = st.l[h] * f1 + l2 * f2;
        const uint64_t f1p = f2pack(f1, f1);
        const uint64_t f2p = f2pack(f2, f2);
        const uint64_t z2 = f2pack(0.f, 0.f);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const uint64_t o2 = __shfl_xor_sync(0xffffffffu, st.o[h][i], off);
            st.o[h][i] = ffma2(o2, f2p, ffma2(st.o[h][i], f1p, z2));
        }
        st.m[h] = mn;
    }
}

// Test of the bounded waits (DecodeParams::test_withhold): warp 0 of CTA 0 does
// not issue its first copy, so its wait on it gives up after timeout_ns and the
// CTA reports kErrDecodeCopy. Every other copy is issued and waited for as usual.
struct WaitTest {
    bool withhold;
    uint64_t timeout_ns;
};

// Eight E4M3 codes (8 bytes) as four packed fp32 pairs.
__device__ __forceinline__ void e4m3x8_to_f2(const uint2& c, uint64_t (&r)[4]) {
    const uint32_t w[2] = {c.x, c.y};
#pragma unroll
    for (int i = 0; i < 2; ++i) {
        float a, b, d, e;
        e4m3x2_to_f32(static_cast<uint16_t>(w[i] & 0xFFFFu), a, b);
        e4m3x2_to_f32(static_cast<uint16_t>(w[i] >> 16), d, e);
        r[2 * i] = f2pack(a, b);
        r[2 * i + 1] = f2pack(d, e);
    }
}

// accumulate() for rows held as E4M3 codes (an E4M3 retrieval cache): this
// lane's 8 codes of K and V per row group. The head's scales are applied
// outside (k_scale folded into q2, v_scale into the partial output).
template <int D, int G, int U>
__device__ __forceinline__ void accumulate8(DecState<G>& st, const uint64_t (&q2)[G][4], const uint2 (&kc)[U],
                                            const uint2 (&vc)[U], const bool (&valid)[U]) {
    constexpr int LPR = D / 8;
    float s[U][G];
#pragma unroll
    for (int u = 0; u < U; ++u) {
        uint64_t k2[4];
        e4m3x8_to_f2(kc[u], k2);
#pragma unroll
        for (int h = 0; h < G; ++h) {
            uint64_t acc = f2pack(0.f, 0.f);
#pragma unroll
            for (int i = 0; i < 4; ++i) acc = ffma2(q2[h][i], k2[i], acc);
            float lo, hi;
            f2unpack(acc, lo, hi);
            s[u][h] = lo + hi;
        }
    }
#pragma unroll
    for (int off = LPR / 2; off >= 1; off >>= 1) {
#pragma unroll
        for (int u = 0; u < U; ++u) {
#pragma unroll
            for (int h = 0; h < G; ++h) s[u][h] += __shfl_xor_sync(0xffffffffu, s[u][h], off);
        }
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
        if (!valid[u]) {
#pragma unroll
            for (int h = 0; h < G; ++h) s[u][h] = -INFINITY;
        }
    }
    uint64_t v2[U][4];
#pragma unroll
    for (int u = 0; u < U; ++u) e4m3x8_to_f2(vc[u], v2[u]);
#pragma unroll
    for (int h = 0; h < G; ++h) {
        float mb = s[0][h];
#pragma unroll
        for (int u = 1; u < U; ++u) mb = fmaxf(mb, s[u][h]);
        if (mb > st.m[h] + kDecodeRescale) {
            const float f = fast_exp2(st.m[h] - mb);
            st.m[h] = mb;
            st.l[h] *= f;
            const uint64_t f2 = f2pack(f, f);
            const uint64_t z2 = f2pack(0.f, 0.f);
#pragma unroll
            for (int i = 0; i < 4; ++i) st.o[h][i] = ffma2(st.o[h][i], f2, z2);
        }
        if (st.m[h] == -INFINITY) continue;
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const float pu = fast_exp2(s[u][h] - st.m[h]);
            st.l[h] += pu;
            const uint64_t p2 = f2pack(pu, pu);
#pragma unroll
            for (int i = 0; i < 4; ++i) st.o[h][i] = ffma2(p2, v2[u][i], st.o[h][i]);
        }
    }
}

// warp_stream() for an E4M3 retrieval cache: rows of D one-byte codes, so a
// 4 KB block holds twice the rows; a lane reads 8 codes (8 bytes) of a row.
template <int D, int G>
__device__ bool warp_stream8(DecState<G>& st, const uint64_t (&q2)[G][4], const uint8_t* kbase, const uint8_t* vbase,
                             int64_t r0, int64_t r1, uint32_t ring, uint32_t bars, const WaitTest& wt) {
    using Gm = Geom<D, G>;
    constexpr int BLK8 = Gm::kBlockBytes / D;  // rows per block of codes
    const int lane = threadIdx.x & 31;
    const int sub = lane % Gm::LPR;
    const int rsub = lane / Gm::LPR;
    const int64_t nblk = (r1 - r0 + BLK8 - 1) / BLK8;
    auto issue = [&](int64_t i) {
        if (i == 0 && wt.withhold) return;  // test of the bounded wait: this copy is never issued
        const int stg = static_cast<int>(i % Gm::kStages);
        const int64_t a = r0 + i * BLK8;
        const int64_t n = (r1 - a < BLK8) ? (r1 - a) : BLK8;
        const uint32_t bytes = static_cast<uint32_t>(n * D);
        const uint32_t bar = bars + 8u * stg;
        const uint32_t dst = ring + stg * Gm::kStageBytes;
        mbar_arrive_expect_tx(bar, 2 * bytes);
        bulk_load(dst, kbase + a * D, bytes, bar);
        bulk_load(dst + Gm::kBlockBytes, vbase + a * D, bytes, bar);
    };
    if (lane == 0) {
        for (int64_t i = 0; i < nblk && i < Gm::kStages; ++i) issue(i);
    }
    for (int64_t i = 0; i < nblk; ++i) {
        const int stg = static_cast<int>(i % Gm::kStages);
        if (!mbar_wait(bars + 8u * stg, static_cast<uint32_t>((i / Gm::kStages) & 1), nullptr,
                       i == 0 && wt.withhold ? wt.timeout_ns : kWaitTimeoutNs)) {
            for (int64_t j = i + 1; j < nblk && j < i + Gm::kStages; ++j)
                mbar_wait(bars + 8u * static_cast<uint32_t>(j % Gm::kStages),
                          static_cast<uint32_t>((j / Gm::kStages) & 1), nullptr);
            return false;
        }
        const int64_t a = r0 + i * BLK8;
        const int rows = static_cast<int>((r1 - a < BLK8) ? (r1 - a) : BLK8);
        const uint32_t kst = ring + stg * Gm::kStageBytes;
        const uint32_t vst = kst + Gm::kBlockBytes;
#pragma unroll
        for (int u0 = 0; u0 < BLK8 / Gm::RPW; u0 += kGroupRows) {
            uint2 kc[kGroupRows], vc[kGroupRows];
            bool valid[kGroupRows];
#pragma unroll
            for (int u = 0; u < kGroupRows; ++u) {
                const int row = (u0 + u) * Gm::RPW + rsub;
                valid[u] = row < rows;
                const uint32_t off = static_cast<uint32_t>(row * D + sub * 8);
                kc[u] = valid[u] ? lds64(kst + off) : make_uint2(0, 0);
                vc[u] = valid[u] ? lds64(vst + off) : make_uint2(0, 0);
            }
            accumulate8<D, G, kGroupRows>(st, q2, kc, vc, valid);
        }
        __syncwarp();
        if (lane == 0 && i + Gm::kStages < nblk) {
            fence_proxy_async_smem();
            issue(i + Gm::kStages);
        }
    }
    return true;
}

// Stream rows [r0, r1) (except `skip`) of one head through this warp's ring.
// Returns false if a copy did not complete within the wait limit.
template <int D, int G>
__device__ bool warp_stream(DecState<G>& st, const uint64_t (&q2)[G][4], const bf16* kbase, const bf16* vbase,
                            int64_t r0, int64_t r1, int64_t skip, uint32_t ring, uint32_t bars, const WaitTest& wt) {
    using Gm = Geom<D, G>;
    const int lane = threadIdx.x & 31;
    const int sub = lane % Gm::LPR;
    const int rsub = lane / Gm::LPR;
    const int64_t nblk = (r1 - r0 + Gm::BLK - 1) / Gm::BLK;
    auto issue = [&](int64_t i) {
        if (i == 0 && wt.withhold) return;  // test of the bounded wait: this copy is never issued
        const int stg = static_cast<int>(i % Gm::kStages);
        const int64_t a = r0 + i * Gm::BLK;
        const int64_t n = (r1 - a < Gm::BLK) ? (r1 - a) : Gm::BLK;
        const uint32_t bytes = static_cast<uint32_t>(n * D * 2);
        const uint32_t bar = bars + 8u * stg;
        const uint32_t dst = ring + stg * Gm::kStageBytes;
        mbar_arrive_expect_tx(bar, 2 * bytes);
        bulk_load(dst, kbase + a * D, bytes, bar);
        bulk_load(dst + Gm::kBlockBytes, vbase + a * D, bytes, bar);
    };
    if (lane == 0) {
        for (int64_t i = 0; i < nblk && i < Gm::kStages; ++i) issue(i);
    }
    for (int64_t i = 0; i < nblk; ++i) {
        const int stg = static_cast<int>(i % Gm::kStages);
        if (!mbar_wait(bars + 8u * stg, static_cast<uint32_t>((i / Gm::kStages) & 1), nullptr,
                       i == 0 && wt.withhold ? wt.timeout_ns : kWaitTimeoutNs)) {
            // Give the copies still in flight one more bounded wait before the
            // CTA moves on (and later reuses this shared memory).
            for (int64_t j = i + 1; j < nblk && j < i + Gm::kStages; ++j)
                mbar_wait(bars + 8u * static_cast<uint32_t>(j % Gm::kStages), static_cast<uint32_t>((j / Gm::kStages) & 1),
                          nullptr);
            return false;
        }
        const int64_t a = r0 + i * Gm::BLK;
        const int rows = static_cast<int>((r1 - a < Gm::BLK) ? (r1 - a) : Gm::BLK);
        const uint32_t kst = ring + stg * Gm::kStageBytes;
        const uint32_t vst = kst + Gm::kBlockBytes;
#pragma unroll
        for (int u0 = 0; u0 < Gm::BLK / Gm::RPW; u0 += kGroupRows) {
            uint4 kx[kGroupRows], vx[kGroupRows];
            bool valid[kGroupRows];
#pragma unroll
            for (int u = 0; u < kGroupRows; ++u) {
                const int row = (u0 + u) * Gm::RPW + rsub;
                valid[u] = row < rows && (a + row) != skip;
                const uint32_t off = static_cast<uint32_t>(row * D * 2 + sub * 16);
                kx[u] = valid[u] ? lds128(kst + off) : make_uint4(0, 0, 0, 0);
                vx[u] = valid[u] ? lds128(vst + off) : make_uint4(0, 0, 0, 0);
            }
            accumulate<D, G, kGroupRows>(st, q2, kx, vx, valid);
        }
        __syncwarp();
        if (lane == 0 && i + Gm::kStages < nblk) {
            fence_proxy_async_smem();  // our generic reads of this stage precede the async refill
            issue(i + Gm::kStages);
        }
    }
    return true;
}

// Fp8: the retrieval pools hold E4M3 codes (one instantiation per format, so
// the bf16 kernel carries no code of the other path).
template <int D, int G, bool Fp8>
__device__ __forceinline__ void decode_body(const DecodeParams& p) {
    using Gm = Geom<D, G>;
    constexpr int LPR = Gm::LPR;
    extern __shared__ __align__(128) uint8_t smem[];
    // After the streaming phase the ring is reused for the cross-warp merge.
    float* sm_m = reinterpret_cast<float*>(smem);                 // [kWarps][G]
    float* sm_l = sm_m + kWarps * G;                              // [kWarps][G]
    float* sm_o = sm_l + kWarps * G;                              // [kWarps][G][D]
    int* sm_last = reinterpret_cast<int*>(smem + Gm::kBarOff + kWarps * Gm::kStages * 8);

    const int tid = threadIdx.x;
    const int warp = tid >> 5;
    const int lane = tid & 31;
    const int sub = lane % LPR;
    const uint32_t ring = smem_u32(smem) + warp * Gm::kWarpBytes;
    const uint32_t bars = smem_u32(smem) + Gm::kBarOff + warp * Gm::kStages * 8;
    if (lane == 0) {
        for (int s = 0; s < Gm::kStages; ++s) mbar_init(bars + 8u * s, 1);
        fence_barrier_init();
    }
    __syncwarp();

    const int n_retr_items = p.B * p.n_retr * p.nsplit;
    const bool is_retr = static_cast<int>(blockIdx.x) < n_retr_items;
    int b, g, ri = 0, split = 0;
    if (is_retr) {
        split = blockIdx.x % p.nsplit;
        const int t = blockIdx.x / p.nsplit;
        ri = t % p.n_retr;
        b = t / p.n_retr;
        g = p.retr_list[ri];
    } else {
        const int si = blockIdx.x - n_retr_items;
        b = si / p.n_strm;
        g = p.strm_list[si % p.n_strm];
    }
    const int pool = p.heads.pool_idx[g];
    const int64_t L = p.ragged ? p.seq_len[b] : p.len;  // this sequence's new token position

    // Rows of this item held in the cache, and whether it owns the new token.
    const bf16* kbase;
    const bf16* vbase;
    bf16* new_k_dst;
    bf16* new_v_dst;
    int64_t r0, r1, skip = -1;
    bool owns_new;
    if (is_retr) {
        const int64_t head_off = (static_cast<int64_t>(pool) * p.B + b) * p.max_len * D;
        kbase = p.pools.rk + head_off;
        vbase = p.pools.rv + head_off;
        r0 = split * p.split_rows;
        const int64_t s1 = r0 + p.split_rows;
        // Splits are cut for the longest sequence: in a ragged batch a shorter
        // sequence's last splits hold no rows (they still report to the merge).
        owns_new = r0 <= L && s1 >= L + 1;
        r1 = owns_new ? L : (s1 < L ? s1 : (L > r0 ? L : r0));
        new_k_dst = p.pools.rk + head_off + L * D;
        new_v_dst = p.pools.rv + head_off + L * D;
    } else {
        const int64_t head_off = (static_cast<int64_t>(pool) * p.B + b) * p.W * D;
        kbase = p.pools.sk + head_off;
        vbase = p.pools.sv + head_off;
        r0 = 0;
        r1 = (L + 1 < p.W) ? (L + 1) : p.W;
        skip = (L < p.S) ? L : p.S + (L - p.S) % p.R;
        owns_new = true;
        new_k_dst = p.pools.sk + head_off + skip * D;
        new_v_dst = p.pools.sv + head_off + skip * D;
    }
    const bf16* knew = p.k_new + (static_cast<int64_t>(b) * p.Hkv + g) * D;
    const bf16* vnew = p.v_new + (static_cast<int64_t>(b) * p.Hkv + g) * D;

    // This warp's rows (contiguous, whole 4 KB blocks except at the end).
    const int64_t n_rows = r1 - r0;
    const int64_t per_warp = ((n_rows + kWarps - 1) / kWarps + Gm::BLK - 1) / Gm::BLK * Gm::BLK;
    const int64_t w0 = r0 + warp * per_warp;
    const int64_t w1 = (w0 + per_warp < r1) ? (w0 + per_warp) : r1;

    // Launched with programmatic stream serialization: the CTA may start while
    // the previous kernel of the stream drains. Before waiting for it, only hint
    // the first rows of this warp into L2 (a prefetch reads no data into the CTA,
    // and L2 stays coherent with the previous kernel's writes). Everything the
    // kernel reads or writes comes after the wait.
    if (lane == 0 && w0 < w1) {
        const int64_t pre = (w1 - w0 < kPrefetchRows<D>) ? (w1 - w0) : kPrefetchRows<D>;
        if (Fp8 && is_retr) {  // rows of one-byte codes
            const uint32_t bytes = static_cast<uint32_t>(pre * D);
            bulk_prefetch_l2(reinterpret_cast<const uint8_t*>(p.pools.rk) + (kbase - p.pools.rk) + w0 * D, bytes);
            bulk_prefetch_l2(reinterpret_cast<const uint8_t*>(p.pools.rv) + (vbase - p.pools.rv) + w0 * D, bytes);
        } else {
            const uint32_t bytes = static_cast<uint32_t>(pre * D * 2);
            bulk_prefetch_l2(kbase + w0 * D, bytes);
            bulk_prefetch_l2(vbase + w0 * D, bytes);
        }
    }
    grid_dependency_wait();
    grid_launch_dependents();

    // E4M3 retrieval cache: this head's scales; k_scale is folded into the
    // queries, v_scale into the partial output.
    const bool fp8 = Fp8 && is_retr;
    const float k_scale = fp8 ? p.kv_scale[g * 4 + 0] : 1.f;
    const float v_scale = fp8 ? p.kv_scale[g * 4 + 1] : 1.f;
    const float k_inv = fp8 ? p.kv_scale[g * 4 + 2] : 1.f;
    const float v_inv = fp8 ? p.kv_scale[g * 4 + 3] : 1.f;
    // Codes of this lane's 8 elements of the new K (or V) row.
    auto quantize8 = [&](const bf16* src, float inv) -> uint2 { return e4m3x8_from_bf16x8(ld_nc_v4(src), inv); };

    // Append the new token (D1): warp 1 copies (or quantizes) it into its slot.
    if (owns_new && warp == 1) {
        if (fp8) {
            uint8_t* k8 = reinterpret_cast<uint8_t*>(p.pools.rk) + (new_k_dst - p.pools.rk);
            uint8_t* v8 = reinterpret_cast<uint8_t*>(p.pools.rv) + (new_v_dst - p.pools.rv);
            if (lane < LPR) {
                *reinterpret_cast<uint2*>(k8 + lane * 8) = quantize8(knew + lane * 8, k_inv);
            } else if (lane < 2 * LPR) {
                *reinterpret_cast<uint2*>(v8 + (lane - LPR) * 8) = quantize8(vnew + (lane - LPR) * 8, v_inv);
            }
        } else if (lane < LPR) {
            *reinterpret_cast<uint4*>(new_k_dst + lane * 8) = ld_nc_v4(knew + lane * 8);
        } else if (lane < 2 * LPR) {
            *reinterpret_cast<uint4*>(new_v_dst + (lane - LPR) * 8) = ld_nc_v4(vnew + (lane - LPR) * 8);
        }
    }

    // Queries of the group, pre-scaled into the exp2 domain.
    uint64_t q2[G][4];
#pragma unroll
    for (int h = 0; h < G; ++h) {
        const uint4 qx = ld_nc_v4(p.q + (static_cast<int64_t>(b) * p.Hq + g * G + h) * D + sub * 8);
        const uint32_t w[4] = {qx.x, qx.y, qx.z, qx.w};
#pragma unroll
        for (int i = 0; i < 4; ++i)
            q2[h][i] = f2pack(bf16lo_to_f32(w[i]) * p.scale_log2 * k_scale, bf16hi_to_f32(w[i]) * p.scale_log2 * k_scale);
    }

    DecState<G> st;
    init_state(st);
    bool ok = true;
    const WaitTest wt{p.test_withhold != 0 && blockIdx.x == 0 && warp == 0, p.test_timeout_ns};
    if (w0 < w1) {
        if (fp8) {
            const uint8_t* k8 = reinterpret_cast<const uint8_t*>(p.pools.rk) + (kbase - p.pools.rk);
            const uint8_t* v8 = reinterpret_cast<const uint8_t*>(p.pools.rv) + (vbase - p.pools.rv);
            ok = warp_stream8<D, G>(st, q2, k8, v8, w0, w1, ring, bars, wt);
        } else {
            ok = warp_stream<D, G>(st, q2, kbase, vbase, w0, w1, skip, ring, bars, wt);
        }
    }
    if (!ok && lane == 0) atomicOr(p.err, kErrDecodeCopy);
    if (owns_new && warp == 0) {
        bool valid[1] = {lane < LPR};
        if (fp8) {  // the stored codes, as every later step reads them
            uint2 kc[1] = {quantize8(knew + sub * 8, k_inv)};
            uint2 vc[1] = {quantize8(vnew + sub * 8, v_inv)};
            accumulate8<D, G, 1>(st, q2, kc, vc, valid);
        } else {
            uint4 kx[1] = {ld_nc_v4(knew + sub * 8)};
            uint4 vx[1] = {ld_nc_v4(vnew + sub * 8)};
            accumulate<D, G, 1>(st, q2, kx, vx, valid);
        }
    }

    // Merge the row groups of the warp, then the warps.
#pragma unroll
    for (int off = LPR; off < 32; off <<= 1) merge_lanes<G>(st, off);
    __syncthreads();  // every warp is done with its ring: reuse it for the merge
    if (lane < LPR) {
#pragma unroll
        for (int h = 0; h < G; ++h) {
            if (lane == 0) {
                sm_m[warp * G + h] = st.m[h];
                sm_l[warp * G + h] = st.l[h];
            }
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                float lo, hi;
                f2unpack(st.o[h][i], lo, hi);
                sm_o[(warp * G + h) * D + sub * 8 + 2 * i] = lo;
                sm_o[(warp * G + h) * D + sub * 8 + 2 * i + 1] = hi;
            }
        }
    }
    __syncthreads();

    const int64_t item = (static_cast<int64_t>(b) * p.n_retr + ri) * p.nsplit + split;
    const bool final_now = !is_retr || p.nsplit == 1;
    for (int idx = tid; idx < G * D; idx += kDecodeThreads) {
        const int h = idx / D;
        const int d = idx % D;
        float M = -INFINITY;
#pragma unroll
        for (int w = 0; w < kWarps; ++w) M = fmaxf(M, sm_m[w * G + h]);
        const float Ms = (M == -INFINITY) ? 0.f : M;  // -inf: a split without rows
        float Lsum = 0.f, O = 0.f;
#pragma unroll
        for (int w = 0; w < kWarps; ++w) {
            const float f = fast_exp2(sm_m[w * G + h] - Ms);
            Lsum += f * sm_l[w * G + h];
            O += f * sm_o[(w * G + h) * D + d];
        }
        if (final_now) {
            p.out[(static_cast<int64_t>(b) * p.Hq + g * G + h) * D + d] = __float2bfloat16_rn(O * v_scale / Lsum);
        } else {
            p.part_o[(item * G + h) * D + d] = Lsum > 0.f ? O * v_scale / Lsum : 0.f;
            if (d == 0) p.part_lse[item * G + h] = Lsum > 0.f ? M + __log2f(Lsum) : -INFINITY;
        }
    }
    if (final_now) return;

    // Split-KV merge (D4): the last CTA of this (b, KV head) combines the partials
    // (the handshake's barriers also end every read of the per-warp arrays above).
    if (!split_arrive(&p.counters[b * p.Hkv + g], static_cast<uint32_t>(p.nsplit), sm_last)) return;
    merge_split_partials<G, D, kDecodeThreads>(p, b, g, ri, smem);
    if (tid == 0) p.counters[b * p.Hkv + g] = 0u;  // ready for the next step (stream-ordered)
}

// The kernel, with the register budget its residency needs: three CTAs per SM
// for G = 2 and 4, the compiler's own choice otherwise.
template <int D, int G, bool Fp8>
__global__ void __launch_bounds__(kDecodeThreads) decode_kernel(const DecodeParams p) {
    decode_body<D, G, Fp8>(p);
}
template <int D, int G, bool Fp8>
__global__ void __launch_bounds__(kDecodeThreads, 3) decode_kernel_3(const DecodeParams p) {
    decode_body<D, G, Fp8>(p);
}

template <int D, int G, bool Fp8>
cudaError_t launch_dg(const DecodeParams& p, unsigned grid, cudaStream_t s) {
    constexpr int smem = Geom<D, G>::kSmem;
    static_assert((kWarps * 2 * G + kWarps * G * D) * 4 <= Geom<D, G>::kRingBytes, "warp merge arrays fit in the ring");
    static_assert(16 * (G * D / 4 >= kDecodeThreads ? G * D / 4 : kDecodeThreads) + 4 * (kDecodeMaxSplits + 2) * G <=
                      Geom<D, G>::kRingBytes,
                  "split merge arrays fit in the ring");
    static SmemLimitOnce limit;
    static_assert(decode_ctas_per_sm(G) == 2 || decode_ctas_per_sm(G) == 3, "one of the two kernels");
    if constexpr (decode_ctas_per_sm(G) == 3) {
        const cudaError_t e = limit.apply(reinterpret_cast<const void*>(&decode_kernel_3<D, G, Fp8>), smem);
        if (e != cudaSuccess) return e;
        return launch_pdl(decode_kernel_3<D, G, Fp8>, dim3(grid), dim3(kDecodeThreads), smem, s, p);
    } else {
        const cudaError_t e = limit.apply(reinterpret_cast<const void*>(&decode_kernel<D, G, Fp8>), smem);
        if (e != cudaSuccess) return e;
        return launch_pdl(decode_kernel<D, G, Fp8>, dim3(grid), dim3(kDecodeThreads), smem, s, p);
    }
}

template <int D, bool Fp8>
cudaError_t launch_df(const DecodeParams& p, unsigned grid, cudaStream_t s) {
    switch (p.G) {
        case 1: return launch_dg<D, 1, Fp8>(p, grid, s);
        case 2: return launch_dg<D, 2, Fp8>(p, grid, s);
        case 4: return launch_dg<D, 4, Fp8>(p, grid, s);
        case 8: return launch_dg<D, 8, Fp8>(p, grid, s);
        default: return cudaErrorInvalidValue;
    }
}

template <int D>
cudaError_t launch_d(const DecodeParams& p, unsigned grid, cudaStream_t s) {
    return p.fp8 ? launch_df<D, true>(p, grid, s) : launch_df<D, false>(p, grid, s);
}

}  // namespace

cudaError_t launch_decode(const DecodeParams& p, const DecodeMaps& maps, cudaStream_t s) {
    const unsigned grid = static_cast<unsigned>(p.B * p.n_retr * p.nsplit + p.B * p.n_strm);
    if (grid == 0) return cudaSuccess;
    if (decode_on_tensor_cores(p.G, p.D, p.fp8 != 0) && p.test_withhold == 0) return launch_decode_tc(p, maps, s);
    if (p.D == 128) return launch_d<128>(p, grid, s);
    if (p.D == 64) return launch_d<64>(p, grid, s);
    return cudaErrorInvalidValue;
}

}  // namespace duo
