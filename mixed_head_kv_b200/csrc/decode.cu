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
// Inside a CTA, 4 warps split the key range. A K/V row of D bf16 is read by
// D/8 lanes with 16-byte non-caching loads (2 rows per warp instruction at
// D = 128); each row is read once for all G query heads of its group. Scores
// are reduced with warp shuffles; online softmax (exp2 domain) runs per lane
// group and the groups/warps are merged at the end.
#include <cfloat>

#include "duo_internal.cuh"
#include "sm100.cuh"

namespace duo {

namespace {

constexpr int kUnroll = 4;  // row groups in flight per warp iteration
constexpr int kWarps = kDecodeThreads / 32;

template <int D, int G>
struct DecState {
    float m[G];
    float l[G];
    float o[G][8];
};

template <int D, int G>
__device__ __forceinline__ void init_state(DecState<D, G>& st) {
#pragma unroll
    for (int h = 0; h < G; ++h) {
        st.m[h] = -INFINITY;
        st.l[h] = 0.f;
#pragma unroll
        for (int e = 0; e < 8; ++e) st.o[h][e] = 0.f;
    }
}

// Accumulate rows [r0, r1) (except `skip`) of one head's K/V into the state.
// kbase/vbase point at row 0; row r lives at base + r * D.
template <int D, int G>
__device__ __forceinline__ void process_rows(DecState<D, G>& st, const float (&qf)[G][8], const bf16* kbase,
                                             const bf16* vbase, int64_t r0, int64_t r1, int64_t skip) {
    constexpr int LPR = D / 8;    // lanes per row
    constexpr int RPW = 32 / LPR; // rows per warp instruction
    const int lane = threadIdx.x & 31;
    const int sub = lane % LPR;
    const int rsub = lane / LPR;
    for (int64_t base = r0; base < r1; base += kUnroll * RPW) {
        uint4 kx[kUnroll], vx[kUnroll];
        bool valid[kUnroll];
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
            const int64_t row = base + u * RPW + rsub;
            valid[u] = (row < r1) && (row != skip);
            if (valid[u]) {
                kx[u] = ld_nc_v4(kbase + row * D + sub * 8);
                vx[u] = ld_nc_v4(vbase + row * D + sub * 8);
            } else {
                kx[u] = make_uint4(0, 0, 0, 0);
                vx[u] = make_uint4(0, 0, 0, 0);
            }
        }
        float s[kUnroll][G];
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
            const uint32_t w[4] = {kx[u].x, kx[u].y, kx[u].z, kx[u].w};
            float kf[8];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                kf[2 * i] = bf16lo_to_f32(w[i]);
                kf[2 * i + 1] = bf16hi_to_f32(w[i]);
            }
#pragma unroll
            for (int h = 0; h < G; ++h) {
                float acc = 0.f;
#pragma unroll
                for (int e = 0; e < 8; ++e) acc = fmaf(qf[h][e], kf[e], acc);
                s[u][h] = acc;
            }
        }
#pragma unroll
        for (int off = LPR / 2; off >= 1; off >>= 1) {
#pragma unroll
            for (int u = 0; u < kUnroll; ++u) {
#pragma unroll
                for (int h = 0; h < G; ++h) s[u][h] += __shfl_xor_sync(0xffffffffu, s[u][h], off);
            }
        }
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
            if (!valid[u]) {
#pragma unroll
                for (int h = 0; h < G; ++h) s[u][h] = -INFINITY;
            }
        }
        float vf[kUnroll][8];
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
            const uint32_t w[4] = {vx[u].x, vx[u].y, vx[u].z, vx[u].w};
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                vf[u][2 * i] = bf16lo_to_f32(w[i]);
                vf[u][2 * i + 1] = bf16hi_to_f32(w[i]);
            }
        }
#pragma unroll
        for (int h = 0; h < G; ++h) {
            float mb = s[0][h];
#pragma unroll
            for (int u = 1; u < kUnroll; ++u) mb = fmaxf(mb, s[u][h]);
            const float mn = fmaxf(st.m[h], mb);
            if (mn == -INFINITY) continue;  // nothing valid for this lane group yet
            const float f = fast_exp2(st.m[h] - mn);  // 0 when the old max is -inf
            st.m[h] = mn;
            st.l[h] *= f;
#pragma unroll
            for (int e = 0; e < 8; ++e) st.o[h][e] *= f;
#pragma unroll
            for (int u = 0; u < kUnroll; ++u) {
                const float pu = fast_exp2(s[u][h] - mn);
                st.l[h] += pu;
#pragma unroll
                for (int e = 0; e < 8; ++e) st.o[h][e] = fmaf(pu, vf[u][e], st.o[h][e]);
            }
        }
    }
}

// Merge the partial softmax state of the partner lane (xor `off`) into st.
template <int D, int G>
__device__ __forceinline__ void merge_lanes(DecState<D, G>& st, int off) {
#pragma unroll
    for (int h = 0; h < G; ++h) {
        const float m2 = __shfl_xor_sync(0xffffffffu, st.m[h], off);
        const float l2 = __shfl_xor_sync(0xffffffffu, st.l[h], off);
        const float mn = fmaxf(st.m[h], m2);
        const float ms = (mn == -INFINITY) ? 0.f : mn;
        const float f1 = fast_exp2(st.m[h] - ms);
        const float f2 = fast_exp2(m2 - ms);
        st.l[h] = st.l[h] * f1 + l2 * f2;
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            const float o2 = __shfl_xor_sync(0xffffffffu, st.o[h][e], off);
            st.o[h][e] = st.o[h][e] * f1 + o2 * f2;
        }
        st.m[h] = mn;
    }
}

template <int D, int G>
__global__ void __launch_bounds__(kDecodeThreads) decode_kernel(const DecodeParams p) {
    constexpr int LPR = D / 8;
    __shared__ float sm_m[kWarps][G];
    __shared__ float sm_l[kWarps][G];
    __shared__ float sm_o[kWarps][G][D];
    __shared__ float sm_w[G][kDecodeMaxSplits];
    __shared__ int sm_last;

    const int tid = threadIdx.x;
    const int warp = tid >> 5;
    const int lane = tid & 31;
    const int sub = lane % LPR;

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
    const int64_t L = p.len;  // new token position

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
        owns_new = s1 >= L + 1;
        r1 = owns_new ? L : s1;
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

    // Append the new token (D1): warp 1 copies it into its slot.
    if (owns_new && warp == 1) {
        if (lane < LPR) {
            *reinterpret_cast<uint4*>(new_k_dst + lane * 8) = ld_nc_v4(knew + lane * 8);
        } else if (lane < 2 * LPR) {
            *reinterpret_cast<uint4*>(new_v_dst + (lane - LPR) * 8) = ld_nc_v4(vnew + (lane - LPR) * 8);
        }
    }

    // Queries of the group, pre-scaled into the exp2 domain.
    float qf[G][8];
#pragma unroll
    for (int h = 0; h < G; ++h) {
        const uint4 qx = ld_nc_v4(p.q + (static_cast<int64_t>(b) * p.Hq + g * G + h) * D + sub * 8);
        const uint32_t w[4] = {qx.x, qx.y, qx.z, qx.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            qf[h][2 * i] = bf16lo_to_f32(w[i]) * p.scale_log2;
            qf[h][2 * i + 1] = bf16hi_to_f32(w[i]) * p.scale_log2;
        }
    }

    DecState<D, G> st;
    init_state(st);
    const int64_t n_rows = r1 - r0;
    const int64_t per_warp = (n_rows + kWarps - 1) / kWarps;
    const int64_t w0 = r0 + warp * per_warp;
    const int64_t w1 = (w0 + per_warp < r1) ? (w0 + per_warp) : r1;
    if (w0 < w1) process_rows<D, G>(st, qf, kbase, vbase, w0, w1, skip);
    if (owns_new && warp == 0) process_rows<D, G>(st, qf, knew, vnew, 0, 1, -1);

    // Merge the row groups of the warp, then the warps.
#pragma unroll
    for (int off = LPR; off < 32; off <<= 1) merge_lanes<D, G>(st, off);
    if (lane < LPR) {
#pragma unroll
        for (int h = 0; h < G; ++h) {
            if (lane == 0) {
                sm_m[warp][h] = st.m[h];
                sm_l[warp][h] = st.l[h];
            }
#pragma unroll
            for (int e = 0; e < 8; ++e) sm_o[warp][h][sub * 8 + e] = st.o[h][e];
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
        for (int w = 0; w < kWarps; ++w) M = fmaxf(M, sm_m[w][h]);
        float Lsum = 0.f, O = 0.f;
#pragma unroll
        for (int w = 0; w < kWarps; ++w) {
            const float f = fast_exp2(sm_m[w][h] - M);
            Lsum += f * sm_l[w][h];
            O += f * sm_o[w][h][d];
        }
        if (final_now) {
            p.out[(static_cast<int64_t>(b) * p.Hq + g * G + h) * D + d] = __float2bfloat16_rn(O / Lsum);
        } else {
            p.part_o[(item * G + h) * D + d] = O / Lsum;
            if (d == 0) p.part_lse[item * G + h] = M + __log2f(Lsum);
        }
    }
    if (final_now) return;

    // Split-KV merge (D4): the last CTA of this (b, KV head) combines the partials.
    __threadfence();
    __syncthreads();
    if (tid == 0) {
        const uint32_t prev = atomicAdd(&p.counters[b * p.Hkv + g], 1u);
        sm_last = (prev == static_cast<uint32_t>(p.nsplit - 1));
    }
    __syncthreads();
    if (!sm_last) return;
    __threadfence();
    const int64_t item0 = (static_cast<int64_t>(b) * p.n_retr + ri) * p.nsplit;
    for (int h = warp; h < G; h += kWarps) {
        float M = -INFINITY;
        for (int s = lane; s < p.nsplit; s += 32) M = fmaxf(M, __ldcg(p.part_lse + (item0 + s) * G + h));
#pragma unroll
        for (int off = 16; off >= 1; off >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, off));
        float sum = 0.f;
        for (int s = lane; s < p.nsplit; s += 32) {
            const float w = fast_exp2(__ldcg(p.part_lse + (item0 + s) * G + h) - M);
            sm_w[h][s] = w;
            sum += w;
        }
#pragma unroll
        for (int off = 16; off >= 1; off >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, off);
        const float inv = 1.f / sum;
        for (int s = lane; s < p.nsplit; s += 32) sm_w[h][s] *= inv;
    }
    __syncthreads();
    for (int idx = tid; idx < G * D; idx += kDecodeThreads) {
        const int h = idx / D;
        const int d = idx % D;
        float acc = 0.f;
        for (int s = 0; s < p.nsplit; ++s) acc = fmaf(sm_w[h][s], __ldcg(p.part_o + ((item0 + s) * G + h) * D + d), acc);
        p.out[(static_cast<int64_t>(b) * p.Hq + g * G + h) * D + d] = __float2bfloat16_rn(acc);
    }
    if (tid == 0) p.counters[b * p.Hkv + g] = 0u;  // ready for the next step (stream-ordered)
}

template <int D>
cudaError_t launch_d(const DecodeParams& p, unsigned grid, cudaStream_t s) {
    switch (p.G) {
        case 1: decode_kernel<D, 1><<<grid, kDecodeThreads, 0, s>>>(p); break;
        case 2: decode_kernel<D, 2><<<grid, kDecodeThreads, 0, s>>>(p); break;
        case 4: decode_kernel<D, 4><<<grid, kDecodeThreads, 0, s>>>(p); break;
        case 8: decode_kernel<D, 8><<<grid, kDecodeThreads, 0, s>>>(p); break;
        default: return cudaErrorInvalidValue;
    }
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_decode(const DecodeParams& p, cudaStream_t s) {
    const unsigned grid = static_cast<unsigned>(p.B * p.n_retr * p.nsplit + p.B * p.n_strm);
    if (grid == 0) return cudaSuccess;
    if (p.D == 128) return launch_d<128>(p, grid, s);
    if (p.D == 64) return launch_d<64>(p, grid, s);
    return cudaErrorInvalidValue;
}

}  // namespace duo
