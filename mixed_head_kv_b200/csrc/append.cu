// append.cu — per-head KV-cache append/eviction (DuoAttention abstract: a full
// cache for retrieval heads, a constant-length sink + recent cache for
// streaming heads).
//
// One CTA per (sequence b, appended token c): the token's K and V rows of all
// KV heads are contiguous in the [B][n][Hkv][D] input, so the CTA reads them
// coalesced and writes whole 16-byte pieces of each head's cache row. The slot
// rules are evaluated once per token (uniform over the CTA):
//   retrieval head: slot = position;
//   streaming head: sink slot p < sink, else ring slot sink + (p - sink) mod
//     recent, but only for the last `recent` positions of the call (earlier
//     ring positions would be overwritten within the same call, so they are
//     neither read nor written).
// The threads walk the token's active heads (retrieval heads first, then the
// streaming heads when the token is kept by them), 16 bytes of K and V per
// thread and head, with up to four heads' loads in flight before their stores.
// HBM-bound: bytes = 2 (K,V) x rows written x D x 2 B, read and written.
#include "duo_internal.cuh"
#include "sm100.cuh"

namespace duo {

namespace {

constexpr int kAppendThreads = 128;
constexpr int kAppendUnroll = 4;

// Token c of sequence b, at position pos; `end` = the sequence's length after the call.
template <int D>
__device__ __forceinline__ void append_token(const AppendParams& p, int b, int64_t c, int64_t pos, int64_t end) {
    constexpr int LPR = D / 8;  // threads per row (16 bytes each)
    constexpr int kHeadsPerPass = kAppendThreads / LPR;
    int64_t sslot = -1;  // streaming slot, or -1 when the call itself evicts this position again
    if (pos < p.S) sslot = pos;
    else if (pos >= end - p.R) sslot = p.S + (pos - p.S) % p.R;
    const int n_active = sslot >= 0 ? p.Hkv : p.n_retr;
    const int e = threadIdx.x % LPR;
    const int64_t row0 = (static_cast<int64_t>(b) * p.n + c) * p.Hkv;  // input row of head 0
    for (int i0 = threadIdx.x / LPR; i0 < n_active; i0 += kAppendUnroll * kHeadsPerPass) {
        uint4 kx[kAppendUnroll], vx[kAppendUnroll];
        bf16* dk[kAppendUnroll];
        bf16* dv[kAppendUnroll];
#pragma unroll
        for (int u = 0; u < kAppendUnroll; ++u) {
            const int i = i0 + u * kHeadsPerPass;
            dk[u] = nullptr;
            dv[u] = nullptr;
            if (i < n_active) {
                const int g = p.order[i];
                const int64_t pool = p.heads.pool_idx[g];
                if (i < p.n_retr) {
                    const int64_t off = ((pool * p.B + b) * p.max_len + pos) * D + e * 8;
                    dk[u] = p.pools.rk + off;
                    dv[u] = p.pools.rv + off;
                } else {
                    const int64_t off = ((pool * p.B + b) * p.W + sslot) * D + e * 8;
                    dk[u] = p.pools.sk + off;
                    dv[u] = p.pools.sv + off;
                }
                const int64_t src = (row0 + g) * D + e * 8;
                kx[u] = ld_nc_v4(p.k + src);
                vx[u] = ld_nc_v4(p.v + src);
            }
        }
#pragma unroll
        for (int u = 0; u < kAppendUnroll; ++u) {
            if (dk[u] != nullptr) {
                *reinterpret_cast<uint4*>(dk[u]) = kx[u];
                *reinterpret_cast<uint4*>(dv[u]) = vx[u];
            }
        }
    }
}

template <int D>
__global__ void __launch_bounds__(kAppendThreads) append_kernel(const AppendParams p) {
    grid_dependency_wait();  // launched with programmatic stream serialization
    grid_launch_dependents();
    const int64_t c = blockIdx.x;
    for (int b = blockIdx.y; b < p.B; b += gridDim.y) {
        // Sequence b appends rows [0, n_b) at its own length (ragged batches).
        const int64_t len_b = p.ragged ? p.seq_len[b] : p.len;
        const int64_t n_b = p.ragged ? p.seq_n[b] : p.n;
        if (c < n_b) append_token<D>(p, b, c, len_b + c, len_b + n_b);
    }
}

}  // namespace

cudaError_t launch_append(const AppendParams& p, cudaStream_t s) {
    if (p.B <= 0 || p.n <= 0 || p.Hkv <= 0) return cudaSuccess;
    if (p.n > 0x7FFFFFFF) return cudaErrorInvalidValue;
    const dim3 grid(static_cast<unsigned>(p.n), static_cast<unsigned>(p.B < 65535 ? p.B : 65535));
    if (p.D == 128) return launch_pdl(append_kernel<128>, grid, dim3(kAppendThreads), 0, s, p);
    if (p.D == 64) return launch_pdl(append_kernel<64>, grid, dim3(kAppendThreads), 0, s, p);
    return cudaErrorInvalidValue;
}

}  // namespace duo
