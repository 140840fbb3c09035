// append.cu — per-head KV-cache append/eviction (DuoAttention abstract: a full
// cache for retrieval heads, a constant-length sink + recent cache for
// streaming heads).
//
// One CTA per (sequence b, two consecutive appended tokens): a token's K and V
// rows of all KV heads are contiguous in the [B][n][Hkv][D] input, so the CTA
// reads them coalesced and writes whole 16-byte pieces of each head's cache
// row. The slot rules are evaluated once per token (uniform over the CTA):
//   retrieval head: slot = position;
//   streaming head: sink slot p < sink, else ring slot sink + (p - sink) mod
//     recent, but only for the last `recent` positions of the call (earlier
//     ring positions would be overwritten within the same call, so they are
//     neither read nor written).
// The threads walk the tokens' active heads (retrieval heads first, then the
// streaming heads when the token is kept by them), 16 bytes of K and V per
// thread, head and token, with the loads of both tokens and two head passes in
// flight before their stores. E4M3 retrieval caches store the codes.
// HBM-bound: bytes = 2 (K,V) x rows written x D x 2 B, read and written.
#include "duo_internal.cuh"
#include "sm100.cuh"

namespace duo {

namespace {

constexpr int kAppendThreads = 128;
constexpr int kTokensPerCta = 2;  // tokens of one sequence per CTA, their loads in flight together
constexpr int kPassUnroll = 2;    // head passes per batch of loads

// Where token (sequence b, chunk row c) goes: its position and its streaming
// slot, or -1 when the call itself evicts the position again (ring positions
// below the sequence's length after the call minus recent).
struct TokenSlot {
    int64_t pos, sslot;
    int n_active;  // heads that store it: all heads, or the retrieval heads only
    bool valid;
};

__device__ __forceinline__ TokenSlot token_slot(const AppendParams& p, int b, int64_t c) {
    TokenSlot t;
    const int64_t len_b = p.ragged ? p.seq_len[b] : p.len;
    const int64_t n_b = p.ragged ? p.seq_n[b] : p.n;
    t.valid = c < n_b;
    t.pos = len_b + c;
    t.sslot = -1;
    if (t.pos < p.S) t.sslot = t.pos;
    else if (t.pos >= len_b + n_b - p.R) t.sslot = p.S + (t.pos - p.S) % p.R;
    t.n_active = !t.valid ? 0 : (t.sslot >= 0 ? p.Hkv : p.n_retr);
    return t;
}

// Tokens c0 .. c0 + kTokensPerCta - 1 of sequence b. Thread (head slot i, column
// e) moves 16 bytes of K and of V per token: active head i of the token (the
// layer's heads in order[], retrieval heads first). Retrieval rows go to slot =
// position; in E4M3 caches they are stored as codes (8 bytes per thread).
template <int D>
__device__ __forceinline__ void append_tokens(const AppendParams& p, int b, int64_t c0) {
    constexpr int LPR = D / 8;  // threads per row (16 bytes each)
    constexpr int kHeadsPerPass = kAppendThreads / LPR;
    TokenSlot ts[kTokensPerCta];
    int n_max = 0;
#pragma unroll
    for (int t = 0; t < kTokensPerCta; ++t) {
        ts[t] = token_slot(p, b, c0 + t);
        n_max = ts[t].n_active > n_max ? ts[t].n_active : n_max;
    }
    const int e = threadIdx.x % LPR;
    for (int i0 = threadIdx.x / LPR; i0 < n_max; i0 += kPassUnroll * kHeadsPerPass) {
        uint4 kx[kPassUnroll][kTokensPerCta], vx[kPassUnroll][kTokensPerCta];
        int64_t dst[kPassUnroll][kTokensPerCta];  // element offset in its pool, -1: nothing to store
#pragma unroll
        for (int u = 0; u < kPassUnroll; ++u) {
            const int i = i0 + u * kHeadsPerPass;
            const int g = i < p.Hkv ? p.order[i] : 0;
            const int64_t pool = p.heads.pool_idx[g];
#pragma unroll
            for (int t = 0; t < kTokensPerCta; ++t) {
                dst[u][t] = -1;
                if (i < ts[t].n_active) {
                    dst[u][t] = i < p.n_retr ? ((pool * p.B + b) * p.max_len + ts[t].pos) * D + e * 8
                                             : ((pool * p.B + b) * p.W + ts[t].sslot) * D + e * 8;
                    const int64_t src = ((static_cast<int64_t>(b) * p.n + c0 + t) * p.Hkv + g) * D + e * 8;
                    kx[u][t] = ld_nc_v4(p.k + src);
                    vx[u][t] = ld_nc_v4(p.v + src);
                }
            }
        }
#pragma unroll
        for (int u = 0; u < kPassUnroll; ++u) {
            const bool retr = i0 + u * kHeadsPerPass < p.n_retr;
            const int g = i0 + u * kHeadsPerPass < p.Hkv ? p.order[i0 + u * kHeadsPerPass] : 0;
#pragma unroll
            for (int t = 0; t < kTokensPerCta; ++t) {
                if (dst[u][t] < 0) continue;
                if (retr && p.fp8) {  // E4M3 codes of x * (1 / scale), one byte per element
                    const uint2 kc = e4m3x8_from_bf16x8(kx[u][t], p.kv_scale[g * 4 + 2]);
                    const uint2 vc = e4m3x8_from_bf16x8(vx[u][t], p.kv_scale[g * 4 + 3]);
                    *reinterpret_cast<uint2*>(reinterpret_cast<uint8_t*>(p.pools.rk) + dst[u][t]) = kc;
                    *reinterpret_cast<uint2*>(reinterpret_cast<uint8_t*>(p.pools.rv) + dst[u][t]) = vc;
                } else {
                    *reinterpret_cast<uint4*>((retr ? p.pools.rk : p.pools.sk) + dst[u][t]) = kx[u][t];
                    *reinterpret_cast<uint4*>((retr ? p.pools.rv : p.pools.sv) + dst[u][t]) = vx[u][t];
                }
            }
        }
    }
}

template <int D>
__global__ void __launch_bounds__(kAppendThreads) append_kernel(const AppendParams p) {
    grid_dependency_wait();  // launched with programmatic stream serialization
    grid_launch_dependents();
    const int64_t c0 = static_cast<int64_t>(blockIdx.x) * kTokensPerCta;
    for (int b = blockIdx.y; b < p.B; b += gridDim.y) append_tokens<D>(p, b, c0);
}

}  // namespace

cudaError_t launch_append(const AppendParams& p, cudaStream_t s) {
    if (p.B <= 0 || p.n <= 0 || p.Hkv <= 0) return cudaSuccess;
    if (p.n > 0x7FFFFFFF) return cudaErrorInvalidValue;
    const dim3 grid(static_cast<unsigned>((p.n + kTokensPerCta - 1) / kTokensPerCta),
                    static_cast<unsigned>(p.B < 65535 ? p.B : 65535));
    if (p.D == 128) return launch_pdl(append_kernel<128>, grid, dim3(kAppendThreads), 0, s, p);
    if (p.D == 64) return launch_pdl(append_kernel<64>, grid, dim3(kAppendThreads), 0, s, p);
    return cudaErrorInvalidValue;
}

}  // namespace duo
