// append.cu — per-head KV-cache append/eviction (DuoAttention abstract: a full
// cache for retrieval heads, a constant-length sink + recent cache for
// streaming heads).
//
// One thread moves 16 bytes (8 bf16) of one K row and the same 16 bytes of the
// V row. Reads walk the [B][n][Hkv][D] input in order (fully coalesced);
// writes land in whole 16-byte pieces of 256-byte head rows. Streaming heads
// skip the non-sink positions that a later position of the same call would
// overwrite, so every destination slot is written at most once per call.
// HBM-bound: bytes = 2 (K,V) x rows written x D x 2 B, read and written.
#include "duo_internal.cuh"
#include "sm100.cuh"

namespace duo {

__global__ void __launch_bounds__(256) append_kernel(const AppendParams p) {
    grid_dependency_wait();  // launched with programmatic stream serialization
    grid_launch_dependents();
    const int vec_per_row = p.D / 8;
    const int64_t total = static_cast<int64_t>(p.B) * p.n * p.Hkv * vec_per_row;
    for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < total;
         i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        const int e = static_cast<int>(i % vec_per_row);
        int64_t r = i / vec_per_row;
        const int g = static_cast<int>(r % p.Hkv);
        r /= p.Hkv;
        const int64_t c = r % p.n;
        const int b = static_cast<int>(r / p.n);
        // Sequence b appends rows [0, n_b) at its own length (ragged batches).
        const int64_t len_b = p.ragged ? p.seq_len[b] : p.len;
        const int64_t n_b = p.ragged ? p.seq_n[b] : p.n;
        if (c >= n_b) continue;
        const int64_t pos = len_b + c;
        const int64_t first_kept = len_b + n_b - p.R;  // ring positions below this are overwritten in-call
        const int pool = p.heads.pool_idx[g];
        bf16* dk;
        bf16* dv;
        int64_t off;
        if (p.heads.is_retr[g]) {
            off = ((static_cast<int64_t>(pool) * p.B + b) * p.max_len + pos) * p.D + e * 8;
            dk = p.pools.rk;
            dv = p.pools.rv;
        } else {
            int64_t slot;
            if (pos < p.S) {
                slot = pos;
            } else if (pos >= first_kept) {
                slot = p.S + (pos - p.S) % p.R;
            } else {
                continue;
            }
            off = ((static_cast<int64_t>(pool) * p.B + b) * p.W + slot) * p.D + e * 8;
            dk = p.pools.sk;
            dv = p.pools.sv;
        }
        const int64_t src = i * 8;  // input is [B][n][Hkv][D]: thread i owns elements [8i, 8i+8)
        const uint4 kx = ld_nc_v4(p.k + src);
        const uint4 vx = ld_nc_v4(p.v + src);
        *reinterpret_cast<uint4*>(dk + off) = kx;
        *reinterpret_cast<uint4*>(dv + off) = vx;
    }
}

cudaError_t launch_append(const AppendParams& p, cudaStream_t s) {
    const int64_t total = static_cast<int64_t>(p.B) * p.n * p.Hkv * (p.D / 8);
    if (total == 0) return cudaSuccess;
    const int sms = p.num_sms > 0 ? p.num_sms : 148;
    const int threads = 256;
    int64_t blocks = (total + threads - 1) / threads;
    const int64_t cap = static_cast<int64_t>(sms) * 8;  // grid-stride beyond 8 resident CTAs per SM
    if (blocks > cap) blocks = cap;
    return launch_pdl(append_kernel, dim3(static_cast<unsigned>(blocks)), dim3(threads), 0, s, p);
}

}  // namespace duo
