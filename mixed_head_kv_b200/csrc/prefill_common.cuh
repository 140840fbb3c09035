// prefill_common.cuh — constants and helpers shared by the two prefill kernels
// (prefill.cu: one retrieval work item per CTA; prefill_stream.cu: persistent
// CTAs over the streaming work items). Both use 384 threads with the same warp
// roles, 128 x 128 tiles, split-O softmax (two threads per query row) and the
// same TMEM map: S in two 128-column buffers, P written back into S, O of key
// half h at kTmemO + h * D.
#pragma once

#include "duo_internal.cuh"
#include "mask_rules.cuh"
#include "sm100.cuh"
#include "tile_plan.cuh"

namespace duo {
namespace {

constexpr int kThreads = 384;
constexpr int kTileBytesPerColBlock = kTileQ * 128;  // 128 rows x 64 bf16 (128 B)
constexpr float kRescaleThreshold = 8.0f;             // log2 units: rescale when max grows by > 2^8
constexpr int kHalf = kTileK / 2;                     // keys per softmax thread and tile

constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kTmemO = 256;  // O of key half h at kTmemO + h * D
constexpr uint32_t kTmemP = 32;   // P of a key tile at its S buffer + 32 (64 columns of bf16 pairs)

__device__ __forceinline__ void record_abort(uint32_t* err, volatile int* abort_flag) {
    *abort_flag = 1;
    atomicOr(err, kErrPrefillWait);
}

// Visibility of the 32 keys from `base` of a tile from `src` (0 retrieval
// cache, 1 streaming cache, 2 chunk) for one query row, from its row bounds
// (mask_rules.cuh).
__device__ __forceinline__ uint32_t visible_bits(const RowVis& v, int src, int32_t base) {
    if (src == 2) return chunk_bits_row(v, base);
    if (src == 1) return streaming_cache_bits_row(v, base);
    return retrieval_cache_bits_row(v, base);
}

__device__ __forceinline__ float fmax3(float a, float b, float c) {
    float r;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
    return r;
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

}  // namespace
}  // namespace duo
