// duo_internal.cuh — kernel parameter blocks and launch entry points shared by
// the host ABI (duo_abi.cu) and the kernels (append.cu, decode.cu, prefill.cu).
#pragma once

#include <atomic>
#include <cstdint>
#include <vector>
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "../../include/duo.h"

namespace duo {

using bf16 = __nv_bfloat16;

// Launch `kernel` on stream `s` with programmatic stream serialization: its
// CTAs may start while the previous kernel of the stream drains; the kernel
// itself waits (griddepcontrol.wait) before touching dependent memory.
template <typename Kernel, typename Params>
cudaError_t launch_pdl(Kernel kernel, dim3 grid, dim3 block, size_t smem, cudaStream_t s, const Params& p) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, p);
}

// Sets a kernel's dynamic shared-memory limit once per device (the attribute
// call costs host time on every launch otherwise). One instance per kernel.
struct SmemLimitOnce {
    std::atomic<uint64_t> done{0};
    cudaError_t apply(const void* kernel, int smem) {
        int dev = 0;
        if (cudaGetDevice(&dev) != cudaSuccess) return cudaErrorInvalidDevice;
        const uint64_t bit = (dev >= 0 && dev < 64) ? (1ull << dev) : 0ull;
        if (bit != 0 && (done.load(std::memory_order_acquire) & bit) != 0) return cudaSuccess;
        const cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
        if (e == cudaSuccess && bit != 0) done.fetch_or(bit, std::memory_order_acq_rel);
        return e;
    }
};

// Per-layer KV-head map, passed by value: for every KV head its type and its
// dense index in the retrieval pool or the streaming pool (over all layers).
struct HeadMap {
    int32_t pool_idx[DUO_MAX_KV_HEADS];
    uint8_t is_retr[DUO_MAX_KV_HEADS];
};

// Where one layer's caches live.
struct Pools {
    bf16* rk;  // retrieval K pool [n_retr_all][B][max_len][D]
    bf16* rv;
    bf16* sk;  // streaming K pool [n_strm_all][B][W][D], W = sink + recent
    bf16* sv;
};

// Sequences of a batch may have different lengths (ragged batches) when the
// batch has at most this many sequences; their lengths travel in the launch.
constexpr int kMaxRaggedBatch = DUO_MAX_RAGGED_BATCH;

// ------------------------------------------------------------------ append
struct AppendParams {
    const bf16* k;  // [B][n][Hkv][D]
    const bf16* v;
    Pools pools;
    int64_t len;      // tokens cached before this call (uniform batch)
    int64_t n;        // tokens appended (uniform batch); rows per sequence of k and v
    int64_t max_len;
    int32_t B, Hkv, D, S, R, W;
    int32_t ragged;   // 1: per-sequence seq_len / seq_n below
    int32_t n_retr;   // retrieval KV heads of the layer, listed first in order[]
    int32_t fp8;            // retrieval pools hold E4M3 codes
    const float* kv_scale;  // fp8: [Hkv][k_scale, v_scale, 1/k_scale, 1/v_scale] of this layer
    HeadMap heads;
    int16_t order[DUO_MAX_KV_HEADS];   // KV heads, retrieval heads first
    int64_t seq_len[kMaxRaggedBatch];  // tokens cached before this call, per sequence
    int64_t seq_n[kMaxRaggedBatch];    // tokens appended, per sequence (<= n)
};
cudaError_t launch_append(const AppendParams& p, cudaStream_t s);

// ------------------------------------------------------------------ decode
constexpr int kDecodeMaxSplits = 256;
constexpr int kDecodeThreads = 128;

// Resident decode CTAs per SM for a query-group size (the kernel's shared memory
// and register budget are sized for it).
__host__ __device__ constexpr int decode_ctas_per_sm(int G) { return (G == 2 || G == 4) ? 3 : 2; }

// Query groups of 4 and 8 heads with head_dim 128 decode on the tensor cores
// (decode_tc.cu, one CTA per SM; E4M3 retrieval rows are converted to f16 in
// shared memory); everything else on the CUDA cores.
__host__ __device__ constexpr bool decode_on_tensor_cores(int G, int D, bool /*fp8*/) {
    return (G == 4 || G == 8) && D == 128;
}
__host__ __device__ constexpr int decode_slots_per_sm(int G, int D, bool fp8) {
    return decode_on_tensor_cores(G, D, fp8) ? 1 : decode_ctas_per_sm(G);
}

// Splits per retrieval (b, KV head) for one decode step. Every CTA streams
// its rows at about the same rate, so the step takes about
//   waves * (rows of the longest CTA + a fixed per-CTA cost),
// waves = ceil(CTAs / resident slots). The streaming items are one CTA of up to
// sink + recent rows each. Pick the split count (>= 256 rows per split, at most
// kDecodeMaxSplits) that minimises that estimate.
inline int64_t plan_decode_splits(int64_t batch, int64_t n_retr, int64_t n_strm, int64_t rows, int64_t strm_rows,
                                  int num_sms, int G, int D, bool fp8) {
    if (n_retr <= 0) return 1;
    constexpr int64_t kCtaCostRows = 64;
    const int64_t pairs = batch * n_retr;
    const int64_t strm_items = batch * n_strm;
    const int64_t slots = static_cast<int64_t>(num_sms) * decode_slots_per_sm(G, D, fp8);
    int64_t max_split = (rows + 255) / 256;
    if (max_split > kDecodeMaxSplits) max_split = kDecodeMaxSplits;
    if (max_split < 1) max_split = 1;
    int64_t best = 1, best_cost = -1;
    for (int64_t ns = 1; ns <= max_split; ++ns) {
        const int64_t ctas = pairs * ns + strm_items;
        const int64_t waves = (ctas + slots - 1) / slots;
        int64_t longest = (rows + ns - 1) / ns;
        if (strm_items > 0 && strm_rows > longest) longest = strm_rows;
        const int64_t cost = waves * (longest + kCtaCostRows);
        if (best_cost < 0 || cost < best_cost) {
            best_cost = cost;
            best = ns;
        }
    }
    return best;
}

struct DecodeParams {
    const bf16* q;      // [B][Hq][D]
    const bf16* k_new;  // [B][Hkv][D]
    const bf16* v_new;
    bf16* out;          // [B][Hq][D]
    Pools pools;
    float* part_o;       // [B*Hkv*kDecodeMaxSplits][G][D]  normalised partial outputs
    float* part_lse;     // [B*Hkv*kDecodeMaxSplits][G]     log2-sum-exp2 of the partial
    uint32_t* counters;  // [B*Hkv] splits finished, reset by the merging CTA
    uint32_t* err;
    int64_t len;        // tokens cached before this step; the new token sits at position len
                        // (uniform batch; the longest sequence when ragged)
    int64_t max_len;
    int64_t split_rows;  // rows per retrieval split
    int32_t nsplit;      // splits per retrieval (b, kv head)
    int32_t B, Hq, Hkv, G, D, S, R, W;
    int32_t n_retr, n_strm;  // retrieval / streaming KV heads in this layer
    float scale_log2;        // softmax scale * log2(e)
    int16_t retr_list[DUO_MAX_KV_HEADS];
    int16_t strm_list[DUO_MAX_KV_HEADS];
    HeadMap heads;
    int32_t ragged;                     // 1: per-sequence lengths in seq_len
    int32_t fp8;                        // retrieval pools hold E4M3 codes
    const float* kv_scale;              // fp8: [Hkv][k_scale, v_scale, 1/k_scale, 1/v_scale] of this layer
    int32_t test_withhold;              // 1: a test of the bounded waits (duo_cache_test_wait_timeout)
    uint64_t test_timeout_ns;           // the withheld copy's wait limit
    int64_t seq_len[kMaxRaggedBatch];   // tokens cached before this step, per sequence
};
// TMA maps of the cache pools, for the tensor-core decode: bf16 pools with box
// 64 x 128 rows (128-byte swizzle); for E4M3 caches also the retrieval pools as
// one-byte codes with box D x 128 rows (no swizzle).
struct DecodeMaps {
    CUtensorMap rk, rv, sk, sv;
    CUtensorMap rk8, rv8;
};
// One decode step: on the tensor cores when decode_on_tensor_cores() (and no
// test of the bounded waits is armed), else on the CUDA cores.
cudaError_t launch_decode(const DecodeParams& p, const DecodeMaps& maps, cudaStream_t s);
cudaError_t launch_decode_tc(const DecodeParams& p, const DecodeMaps& maps, cudaStream_t s);

// ------------------------------------------------------------------ prefill
constexpr int kTileQ = 128;   // query rows per CTA (one TMEM lane each)
constexpr int kTileK = 128;   // keys per KV tile

struct PrefillParams {
    bf16* out;  // [B][C][Hq][D]
    uint32_t* err;
    // Two words, zero between launches: [0] next work item, [1] CTAs done (the
    // last CTA of a launch zeroes both). The CTAs of one launch take items in
    // order from [0], so launches on one cache must be stream-ordered.
    uint32_t* work;
    int64_t len;  // tokens cached before the chunk (uniform batch)
    int32_t C;    // chunk length; rows per sequence of q, k, v and out
    int32_t B, Hq, Hkv, G, D, S, R, W;
    int32_t n_qt;      // ceil(C / kTileQ)
    int32_t n_retr_q;  // retrieval query heads (listed first in qhead)
    float scale_log2;
    int16_t qhead[DUO_MAX_Q_HEADS];
    HeadMap heads;
    int32_t ragged;                    // 1: per-sequence seq_len / seq_c below
    int32_t test_withhold;             // 1: a test of the bounded waits (duo_cache_test_wait_timeout)
    uint64_t test_timeout_ns;          // the withheld copy's wait limit
    int64_t seq_len[kMaxRaggedBatch];  // tokens cached before the chunk, per sequence
    int32_t seq_c[kMaxRaggedBatch];    // chunk rows that are tokens, per sequence (<= C)
};

struct PrefillMaps {
    CUtensorMap q;   // chunk q  (D, Hq, C, B), box (64, 1, 128, 1)
    CUtensorMap out; // prefill output, same shape and box as q (tile stores)
    CUtensorMap k;   // chunk k  (D, Hkv, C, B)
    CUtensorMap v;
    CUtensorMap rk;  // retrieval pool (D, max_len, n_retr_all*B), box (64, 128, 1)
    CUtensorMap rv;
    CUtensorMap sk;  // streaming pool (D, W, n_strm_all*B), box (64, 128, 1)
    CUtensorMap sv;
};
cudaError_t launch_prefill(const PrefillParams& p, const PrefillMaps& maps, int num_sms, cudaStream_t s);
// The streaming-head work items of a prefill launch (prefill_stream.cu); `after_retrieval`:
// launched behind the retrieval-item kernel with programmatic dependent launch.
cudaError_t launch_prefill_streaming(const PrefillParams& p, const PrefillMaps& maps, int num_sms,
                                     bool after_retrieval, cudaStream_t s);

}  // namespace duo

// Host object behind the opaque duo_cache handle.
struct duo_cache {
    duo_layout lay;
    int32_t G = 1;
    int32_t W = 0;
    float scale = 0.f;
    int device = 0;
    int num_sms = 148;
    std::vector<uint8_t> is_retr;       // [layers][Hkv]
    std::vector<int32_t> pool_idx;      // [layers][Hkv] dense index within its pool
    std::vector<int64_t> len;           // [layers][batch] tokens cached per sequence
    int64_t n_retr_all = 0, n_strm_all = 0;
    duo::Pools pools{};
    float* part_o = nullptr;
    float* part_lse = nullptr;
    uint32_t* counters = nullptr;
    uint32_t* err = nullptr;
    CUtensorMap map_rk{}, map_rv{}, map_sk{}, map_sv{};
    CUtensorMap map_rk8{}, map_rv8{};   // E4M3 caches: the retrieval pools as one-byte codes
    int32_t test_wait = 0;              // duo_cache_test_wait_timeout: launch kinds still to withhold a copy
    uint64_t test_wait_ns = 0;
    bool fp8 = false;                   // retrieval pools hold E4M3 codes
    float* kv_scales = nullptr;         // device [layers][Hkv][k_scale, v_scale, 1/k_scale, 1/v_scale]
    std::vector<float> kv_scales_host;  // host copy of kv_scales
    std::vector<duo::DecodeParams> decode_tmpl;  // [layers] decode parameters fixed at alloc
    std::vector<int64_t> plan_key;               // [layers] rows / 256 of the cached split plan
    std::vector<int64_t> plan_nsplit;            // [layers] the plan's split count
};

// The pool tensor maps of a cache, as the decode launch takes them.
inline duo::DecodeMaps decode_maps(const duo_cache* c) {
    return duo::DecodeMaps{c->map_rk, c->map_rv, c->map_sk, c->map_sv, c->map_rk8, c->map_rv8};
}

// Per-sequence lengths of one layer ([batch] host values).
inline int64_t* seq_lens(duo_cache* c, int32_t layer) {
    return c->len.data() + static_cast<size_t>(layer) * c->lay.batch;
}
inline const int64_t* seq_lens(const duo_cache* c, int32_t layer) {
    return c->len.data() + static_cast<size_t>(layer) * c->lay.batch;
}

// Longest sequence of a layer, and whether all sequences have that length.
inline int64_t longest_seq(const duo_cache* c, int32_t layer, bool* uniform) {
    const int64_t* L = seq_lens(c, layer);
    int64_t mx = L[0];
    bool uni = true;
    for (int32_t b = 1; b < c->lay.batch; ++b) {
        if (L[b] > mx) mx = L[b];
        uni = uni && (L[b] == L[0]);
    }
    if (uniform) *uniform = uni;
    return mx;
}

// Lengths of a decode step: the longest sequence in p.len and, for a ragged
// batch, every sequence's length. DUO_ERR_STATE if a ragged batch is larger
// than the launch can carry.
inline duo_status fill_decode_lengths(const duo_cache* c, int32_t layer, duo::DecodeParams& p) {
    bool uniform = true;
    p.len = longest_seq(c, layer, &uniform);
    p.ragged = uniform ? 0 : 1;
    if (uniform) return DUO_OK;
    if (c->lay.batch > duo::kMaxRaggedBatch) return DUO_ERR_STATE;
    const int64_t* L = seq_lens(c, layer);
    for (int32_t b = 0; b < c->lay.batch; ++b) p.seq_len[b] = L[b];
    return DUO_OK;
}

// Split count for a decode step over `rows` keys of `layer`. The plan is kept
// per layer and recomputed when rows / 256 changes: any split count is
// correct, the plan only balances the launch.
inline int64_t decode_plan(duo_cache* c, int32_t layer, int64_t rows) {
    const int64_t key = rows >> 8;
    if (c->plan_key[layer] != key) {
        const duo::DecodeParams& t = c->decode_tmpl[layer];
        c->plan_nsplit[layer] =
            duo::plan_decode_splits(c->lay.batch, t.n_retr, t.n_strm, rows, rows < c->W ? rows : c->W, c->num_sms,
                                    c->G, c->lay.head_dim, c->fp8);
        c->plan_key[layer] = key;
    }
    return c->plan_nsplit[layer];
}
