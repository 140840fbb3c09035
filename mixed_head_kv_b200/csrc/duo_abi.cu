// duo_abi.cu — the C ABI of libduo (include/duo.h): argument checks, the head
// maps, carving of the caller's device buffer, TMA tensor maps, split-KV
// planning and kernel launches. No device memory is allocated here.
#include <cmath>
#include <cstring>
#include <mutex>
#include <new>

#include "duo_internal.cuh"

using namespace duo;

namespace {

constexpr size_t kAlign = 256;

size_t align_up(size_t x) { return (x + kAlign - 1) / kAlign * kAlign; }

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Byte sizes of the regions of the cache buffer, in carving order.
struct Regions {
    size_t retr_pool, strm_pool, part_o, part_lse, counters, err, scales, total;
};

// Split-KV partials are written by retrieval (b, KV head, split) items only, indexed
// by the head's rank among the layer's retrieval heads: the scratch holds
// batch x (most retrieval heads of any layer) x kDecodeMaxSplits partials.
Regions regions_for(const duo_layout& L, int64_t n_retr_all, int64_t n_strm_all, int64_t max_retr_layer) {
    Regions r{};
    const size_t D = static_cast<size_t>(L.head_dim);
    const size_t W = static_cast<size_t>(L.sink) + static_cast<size_t>(L.recent);
    const size_t G = static_cast<size_t>(L.num_q_heads / L.num_kv_heads);
    const size_t retr_elem = L.kv_format == DUO_KV_E4M3 ? 1 : 2;  // E4M3 codes or bf16
    r.retr_pool =
        align_up(static_cast<size_t>(n_retr_all) * L.batch * static_cast<size_t>(L.max_len) * D * retr_elem);
    r.strm_pool = align_up(static_cast<size_t>(n_strm_all) * L.batch * W * D * 2);
    const size_t items = static_cast<size_t>(L.batch) * static_cast<size_t>(max_retr_layer) * kDecodeMaxSplits;
    r.part_o = align_up(items * G * D * sizeof(float));
    r.part_lse = align_up(items * G * sizeof(float));
    r.counters = align_up(static_cast<size_t>(L.batch) * L.num_kv_heads * sizeof(uint32_t));
    r.err = align_up(3 * sizeof(uint32_t));  // error word, prefill work counter and done counter
    // E4M3 caches: k_scale, v_scale and their reciprocals per (layer, KV head)
    r.scales = L.kv_format == DUO_KV_E4M3
                   ? align_up(static_cast<size_t>(L.num_layers) * L.num_kv_heads * 4 * sizeof(float))
                   : 0;
    r.total = 2 * r.retr_pool + 2 * r.strm_pool + r.part_o + r.part_lse + r.counters + r.err + r.scales;
    return r;
}

duo_status check_layout(const duo_layout* L, const uint8_t* mask) {
    if (!L || !mask) return DUO_ERR_INVALID_ARG;
    if (L->num_layers < 1 || L->batch < 1) return DUO_ERR_INVALID_ARG;
    if (L->num_kv_heads < 1 || L->num_kv_heads > DUO_MAX_KV_HEADS) return DUO_ERR_INVALID_ARG;
    if (L->num_q_heads < 1 || L->num_q_heads > DUO_MAX_Q_HEADS) return DUO_ERR_INVALID_ARG;
    if (L->num_q_heads % L->num_kv_heads != 0) return DUO_ERR_INVALID_ARG;
    const int G = L->num_q_heads / L->num_kv_heads;
    if (G != 1 && G != 2 && G != 4 && G != 8) return DUO_ERR_INVALID_ARG;
    if (L->head_dim != 64 && L->head_dim != 128) return DUO_ERR_INVALID_ARG;
    if (L->sink < 0 || L->recent < 1) return DUO_ERR_INVALID_ARG;
    if (static_cast<int64_t>(L->sink) + L->recent > (1 << 30)) return DUO_ERR_INVALID_ARG;
    if (L->max_len < 1 || L->max_len > (int64_t{1} << 31) - 1) return DUO_ERR_INVALID_ARG;
    if (!(L->softmax_scale >= 0.f) || !std::isfinite(L->softmax_scale)) return DUO_ERR_INVALID_ARG;
    if (L->kv_format != DUO_KV_BF16 && L->kv_format != DUO_KV_E4M3) return DUO_ERR_INVALID_ARG;
    const int64_t n = static_cast<int64_t>(L->num_layers) * L->num_kv_heads;
    for (int64_t i = 0; i < n; ++i)
        if (mask[i] > 1) return DUO_ERR_INVALID_ARG;
    return DUO_OK;
}

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    });
    return fn;
}

// bf16 tensor map with a 64-element (128-byte) innermost box and 128-byte swizzle.
// dims/box are innermost first; strides are the byte strides of dims 1..rank-1.
bool make_map(CUtensorMap* m, const void* base, int rank, const uint64_t* dims, const uint64_t* strides,
              const uint32_t* box) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    cuuint64_t d[5], s[4];
    cuuint32_t b[5], e[5];
    for (int i = 0; i < rank; ++i) {
        d[i] = dims[i];
        b[i] = box[i];
        e[i] = 1;
    }
    for (int i = 0; i < rank - 1; ++i) s[i] = strides[i];
    CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, static_cast<cuuint32_t>(rank), const_cast<void*>(base), d, s,
                    b, e, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// One-byte-code pool map for E4M3 retrieval caches: (D, slots, heads*B) uint8,
// box (D, 128, 1), no swizzle (the decode converts the codes itself).
bool make_code_pool_map(CUtensorMap* m, const void* base, int64_t D, int64_t slots, int64_t zdim) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    const cuuint64_t d[3] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(slots),
                             static_cast<cuuint64_t>(zdim < 1 ? 1 : zdim)};
    const cuuint64_t st[2] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(D * slots)};
    const cuuint32_t b[3] = {static_cast<cuuint32_t>(D), static_cast<cuuint32_t>(kTileK), 1};
    const cuuint32_t e[3] = {1, 1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(base), d, st, b, e, CU_TENSOR_MAP_INTERLEAVE_NONE,
              CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Pool map: (D, slots, heads*B), box (64, 128, 1).
bool make_pool_map(CUtensorMap* m, const void* base, int64_t D, int64_t slots, int64_t zdim) {
    const uint64_t dims[3] = {static_cast<uint64_t>(D), static_cast<uint64_t>(slots),
                              static_cast<uint64_t>(zdim < 1 ? 1 : zdim)};
    const uint64_t strides[2] = {static_cast<uint64_t>(D * 2), static_cast<uint64_t>(D * 2 * slots)};
    const uint32_t box[3] = {64, static_cast<uint32_t>(kTileK), 1};
    return make_map(m, base, 3, dims, strides, box);
}

// Chunk map over [B][C][H][D]: (D, H, C, B), box (64, 1, 128, 1).
bool make_chunk_map(CUtensorMap* m, const void* base, int64_t D, int64_t H, int64_t C, int64_t B) {
    const uint64_t dims[4] = {static_cast<uint64_t>(D), static_cast<uint64_t>(H), static_cast<uint64_t>(C),
                              static_cast<uint64_t>(B)};
    const uint64_t strides[3] = {static_cast<uint64_t>(D * 2), static_cast<uint64_t>(H * D * 2),
                                 static_cast<uint64_t>(C * H * D * 2)};
    const uint32_t box[4] = {64, 1, static_cast<uint32_t>(kTileQ), 1};
    return make_map(m, base, 4, dims, strides, box);
}

duo_status check_call(const duo_cache* c, int32_t layer) {
    if (!c) return DUO_ERR_INVALID_ARG;
    if (layer < 0 || layer >= c->lay.num_layers) return DUO_ERR_INVALID_ARG;
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess) return DUO_ERR_CUDA;
    if (dev != c->device) return DUO_ERR_STATE;
    return DUO_OK;
}

void fill_heads(const duo_cache* c, int32_t layer, HeadMap* h) {
    std::memset(h, 0, sizeof(*h));
    const int Hkv = c->lay.num_kv_heads;
    for (int g = 0; g < Hkv; ++g) {
        h->is_retr[g] = c->is_retr[static_cast<size_t>(layer) * Hkv + g];
        h->pool_idx[g] = c->pool_idx[static_cast<size_t>(layer) * Hkv + g];
    }
}

}  // namespace

extern "C" {

const char* duo_status_str(duo_status s) {
    switch (s) {
        case DUO_OK: return "ok";
        case DUO_ERR_INVALID_ARG: return "invalid argument";
        case DUO_ERR_CAPACITY: return "retrieval cache capacity (max_len) exceeded";
        case DUO_ERR_ALIGNMENT: return "pointer not 16-byte aligned";
        case DUO_ERR_CUDA: return "CUDA call or kernel launch failed";
        case DUO_ERR_STATE: return "call not valid in the current state (device mismatch)";
        case DUO_ERR_DEVICE: return "a kernel reported a device-side error";
        case DUO_ERR_SCRATCH_LIMIT: return "request exceeds the static decode scratch (DUO_STATIC_SCRATCH_BYTES)";
    }
    return "unknown status";
}

duo_status duo_cache_alloc(const duo_layout* layout, const uint8_t* is_retrieval, void* dev_buf, size_t buf_bytes,
                           size_t* required_bytes, void* stream, duo_cache** out) {
    duo_status st = check_layout(layout, is_retrieval);
    if (st != DUO_OK) return st;
    const duo_layout& L = *layout;
    const int64_t n = static_cast<int64_t>(L.num_layers) * L.num_kv_heads;
    int64_t n_retr = 0, max_retr_layer = 0;
    for (int32_t l = 0; l < L.num_layers; ++l) {
        int64_t nl = 0;
        for (int32_t g = 0; g < L.num_kv_heads; ++g) nl += is_retrieval[static_cast<int64_t>(l) * L.num_kv_heads + g];
        n_retr += nl;
        if (nl > max_retr_layer) max_retr_layer = nl;
    }
    const Regions reg = regions_for(L, n_retr, n - n_retr, max_retr_layer);
    if (required_bytes) *required_bytes = reg.total;
    if (!dev_buf) return DUO_OK;
    if (!out) return DUO_ERR_INVALID_ARG;
    if (buf_bytes < reg.total) return DUO_ERR_INVALID_ARG;
    if ((reinterpret_cast<uintptr_t>(dev_buf) & (kAlign - 1)) != 0) return DUO_ERR_ALIGNMENT;

    duo_cache* c = new (std::nothrow) duo_cache();
    if (!c) return DUO_ERR_INVALID_ARG;
    c->lay = L;
    c->G = L.num_q_heads / L.num_kv_heads;
    c->W = L.sink + L.recent;
    c->scale = L.softmax_scale > 0.f ? L.softmax_scale : 1.0f / std::sqrt(static_cast<float>(L.head_dim));
    c->is_retr.assign(is_retrieval, is_retrieval + n);
    c->pool_idx.resize(n);
    int32_t nr = 0, ns = 0;
    for (int64_t i = 0; i < n; ++i) c->pool_idx[i] = is_retrieval[i] ? nr++ : ns++;
    c->n_retr_all = nr;
    c->n_strm_all = ns;
    c->len.assign(static_cast<size_t>(L.num_layers) * L.batch, 0);
    if (cudaGetDevice(&c->device) != cudaSuccess ||
        cudaDeviceGetAttribute(&c->num_sms, cudaDevAttrMultiProcessorCount, c->device) != cudaSuccess) {
        delete c;
        return DUO_ERR_CUDA;
    }
    uint8_t* p = static_cast<uint8_t*>(dev_buf);
    c->pools.rk = reinterpret_cast<bf16*>(p); p += reg.retr_pool;
    c->pools.rv = reinterpret_cast<bf16*>(p); p += reg.retr_pool;
    c->pools.sk = reinterpret_cast<bf16*>(p); p += reg.strm_pool;
    c->pools.sv = reinterpret_cast<bf16*>(p); p += reg.strm_pool;
    c->part_o = reinterpret_cast<float*>(p); p += reg.part_o;
    c->part_lse = reinterpret_cast<float*>(p); p += reg.part_lse;
    c->counters = reinterpret_cast<uint32_t*>(p); p += reg.counters;
    c->err = reinterpret_cast<uint32_t*>(p); p += reg.err;
    c->fp8 = L.kv_format == DUO_KV_E4M3;
    c->kv_scales = c->fp8 ? reinterpret_cast<float*>(p) : nullptr;

    // Pool tensor maps (bf16 tiles for the prefill kernel). An empty pool gets a
    // map over the other pool, never read; so does an E4M3 retrieval pool, whose
    // cache tiles prefill never reads (it refuses such chunks). A cache with no
    // bf16 pool at all (every head an E4M3 retrieval head) needs no map.
    const int64_t D = L.head_dim;
    const bool bf16_retr = nr > 0 && !c->fp8;
    const bool any_bf16 = bf16_retr || ns > 0;
    const void* rk = bf16_retr ? static_cast<const void*>(c->pools.rk) : c->pools.sk;
    const void* rv = bf16_retr ? static_cast<const void*>(c->pools.rv) : c->pools.sv;
    const void* sk = ns ? static_cast<const void*>(c->pools.sk) : c->pools.rk;
    const void* sv = ns ? static_cast<const void*>(c->pools.sv) : c->pools.rv;
    const int64_t rslots = bf16_retr ? L.max_len : c->W;
    const int64_t sslots = ns ? c->W : L.max_len;
    const int64_t rz = static_cast<int64_t>(bf16_retr ? nr : ns) * L.batch;
    const int64_t sz = static_cast<int64_t>(ns ? ns : nr) * L.batch;
    if (any_bf16 &&
        (!make_pool_map(&c->map_rk, rk, D, rslots, rz) || !make_pool_map(&c->map_rv, rv, D, rslots, rz) ||
         !make_pool_map(&c->map_sk, sk, D, sslots, sz) || !make_pool_map(&c->map_sv, sv, D, sslots, sz))) {
        delete c;
        return DUO_ERR_CUDA;
    }
    if (c->fp8 && nr > 0 &&
        (!make_code_pool_map(&c->map_rk8, c->pools.rk, D, L.max_len, static_cast<int64_t>(nr) * L.batch) ||
         !make_code_pool_map(&c->map_rv8, c->pools.rv, D, L.max_len, static_cast<int64_t>(nr) * L.batch))) {
        delete c;
        return DUO_ERR_CUDA;
    }
    if (cudaMemsetAsync(dev_buf, 0, reg.total, static_cast<cudaStream_t>(stream)) != cudaSuccess) {
        delete c;
        return DUO_ERR_CUDA;
    }
    if (c->fp8) {  // scale 1 for every head until duo_cache_set_kv_scales
        c->kv_scales_host.assign(static_cast<size_t>(L.num_layers) * L.num_kv_heads * 4, 1.0f);
        if (cudaMemcpyAsync(c->kv_scales, c->kv_scales_host.data(), c->kv_scales_host.size() * sizeof(float),
                            cudaMemcpyHostToDevice, static_cast<cudaStream_t>(stream)) != cudaSuccess) {
            delete c;
            return DUO_ERR_CUDA;
        }
    }
    // Decode parameters that do not change between steps, per layer.
    c->decode_tmpl.assign(L.num_layers, DecodeParams{});
    for (int32_t layer = 0; layer < L.num_layers; ++layer) {
        DecodeParams& t = c->decode_tmpl[layer];
        t.pools = c->pools;
        t.part_o = c->part_o;
        t.part_lse = c->part_lse;
        t.counters = c->counters;
        t.err = c->err;
        t.max_len = L.max_len;
        t.B = L.batch;
        t.Hq = L.num_q_heads;
        t.Hkv = L.num_kv_heads;
        t.G = c->G;
        t.D = L.head_dim;
        t.S = L.sink;
        t.R = L.recent;
        t.W = c->W;
        t.scale_log2 = c->scale * 1.4426950408889634f;
        t.fp8 = c->fp8 ? 1 : 0;
        t.kv_scale = c->fp8 ? c->kv_scales + static_cast<size_t>(layer) * L.num_kv_heads * 4 : nullptr;
        fill_heads(c, layer, &t.heads);
        for (int g = 0; g < L.num_kv_heads; ++g) {
            if (t.heads.is_retr[g]) t.retr_list[t.n_retr++] = static_cast<int16_t>(g);
            else t.strm_list[t.n_strm++] = static_cast<int16_t>(g);
        }
    }
    c->plan_key.assign(L.num_layers, -1);
    c->plan_nsplit.assign(L.num_layers, 1);
    *out = c;
    return DUO_OK;
}

duo_status duo_cache_free(duo_cache* cache) {
    delete cache;
    return DUO_OK;
}

duo_status duo_cache_len(const duo_cache* c, int32_t layer, int64_t* len) {
    if (!c || !len || layer < 0 || layer >= c->lay.num_layers) return DUO_ERR_INVALID_ARG;
    bool uniform = true;
    const int64_t mx = longest_seq(c, layer, &uniform);
    if (!uniform) return DUO_ERR_STATE;
    *len = mx;
    return DUO_OK;
}

duo_status duo_cache_set_len(duo_cache* c, int32_t layer, int64_t len) {
    if (!c || layer < 0 || layer >= c->lay.num_layers) return DUO_ERR_INVALID_ARG;
    if (len < 0 || len > c->lay.max_len) return DUO_ERR_INVALID_ARG;
    int64_t* L = seq_lens(c, layer);
    for (int32_t b = 0; b < c->lay.batch; ++b) L[b] = len;
    return DUO_OK;
}

duo_status duo_cache_set_kv_scales(duo_cache* c, int32_t layer, const float* k_scale, const float* v_scale,
                                   void* stream) {
    if (!c || !k_scale || !v_scale || layer < 0 || layer >= c->lay.num_layers) return DUO_ERR_INVALID_ARG;
    if (!c->fp8) return DUO_ERR_STATE;
    const int32_t H = c->lay.num_kv_heads;
    for (int32_t g = 0; g < H; ++g)
        if (!(k_scale[g] > 0.f) || !(v_scale[g] > 0.f) || !std::isfinite(k_scale[g]) || !std::isfinite(v_scale[g]))
            return DUO_ERR_INVALID_ARG;
    float* h = c->kv_scales_host.data() + static_cast<size_t>(layer) * H * 4;
    for (int32_t g = 0; g < H; ++g) {
        h[g * 4 + 0] = k_scale[g];
        h[g * 4 + 1] = v_scale[g];
        h[g * 4 + 2] = 1.0f / k_scale[g];  // fp32 reciprocals: the quantizer multiplies by them
        h[g * 4 + 3] = 1.0f / v_scale[g];
    }
    if (cudaMemcpyAsync(c->kv_scales + static_cast<size_t>(layer) * H * 4, h, static_cast<size_t>(H) * 4 * sizeof(float),
                        cudaMemcpyHostToDevice, static_cast<cudaStream_t>(stream)) != cudaSuccess)
        return DUO_ERR_CUDA;
    return DUO_OK;
}

duo_status duo_cache_test_wait_timeout(duo_cache* c, int32_t launches, uint64_t timeout_ns) {
    if (!c || (launches & ~(DUO_TEST_WAIT_DECODE | DUO_TEST_WAIT_PREFILL)) != 0) return DUO_ERR_INVALID_ARG;
    if (timeout_ns < 1000 || timeout_ns > 1000000000ull) return DUO_ERR_INVALID_ARG;
    c->test_wait = launches;
    c->test_wait_ns = timeout_ns;
    return DUO_OK;
}

duo_status duo_cache_seq_lens(const duo_cache* c, int32_t layer, int64_t* lens) {
    if (!c || !lens || layer < 0 || layer >= c->lay.num_layers) return DUO_ERR_INVALID_ARG;
    const int64_t* L = seq_lens(c, layer);
    for (int32_t b = 0; b < c->lay.batch; ++b) lens[b] = L[b];
    return DUO_OK;
}

duo_status duo_cache_set_seq_lens(duo_cache* c, int32_t layer, const int64_t* lens) {
    if (!c || !lens || layer < 0 || layer >= c->lay.num_layers) return DUO_ERR_INVALID_ARG;
    for (int32_t b = 0; b < c->lay.batch; ++b)
        if (lens[b] < 0 || lens[b] > c->lay.max_len) return DUO_ERR_INVALID_ARG;
    int64_t* L = seq_lens(c, layer);
    for (int32_t b = 0; b < c->lay.batch; ++b) L[b] = lens[b];
    return DUO_OK;
}

duo_status duo_cache_views(const duo_cache* c, int32_t layer, int32_t kv_head, void** k, void** v, int64_t* slots,
                           int32_t* is_retrieval) {
    if (!c || layer < 0 || layer >= c->lay.num_layers || kv_head < 0 || kv_head >= c->lay.num_kv_heads)
        return DUO_ERR_INVALID_ARG;
    const size_t i = static_cast<size_t>(layer) * c->lay.num_kv_heads + kv_head;
    const int64_t D = c->lay.head_dim;
    const bool r = c->is_retr[i] != 0;
    const int64_t nslots = r ? c->lay.max_len : c->W;
    const int64_t off = static_cast<int64_t>(c->pool_idx[i]) * c->lay.batch * nslots * D;  // elements
    if (r && c->fp8) {  // one byte per element
        if (k) *k = reinterpret_cast<uint8_t*>(c->pools.rk) + off;
        if (v) *v = reinterpret_cast<uint8_t*>(c->pools.rv) + off;
    } else {
        if (k) *k = (r ? c->pools.rk : c->pools.sk) + off;
        if (v) *v = (r ? c->pools.rv : c->pools.sv) + off;
    }
    if (slots) *slots = nslots;
    if (is_retrieval) *is_retrieval = r ? 1 : 0;
    return DUO_OK;
}

duo_status duo_cache_error(duo_cache* c, void* stream, uint32_t* flags) {
    if (!c || !flags) return DUO_ERR_INVALID_ARG;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    uint32_t v = 0;
    if (cudaMemcpyAsync(&v, c->err, sizeof(v), cudaMemcpyDeviceToHost, s) != cudaSuccess) return DUO_ERR_CUDA;
    if (cudaStreamSynchronize(s) != cudaSuccess) return DUO_ERR_CUDA;
    if (v != 0 && cudaMemsetAsync(c->err, 0, sizeof(uint32_t), s) != cudaSuccess) return DUO_ERR_CUDA;
    *flags = v;
    return DUO_OK;
}

namespace {

// Append rows [0, n_tok[b]) of sequence b (k, v: [batch][max_tok][Hkv][D]).
duo_status append_impl(duo_cache* c, int32_t layer, const void* k, const void* v, const int64_t* n_tok,
                       int64_t max_tok, void* stream) {
    duo_status st = check_call(c, layer);
    if (st != DUO_OK) return st;
    if (max_tok < 0) return DUO_ERR_INVALID_ARG;
    const int32_t B = c->lay.batch;
    int64_t* L = seq_lens(c, layer);
    bool uniform = true, any = false;
    for (int32_t b = 0; b < B; ++b) {
        if (n_tok[b] < 0 || n_tok[b] > max_tok) return DUO_ERR_INVALID_ARG;
        if (L[b] + n_tok[b] > c->lay.max_len) return DUO_ERR_CAPACITY;
        uniform = uniform && L[b] == L[0] && n_tok[b] == n_tok[0];
        any = any || n_tok[b] > 0;
    }
    if (!any) return DUO_OK;
    if (!k || !v) return DUO_ERR_INVALID_ARG;
    if (!aligned16(k) || !aligned16(v)) return DUO_ERR_ALIGNMENT;
    uniform = uniform && max_tok == n_tok[0];  // else the launch carries the row stride and counts
    if (!uniform && B > kMaxRaggedBatch) return DUO_ERR_STATE;
    AppendParams p{};
    p.k = static_cast<const bf16*>(k);
    p.v = static_cast<const bf16*>(v);
    p.pools = c->pools;
    p.len = L[0];
    p.n = max_tok;
    p.max_len = c->lay.max_len;
    p.B = B;
    p.Hkv = c->lay.num_kv_heads;
    p.D = c->lay.head_dim;
    p.S = c->lay.sink;
    p.R = c->lay.recent;
    p.W = c->W;
    p.fp8 = c->fp8 ? 1 : 0;
    p.kv_scale = c->fp8 ? c->kv_scales + static_cast<size_t>(layer) * c->lay.num_kv_heads * 4 : nullptr;
    p.ragged = uniform ? 0 : 1;
    if (!uniform) {
        for (int32_t b = 0; b < B; ++b) {
            p.seq_len[b] = L[b];
            p.seq_n[b] = n_tok[b];
        }
    }
    fill_heads(c, layer, &p.heads);
    for (int pass = 0; pass < 2; ++pass) {
        int n = pass == 0 ? 0 : p.n_retr;
        for (int g = 0; g < p.Hkv; ++g)
            if ((p.heads.is_retr[g] != 0) == (pass == 0)) p.order[n++] = static_cast<int16_t>(g);
        if (pass == 0) p.n_retr = n;
    }
    if (launch_append(p, static_cast<cudaStream_t>(stream)) != cudaSuccess) return DUO_ERR_CUDA;
    for (int32_t b = 0; b < B; ++b) L[b] += n_tok[b];
    return DUO_OK;
}

}  // namespace

duo_status duo_cache_append(duo_cache* c, int32_t layer, const void* k, const void* v, int64_t n_tok, void* stream) {
    if (!c || layer < 0 || layer >= c->lay.num_layers) return DUO_ERR_INVALID_ARG;
    if (n_tok < 0) return DUO_ERR_INVALID_ARG;
    std::vector<int64_t> n(static_cast<size_t>(c->lay.batch), n_tok);
    return append_impl(c, layer, k, v, n.data(), n_tok, stream);
}

duo_status duo_cache_append_ragged(duo_cache* c, int32_t layer, const void* k, const void* v, const int64_t* n_tok,
                                   int64_t max_tok, void* stream) {
    if (!c || !n_tok || layer < 0 || layer >= c->lay.num_layers) return DUO_ERR_INVALID_ARG;
    return append_impl(c, layer, k, v, n_tok, max_tok, stream);
}

namespace {

// Prefill of sequence b's chunk rows [0, n_tok[b]) at its own length (q, k, v,
// out: [batch][max_tok][H][D]).
duo_status prefill_impl(duo_cache* c, int32_t layer, const void* q, const void* k, const void* v, void* out,
                        const int64_t* n_tok, int64_t max_tok, void* stream) {
    duo_status st = check_call(c, layer);
    if (st != DUO_OK) return st;
    if (max_tok < 0 || max_tok > (int64_t{1} << 30)) return DUO_ERR_INVALID_ARG;
    const int32_t B = c->lay.batch;
    const int64_t* lens = seq_lens(c, layer);
    bool uniform = true, any = false;
    for (int32_t b = 0; b < B; ++b) {
        if (n_tok[b] < 0 || n_tok[b] > max_tok) return DUO_ERR_INVALID_ARG;
        if (lens[b] + n_tok[b] > c->lay.max_len) return DUO_ERR_CAPACITY;
        uniform = uniform && lens[b] == lens[0] && n_tok[b] == max_tok;
        any = any || n_tok[b] > 0;
    }
    if (!any) return DUO_OK;
    if (!q || !k || !v || !out) return DUO_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out)) return DUO_ERR_ALIGNMENT;
    if (!uniform && B > kMaxRaggedBatch) return DUO_ERR_STATE;
    if (c->fp8) {  // the tensor-core prefill reads bf16 cache tiles only
        bool has_retr = false;
        for (int32_t g = 0; g < c->lay.num_kv_heads; ++g)
            has_retr = has_retr || c->is_retr[static_cast<size_t>(layer) * c->lay.num_kv_heads + g];
        for (int32_t b = 0; b < B && has_retr; ++b)
            if (lens[b] > 0) return DUO_ERR_STATE;
    }
    const int64_t n_rows = max_tok;  // rows per sequence of the padded tensors
    const int64_t len0 = lens[0];
    const duo_layout& L = c->lay;
    PrefillParams p{};
    p.out = static_cast<bf16*>(out);
    p.err = c->err;
    p.work = c->err + 1;  // the error word's 256-byte region: words 1 and 2
    p.len = len0;
    p.C = static_cast<int32_t>(n_rows);
    p.ragged = uniform ? 0 : 1;
    if (!uniform) {
        for (int32_t b = 0; b < B; ++b) {
            p.seq_len[b] = lens[b];
            p.seq_c[b] = static_cast<int32_t>(n_tok[b]);
        }
    }
    p.B = L.batch;
    p.Hq = L.num_q_heads;
    p.Hkv = L.num_kv_heads;
    p.G = c->G;
    p.D = L.head_dim;
    p.S = L.sink;
    p.R = L.recent;
    p.W = c->W;
    p.n_qt = static_cast<int32_t>((n_rows + kTileQ - 1) / kTileQ);
    p.scale_log2 = c->scale * 1.4426950408889634f;
    fill_heads(c, layer, &p.heads);
    int nq = 0;
    for (int pass = 0; pass < 2; ++pass) {
        for (int h = 0; h < L.num_q_heads; ++h) {
            const bool r = p.heads.is_retr[h / c->G] != 0;
            if (r == (pass == 0)) p.qhead[nq++] = static_cast<int16_t>(h);
        }
        if (pass == 0) p.n_retr_q = nq;
    }
    if (static_cast<int64_t>(L.batch) * L.num_q_heads * p.n_qt > 0x7FFFFFFF) return DUO_ERR_INVALID_ARG;
    PrefillMaps maps;
    maps.rk = c->map_rk;
    maps.rv = c->map_rv;
    maps.sk = c->map_sk;
    maps.sv = c->map_sv;
    if (!make_chunk_map(&maps.q, q, L.head_dim, L.num_q_heads, n_rows, L.batch) ||
        !make_chunk_map(&maps.out, out, L.head_dim, L.num_q_heads, n_rows, L.batch) ||
        !make_chunk_map(&maps.k, k, L.head_dim, L.num_kv_heads, n_rows, L.batch) ||
        !make_chunk_map(&maps.v, v, L.head_dim, L.num_kv_heads, n_rows, L.batch))
        return DUO_ERR_CUDA;
    if (c->test_wait & DUO_TEST_WAIT_PREFILL) {  // one launch only
        p.test_withhold = 1;
        p.test_timeout_ns = c->test_wait_ns;
        c->test_wait &= ~DUO_TEST_WAIT_PREFILL;
    }
    if (launch_prefill(p, maps, c->num_sms, static_cast<cudaStream_t>(stream)) != cudaSuccess) return DUO_ERR_CUDA;
    return DUO_OK;
}

}  // namespace

duo_status duo_prefill(duo_cache* c, int32_t layer, const void* q, const void* k, const void* v, void* out,
                       int64_t n_tok, void* stream) {
    if (!c || layer < 0 || layer >= c->lay.num_layers) return DUO_ERR_INVALID_ARG;
    if (n_tok < 0) return DUO_ERR_INVALID_ARG;
    std::vector<int64_t> n(static_cast<size_t>(c->lay.batch), n_tok);
    return prefill_impl(c, layer, q, k, v, out, n.data(), n_tok, stream);
}

duo_status duo_prefill_ragged(duo_cache* c, int32_t layer, const void* q, const void* k, const void* v, void* out,
                              const int64_t* n_tok, int64_t max_tok, void* stream) {
    if (!c || !n_tok || layer < 0 || layer >= c->lay.num_layers) return DUO_ERR_INVALID_ARG;
    return prefill_impl(c, layer, q, k, v, out, n_tok, max_tok, stream);
}

duo_status duo_decode(duo_cache* c, int32_t layer, const void* q, const void* k_new, const void* v_new, void* out,
                      void* stream) {
    duo_status st = check_call(c, layer);
    if (st != DUO_OK) return st;
    if (!q || !k_new || !v_new || !out) return DUO_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k_new) || !aligned16(v_new) || !aligned16(out)) return DUO_ERR_ALIGNMENT;
    DecodeParams p = c->decode_tmpl[layer];
    st = fill_decode_lengths(c, layer, p);
    if (st != DUO_OK) return st;
    if (p.len + 1 > c->lay.max_len) return DUO_ERR_CAPACITY;
    p.q = static_cast<const bf16*>(q);
    p.k_new = static_cast<const bf16*>(k_new);
    p.v_new = static_cast<const bf16*>(v_new);
    p.out = static_cast<bf16*>(out);
    if (c->test_wait & DUO_TEST_WAIT_DECODE) {  // one launch only
        p.test_withhold = 1;
        p.test_timeout_ns = c->test_wait_ns;
        c->test_wait &= ~DUO_TEST_WAIT_DECODE;
    }
    const int64_t rows = p.len + 1;
    const int64_t nsplit = decode_plan(c, layer, rows);
    p.split_rows = (rows + nsplit - 1) / nsplit;
    p.nsplit = static_cast<int32_t>((rows + p.split_rows - 1) / p.split_rows);
    if (launch_decode(p, decode_maps(c), static_cast<cudaStream_t>(stream)) != cudaSuccess) return DUO_ERR_CUDA;
    int64_t* L = seq_lens(c, layer);
    for (int32_t b = 0; b < c->lay.batch; ++b) L[b] += 1;
    return DUO_OK;
}

}  // extern "C"
