// decode_static.cu — duo_decode_static_scratch: the decode step of duo_decode,
// for callers that cannot allocate device memory when they call in.
//
// duo_decode keeps its split-KV partial results in the scratch region of the
// caller's cache buffer. This entry point keeps them in a file-scope device
// array instead, so that a caller whose memory is fixed up front (an engine
// plugin that gets a preplanned arena, a service that must not let cudaMalloc
// or cudaFree synchronize the device in its serving loop, a process whose
// device-memory budget is owned by another allocator) can run a decode step
// without any allocation: neither this library nor the caller allocates.
//
// Rules of the shared array:
//  - its size is DUO_STATIC_SCRATCH_BYTES; every GPU that loads libduo keeps
//    that much device memory until the process exits;
//  - every call on a device uses the same array and it keeps the previous
//    call's contents: the split counters are cleared on the call's stream
//    before the launch; the partial results are always written before read;
//  - calls whose kernels overlap on the GPU (other streams, other host
//    threads) race on the array: order them on one stream;
//  - the first call on a device looks up the array's device address with
//    cudaGetSymbolAddress (with that device current); make that first call
//    before any stream capture. The address is kept per device and context:
//    after a device reset, the first call in the new context looks it up again
//    (that call, too, belongs before any stream capture).
#include <cstring>
#include <mutex>

#include "duo_internal.cuh"

using namespace duo;

namespace {

constexpr size_t kStaticBytes = DUO_STATIC_SCRATCH_BYTES;
static_assert(kStaticBytes % 256 == 0, "scratch size must be a multiple of 256 bytes");

// Host code may not use this name as a device address; see scratch_address().
static __device__ __align__(256) unsigned char g_decode_scratch[kStaticBytes];

constexpr int kMaxDevices = 64;
std::mutex g_scratch_mu;
void* g_scratch_addr[kMaxDevices] = {};
CUcontext g_scratch_ctx[kMaxDevices] = {};

size_t round256(size_t x) { return (x + 255) / 256 * 256; }

using CtxGetCurrentFn = CUresult (*)(CUcontext*);

// The driver's cuCtxGetCurrent, found through the runtime (the library links no driver stub).
CtxGetCurrentFn ctx_get_current_fn() {
    static CtxGetCurrentFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<CtxGetCurrentFn>(p);
    });
    return fn;
}

// Device address of g_decode_scratch in the current context of device `dev`,
// looked up once per (device, context): after a device reset the runtime makes
// a new primary context in which the array is loaded again and may move, so a
// changed context handle triggers a new lookup.
cudaError_t scratch_address(int dev, void** out) {
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    CtxGetCurrentFn get_ctx = ctx_get_current_fn();
    if (get_ctx == nullptr) return cudaErrorNotSupported;
    std::lock_guard<std::mutex> lock(g_scratch_mu);
    CUcontext ctx = nullptr;
    if (get_ctx(&ctx) != CUDA_SUCCESS) return cudaErrorInvalidDevice;
    if (g_scratch_addr[dev] == nullptr || ctx == nullptr || g_scratch_ctx[dev] != ctx) {
        void* p = nullptr;
        const cudaError_t e = cudaGetSymbolAddress(&p, g_decode_scratch);  // makes the context current if needed
        if (e != cudaSuccess) return e;
        if (get_ctx(&ctx) != CUDA_SUCCESS || ctx == nullptr) return cudaErrorInvalidDevice;
        g_scratch_addr[dev] = p;
        g_scratch_ctx[dev] = ctx;
    }
    *out = g_scratch_addr[dev];
    return cudaSuccess;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace

extern "C" duo_status duo_decode_static_scratch(duo_cache* c, int32_t layer, const void* q, const void* k_new,
                                                const void* v_new, void* out, void* stream) {
    if (!c || layer < 0 || layer >= c->lay.num_layers) return DUO_ERR_INVALID_ARG;
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess) return DUO_ERR_CUDA;
    if (dev != c->device) return DUO_ERR_STATE;
    if (!q || !k_new || !v_new || !out) return DUO_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k_new) || !aligned16(v_new) || !aligned16(out)) return DUO_ERR_ALIGNMENT;
    const duo_layout& L = c->lay;

    DecodeParams p{};
    p.q = static_cast<const bf16*>(q);
    p.k_new = static_cast<const bf16*>(k_new);
    p.v_new = static_cast<const bf16*>(v_new);
    p.out = static_cast<bf16*>(out);
    p.pools = c->pools;
    p.err = c->err;
    if (fill_decode_lengths(c, layer, p) != DUO_OK) return DUO_ERR_STATE;
    if (p.len + 1 > c->lay.max_len) return DUO_ERR_CAPACITY;
    p.max_len = L.max_len;
    p.B = L.batch;
    p.Hq = L.num_q_heads;
    p.Hkv = L.num_kv_heads;
    p.G = c->G;
    p.D = L.head_dim;
    p.S = L.sink;
    p.R = L.recent;
    p.W = c->W;
    p.scale_log2 = c->scale * 1.4426950408889634f;
    p.fp8 = c->fp8 ? 1 : 0;
    p.kv_scale = c->fp8 ? c->kv_scales + static_cast<size_t>(layer) * L.num_kv_heads * 4 : nullptr;
    std::memset(&p.heads, 0, sizeof(p.heads));
    for (int g = 0; g < L.num_kv_heads; ++g) {
        const size_t i = static_cast<size_t>(layer) * L.num_kv_heads + g;
        p.heads.is_retr[g] = c->is_retr[i];
        p.heads.pool_idx[g] = c->pool_idx[i];
        if (c->is_retr[i]) p.retr_list[p.n_retr++] = static_cast<int16_t>(g);
        else p.strm_list[p.n_strm++] = static_cast<int16_t>(g);
    }

    // Same split plan as duo_decode, then limited to what the array holds.
    const int64_t rows = p.len + 1;
    int64_t nsplit =
        plan_decode_splits(L.batch, p.n_retr, p.n_strm, rows, rows < c->W ? rows : c->W, c->num_sms, c->G, p.D,
                           p.fp8 != 0);
    const size_t counters_bytes = round256(static_cast<size_t>(L.batch) * L.num_kv_heads * sizeof(uint32_t));
    if (p.n_retr > 0) {
        const int64_t pairs = static_cast<int64_t>(L.batch) * p.n_retr;
        // Bytes per split: partial outputs and their log-sum-exp, for every (b, retrieval head, query head).
        const size_t per_split = static_cast<size_t>(pairs) * p.G * (static_cast<size_t>(p.D) + 1) * sizeof(float);
        const size_t room = kStaticBytes - counters_bytes - 256;  // 256: alignment of the second region
        const int64_t fit = static_cast<int64_t>(room / per_split);
        if (counters_bytes + 256 >= kStaticBytes || fit < 1) return DUO_ERR_SCRATCH_LIMIT;
        if (nsplit > fit) nsplit = fit;
    } else if (counters_bytes > kStaticBytes) {
        return DUO_ERR_SCRATCH_LIMIT;
    }
    p.split_rows = (rows + nsplit - 1) / nsplit;
    p.nsplit = static_cast<int32_t>((rows + p.split_rows - 1) / p.split_rows);

    void* base = nullptr;
    if (scratch_address(dev, &base) != cudaSuccess) return DUO_ERR_CUDA;
    uint8_t* s8 = static_cast<uint8_t*>(base);
    const size_t items = static_cast<size_t>(L.batch) * p.n_retr * p.nsplit;
    p.counters = reinterpret_cast<uint32_t*>(s8);
    p.part_lse = reinterpret_cast<float*>(s8 + counters_bytes);
    p.part_o = reinterpret_cast<float*>(s8 + counters_bytes + round256(items * p.G * sizeof(float)));

    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (cudaMemsetAsync(p.counters, 0, counters_bytes, s) != cudaSuccess) return DUO_ERR_CUDA;
    if (launch_decode(p, decode_maps(c), s) != cudaSuccess) return DUO_ERR_CUDA;
    int64_t* lens = seq_lens(c, layer);
    for (int32_t b = 0; b < L.batch; ++b) lens[b] += 1;
    return DUO_OK;
}
