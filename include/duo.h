/*
 * duo.h — C ABI of libduo: mixed-head (DuoAttention) attention on B200 (sm_100a).
 *
 * The method (DuoAttention abstract, pith.science review page, "read the
 * original abstract"; sourcepulse project card, "How It Works"): each KV head
 * of each layer is either a retrieval head, which keeps a full KV cache and
 * attends causally over every previous token, or a streaming head, which keeps
 * a constant-length KV cache of the first `sink` tokens (attention sinks) plus
 * the `recent` most recent tokens, and attends only to those. In GQA models
 * every query head inherits the type of its KV head. The library covers the two
 * phases the pages speed up (pre-filling, in chunks, and decoding) and the
 * per-head cache append/eviction behind them.
 *
 * Conventions (all calls):
 *  - Tensors are bf16, row-major, contiguous, in device memory owned by the
 *    caller, 16-byte aligned (DUO_ERR_ALIGNMENT otherwise).
 *      prefill q / out   [batch][n_tok][num_q_heads][head_dim]
 *      prefill k / v     [batch][n_tok][num_kv_heads][head_dim]
 *      decode  q / out   [batch][num_q_heads][head_dim]
 *      decode  k / v     [batch][num_kv_heads][head_dim]
 *  - `stream` is a cudaStream_t passed as void* (NULL = legacy default stream).
 *    Every call is stream-ordered and asynchronous; host-side cache lengths are
 *    updated when the call is enqueued. Calls on one cache must be issued on
 *    one stream (or ordered by the caller): they share the cache's device state.
 *  - Argument errors are reported before any launch and leave the cache
 *    unchanged. DUO_ERR_CUDA reports a failed launch or CUDA call.
 *  - Positions are absolute token indices within a sequence, starting at 0.
 *    Each sequence of a batch has its own cache length (duo_cache_seq_lens).
 *  - Positional encodings are the caller's: q and k arrive already encoded and
 *    cached tokens keep their original positions (no re-indexing).
 *  - Softmax scale: layout.softmax_scale, or 1/sqrt(head_dim) when it is 0.
 */
#ifndef DUO_H_
#define DUO_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define DUO_API __attribute__((visibility("default")))
#else
#define DUO_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum duo_status {
    DUO_OK = 0,
    DUO_ERR_INVALID_ARG = 1, /* bad layout, mask, layer, size or null pointer */
    DUO_ERR_CAPACITY = 2,    /* a retrieval cache would exceed max_len tokens */
    DUO_ERR_ALIGNMENT = 3,   /* a pointer is not 16-byte aligned */
    DUO_ERR_CUDA = 4,        /* a CUDA call or kernel launch failed */
    DUO_ERR_STATE = 5,       /* call not valid in the cache's current state */
    DUO_ERR_DEVICE = 6,      /* a kernel reported a device-side error (see duo_cache_error) */
    DUO_ERR_SCRATCH_LIMIT = 7 /* the request needs more than DUO_STATIC_SCRATCH_BYTES */
} duo_status;

/* Storage format of the retrieval heads' caches (streaming caches are always
 * bf16). The pages reach their longest contexts only with a quantized KV cache
 * (DuoAttention abstract: 3.3 million tokens on one GPU "combined with
 * quantization"); this library offers FP8 E4M3 with one scale per (layer, KV
 * head) for K and one for V:
 *   DUO_KV_BF16  bf16 rows (default)
 *   DUO_KV_E4M3  each element is stored as the E4M3 code of x * inv_scale (the
 *                product in fp32, inv_scale the fp32 reciprocal of the head's
 *                scale), rounded to nearest with ties to even and saturated to
 *                +-448, and read back as value(code) * scale. Halves the bytes a
 *                decode step reads from retrieval caches. */
#define DUO_KV_BF16 0
#define DUO_KV_E4M3 1

/* Largest head counts the kernels accept. */
#define DUO_MAX_Q_HEADS 256
#define DUO_MAX_KV_HEADS 128

/* Largest batch whose sequences may have different lengths (a ragged batch):
 * the per-sequence lengths travel with each launch. Larger batches keep one
 * length for all sequences. */
#define DUO_MAX_RAGGED_BATCH 64

/* Shape of the model's attention and of the caches.
 *   num_layers    >= 1
 *   batch         >= 1 sequences (each with its own cache length; see
 *                 duo_cache_seq_lens)
 *   num_q_heads   query heads, a multiple of num_kv_heads (GQA group size G)
 *   num_kv_heads  KV heads; the retrieval/streaming type is per (layer, KV head)
 *   head_dim      64 or 128
 *   sink          attention-sink tokens kept by streaming heads (>= 0)
 *   recent        recent tokens kept by streaming heads (>= 1); includes the
 *                 query's own token, so a streaming query at position p attends
 *                 to { j <= p : j < sink or p - j < recent }
 *   kv_format     DUO_KV_BF16 or DUO_KV_E4M3 (retrieval caches; see above)
 *   max_len       capacity of every retrieval cache in tokens
 *   softmax_scale 0 selects 1/sqrt(head_dim) */
typedef struct duo_layout {
    int32_t num_layers;
    int32_t batch;
    int32_t num_q_heads;
    int32_t num_kv_heads;
    int32_t head_dim;
    int32_t sink;
    int32_t recent;
    int32_t kv_format; /* DUO_KV_BF16 or DUO_KV_E4M3: storage of the retrieval caches */
    int64_t max_len;
    float softmax_scale;
    int32_t reserved1;
} duo_layout;

/* Opaque host object: the layout, the per-layer head maps and lengths, and
 * pointers into the caller's device buffer. */
typedef struct duo_cache duo_cache;

/* duo_cache_alloc — set up the two cache kinds of DuoAttention (a full cache per
 * retrieval head, a constant-length sink + recent cache per streaming head;
 * DuoAttention abstract) inside one caller-owned device buffer.
 *   layout        shape (see duo_layout); copied
 *   is_retrieval  host array [num_layers][num_kv_heads]: 1 = retrieval, 0 = streaming
 *   dev_buf       device buffer of at least *required_bytes bytes, 256-byte
 *                 aligned; NULL to only compute *required_bytes
 *   buf_bytes     size of dev_buf
 *   required_bytes out: bytes the cache needs (always written when non-NULL)
 *   stream        stream on which the buffer is zero-filled
 *   out           out: the new cache object (when dev_buf != NULL)
 * Device layout inside dev_buf (offsets in required_bytes order):
 *   retrieval K, V pools  [n_retrieval_heads_all_layers][batch][max_len][head_dim]
 *                         (bf16, or one-byte E4M3 codes for DUO_KV_E4M3)
 *   streaming K, V pools  [n_streaming_heads_all_layers][batch][sink+recent][head_dim]
 *   streaming slot rule   position p < sink -> slot p; otherwise slot
 *                         sink + (p - sink) mod recent (fixed sinks + a ring)
 *   decode scratch        split-KV partial results: batch x R x 256 splits x
 *                         (num_q_heads / num_kv_heads) x (head_dim + 1) fp32,
 *                         R = the most retrieval KV heads of any one layer
 *                         (streaming heads write none); per-(sequence, KV head)
 *                         split counters; an error word and the prefill's
 *                         work-item counters (one 256-byte block)
 *   E4M3 scales           DUO_KV_E4M3 only: [num_layers][num_kv_heads] x 4 fp32
 *                         (k_scale, v_scale and their fp32 reciprocals), 1 until
 *                         duo_cache_set_kv_scales
 * The caller keeps ownership of dev_buf and frees it after duo_cache_free. */
DUO_API duo_status duo_cache_alloc(const duo_layout* layout, const uint8_t* is_retrieval, void* dev_buf,
                           size_t buf_bytes, size_t* required_bytes, void* stream, duo_cache** out);

/* duo_cache_free — release the host object (not the device buffer). NULL is allowed. */
DUO_API duo_status duo_cache_free(duo_cache* cache);

/* duo_cache_append — append n_tok tokens per sequence to every KV head of `layer`
 * (the per-head cache update of DuoAttention: retrieval heads keep everything,
 * streaming heads keep sinks and evict the oldest recent token).
 *   k, v   device [batch][n_tok][num_kv_heads][head_dim] bf16, the tokens at
 *          positions [len_b, len_b + n_tok) of each sequence b (its own length)
 *   n_tok  >= 0 (0 is a no-op)
 * Retrieval heads write position p to slot p. Streaming heads write sink
 * positions to their slots and only the last min(n_tok, recent) non-sink
 * positions to their ring slots (earlier ones would be evicted within the call).
 * DUO_ERR_CAPACITY if some len_b + n_tok > max_len. Then every len_b += n_tok. */
DUO_API duo_status duo_cache_append(duo_cache* cache, int32_t layer, const void* k, const void* v, int64_t n_tok,
                            void* stream);

/* duo_cache_append_ragged — append a different number of tokens to each
 * sequence of `layer` (a ragged batch: sequences of different lengths).
 *   k, v     device [batch][max_tok][num_kv_heads][head_dim]; sequence b's rows
 *            [0, n_tok[b]) are its tokens at positions [len_b, len_b + n_tok[b]),
 *            the remaining rows are not read
 *   n_tok    host [batch], 0 <= n_tok[b] <= max_tok
 * Same slot rules as duo_cache_append, per sequence. Needs batch <=
 * DUO_MAX_RAGGED_BATCH unless every sequence has the same length and
 * n_tok[b] == max_tok for all b. DUO_ERR_CAPACITY if some len_b + n_tok[b] >
 * max_len (nothing is appended). Then len_b += n_tok[b]. */
DUO_API duo_status duo_cache_append_ragged(duo_cache* cache, int32_t layer, const void* k, const void* v,
                                   const int64_t* n_tok, int64_t max_tok, void* stream);

/* duo_prefill — attention of one prefill chunk of `layer` (DuoAttention
 * pre-filling; chunked as in the chunked-prefill work the pages cite).
 *   q      device [batch][n_tok][num_q_heads][head_dim], queries at positions
 *          [len, len + n_tok) with len = duo_cache_len(layer)
 *   k, v   device [batch][n_tok][num_kv_heads][head_dim], the chunk's own tokens
 *   out    device [batch][n_tok][num_q_heads][head_dim], written
 * Retrieval heads attend causally over the cache [0, len) and the chunk;
 * streaming heads over the sinks and the recent window, read from the
 * streaming cache for positions < len and from k/v for the chunk.
 * Does NOT modify the cache: call duo_cache_append(layer, k, v, n_tok) after it.
 * DUO_KV_E4M3 caches: the tensor-core prefill reads bf16 tiles only, so a chunk
 * is refused (DUO_ERR_STATE) once a retrieval head of the layer holds tokens;
 * prefill the prompt in one chunk, then decode.
 * Each sequence's chunk starts at its own length len_b (a ragged batch needs
 * batch <= DUO_MAX_RAGGED_BATCH, else DUO_ERR_STATE).
 * DUO_ERR_CAPACITY if a retrieval head could not hold len_b + n_tok tokens. */
DUO_API duo_status duo_prefill(duo_cache* cache, int32_t layer, const void* q, const void* k, const void* v, void* out,
                       int64_t n_tok, void* stream);

/* duo_prefill_ragged — duo_prefill with a different chunk length per sequence.
 *   q, k, v, out  as duo_prefill with max_tok rows per sequence; sequence b's
 *                 rows [0, n_tok[b]) are its chunk at positions
 *                 [len_b, len_b + n_tok[b]); its other rows are not read and its
 *                 other output rows are not written
 *   n_tok         host [batch], 0 <= n_tok[b] <= max_tok
 * Follow it with duo_cache_append_ragged(layer, k, v, n_tok, max_tok). Needs
 * batch <= DUO_MAX_RAGGED_BATCH unless all lengths and counts are equal. */
DUO_API duo_status duo_prefill_ragged(duo_cache* cache, int32_t layer, const void* q, const void* k, const void* v,
                              void* out, const int64_t* n_tok, int64_t max_tok, void* stream);

/* duo_decode — one decoding step of `layer` (DuoAttention decoding).
 *   q            device [batch][num_q_heads][head_dim], sequence b's query at
 *                position len_b (its cache length)
 *   k_new, v_new device [batch][num_kv_heads][head_dim], the new tokens
 *   out          device [batch][num_q_heads][head_dim], written
 * Appends each sequence's new token to every head's cache at that sequence's
 * own length (as duo_cache_append with one token), then attends: retrieval
 * heads over positions [0, len_b], streaming heads over the sinks and the last
 * `recent` positions. Then every len_b += 1. Sequences of different lengths
 * (a ragged batch) need batch <= DUO_MAX_RAGGED_BATCH, else DUO_ERR_STATE.
 * Uses the cache's decode scratch: decode calls on one cache must not overlap
 * on the device. DUO_ERR_CAPACITY if some len_b + 1 > max_len. */
DUO_API duo_status duo_decode(duo_cache* cache, int32_t layer, const void* q, const void* k_new, const void* v_new,
                      void* out, void* stream);

/* duo_cache_len — tokens appended so far to `layer` (host value; no sync).
 * DUO_ERR_STATE if its sequences have different lengths (see
 * duo_cache_seq_lens). */
DUO_API duo_status duo_cache_len(const duo_cache* cache, int32_t layer, int64_t* len);

/* duo_cache_set_len — set the host-side length of every sequence of `layer`,
 * e.g. to restore a snapshot taken with duo_cache_len (the device contents are
 * the caller's to restore). 0 <= len <= max_len. */
DUO_API duo_status duo_cache_set_len(duo_cache* cache, int32_t layer, int64_t len);

/* duo_cache_set_kv_scales — per-KV-head scales of a DUO_KV_E4M3 cache.
 *   k_scale, v_scale  host [num_kv_heads], finite and > 0 (the entries of
 *                     streaming heads are checked but not used)
 * The scales apply to tokens appended (and decoded) afterwards: set them before
 * the layer's first append. Copies them to the device on `stream`.
 * DUO_ERR_STATE for a bf16 cache; DUO_ERR_INVALID_ARG for a bad scale (nothing
 * changes). */
DUO_API duo_status duo_cache_set_kv_scales(duo_cache* cache, int32_t layer, const float* k_scale,
                                           const float* v_scale, void* stream);

/* duo_cache_seq_lens — per-sequence lengths of `layer`.
 *   lens  host [batch], written (host values; no sync) */
DUO_API duo_status duo_cache_seq_lens(const duo_cache* cache, int32_t layer, int64_t* lens);

/* duo_cache_set_seq_lens — set the per-sequence lengths of `layer`.
 *   lens  host [batch], 0 <= lens[b] <= max_len (nothing changes otherwise) */
DUO_API duo_status duo_cache_set_seq_lens(duo_cache* cache, int32_t layer, const int64_t* lens);

/* duo_cache_views — where one KV head's cache lives, for inspection.
 *   k, v          out: device pointers to [batch][slots][head_dim] bf16
 *                 (uint8 E4M3 codes for a retrieval head of a DUO_KV_E4M3 cache)
 *   slots         out: max_len (retrieval) or sink + recent (streaming)
 *   is_retrieval  out: 1 or 0
 * Any out pointer may be NULL. */
DUO_API duo_status duo_cache_views(const duo_cache* cache, int32_t layer, int32_t kv_head, void** k, void** v,
                           int64_t* slots, int32_t* is_retrieval);

/* duo_cache_error — read and clear the device-side error word of the cache
 * (bit flags set by kernels whose bounded waits ran out: DUO_ERR_BIT_PREFILL_WAIT,
 * DUO_ERR_BIT_DECODE_COPY). Synchronizes `stream`. *flags = 0 when no kernel
 * reported an error. */
DUO_API duo_status duo_cache_error(duo_cache* cache, void* stream, uint32_t* flags);

/* duo_decode_static_scratch — duo_decode for callers that cannot allocate device
 * memory when they call in. The pages have no counterpart to this call: it is a
 * deployment variant of the decode step.
 *
 * Some callers cannot call cudaMalloc at decode time: an inference-engine
 * plugin that only gets a memory arena planned before the run, a serving loop
 * that must not let cudaMalloc/cudaFree synchronize the device, or a process
 * whose device-memory budget belongs to another allocator. This call computes
 * exactly what duo_decode computes (same arguments, same cache update, same
 * result within rounding), but keeps the split-KV partial results in one
 * file-scope device array of DUO_STATIC_SCRATCH_BYTES instead of the cache's
 * scratch region. It allocates nothing and calls no allocating routine.
 *   - Every GPU that loads libduo holds the array until the process exits.
 *   - All calls on a device share the array; it keeps the previous call's
 *     contents (the call clears what must start at zero on `stream`). Calls
 *     whose kernels overlap on the GPU race on it: issue them on one stream.
 *   - The first call on a device looks up the array's address
 *     (cudaGetSymbolAddress, device current): make it before any stream capture.
 *     The address is kept per device and context; after a device reset the
 *     first call in the new context looks it up again (also before any capture).
 *   - DUO_ERR_SCRATCH_LIMIT when even one split per (sequence, retrieval head)
 *     does not fit: batch * retrieval KV heads * G * (head_dim + 1) * 4 bytes
 *     plus batch * num_kv_heads * 4 bytes of counters must stay below the limit.
 *     Long contexts are served with fewer, longer splits when the full split
 *     plan does not fit. */
#define DUO_STATIC_SCRATCH_BYTES (16u * 1024u * 1024u)
DUO_API duo_status duo_decode_static_scratch(duo_cache* cache, int32_t layer, const void* q, const void* k_new,
                                             const void* v_new, void* out, void* stream);

/* duo_cache_test_wait_timeout — a test of the kernels' failure detection; not
 * for production use. Every wait of a kernel on an asynchronous copy is bounded
 * (1 s); when one runs out the kernel sets a bit in the cache's error word
 * (duo_cache_error), finishes without the missing data and returns, and the
 * call that launched it has already returned DUO_OK. This call arms the next
 * launch of the kinds in `launches` on this cache to exercise that path without
 * any fault: one of its CTAs does not issue one of its copies, and the wait for
 * that copy gives up after `timeout_ns` (1 us .. 1 s) instead of 1 s. Every
 * other copy is issued and waited for as usual, so nothing is left in flight.
 *   DUO_TEST_WAIT_DECODE  the next duo_decode launch: warp 0 of its first CTA
 *                         withholds its first K/V block; error bit
 *                         DUO_ERR_BIT_DECODE_COPY; that step's output is wrong,
 *                         the cache update and every later call are not affected
 *   DUO_TEST_WAIT_PREFILL the next duo_prefill launch: its first CTA withholds
 *                         its first K tile; the CTA's MMA issuer gives up, the
 *                         CTA's other roles stop at their next wait and drain
 *                         what they issued; error bit DUO_ERR_BIT_PREFILL_WAIT;
 *                         the output rows of that CTA's work items are not
 *                         written, every other item's rows are
 * 0 disarms. DUO_ERR_INVALID_ARG for an unknown kind or a limit out of range. */
#define DUO_TEST_WAIT_DECODE 1
#define DUO_TEST_WAIT_PREFILL 2
#define DUO_ERR_BIT_PREFILL_WAIT 1u  /* duo_cache_error bits */
#define DUO_ERR_BIT_DECODE_COPY 2u
DUO_API duo_status duo_cache_test_wait_timeout(duo_cache* cache, int32_t launches, uint64_t timeout_ns);

/* duo_status_str — static description of a status code. */
DUO_API const char* duo_status_str(duo_status status);

#ifdef __cplusplus
}
#endif

#endif /* DUO_H_ */
