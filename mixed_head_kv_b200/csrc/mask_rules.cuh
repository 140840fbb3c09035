// mask_rules.cuh — which keys of a prefill key tile a query row may see, one
// bit per key for 32 consecutive keys. Host and device code: the prefill kernel
// masks its edge tiles with these, and a host build of the same functions is
// checked against the key-set and cache-slot definitions on the CPU.
//
// Key sets (DuoAttention abstract: retrieval heads keep and attend to every
// previous token; streaming heads keep a fixed-size cache of the sink tokens
// and the latest tokens): a query at position p sees {0 .. p} (retrieval) or
// {j <= p : j < sink or p - j < recent} (streaming).
#pragma once

#include <cstdint>

#if defined(__CUDACC__)
#define DUO_MASK_FN __host__ __device__ __forceinline__
#else
#define DUO_MASK_FN inline
#endif

namespace duo {

// Bits k of a 32-bit word set for k < x (x clamped to [0, 32]).
DUO_MASK_FN uint32_t bits_below(int64_t x) {
    if (x <= 0) return 0u;
    if (x >= 32) return 0xFFFFFFFFu;
    return (1u << static_cast<uint32_t>(x)) - 1u;
}

// Bits k of a 32-bit word set for base + k in [lo, hi).
DUO_MASK_FN uint32_t bits_in(int64_t lo, int64_t hi, int64_t base) {
    return bits_below(hi - base) & ~bits_below(lo - base);
}

// Ring slots of the streaming cache visible from one query row, as at most two
// slot ranges [a0, b0) and [a1, b1). The ring holds the latest min(recent,
// len - sink) positions p >= sink below len, position p in slot
// sink + (p - sink) mod recent; the query at len + qrow sees those with
// p > len + qrow - recent, a contiguous run of positions [lo, len) that wraps
// at most once in slot order.
struct RingVis {
    int64_t a0, b0, a1, b1;
};

DUO_MASK_FN RingVis ring_visible(int64_t len, int64_t sink, int64_t recent, int qrow) {
    RingVis g{0, 0, 0, 0};
    int64_t lo = len + qrow - recent + 1;
    if (lo < sink) lo = sink;
    const int64_t c = len - lo;
    if (c > 0) {
        // 0 <= lo - sink < len + qrow < 2^31 and recent < 2^31: a 32-bit remainder.
        const int64_t r0 = static_cast<int64_t>(static_cast<uint32_t>(lo - sink) % static_cast<uint32_t>(recent));
        g.a0 = sink + r0;
        if (r0 + c <= recent) {
            g.b0 = sink + r0 + c;
        } else {
            g.b0 = sink + recent;
            g.a1 = sink;
            g.b1 = sink + r0 + c - recent;
        }
    }
    return g;
}

// Keys [base, base + 32) of one source, seen from chunk row `qrow` (absolute
// position len + qrow) of a chunk of C rows:
//   retrieval cache: slot j holds position j, valid for j < len;
//   streaming cache: sink slots j < sink hold position j, valid for j < len;
//     ring slots as in ring_visible (computed once per row);
//   chunk: row c is position len + c, valid for c < C, causal, and for
//     streaming heads a sink (len + c < sink) or inside the window.
DUO_MASK_FN uint32_t retrieval_cache_bits(int64_t len, int64_t base) { return bits_below(len - base); }

DUO_MASK_FN uint32_t streaming_cache_bits(int64_t len, int64_t sink, const RingVis& ring, int64_t base) {
    const int64_t sink_hi = len < sink ? len : sink;
    return bits_in(0, sink_hi, base) | bits_in(ring.a0, ring.b0, base) | bits_in(ring.a1, ring.b1, base);
}

DUO_MASK_FN uint32_t chunk_bits(int retr, int64_t len, int64_t C, int64_t sink, int64_t recent, int64_t qrow,
                                int64_t base) {
    const int64_t hi = (qrow < C - 1 ? qrow : C - 1);
    const uint32_t causal = bits_below(hi + 1 - base);
    if (retr) return causal;
    const uint32_t sinks = bits_below(sink - len - base);
    const uint32_t band = ~bits_below(qrow - recent + 1 - base);
    return causal & (sinks | band);
}

// The same rules with every bound of one query row computed once, in 32-bit
// arithmetic, for kernels that test many words of a row: chunk rows and slot
// indices are below 2^30 (chunk and window sizes), cache positions below 2^31.
// Each *_row function returns exactly what its 64-bit counterpart above returns
// for the same row and word.
DUO_MASK_FN uint32_t bits_below32(int32_t x) {
    if (x <= 0) return 0u;
    if (x >= 32) return 0xFFFFFFFFu;
    return (1u << static_cast<uint32_t>(x)) - 1u;
}

struct RowVis {
    int32_t c_hi;            // chunk rows < c_hi are causal: min(qrow, C - 1) + 1
    int32_t c_sink;          // chunk rows < c_sink hold sinks (streaming): max(sink - len, 0)
    int32_t c_lo;            // chunk rows >= c_lo are inside the window: qrow - recent + 1 (retrieval: -2^30)
    int32_t s_sink;          // streaming cache: sink slots < min(len, sink) are valid
    int32_t a0, b0, a1, b1;  // streaming cache: visible ring slot ranges (ring_visible)
    int32_t r_len;           // retrieval cache: slots < len are valid
};

DUO_MASK_FN RowVis row_visible(int retr, int64_t len, int64_t C, int64_t sink, int64_t recent, int qrow) {
    RowVis v;
    v.c_hi = static_cast<int32_t>((qrow < C - 1 ? qrow : C - 1) + 1);
    v.c_sink = retr ? 0 : static_cast<int32_t>(len < sink ? sink - len : 0);
    v.c_lo = retr ? -(1 << 30) : static_cast<int32_t>(qrow - recent + 1);
    v.s_sink = static_cast<int32_t>(len < sink ? len : sink);
    const RingVis g = ring_visible(len, sink, recent, qrow);
    v.a0 = static_cast<int32_t>(g.a0);
    v.b0 = static_cast<int32_t>(g.b0);
    v.a1 = static_cast<int32_t>(g.a1);
    v.b1 = static_cast<int32_t>(g.b1);
    v.r_len = static_cast<int32_t>(len);
    return v;
}

DUO_MASK_FN uint32_t retrieval_cache_bits_row(const RowVis& v, int32_t base) { return bits_below32(v.r_len - base); }

DUO_MASK_FN uint32_t streaming_cache_bits_row(const RowVis& v, int32_t base) {
    return bits_below32(v.s_sink - base) | (bits_below32(v.b0 - base) & ~bits_below32(v.a0 - base)) |
           (bits_below32(v.b1 - base) & ~bits_below32(v.a1 - base));
}

DUO_MASK_FN uint32_t chunk_bits_row(const RowVis& v, int32_t base) {
    return bits_below32(v.c_hi - base) & (bits_below32(v.c_sink - base) | ~bits_below32(v.c_lo - base));
}

}  // namespace duo
