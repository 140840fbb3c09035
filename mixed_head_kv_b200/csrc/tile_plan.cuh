// tile_plan.cuh — the work items of a prefill launch and the key tiles each
// one visits. Host and device code: the prefill kernel runs one CTA per item,
// and a host build of the same functions is checked on the CPU against the key
// sets (every visible key lies in a listed tile, no listed tile is fully
// masked).
//
// Work item idx = (batch b, query head, 128-query tile qt): retrieval heads
// first, heaviest (last) query tile first. Key tiles of 128 keys:
//   retrieval: cache tiles covering [0, len) of the retrieval pool, then chunk
//              tiles 0 .. qt (the diagonal);
//   streaming: the streaming-cache tiles holding the sinks (and the ring when
//              the window of the first query reaches below len), chunk tiles
//              holding chunk-resident sinks, then the band tiles
//              [first query - recent + 1, last query].
#pragma once

#include "duo_internal.cuh"

#if defined(__CUDACC__)
#define DUO_PLAN_FN __host__ __device__ __forceinline__
#else
#define DUO_PLAN_FN inline
#endif

namespace duo {

// What one work item attends to.
struct Item {
    int b, head, g, qt, retr, pool;
    int64_t L;    // the sequence's cache length (tokens before its chunk)
    int C;        // the sequence's chunk length (rows of the padded chunk that are tokens)
    int q0;       // first chunk row of the query tile
    int n_cache;  // cache tiles
    int src_cache;
    int a;        // streaming: chunk tiles holding chunk-resident sinks
    int b0;       // streaming: first band tile after them
    int n_tiles;
};

DUO_PLAN_FN Item make_item(const PrefillParams& p, int idx) {
    Item it;
    const int n_retr_items = p.n_retr_q * p.B * p.n_qt;
    int nh, hbase;
    if (idx < n_retr_items) {
        nh = p.n_retr_q;
        hbase = 0;
    } else {
        idx -= n_retr_items;
        nh = p.Hq - p.n_retr_q;
        hbase = p.n_retr_q;
    }
    it.qt = p.n_qt - 1 - idx / (nh * p.B);
    const int rem = idx % (nh * p.B);
    it.head = p.qhead[hbase + rem / p.B];
    it.b = rem % p.B;
    it.g = it.head / p.G;
    it.retr = p.heads.is_retr[it.g];
    it.pool = p.heads.pool_idx[it.g];
    it.q0 = it.qt * kTileQ;
    it.L = p.ragged ? p.seq_len[it.b] : p.len;
    it.C = p.ragged ? p.seq_c[it.b] : p.C;
    if (it.q0 >= it.C) {  // a query tile past this sequence's chunk (ragged batch): no work
        it.n_tiles = 0;
        return it;
    }
    const int64_t L = it.L;
    if (it.retr) {
        it.src_cache = 0;
        it.n_cache = static_cast<int>((L + kTileK - 1) / kTileK);
        it.a = 0;
        it.b0 = 0;
        it.n_tiles = it.n_cache + it.qt + 1;
    } else {
        it.src_cache = 1;
        int64_t slots = 0;
        if (L > 0) {
            const bool band_in_cache = (L > p.S) && (it.q0 < p.R - 1);
            slots = band_in_cache ? (L < p.W ? L : p.W) : (L < p.S ? L : p.S);
        }
        it.n_cache = static_cast<int>((slots + kTileK - 1) / kTileK);
        int a = 0;
        if (L < p.S) {
            const int64_t sink_rows = (p.S - L < it.C) ? (p.S - L) : it.C;
            a = static_cast<int>((sink_rows + kTileK - 1) / kTileK);
            if (a > it.qt + 1) a = it.qt + 1;
        }
        const int band_lo = it.q0 - p.R + 1 > 0 ? it.q0 - p.R + 1 : 0;
        const int tb = band_lo / kTileK;
        it.a = a;
        it.b0 = a > tb ? a : tb;
        it.n_tiles = it.n_cache + a + (it.qt + 1 - it.b0);
    }
    return it;
}

// Tile t of an item: source (0 retrieval pool, 1 streaming pool, 2 chunk) and first row.
DUO_PLAN_FN void tile_of(const Item& it, int t, int& src, int& row0) {
    if (t < it.n_cache) {
        src = it.src_cache;
        row0 = t * kTileK;
        return;
    }
    const int u = t - it.n_cache;
    src = 2;
    row0 = (it.retr || u < it.a) ? u * kTileK : (it.b0 + u - it.a) * kTileK;
}

}  // namespace duo
