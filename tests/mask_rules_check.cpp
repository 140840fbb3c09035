// Host build of the prefill kernel's key-visibility rules (mask_rules.cuh):
// prints one line per 32-key word for an enumeration of cache lengths, window
// sizes, chunk lengths and query rows; test_mask_rules.py checks every bit
// against the oracle's key-set and cache-slot definitions. The row-precomputed
// 32-bit forms must give the same words: a difference prints MISMATCH and the
// program exits 1.
#include <cstdio>

#include "mask_rules.cuh"

static int mismatches = 0;

static unsigned same(unsigned a, unsigned b, const char* what, long base) {
    if (a != b) {
        std::printf("MISMATCH %s base %ld: %u vs %u\n", what, base, a, b);
        ++mismatches;
    }
    return a;
}

int main() {
    const long sinks[] = {0, 1, 4, 64};
    const long recents[] = {1, 3, 64, 256};
    const long lens[] = {0, 3, 5, 64, 65, 300};
    const long chunks[] = {65, 300};
    const int rows[] = {0, 5, 63, 64, 200};
    for (long S : sinks)
        for (long R : recents)
            for (long L : lens)
                for (int q : rows) {
                    const duo::RingVis ring = duo::ring_visible(L, S, R, q);
                    const duo::RowVis vs = duo::row_visible(0, L, 300, S, R, q);
                    for (long base = 0; base < S + R + 32; base += 32)
                        std::printf("1 0 %ld %ld %ld 0 %d %ld %u\n", S, R, L, q, base,
                                    same(duo::streaming_cache_bits(L, S, ring, base),
                                         duo::streaming_cache_bits_row(vs, static_cast<int>(base)), "streaming cache",
                                         base));
                    for (long base = 0; base < L + 32; base += 32)
                        std::printf("0 1 %ld %ld %ld 0 %d %ld %u\n", S, R, L, q, base,
                                    same(duo::retrieval_cache_bits(L, base),
                                         duo::retrieval_cache_bits_row(vs, static_cast<int>(base)), "retrieval cache",
                                         base));
                    for (long C : chunks)
                        for (int retr = 0; retr < 2; ++retr) {
                            const duo::RowVis vc = duo::row_visible(retr, L, C, S, R, q);
                            for (long base = 0; base < C + 32; base += 32)
                                std::printf("2 %d %ld %ld %ld %ld %d %ld %u\n", retr, S, R, L, C, q, base,
                                            same(duo::chunk_bits(retr, L, C, S, R, q, base),
                                                 duo::chunk_bits_row(vc, static_cast<int>(base)), "chunk", base));
                        }
                }
    // Cache lengths near the 2^31 - 1 limit (compared with the 64-bit forms only:
    // the oracle check above covers the rules themselves).
    const long big[] = {2147480000L, 2147483000L};
    for (long S : sinks)
        for (long R : recents)
            for (long L : big)
                for (int q : rows) {
                    const duo::RingVis ring = duo::ring_visible(L, S, R, q);
                    const duo::RowVis vs = duo::row_visible(0, L, 300, S, R, q);
                    for (long base = 0; base < S + R + 32; base += 32)
                        same(duo::streaming_cache_bits(L, S, ring, base),
                             duo::streaming_cache_bits_row(vs, static_cast<int>(base)), "streaming cache", base);
                    for (long base = (L - 96) / 32 * 32; base < L + 32; base += 32)
                        same(duo::retrieval_cache_bits(L, base),
                             duo::retrieval_cache_bits_row(vs, static_cast<int>(base)), "retrieval cache", base);
                    for (int retr = 0; retr < 2; ++retr) {
                        const duo::RowVis vc = duo::row_visible(retr, L, 300, S, R, q);
                        for (long base = 0; base < 300 + 32; base += 32)
                            same(duo::chunk_bits(retr, L, 300, S, R, q, base), duo::chunk_bits_row(vc, static_cast<int>(base)),
                                 "chunk", base);
                    }
                }
    return mismatches == 0 ? 0 : 1;
}
