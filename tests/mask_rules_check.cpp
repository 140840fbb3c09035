// Host build of the prefill kernel's key-visibility rules (mask_rules.cuh):
// prints one line per 32-key word for an enumeration of cache lengths, window
// sizes, chunk lengths and query rows; test_mask_rules.py checks every bit
// against the oracle's key-set and cache-slot definitions.
#include <cstdio>

#include "mask_rules.cuh"

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
                    for (long base = 0; base < S + R + 32; base += 32)
                        std::printf("1 0 %ld %ld %ld 0 %d %ld %u\n", S, R, L, q, base,
                                    duo::streaming_cache_bits(L, S, ring, base));
                    for (long base = 0; base < L + 32; base += 32)
                        std::printf("0 1 %ld %ld %ld 0 %d %ld %u\n", S, R, L, q, base,
                                    duo::retrieval_cache_bits(L, base));
                    for (long C : chunks)
                        for (int retr = 0; retr < 2; ++retr)
                            for (long base = 0; base < C + 32; base += 32)
                                std::printf("2 %d %ld %ld %ld %ld %d %ld %u\n", retr, S, R, L, C, q, base,
                                            duo::chunk_bits(retr, L, C, S, R, q, base));
                }
    return 0;
}
