// Host build of the prefill work-item plan (tile_plan.cuh). Reads cases from
// stdin, one per line:
//   B Hq Hkv S R C ragged len_0 C_0 len_1 C_1 ... mask_0 .. mask_{Hkv-1}
// (len_b, C_b only when ragged, else one `len`), and prints for every work
// item: "item b head qt retr L C n_tiles src row0 src row0 ...".
#include <cstdio>
#include <vector>

#include "tile_plan.cuh"

int main() {
    int B, Hq, Hkv, S, R, C, ragged;
    while (std::scanf("%d %d %d %d %d %d %d", &B, &Hq, &Hkv, &S, &R, &C, &ragged) == 7) {
        duo::PrefillParams p{};
        p.B = B;
        p.Hq = Hq;
        p.Hkv = Hkv;
        p.G = Hq / Hkv;
        p.S = S;
        p.R = R;
        p.W = S + R;
        p.C = C;
        p.ragged = ragged;
        if (ragged) {
            for (int b = 0; b < B; ++b) {
                long long l;
                int c;
                if (std::scanf("%lld %d", &l, &c) != 2) return 1;
                p.seq_len[b] = l;
                p.seq_c[b] = c;
            }
        } else {
            long long l;
            if (std::scanf("%lld", &l) != 1) return 1;
            p.len = l;
        }
        int nr = 0, ns = 0;
        for (int g = 0; g < Hkv; ++g) {
            int m;
            if (std::scanf("%d", &m) != 1) return 1;
            p.heads.is_retr[g] = static_cast<uint8_t>(m);
            p.heads.pool_idx[g] = m ? nr++ : ns++;
        }
        p.n_qt = (C + duo::kTileQ - 1) / duo::kTileQ;
        int nq = 0;
        for (int pass = 0; pass < 2; ++pass) {
            for (int h = 0; h < Hq; ++h)
                if ((p.heads.is_retr[h / p.G] != 0) == (pass == 0)) p.qhead[nq++] = static_cast<int16_t>(h);
            if (pass == 0) p.n_retr_q = nq;
        }
        for (int idx = 0; idx < B * Hq * p.n_qt; ++idx) {
            const duo::Item it = duo::make_item(p, idx);
            std::printf("item %d %d %d %d %lld %d %d", it.b, it.head, it.qt, it.retr, static_cast<long long>(it.L),
                        it.C, it.n_tiles);
            for (int t = 0; t < it.n_tiles; ++t) {
                int src, row0;
                duo::tile_of(it, t, src, row0);
                std::printf(" %d %d", src, row0);
            }
            std::printf("\n");
        }
        std::printf("end\n");
    }
    return 0;
}
