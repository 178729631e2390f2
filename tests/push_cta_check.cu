// Host-only check of the fp32 trailing update's launch shapes (push_variant, push_grid, push_cta in
// kg_push_tc.cuh): runs on the CPU, launches nothing.  Reads pieces "D0 mid tgt0 D1 Mt Nt" from
// standard input, one per line, enumerates every CTA of each piece's grid with the same functions
// the kernel and its launch use, and checks, per chain, that every target tile of the band (tile
// (t, b) with t + b in [tgt0, D1)) is written by exactly one CTA when its own K range
// [max(0, D0 - b), min(K, mid - b)) is not empty, by at most one when it is (two CTAs writing one
// tile would race in their read-modify-write), and that the CTA's K range covers the tile's own.
// Prints "ok <pieces> <ctas with work>" and exits 0, or prints the first violation and exits 1.
// With --skip-first-row it leaves out the CTAs with blockIdx.y = 0, so that a test can see the check
// fail.
#include <cstdio>
#include <cstring>
#include <vector>

#include "kg_push_tc.cuh"

using namespace kg;

static bool g_skip_first_row = false;

template <int NB, int MT>
static bool check(int D0, int mid, int tgt0, int D1, int Mt, int Nt, long long& ctas) {
    const dim3 g = push_grid(push_variant(D0, mid, tgt0, D1), tgt0, D1, Mt, Nt);
    if (g.y > 65535u || g.z != 2u) {
        std::printf("bad grid %u %u %u for %d %d %d %d %d %d\n", g.x, g.y, g.z, D0, mid, tgt0, D1, Mt, Nt);
        return false;
    }
    for (int chain = 0; chain < 2; ++chain) {
        const int Bmax = chain ? Nt : Mt, Tmax = chain ? Mt : Nt, Kmax = chain ? Mt : Nt;
        std::vector<int> cnt((size_t)Tmax * Bmax, 0);
        for (unsigned by = g_skip_first_row ? 1u : 0u; by < g.y; ++by)
            for (unsigned bx = 0; bx < g.x; ++bx) {
                PushCta c;
                if (!push_cta<NB, MT>((int)bx, (int)by, (int)g.y, chain, D0, mid, tgt0, D1, Mt, Nt, c)) continue;
                ++ctas;
                if (c.b0 < 0 || c.t0 < 0 || c.k0 < 0 || c.k1 > Kmax) {
                    std::printf("CTA out of range: piece %d %d %d %d shape %d %d chain %d b0 %d t0 %d k %d..%d\n", D0,
                                mid, tgt0, D1, Mt, Nt, chain, c.b0, c.t0, c.k0, c.k1);
                    return false;
                }
                for (int u = 0; u < MT; ++u)
                    for (int h = 0; h < NB; ++h) {
                        const int t = c.t0 + u, b = c.b0 + h;
                        // the epilogue's store predicate
                        if (!(t < Tmax && b < Bmax && t + b >= tgt0 && t + b < D1)) continue;
                        ++cnt[(size_t)t * Bmax + b];
                        const int lo = D0 - b > 0 ? D0 - b : 0, hi = mid - b < Kmax ? mid - b : Kmax;
                        if (lo < hi && (lo < c.k0 || hi > c.k1)) {
                            std::printf("K range of tile (%d, %d) [%d, %d) not inside the CTA's [%d, %d)\n", t, b, lo,
                                        hi, c.k0, c.k1);
                            return false;
                        }
                    }
            }
        for (int t = 0; t < Tmax; ++t)
            for (int b = 0; b < Bmax; ++b) {
                const int n = cnt[(size_t)t * Bmax + b];
                const bool band = t + b >= tgt0 && t + b < D1;
                const int lo = D0 - b > 0 ? D0 - b : 0, hi = mid - b < Kmax ? mid - b : Kmax;
                const int want_min = band && lo < hi ? 1 : 0, want_max = band ? 1 : 0;
                if (n < want_min || n > want_max) {
                    std::printf("tile (%d, %d) of chain %d written %d times: piece %d %d %d %d shape %d %d\n", t, b,
                                chain, n, D0, mid, tgt0, D1, Mt, Nt);
                    return false;
                }
            }
    }
    return true;
}

int main(int argc, char** argv) {
    g_skip_first_row = argc > 1 && std::strcmp(argv[1], "--skip-first-row") == 0;
    int D0, mid, tgt0, D1, Mt, Nt;
    long long pieces = 0, ctas = 0;
    while (std::scanf("%d %d %d %d %d %d", &D0, &mid, &tgt0, &D1, &Mt, &Nt) == 6) {
        const int v = push_variant(D0, mid, tgt0, D1);
        const bool ok = v == PV_PAIR     ? check<2, 2>(D0, mid, tgt0, D1, Mt, Nt, ctas)
                        : v == PV_SINGLE ? check<1, 1>(D0, mid, tgt0, D1, Mt, Nt, ctas)
                                         : check<1, 2>(D0, mid, tgt0, D1, Mt, Nt, ctas);
        if (!ok) return 1;
        ++pieces;
    }
    std::printf("ok %lld %lld\n", pieces, ctas);
    return 0;
}
