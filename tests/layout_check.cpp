// Host-side check of the shard-layout position helpers of the CUDA library (ra_internal.h)
// against brute force: the sequence position of every shard token, that the keys of a
// shard at positions <= q form a prefix of the shard (what the causal schedule relies on),
// the length of that prefix, and the smallest/largest position over a range of
// rank-major rows.  Contiguous layout: "Как работает sequence parallelism в контексте
// LLM?", section 2; zigzag layout: named in "Метод контекстного параллелизма Ulysses",
// introduction (2P segments of Lc/2 tokens, rank i holding segments i and 2P-1-i).
#include <cstdio>
#include "ra_internal.h"

int main() {
    int bad = 0;
    for (int zz = 0; zz < 2; ++zz)
        for (int P = 1; P <= 7; ++P)
            for (int Lc = 2; Lc <= 42; Lc += 2) {
                const long long L = (long long)P * Lc, h = Lc / 2;
                // positions: contiguous j*Lc+u; zigzag segment j then segment 2P-1-j
                for (int j = 0; j < P; ++j)
                    for (long long u = 0; u < Lc; ++u) {
                        const long long want = !zz ? j * Lc + u
                                                   : (u < h ? j * h + u : (2LL * P - 1 - j) * h + u - h);
                        if (ra::shard_pos(zz, P, Lc, j, u) != want) ++bad;
                    }
                for (int j = 0; j < P; ++j)
                    for (long long q = -2; q < L + 2; ++q) {
                        long long cnt = 0;
                        bool outside = false, prefix = true;
                        for (long long u = 0; u < Lc; ++u) {
                            if (ra::shard_pos(zz, P, Lc, j, u) <= q) {
                                ++cnt;
                                if (outside) prefix = false;
                            } else {
                                outside = true;
                            }
                        }
                        if (!prefix || ra::shard_prefix(zz, P, Lc, j, q) != cnt) ++bad;
                    }
                for (long long a = 0; a < L; a += 3)
                    for (long long b = a; b < L; b += 5) {
                        long long mn = L, mx = -1;
                        for (long long r = a; r <= b; ++r) {
                            const long long p = ra::shard_pos(zz, P, Lc, (int)(r / Lc), r % Lc);
                            mn = p < mn ? p : mn;
                            mx = p > mx ? p : mx;
                        }
                        long long pmin, pmax;
                        ra::row_pos_range(zz, P, Lc, a, b, pmin, pmax);
                        if (pmin != mn || pmax != mx) ++bad;
                    }
            }
    std::printf("mismatches: %d\n", bad);
    return bad != 0;
}
