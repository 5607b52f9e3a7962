// Host-side check of the shard-layout position helpers of the CUDA library (ra_internal.h)
// against brute force: the sequence position of every shard token, that the keys of a
// shard at positions <= q form a prefix of the shard (what the causal schedule relies on),
// the length of that prefix, and the smallest/largest position over a range of
// rank-major rows, and the query-tile ranges the backward walks for each key tile.
// Contiguous layout: "Как работает sequence parallelism в контексте
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
    // key_tile_q_ranges: for every key tile, the query tiles holding a row that sees one of
    // its keys must all be covered (zigzag: exactly those), by at most 2P ascending disjoint
    // ranges inside [0, n_qt).  Small tiles so that short sequences span many of them;
    // packed rows from seeded sample lengths (position_ids 0, 1, ... within each sample).
    unsigned seed = 12345u;
    auto rnd = [&](int n) { seed = seed * 1103515245u + 12345u; return (int)((seed >> 8) % (unsigned)n); };
    int cases = 0;
    for (int layout = 1; layout <= 2; ++layout)
        for (int P = 1; P <= 6; ++P)
            for (int Lc = layout == 1 ? 2 : 1; Lc <= 24; Lc += layout == 1 ? 2 : 1)
                for (int tile : {1, 2, 3, 4, 8})
                    for (int causal = layout == 2 ? 1 : 0; causal <= 1; ++causal) {
                        const int L = P * Lc, n_qt = (L + tile - 1) / tile, ntc = (Lc + tile - 1) / tile;
                        int pid[6 * 24];
                        for (int t = 0; t < L;) {
                            const int n = 1 + rnd(L);
                            for (int i = 0; i < n && t < L; ++i) pid[t++] = i;
                        }
                        for (int j = 0; j < P; ++j)
                            for (int kt = 0; kt < ntc; ++kt) {
                                const int key0 = kt * tile, kvalid = Lc - key0 < tile ? Lc - key0 : tile;
                                int lo[2 * 6], hi[2 * 6], nt = -1;
                                const int nr = ra::key_tile_q_ranges(layout, P, Lc, causal, tile, pid, j,
                                                                     key0, kvalid, lo, hi, &nt);
                                ++cases;
                                bool cover[6 * 24] = {};
                                int sum = 0;
                                if (nr < 0 || nr > 2 * P) { ++bad; continue; }
                                for (int i = 0; i < nr; ++i) {
                                    if (lo[i] < 0 || hi[i] > n_qt || lo[i] >= hi[i] || (i > 0 && lo[i] <= hi[i - 1])) ++bad;
                                    for (int q = lo[i]; q < hi[i] && q < n_qt && q >= 0; ++q) cover[q] = true;
                                    sum += hi[i] - lo[i];
                                }
                                if (sum != nt) ++bad;
                                for (int q = 0; q < n_qt; ++q) {
                                    bool need = false;
                                    for (int r = q * tile; r < (q + 1) * tile && r < L; ++r) {
                                        const long long rp = ra::shard_pos(layout == 1, P, Lc, r / Lc, r % Lc);
                                        const int st = layout == 2 ? ra::sample_start(pid, r) : 0;
                                        for (int c = 0; c < kvalid; ++c) {
                                            const long long kp = ra::shard_pos(layout == 1, P, Lc, j, key0 + c);
                                            if ((!causal || kp <= rp) && kp >= st) need = true;
                                        }
                                    }
                                    if (need && !cover[q]) ++bad;            // a visible tile skipped
                                    if (layout == 1 && !need && cover[q]) ++bad;  // zigzag: exact
                                }
                            }
                    }
    std::printf("key tile cases: %d\n", cases);
    std::printf("mismatches: %d\n", bad);
    return bad != 0;
}
