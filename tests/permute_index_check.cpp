// Host-side check of the index arithmetic of the Ulysses transforms' vector kernels
// (permute_index.cuh, shared with the device code): the invariant-integer division
// (Granlund-Montgomery) against the / operator, and the source vector of every output
// vector of seq2head and head2seq against the coordinates written out directly, for G head
// groups over P shards with the GQA copy ("Метод контекстного параллелизма Ulysses": the
// seq<->head all-to-all; G = P is Ulysses, G < P the ring x Ulysses hybrid's head split),
// and the one-rank shares of the scatter kernels against the whole transforms.
#include <cstdint>
#include <cstdio>
#include <random>
#include <vector>
#include "permute_index.cuh"

int main() {
    using namespace ra;
    int bad = 0;
    std::mt19937_64 rng(1);
    for (uint32_t d : {1u, 2u, 3u, 5u, 7u, 8u, 16u, 31u, 64u, 100u, 1000u, 4096u, 16384u,
                       65537u, 131072u, 0x7fffffffu, 0x80000000u, 0xffffffffu}) {
        const FastDiv f = make_fastdiv(d);
        for (int i = 0; i < 200000; ++i) {
            const uint32_t n = i < 1000 ? (uint32_t)i
                               : i < 2000 ? 0xffffffffu - (uint32_t)(i - 1000) : (uint32_t)rng();
            if (fdiv(n, f) != n / d) ++bad;
        }
    }
    for (uint32_t d = 1; d < 5000; ++d) {
        const FastDiv f = make_fastdiv(d);
        for (uint32_t n : {0u, d - 1, d, d + 1, 2 * d - 1, 0xffffffffu, 0xfffffffeu, 123456789u})
            if (fdiv(n, f) != n / d) ++bad;
    }
    // {P, G, B, Lc, H_in, H_out, D, element size}
    const int geos[][8] = {{2, 2, 1, 64, 2, 2, 32, 4},   {4, 4, 1, 1024, 8, 8, 64, 2},
                           {8, 8, 1, 512, 4, 8, 128, 2}, {2, 2, 3, 5, 2, 4, 8, 2},
                           {4, 4, 2, 7, 1, 4, 16, 4},    {8, 8, 2, 3, 8, 16, 64, 2},
                           {3, 3, 2, 5, 3, 6, 32, 2},    {1, 1, 1, 9, 5, 5, 8, 2},
                           {4, 2, 1, 37, 2, 4, 128, 2},  {8, 4, 2, 11, 4, 4, 64, 2},
                           {6, 3, 2, 5, 6, 6, 64, 2},    {3, 1, 2, 50, 4, 4, 32, 4},
                           {8, 2, 1, 33, 4, 4, 128, 2}};
    long long checked = 0;
    for (const auto& g0 : geos) {
        const int P = g0[0], G = g0[1], B = g0[2], Lc = g0[3], Hi = g0[4], Ho = g0[5], D = g0[6],
                  es = g0[7];
        const int VD = D * es / 16, Hl = Ho / G;
        // seq2head: out [G][B][P*Lc][Hl][VD] <- in [P][B][Lc][Hi][VD]
        const PermuteGeom gs = make_seq2head_geom(P, G, B, Lc, Hi, Ho, D, es);
        const uint64_t nout = (uint64_t)G * B * P * Lc * Hl * VD, nin = (uint64_t)P * B * Lc * Hi * VD;
        for (uint64_t v = 0; v < nout; ++v, ++checked) {
            uint64_t x = v;
            const int dv = (int)(x % VD); x /= VD;
            const int hh = (int)(x % Hl); x /= Hl;
            const int gt = (int)(x % ((uint64_t)P * Lc)); x /= (uint64_t)P * Lc;
            const int b = (int)(x % B);
            const int r = (int)(x / B);
            const int s = gt / Lc, t = gt % Lc;
            const int hs = (int)(((long long)(r * Hl + hh) * Hi) / Ho);  // the GQA copy
            const uint64_t want = ((((uint64_t)s * B + b) * Lc + t) * Hi + hs) * VD + dv;
            const uint64_t got = seq2head_src_vec(gs, (uint32_t)v);
            if (got != want || got >= nin) ++bad;
        }
        // head2seq: out [P][B][Lc][Ho][VD] <- in [G][B][P*Lc][Hl][VD]
        const PermuteGeom gh = make_head2seq_geom(P, G, B, Lc, Ho, D, es);
        const uint64_t n2 = (uint64_t)P * B * Lc * Ho * VD;
        for (uint64_t v = 0; v < n2; ++v, ++checked) {
            uint64_t x = v;
            const int dv = (int)(x % VD); x /= VD;
            const int hd = (int)(x % Ho); x /= Ho;
            const int t = (int)(x % Lc); x /= Lc;
            const int b = (int)(x % B);
            const int s = (int)(x / B);
            const int r = hd / Hl, hh = hd % Hl;
            const uint64_t want =
                ((((uint64_t)r * B + b) * ((uint64_t)P * Lc) + (uint64_t)s * Lc + t) * Hl + hh) * VD + dv;
            if (head2seq_src_vec(gh, (uint32_t)v) != want) ++bad;
        }
    }
    // One rank's share of the all-to-all (G = P): every destination vector of every rank's
    // buffer is written exactly once over the P ranks' shares, from the source vector that
    // the whole-tensor transform reads for it.
    for (const auto& g0 : geos) {
        const int P = g0[0], G = g0[1], B = g0[2], Lc = g0[3], Hi = g0[4], Ho = g0[5], D = g0[6],
                  es = g0[7];
        if (G != P) continue;
        const int VD = D * es / 16, Hl = Ho / P;
        const uint64_t share = (uint64_t)P * B * Lc * Hl * VD;
        // seq2head: dst[r] [B][P*Lc][Hl][VD] is block r of the whole output
        const PermuteGeom gs = make_seq2head_geom(P, P, B, Lc, Hi, Ho, D, es);
        const uint64_t blk_out = (uint64_t)B * P * Lc * Hl * VD, blk_in = (uint64_t)B * Lc * Hi * VD;
        std::vector<int> seen(P * blk_out, 0);
        for (int me = 0; me < P; ++me) {
            const ScatterGeom sg = make_scatter_geom(P, me, B, Lc, Hi, Ho, Hl, D, es);
            for (uint64_t v = 0; v < share; ++v, ++checked) {
                const ScatterVec sv = seq2head_scatter_vec(sg, (uint32_t)v);
                if (sv.r >= (uint32_t)P || sv.dst >= blk_out || sv.src >= blk_in) { ++bad; continue; }
                const uint64_t gout = sv.r * blk_out + sv.dst;
                ++seen[gout];
                if (seq2head_src_vec(gs, (uint32_t)gout) != me * blk_in + sv.src) ++bad;
            }
        }
        for (int c : seen) if (c != 1) ++bad;
        // head2seq: dst[r] [B][Lc][P*Hl][VD] is shard r of the whole output; rank me's input is
        // head group me [B][P*Lc][Hl][VD]
        const PermuteGeom gh = make_head2seq_geom(P, P, B, Lc, Ho, D, es);
        const uint64_t shard = (uint64_t)B * Lc * Ho * VD, grp = (uint64_t)B * P * Lc * Hl * VD;
        std::vector<int> seen2(P * shard, 0);
        for (int me = 0; me < P; ++me) {
            const ScatterGeom sg = make_scatter_geom(P, me, B, Lc, Ho, Ho, Hl, D, es);
            for (uint64_t v = 0; v < share; ++v, ++checked) {
                const ScatterVec sv = head2seq_scatter_vec(sg, (uint32_t)v);
                if (sv.r >= (uint32_t)P || sv.dst >= shard || sv.src >= grp) { ++bad; continue; }
                const uint64_t gout = sv.r * shard + sv.dst;
                ++seen2[gout];
                if (head2seq_src_vec(gh, (uint32_t)gout) != me * grp + sv.src) ++bad;
            }
        }
        for (int c : seen2) if (c != 1) ++bad;
    }
    std::printf("vectors checked: %lld\nmismatches: %d\n", checked, bad);
    return bad != 0;
}
