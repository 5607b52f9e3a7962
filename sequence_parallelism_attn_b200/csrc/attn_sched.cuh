// attn_sched.cuh -- the chunk/tile schedule shared by the attention kernels: which
// 128-key tiles of which K/V chunks a block of query rows visits, in ring order
// ("Как работает sequence parallelism в контексте LLM?", section 3: at step s the queries
// of rank i see the chunk of rank (i - s) mod P), with causal, zigzag and packed-sample
// tile skipping.
#pragma once
#include <cstdint>
#include "ra_internal.h"
#include "../../include/ra.h"

namespace ra {

constexpr int kSchedTile = 128;  // keys per tile

// What make_schedule needs to know about a launch.
struct SchedArgs {
    int P, Lc, L, causal, zigzag;
    const int* pid;  // packed samples: position_ids [B][L] (nullptr: none)
};

// The chunk/tile visiting order of one CTA: chunks in ring order j = (i0 - s) mod P, and
// of chunk j the tiles [range[j], range[RA_MAX_P + j]) (filled once per CTA into shared
// memory by make_schedule).
struct Sched {
    const uint32_t* range;
    int P, i0;
};

// One warp fills the schedule of a CTA whose rows are r0 .. last_row (rank-major) of batch
// b: for every chunk j the 128-key tiles holding a key the rows may see.  Causal: keys at
// positions up to the largest row position (a prefix of the shard, positions increase
// along it).  Packed samples (position_ids, contiguous layout): keys from the smallest
// sample start among the rows on (row r's sample starts at r - position_ids[r], clamped
// to [0, r]).  Returns the number of tiles (in every lane).
__device__ __forceinline__ int make_schedule(const SchedArgs& p, int b, long long r0,
                                             long long last_row, uint32_t* range) {
    const int lane = threadIdx.x & 31;
    const int ntc = (p.Lc + kSchedTile - 1) / kSchedTile;
    long long qmin, qmax;
    row_pos_range(p.zigzag, p.P, p.Lc, r0, last_row, qmin, qmax);
    long long smin = p.pid ? last_row : 0;
    if (p.pid)
        for (long long r = r0 + lane; r <= last_row; r += 32) {
            const long long st = r - (long long)p.pid[(long long)b * p.L + r];
            smin = min(smin, st < 0 ? 0 : (st > r ? r : st));
        }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) smin = min(smin, __shfl_xor_sync(0xffffffffu, smin, off));
    int n = 0;
    for (int j = lane; j < p.P; j += 32) {
        long long t_hi = ntc;
        if (p.causal) {
            const long long nk = shard_prefix(p.zigzag, p.P, p.Lc, j, qmax);
            t_hi = min((nk + kSchedTile - 1) / kSchedTile, (long long)ntc);
        }
        const long long k0 = (long long)j * p.Lc;
        long long t_lo = smin > k0 ? min((smin - k0) / kSchedTile, (long long)ntc) : 0;
        t_lo = min(t_lo, t_hi);
        range[j] = (uint32_t)t_lo;
        range[RA_MAX_P + j] = (uint32_t)t_hi;
        n += (int)(t_hi - t_lo);
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) n += __shfl_xor_sync(0xffffffffu, n, off);
    return n;
}

// Walks the schedule tile by tile; the chunk index is recomputed only when the step s
// changes, so a tile costs no integer division.
struct SchedIter {
    Sched S;
    int s, t, nt, j;
    __device__ void load_chunk() {
        j = (S.i0 - s) % S.P;
        j = j < 0 ? j + S.P : j;
        t = (int)S.range[j];
        nt = (int)S.range[RA_MAX_P + j];
    }
    __device__ void begin(const Sched& sched) {
        S = sched;
        s = 0;
        load_chunk();
        skip_empty();
    }
    __device__ void skip_empty() {
        while (s < S.P && t >= nt) {
            ++s;
            if (s < S.P) load_chunk();
        }
    }
    __device__ void next() {
        ++t;
        skip_empty();
    }
    __device__ int chunk() const { return j; }
};

}  // namespace ra
