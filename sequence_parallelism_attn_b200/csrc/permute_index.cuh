// permute_index.cuh -- index arithmetic of the Ulysses transforms, shared by host and
// device code so that it can be checked exhaustively on the CPU.  All indices count
// 16-byte vectors; VD = D * element_size / 16 vectors per head.
#pragma once
#include <cstdint>
#include "ra_internal.h"

#ifdef __CUDACC__
#define RA_HD __host__ __device__ __forceinline__
#else
#define RA_HD inline
#endif

namespace ra {

RA_HD uint32_t umulhi32(uint32_t a, uint32_t b) {
#ifdef __CUDA_ARCH__
    return __umulhi(a, b);
#else
    return (uint32_t)(((uint64_t)a * b) >> 32);
#endif
}

// n / d by the invariant-divisor multiplier; exact for every 32-bit n.
RA_HD uint32_t fdiv(uint32_t n, const FastDiv& f) {
    return (uint32_t)(((uint64_t)umulhi32(n, f.mul) + n) >> f.shift);
}

struct PermuteGeom {
    FastDiv VD;   // vectors per head
    FastDiv Hl;   // heads per rank on the head-sharded side
    FastDiv H;    // heads on the sequence-sharded side of head2seq
    FastDiv PLc;  // global tokens P*Lc
    FastDiv Lc;   // tokens per rank
    FastDiv B;
    FastDiv H_out;
    uint32_t H_in;
};

// G head groups (G = P for the Ulysses transform; fewer for the ring x Ulysses hybrid).
inline PermuteGeom make_seq2head_geom(int P, int G, int B, int Lc, int H_in, int H_out, int D,
                                      int esize) {
    PermuteGeom g;
    g.VD = make_fastdiv((uint32_t)(D * esize / 16));
    g.Hl = make_fastdiv((uint32_t)(H_out / G));
    g.H = make_fastdiv((uint32_t)H_out);
    g.PLc = make_fastdiv((uint32_t)P * (uint32_t)Lc);
    g.Lc = make_fastdiv((uint32_t)Lc);
    g.B = make_fastdiv((uint32_t)B);
    g.H_out = make_fastdiv((uint32_t)H_out);
    g.H_in = (uint32_t)H_in;
    return g;
}

inline PermuteGeom make_head2seq_geom(int P, int G, int B, int Lc, int H, int D, int esize) {
    PermuteGeom g;
    g.VD = make_fastdiv((uint32_t)(D * esize / 16));
    g.Hl = make_fastdiv((uint32_t)(H / G));
    g.H = make_fastdiv((uint32_t)H);
    g.PLc = make_fastdiv((uint32_t)P * (uint32_t)Lc);
    g.Lc = make_fastdiv((uint32_t)Lc);
    g.B = make_fastdiv((uint32_t)B);
    g.H_out = make_fastdiv((uint32_t)H);
    g.H_in = (uint32_t)H;
    return g;
}

// Output vector `vec` of seq2head, out [G][B][P*Lc][Hl][VD] (group r), reads input vector
//   in [s][b][t][hs][dv] with (r, b, s*Lc+t, hh, dv) = coordinates of vec and
//   hs = ((r*Hl + hh) * H_in) / H_out  (the GQA copy).
RA_HD uint64_t seq2head_src_vec(const PermuteGeom& g, uint32_t vec) {
    const uint32_t seg = fdiv(vec, g.VD);
    const uint32_t dv = vec - seg * g.VD.div;
    const uint32_t row = fdiv(seg, g.Hl);
    const uint32_t hh = seg - row * g.Hl.div;
    const uint32_t rb = fdiv(row, g.PLc);
    const uint32_t gt = row - rb * g.PLc.div;
    const uint32_t r = fdiv(rb, g.B);
    const uint32_t b = rb - r * g.B.div;
    const uint32_t s = fdiv(gt, g.Lc);
    const uint32_t t = gt - s * g.Lc.div;
    const uint32_t hs = fdiv((r * g.Hl.div + hh) * g.H_in, g.H_out);
    return ((((uint64_t)s * g.B.div + b) * g.Lc.div + t) * g.H_in + hs) * g.VD.div + dv;
}

// Output vector `vec` of head2seq, out [P][B][Lc][H][VD] (coordinates s, b, t, hd, dv),
// reads in [r][b][s*Lc+t][hh][dv] (group r of G) with hd = r*Hl + hh.
RA_HD uint64_t head2seq_src_vec(const PermuteGeom& g, uint32_t vec) {
    const uint32_t seg = fdiv(vec, g.VD);
    const uint32_t dv = vec - seg * g.VD.div;
    const uint32_t row = fdiv(seg, g.H);
    const uint32_t hd = seg - row * g.H.div;
    const uint32_t r = fdiv(hd, g.Hl);
    const uint32_t hh = hd - r * g.Hl.div;
    const uint32_t sb = fdiv(row, g.Lc);
    const uint32_t t = row - sb * g.Lc.div;
    const uint32_t s = fdiv(sb, g.B);
    const uint32_t b = sb - s * g.B.div;
    return ((((uint64_t)r * g.B.div + b) * g.PLc.div + (uint64_t)s * g.Lc.div + t) * g.Hl.div +
            hh) * g.VD.div + dv;
}

// ------------------------------------------------------------------ scatter (one rank's share)
// One rank `me` of P writes its share of the Ulysses all-to-all straight into the P
// destination buffers (peer memory or local).  The share is enumerated as vectors over
// [P (destination r)][B][Lc][Hl][VD]; every vector has one source and one destination.
//   seq2head: in [B][Lc][H_in][VD] (this rank's sequence shard) -> dst[r] [B][P*Lc][Hl][VD]
//     at token me*Lc + t, head hh of group r (source head hs by the GQA copy).
//   head2seq: in [B][P*Lc][Hl][VD] (this rank's head group) -> dst[r] [B][Lc][P*Hl][VD]
//     (rank r's sequence shard) at head me*Hl + hh, from token r*Lc + t.
struct ScatterGeom {
    FastDiv VD, Hl, Lc, B, H_out;
    uint32_t P, me, H_in;
};

struct ScatterVec {
    uint32_t r;    // destination rank
    uint64_t src;  // vector index into in
    uint64_t dst;  // vector index into dst[r]
};

inline ScatterGeom make_scatter_geom(int P, int me, int B, int Lc, int H_in, int H_out, int Hl,
                                     int D, int esize) {
    ScatterGeom g;
    g.VD = make_fastdiv((uint32_t)(D * esize / 16));
    g.Hl = make_fastdiv((uint32_t)Hl);
    g.Lc = make_fastdiv((uint32_t)Lc);
    g.B = make_fastdiv((uint32_t)B);
    g.H_out = make_fastdiv((uint32_t)H_out);
    g.P = (uint32_t)P;
    g.me = (uint32_t)me;
    g.H_in = (uint32_t)H_in;
    return g;
}

// coordinates (r, b, t, hh, dv) of share vector `vec`
RA_HD void scatter_coords(const ScatterGeom& g, uint32_t vec, uint32_t& r, uint32_t& b,
                          uint32_t& t, uint32_t& hh, uint32_t& dv) {
    const uint32_t seg = fdiv(vec, g.VD);
    dv = vec - seg * g.VD.div;
    const uint32_t row = fdiv(seg, g.Hl);
    hh = seg - row * g.Hl.div;
    const uint32_t rb = fdiv(row, g.Lc);
    t = row - rb * g.Lc.div;
    r = fdiv(rb, g.B);
    b = rb - r * g.B.div;
}

RA_HD ScatterVec seq2head_scatter_vec(const ScatterGeom& g, uint32_t vec) {
    uint32_t r, b, t, hh, dv;
    scatter_coords(g, vec, r, b, t, hh, dv);
    const uint32_t hs = fdiv((r * g.Hl.div + hh) * g.H_in, g.H_out);
    const uint64_t PLc = (uint64_t)g.P * g.Lc.div;
    ScatterVec o;
    o.r = r;
    o.src = (((uint64_t)b * g.Lc.div + t) * g.H_in + hs) * g.VD.div + dv;
    o.dst = (((uint64_t)b * PLc + (uint64_t)g.me * g.Lc.div + t) * g.Hl.div + hh) * g.VD.div + dv;
    return o;
}

RA_HD ScatterVec head2seq_scatter_vec(const ScatterGeom& g, uint32_t vec) {
    uint32_t r, b, t, hh, dv;
    scatter_coords(g, vec, r, b, t, hh, dv);
    const uint64_t PLc = (uint64_t)g.P * g.Lc.div;
    const uint64_t H = (uint64_t)g.P * g.Hl.div;
    ScatterVec o;
    o.r = r;
    o.src = (((uint64_t)b * PLc + (uint64_t)r * g.Lc.div + t) * g.Hl.div + hh) * g.VD.div + dv;
    o.dst = (((uint64_t)b * g.Lc.div + t) * H + (uint64_t)g.me * g.Hl.div + hh) * g.VD.div + dv;
    return o;
}

}  // namespace ra
