// attn_fp32.cu -- ring-chunked exact attention for fp32 inputs on CUDA cores.
//
// Same computation as the tensor-core kernel ("Как работает sequence parallelism в
// контексте LLM?", sections 2, 3 and 5): the queries of virtual rank i visit the K/V
// chunks j = (i - s) mod P for s = 0..P-1 (chunks wholly after the queries skipped when
// causal), and the running (max, normaliser, output) state is rescaled by
// exp(m_old - m_new) whenever a new chunk or tile raises the row maximum, which is the
// log-sum-exp merge of the ring applied one 32-key tile at a time.  Everything is fp32
// with IEEE expf/logf; tf32 tensor cores would not meet a 1e-4 tolerance.
//
// Launch: one CTA = 8 warps = 8 consecutive query rows of one (batch, head); each warp
// owns one row.  K/V tiles of 32 keys are staged in shared memory (K rows padded to
// D+1 floats so that lane c reading key c's row is conflict-free) and shared by the 8
// warps.  Lane c computes the score of key c; the output row is spread over the lanes
// (D/32 values each), and the probabilities are broadcast with shuffles.
#include "ra_internal.h"
#include "../../include/ra.h"
#include <cmath>

namespace ra {
namespace {

constexpr int kRows = 8;   // query rows (warps) per CTA
constexpr int kKeys = 32;  // keys per staged tile

struct Fp32Params {
    const float* q;
    const float* k[RA_MAX_P];
    const float* v[RA_MAX_P];
    float* out;
    float* lse;
    long long q_bstride, kv_bstride;
    int P, B, H_q, H_kv, Lc, L, causal, zigzag;
    const int* pid;  // packed samples: position_ids [B][L] (nullptr: none)
    float scale;
};

template <int D>
__global__ void __launch_bounds__(kRows * 32) attn_fwd_fp32(const __grid_constant__ Fp32Params p) {
    __shared__ float ks[kKeys][D + 1];
    __shared__ float vs[kKeys][D];
    __shared__ float qs[kRows][D];
    constexpr int NPL = D / 32;  // output values per lane

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int bh = blockIdx.y;
    const int b = bh / p.H_q, h = bh % p.H_q, g = h / (p.H_q / p.H_kv);
    const int r0 = blockIdx.x * kRows;
    const int row = r0 + warp;
    const bool active = row < p.L;
    const int last_row = min(r0 + kRows - 1, p.L - 1);
    // sequence positions (the shard layout): this warp's row and the CTA's largest
    const long long my_pos = active ? shard_pos(p.zigzag, p.P, p.Lc, row / p.Lc, row % p.Lc) : 0;
    long long qmin, qmax;
    row_pos_range(p.zigzag, p.P, p.Lc, r0, last_row, qmin, qmax);
    // packed samples: row r's sample starts at r - position_ids[r] (clamped to [0, r]);
    // this warp's row sees no key before its start, and the CTA none before the smallest
    auto sample_start = [&](int r) {
        const int st = r - p.pid[(long long)b * p.L + r];
        return st < 0 ? 0 : (st > r ? r : st);
    };
    const long long my_start = (p.pid && active) ? sample_start(row) : 0;
    long long smin = 0;
    if (p.pid) {
        smin = last_row;
        for (int r = r0; r <= last_row; ++r) smin = min(smin, (long long)sample_start(r));
    }

    for (int i = threadIdx.x; i < kRows * D; i += blockDim.x) {
        const int rr = r0 + i / D;
        qs[i / D][i % D] =
            rr < p.L ? p.q[b * p.q_bstride + ((long long)rr * p.H_q + h) * D + i % D] : 0.f;
    }

    float m_run = -INFINITY, l_run = 0.f, o[NPL];
#pragma unroll
    for (int i = 0; i < NPL; ++i) o[i] = 0.f;

    const int i0 = r0 / p.Lc;  // rank owning the CTA's first query
    for (int s = 0; s < p.P; ++s) {
        const int j = ((i0 - s) % p.P + p.P) % p.P;
        // keys of chunk j at a position <= qmax: a prefix of the chunk (all if not causal)
        const int n_keys = p.causal ? (int)shard_prefix(p.zigzag, p.P, p.Lc, j, qmax) : p.Lc;
        // packed: keys of the chunk before the smallest sample start are skipped too
        const long long key0 = (long long)j * p.Lc;
        const int c_first = smin > key0 ? (int)min(smin - key0, (long long)p.Lc) / kKeys * kKeys : 0;
        if (n_keys <= c_first) continue;  // nothing in the chunk any row may see: skipped
        const float* kc = p.k[j] + b * p.kv_bstride;
        const float* vc = p.v[j] + b * p.kv_bstride;
        for (int c0 = c_first; c0 < n_keys; c0 += kKeys) {
            __syncthreads();  // previous tile fully consumed (and qs written, first time)
            for (int i = threadIdx.x; i < kKeys * D; i += blockDim.x) {
                const int c = i / D, d = i % D;
                const bool in = c0 + c < p.Lc;
                const long long off = ((long long)(c0 + c) * p.H_kv + g) * D + d;
                ks[c][d] = in ? kc[off] : 0.f;
                vs[c][d] = in ? vc[off] : 0.f;
            }
            __syncthreads();
            const long long kpos = shard_pos(p.zigzag, p.P, p.Lc, j, c0 + lane);
            const bool vis = active && (c0 + lane < n_keys) && (!p.causal || kpos <= my_pos) &&
                             kpos >= my_start;
            float sc = -INFINITY;
            if (vis) {
                float dot = 0.f;
#pragma unroll 8
                for (int d = 0; d < D; ++d) dot = fmaf(qs[warp][d], ks[lane][d], dot);
                sc = p.scale * dot;
            }
            float mt = sc;
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) mt = fmaxf(mt, __shfl_xor_sync(0xffffffffu, mt, off));
            const float m_new = fmaxf(m_run, mt);
            if (m_new == -INFINITY) continue;  // nothing visible yet for this row
            const float alpha = expf(m_run - m_new);  // 0 when m_run is -inf
            const float pr = vis ? expf(sc - m_new) : 0.f;
            float ps = pr;
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) ps += __shfl_xor_sync(0xffffffffu, ps, off);
            l_run = l_run * alpha + ps;
#pragma unroll
            for (int i = 0; i < NPL; ++i) o[i] *= alpha;
#pragma unroll 4
            for (int c = 0; c < kKeys; ++c) {
                const float pc = __shfl_sync(0xffffffffu, pr, c);
#pragma unroll
                for (int i = 0; i < NPL; ++i) o[i] = fmaf(pc, vs[c][lane + 32 * i], o[i]);
            }
            m_run = m_new;
        }
    }
    if (active) {
        const float inv = 1.f / l_run;
        float* dst = p.out + ((long long)b * p.L + row) * p.H_q * D + (long long)h * D;
#pragma unroll
        for (int i = 0; i < NPL; ++i) dst[lane + 32 * i] = o[i] * inv;
        if (lane == 0) p.lse[((long long)b * p.H_q + h) * p.L + row] = m_run + logf(l_run);
    }
}

}  // namespace

cudaError_t launch_attn_fp32(const AttnArgs& a) {
    Fp32Params p;
    p.q = (const float*)a.q;
    for (int j = 0; j < a.P; ++j) {
        p.k[j] = (const float*)a.k_chunks[j];
        p.v[j] = (const float*)a.v_chunks[j];
    }
    p.out = (float*)a.out;
    p.lse = a.lse;
    p.q_bstride = a.q_bstride;
    p.kv_bstride = a.kv_bstride;
    p.P = a.P;
    p.B = a.B;
    p.H_q = a.H_q;
    p.H_kv = a.H_kv;
    p.Lc = a.Lc;
    p.L = a.P * a.Lc;
    p.causal = a.causal;
    p.zigzag = a.zigzag;
    p.pid = a.pid;
    p.scale = a.scale;
    dim3 grid((p.L + kRows - 1) / kRows, a.B * a.H_q);
    switch (a.D) {
        case 32: attn_fwd_fp32<32><<<grid, kRows * 32, 0, a.stream>>>(p); break;
        case 64: attn_fwd_fp32<64><<<grid, kRows * 32, 0, a.stream>>>(p); break;
        case 128: attn_fwd_fp32<128><<<grid, kRows * 32, 0, a.stream>>>(p); break;
        default: return cudaErrorInvalidValue;
    }
    return cudaGetLastError();
}

}  // namespace ra
