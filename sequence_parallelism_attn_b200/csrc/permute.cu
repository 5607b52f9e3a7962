// permute.cu -- the Ulysses layout transforms ("Метод контекстного параллелизма Ulysses"):
// sequence-sharded [P][B][Lc][H][D] <-> head-sharded [P][B][P*Lc][H/P][D], with the GQA
// copy of KV heads up to H_out.  Pure data movement; bit-exact by construction.
//
// Each thread moves U 16-byte vectors that lie inside one head's D elements, so the
// per-element index arithmetic is paid once per 16*U bytes; consecutive threads write
// consecutive output addresses (coalesced stores) and read whole head segments of the
// source (D * element size contiguous bytes).  The grid is a multiple of the SM count and
// strides over the output.  HBM-bound: algorithmic bytes = input read once per output
// byte that needs it + output written once.
#include "ra_internal.h"
#include "permute_index.cuh"

namespace ra {

namespace {

int g_sm_count = 0;

int sm_count() {
    if (g_sm_count == 0) {
        int dev = 0, n = 0;
        if (cudaGetDevice(&dev) == cudaSuccess &&
            cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess && n > 0)
            g_sm_count = n;
        else
            g_sm_count = 148;
    }
    return g_sm_count;
}

template <int U>
__global__ void __launch_bounds__(256) seq2head_kernel(const int4* __restrict__ in,
                                                       int4* __restrict__ out, uint32_t n_groups,
                                                       PermuteGeom geo) {
    const uint32_t stride = gridDim.x * blockDim.x;
    for (uint32_t g = blockIdx.x * blockDim.x + threadIdx.x; g < n_groups; g += stride) {
        const uint32_t vec = g * U;
        const uint64_t src = seq2head_src_vec(geo, vec);
        int4 v[U];
#pragma unroll
        for (int u = 0; u < U; ++u) v[u] = __ldg(in + src + u);
#pragma unroll
        for (int u = 0; u < U; ++u) out[(uint64_t)vec + u] = v[u];
    }
}

template <int U>
__global__ void __launch_bounds__(256) head2seq_kernel(const int4* __restrict__ in,
                                                       int4* __restrict__ out, uint32_t n_groups,
                                                       PermuteGeom geo) {
    const uint32_t stride = gridDim.x * blockDim.x;
    for (uint32_t g = blockIdx.x * blockDim.x + threadIdx.x; g < n_groups; g += stride) {
        const uint32_t vec = g * U;
        const uint64_t src = head2seq_src_vec(geo, vec);
        int4 v[U];
#pragma unroll
        for (int u = 0; u < U; ++u) v[u] = __ldg(in + src + u);
#pragma unroll
        for (int u = 0; u < U; ++u) out[(uint64_t)vec + u] = v[u];
    }
}

unsigned grid_for(uint32_t n_groups) {
    const uint32_t per_wave = (uint32_t)sm_count() * 8u;  // 8 resident 256-thread CTAs per SM
    uint32_t blocks = (n_groups + 255u) / 256u;
    if (blocks > per_wave * 4u) blocks = per_wave * 4u;
    return blocks ? blocks : 1u;
}

}  // namespace

cudaError_t launch_seq2head(const void* in, void* out, int P, int B, int Lc, int H_in, int H_out,
                            int D, int esize, cudaStream_t s) {
    PermuteGeom geo = make_seq2head_geom(P, B, Lc, H_in, H_out, D, esize);
    const uint64_t n_vec = (uint64_t)P * B * P * Lc * (uint64_t)(H_out / P) * geo.VD.div;
    if (geo.VD.div % 4 == 0) {
        const uint32_t n_groups = (uint32_t)(n_vec / 4);
        seq2head_kernel<4><<<grid_for(n_groups), 256, 0, s>>>((const int4*)in, (int4*)out,
                                                              n_groups, geo);
    } else {
        const uint32_t n_groups = (uint32_t)n_vec;
        seq2head_kernel<1><<<grid_for(n_groups), 256, 0, s>>>((const int4*)in, (int4*)out,
                                                              n_groups, geo);
    }
    return cudaGetLastError();
}

cudaError_t launch_head2seq(const void* in, void* out, int P, int B, int Lc, int H, int D,
                            int esize, cudaStream_t s) {
    PermuteGeom geo = make_head2seq_geom(P, B, Lc, H, D, esize);
    const uint64_t n_vec = (uint64_t)P * B * Lc * (uint64_t)H * geo.VD.div;
    if (geo.VD.div % 4 == 0) {
        const uint32_t n_groups = (uint32_t)(n_vec / 4);
        head2seq_kernel<4><<<grid_for(n_groups), 256, 0, s>>>((const int4*)in, (int4*)out,
                                                              n_groups, geo);
    } else {
        const uint32_t n_groups = (uint32_t)n_vec;
        head2seq_kernel<1><<<grid_for(n_groups), 256, 0, s>>>((const int4*)in, (int4*)out,
                                                              n_groups, geo);
    }
    return cudaGetLastError();
}

}  // namespace ra
