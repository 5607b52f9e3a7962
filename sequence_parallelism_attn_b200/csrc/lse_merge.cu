// lse_merge.cu -- the merge of two partial attention results over disjoint key sets,
// "Как работает sequence parallelism в контексте LLM?", section 5 (the online-softmax
// merge of the ring loop), taken as the exact log-sum-exp combination:
//   lse = log(e^lse_a + e^lse_b);  o = e^(lse_a - lse) o_a + e^(lse_b - lse) o_b
// with (anything, -inf) as the empty partial.  In place into (o_a, lse_a).
//
// HBM-bound: per row 3*D*4 bytes of O (read a, read b, write a) + 12 bytes of LSE.
// A row is handled by TPR threads of one warp (TPR = the power of two >= D/4, at most
// 32), each moving float4s; every thread of a row reads both LSEs before the row's
// first thread overwrites lse_a, separated by __syncwarp, so the in-place update has no
// race.  The grid is one wave of 256-thread blocks (a multiple of the SM count) and strides
// over rows.
#include "ra_internal.h"
#include "permute_index.cuh"
#include <cmath>

namespace ra {
namespace {

// Two rows per warp slot per iteration, and every load of both rows (the two LSEs and the
// first float4 of O_a and O_b) issued before any arithmetic: the row's addresses do not
// depend on the LSE values, so a warp keeps four independent loads per lane in flight
// instead of waiting for the LSEs before it asks for O.
// FAST: every row index fits in 32 bits, so the row's (b, h, t) come from two
// invariant-divisor multiplications (by L, then by H) instead of 64-bit divisions, which
// would cost more instructions per row than the row's loads and stores.
template <bool FAST>
__global__ void __launch_bounds__(256) lse_merge_kernel(float* __restrict__ o_a,
                                                        float* __restrict__ lse_a,
                                                        const float* __restrict__ o_b,
                                                        const float* __restrict__ lse_b,
                                                        int B, int H, long long L, int D,
                                                        int tpr_log2, FastDiv fH, FastDiv fL) {
    const int tpr = 1 << tpr_log2;
    const int rows_per_warp = 32 >> tpr_log2;
    const int lane = threadIdx.x & 31;
    const int sub = lane >> tpr_log2;         // row slot within the warp
    const int li = lane & (tpr - 1);          // thread within the row
    const long long n_rows = (long long)B * L * H;
    const long long warp_global = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const long long n_warps = ((long long)gridDim.x * blockDim.x) >> 5;
    const long long step = n_warps * rows_per_warp;  // rows between a warp's two rows
    const int D4 = D >> 2;
    const bool has_c = li < D4;  // this lane owns float4 li of each row
    // Every lane of the warp runs the same number of iterations so that __syncwarp is legal.
    for (long long base = warp_global * rows_per_warp; base < n_rows; base += 2 * step) {
        long long orow[2], li_idx[2] = {0, 0};
        bool active[2];
        float la[2] = {-INFINITY, -INFINITY}, lb[2] = {-INFINITY, -INFINITY};
        float4 x[2], y[2];
#pragma unroll
        for (int u = 0; u < 2; ++u) {
            // rows in LSE order [B][H][L]: neighbouring warps read and write neighbouring
            // LSE entries (one 32-byte sector serves eight rows), while each row of O is one
            // contiguous D-float segment of the [B][L][H][D] tensor
            li_idx[u] = base + u * step + sub;
            active[u] = li_idx[u] < n_rows;
            orow[u] = 0;
            if (active[u]) {
                long long h, t, b;
                if (FAST) {
                    const uint32_t r = (uint32_t)li_idx[u];
                    const uint32_t bh = fdiv(r, fL);  // b * H + h
                    const uint32_t bb = fdiv(bh, fH);
                    t = r - bh * (uint32_t)L;
                    h = bh - bb * (uint32_t)H;
                    b = bb;
                } else {
                    t = li_idx[u] % L;
                    h = (li_idx[u] / L) % H;
                    b = li_idx[u] / L / H;
                }
                orow[u] = (b * L + t) * H + h;
                la[u] = lse_a[li_idx[u]];
                lb[u] = lse_b[li_idx[u]];
                if (has_c) {
                    x[u] = reinterpret_cast<const float4*>(o_a + orow[u] * D)[li];
                    y[u] = __ldg(reinterpret_cast<const float4*>(o_b + orow[u] * D) + li);
                }
            }
        }
        __syncwarp();
#pragma unroll
        for (int u = 0; u < 2; ++u) {
            const float m = fmaxf(la[u], lb[u]);
            float wa = 0.f, wb = 0.f, lse = -INFINITY;
            if (m != -INFINITY) {
                const float ea = expf(la[u] - m), eb = expf(lb[u] - m);
                const float z = ea + eb;
                lse = m + logf(z);
                wa = ea / z;
                wb = eb / z;
            }
            if (active[u]) {
                float4* pa = reinterpret_cast<float4*>(o_a + orow[u] * D);
                const float4* pb = reinterpret_cast<const float4*>(o_b + orow[u] * D);
                if (has_c)
                    pa[li] = make_float4(wa * x[u].x + wb * y[u].x, wa * x[u].y + wb * y[u].y,
                                         wa * x[u].z + wb * y[u].z, wa * x[u].w + wb * y[u].w);
                for (int c = li + tpr; c < D4; c += tpr) {  // rows wider than 32 float4s
                    const float4 xc = pa[c], yc = __ldg(pb + c);
                    pa[c] = make_float4(wa * xc.x + wb * yc.x, wa * xc.y + wb * yc.y,
                                        wa * xc.z + wb * yc.z, wa * xc.w + wb * yc.w);
                }
                if (li == 0) lse_a[li_idx[u]] = lse;
            }
        }
    }
}

// Blocks of one full wave: SMs x resident 256-thread blocks per SM.
int wave_blocks_merge() {
    static int n = 0;
    if (n == 0) {
        int dev = 0, sms = 0, per_sm = 0;
        if (cudaGetDevice(&dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
            sms <= 0)
            sms = 148;
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, lse_merge_kernel<true>, 256, 0) !=
                cudaSuccess ||
            per_sm <= 0)
            per_sm = 4;
        n = sms * per_sm;
    }
    return n;
}

}  // namespace

cudaError_t launch_lse_merge(float* o_a, float* lse_a, const float* o_b, const float* lse_b, int B,
                             int H, long long L, int D, cudaStream_t s) {
    int tpr_log2 = 0;
    while ((1 << tpr_log2) < D / 4 && tpr_log2 < 5) ++tpr_log2;
    const long long n_rows = (long long)B * L * H;
    const long long rows_per_block = (256 / 32) * (32 >> tpr_log2);
    long long blocks = (n_rows + rows_per_block - 1) / rows_per_block;
    const long long cap = wave_blocks_merge();
    if (blocks > cap) blocks = cap;
    if (blocks < 1) blocks = 1;
    const FastDiv fH = make_fastdiv((uint32_t)H);
    const bool fast = n_rows <= 0xffffffffLL && L <= 0xffffffffLL;
    const FastDiv fL = make_fastdiv(fast ? (uint32_t)L : 1u);
    if (fast)
        lse_merge_kernel<true><<<(unsigned)blocks, 256, 0, s>>>(o_a, lse_a, o_b, lse_b, B, H, L,
                                                                 D, tpr_log2, fH, fL);
    else
        lse_merge_kernel<false><<<(unsigned)blocks, 256, 0, s>>>(o_a, lse_a, o_b, lse_b, B, H, L,
                                                                  D, tpr_log2, fH, fL);
    return cudaGetLastError();
}

}  // namespace ra
