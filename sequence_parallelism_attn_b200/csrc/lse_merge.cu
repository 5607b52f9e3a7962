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
// race.  The grid is a multiple of the SM count and strides over rows.
#include "ra_internal.h"
#include <cmath>

namespace ra {
namespace {

__global__ void __launch_bounds__(256) lse_merge_kernel(float* __restrict__ o_a,
                                                        float* __restrict__ lse_a,
                                                        const float* __restrict__ o_b,
                                                        const float* __restrict__ lse_b,
                                                        int B, int H, long long L, int D,
                                                        int tpr_log2) {
    const int tpr = 1 << tpr_log2;
    const int rows_per_warp = 32 >> tpr_log2;
    const int lane = threadIdx.x & 31;
    const int sub = lane >> tpr_log2;         // row slot within the warp
    const int li = lane & (tpr - 1);          // thread within the row
    const long long n_rows = (long long)B * L * H;
    const long long warp_global = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const long long n_warps = ((long long)gridDim.x * blockDim.x) >> 5;
    const int D4 = D >> 2;
    // Every lane of the warp runs the same number of iterations so that __syncwarp is legal.
    for (long long base = warp_global * rows_per_warp; base < n_rows;
         base += n_warps * rows_per_warp) {
        const long long row = base + sub;  // row in [B][L][H] order
        const bool active = row < n_rows;
        long long li_idx = 0;
        float la = -INFINITY, lb = -INFINITY;
        if (active) {
            const long long h = row % H;
            const long long t = (row / H) % L;
            const long long b = row / H / L;
            li_idx = (b * H + h) * L + t;
            la = lse_a[li_idx];
            lb = lse_b[li_idx];
        }
        __syncwarp();
        const float m = fmaxf(la, lb);
        float wa = 0.f, wb = 0.f, lse = -INFINITY;
        if (m != -INFINITY) {
            const float ea = expf(la - m), eb = expf(lb - m);
            const float z = ea + eb;
            lse = m + logf(z);
            wa = ea / z;
            wb = eb / z;
        }
        if (active) {
            float4* pa = reinterpret_cast<float4*>(o_a + row * D);
            const float4* pb = reinterpret_cast<const float4*>(o_b + row * D);
            for (int c = li; c < D4; c += tpr) {
                const float4 x = pa[c], y = __ldg(pb + c);
                float4 r;
                r.x = wa * x.x + wb * y.x;
                r.y = wa * x.y + wb * y.y;
                r.z = wa * x.z + wb * y.z;
                r.w = wa * x.w + wb * y.w;
                pa[c] = r;
            }
            if (li == 0) lse_a[li_idx] = lse;
        }
    }
}

int sm_count_merge() {
    static int n = 0;
    if (n == 0) {
        int dev = 0;
        if (cudaGetDevice(&dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
            n = 148;
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
    const long long cap = (long long)sm_count_merge() * 8 * 4;
    if (blocks > cap) blocks = cap;
    if (blocks < 1) blocks = 1;
    lse_merge_kernel<<<(unsigned)blocks, 256, 0, s>>>(o_a, lse_a, o_b, lse_b, B, H, L, D, tpr_log2);
    return cudaGetLastError();
}

}  // namespace ra
