// bwd_static.cu -- ra_ring_attn_bwd_static: the backward pass with its Delta scratch in a
// fixed file-scope device array instead of a caller-provided workspace, so that a call makes
// no device allocation of any kind.  Every call looks the array's address up in the current
// context with cudaGetSymbolAddress (a host-side lookup once the module is loaded; nothing
// is cached, so a context torn down and made again -- cudaDeviceReset -- gives the new
// module's address, never a stale one) and forwards to ra_ring_attn_bwd, whose validation
// and kernels are used unchanged.
//
// Nothing in the scratch has to start at zero: the Delta kernel writes every row that the
// gradient kernel reads, earlier on the same stream.  The one array is shared by every
// call on a device, so calls that overlap in time (different streams, or different host
// threads without ordering) race on it.
#include <cuda_runtime.h>
#include <string>
#include "ra_internal.h"
#include "../../include/ra.h"

namespace {

constexpr long long kMaxRows = RA_BWD_STATIC_MAX_ROWS;

static __device__ __align__(256) float g_bwd_scratch[RA_BWD_STATIC_MAX_ROWS];

// B * H_q * P * Lc, or -1 once the running product passes kMaxRows (each factor is >= 1
// and < 2^31, so no intermediate product exceeds 2^52).
long long rows_or_over(int B, int H_q, int P, int Lc) {
    long long r = 1;
    for (long long f : {(long long)B, (long long)H_q, (long long)P, (long long)Lc}) {
        r *= f;
        if (r > kMaxRows) return -1;
    }
    return r;
}

}  // namespace

extern "C" ra_status ra_ring_attn_bwd_static(
    const void* q, const void* const* k_chunks, const void* const* v_chunks, const void* out,
    const float* lse, const void* dout, int P, int B, int H_q, int H_kv, int Lc, int D,
    long long q_bstride, long long kv_bstride, float scale, int causal, float* dq,
    float* const* dk_chunks, float* const* dv_chunks, void* stream) {
    if (B < 1 || H_q < 1 || P < 1 || Lc < 1)
        return (ra_status)ra::set_last_error(RA_ERR_INVALID, "B, H_q, P and Lc must be >= 1");
    if (rows_or_over(B, H_q, P, Lc) < 0)
        return (ra_status)ra::set_last_error(
            RA_ERR_INVALID,
            "B*H_q*P*Lc exceeds the static backward scratch (RA_BWD_STATIC_MAX_ROWS = " +
                std::to_string(kMaxRows) + " rows, " + std::to_string(kMaxRows * 4 >> 20) +
                " MiB); use ra_ring_attn_bwd with a caller-provided workspace");
    // the address in the context that is current now, looked up on every call
    void* p = nullptr;
    cudaError_t e = cudaGetSymbolAddress(&p, g_bwd_scratch);
    if (e != cudaSuccess || !p)
        return (ra_status)ra::set_last_error(
            RA_ERR_CUDA, std::string("cudaGetSymbolAddress of the backward scratch: ") +
                             cudaGetErrorName(e));
    float* scratch = static_cast<float*>(p);
    return ra_ring_attn_bwd(q, k_chunks, v_chunks, out, lse, dout, P, B, H_q, H_kv, Lc, D,
                            q_bstride, kv_bstride, scale, causal, dq, dk_chunks, dv_chunks,
                            scratch, stream);
}
