// ra_internal.h -- launchers shared between the kernel translation units and the API
// layer (api.cu).  Arguments are validated by the API layer before these are called.
#pragma once
#include <cuda_runtime.h>
#include <cstdint>

namespace ra {

// Runtime divisor for 32-bit unsigned division by an invariant integer (Granlund &
// Montgomery, "Division by invariant integers using multiplication", PLDI 1994, the
// round-up multiplier with one extra add): q = (umulhi(n, mul) + n) >> shift.
struct FastDiv {
    uint32_t div, mul, shift;
};
inline FastDiv make_fastdiv(uint32_t d) {
    FastDiv f;
    f.div = d;
    uint32_t s = 0;
    while ((uint64_t(1) << s) < d) ++s;
    f.shift = s;
    // mul = floor(2^32 * (2^s - d) / d) + 1, which fits in 32 bits for every d >= 1.
    f.mul = (uint32_t)(((uint64_t(1) << 32) * ((uint64_t(1) << s) - d)) / d + 1);
    return f;
}

struct AttnArgs {
    const void* q;
    const void* const* k_chunks;  // host array, P entries
    const void* const* v_chunks;
    int P, B, H_q, H_kv, Lc, D;
    long long q_bstride, kv_bstride;  // elements
    float scale;
    int causal;
    int out_bf16;
    void* out;
    float* lse;
    cudaStream_t stream;
};

// Tensor-core (tcgen05) attention for bf16 inputs, D in {64, 128}.
cudaError_t launch_attn_sm100(const AttnArgs& a, unsigned long long wait_limit_ns,
                              int inject_stall, const char** why);
// CUDA-core fp32 attention, D in {32, 64, 128}.
cudaError_t launch_attn_fp32(const AttnArgs& a);
cudaError_t launch_lse_merge(float* o_a, float* lse_a, const float* o_b, const float* lse_b, int B,
                             int H, long long L, int D, cudaStream_t s);
cudaError_t launch_seq2head(const void* in, void* out, int P, int B, int Lc, int H_in, int H_out,
                            int D, int esize, cudaStream_t s, unsigned long long wait_limit_ns);
cudaError_t launch_head2seq(const void* in, void* out, int P, int B, int Lc, int H, int D,
                            int esize, cudaStream_t s, unsigned long long wait_limit_ns);
// Read and clear the per-device kernel error word (after the caller synchronised).
cudaError_t read_and_clear_error_word(unsigned int* value);
cudaError_t read_and_clear_permute_error(unsigned int* value);

}  // namespace ra
