// api.cu -- the C ABI of include/ra.h: argument validation, dispatch to the kernels,
// status codes and thread-local error messages.  Nothing is launched unless every
// argument check passes.
#include <cuda_runtime.h>
#include <atomic>
#include <cmath>
#include <cstdint>
#include <cstdio>
#include <string>
#include "ra_internal.h"
#include "../../include/ra.h"

namespace {

thread_local std::string g_last_error;
thread_local int g_inject_stall = 0;
constexpr unsigned long long kDefaultWaitLimitNs = 4000000000ull;
std::atomic<unsigned long long> g_wait_limit_ns{kDefaultWaitLimitNs};
std::atomic<int> g_bwd_deterministic{0};

ra_status fail(ra_status s, const std::string& msg) {
    g_last_error = msg;
    return s;
}

ra_status cuda_fail(cudaError_t e, const char* what) {
    g_last_error = std::string(what) + ": " + cudaGetErrorName(e) + " (" + cudaGetErrorString(e) + ")";
    return RA_ERR_CUDA;
}

bool aligned16(const void* p) { return p && (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int elem_size(ra_dtype d) { return d == RA_BF16 ? 2 : (d == RA_FP32 ? 4 : 0); }

}  // namespace

namespace ra {
int set_last_error(int status, const std::string& msg) { return (int)fail((ra_status)status, msg); }
}  // namespace ra

extern "C" {

static ra_status ring_attn(const void* q, const void* const* k_chunks, const void* const* v_chunks,
                           int P, int B, int H_q, int H_kv, int Lc, int D, long long q_bstride,
                           long long kv_bstride, float scale, int causal, ra_dtype in_dtype,
                           ra_dtype out_dtype, void* out, float* lse, void* stream, int zigzag,
                           const int* position_ids) {
    if (P < 1 || P > RA_MAX_P) return fail(RA_ERR_INVALID, "P must be in [1, RA_MAX_P]");
    if (B < 1 || H_q < 1 || H_kv < 1 || Lc < 1 || D < 1)
        return fail(RA_ERR_INVALID, "B, H_q, H_kv, Lc and D must be >= 1");
    if (H_q % H_kv != 0) return fail(RA_ERR_INVALID, "H_q must be a multiple of H_kv");
    if (zigzag && Lc % 2 != 0)
        return fail(RA_ERR_INVALID, "the zigzag layout needs an even chunk length Lc");
    if (position_ids && (reinterpret_cast<uintptr_t>(position_ids) & 3u) != 0)
        return fail(RA_ERR_INVALID, "position_ids must be 4-byte aligned");
    if (causal != 0 && causal != 1) return fail(RA_ERR_INVALID, "causal must be 0 or 1");
    if (!(scale > 0.f) || !std::isfinite(scale))
        return fail(RA_ERR_INVALID, "scale must be finite and > 0");
    if (in_dtype != RA_BF16 && in_dtype != RA_FP32) return fail(RA_ERR_INVALID, "bad in_dtype");
    if (out_dtype != RA_BF16 && out_dtype != RA_FP32) return fail(RA_ERR_INVALID, "bad out_dtype");
    if (in_dtype == RA_FP32 && out_dtype != RA_FP32)
        return fail(RA_ERR_INVALID, "fp32 input requires fp32 output");
    if (in_dtype == RA_BF16 && D != 64 && D != 128)
        return fail(RA_ERR_UNSUPPORTED, "bf16 tensor-core path supports D in {64, 128}");
    if (in_dtype == RA_FP32 && D != 32 && D != 64 && D != 128)
        return fail(RA_ERR_UNSUPPORTED, "fp32 path supports D in {32, 64, 128}");
    const long long L = (long long)P * Lc;
    if (L > (1ll << 30)) return fail(RA_ERR_INVALID, "P*Lc must be <= 2^30");
    if (q_bstride < L * H_q * D) return fail(RA_ERR_INVALID, "q_bstride below the dense size");
    if (kv_bstride < (long long)Lc * H_kv * D)
        return fail(RA_ERR_INVALID, "kv_bstride below the dense size");
    const int es = elem_size(in_dtype);
    if ((q_bstride * es) % 16 != 0 || (kv_bstride * es) % 16 != 0)
        return fail(RA_ERR_INVALID, "batch strides must be multiples of 16 bytes");
    if (!aligned16(q) || !aligned16(out) || !aligned16(lse))
        return fail(RA_ERR_INVALID, "q, out and lse must be non-null and 16-byte aligned");
    if (!k_chunks || !v_chunks) return fail(RA_ERR_INVALID, "k_chunks/v_chunks must be non-null");
    for (int j = 0; j < P; ++j)
        if (!aligned16(k_chunks[j]) || !aligned16(v_chunks[j]))
            return fail(RA_ERR_INVALID, "every K/V chunk pointer must be non-null and 16-byte aligned");
    if (in_dtype == RA_FP32 && (long long)B * H_q > 65535)
        return fail(RA_ERR_UNSUPPORTED, "fp32 path supports B*H_q <= 65535");

    ra::AttnArgs a;
    a.q = q;
    a.k_chunks = k_chunks;
    a.v_chunks = v_chunks;
    a.P = P;
    a.B = B;
    a.H_q = H_q;
    a.H_kv = H_kv;
    a.Lc = Lc;
    a.D = D;
    a.q_bstride = q_bstride;
    a.kv_bstride = kv_bstride;
    a.scale = scale;
    a.causal = causal;
    a.zigzag = zigzag;
    a.pid = position_ids;
    a.out_bf16 = out_dtype == RA_BF16;
    a.out = out;
    a.lse = lse;
    a.stream = (cudaStream_t)stream;
    cudaError_t e;
    if (in_dtype == RA_BF16) {
        const char* why = "launch failed";
        const int stall = g_inject_stall;
        g_inject_stall = 0;
        e = ra::launch_attn_sm100(a, g_wait_limit_ns.load(), stall, &why);
        if (e != cudaSuccess) return cuda_fail(e, why);
    } else {
        e = ra::launch_attn_fp32(a);
        if (e != cudaSuccess) return cuda_fail(e, "fp32 attention launch");
    }
    return RA_OK;
}

ra_status ra_ring_attn_fwd(const void* q, const void* const* k_chunks, const void* const* v_chunks,
                           int P, int B, int H_q, int H_kv, int Lc, int D, long long q_bstride,
                           long long kv_bstride, float scale, int causal, ra_dtype in_dtype,
                           ra_dtype out_dtype, void* out, float* lse, void* stream) {
    return ring_attn(q, k_chunks, v_chunks, P, B, H_q, H_kv, Lc, D, q_bstride, kv_bstride, scale,
                     causal, in_dtype, out_dtype, out, lse, stream, 0, nullptr);
}

ra_status ra_ring_attn_fwd_zigzag(const void* q, const void* const* k_chunks,
                                  const void* const* v_chunks, int P, int B, int H_q, int H_kv,
                                  int Lc, int D, long long q_bstride, long long kv_bstride,
                                  float scale, int causal, ra_dtype in_dtype, ra_dtype out_dtype,
                                  void* out, float* lse, void* stream) {
    return ring_attn(q, k_chunks, v_chunks, P, B, H_q, H_kv, Lc, D, q_bstride, kv_bstride, scale,
                     causal, in_dtype, out_dtype, out, lse, stream, 1, nullptr);
}

ra_status ra_ring_attn_fwd_packed(const void* q, const void* const* k_chunks,
                                  const void* const* v_chunks, const int* position_ids, int P,
                                  int B, int H_q, int H_kv, int Lc, int D, long long q_bstride,
                                  long long kv_bstride, float scale, ra_dtype in_dtype,
                                  ra_dtype out_dtype, void* out, float* lse, void* stream) {
    if (!position_ids) return fail(RA_ERR_INVALID, "position_ids must be non-null");
    return ring_attn(q, k_chunks, v_chunks, P, B, H_q, H_kv, Lc, D, q_bstride, kv_bstride, scale,
                     1, in_dtype, out_dtype, out, lse, stream, 0, position_ids);
}

static ra_status ring_attn_bwd(const void* q, const void* const* k_chunks,
                               const void* const* v_chunks, const void* out, const float* lse,
                               const void* dout, int P, int B, int H_q, int H_kv, int Lc, int D,
                               long long q_bstride, long long kv_bstride, float scale, int causal,
                               float* dq, float* const* dk_chunks, float* const* dv_chunks,
                               float* workspace, void* stream, int zigzag,
                               const int* position_ids, int accumulate = 0) {
    if (P < 1 || P > RA_MAX_P) return fail(RA_ERR_INVALID, "P must be in [1, RA_MAX_P]");
    if (zigzag && Lc % 2 != 0)
        return fail(RA_ERR_INVALID, "the zigzag layout needs an even chunk length Lc");
    if (position_ids && (reinterpret_cast<uintptr_t>(position_ids) & 3u) != 0)
        return fail(RA_ERR_INVALID, "position_ids must be 4-byte aligned");
    if (B < 1 || H_q < 1 || H_kv < 1 || Lc < 1 || D < 1)
        return fail(RA_ERR_INVALID, "B, H_q, H_kv, Lc and D must be >= 1");
    if (H_q % H_kv != 0) return fail(RA_ERR_INVALID, "H_q must be a multiple of H_kv");
    if (causal != 0 && causal != 1) return fail(RA_ERR_INVALID, "causal must be 0 or 1");
    if (!(scale > 0.f) || !std::isfinite(scale))
        return fail(RA_ERR_INVALID, "scale must be finite and > 0");
    if (D != 64 && D != 128)
        return fail(RA_ERR_UNSUPPORTED, "the tensor-core backward supports D in {64, 128}");
    const long long L = (long long)P * Lc;
    if (L > (1ll << 30)) return fail(RA_ERR_INVALID, "P*Lc must be <= 2^30");
    if (q_bstride < L * H_q * D) return fail(RA_ERR_INVALID, "q_bstride below the dense size");
    if (kv_bstride < (long long)Lc * H_kv * D)
        return fail(RA_ERR_INVALID, "kv_bstride below the dense size");
    if ((q_bstride * 2) % 16 != 0 || (kv_bstride * 2) % 16 != 0)
        return fail(RA_ERR_INVALID, "batch strides must be multiples of 16 bytes");
    if (!aligned16(q) || !aligned16(out) || !aligned16(lse) || !aligned16(dout) ||
        !aligned16(dq) || !aligned16(workspace))
        return fail(RA_ERR_INVALID, "q, out, lse, dout, dq and workspace must be non-null and "
                                    "16-byte aligned");
    if (!k_chunks || !v_chunks || !dk_chunks || !dv_chunks)
        return fail(RA_ERR_INVALID, "chunk pointer arrays must be non-null");
    for (int j = 0; j < P; ++j)
        if (!aligned16(k_chunks[j]) || !aligned16(v_chunks[j]) || !aligned16(dk_chunks[j]) ||
            !aligned16(dv_chunks[j]))
            return fail(RA_ERR_INVALID, "every chunk pointer must be non-null and 16-byte aligned");
    ra::AttnBwdArgs a;
    a.q = q;
    a.k_chunks = k_chunks;
    a.v_chunks = v_chunks;
    a.out = out;
    a.lse = lse;
    a.dout = dout;
    a.P = P;
    a.B = B;
    a.H_q = H_q;
    a.H_kv = H_kv;
    a.Lc = Lc;
    a.D = D;
    a.q_bstride = q_bstride;
    a.kv_bstride = kv_bstride;
    a.scale = scale;
    a.causal = causal;
    a.dq = dq;
    a.dk_chunks = dk_chunks;
    a.dv_chunks = dv_chunks;
    a.workspace = workspace;
    a.zigzag = zigzag;
    a.pid = position_ids;
    a.accumulate = accumulate;
    a.deterministic = g_bwd_deterministic.load();
    a.stream = (cudaStream_t)stream;
    const char* why = "launch failed";
    cudaError_t e = ra::launch_attn_bwd_sm100(a, g_wait_limit_ns.load(), &why);
    if (e != cudaSuccess) return cuda_fail(e, why);
    return RA_OK;
}

ra_status ra_ring_attn_bwd(const void* q, const void* const* k_chunks, const void* const* v_chunks,
                           const void* out, const float* lse, const void* dout, int P, int B,
                           int H_q, int H_kv, int Lc, int D, long long q_bstride,
                           long long kv_bstride, float scale, int causal, float* dq,
                           float* const* dk_chunks, float* const* dv_chunks, float* workspace,
                           void* stream) {
    return ring_attn_bwd(q, k_chunks, v_chunks, out, lse, dout, P, B, H_q, H_kv, Lc, D, q_bstride,
                         kv_bstride, scale, causal, dq, dk_chunks, dv_chunks, workspace, stream, 0,
                         nullptr);
}

ra_status ra_ring_attn_bwd_accumulate(const void* q, const void* const* k_chunks,
                                      const void* const* v_chunks, const void* out,
                                      const float* lse, const void* dout, int P, int B, int H_q,
                                      int H_kv, int Lc, int D, long long q_bstride,
                                      long long kv_bstride, float scale, int causal, float* dq,
                                      float* const* dk_chunks, float* const* dv_chunks,
                                      float* workspace, void* stream) {
    return ring_attn_bwd(q, k_chunks, v_chunks, out, lse, dout, P, B, H_q, H_kv, Lc, D, q_bstride,
                         kv_bstride, scale, causal, dq, dk_chunks, dv_chunks, workspace, stream, 0,
                         nullptr, 1);
}

ra_status ra_ring_attn_bwd_zigzag(const void* q, const void* const* k_chunks,
                                  const void* const* v_chunks, const void* out, const float* lse,
                                  const void* dout, int P, int B, int H_q, int H_kv, int Lc, int D,
                                  long long q_bstride, long long kv_bstride, float scale,
                                  int causal, float* dq, float* const* dk_chunks,
                                  float* const* dv_chunks, float* workspace, void* stream) {
    return ring_attn_bwd(q, k_chunks, v_chunks, out, lse, dout, P, B, H_q, H_kv, Lc, D, q_bstride,
                         kv_bstride, scale, causal, dq, dk_chunks, dv_chunks, workspace, stream, 1,
                         nullptr);
}

ra_status ra_ring_attn_bwd_packed(const void* q, const void* const* k_chunks,
                                  const void* const* v_chunks, const int* position_ids,
                                  const void* out, const float* lse, const void* dout, int P, int B,
                                  int H_q, int H_kv, int Lc, int D, long long q_bstride,
                                  long long kv_bstride, float scale, float* dq,
                                  float* const* dk_chunks, float* const* dv_chunks,
                                  float* workspace, void* stream) {
    if (!position_ids) return fail(RA_ERR_INVALID, "position_ids must be non-null");
    return ring_attn_bwd(q, k_chunks, v_chunks, out, lse, dout, P, B, H_q, H_kv, Lc, D, q_bstride,
                         kv_bstride, scale, 1, dq, dk_chunks, dv_chunks, workspace, stream, 0,
                         position_ids);
}

ra_status ra_lse_merge(float* o_a, float* lse_a, const float* o_b, const float* lse_b, int B, int H,
                       long long L, int D, void* stream) {
    if (B < 1 || H < 1 || L < 1 || D < 1) return fail(RA_ERR_INVALID, "sizes must be >= 1");
    if (D % 4 != 0) return fail(RA_ERR_UNSUPPORTED, "D must be a multiple of 4");
    if (!aligned16(o_a) || !aligned16(o_b) || !aligned16(lse_a) || !aligned16(lse_b))
        return fail(RA_ERR_INVALID, "pointers must be non-null and 16-byte aligned");
    if (o_a == o_b || lse_a == lse_b) return fail(RA_ERR_INVALID, "b must not alias a");
    cudaError_t e = ra::launch_lse_merge(o_a, lse_a, o_b, lse_b, B, H, L, D, (cudaStream_t)stream);
    if (e != cudaSuccess) return cuda_fail(e, "lse_merge launch");
    return RA_OK;
}

static ra_status check_permute(const void* in, const void* out, int P, int G, int B, int Lc,
                               int H_small, int H_big, int D, ra_dtype dt) {
    if (P < 1 || G < 1 || B < 1 || Lc < 1 || H_small < 1 || H_big < 1 || D < 1)
        return fail(RA_ERR_INVALID, "sizes must be >= 1");
    if (dt != RA_BF16 && dt != RA_FP32) return fail(RA_ERR_INVALID, "bad dtype");
    if (H_big % G != 0)
        return fail(RA_ERR_INVALID,
                    "head count must be divisible by the number of head groups (ranks P)");
    if (H_big % H_small != 0)
        return fail(RA_ERR_INVALID, "H_out must be a multiple of H_in");
    if ((D * elem_size(dt)) % 16 != 0)
        return fail(RA_ERR_INVALID, "D * element size must be a multiple of 16 bytes");
    if (!aligned16(in) || !aligned16(out))
        return fail(RA_ERR_INVALID, "pointers must be non-null and 16-byte aligned");
    if (in == out) return fail(RA_ERR_INVALID, "in and out must not alias");
    const unsigned long long vecs = (unsigned long long)P * B * P * (unsigned long long)Lc *
                                    (unsigned long long)H_big * D * elem_size(dt) / 16 / P;
    if (vecs >= (1ull << 32)) return fail(RA_ERR_UNSUPPORTED, "tensor larger than 64 GiB");
    return RA_OK;
}

ra_status ra_ulysses_seq2head_grouped(const void* in, void* out, int P, int G, int B, int Lc,
                                      int H_in, int H_out, int D, ra_dtype dt, void* stream) {
    ra_status s = check_permute(in, out, P, G, B, Lc, H_in, H_out, D, dt);
    if (s != RA_OK) return s;
    cudaError_t e = ra::launch_seq2head(in, out, P, G, B, Lc, H_in, H_out, D, elem_size(dt),
                                        (cudaStream_t)stream, g_wait_limit_ns.load());
    if (e != cudaSuccess) return cuda_fail(e, "seq2head launch");
    return RA_OK;
}

ra_status ra_ulysses_head2seq_grouped(const void* in, void* out, int P, int G, int B, int Lc,
                                      int H, int D, ra_dtype dt, void* stream) {
    ra_status s = check_permute(in, out, P, G, B, Lc, H, H, D, dt);
    if (s != RA_OK) return s;
    cudaError_t e = ra::launch_head2seq(in, out, P, G, B, Lc, H, D, elem_size(dt),
                                        (cudaStream_t)stream, g_wait_limit_ns.load());
    if (e != cudaSuccess) return cuda_fail(e, "head2seq launch");
    return RA_OK;
}

static ra_status ulysses_scatter(int mode, const void* in, void* const* dst, int P, int rank,
                                 int B, int Lc, int H_in, int H_out, int D, ra_dtype dt,
                                 void* stream) {
    if (P < 1 || P > RA_MAX_P) return fail(RA_ERR_INVALID, "P must be in [1, RA_MAX_P]");
    if (rank < 0 || rank >= P) return fail(RA_ERR_INVALID, "rank must be in [0, P)");
    if (!dst) return fail(RA_ERR_INVALID, "dst must be a host array of P device pointers");
    ra_status s = check_permute(in, dst[0], P, P, B, Lc, H_in, H_out, D, dt);
    if (s != RA_OK) return s;
    for (int r = 0; r < P; ++r) {
        if (!aligned16(dst[r]))
            return fail(RA_ERR_INVALID, "every dst pointer must be non-null and 16-byte aligned");
        if (dst[r] == in) return fail(RA_ERR_INVALID, "in and a dst buffer must not alias");
        for (int q = 0; q < r; ++q)
            if (dst[q] == dst[r]) return fail(RA_ERR_INVALID, "dst buffers must be distinct");
    }
    cudaError_t e = ra::launch_ulysses_scatter(mode, in, dst, P, rank, B, Lc, H_in, H_out, D,
                                               elem_size(dt), (cudaStream_t)stream);
    if (e != cudaSuccess) return cuda_fail(e, "Ulysses scatter launch");
    return RA_OK;
}

ra_status ra_ulysses_seq2head_scatter(const void* in, void* const* dst, int P, int rank, int B,
                                      int Lc, int H_in, int H_out, int D, ra_dtype dt,
                                      void* stream) {
    return ulysses_scatter(0, in, dst, P, rank, B, Lc, H_in, H_out, D, dt, stream);
}

ra_status ra_ulysses_head2seq_scatter(const void* in, void* const* dst, int P, int rank, int B,
                                      int Lc, int H, int D, ra_dtype dt, void* stream) {
    return ulysses_scatter(1, in, dst, P, rank, B, Lc, H, H, D, dt, stream);
}

ra_status ra_ulysses_replica_sum(const float* in, float* out, long long rows, int H_in, int H_out,
                                 int D, void* stream) {
    if (rows < 1 || H_in < 1 || H_out < 1 || D < 1)
        return fail(RA_ERR_INVALID, "sizes must be >= 1");
    if (H_in % H_out != 0) return fail(RA_ERR_INVALID, "H_in must be a multiple of H_out");
    if (D % 4 != 0) return fail(RA_ERR_INVALID, "D must be a multiple of 4 (16-byte rows)");
    if (!aligned16(in) || !aligned16(out))
        return fail(RA_ERR_INVALID, "pointers must be non-null and 16-byte aligned");
    if (static_cast<const void*>(in) == static_cast<const void*>(out))
        return fail(RA_ERR_INVALID, "in and out must not alias");
    cudaError_t e = ra::launch_replica_sum(in, out, rows, H_in, H_out, D, (cudaStream_t)stream);
    if (e != cudaSuccess) return cuda_fail(e, "replica sum launch");
    return RA_OK;
}

ra_status ra_ulysses_seq2head(const void* in, void* out, int P, int B, int Lc, int H_in, int H_out,
                              int D, ra_dtype dt, void* stream) {
    return ra_ulysses_seq2head_grouped(in, out, P, P, B, Lc, H_in, H_out, D, dt, stream);
}

ra_status ra_ulysses_head2seq(const void* in, void* out, int P, int B, int Lc, int H, int D,
                              ra_dtype dt, void* stream) {
    return ra_ulysses_head2seq_grouped(in, out, P, P, B, Lc, H, D, dt, stream);
}

ra_status ra_sync_status(void* stream) {
    cudaError_t e = cudaStreamSynchronize((cudaStream_t)stream);
    if (e != cudaSuccess) return cuda_fail(e, "stream synchronize");
    unsigned int word = 0, pword = 0, bword = 0;
    e = ra::read_and_clear_error_word(&word);
    if (e == cudaSuccess) e = ra::read_and_clear_permute_error(&pword);
    if (e == cudaSuccess) e = ra::read_and_clear_bwd_error(&bword);
    if (e != cudaSuccess) return cuda_fail(e, "reading the kernel error word");
    word |= (pword ? 16u : 0u) | (bword ? 64u : 0u);
    if (word) {
        char buf[128];
        std::snprintf(buf, sizeof buf,
                      "a kernel gave up on a bounded wait (error bits 0x%x: 1 load, 2 mma, "
                      "4 softmax, 8 drain, 16 permute, 64 backward)", word);
        return fail(RA_ERR_TIMEOUT, buf);
    }
    return RA_OK;
}

const char* ra_last_error(void) { return g_last_error.c_str(); }

unsigned long long ra_set_wait_limit_ns(unsigned long long ns) {
    return g_wait_limit_ns.exchange(ns ? ns : kDefaultWaitLimitNs);
}

void ra_debug_inject_stall(int on) { g_inject_stall = on ? 1 : 0; }

int ra_set_bwd_deterministic(int on) { return g_bwd_deterministic.exchange(on ? 1 : 0); }

const char* ra_version(void) { return "ra_b200 0.1 (sm_100a: tcgen05/TMEM/TMA attention)"; }

}  // extern "C"
