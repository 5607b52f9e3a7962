// ra_internal.h -- launchers shared between the kernel translation units and the API
// layer (api.cu).  Arguments are validated by the API layer before these are called.
#pragma once
#include <cuda_runtime.h>
#include <cstdint>
#include <string>

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
    int zigzag;  // shard layout: 0 contiguous, 1 zigzag (Lc even)
    const int* pid;  // packed samples: device position_ids [B][P*Lc] (nullptr: none)
    int out_bf16;
    void* out;
    float* lse;
    cudaStream_t stream;
};

// The backward pass: gradients of the forward's O given dO, with its LSE.
struct AttnBwdArgs {
    const void* q;                // [B][P*Lc][H_q][D] bf16, batch stride q_bstride
    const void* const* k_chunks;  // host array, P entries, [B][Lc][H_kv][D] bf16
    const void* const* v_chunks;
    const void* out;              // [B][P*Lc][H_q][D] bf16, dense (the forward's O)
    const float* lse;             // [B][H_q][P*Lc]
    const void* dout;             // [B][P*Lc][H_q][D] bf16, dense
    int P, B, H_q, H_kv, Lc, D;
    long long q_bstride, kv_bstride;
    float scale;
    int causal;
    float* dq;                    // [B][P*Lc][H_q][D] fp32, dense
    float* const* dk_chunks;      // host array, P entries, [B][Lc][H_kv][D] fp32, dense
    float* const* dv_chunks;
    float* workspace;             // [B][H_q][P*Lc] fp32 (rowsum(dO * O))
    int zigzag = 0;               // shards in the zigzag layout
    const int* pid = nullptr;     // packed samples: position_ids [B][P*Lc] (causal), else null
    int accumulate = 0;           // add into dq, dk, dv instead of overwriting them
    int deterministic = 0;        // dq from the query-stationary kernel (fixed order)
    cudaStream_t stream;
};

// ---- sequence positions of the shard layouts ("Как работает sequence parallelism в
// контексте LLM?", section 2: rank i owns the contiguous tokens i*Lc .. i*Lc+Lc-1; the
// zigzag layout, named beside the ring in "Метод контекстного параллелизма Ulysses",
// introduction: 2P segments of h = Lc/2 tokens, rank i holding segment i then segment
// 2P-1-i).  Within one shard positions increase with the local index in both layouts,
// which is what lets a causal schedule keep a prefix of each K/V chunk.

// Sequence position of local token u of rank j's shard.
__host__ __device__ inline long long shard_pos(int zigzag, int P, int Lc, int j, long long u) {
    if (!zigzag) return (long long)j * Lc + u;
    const long long h = Lc / 2;
    return u < h ? (long long)j * h + u : (2LL * P - 1 - j) * h + (u - h);
}

// Number of leading tokens of rank j's shard whose position is <= qmax (0 .. Lc).
__host__ __device__ inline long long shard_prefix(int zigzag, int P, int Lc, int j,
                                                  long long qmax) {
    long long n;
    if (!zigzag) {
        n = qmax - (long long)j * Lc + 1;
    } else {
        const long long h = Lc / 2;
        const long long lo = (long long)j * h, hi = (2LL * P - 1 - j) * h;
        n = qmax < hi ? qmax - lo + 1 : h + (qmax - hi + 1);
        if (qmax >= hi) n = n > Lc ? Lc : n;
        else n = n > h ? h : n;
    }
    return n < 0 ? 0 : (n > Lc ? Lc : n);
}

// Smallest and largest position among the rank-major rows a .. b (a <= b), one shard
// slice at a time (positions increase within a slice).
__host__ __device__ inline void row_pos_range(int zigzag, int P, int Lc, long long a, long long b,
                                              long long& pmin, long long& pmax) {
    if (!zigzag) {
        pmin = a;
        pmax = b;
        return;
    }
    pmin = shard_pos(1, P, Lc, (int)(a / Lc), a % Lc);
    pmax = pmin;
    for (long long r = a; r <= b;) {
        const int i = (int)(r / Lc);
        const long long t0 = r - (long long)i * Lc;
        const long long t1 = (b - r) < (Lc - 1 - t0) ? t0 + (b - r) : Lc - 1;
        const long long p0 = shard_pos(1, P, Lc, i, t0), p1 = shard_pos(1, P, Lc, i, t1);
        pmin = p0 < pmin ? p0 : pmin;
        pmax = p1 > pmax ? p1 : pmax;
        r += t1 - t0 + 1;
    }
}

// Sample start of row r of one batch row of packed samples ("Paralelismo de secuencias en
// 🤗 accelerate", section "Configuración del backend SP de ALST/Ulysses"): r minus its
// position_ids entry, clamped to [0, r].
__host__ __device__ inline int sample_start(const int* pid_row, int r) {
    const int st = r - pid_row[r];
    return st < 0 ? 0 : (st > r ? r : st);
}

// The query tiles (of `tile` rows, rank-major) whose rows may see a key of the key tile
// (chunk j, local keys key0 .. key0 + kvalid - 1), as ascending disjoint ranges
// [qr_lo[i], qr_hi[i]) of tile indices (at most 2 P).  Returns the number of ranges and
// sets *n_tiles to the tiles they hold.  layout: 1 zigzag, 2 packed (pid_row: the batch
// row's position_ids).  Not causal: every tile.  Zigzag, causal: rows at a position >= the
// key tile's first position, a suffix of every half-shard.  Packed (causal): rows from the
// tile's first key to the last row whose sample starts at or before its last key (sample
// starts do not decrease along a row, so a binary search over tiles finds it).
__host__ __device__ inline int key_tile_q_ranges(int layout, int P, int Lc, int causal, int tile,
                                                 const int* pid_row, int j, int key0, int kvalid,
                                                 int* qr_lo, int* qr_hi, int* n_tiles) {
    const long long L = (long long)P * Lc;
    const int n_qt = (int)((L + tile - 1) / tile);
    int nr = 0;
    auto add_rows = [&](long long row_lo, long long row_hi) {  // rows [row_lo, row_hi)
        if (row_lo >= row_hi) return;
        const int lo = (int)(row_lo / tile), hi = (int)((row_hi - 1) / tile) + 1;
        if (nr > 0 && lo <= qr_hi[nr - 1]) {
            qr_hi[nr - 1] = qr_hi[nr - 1] > hi ? qr_hi[nr - 1] : hi;
        } else {
            qr_lo[nr] = lo;
            qr_hi[nr] = hi;
            ++nr;
        }
    };
    if (!causal) {
        add_rows(0, L);
    } else if (layout == 1) {
        const long long h = Lc / 2;
        const long long kmin = shard_pos(1, P, Lc, j, key0);
        for (int r = 0; r < P; ++r) {
            const long long base = (long long)r * Lc;
            const long long d1 = kmin - (long long)r * h;  // first half: positions r h + u
            const long long u1 = d1 > 0 ? d1 : 0;
            if (u1 < h) add_rows(base + u1, base + h);
            const long long d2 = kmin - (2LL * P - 1 - r) * h;
            const long long u2 = h + (d2 > 0 ? d2 : 0);
            if (u2 < Lc) add_rows(base + u2, base + Lc);
        }
    } else {
        const int k0 = j * Lc + key0, k_last = k0 + kvalid - 1;
        int lo = k0 / tile, hi = n_qt - 1;
        while (lo < hi) {
            const int mid = (lo + hi + 1) / 2;
            if (sample_start(pid_row, mid * tile) <= k_last) lo = mid;
            else hi = mid - 1;
        }
        add_rows((long long)(k0 / tile) * tile, (long long)(lo + 1) * tile);
    }
    int n = 0;
    for (int i = 0; i < nr; ++i) n += qr_hi[i] - qr_lo[i];
    *n_tiles = n;
    return nr;
}

// Tensor-core (tcgen05) attention for bf16 inputs, D in {64, 128}.
cudaError_t launch_attn_sm100(const AttnArgs& a, unsigned long long wait_limit_ns,
                              int inject_stall, const char** why);
// CUDA-core fp32 attention, D in {32, 64, 128}.
cudaError_t launch_attn_fp32(const AttnArgs& a);
cudaError_t launch_lse_merge(float* o_a, float* lse_a, const float* o_b, const float* lse_b, int B,
                             int H, long long L, int D, cudaStream_t s);
// Ulysses transforms with G head groups (G = P: the Ulysses all-to-all).
cudaError_t launch_seq2head(const void* in, void* out, int P, int G, int B, int Lc, int H_in,
                            int H_out, int D, int esize, cudaStream_t s,
                            unsigned long long wait_limit_ns);
cudaError_t launch_replica_sum(const float* in, float* out, long long rows, int H_in, int H_out,
                               int D, cudaStream_t s);
cudaError_t launch_head2seq(const void* in, void* out, int P, int G, int B, int Lc, int H, int D,
                            int esize, cudaStream_t s, unsigned long long wait_limit_ns);
// One rank's share of the Ulysses all-to-all stored straight into the P destination buffers
// (mode 0: seq2head with the GQA copy H_in -> H_out; mode 1: head2seq, H_in = H_out = H).
cudaError_t launch_ulysses_scatter(int mode, const void* in, void* const* dst, int P, int me,
                                   int B, int Lc, int H_in, int H_out, int D, int esize,
                                   cudaStream_t s);
// Tensor-core backward for bf16 inputs, D in {64, 128}: Delta, dQ, then dK/dV.
cudaError_t launch_attn_bwd_sm100(const AttnBwdArgs& a, unsigned long long wait_limit_ns,
                                  const char** why);
cudaError_t read_and_clear_bwd_error(unsigned int* value);

// Records msg as the calling thread's ra_last_error() text and returns status (for entry
// points defined outside api.cu).
int set_last_error(int status, const std::string& msg);
// Read and clear the per-device kernel error word (after the caller synchronised).
cudaError_t read_and_clear_error_word(unsigned int* value);
cudaError_t read_and_clear_permute_error(unsigned int* value);

}  // namespace ra
