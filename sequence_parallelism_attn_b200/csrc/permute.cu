// permute.cu -- the Ulysses layout transforms ("Метод контекстного параллелизма Ulysses"):
// sequence-sharded [P][B][Lc][H][D] <-> head-sharded [G][B][P*Lc][H/G][D], with the GQA
// copy of KV heads up to H_out.  G = P is the Ulysses all-to-all; G < P head groups is the
// head split of the ring x Ulysses hybrid (every group receives all P shards' tokens and
// the ring runs over them).  Pure data movement; bit-exact by construction.
//
// Each thread moves U 16-byte vectors that lie inside one head's D elements, so the
// per-element index arithmetic is paid once per 16*U bytes; consecutive threads write
// consecutive output addresses (coalesced stores) and read whole head segments of the
// source (D * element size contiguous bytes).  The grid is a multiple of the SM count and
// strides over the output.  HBM-bound: algorithmic bytes = input read once per output
// byte that needs it + output written once.
#include <cuda.h>
#include <cudaTypedefs.h>
#include "ra_internal.h"
#include "permute_index.cuh"
#include "sm100_ptx.cuh"
#include "../../include/ra.h"

namespace ra {

__device__ unsigned int g_permute_error_word = 0;

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


// ---------------------------------------------------------------- TMA bulk-tensor path
// The sequence-sharded side is viewed as a 4-D tensor of 32-bit words
//   {W = D*elem/4, H, Lc, P*B}              (token t of rank s, batch b at (.., t, s*B + b))
// and the head-sharded side as a 5-D tensor
//   {W, Hl, Lc, P, G*B}                      (group r, batch b, global token s*Lc + t at
//                                             (.., t, s, r*B + b))
// so a box of T tokens never crosses a chunk boundary: loads past Lc read zeros and stores
// past Lc are clipped.  One thread per CTA runs a ring of NS shared-memory stages: a tiled
// TMA load fills a stage, a tiled TMA store drains it, and a stage is refilled once the
// store that read it is done.  Each thread issues a handful of instructions per 32 KB.
constexpr int kPermStages = 3;
constexpr int kPermStageBytes = 32 * 1024;
constexpr int kPermSmem = kPermStages * kPermStageBytes + 128 + 64;

struct __align__(64) PermTmaParams {
    CUtensorMap src;
    CUtensorMap dst;
    int P, G, B, Lc, Hl, H_in, H_out, T, n_tblk, per_head;
    int box_bytes;
    long long n_blocks;
    unsigned long long wait_limit_ns;
};

__device__ __forceinline__ bool perm_wait(uint32_t bar, uint32_t parity, unsigned long long limit) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = global_timer_ns();
    for (uint32_t it = 1;; ++it) {
        if (mbar_try_wait(bar, parity)) return true;
        if ((it & 15u) == 0 && global_timer_ns() - t0 > limit) {
            atomicOr(&g_permute_error_word, 1u);
            return false;
        }
    }
}

// MODE 0: seq2head, MODE 1: head2seq
template <int MODE>
__global__ void __launch_bounds__(32) permute_tma_kernel(const __grid_constant__ PermTmaParams p) {
    extern __shared__ uint8_t smem_raw[];
    if (threadIdx.x != 0) return;
    uint32_t base = smem_u32(smem_raw);
    base = (base + 127u) & ~127u;
    const uint32_t bars = base + kPermStages * kPermStageBytes;
    for (int i = 0; i < kPermStages; ++i) mbar_init(bars + 8 * i, 1);
    fence_mbar_init();
    fence_proxy_async_smem();

    const long long n_my =
        p.n_blocks > blockIdx.x ? (p.n_blocks - 1 - blockIdx.x) / gridDim.x + 1 : 0;

    // block -> coordinates (r: head group).  seq2head order: (r, b, s, t-block, head);
    // head2seq: (s, b, t-block, r), so that consecutive blocks write neighbouring
    // destination bytes.
    auto issue_load = [&](long long i) {
        const long long blk = blockIdx.x + i * gridDim.x;
        const uint32_t stage = base + (uint32_t)(i % kPermStages) * kPermStageBytes;
        const uint32_t bar = bars + 8 * (uint32_t)(i % kPermStages);
        mbar_arrive_expect_tx(bar, (uint32_t)p.box_bytes);
        if (MODE == 0 && p.per_head) {
            // GQA copy: one block per (source head, rank s, batch, token block); the
            // source box is read once and stored to every replica of that head.
            long long x = blk;
            const int tb = (int)(x % p.n_tblk); x /= p.n_tblk;
            const int s = (int)(x % p.P); x /= p.P;
            const int b = (int)(x % p.B);
            const int hs = (int)(x / p.B);
            tma_load_4d(stage, &p.src, bar, 0, hs, tb * p.T, s * p.B + b);
        } else if (MODE == 0) {
            long long x = blk;
            const int tb = (int)(x % p.n_tblk); x /= p.n_tblk;
            const int s = (int)(x % p.P); x /= p.P;
            const int b = (int)(x % p.B);
            const int r = (int)(x / p.B);
            tma_load_4d(stage, &p.src, bar, 0, r * p.Hl, tb * p.T, s * p.B + b);
        } else {
            long long x = blk;
            const int r = (int)(x % p.G); x /= p.G;
            const int tb = (int)(x % p.n_tblk); x /= p.n_tblk;
            const int b = (int)(x % p.B);
            const int s = (int)(x / p.B);
            tma_load_5d(stage, &p.src, bar, 0, 0, tb * p.T, s, r * p.B + b);
        }
    };
    auto issue_store = [&](long long i) {
        const long long blk = blockIdx.x + i * gridDim.x;
        const uint32_t stage = base + (uint32_t)(i % kPermStages) * kPermStageBytes;
        if (MODE == 0 && p.per_head) {
            long long x = blk;
            const int tb = (int)(x % p.n_tblk); x /= p.n_tblk;
            const int s = (int)(x % p.P); x /= p.P;
            const int b = (int)(x % p.B);
            const int hs = (int)(x / p.B);
            // replicas j = hs*rep .. hs*rep+rep-1 of the H_out heads copy source head hs
            const int rep = p.H_out / p.H_in;
            for (int jr = 0; jr < rep; ++jr) {
                const int j = hs * rep + jr;
                const int r = j / p.Hl, hh = j % p.Hl;
                tma_store_5d(&p.dst, stage, 0, hh, tb * p.T, s, r * p.B + b);
            }
        } else if (MODE == 0) {
            long long x = blk;
            const int tb = (int)(x % p.n_tblk); x /= p.n_tblk;
            const int s = (int)(x % p.P); x /= p.P;
            const int b = (int)(x % p.B);
            const int r = (int)(x / p.B);
            tma_store_5d(&p.dst, stage, 0, 0, tb * p.T, s, r * p.B + b);
        } else {
            long long x = blk;
            const int r = (int)(x % p.G); x /= p.G;
            const int tb = (int)(x % p.n_tblk); x /= p.n_tblk;
            const int b = (int)(x % p.B);
            const int s = (int)(x / p.B);
            tma_store_4d(&p.dst, stage, 0, r * p.Hl, tb * p.T, s * p.B + b);
        }
    };

    long long issued = 0;
    for (; issued < kPermStages - 1 && issued < n_my; ++issued) issue_load(issued);
    long long n = 0;
    for (; n < n_my; ++n) {
        const uint32_t bar = bars + 8 * (uint32_t)(n % kPermStages);
        if (!perm_wait(bar, (uint32_t)((n / kPermStages) & 1), p.wait_limit_ns)) break;
        issue_store(n);
        bulk_commit();
        if (issued < n_my) {
            bulk_wait_read<1>();  // the store that last read stage (issued % NS) is done
            issue_load(issued);
            ++issued;
        }
    }
    bulk_wait_all();
    // loads issued but never consumed (only after a timeout) must land before exit
    for (long long i = n; i < issued; ++i)
        perm_wait(bars + 8 * (uint32_t)(i % kPermStages), (uint32_t)((i / kPermStages) & 1),
                  p.wait_limit_ns);
}

PFN_cuTensorMapEncodeTiled_v12000 perm_encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    if (!fn) {
        void* ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
    }
    return fn;
}

// rank-4 {W, H, Lc, PB} or rank-5 {W, Hl, Lc, P, PB} tensor of 32-bit words
bool encode_words(CUtensorMap* m, const void* ptr, int rank, const uint64_t* dims,
                  const uint32_t* box) {
    auto enc = perm_encode_fn();
    if (!enc) return false;
    cuuint64_t d[5], st[4];
    cuuint32_t bx[5], es[5] = {1, 1, 1, 1, 1};
    uint64_t stride = 4;
    for (int i = 0; i < rank; ++i) {
        d[i] = dims[i];
        bx[i] = box[i];
        if (i > 0) st[i - 1] = stride;
        stride *= dims[i];
    }
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT32, rank, const_cast<void*>(ptr), d, st, bx, es,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int MODE>
cudaError_t launch_perm_tma(const PermTmaParams& p, cudaStream_t s) {
    static int configured_for = -1;
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (configured_for != dev) {
        e = cudaFuncSetAttribute(permute_tma_kernel<MODE>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize, kPermSmem);
        if (e != cudaSuccess) return e;
        configured_for = dev;
    }
    long long grid = (long long)sm_count() * 2;
    if (grid > p.n_blocks) grid = p.n_blocks;
    if (grid < 1) grid = 1;
    permute_tma_kernel<MODE><<<(unsigned)grid, 32, kPermSmem, s>>>(p);
    return cudaGetLastError();
}

// TMA path usable: a head segment is at most 256 words (the box limit)
bool tma_ok(int D, int esize) { return (D * esize) % 16 == 0 && (D * esize) / 4 <= 256; }

int tokens_per_box(int words, int heads_per_box) {
    int t = kPermStageBytes / (words * 4 * heads_per_box);
    if (t > 256) t = 256;
    return t < 1 ? 1 : t;
}

unsigned grid_for(uint32_t n_groups) {
    const uint32_t per_wave = (uint32_t)sm_count() * 8u;  // 8 resident 256-thread CTAs per SM
    uint32_t blocks = (n_groups + 255u) / 256u;
    if (blocks > per_wave * 4u) blocks = per_wave * 4u;
    return blocks ? blocks : 1u;
}

}  // namespace

cudaError_t launch_seq2head(const void* in, void* out, int P, int G, int B, int Lc, int H_in,
                            int H_out, int D, int esize, cudaStream_t s,
                            unsigned long long wait_limit_ns) {
    const int Hl = H_out / G;
    if (tma_ok(D, esize) && Hl <= 256 && Hl * (D * esize) <= kPermStageBytes) {
        static thread_local PermTmaParams p;
        const int W = D * esize / 4;
        p.per_head = H_in != H_out;
        const int hbox = p.per_head ? 1 : Hl;
        p.T = tokens_per_box(W, hbox);
        const uint64_t sdims[4] = {(uint64_t)W, (uint64_t)H_in, (uint64_t)Lc, (uint64_t)P * B};
        const uint32_t sbox[4] = {(uint32_t)W, (uint32_t)hbox, (uint32_t)p.T, 1};
        const uint64_t ddims[5] = {(uint64_t)W, (uint64_t)Hl, (uint64_t)Lc, (uint64_t)P,
                                   (uint64_t)G * B};
        const uint32_t dbox[5] = {(uint32_t)W, (uint32_t)hbox, (uint32_t)p.T, 1, 1};
        if (encode_words(&p.src, in, 4, sdims, sbox) && encode_words(&p.dst, out, 5, ddims, dbox)) {
            p.P = P; p.G = G; p.B = B; p.Lc = Lc; p.Hl = Hl; p.H_in = H_in; p.H_out = H_out;
            p.n_tblk = (Lc + p.T - 1) / p.T;
            p.box_bytes = W * 4 * hbox * p.T;
            // per_head: one block per source head (its replicas are stored from one load)
            p.n_blocks = (long long)(p.per_head ? H_in : G) * B * P * p.n_tblk;
            p.wait_limit_ns = wait_limit_ns;
            return launch_perm_tma<0>(p, s);
        }
    }
    PermuteGeom geo = make_seq2head_geom(P, G, B, Lc, H_in, H_out, D, esize);
    const uint64_t n_vec = (uint64_t)G * B * P * Lc * (uint64_t)(H_out / G) * geo.VD.div;
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

cudaError_t launch_head2seq(const void* in, void* out, int P, int G, int B, int Lc, int H, int D,
                            int esize, cudaStream_t s, unsigned long long wait_limit_ns) {
    const int Hl = H / G;
    if (tma_ok(D, esize) && Hl <= 256 && Hl * (D * esize) <= kPermStageBytes) {
        static thread_local PermTmaParams p;
        const int W = D * esize / 4;
        p.per_head = 0;
        p.T = tokens_per_box(W, Hl);
        const uint64_t sdims[5] = {(uint64_t)W, (uint64_t)Hl, (uint64_t)Lc, (uint64_t)P,
                                   (uint64_t)G * B};
        const uint32_t sbox[5] = {(uint32_t)W, (uint32_t)Hl, (uint32_t)p.T, 1, 1};
        const uint64_t ddims[4] = {(uint64_t)W, (uint64_t)H, (uint64_t)Lc, (uint64_t)P * B};
        const uint32_t dbox[4] = {(uint32_t)W, (uint32_t)Hl, (uint32_t)p.T, 1};
        if (encode_words(&p.src, in, 5, sdims, sbox) && encode_words(&p.dst, out, 4, ddims, dbox)) {
            p.P = P; p.G = G; p.B = B; p.Lc = Lc; p.Hl = Hl; p.H_in = H; p.H_out = H;
            p.n_tblk = (Lc + p.T - 1) / p.T;
            p.box_bytes = W * 4 * Hl * p.T;
            p.n_blocks = (long long)P * B * p.n_tblk * G;
            p.wait_limit_ns = wait_limit_ns;
            return launch_perm_tma<1>(p, s);
        }
    }
    PermuteGeom geo = make_head2seq_geom(P, G, B, Lc, H, D, esize);
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

// ------------------------------------------------------------------ the GQA copy's gradient
// out[r][g][:] = sum_{k < rep} in[r][g rep + k][:] over fp32 rows of H_in = H_out * rep heads:
// the adjoint of seq->head's repeat-interleave copy, so the gradient of a KV head is the sum
// of its replicas'.  HBM-bound: every input element read once, every output written once;
// one thread per 16-byte vector of out, the replicas added in ascending order (the same bits
// on every call).
__global__ void __launch_bounds__(256) replica_sum_kernel(const float4* __restrict__ in,
                                                          float4* __restrict__ out,
                                                          unsigned long long n_out, int H_out,
                                                          int rep, int D4) {
    const unsigned long long stride = (unsigned long long)gridDim.x * blockDim.x;
    for (unsigned long long i = (unsigned long long)blockIdx.x * blockDim.x + threadIdx.x; i < n_out;
         i += stride) {
        const unsigned long long row_g = i / (unsigned)D4;  // (row, g) pair
        const unsigned d4 = (unsigned)(i - row_g * (unsigned)D4);
        const unsigned long long r = row_g / (unsigned)H_out;
        const unsigned g = (unsigned)(row_g - r * (unsigned)H_out);
        const float4* src = in + ((r * (unsigned)H_out + g) * (unsigned)rep) * (unsigned)D4 + d4;
        float4 acc = src[0];
        for (int k = 1; k < rep; ++k) {
            const float4 x = src[(unsigned long long)k * (unsigned)D4];
            acc.x += x.x;
            acc.y += x.y;
            acc.z += x.z;
            acc.w += x.w;
        }
        out[i] = acc;
    }
}

cudaError_t launch_replica_sum(const float* in, float* out, long long rows, int H_in, int H_out,
                               int D, cudaStream_t s) {
    const int D4 = D / 4, rep = H_in / H_out;
    const unsigned long long n_out = (unsigned long long)rows * H_out * D4;
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) == cudaSuccess)
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const unsigned long long want = (n_out + 255) / 256;
    const unsigned grid = (unsigned)(want < (unsigned long long)sms * 8 ? (want ? want : 1) : (unsigned long long)sms * 8);
    replica_sum_kernel<<<grid, 256, 0, s>>>((const float4*)in, (float4*)out, n_out, H_out, rep, D4);
    return cudaGetLastError();
}

// ------------------------------------------------------------------ one rank's all-to-all share
// The Ulysses exchange as one kernel: rank `me` reads its own tensor and stores each
// destination rank's block straight into that rank's buffer (dst[r]: peer memory mapped
// into this process, or local memory), so the pack, the all-to-all and the unpack become one
// pass.  Plain 16-byte loads from local memory and 16-byte stores; consecutive threads
// store consecutive addresses of one destination (a whole head segment, or Hl of them).
// The kernel ends with a system-scope fence, so that its stores to peers are performed
// before work ordered after the kernel (the caller's cross-rank barrier) signals anyone.
struct ScatterParams {
    int4* dst[RA_MAX_P];
    const int4* in;
    uint32_t n_groups;
    ScatterGeom geo;
};

namespace {
template <int MODE, int U>  // MODE 0: seq2head, 1: head2seq
__global__ void __launch_bounds__(256) scatter_kernel(const __grid_constant__ ScatterParams p) {
    const uint32_t stride = gridDim.x * blockDim.x;
    for (uint32_t g = blockIdx.x * blockDim.x + threadIdx.x; g < p.n_groups; g += stride) {
        const uint32_t vec = g * U;  // U vectors of one head segment (VD % U == 0)
        const ScatterVec sv =
            MODE == 0 ? seq2head_scatter_vec(p.geo, vec) : head2seq_scatter_vec(p.geo, vec);
        int4 v[U];
#pragma unroll
        for (int u = 0; u < U; ++u) v[u] = __ldg(p.in + sv.src + u);
        int4* d = p.dst[sv.r] + sv.dst;
#pragma unroll
        for (int u = 0; u < U; ++u) d[u] = v[u];
    }
    __threadfence_system();
}
}  // namespace

cudaError_t launch_ulysses_scatter(int mode, const void* in, void* const* dst, int P, int me,
                                   int B, int Lc, int H_in, int H_out, int D, int esize,
                                   cudaStream_t s) {
    static thread_local ScatterParams p;
    const int Hl = H_out / P;
    for (int r = 0; r < P; ++r) p.dst[r] = (int4*)dst[r];
    p.in = (const int4*)in;
    p.geo = make_scatter_geom(P, me, B, Lc, H_in, H_out, Hl, D, esize);
    const uint64_t n_vec = (uint64_t)P * B * Lc * (uint64_t)Hl * p.geo.VD.div;
    const int U = p.geo.VD.div % 4 == 0 ? 4 : 1;
    p.n_groups = (uint32_t)(n_vec / U);
    if (p.n_groups == 0) return cudaSuccess;
    const unsigned grid = grid_for(p.n_groups);
    if (mode == 0 && U == 4) scatter_kernel<0, 4><<<grid, 256, 0, s>>>(p);
    else if (mode == 0) scatter_kernel<0, 1><<<grid, 256, 0, s>>>(p);
    else if (U == 4) scatter_kernel<1, 4><<<grid, 256, 0, s>>>(p);
    else scatter_kernel<1, 1><<<grid, 256, 0, s>>>(p);
    return cudaGetLastError();
}

cudaError_t read_and_clear_permute_error(unsigned int* value) {
    cudaError_t e = cudaMemcpyFromSymbol(value, g_permute_error_word, sizeof(unsigned int));
    if (e != cudaSuccess) return e;
    if (*value) {
        const unsigned int zero = 0;
        e = cudaMemcpyToSymbol(g_permute_error_word, &zero, sizeof(unsigned int));
    }
    return e;
}

}  // namespace ra
