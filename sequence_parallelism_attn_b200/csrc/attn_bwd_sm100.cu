// attn_bwd_sm100.cu -- the backward pass of ring-chunked attention on the Blackwell tensor
// cores (sm_100a): dQ, dK, dV of O = softmax(scale Q K^T) V given dO, with the forward's
// LSE ("Как работает sequence parallelism в контексте LLM?" trains with ring attention;
// the gradient is the derivative of the section-5 computation):
//   P  = exp(scale Q K^T - LSE)        (recomputed from the forward's log-sum-exp)
//   dP = dO V^T,  Delta = rowsum(dO * O),  dS = P * (dP - Delta)
//   dQ = scale dS K,   dK = scale dS^T Q,   dV = P^T dO
// Two kernels: Delta (a row reduction, which also zeroes dQ) and one tensor-core kernel
// with the key tile stationary that produces all three gradients.  Its CTA holds one
// 128-key tile of a chunk and visits every query tile of every query head of the kv
// head's group that can see it; per (head, query tile) item it computes S^T and dP^T once,
// accumulates dV and dK in tensor memory, and adds the item's dQ contribution into the
// fp32 dQ in global memory with bulk tensor reduce-adds.  The order of those adds across
// CTAs varies from run to run, so dQ is reproducible up to the rounding of a reordered
// fp32 sum; dK and dV are written once per key and are bit-reproducible.  The kernel is
// compiled per shard layout (contiguous, zigzag, packed samples), like the forward.  Every
// wait is bounded: a role that gives up sets the CTA abort flag and this file's error
// word, every role stops issuing and drains its own work, and the CTA frees its tensor
// memory.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>
#include <climits>
#include <cmath>
#include <cstdint>
#include "ra_internal.h"
#include "attn_sched.cuh"
#include "sm100_ptx.cuh"
#include "../../include/ra.h"

namespace ra {

__device__ unsigned int g_bwd_error_word = 0;

namespace {

constexpr int kThreads = 512;
constexpr int kThreadsQ = 352;  // the deterministic mode's dQ kernel
constexpr int kComputeWarps = 8;  // two warpgroups: one per 64-query half of every item
constexpr int kWarpLoad = 8;
constexpr int kWarpMma = 9;    // MMA-issuing thread A: S^T, dV (owns tensor memory)
constexpr int kWarpMma2 = 10;  // MMA-issuing thread B: dK, dQ
constexpr int kWarpMmaC = 11;  // MMA-issuing thread C: dP^T
constexpr int kWarpRed0 = 12;  // first of the four dQ reduce warps (one per TMEM lane quarter)
// register split (setmaxnreg): launched at 128 per thread (512 x 128 = 65536), the compute
// warpgroups rise to 160, the load / MMA warpgroup and the reduce warpgroup fall to 96
constexpr uint32_t kRegsLaunch = 128, kRegsCompute = 160, kRegsOther = 96, kRegsRed = 96;
static_assert(2 * kRegsCompute + kRegsOther + kRegsRed == 4 * kRegsLaunch,
              "register split must use exactly the launch allocation");
constexpr int kBM = 128;  // query rows per tile
constexpr int kBN = 128;  // keys per tile
static_assert(kBN == kSchedTile, "the schedule counts tiles of kBN keys");
constexpr uint32_t kTmemCols = 512;
constexpr unsigned kErrLoad = 1u, kErrMma = 2u, kErrCompute = 4u, kErrDrain = 8u, kErrReduce = 16u;

struct __align__(64) BwdParams {
    CUtensorMap tm_q;   // [D][H_q][L][B] bf16
    CUtensorMap tm_do;  // [D][H_q][L][B] bf16
    CUtensorMap tm_dq;  // [D][H_q][L][B] fp32, 16-column x 32-row boxes (reduce-add target)
    CUtensorMap tm_k[RA_MAX_P];
    CUtensorMap tm_v[RA_MAX_P];
    const float* lse;    // [B][H_q][L]
    const float* delta;  // [B][H_q][L]
    float* dq;           // [B][L][H_q][D]
    float* dk[RA_MAX_P];  // chunk j: [B][Lc][H_kv][D]
    float* dv[RA_MAX_P];
    int P, B, H_q, H_kv, Lc, L, causal, group, n_qblocks, ntc;
    int zigzag;       // shards in the zigzag layout
    int position_order;  // zigzag, causal, Lc/2 a multiple of 128: grids by sequence position
    const int* pid;   // packed samples: position_ids [B][L] (else null)
    int accumulate;   // dK, dV added to the values in memory (dQ: not zeroed by Delta)
    int skip_dq;      // deterministic mode: dQ from bwd_dq_sm100 (the key-stationary kernel
                      // is then its SKIP_DQ instance)
    float scale, scale_log2;
    unsigned long long wait_limit_ns;
};

// Shard layouts, compiled as separate kernels (the contiguous one keeps plain index
// arithmetic per tile).
constexpr int kLayoutContiguous = 0, kLayoutZigzag = 1, kLayoutPacked = 2;


__device__ __forceinline__ void raise_abort(volatile int* abort_flag, unsigned code) {
    *abort_flag = 1;
    atomicOr(&g_bwd_error_word, code);
}

__device__ __forceinline__ bool wait1(uint32_t bar, uint32_t parity, volatile int* abort_flag,
                                      unsigned long long limit, unsigned code) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = global_timer_ns();
    for (uint32_t it = 1;; ++it) {
        if (mbar_try_wait(bar, parity)) return true;
        if ((it & 15u) == 0) {
            if (*abort_flag) return false;
            if (global_timer_ns() - t0 > limit) {
                raise_abort(abort_flag, code);
                return false;
            }
        }
    }
}

__device__ __forceinline__ bool wait_drain(uint32_t bar, uint32_t parity, volatile int* abort_flag,
                                           unsigned long long limit) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = global_timer_ns();
    for (uint32_t it = 1;; ++it) {
        if (mbar_try_wait(bar, parity)) return true;
        if ((it & 15u) == 0 && global_timer_ns() - t0 > limit) {
            raise_abort(abort_flag, kErrDrain);
            return false;
        }
    }
}

// Warp-uniform bounded wait (every lane polls; the give-up decision is lane 0's).
__device__ __forceinline__ bool wait_warp(uint32_t bar, uint32_t parity, volatile int* abort_flag,
                                          unsigned long long limit, unsigned code) {
    const unsigned FULL = 0xffffffffu;
    bool done = mbar_try_wait(bar, parity);
    if (__all_sync(FULL, done)) return true;
    const uint64_t t0 = global_timer_ns();
    for (uint32_t it = 1;; ++it) {
        if (!done) done = mbar_try_wait(bar, parity);
        if (__all_sync(FULL, done)) return true;
        if ((it & 15u) == 0) {
            int stop = 0;
            if ((threadIdx.x & 31) == 0) {
                if (*abort_flag) stop = 1;
                else if (global_timer_ns() - t0 > limit) {
                    raise_abort(abort_flag, code);
                    stop = 1;
                }
            }
            if (__shfl_sync(FULL, stop, 0)) return false;
        }
    }
}

// Two 32-column TMEM loads of this thread's lane as 32 fp32 pairs (column 2i low).
__device__ __forceinline__ void tmem_ld64(uint32_t taddr, float (&x)[64]) {
    uint32_t a[32], b[32];
    tmem_ld32(taddr, a);
    tmem_ld32(taddr + 32, b);
    tmem_wait_ld();
#pragma unroll
    for (int i = 0; i < 32; ++i) {
        x[i] = __uint_as_float(a[i]);
        x[32 + i] = __uint_as_float(b[i]);
    }
}

// 64 fp32 columns of this thread's TMEM lane as 32 register pairs (column 2i in the low
// half of pair i), loaded and waited for in one block so that every pair is an aligned
// 64-bit register ready for the packed f32x2 instructions.
__device__ __forceinline__ void tmem_ld64_pairs(uint32_t taddr, uint64_t (&o)[32]) {
    asm volatile(
        "{\n\t.reg .b32 r0, r1, r2, r3, r4, r5, r6, r7, r8, r9, r10, r11, r12, r13, r14, r15, r16, r17, r18, r19, r20, r21, r22, r23, r24, r25, r26, r27, r28, r29, r30, r31, r32, r33, r34, r35, r36, r37, r38, r39, r40, r41, r42, r43, r44, r45, r46, r47, r48, r49, r50, r51, r52, r53, r54, r55, r56, r57, r58, r59, r60, r61, r62, r63;\n\t"
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {r0, r1, r2, r3, r4, r5, r6, r7, r8, r9, r10, r11, r12, r13, r14, r15, r16, r17, r18, r19, r20, r21, r22, r23, r24, r25, r26, r27, r28, r29, r30, r31}, [%32];\n\t"
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {r32, r33, r34, r35, r36, r37, r38, r39, r40, r41, r42, r43, r44, r45, r46, r47, r48, r49, r50, r51, r52, r53, r54, r55, r56, r57, r58, r59, r60, r61, r62, r63}, [%33];\n\t"
        "tcgen05.wait::ld.sync.aligned;\n\t"
        "mov.b64 %0, {r0, r1};\n\t"
        "mov.b64 %1, {r2, r3};\n\t"
        "mov.b64 %2, {r4, r5};\n\t"
        "mov.b64 %3, {r6, r7};\n\t"
        "mov.b64 %4, {r8, r9};\n\t"
        "mov.b64 %5, {r10, r11};\n\t"
        "mov.b64 %6, {r12, r13};\n\t"
        "mov.b64 %7, {r14, r15};\n\t"
        "mov.b64 %8, {r16, r17};\n\t"
        "mov.b64 %9, {r18, r19};\n\t"
        "mov.b64 %10, {r20, r21};\n\t"
        "mov.b64 %11, {r22, r23};\n\t"
        "mov.b64 %12, {r24, r25};\n\t"
        "mov.b64 %13, {r26, r27};\n\t"
        "mov.b64 %14, {r28, r29};\n\t"
        "mov.b64 %15, {r30, r31};\n\t"
        "mov.b64 %16, {r32, r33};\n\t"
        "mov.b64 %17, {r34, r35};\n\t"
        "mov.b64 %18, {r36, r37};\n\t"
        "mov.b64 %19, {r38, r39};\n\t"
        "mov.b64 %20, {r40, r41};\n\t"
        "mov.b64 %21, {r42, r43};\n\t"
        "mov.b64 %22, {r44, r45};\n\t"
        "mov.b64 %23, {r46, r47};\n\t"
        "mov.b64 %24, {r48, r49};\n\t"
        "mov.b64 %25, {r50, r51};\n\t"
        "mov.b64 %26, {r52, r53};\n\t"
        "mov.b64 %27, {r54, r55};\n\t"
        "mov.b64 %28, {r56, r57};\n\t"
        "mov.b64 %29, {r58, r59};\n\t"
        "mov.b64 %30, {r60, r61};\n\t"
        "mov.b64 %31, {r62, r63};\n\t"
        "}"
        : "=l"(o[0]), "=l"(o[1]), "=l"(o[2]), "=l"(o[3]), "=l"(o[4]), "=l"(o[5]), "=l"(o[6]), "=l"(o[7]), "=l"(o[8]), "=l"(o[9]), "=l"(o[10]), "=l"(o[11]), "=l"(o[12]), "=l"(o[13]), "=l"(o[14]), "=l"(o[15]), "=l"(o[16]), "=l"(o[17]), "=l"(o[18]), "=l"(o[19]), "=l"(o[20]), "=l"(o[21]), "=l"(o[22]), "=l"(o[23]), "=l"(o[24]), "=l"(o[25]), "=l"(o[26]), "=l"(o[27]), "=l"(o[28]), "=l"(o[29]), "=l"(o[30]), "=l"(o[31])
        : "r"(taddr), "r"(taddr + 32)
        : "memory");
}

// The backward's elementwise step on packed fp32 pairs, in two parts so that P can be
// formed before dP is ready:
//   p  = 2^(s * scale_log2 + neg_lse)     (one packed fma, two MUFU ex2)
//   ds = p * (dp + neg_delta)             (one packed add, one packed multiply)
// p_pair returns bf16x2(p) (lane 0 in the low half) and the fp32 pair in p2; the roundings
// are those of the scalar fma, add and multiply.
__device__ __forceinline__ uint32_t p_pair(uint64_t s2, uint64_t sl2x2, uint64_t nlse2,
                                           uint64_t& p2) {
    uint32_t pp;
    asm("{\n\t.reg .b32 x0, x1, p0, p1;\n\t.reg .b64 x;\n\t"
        "fma.rn.f32x2 x, %2, %3, %4;\n\t"
        "mov.b64 {x0, x1}, x;\n\t"
        "ex2.approx.ftz.f32 p0, x0;\n\t"
        "ex2.approx.ftz.f32 p1, x1;\n\t"
        "cvt.rn.bf16x2.f32 %0, p1, p0;\n\t"
        "mov.b64 %1, {p0, p1};\n\t}"
        : "=r"(pp), "=l"(p2)
        : "l"(s2), "l"(sl2x2), "l"(nlse2));
    return pp;
}

// The second part: bf16x2(p * (dp + neg_delta)) from the fp32 pair p2 of p_pair.
__device__ __forceinline__ uint32_t ds_from_p(uint64_t p2, uint64_t dp2, uint64_t ndelta2) {
    uint32_t pd;
    asm("{\n\t.reg .b32 d0, d1;\n\t.reg .b64 t, d;\n\t"
        "add.rn.f32x2 t, %2, %3;\n\t"
        "mul.rn.f32x2 d, %1, t;\n\t"
        "mov.b64 {d0, d1}, d;\n\t"
        "cvt.rn.bf16x2.f32 %0, d1, d0;\n\t}"
        : "=r"(pd)
        : "l"(p2), "l"(dp2), "l"(ndelta2));
    return pd;
}

// The same without bf16(p): the dQ kernel needs only dS.
__device__ __forceinline__ uint32_t ds_pair(uint64_t s2, uint64_t dp2, uint64_t sl2x2,
                                            uint64_t nlse2, uint64_t ndelta2) {
    uint32_t pd;
    asm("{\n\t.reg .b32 x0, x1, p0, p1, d0, d1;\n\t.reg .b64 x, p, t, d;\n\t"
        "fma.rn.f32x2 x, %1, %3, %4;\n\t"
        "mov.b64 {x0, x1}, x;\n\t"
        "ex2.approx.ftz.f32 p0, x0;\n\t"
        "ex2.approx.ftz.f32 p1, x1;\n\t"
        "mov.b64 p, {p0, p1};\n\t"
        "add.rn.f32x2 t, %2, %5;\n\t"
        "mul.rn.f32x2 d, p, t;\n\t"
        "mov.b64 {d0, d1}, d;\n\t"
        "cvt.rn.bf16x2.f32 %0, d1, d0;\n\t}"
        : "=r"(pd)
        : "l"(s2), "l"(dp2), "l"(sl2x2), "l"(nlse2), "l"(ndelta2));
    return pd;
}

// ------------------------------------------------------------------ layout helpers
// Sample start of row r of batch row b (packed samples).
__device__ __forceinline__ int sample_start(const BwdParams& p, int b, int r) {
    return ra::sample_start(p.pid + (long long)b * p.L, r);
}

// The keys of tile (chunk j, local keys key0 .. key0 + kvalid - 1) that a query at sequence
// position my_pos with sample start my_start sees form one interval [c_lo, c_hi] of tile
// columns (empty when c_lo > c_hi).  Key c sits at position kpos0 + c, except that a zigzag
// tile straddling the shard's two segments continues from c = cs at the second segment's
// start, and a query that sees a key of the second segment sees all of the first.
template <int LAYOUT>
__device__ __forceinline__ void key_interval(const BwdParams& p, int j, int key0, int kvalid,
                                             int my_pos, int my_start, int& c_lo, int& c_hi) {
    constexpr int ZZ = LAYOUT == kLayoutZigzag ? 1 : 0;
    const int kpos0 = (int)shard_pos(ZZ, p.P, p.Lc, j, key0);
    auto clamp_c = [](int x) { return x < -1 ? -1 : (x > kBN ? kBN : x); };
    c_hi = kvalid - 1;
    if (p.causal) {
        int hi = clamp_c(my_pos - kpos0);
        const int hseg = p.Lc / 2;
        if (ZZ && key0 < hseg && key0 + kBN > hseg) {
            const int cs = hseg - key0;
            const int hi2 = clamp_c(my_pos - (int)shard_pos(1, p.P, p.Lc, j, hseg) + cs);
            hi = hi2 >= cs ? hi2 : min(hi, cs - 1);
        }
        c_hi = min(c_hi, hi);
    }
    c_lo = LAYOUT == kLayoutPacked ? clamp_c(my_start - kpos0) : -1;
}

// ------------------------------------------------------------------ Delta = rowsum(dO * O)
// One warp per (b, t, h) row, fp32 accumulation of the bf16 products; the row of dQ is
// zeroed on the way (the backward kernel adds every key tile's contribution into it).
template <int D>
__global__ void __launch_bounds__(256) bwd_delta_kernel(const uint16_t* __restrict__ out,
                                                        const uint16_t* __restrict__ dout,
                                                        float* __restrict__ delta,
                                                        float* __restrict__ dq, int zero_dq,
                                                        int B, int L, int H) {
    const long long row = (long long)blockIdx.x * 8 + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (row >= (long long)B * L * H) return;
    const uint16_t* o = out + row * D;
    const uint16_t* g = dout + row * D;
    if (zero_dq && 4 * lane < D)
        reinterpret_cast<float4*>(dq + row * D)[lane] = make_float4(0.f, 0.f, 0.f, 0.f);
    float acc = 0.f;
#pragma unroll
    for (int i = lane; i < D; i += 32)
        acc = fmaf(__uint_as_float((uint32_t)o[i] << 16), __uint_as_float((uint32_t)g[i] << 16), acc);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
    if (lane == 0) {
        const long long t = (row / H) % L, h = row % H, b = row / H / L;
        delta[(b * H + h) * L + t] = acc;
    }
}

template <int D>
struct QCfg {
    static constexpr int TILE = kBM * D * 2;  // bytes of a 128 x D bf16 tile
    static constexpr int NKB = D / 64;        // 64-column (128-byte) swizzle blocks per tile
    static constexpr int BLK = kBM * 128;     // bytes of one swizzle block
    static constexpr int NS = 2;              // ring stages
    // Q and dO once; a ring of (K, V) stages
    static constexpr int OFF_A = 0;                      // Q
    static constexpr int OFF_B = TILE;                   // dO
    static constexpr int OFF_RING = 2 * TILE;            // NS x (K, V) stages
    static constexpr int STAGE = 2 * TILE;
    static constexpr int OFF_BAR = OFF_RING + NS * STAGE;
    // barriers: fixed_full, full[NS], empty[NS], s_ready (S of a tile complete), dp_ready
    // (dP complete), ds_full[2][2] (dS of each 64-column half stored; two per half, by tile
    // parity), acc_done, drain, dp_free (the compute warps have read all of dP); the indices
    // between are unused
    static constexpr int N_BARS = 1 + 2 * NS + 14;
    static constexpr int OFF_MISC = OFF_BAR + N_BARS * 8;  // tmem base, abort flag, n
    static constexpr int OFF_SCHED = OFF_MISC + 16;   // per-chunk tile ranges
    static constexpr int SMEM = OFF_SCHED + 2 * RA_MAX_P * 4 + 1024;
    static constexpr int BAR_FIXED = 0;
    __host__ __device__ static constexpr int bar_full(int s) { return 1 + s; }
    __host__ __device__ static constexpr int bar_empty(int s) { return 1 + NS + s; }
    static constexpr int BAR_SREADY = 1 + 2 * NS;
    static constexpr int BAR_DPREADY = 2 + 2 * NS;
    // tile i's barrier of a half and its wait parity: the k-th phase of ds(half, par)
    // belongs to tile 2k + par
    __host__ __device__ static constexpr int bar_ds(int half, int i) { return 3 + 2 * NS + 2 * half + (i & 1); }
    __host__ __device__ static constexpr uint32_t par2(int i) { return (uint32_t)(i >> 1) & 1u; }
    static constexpr int BAR_ACC = 11 + 2 * NS;
    static constexpr int BAR_DRAIN = 12 + 2 * NS;
    static constexpr int BAR_DPFREE = 13 + 2 * NS;
    // TMEM: S of even key tiles at column 0, of odd ones at S_ODD (S of the next tile is
    // computed while this tile's dS is formed), dP at 128, dQ at 256.
    static constexpr uint32_t S_ODD = 384;
    __host__ __device__ static constexpr uint32_t s_col(int jt) { return (jt & 1) ? S_ODD : 0u; }
    static_assert(SMEM <= 232448, "shared memory budget");
    static_assert(STAGE % 1024 == 0, "TMA destinations of every stage stay 1024-byte aligned");
    static_assert(256 + D <= (int)S_ODD && S_ODD + kBN <= kTmemCols, "dQ kernel columns");
};

// ------------------------------------------------------------------ dQ, deterministic
// The deterministic mode's dQ: one CTA per 128 query rows of one (batch, head), 352 threads
// (warps 0-7 compute, warp 8 loads, warps 9 and 10 one MMA-issuing thread each).  Q and dO
// stay in shared memory; K and V stream through a two-stage ring in the forward's chunk
// order (causal tiles skipped by the shared schedule).  Per key tile: S = Q K^T and
// dP = dO V^T, dS formed in registers and stored as bf16 over S, dQ += dS K; every dQ
// element is written once, by its CTA, after all key tiles in one fixed order.  The
// key-stationary kernel then runs with its dQ share skipped.
template <int D, int LAYOUT>
__global__ void __launch_bounds__(kThreadsQ, 1) bwd_dq_sm100(const __grid_constant__ BwdParams p) {
    using C = QCfg<D>;
    extern __shared__ uint8_t smem_raw[];
    uint32_t base = smem_u32(smem_raw);
    const uint32_t pad = (1024u - (base & 1023u)) & 1023u;
    base += pad;
    uint8_t* smem = smem_raw + pad;
    volatile uint32_t* tmem_slot = reinterpret_cast<volatile uint32_t*>(smem + C::OFF_MISC);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::OFF_MISC + 4);
    volatile int* n_slot = reinterpret_cast<volatile int*>(smem + C::OFF_MISC + 8);
    uint32_t* sched_range = reinterpret_cast<uint32_t*>(smem + C::OFF_SCHED);
    auto bar = [&](int i) { return base + C::OFF_BAR + 8u * (uint32_t)i; };
    const unsigned long long lim = p.wait_limit_ns;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    // grid: (batch, kv head) outermost, then row blocks heaviest first, then the query
    // heads of the group (they read the same K/V tiles)
    const int per_bg = p.n_qblocks * p.group;
    const int bg = (int)(blockIdx.x / per_bg), rem = (int)(blockIdx.x % per_bg);
    const int b = bg / p.H_kv, g = bg % p.H_kv;
    const int h = g * p.group + rem % p.group;
    int r0 = (p.n_qblocks - 1 - rem / p.group) * kBM;
    if (LAYOUT == kLayoutZigzag && p.position_order) {
        // the k-th block visited is the one at the k-th latest position: segments 2P-1 down
        // to 0 (segment s >= P is the second half of rank 2P-1-s, s < P the first of rank s)
        const int kvis = rem / p.group, hseg = p.Lc / 2, seg_blocks = hseg / kBM;
        const int seg = 2 * p.P - 1 - kvis / seg_blocks;
        const int bis = seg_blocks - 1 - kvis % seg_blocks;
        const int rank = seg < p.P ? seg : 2 * p.P - 1 - seg;
        r0 = rank * p.Lc + (seg < p.P ? 0 : hseg) + bis * kBM;
    }

    if (threadIdx.x == 0) {
        mbar_init(bar(C::BAR_FIXED), 1);
        for (int s = 0; s < C::NS; ++s) {
            mbar_init(bar(C::bar_full(s)), 1);
            mbar_init(bar(C::bar_empty(s)), 1);
        }
        mbar_init(bar(C::BAR_SREADY), 1);   // thread A's commit after S
        mbar_init(bar(C::BAR_DPREADY), 1);  // thread B's commit after dP
        for (int hf = 0; hf < 2; ++hf)
            for (int par = 0; par < 2; ++par) mbar_init(bar(C::bar_ds(hf, par)), 4 * 32);
        mbar_init(bar(C::BAR_ACC), 1);
        mbar_init(bar(C::BAR_DRAIN), 2);
        mbar_init(bar(C::BAR_DPFREE), kComputeWarps * 32);
        *abort_flag = 0;
        fence_mbar_init();
        fence_proxy_async_smem();
    }
    if (warp == kWarpLoad) {
        SchedArgs sa;
        sa.P = p.P; sa.Lc = p.Lc; sa.L = p.L; sa.causal = p.causal;
        sa.zigzag = LAYOUT == kLayoutZigzag ? 1 : 0;
        sa.pid = LAYOUT == kLayoutPacked ? p.pid : nullptr;
        const long long last_row = min((long long)r0 + kBM - 1, (long long)p.L - 1);
        const int nt = make_schedule(sa, b, r0, last_row, sched_range);
        if (lane == 0) *n_slot = nt;
    }
    if (warp == kWarpMma) {
        __syncwarp();
        tmem_alloc(base + C::OFF_MISC, kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    Sched sched;
    sched.range = sched_range;
    sched.P = p.P;
    sched.i0 = r0 / p.Lc;
    const int n = *n_slot;

    if (warp == kWarpLoad) {
        if (lane == 0) {
            // Q and dO once; K and V of each visited tile through an NS-deep ring
            mbar_arrive_expect_tx(bar(C::BAR_FIXED), 2 * C::TILE);
            for (int kb = 0; kb < C::NKB; ++kb) {
                tma_load_4d(base + C::OFF_A + kb * C::BLK, &p.tm_q, bar(C::BAR_FIXED), kb * 64, h, r0, b);
                tma_load_4d(base + C::OFF_B + kb * C::BLK, &p.tm_do, bar(C::BAR_FIXED), kb * 64, h, r0, b);
            }
            int armed[C::NS];
            for (int s = 0; s < C::NS; ++s) armed[s] = -1;
            SchedIter it;
            it.begin(sched);
            for (int jt = 0; jt < n; ++jt, it.next()) {
                const int slot = jt % C::NS;
                if (jt >= C::NS &&
                    !wait1(bar(C::bar_empty(slot)), ((jt / C::NS) - 1) & 1, abort_flag, lim, kErrLoad))
                    break;
                const uint32_t st = base + C::OFF_RING + slot * C::STAGE;
                mbar_arrive_expect_tx(bar(C::bar_full(slot)), 2 * C::TILE);
                for (int kb = 0; kb < C::NKB; ++kb) {
                    tma_load_4d(st + kb * C::BLK, &p.tm_k[it.chunk()], bar(C::bar_full(slot)),
                                kb * 64, g, it.t * kBN, b);
                    tma_load_4d(st + C::TILE + kb * C::BLK, &p.tm_v[it.chunk()],
                                bar(C::bar_full(slot)), kb * 64, g, it.t * kBN, b);
                }
                armed[slot] = jt;
            }
            wait_drain(bar(C::BAR_FIXED), 0, abort_flag, lim);
            for (int s = 0; s < C::NS; ++s)
                if (armed[s] >= 0) wait_drain(bar(C::bar_full(s)), (armed[s] / C::NS) & 1, abort_flag, lim);
        }
    } else if (warp == kWarpMma || warp == kWarpMma2) {
        if (lane == 0) {
            const bool thread_a = warp == kWarpMma;
            constexpr uint32_t IDESC_S = idesc_bf16_f32(kBM, kBN, 0);  // K-major A and B
            constexpr uint32_t IDESC_O = idesc_bf16_f32(kBM, D, 1);    // B MN-major (D contiguous)
            const uint64_t dq_ = desc_sw128(base + C::OFF_A, 16, 1024);
            const uint64_t ddo = desc_sw128(base + C::OFF_B, 16, 1024);
            auto stage = [&](int jt) { return base + C::OFF_RING + (uint32_t)(jt % C::NS) * C::STAGE; };
            auto issue_s = [&](int jt) {  // S(jt) = Q K(jt)^T into its column region
                const uint64_t dk = desc_sw128(stage(jt), 16, 1024);
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t off = ((kk / 4) * C::BLK + (kk % 4) * 32) >> 4;
                    mma_ss(tmem + C::s_col(jt), dq_ + off, dk + off, IDESC_S, kk > 0 ? 1u : 0u);
                }
            };
            auto issue_dp = [&](int jt) {  // dP(jt) = dO V(jt)^T
                const uint64_t dv = desc_sw128(stage(jt) + C::TILE, 16, 1024);
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t off = ((kk / 4) * C::BLK + (kk % 4) * 32) >> 4;
                    mma_ss(tmem + 128, ddo + off, dv + off, IDESC_S, kk > 0 ? 1u : 0u);
                }
            };
            auto dq_half = [&](int jt, int half) {  // dQ += dS(jt) K(jt) over 64 keys
                // dS (bf16 pairs) of the half over the first 32 of its 64 S columns, K as
                // MN-major B
                const uint64_t dkm = desc_sw128(stage(jt), C::BLK, 1024);
#pragma unroll
                for (int kk = 4 * half; kk < 4 * half + 4; ++kk)
                    mma_ts(tmem + 256, tmem + C::s_col(jt) + 64 * half + (kk % 4) * 8,
                           dkm + (uint64_t)((kk * 2048) >> 4), IDESC_O,
                           (jt > 0 || kk > 0) ? 1u : 0u);
            };
            // Two issuing threads (one thread cannot issue 128-wide MMAs fast enough to keep
            // the tensor core busy).  A issues S and dQ, B issues dP; no MMA reads the other
            // thread's output columns.  A, per key tile jt: S(jt+1) into the other S region as
            // soon as K(jt+1) has landed, committed to s_ready once every compute warp has
            // read tile jt (dp_free) -- so the commit waits for S(jt+1) alone, not for dQ(jt),
            // and s_ready cannot complete a phase before the compute warps have waited for
            // the previous one; then dQ over each 64-key half as the compute warps publish it.
            // B, per key tile jt: dP(jt+1) once the compute warps have read dP(jt), committed
            // to dp_ready.  The compute warps can then finish tile jt+1 before A has waited for
            // tile jt's dS, which is why each half's ds barrier alternates by tile parity.
            if (wait1(bar(C::BAR_FIXED), 0, abort_flag, lim, kErrMma) && n > 0 &&
                wait1(bar(C::bar_full(0)), 0, abort_flag, lim, kErrMma)) {
                tc_fence_after();
                if (thread_a) {
                    issue_s(0);
                    tc_commit(bar(C::BAR_SREADY));
                    for (int jt = 0; jt < n; ++jt) {
                        const bool more = jt + 1 < n;
                        if (more) {
                            if (!wait1(bar(C::bar_full((jt + 1) % C::NS)), ((jt + 1) / C::NS) & 1,
                                       abort_flag, lim, kErrMma))
                                break;
                            tc_fence_after();
                            issue_s(jt + 1);
                            if (!wait1(bar(C::BAR_DPFREE), jt & 1, abort_flag, lim, kErrMma)) break;
                            tc_commit(bar(C::BAR_SREADY));
                        }
                        if (!wait1(bar(C::bar_ds(0, jt)), C::par2(jt), abort_flag, lim, kErrMma))
                            break;
                        tc_fence_after();
                        dq_half(jt, 0);
                        if (!wait1(bar(C::bar_ds(1, jt)), C::par2(jt), abort_flag, lim, kErrMma))
                            break;
                        tc_fence_after();
                        dq_half(jt, 1);
                        tc_commit(bar(C::bar_empty(jt % C::NS)));
                    }
                } else {
                    issue_dp(0);
                    tc_commit(bar(C::BAR_DPREADY));
                    for (int jt = 0; jt + 1 < n; ++jt) {
                        if (!wait1(bar(C::BAR_DPFREE), jt & 1, abort_flag, lim, kErrMma)) break;
                        if (!wait1(bar(C::bar_full((jt + 1) % C::NS)), ((jt + 1) / C::NS) & 1,
                                   abort_flag, lim, kErrMma))
                            break;
                        tc_fence_after();
                        issue_dp(jt + 1);
                        tc_commit(bar(C::BAR_DPREADY));
                    }
                }
            }
            if (n > 0) {  // a commit with nothing outstanding arrives at once
                if (thread_a) tc_commit(bar(C::BAR_ACC));
                tc_commit(bar(C::BAR_DRAIN));
                wait_drain(bar(C::BAR_DRAIN), 0, abort_flag, lim);
            }
        }
    } else {
        // compute warps: P and dS for this thread's row over its warpgroup's 64-key half
        // (a warp reaches TMEM lanes 32 (warp % 4) .. + 31)
        const int quarter = warp & 3, c = warp >> 2;
        const int row_t = quarter * 32 + lane;
        const long long my_row = (long long)r0 + row_t;
        const bool row_ok = my_row < p.L;
        const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
        const long long lrow = ((long long)b * p.H_q + h) * p.L + (row_ok ? my_row : 0);
        // rows past L see nothing (lse2 = +inf makes every probability 0)
        const float lse2 = row_ok ? p.lse[lrow] * 1.4426950408889634f : INFINITY;
        const float dlt = row_ok ? p.delta[lrow] : 0.f;
        const float sl2 = p.scale_log2;
        const uint64_t sl2x2 = f2_pack(sl2, sl2), nlse2 = f2_pack(-lse2, -lse2),
                       nd2 = f2_pack(-dlt, -dlt);
        // zigzag / packed: this row's sequence position and sample start (L <= 2^30)
        constexpr int ZZ = LAYOUT == kLayoutZigzag ? 1 : 0;
        const int my_pos = row_ok ? (int)shard_pos(ZZ, p.P, p.Lc, (int)(my_row / p.Lc), my_row % p.Lc)
                                  : p.L;
        const int my_start = (LAYOUT == kLayoutPacked && row_ok) ? sample_start(p, b, (int)my_row) : 0;
        bool ok = true;
        SchedIter it;
        it.begin(sched);
        for (int jt = 0; jt < n; ++jt, it.next()) {
            if (!wait_warp(bar(C::BAR_SREADY), jt & 1, abort_flag, lim, kErrCompute) ||
                !wait_warp(bar(C::BAR_DPREADY), jt & 1, abort_flag, lim, kErrCompute)) {
                ok = false;
                break;
            }
            __syncwarp();
            tc_fence_after();
            const int kvalid = min(kBN, p.Lc - it.t * kBN);
            // this row sees the tile's keys c with c_lo <= c <= c_hi
            int c_lo = -1, c_hi;
            if (LAYOUT == kLayoutContiguous) {
                const long long k0 = (long long)it.chunk() * p.Lc + (long long)it.t * kBN;
                const long long lim = p.causal ? my_row - k0 : (long long)kBN;
                c_hi = (int)min((long long)(kvalid - 1), lim < -1 ? -1LL : lim);
            } else {
                key_interval<LAYOUT>(p, it.chunk(), it.t * kBN, kvalid, my_pos, my_start, c_lo, c_hi);
            }
            const uint32_t scol = C::s_col(jt);
            uint32_t pk[32];
            // warp-uniform: the TMEM loads below are warp-collective
            if (__all_sync(0xffffffffu, 64 * c >= c_lo && 64 * c + 63 <= c_hi)) {
                // every key of this half is visible to every row of the warp: packed pairs
                uint64_t s2[32], d2[32];
                tmem_ld64_pairs(tmem + lane_off + scol + 64 * c, s2);
                tmem_ld64_pairs(tmem + lane_off + 128 + 64 * c, d2);
                // dP is in registers: once both halves are, its columns may take dP(jt+1)
                tc_fence_before();
                mbar_arrive(bar(C::BAR_DPFREE));
#pragma unroll
                for (int i = 0; i < 32; ++i) pk[i] = ds_pair(s2[i], d2[i], sl2x2, nlse2, nd2);
            } else {
                float s[64], dp[64];
                tmem_ld64(tmem + lane_off + scol + 64 * c, s);
                tmem_ld64(tmem + lane_off + 128 + 64 * c, dp);
                tc_fence_before();
                mbar_arrive(bar(C::BAR_DPFREE));
#pragma unroll
                for (int i = 0; i < 32; ++i) {
                    float ds2[2];
#pragma unroll
                    for (int e = 0; e < 2; ++e) {
                        const int col = 64 * c + 2 * i + e;
                        const bool vis = col >= c_lo && col <= c_hi;
                        const float pr = vis ? ex2_approx(s[2 * i + e] * sl2 - lse2) : 0.f;
                        ds2[e] = pr * (dp[2 * i + e] - dlt);
                    }
                    pk[i] = pack_bf16x2(ds2[0], ds2[1]);
                }
            }
            // publish this 64-key half over its own S columns (already read)
            tmem_st32(tmem + lane_off + scol + 64 * c, pk);
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(bar(C::bar_ds(c, jt)));
        }
        if (ok && n > 0 && wait_warp(bar(C::BAR_ACC), 0, abort_flag, lim, kErrCompute)) {
            __syncwarp();
            tc_fence_after();
#pragma unroll
            for (int cb = c * (D / 64); cb < (c + 1) * (D / 64); ++cb) {  // this half's columns
                uint32_t o[32];
                tmem_ld32(tmem + lane_off + 256 + cb * 32, o);
                tmem_wait_ld();
                if (row_ok) {
                    float4* dst = reinterpret_cast<float4*>(
                        p.dq + (((long long)b * p.L + my_row) * p.H_q + h) * D + cb * 32);
#pragma unroll
                    for (int i = 0; i < 8; ++i) {
                        float4 r = make_float4(__uint_as_float(o[4 * i]) * p.scale,
                                               __uint_as_float(o[4 * i + 1]) * p.scale,
                                               __uint_as_float(o[4 * i + 2]) * p.scale,
                                               __uint_as_float(o[4 * i + 3]) * p.scale);
                        if (p.accumulate) {  // this CTA alone owns the row
                            const float4 was = dst[i];
                            r.x += was.x;
                            r.y += was.y;
                            r.z += was.z;
                            r.w += was.w;
                        }
                        dst[i] = r;
                    }
                }
            }
        } else if (ok && n == 0 && row_ok && !p.accumulate) {  // the row sees no key
            float4* dst = reinterpret_cast<float4*>(
                p.dq + (((long long)b * p.L + my_row) * p.H_q + h) * D + c * (D / 2));
            for (int i = 0; i < D / 8; ++i) dst[i] = make_float4(0.f, 0.f, 0.f, 0.f);
        }
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == kWarpMma) {
        __syncwarp();
        tmem_dealloc(tmem, kTmemCols);
    }
}


// ------------------------------------------------------------------ dQ, dK, dV (key tile stationary)
// Per (head, query tile) item i of the CTA, tensor memory holds
//   R_S  [0, 128)     S^T(i); P^T of each 64-query half over the first 32 columns of it
//   R_DP [128, 256)   dP^T(i), one N = 64 MMA per query half; then dQ(i) = dS(i) K (its D
//                     columns), once both halves of dP^T(i) have been read
//   dV [256, 256 + D), dK [256 + D, 256 + 2D)
// and dS^T(i) goes to shared memory (bf16, keys as rows, 128-byte swizzle), where it is the
// K-major A operand of dK += dS^T Q and the MN-major A operand of dQ = dS K.  At D = 128 it
// is written over dO(i) once dV(i) and both dP^T(i) halves have read dO(i) (the shared
// memory holds K, V, two (Q, dO) stages and the dQ staging buffers); at D = 64 each stage
// has its own dS^T slot.
// Roles: warps 0-7 compute P^T and dS^T (one key per thread, warpgroup c the query half c),
// warp 8 loads (TMA, and the per-row LSE, Delta, positions and sample starts), warps 9, 10,
// 11 each issue MMAs from one thread -- A: dV, then S^T of the next item into R_S once dV is
// done; B: dK per half as dS^T is stored, dQ after the second half; C: dP^T of the next
// item per half once the reduce warps have read that half of dQ -- and warps 12-15 (one per
// TMEM lane quarter) read dQ out of tensor memory and reduce it into global memory in
// 32-row x 16-column chunks through three staging buffers per warp.
template <int D>
struct BCfg {
    static constexpr int TILE = kBM * D * 2;   // bytes of a 128 x D bf16 tile
    static constexpr int NKB = D / 64;         // 64-column swizzle blocks per tile
    static constexpr int BLK = kBM * 128;      // bytes of one swizzle block (128 rows)
    static constexpr int NS = 2;               // (Q, dO) stages
    static constexpr int DS_BYTES = kBN * kBM * 2;  // dS^T of one item, bf16
    static constexpr bool DS_IN_DO = TILE >= DS_BYTES;
    static constexpr int OFF_A = 0;            // K
    static constexpr int OFF_B = TILE;         // V
    static constexpr int OFF_RING = 2 * TILE;  // NS x (Q, dO)
    static constexpr int STAGE = 2 * TILE;
    static constexpr int OFF_DS = OFF_RING + NS * STAGE;  // D = 64: NS dS^T slots
    static constexpr int OFF_STG = OFF_DS + (DS_IN_DO ? 0 : NS * DS_BYTES);
    static constexpr int STG_BUF = 32 * 16 * 4;  // 32 rows x 16 fp32, 64-byte swizzle
    static constexpr int STG_NB = 3;             // buffers per reduce warp
    static constexpr int OFF_ROWS = OFF_STG + 4 * STG_NB * STG_BUF;
    // per stage: -LSE log2(e), -Delta, sequence position, sample start per query row, and
    // per 64-row half the smallest position and the largest start
    static constexpr int ROWS_BYTES = 4 * kBM * 4 + 4 * 4;
    static constexpr int OFF_BAR = OFF_ROWS + NS * ROWS_BYTES;
    // barriers: fixed_full, full[NS], empty[NS] (A's and B's release), s_ready, dp_ready[2]
    // (per query half), dv_done, p_full[2], ds_full[2], dq_ready, r_free[2] (per 64-column
    // half of dQ), acc_done, drain
    static constexpr int N_BARS = 1 + 2 * NS + 13;
    static constexpr int OFF_MISC = OFF_BAR + N_BARS * 8;  // tmem base, abort flag, n, nr
    static constexpr int OFF_QR = OFF_MISC + 16;
    static constexpr int SMEM = OFF_QR + 2 * RA_MAX_P * 8 + 1024;
    static constexpr int BAR_FIXED = 0;
    __host__ __device__ static constexpr int bar_full(int s) { return 1 + s; }
    __host__ __device__ static constexpr int bar_empty(int s) { return 1 + NS + s; }
    static constexpr int BAR_SREADY = 1 + 2 * NS;
    __host__ __device__ static constexpr int bar_dpready(int h) { return 2 + 2 * NS + h; }
    static constexpr int BAR_DVDONE = 4 + 2 * NS;
    __host__ __device__ static constexpr int bar_p(int c) { return 5 + 2 * NS + c; }
    __host__ __device__ static constexpr int bar_ds(int c) { return 7 + 2 * NS + c; }
    static constexpr int BAR_DQREADY = 9 + 2 * NS;
    __host__ __device__ static constexpr int bar_rfree(int h) { return 10 + 2 * NS + h; }
    static constexpr int BAR_ACC = 12 + 2 * NS;
    static constexpr int BAR_DRAIN = 13 + 2 * NS;
    static constexpr uint32_t R_S = 0, R_DP = 128, COL_DV = 256, COL_DK = 256 + D;
    static_assert(BAR_DRAIN == N_BARS - 1, "barrier count");
    static_assert(SMEM <= 232448, "shared memory budget");
    static_assert(OFF_RING % 1024 == 0 && STAGE % 1024 == 0 && OFF_DS % 1024 == 0 &&
                  OFF_STG % 1024 == 0, "swizzled buffers stay 1024-byte aligned");
    static_assert(OFF_BAR % 8 == 0, "mbarrier alignment");
    static_assert(COL_DK + D <= kTmemCols, "tensor memory budget");
    static_assert(D <= 128, "dQ of one item fits in the dP^T region");
};

template <int D, int LAYOUT, bool SKIP_DQ>
__global__ void __launch_bounds__(kThreads, 1) bwd_sm100(const __grid_constant__ BwdParams p) {
    using C = BCfg<D>;
    extern __shared__ uint8_t smem_raw[];
    uint32_t base = smem_u32(smem_raw);
    const uint32_t pad = (1024u - (base & 1023u)) & 1023u;
    base += pad;
    uint8_t* smem = smem_raw + pad;
    volatile uint32_t* tmem_slot = reinterpret_cast<volatile uint32_t*>(smem + C::OFF_MISC);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::OFF_MISC + 4);
    volatile int* n_slot = reinterpret_cast<volatile int*>(smem + C::OFF_MISC + 8);
    volatile int* nr_slot = reinterpret_cast<volatile int*>(smem + C::OFF_MISC + 12);
    int* qr_lo = reinterpret_cast<int*>(smem + C::OFF_QR);
    int* qr_hi = qr_lo + 2 * RA_MAX_P;
    auto bar = [&](int i) { return base + C::OFF_BAR + 8u * (uint32_t)i; };
    const unsigned long long lim = p.wait_limit_ns;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    constexpr bool CONTIG = LAYOUT == kLayoutContiguous;

    // grid: (batch, kv head) outermost, then the key tiles (chunk j, tile t) heaviest first
    const int n_kt = p.P * p.ntc;
    const int bg = (int)(blockIdx.x / n_kt), kt = (int)(blockIdx.x % n_kt);
    const int b = bg / p.H_kv, g = bg % p.H_kv;
    int j = kt / p.ntc, t = kt % p.ntc;
    if (LAYOUT == kLayoutZigzag && p.position_order) {
        const int seg_tiles = (p.Lc / 2) / kBN, seg = kt / seg_tiles;
        j = seg < p.P ? seg : 2 * p.P - 1 - seg;
        t = (seg < p.P ? 0 : seg_tiles) + kt % seg_tiles;
    }
    const long long key0 = (long long)j * p.Lc + (long long)t * kBN;
    const int kvalid = min(kBN, p.Lc - t * kBN);
    const int qt0 = p.causal ? (int)(key0 / kBM) : 0;
    const int n_qt = p.n_qblocks - qt0;

    if (threadIdx.x == 0) {
        mbar_init(bar(C::BAR_FIXED), 1);
        for (int s = 0; s < C::NS; ++s) {
            mbar_init(bar(C::bar_full(s)), 1 + 1);  // the load thread's expect_tx + the per-row values
            mbar_init(bar(C::bar_empty(s)), 2);     // A after dV, B after dK and dQ
        }
        mbar_init(bar(C::BAR_SREADY), 1);
        mbar_init(bar(C::bar_dpready(0)), 1);
        mbar_init(bar(C::bar_dpready(1)), 1);
        mbar_init(bar(C::BAR_DVDONE), 1);
        for (int c = 0; c < 2; ++c) {
            mbar_init(bar(C::bar_p(c)), 4 * 32);
            mbar_init(bar(C::bar_ds(c)), 4 * 32);
            mbar_init(bar(C::bar_rfree(c)), 4 * 32);
        }
        mbar_init(bar(C::BAR_DQREADY), 1);
        mbar_init(bar(C::BAR_ACC), 2);    // dV from A, dK from B
        mbar_init(bar(C::BAR_DRAIN), 3);  // A, B, C
        *abort_flag = 0;
        fence_mbar_init();
        fence_proxy_async_smem();
    }
    if (!CONTIG && warp == kWarpLoad && lane == 0) {
        int nt = 0;
        *nr_slot = key_tile_q_ranges(LAYOUT, p.P, p.Lc, p.causal, kBM,
                                     p.pid ? p.pid + (long long)b * p.L : nullptr, j, t * kBN,
                                     kvalid, qr_lo, qr_hi, &nt);
        *n_slot = nt * p.group;
    }
    if (warp == kWarpMma) {
        __syncwarp();
        tmem_alloc(base + C::OFF_MISC, kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const int n = CONTIG ? n_qt * p.group : *n_slot;  // (head, query tile) items, head-major

    // the items in order: (query head, first row of the query tile)
    auto for_items = [&](auto&& fn) {
        if (CONTIG) {
            for (int it = 0; it < n; ++it)
                if (!fn(it, g * p.group + it / n_qt, (qt0 + it % n_qt) * kBM)) return;
        } else {
            const int nr = *nr_slot;
            int it = 0;
            for (int hh = 0; hh < p.group; ++hh)
                for (int ri = 0; ri < nr; ++ri)
                    for (int qt = qr_lo[ri]; qt < qr_hi[ri]; ++qt, ++it)
                        if (!fn(it, g * p.group + hh, qt * kBM)) return;
        }
    };
    auto stage = [&](int i) { return base + C::OFF_RING + (uint32_t)(i % C::NS) * C::STAGE; };
    auto ds_slot = [&](int i) {
        return C::DS_IN_DO ? stage(i) + (uint32_t)C::TILE
                           : base + C::OFF_DS + (uint32_t)(i % C::NS) * C::DS_BYTES;
    };
    auto rows_of = [&](int i) {
        return reinterpret_cast<float*>(smem + C::OFF_ROWS + (i % C::NS) * C::ROWS_BYTES);
    };

    if (warp >= kComputeWarps && warp < kWarpRed0) {
      regs_decrease<kRegsOther>();
      if (warp == kWarpLoad) {
        if (lane == 0) {
            mbar_arrive_expect_tx(bar(C::BAR_FIXED), 2 * C::TILE);
            for (int kb = 0; kb < C::NKB; ++kb) {
                tma_load_4d(base + C::OFF_A + kb * C::BLK, &p.tm_k[j], bar(C::BAR_FIXED), kb * 64, g, t * kBN, b);
                tma_load_4d(base + C::OFF_B + kb * C::BLK, &p.tm_v[j], bar(C::BAR_FIXED), kb * 64, g, t * kBN, b);
            }
        }
        int armed[C::NS];
        for (int s = 0; s < C::NS; ++s) armed[s] = -1;
        for_items([&](int it, int h, int q0) -> bool {
            const int slot = it % C::NS;
            // the item's per-row values into registers first: their global loads are in
            // flight while the warp waits for a free stage.  Negated: the compute warps add
            // them (rows past L give P = 0, dS = 0).  Zigzag / packed: the row's sequence
            // position and sample start (it sees the keys at positions start .. pos; every
            // key when not causal).
            const long long lbase = ((long long)b * p.H_q + h) * p.L;
            float vl[4], vd[4];
            int vp[4], vs[4];
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const long long row = (long long)q0 + lane + 32 * k;
                vl[k] = row < p.L ? -(p.lse[lbase + row] * 1.4426950408889634f) : -INFINITY;
                vd[k] = row < p.L ? -p.delta[lbase + row] : 0.f;
                vp[k] = INT_MAX;
                vs[k] = 0;
                if (!CONTIG && row < p.L && p.causal) {
                    const int ri = (int)row;  // L <= 2^30
                    vp[k] = (int)shard_pos(LAYOUT == kLayoutZigzag ? 1 : 0, p.P, p.Lc, ri / p.Lc,
                                           ri % p.Lc);
                    if (LAYOUT == kLayoutPacked) vs[k] = sample_start(p, b, ri);
                }
            }
            if (it >= C::NS &&
                !wait_warp(bar(C::bar_empty(slot)), ((it / C::NS) - 1) & 1, abort_flag, lim, kErrLoad))
                return false;
            const uint32_t st = stage(it);
            if (lane == 0) {
                mbar_arrive_expect_tx(bar(C::bar_full(slot)), 2 * C::TILE);
                for (int kb = 0; kb < C::NKB; ++kb)
                    tma_load_4d(st + kb * C::BLK, &p.tm_q, bar(C::bar_full(slot)), kb * 64, h, q0, b);
                for (int kb = 0; kb < C::NKB; ++kb)
                    tma_load_4d(st + C::TILE + kb * C::BLK, &p.tm_do, bar(C::bar_full(slot)), kb * 64, h, q0, b);
            }
            float* rows = rows_of(it);
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                rows[lane + 32 * k] = vl[k];
                rows[kBM + lane + 32 * k] = vd[k];
            }
            if (!CONTIG) {
                int pmin0 = min(vp[0], vp[1]), pmin1 = min(vp[2], vp[3]);
                int smax0 = max(vs[0], vs[1]), smax1 = max(vs[2], vs[3]);
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    reinterpret_cast<int*>(rows)[2 * kBM + lane + 32 * k] = vp[k];
                    reinterpret_cast<int*>(rows)[3 * kBM + lane + 32 * k] = vs[k];
                }
#pragma unroll
                for (int off = 16; off > 0; off >>= 1) {
                    pmin0 = min(pmin0, __shfl_xor_sync(0xffffffffu, pmin0, off));
                    pmin1 = min(pmin1, __shfl_xor_sync(0xffffffffu, pmin1, off));
                    smax0 = max(smax0, __shfl_xor_sync(0xffffffffu, smax0, off));
                    smax1 = max(smax1, __shfl_xor_sync(0xffffffffu, smax1, off));
                }
                if (lane == 0) {
                    int* sum = reinterpret_cast<int*>(rows) + 4 * kBM;
                    sum[0] = pmin0; sum[1] = pmin1; sum[2] = smax0; sum[3] = smax1;
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(C::bar_full(slot)));
            armed[slot] = it;
            return true;
        });
        if (lane == 0) {
            wait_drain(bar(C::BAR_FIXED), 0, abort_flag, lim);
            for (int s = 0; s < C::NS; ++s)
                if (armed[s] >= 0) wait_drain(bar(C::bar_full(s)), (armed[s] / C::NS) & 1, abort_flag, lim);
        }
      } else if (lane == 0) {  // warps 9, 10, 11: one MMA-issuing thread each
        constexpr uint32_t IDESC_S = idesc_bf16_f32(kBN, kBM, 0);       // S^T: K-major A, B
        constexpr uint32_t IDESC_DP = idesc_bf16_f32(kBN, kBM / 2, 0);  // dP^T of one half
        constexpr uint32_t IDESC_O = idesc_bf16_f32(kBN, D, 1);         // dV, dK: B MN-major
        constexpr uint32_t IDESC_Q = idesc_bf16_f32_ab(kBM, D, 1, 1);   // dQ: A, B MN-major
        const uint64_t dk_ = desc_sw128(base + C::OFF_A, 16, 1024);      // K as K-major A
        const uint64_t dv_ = desc_sw128(base + C::OFF_B, 16, 1024);      // V as K-major A
        const uint64_t kmn = desc_sw128(base + C::OFF_A, C::BLK, 1024);  // K as MN-major B
        auto koff = [](int kk) { return (uint32_t)(((kk / 4) * C::BLK + (kk % 4) * 32) >> 4); };
        // S^T(i) = K Q(i)^T into R_S
        auto issue_st = [&](int i) {
            const uint64_t dq_ = desc_sw128(stage(i), 16, 1024);
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk)
                mma_ss(tmem + C::R_S, dk_ + koff(kk), dq_ + koff(kk), IDESC_S, kk > 0 ? 1u : 0u);
        };
        // dP^T(i) of query half hq = V dO(rows 64 hq ..)^T into R_DP + 64 hq
        auto issue_dpt = [&](int i, int hq) {
            const uint64_t ddo = desc_sw128(stage(i) + C::TILE + (uint32_t)hq * 64u * 128u, 16, 1024);
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk)
                mma_ss(tmem + C::R_DP + 64u * hq, dv_ + koff(kk), ddo + koff(kk), IDESC_DP,
                       kk > 0 ? 1u : 0u);
        };
        // dV += P^T dO over query half c (P^T from tensor memory, dO MN-major)
        auto issue_dv = [&](int i, int c) {
            const uint64_t bm = desc_sw128(stage(i) + C::TILE, C::BLK, 1024);
            const uint32_t a0 = tmem + C::R_S + 64u * c;
#pragma unroll
            for (int kk = 4 * c; kk < 4 * c + 4; ++kk)
                mma_ts(tmem + C::COL_DV, a0 + (kk % 4) * 8, bm + (uint64_t)((kk * 2048) >> 4),
                       IDESC_O, (i > 0 || kk > 0) ? 1u : 0u);
        };
        // dK += dS^T Q over query half c (dS^T K-major from shared memory, Q MN-major)
        auto issue_dk = [&](int i, int c) {
            const uint64_t a = desc_sw128(ds_slot(i), 16, 1024);
            const uint64_t bq = desc_sw128(stage(i), C::BLK, 1024);
#pragma unroll
            for (int kk = 4 * c; kk < 4 * c + 4; ++kk)
                mma_ss(tmem + C::COL_DK, a + koff(kk), bq + (uint64_t)((kk * 2048) >> 4), IDESC_O,
                       (i > 0 || kk > 0) ? 1u : 0u);
        };
        // dQ(i) = dS K into R_DP (dS: the dS^T slot read MN-major; K MN-major)
        auto issue_dq = [&](int i) {
            const uint64_t a = desc_sw128(ds_slot(i), C::BLK, 1024);
#pragma unroll
            for (int kk = 0; kk < kBN / 16; ++kk)
                mma_ss(tmem + C::R_DP, a + (uint64_t)((kk * 2048) >> 4),
                       kmn + (uint64_t)((kk * 2048) >> 4), IDESC_Q, kk > 0 ? 1u : 0u);
        };
        if (wait1(bar(C::BAR_FIXED), 0, abort_flag, lim, kErrMma) && n > 0) {
            if (warp == kWarpMma) {
                // A: S^T(0); per item: dV per half as its P^T is published, dv_done and the
                // stage's release; once dV(i) is done (it read the P^T that S^T(i+1)
                // overwrites) and the next stage has landed, S^T(i+1)
                if (wait1(bar(C::bar_full(0)), 0, abort_flag, lim, kErrMma)) {
                    tc_fence_after();
                    issue_st(0);
                    tc_commit(bar(C::BAR_SREADY));
                    for (int it = 0; it < n; ++it) {
                        const uint32_t ph = it & 1;
                        if (!wait1(bar(C::bar_p(0)), ph, abort_flag, lim, kErrMma)) break;
                        tc_fence_after();
                        issue_dv(it, 0);
                        if (!wait1(bar(C::bar_p(1)), ph, abort_flag, lim, kErrMma)) break;
                        tc_fence_after();
                        issue_dv(it, 1);
                        tc_commit(bar(C::BAR_DVDONE));
                        tc_commit(bar(C::bar_empty(it % C::NS)));
                        if (it + 1 < n) {
                            if (!wait1(bar(C::BAR_DVDONE), ph, abort_flag, lim, kErrMma)) break;
                            if (!wait1(bar(C::bar_full((it + 1) % C::NS)), ((it + 1) / C::NS) & 1,
                                       abort_flag, lim, kErrMma))
                                break;
                            tc_fence_after();
                            issue_st(it + 1);
                            tc_commit(bar(C::BAR_SREADY));
                        }
                    }
                }
            } else if (warp == kWarpMma2) {
                // B: per item, dK over half 0 once its dS^T is stored; after half 1, dQ,
                // dq_ready, dK over half 1 and the stage's release
                for (int it = 0; it < n; ++it) {
                    const uint32_t ph = it & 1;
                    if (!wait1(bar(C::bar_ds(0)), ph, abort_flag, lim, kErrMma)) break;
                    tc_fence_after();
                    issue_dk(it, 0);
                    if (!wait1(bar(C::bar_ds(1)), ph, abort_flag, lim, kErrMma)) break;
                    tc_fence_after();
                    if (!SKIP_DQ) issue_dq(it);
                    tc_commit(bar(C::BAR_DQREADY));
                    issue_dk(it, 1);
                    tc_commit(bar(C::bar_empty(it % C::NS)));
                }
            } else {
                // C: dP^T(0) per half; per next item, each half once the reduce warps have
                // read the columns of dQ it overwrites
                if (wait1(bar(C::bar_full(0)), 0, abort_flag, lim, kErrMma)) {
                    tc_fence_after();
                    for (int hq = 0; hq < 2; ++hq) {
                        issue_dpt(0, hq);
                        tc_commit(bar(C::bar_dpready(hq)));
                    }
                    bool go = true;
                    for (int it = 0; go && it + 1 < n; ++it) {
                        if (!wait1(bar(C::bar_full((it + 1) % C::NS)), ((it + 1) / C::NS) & 1,
                                   abort_flag, lim, kErrMma))
                            break;
                        for (int hq = 0; hq < 2; ++hq) {
                            if (!wait1(bar(C::bar_rfree(hq)), it & 1, abort_flag, lim, kErrMma)) {
                                go = false;
                                break;
                            }
                            tc_fence_after();
                            issue_dpt(it + 1, hq);
                            tc_commit(bar(C::bar_dpready(hq)));
                        }
                    }
                }
            }
        }
        if (n > 0) {  // a commit with nothing outstanding arrives at once
            if (warp != kWarpMmaC) tc_commit(bar(C::BAR_ACC));
            tc_commit(bar(C::BAR_DRAIN));
            wait_drain(bar(C::BAR_DRAIN), 0, abort_flag, lim);
        }
      }
    } else if (warp >= kWarpRed0) {
        regs_decrease<kRegsRed>();
        // reduce warps: rows 32 q .. 32 q + 31 of each item's dQ (TMEM lanes of quarter q)
        const int quarter = warp & 3;
        const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
        const uint32_t stg = base + C::OFF_STG + (uint32_t)(quarter * C::STG_NB * C::STG_BUF);
        const uint32_t swz = (uint32_t)((lane >> 1) & 3);  // 64-byte swizzle of this row
        const float sc = p.scale;
        uint32_t chunk = 0;  // chunks staged so far (each a committed bulk group)
        for_items([&](int it, int h, int q0) -> bool {
            if (!wait_warp(bar(C::BAR_DQREADY), it & 1, abort_flag, lim, kErrReduce)) return false;
            __syncwarp();
            tc_fence_after();
            const int row0 = q0 + 32 * quarter;
            const bool rows_in = row0 < p.L;  // warp-uniform; rows past L are clipped by TMA
#pragma unroll
            for (int hf = 0; hf < (D + 63) / 64; ++hf) {
                if (SKIP_DQ) {  // no dQ share was computed: only free the columns
                    mbar_arrive(bar(C::bar_rfree(hf)));
                    if (D == 64) mbar_arrive(bar(C::bar_rfree(1)));
                    continue;
                }
                uint32_t va[32], vb[32];
                tmem_ld32(tmem + lane_off + C::R_DP + 64 * hf, va);
                tmem_ld32(tmem + lane_off + C::R_DP + 64 * hf + 32, vb);
                tmem_wait_ld();
                tc_fence_before();
                mbar_arrive(bar(C::bar_rfree(hf)));
                if (D == 64) mbar_arrive(bar(C::bar_rfree(1)));
                if (!rows_in) continue;
#pragma unroll
                for (int ch = 0; ch < 4; ++ch) {
                    const uint32_t buf = stg + (chunk % C::STG_NB) * C::STG_BUF;
                    // the buffer's previous bulk group (three commits ago) has read it
                    if (lane == 0) bulk_wait_read<C::STG_NB - 1>();
                    __syncwarp();
#pragma unroll
                    for (int k4 = 0; k4 < 4; ++k4) {
                        const int c0 = 16 * ch + 4 * k4;  // column within this 64-column half
                        uint32_t w[4];
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const uint32_t x = c0 + e < 32 ? va[c0 + e] : vb[c0 + e - 32];
                            w[e] = __float_as_uint(__uint_as_float(x) * sc);
                        }
                        st_shared_v4(buf + (uint32_t)lane * 64u + (((uint32_t)k4 ^ swz) << 4), w[0],
                                     w[1], w[2], w[3]);
                    }
                    fence_proxy_async_smem();
                    __syncwarp();
                    if (lane == 0) {
                        tma_reduce_add_4d(&p.tm_dq, buf, 64 * hf + 16 * ch, h, row0, b);
                        bulk_commit();
                    }
                    ++chunk;
                }
            }
            return true;
        });
        if (lane == 0) bulk_wait_all();  // the reduce-adds have read and written everything
        __syncwarp();
    } else {
        regs_increase<kRegsCompute>();
        // compute warps: P^T and dS^T for this thread's key against its warpgroup's 64-query
        // half of each item
        const int quarter = warp & 3, c = warp >> 2;
        const int key_t = quarter * 32 + lane;
        const bool key_ok = key_t < kvalid;
        const int my_kpos = key_ok ? (int)shard_pos(LAYOUT == kLayoutZigzag ? 1 : 0, p.P, p.Lc, j,
                                                    t * kBN + key_t)
                                   : INT_MAX;
        const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
        const float sl2 = p.scale_log2;
        const uint64_t sl2x2 = f2_pack(sl2, sl2);
        const uint32_t swz = (uint32_t)(key_t & 7);  // 128-byte swizzle of this key's row
        bool ok = true;
        for (int it = 0; it < n; ++it) {
            const int q0 = (qt0 + it % n_qt) * kBM;
            const uint32_t ph = it & 1;
            if (!wait_warp(bar(C::BAR_SREADY), ph, abort_flag, lim, kErrCompute)) {
                ok = false;
                break;
            }
            __syncwarp();
            tc_fence_after();
            const float* rows = rows_of(it);
            const long long lo_c = p.causal ? (long long)my_kpos - q0 : 0;
            const int* posv = reinterpret_cast<const int*>(rows) + 2 * kBM;
            const int* startv = reinterpret_cast<const int*>(rows) + 3 * kBM;
            const bool half_visible =
                CONTIG ? lo_c <= 64 * c
                       : (my_kpos <= posv[2 * kBM + c] && my_kpos >= posv[2 * kBM + 2 + c]);
            const bool packed = __all_sync(0xffffffffu, key_ok && half_visible);
            uint32_t pp[32];
            uint64_t p2[32];  // the fp32 probabilities as pairs (column 2i low), kept for dS
            if (packed) {
                uint64_t s2[32];
                tmem_ld64_pairs(tmem + lane_off + C::R_S + 64 * c, s2);
                const ulonglong2* nl = reinterpret_cast<const ulonglong2*>(rows + 64 * c);
#pragma unroll
                for (int k = 0; k < 16; ++k) {
                    const ulonglong2 a = nl[k];
                    pp[2 * k] = p_pair(s2[2 * k], sl2x2, a.x, p2[2 * k]);
                    pp[2 * k + 1] = p_pair(s2[2 * k + 1], sl2x2, a.y, p2[2 * k + 1]);
                }
            } else {
                float s[64];
                tmem_ld64(tmem + lane_off + C::R_S + 64 * c, s);
#pragma unroll
                for (int i = 0; i < 32; ++i) {
                    float pr2[2];
#pragma unroll
                    for (int e = 0; e < 2; ++e) {
                        const int col = 64 * c + 2 * i + e;
                        const bool vis =
                            key_ok && (CONTIG ? col >= lo_c
                                              : (my_kpos <= posv[col] && my_kpos >= startv[col]));
                        pr2[e] = vis ? ex2_approx(s[2 * i + e] * sl2 + rows[col]) : 0.f;
                    }
                    pp[i] = pack_bf16x2(pr2[0], pr2[1]);
                    p2[i] = f2_pack(pr2[0], pr2[1]);
                }
            }
            // publish P^T of this half over the S^T columns just read
            tmem_st32(tmem + lane_off + C::R_S + 64 * c, pp);
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(bar(C::bar_p(c)));

            if (!wait_warp(bar(C::bar_dpready(c)), ph, abort_flag, lim, kErrCompute)) {
                ok = false;
                break;
            }
            __syncwarp();
            tc_fence_after();
            uint32_t pd[32];
            if (packed) {
                uint64_t d2[32];
                tmem_ld64_pairs(tmem + lane_off + C::R_DP + 64 * c, d2);
                const ulonglong2* nd = reinterpret_cast<const ulonglong2*>(rows + kBM + 64 * c);
#pragma unroll
                for (int k = 0; k < 16; ++k) {
                    const ulonglong2 d = nd[k];
                    pd[2 * k] = ds_from_p(p2[2 * k], d2[2 * k], d.x);
                    pd[2 * k + 1] = ds_from_p(p2[2 * k + 1], d2[2 * k + 1], d.y);
                }
            } else {
                float dp[64];
                tmem_ld64(tmem + lane_off + C::R_DP + 64 * c, dp);
#pragma unroll
                for (int i = 0; i < 32; ++i) {
                    float pr2[2], ds2[2];
                    f2_unpack(p2[i], pr2[0], pr2[1]);
#pragma unroll
                    for (int e = 0; e < 2; ++e)
                        ds2[e] = pr2[e] * (dp[2 * i + e] + rows[kBM + 64 * c + 2 * i + e]);
                    pd[i] = pack_bf16x2(ds2[0], ds2[1]);
                }
            }
            if (C::DS_IN_DO) {
                // dS^T goes over dO(i): dV(i) and both halves of dP^T(i) must have read it
                if (!wait_warp(bar(C::BAR_DVDONE), ph, abort_flag, lim, kErrCompute) ||
                    !wait_warp(bar(C::bar_dpready(1 - c)), ph, abort_flag, lim, kErrCompute)) {
                    ok = false;
                    break;
                }
            }
            // dS^T of this half: row key_t of swizzle block c (128-byte swizzle)
            const uint32_t drow = ds_slot(it) + (uint32_t)c * C::BLK + (uint32_t)key_t * 128u;
#pragma unroll
            for (int k = 0; k < 8; ++k)
                st_shared_v4(drow + (((uint32_t)k ^ swz) << 4), pd[4 * k], pd[4 * k + 1],
                             pd[4 * k + 2], pd[4 * k + 3]);
            fence_proxy_async_smem();
            tc_fence_before();  // the dP^T loads above precede dQ(i) over the same columns
            mbar_arrive(bar(C::bar_ds(c)));
        }
        if (ok && n > 0 && wait_warp(bar(C::BAR_ACC), 0, abort_flag, lim, kErrCompute)) {
            __syncwarp();
            tc_fence_after();
            const long long orow = (((long long)b * p.Lc + t * kBN + key_t) * p.H_kv + g) * D;
            const int which = c;  // warpgroup 0 writes dV, warpgroup 1 dK (times scale)
            const float mul = which ? p.scale : 1.f;
            float* outp = which ? p.dk[j] : p.dv[j];
#pragma unroll
            for (int cb = 0; cb < D / 32; ++cb) {
                uint32_t o[32];
                tmem_ld32(tmem + lane_off + C::COL_DV + which * D + cb * 32, o);
                tmem_wait_ld();
                if (key_ok) {
                    float4* dst = reinterpret_cast<float4*>(outp + orow + cb * 32);
#pragma unroll
                    for (int i = 0; i < 8; ++i) {
                        float4 r = make_float4(__uint_as_float(o[4 * i]) * mul,
                                               __uint_as_float(o[4 * i + 1]) * mul,
                                               __uint_as_float(o[4 * i + 2]) * mul,
                                               __uint_as_float(o[4 * i + 3]) * mul);
                        if (p.accumulate) {  // this CTA alone owns the key's row
                            const float4 was = dst[i];
                            r.x += was.x;
                            r.y += was.y;
                            r.z += was.z;
                            r.w += was.w;
                        }
                        dst[i] = r;
                    }
                }
            }
        } else if (ok && n == 0 && key_ok && !p.accumulate) {  // no query sees the key
            const long long orow = (((long long)b * p.Lc + t * kBN + key_t) * p.H_kv + g) * D;
            float* outp = c ? p.dk[j] : p.dv[j];
            for (int i = 0; i < D; ++i) outp[orow + i] = 0.f;
        }
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == kWarpMma) {
        __syncwarp();
        tmem_dealloc(tmem, kTmemCols);
    }
}

PFN_cuTensorMapEncodeTiled_v12000 bwd_encode_fn() {
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

// [D][H][rows][B] bf16 tensor, 128-row x 64-column boxes, 128-byte swizzle, zero fill.
bool bwd_tile_map(CUtensorMap* m, const void* ptr, int D, int H, long long rows, int B,
                  long long bstride_elems) {
    auto enc = bwd_encode_fn();
    if (!enc) return false;
    cuuint64_t dims[4] = {(cuuint64_t)D, (cuuint64_t)H, (cuuint64_t)rows, (cuuint64_t)B};
    cuuint64_t strides[3] = {(cuuint64_t)D * 2, (cuuint64_t)H * D * 2, (cuuint64_t)bstride_elems * 2};
    cuuint32_t box[4] = {64, 1, (cuuint32_t)kBM, 1};
    cuuint32_t estr[4] = {1, 1, 1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(ptr), dims, strides, box,
               estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// dQ [B][L][H][D] fp32 as the target of the backward kernel's reduce-adds: 16-column x 32-row
// boxes (64-byte rows, 64-byte swizzle).
bool bwd_dq_reduce_map(CUtensorMap* m, float* ptr, int D, int H, long long rows, int B) {
    auto enc = bwd_encode_fn();
    if (!enc) return false;
    cuuint64_t dims[4] = {(cuuint64_t)D, (cuuint64_t)H, (cuuint64_t)rows, (cuuint64_t)B};
    cuuint64_t strides[3] = {(cuuint64_t)D * 4, (cuuint64_t)H * D * 4,
                             (cuuint64_t)rows * H * D * 4};
    cuuint32_t box[4] = {16, 1, 32, 1};
    cuuint32_t estr[4] = {1, 1, 1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, ptr, dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B,
               CU_TENSOR_MAP_L2_PROMOTION_L2_128B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int D>
cudaError_t launch_bwd_d(const BwdParams& p, const AttnBwdArgs& a, const char** why) {
    static int configured_for = -1;
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    // [skip dQ][layout]: the deterministic mode's key-stationary kernel is compiled apart,
    // so that the default one carries no test of it
    decltype(&bwd_sm100<D, kLayoutContiguous, false>) kern[2][3] = {
        {bwd_sm100<D, kLayoutContiguous, false>, bwd_sm100<D, kLayoutZigzag, false>,
         bwd_sm100<D, kLayoutPacked, false>},
        {bwd_sm100<D, kLayoutContiguous, true>, bwd_sm100<D, kLayoutZigzag, true>,
         bwd_sm100<D, kLayoutPacked, true>}};
    decltype(&bwd_dq_sm100<D, kLayoutContiguous>) kern_dq[3] = {
        bwd_dq_sm100<D, kLayoutContiguous>, bwd_dq_sm100<D, kLayoutZigzag>,
        bwd_dq_sm100<D, kLayoutPacked>};
    if (configured_for != dev) {
        for (int l = 0; l < 3; ++l) {
            for (int sk = 0; sk < 2; ++sk) {
                // the register split assumes the launch allocation: a raise beyond it
                // would never complete
                cudaFuncAttributes fa;
                e = cudaFuncGetAttributes(&fa, kern[sk][l]);
                if (e != cudaSuccess) return e;
                if (fa.numRegs != (int)kRegsLaunch) {
                    *why = "backward kernel compiled with a register count its register split does not assume";
                    return cudaErrorInvalidKernelImage;
                }
                e = cudaFuncSetAttribute(kern[sk][l], cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         BCfg<D>::SMEM);
                if (e != cudaSuccess) return e;
            }
            e = cudaFuncSetAttribute(kern_dq[l], cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     QCfg<D>::SMEM);
            if (e != cudaSuccess) return e;
        }
        configured_for = dev;
    }
    const int layout = p.pid ? kLayoutPacked : (p.zigzag ? kLayoutZigzag : kLayoutContiguous);
    const long long rows = (long long)a.B * p.L * a.H_q;
    bwd_delta_kernel<D><<<(unsigned)((rows + 7) / 8), 256, 0, a.stream>>>(
        (const uint16_t*)a.out, (const uint16_t*)a.dout, a.workspace, a.dq,
        !a.accumulate && !p.skip_dq, a.B, p.L, a.H_q);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    const long long grid_k = (long long)a.B * a.H_kv * a.P * p.ntc;
    kern[p.skip_dq ? 1 : 0][layout]<<<(unsigned)grid_k, kThreads, BCfg<D>::SMEM, a.stream>>>(p);
    e = cudaGetLastError();
    if (e != cudaSuccess || !p.skip_dq) return e;
    // deterministic mode: dQ from the query-stationary kernel, each element written once
    const long long grid_q = (long long)p.n_qblocks * a.B * a.H_q;
    kern_dq[layout]<<<(unsigned)grid_q, kThreadsQ, QCfg<D>::SMEM, a.stream>>>(p);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_attn_bwd_sm100(const AttnBwdArgs& a, unsigned long long wait_limit_ns,
                                  const char** why) {
    static thread_local BwdParams p;
    const long long L = (long long)a.P * a.Lc;
    if (!bwd_tile_map(&p.tm_q, a.q, a.D, a.H_q, L, a.B, a.q_bstride) ||
        !bwd_tile_map(&p.tm_do, a.dout, a.D, a.H_q, L, a.B, L * a.H_q * a.D)) {
        *why = "cuTensorMapEncodeTiled failed for q or dout";
        return cudaErrorInvalidValue;
    }
    if (!bwd_dq_reduce_map(&p.tm_dq, a.dq, a.D, a.H_q, L, a.B)) {
        *why = "cuTensorMapEncodeTiled failed for dq";
        return cudaErrorInvalidValue;
    }
    for (int j = 0; j < a.P; ++j) {
        if (!bwd_tile_map(&p.tm_k[j], a.k_chunks[j], a.D, a.H_kv, a.Lc, a.B, a.kv_bstride) ||
            !bwd_tile_map(&p.tm_v[j], a.v_chunks[j], a.D, a.H_kv, a.Lc, a.B, a.kv_bstride)) {
            *why = "cuTensorMapEncodeTiled failed for a K/V chunk";
            return cudaErrorInvalidValue;
        }
        p.dk[j] = a.dk_chunks[j];
        p.dv[j] = a.dv_chunks[j];
    }
    p.lse = a.lse;
    p.delta = a.workspace;
    p.dq = a.dq;
    p.P = a.P;
    p.B = a.B;
    p.H_q = a.H_q;
    p.H_kv = a.H_kv;
    p.Lc = a.Lc;
    p.L = (int)L;
    p.causal = a.causal;
    p.zigzag = a.zigzag;
    p.position_order = a.zigzag && a.causal && (a.Lc / 2) % kBM == 0;
    p.pid = a.pid;
    p.accumulate = a.accumulate;
    p.skip_dq = a.deterministic ? 1 : 0;
    p.group = a.H_q / a.H_kv;
    p.n_qblocks = (int)((L + kBM - 1) / kBM);
    p.ntc = (a.Lc + kBN - 1) / kBN;
    p.scale = a.scale;
    p.scale_log2 = (float)((double)a.scale * 1.4426950408889634);
    p.wait_limit_ns = wait_limit_ns;
    if ((long long)p.n_qblocks * a.B * a.H_q > 0x7fffffffLL) {
        *why = "problem too large for one launch";
        return cudaErrorInvalidValue;
    }
    if (a.D == 128) return launch_bwd_d<128>(p, a, why);
    if (a.D == 64) return launch_bwd_d<64>(p, a, why);
    *why = "head dimension not supported by the tensor-core backward";
    return cudaErrorInvalidValue;
}

cudaError_t read_and_clear_bwd_error(unsigned int* value) {
    cudaError_t e = cudaMemcpyFromSymbol(value, g_bwd_error_word, sizeof(unsigned int));
    if (e != cudaSuccess) return e;
    if (*value) {
        const unsigned int zero = 0;
        e = cudaMemcpyToSymbol(g_bwd_error_word, &zero, sizeof(unsigned int));
    }
    return e;
}

}  // namespace ra
