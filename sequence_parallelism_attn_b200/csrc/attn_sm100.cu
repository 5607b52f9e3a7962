// attn_sm100.cu -- ring-chunked exact attention on the Blackwell tensor cores (sm_100a).
//
// What it computes ("Как работает sequence parallelism в контексте LLM?"):
//   section 2  -- the sequence of length L = P*Lc is split into P contiguous chunks, rank i
//                 owning tokens [i*Lc, (i+1)*Lc);
//   section 3  -- ring attention: at step s the queries of rank i attend to the K/V chunk
//                 it holds then, chunk j = (i - s) mod P, for s = 0..P-1;
//   section 5  -- per chunk: scores Q.K^T, row max, exp, row sum, and the merge of the new
//                 partial into the running one by rescaling with exp(lse_old - lse_new);
//                 finally the division by the normaliser.
// Here the P ranks are virtual chunk partitions in one GPU's memory.  The merge across
// chunk steps is carried in registers and tensor memory as the running (max, normaliser,
// output) state of an online softmax: rescaling the running output by
// exp2(m_old - m_new) whenever a tile of a new chunk raises the row maximum is exactly the
// ring's log-sum-exp merge, applied at 128-key granularity.  Causal masking (a reading:
// global positions in rank order, key <= query) skips chunk pairs and 128-key tiles that
// lie wholly after the CTA's last query row -- no MMA is issued for them -- and masks
// elements only in tiles that straddle the diagonal or a ragged chunk end.
//
// Kernel organisation (one CTA per 256 query rows of one (batch, head); 384 threads):
//   warps 0-3  softmax for query tile A (rows r0 .. r0+127), one TMEM lane (= row) each
//   warps 4-7  softmax for query tile B (rows r0+128 .. r0+255)
//   warp 8     TMA producer of the Q tiles (once) and the K tiles (NSK-deep ring)
//   warp 9     MMA issuer (one thread) and TMEM owner
//   warp 10    TMA producer of the V tiles (NSV-deep ring)
//   warp 11    idle (it completes the third warpgroup for the register split)
// Registers: launched at 168 per thread (3 warps per SM sub-partition); the softmax
// warpgroups raise their budget to 192 and the third warpgroup drops to 120
// (192 + 192 + 120 = 504 <= 512 per sub-partition; 256*192 + 128*120 = 384*168).
// Tensor memory (512 columns x 128 lanes x 32 bit):
//   S [0,128): one fp32 score buffer shared by the two query tiles; P_A [128,192) and
//   P_B [192,256): bf16 probabilities (two per column); O_A at 256, O_B at 256+D (fp32).
// Per KV tile j the MMA thread issues, in this order,
//   S_A(j+1) = Q_A K(j+1)^T  once softmax B has read S_B(j) out of S,
//   PV_A(j)  = P_A V(j)      once softmax A has written P_A(j),
//   S_B(j+1)                 once softmax A has read S_A(j+1),
//   PV_B(j)                  once softmax B has written P_B(j),
// so a tile's next scores are computed while its softmax still works on the current ones:
// a softmax warpgroup finds S(j+1) ready when it finishes P(j), and the tensor core is
// never waiting on a chain of PV(j) then S(j+1).  A softmax warpgroup reads S, signals that
// S is free, and waits for PV(j-1) (its commit) only before it overwrites P(j-1) with P(j)
// -- and before it rescales O, which it does only when the row max grew by more than 2^8
// (exact: the final normalisation uses the same stale max as the probabilities).
//
// Every wait is bounded (a time limit on %globaltimer): a role that gives up sets a CTA
// abort flag and the per-device error word; every role then stops issuing, the producer
// waits for its own copies in flight, the MMA thread waits for its own MMAs, and the CTA
// frees its tensor memory and exits.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>
#include <cmath>
#include <cstdint>
#include "ra_internal.h"
#include "attn_sched.cuh"
#include "sm100_ptx.cuh"
#include "../../include/ra.h"

namespace ra {

__device__ unsigned int g_ra_error_word = 0;

namespace {

constexpr int kThreads = 384;
// Shard layouts, compiled as separate kernels so that the contiguous layout's per-tile
// softmax keeps plain index arithmetic: positions and sample starts only where they vary.
constexpr int kLayoutContiguous = 0, kLayoutZigzag = 1, kLayoutPacked = 2;
// setmaxnreg split of the launch allocation (168 per thread): the softmax warpgroups rise
// to 192, the third falls to 120 (2 x 128 x 192 + 128 x 120 = 384 x 168).  The host checks
// the compiled register count before the first launch: a raise beyond what the block was
// launched with would never complete.
constexpr uint32_t kRegsLaunch = 168, kRegsSoftmax = 192, kRegsOther = 120;
static_assert(2 * 128 * kRegsSoftmax + 128 * kRegsOther == kThreads * kRegsLaunch,
              "register split must use exactly the launch allocation");
constexpr int kWarpLoad = 8;
constexpr int kWarpMma = 9;
constexpr int kWarpLoadV = 10;
constexpr int kWarpIdle = 11;  // fills the CTA's schedule in the prologue
constexpr int kBM = 128;  // query rows per tile
constexpr int kBN = 128;  // keys per tile
static_assert(kBN == kSchedTile, "the schedule counts tiles of kBN keys");
constexpr uint32_t kTmemCols = 512;
constexpr float kRescaleThreshold = 8.0f;  // log2 units

// error-word bits
constexpr unsigned kErrProducer = 1u, kErrMma = 2u, kErrSoftmax = 4u, kErrDrain = 8u;

struct __align__(64) AttnParams {
    CUtensorMap tm_q;
    CUtensorMap tm_k[RA_MAX_P];
    CUtensorMap tm_v[RA_MAX_P];
    void* out;
    float* lse;
    int P, B, H_q, H_kv, Lc, L;
    int causal, zigzag, out_bf16, group, n_row_blocks;
    int position_order;  // visit row blocks by descending sequence position (zigzag, see below)
    const int* pid;      // packed samples: position_ids [B][L] (nullptr: one sample per row)
    float scale_log2;
    int inject_stall;
    unsigned long long wait_limit_ns;
};

template <int D>
struct Cfg {
    static constexpr int TILE = kBM * D * 2;  // bytes of a 128 x D bf16 tile
    static constexpr int NKB = D / 64;        // 64-column (128-byte) swizzle blocks per tile
    static constexpr int BLK = kBM * 128;     // bytes of one swizzle block (16 KB)
    // K is needed first in each step (S = Q K^T right after the previous P V), so its ring
    // is the deeper one.  D = 128: 64 KB Q + 3 x 32 KB K + 2 x 32 KB V = 224 KB.
    static constexpr int NSK = (D == 128) ? 3 : 4;
    static constexpr int NSV = (D == 128) ? 2 : 4;
    static constexpr int OFF_Q = 0;
    static constexpr int OFF_K = 2 * TILE;
    static constexpr int OFF_V = OFF_K + NSK * TILE;
    static constexpr int OFF_BAR = OFF_V + NSV * TILE;
    // barriers: q_full, k_full[NSK], k_empty[NSK], v_full[NSV], v_empty[NSV], s_full[2],
    // p_full[2], o_full[2], drain, s_free[2] (softmax w has read S), pv_done[2]
    static constexpr int N_BARS = 1 + 2 * NSK + 2 * NSV + 2 + 2 + 2 + 1 + 2 + 2;
    // tmem base (4 B), abort flag (4 B), the schedule's tile count (4 B)
    static constexpr int OFF_MISC = OFF_BAR + N_BARS * 8;
    static constexpr int OFF_SCHED = OFF_MISC + 16;  // tile ranges: RA_MAX_P starts, RA_MAX_P ends
    static constexpr int SMEM = OFF_SCHED + 2 * RA_MAX_P * 4 + 1024;  // + 1024-B alignment slack
    static constexpr int BAR_Q = 0;
    __host__ __device__ static constexpr int bar_kf(int s) { return 1 + s; }
    __host__ __device__ static constexpr int bar_ke(int s) { return 1 + NSK + s; }
    __host__ __device__ static constexpr int bar_vf(int s) { return 1 + 2 * NSK + s; }
    __host__ __device__ static constexpr int bar_ve(int s) { return 1 + 2 * NSK + NSV + s; }
    __host__ __device__ static constexpr int bar_sf(int w) { return 1 + 2 * NSK + 2 * NSV + w; }
    __host__ __device__ static constexpr int bar_pf(int w) { return 3 + 2 * NSK + 2 * NSV + w; }
    __host__ __device__ static constexpr int bar_of(int w) { return 5 + 2 * NSK + 2 * NSV + w; }
    static constexpr int BAR_DRAIN = 7 + 2 * NSK + 2 * NSV;
    __host__ __device__ static constexpr int bar_sfree(int w) { return 8 + 2 * NSK + 2 * NSV + w; }
    __host__ __device__ static constexpr int bar_pvd(int w) { return 10 + 2 * NSK + 2 * NSV + w; }
    static constexpr uint32_t S_COL = 0;
    static constexpr uint32_t P_COL0 = 128, P_COL1 = 192;
    static constexpr uint32_t O_COL0 = 256, O_COL1 = 256 + D;
    static_assert(O_COL1 + D <= kTmemCols, "tensor memory budget");
    static_assert(SMEM <= 232448, "shared memory budget");
};

__device__ __forceinline__ void raise_abort(volatile int* abort_flag, unsigned code) {
    *abort_flag = 1;
    atomicOr(&g_ra_error_word, code);
}

// Single-thread bounded wait.  Gives up when the CTA aborted or after `limit` ns.
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

// Bounded wait that ignores the abort flag: used to drain work this thread started.
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
                                       unsigned long long limit) {
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
                    raise_abort(abort_flag, kErrSoftmax);
                    stop = 1;
                }
            }
            if (__shfl_sync(FULL, stop, 0)) return false;
        }
    }
}

// K/V producer: one thread streams either the K tiles (and first the two Q tiles) or the
// V tiles of the CTA's schedule through its ring, each with its own bounded waits.
template <int D, bool IS_K>
__device__ __forceinline__ void producer(const AttnParams& p, uint32_t base, const Sched& sched,
                                         int n, int b, int h, int g, int r0,
                                         volatile int* abort_flag) {
    using C = Cfg<D>;
    constexpr int NS = IS_K ? C::NSK : C::NSV;
    auto bar = [&](int i) { return base + C::OFF_BAR + 8u * (uint32_t)i; };
    auto bar_full = [&](int s) { return bar(IS_K ? C::bar_kf(s) : C::bar_vf(s)); };
    auto bar_empty = [&](int s) { return bar(IS_K ? C::bar_ke(s) : C::bar_ve(s)); };
    const uint32_t ring = base + (IS_K ? C::OFF_K : C::OFF_V);
    const CUtensorMap* maps = IS_K ? p.tm_k : p.tm_v;
    const unsigned long long lim = p.wait_limit_ns;
    int armed[NS];
#pragma unroll
    for (int s = 0; s < NS; ++s) armed[s] = -1;

    if (IS_K) {
        mbar_arrive_expect_tx(bar(C::BAR_Q), 2 * C::TILE);
#pragma unroll
        for (int kb = 0; kb < C::NKB; ++kb) {
            tma_load_4d(base + C::OFF_Q + kb * C::BLK, &p.tm_q, bar(C::BAR_Q), kb * 64, h, r0, b);
            tma_load_4d(base + C::OFF_Q + C::TILE + kb * C::BLK, &p.tm_q, bar(C::BAR_Q), kb * 64,
                        h, r0 + kBM, b);
        }
    }
    SchedIter it;
    it.begin(sched);
    for (int jt = 0; jt < n; ++jt, it.next()) {
        const int slot = jt % NS;
        if (jt >= NS && !wait1(bar_empty(slot), ((jt / NS) - 1) & 1, abort_flag, lim, kErrProducer))
            break;
        // Test hook: withhold the last K tile so the consumer's bounded wait expires.
        if (IS_K && p.inject_stall && jt == n - 1) continue;
        mbar_arrive_expect_tx(bar_full(slot), C::TILE);
#pragma unroll
        for (int kb = 0; kb < C::NKB; ++kb)
            tma_load_4d(ring + slot * C::TILE + kb * C::BLK, &maps[it.chunk()], bar_full(slot),
                        kb * 64, g, it.t * kBN, b);
        armed[slot] = jt;
    }
    // Drain: every copy this thread started must have landed before the CTA exits.
    if (IS_K) wait_drain(bar(C::BAR_Q), 0, abort_flag, lim);
#pragma unroll
    for (int s = 0; s < NS; ++s)
        if (armed[s] >= 0) wait_drain(bar_full(s), (armed[s] / NS) & 1, abort_flag, lim);
}

template <int D>
__device__ __forceinline__ void mma_issuer(const AttnParams& p, uint32_t base, uint32_t tmem,
                                           int n, volatile int* abort_flag) {
    using C = Cfg<D>;
    auto bar = [&](int i) { return base + C::OFF_BAR + 8u * (uint32_t)i; };
    const unsigned long long lim = p.wait_limit_ns;
    constexpr uint32_t IDESC_S = idesc_bf16_f32(kBM, kBN, 0);  // K-major Q and K
    constexpr uint32_t IDESC_O = idesc_bf16_f32(kBM, D, 1);    // V is MN-major (D contiguous)
    const uint32_t p_col[2] = {C::P_COL0, C::P_COL1};
    const uint32_t o_col[2] = {C::O_COL0, C::O_COL1};

    // Descriptors are built once per operand tile; a K step only moves the start address,
    // which lives in the low 14 bits (address >> 4) and never carries out of them here
    // (shared memory < 256 KB).
    const uint64_t dq[2] = {desc_sw128(base + C::OFF_Q, 16, 1024),
                            desc_sw128(base + C::OFF_Q + C::TILE, 16, 1024)};
    const uint64_t dk0 = desc_sw128(base + C::OFF_K, 16, 1024);
    const uint64_t dv0 = desc_sw128(base + C::OFF_V, C::BLK, 1024);
    // S = Q_w K^T over D in steps of 16: step kk lives in swizzle block kk/4 at byte 32*(kk%4).
    auto issue_s = [&](int w, int slot) {
        const uint64_t dk = dk0 + (uint64_t)((slot * C::TILE) >> 4);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t off = ((kk / 4) * C::BLK + (kk % 4) * 32) >> 4;
            mma_ss(tmem + C::S_COL, dq[w] + off, dk + off, IDESC_S, kk > 0 ? 1u : 0u);
        }
    };
    // O_w (+)= P_w V over 128 keys in steps of 16: P from TMEM (8 columns of bf16 pairs per
    // step), V rows at 128-byte pitch (16 keys = 2048 B), 64-wide D blocks 16 KB apart.
    auto issue_pv = [&](int w, int slot, bool acc) {
        const uint64_t dv = dv0 + (uint64_t)((slot * C::TILE) >> 4);
#pragma unroll
        for (int kk = 0; kk < kBN / 16; ++kk)
            mma_ts(tmem + o_col[w], tmem + p_col[w] + kk * 8, dv + (uint64_t)((kk * 2048) >> 4),
                   IDESC_O, (acc || kk > 0) ? 1u : 0u);
    };

    bool issued = false;
    if (wait1(bar(C::BAR_Q), 0, abort_flag, lim, kErrMma) &&
        wait1(bar(C::bar_kf(0)), 0, abort_flag, lim, kErrMma)) {
        tc_fence_after();
        issue_s(0, 0);
        tc_commit(bar(C::bar_sf(0)));
        issued = true;
        // S_B(0) goes into S once softmax A has read S_A(0) out of it
        if (wait1(bar(C::bar_sfree(0)), 0, abort_flag, lim, kErrMma)) {
            tc_fence_after();
            issue_s(1, 0);
            tc_commit(bar(C::bar_sf(1)));
            tc_commit(bar(C::bar_ke(0)));
            for (int jt = 0; jt < n; ++jt) {
                const int slot_v = jt % C::NSV;
                const int slot_k = (jt + 1) % C::NSK;
                const bool more = jt + 1 < n;
                if (more) {  // S_A(j+1): softmax B has read S_B(j), K(j+1) has landed
                    if (!wait1(bar(C::bar_sfree(1)), jt & 1, abort_flag, lim, kErrMma)) break;
                    if (!wait1(bar(C::bar_kf(slot_k)), ((jt + 1) / C::NSK) & 1, abort_flag, lim,
                               kErrMma))
                        break;
                    tc_fence_after();
                    issue_s(0, slot_k);
                    tc_commit(bar(C::bar_sf(0)));
                }
                if (!wait1(bar(C::bar_vf(slot_v)), (jt / C::NSV) & 1, abort_flag, lim, kErrMma))
                    break;
                if (!wait1(bar(C::bar_pf(0)), jt & 1, abort_flag, lim, kErrMma)) break;
                tc_fence_after();
                issue_pv(0, slot_v, jt > 0);
                tc_commit(bar(C::bar_pvd(0)));
                if (!more) tc_commit(bar(C::bar_of(0)));
                if (more) {  // S_B(j+1): softmax A has read S_A(j+1)
                    if (!wait1(bar(C::bar_sfree(0)), (jt + 1) & 1, abort_flag, lim, kErrMma))
                        break;
                    tc_fence_after();
                    issue_s(1, slot_k);
                    tc_commit(bar(C::bar_sf(1)));
                    tc_commit(bar(C::bar_ke(slot_k)));
                }
                if (!wait1(bar(C::bar_pf(1)), jt & 1, abort_flag, lim, kErrMma)) break;
                tc_fence_after();
                issue_pv(1, slot_v, jt > 0);
                tc_commit(bar(C::bar_pvd(1)));
                tc_commit(bar(C::bar_ve(slot_v)));
                if (!more) tc_commit(bar(C::bar_of(1)));
            }
        }
    }
    if (issued) {  // every MMA this thread issued completes before TMEM is released
        tc_commit(bar(C::BAR_DRAIN));
        wait_drain(bar(C::BAR_DRAIN), 0, abort_flag, lim);
    }
}

template <int D, int LAYOUT>
__device__ __forceinline__ void softmax_wg(const AttnParams& p, uint32_t base, uint32_t tmem,
                                           const Sched& sched, int n, int wg, int b, int h,
                                           int r0, volatile int* abort_flag) {
    using C = Cfg<D>;
    auto bar = [&](int i) { return base + C::OFF_BAR + 8u * (uint32_t)i; };
    const unsigned long long lim = p.wait_limit_ns;
    const unsigned FULL = 0xffffffffu;
    const int wr = (threadIdx.x >> 5) & 3;  // warp within the warpgroup = TMEM lane quarter
    const int lane = threadIdx.x & 31;
    const int q_lo = r0 + wg * kBM;
    const long long my_row = (long long)q_lo + wr * 32 + lane;
    // Sequence positions (L <= 2^30, so 32-bit): this thread's row, and the smallest among
    // the tile's rows (a key tile needs a mask only if some key comes after it).
    constexpr int ZZ = LAYOUT == kLayoutZigzag ? 1 : 0;
    constexpr bool PACKED = LAYOUT == kLayoutPacked;
    const int my_pos =
        my_row < p.L ? (int)shard_pos(ZZ, p.P, p.Lc, (int)(my_row / p.Lc), my_row % p.Lc)
                     : p.L;
    // packed samples: the first key position this row may see (its sample's start)
    int my_start = 0;
    if (PACKED && my_row < p.L) {
        const int r = (int)my_row, st = r - p.pid[(long long)b * p.L + r];
        my_start = st < 0 ? 0 : (st > r ? r : st);
    }
    int tile_qmin = p.L;
    if (q_lo < p.L) {
        long long lo_pos, hi_pos;
        row_pos_range(ZZ, p.P, p.Lc, q_lo, min((long long)q_lo + kBM - 1, (long long)p.L - 1),
                      lo_pos, hi_pos);
        tile_qmin = (int)lo_pos;
    }
    const uint32_t lane_off = (uint32_t)(wr * 32) << 16;
    const uint32_t tS = tmem + lane_off + C::S_COL;
    const uint32_t tP = tmem + lane_off + (wg ? C::P_COL1 : C::P_COL0);
    const uint32_t tO = tmem + lane_off + (wg ? C::O_COL1 : C::O_COL0);
    const float sl2 = p.scale_log2;

    // l_run: normaliser of the fp32 probabilities (gives the LSE); l_used: normaliser of
    // the bf16-rounded probabilities that enter P.V (divides O, so that the weights applied
    // to V sum to one exactly as used).
    float m_run = -INFINITY, l_run = 0.f, l_used = 0.f;
    bool ok = true;
    SchedIter it;
    it.begin(sched);
    for (int jt = 0; jt < n; ++jt, it.next()) {
        if (!wait_warp(bar(C::bar_sf(wg)), jt & 1, abort_flag, lim)) {
            ok = false;
            break;
        }
        __syncwarp();
        tc_fence_after();
        uint64_t s2[64];  // the row's 128 scores as pairs (2i, 2i+1)
        tmem_ld128_pairs(tS, s2);
        // the scores are in registers: S may take the other tile's next scores
        tc_fence_before();
        mbar_arrive(bar(C::bar_sfree(wg)));

        const int j = it.chunk(), key0 = it.t * kBN;  // chunk and first local key of the tile
        const int kvalid = min(kBN, p.Lc - key0);
        const bool need_mask =
            (kvalid < kBN) ||
            (p.causal && (int)shard_pos(ZZ, p.P, p.Lc, j, key0 + kvalid - 1) > tile_qmin) ||
            (PACKED && my_start > (int)shard_pos(ZZ, p.P, p.Lc, j, key0));
        if (need_mask) {
            // The keys of the tile this row sees form one interval [c_lo, c_hi]: key c sits
            // at position kpos0 + c, except that a zigzag tile straddling the shard's two
            // segments continues from c = cs at the second segment's start -- and a row that
            // sees any key of the second segment sees every key of the first.  c_lo > 0
            // only for packed samples (keys before the row's sample start).
            const int kpos0 = (int)shard_pos(ZZ, p.P, p.Lc, j, key0);
            auto clamp_c = [](int x) { return x < -1 ? -1 : (x > kBN ? kBN : x); };
            int c_hi = kvalid - 1;
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
            const int c_lo = PACKED ? clamp_c(my_start - kpos0) : -1;
#pragma unroll
            for (int i = 0; i < 64; ++i) {
                float a, b;
                f2_unpack(s2[i], a, b);
                if (2 * i < c_lo || 2 * i > c_hi) a = -INFINITY;
                if (2 * i + 1 < c_lo || 2 * i + 1 > c_hi) b = -INFINITY;
                s2[i] = f2_pack(a, b);
            }
        }
        // row max over all 128 columns: four chains of three-input max, 8 columns per step
        float mx0, mx1, mx2, mx3;
        {
            float a, b;
            f2_unpack(s2[0], a, b); mx0 = fmaxf(a, b);
            f2_unpack(s2[1], a, b); mx1 = fmaxf(a, b);
            f2_unpack(s2[2], a, b); mx2 = fmaxf(a, b);
            f2_unpack(s2[3], a, b); mx3 = fmaxf(a, b);
#pragma unroll
            for (int i = 4; i < 64; i += 4) {
                f2_unpack(s2[i], a, b); mx0 = fmax3(mx0, a, b);
                f2_unpack(s2[i + 1], a, b); mx1 = fmax3(mx1, a, b);
                f2_unpack(s2[i + 2], a, b); mx2 = fmax3(mx2, a, b);
                f2_unpack(s2[i + 3], a, b); mx3 = fmax3(mx3, a, b);
            }
        }
        const float mx = fmaxf(fmax3(mx0, mx1, mx2), mx3);
        const float m_new = fmaxf(m_run, mx * sl2);
        float alpha = 1.f;
        bool resc = false;
        if (jt == 0) {
            m_run = m_new;
        } else if (m_new - m_run > kRescaleThreshold) {
            alpha = ex2_approx(m_run - m_new);
            m_run = m_new;
            resc = true;
        }
        const float neg_m = (m_run == -INFINITY) ? 0.f : -m_run;
        // P = 2^(s*scale*log2e - m) in bf16 pairs into this tile's P columns, one 64-key
        // half at a time.  P(j-1) there is overwritten only once PV(j-1) has read it.
        const uint64_t sl2x2 = f2_pack(sl2, sl2), negm_x2 = f2_pack(neg_m, neg_m);
        uint64_t sum_a = 0, sum_b = 0, used_a = 0, used_b = 0;  // (0.f, 0.f) pairs
#pragma unroll
        for (int half = 0; half < 2; ++half) {
            uint32_t pk[32];
#pragma unroll
            for (int c2 = 0; c2 < 32; ++c2) {
                if (c2 & 1)
                    pk[c2] = softmax_pair(s2[half * 32 + c2], sl2x2, negm_x2, sum_b, used_b);
                else
                    pk[c2] = softmax_pair(s2[half * 32 + c2], sl2x2, negm_x2, sum_a, used_a);
            }
            if (half == 0 && jt > 0) {
                if (!wait_warp(bar(C::bar_pvd(wg)), (jt - 1) & 1, abort_flag, lim)) {
                    ok = false;
                    break;
                }
                __syncwarp();
                tc_fence_after();
            }
            tmem_st32(tP + half * 32, pk);
        }
        if (!ok) break;
        float s0, s1, u0, u1;
        f2_unpack(f2_add(sum_a, sum_b), s0, s1);
        f2_unpack(f2_add(used_a, used_b), u0, u1);
        l_run = l_run * alpha + (s0 + s1);
        l_used = l_used * alpha + (u0 + u1);
        if (__any_sync(FULL, resc)) {
            // PV of the previous tile is complete: its commit (pv_done) was awaited above.
#pragma unroll
            for (int cb = 0; cb < D / 32; ++cb) {
                uint32_t o[32];
                tmem_ld32(tO + cb * 32, o);
                tmem_wait_ld();
#pragma unroll
                for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
                tmem_st32(tO + cb * 32, o);
            }
        }
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(bar(C::bar_pf(wg)));
    }
    if (ok && !wait_warp(bar(C::bar_of(wg)), 0, abort_flag, lim)) ok = false;
    if (!ok) return;
    __syncwarp();
    tc_fence_after();

    const bool row_ok = my_row < p.L;
    const float inv_l = 1.f / l_used;
    const long long orow = ((long long)b * p.L + my_row) * p.H_q + h;
#pragma unroll
    for (int cb = 0; cb < D / 32; ++cb) {
        uint32_t o[32];
        tmem_ld32(tO + cb * 32, o);
        tmem_wait_ld();
        if (row_ok) {
            if (!p.out_bf16) {
                float4* dst = reinterpret_cast<float4*>((float*)p.out + orow * D + cb * 32);
#pragma unroll
                for (int i = 0; i < 8; ++i)
                    dst[i] = make_float4(__uint_as_float(o[4 * i]) * inv_l,
                                         __uint_as_float(o[4 * i + 1]) * inv_l,
                                         __uint_as_float(o[4 * i + 2]) * inv_l,
                                         __uint_as_float(o[4 * i + 3]) * inv_l);
            } else {
                uint4* dst = reinterpret_cast<uint4*>((uint16_t*)p.out + orow * D + cb * 32);
#pragma unroll
                for (int i = 0; i < 4; ++i)
                    dst[i] = make_uint4(
                        pack_bf16x2(__uint_as_float(o[8 * i]) * inv_l, __uint_as_float(o[8 * i + 1]) * inv_l),
                        pack_bf16x2(__uint_as_float(o[8 * i + 2]) * inv_l, __uint_as_float(o[8 * i + 3]) * inv_l),
                        pack_bf16x2(__uint_as_float(o[8 * i + 4]) * inv_l, __uint_as_float(o[8 * i + 5]) * inv_l),
                        pack_bf16x2(__uint_as_float(o[8 * i + 6]) * inv_l, __uint_as_float(o[8 * i + 7]) * inv_l));
            }
        }
    }
    if (row_ok)
        p.lse[((long long)b * p.H_q + h) * p.L + my_row] =
            (m_run + lg2_approx(l_run)) * 0.69314718055994530942f;
}

template <int D, int LAYOUT>
__global__ void __launch_bounds__(kThreads, 1) attn_fwd_sm100(const __grid_constant__ AttnParams p) {
    using C = Cfg<D>;
    extern __shared__ uint8_t smem_raw[];
    uint32_t base = smem_u32(smem_raw);
    const uint32_t pad = (1024u - (base & 1023u)) & 1023u;
    base += pad;
    uint8_t* smem = smem_raw + pad;
    volatile uint32_t* tmem_slot = reinterpret_cast<volatile uint32_t*>(smem + C::OFF_MISC);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::OFF_MISC + 4);
    auto bar = [&](int i) { return base + C::OFF_BAR + 8u * (uint32_t)i; };

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    // Grid order: (batch, kv head) outermost, then 256-row blocks heaviest first (the rows
    // at the latest sequence positions see the most keys when causal), then the query heads
    // sharing that kv head.  The CTAs resident at any time then stream the same K/V tiles
    // in near lockstep, so K/V are read from HBM about once per (batch, kv head) and served
    // from L2 after that.  In the contiguous layout the latest positions are the last rows;
    // in the zigzag layout (when each Lc/2-token segment holds whole blocks) the k-th block
    // visited is the one at the k-th latest position: segments 2P-1 down to 0, segment
    // s >= P being the second half of rank 2P-1-s and segment s < P the first half of
    // rank s.
    const int per_bg = p.n_row_blocks * p.group;
    const int bg = (int)(blockIdx.x / per_bg);
    const int rem = (int)(blockIdx.x % per_bg);
    const int kvis = rem / p.group;  // 0 = visited first
    const int b = bg / p.H_kv, g = bg % p.H_kv;
    const int h = g * p.group + rem % p.group;
    int r0 = (p.n_row_blocks - 1 - kvis) * 2 * kBM;
    if (p.position_order) {
        const int hseg = p.Lc / 2, seg_blocks = hseg / (2 * kBM);
        const int seg = 2 * p.P - 1 - kvis / seg_blocks;
        const int bis = seg_blocks - 1 - kvis % seg_blocks;
        const int rank = seg < p.P ? seg : 2 * p.P - 1 - seg;
        r0 = rank * p.Lc + (seg < p.P ? 0 : hseg) + bis * 2 * kBM;
    }

    if (threadIdx.x == 0) {
        mbar_init(bar(C::BAR_Q), 1);
        for (int s = 0; s < C::NSK; ++s) {
            mbar_init(bar(C::bar_kf(s)), 1);
            mbar_init(bar(C::bar_ke(s)), 1);
        }
        for (int s = 0; s < C::NSV; ++s) {
            mbar_init(bar(C::bar_vf(s)), 1);
            mbar_init(bar(C::bar_ve(s)), 1);
        }
        for (int w = 0; w < 2; ++w) {
            mbar_init(bar(C::bar_sf(w)), 1);
            mbar_init(bar(C::bar_pf(w)), 4 * 32);
            mbar_init(bar(C::bar_of(w)), 1);
            mbar_init(bar(C::bar_sfree(w)), 4 * 32);
            mbar_init(bar(C::bar_pvd(w)), 1);
        }
        mbar_init(bar(C::BAR_DRAIN), 1);
        *abort_flag = 0;
        fence_mbar_init();
        fence_proxy_async_smem();
    }
    if (warp == kWarpLoad && lane == 0) {
        tma_prefetch_desc(&p.tm_q);
    }
    uint32_t* sched_range = reinterpret_cast<uint32_t*>(smem + C::OFF_SCHED);
    volatile int* n_slot = reinterpret_cast<volatile int*>(smem + C::OFF_MISC + 8);
    if (warp == kWarpIdle) {
        const long long last_row = min((long long)r0 + 2 * kBM - 1, (long long)p.L - 1);
        SchedArgs sa;
        sa.P = p.P;
        sa.Lc = p.Lc;
        sa.L = p.L;
        sa.causal = p.causal;
        sa.zigzag = p.zigzag;
        sa.pid = p.pid;
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

    if (warp >= 8) {
        regs_decrease<kRegsOther>();
        if (warp == kWarpLoad) {
            if (lane == 0) producer<D, true>(p, base, sched, n, b, h, g, r0, abort_flag);
        } else if (warp == kWarpLoadV) {
            if (lane == 0) producer<D, false>(p, base, sched, n, b, h, g, r0, abort_flag);
        } else if (warp == kWarpMma) {
            if (lane == 0) mma_issuer<D>(p, base, tmem, n, abort_flag);
        }
    } else {
        regs_increase<kRegsSoftmax>();
        softmax_wg<D, LAYOUT>(p, base, tmem, sched, n, warp >> 2, b, h, r0, abort_flag);
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == kWarpMma) {
        __syncwarp();
        tmem_dealloc(tmem, kTmemCols);
    }
}

PFN_cuTensorMapEncodeTiled_v12000 get_encode_fn() {
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
bool encode_tile_map(CUtensorMap* m, const void* ptr, int D, int H, long long rows, int B,
                     long long bstride_elems) {
    auto enc = get_encode_fn();
    if (!enc) return false;
    cuuint64_t dims[4] = {(cuuint64_t)D, (cuuint64_t)H, (cuuint64_t)rows, (cuuint64_t)B};
    cuuint64_t strides[3] = {(cuuint64_t)D * 2, (cuuint64_t)H * D * 2, (cuuint64_t)bstride_elems * 2};
    cuuint32_t box[4] = {64, 1, (cuuint32_t)kBM, 1};
    cuuint32_t estr[4] = {1, 1, 1, 1};
    CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(ptr), dims, strides,
                     box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                     CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

template <int D>
cudaError_t launch_d(const AttnParams& p, int grid, cudaStream_t stream, const char** why) {
    using C = Cfg<D>;
    static int configured_for = -1;
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    decltype(&attn_fwd_sm100<D, kLayoutContiguous>) kernels[3] = {
        attn_fwd_sm100<D, kLayoutContiguous>, attn_fwd_sm100<D, kLayoutZigzag>,
        attn_fwd_sm100<D, kLayoutPacked>};
    if (configured_for != dev) {
        for (auto k : kernels) {
            cudaFuncAttributes fa;
            e = cudaFuncGetAttributes(&fa, k);
            if (e != cudaSuccess) return e;
            if (fa.numRegs != (int)kRegsLaunch) {
                *why = "attention kernel compiled with a register count its register split does not assume";
                return cudaErrorInvalidKernelImage;
            }
            e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
            if (e != cudaSuccess) return e;
        }
        configured_for = dev;
    }
    const int layout = p.pid ? kLayoutPacked : (p.zigzag ? kLayoutZigzag : kLayoutContiguous);
    kernels[layout]<<<grid, kThreads, C::SMEM, stream>>>(p);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_attn_sm100(const AttnArgs& a, unsigned long long wait_limit_ns,
                              int inject_stall, const char** why) {
    static thread_local AttnParams p;  // ~16.6 KB of tensor maps: kept off the stack
    const long long L = (long long)a.P * a.Lc;
    if (!encode_tile_map(&p.tm_q, a.q, a.D, a.H_q, L, a.B, a.q_bstride)) {
        *why = "cuTensorMapEncodeTiled failed for q";
        return cudaErrorInvalidValue;
    }
    for (int j = 0; j < a.P; ++j) {
        if (!encode_tile_map(&p.tm_k[j], a.k_chunks[j], a.D, a.H_kv, a.Lc, a.B, a.kv_bstride) ||
            !encode_tile_map(&p.tm_v[j], a.v_chunks[j], a.D, a.H_kv, a.Lc, a.B, a.kv_bstride)) {
            *why = "cuTensorMapEncodeTiled failed for a K/V chunk";
            return cudaErrorInvalidValue;
        }
    }
    p.out = a.out;
    p.lse = a.lse;
    p.P = a.P;
    p.B = a.B;
    p.H_q = a.H_q;
    p.H_kv = a.H_kv;
    p.Lc = a.Lc;
    p.L = (int)L;
    p.causal = a.causal;
    p.zigzag = a.zigzag;
    p.pid = a.pid;
    p.position_order = a.zigzag && a.causal && a.Lc % (4 * kBM) == 0;
    p.out_bf16 = a.out_bf16;
    p.group = a.H_q / a.H_kv;
    p.n_row_blocks = (int)((L + 2 * kBM - 1) / (2 * kBM));
    p.scale_log2 = (float)((double)a.scale * 1.4426950408889634);
    p.inject_stall = inject_stall;
    p.wait_limit_ns = wait_limit_ns;
    const long long grid = (long long)p.n_row_blocks * a.B * a.H_q;
    if (grid > 0x7fffffffLL) {
        *why = "problem too large for one launch";
        return cudaErrorInvalidValue;
    }
    if (a.D == 128) return launch_d<128>(p, (int)grid, a.stream, why);
    if (a.D == 64) return launch_d<64>(p, (int)grid, a.stream, why);
    *why = "head dimension not supported by the tensor-core path";
    return cudaErrorInvalidValue;
}

cudaError_t read_and_clear_error_word(unsigned int* value) {
    cudaError_t e = cudaMemcpyFromSymbol(value, g_ra_error_word, sizeof(unsigned int));
    if (e != cudaSuccess) return e;
    if (*value) {
        const unsigned int zero = 0;
        e = cudaMemcpyToSymbol(g_ra_error_word, &zero, sizeof(unsigned int));
    }
    return e;
}

}  // namespace ra
