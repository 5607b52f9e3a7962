// sm100_ptx.cuh -- thin inline-PTX wrappers for the Blackwell (sm_100a) features the
// attention kernel uses: mbarriers, TMA tiled loads, tcgen05 (TMEM alloc, MMA, ld/st,
// commit, fences), plus the shared-memory matrix and instruction descriptors.
#pragma once
#include <cstdint>

namespace ra {

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint64_t global_timer_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// ------------------------------------------------------------------ mbarrier
__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}
__device__ __forceinline__ void fence_mbar_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ void fence_proxy_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
                 : "memory");
}
// One non-blocking probe: true once the phase with parity `parity` has completed.
__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    return ok != 0;
}

// ------------------------------------------------------------------ TMA
__device__ __forceinline__ void tma_prefetch_desc(const void* tmap) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(tmap)) : "memory");
}
// 4-D tiled load global -> shared, completion signalled on `bar` as transaction bytes.
__device__ __forceinline__ void tma_load_4d(uint32_t dst, const void* tmap, uint32_t bar, int c0,
                                            int c1, int c2, int c3) {
    asm volatile(
        "cp.async.bulk.tensor.4d.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3, %4, %5}], [%6];" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(tmap)), "r"(c0), "r"(c1), "r"(c2), "r"(c3), "r"(bar)
        : "memory");
}

__device__ __forceinline__ void tma_load_5d(uint32_t dst, const void* tmap, uint32_t bar, int c0,
                                            int c1, int c2, int c3, int c4) {
    asm volatile(
        "cp.async.bulk.tensor.5d.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3, %4, %5, %6}], [%7];" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(tmap)), "r"(c0), "r"(c1), "r"(c2), "r"(c3), "r"(c4), "r"(bar)
        : "memory");
}
// Tiled stores shared -> global (bulk-group completion).  Coordinates are never negative.
__device__ __forceinline__ void tma_store_4d(const void* tmap, uint32_t src, int c0, int c1, int c2,
                                             int c3) {
    asm volatile(
        "cp.async.bulk.tensor.4d.global.shared::cta.bulk_group [%0, {%2, %3, %4, %5}], [%1];" ::"l"(
            reinterpret_cast<uint64_t>(tmap)),
        "r"(src), "r"(c0), "r"(c1), "r"(c2), "r"(c3)
        : "memory");
}
__device__ __forceinline__ void tma_store_5d(const void* tmap, uint32_t src, int c0, int c1, int c2,
                                             int c3, int c4) {
    asm volatile(
        "cp.async.bulk.tensor.5d.global.shared::cta.bulk_group [%0, {%2, %3, %4, %5, %6}], [%1];" ::"l"(
            reinterpret_cast<uint64_t>(tmap)),
        "r"(src), "r"(c0), "r"(c1), "r"(c2), "r"(c3), "r"(c4)
        : "memory");
}
// 4-D tiled reduce-add shared -> global (bulk-group completion): every element of the box is
// added to the global element in the tensor map's type (fp32 here); elements past the
// tensor's extent are skipped.  Coordinates are never negative.
__device__ __forceinline__ void tma_reduce_add_4d(const void* tmap, uint32_t src, int c0, int c1,
                                                  int c2, int c3) {
    asm volatile(
        "cp.reduce.async.bulk.tensor.4d.global.shared::cta.add.tile.bulk_group"
        " [%0, {%2, %3, %4, %5}], [%1];" ::"l"(reinterpret_cast<uint64_t>(tmap)),
        "r"(src), "r"(c0), "r"(c1), "r"(c2), "r"(c3)
        : "memory");
}
__device__ __forceinline__ void st_shared_v4(uint32_t addr, uint32_t a, uint32_t b, uint32_t c,
                                             uint32_t d) {
    asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(a), "r"(b), "r"(c),
                 "r"(d)
                 : "memory");
}
__device__ __forceinline__ void bulk_commit() {
    asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}
// Wait until at most N committed bulk groups still read shared memory.
template <int N>
__device__ __forceinline__ void bulk_wait_read() {
    asm volatile("cp.async.bulk.wait_group.read %0;" ::"n"(N) : "memory");
}
// Wait until every committed bulk group has completed (writes done).
__device__ __forceinline__ void bulk_wait_all() {
    asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
}

// ------------------------------------------------------------------ tcgen05
__device__ __forceinline__ void tmem_alloc(uint32_t dst_smem, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst_smem),
                 "r"(ncols)
                 : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
                 : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
// Arrive once on `bar` when every tcgen05 async op issued so far by this thread is done.
__device__ __forceinline__ void tc_commit(uint32_t bar) {
    asm volatile(
        "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
        : "memory");
}
// D[tmem] (+)= A[smem desc] * B[smem desc]^T, kind::f16 (bf16 in, fp32 accumulate).
__device__ __forceinline__ void mma_ss(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                       uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}
// D[tmem] (+)= A[tmem] * B[smem desc], kind::f16.
__device__ __forceinline__ void mma_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc,
                                       uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
        "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}

#define RA_R32(a) "=r"(a[0]), "=r"(a[1]), "=r"(a[2]), "=r"(a[3]), "=r"(a[4]), "=r"(a[5]), \
    "=r"(a[6]), "=r"(a[7]), "=r"(a[8]), "=r"(a[9]), "=r"(a[10]), "=r"(a[11]), "=r"(a[12]), \
    "=r"(a[13]), "=r"(a[14]), "=r"(a[15]), "=r"(a[16]), "=r"(a[17]), "=r"(a[18]), "=r"(a[19]), \
    "=r"(a[20]), "=r"(a[21]), "=r"(a[22]), "=r"(a[23]), "=r"(a[24]), "=r"(a[25]), "=r"(a[26]), \
    "=r"(a[27]), "=r"(a[28]), "=r"(a[29]), "=r"(a[30]), "=r"(a[31])
#define RA_W32(a) "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(a[4]), "r"(a[5]), "r"(a[6]), \
    "r"(a[7]), "r"(a[8]), "r"(a[9]), "r"(a[10]), "r"(a[11]), "r"(a[12]), "r"(a[13]), "r"(a[14]), \
    "r"(a[15]), "r"(a[16]), "r"(a[17]), "r"(a[18]), "r"(a[19]), "r"(a[20]), "r"(a[21]), \
    "r"(a[22]), "r"(a[23]), "r"(a[24]), "r"(a[25]), "r"(a[26]), "r"(a[27]), "r"(a[28]), \
    "r"(a[29]), "r"(a[30]), "r"(a[31])

// Each thread of the warp reads 32 consecutive 32-bit columns of its own TMEM lane.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "
        "%11, %12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, "
        "%28, %29, %30, %31}, [%32];"
        : RA_R32(r)
        : "r"(taddr));
}
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "
        "%11, %12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, "
        "%28, %29, %30, %31, %32};" ::"r"(taddr),
        RA_W32(r)
        : "memory");
}
__device__ __forceinline__ void tmem_wait_ld() {
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_wait_st() {
    asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}


// All 128 fp32 columns of this thread's TMEM lane as 64 register pairs (column 2i in the
// low half of pair i), loaded and waited for in one block so that every pair is an
// aligned 64-bit register ready for the packed f32x2 instructions.
__device__ __forceinline__ void tmem_ld128_pairs(uint32_t taddr, uint64_t (&o)[64]) {
    asm volatile(
        "{\n\t.reg .b32 r0, r1, r2, r3, r4, r5, r6, r7, r8, r9, r10, r11, r12, r13, r14, r15, r16, r17, r18, r19, r20, r21, r22, r23, r24, r25, r26, r27, r28, r29, r30, r31, r32, r33, r34, r35, r36, r37, r38, r39, r40, r41, r42, r43, r44, r45, r46, r47, r48, r49, r50, r51, r52, r53, r54, r55, r56, r57, r58, r59, r60, r61, r62, r63, r64, r65, r66, r67, r68, r69, r70, r71, r72, r73, r74, r75, r76, r77, r78, r79, r80, r81, r82, r83, r84, r85, r86, r87, r88, r89, r90, r91, r92, r93, r94, r95, r96, r97, r98, r99, r100, r101, r102, r103, r104, r105, r106, r107, r108, r109, r110, r111, r112, r113, r114, r115, r116, r117, r118, r119, r120, r121, r122, r123, r124, r125, r126, r127;\n\t"
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {r0, r1, r2, r3, r4, r5, r6, r7, r8, r9, r10, r11, r12, r13, r14, r15, r16, r17, r18, r19, r20, r21, r22, r23, r24, r25, r26, r27, r28, r29, r30, r31}, [%64];\n\t"
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {r32, r33, r34, r35, r36, r37, r38, r39, r40, r41, r42, r43, r44, r45, r46, r47, r48, r49, r50, r51, r52, r53, r54, r55, r56, r57, r58, r59, r60, r61, r62, r63}, [%65];\n\t"
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {r64, r65, r66, r67, r68, r69, r70, r71, r72, r73, r74, r75, r76, r77, r78, r79, r80, r81, r82, r83, r84, r85, r86, r87, r88, r89, r90, r91, r92, r93, r94, r95}, [%66];\n\t"
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {r96, r97, r98, r99, r100, r101, r102, r103, r104, r105, r106, r107, r108, r109, r110, r111, r112, r113, r114, r115, r116, r117, r118, r119, r120, r121, r122, r123, r124, r125, r126, r127}, [%67];\n\t"
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
        "mov.b64 %32, {r64, r65};\n\t"
        "mov.b64 %33, {r66, r67};\n\t"
        "mov.b64 %34, {r68, r69};\n\t"
        "mov.b64 %35, {r70, r71};\n\t"
        "mov.b64 %36, {r72, r73};\n\t"
        "mov.b64 %37, {r74, r75};\n\t"
        "mov.b64 %38, {r76, r77};\n\t"
        "mov.b64 %39, {r78, r79};\n\t"
        "mov.b64 %40, {r80, r81};\n\t"
        "mov.b64 %41, {r82, r83};\n\t"
        "mov.b64 %42, {r84, r85};\n\t"
        "mov.b64 %43, {r86, r87};\n\t"
        "mov.b64 %44, {r88, r89};\n\t"
        "mov.b64 %45, {r90, r91};\n\t"
        "mov.b64 %46, {r92, r93};\n\t"
        "mov.b64 %47, {r94, r95};\n\t"
        "mov.b64 %48, {r96, r97};\n\t"
        "mov.b64 %49, {r98, r99};\n\t"
        "mov.b64 %50, {r100, r101};\n\t"
        "mov.b64 %51, {r102, r103};\n\t"
        "mov.b64 %52, {r104, r105};\n\t"
        "mov.b64 %53, {r106, r107};\n\t"
        "mov.b64 %54, {r108, r109};\n\t"
        "mov.b64 %55, {r110, r111};\n\t"
        "mov.b64 %56, {r112, r113};\n\t"
        "mov.b64 %57, {r114, r115};\n\t"
        "mov.b64 %58, {r116, r117};\n\t"
        "mov.b64 %59, {r118, r119};\n\t"
        "mov.b64 %60, {r120, r121};\n\t"
        "mov.b64 %61, {r122, r123};\n\t"
        "mov.b64 %62, {r124, r125};\n\t"
        "mov.b64 %63, {r126, r127};\n\t"
        "}"
        : "=l"(o[0]), "=l"(o[1]), "=l"(o[2]), "=l"(o[3]), "=l"(o[4]), "=l"(o[5]), "=l"(o[6]), "=l"(o[7]), "=l"(o[8]), "=l"(o[9]), "=l"(o[10]), "=l"(o[11]), "=l"(o[12]), "=l"(o[13]), "=l"(o[14]), "=l"(o[15]), "=l"(o[16]), "=l"(o[17]), "=l"(o[18]), "=l"(o[19]), "=l"(o[20]), "=l"(o[21]), "=l"(o[22]), "=l"(o[23]), "=l"(o[24]), "=l"(o[25]), "=l"(o[26]), "=l"(o[27]), "=l"(o[28]), "=l"(o[29]), "=l"(o[30]), "=l"(o[31]), "=l"(o[32]), "=l"(o[33]), "=l"(o[34]), "=l"(o[35]), "=l"(o[36]), "=l"(o[37]), "=l"(o[38]), "=l"(o[39]), "=l"(o[40]), "=l"(o[41]), "=l"(o[42]), "=l"(o[43]), "=l"(o[44]), "=l"(o[45]), "=l"(o[46]), "=l"(o[47]), "=l"(o[48]), "=l"(o[49]), "=l"(o[50]), "=l"(o[51]), "=l"(o[52]), "=l"(o[53]), "=l"(o[54]), "=l"(o[55]), "=l"(o[56]), "=l"(o[57]), "=l"(o[58]), "=l"(o[59]), "=l"(o[60]), "=l"(o[61]), "=l"(o[62]), "=l"(o[63])
        : "r"(taddr), "r"(taddr + 32), "r"(taddr + 64), "r"(taddr + 96)
        : "memory");
}

// One column pair of the softmax: x = s * scale_log2 - m (packed), p = 2^x (two MUFU ops),
// pp = bf16x2(p) (the P.V operand), sum += p (fp32, packed) and used += (float)pp (the
// bf16 values as used, each added to its fp32 lane by a mixed-precision add).  All pair
// traffic stays in 64-bit registers.
__device__ __forceinline__ uint32_t softmax_pair(uint64_t s2, uint64_t scale2, uint64_t negm2,
                                                 uint64_t& sum, uint64_t& used) {
    uint32_t pp;
    asm("{\n\t.reg .b32 x0, x1, p0, p1, u0, u1;\n\t.reg .b16 h0, h1;\n\t.reg .b64 x, p;\n\t"
        "fma.rn.f32x2 x, %3, %4, %5;\n\t"
        "mov.b64 {x0, x1}, x;\n\t"
        "ex2.approx.ftz.f32 p0, x0;\n\t"
        "ex2.approx.ftz.f32 p1, x1;\n\t"
        "cvt.rn.bf16x2.f32 %0, p1, p0;\n\t"
        "mov.b64 p, {p0, p1};\n\t"
        "add.rn.f32x2 %1, %1, p;\n\t"
        "mov.b32 {h0, h1}, %0;\n\t"
        "mov.b64 {u0, u1}, %2;\n\t"
        "add.rn.f32.bf16 u0, h0, u0;\n\t"
        "add.rn.f32.bf16 u1, h1, u1;\n\t"
        "mov.b64 %2, {u0, u1};\n\t}"
        : "=r"(pp), "+l"(sum), "+l"(used)
        : "l"(s2), "l"(scale2), "l"(negm2));
    return pp;
}


// ------------------------------------------------------------------ register split
// Per-warpgroup register budget change (all 4 warps of the warpgroup execute it).  The
// sum over the block must stay within what the block was launched with.
template <uint32_t N>
__device__ __forceinline__ void regs_increase() {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(N));
}
template <uint32_t N>
__device__ __forceinline__ void regs_decrease() {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(N));
}

// ------------------------------------------------------------------ math
__device__ __forceinline__ float ex2_approx(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}
__device__ __forceinline__ float lg2_approx(float x) {
    float y;
    asm("lg2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}
// Packed fp32 pairs (sm_100 f32x2 instructions: one issue slot for two lanes of work).
__device__ __forceinline__ uint64_t f2_pack(float lo, float hi) {
    uint64_t r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
    return r;
}
__device__ __forceinline__ void f2_unpack(uint64_t v, float& lo, float& hi) {
    asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
__device__ __forceinline__ uint64_t f2_fma(uint64_t a, uint64_t b, uint64_t c) {
    uint64_t d;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
    return d;
}
__device__ __forceinline__ uint64_t f2_add(uint64_t a, uint64_t b) {
    uint64_t d;
    asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}
// max of three fp32 values in one instruction
__device__ __forceinline__ float fmax3(float a, float b, float c) {
    float d;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
    return d;
}

// Pack two fp32 into bf16x2 (round to nearest even): `lo` in bits 0..15, `hi` in 16..31.
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    uint32_t r;
    asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
    return r;
}

// ------------------------------------------------------------------ descriptors
// Shared-memory matrix descriptor (tcgen05 format): start address, leading and stride
// byte offsets (all >> 4), descriptor version 1 at bits 46-47, 128-byte swizzle (2) at
// bits 61-63.  Base offset 0: every swizzle atom we point into is 1024-byte aligned.
__device__ __forceinline__ uint64_t desc_sw128(uint32_t smem_addr, uint32_t lbo_bytes,
                                               uint32_t sbo_bytes) {
    uint64_t d = 0;
    d |= (uint64_t)((smem_addr >> 4) & 0x3FFFu);
    d |= (uint64_t)((lbo_bytes >> 4) & 0x3FFFu) << 16;
    d |= (uint64_t)((sbo_bytes >> 4) & 0x3FFFu) << 32;
    d |= (uint64_t)1u << 46;
    d |= (uint64_t)2u << 61;
    return d;
}

// Instruction descriptor, kind::f16 with bf16 A/B and fp32 accumulator.
//   bits 4-5 D format (1 = f32), 7-9 A format (1 = bf16), 10-12 B format (1 = bf16),
//   15 A major (0 = K), 16 B major (1 = MN), 17-22 N >> 3, 24-28 M >> 4.
__host__ __device__ constexpr uint32_t idesc_bf16_f32(int M, int N, int b_mn_major) {
    return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)b_mn_major << 16) |
           ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

// The same with A also MN-major (bit 15): both operands with their M / N dimension
// contiguous in shared memory.
__host__ __device__ constexpr uint32_t idesc_bf16_f32_ab(int M, int N, int a_mn_major,
                                                         int b_mn_major) {
    return idesc_bf16_f32(M, N, b_mn_major) | ((uint32_t)a_mn_major << 15);
}

}  // namespace ra
