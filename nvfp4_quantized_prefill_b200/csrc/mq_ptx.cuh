// mq_ptx.cuh -- thin inline-PTX wrappers for sm_100a: mbarriers, TMA and bulk
// copies, and the tcgen05 (5th-generation tensor core / tensor memory)
// instructions used by the block-scaled GEMM.  Every wait is bounded.
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

namespace mq {

// Error bits latched in the per-device error word.
constexpr unsigned kDevErrTimeout = 1u;

// A bounded wait gives up after this many nanoseconds of %globaltimer.
constexpr unsigned long long kWaitLimitNs = 2000000000ull;

__device__ __forceinline__ uint32_t smem_u32(const void *p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ unsigned long long global_timer_ns() {
    unsigned long long t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// ---- mbarrier ---------------------------------------------------------------

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_barrier_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

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

// Waits until the phase with the given parity of the barrier has completed.
// Returns false (after latching kDevErrTimeout and raising *abort) if it takes
// longer than kWaitLimitNs, or if another role already raised *abort.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, volatile int *abort,
                                          unsigned *err, unsigned long long limit_ns = kWaitLimitNs) {
    if (mbar_try_wait(bar, parity)) return true;
    unsigned long long t0 = global_timer_ns();
    for (uint32_t i = 1;; ++i) {
        if (mbar_try_wait(bar, parity)) return true;
        if ((i & 255u) == 0) {
            if (*abort) return false;
            if (global_timer_ns() - t0 > limit_ns) {
                atomicOr(err, kDevErrTimeout);
                *abort = 1;
                return false;
            }
        }
    }
}

// ---- TMA / bulk copies -------------------------------------------------------

__device__ __forceinline__ void tma_load_2d(uint32_t dst, const void *tmap, int32_t x, int32_t y,
                                            uint32_t bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3}], [%4];" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(tmap)), "r"(x), "r"(y), "r"(bar)
        : "memory");
}

// Plain (untiled) bulk copy global -> shared; both addresses 16-byte aligned,
// bytes a multiple of 16.
__device__ __forceinline__ void bulk_load(uint32_t dst, const void *src, uint32_t bytes,
                                          uint32_t bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::
            "r"(dst),
        "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(bar)
        : "memory");
}

// TMA tile store shared -> global (bulk async-group completion); rows or
// columns outside the tensor are not written.
__device__ __forceinline__ void tma_store_2d(const void *tmap, int32_t x, int32_t y, uint32_t src) {
    asm volatile(
        "cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%1, %2}], [%3];" ::"l"(
            reinterpret_cast<uint64_t>(tmap)),
        "r"(x), "r"(y), "r"(src)
        : "memory");
}

// 3-D TMA tile store shared -> global (coordinates innermost first).
__device__ __forceinline__ void tma_store_3d(const void *tmap, int32_t x, int32_t y, int32_t z,
                                             uint32_t src) {
    asm volatile(
        "cp.async.bulk.tensor.3d.global.shared::cta.bulk_group [%0, {%1, %2, %3}], [%4];" ::"l"(
            reinterpret_cast<uint64_t>(tmap)),
        "r"(x), "r"(y), "r"(z), "r"(src)
        : "memory");
}

__device__ __forceinline__ void bulk_commit_group() {
    asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}

// Waits until every committed bulk store of this thread has finished reading
// its shared-memory source.
__device__ __forceinline__ void bulk_wait_group_read0() {
    asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
}

// Waits until every committed bulk store of this thread has completed.
__device__ __forceinline__ void bulk_wait_group0() {
    asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
}

// Orders this thread's generic-proxy shared-memory writes before later
// async-proxy (TMA) reads of them.
__device__ __forceinline__ void fence_proxy_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void st_shared_v4(uint32_t addr, uint32_t a, uint32_t b, uint32_t c,
                                             uint32_t d) {
    asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(a), "r"(b), "r"(c),
                 "r"(d)
                 : "memory");
}

__device__ __forceinline__ void prefetch_tmap(const void *tmap) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(tmap)) : "memory");
}

// ---- clusters (CTA pairs) -------------------------------------------------------

__device__ __forceinline__ uint32_t cluster_ctarank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}

// Address of the same shared-memory offset in CTA `rank` of the cluster.
__device__ __forceinline__ uint32_t mapa_shared(uint32_t addr, uint32_t rank) {
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(addr), "r"(rank));
    return r;
}

// Arrive on an mbarrier given by a shared::cluster address (any CTA of the cluster).
// Arrive on a barrier of the peer CTA with release semantics at CTA scope:
// the signal carries no data the waiter reads through memory, and the
// cluster-scope release form stalls the arriving thread for several hundred
// nanoseconds.
__device__ __forceinline__ void mbar_arrive_remote(uint32_t cluster_addr) {
    asm volatile("mbarrier.arrive.release.cta.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr)
                 : "memory");
}

__device__ __forceinline__ void cluster_sync() {
    asm volatile("barrier.cluster.arrive.release;\n\tbarrier.cluster.wait.acquire;" ::: "memory");
}

// ---- tcgen05, CTA-pair forms (cta_group::2) ----------------------------------------
// Every tcgen05 instruction of a kernel uses the same cta_group; the pair forms
// below are issued by one thread of the even CTA and act on both CTAs' tensor
// memory (each CTA's shared memory supplies its half at the same offset).

__device__ __forceinline__ void tmem_alloc_pair(uint32_t dst, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst),
                 "r"(ncols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_dealloc_pair(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
                 : "memory");
}

// ---- warp-issued forms -------------------------------------------------------------
// Called by all 32 lanes of a warp with warp-uniform operands; one elected lane
// issues the instruction.  Keeping the issuing loop warp-wide lets the operands
// stay warp-uniform instead of being moved per instruction from one lane.

__device__ __forceinline__ void warp_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
    asm volatile(
        "{\n\t.reg .pred e;\n\telect.sync _|e, 0xffffffff;\n\t"
        "@e mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;\n\t}" ::"r"(bar),
        "r"(bytes)
        : "memory");
}

__device__ __forceinline__ void warp_tma_load_2d_pair(uint32_t dst, const void *tmap, int32_t x,
                                                      int32_t y, uint32_t bar_cluster) {
    asm volatile(
        "{\n\t.reg .pred e;\n\telect.sync _|e, 0xffffffff;\n\t"
        "@e cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3}], [%4];\n\t}" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(tmap)), "r"(x), "r"(y), "r"(bar_cluster)
        : "memory");
}

__device__ __forceinline__ void warp_cp_sf_pair(uint32_t taddr, uint64_t sdesc) {
    asm volatile(
        "{\n\t.reg .pred e;\n\telect.sync _|e, 0xffffffff;\n\t"
        "@e tcgen05.cp.cta_group::2.32x128b.warpx4 [%0], %1;\n\t}" ::"r"(taddr),
        "l"(sdesc)
        : "memory");
}

__device__ __forceinline__ void warp_mma_nvf4_pair(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                                   uint32_t idesc, uint32_t sfa_tmem,
                                                   uint32_t sfb_tmem, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p, e;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "elect.sync _|e, 0xffffffff;\n\t"
        "@e tcgen05.mma.cta_group::2.kind::mxf4nvf4.block_scale.block16"
        " [%0], %1, %2, %3, [%5], [%6], p;\n\t}" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(sfa_tmem), "r"(sfb_tmem)
        : "memory");
}

// One K = 256 stage: four paired MMAs (K = 64 each; the A / B descriptors
// advance 32 bytes = 2 descriptor units, the scale columns by 4 / 8) and the
// commit that frees the stage in both CTAs, from one elected lane.  The first
// MMA overwrites the accumulator when `accumulate` is 0.
__device__ __forceinline__ void warp_mma4_commit_pair(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                                      uint32_t idesc, uint32_t sfa_tmem,
                                                      uint32_t sfb_tmem, uint32_t accumulate,
                                                      uint32_t bar, uint16_t cta_mask) {
    asm volatile(
        "{\n\t.reg .pred p, t, e;\n\t"
        ".reg .b64 a1, a2, a3, b1, b2, b3;\n\t"
        ".reg .b32 sa1, sa2, sa3, sb1, sb2, sb3;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "setp.eq.b32 t, 0, 0;\n\t"
        "add.s64 a1, %1, 2;\n\tadd.s64 a2, %1, 4;\n\tadd.s64 a3, %1, 6;\n\t"
        "add.s64 b1, %2, 2;\n\tadd.s64 b2, %2, 4;\n\tadd.s64 b3, %2, 6;\n\t"
        "add.u32 sa1, %5, 4;\n\tadd.u32 sa2, %5, 8;\n\tadd.u32 sa3, %5, 12;\n\t"
        "add.u32 sb1, %6, 8;\n\tadd.u32 sb2, %6, 16;\n\tadd.u32 sb3, %6, 24;\n\t"
        "elect.sync _|e, 0xffffffff;\n\t"
        "@e tcgen05.mma.cta_group::2.kind::mxf4nvf4.block_scale.block16"
        " [%0], %1, %2, %3, [%5], [%6], p;\n\t"
        "@e tcgen05.mma.cta_group::2.kind::mxf4nvf4.block_scale.block16"
        " [%0], a1, b1, %3, [sa1], [sb1], t;\n\t"
        "@e tcgen05.mma.cta_group::2.kind::mxf4nvf4.block_scale.block16"
        " [%0], a2, b2, %3, [sa2], [sb2], t;\n\t"
        "@e tcgen05.mma.cta_group::2.kind::mxf4nvf4.block_scale.block16"
        " [%0], a3, b3, %3, [sa3], [sb3], t;\n\t"
        "@e tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64"
        " [%7], %8;\n\t}" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(sfa_tmem), "r"(sfb_tmem),
        "r"(bar), "h"(cta_mask)
        : "memory");
}

// A copier's share of one stage when two copiers split its four K-blocks:
// K-blocks kb and kb + 2, each its A scale tile and the two B scale tiles
// (512-byte tiles; kb + 2 is 1024 bytes = 64 descriptor units further, and
// 8 / 16 TMEM columns further), from one elected lane.
__device__ __forceinline__ void warp_cp6_pair(uint32_t tsfa, uint32_t tsfb, uint64_t da,
                                              uint64_t db_lo, uint64_t db_hi) {
    asm volatile(
        "{\n\t.reg .pred e;\n\t"
        ".reg .b64 a2, l2, h2;\n\t"
        ".reg .b32 ta2, tb1, tb2, tb3;\n\t"
        "add.s64 a2, %2, 64;\n\tadd.s64 l2, %3, 64;\n\tadd.s64 h2, %4, 64;\n\t"
        "add.u32 ta2, %0, 8;\n\tadd.u32 tb1, %1, 4;\n\t"
        "add.u32 tb2, %1, 16;\n\tadd.u32 tb3, %1, 20;\n\t"
        "elect.sync _|e, 0xffffffff;\n\t"
        "@e tcgen05.cp.cta_group::2.32x128b.warpx4 [%0], %2;\n\t"
        "@e tcgen05.cp.cta_group::2.32x128b.warpx4 [%1], %3;\n\t"
        "@e tcgen05.cp.cta_group::2.32x128b.warpx4 [tb1], %4;\n\t"
        "@e tcgen05.cp.cta_group::2.32x128b.warpx4 [ta2], a2;\n\t"
        "@e tcgen05.cp.cta_group::2.32x128b.warpx4 [tb2], l2;\n\t"
        "@e tcgen05.cp.cta_group::2.32x128b.warpx4 [tb3], h2;\n\t}"
        ::"r"(tsfa), "r"(tsfb), "l"(da), "l"(db_lo), "l"(db_hi)
        : "memory");
}

__device__ __forceinline__ void warp_commit_pair_mc(uint32_t bar, uint16_t cta_mask) {
    asm volatile(
        "{\n\t.reg .pred e;\n\telect.sync _|e, 0xffffffff;\n\t"
        "@e tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64"
        " [%0], %1;\n\t}" ::"r"(bar),
        "h"(cta_mask)
        : "memory");
}

__device__ __forceinline__ void warp_commit_pair(uint32_t bar) {
    asm volatile(
        "{\n\t.reg .pred e;\n\telect.sync _|e, 0xffffffff;\n\t"
        "@e tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%0];\n\t}" ::"r"(
            bar)
        : "memory");
}

// Warp-uniform bounded wait: every lane polls; the warp agrees on the result.
__device__ __forceinline__ bool warp_mbar_wait(uint32_t bar, uint32_t parity, volatile int *abort,
                                               unsigned *err,
                                               unsigned long long limit_ns = kWaitLimitNs) {
    return __all_sync(0xFFFFFFFFu, mbar_wait(bar, parity, abort, err, limit_ns));
}

// ---- tcgen05 -------------------------------------------------------------------

// Allocates `ncols` TMEM columns (power of two >= 32); the whole warp calls it.
// The TMEM address is written to shared memory at `dst`.
__device__ __forceinline__ void tmem_alloc(uint32_t dst, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst),
                 "r"(ncols)
                 : "memory");
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

// Arrive on an mbarrier once every tcgen05 operation issued so far by this
// thread (MMAs, copies) has completed.
__device__ __forceinline__ void tc_commit(uint32_t bar) {
    asm volatile(
        "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
        : "memory");
}

// Copy one 512-byte scale-factor tile (32 rows x 128 bits in shared memory)
// into TMEM columns [taddr, taddr+4), replicated into all four 32-lane groups.
__device__ __forceinline__ void tc_cp_sf(uint32_t taddr, uint64_t sdesc) {
    asm volatile("tcgen05.cp.cta_group::1.32x128b.warpx4 [%0], %1;" ::"r"(taddr), "l"(sdesc)
                 : "memory");
}

// D (TMEM, FP32) (+)= A * B with E2M1 operands from shared memory and UE4M3
// block scales (one per 16 K-elements) from TMEM; M=128, K=64 per call.
__device__ __forceinline__ void tc_mma_nvf4(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                            uint32_t idesc, uint32_t sfa_tmem, uint32_t sfb_tmem,
                                            uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::mxf4nvf4.block_scale.block16"
        " [%0], %1, %2, %3, [%5], [%6], p;\n\t}" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(sfa_tmem), "r"(sfb_tmem)
        : "memory");
}

// 32 lanes x 32 consecutive 32-bit columns: thread t of the warp receives lane
// (warp's lane group base + t), columns [col, col+32).
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32"
        " {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15,"
        " %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31},"
        " [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
          "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]),
          "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
          "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]),
          "=r"(r[31])
        : "r"(taddr));
}

// 32 lanes x 16 consecutive 32-bit columns from registers.
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&r)[16]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0],"
        " {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16};" ::"r"(taddr),
        "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
        "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
        : "memory");
}

__device__ __forceinline__ void tmem_ld_wait() {
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// 32 lanes x 32 consecutive 32-bit columns from registers: thread t of the
// warp writes lane (warp's lane group base + t), columns [col, col+32).
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0],"
        " {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16,"
        " %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32};" ::"r"(taddr),
        "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
        "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]),
        "r"(r[16]), "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]),
        "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31])
        : "memory");
}

// Waits until this thread's tcgen05.st writes have completed.
__device__ __forceinline__ void tmem_st_wait() {
    asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

// ---- tcgen05, single-CTA BF16 forms (kind::f16) -------------------------------------

// D (TMEM, FP32) (+)= A * B over K = 128: eight chained BF16 MMAs (M = 128,
// K = 16 each) with A and B K-major 128-byte-swizzled shared-memory operands
// (descriptors advanced by 32 bytes per step within a 64-column half of the
// 128-column tile, and by 16 KB to the tile's second half after four steps),
// then two commits: each barrier arrives once the MMAs have completed.
__device__ __forceinline__ void tc_mma8_bf16_ss_commit2(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                                        uint32_t idesc, uint32_t accumulate,
                                                        uint32_t bar0, uint32_t bar1) {
    asm volatile(
        "{\n\t.reg .pred p, t;\n\t"
        ".reg .b64 a1, a2, a3, a4, a5, a6, a7, b1, b2, b3, b4, b5, b6, b7;\n\t"
        "setp.ne.b32 p, %4, 0;\n\tsetp.eq.b32 t, 0, 0;\n\t"
        "add.s64 a1, %1, 2;\n\tadd.s64 a2, %1, 4;\n\tadd.s64 a3, %1, 6;\n\t"
        "add.s64 a4, %1, 1024;\n\tadd.s64 a5, %1, 1026;\n\tadd.s64 a6, %1, 1028;\n\t"
        "add.s64 a7, %1, 1030;\n\t"
        "add.s64 b1, %2, 2;\n\tadd.s64 b2, %2, 4;\n\tadd.s64 b3, %2, 6;\n\t"
        "add.s64 b4, %2, 1024;\n\tadd.s64 b5, %2, 1026;\n\tadd.s64 b6, %2, 1028;\n\t"
        "add.s64 b7, %2, 1030;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], a1, b1, %3, t;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], a2, b2, %3, t;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], a3, b3, %3, t;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], a4, b4, %3, t;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], a5, b5, %3, t;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], a6, b6, %3, t;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], a7, b7, %3, t;\n\t"
        "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%5];\n\t"
        "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%6];\n\t}" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(bar0), "r"(bar1)
        : "memory");
}

// Eight chained BF16 MMAs with A from tensor memory (8 columns per K = 16
// step) and B an MN-major shared-memory operand whose K steps are 2048 bytes
// apart (two 8-row groups), then two commits.
__device__ __forceinline__ void tc_mma8_bf16_ts_commit2(uint32_t d_tmem, uint32_t a_tmem, uint64_t bdesc,
                                                        uint32_t idesc, uint32_t accumulate,
                                                        uint32_t bar0, uint32_t bar1) {
    asm volatile(
        "{\n\t.reg .pred p, t;\n\t"
        ".reg .b32 a1, a2, a3, a4, a5, a6, a7;\n\t"
        ".reg .b64 b1, b2, b3, b4, b5, b6, b7;\n\t"
        "setp.ne.b32 p, %4, 0;\n\tsetp.eq.b32 t, 0, 0;\n\t"
        "add.u32 a1, %1, 8;\n\tadd.u32 a2, %1, 16;\n\tadd.u32 a3, %1, 24;\n\t"
        "add.u32 a4, %1, 32;\n\tadd.u32 a5, %1, 40;\n\tadd.u32 a6, %1, 48;\n\t"
        "add.u32 a7, %1, 56;\n\t"
        "add.s64 b1, %2, 128;\n\tadd.s64 b2, %2, 256;\n\tadd.s64 b3, %2, 384;\n\t"
        "add.s64 b4, %2, 512;\n\tadd.s64 b5, %2, 640;\n\tadd.s64 b6, %2, 768;\n\t"
        "add.s64 b7, %2, 896;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [a1], b1, %3, t;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [a2], b2, %3, t;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [a3], b3, %3, t;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [a4], b4, %3, t;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [a5], b5, %3, t;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [a6], b6, %3, t;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [a7], b7, %3, t;\n\t"
        "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%5];\n\t"
        "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%6];\n\t}" ::"r"(d_tmem),
        "r"(a_tmem), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(bar0), "r"(bar1)
        : "memory");
}

// Instruction descriptor of kind::f16 with BF16 A and B and FP32 D: D format
// 1 at bits [4,6), A / B format 1 (BF16) at [7,10) / [10,13), A / B major
// (0 K-major, 1 MN-major) at bits 15 / 16, N >> 3 at [17,23), M >> 4 at [24,29).
__host__ __device__ constexpr uint32_t idesc_bf16(uint32_t M, uint32_t N, uint32_t a_mn,
                                                  uint32_t b_mn) {
    return (1u << 4) | (1u << 7) | (1u << 10) | (a_mn << 15) | (b_mn << 16) | ((N >> 3) << 17) |
           ((M >> 4) << 24);
}

// ---- shared-memory matrix descriptors (tcgen05) ---------------------------------
// Fields: start address >> 4 in bits [0,14), leading byte offset >> 4 in
// [16,30), stride byte offset >> 4 in [32,46), fixed version 1 at bit 46,
// base offset [49,52) = 0, layout type in [61,64) (0 none, 2 = 128-byte swizzle).

// K-major operand tile whose rows are 128 bytes wide, 128-byte swizzled, with
// 8-row groups 1024 bytes apart (the TMA SWIZZLE_128B image of a [rows, 128 B]
// box).  The tile must start on a 1024-byte boundary; a K offset inside the
// 128-byte row is added to the start address.
__device__ __forceinline__ uint64_t sdesc_kmajor_sw128(uint32_t saddr) {
    uint64_t d = 0;
    d |= static_cast<uint64_t>((saddr >> 4) & 0x3FFFu);
    d |= static_cast<uint64_t>(1u) << 16;            // LBO (unused for swizzled K-major)
    d |= static_cast<uint64_t>(1024u >> 4) << 32;    // SBO: 8 rows x 128 B
    d |= static_cast<uint64_t>(1u) << 46;            // version
    d |= static_cast<uint64_t>(2u) << 61;            // SWIZZLE_128B
    return d;
}

// MN-major operand tile with 128-byte swizzle: 64 consecutive MN elements
// (128 bytes) per K row, K rows 128 bytes apart, 8-row groups 1024 bytes apart
// (SBO), the next 64 MN elements `mn_stride` bytes further (LBO) -- the TMA
// SWIZZLE_128B image of [K rows, 64 elements] boxes placed mn_stride apart.
__device__ __forceinline__ uint64_t sdesc_mnmajor_sw128(uint32_t saddr, uint32_t mn_stride) {
    uint64_t d = 0;
    d |= static_cast<uint64_t>((saddr >> 4) & 0x3FFFu);
    d |= static_cast<uint64_t>((mn_stride >> 4) & 0x3FFFu) << 16;   // LBO
    d |= static_cast<uint64_t>(1024u >> 4) << 32;                   // SBO: 8 rows x 128 B
    d |= static_cast<uint64_t>(1u) << 46;
    d |= static_cast<uint64_t>(2u) << 61;                           // SWIZZLE_128B
    return d;
}

// Source of a 32x128b scale-factor copy: 32 rows of 16 bytes, contiguous.
__device__ __forceinline__ uint64_t sdesc_sf_tile(uint32_t saddr) {
    uint64_t d = 0;
    d |= static_cast<uint64_t>((saddr >> 4) & 0x3FFFu);
    d |= static_cast<uint64_t>(128u >> 4) << 32;     // SBO: 8 rows x 16 B
    d |= static_cast<uint64_t>(1u) << 46;
    return d;
}

// Instruction descriptor of kind::mxf4nvf4 (E2M1 x E2M1, UE4M3 scales, FP32
// accumulate, both operands K-major, dense): a/b format 1 at bits [7,10) and
// [10,13), N >> 3 at [17,23), scale format 0 (UE4M3) at bit 23, M >> 4 at
// [24,29), scale-factor ids 0.
__host__ __device__ constexpr uint32_t idesc_nvf4(uint32_t M, uint32_t N) {
    return (1u << 7) | (1u << 10) | ((N >> 3) << 17) | ((M >> 4) << 24);
}

}  // namespace mq
