// ptx.cuh -- thin inline-PTX wrappers for sm_100a: mbarriers with bounded
// waits, TMA / bulk copies, and the tcgen05 family (TMEM allocation, the
// block-scaled FP4 MMA, shared->TMEM scale copies, TMEM loads).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace nvfp4 {

// Device status word values (written by kernels whose bounded waits give up).
enum : int { kDevOk = 0, kDevTimeout = 1 };

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// ----------------------------------------------------------------------------
// mbarrier
// ----------------------------------------------------------------------------
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}

__device__ __forceinline__ void fence_mbar_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
                 "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

// Suspend-time hint for try_wait, in ns: a waiting thread sleeps in hardware
// until the phase completes (it is woken then) or this much time has passed,
// instead of spinning and loading the shared-memory pipe the working warps need.
constexpr uint32_t kWaitHintNs = 20000;

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
    uint32_t done;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(done)
        : "r"(smem_u32(bar)), "r"(parity), "r"(kWaitHintNs)
        : "memory");
    return done != 0;
}

// SM cycle counter: cheap to read (unlike %globaltimer, whose reads are slow
// and which advances in coarse steps), so polling loops can consult it on
// every iteration without adding latency to the handshake they wait for.
__device__ __forceinline__ uint64_t clock_cycles() {
    uint64_t c;
    asm volatile("mov.u64 %0, %%clock64;" : "=l"(c));
    return c;
}

// A wait limit given in nanoseconds as SM cycles: 2 cycles per ns, so the
// bound is the requested time at 2 GHz and proportionally longer at lower
// clocks -- always finite.
__device__ __forceinline__ uint64_t limit_cycles(uint64_t limit_ns) { return limit_ns * 2; }

// Wait until the phase with the given parity has completed, or give up after
// `limit_ns` (see limit_cycles) or when *abort becomes non-zero.  On a
// timeout the device status word is set and *abort raised so that every role
// of the CTA stops.  Returns true when the phase completed.
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t* bar, uint32_t parity,
                                                  uint64_t limit_ns, volatile int* abort,
                                                  int* dev_status) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = clock_cycles();
    const uint64_t lim = limit_cycles(limit_ns);
    while (true) {
        if (mbar_try_wait(bar, parity)) return true;
        if (*abort) return false;
        if (clock_cycles() - t0 > lim) {
            *abort = 1;
            atomicExch(dev_status, kDevTimeout);
            return false;
        }
    }
}

// Wait variant for barriers that other CTAs of the cluster arrive on (with
// release.cluster) after writing into this CTA's shared memory: the acquire
// is at cluster scope so those writes are visible once the phase completes.
__device__ __forceinline__ bool mbar_try_wait_cluster(uint64_t* bar, uint32_t parity) {
    uint32_t done;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2, %3;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(done)
        : "r"(smem_u32(bar)), "r"(parity), "r"(kWaitHintNs)
        : "memory");
    return done != 0;
}

__device__ __forceinline__ bool mbar_wait_cluster_bounded(uint64_t* bar, uint32_t parity,
                                                          uint64_t limit_ns, volatile int* abort,
                                                          int* dev_status) {
    if (mbar_try_wait_cluster(bar, parity)) return true;
    const uint64_t t0 = clock_cycles();
    const uint64_t lim = limit_cycles(limit_ns);
    while (true) {
        if (mbar_try_wait_cluster(bar, parity)) return true;
        if (*abort) return false;
        if (clock_cycles() - t0 > lim) {
            *abort = 1;
            atomicExch(dev_status, kDevTimeout);
            return false;
        }
    }
}

// True in exactly one active lane of the warp.  Issue code of the form
// "the whole warp computes, one elected lane issues" keeps descriptors and
// addresses warp-uniform, so tensor-core and TMA instructions take them from
// uniform registers without per-instruction moves.
__device__ __forceinline__ bool elect_one() {
    uint32_t pred = 0;
    asm volatile(
        "{\n\t.reg .pred P;\n\t"
        "elect.sync _|P, 0xffffffff;\n\t"
        "selp.u32 %0, 1, 0, P;\n\t}"
        : "=r"(pred));
    return pred != 0;
}

// Non-blocking test of a phase: never suspends the thread.
__device__ __forceinline__ bool mbar_test_wait(uint64_t* bar, uint32_t parity) {
    uint32_t done;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(done)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return done != 0;
}

// try_wait without a suspend-time hint (the system's own short limit).
__device__ __forceinline__ bool mbar_try_wait_nohint(uint64_t* bar, uint32_t parity) {
    uint32_t done;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(done)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return done != 0;
}

#ifndef NVFP4_PIPE_WAIT
#define NVFP4_PIPE_WAIT 0
#endif

// Bounded wait for the GEMM feed loop (TMA producer <-> MMA issuer), where the
// wake-up latency of every hop adds to the time a stage stays out of use.
__device__ __forceinline__ bool mbar_wait_pipe(uint64_t* bar, uint32_t parity, uint64_t limit_ns,
                                               volatile int* abort, int* dev_status) {
#if NVFP4_PIPE_WAIT == 0
    return mbar_wait_bounded(bar, parity, limit_ns, abort, dev_status);
#else
    const uint64_t t0 = clock_cycles();
    const uint64_t lim = limit_cycles(limit_ns);
    while (true) {
#if NVFP4_PIPE_WAIT == 1
        if (mbar_try_wait_nohint(bar, parity)) return true;
#else
        if (mbar_test_wait(bar, parity)) return true;
#endif
        if (*abort) return false;
        if (clock_cycles() - t0 > lim) {
            *abort = 1;
            atomicExch(dev_status, kDevTimeout);
            return false;
        }
    }
#endif
}

__device__ __forceinline__ bool mbar_wait_warp_pipe(uint64_t* bar, uint32_t parity,
                                                    uint64_t limit_ns, volatile int* abort,
                                                    int* dev_status) {
    int ok = 1;
    if ((threadIdx.x & 31) == 0) ok = mbar_wait_pipe(bar, parity, limit_ns, abort, dev_status);
    return __shfl_sync(0xFFFFFFFFu, ok, 0) != 0;
}

// Whole-warp bounded wait that never suspends: every lane tests the phase
// (one broadcast read) until it completes.  For the feed loop of the
// few-token GEMM, where each stage crosses two handshakes and the wake-up
// latency of a suspended try_wait would add to every one of them.  Same
// limits as mbar_wait_bounded; all 32 lanes must call it.
__device__ __forceinline__ bool mbar_spin_warp(uint64_t* bar, uint32_t parity, uint64_t limit_ns,
                                               volatile int* abort, int* dev_status) {
    if (__shfl_sync(0xFFFFFFFFu, mbar_test_wait(bar, parity) ? 1 : 0, 0)) return true;
    const uint64_t t0 = clock_cycles();
    const uint64_t lim = limit_cycles(limit_ns);
    while (true) {
        if (__shfl_sync(0xFFFFFFFFu, mbar_test_wait(bar, parity) ? 1 : 0, 0)) return true;
        int stop = 0;
        if ((threadIdx.x & 31) == 0) {
            if (*abort) {
                stop = 1;
            } else if (clock_cycles() - t0 > lim) {
                *abort = 1;
                atomicExch(dev_status, kDevTimeout);
                stop = 1;
            }
        }
        if (__shfl_sync(0xFFFFFFFFu, stop, 0)) return false;
    }
}

// Bounded wait by the whole warp: lane 0 polls, the outcome is broadcast.
__device__ __forceinline__ bool mbar_wait_warp(uint64_t* bar, uint32_t parity, uint64_t limit_ns,
                                               volatile int* abort, int* dev_status) {
    int ok = 1;
    if ((threadIdx.x & 31) == 0) ok = mbar_wait_bounded(bar, parity, limit_ns, abort, dev_status);
    return __shfl_sync(0xFFFFFFFFu, ok, 0) != 0;
}

// ----------------------------------------------------------------------------
// TMA and bulk copies (global -> shared), completion counted in bytes on an
// mbarrier.  No multicast anywhere: each CTA loads its own tiles.
// ----------------------------------------------------------------------------
__device__ __forceinline__ void prefetch_tmap(const CUtensorMap* m) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(m) : "memory");
}

__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, uint64_t* bar,
                                            int32_t x, int32_t y, uint64_t policy) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        ".L2::cache_hint [%0], [%1, {%3, %4}], [%2], %5;" ::"r"(smem_u32(dst)),
        "l"(map), "r"(smem_u32(bar)), "r"(x), "r"(y), "l"(policy)
        : "memory");
}

__device__ __forceinline__ void bulk_load(void* dst, const void* src, uint32_t bytes,
                                          uint64_t* bar, uint64_t policy) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
        " [%0], [%1], %2, [%3], %4;" ::"r"(smem_u32(dst)),
        "l"(src), "r"(bytes), "r"(smem_u32(bar)), "l"(policy)
        : "memory");
}

__device__ __forceinline__ uint64_t l2_policy_evict_last() {
    uint64_t p;
    asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(p));
    return p;
}

__device__ __forceinline__ uint64_t l2_policy_evict_first() {
    uint64_t p;
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
    return p;
}

// 16-byte global store that bypasses L1 and carries an L2 eviction policy.
__device__ __forceinline__ void st_global_v4_hint(void* p, uint32_t a, uint32_t b, uint32_t c,
                                                  uint32_t d, uint64_t policy) {
    asm volatile("st.global.L1::no_allocate.L2::cache_hint.v4.b32 [%0], {%1, %2, %3, %4}, %5;" ::"l"(p),
                 "r"(a), "r"(b), "r"(c), "r"(d), "l"(policy)
                 : "memory");
}

// TMA store of a 2-D box from this CTA's shared memory, completion tracked
// by bulk groups of the issuing thread.
__device__ __forceinline__ void tma_store_2d(const CUtensorMap* map, const void* src, int32_t x,
                                             int32_t y, uint64_t policy) {
    asm volatile(
        "cp.async.bulk.tensor.2d.global.shared::cta.bulk_group.L2::cache_hint"
        " [%0, {%2, %3}], [%1], %4;" ::"l"(map),
        "r"(smem_u32(src)), "r"(x), "r"(y), "l"(policy)
        : "memory");
}

__device__ __forceinline__ void bulk_commit_group() {
    asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}

// Wait until every bulk group of this thread has finished reading its
// shared-memory source (the buffer may be rewritten).
__device__ __forceinline__ void bulk_wait_read_all() {
    asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
}

// Wait until every bulk group of this thread has completed (writes done).
__device__ __forceinline__ void bulk_wait_all() {
    asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
}

// Make this thread's generic-proxy shared-memory writes visible to the async
// proxy (TMA) before a bulk copy reads them.
__device__ __forceinline__ void fence_proxy_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// 16-byte shared-memory store.
__device__ __forceinline__ void sts128(uint32_t saddr, uint32_t a, uint32_t b, uint32_t c,
                                       uint32_t d) {
    asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(saddr), "r"(a), "r"(b), "r"(c),
                 "r"(d)
                 : "memory");
}

// ----------------------------------------------------------------------------
// tcgen05: tensor memory, MMA, copies, loads (single-CTA group)
// ----------------------------------------------------------------------------
__device__ __forceinline__ void tmem_alloc(uint32_t* dst_smem, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(dst_smem)),
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

// Arrive once on `bar` when every tcgen05 operation this thread issued so far
// (MMAs and shared->TMEM copies) has completed.
__device__ __forceinline__ void tc_commit(uint64_t* bar) {
    asm volatile(
        "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
            smem_u32(bar))
        : "memory");
}

// Copy one 512-byte scale atom (32 rows x 16 bytes in shared memory) into 4
// TMEM columns, replicated to the four 32-lane quarters of TMEM.
__device__ __forceinline__ void tc_copy_scales(uint32_t taddr, uint64_t sdesc) {
    asm volatile("tcgen05.cp.cta_group::1.32x128b.warpx4 [%0], %1;" ::"r"(taddr), "l"(sdesc)
                 : "memory");
}

// D[tmem] (+)= A[smem] * B[smem]^T with E2M1 operands and UE4M3 scales per 16
// elements (K = 64 per instruction).
__device__ __forceinline__ void tc_mma_nvf4(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                            uint32_t idesc, uint32_t sfa_tmem,
                                            uint32_t sfb_tmem, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::mxf4nvf4.block_scale.block16 [%0], %1, %2, %3, [%5], "
        "[%6], p;\n\t}" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(sfa_tmem), "r"(sfb_tmem)
        : "memory");
}

// Each thread of the warp reads 32 consecutive 32-bit columns of its own TMEM
// lane (the warp's 32-lane quarter).
__device__ __forceinline__ void tmem_ld_32cols(uint32_t taddr, uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
        "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
        "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, "
        "[%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
          "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]),
          "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
          "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]),
          "=r"(r[31])
        : "r"(taddr));
}

__device__ __forceinline__ void tmem_ld_wait() {
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// ----------------------------------------------------------------------------
// Shared-memory matrix descriptors (tcgen05 format, version 1)
// ----------------------------------------------------------------------------
// K-major operand tile, rows of exactly 128 bytes (256 packed FP4 values),
// 128-byte swizzle, 8-row groups 1024 bytes apart.  The tile base must be
// 1024-byte aligned; stepping K by 64 values inside the row adds 32 bytes to
// the start address.
__device__ __forceinline__ uint64_t sdesc_kmajor_sw128(uint32_t saddr) {
    uint64_t d = 0;
    d |= static_cast<uint64_t>((saddr >> 4) & 0x3FFF);      // start address
    d |= static_cast<uint64_t>(1024 >> 4) << 32;             // stride between 8-row groups
    d |= static_cast<uint64_t>(1) << 46;                     // descriptor version
    d |= static_cast<uint64_t>(2) << 61;                     // 128-byte swizzle
    return d;
}

// K-major operand tile, rows of exactly 64 bytes (128 packed FP4 values),
// 64-byte swizzle, 8-row groups 512 bytes apart; the base must be 512-byte
// aligned and K steps of 64 values add 32 bytes to the start address.
__device__ __forceinline__ uint64_t sdesc_kmajor_sw64(uint32_t saddr) {
    uint64_t d = 0;
    d |= static_cast<uint64_t>((saddr >> 4) & 0x3FFF);      // start address
    d |= static_cast<uint64_t>(512 >> 4) << 32;              // stride between 8-row groups
    d |= static_cast<uint64_t>(1) << 46;                     // descriptor version
    d |= static_cast<uint64_t>(4) << 61;                     // 64-byte swizzle
    return d;
}

// Source of a 32x128b scale copy: 32 rows of 16 bytes, contiguous, no swizzle
// (8-row core matrices 128 bytes apart).
__device__ __forceinline__ uint64_t sdesc_scales(uint32_t saddr) {
    uint64_t d = 0;
    d |= static_cast<uint64_t>((saddr >> 4) & 0x3FFF);
    d |= static_cast<uint64_t>(128 >> 4) << 32;
    d |= static_cast<uint64_t>(1) << 46;
    return d;
}

// ----------------------------------------------------------------------------
// CTA pairs (cluster of two): the even CTA issues the pair's MMAs
// ----------------------------------------------------------------------------
__device__ __forceinline__ uint32_t cluster_ctarank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}

// Shared-memory address of the same variable in CTA `rank` of the cluster.
__device__ __forceinline__ uint32_t mapa_shared(uint32_t saddr, uint32_t rank) {
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(saddr), "r"(rank));
    return r;
}

// Arrive on an mbarrier that may live in another CTA of the cluster.
__device__ __forceinline__ void mbar_arrive_cluster(uint32_t cluster_saddr) {
    asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_saddr)
                 : "memory");
}

// Arrive with relaxed ordering: for signals that only say "I have finished
// reading" where every value read was already consumed by this thread before
// the arrive issues.  Unlike the release form it does not wait for this
// thread's earlier global stores to complete.
__device__ __forceinline__ void mbar_arrive_cluster_relaxed(uint32_t cluster_saddr) {
    asm volatile("mbarrier.arrive.relaxed.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_saddr)
                 : "memory");
}

// The two halves of cluster_sync, for roles that can start before their
// peers: arrive (release: this thread's earlier writes, barrier set-up
// included, become visible to the cluster) and, later, wait (acquire).
__device__ __forceinline__ void cluster_arrive() {
    asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory");
}

__device__ __forceinline__ void cluster_wait() {
    asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// Arrive on named barrier `id` without waiting; the calling thread's earlier
// writes are visible to the threads that wait on the barrier.
__device__ __forceinline__ void named_barrier_arrive(int id, int count) {
    asm volatile("bar.arrive %0, %1;" ::"r"(id), "r"(count) : "memory");
}

// Programmatic dependent launch.  launch_dependents lets the next grid on the
// stream (when it was launched as a programmatic dependent) be scheduled now,
// so its CTAs start on SMs as this grid's CTAs leave them; dependency_wait
// returns once the previous grid has completed and its memory writes are
// visible (at once when this grid was launched the ordinary way).
__device__ __forceinline__ void grid_launch_dependents() {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}
__device__ __forceinline__ void grid_dependency_wait() {
    asm volatile("griddepcontrol.wait;" ::: "memory");
}

// Barrier among `count` threads of the CTA on named barrier `id` (1..15).
__device__ __forceinline__ void named_barrier_sync(int id, int count) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(count) : "memory");
}

__device__ __forceinline__ void cluster_sync() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::
                     : "memory");
}

// 2-D tiled TMA load for a CTA pair: the bytes are counted on the mbarrier
// at `bar_cluster` (a shared::cluster address, normally the even CTA's).
__device__ __forceinline__ void tma_load_2d_pair(void* dst, const CUtensorMap* map,
                                                 uint32_t bar_cluster, int32_t x, int32_t y,
                                                 uint64_t policy) {
    asm volatile(
        "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        ".L2::cache_hint [%0], [%1, {%3, %4}], [%2], %5;" ::"r"(smem_u32(dst)),
        "l"(map), "r"(bar_cluster), "r"(x), "r"(y), "l"(policy)
        : "memory");
}

__device__ __forceinline__ void tmem_alloc_pair(uint32_t* dst_smem, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(dst_smem)),
                 "r"(ncols)
                 : "memory");
}

__device__ __forceinline__ void tmem_relinquish_pair() {
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_dealloc_pair(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
                 : "memory");
}

// Arrive once on the mbarrier at the same shared offset in every CTA of
// `cta_mask` when the pair's tcgen05 operations issued so far have completed.
__device__ __forceinline__ void tc_commit_pair(uint64_t* bar, uint16_t cta_mask) {
    asm volatile(
        "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64"
        " [%0], %1;" ::"r"(smem_u32(bar)),
        "h"(cta_mask)
        : "memory");
}

// Scale atom copy for the pair: each CTA's shared memory at this offset into
// its own tensor memory.
__device__ __forceinline__ void tc_copy_scales_pair(uint32_t taddr, uint64_t sdesc) {
    asm volatile("tcgen05.cp.cta_group::2.32x128b.warpx4 [%0], %1;" ::"r"(taddr), "l"(sdesc)
                 : "memory");
}

// Pair MMA: M = 256 (128 rows of A from each CTA), B split along N between
// the two CTAs, accumulators in each CTA's tensor memory.
__device__ __forceinline__ void tc_mma_nvf4_pair(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                                 uint32_t idesc, uint32_t sfa_tmem,
                                                 uint32_t sfb_tmem, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::2.kind::mxf4nvf4.block_scale.block16 [%0], %1, %2, %3, [%5], "
        "[%6], p;\n\t}" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(sfa_tmem), "r"(sfb_tmem)
        : "memory");
}

// Each thread of the warp writes 16 / 32 consecutive 32-bit columns of its own
// TMEM lane (the warp's 32-lane quarter).
__device__ __forceinline__ void tmem_st_16cols(uint32_t taddr, const uint32_t (&r)[16]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
        "{%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16};" ::"r"(taddr),
        "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
        "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
        : "memory");
}

__device__ __forceinline__ void tmem_st_wait() {
    asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

// 16-byte shared-memory load.
__device__ __forceinline__ uint4 lds128(uint32_t saddr) {
    uint4 v;
    asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "r"(saddr));
    return v;
}

// 32-bit store into the shared memory of a CTA of the cluster (a
// shared::cluster address from mapa_shared).
__device__ __forceinline__ void st_shared_cluster_f32(uint32_t cluster_saddr, float v) {
    asm volatile("st.shared::cluster.f32 [%0], %1;" ::"r"(cluster_saddr), "f"(v) : "memory");
}

// Each thread of the warp reads 16 consecutive 32-bit columns of its own TMEM
// lane (the warp's 32-lane quarter).
__device__ __forceinline__ void tmem_ld_16cols(uint32_t taddr, uint32_t (&r)[16]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
        "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
          "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr));
}

}  // namespace nvfp4
