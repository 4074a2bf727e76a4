// Device helpers shared by the kernels: status word, bounded waits, and thin
// inline-PTX wrappers for mbarrier, TMA, tcgen05 (UMMA + TMEM) and clusters
// on sm_100a.
#pragma once
#include <climits>
#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

#include "lb.h"

namespace lb {

// Per-device status word (LB_DEV_* bits).  Kernels never trap: they skip the
// offending element and OR a bit in here.
__device__ int g_status;

__device__ __forceinline__ void flag(int bits) { atomicOr(&g_status, bits); }

// Phase timestamps of block 0 for latency analysis builds (-DLB_TIMING);
// compiled out otherwise.
#ifdef LB_TIMING
// [0, 64): phase stamps of block 0; [64, 64 + 1024): start and end
// (globaltimer, ns) of CTAs 0..511 of the kernels that record them
__device__ long long g_ticks[64 + 1024];
// (the clock read carries a memory clobber, so it stays between the memory
// operations and barriers around it)
__device__ __forceinline__ long long lb_clock() {
    long long t;
    asm volatile("mov.u64 %0, %%clock64;" : "=l"(t)::"memory");
    return t;
}
#define LB_TICK(slot)                                                                          \
    do {                                                                                       \
        if (threadIdx.x == 0 && blockIdx.x == 0 && blockIdx.y == 0) lb::g_ticks[slot] = lb::lb_clock(); \
    } while (0)
#define LB_CTA_TIME(which)                                                                     \
    do {                                                                                       \
        const unsigned cta_ = blockIdx.x + blockIdx.y * gridDim.x;                             \
        if (cta_ < 512u) {                                                                     \
            long long t_;                                                                      \
            asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t_)::"memory");                   \
            lb::g_ticks[64 + 2 * cta_ + (which)] = t_;                                         \
        }                                                                                      \
    } while (0)
// stamp by whichever thread of block 0 calls it (the caller picks the thread)
#define LB_TICK_ANY(slot)                                                      \
    do {                                                                       \
        if (blockIdx.x == 0 && blockIdx.y == 0) lb::g_ticks[slot] = lb::lb_clock(); \
    } while (0)
#else
#define LB_TICK(slot) \
    do {              \
    } while (0)
#define LB_TICK_ANY(slot) \
    do {                  \
    } while (0)
#define LB_CTA_TIME(which) \
    do {                   \
    } while (0)
#endif

// About one second at the B200's top SM clock: longer than any legitimate
// wait inside one launch, short enough to keep a broken launch from hanging.
constexpr long long kWaitCycles = 2000000000LL;

constexpr unsigned kFull = 0xffffffffu;

// Programmatic dependent launch.  Every kernel of the library calls
// pdl_begin(), which waits until the previous kernel on the stream has
// completed and its memory operations are visible (a no-op for a kernel
// launched without programmatic stream serialization), before it touches
// global memory, so a kernel never reads an input, or overwrites a buffer,
// that its predecessor is still using.  The one exception is the assign's
// scatter: its predecessor signals its dependents once past its own wait,
// and the scatter reads, before its wait, only inputs that were final before
// that predecessor started (through L2; assign.cuh names them).  No other
// kernel signals early (measured: an early signal let the next kernels'
// blocks sit waiting on the SMs and made the step slower); the gain there is
// the launch processing of the next kernel, which overlaps the previous
// one's exit.
__device__ __forceinline__ void pdl_begin() {
    asm volatile("griddepcontrol.wait;" ::: "memory");
}

__device__ __forceinline__ uint32_t smem_u32(const void *p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// ---------------------------------------------------------------- mbarrier
__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}

__device__ __forceinline__ void fence_mbar_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t addr, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(addr), "r"(parity)
        : "memory");
    return ok != 0;
}

// Wait for the phase with the given parity to complete; false after about a
// second (the caller then records LB_DEV_TIMEOUT and unwinds).
__device__ __forceinline__ bool mbar_wait(uint64_t *bar, uint32_t parity) {
    const uint32_t addr = smem_u32(bar);
    if (mbar_try_wait(addr, parity)) return true;
    const long long t0 = clock64();
    while (!mbar_try_wait(addr, parity)) {
        if (clock64() - t0 > kWaitCycles) return false;
    }
    return true;
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t *bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
                 "r"(bytes)
                 : "memory");
}

// ---------------------------------------------------------------- TMA
__device__ __forceinline__ void tma_prefetch_desc(const CUtensorMap *map) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// 3-D tiled load into this CTA's shared memory, completing on `bar`.
__device__ __forceinline__ void tma_load_3d(const CUtensorMap *map, void *dst, uint64_t *bar,
                                            int c0, int c1, int c2) {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4, %5}], [%2];" ::"r"(smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(c0), "r"(c1), "r"(c2)
        : "memory");
}

// Same load with an L2 eviction-priority hint (a policy from l2_policy_*).
__device__ __forceinline__ void tma_load_3d_hint(const CUtensorMap *map, void *dst, uint64_t *bar, int c0, int c1,
                                                 int c2, uint64_t policy) {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes.L2::cache_hint"
        " [%0], [%1, {%3, %4, %5}], [%2], %6;" ::"r"(smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(c0), "r"(c1), "r"(c2), "l"(policy)
        : "memory");
}
__device__ __forceinline__ uint64_t l2_policy_evict_first() {
    uint64_t p;
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
    return p;
}
__device__ __forceinline__ uint64_t l2_policy_evict_last() {
    uint64_t p;
    asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(p));
    return p;
}

__device__ __forceinline__ void mbar_arrive(uint64_t *bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

// ---------------------------------------------------------------- tcgen05
__device__ __forceinline__ void tmem_alloc(uint32_t *slot, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(slot)),
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

// D[tmem] (+)= A[smem] * B[smem]^T, bf16 inputs, fp32 accumulator in TMEM.
__device__ __forceinline__ void umma_bf16(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                          uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// Arrive on `bar` once every tcgen05.mma issued so far by this thread is done.
__device__ __forceinline__ void umma_commit(uint64_t *bar) {
    asm volatile(
        "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
            smem_u32(bar))
        : "memory");
}

// Warp-collective: 32 TMEM lanes x 16 consecutive 32-bit columns; thread i of
// the warp receives lane (base lane + i).
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&r)[16]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
          "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr)
        : "memory");
}
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
        "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
          "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
          "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr)
        : "memory");
}
__device__ __forceinline__ void tmem_wait_ld() {
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// Shared-memory matrix descriptor: K-major operand staged by TMA with the
// 128-byte swizzle (8 rows x 128 B atoms, 1024 B apart).
__device__ __forceinline__ uint64_t sw128_kmajor_desc(uint32_t saddr) {
    return static_cast<uint64_t>((saddr & 0x3FFFFu) >> 4)     // start address
           | (static_cast<uint64_t>(1) << 16)                  // leading byte offset (unused)
           | (static_cast<uint64_t>(1024 >> 4) << 32)          // stride byte offset
           | (static_cast<uint64_t>(1) << 46)                  // descriptor version
           | (static_cast<uint64_t>(2) << 61);                 // 128-byte swizzle
}

// Instruction descriptor: bf16 x bf16 -> fp32, both operands K-major.
__host__ __device__ constexpr uint32_t umma_idesc_bf16(int M, int N) {
    return (1u << 4)                                  // D format fp32
           | (1u << 7)                                // A format bf16
           | (1u << 10)                               // B format bf16
           | (static_cast<uint32_t>(N >> 3) << 17)    // N / 8
           | (static_cast<uint32_t>(M >> 4) << 24);   // M / 16
}

// ---------------------------------------------------------------- CTA pairs (cta_group::2)
// Two CTAs of a cluster (ranks 0 and 1) share one MMA of M = 256: rank 0
// issues it, each CTA holds its 128 rows of A and half of B's N rows in its
// own shared memory at the same offsets, and each CTA's TMEM receives its
// 128 rows of the accumulator.  These forms are used by the paired gate
// kernel only; a kernel uses one cta_group for all its tcgen05 operations.

// 3-D tiled load into this CTA's shared memory whose completion is counted
// on an mbarrier that may be the pair leader's (a shared::cluster address).
// No multicast: every CTA loads its own boxes.
__device__ __forceinline__ void tma_load_3d_pair(const CUtensorMap *map, void *dst, uint32_t bar_cluster, int c0,
                                                 int c1, int c2, uint64_t policy) {
    asm volatile(
        "cp.async.bulk.tensor.3d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
        " [%0], [%1, {%3, %4, %5}], [%2], %6;" ::"r"(smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(bar_cluster), "r"(c0), "r"(c1), "r"(c2), "l"(policy)
        : "memory");
}
__device__ __forceinline__ void tmem_alloc_pair(uint32_t *slot, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(slot)),
                 "r"(ncols)
                 : "memory");
}
__device__ __forceinline__ void tmem_relinquish_pair() {
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc_pair(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
// D[tmem of both CTAs] (+)= A[256 rows, 128 per CTA] * B[N rows, N/2 per CTA]^T.
__device__ __forceinline__ void umma_bf16_pair(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                               uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}
// Arrive on the mbarrier at `bar`'s offset in every CTA of `cta_mask` once
// every tcgen05.mma this thread issued so far is done.
__device__ __forceinline__ void umma_commit_pair(uint64_t *bar, uint16_t cta_mask) {
    asm volatile(
        "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;" ::"r"(
            smem_u32(bar)),
        "h"(cta_mask)
        : "memory");
}
// Arrive on an mbarrier of another CTA of the cluster (shared::cluster address).
__device__ __forceinline__ void mbar_arrive_cluster(uint32_t bar_cluster) {
    asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(bar_cluster) : "memory");
}

// ---------------------------------------------------------------- clusters
__device__ __forceinline__ uint32_t cluster_ctarank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}
__device__ __forceinline__ void cluster_sync() {
    asm volatile(
        "barrier.cluster.arrive.release.aligned;\n\t"
        "barrier.cluster.wait.acquire.aligned;" ::
            : "memory");
}
__device__ __forceinline__ uint32_t mapa_shared(uint32_t saddr, uint32_t rank) {
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(saddr), "r"(rank));
    return r;
}
__device__ __forceinline__ int ld_cluster_i32(uint32_t addr) {
    int v;
    asm volatile("ld.shared::cluster.s32 %0, [%1];" : "=r"(v) : "r"(addr) : "memory");
    return v;
}
// Bulk copy of `bytes` (a multiple of 16, both addresses 16-byte aligned)
// from this CTA's shared memory into another CTA's of the cluster (dst and
// bar are cluster addresses from mapa); completes on the receiver's mbarrier.
__device__ __forceinline__ void bulk_copy_to_cta(uint32_t dst, uint32_t src, uint32_t bytes, uint32_t bar) {
    asm volatile("cp.async.bulk.shared::cluster.shared::cta.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
                 "r"(src), "r"(bytes), "r"(bar)
                 : "memory");
}
// Order this thread's shared-memory writes before later async-proxy reads
// of them (a bulk copy issued after a barrier).
__device__ __forceinline__ void fence_proxy_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
__device__ __forceinline__ float4 ld_cluster_f4(uint32_t addr) {
    float4 v;
    asm volatile("ld.shared::cluster.v4.f32 {%0,%1,%2,%3}, [%4];"
                 : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
                 : "r"(addr)
                 : "memory");
    return v;
}

// ---------------------------------------------------------------- staging
// Copy n int32 from global to shared memory with the whole CTA: 16-byte
// loads when both sides are 16-byte aligned, four loads in flight per thread.
// Plain (coherent) loads: the source may have been written earlier in the
// same kernel by this CTA.
__device__ __forceinline__ void stage_i32(int32_t *dst, const int32_t *src, int n) {
    const int t = threadIdx.x, nt = blockDim.x;
    if (((reinterpret_cast<uintptr_t>(dst) | reinterpret_cast<uintptr_t>(src)) & 15) == 0) {
        const int n4 = n >> 2;
        const int4 *s4 = reinterpret_cast<const int4 *>(src);
        int4 *d4 = reinterpret_cast<int4 *>(dst);
        int i = t;
        for (; i + 3 * nt < n4; i += 4 * nt) {
            const int4 a = s4[i], b = s4[i + nt], c = s4[i + 2 * nt],
                       d = s4[i + 3 * nt];
            d4[i] = a;
            d4[i + nt] = b;
            d4[i + 2 * nt] = c;
            d4[i + 3 * nt] = d;
        }
        for (; i < n4; i += nt) d4[i] = s4[i];
        for (int j = (n4 << 2) + t; j < n; j += nt) dst[j] = src[j];
    } else {
        int i = t;
        for (; i + 3 * nt < n; i += 4 * nt) {
            const int a = src[i], b = src[i + nt], c = src[i + 2 * nt],
                      d = src[i + 3 * nt];
            dst[i] = a;
            dst[i + nt] = b;
            dst[i + 2 * nt] = c;
            dst[i + 3 * nt] = d;
        }
        for (; i < n; i += nt) dst[i] = src[i];
    }
}

// ---------------------------------------------------------------- warp helpers
__device__ __forceinline__ unsigned lanemask_lt() {
    unsigned m;
    asm("mov.u32 %0, %%lanemask_lt;" : "=r"(m));
    return m;
}

}  // namespace lb
