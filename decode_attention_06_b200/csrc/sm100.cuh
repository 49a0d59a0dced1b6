// sm100.cuh -- thin inline-PTX wrappers for the Blackwell (sm_100a) features
// the decode kernels use: mbarriers with bounded waits, TMA tiled loads,
// tcgen05 tensor-memory allocation, MMA, commit, loads and stores, and the
// shared-memory matrix / instruction descriptors of tcgen05.mma.
#pragma once

#include <cuda.h>
#include <cuda_fp16.h>
#include <stdint.h>

namespace gqla {
namespace sm100 {

__device__ __forceinline__ uint32_t smem_u32(const void *p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// ------------------------------------------------------------------ mbarrier

__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}

__device__ __forceinline__ void fence_barrier_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t *bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t *bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
                 "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t *bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}

// Non-blocking probe of the phase with the given parity (never suspends the thread).
__device__ __forceinline__ bool mbar_test_wait(uint64_t *bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}

// About two seconds at B200 clocks: a wait that takes longer is a bug, and
// the kernel gives up instead of hanging the GPU.
constexpr long long kWaitCycles = 4000000000LL;

// Bounded wait for the phase with the given parity.  Returns false when the
// limit ran out or another thread of the CTA has already given up (*abort).
__device__ __forceinline__ bool mbar_wait(uint64_t *bar, uint32_t parity, volatile int *abort) {
    if (mbar_try_wait(bar, parity)) return true;
    const long long t0 = clock64();
    while (true) {
        if (mbar_try_wait(bar, parity)) return true;
        if (*abort) return false;
        if (clock64() - t0 > kWaitCycles) return false;
    }
}

// Wait-site profiling hook: compiled to the plain bounded wait unless the
// translation unit defines GQLA_WAIT_PROFILE (a diagnostic build), in which
// case each thread accumulates the cycles spent per numbered site in
// registers and lane 0 of every warp adds them to a global table at exit.
#ifdef GQLA_WAIT_PROFILE
__device__ unsigned long long g_wait_cycles[32];
__device__ unsigned long long g_wait_count[32];
// per-warp accumulators in shared memory (lane 0 of each warp writes its own
// row; kernels of up to 20 warps)
#define GQLA_PROF_DECL                                                       \
    __shared__ unsigned int gqla_prof_c_[20][24];                           \
    __shared__ unsigned int gqla_prof_n_[20][24];                           \
    if ((threadIdx.x & 31) == 0)                                            \
        for (int i_ = 0; i_ < 24; ++i_)                                     \
            gqla_prof_c_[threadIdx.x >> 5][i_] = 0, gqla_prof_n_[threadIdx.x >> 5][i_] = 0
#define GQLA_PROF_ADD(site, dt)                                              \
    do {                                                                     \
        if ((threadIdx.x & 31) == 0) {                                       \
            gqla_prof_c_[threadIdx.x >> 5][site] += (unsigned int)(dt);      \
            gqla_prof_n_[threadIdx.x >> 5][site] += 1;                       \
        }                                                                    \
    } while (0)
#define GQLA_WAIT(site, bar, parity, abort)                                  \
    ({                                                                       \
        const long long t0_ = clock64();                                     \
        const bool ok_ = ::gqla::sm100::mbar_wait(bar, parity, abort);       \
        GQLA_PROF_ADD(site, clock64() - t0_);                                \
        ok_;                                                                 \
    })
#define GQLA_WAITC(site, bar, parity, abort)                                 \
    ({                                                                       \
        const long long t0_ = clock64();                                     \
        const bool ok_ = ::gqla::sm100::mbar_wait_cluster(bar, parity, abort); \
        GQLA_PROF_ADD(site, clock64() - t0_);                                \
        ok_;                                                                 \
    })
#define GQLA_SPAN_BEGIN(v) const long long v = clock64()
#define GQLA_SPAN_END(site, v) GQLA_PROF_ADD(site, clock64() - v)
#define GQLA_PROF_FLUSH                                                                     \
    do {                                                                                    \
        if ((threadIdx.x & 31) == 0)                                                        \
            for (int i_ = 0; i_ < 24; ++i_)                                                 \
                if (gqla_prof_n_[threadIdx.x >> 5][i_]) {                                   \
                    atomicAdd(&::gqla::sm100::g_wait_cycles[i_],                            \
                              (unsigned long long)gqla_prof_c_[threadIdx.x >> 5][i_]);      \
                    atomicAdd(&::gqla::sm100::g_wait_count[i_],                             \
                              (unsigned long long)gqla_prof_n_[threadIdx.x >> 5][i_]);      \
                }                                                                           \
    } while (0)
#else
#define GQLA_PROF_DECL (void)0
#define GQLA_WAIT(site, bar, parity, abort) ::gqla::sm100::mbar_wait(bar, parity, abort)
#define GQLA_WAITC(site, bar, parity, abort) ::gqla::sm100::mbar_wait_cluster(bar, parity, abort)
#define GQLA_SPAN_BEGIN(v) (void)0
#define GQLA_SPAN_END(site, v) (void)0
#define GQLA_PROF_FLUSH (void)0
#endif

// ------------------------------------------------------------------ dependent launch

// Wait until the grids this one depends on (the previous kernel in the stream,
// when it was launched with programmatic serialization) have completed and
// their writes are visible.  A no-op otherwise.  Every global access of a
// kernel comes after it.
__device__ __forceinline__ void griddep_wait() {
    asm volatile("griddepcontrol.wait;" ::: "memory");
}

// Allow the next kernel in the stream to start its set-up (its own accesses of
// global memory still wait for this grid to complete).
__device__ __forceinline__ void griddep_launch_dependents() {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// ------------------------------------------------------------------ TMA

__device__ __forceinline__ void tma_load_2d(void *dst, const CUtensorMap *map, uint64_t *bar, int x,
                                            int y) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4}], [%2];" ::"r"(smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(x), "r"(y)
        : "memory");
}

// Four rows (y0..y3) of a 2D tensor, `x` the first column of a one-row box,
// into four consecutive box rows at `dst` (the map's swizzle applies as for a
// four-row box); completes their bytes on `bar`.  Rows outside the tensor
// read as zeros.
__device__ __forceinline__ void tma_gather4_hint(void *dst, const CUtensorMap *map, uint64_t *bar, int x,
                                                 int y0, int y1, int y2, int y3, uint64_t policy) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile::gather4.mbarrier::complete_tx::bytes.L2::cache_hint"
        " [%0], [%1, {%3, %4, %5, %6, %7}], [%2], %8;" ::"r"(smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(x), "r"(y0), "r"(y1), "r"(y2),
        "r"(y3), "l"(policy)
        : "memory");
}

// L2 policy for data read once per launch (a KV cache stream): its lines are the
// first to go, so that what is reused (queries, partials, weights) stays in L2.
__device__ __forceinline__ uint64_t l2_evict_first_policy() {
    uint64_t pol;
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
    return pol;
}

// tma_load_2d with an L2 cache policy (from l2_evict_first_policy and the like).
__device__ __forceinline__ void tma_load_2d_hint(void *dst, const CUtensorMap *map, uint64_t *bar,
                                                 int x, int y, uint64_t policy) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes.L2::cache_hint"
        " [%0], [%1, {%3, %4}], [%2], %5;" ::"r"(smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(x), "r"(y), "l"(policy)
        : "memory");
}

__device__ __forceinline__ void tma_load_3d(void *dst, const CUtensorMap *map, uint64_t *bar, int x,
                                            int y, int z) {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4, %5}], [%2];" ::"r"(smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(x), "r"(y), "r"(z)
        : "memory");
}

// tma_load_3d with an L2 cache policy.
__device__ __forceinline__ void tma_load_3d_hint(void *dst, const CUtensorMap *map, uint64_t *bar, int x,
                                                 int y, int z, uint64_t policy) {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes.L2::cache_hint"
        " [%0], [%1, {%3, %4, %5}], [%2], %6;" ::"r"(smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(x), "r"(y), "r"(z), "l"(policy)
        : "memory");
}

// Tiled TMA store of a box from shared memory, tracked by the bulk async-group
// of the issuing thread.
__device__ __forceinline__ void tma_store_2d(const CUtensorMap *map, const void *src, int x, int y) {
    asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%2, %3}], [%1];" ::"l"(
                     reinterpret_cast<uint64_t>(map)),
                 "r"(smem_u32(src)), "r"(x), "r"(y)
                 : "memory");
}

__device__ __forceinline__ void bulk_commit_group() {
    asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}

// Wait until at most N bulk groups of this thread still read shared memory.
template <int N>
__device__ __forceinline__ void bulk_wait_group_read() {
    asm volatile("cp.async.bulk.wait_group.read %0;" ::"n"(N) : "memory");
}

// Wait until at most N bulk groups of this thread are incomplete.
template <int N>
__device__ __forceinline__ void bulk_wait_group() {
    asm volatile("cp.async.bulk.wait_group %0;" ::"n"(N) : "memory");
}

// Bring the 128-byte line holding `ptr` into L2.
__device__ __forceinline__ void prefetch_l2(const void *ptr) {
    asm volatile("prefetch.global.L2 [%0];" ::"l"(ptr) : "memory");
}

__device__ __forceinline__ void prefetch_tensormap(const CUtensorMap *map) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

__device__ __forceinline__ void fence_proxy_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// ------------------------------------------------------------------ tcgen05

// Warp-collective: allocate `ncols` (power of two >= 32) TMEM columns; the
// base address is written to *dst (shared memory).
__device__ __forceinline__ void tmem_alloc(uint32_t *dst, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(dst)),
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

// D[tmem] (+)= A[smem] * B[smem], kind::f16 (bf16 inputs, fp32 accumulate), issued by one thread.
__device__ __forceinline__ void mma_bf16(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                         uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// Arrive once on `bar` when every tcgen05.mma issued so far by this thread has completed.
__device__ __forceinline__ void mma_commit(uint64_t *bar) {
    asm volatile(
        "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
            smem_u32(bar))
        : "memory");
}

// Commit arriving on the mbarrier at the same shared-memory offset in every CTA
// of `cta_mask` (bit r: cluster rank r).
__device__ __forceinline__ void mma_commit_multicast(uint64_t *bar, uint16_t cta_mask) {
    asm volatile(
        "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64"
        " [%0], %1;" ::"r"(smem_u32(bar)),
        "h"(cta_mask)
        : "memory");
}

__device__ __forceinline__ void tmem_wait_ld() {
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_wait_st() {
    asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

// Warp-collective: thread i reads lane (taddr.lane + i), 16 consecutive 32-bit columns.
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t *r) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
          "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr));
}

__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t *r) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
        "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(taddr),
        "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
        "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]),
        "r"(r[15])
        : "memory");
}

// Warp-collective: thread i reads lane (taddr.lane + i), 32 consecutive 32-bit columns.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t *r) {
    tmem_ld16(taddr, r);
    tmem_ld16(taddr + 16, r + 16);
}

// D[tmem] (+)= A[tmem] * B[smem] (A read from tensor memory, K-major), kind::f16.
__device__ __forceinline__ void mma_bf16_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t bdesc,
                                            uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
        "r"(a_tmem), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// ------------------------------------------------------------------ clusters / DSMEM

__device__ __forceinline__ uint32_t cluster_rank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}

// Shared-memory address of the same variable in CTA `rank` of this cluster.
__device__ __forceinline__ uint32_t map_peer(uint32_t saddr, uint32_t rank) {
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(saddr), "r"(rank));
    return r;
}

__device__ __forceinline__ void st_cluster_v4(uint32_t addr, uint4 v) {
    asm volatile("st.shared::cluster.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(v.x),
                 "r"(v.y), "r"(v.z), "r"(v.w)
                 : "memory");
}

__device__ __forceinline__ void st_cluster_b32(uint32_t addr, uint32_t v) {
    asm volatile("st.shared::cluster.b32 [%0], %1;" ::"r"(addr), "r"(v) : "memory");
}

__device__ __forceinline__ float4 ld_cluster_f4(uint32_t addr) {
    float4 v;
    asm volatile("ld.shared::cluster.v4.f32 {%0, %1, %2, %3}, [%4];"
                 : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
                 : "r"(addr));
    return v;
}

// Arrive on an mbarrier of another CTA of the cluster, releasing this thread's
// earlier shared::cluster stores to whoever acquires the phase.
__device__ __forceinline__ void mbar_arrive_remote(uint32_t cluster_addr) {
    asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr)
                 : "memory");
}

__device__ __forceinline__ bool mbar_try_wait_cluster(uint64_t *bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}

// Non-blocking probe with cluster-scope acquire of the phase with the given parity.
__device__ __forceinline__ bool mbar_test_wait_cluster(uint64_t *bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.test_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}

// Bounded wait with cluster-scope acquire (data written by the peer CTA).
__device__ __forceinline__ bool mbar_wait_cluster(uint64_t *bar, uint32_t parity,
                                                  volatile int *abort) {
    if (mbar_try_wait_cluster(bar, parity)) return true;
    const long long t0 = clock64();
    while (true) {
        if (mbar_try_wait_cluster(bar, parity)) return true;
        if (*abort) return false;
        if (clock64() - t0 > kWaitCycles) return false;
    }
}

// Bulk copy of `bytes` (multiple of 16) from this CTA's shared memory into a
// peer CTA's shared memory; completes `bytes` of transaction count on the
// peer's mbarrier.  Asynchronous: the issuing thread does not wait.
__device__ __forceinline__ void bulk_copy_to_peer(uint32_t dst_cluster, const void *src,
                                                  uint32_t bytes, uint32_t mbar_cluster) {
    asm volatile(
        "cp.async.bulk.shared::cluster.shared::cta.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::
            "r"(dst_cluster),
        "r"(smem_u32(src)), "r"(bytes), "r"(mbar_cluster)
        : "memory");
}

// Asynchronous 16-byte store into a peer CTA's shared memory; completes 16
// bytes of transaction count on the peer's mbarrier `mbar_cluster`.
__device__ __forceinline__ void st_async_v4(uint32_t dst_cluster, uint4 v, uint32_t mbar_cluster) {
    asm volatile(
        "st.async.shared::cluster.mbarrier::complete_tx::bytes.v4.b32 [%0], {%1, %2, %3, %4}, [%5];" ::"r"(
            dst_cluster),
        "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w), "r"(mbar_cluster)
        : "memory");
}

// Asynchronous 8-byte store into a peer CTA's shared memory; completes 8 bytes
// of the transaction count of the peer's mbarrier.
__device__ __forceinline__ void st_async_v2(uint32_t dst_cluster, uint2 v, uint32_t mbar_cluster) {
    asm volatile("st.async.shared::cluster.mbarrier::complete_tx::bytes.v2.b32 [%0], {%1, %2}, [%3];" ::"r"(
                     dst_cluster),
                 "r"(v.x), "r"(v.y), "r"(mbar_cluster)
                 : "memory");
}

// Asynchronous 4-byte store into a peer CTA's shared memory; completes 4 bytes
// of the transaction count of the peer's mbarrier.
__device__ __forceinline__ void st_async_b32(uint32_t dst_cluster, uint32_t v, uint32_t mbar_cluster) {
    asm volatile("st.async.shared::cluster.mbarrier::complete_tx::bytes.b32 [%0], %1, [%2];" ::"r"(
                     dst_cluster),
                 "r"(v), "r"(mbar_cluster)
                 : "memory");
}

// Arrive on a peer CTA's mbarrier without ordering this thread's memory accesses.
__device__ __forceinline__ void mbar_arrive_remote_relaxed(uint32_t cluster_addr) {
    asm volatile("mbarrier.arrive.relaxed.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr)
                 : "memory");
}

// All threads of all CTAs of the cluster (aligned: every thread executes it).
__device__ __forceinline__ void cluster_sync() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::
                     : "memory");
}

// The arrive half of cluster_sync without its release ordering, for a CTA that
// only lets the others go on (it may exit without the matching wait).
__device__ __forceinline__ void cluster_arrive_relaxed() {
    asm volatile("barrier.cluster.arrive.relaxed.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_st8(uint32_t taddr, const uint32_t *r) {
    asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};" ::"r"(taddr),
                 "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7])
                 : "memory");
}

// 2^x with the hardware approximation (a single MUFU.EX2; flushes subnormal
// results to zero, which is harmless for softmax weights that are rounded to
// bf16 afterwards).
__device__ __forceinline__ float fast_exp2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// Two 2^x at once in fp16 (one MUFU.EX2 for both halves).
__device__ __forceinline__ __half2 fast_exp2_h2(__half2 x) {
    uint32_t y;
    asm("ex2.approx.f16x2 %0, %1;" : "=r"(y) : "r"(*reinterpret_cast<uint32_t *>(&x)));
    return *reinterpret_cast<__half2 *>(&y);
}

// ------------------------------------------------------------------ descriptors

enum Swizzle : uint32_t { kSwNone = 0, kSw128 = 2, kSw64 = 4, kSw32 = 6 };

// Shared-memory matrix descriptor of tcgen05.mma: start address, leading and
// stride byte offsets (16-byte units), descriptor version 1, swizzle mode.
__device__ __forceinline__ uint64_t smem_desc(uint32_t saddr, uint32_t lbo, uint32_t sbo,
                                              uint32_t swizzle) {
    uint64_t d = 0;
    d |= static_cast<uint64_t>((saddr >> 4) & 0x3FFFu);
    d |= static_cast<uint64_t>((lbo >> 4) & 0x3FFFu) << 16;
    d |= static_cast<uint64_t>((sbo >> 4) & 0x3FFFu) << 32;
    d |= static_cast<uint64_t>(1u) << 46;
    d |= static_cast<uint64_t>(swizzle & 7u) << 61;
    return d;
}

// The descriptor of the same layout `bytes` further on (the start address field,
// bits 0-13, holds address / 16 and stays below 2^14 for every shared address).
__device__ __forceinline__ uint64_t desc_advance(uint64_t desc, uint32_t bytes) {
    return desc + static_cast<uint64_t>(bytes >> 4);
}

// Instruction descriptor, kind::f16: bf16 x bf16 -> fp32, M x N, operand majors
// (0 = K-major, 1 = MN-major).
__host__ __device__ constexpr uint32_t idesc_bf16(int M, int N, int a_mn, int b_mn) {
    return (1u << 4)                              // D format fp32
           | (1u << 7)                            // A format bf16
           | (1u << 10)                           // B format bf16
           | (static_cast<uint32_t>(a_mn) << 15)  // A major
           | (static_cast<uint32_t>(b_mn) << 16)  // B major
           | (static_cast<uint32_t>(N >> 3) << 17) | (static_cast<uint32_t>(M >> 4) << 24);
}

// Physical byte offset of logical offset `logical` inside a tile stored with
// the 32/64/128-byte swizzle (row_bytes = the swizzle width): the 16-byte
// chunk index bits [4, 4+k) are XORed with address bits [7, 7+k), k =
// log2(row_bytes / 16).  The tile base must be aligned to the swizzle atom.
__device__ __forceinline__ uint32_t swz(uint32_t logical, uint32_t row_bytes) {
    const uint32_t mask = row_bytes / 16 - 1;
    return logical ^ (((logical >> 7) & mask) << 4);
}

}  // namespace sm100
}  // namespace gqla
