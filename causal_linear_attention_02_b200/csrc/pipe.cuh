// Pipeline helpers shared by the persistent tcgen05 kernels: bounded
// mbarrier waits with a launch-wide abort, L2 eviction-priority policies,
// TMA loads with cache hints, TMA tensor stores and bulk-group waits.
#pragma once

#include <cuda.h>
#include <stdint.h>

#include "common.cuh"
#include "sm100.cuh"

namespace la {
namespace sm100 {

// Warp-uniform AND: every decision that guards a .sync.aligned tcgen05
// instruction must be the same in all 32 lanes, even on an abort path.
__device__ __forceinline__ bool warp_all(bool x) { return __all_sync(0xffffffffu, x) != 0; }

__device__ __forceinline__ uint64_t policy_evict_first() {
    uint64_t pol;
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
    return pol;
}
__device__ __forceinline__ uint64_t policy_evict_last() {
    uint64_t pol;
    asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(pol));
    return pol;
}

__device__ __forceinline__ void tma_load_3d_hint(void* dst, const CUtensorMap* map, uint64_t* bar,
                                                 int32_t c0, int32_t c1, int32_t c2, uint64_t pol) {
    asm volatile("cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
                 " [%0], [%1, {%3, %4, %5}], [%2], %6;"
                 :: "r"(smem_u32(dst)), "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)),
                    "r"(c0), "r"(c1), "r"(c2), "l"(pol)
                 : "memory");
}

// Abort state of one launch: a CTA-local flag in shared memory and a
// launch-wide flag in the workspace. The first wait that runs out of time
// raises both (and records LA_ERR_TIMEOUT); every other wait of every CTA
// then gives up at its next check, so the launch ends promptly.
struct Abort {
    volatile int* cta;
    volatile int* global;
    uint64_t limit_ns;
    __device__ __forceinline__ bool raised() const { return *cta || *global; }
    __device__ __forceinline__ void raise() const {
        if (!*cta) { *cta = 1; *global = 1; record_status(LA_ERR_TIMEOUT); }
    }
};

// The waiting loop of wait_bar, out of line: every role's wait shares one copy of it.
__device__ __noinline__ bool wait_bar_slow(uint64_t* bar, uint32_t parity, volatile int* cta, volatile int* global,
                                           uint64_t limit_ns) {
    const Abort ab{cta, global, limit_ns};
    const uint64_t t0 = globaltimer_ns();
    for (uint32_t it = 1;; ++it) {
        if (mbar_try_wait(bar, parity)) return true;
        if ((it & 31u) == 0) {
            if (ab.raised()) { *ab.cta = 1; return false; }
            if (globaltimer_ns() - t0 > ab.limit_ns) { ab.raise(); return false; }
        }
    }
}
__device__ __forceinline__ bool wait_bar(uint64_t* bar, uint32_t parity, const Abort& ab) {
    if (mbar_try_wait(bar, parity)) return true;
    return wait_bar_slow(bar, parity, ab.cta, ab.global, ab.limit_ns);
}

__device__ __forceinline__ void tma_store_3d(const CUtensorMap* map, const void* src, int32_t c0, int32_t c1,
                                             int32_t c2) {
    asm volatile("cp.async.bulk.tensor.3d.global.shared::cta.bulk_group [%0, {%2, %3, %4}], [%1];"
                 :: "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(src)), "r"(c0), "r"(c1), "r"(c2)
                 : "memory");
}
__device__ __forceinline__ void tma_store_3d_hint(const CUtensorMap* map, const void* src, int32_t c0, int32_t c1,
                                                  int32_t c2, uint64_t pol) {
    asm volatile("cp.async.bulk.tensor.3d.global.shared::cta.bulk_group.L2::cache_hint [%0, {%2, %3, %4}], [%1], %5;"
                 :: "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(src)), "r"(c0), "r"(c1), "r"(c2), "l"(pol)
                 : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait_read0() { asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait0() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

__device__ __forceinline__ void tma_prefetch_l2_3d(const CUtensorMap* map, int32_t c0, int32_t c1, int32_t c2) {
    asm volatile("cp.async.bulk.prefetch.tensor.3d.L2.global [%0, {%1, %2, %3}];"
                 :: "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(c2) : "memory");
}

// Bounded barrier of one 128-thread group built on an mbarrier (arrive, then
// wait for the phase). Unlike bar.sync it cannot hang if a member has left
// after an abort: the wait gives up at the time limit. Returns false then.
__device__ __forceinline__ bool group_sync(uint64_t* bar, uint32_t& phase, const Abort& ab) {
    mbar_arrive(bar);
    const bool ok = wait_bar(bar, phase, ab);
    phase ^= 1u;
    return ok;
}

__device__ __forceinline__ void bulk_wait_read1() { asm volatile("cp.async.bulk.wait_group.read 1;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait_read2() { asm volatile("cp.async.bulk.wait_group.read 2;" ::: "memory"); }

// Untiled bulk copies (addresses 16-byte aligned, sizes multiples of 16 bytes):
// global -> this CTA's shared memory, completing `bytes` of transactions on `bar`;
// and this CTA's shared memory -> global, in the thread's current bulk group.
__device__ __forceinline__ void bulk_load(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
                 :: "r"(smem_u32(dst)), "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(smem_u32(bar))
                 : "memory");
}
__device__ __forceinline__ void bulk_load_hint(void* dst, const void* src, uint32_t bytes, uint64_t* bar, uint64_t pol) {
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint [%0], [%1], %2, [%3], %4;"
                 :: "r"(smem_u32(dst)), "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(smem_u32(bar)), "l"(pol)
                 : "memory");
}
__device__ __forceinline__ void bulk_store_hint(void* dst, const void* src, uint32_t bytes, uint64_t pol) {
    asm volatile("cp.async.bulk.global.shared::cta.bulk_group.L2::cache_hint [%0], [%1], %2, %3;"
                 :: "l"(reinterpret_cast<uint64_t>(dst)), "r"(smem_u32(src)), "r"(bytes), "l"(pol) : "memory");
}
// Named barrier `id` of `count` threads; returns whether any of them passed `pred` true.
__device__ __forceinline__ bool bar_red_or(int id, int count, bool pred) {
    uint32_t r;
    asm volatile("{\n\t.reg .pred p, q;\n\t"
                 "setp.ne.b32 p, %1, 0;\n\t"
                 "bar.red.or.pred q, %2, %3, p;\n\t"
                 "selp.u32 %0, 1, 0, q;\n\t}"
                 : "=r"(r) : "r"((uint32_t)pred), "r"(id), "r"(count) : "memory");
    return r != 0;
}
__device__ __forceinline__ void bar_named(int id, int count) {
    asm volatile("bar.sync %0, %1;" :: "r"(id), "r"(count) : "memory");
}
__device__ __forceinline__ void bulk_store(void* dst, const void* src, uint32_t bytes) {
    asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;"
                 :: "l"(reinterpret_cast<uint64_t>(dst)), "r"(smem_u32(src)), "r"(bytes) : "memory");
}

}  // namespace sm100
}  // namespace la
