// Inline-PTX helpers shared by the tensor-pipe kernels: shared-memory
// addressing, mbarriers (bounded waits), TMA copies and vector shared loads.
#pragma once

#include "common.cuh"

#include <cuda.h>

namespace lora {

// Tries of a bounded mbarrier wait (each try suspends for up to ~20 us).
constexpr unsigned WAIT_LIMIT = 1u << 16;

__device__ __forceinline__ uint32_t smem_u32(const void *p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint32_t bar, unsigned count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;\n" ::"r"(bar), "r"(count));
}
__device__ __forceinline__ void mbar_expect_tx(uint32_t bar, unsigned bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;\n" ::"r"(bar), "r"(bytes)
                 : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];\n" ::"r"(bar) : "memory");
}
template <bool CLUSTER_ACQUIRE>
__device__ __forceinline__ bool mbar_try(uint32_t bar, unsigned parity) {
    uint32_t ok;
    if (CLUSTER_ACQUIRE)
        asm volatile(
            "{\n\t.reg .pred p;\n\t"
            "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2, 20000;\n\t"
            "selp.u32 %0, 1, 0, p;\n\t}\n"
            : "=r"(ok)
            : "r"(bar), "r"(parity)
            : "memory");
    else
        asm volatile(
            "{\n\t.reg .pred p;\n\t"
            "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, 20000;\n\t"
            "selp.u32 %0, 1, 0, p;\n\t}\n"
            : "=r"(ok)
            : "r"(bar), "r"(parity)
            : "memory");
    return ok != 0;
}
// Bounded wait; false (and the status bit) once `limit` tries have failed.
template <bool CLUSTER_ACQUIRE = false>
__device__ __forceinline__ bool mbar_wait(uint32_t bar, unsigned parity, int32_t *status,
                                          bool &failed, unsigned limit = WAIT_LIMIT) {
    if (failed) return false;
    for (unsigned it = 0; it < limit; ++it)
        if (mbar_try<CLUSTER_ACQUIRE>(bar, parity)) return true;
    atomicOr(status, LORA_DEV_TIMEOUT);
    failed = true;
    return false;
}

// 1-D bulk copy global -> shared through the TMA engine, completing on bar.
__device__ __forceinline__ void bulk_g2s(uint32_t dst, const void *src, unsigned bytes,
                                         uint32_t bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];\n" ::"r"(
            dst),
        "l"(src), "r"(bytes), "r"(bar)
        : "memory");
}
// 16 bytes global -> shared on the load/store path (L2 only), completion tracked by
// cp_async_arrive.
__device__ __forceinline__ void cp_async16(uint32_t dst, const void *src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(dst), "l"(src) : "memory");
}
// One arrival on bar once every cp.async this thread issued so far has landed (the
// barrier's expected arrival count includes it).
__device__ __forceinline__ void cp_async_arrive(uint32_t bar) {
    asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];\n" ::"r"(bar) : "memory");
}
// Pull a tensor map (kernel parameter) into the TMA unit's descriptor cache
// ahead of its first copy.
__device__ __forceinline__ void prefetch_tmap(const CUtensorMap *map) {
    asm volatile("prefetch.tensormap [%0];\n" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}
// 2-D tensor copy (one box) global -> shared through the TMA engine.
__device__ __forceinline__ void tma_2d(uint32_t dst, const CUtensorMap *map, int x, int y,
                                       uint32_t bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, "
        "{%2, %3}], [%4];\n" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(bar)
        : "memory");
}
// 3-D tensor copy (one box) global -> shared through the TMA engine.
__device__ __forceinline__ void tma_3d(uint32_t dst, const CUtensorMap *map, int x, int y, int z,
                                       uint32_t bar) {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, "
        "{%2, %3, %4}], [%5];\n" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(z), "r"(bar)
        : "memory");
}

__device__ __forceinline__ uint4 lds128(uint32_t a) {
    uint4 r;
    asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];\n"
                 : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
                 : "r"(a));
    return r;
}
__device__ __forceinline__ uint2 lds64(uint32_t a) {
    uint2 r;
    asm volatile("ld.shared.v2.u32 {%0,%1}, [%2];\n" : "=r"(r.x), "=r"(r.y) : "r"(a));
    return r;
}
__device__ __forceinline__ uint32_t lds32(uint32_t a) {
    uint32_t r;
    asm volatile("ld.shared.u32 %0, [%1];\n" : "=r"(r) : "r"(a));
    return r;
}
__device__ __forceinline__ void sts32(uint32_t a, uint32_t v) {
    asm volatile("st.shared.u32 [%0], %1;\n" ::"r"(a), "r"(v) : "memory");
}
__device__ __forceinline__ uint32_t map_rank(uint32_t addr, uint32_t rank) {
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;\n" : "=r"(r) : "r"(addr), "r"(rank));
    return r;
}
// 16 bytes into the shared memory of a block of the cluster (address and
// mbarrier both mapped with map_rank), completing 16 transaction bytes on that
// mbarrier: its waiters see the data once the phase completes, with no fence
// on either side (measured on B200: a cluster-scope fence or acquire costs
// ~1-2 us under this kernel's load, several per tile with plain stores).
__device__ __forceinline__ void st_async_f4(uint32_t addr, float a, float b, float c, float d,
                                            uint32_t bar) {
    asm volatile(
        "st.async.shared::cluster.mbarrier::complete_tx::bytes.v4.f32 [%0], {%1,%2,%3,%4}, [%5];\n" ::"r"(
            addr),
        "f"(a), "f"(b), "f"(c), "f"(d), "r"(bar)
        : "memory");
}
// 4 bytes into the shared memory of a block of the cluster, completing 4
// transaction bytes on that block's mbarrier (see st_async_f4)
__device__ __forceinline__ void st_async_f32(uint32_t addr, float v, uint32_t bar) {
    asm volatile("st.async.shared::cluster.mbarrier::complete_tx::bytes.f32 [%0], %1, [%2];\n" ::"r"(addr),
                 "f"(v), "r"(bar)
                 : "memory");
}

}  // namespace lora
