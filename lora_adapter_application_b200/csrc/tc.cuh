// tcgen05 (5th-generation tensor core) helpers shared by the tensor-core
// kernels: shared-memory matrix descriptors, the instruction descriptor, MMA
// issue / commit / tensor-memory loads, and a few bulk-copy and shared-memory
// PTX wrappers.  Field layouts restate the PTX ISA's tcgen05 descriptor
// formats.
#pragma once

#include "ptx.cuh"

namespace lora {

// ------------------------------------------------------------------ descriptors
// Shared-memory matrix descriptor (tcgen05), K-major, 128-byte swizzle: rows of
// 128 bytes in 8-row atoms of 1 KB (the layout a TMA box of 64 bf16 columns
// with 128-byte swizzle leaves behind); the next 8 rows start 1 KB later.
// Fields: start address >> 4 [0,14), leading offset >> 4 [16,30) (unused
// here), stride offset >> 4 [32,46), descriptor version 1 [46,48), layout
// 2 = 128-byte swizzle [61,64).
__device__ __forceinline__ uint64_t desc_sw128(uint32_t addr) {
    return (uint64_t)((addr >> 4) & 0x3FFFu) | (1ull << 16) | ((uint64_t)(1024 >> 4) << 32) |
           (1ull << 46) | (2ull << 61);
}
// K-major without swizzle: 8-row x 16-byte core matrices stored as 128
// contiguous bytes; the next 8 rows start 128 B later (stride offset) and the
// next 8 K elements 2 KB later (leading offset) - a TMA box of 8 bf16 columns
// x 128 rows, or the s v buffer below.
__device__ __forceinline__ uint64_t desc_plain(uint32_t addr) {
    return (uint64_t)((addr >> 4) & 0x3FFFu) | ((uint64_t)(2048 >> 4) << 16) |
           ((uint64_t)(128 >> 4) << 32) | (1ull << 46);
}
// Instruction descriptor, kind::f16: fp32 accumulator [4,6) = 1, A and B bf16
// [7,10) = [10,13) = 1, both K-major (bits 15, 16 clear), N >> 3 at [17,23),
// M >> 4 at [24,29).
__host__ __device__ constexpr uint32_t idesc_bf16(int M, int N) {
    return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(N >> 3) << 17) |
           ((uint32_t)(M >> 4) << 24);
}

// ------------------------------------------------------------------ tcgen05
__device__ __forceinline__ void tc_mma(uint32_t d, uint64_t a, uint64_t b, uint32_t idesc,
                                       uint32_t acc) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d),
        "l"(a), "l"(b), "r"(idesc), "r"(acc)
        : "memory");
}
// mbarrier arrival once every tcgen05 operation this thread issued has completed
__device__ __forceinline__ void tc_commit(uint32_t bar) {
    asm volatile(
        "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n" ::"r"(bar)
        : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
    asm volatile("tcgen05.fence::before_thread_sync;\n" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
    asm volatile("tcgen05.fence::after_thread_sync;\n" ::: "memory");
}
__device__ __forceinline__ void tc_wait_ld() {
    asm volatile("tcgen05.wait::ld.sync.aligned;\n" ::: "memory");
}
// 8 / 16 consecutive fp32 columns of this thread's tensor-memory lane
__device__ __forceinline__ void tc_ld8(uint32_t taddr, float *v) {
    uint32_t r[8];
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];\n"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]),
                   "=r"(r[6]), "=r"(r[7])
                 : "r"(taddr)
                 : "memory");
#pragma unroll
    for (int i = 0; i < 8; ++i) v[i] = __uint_as_float(r[i]);
}
__device__ __forceinline__ void tc_ld16(uint32_t taddr, float *v) {
    uint32_t r[16];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];\n"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
          "=r"(r[14]), "=r"(r[15])
        : "r"(taddr)
        : "memory");
#pragma unroll
    for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
}

// ------------------------------------------------------------------ misc PTX
__device__ __forceinline__ uint32_t cluster_rank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;\n" : "=r"(r));
    return r;
}
__device__ __forceinline__ void cluster_sync_all() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n"
                 "barrier.cluster.wait.acquire.aligned;\n" ::: "memory");
}
__device__ __forceinline__ float4 lds128f(uint32_t a) {
    float4 r;
    asm volatile("ld.shared.v4.f32 {%0,%1,%2,%3}, [%4];\n"
                 : "=f"(r.x), "=f"(r.y), "=f"(r.z), "=f"(r.w)
                 : "r"(a));
    return r;
}
__device__ __forceinline__ void sts128(uint32_t a, uint4 v) {
    asm volatile("st.shared.v4.u32 [%0], {%1,%2,%3,%4};\n" ::"r"(a), "r"(v.x), "r"(v.y), "r"(v.z),
                 "r"(v.w)
                 : "memory");
}
__device__ __forceinline__ void fence_proxy_async() {
    asm volatile("fence.proxy.async.shared::cta;\n" ::: "memory");
}
// 2-D tensor store (one box) shared -> global, tracked by this thread's bulk groups
__device__ __forceinline__ void tma_store_2d(const CUtensorMap *map, int x, int y, uint32_t src) {
    asm volatile(
        "cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%1, %2}], [%3];\n" ::"l"(
            reinterpret_cast<uint64_t>(map)),
        "r"(x), "r"(y), "r"(src)
        : "memory");
}
__device__ __forceinline__ void bulk_commit() {
    asm volatile("cp.async.bulk.commit_group;\n" ::: "memory");
}
__device__ __forceinline__ void bulk_wait_read() {
    asm volatile("cp.async.bulk.wait_group.read 0;\n" ::: "memory");
}
// every bulk group but the most recent one has finished reading shared memory
__device__ __forceinline__ void bulk_wait_read_but1() {
    asm volatile("cp.async.bulk.wait_group.read 1;\n" ::: "memory");
}
__device__ __forceinline__ void bulk_wait_all() {
    asm volatile("cp.async.bulk.wait_group 0;\n" ::: "memory");
}

// Bounded wait taken by a whole warp: every lane sees the same outcome.
template <bool CLUSTER_ACQUIRE = false>
__device__ __forceinline__ bool warp_wait(uint32_t bar, unsigned parity, int32_t *status,
                                          bool &failed) {
    bool ok = mbar_wait<CLUSTER_ACQUIRE>(bar, parity, status, failed);
    ok = __all_sync(FULL, ok);
    if (!ok) failed = true;
    return ok;
}

// y += d for 8 bf16 columns (fp32 add, one rounding)
__device__ __forceinline__ uint4 add8(uint4 y, const float *d) {
    uint4 o;
    o.x = pack_bf16x2(bf16_lo(y.x) + d[0], bf16_hi(y.x) + d[1]);
    o.y = pack_bf16x2(bf16_lo(y.y) + d[2], bf16_hi(y.y) + d[3]);
    o.z = pack_bf16x2(bf16_lo(y.z) + d[4], bf16_hi(y.z) + d[5]);
    o.w = pack_bf16x2(bf16_lo(y.w) + d[6], bf16_hi(y.w) + d[7]);
    return o;
}
// keep the first `keep` (0..8) bf16 elements of 8, zero the rest
__device__ __forceinline__ uint4 keep8(uint4 v, int keep) {
    uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        if (2 * i >= keep) w[i] = 0u;
        else if (2 * i + 1 >= keep) w[i] &= 0xffffu;
    }
    return make_uint4(w[0], w[1], w[2], w[3]);
}

}  // namespace lora
