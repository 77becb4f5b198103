// sm100.cuh -- thin inline-PTX wrappers for the Blackwell (sm_100a) features
// the kernels use: mbarriers, bulk async copies (TMA engine), programmatic
// dependent launch, warp-level MMA and small bit tricks.
//
// Every wait is bounded: a wait that runs out of its clock budget sets a
// flag in global memory and returns false, so a kernel never spins forever.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/moe.h"

namespace moe {

// status word values written into a kernel's error flag (moe_device_status)
enum : int { kErrNone = MOE_DEV_OK, kErrTimeoutFull = MOE_DEV_TIMEOUT_FULL,
             kErrTimeoutEmpty = MOE_DEV_TIMEOUT_EMPTY, kErrTimeoutDrain = MOE_DEV_TIMEOUT_DRAIN,
             kErrBadSlot = MOE_DEV_BAD_SLOT, kErrTimeoutMma = MOE_DEV_TIMEOUT_MMA };

// ~4 s at 2 GHz: far above any legitimate wait in these kernels
constexpr long long kWaitBudgetCycles = 8000000000LL;

__device__ __forceinline__ uint32_t smem_u32(const void *p) {
    return (uint32_t)__cvta_generic_to_shared(p);
}

__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}

__device__ __forceinline__ void fence_mbar_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t *bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
                 "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t *bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t *bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n .reg .pred p;\n"
        " mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n"
        " selp.u32 %0, 1, 0, p;\n}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}

// try_wait that lets the hardware suspend the thread until the phase
// completes or about `ns` nanoseconds pass: a waiting warp then takes no
// issue slots from the warps doing the work.
__device__ __forceinline__ bool mbar_try_wait_sleep(uint64_t *bar, uint32_t parity, uint32_t ns) {
    uint32_t ok;
    asm volatile(
        "{\n .reg .pred p;\n"
        " mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n"
        " selp.u32 %0, 1, 0, p;\n}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity), "r"(ns)
        : "memory");
    return ok != 0;
}

// Bounded wait on a phase parity; on timeout records `code` in *err (first
// error wins) and returns false.
// budget: clock cycles before giving up (the kernels pass kWaitBudgetCycles)
__device__ __forceinline__ bool mbar_wait_budget(uint64_t *bar, uint32_t parity, int *err, int code,
                                                 long long budget) {
    if (mbar_try_wait(bar, parity)) return true;
    const long long t0 = clock64();
    while (!mbar_try_wait_sleep(bar, parity, 100000u)) {
        if (clock64() - t0 > budget) {
            if (err) atomicCAS(err, 0, code);
            return false;
        }
    }
    return true;
}
__device__ __forceinline__ bool mbar_wait(uint64_t *bar, uint32_t parity, int *err, int code) {
    return mbar_wait_budget(bar, parity, err, code, kWaitBudgetCycles);
}

// mbar_wait by every lane of a warp with one outcome for the whole warp (a
// lane that timed out makes all lanes report the timeout), so warp-wide
// synchronisation after it never waits for a lane that left.
__device__ __forceinline__ bool mbar_wait_warp(uint64_t *bar, uint32_t parity, int *err, int code) {
    return __all_sync(0xffffffffu, mbar_wait(bar, parity, err, code));
}

// Bulk async copy global -> shared (TMA engine), completion counted in bytes
// on `bar`.  dst, src 16-byte aligned; bytes a multiple of 16.
__device__ __forceinline__ void bulk_g2s(void *dst, const void *src, uint32_t bytes, uint64_t *bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
            smem_u32(dst)),
        "l"(src), "r"(bytes), "r"(smem_u32(bar))
        : "memory");
}

// 2-D tensor copy global -> shared (TMA engine) through a tensor map passed
// as a __grid_constant__ kernel parameter; box placed densely at dst.
// Coordinates in elements; x * element size must be a multiple of 16.
__device__ __forceinline__ void tma_load_2d(void *dst, const void *tmap, int x, int y, uint64_t *bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3}], [%4];" ::"r"(smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(tmap)), "r"(x), "r"(y), "r"(smem_u32(bar))
        : "memory");
}

// L2 eviction priority for data read once per call (expert weights): lines
// loaded under this policy are the first candidates for replacement, so a
// weight stream far larger than L2 does not push out what the following
// kernels reuse (their code, the router weights, activations, routing
// tables).
__device__ __forceinline__ uint64_t l2_evict_first_policy() {
    uint64_t p;
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
    return p;
}

// tma_load_2d with an L2 cache-policy hint
__device__ __forceinline__ void tma_load_2d_hint(void *dst, const void *tmap, int x, int y,
                                                 uint64_t *bar, uint64_t policy) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        ".L2::cache_hint [%0], [%1, {%2, %3}], [%4], %5;" ::"r"(smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(tmap)), "r"(x), "r"(y), "r"(smem_u32(bar)), "l"(policy)
        : "memory");
}

// 3-D tensor copy with an L2 cache-policy hint (coordinates in elements;
// x * element size a multiple of 16)
__device__ __forceinline__ void tma_load_3d_hint(void *dst, const void *tmap, int x, int y, int z,
                                                 uint64_t *bar, uint64_t policy) {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        ".L2::cache_hint [%0], [%1, {%2, %3, %4}], [%5], %6;" ::"r"(smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(tmap)), "r"(x), "r"(y), "r"(z), "r"(smem_u32(bar)),
        "l"(policy)
        : "memory");
}

// Programmatic dependent launch.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_launch_dependents() {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// D = A(16x16 f16, row) * B(16x8 f16, col) + C (f32), warp-wide.
__device__ __forceinline__ void mma_16816(float *d, const uint32_t *a, uint32_t b0, uint32_t b1,
                                          const float *c) {
    asm(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
        "{%8,%9}, {%10,%11,%12,%13};"
        : "=f"(d[0]), "=f"(d[1]), "=f"(d[2]), "=f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1), "f"(c[0]), "f"(c[1]),
          "f"(c[2]), "f"(c[3]));
}

// int8 tensor-core products, int32 accumulate: A 16x32 (row), B 32x8 (col).
// Fragments: a[0] row g, k 4c..4c+3; a[1] row g+8, same k; a[2], a[3] the
// same rows at k 16+4c..; b0 k 4c..4c+3 of column g, b1 k 16+4c..; c/d as
// the f16 shape (rows g, g+8; columns 2c, 2c+1).
__device__ __forceinline__ void imma_s8s8(int *d, const uint32_t *a, uint32_t b0, uint32_t b1,
                                          const int *c) {
    asm("mma.sync.aligned.m16n8k32.row.col.s32.s8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
        "{%8,%9}, {%10,%11,%12,%13};"
        : "=r"(d[0]), "=r"(d[1]), "=r"(d[2]), "=r"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1), "r"(c[0]), "r"(c[1]),
          "r"(c[2]), "r"(c[3]));
}
// the same with unsigned 8-bit A (Q4_0 nibble codes)
__device__ __forceinline__ void imma_u8s8(int *d, const uint32_t *a, uint32_t b0, uint32_t b1,
                                          const int *c) {
    asm("mma.sync.aligned.m16n8k32.row.col.s32.u8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
        "{%8,%9}, {%10,%11,%12,%13};"
        : "=r"(d[0]), "=r"(d[1]), "=r"(d[2]), "=r"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1), "r"(c[0]), "r"(c[1]),
          "r"(c[2]), "r"(c[3]));
}

__device__ __forceinline__ uint32_t lop3_and_or(uint32_t a, uint32_t mask, uint32_t magic) {
    uint32_t r;
    // (a & mask) | magic  -> lut 0xEA for (a & b) | c
    asm("lop3.b32 %0, %1, %2, %3, 0xEA;" : "=r"(r) : "r"(a), "r"(mask), "r"(magic));
    return r;
}

// Bit k of x (x < 16) to bit 4 of byte k: the four copies of x in
// x * (2^4 + 2^11 + 2^18 + 2^25) sit 7 bits apart (no overlap, no carries)
// and copy k puts bit k on bit 8k + 4.  The fifth bit of four 5-bit codes
// held as bytes.
__device__ __forceinline__ uint32_t spread4_bit4(uint32_t x) {
    return (x * 0x02040810u) & 0x10101010u;
}

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
    uint32_t r;
    asm("prmt.b32 %0, %1, %2, %3;" : "=r"(r) : "r"(a), "r"(b), "r"(sel));
    return r;
}

__device__ __forceinline__ uint32_t hsub2_u(uint32_t a, uint32_t b) {
    uint32_t r;
    asm("sub.rn.f16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
    return r;
}

__device__ __forceinline__ uint32_t hmul2_u(uint32_t a, uint32_t b) {
    uint32_t r;
    asm("mul.rn.f16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
    return r;
}

// a * b + c in fp16x2, one rounding
__device__ __forceinline__ uint32_t hfma2_u(uint32_t a, uint32_t b, uint32_t c) {
    uint32_t r;
    asm("fma.rn.f16x2 %0, %1, %2, %3;" : "=r"(r) : "r"(a), "r"(b), "r"(c));
    return r;
}

}  // namespace moe
