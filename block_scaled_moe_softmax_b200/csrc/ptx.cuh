// ptx.cuh -- thin inline-PTX wrappers for sm_100a: mbarriers, TMA, cp.async,
// tcgen05 (TMEM allocation, MMA, commit, loads) and the MX conversions.
// Written from the PTX ISA (version 8.7/8.8) descriptions of these instructions.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <stdint.h>

namespace moe_mx {

__device__ __forceinline__ uint32_t smem_u32(const void *p)
{
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint64_t global_timer_ns()
{
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// ----------------------------------------------------------------- mbarrier
__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count)
{
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_mbar_init()
{
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void fence_proxy_async_smem()
{
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar)
{
    asm volatile("mbarrier.arrive.release.cta.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes)
{
    asm volatile("mbarrier.arrive.expect_tx.release.cta.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity)
{
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.acquire.cta.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    return ok != 0;
}

// Error word bits written by bounded waits that gave up.
constexpr uint32_t kErrTimeout = 1u;

// Wait for phase `parity` of an mbarrier to complete, for at most timeout_ns
// of wall time (measured on the SM cycle counter, taken as 1 cycle per ns: at
// clocks above 1 GHz the limit only gets longer).  With a non-null global error
// word `err`, a wait that has already lasted 100 us also gives up once another
// thread has flagged an error, and a wait that runs out of time records
// kErrTimeout there.  Healthy waits never touch global memory.  Returns false
// when the wait gave up.
__device__ __forceinline__ bool mbar_wait_bounded(uint32_t bar, uint32_t parity, uint32_t *err,
                                                  uint64_t timeout_ns)
{
    if (mbar_try_wait(bar, parity))
        return true;
    const long long t0 = clock64();
    for (uint32_t it = 1;; ++it) {
        if (mbar_try_wait(bar, parity))
            return true;
        if ((it & 255) == 0) {
            const unsigned long long dt = (unsigned long long)(clock64() - t0);
            if (dt > 100000ull && err != nullptr && *(volatile uint32_t *)err != 0)
                return false;
            if (dt > timeout_ns) {
                if (err != nullptr)
                    atomicOr(err, kErrTimeout);
                return false;
            }
        }
    }
}

// ----------------------------------------------------------------- programmatic dependent launch
// A kernel launched with programmatic stream serialization may start before the kernel ahead
// of it in the stream has finished.  griddepcontrol.wait blocks the executing thread until
// every prerequisite grid has completed and its memory operations are visible (it returns at
// once when there is none); griddepcontrol.launch_dependents lets the next such kernel launch
// once every CTA of this grid has issued it or exited.
__device__ __forceinline__ void grid_dep_wait()
{
    asm volatile("griddepcontrol.wait;" ::: "memory");
}

__device__ __forceinline__ void grid_dep_launch()
{
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// ----------------------------------------------------------------- TMA / cp.async
__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap *map, int32_t x, int32_t y,
                                            uint32_t bar)
{
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3}], [%4];" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(bar)
        : "memory");
}

__device__ __forceinline__ void tma_load_3d(uint32_t dst, const CUtensorMap *map, int32_t x, int32_t y, int32_t z,
                                            uint32_t bar)
{
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3, %4}], [%5];" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(z), "r"(bar)
        : "memory");
}

__device__ __forceinline__ void prefetch_tensormap(const CUtensorMap *map)
{
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

__device__ __forceinline__ void cp_async_4(uint32_t dst, const void *src)
{
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(dst), "l"(src) : "memory");
}

// The mbarrier receives one arrival (counted against its expected count) once
// all prior cp.async of this thread have landed.
__device__ __forceinline__ void cp_async_mbar_arrive_noinc(uint32_t bar)
{
    asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(bar) : "memory");
}

// ----------------------------------------------------------------- tcgen05
__device__ __forceinline__ void tmem_alloc(uint32_t dst_smem, uint32_t ncols)
{
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst_smem),
                 "r"(ncols)
                 : "memory");
}

__device__ __forceinline__ void tmem_relinquish()
{
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols)
{
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}

__device__ __forceinline__ void tc_fence_before()
{
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}

__device__ __forceinline__ void tc_fence_after()
{
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// Arrive once on an mbarrier when all previously issued tcgen05 async ops of
// this thread have completed.
__device__ __forceinline__ void umma_commit(uint32_t bar)
{
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
                 : "memory");
}

__device__ __forceinline__ void tmem_wait_ld()
{
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// Each thread of the warp reads 16 consecutive 32-bit columns of its own lane.
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&r)[16])
{
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr)
        : "memory");
}

// Shared-memory matrix descriptor (tcgen05 "matrix descriptor"): K-major
// operand in the 128-byte swizzled canonical layout, 8-row groups 1024 bytes
// apart.  Bits: [0,14) start>>4, [16,30) leading offset>>4, [32,46) stride
// offset>>4, [46,48) version 1, [61,64) swizzle mode 2 (128B).
__device__ __forceinline__ uint64_t smem_desc_sw128(uint32_t saddr)
{
    uint64_t d = 0;
    d |= (uint64_t)((saddr >> 4) & 0x3FFF);
    d |= (uint64_t)1 << 16;           // leading byte offset (unused for swizzled K-major)
    d |= (uint64_t)(1024 >> 4) << 32; // stride byte offset: next 8-row group
    d |= (uint64_t)1 << 46;           // descriptor version
    d |= (uint64_t)2 << 61;           // 128-byte swizzle
    return d;
}

// ----------------------------------------------------------------- MX helpers
// floor(log2(a)) for a finite a > 0, read from the float's bits (handles subnormals).
__device__ __forceinline__ int floor_log2_pos(float a)
{
    uint32_t u = __float_as_uint(a);
    int e = (int)((u >> 23) & 0xFF);
    if (e != 0)
        return e - 127;
    uint32_t m = u & 0x7FFFFF;
    return -149 + (31 - __clz(m));
}

// 2^n as a float for n in [-149, 127].
__device__ __forceinline__ float exp2_int(int n)
{
    if (n >= -126)
        return __uint_as_float((uint32_t)(n + 127) << 23);
    return __uint_as_float(1u << (n + 149));
}

// max(a, b) that propagates NaN (a NaN operand gives NaN; fmaxf would drop it).
__device__ __forceinline__ float fmax_nan(float a, float b)
{
    float r;
    asm("max.NaN.f32 %0, %1, %2;" : "=f"(r) : "f"(a), "f"(b));
    return r;
}

// Round to the nearest E4M3 code (ties to even), saturating to +-448.
__device__ __forceinline__ uint32_t f32_to_e4m3(float t)
{
    uint16_t r;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %1;" : "=h"(r) : "f"(t));
    return r & 0xFF;
}

// Round to the nearest E2M1 code (ties to even), saturating to +-6.
__device__ __forceinline__ uint32_t f32_to_e2m1(float t)
{
    uint32_t r;
    asm("{\n\t.reg .b8 q;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 q, %1, %1;\n\t"
        "mov.b32 %0, {q, q, q, q};\n\t}"
        : "=r"(r)
        : "f"(t));
    return r & 0xF;
}

// Two values rounded to E4M3 codes (ties to even, saturating to +-448): a's code in
// bits [0, 8), b's in bits [8, 16) (the conversion puts its first source operand in the
// upper byte).
__device__ __forceinline__ uint32_t f32x2_to_e4m3x2(float a, float b)
{
    uint16_t r;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(b), "f"(a));
    return r;
}

// Values of the two E4M3 codes in bits [0, 8) (.x) and [8, 16) (.y) of p (exact), via
// the hardware e4m3 -> f16 conversion, which keeps each byte's position.
__device__ __forceinline__ float2 e4m3x2_to_f32x2(uint32_t p)
{
    uint32_t h2;
    asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h2) : "h"((uint16_t)(p & 0xFFFF)));
    return make_float2(__half2float(__ushort_as_half((unsigned short)(h2 & 0xFFFF))),
                       __half2float(__ushort_as_half((unsigned short)(h2 >> 16))));
}

// Value of an E4M3 code (exact), via the hardware e4m3 -> f16 conversion.
__device__ __forceinline__ float e4m3_to_f32(uint32_t code)
{
    uint32_t h2;
    uint16_t in = (uint16_t)((code & 0xFF) * 0x0101u); // same code in both bytes
    asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h2) : "h"(in));
    return __half2float(__ushort_as_half((unsigned short)(h2 & 0xFFFF)));
}

} // namespace moe_mx
