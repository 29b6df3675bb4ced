// tcgen05 (tensor-core MMA with tensor-memory accumulators), 2-D TMA and
// CTA-abort helpers of the fused core + projection kernels (sm_100a).
#pragma once

#include <cuda.h>
#include <stdint.h>

#include "dcn_tma.cuh"

namespace dcnb {

__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap *map, uint32_t bar, int c0, int c1) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];" ::"r"(
            dst),
        "l"(map), "r"(c0), "r"(c1), "r"(bar)
        : "memory");
}

__device__ __forceinline__ void tc_fence_before() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// Shared-memory matrix descriptor: K-major operand in the 128-byte swizzle
// layout, 8-row groups 1024 bytes apart (the leading-byte offset is unused
// for this layout), descriptor version 1.
__device__ __forceinline__ uint64_t smem_desc_sw128(uint32_t addr) {
    uint64_t d = (uint64_t)((addr & 0x3FFFFu) >> 4);
    d |= (uint64_t)1 << 16;           // leading byte offset (16 bytes, ignored here)
    d |= (uint64_t)(1024 >> 4) << 32; // stride byte offset
    d |= (uint64_t)1 << 46;           // version
    d |= (uint64_t)2 << 61;           // 128-byte swizzle
    return d;
}

// Instruction descriptor of kind::f16: fp32 accumulator, A and B both fp16
// (fmt 0) or both bf16 (fmt 1), both K-major, M = 128, N = n.
__device__ __forceinline__ uint32_t instr_desc_f16(int fmt, int n) {
    return (1u << 4) | ((uint32_t)fmt << 7) | ((uint32_t)fmt << 10) | ((uint32_t)(n >> 3) << 17) |
           ((uint32_t)(128 >> 4) << 24);
}

__device__ __forceinline__ void mma_f16(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                        uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// Arrive on `bar` once every tcgen05.mma this thread issued so far is complete.
__device__ __forceinline__ void mma_commit(uint32_t bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
                 : "memory");
}

__device__ __forceinline__ void tmem_ld16(uint32_t taddr, float *v) {
    uint32_t r[16];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
    for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
}

// Bounded wait (1 s) that also gives up as soon as another role of the CTA
// has raised the abort flag.
constexpr uint64_t kTcWaitNs = 1000000000ull;
__device__ __forceinline__ bool wait_or_abort(uint32_t bar, uint32_t parity, volatile int *abort_flag) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = global_timer_ns();
    while (true) {
        if (mbar_try_wait(bar, parity)) return true;
        if (*abort_flag) return false;
        if (global_timer_ns() - t0 > kTcWaitNs) return false;
        __nanosleep(64);
    }
}

__device__ __forceinline__ void raise_abort(volatile int *abort_flag, unsigned int *err) {
    *abort_flag = 1;
    atomicOr(err, kDevErrTmaTimeout);
}

// Chunk c of n of the pixel range [r0, r1).
__device__ __forceinline__ void chunk_range(long long r0, long long r1, int c, int n, long long &c0, long long &c1) {
    const long long len = r1 - r0;
    c0 = r0 + len * c / n;
    c1 = r0 + len * (c + 1) / n;
}

}  // namespace dcnb
