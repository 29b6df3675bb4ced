// Vector reductions into global memory (sm_90+ forms): one instruction adds
// 16 bytes of contributions, fp32 x4 or packed half/bfloat x8.
#pragma once

#include "dcn_common.cuh"

namespace dcnb {

template <typename T> __device__ __forceinline__ void red_add16(T *dst, const float *f);

template <> __device__ __forceinline__ void red_add16<float>(float *dst, const float *f) {
    asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};"
                 :
                 : "l"(dst), "f"(f[0]), "f"(f[1]), "f"(f[2]), "f"(f[3])
                 : "memory");
}

template <> __device__ __forceinline__ void red_add16<__half>(__half *dst, const float *f) {
    const uint4 v = pack16<__half>(f);
    asm volatile("red.global.add.noftz.v4.f16x2 [%0], {%1, %2, %3, %4};"
                 :
                 : "l"(dst), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w)
                 : "memory");
}

template <> __device__ __forceinline__ void red_add16<__nv_bfloat16>(__nv_bfloat16 *dst, const float *f) {
    const uint4 v = pack16<__nv_bfloat16>(f);
    asm volatile("red.global.add.noftz.v4.bf16x2 [%0], {%1, %2, %3, %4};"
                 :
                 : "l"(dst), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w)
                 : "memory");
}

// Sum over the `width` lanes of an aligned sub-warp (width a power of two).
template <int WIDTH> __device__ __forceinline__ float subwarp_sum(float v) {
#pragma unroll
    for (int o = WIDTH / 2; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

}  // namespace dcnb
