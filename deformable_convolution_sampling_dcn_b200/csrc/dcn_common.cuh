// Shared device helpers of the sm_100a deformable sampling kernels: storage
// types, 16-byte vector loads/stores with fp32 conversion, and the tap
// geometry (sampling position, bilinear corner weights) used by every kernel.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace dcnb {

// Storage types.  Every tensor of one call shares one of them; arithmetic is
// fp32 throughout.
template <typename T> struct Storage;
template <> struct Storage<float> {
    static constexpr int kVec = 4;  // elements per 16-byte vector
};
template <> struct Storage<__half> {
    static constexpr int kVec = 8;
};
template <> struct Storage<__nv_bfloat16> {
    static constexpr int kVec = 8;
};

// Unsigned division by a divisor fixed for a launch (or a chunk of work), without the
// hardware division sequence: q = mulhi(n, m) with m = floor((2^32 - 1) / d)
// underestimates n / d by at most one for n < 2^31 (n*m/2^32 lies in
// (n/d - 1, n/d)), so one remainder check makes it exact (the round-down
// reciprocal method of Granlund and Montgomery, "Division by invariant
// integers using multiplication", 1994).
struct FastDiv {
    unsigned d, m;
};
__host__ __device__ inline FastDiv make_fastdiv(unsigned d) { return FastDiv{d, 0xFFFFFFFFu / d}; }
__device__ __forceinline__ unsigned fdiv(unsigned n, FastDiv f, unsigned &r) {
    unsigned q = __umulhi(n, f.m);
    r = n - q * f.d;
    if (r >= f.d) {
        ++q;
        r -= f.d;
    }
    return q;
}

// Divisors of a flat (b, ho, wo, g) item index (g fastest), for item indices
// below 2^31.
struct ItemDecode {
    FastDiv g, wo, ho;
};
inline ItemDecode make_item_decode(int G, int Wo, int Ho) {
    return ItemDecode{make_fastdiv((unsigned)G), make_fastdiv((unsigned)Wo), make_fastdiv((unsigned)Ho)};
}

__device__ __forceinline__ float to_f32(float v) { return v; }
__device__ __forceinline__ float to_f32(__half v) { return __half2float(v); }
__device__ __forceinline__ float to_f32(__nv_bfloat16 v) { return __bfloat162float(v); }

template <typename T> __device__ __forceinline__ T from_f32(float v);
template <> __device__ __forceinline__ float from_f32<float>(float v) { return v; }
template <> __device__ __forceinline__ __half from_f32<__half>(float v) { return __float2half_rn(v); }
template <> __device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float v) {
    return __float2bfloat16_rn(v);
}

// 16 bytes through the read-only path (L1-cached, non-coherent).
__device__ __forceinline__ uint4 ld_nc16(const void *p) {
    uint4 r;
    asm volatile("ld.global.nc.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
                 : "l"(p));
    return r;
}

// Unpack a 16-byte vector into fp32 values.
template <typename T> __device__ __forceinline__ void unpack16(const uint4 &v, float *f);
template <> __device__ __forceinline__ void unpack16<float>(const uint4 &v, float *f) {
    f[0] = __uint_as_float(v.x);
    f[1] = __uint_as_float(v.y);
    f[2] = __uint_as_float(v.z);
    f[3] = __uint_as_float(v.w);
}
template <> __device__ __forceinline__ void unpack16<__half>(const uint4 &v, float *f) {
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float2 t = __half22float2(*reinterpret_cast<const __half2 *>(&w[i]));
        f[2 * i] = t.x;
        f[2 * i + 1] = t.y;
    }
}
template <> __device__ __forceinline__ void unpack16<__nv_bfloat16>(const uint4 &v, float *f) {
    // bf16 is the top half of an fp32 word: widening is a shift or a mask.
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        f[2 * i] = __uint_as_float(w[i] << 16);
        f[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
    }
}

// Unpack a 16-byte vector into V/2 fp32 pairs (for packed fp32x2 math).
template <typename T> __device__ __forceinline__ void unpack16x2(const uint4 &v, float2 *f);
template <> __device__ __forceinline__ void unpack16x2<float>(const uint4 &v, float2 *f) {
    f[0] = make_float2(__uint_as_float(v.x), __uint_as_float(v.y));
    f[1] = make_float2(__uint_as_float(v.z), __uint_as_float(v.w));
}
template <> __device__ __forceinline__ void unpack16x2<__half>(const uint4 &v, float2 *f) {
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i)
        asm("{.reg .f16 lo, hi;\n\tmov.b32 {lo, hi}, %2;\n\tcvt.f32.f16 %0, lo;\n\tcvt.f32.f16 %1, hi;}"
            : "=f"(f[i].x), "=f"(f[i].y)
            : "r"(w[i]));
}
template <> __device__ __forceinline__ void unpack16x2<__nv_bfloat16>(const uint4 &v, float2 *f) {
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) f[i] = make_float2(__uint_as_float(w[i] << 16), __uint_as_float(w[i] & 0xffff0000u));
}

// Pack fp32 values into a 16-byte vector, rounding nearest-even.
template <typename T> __device__ __forceinline__ uint4 pack16(const float *f);
template <> __device__ __forceinline__ uint4 pack16<float>(const float *f) {
    return make_uint4(__float_as_uint(f[0]), __float_as_uint(f[1]), __float_as_uint(f[2]),
                      __float_as_uint(f[3]));
}
template <> __device__ __forceinline__ uint4 pack16<__half>(const float *f) {
    uint32_t w[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const __half2 h = __floats2half2_rn(f[2 * i], f[2 * i + 1]);
        w[i] = *reinterpret_cast<const uint32_t *>(&h);
    }
    return make_uint4(w[0], w[1], w[2], w[3]);
}
template <> __device__ __forceinline__ uint4 pack16<__nv_bfloat16>(const float *f) {
    uint32_t w[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const __nv_bfloat162 h = __floats2bfloat162_rn(f[2 * i], f[2 * i + 1]);
        w[i] = *reinterpret_cast<const uint32_t *>(&h);
    }
    return make_uint4(w[0], w[1], w[2], w[3]);
}

// Load an (dx, dy) offset pair as fp32.
__device__ __forceinline__ float2 load_pair(const float *p) { return __ldg(reinterpret_cast<const float2 *>(p)); }
__device__ __forceinline__ float2 load_pair(const __half *p) {
    return __half22float2(__ldg(reinterpret_cast<const __half2 *>(p)));
}
__device__ __forceinline__ float2 load_pair(const __nv_bfloat16 *p) {
    const uint32_t w = __ldg(reinterpret_cast<const unsigned int *>(p));
    return make_float2(__uint_as_float(w << 16), __uint_as_float(w & 0xffff0000u));
}
template <typename T> __device__ __forceinline__ float load_scalar(const T *p) { return to_f32(__ldg(p)); }

// One bilinear tap.  Given the fp32 sampling position (py, px) of a map of
// size H x W, decide whether any of the four grid neighbours floor(p)+{0,1}^2
// lies inside the map, and if so return the upper-left corner (y0, x0) and
// the fractional parts.  g(a,b) = max(0, 1-|a-b|) evaluated on the four
// neighbours gives the weights (1-ly)(1-lx), (1-ly)lx, ly(1-lx), ly lx.
struct Tap {
    int y0, x0;
    float ly, lx;
};

// Returns 1 if the tap may contribute, 0 if every neighbour lies outside the
// map (or p is infinite), and -1 if p is not a number.  The support is
// floor(p) in [-1, size-1], i.e. -1 <= p < size: at p = -1 exactly the
// in-map corner has weight zero but, with the derivative taken from the
// right, a non-zero position gradient.
__device__ __forceinline__ int make_tap(float py, float px, int H, int W, Tap &t) {
    if (py != py || px != px) return -1;
    if (!(py >= -1.0f && py < (float)H && px >= -1.0f && px < (float)W)) return 0;
    const float fy = floorf(py), fx = floorf(px);
    t.y0 = (int)fy;
    t.x0 = (int)fx;
    t.ly = py - fy;
    t.lx = px - fx;
    return 1;
}

}  // namespace dcnb
