// Deformable RoI pooling, forward ("用PyTorch实战DCNv1：从零构建可变形卷积与ROI池化模块",
// section 3): each of the PH x PW bins of a region of interest is moved by
// dp = gamma * dp_hat o (w, h), the learned offset normalised by the region
// size, and averages S x S bilinear samples of the NHWC map (the bilinear
// kernel of section 2, zeros outside the map).
//
// One warp per (roi, bin); lanes own 16-byte channel chunks, so each corner
// read is a coalesced C-contiguous row.  The sample positions are formed in
// fp32 with one rounding per operation in a fixed order (no contraction),
// so the floor() decisions are reproducible.
#include "dcn_common.cuh"
#include "dcn_launch.h"

namespace dcnb {
namespace {

// One warp per (roi, bin); lane l owns channel chunks l, l+32, ... of
// 16 * W16 bytes (CPL of them, one channel block of 32*CPL chunks at a time;
// W16 = 2 reads each chunk with one 32-byte load, sm_100's ld.global.v8, for
// which L1 returns twice the bytes per clock of 16-byte loads).  The bin
// geometry is computed by every lane (same values).  For each sample the
// four corner loads of all the lane's chunks are independent and issued
// together (an out-of-map corner loads nothing and gets weight zero); the
// sample loop is unrolled by two to keep more loads in flight.
template <int W16> struct Chunk { uint4 h[W16]; };

template <int W16> __device__ __forceinline__ Chunk<W16> ld_chunk(const void *p);
template <> __device__ __forceinline__ Chunk<1> ld_chunk<1>(const void *p) { return Chunk<1>{{ld_nc16(p)}}; }
template <> __device__ __forceinline__ Chunk<2> ld_chunk<2>(const void *p) {
    uint32_t q[8];
    asm volatile("ld.global.nc.v8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
                 : "=r"(q[0]), "=r"(q[1]), "=r"(q[2]), "=r"(q[3]), "=r"(q[4]), "=r"(q[5]), "=r"(q[6]), "=r"(q[7])
                 : "l"(p));
    return Chunk<2>{{make_uint4(q[0], q[1], q[2], q[3]), make_uint4(q[4], q[5], q[6], q[7])}};
}

template <typename T, int CPL, int W16>
__global__ void __launch_bounds__(256) roi_pool_forward_kernel(RoiArgs a) {
    constexpr int V16 = Storage<T>::kVec;  // elements per 16 bytes
    constexpr int V = V16 * W16;           // elements per chunk
    const int lane = threadIdx.x & 31;
    // N * PH * PW <= 2^31 (checked on the host): 32-bit index arithmetic
    const unsigned bins = (unsigned)a.N * (unsigned)(a.PH * a.PW);
    const unsigned bin = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    if (bin >= bins) return;
    const unsigned ij = bin % (unsigned)(a.PH * a.PW);
    const unsigned n = bin / (unsigned)(a.PH * a.PW);
    const int i = (int)(ij / (unsigned)a.PW), j = (int)(ij % (unsigned)a.PW);
    const float *r = a.rois + (long long)n * 5;
    const float rb = __ldg(r);
    const int chunks = a.C / V;
    for (int cb = 0; cb < chunks; cb += 32 * CPL) {
        T *o = static_cast<T *>(a.out) + (long long)bin * a.C + cb * V;
        const int left = chunks - cb;
        float acc[CPL][V];
#pragma unroll
        for (int q = 0; q < CPL; ++q)
#pragma unroll
            for (int v = 0; v < V; ++v) acc[q][v] = 0.0f;
        bool nan_pos = false;
        if (rb >= 0.0f && rb < (float)a.B) {  // else: batch index outside the input, nothing to read
            const int b = (int)rb;
            const float x1 = __fmul_rn(__ldg(r + 1), a.spatial_scale), y1 = __fmul_rn(__ldg(r + 2), a.spatial_scale);
            const float x2 = __fmul_rn(__ldg(r + 3), a.spatial_scale), y2 = __fmul_rn(__ldg(r + 4), a.spatial_scale);
            float rw = __fsub_rn(x2, x1), rh = __fsub_rn(y2, y1);
            if (!(rw >= 1.0f)) rw = 1.0f;
            if (!(rh >= 1.0f)) rh = 1.0f;
            const float bw = __fdiv_rn(rw, (float)a.PW), bh = __fdiv_rn(rh, (float)a.PH);
            const float sw = __fdiv_rn(bw, (float)a.S), sh = __fdiv_rn(bh, (float)a.S);
            const float2 d = __ldg(reinterpret_cast<const float2 *>(a.offset) + bin);
            const float dx = __fmul_rn(__fmul_rn(a.gamma, d.x), rw), dy = __fmul_rn(__fmul_rn(a.gamma, d.y), rh);
            const float bx0 = __fadd_rn(x1, __fmul_rn((float)j, bw)), by0 = __fadd_rn(y1, __fmul_rn((float)i, bh));
            const T *xb = static_cast<const T *>(a.x) + (long long)b * a.H * a.W * a.C + (cb + lane) * V;
            for (int sy = 0; sy < a.S; ++sy) {
                const float py = __fadd_rn(__fadd_rn(by0, __fmul_rn((float)sy + 0.5f, sh)), dy);
#pragma unroll 2
                for (int sx = 0; sx < a.S; ++sx) {
                    const float px = __fadd_rn(__fadd_rn(bx0, __fmul_rn((float)sx + 0.5f, sw)), dx);
                    Tap tp{0, 0, 0.0f, 0.0f};
                    const int st = make_tap(py, px, a.H, a.W, tp);
                    nan_pos |= st < 0;
                    float g[4];
                    long long off[4];
#pragma unroll
                    for (int c = 0; c < 4; ++c) {
                        const int y = tp.y0 + (c >> 1), x = tp.x0 + (c & 1);
                        const bool ok = st > 0 && y >= 0 && y < a.H && x >= 0 && x < a.W;
                        g[c] = ok ? ((c >> 1) ? tp.ly : 1.0f - tp.ly) * ((c & 1) ? tp.lx : 1.0f - tp.lx) : 0.0f;
                        off[c] = ok ? ((long long)y * a.W + x) * a.C : -1;
                    }
#pragma unroll
                    for (int q = 0; q < CPL; ++q) {
                        if (lane + 32 * q >= left) break;
                        Chunk<W16> raw[4];
#pragma unroll
                        for (int c = 0; c < 4; ++c) {
                            if (off[c] >= 0) {
                                raw[c] = ld_chunk<W16>(xb + off[c] + 32 * q * V);
                            } else {
#pragma unroll
                                for (int h = 0; h < W16; ++h) raw[c].h[h] = make_uint4(0, 0, 0, 0);
                            }
                        }
#pragma unroll
                        for (int c = 0; c < 4; ++c) {
                            float f[V];
#pragma unroll
                            for (int h = 0; h < W16; ++h) unpack16<T>(raw[c].h[h], f + h * V16);
#pragma unroll
                            for (int v = 0; v < V; ++v) acc[q][v] = fmaf(g[c], f[v], acc[q][v]);
                        }
                    }
                }
            }
        }
        const float inv = 1.0f / (float)(a.S * a.S);
#pragma unroll
        for (int q = 0; q < CPL; ++q) {
            const int c = lane + 32 * q;
            if (c >= left) break;
#pragma unroll
            for (int v = 0; v < V; ++v) acc[q][v] = nan_pos ? __int_as_float(0x7fc00000) : acc[q][v] * inv;
#pragma unroll
            for (int h = 0; h < W16; ++h)
                *reinterpret_cast<uint4 *>(o + c * V + h * V16) = pack16<T>(acc[q] + h * V16);
        }
    }
}

template <typename T, int W16>
cudaError_t launch_w(const RoiArgs &a, cudaStream_t stream) {
    const long long bins = (long long)a.N * a.PH * a.PW;
    const unsigned blocks = (unsigned)((bins + 7) / 8);
    const int cpl = (a.C / (Storage<T>::kVec * W16) + 31) / 32;
    if (cpl <= 1) roi_pool_forward_kernel<T, 1, W16><<<blocks, 256, 0, stream>>>(a);
    else if (cpl == 2) roi_pool_forward_kernel<T, 2, W16><<<blocks, 256, 0, stream>>>(a);
    else if (cpl <= 4) roi_pool_forward_kernel<T, 4, W16><<<blocks, 256, 0, stream>>>(a);
    else roi_pool_forward_kernel<T, 8, W16><<<blocks, 256, 0, stream>>>(a);
    return cudaGetLastError();
}

template <typename T>
cudaError_t launch_t(const RoiArgs &a, cudaStream_t stream) {
    // 32-byte chunks where every lane still gets one (rows of at least 1 KB)
    // and x sits on a 32-byte boundary (rows are then 32-byte multiples too)
    const long long row = (long long)a.C * sizeof(T);
    if (row % 32 == 0 && row >= 1024 && (reinterpret_cast<uintptr_t>(a.x) & 31) == 0)
        return launch_w<T, 2>(a, stream);
    return launch_w<T, 1>(a, stream);
}

}  // namespace

cudaError_t launch_roi_pool_forward(const RoiArgs &a, cudaStream_t stream) {
    switch (a.dtype) {
        case DType::F32: return launch_t<float>(a, stream);
        case DType::F16: return launch_t<__half>(a, stream);
        case DType::BF16: return launch_t<__nv_bfloat16>(a, stream);
    }
    return cudaErrorInvalidValue;
}

}  // namespace dcnb
