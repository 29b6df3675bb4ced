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

// One warp per (roi, bin); lane l owns 16-byte channel chunks l, l+32, ...
// (CPL of them, one channel block of 32*CPL chunks at a time).  The bin
// geometry is computed by every lane (same values).  For each sample the
// four corner loads of all the lane's chunks are independent and issued
// together (an out-of-map corner loads nothing and gets weight zero); the
// sample loop is unrolled by two to keep more loads in flight.
template <typename T, int CPL>
__global__ void __launch_bounds__(256) roi_pool_forward_kernel(RoiArgs a) {
    constexpr int V = Storage<T>::kVec;
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
                        uint4 raw[4];
#pragma unroll
                        for (int c = 0; c < 4; ++c)
                            raw[c] = off[c] >= 0 ? ld_nc16(xb + off[c] + 32 * q * V) : make_uint4(0, 0, 0, 0);
#pragma unroll
                        for (int c = 0; c < 4; ++c) {
                            float f[V];
                            unpack16<T>(raw[c], f);
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
            *reinterpret_cast<uint4 *>(o + c * V) = pack16<T>(acc[q]);
        }
    }
}

template <typename T>
cudaError_t launch_t(const RoiArgs &a, cudaStream_t stream) {
    const long long bins = (long long)a.N * a.PH * a.PW;
    const unsigned blocks = (unsigned)((bins + 7) / 8);
    const int cpl = (a.C / Storage<T>::kVec + 31) / 32;
    if (cpl <= 1) roi_pool_forward_kernel<T, 1><<<blocks, 256, 0, stream>>>(a);
    else if (cpl == 2) roi_pool_forward_kernel<T, 2><<<blocks, 256, 0, stream>>>(a);
    else if (cpl <= 4) roi_pool_forward_kernel<T, 4><<<blocks, 256, 0, stream>>>(a);
    else roi_pool_forward_kernel<T, 8><<<blocks, 256, 0, stream>>>(a);
    return cudaGetLastError();
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
