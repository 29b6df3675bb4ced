// Multi-camera, multi-scale deformable aggregation (Sparse4D
// deformable_aggregation article, sections 1, 2.1, 2.2 and 4).
//
// One warp per (b, anchor, group).  The warp's 32/LPI sub-warps split the
// anchor's (point, camera) pairs between them; each sub-warp walks the
// scales of its pair, so the normalised location is read once per pair.
// Lane s of a sub-warp owns 16 bytes of the group's channels, so every
// bilinear corner fetch is one 16-byte load per lane over a C-contiguous row
// of the flattened [B, rows, G*C] features.  Partial sums of the sub-warps
// are combined with shuffles at the end (forward) or per pair (backward).
#include <stdlib.h>

#include "dcn_atomic.cuh"
#include "dcn_launch.h"

namespace dcnb {
namespace {

struct AggTap {
    int st;   // 1 contributes, 0 outside, -1 not a number
    Tap t;
    int Hs, Ws, start;
};

__device__ __forceinline__ AggTap agg_tap(const AggArgs &a, float u, float v, int cam, int s) {
    AggTap r;
    const int cs = cam * a.scales + s;
    r.Hs = __ldg(a.spatial_shape + 2 * cs + 0);
    r.Ws = __ldg(a.spatial_shape + 2 * cs + 1);
    r.start = __ldg(a.scale_start + cs);
    // position (u*W_s - 0.5, v*H_s - 0.5), pixel centres at integers
    const float px = fmaf(u, (float)r.Ws, -0.5f);
    const float py = fmaf(v, (float)r.Hs, -0.5f);
    r.st = make_tap(py, px, r.Hs, r.Ws, r.t);
    return r;
}

template <typename T, int LPI>
__global__ void __launch_bounds__(256) agg_forward_kernel(AggArgs a) {
    constexpr int V = Storage<T>::kVec;
    constexpr int NSUB = 32 / LPI;
    const int lane = threadIdx.x & 31;
    const int sub = lane % LPI;
    const int sw = lane / LPI;
    const int GC = a.G * a.C;
    const long long n_items = (long long)a.B * a.A * a.G;
    const long long warps_total = (long long)gridDim.x * (blockDim.x >> 5);
    const T *__restrict__ feat = static_cast<const T *>(a.feat);
    const T *__restrict__ wts = static_cast<const T *>(a.weights);
    T *__restrict__ out = static_cast<T *>(a.out);
    const int pairs = a.P * a.cams;

    for (long long item = (long long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); item < n_items;
         item += warps_total) {
        const int g = (int)(item % a.G);
        const long long ba = item / a.G;  // b * A + anchor
        const int b = (int)(ba / a.A);
        const T *fb = feat + (long long)b * a.rows * GC + g * a.C + sub * V;
        float acc[V];
#pragma unroll
        for (int v = 0; v < V; ++v) acc[v] = 0.0f;
        bool nan_pos = false;
        for (int pc = sw; pc < pairs; pc += NSUB) {
            const int cam = pc % a.cams;
            const float2 uv = __ldg(reinterpret_cast<const float2 *>(a.loc) + ba * pairs + pc);
            for (int s = 0; s < a.scales; ++s) {
                const AggTap tp = agg_tap(a, uv.x, uv.y, cam, s);
                if (tp.st < 0) nan_pos = true;
                if (tp.st <= 0) continue;
                const float w = load_scalar(wts + ((ba * pairs + pc) * a.scales + s) * a.G + g);
                const float gyv[2] = {1.0f - tp.t.ly, tp.t.ly};
                const float gxv[2] = {1.0f - tp.t.lx, tp.t.lx};
#pragma unroll
                for (int cy = 0; cy < 2; ++cy) {
#pragma unroll
                    for (int cx = 0; cx < 2; ++cx) {
                        const int y = tp.t.y0 + cy, xx = tp.t.x0 + cx;
                        if (y < 0 || y >= tp.Hs || xx < 0 || xx >= tp.Ws) continue;
                        const long long row = (long long)tp.start + (long long)y * tp.Ws + xx;
                        if (row < 0 || row >= a.rows) continue;
                        float f[V];
                        unpack16<T>(ld_nc16(fb + row * GC), f);
                        const float wc = w * gyv[cy] * gxv[cx];
#pragma unroll
                        for (int v = 0; v < V; ++v) acc[v] = fmaf(wc, f[v], acc[v]);
                    }
                }
            }
        }
        // combine the sub-warps (lanes with equal `sub`)
#pragma unroll
        for (int o = LPI; o < 32; o <<= 1) {
#pragma unroll
            for (int v = 0; v < V; ++v) acc[v] += __shfl_xor_sync(0xffffffffu, acc[v], o);
            nan_pos |= __shfl_xor_sync(0xffffffffu, (int)nan_pos, o) != 0;
        }
        if (nan_pos) {
#pragma unroll
            for (int v = 0; v < V; ++v) acc[v] = __int_as_float(0x7fc00000);
        }
        if (sw == 0) *reinterpret_cast<uint4 *>(out + ba * GC + g * a.C + sub * V) = pack16<T>(acc);
    }
}

template <typename T, int LPI>
__global__ void __launch_bounds__(256) agg_backward_kernel(AggArgs a) {
    constexpr int V = Storage<T>::kVec;
    constexpr int NSUB = 32 / LPI;
    const int lane = threadIdx.x & 31;
    const int sub = lane % LPI;
    const int sw = lane / LPI;
    const int GC = a.G * a.C;
    const long long n_items = (long long)a.B * a.A * a.G;
    const long long warps_total = (long long)gridDim.x * (blockDim.x >> 5);
    const T *__restrict__ feat = static_cast<const T *>(a.feat);
    const T *__restrict__ wts = static_cast<const T *>(a.weights);
    const T *__restrict__ gout = static_cast<const T *>(a.grad_out);
    T *__restrict__ gfeat = static_cast<T *>(a.grad_feat);
    T *__restrict__ gw = static_cast<T *>(a.grad_weights);
    const int pairs = a.P * a.cams;
    const int rounds = (pairs + NSUB - 1) / NSUB;

    for (long long item = (long long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); item < n_items;
         item += warps_total) {
        const int g = (int)(item % a.G);
        const long long ba = item / a.G;
        const int b = (int)(ba / a.A);
        const long long fofs = (long long)b * a.rows * GC + g * a.C + sub * V;
        float go[V];
        unpack16<T>(ld_nc16(gout + ba * GC + g * a.C + sub * V), go);
        for (int r = 0; r < rounds; ++r) {  // warp-uniform
            const int pc = r * NSUB + sw;
            const bool active = pc < pairs;
            const int cam = active ? pc % a.cams : 0;
            const float2 uv = active ? __ldg(reinterpret_cast<const float2 *>(a.loc) + ba * pairs + pc)
                                     : make_float2(0.0f, 0.0f);
            float glx = 0.0f, gly = 0.0f;
            for (int s = 0; s < a.scales; ++s) {
                AggTap tp = agg_tap(a, uv.x, uv.y, cam, s);
                if (!active) tp.st = 0;
                const long long wi = ((ba * pairs + pc) * a.scales + s) * a.G + g;
                const float w = active ? load_scalar(wts + wi) : 0.0f;
                float val = 0.0f, dpx = 0.0f, dpy = 0.0f;
                if (tp.st > 0) {
                    const float gyv[2] = {1.0f - tp.t.ly, tp.t.ly};
                    const float gxv[2] = {1.0f - tp.t.lx, tp.t.lx};
#pragma unroll
                    for (int cy = 0; cy < 2; ++cy) {
#pragma unroll
                        for (int cx = 0; cx < 2; ++cx) {
                            const int y = tp.t.y0 + cy, xx = tp.t.x0 + cx;
                            if (y < 0 || y >= tp.Hs || xx < 0 || xx >= tp.Ws) continue;
                            const long long row = (long long)tp.start + (long long)y * tp.Ws + xx;
                            if (row < 0 || row >= a.rows) continue;
                            float f[V];
                            unpack16<T>(ld_nc16(feat + fofs + row * GC), f);
                            float dc = 0.0f;
#pragma unroll
                            for (int v = 0; v < V; ++v) dc = fmaf(go[v], f[v], dc);
                            const float Gc = gyv[cy] * gxv[cx];
                            val = fmaf(Gc, dc, val);
                            dpx = fmaf(cx ? gyv[cy] : -gyv[cy], dc, dpx);
                            dpy = fmaf(cy ? gxv[cx] : -gxv[cx], dc, dpy);
                            const float wg = w * Gc;
                            float contrib[V];
#pragma unroll
                            for (int v = 0; v < V; ++v) contrib[v] = wg * go[v];
                            red_add16<T>(gfeat + fofs + row * GC, contrib);
                        }
                    }
                }
                val = subwarp_sum<LPI>(val);
                dpx = subwarp_sum<LPI>(dpx);
                dpy = subwarp_sum<LPI>(dpy);
                if (tp.st < 0) val = dpx = dpy = __int_as_float(0x7fc00000);
                if (active && sub == 0) gw[wi] = from_f32<T>(val);
                glx = fmaf(w * (float)tp.Ws, dpx, glx);
                gly = fmaf(w * (float)tp.Hs, dpy, gly);
            }
            if (active && sub == 0) {
                float *gl = a.grad_loc + (ba * pairs + pc) * 2;
                atomicAdd(gl + 0, glx);
                atomicAdd(gl + 1, gly);
            }
        }
    }
}

template <typename T, int LPI>
cudaError_t launch_fwd(const AggArgs &a, cudaStream_t stream) {
    const long long n_items = (long long)a.B * a.A * a.G;
    long long blocks = (n_items + 7) / 8;
    if (blocks > 148LL * 64) blocks = 148LL * 64;
    agg_forward_kernel<T, LPI><<<(unsigned)blocks, 256, 0, stream>>>(a);
    return cudaGetLastError();
}

template <typename T, int LPI>
cudaError_t launch_bwd(const AggArgs &a, cudaStream_t stream) {
    cudaError_t e = cudaMemsetAsync(a.grad_feat, 0, (size_t)a.B * a.rows * a.G * a.C * sizeof(T), stream);
    if (e != cudaSuccess) return e;
    e = cudaMemsetAsync(a.grad_loc, 0, (size_t)a.B * a.A * a.P * a.cams * 2 * sizeof(float), stream);
    if (e != cudaSuccess) return e;
    const long long n_items = (long long)a.B * a.A * a.G;
    long long blocks = (n_items + 7) / 8;
    if (blocks > 148LL * 64) blocks = 148LL * 64;
    agg_backward_kernel<T, LPI><<<(unsigned)blocks, 256, 0, stream>>>(a);
    return cudaGetLastError();
}

template <typename T, bool BWD>
cudaError_t dispatch(const AggArgs &a, cudaStream_t stream) {
    switch (a.C * (int)sizeof(T) / 16) {
        case 1: return BWD ? launch_bwd<T, 1>(a, stream) : launch_fwd<T, 1>(a, stream);
        case 2: return BWD ? launch_bwd<T, 2>(a, stream) : launch_fwd<T, 2>(a, stream);
        case 4: return BWD ? launch_bwd<T, 4>(a, stream) : launch_fwd<T, 4>(a, stream);
        case 8: return BWD ? launch_bwd<T, 8>(a, stream) : launch_fwd<T, 8>(a, stream);
        case 16: return BWD ? launch_bwd<T, 16>(a, stream) : launch_fwd<T, 16>(a, stream);
        default: return cudaErrorInvalidValue;
    }
}

template <bool BWD>
cudaError_t dispatch_dtype(const AggArgs &a, cudaStream_t stream) {
    switch (a.dtype) {
        case DType::F32: return dispatch<float, BWD>(a, stream);
        case DType::F16: return dispatch<__half, BWD>(a, stream);
        case DType::BF16: return dispatch<__nv_bfloat16, BWD>(a, stream);
    }
    return cudaErrorInvalidValue;
}

}  // namespace

cudaError_t launch_agg_forward(const AggArgs &a, cudaStream_t stream) {
    bool handled = false;
    const char *force = getenv("DCN_B200_FORCE_GENERIC");
    if (!(force && force[0] == '1')) {
        const cudaError_t e = launch_agg_wide(a, false, stream, &handled);
        if (handled) return e;
    }
    return dispatch_dtype<false>(a, stream);
}

cudaError_t launch_agg_backward(const AggArgs &a, cudaStream_t stream) {
    bool handled = false;
    const char *force = getenv("DCN_B200_FORCE_GENERIC");
    if (!(force && force[0] == '1')) {
        const cudaError_t e = launch_agg_wide(a, true, stream, &handled);
        if (handled) return e;
    }
    return dispatch_dtype<true>(a, stream);
}

}  // namespace dcnb
