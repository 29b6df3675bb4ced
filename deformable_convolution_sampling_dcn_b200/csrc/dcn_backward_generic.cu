// Generic backward core: any shape the ABI accepts, global atomic scatter.
//
// Same item mapping as the generic forward (one LPI-lane sub-warp per
// (pixel, group), 16 bytes of channels per lane).  Per tap each lane forms
// the dot products d_c = <grad_out, x(corner c)> over its channels for the
// four corners; the sample value and its two position derivatives are
// linear combinations of the d_c:
//   value = sum_c G_c d_c,  d/dpx = sum_c dG_c/dpx d_c,  d/dpy likewise,
// with G_c = g(qx,px) g(qy,py) and dg/dp = -1 on floor(p), +1 on floor(p)+1
// (the bilinear kernel of the DCNv1 page, section 2, differentiated from the
// right on grid lines).  The three partial sums are reduced over the
// sub-warp with shuffles, and the input gradient m_k G_c grad_out is added
// with 16-byte vector reductions, following the thread-local accumulation +
// one atomic add per value of the Sparse4D article (section 4.2).
#include "dcn_atomic.cuh"
#include "dcn_launch.h"

namespace dcnb {
namespace {

template <typename T, int LPI, bool SOFTMAX>
__global__ void __launch_bounds__(256) core_backward_generic(CoreArgs a, ItemDecode dd) {
    constexpr int V = Storage<T>::kVec;
    constexpr int IPW = 32 / LPI;
    const int lane = threadIdx.x & 31;
    const int sub = lane % LPI;
    const int slot = lane / LPI;
    const int K = a.kh * a.kw;
    const int GC = a.G * a.C;
    const long long n_items = (long long)a.B * a.Ho * a.Wo * a.G;
    const long long warps_total = (long long)gridDim.x * (blockDim.x >> 5);
    const T *__restrict__ x = static_cast<const T *>(a.x);
    const T *__restrict__ off = static_cast<const T *>(a.offset);
    const T *__restrict__ msk = static_cast<const T *>(a.mask);
    const T *__restrict__ gout = static_cast<const T *>(a.grad_out);
    T *__restrict__ gx = static_cast<T *>(a.grad_x);
    T *__restrict__ goff = static_cast<T *>(a.grad_offset);
    T *__restrict__ gmsk = static_cast<T *>(a.grad_mask);
    float gk[SOFTMAX ? kMaxSoftmaxK : 1];

    // Warp-uniform loop: every lane runs the same iterations so that the
    // sub-warp shuffles always see all 32 lanes.
    for (long long base = ((long long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5)) * IPW;
         base < n_items; base += warps_total * IPW) {
        const long long item = base + slot;
        const bool active = item < n_items;
        const long long it = active ? item : 0;
        int g, wo, ho, b;
        if (n_items < (1LL << 31)) {  // 32-bit decode by multiply-high (the common case)
            unsigned r;
            unsigned t = fdiv((unsigned)it, dd.g, r);
            g = (int)r;
            t = fdiv(t, dd.wo, r);
            wo = (int)r;
            b = (int)fdiv(t, dd.ho, r);
            ho = (int)r;
        } else {
            long long t = it;
            g = (int)(t % a.G);
            t /= a.G;
            wo = (int)(t % a.Wo);
            t /= a.Wo;
            ho = (int)(t % a.Ho);
            b = (int)(t / a.Ho);
        }
        const T *o_item = off + it * K * 2;
        const T *m_item = msk + it * K;

        float mx = 0.0f, inv_sum = 1.0f;
        if (SOFTMAX) {
            mx = -INFINITY;
            for (int k = 0; k < K; ++k) mx = fmaxf(mx, load_scalar(m_item + k));
            float s = 0.0f;
            for (int k = 0; k < K; ++k) s += expf(load_scalar(m_item + k) - mx);
            inv_sum = 1.0f / s;
        }

        float go[V];
        const long long orow = (((long long)b * a.Ho + ho) * a.Wo + wo) * GC + g * a.C + sub * V;
        unpack16<T>(ld_nc16(gout + orow), go);
        const long long xplane = (long long)b * a.H * a.W * GC + g * a.C + sub * V;
        float dot_mg = 0.0f;  // sum_k m_k g_k, for the softmax Jacobian

        for (int i = 0; i < a.kh; ++i) {
            const int by = ho * a.sh - a.ph + i * a.dh;
            for (int j = 0; j < a.kw; ++j) {
                const int k = i * a.kw + j;
                const int bx = wo * a.sw - a.pw + j * a.dw;
                const float2 d = load_pair(o_item + 2 * k);
                float m = load_scalar(m_item + k);
                if (SOFTMAX) m = expf(m - mx) * inv_sum;
                const float px = fmaf(a.offset_scale, d.x, (float)bx);
                const float py = fmaf(a.offset_scale, d.y, (float)by);
                Tap tp{0, 0, 0.0f, 0.0f};
                int st = make_tap(py, px, a.H, a.W, tp);
                if (!active) st = 0;
                float val = 0.0f, dpx = 0.0f, dpy = 0.0f;
                // the four corner rows are loaded first (an out-of-map corner
                // loads nothing), then the dots and the reductions follow
                const float gyv[2] = {1.0f - tp.ly, tp.ly};
                const float gxv[2] = {1.0f - tp.lx, tp.lx};
                bool ok[4];
                long long r[4];
                uint4 raw[4];
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    const int y = tp.y0 + (c >> 1), xx = tp.x0 + (c & 1);
                    ok[c] = st > 0 && (unsigned)y < (unsigned)a.H && (unsigned)xx < (unsigned)a.W;
                    r[c] = xplane + ((long long)y * a.W + xx) * GC;
                    raw[c] = ok[c] ? ld_nc16(x + r[c]) : make_uint4(0, 0, 0, 0);
                }
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    const int cy = c >> 1, cx = c & 1;
                    float f[V];
                    unpack16<T>(raw[c], f);
                    float dc = 0.0f;
#pragma unroll
                    for (int v = 0; v < V; ++v) dc = fmaf(go[v], f[v], dc);
                    const float Gc = ok[c] ? gyv[cy] * gxv[cx] : 0.0f;
                    val = fmaf(Gc, dc, val);
                    dpx = fmaf(ok[c] ? (cx ? gyv[cy] : -gyv[cy]) : 0.0f, dc, dpx);
                    dpy = fmaf(ok[c] ? (cy ? gxv[cx] : -gxv[cx]) : 0.0f, dc, dpy);
                    if (ok[c]) {
                        const float mg = m * Gc;
                        float contrib[V];
#pragma unroll
                        for (int v = 0; v < V; ++v) contrib[v] = mg * go[v];
                        red_add16<T>(gx + r[c], contrib);
                    }
                }
                val = subwarp_sum<LPI>(val);
                dpx = subwarp_sum<LPI>(dpx);
                dpy = subwarp_sum<LPI>(dpy);
                if (st < 0) val = dpx = dpy = __int_as_float(0x7fc00000);
                if (active && sub == 0) {
                    const float sm = a.offset_scale * m;
                    goff[(it * K + k) * 2 + 0] = from_f32<T>(sm * dpx);
                    goff[(it * K + k) * 2 + 1] = from_f32<T>(sm * dpy);
                    if (!SOFTMAX) gmsk[it * K + k] = from_f32<T>(val);
                }
                if (SOFTMAX) {
                    gk[k] = val;
                    dot_mg = fmaf(m, val, dot_mg);
                }
            }
        }
        if (SOFTMAX && active && sub == 0) {
            for (int k = 0; k < K; ++k) {
                const float m = expf(load_scalar(m_item + k) - mx) * inv_sum;
                gmsk[it * K + k] = from_f32<T>(m * (gk[k] - dot_mg));
            }
        }
    }
}

template <typename T, int LPI>
cudaError_t launch_lpi(const CoreArgs &a, cudaStream_t stream) {
    const long long n_items = (long long)a.B * a.Ho * a.Wo * a.G;
    const int threads = 256;
    const long long items_per_block = (threads / 32) * (32 / LPI);
    long long blocks = (n_items + items_per_block - 1) / items_per_block;
    if (blocks > 148LL * 64) blocks = 148LL * 64;
    const ItemDecode dd = make_item_decode(a.G, a.Wo, a.Ho);
    if (a.softmax)
        core_backward_generic<T, LPI, true><<<(unsigned)blocks, threads, 0, stream>>>(a, dd);
    else
        core_backward_generic<T, LPI, false><<<(unsigned)blocks, threads, 0, stream>>>(a, dd);
    return cudaGetLastError();
}

template <typename T>
cudaError_t launch_t(const CoreArgs &a, cudaStream_t stream) {
    const size_t gx_bytes = (size_t)a.B * a.H * a.W * a.G * a.C * sizeof(T);
    cudaError_t e = cudaMemsetAsync(a.grad_x, 0, gx_bytes, stream);
    if (e != cudaSuccess) return e;
    switch (a.C * (int)sizeof(T) / 16) {
        case 1: return launch_lpi<T, 1>(a, stream);
        case 2: return launch_lpi<T, 2>(a, stream);
        case 4: return launch_lpi<T, 4>(a, stream);
        case 8: return launch_lpi<T, 8>(a, stream);
        case 16: return launch_lpi<T, 16>(a, stream);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace

cudaError_t launch_core_backward_generic(const CoreArgs &a, cudaStream_t stream) {
    switch (a.dtype) {
        case DType::F32: return launch_t<float>(a, stream);
        case DType::F16: return launch_t<__half>(a, stream);
        case DType::BF16: return launch_t<__nv_bfloat16>(a, stream);
    }
    return cudaErrorInvalidValue;
}

}  // namespace dcnb
