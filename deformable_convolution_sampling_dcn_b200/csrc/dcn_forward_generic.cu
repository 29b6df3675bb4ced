// Generic forward core: any shape the ABI accepts.
//
// Work mapping: one sub-warp of LPI lanes per (pixel, group) item; lane s of
// the sub-warp owns channels [s*V, (s+1)*V) of the group, V = 16 bytes of the
// storage type, so every bilinear corner fetch is one 16-byte load per lane
// and the LPI lanes of an item together read the C-contiguous corner row.
// Items are enumerated in output memory order (b, ho, wo, g), so a warp's
// stores cover consecutive 16-byte chunks.  Out-of-map corners load nothing
// and get weight zero (the four corner loads of a tap are issued together);
// sampling follows the bilinear definition of the DCNv1 page (section 2) and
// the modulation of the DCNv2 page (section 1) and the YOLOv11 + DCNv4 page
// (section 1.1: softmax over K for DCNv3, raw for DCNv4).
#include "dcn_common.cuh"
#include "dcn_launch.h"

namespace dcnb {
namespace {

template <typename T, int LPI, bool SOFTMAX>
__global__ void __launch_bounds__(256) core_forward_generic(CoreArgs a, ItemDecode dd) {
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
    T *__restrict__ out = static_cast<T *>(a.out);

    for (long long item = ((long long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5)) * IPW + slot;
         item < n_items; item += warps_total * IPW) {
        int g, wo, ho, b;
        if (n_items < (1LL << 31)) {  // 32-bit decode by multiply-high (the common case)
            unsigned r;
            unsigned t = fdiv((unsigned)item, dd.g, r);
            g = (int)r;
            t = fdiv(t, dd.wo, r);
            wo = (int)r;
            b = (int)fdiv(t, dd.ho, r);
            ho = (int)r;
        } else {
            long long t = item;
            g = (int)(t % a.G);
            t /= a.G;
            wo = (int)(t % a.Wo);
            t /= a.Wo;
            ho = (int)(t % a.Ho);
            b = (int)(t / a.Ho);
        }
        const T *o_item = off + item * K * 2;
        const T *m_item = msk + item * K;

        float mx = 0.0f, inv_sum = 1.0f;
        if (SOFTMAX) {
            mx = -INFINITY;
            for (int k = 0; k < K; ++k) mx = fmaxf(mx, load_scalar(m_item + k));
            float s = 0.0f;
            for (int k = 0; k < K; ++k) s += expf(load_scalar(m_item + k) - mx);
            inv_sum = 1.0f / s;
        }

        float acc[V];
#pragma unroll
        for (int v = 0; v < V; ++v) acc[v] = 0.0f;
        bool nan_pos = false;
        const T *xb = x + (long long)b * a.H * a.W * GC + g * a.C + sub * V;

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
                const int st = make_tap(py, px, a.H, a.W, tp);
                if (st < 0) nan_pos = true;
                // the four corner loads are issued together; an out-of-map
                // corner loads nothing and gets weight zero
                const float hy = 1.0f - tp.ly, hx = 1.0f - tp.lx;
                const float wc[4] = {hy * hx * m, hy * tp.lx * m, tp.ly * hx * m, tp.ly * tp.lx * m};
                uint4 raw[4];
                float w[4];
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    const int y = tp.y0 + (c >> 1), xx = tp.x0 + (c & 1);
                    const bool ok = st > 0 && (unsigned)y < (unsigned)a.H && (unsigned)xx < (unsigned)a.W;
                    w[c] = ok ? wc[c] : 0.0f;
                    raw[c] = ok ? ld_nc16(xb + ((long long)y * a.W + xx) * GC) : make_uint4(0, 0, 0, 0);
                }
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    float f[V];
                    unpack16<T>(raw[c], f);
#pragma unroll
                    for (int v = 0; v < V; ++v) acc[v] = fmaf(w[c], f[v], acc[v]);
                }
            }
        }
        if (nan_pos) {
#pragma unroll
            for (int v = 0; v < V; ++v) acc[v] = __int_as_float(0x7fc00000);
        }
        T *o = out + (((long long)b * a.Ho + ho) * a.Wo + wo) * GC + g * a.C + sub * V;
        *reinterpret_cast<uint4 *>(o) = pack16<T>(acc);
    }
}

template <typename T, int LPI>
cudaError_t launch_lpi(const CoreArgs &a, cudaStream_t stream) {
    const long long n_items = (long long)a.B * a.Ho * a.Wo * a.G;
    const int threads = 256;
    const long long items_per_block = (threads / 32) * (32 / LPI);
    long long blocks = (n_items + items_per_block - 1) / items_per_block;
    if (blocks > 148LL * 64) blocks = 148LL * 64;  // grid-stride beyond this
    const ItemDecode dd = make_item_decode(a.G, a.Wo, a.Ho);
    if (a.softmax)
        core_forward_generic<T, LPI, true><<<(unsigned)blocks, threads, 0, stream>>>(a, dd);
    else
        core_forward_generic<T, LPI, false><<<(unsigned)blocks, threads, 0, stream>>>(a, dd);
    return cudaGetLastError();
}

template <typename T>
cudaError_t launch_t(const CoreArgs &a, cudaStream_t stream) {
    const int lpi = a.C * (int)sizeof(T) / 16;
    switch (lpi) {
        case 1: return launch_lpi<T, 1>(a, stream);
        case 2: return launch_lpi<T, 2>(a, stream);
        case 4: return launch_lpi<T, 4>(a, stream);
        case 8: return launch_lpi<T, 8>(a, stream);
        case 16: return launch_lpi<T, 16>(a, stream);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace

cudaError_t launch_core_forward_generic(const CoreArgs &a, cudaStream_t stream) {
    switch (a.dtype) {
        case DType::F32: return launch_t<float>(a, stream);
        case DType::F16: return launch_t<__half>(a, stream);
        case DType::BF16: return launch_t<__nv_bfloat16>(a, stream);
    }
    return cudaErrorInvalidValue;
}

}  // namespace dcnb
