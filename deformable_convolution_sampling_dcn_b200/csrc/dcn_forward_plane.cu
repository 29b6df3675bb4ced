// Staged forward core for sm_100a: the (b, g) input plane goes through
// shared memory by TMA, and the gather reads bilinear corner pairs from it.
//
// Work split.  Items are (b, g, ho, wo) in plane-major order; the grid is
// persistent (one or two CTAs per SM) and CTA c owns the contiguous item range
// [T*c/NC, T*(c+1)/NC), so every SM gets the same number of taps.  A range is
// cut into segments, each inside one (b, g) plane and at most seg_rows output
// rows tall.
//
// Staging.  For a segment, the input rows its taps can reach (the kernel
// window plus a halo of `halo` rows for the offsets, plus one row for the
// lower bilinear corner) are loaded by 4-D TMA boxes {C, W+2, 8 rows, 1}
// starting at column -1: the out-of-range column on each side and the rows
// outside the map arrive as zeros, so a corner that leaves the map reads a
// zero and needs no test.  In shared memory pixel (y, x) of the band sits at
// ((y - ys) * (W+2) + (x+1)) * RB bytes, RB = C * sizeof(T), so the two
// horizontal corners (x0, x0+1) of a tap are one contiguous 2*RB row.
//
// Records.  Per chunk of IPW items a warp first turns every (item, point)
// into a 16-byte record {code, ly, lx, m}: code >= 0 is the byte offset of
// the corner pair (x0, x0+1) on row y0 in the band; -1 means the tap
// contributes nothing (every neighbour outside the map); -2 a NaN position;
// <= -3 a tap inside the map but outside the staged rows, encoding y0 and
// x0 for a direct read from global memory.  The modulation m is the raw mask
// or its softmax over the item's K points.
//
// Gather.  2*LPC lanes per item (LPC = RB/16): lanes [0, LPC) read the x0
// corner, lanes [LPC, 2*LPC) the x0+1 corner, 16 bytes each, so one quarter
// warp reads one 128-byte pair row: no bank conflicts.  Each lane applies
// the two vertical weights (1-ly) and ly times its horizontal weight and m,
// accumulates in fp32, and the two halves are summed with one shuffle before
// the 16-byte store.  Sampling follows the bilinear definition of the DCNv1
// page (section 2) and the modulation of the DCNv2 page (section 1) and the
// YOLOv11 + DCNv4 page (section 1.1).
#include <cudaTypedefs.h>

#include <mutex>

#include "dcn_common.cuh"
#include "dcn_launch.h"
#include "dcn_tma.cuh"

namespace dcnb {

// Set (bitwise OR) by a kernel whose bounded wait ran out.
__device__ unsigned int g_device_error = 0;

cudaError_t take_device_error(unsigned int *value) {
    unsigned int zero = 0;
    cudaError_t e = cudaMemcpyFromSymbol(value, g_device_error, sizeof(unsigned int));
    if (e != cudaSuccess) return e;
    return cudaMemcpyToSymbol(g_device_error, &zero, sizeof(unsigned int));
}

namespace {

constexpr int kBoxRows = 8;       // rows per TMA box
constexpr int kHaloMax = 8;       // rows of margin for the offsets
constexpr int kMaxK = 64;         // kernel points supported by this path
constexpr uint64_t kWaitNs = 1000000000ull;  // bounded TMA wait: 1 s

struct StagedParams {
    CoreArgs a;
    long long n_items;      // B * G * Ho * Wo
    int n_cta;              // persistent grid size
    int row_bytes;          // (W + 2) * RB: one staged row
    int buf_rows;           // staged rows the buffer holds (multiple of kBoxRows)
    int halo;               // margin rows
    int seg_rows;           // output rows per segment at most
    int rec_bytes_per_warp; // IPW * K * 16
};

struct Segment {
    long long i0, i1;  // plane-major item range
    int b, g, ho_a, ys, ye, nbox;
};

__device__ __forceinline__ Segment make_segment(long long i0, long long iend, const StagedParams &s) {
    const CoreArgs &a = s.a;
    Segment sg;
    const long long hw = (long long)a.Ho * a.Wo;
    const long long plane = i0 / hw;
    const int lp = (int)(i0 - plane * hw);
    sg.i0 = i0;
    sg.ho_a = lp / a.Wo;
    long long lim = plane * hw + (long long)(sg.ho_a + s.seg_rows) * a.Wo;
    long long pend = (plane + 1) * hw;
    sg.i1 = iend < pend ? iend : pend;
    if (lim < sg.i1) sg.i1 = lim;
    const int ho_b = (int)((sg.i1 - 1 - plane * hw) / a.Wo);
    sg.b = (int)(plane / a.G);
    sg.g = (int)(plane % a.G);
    int ys = sg.ho_a * a.sh - a.ph - s.halo;
    int ye = ho_b * a.sh - a.ph + (a.kh - 1) * a.dh + 1 + s.halo;
    sg.ys = ys < -1 ? -1 : ys;
    sg.ye = ye > a.H ? a.H : ye;
    sg.nbox = sg.ye >= sg.ys ? (sg.ye - sg.ys + kBoxRows) / kBoxRows : 0;
    return sg;
}

template <typename T, int RB, bool SOFTMAX, int THREADS, int MINB>
__global__ void __launch_bounds__(THREADS, MINB)
    core_forward_staged(const __grid_constant__ CUtensorMap tmap, const StagedParams s) {
    constexpr int V = Storage<T>::kVec;
    constexpr int LPC = RB / 16;       // lanes per corner
    constexpr int SUB = 2 * LPC;       // lanes per item
    constexpr int IPW = 32 / SUB;      // items per warp chunk
    constexpr int NW = THREADS / 32;
    const CoreArgs &a = s.a;
    const int K = a.kh * a.kw;
    const int GC = a.G * a.C;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    extern __shared__ __align__(1024) unsigned char smem[];
    // layout: [x band buffer][records per warp][softmax stats per warp][kernel table][barrier]
    unsigned char *buf = smem;
    const int buf_bytes = s.buf_rows * s.row_bytes;
    float4 *recs = reinterpret_cast<float4 *>(smem + buf_bytes) + warp * (IPW * K);
    float2 *stats = reinterpret_cast<float2 *>(smem + buf_bytes + NW * s.rec_bytes_per_warp) + warp * IPW;
    int2 *ktab = reinterpret_cast<int2 *>(smem + buf_bytes + NW * s.rec_bytes_per_warp + NW * IPW * 8);
    uint64_t *bar = reinterpret_cast<uint64_t *>(ktab + kMaxK);
    const uint32_t bar_a = smem_u32(bar);
    const uint32_t buf_a = smem_u32(buf);

    for (int k = threadIdx.x; k < K; k += THREADS) ktab[k] = make_int2((k / a.kw) * a.dh, (k % a.kw) * a.dw);
    if (threadIdx.x == 0) {
        mbar_init(bar_a, 1);
        fence_mbar_init();
    }
    __syncthreads();

    const T *__restrict__ xg = static_cast<const T *>(a.x);
    const T *__restrict__ off = static_cast<const T *>(a.offset);
    const T *__restrict__ msk = static_cast<const T *>(a.mask);
    T *__restrict__ out = static_cast<T *>(a.out);

    const long long r0 = s.n_items * blockIdx.x / s.n_cta;
    const long long r1 = s.n_items * (blockIdx.x + 1) / s.n_cta;
    const int sub = lane % SUB, slot = lane / SUB;
    const int half = sub / LPC, q = sub % LPC;
    const long long hw = (long long)a.Ho * a.Wo;
    uint32_t phase = 0;

    for (long long i0 = r0; i0 < r1;) {
        const Segment sg = make_segment(i0, r1, s);
        if (threadIdx.x == 0) {
            fence_proxy_async_smem();  // earlier reads of the buffer precede the new writes
            mbar_arrive_expect_tx(bar_a, (uint32_t)(sg.nbox * kBoxRows * s.row_bytes));
            for (int bx = 0; bx < sg.nbox; ++bx)
                tma_load_4d(buf_a + bx * kBoxRows * s.row_bytes, &tmap, bar_a, sg.g * a.C, -1,
                            sg.ys + bx * kBoxRows, sg.b);
        }
        const long long plane_base = (long long)(sg.b * a.G + sg.g) * hw;
        const int n_chunks = (int)((sg.i1 - sg.i0 + IPW - 1) / IPW);
        bool waited = false;

        for (int ch = warp; ch < n_chunks || !waited; ch += NW) {
            const bool have = ch < n_chunks;
            const long long c0 = sg.i0 + (long long)ch * IPW;
            if (have) {
                // ---- softmax statistics (one lane per item)
                if (SOFTMAX && lane < IPW) {
                    const long long it = c0 + lane;
                    float mx = -INFINITY, sum = 0.0f;
                    if (it < sg.i1) {
                        const int lp = (int)(it - plane_base);
                        const long long mi = ((long long)sg.b * hw + lp) * a.G + sg.g;
                        const T *ml = msk + mi * K;
                        for (int k = 0; k < K; ++k) mx = fmaxf(mx, load_scalar(ml + k));
                        for (int k = 0; k < K; ++k) sum += expf(load_scalar(ml + k) - mx);
                    }
                    stats[lane] = make_float2(mx, 1.0f / sum);
                }
                if (SOFTMAX) __syncwarp();
                // ---- records: one (item, point) per lane
                for (int r = lane; r < IPW * K; r += 32) {
                    const int is = r / K, k = r - is * K;
                    const long long it = c0 + is;
                    float4 rec = make_float4(__int_as_float(-1), 0.0f, 0.0f, 0.0f);
                    if (it < sg.i1) {
                        const int lp = (int)(it - plane_base);
                        const int ho = lp / a.Wo, wo = lp - ho * a.Wo;
                        const long long mi = ((long long)sg.b * hw + lp) * a.G + sg.g;
                        const int2 kt = ktab[k];
                        const float2 d = load_pair(off + (mi * K + k) * 2);
                        float m = load_scalar(msk + mi * K + k);
                        if (SOFTMAX) {
                            const float2 st = stats[is];
                            m = expf(m - st.x) * st.y;
                        }
                        const float px = fmaf(a.offset_scale, d.x, (float)(wo * a.sw - a.pw + kt.y));
                        const float py = fmaf(a.offset_scale, d.y, (float)(ho * a.sh - a.ph + kt.x));
                        Tap tp{0, 0, 0.0f, 0.0f};
                        const int st = make_tap(py, px, a.H, a.W, tp);
                        int code = -1;
                        if (st < 0) {
                            code = -2;
                        } else if (st > 0) {
                            if (tp.y0 >= sg.ys && tp.y0 + 1 <= sg.ye)
                                code = ((tp.y0 - sg.ys) * (a.W + 2) + tp.x0 + 1) * RB;
                            else
                                code = -3 - ((tp.y0 + 1) * (a.W + 2) + tp.x0 + 1);
                        }
                        rec = make_float4(__int_as_float(code), tp.ly, tp.lx, m);
                    }
                    recs[r] = rec;
                }
            }
            if (!waited) {
                // every thread takes part: the CTA agrees on success before reading the band
                const bool ok = mbar_wait_bounded(bar_a, phase, kWaitNs);
                if (__syncthreads_or(!ok)) {
                    if (threadIdx.x == 0) atomicOr(&g_device_error, kDevErrTmaTimeout);
                    mbar_wait_bounded(bar_a, phase, kWaitNs);  // let copies in flight land
                    return;
                }
                waited = true;
            }
            __syncwarp();
            if (!have) continue;

            // ---- gather
            const long long it = c0 + slot;
            const bool active = it < sg.i1;
            float acc[V];
#pragma unroll
            for (int v = 0; v < V; ++v) acc[v] = 0.0f;
            bool nan_pos = false;
            const float4 *rr = recs + slot * K;
            const uint32_t lane_off = (uint32_t)(half * RB + q * 16);
            for (int k = 0; k < K; ++k) {
                const float4 rec = rr[k];
                const int code = __float_as_int(rec.x);
                if (code == -1) continue;
                if (code == -2) {
                    nan_pos = true;
                    continue;
                }
                const float wx = half ? rec.z : 1.0f - rec.z;
                const float t = wx * rec.w;
                const float wt = fmaf(-t, rec.y, t), wb = t * rec.y;
                float ft[V], fb[V];
                if (code >= 0) {
                    const unsigned char *p = buf + code + lane_off;
                    unpack16<T>(*reinterpret_cast<const uint4 *>(p), ft);
                    unpack16<T>(*reinterpret_cast<const uint4 *>(p + s.row_bytes), fb);
                } else {
                    // inside the map, outside the staged rows: read global memory
                    const int tcode = -3 - code;
                    const int y0 = tcode / (a.W + 2) - 1;
                    const int xc = tcode % (a.W + 2) - 1 + half;
                    const bool vx = xc >= 0 && xc < a.W;
                    const T *base = xg + (long long)sg.b * a.H * a.W * GC + sg.g * a.C + q * V;
#pragma unroll
                    for (int v = 0; v < V; ++v) ft[v] = fb[v] = 0.0f;
                    if (vx && y0 >= 0) unpack16<T>(ld_nc16(base + ((long long)y0 * a.W + xc) * GC), ft);
                    if (vx && y0 + 1 < a.H) unpack16<T>(ld_nc16(base + ((long long)(y0 + 1) * a.W + xc) * GC), fb);
                }
#pragma unroll
                for (int v = 0; v < V; ++v) acc[v] = fmaf(wt, ft[v], fmaf(wb, fb[v], acc[v]));
            }
#pragma unroll
            for (int v = 0; v < V; ++v) acc[v] += __shfl_xor_sync(0xffffffffu, acc[v], LPC);
            nan_pos = __shfl_xor_sync(0xffffffffu, (int)nan_pos, LPC) != 0 || nan_pos;
            if (active && half == 0) {
                if (nan_pos) {
#pragma unroll
                    for (int v = 0; v < V; ++v) acc[v] = __int_as_float(0x7fc00000);
                }
                const int lp = (int)(it - plane_base);
                const long long mi = ((long long)sg.b * hw + lp) * a.G + sg.g;
                *reinterpret_cast<uint4 *>(out + mi * a.C + q * V) = pack16<T>(acc);
            }
            __syncwarp();
        }
        __syncthreads();  // the band is free for the next segment
        phase ^= 1u;
        i0 = sg.i1;
    }
}

// ------------------------------------------------------------------ host side
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    });
    return fn;
}

struct DeviceInfo {
    int sms = 0, smem_optin = 0, smem_per_sm = 0;
};

DeviceInfo device_info() {
    DeviceInfo d;
    int dev = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&d.sms, cudaDevAttrMultiProcessorCount, dev);
    cudaDeviceGetAttribute(&d.smem_optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
    cudaDeviceGetAttribute(&d.smem_per_sm, cudaDevAttrMaxSharedMemoryPerMultiprocessor, dev);
    return d;
}

template <typename T, int RB, bool SOFTMAX, int THREADS, int MINB>
cudaError_t launch_staged(const CUtensorMap &map, const StagedParams &s, size_t smem, cudaStream_t stream) {
    auto kern = core_forward_staged<T, RB, SOFTMAX, THREADS, MINB>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    kern<<<s.n_cta, THREADS, smem, stream>>>(map, s);
    return cudaGetLastError();
}

template <typename T, int RB>
cudaError_t launch_rb(const CoreArgs &a, cudaStream_t stream, bool *handled) {
    constexpr int SUB = 2 * (RB / 16);
    constexpr int IPW = 32 / SUB;
    const int K = a.kh * a.kw;
    if (K > kMaxK || a.W + 2 > 256) return cudaSuccess;
    auto enc = encode_fn();
    if (!enc) return cudaSuccess;
    const DeviceInfo dev = device_info();
    const int row_bytes = (a.W + 2) * RB;

    // Two CTAs per SM (256 threads each) when the band still holds segments
    // of >= 8 output rows with the full halo; otherwise one CTA (512 threads).
    StagedParams s;
    s.a = a;
    s.n_items = (long long)a.B * a.G * a.Ho * a.Wo;
    s.row_bytes = row_bytes;
    s.rec_bytes_per_warp = IPW * K * 16;
    int chosen = 0;
    size_t smem = 0;
    for (int per_sm = 2; per_sm >= 1; --per_sm) {
        const int threads = per_sm == 2 ? 256 : 512;
        const int nw = threads / 32;
        const size_t other = (size_t)nw * s.rec_bytes_per_warp + (size_t)nw * IPW * 8 + kMaxK * 8 + 16;
        const long long budget = (long long)(per_sm == 2 ? (dev.smem_per_sm / 2 - 1024) : dev.smem_optin) -
                                 (long long)other;
        if (budget <= 0) continue;
        int rows = (int)(budget / row_bytes) / kBoxRows * kBoxRows;
        const int fixed = (a.kh - 1) * a.dh + 2;  // window extent + lower corner
        int halo = kHaloMax;
        if (rows - fixed - 2 * halo < 0) halo = (rows - fixed) / 2;
        if (halo < 2) continue;
        const int seg_rows = 1 + (rows - fixed - 2 * halo) / a.sh;
        if (per_sm == 2 && (seg_rows < 8 || halo < kHaloMax) && seg_rows < a.Ho) continue;
        s.buf_rows = rows;
        s.halo = halo;
        s.seg_rows = seg_rows;
        smem = (size_t)rows * row_bytes + other;
        chosen = per_sm;
        break;
    }
    if (!chosen) return cudaSuccess;
    long long n_cta = (long long)dev.sms * chosen;
    const long long min_items = 64;
    if (n_cta * min_items > s.n_items) n_cta = (s.n_items + min_items - 1) / min_items;
    if (n_cta < 1) n_cta = 1;
    s.n_cta = (int)n_cta;

    CUtensorMap map;
    const cuuint64_t es = sizeof(T);
    const cuuint64_t dims[4] = {(cuuint64_t)a.G * a.C, (cuuint64_t)a.W, (cuuint64_t)a.H, (cuuint64_t)a.B};
    const cuuint64_t strides[3] = {dims[0] * es, dims[0] * dims[1] * es, dims[0] * dims[1] * dims[2] * es};
    const cuuint32_t box[4] = {(cuuint32_t)a.C, (cuuint32_t)(a.W + 2), (cuuint32_t)kBoxRows, 1};
    const cuuint32_t estr[4] = {1, 1, 1, 1};
    const CUtensorMapDataType dt = sizeof(T) == 4 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_UINT16;
    const CUresult r = enc(&map, dt, 4, const_cast<void *>(a.x), dims, strides, box, estr,
                           CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                           CU_TENSOR_MAP_L2_PROMOTION_L2_128B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return cudaSuccess;  // not expressible as a tensor map: generic path
    *handled = true;
    if (chosen == 2)
        return a.softmax ? launch_staged<T, RB, true, 256, 2>(map, s, smem, stream)
                         : launch_staged<T, RB, false, 256, 2>(map, s, smem, stream);
    return a.softmax ? launch_staged<T, RB, true, 512, 1>(map, s, smem, stream)
                     : launch_staged<T, RB, false, 512, 1>(map, s, smem, stream);
}

template <typename T>
cudaError_t launch_t(const CoreArgs &a, cudaStream_t stream, bool *handled) {
    switch (a.C * (int)sizeof(T)) {
        case 32: return launch_rb<T, 32>(a, stream, handled);
        case 64: return launch_rb<T, 64>(a, stream, handled);
        case 128: return launch_rb<T, 128>(a, stream, handled);
        case 256: return launch_rb<T, 256>(a, stream, handled);
        default: return cudaSuccess;  // 16-byte groups: generic path
    }
}

}  // namespace

cudaError_t launch_core_forward_plane(const CoreArgs &a, cudaStream_t stream, bool *handled) {
    *handled = false;
    switch (a.dtype) {
        case DType::F32: return launch_t<float>(a, stream, handled);
        case DType::F16: return launch_t<__half>(a, stream, handled);
        case DType::BF16: return launch_t<__nv_bfloat16>(a, stream, handled);
    }
    return cudaSuccess;
}

}  // namespace dcnb
