// Staged backward core: the forward's staging with the backward's arithmetic
// (fp32 storage, 128-byte groups, K <= 9; other shapes take the generic kernel).
//
// Work split, staging and records follow the staged forward
// (dcn_forward_staged.cuh): a persistent grid over plane-major (b, g, ho, wo)
// items, segments of output rows inside one (b, g) plane, the input rows a
// segment's taps can reach loaded by TMA into shared memory, and per chunk of
// IPW items one record per (item, point) built by the warp.  A record holds
// the two band addresses of the tap's upper corners, the fractional parts
// (ly, lx), the modulation m_k (after the softmax over K in DCNv3 mode), the
// global pixel index of the corner (y0, x0) and one validity bit per corner.
//
// Per tap, lane q of an item reads its 16 bytes of channels of the four
// corners from the band (from global memory for the rare tap inside the map
// but beyond the staged rows) and forms the dot products d_c = <grad_out,
// x(corner c)> over them; the sample value sum_c G_c d_c and the two position
// derivatives sum_c dG_c/dp d_c follow (the bilinear kernel of the DCNv1 page,
// section 2, differentiated from the right on grid lines) and are summed over
// the item's lanes with shuffles: grad_mask (through the softmax Jacobian in
// DCNv3 mode) and grad_offset = offset_scale * m_k * (d/dpx, d/dpy) are stored
// once.  The input gradient m_k G_c grad_out goes to grad_x with 16-byte
// vector reductions (the thread-local accumulation and one atomic add per value
// of the Sparse4D article, section 4.2).  Reading the corners from shared
// memory takes them off the SM's global load path, which the reductions need.
#include "dcn_atomic.cuh"
#include "dcn_device.h"
#include "dcn_forward_staged.cuh"

namespace dcnb {
namespace {

constexpr int kBwdThreads = 640;         // CTA size: one CTA per SM (19 consumer warps)
constexpr unsigned kFlagFallback = 16u;  // in the map, outside the staged rows
constexpr unsigned kFlagNaN = 32u;       // NaN position

template <typename T, int RB, bool SOFTMAX, int KMAX>
__global__ void __launch_bounds__(kBwdThreads, 1)
    core_backward_staged(const __grid_constant__ CUtensorMap tmap, const StagedParams s) {
    constexpr int V = Storage<T>::kVec;     // elements per 16-byte chunk
    constexpr int L = RB / 16;              // lanes per item
    constexpr int IPW = 32 / L;             // items per warp chunk
    constexpr int NT = (KMAX + L - 1) / L;  // record taps per lane
    const int NW = blockDim.x >> 5;         // warps: NW - 1 consumers and one producer
    const int NC = NW - 1;
    const CoreArgs &a = s.a;
    const int K = a.kh * a.kw;
    const int GC = a.G * a.C;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    extern __shared__ __align__(1024) unsigned char smem[];
    // [band 0][band 1 if nbuf == 2][rec (ly, lx, m): NC x KMAX x IPW float4]
    // [rec band addresses: NC x KMAX x IPW int2][rec (pixel, flags): NC x KMAX x IPW int2][ktab][4 barriers]
    const int buf_bytes = s.buf_rows * s.row_bytes;
    const int nbuf = s.nbuf;
    unsigned char *rp = smem + nbuf * buf_bytes;
    float4 *rec_g = reinterpret_cast<float4 *>(rp) + warp * KMAX * IPW;
    rp += NC * KMAX * IPW * 16;
    int2 *rec_a = reinterpret_cast<int2 *>(rp) + warp * KMAX * IPW;
    rp += NC * KMAX * IPW * 8;
    int2 *rec_p = reinterpret_cast<int2 *>(rp) + warp * KMAX * IPW;
    rp += NC * KMAX * IPW * 8;
    int2 *ktab = reinterpret_cast<int2 *>(rp);
    uint64_t *bars = reinterpret_cast<uint64_t *>(ktab + KMAX);  // full[0], full[1], empty[0], empty[1]
    const uint32_t full_a = smem_u32(bars), empty_a = smem_u32(bars + 2);

    for (int k = threadIdx.x; k < K; k += blockDim.x) ktab[k] = make_int2((k / a.kw) * a.dh, (k % a.kw) * a.dw);
    if (threadIdx.x == 0) {
        mbar_init(full_a, 1);
        mbar_init(full_a + 8, 1);
        mbar_init(empty_a, NC);
        mbar_init(empty_a + 8, NC);
        fence_mbar_init();
    }
    __syncthreads();

    const long long r0 = s.n_items * blockIdx.x / s.n_cta;
    const long long r1 = s.n_items * (blockIdx.x + 1) / s.n_cta;

    if (warp == NW - 1) {
        // ---- producer: stage the band of every segment (as in the forward)
        if (lane == 0) {
            int n = 0;
            for (long long i0 = r0; i0 < r1; ++n) {
                const Segment sg = make_segment(i0, r1, s);
                const int b = n % nbuf, u = n / nbuf;
                if (u >= 1 && !mbar_wait_bounded(empty_a + 8 * b, (u - 1) & 1, kStagedWaitNs)) {
                    atomicOr(s.err, kDevErrTmaTimeout);
                    break;
                }
                if (n == 1 && nbuf == 2 && !mbar_wait_bounded(full_a, 0, kStagedWaitNs)) {
                    atomicOr(s.err, kDevErrTmaTimeout);
                    break;
                }
                fence_proxy_async_smem();
                mbar_arrive_expect_tx(full_a + 8 * b, (uint32_t)(sg.nbox * s.box_rows * s.row_bytes));
                const uint32_t dst = smem_u32(smem + b * buf_bytes);
                for (int bx = 0; bx < sg.nbox; ++bx)
                    tma_load_4d(dst + bx * s.box_rows * s.row_bytes, &tmap, full_a + 8 * b, sg.g * a.C, -1,
                                sg.ys + bx * s.box_rows, sg.b);
                i0 = sg.i1;
            }
        }
        return;
    }

    // ---- consumers
    const T *__restrict__ xg = static_cast<const T *>(a.x);
    const T *__restrict__ off = static_cast<const T *>(a.offset);
    const T *__restrict__ msk = static_cast<const T *>(a.mask);
    const T *__restrict__ gout = static_cast<const T *>(a.grad_out);
    T *__restrict__ gx = static_cast<T *>(a.grad_x);
    T *__restrict__ goff = static_cast<T *>(a.grad_offset);
    T *__restrict__ gmsk = static_cast<T *>(a.grad_mask);
    const long long hw = (long long)a.Ho * a.Wo;
    const int gi = lane / L, q = lane % L;       // gather role
    const int ri = lane % IPW, k0 = lane / IPW;  // record role: item ri, points k0 + j*L
    const int W2 = a.W + 2;

    RawTap<T> raw[NT];
    int r_ho = 0, r_wo = 0;
    bool r_ok = false;
    auto fetch = [&](const Segment &sg, int ch) {
        const long long it = sg.i0 + (long long)ch * IPW + ri;
        r_ok = sg.i0 < sg.i1 && it < sg.i1;
        if (!r_ok) return;
        const int lp = (int)(it - ((long long)sg.b * a.G + sg.g) * hw);
        unsigned wo_u;
        r_ho = (int)fdiv((unsigned)lp, s.fd_wo, wo_u);
        r_wo = (int)wo_u;
        const long long mi = ((long long)sg.b * hw + lp) * a.G + sg.g;
#pragma unroll
        for (int j = 0; j < NT; ++j) {
            const int k = k0 + j * L;
            if (k < K) raw[j].load(off + (mi * K + k) * 2, msk + mi * K + k);
        }
    };

    Segment sg = r0 < r1 ? make_segment(r0, r1, s) : Segment{r1, r1, 0, 0, 0, 0, 0};
    int n = 0;
    fetch(sg, warp);
    while (sg.i0 < r1) {
        const int b = n % nbuf;
        const uint32_t par = (uint32_t)(n / nbuf) & 1;
        const unsigned char *band = smem + b * buf_bytes;
        const Segment nx = sg.i1 < r1 ? make_segment(sg.i1, r1, s) : Segment{r1, r1, 0, 0, 0, 0, 0};
        const long long plane_base = ((long long)sg.b * a.G + sg.g) * hw;
        const long long pix_base = (long long)sg.b * hw;
        // this segment's image in x and grad_x, at the group's channels and this lane's chunk
        const long long img = (long long)sg.b * a.H * a.W;
        const T *xq = xg + img * GC + sg.g * a.C + q * V;
        T *gxq = gx + img * GC + sg.g * a.C + q * V;
        const int n_chunks = (int)((sg.i1 - sg.i0 + IPW - 1) / IPW);
        bool ready = false;
        for (int ch = warp; ch < n_chunks || !ready; ch += NC) {
            const bool have = ch < n_chunks;
            if (have) {
                // ---- records for this chunk from the prefetched raw taps
                float m[NT];
#pragma unroll
                for (int j = 0; j < NT; ++j) m[j] = (k0 + j * L < K) ? raw[j].mask() : -INFINITY;
                if (SOFTMAX) {
                    float mx = -INFINITY;
#pragma unroll
                    for (int j = 0; j < NT; ++j) mx = fmaxf(mx, m[j]);
#pragma unroll
                    for (int o = IPW; o < 32; o <<= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
                    float sum = 0.0f;
#pragma unroll
                    for (int j = 0; j < NT; ++j) {
                        m[j] = (k0 + j * L < K) ? expf(m[j] - mx) : 0.0f;
                        sum += m[j];
                    }
#pragma unroll
                    for (int o = IPW; o < 32; o <<= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
                    const float inv = 1.0f / sum;
#pragma unroll
                    for (int j = 0; j < NT; ++j) m[j] *= inv;
                }
#pragma unroll
                for (int j = 0; j < NT; ++j) {
                    const int k = k0 + j * L;
                    if (k >= K) continue;
                    const int2 kt = ktab[k];
                    const float2 d = raw[j].pair();
                    const float px = fmaf(a.offset_scale, d.x, (float)(r_wo * a.sw - a.pw + kt.y));
                    const float py = fmaf(a.offset_scale, d.y, (float)(r_ho * a.sh - a.ph + kt.x));
                    // floor(p) by a round-down add of 1.5 * 2^23 (see the forward): every
                    // position whose floor lies outside [-1, size-1], infinite and NaN ones
                    // included, fails the unsigned map test
                    constexpr float kMagic = 12582912.0f;
                    const float tx = __fadd_rd(px, kMagic), ty = __fadd_rd(py, kMagic);
                    const unsigned x0u = (unsigned)__float_as_int(tx) - 0x4B400000u;
                    const unsigned y0u = (unsigned)__float_as_int(ty) - 0x4B400000u;
                    const float ly = py - (ty - kMagic), lx = px - (tx - kMagic);
                    const bool nanp = (px != px) | (py != py);
                    const bool inmap = (x0u + 1u <= (unsigned)a.W) & (y0u + 1u <= (unsigned)a.H);
                    const int y0 = (int)y0u, x0 = (int)x0u;
                    const bool inband = (unsigned)y0 - (unsigned)sg.ys < (unsigned)(sg.ye - sg.ys);
                    const bool tap = r_ok & inmap;
                    // corner c = 2*cy + cx at (y0 + cy, x0 + cx)
                    unsigned flags = 0;
                    if (tap) {
                        flags |= (unsigned)(y0u < (unsigned)a.H && x0u < (unsigned)a.W);
                        flags |= (unsigned)(y0u < (unsigned)a.H && x0u + 1u < (unsigned)a.W) << 1;
                        flags |= (unsigned)(y0u + 1u < (unsigned)a.H && x0u < (unsigned)a.W) << 2;
                        flags |= (unsigned)(y0u + 1u < (unsigned)a.H && x0u + 1u < (unsigned)a.W) << 3;
                        if (!inband) flags |= kFlagFallback;
                    }
                    if (r_ok & nanp) flags |= kFlagNaN;
                    const int P = (int)((((unsigned)y0 - (unsigned)sg.ys) * (unsigned)W2 + (unsigned)x0 + 1u) *
                                        (unsigned)RB);
                    rec_a[k * IPW + ri] = (tap & inband) ? make_int2(P, P + RB) : make_int2(0, 0);
                    rec_g[k * IPW + ri] = make_float4(tap ? ly : 0.0f, tap ? lx : 0.0f, m[j], 0.0f);
                    rec_p[k * IPW + ri] = make_int2(tap ? y0 * a.W + x0 : 0, (int)flags);
                }
                if (ch + NC < n_chunks) fetch(sg, ch + NC);
                else fetch(nx, warp);
            } else {
                fetch(nx, warp);
            }
            if (!ready) {
                if (!mbar_wait_bounded(full_a + 8 * b, par, kStagedWaitNs)) {
                    if (lane == 0) atomicOr(s.err, kDevErrTmaTimeout);
                    mbar_wait_bounded(full_a + 8 * b, par, kStagedWaitNs);
                    return;
                }
                ready = true;
            }
            __syncwarp();
            if (!have) continue;

            // ---- gradients of the chunk's items
            const long long it = sg.i0 + (long long)ch * IPW + gi;
            const bool active = it < sg.i1;
            const int lp = active ? (int)(it - plane_base) : 0;
            const long long mi = (pix_base + lp) * a.G + sg.g;
            float go[V];
            unpack16<T>(active ? ld_nc16(gout + mi * a.C + q * V) : make_uint4(0, 0, 0, 0), go);
            const uint32_t bq = smem_u32(band) + q * 16;
            float gk[SOFTMAX ? KMAX : 1];
            float dot_mg = 0.0f;
#pragma unroll
            for (int k = 0; k < KMAX; ++k) {
                if (k >= K) break;
                const float4 rg = rec_g[k * IPW + gi];
                const int2 ad = rec_a[k * IPW + gi];
                const int2 pf = rec_p[k * IPW + gi];
                const unsigned flags = (unsigned)pf.y;
                uint4 raw4[4];
                if (flags & kFlagFallback) {
                    const int coff[4] = {0, 1, a.W, a.W + 1};
#pragma unroll
                    for (int c = 0; c < 4; ++c)
                        raw4[c] = (flags >> c) & 1u ? ld_nc16(xq + (long long)(pf.x + coff[c]) * GC)
                                                    : make_uint4(0, 0, 0, 0);
                } else {
                    raw4[0] = lds16(bq + ad.x);
                    raw4[1] = lds16(bq + ad.y);
                    raw4[2] = lds16(bq + ad.x + s.row_bytes);
                    raw4[3] = lds16(bq + ad.y + s.row_bytes);
                }
                const float gyv[2] = {1.0f - rg.x, rg.x};
                const float gxv[2] = {1.0f - rg.y, rg.y};
                const float mk = rg.z;
                float val = 0.0f, dpx = 0.0f, dpy = 0.0f;
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    const int cy = c >> 1, cx = c & 1;
                    const bool ok = (flags >> c) & 1u;
                    float f[V];
                    unpack16<T>(raw4[c], f);
                    float dc = 0.0f;
#pragma unroll
                    for (int v = 0; v < V; ++v) dc = fmaf(go[v], f[v], dc);
                    const float Gc = ok ? gyv[cy] * gxv[cx] : 0.0f;
                    val = fmaf(Gc, dc, val);
                    dpx = fmaf(ok ? (cx ? gyv[cy] : -gyv[cy]) : 0.0f, dc, dpx);
                    dpy = fmaf(ok ? (cy ? gxv[cx] : -gxv[cx]) : 0.0f, dc, dpy);
                    if (ok && active) {
                        const float mg = mk * Gc;
                        float contrib[V];
#pragma unroll
                        for (int v = 0; v < V; ++v) contrib[v] = mg * go[v];
                        const int coff = cy * a.W + cx;
                        red_add16<T>(gxq + (long long)(pf.x + coff) * GC, contrib);
                    }
                }
                val = subwarp_sum<L>(val);
                dpx = subwarp_sum<L>(dpx);
                dpy = subwarp_sum<L>(dpy);
                if (flags & kFlagNaN) val = dpx = dpy = __int_as_float(0x7fc00000);
                if (active && q == 0) {
                    const float sm = a.offset_scale * mk;
                    goff[(mi * K + k) * 2 + 0] = from_f32<T>(sm * dpx);
                    goff[(mi * K + k) * 2 + 1] = from_f32<T>(sm * dpy);
                    if (!SOFTMAX) gmsk[mi * K + k] = from_f32<T>(val);
                }
                if (SOFTMAX) {
                    gk[k] = val;
                    dot_mg = fmaf(mk, val, dot_mg);
                }
            }
            if (SOFTMAX && active && q == 0) {
#pragma unroll
                for (int k = 0; k < KMAX; ++k) {
                    if (k >= K) break;
                    const float mk = rec_g[k * IPW + gi].z;
                    gmsk[mi * K + k] = from_f32<T>(mk * (gk[k] - dot_mg));
                }
            }
            __syncwarp();
        }
        // this warp is done with the band: the producer may refill it
        __syncwarp();
        if (lane == 0) mbar_arrive(empty_a + 8 * b);
        sg = nx;
        ++n;
    }
}

template <typename T, int RB, bool SOFTMAX, int KMAX>
cudaError_t launch_one(const CUtensorMap &map, const StagedParams &s, size_t smem, cudaStream_t stream) {
    auto kern = core_backward_staged<T, RB, SOFTMAX, KMAX>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    kern<<<s.n_cta, s.threads, smem, stream>>>(map, s);
    return cudaGetLastError();
}

constexpr int kHaloMax = 8;  // rows of margin for the offsets
constexpr int kBoxRows = 4;  // rows per TMA box

// Taken for fp32 storage with 128-byte groups (C = 32), where it measured
// faster than the generic kernel (P4 backward: 183.6 against 191.2 us).  With
// 16-bit storage the plane-major order makes the packed half-precision
// reductions of neighbouring items contend (DCNv3 P3 bf16 backward: 559 against
// 488 us), so those shapes keep the generic kernel's pixel-major order.
template <typename T>
cudaError_t launch_t(const CoreArgs &a, cudaStream_t stream, bool *handled) {
    const int RB = a.C * (int)sizeof(T);
    if (sizeof(T) != 4 || RB != 128) return cudaSuccess;
    const int K = a.kh * a.kw;
    if (K > 9 || a.W + 2 > 256) return cudaSuccess;
    if ((long long)a.Ho * a.Wo >= (1LL << 31) || (long long)a.H * a.W >= (1LL << 31)) return cudaSuccess;
    constexpr int kmax = 9;
    auto enc = encode_fn();
    const DeviceInfo *dev = device_info();
    if (!enc || !dev) return cudaSuccess;
    const int L = RB / 16, IPW = 32 / L;

    StagedParams s;
    s.a = a;
    s.n_items = (long long)a.B * a.G * a.Ho * a.Wo;
    s.row_bytes = (a.W + 2) * RB;
    s.box_rows = kBoxRows;
    s.err = dev->err;
    s.fd_wo = make_fastdiv((unsigned)a.Wo);
    s.fd_hw = make_fastdiv((unsigned)(a.Ho * a.Wo));
    s.fd_g = make_fastdiv((unsigned)a.G);
    s.fd_box = make_fastdiv((unsigned)kBoxRows);
    const int threads = kBwdThreads, nc = threads / 32 - 1;
    const size_t other = (size_t)nc * (kmax * IPW * 32) + (size_t)kmax * 8 + 32;
    const long long budget = (long long)dev->smem_optin - (long long)other;
    if (budget <= 0) return cudaSuccess;
    const int fixed = (a.kh - 1) * a.dh + 2;  // window extent + lower corner
    int chosen = 0;
    for (int nbuf = 2; nbuf >= 1; --nbuf) {
        const int rows = (int)(budget / nbuf / s.row_bytes) / kBoxRows * kBoxRows;
        int halo = kHaloMax;
        if (rows - fixed - 2 * halo < 0) halo = (rows - fixed) / 2;
        if (halo < 2) continue;
        const int seg_rows = 1 + (rows - fixed - 2 * halo) / a.sh;
        if (nbuf == 2 && (seg_rows < 8 || halo < kHaloMax) && seg_rows < a.Ho) continue;
        s.buf_rows = rows;
        s.halo = halo;
        s.seg_rows = seg_rows;
        s.nbuf = nbuf;
        chosen = 1;
        break;
    }
    if (!chosen) return cudaSuccess;
    s.threads = threads;
    const size_t smem = (size_t)s.nbuf * s.buf_rows * s.row_bytes + other;
    long long n_cta = dev->sms;
    const long long min_items = 64;
    if (n_cta * min_items > s.n_items) n_cta = (s.n_items + min_items - 1) / min_items;
    s.n_cta = (int)(n_cta < 1 ? 1 : n_cta);

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
    const size_t gx_bytes = (size_t)a.B * a.H * a.W * a.G * a.C * sizeof(T);
    cudaError_t e = cudaMemsetAsync(a.grad_x, 0, gx_bytes, stream);
    if (e != cudaSuccess) return e;
    return a.softmax ? launch_one<T, 128, true, kmax>(map, s, smem, stream)
                     : launch_one<T, 128, false, kmax>(map, s, smem, stream);
}

}  // namespace

cudaError_t launch_core_backward_staged(const CoreArgs &a, cudaStream_t stream, bool *handled) {
    *handled = false;
    if (a.dtype == DType::F32) return launch_t<float>(a, stream, handled);
    return cudaSuccess;
}

}  // namespace dcnb
