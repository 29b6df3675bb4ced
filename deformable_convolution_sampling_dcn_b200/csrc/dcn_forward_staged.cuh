// Staged forward core for sm_100a (kernel template; instantiated per storage
// type in dcn_forward_staged_{f32,f16,bf16}.cu, planned and launched from
// dcn_forward_plane.cu).
//
// Work split.  Items are (b, g, ho, wo) in plane-major order; the grid is
// persistent and CTA c owns the contiguous item range [T*c/NC, T*(c+1)/NC),
// so every SM gets the same number of taps.  A range is cut into segments,
// each inside one (b, g) plane and at most seg_rows output rows tall.
//
// Staging.  For a segment, the input rows its taps can reach (the kernel
// window, a halo for the offsets, one more row for the lower bilinear corner)
// are loaded by 4-D TMA boxes {C, W+2, box_rows, 1} that start at column -1:
// the out-of-range column on each side and the rows outside the map arrive as
// zeros.  Pixel (y, x) of the band sits at ((y - ys)*(W+2) + x + 1)*RB bytes,
// RB = C*sizeof(T), so the two horizontal corners of a tap are one contiguous
// 2*RB row, and column 0 of every staged row is zero.
//
// Records.  Per chunk of IPW items, the warp turns every (item, point) into a
// record: two corner addresses (A, B) in the band and the four bilinear
// weights g(qx,px) g(qy,py) m for (A top, A bottom, B top, B bottom).  A tap
// whose neighbours all lie outside the map points both corners at column 0
// with zero weights; a NaN position does the same with NaN weights (so the
// item's output becomes NaN); a tap inside the map but outside the staged
// rows stores negative addresses that encode its row and columns, and is read
// from global memory in a separate, rarely taken pass.  Records are stored
// point-major ([k][item]) so that one shared load serves the IPW items of a
// point.  Offsets and masks of the warp's next chunk are loaded into
// registers while the current chunk is gathered.
//
// Gather.  L = RB/16 lanes per item; lane q owns bytes [16q, 16q+16) of the
// group's channels and reads them from both corners on both rows (4 shared
// loads per tap), so it accumulates its channels completely and stores them
// without any exchange.  With RB = 64 a quarter warp covers two items; each
// item reads first the corner that lies in the bank half matching its slot
// parity, so the two 64-byte reads of a quarter warp never share a bank.
//
// Definitions: bilinear sampling per the DCNv1 page (section 2), modulation
// per the DCNv2 page (section 1), softmax over K (DCNv3) or raw (DCNv4) per
// the YOLOv11 + DCNv4 page (section 1.1).
#pragma once

#include "dcn_common.cuh"
#include "dcn_launch.h"
#include "dcn_tma.cuh"

namespace dcnb {

constexpr uint64_t kStagedWaitNs = 1000000000ull;  // bounded TMA wait: 1 s
// CTA size, one CTA per SM: 15 consumer warps, or 19 in softmax mode, whose
// longer record phase (a max, exponentials and a sum over K per item) leaves
// more latency to hide (DCNv3 P3: 167 -> 161 us; the raw-mode P4 instance
// loses with 640 threads, 41.8 -> 43.5 us, so it keeps 512).  16-byte groups
// with K > 9 hold 13 raw taps per lane and would spill at 640.
__host__ __device__ constexpr int staged_threads(bool softmax, int rb, int kmax) {
    return softmax && !(rb == 32 && kmax > 9) ? 640 : 512;
}

struct StagedParams {
    CoreArgs a;
    long long n_items;  // B * G * Ho * Wo
    int n_cta;          // persistent grid size
    int row_bytes;      // (W + 2) * RB: one staged row
    int buf_rows;       // staged rows the buffer holds (multiple of box_rows)
    int box_rows;       // rows per TMA box
    int halo;           // margin rows
    int seg_rows;       // output rows per segment at most
    unsigned int *err;  // device error word (bit 0: a TMA wait ran out)
    int threads;        // CTA size: staged_threads(softmax, RB, KMAX)
    int nbuf;           // band buffers (1 or 2): segment n uses buffer n % nbuf
    FastDiv fd_wo;      // division by Wo
    FastDiv fd_hw;      // division by Ho * Wo (used when n_items < 2^31)
    FastDiv fd_g;       // division by G (used when n_items < 2^31)
    FastDiv fd_box;     // division by box_rows
};

struct Segment {
    long long i0, i1;  // plane-major item range
    int b, g, ys, ye, nbox;
};

__device__ __forceinline__ Segment make_segment(long long i0, long long iend, const StagedParams &s) {
    const CoreArgs &a = s.a;
    Segment sg;
    const long long hw = (long long)a.Ho * a.Wo;
    const bool small = s.n_items < (1LL << 31);  // 32-bit decode by multiply-high
    unsigned r;
    const long long plane = small ? (long long)fdiv((unsigned)i0, s.fd_hw, r) : i0 / hw;
    const int lp = (int)(i0 - plane * hw);
    sg.i0 = i0;
    const int ho_a = (int)fdiv((unsigned)lp, s.fd_wo, r);
    const long long lim = plane * hw + (long long)(ho_a + s.seg_rows) * a.Wo;
    const long long pend = (plane + 1) * hw;
    sg.i1 = iend < pend ? iend : pend;
    if (lim < sg.i1) sg.i1 = lim;
    const int ho_b = (int)fdiv((unsigned)(sg.i1 - 1 - plane * hw), s.fd_wo, r);
    if (small) {
        sg.b = (int)fdiv((unsigned)plane, s.fd_g, r);
        sg.g = (int)r;
    } else {
        sg.b = (int)(plane / a.G);
        sg.g = (int)(plane % a.G);
    }
    const int ys = ho_a * a.sh - a.ph - s.halo;
    const int ye = ho_b * a.sh - a.ph + (a.kh - 1) * a.dh + 1 + s.halo;
    sg.ys = ys < -1 ? -1 : ys;
    sg.ye = ye > a.H ? a.H : ye;
    // at least one box, so that column 0 of rows 0 and 1 always exists as zeros
    sg.nbox = sg.ye >= sg.ys ? (int)fdiv((unsigned)(sg.ye - sg.ys + s.box_rows), s.fd_box, r) : 1;
    return sg;
}

// acc += w * f for a channel pair: two fp32 FMAs, or one paired fp32 FMA for
// bf16 storage, whose widening runs on the integer pipe and leaves the FMA
// pipe's issue slots to the pair (measured 175.8 -> 167.2 us on the DCNv3 P3
// workload; for fp16, whose widening shares the FMA pipe, the pair is slower).
template <typename T> __device__ __forceinline__ void fma2_bcast(float2 &acc, float w, const float2 &f) {
    acc.x = fmaf(w, f.x, acc.x);
    acc.y = fmaf(w, f.y, acc.y);
}
template <> __device__ __forceinline__ void fma2_bcast<__nv_bfloat16>(float2 &acc, float w, const float2 &f) {
    acc = __ffma2_rn(f, make_float2(w, w), acc);
}

// Raw offset pair / mask of one tap as loaded (converted at use).
template <typename T> struct RawTap;
template <> struct RawTap<float> {
    float2 d;
    float m;
    __device__ __forceinline__ void load(const float *o, const float *mk) {
        d = __ldg(reinterpret_cast<const float2 *>(o));
        m = __ldg(mk);
    }
    __device__ __forceinline__ float2 pair() const { return d; }
    __device__ __forceinline__ float mask() const { return m; }
};
template <> struct RawTap<__half> {
    uint32_t d;
    unsigned short m;
    __device__ __forceinline__ void load(const __half *o, const __half *mk) {
        d = __ldg(reinterpret_cast<const unsigned int *>(o));
        m = __ldg(reinterpret_cast<const unsigned short *>(mk));
    }
    __device__ __forceinline__ float2 pair() const {
        return __half22float2(*reinterpret_cast<const __half2 *>(&d));
    }
    __device__ __forceinline__ float mask() const { return __half2float(__ushort_as_half(m)); }
};
template <> struct RawTap<__nv_bfloat16> {
    uint32_t d;
    unsigned short m;
    __device__ __forceinline__ void load(const __nv_bfloat16 *o, const __nv_bfloat16 *mk) {
        d = __ldg(reinterpret_cast<const unsigned int *>(o));
        m = __ldg(reinterpret_cast<const unsigned short *>(mk));
    }
    __device__ __forceinline__ float2 pair() const {
        return make_float2(__uint_as_float(d << 16), __uint_as_float(d & 0xffff0000u));
    }
    __device__ __forceinline__ float mask() const { return __uint_as_float((uint32_t)m << 16); }
};

template <typename T, int RB, bool SOFTMAX, int KMAX>
__global__ void __launch_bounds__(staged_threads(SOFTMAX, RB, KMAX), 1)
    core_forward_staged(const __grid_constant__ CUtensorMap tmap, const StagedParams s) {
    constexpr int V = Storage<T>::kVec;  // elements per 16-byte chunk
    constexpr int V2 = V / 2;            // fp32 pairs per chunk
    constexpr int L = RB / 16;           // lanes per item
    constexpr int IPW = 32 / L;          // items per warp chunk
    constexpr int NT = (KMAX + L - 1) / L;  // record taps per lane
    const int NW = blockDim.x >> 5;      // warps: NW - 1 consumers and one producer
    const int NC = NW - 1;
    const CoreArgs &a = s.a;
    const int K = a.kh * a.kw;
    const int GC = a.G * a.C;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    // a programmatic dependent on the stream (the projection GEMM) may launch
    // now; it waits for this grid's completion before reading its output
    asm volatile("griddepcontrol.launch_dependents;");

    extern __shared__ __align__(1024) unsigned char smem[];
    // [band 0][band 1 if nbuf == 2][rec weights: NC x KMAX x IPW float4][rec addrs: NC x KMAX x IPW int2]
    // [fallback descriptors: NC x KMAX x IPW int][fallback masks: NC x IPW uint][ktab][4 barriers]
    const int buf_bytes = s.buf_rows * s.row_bytes;
    const int nbuf = s.nbuf;
    unsigned char *rp = smem + nbuf * buf_bytes;
    float4 *rec_w = reinterpret_cast<float4 *>(rp) + warp * KMAX * IPW;
    rp += NC * KMAX * IPW * 16;
    int2 *rec_a = reinterpret_cast<int2 *>(rp) + warp * KMAX * IPW;
    rp += NC * KMAX * IPW * 8;
    int *rec_f = reinterpret_cast<int *>(rp) + warp * KMAX * IPW;
    rp += NC * KMAX * IPW * 4;
    unsigned *fbm = reinterpret_cast<unsigned *>(rp) + warp * IPW;
    rp += NC * IPW * 4;
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
        // ---- producer: stage the band of every segment, two buffers ahead
        if (lane == 0) {
            int n = 0;
            for (long long i0 = r0; i0 < r1; ++n) {
                const Segment sg = make_segment(i0, r1, s);
                const int b = n % nbuf, u = n / nbuf;  // buffer and its use count
                // wait until every consumer released this buffer's previous use
                if (u >= 1 && !mbar_wait_bounded(empty_a + 8 * b, (u - 1) & 1, kStagedWaitNs)) {
                    atomicOr(s.err, kDevErrTmaTimeout);
                    break;
                }
                // the second band of the CTA starts after the first has landed, so the
                // first one is not slowed down by it at kernel start
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
    T *__restrict__ out = static_cast<T *>(a.out);
    const long long hw = (long long)a.Ho * a.Wo;
    const int gi = lane / L, q = lane % L;        // gather role
    const int ri = lane % IPW, k0 = lane / IPW;   // record role: item ri, points k0 + j*L
    const int W2 = a.W + 2;

    // raw taps of the record role's next chunk, loaded one chunk ahead
    RawTap<T> raw[NT];
    int r_ho = 0, r_wo = 0;
    bool r_ok = false;
    auto fetch = [&](const Segment &sg, int ch) {
        const long long it = sg.i0 + (long long)ch * IPW + ri;
        r_ok = sg.i0 < sg.i1 && it < sg.i1;
        if (!r_ok) return;
        // pixel index inside the segment's (b, g) plane
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
                unsigned fmask = 0;  // points of item ri read from global memory (this lane's share)
#pragma unroll
                for (int j = 0; j < NT; ++j) {
                    const int k = k0 + j * L;
                    if (k >= K) continue;
                    // Branch-free: every lane of the warp takes the same instructions,
                    // whatever case its tap falls in.
                    const int2 kt = ktab[k];
                    const float2 d = raw[j].pair();
                    const float px = fmaf(a.offset_scale, d.x, (float)(r_wo * a.sw - a.pw + kt.y));
                    const float py = fmaf(a.offset_scale, d.y, (float)(r_ho * a.sh - a.ph + kt.x));
                    // floor by a round-down add of 1.5 * 2^23: exact for |p| < 2^22 (then the
                    // integer is the low mantissa bits); every other position, infinite and NaN
                    // ones included, yields a corner index outside [-1, size-1], so the
                    // unsigned tests below are the map test
                    constexpr float kMagic = 12582912.0f;
                    const float tx = __fadd_rd(px, kMagic), ty = __fadd_rd(py, kMagic);
                    const unsigned x0u = (unsigned)__float_as_int(tx) - 0x4B400000u;
                    const unsigned y0u = (unsigned)__float_as_int(ty) - 0x4B400000u;
                    const float ly = py - (ty - kMagic), lx = px - (tx - kMagic);  // NaN for a NaN position
                    const bool nanp = (px != px) | (py != py);
                    // floor(p) in [-1, size-1], i.e. -1 <= p < size
                    const bool inmap = (x0u + 1u <= (unsigned)a.W) & (y0u + 1u <= (unsigned)a.H);
                    const int y0 = (int)y0u, x0 = (int)x0u;  // meaningful only when inmap
                    const bool inband = (unsigned)y0 - (unsigned)sg.ys < (unsigned)(sg.ye - sg.ys);
                    const bool smem_tap = r_ok & inmap & inband;
                    const bool fb_tap = r_ok & inmap & !inband;
                    const float mk = m[j];
                    const float tx0 = (1.0f - lx) * mk, tx1 = lx * mk;
                    const float w00 = fmaf(-tx0, ly, tx0), w10 = tx0 * ly;
                    const float w01 = fmaf(-tx1, ly, tx1), w11 = tx1 * ly;
                    const int P = (int)((((unsigned)y0 - (unsigned)sg.ys) * (unsigned)W2 + (unsigned)x0 + 1u) *
                                        (unsigned)RB);
                    const bool order = (RB == 64) && ((((unsigned)P >> 6) ^ (unsigned)ri) & 1u);
                    int2 ad = order ? make_int2(P + RB, P) : make_int2(P, P + RB);
                    if (!smem_tap) ad = make_int2(0, 0);  // column 0 of the band: zeros
                    float4 w = (smem_tap && order) ? make_float4(w01, w11, w00, w10) : make_float4(w00, w10, w01, w11);
                    if (!(r_ok & (inmap | nanp))) w = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
                    // inside the map, outside the staged rows: the staged pass reads zeros
                    // here and the fallback pass adds the global corners
                    if (fb_tap) rec_f[k * IPW + ri] = (y0 + 1) * W2 + x0 + 1;
                    fmask |= (unsigned)fb_tap << k;
                    rec_w[k * IPW + ri] = w;
                    rec_a[k * IPW + ri] = ad;
                }
#pragma unroll
                for (int o = IPW; o < 32; o <<= 1) fmask |= __shfl_xor_sync(0xffffffffu, fmask, o);
                if (k0 == 0) fbm[ri] = fmask;
                // next chunk of this warp: later in this segment, or its first chunk of the next
                if (ch + NC < n_chunks) fetch(sg, ch + NC);
                else fetch(nx, warp);
            } else {
                fetch(nx, warp);  // no chunk here: prefetch this warp's first chunk of the next segment
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

            // ---- gather: staged corners for every point, branch-free
            const long long it = sg.i0 + (long long)ch * IPW + gi;
            float2 acc[V2];
#pragma unroll
            for (int v = 0; v < V2; ++v) acc[v] = make_float2(0.0f, 0.0f);
            const uint32_t bqa = smem_u32(band) + q * 16;  // 32-bit shared addresses
#pragma unroll
            for (int k = 0; k < KMAX; ++k) {
                if (k >= K) break;
                const float4 w = rec_w[k * IPW + gi];
                const int2 ad = rec_a[k * IPW + gi];
                const uint4 va = lds16(bqa + ad.x);
                const uint4 vb = lds16(bqa + ad.x + s.row_bytes);
                const uint4 vc = lds16(bqa + ad.y);
                const uint4 vd = lds16(bqa + ad.y + s.row_bytes);
                float2 f[V2];
                unpack16x2<T>(va, f);
#pragma unroll
                for (int v = 0; v < V2; ++v) fma2_bcast<T>(acc[v], w.x, f[v]);
                unpack16x2<T>(vb, f);
#pragma unroll
                for (int v = 0; v < V2; ++v) fma2_bcast<T>(acc[v], w.y, f[v]);
                unpack16x2<T>(vc, f);
#pragma unroll
                for (int v = 0; v < V2; ++v) fma2_bcast<T>(acc[v], w.z, f[v]);
                unpack16x2<T>(vd, f);
#pragma unroll
                for (int v = 0; v < V2; ++v) fma2_bcast<T>(acc[v], w.w, f[v]);
            }
            // ---- taps inside the map but outside the staged rows (rare)
            for (unsigned fm = fbm[gi]; fm; fm &= fm - 1) {
                const int k = __ffs(fm) - 1;
                const float4 w = rec_w[k * IPW + gi];
                const int t0 = rec_f[k * IPW + gi];
                const int y0 = t0 / W2 - 1;
                const int x0 = t0 - (y0 + 1) * W2 - 1;
                const T *base = xg + (long long)sg.b * a.H * a.W * GC + sg.g * a.C + q * V;
                const float wv[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
                for (int c = 0; c < 2; ++c) {
#pragma unroll
                    for (int r = 0; r < 2; ++r) {
                        const int yy = y0 + r, xx = x0 + c;
                        if (yy < 0 || yy >= a.H || xx < 0 || xx >= a.W) continue;
                        float2 f[V2];
                        unpack16x2<T>(ld_nc16(base + ((long long)yy * a.W + xx) * GC), f);
#pragma unroll
                        for (int v = 0; v < V2; ++v) fma2_bcast<T>(acc[v], wv[2 * c + r], f[v]);
                    }
                }
            }
            if (it < sg.i1) {
                const int lp = (int)(it - plane_base);
                const long long mi = (pix_base + lp) * a.G + sg.g;
                *reinterpret_cast<uint4 *>(out + mi * a.C + q * V) = pack16<T>(reinterpret_cast<const float *>(acc));
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

// Launch one instance: RB in {32, 64, 128, 256}, kmax in {9, 25}.
template <typename T>
cudaError_t launch_staged_instance(const CUtensorMap &map, const StagedParams &s, int RB, bool softmax, int kmax,
                                   size_t smem, cudaStream_t stream);

template <typename T, int RB, bool SOFTMAX, int KMAX>
cudaError_t launch_staged_one(const CUtensorMap &map, const StagedParams &s, size_t smem, cudaStream_t stream) {
    auto kern = core_forward_staged<T, RB, SOFTMAX, KMAX>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    kern<<<s.n_cta, s.threads, smem, stream>>>(map, s);
    return cudaGetLastError();
}

#define DCNB_STAGED_INSTANCE(T)                                                                                     \
    template <>                                                                                                     \
    cudaError_t launch_staged_instance<T>(const CUtensorMap &map, const StagedParams &s, int RB, bool softmax,      \
                                          int kmax, size_t smem, cudaStream_t stream) {                             \
        _Pragma("nv_diag_suppress 128")                                                                             \
        switch (RB * 4 + (softmax ? 2 : 0) + (kmax > 9 ? 1 : 0)) {                                                  \
            case 32 * 4 + 0: return launch_staged_one<T, 32, false, 9>(map, s, smem, stream);                      \
            case 32 * 4 + 1: return launch_staged_one<T, 32, false, 25>(map, s, smem, stream);                     \
            case 32 * 4 + 2: return launch_staged_one<T, 32, true, 9>(map, s, smem, stream);                       \
            case 32 * 4 + 3: return launch_staged_one<T, 32, true, 25>(map, s, smem, stream);                      \
            case 64 * 4 + 0: return launch_staged_one<T, 64, false, 9>(map, s, smem, stream);                      \
            case 64 * 4 + 1: return launch_staged_one<T, 64, false, 25>(map, s, smem, stream);                     \
            case 64 * 4 + 2: return launch_staged_one<T, 64, true, 9>(map, s, smem, stream);                       \
            case 64 * 4 + 3: return launch_staged_one<T, 64, true, 25>(map, s, smem, stream);                      \
            case 128 * 4 + 0: return launch_staged_one<T, 128, false, 9>(map, s, smem, stream);                    \
            case 128 * 4 + 1: return launch_staged_one<T, 128, false, 25>(map, s, smem, stream);                   \
            case 128 * 4 + 2: return launch_staged_one<T, 128, true, 9>(map, s, smem, stream);                     \
            case 128 * 4 + 3: return launch_staged_one<T, 128, true, 25>(map, s, smem, stream);                    \
            case 256 * 4 + 0: return launch_staged_one<T, 256, false, 9>(map, s, smem, stream);                    \
            case 256 * 4 + 1: return launch_staged_one<T, 256, false, 25>(map, s, smem, stream);                   \
            case 256 * 4 + 2: return launch_staged_one<T, 256, true, 9>(map, s, smem, stream);                     \
            case 256 * 4 + 3: return launch_staged_one<T, 256, true, 25>(map, s, smem, stream);                    \
        }                                                                                                           \
        return cudaErrorInvalidValue;                                                                               \
    }

}  // namespace dcnb
