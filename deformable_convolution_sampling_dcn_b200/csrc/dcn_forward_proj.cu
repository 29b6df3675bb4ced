// Forward core fused with the pointwise projection that follows it in the
// DCNv4 module (YOLOv11 + DCNv4 article, section 3.2: the core's output goes
// through a 1x1 convolution with bias):
//     out[p, o] = bias[o] + sum_j Wt[o, j] * core[p, j],  j = g*C + c.
// The core tile never leaves the SM.
//
// The same kernel runs the modulated deformable convolution (DCNv2 page,
// section 1: every kernel point has its own dense weight):
//     out[p, o] = bias[o] + sum_k sum_j Wt[o, k, j] * m_k * x_j(p + p_k + dp_k).
// There the K-blocks run over (kernel point, 64 channels) and each item
// samples only its K-block's point, so the tensor core contracts over all
// K * G * C sampled values instead of the G * C core values.
//
// Work split.  The B*Ho*Wo pixels are cut into one contiguous range per CTA
// (persistent grid, one CTA per SM), processed in chunks of at most 128
// pixels.  Per chunk:
//   1. Twenty gather warps sample the core for every (pixel, group) of the
//      chunk (sub-warp per item, as in the generic kernel), in K-blocks of 64
//      channels.  Each result is rounded once to the storage type (the value
//      an unfused core would store) and written straight into shared memory
//      as the tensor-core B operand: rows = pixels, 128 bytes of channels per
//      row and K-block, in the 128-byte-swizzled K-major layout (16-byte chunk
//      c of row n sits at chunk c ^ (n mod 8)).  When a warp has finished its
//      part of a K-block it arrives on that K-block's barrier.
//   2. A producer warp streams 128 x 64 tiles of the weight (A operand,
//      rows = output channels) with TMA into a four-stage ring.
//   3. One thread of the MMA warp issues tcgen05.mma (kind::f16, M = 128 output
//      channels, N = chunk pixels padded to 16, K = 16 per instruction) for
//      each K-block as soon as it is complete, so the products overlap the
//      gather of the next K-block.  The fp32 accumulators live in tensor
//      memory: output-channel block mb occupies columns [mb*N, (mb+1)*N).
//   4. The gather warps read the accumulators back (tcgen05.ld, 32 lanes x 16
//      columns per load), add the bias, round and store the output rows.
// Every wait is bounded (1 s); a wait that runs out sets the device error
// word, stops the CTA's remaining work, drains the copies and products it
// already issued and frees its tensor memory.
#include <type_traits>

#include "dcn_common.cuh"
#include "dcn_device.h"
#include "dcn_launch.h"
#include "dcn_tcgen05.cuh"
#include "dcn_tma.cuh"

namespace dcnb {
namespace {

constexpr int kGatherWarps = 20;
constexpr int kProducerWarp = kGatherWarps;
constexpr int kMmaWarp = kGatherWarps + 1;
constexpr int kProjThreads = (kGatherWarps + 2) * 32;
constexpr int kWStages = 4;
constexpr int kWTileBytes = 128 * 128;  // 128 rows x 64 elements x 2 bytes
constexpr int kWTileBytesSwap = 256 * 128;  // 256 output channels x 64 elements x 2 bytes
constexpr int kMaxChunk = 128;          // pixels per chunk (MMA N <= 128)
constexpr int kBSlots = 4;             // B-operand ring: K-blocks in flight
constexpr uint64_t kProjWaitNs = 1000000000ull;

struct ProjParams {
    CoreArgs a;
    const void *bias;   // [Cout] storage type, or nullptr
    long long P;        // output pixels B*Ho*Wo
    int Cout;
    int MB;             // ceil(Cout / 128) output-channel blocks
    int KB;             // 64-channel K-blocks of the contraction
    int cbk;            // K-blocks per kernel point (KB when the points are summed first)
    int per_point;      // 1: deformable convolution, one K-block per (point, channel block)
    int lg_gpb;         // log2 of the groups per K-block (64 / C)
    int pp_records;     // per-point mode with one record per item (32-item steps)
    FastDiv fd_cbk, fd_howo, fd_wo;  // K-blocks per point, Ho*Wo, Wo
    int n_cta;
    int npad_max;       // largest padded chunk of any CTA (B operand rows)
    int tmem_cols;      // allocated tensor-memory columns (power of two >= 32)
    int w_box_rows;     // rows per weight TMA box: min(Cout, 128), or min(Cout16, 256) when swapped
    int cout16;         // Cout rounded up to a multiple of 16
    unsigned int *err;
};

// Zeros read by the corners of a tap that lie outside the map (one group row
// of at most 128 bytes).
__device__ __align__(16) unsigned char g_zero_row[128];

// Work of a chunk: its n_px * G (pixel, group) items in one flat list,
// K-block by K-block and group-major inside a K-block (pixels fastest), so
// consecutive items of a warp sample neighbouring pixels of one group.  The
// list is dealt to the gather warps in steps of IPW items, round-robin, so
// every warp gets the same number of steps whatever the K-block sizes.
struct ItemPos {
    int kb, k, g, px;  // K-block, kernel point (per-point mode), group, pixel in the chunk
};
__device__ __forceinline__ ItemPos item_pos(int item, FastDiv fd_npx, const ProjParams &p) {
    // item = (kb * gpb + gl) * n_px + px, kb = k * cbk + cb, g = cb * gpb + gl
    ItemPos r;
    unsigned px, cb;
    const unsigned q = fdiv((unsigned)item, fd_npx, px);
    r.px = (int)px;
    r.kb = (int)(q >> p.lg_gpb);
    const int gl = (int)(q & ((1u << p.lg_gpb) - 1u));
    r.k = (int)fdiv((unsigned)r.kb, p.fd_cbk, cb);
    r.g = ((int)cb << p.lg_gpb) + gl;
    return r;
}

// Offsets and masks of points k0, k0 + LPI, ... of flat item `item` (the
// record role's raw taps), loaded one step ahead of their use.
template <typename T, int LPI, bool SOFTMAX, int NT>
__device__ __forceinline__ void load_raw(const ProjParams &p, long long c0, FastDiv fd_npx, int total,
                                         int item, int k0, float *dx, float *dy, float *m) {
    const CoreArgs &a = p.a;
    const int K = a.kh * a.kw;
    const bool valid = item < total;
    const ItemPos ip = item_pos(valid ? item : 0, fd_npx, p);
    const long long mi = (c0 + ip.px) * a.G + ip.g;
    const T *off = static_cast<const T *>(a.offset);
    const T *msk = static_cast<const T *>(a.mask);
#pragma unroll
    for (int j = 0; j < NT; ++j) {
        const int k = k0 + j * LPI;
        dx[j] = dy[j] = 0.0f;
        m[j] = SOFTMAX ? -INFINITY : 0.0f;
        if (valid && k < K) {
            const float2 d = load_pair(off + (mi * K + k) * 2);
            dx[j] = d.x;
            dy[j] = d.y;
            m[j] = load_scalar(msk + mi * K + k);
        }
    }
}

// One step: items [base, base + IPW) of the chunk's flat list, sampled into
// the B-operand slots of their K-blocks.
//
// RECORDS (K <= 9, 2..8 lanes per item): the lanes first turn every (item,
// point) into a record in shared memory - the four bilinear weights with the
// modulation folded in and the four corner pixel indices (-1: outside the
// map, read from the zero row) - computed once by one lane from the raw
// taps loaded one step earlier; then the LPI lanes of each item read the
// records and gather their 16-byte channel chunks of the four corners
// through L1.  Otherwise every lane of an item computes the taps itself.
template <typename T, int LPI, bool SOFTMAX, int KMAX, bool RECORDS, int NT>
__device__ __forceinline__ void gather_step(const ProjParams &p, int ci, long long c0, FastDiv fd_npx, int total,
                                            int base, int lane, unsigned char *bring, int slot_bytes,
                                            float4 *rec_w, int4 *rec_o, const int2 *ktab, const float *dx,
                                            const float *dy, const float *m_raw) {
    constexpr int V = Storage<T>::kVec;
    constexpr int IPW = 32 / LPI;
    const CoreArgs &a = p.a;
    const int K = a.kh * a.kw;
    const int GC = a.G * a.C;
    const T *__restrict__ xg = static_cast<const T *>(a.x);
    const int gi = lane / LPI, q = lane % LPI;  // gather role
    const int item = base + gi;
    const bool valid = item < total;
    const ItemPos ip = item_pos(valid ? item : 0, fd_npx, p);
    const unsigned pix = (unsigned)(c0 + ip.px);
    unsigned rem;
    const unsigned b = fdiv(pix, p.fd_howo, rem);
    const T *xb = xg + (long long)b * a.H * a.W * GC + ip.g * a.C + q * V;
    float acc[V];
#pragma unroll
    for (int v = 0; v < V; ++v) acc[v] = 0.0f;
    if (RECORDS) {
        // ---- records: lane (ri, k0) builds points k0, k0 + LPI, ... of item ri
        const int ri = lane % IPW, k0 = lane / IPW;
        const int item_r = base + ri;
        const bool valid_r = item_r < total;
        const ItemPos ipr = item_pos(valid_r ? item_r : 0, fd_npx, p);
        unsigned rem_r, wo_r;
        fdiv((unsigned)(c0 + ipr.px), p.fd_howo, rem_r);
        const int ho = (int)fdiv(rem_r, p.fd_wo, wo_r), wo = (int)wo_r;
        float m[NT];
#pragma unroll
        for (int j = 0; j < NT; ++j) m[j] = m_raw[j];
        if (SOFTMAX) {
            float mx = -INFINITY;
#pragma unroll
            for (int j = 0; j < NT; ++j) mx = fmaxf(mx, m[j]);
#pragma unroll
            for (int o = IPW; o < 32; o <<= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
            float sum = 0.0f;
#pragma unroll
            for (int j = 0; j < NT; ++j) {
                m[j] = (k0 + j * LPI < K && valid_r) ? expf(m[j] - mx) : 0.0f;
                sum += m[j];
            }
#pragma unroll
            for (int o = IPW; o < 32; o <<= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
            const float inv = sum > 0.0f ? 1.0f / sum : 0.0f;
#pragma unroll
            for (int j = 0; j < NT; ++j) m[j] *= inv;
        }
        const float Hf = (float)a.H, Wf = (float)a.W;
#pragma unroll
        for (int j = 0; j < NT; ++j) {
            const int k = k0 + j * LPI;
            if (k >= K) continue;
            const int2 kt = ktab[k];
            const float pxf = fmaf(a.offset_scale, dx[j], (float)(wo * a.sw - a.pw + kt.y));
            const float pyf = fmaf(a.offset_scale, dy[j], (float)(ho * a.sh - a.ph + kt.x));
            const float fy = floorf(pyf), fx = floorf(pxf);
            const float ly = pyf - fy, lx = pxf - fx;  // NaN for a NaN position
            const bool nanp = (pxf != pxf) | (pyf != pyf);
            const bool inmap = (pyf >= -1.0f) & (pyf < Hf) & (pxf >= -1.0f) & (pxf < Wf);
            const int y0 = inmap ? (int)fy : -2, x0 = inmap ? (int)fx : -2;
            const bool vy0 = (unsigned)y0 < (unsigned)a.H, vy1 = (unsigned)(y0 + 1) < (unsigned)a.H;
            const bool vx0 = (unsigned)x0 < (unsigned)a.W, vx1 = (unsigned)(x0 + 1) < (unsigned)a.W;
            const int r00 = y0 * a.W + x0;
            int4 o4 = make_int4(vy0 & vx0 ? r00 : -1, vy0 & vx1 ? r00 + 1 : -1, vy1 & vx0 ? r00 + a.W : -1,
                                vy1 & vx1 ? r00 + a.W + 1 : -1);
            const float mk = m[j];
            const float tx0 = (1.0f - lx) * mk, tx1 = lx * mk;
            float4 w4 = make_float4(fmaf(-tx0, ly, tx0), fmaf(-tx1, ly, tx1), tx0 * ly, tx1 * ly);
            if (!(valid_r & (inmap | nanp))) w4 = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
            if (!valid_r) o4 = make_int4(-1, -1, -1, -1);
            rec_w[k * IPW + ri] = w4;  // a NaN position keeps NaN weights and zero-row corners
            rec_o[k * IPW + ri] = o4;
        }
        __syncwarp();
        // ---- gather
        const unsigned char *zrow = g_zero_row + q * 16;
#pragma unroll
        for (int k = 0; k < KMAX; ++k) {
            if (k >= K) break;
            const float4 w = rec_w[k * IPW + gi];
            const int4 o = rec_o[k * IPW + gi];
            const uint4 v0 = ld_nc16(o.x >= 0 ? (const void *)(xb + (long long)o.x * GC) : (const void *)zrow);
            const uint4 v1 = ld_nc16(o.y >= 0 ? (const void *)(xb + (long long)o.y * GC) : (const void *)zrow);
            const uint4 v2 = ld_nc16(o.z >= 0 ? (const void *)(xb + (long long)o.z * GC) : (const void *)zrow);
            const uint4 v3 = ld_nc16(o.w >= 0 ? (const void *)(xb + (long long)o.w * GC) : (const void *)zrow);
            float f[V];
            unpack16<T>(v0, f);
#pragma unroll
            for (int v = 0; v < V; ++v) acc[v] = fmaf(w.x, f[v], acc[v]);
            unpack16<T>(v1, f);
#pragma unroll
            for (int v = 0; v < V; ++v) acc[v] = fmaf(w.y, f[v], acc[v]);
            unpack16<T>(v2, f);
#pragma unroll
            for (int v = 0; v < V; ++v) acc[v] = fmaf(w.z, f[v], acc[v]);
            unpack16<T>(v3, f);
#pragma unroll
            for (int v = 0; v < V; ++v) acc[v] = fmaf(w.w, f[v], acc[v]);
        }
    } else if (valid) {
        // ---- every lane computes the taps of its item
        unsigned wo_u;
        const int ho = (int)fdiv(rem, p.fd_wo, wo_u), wo = (int)wo_u;
        const long long mi = (long long)pix * a.G + ip.g;
        const T *o_item = static_cast<const T *>(a.offset) + mi * K * 2;
        const T *m_item = static_cast<const T *>(a.mask) + mi * K;
        float mx = 0.0f, inv_sum = 1.0f;
        if (SOFTMAX) {
            mx = -INFINITY;
            for (int k = 0; k < K; ++k) mx = fmaxf(mx, load_scalar(m_item + k));
            float sum = 0.0f;
            for (int k = 0; k < K; ++k) sum += expf(load_scalar(m_item + k) - mx);
            inv_sum = 1.0f / sum;
        }
        bool nan_pos = false;
        // all K points summed (core + projection), or only this K-block's point
        // (deformable convolution: the points are contracted by the weight)
        const int k_lo = p.per_point ? ip.k : 0, k_hi = p.per_point ? ip.k + 1 : K;
        for (int k = k_lo; k < k_hi; ++k) {
            const int2 kt = ktab[k];
            const float2 d = load_pair(o_item + 2 * k);
            float m = load_scalar(m_item + k);
            if (SOFTMAX) m = expf(m - mx) * inv_sum;
            const float pxf = fmaf(a.offset_scale, d.x, (float)(wo * a.sw - a.pw + kt.y));
            const float pyf = fmaf(a.offset_scale, d.y, (float)(ho * a.sh - a.ph + kt.x));
            Tap tp{0, 0, 0.0f, 0.0f};
            const int st = make_tap(pyf, pxf, a.H, a.W, tp);
            nan_pos |= st < 0;
            uint4 raw[4];
            float w[4];
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                const int y = tp.y0 + (c >> 1), x = tp.x0 + (c & 1);
                const bool ok = st > 0 && (unsigned)y < (unsigned)a.H && (unsigned)x < (unsigned)a.W;
                w[c] = ok ? ((c >> 1) ? tp.ly : 1.0f - tp.ly) * ((c & 1) ? tp.lx : 1.0f - tp.lx) * m : 0.0f;
                raw[c] = ok ? ld_nc16(xb + ((long long)y * a.W + x) * GC) : make_uint4(0, 0, 0, 0);
            }
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                float f[V];
                unpack16<T>(raw[c], f);
#pragma unroll
                for (int v = 0; v < V; ++v) acc[v] = fmaf(w[c], f[v], acc[v]);
            }
        }
        if (nan_pos) {
#pragma unroll
            for (int v = 0; v < V; ++v) acc[v] = __int_as_float(0x7fc00000);
        }
    }
    if (valid) {
        // 16-byte chunk of row px inside its K-block's slot, swizzled
        unsigned char *slot = bring + ((ci * p.KB + ip.kb) % kBSlots) * slot_bytes;
        const int chunk = ((ip.g * a.C) & 63) / V + q;
        *reinterpret_cast<uint4 *>(slot + ip.px * 128 + ((chunk ^ (ip.px & 7)) << 4)) = pack16<T>(acc);
    }
    if (RECORDS) __syncwarp();  // records are rewritten by the next step
}

// Per-point records (deformable convolution: every item is one kernel point
// of one (pixel, group)).  A step is 32 consecutive items of the chunk's flat
// list.  Lane l first turns item base + l into a record: its four corner
// pixels (image-wide index, -1 outside the map), its four bilinear weights with
// the modulation folded in, and where its 16-byte chunks go in the B-operand
// slot.  Then the LPI lanes of each item gather its channel chunks, IPW items
// per round, LPI rounds, so every tap is computed once instead of once per lane.
template <typename T, int LPI, bool SOFTMAX>
__device__ __forceinline__ void gather_step_pp(const ProjParams &p, int ci, long long c0, FastDiv fd_npx, int total,
                                               int base, int lane, unsigned char *bring, int slot_bytes,
                                               float4 *rec_w, int4 *rec_o, int2 *rec_d, const int2 *ktab) {
    constexpr int V = Storage<T>::kVec;
    constexpr int IPW = 32 / LPI;
    const CoreArgs &a = p.a;
    const int K = a.kh * a.kw;
    const int GC = a.G * a.C;
    {
        // ---- record of item base + lane
        const int item = base + lane;
        const bool valid = item < total;
        const ItemPos ip = item_pos(valid ? item : 0, fd_npx, p);
        const unsigned pix = (unsigned)(c0 + ip.px);
        unsigned rem, wo_u;
        const unsigned b = fdiv(pix, p.fd_howo, rem);
        const int ho = (int)fdiv(rem, p.fd_wo, wo_u), wo = (int)wo_u;
        const long long mi = (long long)pix * a.G + ip.g;
        const T *m_item = static_cast<const T *>(a.mask) + mi * K;
        const float2 d = load_pair(static_cast<const T *>(a.offset) + (mi * K + ip.k) * 2);
        float mk = load_scalar(m_item + ip.k);
        if (SOFTMAX) {
            float mx = -INFINITY;
            for (int k = 0; k < K; ++k) mx = fmaxf(mx, load_scalar(m_item + k));
            float sum = 0.0f;
            for (int k = 0; k < K; ++k) sum += expf(load_scalar(m_item + k) - mx);
            mk = expf(mk - mx) * (1.0f / sum);
        }
        const int2 kt = ktab[ip.k];
        const float pxf = fmaf(a.offset_scale, d.x, (float)(wo * a.sw - a.pw + kt.y));
        const float pyf = fmaf(a.offset_scale, d.y, (float)(ho * a.sh - a.ph + kt.x));
        const float fy = floorf(pyf), fx = floorf(pxf);
        const float ly = pyf - fy, lx = pxf - fx;  // NaN for a NaN position
        const bool nanp = (pxf != pxf) | (pyf != pyf);
        const bool inmap = (pyf >= -1.0f) & (pyf < (float)a.H) & (pxf >= -1.0f) & (pxf < (float)a.W);
        const int y0 = inmap ? (int)fy : -2, x0 = inmap ? (int)fx : -2;
        const bool vy0 = (unsigned)y0 < (unsigned)a.H, vy1 = (unsigned)(y0 + 1) < (unsigned)a.H;
        const bool vx0 = (unsigned)x0 < (unsigned)a.W, vx1 = (unsigned)(x0 + 1) < (unsigned)a.W;
        const int r00 = ((int)b * a.H + y0) * a.W + x0;  // B*H*W < 2^31
        int4 o4 = make_int4(vy0 & vx0 ? r00 : -1, vy0 & vx1 ? r00 + 1 : -1, vy1 & vx0 ? r00 + a.W : -1,
                            vy1 & vx1 ? r00 + a.W + 1 : -1);
        const float tx0 = (1.0f - lx) * mk, tx1 = lx * mk;
        float4 w4 = make_float4(fmaf(-tx0, ly, tx0), fmaf(-tx1, ly, tx1), tx0 * ly, tx1 * ly);
        if (!(valid & (inmap | nanp))) w4 = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
        if (!valid) o4 = make_int4(-1, -1, -1, -1);
        rec_w[lane] = w4;  // a NaN position keeps NaN weights and zero-row corners
        rec_o[lane] = o4;
        // slot row of the item's K-block and the group's first channel (-1: no item)
        rec_d[lane] = make_int2(((ci * p.KB + ip.kb) % kBSlots) * slot_bytes + ip.px * 128, valid ? ip.g * a.C : -1);
    }
    __syncwarp();
    // ---- gather: lanes (gi, q) take the 16-byte chunk q of item r * IPW + gi
    const int gi = lane / LPI, q = lane % LPI;
    const T *__restrict__ xq = static_cast<const T *>(a.x) + q * V;
    const unsigned char *zrow = g_zero_row + q * 16;
#pragma unroll
    for (int r = 0; r < LPI; ++r) {
        const int idx = r * IPW + gi;
        const float4 w = rec_w[idx];
        const int4 o = rec_o[idx];
        const int2 dd = rec_d[idx];
        const T *xb = xq + (dd.y < 0 ? 0 : dd.y);
        const uint4 v0 = ld_nc16(o.x >= 0 ? (const void *)(xb + (long long)o.x * GC) : (const void *)zrow);
        const uint4 v1 = ld_nc16(o.y >= 0 ? (const void *)(xb + (long long)o.y * GC) : (const void *)zrow);
        const uint4 v2 = ld_nc16(o.z >= 0 ? (const void *)(xb + (long long)o.z * GC) : (const void *)zrow);
        const uint4 v3 = ld_nc16(o.w >= 0 ? (const void *)(xb + (long long)o.w * GC) : (const void *)zrow);
        float acc[V], f[V];
        unpack16<T>(v0, f);
#pragma unroll
        for (int v = 0; v < V; ++v) acc[v] = w.x * f[v];
        unpack16<T>(v1, f);
#pragma unroll
        for (int v = 0; v < V; ++v) acc[v] = fmaf(w.y, f[v], acc[v]);
        unpack16<T>(v2, f);
#pragma unroll
        for (int v = 0; v < V; ++v) acc[v] = fmaf(w.z, f[v], acc[v]);
        unpack16<T>(v3, f);
#pragma unroll
        for (int v = 0; v < V; ++v) acc[v] = fmaf(w.w, f[v], acc[v]);
        if (dd.y >= 0) {
            // 16-byte chunk of the item's slot row, swizzled (slot bytes are a multiple of 1024)
            const int chunk = (dd.y & 63) / V + q;
            *reinterpret_cast<uint4 *>(bring + dd.x + ((chunk ^ ((dd.x >> 7) & 7)) << 4)) = pack16<T>(acc);
        }
    }
    __syncwarp();  // records are rewritten by the next step
}

template <typename T, int LPI, bool SOFTMAX, int KMAX, bool RECORDS, bool PP>
__global__ void __launch_bounds__(kProjThreads, 1)
    core_forward_proj(const __grid_constant__ CUtensorMap wmap, const ProjParams p) {
    constexpr int IPW = 32 / LPI;
    const CoreArgs &a = p.a;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    extern __shared__ unsigned char smem_raw[];
    // 1024-byte aligned base (the swizzle pattern repeats every 1024 bytes):
    // [sample ring: kBSlots x npad_max x 128][weight ring: kWStages x 16 KB (32 KB swapped)]
    // [records: weights, corners][kernel-point table][barriers, tensor-memory address, abort flag]
    const uint32_t raw_a = smem_u32(smem_raw);
    unsigned char *smem = smem_raw + (((raw_a + 1023u) & ~1023u) - raw_a);
    const int slot_bytes = p.npad_max * 128;
    unsigned char *bring = smem;
    unsigned char *wst = bring + (size_t)kBSlots * slot_bytes;
    // Per-point records swap the roles: the sampled pixels are the M = 128 operand
    // and up to 256 output channels of the weight the N operand, so that each
    // weight tile feeds products of N = 256 (a 4-product tile costs a fixed few
    // hundred cycles of hand-over, which only products of N >= 128 cover).
    constexpr bool SWAP = PP;
    constexpr int WTILE = SWAP ? kWTileBytesSwap : kWTileBytes;
    unsigned char *rp = wst + kWStages * WTILE;
    // records per gather warp: one per (item, point) of a step, or one per item of a per-point step
    constexpr int RECS = PP ? 32 : (RECORDS ? KMAX * IPW : 0);
    const int wsel = warp < kGatherWarps ? warp : 0;
    float4 *rec_w = reinterpret_cast<float4 *>(rp) + wsel * RECS;
    int4 *rec_o = reinterpret_cast<int4 *>(rp + kGatherWarps * RECS * 16) + wsel * RECS;
    int2 *rec_d = reinterpret_cast<int2 *>(rp + kGatherWarps * RECS * 32) + wsel * RECS;
    rp += kGatherWarps * RECS * (PP ? 40 : 32);
    int2 *ktab = reinterpret_cast<int2 *>(rp);
    uint64_t *bars = reinterpret_cast<uint64_t *>(ktab + KMAX);
    constexpr int kBars = 2 * kWStages + 2 * kBSlots + 3;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + kBars);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);
    const uint32_t wfull = smem_u32(bars), wempty = wfull + 8 * kWStages;
    const uint32_t kready = wempty + 8 * kWStages, bfree = kready + 8 * kBSlots;
    const uint32_t dfull = bfree + 8 * kBSlots, tempty = dfull + 8, drain = dfull + 16;
    const uint32_t bring_a = smem_u32(bring), wst_a = smem_u32(wst);

    for (int k = threadIdx.x; k < a.kh * a.kw; k += blockDim.x)
        ktab[k] = make_int2((k / a.kw) * a.dh, (k % a.kw) * a.dw);
    if (threadIdx.x == 0) {
        for (int i = 0; i < kWStages; ++i) {
            mbar_init(wfull + 8 * i, 1);
            mbar_init(wempty + 8 * i, 1);
        }
        for (int i = 0; i < kBSlots; ++i) {
            mbar_init(kready + 8 * i, kGatherWarps);
            mbar_init(bfree + 8 * i, 1);
        }
        mbar_init(dfull, 1);
        mbar_init(tempty, kGatherWarps);
        mbar_init(drain, 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == kMmaWarp) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                     "r"(p.tmem_cols)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    const long long r0 = p.P * blockIdx.x / p.n_cta, r1 = p.P * (blockIdx.x + 1) / p.n_cta;
    const int n_chunks = (int)((r1 - r0 + kMaxChunk - 1) / kMaxChunk);

    if (warp == kProducerWarp) {
        // ---- weight tiles, in the order the MMA thread consumes them
        if (lane == 0) {
            int it = 0;
            uint32_t s = 0, pass = 0;  // stage of the next tile and how often the ring has wrapped
            const uint32_t tx = (uint32_t)p.w_box_rows * 128u;
            for (int ci = 0; ci < n_chunks && !*abort_flag; ++ci)
                for (int kb = 0; kb < p.KB && !*abort_flag; ++kb)
                    for (int mb = 0; mb < p.MB; ++mb, ++it) {
                        if (pass >= 1 && !wait_or_abort(wempty + 8 * s, (pass - 1) & 1, abort_flag)) {
                            raise_abort(abort_flag, p.err);
                            break;
                        }
                        mbar_arrive_expect_tx(wfull + 8 * s, tx);
                        tma_load_2d(wst_a + s * WTILE, &wmap, wfull + 8 * s, kb * 64, mb * (SWAP ? 256 : 128));
                        if (++s == kWStages) {
                            s = 0;
                            ++pass;
                        }
                    }
            // drain: the last load issued into each stage has landed
            for (int j = it - 1; j >= 0 && j >= it - kWStages; --j)
                mbar_wait_bounded(wfull + 8 * (j % kWStages), (j / kWStages) & 1, kProjWaitNs);
        }
        __syncwarp();
    } else if (warp == kMmaWarp) {
        // ---- tensor-core products, one thread
        if (lane == 0) {
            // One thread issues every product, so its own instruction latency paces
            // the tensor core: between products it only steps counters and adds
            // precomputed descriptor offsets (no division, no descriptor rebuild).
            uint32_t ws = 0, wph = 0;  // weight stage of the next tile, its phase parity
            uint32_t bsl = 0, bph = 0; // B slot of the next K-block, its phase parity
            // descriptors are linear in the address (start address >> 4 in the low field)
            const uint64_t adesc0 = smem_desc_sw128(wst_a), bdesc0 = smem_desc_sw128(bring_a);
            const uint32_t slot_step = (uint32_t)slot_bytes >> 4, stage_step = WTILE >> 4;
            bool issued = false;
            const int fmt = std::is_same<T, __nv_bfloat16>::value ? 1 : 0;
            for (int ci = 0; ci < n_chunks && !*abort_flag; ++ci) {
                long long c0, c1;
                chunk_range(r0, r1, ci, n_chunks, c0, c1);
                const int npad = ((int)(c1 - c0) + 15) & ~15;
                // swapped: N = 256 output channels per tile, the last tile the rest
                const int n_last = p.cout16 - 256 * (p.MB - 1);
                const uint32_t idesc = instr_desc_f16(fmt, SWAP ? (p.MB > 1 ? 256 : n_last) : npad);
                const uint32_t idesc_last = SWAP ? instr_desc_f16(fmt, n_last) : idesc;
                const uint32_t dstep = SWAP ? 256u : (uint32_t)npad;
                // the epilogue has read the previous chunk's accumulators
                if (ci > 0 && !wait_or_abort(tempty, (ci - 1) & 1, abort_flag)) {
                    raise_abort(abort_flag, p.err);
                    break;
                }
                tc_fence_after();
                bool ok = true;
                for (int kb = 0; kb < p.KB && ok; ++kb) {
                    if (!wait_or_abort(kready + 8 * bsl, bph, abort_flag)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint64_t bdesc = bdesc0 + bsl * slot_step;
                    uint32_t dcol = tmem;
                    for (int mb = 0; mb < p.MB; ++mb, dcol += dstep) {
                        if (!wait_or_abort(wfull + 8 * ws, wph, abort_flag)) {
                            ok = false;
                            break;
                        }
                        tc_fence_after();
                        // k-steps of 16 elements = 32 bytes = 2 descriptor units
                        const uint64_t wdesc = adesc0 + ws * stage_step;
                        if (SWAP) {  // D[pixel, channel] += samples . weight^T
                            const uint32_t id = mb + 1 < p.MB ? idesc : idesc_last;
                            mma_f16(dcol, bdesc, wdesc, id, kb != 0);
                            mma_f16(dcol, bdesc + 2, wdesc + 2, id, 1u);
                            mma_f16(dcol, bdesc + 4, wdesc + 4, id, 1u);
                            mma_f16(dcol, bdesc + 6, wdesc + 6, id, 1u);
                        } else {     // D[channel, pixel] += weight . samples^T
                            mma_f16(dcol, wdesc, bdesc, idesc, kb != 0);
                            mma_f16(dcol, wdesc + 2, bdesc + 2, idesc, 1u);
                            mma_f16(dcol, wdesc + 4, bdesc + 4, idesc, 1u);
                            mma_f16(dcol, wdesc + 6, bdesc + 6, idesc, 1u);
                        }
                        issued = true;
                        mma_commit(wempty + 8 * ws);  // weight stage free once these products are done
                        if (++ws == kWStages) {
                            ws = 0;
                            wph ^= 1u;
                        }
                    }
                    if (!ok) break;
                    mma_commit(bfree + 8 * bsl);  // B slot free once this K-block's products are done
                    if (++bsl == kBSlots) {
                        bsl = 0;
                        bph ^= 1u;
                    }
                }
                if (!ok) {
                    raise_abort(abort_flag, p.err);
                    break;
                }
                if (*abort_flag) break;
                mma_commit(dfull);  // accumulators of this chunk complete
            }
            if (issued && *abort_flag) {  // let the products already issued finish
                mma_commit(drain);
                mbar_wait_bounded(drain, 0, kProjWaitNs);
            }
        }
        __syncwarp();
    } else {
        // ---- gather warps: core samples into the B ring, then the epilogue
        constexpr int NT = (KMAX + LPI - 1) / LPI;
        const T *__restrict__ bias = static_cast<const T *>(p.bias);
        T *__restrict__ out = static_cast<T *>(a.out);
        const int ri = lane % IPW, k0 = lane / IPW;
        bool stop = false;
        for (int ci = 0; ci < n_chunks && !stop; ++ci) {
            long long c0, c1;
            chunk_range(r0, r1, ci, n_chunks, c0, c1);
            const int n_px = (int)(c1 - c0);
            const int npad = (n_px + 15) & ~15;
            const int per_kb = n_px << p.lg_gpb;
            const int total = per_kb * p.KB;
            const FastDiv fd_npx = make_fastdiv((unsigned)n_px), fd_pkb = make_fastdiv((unsigned)per_kb);
            unsigned fr;
            constexpr int SI = PP ? 32 : IPW;  // items per step
            const int n_steps = (total + SI - 1) / SI;
            int waited = -1;    // slots of K-blocks <= waited are known to be free
            int signaled = 0;   // K-blocks < signaled are handed to the tensor core by this warp
            // wait until the products that read K-block kb's slot before are done
            auto slot_free = [&](int kb) -> bool {
                while (waited < kb) {
                    ++waited;
                    const int t = ci * p.KB + waited, use = t / kBSlots;
                    if (use >= 1 && !wait_or_abort(bfree + 8 * (t % kBSlots), (use - 1) & 1, abort_flag)) {
                        if (lane == 0) raise_abort(abort_flag, p.err);
                        return false;
                    }
                }
                return true;
            };
            // hand K-blocks [signaled, upto) to the tensor core
            auto signal = [&](int upto) -> bool {
                if (upto <= signaled) return true;
                fence_proxy_async_smem();  // this thread's slot writes before the tensor core reads
                __syncwarp();
                for (; signaled < upto; ++signaled) {
                    // the slot's previous phase is complete before this warp arrives on it again
                    if (!slot_free(signaled)) return false;
                    if (lane == 0) mbar_arrive(kready + 8 * ((ci * p.KB + signaled) % kBSlots));
                }
                return true;
            };
            float dx[NT], dy[NT], m[NT];
            if (RECORDS) load_raw<T, LPI, SOFTMAX, NT>(p, c0, fd_npx, total, warp * IPW + ri, k0, dx, dy, m);
            for (int st = warp; st < n_steps; st += kGatherWarps) {
                const int first = st * SI;
                const int last = (first + SI < total ? first + SI : total) - 1;
                // K-blocks before this step's first one hold nothing more of this
                // warp: hand them over before waiting for any slot, so that every
                // wait below depends only on K-blocks this warp has already
                // handed over (a step spans at most four K-blocks, the ring size)
                if (!signal((int)fdiv((unsigned)first, fd_pkb, fr)) ||
                    !slot_free((int)fdiv((unsigned)last, fd_pkb, fr))) {
                    stop = true;
                    break;
                }
                float cdx[NT], cdy[NT], cm[NT];
#pragma unroll
                for (int j = 0; j < NT; ++j) {
                    cdx[j] = dx[j];
                    cdy[j] = dy[j];
                    cm[j] = m[j];
                }
                const int nxt = st + kGatherWarps;
                if (RECORDS && nxt < n_steps)
                    load_raw<T, LPI, SOFTMAX, NT>(p, c0, fd_npx, total, nxt * IPW + ri, k0, dx, dy, m);
                if constexpr (PP)
                    gather_step_pp<T, LPI, SOFTMAX>(p, ci, c0, fd_npx, total, first, lane, bring, slot_bytes, rec_w,
                                                    rec_o, rec_d, ktab);
                else
                    gather_step<T, LPI, SOFTMAX, KMAX, RECORDS, NT>(p, ci, c0, fd_npx, total, first, lane, bring,
                                                                     slot_bytes, rec_w, rec_o, ktab, cdx, cdy, cm);
                // every K-block before the one this warp's next step starts in is done
                if (!signal(nxt < n_steps ? (int)fdiv((unsigned)(nxt * SI), fd_pkb, fr) : p.KB)) {
                    stop = true;
                    break;
                }
            }
            if (!stop && !signal(p.KB)) stop = true;
            if (stop) break;
            // ---- epilogue: accumulators -> + bias -> storage type
            if (!wait_or_abort(dfull, ci & 1, abort_flag)) {
                if (lane == 0) raise_abort(abort_flag, p.err);
                break;
            }
            tc_fence_after();
            const int quad = warp & 3, part = warp >> 2;
            if (SWAP) {
                // tensor-memory lane = pixel of the chunk, column = output channel
                const int px = 32 * quad + lane;
                if (32 * quad < n_px) {
                    T *orow = out + (c0 + (px < n_px ? px : 0)) * p.Cout;
                    for (int cc = part; cc < p.cout16 / 16; cc += kGatherWarps / 4) {
                        float v[16];
                        tmem_ld16(tmem + ((uint32_t)(32 * quad) << 16) + (uint32_t)(cc * 16), v);
                        const int o0 = cc * 16;
                        if (px < n_px) {
#pragma unroll
                            for (int j = 0; j < 16; ++j)
                                if (o0 + j < p.Cout) v[j] += bias ? load_scalar(bias + o0 + j) : 0.0f;
                            if (o0 + 16 <= p.Cout) {  // rows are 16-byte aligned (Cout % 8 == 0)
                                uint4 *dst = reinterpret_cast<uint4 *>(orow + o0);
                                dst[0] = pack16<T>(v);
                                dst[1] = pack16<T>(v + 8);
                            } else {
#pragma unroll
                                for (int j = 0; j < 16; ++j)
                                    if (o0 + j < p.Cout) orow[o0 + j] = from_f32<T>(v[j]);
                            }
                        }
                    }
                }
            } else
            for (int blk = part; blk < npad / 16; blk += kGatherWarps / 4) {
                for (int mb = 0; mb < p.MB; ++mb) {
                    float v[16];
                    tmem_ld16(tmem + ((uint32_t)(32 * quad) << 16) + (uint32_t)(mb * npad + blk * 16), v);
                    const int o = mb * 128 + 32 * quad + lane;
                    if (o < p.Cout) {
                        const float bo = bias ? load_scalar(bias + o) : 0.0f;
#pragma unroll
                        for (int r = 0; r < 16; ++r) {
                            const int px = blk * 16 + r;
                            if (px < n_px) out[(c0 + px) * p.Cout + o] = from_f32<T>(v[r] + bo);
                        }
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(tempty);
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == kMmaWarp) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(p.tmem_cols)
                     : "memory");
    }
}

template <typename T, int LPI, bool SOFTMAX, int KMAX, bool RECORDS, bool PP = false>
cudaError_t launch_one(const CUtensorMap &map, const ProjParams &p, size_t smem, cudaStream_t stream) {
    auto kern = core_forward_proj<T, LPI, SOFTMAX, KMAX, RECORDS, PP>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    kern<<<p.n_cta, kProjThreads, smem, stream>>>(map, p);
    return cudaGetLastError();
}

// Shared memory of one instance: B ring + weight ring + records + table + barriers, plus alignment slack.
constexpr size_t proj_smem(int npad_max, int lpi, int kmax, bool records, bool pp = false) {
    return (size_t)kBSlots * npad_max * 128 + (size_t)kWStages * (pp ? kWTileBytesSwap : kWTileBytes) +
           (pp ? (size_t)kGatherWarps * 32 * 40 : records ? (size_t)kGatherWarps * kmax * (32 / lpi) * 32 : 0) +
           (size_t)kmax * 8 + 256 + 1024;
}

template <typename T, int LPI>
cudaError_t launch_lpi(const CUtensorMap &map, const ProjParams &p, size_t min_smem, cudaStream_t stream) {
    const int K = p.a.kh * p.a.kw;
    auto pick = [&](size_t need) { return need > min_smem ? need : min_smem; };
    if (p.per_point && p.pp_records) {
        // one tap per item, built once per item into a record
        const size_t smem = pick(proj_smem(p.npad_max, LPI, 25, false, true));
        return p.a.softmax ? launch_one<T, LPI, true, 25, false, true>(map, p, smem, stream)
                           : launch_one<T, LPI, false, 25, false, true>(map, p, smem, stream);
    }
    if (p.per_point) {
        // one tap per item: every lane computes its own
        const size_t smem = pick(proj_smem(p.npad_max, LPI, 25, false));
        return p.a.softmax ? launch_one<T, LPI, true, 25, false>(map, p, smem, stream)
                           : launch_one<T, LPI, false, 25, false>(map, p, smem, stream);
    }
    if (K <= 9) {
        // records for 2..8 lanes per item; a single-lane item computes its own taps
        constexpr bool R = LPI >= 2;
        const size_t smem = pick(proj_smem(p.npad_max, LPI, 9, R));
        return p.a.softmax ? launch_one<T, LPI, true, 9, R>(map, p, smem, stream)
                           : launch_one<T, LPI, false, 9, R>(map, p, smem, stream);
    }
    const size_t smem = pick(proj_smem(p.npad_max, LPI, 25, false));
    return p.a.softmax ? launch_one<T, LPI, true, 25, false>(map, p, smem, stream)
                       : launch_one<T, LPI, false, 25, false>(map, p, smem, stream);
}

template <typename T>
cudaError_t launch_t(const ProjArgs &pa, cudaStream_t stream) {
    const CoreArgs &a = pa.core;
    const DeviceInfo *dev = device_info();
    auto enc = encode_fn();
    if (!dev || !enc) return cudaErrorNotSupported;
    ProjParams p;
    p.a = a;
    p.bias = pa.bias;
    p.P = (long long)a.B * a.Ho * a.Wo;
    p.Cout = pa.Cout;
    p.MB = (pa.Cout + 127) / 128;
    const int K = a.kh * a.kw;
    p.per_point = pa.per_point ? 1 : 0;
    p.cbk = a.G * a.C / 64;
    p.KB = pa.per_point ? K * p.cbk : p.cbk;
    p.lg_gpb = 0;
    while ((a.C << p.lg_gpb) < 64) ++p.lg_gpb;
    p.fd_cbk = make_fastdiv((unsigned)p.cbk);
    p.fd_howo = make_fastdiv((unsigned)(a.Ho * a.Wo));
    p.fd_wo = make_fastdiv((unsigned)a.Wo);
    p.err = dev->err;
    long long n_cta = dev->sms;
    if (n_cta * 16 > p.P) n_cta = (p.P + 15) / 16;  // at least 16 pixels per CTA
    p.n_cta = (int)(n_cta < 1 ? 1 : n_cta);
    // every chunk holds at most min(range, 128) pixels, and no range exceeds
    // ceil(P / n_cta)
    const long long max_range = (p.P + p.n_cta - 1) / p.n_cta;
    // A per-point step of 32 items must span at most four K-blocks (the slot
    // ring): every chunk needs at least 11 items per K-block.  A chunk holds
    // min(range, 128) pixels when its range is at most 128, else at least 64;
    // every range holds at least floor(P / n_cta) pixels.
    const long long min_range = p.P / p.n_cta;
    const long long min_px = min_range > kMaxChunk ? 64 : min_range;
    p.pp_records = pa.per_point && (min_px << p.lg_gpb) >= 11 ? 1 : 0;
    p.cout16 = (pa.Cout + 15) & ~15;
    int cols = 32;
    if (p.pp_records) {
        // swapped products: 128 sample rows (M), output channels in tiles of 256 (N)
        p.npad_max = kMaxChunk;
        p.MB = (p.cout16 + 255) / 256;
        p.w_box_rows = p.cout16 < 256 ? p.cout16 : 256;
        while (cols < p.cout16) cols <<= 1;
    } else {
        p.npad_max = (int)(((max_range < kMaxChunk ? max_range : kMaxChunk) + 15) & ~15LL);
        p.w_box_rows = pa.Cout < 128 ? pa.Cout : 128;
        while (cols < p.MB * p.npad_max) cols <<= 1;
    }
    p.tmem_cols = cols;

    // at least half an SM's shared memory, so that one CTA owns the SM's
    // tensor memory (the largest instance needs about 200 KB)
    const size_t half_sm = (size_t)dev->smem_per_sm / 2 + 1024;
    if (proj_smem(p.npad_max, 2, 9, true) > (size_t)dev->smem_optin) return cudaErrorInvalidConfiguration;

    CUtensorMap map;
    // weight [Cout, G*C] (projection) or [Cout, K, G*C] (deformable convolution)
    const cuuint64_t dims[2] = {(cuuint64_t)(pa.per_point ? K : 1) * a.G * a.C, (cuuint64_t)pa.Cout};
    const cuuint64_t strides[1] = {dims[0] * 2};
    const cuuint32_t box[2] = {64, (cuuint32_t)p.w_box_rows};
    const cuuint32_t estr[2] = {1, 1};
    const CUresult r = enc(&map, CU_TENSOR_MAP_DATA_TYPE_UINT16, 2, const_cast<void *>(pa.weight), dims, strides, box,
                           estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                           CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return cudaErrorInvalidValue;
    switch (a.C * (int)sizeof(T) / 16) {
        case 1: return launch_lpi<T, 1>(map, p, half_sm, stream);
        case 2: return launch_lpi<T, 2>(map, p, half_sm, stream);
        case 4: return launch_lpi<T, 4>(map, p, half_sm, stream);
        case 8: return launch_lpi<T, 8>(map, p, half_sm, stream);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace

cudaError_t launch_core_forward_proj(const ProjArgs &pa, cudaStream_t stream) {
    switch (pa.core.dtype) {
        case DType::F16: return launch_t<__half>(pa, stream);
        case DType::BF16: return launch_t<__nv_bfloat16>(pa, stream);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace dcnb
