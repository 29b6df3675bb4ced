// Multi-camera multi-scale aggregation, anchor-wide kernels (Sparse4D
// deformable_aggregation article, sections 1, 2.1, 2.2 and 4).
//
// The sampling position of (anchor, point, camera, scale) does not depend on
// the group, so these kernels handle all G groups of a sample at once: the
// tap geometry (corner rows, bilinear weights) is computed once per
// sample instead of once per group, and each bilinear corner of all groups is
// one contiguous G*C row that the 32 lanes of a warp read as CPL coalesced
// 512-byte transactions (lane l, chunk j owns elements (32*j + l)*V ...).
// For 16-bit storage the forward runs one CTA per anchor: its warps split the
// anchor's (point, camera) pairs, each warp walks the scales of its pairs, and
// the warps' partial rows are summed through shared memory at the end.  The
// fp32 forward and the backward are persistent and pair-granular (below); the
// fp32 forward decodes each tap once per warp (agg_forward_coop_f32) where
// the shape allows, else once per lane (agg_forward_pairs_f32).  In
// the backward each pair belongs to exactly one warp, so the location
// gradient of a pair is reduced inside the warp and stored without atomics;
// the weight gradient of (sample, group) is reduced over the lanes of the
// group; the feature gradient is scattered with 16-byte vector reductions.
//
// Taken when G*C*sizeof(T) is 512, 1024 or 2048 bytes; other widths use the
// per-group kernels in deform_agg.cu.
#include "dcn_atomic.cuh"
#include "dcn_launch.h"

namespace dcnb {
namespace {

constexpr int kAggWarps = 8;        // warps per anchor CTA
constexpr int kAggTableMax = 512;   // (camera, scale) entries cached in shared memory

__device__ __forceinline__ int4 load_table(const AggArgs &a, int cs) {
    return make_int4(__ldg(a.spatial_shape + 2 * cs), __ldg(a.spatial_shape + 2 * cs + 1), __ldg(a.scale_start + cs), 0);
}

template <typename T, int CPL>
__global__ void __launch_bounds__(kAggWarps * 32) agg_forward_wide(AggArgs a) {
    constexpr int V = Storage<T>::kVec;
    constexpr int ROW = CPL * 32 * V;  // elements in one feature row (G*C)
    __shared__ int4 tab[kAggTableMax];
    __shared__ float part[kAggWarps][ROW];
    __shared__ int nan_any;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int CS = a.cams * a.scales;
    const bool tab_smem = CS <= kAggTableMax;
    if (tab_smem)
        for (int i = threadIdx.x; i < CS; i += blockDim.x) tab[i] = load_table(a, i);
    if (threadIdx.x == 0) nan_any = 0;
    __syncthreads();

    const long long ba = blockIdx.x;  // b * A + anchor
    const int b = (int)(ba / a.A);
    const T *__restrict__ feat = static_cast<const T *>(a.feat) + (long long)b * a.rows * ROW;
    const T *__restrict__ wts = static_cast<const T *>(a.weights);
    const int pairs = a.P * a.cams;
    int grp[CPL];
#pragma unroll
    for (int j = 0; j < CPL; ++j) grp[j] = (32 * j + lane) * V / a.C;
    float acc[CPL][V];
#pragma unroll
    for (int j = 0; j < CPL; ++j)
#pragma unroll
        for (int v = 0; v < V; ++v) acc[j][v] = 0.0f;
    bool nan_pos = false;

    for (int pc = warp; pc < pairs; pc += kAggWarps) {
        const int cam = pc % a.cams;
        const float2 uv = __ldg(reinterpret_cast<const float2 *>(a.loc) + ba * pairs + pc);
        const long long wbase = (ba * pairs + pc) * a.scales;
#pragma unroll 4
        for (int s = 0; s < a.scales; ++s) {
            const int4 t = tab_smem ? tab[cam * a.scales + s] : load_table(a, cam * a.scales + s);
            const float px = fmaf(uv.x, (float)t.y, -0.5f);
            const float py = fmaf(uv.y, (float)t.x, -0.5f);
            Tap tp{0, 0, 0.0f, 0.0f};
            const int st = make_tap(py, px, t.x, t.y, tp);
            if (st < 0) nan_pos = true;
            if (st <= 0) continue;
            float w[CPL];
#pragma unroll
            for (int j = 0; j < CPL; ++j) w[j] = load_scalar(wts + (wbase + s) * a.G + grp[j]);
            const float gyv[2] = {1.0f - tp.ly, tp.ly};
            const float gxv[2] = {1.0f - tp.lx, tp.lx};
#pragma unroll
            for (int cy = 0; cy < 2; ++cy) {
#pragma unroll
                for (int cx = 0; cx < 2; ++cx) {
                    const int y = tp.y0 + cy, x = tp.x0 + cx;
                    if (y < 0 || y >= t.x || x < 0 || x >= t.y) continue;
                    const long long row = (long long)t.z + (long long)y * t.y + x;
                    if (row < 0 || row >= a.rows) continue;
                    const float g = gyv[cy] * gxv[cx];
                    const T *r = feat + row * ROW + lane * V;
#pragma unroll
                    for (int j = 0; j < CPL; ++j) {
                        float f[V];
                        unpack16<T>(ld_nc16(r + 32 * j * V), f);
                        const float wg = w[j] * g;
#pragma unroll
                        for (int v = 0; v < V; ++v) acc[j][v] = fmaf(wg, f[v], acc[j][v]);
                    }
                }
            }
        }
    }
#pragma unroll
    for (int j = 0; j < CPL; ++j)
#pragma unroll
        for (int v = 0; v < V; ++v) part[warp][(32 * j + lane) * V + v] = acc[j][v];
    if (nan_pos) atomicOr(&nan_any, 1);
    __syncthreads();
    // sum the warps' partial rows; each thread produces 16-byte chunks
    T *__restrict__ out = static_cast<T *>(a.out) + ba * ROW;
    for (int c = threadIdx.x; c < ROW / V; c += blockDim.x) {
        float f[V];
#pragma unroll
        for (int v = 0; v < V; ++v) {
            float sum = 0.0f;
#pragma unroll
            for (int w = 0; w < kAggWarps; ++w) sum += part[w][c * V + v];
            f[v] = nan_any ? __int_as_float(0x7fc00000) : sum;
        }
        *reinterpret_cast<uint4 *>(out + c * V) = pack16<T>(f);
    }
}

// fp32 variant with pair-granular persistent work: warp w of the grid owns the
// contiguous range of (anchor, pair) units [U*w/NW, U*(w+1)/NW), so every warp
// gets the same number of samples whatever the anchor count.  Consecutive
// units of one anchor accumulate in registers; when the anchor changes the
// partial row is added to the (zeroed) output with 16-byte reductions, so an
// anchor split between two warps is summed in L2 (a few flushes per warp).
// The next unit's location is loaded one unit ahead, and the four corner
// loads of a sample are issued unconditionally (an out-of-map corner loads
// nothing and gets weight zero), so the unrolled scale loop keeps several
// samples' loads in flight.
template <int CPL>
__global__ void __launch_bounds__(kAggWarps * 32) agg_forward_pairs_f32(AggArgs a, long long units, int total_warps) {
    constexpr int V = 4;
    constexpr int ROW = CPL * 32 * V;
    __shared__ int4 tab[kAggTableMax];
    const int lane = threadIdx.x & 31;
    const int CS = a.cams * a.scales;
    const bool tab_smem = CS <= kAggTableMax;
    if (tab_smem)
        for (int i = threadIdx.x; i < CS; i += blockDim.x) tab[i] = load_table(a, i);
    __syncthreads();

    const int gw = blockIdx.x * kAggWarps + (threadIdx.x >> 5);
    const long long u0 = units * gw / total_warps, u1 = units * (gw + 1) / total_warps;
    if (u0 >= u1) return;
    const int pairs = a.P * a.cams;
    const float *__restrict__ wts = static_cast<const float *>(a.weights);
    float *__restrict__ out = static_cast<float *>(a.out);
    int grp[CPL];
#pragma unroll
    for (int j = 0; j < CPL; ++j) grp[j] = (32 * j + lane) * V / a.C;
    float acc[CPL][V];
#pragma unroll
    for (int j = 0; j < CPL; ++j)
#pragma unroll
        for (int v = 0; v < V; ++v) acc[j][v] = 0.0f;
    bool nan_pos = false;

    const float2 *locp = reinterpret_cast<const float2 *>(a.loc);
    float2 uv_next = __ldg(locp + u0);  // unit index == (b*A + anchor)*pairs + pair
    // (anchor, pair, camera) of the current unit, advanced incrementally
    long long ba = u0 / pairs;
    int pc = (int)(u0 - ba * pairs);
    int cam = pc % a.cams;
    int anchor = (int)(ba % a.A);
    const float *feat = static_cast<const float *>(a.feat) + (ba / a.A) * a.rows * ROW;
    bool dirty = false;  // acc holds contributions not yet added to the output
    auto flush = [&]() {
        float *o = out + ba * ROW + lane * V;
#pragma unroll
        for (int j = 0; j < CPL; ++j) {
            if (nan_pos) {
#pragma unroll
                for (int v = 0; v < V; ++v) acc[j][v] = __int_as_float(0x7fc00000);
            }
            red_add16<float>(o + 32 * j * V, acc[j]);
#pragma unroll
            for (int v = 0; v < V; ++v) acc[j][v] = 0.0f;
        }
        nan_pos = false;
        dirty = false;
    };
    for (long long u = u0; u < u1; ++u) {
        const float2 uv = uv_next;
        if (u + 1 < u1) uv_next = __ldg(locp + u + 1);
        const long long wbase = u * a.scales;
        dirty = true;
#pragma unroll 4
        for (int s = 0; s < a.scales; ++s) {
            const int4 t = tab_smem ? tab[cam * a.scales + s] : load_table(a, cam * a.scales + s);
            const float px = fmaf(uv.x, (float)t.y, -0.5f);
            const float py = fmaf(uv.y, (float)t.x, -0.5f);
            Tap tp{0, 0, 0.0f, 0.0f};
            const int st = make_tap(py, px, t.x, t.y, tp);
            nan_pos |= st < 0;
            float w[CPL];
#pragma unroll
            for (int j = 0; j < CPL; ++j) w[j] = __ldg(wts + (wbase + s) * a.G + grp[j]);
            float g[4];
            float4 f[4][CPL];
            const long long row00 = (long long)t.z + (long long)tp.y0 * t.y + tp.x0;
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                const int y = tp.y0 + (c >> 1), x = tp.x0 + (c & 1);
                const long long row = row00 + (c >> 1) * t.y + (c & 1);
                const bool ok = st > 0 && (unsigned)y < (unsigned)t.x && (unsigned)x < (unsigned)t.y &&
                                (unsigned long long)row < (unsigned long long)a.rows;
                g[c] = ok ? ((c >> 1) ? tp.ly : 1.0f - tp.ly) * ((c & 1) ? tp.lx : 1.0f - tp.lx) : 0.0f;
                const float *r = feat + (ok ? row : 0) * ROW + lane * V;
#pragma unroll
                for (int j = 0; j < CPL; ++j) {
                    f[c][j] = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
                    if (ok) f[c][j] = __ldg(reinterpret_cast<const float4 *>(r + 32 * j * V));
                }
            }
#pragma unroll
            for (int c = 0; c < 4; ++c)
#pragma unroll
                for (int j = 0; j < CPL; ++j) {
                    const float wg = w[j] * g[c];
                    acc[j][0] = fmaf(wg, f[c][j].x, acc[j][0]);
                    acc[j][1] = fmaf(wg, f[c][j].y, acc[j][1]);
                    acc[j][2] = fmaf(wg, f[c][j].z, acc[j][2]);
                    acc[j][3] = fmaf(wg, f[c][j].w, acc[j][3]);
                }
        }
        // next unit: next pair of this anchor, or the first pair of the next one
        if (++cam == a.cams) cam = 0;
        if (++pc == pairs) {
            flush();
            pc = 0;
            ++ba;
            if (++anchor == a.A) {
                anchor = 0;
                feat += (long long)a.rows * ROW;
            }
        }
    }
    if (dirty) flush();
}

// fp32 forward with the tap decode shared by the warp.  Warp w takes units
// [U*w/NW, U*(w+1)/NW) (unit = (b*A + anchor)*P*cams + point*cams + camera,
// so consecutive units mostly share an anchor).  The (unit, scale) taps of a
// batch of 32 / S units are decoded one per lane (location, table entry,
// floor, the four corner rows and their bilinear weights); the lanes then walk
// the batch's taps together, taking each tap's rows and weights by shuffle,
// so the decode runs once per tap instead of once per lane.  Each unit's
// scales are unrolled so that their corner loads are in flight together.  The
// partial row of an anchor is added to the zeroed output when the next unit
// belongs to another anchor.
// A lane holds VW consecutive channels per load: VW = 8 (one 32-byte load,
// sm_100's ld.global.v8.f32) where the group width C allows it, else 4.
// Needs S <= 32, fewer than 2^31 units and B*num_rows < 2^31.
__device__ __forceinline__ void ldg_v(const float *p, float (&v)[8]) {
    asm volatile("ld.global.nc.v8.f32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
                 : "=f"(v[0]), "=f"(v[1]), "=f"(v[2]), "=f"(v[3]), "=f"(v[4]), "=f"(v[5]), "=f"(v[6]), "=f"(v[7])
                 : "l"(p));
}
__device__ __forceinline__ void ldg_v(const float *p, float (&v)[4]) {
    const float4 t = __ldg(reinterpret_cast<const float4 *>(p));
    v[0] = t.x; v[1] = t.y; v[2] = t.z; v[3] = t.w;
}

template <int CPL, int VW>
__global__ void __launch_bounds__(kAggWarps * 32) agg_forward_coop_f32(AggArgs a, long long units, int total_warps) {
    constexpr int V = VW;                  // channels per lane and load
    constexpr int NL = CPL * 4 / VW;       // loads per lane and corner row
    constexpr int ROW = CPL * 32 * 4;      // channels of a row
    __shared__ int4 tab[kAggTableMax];
    const int lane = threadIdx.x & 31;
    const int warp = threadIdx.x >> 5;
    const int S = a.scales;
    const int CS = a.cams * S;
    const bool tab_smem = CS <= kAggTableMax;
    if (tab_smem)
        for (int i = threadIdx.x; i < CS; i += blockDim.x) tab[i] = load_table(a, i);
    __syncthreads();

    const int NB = 32 / S;                              // units per batch
    const int my_bu = lane / S, my_s = lane - my_bu * S;  // this lane's tap of a batch
    const int gw = blockIdx.x * kAggWarps + warp;
    const long long p0 = units * gw / total_warps, p1 = units * (gw + 1) / total_warps;
    const int pairs = a.P * a.cams;
    const float *__restrict__ wts = static_cast<const float *>(a.weights);
    const float *__restrict__ feat = static_cast<const float *>(a.feat);
    const float2 *__restrict__ locp = reinterpret_cast<const float2 *>(a.loc);
    float *__restrict__ out = static_cast<float *>(a.out);
    int grp[NL];
#pragma unroll
    for (int j = 0; j < NL; ++j) grp[j] = (32 * j + lane) * V / a.C;
    float acc[NL][V];
#pragma unroll
    for (int j = 0; j < NL; ++j)
#pragma unroll
        for (int v = 0; v < V; ++v) acc[j][v] = 0.0f;
    bool nan_acc = false;
    int cur_ba = -1;  // anchor (b*A + a) whose partial row acc holds

    for (long long pb = p0; pb < p1; pb += NB) {
        const int nb = (int)min((long long)NB, p1 - pb);
        // ---- decode: lane = (unit my_bu, scale my_s) of this batch
        const bool tv = my_bu < nb;
        int uid = 0;
        if (tv) uid = (int)(pb + my_bu);
        const int ba = uid / pairs;
        const int cam = (uid - ba * pairs) % a.cams;
        const int b = ba / a.A;
        const float2 uv = tv ? __ldg(locp + uid) : make_float2(0.0f, 0.0f);
        const int4 t = tab_smem ? tab[cam * S + my_s] : load_table(a, cam * S + my_s);
        Tap tp{0, 0, 0.0f, 0.0f};
        int st = make_tap(fmaf(uv.y, (float)t.x, -0.5f), fmaf(uv.x, (float)t.y, -0.5f), t.x, t.y, tp);
        if (!tv) st = 0;
        const unsigned nanm = __ballot_sync(0xffffffffu, st < 0);
        int rw[4];
        float gw4[4];
        const long long row00 = (long long)t.z + (long long)tp.y0 * t.y + tp.x0;
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            const int y = tp.y0 + (c >> 1), x = tp.x0 + (c & 1);
            const long long row = row00 + (c >> 1) * t.y + (c & 1);
            const bool ok = st > 0 && (unsigned)y < (unsigned)t.x && (unsigned)x < (unsigned)t.y &&
                            (unsigned long long)row < (unsigned long long)a.rows;
            rw[c] = ok ? (int)((long long)b * a.rows + row) : -1;
            gw4[c] = ok ? ((c >> 1) ? tp.ly : 1.0f - tp.ly) * ((c & 1) ? tp.lx : 1.0f - tp.lx) : 0.0f;
        }
        // ---- sample: every lane, every tap of the batch
        for (int bu = 0; bu < nb; ++bu) {
            const int kb = bu * S;
            const int ba_k = __shfl_sync(0xffffffffu, ba, kb);
            const int uid_k = __shfl_sync(0xffffffffu, uid, kb);
            if (ba_k != cur_ba) {
                if (cur_ba >= 0) {
                    float *o = out + (long long)cur_ba * ROW + lane * V;
#pragma unroll
                    for (int j = 0; j < NL; ++j) {
                        if (nan_acc) {
#pragma unroll
                            for (int v = 0; v < V; ++v) acc[j][v] = __int_as_float(0x7fc00000);
                        }
#pragma unroll
                        for (int h = 0; h < V; h += 4) red_add16<float>(o + 32 * j * V + h, acc[j] + h);
#pragma unroll
                        for (int v = 0; v < V; ++v) acc[j][v] = 0.0f;
                    }
                    nan_acc = false;
                }
                cur_ba = ba_k;
            }
            const unsigned um = S == 32 ? 0xffffffffu : ((1u << S) - 1u) << kb;
            nan_acc |= (nanm & um) != 0;
            const float *wu = wts + (long long)uid_k * S * a.G;
#pragma unroll 4
            for (int s = 0; s < S; ++s) {
                const int k = kb + s;
                float w[NL];
#pragma unroll
                for (int j = 0; j < NL; ++j) w[j] = __ldg(wu + s * a.G + grp[j]);
                float g[4];
                float f[4][NL][V];
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    const int r = __shfl_sync(0xffffffffu, rw[c], k);
                    g[c] = __shfl_sync(0xffffffffu, gw4[c], k);
                    const float *src = feat + (long long)(r < 0 ? 0 : r) * ROW + lane * V;
#pragma unroll
                    for (int j = 0; j < NL; ++j) {
#pragma unroll
                        for (int v = 0; v < V; ++v) f[c][j][v] = 0.0f;
                        if (r >= 0) ldg_v(src + 32 * j * V, f[c][j]);
                    }
                }
#pragma unroll
                for (int c = 0; c < 4; ++c)
#pragma unroll
                    for (int j = 0; j < NL; ++j) {
                        const float wg = w[j] * g[c];
#pragma unroll
                        for (int v = 0; v < V; ++v) acc[j][v] = fmaf(wg, f[c][j][v], acc[j][v]);
                    }
            }
        }
    }
    if (cur_ba >= 0) {
        float *o = out + (long long)cur_ba * ROW + lane * V;
#pragma unroll
        for (int j = 0; j < NL; ++j) {
            if (nan_acc) {
#pragma unroll
                for (int v = 0; v < V; ++v) acc[j][v] = __int_as_float(0x7fc00000);
            }
#pragma unroll
            for (int h = 0; h < V; h += 4) red_add16<float>(o + 32 * j * V + h, acc[j] + h);
        }
    }
}

// Backward with pair-granular persistent work (every storage type): warp w
// of the grid owns the contiguous (anchor, pair) units [U*w/NW, U*(w+1)/NW),
// so every warp has the same number of samples whatever the anchor count.
// A unit belongs to exactly one warp, so its location gradient is stored
// without atomics; the grad_out row is reloaded when the anchor changes.
// Per sample the four corner rows are loaded first (out-of-map corners load
// nothing and get weight zero), then the dot products and the 16-byte vector
// reductions into grad_feat follow.
template <typename T, int CPL>
__global__ void __launch_bounds__(kAggWarps * 32) agg_backward_pairs(AggArgs a, long long units, int total_warps) {
    constexpr int V = Storage<T>::kVec;
    constexpr int ROW = CPL * 32 * V;
    __shared__ int4 tab[kAggTableMax];
    const int lane = threadIdx.x & 31;
    const int CS = a.cams * a.scales;
    const bool tab_smem = CS <= kAggTableMax;
    if (tab_smem)
        for (int i = threadIdx.x; i < CS; i += blockDim.x) tab[i] = load_table(a, i);
    __syncthreads();

    const int gw_idx = blockIdx.x * kAggWarps + (threadIdx.x >> 5);
    const long long u0 = units * gw_idx / total_warps, u1 = units * (gw_idx + 1) / total_warps;
    if (u0 >= u1) return;
    const int pairs = a.P * a.cams;
    const T *__restrict__ wts = static_cast<const T *>(a.weights);
    T *__restrict__ gw = static_cast<T *>(a.grad_weights);
    const int gl = a.C / V;  // lanes of one group inside a chunk (a power of two)
    int grp[CPL];
#pragma unroll
    for (int j = 0; j < CPL; ++j) grp[j] = (32 * j + lane) * V / a.C;

    long long ba = u0 / pairs;
    int pc = (int)(u0 - ba * pairs);
    int cam = pc % a.cams;
    int anchor = (int)(ba % a.A);
    long long fofs = (ba / a.A) * a.rows * ROW;
    float go[CPL][V];
    auto load_go = [&]() {
        const T *gout = static_cast<const T *>(a.grad_out) + ba * ROW;
#pragma unroll
        for (int j = 0; j < CPL; ++j) unpack16<T>(ld_nc16(gout + (32 * j + lane) * V), go[j]);
    };
    load_go();
    for (long long u = u0; u < u1; ++u) {
        const T *__restrict__ feat = static_cast<const T *>(a.feat) + fofs;
        T *__restrict__ gfeat = static_cast<T *>(a.grad_feat) + fofs;
        const float2 uv = __ldg(reinterpret_cast<const float2 *>(a.loc) + u);
        const long long wbase = u * a.scales;
        float glx = 0.0f, gly = 0.0f;
        bool nan_pos = false;
        for (int s = 0; s < a.scales; ++s) {
            const int4 t = tab_smem ? tab[cam * a.scales + s] : load_table(a, cam * a.scales + s);
            const float px = fmaf(uv.x, (float)t.y, -0.5f);
            const float py = fmaf(uv.y, (float)t.x, -0.5f);
            Tap tp{0, 0, 0.0f, 0.0f};
            const int st = make_tap(py, px, t.x, t.y, tp);
            nan_pos |= st < 0;
            float w[CPL];
#pragma unroll
            for (int j = 0; j < CPL; ++j) w[j] = load_scalar(wts + (wbase + s) * a.G + grp[j]);
            const float gyv[2] = {1.0f - tp.ly, tp.ly};
            const float gxv[2] = {1.0f - tp.lx, tp.lx};
            const long long row00 = (long long)t.z + (long long)tp.y0 * t.y + tp.x0;
            bool ok[4];
            long long e0[4];
            uint4 raw[4][CPL];
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                const int y = tp.y0 + (c >> 1), x = tp.x0 + (c & 1);
                const long long row = row00 + (c >> 1) * t.y + (c & 1);
                ok[c] = st > 0 && (unsigned)y < (unsigned)t.x && (unsigned)x < (unsigned)t.y &&
                        (unsigned long long)row < (unsigned long long)a.rows;
                e0[c] = (ok[c] ? row : 0) * ROW + lane * V;
#pragma unroll
                for (int j = 0; j < CPL; ++j) {
                    raw[c][j] = make_uint4(0, 0, 0, 0);
                    if (ok[c]) raw[c][j] = ld_nc16(feat + e0[c] + 32 * j * V);
                }
            }
            float val[CPL], dpx[CPL], dpy[CPL];
#pragma unroll
            for (int j = 0; j < CPL; ++j) val[j] = dpx[j] = dpy[j] = 0.0f;
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                const int cy = c >> 1, cx = c & 1;
                const float G = ok[c] ? gyv[cy] * gxv[cx] : 0.0f;
                const float sx = ok[c] ? (cx ? gyv[cy] : -gyv[cy]) : 0.0f;
                const float sy = ok[c] ? (cy ? gxv[cx] : -gxv[cx]) : 0.0f;
#pragma unroll
                for (int j = 0; j < CPL; ++j) {
                    float f[V];
                    unpack16<T>(raw[c][j], f);
                    float dc = 0.0f;
#pragma unroll
                    for (int v = 0; v < V; ++v) dc = fmaf(go[j][v], f[v], dc);
                    val[j] = fmaf(G, dc, val[j]);
                    dpx[j] = fmaf(sx, dc, dpx[j]);
                    dpy[j] = fmaf(sy, dc, dpy[j]);
                    if (ok[c]) {
                        const float wg = w[j] * G;
                        float cv[V];
#pragma unroll
                        for (int v = 0; v < V; ++v) cv[v] = wg * go[j][v];
                        red_add16<T>(gfeat + e0[c] + 32 * j * V, cv);
                    }
                }
            }
            // weight gradient of (sample, group): sum over the group's lanes
#pragma unroll
            for (int j = 0; j < CPL; ++j) {
                float v = val[j];
                for (int o = 1; o < gl; o <<= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
                if (st < 0) v = __int_as_float(0x7fc00000);
                if ((lane & (gl - 1)) == 0) gw[(wbase + s) * a.G + grp[j]] = from_f32<T>(v);
                glx = fmaf(w[j] * (float)t.y, dpx[j], glx);
                gly = fmaf(w[j] * (float)t.x, dpy[j], gly);
            }
        }
        // location gradient of the pair: all groups and scales, one warp
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            glx += __shfl_xor_sync(0xffffffffu, glx, o);
            gly += __shfl_xor_sync(0xffffffffu, gly, o);
        }
        nan_pos = __any_sync(0xffffffffu, nan_pos);
        if (lane == 0) {
            const float nan = __int_as_float(0x7fc00000);
            reinterpret_cast<float2 *>(a.grad_loc)[u] = nan_pos ? make_float2(nan, nan) : make_float2(glx, gly);
        }
        // next unit
        if (++cam == a.cams) cam = 0;
        if (++pc == pairs) {
            pc = 0;
            ++ba;
            if (++anchor == a.A) {
                anchor = 0;
                fofs += (long long)a.rows * ROW;
            }
            if (u + 1 < u1) load_go();
        }
    }
}

// Shapes the warp-shared tap decode takes: one tap per lane needs S <= 32;
// unit and row indices travel as int32.
bool coop_fits(const AggArgs &a) {
    return a.scales <= 32 && (long long)a.B * a.A * a.P * a.cams <= 0x7fffffffLL &&
           (long long)a.B * a.rows <= 0x7fffffffLL;
}

template <int CPL, int VW>
cudaError_t launch_coop_k(const AggArgs &a, cudaStream_t stream) {
    int dev = 0, sms = 148, per_sm = 1;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, agg_forward_coop_f32<CPL, VW>, kAggWarps * 32, 0);
    if (per_sm < 1) per_sm = 1;
    const long long units = (long long)a.B * a.A * a.P * a.cams;
    long long ctas = (long long)sms * per_sm;
    if (ctas * kAggWarps > units) ctas = (units + kAggWarps - 1) / kAggWarps;
    cudaError_t e = cudaMemsetAsync(a.out, 0, (size_t)a.B * a.A * a.G * a.C * sizeof(float), stream);
    if (e != cudaSuccess) return e;
    agg_forward_coop_f32<CPL, VW><<<(unsigned)ctas, kAggWarps * 32, 0, stream>>>(a, units, (int)(ctas * kAggWarps));
    return cudaGetLastError();
}

template <int CPL>
cudaError_t launch_coop(const AggArgs &a, cudaStream_t stream) {
    // 32-byte loads need 8 channels of one group per lane and a 32-byte aligned
    // feat (the ABI guarantees 16; rows are multiples of 32 bytes)
    constexpr int VW8 = CPL % 2 == 0 ? 8 : 4;
    if (CPL % 2 == 0 && a.C % 8 == 0 && (reinterpret_cast<uintptr_t>(a.feat) & 31) == 0)
        return launch_coop_k<CPL, VW8>(a, stream);
    return launch_coop_k<CPL, 4>(a, stream);
}

template <typename T, int CPL>
cudaError_t launch(const AggArgs &a, bool bwd, cudaStream_t stream) {
    const unsigned grid = (unsigned)((long long)a.B * a.A);
    if (bwd) {
        cudaError_t e = cudaMemsetAsync(a.grad_feat, 0, (size_t)a.B * a.rows * a.G * a.C * sizeof(T), stream);
        if (e != cudaSuccess) return e;
        int dev = 0, sms = 148, per_sm = 1;
        cudaGetDevice(&dev);
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
        cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, agg_backward_pairs<T, CPL>, kAggWarps * 32, 0);
        if (per_sm < 1) per_sm = 1;
        const long long units = (long long)a.B * a.A * a.P * a.cams;
        long long ctas = (long long)sms * per_sm;
        if (ctas * kAggWarps > units) ctas = (units + kAggWarps - 1) / kAggWarps;
        agg_backward_pairs<T, CPL><<<(unsigned)ctas, kAggWarps * 32, 0, stream>>>(a, units, (int)(ctas * kAggWarps));
    } else if (sizeof(T) == 4 && coop_fits(a)) {
        return launch_coop<CPL>(a, stream);
    } else if (sizeof(T) == 4) {
        // fp32 output: pair-granular persistent warps, partial rows added in L2
        int dev = 0, sms = 148, per_sm = 1;
        cudaGetDevice(&dev);
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
        cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, agg_forward_pairs_f32<CPL>, kAggWarps * 32, 0);
        if (per_sm < 1) per_sm = 1;
        const long long units = (long long)a.B * a.A * a.P * a.cams;
        long long ctas = (long long)sms * per_sm;
        if (ctas * kAggWarps > units) ctas = (units + kAggWarps - 1) / kAggWarps;
        cudaError_t e = cudaMemsetAsync(a.out, 0, (size_t)a.B * a.A * a.G * a.C * sizeof(float), stream);
        if (e != cudaSuccess) return e;
        agg_forward_pairs_f32<CPL><<<(unsigned)ctas, kAggWarps * 32, 0, stream>>>(a, units, (int)(ctas * kAggWarps));
    } else {
        agg_forward_wide<T, CPL><<<grid, kAggWarps * 32, 0, stream>>>(a);
    }
    return cudaGetLastError();
}

template <typename T>
cudaError_t launch_t(const AggArgs &a, bool bwd, cudaStream_t stream, bool *handled) {
    const long long row_bytes = (long long)a.G * a.C * sizeof(T);
    if ((long long)a.B * a.A > 0x7fffffffLL) return cudaSuccess;
    *handled = true;
    switch (row_bytes) {
        case 512: return launch<T, 1>(a, bwd, stream);
        case 1024: return launch<T, 2>(a, bwd, stream);
        case 2048: return launch<T, 4>(a, bwd, stream);
    }
    *handled = false;
    return cudaSuccess;
}

}  // namespace

cudaError_t launch_agg_wide(const AggArgs &a, bool bwd, cudaStream_t stream, bool *handled) {
    *handled = false;
    switch (a.dtype) {
        case DType::F32: return launch_t<float>(a, bwd, stream, handled);
        case DType::F16: return launch_t<__half>(a, bwd, stream, handled);
        case DType::BF16: return launch_t<__nv_bfloat16>(a, bwd, stream, handled);
    }
    return cudaSuccess;
}

}  // namespace dcnb
