// Forward core fused with the pointwise projection that follows it in the
// DCNv4 module (YOLOv11 + DCNv4 article, section 3.2: the core's output goes
// through a 1x1 convolution with bias):
//     out[p, o] = bias[o] + sum_j Wt[o, j] * core[p, j],  j = g*C + c.
// The core tile never leaves the SM.
//
// Work split.  The B*Ho*Wo pixels are cut into one contiguous range per CTA
// (persistent grid, one CTA per SM), processed in chunks of at most 128
// pixels.  Per chunk:
//   1. Sixteen gather warps sample the core for every (pixel, group) of the
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
#include "dcn_tma.cuh"

namespace dcnb {
namespace {

constexpr int kGatherWarps = 16;
constexpr int kProducerWarp = kGatherWarps;
constexpr int kMmaWarp = kGatherWarps + 1;
constexpr int kProjThreads = (kGatherWarps + 2) * 32;
constexpr int kWStages = 4;
constexpr int kWTileBytes = 128 * 128;  // 128 rows x 64 elements x 2 bytes
constexpr int kMaxChunk = 128;          // pixels per chunk (MMA N <= 128)
constexpr int kMaxKBlocks = 8;          // G*C <= 512
constexpr uint64_t kProjWaitNs = 1000000000ull;

struct ProjParams {
    CoreArgs a;
    const void *bias;   // [Cout] storage type, or nullptr
    long long P;        // output pixels B*Ho*Wo
    int Cout;
    int MB;             // ceil(Cout / 128) output-channel blocks
    int KB;             // G*C / 64 channel blocks
    int n_cta;
    int npad_max;       // largest padded chunk of any CTA (B operand rows)
    int tmem_cols;      // allocated tensor-memory columns (power of two >= 32)
    int w_box_rows;     // rows per weight TMA box (min(Cout, 128))
    unsigned int *err;
};

// ---- tcgen05 / TMA helpers ----------------------------------------------------

__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap *map, uint32_t bar, int c0, int c1) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];" ::"r"(
            dst),
        "l"(map), "r"(c0), "r"(c1), "r"(bar)
        : "memory");
}

__device__ __forceinline__ void tc_fence_before() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// Shared-memory matrix descriptor: K-major operand in the 128-byte swizzle
// layout, 8-row groups 1024 bytes apart (the leading-byte offset is unused
// for this layout), descriptor version 1.
__device__ __forceinline__ uint64_t smem_desc_sw128(uint32_t addr) {
    uint64_t d = (uint64_t)((addr & 0x3FFFFu) >> 4);
    d |= (uint64_t)1 << 16;           // leading byte offset (16 bytes, ignored here)
    d |= (uint64_t)(1024 >> 4) << 32; // stride byte offset
    d |= (uint64_t)1 << 46;           // version
    d |= (uint64_t)2 << 61;           // 128-byte swizzle
    return d;
}

// Instruction descriptor of kind::f16: fp32 accumulator, A and B both fp16
// (fmt 0) or both bf16 (fmt 1), both K-major, M = 128, N = n.
__device__ __forceinline__ uint32_t instr_desc_f16(int fmt, int n) {
    return (1u << 4) | ((uint32_t)fmt << 7) | ((uint32_t)fmt << 10) | ((uint32_t)(n >> 3) << 17) |
           ((uint32_t)(128 >> 4) << 24);
}

__device__ __forceinline__ void mma_f16(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                        uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// Arrive on `bar` once every tcgen05.mma this thread issued so far is complete.
__device__ __forceinline__ void mma_commit(uint32_t bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
                 : "memory");
}

__device__ __forceinline__ void tmem_ld16(uint32_t taddr, float *v) {
    uint32_t r[16];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
    for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
}

// Bounded wait that also gives up as soon as another role has aborted.
__device__ __forceinline__ bool wait_or_abort(uint32_t bar, uint32_t parity, volatile int *abort_flag) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = global_timer_ns();
    while (true) {
        if (mbar_try_wait(bar, parity)) return true;
        if (*abort_flag) return false;
        if (global_timer_ns() - t0 > kProjWaitNs) return false;
        __nanosleep(64);
    }
}

__device__ __forceinline__ void raise_abort(volatile int *abort_flag, unsigned int *err) {
    *abort_flag = 1;
    atomicOr(err, kDevErrTmaTimeout);
}

// Chunk c of n of the pixel range [r0, r1).
__device__ __forceinline__ void chunk_range(long long r0, long long r1, int c, int n, long long &c0, long long &c1) {
    const long long len = r1 - r0;
    c0 = r0 + len * c / n;
    c1 = r0 + len * (c + 1) / n;
}

template <typename T, int LPI, bool SOFTMAX, int KMAX>
__global__ void __launch_bounds__(kProjThreads, 1)
    core_forward_proj(const __grid_constant__ CUtensorMap wmap, const ProjParams p) {
    constexpr int V = Storage<T>::kVec;  // 8 channels per 16-byte chunk
    constexpr int IPW = 32 / LPI;        // items per warp step
    const CoreArgs &a = p.a;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    extern __shared__ unsigned char smem_raw[];
    // 1024-byte aligned base (the swizzle pattern repeats every 1024 bytes)
    const uint32_t raw_a = smem_u32(smem_raw);
    unsigned char *smem = smem_raw + (((raw_a + 1023u) & ~1023u) - raw_a);
    unsigned char *btile = smem;                                    // KB x npad_max x 128 bytes
    unsigned char *wst = btile + (size_t)p.KB * p.npad_max * 128;  // kWStages x kWTileBytes
    uint64_t *bars = reinterpret_cast<uint64_t *>(wst + kWStages * kWTileBytes);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + 2 * kWStages + kMaxKBlocks + 3);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);
    const uint32_t wfull = smem_u32(bars), wempty = wfull + 8 * kWStages;
    const uint32_t kready = wempty + 8 * kWStages, dfull = kready + 8 * kMaxKBlocks;
    const uint32_t tempty = dfull + 8, drain = dfull + 16;
    const uint32_t btile_a = smem_u32(btile), wst_a = smem_u32(wst);

    if (threadIdx.x == 0) {
        for (int i = 0; i < kWStages; ++i) {
            mbar_init(wfull + 8 * i, 1);
            mbar_init(wempty + 8 * i, 1);
        }
        for (int i = 0; i < kMaxKBlocks; ++i) mbar_init(kready + 8 * i, kGatherWarps);
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
            const uint32_t tx = (uint32_t)p.w_box_rows * 128u;
            for (int ci = 0; ci < n_chunks && !*abort_flag; ++ci)
                for (int kb = 0; kb < p.KB && !*abort_flag; ++kb)
                    for (int mb = 0; mb < p.MB; ++mb, ++it) {
                        const int s = it % kWStages, u = it / kWStages;
                        if (u >= 1 && !wait_or_abort(wempty + 8 * s, (u - 1) & 1, abort_flag)) {
                            raise_abort(abort_flag, p.err);
                            break;
                        }
                        mbar_arrive_expect_tx(wfull + 8 * s, tx);
                        tma_load_2d(wst_a + s * kWTileBytes, &wmap, wfull + 8 * s, kb * 64, mb * 128);
                    }
            // drain: the last load issued into each stage has landed
            for (int j = it - 1; j >= 0 && j >= it - kWStages; --j)
                mbar_wait_bounded(wfull + 8 * (j % kWStages), (j / kWStages) & 1, kProjWaitNs);
        }
        __syncwarp();
    } else if (warp == kMmaWarp) {
        // ---- tensor-core products, one thread
        if (lane == 0) {
            int it = 0;
            bool issued = false;
            const int fmt = std::is_same<T, __nv_bfloat16>::value ? 1 : 0;
            for (int ci = 0; ci < n_chunks && !*abort_flag; ++ci) {
                long long c0, c1;
                chunk_range(r0, r1, ci, n_chunks, c0, c1);
                const int npad = ((int)(c1 - c0) + 15) & ~15;
                const uint32_t idesc = instr_desc_f16(fmt, npad);
                // the epilogue has read the previous chunk's accumulators
                if (ci > 0 && !wait_or_abort(tempty, (ci - 1) & 1, abort_flag)) {
                    raise_abort(abort_flag, p.err);
                    break;
                }
                tc_fence_after();
                for (int kb = 0; kb < p.KB && !*abort_flag; ++kb) {
                    if (!wait_or_abort(kready + 8 * kb, ci & 1, abort_flag)) {
                        raise_abort(abort_flag, p.err);
                        break;
                    }
                    tc_fence_after();
                    const uint32_t b_kb = btile_a + (uint32_t)(kb * npad * 128);
                    for (int mb = 0; mb < p.MB; ++mb, ++it) {
                        const int s = it % kWStages;
                        if (!wait_or_abort(wfull + 8 * s, (it / kWStages) & 1, abort_flag)) {
                            raise_abort(abort_flag, p.err);
                            break;
                        }
                        tc_fence_after();
                        const uint32_t a_s = wst_a + s * kWTileBytes;
#pragma unroll
                        for (int k = 0; k < 4; ++k)
                            mma_f16(tmem + (uint32_t)(mb * npad), smem_desc_sw128(a_s + k * 32),
                                    smem_desc_sw128(b_kb + k * 32), idesc, (kb | k) != 0);
                        issued = true;
                        mma_commit(wempty + 8 * s);  // weight stage free once these products are done
                    }
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
        // ---- gather warps: core samples into the B operand, then the epilogue
        const int sub = lane % LPI, slot = lane / LPI;
        const int K = a.kh * a.kw;
        const int GC = a.G * a.C;
        const int gpb = 64 / a.C;  // groups per K-block
        const T *__restrict__ xg = static_cast<const T *>(a.x);
        const T *__restrict__ off = static_cast<const T *>(a.offset);
        const T *__restrict__ msk = static_cast<const T *>(a.mask);
        const T *__restrict__ bias = static_cast<const T *>(p.bias);
        T *__restrict__ out = static_cast<T *>(a.out);
        for (int ci = 0; ci < n_chunks; ++ci) {
            long long c0, c1;
            chunk_range(r0, r1, ci, n_chunks, c0, c1);
            const int n_px = (int)(c1 - c0);
            const int npad = (n_px + 15) & ~15;
            for (int kb = 0; kb < p.KB; ++kb) {
                const int items = n_px * gpb;
                for (int base = warp * IPW; base < items; base += kGatherWarps * IPW) {
                    const int item = base + slot;
                    if (item < items) {
                        const int px = item / gpb;
                        const int g = kb * gpb + (item - px * gpb);
                        long long t = c0 + px;
                        const int wo = (int)(t % a.Wo);
                        t /= a.Wo;
                        const int ho = (int)(t % a.Ho);
                        const int b = (int)(t / a.Ho);
                        const long long mi = (c0 + px) * a.G + g;
                        const T *o_item = off + mi * K * 2;
                        const T *m_item = msk + mi * K;
                        float mx = 0.0f, inv_sum = 1.0f;
                        if (SOFTMAX) {
                            mx = -INFINITY;
                            for (int k = 0; k < K; ++k) mx = fmaxf(mx, load_scalar(m_item + k));
                            float sum = 0.0f;
                            for (int k = 0; k < K; ++k) sum += expf(load_scalar(m_item + k) - mx);
                            inv_sum = 1.0f / sum;
                        }
                        float acc[V];
#pragma unroll
                        for (int v = 0; v < V; ++v) acc[v] = 0.0f;
                        bool nan_pos = false;
                        const T *xb = xg + (long long)b * a.H * a.W * GC + g * a.C + sub * V;
                        int i = 0, j = 0;
#pragma unroll
                        for (int k = 0; k < KMAX; ++k) {
                            if (k >= K) break;
                            const int by = ho * a.sh - a.ph + i * a.dh;
                            const int bx = wo * a.sw - a.pw + j * a.dw;
                            if (++j == a.kw) {
                                j = 0;
                                ++i;
                            }
                            const float2 d = load_pair(o_item + 2 * k);
                            float m = load_scalar(m_item + k);
                            if (SOFTMAX) m = expf(m - mx) * inv_sum;
                            const float pxf = fmaf(a.offset_scale, d.x, (float)bx);
                            const float pyf = fmaf(a.offset_scale, d.y, (float)by);
                            Tap tp{0, 0, 0.0f, 0.0f};
                            const int st = make_tap(pyf, pxf, a.H, a.W, tp);
                            nan_pos |= st < 0;
                            uint4 raw[4];
                            float w[4];
#pragma unroll
                            for (int c = 0; c < 4; ++c) {
                                const int y = tp.y0 + (c >> 1), x = tp.x0 + (c & 1);
                                const bool ok = st > 0 && y >= 0 && y < a.H && x >= 0 && x < a.W;
                                w[c] = ok ? ((c >> 1) ? tp.ly : 1.0f - tp.ly) * ((c & 1) ? tp.lx : 1.0f - tp.lx) * m
                                          : 0.0f;
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
                        // 16-byte chunk of row px inside this K-block, swizzled
                        const int chunk = ((g * a.C) & 63) / V + sub;
                        unsigned char *dst =
                            btile + (size_t)kb * npad * 128 + px * 128 + ((chunk ^ (px & 7)) << 4);
                        *reinterpret_cast<uint4 *>(dst) = pack16<T>(acc);
                    }
                }
                fence_proxy_async_smem();  // this thread's tile writes before the tensor core reads
                __syncwarp();
                if (lane == 0) mbar_arrive(kready + 8 * kb);
            }
            // ---- epilogue: accumulators -> + bias -> storage type
            if (!wait_or_abort(dfull, ci & 1, abort_flag)) {
                if (lane == 0) raise_abort(abort_flag, p.err);
                break;
            }
            tc_fence_after();
            const int quad = warp & 3, part = warp >> 2;
            for (int blk = part; blk < npad / 16; blk += kGatherWarps / 4) {
                for (int mb = 0; mb < p.MB; ++mb) {
                    float v[16];
                    tmem_ld16(tmem + ((uint32_t)(32 * quad) << 16) + (uint32_t)(mb * npad + blk * 16), v);
                    const int o = mb * 128 + 32 * quad + lane;
                    if (o < p.Cout) {
                        const float bo = bias ? load_scalar(bias + o) : 0.0f;
#pragma unroll
                        for (int q = 0; q < 16; ++q) {
                            const int px = blk * 16 + q;
                            if (px < n_px) out[(c0 + px) * p.Cout + o] = from_f32<T>(v[q] + bo);
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

template <typename T, int LPI, bool SOFTMAX, int KMAX>
cudaError_t launch_one(const CUtensorMap &map, const ProjParams &p, size_t smem, cudaStream_t stream) {
    auto kern = core_forward_proj<T, LPI, SOFTMAX, KMAX>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    kern<<<p.n_cta, kProjThreads, smem, stream>>>(map, p);
    return cudaGetLastError();
}

template <typename T, int LPI>
cudaError_t launch_lpi(const CUtensorMap &map, const ProjParams &p, size_t smem, cudaStream_t stream) {
    const int K = p.a.kh * p.a.kw;
    if (K <= 9) {
        return p.a.softmax ? launch_one<T, LPI, true, 9>(map, p, smem, stream)
                           : launch_one<T, LPI, false, 9>(map, p, smem, stream);
    }
    return p.a.softmax ? launch_one<T, LPI, true, 25>(map, p, smem, stream)
                       : launch_one<T, LPI, false, 25>(map, p, smem, stream);
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
    p.KB = a.G * a.C / 64;
    p.err = dev->err;
    long long n_cta = dev->sms;
    if (n_cta * 16 > p.P) n_cta = (p.P + 15) / 16;  // at least 16 pixels per CTA
    p.n_cta = (int)(n_cta < 1 ? 1 : n_cta);
    // every chunk holds at most min(range, 128) pixels, and no range exceeds
    // ceil(P / n_cta)
    const long long max_range = (p.P + p.n_cta - 1) / p.n_cta;
    p.npad_max = (int)(((max_range < kMaxChunk ? max_range : kMaxChunk) + 15) & ~15LL);
    int cols = 32;
    while (cols < p.MB * p.npad_max) cols <<= 1;
    p.tmem_cols = cols;
    p.w_box_rows = pa.Cout < 128 ? pa.Cout : 128;

    // B operand + weight ring + barriers, plus the alignment slack; at least
    // half an SM's shared memory so that one CTA owns the SM's tensor memory
    size_t smem = (size_t)p.KB * p.npad_max * 128 + (size_t)kWStages * kWTileBytes + 256 + 1024;
    const size_t half_sm = (size_t)dev->smem_per_sm / 2 + 1024;
    if (smem < half_sm) smem = half_sm;
    if (smem > (size_t)dev->smem_optin) return cudaErrorInvalidConfiguration;

    CUtensorMap map;
    const cuuint64_t dims[2] = {(cuuint64_t)a.G * a.C, (cuuint64_t)pa.Cout};
    const cuuint64_t strides[1] = {dims[0] * 2};
    const cuuint32_t box[2] = {64, (cuuint32_t)p.w_box_rows};
    const cuuint32_t estr[2] = {1, 1};
    const CUresult r = enc(&map, CU_TENSOR_MAP_DATA_TYPE_UINT16, 2, const_cast<void *>(pa.weight), dims, strides, box,
                           estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                           CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return cudaErrorInvalidValue;
    switch (a.C * (int)sizeof(T) / 16) {
        case 1: return launch_lpi<T, 1>(map, p, smem, stream);
        case 2: return launch_lpi<T, 2>(map, p, smem, stream);
        case 4: return launch_lpi<T, 4>(map, p, smem, stream);
        case 8: return launch_lpi<T, 8>(map, p, smem, stream);
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
