// Pointwise projection on the tensor cores (sm_100a): the 1x1 convolution
// with bias that follows the sampling core in the DCNv4 module (YOLOv11 +
// DCNv4 page, section 3.2, proj_conv), as a plain GEMM over a core output
// that already sits in device memory:
//   out[p, o] = bias[o] + sum_j core[p, j] * weight[o, j]
// core [P, KD] and weight [Cout, KD] are both K-major (row-major with the
// contraction index fastest), fp16 or bf16; out [P, Cout] in the same type.
//
// Persistent, warp-specialised: every CTA works on one tile of up to 128
// output channels, whose weight rows (all K-blocks, at most 128 KB) warp 0
// loads once into shared memory by TMA; it then streams the CTA's pixel
// tiles, K-block by K-block (64 channels, 128-byte swizzle), through a
// 4-stage ring.  One thread of warp 1 issues tcgen05.mma (M = 128 pixels,
// N = up to 128 output channels, K = 16) into one of two tensor-memory
// accumulators, and
// warps 2..5 (one per 32-lane quarter of tensor memory) read the finished
// accumulator back with tcgen05.ld, add the bias in fp32, round once to the
// storage type and store, while the products of the next tile already run
// into the other accumulator.  Every wait is bounded and gives up when
// another role has aborted; a role that gives up sets the device error word.
#include <cudaTypedefs.h>

#include <type_traits>

#include "dcn_common.cuh"
#include "dcn_device.h"
#include "dcn_launch.h"
#include "dcn_tcgen05.cuh"

namespace dcnb {

PFN_cuTensorMapEncodeTiled_v12000 encode_fn();  // dcn_forward_plane.cu
const DeviceInfo *device_info();

namespace {

constexpr int kGStages = 4;
constexpr int kBM = 128;                 // pixels per tile (the MMA's M)
constexpr int kBK = 64;                  // channels per K-block (128 bytes: one swizzle row)
constexpr int kABytes = kBM * kBK * 2;   // 16 KB
constexpr int kBNMax = 128;              // output channels per tile (resident weight rows)
constexpr int kMaxKB = 8;                // K-blocks of the contraction (G*C <= 512)
constexpr int kGThreads = 6 * 32;

// 32 consecutive fp32 accumulator columns of this warp's 32 tensor-memory lanes.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float *v) {
    uint32_t r[32];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
        "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
          "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
          "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
    for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}

struct GemmParams {
    long long P;       // pixels (rows of core and out)
    int KD, Cout;      // contraction length, output channels
    int BN;            // output channels per tile (multiple of 32, <= 128)
    int NT;            // output-channel tiles
    long long PT;      // pixel tiles
    int n_cta;         // a multiple of NT: CTA c works on output-channel tile c % NT
    int tmem_cols;     // 2 * BN rounded up to a power of two
    const void *bias;  // [Cout] or nullptr
    void *out;
    unsigned int *err;
    int store32;       // out rows start on 32-byte boundaries: 32-byte stores (whole L2 sectors)
};

template <typename T>
__global__ void __launch_bounds__(kGThreads, 1)
    proj_gemm_kernel(const __grid_constant__ CUtensorMap amap, const __grid_constant__ CUtensorMap bmap,
                     const GemmParams p) {
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    // 1024-byte alignment of the swizzled tiles
    unsigned char *smem = reinterpret_cast<unsigned char *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
    const int KB = p.KD / kBK;
    const int wblk = p.BN * kBK * 2;  // one resident weight K-block
    unsigned char *wres = smem;       // [KB][BN rows x 128 bytes], swizzled
    unsigned char *ring = smem + KB * wblk;
    uint64_t *bars = reinterpret_cast<uint64_t *>(ring + kGStages * kABytes);
    // full[s], empty[s], acc_full[2], acc_empty[2], drain, weights[kMaxKB] (one per resident K-block)
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + 2 * kGStages + 5 + kMaxKB);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);
    // [NT * BN] fp32 bias, zero past Cout, at the next 16-byte boundary after the slot and the flag
    float *bias_s = reinterpret_cast<float *>((reinterpret_cast<uintptr_t>(tmem_slot + 2) + 15) & ~(uintptr_t)15);
    const uint32_t full0 = smem_u32(bars), empty0 = full0 + 8 * kGStages;
    const uint32_t accf0 = empty0 + 8 * kGStages, acce0 = accf0 + 16, drain = acce0 + 16, wfull = drain + 8;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int nt = blockIdx.x % p.NT;  // this CTA's output-channel tile
    const long long pt0 = blockIdx.x / p.NT, pstep = p.n_cta / p.NT;

    if (threadIdx.x == 0) {
        for (int i = 0; i < kGStages; ++i) {
            mbar_init(full0 + 8 * i, 1);
            mbar_init(empty0 + 8 * i, 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(accf0 + 8 * i, 1);
            mbar_init(acce0 + 8 * i, 4);  // one arrival per epilogue warp
        }
        mbar_init(drain, 1);
        for (int i = 0; i < kMaxKB; ++i) mbar_init(wfull + 8 * i, 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                     "r"(p.tmem_cols)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    // The launcher makes this kernel a programmatic dependent of the core kernel
    // that writes the pixel matrix, so it may start while that kernel's last CTAs
    // run: the producer issues this CTA's weight rows (which the core kernel does
    // not write) first, then every thread waits for the core kernel to complete
    // before any wait of its own starts (the instruction returns at once when the
    // launch was an ordinary one).
    int wissued = 0;  // weight K-blocks issued (producer thread)
    if (warp == 0 && lane == 0 && pt0 < p.PT)
        for (int j = 0; j < KB; ++j, ++wissued) {
            mbar_arrive_expect_tx(wfull + 8 * j, (uint32_t)wblk);
            tma_load_2d(smem_u32(wres + j * wblk), &bmap, wfull + 8 * j, j * kBK, nt * p.BN);
        }
    asm volatile("griddepcontrol.wait;" ::: "memory");

    if (warp == 0) {
        // ---- producer: the pixel K-blocks of this CTA's tiles
        if (lane == 0) {
            uint32_t s = 0, pass = 0;
            long long issued = 0;
            for (long long pt = pt0; pt < p.PT && !*abort_flag; pt += pstep) {
                for (int kb = 0; kb < KB; ++kb) {
                    if (pass >= 1 && !wait_or_abort(empty0 + 8 * s, (pass - 1) & 1, abort_flag)) {
                        raise_abort(abort_flag, p.err);
                        break;
                    }
                    mbar_arrive_expect_tx(full0 + 8 * s, (uint32_t)kABytes);
                    tma_load_2d(smem_u32(ring + s * kABytes), &amap, full0 + 8 * s, kb * kBK, (int)pt * kBM);
                    ++issued;
                    if (++s == kGStages) {
                        s = 0;
                        ++pass;
                    }
                }
            }
            // drain: the weights and the last load of every stage have landed before the CTA may exit
            for (int kb = 0; kb < wissued; ++kb) mbar_wait_bounded(wfull + 8 * kb, 0, kTcWaitNs);
            for (long long j = issued - 1; j >= 0 && j >= issued - kGStages; --j)
                mbar_wait_bounded(full0 + 8 * (uint32_t)(j % kGStages), (uint32_t)(j / kGStages) & 1, kTcWaitNs);
        }
        __syncwarp();
    } else if (warp == 1) {
        // ---- one thread issues the products
        if (lane == 0) {
            const int fmt = std::is_same<T, __nv_bfloat16>::value ? 1 : 0;
            const uint32_t idesc = instr_desc_f16(fmt, p.BN);
            const uint64_t a0 = smem_desc_sw128(smem_u32(ring)), b0 = smem_desc_sw128(smem_u32(wres));
            const uint32_t sstep = (uint32_t)kABytes >> 4, wstep = (uint32_t)wblk >> 4;
            uint32_t s = 0, ph = 0;
            int local = 0;
            bool ok = true, issued = false;
            for (long long pt = pt0; pt < p.PT && ok; pt += pstep, ++local) {
                const int buf = local & 1;
                // the epilogue has emptied this accumulator (used two tiles ago)
                if (local >= 2 && !wait_or_abort(acce0 + 8 * buf, ((local >> 1) - 1) & 1, abort_flag)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t dcol = tmem + (uint32_t)(buf * p.BN);
                for (int kb = 0; kb < KB; ++kb) {
                    if ((local == 0 && !wait_or_abort(wfull + 8 * kb, 0, abort_flag)) ||
                        !wait_or_abort(full0 + 8 * s, ph, abort_flag)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint64_t ad = a0 + s * sstep, bd = b0 + kb * wstep;
                    // k-steps of 16 elements = 32 bytes = 2 descriptor units
                    mma_f16(dcol, ad, bd, idesc, kb != 0);
                    mma_f16(dcol, ad + 2, bd + 2, idesc, 1u);
                    mma_f16(dcol, ad + 4, bd + 4, idesc, 1u);
                    mma_f16(dcol, ad + 6, bd + 6, idesc, 1u);
                    issued = true;
                    mma_commit(empty0 + 8 * s);  // stage free once these products are done
                    if (++s == kGStages) {
                        s = 0;
                        ph ^= 1u;
                    }
                }
                if (!ok) break;
                mma_commit(accf0 + 8 * buf);  // accumulator complete
            }
            if (!ok) raise_abort(abort_flag, p.err);
            if (issued) {
                // every product this thread issued has finished before tensor memory is freed
                mma_commit(drain);
                mbar_wait_bounded(drain, 0, kTcWaitNs);
            }
        }
        __syncwarp();
    } else {
        // ---- epilogue: warp w reads tensor-memory lanes 32*(w % 4) .. +31 = pixel rows of the tile
        const int quad = warp & 3;
        const T *bias = static_cast<const T *>(p.bias);
        T *out = static_cast<T *>(p.out);
        // the bias, once per CTA, in fp32 (zero past Cout or without bias)
        for (int i = threadIdx.x - 64; i < p.NT * p.BN; i += 128)
            bias_s[i] = (bias && i < p.Cout) ? to_f32(bias[i]) : 0.0f;
        asm volatile("bar.sync 1, 128;" ::: "memory");  // the four epilogue warps
        int local = 0;
        for (long long pt = pt0; pt < p.PT; pt += pstep, ++local) {
            const int buf = local & 1;
            if (!wait_or_abort(accf0 + 8 * buf, (local >> 1) & 1, abort_flag)) {
                raise_abort(abort_flag, p.err);
                break;
            }
            tc_fence_after();
            const long long row = pt * kBM + quad * 32 + lane;
            for (int c = 0; c < p.BN; c += 32) {
                float v[32];
                tmem_ld32(tmem + ((uint32_t)(32 * quad) << 16) + (uint32_t)(buf * p.BN + c), v);
                const int o0 = nt * p.BN + c;
                if (o0 >= p.Cout) continue;  // warp-uniform
                const float4 *bb = reinterpret_cast<const float4 *>(bias_s + o0);
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const float4 b4 = bb[i];
                    v[4 * i] += b4.x;
                    v[4 * i + 1] += b4.y;
                    v[4 * i + 2] += b4.z;
                    v[4 * i + 3] += b4.w;
                }
                if (row < p.P) {
                    T *dst = out + row * p.Cout + o0;
                    const int n16 = (p.Cout - o0) >= 32 ? 4 : (p.Cout - o0) / 8;  // Cout is a multiple of 8
                    if (p.store32 && n16 == 4) {
                        // two 32-byte stores: every store fills whole 32-byte sectors of L2
#pragma unroll
                        for (int i = 0; i < 2; ++i) {
                            const uint4 lo = pack16<T>(v + 16 * i), hi = pack16<T>(v + 16 * i + 8);
                            asm volatile("st.global.v8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};" ::"l"(dst + 16 * i),
                                         "r"(lo.x), "r"(lo.y), "r"(lo.z), "r"(lo.w), "r"(hi.x), "r"(hi.y), "r"(hi.z),
                                         "r"(hi.w)
                                         : "memory");
                        }
                    } else {
#pragma unroll
                        for (int i = 0; i < 4; ++i)
                            if (i < n16) reinterpret_cast<uint4 *>(dst)[i] = pack16<T>(v + 8 * i);
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(acce0 + 8 * buf);
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(p.tmem_cols)
                     : "memory");
    }
}

template <typename T>
cudaError_t launch_t(const void *core, const void *weight, const void *bias, void *out, long long P, int KD,
                     int Cout, cudaStream_t stream) {
    auto enc = encode_fn();
    const DeviceInfo *dev = device_info();
    if (!enc || !dev) return cudaErrorNotSupported;
    GemmParams p;
    p.P = P;
    p.KD = KD;
    p.Cout = Cout;
    // a multiple of 32, so the epilogue's 32-column loads stay inside the tile
    const int c32 = (Cout + 31) & ~31;
    p.BN = c32 <= kBNMax ? c32 : kBNMax;
    p.NT = (Cout + p.BN - 1) / p.BN;
    p.PT = (P + kBM - 1) / kBM;
    long long per_nt = dev->sms / p.NT;  // CTAs per output-channel tile
    if (per_nt > p.PT) per_nt = p.PT;
    if (per_nt < 1) per_nt = 1;
    p.n_cta = (int)(per_nt * p.NT);
    int cols = 32;
    while (cols < 2 * p.BN) cols <<= 1;
    p.tmem_cols = cols;
    p.bias = bias;
    p.out = out;
    p.err = dev->err;
    p.store32 = Cout % 16 == 0 && (reinterpret_cast<uintptr_t>(out) & 31) == 0;

    CUtensorMap amap, bmap;
    const cuuint32_t estr[2] = {1, 1};
    const cuuint64_t adims[2] = {(cuuint64_t)KD, (cuuint64_t)P};
    const cuuint64_t astr[1] = {(cuuint64_t)KD * 2};
    const cuuint32_t abox[2] = {(cuuint32_t)kBK, (cuuint32_t)kBM};
    const cuuint64_t bdims[2] = {(cuuint64_t)KD, (cuuint64_t)Cout};
    const cuuint64_t bstr[1] = {(cuuint64_t)KD * 2};
    const cuuint32_t bbox[2] = {(cuuint32_t)kBK, (cuuint32_t)p.BN};
    const CUtensorMapDataType dt = std::is_same<T, __half>::value ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16
                                                                  : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
    if (enc(&amap, dt, 2, const_cast<void *>(core), adims, astr, abox, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
            CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
        return cudaErrorInvalidValue;
    if (enc(&bmap, dt, 2, const_cast<void *>(weight), bdims, bstr, bbox, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
            CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
        return cudaErrorInvalidValue;
    const size_t smem = 1024 + (size_t)(KD / kBK) * p.BN * kBK * 2 + (size_t)kGStages * kABytes +
                        (2 * kGStages + 5 + kMaxKB) * 8 + 32 + (size_t)p.NT * p.BN * 4;
    auto kern = proj_gemm_kernel<T>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    // programmatic dependent launch: the CTAs may start (and fetch their weight
    // rows) as the preceding kernel on the stream finishes
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)p.n_cta);
    cfg.blockDim = dim3(kGThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, amap, bmap, p);
}

}  // namespace

cudaError_t launch_proj_gemm(const void *core, const void *weight, const void *bias, void *out, long long P, int KD,
                             int Cout, DType dtype, cudaStream_t stream) {
    if (P <= 0) return cudaSuccess;
    switch (dtype) {
        case DType::F16: return launch_t<__half>(core, weight, bias, out, P, KD, Cout, stream);
        case DType::BF16: return launch_t<__nv_bfloat16>(core, weight, bias, out, P, KD, Cout, stream);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace dcnb
