// Host-side planning of the staged forward (kernel in dcn_forward_staged.cuh):
// picks the band height, the halo and one or two band buffers from the shared
// memory budget left by the records of staged_threads() warps, builds the 4-D
// TMA tensor map of x, and launches the persistent grid of one CTA per SM.  Shapes the staged kernel does not cover (W > 254,
// K > 25, 16-byte groups, a map the tensor-map encoder rejects) are left to
// the generic kernel.
#include <cudaTypedefs.h>

#include <mutex>

#include "dcn_device.h"
#include "dcn_forward_staged.cuh"

namespace dcnb {

// Set (bitwise OR) by a kernel whose bounded wait ran out.
__device__ unsigned int g_device_error = 0;

cudaError_t take_device_error(unsigned int *value) {
    // The symbol copies below run on the legacy default stream, which does not
    // wait for work on non-blocking streams (torch's pool streams are such):
    // without a device-wide synchronisation the read could miss the bit of a
    // kernel still running there, and the clear could wipe it.
    cudaError_t e = cudaDeviceSynchronize();
    if (e != cudaSuccess) return e;
    unsigned int zero = 0;
    e = cudaMemcpyFromSymbol(value, g_device_error, sizeof(unsigned int));
    if (e != cudaSuccess) return e;
    return cudaMemcpyToSymbol(g_device_error, &zero, sizeof(unsigned int));
}

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

const DeviceInfo *device_info() {
    constexpr int kMaxDev = 64;
    static DeviceInfo info[kMaxDev];
    static std::once_flag once[kMaxDev];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDev) return nullptr;
    std::call_once(once[dev], [dev] {
        DeviceInfo &d = info[dev];
        cudaDeviceGetAttribute(&d.sms, cudaDevAttrMultiProcessorCount, dev);
        cudaDeviceGetAttribute(&d.smem_optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
        cudaDeviceGetAttribute(&d.smem_per_sm, cudaDevAttrMaxSharedMemoryPerMultiprocessor, dev);
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_device_error) == cudaSuccess) d.err = static_cast<unsigned int *>(p);
    });
    return info[dev].err ? &info[dev] : nullptr;
}

namespace {

constexpr int kHaloMax = 8;   // rows of margin for the offsets
constexpr int kBoxRows = 4;   // rows per TMA box

template <typename T>
cudaError_t launch_t(const CoreArgs &a, cudaStream_t stream, bool *handled) {
    const int RB = a.C * (int)sizeof(T);
    if (RB != 32 && RB != 64 && RB != 128 && RB != 256) return cudaSuccess;
    const int K = a.kh * a.kw;
    if (K > 25 || a.W + 2 > 256) return cudaSuccess;
    if ((long long)a.Ho * a.Wo >= (1LL << 31)) return cudaSuccess;  // plane index decode is 32-bit
    const int kmax = K <= 9 ? 9 : 25;
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
    // One CTA of staged_threads() per SM: a producer warp stages the bands of
    // consecutive segments while the consumer warps gather.  Two band buffers
    // (the next segment loads while the current one is gathered) when they
    // still hold segments of >= 8 output rows with the full halo, else one.
    const int threads = staged_threads(a.softmax, RB, kmax), nc = threads / 32 - 1;
    const size_t other = (size_t)nc * (kmax * IPW * 28 + IPW * 4) + (size_t)kmax * 8 + 32;
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
    long long n_cta = (long long)dev->sms * chosen;
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
    return launch_staged_instance<T>(map, s, RB, a.softmax, kmax, smem, stream);
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
