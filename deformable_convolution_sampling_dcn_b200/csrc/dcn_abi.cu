// C ABI of the library: host-side argument checks, then one launch (or a
// memset and a launch) on the caller's stream.  No allocation, no
// synchronisation.  See include/dcn_b200.h for the contract.
#include <math.h>
#include <stdarg.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include <mutex>

#include "dcn_b200.h"
#include "dcn_launch.h"

namespace {

thread_local char g_detail[256] = "no error";

dcn_status fail(dcn_status s, const char *fmt, ...) __attribute__((format(printf, 2, 3)));
dcn_status fail(dcn_status s, const char *fmt, ...) {
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_detail, sizeof(g_detail), fmt, ap);
    va_end(ap);
    return s;
}

dcn_status cuda_status(cudaError_t e, const char *what) {
    if (e == cudaSuccess) return DCN_OK;
    return fail(DCN_ERR_CUDA, "%s: %s (%s)", what, cudaGetErrorName(e), cudaGetErrorString(e));
}

size_t dtype_size(int32_t dt) { return dt == DCN_F32 ? 4 : 2; }

bool aligned(const void *p, size_t a) { return ((uintptr_t)p % a) == 0; }

const int kMaxDim = 1 << 20;

// Checks shared by the core calls; fills Ho/Wo.
dcn_status check_core(const dcn_params *p, int *Ho, int *Wo) {
    if (!p) return fail(DCN_ERR_NULL, "params is NULL");
    if (p->dtype < DCN_F32 || p->dtype > DCN_BF16) return fail(DCN_ERR_UNSUPPORTED, "dtype %d", p->dtype);
    if (p->mask_mode != DCN_MASK_RAW && p->mask_mode != DCN_MASK_SOFTMAX)
        return fail(DCN_ERR_UNSUPPORTED, "mask_mode %d", p->mask_mode);
    if (p->B < 0 || p->H < 1 || p->W < 1 || p->G < 1 || p->C < 1 || p->kh < 1 || p->kw < 1)
        return fail(DCN_ERR_SHAPE, "sizes must be positive (B may be 0)");
    if (p->B > kMaxDim || p->H > kMaxDim || p->W > kMaxDim || p->G > kMaxDim || p->C > kMaxDim ||
        p->kh > 64 || p->kw > 64)
        return fail(DCN_ERR_SHAPE, "a size exceeds its limit");
    if (p->stride_h < 1 || p->stride_w < 1 || p->dil_h < 1 || p->dil_w < 1)
        return fail(DCN_ERR_SHAPE, "stride and dilation must be >= 1");
    if (p->pad_h < 0 || p->pad_w < 0 || p->pad_h > kMaxDim || p->pad_w > kMaxDim)
        return fail(DCN_ERR_SHAPE, "padding must be in [0, 2^20]");
    if (!isfinite(p->offset_scale)) return fail(DCN_ERR_SHAPE, "offset_scale is not finite");
    const long long eh = (long long)p->dil_h * (p->kh - 1) + 1, ew = (long long)p->dil_w * (p->kw - 1) + 1;
    const long long ho = ((long long)p->H + 2LL * p->pad_h - eh), wo = ((long long)p->W + 2LL * p->pad_w - ew);
    if (ho < 0 || wo < 0) return fail(DCN_ERR_SHAPE, "kernel extent exceeds the padded input");
    *Ho = (int)(ho / p->stride_h + 1);
    *Wo = (int)(wo / p->stride_w + 1);
    const size_t es = dtype_size(p->dtype);
    const size_t row = (size_t)p->C * es;
    if (row % 16 != 0 || row / 16 > 16 || ((row / 16) & (row / 16 - 1)) != 0)
        return fail(DCN_ERR_UNSUPPORTED, "C*sizeof(dtype) = %zu bytes; supported: 16, 32, 64, 128, 256", row);
    if ((long long)p->G * p->C > kMaxDim) return fail(DCN_ERR_SHAPE, "G*C exceeds 2^20");
    return DCN_OK;
}

dcnb::CoreArgs core_args(const dcn_params *p, int Ho, int Wo) {
    dcnb::CoreArgs a;
    memset(&a, 0, sizeof(a));
    a.B = p->B; a.H = p->H; a.W = p->W; a.G = p->G; a.C = p->C; a.kh = p->kh; a.kw = p->kw;
    a.sh = p->stride_h; a.sw = p->stride_w; a.ph = p->pad_h; a.pw = p->pad_w;
    a.dh = p->dil_h; a.dw = p->dil_w; a.Ho = Ho; a.Wo = Wo;
    a.offset_scale = p->offset_scale;
    a.softmax = p->mask_mode == DCN_MASK_SOFTMAX;
    a.dtype = (dcnb::DType)p->dtype;
    return a;
}

dcn_status check_agg(const dagg_params *p) {
    if (!p) return fail(DCN_ERR_NULL, "params is NULL");
    if (p->dtype < DCN_F32 || p->dtype > DCN_BF16) return fail(DCN_ERR_UNSUPPORTED, "dtype %d", p->dtype);
    if (p->B < 0 || p->num_cams < 1 || p->num_scales < 1 || p->num_rows < 1 || p->num_anchors < 0 ||
        p->num_pts < 1 || p->G < 1 || p->C < 1)
        return fail(DCN_ERR_SHAPE, "sizes must be positive (B and num_anchors may be 0)");
    if ((long long)p->num_cams * p->num_scales > 4096 || (long long)p->num_pts * p->num_cams > (1 << 20) ||
        (long long)p->G * p->C > kMaxDim)
        return fail(DCN_ERR_SHAPE, "a size exceeds its limit");
    const size_t row = (size_t)p->C * dtype_size(p->dtype);
    if (row % 16 != 0 || row / 16 > 16 || ((row / 16) & (row / 16 - 1)) != 0)
        return fail(DCN_ERR_UNSUPPORTED, "C*sizeof(dtype) = %zu bytes; supported: 16, 32, 64, 128, 256", row);
    return DCN_OK;
}

dcnb::AggArgs agg_args(const dagg_params *p) {
    dcnb::AggArgs a;
    memset(&a, 0, sizeof(a));
    a.B = p->B; a.cams = p->num_cams; a.scales = p->num_scales; a.rows = p->num_rows;
    a.A = p->num_anchors; a.P = p->num_pts; a.G = p->G; a.C = p->C;
    a.dtype = (dcnb::DType)p->dtype;
    return a;
}

}  // namespace

extern "C" {

int32_t dcn_abi_version(void) { return DCN_ABI_VERSION; }

int32_t dcn_take_device_error(void) {
    unsigned int v = 0;
    if (dcnb::take_device_error(&v) != cudaSuccess) return -1;
    return (int32_t)v;
}

const char *dcn_last_error_detail(void) { return g_detail; }

dcn_status dcn_selftest_bounded_wait(int32_t limit_us, dcn_stream_t stream) {
    if (limit_us < 1 || limit_us > 10000000) return fail(DCN_ERR_SHAPE, "limit_us must be in [1, 10^7]");
    return cuda_status(dcnb::launch_bounded_wait_selftest((long long)limit_us * 1000, (cudaStream_t)stream),
                       "dcn_selftest_bounded_wait launch");
}

const char *dcn_status_string(dcn_status s) {
    switch (s) {
        case DCN_OK: return "DCN_OK";
        case DCN_ERR_NULL: return "DCN_ERR_NULL: a required pointer is NULL";
        case DCN_ERR_SHAPE: return "DCN_ERR_SHAPE: invalid sizes";
        case DCN_ERR_UNSUPPORTED: return "DCN_ERR_UNSUPPORTED: configuration not implemented";
        case DCN_ERR_ALIGN: return "DCN_ERR_ALIGN: misaligned pointer";
        case DCN_ERR_CUDA: return "DCN_ERR_CUDA: CUDA runtime error";
    }
    return "unknown dcn_status";
}

dcn_status dcn_core_output_hw(const dcn_params *p, int32_t *Ho, int32_t *Wo) {
    int ho = 0, wo = 0;
    const dcn_status s = check_core(p, &ho, &wo);
    if (s != DCN_OK) return s;
    if (!Ho || !Wo) return fail(DCN_ERR_NULL, "Ho/Wo output pointer is NULL");
    *Ho = ho;
    *Wo = wo;
    return DCN_OK;
}

dcn_status dcn_core_forward(const dcn_params *p, const void *x, const void *offset, const void *mask,
                            void *out, dcn_stream_t stream) {
    int Ho = 0, Wo = 0;
    dcn_status s = check_core(p, &Ho, &Wo);
    if (s != DCN_OK) return s;
    if (p->B == 0) return DCN_OK;
    if (!x || !offset || !mask || !out) return fail(DCN_ERR_NULL, "x, offset, mask and out are required");
    const size_t es = dtype_size(p->dtype);
    if (!aligned(x, 16) || !aligned(out, 16)) return fail(DCN_ERR_ALIGN, "x and out must be 16-byte aligned");
    if (!aligned(offset, 2 * es) || !aligned(mask, es))
        return fail(DCN_ERR_ALIGN, "offset must be aligned to 2*sizeof(dtype), mask to sizeof(dtype)");
    dcnb::CoreArgs a = core_args(p, Ho, Wo);
    a.x = x; a.offset = offset; a.mask = mask; a.out = out;
    bool handled = false;
    cudaError_t e = cudaSuccess;
    const char *force = getenv("DCN_B200_FORCE_GENERIC");
    if (!(force && force[0] == '1')) e = dcnb::launch_core_forward_plane(a, (cudaStream_t)stream, &handled);
    if (!handled) e = dcnb::launch_core_forward_generic(a, (cudaStream_t)stream);
    return cuda_status(e, "dcn_core_forward launch");
}

namespace {

// Bytes of the core output [B, Ho, Wo, G*C] (-1 for invalid params).
long long core_out_bytes(const dcn_params *p) {
    int Ho = 0, Wo = 0;
    if (check_core(p, &Ho, &Wo) != DCN_OK) return -1;
    return (long long)p->B * Ho * Wo * p->G * p->C * (long long)dtype_size(p->dtype);
}

dcn_status proj_call(const dcn_params *p, int32_t Cout, const void *x, const void *offset, const void *mask,
                     const void *weight, const void *bias, void *out, void *workspace, int64_t workspace_bytes,
                     dcn_stream_t stream, bool per_point, const char *what) {
    int Ho = 0, Wo = 0;
    dcn_status s = check_core(p, &Ho, &Wo);
    if (s != DCN_OK) return s;
    if (p->dtype != DCN_F16 && p->dtype != DCN_BF16)
        return fail(DCN_ERR_UNSUPPORTED, "the fused contraction takes fp16 or bf16 (dtype %d)", p->dtype);
    if (p->C > 64) return fail(DCN_ERR_UNSUPPORTED, "the fused contraction takes C <= 64 (C = %d)", p->C);
    const long long GC = (long long)p->G * p->C;
    if (GC % 64 != 0 || GC > 512)
        return fail(DCN_ERR_UNSUPPORTED, "the fused contraction takes G*C in {64, 128, ..., 512} (G*C = %lld)", GC);
    if ((long long)p->kh * p->kw > 25)
        return fail(DCN_ERR_UNSUPPORTED, "the fused contraction takes kh*kw <= 25");
    if (Cout < 8 || Cout > 512 || Cout % 8 != 0)
        return fail(DCN_ERR_UNSUPPORTED, "Cout must be a multiple of 8 in [8, 512] (Cout = %d)", Cout);
    if ((long long)p->B * p->H * p->W >= (1LL << 31) || (long long)p->B * Ho * Wo >= (1LL << 31))
        return fail(DCN_ERR_UNSUPPORTED, "the fused contraction takes B*H*W and B*Ho*Wo below 2^31");
    if (p->B == 0) return DCN_OK;
    if (!x || !offset || !mask || !weight || !out)
        return fail(DCN_ERR_NULL, "x, offset, mask, weight and out are required");
    if (!aligned(x, 16) || !aligned(out, 16) || !aligned(weight, 16))
        return fail(DCN_ERR_ALIGN, "x, weight and out must be 16-byte aligned");
    if (!aligned(offset, 4) || !aligned(mask, 2) || !aligned(bias, 2))
        return fail(DCN_ERR_ALIGN, "offset must be 4-byte aligned, mask and bias 2-byte aligned");
    const long long need = core_out_bytes(p);
    if (!per_point && workspace && workspace_bytes >= need) {
        // two launches: the core into the workspace (staged kernel where it applies),
        // then the tensor-core projection of that [B*Ho*Wo, G*C] matrix
        if (!aligned(workspace, 16)) return fail(DCN_ERR_ALIGN, "workspace must be 16-byte aligned");
        dcnb::CoreArgs c = core_args(p, Ho, Wo);
        c.x = x; c.offset = offset; c.mask = mask; c.out = workspace;
        bool handled = false;
        cudaError_t e = dcnb::launch_core_forward_plane(c, (cudaStream_t)stream, &handled);
        if (e == cudaSuccess && !handled) e = dcnb::launch_core_forward_generic(c, (cudaStream_t)stream);
        if (e == cudaSuccess)
            e = dcnb::launch_proj_gemm(workspace, weight, bias, out, (long long)p->B * Ho * Wo, (int)GC, Cout,
                                       (dcnb::DType)p->dtype, (cudaStream_t)stream);
        return cuda_status(e, what);
    }
    dcnb::ProjArgs a;
    a.core = core_args(p, Ho, Wo);
    a.core.x = x; a.core.offset = offset; a.core.mask = mask; a.core.out = out;
    a.weight = weight;
    a.bias = bias;
    a.Cout = Cout;
    a.per_point = per_point;
    return cuda_status(dcnb::launch_core_forward_proj(a, (cudaStream_t)stream), what);
}

}  // namespace

dcn_status dcn_core_forward_proj(const dcn_params *p, int32_t Cout, const void *x, const void *offset,
                                 const void *mask, const void *weight, const void *bias, void *out,
                                 void *workspace, int64_t workspace_bytes, dcn_stream_t stream) {
    if (workspace_bytes < 0) return fail(DCN_ERR_SHAPE, "workspace_bytes is negative");
    return proj_call(p, Cout, x, offset, mask, weight, bias, out, workspace, workspace_bytes, stream, false,
                     "dcn_core_forward_proj launch");
}

}  // extern "C"

namespace {

// Scratch of dcn_core_forward_proj_noalloc: a fixed array in device memory,
// one per GPU that loads the library, kept until the process exits.  Host code
// may not pass the symbol itself to a kernel (on the host it names a shadow
// variable, not device memory): noalloc_scratch() looks its device address up
// once per device, with that device current.
constexpr size_t kNoAllocScratchBytes = (size_t)DCN_NOALLOC_SCRATCH_BYTES;
__device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

void *noalloc_scratch(cudaError_t *err) {
    constexpr int kMaxDev = 64;
    static void *addr[kMaxDev];
    static cudaError_t status[kMaxDev];
    static std::once_flag once[kMaxDev];
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess || dev < 0 || dev >= kMaxDev) {
        *err = e != cudaSuccess ? e : cudaErrorInvalidDevice;
        return nullptr;
    }
    std::call_once(once[dev], [dev] {
        void *p = nullptr;
        status[dev] = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        addr[dev] = status[dev] == cudaSuccess ? p : nullptr;
    });
    *err = status[dev];
    return addr[dev];
}

}  // namespace

extern "C" {

dcn_status dcn_core_forward_proj_noalloc(const dcn_params *p, int32_t Cout, const void *x, const void *offset,
                                         const void *mask, const void *weight, const void *bias, void *out,
                                         dcn_stream_t stream) {
    const long long need = core_out_bytes(p);
    if (need < 0) {
        int Ho = 0, Wo = 0;
        return check_core(p, &Ho, &Wo);  // the same status and detail as the other calls
    }
    if ((size_t)need > kNoAllocScratchBytes)
        return fail(DCN_ERR_UNSUPPORTED,
                    "dcn_core_forward_proj_noalloc: the core output needs %lld bytes, more than its fixed "
                    "%zu-byte scratch; use dcn_core_forward_proj with a workspace",
                    need, kNoAllocScratchBytes);
    if (p->B == 0) return proj_call(p, Cout, x, offset, mask, weight, bias, out, nullptr, 0, stream, false,
                                    "dcn_core_forward_proj_noalloc");
    cudaError_t e = cudaSuccess;
    void *scratch = noalloc_scratch(&e);
    if (!scratch) return cuda_status(e == cudaSuccess ? cudaErrorInvalidSymbol : e,
                                     "dcn_core_forward_proj_noalloc scratch address");
    // the workspace route of dcn_core_forward_proj with the fixed array as workspace
    return proj_call(p, Cout, x, offset, mask, weight, bias, out, scratch, (int64_t)kNoAllocScratchBytes, stream,
                     false, "dcn_core_forward_proj_noalloc launch");
}

int64_t dcn_core_forward_proj_workspace_bytes(const dcn_params *p) {
    const long long n = core_out_bytes(p);
    if (n < 0) fail(DCN_ERR_SHAPE, "invalid params");
    return n;
}

dcn_status dcn_deform_conv_forward(const dcn_params *p, int32_t Cout, const void *x, const void *offset,
                                   const void *mask, const void *weight, const void *bias, void *out,
                                   dcn_stream_t stream) {
    return proj_call(p, Cout, x, offset, mask, weight, bias, out, nullptr, 0, stream, true,
                     "dcn_deform_conv_forward launch");
}

dcn_status dcn_core_backward(const dcn_params *p, const void *x, const void *offset, const void *mask,
                             const void *grad_out, void *grad_x, void *grad_offset, void *grad_mask,
                             dcn_stream_t stream) {
    int Ho = 0, Wo = 0;
    dcn_status s = check_core(p, &Ho, &Wo);
    if (s != DCN_OK) return s;
    if (p->B == 0) return DCN_OK;
    if (!x || !offset || !mask || !grad_out || !grad_x || !grad_offset || !grad_mask)
        return fail(DCN_ERR_NULL, "x, offset, mask, grad_out and the three gradients are required");
    const size_t es = dtype_size(p->dtype);
    if (!aligned(x, 16) || !aligned(grad_out, 16) || !aligned(grad_x, 16))
        return fail(DCN_ERR_ALIGN, "x, grad_out and grad_x must be 16-byte aligned");
    if (!aligned(offset, 2 * es) || !aligned(mask, es) || !aligned(grad_offset, 2 * es) || !aligned(grad_mask, es))
        return fail(DCN_ERR_ALIGN, "offset/grad_offset need 2*sizeof(dtype), mask/grad_mask sizeof(dtype) alignment");
    if (p->mask_mode == DCN_MASK_SOFTMAX && p->kh * p->kw > dcnb::kMaxSoftmaxK)
        return fail(DCN_ERR_UNSUPPORTED, "softmax-mode backward supports K <= %d", dcnb::kMaxSoftmaxK);
    dcnb::CoreArgs a = core_args(p, Ho, Wo);
    a.x = x; a.offset = offset; a.mask = mask; a.grad_out = grad_out;
    a.grad_x = grad_x; a.grad_offset = grad_offset; a.grad_mask = grad_mask;
    bool handled = false;
    cudaError_t e = cudaSuccess;
    const char *force = getenv("DCN_B200_FORCE_GENERIC");
    if (!(force && force[0] == '1')) e = dcnb::launch_core_backward_staged(a, (cudaStream_t)stream, &handled);
    if (!handled) e = dcnb::launch_core_backward_generic(a, (cudaStream_t)stream);
    return cuda_status(e, "dcn_core_backward launch");
}

dcn_status deform_agg_forward(const dagg_params *p, const void *feat, const int32_t *spatial_shape,
                              const int32_t *scale_start_index, const float *sampling_location,
                              const void *weights, void *out, dcn_stream_t stream) {
    dcn_status s = check_agg(p);
    if (s != DCN_OK) return s;
    if (p->B == 0 || p->num_anchors == 0) return DCN_OK;
    if (!feat || !spatial_shape || !scale_start_index || !sampling_location || !weights || !out)
        return fail(DCN_ERR_NULL, "all tensor pointers are required");
    const size_t es = dtype_size(p->dtype);
    if (!aligned(feat, 16) || !aligned(out, 16)) return fail(DCN_ERR_ALIGN, "feat and out must be 16-byte aligned");
    if (!aligned(sampling_location, 8) || !aligned(weights, es) || !aligned(spatial_shape, 4) ||
        !aligned(scale_start_index, 4))
        return fail(DCN_ERR_ALIGN, "sampling_location needs 8-byte, weights sizeof(dtype), tables 4-byte alignment");
    dcnb::AggArgs a = agg_args(p);
    a.feat = feat; a.spatial_shape = spatial_shape; a.scale_start = scale_start_index;
    a.loc = sampling_location; a.weights = weights; a.out = out;
    return cuda_status(dcnb::launch_agg_forward(a, (cudaStream_t)stream), "deform_agg_forward launch");
}

dcn_status deform_roi_pool_forward(const droi_params *p, const void *x, const float *rois, const float *offset,
                                   void *out, dcn_stream_t stream) {
    if (!p) return fail(DCN_ERR_NULL, "params is NULL");
    if (p->dtype < DCN_F32 || p->dtype > DCN_BF16) return fail(DCN_ERR_UNSUPPORTED, "dtype %d", p->dtype);
    if (p->B < 1 || p->H < 1 || p->W < 1 || p->C < 1 || p->num_rois < 0 || p->pooled_h < 1 || p->pooled_w < 1 ||
        p->sampling < 1)
        return fail(DCN_ERR_SHAPE, "sizes must be positive (num_rois may be 0)");
    if (p->B > kMaxDim || p->H > kMaxDim || p->W > kMaxDim || p->C > 65536 || p->pooled_h > 1024 ||
        p->pooled_w > 1024 || p->sampling > 64 || p->num_rois > (1 << 24))
        return fail(DCN_ERR_SHAPE, "a size exceeds its limit");
    if (!isfinite(p->spatial_scale) || !isfinite(p->gamma)) return fail(DCN_ERR_SHAPE, "scale/gamma not finite");
    if ((long long)p->num_rois * p->pooled_h * p->pooled_w > (1LL << 31))
        return fail(DCN_ERR_SHAPE, "num_rois * pooled_h * pooled_w exceeds 2^31");
    if (((size_t)p->C * dtype_size(p->dtype)) % 16 != 0)
        return fail(DCN_ERR_UNSUPPORTED, "C*sizeof(dtype) must be a multiple of 16 bytes");
    if (p->num_rois == 0) return DCN_OK;
    if (!x || !rois || !offset || !out) return fail(DCN_ERR_NULL, "x, rois, offset and out are required");
    if (!aligned(x, 16) || !aligned(out, 16)) return fail(DCN_ERR_ALIGN, "x and out must be 16-byte aligned");
    if (!aligned(rois, 4) || !aligned(offset, 8)) return fail(DCN_ERR_ALIGN, "rois 4-byte, offset 8-byte alignment");
    dcnb::RoiArgs a;
    a.x = x; a.rois = rois; a.offset = offset; a.out = out;
    a.B = p->B; a.H = p->H; a.W = p->W; a.C = p->C; a.N = p->num_rois;
    a.PH = p->pooled_h; a.PW = p->pooled_w; a.S = p->sampling;
    a.spatial_scale = p->spatial_scale; a.gamma = p->gamma;
    a.dtype = (dcnb::DType)p->dtype;
    return cuda_status(dcnb::launch_roi_pool_forward(a, (cudaStream_t)stream), "deform_roi_pool_forward launch");
}

dcn_status deform_agg_backward(const dagg_params *p, const void *feat, const int32_t *spatial_shape,
                               const int32_t *scale_start_index, const float *sampling_location,
                               const void *weights, const void *grad_out, void *grad_feat, float *grad_loc,
                               void *grad_weights, dcn_stream_t stream) {
    dcn_status s = check_agg(p);
    if (s != DCN_OK) return s;
    if (p->B == 0 || p->num_anchors == 0) return DCN_OK;
    if (!feat || !spatial_shape || !scale_start_index || !sampling_location || !weights || !grad_out ||
        !grad_feat || !grad_loc || !grad_weights)
        return fail(DCN_ERR_NULL, "all tensor pointers are required");
    const size_t es = dtype_size(p->dtype);
    if (!aligned(feat, 16) || !aligned(grad_out, 16) || !aligned(grad_feat, 16))
        return fail(DCN_ERR_ALIGN, "feat, grad_out and grad_feat must be 16-byte aligned");
    if (!aligned(sampling_location, 8) || !aligned(grad_loc, 8) || !aligned(weights, es) ||
        !aligned(grad_weights, es) || !aligned(spatial_shape, 4) || !aligned(scale_start_index, 4))
        return fail(DCN_ERR_ALIGN, "locations need 8-byte, weights sizeof(dtype), tables 4-byte alignment");
    dcnb::AggArgs a = agg_args(p);
    a.feat = feat; a.spatial_shape = spatial_shape; a.scale_start = scale_start_index;
    a.loc = sampling_location; a.weights = weights; a.grad_out = grad_out;
    a.grad_feat = grad_feat; a.grad_loc = grad_loc; a.grad_weights = grad_weights;
    return cuda_status(dcnb::launch_agg_backward(a, (cudaStream_t)stream), "deform_agg_backward launch");
}

}  // extern "C"
