// Internal launcher interface between the C-ABI layer (dcn_abi.cu) and the
// kernels.  Arguments are validated by the ABI layer before any launcher runs.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace dcnb {

enum class DType : int { F32 = 0, F16 = 1, BF16 = 2 };

// Largest K for which the softmax-mode backward keeps per-point gradients.
constexpr int kMaxSoftmaxK = 49;

struct CoreArgs {
    const void *x;
    const void *offset;
    const void *mask;
    void *out;              // forward output
    const void *grad_out;   // backward only
    void *grad_x;           // backward only
    void *grad_offset;      // backward only
    void *grad_mask;        // backward only
    int B, H, W, G, C, kh, kw, sh, sw, ph, pw, dh, dw, Ho, Wo;
    float offset_scale;
    bool softmax;
    DType dtype;
};

// Forward core followed by its pointwise projection (fp16/bf16 only).
struct ProjArgs {
    CoreArgs core;       // core.out is the projected output [B, Ho, Wo, Cout]
    const void *weight;  // [Cout, G*C], or [Cout, K, G*C] when per_point
    const void *bias;    // [Cout] or nullptr
    int Cout;
    bool per_point;      // deformable convolution: a dense weight per kernel point
};

struct AggArgs {
    const void *feat;
    const int32_t *spatial_shape;
    const int32_t *scale_start;
    const float *loc;
    const void *weights;
    void *out;
    const void *grad_out;   // backward only
    void *grad_feat;        // backward only
    float *grad_loc;        // backward only
    void *grad_weights;     // backward only
    int B, cams, scales, rows, A, P, G, C;
    DType dtype;
};

struct RoiArgs {
    const void *x;       // [B, H, W, C]
    const float *rois;   // [N, 5]
    const float *offset; // [N, PH, PW, 2]
    void *out;           // [N, PH, PW, C]
    int B, H, W, C, N, PH, PW, S;
    float spatial_scale, gamma;
    DType dtype;
};

// Each launcher enqueues its kernel(s) on `stream` and returns the
// cudaGetLastError() of the launch.
cudaError_t launch_core_forward_generic(const CoreArgs &a, cudaStream_t stream);
cudaError_t launch_core_backward_generic(const CoreArgs &a, cudaStream_t stream);
// Staged backward (TMA row bands, per-tap records) for fp32 storage with 128-byte
// groups and K <= 9; *handled stays false for other shapes.
cudaError_t launch_core_backward_staged(const CoreArgs &a, cudaStream_t stream, bool *handled);
// Shared-memory path; sets *handled = false (and launches nothing) when the
// problem does not fit it.
cudaError_t launch_core_forward_plane(const CoreArgs &a, cudaStream_t stream, bool *handled);
// Reads and clears the device error word that bounded waits set (bit 0:
// a TMA wait ran out).  Synchronous.
cudaError_t take_device_error(unsigned int *value);
// One thread waits (bounded by limit_ns) on an mbarrier nothing arrives on.
cudaError_t launch_bounded_wait_selftest(long long limit_ns, cudaStream_t stream);
// Fused core + projection (tcgen05 GEMM on the core tile in shared memory).
cudaError_t launch_core_forward_proj(const ProjArgs &a, cudaStream_t stream);
// out[p, o] = bias[o] + sum_j core[p, j] * weight[o, j] on the tensor cores (fp16/bf16;
// core [P, KD], weight [Cout, KD], out [P, Cout]; KD a multiple of 64, Cout of 8 up to 512).
cudaError_t launch_proj_gemm(const void *core, const void *weight, const void *bias, void *out, long long P, int KD,
                             int Cout, DType dtype, cudaStream_t stream);
cudaError_t launch_agg_forward(const AggArgs &a, cudaStream_t stream);
// Anchor-wide aggregation kernels (all groups per CTA); sets *handled = false
// (and launches nothing) when the feature row width does not fit them.
cudaError_t launch_agg_wide(const AggArgs &a, bool bwd, cudaStream_t stream, bool *handled);
cudaError_t launch_agg_backward(const AggArgs &a, cudaStream_t stream);
cudaError_t launch_roi_pool_forward(const RoiArgs &a, cudaStream_t stream);

}  // namespace dcnb
