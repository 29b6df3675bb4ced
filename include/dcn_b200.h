/*
 * dcn_b200.h - C ABI of the B200 (sm_100a) deformable sampling-aggregation
 * library.
 *
 * The operator.  For every output pixel p and channel group g, K kernel
 * points are sampled at p0 + pk + dpk, where pk is the regular kernel grid
 * and dpk a learned fractional offset ("用PyTorch实战DCNv1：从零构建可变形卷积与ROI池化模块",
 * section 1: y(p0) = sum_n w(pn) x(p0 + pn + dpn)).  Each sample is a bilinear
 * interpolation of the NHWC input (same page, section 2:
 * x(p) = sum_q G(q,p) x(q), G(q,p) = g(qx,px) g(qy,py), g(a,b) = max(0, 1-|a-b|),
 * grid points outside the map hold zero).  Each sample is weighted by a
 * per-point modulation (DCNv2 page "DCNv2实战：在YOLOv5中替换普通卷积...", section 1:
 * sum_n m(pn) w(pn) x(p + pn + dpn)), either normalised by a softmax over the K
 * points of the (pixel, group) as in DCNv3 or used raw as in DCNv4 (YOLOv11 +
 * DCNv4 article, section 1.1), and the K samples are summed in fp32.  The
 * pointwise projection that follows the core in the DCNv4 module (1x1
 * convolution with bias) is available fused with it (dcn_core_forward_proj),
 * and so is the dense per-point weight w(pn) of DCNv1/v2 (the modulated
 * deformable convolution, dcn_deform_conv_forward).
 *
 * Conventions shared by every call:
 *   - All tensor pointers are DEVICE pointers to dense, C-contiguous buffers
 *     owned by the caller.  The library never allocates or frees memory.
 *   - Calls are asynchronous on `stream` (0 = the legacy default stream)
 *     and never synchronise.  A non-OK status means nothing was enqueued,
 *     except DCN_ERR_CUDA after a failed launch.
 *   - Every argument check runs on the host before any launch; a failed
 *     check returns its status and touches no memory.
 *   - x, offset, mask, out (and the gradients) share the storage dtype given
 *     in the params; accumulation is fp32; results are rounded once,
 *     nearest-even, to the storage dtype.
 *   - Layouts (row-major, last index fastest):
 *       x      [B, H, W, G*C]          channel = g*C + c
 *       offset [B, Ho, Wo, G, K, 2]    last dim (dx, dy) in input pixels
 *       mask   [B, Ho, Wo, G, K]       raw modulation, or logits (softmax mode)
 *       out    [B, Ho, Wo, G*C]
 *     with K = kh*kw, kernel point k = i*kw + j (i along H),
 *     Ho = (H + 2*pad_h - (dil_h*(kh-1) + 1)) / stride_h + 1 (floor), and
 *     likewise Wo.  Kernel point (i,j) of output (ho,wo) samples
 *       y = ho*stride_h - pad_h + i*dil_h + offset_scale*dy,
 *       x = wo*stride_w - pad_w + j*dil_w + offset_scale*dx,
 *     formed in fp32 with one rounding (fused multiply-add).
 *   - A sampling position that is not a number makes its whole (pixel,
 *     group) output NaN; positions whose four grid neighbours all lie
 *     outside the map (including infinite ones) contribute exactly zero.
 *   - Supported group widths: C*sizeof(dtype) in {16, 32, 64, 128, 256}
 *     bytes, i.e. C in {4,8,16,32,64} for fp32 and {8,16,32,64,128} for
 *     fp16/bf16.  Other C return DCN_ERR_UNSUPPORTED.
 *   - x, out, grad_out and grad_x must be 16-byte aligned; offset and its
 *     gradient aligned to 2*sizeof(dtype); mask and its gradient to
 *     sizeof(dtype).  Otherwise DCN_ERR_ALIGN.
 *   - A problem with no output elements (B == 0) is a no-op returning DCN_OK;
 *     its pointers may be NULL.
 */
#ifndef DCN_B200_H
#define DCN_B200_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as cudaStream_t. */
typedef struct CUstream_st *dcn_stream_t;

typedef enum {
    DCN_OK = 0,
    DCN_ERR_NULL = 1,        /* a required pointer is NULL */
    DCN_ERR_SHAPE = 2,       /* inconsistent or non-positive sizes, Ho or Wo < 1 */
    DCN_ERR_UNSUPPORTED = 3, /* valid but not implemented (group width, dtype, mode) */
    DCN_ERR_ALIGN = 4,       /* a pointer is not aligned as required */
    DCN_ERR_CUDA = 5         /* the CUDA runtime reported an error at launch */
} dcn_status;

typedef enum { DCN_F32 = 0, DCN_F16 = 1, DCN_BF16 = 2 } dcn_dtype;

typedef enum {
    DCN_MASK_RAW = 0,    /* DCNv2/DCNv4: the mask is the modulation itself */
    DCN_MASK_SOFTMAX = 1 /* DCNv3: the mask holds logits, normalised over K */
} dcn_mask_mode;

typedef struct {
    int32_t B, H, W, G, C;   /* batch, input height/width, groups, channels per group */
    int32_t kh, kw;          /* kernel height/width */
    int32_t stride_h, stride_w;
    int32_t pad_h, pad_w;
    int32_t dil_h, dil_w;
    float offset_scale;      /* multiplies every offset (1.0 = offsets in pixels) */
    int32_t mask_mode;       /* dcn_mask_mode */
    int32_t dtype;           /* dcn_dtype: storage type of every tensor */
} dcn_params;

/* Output spatial size for `p`.  Returns DCN_ERR_SHAPE (and leaves the
 * outputs untouched) when the sizes are invalid or Ho/Wo would be < 1. */
dcn_status dcn_core_output_hw(const dcn_params *p, int32_t *Ho, int32_t *Wo);

/*
 * Forward core: out = sum_k m_k * bilinear(x, p_k) per (pixel, group).
 * Reads x, offset, mask; overwrites every element of out.
 * Two kernels implement it: a shared-memory staged one (group rows of 32 to
 * 256 bytes, W <= 254, K <= 25) and a generic one for every other shape.
 * Setting the environment variable DCN_B200_FORCE_GENERIC=1 routes every
 * call to the generic kernel (both give the same result up to fp32
 * summation order).
 */
dcn_status dcn_core_forward(const dcn_params *p, const void *x, const void *offset,
                            const void *mask, void *out, dcn_stream_t stream);

/*
 * Forward core followed by its pointwise projection (the DCNv4 module of the
 * YOLOv11 + DCNv4 article, section 3.2, passes the core's output through a
 * 1x1 convolution with bias):
 *   out[b, ho, wo, o] = bias[o] + sum_j weight[o, j] * core[b, ho, wo, j],
 *   j = g*C + c over the G*C core channels.
 *   weight [Cout, G*C]        storage dtype (a Conv2d weight without its 1x1 extent)
 *   bias   [Cout]             storage dtype, or NULL for no bias
 *   out    [B, Ho, Wo, Cout]  storage dtype
 * x, offset and mask are as for dcn_core_forward.  The core value of each
 * (pixel, channel) is accumulated in fp32 and rounded once to the storage
 * dtype (what dcn_core_forward would store); the projection runs on the
 * tensor cores with fp32 accumulation, adds the bias in fp32 and rounds the
 * result once.
 * workspace (optional): a caller-owned device buffer of at least
 * dcn_core_forward_proj_workspace_bytes(p) bytes (16-byte aligned).  With
 * it, the call enqueues two kernels: the core (the same kernels as
 * dcn_core_forward) writes its rounded output [B*Ho*Wo, G*C] into the
 * workspace, and a tensor-core GEMM projects it; this is the faster route
 * where the sampling gather dominates (the YOLO P4 shape).  Without it (NULL
 * or smaller), one fused kernel runs and the core never reaches device
 * memory.  Both routes compute the same values up to fp32 summation order.
 * The workspace holds the core output after the call.
 * Supported: fp16 and bf16 (fp32 returns DCN_ERR_UNSUPPORTED), C <= 64 with
 * G*C a multiple of 64 up to 512, kh*kw <= 25, Cout a multiple of 8 in
 * [8, 512], B*H*W and B*Ho*Wo below 2^31; both mask modes.  x, weight and out
 * 16-byte aligned, offset 4-byte, mask and bias 2-byte.  A NaN sampling
 * position makes every output channel of its pixel NaN.
 * DCN_ERR_SHAPE for a negative workspace_bytes.
 */
dcn_status dcn_core_forward_proj(const dcn_params *p, int32_t Cout, const void *x, const void *offset,
                                 const void *mask, const void *weight, const void *bias, void *out,
                                 void *workspace, int64_t workspace_bytes, dcn_stream_t stream);

/* Workspace bytes for the two-kernel route of dcn_core_forward_proj: the core
 * output, B*Ho*Wo*G*C*sizeof(dtype).  -1 for invalid params. */
int64_t dcn_core_forward_proj_workspace_bytes(const dcn_params *p);

/*
 * dcn_core_forward_proj for callers that cannot allocate device memory (this
 * entry point is the library's own addition; the pages have no counterpart).
 * Some callers have no way to obtain a workspace: a plugin hosted by a
 * framework or serving runtime whose allocator owns all of the GPU's memory
 * gets no handle to it, and a latency-critical loop cannot afford the
 * device-wide synchronisation that cudaMalloc implies.  This call allocates
 * nothing: it runs the workspace route of dcn_core_forward_proj (core kernel,
 * then the tensor-core GEMM) with a fixed scratch array of
 * DCN_NOALLOC_SCRATCH_BYTES (16 MiB) that the library holds in the memory of
 * every GPU that loads it, until the process exits.  The caller still owns
 * x, offset, mask, weight, bias and out, with the rules of
 * dcn_core_forward_proj.
 * Limit: the core output B*Ho*Wo*G*C*sizeof(dtype) must fit the array (the
 * DCNv4 P4 batch of 8 needs 13,107,200 bytes); a larger problem returns
 * DCN_ERR_UNSUPPORTED with a detail naming both sizes, before any launch.
 * Every call on a device shares the one array and leaves the core output of
 * its problem in it (every byte it reads is written by the same call first):
 * calls whose kernels overlap on the GPU, e.g. on two streams, race on it and
 * give wrong results; order them.  The first call on each device looks up the
 * array's device address (cudaGetSymbolAddress, once per device, with that
 * device current); make that first call before any stream capture.
 */
#define DCN_NOALLOC_SCRATCH_BYTES (16 * 1024 * 1024)
dcn_status dcn_core_forward_proj_noalloc(const dcn_params *p, int32_t Cout, const void *x, const void *offset,
                                         const void *mask, const void *weight, const void *bias, void *out,
                                         dcn_stream_t stream);

/*
 * Modulated deformable convolution with a dense weight per kernel point (the
 * DCNv2 page "DCNv2实战：在YOLOv5中替换普通卷积...", section 1:
 * y(p0) = sum_n w(pn) * x(p0 + pn + dpn) * dm_n; with unit masks it is the DCNv1
 * page's section-1 formula), in one kernel:
 *   out[b, ho, wo, o] = bias[o] + sum_k sum_j weight[o, k, j] * m_k * x_j(p_k),
 *   j = g*C + c; offset and modulation of point k shared by deformable group g.
 *   weight [Cout, K, G*C]     storage dtype (a Conv2d weight [Cout, G*C, kh, kw]
 *                             permuted to point-major)
 *   bias   [Cout]             storage dtype, or NULL
 *   out    [B, Ho, Wo, Cout]  storage dtype
 * x, offset and mask are as for dcn_core_forward (softmax mode normalises the
 * K masks of each (pixel, group) first).  Each sampled, modulated value is
 * formed in fp32 and rounded once to the storage dtype as the tensor-core
 * operand; the contraction over the K*G*C values accumulates in fp32.  The
 * K*G*C-wide column matrix never reaches device memory.  Same support,
 * alignment and error rules as dcn_core_forward_proj.
 */
dcn_status dcn_deform_conv_forward(const dcn_params *p, int32_t Cout, const void *x, const void *offset,
                                   const void *mask, const void *weight, const void *bias, void *out,
                                   dcn_stream_t stream);

/*
 * Backward core: gradients of L = <grad_out, out> with respect to x, offset
 * and mask.  The Sparse4D article (section 4.2) scatters the input gradient
 * with atomic adds and accumulates the position gradients per thread before
 * one write; this library does the same on the GPU.
 *   grad_x      [B, H, W, G*C]        m_k * G(q, p_k) * grad_out, summed over taps
 *   grad_offset [B, Ho, Wo, G, K, 2]  offset_scale * m_k * <grad_out, d x(p_k)/d p>
 *   grad_mask   [B, Ho, Wo, G, K]     <grad_out, x(p_k)>, through the softmax
 *                                     Jacobian m_k (g_k - sum_j m_j g_j) in
 *                                     softmax mode
 * All three are overwritten (grad_x is zeroed on `stream` first).  The
 * derivative of g at a grid line is taken from the right.  The order of the
 * atomic additions is not fixed, so grad_x may differ in the last bits from
 * run to run.  Supported: every dtype and both mask modes.
 */
dcn_status dcn_core_backward(const dcn_params *p, const void *x, const void *offset,
                             const void *mask, const void *grad_out, void *grad_x,
                             void *grad_offset, void *grad_mask, dcn_stream_t stream);

/*
 * Multi-camera, multi-scale deformable aggregation (Sparse4D
 * deformable_aggregation article, sections 1, 2.1 and 2.2).
 *   feat              [B, num_rows, G*C]   features of every camera and scale,
 *                     flattened: camera cam, scale s occupies rows
 *                     scale_start_index[cam][s] + y*W_s + x
 *   spatial_shape     [num_cams, num_scales, 2] int32 (H_s, W_s), device memory
 *   scale_start_index [num_cams, num_scales]    int32, device memory
 *   sampling_location [B, A, P, num_cams, 2]    fp32 (u, v), normalised to [0,1]
 *                     per camera; sampled at (u*W_s - 0.5, v*H_s - 0.5), fp32
 *   weights           [B, A, P, num_cams, num_scales, G], used as given
 *   out               [B, A, G*C]
 * out[b,a,g*C+c] = sum_{p,cam,s} weights[b,a,p,cam,s,g] * bilinear(map(cam,s), pos)[g*C+c].
 * Rows outside [0, num_rows) are never read: a table entry that points
 * there contributes zero.  feat, weights and out share `dtype`; locations
 * are always fp32.  Same group widths and alignment rules as the core.
 */
typedef struct {
    int32_t B, num_cams, num_scales, num_rows, num_anchors, num_pts, G, C;
    int32_t dtype; /* dcn_dtype */
} dagg_params;

dcn_status deform_agg_forward(const dagg_params *p, const void *feat,
                              const int32_t *spatial_shape, const int32_t *scale_start_index,
                              const float *sampling_location, const void *weights, void *out,
                              dcn_stream_t stream);

/*
 * Aggregation backward: gradients of <grad_out, out>.
 *   grad_feat    [B, num_rows, G*C]     scatter of weight * G(q,p) * grad_out (atomic)
 *   grad_loc     [B, A, P, num_cams, 2] fp32; sum over scales and groups of
 *                weight * W_s (resp. H_s) * <grad_out, d x / d px (resp. py)>
 *   grad_weights [B, A, P, num_cams, num_scales, G]  <grad_out, sample>
 * All three are overwritten (grad_feat is zeroed on `stream` first).
 */
dcn_status deform_agg_backward(const dagg_params *p, const void *feat,
                               const int32_t *spatial_shape, const int32_t *scale_start_index,
                               const float *sampling_location, const void *weights,
                               const void *grad_out, void *grad_feat, float *grad_loc,
                               void *grad_weights, dcn_stream_t stream);

/*
 * Deformable RoI pooling, forward ("用PyTorch实战DCNv1：从零构建可变形卷积与ROI池化模块",
 * section 3): bin (i, j) of region n is moved by
 * dp = gamma * dp_hat o (w, h) (the offset normalised by the region's width and
 * height) and averages S x S bilinear samples (zeros outside the map).
 *   x      [B, H, W, C]          NHWC, storage dtype
 *   rois   [N, 5] fp32           (batch index, x1, y1, x2, y2) in input-image units,
 *                                scaled by spatial_scale; a batch index outside
 *                                [0, B) reads nothing and yields zeros
 *   offset [N, PH, PW, 2] fp32   (dx_hat, dy_hat)
 *   out    [N, PH, PW, C]        storage dtype
 * Region size max(x2 - x1, 1) x max(y2 - y1, 1) after scaling; bin (i, j)
 * starts at (x1 + j*w/PW, y1 + i*h/PH); sample (sy, sx) sits at
 * + ((s + 0.5) * bin / S) + dp, pixel centres at integers; positions are
 * formed in fp32, one rounding per operation in that order.  A NaN position
 * makes its bin NaN.  C*sizeof(dtype) must be a multiple of 16 bytes (at most
 * 65536 channels), num_rois*PH*PW at most 2^31; x and out 16-byte aligned,
 * rois 4-byte, offset 8-byte.
 */
typedef struct {
    int32_t B, H, W, C;           /* input map */
    int32_t num_rois;             /* N */
    int32_t pooled_h, pooled_w;   /* PH, PW */
    int32_t sampling;             /* S >= 1 samples per bin side */
    float spatial_scale, gamma;
    int32_t dtype;                /* dcn_dtype */
} droi_params;

dcn_status deform_roi_pool_forward(const droi_params *p, const void *x, const float *rois,
                                   const float *offset, void *out, dcn_stream_t stream);

/* Static, human-readable name of a status. */
const char *dcn_status_string(dcn_status s);

/* Detail of the last non-OK status returned on the calling thread (which
 * check failed, or the CUDA error string).  Never NULL. */
const char *dcn_last_error_detail(void);

/* Device-side error word: kernels that wait on their own asynchronous
 * copies bound every wait (1 s); if one ran out the kernel sets bit 0 of this
 * word and returns without finishing its outputs.  This call synchronises
 * the device, returns the word and clears it; -1 if the read itself failed.
 * 0 after every normal run. */
int32_t dcn_take_device_error(void);

/* Self-test of the bounded-wait error path above (the pages have no
 * counterpart; it exists so that the failure path can be exercised without
 * a fault): enqueues on `stream` one thread that waits on a shared-memory
 * barrier nothing arrives on, for limit_us microseconds (1 .. 10^7).  The wait
 * gives up, the kernel sets bit 0 of the device error word and returns; the
 * next dcn_take_device_error() returns 1 and every later call works as
 * before.  DCN_ERR_SHAPE for a limit outside the range. */
dcn_status dcn_selftest_bounded_wait(int32_t limit_us, dcn_stream_t stream);

/*
 * On-chip rate probes: measurement support for the roofline of the sampling
 * kernels (the pages have no counterpart).  Runs probe number `probe` on one
 * CTA of 512 threads per SM, `reps` (1 .. 2^24) repetitions of its loop, on
 * `stream`:
 *    0  16-byte shared loads (bytes)
 *    1  chunk: two 16-byte shared loads of fp32 + 4 paired FMAs (chunks of 8 channels)
 *    2  fp32 FMAs                          3  paired fp32 FMAs (fma counted)
 *    4  chunk: 16-byte shared load of fp16 + 8 conversions + 8 FMAs (chunks)
 *    5  chunk: load + 8 fp16 conversions + 4 paired FMAs (chunks)
 *    6  chunk: load + bf16 widening by shift and mask + 4 paired FMAs (chunks)
 *    7  chunk: load + 8 fma.rn.f32.f16 with fp16 operands (chunks)
 *    8  16-byte global loads hitting L1 (bytes)
 *    9  gather, 4 lanes per 64-byte item (samples)
 *   10  gather, 8 lanes per item, paired FMAs (samples)
 *   11  gather, 8 lanes per item, FMAs (samples)
 *   12  integer lop3 (ops)
 *   13  32-byte global loads (ld.global.nc.v8.f32) hitting L1 (bytes)
 *   14  red.shared.add.f32, 32 distinct banks per warp (shared reductions)
 * dev_buf is a caller-owned device buffer of at least 36,864 bytes, 256-byte
 * aligned: on completion its first two 64-bit words hold the sum over the
 * CTAs of their SM-clock cycles and the number of CTAs (the rest is scratch
 * of the probe).  *units_per_cta receives the work of one CTA in *unit, so
 * units per SM per clock = units_per_cta * word[1] / word[0].
 * DCN_ERR_SHAPE for an unknown probe, reps out of range or a small buffer.
 */
dcn_status dcn_probe_rate(int32_t probe, int32_t reps, void *dev_buf, int64_t dev_buf_bytes,
                          double *units_per_cta, const char **unit, dcn_stream_t stream);

/* ABI version of this header (bumped on any incompatible change). */
int32_t dcn_abi_version(void);

#define DCN_ABI_VERSION 2

#ifdef __cplusplus
}
#endif

#endif /* DCN_B200_H */
