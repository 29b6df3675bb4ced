/*
 * Plain fp64 CPU oracle for the modulated deformable sampling-aggregation
 * core.  TEST INFRASTRUCTURE ONLY: the tests, the smoke check and the CPU
 * baseline leg of the benchmark call it; the product never does.  It shares
 * no code, header or constant with the CUDA library.
 *
 * What it computes, and where that is defined:
 *
 *   Deformable convolution sampling (DCNv1, "用PyTorch实战DCNv1：从零构建可变形
 *   卷积与ROI池化模块", section 1, the formula y(p0) = sum_n w(pn) x(p0+pn+dpn)):
 *   each output pixel p0 reads the input at the regular grid point p0+pn moved
 *   by a learned fractional offset dpn.
 *
 *   Bilinear interpolation (same page, section 2):
 *       x(p) = sum_q G(q,p) x(q),  G(q,p) = g(qx,px) g(qy,py),
 *       g(a,b) = max(0, 1 - |a-b|),
 *   the sum running over every integer grid point q; points outside the map
 *   hold zero.  g vanishes unless |a-b| < 1, so only the four grid points
 *   floor(p) + {0,1}^2 can contribute; the loops below visit exactly those and
 *   evaluate g itself on them.
 *
 *   Modulation (DCNv2, "DCNv2实战：在YOLOv5中替换普通卷积，目标检测精度能提升多少？",
 *   section 1: output(p) = sum m(pn) w(pn) x(p+pn+dpn)), grouped channels with
 *   a softmax over the K points (DCNv3) or the raw value (DCNv4) (YOLOv11 +
 *   DCNv4 article, section 1.1).
 *
 *   Multi-camera multi-scale aggregation (Sparse4D deformable_aggregation
 *   article, sections 1, 2.1 and 2.2).
 *
 *   The pointwise projection (1x1 convolution with bias) that follows the
 *   core in the DCNv4 module (YOLOv11 + DCNv4 article, section 3.2), and the
 *   modulated deformable convolution with a dense weight per kernel point
 *   (DCNv2 page, section 1; DCNv1 page, section 1).
 *
 * Readings where the pages are silent (each one is listed in the design notes):
 *   - base grid point of kernel point (i,j) at output (ho,wo):
 *       y = ho*stride_h - pad_h + i*dil_h,  x = wo*stride_w - pad_w + j*dil_w,
 *     point index k = i*kw + j; offsets are stored (dx, dy).
 *   - the sampling position p = base + offset_scale * d is formed in fp32 with
 *     one rounding (fmaf), the precision the GPU kernel uses, so that both
 *     sides take the same floor() decision; everything after it is fp64.
 *   - a sampling position that is not a number makes its whole (pixel, group)
 *     output not a number.
 *   - Sparse4D positions: p = loc * size - 0.5 (fp32, one rounding), rows laid
 *     out camera-major with per-(camera, scale) start indices.
 *   - derivatives of g at the kink (p exactly on a grid line) are one-sided
 *     from the right, consistent with the floor() support choice.
 *
 * Pins: closed-form identities, brute force over the whole grid, a library
 * bilinear sampler, finite differences and adjoint identities (see the
 * oracle tests).  Nothing in this file is unpinned.
 */
#include <math.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

int oracle_set_threads(int n)
{
#ifdef _OPENMP
    if (n > 0) omp_set_num_threads(n);
    return omp_get_max_threads();
#else
    (void)n;
    return 1;
#endif
}

/* g(a,b) = max(0, 1 - |a-b|), the one-dimensional bilinear kernel. */
static double g_kernel(double a, double b)
{
    double v = 1.0 - fabs(a - b);
    return v > 0.0 ? v : 0.0;
}

/* d g(q, p) / d p on the support q in {floor(p), floor(p)+1}, one-sided. */
static double g_kernel_dp(int q, int q_floor)
{
    return q == q_floor ? -1.0 : 1.0;
}

/* Modulation of the K points of one (pixel, group): raw or softmax over K. */
static void modulation(const double *logit, int K, int softmax, double *m)
{
    if (!softmax) {
        for (int k = 0; k < K; ++k) m[k] = logit[k];
        return;
    }
    double mx = -INFINITY;
    for (int k = 0; k < K; ++k) mx = logit[k] > mx ? logit[k] : mx;
    double s = 0.0;
    for (int k = 0; k < K; ++k) { m[k] = exp(logit[k] - mx); s += m[k]; }
    for (int k = 0; k < K; ++k) m[k] /= s;
}

/*
 * Forward core.
 *   x      [B, H, W, G*C]
 *   offset [B, Ho, Wo, G, K, 2]   (dx, dy)
 *   mask   [B, Ho, Wo, G, K]      logits if softmax != 0, else the modulation
 *   out    [B, Ho, Wo, G*C]
 */
void oracle_dcn_forward(int B, int H, int W, int G, int C, int kh, int kw,
                        int sh, int sw, int ph, int pw, int dh, int dw,
                        float offset_scale, int softmax,
                        const double *x, const double *offset, const double *mask,
                        double *out)
{
    const int K = kh * kw;
    const int Ho = (H + 2 * ph - (dh * (kh - 1) + 1)) / sh + 1;
    const int Wo = (W + 2 * pw - (dw * (kw - 1) + 1)) / sw + 1;

#pragma omp parallel for collapse(2) schedule(static)
    for (int b = 0; b < B; ++b)
        for (int ho = 0; ho < Ho; ++ho) {
            double *m = (double *)malloc(sizeof(double) * (size_t)K);
            for (int wo = 0; wo < Wo; ++wo)
                for (int g = 0; g < G; ++g) {
                    const size_t item = (((size_t)b * Ho + ho) * Wo + wo) * G + g;
                    double *y = out + item * C;
                    for (int c = 0; c < C; ++c) y[c] = 0.0;
                    modulation(mask + item * K, K, softmax, m);
                    int not_a_number = 0;
                    for (int i = 0; i < kh; ++i)
                        for (int j = 0; j < kw; ++j) {
                            const int k = i * kw + j;
                            const int by = ho * sh - ph + i * dh;
                            const int bx = wo * sw - pw + j * dw;
                            const double *d = offset + (item * K + k) * 2;
                            const float px = fmaf(offset_scale, (float)d[0], (float)bx);
                            const float py = fmaf(offset_scale, (float)d[1], (float)by);
                            if (isnan(px) || isnan(py)) { not_a_number = 1; continue; }
                            const double fy = floor((double)py), fx = floor((double)px);
                            if (!(fy >= -1.0 && fy <= H - 1 && fx >= -1.0 && fx <= W - 1))
                                continue; /* every q with G(q,p) != 0 lies outside the map */
                            const int y0 = (int)fy, x0 = (int)fx;
                            for (int qy = y0; qy <= y0 + 1; ++qy) {
                                if (qy < 0 || qy >= H) continue;
                                const double gy = g_kernel(qy, py);
                                for (int qx = x0; qx <= x0 + 1; ++qx) {
                                    if (qx < 0 || qx >= W) continue;
                                    const double Gq = g_kernel(qx, px) * gy;
                                    const double *xq = x + (((size_t)b * H + qy) * W + qx) * (size_t)G * C
                                                         + (size_t)g * C;
                                    for (int c = 0; c < C; ++c) y[c] += m[k] * Gq * xq[c];
                                }
                            }
                        }
                    if (not_a_number)
                        for (int c = 0; c < C; ++c) y[c] = NAN;
                }
            free(m);
        }
}

/*
 * Pointwise projection after the sampling core (the 1x1 convolution with bias
 * that the DCNv4 module of the YOLOv11 + DCNv4 article, section 3.2, applies
 * to the core's output):
 *     out[p, o] = bias[o] + sum_c Wt[o, c] * in[p, c]
 * for every pixel p of the NHWC map; Wt is [Cout, Cin] (a Conv2d weight with
 * its 1x1 spatial extent dropped); bias may be NULL (no bias).
 */
void oracle_pointwise_projection(long long npix, int Cin, int Cout, const double *in, const double *Wt,
                                 const double *bias, double *out)
{
#pragma omp parallel for schedule(static)
    for (long long p = 0; p < npix; ++p) {
        const double *v = in + (size_t)p * Cin;
        double *y = out + (size_t)p * Cout;
        for (int o = 0; o < Cout; ++o) {
            const double *w = Wt + (size_t)o * Cin;
            double s = bias ? bias[o] : 0.0;
            for (int c = 0; c < Cin; ++c) s += w[c] * v[c];
            y[o] = s;
        }
    }
}

/*
 * Modulated deformable convolution (DCNv2: "DCNv2实战：在YOLOv5中替换普通卷积..."
 * section 1, y(p0) = sum_n w(pn) * x(p0 + pn + dpn) * dm_n; DCNv1 page, section 1,
 * without the modulation): every kernel point k has its own dense weight
 * w_k[o, c] over the input channels,
 *     out[p, o] = bias[o] + sum_k sum_j weight[o, k, j] * m_k * x_j(p + p_k + dp_k),
 * j = g*C + c over the G*C input channels, the offset and modulation of point
 * k shared by the C channels of deformable group g (the same offset/mask
 * tensors and sampling as the core above).  weight is [Cout, K, G*C]; bias
 * may be NULL.  The sampled, modulated values of one output pixel are formed
 * first (K*G*C of them), then contracted with the weight.
 */
void oracle_deform_conv_forward(int B, int H, int W, int G, int C, int kh, int kw,
                                int sh, int sw, int ph, int pw, int dh, int dw,
                                float offset_scale, int softmax, int Cout,
                                const double *x, const double *offset, const double *mask,
                                const double *weight, const double *bias, double *out)
{
    const int K = kh * kw;
    const int GC = G * C;
    const int Ho = (H + 2 * ph - (dh * (kh - 1) + 1)) / sh + 1;
    const int Wo = (W + 2 * pw - (dw * (kw - 1) + 1)) / sw + 1;

#pragma omp parallel for collapse(2) schedule(static)
    for (int b = 0; b < B; ++b)
        for (int ho = 0; ho < Ho; ++ho) {
            double *col = (double *)malloc(sizeof(double) * (size_t)K * GC);
            double *m = (double *)malloc(sizeof(double) * (size_t)K);
            for (int wo = 0; wo < Wo; ++wo) {
                for (int t = 0; t < K * GC; ++t) col[t] = 0.0;
                for (int g = 0; g < G; ++g) {
                    const size_t item = (((size_t)b * Ho + ho) * Wo + wo) * G + g;
                    modulation(mask + item * K, K, softmax, m);
                    for (int i = 0; i < kh; ++i)
                        for (int j = 0; j < kw; ++j) {
                            const int k = i * kw + j;
                            double *ck = col + (size_t)k * GC + (size_t)g * C;
                            const int by = ho * sh - ph + i * dh;
                            const int bx = wo * sw - pw + j * dw;
                            const double *d = offset + (item * K + k) * 2;
                            const float px = fmaf(offset_scale, (float)d[0], (float)bx);
                            const float py = fmaf(offset_scale, (float)d[1], (float)by);
                            if (isnan(px) || isnan(py)) {
                                for (int c = 0; c < C; ++c) ck[c] = NAN;
                                continue;
                            }
                            const double fy = floor((double)py), fx = floor((double)px);
                            if (!(fy >= -1.0 && fy <= H - 1 && fx >= -1.0 && fx <= W - 1)) continue;
                            const int y0 = (int)fy, x0 = (int)fx;
                            for (int qy = y0; qy <= y0 + 1; ++qy) {
                                if (qy < 0 || qy >= H) continue;
                                const double gy = g_kernel(qy, py);
                                for (int qx = x0; qx <= x0 + 1; ++qx) {
                                    if (qx < 0 || qx >= W) continue;
                                    const double Gq = g_kernel(qx, px) * gy;
                                    const double *xq = x + (((size_t)b * H + qy) * W + qx) * (size_t)GC
                                                         + (size_t)g * C;
                                    for (int c = 0; c < C; ++c) ck[c] += m[k] * Gq * xq[c];
                                }
                            }
                        }
                }
                double *y = out + (((size_t)b * Ho + ho) * Wo + wo) * (size_t)Cout;
                for (int o = 0; o < Cout; ++o) {
                    const double *w = weight + (size_t)o * K * GC;
                    double acc = bias ? bias[o] : 0.0;
                    for (int t = 0; t < K * GC; ++t) acc += w[t] * col[t];
                    y[o] = acc;
                }
            }
            free(col);
            free(m);
        }
}

/*
 * Backward core: gradients of L = <grad_out, out> with respect to x, offset
 * and mask (the logits in softmax mode).  The input gradient is the scatter
 * of m_k G(q,p) grad_out onto the four corners; the offset gradient is
 * offset_scale * m_k * sum_c grad_out_c * d x_c(p) / d p; the mask gradient is
 * sum_c grad_out_c * x_c(p), passed through the softmax Jacobian
 * m_k (g_k - sum_j m_j g_j) in softmax mode.  All three outputs are
 * overwritten.
 */
void oracle_dcn_backward(int B, int H, int W, int G, int C, int kh, int kw,
                         int sh, int sw, int ph, int pw, int dh, int dw,
                         float offset_scale, int softmax,
                         const double *x, const double *offset, const double *mask,
                         const double *grad_out,
                         double *grad_x, double *grad_offset, double *grad_mask)
{
    const int K = kh * kw;
    const int Ho = (H + 2 * ph - (dh * (kh - 1) + 1)) / sh + 1;
    const int Wo = (W + 2 * pw - (dw * (kw - 1) + 1)) / sw + 1;
    memset(grad_x, 0, sizeof(double) * (size_t)B * H * W * G * C);

    /* grad_x[b, :, :, g*C:(g+1)*C] only receives from items of the same
     * (b, g), so the (b, g) planes are independent. */
#pragma omp parallel for collapse(2) schedule(dynamic)
    for (int b = 0; b < B; ++b)
        for (int g = 0; g < G; ++g) {
            double *m = (double *)malloc(sizeof(double) * (size_t)K);
            double *gm = (double *)malloc(sizeof(double) * (size_t)K);
            for (int ho = 0; ho < Ho; ++ho)
                for (int wo = 0; wo < Wo; ++wo) {
                    const size_t item = (((size_t)b * Ho + ho) * Wo + wo) * G + g;
                    const double *go = grad_out + item * C;
                    modulation(mask + item * K, K, softmax, m);
                    for (int i = 0; i < kh; ++i)
                        for (int j = 0; j < kw; ++j) {
                            const int k = i * kw + j;
                            const int by = ho * sh - ph + i * dh;
                            const int bx = wo * sw - pw + j * dw;
                            const double *d = offset + (item * K + k) * 2;
                            double *gd = grad_offset + (item * K + k) * 2;
                            const float px = fmaf(offset_scale, (float)d[0], (float)bx);
                            const float py = fmaf(offset_scale, (float)d[1], (float)by);
                            gd[0] = gd[1] = 0.0;
                            gm[k] = 0.0;
                            if (isnan(px) || isnan(py)) { gd[0] = gd[1] = gm[k] = NAN; continue; }
                            const double fy = floor((double)py), fx = floor((double)px);
                            if (!(fy >= -1.0 && fy <= H - 1 && fx >= -1.0 && fx <= W - 1)) continue;
                            const int y0 = (int)fy, x0 = (int)fx;
                            double dpx = 0.0, dpy = 0.0, val = 0.0;
                            for (int qy = y0; qy <= y0 + 1; ++qy) {
                                if (qy < 0 || qy >= H) continue;
                                const double gy = g_kernel(qy, py);
                                const double dgy = g_kernel_dp(qy, y0);
                                for (int qx = x0; qx <= x0 + 1; ++qx) {
                                    if (qx < 0 || qx >= W) continue;
                                    const double gx = g_kernel(qx, px);
                                    const double dgx = g_kernel_dp(qx, x0);
                                    const size_t row = (((size_t)b * H + qy) * W + qx) * (size_t)G * C
                                                       + (size_t)g * C;
                                    const double *xq = x + row;
                                    double *gxq = grad_x + row;
                                    for (int c = 0; c < C; ++c) {
                                        val += go[c] * gx * gy * xq[c];
                                        dpx += go[c] * dgx * gy * xq[c];
                                        dpy += go[c] * gx * dgy * xq[c];
                                        gxq[c] += m[k] * gx * gy * go[c];
                                    }
                                }
                            }
                            gm[k] = val;
                            gd[0] = (double)offset_scale * m[k] * dpx;
                            gd[1] = (double)offset_scale * m[k] * dpy;
                        }
                    double *gl = grad_mask + item * K;
                    if (!softmax) {
                        for (int k = 0; k < K; ++k) gl[k] = gm[k];
                    } else {
                        double dot = 0.0;
                        for (int k = 0; k < K; ++k) dot += m[k] * gm[k];
                        for (int k = 0; k < K; ++k) gl[k] = m[k] * (gm[k] - dot);
                    }
                }
            free(m);
            free(gm);
        }
}

/*
 * Error budget of an input gradient summed by atomic additions: for every
 * grad_x element, the sum of the absolute values of its contributions
 * |m_k G(q,p) grad_out_c| (abs_sum, [B,H,W,G*C]) and how many contributions it
 * receives (terms, [B,H,W,G], the same for every channel of a group).  When a
 * device adds the contributions one by one in a storage precision with unit
 * roundoff u, each partial sum and each contribution is rounded once, and the
 * recursive-summation bound (Higham, "Accuracy and Stability of Numerical
 * Algorithms", 2nd ed., section 4.2) limits the error of the stored result to
 * gamma_(n+1) * abs_sum, gamma_m = m u / (1 - m u), n = terms: whatever the
 * order in which the atomics land.  The taps are enumerated exactly as in
 * oracle_dcn_backward.
 */
void oracle_dcn_grad_x_budget(int B, int H, int W, int G, int C, int kh, int kw,
                              int sh, int sw, int ph, int pw, int dh, int dw,
                              float offset_scale, int softmax,
                              const double *offset, const double *mask, const double *grad_out,
                              double *abs_sum, double *terms)
{
    const int K = kh * kw;
    const int Ho = (H + 2 * ph - (dh * (kh - 1) + 1)) / sh + 1;
    const int Wo = (W + 2 * pw - (dw * (kw - 1) + 1)) / sw + 1;
    memset(abs_sum, 0, sizeof(double) * (size_t)B * H * W * G * C);
    memset(terms, 0, sizeof(double) * (size_t)B * H * W * G);
#pragma omp parallel for collapse(2) schedule(dynamic)
    for (int b = 0; b < B; ++b)
        for (int g = 0; g < G; ++g) {
            double *m = (double *)malloc(sizeof(double) * (size_t)K);
            for (int ho = 0; ho < Ho; ++ho)
                for (int wo = 0; wo < Wo; ++wo) {
                    const size_t item = (((size_t)b * Ho + ho) * Wo + wo) * G + g;
                    const double *go = grad_out + item * C;
                    modulation(mask + item * K, K, softmax, m);
                    for (int i = 0; i < kh; ++i)
                        for (int j = 0; j < kw; ++j) {
                            const int k = i * kw + j;
                            const int by = ho * sh - ph + i * dh;
                            const int bx = wo * sw - pw + j * dw;
                            const double *d = offset + (item * K + k) * 2;
                            const float px = fmaf(offset_scale, (float)d[0], (float)bx);
                            const float py = fmaf(offset_scale, (float)d[1], (float)by);
                            if (isnan(px) || isnan(py)) continue;
                            const double fy = floor((double)py), fx = floor((double)px);
                            if (!(fy >= -1.0 && fy <= H - 1 && fx >= -1.0 && fx <= W - 1)) continue;
                            const int y0 = (int)fy, x0 = (int)fx;
                            for (int qy = y0; qy <= y0 + 1; ++qy) {
                                if (qy < 0 || qy >= H) continue;
                                for (int qx = x0; qx <= x0 + 1; ++qx) {
                                    if (qx < 0 || qx >= W) continue;
                                    const double Gq = g_kernel(qx, px) * g_kernel(qy, py);
                                    const size_t pixel = ((size_t)b * H + qy) * W + qx;
                                    double *aq = abs_sum + pixel * (size_t)G * C + (size_t)g * C;
                                    for (int c = 0; c < C; ++c) aq[c] += fabs(m[k] * Gq * go[c]);
                                    terms[pixel * G + g] += 1.0;
                                }
                            }
                        }
                }
            free(m);
        }
}

/*
 * Multi-camera multi-scale deformable aggregation, forward.
 *   feat    [B, rows, G*C]; camera cam, scale s occupies rows
 *           start[cam*S + s] + y*W_s + x for its H_s x W_s map
 *   shape   [cams, S, 2]  (H_s, W_s) per camera and scale
 *   loc     [B, A, P, cams, 2]  normalised (u, v) in [0,1] per camera (fp32)
 *   weights [B, A, P, cams, S, G]
 *   out     [B, A, G*C]
 * out[b,a,g*C+c] = sum_{p,cam,s} weights * x_{cam,s}(u*W_s - 0.5, v*H_s - 0.5)[g*C+c]
 */
void oracle_agg_forward(int B, int cams, int S, int rows, int A, int P, int G, int C,
                        const double *feat, const int *shape, const int *start,
                        const float *loc, const double *weights, double *out)
{
#pragma omp parallel for collapse(2) schedule(static)
    for (int b = 0; b < B; ++b)
        for (int a = 0; a < A; ++a)
            for (int g = 0; g < G; ++g) {
                double *y = out + (((size_t)b * A + a) * G + g) * C;
                for (int c = 0; c < C; ++c) y[c] = 0.0;
                int not_a_number = 0;
                for (int p = 0; p < P; ++p)
                    for (int cam = 0; cam < cams; ++cam) {
                        const float *l = loc + ((((size_t)b * A + a) * P + p) * cams + cam) * 2;
                        for (int s = 0; s < S; ++s) {
                            const int Hs = shape[(cam * S + s) * 2 + 0];
                            const int Ws = shape[(cam * S + s) * 2 + 1];
                            const float px = fmaf(l[0], (float)Ws, -0.5f);
                            const float py = fmaf(l[1], (float)Hs, -0.5f);
                            const double w = weights[(((((size_t)b * A + a) * P + p) * cams + cam) * S + s) * G + g];
                            if (isnan(px) || isnan(py)) { not_a_number = 1; continue; }
                            const double fy = floor((double)py), fx = floor((double)px);
                            if (!(fy >= -1.0 && fy <= Hs - 1 && fx >= -1.0 && fx <= Ws - 1)) continue;
                            const int y0 = (int)fy, x0 = (int)fx;
                            for (int qy = y0; qy <= y0 + 1; ++qy) {
                                if (qy < 0 || qy >= Hs) continue;
                                const double gy = g_kernel(qy, py);
                                for (int qx = x0; qx <= x0 + 1; ++qx) {
                                    if (qx < 0 || qx >= Ws) continue;
                                    const double Gq = g_kernel(qx, px) * gy;
                                    const size_t row = (size_t)start[cam * S + s] + (size_t)qy * Ws + qx;
                                    const double *f = feat + ((size_t)b * rows + row) * (size_t)G * C
                                                      + (size_t)g * C;
                                    for (int c = 0; c < C; ++c) y[c] += w * Gq * f[c];
                                }
                            }
                        }
                    }
                if (not_a_number)
                    for (int c = 0; c < C; ++c) y[c] = NAN;
            }
    (void)rows;
}

/*
 * Multi-camera aggregation, backward: gradients of <grad_out, out> with
 * respect to feat (scatter), the sampling locations and the weights.
 * grad_loc[.., 0] = sum_{s,g} w * W_s * sum_c grad_out_c d x_c / d px, and
 * likewise with H_s for the second coordinate.  All outputs are overwritten.
 */
void oracle_agg_backward(int B, int cams, int S, int rows, int A, int P, int G, int C,
                         const double *feat, const int *shape, const int *start,
                         const float *loc, const double *weights, const double *grad_out,
                         double *grad_feat, double *grad_loc, double *grad_weights)
{
    memset(grad_feat, 0, sizeof(double) * (size_t)B * rows * G * C);
    memset(grad_loc, 0, sizeof(double) * (size_t)B * A * P * cams * 2);
    /* Columns g*C..(g+1)*C of grad_feat only receive from group g, so the
     * (b, g) slices are independent; grad_loc sums over groups, so each
     * group writes a private copy that is reduced afterwards. */
    double *gl_part = (double *)calloc((size_t)G * B * A * P * cams * 2, sizeof(double));
#pragma omp parallel for collapse(2) schedule(dynamic)
    for (int b = 0; b < B; ++b)
        for (int g = 0; g < G; ++g) {
            double *glp = gl_part + (size_t)g * B * A * P * cams * 2;
            for (int a = 0; a < A; ++a) {
                const double *go = grad_out + (((size_t)b * A + a) * G + g) * C;
                for (int p = 0; p < P; ++p)
                    for (int cam = 0; cam < cams; ++cam) {
                        const size_t li = ((((size_t)b * A + a) * P + p) * cams + cam) * 2;
                        const float *l = loc + li;
                        for (int s = 0; s < S; ++s) {
                            const int Hs = shape[(cam * S + s) * 2 + 0];
                            const int Ws = shape[(cam * S + s) * 2 + 1];
                            const float px = fmaf(l[0], (float)Ws, -0.5f);
                            const float py = fmaf(l[1], (float)Hs, -0.5f);
                            const size_t wi = (((((size_t)b * A + a) * P + p) * cams + cam) * S + s) * G + g;
                            const double w = weights[wi];
                            grad_weights[wi] = 0.0;
                            if (isnan(px) || isnan(py)) {
                                grad_weights[wi] = NAN;
                                glp[li] = glp[li + 1] = NAN;
                                continue;
                            }
                            const double fy = floor((double)py), fx = floor((double)px);
                            if (!(fy >= -1.0 && fy <= Hs - 1 && fx >= -1.0 && fx <= Ws - 1)) continue;
                            const int y0 = (int)fy, x0 = (int)fx;
                            double val = 0.0, dpx = 0.0, dpy = 0.0;
                            for (int qy = y0; qy <= y0 + 1; ++qy) {
                                if (qy < 0 || qy >= Hs) continue;
                                const double gy = g_kernel(qy, py);
                                const double dgy = g_kernel_dp(qy, y0);
                                for (int qx = x0; qx <= x0 + 1; ++qx) {
                                    if (qx < 0 || qx >= Ws) continue;
                                    const double gx = g_kernel(qx, px);
                                    const double dgx = g_kernel_dp(qx, x0);
                                    const size_t row = (size_t)start[cam * S + s] + (size_t)qy * Ws + qx;
                                    const size_t off = ((size_t)b * rows + row) * (size_t)G * C + (size_t)g * C;
                                    for (int c = 0; c < C; ++c) {
                                        val += go[c] * gx * gy * feat[off + c];
                                        dpx += go[c] * dgx * gy * feat[off + c];
                                        dpy += go[c] * gx * dgy * feat[off + c];
                                        grad_feat[off + c] += w * gx * gy * go[c];
                                    }
                                }
                            }
                            grad_weights[wi] = val;
                            glp[li + 0] += w * dpx * Ws;
                            glp[li + 1] += w * dpy * Hs;
                        }
                    }
            }
        }
    const size_t nl = (size_t)B * A * P * cams * 2;
    for (int g = 0; g < G; ++g)
        for (size_t i = 0; i < nl; ++i) grad_loc[i] += gl_part[(size_t)g * nl + i];
    free(gl_part);
}

/*
 * Error budget of the aggregation's feature gradient, summed by atomic
 * additions on a device: per grad_feat element the sum of the absolute values
 * of its contributions |w G(q,p) grad_out_c| (abs_sum, [B, rows, G*C]) and how
 * many it receives (terms, [B, rows, G]); see oracle_dcn_grad_x_budget for the
 * bound these give.  The samples are enumerated exactly as in
 * oracle_agg_backward.
 */
void oracle_agg_grad_feat_budget(int B, int cams, int S, int rows, int A, int P, int G, int C,
                                 const int *shape, const int *start, const float *loc,
                                 const double *weights, const double *grad_out,
                                 double *abs_sum, double *terms)
{
    memset(abs_sum, 0, sizeof(double) * (size_t)B * rows * G * C);
    memset(terms, 0, sizeof(double) * (size_t)B * rows * G);
#pragma omp parallel for collapse(2) schedule(dynamic)
    for (int b = 0; b < B; ++b)
        for (int g = 0; g < G; ++g)
            for (int a = 0; a < A; ++a) {
                const double *go = grad_out + (((size_t)b * A + a) * G + g) * C;
                for (int p = 0; p < P; ++p)
                    for (int cam = 0; cam < cams; ++cam) {
                        const float *l = loc + ((((size_t)b * A + a) * P + p) * cams + cam) * 2;
                        for (int s = 0; s < S; ++s) {
                            const int Hs = shape[(cam * S + s) * 2 + 0];
                            const int Ws = shape[(cam * S + s) * 2 + 1];
                            const float px = fmaf(l[0], (float)Ws, -0.5f);
                            const float py = fmaf(l[1], (float)Hs, -0.5f);
                            const double w = weights[(((((size_t)b * A + a) * P + p) * cams + cam) * S + s) * G + g];
                            if (isnan(px) || isnan(py)) continue;
                            const double fy = floor((double)py), fx = floor((double)px);
                            if (!(fy >= -1.0 && fy <= Hs - 1 && fx >= -1.0 && fx <= Ws - 1)) continue;
                            const int y0 = (int)fy, x0 = (int)fx;
                            for (int qy = y0; qy <= y0 + 1; ++qy) {
                                if (qy < 0 || qy >= Hs) continue;
                                for (int qx = x0; qx <= x0 + 1; ++qx) {
                                    if (qx < 0 || qx >= Ws) continue;
                                    const double Gq = g_kernel(qx, px) * g_kernel(qy, py);
                                    const size_t row = (size_t)b * rows + (size_t)start[cam * S + s] +
                                                       (size_t)qy * Ws + qx;
                                    double *aq = abs_sum + row * (size_t)G * C + (size_t)g * C;
                                    for (int c = 0; c < C; ++c) aq[c] += fabs(w * Gq * go[c]);
                                    terms[row * G + g] += 1.0;
                                }
                            }
                        }
                    }
            }
}

/*
 * Deformable RoI pooling, forward ("用PyTorch实战DCNv1：从零构建可变形卷积与ROI池化模块",
 * section 3): the k x k bins of a region of interest are each moved by a
 * learned offset normalised by the region size, dp = gamma * dp_hat o (w, h),
 * and each bin's value is read by bilinear interpolation (the same kernel
 * g(a,b) = max(0, 1-|a-b|) as the core, zeros outside the map).
 *   x      [B, H, W, C]
 *   rois   [N, 5]      (batch index, x1, y1, x2, y2) in input-image units
 *   offset [N, PH, PW, 2]  (dx_hat, dy_hat), normalised by the region size
 *   out    [N, PH, PW, C]
 * Reading (the page gives the offset normalisation and the interpolation
 * only): coordinates are scaled by spatial_scale, the region is at least one
 * pixel on each side, each bin averages S x S sampling points placed at the
 * centres of an S x S sub-grid of the bin, pixel centres at integers.  All
 * position arithmetic is fp32 with one rounding per operation, in this
 * order, so that both implementations take the same floor() decisions.
 */
void oracle_roi_pool_forward(int B, int H, int W, int C, int N, int PH, int PW, int S,
                             float spatial_scale, float gamma,
                             const double *x, const float *rois, const float *offset, double *out)
{
#pragma omp parallel for schedule(static)
    for (int n = 0; n < N; ++n) {
        const float *r = rois + (size_t)n * 5;
        /* A batch index that names no image of the input (outside [0, B), or
         * not a number) reads nothing: every bin of the region is zero.
         * Inside the range the index is the integer part of the value. */
        if (!(r[0] >= 0.0f && r[0] < (float)B)) {
            for (size_t e = 0; e < (size_t)PH * PW * C; ++e) out[(size_t)n * PH * PW * C + e] = 0.0;
            continue;
        }
        const int b = (int)r[0];
        const float x1 = r[1] * spatial_scale, y1 = r[2] * spatial_scale;
        const float x2 = r[3] * spatial_scale, y2 = r[4] * spatial_scale;
        float rw = x2 - x1, rh = y2 - y1;
        if (!(rw >= 1.0f)) rw = 1.0f;
        if (!(rh >= 1.0f)) rh = 1.0f;
        const float bw = rw / (float)PW, bh = rh / (float)PH;
        const float sw = bw / (float)S, sh = bh / (float)S;
        for (int i = 0; i < PH; ++i)
            for (int j = 0; j < PW; ++j) {
                const float *d = offset + (((size_t)n * PH + i) * PW + j) * 2;
                const float dx = (gamma * d[0]) * rw, dy = (gamma * d[1]) * rh;
                const float bx0 = x1 + (float)j * bw, by0 = y1 + (float)i * bh;
                double *y = out + (((size_t)n * PH + i) * PW + j) * C;
                for (int c = 0; c < C; ++c) y[c] = 0.0;
                int not_a_number = 0;
                for (int sy = 0; sy < S; ++sy)
                    for (int sx = 0; sx < S; ++sx) {
                        const float py = (by0 + ((float)sy + 0.5f) * sh) + dy;
                        const float px = (bx0 + ((float)sx + 0.5f) * sw) + dx;
                        if (isnan(px) || isnan(py)) { not_a_number = 1; continue; }
                        const double fy = floor((double)py), fx = floor((double)px);
                        if (!(fy >= -1.0 && fy <= H - 1 && fx >= -1.0 && fx <= W - 1)) continue;
                        const int y0 = (int)fy, x0 = (int)fx;
                        for (int qy = y0; qy <= y0 + 1; ++qy) {
                            if (qy < 0 || qy >= H) continue;
                            const double gy = g_kernel(qy, py);
                            for (int qx = x0; qx <= x0 + 1; ++qx) {
                                if (qx < 0 || qx >= W) continue;
                                const double Gq = g_kernel(qx, px) * gy;
                                const double *xq = x + (((size_t)b * H + qy) * W + qx) * (size_t)C;
                                for (int c = 0; c < C; ++c) y[c] += Gq * xq[c];
                            }
                        }
                    }
                for (int c = 0; c < C; ++c) y[c] = not_a_number ? NAN : y[c] / (double)(S * S);
            }
    }
}
