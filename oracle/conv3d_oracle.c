/*
 * conv3d_oracle.c -- TEST INFRASTRUCTURE ONLY.
 *
 * A plain, slow, obviously correct CPU statement of the 3-D convolution forward pass,
 * accumulating in double precision.  Only the test suite and the benchmark's
 * CPU-baseline leg load this file's library; the CUDA library never includes, links or
 * calls anything here, and nothing here is shared with it.
 *
 * Sources followed (page title, then section):
 *   - "PyTorch高维张量乘法与conv2d/conv3d维度语义解析" (pwwt.cn/news/6111401) §5.1:
 *     x is (N, C_in, D, H, W), the weight (C_out, C_in/groups, kD, kH, kW), the output
 *     (N, C_out, D_out, H_out, W_out), and the kernel slides over D, H and W alike (the
 *     three spatial directions are treated the same); §4.2's output-size formula holds
 *     in each of the three directions (§6.2 applies it to D, H and W); §4.3's groups.
 *   - The 2-D definition this extends is the "手撕 Conv2D" page's (lpnh.cn/news/2493075)
 *     §1.1-§2.1 six-loop form with bounds-checked zero padding; dilation per its §7.
 * So y[n][oc][od][oh][ow] = bias[oc] + sum over c < C_in/groups, kd, kh, kw of
 * x[n][g*C_in/groups + c][od*s + kd*d - p][oh*s + kh*d - p][ow*s + kw*d - p] * w[oc][c][kd][kh][kw],
 * g = oc / (C_out/groups), a term dropped when its input position is outside the volume.
 * Stride, padding and dilation are one value each, used in all three directions.
 */
#include <stddef.h>
#ifdef _OPENMP
#include <omp.h>
#endif

static long extent(long in, long k, long s, long p, long d)
{
    long numer = in + 2 * p - d * (k - 1) - 1;
    if (in < 1 || k < 1 || s < 1 || p < 0 || d < 1 || numer < 0)
        return -1;
    return numer / s + 1;
}

/* One output element, straight from the definition. */
static double point(const double *x, const double *w, const double *bias, long C_in, long D,
                    long H, long W, long C_out, long Kd, long Kh, long Kw, long stride,
                    long pad, long dilation, long groups, long n, long oc, long od, long oh,
                    long ow)
{
    long cin_g = C_in / groups, cout_g = C_out / groups, g = oc / cout_g;
    double acc = bias ? bias[oc] : 0.0;
    for (long c = 0; c < cin_g; ++c) {
        long ic = g * cin_g + c;
        for (long kd = 0; kd < Kd; ++kd) {
            long id = od * stride + kd * dilation - pad;
            if (id < 0 || id >= D)
                continue;
            for (long kh = 0; kh < Kh; ++kh) {
                long ih = oh * stride + kh * dilation - pad;
                if (ih < 0 || ih >= H)
                    continue;
                for (long kw = 0; kw < Kw; ++kw) {
                    long iw = ow * stride + kw * dilation - pad;
                    if (iw < 0 || iw >= W)
                        continue;
                    acc += x[(((n * C_in + ic) * D + id) * H + ih) * W + iw] *
                           w[(((oc * cin_g + c) * Kd + kd) * Kh + kh) * Kw + kw];
                }
            }
        }
    }
    return acc;
}

static int shape3(long N, long C_in, long D, long H, long W, long C_out, long Kd, long Kh,
                  long Kw, long stride, long pad, long dilation, long groups, long *Do,
                  long *Ho, long *Wo)
{
    if (N < 1 || C_in < 1 || C_out < 1 || groups < 1 || C_in % groups || C_out % groups)
        return -1;
    *Do = extent(D, Kd, stride, pad, dilation);
    *Ho = extent(H, Kh, stride, pad, dilation);
    *Wo = extent(W, Kw, stride, pad, dilation);
    return (*Do < 1 || *Ho < 1 || *Wo < 1) ? -1 : 0;
}

/* The whole output y (N, C_out, Do, Ho, Wo).  bias may be NULL.  Returns 0, or -1 on an
 * invalid shape (y untouched). */
int oracle_conv3d(const double *x, const double *w, const double *bias, double *y, long N,
                  long C_in, long D, long H, long W, long C_out, long Kd, long Kh, long Kw,
                  long stride, long pad, long dilation, long groups)
{
    long Do, Ho, Wo;
    if (!x || !w || !y)
        return -1;
    if (shape3(N, C_in, D, H, W, C_out, Kd, Kh, Kw, stride, pad, dilation, groups, &Do, &Ho,
               &Wo) != 0)
        return -1;
#pragma omp parallel for collapse(2) schedule(dynamic, 1)
    for (long n = 0; n < N; ++n)
        for (long oc = 0; oc < C_out; ++oc)
            for (long od = 0; od < Do; ++od)
                for (long oh = 0; oh < Ho; ++oh)
                    for (long ow = 0; ow < Wo; ++ow)
                        y[(((n * C_out + oc) * Do + od) * Ho + oh) * Wo + ow] =
                            point(x, w, bias, C_in, D, H, W, C_out, Kd, Kh, Kw, stride, pad,
                                  dilation, groups, n, oc, od, oh, ow);
    return 0;
}

/* Selected outputs (n, oc, od, oh, ow given as 5 * count longs).  Returns 0, or -1 on an
 * invalid shape or index. */
int oracle_conv3d_points(const double *x, const double *w, const double *bias, long N, long C_in,
                         long D, long H, long W, long C_out, long Kd, long Kh, long Kw,
                         long stride, long pad, long dilation, long groups, const long *idx,
                         long count, double *out)
{
    long Do, Ho, Wo;
    if (!x || !w || !idx || !out || count < 0)
        return -1;
    if (shape3(N, C_in, D, H, W, C_out, Kd, Kh, Kw, stride, pad, dilation, groups, &Do, &Ho,
               &Wo) != 0)
        return -1;
    for (long i = 0; i < count; ++i) {
        const long *q = idx + 5 * i;
        if (q[0] < 0 || q[0] >= N || q[1] < 0 || q[1] >= C_out || q[2] < 0 || q[2] >= Do ||
            q[3] < 0 || q[3] >= Ho || q[4] < 0 || q[4] >= Wo)
            return -1;
    }
#pragma omp parallel for schedule(static)
    for (long i = 0; i < count; ++i) {
        const long *q = idx + 5 * i;
        out[i] = point(x, w, bias, C_in, D, H, W, C_out, Kd, Kh, Kw, stride, pad, dilation,
                       groups, q[0], q[1], q[2], q[3], q[4]);
    }
    return 0;
}
