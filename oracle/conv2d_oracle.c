/*
 * conv2d_oracle.c -- TEST INFRASTRUCTURE ONLY.
 *
 * A plain, slow, obviously correct CPU statement of the 2-D convolution
 * forward pass, accumulating in double precision.  Only the test suite, the
 * package smoke check and the benchmark's CPU-baseline leg load this file's
 * library; the CUDA library never includes, links or calls anything here, and
 * nothing here is shared with it.
 *
 * Sources followed (page title, then section):
 *   - "手撕 Conv2D" interview page (lpnh.cn/news/2493075) §1.1: the forward
 *     index map  y[n][oc][oh][ow] = bias[oc] + sum_{ic,kh,kw}
 *     x[n][ic][oh*stride + kh - pad][ow*stride + kw - pad] * w[oc][ic][kh][kw];
 *     §1.2 and §2.1: padding by a bounds check (a term whose input row or
 *     column falls outside [0,H) x [0,W) is skipped), accumulator started at
 *     bias[oc]; §7: dilation multiplies the kernel tap index (kh*d, kw*d).
 *   - "PyTorch高维张量乘法与conv2d/conv3d维度语义解析" (pwwt.cn/news/6111401)
 *     §4.1 shapes x (N,C_in,H,W), w (C_out, C_in/groups, kH, kW), bias
 *     (C_out,); §4.2 output size floor((H + 2p - d(k-1) - 1)/s) + 1;
 *     §4.3 groups: output channel block i sees only input channel block i,
 *     both C_in and C_out divisible by groups.
 *   - Conv2d documentation walk-through (dpshk.com/news/5792599, page title
 *     "企业官网建设流程全解析") §3.2 the same size formula with floor, §3.3
 *     dilation spacing, §3.4 groups.
 *
 * Layouts are the pages' own: x NCHW, w OIHW (C_out, C_in/groups, Kh, Kw),
 * y NCHW, all row-major doubles.  Stride, padding and dilation are one value
 * each, used for both spatial dimensions; padding is zeros on both sides.
 */
#include <stddef.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* Output extent along one spatial dimension ("PyTorch高维张量乘法..." §4.2).
 * Returns 0 and stores the size, or -1 if an argument is out of range or the
 * size would be below 1 (the floor of a negative numerator is rejected). */
int oracle_conv2d_out_size(long in, long k, long stride, long pad, long dilation,
                           long *out)
{
    if (in < 1 || k < 1 || stride < 1 || pad < 0 || dilation < 1 || !out)
        return -1;
    long numer = in + 2 * pad - dilation * (k - 1) - 1;
    if (numer < 0)
        return -1;
    *out = numer / stride + 1; /* numer >= 0, so C division is the floor */
    return 0;
}

static int check_shape(long N, long C_in, long H, long W, long C_out, long Kh,
                       long Kw, long stride, long pad, long dilation, long groups,
                       long *Ho, long *Wo)
{
    if (N < 1 || C_in < 1 || C_out < 1 || groups < 1)
        return -1;
    if (C_in % groups != 0 || C_out % groups != 0)
        return -1;
    if (oracle_conv2d_out_size(H, Kh, stride, pad, dilation, Ho) != 0)
        return -1;
    if (oracle_conv2d_out_size(W, Kw, stride, pad, dilation, Wo) != 0)
        return -1;
    return 0;
}

/* One output element, straight from the definition. */
static double point(const double *x, const double *w, const double *bias,
                    long C_in, long H, long W, long C_out, long Kh, long Kw,
                    long stride, long pad, long dilation, long groups,
                    long n, long oc, long oh, long ow)
{
    long cin_g = C_in / groups;        /* input channels seen by one group  */
    long cout_g = C_out / groups;      /* output channels made by one group */
    long g = oc / cout_g;              /* the group this output belongs to  */
    double acc = bias ? bias[oc] : 0.0;
    for (long c = 0; c < cin_g; ++c) {
        long ic = g * cin_g + c;
        for (long kh = 0; kh < Kh; ++kh) {
            long ih = oh * stride + kh * dilation - pad;
            if (ih < 0 || ih >= H)
                continue; /* zero padding */
            for (long kw = 0; kw < Kw; ++kw) {
                long iw = ow * stride + kw * dilation - pad;
                if (iw < 0 || iw >= W)
                    continue; /* zero padding */
                double xv = x[((n * C_in + ic) * H + ih) * W + iw];
                double wv = w[((oc * cin_g + c) * Kh + kh) * Kw + kw];
                acc += xv * wv;
            }
        }
    }
    return acc;
}

/* The whole output y (N, C_out, Ho, Wo).  bias may be NULL (no bias).
 * Returns 0, or -1 on an invalid shape (y untouched). */
int oracle_conv2d_nchw(const double *x, const double *w, const double *bias,
                       double *y, long N, long C_in, long H, long W, long C_out,
                       long Kh, long Kw, long stride, long pad, long dilation,
                       long groups)
{
    long Ho, Wo;
    if (!x || !w || !y)
        return -1;
    if (check_shape(N, C_in, H, W, C_out, Kh, Kw, stride, pad, dilation, groups,
                    &Ho, &Wo) != 0)
        return -1;
#pragma omp parallel for collapse(2) schedule(dynamic, 1)
    for (long n = 0; n < N; ++n)
        for (long oc = 0; oc < C_out; ++oc)
            for (long oh = 0; oh < Ho; ++oh)
                for (long ow = 0; ow < Wo; ++ow)
                    y[((n * C_out + oc) * Ho + oh) * Wo + ow] =
                        point(x, w, bias, C_in, H, W, C_out, Kh, Kw, stride, pad,
                              dilation, groups, n, oc, oh, ow);
    return 0;
}

/* A list of single output elements (n, oc, oh, ow given as 4 * count longs),
 * for checking sampled outputs of problems too large to compute whole.
 * Returns 0, or -1 on an invalid shape or an index out of range. */
int oracle_conv2d_points(const double *x, const double *w, const double *bias,
                         long N, long C_in, long H, long W, long C_out, long Kh,
                         long Kw, long stride, long pad, long dilation,
                         long groups, const long *idx, long count, double *out)
{
    long Ho, Wo;
    if (!x || !w || !idx || !out || count < 0)
        return -1;
    if (check_shape(N, C_in, H, W, C_out, Kh, Kw, stride, pad, dilation, groups,
                    &Ho, &Wo) != 0)
        return -1;
    for (long i = 0; i < count; ++i) {
        const long *p = idx + 4 * i;
        if (p[0] < 0 || p[0] >= N || p[1] < 0 || p[1] >= C_out || p[2] < 0 ||
            p[2] >= Ho || p[3] < 0 || p[3] >= Wo)
            return -1;
    }
#pragma omp parallel for schedule(static)
    for (long i = 0; i < count; ++i) {
        const long *p = idx + 4 * i;
        out[i] = point(x, w, bias, C_in, H, W, C_out, Kh, Kw, stride, pad,
                       dilation, groups, p[0], p[1], p[2], p[3]);
    }
    return 0;
}

/* Threads the parallel loops above will use. */
int oracle_num_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
