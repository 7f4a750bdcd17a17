/*
 * conv2d_backward_oracle.c -- TEST INFRASTRUCTURE ONLY.
 *
 * A plain, slow, obviously correct CPU statement of the 2-D convolution's backward
 * pass -- the gradients of a loss L with respect to the input, the weights and the
 * bias, given dL/dy -- accumulating in double precision.  Only the test suite and the
 * benchmark's CPU-baseline leg load this file's library; the CUDA library never
 * includes, links or calls anything here, and nothing here is shared with it.
 *
 * Sources followed (page title, then section):
 *   - "手撕 Conv2D" interview page (lpnh.cn/news/2493075) §5.1: the three gradients,
 *       db[oc]             = sum_{n, oh, ow} dout[n][oc][oh][ow]
 *       dW[oc][ic][kh][kw] = sum_{n, oh, ow} dout[n][oc][oh][ow] * x[n][ic][oh*s + kh - p][ow*s + kw - p]
 *       dx                 : every dout[n][oc][oh][ow] is scattered back, times the
 *                            weight, onto each input position of its window, the
 *                            contributions of overlapping windows added up;
 *     input positions outside the image take no part (the padding); §5.2: the naive
 *     loops -- db first, then one loop nest over (n, oc, oh, ow) that, for each
 *     (ic, kh, kw) inside the image, adds x * dout into dW and w * dout into dx;
 *     §7: dilation multiplies the tap index (kh*d, kw*d); groups restrict output
 *     channel oc to the input channels of its group.
 *   - The im2col/GEMM tutorial (zskr.cn/news/1820658) §3.3 states the same three
 *     gradients in matrix form (dW_row = dout_col X_col^T, db = sum of dout,
 *     dx = col2im(W_row^T dout_col)); the tests use that form as an independent pin.
 *
 * The §5.2 loop nest updates dx and dW together; here it is run twice with the same
 * inner order -- once parallel over images (each thread owns dx[n], so the scatter
 * needs no atomics) updating dx, once parallel over output channels (each thread owns
 * dW[oc]) updating dW.  Splitting one loop into two changes no sum.
 *
 * Layouts are the pages' own: x and dx NCHW, w and dW OIHW (C_out, C_in/groups, Kh,
 * Kw), dy NCHW (N, C_out, Ho, Wo), all row-major doubles.  Stride, padding and
 * dilation are one value each, used for both spatial dimensions.
 */
#include <stddef.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* Output extent along one spatial dimension, floor((in + 2p - d(k-1) - 1)/s) + 1
 * ("PyTorch高维张量乘法与conv2d/conv3d维度语义解析" §4.2); -1 if below 1. */
static long out_extent(long in, long k, long s, long p, long d)
{
    long numer = in + 2 * p - d * (k - 1) - 1;
    if (in < 1 || k < 1 || s < 1 || p < 0 || d < 1 || numer < 0)
        return -1;
    return numer / s + 1;
}

static int check_shape(long N, long C_in, long H, long W, long C_out, long Kh,
                       long Kw, long stride, long pad, long dilation, long groups,
                       long *Ho, long *Wo)
{
    if (N < 1 || C_in < 1 || C_out < 1 || groups < 1)
        return -1;
    if (C_in % groups != 0 || C_out % groups != 0)
        return -1;
    *Ho = out_extent(H, Kh, stride, pad, dilation);
    *Wo = out_extent(W, Kw, stride, pad, dilation);
    return (*Ho < 1 || *Wo < 1) ? -1 : 0;
}

/* dx (N, C_in, H, W), dW (C_out, C_in/groups, Kh, Kw) and db (C_out) from dy, x and w.
 * Any of dx, dW, db may be NULL (that gradient is skipped).  Returns 0, or -1 on an
 * invalid shape (outputs untouched). */
int oracle_conv2d_backward(const double *dy, const double *x, const double *w,
                           double *dx, double *dW, double *db, long N, long C_in,
                           long H, long W, long C_out, long Kh, long Kw, long stride,
                           long pad, long dilation, long groups)
{
    long Ho, Wo;
    if (!dy || !x || !w)
        return -1;
    if (check_shape(N, C_in, H, W, C_out, Kh, Kw, stride, pad, dilation, groups,
                    &Ho, &Wo) != 0)
        return -1;
    const long cin_g = C_in / groups, cout_g = C_out / groups;

    /* bias gradient: sum of dout over images and output positions */
    if (db) {
        for (long oc = 0; oc < C_out; ++oc) {
            double acc = 0.0;
            for (long n = 0; n < N; ++n)
                for (long oh = 0; oh < Ho; ++oh)
                    for (long ow = 0; ow < Wo; ++ow)
                        acc += dy[((n * C_out + oc) * Ho + oh) * Wo + ow];
            db[oc] = acc;
        }
    }

    /* input gradient: scatter every dout back onto its window */
    if (dx) {
#pragma omp parallel for schedule(dynamic, 1)
        for (long n = 0; n < N; ++n) {
            for (long i = 0; i < C_in * H * W; ++i)
                dx[n * C_in * H * W + i] = 0.0;
            for (long oc = 0; oc < C_out; ++oc) {
                long g = oc / cout_g;
                for (long oh = 0; oh < Ho; ++oh)
                    for (long ow = 0; ow < Wo; ++ow) {
                        double grad_out = dy[((n * C_out + oc) * Ho + oh) * Wo + ow];
                        for (long c = 0; c < cin_g; ++c) {
                            long ic = g * cin_g + c;
                            for (long kh = 0; kh < Kh; ++kh) {
                                long ih = oh * stride + kh * dilation - pad;
                                if (ih < 0 || ih >= H)
                                    continue;
                                for (long kw = 0; kw < Kw; ++kw) {
                                    long iw = ow * stride + kw * dilation - pad;
                                    if (iw < 0 || iw >= W)
                                        continue;
                                    dx[((n * C_in + ic) * H + ih) * W + iw] +=
                                        w[((oc * cin_g + c) * Kh + kh) * Kw + kw] * grad_out;
                                }
                            }
                        }
                    }
            }
        }
    }

    /* weight gradient: dout times the input value each tap saw */
    if (dW) {
#pragma omp parallel for schedule(dynamic, 1)
        for (long oc = 0; oc < C_out; ++oc) {
            long g = oc / cout_g;
            for (long i = 0; i < cin_g * Kh * Kw; ++i)
                dW[oc * cin_g * Kh * Kw + i] = 0.0;
            for (long n = 0; n < N; ++n)
                for (long oh = 0; oh < Ho; ++oh)
                    for (long ow = 0; ow < Wo; ++ow) {
                        double grad_out = dy[((n * C_out + oc) * Ho + oh) * Wo + ow];
                        for (long c = 0; c < cin_g; ++c) {
                            long ic = g * cin_g + c;
                            for (long kh = 0; kh < Kh; ++kh) {
                                long ih = oh * stride + kh * dilation - pad;
                                if (ih < 0 || ih >= H)
                                    continue;
                                for (long kw = 0; kw < Kw; ++kw) {
                                    long iw = ow * stride + kw * dilation - pad;
                                    if (iw < 0 || iw >= W)
                                        continue;
                                    dW[((oc * cin_g + c) * Kh + kh) * Kw + kw] +=
                                        x[((n * C_in + ic) * H + ih) * W + iw] * grad_out;
                                }
                            }
                        }
                    }
        }
    }
    return 0;
}

/* Selected input-gradient elements dx[n][ic][ih][iw] (rows of idx), for problems too
 * large to compute whole.  dx at one input position is the sum, over the output
 * channels of its group and the filter taps, of dout at the output position whose
 * window puts that tap on it (oh*s + kh*d - p = ih, the same for columns) times the
 * tap's weight -- the scatter of §5.1 read from the receiving side.
 * Returns 0, or -1 on an invalid shape or index. */
int oracle_conv2d_backward_data_points(const double *dy, const double *w, long N,
                                       long C_in, long H, long W, long C_out, long Kh,
                                       long Kw, long stride, long pad, long dilation,
                                       long groups, const long *idx, long count,
                                       double *out)
{
    long Ho, Wo;
    if (!dy || !w || !idx || !out || count < 0)
        return -1;
    if (check_shape(N, C_in, H, W, C_out, Kh, Kw, stride, pad, dilation, groups,
                    &Ho, &Wo) != 0)
        return -1;
    const long cin_g = C_in / groups, cout_g = C_out / groups;
    for (long i = 0; i < count; ++i) {
        const long *q = idx + 4 * i;
        if (q[0] < 0 || q[0] >= N || q[1] < 0 || q[1] >= C_in || q[2] < 0 ||
            q[2] >= H || q[3] < 0 || q[3] >= W)
            return -1;
    }
#pragma omp parallel for schedule(static)
    for (long i = 0; i < count; ++i) {
        const long n = idx[4 * i], ic = idx[4 * i + 1], ih = idx[4 * i + 2], iw = idx[4 * i + 3];
        const long g = ic / cin_g, c = ic - g * cin_g;
        double acc = 0.0;
        for (long oc = g * cout_g; oc < (g + 1) * cout_g; ++oc)
            for (long kh = 0; kh < Kh; ++kh) {
                long th = ih + pad - kh * dilation; /* = oh * stride if some oh reaches ih */
                if (th < 0 || th % stride != 0 || th / stride >= Ho)
                    continue;
                long oh = th / stride;
                for (long kw = 0; kw < Kw; ++kw) {
                    long tw = iw + pad - kw * dilation;
                    if (tw < 0 || tw % stride != 0 || tw / stride >= Wo)
                        continue;
                    long ow = tw / stride;
                    acc += dy[((n * C_out + oc) * Ho + oh) * Wo + ow] *
                           w[((oc * cin_g + c) * Kh + kh) * Kw + kw];
                }
            }
        out[i] = acc;
    }
    return 0;
}

/* Selected weight-gradient elements dW[oc][c][kh][kw] (rows of idx), straight from the
 * §5.1 formula: the sum over images and output positions of dout times the input value
 * under that tap.  Returns 0, or -1 on an invalid shape or index. */
int oracle_conv2d_backward_weight_points(const double *dy, const double *x, long N,
                                         long C_in, long H, long W, long C_out, long Kh,
                                         long Kw, long stride, long pad, long dilation,
                                         long groups, const long *idx, long count,
                                         double *out)
{
    long Ho, Wo;
    if (!dy || !x || !idx || !out || count < 0)
        return -1;
    if (check_shape(N, C_in, H, W, C_out, Kh, Kw, stride, pad, dilation, groups,
                    &Ho, &Wo) != 0)
        return -1;
    const long cin_g = C_in / groups, cout_g = C_out / groups;
    for (long i = 0; i < count; ++i) {
        const long *q = idx + 4 * i;
        if (q[0] < 0 || q[0] >= C_out || q[1] < 0 || q[1] >= cin_g || q[2] < 0 ||
            q[2] >= Kh || q[3] < 0 || q[3] >= Kw)
            return -1;
    }
#pragma omp parallel for schedule(static)
    for (long i = 0; i < count; ++i) {
        const long oc = idx[4 * i], c = idx[4 * i + 1], kh = idx[4 * i + 2], kw = idx[4 * i + 3];
        const long ic = (oc / cout_g) * cin_g + c;
        double acc = 0.0;
        for (long n = 0; n < N; ++n)
            for (long oh = 0; oh < Ho; ++oh) {
                long ih = oh * stride + kh * dilation - pad;
                if (ih < 0 || ih >= H)
                    continue;
                for (long ow = 0; ow < Wo; ++ow) {
                    long iw = ow * stride + kw * dilation - pad;
                    if (iw < 0 || iw >= W)
                        continue;
                    acc += dy[((n * C_out + oc) * Ho + oh) * Wo + ow] *
                           x[((n * C_in + ic) * H + ih) * W + iw];
                }
            }
        out[i] = acc;
    }
    return 0;
}

/* Threads the parallel loops above will use. */
int oracle_backward_num_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
