/*
 * conv2d_b200.h -- C ABI of the B200 (sm_100a) 2-D convolution forward library.
 *
 * The operation is the 2-D convolution forward pass
 *     y[n][oc][oh][ow] = bias[oc] + sum_{c < C_in/groups, kh < Kh, kw < Kw}
 *         x[n][g*C_in/groups + c][oh*stride + kh*dilation - pad]
 *                                [ow*stride + kw*dilation - pad] * w[oc][c][kh][kw]
 * with g = oc / (C_out/groups) and terms whose input row or column falls outside
 * the image dropped (zero padding).  Definition: "手撕 Conv2D" interview page
 * (lpnh.cn/news/2493075) §1.1 (index map) and §2.1 (bounds-checked padding, bias
 * added once per output); dilation per the same page §7; groups and shapes per
 * "PyTorch高维张量乘法与conv2d/conv3d维度语义解析" (pwwt.cn/news/6111401) §4.1 and
 * §4.3; output size per the same page §4.2.  The im2col + matrix-product view
 * Y = W_row @ X_col is the one the im2col/GEMM tutorial (zskr.cn/news/1820658)
 * §2.2-§2.3 gives; conv2d_forward computes that product without forming X_col.
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 * - Pointers named x, y, w_*, bias, workspace are DEVICE pointers owned by the
 *   caller (cudaMalloc or any allocator of device memory); the library never
 *   frees or keeps them.  Pointers named *_host are host pointers (pinned memory
 *   gives asynchronous copies).  Every device pointer must be 16-byte aligned.
 * - `stream` is a cudaStream_t (NULL = the legacy default stream).  Every call
 *   that takes a stream only enqueues work on it and returns; results are ready
 *   once the stream reaches that point.  Device-side watchdog failures are
 *   reported by conv2d_sync_status().
 * - dtype CONV_BF16: x, w, bias and y hold bfloat16; products are accumulated
 *   in fp32 and bias is added in fp32 before one round-to-nearest-even to bf16.
 *   dtype CONV_F32: all tensors are fp32; the products run on tensor cores with
 *   the three-term TF32 split (a*b ~ a_hi*b_hi + a_hi*b_lo + a_lo*b_hi) and
 *   fp32 accumulation.
 * - layout CONV_NCHW: x is (N, C_in, H, W) and y is (N, C_out, Ho, Wo).
 *   layout CONV_NHWC: x is (N, H, W, C_in) and y is (N, Ho, Wo, C_out).
 * - Stride, pad and dilation apply to both spatial dimensions; padding is zero
 *   padding on both sides.
 * - Every function returns a conv_status_t.  On any status other than CONV_OK
 *   nothing has been enqueued and no output byte has been written;
 *   conv2d_last_error() then returns a message for the calling thread.
 */
#ifndef CONV2D_B200_H
#define CONV2D_B200_H

#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

/* A cudaStream_t; declared here so that this header needs no CUDA header. */
typedef struct CUstream_st *conv_stream_t;

typedef enum {
    CONV_OK = 0,
    CONV_ERR_INVALID_ARG = 1, /* a shape, size or pointer argument is invalid   */
    CONV_ERR_UNSUPPORTED = 2, /* valid, but outside what the kernels cover      */
    CONV_ERR_CUDA = 3,        /* a CUDA runtime or driver call failed           */
    CONV_ERR_TIMEOUT = 4,     /* a device-side wait ran out (see sync_status)   */
    CONV_ERR_WORKSPACE = 5    /* the workspace passed in is too small           */
} conv_status_t;

typedef enum { CONV_F32 = 0, CONV_BF16 = 1 } conv_dtype_t;
typedef enum { CONV_NHWC = 0, CONV_NCHW = 1 } conv_layout_t;

/* Output extent along one spatial dimension,
 *     *out = floor((in + 2*pad - dilation*(k - 1) - 1) / stride) + 1,
 * the formula of "PyTorch高维张量乘法与conv2d/conv3d维度语义解析" §4.2 (and of the
 * Conv2d documentation walk-through, dpshk.com/news/5792599, §3.2).
 * CONV_ERR_INVALID_ARG if in, k, stride or dilation < 1, pad < 0, out is NULL,
 * or the result would be below 1 (a negative numerator is rejected, not floored). */
int conv2d_output_size(int in, int k, int stride, int pad, int dilation, int *out);

/* Bytes of the packed weight buffer that conv2d_pack_weight writes:
 * C_out * Kh * Kw * Cpg elements of dtype, where Cpg is C_in/groups rounded up
 * to a multiple of 8 (bf16) or 4 (fp32), followed -- for groups = 1 and fewer
 * than 32 bytes of input channels per pixel -- by ready-made shared-memory images
 * of the weight matrix for the few-channel kernel.  Narrow bf16 groups (fewer than 64
 * output channels each, C_in/groups a multiple of 8) are packed gm at
 * a time as one block-diagonal group, Cpg = gm * C_in/groups, with gm the largest
 * divisor of groups that keeps gm * C_out/groups <= 128 and gm * C_in/groups * the
 * element size <= 256 bytes; the forward pass then computes gm groups per product. */
int conv2d_packed_weight_size(int C_out, int C_in, int Kh, int Kw, int groups,
                              conv_dtype_t dtype, size_t *bytes);

/* Packs w_oihw (C_out, C_in/groups, Kh, Kw) -- the pages' weight layout
 * ("PyTorch高维张量乘法..." §4.1) -- into the layout the kernels read: for each
 * output channel the taps in (kh, kw) order, each tap's input channels
 * contiguous and zero-padded to Cpg (the OHWI order the Conv2d documentation
 * walk-through, dpshk.com/news/5792599, §5.2 describes for channels-last
 * frameworks).  Done once per weight, outside the timed path.
 * w_packed must hold conv2d_packed_weight_size() bytes; the two buffers must
 * not overlap. */
int conv2d_pack_weight(const void *w_oihw, void *w_packed, int C_out, int C_in,
                       int Kh, int Kw, int groups, conv_dtype_t dtype,
                       conv_stream_t stream);

/* Device scratch bytes conv2d_forward needs for this problem (0 when none).
 * Scratch holds a channels-last, channel-padded copy of x when layout is
 * CONV_NCHW or C_in/groups is not a multiple of 8 (bf16) / 4 (fp32), and fp32
 * partial sums when the reduction over C_in*Kh*Kw is split across SMs to fill
 * the machine.  Arguments are validated as in conv2d_forward. */
int conv2d_workspace_size(int N, int C_in, int H, int W, int C_out, int Kh, int Kw,
                          int stride, int pad, int dilation, int groups,
                          conv_dtype_t dtype, conv_layout_t layout, size_t *bytes);

/* The convolution forward pass as an implicit matrix product that never forms
 * the im2col matrix: rows are output pixels (N*Ho*Wo), columns output channels
 * of a group, and the reduction runs over (kh, kw, c).  Input patches are staged
 * tile by tile into shared memory by the tensor memory accelerator's im2col mode
 * (out-of-image reads return zero: the zero padding), weights by tiled loads,
 * tcgen05 tensor-core instructions accumulate in tensor memory, and the epilogue
 * adds bias and stores y in `layout`.  Depthwise problems (groups = C_in = C_out:
 * one filter per channel) instead run a direct stencil kernel over channels-last
 * tiles staged in shared memory -- the case the im2col/GEMM tutorial §4.2 names as
 * one where im2col only adds traffic -- with the same arguments and results.
 *   x         : input, layout as above, dtype elements
 *   w_packed  : weights from conv2d_pack_weight (same C_out, C_in, Kh, Kw, groups, dtype)
 *   bias      : (C_out,) dtype elements, or NULL for no bias
 *   y         : output, layout as above; must not overlap any input
 *   workspace : at least conv2d_workspace_size() bytes (may be NULL when that is 0)
 * Errors: CONV_ERR_INVALID_ARG for a non-positive size, stride < 1, dilation < 1,
 * pad < 0, C_in or C_out not divisible by groups (pwwt §4.3), an empty output,
 * or a NULL x / w_packed / y; CONV_ERR_WORKSPACE when workspace_bytes is too
 * small; CONV_ERR_UNSUPPORTED for a misaligned pointer, stride > 8,
 * pad > 127, dilation*(K-1) - pad outside [-128, 127] (limits of the hardware
 * im2col addressing), or C_in/groups not a multiple of 8 (bf16) / 4 (fp32)
 * when groups > 1; CONV_ERR_CUDA if the launch fails. */
int conv2d_forward(const void *x, const void *w_packed, const void *bias, void *y,
                   int N, int C_in, int H, int W, int C_out, int Kh, int Kw,
                   int stride, int pad, int dilation, int groups,
                   conv_dtype_t dtype, conv_layout_t layout,
                   void *workspace, size_t workspace_bytes, conv_stream_t stream);

/* Device scratch bytes conv2d_forward_im2col_gemm needs: the explicit im2col
 * matrix (N*Ho*Wo rows of groups*Kh*Kw*Cpg elements) plus what conv2d_forward
 * would need. */
int conv2d_im2col_workspace_size(int N, int C_in, int H, int W, int C_out, int Kh,
                                 int Kw, int stride, int pad, int dilation,
                                 int groups, conv_dtype_t dtype, conv_layout_t layout,
                                 size_t *bytes);

/* The pages' own formulation, kept as a comparison point: an im2col kernel
 * writes X_col (one row per output pixel, (kh, kw, c) along the row -- the
 * transpose of zskr §2.2's column matrix) into the workspace, then the same
 * tensor-core matrix product Y = X_col * W_row^T + bias runs over it (zskr
 * §2.3, lpnh §4.2).  Arguments and errors as conv2d_forward; the workspace must
 * hold conv2d_im2col_workspace_size() bytes. */
int conv2d_forward_im2col_gemm(const void *x, const void *w_packed, const void *bias,
                               void *y, int N, int C_in, int H, int W, int C_out,
                               int Kh, int Kw, int stride, int pad, int dilation,
                               int groups, conv_dtype_t dtype, conv_layout_t layout,
                               void *workspace, size_t workspace_bytes,
                               conv_stream_t stream);

/* End-to-end call for host-resident activations: enqueues the copy of x_host into
 * x_dev, conv2d_forward(x_dev, ...) into y_dev, and the copy of y_dev back into
 * y_host, ordered after the work already on `stream` and before the work enqueued on it
 * later.  x_host/y_host are host buffers of the x and y sizes (pinned for asynchronous
 * copies); x_dev/y_dev are caller-owned device buffers of the same sizes.  Weights and
 * bias stay resident on the device.  With at least 16 MB of input (and images of whole
 * 16-byte multiples) the batch is cut into up to 16 chunks of >= 8 MB along N, each
 * chunk's input copy, product and output copy chained through two internal copy streams
 * of the device, so that the two copy directions and the products overlap (only chunk
 * sizes whose plans fit workspace_bytes are used; otherwise one chunk).  The products run
 * on `stream`.  Returns after enqueuing; y_host is valid once the stream is
 * synchronised.  Errors as conv2d_forward. */
int conv2d_forward_hostio(const void *x_host, void *y_host, void *x_dev, void *y_dev,
                          const void *w_packed, const void *bias,
                          int N, int C_in, int H, int W, int C_out, int Kh, int Kw,
                          int stride, int pad, int dilation, int groups,
                          conv_dtype_t dtype, conv_layout_t layout,
                          void *workspace, size_t workspace_bytes,
                          conv_stream_t stream);

/* Layout change NCHW -> channels-last: dst[n][h][w][g*Cpg + c] = src[n][g*Cg + c][h][w]
 * for c < Cg = C/groups and zero for Cg <= c < Cpg (Cpg >= Cg).  This is the
 * "layout in" step for NCHW callers (pwwt §6.3 on channels_last; zero channels
 * make every pixel row a multiple of 16 bytes).  dst holds N*H*W*groups*Cpg
 * elements. */
int conv2d_nchw_to_nhwc(const void *src, void *dst, int N, int C, int H, int W,
                        int groups, int Cpg, conv_dtype_t dtype, conv_stream_t stream);

/* Layout change channels-last -> NCHW: dst[n][c][h][w] = src[n][h][w][c]
 * (the final transpose of zskr §3.2 step 5). */
int conv2d_nhwc_to_nchw(const void *src, void *dst, int N, int C, int H, int W,
                        conv_dtype_t dtype, conv_stream_t stream);

/* Waits for `stream`, then reports and clears the device watchdog status:
 * CONV_ERR_TIMEOUT if a kernel of this library gave up on a wait since the
 * last call (its output is then incomplete), CONV_ERR_CUDA if the stream
 * reported an error, else CONV_OK. */
int conv2d_sync_status(conv_stream_t stream);

/* Message describing the last non-OK status returned on the calling thread
 * (empty string if none).  The pointer stays valid until the thread's next call. */
const char *conv2d_last_error(void);

/* Bytes of the device scratch built into the library for conv2d_forward_noalloc. */
#define CONV2D_NOALLOC_SCRATCH_BYTES (32u * 1024u * 1024u)

/* conv2d_forward for callers that cannot allocate device memory -- code running
 * where cudaMalloc is not allowed or not wanted (while a CUDA graph is being
 * captured, under an allocator that owns all device memory, or in a plugin whose
 * host gives it only input and output buffers).  The pages describe no such
 * entry point; it exists for deployment.
 * Arguments and results are those of conv2d_forward without the workspace: the
 * scratch it needs (a channels-last copy of x, split partial sums) comes from a
 * CONV2D_NOALLOC_SCRATCH_BYTES array compiled into the library, which every GPU
 * that loads the library holds until the process exits.  A problem needing more
 * scratch than that is rejected with CONV_ERR_WORKSPACE before anything is
 * enqueued.  Nothing in this call allocates memory.
 * The first call on a device looks up the array's device address (once per
 * device, with that device current); make that first call before any stream
 * capture.  All calls share the one array and it keeps the last call's contents
 * (every byte a call reads it has written first, so nothing needs clearing):
 * calls whose work overlaps on the GPU -- on different streams without ordering
 * between them -- race on it and must not be made. */
int conv2d_forward_noalloc(const void *x, const void *w_packed, const void *bias, void *y,
                           int N, int C_in, int H, int W, int C_out, int Kh, int Kw,
                           int stride, int pad, int dilation, int groups,
                           conv_dtype_t dtype, conv_layout_t layout, conv_stream_t stream);

/* ------------------------------------------------------------ backward pass ---
 * The gradients of a loss L with respect to the input, the weights and the bias of
 * y = conv2d(x, w) + bias, given dy = dL/dy: the three formulas of the "手撕 Conv2D"
 * page (lpnh.cn/news/2493075) §5.1 -- db[oc] = sum over n, oh, ow of dy;
 * dW[oc][c][kh][kw] = sum over n, oh, ow of dy[n][oc][oh][ow] * x[n][c][oh*s + kh*d - p][ow*s + kw*d - p];
 * dx = every dy scattered back, times its weight, onto the input positions of its
 * window -- which the im2col/GEMM tutorial (zskr.cn/news/1820658) §3.3 writes as
 * dW_row = dout_col X_col^T, db = sum of dout, dx = col2im(W_row^T dout_col).
 * Shapes, dtypes, layouts and the shape arguments are those of conv2d_forward for the
 * same convolution: dy has y's shape and layout, dx has x's.  Gradients are
 * accumulated in fp32 (fp32: three TF32 products per multiply-add, as the forward
 * pass) and rounded once to the dtype. */

/* Bytes of the kernel conv2d_pack_weight_backward_data writes: C_in * Kh * Kw * Cpg
 * elements of dtype with Cpg = C_out/groups rounded up to a multiple of 8 (bf16) / 4
 * (fp32), times the group merge factor described at conv2d_packed_weight_size for a
 * convolution of C_in output and C_out input channels. */
int conv2d_packed_weight_backward_data_size(int C_out, int C_in, int Kh, int Kw, int groups,
                                            conv_dtype_t dtype, size_t *bytes);

/* Packs w_oihw (C_out, C_in/groups, Kh, Kw) for conv2d_backward_data: the kernel of the
 * transposed convolution, w_t[ic][kh][kw][oc] = w[oc][ic][Kh-1-kh][Kw-1-kw] within each
 * group (spatially flipped, input and output channels exchanged), in the packed
 * channels-last layout.  Done once per weight; w_packed_t holds
 * conv2d_packed_weight_backward_data_size() bytes and must not overlap w_oihw. */
int conv2d_pack_weight_backward_data(const void *w_oihw, void *w_packed_t, int C_out, int C_in,
                                     int Kh, int Kw, int groups, conv_dtype_t dtype,
                                     conv_stream_t stream);

/* Device scratch bytes conv2d_backward_data needs (0 when none). */
int conv2d_backward_data_workspace_size(int N, int C_in, int H, int W, int C_out, int Kh, int Kw,
                                        int stride, int pad, int dilation, int groups,
                                        conv_dtype_t dtype, conv_layout_t layout, size_t *bytes);

/* Input gradient dx (x's shape and layout) from dy (y's shape and layout): the
 * transposed convolution, computed as a forward convolution of dy with the packed
 * kernel of conv2d_pack_weight_backward_data, stride 1 and padding
 * dilation*(K-1) - pad in each dimension, on the same tensor-core kernels as
 * conv2d_forward (or the depthwise kernel).  For stride s > 1, dy is first expanded
 * in the workspace with s-1 zero rows and columns between its rows and columns (so
 * the product does s*s times the multiply-adds of the gradient's own count).
 * Errors as conv2d_forward, plus CONV_ERR_UNSUPPORTED when the transposed
 * convolution falls outside the kernels' addressing limits (padding beyond +-127). */
int conv2d_backward_data(const void *dy, const void *w_packed_t, void *dx,
                         int N, int C_in, int H, int W, int C_out, int Kh, int Kw,
                         int stride, int pad, int dilation, int groups,
                         conv_dtype_t dtype, conv_layout_t layout,
                         void *workspace, size_t workspace_bytes, conv_stream_t stream);

/* Device scratch bytes conv2d_backward_weight needs; with_bias != 0 includes the bias
 * gradient's partial sums. */
int conv2d_backward_weight_workspace_size(int N, int C_in, int H, int W, int C_out, int Kh,
                                          int Kw, int stride, int pad, int dilation, int groups,
                                          conv_dtype_t dtype, conv_layout_t layout, int with_bias,
                                          size_t *bytes);

/* Weight gradient dw (C_out, C_in/groups, Kh, Kw) -- the pages' OIHW layout -- and,
 * when db is not NULL, the bias gradient db (C_out,), from x and dy.  With at least 32
 * bytes of input channels per group the product dW_row = dout_col X_col^T runs on the
 * tensor cores with its reduction over output pixels split across SMs (input patches
 * staged by the tensor memory accelerator's im2col mode, never formed in memory);
 * fewer channels per group (depthwise and the like) run on the CUDA cores.  Errors as
 * conv2d_forward; the workspace must hold conv2d_backward_weight_workspace_size() bytes
 * (with_bias = db != NULL). */
int conv2d_backward_weight(const void *x, const void *dy, void *dw, void *db,
                           int N, int C_in, int H, int W, int C_out, int Kh, int Kw,
                           int stride, int pad, int dilation, int groups,
                           conv_dtype_t dtype, conv_layout_t layout,
                           void *workspace, size_t workspace_bytes, conv_stream_t stream);

/* Device scratch bytes conv2d_backward_bias needs (partial sums). */
int conv2d_backward_bias_workspace_size(int N, int C_out, int Ho, int Wo, conv_layout_t layout,
                                        size_t *bytes);

/* Bias gradient alone: db[oc] = sum of dy[n][oc][oh][ow] over n, oh, ow (lpnh §5.1),
 * summed in fp32 and rounded once to dtype.  dy is (N, C_out, Ho, Wo) in `layout`. */
int conv2d_backward_bias(const void *dy, void *db, int N, int C_out, int Ho, int Wo,
                         conv_dtype_t dtype, conv_layout_t layout, void *workspace,
                         size_t workspace_bytes, conv_stream_t stream);

/* ------------------------------------------------------------------- conv3d ---
 * The 3-D convolution forward pass of "PyTorch高维张量乘法与conv2d/conv3d维度语义解析"
 * (pwwt.cn/news/6111401) §5.1: x (N, C_in, D, H, W), w (C_out, C_in/groups, Kd, Kh, Kw),
 * y (N, C_out, Do, Ho, Wo); the kernel slides over depth, height and width alike, each
 * output extent given by conv2d_output_size's formula (§6.2 applies it to D, H and W):
 *     y[n][oc][od][oh][ow] = bias[oc] + sum_{c, kd, kh, kw}
 *         x[n][g*C_in/groups + c][od*s + kd*d - p][oh*s + kh*d - p][ow*s + kw*d - p] * w[oc][c][kd][kh][kw],
 * terms outside the volume dropped.  Stride, pad and dilation apply to all three
 * directions.  layout CONV_NCHW means NCDHW tensors, CONV_NHWC means NDHWC.  The same
 * implicit matrix product as conv2d_forward runs over output voxels, its input patches
 * staged by the tensor memory accelerator's 5-D im2col mode.  bf16 NDHWC problems with
 * stride 1, unit dilation, 64 input channels, groups 1 and at most 128 output channels
 * (a multiple of 32; Ho*Wo a multiple of 32 and >= 128)
 * run on a kernel that loads each input depth slice once for all the depth taps that read
 * it (J output slices per unit of work; the sums are the same, their fp32 rounding order
 * is per tap as elsewhere).  Beyond conv2d_forward's
 * errors: CONV_ERR_UNSUPPORTED when pad or pad - dilation*(K-1) lies outside
 * [-16, 15] in any direction (the 5-D im2col addressing range). */

/* Bytes of conv3d_pack_weight's output: C_out * Kd * Kh * Kw * Cpg elements of dtype, Cpg
 * as for conv2d_packed_weight_size (group merging included, no few-channel images). */
int conv3d_packed_weight_size(int C_out, int C_in, int Kd, int Kh, int Kw, int groups,
                              conv_dtype_t dtype, size_t *bytes);

/* Packs w_oidhw (C_out, C_in/groups, Kd, Kh, Kw) into (C_out, Kd, Kh, Kw, Cpg), each tap's
 * input channels contiguous and zero-padded (the channels-last filter order). */
int conv3d_pack_weight(const void *w_oidhw, void *w_packed, int C_out, int C_in, int Kd, int Kh,
                       int Kw, int groups, conv_dtype_t dtype, conv_stream_t stream);

/* Device scratch bytes conv3d_forward needs (channels-last copy of an NCDHW or
 * channel-unaligned x, split partial sums). */
int conv3d_workspace_size(int N, int C_in, int D, int H, int W, int C_out, int Kd, int Kh,
                          int Kw, int stride, int pad, int dilation, int groups,
                          conv_dtype_t dtype, conv_layout_t layout, size_t *bytes);

/* The 3-D forward pass; arguments as conv2d_forward with the depth extents added. */
int conv3d_forward(const void *x, const void *w_packed, const void *bias, void *y,
                   int N, int C_in, int D, int H, int W, int C_out, int Kd, int Kh, int Kw,
                   int stride, int pad, int dilation, int groups,
                   conv_dtype_t dtype, conv_layout_t layout,
                   void *workspace, size_t workspace_bytes, conv_stream_t stream);

/* The plan conv3d_forward makes for a problem (conv2d_describe_plan's JSON object, with
 * "kernel": "vol_reuse" for the kernel that loads each input depth slice once for all
 * the depth taps that read it, "igemm" for the implicit GEMM over output voxels).
 * Arguments as conv3d_forward; sms and buf as conv2d_describe_plan.  Nothing runs on
 * a GPU. */
int conv3d_describe_plan(int N, int C_in, int D, int H, int W, int C_out, int Kd, int Kh, int Kw,
                         int stride, int pad, int dilation, int groups, conv_dtype_t dtype,
                         conv_layout_t layout, int sms, char *buf, size_t buflen);

/* ----------------------------------------------------------------- Winograd ---
 * The minimal-filtering form of a 3x3, stride-1, unit-dilation, ungrouped convolution
 * that the im2col/GEMM tutorial (zskr.cn/news/1820658) §5.1 sets beside im2col + GEMM:
 * F(m x m, 3 x 3) with m = 2 (16 multiplications per 2x2 output block instead of 36) or
 * m = 4 (36 instead of 144), using the published transforms of Lavin & Gray (2016),
 * Y = A^T [ (G g G^T) o (B^T d B) ] A over (m+2) x (m+2) input tiles.  The input
 * transform, the (m+2)^2 channel products (on the tensor cores, fp32 results) and the
 * output transform (+ bias, one rounding) run as three steps through the workspace.
 * Results equal conv2d_forward's up to rounding; the transforms enlarge the rounding
 * error, more for m = 4 (§5.1's numerical caveat): with bf16 data, m = 2 keeps its
 * transformed tiles and filters in bf16, while m = 4 keeps them, and runs their product,
 * in fp32 (three TF32 products), since in bf16 its error exceeds the bf16 tolerance of
 * this library (measured 6% of max |y| against 2%).  Arguments as conv2d_forward for a
 * 3x3 filter with stride 1, dilation 1 and groups 1; CONV_ERR_INVALID_ARG for m other
 * than 2 or 4. */

/* Bytes of conv2d_pack_weight_winograd's output: (m+2)^2 * C_out rows of C_in channels
 * padded to 16 bytes (times the group merge factor of conv2d_packed_weight_size for
 * C_out < 64), elements of the transform type (dtype for m = 2, fp32 for m = 4). */
int conv2d_winograd_packed_weight_size(int C_out, int C_in, int m, conv_dtype_t dtype, size_t *bytes);

/* The transformed filters U = G g G^T of w_oihw (C_out, C_in, 3, 3), packed for the
 * product.  Done once per weight. */
int conv2d_pack_weight_winograd(const void *w_oihw, void *u_packed, int C_out, int C_in, int m,
                                conv_dtype_t dtype, conv_stream_t stream);

/* Device scratch bytes conv2d_forward_winograd needs: the transformed input, the fp32
 * products and the product's own scratch. */
int conv2d_winograd_workspace_size(int N, int C_in, int H, int W, int C_out, int pad, int m,
                                   conv_dtype_t dtype, conv_layout_t layout, size_t *bytes);

/* The forward pass of a 3x3 stride-1 convolution by F(m x m, 3 x 3). */
int conv2d_forward_winograd(const void *x, const void *u_packed, const void *bias, void *y,
                            int N, int C_in, int H, int W, int C_out, int pad, int m,
                            conv_dtype_t dtype, conv_layout_t layout, void *workspace,
                            size_t workspace_bytes, conv_stream_t stream);

/* The plan of conv2d_forward_winograd's channel product (the (m+2)^2-group 1x1 product of
 * the transformed tiles), as conv2d_describe_plan's JSON object: "pointwise" where the
 * product runs on the kernel with resident weights (bf16 transforms, C_in a multiple of 64
 * up to 256, C_out a multiple of 256), else "igemm".  Arguments as conv2d_forward_winograd;
 * sms and buf as conv2d_describe_plan.  Nothing runs on the device. */
int conv2d_winograd_describe_plan(int N, int C_in, int H, int W, int C_out, int pad, int m,
                                  conv_dtype_t dtype, conv_layout_t layout, int sms, char *buf,
                                  size_t buflen);

/* Measurement aid: when `start` and `stop` (cudaEvent_t handles the caller created
 * with timing enabled) are both non-NULL, every later forward call records `start`
 * on its stream immediately before launching its tensor-core kernel and `stop`
 * immediately after it, so that the caller can time that kernel alone inside a
 * longer sequence of work.  Passing NULL, NULL turns this off.  The setting is
 * per process; events are only recorded, never waited on. */
int conv2d_set_main_kernel_events(void *start, void *stop);

/* Total number of kernels this library has launched (or, under stream capture,
 * added to a graph) in this process, written to *count. */
int conv2d_kernel_launch_count(unsigned long long *count);

/* Test hook for the watchdog: every later launch uses `timeout_ns` as the limit
 * of each device-side wait (<= 0 restores the default of 2 s) and, if
 * `starve_loads` is non-zero, issues no input loads, so the waits for them run
 * out.  Used only by the tests that check that a kernel returns an error status
 * instead of hanging. */
int conv2d_debug_set_watchdog(long long timeout_ns, int starve_loads);

/* Test hook for the choice of kernel on bf16 problems: mode 0 (the default) uses
 * the CTA-pair tensor-core kernel (clusters of two CTAs on an SM pair, M = 256
 * products) when its 256-row units still give every SM pair work, 1 uses it
 * whenever the tile shape allows it (also on problems too small to fill the
 * device, so that the tests can compare it with the oracle in full), and 2 never
 * uses it.  Results are the same in every mode up to the order of fp32 additions.
 * Returns CONV_ERR_INVALID_ARG for any other mode. */
int conv2d_debug_set_pair_mode(int mode);

/* The plan the library makes for a problem, written into buf (buflen bytes, owned by
 * the caller) as one JSON object: "kernel" ("igemm" = the implicit-GEMM tensor-core
 * kernel, "gather" = the few-channel kernel), "pair" (1: CTA-pair launch), "a_load"
 * (how the im2col operand is read: "im2col" = TMA im2col mode, "tiled_x" = x itself
 * through tiled loads, "xcol" = the explicit X_col, "gather" = software gather), "BN"
 * (output channels per tile), "cb" (bytes of channels per plane), "stages", "splits",
 * "units", "xcopy" (1: a channels-last copy of x comes first), "halo", "tma_out",
 * "Kpad", "smem" (bytes of shared memory per CTA), "workspace" (bytes) and "sms".
 * The tile and launch choices follow the same rules the forward pass applies (zskr
 * §4.3 implicit GEMM; output size per pwwt §4.2).  sms < 0 plans for this process's
 * current CUDA device (with no device: as if it had none, so without reduction splits
 * or CTA pairs); sms >= 0 plans as if the device had that many SMs.  The forward pass
 * may still fall back from CTA pairs if the device cannot co-schedule them.
 * explicit_im2col != 0 describes conv2d_forward_im2col_gemm.  Returns
 * CONV_ERR_INVALID_ARG for invalid shapes (as conv2d_forward) or a NULL / too small
 * buffer, CONV_ERR_UNSUPPORTED for unsupported problems; nothing runs on a GPU. */
int conv2d_describe_plan(int N, int C_in, int H, int W, int C_out, int Kh, int Kw, int stride,
                         int pad, int dilation, int groups, conv_dtype_t dtype, conv_layout_t layout,
                         int explicit_im2col, int sms, char *buf, size_t buflen);

#ifdef __cplusplus
}
#endif

#endif /* CONV2D_B200_H */
