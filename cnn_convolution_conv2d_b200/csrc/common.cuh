// common.cuh -- definitions shared by the kernels and the host-side dispatcher.
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

namespace conv2d_b200 {

// Output forms of the matrix-product epilogue.
enum OutMode : int {
    kOutNHWC = 0,     // y[m][oc], m = (n, oh, ow)
    kOutNCHW = 1,     // y[n][oc][oh][ow]
    kOutPartial = 2,  // fp32 partial sums ws[split][m][oc], no bias
};

// Watchdog status codes written by device code (0 = fine).
enum DeviceStatus : int {
    kDevOk = 0,
    kDevTimeoutFull = 1,     // the tensor-core warp waited too long for a stage's loads
    kDevTimeoutEmpty = 2,    // the load warp waited too long for a free stage
    kDevTimeoutAccFull = 3,  // the epilogue waited too long for an accumulator
    kDevTimeoutAccEmpty = 4, // the tensor-core warp waited too long for a free accumulator
    kDevTimeoutConvert = 5,  // fp32 split warps waited too long
    kDevBadCoordinate = 6,   // a load coordinate failed the 16-byte rule (load skipped)
};

// Everything one launch of the implicit-GEMM kernel needs.  Rows of the
// product are output pixels m = (n*Ho + oh)*Wo + ow; columns are the output
// channels of one group; the reduction runs over planes, a plane being one
// filter tap times one block of CB bytes of input channels.
struct IgemmParams {
    CUtensorMap tmap_a;  // A operand: im2col-mode map of x (NHWC) or tiled map of X_col
    CUtensorMap tmap_b;  // B operand: tiled map of the packed weights {Kp, Cout_g, groups}
    int M;               // N * Ho * Wo
    int HoWo, Wo;
    int stride, pad, dilation;
    int Kw, taps;        // taps = Kh * Kw
    int Cpg;             // padded input channels per group (elements)
    int nCB;             // channel blocks per tap
    int planes;          // taps * nCB
    int kstages;         // ceil(planes / planes-per-stage)
    int Kp;              // taps * Cpg: reduction length of one group (elements)
    int groups, Cout_g, Cout;
    int BN;              // output channels per tile (multiple of 16, <= 256)
    int n_mtiles, n_ntiles, splits, units;
    int stages;          // depth of the shared-memory ring
    uint32_t tmem_cols;  // tensor-memory columns allocated (two accumulators)
    void *y;
    const void *bias;
    int out_mode;
    int vec_ok;          // 16-byte stores allowed for full chunks in NHWC / partial mode
    int *status;
    long long timeout_ns;
    int starve;          // test hook: issue no loads
};

// Launchers (igemm.cu, layout.cu).  All return cudaSuccess or the launch error.
cudaError_t launch_igemm(const IgemmParams &p, bool f32, int cb_bytes, bool im2col, int grid,
                         size_t smem_bytes, cudaStream_t stream);
size_t igemm_smem_bytes(bool f32, int BN, int stages);
int igemm_threads(bool f32);

cudaError_t launch_nchw_to_nhwc(const void *src, void *dst, int N, int C, int H, int W,
                                int groups, int Cpg, int elt, cudaStream_t s);
cudaError_t launch_nhwc_pad(const void *src, void *dst, int N, int C, int H, int W, int groups,
                            int Cpg, int elt, cudaStream_t s);
cudaError_t launch_nhwc_to_nchw(const void *src, void *dst, int N, int C, int H, int W, int elt,
                                cudaStream_t s);
cudaError_t launch_pack_weight(const void *w, void *wp, int Cout, int Cin_g, int Kh, int Kw,
                               int Cpg, int elt, cudaStream_t s);
cudaError_t launch_im2col(const void *x_nhwc, void *xcol, int N, int H, int W, int groups,
                          int Cpg, int Ho, int Wo, int Kh, int Kw, int stride, int pad,
                          int dilation, int elt, cudaStream_t s);
cudaError_t launch_splitk_reduce(const float *ws, const void *bias, void *y, int M, int Cout,
                                 int HoWo, int splits, int out_mode, bool f32, cudaStream_t s);

}  // namespace conv2d_b200
