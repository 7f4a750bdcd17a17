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
    CUtensorMap tmap_y;  // tma_out: y as {C_out, M}, 32 x 32 boxes with 64-byte swizzle
    int M;               // N * Ho * Wo (volumes: N * Do * Ho * Wo)
    int HoWo, Wo;        // HoWo: output pixels per image (volumes: Do * Ho * Wo)
    int HoWo2, Kh;       // volumes: Ho * Wo per output depth slice, and the filter height
    int stride, pad, dilation;  // stride: rows (and depth); columns: stride_w
    int stride_w;
    int pad_w;           // column padding (pad: row padding)
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
    int chunk_stages;    // > 0: restart the tensor-memory accumulator every this many
                         // stages and sum the chunks in fp32 registers (fp32 path)
    uint32_t tmem_cols;  // tensor-memory columns allocated (two accumulators)
    void *y;
    const void *bias;
    int out_mode;
    int vec_ok;          // 16-byte stores allowed for full chunks in NHWC / partial mode
    int tma_out;         // bf16 NHWC output staged in shared memory and stored by TMA
    int *status;
    long long timeout_ns;
    int starve;          // test hook: issue no loads
};

// One launch of the volume kernel with input-slice reuse (vol.cu): 3-D, bf16, stride 1,
// unit dilation, C_in = 64, groups = 1, channels-last.  A unit is J output depth slices
// of one 128-voxel tile of a depth slice; u = (n*n_odb + b)*n_k + k.
struct VolParams {
    CUtensorMap tmap_a;  // 5-D im2col map of x (c, w, h, d, n), boxes of 128 voxels x 64 channels
    CUtensorMap tmap_b;  // packed weights {taps*64, C_out, 1}, boxes of 64 x C_out
    CUtensorMap tmap_y;  // y as {C_out, M}, 32 x 32 boxes with 64-byte swizzle
    int M, Do, HoWo2, Wo;
    int Kd, Kh, Kw, taps, pad, pad_w;
    int BN;              // = C_out (a multiple of 32, <= 128)
    int J;               // output depth slices per unit (accumulators: nacc*J*BN columns)
    int nacc;            // accumulator sets: 2 (the epilogue of one unit overlaps the next) or 1
    int n_k, n_odb, units, stages;
    uint32_t tmem_cols;
    const void *bias;
    int *status;
    long long timeout_ns;
    int starve;
};

// One launch of the pointwise kernel (pw.cu): 1x1, stride 1, no padding, bf16 operands,
// channels-last, per group C_in = 64*nk (nk <= 4) and C_out a multiple of BN = 256, CTA
// pairs.  Cluster c keeps (group, column tile) c % (groups*n_ntiles) resident and takes row
// tiles c / (groups*n_ntiles) + i*cpn.
struct PwParams {
    CUtensorMap tmap_a;  // x as X_col {groups*Kp, M}, boxes of {64, 128}, 128-byte swizzle
    CUtensorMap tmap_b;  // packed weights {Kp, Cout_g, groups}, boxes of {64, BN/2, 1}, 128-byte swizzle
    CUtensorMap tmap_y;  // y as {C_out, M}, boxes of 32 rows x 128 bytes, 128-byte swizzle
    int M, nk, BN, n_ntiles, m_tiles, cpn, stages;
    int groups, Kp, Cout_g;
    int out_f32;         // the raw fp32 sums (no bias) instead of bf16 + bias
    int ybufs;           // output staging blocks per epilogue warp (1 or 2)
    uint32_t tmem_cols;
    const void *bias;
    int *status;
    long long timeout_ns;
    int starve;
};

// One launch of the software-gather kernel (gather.cu) for inputs with few
// channels: groups = 1, reduction index k = (kh*Kw + kw)*C + c (or the row-vector
// order), padded to Kpad.
struct GatherParams {
    CUtensorMap tmap_x;    // halo mode: 4-D tiled map of x (W, H, C, N)
    CUtensorMap tmap_y;    // tma_out mode: 3-D tiled map of y (Ho*Wo, C_out, N); gather_t: 4-D (Wo, Ho, C_out, N)
    const void *x;
    const void *w_packed;  // (C_out, Kh, Kw, Cpg) from conv2d_pack_weight
    const void *w_image;   // the kernel's shared-memory weight image (written by the pack)
    int N, C, H, W, Kh, Kw, stride, pad, dilation;
    int Ho, Wo, M;
    int Cpg;               // channel pitch of w_packed
    int Kc, Kpad;          // C*Kh*Kw and its length padded to a 32-byte multiple
    int BN, n_mtiles;
    int stages;            // A slots in tensor memory
    int acols;             // tensor-memory columns per A slot
    int in_nchw;
    int vec_rows;          // row-vector gather: k = (c*Kh + kh)*(16/elt) + kw, see gather.cu
    int halo;              // input rows staged in shared memory by TMA (needs vec_rows)
    int R, BW, ME;         // halo rows, row width (elements) and left zero margin
    int tma_out;           // epilogue stages each tile channel-major and stores it by TMA
    int cw;                // output channels per epilogue group
    int tpix;              // transposed kernel (gather_t.cu): pixels per tile, Wo rounded up to 16
    int nhalo;             // ... its staged-row buffers (loads run this many tiles ahead)
    int nacc;              // ... its accumulators in tensor memory
    int nout;              // ... its output images (tma_out)
    int rt;                // ... output rows per tile (1, or 2 when C_out <= 64)
    int kt;                // ... the reduction length of a tile's product (padded)
    int a_tmem;            // ... and whether A is resident in tensor memory
    uint32_t tmem_cols;
    void *y;
    const void *bias;
    int Cout, out_mode, vec_ok;
    int *status;
    long long timeout_ns;
    int starve;
};

// One launch of the depthwise kernel (depthwise.cu): groups = C_in = C_out, x
// channels-last with Cp >= C channels per pixel (a multiple of 16 bytes).  Tiles are
// TH x TW output pixels x 128 bytes of channels; tile u = ((chunk*N + n)*n_th + th)*n_tw + tw.
struct DwParams {
    CUtensorMap tmap_x;    // x as {Cp, W, H, N}, boxes of {128 bytes, IW, IH, 1}
    const void *w_packed;  // (C, Kh, Kw, Cpg) from conv2d_pack_weight
    const void *bias;
    void *y;
    int N, C, Ho, Wo, Kh, Kw, stride, pad, dilation;
    int pad_w;             // column padding (pad: row padding)
    int Cpg;               // channel pitch of w_packed
    int TH, TW, IH, IW;    // output tile and the staged input box
    int n_th, n_tw, units, stages;
    int wregion;           // bytes of the per-warp weight copies ahead of the stage ring
    int out_nchw, vec_ok;
    int *status;
    long long timeout_ns;
    int starve;
};

// One launch of the weight-gradient kernel (wgrad.cu): per group, dW_row = dout_col X_col^T
// with the reduction over output pixels in stages of PK (64 bf16 / 32 fp32), written as
// fp32 partial sums ws[split][C_out][taps][Cpg].  Unit u = (((split*n_otiles + otile)*groups
// + g)*taps + tap)*n_ctiles + ctile.
struct WgradParams {
    CUtensorMap tmap_dy;   // dy channels-last as {groups*dy_cpg, M}, boxes of {128 bytes, PK}, 128-byte swizzle
    CUtensorMap tmap_x;    // im2col map of channels-last x ({groups*Cpg, W, H, N}), PK pixels x 128 bytes
    float *ws;
    int M, HoWo, Wo, stride, pad, dilation, Kw, taps;
    int Cpg;               // channels per group of the x tensor read (multiple of 128 bytes)
    int dy_cpg;            // channels per group of the dy tensor read (multiple of 16 bytes)
    int Cout, Cout_g, groups;
    int BN;                // channels per tile (multiple of 128 bytes; <= 256 bf16, <= 128 fp32)
    int n_ctiles, n_otiles, kstages, splits, units, stages, chunk_stages;
    int om;                // 128-row output-channel tiles per unit (1, or 2 in bf16); n_otiles counts units' worth
    uint32_t tmem_cols;
    int *status;
    long long timeout_ns;
    int starve;
};

// Launchers (igemm.cu, gather.cu, layout.cu).  All return cudaSuccess or the launch error.
// pair: bf16 only, grid even, launched as clusters of two CTAs (p.n_mtiles counts
// 256-row units, the tensor map of B has boxes of BN/2 rows).  vol: 5-D (volumetric)
// im2col map, filter taps stepped over (kd, kh, kw); needs im2col.
cudaError_t launch_igemm(const IgemmParams &p, bool f32, int cb_bytes, bool im2col, bool pair, int grid,
                         size_t smem_bytes, cudaStream_t stream, bool vol = false);
// Bytes of dynamic shared memory for `stages` stages holding BN rows of B each.
size_t igemm_smem_bytes(bool f32, int BN, int stages, bool tma_out);
// Two-CTA clusters of the pair kernel that can be resident at once.
cudaError_t igemm_pair_max_clusters(int cb_bytes, bool im2col, size_t smem_bytes, int *clusters, bool vol = false);
cudaError_t launch_gather(const GatherParams &p, bool f32, int grid, size_t smem, cudaStream_t stream);
// The (kd, kh)-fold of a few-channel 3-D input into xf [N][Do*Ho][W][Cf] (channels-last),
// and of its packed weights wp [Cout][Kd*Kh*Kw][cpg] into the 2-D packed layout
// wf [Cout][Kw][Cf], in one launch (layout.cu).
cudaError_t launch_fold3d(const void *x, void *xf, const void *wp, void *wf, int N, int C, int D, int H, int W,
                          int Do, int Ho, int Cout, int Kd, int Kh, int Kw, int cpg, int stride, int pad, int dilation,
                          int Cf, int elt, bool nchw, cudaStream_t s);
size_t gather_smem_bytes(bool f32, int BN, int Kpad, size_t halo_bytes, size_t out_stage_bytes);
// The transposed few-channel kernel (gather_t.cu): bf16, NCHW in and out, one output row
// per tile, output channels on the tensor-memory lanes.
cudaError_t launch_gather_t(const GatherParams &p, int grid, size_t smem, cudaStream_t stream);
cudaError_t launch_vol_reuse(const VolParams &p, int grid, size_t smem, cudaStream_t stream);
cudaError_t launch_pw(const PwParams &p, size_t smem, cudaStream_t stream);
cudaError_t pw_max_clusters(size_t smem, bool out_f32, int *clusters);
size_t pw_smem_bytes(int nk, int BN, int stages, bool out_f32, int ybufs);
int pw_max_stages();
int pw_max_planes();
size_t vol_reuse_smem_bytes(int Kd, int BN, int stages);
int vol_reuse_max_stages();
int vol_reuse_max_j();
size_t gather_t_smem_bytes(int kt, int tpix, size_t halo_bytes, int nhalo, size_t out_bytes, int nout, bool a_tmem);
int gather_t_max_halo();
int gather_t_max_acc();
int gather_t_max_chunks();
int gather_max_stages();
int igemm_threads(bool f32);

// window_k: 3, 5 or 7 for the register-window form (stride 1, unit dilation, square
// filter), 0 for the general form.
cudaError_t launch_depthwise(const DwParams &p, bool f32, int window_k, int grid, size_t smem,
                             cudaStream_t stream);
int dw_pixels_per_thread();
int dw_threads();
int dw_compute_warps();
int dw_max_stages();
size_t dw_header_bytes();

cudaError_t launch_wgrad(const WgradParams &p, bool f32, int grid, size_t smem, cudaStream_t stream);
size_t wgrad_smem_bytes(bool f32, int BN, int stages, int om);
int wgrad_pixels_per_stage(bool f32);
int wgrad_max_stages();
// Weight gradient on the CUDA cores for few channels per group: partial sums
// ws[split][C_out][Kh*Kw][C_in/groups] from channels-last x and dy.
cudaError_t launch_wgrad_direct(const void *x, const void *dy, float *ws, int N, int C_in, int H, int W, int C_out,
                                int Ho, int Wo, int Kh, int Kw, int stride, int pad, int dilation, int groups,
                                int splits, bool f32, cudaStream_t s);
cudaError_t launch_wgrad_reduce(const float *ws, void *dw, int Cout, int Cin_g, int taps, int Cpg, int splits,
                                bool f32, cudaStream_t s);
// Bias gradient db[c] = sum of dy over images and output positions: partials (count from
// bias_grad_partials, times C floats of scratch), then their sum in the bias type.
int bias_grad_partials(long long rows, int C, int N, bool nchw);
cudaError_t launch_bias_grad(const void *dy, float *partial, void *db, int N, int C, long long plane, bool nchw,
                             bool f32, cudaStream_t s);
cudaError_t launch_zero_insert(const void *dy, void *dyz, int N, int C, int Ho, int Wo, int Hz, int Wz, int stride,
                               bool nchw, int elt, cudaStream_t s);
cudaError_t launch_pack_weight_t(const void *w, void *wp, int O, int R, int Cin_g, int gm, int Kh, int Kw, int Cpg,
                                 int elt, cudaStream_t s);

// Winograd F(m x m, 3 x 3) transforms (winograd.cu), m = 2 or 4.
// f32: the data type; v_f32 / u_f32: the transform type (fp32 whenever the data is fp32).
cudaError_t launch_wino_input(const void *x, void *v, int N, int C, int H, int W, int Cpg, int TH, int TW, int pad,
                              int m, bool nchw, bool f32, bool v_f32, cudaStream_t s);
cudaError_t launch_wino_weight(const void *w, void *u, int C_out, int C, int Cpg, int gm, int m, bool f32, bool u_f32,
                               cudaStream_t s);
cudaError_t launch_wino_output(const float *mp, const void *bias, void *y, int N, int C_out, int Ho, int Wo, int TH,
                               int TW, int splits, int m, bool nchw, bool f32, cudaStream_t s);

cudaError_t launch_nchw_to_nhwc(const void *src, void *dst, int N, int C, int H, int W,
                                int groups, int Cpg, int elt, cudaStream_t s);
cudaError_t launch_nhwc_pad(const void *src, void *dst, int N, int C, int H, int W, int groups,
                            int Cpg, int elt, cudaStream_t s);
cudaError_t launch_nhwc_to_nchw(const void *src, void *dst, int N, int C, int H, int W, int elt,
                                cudaStream_t s);
// gm > 1: groups merged gm at a time, block-diagonal (see group_merge in abi.cu).
cudaError_t launch_pack_weight(const void *w, void *wp, int Cout, int Cin_g, int Cout_g, int gm, int Kh,
                               int Kw, int Cpg, int elt, cudaStream_t s);
cudaError_t launch_pack_gather_image(const void *w, void *img, int Cout, int C, int Kh, int Kw,
                                     int BN, int Kpad, bool rowvec, int elt, cudaStream_t s);
cudaError_t launch_im2col(const void *x_nhwc, void *xcol, int N, int H, int W, int groups,
                          int Cpg, int Ho, int Wo, int Kh, int Kw, int stride, int pad,
                          int dilation, int elt, cudaStream_t s);
cudaError_t launch_splitk_reduce(const float *ws, const void *bias, void *y, int M, int Cout,
                                 int HoWo, int splits, int out_mode, bool f32, cudaStream_t s);

}  // namespace conv2d_b200
