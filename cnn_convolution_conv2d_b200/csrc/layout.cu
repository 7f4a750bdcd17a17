// layout.cu -- bandwidth-bound helper kernels around the tensor-core product:
//   * NCHW -> channels-last with per-group zero channel padding ("layout in");
//   * channels-last -> NCHW ("layout out", zskr §3.2 step 5);
//   * weight packing OIHW -> (oc, kh, kw, c) with zero channel padding;
//   * explicit im2col (the pages' X_col, one row per output pixel);
//   * the depth-and-row fold of a few-channel 3-D input (partial im2col) and its weights;
//   * the fp32 reduction of split partial sums, + bias, in the output layout.
// All are plain coalesced CUDA-core kernels with grid-stride loops; none reads or
// writes outside the extents passed in.
#include <cuda_bf16.h>

#include "common.cuh"

namespace conv2d_b200 {
namespace {

constexpr int kThreads = 256;
constexpr int kBiasRows = 512;  // rows of channels-last dy summed per block of the bias gradient

inline int grid_for(long long work, int per_block = kThreads) {
    long long g = (work + per_block - 1) / per_block;
    if (g < 1) g = 1;
    if (g > 148LL * 64) g = 148LL * 64;  // grid-stride loops cover the rest
    return static_cast<int>(g);
}

// --- Transpose of the two inner dimensions of a [B][R][S] array of 2-byte elements
// into [B][S][R] (NCHW -> NHWC with R = C, S = H*W; NHWC -> NCHW with R = H*W, S = C),
// for R and S multiples of 8.  64 x 64 tiles through shared memory; every global access
// is a 16-byte vector, and each warp touches four 128-byte rows per instruction.  In
// shared memory the tile is 64 rows of 32 words (two elements per word); word w of row r
// sits at column w ^ (r & 31), so that the row-wise stores are conflict-free and the
// column-wise reads at most two-way.
__global__ void __launch_bounds__(256) transpose_b16_kernel(const uint16_t *__restrict__ src,
                                                            uint16_t *__restrict__ dst, int B, int R, int S) {
    __shared__ uint32_t tile[64][32];
    const int tiles_r = (R + 63) / 64, tiles_s = (S + 63) / 64;
    const long long per_b = static_cast<long long>(tiles_r) * tiles_s;
    const long long ntiles = static_cast<long long>(B) * per_b;
    const int t = threadIdx.x;
    for (long long tt = blockIdx.x; tt < ntiles; tt += gridDim.x) {
        const long long b = tt / per_b;
        const int rem = static_cast<int>(tt - b * per_b);
        const int r0 = (rem / tiles_s) * 64, s0 = (rem - (rem / tiles_s) * tiles_s) * 64;
        const uint16_t *sb = src + b * static_cast<long long>(R) * S;
        uint16_t *db = dst + b * static_cast<long long>(R) * S;
#pragma unroll
        for (int k = 0; k < 2; ++k) {  // 64 source rows x 8 vectors of 8 elements
            const int row = (t >> 3) + 32 * k, vec = t & 7;
            const int r = r0 + row, c = s0 + 8 * vec;
            uint4 v = make_uint4(0u, 0u, 0u, 0u);
            if (r < R && c < S) v = __ldg(reinterpret_cast<const uint4 *>(sb + static_cast<long long>(r) * S + c));
            const int sw = row & 31;
            tile[row][(4 * vec + 0) ^ sw] = v.x;
            tile[row][(4 * vec + 1) ^ sw] = v.y;
            tile[row][(4 * vec + 2) ^ sw] = v.z;
            tile[row][(4 * vec + 3) ^ sw] = v.w;
        }
        __syncthreads();
        {  // 64 destination rows (pairs per thread) x 8 vectors of 8 elements
            const int vec = t & 7, wj = t >> 3;  // source rows 8*vec..+7, source word column wj
            uint32_t w[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const int row = 8 * vec + i;
                w[i] = tile[row][wj ^ (row & 31)];
            }
            const int r = r0 + 8 * vec;
            const int c = s0 + 2 * wj;  // destination rows c and c + 1
            if (r < R) {
                if (c < S) {
                    const uint4 lo = make_uint4(__byte_perm(w[0], w[1], 0x5410), __byte_perm(w[2], w[3], 0x5410),
                                                __byte_perm(w[4], w[5], 0x5410), __byte_perm(w[6], w[7], 0x5410));
                    *reinterpret_cast<uint4 *>(db + static_cast<long long>(c) * R + r) = lo;
                }
                if (c + 1 < S) {
                    const uint4 hi = make_uint4(__byte_perm(w[0], w[1], 0x7632), __byte_perm(w[2], w[3], 0x7632),
                                                __byte_perm(w[4], w[5], 0x7632), __byte_perm(w[6], w[7], 0x7632));
                    *reinterpret_cast<uint4 *>(db + static_cast<long long>(c + 1) * R + r) = hi;
                }
            }
        }
        __syncthreads();
    }
}

// --- The same for 4-byte elements (R and S multiples of 4): 32 x 32 tiles, one
// 16-byte vector (4 elements) per thread in each direction; word c of row r sits at
// column c ^ (r & 31), conflict-free both ways.
__global__ void __launch_bounds__(256) transpose_b32_kernel(const uint32_t *__restrict__ src,
                                                            uint32_t *__restrict__ dst, int B, int R, int S) {
    __shared__ uint32_t tile[32][32];
    const int tiles_r = (R + 31) / 32, tiles_s = (S + 31) / 32;
    const long long per_b = static_cast<long long>(tiles_r) * tiles_s;
    const long long ntiles = static_cast<long long>(B) * per_b;
    const int t = threadIdx.x;
    for (long long tt = blockIdx.x; tt < ntiles; tt += gridDim.x) {
        const long long b = tt / per_b;
        const int rem = static_cast<int>(tt - b * per_b);
        const int r0 = (rem / tiles_s) * 32, s0 = (rem - (rem / tiles_s) * tiles_s) * 32;
        const uint32_t *sb = src + b * static_cast<long long>(R) * S;
        uint32_t *db = dst + b * static_cast<long long>(R) * S;
        {  // 32 source rows x 8 vectors of 4 elements
            const int row = t >> 3, vec = t & 7;
            const int r = r0 + row, c = s0 + 4 * vec;
            uint4 v = make_uint4(0u, 0u, 0u, 0u);
            if (r < R && c < S) v = __ldg(reinterpret_cast<const uint4 *>(sb + static_cast<long long>(r) * S + c));
            const int sw = row & 31;
            tile[row][(4 * vec + 0) ^ sw] = v.x;
            tile[row][(4 * vec + 1) ^ sw] = v.y;
            tile[row][(4 * vec + 2) ^ sw] = v.z;
            tile[row][(4 * vec + 3) ^ sw] = v.w;
        }
        __syncthreads();
        {  // 32 destination rows x 8 vectors of 4 elements
            const int vec = t & 7, col = t >> 3;  // source rows 4*vec..+3, source column col
            uint32_t w[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int row = 4 * vec + i;
                w[i] = tile[row][col ^ (row & 31)];
            }
            const int r = r0 + 4 * vec, c = s0 + col;
            if (r < R && c < S)
                *reinterpret_cast<uint4 *>(db + static_cast<long long>(c) * R + r) = make_uint4(w[0], w[1], w[2], w[3]);
        }
        __syncthreads();
    }
}

void launch_transpose_b32(const void *src, void *dst, int B, int R, int S, cudaStream_t s) {
    const long long tiles = static_cast<long long>(B) * ((R + 31) / 32) * ((S + 31) / 32);
    const int grid = static_cast<int>(tiles < 148LL * 8 ? tiles : 148LL * 8);
    transpose_b32_kernel<<<grid, 256, 0, s>>>(static_cast<const uint32_t *>(src), static_cast<uint32_t *>(dst), B, R, S);
}

void launch_transpose_b16(const void *src, void *dst, int B, int R, int S, cudaStream_t s) {
    const long long tiles = static_cast<long long>(B) * ((R + 63) / 64) * ((S + 63) / 64);
    const int grid = static_cast<int>(tiles < 148LL * 8 ? tiles : 148LL * 8);
    transpose_b16_kernel<<<grid, 256, 0, s>>>(static_cast<const uint16_t *>(src), static_cast<uint16_t *>(dst), B, R, S);
}

template <int kElt> struct Word;
template <> struct Word<2> { using T = uint16_t; };
template <> struct Word<4> { using T = uint32_t; };

// --- NCHW -> channels-last, small padded channel counts (Ctot * elt <= 64 bytes):
// one thread per pixel; reads are coalesced across the warp (consecutive pixels of
// one channel plane), each pixel's Ctot channels are written as 16-byte words.
template <int kElt>
__global__ void nchw_to_nhwc_small(const void *__restrict__ src, void *__restrict__ dst, int N,
                                   int C, int HW, int groups, int Cpg) {
    using T = typename Word<kElt>::T;
    const T *s = static_cast<const T *>(src);
    T *d = static_cast<T *>(dst);
    const int Cg = C / groups;
    const int Ctot = groups * Cpg;
    const long long total = static_cast<long long>(N) * HW;
    for (long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; i < total;
         i += static_cast<long long>(gridDim.x) * blockDim.x) {
        const long long n = i / HW;
        const long long pix = i - n * HW;
        alignas(16) T vals[64 / kElt];
        for (int cc = 0; cc < Ctot; ++cc) {
            const int g = cc / Cpg, c = cc - g * Cpg;
            vals[cc] = c < Cg ? s[(n * C + g * Cg + c) * HW + pix] : T(0);
        }
        uint4 *d4 = reinterpret_cast<uint4 *>(d + i * Ctot);
        const uint4 *v4 = reinterpret_cast<const uint4 *>(vals);
        for (int k = 0; k < Ctot * kElt / 16; ++k) d4[k] = v4[k];
    }
}

// --- NCHW -> channels-last, general: 32 x 32 tiles through shared memory.
// Block (32, 8); tile = 32 destination channels x 32 pixels of one image.
template <int kElt>
__global__ void nchw_to_nhwc_tiled(const void *__restrict__ src, void *__restrict__ dst, int N,
                                   int C, int HW, int groups, int Cpg) {
    using T = typename Word<kElt>::T;
    __shared__ T tile[32][33];
    const T *s = static_cast<const T *>(src);
    T *d = static_cast<T *>(dst);
    const int Cg = C / groups;
    const int Ctot = groups * Cpg;
    const int tiles_c = (Ctot + 31) / 32, tiles_p = (HW + 31) / 32;
    const long long ntiles = static_cast<long long>(N) * tiles_c * tiles_p;
    for (long long t = blockIdx.x; t < ntiles; t += gridDim.x) {
        const long long n = t / (static_cast<long long>(tiles_c) * tiles_p);
        const int r = static_cast<int>(t - n * tiles_c * tiles_p);
        const int c0 = (r / tiles_p) * 32, p0 = (r % tiles_p) * 32;
        for (int k = threadIdx.y; k < 32; k += 8) {  // read: channel rows, pixel columns
            const int cc = c0 + k, pix = p0 + threadIdx.x;
            T v = T(0);
            if (cc < Ctot && pix < HW) {
                const int g = cc / Cpg, c = cc - g * Cpg;
                if (c < Cg) v = s[(n * C + g * Cg + c) * HW + pix];
            }
            tile[k][threadIdx.x] = v;
        }
        __syncthreads();
        for (int k = threadIdx.y; k < 32; k += 8) {  // write: pixel rows, channel columns
            const int pix = p0 + k, cc = c0 + threadIdx.x;
            if (pix < HW && cc < Ctot) d[(n * HW + pix) * Ctot + cc] = tile[threadIdx.x][k];
        }
        __syncthreads();
    }
}

// --- channels-last C -> channels-last groups*Cpg (zero channels appended per group).
template <int kElt>
__global__ void nhwc_pad_kernel(const void *__restrict__ src, void *__restrict__ dst,
                                long long pixels, int C, int groups, int Cpg) {
    using T = typename Word<kElt>::T;
    const T *s = static_cast<const T *>(src);
    T *d = static_cast<T *>(dst);
    const int Cg = C / groups;
    const int Ctot = groups * Cpg;
    const long long total = pixels * Ctot;
    for (long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; i < total;
         i += static_cast<long long>(gridDim.x) * blockDim.x) {
        const long long pix = i / Ctot;
        const int cc = static_cast<int>(i - pix * Ctot);
        const int g = cc / Cpg, c = cc - g * Cpg;
        d[i] = c < Cg ? s[pix * C + g * Cg + c] : T(0);
    }
}

// --- channels-last -> NCHW: 32 x 32 tiles through shared memory.
template <int kElt>
__global__ void nhwc_to_nchw_tiled(const void *__restrict__ src, void *__restrict__ dst, int N,
                                   int C, int HW) {
    using T = typename Word<kElt>::T;
    __shared__ T tile[32][33];
    const T *s = static_cast<const T *>(src);
    T *d = static_cast<T *>(dst);
    const int tiles_c = (C + 31) / 32, tiles_p = (HW + 31) / 32;
    const long long ntiles = static_cast<long long>(N) * tiles_c * tiles_p;
    for (long long t = blockIdx.x; t < ntiles; t += gridDim.x) {
        const long long n = t / (static_cast<long long>(tiles_c) * tiles_p);
        const int r = static_cast<int>(t - n * tiles_c * tiles_p);
        const int c0 = (r / tiles_p) * 32, p0 = (r % tiles_p) * 32;
        for (int k = threadIdx.y; k < 32; k += 8) {  // read: pixel rows, channel columns
            const int pix = p0 + k, c = c0 + threadIdx.x;
            tile[k][threadIdx.x] = (pix < HW && c < C) ? s[(n * HW + pix) * C + c] : T(0);
        }
        __syncthreads();
        for (int k = threadIdx.y; k < 32; k += 8) {  // write: channel rows, pixel columns
            const int c = c0 + k, pix = p0 + threadIdx.x;
            if (c < C && pix < HW) d[(n * C + c) * HW + pix] = tile[threadIdx.x][k];
        }
        __syncthreads();
    }
}

// --- weights OIHW (Cout, Cin_g, Kh, Kw) -> (Cout, Kh, Kw, Cpg), zero for c >= Cin_g.  With
// groups merged gm at a time (gm > 1), Cpg = gm * Cin_g and output channel oc keeps its
// weights in block j = (oc / Cout_g) % gm of its row, zeros elsewhere (block-diagonal).
template <int kElt>
__global__ void pack_weight_kernel(const void *__restrict__ w, void *__restrict__ wp, int Cout,
                                   int Cin_g, int Cout_g, int gm, int Kh, int Kw, int Cpg) {
    using T = typename Word<kElt>::T;
    const T *s = static_cast<const T *>(w);
    T *d = static_cast<T *>(wp);
    const long long total = static_cast<long long>(Cout) * Kh * Kw * Cpg;
    for (long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; i < total;
         i += static_cast<long long>(gridDim.x) * blockDim.x) {
        const int c = static_cast<int>(i % Cpg);
        long long r = i / Cpg;
        const int kw = static_cast<int>(r % Kw);
        r /= Kw;
        const int kh = static_cast<int>(r % Kh);
        const long long oc = r / Kh;
        // merged groups: output channel oc belongs to sub-group j of its merged group and
        // sees only that sub-group's Cin_g channels (block-diagonal)
        const int j = static_cast<int>((oc / Cout_g) % gm);
        const int cl = c - j * Cin_g;
        d[i] = (cl >= 0 && cl < Cin_g) ? s[((oc * Cin_g + cl) * Kh + kh) * Kw + kw] : T(0);
    }
}

// --- weight image of the software-gather kernel: OIHW (Cout, C, Kh, Kw) ->
// the tensor cores' no-swizzle K-major shared-memory layout of a BN x Kpad matrix
// (8-row groups `nchunks * 128` bytes apart, 16-byte k chunks 128 bytes apart,
// rows 16 bytes apart), k in the compact order (kh*Kw + kw)*C + c or the row-vector
// order (c*Kh + kh)*kPer + kw, zero where k or the row is padding.  fp32 weights
// become two images, tf32 hi then lo.
template <int kElt>
__global__ void pack_gather_image_kernel(const void *__restrict__ w, uint8_t *__restrict__ img,
                                         int Cout, int C, int Kh, int Kw, int BN, int Kpad,
                                         int rowvec) {
    constexpr int kPer = 16 / kElt;
    const int nchunks = Kpad / kPer;
    const size_t image_bytes = static_cast<size_t>(BN) * Kpad * kElt;
    for (long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x;
         i < static_cast<long long>(BN) * nchunks; i += static_cast<long long>(gridDim.x) * blockDim.x) {
        const int oc = static_cast<int>(i / nchunks), j = static_cast<int>(i % nchunks);
        float v[kPer];
        uint32_t u[kPer];
        for (int e = 0; e < kPer; ++e) {
            int c, kh, kw;
            bool real = oc < Cout;
            if (rowvec) {
                c = j / Kh;
                kh = j % Kh;
                kw = e;
                real = real && j < C * Kh && e < Kw;
            } else {
                const int k = j * kPer + e;
                const int tap = k / C;
                c = k % C;
                kh = tap / Kw;
                kw = tap % Kw;
                real = real && k < C * Kh * Kw;
            }
            const size_t src = ((static_cast<size_t>(oc) * C + c) * Kh + kh) * Kw + kw;
            if (kElt == 4) {
                v[e] = real ? static_cast<const float *>(w)[src] : 0.f;
            } else {
                u[e] = real ? static_cast<const unsigned short *>(w)[src] : 0u;
            }
        }
        const size_t off = static_cast<size_t>(oc >> 3) * nchunks * 128 + static_cast<size_t>(j) * 128 +
                           static_cast<size_t>(oc & 7) * 16;
        if (kElt == 4) {
            float hi[4], lo[4];
            for (int e = 0; e < 4; ++e) {
                hi[e] = __uint_as_float((__float_as_uint(v[e]) + 0x1000u) & 0xFFFFE000u);
                const float r = v[e] - hi[e];
                lo[e] = __uint_as_float((__float_as_uint(r) + 0x1000u) & 0xFFFFE000u);
            }
            *reinterpret_cast<float4 *>(img + off) = make_float4(hi[0], hi[1], hi[2], hi[3]);
            *reinterpret_cast<float4 *>(img + image_bytes + off) = make_float4(lo[0], lo[1], lo[2], lo[3]);
        } else {
            uint32_t wds[4];
            for (int e = 0; e < 4; ++e) wds[e] = u[2 * e] | (u[2 * e + 1] << 16);
            *reinterpret_cast<uint4 *>(img + off) = make_uint4(wds[0], wds[1], wds[2], wds[3]);
        }
    }
}

// --- explicit im2col: xcol[m][g*Kp + (kh*Kw + kw)*Cpg + c] = x[n][ih][iw][g*Cpg + c]
// (0 outside the image), m = (n*Ho + oh)*Wo + ow.  One thread per 16-byte chunk; a
// chunk never straddles two taps because Cpg*elt is a multiple of 16.
template <int kElt>
__global__ void im2col_kernel(const void *__restrict__ x, void *__restrict__ xcol, int N, int H,
                              int W, int groups, int Cpg, int Ho, int Wo, int Kh, int Kw,
                              int stride, int pad, int dilation) {
    constexpr int kPer = 16 / kElt;  // elements per chunk
    const int Kp = Kh * Kw * Cpg;
    const int row_chunks = groups * Kp / kPer;
    const int Ctot = groups * Cpg;
    const long long total = static_cast<long long>(N) * Ho * Wo * row_chunks;
    const uint4 *xs = static_cast<const uint4 *>(x);
    uint4 *d = static_cast<uint4 *>(xcol);
    for (long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; i < total;
         i += static_cast<long long>(gridDim.x) * blockDim.x) {
        const long long m = i / row_chunks;
        const int k = static_cast<int>(i - m * row_chunks) * kPer;  // element column
        const int g = k / Kp;
        const int kr = k - g * Kp;
        const int tap = kr / Cpg, c = kr - tap * Cpg;
        const int kh = tap / Kw, kw = tap - kh * Kw;
        const int n = static_cast<int>(m / (static_cast<long long>(Ho) * Wo));
        const int rem = static_cast<int>(m - static_cast<long long>(n) * Ho * Wo);
        const int oh = rem / Wo, ow = rem - (rem / Wo) * Wo;
        const int ih = oh * stride + kh * dilation - pad;
        const int iw = ow * stride + kw * dilation - pad;
        uint4 v = make_uint4(0, 0, 0, 0);
        if (ih >= 0 && ih < H && iw >= 0 && iw < W)
            v = xs[((static_cast<long long>(n) * H + ih) * W + iw) * Ctot / kPer + (g * Cpg + c) / kPer];
        d[i] = v;
    }
}

// --- depth-and-row fold of a few-channel 3-D input: the (kd, kh) part of the volume's
// im2col moved into the channels, so that a 1 x Kw convolution with column stride s over
// the folded image gives the 3-D result:
//   xf[n][od*Ho + oh][w][(kd*Kh + kh)*C + c] = x[n][c][od*s - pad + kd*dil][oh*s - pad + kh*dil][w]
// (0 outside the volume and for the channel padding up to Cf).  x is NCDHW, or NDHWC with
// C channels per voxel.  One thread per folded voxel (neighbouring threads read
// neighbouring w of each tap and channel); each block first tabulates, per folded channel,
// its offset in x and its depth and row shifts.
template <typename T>
__global__ void fold3d_kernel(const T *__restrict__ x, T *__restrict__ xf, const T *__restrict__ wp,
                              T *__restrict__ wf, int N, int C, int D, int H, int W, int Do, int Ho, int Cout, int Kd,
                              int Kh, int Kw, int cpg, int stride, int pad, int dilation, int Cf, bool nchw) {
    constexpr int kPer = 16 / sizeof(T);
    extern __shared__ int4 tab[];  // per folded channel k < Kd*Kh*C: {offset in x, kd*dil, kh*dil, 0}
    const int kc = Kd * Kh * C;
    // the folded weights (a few thousand elements) ride along on the first threads:
    // wf[oc][kw][(kd*Kh + kh)*C + c] = wp[oc][(kd*Kh + kh)*Kw + kw][c], zero past Kd*Kh*C
    const long long wtotal = static_cast<long long>(Cout) * Kw * Cf;
    for (long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; i < wtotal;
         i += static_cast<long long>(gridDim.x) * blockDim.x) {
        const int k = static_cast<int>(i % Cf);
        const long long r = i / Cf;
        const int kw = static_cast<int>(r % Kw);
        const int oc = static_cast<int>(r / Kw);
        T e = T(0.f);
        if (k < kc) {
            const int t = k / C, c = k - (k / C) * C;
            e = wp[(static_cast<long long>(oc) * Kd * Kh * Kw + static_cast<long long>(t) * Kw + kw) * cpg + c];
        }
        wf[i] = e;
    }
    const long long HW = static_cast<long long>(H) * W;
    for (int k = threadIdx.x; k < kc; k += blockDim.x) {
        const int t = k / C, c = k - (k / C) * C;
        const int kd = t / Kh, kh = t - (t / Kh) * Kh;
        const long long off = nchw ? (static_cast<long long>(c) * D + kd * dilation) * HW + static_cast<long long>(kh) * dilation * W
                                   : (static_cast<long long>(kd) * dilation * HW + static_cast<long long>(kh) * dilation * W) * C + c;
        tab[k] = make_int4(static_cast<int>(off), kd * dilation, kh * dilation, 0);
    }
    __syncthreads();
    if (!nchw && (C * static_cast<int>(sizeof(T))) % 16 == 0) {
        // channels-last, whole 16-byte pieces per voxel: one thread per (voxel, tap slot)
        // copies the slot's C channels as 16-byte vectors (slots past Kd*Kh are the zero
        // channel padding; Cf is a multiple of C here)
        // 32-bit indices: the host keeps voxels x slots below 2^31
        const unsigned slots = static_cast<unsigned>(Cf / C), q = C * static_cast<unsigned>(sizeof(T)) / 16;
        const unsigned total = static_cast<unsigned>(N * Do * Ho * W) * slots;
        for (unsigned i = blockIdx.x * blockDim.x + threadIdx.x; i < total; i += gridDim.x * blockDim.x) {
            const unsigned vox = i / slots;
            const int slot = static_cast<int>(i - vox * slots);
            const unsigned r = vox / static_cast<unsigned>(W);
            const int w = static_cast<int>(vox - r * static_cast<unsigned>(W));
            const unsigned r2 = r / static_cast<unsigned>(Ho);
            const int oh = static_cast<int>(r - r2 * static_cast<unsigned>(Ho));
            const int n = static_cast<int>(r2 / static_cast<unsigned>(Do));
            const int od = static_cast<int>(r2 - static_cast<unsigned>(n) * static_cast<unsigned>(Do));
            uint4 *dst = reinterpret_cast<uint4 *>(xf + static_cast<size_t>(vox) * Cf + static_cast<size_t>(slot) * C);
            const int kd = slot / Kh, kh = slot - (slot / Kh) * Kh;
            const int id = od * stride - pad + kd * dilation, ih = oh * stride - pad + kh * dilation;
            if (slot < Kd * Kh && id >= 0 && id < D && ih >= 0 && ih < H) {
                const uint4 *src = reinterpret_cast<const uint4 *>(
                    x + (((static_cast<long long>(n) * D + id) * H + ih) * W + w) * C);
                for (unsigned j = 0; j < q; ++j) dst[j] = __ldg(src + j);
            } else {
                for (unsigned j = 0; j < q; ++j) dst[j] = make_uint4(0u, 0u, 0u, 0u);
            }
        }
        return;
    }
    const long long total = static_cast<long long>(N) * Do * Ho * W;
    for (long long vox = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; vox < total;
         vox += static_cast<long long>(gridDim.x) * blockDim.x) {
        const int w = static_cast<int>(vox % W);
        const long long r = vox / W;                   // n * (Do*Ho) + od*Ho + oh
        const int oh = static_cast<int>(r % Ho);
        const long long r2 = r / Ho;
        const int od = static_cast<int>(r2 % Do);
        const int n = static_cast<int>(r2 / Do);
        const int d0 = od * stride - pad, h0 = oh * stride - pad;  // the window's first depth and row
        // x offset of (n, c = 0, d0, h0, w), possibly outside x: only in-range taps read it
        const long long base = nchw ? ((static_cast<long long>(n) * C * D + d0) * H + h0) * W + w
                                    : (((static_cast<long long>(n) * D + d0) * H + h0) * W + w) * C;
        uint4 *dst = reinterpret_cast<uint4 *>(xf + vox * Cf);
        for (int k0 = 0; k0 < Cf; k0 += kPer) {
            alignas(16) T v[kPer];
#pragma unroll
            for (int j = 0; j < kPer; ++j) {
                const int k = k0 + j;
                T e = T(0.f);
                if (k < kc) {
                    const int4 tk = tab[k];
                    if (static_cast<unsigned>(d0 + tk.y) < static_cast<unsigned>(D) &&
                        static_cast<unsigned>(h0 + tk.z) < static_cast<unsigned>(H))
                        e = x[base + tk.x];
                }
                v[j] = e;
            }
            dst[k0 / kPer] = *reinterpret_cast<const uint4 *>(v);
        }
    }
}

// --- the same fold for a fixed channel count kC and kT = Kd*Kh folded taps (3x3 depth
// and row taps of an RGB-like input): every index of the folded row is a compile-time
// constant, the taps' shifts and offsets are computed once per thread, and each thread
// issues all kT*kC loads of its voxel before its 16-byte stores.
template <typename T, int kC, int kT>
__global__ void __launch_bounds__(kThreads) fold3d_fixed_kernel(
    const T *__restrict__ x, T *__restrict__ xf, const T *__restrict__ wp, T *__restrict__ wf, int N, int D, int H,
    int W, int Do, int Ho, int Cout, int Kh, int Kw, int cpg, int stride, int pad, int dilation, bool nchw) {
    constexpr int kPer = 16 / sizeof(T);
    constexpr int kc = kT * kC;
    constexpr int kAlign = 64 / sizeof(T);
    constexpr int kCf = (kc + kAlign - 1) / kAlign * kAlign;
    const long long wtotal = static_cast<long long>(Cout) * Kw * kCf;
    for (long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; i < wtotal;
         i += static_cast<long long>(gridDim.x) * blockDim.x) {
        const int k = static_cast<int>(i % kCf);
        const long long r = i / kCf;
        const int kw = static_cast<int>(r % Kw);
        const int oc = static_cast<int>(r / Kw);
        T e = T(0.f);
        if (k < kc)
            e = wp[(static_cast<long long>(oc) * kT * Kw + static_cast<long long>(k / kC) * Kw + kw) * cpg + k % kC];
        wf[i] = e;
    }
    const int HW = H * W;          // one image's C*D*H*W < 2^31 (host)
    const int cstep = nchw ? D * HW : 1;
    int dd[kT], hh[kT], off[kT];
#pragma unroll
    for (int t = 0; t < kT; ++t) {
        const int kd = t / Kh, kh = t - (t / Kh) * Kh;
        dd[t] = kd * dilation;
        hh[t] = kh * dilation;
        off[t] = (kd * dilation * HW + kh * dilation * W) * (nchw ? 1 : kC);
    }
    const unsigned total = static_cast<unsigned>(N * Do * Ho * W);  // < 2^31 (host)
    for (unsigned vox = blockIdx.x * blockDim.x + threadIdx.x; vox < total; vox += gridDim.x * blockDim.x) {
        const unsigned r = vox / static_cast<unsigned>(W);
        const int w = static_cast<int>(vox - r * static_cast<unsigned>(W));
        const unsigned r2 = r / static_cast<unsigned>(Ho);
        const int oh = static_cast<int>(r - r2 * static_cast<unsigned>(Ho));
        const int n = static_cast<int>(r2 / static_cast<unsigned>(Do));
        const int od = static_cast<int>(r2 - static_cast<unsigned>(n) * static_cast<unsigned>(Do));
        const int d0 = od * stride - pad, h0 = oh * stride - pad;
        const long long base = nchw ? ((static_cast<long long>(n) * kC * D + d0) * H + h0) * W + w
                                    : (((static_cast<long long>(n) * D + d0) * H + h0) * W + w) * kC;
        alignas(16) T v[kCf];
#pragma unroll
        for (int t = 0; t < kT; ++t) {
            const bool in = static_cast<unsigned>(d0 + dd[t]) < static_cast<unsigned>(D) &&
                            static_cast<unsigned>(h0 + hh[t]) < static_cast<unsigned>(H);
#pragma unroll
            for (int c = 0; c < kC; ++c) v[t * kC + c] = in ? x[base + off[t] + c * cstep] : T(0.f);
        }
#pragma unroll
        for (int k = kc; k < kCf; ++k) v[k] = T(0.f);
        uint4 *dst = reinterpret_cast<uint4 *>(xf + static_cast<size_t>(vox) * kCf);
#pragma unroll
        for (int q = 0; q < kCf / kPer; ++q) dst[q] = reinterpret_cast<const uint4 *>(v)[q];
    }
}

template <typename T>
cudaError_t launch_fold3d_fixed(int C, const void *x, void *xf, const void *wp, void *wf, int N, int D, int H, int W,
                                int Do, int Ho, int Cout, int Kh, int Kw, int cpg, int stride, int pad, int dilation,
                                bool nchw, int grid, cudaStream_t s) {
    const T *xt = static_cast<const T *>(x);
    const T *wt = static_cast<const T *>(wp);
    T *xo = static_cast<T *>(xf);
    T *wo = static_cast<T *>(wf);
    switch (C) {
        case 1: fold3d_fixed_kernel<T, 1, 9><<<grid, kThreads, 0, s>>>(xt, xo, wt, wo, N, D, H, W, Do, Ho, Cout, Kh, Kw, cpg, stride, pad, dilation, nchw); break;
        case 2: fold3d_fixed_kernel<T, 2, 9><<<grid, kThreads, 0, s>>>(xt, xo, wt, wo, N, D, H, W, Do, Ho, Cout, Kh, Kw, cpg, stride, pad, dilation, nchw); break;
        case 3: fold3d_fixed_kernel<T, 3, 9><<<grid, kThreads, 0, s>>>(xt, xo, wt, wo, N, D, H, W, Do, Ho, Cout, Kh, Kw, cpg, stride, pad, dilation, nchw); break;
        case 4: fold3d_fixed_kernel<T, 4, 9><<<grid, kThreads, 0, s>>>(xt, xo, wt, wo, N, D, H, W, Do, Ho, Cout, Kh, Kw, cpg, stride, pad, dilation, nchw); break;
        default: return cudaErrorInvalidValue;
    }
    return cudaGetLastError();
}

// --- split reduction: y = bias + sum_s ws[s][m][oc], in the output layout.
template <bool kF32>
__global__ void splitk_reduce_kernel(const float *__restrict__ ws, const void *__restrict__ bias,
                                     void *__restrict__ y, int M, int Cout, int HoWo, int splits,
                                     int nchw) {
    const long long total = static_cast<long long>(M) * Cout;
    for (long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; i < total;
         i += static_cast<long long>(gridDim.x) * blockDim.x) {
        long long m, oc;
        if (nchw) {  // consecutive threads walk pixels of one channel: coalesced writes
            const long long plane = static_cast<long long>(HoWo);
            const long long n = i / (plane * Cout);
            const long long r = i - n * plane * Cout;
            oc = r / plane;
            m = n * plane + (r - oc * plane);
        } else {
            m = i / Cout;
            oc = i - m * Cout;
        }
        float acc = 0.f;
        if (bias)
            acc = kF32 ? static_cast<const float *>(bias)[oc]
                       : __bfloat162float(static_cast<const __nv_bfloat16 *>(bias)[oc]);
        for (int s = 0; s < splits; ++s) acc += ws[(static_cast<long long>(s) * M + m) * Cout + oc];
        if (kF32)
            static_cast<float *>(y)[i] = acc;
        else
            static_cast<__nv_bfloat16 *>(y)[i] = __float2bfloat16_rn(acc);
    }
}


// --- weight gradient: dW[oc][c][kh][kw] = sum_s ws[s][oc][tap][c] (the splits of the
// tensor-core kernel's reduction over pixels), c < Cin_g, written OIHW in the weight type.
template <bool kF32>
__global__ void wgrad_reduce_kernel(const float *__restrict__ ws, void *__restrict__ dw, int Cout, int Cin_g,
                                    int taps, int Cpg, int splits) {
    const long long total = static_cast<long long>(Cout) * Cin_g * taps;
    const long long slice = static_cast<long long>(Cout) * taps * Cpg;
    for (long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; i < total;
         i += static_cast<long long>(gridDim.x) * blockDim.x) {
        const int tap = static_cast<int>(i % taps);
        const long long r = i / taps;
        const int c = static_cast<int>(r % Cin_g);
        const long long oc = r / Cin_g;
        const float *src = ws + (oc * taps + tap) * Cpg + c;
        float acc = 0.f;
        for (int s = 0; s < splits; ++s) acc += src[s * slice];
        if (kF32)
            static_cast<float *>(dw)[i] = acc;
        else
            static_cast<__nv_bfloat16 *>(dw)[i] = __float2bfloat16_rn(acc);
    }
}

// --- bias gradient, first pass: partial[b][c] = sum over a block of rows of dy.
// Channels-last dy is [rows][C]; each block sums `rows_per_block` rows, one thread per
// channel (consecutive threads read consecutive channels: coalesced).
template <bool kF32>
__global__ void bias_grad_rows_kernel(const void *__restrict__ dy, float *__restrict__ partial, long long rows,
                                      int C, int rows_per_block) {
    const long long r0 = static_cast<long long>(blockIdx.x) * rows_per_block;
    const long long r1 = r0 + rows_per_block < rows ? r0 + rows_per_block : rows;
    for (int c = threadIdx.x; c < C; c += blockDim.x) {
        float acc = 0.f;
        for (long long r = r0; r < r1; ++r) {
            const long long at = r * C + c;
            acc += kF32 ? static_cast<const float *>(dy)[at]
                        : __bfloat162float(static_cast<const __nv_bfloat16 *>(dy)[at]);
        }
        partial[static_cast<long long>(blockIdx.x) * C + c] = acc;
    }
}

// NCHW dy is [N][C][plane]: one warp sums one (n, c) plane; partial[n][c].
template <bool kF32>
__global__ void bias_grad_planes_kernel(const void *__restrict__ dy, float *__restrict__ partial, int N, int C,
                                        long long plane) {
    const int lane = threadIdx.x & 31;
    const long long warps = static_cast<long long>(gridDim.x) * (blockDim.x / 32);
    for (long long wi = (static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x) / 32;
         wi < static_cast<long long>(N) * C; wi += warps) {
        float acc = 0.f;
        for (long long k = lane; k < plane; k += 32) {
            const long long at = wi * plane + k;
            acc += kF32 ? static_cast<const float *>(dy)[at]
                        : __bfloat162float(static_cast<const __nv_bfloat16 *>(dy)[at]);
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
        if (lane == 0) partial[wi] = acc;
    }
}

// Second pass: db[c] = sum_b partial[b][c], in the bias type.
template <bool kF32>
__global__ void bias_grad_final_kernel(const float *__restrict__ partial, void *__restrict__ db, int blocks, int C) {
    for (int c = blockIdx.x * blockDim.x + threadIdx.x; c < C; c += gridDim.x * blockDim.x) {
        float acc = 0.f;
        for (int b = 0; b < blocks; ++b) acc += partial[static_cast<long long>(b) * C + c];
        if (kF32)
            static_cast<float *>(db)[c] = acc;
        else
            static_cast<__nv_bfloat16 *>(db)[c] = __float2bfloat16_rn(acc);
    }
}

// --- zero insertion for the input gradient of a strided convolution: dyz (Hz x Wz) has
// dy[n][c][oh][ow] at (oh*s, ow*s) and zeros elsewhere, in dy's layout.
template <int kElt>
__global__ void zero_insert_kernel(const void *__restrict__ dy, void *__restrict__ dyz, int N, int C, int Ho, int Wo,
                                   int Hz, int Wz, int s, int nchw) {
    using T = typename Word<kElt>::T;
    const T *src = static_cast<const T *>(dy);
    T *dst = static_cast<T *>(dyz);
    const long long total = static_cast<long long>(N) * C * Hz * Wz;
    for (long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; i < total;
         i += static_cast<long long>(gridDim.x) * blockDim.x) {
        long long n, c, j, k;
        if (nchw) {
            k = i % Wz;
            long long r = i / Wz;
            j = r % Hz;
            r /= Hz;
            c = r % C;
            n = r / C;
        } else {
            c = i % C;
            long long r = i / C;
            k = r % Wz;
            r /= Wz;
            j = r % Hz;
            n = r / Hz;
        }
        T v = T(0);
        if (j % s == 0 && k % s == 0 && j / s < Ho && k / s < Wo) {
            const long long oh = j / s, ow = k / s;
            v = nchw ? src[((n * C + c) * Ho + oh) * Wo + ow] : src[((n * Ho + oh) * Wo + ow) * C + c];
        }
        dst[i] = v;
    }
}

// --- weights of the input gradient: the kernel of the transposed convolution, packed
// like pack_weight_kernel's output for a convolution with O = C_in output channels and
// R = C_out/groups reduction channels per group: entry (o, kh, kw, c) holds
// w[g*R + cl][o % Cin_g][Kh-1-kh][Kw-1-kw] with g = o / Cin_g (spatially flipped,
// input and output channels exchanged within each group), zero for padding channels
// and, with groups merged gm at a time, outside the diagonal block.
template <int kElt>
__global__ void pack_weight_t_kernel(const void *__restrict__ w, void *__restrict__ wp, int O, int R, int Cin_g,
                                     int gm, int Kh, int Kw, int Cpg) {
    using T = typename Word<kElt>::T;
    const T *s = static_cast<const T *>(w);
    T *d = static_cast<T *>(wp);
    const long long total = static_cast<long long>(O) * Kh * Kw * Cpg;
    for (long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; i < total;
         i += static_cast<long long>(gridDim.x) * blockDim.x) {
        const int c = static_cast<int>(i % Cpg);
        long long r = i / Cpg;
        const int kw = static_cast<int>(r % Kw);
        r /= Kw;
        const int kh = static_cast<int>(r % Kh);
        const long long o = r / Kh;
        const long long g = o / Cin_g;
        const int j = static_cast<int>(g % gm);
        const int cl = c - j * R;
        T v = T(0);
        if (cl >= 0 && cl < R)
            v = s[(((g * R + cl) * Cin_g + (o - g * Cin_g)) * Kh + (Kh - 1 - kh)) * Kw + (Kw - 1 - kw)];
        d[i] = v;
    }
}

// --- weight gradient for few channels per group (depthwise and the like), on the CUDA
// cores: one thread per (split, oc, tap, c), c fastest, summing dy * x over the split's
// rows of output pixels (lpnh §5.1's formula); x and dy channels-last.  Partial sums go to
// ws[split][oc][tap][c] (Cpg = Cin_g), reduced by wgrad_reduce_kernel.
template <bool kF32>
__global__ void wgrad_direct_kernel(const void *__restrict__ x, const void *__restrict__ dy, float *__restrict__ ws,
                                    int N, int C_in, int H, int W, int C_out, int Ho, int Wo, int Kh, int Kw,
                                    int stride, int pad, int dilation, int groups, int splits) {
    const int cin_g = C_in / groups, cout_g = C_out / groups, taps = Kh * Kw;
    const long long per_split = static_cast<long long>(C_out) * taps * cin_g;
    const long long total = per_split * splits;
    const long long rows = static_cast<long long>(N) * Ho;
    for (long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; i < total;
         i += static_cast<long long>(gridDim.x) * blockDim.x) {
        const int split = static_cast<int>(i / per_split);
        long long r = i - split * per_split;
        const int c = static_cast<int>(r % cin_g);
        r /= cin_g;
        const int tap = static_cast<int>(r % taps);
        const int oc = static_cast<int>(r / taps);
        const int kh = tap / Kw, kw = tap - (tap / Kw) * Kw;
        const int ic = (oc / cout_g) * cin_g + c;
        const long long r0 = rows * split / splits, r1 = rows * (split + 1) / splits;
        float acc = 0.f;
        for (long long row = r0; row < r1; ++row) {
            const int n = static_cast<int>(row / Ho), oh = static_cast<int>(row - static_cast<long long>(n) * Ho);
            const int ih = oh * stride + kh * dilation - pad;
            if (ih < 0 || ih >= H) continue;
            for (int ow = 0; ow < Wo; ++ow) {
                const int iw = ow * stride + kw * dilation - pad;
                if (iw < 0 || iw >= W) continue;
                const long long dyi = (row * Wo + ow) * C_out + oc;
                const long long xi = ((static_cast<long long>(n) * H + ih) * W + iw) * C_in + ic;
                if (kF32)
                    acc = fmaf(static_cast<const float *>(dy)[dyi], static_cast<const float *>(x)[xi], acc);
                else
                    acc = fmaf(__bfloat162float(static_cast<const __nv_bfloat16 *>(dy)[dyi]),
                               __bfloat162float(static_cast<const __nv_bfloat16 *>(x)[xi]), acc);
            }
        }
        ws[((static_cast<long long>(split) * C_out + oc) * taps + tap) * cin_g + c] = acc;
    }
}
}  // namespace

cudaError_t launch_nchw_to_nhwc(const void *src, void *dst, int N, int C, int H, int W,
                                int groups, int Cpg, int elt, cudaStream_t s) {
    const int HW = H * W;
    const int Ctot = groups * Cpg;
    const long long pixels = static_cast<long long>(N) * HW;
    if (elt == 2 && Cpg == C / groups && C % 8 == 0 && HW % 8 == 0 && C * elt > 64) {
        launch_transpose_b16(src, dst, N, C, HW, s);  // no channel padding: a plain transpose
    } else if (elt == 4 && Cpg == C / groups && C % 4 == 0 && HW % 4 == 0 && C * elt > 64) {
        launch_transpose_b32(src, dst, N, C, HW, s);
    } else if (Ctot * elt <= 64 && (Ctot * elt) % 16 == 0) {
        if (elt == 2)
            nchw_to_nhwc_small<2><<<grid_for(pixels), kThreads, 0, s>>>(src, dst, N, C, HW, groups, Cpg);
        else
            nchw_to_nhwc_small<4><<<grid_for(pixels), kThreads, 0, s>>>(src, dst, N, C, HW, groups, Cpg);
    } else {
        const long long tiles = static_cast<long long>(N) * ((Ctot + 31) / 32) * ((HW + 31) / 32);
        const int grid = static_cast<int>(tiles < 148LL * 32 ? tiles : 148LL * 32);
        if (elt == 2)
            nchw_to_nhwc_tiled<2><<<grid, dim3(32, 8), 0, s>>>(src, dst, N, C, HW, groups, Cpg);
        else
            nchw_to_nhwc_tiled<4><<<grid, dim3(32, 8), 0, s>>>(src, dst, N, C, HW, groups, Cpg);
    }
    return cudaGetLastError();
}

cudaError_t launch_nhwc_pad(const void *src, void *dst, int N, int C, int H, int W, int groups,
                            int Cpg, int elt, cudaStream_t s) {
    const long long pixels = static_cast<long long>(N) * H * W;
    const long long total = pixels * groups * Cpg;
    if (elt == 2)
        nhwc_pad_kernel<2><<<grid_for(total), kThreads, 0, s>>>(src, dst, pixels, C, groups, Cpg);
    else
        nhwc_pad_kernel<4><<<grid_for(total), kThreads, 0, s>>>(src, dst, pixels, C, groups, Cpg);
    return cudaGetLastError();
}

cudaError_t launch_nhwc_to_nchw(const void *src, void *dst, int N, int C, int H, int W, int elt,
                                cudaStream_t s) {
    const int HW = H * W;
    if (elt == 2 && C % 8 == 0 && HW % 8 == 0) {
        launch_transpose_b16(src, dst, N, HW, C, s);
        return cudaGetLastError();
    }
    if (elt == 4 && C % 4 == 0 && HW % 4 == 0) {
        launch_transpose_b32(src, dst, N, HW, C, s);
        return cudaGetLastError();
    }
    const long long tiles = static_cast<long long>(N) * ((C + 31) / 32) * ((HW + 31) / 32);
    const int grid = static_cast<int>(tiles < 148LL * 32 ? tiles : 148LL * 32);
    if (elt == 2)
        nhwc_to_nchw_tiled<2><<<grid, dim3(32, 8), 0, s>>>(src, dst, N, C, HW);
    else
        nhwc_to_nchw_tiled<4><<<grid, dim3(32, 8), 0, s>>>(src, dst, N, C, HW);
    return cudaGetLastError();
}

cudaError_t launch_pack_weight(const void *w, void *wp, int Cout, int Cin_g, int Cout_g, int gm, int Kh,
                               int Kw, int Cpg, int elt, cudaStream_t s) {
    const long long total = static_cast<long long>(Cout) * Kh * Kw * Cpg;
    if (elt == 2)
        pack_weight_kernel<2><<<grid_for(total), kThreads, 0, s>>>(w, wp, Cout, Cin_g, Cout_g, gm, Kh, Kw, Cpg);
    else
        pack_weight_kernel<4><<<grid_for(total), kThreads, 0, s>>>(w, wp, Cout, Cin_g, Cout_g, gm, Kh, Kw, Cpg);
    return cudaGetLastError();
}

cudaError_t launch_pack_gather_image(const void *w, void *img, int Cout, int C, int Kh, int Kw,
                                     int BN, int Kpad, bool rowvec, int elt, cudaStream_t s) {
    const long long work = static_cast<long long>(BN) * Kpad * elt / 16;
    if (elt == 2)
        pack_gather_image_kernel<2><<<grid_for(work), kThreads, 0, s>>>(
            w, static_cast<uint8_t *>(img), Cout, C, Kh, Kw, BN, Kpad, rowvec ? 1 : 0);
    else
        pack_gather_image_kernel<4><<<grid_for(work), kThreads, 0, s>>>(
            w, static_cast<uint8_t *>(img), Cout, C, Kh, Kw, BN, Kpad, rowvec ? 1 : 0);
    return cudaGetLastError();
}

cudaError_t launch_im2col(const void *x_nhwc, void *xcol, int N, int H, int W, int groups,
                          int Cpg, int Ho, int Wo, int Kh, int Kw, int stride, int pad,
                          int dilation, int elt, cudaStream_t s) {
    const long long chunks = static_cast<long long>(N) * Ho * Wo * groups * Kh * Kw * Cpg * elt / 16;
    if (elt == 2)
        im2col_kernel<2><<<grid_for(chunks), kThreads, 0, s>>>(x_nhwc, xcol, N, H, W, groups, Cpg,
                                                              Ho, Wo, Kh, Kw, stride, pad, dilation);
    else
        im2col_kernel<4><<<grid_for(chunks), kThreads, 0, s>>>(x_nhwc, xcol, N, H, W, groups, Cpg,
                                                              Ho, Wo, Kh, Kw, stride, pad, dilation);
    return cudaGetLastError();
}

cudaError_t launch_fold3d(const void *x, void *xf, const void *wp, void *wf, int N, int C, int D, int H, int W,
                          int Do, int Ho, int Cout, int Kd, int Kh, int Kw, int cpg, int stride, int pad, int dilation,
                          int Cf, int elt, bool nchw, cudaStream_t s) {
    const int kc = Kd * Kh * C;
    // the per-channel offsets are 32-bit: one image's C*D*H*W elements, and the largest tap
    // shift, stay below 2^31
    if (Cf % (16 / elt) != 0 || Cf < kc || kc > 4096 || cpg < C ||
        static_cast<long long>(C) * (D + Kd * dilation) * (H + Kh * dilation) * W >= (1LL << 31))
        return cudaErrorInvalidValue;
    const long long voxels = static_cast<long long>(N) * Do * Ho * W;
    const bool vec = !nchw && (C * elt) % 16 == 0;  // the kernel's 16-byte copy path
    if (vec && (Cf % C != 0 || voxels * (Cf / C) >= (1LL << 31))) return cudaErrorInvalidValue;
    const long long work = vec ? voxels * (Cf / C) : voxels;
    // three-by-three depth and row taps of one to four channels (an RGB-like input): the
    // kernel with every folded index fixed at compile time (same Cf formula)
    if (!vec && Kd * Kh == 9 && C >= 1 && C <= 4 && voxels < (1LL << 31))
        return elt == 2 ? launch_fold3d_fixed<__nv_bfloat16>(C, x, xf, wp, wf, N, D, H, W, Do, Ho, Cout, Kh, Kw, cpg,
                                                              stride, pad, dilation, nchw, grid_for(voxels), s)
                        : launch_fold3d_fixed<float>(C, x, xf, wp, wf, N, D, H, W, Do, Ho, Cout, Kh, Kw, cpg, stride,
                                                      pad, dilation, nchw, grid_for(voxels), s);
    const size_t tab = static_cast<size_t>(kc) * sizeof(int4);
    if (elt == 2)
        fold3d_kernel<__nv_bfloat16><<<grid_for(work), kThreads, tab, s>>>(
            static_cast<const __nv_bfloat16 *>(x), static_cast<__nv_bfloat16 *>(xf),
            static_cast<const __nv_bfloat16 *>(wp), static_cast<__nv_bfloat16 *>(wf), N, C, D, H, W, Do, Ho, Cout, Kd,
            Kh, Kw, cpg, stride, pad, dilation, Cf, nchw);
    else
        fold3d_kernel<float><<<grid_for(work), kThreads, tab, s>>>(
            static_cast<const float *>(x), static_cast<float *>(xf), static_cast<const float *>(wp),
            static_cast<float *>(wf), N, C, D, H, W, Do, Ho, Cout, Kd, Kh, Kw, cpg, stride, pad, dilation, Cf, nchw);
    return cudaGetLastError();
}

cudaError_t launch_splitk_reduce(const float *ws, const void *bias, void *y, int M, int Cout,
                                 int HoWo, int splits, int out_mode, bool f32, cudaStream_t s) {
    const long long total = static_cast<long long>(M) * Cout;
    const int nchw = out_mode == kOutNCHW ? 1 : 0;
    if (f32)
        splitk_reduce_kernel<true><<<grid_for(total), kThreads, 0, s>>>(ws, bias, y, M, Cout, HoWo,
                                                                        splits, nchw);
    else
        splitk_reduce_kernel<false><<<grid_for(total), kThreads, 0, s>>>(ws, bias, y, M, Cout, HoWo,
                                                                         splits, nchw);
    return cudaGetLastError();
}


cudaError_t launch_wgrad_reduce(const float *ws, void *dw, int Cout, int Cin_g, int taps, int Cpg, int splits,
                                bool f32, cudaStream_t s) {
    const long long total = static_cast<long long>(Cout) * Cin_g * taps;
    if (f32)
        wgrad_reduce_kernel<true><<<grid_for(total), kThreads, 0, s>>>(ws, dw, Cout, Cin_g, taps, Cpg, splits);
    else
        wgrad_reduce_kernel<false><<<grid_for(total), kThreads, 0, s>>>(ws, dw, Cout, Cin_g, taps, Cpg, splits);
    return cudaGetLastError();
}

int bias_grad_partials(long long rows, int C, int N, bool nchw) {
    return nchw ? N : static_cast<int>((rows + kBiasRows - 1) / kBiasRows);
}

cudaError_t launch_bias_grad(const void *dy, float *partial, void *db, int N, int C, long long plane, bool nchw,
                             bool f32, cudaStream_t s) {
    const long long rows = static_cast<long long>(N) * plane;
    const int blocks = bias_grad_partials(rows, C, N, nchw);
    if (nchw) {
        const int grid = grid_for(static_cast<long long>(N) * C * 32);
        if (f32)
            bias_grad_planes_kernel<true><<<grid, kThreads, 0, s>>>(dy, partial, N, C, plane);
        else
            bias_grad_planes_kernel<false><<<grid, kThreads, 0, s>>>(dy, partial, N, C, plane);
    } else {
        if (f32)
            bias_grad_rows_kernel<true><<<blocks, kThreads, 0, s>>>(dy, partial, rows, C, kBiasRows);
        else
            bias_grad_rows_kernel<false><<<blocks, kThreads, 0, s>>>(dy, partial, rows, C, kBiasRows);
    }
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    if (f32)
        bias_grad_final_kernel<true><<<grid_for(C), kThreads, 0, s>>>(partial, db, blocks, C);
    else
        bias_grad_final_kernel<false><<<grid_for(C), kThreads, 0, s>>>(partial, db, blocks, C);
    return cudaGetLastError();
}

cudaError_t launch_zero_insert(const void *dy, void *dyz, int N, int C, int Ho, int Wo, int Hz, int Wz, int stride,
                               bool nchw, int elt, cudaStream_t s) {
    const long long total = static_cast<long long>(N) * C * Hz * Wz;
    if (elt == 2)
        zero_insert_kernel<2><<<grid_for(total), kThreads, 0, s>>>(dy, dyz, N, C, Ho, Wo, Hz, Wz, stride, nchw ? 1 : 0);
    else
        zero_insert_kernel<4><<<grid_for(total), kThreads, 0, s>>>(dy, dyz, N, C, Ho, Wo, Hz, Wz, stride, nchw ? 1 : 0);
    return cudaGetLastError();
}

cudaError_t launch_pack_weight_t(const void *w, void *wp, int O, int R, int Cin_g, int gm, int Kh, int Kw, int Cpg,
                                 int elt, cudaStream_t s) {
    const long long total = static_cast<long long>(O) * Kh * Kw * Cpg;
    if (elt == 2)
        pack_weight_t_kernel<2><<<grid_for(total), kThreads, 0, s>>>(w, wp, O, R, Cin_g, gm, Kh, Kw, Cpg);
    else
        pack_weight_t_kernel<4><<<grid_for(total), kThreads, 0, s>>>(w, wp, O, R, Cin_g, gm, Kh, Kw, Cpg);
    return cudaGetLastError();
}


cudaError_t launch_wgrad_direct(const void *x, const void *dy, float *ws, int N, int C_in, int H, int W, int C_out,
                                int Ho, int Wo, int Kh, int Kw, int stride, int pad, int dilation, int groups,
                                int splits, bool f32, cudaStream_t s) {
    const long long total = static_cast<long long>(C_out) * Kh * Kw * (C_in / groups) * splits;
    const int grid = grid_for(total, 128);
    if (f32)
        wgrad_direct_kernel<true><<<grid, 128, 0, s>>>(x, dy, ws, N, C_in, H, W, C_out, Ho, Wo, Kh, Kw, stride, pad,
                                                      dilation, groups, splits);
    else
        wgrad_direct_kernel<false><<<grid, 128, 0, s>>>(x, dy, ws, N, C_in, H, W, C_out, Ho, Wo, Kh, Kw, stride,
                                                       pad, dilation, groups, splits);
    return cudaGetLastError();
}

}  // namespace conv2d_b200
