// winograd.cu -- the minimal-filtering (Winograd) form of the 3x3, stride-1, unit-
// dilation convolution: F(2x2, 3x3) and F(4x4, 3x3).
//
// The im2col/GEMM tutorial (zskr.cn/news/1820658) §5.1 describes it: an m x m block of
// outputs of an r x r filter needs m^2 r^2 multiplications directly but only (m+r-1)^2
// after linear transforms of the input tile and the filter (36 -> 16 for F(2x2,3x3),
// 2.25x), and it applies only to small filters with stride 1 and dilation 1, with larger
// rounding error from the transforms; the "手撕 Conv2D" page (lpnh.cn/news/2493075) §7
// names F(2,3) and F(4,3).  The transforms are the published ones of Lavin & Gray,
// "Fast Algorithms for Convolutional Neural Networks" (2016):
//     Y = A^T [ (G g G^T) o (B^T d B) ] A
// with d an alpha x alpha input tile (alpha = m + 2), g the 3 x 3 filter and o the
// elementwise product.  Summed over input channels, the elementwise product becomes,
// for each of the alpha^2 tile positions xi, one matrix product
//     M[xi][tile][oc] = sum_c V[xi][tile][c] * U[xi][oc][c],
// which runs here on the same tensor-core kernel as the forward pass (a grouped 1x1
// convolution with alpha^2 groups over the transformed tiles).  The three steps:
//   1. input transform (this file): V = B^T d B per tile and channel vector, written
//      channels-last as [tile][xi][Cpg] (Cpg: channels padded to 16 bytes), in the
//      transform type: bf16 for F(2x2,3x3) on bf16 data (one more rounding), fp32
//      otherwise -- F(4x4,3x3)'s larger transform entries make bf16 V and U miss the bf16
//      tolerance (measured), so its transforms and product stay in fp32 (3xTF32);
//   2. the product on the tensor cores, fp32 results [tile][xi][oc];
//   3. output transform (this file): Y = A^T M A + bias per tile and output channel
//      vector, one rounding to the output dtype, written NHWC or NCHW.
// U = G g G^T is computed once when the weights are packed.  All three kernels are
// memory-bound CUDA-core loops; the transformed tensors (V, M) are alpha^2/m^2 times
// the size of x and y, which is the cost of not fusing the transforms into the product.
#include <cuda_bf16.h>

#include "common.cuh"

namespace conv2d_b200 {
namespace {

constexpr int kWgThreads256 = 256;

inline int wino_grid(long long work) {
    long long g = (work + kWgThreads256 - 1) / kWgThreads256;
    if (g < 1) g = 1;
    if (g > 148LL * 32) g = 148LL * 32;
    return static_cast<int>(g);
}

// B^T rows (alpha x alpha), G (alpha x 3) and A^T (m x alpha) of F(m x m, 3 x 3).
template <int kM>
struct WinoMats;

template <>
struct WinoMats<2> {
    static constexpr int kA = 4;
    __device__ static float bt(int i, int j) {
        constexpr float t[4][4] = {{1, 0, -1, 0}, {0, 1, 1, 0}, {0, -1, 1, 0}, {0, 1, 0, -1}};
        return t[i][j];
    }
    __device__ static float g(int i, int j) {
        constexpr float t[4][3] = {{1, 0, 0}, {0.5f, 0.5f, 0.5f}, {0.5f, -0.5f, 0.5f}, {0, 0, 1}};
        return t[i][j];
    }
    __device__ static float at(int i, int j) {
        constexpr float t[2][4] = {{1, 1, 1, 0}, {0, 1, -1, -1}};
        return t[i][j];
    }
};

template <>
struct WinoMats<4> {
    static constexpr int kA = 6;
    __device__ static float bt(int i, int j) {
        constexpr float t[6][6] = {{4, 0, -5, 0, 1, 0},  {0, -4, -4, 1, 1, 0}, {0, 4, -4, -1, 1, 0},
                                   {0, -2, -1, 2, 1, 0}, {0, 2, -1, -2, 1, 0}, {0, 4, 0, -5, 0, 1}};
        return t[i][j];
    }
    __device__ static float g(int i, int j) {
        constexpr float t[6][3] = {{1.f / 4, 0, 0},
                                   {-1.f / 6, -1.f / 6, -1.f / 6},
                                   {-1.f / 6, 1.f / 6, -1.f / 6},
                                   {1.f / 24, 1.f / 12, 1.f / 6},
                                   {1.f / 24, -1.f / 12, 1.f / 6},
                                   {0, 0, 1}};
        return t[i][j];
    }
    __device__ static float at(int i, int j) {
        constexpr float t[4][6] = {{1, 1, 1, 1, 1, 0}, {0, 1, -1, 2, -2, 0}, {0, 1, 1, 4, 4, 0}, {0, 1, -1, 8, -8, 1}};
        return t[i][j];
    }
};

template <bool kF32>
__device__ __forceinline__ float ld1(const void *p, long long i) {
    if constexpr (kF32)
        return static_cast<const float *>(p)[i];
    else
        return __bfloat162float(static_cast<const __nv_bfloat16 *>(p)[i]);
}

template <bool kF32>
__device__ __forceinline__ void st1(void *p, long long i, float v) {
    if constexpr (kF32)
        static_cast<float *>(p)[i] = v;
    else
        static_cast<__nv_bfloat16 *>(p)[i] = __float2bfloat16_rn(v);
}

// kV consecutive elements at element index i (i a multiple of kV, the base aligned):
// one 4-, 8- or 16-byte access instead of kV scalar ones.
template <bool kF32, int kV>
__device__ __forceinline__ void ldv(const void *p, long long i, float *f) {
    if constexpr (kF32) {
        if constexpr (kV == 4) {
            const float4 v = *reinterpret_cast<const float4 *>(static_cast<const float *>(p) + i);
            f[0] = v.x; f[1] = v.y; f[2] = v.z; f[3] = v.w;
        } else {
            const float2 v = *reinterpret_cast<const float2 *>(static_cast<const float *>(p) + i);
            f[0] = v.x; f[1] = v.y;
        }
    } else {
        const unsigned short *q = static_cast<const unsigned short *>(p) + i;
        if constexpr (kV == 4) {
            const uint2 v = *reinterpret_cast<const uint2 *>(q);
            f[0] = __uint_as_float(v.x << 16); f[1] = __uint_as_float(v.x & 0xFFFF0000u);
            f[2] = __uint_as_float(v.y << 16); f[3] = __uint_as_float(v.y & 0xFFFF0000u);
        } else {
            const uint32_t v = *reinterpret_cast<const uint32_t *>(q);
            f[0] = __uint_as_float(v << 16); f[1] = __uint_as_float(v & 0xFFFF0000u);
        }
    }
}

template <bool kF32, int kV>
__device__ __forceinline__ void stv(void *p, long long i, const float *f) {
    if constexpr (kF32) {
        if constexpr (kV == 4)
            *reinterpret_cast<float4 *>(static_cast<float *>(p) + i) = make_float4(f[0], f[1], f[2], f[3]);
        else
            *reinterpret_cast<float2 *>(static_cast<float *>(p) + i) = make_float2(f[0], f[1]);
    } else {
        uint32_t w[kV / 2];
#pragma unroll
        for (int k = 0; k < kV / 2; ++k) {
            __nv_bfloat162 h = __floats2bfloat162_rn(f[2 * k], f[2 * k + 1]);
            w[k] = *reinterpret_cast<uint32_t *>(&h);
        }
        unsigned short *q = static_cast<unsigned short *>(p) + i;
        if constexpr (kV == 4)
            *reinterpret_cast<uint2 *>(q) = make_uint2(w[0], w[1]);
        else
            *reinterpret_cast<uint32_t *>(q) = w[0];
    }
}

// 1. V[tile][xi][c] = (B^T d B)[xi] for each tile (n, th, tw) and channel c < Cpg (zero
// for c >= C): d[a][b] = x[n][th*m - pad + a][tw*m - pad + b][c], zero outside the image.
// One thread per (tile, group of kV consecutive channels).  All alpha^2 loads of a tile are
// issued before any arithmetic (they are independent, and so in flight together), then
// B^T is applied to the columns in place and B to the rows on the way out.
template <bool kF32, bool kVF32, int kM, int kV>
__global__ void __launch_bounds__(kWgThreads256) wino_input_kernel(const void *__restrict__ x, void *__restrict__ v,
                                                                 int N, int C, int H, int W, int Cpg, int TH, int TW,
                                                                 int pad, int nchw) {
    using Mt = WinoMats<kM>;
    constexpr int kA = Mt::kA;
    const int cgroups = Cpg / kV;
    const long long total = static_cast<long long>(N) * TH * TW * cgroups;
    const bool vec = !nchw && C % kV == 0;
    for (long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; i < total;
         i += static_cast<long long>(gridDim.x) * blockDim.x) {
        const int cg = static_cast<int>(i % cgroups);
        const long long tile = i / cgroups;
        const int tw = static_cast<int>(tile % TW);
        const long long r = tile / TW;
        const int th = static_cast<int>(r % TH);
        const int n = static_cast<int>(r / TH);
        const int c0 = cg * kV;
        const int h0 = th * kM - pad, w0 = tw * kM - pad;
        float d[kA][kA][kV];
#pragma unroll
        for (int k = 0; k < kA; ++k) {
            const int ih = h0 + k;
#pragma unroll
            for (int b = 0; b < kA; ++b) {
                const int iw = w0 + b;
                const bool in = ih >= 0 && ih < H && iw >= 0 && iw < W;
                if (vec) {  // channels-last, C a multiple of kV: one vector access
                    if (in && c0 < C) {
                        ldv<kF32, kV>(x, ((static_cast<long long>(n) * H + ih) * W + iw) * C + c0, d[k][b]);
                    } else {
#pragma unroll
                        for (int e = 0; e < kV; ++e) d[k][b][e] = 0.f;
                    }
                } else {
#pragma unroll
                    for (int e = 0; e < kV; ++e) {
                        const int c = c0 + e;
                        float val = 0.f;
                        if (in && c < C) {
                            const long long at = nchw ? ((static_cast<long long>(n) * C + c) * H + ih) * W + iw
                                                      : ((static_cast<long long>(n) * H + ih) * W + iw) * C + c;
                            val = ld1<kF32>(x, at);
                        }
                        d[k][b][e] = val;
                    }
                }
            }
        }
        // columns: d[.][b] <- B^T d[.][b]
#pragma unroll
        for (int b = 0; b < kA; ++b) {
            float t[kA][kV];
#pragma unroll
            for (int a = 0; a < kA; ++a)
#pragma unroll
                for (int e = 0; e < kV; ++e) {
                    float sum = 0.f;
#pragma unroll
                    for (int k = 0; k < kA; ++k) sum += Mt::bt(a, k) * d[k][b][e];
                    t[a][e] = sum;
                }
#pragma unroll
            for (int a = 0; a < kA; ++a)
#pragma unroll
                for (int e = 0; e < kV; ++e) d[a][b][e] = t[a][e];
        }
        // rows: V[a][b] = sum_k (B^T d)[a][k] B[k][b]
        const long long base = tile * kA * kA * Cpg + c0;
#pragma unroll
        for (int a = 0; a < kA; ++a)
#pragma unroll
            for (int b = 0; b < kA; ++b) {
                float o[kV];
#pragma unroll
                for (int e = 0; e < kV; ++e) {
                    float sum = 0.f;
#pragma unroll
                    for (int k = 0; k < kA; ++k) sum += d[a][k][e] * Mt::bt(b, k);
                    o[e] = sum;
                }
                stv<kVF32, kV>(v, base + static_cast<long long>(a * kA + b) * Cpg, o);  // Cpg % kV == 0
            }
    }
}

// U packed for the product: rows o = xi * C_out + oc (alpha^2 groups of C_out), each
// row Cpgw entries; entry c of row o holds (G g[oc][c] G^T)[xi] for c < C, zero for the
// padding channels and -- with groups merged gm at a time -- outside the diagonal block.
template <bool kF32, bool kUF32, int kM>
__global__ void __launch_bounds__(kWgThreads256) wino_weight_kernel(const void *__restrict__ w, void *__restrict__ u,
                                                                  int C_out, int C, int Cpg, int gm, int Cpgw) {
    using Mt = WinoMats<kM>;
    constexpr int kA = Mt::kA;
    const long long total = static_cast<long long>(kA) * kA * C_out * Cpgw;
    for (long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; i < total;
         i += static_cast<long long>(gridDim.x) * blockDim.x) {
        const int cw = static_cast<int>(i % Cpgw);
        const long long o = i / Cpgw;
        const int xi = static_cast<int>(o / C_out);
        const int oc = static_cast<int>(o - static_cast<long long>(xi) * C_out);
        const int j = xi % gm;
        const int c = cw - j * Cpg;
        float val = 0.f;
        if (c >= 0 && c < C) {
            const int a = xi / kA, b = xi - (xi / kA) * kA;
            const long long g0 = (static_cast<long long>(oc) * C + c) * 9;
#pragma unroll
            for (int p = 0; p < 3; ++p)
#pragma unroll
                for (int q = 0; q < 3; ++q) val += Mt::g(a, p) * ld1<kF32>(w, g0 + p * 3 + q) * Mt::g(b, q);
        }
        st1<kUF32>(u, i, val);
    }
}

// 3. y[n][th*m + i][tw*m + j][oc] = bias[oc] + (A^T M A)[i][j], M[xi] summed over the
// product's splits (fp32 partial sums [split][tile][alpha^2 * C_out]).  As in the input
// transform, all alpha^2 loads of a tile (per split) are issued before any arithmetic.
template <bool kF32, int kM, int kV>
__global__ void __launch_bounds__(kWgThreads256) wino_output_kernel(const float *__restrict__ mp,
                                                                  const void *__restrict__ bias, void *__restrict__ y,
                                                                  int N, int C_out, int Ho, int Wo, int TH, int TW,
                                                                  int splits, int nchw) {
    using Mt = WinoMats<kM>;
    constexpr int kA = Mt::kA;
    const int cgroups = (C_out + kV - 1) / kV;
    const long long tiles = static_cast<long long>(N) * TH * TW;
    const long long total = tiles * cgroups;
    const long long row = static_cast<long long>(kA) * kA * C_out;
    const bool vec = C_out % kV == 0;
    for (long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; i < total;
         i += static_cast<long long>(gridDim.x) * blockDim.x) {
        const int cg = static_cast<int>(i % cgroups);
        const long long tile = i / cgroups;
        const int tw = static_cast<int>(tile % TW);
        const long long r = tile / TW;
        const int th = static_cast<int>(r % TH);
        const int n = static_cast<int>(r / TH);
        const int c0 = cg * kV;
        // the first split straight into m, all loads in flight together; later splits
        // (rare) added one vector at a time
        float m[kA][kA][kV];
        for (int sp = 0; sp < splits; ++sp) {
            const float *src = mp + (sp * tiles + tile) * row + c0;
#pragma unroll
            for (int k = 0; k < kA; ++k)
#pragma unroll
                for (int b = 0; b < kA; ++b) {
                    const long long at = static_cast<long long>(k * kA + b) * C_out;
                    float f[kV];
                    if (vec) {
                        ldv<true, kV>(src, at, f);
                    } else {
#pragma unroll
                        for (int e = 0; e < kV; ++e) f[e] = c0 + e < C_out ? src[at + e] : 0.f;
                    }
#pragma unroll
                    for (int e = 0; e < kV; ++e) m[k][b][e] = sp == 0 ? f[e] : m[k][b][e] + f[e];
                }
        }
        // columns: m[a][b] <- (A^T M)[a][b] for a < m
#pragma unroll
        for (int b = 0; b < kA; ++b) {
            float t[kM][kV];
#pragma unroll
            for (int a = 0; a < kM; ++a)
#pragma unroll
                for (int e = 0; e < kV; ++e) {
                    float sum = 0.f;
#pragma unroll
                    for (int k = 0; k < kA; ++k) sum += Mt::at(a, k) * m[k][b][e];
                    t[a][e] = sum;
                }
#pragma unroll
            for (int a = 0; a < kM; ++a)
#pragma unroll
                for (int e = 0; e < kV; ++e) m[a][b][e] = t[a][e];
        }
        float bv[kV];
#pragma unroll
        for (int e = 0; e < kV; ++e) bv[e] = (bias && c0 + e < C_out) ? ld1<kF32>(bias, c0 + e) : 0.f;
#pragma unroll
        for (int a = 0; a < kM; ++a) {
            const int oh = th * kM + a;
            if (oh >= Ho) break;
#pragma unroll
            for (int b = 0; b < kM; ++b) {
                const int ow = tw * kM + b;
                if (ow >= Wo) break;
                float o[kV];
#pragma unroll
                for (int e = 0; e < kV; ++e) {
                    float s = bv[e];
#pragma unroll
                    for (int k = 0; k < kA; ++k) s += m[a][k][e] * Mt::at(b, k);
                    o[e] = s;
                }
                if (vec && !nchw) {
                    stv<kF32, kV>(y, ((static_cast<long long>(n) * Ho + oh) * Wo + ow) * C_out + c0, o);
                } else {
#pragma unroll
                    for (int e = 0; e < kV; ++e) {
                        const int oc = c0 + e;
                        if (oc >= C_out) break;
                        const long long at = nchw ? ((static_cast<long long>(n) * C_out + oc) * Ho + oh) * Wo + ow
                                                  : ((static_cast<long long>(n) * Ho + oh) * Wo + ow) * C_out + oc;
                        st1<kF32>(y, at, o[e]);
                    }
                }
            }
        }
    }
}

template <bool kF32, bool kVF32, int kM>
cudaError_t input_t(const void *x, void *v, int N, int C, int H, int W, int Cpg, int TH, int TW, int pad, bool nchw,
                    cudaStream_t s) {
    constexpr int kV = kM == 2 ? 4 : 2;  // channels per thread
    const long long work = static_cast<long long>(N) * TH * TW * (Cpg / kV);
    wino_input_kernel<kF32, kVF32, kM, kV><<<wino_grid(work), kWgThreads256, 0, s>>>(x, v, N, C, H, W, Cpg, TH, TW,
                                                                                   pad, nchw ? 1 : 0);
    return cudaGetLastError();
}

template <bool kF32, int kM>
cudaError_t output_t(const float *mp, const void *bias, void *y, int N, int C_out, int Ho, int Wo, int TH, int TW,
                     int splits, bool nchw, cudaStream_t s) {
    constexpr int kV = kM == 2 ? 4 : 2;
    const long long work = static_cast<long long>(N) * TH * TW * ((C_out + kV - 1) / kV);
    wino_output_kernel<kF32, kM, kV><<<wino_grid(work), kWgThreads256, 0, s>>>(mp, bias, y, N, C_out, Ho, Wo, TH, TW,
                                                                             splits, nchw ? 1 : 0);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_wino_input(const void *x, void *v, int N, int C, int H, int W, int Cpg, int TH, int TW, int pad,
                              int m, bool nchw, bool f32, bool v_f32, cudaStream_t s) {
    if (Cpg % 4 != 0) return cudaErrorInvalidValue;  // a multiple of both vector widths
    if (f32 && !v_f32) return cudaErrorInvalidValue;
    if (m == 2) return f32 ? input_t<true, true, 2>(x, v, N, C, H, W, Cpg, TH, TW, pad, nchw, s)
                           : v_f32 ? input_t<false, true, 2>(x, v, N, C, H, W, Cpg, TH, TW, pad, nchw, s)
                                   : input_t<false, false, 2>(x, v, N, C, H, W, Cpg, TH, TW, pad, nchw, s);
    if (m == 4) return f32 ? input_t<true, true, 4>(x, v, N, C, H, W, Cpg, TH, TW, pad, nchw, s)
                           : v_f32 ? input_t<false, true, 4>(x, v, N, C, H, W, Cpg, TH, TW, pad, nchw, s)
                                   : input_t<false, false, 4>(x, v, N, C, H, W, Cpg, TH, TW, pad, nchw, s);
    return cudaErrorInvalidValue;
}

template <bool kF32, bool kUF32, int kM>
cudaError_t weight_t(const void *w, void *u, int C_out, int C, int Cpg, int gm, cudaStream_t s) {
    const long long work = static_cast<long long>(kM + 2) * (kM + 2) * C_out * Cpg * gm;
    wino_weight_kernel<kF32, kUF32, kM><<<wino_grid(work), kWgThreads256, 0, s>>>(w, u, C_out, C, Cpg, gm, Cpg * gm);
    return cudaGetLastError();
}

cudaError_t launch_wino_weight(const void *w, void *u, int C_out, int C, int Cpg, int gm, int m, bool f32, bool u_f32,
                               cudaStream_t s) {
    if (f32 && !u_f32) return cudaErrorInvalidValue;
    if (m == 2) return f32 ? weight_t<true, true, 2>(w, u, C_out, C, Cpg, gm, s)
                           : u_f32 ? weight_t<false, true, 2>(w, u, C_out, C, Cpg, gm, s)
                                   : weight_t<false, false, 2>(w, u, C_out, C, Cpg, gm, s);
    if (m == 4) return f32 ? weight_t<true, true, 4>(w, u, C_out, C, Cpg, gm, s)
                           : u_f32 ? weight_t<false, true, 4>(w, u, C_out, C, Cpg, gm, s)
                                   : weight_t<false, false, 4>(w, u, C_out, C, Cpg, gm, s);
    return cudaErrorInvalidValue;
}

cudaError_t launch_wino_output(const float *mp, const void *bias, void *y, int N, int C_out, int Ho, int Wo, int TH,
                               int TW, int splits, int m, bool nchw, bool f32, cudaStream_t s) {
    if (m == 2) return f32 ? output_t<true, 2>(mp, bias, y, N, C_out, Ho, Wo, TH, TW, splits, nchw, s)
                           : output_t<false, 2>(mp, bias, y, N, C_out, Ho, Wo, TH, TW, splits, nchw, s);
    if (m == 4) return f32 ? output_t<true, 4>(mp, bias, y, N, C_out, Ho, Wo, TH, TW, splits, nchw, s)
                           : output_t<false, 4>(mp, bias, y, N, C_out, Ho, Wo, TH, TW, splits, nchw, s);
    return cudaErrorInvalidValue;
}

}  // namespace conv2d_b200
