// depthwise.cu -- depthwise convolution (groups = C_in = C_out: every channel is filtered
// by its own Kh x Kw kernel), written as a direct stencil over channels-last tiles.
//
// The tutorial page (zskr.cn/news/1820658) §4.2 names depthwise convolution as the case
// where im2col + GEMM is the wrong tool: each output reads only Kh*Kw values of its own
// channel, so the "matrix product" has a reduction of Kh*Kw and im2col only multiplies the
// memory traffic; §4.3 item 4 recommends a direct kernel that stages data in shared
// memory.  The "手撕 Conv2D" page (lpnh.cn/news/2493075) §7 gives the variant: groups =
// input channels, so output channel c sees input channel c alone.  The sum computed is the
// convolution's definition with that grouping,
//     y[n][oh][ow][c] = bias[c] + sum_{kh, kw} x[n][oh*s + kh*d - p][ow*s + kw*d - p][c] * w[c][kh][kw],
// terms outside the image dropped.  It is memory-bound (2*Kh*Kw FLOPs per 2-4 bytes of
// output), so it runs on the CUDA cores; tensor cores would only add traffic here.
//
// Persistent CTAs, one per SM, warp-specialised:
//   warp 0     : one thread issues a tiled TMA load per tile -- a box of IH x IW input
//                pixels x 128 bytes of channels, starting at (oh0*s - p, ow0*s - p); the
//                part of the box outside the image is filled with zeros by the copy engine,
//                which is the zero padding -- into a ring of shared-memory stages;
//   warps 1..15: compute.  Each thread owns R consecutive output pixels of one row and 16
//                bytes of channels; for stride 1 and unit dilation it reads each input row
//                once into a register window of R + Kw - 1 pixels and reuses it for every
//                filter column.  Weights of the tile's channels are kept per warp in shared
//                memory; accumulation is fp32 (bf16 inputs by mixed-precision FMAs straight
//                from their packed words, fp32 by paired FMAs), bias is added in fp32 and
//                the result is rounded once to the output type and stored with 16-byte
//                stores (NHWC).
// Every wait is bounded (see ptx.cuh).
#include <cuda_bf16.h>

#include "common.cuh"
#include "ptx.cuh"

namespace conv2d_b200 {
namespace {

using namespace ptx;

constexpr int kDwRowBytes = 128;  // bytes of channels per staged pixel
// 16 warps in all: four per SM sub-partition, so each thread may use 128 registers
// (a 17th warp would put five on one sub-partition and cap every thread at 96)
constexpr int kDwComputeWarps = 15;
constexpr int kDwThreads = 32 * (1 + kDwComputeWarps);
constexpr int kDwMaxStages = 6;
constexpr int kDwHeader = 1024;   // barriers, ahead of the weights and the stage ring

struct DwShared {
    uint64_t full[kDwMaxStages];
    uint64_t empty[kDwMaxStages];
    int abort;
};
static_assert(sizeof(DwShared) <= kDwHeader, "header too small");

// 16 bytes of channels as fp32 values (8 bf16 or 4 fp32).
template <bool kF32>
__device__ __forceinline__ void unpack16(const uint4 &u, float *f) {
    if constexpr (kF32) {
        f[0] = __uint_as_float(u.x);
        f[1] = __uint_as_float(u.y);
        f[2] = __uint_as_float(u.z);
        f[3] = __uint_as_float(u.w);
    } else {
        const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            f[2 * i] = __uint_as_float(w[i] << 16);
            f[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
        }
    }
}

// Paired fp32 arithmetic: a 64-bit register holds two fp32 lanes (channels 2i, 2i+1).
// fma2 is one fma.rn.f32x2 -- two fused multiply-adds per instruction, each lane rounded
// as fmaf rounds it.
__device__ __forceinline__ uint64_t pair(uint32_t lo, uint32_t hi) {
    uint64_t r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "r"(lo), "r"(hi));
    return r;
}

__device__ __forceinline__ void fma2(uint64_t &acc, uint64_t x, uint64_t w) {
    asm("fma.rn.f32x2 %0, %1, %2, %0;" : "+l"(acc) : "l"(x), "l"(w));
}

__device__ __forceinline__ void unpair(uint64_t v, float &lo, float &hi) {
    uint32_t a, b;
    asm("mov.b64 {%0, %1}, %2;" : "=r"(a), "=r"(b) : "l"(v));
    lo = __uint_as_float(a);
    hi = __uint_as_float(b);
}

// acc0 += lo(x) * lo(w), acc1 += hi(x) * hi(w) on the bf16 halves of two 32-bit words:
// sm_100's mixed-precision fma (bf16 operands, fp32 addend and result; the product of two
// bf16 values is exact in fp32, so each is one rounding, as after converting them).
__device__ __forceinline__ void fma_bf16x2_f32(float &acc0, float &acc1, uint32_t x, uint32_t w) {
    asm("{\n\t.reg .b16 x0, x1, w0, w1;\n\t"
        "mov.b32 {x0, x1}, %2;\n\t"
        "mov.b32 {w0, w1}, %3;\n\t"
        "fma.rn.f32.bf16 %0, x0, w0, %0;\n\t"
        "fma.rn.f32.bf16 %1, x1, w1, %1;\n\t}"
        : "+f"(acc0), "+f"(acc1)
        : "r"(x), "r"(w));
}

// 16 bytes of channels as kV/2 fp32 pairs (bf16: each 32-bit word holds channels 2i, 2i+1).
template <bool kF32>
__device__ __forceinline__ void unpack16_pairs(const uint4 &u, uint64_t *p) {
    if constexpr (kF32) {
        p[0] = pair(u.x, u.y);
        p[1] = pair(u.z, u.w);
    } else {
        const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) p[i] = pair(w[i] << 16, w[i] & 0xFFFF0000u);
    }
}

// Stores kV consecutive channels (c ..) of output pixel pix (= (n*Ho + oh)*Wo + ow), rounded
// once to the output type; vector stores for whole groups in channels-last output.
template <bool kF32, int kV>
__device__ __forceinline__ void dw_store(const DwParams &p, size_t pix, size_t n, int oh, int ow, int c,
                                         const float *o, bool whole) {
    if (!p.out_nchw) {
        if constexpr (kF32) {
            float *dst = static_cast<float *>(p.y) + pix * p.C + c;
            if (whole) {
                *reinterpret_cast<float4 *>(dst) = make_float4(o[0], o[1], o[2], o[3]);
            } else {
#pragma unroll
                for (int v = 0; v < kV; ++v)
                    if (c + v < p.C) dst[v] = o[v];
            }
        } else {
            __nv_bfloat16 *dst = static_cast<__nv_bfloat16 *>(p.y) + pix * p.C + c;
            if (whole) {
                uint32_t pk[kV / 2];
#pragma unroll
                for (int i = 0; i < kV / 2; ++i) {
                    __nv_bfloat162 h = __floats2bfloat162_rn(o[2 * i], o[2 * i + 1]);
                    pk[i] = *reinterpret_cast<uint32_t *>(&h);
                }
                *reinterpret_cast<uint4 *>(dst) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
            } else {
#pragma unroll
                for (int v = 0; v < kV; ++v)
                    if (c + v < p.C) dst[v] = __float2bfloat16_rn(o[v]);
            }
        }
    } else {  // NCHW: y[n][c][oh][ow]
        const size_t plane = static_cast<size_t>(p.Ho) * p.Wo;
        const size_t at = (n * p.C + c) * plane + static_cast<size_t>(oh) * p.Wo + ow;
#pragma unroll
        for (int v = 0; v < kV; ++v) {
            if (c + v >= p.C) break;
            if constexpr (kF32)
                static_cast<float *>(p.y)[at + v * plane] = o[v];
            else
                static_cast<__nv_bfloat16 *>(p.y)[at + v * plane] = __float2bfloat16_rn(o[v]);
        }
    }
}

struct DwTile {
    int chunk, n, th, tw;
};

__device__ __forceinline__ DwTile dw_decode(const DwParams &p, int u) {
    DwTile t;
    const int per_img = p.n_th * p.n_tw;
    const int per_chunk = p.N * per_img;
    t.chunk = u / per_chunk;
    int r = u - t.chunk * per_chunk;
    t.n = r / per_img;
    r -= t.n * per_img;
    t.th = r / p.n_tw;
    t.tw = r - t.th * p.n_tw;
    return t;
}

__device__ __forceinline__ void dw_wait_quiet(uint64_t *bar, uint32_t parity, uint64_t limit_ns) {
    const uint64_t start = globaltimer_ns();
    while (!mbar_try_wait(bar, parity)) {
        if (globaltimer_ns() - start > limit_ns) return;
    }
}

// kR: output pixels per thread along a row.  kKW > 0: stride 1, unit dilation and a
// kKW x kKW filter, read through a register window; kKW = 0: any stride, dilation and
// filter, one shared-memory read per (pixel, filter column).
template <bool kF32, int kR, int kKW>
__global__ void __launch_bounds__(kDwThreads, 1) dw_kernel(const __grid_constant__ DwParams p) {
    constexpr int kV = kF32 ? 4 : 8;          // channels per 16-byte vector
    constexpr int kCC = kDwRowBytes / (kF32 ? 4 : 2);  // channels per tile
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_addr = smem_addr(smem_raw);
    uint8_t *base = smem_raw + (((raw_addr + 1023u) & ~1023u) - raw_addr);
    DwShared &sb = *reinterpret_cast<DwShared *>(base);
    const int taps = p.Kh * p.Kw;
    const int wbytes = taps * kDwRowBytes + kCC * 4;  // one warp's weights + biases
    uint8_t *wbase = base + kDwHeader;
    uint8_t *ring = wbase + p.wregion;
    const uint32_t sbytes = static_cast<uint32_t>(p.IH) * p.IW * kDwRowBytes;

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        for (int s = 0; s < p.stages; ++s) {
            mbar_init(&sb.full[s], 1);
            mbar_init(&sb.empty[s], kDwComputeWarps);
        }
        sb.abort = 0;
        fence_mbar_init();
    }
    __syncthreads();

    Watchdog wd;
    wd.abort = &sb.abort;
    wd.status = p.status;
    wd.timeout_ns = static_cast<uint64_t>(p.timeout_ns);

    if (warp == 0) {
        // ------------------------------------------------------------ TMA loads ---
        if (lane == 0) {
            prefetch_tensormap(&p.tmap_x);
            int stage = 0;
            uint32_t phase = 0;
            long long issued = 0;
            for (int u = blockIdx.x; u < p.units; u += gridDim.x) {
                const DwTile t = dw_decode(p, u);
                if (!mbar_wait(&sb.empty[stage], phase ^ 1u, wd, kDevTimeoutEmpty)) break;
                if (!p.starve) {
                    mbar_arrive_expect_tx(&sb.full[stage], sbytes);
                    tma_load_4d(ring + static_cast<size_t>(stage) * sbytes, &p.tmap_x, &sb.full[stage],
                                t.chunk * kCC, t.tw * p.TW * p.stride - p.pad_w,
                                t.th * p.TH * p.stride - p.pad, t.n);
                    ++issued;
                }
                if (++stage == p.stages) {
                    stage = 0;
                    phase ^= 1u;
                }
            }
            if (*wd.abort && issued > 0) {
                // let the copies still in flight land before the CTA goes away
                const long long first = issued > p.stages ? issued - p.stages : 0;
                for (long long i = first; i < issued; ++i)
                    dw_wait_quiet(&sb.full[i % p.stages], static_cast<uint32_t>((i / p.stages) & 1),
                                  wd.timeout_ns);
            }
        }
    } else {
        // -------------------------------------------------------------- compute ---
        const int cw = warp - 1;
        const int tid = threadIdx.x - 32;
        uint8_t *wsm = wbase + cw * wbytes;               // [taps][kCC] weights (dtype)
        float *bsm = reinterpret_cast<float *>(wsm + taps * kDwRowBytes);  // [kCC] biases
        const int groups_per_row = p.TW / kR;
        const int items = groups_per_row * p.TH * 8;
        int cur_chunk = -1;
        int stage = 0;
        uint32_t phase = 0;
        for (int u = blockIdx.x; u < p.units; u += gridDim.x) {
            const DwTile t = dw_decode(p, u);
            if (t.chunk != cur_chunk) {
                // this warp's copy of the tile's weights and biases (warp-private, so
                // no other warp can still be reading the previous chunk's)
                __syncwarp();
                const int c0 = t.chunk * kCC;
                for (int i = lane; i < taps * kCC; i += 32) {
                    const int tap = i / kCC, cc = i - tap * kCC, c = c0 + cc;
                    if constexpr (kF32) {
                        const float v = c < p.C ? __ldg(static_cast<const float *>(p.w_packed) +
                                                        (static_cast<size_t>(c) * taps + tap) * p.Cpg)
                                                : 0.f;
                        reinterpret_cast<float *>(wsm)[i] = v;
                    } else {
                        const unsigned short v =
                            c < p.C ? __ldg(static_cast<const unsigned short *>(p.w_packed) +
                                            (static_cast<size_t>(c) * taps + tap) * p.Cpg)
                                    : static_cast<unsigned short>(0);
                        reinterpret_cast<unsigned short *>(wsm)[i] = v;
                    }
                }
                for (int i = lane; i < kCC; i += 32) {
                    const int c = c0 + i;
                    float b = 0.f;
                    if (p.bias && c < p.C) {
                        if constexpr (kF32)
                            b = __ldg(static_cast<const float *>(p.bias) + c);
                        else
                            b = __uint_as_float(static_cast<uint32_t>(
                                                    __ldg(static_cast<const unsigned short *>(p.bias) + c))
                                                << 16);
                    }
                    bsm[i] = b;
                }
                __syncwarp();
                cur_chunk = t.chunk;
            }
            const bool ok = mbar_wait(&sb.full[stage], phase, wd, kDevTimeoutFull);
            if (!__all_sync(0xffffffffu, ok)) break;
            const uint8_t *stg = ring + static_cast<size_t>(stage) * sbytes;
            if constexpr (kKW == 0) {
                // general form: 16 bytes of channels of kR pixels of one output row per item
                for (int it = tid; it < items; it += 32 * kDwComputeWarps) {
                    const int cg = it & 7, pg = it >> 3;
                    const int py = pg / groups_per_row;
                    const int px0 = (pg - py * groups_per_row) * kR;
                    const int oh = t.th * p.TH + py;
                    const int ow0 = t.tw * p.TW + px0;
                    if (oh >= p.Ho || ow0 >= p.Wo) continue;
                    float acc[kR][kV];
                    {
    #pragma unroll
                        for (int r = 0; r < kR; ++r)
    #pragma unroll
                            for (int v = 0; v < kV; ++v) acc[r][v] = 0.f;
                        for (int kh = 0; kh < p.Kh; ++kh) {
                            const int row = py * p.stride + kh * p.dilation;
                            const uint8_t *rp = stg + static_cast<size_t>(row) * p.IW * kDwRowBytes + cg * 16;
                            const uint8_t *wp = wsm + kh * p.Kw * kDwRowBytes + cg * 16;
                            for (int kw = 0; kw < p.Kw; ++kw) {
                                if constexpr (kF32) {
                                    float wv[kV];
                                    unpack16<kF32>(*reinterpret_cast<const uint4 *>(wp + kw * kDwRowBytes), wv);
    #pragma unroll
                                    for (int r = 0; r < kR; ++r) {
                                        const int col = (px0 + r) * p.stride + kw * p.dilation;
                                        float xv[kV];
                                        unpack16<kF32>(*reinterpret_cast<const uint4 *>(rp + col * kDwRowBytes), xv);
    #pragma unroll
                                        for (int v = 0; v < kV; ++v) acc[r][v] = fmaf(xv[v], wv[v], acc[r][v]);
                                    }
                                } else {
                                    // bf16: mixed-precision FMAs on the packed words (the same
                                    // exact products and roundings as converting them first)
                                    const uint4 wq = *reinterpret_cast<const uint4 *>(wp + kw * kDwRowBytes);
    #pragma unroll
                                    for (int r = 0; r < kR; ++r) {
                                        const int col = (px0 + r) * p.stride + kw * p.dilation;
                                        const uint4 xq = *reinterpret_cast<const uint4 *>(rp + col * kDwRowBytes);
                                        fma_bf16x2_f32(acc[r][0], acc[r][1], xq.x, wq.x);
                                        fma_bf16x2_f32(acc[r][2], acc[r][3], xq.y, wq.y);
                                        fma_bf16x2_f32(acc[r][4], acc[r][5], xq.z, wq.z);
                                        fma_bf16x2_f32(acc[r][6], acc[r][7], xq.w, wq.w);
                                    }
                                }
                            }
                        }
                    }
                    // epilogue: + bias, one rounding, store
                    const int c = t.chunk * kCC + cg * kV;
                    if (c >= p.C) continue;
                    float bv[kV];
    #pragma unroll
                    for (int v = 0; v < kV; ++v) bv[v] = bsm[cg * kV + v];
                    const bool whole = c + kV <= p.C && p.vec_ok;
    #pragma unroll
                    for (int r = 0; r < kR; ++r) {
                        const int ow = ow0 + r;
                        if (ow >= p.Wo) break;
                        float o[kV];
    #pragma unroll
                        for (int v = 0; v < kV; ++v) o[v] = acc[r][v] + bv[v];
                        const size_t pix = (static_cast<size_t>(t.n) * p.Ho + oh) * p.Wo + ow;
                        if (!p.out_nchw) {
                            if constexpr (kF32) {
                                float *dst = static_cast<float *>(p.y) + pix * p.C + c;
                                if (whole) {
                                    *reinterpret_cast<float4 *>(dst) = make_float4(o[0], o[1], o[2], o[3]);
                                } else {
    #pragma unroll
                                    for (int v = 0; v < kV; ++v)
                                        if (c + v < p.C) dst[v] = o[v];
                                }
                            } else {
                                __nv_bfloat16 *dst = static_cast<__nv_bfloat16 *>(p.y) + pix * p.C + c;
                                if (whole) {
                                    uint32_t pk[4];
    #pragma unroll
                                    for (int i = 0; i < 4; ++i) {
                                        __nv_bfloat162 h = __floats2bfloat162_rn(o[2 * i], o[2 * i + 1]);
                                        pk[i] = *reinterpret_cast<uint32_t *>(&h);
                                    }
                                    *reinterpret_cast<uint4 *>(dst) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
                                } else {
    #pragma unroll
                                    for (int v = 0; v < kV; ++v)
                                        if (c + v < p.C) dst[v] = __float2bfloat16_rn(o[v]);
                                }
                            }
                        } else {  // NCHW: y[n][c][oh][ow]
                            const size_t plane = static_cast<size_t>(p.Ho) * p.Wo;
                            const size_t at = (static_cast<size_t>(t.n) * p.C + c) * plane +
                                              static_cast<size_t>(oh) * p.Wo + ow;
    #pragma unroll
                            for (int v = 0; v < kV; ++v) {
                                if (c + v >= p.C) break;
                                if constexpr (kF32)
                                    static_cast<float *>(p.y)[at + v * plane] = o[v];
                                else
                                    static_cast<__nv_bfloat16 *>(p.y)[at + v * plane] = __float2bfloat16_rn(o[v]);
                            }
                        }
                    }
                }
            }
            if constexpr (kKW > 0) {
                // Stride 1, unit dilation, kKW x kKW: every filter row reads a window of
                // kR + kKW - 1 input pixels once; products accumulate in fp32 started from
                // the bias (bf16: mixed-precision FMAs on the raw words; fp32: paired FMAs).
                // A tile row holds two groups of kR pixels (TW = 2*kR).
                constexpr int kP = kV / 2;
                for (int it = tid; it < items; it += 32 * kDwComputeWarps) {
                    const int cg = it & 7, pg = it >> 3;
                    const int py = pg >> 1, px0 = (pg & 1) * kR;
                    const int oh = t.th * p.TH + py;
                    const int ow0 = t.tw * p.TW + px0;
                    const int c = t.chunk * kCC + cg * kV;
                    if (oh >= p.Ho || ow0 >= p.Wo || c >= p.C) continue;
                    const uint8_t *rp0 = stg + (static_cast<uint32_t>(py) * p.IW + px0) * kDwRowBytes + cg * 16;
                    const uint8_t *wp0 = wsm + cg * 16;
                    float o_all[kR][kV];
                    if constexpr (!kF32) {
                        // bf16: the window's words as they are, mixed-precision FMAs into
                        // fp32 accumulators started from the bias (no unpacking)
                        const float *bq = bsm + cg * kV;
#pragma unroll
                        for (int r = 0; r < kR; ++r)
#pragma unroll
                            for (int v = 0; v < kV; ++v) o_all[r][v] = bq[v];
#pragma unroll
                        for (int kh = 0; kh < kKW; ++kh) {
                            const uint8_t *rp = rp0 + static_cast<uint32_t>(kh) * p.IW * kDwRowBytes;
                            const uint8_t *wp = wp0 + kh * kKW * kDwRowBytes;
                            uint4 win[kR + kKW - 1];
#pragma unroll
                            for (int j = 0; j < kR + kKW - 1; ++j)
                                win[j] = *reinterpret_cast<const uint4 *>(rp + j * kDwRowBytes);
#pragma unroll
                            for (int kw = 0; kw < kKW; ++kw) {
                                const uint4 wv = *reinterpret_cast<const uint4 *>(wp + kw * kDwRowBytes);
#pragma unroll
                                for (int r = 0; r < kR; ++r) {
                                    const uint4 xv = win[r + kw];
                                    fma_bf16x2_f32(o_all[r][0], o_all[r][1], xv.x, wv.x);
                                    fma_bf16x2_f32(o_all[r][2], o_all[r][3], xv.y, wv.y);
                                    fma_bf16x2_f32(o_all[r][4], o_all[r][5], xv.z, wv.z);
                                    fma_bf16x2_f32(o_all[r][6], o_all[r][7], xv.w, wv.w);
                                }
                            }
                        }
                    } else {
                        uint64_t accp[kR][kP];
                        {
                            const float *bq = bsm + cg * kV;
                            uint64_t b2[kP];
#pragma unroll
                            for (int v = 0; v < kP; ++v) b2[v] = pair(__float_as_uint(bq[2 * v]), __float_as_uint(bq[2 * v + 1]));
#pragma unroll
                            for (int r = 0; r < kR; ++r)
#pragma unroll
                                for (int v = 0; v < kP; ++v) accp[r][v] = b2[v];
                        }
#pragma unroll
                        for (int kh = 0; kh < kKW; ++kh) {
                            const uint8_t *rp = rp0 + static_cast<uint32_t>(kh) * p.IW * kDwRowBytes;
                            const uint8_t *wp = wp0 + kh * kKW * kDwRowBytes;
                            uint64_t win[kR + kKW - 1][kP];
#pragma unroll
                            for (int j = 0; j < kR + kKW - 1; ++j)
                                unpack16_pairs<kF32>(*reinterpret_cast<const uint4 *>(rp + j * kDwRowBytes), win[j]);
#pragma unroll
                            for (int kw = 0; kw < kKW; ++kw) {
                                uint64_t wv[kP];
                                unpack16_pairs<kF32>(*reinterpret_cast<const uint4 *>(wp + kw * kDwRowBytes), wv);
#pragma unroll
                                for (int r = 0; r < kR; ++r)
#pragma unroll
                                    for (int v = 0; v < kP; ++v) fma2(accp[r][v], win[r + kw][v], wv[v]);
                            }
                        }
#pragma unroll
                        for (int r = 0; r < kR; ++r)
#pragma unroll
                            for (int v = 0; v < kP; ++v) unpair(accp[r][v], o_all[r][2 * v], o_all[r][2 * v + 1]);
                    }
                    // epilogue: one rounding, store (the bias is already in)
                    const bool whole = c + kV <= p.C && p.vec_ok;
                    const size_t pix0 = (static_cast<size_t>(t.n) * p.Ho + oh) * p.Wo + ow0;
#pragma unroll
                    for (int r = 0; r < kR; ++r) {
                        if (ow0 + r >= p.Wo) break;
                        dw_store<kF32, kV>(p, pix0 + r, static_cast<size_t>(t.n), oh, ow0 + r, c, o_all[r], whole);
                    }
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&sb.empty[stage]);
            if (++stage == p.stages) {
                stage = 0;
                phase ^= 1u;
            }
        }
    }
    __syncthreads();
}

template <bool kF32, int kR, int kKW>
cudaError_t dw_launch_one(const DwParams &p, int grid, size_t smem, cudaStream_t s) {
    auto kern = dw_kernel<kF32, kR, kKW>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    kern<<<grid, kDwThreads, smem, s>>>(p);
    return cudaGetLastError();
}

template <bool kF32>
cudaError_t dw_launch_t(const DwParams &p, int window_k, int grid, size_t smem, cudaStream_t s) {
    switch (window_k) {
        case 3: return dw_launch_one<kF32, 4, 3>(p, grid, smem, s);
        case 5: return dw_launch_one<kF32, 4, 5>(p, grid, smem, s);
        case 7: return dw_launch_one<kF32, 4, 7>(p, grid, smem, s);
        case 0: return dw_launch_one<kF32, 4, 0>(p, grid, smem, s);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace

int dw_pixels_per_thread() { return 4; }
int dw_threads() { return kDwThreads; }
int dw_compute_warps() { return kDwComputeWarps; }
int dw_max_stages() { return kDwMaxStages; }
size_t dw_header_bytes() { return 1024 /* alignment slack */ + kDwHeader; }

cudaError_t launch_depthwise(const DwParams &p, bool f32, int window_k, int grid, size_t smem,
                             cudaStream_t stream) {
    if (p.stages < 2 || p.stages > kDwMaxStages) return cudaErrorInvalidValue;
    return f32 ? dw_launch_t<true>(p, window_k, grid, smem, stream)
               : dw_launch_t<false>(p, window_k, grid, smem, stream);
}

}  // namespace conv2d_b200
