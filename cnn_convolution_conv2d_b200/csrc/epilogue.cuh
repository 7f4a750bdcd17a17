// epilogue.cuh -- storing accumulator rows of the convolution's matrix product:
// bias add in fp32, one rounding to the output type, and the write in the
// requested layout.  Shared by the tensor-core kernels.
#pragma once

#include <cuda_bf16.h>

#include "common.cuh"

namespace conv2d_b200 {

// Where and how a kernel writes its output rows.
struct OutDesc {
    void *y;
    const void *bias;
    int M, HoWo, Cout, Cout_g;
    int out_mode;
    int vec_ok;
};

// Rounds to the nearest value with 10 explicit mantissa bits (ties away from
// zero): the operand precision of the tensor cores' tf32 mode.
__device__ __forceinline__ float tf32_round(float v) {
    return __uint_as_float((__float_as_uint(v) + 0x1000u) & 0xFFFFE000u);
}

// Stores 16 consecutive accumulator columns [col0, col0 + 16) of output row m
// (group g), adding bias unless the output is a split partial sum.
template <bool kF32>
__device__ __forceinline__ void store16(const OutDesc &p, int m, int g, int col0, int split,
                                        const float *vin) {
    if (m >= p.M) return;
    const int nvalid = min(16, p.Cout_g - col0);
    if (nvalid <= 0) return;
    const int oc0 = g * p.Cout_g + col0;
    float v[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) v[i] = vin[i];

    if (p.out_mode == kOutPartial) {
        float *dst = static_cast<float *>(p.y) +
                     (static_cast<size_t>(split) * p.M + m) * p.Cout + oc0;
        if (nvalid == 16 && p.vec_ok) {
            float4 *d4 = reinterpret_cast<float4 *>(dst);
#pragma unroll
            for (int i = 0; i < 4; ++i)
                d4[i] = make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
        } else {
#pragma unroll
            for (int i = 0; i < 16; ++i)
                if (i < nvalid) dst[i] = v[i];
        }
        return;
    }
    if (p.bias) {
        if constexpr (kF32) {
            const float *b = static_cast<const float *>(p.bias) + oc0;
#pragma unroll
            for (int i = 0; i < 16; ++i)
                if (i < nvalid) v[i] += __ldg(b + i);
        } else {
            const __nv_bfloat16 *b = static_cast<const __nv_bfloat16 *>(p.bias) + oc0;
#pragma unroll
            for (int i = 0; i < 16; ++i)
                if (i < nvalid) v[i] += __bfloat162float(b[i]);
        }
    }
    if (p.out_mode == kOutNHWC) {
        if constexpr (kF32) {
            float *dst = static_cast<float *>(p.y) + static_cast<size_t>(m) * p.Cout + oc0;
            if (nvalid == 16 && p.vec_ok) {
                float4 *d4 = reinterpret_cast<float4 *>(dst);
#pragma unroll
                for (int i = 0; i < 4; ++i)
                    d4[i] = make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
            } else {
#pragma unroll
                for (int i = 0; i < 16; ++i)
                    if (i < nvalid) dst[i] = v[i];
            }
        } else {
            __nv_bfloat16 *dst =
                static_cast<__nv_bfloat16 *>(p.y) + static_cast<size_t>(m) * p.Cout + oc0;
            if (nvalid == 16 && p.vec_ok) {
                uint32_t packed[8];
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    __nv_bfloat162 h = __floats2bfloat162_rn(v[2 * i], v[2 * i + 1]);
                    packed[i] = *reinterpret_cast<uint32_t *>(&h);
                }
                uint4 *d4 = reinterpret_cast<uint4 *>(dst);
                d4[0] = make_uint4(packed[0], packed[1], packed[2], packed[3]);
                d4[1] = make_uint4(packed[4], packed[5], packed[6], packed[7]);
            } else {
#pragma unroll
                for (int i = 0; i < 16; ++i)
                    if (i < nvalid) dst[i] = __float2bfloat16_rn(v[i]);
            }
        }
    } else {  // kOutNCHW: lanes hold consecutive pixels, so each column is a coalesced row
        const int n = m / p.HoWo;
        const int pix = m - n * p.HoWo;
        const size_t base = (static_cast<size_t>(n) * p.Cout + oc0) * p.HoWo + pix;
        if constexpr (kF32) {
            float *dst = static_cast<float *>(p.y) + base;
#pragma unroll
            for (int i = 0; i < 16; ++i)
                if (i < nvalid) dst[static_cast<size_t>(i) * p.HoWo] = v[i];
        } else {
            __nv_bfloat16 *dst = static_cast<__nv_bfloat16 *>(p.y) + base;
#pragma unroll
            for (int i = 0; i < 16; ++i)
                if (i < nvalid) dst[static_cast<size_t>(i) * p.HoWo] = __float2bfloat16_rn(v[i]);
        }
    }
}

}  // namespace conv2d_b200
