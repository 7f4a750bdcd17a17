// wgrad.cu -- the weight gradient of the convolution as a tcgen05 matrix product whose
// reduction runs over the output pixels.
//
// The im2col/GEMM tutorial (zskr.cn/news/1820658) §3.3 writes the weight gradient as
// dW_row = dout_col @ X_col^T: rows are output channels, columns are the (c, kh, kw)
// entries of one filter, and the reduction runs over every output pixel of every image.
// The "手撕 Conv2D" page (lpnh.cn/news/2493075) §5.1 gives the same sum element by
// element, dW[oc][c][kh][kw] = sum_{n, oh, ow} dout[n][oc][oh][ow] * x[n][c][oh*s + kh*d - p][ow*s + kw*d - p].
// Here X_col is never formed: for one filter tap (kh, kw) the X_col^T block of PK
// consecutive output pixels is exactly what the tensor memory accelerator's im2col mode
// delivers (PK pixels x 128 bytes of channels, zero outside the image), and the dout_col
// block is a tiled load of the channels-last dout (PK pixels x 128 bytes of output
// channels).  Both land in shared memory with the pixel index along the rows and the
// channel contiguous, i.e. with the MN dimension contiguous and the reduction (pixels)
// strided, which tcgen05.mma reads directly as "MN-major" operands (transpose bits of
// the instruction descriptor), so neither operand is transposed in memory.
//
// Tiles: M = 128 output channels of one group (tensor-memory lanes), N = BN channels of
// one filter tap (columns), reduction = pixels in stages of PK (64 bf16, 32 fp32).  In bf16
// a unit may take two such row tiles (OM = 2: 256 output channels, two products per step
// into two accumulators, one accumulator set -- a unit's reduction is long, so the drain
// need not overlap it): each staged block of x then feeds twice the products, which cuts
// the bytes brought into the SM per multiply-add by a third.  (Measured on the 3x3 layer:
// 263.9 -> 193.7 us; with stages of 32 pixels instead, 277 us.)  The
// reduction over all pixels is long and the tile count small, so it is split across SMs;
// each unit writes fp32 partial sums [split][C_out][taps][Cpg] and a reduction kernel
// (layout.cu) adds the splits and writes dW in the weight's own OIHW layout.
//
// Persistent and warp-specialised like the forward kernel (igemm.cu): warp 0 issues the
// TMA loads, warp 1 allocates tensor memory and issues the MMAs from one thread, warps
// 2..9 (bf16) or 2..5 (fp32) drain the double-buffered accumulator.  fp32: the tensor
// cores read tf32 operands MN-major only in a 32-byte-atom swizzle that these loads do not
// produce, so warps 6..9 rewrite every staged block K-major (pixels contiguous, the
// forward kernel's 128-byte swizzle), split into tf32 hi and lo parts for three products
// per multiply-add, and the accumulator restarts every few stages with the chunks summed
// in fp32 registers (as in the forward fp32 path).  Every wait is bounded (see ptx.cuh).
#include "common.cuh"
#include "epilogue.cuh"
#include "ptx.cuh"

namespace conv2d_b200 {
namespace {

using namespace ptx;

constexpr int kWgMaxStages = 8;
constexpr int kWgHeader = 1024;
constexpr int kWgThreads = 320;
constexpr int kWgMaxBNf32 = 128;

struct WgShared {
    uint64_t full[kWgMaxStages];
    uint64_t empty[kWgMaxStages];
    uint64_t converted[kWgMaxStages];
    uint64_t acc_full[2];
    uint64_t acc_empty[2];
    uint64_t drain;
    uint32_t tmem_base;
    int abort;
};
static_assert(sizeof(WgShared) <= kWgHeader, "header too small");

template <bool kF32>
__host__ __device__ constexpr int wg_pk() { return kF32 ? 32 : 64; }  // pixels per stage
template <bool kF32>
__host__ __device__ constexpr int wg_epi_warps() { return kF32 ? 4 : 8; }

// bytes of one operand block of PK pixel rows x 128 bytes of channels
template <bool kF32>
__host__ __device__ constexpr uint32_t wg_block_bytes() { return static_cast<uint32_t>(wg_pk<kF32>()) * 128u; }

struct WgUnit {
    int split, otile, g, tap, ctile, k0, k1;
};

__device__ __forceinline__ WgUnit wg_decode(const WgradParams &p, int u) {
    WgUnit t;
    const int per_split = p.units / p.splits;
    t.split = u / per_split;
    int r = u - t.split * per_split;
    t.ctile = r % p.n_ctiles;
    r /= p.n_ctiles;
    t.tap = r % p.taps;
    r /= p.taps;
    t.g = r % p.groups;
    t.otile = r / p.groups;
    t.k0 = static_cast<int>((static_cast<long long>(t.split) * p.kstages) / p.splits);
    t.k1 = static_cast<int>((static_cast<long long>(t.split + 1) * p.kstages) / p.splits);
    return t;
}

__device__ __forceinline__ void wg_wait_quiet(uint64_t *bar, uint32_t parity, uint64_t limit_ns) {
    const uint64_t start = globaltimer_ns();
    while (!mbar_try_wait(bar, parity)) {
        if (globaltimer_ns() - start > limit_ns) return;
    }
}

template <bool kF32, bool kM2>
__global__ void __launch_bounds__(kWgThreads, 1) wgrad_kernel(const __grid_constant__ WgradParams p) {
    static_assert(!(kF32 && kM2), "two row tiles per unit: bf16 only");
    constexpr int kOM = kM2 ? 2 : 1;                     // 128-row tiles of output channels per unit
    constexpr int kNBuf = kM2 ? 1 : 2;                   // accumulator sets in tensor memory
    constexpr int kPK = wg_pk<kF32>();
    constexpr uint32_t kBlk = wg_block_bytes<kF32>();   // one 128-byte-wide operand block
    constexpr int kCC = kF32 ? 32 : 64;                  // channels per 128 bytes
    constexpr int kKS = kF32 ? 8 : 16;                   // pixels per MMA (K of one instruction)
    constexpr int kEpi = wg_epi_warps<kF32>();
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_addr = smem_addr(smem_raw);
    uint8_t *base = smem_raw + (((raw_addr + 1023u) & ~1023u) - raw_addr);
    WgShared &sb = *reinterpret_cast<WgShared *>(base);
    uint8_t *ring = base + kWgHeader;

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int BN = p.BN;
    const int a_blocks = kOM * 128 / kCC;               // 128 output channels per row tile
    const int b_blocks = BN / kCC;
    const uint32_t a_bytes = a_blocks * kBlk, b_bytes = b_blocks * kBlk;
    const uint32_t tx_bytes = a_bytes + b_bytes;
    // fp32: the raw (MN-major) blocks, then K-major hi and lo copies of both operands
    const uint32_t sbytes = tx_bytes * (kF32 ? 3u : 1u);

    if (threadIdx.x == 0) {
        for (int s = 0; s < p.stages; ++s) {
            mbar_init(&sb.full[s], 1);
            mbar_init(&sb.empty[s], 1);
            mbar_init(&sb.converted[s], 128);
        }
        for (int i = 0; i < kNBuf; ++i) {
            mbar_init(&sb.acc_full[i], 1);
            mbar_init(&sb.acc_empty[i], kEpi);
        }
        mbar_init(&sb.drain, 1);
        sb.abort = 0;
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc(&sb.tmem_base, p.tmem_cols);
        tmem_relinquish();
    }
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    const uint32_t tmem_base = sb.tmem_base;

    Watchdog wd;
    wd.abort = &sb.abort;
    wd.status = p.status;
    wd.timeout_ns = static_cast<uint64_t>(p.timeout_ns);

    if (warp == 0) {
        // ------------------------------------------------------ TMA producer ---
        if (lane == 0) {
            prefetch_tensormap(&p.tmap_dy);
            prefetch_tensormap(&p.tmap_x);
            int stage = 0;
            uint32_t phase = 0;
            long long issued = 0;
            bool ok = true;
            for (int u = blockIdx.x; ok && u < p.units; u += gridDim.x) {
                const WgUnit t = wg_decode(p, u);
                const int kh = t.tap / p.Kw, kw = t.tap - (t.tap / p.Kw) * p.Kw;
                const int oc0 = t.g * p.dy_cpg + t.otile * kOM * 128;
                const int c0 = t.g * p.Cpg + t.ctile * BN;
                for (int kb = t.k0; kb < t.k1; ++kb) {
                    if (!mbar_wait(&sb.empty[stage], phase ^ 1u, wd, kDevTimeoutEmpty)) {
                        ok = false;
                        break;
                    }
                    uint8_t *st = ring + static_cast<size_t>(stage) * sbytes;
                    if (!p.starve) {
                        mbar_arrive_expect_tx(&sb.full[stage], tx_bytes);
                        const int m0 = kb * kPK;
                        for (int j = 0; j < a_blocks; ++j)
                            tma_load_2d(st + j * kBlk, &p.tmap_dy, &sb.full[stage], oc0 + j * kCC, m0);
                        const int img = m0 / p.HoWo;
                        const int rem = m0 - img * p.HoWo;
                        const int oh = rem / p.Wo;
                        const int ow = rem - oh * p.Wo;
                        for (int j = 0; j < b_blocks; ++j)
                            tma_load_im2col_4d(st + a_bytes + j * kBlk, &p.tmap_x, &sb.full[stage],
                                               c0 + j * kCC, ow * p.stride - p.pad, oh * p.stride - p.pad, img,
                                               static_cast<uint16_t>(kw * p.dilation),
                                               static_cast<uint16_t>(kh * p.dilation));
                        ++issued;
                    }
                    if (++stage == p.stages) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
            }
            if (*wd.abort && issued > 0) {
                const long long first = issued > p.stages ? issued - p.stages : 0;
                for (long long i = first; i < issued; ++i)
                    wg_wait_quiet(&sb.full[i % p.stages], static_cast<uint32_t>((i / p.stages) & 1), wd.timeout_ns);
            }
        }
    } else if (warp == 1) {
        // --------------------------------------------------- tensor-core issue ---
        if (lane == 0) {
            // bf16: MN-major A (output channels contiguous) and B (input channels
            // contiguous); fp32: the converted K-major copies
            const uint32_t idesc = kF32 ? instr_desc(2u, 128, static_cast<uint32_t>(BN))
                                        : (instr_desc(1u, 128, static_cast<uint32_t>(BN)) | (1u << 15) | (1u << 16));
            int stage = 0;
            uint32_t phase = 0;
            int abuf = 0;
            uint32_t aphase = 0;
            bool ok = true;
            for (int u = blockIdx.x; ok && u < p.units; u += gridDim.x) {
                const WgUnit t = wg_decode(p, u);
                const int cs = p.chunk_stages > 0 ? p.chunk_stages : t.k1 - t.k0;
                for (int c0 = t.k0; ok && c0 < t.k1; c0 += cs) {
                    const int c1 = min(c0 + cs, t.k1);
                    if (!mbar_wait(&sb.acc_empty[abuf], aphase ^ 1u, wd, kDevTimeoutAccEmpty)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after_sync();
                    const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(abuf * kOM * BN);
                    for (int kb = c0; kb < c1; ++kb) {
                        uint64_t *ready = kF32 ? &sb.converted[stage] : &sb.full[stage];
                        if (!mbar_wait(ready, phase, wd, kF32 ? kDevTimeoutConvert : kDevTimeoutFull)) {
                            ok = false;
                            break;
                        }
                        tc_fence_after_sync();
                        const uint32_t a = smem_addr(ring + static_cast<size_t>(stage) * sbytes);
                        const uint32_t b = a + a_bytes;
#pragma unroll
                        for (int ks = 0; ks < kPK / kKS; ++ks) {
                            const uint32_t off = static_cast<uint32_t>(ks * kKS * 128);
                            const uint32_t acc = (kb == c0 && ks == 0) ? 0u : 1u;
                            if constexpr (kF32) {
                                // K-major copies: rows of 32 pixels (128 bytes), 32 bytes of k per MMA
                                const uint32_t ah = a + tx_bytes, bh = ah + a_bytes;
                                const uint32_t al = a + 2 * tx_bytes, bl = al + a_bytes;
                                const uint32_t ko = static_cast<uint32_t>(ks * 32);
                                mma_tf32(d_tmem, smem_desc(al + ko, 16, 1024, kSw128),
                                         smem_desc(bh + ko, 16, 1024, kSw128), idesc, acc);
                                mma_tf32(d_tmem, smem_desc(ah + ko, 16, 1024, kSw128),
                                         smem_desc(bl + ko, 16, 1024, kSw128), idesc, 1u);
                                mma_tf32(d_tmem, smem_desc(ah + ko, 16, 1024, kSw128),
                                         smem_desc(bh + ko, 16, 1024, kSw128), idesc, 1u);
                            } else {
#pragma unroll
                                for (int o = 0; o < kOM; ++o)  // row tile o: A blocks 2o, 2o+1
                                    mma_bf16(d_tmem + static_cast<uint32_t>(o * BN),
                                             smem_desc(a + static_cast<uint32_t>(o * 2) * kBlk + off, kBlk, 1024, kSw128),
                                             smem_desc(b + off, kBlk, 1024, kSw128), idesc, acc);
                            }
                        }
                        mma_commit(&sb.empty[stage]);
                        if (++stage == p.stages) {
                            stage = 0;
                            phase ^= 1u;
                        }
                    }
                    if (!ok) break;
                    mma_commit(&sb.acc_full[abuf]);
                    if (++abuf == kNBuf) {
                        abuf = 0;
                        aphase ^= 1u;
                    }
                }
            }
            if (!ok || *wd.abort) {
                mma_commit(&sb.drain);
                wg_wait_quiet(&sb.drain, 0, wd.timeout_ns);
            }
        }
        __syncwarp();
    } else if (warp < 2 + kEpi) {
        // ------------------------------------------------------------ epilogue ---
        const int quarter = warp & 3;
        const int half = (warp - 2) >> 2;
        const int cspan = kF32 ? BN : BN / 2;  // BN is a multiple of 64
        const int c_lo = half * cspan, c_hi = min(BN, c_lo + cspan);
        const int row = quarter * 32 + lane;   // output channel within the 128-row tile
        const uint32_t lane_base = static_cast<uint32_t>(quarter * 32) << 16;
        int abuf = 0;
        uint32_t aphase = 0;
        for (int u = blockIdx.x; u < p.units; u += gridDim.x) {
            const WgUnit t = wg_decode(p, u);
            if constexpr (kF32) {
                const int oc_l = t.otile * 128 + row;
                const bool valid = oc_l < p.Cout_g;
                float *dst = p.ws + ((static_cast<size_t>(t.split) * p.Cout + t.g * p.Cout_g + (valid ? oc_l : 0)) *
                                         p.taps + t.tap) * p.Cpg + t.ctile * BN;
                const int cs = p.chunk_stages > 0 ? p.chunk_stages : t.k1 - t.k0;
                const int nch = (t.k1 - t.k0 + cs - 1) / cs;
                float acc[kWgMaxBNf32];
#pragma unroll
                for (int i = 0; i < kWgMaxBNf32; ++i) acc[i] = 0.f;
                bool ok = true;
                for (int ch = 0; ch < nch; ++ch) {
                    ok = mbar_wait(&sb.acc_full[abuf], aphase, wd, kDevTimeoutAccFull);
                    if (!__all_sync(0xffffffffu, ok)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after_sync();
                    const uint32_t taddr = tmem_base + lane_base + static_cast<uint32_t>(abuf * BN);
#pragma unroll
                    for (int c = 0; c < kWgMaxBNf32 / 16; ++c) {
                        if (c * 16 < BN) {
                            uint32_t r[16];
                            tmem_ld_x16(taddr + static_cast<uint32_t>(c * 16), r);
                            tmem_ld_wait();
#pragma unroll
                            for (int i = 0; i < 16; ++i) acc[c * 16 + i] += __uint_as_float(r[i]);
                        }
                    }
                    tc_fence_before_sync();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&sb.acc_empty[abuf]);
                    abuf ^= 1;
                    if (abuf == 0) aphase ^= 1u;
                }
                if (!ok) break;
                if (valid) {
#pragma unroll
                    for (int c = 0; c < kWgMaxBNf32 / 4; ++c)
                        if (c * 4 < BN)
                            *reinterpret_cast<float4 *>(dst + 4 * c) =
                                make_float4(acc[4 * c], acc[4 * c + 1], acc[4 * c + 2], acc[4 * c + 3]);
                }
            } else {
                const bool ok = mbar_wait(&sb.acc_full[abuf], aphase, wd, kDevTimeoutAccFull);
                if (!__all_sync(0xffffffffu, ok)) break;
                tc_fence_after_sync();
#pragma unroll
                for (int o = 0; o < kOM; ++o) {
                    const int oc_l = (t.otile * kOM + o) * 128 + row;
                    const bool valid = oc_l < p.Cout_g;
                    float *dst = p.ws + ((static_cast<size_t>(t.split) * p.Cout + t.g * p.Cout_g + (valid ? oc_l : 0)) *
                                             p.taps + t.tap) * p.Cpg + t.ctile * BN;
                    const uint32_t taddr = tmem_base + lane_base + static_cast<uint32_t>((abuf * kOM + o) * BN);
                    for (int c = c_lo; c < c_hi; c += 16) {
                        uint32_t r[16];
                        tmem_ld_x16(taddr + static_cast<uint32_t>(c), r);
                        tmem_ld_wait();
                        if (valid) {
#pragma unroll
                            for (int i = 0; i < 4; ++i)
                                *reinterpret_cast<float4 *>(dst + c + 4 * i) =
                                    make_float4(__uint_as_float(r[4 * i]), __uint_as_float(r[4 * i + 1]),
                                                __uint_as_float(r[4 * i + 2]), __uint_as_float(r[4 * i + 3]));
                        }
                    }
                }
                tc_fence_before_sync();
                __syncwarp();
                if (lane == 0) mbar_arrive(&sb.acc_empty[abuf]);
                if (++abuf == kNBuf) {
                    abuf = 0;
                    aphase ^= 1u;
                }
            }
        }
    } else if constexpr (kF32) {
        // ------------------------------------------- fp32 -> tf32 hi/lo split ---
        const int tid = (warp - 6) * 32 + lane;  // 0..127
        int stage = 0;
        uint32_t phase = 0;
        bool ok = true;
        for (int u = blockIdx.x; ok && u < p.units; u += gridDim.x) {
            const WgUnit t = wg_decode(p, u);
            for (int kb = t.k0; kb < t.k1; ++kb) {
                if (!mbar_wait(&sb.full[stage], phase, wd, kDevTimeoutFull)) {
                    ok = false;
                    break;
                }
                // Raw block j of an operand: PK pixel rows of 128 bytes (32 MN elements),
                // 16-byte chunk q of row p at chunk q ^ (p & 7).  K-major copy: MN element
                // r of the operand is row r (128 bytes = 32 pixels), 16-byte chunk q of row r
                // at q ^ (r & 7), 8-row groups 1024 bytes apart.  Each thread moves one
                // 16-byte raw chunk (four MN elements of one pixel) per step.
                const uint8_t *raw = ring + static_cast<size_t>(stage) * sbytes;
                uint8_t *hi = const_cast<uint8_t *>(raw) + tx_bytes;
                uint8_t *lo = const_cast<uint8_t *>(raw) + 2 * tx_bytes;
                const int chunks = static_cast<int>(tx_bytes / 16);
                for (int i = tid; i < chunks; i += 128) {
                    const int blk = i / (kPK * 8);          // 8 chunks per 128-byte row
                    const int rem = i - blk * (kPK * 8);
                    const int px = rem >> 3, q = rem & 7;
                    const float4 v = *reinterpret_cast<const float4 *>(raw + blk * kBlk + px * 128 +
                                                                       ((q ^ (px & 7)) << 4));
                    const float vv[4] = {v.x, v.y, v.z, v.w};
                    // operand row of MN element (blk*32 + 4q + e); B follows A's 128 rows
                    const uint32_t region = blk < a_blocks ? 0u : a_bytes;
                    const int r0 = (blk < a_blocks ? blk : blk - a_blocks) * 32 + 4 * q;
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const int r = r0 + e;
                        const uint32_t off = region + static_cast<uint32_t>(r >> 3) * 1024u +
                                             static_cast<uint32_t>(r & 7) * 128u +
                                             static_cast<uint32_t>(((px >> 2) ^ (r & 7)) << 4) +
                                             static_cast<uint32_t>(px & 3) * 4u;
                        const float h = tf32_round(vv[e]);
                        *reinterpret_cast<float *>(hi + off) = h;
                        *reinterpret_cast<float *>(lo + off) = tf32_round(vv[e] - h);
                    }
                }
                fence_proxy_async_smem();
                mbar_arrive(&sb.converted[stage]);
                if (++stage == p.stages) {
                    stage = 0;
                    phase ^= 1u;
                }
            }
        }
    }

    tc_fence_before_sync();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after_sync();
        tmem_dealloc(tmem_base, p.tmem_cols);
    }
}

template <bool kF32, bool kM2>
cudaError_t wgrad_launch_t(const WgradParams &p, int grid, size_t smem, cudaStream_t s) {
    auto kern = wgrad_kernel<kF32, kM2>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    kern<<<grid, kWgThreads, smem, s>>>(p);
    return cudaGetLastError();
}

}  // namespace

int wgrad_pixels_per_stage(bool f32) { return f32 ? wg_pk<true>() : wg_pk<false>(); }
int wgrad_max_stages() { return kWgMaxStages; }

// Shared memory for `stages` stages of A (om x 128 output channels) and B (BN channels).
size_t wgrad_smem_bytes(bool f32, int BN, int stages, int om) {
    const size_t blk = static_cast<size_t>(wgrad_pixels_per_stage(f32)) * 128;
    const int cc = f32 ? 32 : 64;
    const size_t stage = (om * 128 / cc + BN / cc) * blk * (f32 ? 3 : 1);
    return 1024 /* alignment slack */ + kWgHeader + static_cast<size_t>(stages) * stage;
}

cudaError_t launch_wgrad(const WgradParams &p, bool f32, int grid, size_t smem, cudaStream_t stream) {
    if (p.stages < 2 || p.stages > kWgMaxStages || (p.om != 1 && p.om != 2) || (f32 && p.om != 1) ||
        (p.om == 2 && (p.BN > 256 || 2 * p.BN > static_cast<int>(p.tmem_cols))))
        return cudaErrorInvalidValue;
    if (f32) return wgrad_launch_t<true, false>(p, grid, smem, stream);
    return p.om == 2 ? wgrad_launch_t<false, true>(p, grid, smem, stream) : wgrad_launch_t<false, false>(p, grid, smem, stream);
}

}  // namespace conv2d_b200
