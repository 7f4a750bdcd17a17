// gather_t.cu -- the few-channel first layer (bf16, NCHW in and out) as the transposed
// product: output channels on the tensor-memory lanes, output pixels along the columns.
//
// The first layer of an image network reads 3 colour channels ("PyTorch高维张量乘法与
// conv2d/conv3d维度语义解析" §6.3: channels-last brings nothing there) and writes many
// more; the im2col/GEMM tutorial (zskr.cn/news/1820658) §2.3 writes its product as
// Y = W_row @ X_col with W_row (C_out x C_in*Kh*Kw) on the left.  Computed that way round
// on the tensor cores, each accumulator lane holds one output channel and its columns
// are consecutive output pixels of one output row, so the epilogue stores each channel's
// row with 16-byte vector stores straight into the NCHW output: no transposition, no
// staging, one bias per thread.  (The other few-channel kernel, gather.cu, has pixels on
// the lanes and must turn each tile channel-major before storing it.)
//
//   A (M = 128 x K): the weight image that conv2d_pack_weight wrote (C_out rows, K in the
//      row-vector order k = (c*Kh + kh)*8 + kw, 16-byte k chunks), rows C_out..127 zero,
//      resident in shared memory (one bulk copy);
//   B (N = Wo padded to 16, x K): the im2col rows of one output row, gathered by the
//      gather warps from input rows staged in shared memory by one TMA box load per tile
//      (all channels, the Kh rows the output row reads, with a zero margin on the left;
//      outside the image the box reads zeros: the padding), double-buffered;
//   D (tensor memory, fp32): lanes = output channels, columns = pixels, double-buffered.
//
//   gather warps 0..7 : thread t builds pixel row (t % 128), chunks of half (t / 128);
//   warp 8            : tensor-memory allocation, TMA loads of the staged input rows (two
//                       tiles ahead), tcgen05.mma from one thread;
//   warps 9..16       : epilogue, two warps per lane quarter (each half of the columns):
//                       tcgen05.ld, + bias, one rounding to bf16, 16-byte stores.
// Every wait is bounded (ptx.cuh).
#include <cuda_bf16.h>

#include "common.cuh"
#include "ptx.cuh"

namespace conv2d_b200 {
namespace {

using namespace ptx;

constexpr int kGtProd = 8;
constexpr int kGtMma = 8;
constexpr int kGtEpi = 8;
constexpr int kGtThreads = (kGtProd + 1 + kGtEpi) * 32;
constexpr int kGtHeader = 1024;
constexpr int kGtMaxChunks = 32;   // Kpad <= 256 bf16

struct GtShared {
    uint64_t halo_full[2];
    uint64_t b_full[2];
    uint64_t b_empty[2];
    uint64_t acc_full[2];
    uint64_t acc_empty[2];
    uint64_t a_ready;
    uint64_t drain;
    uint32_t tmem_base;
    int abort;
    int cwo[kGtMaxChunks];   // word offset of each chunk's staged row
};
static_assert(sizeof(GtShared) <= kGtHeader, "header too small");

__device__ __forceinline__ uint32_t gt_align1k(uint32_t v) { return (v + 1023u) & ~1023u; }

__device__ __forceinline__ void gt_wait_quiet(uint64_t *bar, uint32_t parity, uint64_t limit_ns) {
    const uint64_t start = globaltimer_ns();
    while (!mbar_try_wait(bar, parity)) {
        if (globaltimer_ns() - start > limit_ns) return;
    }
}

__global__ void __launch_bounds__(kGtThreads, 1) gather_t_kernel(const __grid_constant__ GatherParams p) {
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_addr = smem_addr(smem_raw);
    uint8_t *base = smem_raw + (((raw_addr + 1023u) & ~1023u) - raw_addr);
    GtShared &sb = *reinterpret_cast<GtShared *>(base);
    const int nchunks = p.Kpad / 8;
    const uint32_t sbo = static_cast<uint32_t>(nchunks) * 128u;  // one 8-row group of a K-major operand
    const int tpix = p.tpix;                                     // B rows (pixels), a multiple of 16
    uint8_t *a_sm = base + kGtHeader;
    const uint32_t a_bytes = 16u * sbo;                          // 128 rows
    uint8_t *b_sm = a_sm + gt_align1k(a_bytes);
    const uint32_t b_bytes = static_cast<uint32_t>(tpix / 8) * sbo;
    const uint32_t b_stride = gt_align1k(b_bytes);
    uint8_t *halo_sm = b_sm + 2 * b_stride;
    const uint32_t halo_bytes = static_cast<uint32_t>(p.C) * p.R * p.BW * 2u;
    const uint32_t halo_stride = gt_align1k(halo_bytes);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int i = 0; i < 2; ++i) {
            mbar_init(&sb.halo_full[i], 1);
            mbar_init(&sb.b_full[i], kGtProd);
            mbar_init(&sb.b_empty[i], 1);
            mbar_init(&sb.acc_full[i], 1);
            mbar_init(&sb.acc_empty[i], kGtEpi);
        }
        mbar_init(&sb.a_ready, 1);
        mbar_init(&sb.drain, 1);
        sb.abort = 0;
        fence_mbar_init();
    }
    // chunk j = c*Kh + kh reads staged row c*R + kh*d (word offsets; BW is even)
    for (int j = threadIdx.x; j < kGtMaxChunks; j += blockDim.x) {
        const int c = j / p.Kh, kh = j - (j / p.Kh) * p.Kh;
        sb.cwo[j] = j < p.C * p.Kh ? (c * p.R + kh * p.dilation) * (p.BW / 2) : -1;
    }
    // weight rows past the image's (C_out rounded up to 16) are zero: output channels
    // that do not exist come out as zeros and are not stored
    {
        const uint32_t img_bytes = static_cast<uint32_t>(p.BN / 8) * sbo;
        uint4 *z = reinterpret_cast<uint4 *>(a_sm + img_bytes);
        for (uint32_t i = threadIdx.x; i < (a_bytes - img_bytes) / 16u; i += blockDim.x) z[i] = make_uint4(0, 0, 0, 0);
        fence_proxy_async_smem();
    }
    if (warp == kGtMma) {
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

    if (warp < kGtProd) {
        // ------------------------------------------------------------- gather ---
        const int row = threadIdx.x & 127;          // pixel (B row) of this thread
        const int part = threadIdx.x >> 7;          // which half of the chunks
        const int half = ((nchunks + 1) / 2 + 1) & ~1;
        const int jb = part == 0 ? 0 : half, je = part == 0 ? min(half, nchunks) : nchunks;
        const bool active = row < p.Wo;             // rows past Wo feed columns never stored
        int li = 0;
        for (int t = blockIdx.x; t < p.n_mtiles; t += gridDim.x, ++li) {
            const int b = li & 1;
            const uint32_t ph = static_cast<uint32_t>(li >> 1) & 1u;
            const bool ok = mbar_wait(&sb.b_empty[b], ph ^ 1u, wd, kDevTimeoutEmpty) &&
                            mbar_wait(&sb.halo_full[b], ph, wd, kDevTimeoutFull);
            if (!__all_sync(0xffffffffu, ok)) break;
            if (active) {
                const uint32_t *h32 = reinterpret_cast<const uint32_t *>(halo_sm + b * halo_stride);
                const int e0 = row * p.stride - p.pad + p.ME;   // staged column of kw = 0
                const uint32_t *hrow = h32 + (e0 >> 1);
                const uint32_t sh = (e0 & 1) * 16u;
                uint8_t *dst = b_sm + b * b_stride + static_cast<uint32_t>(row >> 3) * sbo +
                               static_cast<uint32_t>(row & 7) * 16u;
#pragma unroll 4
                for (int j = jb; j < je; ++j) {
                    const int wo = sb.cwo[j];
                    uint4 v = make_uint4(0, 0, 0, 0);
                    if (wo >= 0) {
                        uint32_t w[5];
#pragma unroll
                        for (int i = 0; i < 5; ++i) w[i] = hrow[wo + i];
                        v.x = __funnelshift_r(w[0], w[1], sh);
                        v.y = __funnelshift_r(w[1], w[2], sh);
                        v.z = __funnelshift_r(w[2], w[3], sh);
                        v.w = __funnelshift_r(w[3], w[4], sh);
                    }
                    *reinterpret_cast<uint4 *>(dst + j * 128) = v;
                }
            }
            fence_proxy_async_smem();   // the tensor cores read these rows
            __syncwarp();
            if (lane == 0 && !p.starve) mbar_arrive(&sb.b_full[b]);
        }
    } else if (warp == kGtMma) {
        // ------------------------------------------- loads and tensor-core issue ---
        if (lane == 0) {
            const uint32_t idesc = instr_desc(1u, 128, static_cast<uint32_t>(tpix));
            const uint32_t a_addr = smem_addr(a_sm);
            const int ksteps = nchunks / 2;       // 32 bytes of k per instruction
            int issued[2] = {0, 0};
            auto issue_halo = [&](int t, int b) {
                const int img = t / p.Ho;
                const int oh = t - img * p.Ho;
                ++issued[b];
                mbar_arrive_expect_tx(&sb.halo_full[b], halo_bytes);
                tma_load_4d(halo_sm + b * halo_stride, &p.tmap_x, &sb.halo_full[b], -p.ME, oh * p.stride - p.pad,
                            0, img);
            };
            bool ok = true;
            if (!p.starve) {
                prefetch_tensormap(&p.tmap_x);
                for (int k = 0; k < 2; ++k)
                    if (blockIdx.x + k * static_cast<int>(gridDim.x) < p.n_mtiles) issue_halo(blockIdx.x + k * gridDim.x, k);
                const uint32_t img_bytes = static_cast<uint32_t>(p.BN / 8) * sbo;
                mbar_arrive_expect_tx(&sb.a_ready, img_bytes);
                bulk_load(a_sm, p.w_image, img_bytes, &sb.a_ready);
            }
            if (!mbar_wait(&sb.a_ready, 0, wd, kDevTimeoutFull)) ok = false;
            int li = 0;
            for (int t = blockIdx.x; ok && t < p.n_mtiles; t += gridDim.x, ++li) {
                const int b = li & 1;
                const uint32_t ph = static_cast<uint32_t>(li >> 1) & 1u;
                if (!mbar_wait(&sb.acc_empty[b], ph ^ 1u, wd, kDevTimeoutAccEmpty) ||
                    !mbar_wait(&sb.b_full[b], ph, wd, kDevTimeoutFull)) {
                    ok = false;
                    break;
                }
                tc_fence_after_sync();
                // the gather warps are done with halo buffer b: it takes tile t + 2
                const int t2 = t + 2 * static_cast<int>(gridDim.x);
                if (!p.starve && t2 < p.n_mtiles) issue_halo(t2, b);
                const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(b * tpix);
                const uint32_t b_addr = smem_addr(b_sm + b * b_stride);
                for (int ks = 0; ks < ksteps; ++ks) {
                    const uint32_t off = static_cast<uint32_t>(ks) * 256u;  // two 16-byte k chunks
                    mma_bf16(d_tmem, smem_desc(a_addr + off, 128, sbo, kSwNone),
                             smem_desc(b_addr + off, 128, sbo, kSwNone), idesc, ks > 0 ? 1u : 0u);
                }
                mma_commit(&sb.b_empty[b]);
                mma_commit(&sb.acc_full[b]);
            }
            if (!ok || *wd.abort) {
                mma_commit(&sb.drain);
                gt_wait_quiet(&sb.drain, 0, wd.timeout_ns);
                if (!p.starve) gt_wait_quiet(&sb.a_ready, 0, wd.timeout_ns);
                for (int b = 0; b < 2; ++b)  // let the staged-row loads still in flight land
                    if (issued[b] > 0)
                        gt_wait_quiet(&sb.halo_full[b], static_cast<uint32_t>(issued[b] - 1) & 1u, wd.timeout_ns);
            }
        }
        __syncwarp();
    } else {
        // ----------------------------------------------------------- epilogue ---
        const int e = warp - kGtMma - 1;            // 0..7
        const int quarter = warp & 3;               // tensor-memory lanes of this warp
        const int oc = quarter * 32 + lane;         // output channel of this thread
        const int cspan = ((p.Wo + 15) / 16) * 8;   // columns per half, a multiple of 8
        const int c_lo = (e >> 2) * cspan, c_hi = min(p.Wo, c_lo + cspan);
        const bool valid = oc < p.Cout;
        const float bv = (valid && p.bias)
                             ? __uint_as_float(static_cast<uint32_t>(static_cast<const unsigned short *>(p.bias)[oc]) << 16)
                             : 0.f;
        const uint32_t lane_base = static_cast<uint32_t>(quarter * 32) << 16;
        const bool any = __any_sync(0xffffffffu, valid) && c_lo < c_hi;
        int li = 0;
        for (int t = blockIdx.x; t < p.n_mtiles; t += gridDim.x, ++li) {
            const int b = li & 1;
            const uint32_t ph = static_cast<uint32_t>(li >> 1) & 1u;
            const bool ok = mbar_wait(&sb.acc_full[b], ph, wd, kDevTimeoutAccFull);
            if (!__all_sync(0xffffffffu, ok)) break;
            tc_fence_after_sync();
            if (any) {
                const int img = t / p.Ho;
                const int oh = t - img * p.Ho;
                __nv_bfloat16 *yrow = static_cast<__nv_bfloat16 *>(p.y) +
                                      ((static_cast<size_t>(img) * p.Cout + (valid ? oc : 0)) * p.Ho + oh) * p.Wo;
                const uint32_t taddr = tmem_base + lane_base + static_cast<uint32_t>(b * tpix);
                // eight columns (pixels) per load and per 16-byte store; c_hi <= Wo <= tpix,
                // so no load leaves this accumulator's columns
                for (int c = c_lo; c < c_hi; c += 8) {
                    uint32_t r[8];
                    tmem_ld_x8(taddr + static_cast<uint32_t>(c), r);
                    tmem_ld_wait();
                    if (valid) {
                        uint32_t pk[4];
#pragma unroll
                        for (int i = 0; i < 4; ++i) {
                            __nv_bfloat162 v = __floats2bfloat162_rn(__uint_as_float(r[2 * i]) + bv,
                                                                     __uint_as_float(r[2 * i + 1]) + bv);
                            pk[i] = *reinterpret_cast<uint32_t *>(&v);
                        }
                        *reinterpret_cast<uint4 *>(yrow + c) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
                    }
                }
            }
            tc_fence_before_sync();
            __syncwarp();
            if (lane == 0) mbar_arrive(&sb.acc_empty[b]);
        }
    }

    tc_fence_before_sync();
    __syncthreads();
    if (warp == kGtMma) {
        tc_fence_after_sync();
        tmem_dealloc(tmem_base, p.tmem_cols);
    }
}

}  // namespace

size_t gather_t_smem_bytes(int Kpad, int tpix, size_t halo_bytes) {
    auto a1k = [](size_t v) { return (v + 1023) / 1024 * 1024; };
    const size_t sbo = static_cast<size_t>(Kpad / 8) * 128;
    return 1024 /* alignment slack */ + kGtHeader + a1k(16 * sbo) + 2 * a1k(static_cast<size_t>(tpix / 8) * sbo) +
           2 * a1k(halo_bytes);
}

cudaError_t launch_gather_t(const GatherParams &p, int grid, size_t smem, cudaStream_t s) {
    if (p.Kpad > 8 * kGtMaxChunks || p.Kpad % 16 != 0 || p.tpix % 16 != 0 || p.tpix > 256 || p.Wo > 256 ||
        p.Wo % 8 != 0 || p.Cout > 128 || p.BN > 128 || p.C * p.Kh > kGtMaxChunks || 2 * p.tpix > static_cast<int>(p.tmem_cols))
        return cudaErrorInvalidValue;
    cudaError_t e = cudaFuncSetAttribute(gather_t_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    gather_t_kernel<<<grid, kGtThreads, smem, s>>>(p);
    return cudaGetLastError();
}

}  // namespace conv2d_b200
