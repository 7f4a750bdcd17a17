// pw.cu -- the pointwise (1x1, stride 1, no padding) convolution with its weights resident
// in shared memory.
//
// A 1x1 filter makes the convolution a plain channel matrix product ("PyTorch高维张量乘法与
// conv2d/conv3d维度语义解析" §1.2; the im2col/GEMM tutorial, zskr.cn/news/1820658, §4.2):
// the channels-last input x (M = N*H*W rows of C_in) is itself X_col, and y = X_col W^T.
// With a short reduction (C_in <= 256) every 256-row tile of the implicit GEMM in igemm.cu
// re-loads its whole weight tile (256 output channels x C_in) next to its A rows: half of
// the 128-byte rows the TMA engines bring in are weights, and that row rate is what bounds
// the layer before its output writes do.  Here each two-CTA cluster keeps one 256-column
// tile of W^T resident (each CTA its 128 columns, loaded once) and streams only the A rows
// of the row tiles it owns; the clusters are split evenly over the column tiles.
//
// CTA pairs on SM pairs (cta_group::2, M = 256 rows, N = 256 columns), bf16 operands, per
// group C_in a multiple of 64 up to 256 and C_out a multiple of 256; the clusters are split
// evenly over (group, column tile).  Output through swizzled shared-memory blocks and TMA
// stores: bf16 channels-last with the bias added in fp32, or the raw fp32 sums (the
// Winograd path's channel products, finished by its output transform).  fp32 layers stay on
// the general kernel: their three-product tf32 split needs the weights' low parts resident
// too, which does not fit beside the input ring.
//   warp 0     : loads: the resident weight planes once, then one A plane per stage;
//   warp 1     : tensor-memory allocation; the even CTA issues the products;
//   warps 2..9 : epilogue, two warps per tensor-memory lane quarter (halves of the columns).
// Every wait is bounded (ptx.cuh).
#include <cuda_bf16.h>

#include "common.cuh"
#include "ptx.cuh"

namespace conv2d_b200 {
namespace {

using namespace ptx;

constexpr int kPRows = 128;                 // A rows per CTA per tile
constexpr int kPPlane = 128;                // bytes of one 64-channel plane row
constexpr int kPAStage = kPRows * kPPlane;
constexpr int kPMaxStages = 8;
constexpr int kPMaxPlanes = 4;              // 128-byte planes: C_in <= 256
constexpr int kPHeader = 1024;
constexpr int kPThreads = 320;
constexpr int kPEpiWarp0 = 2;
constexpr int kPEpiWarps = 8;
// one output block of 32 rows x 128 bytes (64 bf16 or 32 fp32 columns): whole 128-byte
// lines of y per row; one or two staging buffers per epilogue warp
constexpr int kPStageBuf = 32 * 128;

struct PwShared {
    uint64_t full[kPMaxStages];
    uint64_t empty[kPMaxStages];
    uint64_t acc_full[2];
    uint64_t acc_empty[2];
    uint64_t b_ready;
    uint64_t drain;
    uint32_t tmem_base;
    int abort;
};
static_assert(sizeof(PwShared) <= kPHeader, "header too small");

__device__ __forceinline__ void pw_wait_quiet(uint64_t *bar, uint32_t parity, uint64_t limit_ns) {
    const uint64_t start = globaltimer_ns();
    while (!mbar_try_wait(bar, parity)) {
        if (globaltimer_ns() - start > limit_ns) return;
    }
}

template <bool kOutF32>
__global__ void __launch_bounds__(kPThreads, 1) pw_kernel(const __grid_constant__ PwParams p) {
    constexpr int kBW = kOutF32 ? 32 : 64;  // columns per output block
    constexpr int kPlaneElems = 64;  // channels in one 128-byte plane row
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_addr = smem_addr(smem_raw);
    uint8_t *base = smem_raw + (((raw_addr + 1023u) & ~1023u) - raw_addr);
    PwShared &sb = *reinterpret_cast<PwShared *>(base);
    const int BN = p.BN;
    const int BNl = BN / 2;                                   // weight columns resident per CTA
    const uint32_t plane_bytes = static_cast<uint32_t>(BNl) * kPPlane;
    uint8_t *bres = base + kPHeader;                          // resident weights: [plane][BNl][128 B]
    uint8_t *ring = bres + static_cast<uint32_t>(p.nk) * plane_bytes;
    uint8_t *ystage = ring + p.stages * kPAStage;                  // 1024-aligned: swizzled blocks

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank();
    // cluster c owns (group, column tile) c % (groups * n_ntiles) and row tiles
    // c / (groups * n_ntiles) + i * cpn
    const int cl = static_cast<int>(blockIdx.x >> 1);
    const int gn = cl % (p.groups * p.n_ntiles);
    const int g = gn / p.n_ntiles, ntile = gn - (gn / p.n_ntiles) * p.n_ntiles;
    const int mt0 = cl / (p.groups * p.n_ntiles);

    if (threadIdx.x == 0) {
        for (int s = 0; s < p.stages; ++s) {
            mbar_init(&sb.full[s], 1);
            mbar_init(&sb.empty[s], 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&sb.acc_full[i], 1);
            mbar_init(&sb.acc_empty[i], 2 * kPEpiWarps);
        }
        mbar_init(&sb.b_ready, 1);
        mbar_init(&sb.drain, 1);
        sb.abort = 0;
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc_pair(&sb.tmem_base, p.tmem_cols);
        tmem_relinquish_pair();
    }
    tc_fence_before_sync();
    __syncthreads();
    cluster_sync();  // the peer's barriers exist before anyone signals them
    tc_fence_after_sync();
    const uint32_t tmem_base = sb.tmem_base;
    const uint32_t full0 = mapa_shared(smem_addr(&sb.full[0]), 0u);
    const uint32_t acc_empty0 = mapa_shared(smem_addr(&sb.acc_empty[0]), 0u);
    const uint32_t bready0 = mapa_shared(smem_addr(&sb.b_ready), 0u);

    Watchdog wd;
    wd.abort = &sb.abort;
    wd.status = p.status;
    wd.timeout_ns = static_cast<uint64_t>(p.timeout_ns);

    if (warp == 0) {
        // ------------------------------------------------------------- loads ---
        if (lane == 0) {
            prefetch_tensormap(&p.tmap_a);
            prefetch_tensormap(&p.tmap_b);
            bool b_issued = false;
            if (!p.starve) {
                // this CTA's half of the column tile, every plane of the reduction, once;
                // both CTAs' copies count on the even CTA's barrier (armed there for both)
                if (rank == 0) mbar_arrive_expect_tx(&sb.b_ready, 2u * static_cast<uint32_t>(p.nk) * plane_bytes);
                for (int kp = 0; kp < p.nk; ++kp)
                    tma_load_3d_pair(bres + kp * plane_bytes, &p.tmap_b, bready0, kp * kPlaneElems,
                                     ntile * BN + static_cast<int>(rank) * BNl, g);
                b_issued = true;
            }
            int stage = 0;
            uint32_t phase = 0;
            long long loads_issued = 0;
            bool ok = true;
            for (int mt = mt0; ok && mt < p.m_tiles; mt += p.cpn) {
                // this CTA's 128 rows; the odd CTA past the last row reloads the last full
                // 128 rows (its results are never stored)
                int m0 = mt * 2 * kPRows + static_cast<int>(rank) * kPRows;
                if (m0 >= p.M) m0 = ((p.M - 1) / kPRows) * kPRows;
                for (int kp = 0; kp < p.nk; ++kp) {
                    if (!mbar_wait(&sb.empty[stage], phase ^ 1u, wd, kDevTimeoutEmpty)) {
                        ok = false;
                        break;
                    }
                    if (!p.starve) {
                        if (rank == 0) mbar_arrive_expect_tx(&sb.full[stage], 2u * kPAStage);
                        tma_load_2d_pair(ring + stage * kPAStage, &p.tmap_a, full0 + 8u * static_cast<uint32_t>(stage),
                                         g * p.Kp + kp * kPlaneElems, m0);
                        ++loads_issued;
                    }
                    if (++stage == p.stages) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
            }
            if (!*wd.abort) {
                // wait until the products have released every slot, so that no commit
                // from the even CTA is still on its way to this CTA's barriers at exit
                for (int i = 0; i < p.stages; ++i) {
                    if (!mbar_wait(&sb.empty[stage], phase ^ 1u, wd, kDevTimeoutEmpty)) break;
                    if (++stage == p.stages) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
            }
            if (*wd.abort) {
                if (rank == 0) {
                    // every copy of either CTA counts on the even CTA's barriers: wait
                    // (bounded) for each armed phase not yet seen complete
                    const long long first = loads_issued > p.stages ? loads_issued - p.stages : 0;
                    for (long long i = first; i < loads_issued; ++i)
                        pw_wait_quiet(&sb.full[i % p.stages], static_cast<uint32_t>((i / p.stages) & 1),
                                      wd.timeout_ns);
                    if (b_issued) pw_wait_quiet(&sb.b_ready, 0, wd.timeout_ns);
                } else if (loads_issued > 0 || b_issued) {
                    // the odd CTA cannot observe its own copies: a fixed time to land
                    const uint64_t t0 = globaltimer_ns();
                    while (globaltimer_ns() - t0 < 200000u) {
                    }
                }
            }
        }
    } else if (warp == 1) {
        // ---------------------------------------------------- tensor-core issue ---
        if (lane == 0 && rank == 0) {
            const uint32_t idesc = instr_desc(1u, 2 * kPRows, static_cast<uint32_t>(BN));
            const uint32_t bres_addr = smem_addr(bres);
            bool ok = mbar_wait(&sb.b_ready, 0, wd, kDevTimeoutFull);
            int stage = 0;
            uint32_t phase = 0;
            int abuf = 0;
            uint32_t aphase = 0;
            for (int mt = mt0; ok && mt < p.m_tiles; mt += p.cpn) {
                if (!mbar_wait(&sb.acc_empty[abuf], aphase ^ 1u, wd, kDevTimeoutAccEmpty)) {
                    ok = false;
                    break;
                }
                tc_fence_after_sync();
                const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(abuf * BN);
                for (int kp = 0; kp < p.nk; ++kp) {
                    if (!mbar_wait(&sb.full[stage], phase, wd, kDevTimeoutFull)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after_sync();
                    const uint32_t a_addr = smem_addr(ring + stage * kPAStage);
                    const uint32_t b_addr = bres_addr + static_cast<uint32_t>(kp) * plane_bytes;
#pragma unroll
                    for (int q = 0; q < 4; ++q)  // 64 channels = 4 x 16
                        mma_bf16_pair(d_tmem, smem_desc(a_addr + q * 32, 16, 1024, kSw128),
                                      smem_desc(b_addr + q * 32, 16, 1024, kSw128), idesc,
                                      (kp == 0 && q == 0) ? 0u : 1u);
                    mma_commit_pair(&sb.empty[stage], 0x3);   // both CTAs' slots
                    if (++stage == p.stages) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
                if (!ok) break;
                mma_commit_pair(&sb.acc_full[abuf], 0x3);
                abuf ^= 1;
                if (abuf == 0) aphase ^= 1u;
            }
            if (!ok || *wd.abort) {
                mma_commit_pair(&sb.drain, 0x1);
                pw_wait_quiet(&sb.drain, 0, wd.timeout_ns);
            }
        }
        __syncwarp();
    } else {
        // ------------------------------------------------------------ epilogue ---
        // Warp e drains lane quarter (warp % 4) and columns [128*(e/4), + 128) of the
        // accumulator; every 32-row x 128-byte block goes out by one TMA store.
        const int e = warp - kPEpiWarp0;
        const int quarter = warp & 3;
        const int cspan = ((BN / 2 + 31) & ~31);
        const int c_lo = min(BN, (e >> 2) * cspan), c_hi = min(BN, c_lo + cspan);
        const uint32_t lane_base = static_cast<uint32_t>(quarter * 32) << 16;
        const int col0 = g * p.Cout_g + ntile * BN;
        int abuf = 0;
        uint32_t aphase = 0;
        int sbi = 0;
        for (int mt = mt0; mt < p.m_tiles; mt += p.cpn) {
            const bool ok = mbar_wait(&sb.acc_full[abuf], aphase, wd, kDevTimeoutAccFull);
            if (!__all_sync(0xffffffffu, ok)) break;
            tc_fence_after_sync();
            const int mrow0 = mt * 2 * kPRows + static_cast<int>(rank) * kPRows + quarter * 32;
            const uint32_t taddr = tmem_base + lane_base + static_cast<uint32_t>(abuf * BN);
            for (int c = c_lo; c < c_hi; c += kBW) {
                uint32_t r[kBW / 16][16];
#pragma unroll
                for (int h = 0; h < kBW / 16; ++h) tmem_ld_x16(taddr + static_cast<uint32_t>(c + 16 * h), r[h]);
                tmem_ld_wait();
                if (c + kBW >= c_hi) {  // this warp's part of the accumulator is read
                    tc_fence_before_sync();
                    __syncwarp();
                    if (lane == 0) mbar_arrive_cluster(acc_empty0 + 8u * static_cast<uint32_t>(abuf));
                }
                if (mrow0 >= p.M) continue;
                if (lane == 0) {  // this buffer's previous store has read it
                    if (p.ybufs == 2)
                        bulk_wait_group_read<1>();
                    else
                        bulk_wait_group_read<0>();
                }
                __syncwarp();
                uint8_t *buf = ystage + (e * p.ybufs + sbi) * kPStageBuf;
                // 128-byte swizzle: 16-byte chunk q of row r goes to chunk q ^ (r & 7)
                if constexpr (kOutF32) {
#pragma unroll
                    for (int q = 0; q < 8; ++q)
                        *reinterpret_cast<uint4 *>(buf + lane * 128 + ((q ^ (lane & 7)) * 16)) =
                            make_uint4(r[q >> 2][4 * (q & 3)], r[q >> 2][4 * (q & 3) + 1], r[q >> 2][4 * (q & 3) + 2],
                                       r[q >> 2][4 * (q & 3) + 3]);
                } else {
                    // chunk q holds columns [8q, 8q + 8): + bias, one rounding to bf16
                    const uint4 *b4 = p.bias ? reinterpret_cast<const uint4 *>(
                                                   static_cast<const __nv_bfloat16 *>(p.bias) + col0 + c)
                                             : nullptr;
#pragma unroll
                    for (int q = 0; q < 8; ++q) {
                        uint32_t ws[4] = {0u, 0u, 0u, 0u};
                        if (b4) {
                            const uint4 w = __ldg(b4 + q);
                            ws[0] = w.x;
                            ws[1] = w.y;
                            ws[2] = w.z;
                            ws[3] = w.w;
                        }
                        uint32_t pk[4];
#pragma unroll
                        for (int i = 0; i < 4; ++i) {
                            const float v0 = __uint_as_float(r[q >> 1][(q & 1) * 8 + 2 * i]) + __uint_as_float(ws[i] << 16);
                            const float v1 = __uint_as_float(r[q >> 1][(q & 1) * 8 + 2 * i + 1]) +
                                             __uint_as_float(ws[i] & 0xFFFF0000u);
                            __nv_bfloat162 h = __floats2bfloat162_rn(v0, v1);
                            pk[i] = *reinterpret_cast<uint32_t *>(&h);
                        }
                        *reinterpret_cast<uint4 *>(buf + lane * 128 + ((q ^ (lane & 7)) * 16)) =
                            make_uint4(pk[0], pk[1], pk[2], pk[3]);
                    }
                }
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) {
                    tma_store_2d(&p.tmap_y, buf, col0 + c, mrow0);
                    bulk_commit_group();
                }
                sbi ^= p.ybufs - 1;
            }
            if (c_lo >= c_hi) {  // nothing to drain in this half: release at once
                tc_fence_before_sync();
                __syncwarp();
                if (lane == 0) mbar_arrive_cluster(acc_empty0 + 8u * static_cast<uint32_t>(abuf));
            }
            abuf ^= 1;
            if (abuf == 0) aphase ^= 1u;
        }
        if (lane == 0) bulk_wait_group_all();  // stores done before exit
    }

    tc_fence_before_sync();
    __syncthreads();
    cluster_sync();  // neither CTA leaves while the pair still works
    if (warp == 1) {
        tc_fence_after_sync();
        tmem_dealloc_pair(tmem_base, p.tmem_cols);
    }
}

}  // namespace

size_t pw_smem_bytes(int nk, int BN, int stages, bool out_f32, int ybufs) {
    return 1024 /* alignment slack */ + kPHeader + static_cast<size_t>(nk) * (BN / 2) * kPPlane +
           static_cast<size_t>(stages) * kPAStage + static_cast<size_t>(kPEpiWarps) * ybufs * kPStageBuf;
}

namespace {
using PwKernel = void (*)(PwParams);
PwKernel pw_kernel_for(bool out_f32) { return out_f32 ? pw_kernel<true> : pw_kernel<false>; }
}  // namespace

int pw_max_stages() { return kPMaxStages; }
int pw_max_planes() { return kPMaxPlanes; }

cudaError_t pw_max_clusters(size_t smem, bool out_f32, int *out) {
    *out = 0;
    const PwKernel kern = pw_kernel_for(out_f32);
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2);
    cfg.blockDim = dim3(kPThreads);
    cfg.dynamicSmemBytes = smem;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaOccupancyMaxActiveClusters(out, kern, &cfg);
}

cudaError_t launch_pw(const PwParams &p, size_t smem, cudaStream_t stream) {
    if (p.stages < 2 || p.stages > kPMaxStages || p.nk < 1 || p.nk > kPMaxPlanes || p.BN != 256 ||
        p.n_ntiles < 1 || p.groups < 1 || p.cpn < 1 || p.m_tiles < 1 || 2 * p.BN > static_cast<int>(p.tmem_cols) ||
        p.Kp < 64 * p.nk || p.Cout_g < p.BN * p.n_ntiles || (p.ybufs != 1 && p.ybufs != 2) ||
        (p.bias && p.out_f32))
        return cudaErrorInvalidValue;
    const PwKernel kern = pw_kernel_for(p.out_f32 != 0);
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(2 * p.cpn * p.n_ntiles * p.groups));
    cfg.blockDim = dim3(kPThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    e = cudaLaunchKernelEx(&cfg, kern, p);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

}  // namespace conv2d_b200
