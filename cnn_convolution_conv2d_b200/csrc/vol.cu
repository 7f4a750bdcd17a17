// vol.cu -- the 3-D convolution (pwwt.cn/news/6111401 §5.1: a filter of Kd x Kh x Kw
// taps over a (D, H, W) volume) as an implicit matrix product that loads each input
// depth slice once for all the depth taps that read it.
//
// In the implicit product of igemm.cu every filter tap re-reads the input through its
// own im2col box: Kd*Kh*Kw boxes of 128 voxels x 128 bytes per output tile.  With 64 input
// channels that is one 128-byte row per voxel and tap, and the rate at which an SM's TMA
// engine brings in im2col rows (about 5.4 cycles per row, measured) bounds the layer:
// the video layer takes the same ~213 us with 64 or 128 output channels.  Here a unit of
// work is J output depth slices (od0 .. od0 + J - 1) of one 128-voxel tile of a depth
// slice (Ho*Wo voxels; tiles start on slice boundaries, the last tile of a slice is
// partial).  At stride 1 and unit dilation, output slice od0 + j read through depth tap kd
// sees input slice od0 + j + kd - pad: with s = j + kd, one im2col box per (s, kh, kw)
// serves every (j, kd) pair on that diagonal, so a unit loads (J + Kd - 1)*Kh*Kw boxes
// instead of J*Kd*Kh*Kw.  The accumulators of the J slices sit in tensor memory in
// descending j order, so the pairs of one box -- j = s - kd for consecutive kd -- are
// consecutive column blocks, and with the weights of one (kh, kw) staged kd-major they
// are one product of N = (number of kd) x C_out.  Each box is addressed through an output
// slice that exists (od0 + j < Do): an im2col box must start at an output position
// inside the tensor map's bounding box.
//
// One CTA per SM (M = 128 voxels per product), bf16, C_in = 64 (one 128-byte swizzled
// channel row per voxel), groups = 1, channels-last output stored through 64-byte-swizzled
// shared-memory blocks by TMA.
//   warp 0     : loads: per (kh, kw) the Kd weight tiles into one of two slots, then one
//                im2col box per (input slice, kh, kw) into the stage ring;
//   warp 1     : tensor-memory allocation; one thread issues the products;
//   warps 2..9 : epilogue, two warps per tensor-memory lane quarter (halves of the
//                columns), J accumulators per unit.
// Every wait is bounded (ptx.cuh).
#include <cuda_bf16.h>

#include "common.cuh"
#include "ptx.cuh"

namespace conv2d_b200 {
namespace {

using namespace ptx;

constexpr int kVRows = 128;                 // voxels per tile (M)
constexpr int kVRowBytes = 128;             // one voxel's 64 bf16 channels
constexpr int kVAStage = kVRows * kVRowBytes;
constexpr int kVMaxStages = 8;
constexpr int kVMaxJ = 8;
constexpr int kVHeader = 1024;
constexpr int kVThreads = 320;
constexpr int kVEpiWarp0 = 2;
constexpr int kVEpiWarps = 8;
constexpr int kVStageBuf = 32 * 64;         // one 32 x 32 bf16 output block
constexpr int kVYStage = kVEpiWarps * 2 * kVStageBuf;

struct VolShared {
    uint64_t full[kVMaxStages];
    uint64_t empty[kVMaxStages];
    uint64_t b_full[2];
    uint64_t b_empty[2];
    uint64_t acc_full[2];
    uint64_t acc_empty[2];
    uint64_t drain;
    uint32_t tmem_base;
    int abort;
};
static_assert(sizeof(VolShared) <= kVHeader, "header too small");

struct VolUnit {
    int n, od0, v0;   // image, first output depth slice, first voxel of the tile in its slice
};

__device__ __forceinline__ VolUnit vol_decode(const VolParams &p, int u) {
    VolUnit t;
    const int k = u % p.n_k;
    const int r = u / p.n_k;
    const int b = r % p.n_odb;
    t.n = r / p.n_odb;
    t.od0 = b * p.J;
    t.v0 = k * kVRows;
    return t;
}

__device__ __forceinline__ void vol_wait_quiet(uint64_t *bar, uint32_t parity, uint64_t limit_ns) {
    const uint64_t start = globaltimer_ns();
    while (!mbar_try_wait(bar, parity)) {
        if (globaltimer_ns() - start > limit_ns) return;
    }
}

__global__ void __launch_bounds__(kVThreads, 1) vol_reuse_kernel(const __grid_constant__ VolParams p) {
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_addr = smem_addr(smem_raw);
    uint8_t *base = smem_raw + (((raw_addr + 1023u) & ~1023u) - raw_addr);
    VolShared &sb = *reinterpret_cast<VolShared *>(base);
    const int BN = p.BN;
    const uint32_t tap_bytes = static_cast<uint32_t>(BN) * kVRowBytes;  // one tap's weight tile
    const uint32_t slot_bytes = static_cast<uint32_t>(p.Kd) * tap_bytes;  // the Kd taps of one (kh, kw)
    uint8_t *bslots = base + kVHeader;
    uint8_t *ring = bslots + 2 * slot_bytes;
    uint8_t *ystage = ring + p.stages * kVAStage;

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int khkw = p.Kh * p.Kw;

    if (threadIdx.x == 0) {
        for (int s = 0; s < p.stages; ++s) {
            mbar_init(&sb.full[s], 1);
            mbar_init(&sb.empty[s], 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&sb.b_full[i], 1);
            mbar_init(&sb.b_empty[i], 1);
            mbar_init(&sb.acc_full[i], 1);
            mbar_init(&sb.acc_empty[i], kVEpiWarps);
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
        // ------------------------------------------------------------- loads ---
        if (lane == 0) {
            prefetch_tensormap(&p.tmap_a);
            prefetch_tensormap(&p.tmap_b);
            int stage = 0, slot = 0;
            uint32_t phase = 0, bphase = 0;
            long long loads_issued = 0, b_issued = 0;
            bool ok = true;
            for (int u = blockIdx.x; ok && u < p.units; u += gridDim.x) {
                const VolUnit t = vol_decode(p, u);
                const int oh = t.v0 / p.Wo, ow = t.v0 - (t.v0 / p.Wo) * p.Wo;
                // the unit's input slices: those its existing output slices read
                const int jmax = min(p.J, p.Do - t.od0);
                const int nslices = jmax + p.Kd - 1;
                for (int g = 0; g < khkw && ok; ++g) {
                    const int kh = g / p.Kw, kw = g - (g / p.Kw) * p.Kw;
                    // the Kd weight tiles of (kh, kw), kd-major
                    if (!mbar_wait(&sb.b_empty[slot], bphase ^ 1u, wd, kDevTimeoutEmpty)) {
                        ok = false;
                        break;
                    }
                    if (!p.starve) {
                        mbar_arrive_expect_tx(&sb.b_full[slot], slot_bytes);
                        for (int kd = 0; kd < p.Kd; ++kd)
                            tma_load_3d(bslots + slot * slot_bytes + kd * tap_bytes, &p.tmap_b, &sb.b_full[slot],
                                        ((kd * p.Kh + kh) * p.Kw + kw) * 64, 0, 0);
                        ++b_issued;
                    }
                    if (++slot == 2) {
                        slot = 0;
                        bphase ^= 1u;
                    }
                    for (int s = 0; s < nslices; ++s) {
                        // any (j, kd) with j + kd = s names the same input slice: address it
                        // through an existing output slice j
                        const int j = s - (p.Kd - 1) > 0 ? s - (p.Kd - 1) : 0;   // j <= jmax - 1
                        const int kd = s - j;                                  // 0 <= kd < Kd
                        if (!mbar_wait(&sb.empty[stage], phase ^ 1u, wd, kDevTimeoutEmpty)) {
                            ok = false;
                            break;
                        }
                        if (!p.starve) {
                            mbar_arrive_expect_tx(&sb.full[stage], kVAStage);
                            tma_load_im2col_5d(ring + stage * kVAStage, &p.tmap_a, &sb.full[stage], 0,
                                               ow - p.pad_w, oh - p.pad, t.od0 + j - p.pad, t.n,
                                               static_cast<uint16_t>(kw), static_cast<uint16_t>(kh),
                                               static_cast<uint16_t>(kd));
                            ++loads_issued;
                        }
                        if (++stage == p.stages) {
                            stage = 0;
                            phase ^= 1u;
                        }
                    }
                }
            }
            if (*wd.abort) {
                // let the copies still in flight land before the CTA goes away
                const long long first = loads_issued > p.stages ? loads_issued - p.stages : 0;
                for (long long i = first; i < loads_issued; ++i)
                    vol_wait_quiet(&sb.full[i % p.stages], static_cast<uint32_t>((i / p.stages) & 1), wd.timeout_ns);
                const long long bfirst = b_issued > 2 ? b_issued - 2 : 0;
                for (long long i = bfirst; i < b_issued; ++i)
                    vol_wait_quiet(&sb.b_full[i % 2], static_cast<uint32_t>((i / 2) & 1), wd.timeout_ns);
            }
        }
    } else if (warp == 1) {
        // ---------------------------------------------------- tensor-core issue ---
        if (lane == 0) {
            const int max_blocks = 256 / BN;               // kd blocks one product may cover
            int stage = 0, slot = 0;
            uint32_t phase = 0, bphase = 0;
            int abuf = 0;
            uint32_t aphase = 0;
            bool ok = true;
            for (int u = blockIdx.x; ok && u < p.units; u += gridDim.x) {
                const VolUnit t = vol_decode(p, u);
                if (!mbar_wait(&sb.acc_empty[abuf], aphase ^ 1u, wd, kDevTimeoutAccEmpty)) {
                    ok = false;
                    break;
                }
                tc_fence_after_sync();
                const int jmax = min(p.J, p.Do - t.od0);          // output slices of this unit
                const int nslices = jmax + p.Kd - 1;               // as the loads
                // accumulator of slice j: columns [(J - 1 - j)*BN, + BN) of this buffer
                const uint32_t acc0 = tmem_base + static_cast<uint32_t>(abuf * p.J * BN);
                for (int g = 0; g < khkw && ok; ++g) {
                    if (!mbar_wait(&sb.b_full[slot], bphase, wd, kDevTimeoutFull)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after_sync();
                    const uint32_t b_addr = smem_addr(bslots + slot * slot_bytes);
                    for (int s = 0; s < nslices; ++s) {
                        if (!mbar_wait(&sb.full[stage], phase, wd, kDevTimeoutFull)) {
                            ok = false;
                            break;
                        }
                        tc_fence_after_sync();
                        const uint32_t a_addr = smem_addr(ring + stage * kVAStage);
                        // depth taps whose output slice j = s - kd exists
                        const int kd_lo = s - (jmax - 1) > 0 ? s - (jmax - 1) : 0;
                        const int kd_hi = s < p.Kd - 1 ? s : p.Kd - 1;
                        for (int k0 = kd_lo; k0 <= kd_hi;) {
                            // the kd = 0 block of the first (kh, kw) starts its accumulator
                            // (the other blocks of that product were started at an earlier s)
                            const bool first = g == 0 && k0 == 0;
                            int k1 = first ? 0 : kd_hi;
                            if (k1 - k0 + 1 > max_blocks) k1 = k0 + max_blocks - 1;
                            const int nb = k1 - k0 + 1;
                            const uint32_t idesc = instr_desc(1u, kVRows, static_cast<uint32_t>(nb * BN));
                            const uint32_t d_tmem = acc0 + static_cast<uint32_t>((p.J - 1 - (s - k0)) * BN);
                            const uint32_t b0 = b_addr + static_cast<uint32_t>(k0) * tap_bytes;
#pragma unroll
                            for (int q = 0; q < 4; ++q)  // 64 channels = 4 x 16
                                mma_bf16(d_tmem, smem_desc(a_addr + q * 32, 16, 1024, kSw128),
                                         smem_desc(b0 + q * 32, 16, 1024, kSw128), idesc,
                                         (first && q == 0) ? 0u : 1u);
                            k0 = k1 + 1;
                        }
                        mma_commit(&sb.empty[stage]);
                        if (++stage == p.stages) {
                            stage = 0;
                            phase ^= 1u;
                        }
                    }
                    if (!ok) break;
                    mma_commit(&sb.b_empty[slot]);
                    if (++slot == 2) {
                        slot = 0;
                        bphase ^= 1u;
                    }
                }
                if (!ok) break;
                mma_commit(&sb.acc_full[abuf]);
                if (++abuf == p.nacc) {  // one or two accumulator sets
                    abuf = 0;
                    aphase ^= 1u;
                }
            }
            if (!ok || *wd.abort) {
                mma_commit(&sb.drain);
                vol_wait_quiet(&sb.drain, 0, wd.timeout_ns);
            }
        }
        __syncwarp();
    } else {
        // ------------------------------------------------------------ epilogue ---
        // Warp e drains lane quarter (warp % 4) and columns [cspan*(e/4) ... ) of each of
        // the unit's accumulators; every 32 x 32 block goes out by one TMA store (rows are
        // voxels, all inside one depth slice: Ho*Wo is a multiple of 32).
        const int e = warp - kVEpiWarp0;
        const int quarter = warp & 3;
        const int cspan = ((BN / 2 + 31) & ~31);
        const int c_lo = min(BN, (e >> 2) * cspan), c_hi = min(BN, c_lo + cspan);
        const uint32_t lane_base = static_cast<uint32_t>(quarter * 32) << 16;
        int abuf = 0;
        uint32_t aphase = 0;
        int sbi = 0;
        for (int u = blockIdx.x; u < p.units; u += gridDim.x) {
            const VolUnit t = vol_decode(p, u);
            const bool ok = mbar_wait(&sb.acc_full[abuf], aphase, wd, kDevTimeoutAccFull);
            if (!__all_sync(0xffffffffu, ok)) break;
            tc_fence_after_sync();
            const int jmax = min(p.J, p.Do - t.od0);
            const int vrow = t.v0 + quarter * 32;                 // first voxel of this warp's block
            const bool rows_in = vrow < p.HoWo2;
            for (int j = 0; j < jmax && rows_in; ++j) {
                const uint32_t taddr = tmem_base + lane_base +
                                       static_cast<uint32_t>((abuf * p.J + (p.J - 1 - j)) * BN);
                const int mrow0 = (t.n * p.Do + t.od0 + j) * p.HoWo2 + vrow;
                for (int c = c_lo; c < c_hi; c += 32) {
                    uint32_t r[2][16];
                    tmem_ld_x16(taddr + static_cast<uint32_t>(c), r[0]);
                    tmem_ld_x16(taddr + static_cast<uint32_t>(c + 16), r[1]);
                    tmem_ld_wait();
                    float bv[32];
                    if (p.bias) {
                        const uint4 *b4 = reinterpret_cast<const uint4 *>(static_cast<const __nv_bfloat16 *>(p.bias) + c);
#pragma unroll
                        for (int q = 0; q < 4; ++q) {
                            const uint4 w = __ldg(b4 + q);
                            const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
                            for (int h = 0; h < 4; ++h) {
                                bv[8 * q + 2 * h] = __uint_as_float(ws[h] << 16);
                                bv[8 * q + 2 * h + 1] = __uint_as_float(ws[h] & 0xFFFF0000u);
                            }
                        }
                    } else {
#pragma unroll
                        for (int i = 0; i < 32; ++i) bv[i] = 0.f;
                    }
                    uint32_t pk[16];
#pragma unroll
                    for (int i = 0; i < 16; ++i) {
                        const float v0 = __uint_as_float(r[(2 * i) >> 4][(2 * i) & 15]) + bv[2 * i];
                        const float v1 = __uint_as_float(r[(2 * i + 1) >> 4][(2 * i + 1) & 15]) + bv[2 * i + 1];
                        __nv_bfloat162 h = __floats2bfloat162_rn(v0, v1);
                        pk[i] = *reinterpret_cast<uint32_t *>(&h);
                    }
                    if (lane == 0) bulk_wait_group_read<1>();  // this buffer's previous store has read it
                    __syncwarp();
                    // 64-byte swizzle: 16-byte chunk q of row r goes to chunk q ^ ((r >> 1) & 3)
                    uint8_t *buf = ystage + (e * 2 + sbi) * kVStageBuf;
#pragma unroll
                    for (int q = 0; q < 4; ++q)
                        *reinterpret_cast<uint4 *>(buf + lane * 64 + ((q ^ ((lane >> 1) & 3)) * 16)) =
                            make_uint4(pk[4 * q], pk[4 * q + 1], pk[4 * q + 2], pk[4 * q + 3]);
                    fence_proxy_async_smem();
                    __syncwarp();
                    if (lane == 0) {
                        tma_store_2d(&p.tmap_y, buf, c, mrow0);
                        bulk_commit_group();
                    }
                    sbi ^= 1;
                }
            }
            tc_fence_before_sync();
            __syncwarp();
            if (lane == 0) mbar_arrive(&sb.acc_empty[abuf]);
            if (++abuf == p.nacc) {
                abuf = 0;
                aphase ^= 1u;
            }
        }
        if (lane == 0) bulk_wait_group_all();  // stores done before exit
    }

    tc_fence_before_sync();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after_sync();
        tmem_dealloc(tmem_base, p.tmem_cols);
    }
}

}  // namespace

size_t vol_reuse_smem_bytes(int Kd, int BN, int stages) {
    return 1024 /* alignment slack */ + kVHeader + 2 * static_cast<size_t>(Kd) * BN * kVRowBytes +
           static_cast<size_t>(stages) * kVAStage + kVYStage;
}

int vol_reuse_max_stages() { return kVMaxStages; }
int vol_reuse_max_j() { return kVMaxJ; }

cudaError_t launch_vol_reuse(const VolParams &p, int grid, size_t smem, cudaStream_t stream) {
    if (p.stages < 2 || p.stages > kVMaxStages || p.J < 1 || p.J > kVMaxJ || p.BN % 32 != 0 || p.BN > 256 ||
        p.HoWo2 % 32 != 0 || p.HoWo2 < kVRows || (p.nacc != 1 && p.nacc != 2) ||
        p.nacc * p.J * p.BN > static_cast<int>(p.tmem_cols) ||
        p.Kd < 1 || p.Kh < 1 || p.Kw < 1 || p.taps != p.Kd * p.Kh * p.Kw)
        return cudaErrorInvalidValue;
    cudaError_t e = cudaFuncSetAttribute(vol_reuse_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    vol_reuse_kernel<<<grid, kVThreads, smem, stream>>>(p);
    return cudaGetLastError();
}

}  // namespace conv2d_b200
