// igemm.cu -- the convolution forward pass as an implicit matrix product on the
// sm_100a tensor cores (tcgen05), never forming the im2col matrix in memory.
//
// The product is the one of the im2col/GEMM tutorial (zskr.cn/news/1820658) §2.3,
// Y = W_row @ X_col, computed transposed: rows are output pixels
// m = (n*Ho + oh)*Wo + ow (tcgen05 M = 128 per CTA), columns are the output channels
// of one group (tcgen05 N = BN), and the reduction runs over the filter taps
// (kh, kw) and the input channels of the group -- the "expand per tile, multiply,
// discard" scheme the "手撕 Conv2D" page (lpnh.cn/news/2493075) §4.1 mentions, with
// the expansion done by the tensor memory accelerator's im2col mode (or, for a 1x1
// filter at stride 1 without padding, by tiled loads of x, which is then X_col).
//
// Persistent and warp-specialised, one CTA per SM:
//   warp 0      : TMA producer -- per stage, one im2col load of 128 output pixels x
//                 CB bytes of channels per plane (filter-tap offsets kw*d, kh*d; reads
//                 outside the image return zero, which is the zero padding) and one
//                 tiled load of the weight rows x CB bytes per plane;
//   warp 1      : allocates tensor memory and issues tcgen05.mma from one thread,
//                 releasing each stage with tcgen05.commit;
//   warps 2..9  : (bf16) epilogue -- tcgen05.ld of the fp32 accumulator, + bias, round,
//                 store (channels-last through shared memory and TMA stores), two
//                 warps per tensor-memory lane quarter, each draining half the columns;
//   warps 2..5  : (fp32) epilogue, with warps 6..9 splitting every staged fp32 value v
//                 into tf32 parts hi = tf32(v), lo = tf32(v - hi) for three products.
// Two accumulators in tensor memory let the epilogue of one tile overlap the
// main loop of the next.  Every wait is bounded (see ptx.cuh).
//
// CTA pairs (kPair, bf16): the grid is launched in clusters of two CTAs on an SM pair.
// A unit of work is 256 output pixels; each CTA stages its own 128 rows of A and half
// of the BN weight rows, all loads count on the even CTA's full barrier, the even CTA
// issues M = 256 tcgen05.mma.cta_group::2 that read both CTAs' shared memory and write
// each CTA's 128 accumulator rows into its own tensor memory, and its commits release
// both CTAs' ring slots and accumulators by multicast arrive.  Both CTAs' epilogue
// warps hand the accumulator back on the even CTA's barrier.
#include <cuda_bf16.h>

#include "common.cuh"
#include "epilogue.cuh"
#include "ptx.cuh"

namespace conv2d_b200 {
namespace {

using namespace ptx;

constexpr int kBM = 128;                  // output pixels per tile
constexpr int kStageRowBytes = 128;       // reduction bytes per operand row per stage
constexpr int kAStageBytes = kBM * kStageRowBytes;
constexpr int kMaxStages = 8;
constexpr int kBarrierBlock = 1024;       // barriers + flags, ahead of the stage ring

constexpr int kProducerWarp = 0;
constexpr int kMmaWarp = 1;
constexpr int kEpiWarp0 = 2;
constexpr int kCvtWarp0 = 6;
constexpr int kMaxBNf32 = 128;            // widest fp32 tile: its accumulator row lives in registers
constexpr int kStageBufBytes = 32 * 64;   // tma_out: one 32-row x 32-column bf16 block
constexpr int kYStageBytes = 8 * 2 * kStageBufBytes;  // two buffers per epilogue warp

// bf16: warps 2..9 drain the accumulator (two per tensor-memory lane quarter, each
// taking half of the columns); fp32: warps 2..5 drain, warps 6..9 split operands.
template <bool kF32>
__host__ __device__ constexpr int epi_warps() { return kF32 ? 4 : 8; }
template <bool kF32>
__host__ __device__ constexpr int threads_for() { return 320; }

__host__ __device__ inline uint32_t stage_bytes(bool f32, int BN) {
    return static_cast<uint32_t>((kAStageBytes + BN * kStageRowBytes) * (f32 ? 2 : 1));
}

struct SharedBlock {  // lives at the start of the 1024-aligned dynamic shared memory
    uint64_t full[kMaxStages];
    uint64_t empty[kMaxStages];
    uint64_t converted[kMaxStages];
    uint64_t acc_full[2];
    uint64_t acc_empty[2];
    uint64_t drain;
    uint32_t tmem_base;
    int abort;
};
static_assert(sizeof(SharedBlock) <= kBarrierBlock, "barrier block too small");

__device__ __forceinline__ OutDesc out_desc(const IgemmParams &p) {
    OutDesc o;
    o.y = p.y;
    o.bias = p.bias;
    o.M = p.M;
    o.HoWo = p.HoWo;
    o.Cout = p.Cout;
    o.Cout_g = p.Cout_g;
    o.out_mode = p.out_mode;
    o.vec_ok = p.vec_ok;
    return o;
}

struct Unit {
    int mtile, g, ntile, split, k0, k1;
};

__device__ __forceinline__ Unit decode_unit(const IgemmParams &p, int u) {
    // 32-bit arithmetic, and no division where a factor is 1: this runs once per
    // tile on the issuing threads, where a 64-bit division costs about as much as
    // a stage of MMAs.
    Unit t;
    int r = u;
    t.split = 0;
    t.ntile = 0;
    t.g = 0;
    if (p.splits > 1) {
        const int q = r / p.splits;
        t.split = r - q * p.splits;
        r = q;
    }
    if (p.n_ntiles > 1) {
        const int q = r / p.n_ntiles;
        t.ntile = r - q * p.n_ntiles;
        r = q;
    }
    if (p.groups > 1) {
        const int q = r / p.groups;
        t.g = r - q * p.groups;
        r = q;
    }
    t.mtile = r;
    if (p.splits > 1) {
        t.k0 = (t.split * p.kstages) / p.splits;  // kstages * splits < 2^31 (checked by the host)
        t.k1 = ((t.split + 1) * p.kstages) / p.splits;
    } else {
        t.k0 = 0;
        t.k1 = p.kstages;
    }
    return t;
}

// Bounded wait that ignores the abort flag: used only while tearing down after an
// abort, to let copies already in flight land before the CTA exits.
__device__ __forceinline__ void wait_quiet(uint64_t *bar, uint32_t parity, uint64_t limit_ns) {
    const uint64_t start = globaltimer_ns();
    while (!mbar_try_wait(bar, parity)) {
        if (globaltimer_ns() - start > limit_ns) return;
    }
}

// ------------------------------------------------------------------ MMAs ---
// Issues the tensor-core instructions for one staged block of the reduction
// (128 bytes per operand row: kNP planes of kCB bytes).
// `BNl` is the number of B rows staged in this CTA (all BN columns, or half of
// them for a CTA pair, whose MMAs read the other half from the peer CTA).
template <bool kF32, int kCB, bool kPair>
__device__ __forceinline__ void mma_one(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                        uint32_t idesc, uint32_t acc) {
    if constexpr (kPair) {
        mma_bf16_pair(d_tmem, a_desc, b_desc, idesc, acc);
    } else if constexpr (kF32) {
        mma_tf32(d_tmem, a_desc, b_desc, idesc, acc);
    } else {
        mma_bf16(d_tmem, a_desc, b_desc, idesc, acc);
    }
}

template <bool kF32, int kCB, bool kPair>
__device__ __forceinline__ void issue_stage(uint32_t a, uint32_t b, uint32_t alo, uint32_t blo,
                                            int BNl, uint32_t d_tmem, uint32_t idesc,
                                            bool first) {
    static_assert(!(kF32 && kPair), "CTA pairs are bf16 only");
    constexpr int kNP = kStageRowBytes / kCB;
    const uint32_t a_plane = kBM * kCB;
    const uint32_t b_plane = static_cast<uint32_t>(BNl) * kCB;
    if constexpr (kCB >= 32) {
        constexpr uint32_t kSw = kCB == 128 ? kSw128 : (kCB == 64 ? kSw64 : kSw32);
        constexpr uint32_t kSbo = 8 * kCB;  // eight rows of one swizzle atom
#pragma unroll
        for (int j = 0; j < kNP; ++j) {
#pragma unroll
            for (int kk = 0; kk < kCB / 32; ++kk) {
                const uint32_t ao = j * a_plane + kk * 32;
                const uint32_t bo = j * b_plane + kk * 32;
                const uint32_t acc = (first && j == 0 && kk == 0) ? 0u : 1u;
                if constexpr (kF32) {
                    mma_tf32(d_tmem, smem_desc(alo + ao, 16, kSbo, kSw),
                             smem_desc(b + bo, 16, kSbo, kSw), idesc, acc);
                    mma_tf32(d_tmem, smem_desc(a + ao, 16, kSbo, kSw),
                             smem_desc(blo + bo, 16, kSbo, kSw), idesc, 1u);
                    mma_tf32(d_tmem, smem_desc(a + ao, 16, kSbo, kSw),
                             smem_desc(b + bo, 16, kSbo, kSw), idesc, 1u);
                } else {
                    mma_one<false, kCB, kPair>(d_tmem, smem_desc(a + ao, 16, kSbo, kSw),
                                               smem_desc(b + bo, 16, kSbo, kSw), idesc, acc);
                }
            }
        }
    } else {
        // 16-byte planes, no swizzle: core matrices of 8 rows x 16 bytes stacked every
        // 128 bytes (SBO); one instruction's 32-byte K slice spans two planes (LBO).
#pragma unroll
        for (int j = 0; j < kNP; j += 2) {
            const uint32_t acc = (first && j == 0) ? 0u : 1u;
            const uint32_t ao = j * a_plane, bo = j * b_plane;
            if constexpr (kF32) {
                mma_tf32(d_tmem, smem_desc(alo + ao, a_plane, 128, kSwNone),
                         smem_desc(b + bo, b_plane, 128, kSwNone), idesc, acc);
                mma_tf32(d_tmem, smem_desc(a + ao, a_plane, 128, kSwNone),
                         smem_desc(blo + bo, b_plane, 128, kSwNone), idesc, 1u);
                mma_tf32(d_tmem, smem_desc(a + ao, a_plane, 128, kSwNone),
                         smem_desc(b + bo, b_plane, 128, kSwNone), idesc, 1u);
            } else {
                mma_one<false, kCB, kPair>(d_tmem, smem_desc(a + ao, a_plane, 128, kSwNone),
                                           smem_desc(b + bo, b_plane, 128, kSwNone), idesc, acc);
            }
        }
    }
}

// ---------------------------------------------------------------- kernel ---
// kPair: launched in clusters of two CTAs on an SM pair; each unit of work is 256
// output pixels (128 per CTA) x BN channels, computed by M = 256 pair MMAs issued from
// the even CTA, with each CTA staging its own 128 rows of A and BN/2 rows of B.
// kVol (with kIm2col): the input is a 5-D channels-last volume (c, w, h, d, n), rows
// are output voxels and the filter taps run over (kd, kh, kw) -- the 3-D convolution.
template <bool kF32, int kCB, bool kIm2col, bool kPair, bool kVol = false>
__global__ void __launch_bounds__(threads_for<kF32>(), 1)
    igemm_kernel(const __grid_constant__ IgemmParams p) {
    static_assert(kIm2col || !kVol, "volumes are read through im2col-mode loads");
    static_assert(!(kF32 && kPair), "CTA pairs are bf16 only");
    constexpr int kElt = kF32 ? 4 : 2;
    constexpr int kCBe = kCB / kElt;              // channels (elements) per plane row
    constexpr int kNP = kStageRowBytes / kCB;     // planes per stage

    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_addr = smem_addr(smem_raw);
    uint8_t *base = smem_raw + (((raw_addr + 1023u) & ~1023u) - raw_addr);
    SharedBlock &sb = *reinterpret_cast<SharedBlock *>(base);
    uint8_t *ring = base + kBarrierBlock;

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int BN = p.BN;
    // CTA pairs: rank 0 issues the MMAs and owns the full / acc_empty barriers
    const uint32_t rank = kPair ? cluster_ctarank() : 0u;
    const int unit0 = kPair ? static_cast<int>(blockIdx.x >> 1) : static_cast<int>(blockIdx.x);
    const int ustep = kPair ? static_cast<int>(gridDim.x >> 1) : static_cast<int>(gridDim.x);
    constexpr int kUnitRows = kPair ? 2 * kBM : kBM;  // output pixels per unit of work
    const int row_off = static_cast<int>(rank) * kBM;  // this CTA's rows within a unit
    const int BNl = kPair ? BN / 2 : BN;               // B rows staged in this CTA
    const uint32_t sbytes = stage_bytes(kF32, BNl);
    const uint32_t b_off = kAStageBytes;
    const uint32_t alo_off = kAStageBytes + BNl * kStageRowBytes;
    const uint32_t blo_off = alo_off + kAStageBytes;
    const uint32_t tx_bytes = (kAStageBytes + BNl * kStageRowBytes) * (kPair ? 2u : 1u);

    if (threadIdx.x == 0) {
        for (int s = 0; s < p.stages; ++s) {
            mbar_init(&sb.full[s], 1);
            mbar_init(&sb.empty[s], 1);
            mbar_init(&sb.converted[s], 128);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&sb.acc_full[i], 1);
            mbar_init(&sb.acc_empty[i], epi_warps<kF32>() * (kPair ? 2 : 1));
        }
        mbar_init(&sb.drain, 1);
        sb.abort = 0;
        fence_mbar_init();
    }
    if (warp == kMmaWarp) {
        if constexpr (kPair) {
            tmem_alloc_pair(&sb.tmem_base, p.tmem_cols);
            tmem_relinquish_pair();
        } else {
            tmem_alloc(&sb.tmem_base, p.tmem_cols);
            tmem_relinquish();
        }
    }
    tc_fence_before_sync();
    __syncthreads();
    if constexpr (kPair) cluster_sync();  // the peer's barriers exist before anyone signals them
    tc_fence_after_sync();
    const uint32_t tmem_base = sb.tmem_base;
    // shared::cluster addresses of rank 0's full and acc_empty barriers
    const uint32_t full0 = kPair ? mapa_shared(smem_addr(&sb.full[0]), 0u) : 0u;
    const uint32_t acc_empty0 = kPair ? mapa_shared(smem_addr(&sb.acc_empty[0]), 0u) : 0u;

    Watchdog wd;
    wd.abort = &sb.abort;
    wd.status = p.status;
    wd.timeout_ns = static_cast<uint64_t>(p.timeout_ns);

    if (warp == kProducerWarp) {
        // ------------------------------------------------------ TMA producer ---
        if (lane == 0) {
            prefetch_tensormap(&p.tmap_a);
            prefetch_tensormap(&p.tmap_b);
            int stage = 0;
            uint32_t phase = 0;
            long long loads_issued = 0;
            bool ok = true;
            for (int u = unit0; ok && u < p.units; u += ustep) {
                const Unit t = decode_unit(p, u);
                // A rows of this CTA; the odd CTA of a pair past the last row tile
                // reloads that tile (its results are never stored)
                const int m0 = kPair ? min(t.mtile * kUnitRows + row_off, ((p.M - 1) / kBM) * kBM)
                                     : t.mtile * kBM;
                int img = 0, d0 = 0, h0 = 0, w0 = 0;
                if constexpr (kIm2col) {
                    img = m0 / p.HoWo;
                    int rem = m0 - img * p.HoWo;
                    if constexpr (kVol) {
                        const int od = rem / p.HoWo2;
                        rem -= od * p.HoWo2;
                        d0 = od * p.stride - p.pad;
                    }
                    const int oh = rem / p.Wo;
                    const int ow = rem - oh * p.Wo;
                    h0 = oh * p.stride - p.pad;
                    w0 = ow * p.stride_w - p.pad_w;
                }
                // Filter tap (kh, kw) and channel block of the next plane, stepped
                // along instead of divided out per plane; past the last plane (the
                // padding of the last stage, whose weights are zero) the tap stays at
                // the last one so that the load is still well formed.
                int cblk = 0, kd = 0, kh = 0, kw = 0, tap = 0;
                if constexpr (kIm2col) {
                    if (t.k0 > 0) {
                        const int plane0 = t.k0 * kNP;
                        tap = plane0 / p.nCB;
                        cblk = plane0 - tap * p.nCB;
                        int r = tap;
                        if constexpr (kVol) {
                            kd = r / (p.Kh * p.Kw);
                            r -= kd * p.Kh * p.Kw;
                        }
                        kh = r / p.Kw;
                        kw = r - kh * p.Kw;
                    }
                }
                for (int ks = t.k0; ks < t.k1; ++ks) {
                    if (!mbar_wait(&sb.empty[stage], phase ^ 1u, wd, kDevTimeoutEmpty)) {
                        ok = false;
                        break;
                    }
                    uint8_t *st = ring + static_cast<size_t>(stage) * sbytes;
                    if (!p.starve) {
                        // a pair's loads all count on rank 0's barrier, armed once for both
                        if (!kPair || rank == 0) mbar_arrive_expect_tx(&sb.full[stage], tx_bytes);
                        const uint32_t fbar = full0 + 8u * static_cast<uint32_t>(stage);
#pragma unroll
                        for (int j = 0; j < kNP; ++j) {
                            const int plane = ks * kNP + j;
                            const int kelem = plane * kCBe;  // offset in the group's reduction
                            if constexpr (kIm2col) {
                                const bool in = tap < p.taps;
                                // past the last plane: the last tap, so the load stays well formed
                                const int kdc = in ? kd : (kVol ? (p.taps - 1) / (p.Kh * p.Kw) : 0);
                                const int khc = in ? kh : (kVol ? p.Kh - 1 : (p.taps - 1) / p.Kw);
                                const int kwc = in ? kw : p.Kw - 1;
                                const int c = t.g * p.Cpg + cblk * kCBe;
                                const uint16_t ow_ = static_cast<uint16_t>(kwc * p.dilation);
                                const uint16_t oh_ = static_cast<uint16_t>(khc * p.dilation);
                                if constexpr (kVol) {
                                    const uint16_t od_ = static_cast<uint16_t>(kdc * p.dilation);
                                    if constexpr (kPair)
                                        tma_load_im2col_5d_pair(st + j * (kBM * kCB), &p.tmap_a, fbar, c, w0, h0, d0,
                                                                img, ow_, oh_, od_);
                                    else
                                        tma_load_im2col_5d(st + j * (kBM * kCB), &p.tmap_a, &sb.full[stage], c, w0,
                                                           h0, d0, img, ow_, oh_, od_);
                                } else if constexpr (kPair) {
                                    tma_load_im2col_4d_pair(st + j * (kBM * kCB), &p.tmap_a, fbar, c, w0, h0,
                                                            img, ow_, oh_);
                                } else {
                                    tma_load_im2col_4d(st + j * (kBM * kCB), &p.tmap_a, &sb.full[stage],
                                                       c, w0, h0, img, ow_, oh_);
                                }
                                if (++cblk == p.nCB) {
                                    cblk = 0;
                                    ++tap;
                                    if (++kw == p.Kw) {
                                        kw = 0;
                                        if (++kh == p.Kh && kVol) {
                                            kh = 0;
                                            ++kd;
                                        }
                                    }
                                }
                            } else {
                                if constexpr (kPair)
                                    tma_load_2d_pair(st + j * (kBM * kCB), &p.tmap_a, fbar, t.g * p.Kp + kelem, m0);
                                else
                                    tma_load_2d(st + j * (kBM * kCB), &p.tmap_a, &sb.full[stage],
                                                t.g * p.Kp + kelem, m0);
                            }
                            if constexpr (kPair)
                                tma_load_3d_pair(st + b_off + j * (BNl * kCB), &p.tmap_b, fbar, kelem,
                                                 t.ntile * BN + static_cast<int>(rank) * BNl, t.g);
                            else
                                tma_load_3d(st + b_off + j * (BN * kCB), &p.tmap_b, &sb.full[stage],
                                            kelem, t.ntile * BN, t.g);
                        }
                        ++loads_issued;
                    }
                    if (++stage == p.stages) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
            }
            if constexpr (kPair) {
                if (!*wd.abort) {
                    // Wait until the MMAs have released every slot, so that no commit
                    // from rank 0 is still on its way to this CTA's barriers at exit.
                    for (int i = 0; i < p.stages; ++i) {
                        if (!mbar_wait(&sb.empty[stage], phase ^ 1u, wd, kDevTimeoutEmpty)) break;
                        if (++stage == p.stages) {
                            stage = 0;
                            phase ^= 1u;
                        }
                    }
                }
                if (*wd.abort && loads_issued > 0) {
                    if (rank == 0) {
                        // Both CTAs' loads of a stage complete on rank 0's full barrier:
                        // wait (bounded) for every phase this CTA armed and has not seen
                        // complete, so that no copy of either CTA is still writing into a
                        // stage of an armed phase.  The odd CTA leaves only after the
                        // final cluster barrier, i.e. after these waits.
                        const long long first = loads_issued > p.stages ? loads_issued - p.stages : 0;
                        for (long long i = first; i < loads_issued; ++i)
                            wait_quiet(&sb.full[i % p.stages], static_cast<uint32_t>((i / p.stages) & 1),
                                       wd.timeout_ns);
                    } else {
                        // The odd CTA cannot observe its own copies (they count on the even
                        // CTA's barrier).  Copies it issued for a phase the even CTA never
                        // armed get a fixed time to land: the one remaining bounded case.
                        const uint64_t t0 = globaltimer_ns();
                        while (globaltimer_ns() - t0 < 200000u) {
                        }
                    }
                }
            } else if (*wd.abort && loads_issued > 0) {
                // Let the copies still in flight land before the CTA goes away.
                const long long first = loads_issued > p.stages ? loads_issued - p.stages : 0;
                for (long long i = first; i < loads_issued; ++i)
                    wait_quiet(&sb.full[i % p.stages], static_cast<uint32_t>((i / p.stages) & 1),
                               wd.timeout_ns);
            }
        }
    } else if (warp == kMmaWarp) {
        // --------------------------------------------------- tensor-core issue ---
        if (lane == 0 && rank == 0) {
            const uint32_t idesc = instr_desc(kF32 ? 2u : 1u, kUnitRows, static_cast<uint32_t>(BN));
            int stage = 0;
            uint32_t phase = 0;
            int abuf = 0;
            uint32_t aphase = 0;
            bool ok = true;
            for (int u = unit0; ok && u < p.units; u += ustep) {
                const Unit t = decode_unit(p, u);
                const int cs = p.chunk_stages > 0 ? p.chunk_stages : t.k1 - t.k0;
                // Each chunk of the reduction goes into a fresh accumulator; the
                // epilogue adds the chunks up (see the fp32 epilogue).
                for (int c0 = t.k0; ok && c0 < t.k1; c0 += cs) {
                    const int c1 = min(c0 + cs, t.k1);
                    if (!mbar_wait(&sb.acc_empty[abuf], aphase ^ 1u, wd, kDevTimeoutAccEmpty)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after_sync();
                    const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(abuf * BN);
                    for (int ks = c0; ks < c1; ++ks) {
                        uint64_t *ready = kF32 ? &sb.converted[stage] : &sb.full[stage];
                        if (!mbar_wait(ready, phase, wd, kF32 ? kDevTimeoutConvert : kDevTimeoutFull)) {
                            ok = false;
                            break;
                        }
                        tc_fence_after_sync();
                        const uint32_t st = smem_addr(ring + static_cast<size_t>(stage) * sbytes);
                        issue_stage<kF32, kCB, kPair>(st, st + b_off, st + alo_off, st + blo_off, BNl,
                                                      d_tmem, idesc, ks == c0);
                        if constexpr (kPair)
                            mma_commit_pair(&sb.empty[stage], 0x3);  // both CTAs' slots
                        else
                            mma_commit(&sb.empty[stage]);
                        if (++stage == p.stages) {
                            stage = 0;
                            phase ^= 1u;
                        }
                    }
                    if (!ok) break;
                    if constexpr (kPair)
                        mma_commit_pair(&sb.acc_full[abuf], 0x3);
                    else
                        mma_commit(&sb.acc_full[abuf]);
                    abuf ^= 1;
                    if (abuf == 0) aphase ^= 1u;
                }
            }
            if (!ok || *wd.abort) {
                if constexpr (kPair)
                    mma_commit_pair(&sb.drain, 0x1);
                else
                    mma_commit(&sb.drain);
                wait_quiet(&sb.drain, 0, wd.timeout_ns);
            }
        }
        __syncwarp();
    } else if (warp < kEpiWarp0 + epi_warps<kF32>()) {
        // ------------------------------------------------------------ epilogue ---
        const int quarter = warp & 3;  // tensor-memory lanes [32*quarter, 32*quarter + 32)
        // columns of the tile this warp drains: all (fp32), or one half (bf16), in
        // multiples of 32 so that TMA-store blocks never straddle two warps
        const int half = (warp - kEpiWarp0) >> 2;
        const int cspan = kF32 ? BN : ((BN / 2 + 31) & ~31);
        const int c_lo = min(BN, half * cspan), c_hi = min(BN, c_lo + cspan);
        const int row = quarter * 32 + lane;
        int abuf = 0;
        uint32_t aphase = 0;
        const uint32_t lane_base = static_cast<uint32_t>(quarter * 32) << 16;
        const OutDesc out = out_desc(p);
        uint8_t *ystage = ring + static_cast<size_t>(p.stages) * sbytes;  // tma_out staging
        // hands accumulator `b` back to the MMA issuer (rank 0 of a pair)
        auto release_acc = [&](int b) {
            if constexpr (kPair)
                mbar_arrive_cluster(acc_empty0 + 8u * static_cast<uint32_t>(b));
            else
                mbar_arrive(&sb.acc_empty[b]);
        };
        int sbi = 0;
        for (int u = unit0; u < p.units; u += ustep) {
            const Unit t = decode_unit(p, u);
            const int m = t.mtile * kUnitRows + row_off + row;
            if constexpr (kF32) {
                // The tensor cores' own accumulation loses accuracy over long
                // reductions, so each chunk of p.chunk_stages stages is accumulated afresh
                // in tensor memory and the chunks are summed here with IEEE fp32 adds.
                const int cs = p.chunk_stages > 0 ? p.chunk_stages : t.k1 - t.k0;
                const int nch = (t.k1 - t.k0 + cs - 1) / cs;
                float acc[kMaxBNf32];
#pragma unroll
                for (int i = 0; i < kMaxBNf32; ++i) acc[i] = 0.f;
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
                    for (int c = 0; c < kMaxBNf32 / 16; ++c) {
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
                    if (lane == 0) release_acc(abuf);
                    abuf ^= 1;
                    if (abuf == 0) aphase ^= 1u;
                }
                if (!ok) break;
#pragma unroll
                for (int c = 0; c < kMaxBNf32 / 16; ++c)
                    if (c * 16 < BN) store16<kF32>(out, m, t.g, t.ntile * BN + c * 16, t.split, &acc[c * 16]);
            } else if (p.tma_out) {
                // bf16 channels-last output through shared memory: per block of 32 columns
                // each thread writes its row's 64 bytes into this warp's staging buffer
                // (64-byte swizzle: 16-byte chunk q of row r goes to chunk q ^ ((r >> 1) & 3),
                // conflict-free), then one lane stores the 32 x 32 block with TMA; two
                // buffers per warp let the next block fill while the previous store reads.
                const bool ok = mbar_wait(&sb.acc_full[abuf], aphase, wd, kDevTimeoutAccFull);
                if (!__all_sync(0xffffffffu, ok)) break;
                tc_fence_after_sync();
                const uint32_t taddr = tmem_base + lane_base + static_cast<uint32_t>(abuf * BN);
                const int mrow0 = t.mtile * kUnitRows + row_off + quarter * 32;
                const int col0 = t.g * p.Cout_g + t.ntile * BN;
                if (c_lo >= c_hi) {  // nothing to drain in this half: release at once
                    tc_fence_before_sync();
                    __syncwarp();
                    if (lane == 0) release_acc(abuf);
                }
                for (int c = c_lo; c < c_hi; c += 32) {
                    uint32_t r[2][16];
                    tmem_ld_x16(taddr + static_cast<uint32_t>(c), r[0]);
                    tmem_ld_x16(taddr + static_cast<uint32_t>(c + 16), r[1]);
                    tmem_ld_wait();
                    if (c + 32 >= c_hi) {  // this warp's part of the accumulator is read
                        tc_fence_before_sync();
                        __syncwarp();
                        if (lane == 0) release_acc(abuf);
                    }
                    float bv[32];
                    if (p.bias) {
                        const uint4 *b4 = reinterpret_cast<const uint4 *>(
                            static_cast<const __nv_bfloat16 *>(p.bias) + col0 + c);
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
                    uint8_t *buf = ystage + ((warp - kEpiWarp0) * 2 + sbi) * kStageBufBytes;
#pragma unroll
                    for (int q = 0; q < 4; ++q)
                        *reinterpret_cast<uint4 *>(buf + lane * 64 + ((q ^ ((lane >> 1) & 3)) * 16)) =
                            make_uint4(pk[4 * q], pk[4 * q + 1], pk[4 * q + 2], pk[4 * q + 3]);
                    fence_proxy_async_smem();
                    __syncwarp();
                    if (lane == 0 && mrow0 < p.M) {
                        tma_store_2d(&p.tmap_y, buf, col0 + c, mrow0);
                        bulk_commit_group();
                    }
                    sbi ^= 1;
                }
                abuf ^= 1;
                if (abuf == 0) aphase ^= 1u;
            } else {
                const bool ok = mbar_wait(&sb.acc_full[abuf], aphase, wd, kDevTimeoutAccFull);
                if (!__all_sync(0xffffffffu, ok)) break;
                tc_fence_after_sync();
                const uint32_t taddr = tmem_base + lane_base + static_cast<uint32_t>(abuf * BN);
                for (int c = c_lo; c < c_hi; c += 16) {
                    uint32_t r[16];
                    tmem_ld_x16(taddr + static_cast<uint32_t>(c), r);
                    tmem_ld_wait();
                    float v[16];
#pragma unroll
                    for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
                    store16<kF32>(out, m, t.g, t.ntile * BN + c, t.split, v);
                }
                tc_fence_before_sync();
                __syncwarp();
                if (lane == 0) release_acc(abuf);
                abuf ^= 1;
                if (abuf == 0) aphase ^= 1u;
            }
        }
        if (p.tma_out && lane == 0) bulk_wait_group_all();  // stores done before exit
    } else if constexpr (kF32) {
        // ------------------------------------------- fp32 -> tf32 hi/lo split ---
        const int tid = (warp - kCvtWarp0) * 32 + lane;  // 0..127
        int stage = 0;
        uint32_t phase = 0;
        bool ok = true;
        for (int u = unit0; ok && u < p.units; u += ustep) {
            const Unit t = decode_unit(p, u);
            for (int ks = t.k0; ks < t.k1; ++ks) {
                if (!mbar_wait(&sb.full[stage], phase, wd, kDevTimeoutFull)) {
                    ok = false;
                    break;
                }
                uint8_t *st = ring + static_cast<size_t>(stage) * sbytes;
                float4 *a = reinterpret_cast<float4 *>(st);
                float4 *alo = reinterpret_cast<float4 *>(st + alo_off);
                for (int i = tid; i < kAStageBytes / 16; i += 128) {
                    const float4 v = a[i];
                    float4 h, l;
                    h.x = tf32_round(v.x); l.x = tf32_round(v.x - h.x);
                    h.y = tf32_round(v.y); l.y = tf32_round(v.y - h.y);
                    h.z = tf32_round(v.z); l.z = tf32_round(v.z - h.z);
                    h.w = tf32_round(v.w); l.w = tf32_round(v.w - h.w);
                    a[i] = h;
                    alo[i] = l;
                }
                float4 *b = reinterpret_cast<float4 *>(st + b_off);
                float4 *blo = reinterpret_cast<float4 *>(st + blo_off);
                const int nb = BN * kStageRowBytes / 16;
                for (int i = tid; i < nb; i += 128) {
                    const float4 v = b[i];
                    float4 h, l;
                    h.x = tf32_round(v.x); l.x = tf32_round(v.x - h.x);
                    h.y = tf32_round(v.y); l.y = tf32_round(v.y - h.y);
                    h.z = tf32_round(v.z); l.z = tf32_round(v.z - h.z);
                    h.w = tf32_round(v.w); l.w = tf32_round(v.w - h.w);
                    b[i] = h;
                    blo[i] = l;
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
    if constexpr (kPair) cluster_sync();  // neither CTA leaves while the pair still works
    if (warp == kMmaWarp) {
        tc_fence_after_sync();
        if constexpr (kPair)
            tmem_dealloc_pair(tmem_base, p.tmem_cols);
        else
            tmem_dealloc(tmem_base, p.tmem_cols);
    }
}

template <bool kF32, int kCB, bool kIm2col, bool kPair, bool kVol = false>
cudaError_t launch_one(const IgemmParams &p, int grid, size_t smem, cudaStream_t stream) {
    auto kern = igemm_kernel<kF32, kCB, kIm2col, kPair, kVol>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    if constexpr (kPair) {
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(static_cast<unsigned>(grid));
        cfg.blockDim = dim3(threads_for<kF32>());
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
    } else {
        kern<<<grid, threads_for<kF32>(), smem, stream>>>(p);
    }
    return cudaGetLastError();
}

// How many two-CTA clusters of the pair kernel fit on the device at once.
template <int kCB, bool kIm2col, bool kVol = false>
cudaError_t pair_clusters_one(size_t smem, int *out) {
    auto kern = igemm_kernel<false, kCB, kIm2col, true, kVol>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2);
    cfg.blockDim = dim3(threads_for<false>());
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

template <bool kF32, bool kIm2col, bool kPair, bool kVol = false>
cudaError_t launch_cb(const IgemmParams &p, int cb, int grid, size_t smem, cudaStream_t s) {
    switch (cb) {
        case 128: return launch_one<kF32, 128, kIm2col, kPair, kVol>(p, grid, smem, s);
        case 64: return launch_one<kF32, 64, kIm2col, kPair, kVol>(p, grid, smem, s);
        case 32: return launch_one<kF32, 32, kIm2col, kPair, kVol>(p, grid, smem, s);
        case 16: return launch_one<kF32, 16, kIm2col, kPair, kVol>(p, grid, smem, s);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace

size_t igemm_smem_bytes(bool f32, int BN, int stages, bool tma_out) {
    return 1024 /* alignment slack */ + kBarrierBlock +
           static_cast<size_t>(stages) * stage_bytes(f32, BN) + (tma_out ? kYStageBytes : 0);
}

int igemm_threads(bool f32) { return f32 ? threads_for<true>() : threads_for<false>(); }

cudaError_t igemm_pair_max_clusters(int cb_bytes, bool im2col, size_t smem_bytes, int *clusters, bool vol) {
    *clusters = 0;
    if (vol) {
        switch (cb_bytes) {
            case 128: return pair_clusters_one<128, true, true>(smem_bytes, clusters);
            case 64: return pair_clusters_one<64, true, true>(smem_bytes, clusters);
            case 32: return pair_clusters_one<32, true, true>(smem_bytes, clusters);
            case 16: return pair_clusters_one<16, true, true>(smem_bytes, clusters);
            default: return cudaErrorInvalidValue;
        }
    }
    switch (cb_bytes) {
        case 128: return im2col ? pair_clusters_one<128, true>(smem_bytes, clusters)
                                : pair_clusters_one<128, false>(smem_bytes, clusters);
        case 64: return im2col ? pair_clusters_one<64, true>(smem_bytes, clusters)
                               : pair_clusters_one<64, false>(smem_bytes, clusters);
        case 32: return im2col ? pair_clusters_one<32, true>(smem_bytes, clusters)
                               : pair_clusters_one<32, false>(smem_bytes, clusters);
        case 16: return im2col ? pair_clusters_one<16, true>(smem_bytes, clusters)
                               : pair_clusters_one<16, false>(smem_bytes, clusters);
        default: return cudaErrorInvalidValue;
    }
}

cudaError_t launch_igemm(const IgemmParams &p, bool f32, int cb_bytes, bool im2col, bool pair, int grid,
                         size_t smem_bytes, cudaStream_t stream, bool vol) {
    if (p.stages < 2 || p.stages > kMaxStages) return cudaErrorInvalidValue;
    if (vol) {
        if (!im2col) return cudaErrorInvalidValue;
        if (pair) {
            if (f32 || grid % 2 != 0) return cudaErrorInvalidValue;
            return launch_cb<false, true, true, true>(p, cb_bytes, grid, smem_bytes, stream);
        }
        return f32 ? launch_cb<true, true, false, true>(p, cb_bytes, grid, smem_bytes, stream)
                   : launch_cb<false, true, false, true>(p, cb_bytes, grid, smem_bytes, stream);
    }
    if (pair) {
        if (f32 || grid % 2 != 0) return cudaErrorInvalidValue;
        return im2col ? launch_cb<false, true, true>(p, cb_bytes, grid, smem_bytes, stream)
                      : launch_cb<false, false, true>(p, cb_bytes, grid, smem_bytes, stream);
    }
    if (f32) {
        return im2col ? launch_cb<true, true, false>(p, cb_bytes, grid, smem_bytes, stream)
                      : launch_cb<true, false, false>(p, cb_bytes, grid, smem_bytes, stream);
    }
    return im2col ? launch_cb<false, true, false>(p, cb_bytes, grid, smem_bytes, stream)
                  : launch_cb<false, false, false>(p, cb_bytes, grid, smem_bytes, stream);
}

}  // namespace conv2d_b200
