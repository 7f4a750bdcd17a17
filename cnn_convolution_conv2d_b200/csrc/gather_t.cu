// gather_t.cu -- the few-channel first layer (bf16, NCHW in and out) as the transposed
// product: output channels on the tensor-memory lanes, output pixels along the columns.
//
// The first layer of an image network reads 3 colour channels ("PyTorch高维张量乘法与
// conv2d/conv3d维度语义解析" §6.3: channels-last brings nothing there) and writes many
// more; the im2col/GEMM tutorial (zskr.cn/news/1820658) §2.3 writes its product as
// Y = W_row @ X_col with W_row (C_out x C_in*Kh*Kw) on the left.  Computed that way round
// on the tensor cores, each accumulator lane holds one output channel and its columns
// are consecutive output pixels of one output row, so each thread owns one channel's
// row: it adds one bias and writes whole 16-byte pieces of that row, into a
// shared-memory image of the tile's block of y from which one TMA box store per tile
// writes the NCHW output (or, when the image does not fit, straight into y).  No
// transposition anywhere.  (The other few-channel kernel, gather.cu, has pixels on the
// lanes and must turn each tile channel-major before storing it.)
//
// A tile is RT output rows (oh0 .. oh0 + RT - 1) of one image.  With C_out <= 64 a tile
// takes two rows (RT = 2): the product's 128 lanes hold both rows' channels, rows
// 0..63 of A being the filter and rows 64..127 the same filter moved down by one stride
// of input rows, so that one reduction over the Kh + stride input rows the pair reads
// gives both output rows: no half-empty accumulator, and the pair's input rows are
// gathered once.
//
//   A (M = 128 x K): RT = 1: the weight image that conv2d_pack_weight wrote (C_out rows,
//      K in the row-vector order k = (c*Kh + kh)*8 + kw, 16-byte k chunks), rows
//      C_out..127 zero, one bulk copy; RT = 2: built from that image at the start
//      (row r*64 + oc, chunk c*R + kh + r*stride).  Resident for the whole launch: in
//      tensor memory beside the accumulators when it fits there (built in the B buffers'
//      space, which is free at the start, then copied lane by lane), so that the tensor
//      cores read only B from shared memory; otherwise in shared memory;
//   B (N = Wo padded to 16, x K): the im2col rows of the tile's output pixels, gathered by
//      the gather warps from input rows staged in shared memory by one TMA box load per
//      tile (all channels, the R = Kh + (RT-1)*stride rows the tile reads, with a zero
//      margin on the left; outside the image the box reads zeros: the padding), chunk j
//      reading staged row j; double-buffered;
//   D (tensor memory, fp32): lanes = (output row, output channel), columns = pixels, a ring
//      of up to four accumulators (as many as 512 columns hold beside A).
//
//   gather warps 0..7 : two groups of four on alternate tiles, thread t of a group builds
//                       pixel rows t (+ 128); a group's first thread reloads each staged-row
//                       buffer it has read with the rows of its tile nhalo ahead (up to
//                       eight: a tile's own work is shorter than the latency of its load;
//                       the first round is issued at the start);
//   warp 8            : tensor-memory allocation, tcgen05.mma from one thread;
//   warps 9..16       : epilogue, two warps per lane quarter (each half of the columns):
//                       tcgen05.ld, + bias, one rounding to bf16, 16-byte writes into
//                       the output image (64-pixel parts, 128-byte swizzled), then one TMA
//                       store per part.
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
constexpr int kGtMaxChunks = 32;   // K <= 256 bf16
constexpr int kGtMaxHalo = 8;      // staged-row buffers: loads run up to this many tiles ahead
constexpr int kGtMaxAcc = 4;       // accumulators in tensor memory

struct GtShared {
    uint64_t halo_full[kGtMaxHalo];
    uint64_t b_full[2];
    uint64_t b_empty[2];
    uint64_t acc_full[kGtMaxAcc];
    uint64_t acc_empty[kGtMaxAcc];
    uint64_t a_ready;
    uint64_t a_tm_ready;   // A is in tensor memory (four epilogue warps)
    uint64_t drain;
    uint32_t tmem_base;
    int abort;
};
static_assert(sizeof(GtShared) <= kGtHeader, "header too small");

__device__ __forceinline__ uint32_t gt_align1k(uint32_t v) { return (v + 1023u) & ~1023u; }

// Offset of (row m, 16-byte chunk j) in a no-swizzle K-major operand whose 8-row groups
// are `sbo` bytes apart.
__device__ __forceinline__ uint32_t gt_core(int m, int j, uint32_t sbo) {
    return static_cast<uint32_t>(m >> 3) * sbo + static_cast<uint32_t>(j) * 128u + static_cast<uint32_t>(m & 7) * 16u;
}

// Arrival on hardware barrier `id` without waiting: the other side of a named_barrier that
// one warp waits on while the rest of its group go on.
__device__ __forceinline__ void gt_barrier_arrive(int id, int count) {
    asm volatile("bar.arrive %0, %1;" ::"r"(id), "r"(count) : "memory");
}

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
    const int nchunks = p.kt / 8;                                // chunks of the tile's reduction
    const uint32_t sbo = static_cast<uint32_t>(nchunks) * 128u;  // one 8-row group of a K-major operand
    const int tpix = p.tpix;                                     // B rows (pixels), a multiple of 16
    const int rt = p.rt;                                         // output rows per tile
    const bool a_tmem = p.a_tmem != 0;                           // A resident in tensor memory
    const uint32_t a_bytes = 16u * sbo;                          // 128 rows
    uint8_t *b_sm = base + kGtHeader + (a_tmem ? 0u : gt_align1k(a_bytes));
    uint8_t *a_sm = a_tmem ? b_sm : base + kGtHeader;            // A is built in B's space first
    const uint32_t b_bytes = static_cast<uint32_t>(tpix / 8) * sbo;
    const uint32_t b_stride = gt_align1k(b_bytes);
    uint8_t *halo_sm = b_sm + 2 * b_stride;
    const uint32_t halo_bytes = static_cast<uint32_t>(p.C) * p.R * p.BW * 2u;
    const uint32_t halo_stride = gt_align1k(halo_bytes);
    uint8_t *out_sm = halo_sm + p.nhalo * halo_stride;            // output images (tma_out)
    // an output image: ceil(Wo / 64) parts of (rt x BN) 128-byte rows (64 pixels), each the
    // 128-byte-swizzled box of one TMA store
    const int oparts = (p.Wo + 63) / 64;
    const uint32_t opart_bytes = static_cast<uint32_t>(rt * p.BN) * 128u;
    const uint32_t out_stride = gt_align1k(static_cast<uint32_t>(oparts) * opart_bytes);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int i = 0; i < p.nhalo; ++i) mbar_init(&sb.halo_full[i], 1);
        for (int i = 0; i < 2; ++i) {
            mbar_init(&sb.b_full[i], kGtProd / 2);  // the gather group of the tile (four warps)
            mbar_init(&sb.b_empty[i], 1);
        }
        for (int i = 0; i < p.nacc; ++i) {
            mbar_init(&sb.acc_full[i], 1);
            // every epilogue warp of the tile's group hands the accumulator back
            mbar_init(&sb.acc_empty[i], (p.tma_out && p.nout == 2) ? kGtEpi / 2 : kGtEpi);
        }
        mbar_init(&sb.a_ready, 1);
        mbar_init(&sb.a_tm_ready, 4);
        mbar_init(&sb.drain, 1);
        sb.abort = 0;
        fence_mbar_init();
    }
    const int tiles_per_img = (p.Ho + rt - 1) / rt;
    auto issue_halo = [&](int t, int hb) {
        const int img = t / tiles_per_img;
        const int oh0 = (t - img * tiles_per_img) * rt;
        mbar_arrive_expect_tx(&sb.halo_full[hb], halo_bytes);
        tma_load_4d(halo_sm + hb * halo_stride, &p.tmap_x, &sb.halo_full[hb], -p.ME, oh0 * p.stride - p.pad, 0, img);
    };
    // A from the weight image.  Every CTA reads the same image at the same moment: it comes
    // into shared memory by one bulk copy, issued ahead of the staged input rows so that it
    // does not queue behind them, rather than by a global load per 16-byte piece (a per-role
    // clock record put that form at ~6.5 K cycles of the launch's start).  With A in tensor
    // memory the image lands in the output images (free until the first tile's accumulator,
    // which needs A) and four epilogue warps write A's rows from it straight into tensor
    // memory while the gather warps start on the first tiles; otherwise A is built in
    // shared memory before the roles split (two rows per tile: from the image staged beside
    // it; one row: the image is A, loaded by the product warp).
    const int ichunks = p.Kpad / 8;                                // the image's chunks
    const uint32_t isbo = static_cast<uint32_t>(ichunks) * 128u;
    const uint32_t img_bytes = static_cast<uint32_t>(p.BN / 8) * isbo;
    uint8_t *stage = nullptr;
    if (a_tmem) {
        if (static_cast<uint32_t>(p.nout) * out_stride >= img_bytes) stage = out_sm;
    } else if (rt == 2) {
        if (2 * b_stride >= img_bytes) stage = b_sm;
        else if (static_cast<uint32_t>(p.nout) * out_stride >= img_bytes) stage = out_sm;
    }
    if (stage != nullptr && threadIdx.x == 0 && !p.starve) {
        mbar_arrive_expect_tx(&sb.a_ready, img_bytes);
        bulk_load(stage, p.w_image, img_bytes, &sb.a_ready);
    }
    const bool a_staged = stage != nullptr;
    if (threadIdx.x == 0 && !p.starve) {
        // the first tiles' input rows are on their way while A is being set up
        prefetch_tensormap(&p.tmap_x);
        for (int k = 0; k < p.nhalo; ++k)
            if (blockIdx.x + k * static_cast<int>(gridDim.x) < p.n_mtiles) issue_halo(blockIdx.x + k * gridDim.x, k);
    }
    Watchdog wd;
    wd.abort = &sb.abort;
    wd.status = p.status;
    wd.timeout_ns = static_cast<uint64_t>(p.timeout_ns);
    if (!a_tmem && rt == 1) {
        // weight rows past the image's (C_out rounded up to 16) are zero: output channels
        // that do not exist come out as zeros and are not stored
        uint4 *z = reinterpret_cast<uint4 *>(a_sm + img_bytes);
        for (uint32_t i = threadIdx.x; i < (a_bytes - img_bytes) / 16u; i += blockDim.x) z[i] = make_uint4(0, 0, 0, 0);
    } else if (!a_tmem) {
        // Two rows per tile: row r*64 + oc of A, chunk c*R + kh + r*stride, holds the
        // image's row oc, chunk c*Kh + kh (R = Kh + stride staged rows); all else is zero.
        uint4 *z = reinterpret_cast<uint4 *>(a_sm);
        for (uint32_t i = threadIdx.x; i < a_bytes / 16u; i += blockDim.x) z[i] = make_uint4(0, 0, 0, 0);
        __syncthreads();
        // a copy that never lands leaves A zero and the watchdog's status set
        const bool img_ok = !a_staged || mbar_wait(&sb.a_ready, 0, wd, kDevTimeoutFull);
        const int real = p.C * p.Kh;
        const uint8_t *img = a_staged ? stage : static_cast<const uint8_t *>(p.w_image);
        for (int i = threadIdx.x; img_ok && i < p.BN * real; i += blockDim.x) {
            const int oc = i / real, j = i - (i / real) * real;
            const int c = j / p.Kh, kh = j - (j / p.Kh) * p.Kh;
            const uint4 *q = reinterpret_cast<const uint4 *>(img + gt_core(oc, j, isbo));
            const uint4 v = a_staged ? *q : __ldg(q);
            const int j0 = c * p.R + kh;
            *reinterpret_cast<uint4 *>(a_sm + gt_core(oc, j0, sbo)) = v;
            *reinterpret_cast<uint4 *>(a_sm + gt_core(64 + oc, j0 + p.stride, sbo)) = v;
        }
    }
    fence_proxy_async_smem();
    if (warp == kGtMma) {
        tmem_alloc(&sb.tmem_base, p.tmem_cols);
        tmem_relinquish();
    }
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    const uint32_t tmem_base = sb.tmem_base;
    const uint32_t a_col = static_cast<uint32_t>(p.nacc * tpix);   // A's first tensor-memory column

    if (warp < kGtProd) {
        // ------------------------------------------------------------- gather ---
        // Two groups of four warps on alternate tiles, each with its own B buffer, so that one
        // tile's waits overlap the other's gather; a thread builds all chunks of its rows.
        const int grp = warp / (kGtProd / 2);
        const int row0 = threadIdx.x & 127;         // first pixel (B row) of this thread; then +128
        const int jb = 0, je = nchunks;
        // rows past Wo feed columns that are never stored
        // chunk j = c*R + r reads staged row j (unit dilation); chunks past C*R are the
        // reduction's zero padding
        const int crow = p.C * p.R;
        const int bww = p.BW / 2;                   // 32-bit words per staged row (BW is even)
        // Once the group has read a staged-row buffer, its first thread reloads it with the
        // rows of the group's tile nhalo ahead (nhalo is even, so a buffer serves one group
        // and has one issuer).  last[k]: the tile count of the last load into buffer k.
        const bool lead_warp = warp % (kGtProd / 2) == 0;
        int last[kGtMaxHalo];
        for (int k = 0; k < kGtMaxHalo; ++k)
            last[k] = (k < p.nhalo && k % 2 == grp && !p.starve &&
                       blockIdx.x + k * static_cast<int>(gridDim.x) < p.n_mtiles) ? k : -1;
        int li = grp;
        for (int t = blockIdx.x + grp * static_cast<int>(gridDim.x); t < p.n_mtiles;
             t += 2 * static_cast<int>(gridDim.x), li += 2) {
            const int b = li & 1;                   // = grp
            const uint32_t ph = static_cast<uint32_t>(li >> 1) & 1u;
            const int hb = li % p.nhalo;
            const uint32_t hph = static_cast<uint32_t>(li / p.nhalo) & 1u;
            const bool ok = mbar_wait(&sb.b_empty[b], ph ^ 1u, wd, kDevTimeoutEmpty) &&
                            mbar_wait(&sb.halo_full[hb], hph, wd, kDevTimeoutFull);
            // the group's four warps leave together (they meet at the reload below)
            if (!named_barrier_all(7 + grp, (kGtProd / 2) * 32, ok)) break;
            for (int row = row0; row < p.Wo; row += 128) {
                const uint32_t *h32 = reinterpret_cast<const uint32_t *>(halo_sm + hb * halo_stride);
                const int e0 = row * p.stride - p.pad + p.ME;   // staged column of kw = 0
                const uint32_t *hrow = h32 + (e0 >> 1);
                const uint32_t sh = (e0 & 1) * 16u;
                uint8_t *dst = b_sm + b * b_stride + gt_core(row, 0, sbo);
                // at most kGtMaxChunks chunks per thread, in batches of 8: all of a
                // batch's loads are issued before any of its stores (a store could alias a
                // later load as far as the compiler knows, which would serialise them)
#pragma unroll
                for (int g0 = 0; g0 < kGtMaxChunks; g0 += 8) {
                    if (jb + g0 >= je) break;
                    uint32_t w[8][5];
#pragma unroll
                    for (int i = 0; i < 8; ++i) {
                        const int j = jb + g0 + i;
                        const bool real = j < je && j < crow;
                        const uint32_t *q = hrow + (real ? j : 0) * bww;
#pragma unroll
                        for (int k = 0; k < 5; ++k) w[i][k] = real ? q[k] : 0u;
                    }
#pragma unroll
                    for (int i = 0; i < 8; ++i) {
                        const int j = jb + g0 + i;
                        if (j < je) {
                            uint4 v;
                            v.x = __funnelshift_r(w[i][0], w[i][1], sh);
                            v.y = __funnelshift_r(w[i][1], w[i][2], sh);
                            v.z = __funnelshift_r(w[i][2], w[i][3], sh);
                            v.w = __funnelshift_r(w[i][3], w[i][4], sh);
                            *reinterpret_cast<uint4 *>(dst + j * 128) = v;
                        }
                    }
                }
            }
            fence_proxy_async_smem();   // the tensor cores read these rows
            __syncwarp();
            if (lane == 0 && !p.starve) mbar_arrive(&sb.b_full[b]);
            const int t2 = t + p.nhalo * static_cast<int>(gridDim.x);
            if (!p.starve && t2 < p.n_mtiles) {
                if (lead_warp) {
                    named_barrier(5 + grp, (kGtProd / 2) * 32);
                    if (lane == 0) {
                        issue_halo(t2, hb);
                        last[hb] = li + p.nhalo;
                    }
                } else {
                    gt_barrier_arrive(5 + grp, (kGtProd / 2) * 32);
                }
            }
        }
        if (lead_warp && lane == 0 && *wd.abort)   // let this group's loads still in flight land
            for (int k = 0; k < p.nhalo; ++k)
                if (last[k] >= 0)
                    gt_wait_quiet(&sb.halo_full[k], static_cast<uint32_t>(last[k] / p.nhalo) & 1u, wd.timeout_ns);
    } else if (warp == kGtMma) {
        // ------------------------------------------- loads and tensor-core issue ---
        if (lane == 0) {
            const uint32_t idesc = instr_desc(1u, 128, static_cast<uint32_t>(tpix));
            const uint32_t a_addr = smem_addr(a_sm);
            const int ksteps = nchunks / 2;       // 32 bytes of k per instruction
            // descriptors' fields but the start address, set once (the issue of a tile's
            // products is on its critical path)
            const uint64_t bd0 = smem_desc(0u, 128, sbo, kSwNone);
            bool ok = !*wd.abort;
            if (a_tmem && !mbar_wait(&sb.a_tm_ready, 0, wd, kDevTimeoutFull)) ok = false;
            tc_fence_after_sync();
            if (!a_tmem && rt == 1 && !p.starve) {
                const uint32_t img_bytes = static_cast<uint32_t>(p.BN / 8) * sbo;
                mbar_arrive_expect_tx(&sb.a_ready, img_bytes);
                bulk_load(a_sm, p.w_image, img_bytes, &sb.a_ready);
            }
            if (!a_tmem && rt == 1 && !mbar_wait(&sb.a_ready, 0, wd, kDevTimeoutFull)) ok = false;
            int li = 0, ab = 0;
            uint32_t aph = 0;                     // accumulator ab's phase
            for (int t = blockIdx.x; ok && t < p.n_mtiles; t += gridDim.x, ++li) {
                const int b = li & 1;
                const uint32_t ph = static_cast<uint32_t>(li >> 1) & 1u;
                if (!mbar_wait(&sb.acc_empty[ab], aph ^ 1u, wd, kDevTimeoutAccEmpty) ||
                    !mbar_wait(&sb.b_full[b], ph, wd, kDevTimeoutFull)) {
                    ok = false;
                    break;
                }
                tc_fence_after_sync();
                const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(ab * tpix);
                const uint32_t b_addr = smem_addr(b_sm + b * b_stride);
                if (a_tmem) {
                    for (int ks = 0; ks < ksteps; ++ks)   // 16 k = 8 columns of A per instruction
                        mma_bf16_tmem_a(d_tmem, tmem_base + a_col + static_cast<uint32_t>(ks) * 8u,
                                        bd0 | ((b_addr + static_cast<uint32_t>(ks) * 256u) >> 4), idesc,
                                        ks > 0 ? 1u : 0u);
                } else {
                    for (int ks = 0; ks < ksteps; ++ks) {
                        const uint32_t off = static_cast<uint32_t>(ks) * 256u;  // two 16-byte k chunks
                        mma_bf16(d_tmem, bd0 | ((a_addr + off) >> 4), bd0 | ((b_addr + off) >> 4), idesc,
                                 ks > 0 ? 1u : 0u);
                    }
                }
                mma_commit(&sb.b_empty[b]);
                mma_commit(&sb.acc_full[ab]);
                if (++ab == p.nacc) {
                    ab = 0;
                    aph ^= 1u;
                }
            }
            if (!ok || *wd.abort) {
                mma_commit(&sb.drain);
                gt_wait_quiet(&sb.drain, 0, wd.timeout_ns);
                if (!p.starve && ((rt == 1 && !a_tmem) || a_staged)) gt_wait_quiet(&sb.a_ready, 0, wd.timeout_ns);
            }
        }
        __syncwarp();
    } else {
        // ----------------------------------------------------------- epilogue ---
        const int e = warp - kGtMma - 1;            // 0..7
        const int quarter = warp & 3;               // tensor-memory lanes of this warp
        if (a_tmem && e < 4) {
            // A's rows into tensor memory, thread = row of this warp's lane quarter: chunk jj
            // of row r*64 + oc (or oc) is the image's piece (oc, c*Kh + kh) when jj =
            // c*R + kh + r*stride names one, else zero; two chunks (8 columns) per store
            const bool img_ok = !a_staged || mbar_wait(&sb.a_ready, 0, wd, kDevTimeoutFull);
            const int m = quarter * 32 + lane;
            const int ar = rt == 2 ? m >> 6 : 0;
            const int aoc = rt == 2 ? m & 63 : m;
            const uint8_t *img = a_staged ? stage : static_cast<const uint8_t *>(p.w_image);
            const uint32_t taddr = tmem_base + (static_cast<uint32_t>(quarter * 32) << 16) + a_col;
            if (img_ok) {
                int c = 0, khp = 0;                 // chunk jj = c*R + khp
                for (int j = 0; j < nchunks; j += 2) {
                    uint32_t w8[8];
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        const int kh = khp - ar * p.stride;
                        uint4 v = make_uint4(0, 0, 0, 0);
                        if (aoc < p.BN && c < p.C && kh >= 0 && kh < p.Kh) {
                            const uint4 *q = reinterpret_cast<const uint4 *>(img + gt_core(aoc, c * p.Kh + kh, isbo));
                            v = a_staged ? *q : __ldg(q);
                        }
                        w8[4 * h] = v.x;
                        w8[4 * h + 1] = v.y;
                        w8[4 * h + 2] = v.z;
                        w8[4 * h + 3] = v.w;
                        if (++khp == p.R) {
                            khp = 0;
                            ++c;
                        }
                    }
                    tmem_st_x8(taddr + static_cast<uint32_t>(j * 4), w8);
                }
                tmem_st_wait();
            }
            tc_fence_before_sync();
            __syncwarp();
            if (lane == 0) mbar_arrive(&sb.a_tm_ready);
        }
        // lane quarter -> (output row of the tile, output channel)
        const int r = rt == 2 ? quarter >> 1 : 0;
        const int oc = (rt == 2 ? (quarter & 1) * 32 : quarter * 32) + lane;
        const bool staged = p.tma_out != 0;
        // With two output images the epilogue runs as two groups of four warps on alternate
        // tiles (each group its own image, barriers and store), so that one tile's waits
        // overlap the other's work; each warp then drains all columns of its lane quarter.
        // Otherwise all eight warps take every tile, each half of the columns.
        const int ngroups = (staged && p.nout == 2) ? 2 : 1;
        const int gsize = kGtEpi / ngroups;         // warps per group
        const int group = e / gsize;
        int c_lo = 0, c_hi = p.Wo;
        if (ngroups == 1) {
            const int cspan = ((p.Wo + 15) / 16) * 8;   // columns per half, a multiple of 8
            c_lo = (e >> 2) * cspan;
            c_hi = min(p.Wo, c_lo + cspan);
        }
        const bool ch_ok = oc < p.Cout;
        const bool issuer = e % gsize == 0 && lane == 0;    // issues the group's TMA stores
        const int bar_a = 1 + 2 * group, bar_b = 2 + 2 * group;
        const float bv = (ch_ok && p.bias)
                             ? __uint_as_float(static_cast<uint32_t>(static_cast<const unsigned short *>(p.bias)[oc]) << 16)
                             : 0.f;
        const uint32_t lane_base = static_cast<uint32_t>(quarter * 32) << 16;
        int li = group;                             // this CTA's tile count (li-th tile: t)
        for (int t = blockIdx.x + group * static_cast<int>(gridDim.x); t < p.n_mtiles;
             t += ngroups * static_cast<int>(gridDim.x), li += ngroups) {
            const int ab = li % p.nacc;
            const uint32_t aph = static_cast<uint32_t>(li / p.nacc) & 1u;
            const int ob = li % p.nout;             // output image of this tile (the group's own with two)
            bool ok = mbar_wait(&sb.acc_full[ab], aph, wd, kDevTimeoutAccFull);
            if (staged) {
                // this tile's output image was last read by the TMA store of nout tiles
                // back (with two groups: the group's previous store); the group's warps
                // leave together when any wait gave up
                if (issuer) {
                    if (p.nout == 1 || ngroups == 2)
                        bulk_wait_group_read<0>();
                    else
                        bulk_wait_group_read<1>();
                }
                if (!named_barrier_all(bar_a, gsize * 32, ok)) break;
            } else if (!__all_sync(0xffffffffu, ok)) {
                break;
            }
            tc_fence_after_sync();
            const int img = t / tiles_per_img;
            const int oh0 = (t - img * tiles_per_img) * rt;
            const bool valid = ch_ok && oh0 + r < p.Ho;
            if (__any_sync(0xffffffffu, valid) && c_lo < c_hi) {
                // image row (r*BN + oc) of each part; 16-byte chunk k of a row sits at chunk
                // k ^ (row & 7) (the store's 128-byte swizzle): the eight rows a quarter-warp
                // writes at once land in eight different bank groups
                const uint32_t irow = static_cast<uint32_t>(r * p.BN + (valid ? oc : 0));
                uint8_t *orow = out_sm + ob * out_stride + irow * 128u;
                __nv_bfloat16 *yrow = static_cast<__nv_bfloat16 *>(p.y) +
                                      ((static_cast<size_t>(img) * p.Cout + (valid ? oc : 0)) * p.Ho +
                                       (valid ? oh0 + r : 0)) * p.Wo;
                const uint32_t taddr = tmem_base + lane_base + static_cast<uint32_t>(ab * tpix);
                // Up to 64 columns (pixels) per batch: all their loads are issued before one
                // wait, so the tensor-memory latency is paid once per batch, not per 8 columns.
                // c_hi <= Wo <= tpix: no load leaves this accumulator's columns.
                for (int cb = c_lo; cb < c_hi; cb += 64) {
                    uint32_t v[8][8];
#pragma unroll
                    for (int q = 0; q < 8; ++q)
                        if (cb + 8 * q < c_hi) tmem_ld_x8(taddr + static_cast<uint32_t>(cb + 8 * q), v[q]);
                    tmem_ld_wait();
                    if (valid) {
#pragma unroll
                        for (int q = 0; q < 8; ++q) {
                            if (cb + 8 * q < c_hi) {
                                uint32_t pk[4];
#pragma unroll
                                for (int i = 0; i < 4; ++i) {
                                    __nv_bfloat162 h = __floats2bfloat162_rn(__uint_as_float(v[q][2 * i]) + bv,
                                                                             __uint_as_float(v[q][2 * i + 1]) + bv);
                                    pk[i] = *reinterpret_cast<uint32_t *>(&h);
                                }
                                const uint4 v4 = make_uint4(pk[0], pk[1], pk[2], pk[3]);
                                if (staged) {
                                    const int col = cb + 8 * q;
                                    const uint32_t k = static_cast<uint32_t>((col & 63) >> 3);
                                    *reinterpret_cast<uint4 *>(orow + static_cast<uint32_t>(col >> 6) * opart_bytes +
                                                               ((k ^ (irow & 7u)) << 4)) = v4;
                                } else
                                    *reinterpret_cast<uint4 *>(yrow + cb + 8 * q) = v4;
                            }
                        }
                    }
                }
            }
            tc_fence_before_sync();
            __syncwarp();
            if (lane == 0) mbar_arrive(&sb.acc_empty[ab]);
            if (staged) {
                // rows past C_out or Ho of the image are never written: the store clips them
                fence_proxy_async_smem();
                named_barrier(bar_b, gsize * 32);
                if (issuer) {
                    for (int part = 0; part < oparts; ++part)
                        tma_store_4d(&p.tmap_y, out_sm + ob * out_stride + part * opart_bytes, part * 64, 0, oh0, img);
                    bulk_commit_group();
                }
            }
        }
        if (issuer && staged) bulk_wait_group_all();
    }

    tc_fence_before_sync();
    __syncthreads();
    if (warp == kGtMma) {
        tc_fence_after_sync();
        tmem_dealloc(tmem_base, p.tmem_cols);
    }
}

}  // namespace

size_t gather_t_smem_bytes(int kt, int tpix, size_t halo_bytes, int nhalo, size_t out_bytes, int nout, bool a_tmem) {
    auto a1k = [](size_t v) { return (v + 1023) / 1024 * 1024; };
    const size_t sbo = static_cast<size_t>(kt / 8) * 128;
    const size_t b = 2 * a1k(static_cast<size_t>(tpix / 8) * sbo);
    const size_t a = a_tmem ? 0 : a1k(16 * sbo);
    if (a_tmem && b < 16 * sbo) return ~static_cast<size_t>(0);  // A is built in B's space
    return 1024 /* alignment slack */ + kGtHeader + a + b + static_cast<size_t>(nhalo) * a1k(halo_bytes) +
           static_cast<size_t>(nout) * a1k(out_bytes);
}

int gather_t_max_halo() { return kGtMaxHalo; }
int gather_t_max_acc() { return kGtMaxAcc; }
int gather_t_max_chunks() { return kGtMaxChunks; }

cudaError_t launch_gather_t(const GatherParams &p, int grid, size_t smem, cudaStream_t s) {
    const bool rt_ok = p.rt == 1 ? (p.kt == p.Kpad && p.R == p.Kh && p.BN <= 128)
                                 : (p.rt == 2 && p.BN <= 64 && p.R == p.Kh + p.stride && p.kt >= 8 * p.C * p.R);
    if (!rt_ok || p.Kpad > 8 * kGtMaxChunks || p.Kpad % 16 != 0 || p.kt > 8 * kGtMaxChunks || p.kt % 16 != 0 ||
        p.tpix % 16 != 0 || p.tpix > 256 || p.Wo > 256 || p.Wo % 8 != 0 || p.Cout > p.BN ||
        p.C * p.R > kGtMaxChunks || 2 * p.tpix > static_cast<int>(p.tmem_cols) || p.dilation != 1 ||
        p.nhalo < 2 || p.nhalo > kGtMaxHalo || p.nhalo % 2 != 0 || p.nacc < 2 || p.nacc > kGtMaxAcc ||
        p.nacc * p.tpix + (p.a_tmem ? p.kt / 2 : 0) > static_cast<int>(p.tmem_cols) ||
        (p.a_tmem && p.tpix < 64) || (p.tma_out && (p.nout < 1 || p.nout > 2)) ||
        (!p.tma_out && p.nout != 1))
        return cudaErrorInvalidValue;
    cudaError_t e = cudaFuncSetAttribute(gather_t_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    gather_t_kernel<<<grid, kGtThreads, smem, s>>>(p);
    return cudaGetLastError();
}

}  // namespace conv2d_b200
