// gather.cu -- convolutions whose input has too few channels for the hardware
// im2col path: fewer than 32 bytes of channels per pixel, as in the first layer of
// an image network (3 colour channels, "PyTorch高维张量乘法与conv2d/conv3d维度语义解析"
// §6.3 notes that channels-last brings nothing there).  There a hardware im2col
// load moves one narrow pixel row per step, so the tensor memory accelerator, not
// HBM, sets the pace.
//
// This kernel gathers the im2col rows in software instead, straight from x in its
// own layout (NCHW or NHWC, no layout-change pass), and hands them to the tensor
// cores through tensor memory: the A operand of tcgen05.mma is read from tensor
// memory (one tile row per lane), the whole weight matrix (C_out x K) stays
// resident in shared memory as the B operand, fetched by one bulk copy of the image
// the weight pack wrote in exactly that layout.  The reduction index is the compact
// k = (kh*Kw + kw)*C + c, or, for NCHW inputs with 16-byte-aligned rows, the
// row-vector order k = (c*Kh + kh)*8 + kw (bf16; 4 for fp32) whose 16-byte chunks
// are contiguous runs of one input row.  When every 128-pixel tile lies inside one
// image, the rows a tile reads are first staged in shared memory by one TMA box
// load, double-buffered one tile ahead.
//   gather warps (8 for bf16, 4 for fp32): each thread builds (part of) one tile
//                row in registers (8 bf16 or 4 fp32 values, split into tf32 hi/lo,
//                per chunk) and writes it to its tensor-memory lane with tcgen05.st;
//   next warp  : tensor memory allocation and tcgen05.mma issue from one thread;
//   epilogue warps (8 / 4): tcgen05.ld, + bias, round, store (NCHW or NHWC).
// Every wait is bounded (ptx.cuh).
#include <cuda_bf16.h>

#include "common.cuh"
#include "epilogue.cuh"
#include "ptx.cuh"

namespace conv2d_b200 {
namespace {

using namespace ptx;

constexpr int kBM = 128;
// Warp roles: kProd gather warps, one tensor-core warp, kEpi epilogue warps.  bf16
// doubles the gather and epilogue warps (two per tensor-memory lane quarter, each
// taking half of the chunks or columns) to hide latency; fp32 needs more registers.
template <bool kF32> __host__ __device__ constexpr int prod_warps() { return kF32 ? 4 : 8; }
template <bool kF32> __host__ __device__ constexpr int epi_warps() { return kF32 ? 4 : 8; }
template <bool kF32> __host__ __device__ constexpr int threads_for() { return (prod_warps<kF32>() + 1 + epi_warps<kF32>()) * 32; }
constexpr int kMaxStages = 4;        // A slots in tensor memory
constexpr int kHeader = 1024;          // barriers and flags
constexpr int kTableBytes = 4096;      // one int4 per reduction index, up to 256
constexpr int kBiasBytes = 1024;       // fp32 bias of up to 256 output channels

struct SharedBlock {
    uint64_t full[kMaxStages];
    uint64_t empty[kMaxStages];
    uint64_t halo_full[2];
    uint64_t acc_full[2];
    uint64_t acc_empty[2];
    uint64_t b_ready;
    uint64_t drain;
    uint32_t tmem_base;
    int abort;
};
static_assert(sizeof(SharedBlock) <= kHeader, "header too small");

__host__ __device__ inline uint32_t align1k(uint32_t v) { return (v + 1023u) & ~1023u; }

// Byte offset of element (row, k) in the no-swizzle K-major layout: 8-row groups
// `sbo` bytes apart, 16-byte k chunks 128 bytes apart inside a group.
__device__ __forceinline__ uint32_t canon_offset(int row, int chunk, uint32_t sbo) {
    return static_cast<uint32_t>(row >> 3) * sbo + static_cast<uint32_t>(chunk) * 128u +
           static_cast<uint32_t>(row & 7) * 16u;
}

// Picks word (q + i) of w[0..7] for q in [0, 3] without indexing registers at run time.
__device__ __forceinline__ uint32_t pick(const uint32_t (&w)[8], int q, int i) {
    const uint32_t a = w[i], b = w[i + 1], c = w[i + 2], d = w[i + 3];
    return q == 0 ? a : (q == 1 ? b : (q == 2 ? c : d));
}

template <bool kF32>
__global__ void __launch_bounds__(threads_for<kF32>(), 1) gather_kernel(const __grid_constant__ GatherParams p) {
    constexpr int kProd = prod_warps<kF32>();
    constexpr int kEpi = epi_warps<kF32>();
    constexpr int kMmaWarp = kProd;
    constexpr int kElt = kF32 ? 4 : 2;
    constexpr int kPer = 16 / kElt;  // elements per 16-byte chunk (four 32-bit columns)

    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_addr = smem_addr(smem_raw);
    uint8_t *base = smem_raw + (((raw_addr + 1023u) & ~1023u) - raw_addr);
    SharedBlock &sb = *reinterpret_cast<SharedBlock *>(base);
    int4 *table = reinterpret_cast<int4 *>(base + kHeader);
    float *sbias = reinterpret_cast<float *>(base + kHeader + kTableBytes);
    uint8_t *bsm = base + kHeader + kTableBytes + kBiasBytes;
    const uint32_t b_bytes = static_cast<uint32_t>(p.BN) * p.Kpad * kElt;
    uint8_t *bsm_lo = bsm + b_bytes;
    const uint32_t halo_bytes = p.halo ? static_cast<uint32_t>(p.C) * p.R * p.BW * kElt : 0u;
    uint8_t *halo_buf = base + align1k(kHeader + kTableBytes + kBiasBytes + b_bytes * (kF32 ? 2 : 1));
    // tma_out: per epilogue warp two staging buffers of cw x 32 outputs
    uint8_t *stage_out = halo_buf + 2 * align1k(halo_bytes);
    const int nchunks = p.Kpad / kPer;
    const uint32_t sbo = static_cast<uint32_t>(nchunks) * 128u;
    // Tensor memory: accumulators in columns [0, 2*BN), then `stages` A slots of
    // `acols` columns (bf16: two elements per column; fp32: the tf32 hi part, then
    // the lo part from column lo_off).  Every store's first column is a multiple of
    // its width.
    const uint32_t a_first = static_cast<uint32_t>(2 * p.BN);    // a multiple of 32
    const uint32_t acols = static_cast<uint32_t>(p.acols);        // a multiple of 32
    const uint32_t lo_off = static_cast<uint32_t>((p.Kpad + 31) & ~31);  // fp32 lo half

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    // ---------------------------------------------------------------- prologue ---
    if (threadIdx.x == 0) {
        for (int s = 0; s < p.stages; ++s) {
            mbar_init(&sb.full[s], kProd * 32);
            mbar_init(&sb.empty[s], 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&sb.acc_full[i], 1);
            mbar_init(&sb.acc_empty[i], kEpi);
            mbar_init(&sb.halo_full[i], 1);
        }
        mbar_init(&sb.b_ready, 1);
        mbar_init(&sb.drain, 1);
        sb.abort = 0;
        fence_mbar_init();
    }
    // Reduction-index table.  Scalar order, per index k = (kh*Kw + kw)*C + c: the
    // input offset relative to the window's top-left element, row and column tap
    // offsets, and whether k is real.  Row-vector order, per 16-byte chunk
    // j = c*Kh + kh: the offset of row kh*d of channel c (in x, or in the staged
    // rows) relative to the window's first row, and that row's tap offset.
    for (int k = threadIdx.x; k < p.Kpad; k += blockDim.x) {
        int4 e = make_int4(0, 0, 0, 0);
        if (p.vec_rows) {
            if (k < p.C * p.Kh) {
                const int c = k / p.Kh, kh = k - (k / p.Kh) * p.Kh;
                // staged rows: offset in 32-bit words (BW is even, so bf16 rows start on words)
                e.x = p.halo ? (c * p.R + kh * p.dilation) * p.BW / (kF32 ? 1 : 2)
                             : (c * p.H + kh * p.dilation) * p.W;
                e.y = kh * p.dilation;
                e.w = 1;
            }
        } else if (k < p.Kc) {
            const int tap = k / p.C, c = k - (k / p.C) * p.C;
            const int kh = tap / p.Kw, kw = tap - (tap / p.Kw) * p.Kw;
            const int dh = kh * p.dilation, dw = kw * p.dilation;
            e.x = p.in_nchw ? c * p.H * p.W + dh * p.W + dw : (dh * p.W + dw) * p.C + c;
            e.y = dh;
            e.z = dw;
            e.w = 1;
        }
        table[k] = e;
    }
    for (int oc = threadIdx.x; oc < p.BN; oc += blockDim.x) {
        float bv = 0.f;
        if (p.bias && oc < p.Cout)
            bv = kF32 ? static_cast<const float *>(p.bias)[oc]
                      : __bfloat162float(static_cast<const __nv_bfloat16 *>(p.bias)[oc]);
        sbias[oc] = bv;
    }
    if (warp == kMmaWarp) {
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

    if (warp < kProd) {
        // -------------------------------------------------------------- gather ---
        // Thread (warp w, lane l) builds chunks [jb, je) of tile row tid = (w % 4)*32 + l:
        // per 16-byte chunk four 32-bit words, in batches of up to eight chunks that go
        // to its tensor-memory lane with one store (x32 when 32-column aligned, else
        // x8 per chunk pair).
        const int tid = (warp & 3) * 32 + lane;
        const int part = warp >> 2;
        const int half = ((nchunks / (kProd / 4)) + 1) & ~1;  // even split point
        const int jb = part == 0 ? 0 : half;
        const int je = (kProd == 4 || part == 1) ? nchunks : half;
        const uint32_t lane_addr = tmem_base + (static_cast<uint32_t>((warp & 3) * 32) << 16);
        auto build_row = [&](uint32_t slot, auto &&chunk) {
            for (int j0 = jb; j0 < je; j0 += 8) {
                uint32_t hw[32], lw[32];
#pragma unroll
                for (int u = 0; u < 8; ++u)
                    if (j0 + u < je) chunk(j0 + u, &hw[4 * u], &lw[4 * u]);
                const uint32_t col = lane_addr + slot + static_cast<uint32_t>(4 * j0);
                if (j0 + 8 <= je && (j0 & 7) == 0) {
                    tmem_st_x32(col, hw);
                    if constexpr (kF32) tmem_st_x32(col + lo_off, lw);
                } else {  // chunk pairs (every range boundary is even)
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        if (j0 + 2 * q < je) {
                            tmem_st_x8(col + 8 * q, &hw[8 * q]);
                            if constexpr (kF32) tmem_st_x8(col + lo_off + 8 * q, &lw[8 * q]);
                        }
                    }
                }
            }
            tmem_st_wait();
        };
        // fp32 values -> tf32 hi and lo words
        auto split4 = [](const float (&v)[4], uint32_t *h, uint32_t *l) {
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const float hv = tf32_round(v[i]);
                h[i] = __float_as_uint(hv);
                l[i] = __float_as_uint(tf32_round(v[i] - hv));
            }
        };
        const size_t img_elems = static_cast<size_t>(p.C) * p.H * p.W;

        if (p.halo) {
            // Each tile (128 pixels inside one image) reads rows [ih_first, ih_first + R)
            // of every channel, staged in halo buffer (tile % 2) by the tensor-core warp
            // (see there).  Chunk j = c*Kh + kh of this thread's row is the 8 (bf16) or 4
            // (fp32) elements starting at column ow*stride - pad + ME of staged row
            // (c*R + kh*d + (oh - oh_first)*stride); chunks j >= C*Kh are padding.
            const uint32_t hstride = align1k(halo_bytes);
            const int nreal = p.C * p.Kh;
            // bf16: word offsets of this thread's chunks [jb, je) in a staged row, and
            // whether each is a real one (padding chunks read word 0 and are zeroed)
            int cwo[16];
            bool creal[16];
#pragma unroll
            for (int u = 0; u < 16; ++u) {
                const int j = jb + u;
                creal[u] = j < je && j < nreal;
                cwo[u] = creal[u] ? table[j].x : 0;
            }
            int stage = 0, li = 0;
            uint32_t phase = 0;
            for (int t = blockIdx.x; t < p.n_mtiles; t += gridDim.x, ++li) {
                const int b = li & 1;
                const bool ok = mbar_wait(&sb.empty[stage], phase ^ 1u, wd, kDevTimeoutEmpty) &&
                                mbar_wait(&sb.halo_full[b], (li >> 1) & 1, wd, kDevTimeoutFull);
                if (!__all_sync(0xffffffffu, ok)) break;
                const int m0 = t * kBM;
                const int img = m0 / (p.Ho * p.Wo);
                const int r0 = m0 - img * p.Ho * p.Wo;
                const int r = r0 + tid;
                const int oh = r / p.Wo, ow = r - (r / p.Wo) * p.Wo;
                const int ebase = (oh - r0 / p.Wo) * p.stride * p.BW + ow * p.stride - p.pad + p.ME;
                const uint32_t *h32 = reinterpret_cast<const uint32_t *>(halo_buf + b * hstride);
                const uint32_t *hrow = h32 + (kF32 ? ebase : (ebase >> 1));
                const uint32_t sh = (ebase & 1) * 16u;  // bf16: half-word start within the word
                if constexpr (!kF32) {
                    // At most two batches of eight chunks per thread (nchunks <= 32):
                    // all forty word loads of a batch are issued before any is used.
                    const uint32_t slot = lane_addr + a_first + static_cast<uint32_t>(stage) * acols;
#pragma unroll
                    for (int bt = 0; bt < 2; ++bt) {
                        const int j0 = jb + 8 * bt;
                        if (j0 < je) {
                            uint32_t w[8][5];
#pragma unroll
                            for (int u = 0; u < 8; ++u)
#pragma unroll
                                for (int i = 0; i < 5; ++i) w[u][i] = hrow[cwo[8 * bt + u] + i];
                            uint32_t hw[32];
#pragma unroll
                            for (int u = 0; u < 8; ++u)
#pragma unroll
                                for (int i = 0; i < 4; ++i)
                                    hw[4 * u + i] = creal[8 * bt + u] ? __funnelshift_r(w[u][i], w[u][i + 1], sh) : 0u;
                            const uint32_t col = slot + static_cast<uint32_t>(4 * j0);
                            if (j0 + 8 <= je && (j0 & 7) == 0) {
                                tmem_st_x32(col, hw);
                            } else {  // chunk pairs (every range boundary is even)
#pragma unroll
                                for (int q = 0; q < 4; ++q)
                                    if (j0 + 2 * q < je) tmem_st_x8(col + 8 * q, &hw[8 * q]);
                            }
                        }
                    }
                    tmem_st_wait();
                } else
                build_row(a_first + static_cast<uint32_t>(stage) * acols, [&](int j, uint32_t *h, uint32_t *l) {
                    if (j < nreal) {
                        const int wo = table[j].x;
                        if constexpr (kF32) {
                            float v[4];
#pragma unroll
                            for (int i = 0; i < 4; ++i) v[i] = __uint_as_float(hrow[wo + i]);
                            split4(v, h, l);
                        } else {
                            uint32_t w[5];
#pragma unroll
                            for (int i = 0; i < 5; ++i) w[i] = hrow[wo + i];
#pragma unroll
                            for (int i = 0; i < 4; ++i) h[i] = __funnelshift_r(w[i], w[i + 1], sh);
                        }
                    } else {
#pragma unroll
                        for (int i = 0; i < 4; ++i) h[i] = l[i] = 0u;
                    }
                });
                tc_fence_before_sync();
                if (!p.starve) mbar_arrive(&sb.full[stage]);
                if (++stage == p.stages) {
                    stage = 0;
                    phase ^= 1u;
                }
            }
        } else {
            int stage = 0;
            uint32_t phase = 0;
            for (int t = blockIdx.x; t < p.n_mtiles; t += gridDim.x) {
                const bool ok = mbar_wait(&sb.empty[stage], phase ^ 1u, wd, kDevTimeoutEmpty);
                if (!__all_sync(0xffffffffu, ok)) break;
                const int m = t * kBM + tid;
                const bool valid = m < p.M;
                int n = 0, oh = 0, ow = 0;
                if (valid) {
                    n = m / (p.Ho * p.Wo);
                    const int r = m - n * p.Ho * p.Wo;
                    oh = r / p.Wo;
                    ow = r - oh * p.Wo;
                }
                const int ih0 = oh * p.stride - p.pad, iw0 = ow * p.stride - p.pad;
                const uint32_t slot = a_first + static_cast<uint32_t>(stage) * acols;
                if (p.vec_rows) {
                    // NCHW rows 16-byte aligned, unit column dilation: chunk j = c*Kh + kh is
                    // the kPer elements [iw0, iw0 + kPer) of row ih0 + kh*d of channel c, from
                    // the two aligned 16-byte words that cover them.  A word lies wholly inside
                    // or wholly outside the row, so words outside read as zero and the zero
                    // padding needs no per-element test; slots kw >= Kw meet zero weights.
                    const int aligned = iw0 & ~(kPer - 1);
                    const int o = iw0 - aligned;
                    const bool in0 = aligned >= 0 && aligned + kPer <= p.W;
                    const bool in1 = aligned + kPer >= 0 && aligned + 2 * kPer <= p.W;
                    const long long img_base = static_cast<long long>(n) * img_elems;
                    build_row(slot, [&](int j, uint32_t *h, uint32_t *l) {
                        const int4 te = table[j];
                        const int ih = ih0 + te.y;
                        uint4 lo = make_uint4(0, 0, 0, 0), hi = lo;
                        if (valid && te.w && static_cast<unsigned>(ih) < static_cast<unsigned>(p.H)) {
                            const long long e0 = img_base + te.x + static_cast<long long>(ih0) * p.W + aligned;
                            const uint4 *src = reinterpret_cast<const uint4 *>(static_cast<const uint8_t *>(p.x) + e0 * kElt);
                            if (in0) lo = __ldg(src);
                            if (in1) hi = __ldg(src + 1);
                        }
                        const uint32_t w[8] = {lo.x, lo.y, lo.z, lo.w, hi.x, hi.y, hi.z, hi.w};
                        if constexpr (kF32) {
                            float v[4];
#pragma unroll
                            for (int i = 0; i < 4; ++i) v[i] = __uint_as_float(pick(w, o, i));
                            split4(v, h, l);
                        } else {
                            const int q = o >> 1;
                            const uint32_t sh = (o & 1) * 16u;
#pragma unroll
                            for (int i = 0; i < 4; ++i) h[i] = __funnelshift_r(pick(w, q, i), pick(w, q, i + 1), sh);
                        }
                    });
                } else {
                    const long long row_base =
                        static_cast<long long>(n) * img_elems +
                        (p.in_nchw ? static_cast<long long>(ih0) * p.W + iw0
                                   : (static_cast<long long>(ih0) * p.W + iw0) * p.C);
                    build_row(slot, [&](int j, uint32_t *h, uint32_t *l) {
                        if constexpr (kF32) {
                            const float *xs = static_cast<const float *>(p.x);
                            float v[4];
#pragma unroll
                            for (int e = 0; e < 4; ++e) {
                                const int4 te = table[j * 4 + e];
                                const int ih = ih0 + te.y, iw = iw0 + te.z;
                                v[e] = (valid && te.w && static_cast<unsigned>(ih) < static_cast<unsigned>(p.H) &&
                                        static_cast<unsigned>(iw) < static_cast<unsigned>(p.W))
                                           ? __ldg(xs + (row_base + te.x))
                                           : 0.f;
                            }
                            split4(v, h, l);
                        } else {
                            const unsigned short *xs = static_cast<const unsigned short *>(p.x);
#pragma unroll
                            for (int e = 0; e < 4; ++e) {
                                uint32_t pair = 0;
#pragma unroll
                                for (int hh = 0; hh < 2; ++hh) {
                                    const int4 te = table[j * 8 + e * 2 + hh];
                                    const int ih = ih0 + te.y, iw = iw0 + te.z;
                                    const uint32_t v =
                                        (valid && te.w && static_cast<unsigned>(ih) < static_cast<unsigned>(p.H) &&
                                         static_cast<unsigned>(iw) < static_cast<unsigned>(p.W))
                                            ? __ldg(xs + (row_base + te.x))
                                            : 0u;
                                    pair |= v << (16 * hh);
                                }
                                h[e] = pair;
                            }
                        }
                    });
                }
                tc_fence_before_sync();
                if (!p.starve) mbar_arrive(&sb.full[stage]);
                if (++stage == p.stages) {
                    stage = 0;
                    phase ^= 1u;
                }
            }
        }
    } else if (warp == kMmaWarp) {
        // --------------------------------------------------- tensor-core issue ---
        if (lane == 0) {
            const uint32_t idesc = instr_desc(kF32 ? 2u : 1u, kBM, static_cast<uint32_t>(p.BN));
            const uint32_t b_hi = smem_addr(bsm), b_lo = smem_addr(bsm_lo);
            const int ksteps = p.Kpad * kElt / 32;  // 32 bytes of k per instruction
            int stage = 0, abuf = 0;
            uint32_t phase = 0, aphase = 0;
            bool ok = true;
            // Staged input rows: tile li reads halo buffer li % 2.  Loads go two tiles
            // ahead; the gather warps' arrival for tile li (full[stage]) also means they
            // are done with its buffer, which then takes tile li + 2.
            const uint32_t hstride = align1k(halo_bytes);
            int issued0 = 0, issued1 = 0;
            auto issue_halo = [&](int t, int b) {
                const int m0 = t * kBM;
                const int img = m0 / (p.Ho * p.Wo);
                const int oh0 = (m0 - img * p.Ho * p.Wo) / p.Wo;
                if (b == 0) ++issued0; else ++issued1;
                mbar_arrive_expect_tx(&sb.halo_full[b], halo_bytes);
                tma_load_4d(halo_buf + b * hstride, &p.tmap_x, &sb.halo_full[b], -p.ME,
                            oh0 * p.stride - p.pad, 0, img);
            };
            if (p.halo && !p.starve) {
                prefetch_tensormap(&p.tmap_x);
                for (int k = 0; k < 2; ++k)
                    if (blockIdx.x + k * static_cast<int>(gridDim.x) < p.n_mtiles)
                        issue_halo(blockIdx.x + k * gridDim.x, k);
            }
            // The weight image (written by the weight pack in this layout) arrives by one
            // bulk copy while the gather warps build the first tile.
            if (!p.starve) {
                const uint32_t img_bytes = b_bytes * (kF32 ? 2u : 1u);
                mbar_arrive_expect_tx(&sb.b_ready, img_bytes);
                bulk_load(bsm, p.w_image, img_bytes, &sb.b_ready);
            }
            if (!mbar_wait(&sb.b_ready, 0, wd, kDevTimeoutFull)) ok = false;
            int li = 0;
            for (int t = blockIdx.x; ok && t < p.n_mtiles; t += gridDim.x, ++li) {
                if (!mbar_wait(&sb.acc_empty[abuf], aphase ^ 1u, wd, kDevTimeoutAccEmpty) ||
                    !mbar_wait(&sb.full[stage], phase, wd, kDevTimeoutFull)) {
                    ok = false;
                    break;
                }
                tc_fence_after_sync();
                const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(abuf * p.BN);
                const uint32_t a_hi = tmem_base + a_first + static_cast<uint32_t>(stage) * acols;
                const uint32_t a_lo = a_hi + lo_off;
                for (int ks = 0; ks < ksteps; ++ks) {
                    const uint32_t boff = static_cast<uint32_t>(ks) * 256u;  // two 16-byte chunks
                    const uint32_t aoff = static_cast<uint32_t>(ks) * 8u;    // eight 32-bit columns
                    const uint32_t acc = ks > 0 ? 1u : 0u;
                    if constexpr (kF32) {
                        mma_tf32_tmem_a(d_tmem, a_lo + aoff, smem_desc(b_hi + boff, 128, sbo, kSwNone), idesc, acc);
                        mma_tf32_tmem_a(d_tmem, a_hi + aoff, smem_desc(b_lo + boff, 128, sbo, kSwNone), idesc, 1u);
                        mma_tf32_tmem_a(d_tmem, a_hi + aoff, smem_desc(b_hi + boff, 128, sbo, kSwNone), idesc, 1u);
                    } else {
                        mma_bf16_tmem_a(d_tmem, a_hi + aoff, smem_desc(b_hi + boff, 128, sbo, kSwNone), idesc, acc);
                    }
                }
                mma_commit(&sb.empty[stage]);
                mma_commit(&sb.acc_full[abuf]);
                // The gather warps are done with this tile's staged rows (they arrived
                // on full[stage]), so its buffer takes tile t + 2; issued after the
                // products so that they are not held up by the address arithmetic.
                const int t2 = t + 2 * static_cast<int>(gridDim.x);
                if (p.halo && !p.starve && t2 < p.n_mtiles) issue_halo(t2, li & 1);
                if (++stage == p.stages) {
                    stage = 0;
                    phase ^= 1u;
                }
                abuf ^= 1;
                if (abuf == 0) aphase ^= 1u;
            }
            if (!ok || *wd.abort) {
                mma_commit(&sb.drain);
                const uint64_t start = globaltimer_ns();
                while (!mbar_try_wait(&sb.drain, 0) && globaltimer_ns() - start < wd.timeout_ns) {
                }
                {  // the weight image copy, if it is still in flight
                    const uint64_t t0 = globaltimer_ns();
                    while (!p.starve && !mbar_try_wait(&sb.b_ready, 0) && globaltimer_ns() - t0 < wd.timeout_ns) {
                    }
                }
                for (int b = 0; b < 2; ++b) {  // let the halo loads still in flight land
                    const int n_issued = b == 0 ? issued0 : issued1;
                    if (n_issued == 0) continue;
                    const uint32_t parity = static_cast<uint32_t>(n_issued - 1) & 1u;
                    const uint64_t t0 = globaltimer_ns();
                    while (!mbar_try_wait(&sb.halo_full[b], parity) && globaltimer_ns() - t0 < wd.timeout_ns) {
                    }
                }
            }
        }
        __syncwarp();
    } else {
        // ------------------------------------------------------------ epilogue ---
        // Warp e of the epilogue reads lane quarter (warp % 4) and column block e / 4.
        const int quarter = warp & 3;
        const int row = quarter * 32 + lane;
        const int eb = (warp - kMmaWarp - 1) >> 2;
        const int cw = (kEpi == 4) ? p.BN : ((p.BN / 2 + 15) & ~15);
        const int cb0 = eb * cw;
        const int cb1 = min(p.BN, cb0 + cw);
        const uint32_t lane_base = static_cast<uint32_t>(quarter * 32) << 16;
        OutDesc out;
        out.y = p.y;
        out.bias = nullptr;  // added from shared memory below
        out.M = p.M;
        out.HoWo = p.Ho * p.Wo;
        out.Cout = p.Cout;
        out.Cout_g = p.Cout;
        out.out_mode = p.out_mode;
        out.vec_ok = p.vec_ok;
        int abuf = 0;
        uint32_t aphase = 0;
        if constexpr (!kF32) {
            if (p.tma_out) {
                // Tiles lie inside one image: each warp writes its 32 rows (pixels) x
                // columns [cb0, cb1) channel-major into its own staging buffer and
                // stores them with one TMA box store (y seen as (Ho*Wo, C_out, N));
                // columns past C_out are clipped by the TMA.
                const bool active = cb0 < p.BN;
                const uint32_t wstride = static_cast<uint32_t>(p.cw) * 32u * kElt;
                uint8_t *wstage = stage_out + (warp - kMmaWarp - 1) * 2 * wstride;
                int sbi = 0;
                if (cb1 - cb0 == 32) {
                    // A full 32-channel block (the first-layer shape): its biases stay in
                    // registers, and lanes swap values in pairs so that each thread writes
                    // whole 32-bit words (two pixels of one channel) into the
                    // channel-major staging buffer: half the conversions and stores.
                    uint32_t bsel[16];  // bf16 biases (exact: they came from bf16), two per word
#pragma unroll
                    for (int i = 0; i < 16; ++i) {
                        __nv_bfloat162 b2 = __floats2bfloat162_rn(sbias[cb0 + 2 * i], sbias[cb0 + 2 * i + 1]);
                        bsel[i] = *reinterpret_cast<uint32_t *>(&b2);
                    }
                    const bool odd = (lane & 1) != 0;
                    for (int t = blockIdx.x; t < p.n_mtiles; t += gridDim.x) {
                        const bool ok = mbar_wait(&sb.acc_full[abuf], aphase, wd, kDevTimeoutAccFull);
                        if (!__all_sync(0xffffffffu, ok)) break;
                        tc_fence_after_sync();
                        const uint32_t taddr = tmem_base + lane_base + static_cast<uint32_t>(abuf * p.BN + cb0);
                        uint32_t r[2][16];
                        tmem_ld_x16(taddr, r[0]);
                        tmem_ld_x16(taddr + 16u, r[1]);
                        tmem_ld_wait();
                        tc_fence_before_sync();
                        __syncwarp();
                        if (lane == 0) mbar_arrive(&sb.acc_empty[abuf]);
                        abuf ^= 1;
                        if (abuf == 0) aphase ^= 1u;
                        if (lane == 0) bulk_wait_group_read<1>();  // this buffer's previous store has read it
                        __syncwarp();
                        uint32_t *stg32 = reinterpret_cast<uint32_t *>(wstage + sbi * wstride);
#pragma unroll
                        for (int k = 0; k < 16; ++k) {
                            const float v0 = __uint_as_float(r[k >> 3][(2 * k) & 15]) + __uint_as_float(bsel[k] << 16);
                            const float v1 = __uint_as_float(r[k >> 3][(2 * k + 1) & 15]) +
                                             __uint_as_float(bsel[k] & 0xFFFF0000u);
                            // even lane (pixel 2w): channel 2k of pixels 2w, 2w+1;
                            // odd lane (pixel 2w+1): channel 2k+1 of pixels 2w, 2w+1
                            const float recv = __shfl_xor_sync(0xffffffffu, odd ? v0 : v1, 1);
                            __nv_bfloat162 h = odd ? __floats2bfloat162_rn(recv, v1) : __floats2bfloat162_rn(v0, recv);
                            stg32[(2 * k + (odd ? 1 : 0)) * 16 + (lane >> 1)] = *reinterpret_cast<uint32_t *>(&h);
                        }
                        fence_proxy_async_smem();
                        __syncwarp();
                        if (lane == 0) {
                            const int m0 = t * kBM;
                            const int img = m0 / (p.Ho * p.Wo);
                            tma_store_3d(&p.tmap_y, stg32, m0 - img * p.Ho * p.Wo + quarter * 32, cb0, img);
                            bulk_commit_group();
                        }
                        sbi ^= 1;
                    }
                }
                for (int t = blockIdx.x; t < p.n_mtiles && cb1 - cb0 != 32; t += gridDim.x) {
                    const bool ok = mbar_wait(&sb.acc_full[abuf], aphase, wd, kDevTimeoutAccFull);
                    if (!__all_sync(0xffffffffu, ok)) break;
                    tc_fence_after_sync();
                    const uint32_t taddr = tmem_base + lane_base + static_cast<uint32_t>(abuf * p.BN);
                    uint32_t r[4][16];
#pragma unroll
                    for (int q = 0; q < 4; ++q)
                        if (cb0 + q * 16 < cb1) tmem_ld_x16(taddr + static_cast<uint32_t>(cb0 + q * 16), r[q]);
                    tmem_ld_wait();
                    tc_fence_before_sync();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&sb.acc_empty[abuf]);
                    abuf ^= 1;
                    if (abuf == 0) aphase ^= 1u;
                    if (!active) continue;
                    if (lane == 0) bulk_wait_group_read<1>();  // this buffer's previous store has read it
                    __syncwarp();
                    uint16_t *stg = reinterpret_cast<uint16_t *>(wstage + sbi * wstride);
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        if (cb0 + q * 16 < cb1) {
#pragma unroll
                            for (int i = 0; i < 16; ++i) {
                                const int lc = q * 16 + i;
                                __nv_bfloat16 h = __float2bfloat16_rn(__uint_as_float(r[q][i]) + sbias[cb0 + lc]);
                                stg[lc * 32 + lane] = *reinterpret_cast<uint16_t *>(&h);
                            }
                        }
                    }
                    fence_proxy_async_smem();
                    __syncwarp();
                    if (lane == 0) {
                        const int m0 = t * kBM;
                        const int img = m0 / (p.Ho * p.Wo);
                        tma_store_3d(&p.tmap_y, stg, m0 - img * p.Ho * p.Wo + quarter * 32, cb0, img);
                        bulk_commit_group();
                    }
                    sbi ^= 1;
                }
                if (lane == 0 && active) bulk_wait_group_all();
            }
        }
        for (int t = blockIdx.x; t < p.n_mtiles && !(!kF32 && p.tma_out); t += gridDim.x) {
            const bool ok = mbar_wait(&sb.acc_full[abuf], aphase, wd, kDevTimeoutAccFull);
            if (!__all_sync(0xffffffffu, ok)) break;
            tc_fence_after_sync();
            const int m = t * kBM + row;
            const uint32_t taddr = tmem_base + lane_base + static_cast<uint32_t>(abuf * p.BN);
            for (int c0 = cb0; c0 < cb1; c0 += 64) {
                uint32_t r[4][16];
#pragma unroll
                for (int q = 0; q < 4; ++q)
                    if (c0 + q * 16 < cb1) tmem_ld_x16(taddr + static_cast<uint32_t>(c0 + q * 16), r[q]);
                tmem_ld_wait();
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    if (c0 + q * 16 < cb1) {
                        const float4 *b4 = reinterpret_cast<const float4 *>(sbias + c0 + q * 16);
                        float v[16];
#pragma unroll
                        for (int i = 0; i < 4; ++i) {
                            const float4 bb = b4[i];
                            v[4 * i + 0] = __uint_as_float(r[q][4 * i + 0]) + bb.x;
                            v[4 * i + 1] = __uint_as_float(r[q][4 * i + 1]) + bb.y;
                            v[4 * i + 2] = __uint_as_float(r[q][4 * i + 2]) + bb.z;
                            v[4 * i + 3] = __uint_as_float(r[q][4 * i + 3]) + bb.w;
                        }
                        store16<kF32>(out, m, 0, c0 + q * 16, 0, v);
                    }
                }
            }
            tc_fence_before_sync();
            __syncwarp();
            if (lane == 0) mbar_arrive(&sb.acc_empty[abuf]);
            abuf ^= 1;
            if (abuf == 0) aphase ^= 1u;
        }
    }

    tc_fence_before_sync();
    __syncthreads();
    if (warp == kMmaWarp) {
        tc_fence_after_sync();
        tmem_dealloc(tmem_base, p.tmem_cols);
    }
}

}  // namespace

size_t gather_smem_bytes(bool f32, int BN, int Kpad, size_t halo_bytes, size_t out_stage_bytes) {
    const int elt = f32 ? 4 : 2;
    const uint32_t b = static_cast<uint32_t>(BN) * Kpad * elt * (f32 ? 2 : 1);
    return 1024 /* alignment slack */ + align1k(kHeader + kTableBytes + kBiasBytes + b) +
           2 * static_cast<size_t>(align1k(static_cast<uint32_t>(halo_bytes))) +
           4 * static_cast<size_t>(align1k(static_cast<uint32_t>(out_stage_bytes)));
}

int gather_max_stages() { return kMaxStages; }

cudaError_t launch_gather(const GatherParams &p, bool f32, int grid, size_t smem, cudaStream_t s) {
    if (p.stages < 2 || p.stages > kMaxStages || p.Kpad > kTableBytes / 16 ||
        2 * p.BN + p.stages * p.acols > static_cast<int>(p.tmem_cols))
        return cudaErrorInvalidValue;
    auto kern = f32 ? gather_kernel<true> : gather_kernel<false>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    kern<<<grid, f32 ? threads_for<true>() : threads_for<false>(), smem, s>>>(p);
    return cudaGetLastError();
}

}  // namespace conv2d_b200
