// gather.cu -- convolutions whose input has too few channels for the hardware
// im2col path: fewer than 32 bytes of channels per pixel, as in the first layer of
// an image network (3 colour channels, "PyTorch高维张量乘法与conv2d/conv3d维度语义解析"
// §6.3 notes that channels-last brings nothing there).  There a hardware im2col
// load moves one narrow pixel row per step, so the tensor memory accelerator, not
// HBM, sets the pace.
//
// This kernel gathers the im2col rows in software instead, straight from x in its
// own layout (NCHW or NHWC, no layout-change pass): the reduction index is the
// compact k = (kh*Kw + kw)*C + c, padded only to the tensor-core step, and the
// whole weight matrix (C_out x K) stays resident in shared memory.  The product is
// the same one as in igemm.cu (rows = output pixels, columns = output channels):
//   warps 0..3 : gather -- each thread builds one 128-row tile row per stage, eight
//                (bf16) or four (fp32, split into tf32 hi/lo) k values per 16-byte
//                shared-memory store, in the tensor cores' no-swizzle K-major layout;
//   warp 4     : tensor memory allocation and tcgen05.mma issue from one thread;
//   warps 5..8 : epilogue -- tcgen05.ld, + bias, round, store (NCHW or NHWC).
// Every wait is bounded (ptx.cuh).
#include <cuda_bf16.h>

#include "common.cuh"
#include "epilogue.cuh"
#include "ptx.cuh"

namespace conv2d_b200 {
namespace {

using namespace ptx;

constexpr int kBM = 128;
constexpr int kMmaWarp = 4;
constexpr int kEpiWarp0 = 5;
constexpr int kThreads = 9 * 32;
constexpr int kMaxStages = 8;
constexpr int kHeader = 1024;          // barriers and flags
constexpr int kTableBytes = 4096;      // one int4 per reduction index, up to 256
constexpr int kBiasBytes = 1024;       // fp32 bias of up to 256 output channels

struct SharedBlock {
    uint64_t full[kMaxStages];
    uint64_t empty[kMaxStages];
    uint64_t halo_full[2];
    uint64_t halo_empty[2];
    uint64_t acc_full[2];
    uint64_t acc_empty[2];
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

// Row-vector gather for NCHW inputs with 16-byte-aligned rows and unit column
// dilation: chunk j = c*Kh + kh of a tile row is the kPer input elements
// [iw0, iw0 + kPer) of row ih0 + kh*d of channel c, taken from the two aligned
// 16-byte words that cover it.  A word lies wholly inside or wholly outside the
// row, so words outside are zero and the zero padding needs no per-element test;
// window slots kw >= Kw meet zero weights.
template <bool kF32>
__device__ __forceinline__ void gather_rows(const GatherParams &p, const int4 *table, uint8_t *arow,
                                            uint32_t a_bytes, int nchunks, bool valid,
                                            long long img_base, int ih0, int iw0) {
    constexpr int kPer = kF32 ? 4 : 8;
    const int aligned = iw0 & ~(kPer - 1);  // floor to a word boundary (also for iw0 < 0)
    const int o = iw0 - aligned;            // first element inside the two words
    const bool in0 = aligned >= 0 && aligned + kPer <= p.W;
    const bool in1 = aligned + kPer >= 0 && aligned + 2 * kPer <= p.W;
    const unsigned short *x16 = static_cast<const unsigned short *>(p.x);
    const float *x32 = static_cast<const float *>(p.x);
    for (int j0 = 0; j0 < nchunks; j0 += 4) {
        uint4 lo[4], hi[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            lo[u] = hi[u] = make_uint4(0, 0, 0, 0);
            const int j = j0 + u;
            if (j < nchunks) {
                const int4 te = table[j];
                const int ih = ih0 + te.y;
                if (valid && te.w && static_cast<unsigned>(ih) < static_cast<unsigned>(p.H)) {
                    const long long e0 = img_base + te.x + static_cast<long long>(ih0) * p.W + aligned;
                    const uint4 *src = kF32 ? reinterpret_cast<const uint4 *>(x32 + e0)
                                            : reinterpret_cast<const uint4 *>(x16 + e0);
                    if (in0) lo[u] = __ldg(src);
                    if (in1) hi[u] = __ldg(src + 1);
                }
            }
        }
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const int j = j0 + u;
            if (j >= nchunks) break;
            const uint32_t w[8] = {lo[u].x, lo[u].y, lo[u].z, lo[u].w, hi[u].x, hi[u].y, hi[u].z, hi[u].w};
            if constexpr (kF32) {  // four fp32 elements starting at word o
                float v[4];
#pragma unroll
                for (int i = 0; i < 4; ++i) v[i] = __uint_as_float(pick(w, o, i));
                float4 h, l;
                h.x = tf32_round(v[0]); l.x = tf32_round(v[0] - h.x);
                h.y = tf32_round(v[1]); l.y = tf32_round(v[1] - h.y);
                h.z = tf32_round(v[2]); l.z = tf32_round(v[2] - h.z);
                h.w = tf32_round(v[3]); l.w = tf32_round(v[3] - h.w);
                *reinterpret_cast<float4 *>(arow + j * 128) = h;
                *reinterpret_cast<float4 *>(arow + a_bytes + j * 128) = l;
            } else {  // eight bf16 elements starting at half-word o
                const int q = o >> 1;
                const uint32_t sh = (o & 1) * 16u;
                uint32_t r[4];
#pragma unroll
                for (int i = 0; i < 4; ++i) r[i] = __funnelshift_r(pick(w, q, i), pick(w, q, i + 1), sh);
                *reinterpret_cast<uint4 *>(arow + j * 128) = make_uint4(r[0], r[1], r[2], r[3]);
            }
        }
    }
}

template <bool kF32>
__global__ void __launch_bounds__(kThreads, 1) gather_kernel(const __grid_constant__ GatherParams p) {
    constexpr int kElt = kF32 ? 4 : 2;
    constexpr int kPer = 16 / kElt;  // elements per 16-byte chunk

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
    uint8_t *ring = halo_buf + 2 * align1k(halo_bytes);
    const uint32_t a_bytes = static_cast<uint32_t>(kBM) * p.Kpad * kElt;
    const uint32_t sbytes = a_bytes * (kF32 ? 2 : 1);
    const int nchunks = p.Kpad / kPer;
    const uint32_t sbo = static_cast<uint32_t>(nchunks) * 128u;

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    // ---------------------------------------------------------------- prologue ---
    if (threadIdx.x == 0) {
        for (int s = 0; s < p.stages; ++s) {
            mbar_init(&sb.full[s], 128);
            mbar_init(&sb.empty[s], 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&sb.acc_full[i], 1);
            mbar_init(&sb.acc_empty[i], 4);
            mbar_init(&sb.halo_full[i], 1);
            mbar_init(&sb.halo_empty[i], 128);
        }
        mbar_init(&sb.drain, 1);
        sb.abort = 0;
        fence_mbar_init();
    }
    // Scalar order: per reduction index k = (kh*Kw + kw)*C + c, the input offset
    // relative to the window's top-left element, the row and column tap offsets,
    // and whether the index is real (not padding).
    // Row-vector order: per 16-byte chunk j = c*Kh + kh, the offset of row kh*d of
    // channel c relative to the window's first row, and that row's tap offset.
    for (int k = threadIdx.x; k < p.Kpad; k += blockDim.x) {
        int4 e = make_int4(0, 0, 0, 0);
        if (p.vec_rows) {
            if (k < p.C * p.Kh) {
                const int c = k / p.Kh, kh = k - (k / p.Kh) * p.Kh;
                e.x = p.halo ? (c * p.R + kh * p.dilation) * p.BW : (c * p.H + kh * p.dilation) * p.W;
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
    // The whole weight matrix in the same reduction order, zero where k is padding.
    const int taps = p.Kh * p.Kw;
    for (int i = threadIdx.x; i < p.BN * p.Kpad; i += blockDim.x) {
        const int oc = i / p.Kpad, k = i - (i / p.Kpad) * p.Kpad;
        const uint32_t off = canon_offset(oc, k / kPer, sbo) + static_cast<uint32_t>(k % kPer) * kElt;
        int c, tap;
        bool real = oc < p.Cout;
        if (p.vec_rows) {  // k = (c*Kh + kh)*kPer + kw
            const int j = k / kPer, kw = k - j * kPer;
            c = j / p.Kh;
            tap = (j - c * p.Kh) * p.Kw + kw;
            real = real && j < p.C * p.Kh && kw < p.Kw;
        } else {           // k = (kh*Kw + kw)*C + c
            tap = k / p.C;
            c = k - tap * p.C;
            real = real && k < p.Kc;
        }
        const size_t src = real ? (static_cast<size_t>(oc) * taps + tap) * p.Cpg + c : 0;
        if constexpr (kF32) {
            const float v = real ? __ldg(static_cast<const float *>(p.w_packed) + src) : 0.f;
            const float hi = tf32_round(v);
            *reinterpret_cast<float *>(bsm + off) = hi;
            *reinterpret_cast<float *>(bsm_lo + off) = tf32_round(v - hi);
        } else {
            const uint16_t v = real ? __ldg(static_cast<const unsigned short *>(p.w_packed) + src) : 0;
            *reinterpret_cast<uint16_t *>(bsm + off) = v;
        }
    }
    fence_proxy_async_smem();
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

    if (warp < 4 && p.halo) {
        // ------------------------------------- gather from TMA-staged input rows ---
        // Each tile (128 pixels inside one image) needs rows [ih_first, ih_first + R)
        // of every channel; one TMA box load brings them, with ME zero columns on the
        // left and zeros past the right edge and outside the image (TMA fills), into
        // one of two halo buffers.  Thread 0 issues the load for the next tile before
        // the threads gather the current one.
        const int tid = threadIdx.x;
        const uint32_t hstride = align1k(halo_bytes);
        auto tile_origin = [&](int t, int &img, int &oh_first) {
            const int m0 = t * kBM;
            img = m0 / (p.Ho * p.Wo);
            oh_first = (m0 - img * p.Ho * p.Wo) / p.Wo;
        };
        int issued0 = 0, issued1 = 0;  // halo loads issued per buffer (thread 0)
        auto issue_halo = [&](int t, int b) {
            int img, oh0;
            tile_origin(t, img, oh0);
            if (b == 0) ++issued0; else ++issued1;
            mbar_arrive_expect_tx(&sb.halo_full[b], halo_bytes);
            tma_load_4d(halo_buf + b * hstride, &p.tmap_x, &sb.halo_full[b], -p.ME,
                        oh0 * p.stride - p.pad, 0, img);
        };
        if (tid == 0) prefetch_tensormap(&p.tmap_x);
        if (tid == 0 && blockIdx.x < p.n_mtiles && !p.starve) issue_halo(blockIdx.x, 0);
        int stage = 0;
        uint32_t phase = 0;
        int li = 0;
        for (int t = blockIdx.x; t < p.n_mtiles; t += gridDim.x, ++li) {
            const int b = li & 1;
            if (tid == 0 && t + static_cast<int>(gridDim.x) < p.n_mtiles && !p.starve) {
                // the other buffer was last read for tile li - 1
                if (li >= 1 && !mbar_wait(&sb.halo_empty[b ^ 1], ((li - 1) >> 1) & 1, wd, kDevTimeoutEmpty))
                    break;
                issue_halo(t + gridDim.x, b ^ 1);
            }
            if (!mbar_wait(&sb.empty[stage], phase ^ 1u, wd, kDevTimeoutEmpty)) break;
            if (!mbar_wait(&sb.halo_full[b], (li >> 1) & 1, wd, kDevTimeoutFull)) break;
            int img, oh0;
            tile_origin(t, img, oh0);
            const int m = t * kBM + tid;
            const int r = m - img * p.Ho * p.Wo;
            const int oh = r / p.Wo, ow = r - (r / p.Wo) * p.Wo;
            const int ebase = (oh - oh0) * p.stride * p.BW + ow * p.stride - p.pad + p.ME;
            const uint32_t *h32 = reinterpret_cast<const uint32_t *>(halo_buf + b * hstride);
            uint8_t *arow = ring + static_cast<size_t>(stage) * sbytes + canon_offset(tid, 0, sbo);
            // Batches of chunks: all shared-memory reads of a batch are issued before
            // its stores, so they overlap instead of queuing behind each store.
            constexpr int kBatch = 8;
            for (int j0 = 0; j0 < nchunks; j0 += kBatch) {
                uint32_t wv[kBatch][5];
                uint32_t shift[kBatch];
                bool live[kBatch];
#pragma unroll
                for (int u = 0; u < kBatch; ++u) {
                    const int j = j0 + u;
                    live[u] = false;
                    shift[u] = 0;
                    if (j < nchunks) {
                        const int4 te = table[j];
                        const int e = ebase + te.x;  // a valid index even for padding chunks
                        live[u] = te.w != 0;
                        if constexpr (kF32) {
#pragma unroll
                            for (int i = 0; i < 4; ++i) wv[u][i] = h32[e + i];
                        } else {
                            const int wi = e >> 1;
                            shift[u] = (e & 1) * 16u;
#pragma unroll
                            for (int i = 0; i < 5; ++i) wv[u][i] = h32[wi + i];
                        }
                    }
                }
#pragma unroll
                for (int u = 0; u < kBatch; ++u) {
                    const int j = j0 + u;
                    if (j >= nchunks) break;
                    if constexpr (kF32) {
                        float4 h = make_float4(0.f, 0.f, 0.f, 0.f), l = h;
                        if (live[u]) {
                            const float v0 = __uint_as_float(wv[u][0]), v1 = __uint_as_float(wv[u][1]);
                            const float v2 = __uint_as_float(wv[u][2]), v3 = __uint_as_float(wv[u][3]);
                            h.x = tf32_round(v0); l.x = tf32_round(v0 - h.x);
                            h.y = tf32_round(v1); l.y = tf32_round(v1 - h.y);
                            h.z = tf32_round(v2); l.z = tf32_round(v2 - h.z);
                            h.w = tf32_round(v3); l.w = tf32_round(v3 - h.w);
                        }
                        *reinterpret_cast<float4 *>(arow + j * 128) = h;
                        *reinterpret_cast<float4 *>(arow + a_bytes + j * 128) = l;
                    } else {
                        uint4 out = make_uint4(0, 0, 0, 0);
                        if (live[u]) {
                            const uint32_t sh = shift[u];
                            out = make_uint4(__funnelshift_r(wv[u][0], wv[u][1], sh),
                                             __funnelshift_r(wv[u][1], wv[u][2], sh),
                                             __funnelshift_r(wv[u][2], wv[u][3], sh),
                                             __funnelshift_r(wv[u][3], wv[u][4], sh));
                        }
                        *reinterpret_cast<uint4 *>(arow + j * 128) = out;
                    }
                }
            }
            fence_proxy_async_smem();
            mbar_arrive(&sb.halo_empty[b]);
            if (!p.starve) mbar_arrive(&sb.full[stage]);
            if (++stage == p.stages) {
                stage = 0;
                phase ^= 1u;
            }
        }
        if (tid == 0 && *wd.abort) {  // let the halo loads still in flight land
            for (int b = 0; b < 2; ++b) {
                const int n_issued = b == 0 ? issued0 : issued1;
                if (n_issued == 0) continue;
                const uint32_t parity = static_cast<uint32_t>(n_issued - 1) & 1u;
                const uint64_t start = globaltimer_ns();
                while (!mbar_try_wait(&sb.halo_full[b], parity) && globaltimer_ns() - start < wd.timeout_ns) {
                }
            }
        }
    } else if (warp < 4) {
        // -------------------------------------------------------------- gather ---
        const int tid = threadIdx.x;  // the tile row this thread builds
        const size_t img_elems = static_cast<size_t>(p.C) * p.H * p.W;
        int stage = 0;
        uint32_t phase = 0;
        for (int t = blockIdx.x; t < p.n_mtiles; t += gridDim.x) {
            if (!mbar_wait(&sb.empty[stage], phase ^ 1u, wd, kDevTimeoutEmpty)) break;
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
            const long long row_base =
                static_cast<long long>(n) * img_elems +
                (p.in_nchw ? static_cast<long long>(ih0) * p.W + iw0
                           : (static_cast<long long>(ih0) * p.W + iw0) * p.C);
            uint8_t *arow = ring + static_cast<size_t>(stage) * sbytes + canon_offset(tid, 0, sbo);
            if (p.vec_rows) {
                gather_rows<kF32>(p, table, arow, a_bytes, nchunks, valid,
                                  static_cast<long long>(n) * img_elems, ih0, iw0);
            } else {
#pragma unroll 2
            for (int j = 0; j < nchunks; ++j) {
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
                    float4 hi, lo;
                    hi.x = tf32_round(v[0]); lo.x = tf32_round(v[0] - hi.x);
                    hi.y = tf32_round(v[1]); lo.y = tf32_round(v[1] - hi.y);
                    hi.z = tf32_round(v[2]); lo.z = tf32_round(v[2] - hi.z);
                    hi.w = tf32_round(v[3]); lo.w = tf32_round(v[3] - hi.w);
                    *reinterpret_cast<float4 *>(arow + j * 128) = hi;
                    *reinterpret_cast<float4 *>(arow + a_bytes + j * 128) = lo;
                } else {
                    const unsigned short *xs = static_cast<const unsigned short *>(p.x);
                    uint32_t w2[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        uint32_t pair = 0;
#pragma unroll
                        for (int h = 0; h < 2; ++h) {
                            const int4 te = table[j * 8 + e * 2 + h];
                            const int ih = ih0 + te.y, iw = iw0 + te.z;
                            const uint32_t v =
                                (valid && te.w && static_cast<unsigned>(ih) < static_cast<unsigned>(p.H) &&
                                 static_cast<unsigned>(iw) < static_cast<unsigned>(p.W))
                                    ? __ldg(xs + (row_base + te.x))
                                    : 0u;
                            pair |= v << (16 * h);
                        }
                        w2[e] = pair;
                    }
                    *reinterpret_cast<uint4 *>(arow + j * 128) = make_uint4(w2[0], w2[1], w2[2], w2[3]);
                }
            }
            }
            fence_proxy_async_smem();
            if (!p.starve) mbar_arrive(&sb.full[stage]);
            if (++stage == p.stages) {
                stage = 0;
                phase ^= 1u;
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
            for (int t = blockIdx.x; t < p.n_mtiles; t += gridDim.x) {
                if (!mbar_wait(&sb.acc_empty[abuf], aphase ^ 1u, wd, kDevTimeoutAccEmpty) ||
                    !mbar_wait(&sb.full[stage], phase, wd, kDevTimeoutFull)) {
                    ok = false;
                    break;
                }
                tc_fence_after_sync();
                const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(abuf * p.BN);
                const uint32_t a_hi = smem_addr(ring + static_cast<size_t>(stage) * sbytes);
                const uint32_t a_lo = a_hi + a_bytes;
                for (int ks = 0; ks < ksteps; ++ks) {
                    const uint32_t off = static_cast<uint32_t>(ks) * 256u;  // two 16-byte chunks
                    const uint32_t acc = ks > 0 ? 1u : 0u;
                    if constexpr (kF32) {
                        mma_tf32(d_tmem, smem_desc(a_lo + off, 128, sbo, kSwNone),
                                 smem_desc(b_hi + off, 128, sbo, kSwNone), idesc, acc);
                        mma_tf32(d_tmem, smem_desc(a_hi + off, 128, sbo, kSwNone),
                                 smem_desc(b_lo + off, 128, sbo, kSwNone), idesc, 1u);
                        mma_tf32(d_tmem, smem_desc(a_hi + off, 128, sbo, kSwNone),
                                 smem_desc(b_hi + off, 128, sbo, kSwNone), idesc, 1u);
                    } else {
                        mma_bf16(d_tmem, smem_desc(a_hi + off, 128, sbo, kSwNone),
                                 smem_desc(b_hi + off, 128, sbo, kSwNone), idesc, acc);
                    }
                }
                mma_commit(&sb.empty[stage]);
                mma_commit(&sb.acc_full[abuf]);
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
            }
        }
        __syncwarp();
    } else {
        // ------------------------------------------------------------ epilogue ---
        const int quarter = warp & 3;
        const int row = quarter * 32 + lane;
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
        for (int t = blockIdx.x; t < p.n_mtiles; t += gridDim.x) {
            const bool ok = mbar_wait(&sb.acc_full[abuf], aphase, wd, kDevTimeoutAccFull);
            if (!__all_sync(0xffffffffu, ok)) break;
            tc_fence_after_sync();
            const int m = t * kBM + row;
            const uint32_t taddr = tmem_base + lane_base + static_cast<uint32_t>(abuf * p.BN);
            for (int c0 = 0; c0 < p.BN; c0 += 64) {
                uint32_t r[4][16];
#pragma unroll
                for (int q = 0; q < 4; ++q)
                    if (c0 + q * 16 < p.BN) tmem_ld_x16(taddr + static_cast<uint32_t>(c0 + q * 16), r[q]);
                tmem_ld_wait();
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    if (c0 + q * 16 < p.BN) {
                        float v[16];
#pragma unroll
                        for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[q][i]) + sbias[c0 + q * 16 + i];
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

size_t gather_smem_bytes(bool f32, int BN, int Kpad, int stages, size_t halo_bytes) {
    const int elt = f32 ? 4 : 2;
    const uint32_t b = static_cast<uint32_t>(BN) * Kpad * elt * (f32 ? 2 : 1);
    const size_t a_stage = static_cast<size_t>(kBM) * Kpad * elt * (f32 ? 2 : 1);
    return 1024 /* alignment slack */ + align1k(kHeader + kTableBytes + kBiasBytes + b) +
           2 * static_cast<size_t>(align1k(static_cast<uint32_t>(halo_bytes))) + stages * a_stage;
}

cudaError_t launch_gather(const GatherParams &p, bool f32, int grid, size_t smem, cudaStream_t s) {
    if (p.stages < 2 || p.stages > kMaxStages || p.Kpad > kTableBytes / 16) return cudaErrorInvalidValue;
    auto kern = f32 ? gather_kernel<true> : gather_kernel<false>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    kern<<<grid, kThreads, smem, s>>>(p);
    return cudaGetLastError();
}

}  // namespace conv2d_b200
