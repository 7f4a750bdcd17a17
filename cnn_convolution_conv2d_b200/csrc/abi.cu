// abi.cu -- the C ABI declared in include/conv2d_b200.h: argument validation, the
// per-problem plan (tile shapes, pipeline depth, split of the reduction, scratch
// layout), tensor-map encoding and kernel dispatch.  Host code only; every step of
// the convolution itself runs in the kernels of igemm.cu and layout.cu.
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <algorithm>
#include <atomic>
#include <map>
#include <mutex>
#include <string>

#include "common.cuh"
#include "conv2d_b200.h"

namespace conv2d_b200 {
namespace {

// ------------------------------------------------------------ error state ---
thread_local std::string t_last_error;

int fail(int status, const char *fmt, ...) {
    char buf[512];
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(buf, sizeof(buf), fmt, ap);
    va_end(ap);
    t_last_error = buf;
    return status;
}

int ok() {
    t_last_error.clear();
    return CONV_OK;
}

// Watchdog status word written by device code when a bounded wait runs out.
__device__ int g_device_status;

// Scratch of conv2d_forward_noalloc: callers without an allocator get their
// workspace from here.  Host code passes its device address (looked up once per
// device), never the name itself.
constexpr size_t kNoAllocScratchBytes = CONV2D_NOALLOC_SCRATCH_BYTES;
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

constexpr int kMaxDevices = 64;
constexpr size_t kSmemBudget = 227 * 1024;
constexpr long long kDefaultTimeoutNs = 2000000000LL;

constexpr int kHostioChunks = 16;  // most batch chunks one host-buffer call pipelines

// Streams and events of the host-buffer entry point's copy pipeline, made on first use.
struct HostioPipe {
    std::mutex m;  // one call's enqueue at a time per device: the events below are shared
    bool ready = false;
    cudaStream_t in = nullptr, out = nullptr;  // host -> device, device -> host copies
    cudaEvent_t start = nullptr, done = nullptr;
    cudaEvent_t ev_in[kHostioChunks] = {}, ev_comp[kHostioChunks] = {};
};

struct DeviceInfo {
    bool ready = false;
    int sms = 0;
    int *status = nullptr;
    void *noalloc_scratch = nullptr;  // device address of g_noalloc_scratch
    HostioPipe hio;
};
DeviceInfo g_devices[kMaxDevices];
std::mutex g_mutex;
// Test-hook settings: written by the conv2d_debug_* setters, read once per call
// (see Settings) so that one call never mixes two settings.
std::atomic<long long> g_timeout_ns{kDefaultTimeoutNs};
std::atomic<int> g_starve{0};
std::atomic<int> g_pair_mode{0};  // CTA pairs: 0 when they pay, 1 whenever eligible, 2 never
std::map<long long, int> g_pair_clusters;  // see pair_cluster_limit

// The test-hook settings as one call sees them.
struct Settings {
    long long timeout_ns;
    int starve;
    int pair_mode;
};

Settings settings_now() {
    Settings s;
    s.timeout_ns = g_timeout_ns.load(std::memory_order_relaxed);
    s.starve = g_starve.load(std::memory_order_relaxed);
    s.pair_mode = g_pair_mode.load(std::memory_order_relaxed);
    return s;
}
cudaEvent_t g_main_start = nullptr, g_main_stop = nullptr;
std::atomic<unsigned long long> g_launches{0};

using EncodeTiledFn = CUresult (*)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                   const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                   const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
using EncodeIm2colFn = CUresult (*)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                    const cuuint64_t *, const cuuint64_t *, const int *,
                                    const int *, cuuint32_t, cuuint32_t, const cuuint32_t *,
                                    CUtensorMapInterleave, CUtensorMapSwizzle,
                                    CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
EncodeTiledFn g_encode_tiled = nullptr;
EncodeIm2colFn g_encode_im2col = nullptr;

// Looks up the current device's SM count and status word, and the driver's
// tensor-map encoders, once.
int device_info(DeviceInfo **out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return fail(CONV_ERR_CUDA, "cudaGetDevice: %s", cudaGetErrorString(e));
    if (dev < 0 || dev >= kMaxDevices) return fail(CONV_ERR_UNSUPPORTED, "device index %d", dev);
    std::lock_guard<std::mutex> lock(g_mutex);
    DeviceInfo &d = g_devices[dev];
    if (!d.ready) {
        int major = 0, minor = 0;
        cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev);
        if (major != 10 || minor != 0)
            return fail(CONV_ERR_UNSUPPORTED, "device %d is sm_%d%d; this library is built for sm_100a",
                        dev, major, minor);
        e = cudaDeviceGetAttribute(&d.sms, cudaDevAttrMultiProcessorCount, dev);
        if (e != cudaSuccess) return fail(CONV_ERR_CUDA, "SM count: %s", cudaGetErrorString(e));
        e = cudaGetSymbolAddress(reinterpret_cast<void **>(&d.status), g_device_status);
        if (e != cudaSuccess)
            return fail(CONV_ERR_CUDA, "status word address: %s", cudaGetErrorString(e));
        if (!g_encode_tiled || !g_encode_im2col) {
            cudaDriverEntryPointQueryResult q1, q2;
            void *f1 = nullptr, *f2 = nullptr;
            e = cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &f1, 12000,
                                                 cudaEnableDefault, &q1);
            if (e != cudaSuccess || q1 != cudaDriverEntryPointSuccess || !f1)
                return fail(CONV_ERR_CUDA, "cuTensorMapEncodeTiled entry point unavailable");
            e = cudaGetDriverEntryPointByVersion("cuTensorMapEncodeIm2col", &f2, 12000,
                                                 cudaEnableDefault, &q2);
            if (e != cudaSuccess || q2 != cudaDriverEntryPointSuccess || !f2)
                return fail(CONV_ERR_CUDA, "cuTensorMapEncodeIm2col entry point unavailable");
            g_encode_tiled = reinterpret_cast<EncodeTiledFn>(f1);
            g_encode_im2col = reinterpret_cast<EncodeIm2colFn>(f2);
        }
        d.ready = true;
    }
    *out = &d;
    return CONV_OK;
}

// ------------------------------------------------------------------- plan ---
struct Plan {
    int stride_w;   // column stride (the row stride is `stride`)
    int N, C_in, H, W, C_out, Kh, Kw, stride, pad, dilation, groups;
    int pad_w;      // column padding (= pad, the row padding, for every caller-facing entry)
    bool vol;       // 3-D convolution: input depth D, filter depth Kd, output depth Do
    bool vreuse;    // ... on the input-slice-reuse kernel (vol.cu)
    bool pw;        // 1x1 on the kernel with resident weights (pw.cu)
    int pw_ybufs;   // its output staging blocks per epilogue warp
    int vJ, vn_k, vn_odb;  // its output slices per unit, tiles per slice, slice blocks
    int vnacc;             // its accumulator sets (tensor memory: vnacc * vJ * C_out columns)
    int D, Kd, Do;
    bool f32;
    int elt;
    conv_layout_t layout;
    int Ho, Wo;
    long long M;
    int Cin_g, Cout_g, Cpg;  // per group the kernels see (merged groups: gm of the caller's)
    int gm;                  // caller's groups merged into one (see group_merge)
    bool gather;    // few input channels: the software-gather kernel reads x directly
    bool gather_t;  // ... in its transposed form (gather_t.cu): bf16 NCHW, one output row per tile
    int tpix;       // its pixels per tile (Wo rounded up to 16)
    int nhalo;      // its staged-row buffers
    int nacc;       // its accumulators
    int nout;       // its output images
    int rt;         // its output rows per tile
    int kt;         // its reduction length per tile
    bool a_tmem;    // its A operand resident in tensor memory
    bool vec_rows;  // ... with 16-byte row loads (NCHW, aligned rows, unit dilation)
    bool halo;      // ... from input rows staged in shared memory by TMA
    int R, BW, ME;  // halo rows per tile, staged row width, left zero margin (elements)
    int acols;      // tensor-memory columns per gathered A slot
    bool tma_out;   // epilogue stores through shared memory and TMA (both kernels)
    size_t w_image_off;  // offset of the gather kernel's weight image in w_packed
    int cw;         // output channels per gather epilogue group
    int Kc, Kpad;   // its compact reduction length and padded length
    bool xcopy;     // x goes through the channels-last padding kernel first
    bool direct_a;  // 1x1, stride 1, no padding: X_col is x itself, read with tiled loads
    bool pair;      // CTA-pair kernel: units of 256 rows, M = 256 MMAs over an SM pair
    int cb;         // bytes of channels per plane row (16, 32, 64 or 128)
    int BN, taps, nCB, planes, kstages, Kp;
    int n_mtiles, n_ntiles, splits, units, stages;
    size_t smem;
    size_t off_xcopy, off_partial, off_xcol, ws_total;
    int pair_clusters;  // resident two-CTA clusters of the pair kernel (pair plans only)
    // depthwise kernel (groups = C_in = C_out)
    bool dw;
    int dw_window;      // 3, 5, 7: register-window form; 0: general form
    int dw_Cp;          // channels per pixel of the staged tensor (multiple of 16 bytes)
    int TH, TW, IH, IW, n_th, n_tw, dw_wregion, dw_ctas_per_sm;
};

size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }
int round_up(int v, int a) { return (v + a - 1) / a * a; }

int out_size(int in, int k, int s, int p, int d, int *out) {
    const long long numer = static_cast<long long>(in) + 2LL * p - static_cast<long long>(d) * (k - 1) - 1;
    if (numer < 0) return -1;
    *out = static_cast<int>(numer / s + 1);
    return 0;
}

// Narrow groups -- fewer than 64 output channels each, 16-byte rows of input channels --
// are merged gm at a time into one wider group whose packed weights are block-diagonal
// (zero where an output channel meets another group's input channels).  The product then
// runs with N = gm * C_out/groups columns instead of a handful, which the tensor cores
// execute at full rate; the zeros cost tensor-core cycles but no memory traffic beyond the
// gm-times larger (still small) packed weights.  Depends only on the weight's shape, so
// that conv2d_pack_weight and the forward pass agree.
int group_merge(int C_out, int C_in, int groups, int elt) {
    // fp32 runs three products per multiply-add and splits every staged weight into tf32
    // hi and lo parts: there the block-diagonal zeros cost more than the wider N saves
    // (measured on the grouped layer: 34 -> 46 us), so only bf16 groups are merged.
    if (groups <= 1 || elt != 2) return 1;
    const int cin_g = C_in / groups, cout_g = C_out / groups;
    if (cout_g >= 64 || (cin_g * elt) % 16 != 0) return 1;
    // At most one 128-byte channel row per pixel and tap: a second plane would double the
    // rows the TMA engines load per output (their row rate bounds these layers) and the
    // block-diagonal zeros the weight tiles carry.
    int best = 1;
    for (int gm = 2; gm <= groups; ++gm)
        if (groups % gm == 0 && gm * cout_g <= 128 && gm * cin_g * elt <= 128) best = gm;
    return best;
}

// The software-gather kernel reads its weights as ready-made shared-memory images
// that conv2d_pack_weight writes after the packed OHWI weights: one per reduction
// order (compact; row-vector) whose padded length fits the kernel's tables.
struct GatherImages {
    int bn = 0;              // image rows: C_out rounded up to 16
    int kpad[2] = {0, 0};    // [0] compact order, [1] row-vector order; 0 = absent
    size_t off[2] = {0, 0};  // byte offsets in the packed buffer
    size_t total = 0;        // packed bytes including the images
};

GatherImages gather_images(int C_out, int C_in, int Kh, int Kw, int groups, int elt) {
    GatherImages g;
    const int gm = group_merge(C_out, C_in, groups, elt);
    const int cpg = round_up(C_in / groups, 16 / elt) * gm;
    size_t off = static_cast<size_t>(C_out) * Kh * Kw * cpg * elt;
    g.total = off;
    if (groups != 1 || C_in * elt >= 32 || C_out > (elt == 4 ? 128 : 256)) return g;
    g.bn = round_up(C_out, 16);
    const int per16 = 16 / elt;
    const int kp[2] = {round_up(C_in * Kh * Kw, 32 / elt),
                       Kw <= per16 ? round_up(C_in * Kh * per16, 32 / elt) : 0};
    for (int o = 0; o < 2; ++o) {
        if (kp[o] == 0 || kp[o] > 256) continue;
        off = align_up(off, 256);
        g.kpad[o] = kp[o];
        g.off[o] = off;
        off += static_cast<size_t>(g.bn) * kp[o] * elt * (elt == 4 ? 2 : 1);
    }
    g.total = off;
    return g;
}

// Depthwise problems (groups = C_in = C_out) go to the direct stencil kernel when its
// staged input box fits: tiles of TH (<= 30) x 8 output pixels x 128 bytes of channels, one
// persistent CTA per SM with as many stages as fit.  Returns false (and
// the problem goes to the general kernels) when no tile shape fits.
bool plan_depthwise(Plan *pp) {
    Plan &p = *pp;
    const int per16 = 16 / p.elt;
    p.dw_Cp = round_up(p.C_in, per16);
    p.dw_window = (p.stride == 1 && p.dilation == 1 && p.Kh == p.Kw &&
                   (p.Kh == 3 || p.Kh == 5 || p.Kh == 7)) ? p.Kh : 0;
    p.TW = 2 * dw_pixels_per_thread();
    p.IW = (p.TW - 1) * p.stride + (p.Kw - 1) * p.dilation + 1;
    if (p.IW > 256) return false;
    const int taps = p.Kh * p.Kw;
    const int cc = 128 / p.elt;
    const size_t wbytes = static_cast<size_t>(taps) * 128 + cc * 4;
    p.dw_wregion = static_cast<int>(align_up(wbytes * dw_compute_warps(), 1024));
    const size_t fixed = dw_header_bytes() + p.dw_wregion;
    // the tallest tile (30 rows: one item per compute thread) whose staged box fits twice
    size_t stage = 0;
    const int th_choices[6] = {30, 15, 8, 4, 2, 1};
    p.TH = 0;
    for (int th : th_choices) {
        const int ih = (th - 1) * p.stride + (p.Kh - 1) * p.dilation + 1;
        stage = static_cast<size_t>(ih) * p.IW * 128;
        if (ih <= 256 && fixed + 2 * stage <= kSmemBudget) {
            p.TH = th;
            p.IH = ih;
            break;
        }
    }
    if (p.TH < 1) return false;
    p.dw_ctas_per_sm = 1;
    int stages = static_cast<int>((kSmemBudget - fixed) / stage);
    stages = stages > dw_max_stages() ? dw_max_stages() : stages;
    p.stages = stages;
    p.smem = fixed + static_cast<size_t>(stages) * stage;
    p.n_th = (p.Ho + p.TH - 1) / p.TH;
    p.n_tw = (p.Wo + p.TW - 1) / p.TW;
    const long long units = static_cast<long long>((p.dw_Cp + cc - 1) / cc) * p.N * p.n_th * p.n_tw;
    if (units >= (1LL << 31)) return false;
    p.units = static_cast<int>(units);
    p.dw = true;
    p.gather = false;
    p.pair = false;
    p.direct_a = false;
    p.tma_out = false;
    p.splits = 1;
    p.BN = 0;
    p.cb = 128;
    p.n_mtiles = p.units;
    p.xcopy = p.layout == CONV_NCHW || p.dw_Cp != p.C_in;
    p.off_xcopy = 0;
    p.off_partial = p.off_xcol = 0;
    p.ws_total = p.xcopy ? align_up(static_cast<size_t>(p.N) * p.H * p.W * p.dw_Cp * p.elt, 256) : 0;
    return true;
}

// A convolution the backward entry points run internally: its column padding may differ
// from its row padding (the transposed convolution of a non-square filter) and either may
// be negative (the window starts inside the image).  Internal convolutions never take the
// few-channel gather kernel, whose weight images exist only for caller-packed weights.
struct PadW {
    int pad_w;
    // when set: the product's fp32 results [split][M][C_out] go here (no bias, no
    // split reduction) for a later pass to finish -- the Winograd path's output transform
    float *partial_out = nullptr;
    // x is channels-last with Cpg channels per group whatever `layout` says (which then
    // names y's layout only) -- the folded 3-D input
    bool x_nhwc = false;
    // > 0: the column stride, `stride` then being the row stride (the folded 3-D input,
    // whose rows are already strided)
    int stride_w = 0;
};

// The depth of a 3-D convolution: input depth D and filter depth Kd (stride, padding and
// dilation are shared with the other two directions).
struct Vol {
    int D, Kd;
};

// Validates a problem and fills the plan.  `explicit_im2col` adds the X_col
// buffer to the scratch layout.  `sms` = 0 plans without split (size queries
// made before a device is known use the device's count when one is current).
int make_plan(int N, int C_in, int H, int W, int C_out, int Kh, int Kw, int stride, int pad,
              int dilation, int groups, conv_dtype_t dtype, conv_layout_t layout,
              bool explicit_im2col, int sms, Plan *P, int pair_mode, bool allow_pair = true,
              const PadW *padw = nullptr, const Vol *vol = nullptr) {
    const int pad_w = padw ? padw->pad_w : pad;
    if (N < 1 || C_in < 1 || H < 1 || W < 1 || C_out < 1 || Kh < 1 || Kw < 1)
        return fail(CONV_ERR_INVALID_ARG, "sizes must be >= 1 (N=%d C_in=%d H=%d W=%d C_out=%d Kh=%d Kw=%d)",
                    N, C_in, H, W, C_out, Kh, Kw);
    if (stride < 1 || dilation < 1 || (!padw && pad < 0) || groups < 1)
        return fail(CONV_ERR_INVALID_ARG, "need stride >= 1, dilation >= 1, pad >= 0, groups >= 1");
    if (C_in % groups != 0 || C_out % groups != 0)
        return fail(CONV_ERR_INVALID_ARG, "C_in (%d) and C_out (%d) must be divisible by groups (%d)",
                    C_in, C_out, groups);
    if (dtype != CONV_F32 && dtype != CONV_BF16)
        return fail(CONV_ERR_INVALID_ARG, "unknown dtype %d", static_cast<int>(dtype));
    if (layout != CONV_NHWC && layout != CONV_NCHW)
        return fail(CONV_ERR_INVALID_ARG, "unknown layout %d", static_cast<int>(layout));
    Plan p{};
    p.N = N; p.C_in = C_in; p.H = H; p.W = W; p.C_out = C_out; p.Kh = Kh; p.Kw = Kw;
    p.stride = stride; p.pad = pad; p.pad_w = pad_w; p.dilation = dilation; p.groups = groups;
    p.stride_w = (padw && padw->stride_w > 0) ? padw->stride_w : stride;
    p.vol = vol != nullptr;
    p.D = vol ? vol->D : 1;
    p.Kd = vol ? vol->Kd : 1;
    p.Do = 1;
    if (vol && (p.D < 1 || p.Kd < 1)) return fail(CONV_ERR_INVALID_ARG, "D and Kd must be >= 1");
    if (vol && explicit_im2col) return fail(CONV_ERR_UNSUPPORTED, "no explicit im2col for volumes");
    if (vol && out_size(p.D, p.Kd, stride, pad, dilation, &p.Do))
        return fail(CONV_ERR_INVALID_ARG, "empty output: the dilated kernel is deeper than the padded input");
    p.f32 = dtype == CONV_F32;
    p.elt = p.f32 ? 4 : 2;
    p.layout = layout;
    if (out_size(H, Kh, stride, pad, dilation, &p.Ho) || out_size(W, Kw, p.stride_w, pad_w, dilation, &p.Wo))
        return fail(CONV_ERR_INVALID_ARG, "empty output: the dilated kernel is larger than the padded input");
    p.M = static_cast<long long>(N) * p.Do * p.Ho * p.Wo;
    // Limits of the hardware im2col addressing (traversal stride <= 8, bounding-box
    // corners in [-128, 127] for a 4-D tensor) and of 32-bit indexing.
    if (stride > 8 || p.stride_w > 8) return fail(CONV_ERR_UNSUPPORTED, "stride %d > 8", std::max(stride, p.stride_w));
    if (p.stride_w != stride && (vol || explicit_im2col))
        return fail(CONV_ERR_UNSUPPORTED, "a separate column stride needs the 2-D implicit form");
    if (pad > 127 || pad_w > 127 || pad < -127 || pad_w < -127)
        return fail(CONV_ERR_UNSUPPORTED, "pad %d > 127", pad > pad_w ? pad : pad_w);
    const long long up_h = pad - static_cast<long long>(Kh - 1) * dilation;
    const long long up_w = pad_w - static_cast<long long>(Kw - 1) * dilation;
    if (up_h < -128 || up_w < -128)
        return fail(CONV_ERR_UNSUPPORTED, "dilation*(K-1) - pad exceeds 128");
    if (vol) {  // corners of a 5-D im2col bounding box lie in [-16, 15]
        const long long up_d = pad - static_cast<long long>(p.Kd - 1) * dilation;
        if (pad > 16 || up_h < -16 || up_w < -16 || up_d < -16 || up_h > 15 || up_w > 15 || up_d > 15)
            return fail(CONV_ERR_UNSUPPORTED, "3-D: pad and pad - dilation*(K-1) must lie in [-16, 15]");
    }
    if (p.M >= (1LL << 31) - 256) return fail(CONV_ERR_UNSUPPORTED, "N*Ho*Wo too large");
    if (static_cast<long long>(N) * p.D * H * W * C_in >= (1LL << 40))
        return fail(CONV_ERR_UNSUPPORTED, "input too large");

    p.Cin_g = C_in / groups;
    p.Cout_g = C_out / groups;
    const int align = 16 / p.elt;
    p.Cpg = round_up(p.Cin_g, align);
    p.dw = false;
    if (!vol && !explicit_im2col && groups == C_in && C_out == C_in && plan_depthwise(&p)) {
        *P = p;
        return CONV_OK;
    }
    // From here on `p.groups` is the number of (possibly merged) groups the kernels see.
    p.gm = group_merge(C_out, C_in, groups, p.elt);
    if (p.gm > 1) {
        p.groups = groups / p.gm;
        p.Cin_g *= p.gm;
        p.Cout_g *= p.gm;
        p.Cpg = p.Cin_g;
    }
    // Fewer than 32 bytes of channels per pixel: hardware im2col rows would be too
    // narrow, so the gather kernel builds the rows from x in place (groups = 1, the
    // whole C_out x K weight matrix resident in shared memory).
    // Row-vector order when x is NCHW with 16-byte-aligned rows and the column taps
    // are contiguous (unit dilation) and fit one 16-byte word.
    const int per16 = 16 / p.elt;
    p.vec_rows = layout == CONV_NCHW && dilation == 1 && (W * p.elt) % 16 == 0 && Kw <= per16;
    p.Kc = p.vec_rows ? C_in * Kh * per16 : C_in * Kh * Kw;
    p.Kpad = round_up(p.Kc, 32 / p.elt);
    p.gather = false;
    if (!padw && !vol && !explicit_im2col && groups == 1 && C_in * p.elt < 32 && p.Kpad <= 256 &&
        C_out <= (p.f32 ? 128 : 256)) {
        const int bn = round_up(C_out, 16);
        // Tensor memory (512 columns): two accumulators of bn columns, then A slots
        // of Kpad/2 (bf16, two elements per column) or 2*Kpad (fp32 hi + lo) columns.
        const int acols = p.f32 ? 2 * round_up(p.Kpad, 32) : round_up(p.Kpad / 2, 32);
        int slots = (512 - 2 * bn) / acols;
        slots = slots < gather_max_stages() ? slots : gather_max_stages();
        // Halo staging: every 128-pixel tile lies inside one image (Ho*Wo a multiple
        // of 128) and the rows it reads fit one TMA box, with ME zero columns on the
        // left covering the padding.
        p.halo = false;
        size_t halo_bytes = 0;
        const int HoWo = p.Ho * p.Wo;
        if (p.vec_rows && HoWo % 128 == 0 && pad <= per16) {
            int span = 1;
            for (int m0 = 0; m0 < HoWo; m0 += 128) {
                const int s_rows = (m0 + 127) / p.Wo - m0 / p.Wo + 1;
                span = s_rows > span ? s_rows : span;
            }
            const int R = (span - 1) * stride + (Kh - 1) * dilation + 1;
            const int iw0_max = (p.Wo - 1) * stride - pad;
            const int BW = round_up(iw0_max + per16 + per16 + 2, per16);
            const size_t hb = static_cast<size_t>(C_in) * R * BW * p.elt;
            if (R <= 256 && BW <= 256 && C_in <= 256 && W <= BW &&
                gather_smem_bytes(p.f32, bn, p.Kpad, hb, 0) <= kSmemBudget) {
                p.halo = true;
                p.R = R;
                p.BW = BW;
                p.ME = per16;
                halo_bytes = hb;
            }
        }
        // Staged tiles lie inside one image, so a bf16 epilogue can store each tile
        // with TMA (NCHW output rows of 128 pixels).
        p.cw = round_up((bn + 1) / 2, 16);
        p.tma_out = p.halo && !p.f32;
        size_t smem = gather_smem_bytes(p.f32, bn, p.Kpad, halo_bytes,
                                        p.tma_out ? static_cast<size_t>(p.cw) * 128 * p.elt : 0);
        if (p.tma_out && smem > kSmemBudget) {
            p.tma_out = false;
            smem = gather_smem_bytes(p.f32, bn, p.Kpad, halo_bytes, 0);
        }
        const GatherImages gi = gather_images(C_out, C_in, Kh, Kw, groups, p.elt);
        const int order = p.vec_rows ? 1 : 0;
        if (slots >= 2 && smem <= kSmemBudget && gi.kpad[order] == p.Kpad) {
            p.gather = true;
            // Transposed form: output channels on the lanes, one or two output rows per
            // tile, channel rows stored into NCHW y without transposition.  Needs the
            // row-vector order, whole 16-byte pieces per row (Wo % 8 == 0) and the tile's
            // staged input box.
            p.gather_t = false;
            if (!p.f32 && p.vec_rows && p.Wo % 8 == 0 && p.Wo <= 256 && C_out <= 128 && pad <= per16) {
                const int iw0_max = (p.Wo - 1) * stride - pad;
                const int BW = round_up(iw0_max + per16 + per16 + 2, per16);
                const int tpix = round_up(p.Wo, 16);
                // Two output rows per tile when the channels fill half the lanes, else one.
                // The output block of a tile goes out by TMA stores from double-buffered
                // output images when they fit beside at least four staged-row buffers,
                // else from one image, else straight from the registers; then as many
                // staged-row buffers as fit (up to the kernel's limit), an even number (a
                // buffer serves one of the kernel's two gather groups): one tile's work is
                // shorter than the latency of its rows' load.
                for (int rt = C_out <= 64 ? 2 : 1; rt >= 1 && !p.gather_t; --rt) {
                    const int R = Kh + (rt - 1) * stride;
                    if (C_in * R > gather_t_max_chunks() || BW > 256 || W > BW || R > 256) continue;
                    const int kt = rt == 1 ? p.Kpad : round_up(C_in * R * per16, 32 / p.elt);
                    const size_t hb = static_cast<size_t>(C_in) * R * BW * p.elt;
                    const size_t ob = static_cast<size_t>((p.Wo + 63) / 64) * bn * rt * 128;  // 64-pixel parts
                    // A in tensor memory when at least two accumulators fit beside it (its
                    // kt/2 columns), else in shared memory
                    const int acc_tm = (512 - kt / 2) / tpix;
                    for (int a_tm = (tpix >= 64 && acc_tm >= 2) ? 1 : 0; a_tm >= 0 && !p.gather_t; --a_tm) {
                        const int opts[3][3] = {{1, 2, 4}, {1, 1, 2}, {0, 1, 2}};  // tma_out, images, fewest row buffers
                        for (const auto &o : opts) {
                            const size_t obytes = o[0] ? ob : 0;
                            int nhalo = gather_t_max_halo();
                            while (nhalo > o[2] &&
                                   gather_t_smem_bytes(kt, tpix, hb, nhalo, obytes, o[1], a_tm != 0) > kSmemBudget)
                                --nhalo;
                            nhalo &= ~1;
                            const size_t tsmem = gather_t_smem_bytes(kt, tpix, hb, nhalo, obytes, o[1], a_tm != 0);
                            if (tsmem > kSmemBudget) continue;
                            p.gather_t = true;
                            p.rt = rt;
                            p.kt = kt;
                            p.a_tmem = a_tm != 0;
                            p.nhalo = nhalo;
                            p.nout = o[1];
                            p.tma_out = o[0] != 0;
                            // as many accumulators as the 512 tensor-memory columns hold
                            const int acc = a_tm ? acc_tm : 512 / tpix;
                            p.nacc = acc < gather_t_max_acc() ? acc : gather_t_max_acc();
                            p.halo = true;
                            p.R = R;
                            p.BW = BW;
                            p.ME = per16;
                            p.tpix = tpix;
                            smem = tsmem;
                            break;
                        }
                    }
                }
            }
            p.w_image_off = gi.off[order];
            p.BN = bn;
            p.stages = slots;
            p.acols = acols;
            // at least 120 KB, so that one CTA (holding all tensor memory) runs per SM
            p.smem = smem > 120 * 1024 ? smem : 120 * 1024;
            p.n_mtiles = p.gather_t ? N * ((p.Ho + p.rt - 1) / p.rt) : static_cast<int>((p.M + 127) / 128);
            p.n_ntiles = 1;
            p.splits = 1;
            p.units = p.n_mtiles;
            p.xcopy = false;
            p.off_xcopy = p.off_partial = p.off_xcol = p.ws_total = 0;
            *P = p;
            return CONV_OK;
        }
    }
    p.xcopy = (layout == CONV_NCHW && !(padw && padw->x_nhwc)) || p.Cpg != p.Cin_g;
    if (p.xcopy && padw && padw->x_nhwc)
        return fail(CONV_ERR_UNSUPPORTED, "channels-last input without its channel padding");
    // A 1x1 filter at stride 1 without padding makes the im2col matrix the
    // channels-last input itself (one row per pixel), so the tensor-core kernel reads
    // it with plain tiled loads, which stream far faster than im2col-mode loads.
    p.direct_a = !explicit_im2col && p.Kd == 1 && Kh == 1 && Kw == 1 && stride == 1 && p.stride_w == 1 && pad == 0 &&
                 pad_w == 0;
    const int row_bytes = p.Cpg * p.elt;
    p.cb = row_bytes % 128 == 0 ? 128 : row_bytes % 64 == 0 ? 64 : row_bytes % 32 == 0 ? 32 : 16;
    const int cap = p.f32 ? 128 : 256;
    const int nt = (p.Cout_g + cap - 1) / cap;
    p.BN = round_up((p.Cout_g + nt - 1) / nt, 16);
    p.n_ntiles = (p.Cout_g + p.BN - 1) / p.BN;
    p.taps = p.Kd * Kh * Kw;
    p.nCB = row_bytes / p.cb;
    p.planes = p.taps * p.nCB;
    const int np = 128 / p.cb;
    p.kstages = (p.planes + np - 1) / np;
    p.Kp = p.taps * p.Cpg;
    if (p.kstages > (1 << 26)) return fail(CONV_ERR_UNSUPPORTED, "reduction too long (%d stages)", p.kstages);
    p.n_mtiles = static_cast<int>((p.M + 127) / 128);
    long long base = static_cast<long long>(p.n_mtiles) * p.n_ntiles * p.groups;
    if (base >= (1LL << 31)) return fail(CONV_ERR_UNSUPPORTED, "too many tiles");
    p.splits = 1;
    if (sms > 0 && base < sms) {
        int s = static_cast<int>(sms / base);
        s = s < p.kstages / 4 ? s : p.kstages / 4;
        s = s < 16 ? s : 16;
        if (s >= 2) p.splits = s;
    }
    // CTA pairs (bf16): each SM stages half of the weight tile and the pair's MMAs
    // read the other half from the peer, which halves the weight traffic and the
    // shared-memory bandwidth spent on it.  Used when the 256-row units still give
    // every SM pair work and the tile has at least 128 columns: narrower pair products
    // (M = 256, N = 64) issue no faster than single-CTA ones and gain nothing (measured:
    // the grouped layer 10.8 against 10.2 us, the 3-D video layer 218 against 213 us); the
    // test hook can force or forbid them.
    const long long pair_units = ((p.M + 255) / 256) * p.n_ntiles * p.groups;
    const bool pair_ok = allow_pair && !p.f32 && p.BN % 32 == 0 && pair_mode != 2;
    if (pair_ok && ((p.splits == 1 && sms > 0 && pair_units >= sms / 2 && p.BN >= 128) || pair_mode == 1)) {
        p.pair = true;
        p.splits = 1;
        p.n_mtiles = static_cast<int>((p.M + 255) / 256);
        base = pair_units;
    }
    p.units = static_cast<int>(base * p.splits);
    // 3-D, stride 1, unit dilation, 64 input channels, at most 128 output channels: the
    // kernel that loads each input depth slice once for all the depth taps that read it
    // (vol.cu), with accumulator sets of J slices in tensor memory and at least three
    // stages beside the weights of two (kh, kw).
    p.vreuse = false;
    if (vol && !p.f32 && !padw && !explicit_im2col && groups == 1 && layout == CONV_NHWC && stride == 1 &&
        dilation == 1 && C_in == 64 && C_out % 32 == 0 && C_out <= 128 && (p.Ho * p.Wo) % 32 == 0 &&
        p.Ho * p.Wo >= 128) {
        // As many output slices per unit as tensor memory holds (each input slice then serves
        // more of them: (J + Kd - 1) boxes per J slices); two accumulator sets when they fit.
        int J = 512 / C_out < vol_reuse_max_j() ? 512 / C_out : vol_reuse_max_j();
        J = J < p.Do ? J : p.Do;
        const int nacc = 2 * J * C_out <= 512 ? 2 : 1;
        int vst = vol_reuse_max_stages();
        while (vst > 3 && vol_reuse_smem_bytes(p.Kd, C_out, vst) > kSmemBudget) --vst;
        if (vol_reuse_smem_bytes(p.Kd, C_out, vst) <= kSmemBudget) {
            p.vreuse = true;
            p.vJ = J;
            p.vnacc = nacc;
            p.vn_k = (p.Ho * p.Wo + 127) / 128;
            p.vn_odb = (p.Do + J - 1) / J;
            p.pair = false;
            p.splits = 1;
            p.BN = C_out;
            p.n_ntiles = 1;
            p.units = N * p.vn_odb * p.vn_k;
            p.stages = vst;
            p.tma_out = true;
            p.smem = vol_reuse_smem_bytes(p.Kd, C_out, vst);
            p.ws_total = 0;
            p.xcopy = false;
            *P = p;
            return CONV_OK;
        }
    }
    // bf16 channels-last output leaves through shared memory and TMA stores when
    // every 32-column block of a tile lies inside its group's columns.
    p.tma_out = !p.f32 && layout == CONV_NHWC && p.splits == 1 && !(padw && padw->partial_out) &&
                p.BN % 32 == 0 && p.Cout_g % p.BN == 0 && (C_out * p.elt) % 16 == 0;
    const int bn_local = p.pair ? p.BN / 2 : p.BN;  // B rows staged per CTA
    const size_t stage = static_cast<size_t>(128 + bn_local) * 128 * (p.f32 ? 2 : 1);
    const size_t ystage = igemm_smem_bytes(p.f32, bn_local, 0, p.tma_out) - igemm_smem_bytes(p.f32, bn_local, 0, false);
    int stages = static_cast<int>((kSmemBudget - 2048 - ystage) / stage);
    p.stages = stages > 8 ? 8 : stages;
    if (p.stages < 2) return fail(CONV_ERR_UNSUPPORTED, "tile does not fit in shared memory");
    p.smem = igemm_smem_bytes(p.f32, bn_local, p.stages, p.tma_out);
    // A pointwise layer with a short reduction on CTA pairs: the kernel that keeps each
    // cluster's 256-column weight tile resident and streams only the input rows (pw.cu);
    // bf16 channels-last output, or the raw fp32 sums a later pass finishes (Winograd).
    p.pw = false;
    p.pw_ybufs = 2;
    const bool partial_ext = padw && padw->partial_out;
    const int pw_nk = p.Cin_g / 64;
    if (p.pair && p.direct_a && !p.f32 && p.splits == 1 && p.gm == 1 && layout == CONV_NHWC &&
        (partial_ext || p.tma_out) && p.Cin_g % 64 == 0 && p.Cin_g == p.Cpg && pw_nk <= pw_max_planes() &&
        p.Cout_g % 256 == 0 && p.BN == 256) {
        // two staging blocks per epilogue warp while that leaves four input stages, else one
        for (int yb = 2; yb >= 1 && !p.pw; --yb) {
            int pst = pw_max_stages();
            while (pst > 4 && pw_smem_bytes(pw_nk, 256, pst, partial_ext, yb) > kSmemBudget) --pst;
            if (pw_smem_bytes(pw_nk, 256, pst, partial_ext, yb) <= kSmemBudget) {
                p.pw = true;
                p.pw_ybufs = yb;
                p.stages = pst;
                p.smem = pw_smem_bytes(pw_nk, 256, pst, partial_ext, yb);
            }
        }
        if (p.pw) p.tma_out = true;
    }
    size_t off = 0;
    p.off_xcopy = off;
    if (p.xcopy) off = align_up(off + static_cast<size_t>(N) * p.D * H * W * p.groups * p.Cpg * p.elt, 256);
    p.off_partial = off;
    if (p.splits > 1) off = align_up(off + static_cast<size_t>(p.splits) * p.M * C_out * 4, 256);
    p.off_xcol = off;
    if (explicit_im2col) off = align_up(off + static_cast<size_t>(p.M) * p.groups * p.Kp * p.elt, 256);
    p.ws_total = off;
    *P = p;
    return CONV_OK;
}

bool aligned16(const void *ptr) { return (reinterpret_cast<uintptr_t>(ptr) & 15u) == 0; }

CUtensorMapSwizzle swizzle_for(int cb) {
    switch (cb) {
        case 128: return CU_TENSOR_MAP_SWIZZLE_128B;
        case 64: return CU_TENSOR_MAP_SWIZZLE_64B;
        case 32: return CU_TENSOR_MAP_SWIZZLE_32B;
        default: return CU_TENSOR_MAP_SWIZZLE_NONE;
    }
}

CUtensorMapDataType tma_type(const Plan &p) {
    return p.f32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
}

// A operand, implicit: im2col view of the channels-last input.
int encode_a_im2col(const Plan &p, const void *x_nhwc, CUtensorMap *map) {
    const cuuint64_t ctot = static_cast<cuuint64_t>(p.groups) * p.Cpg;
    cuuint64_t dims[4] = {ctot, static_cast<cuuint64_t>(p.W), static_cast<cuuint64_t>(p.H),
                          static_cast<cuuint64_t>(p.N)};
    cuuint64_t strides[3] = {ctot * p.elt, ctot * p.elt * p.W, ctot * p.elt * p.W * p.H};
    int lower[2] = {-p.pad_w, -p.pad};  // (w, h)
    int upper[2] = {p.pad_w - (p.Kw - 1) * p.dilation, p.pad - (p.Kh - 1) * p.dilation};
    cuuint32_t estr[4] = {1, static_cast<cuuint32_t>(p.stride_w), static_cast<cuuint32_t>(p.stride), 1};
    CUresult r = g_encode_im2col(map, tma_type(p), 4, const_cast<void *>(x_nhwc), dims, strides, lower,
                                 upper, static_cast<cuuint32_t>(p.cb / p.elt), 128, estr,
                                 CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle_for(p.cb),
                                 CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(CONV_ERR_CUDA, "cuTensorMapEncodeIm2col failed (%d)", static_cast<int>(r));
    return CONV_OK;
}

// A operand, implicit, volumes: 5-D im2col view of the channels-last input (c, w, h, d, n).
int encode_a_im2col_5d(const Plan &p, const void *x_ndhwc, CUtensorMap *map) {
    const cuuint64_t ctot = static_cast<cuuint64_t>(p.groups) * p.Cpg;
    cuuint64_t dims[5] = {ctot, static_cast<cuuint64_t>(p.W), static_cast<cuuint64_t>(p.H),
                          static_cast<cuuint64_t>(p.D), static_cast<cuuint64_t>(p.N)};
    cuuint64_t strides[4] = {ctot * p.elt, ctot * p.elt * p.W, ctot * p.elt * p.W * p.H,
                             ctot * p.elt * p.W * p.H * p.D};
    int lower[3] = {-p.pad_w, -p.pad, -p.pad};  // (w, h, d)
    int upper[3] = {p.pad_w - (p.Kw - 1) * p.dilation, p.pad - (p.Kh - 1) * p.dilation,
                    p.pad - (p.Kd - 1) * p.dilation};
    cuuint32_t estr[5] = {1, static_cast<cuuint32_t>(p.stride), static_cast<cuuint32_t>(p.stride),
                          static_cast<cuuint32_t>(p.stride), 1};
    CUresult r = g_encode_im2col(map, tma_type(p), 5, const_cast<void *>(x_ndhwc), dims, strides, lower, upper,
                                 static_cast<cuuint32_t>(p.cb / p.elt), 128, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                                 swizzle_for(p.cb), CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                                 CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(CONV_ERR_CUDA, "cuTensorMapEncodeIm2col (5-D) failed (%d)", static_cast<int>(r));
    return CONV_OK;
}

// A operand, explicit: the X_col matrix (M rows of groups*Kp elements).
int encode_a_xcol(const Plan &p, const void *xcol, CUtensorMap *map) {
    const cuuint64_t cols = static_cast<cuuint64_t>(p.groups) * p.Kp;
    cuuint64_t dims[2] = {cols, static_cast<cuuint64_t>(p.M)};
    cuuint64_t strides[1] = {cols * p.elt};
    cuuint32_t box[2] = {static_cast<cuuint32_t>(p.cb / p.elt), 128};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = g_encode_tiled(map, tma_type(p), 2, const_cast<void *>(xcol), dims, strides, box, estr,
                                CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle_for(p.cb),
                                CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(CONV_ERR_CUDA, "cuTensorMapEncodeTiled (X_col) failed (%d)", static_cast<int>(r));
    return CONV_OK;
}

// B operand: packed weights viewed as {Kp, Cout_g, groups}.
int encode_b(const Plan &p, const void *w_packed, CUtensorMap *map) {
    cuuint64_t dims[3] = {static_cast<cuuint64_t>(p.Kp), static_cast<cuuint64_t>(p.Cout_g),
                          static_cast<cuuint64_t>(p.groups)};
    cuuint64_t strides[2] = {static_cast<cuuint64_t>(p.Kp) * p.elt,
                             static_cast<cuuint64_t>(p.Kp) * p.elt * p.Cout_g};
    cuuint32_t box[3] = {static_cast<cuuint32_t>(p.cb / p.elt), static_cast<cuuint32_t>(p.pair ? p.BN / 2 : p.BN), 1};
    cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = g_encode_tiled(map, tma_type(p), 3, const_cast<void *>(w_packed), dims, strides, box,
                                estr, CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle_for(p.cb),
                                CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(CONV_ERR_CUDA, "cuTensorMapEncodeTiled (weights) failed (%d)", static_cast<int>(r));
    return CONV_OK;
}

int check_launch(cudaError_t e, const char *what) {
    if (e != cudaSuccess) return fail(CONV_ERR_CUDA, "%s launch: %s", what, cudaGetErrorString(e));
    g_launches.fetch_add(1, std::memory_order_relaxed);
    return CONV_OK;
}

// Records a timing event on `stream`; under stream capture it is recorded as an
// external event so that it becomes a timing node of the graph.
int record_event(cudaEvent_t ev, cudaStream_t stream) {
    cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
    cudaError_t e = cudaStreamIsCapturing(stream, &cap);
    if (e == cudaSuccess)
        e = cap == cudaStreamCaptureStatusActive
                ? cudaEventRecordWithFlags(ev, stream, cudaEventRecordExternal)
                : cudaEventRecord(ev, stream);
    if (e != cudaSuccess) return fail(CONV_ERR_CUDA, "timing event record: %s", cudaGetErrorString(e));
    return CONV_OK;
}

// The software-gather path (few input channels): one kernel, no scratch.
int gather_impl(const Plan &p, const void *x, const void *w_packed, const void *bias, void *y,
                DeviceInfo *dev, const Settings &cfg, cudaStream_t stream) {
    GatherParams g;
    std::memset(&g, 0, sizeof(g));
    g.x = x;
    g.w_packed = w_packed;
    g.w_image = static_cast<const uint8_t *>(w_packed) + p.w_image_off;
    g.N = p.N; g.C = p.C_in; g.H = p.H; g.W = p.W; g.Kh = p.Kh; g.Kw = p.Kw;
    g.stride = p.stride; g.pad = p.pad; g.dilation = p.dilation;
    g.Ho = p.Ho; g.Wo = p.Wo; g.M = static_cast<int>(p.M);
    g.Cpg = p.Cpg;
    g.Kc = p.Kc;
    g.Kpad = p.Kpad;
    g.BN = p.BN;
    g.n_mtiles = p.n_mtiles;
    g.stages = p.stages;
    g.acols = p.acols;
    g.in_nchw = p.layout == CONV_NCHW ? 1 : 0;
    g.vec_rows = p.vec_rows ? 1 : 0;
    g.halo = p.halo ? 1 : 0;
    if (p.halo) {
        g.R = p.R;
        g.BW = p.BW;
        g.ME = p.ME;
        cuuint64_t dims[4] = {static_cast<cuuint64_t>(p.W), static_cast<cuuint64_t>(p.H),
                              static_cast<cuuint64_t>(p.C_in), static_cast<cuuint64_t>(p.N)};
        cuuint64_t strides[3] = {static_cast<cuuint64_t>(p.W) * p.elt,
                                 static_cast<cuuint64_t>(p.W) * p.H * p.elt,
                                 static_cast<cuuint64_t>(p.W) * p.H * p.C_in * p.elt};
        cuuint32_t box[4] = {static_cast<cuuint32_t>(p.BW), static_cast<cuuint32_t>(p.R),
                             static_cast<cuuint32_t>(p.C_in), 1};
        cuuint32_t estr[4] = {1, 1, 1, 1};
        CUresult r = g_encode_tiled(&g.tmap_x, tma_type(p), 4, const_cast<void *>(x), dims, strides,
                                    box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
        if (r != CUDA_SUCCESS)
            return fail(CONV_ERR_CUDA, "cuTensorMapEncodeTiled (input rows) failed (%d)", static_cast<int>(r));
    }
    g.tmem_cols = 512;  // accumulators and A slots
    if (p.gather_t) {
        g.tpix = p.tpix;
        g.nhalo = p.nhalo;
        g.nacc = p.nacc;
        g.nout = p.nout;
        g.rt = p.rt;
        g.kt = p.kt;
        g.a_tmem = p.a_tmem ? 1 : 0;
        g.tmem_cols = 32;
        while (g.tmem_cols < static_cast<uint32_t>(p.nacc * p.tpix + (p.a_tmem ? p.kt / 2 : 0))) g.tmem_cols <<= 1;
    }
    g.cw = p.cw;
    g.tma_out = p.tma_out ? 1 : 0;
    if (p.tma_out && p.gather_t) {
        // y as (Wo, C_out, Ho, N); boxes of 64 pixels x every channel x the tile's output
        // rows, 128-byte swizzled (rows of the box: row-of-tile-major, then channel)
        const cuuint64_t wo = static_cast<cuuint64_t>(p.Wo), ho = static_cast<cuuint64_t>(p.Ho);
        cuuint64_t dims[4] = {wo, static_cast<cuuint64_t>(p.C_out), ho, static_cast<cuuint64_t>(p.N)};
        cuuint64_t strides[3] = {wo * ho * p.elt, wo * p.elt, wo * ho * p.elt * p.C_out};
        cuuint32_t box[4] = {64, static_cast<cuuint32_t>(p.BN), static_cast<cuuint32_t>(p.rt), 1};
        cuuint32_t estr[4] = {1, 1, 1, 1};
        CUresult r = g_encode_tiled(&g.tmap_y, tma_type(p), 4, y, dims, strides, box, estr,
                                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                                    CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
        if (r != CUDA_SUCCESS)
            return fail(CONV_ERR_CUDA, "cuTensorMapEncodeTiled (output rows) failed (%d)", static_cast<int>(r));
    } else if (p.tma_out) {
        const cuuint64_t howo = static_cast<cuuint64_t>(p.Ho) * p.Wo;
        cuuint64_t dims[3] = {howo, static_cast<cuuint64_t>(p.C_out), static_cast<cuuint64_t>(p.N)};
        cuuint64_t strides[2] = {howo * p.elt, howo * p.elt * p.C_out};
        cuuint32_t box[3] = {32, static_cast<cuuint32_t>(p.cw), 1};  // one warp: 32 pixels x cw channels
        cuuint32_t estr[3] = {1, 1, 1};
        CUresult r = g_encode_tiled(&g.tmap_y, tma_type(p), 3, y, dims, strides, box, estr,
                                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                                    CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
        if (r != CUDA_SUCCESS)
            return fail(CONV_ERR_CUDA, "cuTensorMapEncodeTiled (output) failed (%d)", static_cast<int>(r));
    }
    g.y = y;
    g.bias = bias;
    g.Cout = p.C_out;
    g.out_mode = p.layout == CONV_NCHW ? kOutNCHW : kOutNHWC;
    g.vec_ok = (p.C_out % (16 / p.elt) == 0) ? 1 : 0;
    g.status = dev->status;
    g.timeout_ns = cfg.timeout_ns;
    g.starve = cfg.starve;
    const int grid = p.n_mtiles < dev->sms ? p.n_mtiles : dev->sms;
    int st;
    cudaEvent_t ev_start = g_main_start, ev_stop = g_main_stop;
    if (ev_start && ev_stop && (st = record_event(ev_start, stream)) != CONV_OK) return st;
    cudaError_t e = p.gather_t ? launch_gather_t(g, grid, p.smem, stream) : launch_gather(g, p.f32, grid, p.smem, stream);
    if ((st = check_launch(e, "gather tensor-core product")) != CONV_OK) return st;
    if (ev_start && ev_stop && (st = record_event(ev_stop, stream)) != CONV_OK) return st;
    return ok();
}

// The depthwise path: an optional channels-last (padded) copy of x, then one kernel.
int dw_impl(const Plan &p, const void *x, const void *w_packed, const void *bias, void *y, void *workspace,
            DeviceInfo *dev, const Settings &cfg, cudaStream_t stream) {
    DwParams d;
    std::memset(&d, 0, sizeof(d));
    const void *x_nhwc = x;
    int st;
    if (p.xcopy) {
        x_nhwc = workspace;
        cudaError_t e = p.layout == CONV_NCHW
                            ? launch_nchw_to_nhwc(x, workspace, p.N, p.C_in, p.H, p.W, 1, p.dw_Cp, p.elt, stream)
                            : launch_nhwc_pad(x, workspace, p.N, p.C_in, p.H, p.W, 1, p.dw_Cp, p.elt, stream);
        if ((st = check_launch(e, "channels-last copy")) != CONV_OK) return st;
    }
    cuuint64_t dims[4] = {static_cast<cuuint64_t>(p.dw_Cp), static_cast<cuuint64_t>(p.W),
                          static_cast<cuuint64_t>(p.H), static_cast<cuuint64_t>(p.N)};
    cuuint64_t strides[3] = {static_cast<cuuint64_t>(p.dw_Cp) * p.elt,
                             static_cast<cuuint64_t>(p.dw_Cp) * p.elt * p.W,
                             static_cast<cuuint64_t>(p.dw_Cp) * p.elt * p.W * p.H};
    cuuint32_t box[4] = {static_cast<cuuint32_t>(128 / p.elt), static_cast<cuuint32_t>(p.IW),
                         static_cast<cuuint32_t>(p.IH), 1};
    cuuint32_t estr[4] = {1, 1, 1, 1};
    CUresult r = g_encode_tiled(&d.tmap_x, tma_type(p), 4, const_cast<void *>(x_nhwc), dims, strides, box, estr,
                                CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                                CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS)
        return fail(CONV_ERR_CUDA, "cuTensorMapEncodeTiled (depthwise input) failed (%d)", static_cast<int>(r));
    d.w_packed = w_packed;
    d.bias = bias;
    d.y = y;
    d.N = p.N; d.C = p.C_in; d.Ho = p.Ho; d.Wo = p.Wo; d.Kh = p.Kh; d.Kw = p.Kw;
    d.stride = p.stride; d.pad = p.pad; d.pad_w = p.pad_w; d.dilation = p.dilation;
    d.Cpg = p.Cpg;
    d.TH = p.TH; d.TW = p.TW; d.IH = p.IH; d.IW = p.IW;
    d.n_th = p.n_th; d.n_tw = p.n_tw; d.units = p.units; d.stages = p.stages;
    d.wregion = p.dw_wregion;
    d.out_nchw = p.layout == CONV_NCHW ? 1 : 0;
    d.vec_ok = (p.C_in % (16 / p.elt)) == 0 ? 1 : 0;
    d.status = dev->status;
    d.timeout_ns = cfg.timeout_ns;
    d.starve = cfg.starve;
    const long long slots = static_cast<long long>(dev->sms) * p.dw_ctas_per_sm;
    const int grid = static_cast<int>(p.units < slots ? p.units : slots);
    cudaEvent_t ev_start = g_main_start, ev_stop = g_main_stop;
    if (ev_start && ev_stop && (st = record_event(ev_start, stream)) != CONV_OK) return st;
    cudaError_t e = launch_depthwise(d, p.f32, p.dw_window, grid, p.smem, stream);
    if ((st = check_launch(e, "depthwise")) != CONV_OK) return st;
    if (ev_start && ev_stop && (st = record_event(ev_stop, stream)) != CONV_OK) return st;
    return ok();
}

// Resident two-CTA clusters of the pair kernel for one configuration, asked of the
// runtime once per configuration and device and remembered.
int pair_cluster_limit(int cb, bool im2col, size_t smem, bool vol = false) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 0;
    const long long key = (((static_cast<long long>(dev) * 256 + cb) * 2 + (im2col ? 1 : 0)) * 2 + (vol ? 1 : 0)) *
                              1048576 + static_cast<long long>(smem);
    {
        std::lock_guard<std::mutex> lock(g_mutex);
        auto it = g_pair_clusters.find(key);
        if (it != g_pair_clusters.end()) return it->second;
    }
    int n = 0;
    if (igemm_pair_max_clusters(cb, im2col, smem, &n, vol) != cudaSuccess) {
        (void)cudaGetLastError();
        n = 0;
    }
    std::lock_guard<std::mutex> lock(g_mutex);
    g_pair_clusters[key] = n;
    return n;
}

// Resident two-CTA clusters of the pointwise kernel (pw.cu) at this shared-memory size,
// asked of the runtime once per device and size and remembered.
int pw_cluster_limit(size_t smem, bool out_f32) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 0;
    const long long key = -(((static_cast<long long>(dev) + 1) * 2 + (out_f32 ? 1 : 0)) * 1048576 + static_cast<long long>(smem));
    {
        std::lock_guard<std::mutex> lock(g_mutex);
        auto it = g_pair_clusters.find(key);
        if (it != g_pair_clusters.end()) return it->second;
    }
    int n = 0;
    if (pw_max_clusters(smem, out_f32, &n) != cudaSuccess) {
        (void)cudaGetLastError();
        n = 0;
    }
    std::lock_guard<std::mutex> lock(g_mutex);
    g_pair_clusters[key] = n;
    return n;
}

// The plan a forward call on the current device makes, including the fall-back
// from CTA pairs to single CTAs when the device cannot co-schedule the pair kernel.
// Size queries and the forward pass share it, so that they always agree.
int device_plan(bool explicit_im2col, int N, int C_in, int H, int W, int C_out, int Kh, int Kw,
                int stride, int pad, int dilation, int groups, conv_dtype_t dtype,
                conv_layout_t layout, DeviceInfo *dev, const Settings &cfg, Plan *p,
                const PadW *padw = nullptr, const Vol *vol = nullptr) {
    int st = make_plan(N, C_in, H, W, C_out, Kh, Kw, stride, pad, dilation, groups, dtype, layout,
                       explicit_im2col, dev ? dev->sms : 0, p, cfg.pair_mode, true, padw, vol);
    if (st != CONV_OK) return st;
    p->pair_clusters = 0;
    if (p->vreuse) return CONV_OK;
    if (p->pw && dev) {
        // clusters split evenly over the column tiles
        const int per = p->n_ntiles * p->groups;  // (group, column tile) pairs
        const int n = pw_cluster_limit(p->smem, padw && padw->partial_out);
        p->pair_clusters = (n / per) * per;
        if (p->pair_clusters >= per) return CONV_OK;
        return make_plan(N, C_in, H, W, C_out, Kh, Kw, stride, pad, dilation, groups, dtype, layout,
                         explicit_im2col, dev->sms, p, cfg.pair_mode, false, padw, vol);
    }
    if (p->pair && dev) {
        const bool a_im2col = !(explicit_im2col || p->direct_a);
        p->pair_clusters = pair_cluster_limit(p->cb, a_im2col, p->smem, p->vol && a_im2col);
        if (p->pair_clusters < 1)  // the device cannot co-schedule the pair kernel: single CTAs
            return make_plan(N, C_in, H, W, C_out, Kh, Kw, stride, pad, dilation, groups, dtype, layout,
                             explicit_im2col, dev->sms, p, cfg.pair_mode, false, padw, vol);
    }
    return CONV_OK;
}

// The current device, or NULL (and no error) when this process has none.
DeviceInfo *current_device_or_null() {
    DeviceInfo *dev = nullptr;
    int ndev = 0;
    if (cudaGetDeviceCount(&ndev) == cudaSuccess && ndev > 0 && device_info(&dev) == CONV_OK) return dev;
    cudaGetLastError();
    return nullptr;
}

// The 3-D path with input-slice reuse (vol.cu): one kernel, no scratch.
int vol_impl(const Plan &p, const void *x, const void *w_packed, const void *bias, void *y, DeviceInfo *dev,
             const Settings &cfg, cudaStream_t stream) {
    VolParams v;
    std::memset(&v, 0, sizeof(v));
    int st = encode_a_im2col_5d(p, x, &v.tmap_a);
    if (st != CONV_OK) return st;
    st = encode_b(p, w_packed, &v.tmap_b);
    if (st != CONV_OK) return st;
    {
        cuuint64_t dims[2] = {static_cast<cuuint64_t>(p.C_out), static_cast<cuuint64_t>(p.M)};
        cuuint64_t strides[1] = {static_cast<cuuint64_t>(p.C_out) * p.elt};
        cuuint32_t box[2] = {32, 32};
        cuuint32_t estr[2] = {1, 1};
        CUresult r = g_encode_tiled(&v.tmap_y, tma_type(p), 2, y, dims, strides, box, estr,
                                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B,
                                    CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
        if (r != CUDA_SUCCESS)
            return fail(CONV_ERR_CUDA, "cuTensorMapEncodeTiled (output) failed (%d)", static_cast<int>(r));
    }
    v.M = static_cast<int>(p.M);
    v.Do = p.Do;
    v.HoWo2 = p.Ho * p.Wo;
    v.Wo = p.Wo;
    v.Kd = p.Kd;
    v.Kh = p.Kh;
    v.Kw = p.Kw;
    v.taps = p.Kd * p.Kh * p.Kw;
    v.pad = p.pad;
    v.pad_w = p.pad_w;
    v.BN = p.BN;
    v.J = p.vJ;
    v.nacc = p.vnacc;
    v.n_k = p.vn_k;
    v.n_odb = p.vn_odb;
    v.units = p.units;
    v.stages = p.stages;
    uint32_t cols = 32;
    while (cols < static_cast<uint32_t>(p.vnacc * p.vJ * p.BN)) cols <<= 1;
    v.tmem_cols = cols;
    v.bias = bias;
    v.status = dev->status;
    v.timeout_ns = cfg.timeout_ns;
    v.starve = cfg.starve;
    const int grid = p.units < dev->sms ? p.units : dev->sms;
    cudaEvent_t ev_start = g_main_start, ev_stop = g_main_stop;
    if (ev_start && ev_stop && (st = record_event(ev_start, stream)) != CONV_OK) return st;
    cudaError_t e = launch_vol_reuse(v, grid, p.smem, stream);
    if ((st = check_launch(e, "3-D product with input-slice reuse")) != CONV_OK) return st;
    if (ev_start && ev_stop && (st = record_event(ev_stop, stream)) != CONV_OK) return st;
    return ok();
}

// The pointwise path with resident weights (pw.cu): one kernel, no scratch.
int pw_impl(const Plan &p, const void *x, const void *w_packed, const void *bias, void *y, DeviceInfo *dev,
            const Settings &cfg, cudaStream_t stream, float *partial_out) {
    const bool out_f32 = partial_out != nullptr;
    void *dst = out_f32 ? static_cast<void *>(partial_out) : y;
    PwParams k;
    std::memset(&k, 0, sizeof(k));
    int st = encode_a_xcol(p, x, &k.tmap_a);
    if (st != CONV_OK) return st;
    st = encode_b(p, w_packed, &k.tmap_b);
    if (st != CONV_OK) return st;
    {
        const int oelt = out_f32 ? 4 : p.elt;
        cuuint64_t dims[2] = {static_cast<cuuint64_t>(p.C_out), static_cast<cuuint64_t>(p.M)};
        cuuint64_t strides[1] = {static_cast<cuuint64_t>(p.C_out) * oelt};
        cuuint32_t box[2] = {out_f32 ? 32u : 64u, 32};  // 32 rows x 128 bytes
        cuuint32_t estr[2] = {1, 1};
        CUresult r = g_encode_tiled(&k.tmap_y, out_f32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : tma_type(p), 2, dst, dims,
                                    strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                                    CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
        if (r != CUDA_SUCCESS)
            return fail(CONV_ERR_CUDA, "cuTensorMapEncodeTiled (output) failed (%d)", static_cast<int>(r));
    }
    k.M = static_cast<int>(p.M);
    k.nk = p.Cin_g / 64;
    k.groups = p.groups;
    k.Kp = p.Kp;
    k.Cout_g = p.Cout_g;
    k.out_f32 = out_f32 ? 1 : 0;
    k.ybufs = p.pw_ybufs;
    k.BN = p.BN;
    k.n_ntiles = p.n_ntiles;
    k.m_tiles = static_cast<int>((p.M + 255) / 256);
    k.cpn = p.pair_clusters / (p.n_ntiles * p.groups);
    k.stages = p.stages;
    k.tmem_cols = 512;
    k.bias = out_f32 ? nullptr : bias;
    k.status = dev->status;
    k.timeout_ns = cfg.timeout_ns;
    k.starve = cfg.starve;
    cudaEvent_t ev_start = g_main_start, ev_stop = g_main_stop;
    if (ev_start && ev_stop && (st = record_event(ev_start, stream)) != CONV_OK) return st;
    cudaError_t e = launch_pw(k, p.smem, stream);
    if ((st = check_launch(e, "pointwise product with resident weights")) != CONV_OK) return st;
    if (ev_start && ev_stop && (st = record_event(ev_stop, stream)) != CONV_OK) return st;
    return ok();
}

// Shared body of conv2d_forward and conv2d_forward_im2col_gemm.
int forward_impl(bool explicit_im2col, const void *x, const void *w_packed, const void *bias, void *y,
                 int N, int C_in, int H, int W, int C_out, int Kh, int Kw, int stride, int pad,
                 int dilation, int groups, conv_dtype_t dtype, conv_layout_t layout, void *workspace,
                 size_t workspace_bytes, cudaStream_t stream, const PadW *padw = nullptr,
                 const Vol *vol = nullptr) {
    const Settings cfg = settings_now();
    DeviceInfo *dev = nullptr;
    Plan p;
    int st = make_plan(N, C_in, H, W, C_out, Kh, Kw, stride, pad, dilation, groups, dtype, layout,
                       explicit_im2col, 0, &p, cfg.pair_mode, true, padw, vol);
    if (st != CONV_OK) return st;
    if (!x || !w_packed || !y) return fail(CONV_ERR_INVALID_ARG, "x, w_packed and y must not be NULL");
    st = device_info(&dev);
    if (st != CONV_OK) return st;
    st = device_plan(explicit_im2col, N, C_in, H, W, C_out, Kh, Kw, stride, pad, dilation, groups, dtype,
                     layout, dev, cfg, &p, padw, vol);
    if (st != CONV_OK) return st;
    const bool a_im2col = !(explicit_im2col || p.direct_a);
    const int pair_clusters = p.pair_clusters;
    if (p.ws_total > 0 && (!workspace || workspace_bytes < p.ws_total))
        return fail(CONV_ERR_WORKSPACE, "workspace of %zu bytes needed, %zu given", p.ws_total,
                    workspace ? workspace_bytes : static_cast<size_t>(0));
    if (!aligned16(x) || !aligned16(w_packed) || !aligned16(y) || (bias && !aligned16(bias)) ||
        (workspace && !aligned16(workspace)))
        return fail(CONV_ERR_UNSUPPORTED, "device pointers must be 16-byte aligned");

    if (p.gather) return gather_impl(p, x, w_packed, bias, y, dev, cfg, stream);
    if (p.dw) return dw_impl(p, x, w_packed, bias, y, workspace, dev, cfg, stream);
    if (p.vreuse) return vol_impl(p, x, w_packed, bias, y, dev, cfg, stream);
    if (p.pw) return pw_impl(p, x, w_packed, bias, y, dev, cfg, stream, padw ? padw->partial_out : nullptr);

    uint8_t *ws = static_cast<uint8_t *>(workspace);
    const void *x_nhwc = p.xcopy ? static_cast<const void *>(ws + p.off_xcopy) : x;
    void *xcol = explicit_im2col ? static_cast<void *>(ws + p.off_xcol) : nullptr;

    IgemmParams kp;
    std::memset(&kp, 0, sizeof(kp));
    st = explicit_im2col ? encode_a_xcol(p, xcol, &kp.tmap_a)
         : p.direct_a    ? encode_a_xcol(p, x_nhwc, &kp.tmap_a)
         : p.vol         ? encode_a_im2col_5d(p, x_nhwc, &kp.tmap_a)
                         : encode_a_im2col(p, x_nhwc, &kp.tmap_a);
    if (st != CONV_OK) return st;
    st = encode_b(p, w_packed, &kp.tmap_b);
    if (st != CONV_OK) return st;
    kp.M = static_cast<int>(p.M);
    kp.HoWo = p.Do * p.Ho * p.Wo;
    kp.HoWo2 = p.Ho * p.Wo;
    kp.Kh = Kh;
    kp.Wo = p.Wo;
    kp.stride = stride;
    kp.stride_w = p.stride_w;
    kp.pad = p.pad;
    kp.pad_w = p.pad_w;
    kp.dilation = dilation;
    kp.Kw = Kw;
    kp.taps = p.taps;
    kp.Cpg = p.Cpg;
    kp.nCB = p.nCB;
    kp.planes = p.planes;
    kp.kstages = p.kstages;
    kp.Kp = p.Kp;
    kp.groups = p.groups;
    kp.Cout_g = p.Cout_g;
    kp.Cout = C_out;
    kp.BN = p.BN;
    kp.n_mtiles = p.n_mtiles;
    kp.n_ntiles = p.n_ntiles;
    kp.splits = p.splits;
    kp.units = p.units;
    kp.stages = p.stages;
    // fp32: four stages (16 TF32 k-steps, 48 instructions) per tensor-memory chunk.
    kp.chunk_stages = p.f32 ? 4 : 0;
    uint32_t cols = 32;
    while (cols < static_cast<uint32_t>(2 * p.BN)) cols <<= 1;
    kp.tmem_cols = cols;
    kp.bias = bias;
    const bool external_partial = padw && padw->partial_out;
    if (p.splits > 1 || external_partial) {
        kp.y = external_partial ? static_cast<void *>(padw->partial_out) : static_cast<void *>(ws + p.off_partial);
        kp.out_mode = kOutPartial;
        kp.vec_ok = (C_out % 4 == 0 && p.Cout_g % 4 == 0) ? 1 : 0;
    } else {
        kp.y = y;
        kp.out_mode = layout == CONV_NCHW ? kOutNCHW : kOutNHWC;
        const int per16 = 16 / p.elt;
        kp.vec_ok = (C_out % per16 == 0 && p.Cout_g % per16 == 0) ? 1 : 0;
    }
    kp.status = dev->status;
    kp.timeout_ns = cfg.timeout_ns;
    kp.starve = cfg.starve;
    kp.tma_out = (p.tma_out && p.splits == 1) ? 1 : 0;
    if (kp.tma_out) {
        cuuint64_t dims[2] = {static_cast<cuuint64_t>(C_out), static_cast<cuuint64_t>(p.M)};
        cuuint64_t strides[1] = {static_cast<cuuint64_t>(C_out) * p.elt};
        cuuint32_t box[2] = {32, 32};
        cuuint32_t estr[2] = {1, 1};
        CUresult r = g_encode_tiled(&kp.tmap_y, tma_type(p), 2, y, dims, strides, box, estr,
                                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B,
                                    CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
        if (r != CUDA_SUCCESS)
            return fail(CONV_ERR_CUDA, "cuTensorMapEncodeTiled (output) failed (%d)", static_cast<int>(r));
    }

    if (p.xcopy) {
        cudaError_t e = layout == CONV_NCHW
                            ? launch_nchw_to_nhwc(x, ws + p.off_xcopy, N, C_in, p.D * H, W, p.groups, p.Cpg, p.elt,
                                                  stream)
                            : launch_nhwc_pad(x, ws + p.off_xcopy, N, C_in, p.D * H, W, p.groups, p.Cpg, p.elt, stream);
        if ((st = check_launch(e, "channels-last copy")) != CONV_OK) return st;
    }
    if (explicit_im2col) {
        cudaError_t e = launch_im2col(x_nhwc, xcol, N, H, W, p.groups, p.Cpg, p.Ho, p.Wo, Kh, Kw,
                                      stride, pad, dilation, p.elt, stream);
        if ((st = check_launch(e, "im2col")) != CONV_OK) return st;
    }
    // one CTA per SM, or one cluster per SM pair, each looping over units of work
    const int grid = p.pair ? 2 * (p.units < pair_clusters ? p.units : pair_clusters)
                            : (p.units < dev->sms ? p.units : dev->sms);
    cudaEvent_t ev_start = g_main_start, ev_stop = g_main_stop;
    if (ev_start && ev_stop && (st = record_event(ev_start, stream)) != CONV_OK) return st;
    // a 1x1x1 stride-1 unpadded volume reads x itself as X_col (tiled loads), like 2-D
    cudaError_t e = launch_igemm(kp, p.f32, p.cb, a_im2col, p.pair, grid, p.smem, stream, p.vol && a_im2col);
    if ((st = check_launch(e, "tensor-core product")) != CONV_OK) return st;
    if (ev_start && ev_stop && (st = record_event(ev_stop, stream)) != CONV_OK) return st;
    if (p.splits > 1 && !external_partial) {
        e = launch_splitk_reduce(reinterpret_cast<const float *>(ws + p.off_partial), bias, y,
                                 static_cast<int>(p.M), C_out, p.Do * p.Ho * p.Wo, p.splits,
                                 layout == CONV_NCHW ? kOutNCHW : kOutNHWC, p.f32, stream);
        if ((st = check_launch(e, "split reduction")) != CONV_OK) return st;
    }
    return ok();
}

// The plan as a JSON object, for callers and tests that want to know which kernel,
// tile shape and passes a problem gets.  sms < 0: this process's current device (none:
// no device-dependent choices); sms >= 0: as if the device had that many SMs.
int describe_impl(bool explicit_im2col, int N, int C_in, int H, int W, int C_out, int Kh, int Kw,
                  int stride, int pad, int dilation, int groups, conv_dtype_t dtype,
                  conv_layout_t layout, int sms, char *buf, size_t buflen, const Vol *vol = nullptr,
                  const PadW *padw = nullptr, int fold = 0, size_t ws_extra = 0) {
    if (!buf || buflen == 0) return fail(CONV_ERR_INVALID_ARG, "buf must not be NULL");
    const Settings cfg = settings_now();
    Plan p;
    int st = make_plan(N, C_in, H, W, C_out, Kh, Kw, stride, pad, dilation, groups, dtype, layout,
                       explicit_im2col, 0, &p, cfg.pair_mode, true, padw, vol);
    if (st != CONV_OK) return st;
    if (sms < 0) {
        DeviceInfo *dev = current_device_or_null();
        sms = dev ? dev->sms : 0;
        st = device_plan(explicit_im2col, N, C_in, H, W, C_out, Kh, Kw, stride, pad, dilation, groups,
                         dtype, layout, dev, cfg, &p, padw, vol);
    } else {
        st = make_plan(N, C_in, H, W, C_out, Kh, Kw, stride, pad, dilation, groups, dtype, layout,
                       explicit_im2col, sms, &p, cfg.pair_mode, true, padw, vol);
    }
    if (st != CONV_OK) return st;
    const char *a_load = p.dw ? "tile" : p.gather ? "gather" : explicit_im2col ? "xcol" : p.direct_a ? "tiled_x" : "im2col";
    const char *kernel = p.dw ? "depthwise" : p.vreuse ? "vol_reuse" : p.pw ? "pointwise" : p.gather_t ? "gather_t" : p.gather ? "gather" : "igemm";
    const int n = std::snprintf(
        buf, buflen,
        "{\"kernel\": \"%s\", \"pair\": %d, \"a_load\": \"%s\", \"BN\": %d, \"cb\": %d, "
        "\"stages\": %d, \"splits\": %d, \"units\": %d, \"xcopy\": %d, \"halo\": %d, "
        "\"tma_out\": %d, \"Kpad\": %d, \"smem\": %zu, \"workspace\": %zu, \"sms\": %d, "
        "\"rows\": %d, \"out_images\": %d, \"a_tmem\": %d, \"fold\": %d}",
        kernel, p.pair ? 1 : 0, a_load, p.BN, p.gather ? 0 : p.cb,
        p.stages, p.gather ? 1 : p.splits, p.gather ? p.n_mtiles : p.units, p.xcopy ? 1 : 0,
        p.halo ? 1 : 0, p.tma_out ? 1 : 0, p.gather ? p.Kpad : 0, p.smem, p.ws_total + ws_extra, sms,
        p.gather_t ? p.rt : 0, p.gather_t && p.tma_out ? p.nout : 0, p.gather_t && p.a_tmem ? 1 : 0, fold);
    if (n < 0 || static_cast<size_t>(n) >= buflen)
        return fail(CONV_ERR_INVALID_ARG, "buf of %zu bytes is too small (%d needed)", buflen, n + 1);
    return ok();
}

int workspace_impl(bool explicit_im2col, int N, int C_in, int H, int W, int C_out, int Kh, int Kw,
                   int stride, int pad, int dilation, int groups, conv_dtype_t dtype,
                   conv_layout_t layout, size_t *bytes, const PadW *padw = nullptr, const Vol *vol = nullptr) {
    if (!bytes) return fail(CONV_ERR_INVALID_ARG, "bytes must not be NULL");
    const Settings cfg = settings_now();
    Plan p;
    int st = make_plan(N, C_in, H, W, C_out, Kh, Kw, stride, pad, dilation, groups, dtype, layout,
                       explicit_im2col, 0, &p, cfg.pair_mode, true, padw, vol);
    if (st != CONV_OK) return st;
    // with no usable device: sized without reduction splits or CTA pairs
    st = device_plan(explicit_im2col, N, C_in, H, W, C_out, Kh, Kw, stride, pad, dilation, groups, dtype,
                     layout, current_device_or_null(), cfg, &p, padw, vol);
    if (st != CONV_OK) return st;
    *bytes = p.ws_total;
    return ok();
}

int elt_of(conv_dtype_t dtype) { return dtype == CONV_F32 ? 4 : dtype == CONV_BF16 ? 2 : 0; }

// Device address of the built-in scratch on the current device, looked up on the
// first use per device (with that device current) and cached.
int noalloc_scratch(void **out) {
    DeviceInfo *dev = nullptr;
    int st = device_info(&dev);
    if (st != CONV_OK) return st;
    std::lock_guard<std::mutex> lock(g_mutex);
    if (!dev->noalloc_scratch) {
        void *ptr = nullptr;
        cudaError_t e = cudaGetSymbolAddress(&ptr, g_noalloc_scratch);
        if (e != cudaSuccess || !ptr)
            return fail(CONV_ERR_CUDA, "built-in scratch address: %s", cudaGetErrorString(e));
        dev->noalloc_scratch = ptr;
    }
    *out = dev->noalloc_scratch;
    return CONV_OK;
}


// ----------------------------------------------------------------- backward ---
// Weight gradient plan: the tensor-core kernel (wgrad.cu) when a group has at least 32
// bytes of input channels, else the CUDA-core kernel (depthwise and other few-channel
// groups).  Scratch: [x copy][dy copy][fp32 partial sums][bias-gradient partials].
struct WgPlan {
    Plan f;                       // the forward problem: validation, Ho, Wo, M
    bool tc;                      // tensor-core kernel
    int Cin_g, Cout_g, Cpg, dy_cpg, BN, n_ctiles, n_otiles, taps, kstages, splits, units, stages;
    int om;                       // 128-row output-channel tiles per unit (n_otiles counts units' worth)
    bool xcopy, dycopy;
    size_t smem, off_xcopy, off_dycopy, off_ws, off_db, ws_total;
    int db_partials;
};

int wgrad_plan(int N, int C_in, int H, int W, int C_out, int Kh, int Kw, int stride, int pad, int dilation,
               int groups, conv_dtype_t dtype, conv_layout_t layout, bool want_db, int sms, WgPlan *out) {
    WgPlan w{};
    int st = make_plan(N, C_in, H, W, C_out, Kh, Kw, stride, pad, dilation, groups, dtype, layout, false, 0,
                       &w.f, 2);
    if (st != CONV_OK) return st;
    const Plan &f = w.f;
    const int elt = f.elt;
    w.Cin_g = C_in / groups;
    w.Cout_g = C_out / groups;
    w.taps = Kh * Kw;
    w.tc = w.Cin_g * elt >= 32;
    const int align = 16 / elt;
    size_t off = 0;
    if (w.tc) {
        const int cc = 128 / elt;
        w.Cpg = round_up(w.Cin_g, cc);
        w.dy_cpg = round_up(w.Cout_g, align);
        w.xcopy = layout == CONV_NCHW || w.Cpg != w.Cin_g;
        w.dycopy = layout == CONV_NCHW || w.dy_cpg != w.Cout_g;
        const int cap = f.f32 ? 64 : 256;  // fp32 stages hold raw, hi and lo copies
        for (w.BN = cap; w.BN > cc && w.Cpg % w.BN != 0; w.BN -= cc) {
        }
        w.n_ctiles = w.Cpg / w.BN;
        w.n_otiles = (w.Cout_g + 127) / 128;
        // bf16 with an even number of 128-row tiles: two per unit (one staged block of x
        // feeds both), when both accumulators fit in tensor memory
        w.om = (!f.f32 && w.n_otiles % 2 == 0 && 2 * w.BN <= 512) ? 2 : 1;
        w.n_otiles /= w.om;
        const int pk = wgrad_pixels_per_stage(f.f32);
        const long long kst = (f.M + pk - 1) / pk;
        const long long base = static_cast<long long>(w.n_otiles) * groups * w.taps * w.n_ctiles;
        if (base * 64 >= (1LL << 31) || kst >= (1LL << 30)) return fail(CONV_ERR_UNSUPPORTED, "too many tiles");
        w.kstages = static_cast<int>(kst);
        w.splits = 1;
        if (sms > 0 && base < sms) {
            long long sp = sms / base;
            sp = sp < w.kstages / 4 ? sp : w.kstages / 4;
            sp = sp < 64 ? sp : 64;
            w.splits = sp > 1 ? static_cast<int>(sp) : 1;
        }
        w.units = static_cast<int>(base * w.splits);
        const size_t fixed = wgrad_smem_bytes(f.f32, w.BN, 0, w.om);
        const size_t stage = wgrad_smem_bytes(f.f32, w.BN, 1, w.om) - fixed;
        int stages = static_cast<int>((kSmemBudget - fixed) / stage);
        w.stages = stages > wgrad_max_stages() ? wgrad_max_stages() : stages;
        if (w.stages < 2) return fail(CONV_ERR_UNSUPPORTED, "weight-gradient tile does not fit in shared memory");
        w.smem = wgrad_smem_bytes(f.f32, w.BN, w.stages, w.om);
    } else {
        // CUDA cores: channels-last copies without padding, splits over rows of pixels
        w.Cpg = w.Cin_g;
        w.dy_cpg = w.Cout_g;
        w.xcopy = w.dycopy = layout == CONV_NCHW;
        const long long elems = static_cast<long long>(C_out) * w.taps * w.Cin_g;
        const long long rows = static_cast<long long>(N) * f.Ho;
        long long sp = (148LL * 1024 + elems - 1) / elems;
        sp = sp < rows ? sp : rows;
        sp = sp < 256 ? sp : 256;
        w.splits = sp > 1 ? static_cast<int>(sp) : 1;
    }
    w.off_xcopy = off;
    if (w.xcopy) off = align_up(off + static_cast<size_t>(N) * H * W * groups * w.Cpg * elt, 256);
    w.off_dycopy = off;
    if (w.dycopy) off = align_up(off + static_cast<size_t>(f.M) * groups * w.dy_cpg * elt, 256);
    w.off_ws = off;
    off = align_up(off + static_cast<size_t>(w.splits) * C_out * w.taps * w.Cpg * 4, 256);
    w.off_db = off;
    w.db_partials = want_db ? bias_grad_partials(f.M, C_out, N, layout == CONV_NCHW) : 0;
    if (want_db) off = align_up(off + static_cast<size_t>(w.db_partials) * C_out * 4, 256);
    w.ws_total = off;
    *out = w;
    return CONV_OK;
}

// Copies x or dy into channels-last with `cpg` channels per group (zero padding) when the
// plan asks for it; returns the tensor the kernels read.
int to_channels_last(bool copy, const void *src, uint8_t *dst, int N, int C, int H, int W, int groups, int cpg,
                     const Plan &f, cudaStream_t stream, const void **out) {
    *out = src;
    if (!copy) return CONV_OK;
    cudaError_t e = f.layout == CONV_NCHW ? launch_nchw_to_nhwc(src, dst, N, C, H, W, groups, cpg, f.elt, stream)
                                          : launch_nhwc_pad(src, dst, N, C, H, W, groups, cpg, f.elt, stream);
    int st = check_launch(e, "channels-last copy");
    if (st != CONV_OK) return st;
    *out = dst;
    return CONV_OK;
}

int bias_grad_impl(const Plan &f, const void *dy, void *db, float *partials, cudaStream_t stream) {
    return check_launch(launch_bias_grad(dy, partials, db, f.N, f.C_out, static_cast<long long>(f.Ho) * f.Wo,
                                         f.layout == CONV_NCHW, f.f32, stream),
                        "bias gradient");
}

int backward_weight_impl(const void *x, const void *dy, void *dw, void *db, int N, int C_in, int H, int W,
                         int C_out, int Kh, int Kw, int stride, int pad, int dilation, int groups,
                         conv_dtype_t dtype, conv_layout_t layout, void *workspace, size_t workspace_bytes,
                         cudaStream_t stream) {
    const Settings cfg = settings_now();
    WgPlan w;
    int st = wgrad_plan(N, C_in, H, W, C_out, Kh, Kw, stride, pad, dilation, groups, dtype, layout, db != nullptr,
                        0, &w);
    if (st != CONV_OK) return st;
    if (!x || !dy || !dw) return fail(CONV_ERR_INVALID_ARG, "x, dy and dw must not be NULL");
    DeviceInfo *dev = nullptr;
    if ((st = device_info(&dev)) != CONV_OK) return st;
    st = wgrad_plan(N, C_in, H, W, C_out, Kh, Kw, stride, pad, dilation, groups, dtype, layout, db != nullptr,
                    dev->sms, &w);
    if (st != CONV_OK) return st;
    if (!workspace || workspace_bytes < w.ws_total)
        return fail(CONV_ERR_WORKSPACE, "workspace of %zu bytes needed, %zu given", w.ws_total,
                    workspace ? workspace_bytes : static_cast<size_t>(0));
    if (!aligned16(x) || !aligned16(dy) || !aligned16(dw) || (db && !aligned16(db)) || !aligned16(workspace))
        return fail(CONV_ERR_UNSUPPORTED, "device pointers must be 16-byte aligned");
    const Plan &f = w.f;
    uint8_t *ws = static_cast<uint8_t *>(workspace);
    float *partial = reinterpret_cast<float *>(ws + w.off_ws);
    if (db && (st = bias_grad_impl(f, dy, db, reinterpret_cast<float *>(ws + w.off_db), stream)) != CONV_OK)
        return st;
    const void *xl = nullptr, *dyl = nullptr;
    if ((st = to_channels_last(w.xcopy, x, ws + w.off_xcopy, N, C_in, H, W, w.tc ? groups : 1,
                               w.tc ? w.Cpg : C_in, f, stream, &xl)) != CONV_OK)
        return st;
    if ((st = to_channels_last(w.dycopy, dy, ws + w.off_dycopy, N, C_out, f.Ho, f.Wo, w.tc ? groups : 1,
                               w.tc ? w.dy_cpg : C_out, f, stream, &dyl)) != CONV_OK)
        return st;
    cudaEvent_t ev_start = g_main_start, ev_stop = g_main_stop;
    if (!w.tc) {
        if (ev_start && ev_stop && (st = record_event(ev_start, stream)) != CONV_OK) return st;
        if ((st = check_launch(launch_wgrad_direct(xl, dyl, partial, N, C_in, H, W, C_out, f.Ho, f.Wo, Kh, Kw, stride,
                                                   pad, dilation, groups, w.splits, f.f32, stream),
                               "weight gradient (CUDA cores)")) != CONV_OK)
            return st;
        if (ev_start && ev_stop && (st = record_event(ev_stop, stream)) != CONV_OK) return st;
    } else {
        WgradParams k;
        std::memset(&k, 0, sizeof(k));
        const int elt = f.elt, cc = 128 / elt, pk = wgrad_pixels_per_stage(f.f32);
        {
            cuuint64_t dims[2] = {static_cast<cuuint64_t>(groups) * w.dy_cpg, static_cast<cuuint64_t>(f.M)};
            cuuint64_t strides[1] = {static_cast<cuuint64_t>(groups) * w.dy_cpg * elt};
            cuuint32_t box[2] = {static_cast<cuuint32_t>(cc), static_cast<cuuint32_t>(pk)};
            cuuint32_t estr[2] = {1, 1};
            CUresult r = g_encode_tiled(&k.tmap_dy, tma_type(f), 2, const_cast<void *>(dyl), dims, strides, box, estr,
                                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
            if (r != CUDA_SUCCESS)
                return fail(CONV_ERR_CUDA, "cuTensorMapEncodeTiled (output gradient) failed (%d)", static_cast<int>(r));
        }
        {
            const cuuint64_t ctot = static_cast<cuuint64_t>(groups) * w.Cpg;
            cuuint64_t dims[4] = {ctot, static_cast<cuuint64_t>(W), static_cast<cuuint64_t>(H),
                                  static_cast<cuuint64_t>(N)};
            cuuint64_t strides[3] = {ctot * elt, ctot * elt * W, ctot * elt * W * H};
            int lower[2] = {-pad, -pad};
            int upper[2] = {pad - (Kw - 1) * dilation, pad - (Kh - 1) * dilation};
            cuuint32_t estr[4] = {1, static_cast<cuuint32_t>(stride), static_cast<cuuint32_t>(stride), 1};
            CUresult r = g_encode_im2col(&k.tmap_x, tma_type(f), 4, const_cast<void *>(xl), dims, strides, lower, upper,
                                         static_cast<cuuint32_t>(cc), static_cast<cuuint32_t>(pk), estr,
                                         CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                                         CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
            if (r != CUDA_SUCCESS)
                return fail(CONV_ERR_CUDA, "cuTensorMapEncodeIm2col (input) failed (%d)", static_cast<int>(r));
        }
        k.ws = partial;
        k.M = static_cast<int>(f.M);
        k.HoWo = f.Ho * f.Wo;
        k.Wo = f.Wo;
        k.stride = stride;
        k.pad = pad;
        k.dilation = dilation;
        k.Kw = Kw;
        k.taps = w.taps;
        k.Cpg = w.Cpg;
        k.dy_cpg = w.dy_cpg;
        k.Cout = C_out;
        k.Cout_g = w.Cout_g;
        k.groups = groups;
        k.BN = w.BN;
        k.n_ctiles = w.n_ctiles;
        k.n_otiles = w.n_otiles;
        k.om = w.om;
        k.kstages = w.kstages;
        k.splits = w.splits;
        k.units = w.units;
        k.stages = w.stages;
        k.chunk_stages = f.f32 ? 4 : 0;
        k.tmem_cols = 2 * w.BN <= 256 ? (2 * w.BN <= 128 ? 128 : 256) : 512;  // two sets, or two tiles
        k.status = dev->status;
        k.timeout_ns = cfg.timeout_ns;
        k.starve = cfg.starve;
        const int grid = w.units < dev->sms ? w.units : dev->sms;
        if (ev_start && ev_stop && (st = record_event(ev_start, stream)) != CONV_OK) return st;
        if ((st = check_launch(launch_wgrad(k, f.f32, grid, w.smem, stream), "weight gradient")) != CONV_OK) return st;
        if (ev_start && ev_stop && (st = record_event(ev_stop, stream)) != CONV_OK) return st;
    }
    if ((st = check_launch(launch_wgrad_reduce(partial, dw, C_out, w.Cin_g, w.taps, w.Cpg, w.splits, f.f32, stream),
                           "weight-gradient reduction")) != CONV_OK)
        return st;
    return ok();
}

// Input gradient: the transposed convolution, run as a forward convolution of dy (or of
// dy with s-1 zeros inserted between its rows and columns when stride s > 1) with the
// spatially flipped, channel-exchanged kernel, stride 1 and padding d*(K-1) - pad.
struct DgradShape {
    int Hi, Wi;          // extent of the tensor the inner convolution reads
    int pad_h, pad_w;    // its padding
    bool zeros;          // dy goes through zero insertion first
    size_t zbytes;       // bytes of the zero-inserted dy
};

int dgrad_shape(const Plan &f, DgradShape *d) {
    d->pad_h = f.dilation * (f.Kh - 1) - f.pad;
    d->pad_w = f.dilation * (f.Kw - 1) - f.pad;
    d->zeros = f.stride > 1;
    if (d->zeros) {
        d->Hi = f.H - f.dilation * (f.Kh - 1) + 2 * f.pad;
        d->Wi = f.W - f.dilation * (f.Kw - 1) + 2 * f.pad;
    } else {
        d->Hi = f.Ho;
        d->Wi = f.Wo;
    }
    d->zbytes = d->zeros ? align_up(static_cast<size_t>(f.N) * d->Hi * d->Wi * f.C_out * f.elt, 256) : 0;
    return CONV_OK;
}

int backward_data_impl(const void *dy, const void *w_packed_t, void *dx, int N, int C_in, int H, int W, int C_out,
                       int Kh, int Kw, int stride, int pad, int dilation, int groups, conv_dtype_t dtype,
                       conv_layout_t layout, void *workspace, size_t workspace_bytes, cudaStream_t stream,
                       size_t *bytes_only) {
    Plan f;
    int st = make_plan(N, C_in, H, W, C_out, Kh, Kw, stride, pad, dilation, groups, dtype, layout, false, 0, &f, 2);
    if (st != CONV_OK) return st;
    DgradShape d;
    dgrad_shape(f, &d);
    const PadW pw{d.pad_w};
    if (bytes_only) {
        size_t inner = 0;
        st = workspace_impl(false, N, C_out, d.Hi, d.Wi, C_in, Kh, Kw, 1, d.pad_h, dilation, groups, dtype, layout,
                            &inner, &pw);
        if (st != CONV_OK) return st;
        *bytes_only = d.zbytes + inner;
        return ok();
    }
    if (!dy || !w_packed_t || !dx) return fail(CONV_ERR_INVALID_ARG, "dy, w_packed_t and dx must not be NULL");
    if (d.zbytes > 0 && (!workspace || workspace_bytes < d.zbytes))
        return fail(CONV_ERR_WORKSPACE, "workspace of at least %zu bytes needed, %zu given", d.zbytes,
                    workspace ? workspace_bytes : static_cast<size_t>(0));
    if (!aligned16(dy) || !aligned16(w_packed_t) || !aligned16(dx) || (workspace && !aligned16(workspace)))
        return fail(CONV_ERR_UNSUPPORTED, "device pointers must be 16-byte aligned");
    const void *src = dy;
    uint8_t *ws = static_cast<uint8_t *>(workspace);
    if (d.zeros) {
        // validate the inner convolution before anything is enqueued
        size_t inner = 0;
        st = workspace_impl(false, N, C_out, d.Hi, d.Wi, C_in, Kh, Kw, 1, d.pad_h, dilation, groups, dtype, layout,
                            &inner, &pw);
        if (st != CONV_OK) return st;
        if (workspace_bytes < d.zbytes + inner)
            return fail(CONV_ERR_WORKSPACE, "workspace of %zu bytes needed, %zu given", d.zbytes + inner,
                        workspace_bytes);
        if ((st = check_launch(launch_zero_insert(dy, ws, N, C_out, f.Ho, f.Wo, d.Hi, d.Wi, stride,
                                                  layout == CONV_NCHW, f.elt, stream),
                               "zero insertion")) != CONV_OK)
            return st;
        src = ws;
    }
    return forward_impl(false, src, w_packed_t, nullptr, dx, N, C_out, d.Hi, d.Wi, C_in, Kh, Kw, 1, d.pad_h,
                        dilation, groups, dtype, layout, ws ? ws + d.zbytes : nullptr,
                        workspace_bytes > d.zbytes ? workspace_bytes - d.zbytes : 0, stream, &pw);
}

// A few-channel 3-D layer as a 2-D one over its (kd, kh)-folded input (layout.cu's
// fold3d): hardware im2col would move one narrow row (C_in channels, at most 16 bytes) per
// voxel and tap, Kd*Kh*Kw of them; folded, each voxel row holds the Kd*Kh taps' channels
// (Cf, padded to 64 bytes) and a 1 x Kw convolution with column stride s over an image of
// Do*Ho rows gives the same sums (the volume's im2col, pwwt §5, done in two steps; the
// depth and row strides are taken by the fold).
struct Fold3d {
    int Cf, Do, Ho;
    PadW pw;                       // columns padded by `pad` and strided by s, x channels-last
    size_t off_x, off_w, off_inner, ws_total;
};

bool fold3d_applies(int C_in, int Kd, int Kh, int stride, int groups, conv_dtype_t dtype) {
    const int elt = dtype == CONV_F32 ? 4 : 2;
    // (at 32 bytes per voxel -- the stride-2 layer of 16 channels -- the fold's writes cost
    // more than the rows it saves: 32.6 against 22.6 us per step, so only narrower rows fold)
    return groups == 1 && stride <= 8 && C_in * elt <= 16 && Kd * Kh > 1;
}

int fold3d_plan(int N, int C_in, int D, int H, int W, int C_out, int Kd, int Kh, int Kw, int stride, int pad,
                int dilation, conv_dtype_t dtype, conv_layout_t layout, DeviceInfo *dev, const Settings &cfg,
                Fold3d *f, Plan *inner) {
    const int elt = dtype == CONV_F32 ? 4 : 2;
    if (out_size(D, Kd, stride, pad, dilation, &f->Do) != 0 || out_size(H, Kh, stride, pad, dilation, &f->Ho) != 0)
        return fail(CONV_ERR_INVALID_ARG, "the dilated kernel is larger than the padded input");
    f->Cf = round_up(Kd * Kh * C_in, 64 / elt);
    f->pw = PadW{pad, nullptr, true, stride};
    if (static_cast<long long>(f->Do) * f->Ho >= (1LL << 31) / (W > 0 ? W : 1))
        return fail(CONV_ERR_UNSUPPORTED, "folded volume too large");
    int st = device_plan(false, N, f->Cf, f->Do * f->Ho, W, C_out, 1, Kw, 1, 0, dilation, 1, dtype, layout, dev,
                         cfg, inner, &f->pw);
    if (st != CONV_OK) return st;
    f->off_x = 0;
    size_t off = align_up(static_cast<size_t>(N) * f->Do * f->Ho * W * f->Cf * elt, 256);
    f->off_w = off;
    off = align_up(off + static_cast<size_t>(C_out) * Kw * f->Cf * elt, 256);
    f->off_inner = off;
    f->ws_total = off + inner->ws_total;
    return CONV_OK;
}

int fold3d_forward(const void *x, const void *w_packed, const void *bias, void *y, int N, int C_in, int D, int H,
                   int W, int C_out, int Kd, int Kh, int Kw, int stride, int pad, int dilation, conv_dtype_t dtype,
                   conv_layout_t layout, void *workspace, size_t workspace_bytes, cudaStream_t stream) {
    const Settings cfg = settings_now();
    Fold3d f;
    Plan inner;
    // argument errors first, then the device's plan
    int st = fold3d_plan(N, C_in, D, H, W, C_out, Kd, Kh, Kw, stride, pad, dilation, dtype, layout, nullptr, cfg, &f,
                         &inner);
    if (st != CONV_OK) return st;
    DeviceInfo *dev = nullptr;
    if ((st = device_info(&dev)) != CONV_OK) return st;
    if ((st = fold3d_plan(N, C_in, D, H, W, C_out, Kd, Kh, Kw, stride, pad, dilation, dtype, layout, dev, cfg, &f,
                          &inner)) != CONV_OK)
        return st;
    if (!x || !w_packed || !y) return fail(CONV_ERR_INVALID_ARG, "x, w_packed and y must not be NULL");
    if (!workspace || workspace_bytes < f.ws_total)
        return fail(CONV_ERR_WORKSPACE, "workspace of %zu bytes needed, %zu given", f.ws_total,
                    workspace ? workspace_bytes : static_cast<size_t>(0));
    if (!aligned16(x) || !aligned16(w_packed) || !aligned16(y) || (bias && !aligned16(bias)) || !aligned16(workspace))
        return fail(CONV_ERR_UNSUPPORTED, "device pointers must be 16-byte aligned");
    const int elt = elt_of(dtype);
    uint8_t *ws = static_cast<uint8_t *>(workspace);
    if ((st = check_launch(launch_fold3d(x, ws + f.off_x, w_packed, ws + f.off_w, N, C_in, D, H, W, f.Do, f.Ho, C_out,
                                         Kd, Kh, Kw, round_up(C_in, 16 / elt), stride, pad, dilation, f.Cf, elt,
                                         layout == CONV_NCHW, stream),
                           "depth-and-row fold")) != CONV_OK)
        return st;
    return forward_impl(false, ws + f.off_x, ws + f.off_w, bias, y, N, f.Cf, f.Do * f.Ho, W, C_out, 1, Kw, 1, 0,
                        dilation, 1, dtype, layout, ws + f.off_inner, workspace_bytes - f.off_inner, stream, &f.pw);
}

// ------------------------------------------------------------------ Winograd ---
// F(m x m, 3 x 3), m = 2 or 4 (winograd.cu): input transform -> the tensor-core product
// as a grouped 1x1 convolution with alpha^2 groups over the transformed tiles, fp32
// results -> output transform.  Scratch: [V][M partial sums][the product's own scratch].
struct WinoPlan {
    Plan f;          // the 3x3 problem: validation, Ho, Wo
    Plan g;          // the product
    conv_dtype_t tdt;  // transform and product type (see wino_tdt)
    int m, a, Cpg, TH, TW, T;
    size_t off_v, off_m, off_inner, ws_total;
};

// Type of the transformed tiles and filters and of their product: the data's own for
// F(2x2,3x3), fp32 for F(4x4,3x3) (its bf16 transforms miss the bf16 tolerance).
conv_dtype_t wino_tdt(conv_dtype_t dtype, int m) { return m == 4 ? CONV_F32 : dtype; }

int wino_plan(int N, int C_in, int H, int W, int C_out, int pad, int m, conv_dtype_t dtype, conv_layout_t layout,
              DeviceInfo *dev, const Settings &cfg, WinoPlan *out) {
    WinoPlan w{};
    if (m != 2 && m != 4) return fail(CONV_ERR_INVALID_ARG, "Winograd tile m must be 2 or 4 (F(2x2,3x3), F(4x4,3x3))");
    int st = make_plan(N, C_in, H, W, C_out, 3, 3, 1, pad, 1, 1, dtype, layout, false, 0, &w.f, 2);
    if (st != CONV_OK) return st;
    w.m = m;
    w.a = m + 2;
    w.tdt = wino_tdt(dtype, m);
    const int telt = w.tdt == CONV_F32 ? 4 : 2;
    w.Cpg = round_up(C_in, 16 / telt);
    w.TH = (w.f.Ho + m - 1) / m;
    w.TW = (w.f.Wo + m - 1) / m;
    const long long T = static_cast<long long>(N) * w.TH * w.TW;
    if (T >= (1LL << 31) - 256) return fail(CONV_ERR_UNSUPPORTED, "too many Winograd tiles");
    w.T = static_cast<int>(T);
    const int a2 = w.a * w.a;
    const PadW pw{0, reinterpret_cast<float *>(16)};  // placeholder address: plans the external-partial form
    st = device_plan(false, 1, a2 * w.Cpg, 1, w.T, a2 * C_out, 1, 1, 1, 0, 1, a2, w.tdt, CONV_NHWC, dev, cfg, &w.g,
                     &pw);
    if (st != CONV_OK) return st;
    size_t off = 0;
    w.off_v = off;
    off = align_up(off + static_cast<size_t>(T) * a2 * w.Cpg * telt, 256);
    w.off_m = off;
    off = align_up(off + static_cast<size_t>(w.g.splits) * T * a2 * C_out * 4, 256);
    w.off_inner = off;
    w.ws_total = off + w.g.ws_total;
    *out = w;
    return CONV_OK;
}

int winograd_impl(const void *x, const void *u_packed, const void *bias, void *y, int N, int C_in, int H, int W,
                  int C_out, int pad, int m, conv_dtype_t dtype, conv_layout_t layout, void *workspace,
                  size_t workspace_bytes, cudaStream_t stream, size_t *bytes_only) {
    const Settings cfg = settings_now();
    WinoPlan w;
    int st;
    if (bytes_only) {
        if ((st = wino_plan(N, C_in, H, W, C_out, pad, m, dtype, layout, current_device_or_null(), cfg, &w)) != CONV_OK)
            return st;
        *bytes_only = w.ws_total;
        return ok();
    }
    if ((st = wino_plan(N, C_in, H, W, C_out, pad, m, dtype, layout, nullptr, cfg, &w)) != CONV_OK) return st;
    if (!x || !u_packed || !y) return fail(CONV_ERR_INVALID_ARG, "x, u_packed and y must not be NULL");
    DeviceInfo *dev = nullptr;
    if ((st = device_info(&dev)) != CONV_OK) return st;
    if ((st = wino_plan(N, C_in, H, W, C_out, pad, m, dtype, layout, dev, cfg, &w)) != CONV_OK) return st;
    if (!workspace || workspace_bytes < w.ws_total)
        return fail(CONV_ERR_WORKSPACE, "workspace of %zu bytes needed, %zu given", w.ws_total,
                    workspace ? workspace_bytes : static_cast<size_t>(0));
    if (!aligned16(x) || !aligned16(u_packed) || !aligned16(y) || (bias && !aligned16(bias)) || !aligned16(workspace))
        return fail(CONV_ERR_UNSUPPORTED, "device pointers must be 16-byte aligned");
    uint8_t *ws = static_cast<uint8_t *>(workspace);
    float *mp = reinterpret_cast<float *>(ws + w.off_m);
    const bool nchw = layout == CONV_NCHW;
    if ((st = check_launch(launch_wino_input(x, ws + w.off_v, N, C_in, H, W, w.Cpg, w.TH, w.TW, pad, m, nchw,
                                             w.f.f32, w.tdt == CONV_F32, stream),
                           "Winograd input transform")) != CONV_OK)
        return st;
    const int a2 = w.a * w.a;
    const PadW pw{0, mp};
    if ((st = forward_impl(false, ws + w.off_v, u_packed, nullptr, mp, 1, a2 * w.Cpg, 1, w.T, a2 * C_out, 1, 1, 1, 0,
                           1, a2, w.tdt, CONV_NHWC, ws + w.off_inner, workspace_bytes - w.off_inner, stream, &pw)) !=
        CONV_OK)
        return st;
    return check_launch(launch_wino_output(mp, bias, y, N, C_out, w.f.Ho, w.f.Wo, w.TH, w.TW, w.g.splits, m, nchw,
                                           w.f.f32, stream),
                        "Winograd output transform") == CONV_OK
               ? ok()
               : CONV_ERR_CUDA;
}

// Packed size of the transposed convolution's kernel: C_in output channels of
// C_out/groups reduction channels per group (merged like any narrow group).
int packed_weight_t_bytes(int C_out, int C_in, int Kh, int Kw, int groups, int elt, int *cpg, int *gm) {
    *gm = group_merge(C_in, C_out, groups, elt);
    *cpg = round_up(C_out / groups, 16 / elt) * *gm;
    return 0;
}
}  // namespace
}  // namespace conv2d_b200

using namespace conv2d_b200;

#pragma GCC visibility push(default)
extern "C" {

int conv2d_output_size(int in, int k, int stride, int pad, int dilation, int *out) {
    if (!out || in < 1 || k < 1 || stride < 1 || pad < 0 || dilation < 1)
        return fail(CONV_ERR_INVALID_ARG, "output size: invalid argument");
    int v = 0;
    if (out_size(in, k, stride, pad, dilation, &v) != 0)
        return fail(CONV_ERR_INVALID_ARG, "output size: the dilated kernel is larger than the padded input");
    *out = v;
    return ok();
}

int conv2d_packed_weight_size(int C_out, int C_in, int Kh, int Kw, int groups, conv_dtype_t dtype,
                              size_t *bytes) {
    const int elt = elt_of(dtype);
    if (!bytes || elt == 0 || C_out < 1 || C_in < 1 || Kh < 1 || Kw < 1 || groups < 1 ||
        C_in % groups || C_out % groups)
        return fail(CONV_ERR_INVALID_ARG, "packed weight size: invalid argument");
    *bytes = gather_images(C_out, C_in, Kh, Kw, groups, elt).total;
    return ok();
}

int conv2d_pack_weight(const void *w_oihw, void *w_packed, int C_out, int C_in, int Kh, int Kw,
                       int groups, conv_dtype_t dtype, conv_stream_t stream) {
    size_t bytes = 0;
    int st = conv2d_packed_weight_size(C_out, C_in, Kh, Kw, groups, dtype, &bytes);
    if (st != CONV_OK) return st;
    if (!w_oihw || !w_packed) return fail(CONV_ERR_INVALID_ARG, "weight pointers must not be NULL");
    const int elt = elt_of(dtype);
    const int gm = group_merge(C_out, C_in, groups, elt);
    const int cpg = round_up(C_in / groups, 16 / elt) * gm;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if ((st = check_launch(launch_pack_weight(w_oihw, w_packed, C_out, C_in / groups, C_out / groups, gm, Kh,
                                              Kw, cpg, elt, s),
                           "weight pack")) != CONV_OK)
        return st;
    const GatherImages gi = gather_images(C_out, C_in, Kh, Kw, groups, elt);
    for (int o = 0; o < 2; ++o) {
        if (gi.kpad[o] == 0) continue;
        if ((st = check_launch(launch_pack_gather_image(w_oihw, static_cast<uint8_t *>(w_packed) + gi.off[o],
                                                        C_out, C_in, Kh, Kw, gi.bn, gi.kpad[o], o == 1, elt, s),
                               "weight image")) != CONV_OK)
            return st;
    }
    return ok();
}

int conv2d_workspace_size(int N, int C_in, int H, int W, int C_out, int Kh, int Kw, int stride,
                          int pad, int dilation, int groups, conv_dtype_t dtype,
                          conv_layout_t layout, size_t *bytes) {
    return workspace_impl(false, N, C_in, H, W, C_out, Kh, Kw, stride, pad, dilation, groups, dtype,
                          layout, bytes);
}

int conv2d_im2col_workspace_size(int N, int C_in, int H, int W, int C_out, int Kh, int Kw,
                                 int stride, int pad, int dilation, int groups,
                                 conv_dtype_t dtype, conv_layout_t layout, size_t *bytes) {
    return workspace_impl(true, N, C_in, H, W, C_out, Kh, Kw, stride, pad, dilation, groups, dtype,
                          layout, bytes);
}

int conv2d_forward(const void *x, const void *w_packed, const void *bias, void *y, int N, int C_in,
                   int H, int W, int C_out, int Kh, int Kw, int stride, int pad, int dilation,
                   int groups, conv_dtype_t dtype, conv_layout_t layout, void *workspace,
                   size_t workspace_bytes, conv_stream_t stream) {
    return forward_impl(false, x, w_packed, bias, y, N, C_in, H, W, C_out, Kh, Kw, stride, pad,
                        dilation, groups, dtype, layout, workspace, workspace_bytes,
                        reinterpret_cast<cudaStream_t>(stream));
}

int conv2d_forward_im2col_gemm(const void *x, const void *w_packed, const void *bias, void *y,
                               int N, int C_in, int H, int W, int C_out, int Kh, int Kw,
                               int stride, int pad, int dilation, int groups, conv_dtype_t dtype,
                               conv_layout_t layout, void *workspace, size_t workspace_bytes,
                               conv_stream_t stream) {
    return forward_impl(true, x, w_packed, bias, y, N, C_in, H, W, C_out, Kh, Kw, stride, pad,
                        dilation, groups, dtype, layout, workspace, workspace_bytes,
                        reinterpret_cast<cudaStream_t>(stream));
}

int conv2d_forward_noalloc(const void *x, const void *w_packed, const void *bias, void *y, int N,
                           int C_in, int H, int W, int C_out, int Kh, int Kw, int stride, int pad,
                           int dilation, int groups, conv_dtype_t dtype, conv_layout_t layout,
                           conv_stream_t stream) {
    size_t need = 0;
    int st = workspace_impl(false, N, C_in, H, W, C_out, Kh, Kw, stride, pad, dilation, groups, dtype,
                            layout, &need);
    if (st != CONV_OK) return st;
    if (need > kNoAllocScratchBytes)
        return fail(CONV_ERR_WORKSPACE,
                    "this problem needs %zu bytes of scratch; the built-in scratch of "
                    "conv2d_forward_noalloc holds %zu (use conv2d_forward with a workspace)",
                    need, kNoAllocScratchBytes);
    // The whole array goes to the forward pass, which checks its own plan against it.
    void *scratch = nullptr;
    if ((st = noalloc_scratch(&scratch)) != CONV_OK) return st;
    return forward_impl(false, x, w_packed, bias, y, N, C_in, H, W, C_out, Kh, Kw, stride, pad,
                        dilation, groups, dtype, layout, scratch, kNoAllocScratchBytes,
                        reinterpret_cast<cudaStream_t>(stream));
}

int conv2d_forward_hostio(const void *x_host, void *y_host, void *x_dev, void *y_dev,
                          const void *w_packed, const void *bias, int N, int C_in, int H, int W,
                          int C_out, int Kh, int Kw, int stride, int pad, int dilation, int groups,
                          conv_dtype_t dtype, conv_layout_t layout, void *workspace,
                          size_t workspace_bytes, conv_stream_t stream) {
    Plan p;
    int st = make_plan(N, C_in, H, W, C_out, Kh, Kw, stride, pad, dilation, groups, dtype, layout,
                       false, 0, &p, 0);
    if (st != CONV_OK) return st;
    if (!x_host || !y_host || !x_dev || !y_dev)
        return fail(CONV_ERR_INVALID_ARG, "host and device activation buffers must not be NULL");
    const size_t xi = static_cast<size_t>(C_in) * H * W * p.elt;             // bytes per image
    const size_t yi = static_cast<size_t>(p.Ho) * p.Wo * C_out * p.elt;
    const size_t xb = xi * N, yb = yi * N;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    // Batch chunks of at least 8 MB of input, so that the input copy of one chunk, the
    // product of the one before and the output copy of the one before that run at once
    // (the two copy directions on their own engines).  Chunks start on 16-byte
    // boundaries and must fit the caller's workspace; otherwise one chunk.
    const Settings cfg = settings_now();
    DeviceInfo *dev = nullptr;
    if ((st = device_info(&dev)) != CONV_OK) return st;
    int nch = static_cast<int>(std::min<size_t>(std::min<size_t>(xb / (8u << 20), kHostioChunks), N));
    if (xi % 16 != 0 || yi % 16 != 0) nch = 1;
    while (nch > 1) {
        bool fits = true;
        for (int nc : {N / nch, (N + nch - 1) / nch}) {
            Plan q;
            if (device_plan(false, nc, C_in, H, W, C_out, Kh, Kw, stride, pad, dilation, groups, dtype, layout, dev,
                            cfg, &q) != CONV_OK ||
                q.ws_total > (workspace ? workspace_bytes : 0))
                fits = false;
        }
        if (fits) break;
        nch /= 2;
    }
    if (nch <= 1) {
        cudaError_t e = cudaMemcpyAsync(x_dev, x_host, xb, cudaMemcpyHostToDevice, s);
        if (e != cudaSuccess) return fail(CONV_ERR_CUDA, "input copy: %s", cudaGetErrorString(e));
        st = forward_impl(false, x_dev, w_packed, bias, y_dev, N, C_in, H, W, C_out, Kh, Kw, stride,
                          pad, dilation, groups, dtype, layout, workspace, workspace_bytes, s);
        if (st != CONV_OK) return st;
        e = cudaMemcpyAsync(y_host, y_dev, yb, cudaMemcpyDeviceToHost, s);
        if (e != cudaSuccess) return fail(CONV_ERR_CUDA, "output copy: %s", cudaGetErrorString(e));
        return ok();
    }
    HostioPipe &hp = dev->hio;
    std::lock_guard<std::mutex> pipe_lock(hp.m);
    {
        if (!hp.ready) {
            cudaError_t e = cudaStreamCreateWithFlags(&hp.in, cudaStreamNonBlocking);
            if (e == cudaSuccess) e = cudaStreamCreateWithFlags(&hp.out, cudaStreamNonBlocking);
            if (e == cudaSuccess) e = cudaEventCreateWithFlags(&hp.start, cudaEventDisableTiming);
            if (e == cudaSuccess) e = cudaEventCreateWithFlags(&hp.done, cudaEventDisableTiming);
            for (int i = 0; e == cudaSuccess && i < kHostioChunks; ++i) {
                e = cudaEventCreateWithFlags(&hp.ev_in[i], cudaEventDisableTiming);
                if (e == cudaSuccess) e = cudaEventCreateWithFlags(&hp.ev_comp[i], cudaEventDisableTiming);
            }
            if (e != cudaSuccess) return fail(CONV_ERR_CUDA, "copy pipeline streams: %s", cudaGetErrorString(e));
            hp.ready = true;
        }
    }
    // fork: both copy streams start after the work already on the caller's stream
    cudaError_t e = cudaEventRecord(hp.start, s);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(hp.in, hp.start, 0);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(hp.out, hp.start, 0);
    if (e != cudaSuccess) return fail(CONV_ERR_CUDA, "copy pipeline fork: %s", cudaGetErrorString(e));
    const uint8_t *xh = static_cast<const uint8_t *>(x_host);
    uint8_t *yh = static_cast<uint8_t *>(y_host);
    uint8_t *xd = static_cast<uint8_t *>(x_dev);
    uint8_t *yd = static_cast<uint8_t *>(y_dev);
    int n0 = 0;
    for (int c = 0; c < nch && st == CONV_OK && e == cudaSuccess; ++c) {
        const int nc = N / nch + (c < N % nch ? 1 : 0);
        const size_t xo = static_cast<size_t>(n0) * xi, yo = static_cast<size_t>(n0) * yi;
        e = cudaMemcpyAsync(xd + xo, xh + xo, nc * xi, cudaMemcpyHostToDevice, hp.in);
        if (e == cudaSuccess) e = cudaEventRecord(hp.ev_in[c], hp.in);
        if (e == cudaSuccess) e = cudaStreamWaitEvent(s, hp.ev_in[c], 0);
        if (e != cudaSuccess) break;
        st = forward_impl(false, xd + xo, w_packed, bias, yd + yo, nc, C_in, H, W, C_out, Kh, Kw, stride, pad,
                          dilation, groups, dtype, layout, workspace, workspace_bytes, s);
        if (st != CONV_OK) break;
        e = cudaEventRecord(hp.ev_comp[c], s);
        if (e == cudaSuccess) e = cudaStreamWaitEvent(hp.out, hp.ev_comp[c], 0);
        if (e == cudaSuccess) e = cudaMemcpyAsync(yh + yo, yd + yo, nc * yi, cudaMemcpyDeviceToHost, hp.out);
        n0 += nc;
    }
    // join: the caller's stream continues after the last output copy (also on failure,
    // so that no copy stream is left behind a capture or ahead of later work)
    cudaError_t ej = cudaEventRecord(hp.done, hp.out);
    if (ej == cudaSuccess) ej = cudaStreamWaitEvent(s, hp.done, 0);
    if (ej == cudaSuccess) ej = cudaEventRecord(hp.done, hp.in);
    if (ej == cudaSuccess) ej = cudaStreamWaitEvent(s, hp.done, 0);
    if (st != CONV_OK) return st;
    if (e != cudaSuccess) return fail(CONV_ERR_CUDA, "pipelined copies: %s", cudaGetErrorString(e));
    if (ej != cudaSuccess) return fail(CONV_ERR_CUDA, "copy pipeline join: %s", cudaGetErrorString(ej));
    return ok();
}

int conv2d_nchw_to_nhwc(const void *src, void *dst, int N, int C, int H, int W, int groups,
                        int Cpg, conv_dtype_t dtype, conv_stream_t stream) {
    const int elt = elt_of(dtype);
    if (!src || !dst || elt == 0 || N < 1 || C < 1 || H < 1 || W < 1 || groups < 1 ||
        C % groups || Cpg < C / groups)
        return fail(CONV_ERR_INVALID_ARG, "nchw_to_nhwc: invalid argument");
    if (!aligned16(src) || !aligned16(dst))
        return fail(CONV_ERR_UNSUPPORTED, "device pointers must be 16-byte aligned");
    return check_launch(launch_nchw_to_nhwc(src, dst, N, C, H, W, groups, Cpg, elt,
                                            reinterpret_cast<cudaStream_t>(stream)),
                        "nchw_to_nhwc") == CONV_OK
               ? ok()
               : CONV_ERR_CUDA;
}

int conv2d_nhwc_to_nchw(const void *src, void *dst, int N, int C, int H, int W,
                        conv_dtype_t dtype, conv_stream_t stream) {
    const int elt = elt_of(dtype);
    if (!src || !dst || elt == 0 || N < 1 || C < 1 || H < 1 || W < 1)
        return fail(CONV_ERR_INVALID_ARG, "nhwc_to_nchw: invalid argument");
    return check_launch(launch_nhwc_to_nchw(src, dst, N, C, H, W, elt,
                                            reinterpret_cast<cudaStream_t>(stream)),
                        "nhwc_to_nchw") == CONV_OK
               ? ok()
               : CONV_ERR_CUDA;
}

int conv2d_sync_status(conv_stream_t stream) {
    cudaError_t e = cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return fail(CONV_ERR_CUDA, "stream: %s", cudaGetErrorString(e));
    DeviceInfo *dev = nullptr;
    int st = device_info(&dev);
    if (st != CONV_OK) return st;
    int v = 0;
    e = cudaMemcpy(&v, dev->status, sizeof(int), cudaMemcpyDeviceToHost);
    if (e != cudaSuccess) return fail(CONV_ERR_CUDA, "status read: %s", cudaGetErrorString(e));
    if (v != 0) {
        const int zero = 0;
        cudaMemcpy(dev->status, &zero, sizeof(int), cudaMemcpyHostToDevice);
        return fail(CONV_ERR_TIMEOUT, "device watchdog fired (code %d)", v);
    }
    return ok();
}

const char *conv2d_last_error(void) { return t_last_error.c_str(); }

int conv2d_set_main_kernel_events(void *start, void *stop) {
    std::lock_guard<std::mutex> lock(g_mutex);
    if (start && stop) {
        g_main_start = static_cast<cudaEvent_t>(start);
        g_main_stop = static_cast<cudaEvent_t>(stop);
    } else {
        g_main_start = g_main_stop = nullptr;
    }
    return ok();
}

int conv2d_kernel_launch_count(unsigned long long *count) {
    if (!count) return fail(CONV_ERR_INVALID_ARG, "count must not be NULL");
    *count = g_launches.load(std::memory_order_relaxed);
    return ok();
}

int conv2d_debug_set_watchdog(long long timeout_ns, int starve_loads) {
    g_timeout_ns.store(timeout_ns > 0 ? timeout_ns : kDefaultTimeoutNs, std::memory_order_relaxed);
    g_starve.store(starve_loads ? 1 : 0, std::memory_order_relaxed);
    return ok();
}

int conv2d_describe_plan(int N, int C_in, int H, int W, int C_out, int Kh, int Kw, int stride,
                         int pad, int dilation, int groups, conv_dtype_t dtype, conv_layout_t layout,
                         int explicit_im2col, int sms, char *buf, size_t buflen) {
    return describe_impl(explicit_im2col != 0, N, C_in, H, W, C_out, Kh, Kw, stride, pad, dilation,
                         groups, dtype, layout, sms, buf, buflen);
}

int conv3d_describe_plan(int N, int C_in, int D, int H, int W, int C_out, int Kd, int Kh, int Kw, int stride,
                         int pad, int dilation, int groups, conv_dtype_t dtype, conv_layout_t layout, int sms,
                         char *buf, size_t buflen) {
    if (fold3d_applies(C_in, Kd, Kh, stride, groups, dtype)) {
        // the 2-D plan of the folded problem, with the fold's buffers in its workspace
        Plan inner;
        Fold3d f;
        int st = fold3d_plan(N, C_in, D, H, W, C_out, Kd, Kh, Kw, stride, pad, dilation, dtype, layout, nullptr,
                             settings_now(), &f, &inner);
        if (st != CONV_OK) return st;
        return describe_impl(false, N, f.Cf, f.Do * f.Ho, W, C_out, 1, Kw, 1, 0, dilation, 1, dtype, layout, sms, buf,
                             buflen, nullptr, &f.pw, 1, f.off_inner);
    }
    const Vol vol{D, Kd};
    return describe_impl(false, N, C_in, H, W, C_out, Kh, Kw, stride, pad, dilation, groups, dtype, layout, sms, buf,
                         buflen, &vol);
}

int conv2d_winograd_describe_plan(int N, int C_in, int H, int W, int C_out, int pad, int m, conv_dtype_t dtype,
                                  conv_layout_t layout, int sms, char *buf, size_t buflen) {
    WinoPlan w;
    int st = wino_plan(N, C_in, H, W, C_out, pad, m, dtype, layout, nullptr, settings_now(), &w);
    if (st != CONV_OK) return st;
    const int a2 = w.a * w.a;
    const PadW pw{0, reinterpret_cast<float *>(16)};  // placeholder address: plans the external-partial form
    return describe_impl(false, 1, a2 * w.Cpg, 1, w.T, a2 * C_out, 1, 1, 1, 0, 1, a2, w.tdt, CONV_NHWC, sms, buf,
                         buflen, nullptr, &pw);
}

int conv2d_debug_set_pair_mode(int mode) {
    if (mode < 0 || mode > 2) return fail(CONV_ERR_INVALID_ARG, "pair mode must be 0, 1 or 2");
    g_pair_mode.store(mode, std::memory_order_relaxed);
    return ok();
}


int conv2d_packed_weight_backward_data_size(int C_out, int C_in, int Kh, int Kw, int groups, conv_dtype_t dtype,
                                            size_t *bytes) {
    const int elt = elt_of(dtype);
    if (!bytes || elt == 0 || C_out < 1 || C_in < 1 || Kh < 1 || Kw < 1 || groups < 1 || C_in % groups ||
        C_out % groups)
        return fail(CONV_ERR_INVALID_ARG, "packed weight size: invalid argument");
    int cpg = 0, gm = 1;
    packed_weight_t_bytes(C_out, C_in, Kh, Kw, groups, elt, &cpg, &gm);
    *bytes = static_cast<size_t>(C_in) * Kh * Kw * cpg * elt;
    return ok();
}

int conv2d_pack_weight_backward_data(const void *w_oihw, void *w_packed_t, int C_out, int C_in, int Kh, int Kw,
                                     int groups, conv_dtype_t dtype, conv_stream_t stream) {
    size_t bytes = 0;
    int st = conv2d_packed_weight_backward_data_size(C_out, C_in, Kh, Kw, groups, dtype, &bytes);
    if (st != CONV_OK) return st;
    if (!w_oihw || !w_packed_t) return fail(CONV_ERR_INVALID_ARG, "weight pointers must not be NULL");
    const int elt = elt_of(dtype);
    int cpg = 0, gm = 1;
    packed_weight_t_bytes(C_out, C_in, Kh, Kw, groups, elt, &cpg, &gm);
    if ((st = check_launch(launch_pack_weight_t(w_oihw, w_packed_t, C_in, C_out / groups, C_in / groups, gm, Kh, Kw,
                                                cpg, elt, reinterpret_cast<cudaStream_t>(stream)),
                           "transposed weight pack")) != CONV_OK)
        return st;
    return ok();
}

int conv2d_backward_data_workspace_size(int N, int C_in, int H, int W, int C_out, int Kh, int Kw, int stride,
                                        int pad, int dilation, int groups, conv_dtype_t dtype,
                                        conv_layout_t layout, size_t *bytes) {
    if (!bytes) return fail(CONV_ERR_INVALID_ARG, "bytes must not be NULL");
    return backward_data_impl(nullptr, nullptr, nullptr, N, C_in, H, W, C_out, Kh, Kw, stride, pad, dilation,
                              groups, dtype, layout, nullptr, 0, nullptr, bytes);
}

int conv2d_backward_data(const void *dy, const void *w_packed_t, void *dx, int N, int C_in, int H, int W,
                         int C_out, int Kh, int Kw, int stride, int pad, int dilation, int groups,
                         conv_dtype_t dtype, conv_layout_t layout, void *workspace, size_t workspace_bytes,
                         conv_stream_t stream) {
    return backward_data_impl(dy, w_packed_t, dx, N, C_in, H, W, C_out, Kh, Kw, stride, pad, dilation, groups,
                              dtype, layout, workspace, workspace_bytes, reinterpret_cast<cudaStream_t>(stream),
                              nullptr);
}

int conv2d_backward_weight_workspace_size(int N, int C_in, int H, int W, int C_out, int Kh, int Kw, int stride,
                                          int pad, int dilation, int groups, conv_dtype_t dtype,
                                          conv_layout_t layout, int with_bias, size_t *bytes) {
    if (!bytes) return fail(CONV_ERR_INVALID_ARG, "bytes must not be NULL");
    WgPlan w;
    DeviceInfo *dev = current_device_or_null();
    int st = wgrad_plan(N, C_in, H, W, C_out, Kh, Kw, stride, pad, dilation, groups, dtype, layout, with_bias != 0,
                        dev ? dev->sms : 0, &w);
    if (st != CONV_OK) return st;
    *bytes = w.ws_total;
    return ok();
}

int conv2d_backward_weight(const void *x, const void *dy, void *dw, void *db, int N, int C_in, int H, int W,
                           int C_out, int Kh, int Kw, int stride, int pad, int dilation, int groups,
                           conv_dtype_t dtype, conv_layout_t layout, void *workspace, size_t workspace_bytes,
                           conv_stream_t stream) {
    return backward_weight_impl(x, dy, dw, db, N, C_in, H, W, C_out, Kh, Kw, stride, pad, dilation, groups, dtype,
                                layout, workspace, workspace_bytes, reinterpret_cast<cudaStream_t>(stream));
}

int conv2d_backward_bias_workspace_size(int N, int C_out, int Ho, int Wo, conv_layout_t layout, size_t *bytes) {
    if (!bytes || N < 1 || C_out < 1 || Ho < 1 || Wo < 1 || (layout != CONV_NHWC && layout != CONV_NCHW))
        return fail(CONV_ERR_INVALID_ARG, "bias gradient size: invalid argument");
    const long long rows = static_cast<long long>(N) * Ho * Wo;
    *bytes = static_cast<size_t>(bias_grad_partials(rows, C_out, N, layout == CONV_NCHW)) * C_out * 4;
    return ok();
}

int conv2d_backward_bias(const void *dy, void *db, int N, int C_out, int Ho, int Wo, conv_dtype_t dtype,
                         conv_layout_t layout, void *workspace, size_t workspace_bytes, conv_stream_t stream) {
    size_t need = 0;
    int st = conv2d_backward_bias_workspace_size(N, C_out, Ho, Wo, layout, &need);
    if (st != CONV_OK) return st;
    const int elt = elt_of(dtype);
    if (!dy || !db || elt == 0) return fail(CONV_ERR_INVALID_ARG, "dy and db must not be NULL; dtype must be valid");
    if (!workspace || workspace_bytes < need)
        return fail(CONV_ERR_WORKSPACE, "workspace of %zu bytes needed, %zu given", need,
                    workspace ? workspace_bytes : static_cast<size_t>(0));
    if (!aligned16(workspace)) return fail(CONV_ERR_UNSUPPORTED, "device pointers must be 16-byte aligned");
    return check_launch(launch_bias_grad(dy, static_cast<float *>(workspace), db, N, C_out,
                                         static_cast<long long>(Ho) * Wo, layout == CONV_NCHW, dtype == CONV_F32,
                                         reinterpret_cast<cudaStream_t>(stream)),
                        "bias gradient") == CONV_OK
               ? ok()
               : CONV_ERR_CUDA;
}


// ------------------------------------------------------------------ conv3d ---
int conv3d_packed_weight_size(int C_out, int C_in, int Kd, int Kh, int Kw, int groups, conv_dtype_t dtype,
                              size_t *bytes) {
    const int elt = elt_of(dtype);
    if (!bytes || elt == 0 || C_out < 1 || C_in < 1 || Kd < 1 || Kh < 1 || Kw < 1 || groups < 1 ||
        C_in % groups || C_out % groups)
        return fail(CONV_ERR_INVALID_ARG, "packed weight size: invalid argument");
    const int gm = group_merge(C_out, C_in, groups, elt);
    const int cpg = round_up(C_in / groups, 16 / elt) * gm;
    *bytes = static_cast<size_t>(C_out) * Kd * Kh * Kw * cpg * elt;
    return ok();
}

int conv3d_pack_weight(const void *w_oidhw, void *w_packed, int C_out, int C_in, int Kd, int Kh, int Kw,
                       int groups, conv_dtype_t dtype, conv_stream_t stream) {
    size_t bytes = 0;
    int st = conv3d_packed_weight_size(C_out, C_in, Kd, Kh, Kw, groups, dtype, &bytes);
    if (st != CONV_OK) return st;
    if (!w_oidhw || !w_packed) return fail(CONV_ERR_INVALID_ARG, "weight pointers must not be NULL");
    const int elt = elt_of(dtype);
    const int gm = group_merge(C_out, C_in, groups, elt);
    const int cpg = round_up(C_in / groups, 16 / elt) * gm;
    // (kd, kh) flattened: the OIDHW weight is an OIHW weight of filter height Kd*Kh
    if ((st = check_launch(launch_pack_weight(w_oidhw, w_packed, C_out, C_in / groups, C_out / groups, gm, Kd * Kh,
                                              Kw, cpg, elt, reinterpret_cast<cudaStream_t>(stream)),
                           "weight pack")) != CONV_OK)
        return st;
    return ok();
}

int conv3d_workspace_size(int N, int C_in, int D, int H, int W, int C_out, int Kd, int Kh, int Kw, int stride,
                          int pad, int dilation, int groups, conv_dtype_t dtype, conv_layout_t layout,
                          size_t *bytes) {
    if (fold3d_applies(C_in, Kd, Kh, stride, groups, dtype)) {
        if (!bytes) return fail(CONV_ERR_INVALID_ARG, "bytes must not be NULL");
        Plan inner;
        Fold3d f;
        int st = fold3d_plan(N, C_in, D, H, W, C_out, Kd, Kh, Kw, stride, pad, dilation, dtype, layout,
                             current_device_or_null(), settings_now(), &f, &inner);
        if (st != CONV_OK) return st;
        *bytes = f.ws_total;
        return ok();
    }
    const Vol vol{D, Kd};
    return workspace_impl(false, N, C_in, H, W, C_out, Kh, Kw, stride, pad, dilation, groups, dtype, layout, bytes,
                          nullptr, &vol);
}

int conv3d_forward(const void *x, const void *w_packed, const void *bias, void *y, int N, int C_in, int D, int H,
                   int W, int C_out, int Kd, int Kh, int Kw, int stride, int pad, int dilation, int groups,
                   conv_dtype_t dtype, conv_layout_t layout, void *workspace, size_t workspace_bytes,
                   conv_stream_t stream) {
    if (fold3d_applies(C_in, Kd, Kh, stride, groups, dtype))
        return fold3d_forward(x, w_packed, bias, y, N, C_in, D, H, W, C_out, Kd, Kh, Kw, stride, pad, dilation, dtype,
                              layout, workspace, workspace_bytes, reinterpret_cast<cudaStream_t>(stream));
    const Vol vol{D, Kd};
    return forward_impl(false, x, w_packed, bias, y, N, C_in, H, W, C_out, Kh, Kw, stride, pad, dilation, groups,
                        dtype, layout, workspace, workspace_bytes, reinterpret_cast<cudaStream_t>(stream), nullptr,
                        &vol);
}


// ---------------------------------------------------------------- Winograd ---
int conv2d_winograd_packed_weight_size(int C_out, int C_in, int m, conv_dtype_t dtype, size_t *bytes) {
    const int elt = elt_of(dtype);
    if (!bytes || elt == 0 || C_out < 1 || C_in < 1 || (m != 2 && m != 4))
        return fail(CONV_ERR_INVALID_ARG, "Winograd packed weight size: invalid argument");
    const int a2 = (m + 2) * (m + 2);
    const int telt = wino_tdt(dtype, m) == CONV_F32 ? 4 : 2;
    const int cpg = round_up(C_in, 16 / telt);
    const int gm = group_merge(a2 * C_out, a2 * cpg, a2, telt);
    *bytes = static_cast<size_t>(a2) * C_out * cpg * gm * telt;
    return ok();
}

int conv2d_pack_weight_winograd(const void *w_oihw, void *u_packed, int C_out, int C_in, int m, conv_dtype_t dtype,
                                conv_stream_t stream) {
    size_t bytes = 0;
    int st = conv2d_winograd_packed_weight_size(C_out, C_in, m, dtype, &bytes);
    if (st != CONV_OK) return st;
    if (!w_oihw || !u_packed) return fail(CONV_ERR_INVALID_ARG, "weight pointers must not be NULL");
    const int a2 = (m + 2) * (m + 2);
    const bool u_f32 = wino_tdt(dtype, m) == CONV_F32;
    const int telt = u_f32 ? 4 : 2;
    const int cpg = round_up(C_in, 16 / telt);
    const int gm = group_merge(a2 * C_out, a2 * cpg, a2, telt);
    return check_launch(launch_wino_weight(w_oihw, u_packed, C_out, C_in, cpg, gm, m, dtype == CONV_F32, u_f32,
                                           reinterpret_cast<cudaStream_t>(stream)),
                        "Winograd weight transform") == CONV_OK
               ? ok()
               : CONV_ERR_CUDA;
}

int conv2d_winograd_workspace_size(int N, int C_in, int H, int W, int C_out, int pad, int m, conv_dtype_t dtype,
                                   conv_layout_t layout, size_t *bytes) {
    if (!bytes) return fail(CONV_ERR_INVALID_ARG, "bytes must not be NULL");
    return winograd_impl(nullptr, nullptr, nullptr, nullptr, N, C_in, H, W, C_out, pad, m, dtype, layout, nullptr, 0,
                         nullptr, bytes);
}

int conv2d_forward_winograd(const void *x, const void *u_packed, const void *bias, void *y, int N, int C_in, int H,
                            int W, int C_out, int pad, int m, conv_dtype_t dtype, conv_layout_t layout,
                            void *workspace, size_t workspace_bytes, conv_stream_t stream) {
    return winograd_impl(x, u_packed, bias, y, N, C_in, H, W, C_out, pad, m, dtype, layout, workspace,
                         workspace_bytes, reinterpret_cast<cudaStream_t>(stream), nullptr);
}

}  // extern "C"
#pragma GCC visibility pop
