"""The C-ABI library on the host, without a GPU: it loads, exports every function the
header declares, and rejects invalid arguments before touching the device."""
import ctypes
import os
import re

import pytest

import cnn_convolution_conv2d_b200 as cb
import oracle_pins

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "conv2d_b200.h")


def declared_functions():
    text = open(HEADER, encoding="utf-8").read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:const\s+)?\w+\s*\*?\s*(conv[23]d_\w+)\s*\(", text, flags=re.M)))


@pytest.fixture(scope="module")
def lib():
    from cnn_convolution_conv2d_b200 import build
    build.build()
    return cb.load()


def test_header_declares_the_abi():
    names = declared_functions()
    assert "conv2d_forward" in names and "conv2d_sync_status" in names
    assert set(names) == set(cb.SIGNATURES), set(names) ^ set(cb.SIGNATURES)


def test_library_exports_every_declared_symbol(lib):
    for name in declared_functions():
        assert hasattr(lib, name), name


def test_output_size_matches_the_pages(lib):
    for size, k, s, p, d, expected, src in oracle_pins.read_output_size_cases():
        out = ctypes.c_int(-7)
        st = lib.conv2d_output_size(size, k, s, p, d, ctypes.byref(out))
        if expected < 0:
            assert st == cb.CONV_ERR_INVALID_ARG, src
        else:
            assert st == cb.CONV_OK and out.value == expected, (src, st, out.value)


@pytest.mark.parametrize("args", [
    (0, 3, 1, 0, 1), (5, 0, 1, 0, 1), (5, 3, 0, 0, 1), (5, 3, 1, -1, 1), (5, 3, 1, 0, 0),
    (2, 5, 1, 0, 1),  # kernel larger than the input
])
def test_output_size_rejects(lib, args):
    out = ctypes.c_int(0)
    assert lib.conv2d_output_size(*args, ctypes.byref(out)) == cb.CONV_ERR_INVALID_ARG
    assert cb.conv2d_last_error()


def test_packed_weight_size(lib):
    # many channels or groups: only the (C_out, Kh, Kw, Cpg) weights
    # 32 groups of 16 -> 16 channels: merged 4 at a time (one 128-byte channel row),
    # block-diagonal rows of 4 * 16 channels
    assert cb.conv2d_packed_weight_size(512, 512, 3, 3, 32, cb.CONV_BF16) == 512 * 9 * 16 * 4 * 2
    assert cb.conv2d_packed_weight_size(512, 512, 3, 3, 32, cb.CONV_F32) == 512 * 9 * 16 * 4  # fp32: no merge
    assert cb.conv2d_packed_weight_size(24, 24, 3, 3, 4, cb.CONV_BF16) == 24 * 9 * 8 * 2  # 12-byte rows: no merge
    assert cb.conv2d_packed_weight_size(256, 256, 3, 3, 1, cb.CONV_BF16) == 256 * 9 * 256 * 2
    # few input channels: followed (256-byte aligned) by the gather kernel's images,
    # 16-row x Kpad matrices for the compact and row-vector reduction orders
    main = 64 * 49 * 8 * 2                       # stem: Cpg = 8
    compact = 64 * 160 * 2                       # 3*7*7 = 147 -> 160
    rowvec = 64 * 176 * 2                        # 3*7*8 = 168 -> 176
    assert cb.conv2d_packed_weight_size(64, 3, 7, 7, 1, cb.CONV_BF16) == main + compact + rowvec
    main32 = 4 * 9 * 4 * 4                       # fp32 tiny: Cpg = 4 -> 576 bytes
    img_c = 16 * 32 * 4 * 2                      # 27 -> 32, tf32 hi + lo
    img_r = 16 * 40 * 4 * 2                      # 3*3*4 = 36 -> 40
    assert main32 == 576
    assert cb.conv2d_packed_weight_size(4, 3, 3, 3, 1, cb.CONV_F32) == 768 + img_c + img_r
    with pytest.raises(cb.Conv2dError):
        cb.conv2d_packed_weight_size(6, 4, 3, 3, 4, cb.CONV_BF16)   # C_out % groups


GOOD = dict(N=2, C_in=8, H=9, W=9, C_out=16, Kh=3, Kw=3, stride=1, pad=1, dilation=1, groups=1)
BAD = [
    dict(N=0), dict(C_in=0), dict(H=0), dict(W=-1), dict(C_out=0), dict(Kh=0), dict(Kw=0),
    dict(stride=0), dict(pad=-1), dict(dilation=0), dict(groups=0), dict(groups=3),
    dict(C_out=12, groups=8),  # C_out % groups
    dict(Kh=12),               # empty output
    dict(H=2, W=2, pad=0),     # kernel larger than the image
]


def _call_forward(lib, shape, x=16, w=16, y=16, dtype=cb.CONV_BF16, layout=cb.CONV_NHWC):
    s = dict(GOOD, **shape)
    return lib.conv2d_forward(x, w, None, y, s["N"], s["C_in"], s["H"], s["W"], s["C_out"], s["Kh"],
                              s["Kw"], s["stride"], s["pad"], s["dilation"], s["groups"], dtype,
                              layout, None, 0, None)


@pytest.mark.parametrize("shape", BAD, ids=lambda d: ",".join(f"{k}={v}" for k, v in d.items()))
def test_forward_rejects_invalid_shapes(lib, shape):
    assert _call_forward(lib, shape) == cb.CONV_ERR_INVALID_ARG
    assert cb.conv2d_last_error()


def test_forward_rejects_null_pointers_and_bad_enums(lib):
    assert _call_forward(lib, {}, x=None) == cb.CONV_ERR_INVALID_ARG
    assert _call_forward(lib, {}, w=None) == cb.CONV_ERR_INVALID_ARG
    assert _call_forward(lib, {}, y=None) == cb.CONV_ERR_INVALID_ARG
    assert _call_forward(lib, {}, dtype=7) == cb.CONV_ERR_INVALID_ARG
    assert _call_forward(lib, {}, layout=5) == cb.CONV_ERR_INVALID_ARG


def test_forward_reports_unsupported_limits(lib):
    assert _call_forward(lib, dict(stride=9, H=40, W=40)) == cb.CONV_ERR_UNSUPPORTED
    assert _call_forward(lib, dict(pad=128, H=4, W=4)) == cb.CONV_ERR_UNSUPPORTED


def test_workspace_size_without_device(lib):
    # channels-last input with C_in a multiple of 8: no scratch at all
    assert cb.conv2d_workspace_size(2, 8, 9, 9, 16, 3, 3, 1, 1, 1, 1, cb.CONV_BF16, "nhwc") == 0
    # NCHW input with 16 channels: a channels-last copy
    assert cb.conv2d_workspace_size(2, 16, 9, 9, 16, 3, 3, 1, 1, 1, 1, cb.CONV_BF16, "nchw") >= 2 * 9 * 9 * 16 * 2
    # 12 channels in groups of 3: a channels-last copy with each group padded to 8
    assert cb.conv2d_workspace_size(2, 12, 9, 9, 16, 3, 3, 1, 1, 1, 4, cb.CONV_BF16, "nhwc") >= 2 * 9 * 9 * 32 * 2
    # 3 channels (first layer): gathered straight from x, no scratch
    assert cb.conv2d_workspace_size(2, 3, 9, 9, 16, 3, 3, 1, 1, 1, 1, cb.CONV_BF16, "nchw") == 0
    # explicit im2col adds X_col: M rows of Kh*Kw*Cpg elements
    xcol = 2 * 9 * 9 * 9 * 8 * 2
    assert cb.conv2d_im2col_workspace_size(2, 8, 9, 9, 16, 3, 3, 1, 1, 1, 1, cb.CONV_BF16, "nhwc") >= xcol
    with pytest.raises(cb.Conv2dError):
        cb.conv2d_workspace_size(2, 8, 9, 9, 16, 3, 3, 1, 1, 1, 3, cb.CONV_BF16, "nhwc")


def test_watchdog_hook_accepts_settings(lib):
    cb.conv2d_debug_set_watchdog(1000, False)
    cb.conv2d_debug_set_watchdog(0, False)   # back to the default


def test_pair_mode_hook_checks_its_argument(lib):
    for mode in (1, 2, 0):                  # ends on the default
        cb.conv2d_debug_set_pair_mode(mode)
    for bad in (-1, 3):
        with pytest.raises(cb.Conv2dError) as err:
            cb.conv2d_debug_set_pair_mode(bad)
        assert err.value.status == cb.CONV_ERR_INVALID_ARG


def test_pair_mode_leaves_workspace_of_split_free_problems_unchanged(lib):
    # the 1x1 layer needs no scratch whichever kernel runs it
    shape = (64, 256, 56, 56, 1024, 1, 1, 1, 0, 1, 1)
    try:
        for mode in (0, 1, 2):
            cb.conv2d_debug_set_pair_mode(mode)
            assert cb.conv2d_workspace_size(*shape, cb.CONV_BF16, "nhwc") == 0
    finally:
        cb.conv2d_debug_set_pair_mode(0)


def _plan(shape, dtype=cb.CONV_BF16, layout="nhwc", **kw):
    return cb.conv2d_describe_plan(*shape, dtype, layout, **kw)


def test_plan_for_the_workloads_on_a_148_sm_device(lib):
    """The kernel and tile choices the forward pass makes, pinned on the CPU."""
    p1 = _plan((64, 256, 56, 56, 1024, 1, 1, 1, 0, 1, 1), sms=148)   # 1x1: x is X_col, weights resident
    assert (p1["kernel"], p1["pair"], p1["a_load"], p1["BN"], p1["stages"], p1["tma_out"]) == \
        ("pointwise", 1, "tiled_x", 256, 6, 1)
    assert p1["units"] == (64 * 56 * 56 // 256) * 4 and p1["workspace"] == 0
    p3 = _plan((64, 256, 56, 56, 256, 3, 3, 1, 1, 1, 1), sms=148)    # 3x3: hardware im2col, pairs
    assert (p3["kernel"], p3["pair"], p3["a_load"], p3["BN"], p3["units"]) == ("igemm", 1, "im2col", 256, 784)
    stem = _plan((32, 3, 224, 224, 64, 7, 7, 2, 3, 1, 1), layout="nchw", sms=148)
    # the transposed few-channel kernel: 64 channels fill half the lanes, so a tile is two
    # output rows (2 x 112 pixels), stored from double-buffered output images by TMA; the
    # weights stay in tensor memory
    assert (stem["kernel"], stem["halo"], stem["BN"], stem["workspace"], stem["units"], stem["rows"],
            stem["out_images"], stem["a_tmem"]) == ("gather_t", 1, 64, 0, 32 * 56, 2, 2, 1)
    nhwc_out = _plan((32, 3, 224, 224, 64, 7, 7, 2, 3, 1, 1), layout="nhwc", sms=148)
    assert nhwc_out["kernel"] == "gather"                              # channels-last: the lane-per-pixel form
    assert stem["Kpad"] == 176                                         # 3 channels x 7 rows x 8 (7 taps + 1) -> 168 -> 176
    k7 = _plan((16, 512, 17, 17, 512, 7, 7, 1, 3, 1, 1), sms=148)     # 19 pair units < 74: single CTAs, split
    assert (k7["pair"], k7["splits"], k7["units"]) == (0, 2, 37 * 2 * 2)
    assert k7["workspace"] == 2 * 16 * 17 * 17 * 512 * 4               # fp32 partial sums per split
    g = _plan((16, 512, 28, 28, 512, 3, 3, 2, 2, 2, 32), sms=148)     # 16 channels per group, merged 4 at a time
    assert (g["pair"], g["BN"], g["cb"], g["units"]) == (0, 64, 128, 25 * 8)
    ex = _plan((64, 256, 56, 56, 256, 3, 3, 1, 1, 1, 1), explicit_im2col=True, sms=148)
    assert ex["a_load"] == "xcol" and ex["workspace"] >= 924_844_032   # the 924.8 MB X_col
    f32 = _plan((16, 512, 17, 17, 512, 7, 7, 1, 3, 1, 1), dtype=cb.CONV_F32, sms=148)
    assert f32["pair"] == 0 and f32["BN"] == 128                        # CTA pairs are bf16 only


def test_winograd_product_plans(lib):
    """The Winograd channel product on the 3x3 layer: F(2x2,3x3) (bf16 transforms) on the
    resident-weight pair kernel, 16 groups of 256 -> 256 over 64 x 28 x 28 tiles; F(4x4,3x3)
    (fp32 transforms, three tf32 products) on the general kernel."""
    p2 = cb.conv2d_winograd_describe_plan(64, 256, 56, 56, 256, 1, 2, cb.CONV_BF16, "nhwc", sms=148)
    assert (p2["kernel"], p2["pair"], p2["BN"], p2["units"]) == ("pointwise", 1, 256, 16 * (64 * 28 * 28 // 256))
    p4 = cb.conv2d_winograd_describe_plan(64, 256, 56, 56, 256, 1, 4, cb.CONV_BF16, "nhwc", sms=148)
    assert (p4["kernel"], p4["pair"]) == ("igemm", 0)
    p2n = cb.conv2d_winograd_describe_plan(1, 96, 9, 9, 512, 1, 2, cb.CONV_BF16, "nchw", sms=148)
    assert p2n["kernel"] == "igemm"                      # 96 channels: not whole 64-channel planes
    with pytest.raises(cb.Conv2dError):
        cb.conv2d_winograd_describe_plan(1, 8, 8, 8, 8, 1, 3, cb.CONV_BF16, "nhwc")


def test_plan_without_a_device_count_makes_no_device_choices(lib):
    p = _plan((64, 256, 56, 56, 256, 3, 3, 1, 1, 1, 1), sms=0)
    assert p["pair"] == 0 and p["splits"] == 1 and p["units"] == 1568 and p["sms"] == 0


def test_pair_mode_hook_changes_the_plan(lib):
    small = (2, 64, 20, 20, 64, 3, 3, 1, 1, 1, 1)
    try:
        assert _plan(small, sms=148)["pair"] == 0        # 4 units of 256 rows: not enough work
        cb.conv2d_debug_set_pair_mode(1)
        assert _plan(small, sms=148)["pair"] == 1
        assert _plan((2, 64, 20, 20, 48, 3, 3, 1, 1, 1, 1), sms=148)["pair"] == 0  # BN = 48: no even split
        cb.conv2d_debug_set_pair_mode(2)
        assert _plan((64, 256, 56, 56, 256, 3, 3, 1, 1, 1, 1), sms=148)["pair"] == 0
    finally:
        cb.conv2d_debug_set_pair_mode(0)


def test_describe_plan_rejects_bad_arguments(lib):
    with pytest.raises(cb.Conv2dError) as err:
        _plan((1, 8, 4, 4, 8, 7, 7, 1, 0, 1, 1))          # empty output
    assert err.value.status == cb.CONV_ERR_INVALID_ARG
    buf = ctypes.create_string_buffer(8)
    st = lib.conv2d_describe_plan(1, 8, 4, 4, 8, 3, 3, 1, 1, 1, 1, cb.CONV_BF16, cb.CONV_NHWC, 0, 0, buf, 8)
    assert st == cb.CONV_ERR_INVALID_ARG                   # buffer too small


def test_bench_mirror_of_the_gather_choice_agrees_with_the_library(lib):
    """bench.py labels the kernel and counts its bytes with a Python copy of the
    library's few-channel rule; keep the two in step for every workload."""
    import bench
    from cnn_convolution_conv2d_b200 import workloads
    for name, c in workloads.CONFIGS.items():
        plan = cb.conv2d_describe_plan(c.N, c.C_in, c.H, c.W, c.C_out, c.Kh, c.Kw, c.stride, c.pad, c.dilation,
                                       c.groups, cb.CONV_BF16 if c.dtype == "bf16" else cb.CONV_F32, c.layout,
                                       sms=148)
        assert (plan["kernel"] in ("gather", "gather_t")) == bench.uses_gather(c), name
        assert (plan["kernel"] == "depthwise") == bench.uses_depthwise(c), name


def test_depthwise_plans(lib):
    """groups = C_in = C_out goes to the depthwise stencil kernel: register-window form for
    stride-1 square 3/5/7 filters, channel-padded copy when 16-byte rows need it."""
    d = _plan((64, 256, 56, 56, 256, 3, 3, 1, 1, 1, 256), sms=148)
    assert (d["kernel"], d["a_load"], d["xcopy"], d["workspace"]) == ("depthwise", "tile", 0, 0)
    assert d["units"] == 4 * 64 * 2 * 7            # 64-channel chunks x images x 30x8 output tiles
    odd = _plan((2, 20, 9, 9, 20, 5, 3, 2, 2, 2, 20), sms=148)   # 40-byte rows: padded copy
    assert odd["kernel"] == "depthwise" and odd["xcopy"] == 1
    assert odd["workspace"] == 2 * 9 * 9 * 24 * 2 + (256 - (2 * 9 * 9 * 24 * 2) % 256) % 256
    nchw = _plan((4, 32, 10, 10, 32, 3, 3, 1, 1, 1, 32), dtype=cb.CONV_F32, layout="nchw", sms=148)
    assert nchw["kernel"] == "depthwise" and nchw["xcopy"] == 1
    mult = _plan((2, 16, 8, 8, 32, 3, 3, 1, 1, 1, 16), sms=148)  # channel multiplier 2: general kernel
    assert mult["kernel"] == "igemm"


def test_backward_sizes_on_the_host(lib):
    """Sizes of the backward entry points, without a device."""
    # transposed kernel: C_in output channels of C_out/groups (padded) reduction channels
    assert cb.conv2d_packed_weight_backward_data_size(64, 32, 3, 3, 1, cb.CONV_BF16) == 32 * 9 * 64 * 2
    assert cb.conv2d_packed_weight_backward_data_size(6, 3, 3, 3, 1, cb.CONV_BF16) == 3 * 9 * 8 * 2  # 6 -> 8
    assert cb.conv2d_packed_weight_backward_data_size(12, 12, 3, 3, 12, cb.CONV_F32) == 12 * 9 * 4 * 4  # depthwise
    # stride 2: the zero-inserted dy (Hz = H - d(K-1) + 2p = 9 - 2 + 2 = 9, same for W) comes first
    base = cb.conv2d_backward_data_workspace_size(2, 16, 9, 9, 32, 3, 3, 1, 1, 1, 1, cb.CONV_BF16, "nhwc")
    assert base == 0
    s2 = cb.conv2d_backward_data_workspace_size(2, 16, 9, 9, 32, 3, 3, 2, 1, 1, 1, cb.CONV_BF16, "nhwc")
    assert s2 >= 2 * 9 * 9 * 32 * 2
    # weight gradient: padded channels-last copies and one split of fp32 partials without a device
    wg = cb.conv2d_backward_weight_workspace_size(2, 16, 9, 9, 32, 3, 3, 1, 1, 1, 1, cb.CONV_BF16, "nhwc")
    assert wg >= 2 * 9 * 9 * 64 * 2 + 32 * 9 * 64 * 4     # x padded to 64 channels; partials [C_out][taps][64]
    assert cb.conv2d_backward_weight_workspace_size(2, 16, 9, 9, 32, 3, 3, 1, 1, 1, 1, cb.CONV_BF16, "nhwc",
                                                    with_bias=True) > wg
    assert cb.conv2d_backward_bias_workspace_size(2, 32, 9, 9, "nchw") == 2 * 32 * 4


def test_backward_rejects_bad_arguments(lib):
    with pytest.raises(cb.Conv2dError) as err:
        cb.conv2d_backward_data_workspace_size(2, 16, 9, 9, 32, 3, 3, 1, 1, 1, 3, cb.CONV_BF16, "nhwc")
    assert err.value.status == cb.CONV_ERR_INVALID_ARG        # groups must divide both channel counts
    st = lib.conv2d_backward_weight(None, None, None, None, 2, 16, 9, 9, 32, 3, 3, 1, 1, 1, 1, cb.CONV_BF16,
                                    cb.CONV_NHWC, None, 0, None)
    assert st == cb.CONV_ERR_INVALID_ARG


def test_conv3d_sizes_and_limits_on_the_host(lib):
    assert cb.conv3d_packed_weight_size(16, 3, 3, 3, 3, 1, cb.CONV_BF16) == 16 * 27 * 8 * 2
    # three channels at stride 1: the (kd, kh)-folded input (27 channels padded to 32) and
    # its 16 x 3 x 32 weights are the workspace; the 2-D product of the fold needs none
    assert cb.conv3d_workspace_size(4, 3, 16, 64, 64, 16, 3, 3, 3, 1, 1, 1, 1, cb.CONV_BF16, "nchw") == \
        4 * 16 * 64 * 64 * 32 * 2 + 16 * 3 * 32 * 2
    p = cb.conv3d_describe_plan(4, 3, 16, 64, 64, 16, 3, 3, 3, 1, 1, 1, 1, cb.CONV_BF16, "nchw", sms=148)
    assert (p["fold"], p["kernel"], p["a_load"], p["cb"], p["BN"], p["units"]) == (1, "igemm", "im2col", 64, 16, 2048)
    # eight channels (16-byte rows) at stride 2 fold as well: 72 -> 96 channels over the
    # strided rows, full input width (the product takes the column stride)
    p2 = cb.conv3d_describe_plan(4, 8, 16, 64, 64, 32, 3, 3, 3, 2, 1, 1, 1, cb.CONV_BF16, "nhwc", sms=148)
    assert (p2["fold"], p2["cb"], p2["BN"], p2["units"]) == (1, 64, 32, 4 * 8 * 32 * 32 // 128)
    assert cb.conv3d_workspace_size(4, 8, 16, 64, 64, 32, 3, 3, 3, 2, 1, 1, 1, cb.CONV_BF16, "nhwc") == \
        4 * 8 * 32 * 64 * 96 * 2 + 32 * 3 * 96 * 2
    # 16 channels (32-byte rows; the stride-2 3-D layer), or groups: no fold; NCDHW input then
    # goes through the channels-last copy
    p3 = cb.conv3d_describe_plan(4, 16, 16, 64, 64, 32, 3, 3, 3, 2, 1, 1, 1, cb.CONV_BF16, "nchw", sms=148)
    assert (p3["fold"], p3["xcopy"]) == (0, 1)
    assert cb.conv3d_describe_plan(2, 8, 8, 16, 16, 32, 3, 3, 3, 1, 1, 1, 2, cb.CONV_BF16, "nhwc", sms=148)["fold"] == 0
    # the 5-D im2col addressing range: pad 17 is out of it
    st = lib.conv3d_forward(16, 16, None, 16, 1, 32, 40, 40, 40, 8, 3, 3, 3, 1, 17, 1, 1, cb.CONV_BF16,
                            cb.CONV_NHWC, None, 0, None)
    assert st == cb.CONV_ERR_UNSUPPORTED
    st = lib.conv3d_forward(16, 16, None, 16, 1, 8, 2, 8, 8, 8, 5, 3, 3, 1, 0, 1, 1, cb.CONV_BF16,
                            cb.CONV_NHWC, None, 0, None)
    assert st == cb.CONV_ERR_INVALID_ARG                       # filter deeper than the input


def test_winograd_sizes_on_the_host(lib):
    # F(2x2,3x3): 16 transformed filters per (oc, c); 64 channels each way, no group merge
    assert cb.conv2d_winograd_packed_weight_size(64, 64, 2, cb.CONV_BF16) == 16 * 64 * 64 * 2
    assert cb.conv2d_winograd_packed_weight_size(64, 64, 4, cb.CONV_F32) == 36 * 64 * 64 * 4
    assert cb.conv2d_winograd_packed_weight_size(64, 64, 4, cb.CONV_BF16) == 36 * 64 * 64 * 4  # fp32 transforms
    for m in (3, 6):
        with pytest.raises(cb.Conv2dError):
            cb.conv2d_winograd_packed_weight_size(8, 8, m, cb.CONV_BF16)
    ws = cb.conv2d_winograd_workspace_size(2, 64, 12, 12, 64, 1, 2, cb.CONV_BF16, "nhwc")
    tiles = 2 * 6 * 6
    assert ws >= tiles * 16 * 64 * 2 + tiles * 16 * 64 * 4  # V (bf16) and the fp32 products


def test_binding_signatures_match_the_header_argument_counts():
    """Every ctypes signature of the binding has as many arguments as the header's
    declaration (a missing or extra argument would shift every later one)."""
    text = open(HEADER, encoding="utf-8").read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    decls = re.findall(r"^\s*(?:const\s+)?\w+\s*\*?\s*(conv[23]d_\w+)\s*\(([^)]*)\)\s*;", text, flags=re.M)
    assert decls
    for name, params in decls:
        params = params.strip()
        count = 0 if params in ("", "void") else len([p for p in params.split(",") if p.strip()])
        assert len(cb.SIGNATURES[name][0]) == count, (name, count, len(cb.SIGNATURES[name][0]))
