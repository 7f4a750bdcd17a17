"""CUDA path vs the fp64 oracle, element by element, through the C ABI (needs a B200).

Small cases span several 128-row tiles with a ragged last tile and finish in the
oracle within seconds; full-size cases run in the launch configuration the
benchmark times and are checked on sampled outputs plus every corner."""
import numpy as np
import pytest

import cnn_convolution_conv2d_b200 as cb
from cnn_convolution_conv2d_b200 import workloads
import oracle
import parity

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def cuda_ready():
    import torch
    assert torch.cuda.is_available(), "these tests need a CUDA device (run with -m 'not gpu' on CPU)"
    from cnn_convolution_conv2d_b200 import build
    build.build()
    cb.load()
    cb.conv2d_debug_set_watchdog(0, False)
    yield
    cb.conv2d_sync_status()


SMALL = {  # oracle-sized versions of every workload (same seeds and distributions)
    "tiny_f32_nchw": {},
    "stem_bf16": dict(N=2, H=62, W=62),                        # M = 1922: 16 tiles, 2 rows in the last
    "resnet3x3_bf16_nhwc": dict(N=2, H=20, W=20),              # M = 800
    "pointwise1x1_bf16": dict(N=2, H=20, W=20),                # 4 column tiles of 256
    "grouped_dilated_bf16": dict(N=2),                         # 32 groups x 16 channels, s2 p2 d2
    "grouped_dilated_f32": dict(N=2),
    "k7_17x17_bf16": dict(N=1, C_in=128, C_out=128),           # split reduction across SMs
    "k7_17x17_f32": dict(N=1, C_in=128, C_out=128),
}


@pytest.mark.parametrize("name", sorted(SMALL))
def test_small_workloads(name):
    cfg = parity.config(name, **SMALL[name])
    inp = workloads.make_inputs(cfg)
    ref = parity.run_oracle(cfg, inp)
    got = parity.run_gpu(cfg, inp)
    parity.assert_close(cfg, got, ref, name)


@pytest.mark.parametrize("name", sorted(SMALL))
def test_small_workloads_other_layout(name):
    base = parity.config(name, **SMALL[name])
    cfg = base.scaled(layout="nhwc" if base.layout == "nchw" else "nchw")
    inp = workloads.make_inputs(cfg)
    parity.assert_close(cfg, parity.run_gpu(cfg, inp), parity.run_oracle(cfg, inp), name)


@pytest.mark.parametrize("name", ["tiny_f32_nchw", "stem_bf16", "resnet3x3_bf16_nhwc",
                                  "grouped_dilated_bf16", "k7_17x17_f32"])
def test_explicit_im2col_gemm(name):
    cfg = parity.config(name, **SMALL[name])
    inp = workloads.make_inputs(cfg)
    ref = parity.run_oracle(cfg, inp)
    got = parity.run_gpu(cfg, inp, explicit_im2col=True)
    parity.assert_close(cfg, got, ref, name + " (explicit im2col)")


EDGE = [  # N, C_in, H, W, C_out, Kh, Kw, stride, pad, dilation, groups
    (1, 8, 1, 1, 16, 1, 1, 1, 0, 1, 1),      # a single pixel
    (1, 3, 1, 1, 4, 3, 3, 2, 1, 1, 1),       # single pixel, only the centre tap in the image
    (3, 5, 13, 11, 40, 3, 3, 1, 1, 1, 1),    # odd C_in, C_out not a multiple of 16
    (2, 12, 10, 14, 24, 3, 5, 2, 2, 1, 1),   # non-square kernel, stride 2
    (2, 16, 15, 15, 32, 3, 3, 3, 4, 3, 1),   # stride 3, dilation 3, large pad
    (2, 64, 9, 9, 48, 1, 1, 2, 0, 1, 1),     # 1x1 with stride 2
    (1, 24, 12, 12, 36, 3, 3, 1, 1, 1, 4),   # groups with 6 input / 9 output channels each
    (2, 64, 8, 8, 64, 3, 3, 1, 1, 2, 8),     # 8 channels per group, dilation 2
    (1, 32, 30, 30, 8, 5, 5, 1, 0, 1, 1),    # C_out 8 < one 16-wide column tile
    (1, 96, 7, 9, 200, 2, 2, 1, 0, 1, 1),    # even kernel, C_out not a multiple of the tile
    (1, 16, 40, 3, 16, 7, 1, 8, 3, 1, 1),    # stride 8 (the largest supported), thin image
    (5, 8, 6, 6, 16, 3, 3, 1, 1, 1, 1),      # several images inside one 128-row tile
    (1, 16, 9, 9, 16, 3, 3, 1, 1, 1, 4),     # 4 channels per group: 16-byte rows, hardware im2col
    (2, 12, 11, 10, 20, 5, 3, 2, 2, 1, 1),   # 12 channels: software gather, reduction 180
    (2, 3, 16, 32, 24, 7, 7, 2, 3, 1, 1),    # first-layer shape, 16-byte rows: row-vector gather (bf16)
    (2, 3, 12, 16, 8, 3, 3, 1, 1, 1, 1),     # 16-byte rows, 3x3: row-vector gather (fp32 too)
    (3, 2, 9, 24, 16, 5, 5, 3, 2, 1, 1),     # row-vector gather with stride 3, two channels
    (2, 3, 32, 32, 24, 7, 7, 2, 3, 1, 1),    # Ho*Wo = 256: input rows staged by TMA (bf16)
    (2, 3, 16, 32, 8, 3, 3, 1, 1, 1, 1),     # Ho*Wo = 512: staged rows, 3x3 (fp32 too)
    (1, 2, 48, 48, 16, 5, 5, 3, 2, 1, 1),    # staged rows with stride 3
    (2, 48, 7, 9, 40, 1, 1, 1, 0, 1, 1),     # 1x1 stride 1: x read as the im2col matrix, M < one tile
    (3, 40, 10, 13, 24, 1, 1, 1, 0, 1, 1),   # ... 40 channels (80- or 160-byte rows), ragged last tile
    (1, 64, 15, 15, 96, 1, 1, 1, 0, 1, 4),   # ... grouped, 16 channels per group
    (1, 32, 6, 6, 32, 1, 1, 1, 0, 3, 1),     # ... dilation has no effect on a 1x1 filter
]


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("layout", ["nhwc", "nchw"])
@pytest.mark.parametrize("shape", EDGE, ids=lambda s: "x".join(map(str, s)))
def test_edge_shapes(shape, layout, dtype):
    N, C_in, H, W, C_out, Kh, Kw, s, p, d, g = shape
    cfg = workloads.ConvConfig("edge", N, C_in, H, W, C_out, Kh, Kw, s, p, d, g, True, dtype, layout,
                               seed=sum(shape))
    inp = workloads.make_inputs(cfg)
    parity.assert_close(cfg, parity.run_gpu(cfg, inp), parity.run_oracle(cfg, inp), str(shape))


TRANSPOSED_FIRST_LAYER = [  # bf16 NCHW, few channels, Wo % 8 == 0: the transposed kernel
    # shape, (output rows per tile, output images (0: stored straight from the registers),
    #         A in tensor memory)
    ((12, 3, 128, 128, 64, 7, 7, 2, 3, 1, 1), (2, 2, 1)),   # 384 row-pair tiles: each CTA wraps its rings
    ((3, 3, 64, 80, 40, 5, 5, 1, 2, 1, 1), (2, 2, 1)),      # stride 1; C_out 40: image rows 40..47 clipped
    ((2, 3, 40, 96, 24, 3, 3, 2, 1, 1, 1), (2, 2, 0)),      # 3x3 stride 2, C_out 24, 48 pixels: A in shared memory
    ((2, 3, 30, 64, 32, 7, 7, 2, 3, 1, 1), (2, 2, 0)),      # Ho = 15: the last pair's second row clipped
    ((2, 3, 40, 96, 96, 3, 3, 2, 1, 1, 1), (1, 2, 0)),      # C_out 96: one row per tile, A in shared memory
    ((2, 4, 64, 128, 128, 7, 7, 1, 3, 1, 1), (1, 2, 1)),    # C_out 128, reduction 224
    ((1, 4, 17, 160, 128, 7, 7, 1, 3, 1, 1), (1, 1, 1)),    # 160 pixels (three 64-pixel parts): room for one image
    ((1, 3, 17, 160, 64, 7, 7, 1, 3, 1, 1), (2, 1, 1)),     # ... two rows per tile, one image
    ((1, 4, 17, 192, 128, 8, 7, 1, 3, 1, 1), (1, 0, 1)),    # reduction 256, 192 pixels: no room for an image
]


@pytest.mark.parametrize("shape,form", TRANSPOSED_FIRST_LAYER, ids=lambda s: "x".join(map(str, s)))
def test_transposed_first_layer(shape, form):
    N, C_in, H, W, C_out, Kh, Kw, s, p, d, g = shape
    plan = cb.conv2d_describe_plan(*shape, cb.CONV_BF16, "nchw")
    assert (plan["kernel"], plan["rows"], plan["out_images"], plan["a_tmem"]) == ("gather_t",) + form, plan
    cfg = workloads.ConvConfig("first", N, C_in, H, W, C_out, Kh, Kw, s, p, d, g, True, "bf16", "nchw",
                               seed=sum(shape))
    inp = workloads.make_inputs(cfg)
    parity.assert_close(cfg, parity.run_gpu(cfg, inp), parity.run_oracle(cfg, inp), str(shape))


def test_transposed_first_layer_watchdog_returns_timeout():
    """The transposed first-layer kernel with loads withheld: its first wait (the bulk copy
    of the weight image that two-row tiles build A from) runs out after 1 ms, every later
    wait gives up at once, the status reads TIMEOUT, and the next normal call is right."""
    shape = (2, 3, 30, 64, 32, 7, 7, 2, 3, 1, 1)
    plan = cb.conv2d_describe_plan(*shape, cb.CONV_BF16, "nchw")
    assert (plan["kernel"], plan["rows"]) == ("gather_t", 2), plan
    N, C_in, H, W, C_out, Kh, Kw, s, p, d, g = shape
    cfg = workloads.ConvConfig("first", N, C_in, H, W, C_out, Kh, Kw, s, p, d, g, True, "bf16", "nchw",
                               seed=sum(shape))
    inp = workloads.make_inputs(cfg)
    layer = parity.make_layer(cfg, inp)
    x = parity.to_device_x(cfg, inp["x"])
    try:
        cb.conv2d_debug_set_watchdog(1_000_000, True)
        layer(x)
        with pytest.raises(cb.Conv2dError) as err:
            cb.conv2d_sync_status()
        assert err.value.status == cb.CONV_ERR_TIMEOUT
    finally:
        cb.conv2d_debug_set_watchdog(0, False)
    cb.conv2d_sync_status()  # status was cleared
    parity.assert_close(cfg, parity.run_gpu(cfg, inp, layer=layer), parity.run_oracle(cfg, inp), "after timeout")


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("explicit", [False, True])
@pytest.mark.parametrize("shape", [(2, 3, 9, 11, 4, 3, 3, 2, 1, 1, 1), (2, 16, 12, 12, 32, 3, 3, 1, 1, 1, 1),
                                   (1, 32, 10, 10, 64, 3, 3, 1, 1, 2, 4), (2, 64, 11, 12, 48, 1, 1, 1, 0, 1, 1)],
                         ids=lambda s: "x".join(map(str, s)))
def test_small_integers_bit_exact(shape, explicit, dtype):
    """Integer inputs in [-2, 2]: every partial sum is exact, so outputs match exactly."""
    N, C_in, H, W, C_out, Kh, Kw, s, p, d, g = shape
    cfg = workloads.ConvConfig("ints", N, C_in, H, W, C_out, Kh, Kw, s, p, d, g, True, dtype, "nhwc",
                               ("integers", -2, 2), ("integers", -2, 2), ("integers", -2, 2), seed=7)
    inp = workloads.make_inputs(cfg)
    ref = parity.run_oracle(cfg, inp)
    assert np.abs(ref).max() <= 256  # exactly representable in bf16 as well
    got = parity.run_gpu(cfg, inp, explicit_im2col=explicit)
    assert np.array_equal(got, ref)


# Full-size workloads whose whole output the oracle computes in seconds (at most ~120
# GFLOP): compared element by element over the entire tensor, the fp32 normwise bar
# taken over the whole output as it is defined.
FULL_WHOLE = ["tiny_f32_nchw", "grouped_dilated_bf16", "grouped_dilated_f32", "k7_17x17_bf16", "k7_17x17_f32"]
# The three largest, whose full oracle would take minutes: sampled outputs plus every corner.
FULL_SAMPLED = ["stem_bf16", "resnet3x3_bf16_nhwc", "pointwise1x1_bf16"]


@pytest.mark.parametrize("name", FULL_WHOLE)
def test_full_size_whole_output(name):
    cfg = workloads.CONFIGS[name]
    inp = workloads.make_inputs(cfg)
    got = parity.run_gpu(cfg, inp)
    parity.assert_close(cfg, got, parity.run_oracle(cfg, inp), name + " (whole output)")


@pytest.mark.parametrize("name", FULL_SAMPLED)
def test_full_size_sampled(name):
    import torch
    cfg = workloads.CONFIGS[name]
    inp = workloads.make_inputs(cfg)
    layer = parity.make_layer(cfg, inp)
    y = layer(parity.to_device_x(cfg, inp["x"]))
    cb.conv2d_sync_status()
    shape = (cfg.N, cfg.C_out, cfg.Ho, cfg.Wo)
    assert tuple(y.shape) == (shape if cfg.layout == "nchw" else (cfg.N, cfg.Ho, cfg.Wo, cfg.C_out))
    assert bool(torch.isfinite(y).all())
    idx = parity.sample_indices(shape, 512, seed=99)
    n, oc, oh, ow = (torch.from_numpy(idx[:, i]).cuda() for i in range(4))
    got = (y[n, oc, oh, ow] if cfg.layout == "nchw" else y[n, oh, ow, oc]).float().cpu().numpy()
    ref = oracle.conv2d_points(inp["x"], inp["w"], inp["b"], idx, cfg.stride, cfg.pad, cfg.dilation,
                               cfg.groups)
    if cfg.dtype == "f32":
        err = np.linalg.norm(got - ref) / np.linalg.norm(ref)
        assert err <= parity.F32_NORMWISE, err
    else:
        assert np.abs(got - ref).max() <= parity.BF16_MAXABS * np.abs(ref).max()


def test_layout_kernels_round_trip():
    import torch
    x = torch.randn(3, 5, 7, 9, dtype=torch.float32).to(torch.bfloat16).cuda()
    nhwc = torch.empty(3, 7, 9, 8, dtype=torch.bfloat16, device="cuda")
    cb.conv2d_nchw_to_nhwc(x, nhwc, 3, 5, 7, 9, 1, 8, cb.CONV_BF16)
    back = torch.empty_like(x)
    cb.conv2d_nhwc_to_nchw(nhwc[..., :5].contiguous(), back, 3, 5, 7, 9, cb.CONV_BF16)
    cb.conv2d_sync_status()
    assert torch.equal(back, x)
    assert torch.equal(nhwc[..., :5], x.permute(0, 2, 3, 1))
    assert bool((nhwc[..., 5:] == 0).all())
    # wide channel counts take the shared-memory tiled path
    x2 = torch.randn(2, 70, 33, 31, dtype=torch.float32).cuda()
    y2 = torch.empty(2, 33, 31, 70, dtype=torch.float32, device="cuda")
    cb.conv2d_nchw_to_nhwc(x2, y2, 2, 70, 33, 31, 1, 70, cb.CONV_F32)
    b2 = torch.empty_like(x2)
    cb.conv2d_nhwc_to_nchw(y2, b2, 2, 70, 33, 31, cb.CONV_F32)
    cb.conv2d_sync_status()
    assert torch.equal(y2, x2.permute(0, 2, 3, 1)) and torch.equal(b2, x2)


def test_pack_weight_layout():
    import torch
    w = torch.randn(6, 3, 2, 5, dtype=torch.float32).cuda()
    wp = cb.conv2d_pack_weight(w, groups=1)
    cb.conv2d_sync_status()
    ref = torch.zeros(6, 2, 5, 4, device="cuda")
    ref[..., :3] = w.permute(0, 2, 3, 1)
    assert torch.equal(wp[:6 * 2 * 5 * 4].view(6, 2, 5, 4), ref)  # images for the gather kernel follow


def test_hostio_matches_device_call():
    import torch
    cfg = parity.config("stem_bf16", N=2, H=62, W=62)
    inp = workloads.make_inputs(cfg)
    layer = parity.make_layer(cfg, inp)
    x_dev = parity.to_device_x(cfg, inp["x"])
    y_dev_ref = layer(x_dev)
    x_host = x_dev.cpu().pin_memory()
    y_host = torch.empty(y_dev_ref.shape, dtype=y_dev_ref.dtype).pin_memory()
    x2 = torch.empty_like(x_dev)
    y2 = torch.empty_like(y_dev_ref)
    layer.forward_hostio(x_host, y_host, x2, y2)
    cb.conv2d_sync_status()
    assert torch.equal(y_host, y_dev_ref.cpu())



@pytest.mark.parametrize("shape,layout", [
    ((35, 64, 64, 64, 64, 3, 3, 1, 1, 1, 1), "nhwc"),     # 18.4 MB of input: two chunks of 18 and 17 images
    ((100, 64, 48, 48, 32, 3, 3, 2, 1, 1, 1), "nchw"),    # 29.5 MB, NCHW, stride 2: three chunks (34, 33, 33)
])
def test_hostio_pipelined_chunks_bit_exact(shape, layout):
    """The host-buffer call cuts large batches into chunks whose copies and products
    overlap; with integer inputs every order of summation is exact, so the result equals
    the oracle's whatever the chunks' plans."""
    import torch
    N, C_in, H, W, C_out, Kh, Kw, s_, p_, d_, g_ = shape
    ints = ("integers", -2, 2)
    cfg = workloads.ConvConfig("hostio", *shape, True, "bf16", layout, ints, ints, ints, seed=23)
    inp = workloads.make_inputs(cfg)
    layer = parity.make_layer(cfg, inp)
    x_dev = parity.to_device_x(cfg, inp["x"])
    y_dev = layer(x_dev)
    x_host = x_dev.cpu().pin_memory()
    y_host = torch.empty(y_dev.shape, dtype=y_dev.dtype).pin_memory()
    x2 = torch.empty_like(x_dev)
    y2 = torch.full_like(y_dev, float("nan"))
    layer.forward_hostio(x_host, y_host, x2, y2)
    cb.conv2d_sync_status()
    ref = parity.run_oracle(cfg, inp)
    assert np.abs(ref).max() <= 256
    got = y_host.float().numpy().astype(np.float64)
    if layout == "nhwc":
        got = got.transpose(0, 3, 1, 2)
    assert np.array_equal(got, ref)



def test_hostio_pipelined_under_graph_capture():
    """The pipelined host-buffer call forks its copies onto two internal streams and joins
    them back; captured into a CUDA graph and replayed, it gives the eager result."""
    import torch
    shape = (35, 64, 64, 64, 64, 3, 3, 1, 1, 1, 1)
    ints = ("integers", -2, 2)
    cfg = workloads.ConvConfig("hostio_graph", *shape, True, "bf16", "nhwc", ints, ints, ints, seed=29)
    inp = workloads.make_inputs(cfg)
    layer = parity.make_layer(cfg, inp)
    x_dev = parity.to_device_x(cfg, inp["x"])
    y_ref = layer(x_dev).cpu()
    x_host = x_dev.cpu().pin_memory()
    y_host = torch.zeros(y_ref.shape, dtype=y_ref.dtype).pin_memory()
    x2 = torch.empty_like(x_dev)
    y2 = torch.empty(y_ref.shape, dtype=y_ref.dtype, device="cuda")
    layer.forward_hostio(x_host, y_host, x2, y2)   # sizes the layer's scratch before capture
    torch.cuda.synchronize()
    y_host.zero_()
    stream = torch.cuda.Stream()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=stream):
        layer.forward_hostio(x_host, y_host, x2, y2, stream=stream)
    graph.replay()
    torch.cuda.synchronize()
    cb.conv2d_sync_status()
    assert torch.equal(y_host, y_ref)

def test_repeated_calls_are_identical():
    import torch
    cfg = parity.config("k7_17x17_bf16", N=1, C_in=128, C_out=128)
    inp = workloads.make_inputs(cfg)
    layer = parity.make_layer(cfg, inp)
    x = parity.to_device_x(cfg, inp["x"])
    a = layer(x)
    b = layer(x)
    cb.conv2d_sync_status()
    assert torch.equal(a, b)


def test_watchdog_returns_timeout_instead_of_hanging():
    """With loads withheld, every wait in the kernel runs out after 1 ms; the kernel
    exits, the status reads TIMEOUT, and the next normal call works."""
    cfg = parity.config("resnet3x3_bf16_nhwc", N=1, H=12, W=12)
    inp = workloads.make_inputs(cfg)
    layer = parity.make_layer(cfg, inp)
    x = parity.to_device_x(cfg, inp["x"])
    try:
        cb.conv2d_debug_set_watchdog(1_000_000, True)
        layer(x)
        with pytest.raises(cb.Conv2dError) as err:
            cb.conv2d_sync_status()
        assert err.value.status == cb.CONV_ERR_TIMEOUT
    finally:
        cb.conv2d_debug_set_watchdog(0, False)
    cb.conv2d_sync_status()  # status was cleared
    parity.assert_close(cfg, parity.run_gpu(cfg, inp, layer=layer), parity.run_oracle(cfg, inp), "after timeout")


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("shape", [(2, 64, 8, 8), (1, 72, 17, 8), (3, 200, 5, 24), (1, 256, 56, 56), (1, 36, 3, 4)],
                         ids=lambda s: "x".join(map(str, s)))
def test_vector_transpose_both_ways(shape, dtype):
    """No channel padding, C and H*W multiples of the 16-byte vector (8 bf16 / 4 fp32):
    the vector tile transposes, full and partial tiles, against torch's permute (a pure
    data movement, so the results must be identical)."""
    import torch
    N, C, H, W = shape
    tdt, code = (torch.bfloat16, cb.CONV_BF16) if dtype == "bf16" else (torch.float32, cb.CONV_F32)
    x = (torch.randn(N, C, H, W) * 3).to(tdt).cuda()
    nhwc = torch.full((N, H, W, C), 7.0, dtype=tdt, device="cuda")
    cb.conv2d_nchw_to_nhwc(x, nhwc, N, C, H, W, 1, C, code)
    back = torch.full_like(x, 7.0)
    cb.conv2d_nhwc_to_nchw(nhwc, back, N, C, H, W, code)
    cb.conv2d_sync_status()
    assert torch.equal(nhwc, x.permute(0, 2, 3, 1))
    assert torch.equal(back, x)


def test_forward_rejects_misaligned_pointers_and_small_workspace_without_writing():
    """Host-side checks that need a device (they follow the device query): a pointer off
    a 16-byte boundary is UNSUPPORTED, a workspace below conv2d_workspace_size is
    WORKSPACE, and y is left untouched in both cases."""
    import torch
    cfg = parity.config("resnet3x3_bf16_nhwc", N=1, H=8, W=8, layout="nchw")  # NCHW: needs a workspace
    inp = workloads.make_inputs(cfg)
    layer = parity.make_layer(cfg, inp)
    x = parity.to_device_x(cfg, inp["x"])
    shape = (cfg.N, layer.C_in, cfg.H, cfg.W, layer.C_out, layer.Kh, layer.Kw, layer.stride, layer.pad,
             layer.dilation, layer.groups)
    need = cb.conv2d_workspace_size(*shape, layer.dtype, layer.layout)
    assert need > 0
    ws = torch.empty(need + 64, dtype=torch.uint8, device="cuda")
    y = torch.full(layer.out_shape(cfg.N, cfg.H, cfg.W), 3.0, dtype=torch.bfloat16, device="cuda")
    lib = cb.load()
    args = [*shape, layer.dtype, layer.layout]
    odd_x = x.data_ptr() + 2  # still inside x's allocation, 2 bytes off a 16-byte boundary
    st = lib.conv2d_forward(odd_x, layer.w_packed.data_ptr(), None, y.data_ptr(), *args, ws.data_ptr(), need, None)
    assert st == cb.CONV_ERR_UNSUPPORTED and "aligned" in cb.conv2d_last_error()
    st = lib.conv2d_forward(x.data_ptr(), layer.w_packed.data_ptr(), None, y.data_ptr(), *args, ws.data_ptr(),
                            need - 16, None)
    assert st == cb.CONV_ERR_WORKSPACE
    cb.conv2d_sync_status()
    assert bool((y == 3.0).all())
