"""The backward pass (dx, dW, db) through the C ABI against the fp64 backward oracle
(needs a B200).

The oracle follows the naive backward loops of the "手撕 Conv2D" page
(lpnh.cn/news/2493075) §5.1-§5.2 and is pinned on the CPU (tests/oracle_pins_backward.py).
Small cases span several tiles, stages and reduction splits with ragged edges; the
full-size 3x3 layer is checked on sampled gradient entries, each evaluated by the
oracle from its definition.  Tolerances are the forward pass's: fp32 normwise relative
error <= 1e-5 per gradient tensor, bf16 max |err| <= 2e-2 * max |ref|."""
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


def draw_dy(cfg, seed, dist=None):
    """Seeded dy (NCHW float32), bf16-rounded for bf16 configs."""
    rng = np.random.default_rng(seed)
    shape = (cfg.N, cfg.C_out, cfg.Ho, cfg.Wo)
    if dist and dist[0] == "integers":
        dy = rng.integers(dist[1], dist[2] + 1, shape).astype(np.float32)
    else:
        dy = rng.standard_normal(shape, dtype=np.float32)
    return workloads.bf16_round(dy) if cfg.dtype == "bf16" else dy


def to_dev(cfg, a_nchw):
    """NCHW float array -> device tensor in the config's dtype and layout."""
    return parity.to_device_x(cfg, a_nchw)


def run_backward(cfg, inp, dy):
    """(dx NCHW, dW OIHW, db) from the CUDA path, as float64 arrays."""
    layer = parity.make_layer(cfg, inp)
    x = to_dev(cfg, inp["x"])
    dyd = to_dev(cfg, dy)
    dx = layer.backward_data(dyd, cfg.H, cfg.W)
    dw, db = layer.backward_weight(x, dyd)
    cb.conv2d_sync_status()
    return (parity.from_device_y(cfg, dx), dw.float().cpu().numpy().astype(np.float64),
            None if db is None else db.float().cpu().numpy().astype(np.float64))


def assert_grad(cfg, got, ref, what):
    assert got.shape == ref.shape, (what, got.shape, ref.shape)
    assert np.all(np.isfinite(got)), what
    e = parity.errors(got, ref)
    if cfg.dtype == "f32":
        assert e["normwise"] <= parity.F32_NORMWISE, (what, e)
    else:
        assert e["max_abs"] <= parity.BF16_MAXABS * e["max_ref"], (what, e)


BWD = [  # N, C_in, H, W, C_out, Kh, Kw, stride, pad, dilation, groups
    (2, 64, 12, 12, 64, 3, 3, 1, 1, 1, 1),     # 128-byte channel rows: tensor-core weight gradient
    (4, 64, 28, 28, 64, 3, 3, 1, 1, 1, 1),     # 49 pixel stages of 64, split across SMs, ragged last stage
    (2, 32, 9, 11, 48, 3, 3, 2, 1, 1, 1),      # stride 2: zero-inserted dy; 48 output channels
    (1, 128, 17, 17, 96, 7, 7, 1, 3, 1, 1),    # 49 taps, 17x17 (M-edge), 96 output channels
    (2, 16, 10, 8, 24, 3, 5, 1, 2, 2, 1),      # non-square filter, dilation 2: row and column pads differ
    (2, 64, 8, 8, 64, 3, 3, 1, 1, 1, 4),       # groups of 16 channels
    (1, 32, 9, 9, 32, 3, 3, 1, 1, 1, 32),      # depthwise: CUDA-core weight gradient, depthwise input gradient
    (2, 3, 16, 16, 8, 3, 3, 1, 1, 1, 1),       # three input channels
    (2, 48, 7, 9, 40, 1, 1, 1, 0, 1, 1),       # 1x1
    (1, 16, 12, 12, 16, 3, 3, 1, 3, 1, 1),     # pad 3 > K-1: the transposed convolution starts inside dy
    (2, 24, 15, 13, 16, 5, 5, 3, 2, 1, 1),     # stride 3, rows the windows never reach (zero gradient)
    (1, 256, 6, 6, 320, 3, 3, 1, 1, 1, 1),     # two 256-channel tiles of C_in, three 128-row tiles of C_out
    (2, 64, 10, 10, 256, 3, 3, 1, 1, 1, 1),    # bf16: both 128-row tiles of C_out in one unit
    (1, 64, 9, 9, 200, 3, 3, 1, 1, 1, 1),      # ... the second of them partial (200 channels)
    (1, 128, 6, 6, 512, 3, 3, 1, 1, 1, 2),     # ... per group of 256 output channels
]


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("layout", ["nhwc", "nchw"])
@pytest.mark.parametrize("shape", BWD, ids=lambda s: "x".join(map(str, s)))
def test_backward_matches_oracle(shape, layout, dtype):
    N, C_in, H, W, C_out, Kh, Kw, s, p, d, g = shape
    cfg = workloads.ConvConfig("bwd", N, C_in, H, W, C_out, Kh, Kw, s, p, d, g, True, dtype, layout,
                               seed=sum(shape) + 1)
    inp = workloads.make_inputs(cfg)
    dy = draw_dy(cfg, seed=sum(shape) + 2)
    dx, dw, db = run_backward(cfg, inp, dy)
    rdx, rdw, rdb = oracle.conv2d_backward(dy, inp["x"], inp["w"], s, p, d, g)
    assert_grad(cfg, dx, rdx, f"dx {shape}")
    assert_grad(cfg, dw, rdw, f"dW {shape}")
    assert_grad(cfg, db, rdb, f"db {shape}")


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("shape", [(1, 64, 6, 6, 64, 3, 3, 1, 1, 1, 1), (2, 32, 7, 7, 16, 3, 3, 2, 1, 1, 1),
                                   (1, 16, 6, 6, 16, 3, 3, 1, 1, 1, 16), (1, 64, 6, 6, 256, 3, 3, 1, 1, 1, 1)],
                         ids=lambda s: "x".join(map(str, s)))
def test_backward_small_integers_bit_exact(shape, dtype):
    """Integer inputs in [-1, 1] and a short pixel reduction: every sum is an integer of
    magnitude <= 256, exact in fp32 accumulation and in bf16, so gradients match exactly."""
    N, C_in, H, W, C_out, Kh, Kw, s, p, d, g = shape
    ints = ("integers", -1, 1)
    cfg = workloads.ConvConfig("bwd_ints", N, C_in, H, W, C_out, Kh, Kw, s, p, d, g, True, dtype, "nhwc",
                               ints, ints, ints, seed=5)
    inp = workloads.make_inputs(cfg)
    dy = draw_dy(cfg, seed=6, dist=ints)
    dx, dw, db = run_backward(cfg, inp, dy)
    rdx, rdw, rdb = oracle.conv2d_backward(dy, inp["x"], inp["w"], s, p, d, g)
    for got, ref in ((dx, rdx), (dw, rdw), (db, rdb)):
        assert np.abs(ref).max() <= 256
        assert np.array_equal(got, ref)


def test_backward_full_size_3x3_sampled():
    """The ResNet-style 3x3 layer at full size (the forward benchmark's workload):
    sampled dx and dW entries plus the whole db against the oracle's definition."""
    import torch
    cfg = workloads.CONFIGS["resnet3x3_bf16_nhwc"].scaled(bias=True)
    inp = workloads.make_inputs(cfg)
    dy = draw_dy(cfg, seed=77)
    layer = parity.make_layer(cfg, inp)
    x = to_dev(cfg, inp["x"])
    dyd = to_dev(cfg, dy)
    dx = layer.backward_data(dyd, cfg.H, cfg.W)
    dw, db = layer.backward_weight(x, dyd)
    cb.conv2d_sync_status()
    assert bool(torch.isfinite(dx).all()) and bool(torch.isfinite(dw).all())
    ix = parity.sample_indices((cfg.N, cfg.C_in, cfg.H, cfg.W), 512, seed=3)
    got = dx[tuple(torch.from_numpy(ix[:, i]).cuda() for i in (0, 2, 3, 1))].float().cpu().numpy()
    ref = oracle.conv2d_backward_data_points(dy, inp["w"], inp["x"].shape, ix, cfg.stride, cfg.pad, cfg.dilation,
                                             cfg.groups)
    assert np.abs(got - ref).max() <= parity.BF16_MAXABS * np.abs(ref).max()
    iw = parity.sample_indices(tuple(inp["w"].shape), 256, seed=4)
    got = dw[tuple(torch.from_numpy(iw[:, i]).cuda() for i in range(4))].float().cpu().numpy()
    ref = oracle.conv2d_backward_weight_points(dy, inp["x"], inp["w"].shape, iw, cfg.stride, cfg.pad,
                                               cfg.dilation, cfg.groups)
    assert np.abs(got - ref).max() <= parity.BF16_MAXABS * np.abs(ref).max()
    rdb = dy.astype(np.float64).sum(axis=(0, 2, 3))
    assert np.abs(db.float().cpu().numpy() - rdb).max() <= parity.BF16_MAXABS * np.abs(rdb).max()


def test_bias_gradient_alone_both_layouts():
    import torch
    rng = np.random.default_rng(9)
    for layout in ("nhwc", "nchw"):
        dy = rng.standard_normal((3, 40, 7, 9)).astype(np.float32)
        t = torch.from_numpy(dy)
        t = (t.permute(0, 2, 3, 1) if layout == "nhwc" else t).contiguous().cuda()
        nbytes = cb.conv2d_backward_bias_workspace_size(3, 40, 7, 9, layout)
        ws = torch.empty(max(nbytes, 16), dtype=torch.uint8, device="cuda")
        db = torch.empty(40, dtype=torch.float32, device="cuda")
        cb.conv2d_backward_bias(t, db, 3, 40, 7, 9, cb.CONV_F32, layout, ws)
        cb.conv2d_sync_status()
        ref = dy.astype(np.float64).sum(axis=(0, 2, 3))
        assert np.linalg.norm(db.cpu().numpy() - ref) / np.linalg.norm(ref) <= 1e-6
