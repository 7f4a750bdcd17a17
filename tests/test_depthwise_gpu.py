"""Depthwise convolution (groups = C_in = C_out) on the direct stencil kernel, against the
fp64 oracle through the C ABI (needs a B200).

The oracle is the same six-loop definition as for every other convolution, with one
input channel per group ("手撕 Conv2D" page, lpnh.cn/news/2493075, §7).  Each case first
checks that the library's plan really sends it to the depthwise kernel."""
import numpy as np
import pytest

import cnn_convolution_conv2d_b200 as cb
from cnn_convolution_conv2d_b200 import workloads
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


def dw_config(shape, dtype, layout, dists=None, seed=None):
    N, C, H, W, Kh, Kw, s, p, d = shape
    kw = {}
    if dists:
        kw = dict(x_dist=dists, w_dist=dists, b_dist=dists)
    return workloads.ConvConfig("dw", N, C, H, W, C, Kh, Kw, s, p, d, C, True, dtype, layout,
                                seed=sum(shape) if seed is None else seed, **kw)


def assert_depthwise_plan(cfg):
    plan = cb.conv2d_describe_plan(cfg.N, cfg.C_in, cfg.H, cfg.W, cfg.C_out, cfg.Kh, cfg.Kw, cfg.stride,
                                   cfg.pad, cfg.dilation, cfg.groups,
                                   cb.CONV_BF16 if cfg.dtype == "bf16" else cb.CONV_F32, cfg.layout)
    assert plan["kernel"] == "depthwise", plan


DW_EDGE = [  # N, C, H, W, Kh, Kw, stride, pad, dilation
    (2, 64, 20, 20, 3, 3, 1, 1, 1),     # register-window form, ragged last column tile
    (1, 128, 40, 33, 3, 3, 1, 1, 1),    # two channel chunks (bf16), two row tiles, ragged columns
    (2, 24, 9, 9, 5, 5, 1, 2, 1),       # 48-byte bf16 rows: channel-padded copy; 5x5 window
    (1, 32, 17, 19, 7, 7, 1, 3, 1),     # 7x7 window
    (2, 64, 15, 15, 3, 3, 2, 1, 1),     # stride 2: general form
    (2, 40, 14, 12, 3, 3, 1, 2, 2),     # dilation 2
    (1, 8, 1, 1, 3, 3, 1, 1, 1),        # a single pixel: only the centre tap inside the image
    (3, 16, 6, 7, 1, 1, 1, 0, 1),       # 1x1: a per-channel scale plus bias
    (2, 20, 11, 10, 5, 3, 2, 2, 2),     # non-square filter, stride 2, dilation 2, 20 channels
    (1, 200, 5, 70, 3, 3, 1, 1, 1),     # 200 channels: partial last chunk; wide image
    (2, 64, 40, 12, 3, 3, 3, 4, 1),     # stride 3, pad larger than the filter's reach
    (1, 8, 300, 9, 3, 1, 1, 1, 1),      # tall image: ten 32-row tiles, 3x1 filter
    (1, 6, 7, 9, 3, 3, 1, 1, 1),        # 6 channels (not a multiple of 4), odd output rows
    (2, 12, 11, 13, 5, 5, 1, 2, 1),     # 5x5 window, odd output rows, ragged columns
]


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("layout", ["nhwc", "nchw"])
@pytest.mark.parametrize("shape", DW_EDGE, ids=lambda s: "x".join(map(str, s)))
def test_depthwise_edge_shapes(shape, layout, dtype):
    cfg = dw_config(shape, dtype, layout)
    assert_depthwise_plan(cfg)
    inp = workloads.make_inputs(cfg)
    parity.assert_close(cfg, parity.run_gpu(cfg, inp), parity.run_oracle(cfg, inp), str(shape))


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("shape", [(2, 64, 20, 20, 3, 3, 1, 1, 1), (2, 24, 9, 9, 5, 5, 2, 2, 2)],
                         ids=lambda s: "x".join(map(str, s)))
def test_depthwise_small_integers_bit_exact(shape, dtype):
    """Integer inputs in [-2, 2]: every partial sum is exact, so outputs match exactly."""
    cfg = dw_config(shape, dtype, "nhwc", dists=("integers", -2, 2), seed=11)
    assert_depthwise_plan(cfg)
    inp = workloads.make_inputs(cfg)
    ref = parity.run_oracle(cfg, inp)
    assert np.array_equal(parity.run_gpu(cfg, inp), ref)


@pytest.mark.parametrize("name", ["depthwise3x3_bf16", "depthwise3x3_f32"])
def test_depthwise_workload_whole_output(name):
    """The full-size workload, in the launch configuration the benchmark times, against the
    oracle's whole output (0.9 GFLOP: seconds on the host)."""
    cfg = workloads.CONFIGS[name]
    assert_depthwise_plan(cfg)
    inp = workloads.make_inputs(cfg)
    parity.assert_close(cfg, parity.run_gpu(cfg, inp), parity.run_oracle(cfg, inp), name)


@pytest.mark.parametrize("name", ["depthwise3x3_bf16", "depthwise3x3_f32"])
def test_depthwise_workload_other_layout(name):
    cfg = workloads.CONFIGS[name].scaled(N=4, layout="nchw")
    assert_depthwise_plan(cfg)
    inp = workloads.make_inputs(cfg)
    parity.assert_close(cfg, parity.run_gpu(cfg, inp), parity.run_oracle(cfg, inp), name + " nchw")


def test_depthwise_watchdog_returns_timeout_instead_of_hanging():
    """With loads withheld every wait runs out after 1 ms; the call reports TIMEOUT and the
    next normal call is correct."""
    cfg = workloads.CONFIGS["depthwise3x3_bf16"].scaled(N=2, H=24, W=24)
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
    cb.conv2d_sync_status()
    parity.assert_close(cfg, parity.run_gpu(cfg, inp, layer=layer), parity.run_oracle(cfg, inp), "after timeout")
