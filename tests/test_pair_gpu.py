"""The CTA-pair tensor-core kernel against the oracle, through the C ABI (needs a B200).

On bf16 problems large enough to give every SM pair work, the library runs the
implicit GEMM in clusters of two CTAs: each unit is 256 output pixels, the even
CTA issues M = 256 tensor-core products that read 128 rows of A and half of the
weight tile from each CTA's shared memory.  Full-size workloads take that path by
default (and are sampled in test_parity_gpu.py); here the test hook
conv2d_debug_set_pair_mode(1) forces it onto problems small enough for the oracle
to check every output, including ragged last units and a unit whose second half
lies wholly past the last pixel.
"""
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
    cb.conv2d_debug_set_pair_mode(0)
    cb.conv2d_sync_status()


@pytest.fixture
def pairs_forced():
    cb.conv2d_debug_set_pair_mode(1)
    yield
    cb.conv2d_debug_set_pair_mode(0)


SMALL = {
    "resnet3x3_bf16_nhwc": dict(N=2, H=20, W=20),   # M = 800: 4 units, the last one ragged
    "pointwise1x1_bf16": dict(N=2, H=20, W=20),     # four column tiles of 256, tiled A loads
    "k7_17x17_bf16": dict(N=1, C_in=128, C_out=128),  # long reduction (49 taps), one unit
}


@pytest.mark.parametrize("layout", ["nhwc", "nchw"])
@pytest.mark.parametrize("name", sorted(SMALL))
def test_pair_small_workloads(name, layout, pairs_forced):
    cfg = parity.config(name, **SMALL[name]).scaled(layout=layout)
    inp = workloads.make_inputs(cfg)
    parity.assert_close(cfg, parity.run_gpu(cfg, inp), parity.run_oracle(cfg, inp), name + " (pair)")


PAIR_EDGE = [  # N, C_in, H, W, C_out, Kh, Kw, stride, pad, dilation, groups
    (3, 64, 10, 13, 64, 3, 3, 1, 1, 1, 1),     # M = 390: second unit ends 122 rows short
    (1, 32, 9, 9, 96, 1, 1, 1, 0, 1, 1),       # M = 81: the odd CTA's rows all lie past M
    (2, 128, 12, 12, 256, 3, 3, 2, 1, 1, 1),   # stride 2, BN = 256 (128 weight rows per CTA)
    (2, 64, 11, 11, 64, 3, 3, 1, 2, 2, 2),     # 2 groups of 32 channels, dilation 2
    (1, 48, 16, 16, 32, 5, 5, 1, 2, 1, 1),     # 96-byte rows (32-byte planes), BN = 32
    (1, 40, 8, 8, 64, 1, 1, 1, 0, 1, 1),       # 1x1 direct loads, 80-byte rows (16-byte planes)
    (2, 96, 9, 9, 160, 2, 3, 1, 0, 1, 1),      # even kernel height, BN = 160
]


@pytest.mark.parametrize("layout", ["nhwc", "nchw"])
@pytest.mark.parametrize("shape", PAIR_EDGE, ids=lambda s: "x".join(map(str, s)))
def test_pair_edge_shapes(shape, layout, pairs_forced):
    N, C_in, H, W, C_out, Kh, Kw, s, p, d, g = shape
    cfg = workloads.ConvConfig("pair_edge", N, C_in, H, W, C_out, Kh, Kw, s, p, d, g, True, "bf16", layout,
                               seed=sum(shape) + 11)
    inp = workloads.make_inputs(cfg)
    parity.assert_close(cfg, parity.run_gpu(cfg, inp), parity.run_oracle(cfg, inp), str(shape) + " (pair)")


@pytest.mark.parametrize("shape", [(2, 32, 10, 10, 64, 3, 3, 1, 1, 1, 1), (3, 64, 9, 7, 96, 1, 1, 1, 0, 1, 1)],
                         ids=lambda s: "x".join(map(str, s)))
def test_pair_small_integers_bit_exact(shape, pairs_forced):
    """Integer inputs in [-2, 2]: every partial sum is exact, so the pair kernel's
    outputs equal the oracle's exactly."""
    N, C_in, H, W, C_out, Kh, Kw, s, p, d, g = shape
    cfg = workloads.ConvConfig("ints", N, C_in, H, W, C_out, Kh, Kw, s, p, d, g, True, "bf16", "nhwc",
                               ("integers", -2, 2), ("integers", -2, 2), ("integers", -2, 2), seed=5)
    inp = workloads.make_inputs(cfg)
    ref = parity.run_oracle(cfg, inp)
    assert np.abs(ref).max() <= 256
    assert np.array_equal(parity.run_gpu(cfg, inp), ref)


def test_pair_and_single_cta_kernels_agree_on_repeated_calls():
    """The same layer run with pairs forbidden, forced and back: the three results
    agree to the bf16 rounding of one output, and repeated pair calls are identical."""
    cfg = parity.config("resnet3x3_bf16_nhwc", N=3, H=14, W=14)
    inp = workloads.make_inputs(cfg)
    outs = []
    try:
        for mode in (2, 1, 1, 0):
            cb.conv2d_debug_set_pair_mode(mode)
            outs.append(parity.run_gpu(cfg, inp))
    finally:
        cb.conv2d_debug_set_pair_mode(0)
    assert np.array_equal(outs[1], outs[2])
    for o in (outs[0], outs[3]):
        assert np.abs(o - outs[1]).max() <= 2 ** -7 * max(1.0, np.abs(o).max())


def test_pair_watchdog_returns_timeout_instead_of_hanging(pairs_forced):
    """With loads withheld the waits of both CTAs of every pair run out; the kernel
    exits with TIMEOUT and the next normal call works."""
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
    cb.conv2d_sync_status()
    parity.assert_close(cfg, parity.run_gpu(cfg, inp, layer=layer), parity.run_oracle(cfg, inp), "after timeout")


@pytest.mark.parametrize("name", ["resnet3x3_bf16_nhwc", "k7_17x17_bf16"])
def test_pair_explicit_im2col_gemm(name, pairs_forced):
    """The pages' formulation (X_col in memory, then the GEMM) with the GEMM on CTA
    pairs reading X_col through tiled loads."""
    cfg = parity.config(name, **SMALL[name])
    inp = workloads.make_inputs(cfg)
    got = parity.run_gpu(cfg, inp, explicit_im2col=True)
    parity.assert_close(cfg, got, parity.run_oracle(cfg, inp), name + " (pair, explicit im2col)")


PW_SHAPES = [  # 1x1, stride 1, no padding: the kernel with each cluster's weight tile resident (bf16)
    ((2, 64, 9, 9, 256, 1, 1, 1, 0, 1, 1), True, "bf16"),     # M = 162: one row tile, the odd CTA's rows partly past M
    ((3, 128, 10, 11, 512, 1, 1, 1, 0, 1, 1), True, "bf16"),  # two column tiles, M = 330: a ragged second row tile
    ((1, 256, 12, 12, 768, 1, 1, 1, 0, 1, 1), False, "bf16"), # reduction 256 (four planes), three column tiles, no bias
    ((2, 192, 8, 8, 256, 1, 1, 1, 0, 1, 1), True, "bf16"),    # three planes
    ((2, 128, 8, 9, 512, 1, 1, 1, 0, 1, 2), True, "bf16"),    # two groups of 64 -> 256: clusters over (group, tile)
]


@pytest.mark.parametrize("shape,bias,dtype", PW_SHAPES,
                         ids=lambda s: "x".join(map(str, s)) if isinstance(s, tuple) else str(s))
def test_pointwise_resident_weights(shape, bias, dtype, pairs_forced):
    N, C_in, H, W, C_out, Kh, Kw, s, p, d, g = shape
    plan = cb.conv2d_describe_plan(*shape, cb.CONV_BF16 if dtype == "bf16" else cb.CONV_F32, "nhwc")
    assert plan["kernel"] == "pointwise", plan
    cfg = workloads.ConvConfig("pw", N, C_in, H, W, C_out, Kh, Kw, s, p, d, g, bias, dtype, "nhwc",
                               seed=sum(shape) + 21)
    inp = workloads.make_inputs(cfg)
    parity.assert_close(cfg, parity.run_gpu(cfg, inp), parity.run_oracle(cfg, inp), str(shape) + " (pointwise)")


def test_pointwise_resident_weights_integers_bit_exact(pairs_forced):
    shape = (3, 128, 9, 7, 512, 1, 1, 1, 0, 1, 1)
    assert cb.conv2d_describe_plan(*shape, cb.CONV_BF16, "nhwc")["kernel"] == "pointwise"
    ints = ("integers", -2, 2)
    cfg = workloads.ConvConfig("pw_ints", *shape, True, "bf16", "nhwc", ints, ints, ints, seed=9)
    inp = workloads.make_inputs(cfg)
    ref = parity.run_oracle(cfg, inp)
    assert np.abs(ref).max() <= 256
    assert np.array_equal(parity.run_gpu(cfg, inp), ref)


def test_pointwise_workload_takes_resident_weights():
    cfg = workloads.CONFIGS["pointwise1x1_bf16"]
    plan = cb.conv2d_describe_plan(cfg.N, cfg.C_in, cfg.H, cfg.W, cfg.C_out, cfg.Kh, cfg.Kw, cfg.stride, cfg.pad,
                                   cfg.dilation, cfg.groups, cb.CONV_BF16, cfg.layout)
    assert plan["kernel"] == "pointwise", plan
