"""Winograd F(2x2, 3x3) and F(4x4, 3x3) through the C ABI against the fp64 oracle
(needs a B200).

Winograd's minimal filtering reaches the convolution's own result (up to rounding), so
the oracle is the direct convolution (the same pinned six-loop oracle as the forward
pass), under the forward pass's tolerances."""
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


def run_wino(cfg, inp, m):
    import torch
    dt = torch.bfloat16 if cfg.dtype == "bf16" else torch.float32
    w = torch.from_numpy(inp["w"]).to(dt).cuda()
    b = None if inp["b"] is None else torch.from_numpy(inp["b"]).to(dt).cuda()
    layer = cb.WinogradConv2dB200(w, b, cfg.pad, m, cfg.layout)
    y = layer(parity.to_device_x(cfg, inp["x"]))
    cb.conv2d_sync_status()
    return parity.from_device_y(cfg, y)


WINO = [  # N, C_in, H, W, C_out, pad
    (2, 64, 12, 12, 64, 1),      # whole tiles for m = 2 and m = 4
    (1, 32, 17, 19, 48, 1),      # ragged last tiles in both directions
    (2, 3, 9, 11, 8, 1),         # three input channels (padded to 16 bytes), eight output channels
    (1, 64, 8, 8, 16, 0),        # no padding: 6x6 outputs
    (1, 16, 7, 7, 200, 2),       # pad 2, 200 output channels
    (1, 256, 14, 14, 256, 1),    # 256 channels each way
    (1, 96, 9, 9, 512, 1),       # 96 input channels, two 256-column tiles per transformed channel
]


@pytest.mark.parametrize("m", [2, 4])
@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("layout", ["nhwc", "nchw"])
@pytest.mark.parametrize("shape", WINO, ids=lambda s: "x".join(map(str, s)))
def test_winograd_matches_oracle(shape, layout, dtype, m):
    N, C_in, H, W, C_out, pad = shape
    cfg = workloads.ConvConfig("wino", N, C_in, H, W, C_out, 3, 3, 1, pad, 1, 1, True, dtype, layout,
                               seed=sum(shape) + m)
    inp = workloads.make_inputs(cfg)
    parity.assert_close(cfg, run_wino(cfg, inp, m), parity.run_oracle(cfg, inp), f"F({m}x{m},3x3) {shape}")


@pytest.mark.parametrize("m", [2, 4])
def test_winograd_full_size_3x3_sampled(m):
    """The ResNet-style 3x3 layer (the forward benchmark's workload) by Winograd: sampled
    outputs plus every corner against the oracle's definition."""
    import torch
    cfg = workloads.CONFIGS["resnet3x3_bf16_nhwc"]
    inp = workloads.make_inputs(cfg)
    w = torch.from_numpy(inp["w"]).to(torch.bfloat16).cuda()
    layer = cb.WinogradConv2dB200(w, None, cfg.pad, m, cfg.layout)
    y = layer(parity.to_device_x(cfg, inp["x"]))
    cb.conv2d_sync_status()
    idx = parity.sample_indices((cfg.N, cfg.C_out, cfg.Ho, cfg.Wo), 512, seed=12)
    got = y[tuple(torch.from_numpy(idx[:, i]).cuda() for i in (0, 2, 3, 1))].float().cpu().numpy()
    ref = oracle.conv2d_points(inp["x"], inp["w"], None, idx, 1, cfg.pad, 1, 1)
    assert np.abs(got - ref).max() <= parity.BF16_MAXABS * np.abs(ref).max()


def test_winograd_product_on_the_resident_weight_kernel():
    """bf16 F(2x2,3x3) with 256 channels each way and 2048 tiles (enough 256-row pair units for
    every SM pair): the product runs on the pair kernel with resident weights, writing the fp32
    M blocks by TMA stores; the whole output is checked against the oracle."""
    shape = (2, 256, 64, 64, 256, 1)
    assert cb.conv2d_winograd_describe_plan(*shape, 2, cb.CONV_BF16, "nhwc")["kernel"] == "pointwise"
    N, C_in, H, W, C_out, pad = shape
    cfg = workloads.ConvConfig("wino_pw", N, C_in, H, W, C_out, 3, 3, 1, pad, 1, 1, False, "bf16", "nhwc", seed=77)
    inp = workloads.make_inputs(cfg)
    parity.assert_close(cfg, run_wino(cfg, inp, 2), parity.run_oracle(cfg, inp), "F(2x2,3x3) on the pointwise kernel")


def test_winograd_rejects_other_tiles():
    with pytest.raises(cb.Conv2dError) as err:
        cb.conv2d_winograd_packed_weight_size(8, 8, 3, cb.CONV_BF16)
    assert err.value.status == cb.CONV_ERR_INVALID_ARG
