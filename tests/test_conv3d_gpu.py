"""The 3-D convolution forward pass through the C ABI against the fp64 conv3d oracle
(needs a B200).

The oracle is pinned on the CPU (tests/oracle_pins_conv3d.py).  Cases span several
128-row tiles with ragged ends, non-cubic filters, strides, dilation and groups; the
workloads of "PyTorch高维张量乘法与conv2d/conv3d维度语义解析" §6.2 and the wider video
block are compared element by element over the whole output."""
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


def run_gpu3d(cfg, inp):
    import torch
    dt = torch.bfloat16 if cfg.dtype == "bf16" else torch.float32
    w = torch.from_numpy(inp["w"]).to(dt).cuda()
    b = None if inp["b"] is None else torch.from_numpy(inp["b"]).to(dt).cuda()
    layer = cb.Conv3dB200(w, b, cfg.stride, cfg.pad, cfg.dilation, cfg.groups, cfg.layout)
    x = torch.from_numpy(inp["x"]).to(dt)
    if cfg.layout == "nhwc":
        x = x.permute(0, 2, 3, 4, 1)
    y = layer(x.contiguous().cuda())
    cb.conv2d_sync_status()
    y = y.float().cpu()
    if cfg.layout == "nhwc":
        y = y.permute(0, 4, 1, 2, 3)
    return y.contiguous().numpy().astype(np.float64)


def run_oracle3d(cfg, inp):
    return oracle.conv3d(inp["x"], inp["w"], inp["b"], cfg.stride, cfg.pad, cfg.dilation, cfg.groups)


EDGE3D = [  # N, C_in, D, H, W, C_out, Kd, Kh, Kw, stride, pad, dilation, groups
    (2, 16, 6, 9, 8, 32, 3, 3, 3, 1, 1, 1, 1),      # ragged last tile (864 voxels)
    (1, 64, 7, 10, 11, 48, 3, 3, 3, 2, 1, 1, 1),    # stride 2, 128-byte channel rows, C_out 48
    (2, 3, 5, 12, 12, 8, 3, 3, 3, 1, 1, 1, 1),      # three input channels: the (kd, kh)-folded 2-D form
    (1, 3, 6, 10, 10, 16, 3, 3, 3, 2, 1, 1, 1),     # three input channels at stride 2 (folded, column stride 2)
    (1, 32, 8, 8, 8, 16, 2, 3, 5, 1, 2, 2, 1),      # non-cubic filter, dilation 2
    (1, 64, 4, 9, 9, 64, 1, 3, 3, 1, 1, 1, 4),      # (1, 3, 3) filter, groups of 16
    (2, 24, 9, 6, 7, 40, 3, 1, 3, 3, 2, 1, 1),      # stride 3, filter of height 1
    (1, 32, 5, 5, 5, 32, 1, 1, 1, 1, 0, 1, 1),      # 1x1x1: the input read as the im2col matrix
    (3, 8, 1, 7, 7, 16, 1, 3, 3, 1, 1, 1, 1),       # a single frame
]


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("layout", ["nhwc", "nchw"])
@pytest.mark.parametrize("shape", EDGE3D, ids=lambda s: "x".join(map(str, s)))
def test_conv3d_edge_shapes(shape, layout, dtype):
    cfg = workloads.Conv3dConfig("edge3d", *shape, True, dtype, layout, seed=sum(shape))
    inp = workloads.make_inputs3d(cfg)
    parity.assert_close(cfg, run_gpu3d(cfg, inp), run_oracle3d(cfg, inp), str(shape))


FOLDED = [  # few-channel inputs at stride 1: (kd, kh) folded into the channels, then a 1 x Kw product
    ((2, 3, 7, 13, 11, 16, 3, 3, 3, 1, 1, 1, 1), "nchw", "bf16"),   # the first 3-D layer's form, ragged tiles
    ((1, 3, 6, 9, 10, 16, 3, 3, 3, 1, 1, 1, 1), "nhwc", "f32"),     # fp32 (three tf32 products), channels-last
    ((1, 1, 8, 9, 9, 8, 3, 5, 3, 1, 2, 2, 1), "nchw", "bf16"),      # one channel, non-cubic filter, dilation 2
    ((2, 8, 5, 6, 7, 32, 2, 2, 3, 1, 0, 1, 1), "nhwc", "bf16"),     # eight channels (16-byte rows), no padding
    ((1, 4, 5, 7, 8, 24, 3, 3, 1, 1, 1, 1, 1), "nchw", "f32"),      # Kw = 1: the folded product is 1x1
    ((1, 2, 4, 8, 8, 16, 1, 3, 3, 1, 1, 1, 1), "nhwc", "bf16"),     # Kd = 1: only the rows fold
    ((2, 8, 9, 12, 13, 32, 3, 3, 3, 2, 1, 1, 1), "nhwc", "bf16"),   # eight channels, stride 2 (16-byte copy path)
    ((1, 3, 7, 11, 12, 16, 3, 3, 3, 3, 2, 1, 1), "nchw", "bf16"),   # stride 3, pad 2
    ((1, 4, 6, 9, 10, 24, 3, 3, 3, 2, 1, 2, 1), "nhwc", "f32"),     # fp32 four channels, stride 2, dilation 2
]


@pytest.mark.parametrize("shape,layout,dtype", FOLDED, ids=lambda s: "x".join(map(str, s)) if isinstance(s, tuple) else s)
def test_conv3d_folded_few_channels(shape, layout, dtype):
    plan = cb.conv3d_describe_plan(*shape, cb.CONV_BF16 if dtype == "bf16" else cb.CONV_F32, layout)
    assert plan["fold"] == 1 and plan["xcopy"] == 0, plan
    cfg = workloads.Conv3dConfig("fold", *shape, True, dtype, layout, seed=sum(shape) + 5)
    inp = workloads.make_inputs3d(cfg)
    parity.assert_close(cfg, run_gpu3d(cfg, inp), run_oracle3d(cfg, inp), str(shape) + " (folded)")


def test_conv3d_folded_integers_bit_exact():
    shape = (2, 3, 6, 10, 9, 16, 3, 3, 3, 1, 1, 1, 1)
    assert cb.conv3d_describe_plan(*shape, cb.CONV_BF16, "nchw")["fold"] == 1
    ints = ("integers", -2, 2)
    cfg = workloads.Conv3dConfig("fold_ints", *shape, True, "bf16", "nchw", ints, ints, ints, seed=11)
    inp = workloads.make_inputs3d(cfg)
    ref = run_oracle3d(cfg, inp)
    assert np.abs(ref).max() <= 256
    assert np.array_equal(run_gpu3d(cfg, inp), ref)


VOL_REUSE = [  # N, C_in, D, H, W, C_out, Kd, Kh, Kw, stride, pad, dilation, groups; bias
    ((2, 64, 7, 16, 16, 64, 3, 3, 3, 1, 1, 1, 1), True),    # Do = 7: the last unit has 3 of 4 slices
    ((2, 64, 7, 16, 16, 64, 3, 3, 3, 1, 1, 1, 1), False),   # ... without bias
    ((1, 64, 5, 12, 24, 32, 3, 3, 3, 1, 1, 1, 1), True),    # 288 voxels a slice: a 32-voxel tile; C_out 32
    ((1, 64, 6, 16, 20, 96, 1, 3, 3, 1, 1, 1, 1), True),    # one depth tap, C_out 96 (2 slices per unit)
    ((1, 64, 8, 18, 34, 64, 3, 3, 3, 1, 0, 1, 1), True),    # no padding, 512 voxels a slice
    ((1, 64, 6, 16, 16, 128, 3, 1, 1, 1, 0, 1, 1), True),   # C_out 128, a (3, 1, 1) filter
    ((1, 64, 4, 16, 16, 128, 3, 3, 3, 1, 1, 1, 1), True),   # C_out 128: products one depth tap wide
    ((2, 64, 3, 18, 18, 64, 3, 3, 3, 1, 0, 1, 1), True),    # one output slice per image (J = 1)
]


@pytest.mark.parametrize("shape,bias", VOL_REUSE, ids=lambda s: "x".join(map(str, s)) if isinstance(s, tuple) else str(s))
def test_conv3d_input_slice_reuse(shape, bias):
    """bf16 NDHWC, stride 1, 64 input channels: the kernel that loads each input depth
    slice once for every depth tap that reads it, over the whole output."""
    plan = cb.conv3d_describe_plan(*shape, cb.CONV_BF16, "nhwc")
    assert plan["kernel"] == "vol_reuse", plan
    cfg = workloads.Conv3dConfig("reuse3d", *shape, bias, "bf16", "nhwc", seed=sum(shape))
    inp = workloads.make_inputs3d(cfg)
    parity.assert_close(cfg, run_gpu3d(cfg, inp), run_oracle3d(cfg, inp), str(shape))


def test_conv3d_input_slice_reuse_integers_bit_exact():
    ints = ("integers", -1, 1)
    cfg = workloads.Conv3dConfig("ints3d", 1, 64, 6, 16, 16, 64, 3, 3, 3, 1, 1, 1, 1, True, "bf16", "nhwc",
                                 ints, ints, ints, seed=5)
    assert cb.conv3d_describe_plan(1, 64, 6, 16, 16, 64, 3, 3, 3, 1, 1, 1, 1, cb.CONV_BF16, "nhwc")["kernel"] == "vol_reuse"
    inp = workloads.make_inputs3d(cfg)
    ref = run_oracle3d(cfg, inp)
    assert np.abs(ref).max() <= 256
    assert np.array_equal(run_gpu3d(cfg, inp), ref)


def test_conv3d_video_layer_takes_input_slice_reuse():
    cfg = workloads.CONFIGS3D["conv3d_video_bf16"]
    plan = cb.conv3d_describe_plan(cfg.N, cfg.C_in, cfg.D, cfg.H, cfg.W, cfg.C_out, cfg.Kd, cfg.Kh, cfg.Kw,
                                   cfg.stride, cfg.pad, cfg.dilation, cfg.groups, cb.CONV_BF16, cfg.layout)
    assert plan["kernel"] == "vol_reuse", plan


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_conv3d_small_integers_bit_exact(dtype):
    ints = ("integers", -2, 2)
    cfg = workloads.Conv3dConfig("ints3d", 2, 16, 5, 6, 7, 16, 3, 3, 3, 1, 1, 1, 1, True, dtype, "nhwc",
                                 ints, ints, ints, seed=3)
    inp = workloads.make_inputs3d(cfg)
    ref = run_oracle3d(cfg, inp)
    assert np.abs(ref).max() <= 256
    assert np.array_equal(run_gpu3d(cfg, inp), ref)


def test_conv3d_one_frame_filter_is_per_frame_conv2d():
    """pwwt §5.3 on the GPU: a (1, 3, 3) filter gives, frame by frame, what the 2-D
    forward pass gives on that frame (with depth padding 1 the real frames are 1..D)."""
    import torch
    cfg = workloads.Conv3dConfig("frames", 2, 32, 4, 10, 9, 16, 1, 3, 3, 1, 1, 1, 1, True, "bf16", "nchw", seed=4)
    inp = workloads.make_inputs3d(cfg)
    got = run_gpu3d(cfg, inp)                      # pad 1 in depth too: frames 1..D are the real ones
    w2 = torch.from_numpy(inp["w"][:, :, 0]).to(torch.bfloat16).cuda()
    b2 = torch.from_numpy(inp["b"]).to(torch.bfloat16).cuda()
    layer2 = cb.Conv2dB200(w2, b2, 1, 1, 1, 1, "nchw")
    for f in range(cfg.D):
        x2 = torch.from_numpy(np.ascontiguousarray(inp["x"][:, :, f])).to(torch.bfloat16).cuda()
        y2 = layer2(x2).float().cpu().numpy().astype(np.float64)
        # the two paths may tile and split the reduction differently: equal up to the
        # order of fp32 additions, i.e. within the bf16 bar
        assert np.abs(got[:, :, f + 1] - y2).max() <= parity.BF16_MAXABS * np.abs(y2).max(), f


@pytest.mark.parametrize("name", sorted(workloads.CONFIGS3D))
def test_conv3d_workloads_whole_output(name):
    cfg = workloads.CONFIGS3D[name]
    inp = workloads.make_inputs3d(cfg)
    parity.assert_close(cfg, run_gpu3d(cfg, inp), run_oracle3d(cfg, inp), name)
