"""conv2d_forward_noalloc against conv2d_forward, through the C ABI (needs a B200).

Some callers cannot allocate device memory: code that runs while a CUDA graph is
being captured, code under a framework allocator that owns all device memory, or a
plugin whose host hands it only input and output buffers.  They call
conv2d_forward_noalloc, whose scratch is a fixed array compiled into the library
instead of a workspace they would have to allocate.

This file is named to be collected last, so that if it fails, a run that stops at
the first failure has already run every other test.
"""
import numpy as np
import pytest

import cnn_convolution_conv2d_b200 as cb
import parity

pytestmark = pytest.mark.gpu

CASES = {
    # NCHW input with 256 channels: the scratch holds the channels-last copy of x
    "nchw_copy_bf16": ("resnet3x3_bf16_nhwc", dict(N=2, H=20, W=20, layout="nchw")),
    # few output tiles, long reduction: the scratch holds split partial sums
    "split_sums_bf16": ("k7_17x17_bf16", dict(N=1, C_in=128, C_out=128)),
    # both at once, in fp32
    "copy_and_split_f32": ("k7_17x17_f32", dict(N=1, C_in=128, C_out=128, layout="nchw")),
}


@pytest.fixture(scope="module", autouse=True)
def cuda_ready():
    import torch
    assert torch.cuda.is_available(), "these tests need a CUDA device"
    from cnn_convolution_conv2d_b200 import build
    build.build()
    cb.load()
    cb.conv2d_debug_set_watchdog(0, False)


def _shape(layer, cfg):
    return (cfg.N, layer.C_in, cfg.H, cfg.W, layer.C_out, layer.Kh, layer.Kw, layer.stride, layer.pad,
            layer.dilation, layer.groups)


@pytest.fixture(params=[0, 1], ids=["auto", "pairs"])
def pair_mode(request):
    """Each case once with the library's own kernel choice and once with the CTA-pair
    kernel forced wherever the tile shape allows it (bf16 cases)."""
    cb.conv2d_debug_set_pair_mode(request.param)
    yield request.param
    cb.conv2d_debug_set_pair_mode(0)


@pytest.mark.parametrize("case", sorted(CASES))
def test_noalloc_matches_forward_on_two_calls(case, pair_mode):
    import torch
    name, kw = CASES[case]
    cfg = parity.config(name, **kw)
    inp = parity.workloads.make_inputs(cfg)
    layer = parity.make_layer(cfg, inp)
    x = parity.to_device_x(cfg, inp["x"])
    shape = _shape(layer, cfg)
    need = cb.conv2d_workspace_size(*shape, layer.dtype, layer.layout)
    assert need <= cb.NOALLOC_SCRATCH_BYTES
    if pair_mode == 0:
        assert need > 0  # the case exercises the built-in scratch (pairs need no split sums)
    ref = layer(x)                               # existing entry point, allocated workspace
    cb.conv2d_sync_status()
    want = parity.from_device_y(cfg, ref)
    for _ in range(2):                           # the second call finds the first call's scratch
        y = torch.full_like(ref, float("nan"))
        cb.conv2d_forward_noalloc(x, layer.w_packed, layer.bias, y, *shape, layer.dtype, layer.layout)
        cb.conv2d_sync_status()
        parity.assert_close(cfg, parity.from_device_y(cfg, y), want, case)


def test_noalloc_rejects_problems_beyond_its_scratch():
    import torch
    # NCHW input of 16 x 64 x 256 x 256 bf16: its channels-last copy alone is 128 MiB
    shape = (16, 64, 256, 256, 64, 3, 3, 1, 1, 1, 1)
    assert cb.conv2d_workspace_size(*shape, cb.CONV_BF16, "nchw") > cb.NOALLOC_SCRATCH_BYTES
    x = torch.empty(16 * 64 * 256 * 256, dtype=torch.bfloat16, device="cuda")
    w = torch.zeros(64, 64, 3, 3, dtype=torch.bfloat16, device="cuda")
    wp = cb.conv2d_pack_weight(w)
    y = torch.full((16, 64, 256, 256), 7.0, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(cb.Conv2dError) as err:
        cb.conv2d_forward_noalloc(x, wp, None, y, *shape, cb.CONV_BF16, "nchw")
    assert err.value.status == cb.CONV_ERR_WORKSPACE
    assert "scratch" in str(err.value)
    cb.conv2d_sync_status()
    assert bool((y == 7.0).all())                # nothing was written
