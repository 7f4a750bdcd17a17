"""Helpers shared by the GPU parity tests: run the CUDA path through the C ABI on
seeded inputs and compare with the oracle under the stated tolerances.

Tolerances (the bars the convolution must meet against the fp64 oracle):
  fp32 : normwise relative error ||y - y_ref||_2 / ||y_ref||_2 <= 1e-5
  bf16 : max |y - y_ref| <= 2e-2 * max |y_ref|, with the oracle run on the same
         bf16-rounded x, w and bias.
"""
from __future__ import annotations

import numpy as np

import cnn_convolution_conv2d_b200 as cb
from cnn_convolution_conv2d_b200 import workloads

F32_NORMWISE = 1e-5
BF16_MAXABS = 2e-2


def torch_dtype(cfg):
    import torch
    return torch.bfloat16 if cfg.dtype == "bf16" else torch.float32


def to_device_x(cfg, x_nchw):
    import torch
    t = torch.from_numpy(np.ascontiguousarray(x_nchw)).to(torch_dtype(cfg))
    if cfg.layout == "nhwc":
        t = t.permute(0, 2, 3, 1).contiguous()
    return t.cuda()


def from_device_y(cfg, y):
    import torch
    y = y.to(torch.float32).cpu()
    if cfg.layout == "nhwc":
        y = y.permute(0, 3, 1, 2)
    return y.contiguous().numpy().astype(np.float64)


def make_layer(cfg, inp):
    import torch
    dt = torch_dtype(cfg)
    w = torch.from_numpy(inp["w"]).to(dt).cuda()
    b = None if inp["b"] is None else torch.from_numpy(inp["b"]).to(dt).cuda()
    return cb.Conv2dB200(w, b, cfg.stride, cfg.pad, cfg.dilation, cfg.groups, cfg.layout)


def run_gpu(cfg, inp, explicit_im2col=False, layer=None):
    """y (NCHW float64) from the CUDA path for the config's layout and dtype."""
    layer = layer or make_layer(cfg, inp)
    y = layer(to_device_x(cfg, inp["x"]), explicit_im2col=explicit_im2col)
    cb.conv2d_sync_status()
    return from_device_y(cfg, y)


def run_oracle(cfg, inp):
    import oracle
    return oracle.conv2d(inp["x"], inp["w"], inp["b"], cfg.stride, cfg.pad, cfg.dilation, cfg.groups)


def errors(got, ref):
    diff = np.abs(got - ref)
    return {
        "max_abs": float(diff.max()) if diff.size else 0.0,
        "max_ref": float(np.abs(ref).max()) if ref.size else 0.0,
        "normwise": float(np.linalg.norm((got - ref).ravel()) / max(np.linalg.norm(ref.ravel()), 1e-300)),
    }


def assert_close(cfg, got, ref, what=""):
    assert got.shape == ref.shape, (what, got.shape, ref.shape)
    assert np.all(np.isfinite(got)), f"{what}: non-finite output"
    e = errors(got, ref)
    if cfg.dtype == "f32":
        assert e["normwise"] <= F32_NORMWISE, (what, e)
    else:
        assert e["max_abs"] <= BF16_MAXABS * e["max_ref"], (what, e)
    return e


def sample_indices(shape, count, seed):
    """Random output indices plus the corners of every dimension (first/last image,
    channel, row and column), as rows (n, oc, oh, ow)."""
    rng = np.random.default_rng(seed)
    idx = [rng.integers(0, n, count) for n in shape]
    rand = np.stack(idx, axis=1)
    corners = np.array([[a, b, c, d] for a in (0, shape[0] - 1) for b in (0, shape[1] - 1)
                        for c in (0, shape[2] - 1) for d in (0, shape[3] - 1)])
    return np.concatenate([rand, corners]).astype(np.int64)


def config(name, **kw):
    return workloads.CONFIGS[name].scaled(**kw) if kw else workloads.CONFIGS[name]
