"""Named convolution workloads and their seeded synthetic inputs.

This module only describes shapes and draws random inputs; it holds none of the
convolution's arithmetic, so both the CUDA path and the CPU oracle can be fed
from it.  Inputs are drawn with numpy's PCG64 generator (``default_rng(seed)``)
as float32, x first, then w, then bias, and rounded to nearest-even bfloat16 for
bf16 workloads so that both sides see identical values.

Shapes follow the pages' layouts: x is (N, C_in, H, W), w is
(C_out, C_in/groups, Kh, Kw), bias is (C_out,)  ("PyTorch高维张量乘法与
conv2d/conv3d维度语义解析" §4.1).  ``layout`` says how the CUDA path receives x
and returns y: "nchw" (as drawn) or "nhwc" (channels last).
"""
from __future__ import annotations

import dataclasses
import math

import numpy as np


@dataclasses.dataclass(frozen=True)
class ConvConfig:
    name: str
    N: int
    C_in: int
    H: int
    W: int
    C_out: int
    Kh: int
    Kw: int
    stride: int = 1
    pad: int = 0
    dilation: int = 1
    groups: int = 1
    bias: bool = True
    dtype: str = "bf16"          # "bf16" (fp32 accumulate) or "f32"
    layout: str = "nhwc"         # how x and y cross the C ABI
    x_dist: tuple = ("normal", 1.0)      # ("normal", variance) or ("uniform", lo, hi)
    w_dist: tuple = ("normal", 1.0)
    b_dist: tuple = ("normal", 1.0)
    seed: int = 0

    @property
    def Ho(self) -> int:
        return (self.H + 2 * self.pad - self.dilation * (self.Kh - 1) - 1) // self.stride + 1

    @property
    def Wo(self) -> int:
        return (self.W + 2 * self.pad - self.dilation * (self.Kw - 1) - 1) // self.stride + 1

    def scaled(self, **kw) -> "ConvConfig":
        """The same workload with some fields replaced (e.g. a smaller N or H)."""
        return dataclasses.replace(self, **kw)

    def params(self) -> dict:
        return {k: getattr(self, k) for k in ("N", "C_in", "H", "W", "C_out", "Kh", "Kw",
                                                "stride", "pad", "dilation", "groups")}


def _he(fan_in: int) -> tuple:
    return ("normal", 2.0 / fan_in)


CONFIGS = {
    # N=2, C_in=3, 9x11, C_out=4, 3x3, stride 2, pad 1, bias; U(-1,1); seed 0
    "tiny_f32_nchw": ConvConfig("tiny_f32_nchw", 2, 3, 9, 11, 4, 3, 3, 2, 1, 1, 1, True, "f32", "nchw",
                                ("uniform", -1.0, 1.0), ("uniform", -1.0, 1.0), ("uniform", -1.0, 1.0), 0),
    # first layer: 32x3x224x224 -> 64, 7x7, stride 2, pad 3; w ~ N(0, 1/(3*49))
    "stem_bf16": ConvConfig("stem_bf16", 32, 3, 224, 224, 64, 7, 7, 2, 3, 1, 1, True, "bf16", "nchw",
                            ("normal", 1.0), ("normal", 1.0 / 147), ("normal", 1.0), 1),
    # ResNet 3x3: 64x256x56x56 -> 256, stride 1, pad 1, no bias; w ~ N(0, 2/(256*9))
    "resnet3x3_bf16_nhwc": ConvConfig("resnet3x3_bf16_nhwc", 64, 256, 56, 56, 256, 3, 3, 1, 1, 1, 1, False,
                                      "bf16", "nhwc", ("normal", 1.0), _he(2304), ("normal", 1.0), 2),
    # pointwise 1x1: 64x256x56x56 -> 1024, bias
    "pointwise1x1_bf16": ConvConfig("pointwise1x1_bf16", 64, 256, 56, 56, 1024, 1, 1, 1, 0, 1, 1, True,
                                    "bf16", "nhwc", ("normal", 1.0), _he(256), ("normal", 1.0), 3),
    # strided + dilated + grouped: 16x512x28x28 -> 512, 3x3, s2 p2 d2 g32, bias
    "grouped_dilated_bf16": ConvConfig("grouped_dilated_bf16", 16, 512, 28, 28, 512, 3, 3, 2, 2, 2, 32, True,
                                       "bf16", "nhwc", ("normal", 1.0), _he(144), ("normal", 1.0), 4),
    "grouped_dilated_f32": ConvConfig("grouped_dilated_f32", 16, 512, 28, 28, 512, 3, 3, 2, 2, 2, 32, True,
                                      "f32", "nhwc", ("normal", 1.0), _he(144), ("normal", 1.0), 4),
    # 7x7, stride 1, pad 3 on 17x17 (non-divisible M edge): 16x512 -> 512, groups 1
    "k7_17x17_bf16": ConvConfig("k7_17x17_bf16", 16, 512, 17, 17, 512, 7, 7, 1, 3, 1, 1, True,
                                "bf16", "nhwc", ("normal", 1.0), _he(512 * 49), ("normal", 1.0), 5),
    "k7_17x17_f32": ConvConfig("k7_17x17_f32", 16, 512, 17, 17, 512, 7, 7, 1, 3, 1, 1, True,
                               "f32", "nhwc", ("normal", 1.0), _he(512 * 49), ("normal", 1.0), 5),
    # depthwise 3x3 (groups = C_in = C_out, one filter per channel): the variant the
    # im2col/GEMM tutorial (zskr.cn/news/1820658) §4.2 and "手撕 Conv2D" §7 single out;
    # the 3x3 layer's activations, 64x256x56x56, stride 1, pad 1, bias; w ~ N(0, 2/9)
    "depthwise3x3_bf16": ConvConfig("depthwise3x3_bf16", 64, 256, 56, 56, 256, 3, 3, 1, 1, 1, 256, True,
                                    "bf16", "nhwc", ("normal", 1.0), _he(9), ("normal", 1.0), 6),
    "depthwise3x3_f32": ConvConfig("depthwise3x3_f32", 64, 256, 56, 56, 256, 3, 3, 1, 1, 1, 256, True,
                                   "f32", "nhwc", ("normal", 1.0), _he(9), ("normal", 1.0), 6),
}


def bf16_round(a: np.ndarray) -> np.ndarray:
    """Round float32 values to the nearest bfloat16 (ties to even); returns float32."""
    bits = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32).astype(np.uint64)
    bits = (bits + 0x7FFF + ((bits >> 16) & 1)) >> 16
    return (bits.astype(np.uint32) << 16).view(np.float32)


def bf16_bits(a: np.ndarray) -> np.ndarray:
    """The bfloat16 bit patterns of float32 values that are already bf16-exact."""
    return (np.ascontiguousarray(a, dtype=np.float32).view(np.uint32) >> 16).astype(np.uint16)


def _draw(rng, dist, shape):
    if dist[0] == "normal":
        return (rng.standard_normal(shape, dtype=np.float32) * np.float32(math.sqrt(dist[1])))
    if dist[0] == "uniform":
        return rng.uniform(dist[1], dist[2], shape).astype(np.float32)
    if dist[0] == "integers":  # small integers: every partial sum is exact in fp32
        return rng.integers(dist[1], dist[2] + 1, shape).astype(np.float32)
    raise ValueError(dist)


def make_inputs(cfg: ConvConfig, seed: int | None = None) -> dict:
    """Seeded x (NCHW), w (OIHW) and bias (or None) as float32 arrays.

    For bf16 workloads every value is already rounded to bfloat16."""
    rng = np.random.default_rng(cfg.seed if seed is None else seed)
    x = _draw(rng, cfg.x_dist, (cfg.N, cfg.C_in, cfg.H, cfg.W))
    w = _draw(rng, cfg.w_dist, (cfg.C_out, cfg.C_in // cfg.groups, cfg.Kh, cfg.Kw))
    b = _draw(rng, cfg.b_dist, (cfg.C_out,)) if cfg.bias else None
    if cfg.dtype == "bf16":
        x, w = bf16_round(x), bf16_round(w)
        b = None if b is None else bf16_round(b)
    return {"x": x, "w": w, "b": b}


@dataclasses.dataclass(frozen=True)
class Conv3dConfig:
    """A 3-D convolution workload: x (N, C_in, D, H, W), w (C_out, C_in/groups, Kd, Kh, Kw)
    ("PyTorch高维张量乘法与conv2d/conv3d维度语义解析" §5.1).  ``layout`` "nchw" means NCDHW,
    "nhwc" NDHWC."""
    name: str
    N: int
    C_in: int
    D: int
    H: int
    W: int
    C_out: int
    Kd: int
    Kh: int
    Kw: int
    stride: int = 1
    pad: int = 0
    dilation: int = 1
    groups: int = 1
    bias: bool = True
    dtype: str = "bf16"
    layout: str = "nhwc"
    x_dist: tuple = ("normal", 1.0)
    w_dist: tuple = ("normal", 1.0)
    b_dist: tuple = ("normal", 1.0)
    seed: int = 0

    def _o(self, v, k):
        return (v + 2 * self.pad - self.dilation * (k - 1) - 1) // self.stride + 1

    @property
    def Do(self) -> int:
        return self._o(self.D, self.Kd)

    @property
    def Ho(self) -> int:
        return self._o(self.H, self.Kh)

    @property
    def Wo(self) -> int:
        return self._o(self.W, self.Kw)

    def scaled(self, **kw) -> "Conv3dConfig":
        return dataclasses.replace(self, **kw)


CONFIGS3D = {
    # the two layers of the network "PyTorch高维张量乘法与conv2d/conv3d维度语义解析" §6.2 runs:
    # x (4, 3, 16, 64, 64) -> 16 channels, 3x3x3, stride 1, pad 1 -> 32 channels, stride 2
    "conv3d_l1_bf16": Conv3dConfig("conv3d_l1_bf16", 4, 3, 16, 64, 64, 16, 3, 3, 3, 1, 1, 1, 1, True, "bf16",
                                   "nchw", ("normal", 1.0), ("normal", 2.0 / 81), ("normal", 1.0), 7),
    "conv3d_l2_bf16": Conv3dConfig("conv3d_l2_bf16", 4, 16, 16, 64, 64, 32, 3, 3, 3, 2, 1, 1, 1, True, "bf16",
                                   "nhwc", ("normal", 1.0), ("normal", 2.0 / 432), ("normal", 1.0), 8),
    # a wider video block of the same kind (64 channels, 16 frames of 56x56): the
    # throughput workload of the 3-D path
    "conv3d_video_bf16": Conv3dConfig("conv3d_video_bf16", 8, 64, 16, 56, 56, 64, 3, 3, 3, 1, 1, 1, 1, True, "bf16",
                                      "nhwc", ("normal", 1.0), ("normal", 2.0 / 1728), ("normal", 1.0), 9),
    "conv3d_video_f32": Conv3dConfig("conv3d_video_f32", 8, 64, 16, 56, 56, 64, 3, 3, 3, 1, 1, 1, 1, True, "f32",
                                     "nhwc", ("normal", 1.0), ("normal", 2.0 / 1728), ("normal", 1.0), 9),
}


def make_inputs3d(cfg: Conv3dConfig, seed: int | None = None) -> dict:
    """Seeded x (NCDHW), w (OIDHW) and bias as float32 (bf16-rounded for bf16 workloads)."""
    rng = np.random.default_rng(cfg.seed if seed is None else seed)
    x = _draw(rng, cfg.x_dist, (cfg.N, cfg.C_in, cfg.D, cfg.H, cfg.W))
    w = _draw(rng, cfg.w_dist, (cfg.C_out, cfg.C_in // cfg.groups, cfg.Kd, cfg.Kh, cfg.Kw))
    b = _draw(rng, cfg.b_dist, (cfg.C_out,)) if cfg.bias else None
    if cfg.dtype == "bf16":
        x, w = bf16_round(x), bf16_round(w)
        b = None if b is None else bf16_round(b)
    return {"x": x, "w": w, "b": b}
