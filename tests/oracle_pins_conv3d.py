"""Pins for the conv3d oracle: facts the pages and the mathematics fix, each reached by
a route other than the oracle's own loops.

  * the shapes "PyTorch高维张量乘法与conv2d/conv3d维度语义解析" (pwwt.cn/news/6111401)
    prints: §5.1's (2, 3, 16, 64, 64) input through a 3x3x3 stride-1 pad-1 layer to
    (2, 16, 16, 64, 64); §6.2's two-layer network, D/H/W 16/64/64 after the first layer
    and 8/32/32 after the stride-2 second;
  * §5.3's equivalence: a (1, 3, 3) kernel is per-frame conv2d -- checked against the
    (separately pinned) conv2d oracle frame by frame;
  * the depth decomposition: the 3-D sum splits over kd into 2-D convolutions of single
    input frames with the kernel's kd-th slice (conv2d oracle again);
  * an explicit pad + strided-slice im2col + matrix product in NumPy;
  * PyTorch's float64 CPU conv3d (library special case);
  * all-ones kernels as box sums over a 3-D integral image.
"""
from __future__ import annotations

import numpy as np

import oracle


def _out(size, k, s, p, d):
    return (size + 2 * p - d * (k - 1) - 1) // s + 1


def im2col3d(x, w, b, s, p, d, g):
    """Explicit pad, im2col by strided slices, one matrix product per group."""
    N, C, D, H, W = x.shape
    Co, Cg, Kd, Kh, Kw = w.shape
    Do, Ho, Wo = _out(D, Kd, s, p, d), _out(H, Kh, s, p, d), _out(W, Kw, s, p, d)
    xp = np.pad(x, ((0, 0), (0, 0), (p, p), (p, p), (p, p)))
    cols = np.empty((N, C, Kd, Kh, Kw, Do, Ho, Wo))
    for a in range(Kd):
        for i in range(Kh):
            for j in range(Kw):
                cols[:, :, a, i, j] = xp[:, :, a * d: a * d + s * (Do - 1) + 1: s,
                                         i * d: i * d + s * (Ho - 1) + 1: s, j * d: j * d + s * (Wo - 1) + 1: s]
    y = np.empty((N, Co, Do, Ho, Wo))
    cog = Co // g
    for gi in range(g):
        xcol = cols[:, gi * Cg:(gi + 1) * Cg].transpose(1, 2, 3, 4, 0, 5, 6, 7).reshape(Cg * Kd * Kh * Kw, -1)
        wrow = w[gi * cog:(gi + 1) * cog].reshape(cog, -1)
        y[:, gi * cog:(gi + 1) * cog] = (wrow @ xcol).reshape(cog, N, Do, Ho, Wo).transpose(1, 0, 2, 3, 4)
    if b is not None:
        y = y + b[None, :, None, None, None]
    return y


CASES = [  # N, C, D, H, W, Co, Kd, Kh, Kw, s, p, d, g
    (2, 3, 6, 9, 8, 4, 3, 3, 3, 1, 1, 1, 1),     # pwwt §5.1's layer, small
    (1, 4, 9, 10, 11, 6, 3, 3, 3, 2, 1, 1, 2),   # stride 2 (pwwt §6.2's second layer), groups
    (2, 2, 5, 7, 6, 3, 1, 3, 3, 1, 1, 1, 1),     # (1, 3, 3): per-frame
    (1, 3, 8, 8, 8, 2, 2, 3, 2, 1, 2, 2, 1),     # non-cubic kernel, dilation 2
    (1, 4, 7, 6, 9, 4, 3, 1, 3, 3, 2, 1, 4),     # stride 3, depthwise-style groups
]


def _rand(rng, case, bias=True):
    N, C, D, H, W, Co, Kd, Kh, Kw, s, p, d, g = case
    x = rng.standard_normal((N, C, D, H, W))
    w = rng.standard_normal((Co, C // g, Kd, Kh, Kw))
    b = rng.standard_normal(Co) if bias else None
    return x, w, b, s, p, d, g


def pin_c3d_printed_shapes(lib):
    """pwwt §5.1 and §6.2's printed shapes."""
    x = np.zeros((2, 3, 16, 64, 64))
    y = oracle.conv3d(x, np.zeros((16, 3, 3, 3, 3)), None, 1, 1, 1, 1, lib=lib)
    assert y.shape == (2, 16, 16, 64, 64)
    x = np.zeros((1, 3, 16, 64, 64))
    y1 = oracle.conv3d(x, np.zeros((2, 3, 3, 3, 3)), None, 1, 1, 1, 1, lib=lib)
    assert y1.shape[2:] == (16, 64, 64)
    y2 = oracle.conv3d(y1, np.zeros((2, 2, 3, 3, 3)), None, 2, 1, 1, 1, lib=lib)
    assert y2.shape[2:] == (8, 32, 32)


def pin_c3d_per_frame(lib):
    """pwwt §5.3: with a (1, 3, 3) kernel and no depth padding every output frame is the
    conv2d of its input frame; with padding p the p outer frames on each side see only
    zero frames (bias alone) and the rest are still per-frame conv2d."""
    rng = np.random.default_rng(31)
    N, C, D, H, W, Co = 2, 3, 5, 8, 7, 4
    x = rng.standard_normal((N, C, D, H, W))
    w = rng.standard_normal((Co, C, 1, 3, 3))
    b = rng.standard_normal(Co)
    for p in (0, 1):
        y = oracle.conv3d(x, w, b, 1, p, 1, 1, lib=lib)
        assert y.shape[2] == D + 2 * p
        for f in range(D):
            want = oracle.conv2d(x[:, :, f], w[:, :, 0], b, 1, p, 1, 1)
            assert np.allclose(y[:, :, f + p], want, rtol=1e-13, atol=1e-12), (p, f)
        for f in list(range(p)) + list(range(D + p, D + 2 * p)):
            assert np.allclose(y[:, :, f], b[None, :, None, None] + 0 * y[:, :, f], rtol=0, atol=1e-15)


def pin_c3d_depth_decomposition(lib):
    """y[:, :, od] = bias + sum over kd of conv2d(x[:, :, od*s + kd*d - p], w[:, :, kd])
    (frames outside the volume dropped), with the conv2d oracle."""
    rng = np.random.default_rng(32)
    for case in CASES:
        x, w, b, s, p, d, g = _rand(rng, case)
        y = oracle.conv3d(x, w, b, s, p, d, g, lib=lib)
        D, Kd = x.shape[2], w.shape[2]
        for od in range(y.shape[2]):
            want = np.broadcast_to(b[None, :, None, None], y[:, :, od].shape).copy()
            for kd in range(Kd):
                f = od * s + kd * d - p
                if 0 <= f < D:
                    want += oracle.conv2d(x[:, :, f], w[:, :, kd], None, s, p, d, g)
            assert np.allclose(y[:, :, od], want, rtol=1e-12, atol=1e-11), (case, od)


def pin_c3d_im2col(lib):
    """Explicit pad + im2col + matrix product agrees to ~1e-13."""
    rng = np.random.default_rng(33)
    for case in CASES:
        x, w, b, s, p, d, g = _rand(rng, case)
        got = oracle.conv3d(x, w, b, s, p, d, g, lib=lib)
        want = im2col3d(x, w, b, s, p, d, g)
        assert got.shape == want.shape, case
        assert np.abs(got - want).max() / max(1.0, np.abs(want).max()) < 1e-13, case


def pin_c3d_torch_f64(lib):
    """PyTorch's float64 CPU conv3d (library special case)."""
    import torch
    rng = np.random.default_rng(34)
    for case in CASES:
        x, w, b, s, p, d, g = _rand(rng, case)
        want = torch.nn.functional.conv3d(torch.from_numpy(x), torch.from_numpy(w), torch.from_numpy(b), stride=s,
                                          padding=p, dilation=d, groups=g).numpy()
        got = oracle.conv3d(x, w, b, s, p, d, g, lib=lib)
        assert np.allclose(got, want, rtol=1e-12, atol=1e-10), case


def pin_c3d_box_sum(lib):
    """All-ones kernels: every output is the sum of the input over its (clipped) box,
    read off a 3-D integral image."""
    rng = np.random.default_rng(35)
    N, C, D, H, W, Co, K, s, p = 2, 3, 7, 8, 9, 2, 3, 2, 1
    x = rng.standard_normal((N, C, D, H, W))
    y = oracle.conv3d(x, np.ones((Co, C, K, K, K)), None, s, p, 1, 1, lib=lib)
    plane = np.pad(x.sum(1), ((0, 0), (p, p), (p, p), (p, p)))
    I = np.zeros((N,) + tuple(v + 1 for v in plane.shape[1:]))
    I[:, 1:, 1:, 1:] = plane.cumsum(1).cumsum(2).cumsum(3)
    for od in range(y.shape[2]):
        for oh in range(y.shape[3]):
            for ow in range(y.shape[4]):
                a0, b0, c0 = od * s, oh * s, ow * s
                a1, b1, c1 = a0 + K, b0 + K, c0 + K
                box = (I[:, a1, b1, c1] - I[:, a0, b1, c1] - I[:, a1, b0, c1] - I[:, a1, b1, c0]
                       + I[:, a0, b0, c1] + I[:, a0, b1, c0] + I[:, a1, b0, c0] - I[:, a0, b0, c0])
                assert np.allclose(y[:, 0, od, oh, ow], box, rtol=1e-12, atol=1e-11)
                assert np.allclose(y[:, 1, od, oh, ow], box, rtol=1e-12, atol=1e-11)


def pin_c3d_points_match_full(lib):
    rng = np.random.default_rng(36)
    for case in CASES:
        x, w, b, s, p, d, g = _rand(rng, case)
        y = oracle.conv3d(x, w, b, s, p, d, g, lib=lib)
        idx = np.stack([rng.integers(0, n, 30) for n in y.shape], axis=1)
        got = oracle.conv3d_points(x, w, b, idx, s, p, d, g, lib=lib)
        assert np.allclose(got, y[tuple(idx.T)], rtol=1e-14, atol=1e-13), case


ALL_PINS = [pin_c3d_printed_shapes, pin_c3d_per_frame, pin_c3d_depth_decomposition, pin_c3d_im2col,
            pin_c3d_torch_f64, pin_c3d_box_sum, pin_c3d_points_match_full]
