"""Pins for the CPU oracle: checks against facts the pages and the mathematics fix.

Every pin takes an oracle library handle (``oracle.load()`` or a deliberately
mutated build) and raises AssertionError when the oracle disagrees.  None of them
re-types the oracle's own loop: each uses a different route to the same number
(values printed on the pages, an integral-image box sum, an explicit
pad + im2col + matrix product, PyTorch's CPU convolution in float64, exact integer
arithmetic, or an invariant of the definition).

Page names used below:
  pwwt  = "PyTorch高维张量乘法与conv2d/conv3d维度语义解析" (pwwt.cn/news/6111401)
  dpshk = Conv2d documentation walk-through (dpshk.com/news/5792599,
          page title "企业官网建设流程全解析")
  lpnh  = "手撕 Conv2D" interview page (lpnh.cn/news/2493075)
  zskr  = im2col + GEMM tutorial (zskr.cn/news/1820658)
"""
from __future__ import annotations

import os

import numpy as np

import oracle

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


# ---------------------------------------------------------------- fixtures ---
def read_output_size_cases():
    """Rows (in, k, stride, pad, dilation, expected, source) of output_size.txt."""
    rows = []
    with open(os.path.join(GOLDEN, "output_size.txt"), encoding="utf-8") as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            parts = line.split(None, 6)
            nums = [int(v) for v in parts[:6]]
            rows.append((*nums, parts[6] if len(parts) > 6 else ""))
    return rows


def read_worked_example():
    """Parsed contents of conv2d_docs_worked_example.txt."""
    data = {"padded_c0": [], "window_c0": []}
    with open(os.path.join(GOLDEN, "conv2d_docs_worked_example.txt"), encoding="utf-8") as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            key, *vals = line.split()
            vals = [int(v) for v in vals]
            if key in data:
                data[key].append(vals)
            else:
                data[key] = vals
    data["padded_c0"] = np.array(data["padded_c0"], dtype=np.float64)
    data["window_c0"] = np.array(data["window_c0"], dtype=np.float64)
    return data


# ------------------------------------------------- independent computations ---
def _out(size, k, s, p, d):
    return (size + 2 * p - d * (k - 1) - 1) // s + 1


def im2col_conv(x, w, b, s, p, d, g, dtype=np.float64):
    """Explicit zero pad, im2col by strided slices, then one matrix product per group.

    The formulation of zskr §2.2-§2.3 (Y = W_row @ X_col) and the sliced im2col of
    lpnh §4.2, extended with dilation (slice start kh*d) and groups (one product per
    channel block, pwwt §4.3)."""
    x = np.asarray(x, dtype=dtype)
    w = np.asarray(w, dtype=dtype)
    N, C, H, W = x.shape
    Co, Cg, Kh, Kw = w.shape
    Ho, Wo = _out(H, Kh, s, p, d), _out(W, Kw, s, p, d)
    xp = np.pad(x, ((0, 0), (0, 0), (p, p), (p, p)))
    cols = np.empty((N, C, Kh, Kw, Ho, Wo), dtype=dtype)
    for i in range(Kh):
        for j in range(Kw):
            cols[:, :, i, j] = xp[:, :, i * d: i * d + s * (Ho - 1) + 1: s,
                                  j * d: j * d + s * (Wo - 1) + 1: s]
    y = np.empty((N, Co, Ho, Wo), dtype=dtype)
    cog = Co // g
    for gi in range(g):
        xcol = cols[:, gi * Cg:(gi + 1) * Cg].transpose(1, 2, 3, 0, 4, 5).reshape(Cg * Kh * Kw, N * Ho * Wo)
        wrow = w[gi * cog:(gi + 1) * cog].reshape(cog, Cg * Kh * Kw)
        y[:, gi * cog:(gi + 1) * cog] = (wrow @ xcol).reshape(cog, N, Ho, Wo).transpose(1, 0, 2, 3)
    if b is not None:
        y = y + np.asarray(b, dtype=dtype)[None, :, None, None]
    return y


def box_sum_conv(x, Co, Kh, Kw, s, p, g, b=None):
    """Convolution with an all-ones kernel as a box sum over an integral image."""
    x = np.asarray(x, dtype=np.float64)
    N, C, H, W = x.shape
    Cg, cog = C // g, Co // g
    Ho, Wo = _out(H, Kh, s, p, 1), _out(W, Kw, s, p, 1)
    y = np.empty((N, Co, Ho, Wo))
    r0 = np.arange(Ho) * s
    c0 = np.arange(Wo) * s
    for gi in range(g):
        plane = x[:, gi * Cg:(gi + 1) * Cg].sum(axis=1)
        plane = np.pad(plane, ((0, 0), (p, p), (p, p)))
        integ = np.zeros((N, plane.shape[1] + 1, plane.shape[2] + 1))
        integ[:, 1:, 1:] = plane.cumsum(1).cumsum(2)
        R0, C0 = np.meshgrid(r0, c0, indexing="ij")
        R1, C1 = R0 + Kh, C0 + Kw
        box = integ[:, R1, C1] - integ[:, R0, C1] - integ[:, R1, C0] + integ[:, R0, C0]
        y[:, gi * cog:(gi + 1) * cog] = box[:, None]
    if b is not None:
        y = y + np.asarray(b, dtype=np.float64)[None, :, None, None]
    return y


# ------------------------------------------------------------------- pins ---
def pin_output_size(lib):
    """Every output size the pages print (misprints corrected by their own formula)."""
    for size, k, s, p, d, expected, src in read_output_size_cases():
        if expected < 0:
            try:
                got = oracle.out_size(size, k, s, p, d, lib=lib)
            except ValueError:
                continue
            raise AssertionError(f"{src}: expected rejection, got {got}")
        got = oracle.out_size(size, k, s, p, d, lib=lib)
        assert got == expected, f"{src}: out_size({size},{k},{s},{p},{d}) = {got}, want {expected}"


def pin_worked_example(lib):
    """dpshk §4.1-§4.3: shapes, the printed padded plane, the first window and its sum 12."""
    ex = read_worked_example()
    x = np.arange(75, dtype=np.float64).reshape(ex["input_shape"])
    w = np.ones(ex["weight_shape"])
    stride, pad = ex["stride"][-1], ex["pad"][0]
    y = oracle.conv2d(x, w, None, stride, pad, lib=lib)
    assert list(y.shape) == ex["output_shape"], (y.shape, ex["output_shape"])
    y0 = oracle.conv2d(x[:, 0:1], np.ones((2, 1, 3, 3)), None, stride, pad, lib=lib)
    assert y0[0, 0, 0, 0] == ex["out0_channel0_only"][0], y0[0, 0, 0, 0]
    assert y0[0, 1, 0, 0] == ex["out0_channel0_only"][0]
    # A unit tap at (a, b) with stride 1 and padding 1 copies padded[oh + a, ow + b]:
    # together the nine taps rebuild the whole printed 7x7 padded plane.
    padded = ex["padded_c0"]
    rebuilt = np.full(padded.shape, np.nan)
    for a in range(3):
        for bb in range(3):
            wd = np.zeros((1, 1, 3, 3))
            wd[0, 0, a, bb] = 1.0
            yd = oracle.conv2d(x[:, 0:1], wd, None, 1, pad, lib=lib)[0, 0]
            rebuilt[a:a + 5, bb:bb + 5] = yd
    assert np.array_equal(rebuilt, padded), rebuilt
    # With the page's stride 2, the unit taps read the printed first window.
    for a in range(3):
        for bb in range(3):
            wd = np.zeros((1, 1, 3, 3))
            wd[0, 0, a, bb] = 1.0
            yd = oracle.conv2d(x[:, 0:1], wd, None, stride, pad, lib=lib)
            assert yd[0, 0, 0, 0] == ex["window_c0"][a, bb], (a, bb, yd[0, 0, 0, 0])


def read_hand_example():
    """Rows of hand_example_5x5_pad1.txt: the 5x5 output worked by hand."""
    rows = []
    with open(os.path.join(GOLDEN, "hand_example_5x5_pad1.txt"), encoding="utf-8") as f:
        for line in f:
            parts = line.split()
            if parts and parts[0] == "out":
                rows.append([float(v) for v in parts[1:]])
    return np.array(rows)


def pin_hand_example_5x5(lib):
    """lpnh §1.1's hand-drawn case: 5x5 arange input, 3x3 ones, stride 1, pad 1 -- the
    25 window sums worked by hand (tests/golden/hand_example_5x5_pad1.txt)."""
    want = read_hand_example()
    assert want.shape == (5, 5)
    x = np.arange(25, dtype=np.float64).reshape(1, 1, 5, 5)
    y = oracle.conv2d(x, np.ones((1, 1, 3, 3)), None, 1, 1, 1, 1, lib=lib)
    assert y.shape == (1, 1, 5, 5)
    assert np.array_equal(y[0, 0], want), y[0, 0]


def pin_box_sum(lib):
    """All-ones kernels equal integral-image box sums (incl. the 3-channel worked example)."""
    rng = np.random.default_rng(11)
    cases = [  # N, C, H, W, Co, Kh, Kw, s, p, g
        (1, 3, 5, 5, 2, 3, 3, 2, 1, 1),
        (2, 4, 9, 7, 6, 3, 2, 1, 1, 2),
        (1, 2, 11, 13, 2, 5, 3, 3, 2, 1),
        (2, 6, 8, 8, 4, 1, 4, 2, 0, 2),
        (1, 1, 1, 1, 1, 3, 3, 2, 1, 1),
    ]
    for i, (N, C, H, W, Co, Kh, Kw, s, p, g) in enumerate(cases):
        x = np.arange(N * C * H * W, dtype=np.float64).reshape(N, C, H, W) if i == 0 \
            else rng.standard_normal((N, C, H, W))
        b = rng.standard_normal(Co)
        w = np.ones((Co, C // g, Kh, Kw))
        got = oracle.conv2d(x, w, b, s, p, 1, g, lib=lib)
        want = box_sum_conv(x, Co, Kh, Kw, s, p, g, b)
        assert got.shape == want.shape, (got.shape, want.shape)
        assert np.allclose(got, want, rtol=1e-13, atol=1e-11), (i, np.abs(got - want).max())


BRUTE_CASES = [  # N, C, H, W, Co, Kh, Kw, s, p, d, g, bias
    (2, 3, 9, 11, 4, 3, 3, 2, 1, 1, 1, True),     # lpnh §3.2 test shape
    (2, 3, 9, 11, 4, 3, 3, 1, 0, 1, 1, False),    # lpnh §6.2: stride 1 / pad 0 ...
    (2, 3, 9, 11, 4, 3, 3, 2, 1, 1, 1, False),    # ... and stride 2 / pad 1
    (1, 4, 10, 8, 6, 3, 3, 1, 2, 2, 2, True),     # dilation + groups
    (2, 8, 12, 9, 8, 3, 5, 3, 3, 1, 4, True),     # non-square kernel, stride 3
    (1, 2, 7, 13, 3, 7, 3, 1, 3, 1, 1, True),     # 7-tall kernel
    (1, 6, 15, 15, 6, 3, 3, 2, 2, 2, 3, True),    # stride + pad + dilation + groups (config-5a shape, small)
    (3, 5, 6, 5, 2, 1, 1, 1, 0, 1, 1, True),      # 1x1
    (1, 4, 8, 8, 4, 2, 2, 2, 0, 3, 4, True),      # depthwise-style groups == C
    (1, 3, 17, 17, 5, 7, 7, 1, 3, 1, 1, True),    # 7x7 on 17x17 (config-5b shape, small)
]


def _rand_case(rng, case):
    N, C, H, W, Co, Kh, Kw, s, p, d, g, has_b = case
    x = rng.standard_normal((N, C, H, W))
    w = rng.standard_normal((Co, C // g, Kh, Kw))
    b = rng.standard_normal(Co) if has_b else None
    return x, w, b, s, p, d, g


def pin_brute_force(lib):
    """Explicit pad + im2col + matrix product agrees to ~1e-13 on random shapes."""
    rng = np.random.default_rng(12)
    for case in BRUTE_CASES:
        x, w, b, s, p, d, g = _rand_case(rng, case)
        got = oracle.conv2d(x, w, b, s, p, d, g, lib=lib)
        want = im2col_conv(x, w, b, s, p, d, g)
        assert got.shape == want.shape, (case, got.shape, want.shape)
        err = np.abs(got - want).max() / max(1.0, np.abs(want).max())
        assert err < 1e-13, (case, err)


def pin_torch_f64(lib):
    """PyTorch's CPU convolution in float64 agrees on the same random shapes."""
    import torch
    import torch.nn.functional as F
    rng = np.random.default_rng(13)
    for case in BRUTE_CASES:
        x, w, b, s, p, d, g = _rand_case(rng, case)
        got = oracle.conv2d(x, w, b, s, p, d, g, lib=lib)
        want = F.conv2d(torch.from_numpy(x), torch.from_numpy(w),
                        None if b is None else torch.from_numpy(b),
                        stride=s, padding=p, dilation=d, groups=g).numpy()
        assert got.shape == want.shape, (case, got.shape, want.shape)
        err = np.abs(got - want).max() / max(1.0, np.abs(want).max())
        assert err < 1e-12, (case, err)


def pin_pointwise_matmul(lib):
    """A 1x1 convolution is a channel matrix product at every pixel (zskr §4.2, pwwt §1.2)."""
    rng = np.random.default_rng(14)
    x = rng.standard_normal((2, 16, 5, 7))
    w = rng.standard_normal((24, 16, 1, 1))
    b = rng.standard_normal(24)
    got = oracle.conv2d(x, w, b, 1, 0, lib=lib)
    want = np.einsum("oc,nchw->nohw", w[:, :, 0, 0], x) + b[None, :, None, None]
    assert np.allclose(got, want, rtol=1e-13, atol=1e-12), np.abs(got - want).max()
    # and with stride 2 it is the same product on the subsampled pixels
    got2 = oracle.conv2d(x, w, b, 2, 0, lib=lib)
    assert np.allclose(got2, want[:, :, ::2, ::2], rtol=1e-13, atol=1e-12)


def pin_delta_shift(lib):
    """A unit tap at (a, b) copies x[c, oh*s + a*d - p, ow*s + b*d - p], zero outside."""
    rng = np.random.default_rng(15)
    N, C, H, W = 2, 3, 9, 8
    x = rng.standard_normal((N, C, H, W))
    for (Kh, Kw, s, p, d) in [(3, 3, 1, 1, 1), (3, 5, 2, 2, 1), (3, 3, 2, 2, 2), (5, 2, 3, 4, 2)]:
        Ho, Wo = _out(H, Kh, s, p, d), _out(W, Kw, s, p, d)
        for a in range(Kh):
            for bb in range(Kw):
                w = np.zeros((C, C, Kh, Kw))
                for c in range(C):
                    w[c, c, a, bb] = 1.0
                got = oracle.conv2d(x, w, None, s, p, d, lib=lib)
                want = np.zeros((N, C, Ho, Wo))
                for oh in range(Ho):
                    ih = oh * s + a * d - p
                    if not 0 <= ih < H:
                        continue
                    for ow in range(Wo):
                        iw = ow * s + bb * d - p
                        if 0 <= iw < W:
                            want[:, :, oh, ow] = x[:, :, ih, iw]
                assert np.array_equal(got, want), (Kh, Kw, s, p, d, a, bb)


def pin_zero_weight(lib):
    """With w = 0 the output is the bias at every pixel."""
    rng = np.random.default_rng(16)
    x = rng.standard_normal((2, 4, 7, 6))
    b = rng.standard_normal(6)
    y = oracle.conv2d(x, np.zeros((6, 2, 3, 3)), b, 2, 1, 1, 2, lib=lib)
    assert np.array_equal(y, np.broadcast_to(b[None, :, None, None], y.shape))


def pin_linearity(lib):
    """Without bias the output is linear in x and in w."""
    rng = np.random.default_rng(17)
    x1, x2 = rng.standard_normal((2, 2, 4, 8, 7))
    w1, w2 = rng.standard_normal((2, 6, 2, 3, 3))
    al, be = 0.75, -1.5
    f = lambda x, w: oracle.conv2d(x, w, None, 2, 1, 2, 2, lib=lib)
    assert np.allclose(f(al * x1 + be * x2, w1), al * f(x1, w1) + be * f(x2, w1), rtol=1e-12, atol=1e-12)
    assert np.allclose(f(x1, al * w1 + be * w2), al * f(x1, w1) + be * f(x1, w2), rtol=1e-12, atol=1e-12)


def pin_groups_split(lib):
    """groups = g is g separate convolutions on channel slices (pwwt §4.3, dpshk §3.4)."""
    rng = np.random.default_rng(18)
    g, C, Co = 4, 8, 12
    x = rng.standard_normal((2, C, 9, 9))
    w = rng.standard_normal((Co, C // g, 3, 3))
    b = rng.standard_normal(Co)
    got = oracle.conv2d(x, w, b, 2, 2, 2, g, lib=lib)
    cg, og = C // g, Co // g
    for gi in range(g):
        part = oracle.conv2d(x[:, gi * cg:(gi + 1) * cg], w[gi * og:(gi + 1) * og],
                             b[gi * og:(gi + 1) * og], 2, 2, 2, 1, lib=lib)
        assert np.allclose(got[:, gi * og:(gi + 1) * og], part, rtol=1e-13, atol=1e-13), gi


def pin_exact_integers(lib):
    """Small-integer inputs: the double result equals exact integer arithmetic."""
    rng = np.random.default_rng(19)
    for case in BRUTE_CASES[:6]:
        N, C, H, W, Co, Kh, Kw, s, p, d, g, has_b = case
        x = rng.integers(-2, 3, (N, C, H, W))
        w = rng.integers(-2, 3, (Co, C // g, Kh, Kw))
        b = rng.integers(-2, 3, Co) if has_b else None
        got = oracle.conv2d(x, w, b, s, p, d, g, lib=lib)
        want = im2col_conv(x, w, b, s, p, d, g, dtype=np.int64)
        assert np.array_equal(got, want.astype(np.float64)), case


def pin_single_pixel(lib):
    """lpnh §6.1: a 1x1 input, 3x3 kernel, stride 2, pad 1 touches only the centre tap."""
    w = np.arange(1.0, 10.0).reshape(1, 1, 3, 3)
    y = oracle.conv2d(np.array([[[[3.0]]]]), w, np.array([0.5]), 2, 1, lib=lib)
    assert y.shape == (1, 1, 1, 1) and y[0, 0, 0, 0] == 0.5 + 3.0 * w[0, 0, 1, 1], y


def pin_points_match_full(lib):
    """Sampled single outputs equal the same entries of the full output."""
    rng = np.random.default_rng(20)
    x, w, b, s, p, d, g = _rand_case(rng, BRUTE_CASES[3])
    y = oracle.conv2d(x, w, b, s, p, d, g, lib=lib)
    idx = np.stack([rng.integers(0, n, 50) for n in y.shape], axis=1)
    pts = oracle.conv2d_points(x, w, b, idx, s, p, d, g, lib=lib)
    assert np.array_equal(pts, y[tuple(idx.T)])


ALL_PINS = [pin_output_size, pin_worked_example, pin_hand_example_5x5, pin_box_sum, pin_brute_force, pin_torch_f64,
            pin_pointwise_matmul, pin_delta_shift, pin_zero_weight, pin_linearity,
            pin_groups_split, pin_exact_integers, pin_single_pixel, pin_points_match_full]
