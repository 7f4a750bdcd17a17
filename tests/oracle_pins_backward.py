"""Pins for the backward oracle (dx, dW, db): checks against facts the pages and the
mathematics fix, each by a route other than the oracle's own loops.

  * the matrix form of the im2col/GEMM tutorial (zskr.cn/news/1820658) §3.3:
    dW_row = dout_col @ X_col^T, db = the sum of dout, dx = col2im(W_row^T @ dout_col),
    with an im2col and a col2im written here in NumPy (strided slices);
  * PyTorch's float64 CPU autograd (a library special case, tiny shapes);
  * the adjoint identity of a linear map: the forward oracle y = conv(x, w) is linear
    in x and in w, so for any g, <x, dx(g)> = <w, dW(g)> = <g, conv(x, w)>;
  * central differences of L = <g, conv(x, w)> through the forward oracle, exact up
    to rounding because L is linear in each entry;
  * the set-up of "手撕 Conv2D" (lpnh.cn/news/2493075) §5.3 (dout all ones), for which
    db, dx and dW have closed forms (counts of covering windows, sums of x over
    shifted rectangles);
  * the point evaluators against the whole-tensor loops.
Every pin takes a backward-oracle library handle and raises AssertionError when the
oracle disagrees.
"""
from __future__ import annotations

import numpy as np

import oracle
import oracle_pins


def _out(size, k, s, p, d):
    return (size + 2 * p - d * (k - 1) - 1) // s + 1


def im2col_cols(x, Kh, Kw, s, p, d):
    """cols[n, c, kh, kw, oh, ow] = padded x at (oh*s + kh*d, ow*s + kw*d) (zskr §2.2)."""
    N, C, H, W = x.shape
    Ho, Wo = _out(H, Kh, s, p, d), _out(W, Kw, s, p, d)
    xp = np.pad(x, ((0, 0), (0, 0), (p, p), (p, p)))
    cols = np.empty((N, C, Kh, Kw, Ho, Wo))
    for i in range(Kh):
        for j in range(Kw):
            cols[:, :, i, j] = xp[:, :, i * d: i * d + s * (Ho - 1) + 1: s, j * d: j * d + s * (Wo - 1) + 1: s]
    return cols


def col2im(cols, x_shape, s, p, d):
    """Inverse scatter of im2col: every column entry is added back onto the padded
    input position it was read from, overlapping windows accumulating (zskr §3.3),
    then the padding is cut off."""
    N, C, H, W = x_shape
    _, _, Kh, Kw, Ho, Wo = cols.shape
    dxp = np.zeros((N, C, H + 2 * p, W + 2 * p))
    for i in range(Kh):
        for j in range(Kw):
            dxp[:, :, i * d: i * d + s * (Ho - 1) + 1: s, j * d: j * d + s * (Wo - 1) + 1: s] += cols[:, :, i, j]
    return dxp[:, :, p: p + H, p: p + W]


def im2col_backward(dy, x, w, s, p, d, g):
    """(dx, dW, db) in the tutorial's matrix form, one product per group."""
    N, C, H, W = x.shape
    Co, Cg, Kh, Kw = w.shape
    Ho, Wo = dy.shape[2], dy.shape[3]
    cols = im2col_cols(x, Kh, Kw, s, p, d)
    cog = Co // g
    dW = np.empty_like(w)
    dcols = np.empty_like(cols)
    for gi in range(g):
        xcol = cols[:, gi * Cg:(gi + 1) * Cg].transpose(1, 2, 3, 0, 4, 5).reshape(Cg * Kh * Kw, N * Ho * Wo)
        dout_col = dy[:, gi * cog:(gi + 1) * cog].transpose(1, 0, 2, 3).reshape(cog, N * Ho * Wo)
        wrow = w[gi * cog:(gi + 1) * cog].reshape(cog, Cg * Kh * Kw)
        dW[gi * cog:(gi + 1) * cog] = (dout_col @ xcol.T).reshape(cog, Cg, Kh, Kw)
        dxc = (wrow.T @ dout_col).reshape(Cg, Kh, Kw, N, Ho, Wo).transpose(3, 0, 1, 2, 4, 5)
        dcols[:, gi * Cg:(gi + 1) * Cg] = dxc
    dx = col2im(dcols, x.shape, s, p, d)
    db = dy.sum(axis=(0, 2, 3))
    return dx, dW, db


CASES = [  # N, C, H, W, Co, Kh, Kw, s, p, d, g
    (2, 3, 8, 10, 4, 3, 3, 1, 1, 1, 1),    # lpnh §5.3's shape
    (2, 3, 9, 11, 4, 3, 3, 2, 1, 1, 1),    # stride 2, pad 1 (lpnh §6.2 asks for both)
    (1, 4, 10, 8, 6, 3, 3, 1, 2, 2, 2),    # dilation + groups
    (2, 8, 12, 9, 8, 3, 5, 3, 3, 1, 4),    # non-square kernel, stride 3
    (1, 6, 15, 15, 6, 3, 3, 2, 2, 2, 3),   # stride + pad + dilation + groups
    (3, 5, 6, 5, 2, 1, 1, 1, 0, 1, 1),     # 1x1
    (1, 4, 8, 8, 4, 3, 3, 1, 1, 1, 4),     # depthwise
    (1, 2, 11, 10, 3, 4, 2, 2, 0, 1, 1),   # even kernel, stride 2, rows the windows never reach
]


def _rand(rng, case):
    N, C, H, W, Co, Kh, Kw, s, p, d, g = case
    Ho, Wo = _out(H, Kh, s, p, d), _out(W, Kw, s, p, d)
    x = rng.standard_normal((N, C, H, W))
    w = rng.standard_normal((Co, C // g, Kh, Kw))
    dy = rng.standard_normal((N, Co, Ho, Wo))
    return dy, x, w, s, p, d, g


def pin_bwd_im2col_matrix_form(lib):
    """zskr §3.3's matrix form agrees to ~1e-13 on random shapes."""
    rng = np.random.default_rng(21)
    for case in CASES:
        dy, x, w, s, p, d, g = _rand(rng, case)
        got = oracle.conv2d_backward(dy, x, w, s, p, d, g, lib=lib)
        want = im2col_backward(dy, x, w, s, p, d, g)
        for name, a, b in zip(("dx", "dW", "db"), got, want):
            assert a.shape == b.shape, (case, name)
            err = np.abs(a - b).max() / max(1.0, np.abs(b).max())
            assert err < 1e-13, (case, name, err)


def pin_bwd_torch_f64(lib):
    """PyTorch's float64 CPU autograd of conv2d (library special case)."""
    import torch
    rng = np.random.default_rng(22)
    for case in CASES:
        dy, x, w, s, p, d, g = _rand(rng, case)
        xt = torch.from_numpy(x).requires_grad_(True)
        wt = torch.from_numpy(w).requires_grad_(True)
        bt = torch.zeros(w.shape[0], dtype=torch.float64, requires_grad=True)
        y = torch.nn.functional.conv2d(xt, wt, bt, stride=s, padding=p, dilation=d, groups=g)
        y.backward(torch.from_numpy(dy))
        got = oracle.conv2d_backward(dy, x, w, s, p, d, g, lib=lib)
        for name, a, b in zip(("dx", "dW", "db"), got, (xt.grad, wt.grad, bt.grad)):
            b = b.numpy()
            assert np.allclose(a, b, rtol=1e-12, atol=1e-10), (case, name, np.abs(a - b).max())


def pin_bwd_adjoint(lib):
    """<x, dx(g)> = <w, dW(g)> = <g, conv(x, w)> with the (pinned) forward oracle."""
    rng = np.random.default_rng(23)
    for case in CASES:
        dy, x, w, s, p, d, g = _rand(rng, case)
        dx, dW, db = oracle.conv2d_backward(dy, x, w, s, p, d, g, lib=lib)
        L = float((dy * oracle.conv2d(x, w, None, s, p, d, g)).sum())
        scale = max(1.0, abs(L), float(np.abs(dy).sum()))
        assert abs(float((x * dx).sum()) - L) < 1e-11 * scale, (case, "dx")
        assert abs(float((w * dW).sum()) - L) < 1e-11 * scale, (case, "dW")
        # bias enters y once per output position: <1, db> = sum of dout
        assert abs(float(db.sum()) - float(dy.sum())) < 1e-11 * scale, (case, "db")


def pin_bwd_central_difference(lib):
    """dL/dx_i and dL/dw_j by central differences of L = <g, conv(x, w)> through the
    forward oracle, at a handful of entries (exact up to rounding: L is linear)."""
    rng = np.random.default_rng(24)
    for case in CASES[:5]:
        dy, x, w, s, p, d, g = _rand(rng, case)
        dx, dW, _ = oracle.conv2d_backward(dy, x, w, s, p, d, g, lib=lib)

        def L(xv, wv):
            return float((dy * oracle.conv2d(xv, wv, None, s, p, d, g)).sum())

        for _ in range(4):
            i = tuple(int(rng.integers(0, n)) for n in x.shape)
            e = np.zeros_like(x)
            e[i] = 1.0
            fd = (L(x + e, w) - L(x - e, w)) / 2.0
            assert abs(fd - dx[i]) < 1e-10 * max(1.0, abs(fd)), (case, "dx", i)
            j = tuple(int(rng.integers(0, n)) for n in w.shape)
            e = np.zeros_like(w)
            e[j] = 1.0
            fd = (L(x, w + e) - L(x, w - e)) / 2.0
            assert abs(fd - dW[j]) < 1e-10 * max(1.0, abs(fd)), (case, "dW", j)


def pin_bwd_ones_closed_form(lib):
    """lpnh §5.3: N=2, C_in=3, 8x10, C_out=4, 3x3, stride 1, pad 1, dout all ones.
    db[oc] = N*Ho*Wo; with w all ones, dx at (ih, iw) = C_out * (rows of the filter that
    land inside) * (columns that land inside); dW[oc][c][kh][kw] = the sum of x over the
    rectangle the tap (kh, kw) sweeps, clipped to the image (integral image)."""
    rng = np.random.default_rng(25)
    N, C, H, W, Co, K = 2, 3, 8, 10, 4, 3
    x = rng.standard_normal((N, C, H, W))
    w = np.ones((Co, C, K, K))
    dy = np.ones((N, Co, H, W))
    dx, dW, db = oracle.conv2d_backward(dy, x, w, 1, 1, 1, 1, lib=lib)
    assert np.array_equal(db, np.full(Co, float(N * H * W)))
    rows = np.array([sum(1 for kh in range(K) if 0 <= ih + 1 - kh < H) for ih in range(H)])
    cols = np.array([sum(1 for kw in range(K) if 0 <= iw + 1 - kw < W) for iw in range(W)])
    assert np.array_equal(dx, np.broadcast_to(Co * np.outer(rows, cols), dx.shape))
    integ = np.zeros((N, C, H + 1, W + 1))
    integ[:, :, 1:, 1:] = x.cumsum(2).cumsum(3)
    for kh in range(K):
        for kw in range(K):
            r0, r1 = max(0, kh - 1), min(H, kh - 1 + H)
            c0, c1 = max(0, kw - 1), min(W, kw - 1 + W)
            box = (integ[:, :, r1, c1] - integ[:, :, r0, c1] - integ[:, :, r1, c0] + integ[:, :, r0, c0]).sum(0)
            for oc in range(Co):
                assert np.allclose(dW[oc, :, kh, kw], box, rtol=1e-13, atol=1e-12), (kh, kw)


def pin_bwd_points_match_full(lib):
    """The point evaluators agree with the whole-tensor loops."""
    rng = np.random.default_rng(26)
    for case in CASES:
        dy, x, w, s, p, d, g = _rand(rng, case)
        dx, dW, _ = oracle.conv2d_backward(dy, x, w, s, p, d, g, lib=lib)
        ix = np.stack([rng.integers(0, n, 40) for n in x.shape], axis=1)
        iw = np.stack([rng.integers(0, n, 40) for n in w.shape], axis=1)
        gx = oracle.conv2d_backward_data_points(dy, w, x.shape, ix, s, p, d, g, lib=lib)
        gw = oracle.conv2d_backward_weight_points(dy, x, w.shape, iw, s, p, d, g, lib=lib)
        assert np.allclose(gx, dx[tuple(ix.T)], rtol=1e-13, atol=1e-12), case
        assert np.allclose(gw, dW[tuple(iw.T)], rtol=1e-13, atol=1e-12), case


def pin_bwd_exact_integers(lib):
    """Small-integer inputs: every sum is exact, so the matrix form matches bit for bit."""
    rng = np.random.default_rng(27)
    for case in CASES:
        N, C, H, W, Co, Kh, Kw, s, p, d, g = case
        Ho, Wo = _out(H, Kh, s, p, d), _out(W, Kw, s, p, d)
        x = rng.integers(-3, 4, (N, C, H, W)).astype(np.float64)
        w = rng.integers(-3, 4, (Co, C // g, Kh, Kw)).astype(np.float64)
        dy = rng.integers(-3, 4, (N, Co, Ho, Wo)).astype(np.float64)
        got = oracle.conv2d_backward(dy, x, w, s, p, d, g, lib=lib)
        want = im2col_backward(dy, x, w, s, p, d, g)
        for a, b in zip(got, want):
            assert np.array_equal(a, b), case


ALL_PINS = [pin_bwd_im2col_matrix_form, pin_bwd_torch_f64, pin_bwd_adjoint, pin_bwd_central_difference,
            pin_bwd_ones_closed_form, pin_bwd_points_match_full, pin_bwd_exact_integers]

# the forward oracle the adjoint and difference pins lean on is pinned on its own
assert oracle_pins.ALL_PINS
