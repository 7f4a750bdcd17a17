"""CPU oracle for the 2-D convolution forward pass -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The CUDA library and its Python binding
never import it; the two share no code.

The arithmetic lives in C files compiled with gcc (no -ffast-math, so IEEE double
arithmetic is kept) and exposed through ctypes:
  * ``conv2d_oracle.c``: the forward pass, six nested loops with bounds-checked zero
    padding, after the "手撕 Conv2D" page (lpnh.cn/news/2493075) §1.1-§2.1;
  * ``conv2d_backward_oracle.c``: the gradients dx, dW, db, after the same page's
    §5.1-§5.2 naive backward loops;
  * ``conv3d_oracle.c``: the 3-D forward pass of "PyTorch高维张量乘法与conv2d/conv3d
    维度语义解析" §5.1, the same loops with a depth dimension.
Inputs are widened to float64 before the call; widening bf16- or fp32-valued data
is exact.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
SOURCE = os.path.join(_HERE, "conv2d_oracle.c")
LIBRARY = os.path.join(_HERE, "liboracle.so")
BWD_SOURCE = os.path.join(_HERE, "conv2d_backward_oracle.c")
BWD_LIBRARY = os.path.join(_HERE, "liboracle_backward.so")
C3D_SOURCE = os.path.join(_HERE, "conv3d_oracle.c")
C3D_LIBRARY = os.path.join(_HERE, "liboracle_conv3d.so")

_lib = None
_bwd = None
_c3d = None


def build(source: str = SOURCE, output: str = LIBRARY, extra_flags=()) -> str:
    """Compile ``source`` into the shared library ``output`` and return its path."""
    cmd = ["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11", *extra_flags,
           "-o", output, source]
    subprocess.run(cmd, check=True)
    return output


def build_all() -> None:
    """Compile every C oracle of this package."""
    build(SOURCE, LIBRARY)
    build(BWD_SOURCE, BWD_LIBRARY)
    build(C3D_SOURCE, C3D_LIBRARY)


def load(path: str | None = None):
    """Load (building first if needed) the oracle library; returns a ctypes handle."""
    global _lib
    if path is not None:
        return _bind(ctypes.CDLL(path))
    if _lib is None:
        if (not os.path.exists(LIBRARY)
                or os.path.getmtime(LIBRARY) < os.path.getmtime(SOURCE)):
            build()
        _lib = _bind(ctypes.CDLL(LIBRARY))
    return _lib


def _bind(lib):
    L = ctypes.c_long
    P = ctypes.c_void_p
    lib.oracle_conv2d_out_size.argtypes = [L, L, L, L, L, ctypes.POINTER(L)]
    lib.oracle_conv2d_out_size.restype = ctypes.c_int
    lib.oracle_conv2d_nchw.argtypes = [P, P, P, P] + [L] * 11
    lib.oracle_conv2d_nchw.restype = ctypes.c_int
    lib.oracle_conv2d_points.argtypes = [P, P, P] + [L] * 11 + [P, L, P]
    lib.oracle_conv2d_points.restype = ctypes.c_int
    lib.oracle_num_threads.argtypes = []
    lib.oracle_num_threads.restype = ctypes.c_int
    return lib


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _f64(a):
    return None if a is None else np.ascontiguousarray(a, dtype=np.float64)


def out_size(size, k, stride=1, pad=0, dilation=1, lib=None):
    """Output extent along one dimension; raises ValueError when it is below 1."""
    lib = lib or load()
    out = ctypes.c_long(0)
    if lib.oracle_conv2d_out_size(size, k, stride, pad, dilation, ctypes.byref(out)) != 0:
        raise ValueError(f"no valid output for in={size} k={k} s={stride} p={pad} d={dilation}")
    return out.value


def conv2d(x, w, bias=None, stride=1, pad=0, dilation=1, groups=1, lib=None):
    """y = conv2d(x, w, bias) in float64; x NCHW, w OIHW (C_out, C_in/groups, Kh, Kw)."""
    lib = lib or load()
    x, w, bias = _f64(x), _f64(w), _f64(bias)
    N, C_in, H, W = x.shape
    C_out, cin_g, Kh, Kw = w.shape
    if cin_g * groups != C_in:
        raise ValueError("weight shape does not match C_in / groups")
    if bias is not None and bias.shape != (C_out,):
        raise ValueError("bias must have shape (C_out,)")
    Ho = out_size(H, Kh, stride, pad, dilation, lib)
    Wo = out_size(W, Kw, stride, pad, dilation, lib)
    y = np.empty((N, C_out, Ho, Wo), dtype=np.float64)
    rc = lib.oracle_conv2d_nchw(_ptr(x), _ptr(w), _ptr(bias), _ptr(y), N, C_in, H, W,
                                C_out, Kh, Kw, stride, pad, dilation, groups)
    if rc != 0:
        raise ValueError("oracle rejected the shape")
    return y


def conv2d_points(x, w, bias, idx, stride=1, pad=0, dilation=1, groups=1, lib=None):
    """Selected outputs y[n, oc, oh, ow] for the rows (n, oc, oh, ow) of ``idx``."""
    lib = lib or load()
    x, w, bias = _f64(x), _f64(w), _f64(bias)
    idx = np.ascontiguousarray(idx, dtype=np.int64).reshape(-1, 4)
    N, C_in, H, W = x.shape
    C_out, _, Kh, Kw = w.shape
    out = np.empty(idx.shape[0], dtype=np.float64)
    rc = lib.oracle_conv2d_points(_ptr(x), _ptr(w), _ptr(bias), N, C_in, H, W, C_out,
                                  Kh, Kw, stride, pad, dilation, groups, _ptr(idx),
                                  idx.shape[0], _ptr(out))
    if rc != 0:
        raise ValueError("oracle rejected the shape or an index")
    return out


def num_threads(lib=None) -> int:
    """OpenMP threads the oracle's loops use."""
    return int((lib or load()).oracle_num_threads())


# ---------------------------------------------------------------- backward ---
def _bind_backward(lib):
    L = ctypes.c_long
    P = ctypes.c_void_p
    lib.oracle_conv2d_backward.argtypes = [P] * 6 + [L] * 11
    lib.oracle_conv2d_backward.restype = ctypes.c_int
    lib.oracle_conv2d_backward_data_points.argtypes = [P, P] + [L] * 11 + [P, L, P]
    lib.oracle_conv2d_backward_data_points.restype = ctypes.c_int
    lib.oracle_conv2d_backward_weight_points.argtypes = [P, P] + [L] * 11 + [P, L, P]
    lib.oracle_conv2d_backward_weight_points.restype = ctypes.c_int
    lib.oracle_backward_num_threads.argtypes = []
    lib.oracle_backward_num_threads.restype = ctypes.c_int
    return lib


def load_backward(path: str | None = None):
    """Load (building first if needed) the backward oracle library."""
    global _bwd
    if path is not None:
        return _bind_backward(ctypes.CDLL(path))
    if _bwd is None:
        if (not os.path.exists(BWD_LIBRARY)
                or os.path.getmtime(BWD_LIBRARY) < os.path.getmtime(BWD_SOURCE)):
            build(BWD_SOURCE, BWD_LIBRARY)
        _bwd = _bind_backward(ctypes.CDLL(BWD_LIBRARY))
    return _bwd


def _bwd_shape(dy, x_shape, w):
    N, C_in, H, W = x_shape
    C_out, cin_g, Kh, Kw = w.shape
    if dy.shape[0] != N or dy.shape[1] != C_out:
        raise ValueError("dy does not match x and w")
    groups = C_in // cin_g
    if cin_g * groups != C_in:
        raise ValueError("weight shape does not match C_in / groups")
    return N, C_in, H, W, C_out, Kh, Kw, groups


def conv2d_backward(dy, x, w, stride=1, pad=0, dilation=1, groups=1, lib=None):
    """(dx, dW, db) in float64 for y = conv2d(x, w, b): dy (N, C_out, Ho, Wo) NCHW,
    x NCHW, w OIHW (C_out, C_in/groups, Kh, Kw)."""
    lib = lib or load_backward()
    dy, x, w = _f64(dy), _f64(x), _f64(w)
    N, C_in, H, W, C_out, Kh, Kw, g = _bwd_shape(dy, x.shape, w)
    if g != groups:
        raise ValueError("weight shape does not match C_in / groups")
    Ho = out_size(H, Kh, stride, pad, dilation)
    Wo = out_size(W, Kw, stride, pad, dilation)
    if dy.shape != (N, C_out, Ho, Wo):
        raise ValueError(f"dy must have shape {(N, C_out, Ho, Wo)}")
    dx = np.empty_like(x)
    dW = np.empty_like(w)
    db = np.empty(C_out)
    rc = lib.oracle_conv2d_backward(_ptr(dy), _ptr(x), _ptr(w), _ptr(dx), _ptr(dW), _ptr(db), N, C_in,
                                    H, W, C_out, Kh, Kw, stride, pad, dilation, groups)
    if rc != 0:
        raise ValueError("oracle rejected the shape")
    return dx, dW, db


def conv2d_backward_data_points(dy, w, x_shape, idx, stride=1, pad=0, dilation=1, groups=1, lib=None):
    """Selected dx[n, ic, ih, iw] for the rows (n, ic, ih, iw) of ``idx``."""
    lib = lib or load_backward()
    dy, w = _f64(dy), _f64(w)
    N, C_in, H, W, C_out, Kh, Kw, _ = _bwd_shape(dy, x_shape, w)
    idx = np.ascontiguousarray(idx, dtype=np.int64).reshape(-1, 4)
    out = np.empty(idx.shape[0])
    rc = lib.oracle_conv2d_backward_data_points(_ptr(dy), _ptr(w), N, C_in, H, W, C_out, Kh, Kw, stride,
                                                pad, dilation, groups, _ptr(idx), idx.shape[0], _ptr(out))
    if rc != 0:
        raise ValueError("oracle rejected the shape or an index")
    return out


def conv2d_backward_weight_points(dy, x, w_shape, idx, stride=1, pad=0, dilation=1, groups=1, lib=None):
    """Selected dW[oc, c, kh, kw] for the rows (oc, c, kh, kw) of ``idx``."""
    lib = lib or load_backward()
    dy, x = _f64(dy), _f64(x)
    N, C_in, H, W = x.shape
    C_out, cin_g, Kh, Kw = w_shape
    idx = np.ascontiguousarray(idx, dtype=np.int64).reshape(-1, 4)
    out = np.empty(idx.shape[0])
    rc = lib.oracle_conv2d_backward_weight_points(_ptr(dy), _ptr(x), N, C_in, H, W, C_out, Kh, Kw, stride,
                                                  pad, dilation, groups, _ptr(idx), idx.shape[0], _ptr(out))
    if rc != 0:
        raise ValueError("oracle rejected the shape or an index")
    return out


# ------------------------------------------------------------------ conv3d ---
def _bind_conv3d(lib):
    L = ctypes.c_long
    P = ctypes.c_void_p
    lib.oracle_conv3d.argtypes = [P, P, P, P] + [L] * 13
    lib.oracle_conv3d.restype = ctypes.c_int
    lib.oracle_conv3d_points.argtypes = [P, P, P] + [L] * 13 + [P, L, P]
    lib.oracle_conv3d_points.restype = ctypes.c_int
    return lib


def load_conv3d(path: str | None = None):
    """Load (building first if needed) the conv3d oracle library."""
    global _c3d
    if path is not None:
        return _bind_conv3d(ctypes.CDLL(path))
    if _c3d is None:
        if (not os.path.exists(C3D_LIBRARY)
                or os.path.getmtime(C3D_LIBRARY) < os.path.getmtime(C3D_SOURCE)):
            build(C3D_SOURCE, C3D_LIBRARY)
        _c3d = _bind_conv3d(ctypes.CDLL(C3D_LIBRARY))
    return _c3d


def conv3d(x, w, bias=None, stride=1, pad=0, dilation=1, groups=1, lib=None):
    """y = conv3d(x, w, bias) in float64; x NCDHW, w OIDHW (C_out, C_in/groups, Kd, Kh, Kw)."""
    lib = lib or load_conv3d()
    x, w, bias = _f64(x), _f64(w), _f64(bias)
    N, C_in, D, H, W = x.shape
    C_out, cin_g, Kd, Kh, Kw = w.shape
    if cin_g * groups != C_in:
        raise ValueError("weight shape does not match C_in / groups")
    if bias is not None and bias.shape != (C_out,):
        raise ValueError("bias must have shape (C_out,)")
    Do, Ho, Wo = (out_size(v, k, stride, pad, dilation) for v, k in ((D, Kd), (H, Kh), (W, Kw)))
    y = np.empty((N, C_out, Do, Ho, Wo), dtype=np.float64)
    rc = lib.oracle_conv3d(_ptr(x), _ptr(w), _ptr(bias), _ptr(y), N, C_in, D, H, W, C_out, Kd, Kh, Kw, stride,
                           pad, dilation, groups)
    if rc != 0:
        raise ValueError("oracle rejected the shape")
    return y


def conv3d_points(x, w, bias, idx, stride=1, pad=0, dilation=1, groups=1, lib=None):
    """Selected outputs y[n, oc, od, oh, ow] for the rows of ``idx``."""
    lib = lib or load_conv3d()
    x, w, bias = _f64(x), _f64(w), _f64(bias)
    idx = np.ascontiguousarray(idx, dtype=np.int64).reshape(-1, 5)
    N, C_in, D, H, W = x.shape
    C_out, _, Kd, Kh, Kw = w.shape
    out = np.empty(idx.shape[0])
    rc = lib.oracle_conv3d_points(_ptr(x), _ptr(w), _ptr(bias), N, C_in, D, H, W, C_out, Kd, Kh, Kw, stride, pad,
                                  dilation, groups, _ptr(idx), idx.shape[0], _ptr(out))
    if rc != 0:
        raise ValueError("oracle rejected the shape or an index")
    return out
