"""B200-native 2-D convolution forward: a thin Python binding of libconv2d_b200.so.

The functions below carry the names of the C ABI in ``include/conv2d_b200.h`` and
only marshal arguments: torch tensors become device pointers, the current CUDA
stream becomes the stream argument, and a non-OK status becomes
``Conv2dError``.  Every step of the convolution runs in the library's CUDA
kernels; there is no CPU or PyTorch fallback, and a missing library is an error.

``Conv2dB200`` is a small convenience that packs the weights once and owns the
scratch buffer, so that a call is ``y = conv(x)``.
"""
from __future__ import annotations

import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIBRARY = os.path.join(_HERE, "libconv2d_b200.so")

CONV_OK = 0
CONV_ERR_INVALID_ARG = 1
CONV_ERR_UNSUPPORTED = 2
CONV_ERR_CUDA = 3
CONV_ERR_TIMEOUT = 4
CONV_ERR_WORKSPACE = 5
STATUS_NAMES = {0: "OK", 1: "INVALID_ARG", 2: "UNSUPPORTED", 3: "CUDA", 4: "TIMEOUT", 5: "WORKSPACE"}

CONV_F32 = 0
CONV_BF16 = 1
CONV_NHWC = 0
CONV_NCHW = 1

# Every symbol the header declares, with its ctypes signature.
_I, _P, _S, _L = ctypes.c_int, ctypes.c_void_p, ctypes.c_size_t, ctypes.c_longlong
_SHAPE = [_I] * 11
SIGNATURES = {
    "conv2d_output_size": ([_I, _I, _I, _I, _I, ctypes.POINTER(_I)], _I),
    "conv2d_packed_weight_size": ([_I, _I, _I, _I, _I, _I, ctypes.POINTER(_S)], _I),
    "conv2d_pack_weight": ([_P, _P, _I, _I, _I, _I, _I, _I, _P], _I),
    "conv2d_workspace_size": (_SHAPE + [_I, _I, ctypes.POINTER(_S)], _I),
    "conv2d_forward": ([_P, _P, _P, _P] + _SHAPE + [_I, _I, _P, _S, _P], _I),
    "conv2d_im2col_workspace_size": (_SHAPE + [_I, _I, ctypes.POINTER(_S)], _I),
    "conv2d_forward_im2col_gemm": ([_P, _P, _P, _P] + _SHAPE + [_I, _I, _P, _S, _P], _I),
    "conv2d_forward_hostio": ([_P, _P, _P, _P, _P, _P] + _SHAPE + [_I, _I, _P, _S, _P], _I),
    "conv2d_forward_noalloc": ([_P, _P, _P, _P] + _SHAPE + [_I, _I, _P], _I),
    "conv2d_nchw_to_nhwc": ([_P, _P, _I, _I, _I, _I, _I, _I, _I, _P], _I),
    "conv2d_nhwc_to_nchw": ([_P, _P, _I, _I, _I, _I, _I, _P], _I),
    "conv2d_sync_status": ([_P], _I),
    "conv2d_last_error": ([], ctypes.c_char_p),
    "conv2d_set_main_kernel_events": ([_P, _P], _I),
    "conv2d_kernel_launch_count": ([ctypes.POINTER(ctypes.c_ulonglong)], _I),
    "conv2d_debug_set_watchdog": ([_L, _I], _I),
    "conv2d_debug_set_pair_mode": ([_I], _I),
    "conv2d_describe_plan": ([_I] * 11 + [_I, _I, _I, _I, ctypes.c_char_p, ctypes.c_size_t], _I),
    "conv2d_packed_weight_backward_data_size": ([_I, _I, _I, _I, _I, _I, ctypes.POINTER(_S)], _I),
    "conv2d_pack_weight_backward_data": ([_P, _P, _I, _I, _I, _I, _I, _I, _P], _I),
    "conv2d_backward_data_workspace_size": (_SHAPE + [_I, _I, ctypes.POINTER(_S)], _I),
    "conv2d_backward_data": ([_P, _P, _P] + _SHAPE + [_I, _I, _P, _S, _P], _I),
    "conv2d_backward_weight_workspace_size": (_SHAPE + [_I, _I, _I, ctypes.POINTER(_S)], _I),
    "conv2d_backward_weight": ([_P, _P, _P, _P] + _SHAPE + [_I, _I, _P, _S, _P], _I),
    "conv2d_backward_bias_workspace_size": ([_I, _I, _I, _I, _I, ctypes.POINTER(_S)], _I),
    "conv2d_backward_bias": ([_P, _P, _I, _I, _I, _I, _I, _I, _P, _S, _P], _I),
    "conv3d_packed_weight_size": ([_I] * 7 + [ctypes.POINTER(_S)], _I),
    "conv3d_pack_weight": ([_P, _P] + [_I] * 7 + [_P], _I),
    "conv3d_workspace_size": ([_I] * 13 + [_I, _I, ctypes.POINTER(_S)], _I),
    "conv3d_forward": ([_P, _P, _P, _P] + [_I] * 13 + [_I, _I, _P, _S, _P], _I),
    "conv3d_describe_plan": ([_I] * 13 + [_I, _I, _I, ctypes.c_char_p, ctypes.c_size_t], _I),
    "conv2d_winograd_packed_weight_size": ([_I, _I, _I, _I, ctypes.POINTER(_S)], _I),
    "conv2d_pack_weight_winograd": ([_P, _P, _I, _I, _I, _I, _P], _I),
    "conv2d_winograd_workspace_size": ([_I] * 7 + [_I, _I, ctypes.POINTER(_S)], _I),
    "conv2d_forward_winograd": ([_P, _P, _P, _P] + [_I] * 7 + [_I, _I, _P, _S, _P], _I),
    "conv2d_winograd_describe_plan": ([_I] * 7 + [_I, _I, _I, ctypes.c_char_p, ctypes.c_size_t], _I),
}

_lib = None


class Conv2dError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(f"{STATUS_NAMES.get(status, status)}: {message}")
        self.status = status


def load():
    """The ctypes handle of libconv2d_b200.so; raises if the library was not built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIBRARY):
            raise RuntimeError(
                f"{LIBRARY} is missing: build it with `python -m cnn_convolution_conv2d_b200.build` "
                "(there is no fallback implementation)")
        lib = ctypes.CDLL(LIBRARY)
        for name, (args, res) in SIGNATURES.items():
            fn = getattr(lib, name)
            fn.argtypes = args
            fn.restype = res
        _lib = lib
    return _lib


def _check(status: int):
    if status != CONV_OK:
        raise Conv2dError(status, load().conv2d_last_error().decode(errors="replace"))


def _dtype_code(t) -> int:
    import torch
    if t == torch.bfloat16:
        return CONV_BF16
    if t == torch.float32:
        return CONV_F32
    raise TypeError(f"unsupported dtype {t}; use torch.bfloat16 or torch.float32")


def _ptr(t):
    if t is None:
        return None
    if isinstance(t, int):
        return t
    if not t.is_cuda or not t.is_contiguous():
        raise ValueError("tensors passed to the library must be contiguous CUDA tensors")
    return t.data_ptr()


def _stream(stream):
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    return stream if isinstance(stream, int) else stream.cuda_stream


def _layout_code(layout) -> int:
    if layout in (CONV_NHWC, "nhwc"):
        return CONV_NHWC
    if layout in (CONV_NCHW, "nchw"):
        return CONV_NCHW
    raise ValueError(f"unknown layout {layout!r}")


# ------------------------------------------------------- same-name wrappers ---
def conv2d_output_size(size: int, k: int, stride: int = 1, pad: int = 0, dilation: int = 1) -> int:
    out = ctypes.c_int(0)
    _check(load().conv2d_output_size(size, k, stride, pad, dilation, ctypes.byref(out)))
    return out.value


def conv2d_packed_weight_size(C_out, C_in, Kh, Kw, groups, dtype) -> int:
    out = ctypes.c_size_t(0)
    _check(load().conv2d_packed_weight_size(C_out, C_in, Kh, Kw, groups, dtype, ctypes.byref(out)))
    return out.value


def conv2d_pack_weight(w_oihw, groups: int = 1, w_packed=None, stream=None):
    """Packs an OIHW weight tensor; returns the packed tensor (allocated if not given)."""
    import torch
    C_out, cin_g, Kh, Kw = w_oihw.shape
    code = _dtype_code(w_oihw.dtype)
    nbytes = conv2d_packed_weight_size(C_out, cin_g * groups, Kh, Kw, groups, code)
    if w_packed is None:
        w_packed = torch.empty(nbytes // w_oihw.element_size(), dtype=w_oihw.dtype, device=w_oihw.device)
    _check(load().conv2d_pack_weight(_ptr(w_oihw), _ptr(w_packed), C_out, cin_g * groups, Kh, Kw,
                                     groups, code, _stream(stream)))
    return w_packed


def conv2d_workspace_size(N, C_in, H, W, C_out, Kh, Kw, stride, pad, dilation, groups, dtype,
                          layout) -> int:
    out = ctypes.c_size_t(0)
    _check(load().conv2d_workspace_size(N, C_in, H, W, C_out, Kh, Kw, stride, pad, dilation, groups,
                                        dtype, _layout_code(layout), ctypes.byref(out)))
    return out.value


def conv2d_im2col_workspace_size(N, C_in, H, W, C_out, Kh, Kw, stride, pad, dilation, groups, dtype,
                                 layout) -> int:
    out = ctypes.c_size_t(0)
    _check(load().conv2d_im2col_workspace_size(N, C_in, H, W, C_out, Kh, Kw, stride, pad, dilation,
                                               groups, dtype, _layout_code(layout), ctypes.byref(out)))
    return out.value


def _ws(workspace):
    if workspace is None:
        return None, 0
    if isinstance(workspace, tuple):  # (pointer, bytes)
        return workspace
    return _ptr(workspace), workspace.numel() * workspace.element_size()


def conv2d_forward(x, w_packed, bias, y, N, C_in, H, W, C_out, Kh, Kw, stride, pad, dilation,
                   groups, dtype, layout, workspace=None, stream=None):
    wp, wb = _ws(workspace)
    _check(load().conv2d_forward(_ptr(x), _ptr(w_packed), _ptr(bias), _ptr(y), N, C_in, H, W, C_out,
                                 Kh, Kw, stride, pad, dilation, groups, dtype, _layout_code(layout),
                                 wp, wb, _stream(stream)))
    return y


def conv2d_forward_im2col_gemm(x, w_packed, bias, y, N, C_in, H, W, C_out, Kh, Kw, stride, pad,
                               dilation, groups, dtype, layout, workspace=None, stream=None):
    wp, wb = _ws(workspace)
    _check(load().conv2d_forward_im2col_gemm(_ptr(x), _ptr(w_packed), _ptr(bias), _ptr(y), N, C_in,
                                             H, W, C_out, Kh, Kw, stride, pad, dilation, groups, dtype,
                                             _layout_code(layout), wp, wb, _stream(stream)))
    return y


NOALLOC_SCRATCH_BYTES = 32 * 1024 * 1024  # CONV2D_NOALLOC_SCRATCH_BYTES


def conv2d_forward_noalloc(x, w_packed, bias, y, N, C_in, H, W, C_out, Kh, Kw, stride, pad, dilation,
                           groups, dtype, layout, stream=None):
    """conv2d_forward without a workspace: for callers that cannot allocate device
    memory; its scratch is the library's built-in NOALLOC_SCRATCH_BYTES array."""
    _check(load().conv2d_forward_noalloc(_ptr(x), _ptr(w_packed), _ptr(bias), _ptr(y), N, C_in, H, W,
                                         C_out, Kh, Kw, stride, pad, dilation, groups, dtype,
                                         _layout_code(layout), _stream(stream)))
    return y


def conv2d_forward_hostio(x_host, y_host, x_dev, y_dev, w_packed, bias, N, C_in, H, W, C_out, Kh,
                          Kw, stride, pad, dilation, groups, dtype, layout, workspace=None,
                          stream=None):
    wp, wb = _ws(workspace)
    _check(load().conv2d_forward_hostio(x_host.data_ptr(), y_host.data_ptr(), _ptr(x_dev), _ptr(y_dev),
                                        _ptr(w_packed), _ptr(bias), N, C_in, H, W, C_out, Kh, Kw,
                                        stride, pad, dilation, groups, dtype, _layout_code(layout),
                                        wp, wb, _stream(stream)))
    return y_host


def conv2d_nchw_to_nhwc(src, dst, N, C, H, W, groups, Cpg, dtype, stream=None):
    _check(load().conv2d_nchw_to_nhwc(_ptr(src), _ptr(dst), N, C, H, W, groups, Cpg, dtype,
                                      _stream(stream)))
    return dst


def conv2d_nhwc_to_nchw(src, dst, N, C, H, W, dtype, stream=None):
    _check(load().conv2d_nhwc_to_nchw(_ptr(src), _ptr(dst), N, C, H, W, dtype, _stream(stream)))
    return dst


def conv2d_sync_status(stream=None):
    """Synchronises the stream and raises Conv2dError if a device watchdog fired."""
    _check(load().conv2d_sync_status(_stream(stream)))


def conv2d_last_error() -> str:
    return load().conv2d_last_error().decode(errors="replace")


def conv2d_set_main_kernel_events(start=None, stop=None):
    """Record torch.cuda.Event `start`/`stop` around each later tensor-core launch (None: off)."""
    def handle(ev):
        return None if ev is None else (ev if isinstance(ev, int) else ev.cuda_event)
    _check(load().conv2d_set_main_kernel_events(handle(start), handle(stop)))


def conv2d_kernel_launch_count() -> int:
    out = ctypes.c_ulonglong(0)
    _check(load().conv2d_kernel_launch_count(ctypes.byref(out)))
    return out.value


def conv2d_debug_set_watchdog(timeout_ns: int = 0, starve_loads: bool = False):
    _check(load().conv2d_debug_set_watchdog(int(timeout_ns), 1 if starve_loads else 0))


def conv2d_describe_plan(N, C_in, H, W, C_out, Kh, Kw, stride, pad, dilation, groups, dtype, layout,
                         explicit_im2col=False, sms=-1) -> dict:
    """The library's plan for a problem (kernel, tile shape, passes) as a dict."""
    import json
    buf = ctypes.create_string_buffer(512)
    _check(load().conv2d_describe_plan(N, C_in, H, W, C_out, Kh, Kw, stride, pad, dilation, groups, dtype,
                                       _layout_code(layout), 1 if explicit_im2col else 0, int(sms), buf,
                                       ctypes.sizeof(buf)))
    return json.loads(buf.value.decode())


def conv3d_describe_plan(N, C_in, D, H, W, C_out, Kd, Kh, Kw, stride, pad, dilation, groups, dtype, layout,
                         sms=-1) -> dict:
    """conv3d_forward's plan for a problem (kernel, tile shape, passes) as a dict."""
    import json
    buf = ctypes.create_string_buffer(512)
    _check(load().conv3d_describe_plan(N, C_in, D, H, W, C_out, Kd, Kh, Kw, stride, pad, dilation, groups, dtype,
                                       _layout_code(layout), int(sms), buf, ctypes.sizeof(buf)))
    return json.loads(buf.value.decode())


def conv2d_winograd_describe_plan(N, C_in, H, W, C_out, pad, m, dtype, layout, sms=-1) -> dict:
    """The plan of conv2d_forward_winograd's channel product as a dict."""
    import json
    buf = ctypes.create_string_buffer(512)
    _check(load().conv2d_winograd_describe_plan(N, C_in, H, W, C_out, pad, m, dtype, _layout_code(layout), int(sms),
                                                buf, ctypes.sizeof(buf)))
    return json.loads(buf.value.decode())


def conv2d_debug_set_pair_mode(mode: int = 0):
    """0: CTA-pair kernel when it pays, 1: whenever eligible, 2: never (test hook)."""
    _check(load().conv2d_debug_set_pair_mode(int(mode)))


# ---------------------------------------------------------------- backward ---
def conv2d_packed_weight_backward_data_size(C_out, C_in, Kh, Kw, groups, dtype) -> int:
    out = ctypes.c_size_t(0)
    _check(load().conv2d_packed_weight_backward_data_size(C_out, C_in, Kh, Kw, groups, dtype, ctypes.byref(out)))
    return out.value


def conv2d_pack_weight_backward_data(w_oihw, groups: int = 1, w_packed_t=None, stream=None):
    """Packs an OIHW weight tensor for conv2d_backward_data (flipped, channels exchanged)."""
    import torch
    C_out, cin_g, Kh, Kw = w_oihw.shape
    code = _dtype_code(w_oihw.dtype)
    nbytes = conv2d_packed_weight_backward_data_size(C_out, cin_g * groups, Kh, Kw, groups, code)
    if w_packed_t is None:
        w_packed_t = torch.empty(nbytes // w_oihw.element_size(), dtype=w_oihw.dtype, device=w_oihw.device)
    _check(load().conv2d_pack_weight_backward_data(_ptr(w_oihw), _ptr(w_packed_t), C_out, cin_g * groups, Kh, Kw,
                                                   groups, code, _stream(stream)))
    return w_packed_t


def conv2d_backward_data_workspace_size(N, C_in, H, W, C_out, Kh, Kw, stride, pad, dilation, groups, dtype,
                                        layout) -> int:
    out = ctypes.c_size_t(0)
    _check(load().conv2d_backward_data_workspace_size(N, C_in, H, W, C_out, Kh, Kw, stride, pad, dilation, groups,
                                                      dtype, _layout_code(layout), ctypes.byref(out)))
    return out.value


def conv2d_backward_data(dy, w_packed_t, dx, N, C_in, H, W, C_out, Kh, Kw, stride, pad, dilation, groups, dtype,
                         layout, workspace=None, stream=None):
    wp, wb = _ws(workspace)
    _check(load().conv2d_backward_data(_ptr(dy), _ptr(w_packed_t), _ptr(dx), N, C_in, H, W, C_out, Kh, Kw, stride,
                                       pad, dilation, groups, dtype, _layout_code(layout), wp, wb, _stream(stream)))
    return dx


def conv2d_backward_weight_workspace_size(N, C_in, H, W, C_out, Kh, Kw, stride, pad, dilation, groups, dtype,
                                          layout, with_bias=False) -> int:
    out = ctypes.c_size_t(0)
    _check(load().conv2d_backward_weight_workspace_size(N, C_in, H, W, C_out, Kh, Kw, stride, pad, dilation, groups,
                                                        dtype, _layout_code(layout), 1 if with_bias else 0,
                                                        ctypes.byref(out)))
    return out.value


def conv2d_backward_weight(x, dy, dw, db, N, C_in, H, W, C_out, Kh, Kw, stride, pad, dilation, groups, dtype,
                           layout, workspace=None, stream=None):
    wp, wb = _ws(workspace)
    _check(load().conv2d_backward_weight(_ptr(x), _ptr(dy), _ptr(dw), _ptr(db), N, C_in, H, W, C_out, Kh, Kw,
                                         stride, pad, dilation, groups, dtype, _layout_code(layout), wp, wb,
                                         _stream(stream)))
    return dw


def conv2d_backward_bias_workspace_size(N, C_out, Ho, Wo, layout) -> int:
    out = ctypes.c_size_t(0)
    _check(load().conv2d_backward_bias_workspace_size(N, C_out, Ho, Wo, _layout_code(layout), ctypes.byref(out)))
    return out.value


def conv2d_backward_bias(dy, db, N, C_out, Ho, Wo, dtype, layout, workspace=None, stream=None):
    wp, wb = _ws(workspace)
    _check(load().conv2d_backward_bias(_ptr(dy), _ptr(db), N, C_out, Ho, Wo, dtype, _layout_code(layout), wp, wb,
                                       _stream(stream)))
    return db


# ---------------------------------------------------------------- Winograd ---
def conv2d_winograd_packed_weight_size(C_out, C_in, m, dtype) -> int:
    out = ctypes.c_size_t(0)
    _check(load().conv2d_winograd_packed_weight_size(C_out, C_in, m, dtype, ctypes.byref(out)))
    return out.value


def conv2d_pack_weight_winograd(w_oihw, m: int = 2, u_packed=None, stream=None):
    """U = G g G^T of an OIHW 3x3 weight for F(m x m, 3 x 3); returns the packed tensor."""
    import torch
    C_out, C_in, Kh, Kw = w_oihw.shape
    if (Kh, Kw) != (3, 3):
        raise ValueError("Winograd F(m x m, 3 x 3) needs a 3x3 filter")
    code = _dtype_code(w_oihw.dtype)
    nbytes = conv2d_winograd_packed_weight_size(C_out, C_in, m, code)
    if u_packed is None:  # raw bytes: the transform type can differ from the weight's
        u_packed = torch.empty(max(nbytes, 16), dtype=torch.uint8, device=w_oihw.device)
    _check(load().conv2d_pack_weight_winograd(_ptr(w_oihw), _ptr(u_packed), C_out, C_in, m, code, _stream(stream)))
    return u_packed


def conv2d_winograd_workspace_size(N, C_in, H, W, C_out, pad, m, dtype, layout) -> int:
    out = ctypes.c_size_t(0)
    _check(load().conv2d_winograd_workspace_size(N, C_in, H, W, C_out, pad, m, dtype, _layout_code(layout),
                                                 ctypes.byref(out)))
    return out.value


def conv2d_forward_winograd(x, u_packed, bias, y, N, C_in, H, W, C_out, pad, m, dtype, layout, workspace=None,
                            stream=None):
    wp, wb = _ws(workspace)
    _check(load().conv2d_forward_winograd(_ptr(x), _ptr(u_packed), _ptr(bias), _ptr(y), N, C_in, H, W, C_out, pad, m,
                                          dtype, _layout_code(layout), wp, wb, _stream(stream)))
    return y


class WinogradConv2dB200:
    """A 3x3, stride-1 convolution layer computed by F(m x m, 3 x 3): transformed
    filters and scratch on the device.  ``w`` is OIHW (C_out, C_in, 3, 3)."""

    def __init__(self, w, bias=None, pad=1, m=2, layout="nhwc"):
        self.C_out, self.C_in = int(w.shape[0]), int(w.shape[1])
        self.pad, self.m = pad, m
        self.layout = _layout_code(layout)
        self.torch_dtype = w.dtype
        self.dtype = _dtype_code(w.dtype)
        self.u_packed = conv2d_pack_weight_winograd(w.contiguous(), m)
        self.bias = None if bias is None else bias.to(w.dtype).contiguous()
        self._ws = {}

    def __call__(self, x, y=None, stream=None):
        import torch
        if self.layout == CONV_NCHW:
            N, C, H, W = (int(v) for v in x.shape)
        else:
            N, H, W, C = (int(v) for v in x.shape)
        Ho = conv2d_output_size(H, 3, 1, self.pad, 1)
        Wo = conv2d_output_size(W, 3, 1, self.pad, 1)
        if y is None:
            shape = (N, self.C_out, Ho, Wo) if self.layout == CONV_NCHW else (N, Ho, Wo, self.C_out)
            y = torch.empty(shape, dtype=self.torch_dtype, device=x.device)
        key = (N, H, W)
        if key not in self._ws:
            nbytes = conv2d_winograd_workspace_size(N, self.C_in, H, W, self.C_out, self.pad, self.m, self.dtype,
                                                    self.layout)
            self._ws[key] = torch.empty(max(nbytes, 16), dtype=torch.uint8, device=x.device)
        conv2d_forward_winograd(x, self.u_packed, self.bias, y, N, self.C_in, H, W, self.C_out, self.pad, self.m,
                                self.dtype, self.layout, self._ws[key], stream)
        return y


# ------------------------------------------------------------------ conv3d ---
def conv3d_packed_weight_size(C_out, C_in, Kd, Kh, Kw, groups, dtype) -> int:
    out = ctypes.c_size_t(0)
    _check(load().conv3d_packed_weight_size(C_out, C_in, Kd, Kh, Kw, groups, dtype, ctypes.byref(out)))
    return out.value


def conv3d_pack_weight(w_oidhw, groups: int = 1, w_packed=None, stream=None):
    """Packs an OIDHW weight tensor; returns the packed tensor (allocated if not given)."""
    import torch
    C_out, cin_g, Kd, Kh, Kw = w_oidhw.shape
    code = _dtype_code(w_oidhw.dtype)
    nbytes = conv3d_packed_weight_size(C_out, cin_g * groups, Kd, Kh, Kw, groups, code)
    if w_packed is None:
        w_packed = torch.empty(nbytes // w_oidhw.element_size(), dtype=w_oidhw.dtype, device=w_oidhw.device)
    _check(load().conv3d_pack_weight(_ptr(w_oidhw), _ptr(w_packed), C_out, cin_g * groups, Kd, Kh, Kw, groups, code,
                                     _stream(stream)))
    return w_packed


def conv3d_workspace_size(N, C_in, D, H, W, C_out, Kd, Kh, Kw, stride, pad, dilation, groups, dtype, layout) -> int:
    out = ctypes.c_size_t(0)
    _check(load().conv3d_workspace_size(N, C_in, D, H, W, C_out, Kd, Kh, Kw, stride, pad, dilation, groups, dtype,
                                        _layout_code(layout), ctypes.byref(out)))
    return out.value


def conv3d_forward(x, w_packed, bias, y, N, C_in, D, H, W, C_out, Kd, Kh, Kw, stride, pad, dilation, groups, dtype,
                   layout, workspace=None, stream=None):
    wp, wb = _ws(workspace)
    _check(load().conv3d_forward(_ptr(x), _ptr(w_packed), _ptr(bias), _ptr(y), N, C_in, D, H, W, C_out, Kd, Kh, Kw,
                                 stride, pad, dilation, groups, dtype, _layout_code(layout), wp, wb, _stream(stream)))
    return y


class Conv3dB200:
    """One 3-D convolution layer: packed weights, bias and scratch on the device.

    ``w`` is an OIDHW tensor (C_out, C_in/groups, Kd, Kh, Kw) of dtype bf16 or fp32;
    ``layout`` is "nhwc" (NDHWC tensors) or "nchw" (NCDHW)."""

    def __init__(self, w, bias=None, stride=1, pad=0, dilation=1, groups=1, layout="nhwc"):
        self.C_out, cin_g, self.Kd, self.Kh, self.Kw = (int(v) for v in w.shape)
        self.C_in = cin_g * groups
        self.stride, self.pad, self.dilation, self.groups = stride, pad, dilation, groups
        self.layout = _layout_code(layout)
        self.torch_dtype = w.dtype
        self.dtype = _dtype_code(w.dtype)
        self.w_packed = conv3d_pack_weight(w.contiguous(), groups)
        self.bias = None if bias is None else bias.to(w.dtype).contiguous()
        self._ws = {}

    def out_shape(self, N, D, H, W):
        o = [conv2d_output_size(v, k, self.stride, self.pad, self.dilation)
             for v, k in ((D, self.Kd), (H, self.Kh), (W, self.Kw))]
        return (N, self.C_out, *o) if self.layout == CONV_NCHW else (N, *o, self.C_out)

    def __call__(self, x, y=None, stream=None):
        import torch
        if self.layout == CONV_NCHW:
            N, C, D, H, W = (int(v) for v in x.shape)
        else:
            N, D, H, W, C = (int(v) for v in x.shape)
        if C != self.C_in:
            raise ValueError(f"x has {C} channels, the layer expects {self.C_in}")
        if y is None:
            y = torch.empty(self.out_shape(N, D, H, W), dtype=self.torch_dtype, device=x.device)
        args = (N, self.C_in, D, H, W, self.C_out, self.Kd, self.Kh, self.Kw, self.stride, self.pad, self.dilation,
                self.groups)
        key = (N, D, H, W)
        if key not in self._ws:
            nbytes = conv3d_workspace_size(*args, self.dtype, self.layout)
            self._ws[key] = torch.empty(max(nbytes, 16), dtype=torch.uint8, device=x.device)
        conv3d_forward(x, self.w_packed, self.bias, y, *args, self.dtype, self.layout, self._ws[key], stream)
        return y


# ------------------------------------------------------------- convenience ---
class Conv2dB200:
    """One convolution layer: packed weights, bias and scratch live on the device.

    ``w`` is an OIHW tensor (C_out, C_in/groups, Kh, Kw) of dtype bf16 or fp32 on
    the current CUDA device; ``layout`` is "nhwc" or "nchw" for x and y."""

    def __init__(self, w, bias=None, stride=1, pad=0, dilation=1, groups=1, layout="nhwc"):
        self.C_out, cin_g, self.Kh, self.Kw = (int(v) for v in w.shape)
        self.C_in = cin_g * groups
        self.stride, self.pad, self.dilation, self.groups = stride, pad, dilation, groups
        self.layout = _layout_code(layout)
        self.torch_dtype = w.dtype
        self.dtype = _dtype_code(w.dtype)
        self._w_oihw = w.contiguous()
        self.w_packed = conv2d_pack_weight(self._w_oihw, groups)
        self.w_packed_t = None
        self.bias = None if bias is None else bias.to(w.dtype).contiguous()
        self._ws = {}

    def out_shape(self, N, H, W):
        Ho = conv2d_output_size(H, self.Kh, self.stride, self.pad, self.dilation)
        Wo = conv2d_output_size(W, self.Kw, self.stride, self.pad, self.dilation)
        if self.layout == CONV_NCHW:
            return (N, self.C_out, Ho, Wo)
        return (N, Ho, Wo, self.C_out)

    def _shape_args(self, N, H, W):
        return (N, self.C_in, H, W, self.C_out, self.Kh, self.Kw, self.stride, self.pad,
                self.dilation, self.groups)

    def workspace(self, N, H, W, explicit_im2col=False):
        import torch
        key = (N, H, W, explicit_im2col)
        if key not in self._ws:
            fn = conv2d_im2col_workspace_size if explicit_im2col else conv2d_workspace_size
            nbytes = fn(*self._shape_args(N, H, W), self.dtype, self.layout)
            self._ws[key] = torch.empty(max(nbytes, 16), dtype=torch.uint8, device=self.w_packed.device)
        return self._ws[key]

    def _nhw(self, x):
        if self.layout == CONV_NCHW:
            N, C, H, W = x.shape
        else:
            N, H, W, C = x.shape
        if C != self.C_in:
            raise ValueError(f"x has {C} channels, the layer expects {self.C_in}")
        return int(N), int(H), int(W)

    def __call__(self, x, y=None, explicit_im2col=False, stream=None):
        import torch
        N, H, W = self._nhw(x)
        if y is None:
            y = torch.empty(self.out_shape(N, H, W), dtype=self.torch_dtype, device=x.device)
        fn = conv2d_forward_im2col_gemm if explicit_im2col else conv2d_forward
        fn(x, self.w_packed, self.bias, y, *self._shape_args(N, H, W), self.dtype, self.layout,
           self.workspace(N, H, W, explicit_im2col), stream)
        return y

    def _scratch(self, key, nbytes):
        import torch
        if key not in self._ws or self._ws[key].numel() < nbytes:
            self._ws[key] = torch.empty(max(nbytes, 16), dtype=torch.uint8, device=self.w_packed.device)
        return self._ws[key]

    def backward_data(self, dy, H, W, dx=None, stream=None):
        """dx for dy (y's shape and layout); the transposed kernel is packed on first use."""
        import torch
        N = int(dy.shape[0])
        if getattr(self, "w_packed_t", None) is None:
            self.w_packed_t = conv2d_pack_weight_backward_data(self._w_oihw, self.groups)
        shape = (N, self.C_in, H, W) if self.layout == CONV_NCHW else (N, H, W, self.C_in)
        if dx is None:
            dx = torch.empty(shape, dtype=self.torch_dtype, device=dy.device)
        args = self._shape_args(N, H, W)
        ws = self._scratch(("dgrad", N, H, W), conv2d_backward_data_workspace_size(*args, self.dtype, self.layout))
        return conv2d_backward_data(dy, self.w_packed_t, dx, *args, self.dtype, self.layout, ws, stream)

    def backward_weight(self, x, dy, dw=None, db=None, stream=None):
        """(dw, db) for input x and dy; dw is OIHW like the layer's weight; db only with a bias."""
        import torch
        N, H, W = self._nhw(x)
        if dw is None:
            dw = torch.empty(self.C_out, self.C_in // self.groups, self.Kh, self.Kw, dtype=self.torch_dtype,
                             device=x.device)
        if db is None and self.bias is not None:
            db = torch.empty(self.C_out, dtype=self.torch_dtype, device=x.device)
        args = self._shape_args(N, H, W)
        nbytes = conv2d_backward_weight_workspace_size(*args, self.dtype, self.layout, db is not None)
        ws = self._scratch(("wgrad", N, H, W, db is not None), nbytes)
        conv2d_backward_weight(x, dy, dw, db, *args, self.dtype, self.layout, ws, stream)
        return dw, db

    def forward_hostio(self, x_host, y_host, x_dev, y_dev, stream=None):
        N, H, W = self._nhw(x_host)
        return conv2d_forward_hostio(x_host, y_host, x_dev, y_dev, self.w_packed, self.bias,
                                     *self._shape_args(N, H, W), self.dtype, self.layout,
                                     self.workspace(N, H, W), stream)
