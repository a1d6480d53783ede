"""Oracle for grouped / depthwise convolution -- TEST INFRASTRUCTURE ONLY.

A plain fp64 CPU implementation (``oracle.c``, nested loops, OpenMP over the outermost
output loop) of what the CUDA library computes. Only the tests, the package smoke check
and the benchmark's CPU-baseline leg import this module; the product path never does,
and the two share no code.

Definitions followed (see the header of ``oracle.c`` for the full statement):
  * grouped conv2d -- "Grouped convolutions" (neon issue #296): channels, filters and
    outputs split into groups with no cross-group connections, group-major channel
    order; cross-correlation with zero padding as ``F.conv2d(..., groups=g)`` in
    "F.conv2d runs x15 slower in mixed-precision/half-precision mode";
  * the data and weight gradients of grouped conv2d (scatter / direct-sum forms of the
    forward sum's adjoint), for the training uses of grouped layers on the pages;
  * the neon thread's output variants: interleaved (1234...) output order and average / max
    merges across groups;
  * the depthwise-separable block (depthwise conv, then a pointwise 1x1 conv over channels)
    of the same Conformer thread, 1-D and 2-D;
  * depthwise conv1d on (batch, steps, channels), forward and backward -- "Investigate
    custom Triton kernels for depthwise-separable convolutions in Conformer".

Every function takes and returns float64 numpy arrays (inputs are the exact values the
GPU receives, widened to fp64).
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")

NCHW = 0
NHWC = 1

_lib = None


def build(force: bool = False) -> str:
    """Compile ``oracle.c`` into ``liboracle.so`` with gcc (OpenMP on)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c99",
                               "-Wall", "-Wno-unknown-pragmas", _SRC, "-o", tmp])
        os.replace(tmp, _LIB)
    return _LIB


def _configure(lib):
    """Declare the C signatures on a loaded oracle library."""
    L, I, P = ctypes.c_long, ctypes.c_int, ctypes.c_void_p
    lib.oracle_conv2d.argtypes = [P, P, P, P] + [L] * 11 + [I]
    lib.oracle_conv2d.restype = I
    lib.oracle_conv2d_points.argtypes = [P, P, P, P, P, L] + [L] * 11 + [I]
    lib.oracle_conv2d_points.restype = I
    for name in ("oracle_conv2d_bwd_data", "oracle_conv2d_bwd_weight"):
        f = getattr(lib, name)
        f.argtypes = [P, P, P] + [L] * 11 + [I]
        f.restype = I
    for name in ("oracle_conv2d_bwd_data_points", "oracle_conv2d_bwd_weight_points"):
        f = getattr(lib, name)
        f.argtypes = [P, P, P, P, L] + [L] * 11 + [I]
        f.restype = I
    for name in ("oracle_dwconv1d_fwd", "oracle_dwconv1d_bwd_data",
                 "oracle_dwconv1d_bwd_weight"):
        f = getattr(lib, name)
        f.argtypes = [P, P, P] + [L] * 6
        f.restype = I
    lib.oracle_conv2d_interleaved.argtypes = [P, P, P, P] + [L] * 11 + [I]
    lib.oracle_conv2d_interleaved.restype = I
    lib.oracle_conv2d_group_merge.argtypes = [P, P, P, P] + [L] * 11 + [I, I]
    lib.oracle_conv2d_group_merge.restype = I
    lib.oracle_dwsep1d_fwd.argtypes = [P] * 6 + [L] * 7
    lib.oracle_dwsep1d_fwd.restype = I
    lib.oracle_dwsep1d_points.argtypes = [P] * 6 + [L] * 8
    lib.oracle_dwsep1d_points.restype = I
    lib.oracle_dwsep2d_fwd.argtypes = [P] * 6 + [L] * 10 + [I]
    lib.oracle_dwsep2d_fwd.restype = I
    lib.oracle_conv_out_extent.argtypes = [L] * 5
    lib.oracle_conv_out_extent.restype = L
    lib.oracle_num_threads.argtypes = []
    lib.oracle_num_threads.restype = I
    return lib


def _load():
    global _lib
    if _lib is None:
        _lib = _configure(ctypes.CDLL(build()))
    return _lib


def _f64(a):
    return np.ascontiguousarray(a, dtype=np.float64)


def _ptr(a):
    return None if a is None else a.ctypes.data


def num_threads() -> int:
    return int(_load().oracle_num_threads())


def out_extent(size: int, k: int, stride: int, pad: int, dilation: int) -> int:
    return int(_load().oracle_conv_out_extent(size, k, stride, pad, dilation))


def conv2d_out_shape(x_shape, w_shape, stride, pad, dilation, groups, layout):
    if layout == NCHW:
        N, C_in, H, W = x_shape
        C_out, _, kH, kW = w_shape
    else:
        N, H, W, C_in = x_shape
        C_out, kH, kW, _ = w_shape
    Ho = out_extent(H, kH, stride, pad, dilation)
    Wo = out_extent(W, kW, stride, pad, dilation)
    return (N, C_out, Ho, Wo) if layout == NCHW else (N, Ho, Wo, C_out)


def _conv_args(x, w, groups, layout):
    if layout == NCHW:
        N, C_in, H, W = x.shape
        C_out, cpg_in, kH, kW = w.shape
    elif layout == NHWC:
        N, H, W, C_in = x.shape
        C_out, kH, kW, cpg_in = w.shape
    else:
        raise ValueError("layout must be NCHW (0) or NHWC (1)")
    if groups <= 0 or C_in % groups or C_out % groups or cpg_in * groups != C_in:
        raise ValueError("inconsistent groups / channel counts")
    return N, C_in, H, W, C_out, kH, kW


def conv2d(x, w, bias=None, stride=1, pad=0, dilation=1, groups=1, layout=NCHW):
    """Grouped conv2d in fp64; x, w, y in the layouts of ``layout``."""
    x, w = _f64(x), _f64(w)
    b = None if bias is None else _f64(bias)
    N, C_in, H, W, C_out, kH, kW = _conv_args(x, w, groups, layout)
    y = np.empty(conv2d_out_shape(x.shape, w.shape, stride, pad, dilation, groups, layout))
    rc = _load().oracle_conv2d(_ptr(x), _ptr(w), _ptr(b), _ptr(y), N, C_in, H, W, C_out, kH,
                               kW, stride, pad, dilation, groups, layout)
    if rc != 0:
        raise ValueError("oracle_conv2d rejected the shape")
    return y


def conv2d_points(x, w, idx, bias=None, stride=1, pad=0, dilation=1, groups=1, layout=NCHW):
    """Outputs of grouped conv2d at idx[i] = (n, co, ho, wo) (logical indices)."""
    x, w = _f64(x), _f64(w)
    b = None if bias is None else _f64(bias)
    idx = np.ascontiguousarray(idx, dtype=np.int64).reshape(-1, 4)
    N, C_in, H, W, C_out, kH, kW = _conv_args(x, w, groups, layout)
    out = np.empty(idx.shape[0])
    rc = _load().oracle_conv2d_points(_ptr(x), _ptr(w), _ptr(b), _ptr(out), _ptr(idx),
                                      idx.shape[0], N, C_in, H, W, C_out, kH, kW, stride, pad,
                                      dilation, groups, layout)
    if rc != 0:
        raise ValueError("oracle_conv2d_points rejected the shape or an index")
    return out


def conv2d_interleaved(x, w, bias=None, stride=1, pad=0, dilation=1, groups=1, layout=NCHW):
    """Grouped conv2d with the interleaved output order: position j*groups + i holds filter j
    of group i (group-major channel i*cpg_out + j)."""
    x, w = _f64(x), _f64(w)
    b = None if bias is None else _f64(bias)
    N, C_in, H, W, C_out, kH, kW = _conv_args(x, w, groups, layout)
    y = np.empty(conv2d_out_shape(x.shape, w.shape, stride, pad, dilation, groups, layout))
    if _load().oracle_conv2d_interleaved(_ptr(x), _ptr(w), _ptr(b), _ptr(y), N, C_in, H, W,
                                         C_out, kH, kW, stride, pad, dilation, groups,
                                         layout) != 0:
        raise ValueError("oracle_conv2d_interleaved rejected the shape")
    return y


def conv2d_group_merge(x, w, bias=None, stride=1, pad=0, dilation=1, groups=1, layout=NCHW,
                       mode="avg"):
    """Grouped conv2d merged across groups: channel j = mean ('avg') or max ('max') over
    groups i of group-major channel i*cpg_out + j; cpg_out output channels."""
    x, w = _f64(x), _f64(w)
    b = None if bias is None else _f64(bias)
    N, C_in, H, W, C_out, kH, kW = _conv_args(x, w, groups, layout)
    full = conv2d_out_shape(x.shape, w.shape, stride, pad, dilation, groups, layout)
    cpg_out = C_out // groups
    shape = (full[0], cpg_out, full[2], full[3]) if layout == NCHW else (
        full[0], full[1], full[2], cpg_out)
    y = np.empty(shape)
    code = {"avg": 0, "max": 1}[mode]
    if _load().oracle_conv2d_group_merge(_ptr(x), _ptr(w), _ptr(b), _ptr(y), N, C_in, H, W,
                                         C_out, kH, kW, stride, pad, dilation, groups, layout,
                                         code) != 0:
        raise ValueError("oracle_conv2d_group_merge rejected the shape")
    return y


def _bwd_dims(dy_shape, w_shape, in_hw, stride, pad, dilation, groups, layout):
    """(N, C_in, H, W, C_out, kH, kW) of the forward problem behind a backward call, checking
    that dy has that problem's output shape."""
    H, W = in_hw
    if layout == NCHW:
        N, C_out = dy_shape[0], dy_shape[1]
        C_out2, cpg_in, kH, kW = w_shape
    elif layout == NHWC:
        N, C_out = dy_shape[0], dy_shape[3]
        C_out2, kH, kW, cpg_in = w_shape
    else:
        raise ValueError("layout must be NCHW (0) or NHWC (1)")
    C_in = cpg_in * groups
    if C_out2 != C_out or groups <= 0 or C_out % groups:
        raise ValueError("inconsistent groups / channel counts")
    x_shape = (N, C_in, H, W) if layout == NCHW else (N, H, W, C_in)
    if tuple(dy_shape) != conv2d_out_shape(x_shape, w_shape, stride, pad, dilation, groups,
                                           layout):
        raise ValueError("dy does not have the forward output's shape")
    return (N, C_in, H, W, C_out, kH, kW), x_shape


def conv2d_bwd_data(dy, w, in_hw, stride=1, pad=0, dilation=1, groups=1, layout=NCHW):
    """dx of grouped conv2d (input spatial size ``in_hw`` = (H, W)), in x's layout."""
    dy, w = _f64(dy), _f64(w)
    dims, x_shape = _bwd_dims(dy.shape, w.shape, in_hw, stride, pad, dilation, groups, layout)
    dx = np.empty(x_shape)
    if _load().oracle_conv2d_bwd_data(_ptr(dy), _ptr(w), _ptr(dx), *dims, stride, pad,
                                      dilation, groups, layout) != 0:
        raise ValueError("oracle_conv2d_bwd_data rejected the shape")
    return dx


def conv2d_bwd_data_points(dy, w, in_hw, idx, stride=1, pad=0, dilation=1, groups=1,
                           layout=NCHW):
    """dx at idx[i] = (n, c, h, w) (logical indices)."""
    dy, w = _f64(dy), _f64(w)
    dims, _ = _bwd_dims(dy.shape, w.shape, in_hw, stride, pad, dilation, groups, layout)
    idx = np.ascontiguousarray(idx, dtype=np.int64).reshape(-1, 4)
    out = np.empty(idx.shape[0])
    if _load().oracle_conv2d_bwd_data_points(_ptr(dy), _ptr(w), _ptr(out), _ptr(idx),
                                             idx.shape[0], *dims, stride, pad, dilation, groups,
                                             layout) != 0:
        raise ValueError("oracle_conv2d_bwd_data_points rejected the shape or an index")
    return out


def conv2d_bwd_weight(x, dy, kernel_hw, stride=1, pad=0, dilation=1, groups=1, layout=NCHW):
    """dw of grouped conv2d (kernel size ``kernel_hw`` = (kH, kW)), in w's layout."""
    x, dy = _f64(x), _f64(dy)
    w_shape = _wgrad_w_shape(x.shape, dy.shape, kernel_hw, groups, layout)
    dims, _ = _bwd_dims(dy.shape, w_shape, _hw(x.shape, layout), stride, pad, dilation, groups,
                        layout)
    dw = np.empty(w_shape)
    if _load().oracle_conv2d_bwd_weight(_ptr(x), _ptr(dy), _ptr(dw), *dims, stride, pad,
                                        dilation, groups, layout) != 0:
        raise ValueError("oracle_conv2d_bwd_weight rejected the shape")
    return dw


def conv2d_bwd_weight_points(x, dy, kernel_hw, idx, stride=1, pad=0, dilation=1, groups=1,
                             layout=NCHW):
    """dw at idx[i] = (co, ci, kh, kw) (logical indices, ci within the group)."""
    x, dy = _f64(x), _f64(dy)
    w_shape = _wgrad_w_shape(x.shape, dy.shape, kernel_hw, groups, layout)
    dims, _ = _bwd_dims(dy.shape, w_shape, _hw(x.shape, layout), stride, pad, dilation, groups,
                        layout)
    idx = np.ascontiguousarray(idx, dtype=np.int64).reshape(-1, 4)
    out = np.empty(idx.shape[0])
    if _load().oracle_conv2d_bwd_weight_points(_ptr(x), _ptr(dy), _ptr(out), _ptr(idx),
                                               idx.shape[0], *dims, stride, pad, dilation,
                                               groups, layout) != 0:
        raise ValueError("oracle_conv2d_bwd_weight_points rejected the shape or an index")
    return out


def _hw(x_shape, layout):
    return (x_shape[2], x_shape[3]) if layout == NCHW else (x_shape[1], x_shape[2])


def _wgrad_w_shape(x_shape, dy_shape, kernel_hw, groups, layout):
    kH, kW = kernel_hw
    C_in = x_shape[1] if layout == NCHW else x_shape[3]
    C_out = dy_shape[1] if layout == NCHW else dy_shape[3]
    if groups <= 0 or C_in % groups:
        raise ValueError("inconsistent groups / channel counts")
    cpg_in = C_in // groups
    return (C_out, cpg_in, kH, kW) if layout == NCHW else (C_out, kH, kW, cpg_in)


def _conv1d_check(x_shape, w_shape):
    B, T, C = x_shape
    C2, K = w_shape
    if C2 != C:
        raise ValueError("w must be [C, K]")
    return B, T, C, K


def dwconv1d_fwd(x, w, pad_left, pad_right):
    """y[b,t,c] = sum_k w[c,k] x[b,t+k-pad_left,c] on (batch, steps, channels)."""
    x, w = _f64(x), _f64(w)
    B, T, C, K = _conv1d_check(x.shape, w.shape)
    T_out = T + pad_left + pad_right - K + 1
    y = np.empty((B, T_out, C))
    if _load().oracle_dwconv1d_fwd(_ptr(x), _ptr(w), _ptr(y), B, T, C, K, pad_left,
                                   pad_right) != 0:
        raise ValueError("oracle_dwconv1d_fwd rejected the shape")
    return y


def dwconv1d_bwd_data(dy, w, T, pad_left, pad_right):
    """dx for dwconv1d_fwd, given dy [B, T_out, C] and the input length T."""
    dy, w = _f64(dy), _f64(w)
    B, T_out, C = dy.shape
    K = w.shape[1]
    if T_out != T + pad_left + pad_right - K + 1:
        raise ValueError("dy has the wrong number of steps")
    dx = np.empty((B, T, C))
    if _load().oracle_dwconv1d_bwd_data(_ptr(dy), _ptr(w), _ptr(dx), B, T, C, K, pad_left,
                                        pad_right) != 0:
        raise ValueError("oracle_dwconv1d_bwd_data rejected the shape")
    return dx


def dwconv1d_bwd_weight(x, dy, K, pad_left, pad_right):
    """dw [C, K] for dwconv1d_fwd, given x [B, T, C] and dy [B, T_out, C]."""
    x, dy = _f64(x), _f64(dy)
    B, T, C = x.shape
    if dy.shape != (B, T + pad_left + pad_right - K + 1, C):
        raise ValueError("dy has the wrong shape")
    dw = np.empty((C, K))
    if _load().oracle_dwconv1d_bwd_weight(_ptr(x), _ptr(dy), _ptr(dw), B, T, C, K, pad_left,
                                          pad_right) != 0:
        raise ValueError("oracle_dwconv1d_bwd_weight rejected the shape")
    return dw


def _dwsep_pw(w_pw, bias, C):
    w_pw = _f64(w_pw)
    if w_pw.ndim != 2 or w_pw.shape[1] != C:
        raise ValueError("w_pw must be [C_out, C]")
    b = None if bias is None else _f64(bias)
    if b is not None and b.shape != (w_pw.shape[0],):
        raise ValueError("bias must be [C_out]")
    return w_pw, b


def dwsep1d_fwd(x, w_dw, w_pw, bias, pad_left, pad_right):
    """Depthwise-separable block on (batch, steps, channels): z = pointwise(dwconv1d(x)),
    z[b,t,o] = bias[o] + sum_c w_pw[o,c] * dwconv1d_fwd(x, w_dw)[b,t,c]."""
    x, w_dw = _f64(x), _f64(w_dw)
    B, T, C, K = _conv1d_check(x.shape, w_dw.shape)
    w_pw, b = _dwsep_pw(w_pw, bias, C)
    T_out = T + pad_left + pad_right - K + 1
    y = np.empty((B, max(T_out, 0), C))
    z = np.empty((B, max(T_out, 0), w_pw.shape[0]))
    if _load().oracle_dwsep1d_fwd(_ptr(x), _ptr(w_dw), _ptr(w_pw), _ptr(b), _ptr(y), _ptr(z), B,
                                  T, C, K, pad_left, pad_right, w_pw.shape[0]) != 0:
        raise ValueError("oracle_dwsep1d_fwd rejected the shape")
    return z


def dwsep1d_points(x, w_dw, w_pw, bias, idx, pad_left, pad_right):
    """Outputs of the 1-D depthwise-separable block at idx[i] = (b, t, o)."""
    x, w_dw = _f64(x), _f64(w_dw)
    B, T, C, K = _conv1d_check(x.shape, w_dw.shape)
    w_pw, b = _dwsep_pw(w_pw, bias, C)
    idx = np.ascontiguousarray(idx, dtype=np.int64).reshape(-1, 3)
    out = np.empty(idx.shape[0])
    if _load().oracle_dwsep1d_points(_ptr(x), _ptr(w_dw), _ptr(w_pw), _ptr(b), _ptr(out),
                                     _ptr(idx), idx.shape[0], B, T, C, K, pad_left, pad_right,
                                     w_pw.shape[0]) != 0:
        raise ValueError("oracle_dwsep1d_points rejected the shape or an index")
    return out


def dwsep2d_fwd(x, w_dw, w_pw, bias=None, stride=1, pad=0, dilation=1, layout=NCHW):
    """2-D depthwise-separable block: z = pointwise(depthwise conv2d(x)); x and z in `layout`,
    w_dw the depthwise weight of that layout ([C,1,kH,kW] / [C,kH,kW,1]), w_pw [C_out, C]."""
    x, w_dw = _f64(x), _f64(w_dw)
    if layout == NCHW:
        N, C, H, W = x.shape
        C2, one, kH, kW = w_dw.shape
    else:
        N, H, W, C = x.shape
        C2, kH, kW, one = w_dw.shape
    if C2 != C or one != 1:
        raise ValueError("w_dw must be the depthwise weight of x's channels")
    w_pw, b = _dwsep_pw(w_pw, bias, C)
    y_shape = conv2d_out_shape(x.shape, w_dw.shape, stride, pad, dilation, C, layout)
    y = np.empty(y_shape)
    C_out = w_pw.shape[0]
    z_shape = (y_shape[0], C_out, y_shape[2], y_shape[3]) if layout == NCHW else (
        y_shape[0], y_shape[1], y_shape[2], C_out)
    z = np.empty(z_shape)
    if _load().oracle_dwsep2d_fwd(_ptr(x), _ptr(w_dw), _ptr(w_pw), _ptr(b), _ptr(y), _ptr(z), N,
                                  C, H, W, kH, kW, stride, pad, dilation, C_out, layout) != 0:
        raise ValueError("oracle_dwsep2d_fwd rejected the shape")
    return z
