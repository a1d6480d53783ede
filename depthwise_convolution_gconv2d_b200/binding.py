"""ctypes binding over libgconv.so (include/gconv.h).

Argument marshalling only: each function reads sizes from torch CUDA tensors, allocates
outputs (and the workspace the library asks for) with torch, and passes raw device
pointers, sizes and the current CUDA stream to the C ABI. Every step of the computation
runs in the library's kernels. There is no fallback: if the library cannot be loaded,
``load_library`` raises RuntimeError.

Tensors are taken in their physical (contiguous) layout:
  NCHW  x [N, C_in, H, W], w [C_out, C_in/g, kH, kW] -> y [N, C_out, Ho, Wo]
  NHWC  x [N, H, W, C_in], w [C_out, kH, kW, C_in/g] -> y [N, Ho, Wo, C_out]
  conv1d  x [B, T, C], w [C, K], dy [B, T_out, C]
"""
from __future__ import annotations

import ctypes
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
_LIB_PATH = os.path.join(_PKG, "libgconv.so")

NCHW, NHWC = 0, 1
F32, F16, BF16 = 0, 1, 2
PATH_AUTO, PATH_DIRECT, PATH_IGEMM, PATH_GENERIC = 0, 1, 2, 3
KERNEL_NAMES = {1: "direct_generic", 2: "depthwise_nhwc", 3: "igemm_tc", 4: "igemm_tc_nchw",
                5: "conv1d_generic", 6: "conv1d_ring", 7: "conv1d_tc", 8: "grouped_nhwc",
                9: "dgrad_generic", 10: "wgrad_generic", 11: "wgrad_depthwise_nhwc",
                12: "dgrad_depthwise_nhwc", 13: "wgrad_tiled_nhwc", 14: "wgrad_dw3_tma",
                15: "wgrad_tiled_nchw", 16: "dwsep1d_fused", 17: "dwsep_unfused",
                18: "wgrad_tc_nhwc", 19: "wgrad_tc_nchw", 20: "conv1d_strip",
                21: "dwsep2d_fused", 22: "dgrad_dw3s2_tma", 23: "merge_max_two_pass"}
STATUS = {0: "GCONV_OK", 1: "GCONV_ERR_INVALID_ARG", 2: "GCONV_ERR_UNSUPPORTED",
          3: "GCONV_ERR_MISALIGNED", 4: "GCONV_ERR_WORKSPACE", 5: "GCONV_ERR_CUDA",
          6: "GCONV_ERR_DEVICE_TIMEOUT"}

EXPORTS = ["gconv2d_fwd", "gconv2d_fwd_path", "gconv2d_fwd_workspace_size",
           "gconv2d_select_path", "gconv2d_bwd_data", "gconv2d_bwd_data_path",
           "gconv2d_bwd_data_workspace_size", "gconv2d_bwd_data_select_path",
           "gconv2d_bwd_weight", "gconv2d_bwd_weight_path", "gconv2d_bwd_weight_workspace_size",
           "gconv2d_bwd_weight_select_path", "dwconv1d_fwd", "dwconv1d_bwd_data", "dwconv1d_fwd_path",
           "dwconv1d_bwd_data_path", "dwconv1d_select_path",
           "dwconv1d_bwd_weight", "dwconv1d_bwd_weight_workspace_size",
           "dwconv1d_bwd_weight_noalloc", "gconv2d_out_shape", "dwconv1d_out_steps",
           "gconv_debug_set_tx_surplus", "gconv2d_fwd_out", "gconv2d_fwd_out_workspace_size",
           "gconv2d_fwd_out_select_path", "dwsep1d_fwd", "dwsep1d_fwd_workspace_size",
           "dwsep1d_select_path", "dwsep2d_fwd", "dwsep2d_fwd_workspace_size",
           "dwsep2d_select_path",
           "gconv_get_device_error", "gconv_status_string", "gconv_version"]

_lib = None


class GconvError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {STATUS.get(status, status)}")


def library_path() -> str:
    return _LIB_PATH


def load_library():
    """Load libgconv.so once and declare the C signatures."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(_LIB_PATH):
        raise RuntimeError(f"{_LIB_PATH} is missing: build it with "
                           "`python -m depthwise_convolution_gconv2d_b200.build`")
    try:
        lib = ctypes.CDLL(_LIB_PATH)
    except OSError as e:
        raise RuntimeError(f"cannot load {_LIB_PATH}: {e}") from e
    I, P, Z = ctypes.c_int, ctypes.c_void_p, ctypes.c_size_t
    conv = [I] * 11
    lib.gconv2d_fwd_workspace_size.argtypes = conv + [I, I, I]
    lib.gconv2d_fwd_workspace_size.restype = Z
    lib.gconv2d_fwd.argtypes = [P, P, P, P] + conv + [I, I, P, Z, P]
    lib.gconv2d_fwd.restype = I
    lib.gconv2d_fwd_path.argtypes = [P, P, P, P] + conv + [I, I, I, P, Z, P]
    lib.gconv2d_fwd_path.restype = I
    lib.gconv2d_select_path.argtypes = conv + [I, I, I]
    lib.gconv2d_select_path.restype = I
    for name in ("gconv2d_bwd_data", "gconv2d_bwd_weight"):
        getattr(lib, name).argtypes = [P, P, P] + conv + [I, I, P, Z, P]
        getattr(lib, name).restype = I
    for name in ("gconv2d_bwd_data_path", "gconv2d_bwd_weight_path"):
        getattr(lib, name).argtypes = [P, P, P] + conv + [I, I, I, P, Z, P]
        getattr(lib, name).restype = I
    for name in ("gconv2d_bwd_data_workspace_size", "gconv2d_bwd_weight_workspace_size"):
        getattr(lib, name).argtypes = conv + [I, I, I]
        getattr(lib, name).restype = Z
    for name in ("gconv2d_bwd_data_select_path", "gconv2d_bwd_weight_select_path"):
        getattr(lib, name).argtypes = conv + [I, I, I]
        getattr(lib, name).restype = I
    lib.dwconv1d_fwd.argtypes = [P, P, P] + [I] * 6 + [I, P]
    lib.dwconv1d_fwd.restype = I
    lib.dwconv1d_bwd_data.argtypes = [P, P, P] + [I] * 6 + [I, P]
    lib.dwconv1d_bwd_data.restype = I
    lib.dwconv1d_fwd_path.argtypes = [P, P, P] + [I] * 6 + [I, I, P]
    lib.dwconv1d_fwd_path.restype = I
    lib.dwconv1d_bwd_data_path.argtypes = [P, P, P] + [I] * 6 + [I, I, P]
    lib.dwconv1d_bwd_data_path.restype = I
    lib.dwconv1d_select_path.argtypes = [I] * 8
    lib.dwconv1d_select_path.restype = I
    lib.dwconv1d_bwd_weight_workspace_size.argtypes = [I] * 7
    lib.dwconv1d_bwd_weight_workspace_size.restype = Z
    lib.dwconv1d_bwd_weight.argtypes = [P, P, P, P, Z] + [I] * 6 + [I, P]
    lib.dwconv1d_bwd_weight.restype = I
    lib.dwconv1d_bwd_weight_noalloc.argtypes = [P, P, P] + [I] * 6 + [I, P]
    lib.dwconv1d_bwd_weight_noalloc.restype = I
    lib.gconv2d_out_shape.argtypes = conv + [I, I, I] + [ctypes.POINTER(I)] * 3
    lib.gconv2d_out_shape.restype = I
    lib.gconv2d_fwd_out.argtypes = [P, P, P, P] + conv + [I, I, I, I, P, Z, P]
    lib.gconv2d_fwd_out.restype = I
    lib.gconv2d_fwd_out_workspace_size.argtypes = conv + [I, I, I, I]
    lib.gconv2d_fwd_out_workspace_size.restype = Z
    lib.gconv2d_fwd_out_select_path.argtypes = conv + [I, I, I, I]
    lib.gconv2d_fwd_out_select_path.restype = I
    lib.dwconv1d_out_steps.argtypes = [I] * 7 + [ctypes.POINTER(I)]
    lib.dwconv1d_out_steps.restype = I
    lib.gconv_debug_set_tx_surplus.argtypes = [ctypes.c_uint]
    lib.gconv_debug_set_tx_surplus.restype = I
    lib.dwsep1d_fwd_workspace_size.argtypes = [I] * 9
    lib.dwsep1d_fwd_workspace_size.restype = Z
    lib.dwsep1d_select_path.argtypes = [I] * 9
    lib.dwsep1d_select_path.restype = I
    lib.dwsep1d_fwd.argtypes = [P] * 5 + [I] * 9 + [P, Z, P]
    lib.dwsep1d_fwd.restype = I
    lib.dwsep2d_fwd_workspace_size.argtypes = [I] * 13
    lib.dwsep2d_fwd_workspace_size.restype = Z
    lib.dwsep2d_select_path.argtypes = [I] * 13
    lib.dwsep2d_select_path.restype = I
    lib.dwsep2d_fwd.argtypes = [P] * 5 + [I] * 13 + [P, Z, P]
    lib.dwsep2d_fwd.restype = I
    lib.gconv_get_device_error.argtypes = [P, ctypes.POINTER(I)]
    lib.gconv_get_device_error.restype = I
    lib.gconv_status_string.argtypes = [I]
    lib.gconv_status_string.restype = ctypes.c_char_p
    lib.gconv_version.argtypes = []
    lib.gconv_version.restype = I
    _lib = lib
    return lib


def _dtype_code(t: torch.dtype) -> int:
    if t == torch.float32:
        return F32
    if t == torch.float16:
        return F16
    if t == torch.bfloat16:
        return BF16
    raise TypeError(f"unsupported dtype {t}")


def _layout_code(layout) -> int:
    if isinstance(layout, str):
        return {"NCHW": NCHW, "NHWC": NHWC}[layout.upper()]
    return int(layout)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _check(status: int, where: str):
    if status != 0:
        raise GconvError(status, where)


def _need(t, name, dtype=None):
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TypeError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous in its physical layout")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} has dtype {t.dtype}, expected {dtype}")


OUT_GROUP_MAJOR, OUT_INTERLEAVED, OUT_MERGE_AVG, OUT_MERGE_MAX = 0, 1, 2, 3
OUT_MODES = {"group_major": OUT_GROUP_MAJOR, "interleaved": OUT_INTERLEAVED,
             "avg": OUT_MERGE_AVG, "max": OUT_MERGE_MAX}


def _out_mode(mode) -> int:
    return OUT_MODES[mode] if isinstance(mode, str) else int(mode)


def out_shape(N, C_in, H, W, C_out, kH, kW, stride, padding, dilation, groups, layout,
              dtype, out_mode=OUT_GROUP_MAJOR, channels=False):
    """(Ho, Wo) -- or (C_y, Ho, Wo) with channels=True -- of a conv2d problem from the
    library's own shape logic (gconv2d_out_shape); raises GconvError(GCONV_ERR_INVALID_ARG)
    for a problem the library rejects."""
    Cy, Ho, Wo = ctypes.c_int(0), ctypes.c_int(0), ctypes.c_int(0)
    dt = dtype if isinstance(dtype, int) else _dtype_code(dtype)
    st = load_library().gconv2d_out_shape(N, C_in, H, W, C_out, kH, kW, stride, padding,
                                          dilation, groups, _layout_code(layout), dt,
                                          _out_mode(out_mode), ctypes.byref(Cy),
                                          ctypes.byref(Ho), ctypes.byref(Wo))
    _check(st, "gconv2d_out_shape")
    return (Cy.value, Ho.value, Wo.value) if channels else (Ho.value, Wo.value)


def out_steps(B, T, C, K, pad_left, pad_right, dtype):
    """T_out of a depthwise conv1d problem (dwconv1d_out_steps); raises GconvError for a
    problem the library rejects."""
    T_out = ctypes.c_int(0)
    dt = dtype if isinstance(dtype, int) else _dtype_code(dtype)
    st = load_library().dwconv1d_out_steps(B, T, C, K, pad_left, pad_right, dt,
                                           ctypes.byref(T_out))
    _check(st, "dwconv1d_out_steps")
    return T_out.value


def conv2d_dims(x, w, stride, padding, dilation, groups, layout):
    lay = _layout_code(layout)
    if lay == NCHW:
        N, C_in, H, W = x.shape
        C_out, cpg_in, kH, kW = w.shape
    else:
        N, H, W, C_in = x.shape
        C_out, kH, kW, cpg_in = w.shape
    if cpg_in * groups != C_in:
        raise ValueError(f"weight has {cpg_in} input channels per group; x has {C_in} channels "
                         f"in {groups} groups")
    Ho, Wo = out_shape(N, C_in, H, W, C_out, kH, kW, stride, padding, dilation, groups, lay,
                       _dtype_code(x.dtype))
    y_shape = (N, C_out, Ho, Wo) if lay == NCHW else (N, Ho, Wo, C_out)
    return lay, (N, C_in, H, W, C_out, kH, kW), y_shape


def gconv2d_fwd_workspace_size(N, C_in, H, W, C_out, kH, kW, stride, padding, dilation, groups,
                               layout, dtype, path=PATH_AUTO) -> int:
    return int(load_library().gconv2d_fwd_workspace_size(
        N, C_in, H, W, C_out, kH, kW, stride, padding, dilation, groups,
        _layout_code(layout), dtype if isinstance(dtype, int) else _dtype_code(dtype), path))


def gconv2d_select_path(N, C_in, H, W, C_out, kH, kW, stride, padding, dilation, groups, layout,
                        dtype, path=PATH_AUTO) -> int:
    return int(load_library().gconv2d_select_path(
        N, C_in, H, W, C_out, kH, kW, stride, padding, dilation, groups, _layout_code(layout),
        dtype if isinstance(dtype, int) else _dtype_code(dtype), path))


def gconv2d_fwd(x, w, bias=None, stride=1, padding=0, dilation=1, groups=1, layout="NCHW",
                out=None, workspace=None, path=PATH_AUTO, stream=None):
    """Grouped conv2d forward through the C ABI; returns y."""
    lib = load_library()
    _need(x, "x")
    _need(w, "w", x.dtype)
    if bias is not None:
        _need(bias, "bias", x.dtype)
    lay, dims, y_shape = conv2d_dims(x, w, stride, padding, dilation, groups, layout)
    dt = _dtype_code(x.dtype)
    y = torch.empty(y_shape, dtype=x.dtype, device=x.device) if out is None else out
    _need(y, "out", x.dtype)
    if tuple(y.shape) != y_shape:
        raise ValueError(f"out has shape {tuple(y.shape)}, expected {y_shape}")
    ws_need = lib.gconv2d_fwd_workspace_size(*dims, stride, padding, dilation, groups, lay, dt,
                                             path)
    if ws_need and workspace is None:
        workspace = torch.empty(ws_need, dtype=torch.uint8, device=x.device)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    st = lib.gconv2d_fwd_path(_ptr(x), _ptr(w), _ptr(bias), _ptr(y), *dims, stride, padding,
                              dilation, groups, lay, dt, path, _ptr(workspace), ws_bytes,
                              _stream(stream))
    _check(st, "gconv2d_fwd")
    return y


def gconv2d_fwd_out_select_path(N, C_in, H, W, C_out, kH, kW, stride, padding, dilation,
                                groups, layout, dtype, out_mode, path=PATH_AUTO) -> int:
    return int(load_library().gconv2d_fwd_out_select_path(
        N, C_in, H, W, C_out, kH, kW, stride, padding, dilation, groups, _layout_code(layout),
        dtype if isinstance(dtype, int) else _dtype_code(dtype), _out_mode(out_mode), path))


def gconv2d_fwd_out(x, w, bias=None, stride=1, padding=0, dilation=1, groups=1, layout="NCHW",
                    out_mode="interleaved", out=None, workspace=None, path=PATH_AUTO,
                    stream=None):
    """Grouped conv2d forward with the output in another channel order or merged across
    groups (out_mode: 'group_major', 'interleaved', 'avg', 'max'); returns y."""
    lib = load_library()
    _need(x, "x")
    _need(w, "w", x.dtype)
    if bias is not None:
        _need(bias, "bias", x.dtype)
    lay, dims, _ = conv2d_dims(x, w, stride, padding, dilation, groups, layout)
    dt = _dtype_code(x.dtype)
    mode = _out_mode(out_mode)
    Cy, Ho, Wo = out_shape(*dims, stride, padding, dilation, groups, lay, dt, mode, True)
    y_shape = (dims[0], Cy, Ho, Wo) if lay == NCHW else (dims[0], Ho, Wo, Cy)
    y = torch.empty(y_shape, dtype=x.dtype, device=x.device) if out is None else out
    _need(y, "out", x.dtype)
    if tuple(y.shape) != y_shape:
        raise ValueError(f"out has shape {tuple(y.shape)}, expected {y_shape}")
    need = lib.gconv2d_fwd_out_workspace_size(*dims, stride, padding, dilation, groups, lay, dt,
                                              mode, path)
    workspace, ws_bytes = _workspace(need, workspace, x.device)
    st = lib.gconv2d_fwd_out(_ptr(x), _ptr(w), _ptr(bias), _ptr(y), *dims, stride, padding,
                             dilation, groups, lay, dt, mode, path, _ptr(workspace), ws_bytes,
                             _stream(stream))
    _check(st, "gconv2d_fwd_out")
    return y


def _bwd_dims(dy, w, in_hw, stride, padding, dilation, groups, layout):
    """(layout code, forward dims, x shape) for a backward call; checks dy's shape."""
    lay = _layout_code(layout)
    H, W = in_hw
    if lay == NCHW:
        N, C_out = dy.shape[0], dy.shape[1]
        C_out2, cpg_in, kH, kW = w.shape
    else:
        N, C_out = dy.shape[0], dy.shape[3]
        C_out2, kH, kW, cpg_in = w.shape
    if C_out2 != C_out:
        raise ValueError(f"w has {C_out2} filters; dy has {C_out} channels")
    C_in = cpg_in * groups
    Ho, Wo = out_shape(N, C_in, H, W, C_out, kH, kW, stride, padding, dilation, groups, lay,
                       _dtype_code(dy.dtype))
    want = (N, C_out, Ho, Wo) if lay == NCHW else (N, Ho, Wo, C_out)
    if tuple(dy.shape) != want:
        raise ValueError(f"dy has shape {tuple(dy.shape)}, expected {want}")
    x_shape = (N, C_in, H, W) if lay == NCHW else (N, H, W, C_in)
    return lay, (N, C_in, H, W, C_out, kH, kW), x_shape


def _workspace(need, workspace, device):
    if need and workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=device)
    return workspace, 0 if workspace is None else workspace.numel() * workspace.element_size()


def gconv2d_bwd_data_workspace_size(N, C_in, H, W, C_out, kH, kW, stride, padding, dilation,
                                    groups, layout, dtype, path=PATH_AUTO) -> int:
    return int(load_library().gconv2d_bwd_data_workspace_size(
        N, C_in, H, W, C_out, kH, kW, stride, padding, dilation, groups, _layout_code(layout),
        dtype if isinstance(dtype, int) else _dtype_code(dtype), path))


def gconv2d_bwd_data_select_path(N, C_in, H, W, C_out, kH, kW, stride, padding, dilation,
                                 groups, layout, dtype, path=PATH_AUTO) -> int:
    return int(load_library().gconv2d_bwd_data_select_path(
        N, C_in, H, W, C_out, kH, kW, stride, padding, dilation, groups, _layout_code(layout),
        dtype if isinstance(dtype, int) else _dtype_code(dtype), path))


def gconv2d_bwd_weight_workspace_size(N, C_in, H, W, C_out, kH, kW, stride, padding, dilation,
                                      groups, layout, dtype, path=PATH_AUTO) -> int:
    return int(load_library().gconv2d_bwd_weight_workspace_size(
        N, C_in, H, W, C_out, kH, kW, stride, padding, dilation, groups, _layout_code(layout),
        dtype if isinstance(dtype, int) else _dtype_code(dtype), path))


def gconv2d_bwd_weight_select_path(N, C_in, H, W, C_out, kH, kW, stride, padding, dilation,
                                   groups, layout, dtype, path=PATH_AUTO) -> int:
    return int(load_library().gconv2d_bwd_weight_select_path(
        N, C_in, H, W, C_out, kH, kW, stride, padding, dilation, groups, _layout_code(layout),
        dtype if isinstance(dtype, int) else _dtype_code(dtype), path))


def gconv2d_bwd_data(dy, w, in_hw, stride=1, padding=0, dilation=1, groups=1, layout="NCHW",
                     out=None, workspace=None, path=PATH_AUTO, stream=None):
    """Data gradient of grouped conv2d through the C ABI: dy, w -> dx (input size in_hw)."""
    lib = load_library()
    _need(dy, "dy")
    _need(w, "w", dy.dtype)
    lay, dims, x_shape = _bwd_dims(dy, w, in_hw, stride, padding, dilation, groups, layout)
    dt = _dtype_code(dy.dtype)
    dx = torch.empty(x_shape, dtype=dy.dtype, device=dy.device) if out is None else out
    _need(dx, "out", dy.dtype)
    if tuple(dx.shape) != x_shape:
        raise ValueError(f"out has shape {tuple(dx.shape)}, expected {x_shape}")
    need = lib.gconv2d_bwd_data_workspace_size(*dims, stride, padding, dilation, groups, lay, dt,
                                               path)
    workspace, ws_bytes = _workspace(need, workspace, dy.device)
    st = lib.gconv2d_bwd_data_path(_ptr(dy), _ptr(w), _ptr(dx), *dims, stride, padding,
                                   dilation, groups, lay, dt, path, _ptr(workspace), ws_bytes,
                                   _stream(stream))
    _check(st, "gconv2d_bwd_data")
    return dx


def gconv2d_bwd_weight(x, dy, kernel_hw, stride=1, padding=0, dilation=1, groups=1,
                       layout="NCHW", out=None, workspace=None, path=PATH_AUTO, stream=None):
    """Weight gradient of grouped conv2d through the C ABI: x, dy -> dw (kernel kernel_hw)."""
    lib = load_library()
    _need(x, "x")
    _need(dy, "dy", x.dtype)
    lay = _layout_code(layout)
    kH, kW = kernel_hw
    C_in = x.shape[1] if lay == NCHW else x.shape[3]
    C_out = dy.shape[1] if lay == NCHW else dy.shape[3]
    if groups <= 0 or C_in % groups:
        raise ValueError(f"{C_in} input channels do not split into {groups} groups")
    cpg_in = C_in // groups
    w_shape = (C_out, cpg_in, kH, kW) if lay == NCHW else (C_out, kH, kW, cpg_in)
    in_hw = (x.shape[2], x.shape[3]) if lay == NCHW else (x.shape[1], x.shape[2])
    _, dims, x_shape = _bwd_dims(dy, torch.empty(w_shape, device="meta"), in_hw, stride,
                                 padding, dilation, groups, lay)
    if tuple(x.shape) != x_shape:
        raise ValueError(f"x has shape {tuple(x.shape)}, expected {x_shape}")
    dt = _dtype_code(x.dtype)
    dw = torch.empty(w_shape, dtype=x.dtype, device=x.device) if out is None else out
    _need(dw, "out", x.dtype)
    if tuple(dw.shape) != w_shape:
        raise ValueError(f"out has shape {tuple(dw.shape)}, expected {w_shape}")
    need = lib.gconv2d_bwd_weight_workspace_size(*dims, stride, padding, dilation, groups, lay,
                                                 dt, path)
    workspace, ws_bytes = _workspace(need, workspace, x.device)
    st = lib.gconv2d_bwd_weight_path(_ptr(x), _ptr(dy), _ptr(dw), *dims, stride, padding,
                                     dilation, groups, lay, dt, path, _ptr(workspace), ws_bytes,
                                     _stream(stream))
    _check(st, "gconv2d_bwd_weight")
    return dw


def _conv1d_dims(x, w):
    B, T, C = x.shape
    C2, K = w.shape
    if C2 != C:
        raise ValueError("w must be [C, K] with the channel count of x")
    return B, T, C, K


def dwconv1d_select_path(B, T, C, K, pad_left, pad_right, dtype, path=PATH_AUTO) -> int:
    """Kernel code (5 generic, 6 CUDA-core ring, 7 tensor cores) a conv1d fwd / dgrad call
    would run, or a negative status."""
    dt = dtype if isinstance(dtype, int) else _dtype_code(dtype)
    return int(load_library().dwconv1d_select_path(B, T, C, K, pad_left, pad_right, dt, path))


def dwconv1d_fwd(x, w, pad_left, pad_right, out=None, stream=None, path=PATH_AUTO):
    lib = load_library()
    _need(x, "x")
    _need(w, "w", x.dtype)
    B, T, C, K = _conv1d_dims(x, w)
    T_out = out_steps(B, T, C, K, pad_left, pad_right, _dtype_code(x.dtype))
    y = torch.empty((B, T_out, C), dtype=x.dtype, device=x.device) if out is None else out
    _need(y, "out", x.dtype)
    st = lib.dwconv1d_fwd_path(_ptr(x), _ptr(w), _ptr(y), B, T, C, K, pad_left, pad_right,
                               _dtype_code(x.dtype), path, _stream(stream))
    _check(st, "dwconv1d_fwd")
    return y


def dwconv1d_bwd_data(dy, w, T, pad_left, pad_right, out=None, stream=None, path=PATH_AUTO):
    lib = load_library()
    _need(dy, "dy")
    _need(w, "w", dy.dtype)
    B, T_out, C = dy.shape
    K = w.shape[1]
    if T_out != out_steps(B, T, C, K, pad_left, pad_right, _dtype_code(dy.dtype)):
        raise ValueError("dy has the wrong number of steps for T, K and the pads")
    dx = torch.empty((B, T, C), dtype=dy.dtype, device=dy.device) if out is None else out
    _need(dx, "out", dy.dtype)
    st = lib.dwconv1d_bwd_data_path(_ptr(dy), _ptr(w), _ptr(dx), B, T, C, K, pad_left,
                                    pad_right, _dtype_code(dy.dtype), path, _stream(stream))
    _check(st, "dwconv1d_bwd_data")
    return dx


def dwconv1d_bwd_weight_workspace_size(B, T, C, K, pad_left, pad_right, dtype) -> int:
    dt = dtype if isinstance(dtype, int) else _dtype_code(dtype)
    return int(load_library().dwconv1d_bwd_weight_workspace_size(B, T, C, K, pad_left,
                                                                 pad_right, dt))


def dwconv1d_bwd_weight(x, dy, K, pad_left, pad_right, out=None, workspace=None, stream=None):
    lib = load_library()
    _need(x, "x")
    _need(dy, "dy", x.dtype)
    B, T, C = x.shape
    dt = _dtype_code(x.dtype)
    dw = torch.empty((C, K), dtype=x.dtype, device=x.device) if out is None else out
    _need(dw, "out", x.dtype)
    need = lib.dwconv1d_bwd_weight_workspace_size(B, T, C, K, pad_left, pad_right, dt)
    if need and workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=x.device)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    st = lib.dwconv1d_bwd_weight(_ptr(x), _ptr(dy), _ptr(dw), _ptr(workspace), ws_bytes, B, T,
                                 C, K, pad_left, pad_right, dt, _stream(stream))
    _check(st, "dwconv1d_bwd_weight")
    return dw


def dwconv1d_bwd_weight_noalloc(x, dy, K, pad_left, pad_right, out=None, stream=None):
    """dwconv1d_bwd_weight with the library's fixed device scratch instead of a workspace
    (for callers that cannot allocate device memory); see include/gconv.h."""
    lib = load_library()
    _need(x, "x")
    _need(dy, "dy", x.dtype)
    B, T, C = x.shape
    dw = torch.empty((C, K), dtype=x.dtype, device=x.device) if out is None else out
    _need(dw, "out", x.dtype)
    st = lib.dwconv1d_bwd_weight_noalloc(_ptr(x), _ptr(dy), _ptr(dw), B, T, C, K, pad_left,
                                         pad_right, _dtype_code(x.dtype), _stream(stream))
    _check(st, "dwconv1d_bwd_weight_noalloc")
    return dw


def dwsep1d_select_path(B, T, C, K, pad_left, pad_right, C_out, dtype, path=PATH_AUTO) -> int:
    """Kernel code (16 fused, 17 two launches) of a dwsep1d_fwd call, or a negative status."""
    dt = dtype if isinstance(dtype, int) else _dtype_code(dtype)
    return int(load_library().dwsep1d_select_path(B, T, C, K, pad_left, pad_right, C_out, dt,
                                                   path))


def dwsep1d_fwd(x, w_dw, w_pw, bias, pad_left, pad_right, out=None, workspace=None,
                path=PATH_AUTO, stream=None):
    """Depthwise-separable block on (batch, steps, channels): x [B, T, C], w_dw [C, K],
    w_pw [C_out, C], bias [C_out] or None -> z [B, T_out, C_out]."""
    lib = load_library()
    _need(x, "x")
    _need(w_dw, "w_dw", x.dtype)
    _need(w_pw, "w_pw", x.dtype)
    if bias is not None:
        _need(bias, "bias", x.dtype)
    B, T, C, K = _conv1d_dims(x, w_dw)
    C_out = w_pw.shape[0]
    if w_pw.dim() != 2 or w_pw.shape[1] != C:
        raise ValueError("w_pw must be [C_out, C] with the channel count of x")
    dt = _dtype_code(x.dtype)
    T_out = out_steps(B, T, C, K, pad_left, pad_right, dt)
    z = torch.empty((B, T_out, C_out), dtype=x.dtype, device=x.device) if out is None else out
    _need(z, "out", x.dtype)
    if tuple(z.shape) != (B, T_out, C_out):
        raise ValueError(f"out has shape {tuple(z.shape)}, expected {(B, T_out, C_out)}")
    need = lib.dwsep1d_fwd_workspace_size(B, T, C, K, pad_left, pad_right, C_out, dt, path)
    workspace, ws_bytes = _workspace(need, workspace, x.device)
    st = lib.dwsep1d_fwd(_ptr(x), _ptr(w_dw), _ptr(w_pw), _ptr(bias), _ptr(z), B, T, C, K,
                         pad_left, pad_right, C_out, dt, path, _ptr(workspace), ws_bytes,
                         _stream(stream))
    _check(st, "dwsep1d_fwd")
    return z


def dwsep2d_select_path(N, C, H, W, kH, kW, stride, padding, dilation, C_out, layout, dtype,
                        path=PATH_AUTO) -> int:
    """Kernel code (21 fused, 17 two launches) of a dwsep2d_fwd call, or a negative status."""
    dt = dtype if isinstance(dtype, int) else _dtype_code(dtype)
    return int(load_library().dwsep2d_select_path(N, C, H, W, kH, kW, stride, padding, dilation,
                                                   C_out, _layout_code(layout), dt, path))


def dwsep2d_fwd(x, w_dw, w_pw, bias=None, stride=1, padding=0, dilation=1, layout="NHWC",
                out=None, workspace=None, path=PATH_AUTO, stream=None):
    """2-D depthwise-separable block: x (NCHW or NHWC, C channels), w_dw the depthwise weight
    of that layout, w_pw [C_out, C], bias [C_out] or None -> z (C_out channels)."""
    lib = load_library()
    _need(x, "x")
    _need(w_dw, "w_dw", x.dtype)
    _need(w_pw, "w_pw", x.dtype)
    if bias is not None:
        _need(bias, "bias", x.dtype)
    lay, dims, y_shape = conv2d_dims(x, w_dw, stride, padding, dilation, x.shape[1 if
                                     _layout_code(layout) == NCHW else 3], layout)
    N, C, H, W, C2, kH, kW = dims
    C_out = w_pw.shape[0]
    if C2 != C or w_pw.dim() != 2 or w_pw.shape[1] != C:
        raise ValueError("w_dw must be the depthwise weight of x and w_pw [C_out, C]")
    dt = _dtype_code(x.dtype)
    z_shape = (N, C_out, y_shape[2], y_shape[3]) if lay == NCHW else (N, y_shape[1],
                                                                        y_shape[2], C_out)
    z = torch.empty(z_shape, dtype=x.dtype, device=x.device) if out is None else out
    _need(z, "out", x.dtype)
    if tuple(z.shape) != z_shape:
        raise ValueError(f"out has shape {tuple(z.shape)}, expected {z_shape}")
    need = lib.dwsep2d_fwd_workspace_size(N, C, H, W, kH, kW, stride, padding, dilation, C_out,
                                          lay, dt, path)
    workspace, ws_bytes = _workspace(need, workspace, x.device)
    st = lib.dwsep2d_fwd(_ptr(x), _ptr(w_dw), _ptr(w_pw), _ptr(bias), _ptr(z), N, C, H, W, kH,
                         kW, stride, padding, dilation, C_out, lay, dt, path, _ptr(workspace),
                         ws_bytes, _stream(stream))
    _check(st, "dwsep2d_fwd")
    return z


def device_error(stream=None) -> int:
    """Synchronise and read/clear the library's device error word (0 = none)."""
    code = ctypes.c_int(0)
    st = load_library().gconv_get_device_error(_stream(stream), ctypes.byref(code))
    if st not in (0, 6):
        raise GconvError(st, "gconv_get_device_error")
    return code.value
