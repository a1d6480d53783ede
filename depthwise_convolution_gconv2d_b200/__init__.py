"""Grouped and depthwise convolution for NVIDIA B200 (sm_100a).

The compute lives in ``libgconv.so`` (hand-written CUDA behind a C ABI, declared in
``include/gconv.h``). This package is the thin Python binding over that ABI:
``gconv2d_fwd``, ``dwconv1d_fwd``, ``dwconv1d_bwd_data``, ``dwconv1d_bwd_weight`` and
helpers, taking torch CUDA tensors and passing their device pointers, sizes and the
current stream. Nothing here computes a convolution.

Attributes of the binding load the shared library on first use (so that
``depthwise_convolution_gconv2d_b200.workloads`` can be imported without it); a missing
or unloadable library raises ``RuntimeError`` -- there is no fallback path.
"""
from __future__ import annotations

__all__ = [
    "gconv2d_fwd", "gconv2d_fwd_workspace_size", "gconv2d_select_path",
    "dwconv1d_fwd", "dwconv1d_bwd_data", "dwconv1d_bwd_weight",
    "dwconv1d_bwd_weight_workspace_size", "library_path", "load_library",
]


def __getattr__(name):
    if name in __all__ or name in ("NCHW", "NHWC", "PATH_AUTO", "PATH_DIRECT", "PATH_IGEMM",
                                   "PATH_GENERIC", "GconvError"):
        import importlib
        return getattr(importlib.import_module(".binding", __name__), name)
    raise AttributeError(name)
