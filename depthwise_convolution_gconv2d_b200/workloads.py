"""Seeded synthetic inputs for the convolution workloads.

This module only draws random numbers and rounds them to the storage dtype; it holds
none of the convolution arithmetic. Both the CUDA path (through the tests and the
benchmark) and the fp64 oracle receive exactly the arrays produced here: the GPU gets
the storage bits, the oracle gets the same values widened to float64.

Seeds: workload k draws with ``numpy.random.default_rng(1000*k + role)``, role 0 = x,
1 = w, 2 = bias, 3 = dy (upstream gradient). Values are drawn in fp64, in the logical
NCHW / [C_out, C_in/g, kH, kW] order, rounded to the dtype (round-to-nearest-even), and
then permuted into the requested memory layout, so the NCHW and NHWC variants of a
workload hold the same logical tensors.

Workloads (shapes of the pages' layers; see ``WORKLOADS``):
  1  tiny grouped conv2d, fp32, NCHW, x[2,8,16,16], w[8,8/g,3,3], g in {4, 8, 1}
  2  wide-group conv2d x[1,512,256,256], w[512,128,3,3], g=4, bf16 -- the layer timed in
     "F.conv2d runs x15 slower in mixed-precision/half-precision mode"
  3  Conformer depthwise conv1d x[8,2048,512] on (batch, steps, channels), K=31, bf16
  4  ensemble-as-groups conv2d x[64,2048,32,32], w[4096,32,3,3], g=64, bf16, NHWC
  5  depthwise conv2d x[32,1024,56,56], w[1024,1,3,3], bf16, NHWC, stride 1 and 2, plus a
     groups sweep g in {1024, 256, 64, 16}
"""
from __future__ import annotations

import dataclasses

from typing import Optional

import numpy as np

NCHW = 0
NHWC = 1
F32 = 0
F16 = 1
BF16 = 2

DTYPE_NAMES = {F32: "f32", F16: "f16", BF16: "bf16"}
ROLE = {"x": 0, "w": 1, "bias": 2, "dy": 3}


def seed_for(workload: int, role: str) -> int:
    return 1000 * int(workload) + ROLE[role]


# ----------------------------------------------------------------------------- rounding

def f32_to_bf16_bits(a) -> np.ndarray:
    """Round float values to bfloat16 (nearest-even); returns the uint16 bit patterns."""
    f = np.ascontiguousarray(a, dtype=np.float32)
    u = f.view(np.uint32).astype(np.uint64)
    rounded = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    return rounded.astype(np.uint16)


def bf16_bits_to_f64(bits) -> np.ndarray:
    b = np.ascontiguousarray(bits, dtype=np.uint16)
    return (b.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def to_storage(a64, dtype: int) -> np.ndarray:
    """fp64 values -> storage array: float32 for F32, uint16 bit patterns for F16/BF16."""
    if dtype == F32:
        return np.ascontiguousarray(a64, dtype=np.float32)
    if dtype == F16:
        return np.ascontiguousarray(np.asarray(a64, dtype=np.float16)).view(np.uint16)
    if dtype == BF16:
        return f32_to_bf16_bits(np.asarray(a64, dtype=np.float32))
    raise ValueError(f"unknown dtype {dtype}")


def widen(storage, dtype: int) -> np.ndarray:
    """Storage array -> the exact values it holds, as float64."""
    if dtype == F32:
        return np.asarray(storage, dtype=np.float32).astype(np.float64)
    if dtype == F16:
        return np.ascontiguousarray(storage, dtype=np.uint16).view(np.float16).astype(np.float64)
    if dtype == BF16:
        return bf16_bits_to_f64(storage)
    raise ValueError(f"unknown dtype {dtype}")


def elem_size(dtype: int) -> int:
    return 4 if dtype == F32 else 2


# ----------------------------------------------------------------------------- drawing

def draw(rng: np.random.Generator, shape, dist: str, scale: float = 1.0) -> np.ndarray:
    """fp64 draw: 'normal' N(0, scale^2), 'uniform' U[-scale, scale], 'int' in {-2..2}."""
    if dist == "normal":
        return rng.standard_normal(shape) * scale
    if dist == "uniform":
        return rng.uniform(-scale, scale, shape)
    if dist == "int":
        return rng.integers(-2, 3, shape).astype(np.float64)
    raise ValueError(f"unknown distribution {dist}")


@dataclasses.dataclass(frozen=True)
class Conv2dProblem:
    N: int
    C_in: int
    H: int
    W: int
    C_out: int
    kH: int
    kW: int
    stride: int = 1
    pad: int = 0
    dilation: int = 1
    groups: int = 1
    layout: int = NCHW
    dtype: int = F32
    bias: bool = False

    @property
    def cpg_in(self) -> int:
        return self.C_in // self.groups

    @property
    def cpg_out(self) -> int:
        return self.C_out // self.groups

    def _ext(self, size, k):
        span = size + 2 * self.pad - self.dilation * (k - 1) - 1
        return span // self.stride + 1 if span >= 0 else 0

    @property
    def Ho(self) -> int:
        return self._ext(self.H, self.kH)

    @property
    def Wo(self) -> int:
        return self._ext(self.W, self.kW)

    @property
    def x_shape(self):
        return (self.N, self.C_in, self.H, self.W) if self.layout == NCHW else (
            self.N, self.H, self.W, self.C_in)

    @property
    def w_shape(self):
        return (self.C_out, self.cpg_in, self.kH, self.kW) if self.layout == NCHW else (
            self.C_out, self.kH, self.kW, self.cpg_in)

    @property
    def y_shape(self):
        return (self.N, self.C_out, self.Ho, self.Wo) if self.layout == NCHW else (
            self.N, self.Ho, self.Wo, self.C_out)

    def flops(self) -> int:
        """2 * N * Ho * Wo * C_out * (C_in/g) * kH * kW (padded taps counted)."""
        return 2 * self.N * self.Ho * self.Wo * self.C_out * self.cpg_in * self.kH * self.kW

    def bytes(self) -> int:
        """Algorithmic bytes: read x and w once (+bias), write y once."""
        e = elem_size(self.dtype)
        n = self.N * self.C_in * self.H * self.W + self.C_out * self.cpg_in * self.kH * self.kW
        n += self.N * self.C_out * self.Ho * self.Wo + (self.C_out if self.bias else 0)
        return n * e


@dataclasses.dataclass
class Conv2dInputs:
    problem: Conv2dProblem
    x: np.ndarray          # storage, memory layout of problem.layout
    w: np.ndarray
    bias: np.ndarray | None

    def x64(self):
        return widen(self.x, self.problem.dtype)

    def w64(self):
        return widen(self.w, self.problem.dtype)

    def bias64(self):
        return None if self.bias is None else widen(self.bias, self.problem.dtype)


def make_conv2d_inputs(p: Conv2dProblem, workload: int, x_dist="normal", x_scale=1.0,
                       w_dist="normal", w_scale=None, bias_scale=1.0) -> Conv2dInputs:
    """Seeded x, w (and bias when p.bias) for a conv2d problem.

    Default w scale is 1/sqrt(C_in/g * kH * kW), i.e. w ~ N(0, 1/(cpg_in*kH*kW))."""
    if w_scale is None:
        w_scale = 1.0 / np.sqrt(p.cpg_in * p.kH * p.kW)
    x64 = draw(np.random.default_rng(seed_for(workload, "x")), (p.N, p.C_in, p.H, p.W),
               x_dist, x_scale)
    x = to_storage(x64, p.dtype)
    del x64
    w = to_storage(draw(np.random.default_rng(seed_for(workload, "w")),
                        (p.C_out, p.cpg_in, p.kH, p.kW), w_dist, w_scale), p.dtype)
    if p.layout == NHWC:
        x = np.ascontiguousarray(x.transpose(0, 2, 3, 1))
        w = np.ascontiguousarray(w.transpose(0, 2, 3, 1))
    b = None
    if p.bias:
        b = to_storage(draw(np.random.default_rng(seed_for(workload, "bias")), (p.C_out,),
                            x_dist if x_dist != "normal" else "uniform", bias_scale), p.dtype)
    return Conv2dInputs(p, x, w, b)


def make_conv2d_dy(p: Conv2dProblem, workload: int, dist="normal", scale=1.0) -> np.ndarray:
    """Seeded output gradient dy ~ N(0, scale^2) (or `dist`), storage array in p's y layout."""
    dy = to_storage(draw(np.random.default_rng(seed_for(workload, "dy")),
                         (p.N, p.C_out, p.Ho, p.Wo), dist, scale), p.dtype)
    if p.layout == NHWC:
        dy = np.ascontiguousarray(dy.transpose(0, 2, 3, 1))
    return dy


@dataclasses.dataclass(frozen=True)
class Dwconv1dProblem:
    B: int
    T: int
    C: int
    K: int
    pad_left: int
    pad_right: int
    dtype: int = BF16

    @property
    def T_out(self) -> int:
        return self.T + self.pad_left + self.pad_right - self.K + 1

    def flops(self) -> int:
        """2 * B * T_out * C * K for each of fwd, dgrad and wgrad."""
        return 2 * self.B * self.T_out * self.C * self.K

    def bytes(self, op: str) -> int:
        """Algorithmic bytes: fwd x+w+y, dgrad dy+w+dx, wgrad x+dy+dw."""
        e = elem_size(self.dtype)
        bt = self.B * self.T * self.C
        bto = self.B * self.T_out * self.C
        ck = self.C * self.K
        return e * {"fwd": bt + ck + bto, "dgrad": bto + ck + bt, "wgrad": bt + bto + ck}[op]


@dataclasses.dataclass
class Dwconv1dInputs:
    problem: Dwconv1dProblem
    x: np.ndarray      # [B, T, C] storage
    w: np.ndarray      # [C, K]
    dy: np.ndarray     # [B, T_out, C]


def make_dwconv1d_inputs(p: Dwconv1dProblem, workload: int, dist="normal") -> Dwconv1dInputs:
    """x ~ N(0,1), w ~ N(0, 1/K), dy ~ N(0,1) (or integer-valued for dist='int')."""
    x = to_storage(draw(np.random.default_rng(seed_for(workload, "x")), (p.B, p.T, p.C), dist),
                   p.dtype)
    w = to_storage(draw(np.random.default_rng(seed_for(workload, "w")), (p.C, p.K), dist,
                        1.0 / np.sqrt(p.K)), p.dtype)
    dy = to_storage(draw(np.random.default_rng(seed_for(workload, "dy")), (p.B, p.T_out, p.C),
                         dist), p.dtype)
    return Dwconv1dInputs(p, x, w, dy)


@dataclasses.dataclass
class DwsepInputs:
    """Depthwise-separable block (depthwise conv1d, then pointwise 1x1 over channels)."""
    problem: Dwconv1dProblem
    C_out: int
    x: np.ndarray      # [B, T, C] storage
    w_dw: np.ndarray   # [C, K]
    w_pw: np.ndarray   # [C_out, C]
    bias: Optional[np.ndarray]   # [C_out] or None

    def x64(self):
        return widen(self.x, self.problem.dtype)

    def w_dw64(self):
        return widen(self.w_dw, self.problem.dtype)

    def w_pw64(self):
        return widen(self.w_pw, self.problem.dtype)

    def bias64(self):
        return None if self.bias is None else widen(self.bias, self.problem.dtype)


def make_dwsep1d_inputs(p: Dwconv1dProblem, C_out: int, workload: int, bias: bool = True,
                        dist="normal") -> DwsepInputs:
    """x ~ N(0,1), w_dw ~ N(0, 1/K), w_pw ~ N(0, 1/C), bias ~ N(0,1) (integer-valued for
    dist='int'); the same seeds roles as the other workloads (w_pw takes the 'dy' role)."""
    x = to_storage(draw(np.random.default_rng(seed_for(workload, "x")), (p.B, p.T, p.C), dist),
                   p.dtype)
    w_dw = to_storage(draw(np.random.default_rng(seed_for(workload, "w")), (p.C, p.K), dist,
                           1.0 / np.sqrt(p.K)), p.dtype)
    w_pw = to_storage(draw(np.random.default_rng(seed_for(workload, "dy")), (C_out, p.C), dist,
                           1.0 / np.sqrt(p.C)), p.dtype)
    b = None
    if bias:
        b = to_storage(draw(np.random.default_rng(seed_for(workload, "bias")), (C_out,), dist),
                       p.dtype)
    return DwsepInputs(p, C_out, x, w_dw, w_pw, b)


# ----------------------------------------------------------------------------- workloads

def tiny_grouped(groups: int, layout=NCHW, dtype=F32, bias=False) -> Conv2dProblem:
    return Conv2dProblem(2, 8, 16, 16, 8, 3, 3, 1, 1, 1, groups, layout, dtype, bias)


def wide_group(layout=NHWC, dtype=BF16) -> Conv2dProblem:
    return Conv2dProblem(1, 512, 256, 256, 512, 3, 3, 1, 1, 1, 4, layout, dtype)


def conformer_dw1d(causal: bool = False, dtype=BF16) -> Dwconv1dProblem:
    return Dwconv1dProblem(8, 2048, 512, 31, 30 if causal else 15, 0 if causal else 15, dtype)


def ensemble_groups(layout=NHWC, dtype=BF16) -> Conv2dProblem:
    return Conv2dProblem(64, 2048, 32, 32, 4096, 3, 3, 1, 1, 1, 64, layout, dtype)


def depthwise_56(stride: int = 1, groups: int = 1024, layout=NHWC, dtype=BF16) -> Conv2dProblem:
    return Conv2dProblem(32, 1024, 56, 56, 1024, 3, 3, stride, 1, 1, groups, layout, dtype)


def grouped_linear(tokens: int = 16384, features: int = 4096, groups: int = 4, layout=NHWC,
                   dtype=BF16) -> Conv2dProblem:
    """Grouped linear layer y_g = x_g W_g^T: the grouped conv2d with H = W = 1 and a 1x1
    kernel, one image per token (the batched-GEMM form of grouping)."""
    return Conv2dProblem(tokens, features, 1, 1, features, 1, 1, 1, 0, 1, groups, layout, dtype)


WORKLOADS = {
    "tiny_grouped_g4": (1, lambda: tiny_grouped(4)),
    "tiny_grouped_g8": (1, lambda: tiny_grouped(8)),
    "tiny_grouped_g1": (1, lambda: tiny_grouped(1)),
    "wide_group_nhwc": (2, lambda: wide_group(NHWC)),
    "wide_group_nchw": (2, lambda: wide_group(NCHW)),
    "conformer_dw1d_same": (3, lambda: conformer_dw1d(False)),
    "conformer_dw1d_causal": (3, lambda: conformer_dw1d(True)),
    "ensemble_g64_nhwc": (4, lambda: ensemble_groups()),
    "depthwise56_s1": (5, lambda: depthwise_56(1)),
    "depthwise56_s2": (5, lambda: depthwise_56(2)),
    "sweep56_g256": (5, lambda: depthwise_56(1, 256)),
    "sweep56_g64": (5, lambda: depthwise_56(1, 64)),
    "sweep56_g16": (5, lambda: depthwise_56(1, 16)),
    "grouped_linear": (6, lambda: grouped_linear()),
    "conformer_dwsep1d": (7, lambda: conformer_dw1d(False)),
}
