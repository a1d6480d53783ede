"""GPU parity of the grouped linear layer (y_g = x_g W_g^T + b_g per group, the fully
connected form of grouping that "Grouped convolutions" (neon issue #296) discusses next to
batched GEMM) run through gconv2d_fwd as a 1x1 convolution of 1x1 images, against the fp64
oracle, which a CPU test pins to the per-group matmul. The library runs pointwise problems
as one wide image of all pixels on the tensor cores, so the cases cover the three tile
kernels that then apply (transposed row: 128k filters per group; row: 64-channel blocks;
tile: narrow groups), bias, fp16, ragged token counts, NCHW, and the benchmark's layer on
sampled outputs."""
import numpy as np
import pytest
import torch

import oracle
from depthwise_convolution_gconv2d_b200 import binding as gb
from depthwise_convolution_gconv2d_b200 import workloads as wl
from _util import assert_close, to_dev, to_f64
from test_parity_conv2d import check_sampled, kernel_of, oracle_full, run_gpu

pytestmark = pytest.mark.gpu

CASES = [
    # tokens, features in, features out, groups
    (1000, 512, 512, 2),      # 256 / 256 per group: transposed row kernel
    (300, 256, 256, 4),       # 64 / 64: row kernel
    (40, 96, 96, 3),          # 32 / 32: tile kernel, one partial tile
    (7, 64, 128, 4),          # 16 / 32, fewer tokens than a tile row
    (70000, 128, 128, 2),     # tokens > 65535: factorised into a 2-D pixel grid
]


@pytest.mark.parametrize("case", CASES)
@pytest.mark.parametrize("dtype", [wl.BF16, wl.F16])
def test_grouped_linear_small(case, dtype):
    T, Ci, Co, g = case
    p = wl.Conv2dProblem(T, Ci, 1, 1, Co, 1, 1, 1, 0, 1, g, wl.NHWC, dtype, bias=True)
    assert kernel_of(p) == 3
    inp = wl.make_conv2d_inputs(p, 17)
    y = run_gpu(inp)
    ref = oracle_full(inp)
    assert_close(to_f64(y), ref, dtype, str(case))
    # the same numbers as per-group matmuls of the widened inputs
    x = inp.x64().reshape(T, g, Ci // g)
    w = inp.w64().reshape(g, Co // g, Ci // g)
    mm = np.einsum("tgc,goc->tgo", x, w).reshape(T, Co) + inp.bias64()[None, :]
    assert_close(to_f64(y).reshape(T, Co), mm, dtype, f"{case} vs matmul")


def test_grouped_linear_integer_bit_exact():
    """Integer-valued inputs: every partial sum is exact in fp32, so any summation order
    gives the oracle's value bit for bit (tile edges, group offsets, token flattening)."""
    p = wl.Conv2dProblem(333, 256, 1, 1, 256, 1, 1, 1, 0, 1, 2, wl.NHWC, wl.BF16)
    inp = wl.make_conv2d_inputs(p, 18, "int", 1.0, "int", 1.0)
    got = to_f64(run_gpu(inp))
    assert np.array_equal(got, oracle_full(inp))


@pytest.mark.parametrize("N", [1, 5])
def test_grouped_linear_nchw(N):
    """NCHW activations [N, C, 1, 1] hold the same bytes as NHWC [N, 1, 1, C]."""
    p = wl.Conv2dProblem(N, 128, 1, 1, 256, 1, 1, 1, 0, 1, 4, wl.NCHW, wl.BF16, bias=True)
    inp = wl.make_conv2d_inputs(p, 19)
    assert_close(to_f64(run_gpu(inp)), oracle_full(inp), p.dtype, f"N={N}")


def test_pointwise_conv_across_images():
    """A 1x1 convolution on real images is the same flattened GEMM: tiles then run across
    image rows and image boundaries (NHWC, and one NCHW image)."""
    for layout, N in ((wl.NHWC, 3), (wl.NCHW, 1)):
        p = wl.Conv2dProblem(N, 128, 9, 21, 256, 1, 1, 1, 0, 1, 2, layout, wl.BF16, bias=True)
        inp = wl.make_conv2d_inputs(p, 20)
        assert_close(to_f64(run_gpu(inp)), oracle_full(inp), p.dtype, f"layout {layout}")


def test_grouped_linear_layer_sampled():
    """The benchmark's layer, x[16384, 4096] -> [16384, 4096] in 4 groups, on sampled
    outputs the oracle computes one by one."""
    p = wl.grouped_linear()
    assert kernel_of(p) == 3
    check_sampled(p, 6, 20000)
