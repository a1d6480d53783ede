"""GPU parity of the tcgen05 implicit-GEMM path (gconv2d_fwd, GCONV_PATH_IGEMM and AUTO)
against the fp64 oracle: small shapes covering every tile/swizzle variant (channel blocks of
16/32/64, filters per group 16..256 and > 256, ragged image edges, W > 128, 1x1 / 5x5 /
dilated filters, bias, fp16), exact cases (integer data, delta filters), the wide-group layer
(NHWC and NCHW) and the ensemble-as-groups layer at full size on sampled outputs, and the
ensemble checked against separate dense convs per model."""
import numpy as np
import pytest
import torch

import oracle
from depthwise_convolution_gconv2d_b200 import binding as gb
from depthwise_convolution_gconv2d_b200 import workloads as wl
from _util import assert_close, to_dev, to_f64
from test_parity_conv2d import check_sampled, gather, kernel_of, oracle_full, run_gpu

pytestmark = pytest.mark.gpu

SMALL = [
    # N, C_in, H, W, C_out, k, pad, dil, groups      (cpg_in / cpg_out)
    (1, 32, 8, 8, 32, 3, 1, 1, 2),           # 16 / 16: 32-byte rows, N = 16
    (2, 128, 20, 24, 128, 3, 1, 1, 2),       # 64 / 64
    (1, 64, 9, 7, 96, 3, 1, 1, 2),           # 32 / 48
    (2, 64, 12, 12, 64, 1, 0, 1, 1),         # 1x1
    (1, 32, 11, 13, 64, 5, 2, 1, 1),         # 5x5, 32 / 64
    (1, 64, 10, 10, 64, 3, 2, 2, 2),         # dilation 2
    (1, 256, 5, 130, 512, 3, 1, 1, 1),       # W > 128 (two column tiles), 512 filters (4 N tiles)
    (3, 128, 7, 56, 256, 3, 1, 1, 1),        # 56-wide rows: 112-row tiles; N = 256
    (1, 64, 3, 3, 32, 3, 0, 1, 1),           # single output pixel
    (2, 48, 6, 6, 48, 3, 1, 1, 3),           # 16 / 16 with three groups
    (1, 128, 4, 140, 192, 3, 1, 1, 2),       # row-strip kernel: Wo >= 128, 96 filters per group
    (2, 128, 3, 300, 256, 3, 1, 1, 2),       # transposed row kernel, 2 segments per row
    (1, 64, 6, 140, 128, 3, 2, 2, 1),        # transposed row kernel with dilation 2
    (1, 64, 7, 131, 128, 5, 2, 1, 1),        # transposed row kernel, 5x5
    (1, 64, 12, 16, 64, 3, 2, 2, 2),         # halo tile kernel: Wo = 16, dilation 2
    (2, 96, 9, 32, 96, 5, 2, 1, 3),          # halo tile kernel: 5x5, 32 / 32
    (1, 128, 5, 40, 64, 3, 1, 1, 2),         # halo tile kernel: 64-channel blocks, 3-row tiles
    (2, 128, 9, 24, 128, 3, 1, 1, 2),        # halo: 64 filters a group (TMA-store epilogue), 5-row tiles, ragged
    (1, 64, 6, 16, 256, 3, 1, 1, 2),         # halo: 128 filters a group (two 64-channel stores)
    (2, 64, 8, 16, 64, 3, 1, 1, 2),          # halo, 2 groups packed (32 -> 32 ch): N = 64
    (1, 64, 6, 24, 64, 3, 1, 1, 4),          # halo, 4 groups packed (16 -> 16 ch): N = 64
    (1, 128, 5, 8, 64, 5, 2, 1, 4),          # halo, 2 groups packed, N = 32, 5x5
]


def problem(case, layout=wl.NHWC, dtype=wl.BF16, bias=False):
    N, C_in, H, W, C_out, k, pad, dil, g = case
    return wl.Conv2dProblem(N, C_in, H, W, C_out, k, k, 1, pad, dil, g, layout, dtype, bias)


@pytest.mark.parametrize("case", SMALL)
def test_igemm_small_nhwc(case):
    p = problem(case, bias=True)
    assert kernel_of(p, gb.PATH_IGEMM) == 3
    inp = wl.make_conv2d_inputs(p, 21)
    y = run_gpu(inp, gb.PATH_IGEMM)
    assert gb.device_error() == 0
    assert_close(to_f64(y), oracle_full(inp), p.dtype, str(case))


@pytest.mark.parametrize("case", SMALL[:6] + SMALL[10:])
def test_igemm_small_nchw(case):
    p = problem(case, wl.NCHW, bias=True)
    assert kernel_of(p, gb.PATH_IGEMM) == 4
    inp = wl.make_conv2d_inputs(p, 22)
    y = run_gpu(inp, gb.PATH_IGEMM)
    assert_close(to_f64(y), oracle_full(inp), p.dtype, str(case))


# NCHW problems on the transposed row-strip kernel (through the NHWC staging copy): several
# images and groups, two row segments, dilation, 5x5 with rows outside a 3-row image, the
# wide-group layer's channels on two rows.
NCHW_ROWT = [
    # N, C_in, H, W, C_out, k, pad, dil, groups
    (2, 128, 5, 136, 256, 3, 1, 1, 2),
    (1, 256, 4, 264, 256, 3, 1, 1, 2),
    (1, 128, 6, 128, 128, 3, 2, 2, 1),
    (3, 64, 3, 200, 128, 5, 2, 1, 1),
    (1, 512, 2, 256, 512, 3, 1, 1, 4),
]


@pytest.mark.parametrize("case", NCHW_ROWT)
@pytest.mark.parametrize("dtype", [wl.BF16, wl.F16])
def test_igemm_nchw_rowt(case, dtype):
    p = problem(case, wl.NCHW, dtype=dtype, bias=True)
    assert kernel_of(p, gb.PATH_IGEMM) == 4
    inp = wl.make_conv2d_inputs(p, 23)
    y = run_gpu(inp, gb.PATH_IGEMM)
    assert gb.device_error() == 0
    assert_close(to_f64(y), oracle_full(inp), p.dtype, str(case))


@pytest.mark.parametrize("case", NCHW_ROWT[::2])
def test_igemm_nchw_rowt_integer_bit_exact(case):
    """x in {-1, 0, 1}, sparse filters in {-1, 0, 1} with at most 255 non-zero taps each: every
    sum is an exact integer below 256, exact in bf16, so the NCHW -> NHWC staging and every tap
    must give the oracle's value bit for bit."""
    p = problem(case, wl.NCHW)
    r = np.random.default_rng(25)
    inp = wl.make_conv2d_inputs(p, 24)
    w = r.integers(-1, 2, p.w_shape) * (r.random(p.w_shape) < 1 / 16)
    assert np.abs(w).reshape(p.C_out, -1).sum(axis=1).max() <= 255
    inp.x = wl.to_storage(r.integers(-1, 2, p.x_shape), wl.BF16)
    inp.w = wl.to_storage(w, wl.BF16)
    y = run_gpu(inp, gb.PATH_IGEMM)
    assert np.array_equal(to_f64(y), oracle_full(inp))


@pytest.mark.parametrize("case", SMALL[:4])
def test_igemm_fp16(case):
    p = problem(case, dtype=wl.F16)
    inp = wl.make_conv2d_inputs(p, 23)
    assert_close(to_f64(run_gpu(inp, gb.PATH_IGEMM)), oracle_full(inp), p.dtype, str(case))


@pytest.mark.parametrize("case", [SMALL[0], SMALL[2], SMALL[9]])
def test_igemm_integer_bit_exact(case):
    """x, w in {-1, 0, 1} with at most 16*9 terms: every partial sum is an exact integer and
    the result (|.| <= 144) is exact in bf16, so the tensor-core result equals the oracle."""
    p = problem(case)
    r = np.random.default_rng(24)
    inp = wl.make_conv2d_inputs(p, 24)
    inp.x = wl.to_storage(r.integers(-1, 2, p.x_shape), wl.BF16)
    inp.w = wl.to_storage(r.integers(-1, 2, p.w_shape), wl.BF16)
    assert p.cpg_in * p.kH * p.kW <= 256 or case == SMALL[2]
    got, ref = to_f64(run_gpu(inp, gb.PATH_IGEMM)), oracle_full(inp)
    if p.cpg_in * p.kH * p.kW <= 255:
        assert np.array_equal(got, ref)
    else:
        assert_close(got, ref, p.dtype)


@pytest.mark.parametrize("layout", [wl.NHWC, wl.NCHW])
def test_igemm_delta_filter_is_exact_identity(layout):
    """Per group, filter co has a single 1 at (ci = co % cpg, centre tap): y == x bit for bit,
    which pins the tap-shifted loads, the zero fill at the borders and the group offsets."""
    g, cpg = 4, 32
    p = wl.Conv2dProblem(2, g * cpg, 9, 11, g * cpg, 3, 3, 1, 1, 1, g, layout, wl.BF16)
    inp = wl.make_conv2d_inputs(p, 25)
    w = np.zeros((p.C_out, cpg, 3, 3))
    for co in range(p.C_out):
        w[co, co % cpg, 1, 1] = 1.0
    if layout == wl.NHWC:
        w = w.transpose(0, 2, 3, 1)
    inp.w = wl.to_storage(w, wl.BF16)
    got = to_f64(run_gpu(inp, gb.PATH_IGEMM))
    assert np.array_equal(got, inp.x64())


def test_igemm_offcentre_delta_shift():
    """Tap (0, 2) with pad 1: y[h, w] = x[h-1, w+1], zero where that leaves the image."""
    g, cpg = 2, 16
    p = wl.Conv2dProblem(1, g * cpg, 6, 7, g * cpg, 3, 3, 1, 1, 1, g, wl.NHWC, wl.BF16)
    inp = wl.make_conv2d_inputs(p, 26)
    w = np.zeros((p.C_out, 3, 3, cpg))
    for co in range(p.C_out):
        w[co, 0, 2, co % cpg] = 1.0
    inp.w = wl.to_storage(w, wl.BF16)
    got = to_f64(run_gpu(inp, gb.PATH_IGEMM))
    x = inp.x64()
    ref = np.zeros_like(x)
    ref[:, 1:, :-1, :] = x[:, :-1, 1:, :]
    assert np.array_equal(got, ref)


def test_auto_picks_tensor_cores_for_wide_groups():
    assert kernel_of(wl.wide_group(wl.NHWC)) == 3
    assert kernel_of(wl.wide_group(wl.NCHW)) == 4
    assert kernel_of(wl.ensemble_groups()) == 3
    assert kernel_of(wl.depthwise_56(1, 64)) == 3
    assert kernel_of(wl.depthwise_56(1, 16)) == 3
    assert kernel_of(wl.depthwise_56(1, 256)) == 8   # 4 channels per group: CUDA cores
    assert kernel_of(wl.depthwise_56(1, 1024)) == 2


@pytest.mark.parametrize("layout", [wl.NHWC, wl.NCHW])
def test_wide_group_full_size_sampled(layout):
    check_sampled(wl.wide_group(layout), 2)


def test_ensemble_full_size_sampled_and_per_model():
    """The groups = 64 layer (64 models x 32 -> 64 channels) against the oracle, and the same
    sampled outputs against model m's own dense conv on its 32-channel slice."""
    p = wl.ensemble_groups()
    y = check_sampled(p, 4, 4000)
    inp = wl.make_conv2d_inputs(p, 4)
    x64, w64 = inp.x64(), inp.w64()
    r = np.random.default_rng(27)
    for m in r.choice(64, 4, replace=False):
        xm = np.ascontiguousarray(x64[..., 32 * m:32 * (m + 1)])
        wm = np.ascontiguousarray(w64[64 * m:64 * (m + 1)])
        idx = np.stack([r.integers(0, 64, 500), r.integers(0, 64, 500), r.integers(0, 32, 500),
                        r.integers(0, 32, 500)], 1)
        ref = oracle.conv2d_points(xm, wm, idx, None, 1, 1, 1, 1, wl.NHWC)
        gidx = idx.copy()
        gidx[:, 1] += 64 * m
        assert_close(gather(y, gidx, wl.NHWC), ref, wl.BF16, f"model {m}")


@pytest.mark.parametrize("groups", [64, 16])
def test_groups_sweep_igemm_sampled(groups):
    check_sampled(wl.depthwise_56(1, groups), 5, 5000, gb.PATH_IGEMM)


def test_no_device_error_left():
    assert gb.device_error() == 0
