"""GPU parity of the grouped conv2d backward pass (gconv2d_bwd_data, gconv2d_bwd_weight,
C ABI through the binding) against the fp64 oracle's gradients.

Small shapes cover every dispatch: the data gradient as a forward convolution (tensor cores,
depthwise, narrow-group, and NCHW tensor-core staging behind the flipped filter) and the
gather kernel (strides 2 / 3, pads above dil*(k-1), rectangular kernels, fp32); the weight
gradient on the depthwise kernel (3x3 / 5x5, strides 1 / 2) and the generic kernel. Exact
cases use integer-valued data. Full-size layers (the wide-group layer and the 56x56x1024
depthwise layer) are checked on sampled entries, and the weight gradient is checked to be
bitwise reproducible. Tolerances as for the forward: relative L2 <= 1e-5 (fp32) / 5e-3
(bf16, fp16), max|err| <= 1e-2 * max|ref|."""
import numpy as np
import pytest
import torch

import oracle
from depthwise_convolution_gconv2d_b200 import binding as gb
from depthwise_convolution_gconv2d_b200 import workloads as wl
from _util import assert_close, to_dev, to_f64

pytestmark = pytest.mark.gpu


def dgrad_kernel(p, path=gb.PATH_AUTO):
    return gb.gconv2d_bwd_data_select_path(p.N, p.C_in, p.H, p.W, p.C_out, p.kH, p.kW, p.stride,
                                           p.pad, p.dilation, p.groups, p.layout, p.dtype, path)


def wgrad_kernel(p, path=gb.PATH_AUTO):
    return gb.gconv2d_bwd_weight_select_path(p.N, p.C_in, p.H, p.W, p.C_out, p.kH, p.kW,
                                             p.stride, p.pad, p.dilation, p.groups, p.layout,
                                             p.dtype, path)


def inputs(p, seed, dist="normal"):
    inp = wl.make_conv2d_inputs(p, seed, dist, 1.0, dist, None if dist == "normal" else 1.0)
    dy = wl.make_conv2d_dy(p, seed, dist)
    return inp, dy


def gpu_dgrad(p, inp, dy, path=gb.PATH_AUTO):
    dx = gb.gconv2d_bwd_data(to_dev(dy, p.dtype), to_dev(inp.w, p.dtype), (p.H, p.W), p.stride,
                             p.pad, p.dilation, p.groups, p.layout, path=path)
    torch.cuda.synchronize()
    return dx


def gpu_wgrad(p, inp, dy, path=gb.PATH_AUTO):
    dw = gb.gconv2d_bwd_weight(to_dev(inp.x, p.dtype), to_dev(dy, p.dtype), (p.kH, p.kW),
                               p.stride, p.pad, p.dilation, p.groups, p.layout, path=path)
    torch.cuda.synchronize()
    return dw


def oracle_dgrad(p, inp, dy):
    return oracle.conv2d_bwd_data(wl.widen(dy, p.dtype), inp.w64(), (p.H, p.W), p.stride, p.pad,
                                  p.dilation, p.groups, p.layout)


def oracle_wgrad(p, inp, dy):
    return oracle.conv2d_bwd_weight(inp.x64(), wl.widen(dy, p.dtype), (p.kH, p.kW), p.stride,
                                    p.pad, p.dilation, p.groups, p.layout)


# (case, expected AUTO dgrad kernel, expected AUTO wgrad kernel) for NHWC bf16
CASES = [
    # N, C_in, H, W, C_out, kH, kW, stride, pad, dil, groups
    ((2, 64, 12, 12, 64, 3, 3, 1, 1, 1, 64), 2, 14),       # depthwise 3x3 s1
    ((2, 64, 13, 11, 64, 3, 3, 2, 1, 1, 64), 22, 14),      # depthwise 3x3 s2, ragged
    ((1, 32, 14, 9, 32, 5, 5, 1, 2, 1, 32), 2, 11),        # depthwise 5x5
    ((1, 32, 15, 16, 32, 5, 5, 2, 2, 1, 32), 12, 11),      # depthwise 5x5 s2
    ((2, 48, 10, 9, 48, 3, 3, 1, 0, 1, 48), 2, 14),        # depthwise, no padding (pad' = 2)
    ((2, 64, 9, 10, 64, 3, 3, 1, 1, 1, 16), 8, 10),        # narrow groups (4 ch)
    ((2, 128, 9, 24, 128, 3, 3, 1, 1, 1, 2), 3, 13),       # wide groups: tensor cores
    ((1, 64, 12, 16, 128, 3, 3, 1, 2, 2, 2), 3, 13),       # dilation 2, cpg_in != cpg_out
    ((1, 64, 7, 140, 64, 3, 3, 1, 1, 1, 1), 3, 13),        # W >= 128 (row kernels)
    ((2, 12, 9, 8, 18, 3, 2, 1, 1, 1, 3), 9, 10),          # rectangular kernel
    ((1, 16, 11, 10, 8, 3, 3, 3, 1, 1, 4), 9, 10),         # stride 3
    ((1, 8, 6, 7, 8, 3, 3, 1, 3, 1, 2), 9, 10),            # pad 3 > dil*(k-1)
    ((2, 16, 5, 6, 32, 1, 1, 2, 0, 1, 16), 9, 10),         # 1x1 stride 2, channel multiplier 2
    ((1, 16, 12, 13, 16, 7, 7, 2, 3, 1, 16), 12, 10),      # depthwise 7x7 s2 (4-byte vectors)
    ((2, 24, 9, 9, 24, 3, 3, 1, 3, 1, 24), 12, 11),        # depthwise, pad 3 > k-1
    ((1, 40, 11, 9, 40, 5, 5, 1, 5, 1, 40), 12, 11),       # depthwise 5x5, pad 5
    ((1, 80, 10, 11, 96, 3, 3, 1, 1, 1, 2), 9, 13),        # 40 -> 48 per group: ragged tiles
    ((2, 64, 11, 13, 64, 3, 3, 2, 1, 1, 1), 9, 13),        # tiled weight gradient, stride 2
    ((1, 160, 6, 7, 320, 3, 3, 1, 1, 1, 1), 3, 13),        # 160 -> 320: 3 x 2 tiles, ragged
    ((2, 72, 30, 31, 72, 3, 3, 1, 1, 1, 72), 2, 14),       # C % 64 != 0, Wo > 28 (2 column tiles)
    ((1, 40, 31, 30, 40, 3, 3, 2, 1, 1, 40), 22, 14),      # s2, odd sizes, ragged tiles
    ((2, 72, 18, 60, 72, 3, 3, 2, 1, 1, 72), 22, 14),      # s2: 3 column tiles, 2 channel tiles
    ((1, 64, 16, 16, 64, 3, 3, 2, 2, 1, 64), 12, 14),      # s2 with pad 2: gather kernel
    ((1, 16, 10, 10, 16, 3, 3, 1, 2, 1, 16), 2, 14),       # pad 2 (dgrad pad' = 0)
]


@pytest.mark.parametrize("case,kd,kw", CASES)
def test_bwd_small_nhwc(case, kd, kw):
    p = wl.Conv2dProblem(*case, layout=wl.NHWC, dtype=wl.BF16)
    assert dgrad_kernel(p) == kd and wgrad_kernel(p) == kw
    inp, dy = inputs(p, 31)
    assert_close(to_f64(gpu_dgrad(p, inp, dy)), oracle_dgrad(p, inp, dy), p.dtype, f"dx {case}")
    assert_close(to_f64(gpu_wgrad(p, inp, dy)), oracle_wgrad(p, inp, dy), p.dtype, f"dw {case}")
    assert gb.device_error() == 0


@pytest.mark.parametrize("case,kd,kw", CASES)
def test_bwd_generic_paths_nhwc(case, kd, kw):
    p = wl.Conv2dProblem(*case, layout=wl.NHWC, dtype=wl.BF16)
    inp, dy = inputs(p, 32)
    assert dgrad_kernel(p, gb.PATH_GENERIC) == 9 and wgrad_kernel(p, gb.PATH_GENERIC) == 10
    assert_close(to_f64(gpu_dgrad(p, inp, dy, gb.PATH_GENERIC)), oracle_dgrad(p, inp, dy),
                 p.dtype, f"dx {case}")
    assert_close(to_f64(gpu_wgrad(p, inp, dy, gb.PATH_GENERIC)), oracle_wgrad(p, inp, dy),
                 p.dtype, f"dw {case}")


@pytest.mark.parametrize("case,kd,kw", CASES[5:])
def test_bwd_small_nchw(case, kd, kw):
    p = wl.Conv2dProblem(*case, layout=wl.NCHW, dtype=wl.BF16)
    inp, dy = inputs(p, 33)
    assert dgrad_kernel(p) == (4 if kd == 3 else 9)
    assert wgrad_kernel(p) == (15 if kw == 13 else 10)
    assert_close(to_f64(gpu_dgrad(p, inp, dy)), oracle_dgrad(p, inp, dy), p.dtype, f"dx {case}")
    assert_close(to_f64(gpu_wgrad(p, inp, dy)), oracle_wgrad(p, inp, dy), p.dtype, f"dw {case}")


@pytest.mark.parametrize("case,kd,kw", CASES[:2] + CASES[5:8])
def test_bwd_fp16(case, kd, kw):
    p = wl.Conv2dProblem(*case, layout=wl.NHWC, dtype=wl.F16)
    inp, dy = inputs(p, 34)
    assert_close(to_f64(gpu_dgrad(p, inp, dy)), oracle_dgrad(p, inp, dy), p.dtype, f"dx {case}")
    assert_close(to_f64(gpu_wgrad(p, inp, dy)), oracle_wgrad(p, inp, dy), p.dtype, f"dw {case}")


@pytest.mark.parametrize("groups", [4, 8, 1])
@pytest.mark.parametrize("layout", [wl.NCHW, wl.NHWC])
def test_bwd_tiny_fp32(groups, layout):
    """The fp32 workload shape (x [2, 8, 16, 16], 3x3, pad 1): generic kernels, 1e-5."""
    p = wl.tiny_grouped(groups, layout)
    inp, dy = inputs(p, 35, "uniform")
    assert dgrad_kernel(p) == 9
    assert_close(to_f64(gpu_dgrad(p, inp, dy)), oracle_dgrad(p, inp, dy), p.dtype, "dx")
    assert_close(to_f64(gpu_wgrad(p, inp, dy)), oracle_wgrad(p, inp, dy), p.dtype, "dw")


@pytest.mark.parametrize("case,kd,kw", [CASES[0], CASES[1], CASES[5], CASES[6], CASES[13]])
@pytest.mark.parametrize("path", [gb.PATH_AUTO, gb.PATH_GENERIC])
def test_bwd_integer_bit_exact(case, kd, kw, path):
    """x, w, dy in {-2..2}: every product and partial sum is an integer below 2^24, exact in
    fp32 whatever the summation order, so the result is the exact sum rounded once to bf16
    (which leaves |v| <= 256 unchanged)."""
    p = wl.Conv2dProblem(*case, layout=wl.NHWC, dtype=wl.BF16)
    inp, dy = inputs(p, 36, "int")
    rnd = lambda a: wl.widen(wl.to_storage(a, wl.BF16), wl.BF16)
    ref_dx, ref_dw = oracle_dgrad(p, inp, dy), oracle_wgrad(p, inp, dy)
    assert np.max(np.abs(ref_dx)) < 2 ** 24 and np.max(np.abs(ref_dw)) < 2 ** 24
    assert np.array_equal(to_f64(gpu_dgrad(p, inp, dy, path)), rnd(ref_dx))
    assert np.array_equal(to_f64(gpu_wgrad(p, inp, dy, path)), rnd(ref_dw))


def test_dgrad_delta_filter_is_identity():
    """Depthwise centre-tap filter: dx == dy bit for bit (stride 1, pad 1)."""
    p = wl.Conv2dProblem(2, 64, 9, 11, 64, 3, 3, 1, 1, 1, 64, wl.NHWC, wl.BF16)
    inp, dy = inputs(p, 37)
    w = np.zeros((64, 3, 3, 1))
    w[:, 1, 1, 0] = 1.0
    inp.w = wl.to_storage(w, wl.BF16)
    assert np.array_equal(to_f64(gpu_dgrad(p, inp, dy)), wl.widen(dy, wl.BF16))


def test_wgrad_deterministic_and_n0():
    p = wl.Conv2dProblem(4, 64, 20, 20, 64, 3, 3, 1, 1, 1, 64, wl.NHWC, wl.BF16)
    inp, dy = inputs(p, 38)
    a = gpu_wgrad(p, inp, dy)
    b = gpu_wgrad(p, inp, dy)
    assert torch.equal(a.view(torch.int16), b.view(torch.int16))
    pg = wl.Conv2dProblem(2, 16, 9, 9, 24, 3, 3, 1, 1, 1, 4, wl.NHWC, wl.BF16)
    inp, dy = inputs(pg, 38)
    a = gpu_wgrad(pg, inp, dy)
    b = gpu_wgrad(pg, inp, dy)
    assert torch.equal(a.view(torch.int16), b.view(torch.int16))
    # N = 0: dw is zero, dx is empty
    x0 = torch.empty((0, 9, 9, 16), dtype=torch.bfloat16, device="cuda")
    dy0 = torch.empty((0, 9, 9, 24), dtype=torch.bfloat16, device="cuda")
    dw = torch.full((24, 3, 3, 4), 7.0, dtype=torch.bfloat16, device="cuda")
    gb.gconv2d_bwd_weight(x0, dy0, (3, 3), 1, 1, 1, 4, "NHWC", out=dw)
    torch.cuda.synchronize()
    assert torch.count_nonzero(dw).item() == 0
    w = torch.zeros((24, 3, 3, 4), dtype=torch.bfloat16, device="cuda")
    assert gb.gconv2d_bwd_data(dy0, w, (9, 9), 1, 1, 1, 4, "NHWC").shape == (0, 9, 9, 16)


def test_dgrad_igemm_forced_and_unsupported():
    p = wl.Conv2dProblem(1, 64, 8, 16, 64, 3, 3, 1, 1, 1, 2, wl.NHWC, wl.BF16)
    inp, dy = inputs(p, 39)
    assert dgrad_kernel(p, gb.PATH_IGEMM) == 3
    assert_close(to_f64(gpu_dgrad(p, inp, dy, gb.PATH_IGEMM)), oracle_dgrad(p, inp, dy), p.dtype)
    q = wl.Conv2dProblem(1, 64, 8, 16, 64, 3, 3, 2, 1, 1, 2, wl.NHWC, wl.BF16)
    assert dgrad_kernel(q, gb.PATH_IGEMM) == -2
    assert wgrad_kernel(p, gb.PATH_IGEMM) == -2


# ------------------------------------------------------------ full-size layers, sampled

def sample_x_indices(p, n, seed):
    r = np.random.default_rng(seed)
    idx = np.stack([r.integers(0, p.N, n), r.integers(0, p.C_in, n), r.integers(0, p.H, n),
                    r.integers(0, p.W, n)], 1)
    edges = [(nn, c, h, w) for nn in (0, p.N - 1) for c in (0, p.C_in - 1)
             for h in (0, 1, p.H - 1) for w in (0, 1, p.W - 1)]
    return np.concatenate([idx, np.array(edges)], 0)


def gather_x(dx, idx, layout):
    n, c, h, w = (torch.from_numpy(idx[:, i]).to(dx.device) for i in range(4))
    return to_f64(dx[n, c, h, w] if layout == wl.NCHW else dx[n, h, w, c])


@pytest.mark.parametrize("p", [wl.depthwise_56(1), wl.depthwise_56(2), wl.wide_group(wl.NHWC),
                               wl.wide_group(wl.NCHW)],
                         ids=["depthwise56_s1", "depthwise56_s2", "wide_nhwc", "wide_nchw"])
def test_dgrad_full_size_sampled(p):
    inp, dy = inputs(p, 40)
    dx = gpu_dgrad(p, inp, dy)
    idx = sample_x_indices(p, 6000, 41)
    ref = oracle.conv2d_bwd_data_points(wl.widen(dy, p.dtype), inp.w64(), (p.H, p.W), idx,
                                        p.stride, p.pad, p.dilation, p.groups, p.layout)
    assert_close(gather_x(dx, idx, p.layout), ref, p.dtype, str(p))
    assert gb.device_error() == 0


@pytest.mark.parametrize("stride", [1, 2])
def test_wgrad_depthwise56_full(stride):
    """All 1024 x 9 entries of the 56x56x1024 depthwise layer's weight gradient."""
    p = wl.depthwise_56(stride)
    assert wgrad_kernel(p) == 14
    inp, dy = inputs(p, 42)
    got = to_f64(gpu_wgrad(p, inp, dy))
    assert_close(got, oracle_wgrad(p, inp, dy), p.dtype, str(p))


def test_wgrad_wide_group_sampled():
    p = wl.wide_group(wl.NHWC)
    inp, dy = inputs(p, 43)
    dw = gpu_wgrad(p, inp, dy)
    r = np.random.default_rng(44)
    n = 600
    idx = np.stack([r.integers(0, p.C_out, n), r.integers(0, p.cpg_in, n),
                    r.integers(0, 3, n), r.integers(0, 3, n)], 1)
    ref = oracle.conv2d_bwd_weight_points(inp.x64(), wl.widen(dy, p.dtype), (3, 3), idx,
                                          p.stride, p.pad, p.dilation, p.groups, p.layout)
    t = [torch.from_numpy(idx[:, i]).to(dw.device) for i in range(4)]
    got = to_f64(dw[t[0], t[2], t[3], t[1]])
    assert_close(got, ref, p.dtype, "wide-group dw")


# ------------------------------------------------------------ tensor-core weight gradient

TC_WGRAD_CASES = [
    # N, C_in, H, W, C_out, kH, kW, stride, pad, dil, groups
    (2, 256, 10, 40, 256, 3, 3, 1, 1, 1, 2),      # 128 / 128, one partial 128-pixel segment
    (1, 128, 6, 130, 256, 3, 3, 1, 1, 1, 1),      # 256 filters: two filter blocks; ragged rows
    (1, 192, 5, 64, 128, 5, 5, 1, 2, 1, 1),       # 5x5: 64-channel blocks (3 of them)
    (2, 128, 8, 36, 128, 3, 3, 1, 2, 2, 1),       # dilation 2
    (1, 64, 9, 48, 128, 1, 1, 1, 0, 1, 1),        # 1x1
    (1, 128, 7, 33, 128, 3, 1, 1, 1, 1, 1),       # 3x1
    (3, 256, 4, 34, 512, 3, 3, 1, 0, 1, 4),       # 4 groups, no padding (Wo = 32)
]


@pytest.mark.parametrize("case", TC_WGRAD_CASES)
@pytest.mark.parametrize("layout", [wl.NHWC, wl.NCHW])
def test_wgrad_tensor_cores(case, layout):
    p = wl.Conv2dProblem(*case, layout=layout, dtype=wl.BF16)
    assert wgrad_kernel(p) == (18 if layout == wl.NHWC else 19)
    inp, dy = inputs(p, 45)
    assert_close(to_f64(gpu_wgrad(p, inp, dy)), oracle_wgrad(p, inp, dy), p.dtype, f"dw {case}")
    assert gb.device_error() == 0


def test_wgrad_tensor_cores_fp16_and_forced_paths():
    p = wl.Conv2dProblem(2, 256, 10, 40, 256, 3, 3, 1, 1, 1, 2, wl.NHWC, wl.F16)
    inp, dy = inputs(p, 46)
    ref = oracle_wgrad(p, inp, dy)
    assert_close(to_f64(gpu_wgrad(p, inp, dy)), ref, p.dtype, "fp16")
    assert wgrad_kernel(p, gb.PATH_IGEMM) == 18 and wgrad_kernel(p, gb.PATH_DIRECT) == 13
    assert_close(to_f64(gpu_wgrad(p, inp, dy, gb.PATH_IGEMM)), ref, p.dtype, "forced IGEMM")
    assert_close(to_f64(gpu_wgrad(p, inp, dy, gb.PATH_DIRECT)), ref, p.dtype, "CUDA cores")


def test_wgrad_tensor_cores_integer_exact_and_deterministic():
    """Integer-valued data: every partial sum is an exact integer in fp32, so the slices'
    fixed-order sum is exact and dw equals the oracle's value rounded to bf16; two calls give
    the same bits."""
    p = wl.Conv2dProblem(2, 256, 10, 40, 256, 3, 3, 1, 1, 1, 2, wl.NHWC, wl.BF16)
    inp, dy = inputs(p, 47, "int")
    assert wgrad_kernel(p) == 18
    a = gpu_wgrad(p, inp, dy)
    b = gpu_wgrad(p, inp, dy)
    assert torch.equal(a.view(torch.int16), b.view(torch.int16))
    rnd = lambda v: wl.widen(wl.to_storage(v, wl.BF16), wl.BF16)
    assert np.array_equal(to_f64(a), rnd(oracle_wgrad(p, inp, dy)))


def test_wgrad_wide_group_sampled_nchw():
    p = wl.wide_group(wl.NCHW)
    assert wgrad_kernel(p) == 19
    inp, dy = inputs(p, 48)
    dw = gpu_wgrad(p, inp, dy)
    r = np.random.default_rng(49)
    n = 400
    idx = np.stack([r.integers(0, p.C_out, n), r.integers(0, p.cpg_in, n),
                    r.integers(0, 3, n), r.integers(0, 3, n)], 1)
    ref = oracle.conv2d_bwd_weight_points(inp.x64(), wl.widen(dy, p.dtype), (3, 3), idx,
                                          p.stride, p.pad, p.dilation, p.groups, p.layout)
    t = [torch.from_numpy(idx[:, i]).to(dw.device) for i in range(4)]
    got = to_f64(dw[t[0], t[1], t[2], t[3]])
    assert_close(got, ref, p.dtype, "wide-group dw, NCHW")
