"""GPU parity of the output variants of "Grouped convolutions" (neon issue #296, ibmua's post
on output orderings): the interleaved channel order 1234... and the average / maximum merge
across groups, written by the kernels' epilogues through gconv2d_fwd_out, against the fp64
oracle's oracle_conv2d_interleaved / oracle_conv2d_group_merge (pinned on the CPU to the
page's printed order and to numpy reshapes / means / maxima of the group-major output).

Cases: the tensor-core tile kernel (several filter-block widths, ragged tiles, bias, NHWC
and NCHW, fp16), the transposed row-strip kernel for the interleaved order, the generic
direct kernel (fp32 at 1e-5, and forced), exact integer cases (a permutation, a maximum and
a power-of-two mean of exact sums are exact), the modes that reduce to the plain output, and
the wide-group layer on sampled outputs."""
import numpy as np
import pytest
import torch

import oracle
from depthwise_convolution_gconv2d_b200 import binding as gb
from depthwise_convolution_gconv2d_b200 import workloads as wl
from _util import assert_close, to_dev, to_f64

pytestmark = pytest.mark.gpu

MODES = ["interleaved", "avg", "max"]


def run_out(inp, mode, path=gb.PATH_AUTO):
    p = inp.problem
    y = gb.gconv2d_fwd_out(to_dev(inp.x, p.dtype), to_dev(inp.w, p.dtype),
                           to_dev(inp.bias, p.dtype), p.stride, p.pad, p.dilation, p.groups,
                           p.layout, mode, path=path)
    torch.cuda.synchronize()
    return y


def oracle_out(inp, mode):
    p = inp.problem
    if mode == "interleaved":
        return oracle.conv2d_interleaved(inp.x64(), inp.w64(), inp.bias64(), p.stride, p.pad,
                                         p.dilation, p.groups, p.layout)
    return oracle.conv2d_group_merge(inp.x64(), inp.w64(), inp.bias64(), p.stride, p.pad,
                                     p.dilation, p.groups, p.layout, mode)


def kernel_of(p, mode, path=gb.PATH_AUTO):
    return gb.gconv2d_fwd_out_select_path(p.N, p.C_in, p.H, p.W, p.C_out, p.kH, p.kW, p.stride,
                                          p.pad, p.dilation, p.groups, p.layout, p.dtype, mode,
                                          path)


TC_CASES = [
    # N, C_in, H, W, C_out, k, pad, groups       (cpg_in / cpg_out)
    (2, 128, 10, 12, 128, 3, 1, 2),        # 64 / 64
    (1, 64, 9, 7, 96, 3, 1, 2),            # 32 / 48: merge blocks of 16
    (2, 64, 6, 20, 256, 3, 1, 4),          # 16 / 64
    (1, 256, 5, 9, 512, 1, 0, 2),          # 1x1, 128 / 256: merge blocks of 64, 4 per tile
    (1, 96, 7, 130, 96, 3, 1, 3),          # 32 / 32, rows wider than one tile
    (2, 64, 12, 16, 128, 5, 2, 4),         # 5x5, 16 / 32
]


@pytest.mark.parametrize("case", TC_CASES)
@pytest.mark.parametrize("mode", MODES)
@pytest.mark.parametrize("layout", [wl.NHWC, wl.NCHW])
def test_variants_tensor_cores(case, mode, layout):
    N, Ci, H, W, Co, k, pad, g = case
    p = wl.Conv2dProblem(N, Ci, H, W, Co, k, k, 1, pad, 1, g, layout, wl.BF16, bias=True)
    assert kernel_of(p, mode) in (3, 4)
    inp = wl.make_conv2d_inputs(p, 31)
    assert_close(to_f64(run_out(inp, mode)), oracle_out(inp, mode), p.dtype, f"{case} {mode}")


@pytest.mark.parametrize("mode", MODES)
def test_variants_fp16(mode):
    p = wl.Conv2dProblem(2, 64, 8, 8, 64, 3, 3, 1, 1, 1, 2, wl.NHWC, wl.F16, bias=True)
    inp = wl.make_conv2d_inputs(p, 32)
    assert_close(to_f64(run_out(inp, mode)), oracle_out(inp, mode), p.dtype, mode)


@pytest.mark.parametrize("mode", ["interleaved", "avg"])
def test_row_strip_kernel_variants(mode):
    """Rows of >= 128 outputs with 128k filters per group take the transposed row-strip
    kernel: its epilogue writes each filter to its interleaved channel, and for the average
    merge one tile runs every group's K loop into one accumulator and scales it by 1/groups."""
    for layout in (wl.NHWC, wl.NCHW):
        for g in (2, 4):
            p = wl.Conv2dProblem(1, 128 * g, 4, 160, 128 * g, 3, 3, 1, 1, 1, g, layout, wl.BF16,
                                 bias=True)
            inp = wl.make_conv2d_inputs(p, 33)
            assert_close(to_f64(run_out(inp, mode)), oracle_out(inp, mode), p.dtype,
                         f"layout {layout} groups {g}")


GENERIC_CASES = [
    # N, C_in, H, W, C_out, kH, kW, stride, pad, dil, groups
    (2, 8, 9, 7, 12, 3, 3, 1, 1, 1, 4),
    (1, 6, 11, 13, 9, 3, 2, 2, 1, 1, 3),
    (2, 4, 7, 7, 8, 5, 5, 1, 2, 2, 2),
]


@pytest.mark.parametrize("case", GENERIC_CASES)
@pytest.mark.parametrize("mode", MODES)
@pytest.mark.parametrize("layout", [wl.NCHW, wl.NHWC])
def test_variants_generic_fp32(case, mode, layout):
    p = wl.Conv2dProblem(*case, layout=layout, dtype=wl.F32, bias=True)
    assert kernel_of(p, mode) == 1
    inp = wl.make_conv2d_inputs(p, 34, "uniform", 1.0, "uniform", 1.0)
    assert_close(to_f64(run_out(inp, mode)), oracle_out(inp, mode), p.dtype, f"{case} {mode}")


@pytest.mark.parametrize("mode", MODES)
def test_variants_generic_forced_16bit(mode):
    p = wl.Conv2dProblem(2, 64, 8, 8, 64, 3, 3, 1, 1, 1, 2, wl.NHWC, wl.BF16, bias=True)
    assert kernel_of(p, mode, gb.PATH_GENERIC) == 1
    inp = wl.make_conv2d_inputs(p, 35)
    assert_close(to_f64(run_out(inp, mode, gb.PATH_GENERIC)), oracle_out(inp, mode), p.dtype,
                 mode)


@pytest.mark.parametrize("mode", MODES)
@pytest.mark.parametrize("path", [gb.PATH_AUTO, gb.PATH_GENERIC])
def test_variants_integer_bit_exact(mode, path):
    """Integer-valued data: every sum is exact in fp32, and so are the permutation, the
    maximum and the mean over 4 groups (a power of two); the GPU equals the oracle bit for
    bit, tile edges and group offsets included."""
    p = wl.Conv2dProblem(2, 64, 9, 11, 128, 3, 3, 1, 1, 1, 4, wl.NHWC, wl.BF16)
    inp = wl.make_conv2d_inputs(p, 36, "int", 1.0, "int", 1.0)
    got = to_f64(run_out(inp, mode, path))
    assert np.array_equal(got, oracle_out(inp, mode))


def test_modes_that_equal_the_plain_output():
    """One filter per group (depthwise) makes the interleaved order the group-major one, and
    one group makes every merge the plain output: both run the ordinary kernels."""
    p = wl.Conv2dProblem(2, 64, 14, 14, 64, 3, 3, 1, 1, 1, 64, wl.NHWC, wl.BF16)
    assert kernel_of(p, "interleaved") == 2
    inp = wl.make_conv2d_inputs(p, 37)
    ref = oracle.conv2d(inp.x64(), inp.w64(), None, 1, 1, 1, 64, p.layout)
    assert_close(to_f64(run_out(inp, "interleaved")), ref, p.dtype, "depthwise interleaved")
    q = wl.Conv2dProblem(1, 64, 10, 10, 64, 3, 3, 1, 1, 1, 1, wl.NHWC, wl.BF16)
    inq = wl.make_conv2d_inputs(q, 38)
    ref = oracle.conv2d(inq.x64(), inq.w64(), None, 1, 1, 1, 1, q.layout)
    for mode in ("avg", "max"):
        assert_close(to_f64(run_out(inq, mode)), ref, q.dtype, f"one group, {mode}")


def _sample(p, n, seed, channels):
    r = np.random.default_rng(seed)
    return np.stack([r.integers(0, p.N, n), r.integers(0, channels, n), r.integers(0, p.Ho, n),
                     r.integers(0, p.Wo, n)], 1)


# The max merge in two passes (the transposed row-strip kernel writes the group-major output
# to the workspace, then the maximum over groups): problems that tiling takes (64 input
# channels a group or a multiple, 128 filters a group or a multiple, rows of >= 128 outputs).
MAX_TWO_PASS = [
    # N, C_in, H, W, C_out, k, pad, groups
    (1, 128, 4, 136, 256, 3, 1, 2),
    (2, 256, 3, 130, 512, 3, 1, 4),
    (1, 192, 5, 128, 384, 3, 2, 3),
]


@pytest.mark.parametrize("case", MAX_TWO_PASS)
@pytest.mark.parametrize("layout", [wl.NHWC, wl.NCHW])
@pytest.mark.parametrize("dtype", [wl.BF16, wl.F16])
def test_max_merge_two_pass(case, layout, dtype):
    N, C_in, H, W, C_out, k, pad, g = case
    p = wl.Conv2dProblem(N, C_in, H, W, C_out, k, k, 1, pad, 1, g, layout, dtype, True)
    assert kernel_of(p, "max") == 23 and kernel_of(p, "max", gb.PATH_IGEMM) == 23
    assert kernel_of(p, "max", gb.PATH_DIRECT) == 1
    assert gb.load_library().gconv2d_fwd_out_workspace_size(
        N, C_in, H, W, C_out, k, k, 1, pad, 1, g, layout, dtype, 3, 0) >= \
        N * C_out * p.Ho * p.Wo * 2
    inp = wl.make_conv2d_inputs(p, 61)
    y = run_out(inp, "max")
    assert gb.device_error() == 0
    assert_close(to_f64(y), oracle_out(inp, "max"), p.dtype, f"{case} {layout}")


def test_max_merge_two_pass_integer_bit_exact():
    """Ternary x and sparse ternary filters (at most 255 non-zero taps): every group's sum is
    an exact integer below 256, so the maximum over groups is exact and equals the oracle's."""
    p = wl.Conv2dProblem(1, 128, 4, 136, 256, 3, 3, 1, 1, 1, 2, wl.NHWC, wl.BF16, False)
    r = np.random.default_rng(62)
    inp = wl.make_conv2d_inputs(p, 62)
    w = r.integers(-1, 2, p.w_shape) * (r.random(p.w_shape) < 1 / 8)
    assert np.abs(w).reshape(p.C_out, -1).sum(axis=1).max() <= 255
    inp.x = wl.to_storage(r.integers(-1, 2, p.x_shape), wl.BF16)
    inp.w = wl.to_storage(w, wl.BF16)
    assert np.array_equal(to_f64(run_out(inp, "max")), oracle_out(inp, "max"))


@pytest.mark.parametrize("mode", MODES)
def test_variants_wide_group_layer_sampled(mode):
    """The wide-group layer x[1,512,256,256] * w[512,128,3,3], groups 4 (NHWC), in each
    variant, on sampled outputs: the oracle computes the group-major points the variant
    reads, and the interleave / mean / maximum of them is taken here."""
    p = wl.wide_group(wl.NHWC)
    inp = wl.make_conv2d_inputs(p, 2)
    y = run_out(inp, mode)
    cpg, g = p.cpg_out, p.groups
    nsamp = 4000
    if mode == "interleaved":
        idx = _sample(p, nsamp, 39, p.C_out)
        src = idx.copy()
        src[:, 1] = (idx[:, 1] % g) * cpg + idx[:, 1] // g
        ref = oracle.conv2d_points(inp.x64(), inp.w64(), src, None, 1, 1, 1, g, p.layout)
    else:
        idx = _sample(p, nsamp // g, 40, cpg)
        vals = []
        for i in range(g):
            src = idx.copy()
            src[:, 1] = i * cpg + idx[:, 1]
            vals.append(oracle.conv2d_points(inp.x64(), inp.w64(), src, None, 1, 1, 1, g,
                                             p.layout))
        vals = np.stack(vals, 0)
        ref = vals.mean(0) if mode == "avg" else vals.max(0)
    n, c, ho, wo = (torch.from_numpy(idx[:, k]).to(y.device) for k in range(4))
    assert_close(to_f64(y[n, ho, wo, c]), ref, p.dtype, mode)
