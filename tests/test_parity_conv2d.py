"""GPU parity of gconv2d_fwd (C ABI through the binding) against the fp64 oracle.

Same seeded inputs on both sides; tolerances relative L2 <= 1e-5 (fp32) / 5e-3 (bf16, fp16)
and max|err| <= 1e-2 * max|ref|; bit-exact where the arithmetic is exact (integer-valued
data, delta kernels). Full-size workloads are checked on sampled outputs that the oracle
computes one by one, in the same launch configuration the benchmark times."""
import numpy as np
import pytest
import torch

import oracle
from depthwise_convolution_gconv2d_b200 import binding as gb
from depthwise_convolution_gconv2d_b200 import workloads as wl
from _util import assert_close, to_dev, to_f64

pytestmark = pytest.mark.gpu


def run_gpu(inp, path=gb.PATH_AUTO, out=None):
    p = inp.problem
    y = gb.gconv2d_fwd(to_dev(inp.x, p.dtype), to_dev(inp.w, p.dtype), to_dev(inp.bias, p.dtype),
                       p.stride, p.pad, p.dilation, p.groups, p.layout, out=out, path=path)
    torch.cuda.synchronize()
    return y


def oracle_full(inp):
    p = inp.problem
    return oracle.conv2d(inp.x64(), inp.w64(), inp.bias64(), p.stride, p.pad, p.dilation,
                         p.groups, p.layout)


def kernel_of(p, path=gb.PATH_AUTO):
    return gb.gconv2d_select_path(p.N, p.C_in, p.H, p.W, p.C_out, p.kH, p.kW, p.stride, p.pad,
                                  p.dilation, p.groups, p.layout, p.dtype, path)


# ------------------------------------------------------------ tiny grouped conv, fp32

@pytest.mark.parametrize("groups", [4, 8, 1])
@pytest.mark.parametrize("layout", [wl.NCHW, wl.NHWC])
def test_tiny_grouped_fp32(groups, layout):
    p = wl.tiny_grouped(groups, layout)
    inp = wl.make_conv2d_inputs(p, 1, "uniform", 1.0, "uniform", 1.0)
    assert kernel_of(p) == 1
    assert_close(to_f64(run_gpu(inp)), oracle_full(inp), p.dtype, f"g={groups}")


@pytest.mark.parametrize("groups", [4, 8, 1])
def test_tiny_grouped_fp32_integer_bit_exact(groups):
    p = wl.tiny_grouped(groups, wl.NCHW, bias=True)
    inp = wl.make_conv2d_inputs(p, 1, "int", 1.0, "int", 1.0)
    inp.bias = np.array([1, -2, 0, 2, -1, 1, 2, -2], np.float32)
    got = to_f64(run_gpu(inp))
    assert np.array_equal(got, oracle_full(inp))


# ------------------------------------------------------------ generic kernel, 16-bit

GENERIC_CASES = [
    # N, C_in, H, W, C_out, kH, kW, stride, pad, dil, groups
    (2, 6, 9, 7, 9, 3, 3, 1, 1, 1, 3),
    (1, 8, 11, 13, 4, 3, 2, 2, 1, 1, 2),
    (3, 4, 7, 7, 8, 5, 5, 1, 2, 2, 4),
    (1, 12, 5, 17, 12, 1, 3, 1, 0, 1, 12),
    (2, 16, 10, 10, 32, 3, 3, 2, 0, 1, 16),   # depthwise channel multiplier 2
    (1, 3, 4, 4, 5, 3, 3, 1, 2, 1, 1),
]


@pytest.mark.parametrize("case", GENERIC_CASES)
@pytest.mark.parametrize("layout", [wl.NCHW, wl.NHWC])
@pytest.mark.parametrize("dtype", [wl.BF16, wl.F16])
def test_generic_16bit(case, layout, dtype):
    p = wl.Conv2dProblem(*case, layout=layout, dtype=dtype, bias=True)
    inp = wl.make_conv2d_inputs(p, 11)
    y = run_gpu(inp, gb.PATH_GENERIC)
    assert_close(to_f64(y), oracle_full(inp), dtype, str(case))


# ------------------------------------------------------------ depthwise NHWC vector kernel

DW_CASES = [
    # N, C, H, W, k, stride, pad, dil
    (2, 64, 9, 11, 3, 1, 1, 1),
    (1, 24, 7, 30, 3, 2, 1, 1),
    (3, 520, 6, 5, 3, 1, 1, 1),       # more than one channel block, ragged
    (1, 40, 13, 9, 5, 1, 2, 1),
    (2, 16, 12, 12, 5, 2, 2, 1),
    (1, 30, 9, 10, 7, 1, 3, 1),
    (1, 14, 15, 8, 7, 2, 3, 1),
    (2, 32, 10, 10, 3, 1, 2, 2),      # dilation: no sliding window
    (1, 8, 1, 1, 3, 1, 1, 1),         # 1x1 image, everything padding but the centre
    (1, 256, 3, 300, 3, 1, 0, 1),     # no padding, wide
    (1, 128, 5, 29, 3, 1, 1, 1),      # one output column past a 28-column tile
    (2, 64, 9, 59, 3, 2, 1, 1),       # stride 2: two column tiles, ragged 2-row tiles
    (1, 72, 4, 57, 3, 2, 2, 1),       # stride 2, pad 2
]


@pytest.mark.parametrize("case", DW_CASES)
@pytest.mark.parametrize("dtype", [wl.BF16, wl.F16])
def test_depthwise_nhwc(case, dtype):
    N, C, H, W, k, s, pd, d = case
    p = wl.Conv2dProblem(N, C, H, W, C, k, k, s, pd, d, C, wl.NHWC, dtype, bias=True)
    assert kernel_of(p) == 2
    inp = wl.make_conv2d_inputs(p, 12)
    assert_close(to_f64(run_gpu(inp)), oracle_full(inp), dtype, str(case))


@pytest.mark.parametrize("case", DW_CASES[:6])
def test_depthwise_nhwc_integer_bit_exact(case):
    N, C, H, W, k, s, pd, d = case
    p = wl.Conv2dProblem(N, C, H, W, C, k, k, s, pd, d, C, wl.NHWC, wl.BF16)
    inp = wl.make_conv2d_inputs(p, 13, "int", 1.0, "int", 1.0)
    assert np.array_equal(to_f64(run_gpu(inp)), oracle_full(inp))


# ------------------------------------------------------------ narrow groups (2 / 4 / 8 channels)

NG_CASES = [
    # N, C, H, W, stride, pad, groups          (channels per group = C / groups)
    (2, 64, 9, 30, 1, 1, 16),       # 4 per group, two column tiles (28 + 2)
    (1, 64, 7, 29, 1, 1, 32),       # 2 per group
    (2, 128, 6, 12, 1, 1, 16),      # 8 per group, two channel tiles
    (1, 64, 9, 59, 2, 1, 16),       # stride 2, ragged 2-row tiles
    (1, 72, 5, 9, 1, 1, 18),        # C = 72: the second channel tile holds 8 channels
    (1, 64, 8, 10, 2, 2, 16),       # stride 2, pad 2
    (3, 32, 5, 5, 1, 0, 8),         # no padding, tiny image
]


@pytest.mark.parametrize("case", NG_CASES)
@pytest.mark.parametrize("dtype", [wl.BF16, wl.F16])
def test_narrow_groups_nhwc(case, dtype):
    N, C, H, W, st, pd, g = case
    p = wl.Conv2dProblem(N, C, H, W, C, 3, 3, st, pd, 1, g, wl.NHWC, dtype, bias=True)
    assert kernel_of(p) == 8
    inp = wl.make_conv2d_inputs(p, 15)
    assert_close(to_f64(run_gpu(inp)), oracle_full(inp), dtype, str(case))


@pytest.mark.parametrize("case", NG_CASES[:4])
def test_narrow_groups_integer_bit_exact(case):
    """x, w in {-1, 0, 1}: at most 72 terms per output, every partial sum exact in fp32 and the
    result exact in bf16, so any order of the sum gives the oracle's value bit for bit."""
    N, C, H, W, st, pd, g = case
    p = wl.Conv2dProblem(N, C, H, W, C, 3, 3, st, pd, 1, g, wl.NHWC, wl.BF16)
    r = np.random.default_rng(16)
    inp = wl.make_conv2d_inputs(p, 16)
    inp.x = wl.to_storage(r.integers(-1, 2, p.x_shape), wl.BF16)
    inp.w = wl.to_storage(r.integers(-1, 2, p.w_shape), wl.BF16)
    assert np.array_equal(to_f64(run_gpu(inp)), oracle_full(inp))


@pytest.mark.parametrize("kh,kw", [(1, 1), (0, 2), (2, 0), (2, 2)])
def test_depthwise_delta_kernel_is_exact_shift(kh, kw):
    """A delta tap at (kh, kw) with pad 1 gives y[h, w] = x[h + kh - 1, w + kw - 1] with zero
    fill, bit for bit: the padding and halo logic."""
    N, C, H, W = 2, 72, 9, 13
    p = wl.Conv2dProblem(N, C, H, W, C, 3, 3, 1, 1, 1, C, wl.NHWC, wl.BF16)
    inp = wl.make_conv2d_inputs(p, 14)
    w = np.zeros((C, 3, 3, 1), np.float64)
    w[:, kh, kw, 0] = 1.0
    inp.w = wl.to_storage(w, wl.BF16)
    got = to_f64(run_gpu(inp))
    x = inp.x64()
    ref = np.zeros_like(x)
    dh, dw = kh - 1, kw - 1
    hs, ws = slice(max(0, -dh), H - max(0, dh)), slice(max(0, -dw), W - max(0, dw))
    hd, wd = slice(max(0, dh), H - max(0, -dh)), slice(max(0, dw), W - max(0, -dw))
    ref[:, hs, ws, :] = x[:, hd, wd, :]
    assert np.array_equal(got, ref)


def test_misaligned_pointer_takes_generic_path():
    """An output pointer that is not 16-byte aligned cannot use the vector kernel; AUTO
    still produces the right answer (generic kernel), forcing IGEMM reports it."""
    p = wl.Conv2dProblem(1, 64, 8, 8, 64, 3, 3, 1, 1, 1, 64, wl.NHWC, wl.BF16)
    inp = wl.make_conv2d_inputs(p, 15)
    buf = torch.empty(64 * 8 * 8 + 1, dtype=torch.bfloat16, device="cuda")
    out = buf[1:].view(1, 8, 8, 64)
    y = run_gpu(inp, out=out)
    assert_close(to_f64(y), oracle_full(inp), wl.BF16)


def test_output_guard_bands_untouched():
    p = wl.Conv2dProblem(2, 64, 9, 9, 64, 3, 3, 2, 1, 1, 64, wl.NHWC, wl.BF16)
    inp = wl.make_conv2d_inputs(p, 16)
    n = int(np.prod(p.y_shape))
    guard = 4096
    buf = torch.full((n + 2 * guard,), float("nan"), dtype=torch.bfloat16, device="cuda")
    sentinel = buf[:guard].clone().view(torch.int16)
    out = buf[guard:guard + n].view(p.y_shape)
    for path in (gb.PATH_AUTO, gb.PATH_GENERIC):
        run_gpu(inp, path, out=out)
        assert torch.equal(buf[:guard].view(torch.int16), sentinel)
        assert torch.equal(buf[guard + n:].view(torch.int16), sentinel)
        assert_close(to_f64(out), oracle_full(inp), wl.BF16)


# ------------------------------------------------------------ full-size workloads, sampled

def sample_indices(p, n, seed):
    r = np.random.default_rng(seed)
    idx = np.stack([r.integers(0, p.N, n), r.integers(0, p.C_out, n), r.integers(0, p.Ho, n),
                    r.integers(0, p.Wo, n)], 1)
    # always include the four corners and the edges of the first and last image
    corners = []
    for nn in (0, p.N - 1):
        for co in (0, p.C_out - 1, p.C_out // 2):
            for ho in (0, p.Ho - 1):
                for wo in (0, p.Wo - 1, p.Wo // 2):
                    corners.append((nn, co, ho, wo))
    return np.concatenate([idx, np.array(corners)], 0)


def gather(y, idx, layout):
    n, co, ho, wo = (torch.from_numpy(idx[:, i]).to(y.device) for i in range(4))
    v = y[n, co, ho, wo] if layout == wl.NCHW else y[n, ho, wo, co]
    return to_f64(v)


def check_sampled(p, workload, nsamp=20000, path=gb.PATH_AUTO):
    inp = wl.make_conv2d_inputs(p, workload)
    y = run_gpu(inp, path)
    idx = sample_indices(p, nsamp, workload)
    ref = oracle.conv2d_points(inp.x64(), inp.w64(), idx, inp.bias64(), p.stride, p.pad,
                               p.dilation, p.groups, p.layout)
    assert_close(gather(y, idx, p.layout), ref, p.dtype, f"{p}")
    assert np.all(np.isfinite(to_f64(y.view(-1)[:: max(1, y.numel() // 100000)])))
    return y


@pytest.mark.parametrize("stride", [1, 2])
def test_depthwise56_full_size_sampled(stride):
    p = wl.depthwise_56(stride)
    assert kernel_of(p) == 2
    check_sampled(p, 5)


@pytest.mark.parametrize("groups", [256, 64, 16])
def test_groups_sweep_direct_path_sampled(groups):
    p = wl.depthwise_56(1, groups)
    check_sampled(p, 5, 3000, gb.PATH_DIRECT)
