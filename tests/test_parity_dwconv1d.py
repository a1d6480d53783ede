"""GPU parity of dwconv1d_fwd / dwconv1d_bwd_data / dwconv1d_bwd_weight against the fp64
oracle, on the Conformer workload (x[8, 2048, 512], K = 31, 'same' and causal pads) in full
and on small ragged shapes; the tensor-core forward / data gradient on its edge cases (several
2048-step chunks, ragged chunk ends, every filter-window size up to K = 49, inputs shorter
than a TMA box, pads wider than a box); bit-exact on integer-valued data where sums are
exact; wgrad bitwise reproducible."""
import numpy as np
import pytest
import torch

import oracle
from depthwise_convolution_gconv2d_b200 import binding as gb
from depthwise_convolution_gconv2d_b200 import workloads as wl
from _util import assert_close, to_dev, to_f64

pytestmark = pytest.mark.gpu


def gpu_all(inp, path=gb.PATH_AUTO):
    p = inp.problem
    x, w, dy = (to_dev(a, p.dtype) for a in (inp.x, inp.w, inp.dy))
    y = gb.dwconv1d_fwd(x, w, p.pad_left, p.pad_right, path=path)
    dx = gb.dwconv1d_bwd_data(dy, w, p.T, p.pad_left, p.pad_right, path=path)
    dw = gb.dwconv1d_bwd_weight(x, dy, p.K, p.pad_left, p.pad_right)
    torch.cuda.synchronize()
    return to_f64(y), to_f64(dx), to_f64(dw)


def oracle_all(inp):
    p = inp.problem
    x, w, dy = (wl.widen(a, p.dtype) for a in (inp.x, inp.w, inp.dy))
    return (oracle.dwconv1d_fwd(x, w, p.pad_left, p.pad_right),
            oracle.dwconv1d_bwd_data(dy, w, p.T, p.pad_left, p.pad_right),
            oracle.dwconv1d_bwd_weight(x, dy, p.K, p.pad_left, p.pad_right))


def check(p, workload, dist="normal", path=gb.PATH_AUTO):
    inp = wl.make_dwconv1d_inputs(p, workload, dist)
    for name, got, ref in zip(("fwd", "dgrad", "wgrad"), gpu_all(inp, path), oracle_all(inp)):
        assert_close(got, ref, p.dtype, f"{name} {p}")


def kernel_of(p, path=gb.PATH_AUTO):
    return gb.dwconv1d_select_path(p.B, p.T, p.C, p.K, p.pad_left, p.pad_right, p.dtype, path)


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("path", [gb.PATH_AUTO, gb.PATH_DIRECT])
def test_conformer_full_size(causal, path):
    """The Conformer layer in full on the path the library picks (the tensor-core kernel)
    and forced onto the 128-byte-row CUDA-core kernel."""
    p = wl.conformer_dw1d(causal)
    assert kernel_of(p) == 7 and kernel_of(p, gb.PATH_DIRECT) == 20
    check(p, 3, path=path)


# The 128-byte-row kernels (16-bit, C % 64 == 0, K in {3, 5, 7, 9, 15, 31}): tiles of 64
# channels x 112 steps, a run of tiles per CTA; weight gradient partials per run.
STRIP_CASES = [
    # B, T, C, K, pl, pr
    (2, 300, 64, 31, 15, 15),     # ragged last tile (300 = 2 * 112 + 76)
    (1, 1000, 128, 3, 1, 1),      # two channel blocks
    (3, 117, 192, 5, 4, 0),       # causal-style pads, three channel blocks
    (1, 40, 64, 15, 7, 7),        # fewer steps than a tile
    (2, 500, 64, 7, 0, 0),        # T_out < T
    (1, 300, 64, 31, 30, 30),     # T_out > T
    (1, 100, 64, 9, 200, 0),      # left pad wider than a tile: whole tiles of zero input
    (4, 2048, 128, 31, 15, 15),   # many tiles a run
]


@pytest.mark.parametrize("case", STRIP_CASES)
@pytest.mark.parametrize("dtype", [wl.BF16, wl.F16])
def test_strip_kernels(case, dtype):
    p = wl.Dwconv1dProblem(*case, dtype)
    assert kernel_of(p, gb.PATH_DIRECT) == 20
    check(p, 35, path=gb.PATH_DIRECT)


def test_strip_integer_bit_exact_and_wgrad_deterministic():
    p = wl.Dwconv1dProblem(3, 700, 128, 31, 15, 15, wl.BF16)
    inp = wl.make_dwconv1d_inputs(p, 36, "int")
    inp.w = wl.to_storage(np.random.default_rng(6).integers(-2, 3, (p.C, p.K)), wl.BF16)
    (y, dx, dw), (ry, rdx, rdw) = gpu_all(inp, gb.PATH_DIRECT), oracle_all(inp)
    assert np.array_equal(y, ry) and np.array_equal(dx, rdx)
    rnd = lambda v: wl.widen(wl.to_storage(v, wl.BF16), wl.BF16)
    assert np.array_equal(dw, rnd(rdw))


SMALL = [
    # B, T, C, K, pl, pr
    (2, 300, 72, 31, 15, 15),     # ragged T and C (vector path)
    (1, 129, 64, 31, 30, 0),
    (3, 50, 16, 3, 1, 1),
    (2, 77, 24, 5, 4, 0),
    (1, 200, 136, 7, 3, 3),
    (2, 64, 8, 9, 0, 8),
    (1, 40, 32, 15, 7, 7),
    (2, 100, 40, 31, 0, 0),       # T_out < T
    (1, 20, 8, 31, 15, 15),       # T shorter than the filter
    (2, 90, 5, 31, 15, 15),       # C not a multiple of 8: generic kernels
    (1, 33, 16, 4, 2, 1),         # K without an unrolled wgrad kernel: generic wgrad
    (2, 45, 24, 11, 10, 0),
]

# Tensor-core forward / data gradient (16-bit data, C % 16 == 0, K <= 49): tiles of 16
# channels x 2048 steps, MMA rows of 16-step blocks, 16*KS-step input windows with
# KS = ceil((K + 15) / 16). C % 16 == 8 (e.g. 72, 136 above) takes the CUDA-core ring kernel.
TC_CASES = [
    # B, T, C, K, pl, pr
    (1, 4100, 16, 31, 15, 15),    # three chunks, the last one ragged
    (2, 2049, 16, 17, 8, 8),      # KS = 2 at its largest K; one step into a second chunk
    (2, 2048, 32, 33, 16, 16),    # KS = 3 at its largest K; two channel tiles
    (1, 500, 16, 34, 17, 16),     # KS = 4
    (1, 300, 16, 49, 24, 24),     # K = 49, the largest filter on the tensor cores
    (1, 300, 16, 50, 25, 24),     # K = 50: CUDA-core kernels
    (1, 700, 16, 1, 0, 0),        # K = 1, KS = 1
    (1, 300, 32, 31, 30, 30),     # T_out > T
    (1, 100, 16, 5, 300, 0),      # left pad wider than a TMA box: box skipped, zeros
    (3, 7, 48, 31, 15, 15),       # T far shorter than the window
]


@pytest.mark.parametrize("case", TC_CASES)
@pytest.mark.parametrize("dtype", [wl.BF16, wl.F16])
def test_tensor_core_edges(case, dtype):
    p = wl.Dwconv1dProblem(*case, dtype)
    tc = p.K <= 49
    assert kernel_of(p, gb.PATH_IGEMM) == (7 if tc else -2)      # -2: UNSUPPORTED
    check(p, 33, path=gb.PATH_IGEMM if tc else gb.PATH_AUTO)


# Tensor-core forward / data gradient with C a multiple of 64 (several channel tiles per
# step chunk, as in the Conformer layer) at every KS, on short inputs whose boxes lie outside
# the sequence, pads wider than a box and T_out > T.
TC64_CASES = [
    # B, T, C, K, pl, pr
    (1, 4100, 64, 31, 15, 15),    # three step chunks, the last one ragged
    (2, 2049, 128, 17, 8, 8),     # KS = 2 at its largest K; one step into a second chunk
    (1, 600, 64, 33, 16, 16),     # KS = 3 at its largest K
    (1, 300, 64, 1, 0, 0),        # K = 1, KS = 1
    (2, 700, 64, 3, 1, 1),        # KS = 1
    (3, 7, 64, 31, 15, 15),       # T far shorter than a box
    (1, 100, 64, 5, 300, 0),      # left pad wider than a box
    (1, 300, 64, 31, 30, 30),     # T_out > T
    (2, 1030, 192, 31, 30, 0),    # causal, three channel blocks
]


@pytest.mark.parametrize("case", TC64_CASES)
@pytest.mark.parametrize("dtype", [wl.BF16, wl.F16])
def test_tensor_core_64ch_edges(case, dtype):
    p = wl.Dwconv1dProblem(*case, dtype)
    assert kernel_of(p, gb.PATH_IGEMM) == 7
    check(p, 35, path=gb.PATH_IGEMM)


@pytest.mark.parametrize("case", TC64_CASES[:3] + TC64_CASES[5:7])
def test_tensor_core_64ch_integer_bit_exact(case):
    """Integer-valued data: the tensor-core path gives the oracle's value bit for bit (fwd and
    dgrad) with several channel tiles, so every index, shift and pad is exact."""
    p = wl.Dwconv1dProblem(*case, wl.BF16)
    inp = wl.make_dwconv1d_inputs(p, 36, "int")
    inp.w = wl.to_storage(np.random.default_rng(6).integers(-2, 3, (p.C, p.K)), wl.BF16)
    (y, dx, _), (ry, rdx, _) = gpu_all(inp, gb.PATH_IGEMM), oracle_all(inp)
    assert np.array_equal(y, ry)
    assert np.array_equal(dx, rdx)


def test_tensor_core_tile_buffers_reused_bit_exact():
    """More than two tiles per CTA (4 batches x 3 step chunks x 32 channel tiles = 384 tiles on
    at most 148 CTAs), so each of a CTA's two tile buffers takes a third tile's input after the
    store of its first tile has read it. Integer-valued data: fwd and dgrad bit for bit."""
    p = wl.Dwconv1dProblem(4, 6100, 512, 31, 15, 15, wl.BF16)
    assert kernel_of(p) == 7
    inp = wl.make_dwconv1d_inputs(p, 37, "int")
    inp.w = wl.to_storage(np.random.default_rng(7).integers(-2, 3, (p.C, p.K)), wl.BF16)
    x, w, dy = (to_dev(a, p.dtype) for a in (inp.x, inp.w, inp.dy))
    y = gb.dwconv1d_fwd(x, w, p.pad_left, p.pad_right, path=gb.PATH_IGEMM)
    dx = gb.dwconv1d_bwd_data(dy, w, p.T, p.pad_left, p.pad_right, path=gb.PATH_IGEMM)
    torch.cuda.synchronize()
    xf, wf, dyf = (wl.widen(a, p.dtype) for a in (inp.x, inp.w, inp.dy))
    assert np.array_equal(to_f64(y), oracle.dwconv1d_fwd(xf, wf, p.pad_left, p.pad_right))
    assert np.array_equal(to_f64(dx),
                          oracle.dwconv1d_bwd_data(dyf, wf, p.T, p.pad_left, p.pad_right))


@pytest.mark.parametrize("case", TC_CASES[:4])
def test_ring_and_generic_paths_agree_with_oracle(case):
    """The same problems forced onto the CUDA-core kernels (ring where instantiated, generic
    otherwise) and onto the generic kernel."""
    p = wl.Dwconv1dProblem(*case, wl.BF16)
    check(p, 34, path=gb.PATH_DIRECT)
    check(p, 34, path=gb.PATH_GENERIC)


@pytest.mark.parametrize("case", SMALL)
@pytest.mark.parametrize("dtype", [wl.BF16, wl.F16, wl.F32])
def test_small_shapes(case, dtype):
    check(wl.Dwconv1dProblem(*case, dtype), 30)


@pytest.mark.parametrize("case", SMALL[:8] + TC_CASES[:3])
@pytest.mark.parametrize("path", [gb.PATH_AUTO, gb.PATH_DIRECT, gb.PATH_IGEMM])
def test_integer_valued_bit_exact_fwd_dgrad(case, path):
    """Integers in [-2, 2]: every partial sum is exact in fp32 and the result (|.| <= 132)
    is exact in bf16, so any summation order gives the oracle's value bit for bit."""
    p = wl.Dwconv1dProblem(*case, wl.BF16)
    if path == gb.PATH_IGEMM and kernel_of(p, path) != 7:
        pytest.skip("not a tensor-core problem")
    inp = wl.make_dwconv1d_inputs(p, 31, "int")
    inp.w = wl.to_storage(np.random.default_rng(5).integers(-2, 3, (p.C, p.K)), wl.BF16)
    (y, dx, _), (ry, rdx, _) = gpu_all(inp, path), oracle_all(inp)
    assert np.array_equal(y, ry)
    assert np.array_equal(dx, rdx)


def test_wgrad_deterministic():
    p = wl.conformer_dw1d(False)
    inp = wl.make_dwconv1d_inputs(p, 3)
    x, dy = to_dev(inp.x, p.dtype), to_dev(inp.dy, p.dtype)
    ref = gb.dwconv1d_bwd_weight(x, dy, p.K, p.pad_left, p.pad_right).clone()
    for _ in range(10):
        again = gb.dwconv1d_bwd_weight(x, dy, p.K, p.pad_left, p.pad_right)
        assert torch.equal(again.view(torch.int16), ref.view(torch.int16))


def test_wgrad_workspace_too_small_rejected():
    p = wl.conformer_dw1d(False)
    inp = wl.make_dwconv1d_inputs(p, 3)
    x, dy = to_dev(inp.x, p.dtype), to_dev(inp.dy, p.dtype)
    need = gb.dwconv1d_bwd_weight_workspace_size(p.B, p.T, p.C, p.K, p.pad_left, p.pad_right,
                                                 p.dtype)
    ws = torch.empty(need - 16, dtype=torch.uint8, device="cuda")
    with pytest.raises(gb.GconvError) as e:
        gb.dwconv1d_bwd_weight(x, dy, p.K, p.pad_left, p.pad_right, workspace=ws)
    assert e.value.status == 4


def test_guard_bands_untouched():
    p = wl.Dwconv1dProblem(2, 300, 72, 31, 15, 15, wl.BF16)
    inp = wl.make_dwconv1d_inputs(p, 32)
    x, w, dy = (to_dev(a, p.dtype) for a in (inp.x, inp.w, inp.dy))
    guard = 2048
    for shape, fn in (((p.B, p.T_out, p.C), lambda o: gb.dwconv1d_fwd(x, w, 15, 15, out=o)),
                      ((p.B, p.T, p.C), lambda o: gb.dwconv1d_bwd_data(dy, w, p.T, 15, 15, out=o)),
                      ((p.C, p.K), lambda o: gb.dwconv1d_bwd_weight(x, dy, p.K, 15, 15, out=o))):
        n = int(np.prod(shape))
        buf = torch.full((n + 2 * guard,), float("nan"), dtype=torch.bfloat16, device="cuda")
        sent = buf[:guard].view(torch.int16).clone()
        fn(buf[guard:guard + n].view(shape))
        torch.cuda.synchronize()
        assert torch.equal(buf[:guard].view(torch.int16), sent)
        assert torch.equal(buf[guard + n:].view(torch.int16), sent)
        assert not torch.isnan(buf[guard:guard + n]).any()
