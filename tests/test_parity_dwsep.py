"""GPU parity of the depthwise-separable block (depthwise conv1d on (batch, steps, channels),
then a pointwise 1x1 convolution over channels: the Conformer convolution module's pair of
convolutions, "Investigate custom Triton kernels for depthwise-separable convolutions in
Conformer", speechbrain #2733) against the fp64 oracle's oracle_dwsep1d_fwd, which CPU tests
pin to brute force, to torch's float64 conv1d + 1x1 conv, and to closed forms.

The fused kernel rounds the intermediate once to the data type (the tensor-core operand), the
composition path rounds it once when it stores it: both stay within the bf16 / fp16
tolerance of the fp64 oracle. Cases: the fused kernel over every supported tap count, ragged
step counts, C_out below / at / above 256 (one or two MMA chunks; partial output slabs),
with and without bias, causal pads, fp16; the composition (forced, and where the fused
kernel does not apply: C % 64 != 0, fp32); integer-valued data bit-exact is not claimed
(the rounded intermediate is not an integer in general); the Conformer layer at full size
on sampled outputs in the launch configuration the benchmark times."""
import numpy as np
import pytest
import torch

import oracle
from depthwise_convolution_gconv2d_b200 import binding as gb
from depthwise_convolution_gconv2d_b200 import workloads as wl
from _util import assert_close, to_dev, to_f64

pytestmark = pytest.mark.gpu

FUSED, UNFUSED = 16, 17


def run(inp, path=gb.PATH_AUTO):
    p = inp.problem
    z = gb.dwsep1d_fwd(to_dev(inp.x, p.dtype), to_dev(inp.w_dw, p.dtype),
                       to_dev(inp.w_pw, p.dtype), to_dev(inp.bias, p.dtype), p.pad_left,
                       p.pad_right, path=path)
    torch.cuda.synchronize()
    return z


def ref(inp):
    p = inp.problem
    return oracle.dwsep1d_fwd(inp.x64(), inp.w_dw64(), inp.w_pw64(), inp.bias64(), p.pad_left,
                              p.pad_right)


def sel(p, C_out, path=gb.PATH_AUTO):
    return gb.dwsep1d_select_path(p.B, p.T, p.C, p.K, p.pad_left, p.pad_right, C_out, p.dtype,
                                  path)


FUSED_CASES = [
    # B, T, C, K, pl, pr, C_out
    (2, 300, 128, 31, 15, 15, 128),
    (1, 128, 64, 3, 1, 1, 64),
    (3, 77, 192, 5, 2, 2, 256),
    (2, 200, 64, 7, 6, 0, 320),        # two MMA chunks (256 + 64)
    (1, 513, 128, 9, 4, 4, 512),
    (2, 260, 64, 15, 7, 7, 80),        # partial 64-channel output slab
    (1, 50, 256, 31, 30, 0, 48),       # causal, fewer steps than a tile
    (2, 140, 64, 31, 0, 0, 64),        # T_out < T
]


@pytest.mark.parametrize("case", FUSED_CASES)
def test_dwsep_fused(case):
    B, T, C, K, pl, pr, Co = case
    p = wl.Dwconv1dProblem(B, T, C, K, pl, pr, wl.BF16)
    assert sel(p, Co) == FUSED
    inp = wl.make_dwsep1d_inputs(p, Co, 70)
    assert_close(to_f64(run(inp)), ref(inp), p.dtype, str(case))


def test_dwsep_fused_no_bias_fp16():
    p = wl.Dwconv1dProblem(2, 300, 128, 31, 15, 15, wl.F16)
    inp = wl.make_dwsep1d_inputs(p, 192, 71, bias=False)
    assert sel(p, 192) == FUSED
    assert_close(to_f64(run(inp)), ref(inp), p.dtype, "fp16 no bias")


@pytest.mark.parametrize("case", [(2, 300, 128, 31, 15, 15, 128), (1, 90, 40, 31, 15, 15, 24),
                                  (2, 64, 64, 4, 2, 1, 96)])
@pytest.mark.parametrize("path", [gb.PATH_DIRECT, gb.PATH_GENERIC])
def test_dwsep_composition(case, path):
    B, T, C, K, pl, pr, Co = case
    p = wl.Dwconv1dProblem(B, T, C, K, pl, pr, wl.BF16)
    assert sel(p, Co, path) == UNFUSED
    inp = wl.make_dwsep1d_inputs(p, Co, 72)
    assert_close(to_f64(run(inp, path)), ref(inp), p.dtype, f"{case} path {path}")


def test_dwsep_auto_falls_back_where_fused_does_not_apply():
    for case, dt in (((1, 90, 40, 31, 15, 15), wl.BF16), ((2, 50, 64, 31, 15, 15), wl.F32)):
        p = wl.Dwconv1dProblem(*case, dt)
        assert sel(p, 32) == UNFUSED
        assert sel(p, 32, gb.PATH_IGEMM) == -2          # UNSUPPORTED
        inp = wl.make_dwsep1d_inputs(p, 32, 73)
        assert_close(to_f64(run(inp)), ref(inp), p.dtype, str(case))


def test_dwsep_conformer_layer_sampled():
    """The Conformer block x[8, 2048, 512], K = 31 'same', then 512 -> 512 pointwise, fused,
    on sampled outputs that the oracle computes one by one."""
    p = wl.conformer_dw1d(False)
    assert sel(p, 512) == FUSED
    inp = wl.make_dwsep1d_inputs(p, 512, 7)
    z = run(inp)
    r = np.random.default_rng(74)
    n = 6000
    idx = np.stack([r.integers(0, p.B, n), r.integers(0, p.T_out, n), r.integers(0, 512, n)], 1)
    corners = np.array([(b, t, o) for b in (0, p.B - 1) for t in (0, 1, 127, 128, p.T_out - 1)
                        for o in (0, 255, 256, 511)])
    idx = np.concatenate([idx, corners], 0)
    want = oracle.dwsep1d_points(inp.x64(), inp.w_dw64(), inp.w_pw64(), inp.bias64(), idx,
                                 p.pad_left, p.pad_right)
    b, t, o = (torch.from_numpy(idx[:, k]).to(z.device) for k in range(3))
    assert_close(to_f64(z[b, t, o]), want, p.dtype, "conformer block")
    assert np.all(np.isfinite(to_f64(z.view(-1)[::997])))


# ------------------------------------------------------------------ 2-D block (NHWC)

def make_2d(N, C, H, W, k, stride, pad, C_out, seed, dtype=wl.BF16, bias=True,
            layout=wl.NHWC):
    """Seeded x (layout), w_dw [C, 1, k, k] storage (same bytes as [C, k, k, 1]), w_pw
    [C_out, C], bias; drawn with the depthwise-separable recipe of the 1-D block."""
    p = wl.Dwconv1dProblem(N, H * W, C, k * k, 0, 0, dtype)
    inp = wl.make_dwsep1d_inputs(p, C_out, seed, bias=bias)
    x = inp.x.reshape(N, H, W, C)
    if layout == wl.NCHW:
        x = np.ascontiguousarray(x.transpose(0, 3, 1, 2))
    return x, inp.w_dw, inp.w_pw, inp.bias


def run_2d(x, w_dw, w_pw, bias, k, stride, pad, dtype, layout=wl.NHWC, path=gb.PATH_AUTO):
    C = x.shape[3] if layout == wl.NHWC else x.shape[1]
    wshape = (C, k, k, 1) if layout == wl.NHWC else (C, 1, k, k)
    z = gb.dwsep2d_fwd(to_dev(x, dtype), to_dev(w_dw.reshape(wshape), dtype),
                       to_dev(w_pw, dtype), to_dev(bias, dtype), stride, pad, 1,
                       "NHWC" if layout == wl.NHWC else "NCHW", path=path)
    torch.cuda.synchronize()
    return z


def ref_2d(x, w_dw, w_pw, bias, k, stride, pad, dtype, layout=wl.NHWC):
    C = x.shape[3] if layout == wl.NHWC else x.shape[1]
    wshape = (C, k, k, 1) if layout == wl.NHWC else (C, 1, k, k)
    return oracle.dwsep2d_fwd(wl.widen(x, dtype), wl.widen(w_dw, dtype).reshape(wshape),
                              wl.widen(w_pw, dtype), None if bias is None else
                              wl.widen(bias, dtype), stride, pad, 1, layout)


FUSED_2D = [
    # N, C, H, W, k, stride, pad, C_out
    (2, 64, 12, 40, 3, 1, 1, 64),
    (1, 128, 20, 80, 3, 2, 1, 256),        # a strided downsampler layer (40 output columns)
    (2, 64, 9, 70, 5, 1, 2, 128),
    (1, 64, 11, 70, 5, 2, 2, 96),
    (1, 192, 7, 70, 3, 2, 1, 320),          # two MMA chunks, a partial column tile
    (1, 64, 5, 150, 3, 1, 0, 512),          # 512 outputs: one tile row per CTA
]


@pytest.mark.parametrize("case", FUSED_2D)
def test_dwsep2d_fused(case):
    N, C, H, W, k, s, pad, Co = case
    x, w_dw, w_pw, b = make_2d(N, C, H, W, k, s, pad, Co, 75)
    assert gb.dwsep2d_select_path(N, C, H, W, k, k, s, pad, 1, Co, "NHWC", wl.BF16,
                                  gb.PATH_IGEMM) == 21
    assert_close(to_f64(run_2d(x, w_dw, w_pw, b, k, s, pad, wl.BF16, path=gb.PATH_IGEMM)),
                 ref_2d(x, w_dw, w_pw, b, k, s, pad, wl.BF16), wl.BF16, str(case))


@pytest.mark.parametrize("layout", [wl.NHWC, wl.NCHW])
@pytest.mark.parametrize("path", [gb.PATH_DIRECT, gb.PATH_GENERIC])
def test_dwsep2d_composition(layout, path):
    N, C, H, W, k, s, pad, Co = (2, 64, 9, 13, 3, 2, 1, 48)
    x, w_dw, w_pw, b = make_2d(N, C, H, W, k, s, pad, Co, 76, layout=layout)
    assert gb.dwsep2d_select_path(N, C, H, W, k, k, s, pad, 1, Co, layout, wl.BF16,
                                  path) == 17
    assert_close(to_f64(run_2d(x, w_dw, w_pw, b, k, s, pad, wl.BF16, layout, path)),
                 ref_2d(x, w_dw, w_pw, b, k, s, pad, wl.BF16, layout), wl.BF16,
                 f"{layout} {path}")


def test_dwsep2d_fp16_no_bias_and_fallbacks():
    x, w_dw, w_pw, b = make_2d(1, 64, 10, 72, 3, 2, 1, 64, 77, dtype=wl.F16, bias=False)
    assert gb.dwsep2d_select_path(1, 64, 10, 72, 3, 3, 2, 1, 1, 64, "NHWC", wl.F16,
                                  gb.PATH_IGEMM) == 21
    assert_close(to_f64(run_2d(x, w_dw, w_pw, None, 3, 2, 1, wl.F16, path=gb.PATH_IGEMM)),
                 ref_2d(x, w_dw, w_pw, None, 3, 2, 1, wl.F16), wl.F16, "fp16")
    # C % 64 != 0, a 7x7 kernel and outputs narrower than a 32-column tile take the
    # composition under AUTO
    x, w_dw, w_pw, b = make_2d(1, 64, 12, 40, 3, 2, 1, 64, 79)
    assert gb.dwsep2d_select_path(1, 64, 12, 40, 3, 3, 2, 1, 1, 64, "NHWC", wl.BF16) == 17
    assert gb.dwsep2d_select_path(1, 64, 12, 40, 3, 3, 2, 1, 1, 64, "NHWC", wl.BF16, 2) == -2
    assert_close(to_f64(run_2d(x, w_dw, w_pw, b, 3, 2, 1, wl.BF16)),
                 ref_2d(x, w_dw, w_pw, b, 3, 2, 1, wl.BF16), wl.BF16, "Wo = 20")
    for (C, k) in ((40, 3), (64, 7)):
        x, w_dw, w_pw, b = make_2d(1, C, 12, 12, k, 1, k // 2, 32, 78)
        assert gb.dwsep2d_select_path(1, C, 12, 12, k, k, 1, k // 2, 1, 32, "NHWC",
                                      wl.BF16) == 17
        assert_close(to_f64(run_2d(x, w_dw, w_pw, b, k, 1, k // 2, wl.BF16)),
                     ref_2d(x, w_dw, w_pw, b, k, 1, k // 2, wl.BF16), wl.BF16, f"C={C} k={k}")
