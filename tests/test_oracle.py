"""Pins for the fp64 oracle: it is checked against things other than itself.

Each test ties the oracle to a fact the pages or the mathematics fix: an independent
brute-force evaluator on tiny integer inputs (exact), library routines for special cases
(numpy einsum / correlate / convolve, scipy correlate2d), closed forms (delta kernels,
box sums by integral image), invariants (group concatenation, linearity, adjointness,
ensemble-as-groups), finite differences, the pages' printed facts (tests/golden), and
planted mistakes that the pins must catch. No GPU is needed.
"""
import ctypes
import json
import os
import subprocess
import tempfile

import numpy as np
import pytest
import scipy.signal

import oracle
from depthwise_convolution_gconv2d_b200 import workloads as wl

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
NCHW, NHWC = oracle.NCHW, oracle.NHWC


# ---------------------------------------------------------------- independent evaluators

def n_positions(size, k, stride, pad, dil):
    """Count window start positions by enumeration (no closed-form output-size rule)."""
    span = dil * (k - 1) + 1
    return len(range(0, size + 2 * pad - span + 1, stride))


def brute_conv2d_nchw(x, w, stride, pad, dil, groups):
    """Tap decomposition on an explicitly zero-padded int64 tensor, one group at a time."""
    x = np.asarray(x).astype(np.int64)
    w = np.asarray(w).astype(np.int64)
    N, C_in, H, W = x.shape
    C_out, cpg_in, kH, kW = w.shape
    cpg_out = C_out // groups
    Ho, Wo = n_positions(H, kH, stride, pad, dil), n_positions(W, kW, stride, pad, dil)
    xp = np.zeros((N, C_in, H + 2 * pad, W + 2 * pad), np.int64)
    xp[:, :, pad:pad + H, pad:pad + W] = x
    y = np.zeros((N, C_out, Ho, Wo), np.int64)
    for j in range(groups):
        xg = xp[:, j * cpg_in:(j + 1) * cpg_in]
        wg = w[j * cpg_out:(j + 1) * cpg_out]
        for kh in range(kH):
            for kw in range(kW):
                patch = xg[:, :, kh * dil: kh * dil + stride * (Ho - 1) + 1: stride,
                           kw * dil: kw * dil + stride * (Wo - 1) + 1: stride]
                y[:, j * cpg_out:(j + 1) * cpg_out] += np.einsum("nchw,oc->nohw", patch,
                                                                 wg[:, :, kh, kw])
    return y


def brute_dwconv1d_fwd(x, w, pl, pr):
    """Pure-Python loops over an explicitly padded sequence (integers, exact)."""
    B, T, C = x.shape
    K = w.shape[1]
    xp = np.zeros((B, T + pl + pr, C), np.int64)
    xp[:, pl:pl + T] = x.astype(np.int64)
    T_out = T + pl + pr - K + 1
    y = np.zeros((B, T_out, C), np.int64)
    for b in range(B):
        for t in range(T_out):
            for c in range(C):
                y[b, t, c] = sum(int(w[c, k]) * int(xp[b, t + k, c]) for k in range(K))
    return y


def to_nhwc(x):
    return np.ascontiguousarray(np.transpose(x, (0, 2, 3, 1)))


def from_nhwc(y):
    return np.ascontiguousarray(np.transpose(y, (0, 3, 1, 2)))


def rng_int(seed, shape):
    return np.random.default_rng(seed).integers(-2, 3, shape).astype(np.float64)


# ---------------------------------------------------------------- brute force, all shapes

def _tiny_cases():
    r = np.random.default_rng(7)
    cases = []
    for _ in range(48):
        groups = int(r.choice([1, 2, 3, 4]))
        cpg_in = int(r.integers(1, 4))
        cpg_out = int(r.integers(1, 4))
        k = (int(r.integers(1, 4)), int(r.integers(1, 4)))
        stride, pad, dil = int(r.choice([1, 2])), int(r.choice([0, 1, 2])), int(r.choice([1, 2]))
        H, W = int(r.integers(1, 8)), int(r.integers(1, 8))
        if n_positions(H, k[0], stride, pad, dil) < 1 or n_positions(W, k[1], stride, pad, dil) < 1:
            continue
        cases.append((int(r.integers(1, 3)), groups * cpg_in, H, W, groups * cpg_out, k, stride,
                      pad, dil, groups))
    return cases


@pytest.mark.parametrize("case", _tiny_cases())
@pytest.mark.parametrize("layout", [NCHW, NHWC])
def test_brute_force_conv2d(case, layout):
    N, C_in, H, W, C_out, (kH, kW), s, p, d, g = case
    x = rng_int(1, (N, C_in, H, W))
    w = rng_int(2, (C_out, C_in // g, kH, kW))
    ref = brute_conv2d_nchw(x, w, s, p, d, g)
    if layout == NCHW:
        y = oracle.conv2d(x, w, None, s, p, d, g, NCHW)
    else:
        y = from_nhwc(oracle.conv2d(to_nhwc(x), to_nhwc(w), None, s, p, d, g, NHWC))
    assert y.shape == ref.shape
    assert np.array_equal(y, ref.astype(np.float64))


def test_points_match_full():
    x, w = rng_int(3, (2, 6, 7, 5)), rng_int(4, (9, 2, 3, 2))
    b = rng_int(5, (9,))
    y = oracle.conv2d(x, w, b, 2, 1, 1, 3, NCHW)
    idx = np.array([(n, co, ho, wo) for n in range(2) for co in range(9)
                    for ho in range(y.shape[2]) for wo in range(y.shape[3])])
    pts = oracle.conv2d_points(x, w, idx, b, 2, 1, 1, 3, NCHW)
    assert np.array_equal(pts, y[idx[:, 0], idx[:, 1], idx[:, 2], idx[:, 3]])


# ---------------------------------------------------------------- invariants and library pins

def test_group_concat_of_dense_convs():
    g, cpg_in, cpg_out = 4, 3, 2
    x, w = rng_int(10, (2, g * cpg_in, 6, 5)), rng_int(11, (g * cpg_out, cpg_in, 3, 3))
    y = oracle.conv2d(x, w, None, 1, 1, 1, g, NCHW)
    for j in range(g):
        yj = oracle.conv2d(x[:, j * cpg_in:(j + 1) * cpg_in], w[j * cpg_out:(j + 1) * cpg_out],
                           None, 1, 1, 1, 1, NCHW)
        assert np.array_equal(y[:, j * cpg_out:(j + 1) * cpg_out], yj)


def test_groups1_1x1_is_matmul():
    x, w = rng_int(12, (3, 7, 4, 5)), rng_int(13, (6, 7, 1, 1))
    y = oracle.conv2d(x, w, None, 1, 0, 1, 1, NCHW)
    assert np.array_equal(y, np.einsum("nchw,oc->nohw", x, w[:, :, 0, 0]))


def test_dense_conv_vs_scipy_correlate2d():
    r = np.random.default_rng(14)
    x, w = r.standard_normal((2, 3, 9, 8)), r.standard_normal((4, 3, 3, 2))
    y = oracle.conv2d(x, w, None, 1, 1, 1, 1, NCHW)
    xp = np.pad(x, ((0, 0), (0, 0), (1, 1), (1, 1)))
    ref = np.zeros_like(y)
    for n in range(2):
        for co in range(4):
            for ci in range(3):
                ref[n, co] += scipy.signal.correlate2d(xp[n, ci], w[co, ci], mode="valid")
    np.testing.assert_allclose(y, ref, rtol=1e-12, atol=1e-12)


def test_grouped_conv_vs_scipy_per_group():
    r = np.random.default_rng(15)
    g = 3
    x, w = r.standard_normal((1, 6, 7, 7)), r.standard_normal((9, 2, 3, 3))
    y = oracle.conv2d(x, w, None, 1, 1, 1, g, NCHW)
    xp = np.pad(x, ((0, 0), (0, 0), (1, 1), (1, 1)))
    for co in range(9):
        j = co // 3
        ref = sum(scipy.signal.correlate2d(xp[0, 2 * j + ci], w[co, ci], mode="valid")
                  for ci in range(2))
        np.testing.assert_allclose(y[0, co], ref, rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("layout", [NCHW, NHWC])
def test_centred_delta_is_identity(layout):
    g, C = 4, 8
    cpg = C // g
    x = np.random.default_rng(16).standard_normal((2, C, 6, 7))
    w = np.zeros((C, cpg, 3, 5))
    for co in range(C):
        w[co, co % cpg, 1, 2] = 1.0
    if layout == NCHW:
        y = oracle.conv2d(x, w, None, 1, 0, 1, g, NCHW)  # pad 0 -> interior only
        assert np.array_equal(y, x[:, :, 1:-1, 2:-2])
    xs = to_nhwc(x) if layout == NHWC else x
    w3 = np.zeros((C, cpg, 3, 3))
    for co in range(C):
        w3[co, co % cpg, 1, 1] = 1.0
    y = oracle.conv2d(xs, to_nhwc(w3) if layout == NHWC else w3, None, 1, 1, 1, g, layout)
    assert np.array_equal(y, xs)


def test_offcentre_delta_is_shift_with_zero_fill():
    x = np.random.default_rng(17).standard_normal((1, 2, 5, 6))
    w = np.zeros((2, 1, 3, 3))
    w[:, 0, 0, 2] = 1.0          # tap (kh=0, kw=2) with pad 1: y[h, w] = x[h-1, w+1]
    y = oracle.conv2d(x, w, None, 1, 1, 1, 2, NCHW)
    ref = np.zeros_like(x)
    ref[:, :, 1:, :-1] = x[:, :, :-1, 1:]
    assert np.array_equal(y, ref)


@pytest.mark.parametrize("k,pad", [(3, 1), (5, 2), (3, 0), (4, 3)])
def test_all_ones_depthwise_is_box_sum(k, pad):
    C, H, W = 3, 9, 11
    x = rng_int(18, (2, C, H, W))
    w = np.ones((C, 1, k, k))
    y = oracle.conv2d(x, w, None, 1, pad, 1, C, NCHW)
    # integral image over the zero-padded input
    xp = np.pad(x, ((0, 0), (0, 0), (pad, pad), (pad, pad)))
    S = np.zeros((2, C, xp.shape[2] + 1, xp.shape[3] + 1))
    S[:, :, 1:, 1:] = xp.cumsum(2).cumsum(3)
    Ho, Wo = y.shape[2], y.shape[3]
    ref = (S[:, :, k:k + Ho, k:k + Wo] - S[:, :, :Ho, k:k + Wo] - S[:, :, k:k + Ho, :Wo]
           + S[:, :, :Ho, :Wo])
    assert np.array_equal(y, ref)


def test_linearity_in_x_and_w():
    r = np.random.default_rng(19)
    x1, x2 = r.standard_normal((2, 4, 6, 6)), r.standard_normal((2, 4, 6, 6))
    w1, w2 = r.standard_normal((6, 2, 3, 3)), r.standard_normal((6, 2, 3, 3))
    a, b = 0.75, -1.5
    f = lambda x, w: oracle.conv2d(x, w, None, 2, 1, 2, 2, NCHW)
    np.testing.assert_allclose(f(a * x1 + b * x2, w1), a * f(x1, w1) + b * f(x2, w1),
                               rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(f(x1, a * w1 + b * w2), a * f(x1, w1) + b * f(x1, w2),
                               rtol=1e-12, atol=1e-12)


def test_stride_is_subsampled_stride1():
    x, w = rng_int(20, (2, 4, 9, 10)), rng_int(21, (4, 2, 3, 3))
    y1 = oracle.conv2d(x, w, None, 1, 1, 1, 2, NCHW)
    y2 = oracle.conv2d(x, w, None, 2, 1, 1, 2, NCHW)
    assert np.array_equal(y2, y1[:, :, ::2, ::2])


def test_dilation_is_zero_inserted_kernel():
    x, w = rng_int(22, (1, 3, 11, 12)), rng_int(23, (3, 1, 3, 2))
    y = oracle.conv2d(x, w, None, 1, 2, 2, 3, NCHW)
    wd = np.zeros((3, 1, 5, 3))
    wd[:, :, ::2, ::2] = w
    assert np.array_equal(y, oracle.conv2d(x, wd, None, 1, 2, 1, 3, NCHW))


def test_layouts_agree():
    x, w = rng_int(24, (2, 6, 5, 7)), rng_int(25, (9, 2, 3, 3))
    b = rng_int(26, (9,))
    y = oracle.conv2d(x, w, b, 2, 1, 1, 3, NCHW)
    y2 = oracle.conv2d(to_nhwc(x), to_nhwc(w), b, 2, 1, 1, 3, NHWC)
    assert np.array_equal(from_nhwc(y2), y)


def test_bias_is_broadcast_add():
    x, w, b = rng_int(27, (2, 4, 5, 5)), rng_int(28, (4, 1, 3, 3)), rng_int(29, (4,))
    y0 = oracle.conv2d(x, w, None, 1, 1, 1, 4, NCHW)
    y1 = oracle.conv2d(x, w, b, 1, 1, 1, 4, NCHW)
    assert np.array_equal(y1, y0 + b[None, :, None, None])


def test_ensemble_equals_groups():
    """M models each mapping cin->cout channels, stacked model-major into one groups=M conv
    (the vmap batching rule of "Optimize convolution batching rule performance")."""
    M, cin, cout, B = 4, 3, 5, 2
    r = np.random.default_rng(30)
    xs = [r.integers(-2, 3, (B, cin, 6, 6)).astype(float) for _ in range(M)]
    ws = [r.integers(-2, 3, (cout, cin, 3, 3)).astype(float) for _ in range(M)]
    y = oracle.conv2d(np.concatenate(xs, 1), np.concatenate(ws, 0), None, 1, 1, 1, M, NCHW)
    for m in range(M):
        ym = oracle.conv2d(xs[m], ws[m], None, 1, 1, 1, 1, NCHW)
        assert np.array_equal(y[:, m * cout:(m + 1) * cout], ym)
        assert np.array_equal(ym, brute_conv2d_nchw(xs[m], ws[m], 1, 1, 1, 1))


def test_rejects_bad_shapes():
    with pytest.raises(ValueError):
        oracle.conv2d(np.zeros((1, 6, 4, 4)), np.zeros((4, 3, 3, 3)), groups=4)
    with pytest.raises(ValueError):       # window larger than the padded input
        oracle.conv2d(np.zeros((1, 2, 2, 2)), np.zeros((2, 2, 5, 5)), pad=0)


# ---------------------------------------------------------------- pages' printed facts

def test_group_order_golden():
    """Output channel co of a grouped conv reads input group co // (C_out/g): the usual
    group-major order of the neon thread."""
    gold = json.load(open(os.path.join(GOLDEN, "group_order.json")))
    C, g = gold["C_out"], gold["groups"]
    cpg = C // g
    assert gold["expected"].startswith(gold["printed"])
    x = np.zeros((1, C, 1, 1))
    for c in range(C):
        x[0, c] = c // cpg + 1           # input channel carries its group label
    w = np.ones((C, cpg, 1, 1)) / cpg    # output = mean of the inputs it is connected to
    y = oracle.conv2d(x, w, None, 1, 0, 1, g, NCHW)
    assert "".join(str(int(v)) for v in y[0, :, 0, 0]) == gold["expected"]


def test_p2_layer_golden():
    gold = json.load(open(os.path.join(GOLDEN, "p2_layer.json")))
    xs, ws = gold["input_shape"], gold["weight_shape"]
    assert ws[1] * gold["groups"] == xs[1]
    shape = oracle.conv2d_out_shape(xs, ws, 1, gold["padding"], 1, gold["groups"], NCHW)
    assert list(shape) == gold["expected_output_shape"]
    # a few sampled outputs of the full-size layer against a per-point window sum
    p = wl.wide_group(wl.NCHW, wl.F32)
    r = np.random.default_rng(31)
    x = r.integers(-2, 3, p.x_shape).astype(np.float64)
    w = r.integers(-2, 3, p.w_shape).astype(np.float64)
    idx = np.array([(0, 0, 0, 0), (0, 511, 255, 255), (0, 130, 17, 0), (0, 383, 255, 100)])
    got = oracle.conv2d_points(x, w, idx, None, 1, 1, 1, 4, NCHW)
    xp = np.pad(x, ((0, 0), (0, 0), (1, 1), (1, 1)))
    for (n, co, ho, wo), v in zip(idx, got):
        j = co // 128
        win = xp[n, j * 128:(j + 1) * 128, ho:ho + 3, wo:wo + 3]
        assert v == float((win * w[co]).sum())


# ---------------------------------------------------------------- dwconv1d

CONV1D_CASES = [(2, 9, 3, 3, 1, 1), (1, 12, 4, 5, 4, 0), (3, 7, 2, 31, 15, 15),
                (2, 40, 5, 31, 30, 0), (1, 5, 1, 2, 0, 1), (2, 6, 3, 4, 0, 0)]


@pytest.mark.parametrize("B,T,C,K,pl,pr", CONV1D_CASES)
def test_dwconv1d_fwd_brute_force(B, T, C, K, pl, pr):
    x, w = rng_int(40, (B, T, C)), rng_int(41, (C, K))
    assert np.array_equal(oracle.dwconv1d_fwd(x, w, pl, pr),
                          brute_dwconv1d_fwd(x, w, pl, pr).astype(float))


@pytest.mark.parametrize("B,T,C,K,pl,pr", CONV1D_CASES)
def test_dwconv1d_library_pins(B, T, C, K, pl, pr):
    """fwd = numpy.correlate, dgrad = numpy.convolve ('full', cropped), wgrad =
    numpy.correlate of the padded input with dy, per (batch, channel)."""
    r = np.random.default_rng(42)
    x, w = r.standard_normal((B, T, C)), r.standard_normal((C, K))
    T_out = T + pl + pr - K + 1
    dy = r.standard_normal((B, T_out, C))
    y = oracle.dwconv1d_fwd(x, w, pl, pr)
    dx = oracle.dwconv1d_bwd_data(dy, w, T, pl, pr)
    dw = oracle.dwconv1d_bwd_weight(x, dy, K, pl, pr)
    dw_ref = np.zeros((C, K))
    for b in range(B):
        for c in range(C):
            xp = np.concatenate([np.zeros(pl), x[b, :, c], np.zeros(pr)])
            np.testing.assert_allclose(y[b, :, c], np.correlate(xp, w[c], "valid"),
                                       rtol=1e-12, atol=1e-12)
            full = np.convolve(dy[b, :, c], w[c], "full")
            np.testing.assert_allclose(dx[b, :, c], full[pl:pl + T], rtol=1e-12, atol=1e-12)
            dw_ref[c] += np.correlate(xp, dy[b, :, c], "valid")
    np.testing.assert_allclose(dw, dw_ref, rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("B,T,C,K,pl,pr", CONV1D_CASES)
def test_dwconv1d_adjoint_identity(B, T, C, K, pl, pr):
    """<fwd(x, w), dy> = <x, dgrad(dy, w)> = <w, wgrad(x, dy)>."""
    r = np.random.default_rng(43)
    x, w = r.standard_normal((B, T, C)), r.standard_normal((C, K))
    dy = r.standard_normal((B, T + pl + pr - K + 1, C))
    a = np.vdot(oracle.dwconv1d_fwd(x, w, pl, pr), dy)
    b = np.vdot(x, oracle.dwconv1d_bwd_data(dy, w, T, pl, pr))
    c = np.vdot(w, oracle.dwconv1d_bwd_weight(x, dy, K, pl, pr))
    assert abs(a - b) <= 1e-10 * max(1.0, abs(a))
    assert abs(a - c) <= 1e-10 * max(1.0, abs(a))


def test_dwconv1d_finite_differences():
    """Central differences of L = <fwd(x, w), dy> (the gradcheck idea of the Conformer
    thread) against dgrad and wgrad."""
    B, T, C, K, pl, pr = 2, 7, 2, 4, 2, 1
    r = np.random.default_rng(44)
    x, w = r.standard_normal((B, T, C)), r.standard_normal((C, K))
    dy = r.standard_normal((B, T + pl + pr - K + 1, C))
    L = lambda xx, ww: np.vdot(oracle.dwconv1d_fwd(xx, ww, pl, pr), dy)
    dx = oracle.dwconv1d_bwd_data(dy, w, T, pl, pr)
    dw = oracle.dwconv1d_bwd_weight(x, dy, K, pl, pr)
    h = 1e-6
    for i in np.ndindex(x.shape):
        e = np.zeros_like(x)
        e[i] = h
        assert abs((L(x + e, w) - L(x - e, w)) / (2 * h) - dx[i]) < 1e-6
    for i in np.ndindex(w.shape):
        e = np.zeros_like(w)
        e[i] = h
        assert abs((L(x, w + e) - L(x, w - e)) / (2 * h) - dw[i]) < 1e-6


def test_dwconv1d_same_and_causal_relation():
    """With equal total padding, the causal output is the 'same' output shifted by the
    difference in left padding (here 15 steps), zero-filled where the window leaves x."""
    x, w = rng_int(45, (2, 50, 3)), rng_int(46, (3, 31))
    ys = oracle.dwconv1d_fwd(x, w, 15, 15)
    yc = oracle.dwconv1d_fwd(x, w, 30, 0)
    # yc[t] = sum_k w[k] x[t+k-30] = ys[t-15] for t >= 15
    assert np.array_equal(yc[:, 15:], ys[:, :-15])


def test_dwconv1d_equals_depthwise_conv2d():
    """conv1d on (batch, steps, channels) is the depthwise conv2d with H = 1 (NHWC)."""
    B, T, C, K = 2, 13, 4, 5
    x, w = rng_int(47, (B, T, C)), rng_int(48, (C, K))
    # conv2d pads H as well (scalar pad); with kH = 1 the middle row is the conv1d result
    y2 = oracle.conv2d(x[:, None], w[:, None, :, None], None, 1, 2, 1, C, NHWC)[:, 2]
    assert np.array_equal(y2, oracle.dwconv1d_fwd(x, w, 2, 2))


# ---------------------------------------------------------------- grouped conv2d backward

def brute_bwd_nchw(x, w, dy, stride, pad, dil, groups):
    """dx and dw from the independent forward evaluator alone, by linearity: the forward is
    linear in x and in w, so dx[i] = <brute(e_i, w), dy> and dw[j] = <brute(x, e_j), dy> for
    the unit tensors e_i, e_j (integers, exact)."""
    dyi = np.asarray(dy).astype(np.int64)
    dx = np.zeros(x.shape, np.int64)
    for i in np.ndindex(x.shape):
        e = np.zeros(x.shape)
        e[i] = 1
        dx[i] = np.sum(brute_conv2d_nchw(e, w, stride, pad, dil, groups) * dyi)
    dw = np.zeros(w.shape, np.int64)
    for j in np.ndindex(w.shape):
        e = np.zeros(w.shape)
        e[j] = 1
        dw[j] = np.sum(brute_conv2d_nchw(x, e, stride, pad, dil, groups) * dyi)
    return dx, dw


def _bwd_grads(x, w, dy, s, p, d, g, layout):
    """Oracle dx, dw for NCHW tensors, run in `layout` and returned as NCHW."""
    H, W = x.shape[2], x.shape[3]
    k = (w.shape[2], w.shape[3])
    if layout == NCHW:
        return (oracle.conv2d_bwd_data(dy, w, (H, W), s, p, d, g, NCHW),
                oracle.conv2d_bwd_weight(x, dy, k, s, p, d, g, NCHW))
    dx = oracle.conv2d_bwd_data(to_nhwc(dy), to_nhwc(w), (H, W), s, p, d, g, NHWC)
    dw = oracle.conv2d_bwd_weight(to_nhwc(x), to_nhwc(dy), k, s, p, d, g, NHWC)
    return from_nhwc(dx), from_nhwc(dw)


@pytest.mark.parametrize("case", _tiny_cases()[:20])
@pytest.mark.parametrize("layout", [NCHW, NHWC])
def test_conv2d_bwd_brute_force(case, layout):
    N, C_in, H, W, C_out, (kH, kW), s, p, d, g = case
    x = rng_int(60, (N, C_in, H, W))
    w = rng_int(61, (C_out, C_in // g, kH, kW))
    dy = rng_int(62, brute_conv2d_nchw(x, w, s, p, d, g).shape)
    dx_ref, dw_ref = brute_bwd_nchw(x, w, dy, s, p, d, g)
    dx, dw = _bwd_grads(x, w, dy, s, p, d, g, layout)
    assert np.array_equal(dx, dx_ref.astype(float))
    assert np.array_equal(dw, dw_ref.astype(float))


BWD_CASES = [
    # N, C_in, H, W, C_out, kH, kW, stride, pad, dil, groups
    (2, 6, 9, 8, 9, 3, 3, 1, 1, 1, 3),      # cpg_in 2 != cpg_out 3
    (1, 8, 11, 10, 8, 3, 3, 2, 1, 1, 8),    # depthwise, stride 2, ragged
    (2, 4, 7, 9, 8, 3, 2, 3, 2, 1, 2),      # stride 3, pad larger than needed
    (1, 6, 12, 12, 6, 3, 3, 1, 2, 2, 2),    # dilation 2
    (1, 12, 6, 7, 12, 5, 5, 1, 2, 1, 4),    # 5x5
    (2, 8, 5, 5, 4, 1, 1, 2, 0, 1, 4),      # 1x1 stride 2: rows / columns nobody reads
    (1, 4, 4, 4, 4, 3, 3, 1, 3, 1, 1),      # pad 3 > dil*(k-1): border outputs read only padding
]


@pytest.mark.parametrize("case", BWD_CASES)
def test_conv2d_bwd_vs_torch(case):
    """Library pin: torch's own conv2d input / weight gradients in float64 on the CPU."""
    import torch
    N, C_in, H, W, C_out, kH, kW, s, p, d, g = case
    r = np.random.default_rng(63)
    x = r.standard_normal((N, C_in, H, W))
    w = r.standard_normal((C_out, C_in // g, kH, kW))
    Ho, Wo = n_positions(H, kH, s, p, d), n_positions(W, kW, s, p, d)
    dy = r.standard_normal((N, C_out, Ho, Wo))
    tx, tw, tdy = (torch.from_numpy(a) for a in (x, w, dy))
    dx_ref = torch.nn.grad.conv2d_input(tx.shape, tw, tdy, s, p, d, g).numpy()
    dw_ref = torch.nn.grad.conv2d_weight(tx, tw.shape, tdy, s, p, d, g).numpy()
    for layout in (NCHW, NHWC):
        dx, dw = _bwd_grads(x, w, dy, s, p, d, g, layout)
        np.testing.assert_allclose(dx, dx_ref, rtol=1e-11, atol=1e-11)
        np.testing.assert_allclose(dw, dw_ref, rtol=1e-11, atol=1e-11)


@pytest.mark.parametrize("case", BWD_CASES)
def test_conv2d_bwd_adjoint_identity(case):
    """<conv2d(x, w), dy> = <x, dx> = <w, dw> against the (separately pinned) forward."""
    N, C_in, H, W, C_out, kH, kW, s, p, d, g = case
    r = np.random.default_rng(64)
    x = r.standard_normal((N, H, W, C_in))
    w = r.standard_normal((C_out, kH, kW, C_in // g))
    y = oracle.conv2d(x, w, None, s, p, d, g, NHWC)
    dy = r.standard_normal(y.shape)
    a = np.vdot(y, dy)
    b = np.vdot(x, oracle.conv2d_bwd_data(dy, w, (H, W), s, p, d, g, NHWC))
    c = np.vdot(w, oracle.conv2d_bwd_weight(x, dy, (kH, kW), s, p, d, g, NHWC))
    assert abs(a - b) <= 1e-10 * max(1.0, abs(a))
    assert abs(a - c) <= 1e-10 * max(1.0, abs(a))


def test_conv2d_bwd_1x1_is_matmul():
    """Closed form: for a 1x1, stride-1, unpadded layer, per group dx = W_g^T dy_g and
    dw_g = sum over pixels of dy_g x_g^T (numpy matmul)."""
    N, H, W, g, ci, co = 2, 5, 4, 3, 4, 2
    r = np.random.default_rng(65)
    x = r.standard_normal((N, H, W, g * ci))
    w = r.standard_normal((g * co, 1, 1, ci))
    dy = r.standard_normal((N, H, W, g * co))
    dx = oracle.conv2d_bwd_data(dy, w, (H, W), 1, 0, 1, g, NHWC)
    dw = oracle.conv2d_bwd_weight(x, dy, (1, 1), 1, 0, 1, g, NHWC)
    for j in range(g):
        Wg = w[j * co:(j + 1) * co, 0, 0, :]                      # [co, ci]
        dyg = dy[..., j * co:(j + 1) * co].reshape(-1, co)        # [pixels, co]
        xg = x[..., j * ci:(j + 1) * ci].reshape(-1, ci)          # [pixels, ci]
        np.testing.assert_allclose(dx[..., j * ci:(j + 1) * ci].reshape(-1, ci), dyg @ Wg,
                                   rtol=1e-12, atol=1e-12)
        np.testing.assert_allclose(dw[j * co:(j + 1) * co, 0, 0, :], dyg.T @ xg,
                                   rtol=1e-12, atol=1e-12)


def test_conv2d_bwd_finite_differences():
    """Central differences of L = <conv2d(x, w), dy> against dx and dw."""
    N, C_in, H, W, C_out, k, s, p, d, g = 1, 4, 5, 4, 6, 3, 2, 1, 1, 2
    r = np.random.default_rng(66)
    x = r.standard_normal((N, C_in, H, W))
    w = r.standard_normal((C_out, C_in // g, k, k))
    dy = r.standard_normal(oracle.conv2d(x, w, None, s, p, d, g, NCHW).shape)
    L = lambda xx, ww: np.vdot(oracle.conv2d(xx, ww, None, s, p, d, g, NCHW), dy)
    dx = oracle.conv2d_bwd_data(dy, w, (H, W), s, p, d, g, NCHW)
    dw = oracle.conv2d_bwd_weight(x, dy, (k, k), s, p, d, g, NCHW)
    h = 1e-6
    for a, grad, is_x in ((x, dx, True), (w, dw, False)):
        for i in np.ndindex(a.shape):
            e = np.zeros_like(a)
            e[i] = h
            fd = (L(x + e, w) - L(x - e, w)) if is_x else (L(x, w + e) - L(x, w - e))
            assert abs(fd / (2 * h) - grad[i]) < 1e-6


@pytest.mark.parametrize("case", BWD_CASES)
@pytest.mark.parametrize("layout", [NCHW, NHWC])
def test_conv2d_bwd_points_match_full(case, layout):
    N, C_in, H, W, C_out, kH, kW, s, p, d, g = case
    x = rng_int(67, (N, C_in, H, W))
    w = rng_int(68, (C_out, C_in // g, kH, kW))
    dy = rng_int(69, (N, C_out, n_positions(H, kH, s, p, d), n_positions(W, kW, s, p, d)))
    dx, dw = _bwd_grads(x, w, dy, s, p, d, g, layout)
    xi = np.array(list(np.ndindex(dx.shape)))
    wi = np.array(list(np.ndindex(dw.shape)))
    if layout == NCHW:
        px = oracle.conv2d_bwd_data_points(dy, w, (H, W), xi, s, p, d, g, NCHW)
        pw = oracle.conv2d_bwd_weight_points(x, dy, (kH, kW), wi, s, p, d, g, NCHW)
    else:
        px = oracle.conv2d_bwd_data_points(to_nhwc(dy), to_nhwc(w), (H, W), xi, s, p, d, g, NHWC)
        pw = oracle.conv2d_bwd_weight_points(to_nhwc(x), to_nhwc(dy), (kH, kW), wi, s, p, d, g,
                                             NHWC)
    assert np.array_equal(px, dx[tuple(xi.T)])
    assert np.array_equal(pw, dw[tuple(wi.T)])


# ---------------------------------------------------------------- output order and group merges

def test_interleaved_order_golden():
    """The neon thread's alternative output order, 1234123412341234: each output position
    reads the input group printed at its place."""
    gold = json.load(open(os.path.join(GOLDEN, "interleaved_order.json")))
    C, g = gold["C_out"], gold["groups"]
    cpg = C // g
    assert gold["expected"] == gold["printed"]
    x = np.zeros((1, C, 1, 1))
    for c in range(C):
        x[0, c] = c // cpg + 1           # input channel carries its group label
    w = np.ones((C, cpg, 1, 1)) / cpg
    y = oracle.conv2d_interleaved(x, w, None, 1, 0, 1, g, NCHW)
    assert "".join(str(int(v)) for v in y[0, :, 0, 0]) == gold["expected"]


MERGE_CASES = [(2, 8, 7, 6, 12, 3, 1, 1, 1, 4), (1, 6, 9, 8, 9, 3, 2, 1, 1, 3),
               (2, 4, 5, 5, 8, 1, 1, 0, 1, 2), (1, 16, 6, 7, 16, 3, 1, 2, 2, 16)]


@pytest.mark.parametrize("case", MERGE_CASES)
@pytest.mark.parametrize("layout", [NCHW, NHWC])
def test_interleaved_is_reshape_transpose(case, layout):
    """Interleaved output = the group-major output with its (group, filter) channel axes
    swapped (numpy reshape / transpose)."""
    N, C_in, H, W, C_out, k, s, p, d, g = case
    r = np.random.default_rng(81)
    x, w = r.standard_normal((N, C_in, H, W)), r.standard_normal((C_out, C_in // g, k, k))
    b = r.standard_normal(C_out)
    y = oracle.conv2d(x, w, b, s, p, d, g, NCHW)
    n, _, Ho, Wo = y.shape
    ref = y.reshape(n, g, C_out // g, Ho, Wo).transpose(0, 2, 1, 3, 4).reshape(y.shape)
    if layout == NCHW:
        got = oracle.conv2d_interleaved(x, w, b, s, p, d, g, NCHW)
    else:
        got = from_nhwc(oracle.conv2d_interleaved(to_nhwc(x), to_nhwc(w), b, s, p, d, g, NHWC))
    assert np.array_equal(got, ref)


@pytest.mark.parametrize("case", MERGE_CASES)
@pytest.mark.parametrize("mode", ["avg", "max"])
@pytest.mark.parametrize("layout", [NCHW, NHWC])
def test_group_merge_vs_numpy(case, mode, layout):
    """Merge across groups = numpy mean / max over the group axis of the group-major output."""
    N, C_in, H, W, C_out, k, s, p, d, g = case
    r = np.random.default_rng(82)
    x, w = r.standard_normal((N, C_in, H, W)), r.standard_normal((C_out, C_in // g, k, k))
    y = oracle.conv2d(x, w, None, s, p, d, g, NCHW)
    n, _, Ho, Wo = y.shape
    yg = y.reshape(n, g, C_out // g, Ho, Wo)
    ref = yg.mean(axis=1) if mode == "avg" else yg.max(axis=1)
    if layout == NCHW:
        got = oracle.conv2d_group_merge(x, w, None, s, p, d, g, NCHW, mode)
    else:
        got = from_nhwc(oracle.conv2d_group_merge(to_nhwc(x), to_nhwc(w), None, s, p, d, g,
                                                  NHWC, mode))
    np.testing.assert_allclose(got, ref, rtol=1e-13, atol=1e-13)


def test_group_merge_is_pooling_over_interleaved_order():
    """Average / max pooling over windows of `groups` consecutive channels of the interleaved
    output (the volumetric pooling the thread has in mind) is the merge across groups."""
    N, C_in, H, W, C_out, k, s, p, d, g = MERGE_CASES[0]
    r = np.random.default_rng(83)
    x, w = r.standard_normal((N, C_in, H, W)), r.standard_normal((C_out, C_in // g, k, k))
    yi = oracle.conv2d_interleaved(x, w, None, s, p, d, g, NCHW)
    n, _, Ho, Wo = yi.shape
    win = yi.reshape(n, C_out // g, g, Ho, Wo)
    np.testing.assert_allclose(oracle.conv2d_group_merge(x, w, None, s, p, d, g, NCHW, "avg"),
                               win.mean(axis=2), rtol=1e-13, atol=1e-13)
    assert np.array_equal(oracle.conv2d_group_merge(x, w, None, s, p, d, g, NCHW, "max"),
                          win.max(axis=2))


def test_group_merge_averages_an_ensemble():
    """The ensemble-as-groups layer merged with 'avg' is the mean of the models' own dense
    convolutions (P1's ensemble, averaged)."""
    models, cin, cout = 4, 3, 5
    r = np.random.default_rng(84)
    x = r.standard_normal((2, models * cin, 6, 7))
    w = r.standard_normal((models * cout, cin, 3, 3))
    got = oracle.conv2d_group_merge(x, w, None, 1, 1, 1, models, NCHW, "avg")
    ref = np.mean([oracle.conv2d(x[:, m * cin:(m + 1) * cin], w[m * cout:(m + 1) * cout], None,
                                 1, 1, 1, 1, NCHW) for m in range(models)], axis=0)
    np.testing.assert_allclose(got, ref, rtol=1e-12, atol=1e-12)


def test_grouped_linear_is_per_group_matmul():
    """A grouped linear layer (the neon thread's gemmBatched use) is the grouped conv2d with
    H = W = 1 and a 1x1 kernel: per group, y_g = x_g W_g^T + b_g (numpy matmul)."""
    B, g, i_, o_ = 7, 5, 6, 4
    r = np.random.default_rng(85)
    x = r.standard_normal((B, g * i_))
    w = r.standard_normal((g * o_, i_))
    b = r.standard_normal(g * o_)
    y = oracle.conv2d(x[:, :, None, None], w[:, :, None, None], b, 1, 0, 1, g, NCHW)[:, :, 0, 0]
    for j in range(g):
        np.testing.assert_allclose(y[:, j * o_:(j + 1) * o_],
                                   x[:, j * i_:(j + 1) * i_] @ w[j * o_:(j + 1) * o_].T +
                                   b[j * o_:(j + 1) * o_], rtol=1e-12, atol=1e-12)


# ---------------------------------------------------------------- depthwise-separable block

def brute_dwsep1d(x, wd, wp, b, pl, pr):
    """Pure-Python loops on integers: depthwise over an explicitly padded sequence, then the
    channel mix."""
    B, T, C = x.shape
    K = wd.shape[1]
    O = wp.shape[0]
    T_out = T + pl + pr - K + 1
    xp = [[[0] * C for _ in range(T + pl + pr)] for _ in range(B)]
    for bb in range(B):
        for t in range(T):
            for c in range(C):
                xp[bb][t + pl][c] = int(x[bb, t, c])
    z = np.zeros((B, T_out, O), np.int64)
    for bb in range(B):
        for t in range(T_out):
            y = [sum(int(wd[c, k]) * xp[bb][t + k][c] for k in range(K)) for c in range(C)]
            for o in range(O):
                z[bb, t, o] = int(b[o]) + sum(int(wp[o, c]) * y[c] for c in range(C))
    return z


DWSEP1D_CASES = [(2, 9, 3, 4, 3, 1, 1), (1, 12, 5, 2, 5, 4, 0), (2, 40, 4, 6, 31, 15, 15),
                 (1, 33, 3, 3, 31, 30, 0)]


@pytest.mark.parametrize("B,T,C,O,K,pl,pr", DWSEP1D_CASES)
def test_dwsep1d_brute_force(B, T, C, O, K, pl, pr):
    x, wd = rng_int(70, (B, T, C)), rng_int(71, (C, K))
    wp, b = rng_int(72, (O, C)), rng_int(73, (O,))
    assert np.array_equal(oracle.dwsep1d_fwd(x, wd, wp, b, pl, pr),
                          brute_dwsep1d(x, wd, wp, b, pl, pr).astype(float))


@pytest.mark.parametrize("B,T,C,O,K,pl,pr", DWSEP1D_CASES)
def test_dwsep1d_vs_torch(B, T, C, O, K, pl, pr):
    """Library pin: torch's conv1d (groups = C) then a 1x1 conv1d, float64 on the CPU."""
    import torch
    import torch.nn.functional as F
    r = np.random.default_rng(74)
    x, wd = r.standard_normal((B, T, C)), r.standard_normal((C, K))
    wp, b = r.standard_normal((O, C)), r.standard_normal(O)
    tx = F.pad(torch.from_numpy(x).permute(0, 2, 1), (pl, pr))
    y = F.conv1d(tx, torch.from_numpy(wd)[:, None, :], groups=C)
    z = F.conv1d(y, torch.from_numpy(wp)[:, :, None], torch.from_numpy(b))
    np.testing.assert_allclose(oracle.dwsep1d_fwd(x, wd, wp, b, pl, pr),
                               z.permute(0, 2, 1).numpy(), rtol=1e-11, atol=1e-11)


@pytest.mark.parametrize("stride,pad,dil", [(1, 1, 1), (2, 1, 1), (1, 2, 2), (2, 0, 1)])
@pytest.mark.parametrize("layout", [NCHW, NHWC])
def test_dwsep2d_vs_torch(stride, pad, dil, layout):
    """Library pin: torch's conv2d (groups = C) then a 1x1 conv2d, float64 on the CPU."""
    import torch
    import torch.nn.functional as F
    N, C, H, W, O = 2, 6, 9, 8, 5
    r = np.random.default_rng(75)
    x, wd = r.standard_normal((N, C, H, W)), r.standard_normal((C, 1, 3, 3))
    wp, b = r.standard_normal((O, C)), r.standard_normal(O)
    y = F.conv2d(torch.from_numpy(x), torch.from_numpy(wd), None, stride, pad, dil, C)
    ref = F.conv2d(y, torch.from_numpy(wp)[:, :, None, None], torch.from_numpy(b)).numpy()
    if layout == NCHW:
        got = oracle.dwsep2d_fwd(x, wd, wp, b, stride, pad, dil, NCHW)
    else:
        got = from_nhwc(oracle.dwsep2d_fwd(to_nhwc(x), to_nhwc(wd), wp, b, stride, pad, dil,
                                           NHWC))
    np.testing.assert_allclose(got, ref, rtol=1e-11, atol=1e-11)


def test_dwsep_closed_forms():
    """An identity channel mix leaves the (separately pinned) depthwise result; a depthwise
    filter with one unit tap at k = pad_left leaves the channel mix x @ w_pw^T + b (numpy)."""
    r = np.random.default_rng(76)
    B, T, C, K, pl, pr = 2, 11, 5, 7, 3, 3
    x, wd = r.standard_normal((B, T, C)), r.standard_normal((C, K))
    np.testing.assert_allclose(oracle.dwsep1d_fwd(x, wd, np.eye(C), None, pl, pr),
                               oracle.dwconv1d_fwd(x, wd, pl, pr), rtol=1e-13, atol=1e-13)
    delta = np.zeros((C, K))
    delta[:, pl] = 1.0
    wp, b = r.standard_normal((4, C)), r.standard_normal(4)
    np.testing.assert_allclose(oracle.dwsep1d_fwd(x, delta, wp, b, pl, pr), x @ wp.T + b,
                               rtol=1e-12, atol=1e-12)
    x2 = r.standard_normal((2, 6, 5, C))
    d2 = np.zeros((C, 3, 3, 1))
    d2[:, 1, 1, 0] = 1.0
    np.testing.assert_allclose(oracle.dwsep2d_fwd(x2, d2, wp, b, 1, 1, 1, NHWC), x2 @ wp.T + b,
                               rtol=1e-12, atol=1e-12)


def test_dwsep1d_points_match_full():
    x, wd = rng_int(77, (2, 20, 6)), rng_int(78, (6, 9))
    wp, b = rng_int(79, (5, 6)), rng_int(80, (5,))
    z = oracle.dwsep1d_fwd(x, wd, wp, b, 4, 4)
    idx = np.array(list(np.ndindex(z.shape)))
    assert np.array_equal(oracle.dwsep1d_points(x, wd, wp, b, idx, 4, 4), z[tuple(idx.T)])


# ---------------------------------------------------------------- planted mistakes

MUTANTS = {
    "kh_kw_swapped_in_nchw_weight": ("((co * cpg_in + ci) * s->kH + kh) * s->kW + kw",
                                     "((co * cpg_in + ci) * s->kH + kw) * s->kW + kh"),
    "group_offset_dropped": ("long c = g * cpg_in + ci;", "long c = ci;"),
    "pad_sign_flipped": ("long h = ho * s->stride - s->pad + kh * s->dil;",
                         "long h = ho * s->stride + s->pad + kh * s->dil;"),
    "last_tap_dropped": ("for (long kw = 0; kw < s->kW; ++kw)", "for (long kw = 0; kw < s->kW - 1; ++kw)"),
    "conv_instead_of_correlation_1d": ("acc += w[c * K + k] * x[(b * T + s) * C + c];",
                                       "acc += w[c * K + (K - 1 - k)] * x[(b * T + s) * C + c];"),
    "dgrad_wrong_direction": ("dx[(b * T + s) * C + c] += w[c * K + k]",
                              "dx[(b * T + s) * C + c] += w[c * K + (K - 1 - k)]"),
    "wgrad_sign": ("acc += dy[(b * T_out + t) * C + c] * x[(b * T + s) * C + c];",
                   "acc -= dy[(b * T_out + t) * C + c] * x[(b * T + s) * C + c];"),
    "conv2d_dgrad_group_offset_dropped": ("dx[x_index(&s, n, g * cpg_in + ci, h, wi)]",
                                          "dx[x_index(&s, n, ci, h, wi)]"),
    "conv2d_dgrad_tap_flipped": ("+= w[w_index(&s, co, ci, kh, kw)] * d;",
                                 "+= w[w_index(&s, co, ci, kH - 1 - kh, kw)] * d;"),
    "conv2d_wgrad_group_stride": ("long c = (co / cpg_out) * cpg_in + ci;",
                                  "long c = (co / cpg_out) * cpg_out + ci;"),
    "conv2d_wgrad_dilation_dropped": ("long wi = wo * s->stride - s->pad + kw * s->dil;\n        if (wi < 0 || wi >= s->W) continue;\n        acc += dy",
                                      "long wi = wo * s->stride - s->pad + kw;\n        if (wi < 0 || wi >= s->W) continue;\n        acc += dy"),
    "conv2d_dgrad_points_stride_check": ("if (th < 0 || th % stride != 0 || th / stride >= s.Ho)",
                                         "if (th < 0 || th / stride >= s.Ho)"),
    "dwsep1d_bias_dropped": ("      double acc = bpw ? bpw[o] : 0.0;\n      for (long c = 0; c < C; ++c) acc += wpw[o * C + c] * y[r * C + c];",
                             "      double acc = 0.0;\n      for (long c = 0; c < C; ++c) acc += wpw[o * C + c] * y[r * C + c];"),
    "dwsep2d_channel_reversed": ("(n * HW + hw) * C + c;", "(n * HW + hw) * C + (C - 1 - c);"),
    "interleave_index_swapped": ("long co = i * cpg_out + j;", "long co = j * groups + i;"),
    "merge_max_is_min": ("else if (i == 0 || v > m) m = v;", "else if (i == 0 || v < m) m = v;"),
}


def _pins_pass():
    """A compact run of the pins above; returns False as soon as one fails."""
    try:
        for case in _tiny_cases()[:16]:
            for layout in (NCHW, NHWC):
                test_brute_force_conv2d(case, layout)
        for args in CONV1D_CASES:
            test_dwconv1d_fwd_brute_force(*args)
            test_dwconv1d_library_pins(*args)
        test_group_order_golden()
        for case in _tiny_cases()[:20]:
            test_conv2d_bwd_brute_force(case, NHWC)
        for case in BWD_CASES:
            test_conv2d_bwd_points_match_full(case, NCHW)
        for args in DWSEP1D_CASES:
            test_dwsep1d_brute_force(*args)
        test_dwsep2d_vs_torch(2, 1, 1, NHWC)
        test_interleaved_order_golden()
        for case in MERGE_CASES:
            test_interleaved_is_reshape_transpose(case, NCHW)
            test_group_merge_vs_numpy(case, "max", NCHW)
    except AssertionError:
        return False
    return True


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_planted_mistakes_are_caught(name, monkeypatch):
    old, new = MUTANTS[name]
    src = open(oracle._SRC).read()
    assert src.count(old) >= 1, name
    with tempfile.TemporaryDirectory() as d:
        path = os.path.join(d, "oracle_mutant.c")
        open(path, "w").write(src.replace(old, new, 1))
        so = os.path.join(d, "liboracle_mutant.so")
        subprocess.check_call(["gcc", "-O1", "-fPIC", "-shared", "-std=c99", path, "-o", so])
        monkeypatch.setattr(oracle, "_lib", oracle._configure(ctypes.CDLL(so)))
        assert not _pins_pass(), f"mutant {name} survived the pins"
    monkeypatch.undo()
    assert _pins_pass()
