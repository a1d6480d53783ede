"""CPU checks of the C ABI: the library loads, exports every entry point include/gconv.h
declares, and host-side validation rejects bad arguments before any CUDA call."""
import ctypes
import os
import re

import pytest

from depthwise_convolution_gconv2d_b200 import binding

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_functions():
    names = []
    for fn in sorted(os.listdir(os.path.join(ROOT, "include"))):
        if not fn.endswith(".h"):
            continue
        text = open(os.path.join(ROOT, "include", fn)).read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        names += re.findall(r"^[A-Za-z_][\w \*]*?\b([a-z_][a-z0-9_]*)\s*\(", text, flags=re.M)
    return sorted(set(names))


@pytest.fixture(scope="module")
def lib():
    from depthwise_convolution_gconv2d_b200 import build
    build.build()
    return binding.load_library()


def test_header_declares_the_boundary():
    names = declared_functions()
    for required in ("gconv2d_fwd", "dwconv1d_fwd", "dwconv1d_bwd_data", "dwconv1d_bwd_weight"):
        assert required in names


def test_every_declared_symbol_is_exported(lib):
    for name in declared_functions():
        assert hasattr(lib, name), f"libgconv.so does not export {name}"
    for name in binding.EXPORTS:
        assert name in declared_functions()


def test_status_strings(lib):
    for code, name in binding.STATUS.items():
        assert lib.gconv_status_string(code).decode() == name
    assert lib.gconv_status_string(99).decode() == "GCONV_ERR_UNKNOWN"
    assert lib.gconv_version() >= 100


CONV = dict(N=1, C_in=8, H=16, W=16, C_out=8, kH=3, kW=3, stride=1, pad=1, dil=1, groups=4)


def _conv_args(**over):
    a = dict(CONV, **over)
    return [a[k] for k in ("N", "C_in", "H", "W", "C_out", "kH", "kW", "stride", "pad", "dil",
                           "groups")]


@pytest.mark.parametrize("over", [dict(groups=3), dict(C_out=6), dict(groups=0), dict(kH=0),
                                  dict(stride=0), dict(pad=-1), dict(dil=0), dict(H=1, pad=0),
                                  dict(C_in=0), dict(N=-1), dict(W=2, kW=5, pad=1)])
def test_invalid_conv2d_rejected_before_launch(lib, over):
    args = _conv_args(**over)
    # fake, never-dereferenced pointers: validation must fail before any CUDA call
    p = ctypes.c_void_p(0x1000)
    st = lib.gconv2d_fwd(p, p, None, p, *args, 0, 2, None, 0, None)
    assert st == 1, binding.STATUS.get(st)
    assert lib.gconv2d_select_path(*args, 0, 2, 0) == -1
    assert lib.gconv2d_fwd_workspace_size(*args, 0, 2, 0) == 0


def test_null_pointers_and_bad_enums_rejected(lib):
    p = ctypes.c_void_p(0x1000)
    args = _conv_args()
    assert lib.gconv2d_fwd(None, p, None, p, *args, 0, 2, None, 0, None) == 1
    assert lib.gconv2d_fwd(p, p, None, None, *args, 0, 2, None, 0, None) == 1
    assert lib.gconv2d_fwd(p, p, None, p, *args, 2, 2, None, 0, None) == 1    # layout
    assert lib.gconv2d_fwd(p, p, None, p, *args, 0, 3, None, 0, None) == 1    # dtype
    assert lib.gconv2d_fwd_path(p, p, None, p, *args, 0, 2, 9, None, 0, None) == 1  # path
    assert lib.dwconv1d_fwd(None, p, p, 2, 8, 4, 3, 1, 1, 2, None) == 1
    assert lib.dwconv1d_fwd(p, p, p, 2, 8, 4, 20, 1, 1, 2, None) == 1           # T_out < 1
    assert lib.dwconv1d_bwd_data(p, p, p, 2, 8, 4, 3, -1, 1, 2, None) == 1
    assert lib.dwconv1d_bwd_weight(p, p, p, None, 0, 2, 8, 4, 3, 1, 1, 7, None) == 1
    code = ctypes.c_int(0)
    assert lib.gconv_get_device_error(None, None) == 1


def test_empty_batch_is_a_noop(lib):
    """N = 0 / B = 0: nothing to compute, nothing launched, OK returned."""
    p = ctypes.c_void_p(0x1000)
    assert lib.gconv2d_fwd(None, None, None, None, *_conv_args(N=0), 0, 2, None, 0, None) == 0
    assert lib.dwconv1d_fwd(None, None, None, 0, 8, 4, 3, 1, 1, 2, None) == 0


def test_path_selection(lib):
    sel = lambda path, **over: lib.gconv2d_select_path(*_conv_args(**over), over.get("layout", 0),
                                                       over.get("dtype", 2), path)
    # fp32 always runs the generic direct kernel under AUTO
    assert lib.gconv2d_select_path(*_conv_args(), 0, 0, 0) == 1
    # depthwise NHWC bf16 -> vectorised depthwise kernel
    assert lib.gconv2d_select_path(*_conv_args(C_in=64, C_out=64, groups=64), 1, 2, 0) == 2
    # depthwise NCHW has no vector kernel: generic
    assert lib.gconv2d_select_path(*_conv_args(C_in=64, C_out=64, groups=64), 0, 2, 0) == 1
    # forced generic
    assert lib.gconv2d_select_path(*_conv_args(C_in=64, C_out=64, groups=64), 1, 2, 3) == 1
    # the tensor-core path refuses fp32 and narrow groups
    assert lib.gconv2d_select_path(*_conv_args(), 1, 0, 2) == -2
    assert lib.gconv2d_select_path(*_conv_args(C_in=32, C_out=32, groups=8), 1, 2, 2) == -2


def test_wgrad_workspace_query(lib):
    n = lib.dwconv1d_bwd_weight_workspace_size(8, 2048, 512, 31, 15, 15, 2)
    assert n > 0 and n % 4 == 0
    assert lib.dwconv1d_bwd_weight_workspace_size(8, 2048, 512, 31, 15, 15, 0) == 0   # fp32: generic
    assert lib.dwconv1d_bwd_weight_workspace_size(8, 10, 512, 31, 0, 0, 2) == 0       # invalid


def test_conv1d_path_selection(lib):
    """dwconv1d_select_path: the tensor-core kernel (7) for 16-bit data with C % 16 == 0 and
    K <= 49, else the 128-byte-row CUDA-core kernel (20) for C % 64 == 0 and an instantiated
    K, else the CUDA-core ring kernel (6) where it is instantiated, else the generic kernel
    (5); DIRECT takes the 128-byte-row kernel first; a forced family that cannot run gives
    -UNSUPPORTED."""
    BF16, F32 = 2, 0
    sel = lambda B, T, C, K, pl, pr, dt, path: lib.dwconv1d_select_path(B, T, C, K, pl, pr, dt,
                                                                        path)
    conformer = (8, 2048, 512, 31, 15, 15, BF16)
    assert sel(*conformer, 0) == 7
    assert sel(*conformer, 1) == 20
    assert sel(*conformer, 2) == 7
    assert sel(*conformer, 3) == 5
    assert sel(8, 2048, 512, 33, 16, 16, BF16, 1) == 5          # K = 33: no strip instantiation
    assert sel(8, 2048, 96, 31, 15, 15, BF16, 1) == 6           # C % 64 != 0: ring kernel
    assert sel(8, 2048, 512, 31, 15, 15, F32, 0) == 5
    assert sel(8, 2048, 512, 31, 15, 15, F32, 2) == -2          # UNSUPPORTED
    assert sel(2, 300, 72, 31, 15, 15, BF16, 0) == 6            # C % 16 == 8: ring only
    assert sel(2, 300, 72, 31, 15, 15, BF16, 2) == -2
    assert sel(1, 500, 16, 17, 8, 8, BF16, 0) == 7              # K = 17: no ring instantiation
    assert sel(1, 500, 16, 17, 8, 8, BF16, 1) == 5
    assert sel(1, 500, 16, 50, 25, 24, BF16, 0) == 5            # K = 50: beyond the TC kernel
    assert sel(1, 500, 16, 50, 25, 24, BF16, 2) == -2
    assert sel(1, 8, 16, 31, 0, 0, BF16, 0) == -1               # T_out < 1: INVALID_ARG
    assert sel(*conformer, 9) == -1                             # unknown path
    # a forced path that cannot run is rejected before anything is launched
    assert lib.dwconv1d_fwd_path(None, None, None, 0, 8, 16, 3, 1, 1, F32, 2, None) == 2
    assert lib.dwconv1d_bwd_data_path(None, None, None, 0, 8, 16, 3, 1, 1, BF16, 9, None) == 1


def test_narrow_group_selection(lib):
    """2 / 4 / 8 channels per group, 3x3, stride 1 or 2, 16-bit NHWC -> the narrow-group
    CUDA-core kernel (8) under AUTO and DIRECT; anything else keeps its previous kernel."""
    NHWC, NCHW, BF16, F16, F32 = 1, 0, 2, 1, 0
    sel = lambda path, layout=NHWC, dtype=BF16, **over: lib.gconv2d_select_path(
        *_conv_args(**over), layout, dtype, path)
    for cpg in (2, 4, 8):
        kw = dict(C_in=64, C_out=64, groups=64 // cpg)
        assert sel(0, **kw) == 8 and sel(1, **kw) == 8
        assert sel(0, dtype=F16, **kw) == 8
        assert sel(0, stride=2, **kw) == 8
        assert sel(0, layout=NCHW, **kw) == 1             # NCHW: generic
        assert sel(0, dtype=F32, **kw) == 1               # fp32: generic
        assert sel(0, kH=5, kW=5, pad=2, **kw) == 1       # 5x5: generic
        assert sel(0, dil=2, pad=2, **kw) == 1            # dilation: generic
    assert sel(0, C_in=64, C_out=64, groups=4) == 3       # 16 per group: tensor cores
    assert sel(0, C_in=64, C_out=128, groups=16) != 8     # 4 in / 8 out: not narrow-group


# ------------------------------------------------------------ conv2d backward (host logic)

def test_bwd_invalid_and_workspace_rejected_before_launch(lib):
    p = ctypes.c_void_p(0x1000)
    for over in (dict(groups=3), dict(C_out=6), dict(stride=0), dict(H=1, pad=0)):
        args = _conv_args(**over)
        assert lib.gconv2d_bwd_data(p, p, p, *args, 1, 2, None, 0, None) == 1
        assert lib.gconv2d_bwd_weight(p, p, p, *args, 1, 2, None, 0, None) == 1
        assert lib.gconv2d_bwd_data_select_path(*args, 1, 2, 0) == -1
        assert lib.gconv2d_bwd_weight_workspace_size(*args, 1, 2, 0) == 0
    args = _conv_args(C_in=64, C_out=64, groups=64)
    assert lib.gconv2d_bwd_data(None, p, p, *args, 1, 2, None, 0, None) == 1
    assert lib.gconv2d_bwd_weight(p, p, None, *args, 1, 2, None, 0, None) == 1
    # a kernel that needs workspace, given none (or too little, or unaligned): WORKSPACE
    need = lib.gconv2d_bwd_data_workspace_size(*args, 1, 2, 0)
    assert need == 256 * ((64 * 9 * 2 + 255) // 256)
    assert lib.gconv2d_bwd_data(p, p, p, *args, 1, 2, None, 0, None) == 4
    assert lib.gconv2d_bwd_data(p, p, p, *args, 1, 2, p, need - 1, None) == 4
    assert lib.gconv2d_bwd_data(p, p, p, *args, 1, 2, ctypes.c_void_p(0x1004), need, None) == 4
    assert lib.gconv2d_bwd_weight(p, p, p, *args, 1, 2, None, 0, None) == 4
    # empty batch: the data gradient has nothing to write
    assert lib.gconv2d_bwd_data(None, None, None, *_conv_args(N=0), 1, 2, None, 0, None) == 0


def test_bwd_path_selection(lib):
    def sel(fn, N, C_in, H, W, C_out, k, s, pad, d, g, layout=1, dtype=2, path=0):
        return fn(N, C_in, H, W, C_out, k, k, s, pad, d, g, layout, dtype, path)
    dg, wg = lib.gconv2d_bwd_data_select_path, lib.gconv2d_bwd_weight_select_path
    # depthwise 56x56x1024: stride 1 runs the depthwise forward kernel on the flipped filter,
    # stride 2 (pad 1) the TMA-staged upsampling kernel, stride 2 with pad 2 the gather
    # kernel; the weight gradient has its own depthwise kernel
    assert sel(dg, 32, 1024, 56, 56, 1024, 3, 1, 1, 1, 1024) == 2
    assert sel(dg, 32, 1024, 56, 56, 1024, 3, 2, 1, 1, 1024) == 22
    assert sel(dg, 32, 1024, 56, 56, 1024, 3, 2, 2, 1, 1024) == 12
    assert sel(wg, 32, 1024, 56, 56, 1024, 3, 1, 1, 1, 1024) == 14
    assert sel(wg, 32, 1024, 56, 56, 1024, 3, 2, 1, 1, 1024) == 14
    assert sel(wg, 32, 1024, 56, 56, 1024, 3, 1, 3, 1, 1024) == 11   # pad 3: LDG kernel
    assert sel(wg, 32, 1024, 56, 56, 1024, 5, 1, 2, 1, 1024) == 11   # 5x5: LDG kernel
    # wide groups: tensor cores for both gradients (NHWC, NCHW staging); DIRECT keeps the
    # CUDA-core tiled weight gradient
    assert sel(dg, 1, 512, 256, 256, 512, 3, 1, 1, 1, 4) == 3
    assert sel(dg, 1, 512, 256, 256, 512, 3, 1, 1, 1, 4, layout=0) == 4
    assert sel(wg, 1, 512, 256, 256, 512, 3, 1, 1, 1, 4) == 18
    assert sel(wg, 1, 512, 256, 256, 512, 3, 1, 1, 1, 4, layout=0) == 19   # NCHW: staged
    assert sel(wg, 1, 512, 256, 256, 512, 3, 1, 1, 1, 4, path=2) == 18
    assert sel(wg, 1, 512, 256, 256, 512, 3, 1, 1, 1, 4, path=1) == 13
    assert sel(wg, 1, 512, 256, 256, 512, 3, 1, 1, 1, 4, layout=0, path=1) == 15
    assert sel(wg, 1, 512, 256, 256, 512, 3, 1, 1, 1, 4, path=3) == 10
    assert sel(wg, 1, 256, 64, 64, 128, 3, 1, 1, 1, 4) == 13          # 32 filters a group
    assert sel(wg, 1, 64, 56, 56, 64, 3, 1, 1, 1, 4) == 10          # 16 channels a group
    # narrow groups (4 channels): the narrow-group forward kernel
    assert sel(dg, 32, 1024, 56, 56, 1024, 3, 1, 1, 1, 256) == 8
    # depthwise with pad beyond dil*(k-1): the depthwise gather kernel; grouped: the generic
    # one, as for fp32 under AUTO and for GENERIC
    assert sel(dg, 1, 64, 16, 16, 64, 3, 1, 3, 1, 64) == 12
    assert sel(dg, 1, 64, 16, 16, 64, 3, 1, 3, 1, 16) == 9
    assert sel(dg, 1, 64, 16, 16, 64, 3, 1, 1, 1, 64, dtype=0) == 9
    assert sel(dg, 1, 512, 256, 256, 512, 3, 1, 1, 1, 4, path=3) == 9
    # forced IGEMM where the data gradient is not a stride-1 convolution, or on a weight
    # gradient the tensor-core kernel does not take (stride 2, 32 filters a group): UNSUPPORTED
    assert sel(dg, 1, 512, 64, 64, 512, 3, 2, 1, 1, 4, path=2) == -2
    assert sel(wg, 1, 512, 64, 64, 512, 3, 2, 1, 1, 4, path=2) == -2
    assert sel(wg, 1, 256, 64, 64, 128, 3, 1, 1, 1, 4, path=2) == -2


def test_bwd_workspace_queries(lib):
    # the flipped filter (rounded to 256 bytes), plus the NCHW staging of the exchanged problem
    wt = 512 * 128 * 9 * 2
    assert lib.gconv2d_bwd_data_workspace_size(1, 512, 256, 256, 512, 3, 3, 1, 1, 1, 4, 1, 2,
                                               0) == wt
    assert lib.gconv2d_bwd_data_workspace_size(1, 512, 256, 256, 512, 3, 3, 1, 1, 1, 4, 0, 2,
                                               0) == wt + lib.gconv2d_fwd_workspace_size(
        1, 512, 256, 256, 512, 3, 3, 1, 1, 1, 4, 0, 2, 0)
    # the gather kernels need none
    assert lib.gconv2d_bwd_data_workspace_size(32, 1024, 56, 56, 1024, 3, 3, 2, 1, 1, 1024, 1,
                                               2, 0) == 0
    assert lib.gconv2d_bwd_data_workspace_size(2, 12, 9, 8, 18, 3, 2, 1, 1, 1, 3, 1, 2, 0) == 0
    # weight gradient: fp32 partials, a whole number of slices of every dw entry
    for args in [(32, 1024, 56, 56, 1024, 3, 3, 1, 1, 1, 1024, 1, 2, 0),
                 (1, 512, 256, 256, 512, 3, 3, 1, 1, 1, 4, 1, 2, 0),
                 (2, 12, 9, 8, 18, 3, 2, 1, 1, 1, 3, 0, 0, 0)]:
        n = lib.gconv2d_bwd_weight_workspace_size(*args)
        E = args[4] * (args[1] // args[10]) * args[5] * args[6]
        assert n > 0 and n % (4 * E) == 0
    # NCHW wide groups: x and dy staged as NHWC (256-byte rounded) ahead of the partials
    nchw = (1, 512, 256, 256, 512, 3, 3, 1, 1, 1, 4, 0, 2, 0)
    n = lib.gconv2d_bwd_weight_workspace_size(*nchw)
    staged = 2 * (512 * 256 * 256 * 2)
    assert n > staged and (n - staged) % (4 * 512 * 128 * 9) == 0


def _enumerated_extent(size, k, stride, pad, dil):
    """Output positions counted one by one: o is an output when its whole window
    o*stride - pad + [0, dil*(k-1)] lies inside the zero-padded input [-pad, size + pad)."""
    n = 0
    while n * stride - pad + dil * (k - 1) <= size - 1 + pad:
        n += 1
    return n


def test_out_shape_query_matches_oracle_and_enumeration(lib):
    """gconv2d_out_shape / dwconv1d_out_steps (the binding allocates y and checks dy with
    them) agree with the oracle's output size and with counting window positions."""
    import oracle
    Cy, Ho, Wo = ctypes.c_int(-7), ctypes.c_int(-7), ctypes.c_int(-7)
    for size in (1, 2, 5, 7, 16, 57):
        for k in (1, 2, 3, 5):
            for s in (1, 2, 3):
                for p in (0, 1, 2):
                    for d in (1, 2):
                        want = _enumerated_extent(size, k, s, p, d)
                        assert oracle.out_extent(size, k, s, p, d) == want
                        st = lib.gconv2d_out_shape(2, 4, size, size + 1, 8, k, k, s, p, d, 2, 1, 2,
                                                   0, ctypes.byref(Cy), ctypes.byref(Ho),
                                                   ctypes.byref(Wo))
                        if want < 1:
                            assert st == 1
                            continue
                        assert st == 0
                        assert Ho.value == want
                        assert Wo.value == _enumerated_extent(size + 1, k, s, p, d)
    # argument errors reach the query too
    assert lib.gconv2d_out_shape(1, 6, 8, 8, 8, 3, 3, 1, 1, 1, 4, 1, 2, 0, ctypes.byref(Cy),
                                 ctypes.byref(Ho), ctypes.byref(Wo)) == 1   # 6 ch in 4 groups
    assert lib.gconv2d_out_shape(1, 8, 8, 8, 8, 3, 3, 1, 1, 1, 4, 1, 2, 0, None, None,
                                 None) == 1
    assert lib.gconv2d_out_shape(1, 8, 8, 8, 8, 3, 3, 1, 1, 1, 4, 1, 2, 4, ctypes.byref(Cy),
                                 ctypes.byref(Ho), ctypes.byref(Wo)) == 1   # no mode 4
    # channels of y: C_out for the orders, C_out / groups for the merges
    for mode, want in ((0, 12), (1, 12), (2, 3), (3, 3)):
        assert lib.gconv2d_out_shape(2, 8, 9, 9, 12, 3, 3, 2, 1, 1, 4, 1, 2, mode,
                                     ctypes.byref(Cy), ctypes.byref(Ho), ctypes.byref(Wo)) == 0
        assert (Cy.value, Ho.value, Wo.value) == (want, 5, 5)
    T_out = ctypes.c_int(0)
    for T, K, pl, pr in ((2048, 31, 15, 15), (2048, 31, 30, 0), (10, 3, 0, 0), (5, 9, 4, 4),
                         (3, 31, 15, 15)):
        st = lib.dwconv1d_out_steps(2, T, 8, K, pl, pr, 2, ctypes.byref(T_out))
        want = T + pl + pr - K + 1
        if want < 1:
            assert st == 1
        else:
            assert st == 0 and T_out.value == want
    assert binding.out_shape(1, 512, 256, 256, 512, 3, 3, 1, 1, 1, 4, "NHWC", 2) == (256, 256)
    assert binding.out_steps(8, 2048, 512, 31, 30, 0, 2) == 2048
    with pytest.raises(binding.GconvError):
        binding.out_shape(1, 8, 2, 2, 8, 5, 5, 1, 0, 1, 1, "NCHW", 2)


def test_binding_restates_no_shape_rule():
    """The binding is argument marshalling: output sizes come from the library's query, so
    the output-size formula appears nowhere in the package's Python code."""
    src = open(os.path.join(ROOT, "depthwise_convolution_gconv2d_b200", "binding.py")).read()
    assert "_out_extent" not in src
    assert "pad_left + pad_right - K" not in src
    assert "dilation * (k" not in src


def _declared_param_counts():
    counts = {}
    for fn in sorted(os.listdir(os.path.join(ROOT, "include"))):
        if not fn.endswith(".h"):
            continue
        text = open(os.path.join(ROOT, "include", fn)).read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        for m in re.finditer(r"^[A-Za-z_][\w \*]*?\b([a-z_][a-z0-9_]*)\s*\(([^)]*)\)\s*;", text,
                             flags=re.M | re.S):
            params = m.group(2).strip()
            counts[m.group(1)] = 0 if params in ("", "void") else params.count(",") + 1
    return counts


def test_binding_signatures_match_the_header(lib):
    """Every function the binding declares to ctypes takes as many arguments as the header
    says (a miscount would shift arguments at call time)."""
    counts = _declared_param_counts()
    for name in binding.EXPORTS:
        argtypes = getattr(lib, name).argtypes
        assert argtypes is not None, f"{name} has no argtypes"
        assert len(argtypes) == counts[name], (name, len(argtypes), counts[name])


def test_new_entry_points_validate_before_launch(lib):
    """The output-variant, depthwise-separable and test-hook entry points reject bad
    arguments on the host, with nothing launched (no GPU is touched here)."""
    P = None
    # gconv2d_fwd_out: bad mode, null pointers with N > 0, groups not dividing C
    assert lib.gconv2d_fwd_out(P, P, P, P, 1, 8, 8, 8, 8, 3, 3, 1, 1, 1, 2, 1, 2, 4, 0, P, 0,
                               P) == 1
    assert lib.gconv2d_fwd_out(P, P, P, P, 1, 8, 8, 8, 8, 3, 3, 1, 1, 1, 2, 1, 2, 1, 0, P, 0,
                               P) == 1
    assert lib.gconv2d_fwd_out(P, P, P, P, 0, 8, 8, 8, 8, 3, 3, 1, 1, 1, 2, 1, 2, 2, 0, P, 0,
                               P) == 0   # empty batch: a no-op
    assert lib.gconv2d_fwd_out(P, P, P, P, 1, 6, 8, 8, 8, 3, 3, 1, 1, 1, 4, 1, 2, 2, 0, P, 0,
                               P) == 1
    # variant selection: tensor cores for 16-bit problems the implicit GEMM takes, the generic
    # kernel otherwise; modes equal to the plain output take the ordinary kernels
    sel = lib.gconv2d_fwd_out_select_path
    assert sel(1, 512, 256, 256, 512, 3, 3, 1, 1, 1, 4, 1, 2, 1, 0) == 3
    assert sel(1, 512, 256, 256, 512, 3, 3, 1, 1, 1, 4, 0, 2, 2, 0) == 4
    assert sel(1, 512, 256, 256, 512, 3, 3, 1, 1, 1, 4, 1, 0, 3, 0) == 1    # fp32
    assert sel(1, 512, 256, 256, 512, 3, 3, 1, 1, 1, 4, 1, 2, 2, 1) == 1    # DIRECT: generic
    assert sel(32, 1024, 56, 56, 1024, 3, 3, 1, 1, 1, 1024, 1, 2, 1, 0) == 2  # depthwise
    assert sel(1, 12, 9, 9, 12, 3, 3, 1, 1, 1, 4, 1, 2, 2, 2) == -2         # IGEMM: 3 ch/group
    # depthwise-separable blocks
    assert lib.dwsep1d_select_path(8, 2048, 512, 31, 15, 15, 512, 2, 0) == 16
    assert lib.dwsep1d_select_path(8, 2048, 512, 31, 15, 15, 1024, 2, 0) == 17  # C_out > 512
    assert lib.dwsep1d_select_path(8, 2048, 512, 31, 15, 15, 1024, 2, 2) == -2
    assert lib.dwsep1d_select_path(8, 2048, 512, 31, 15, 15, 0, 2, 0) == -1     # C_out < 1
    assert lib.dwsep1d_fwd_workspace_size(8, 2048, 512, 31, 15, 15, 512, 2, 0) == 0
    assert lib.dwsep1d_fwd_workspace_size(8, 2048, 512, 31, 15, 15, 512, 2, 1) == \
        8 * 2048 * 512 * 2
    assert lib.dwsep1d_fwd(P, P, P, P, P, 2, 64, 64, 31, 15, 15, 64, 2, 0, P, 0, P) == 1
    assert lib.dwsep1d_fwd(P, P, P, P, P, 0, 64, 64, 31, 15, 15, 64, 2, 1, P, 0, P) == 0
    fake = ctypes.c_void_p(1 << 20)   # never dereferenced: the missing workspace is found first
    assert lib.dwsep1d_fwd(fake, fake, fake, P, fake, 2, 64, 64, 31, 15, 15, 64, 2, 1, P, 0,
                           P) == 4
    # AUTO: the fused kernel only when the depthwise output (N*Ho*Wo*C*2 bytes) exceeds 96 MB,
    # the composition when it stays in L2 between its two launches; IGEMM forces the kernel
    assert lib.dwsep2d_select_path(8, 256, 512, 80, 3, 3, 2, 1, 1, 256, 1, 2, 0) == 17   # 42 MB
    assert lib.dwsep2d_select_path(8, 256, 512, 80, 3, 3, 2, 1, 1, 256, 1, 2, 2) == 21
    assert lib.dwsep2d_select_path(8, 256, 1024, 256, 3, 3, 2, 1, 1, 256, 1, 2, 0) == 21  # 268 MB
    assert lib.dwsep2d_select_path(8, 256, 512, 40, 3, 3, 2, 1, 1, 256, 1, 2, 0) == 17  # Wo 20
    assert lib.dwsep2d_select_path(8, 256, 512, 40, 3, 3, 2, 1, 1, 256, 0, 2, 0) == 17   # NCHW
    assert lib.dwsep2d_select_path(8, 256, 512, 40, 7, 7, 2, 3, 1, 256, 1, 2, 2) == -2
    assert lib.dwsep2d_fwd(P, P, P, P, P, 1, 64, 8, 8, 3, 3, 1, 1, 1, 64, 1, 2, 0, P, 0, P) == 1
    # the bounded-wait test hook takes 16-byte multiples up to 64 KiB, and 0 restores
    assert lib.gconv_debug_set_tx_surplus(24) == 1
    assert lib.gconv_debug_set_tx_surplus(1 << 20) == 1
    assert lib.gconv_debug_set_tx_surplus(0) == 0
