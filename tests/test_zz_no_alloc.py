"""The allocation-free weight gradient, dwconv1d_bwd_weight_noalloc, called through the C ABI.

Some callers cannot allocate device memory (runtimes that forbid allocation once running,
plugins with no handle on the host's allocator); this entry point takes its scratch from a
fixed device array inside the library instead of a workspace. Both entry points run the same
fixed-slice kernels, so its dw must be bitwise the workspace entry point's dw (and, a fortiori,
within the bf16 tolerance used throughout: relative L2 <= 5e-3, max |err| <= 1e-2 * max |ref|)
on two calls in a row, and after a call on another shape that left different contents in
the shared array. This file sorts last so a failure here never hides the other GPU tests."""
import ctypes

import numpy as np
import pytest
import torch

from depthwise_convolution_gconv2d_b200 import binding as gb
from depthwise_convolution_gconv2d_b200 import workloads as wl
from _util import assert_close, to_dev, to_f64

pytestmark = pytest.mark.gpu


def same_bits(a, b):
    return torch.equal(a.contiguous().view(torch.int16), b.contiguous().view(torch.int16))


def call_noalloc(lib, x, dy, dw, p):
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    return lib.dwconv1d_bwd_weight_noalloc(
        ctypes.c_void_p(x.data_ptr()), ctypes.c_void_p(dy.data_ptr()),
        ctypes.c_void_p(dw.data_ptr()), p.B, p.T, p.C, p.K, p.pad_left, p.pad_right, p.dtype,
        stream)


@pytest.mark.parametrize("causal", [False, True])
def test_noalloc_wgrad_matches_workspace_entry_point(causal):
    lib = gb.load_library()
    p = wl.conformer_dw1d(causal)
    inp = wl.make_dwconv1d_inputs(p, 3)
    x, dy = to_dev(inp.x, p.dtype), to_dev(inp.dy, p.dtype)
    ref_t = gb.dwconv1d_bwd_weight(x, dy, p.K, p.pad_left, p.pad_right)
    ref = to_f64(ref_t)
    for _ in range(2):
        dw = torch.full((p.C, p.K), float("nan"), dtype=torch.bfloat16, device="cuda")
        assert call_noalloc(lib, x, dy, dw, p) == 0
        torch.cuda.synchronize()
        assert same_bits(dw, ref_t), "noalloc dw differs from the workspace entry point's"
        assert_close(to_f64(dw), ref, p.dtype, "noalloc vs workspace wgrad")


def test_noalloc_wgrad_small_shapes_two_calls():
    """Shapes of different sizes in a row: each call starts from what the previous, larger or
    smaller, call left in the shared array, and must still give the workspace entry point's
    dw bit for bit."""
    lib = gb.load_library()
    for case in [(8, 2048, 512, 31, 15, 15), (2, 300, 72, 31, 15, 15), (3, 50, 16, 3, 1, 1),
                 (2, 90, 5, 31, 15, 15), (4, 700, 64, 31, 30, 0)]:
        p = wl.Dwconv1dProblem(*case, wl.BF16)
        inp = wl.make_dwconv1d_inputs(p, 40)
        x, dy = to_dev(inp.x, p.dtype), to_dev(inp.dy, p.dtype)
        ref_t = gb.dwconv1d_bwd_weight(x, dy, p.K, p.pad_left, p.pad_right)
        ref = to_f64(ref_t)
        for _ in range(2):
            dw = torch.empty((p.C, p.K), dtype=torch.bfloat16, device="cuda")
            assert call_noalloc(lib, x, dy, dw, p) == 0
            torch.cuda.synchronize()
            assert same_bits(dw, ref_t), f"{case}: noalloc dw differs from the workspace one"
            assert_close(to_f64(dw), ref, p.dtype, str(case))


def test_noalloc_rejects_problems_beyond_the_fixed_scratch():
    lib = gb.load_library()
    limit = 4 * 1024 * 1024
    p = wl.Dwconv1dProblem(64, 2048, 4096, 31, 15, 15, wl.BF16)
    assert gb.dwconv1d_bwd_weight_workspace_size(p.B, p.T, p.C, p.K, 15, 15, p.dtype) > limit
    x = torch.zeros(16, dtype=torch.bfloat16, device="cuda")   # never read: rejected first
    dw = torch.zeros(16, dtype=torch.bfloat16, device="cuda")
    assert call_noalloc(lib, x, x, dw, p) == 4                 # GCONV_ERR_WORKSPACE
    assert torch.count_nonzero(dw) == 0
