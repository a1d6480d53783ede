"""The bounded waits' give-up path, made to run on the GPU without a fault.

Every mbarrier wait in the library's kernels gives up after 1 s, sets the device error word
and lets the CTA wind down: it drains its copies and MMAs (bounded by the same limit), frees
its tensor memory and exits. Here the test hook gconv_debug_set_tx_surplus makes the generic
tensor-core tile kernel declare 16 bytes per stage more than its TMA copies deliver, so no
stage ever completes: the call must end within a few seconds, gconv_get_device_error must
report GCONV_ERR_DEVICE_TIMEOUT, and the next normal call in the same process must again
match the fp64 oracle with no error reported. No trap, fault or unbounded wait is involved."""
import ctypes
import time

import pytest
import torch

import oracle
from depthwise_convolution_gconv2d_b200 import binding as gb
from depthwise_convolution_gconv2d_b200 import workloads as wl
from _util import assert_close, to_dev, to_f64

pytestmark = pytest.mark.gpu

# output rows of 12 pixels (narrower than 128, not a multiple of 8): the generic tile kernel
PROBLEM = wl.Conv2dProblem(1, 32, 12, 12, 32, 3, 3, 1, 1, 1, 2, wl.NHWC, wl.BF16)


def _run(p, x, w):
    return gb.gconv2d_fwd(x, w, None, p.stride, p.pad, p.dilation, p.groups, p.layout,
                          path=gb.PATH_IGEMM)


def test_bounded_wait_gives_up_and_the_context_stays_usable():
    lib = gb.load_library()
    p = PROBLEM
    assert gb.gconv2d_select_path(p.N, p.C_in, p.H, p.W, p.C_out, p.kH, p.kW, p.stride, p.pad,
                                  p.dilation, p.groups, p.layout, p.dtype,
                                  gb.PATH_IGEMM) == 3
    inp = wl.make_conv2d_inputs(p, 61)
    x, w = to_dev(inp.x, p.dtype), to_dev(inp.w, p.dtype)
    ref = oracle.conv2d(inp.x64(), inp.w64(), None, p.stride, p.pad, p.dilation, p.groups,
                        p.layout)
    assert gb.device_error() == 0
    assert lib.gconv_debug_set_tx_surplus(8) == 1            # not a multiple of 16
    assert lib.gconv_debug_set_tx_surplus(16) == 0
    try:
        t0 = time.time()
        _run(p, x, w)
        code = ctypes.c_int(0)
        st = lib.gconv_get_device_error(ctypes.c_void_p(torch.cuda.current_stream().cuda_stream),
                                        ctypes.byref(code))
        elapsed = time.time() - t0
    finally:
        assert lib.gconv_debug_set_tx_surplus(0) == 0
    assert st == 6, gb.STATUS.get(st, st)                    # GCONV_ERR_DEVICE_TIMEOUT
    assert code.value != 0
    assert elapsed < 30.0, f"the give-up path took {elapsed:.1f} s"
    # the word is cleared by the read, and the next call on the same context is correct
    assert gb.device_error() == 0
    y = _run(p, x, w)
    torch.cuda.synchronize()
    assert gb.device_error() == 0
    assert_close(to_f64(y), ref, p.dtype, "after a timed-out call")
