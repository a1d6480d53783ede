"""Library calls captured into CUDA graphs give the same bits as the same calls run eagerly.

The kernels launched with programmatic stream serialization (tensor-core forward and weight
gradient, depthwise 3x3, the second kernel of two-kernel calls) become programmatic edges in a
captured graph, and the library's calls must stay capturable (no synchronous call, no
allocation the caller did not ask for). Every kernel here is deterministic, so a graph replay
must reproduce the eager result bit for bit -- twice in a row, with a whole forward and
backward sequence in one graph."""
import numpy as np
import pytest
import torch

from depthwise_convolution_gconv2d_b200 import binding as gb
from depthwise_convolution_gconv2d_b200 import workloads as wl
from _util import to_dev

pytestmark = pytest.mark.gpu


def same_bits(a, b):
    return torch.equal(a.contiguous().view(torch.int16), b.contiguous().view(torch.int16))


def conv2d_tensors(p, seed):
    inp = wl.make_conv2d_inputs(p, seed)
    x, w = to_dev(inp.x, p.dtype), to_dev(inp.w, p.dtype)
    dy = to_dev(wl.make_conv2d_dy(p, seed), p.dtype)
    return x, w, dy


def capture_and_replay(fns):
    """Run every fn(stream) eagerly, then capture them all in one graph on a side stream and
    replay it twice; returns (eager outputs, replay outputs) per fn."""
    eager = [fn(torch.cuda.current_stream(), False) for fn in fns]
    torch.cuda.synchronize()
    eager = [e.clone() for e in eager]
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        for fn in fns:                     # warm-up on the capture stream
            fn(side, True)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=side):
        outs = [fn(side, True) for fn in fns]
    replays = []
    for _ in range(2):
        for o in outs:
            o.zero_()
        torch.cuda.synchronize()
        g.replay()
        torch.cuda.synchronize()
        replays.append([o.clone() for o in outs])
    del g
    return eager, replays


def check(eager, replays, names):
    for rep in replays:
        for name, e, r in zip(names, eager, rep):
            assert same_bits(e, r), f"{name}: graph replay differs from the eager call"


def test_conv2d_forward_and_backward_graph():
    # row-strip GEMM (W >= 128, 128 filters per group), its NCHW form (staging + GEMM), the
    # halo GEMM (32-channel groups), the depthwise 3x3 kernel, the max merge (GEMM + max), the
    # depthwise data gradient (rotated filter) and the tensor-core weight gradient + sum
    pr = wl.Conv2dProblem(1, 256, 8, 160, 256, 3, 3, 1, 1, 1, 2, wl.NHWC, wl.BF16)
    pn = wl.Conv2dProblem(1, 256, 8, 160, 256, 3, 3, 1, 1, 1, 2, wl.NCHW, wl.BF16)
    ph = wl.Conv2dProblem(2, 128, 16, 16, 256, 3, 3, 1, 1, 1, 4, wl.NHWC, wl.BF16)
    pd = wl.Conv2dProblem(2, 128, 20, 24, 128, 3, 3, 1, 1, 1, 128, wl.NHWC, wl.BF16)
    xr, wr, dyr = conv2d_tensors(pr, 61)
    xn, wn, _ = conv2d_tensors(pn, 62)
    xh, wh, _ = conv2d_tensors(ph, 63)
    xd, wd, dyd = conv2d_tensors(pd, 64)
    bufs = {}

    def out(key, like):
        if key not in bufs:
            bufs[key] = torch.empty_like(like)
        return bufs[key]

    def scratch(key, nbytes):
        # allocated on the first (uncaptured) warm-up call, reused inside the capture
        if key not in bufs:
            bufs[key] = torch.empty(max(nbytes, 16), dtype=torch.uint8, device="cuda")
        return bufs[key]

    def fwd(p, x, w, key):
        def run(s, graph):
            y = gb.gconv2d_fwd(x, w, None, p.stride, p.pad, p.dilation, p.groups, p.layout,
                               stream=s) if not graph else None
            if graph:
                y = out(key, bufs[key + "_like"])
                ws_need = gb.gconv2d_fwd_workspace_size(p.N, p.C_in, p.H, p.W, p.C_out, p.kH,
                                                        p.kW, p.stride, p.pad, p.dilation,
                                                        p.groups, p.layout, p.dtype,
                                                        gb.PATH_AUTO)
                ws = scratch(key + "_ws", ws_need)
                gb.gconv2d_fwd(x, w, None, p.stride, p.pad, p.dilation, p.groups, p.layout,
                               out=y, workspace=ws, stream=s)
            else:
                bufs[key + "_like"] = y
            return y
        return run

    def fwd_max(p, x, w, key):
        def run(s, graph):
            if not graph:
                y = gb.gconv2d_fwd_out(x, w, None, p.stride, p.pad, p.dilation, p.groups,
                                       p.layout, "max", stream=s)
                bufs[key + "_like"] = y
                return y
            y = out(key, bufs[key + "_like"])
            need = gb.load_library().gconv2d_fwd_out_workspace_size(
                p.N, p.C_in, p.H, p.W, p.C_out, p.kH, p.kW, p.stride, p.pad, p.dilation,
                p.groups, p.layout, p.dtype, 3, gb.PATH_AUTO)
            ws = scratch(key + "_ws", need)
            gb.gconv2d_fwd_out(x, w, None, p.stride, p.pad, p.dilation, p.groups, p.layout,
                               "max", out=y, workspace=ws, stream=s)
            return y
        return run

    def dgrad(p, dy, w, key):
        def run(s, graph):
            if not graph:
                dx = gb.gconv2d_bwd_data(dy, w, (p.H, p.W), p.stride, p.pad, p.dilation,
                                         p.groups, p.layout, stream=s)
                bufs[key + "_like"] = dx
                return dx
            dx = out(key, bufs[key + "_like"])
            dims = (p.N, p.C_in, p.H, p.W, p.C_out, p.kH, p.kW, p.stride, p.pad, p.dilation,
                    p.groups, p.layout, p.dtype, gb.PATH_AUTO)
            ws = scratch(key + "_ws", gb.gconv2d_bwd_data_workspace_size(*dims))
            gb.gconv2d_bwd_data(dy, w, (p.H, p.W), p.stride, p.pad, p.dilation, p.groups,
                                p.layout, out=dx, workspace=ws, stream=s)
            return dx
        return run

    def wgrad(p, x, dy, key):
        def run(s, graph):
            if not graph:
                dw = gb.gconv2d_bwd_weight(x, dy, (p.kH, p.kW), p.stride, p.pad, p.dilation,
                                           p.groups, p.layout, stream=s)
                bufs[key + "_like"] = dw
                return dw
            dw = out(key, bufs[key + "_like"])
            dims = (p.N, p.C_in, p.H, p.W, p.C_out, p.kH, p.kW, p.stride, p.pad, p.dilation,
                    p.groups, p.layout, p.dtype, gb.PATH_AUTO)
            ws = scratch(key + "_ws", gb.gconv2d_bwd_weight_workspace_size(*dims))
            gb.gconv2d_bwd_weight(x, dy, (p.kH, p.kW), p.stride, p.pad, p.dilation, p.groups,
                                  p.layout, out=dw, workspace=ws, stream=s)
            return dw
        return run

    fns = [fwd(pr, xr, wr, "rowt"), fwd(pn, xn, wn, "nchw"), fwd(ph, xh, wh, "halo"),
           fwd(pd, xd, wd, "dw3x3"), fwd_max(pr, xr, wr, "max"), dgrad(pd, dyd, wd, "dgrad_dw"),
           wgrad(pr, xr, dyr, "wgrad_tc"), dgrad(pr, dyr, wr, "dgrad_rowt")]
    names = ["row-strip", "NCHW", "halo", "depthwise 3x3", "max merge", "depthwise dgrad",
             "tensor-core wgrad", "row-strip dgrad"]
    eager, replays = capture_and_replay(fns)
    check(eager, replays, names)


def test_conv1d_graph():
    # tensor-core conv1d forward and data gradient, and the 128-byte-row weight gradient
    # followed by its fixed-order run sum
    p = wl.Dwconv1dProblem(2, 300, 128, 31, 15, 15, wl.BF16)
    inp = wl.make_dwconv1d_inputs(p, 65)
    x, w, dy = to_dev(inp.x, p.dtype), to_dev(inp.w, p.dtype), to_dev(inp.dy, p.dtype)
    need = gb.dwconv1d_bwd_weight_workspace_size(p.B, p.T, p.C, p.K, p.pad_left, p.pad_right,
                                                 p.dtype)
    ws = torch.empty(max(need, 16), dtype=torch.uint8, device="cuda")
    bufs = {}

    def keep(key, t, graph):
        if not graph:
            bufs[key] = torch.empty_like(t)
        return bufs[key]

    def fwd(s, graph):
        if not graph:
            y = gb.dwconv1d_fwd(x, w, p.pad_left, p.pad_right, stream=s)
            keep("y", y, False)
            return y
        return gb.dwconv1d_fwd(x, w, p.pad_left, p.pad_right, out=bufs["y"], stream=s)

    def dgrad(s, graph):
        if not graph:
            dx = gb.dwconv1d_bwd_data(dy, w, p.T, p.pad_left, p.pad_right, stream=s)
            keep("dx", dx, False)
            return dx
        return gb.dwconv1d_bwd_data(dy, w, p.T, p.pad_left, p.pad_right, out=bufs["dx"],
                                    stream=s)

    def wgrad(s, graph):
        if not graph:
            dw = gb.dwconv1d_bwd_weight(x, dy, p.K, p.pad_left, p.pad_right, workspace=ws,
                                        stream=s)
            keep("dw", dw, False)
            return dw
        return gb.dwconv1d_bwd_weight(x, dy, p.K, p.pad_left, p.pad_right, out=bufs["dw"],
                                      workspace=ws, stream=s)

    eager, replays = capture_and_replay([fwd, dgrad, wgrad])
    check(eager, replays, ["conv1d forward", "conv1d data gradient", "conv1d weight gradient"])
    assert np.isfinite(eager[0].float().cpu().numpy()).all()
