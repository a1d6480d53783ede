"""Shared helpers for the parity tests: host<->device transfer of storage arrays and the
tolerance checks (relative L2 <= 1e-5 for fp32 and <= 5e-3 for bf16/fp16, plus
max|err| <= 1e-2 * max|ref|)."""
import numpy as np
import torch

from depthwise_convolution_gconv2d_b200 import workloads as wl

TORCH_DTYPE = {wl.F32: torch.float32, wl.F16: torch.float16, wl.BF16: torch.bfloat16}
REL_L2 = {wl.F32: 1e-5, wl.F16: 5e-3, wl.BF16: 5e-3}
MAX_ABS_FRAC = 1e-2


def to_dev(storage, dtype, device="cuda"):
    """Numpy storage array (float32, or uint16 bit patterns) -> CUDA tensor of `dtype`."""
    if storage is None:
        return None
    a = np.ascontiguousarray(storage)
    if dtype == wl.F32:
        return torch.from_numpy(a.astype(np.float32)).to(device)
    t = torch.from_numpy(a.view(np.int16)).to(device)
    return t.view(TORCH_DTYPE[dtype])


def to_f64(t):
    """CUDA tensor -> exact float64 numpy values."""
    if t.dtype == torch.float32:
        return t.detach().cpu().numpy().astype(np.float64)
    bits = t.detach().contiguous().view(torch.int16).cpu().numpy().view(np.uint16)
    return wl.widen(bits, wl.F16 if t.dtype == torch.float16 else wl.BF16)


def rel_l2(got, ref):
    den = np.linalg.norm(ref.ravel())
    num = np.linalg.norm((got - ref).ravel())
    return num / den if den > 0 else num


def assert_close(got, ref, dtype, what=""):
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    assert got.shape == ref.shape, (what, got.shape, ref.shape)
    assert np.all(np.isfinite(got)), f"{what}: non-finite output"
    r = rel_l2(got, ref)
    assert r <= REL_L2[dtype], f"{what}: relative L2 error {r:.3e} > {REL_L2[dtype]:.0e}"
    m = np.max(np.abs(got - ref)) if got.size else 0.0
    lim = MAX_ABS_FRAC * (np.max(np.abs(ref)) if ref.size else 0.0)
    assert m <= lim or m == 0.0, f"{what}: max |err| {m:.3e} > {lim:.3e}"
    return r, m
