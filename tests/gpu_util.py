"""Helpers for the GPU parity tests: numpy <-> torch transfers and the comparison rules."""
import numpy as np
import torch

from expert_ffn_layer_router_b200 import inputs


def dev():
    return torch.device("cuda:0")


def to_dev(a):
    if a is None:
        return None
    if a.dtype == np.uint16:
        return torch.from_numpy(a.view(np.int16).copy()).view(torch.bfloat16).to(dev())
    return torch.from_numpy(np.ascontiguousarray(a).copy()).to(dev())


def to_host(t):
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).cpu().numpy().view(np.uint16)
    return t.cpu().numpy()


def as_f64(a):
    if a.dtype == np.uint16:
        return inputs.bf16_bits_to_f32(a).astype(np.float64)
    return a.astype(np.float64)


def tolerance(dtype, ref):
    """max|delta| allowed: 1e-5 for fp32 layers, 1e-2 * max|ref| + 1e-3 for bf16 layers."""
    if dtype == "f32":
        return 1e-5
    return 1e-2 * float(np.abs(ref).max()) + 1e-3


def assert_close(got, ref, dtype, what=""):
    g, r = as_f64(got), as_f64(ref)
    tol = tolerance(dtype, r)
    err = float(np.abs(g - r).max()) if g.size else 0.0
    assert err <= tol, "%s: max|delta| %.3g > tolerance %.3g" % (what, err, tol)
    return err
