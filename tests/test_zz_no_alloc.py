"""The no-allocation router entry point (moe_route_static) against moe_route.

moe_route_static serves callers that cannot allocate device memory (engine plug-ins without an
allocator, serving loops that may not call cudaMalloc on the request path): its scratch is a
fixed array inside the library.  Its outputs must equal moe_route's bit for bit, on two calls in
a row (the array keeps the previous call's contents), whether this file runs alone in a fresh
process or after every other test.  This file is named to be collected last.
"""
import ctypes
import math

import numpy as np
import pytest
import torch

import oracle
from expert_ffn_layer_router_b200 import inputs
from tests.gpu_util import to_dev, to_host

pytestmark = pytest.mark.gpu


def _outputs(p, dev):
    T, k, E = p.T, p.k, p.E
    return dict(ids=torch.full((T, k), -7, dtype=torch.int32, device=dev),
                w=torch.full((T, k), -7.0, dtype=torch.float32, device=dev),
                slot=torch.full((T, k), -7, dtype=torch.int32, device=dev),
                drop=torch.full((T, k), 7, dtype=torch.uint8, device=dev),
                counts=torch.full((2 * E,), -7, dtype=torch.int32, device=dev))


def _call_static(moe, p, logits, o):
    s = torch.cuda.current_stream().cuda_stream
    vp = ctypes.c_void_p
    return moe.lib().moe_route_static(ctypes.byref(p), vp(logits.data_ptr()),
                                      vp(o["ids"].data_ptr()), vp(o["w"].data_ptr()),
                                      vp(o["slot"].data_ptr()), vp(o["drop"].data_ptr()),
                                      vp(o["counts"].data_ptr()), vp(s))


def _check_pair(moe, spec_T, E, k, C, logits_np, flags=0):
    dev = torch.device("cuda:0")
    layer = moe.MoELayer(spec_T, 64, 64, E, k, C, "bf16", device=dev, flags=flags)
    logits = to_dev(logits_np)
    ref = layer.route(logits)                                   # the workspace entry point
    got = _outputs(layer.p, dev)
    assert _call_static(moe, layer.p, logits, got) == 0
    torch.cuda.synchronize()
    assert moe.moe_get_device_status(None) == 0                 # the static status word
    for name in ("ids", "slot", "drop", "counts"):
        assert torch.equal(got[name], ref[name]), name
    assert torch.equal(got["w"].view(torch.int32), ref["w"].view(torch.int32))
    return {n: to_host(v) for n, v in got.items()}


def test_static_route_matches_workspace_route_twice():
    from expert_ffn_layer_router_b200 import moe
    # First call: the skewed E=64 top-6 routing (experts overflow and drop).
    spec = inputs.CONFIGS["skewed_e64_top6"]
    L = inputs.make_layer(spec, seed=0, weights=False)
    lg = oracle.logits(L["x"], L["Wr"], L["br"])
    g1 = _check_pair(moe, spec.T, spec.E, spec.k, spec.C, lg)
    assert g1["drop"].sum() > 0
    # Second call, right after: a different, smaller problem reusing the same scratch.
    lg2 = inputs.random_logits(3000, 20, 5, 2.0)
    g2 = _check_pair(moe, 3000, 20, 3, 0.8, lg2)
    ro = oracle.route(lg2, 3, oracle.capacity(3000, 20, 3, 0.8))
    assert np.array_equal(g2["slot"], ro["slot"])


def test_static_route_rejects_problems_beyond_its_scratch():
    from expert_ffn_layer_router_b200 import moe
    p = moe.problem(65536, 4096, 1536, 128, 8, 1.5, "bf16")    # needs 32 MiB of candidates
    o = _outputs(moe.problem(1, 64, 64, 128, 8, 1.5, "bf16"), torch.device("cuda:0"))
    x = torch.zeros(1, device="cuda:0")
    assert _call_static(moe, p, x, o) == 3                       # MOE_ERR_WORKSPACE


@pytest.mark.parametrize("T,E,k,C,flags", [
    (64, 64, 8, math.inf, 0),       # decode shape: moe_route takes its single-block dispatch
    (8, 4, 1, 1.25, 0),             # the worked example's shape (token 4 is dropped)
    (100, 16, 4, 0.5, 0),           # small batch with drops
    (3000, 20, 3, 0.8, 1),          # renormalised weights
    (3000, 20, 3, 0.8, 2),          # arrival-order capacity
    (120, 10, 3, 0.6, 3),           # both flags, small batch
])
def test_static_route_matches_workspace_route_small_batches_and_flags(T, E, k, C, flags):
    from expert_ffn_layer_router_b200 import moe
    if (T, E) == (8, 4):
        L = inputs.make_layer(inputs.CONFIGS["tiny_f32"], seed=0)["logits"]
    else:
        L = inputs.random_logits(T, E, T + E + flags, 2.0)
    g = _check_pair(moe, T, E, k, C, L, flags=flags)
    ro = oracle.route(L, k, oracle.capacity(T, E, k, C), flags)
    assert np.array_equal(g["slot"], ro["slot"])
    assert np.array_equal(g["w"].view(np.uint32), ro["w"].view(np.uint32))
    if (T, E) == (8, 4):
        assert g["drop"][:, 0].tolist() == [0, 0, 0, 0, 1, 0, 0, 0]
