"""Host-only checks of the C ABI: the library loads, exports what the header declares, and
rejects malformed problems before launching anything.  No compute call needs a GPU here."""
import ctypes
import math
import os
import re

import pytest

import oracle
from expert_ffn_layer_router_b200 import build as lib_build
from expert_ffn_layer_router_b200 import inputs

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "moe_b200.h")


@pytest.fixture(scope="module")
def moe():
    lib_build.build()
    from expert_ffn_layer_router_b200 import moe as m
    return m


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(moe_[a-z_]+)\s*\(", text)))


def test_header_declares_the_calls():
    names = declared_functions()
    for n in ("moe_route", "moe_dispatch", "moe_expert_ffn", "moe_combine", "moe_forward",
              "moe_capacity", "moe_workspace_size"):
        assert n in names


def test_library_exports_every_declared_symbol(moe):
    lib = ctypes.CDLL(moe.LIB_PATH)
    for n in declared_functions():
        assert hasattr(lib, n), n
    assert set(moe.EXPORTS) == set(declared_functions())


@pytest.mark.parametrize("name", inputs.CONFIG_ORDER)
def test_capacity_matches_oracle(moe, name):
    s = inputs.CONFIGS[name]
    p = moe.problem(s.T, s.d_model, s.d_ff, s.E, s.k, s.C, s.dtype)
    assert moe.moe_capacity(p) == oracle.capacity(s.T, s.E, s.k, s.C)


def test_capacity_edges_match_oracle(moe):
    for T, E, k, C in [(8, 4, 1, 1.25), (10, 3, 1, 1.0), (100, 4, 2, 100.0), (100, 4, 2, 0.0),
                       (100, 4, 2, math.inf), (12345, 7, 3, 1.7)]:
        assert moe.moe_capacity(moe.problem(T, 64, 64, E, k, C, "bf16")) == \
            oracle.capacity(T, E, k, C)


def test_workspace_size_covers_buffers(moe):
    s = inputs.CONFIGS["skewed_e64_top6"]
    p = moe.problem(s.T, s.d_model, s.d_ff, s.E, s.k, s.C, s.dtype)
    n = moe.moe_workspace_size(p)
    rows = min(s.T * s.k, s.E * moe.moe_capacity(p))
    assert n >= rows * (s.d_ff + s.d_model) * 2 + s.T * s.E * 4
    assert n % 256 == 0


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_workspace_size_for_any_legal_shape(moe, dtype):
    """Sizing is host arithmetic only; every legal shape (widths the expert GEMMs reject
    included: moe_route and moe_combine take any width) gets a size, without a host fault."""
    for T in (0, 1, 7, 64, 128, 1000, 1024, 1025, 4096):
        for d in (1, 4, 8, 36, 64, 100, 192, 2112, 12288, 12352):
            for E, k in ((1, 1), (8, 2), (64, 8), (256, 4), (1024, 1)):
                n = moe.moe_workspace_size(moe.problem(T, d, 64, E, k, 1.25, dtype))
                assert n >= 256 and n % 256 == 0


@pytest.mark.parametrize("bad", [dict(k=5, E=4), dict(C=-1.0), dict(C=float("nan")),
                                 dict(E=0), dict(E=2000), dict(k=33, E=64), dict(T=-1),
                                 dict(dtype=7), dict(d=0)])
def test_malformed_problems_rejected(moe, bad):
    args = dict(T=16, d=64, F=64, E=4, k=2, C=1.0, dtype=1)
    args.update(bad)
    p = moe.Problem(args["T"], args["d"], args["F"], args["E"], args["k"], args["C"],
                    args["dtype"], 0)
    K = ctypes.c_int64()
    assert moe.lib().moe_capacity(ctypes.byref(p), ctypes.byref(K)) == 1
    n = ctypes.c_size_t()
    assert moe.lib().moe_workspace_size(ctypes.byref(p), ctypes.byref(n)) == 1
    rc = moe.lib().moe_forward(ctypes.byref(p), *([None] * 15), 0, None)
    assert rc == 1


def test_unknown_flags_rejected(moe):
    n = ctypes.c_size_t()
    for bad in (16, 32, 0x80000000):
        p = moe.Problem(16, 64, 64, 4, 2, 1.0, 1, bad)
        assert moe.lib().moe_workspace_size(ctypes.byref(p), ctypes.byref(n)) == 1
    for good in (0, moe.FLAG_RENORMALIZE, moe.FLAG_ARRIVAL_ORDER, moe.FLAG_GATED,
                 moe.FLAG_ROUTER_PREPARED, 15):
        p = moe.Problem(16, 64, 64, 4, 2, 1.0, 1, good)
        assert moe.lib().moe_workspace_size(ctypes.byref(p), ctypes.byref(n)) == 0


def test_status_strings(moe):
    for s in range(6):
        assert moe.lib().moe_status_string(s)
    assert moe.lib().moe_status_string(99) == b"unknown status"


def test_given_routing_and_logits_calls_reject_bad_arguments(moe):
    """moe_capacity_dispatch and moe_router_logits check their arguments before any launch."""
    lib = moe.lib()
    fake = ctypes.c_void_p(4096)                     # never dereferenced: rejected first
    p = moe.Problem(16, 64, 64, 4, 2, 1.0, 1, 0)
    bad = moe.Problem(16, 64, 64, 0, 2, 1.0, 1, 0)
    cd = lib.moe_capacity_dispatch
    # K < 0, a missing input, a malformed problem, rowtok without offsets: invalid argument.
    assert cd(ctypes.byref(p), -1, fake, fake, fake, fake, fake, None, None, fake, 1 << 20,
              None) == 1
    assert cd(ctypes.byref(p), 3, None, fake, fake, fake, fake, None, None, fake, 1 << 20,
              None) == 1
    assert cd(ctypes.byref(bad), 3, fake, fake, fake, fake, fake, None, None, fake, 1 << 20,
              None) == 1
    assert cd(ctypes.byref(p), 3, fake, fake, fake, fake, fake, None, fake, fake, 1 << 20,
              None) == 1
    # No workspace: MOE_ERR_WORKSPACE (3).
    assert cd(ctypes.byref(p), 3, fake, fake, fake, fake, fake, None, None, None, 0, None) == 3
    rl = lib.moe_router_logits
    assert rl(ctypes.byref(bad), fake, fake, None, fake, fake, 1 << 20, None) == 1
    assert rl(ctypes.byref(p), fake, None, None, fake, fake, 1 << 20, None) == 1
    assert rl(ctypes.byref(p), fake, fake, None, fake, None, 0, None) == 3


def test_prepare_router_rejects_bad_arguments(moe):
    lib = moe.lib()
    fake = ctypes.c_void_p(4096)
    p = moe.Problem(2048, 64, 64, 8, 2, 1.0, 1, 0)
    bad = moe.Problem(2048, 64, 64, 0, 2, 1.0, 1, 0)
    assert lib.moe_prepare_router(ctypes.byref(bad), fake, fake, 1 << 30, None) == 1
    assert lib.moe_prepare_router(ctypes.byref(p), None, fake, 1 << 30, None) == 1
    assert lib.moe_prepare_router(ctypes.byref(p), fake, None, 0, None) == 3


def test_bench_flag_word_matches_library_and_oracle(moe):
    """bench.py builds one flag word for the library and the oracle; the bits must mean the same
    thing on both sides."""
    import argparse
    import dataclasses
    import bench
    spec = inputs.CONFIGS["skewed_e64_top6"]
    ns = argparse.Namespace(renormalize=True, drop_policy="arrival")
    f = bench.layer_flags(dataclasses.replace(spec, gated=True), ns)
    assert f == moe.FLAG_RENORMALIZE | moe.FLAG_ARRIVAL_ORDER | moe.FLAG_GATED
    assert f == oracle.RENORMALIZE | oracle.ARRIVAL_ORDER | oracle.GATED
    assert bench.layer_flags(spec, argparse.Namespace(renormalize=False, drop_policy="weight")) == 0
    desc = bench.workload_desc(spec, f)
    assert "arrival-order capacity" in desc and "renormalised top-k weights" in desc
