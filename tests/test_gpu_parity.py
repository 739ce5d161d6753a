"""CUDA path vs CPU oracle, through the C ABI.

Routing (ids, weights, slots, drop flags, counts) and the dispatch layout must match bit for
bit given the same fp32 logits; float outputs must be within 1e-5 (fp32 layers) or
1e-2 * max|ref| + 1e-3 (bf16 layers, fp32 accumulation); a token whose pairs were all dropped
must come out bit for bit equal to its input.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from expert_ffn_layer_router_b200 import inputs
from tests.gpu_util import assert_close, to_dev, to_host

pytestmark = pytest.mark.gpu


def _moe():
    from expert_ffn_layer_router_b200 import moe
    return moe


def _route_both(L, T, E, k, C, dtype="bf16", d=64, F=64, flags=0):
    moe = _moe()
    layer = moe.MoELayer(T, d, F, E, k, C, dtype, flags=flags)
    r = layer.route(to_dev(L))
    torch.cuda.synchronize()
    assert moe.moe_get_device_status(layer.ws) == 0
    ro = oracle.route(L, k, layer.K, flags)
    return layer, {k_: to_host(v) for k_, v in r.items()}, ro


def _assert_route_equal(g, ro, E):
    assert np.array_equal(g["ids"], ro["ids"]), "expert ids differ"
    assert np.array_equal(g["w"].view(np.uint32), ro["w"].view(np.uint32)), "weights differ"
    assert np.array_equal(g["slot"], ro["slot"]), "slot map differs"
    assert np.array_equal(g["drop"], ro["drop"]), "drop mask differs"
    assert np.array_equal(g["counts"][:E], ro["received"]), "received counts differ"
    assert np.array_equal(g["counts"][E:], ro["kept"]), "kept counts differ"


# ------------------------------------------------------------------------------------------
# Routing, bit for bit, on the five workloads (logits from the oracle's x Wr + br).
# ------------------------------------------------------------------------------------------
@pytest.mark.parametrize("name", inputs.CONFIG_ORDER)
def test_route_configs_bit_exact(name):
    spec = inputs.CONFIGS[name]
    L = inputs.make_layer(spec, seed=0, weights=False)
    logits = L["logits"] if L["logits"] is not None else oracle.logits(L["x"], L["Wr"], L["br"])
    _, g, ro = _route_both(logits, spec.T, spec.E, spec.k, spec.C)
    _assert_route_equal(g, ro, spec.E)
    if name == "skewed_e64_top6":
        assert ro["drop"].sum() > 0, "the skewed workload must overflow some experts"


@pytest.mark.parametrize("T,E,k,C,scale,seed", [
    (1, 4, 1, 1.0, 1.0, 0), (7, 5, 2, 0.5, 1.0, 1), (300, 33, 3, 1.0, 2.0, 2),
    (1000, 100, 8, 1.0, 1.5, 3), (257, 1024, 32, 2.0, 1.0, 4), (513, 32, 32, 1.0, 1.0, 5),
    (4000, 8, 2, 0.0, 1.0, 6), (3000, 16, 4, math.inf, 1.0, 7), (2048, 1, 1, 0.5, 1.0, 8),
    (5000, 64, 6, 0.3, 3.0, 9)])
def test_route_shapes_bit_exact(T, E, k, C, scale, seed):
    L = inputs.random_logits(T, E, seed, scale)
    _, g, ro = _route_both(L, T, E, k, C)
    _assert_route_equal(g, ro, E)


def test_route_all_tokens_to_one_expert():
    T, E, k = 5000, 16, 2
    L = inputs.random_logits(T, E, 11, 0.5)
    L[:, 7] += 20.0
    _, g, ro = _route_both(L, T, E, k, 1.0)
    _assert_route_equal(g, ro, E)
    assert ro["received"][7] == T and ro["kept"][7] == 625


def test_route_weight_ties():
    # Identical rows give identical weights; the lower token index must win every tie.
    rng = np.random.default_rng(3)
    proto = rng.standard_normal((4, 12)).astype(np.float32)
    L = proto[rng.integers(0, 4, size=3000)]
    _, g, ro = _route_both(L, 3000, 12, 3, 0.7)
    _assert_route_equal(g, ro, 12)


def test_route_tie_bin_larger_than_a_block():
    # Every token has the same logits: one expert receives all 3000 pairs with the same weight,
    # more than one block of equal keys at the capacity boundary; the lower tokens are kept.
    T, E, k = 3000, 2, 1
    L = np.zeros((T, E), np.float32)
    _, g, ro = _route_both(L, T, E, k, 0.5)
    _assert_route_equal(g, ro, E)
    assert ro["kept"][0] == 750 and (ro["slot"][:750, 0] == np.arange(750)).all()


def test_route_large_batch_global_bitmap():
    # More than 262144 tokens: the capacity selection keeps its token bitmap in the workspace.
    T, E, k = 300000, 4, 2
    L = inputs.random_logits(T, E, 12, 1.0)
    _, g, ro = _route_both(L, T, E, k, 0.5)
    _assert_route_equal(g, ro, E)
    assert ro["drop"].sum() > 0


def test_route_empty():
    moe = _moe()
    layer = moe.MoELayer(0, 64, 64, 8, 2, 1.0, "bf16")
    counts = torch.full((16,), 7, dtype=torch.int32, device="cuda")
    moe.moe_route(layer.p, None, None, None, None, None, counts, layer.ws)
    torch.cuda.synchronize()
    assert (counts == 0).all()


# ------------------------------------------------------------------------------------------
# Dispatch layout and the permuted buffer.
# ------------------------------------------------------------------------------------------
@pytest.mark.parametrize("T,E,k,C,dtype", [(777, 6, 2, 0.8, "bf16"), (64, 64, 8, math.inf, "bf16"),
                                           (300, 5, 3, 0.5, "f32")])
def test_dispatch_bit_exact(T, E, k, C, dtype):
    moe = _moe()
    d = 64
    L = inputs.random_logits(T, E, T)
    K = oracle.capacity(T, E, k, C)
    ro = oracle.route(L, k, K)
    off_ref, rowtok_ref = oracle.dispatch(ro["ids"], ro["slot"], E)
    layer = moe.MoELayer(T, d, 64, E, k, C, dtype)
    rng = np.random.default_rng(0)
    x = rng.standard_normal((T, d)).astype(np.float32)
    if dtype == "bf16":
        x = inputs.f32_to_bf16_bits(x)
    xd = to_dev(x)
    offs, rowtok, xp = layer.dispatch(to_dev(ro["ids"]), to_dev(ro["slot"]), x=xd, permute=True)
    torch.cuda.synchronize()
    n = int(off_ref[-1])
    assert np.array_equal(to_host(offs), off_ref)
    assert np.array_equal(to_host(rowtok)[:n], rowtok_ref)
    assert np.array_equal(to_host(xp)[:n], x[rowtok_ref])


# ------------------------------------------------------------------------------------------
# Expert FFN (tensor cores for bf16, CUDA cores for fp32) against the oracle's double FFN.
# ------------------------------------------------------------------------------------------
@pytest.mark.parametrize("T,d,F,E,k,C,dtype,bias", [
    (300, 128, 192, 5, 2, 1.0, "bf16", 0.05),      # ragged experts, one column tile
    (1000, 256, 1408, 4, 1, 1.25, "bf16", 0.02),   # d_ff = 1408: 256-wide tiles, the last half full
    (700, 512, 320, 3, 3, 0.9, "bf16", 0.0),       # several m-tiles per expert, a ragged column tile
    (129, 64, 64, 2, 1, math.inf, "bf16", 0.1),    # 129 rows: one full tile + one row
    (2000, 256, 1408, 4, 2, 1.25, "bf16", 0.02),   # gathered rows, half-width last tile
    (2000, 640, 256, 4, 2, 1.25, "bf16", 0.02),    # second GEMM on CTA pairs, half-width last tile
    (1024, 128, 192, 4, 1, math.inf, "bf16", 0.05),  # exactly 256 rows per expert: pairs
    (1023, 128, 192, 4, 1, math.inf, "bf16", 0.05),  # one row short of that: single-CTA tiles
    # Weight streaming (at most 64 rows per expert on average): 64-row m-tiles.
    (700, 256, 320, 16, 1, math.inf, "bf16", 0.05),  # experts above 64 rows: two m-tiles
    (200, 128, 192, 8, 2, math.inf, "bf16", 0.05),   # ragged 64-row tiles, half-width last tile
    (128, 64, 64, 2, 1, math.inf, "bf16", 0.1),      # 128 rows over two experts
    (64, 2048, 1024, 64, 8, math.inf, "bf16", 0.0),  # the decode shape
    (40, 16, 24, 4, 2, 1.0, "f32", 0.1),
    (8, 4, 8, 4, 1, 1.25, "f32", 0.1)])
def test_expert_ffn_parity(T, d, F, E, k, C, dtype, bias):
    moe = _moe()
    spec = inputs.LayerSpec("ffn", T, d, F, E, k, C, dtype, router="normal", router_bias=0.5,
                            bias_std=bias)
    L = inputs.make_layer(spec, seed=T)
    logits = oracle.logits(L["x"], L["Wr"], L["br"])
    K = oracle.capacity(T, E, k, C)
    ro = oracle.route(logits, k, K)
    off_ref, rowtok_ref = oracle.dispatch(ro["ids"], ro["slot"], E)
    n = int(off_ref[-1])
    row_exp = np.repeat(np.arange(E, dtype=np.int32), np.diff(off_ref))
    Yref = oracle.expert_rows(L["x"], L["W1"], L["b1"], L["W2"], L["b2"], rowtok_ref, row_exp)
    layer = moe.MoELayer(T, d, F, E, k, C, dtype)
    Y = layer.expert_ffn(to_dev(L["x"]), to_dev(off_ref), to_dev(rowtok_ref), to_dev(L["W1"]),
                         to_dev(L["b1"]), to_dev(L["W2"]), to_dev(L["b2"]))
    torch.cuda.synchronize()
    assert moe.moe_get_device_status(layer.ws) == 0
    assert_close(to_host(Y)[:n], Yref, dtype, "expert outputs")


# ------------------------------------------------------------------------------------------
# Combine given expert outputs.
# ------------------------------------------------------------------------------------------
@pytest.mark.parametrize("T,d,E,k,C,dtype", [(500, 256, 8, 2, 0.6, "bf16"),
                                             (300, 40, 5, 3, 0.5, "f32"),
                                             (200, 36, 4, 2, 0.5, "bf16"),   # unvectorised path
                                             (100, 6, 3, 1, 0.5, "f32")])
def test_combine_parity(T, d, E, k, C, dtype):
    moe = _moe()
    L = inputs.random_logits(T, E, d)
    K = oracle.capacity(T, E, k, C)
    ro = oracle.route(L, k, K)
    off, _ = oracle.dispatch(ro["ids"], ro["slot"], E)
    rng = np.random.default_rng(T + d)
    x = rng.standard_normal((T, d)).astype(np.float32)
    Y = rng.standard_normal((max(int(off[-1]), 1), d)).astype(np.float32)
    if dtype == "bf16":
        x, Y = inputs.f32_to_bf16_bits(x), inputs.f32_to_bf16_bits(Y)
    none_kept = ~(ro["slot"] >= 0).any(axis=1)
    t0 = int(np.nonzero(none_kept)[0][0])
    x[t0, 0] = 0x8000 if dtype == "bf16" else np.float32(-0.0)
    _, ref = oracle.combine_given_y(x, Y, ro, off)
    layer = moe.MoELayer(T, d, 64, E, k, C, dtype)
    out = layer.combine(to_dev(x), to_dev(Y), to_dev(ro["w"]), to_dev(ro["ids"]),
                        to_dev(ro["slot"]), to_dev(off))
    torch.cuda.synchronize()
    got = to_host(out)
    assert got[none_kept].tobytes() == x[none_kept].tobytes(), "dropped tokens must pass through"
    assert_close(got, ref, dtype, "combine")


# ------------------------------------------------------------------------------------------
# The whole forward against the oracle's whole layer.
# ------------------------------------------------------------------------------------------
def _assert_forward_route_equal(g, ro, E):
    """The forward's exported routing against the oracle's routing of the same fp32 logits."""
    assert np.array_equal(g["ids_out"], ro["ids"]), "expert ids differ"
    assert np.array_equal(g["w_out"].view(np.uint32), ro["w"].view(np.uint32)), "weights differ"
    assert np.array_equal(g["slot_out"], ro["slot"]), "slot map differs"
    assert np.array_equal(g["drop_out"], ro["drop"]), "drop mask differs"
    assert np.array_equal(g["counts_out"][:E], ro["received"]), "received counts differ"
    assert np.array_equal(g["counts_out"][E:], ro["kept"]), "kept counts differ"


def _forward_check(spec, seed, tokens=None, logit_rel=1e-4, flags=0):
    """The whole forward against the oracle.

    1. logits_out within logit_rel * max(1, max|L|) of the oracle's float64 x Wr + br;
    2. routing (ids, weight bits, slots, drop mask, counts) bit for bit equal to the oracle's
       routing of the forward's own exported fp32 logits (routing is a function of the logits);
    3. outputs of ``tokens`` (all by default) within the dtype's tolerance of the oracle's
       layer given that routing; tokens with no kept pair bit for bit equal to x;
    4. against the oracle's routing of its own logits: the same expert sets, and capacity
       decisions that differ only where the oracle's weights tie within the logit error at an
       expert's capacity boundary (the logits differ by rounding).
    """
    moe = _moe()
    L = inputs.make_layer(spec, seed=seed)
    layer = moe.MoELayer(spec.T, spec.d_model, spec.d_ff, spec.E, spec.k, spec.C, spec.dtype,
                         flags=flags)
    args = [to_dev(L[n]) for n in ("x", "Wr", "br", "W1", "b1", "W2", "b2")]
    out, rt = layer.forward(*args, want_routing=True)
    torch.cuda.synchronize()
    assert moe.moe_get_device_status(layer.ws) == 0
    g = {k_: to_host(v) for k_, v in rt.items()}
    Lref = oracle.logits(L["x"], L["Wr"], L["br"])
    lerr = np.abs(g["logits_out"] - Lref).max()
    assert lerr <= logit_rel * max(1.0, float(np.abs(Lref).max())), lerr
    rg = oracle.route(g["logits_out"], spec.k, layer.K, flags & 3)
    _assert_forward_route_equal(g, rg, spec.E)
    T = spec.T
    if tokens is None:
        tokens = np.arange(T, dtype=np.int32)
    tokens = np.asarray(tokens, dtype=np.int32)
    _, ref = oracle.combine_tokens(L["x"], L["W1"], L["b1"], L["W2"], L["b2"], rg, tokens,
                                   flags=flags)
    got = to_host(out)
    assert_close(got[tokens], ref, spec.dtype, "layer output")
    none_kept = ~(rg["slot"] >= 0).any(axis=1)
    assert got[none_kept].tobytes() == L["x"][none_kept].tobytes()
    # Against the routing of the oracle's own logits.
    ro = oracle.route(Lref, spec.k, layer.K, flags & 3)
    og = np.argsort(g["ids_out"], axis=1, kind="stable")
    oo = np.argsort(ro["ids"], axis=1, kind="stable")
    gi, gw, gs = (np.take_along_axis(g[n], og, 1) for n in ("ids_out", "w_out", "slot_out"))
    oi, ow, os_ = (np.take_along_axis(ro[n], oo, 1) for n in ("ids", "w", "slot"))
    assert np.array_equal(gi, oi), "expert sets differ"
    dw = np.abs(gw - ow)
    assert dw.max() <= 4 * lerr * max(1.0, float(ow.max())) + 1e-6
    mism = np.nonzero((gs >= 0) != (os_ >= 0))
    for t, j in zip(*mism):
        e = oi[t, j]
        same_e = oi == e
        kept_w = ow[same_e & (os_ >= 0)]
        drop_w = ow[same_e & (os_ < 0)]
        boundary = (kept_w.min() + drop_w.max()) / 2
        assert abs(float(ow[t, j]) - boundary) <= 8 * dw.max() + 1e-7, "not a near-tie"
    assert ((gs >= 0) == (os_ >= 0)).all(axis=1).mean() >= 0.99
    return g, rg


@pytest.mark.parametrize("spec", [
    inputs.LayerSpec("s1", 300, 128, 192, 5, 2, 1.0, "bf16", router="normal", router_bias=0.5,
                     bias_std=0.05),
    inputs.LayerSpec("s2", 1000, 256, 1408, 8, 3, 0.75, "bf16", router="zipf", router_bias=1.1),
    inputs.LayerSpec("s3", 513, 64, 128, 33, 4, 1.0, "bf16", router="normal", router_bias=1.0,
                     bias_std=0.01),
    inputs.LayerSpec("s4", 64, 128, 64, 16, 8, math.inf, "bf16"),
    inputs.LayerSpec("s5", 200, 32, 48, 6, 2, 0.8, "f32", router="normal", router_bias=0.5,
                     bias_std=0.1),
    inputs.LayerSpec("s6", 256, 64, 64, 4, 2, 0.0, "bf16")])
def test_forward_small(spec):
    _forward_check(spec, seed=5)


def test_forward_worked_example_f32():
    moe = _moe()
    spec = inputs.CONFIGS["tiny_f32"]
    L = inputs.make_layer(spec, seed=0)
    layer = moe.MoELayer(8, 4, 8, 4, 1, 1.25, "f32")
    r = layer.route(to_dev(L["logits"]))
    offs, rowtok, _ = layer.dispatch(r["ids"], r["slot"])
    x = to_dev(L["x"])
    Y = layer.expert_ffn(x, offs, rowtok, to_dev(L["W1"]), to_dev(L["b1"]), to_dev(L["W2"]),
                         to_dev(L["b2"]))
    out = layer.combine(x, Y, r["w"], r["ids"], r["slot"], offs)
    torch.cuda.synchronize()
    ro = oracle.route(L["logits"], 1, 2)
    assert to_host(r["drop"])[:, 0].tolist() == [0, 0, 0, 0, 1, 0, 0, 0]
    _, ref = oracle.combine_tokens(L["x"], L["W1"], L["b1"], L["W2"], L["b2"], ro)
    got = to_host(out)
    assert_close(got, ref, "f32", "worked example")
    assert got[4].tobytes() == L["x"][4].tobytes()


def test_unsupported_and_invalid():
    moe = _moe()
    with pytest.raises(moe.MoeError) as ei:
        moe.MoELayer(16, 100, 64, 4, 2, 1.0, "bf16").forward(
            *[torch.zeros(1, device="cuda")] * 7)
    assert ei.value.status in (1, 2)


# ------------------------------------------------------------------------------------------
# The forward's routing (the router that also places the pairs in candidate lists, then the
# histogram-based capacity selection; or the small-batch router and dispatch) must equal, bit
# for bit, both moe_route's and the oracle's routing of the logits the forward exported.
# ------------------------------------------------------------------------------------------
@pytest.mark.parametrize("T,d,E,k,C", [(3000, 128, 64, 6, 1.0), (1000, 256, 8, 2, 1.25),
                                       (777, 64, 33, 4, 0.75), (200, 64, 16, 8, math.inf),
                                       (5000, 64, 64, 6, 0.5), (129, 64, 1, 1, 1.0)])
@pytest.mark.parametrize("flags", [0, 1, 3])
def test_forward_routing_matches_route(T, d, E, k, C, flags):
    moe = _moe()
    spec = inputs.LayerSpec("fwd_route", T, d, 64, E, k, C, "bf16", router="normal",
                            router_bias=0.5)
    L = inputs.make_layer(spec, seed=E + T)
    layer = moe.MoELayer(T, d, 64, E, k, C, "bf16", flags=flags)
    args = [to_dev(L[n]) for n in ("x", "Wr", "br", "W1", "b1", "W2", "b2")]
    _, rt = layer.forward(*args, want_routing=True)
    r = layer.route(rt["logits_out"])
    torch.cuda.synchronize()
    assert moe.moe_get_device_status(layer.ws) == 0
    assert torch.equal(rt["ids_out"], r["ids"])
    assert torch.equal(rt["w_out"].view(torch.int32), r["w"].view(torch.int32))
    assert torch.equal(rt["slot_out"], r["slot"])
    assert torch.equal(rt["drop_out"], r["drop"])
    assert torch.equal(rt["counts_out"], r["counts"])
    g = {k_: to_host(v) for k_, v in rt.items()}
    ro = oracle.route(g["logits_out"], k, layer.K, flags & 3)
    _assert_forward_route_equal(g, ro, E)


# ------------------------------------------------------------------------------------------
# Capacity dispatch of a given routing (moe_capacity_dispatch) against the oracle's selection,
# and the router logits alone (moe_router_logits) against the forward's own logits.
# ------------------------------------------------------------------------------------------
def _given_routing(T, E, k, seed, ties):
    rng = np.random.default_rng(seed)
    ids = np.argsort(rng.random((T, E)), axis=1)[:, :k].astype(np.int32)
    if ties:
        w = (rng.integers(1, 5, size=(T, k)) * 0.125).astype(np.float32)
    else:
        w = rng.random((T, k)).astype(np.float32)
    return ids, w


@pytest.mark.parametrize("T,E,k,K,flags,ties", [
    (300, 8, 2, 50, 0, True),           # single-block path (T k <= 1024)
    (512, 64, 2, 9, 2, False),          # single-block path, arrival order
    (3000, 64, 6, 200, 0, False),       # candidate lists + histogram selection
    (3000, 64, 6, 200, 0, True),        # weight ties: the threshold bin is one value
    (3000, 64, 6, 200, 2, False),       # arrival order (radix path)
    (5000, 16, 1, 400, 0, False),
    (2000, 128, 8, 10000, 0, False),    # nothing dropped
    (1100, 5, 3, 0, 0, False),          # K = 0: everything dropped
    (20000, 32, 1, 700, 0, True)])
def test_capacity_dispatch_matches_oracle(T, E, k, K, flags, ties):
    moe = _moe()
    ids, w = _given_routing(T, E, k, T + E, ties)
    layer = moe.MoELayer(T, 64, 64, E, k, 1.0, "bf16", flags=flags)
    r = layer.capacity_dispatch(to_dev(ids), to_dev(w), K)
    torch.cuda.synchronize()
    assert moe.moe_get_device_status(layer.ws) == 0
    ro = oracle.select(ids, w, E, K, flags)
    assert np.array_equal(to_host(r["slot"]), ro["slot"])
    assert np.array_equal(to_host(r["drop"]), ro["drop"])
    counts = to_host(r["counts"])
    assert np.array_equal(counts[:E], ro["received"]) and np.array_equal(counts[E:], ro["kept"])
    off_ref, rowtok_ref = oracle.dispatch(ids, ro["slot"], E)
    assert np.array_equal(to_host(r["offsets"]), off_ref)
    n = int(off_ref[-1])
    assert np.array_equal(to_host(r["rowtok"])[:n], rowtok_ref)


def test_capacity_dispatch_reports_bad_ids():
    moe = _moe()
    T, E, k = 2000, 8, 2
    ids, w = _given_routing(T, E, k, 5, False)
    ids[17, 1] = E                      # outside [0, E): left out and reported
    layer = moe.MoELayer(T, 64, 64, E, k, 1.0, "bf16")
    layer.capacity_dispatch(to_dev(ids), to_dev(w), 300)
    torch.cuda.synchronize()
    assert moe.moe_get_device_status(layer.ws) == moe.DEV_BAD_INDEX


@pytest.mark.parametrize("T,d,E,dtype", [(64, 2048, 64, "bf16"), (3000, 256, 64, "bf16"),
                                         (2000, 512, 128, "bf16"), (500, 48, 7, "f32")])
def test_router_logits_equal_the_forward_logits(T, d, E, dtype):
    moe = _moe()
    k = min(4, E)
    spec = inputs.LayerSpec("rl", T, d, 64, E, k, 1.0, dtype, router="normal", router_bias=0.5)
    L = inputs.make_layer(spec, seed=T + d)
    layer = moe.MoELayer(T, d, 64, E, k, 1.0, dtype)
    args = [to_dev(L[n]) for n in ("x", "Wr", "br", "W1", "b1", "W2", "b2")]
    _, rt = layer.forward(*args, want_routing=True)
    lg = layer.router_logits(args[0], args[1], args[2])
    torch.cuda.synchronize()
    assert torch.equal(lg, rt["logits_out"])
    ref = oracle.logits(L["x"], L["Wr"], L["br"])
    assert np.abs(to_host(lg) - ref).max() <= 1e-4 * max(1.0, np.abs(ref).max())


@pytest.mark.parametrize("T,d,E,k,C", [(3000, 256, 64, 6, 1.0), (2048, 512, 128, 8, 1.5),
                                       (1500, 128, 16, 2, 1.25), (500, 128, 16, 2, 1.25)])
def test_prepared_router_forward_equals_unprepared(T, d, E, k, C):
    """moe_prepare_router once, then forwards with MOE_FLAG_ROUTER_PREPARED: the same logits,
    routing and outputs, call after call, and again after the router weights change."""
    moe = _moe()
    spec = inputs.LayerSpec("prep", T, d, 128, E, k, C, "bf16", router="normal",
                            router_bias=0.5, bias_std=0.05)
    L = inputs.make_layer(spec, seed=T + E)
    args = [to_dev(L[n]) for n in ("x", "Wr", "br", "W1", "b1", "W2", "b2")]

    def same(a, b):
        (oa, ra), (ob, rb) = a, b
        assert torch.equal(oa.view(torch.int16), ob.view(torch.int16))
        for key in ra:
            assert torch.equal(ra[key], rb[key]), key

    ref = moe.MoELayer(T, d, 128, E, k, C, "bf16")
    layer = moe.MoELayer(T, d, 128, E, k, C, "bf16")
    layer.prepare_router(args[1])
    want = ref.forward(*args, want_routing=True)
    same(layer.forward(*args, want_routing=True), want)
    same(layer.forward(*args, want_routing=True), want)      # counters cleared every call
    args2 = list(args)
    args2[1] = args[1] * 1.5
    layer.prepare_router(args2[1])
    same(layer.forward(*args2, want_routing=True), ref.forward(*args2, want_routing=True))
    torch.cuda.synchronize()
    assert moe.moe_get_device_status(layer.ws) == 0


# ------------------------------------------------------------------------------------------
# Routing-policy flags (renormalised weights, arrival-order capacity), bit for bit.
# ------------------------------------------------------------------------------------------
@pytest.mark.parametrize("flags", [1, 2, 3])
@pytest.mark.parametrize("T,E,k,C,seed", [(3000, 64, 6, 1.0, 1), (1000, 8, 2, 0.5, 2),
                                          (777, 100, 8, 0.75, 3), (513, 32, 32, 1.0, 4),
                                          (2048, 16, 1, 0.25, 5)])
def test_route_flags_bit_exact(flags, T, E, k, C, seed):
    L = inputs.random_logits(T, E, seed, 2.0)
    _, g, ro = _route_both(L, T, E, k, C, flags=flags)
    _assert_route_equal(g, ro, E)


@pytest.mark.parametrize("flags", [1, 2, 3])
def test_forward_with_flags(flags):
    spec = inputs.LayerSpec("flags", 600, 128, 192, 8, 2, 0.75, "bf16", router="normal",
                            router_bias=0.5, bias_std=0.05)
    _forward_check(spec, seed=3, flags=flags)


# ------------------------------------------------------------------------------------------
# Small batches (T*k <= 1024) take the single-launch dispatch; same results, bit for bit.
# ------------------------------------------------------------------------------------------
@pytest.mark.parametrize("flags", [0, 2, 3])
@pytest.mark.parametrize("T,E,k,C,seed", [(128, 8, 8, 0.5, 1), (1024, 64, 1, 0.3, 2),
                                          (100, 1024, 8, 1.0, 3), (64, 64, 8, math.inf, 4),
                                          (512, 16, 2, 0.0, 5), (33, 3, 3, 0.4, 6)])
def test_route_small_batches_bit_exact(flags, T, E, k, C, seed):
    L = inputs.random_logits(T, E, seed, 1.5)
    _, g, ro = _route_both(L, T, E, k, C, flags=flags)
    _assert_route_equal(g, ro, E)


def test_route_small_batch_weight_ties():
    rng = np.random.default_rng(8)
    proto = rng.standard_normal((3, 10)).astype(np.float32)
    L = proto[rng.integers(0, 3, size=200)]
    _, g, ro = _route_both(L, 200, 10, 2, 0.6)
    _assert_route_equal(g, ro, 10)


# ------------------------------------------------------------------------------------------
# The whole forward replayed from a CUDA graph (no host sync or allocation inside the call).
# ------------------------------------------------------------------------------------------
@pytest.mark.parametrize("spec", [inputs.LayerSpec("g1", 64, 256, 128, 16, 4, math.inf, "bf16"),
                                  inputs.LayerSpec("g2", 2000, 128, 192, 8, 2, 1.0, "bf16",
                                                   router="zipf", router_bias=1.1)])
def test_forward_cuda_graph_replay(spec):
    moe = _moe()
    L = inputs.make_layer(spec, seed=2)
    layer = moe.MoELayer(spec.T, spec.d_model, spec.d_ff, spec.E, spec.k, spec.C, spec.dtype)
    args = [to_dev(L[n]) for n in ("x", "Wr", "br", "W1", "b1", "W2", "b2")]
    eager = layer.forward(*args)
    out = torch.empty_like(eager)
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        layer.forward(*args, out=out)                 # warm-up on the capture stream type
    torch.cuda.current_stream().wait_stream(side)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        layer.forward(*args, out=out)
    out.zero_()
    for _ in range(3):
        graph.replay()
    torch.cuda.synchronize()
    assert moe.moe_get_device_status(layer.ws) == 0
    assert torch.equal(out.view(torch.int16), eager.view(torch.int16))


# ------------------------------------------------------------------------------------------
# Stream order with programmatic dependent launch: the first kernel of a call may be scheduled
# while the caller's preceding work drains, but must not read x before that work has written
# it.  x is produced on the same stream right before the call (a copy from pinned host memory,
# then an in-place update by a torch kernel), in a loop, and every output must match.
# ------------------------------------------------------------------------------------------
def test_forward_reads_inputs_written_just_before_on_the_stream():
    moe = _moe()
    spec = inputs.LayerSpec("s1", 3000, 256, 128, 8, 2, 1.0, "bf16")
    L = inputs.make_layer(spec, seed=5)
    layer = moe.MoELayer(spec.T, spec.d_model, spec.d_ff, spec.E, spec.k, spec.C, spec.dtype)
    args = [to_dev(L[n]) for n in ("x", "Wr", "br", "W1", "b1", "W2", "b2")]
    x_host = args[0].cpu().pin_memory()
    refs = []
    for scale in (1.0, -1.0, 0.5):
        xs = (args[0].float() * scale).to(torch.bfloat16)
        refs.append(layer.forward(xs, *args[1:]).clone())
    torch.cuda.synchronize()
    xd = torch.empty_like(args[0])
    out = torch.empty_like(refs[0])
    for rep in range(3):
        for scale, ref in zip((1.0, -1.0, 0.5), refs):
            xd.copy_(x_host, non_blocking=True)       # same stream, no host sync in between
            xd.mul_(scale)                           # exact in bf16 for these scales
            layer.forward(xd, *args[1:], out=out)
            torch.cuda.synchronize()
            assert torch.equal(out.view(torch.int16), ref.view(torch.int16)), (rep, scale)


# ------------------------------------------------------------------------------------------
# Canaries: every byte the forward writes lies inside its outputs and its workspace.  Each
# buffer sits between 4 KB guard regions filled with a pattern, which must survive the call.
# ------------------------------------------------------------------------------------------
def _guarded(n_elems, dtype, fill_byte=0x5A, guard_bytes=4096):
    esz = torch.empty((), dtype=dtype).element_size()
    g = guard_bytes // esz
    raw = torch.full(((2 * guard_bytes + n_elems * esz),), fill_byte, dtype=torch.uint8,
                     device="cuda")
    view = raw[guard_bytes:guard_bytes + n_elems * esz].view(dtype)
    return raw, view, g * esz


def _guards_intact(raw, guard_bytes, fill_byte=0x5A):
    head = raw[:guard_bytes]
    tail = raw[raw.numel() - guard_bytes:]
    return bool((head == fill_byte).all().item()) and bool((tail == fill_byte).all().item())


@pytest.mark.parametrize("spec", [
    inputs.LayerSpec("c1", 64, 256, 128, 16, 8, math.inf, "bf16"),
    inputs.LayerSpec("c2", 3000, 128, 192, 8, 2, 1.0, "bf16", router="zipf", router_bias=1.1),
    inputs.LayerSpec("c3", 1500, 128, 256, 8, 2, 0.7, "bf16", gated=True),
    inputs.LayerSpec("c4", 300, 16, 24, 6, 2, 1.0, "f32"),
])
def test_forward_writes_stay_inside_outputs_and_workspace(spec):
    moe = _moe()
    L = inputs.make_layer(spec, seed=9)
    flags = moe.FLAG_GATED if spec.gated else 0
    p = moe.problem(spec.T, spec.d_model, spec.d_ff, spec.E, spec.k, spec.C, spec.dtype,
                    flags=flags)
    args = [to_dev(L[n]) for n in ("x", "Wr", "br", "W1", "b1", "W2", "b2")]
    x = args[0]
    T, E, k = spec.T, spec.E, spec.k
    bufs = {}
    bufs["ws"] = _guarded(moe.moe_workspace_size(p), torch.uint8)
    bufs["out"] = _guarded(x.numel(), x.dtype)
    bufs["logits"] = _guarded(T * E, torch.float32)
    bufs["ids"] = _guarded(T * k, torch.int32)
    bufs["w"] = _guarded(T * k, torch.float32)
    bufs["slot"] = _guarded(T * k, torch.int32)
    bufs["drop"] = _guarded(T * k, torch.uint8)
    bufs["counts"] = _guarded(2 * E, torch.int32)
    out = bufs["out"][1].view(x.shape)
    moe.moe_reset_device_status(bufs["ws"][1])       # the status word is the caller's to clear
    moe.moe_forward(p, *args, out, bufs["ws"][1], logits_out=bufs["logits"][1],
                    ids_out=bufs["ids"][1], w_out=bufs["w"][1], slot_out=bufs["slot"][1],
                    drop_out=bufs["drop"][1], counts_out=bufs["counts"][1])
    torch.cuda.synchronize()
    assert moe.moe_get_device_status(bufs["ws"][1]) == 0
    for name, (raw, _, gb) in bufs.items():
        assert _guards_intact(raw, gb), name
    layer = moe.MoELayer(spec.T, spec.d_model, spec.d_ff, spec.E, spec.k, spec.C, spec.dtype,
                         flags=flags)
    ref = layer.forward(*args)
    torch.cuda.synchronize()
    if x.dtype == torch.bfloat16:
        assert torch.equal(out.view(torch.int16), ref.view(torch.int16))
    else:
        assert torch.equal(out, ref)


# ------------------------------------------------------------------------------------------
# Caller-supplied dispatch data is checked on the device.  moe_expert_ffn with offsets whose
# total exceeds the row count by one row, or that decrease, stores nothing: the guard regions
# around Y and the workspace (each larger than one 128-row output tile) survive, Y keeps its
# fill pattern, and the status word says MOE_DEV_BAD_INDEX.  Good offsets then run normally.
# ------------------------------------------------------------------------------------------
@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("defect", ["one_row_too_many", "decreasing", "nonzero_start"])
def test_expert_ffn_rejects_bad_offsets(dtype, defect):
    moe = _moe()
    T, d, F, E, k = 300, 128, 192, 5, 2
    spec = inputs.LayerSpec("bad", T, d, F, E, k, math.inf, dtype, router="normal",
                            router_bias=0.5, bias_std=0.05)
    L = inputs.make_layer(spec, seed=1)
    ro = oracle.route(oracle.logits(L["x"], L["Wr"], L["br"]), k, T)
    off, rowtok = oracle.dispatch(ro["ids"], ro["slot"], E)
    R = T * k
    assert int(off[-1]) == R                          # dropless: every row of Y is used
    bad = off.copy()
    if defect == "one_row_too_many":
        bad[-1] = R + 1
    elif defect == "decreasing":
        bad[2], bad[3] = bad[3], bad[2]
    else:
        bad[0] = 1
    p = moe.problem(T, d, F, E, k, math.inf, dtype)
    tdt = torch.bfloat16 if dtype == "bf16" else torch.float32
    guard = 128 * d * 4 * 2                           # bytes: more than one output tile
    ws_raw, ws, gb = _guarded(moe.moe_workspace_size(p), torch.uint8, guard_bytes=guard)
    y_raw, Y, gy = _guarded(R * d, tdt, guard_bytes=guard)
    y_before = y_raw.clone()
    args = [to_dev(L[n]) for n in ("x", "W1", "b1", "W2", "b2")]
    moe.moe_reset_device_status(ws)
    moe.moe_expert_ffn(p, args[0], to_dev(bad), to_dev(rowtok), args[1], args[2], args[3],
                       args[4], Y, ws)
    torch.cuda.synchronize()
    assert moe.moe_get_device_status(ws) == moe.DEV_BAD_INDEX
    assert _guards_intact(ws_raw, gb) and _guards_intact(y_raw, gy)
    assert torch.equal(y_raw, y_before), "nothing may be stored with bad offsets"
    moe.moe_reset_device_status(ws)
    moe.moe_expert_ffn(p, args[0], to_dev(off), to_dev(rowtok), args[1], args[2], args[3],
                       args[4], Y, ws)
    torch.cuda.synchronize()
    assert moe.moe_get_device_status(ws) == 0
    row_exp = np.repeat(np.arange(E, dtype=np.int32), np.diff(off))
    Yref = oracle.expert_rows(L["x"], L["W1"], L["b1"], L["W2"], L["b2"], rowtok, row_exp)
    assert_close(to_host(Y.view(R, d)), Yref, dtype, "expert outputs after bad offsets")


def test_combine_reports_rows_outside_y():
    # The last expert's range is moved so that some of its rows fall past the end of Y: those
    # terms are skipped and reported in the workspace's status word; tokens routed elsewhere
    # are unaffected.
    moe = _moe()
    T, d, E, k, C = 400, 64, 6, 2, 0.8
    L = inputs.random_logits(T, E, 21)
    K = oracle.capacity(T, E, k, C)
    ro = oracle.route(L, k, K)
    off, _ = oracle.dispatch(ro["ids"], ro["slot"], E)
    R = min(T * k, E * K)
    rng = np.random.default_rng(4)
    x = inputs.f32_to_bf16_bits(rng.standard_normal((T, d)).astype(np.float32))
    Y = inputs.f32_to_bf16_bits(rng.standard_normal((R, d)).astype(np.float32))
    layer = moe.MoELayer(T, d, 64, E, k, C, "bf16")
    args = [to_dev(a) for a in (x, Y, ro["w"], ro["ids"], ro["slot"])]
    good = layer.combine(*args, to_dev(off))
    bad = off.copy()
    last_kept = int(off[E] - off[E - 1])
    assert last_kept >= 2
    bad[E - 1] = R - 1                                 # slot s of expert E-1 -> row R - 1 + s
    bad[E] = R + 1000
    moe.moe_reset_device_status(layer.ws)
    out = layer.combine(*args, to_dev(bad))
    torch.cuda.synchronize()
    assert moe.moe_get_device_status(layer.ws) == moe.DEV_BAD_INDEX
    elsewhere = ~((ro["ids"] == E - 1) & (ro["slot"] >= 0)).any(axis=1)
    assert torch.equal(out[torch.from_numpy(elsewhere).cuda()].view(torch.int16),
                       good[torch.from_numpy(elsewhere).cuda()].view(torch.int16))


# ------------------------------------------------------------------------------------------
# Failure detection: a pipeline wait that can never complete gives up, reports a timeout in the
# status word, and leaves the GPU usable (no trap, no fault, no hang).
# ------------------------------------------------------------------------------------------
def test_bounded_wait_reports_timeout_and_gpu_stays_usable():
    moe = _moe()
    layer = moe.MoELayer(256, 64, 64, 8, 2, 1.0, "bf16")
    moe.moe_reset_device_status(layer.ws)
    moe.moe_selftest_wait_timeout(layer.ws, 50000)       # 50 ms
    assert moe.moe_get_device_status(layer.ws) == moe.DEV_TIMEOUT
    moe.moe_reset_device_status(layer.ws)
    L = inputs.random_logits(256, 8, 1)
    r = layer.route(to_dev(L))
    torch.cuda.synchronize()
    assert moe.moe_get_device_status(layer.ws) == 0
    ro = oracle.route(L, 2, layer.K)
    assert np.array_equal(to_host(r["slot"]), ro["slot"])


# ------------------------------------------------------------------------------------------
# Gated experts (MOE_FLAG_GATED): H = SiLU(x W_gate^T + b_gate) * (x W_up^T + b_up).
# ------------------------------------------------------------------------------------------
@pytest.mark.parametrize("T,d,F,E,k,C,dtype", [(300, 128, 256, 5, 2, 1.0, "bf16"),
                                               (700, 256, 384, 3, 3, 0.9, "bf16"),
                                               (40, 16, 24, 4, 2, 1.0, "f32")])
def test_gated_expert_ffn_parity(T, d, F, E, k, C, dtype):
    moe = _moe()
    spec = inputs.LayerSpec("gffn", T, d, F, E, k, C, dtype, router="normal", router_bias=0.5,
                            bias_std=0.05, gated=True)
    L = inputs.make_layer(spec, seed=T + 1)
    logits = oracle.logits(L["x"], L["Wr"], L["br"])
    K = oracle.capacity(T, E, k, C)
    ro = oracle.route(logits, k, K)
    off_ref, rowtok_ref = oracle.dispatch(ro["ids"], ro["slot"], E)
    n = int(off_ref[-1])
    row_exp = np.repeat(np.arange(E, dtype=np.int32), np.diff(off_ref))
    Yref = oracle.expert_rows(L["x"], L["W1"], L["b1"], L["W2"], L["b2"], rowtok_ref, row_exp,
                              flags=oracle.GATED)
    layer = moe.MoELayer(T, d, F, E, k, C, dtype, flags=moe.FLAG_GATED)
    Y = layer.expert_ffn(to_dev(L["x"]), to_dev(off_ref), to_dev(rowtok_ref), to_dev(L["W1"]),
                         to_dev(L["b1"]), to_dev(L["W2"]), to_dev(L["b2"]))
    torch.cuda.synchronize()
    assert moe.moe_get_device_status(layer.ws) == 0
    assert_close(to_host(Y)[:n], Yref, dtype, "gated expert outputs")


@pytest.mark.parametrize("spec", [
    inputs.LayerSpec("gf1", 1000, 256, 384, 8, 2, 1.0, "bf16", router="zipf", router_bias=1.1,
                     bias_std=0.02, gated=True),
    inputs.LayerSpec("gf2", 2500, 128, 128, 16, 4, 0.8, "bf16", router="normal",
                     router_bias=0.5, gated=True)])
def test_forward_gated(spec):
    _forward_check(spec, seed=4, flags=4)


def test_gated_needs_d_ff_multiple_of_128():
    moe = _moe()
    with pytest.raises(moe.MoeError) as ei:
        moe.MoELayer(16, 64, 192, 4, 2, 1.0, "bf16", flags=moe.FLAG_GATED).forward(
            *[torch.zeros(8, device="cuda")] * 7)
    assert ei.value.status == 2
