"""Pins for the CPU oracle: the worked example, brute force, closed forms and invariants.

Each test checks the oracle against something other than itself: values printed on the pages
(``golden/worked_example.json``), torch/numpy library routines in float64, exhaustive search
on tiny inputs, or properties that must hold whatever the inputs.
"""
import json
import math
import os

import numpy as np
import pytest
import torch
import torch.nn.functional as Fnn

import oracle
from expert_ffn_layer_router_b200 import inputs

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _worked():
    with open(os.path.join(GOLDEN, "worked_example.json")) as f:
        return json.load(f)


def _f64(a):
    return inputs.bf16_bits_to_f32(a).astype(np.float64) if a.dtype == np.uint16 else \
        a.astype(np.float64)


def dense_reference(layer, route):
    """Every expert on every token (torch float64 Linear/SiLU), then masked by the routing."""
    x = torch.from_numpy(_f64(layer["x"]))
    W1 = torch.from_numpy(_f64(layer["W1"]))
    W2 = torch.from_numpy(_f64(layer["W2"]))
    b1 = torch.from_numpy(layer["b1"].astype(np.float64))
    b2 = torch.from_numpy(layer["b2"].astype(np.float64))
    E = W1.shape[0]
    Y = torch.stack([Fnn.linear(Fnn.silu(Fnn.linear(x, W1[e], b1[e])), W2[e], b2[e])
                     for e in range(E)])                          # [E, T, d]
    T, k = route["ids"].shape
    out = x.clone()
    contrib = torch.zeros_like(x)
    for t in range(T):
        for j in range(k):
            if route["slot"][t, j] >= 0:
                contrib[t] += float(route["w"][t, j]) * Y[route["ids"][t, j], t]
    return (out + contrib).numpy(), Y.numpy()


# ------------------------------------------------------------------------------------------
# The worked example (T=8, E=4, top-1, C=1.25).
# ------------------------------------------------------------------------------------------

def test_worked_example_capacity_and_drop():
    g = _worked()
    K = oracle.capacity(g["T"], g["E"], g["top_k"], g["capacity_factor"])
    assert K == g["K"]
    assert math.floor(g["K_unrounded"]) == K
    layer = inputs.make_layer(inputs.CONFIGS["tiny_f32"], seed=0)
    r = oracle.route(layer["logits"], g["top_k"], K)
    for e, toks in g["assignment"].items():
        assert sorted(np.nonzero(r["ids"][:, 0] == int(e))[0].tolist()) == toks
    assert r["received"].tolist() == g["loads"]
    dropped = np.nonzero(r["drop"][:, 0])[0].tolist()
    assert dropped == g["dropped_tokens"]
    offsets, rowtok = oracle.dispatch(r["ids"], r["slot"], g["E"])
    for e, toks in g["expert_batches"].items():
        e = int(e)
        assert rowtok[offsets[e]:offsets[e + 1]].tolist() == toks
    # The slowest expert is the one with the most kept tokens.
    assert int(np.argmax(r["kept"])) == g["slowest_expert"]
    # Token 0's weight is the illustrative 0.87.
    assert abs(float(r["w"][0, 0]) - g["w0_illustrative"]) < 5e-3


def test_worked_example_outputs():
    g = _worked()
    layer = inputs.make_layer(inputs.CONFIGS["tiny_f32"], seed=0)
    assert layer["x"][0].tolist() == pytest.approx(g["x0"])
    K = oracle.capacity(8, 4, 1, 1.25)
    r = oracle.route(layer["logits"], 1, K)
    out64, out = oracle.combine_tokens(layer["x"], layer["W1"], layer["b1"], layer["W2"],
                                       layer["b2"], r)
    # Dropped token 4 leaves the layer bit for bit.
    assert out[4].view(np.uint32).tolist() == layer["x"][4].view(np.uint32).tolist()
    # Token 0: x0 + w0 * y0 with y0 = W2 SiLU(W1 x0 + b1) + b2 of expert 0, built from torch.
    x0 = torch.tensor(layer["x"][0], dtype=torch.float64)
    mlp = torch.nn.Sequential(torch.nn.Linear(4, 8), torch.nn.SiLU(), torch.nn.Linear(8, 4)).double()
    with torch.no_grad():
        mlp[0].weight.copy_(torch.from_numpy(layer["W1"][0].astype(np.float64)))
        mlp[0].bias.copy_(torch.from_numpy(layer["b1"][0].astype(np.float64)))
        mlp[2].weight.copy_(torch.from_numpy(layer["W2"][0].astype(np.float64)))
        mlp[2].bias.copy_(torch.from_numpy(layer["b2"][0].astype(np.float64)))
        y0 = mlp(x0).numpy()
    expect = layer["x"][0].astype(np.float64) + float(r["w"][0, 0]) * y0
    np.testing.assert_allclose(out64[0], expect, rtol=0, atol=1e-12)
    ref, _ = dense_reference(layer, r)
    np.testing.assert_allclose(out64, ref, rtol=0, atol=1e-12)


# ------------------------------------------------------------------------------------------
# Capacity
# ------------------------------------------------------------------------------------------

@pytest.mark.parametrize("name,K", [("tiny_f32", 2), ("bf16_e8_top2", 1280),
                                    ("skewed_e64_top6", 1536), ("decode_e64_top8", 64),
                                    ("prefill_e128_top8", 6144)])
def test_capacity_of_configs(name, K):
    s = inputs.CONFIGS[name]
    assert oracle.capacity(s.T, s.E, s.k, s.C) == K


def test_capacity_edges():
    assert oracle.capacity(100, 4, 1, 0.0) == 0
    assert oracle.capacity(100, 4, 2, 100.0) == 100          # clamped to T
    assert oracle.capacity(100, 4, 2, math.inf) == 100       # dropless
    assert oracle.capacity(10, 3, 1, 1.0) == 3               # floor(10/3)
    assert oracle.capacity(10, 4, 1, -1.0) == -1
    assert oracle.capacity(10, 4, 1, float("nan")) == -1


# ------------------------------------------------------------------------------------------
# Own exp and softmax
# ------------------------------------------------------------------------------------------

def _ulp_f32(v64):
    v = np.abs(v64).astype(np.float32)
    return np.spacing(v).astype(np.float64)


def test_own_exp_within_two_ulp():
    rng = np.random.default_rng(5)
    x = np.concatenate([np.linspace(-86.9, 88.7, 400001, dtype=np.float32),
                        rng.uniform(-30, 0, 200000).astype(np.float32),
                        np.array([0.0, -0.0, 1e-30, -1e-30, 0.5, -0.5, 1.0, -1.0], np.float32)])
    y = oracle.own_exp(x).astype(np.float64)
    ref = np.exp(x.astype(np.float64))
    err = np.abs(y - ref) / _ulp_f32(ref)
    assert err.max() <= 2.0, err.max()
    assert oracle.own_exp(np.float32(0.0))[0] == 1.0


def test_own_exp_range_edges():
    y = oracle.own_exp(np.array([-87.5, -100.0, -1e30, 89.0, 1e30, np.nan], np.float32))
    assert y[0] == 0.0 and y[1] == 0.0 and y[2] == 0.0
    assert np.isinf(y[3]) and np.isinf(y[4]) and np.isnan(y[5])


@pytest.mark.parametrize("E", [1, 2, 4, 8, 33, 64, 128, 257, 1024])
def test_softmax_matches_torch_float64(E):
    L = inputs.random_logits(64, E, seed=E, scale=3.0)
    p = oracle.softmax(L).astype(np.float64)
    ref = torch.softmax(torch.from_numpy(L.astype(np.float64)), dim=1).numpy()
    # Relative error budget in units of 2^-24: rounding of L - m (|L - m| each for u_e and, at
    # worst, for the terms of S), own exp (4), the sum S (ceil(E/32) + 5 additions), the divide.
    span = (L.max(axis=1, keepdims=True) - L).astype(np.float64)
    bound = 2.0 ** -24 * (span + span.max(axis=1, keepdims=True) + 4 + math.ceil(E / 32) + 5 + 1)
    assert (np.abs(p - ref) <= bound * ref + 1e-37).all()
    np.testing.assert_allclose(p.sum(axis=1), 1.0, rtol=0, atol=2e-6)


# ------------------------------------------------------------------------------------------
# Top-k, capacity selection and slots against brute force
# ------------------------------------------------------------------------------------------

def brute_route(L, k, K):
    """Exhaustive reference: sort experts per token, sort candidates per expert."""
    T, E = L.shape
    p = torch.softmax(torch.from_numpy(L.astype(np.float64)), dim=1).numpy()
    ids = np.zeros((T, k), np.int64)
    for t in range(T):
        order = sorted(range(E), key=lambda e: (-float(L[t, e]), e))
        ids[t] = order[:k]
    return ids, p


def _tie_logits(T, E, seed):
    # Few distinct values so ties in logits (across experts) and in weights (across tokens) occur.
    rng = np.random.default_rng(seed)
    base = rng.integers(0, 4, size=(T, E)).astype(np.float32) * np.float32(0.5)
    rows = rng.integers(0, 3, size=T)            # tokens share one of 3 rows -> equal weights
    proto = rng.integers(0, 4, size=(3, E)).astype(np.float32) * np.float32(0.5)
    mix = rng.random(T) < 0.6
    base[mix] = proto[rows[mix]]
    return base


@pytest.mark.parametrize("seed", range(6))
@pytest.mark.parametrize("T,E,k,C", [(16, 4, 1, 1.0), (40, 6, 2, 0.75), (64, 8, 3, 1.25),
                                     (33, 5, 5, 0.5), (20, 4, 2, 0.0), (50, 7, 3, math.inf)])
def test_route_matches_brute_force(seed, T, E, k, C):
    L = _tie_logits(T, E, seed) if seed % 2 else inputs.random_logits(T, E, seed)
    K = oracle.capacity(T, E, k, C)
    r = oracle.route(L, k, K)
    ids_ref, p_ref = brute_route(L, k, K)
    assert np.array_equal(r["ids"], ids_ref)
    np.testing.assert_allclose(r["w"], np.take_along_axis(p_ref, ids_ref, 1), rtol=4e-7)
    # Capacity selection by exhaustive sort of each expert's candidates using the oracle's own
    # fp32 weights (the priority is defined on those values).
    w = r["w"]
    for e in range(E):
        cand = [(t, j) for t in range(T) for j in range(k) if r["ids"][t, j] == e]
        ranked = sorted(cand, key=lambda tj: (-float(w[tj]), tj[0]))
        keep = set(ranked[:K])
        kept_sorted = sorted(keep)
        assert r["received"][e] == len(cand)
        assert r["kept"][e] == min(len(cand), K)
        for (t, j) in cand:
            if (t, j) in keep:
                assert r["drop"][t, j] == 0
                assert r["slot"][t, j] == kept_sorted.index((t, j))
            else:
                assert r["drop"][t, j] == 1 and r["slot"][t, j] == -1


def _given_routing(T, E, k, seed, ties):
    """A routing that no router produced: each token's k distinct experts drawn at random, weights
    from a few values (ties across tokens) or continuous."""
    rng = np.random.default_rng(seed)
    ids = np.stack([rng.permutation(E)[:k] for _ in range(T)]).astype(np.int32)
    if ties:
        w = (rng.integers(1, 5, size=(T, k)) * 0.125).astype(np.float32)
    else:
        w = rng.random((T, k)).astype(np.float32)
    return ids, w


@pytest.mark.parametrize("seed", range(4))
@pytest.mark.parametrize("T,E,k,K", [(30, 4, 1, 5), (40, 6, 2, 9), (25, 5, 3, 0), (50, 8, 4, 100),
                                     (64, 3, 2, 17)])
@pytest.mark.parametrize("flags", [0, 2])
def test_select_matches_brute_force(seed, T, E, k, K, flags):
    # Capacity selection of a given routing ("Expert Networks > Worked Example", capacity
    # paragraph: the lowest-confidence tokens drop; "Some Tokens Do Not Get In", "Past the edge":
    # in arrival order) against an exhaustive sort of each expert's candidates.
    ids, w = _given_routing(T, E, k, seed, ties=seed % 2 == 0)
    r = oracle.select(ids, w, E, K, flags)
    for e in range(E):
        cand = [(t, j) for t in range(T) for j in range(k) if ids[t, j] == e]
        if flags & oracle.ARRIVAL_ORDER:
            ranked = sorted(cand)
        else:
            ranked = sorted(cand, key=lambda tj: (-float(w[tj]), tj[0]))
        keep = set(ranked[:K])
        kept_sorted = sorted(keep)
        assert r["received"][e] == len(cand)
        assert r["kept"][e] == min(len(cand), K)
        for tj in cand:
            if tj in keep:
                assert r["drop"][tj] == 0 and r["slot"][tj] == kept_sorted.index(tj)
            else:
                assert r["drop"][tj] == 1 and r["slot"][tj] == -1


def test_select_rejects_ids_outside_the_experts():
    ids = np.array([[0], [4]], np.int32)
    with pytest.raises(ValueError):
        oracle.select(ids, np.ones((2, 1), np.float32), 4, 1)
    with pytest.raises(ValueError):
        oracle.select(-ids, np.ones((2, 1), np.float32), 4, 1)


def test_drop_is_by_confidence_not_arrival():
    # Expert 0 receives tokens 0, 1, 2; token 0 (first to arrive) has the lowest confidence and
    # must be the one dropped; an arrival-order buffer would drop token 2 instead.
    L = np.array([[0.5, 0, 0], [3.0, 0, 0], [2.0, 0, 0], [0, 1.0, 0]], np.float32)
    r = oracle.route(L, 1, 2)
    assert r["drop"][:, 0].tolist() == [1, 0, 0, 0]
    assert r["slot"][:, 0].tolist() == [-1, 0, 1, 0]


def test_weight_tie_keeps_lower_token():
    L = np.array([[1.0, 0.0]] * 5, np.float32)            # five identical tokens, K = 3
    r = oracle.route(L, 1, 3)
    assert r["drop"][:, 0].tolist() == [0, 0, 0, 1, 1]
    assert r["slot"][:, 0].tolist() == [0, 1, 2, -1, -1]


def test_logit_tie_picks_lower_expert():
    L = np.array([[1.0, 2.0, 2.0, 2.0, 0.0]], np.float32)
    r = oracle.route(L, 2, 1)
    assert r["ids"].tolist() == [[1, 2]]


@pytest.mark.parametrize("seed", range(4))
def test_route_invariants(seed):
    T, E, k = 500, 16, 4
    L = inputs.random_logits(T, E, seed, scale=2.0)
    L[:, 3] += 2.0                                         # one hot expert that overflows
    K = oracle.capacity(T, E, k, 1.0)
    r = oracle.route(L, k, K)
    assert (r["kept"] <= K).all()
    assert np.array_equal(r["kept"], np.minimum(r["received"], K))
    assert r["kept"].sum() + r["drop"].sum() == T * k
    assert r["received"].sum() == T * k
    assert r["received"][3] > K                            # the overflow really happened
    for e in range(E):
        m = r["ids"] == e
        kept = m & (r["slot"] >= 0)
        dropped = m & (r["slot"] < 0)
        if dropped.any():
            assert r["w"][kept].min() >= r["w"][dropped].max()
        toks = np.nonzero(kept)[0]
        slots = r["slot"][kept]
        assert sorted(slots.tolist()) == list(range(kept.sum()))
        assert np.array_equal(slots, np.argsort(np.argsort(toks, kind="stable"), kind="stable"))
    # Each token's experts are distinct and ordered by descending logit.
    for t in range(T):
        assert len(set(r["ids"][t].tolist())) == k
        lv = L[t, r["ids"][t]]
        assert (np.diff(lv) <= 0).all()


def test_dispatch_layout():
    T, E, k = 200, 8, 2
    L = inputs.random_logits(T, E, 3)
    K = oracle.capacity(T, E, k, 0.8)
    r = oracle.route(L, k, K)
    offsets, rowtok = oracle.dispatch(r["ids"], r["slot"], E)
    assert offsets[0] == 0 and offsets[-1] == r["kept"].sum()
    assert np.array_equal(np.diff(offsets), r["kept"])
    for e in range(E):
        toks = rowtok[offsets[e]:offsets[e + 1]]
        assert (np.diff(toks) > 0).all()                   # ascending token order
        expect = sorted(t for t in range(T) for j in range(k)
                        if r["ids"][t, j] == e and r["slot"][t, j] >= 0)
        assert toks.tolist() == expect


# ------------------------------------------------------------------------------------------
# FFN and combine against torch float64 (dense all-experts-on-all-tokens, then masked)
# ------------------------------------------------------------------------------------------

@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("T,d,F,E,k,C", [(24, 8, 16, 4, 1, 0.75), (40, 16, 24, 6, 2, 1.0),
                                         (32, 8, 8, 5, 3, 0.5), (16, 4, 12, 3, 3, math.inf)])
def test_forward_matches_dense_reference(dtype, T, d, F, E, k, C):
    spec = inputs.LayerSpec("t", T, d, F, E, k, C, dtype, router="normal", router_bias=0.3,
                            bias_std=0.1)
    layer = inputs.make_layer(spec, seed=T + d)
    res = oracle.forward(layer["x"], layer["Wr"], layer["br"], layer["W1"], layer["b1"],
                         layer["W2"], layer["b2"], k, C)
    ref, Y = dense_reference(layer, res["route"])
    np.testing.assert_allclose(res["out_f64"], ref, rtol=0, atol=1e-12)
    # Per-row expert outputs.
    offsets, rowtok = oracle.dispatch(res["route"]["ids"], res["route"]["slot"], E)
    row_exp = np.repeat(np.arange(E, dtype=np.int32), np.diff(offsets))
    Yo = oracle.expert_rows(layer["x"], layer["W1"], layer["b1"], layer["W2"], layer["b2"],
                            rowtok, row_exp)
    np.testing.assert_allclose(Yo, Y[row_exp, rowtok], rtol=0, atol=1e-12)
    # Rounded output is the nearest value of x's dtype (tokens with a kept pair).
    any_kept = (res["route"]["slot"] >= 0).any(axis=1)
    if dtype == "f32":
        np.testing.assert_array_equal(res["out"][any_kept], ref[any_kept].astype(np.float32))
    else:
        t = torch.from_numpy(ref[any_kept]).to(torch.float32).to(torch.bfloat16)
        got = inputs.bf16_bits_to_f32(res["out"][any_kept])
        # float64 -> float32 -> bf16 may double-round; allow that one-ulp case only.
        diff = np.abs(got - t.float().numpy())
        assert (diff <= np.spacing(np.abs(t.float().numpy())) * 2 ** 16 + 0).all()


def test_single_expert_is_a_plain_mlp():
    # E = 1, k = 1, dropless: softmax over one expert is 1, so out = x + MLP(x).
    spec = inputs.LayerSpec("mlp", 12, 8, 16, 1, 1, math.inf, "f32", router="plain", bias_std=0.2)
    layer = inputs.make_layer(spec, seed=11)
    res = oracle.forward(layer["x"], layer["Wr"], layer["br"], layer["W1"], layer["b1"],
                         layer["W2"], layer["b2"], 1, math.inf)
    assert (res["route"]["w"] == 1.0).all() and (res["route"]["slot"] >= 0).all()
    x = torch.from_numpy(layer["x"].astype(np.float64))
    h = x @ torch.from_numpy(layer["W1"][0].astype(np.float64)).T + torch.from_numpy(
        layer["b1"][0].astype(np.float64))
    a = h * torch.sigmoid(h)
    y = a @ torch.from_numpy(layer["W2"][0].astype(np.float64)).T + torch.from_numpy(
        layer["b2"][0].astype(np.float64))
    np.testing.assert_allclose(res["out_f64"], (x + y).numpy(), rtol=0, atol=1e-12)


def test_fully_dropped_tokens_are_bit_exact():
    spec = inputs.LayerSpec("drop", 30, 8, 8, 2, 2, 0.25, "bf16", router="plain")
    layer = inputs.make_layer(spec, seed=2)
    L = inputs.random_logits(30, 2, 9)
    K = oracle.capacity(30, 2, 2, 0.25)
    r = oracle.route(L, 2, K)
    none_kept = ~(r["slot"] >= 0).any(axis=1)
    assert none_kept.sum() > 0
    t0 = int(np.nonzero(none_kept)[0][0])
    layer["x"][t0, ::2] = 0x8000                             # -0.0 must survive untouched
    _, out = oracle.combine_tokens(layer["x"], layer["W1"], layer["b1"], layer["W2"],
                                   layer["b2"], r)
    assert np.array_equal(out[none_kept], layer["x"][none_kept])


def test_capacity_zero_is_identity():
    spec = inputs.LayerSpec("zero", 16, 8, 8, 4, 2, 0.0, "f32", router="plain", bias_std=0.1)
    layer = inputs.make_layer(spec, seed=4)
    res = oracle.forward(layer["x"], layer["Wr"], layer["br"], layer["W1"], layer["b1"],
                         layer["W2"], layer["b2"], 2, 0.0)
    assert res["K"] == 0 and (res["route"]["drop"] == 1).all()
    assert np.array_equal(res["out"].view(np.uint32), layer["x"].view(np.uint32))


# ------------------------------------------------------------------------------------------
# Combine from given expert outputs (the checker of the standalone combine kernel).
# Definition (worked example, token-0 trace "x0 + w0 * y0" and the dropped token 4; the
# dataflow diagram's moe_sum for top_k > 1): out[t] = x[t] + sum over kept j, ascending, of
# w[t, j] * Y[offsets[ids[t, j]] + slot[t, j]], in float64, rounded once; a token with no kept
# pair is x[t] bit for bit.  The reference below is numpy fancy indexing in float64, written
# from that definition and sharing nothing with the oracle's loops.
# ------------------------------------------------------------------------------------------

def _combine_reference(x64, Y64, route, offsets):
    ids, w, slot = route["ids"], route["w"], route["slot"]
    T, k = ids.shape
    kept = slot >= 0
    rows = np.where(kept, offsets[ids] + slot, 0)
    s = np.zeros_like(x64)
    for j in range(k):                                   # j ascending, as the definition
        s = s + np.where(kept[:, j, None], w[:, j, None].astype(np.float64) * Y64[rows[:, j]],
                         0.0)
    return x64 + s, kept.any(axis=1)


def _bf16_of_f64(v):
    return np.array([oracle.bf16_from_double(float(a)) for a in v.reshape(-1)],
                    dtype=np.uint16).reshape(v.shape)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("T,d,E,k,C,seed", [(60, 12, 5, 3, 0.5, 0), (40, 8, 4, 1, 0.75, 1),
                                             (33, 16, 8, 8, 0.4, 2), (20, 4, 3, 2, 0.0, 3)])
def test_combine_given_y_matches_definition(dtype, T, d, E, k, C, seed):
    L = inputs.random_logits(T, E, seed + 40, 2.0)
    K = oracle.capacity(T, E, k, C)
    r = oracle.route(L, k, K)
    off, _ = oracle.dispatch(r["ids"], r["slot"], E)
    n = int(off[-1])
    rng = np.random.default_rng(seed)
    x32 = rng.standard_normal((T, d)).astype(np.float32)
    # Large expert outputs against a unit residual: a float32 accumulation of the k terms
    # would round away low bits that the float64 sum keeps, and change the rounded output.
    Y32 = (rng.standard_normal((max(n, 1), d)) * 1e4).astype(np.float32)
    none_kept = ~(r["slot"] >= 0).any(axis=1)
    if dtype == "bf16":
        x, Y = inputs.f32_to_bf16_bits(x32), inputs.f32_to_bf16_bits(Y32)
        if none_kept.any():
            x[np.nonzero(none_kept)[0][0], 0] = 0x8000           # -0.0
    else:
        x, Y = x32, Y32
        if none_kept.any():
            x[np.nonzero(none_kept)[0][0], 0] = np.float32(-0.0)
    out64, out = oracle.combine_given_y(x, Y, r, off)
    ref64, any_kept = _combine_reference(_f64(x), _f64(Y), r, off)
    # Same float64 operations in the same order: identical to the last bit.
    assert np.array_equal(out64, ref64)
    if dtype == "f32":
        assert np.array_equal(out[any_kept], ref64[any_kept].astype(np.float32))
    else:
        assert np.array_equal(out[any_kept], _bf16_of_f64(ref64[any_kept]))
    assert out[none_kept].tobytes() == x[none_kept].tobytes()
    if C == 0.0:
        assert none_kept.all()
    elif k > 1:
        partly = (r["slot"] >= 0).any(axis=1) & (r["slot"] < 0).any(axis=1)
        assert partly.any(), "the case must hold partially dropped tokens"


def test_combine_given_y_detects_float_accumulation():
    # w = 0.1f times Y = 2^24 - 1 and -(2^24 - 2): both products are exact in float64 and their
    # sum is exactly w, but each product rounds to a multiple of 1/8 in float32, so a float32
    # accumulation gives 0 or 0.125 instead of 0.1f.  Pins the float64 accumulation.
    w32 = np.float32(0.1)
    x = np.zeros((1, 1), np.float32)
    Y = np.array([[16777215.0], [-16777214.0]], np.float32)
    route = dict(ids=np.array([[0, 1]], np.int32), w=np.array([[w32, w32]], np.float32),
                 slot=np.array([[0, 0]], np.int32))
    off = np.array([0, 1, 2], np.int32)
    out64, out = oracle.combine_given_y(x, Y, route, off)
    f32_sum = np.float32(np.float32(w32 * Y[0, 0]) + np.float32(w32 * Y[1, 0]))
    assert f32_sum != w32
    assert out64[0, 0] == float(w32) and out[0, 0] == w32


def test_combine_given_y_agrees_with_combine_tokens():
    # Expert outputs from the oracle's own FFN rows (pinned against torch float64 above), then
    # the standalone combine: the same layer output as the oracle's whole-layer path.
    spec = inputs.LayerSpec("cg", 48, 16, 24, 6, 2, 0.6, "f32", router="normal",
                            router_bias=0.3, bias_std=0.1)
    layer = inputs.make_layer(spec, seed=3)
    res = oracle.forward(layer["x"], layer["Wr"], layer["br"], layer["W1"], layer["b1"],
                         layer["W2"], layer["b2"], 2, 0.6)
    off, rowtok = oracle.dispatch(res["route"]["ids"], res["route"]["slot"], 6)
    row_exp = np.repeat(np.arange(6, dtype=np.int32), np.diff(off))
    Y = oracle.expert_rows(layer["x"], layer["W1"], layer["b1"], layer["W2"], layer["b2"],
                           rowtok, row_exp).astype(np.float32)
    out64, out = oracle.combine_given_y(layer["x"], Y, res["route"], off)
    np.testing.assert_allclose(out64, res["out_f64"], rtol=0, atol=1e-5)
    dropped = (res["route"]["slot"] < 0).any(axis=1)
    assert dropped.any()


def test_worked_example_combine_given_y():
    # Token 0 keeps its expert: out0 = x0 + w0 * y0 with y0 the row at offsets[0] + slot; token
    # 4 is dropped and comes back unchanged.
    layer = inputs.make_layer(inputs.CONFIGS["tiny_f32"], seed=0)
    r = oracle.route(layer["logits"], 1, 2)
    off, rowtok = oracle.dispatch(r["ids"], r["slot"], 4)
    Y = np.arange(int(off[-1]) * 4, dtype=np.float32).reshape(-1, 4) / 8.0
    out64, out = oracle.combine_given_y(layer["x"], Y, r, off)
    row0 = int(off[r["ids"][0, 0]] + r["slot"][0, 0])
    assert rowtok[row0] == 0
    np.testing.assert_array_equal(
        out64[0], layer["x"][0].astype(np.float64) + float(r["w"][0, 0]) * Y[row0].astype(np.float64))
    assert out[4].tobytes() == layer["x"][4].tobytes()


# ------------------------------------------------------------------------------------------
# Logits and bfloat16 rounding
# ------------------------------------------------------------------------------------------

def test_logits_match_float64_matmul():
    spec = inputs.LayerSpec("lg", 64, 96, 8, 12, 2, 1.0, "bf16", router="normal", router_bias=0.5)
    layer = inputs.make_layer(spec, seed=8)
    L = oracle.logits(layer["x"], layer["Wr"], layer["br"])
    ref = _f64(layer["x"]) @ layer["Wr"].astype(np.float64) + layer["br"].astype(np.float64)
    np.testing.assert_allclose(L, ref, rtol=2 ** -23, atol=1e-9)


def test_bf16_rounding_against_exhaustive_table():
    # Every finite non-negative bfloat16 value, sorted; the nearest (ties to even) is searched.
    pats = np.arange(0, 0x7F80, dtype=np.uint16)
    vals = inputs.bf16_bits_to_f32(pats).astype(np.float64)
    rng = np.random.default_rng(1)
    probe = np.concatenate([rng.standard_normal(3000) * 10 ** rng.uniform(-6, 6, 3000),
                            (vals[1000:1100] + vals[1001:1101]) / 2,         # exact ties
                            np.array([0.0, -0.0, 1e-45, 3.3e38, -2.5])])
    for v in probe:
        a = abs(v)
        i = int(np.searchsorted(vals, a))
        cands = [j for j in (i - 1, i) if 0 <= j < vals.size]
        best = min(cands, key=lambda j: (abs(vals[j] - a), pats[j] & 1))
        expect = int(pats[best]) | (0x8000 if math.copysign(1.0, v) < 0 else 0)
        assert oracle.bf16_from_double(v) == expect, v


# ------------------------------------------------------------------------------------------
# Routing-policy flags: renormalised top-k weights and arrival-order capacity.
# ------------------------------------------------------------------------------------------

@pytest.mark.parametrize("seed", range(4))
def test_renormalized_weights(seed):
    T, E, k = 300, 16, 4
    L = inputs.random_logits(T, E, seed, 2.0)
    K = oracle.capacity(T, E, k, 1.0)
    plain = oracle.route(L, k, K)
    r = oracle.route(L, k, K, oracle.RENORMALIZE)
    assert np.array_equal(r["ids"], plain["ids"])            # same experts, same order
    p = torch.softmax(torch.from_numpy(L.astype(np.float64)), dim=1).numpy()
    top = np.take_along_axis(p, r["ids"].astype(np.int64), 1)
    ref = top / top.sum(axis=1, keepdims=True)
    np.testing.assert_allclose(r["w"], ref, rtol=2e-6, atol=0)
    np.testing.assert_allclose(r["w"].astype(np.float64).sum(axis=1), 1.0, atol=4e-7 * k)
    # Drop priority follows the renormalised weights.
    for e in range(E):
        m = r["ids"] == e
        kept, dropped = m & (r["slot"] >= 0), m & (r["slot"] < 0)
        if dropped.any():
            assert r["w"][kept].min() >= r["w"][dropped].max()


@pytest.mark.parametrize("seed", range(4))
@pytest.mark.parametrize("T,E,k,C", [(200, 8, 2, 0.5), (64, 4, 1, 1.0), (500, 16, 4, 0.25)])
def test_arrival_order_capacity_brute_force(seed, T, E, k, C):
    L = inputs.random_logits(T, E, seed)
    K = oracle.capacity(T, E, k, C)
    r = oracle.route(L, k, K, oracle.ARRIVAL_ORDER)
    for e in range(E):
        cand = [(t, j) for t in range(T) for j in range(k) if r["ids"][t, j] == e]
        for i, (t, j) in enumerate(cand):                    # ascending token order
            if i < K:
                assert r["slot"][t, j] == i and r["drop"][t, j] == 0
            else:
                assert r["slot"][t, j] == -1 and r["drop"][t, j] == 1


def test_arrival_order_drops_the_late_token():
    # The confidence-order example: under arrival order expert 0 keeps tokens 0 and 1 and
    # drops token 2, although token 0 is its least confident.
    L = np.array([[0.5, 0, 0], [3.0, 0, 0], [2.0, 0, 0], [0, 1.0, 0]], np.float32)
    r = oracle.route(L, 1, 2, oracle.ARRIVAL_ORDER)
    assert r["drop"][:, 0].tolist() == [0, 0, 1, 0]
    g = _worked()
    layer = inputs.make_layer(inputs.CONFIGS["tiny_f32"], seed=0)
    r = oracle.route(layer["logits"], 1, g["K"], oracle.ARRIVAL_ORDER)
    assert np.nonzero(r["drop"][:, 0])[0].tolist() == g["dropped_tokens"]   # token 4 is last


def test_both_flags_compose():
    T, E, k = 400, 8, 3
    L = inputs.random_logits(T, E, 9, 1.5)
    K = oracle.capacity(T, E, k, 0.6)
    r = oracle.route(L, k, K, oracle.RENORMALIZE | oracle.ARRIVAL_ORDER)
    rn = oracle.route(L, k, K, oracle.RENORMALIZE)
    ra = oracle.route(L, k, K, oracle.ARRIVAL_ORDER)
    assert np.array_equal(r["w"].view(np.uint32), rn["w"].view(np.uint32))
    assert np.array_equal(r["slot"], ra["slot"])


# ------------------------------------------------------------------------------------------
# Gated experts (the dataflow diagram's GEMM 1 -> "SiLU x mul" -> GEMM 2): a = SiLU(g) * u.
# ------------------------------------------------------------------------------------------

def dense_gated_reference(layer, route):
    x = torch.from_numpy(_f64(layer["x"]))
    W1 = torch.from_numpy(_f64(layer["W1"]))
    W2 = torch.from_numpy(_f64(layer["W2"]))
    b1 = torch.from_numpy(layer["b1"].astype(np.float64))
    b2 = torch.from_numpy(layer["b2"].astype(np.float64))
    E, d, F = W2.shape
    Y = []
    for e in range(E):
        h = Fnn.linear(x, W1[e], b1[e])
        g, u = h[:, :F], h[:, F:]
        Y.append(Fnn.linear(Fnn.silu(g) * u, W2[e], b2[e]))
    Y = torch.stack(Y)
    T, k = route["ids"].shape
    out = x.clone()
    for t in range(T):
        for j in range(k):
            if route["slot"][t, j] >= 0:
                out[t] += float(route["w"][t, j]) * Y[route["ids"][t, j], t]
    return out.numpy(), Y.numpy()


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("T,d,F,E,k,C", [(24, 8, 16, 4, 1, 0.75), (40, 16, 12, 6, 2, 1.0)])
def test_gated_forward_matches_dense_reference(dtype, T, d, F, E, k, C):
    spec = inputs.LayerSpec("g", T, d, F, E, k, C, dtype, router="normal", router_bias=0.3,
                            bias_std=0.1, gated=True)
    layer = inputs.make_layer(spec, seed=T + F)
    assert layer["W1"].shape == (E, 2 * F, d)
    res = oracle.forward(layer["x"], layer["Wr"], layer["br"], layer["W1"], layer["b1"],
                         layer["W2"], layer["b2"], k, C, flags=oracle.GATED)
    ref, Y = dense_gated_reference(layer, res["route"])
    np.testing.assert_allclose(res["out_f64"], ref, rtol=0, atol=1e-12)
    offsets, rowtok = oracle.dispatch(res["route"]["ids"], res["route"]["slot"], E)
    row_exp = np.repeat(np.arange(E, dtype=np.int32), np.diff(offsets))
    Yo, Ho = oracle.expert_rows(layer["x"], layer["W1"], layer["b1"], layer["W2"], layer["b2"],
                                rowtok, row_exp, want_h=True, flags=oracle.GATED)
    np.testing.assert_allclose(Yo, Y[row_exp, rowtok], rtol=0, atol=1e-12)
    # Zero up-projection -> zero expert output but the bias b2.
    layer["W1"][:, F:, :] = 0
    layer["b1"][:, F:] = 0
    Yz = oracle.expert_rows(layer["x"], layer["W1"], layer["b1"], layer["W2"], layer["b2"],
                            rowtok, row_exp, flags=oracle.GATED)
    np.testing.assert_allclose(Yz, layer["b2"][row_exp].astype(np.float64), rtol=0, atol=0)
