"""The oracle's routing against exhaustive references on random small batches (hypothesis,
derandomised; CPU only).

For every drawn batch: the top-k ids are the k largest logits with ties to the lower expert;
the weights are the float64 softmax at those ids (divided by their sum with renormalisation);
each expert keeps min(received, K) pairs, the highest-weight ones with ties to the lower token
(or its first K in token order with arrival order); a kept pair's slot is its rank among the
expert's kept tokens in token order; everything else is dropped with slot -1.  ("Expert Networks >
Worked Example: Expert Specialization", capacity paragraph and token-0 trace; "Some Tokens Do Not
Get In", "Past the edge".)
"""
import math

import numpy as np
import torch
from hypothesis import given, settings
from hypothesis import strategies as st

import oracle


@st.composite
def batches(draw):
    T = draw(st.integers(1, 40))
    E = draw(st.integers(1, 8))
    k = draw(st.integers(1, E))
    C = draw(st.sampled_from([0.0, 0.3, 0.75, 1.0, 1.5, math.inf]))
    flags = draw(st.integers(0, 3))
    levels = draw(st.sampled_from([2, 3, 5, 0]))            # 0: continuous logits
    seed = draw(st.integers(0, 2 ** 20))
    rng = np.random.default_rng(seed)
    if levels:
        L = (rng.integers(0, levels, size=(T, E)) * 0.5).astype(np.float32)
    else:
        L = rng.standard_normal((T, E)).astype(np.float32)
    return L, k, C, flags


@settings(max_examples=300, deadline=None, derandomize=True)
@given(batches())
def test_route_against_exhaustive_reference(case):
    L, k, C, flags = case
    T, E = L.shape
    K = oracle.capacity(T, E, k, C)
    r = oracle.route(L, k, K, flags)
    p = torch.softmax(torch.from_numpy(L.astype(np.float64)), dim=1).numpy()
    ids = np.array([sorted(range(E), key=lambda e: (-float(L[t, e]), e))[:k] for t in range(T)])
    assert np.array_equal(r["ids"], ids)
    wref = np.take_along_axis(p, ids, 1)
    if flags & oracle.RENORMALIZE:
        wref = wref / wref.sum(axis=1, keepdims=True)
    np.testing.assert_allclose(r["w"], wref, rtol=2e-6, atol=1e-30)
    w = r["w"]
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


@st.composite
def small_layers(draw):
    from expert_ffn_layer_router_b200 import inputs
    T = draw(st.integers(1, 24))
    d = draw(st.sampled_from([4, 8, 16]))
    F = draw(st.sampled_from([4, 8, 12]))
    E = draw(st.integers(1, 5))
    k = draw(st.integers(1, E))
    C = draw(st.sampled_from([0.0, 0.5, 1.0, math.inf]))
    flags = draw(st.integers(0, 7))
    dtype = draw(st.sampled_from(["f32", "bf16"]))
    seed = draw(st.integers(0, 2 ** 16))
    spec = inputs.LayerSpec("p", T, d, F, E, k, C, dtype, router="normal", router_bias=0.3,
                            bias_std=0.1, gated=bool(flags & 4))
    return inputs.make_layer(spec, seed=seed), k, C, flags


@settings(max_examples=150, deadline=None, derandomize=True)
@given(small_layers())
def test_forward_against_dense_reference(case):
    """The oracle's layer output (float64, before rounding) equals every expert run on every
    token in torch float64 and masked by the oracle's routing: x + sum over kept j of w * y
    (plain or gated experts)."""
    from tests.test_oracle_pins import dense_gated_reference, dense_reference
    layer, k, C, flags = case
    res = oracle.forward(layer["x"], layer["Wr"], layer["br"], layer["W1"], layer["b1"],
                         layer["W2"], layer["b2"], k, C, flags=flags)
    ref, _ = (dense_gated_reference if flags & oracle.GATED else dense_reference)(
        layer, res["route"])
    np.testing.assert_allclose(res["out_f64"], ref, rtol=0, atol=1e-12)
    none_kept = ~(res["route"]["slot"] >= 0).any(axis=1)
    assert res["out"][none_kept].tobytes() == layer["x"][none_kept].tobytes()


@st.composite
def given_routings(draw):
    T = draw(st.integers(1, 50))
    E = draw(st.integers(1, 8))
    k = draw(st.integers(1, E))
    K = draw(st.integers(0, 2 * T))
    flags = draw(st.sampled_from([0, 2]))
    ties = draw(st.booleans())
    seed = draw(st.integers(0, 2 ** 20))
    rng = np.random.default_rng(seed)
    ids = np.stack([rng.permutation(E)[:k] for _ in range(T)]).astype(np.int32)
    w = ((rng.integers(1, 4, size=(T, k)) * 0.25) if ties else rng.random((T, k))).astype(
        np.float32)
    return ids, w, E, K, flags


@settings(max_examples=300, deadline=None, derandomize=True)
@given(given_routings())
def test_select_against_exhaustive_reference(case):
    """Capacity selection of an arbitrary routing, and its expert-sorted layout: offsets are the
    prefix sums of the kept counts and row offsets[e] + slot holds the kept token."""
    ids, w, E, K, flags = case
    T, k = ids.shape
    r = oracle.select(ids, w, E, K, flags)
    for e in range(E):
        cand = [(t, j) for t in range(T) for j in range(k) if ids[t, j] == e]
        ranked = sorted(cand) if flags & oracle.ARRIVAL_ORDER else \
            sorted(cand, key=lambda tj: (-float(w[tj]), tj[0]))
        keep = set(ranked[:K])
        kept_sorted = sorted(keep)
        assert r["kept"][e] == min(len(cand), K)
        for tj in cand:
            if tj in keep:
                assert r["drop"][tj] == 0 and r["slot"][tj] == kept_sorted.index(tj)
            else:
                assert r["drop"][tj] == 1 and r["slot"][tj] == -1
    offsets, rowtok = oracle.dispatch(ids, r["slot"], E)
    assert offsets[0] == 0 and np.array_equal(np.diff(offsets), r["kept"])
    for t in range(T):
        for j in range(k):
            if r["slot"][t, j] >= 0:
                assert rowtok[offsets[ids[t, j]] + r["slot"][t, j]] == t
