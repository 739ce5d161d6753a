"""Random small layers (hypothesis, derandomised): moe_forward against the oracle.

Each example draws a layer shape, a capacity factor and the flag word, and checks what holds
for every layer: the routing (ids, weight bits, slots, drop mask, counts) equals the oracle's
routing of the forward's own fp32 logits bit for bit, the expert offsets are the prefix sums
of the kept counts, every output row is within the dtype's tolerance of the oracle's layer, and
a token whose pairs were all dropped leaves bit for bit as it came in.  Shapes span the
small-batch and large-batch router and dispatch paths (T*k on both sides of 1024, T on both
sides of 1024 for the bf16 router).
"""
import math

import numpy as np
import pytest
import torch
from hypothesis import HealthCheck, given, settings
from hypothesis import strategies as st

import oracle
from expert_ffn_layer_router_b200 import inputs
from tests.gpu_util import assert_close, to_dev, to_host

pytestmark = pytest.mark.gpu


@st.composite
def layers(draw):
    T = draw(st.one_of(st.integers(1, 700), st.integers(1025, 2600)))
    E = draw(st.integers(1, 40))
    k = draw(st.integers(1, min(E, 8)))
    d = draw(st.sampled_from([64, 128, 192]))
    F = draw(st.sampled_from([64, 128, 320]))
    C = draw(st.sampled_from([0.0, 0.5, 1.0, 1.25, 2.0, math.inf]))
    flags = draw(st.integers(0, 7))
    dtype = draw(st.sampled_from(["bf16", "bf16", "f32"]))
    seed = draw(st.integers(0, 2 ** 16))
    spec = inputs.LayerSpec("h", T, d, F, E, k, C, dtype, router="normal", router_bias=0.5,
                            bias_std=0.05, gated=bool(flags & 4))
    return spec, flags, seed


@settings(max_examples=100, deadline=None, derandomize=True, print_blob=True,
          suppress_health_check=[HealthCheck.too_slow, HealthCheck.data_too_large])
@given(layers())
def test_forward_random_layers(case):
    from expert_ffn_layer_router_b200 import moe
    spec, flags, seed = case
    L = inputs.make_layer(spec, seed=seed)
    layer = moe.MoELayer(spec.T, spec.d_model, spec.d_ff, spec.E, spec.k, spec.C, spec.dtype,
                         flags=flags)
    args = [to_dev(L[n]) for n in ("x", "Wr", "br", "W1", "b1", "W2", "b2")]
    if spec.dtype == "bf16" and spec.gated and spec.d_ff % 128:
        # Gated bf16 tiles hold 128 gate and 128 up rows: the header's documented limit.
        with pytest.raises(moe.MoeError) as exc:
            layer.forward(*args)
        assert exc.value.status == 2           # MOE_ERR_UNSUPPORTED
        return
    out, rt = layer.forward(*args, want_routing=True)
    torch.cuda.synchronize()
    assert moe.moe_get_device_status(layer.ws) == 0
    g = {k_: to_host(v) for k_, v in rt.items()}
    rg = oracle.route(g["logits_out"], spec.k, layer.K, flags & 3)
    assert np.array_equal(g["ids_out"], rg["ids"]), "expert ids differ"
    assert np.array_equal(g["w_out"].view(np.uint32), rg["w"].view(np.uint32)), "weights differ"
    assert np.array_equal(g["slot_out"], rg["slot"]), "slots differ"
    assert np.array_equal(g["drop_out"], rg["drop"]), "drop mask differs"
    received = np.bincount(rg["ids"].ravel(), minlength=spec.E)
    kept = np.bincount(rg["ids"][rg["slot"] >= 0], minlength=spec.E)
    assert np.array_equal(g["counts_out"][:spec.E], received), "received counts differ"
    assert np.array_equal(g["counts_out"][spec.E:], kept), "kept counts differ"
    assert kept.max(initial=0) <= layer.K
    _, ref = oracle.combine_tokens(L["x"], L["W1"], L["b1"], L["W2"], L["b2"], rg, flags=flags)
    got = to_host(out)
    assert_close(got, ref, spec.dtype, "layer output")
    none_kept = ~(rg["slot"] >= 0).any(axis=1)
    assert got[none_kept].tobytes() == L["x"][none_kept].tobytes()


@st.composite
def tied_logits(draw):
    T = draw(st.one_of(st.integers(1, 300), st.integers(1025, 5000)))
    E = draw(st.integers(1, 64))
    k = draw(st.integers(1, min(E, 8)))
    C = draw(st.sampled_from([0.25, 0.5, 1.0, 1.5, math.inf]))
    flags = draw(st.integers(0, 3))
    levels = draw(st.integers(1, 4))           # how many distinct logit values: ties everywhere
    seed = draw(st.integers(0, 2 ** 16))
    rng = np.random.default_rng(seed)
    vals = np.array([-1.0, 0.0, 0.5, 2.0], np.float32)[:levels]
    L = vals[rng.integers(0, levels, size=(T, E))].astype(np.float32)
    return L, T, E, k, C, flags


@settings(max_examples=60, deadline=None, derandomize=True, print_blob=True,
          suppress_health_check=[HealthCheck.too_slow, HealthCheck.data_too_large])
@given(tied_logits())
def test_route_heavy_ties(case):
    """moe_route on logits drawn from at most four values: ties in the top-k (lower expert
    wins) and at every capacity boundary (lower token wins, or the first K with arrival order)
    must match the oracle bit for bit."""
    from expert_ffn_layer_router_b200 import moe
    L, T, E, k, C, flags = case
    layer = moe.MoELayer(T, 64, 64, E, k, C, "bf16", flags=flags)
    r = layer.route(to_dev(L))
    torch.cuda.synchronize()
    assert moe.moe_get_device_status(layer.ws) == 0
    g = {k_: to_host(v) for k_, v in r.items()}
    ro = oracle.route(L, k, layer.K, flags)
    assert np.array_equal(g["ids"], ro["ids"]), "expert ids differ"
    assert np.array_equal(g["w"].view(np.uint32), ro["w"].view(np.uint32)), "weights differ"
    assert np.array_equal(g["slot"], ro["slot"]), "slots differ"
    assert np.array_equal(g["drop"], ro["drop"]), "drop mask differs"
    kept = np.bincount(ro["ids"][ro["slot"] >= 0], minlength=E)
    assert np.array_equal(g["counts"][E:], kept)


@st.composite
def medium_layers(draw):
    T = draw(st.integers(1, 20000))
    E = draw(st.sampled_from([8, 16, 33, 64, 128]))
    k = draw(st.integers(1, min(E, 8)))
    d = 64 * draw(st.integers(1, 32))
    flags = draw(st.integers(0, 7))
    F = (128 if flags & 4 else 64) * draw(st.integers(1, 16 if flags & 4 else 32))
    C = draw(st.sampled_from([0.5, 1.0, 1.25, math.inf]))
    seed = draw(st.integers(0, 2 ** 16))
    spec = inputs.LayerSpec("m", T, d, F, E, k, C, "bf16", router="normal", router_bias=0.5,
                            bias_std=0.05, gated=bool(flags & 4))
    return spec, flags, seed


@settings(max_examples=12, deadline=None, derandomize=True, print_blob=True,
          suppress_health_check=[HealthCheck.too_slow, HealthCheck.data_too_large])
@given(medium_layers())
def test_forward_random_medium_layers(case):
    """Larger random bf16 layers (up to 20,000 tokens, d_model and d_ff up to 2048): several
    m-tiles per expert, pair and single tiles, weight-streaming tiles and the tensor-core router
    all occur.  Routing is checked on every token; outputs on 256 sampled tokens plus every
    token whose pairs were all dropped."""
    from expert_ffn_layer_router_b200 import moe
    spec, flags, seed = case
    L = inputs.make_layer(spec, seed=seed)
    layer = moe.MoELayer(spec.T, spec.d_model, spec.d_ff, spec.E, spec.k, spec.C, spec.dtype,
                         flags=flags)
    args = [to_dev(L[n]) for n in ("x", "Wr", "br", "W1", "b1", "W2", "b2")]
    out, rt = layer.forward(*args, want_routing=True)
    torch.cuda.synchronize()
    assert moe.moe_get_device_status(layer.ws) == 0
    g = {k_: to_host(v) for k_, v in rt.items()}
    rg = oracle.route(g["logits_out"], spec.k, layer.K, flags & 3)
    assert np.array_equal(g["ids_out"], rg["ids"]), "expert ids differ"
    assert np.array_equal(g["w_out"].view(np.uint32), rg["w"].view(np.uint32)), "weights differ"
    assert np.array_equal(g["slot_out"], rg["slot"]), "slots differ"
    assert np.array_equal(g["drop_out"], rg["drop"]), "drop mask differs"
    rng = np.random.default_rng(seed)
    none_kept = ~(rg["slot"] >= 0).any(axis=1)
    tokens = np.unique(np.concatenate([rng.choice(spec.T, size=min(256, spec.T), replace=False),
                                       np.nonzero(none_kept)[0][:64]])).astype(np.int32)
    _, ref = oracle.combine_tokens(L["x"], L["W1"], L["b1"], L["W2"], L["b2"], rg, tokens,
                                   flags=flags)
    got = to_host(out)
    assert_close(got[tokens], ref, spec.dtype, "layer output")
    assert got[none_kept].tobytes() == L["x"][none_kept].tobytes()
