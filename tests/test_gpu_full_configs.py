"""The whole forward (moe_forward) at the workloads' full sizes, in the configuration the bench
times.

Routing is compared in full and bit for bit with the oracle's routing of the fp32 logits the
forward exported (ids, weight bits, slots, drops, counts); outputs on a seeded sample of tokens
(random tokens plus partially and fully dropped ones), since each token's output depends only
on its own row given the routing.  Fully dropped tokens must come out bit for bit equal to their
input.  A second, looser comparison routes the oracle's own float64 logits: expert sets exactly,
capacity decisions exactly except where the oracle's weights tie within the logit error at a
capacity boundary.
"""
import numpy as np
import pytest

import oracle
from expert_ffn_layer_router_b200 import inputs
from tests.test_gpu_parity import _forward_check

pytestmark = pytest.mark.gpu


def _sample_tokens(spec, seed, n_random):
    """Random tokens plus tokens with dropped pairs (from the oracle's own routing)."""
    L = inputs.make_layer(spec, seed=seed, weights=False)
    logits = oracle.logits(L["x"], L["Wr"], L["br"])
    r = oracle.route(logits, spec.k, oracle.capacity(spec.T, spec.E, spec.k, spec.C))
    rng = np.random.default_rng(seed + 17)
    pick = set(rng.choice(spec.T, size=min(n_random, spec.T), replace=False).tolist())
    dropped_any = np.nonzero((r["slot"] < 0).any(axis=1))[0]
    pick.update(rng.permutation(dropped_any)[:64].tolist())
    return np.array(sorted(pick), dtype=np.int32)


@pytest.mark.parametrize("name,n_random", [("bf16_e8_top2", 256), ("skewed_e64_top6", 384),
                                           ("decode_e64_top8", 64),
                                           ("prefill_e128_top8", 192)])
def test_forward_full_size(name, n_random):
    spec = inputs.CONFIGS[name]
    tokens = _sample_tokens(spec, 0, n_random)
    g, ro = _forward_check(spec, seed=0, tokens=tokens)
    if name == "skewed_e64_top6":
        assert (ro["slot"] < 0).sum() > 0
    if name == "decode_e64_top8":
        assert (ro["slot"] >= 0).all()              # dropless
