"""Seeded synthetic inputs for the MoE layer forward.

This module serves both the CUDA library's tests and bench and the CPU oracle's tests.  It holds
none of the layer's arithmetic; it only draws numbers.  The one computation it does is a float64
screen of x @ Wr + br. That screen redraws a token whose k-th and (k+1)-th router logits are
closer than ``GAP``, so that top-k membership cannot depend on how the logits are rounded.

Recipe (every array drawn from ``numpy.random.default_rng(seed)`` in this fixed order:
x, Wr, br, W1, b1, W2, b2):
  * x ~ N(0, 1), rounded to the layer dtype (bfloat16: round to nearest even from float32);
  * Wr ~ N(0, 0.02^2) float32, shape [d_model, E];
  * br: none, a Zipf(s) probability-mass bias over a random permutation of expert ranks
    (b_e = rank_e^-s / sum_j j^-s), or N(0, sd^2);
  * W1 [E, d_ff, d_model], W2 [E, d_model, d_ff] ~ N(0, 1/fan_in), i.e. std = 1/sqrt(fan_in);
  * b1 [E, d_ff], b2 [E, d_model] float32, zero or N(0, sd^2).
Redrawn x rows come from ``default_rng([seed, 7919, t, attempt])``.
"""
from __future__ import annotations

import dataclasses
import math

import numpy as np

GAP = 1e-3


@dataclasses.dataclass
class LayerSpec:
    name: str
    T: int
    d_model: int
    d_ff: int
    E: int
    k: int
    C: float                      # capacity factor; math.inf = dropless
    dtype: str                    # "f32" or "bf16"
    router: str = "plain"         # "plain" | "zipf" | "normal" | "given" (logits handed in)
    router_bias: float = 0.0      # zipf exponent s, or std of the normal router bias
    bias_std: float = 0.0         # std of b1/b2 (0 = zero biases)
    gated: bool = False           # gated experts: W1 [E, 2*d_ff, d_model] (gate rows, up rows)

    @property
    def pairs(self) -> int:
        return self.T * self.k


# The five workloads: the worked example's shape and four bf16 layers.
CONFIGS = {
    "tiny_f32": LayerSpec("tiny_f32", 8, 4, 8, 4, 1, 1.25, "f32", router="given", bias_std=0.1),
    "bf16_e8_top2": LayerSpec("bf16_e8_top2", 4096, 2048, 8192, 8, 2, 1.25, "bf16"),
    "skewed_e64_top6": LayerSpec("skewed_e64_top6", 16384, 2048, 1408, 64, 6, 1.0, "bf16",
                                 router="zipf", router_bias=1.1),
    "decode_e64_top8": LayerSpec("decode_e64_top8", 64, 2048, 1024, 64, 8, math.inf, "bf16"),
    "prefill_e128_top8": LayerSpec("prefill_e128_top8", 65536, 4096, 1536, 128, 8, 1.5, "bf16",
                                   router="normal", router_bias=0.5, bias_std=0.01),
}
CONFIG_ORDER = ["tiny_f32", "bf16_e8_top2", "skewed_e64_top6", "decode_e64_top8",
                "prefill_e128_top8"]


def f32_to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """Round float32 to bfloat16 (nearest, ties to even) and return the raw 16-bit patterns.

    Works in uint32 (no overflow for any non-NaN pattern: the largest, -FLT_MAX, plus 0x8000
    stays below 2^32) in chunks, so multi-GB weight tensors need no 64-bit temporaries."""
    a = np.ascontiguousarray(a, dtype=np.float32)
    flat = a.reshape(-1)
    out = np.empty(flat.size, np.uint16)
    step = 1 << 24
    for i in range(0, flat.size, step):
        b = flat[i:i + step].view(np.uint32)
        r = b + np.uint32(0x7FFF) + ((b >> np.uint32(16)) & np.uint32(1))
        out[i:i + step] = (r >> np.uint32(16)).astype(np.uint16)
        nan = np.isnan(flat[i:i + step])
        if nan.any():
            out[i:i + step][nan] = 0x7FC0
    return out.reshape(a.shape)


def bf16_bits_to_f32(h: np.ndarray) -> np.ndarray:
    return (np.ascontiguousarray(h, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def _to_dtype(a32: np.ndarray, dtype: str) -> np.ndarray:
    return f32_to_bf16_bits(a32) if dtype == "bf16" else np.ascontiguousarray(a32, np.float32)


def _as_f64(a: np.ndarray) -> np.ndarray:
    return bf16_bits_to_f32(a).astype(np.float64) if a.dtype == np.uint16 else a.astype(np.float64)


def _worked_example_logits() -> np.ndarray:
    """Hand-built router logits for the worked example's 8 tokens and 4 experts.

    Tokens 0, 2, 4 pick expert 0; 1, 5 pick expert 1; 3 picks expert 2; 6, 7 pick expert 3.
    Token 0's softmax weight on expert 0 is e^3 / (e^3 + 3) = 0.870, and token 4 has the lowest
    confidence of expert 0's three tokens.
    """
    L = np.zeros((8, 4), np.float32)
    top = {0: (0, 3.0), 1: (1, 2.5), 2: (0, 2.0), 3: (2, 1.5), 4: (0, 1.0), 5: (1, 1.8),
           6: (3, 2.2), 7: (3, 1.2)}
    for t, (e, v) in top.items():
        L[t, e] = v
    return L


def _topk_gap_ok(L64: np.ndarray, k: int) -> np.ndarray:
    """Per token: is the k-th largest logit at least GAP above the (k+1)-th?"""
    E = L64.shape[1]
    if k >= E:
        return np.ones(L64.shape[0], bool)
    part = -np.sort(-L64, axis=1)
    return (part[:, k - 1] - part[:, k]) >= GAP


def make_layer(spec: LayerSpec, seed: int = 0, T: int | None = None,
               weights: bool = True) -> dict:
    """Draw one layer's inputs. ``T`` overrides the token count (x and the gap screen only).

    ``weights=False`` skips W1/b1/W2/b2 (drawn after x, Wr and br, so those are unchanged)."""
    T = spec.T if T is None else T
    d, F, E, k = spec.d_model, spec.d_ff, spec.E, spec.k
    rng = np.random.default_rng(seed)
    x32 = rng.standard_normal((T, d), dtype=np.float32)
    if spec.name == "tiny_f32" and T == 8:
        x32[0] = np.array([0.5, -0.3, 0.8, 0.2], np.float32)
    Wr = (rng.standard_normal((d, E), dtype=np.float32) * np.float32(0.02)).astype(np.float32)
    br = None
    if spec.router == "zipf":
        ranks = rng.permutation(E) + 1
        z = ranks.astype(np.float64) ** (-spec.router_bias)
        br = (z / np.sum(np.arange(1, E + 1, dtype=np.float64) ** (-spec.router_bias))
              ).astype(np.float32)
    elif spec.router == "normal":
        br = (rng.standard_normal(E, dtype=np.float32) * np.float32(spec.router_bias)
              ).astype(np.float32)
    if weights:
        F1 = 2 * F if spec.gated else F
        W1 = rng.standard_normal((E, F1, d), dtype=np.float32)
        W1 *= np.float32(1.0 / math.sqrt(d))
        b1 = (rng.standard_normal((E, F1), dtype=np.float32) * np.float32(spec.bias_std)
              if spec.bias_std > 0 else np.zeros((E, F1), np.float32))
        W2 = rng.standard_normal((E, d, F), dtype=np.float32)
        W2 *= np.float32(1.0 / math.sqrt(F))
        b2 = (rng.standard_normal((E, d), dtype=np.float32) * np.float32(spec.bias_std)
              if spec.bias_std > 0 else np.zeros((E, d), np.float32))
    else:
        W1 = b1 = W2 = b2 = None

    x = _to_dtype(x32, spec.dtype)
    logits = None
    redrawn = 0
    if spec.router == "given":
        logits = _worked_example_logits() if T == 8 else (
            rng.standard_normal((T, E), dtype=np.float32))
    else:
        # Gap screen: redraw x rows whose top-k boundary is a near-tie.
        Wr64 = Wr.astype(np.float64)
        br64 = 0.0 if br is None else br.astype(np.float64)
        L64 = _as_f64(x) @ Wr64 + br64
        bad = np.nonzero(~_topk_gap_ok(L64, k))[0]
        for t in bad:
            for attempt in range(1, 1000):
                sub = np.random.default_rng([seed, 7919, int(t), attempt])
                row = _to_dtype(sub.standard_normal((1, d), dtype=np.float32), spec.dtype)
                l64 = _as_f64(row) @ Wr64 + br64
                if _topk_gap_ok(l64, k)[0]:
                    x[t] = row[0]
                    redrawn += 1
                    break
            else:
                raise RuntimeError("gap screen failed to redraw token %d" % t)
    if weights:
        W1, W2 = _to_dtype(W1, spec.dtype), _to_dtype(W2, spec.dtype)
    return dict(spec=spec, seed=seed, T=T, x=x, Wr=Wr, br=br, W1=W1, b1=b1, W2=W2, b2=b2,
                logits=logits, redrawn=redrawn)


def random_logits(T: int, E: int, seed: int, scale: float = 1.0) -> np.ndarray:
    """Plain N(0, scale^2) float32 router logits (routing-only tests)."""
    rng = np.random.default_rng([seed, 104729])
    return (rng.standard_normal((T, E), dtype=np.float32) * np.float32(scale)).astype(np.float32)
