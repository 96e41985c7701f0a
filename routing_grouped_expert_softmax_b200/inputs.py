"""Seeded synthetic inputs for the MoE layer step.

This module only draws random numbers and rounds them to the storage type the
library receives.  It holds none of the layer's arithmetic, so both the CUDA
path (through the tests and the benchmark) and the CPU oracle can be fed from
it without sharing any of the method's code.

Workload recipe (the pages publish no data and no weights; these stand in for
their sweep of 8 -> 128 experts, 4 active per token, random routing for system
benchmarks):

* ``numpy.random.default_rng(seed)``; draws in fp32 in the order
  x, W_r, W_gate, W_up, W_down, dY;
* x ~ N(0, 1); every weight ~ N(0, 0.02); dY ~ N(0, 1);
* for bf16 workloads every tensor is rounded to bf16 (round to nearest even)
  and both sides receive exactly the rounded values;
* skewed routing adds b_e = 1.5 * ln(1 / (e + 1)) to expert e's logit;
* uniform random routing draws, per token, k distinct experts uniformly
  without replacement, each with gate 1/k.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np


def bf16_bits(a: np.ndarray) -> np.ndarray:
    """Round fp32 values to bf16 (nearest, ties to even); return the raw uint16 bits."""
    u = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32).astype(np.uint64)
    u = u + 0x7FFF + ((u >> 16) & 1)
    return (u >> 16).astype(np.uint16)


def bf16_value(bits: np.ndarray) -> np.ndarray:
    """The fp32 value of raw bf16 bits (exact)."""
    return (bits.astype(np.uint32) << 16).view(np.float32)


def bf16_round(a: np.ndarray) -> np.ndarray:
    """fp32 values rounded to the bf16 grid (returned as fp32, exactly representable)."""
    return bf16_value(bf16_bits(a))


@dataclass
class LayerInputs:
    """One layer's inputs, as fp32 arrays holding exactly the values the GPU receives.

    For ``dtype == "bf16"`` every array is already on the bf16 grid.
    Shapes: x [T,d], w_r [d,E], w_gate/w_up [E,d,f], w_down [E,f,d], dy [T,d],
    bias [E] or None.
    """
    T: int
    d: int
    E: int
    k: int
    f: int
    dtype: str
    x: np.ndarray
    w_r: np.ndarray
    w_gate: np.ndarray
    w_up: np.ndarray
    w_down: np.ndarray
    dy: np.ndarray | None = None
    bias: np.ndarray | None = None
    extra: dict = field(default_factory=dict)


def zipf_bias(E: int) -> np.ndarray:
    """Per-expert additive logit bias b_e = 1.5 * ln(1/(e+1)): expert 0 is the most popular."""
    return (1.5 * np.log(1.0 / (np.arange(E, dtype=np.float64) + 1.0))).astype(np.float32)


def make_layer_inputs(T: int, d: int, E: int, k: int, f: int, dtype: str = "bf16",
                      seed: int = 0, skew: bool = False, with_grad: bool = True,
                      weight_std: float = 0.02) -> LayerInputs:
    """Draw a full set of layer inputs in the fixed order x, W_r, W_gate, W_up, W_down, dY."""
    if dtype not in ("bf16", "f32"):
        raise ValueError(dtype)
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((T, d), dtype=np.float32)
    w_r = (weight_std * rng.standard_normal((d, E), dtype=np.float32)).astype(np.float32)
    w_gate = (weight_std * rng.standard_normal((E, d, f), dtype=np.float32)).astype(np.float32)
    w_up = (weight_std * rng.standard_normal((E, d, f), dtype=np.float32)).astype(np.float32)
    w_down = (weight_std * rng.standard_normal((E, f, d), dtype=np.float32)).astype(np.float32)
    dy = rng.standard_normal((T, d), dtype=np.float32) if with_grad else None
    if dtype == "bf16":
        x, w_r, w_gate, w_up, w_down = (bf16_round(a) for a in (x, w_r, w_gate, w_up, w_down))
        if dy is not None:
            dy = bf16_round(dy)
    bias = zipf_bias(E) if skew else None
    return LayerInputs(T, d, E, k, f, dtype, x, w_r, w_gate, w_up, w_down, dy, bias)


def make_shared_expert(d: int, f: int, dtype: str = "bf16", seed: int = 0,
                       weight_std: float = 0.02):
    """Shared-expert weights W_gate [d,f], W_up [d,f], W_down [f,d], drawn in that order from
    N(0, weight_std^2) with their own seed; rounded to bf16 for bf16 workloads."""
    rng = np.random.default_rng(seed)
    ws = [(weight_std * rng.standard_normal(shape, dtype=np.float32)).astype(np.float32)
          for shape in ((d, f), (d, f), (f, d))]
    if dtype == "bf16":
        ws = [bf16_round(a) for a in ws]
    return tuple(ws)


def uniform_random_routing(T: int, E: int, k: int, seed: int = 0):
    """Per token, k distinct experts drawn uniformly without replacement; gates 1/k.

    Returns (topk_idx int32 [T,k], topk_gate float32 [T,k]).
    """
    rng = np.random.default_rng(seed)
    keys = rng.random((T, E))
    idx = np.argsort(keys, axis=1, kind="stable")[:, :k].astype(np.int32)
    gate = np.full((T, k), 1.0 / k, dtype=np.float32)
    return idx, gate


def tied_logits(T: int, E: int, levels: int = 4, seed: int = 0) -> np.ndarray:
    """fp32 logits drawn from a handful of values, so that ties are frequent."""
    rng = np.random.default_rng(seed)
    return (rng.integers(0, levels, size=(T, E)).astype(np.float32) * 0.25 - 0.5)


def normal_logits(T: int, E: int, seed: int = 0, std: float = 1.0) -> np.ndarray:
    """fp32 logits ~ N(0, std^2)."""
    rng = np.random.default_rng(seed)
    return (std * rng.standard_normal((T, E), dtype=np.float32)).astype(np.float32)


def skewed_routing_idx(T: int, E: int, k: int, seed: int = 0, s: float = 1.2) -> np.ndarray:
    """k distinct experts per token drawn with Zipf-like popularity p_e ~ (e+1)^-s.

    Used to exercise very uneven expert loads (hot and empty experts) directly
    at the metadata and grouped-GEMM entry points.
    """
    rng = np.random.default_rng(seed)
    w = (np.arange(E) + 1.0) ** (-s)
    # Gumbel-top-k draws k distinct experts with probabilities proportional to w.
    g = np.log(w)[None, :] - np.log(-np.log(rng.random((T, E))))
    return np.argsort(-g, axis=1, kind="stable")[:, :k].astype(np.int32)
