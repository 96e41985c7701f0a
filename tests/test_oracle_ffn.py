"""Pins for the oracle's grouped SwiGLU FFN, combine and whole-layer forward (CPU only)."""
import math

import numpy as np
import pytest
import torch

from oracle import moe_ref as ref
from routing_grouped_expert_softmax_b200 import inputs as gen


def test_silu_matches_torch_library():
    h = np.linspace(-30, 30, 2001)
    np.testing.assert_allclose(ref.silu(h), torch.nn.functional.silu(torch.from_numpy(h)).numpy(),
                               rtol=1e-13, atol=1e-300)


def test_one_token_hand_worked_swiglu():
    # d = f = 1: x = 2, W_gate = 1, W_up = 3, W_down = 0.5
    # h = 2, u = 6, a = silu(2) * 6 = 12 / (1 + e^-2), y = 0.5 a
    h, u, a, y = ref.expert_swiglu(np.array([[2.0]]), np.array([[1.0]]), np.array([[3.0]]),
                                   np.array([[0.5]]))
    assert h[0, 0] == 2.0 and u[0, 0] == 6.0
    assert math.isclose(a[0, 0], 12.0 / (1.0 + math.exp(-2.0)), rel_tol=1e-15)
    assert math.isclose(y[0, 0], 6.0 / (1.0 + math.exp(-2.0)), rel_tol=1e-15)


def _dense_swiglu_torch(x, wg, wu, wd):
    """A dense SwiGLU FFN through torch library ops (silu and matmul)."""
    x, wg, wu, wd = (torch.from_numpy(np.asarray(a, np.float64)) for a in (x, wg, wu, wd))
    return ((torch.nn.functional.silu(x @ wg) * (x @ wu)) @ wd).numpy()


@pytest.mark.parametrize("E,k", [(4, 2), (8, 3), (5, 5)])
def test_identical_experts_equal_one_dense_ffn(E, k):
    inp = gen.make_layer_inputs(T=24, d=16, E=E, k=k, f=12, dtype="f32", seed=E, weight_std=0.3)
    wg = np.repeat(inp.w_gate[:1], E, axis=0)
    wu = np.repeat(inp.w_up[:1], E, axis=0)
    wd = np.repeat(inp.w_down[:1], E, axis=0)
    out = ref.layer_fwd(inp.x, inp.w_r, wg, wu, wd, k)
    dense = _dense_swiglu_torch(inp.x, wg[0], wu[0], wd[0])
    np.testing.assert_allclose(out["y"], dense, rtol=1e-12, atol=1e-12)


def test_single_expert_k1_is_dense_ffn():
    inp = gen.make_layer_inputs(T=9, d=8, E=1, k=1, f=6, dtype="f32", seed=1, weight_std=0.5)
    out = ref.layer_fwd(inp.x, inp.w_r, inp.w_gate, inp.w_up, inp.w_down, 1)
    np.testing.assert_allclose(out["gate"], 1.0)
    np.testing.assert_allclose(out["y"], _dense_swiglu_torch(inp.x, inp.w_gate[0], inp.w_up[0],
                                                             inp.w_down[0]), rtol=1e-12)


def test_layer_forward_per_token_against_direct_sum():
    # Y[t] = sum_j g_j FFN_{e_j}(x_t), evaluated token by token with torch ops
    inp = gen.make_layer_inputs(T=20, d=12, E=6, k=2, f=10, dtype="f32", seed=2, weight_std=0.3)
    out = ref.layer_fwd(inp.x, inp.w_r, inp.w_gate, inp.w_up, inp.w_down, 2)
    for t in range(20):
        acc = np.zeros(12)
        for j in range(2):
            e = out["idx"][t, j]
            acc += out["gate"][t, j] * _dense_swiglu_torch(inp.x[t:t + 1], inp.w_gate[e], inp.w_up[e],
                                                           inp.w_down[e])[0]
        np.testing.assert_allclose(out["y"][t], acc, rtol=1e-12, atol=1e-14)


def test_combine_identity_experts_and_k1():
    rng = np.random.default_rng(3)
    x = rng.standard_normal((15, 4))
    idx = gen.skewed_routing_idx(15, 6, 3, seed=3)
    z = rng.standard_normal((15, 6))
    _, g = ref.route_from_logits(z, 3)
    # idx from the generator, gates from the router: the combine only needs them paired
    _, _, sop, pos = ref.routing_metadata(idx, 6)
    xp = ref.permute(x, pos, 3)
    np.testing.assert_allclose(ref.combine(xp, sop, g), x, rtol=1e-13)   # identity experts
    idx1 = gen.skewed_routing_idx(15, 6, 1, seed=4)
    _, _, sop1, pos1 = ref.routing_metadata(idx1, 6)
    g1 = rng.random((15, 1))
    np.testing.assert_allclose(ref.combine(ref.permute(x, pos1, 1) * 3.0, sop1, g1), 3.0 * g1 * x,
                               rtol=1e-13)


def test_empty_experts_are_skipped():
    inp = gen.make_layer_inputs(T=8, d=8, E=4, k=1, f=8, dtype="f32", seed=5, weight_std=0.3)
    idx = np.zeros((8, 1), np.int32)          # everything to expert 0: experts 1..3 empty
    gate = np.ones((8, 1))
    out = ref.layer_fwd_routed(inp.x, idx, gate, inp.w_gate, inp.w_up, inp.w_down)
    assert out["counts"].tolist() == [8, 0, 0, 0]
    np.testing.assert_allclose(out["y"], _dense_swiglu_torch(inp.x, inp.w_gate[0], inp.w_up[0],
                                                             inp.w_down[0]), rtol=1e-12)
