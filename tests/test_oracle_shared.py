"""Pins for the oracle's shared expert (CPU only).

Reading (bigchange.ai, "Olmo-core 3 открывает стек обучения MoE от Ai2 ...", section "Что
инженер может попробовать на практике": the production rows use top-four routing and one
shared expert): a SwiGLU of the routed experts' shape through which every token passes,
added to the routed experts' gate-weighted sum with weight 1.  Checked against an
independently written dense torch layer (forward and autograd), a closed form for identical
experts, and central differences."""
import numpy as np
import pytest
import torch

from oracle import moe_ref as ref
from routing_grouped_expert_softmax_b200 import inputs as gen


def _shared(d, f, seed, std=0.3):
    rng = np.random.default_rng(seed)
    return (std * rng.standard_normal((d, f)), std * rng.standard_normal((d, f)),
            std * rng.standard_normal((f, d)))


def _dense_swiglu_torch(x, sg, su, sd):
    return (torch.nn.functional.silu(x @ sg) * (x @ su)) @ sd


def test_shared_expert_adds_a_dense_swiglu():
    inp = gen.make_layer_inputs(T=24, d=16, E=6, k=2, f=10, dtype="f32", seed=3, weight_std=0.3)
    sh = _shared(16, 10, 4)
    with_s = ref.layer_fwd(inp.x, inp.w_r, inp.w_gate, inp.w_up, inp.w_down, 2, shared=sh)
    without = ref.layer_fwd(inp.x, inp.w_r, inp.w_gate, inp.w_up, inp.w_down, 2)
    dense = _dense_swiglu_torch(*(torch.tensor(np.asarray(a, np.float64)) for a in (inp.x, *sh))).numpy()
    np.testing.assert_allclose(with_s["y"] - without["y"], dense, rtol=1e-12, atol=1e-12)
    # routing and the routed experts are untouched by the shared expert
    assert np.array_equal(with_s["idx"], without["idx"])
    np.testing.assert_array_equal(with_s["y_perm"], without["y_perm"])


def test_identical_experts_and_shared_expert_give_twice_the_dense_ffn():
    # every routed expert and the shared expert carry the same weights: the gates sum to 1,
    # so y = (1 + 1) * SwiGLU(x) whatever the routing
    inp = gen.make_layer_inputs(T=20, d=8, E=5, k=3, f=6, dtype="f32", seed=9, weight_std=0.4)
    sg, su, sd = (np.asarray(a[0], np.float64) for a in (inp.w_gate, inp.w_up, inp.w_down))
    wg, wu, wd = (np.repeat(a[None], 5, axis=0) for a in (sg, su, sd))
    out = ref.layer_fwd(inp.x, inp.w_r, wg, wu, wd, 3, shared=(sg, su, sd))
    dense = _dense_swiglu_torch(*(torch.tensor(np.asarray(a, np.float64)) for a in (inp.x, sg, su, sd))).numpy()
    np.testing.assert_allclose(out["y"], 2.0 * dense, rtol=1e-12, atol=1e-12)


def _torch_loss(x, w_r, wg, wu, wd, sg, su, sd, dy, k):
    """Independent dense formulation: every expert on every token, masked by the routing
    weights, plus the shared expert with weight 1."""
    z = x @ w_r
    topv, topi = torch.topk(z, k, dim=1)
    gates = torch.softmax(topv, dim=1)
    weight = torch.zeros_like(z).scatter(1, topi, gates)
    y = _dense_swiglu_torch(x, sg, su, sd)
    for e in range(w_r.shape[1]):
        y = y + weight[:, e:e + 1] * _dense_swiglu_torch(x, wg[e], wu[e], wd[e])
    return (y * dy).sum()


def test_layer_backward_with_shared_expert_matches_torch_autograd():
    inp = gen.make_layer_inputs(T=32, d=16, E=8, k=3, f=12, dtype="f32", seed=21, weight_std=0.3)
    sh = _shared(16, 12, 5)
    fwd = ref.layer_fwd(inp.x, inp.w_r, inp.w_gate, inp.w_up, inp.w_down, 3, shared=sh)
    bwd = ref.layer_bwd(fwd, inp.dy, inp.x, inp.w_r, inp.w_gate, inp.w_up, inp.w_down, shared=sh)
    ts = [torch.tensor(np.asarray(a, np.float64), requires_grad=True)
          for a in (inp.x, inp.w_r, inp.w_gate, inp.w_up, inp.w_down, *sh)]
    loss = _torch_loss(*ts, torch.tensor(inp.dy, dtype=torch.float64), 3)
    loss.backward()
    names = ["dx", "dw_r", "dw_gate", "dw_up", "dw_down", "dw_shared_gate", "dw_shared_up", "dw_shared_down"]
    for n, t in zip(names, ts):
        np.testing.assert_allclose(bwd[n], t.grad.numpy(), rtol=1e-10, atol=1e-12, err_msg=n)


@pytest.mark.parametrize("seed", [31, 32])
def test_shared_expert_backward_matches_central_differences(seed):
    T, d, E, k, f = 4, 5, 3, 2, 4
    inp = gen.make_layer_inputs(T=T, d=d, E=E, k=k, f=f, dtype="f32", seed=seed, weight_std=0.5)
    z = ref.router_logits(inp.x, inp.w_r)
    zs = -np.sort(-z, axis=1)
    assert np.min(zs[:, k - 1] - zs[:, k]) > 1e-3        # routing stays put under the step
    sh = [np.asarray(a, np.float64) for a in _shared(d, f, seed + 100, std=0.5)]
    x = inp.x.astype(np.float64)
    dy = inp.dy.astype(np.float64)
    weights = [np.asarray(a, np.float64) for a in (inp.w_r, inp.w_gate, inp.w_up, inp.w_down)]

    def loss():
        return float(np.sum(ref.layer_fwd(x, *weights, k, shared=tuple(sh))["y"] * dy))

    fwd = ref.layer_fwd(x, *weights, k, shared=tuple(sh))
    bwd = ref.layer_bwd(fwd, dy, x, *weights, shared=tuple(sh))
    params = dict(dx=x, dw_shared_gate=sh[0], dw_shared_up=sh[1], dw_shared_down=sh[2])
    h = 1e-6
    for name, val in params.items():
        fd = np.zeros_like(val)
        it = np.nditer(val, flags=["multi_index"])
        for _ in it:
            i = it.multi_index
            old = val[i]
            val[i] = old + h
            lp = loss()
            val[i] = old - h
            lm = loss()
            val[i] = old
            fd[i] = (lp - lm) / (2 * h)
        scale = max(1.0, np.max(np.abs(fd)))
        assert np.max(np.abs(fd - bwd[name])) <= 1e-6 * scale, name


def test_routed_backward_with_shared_expert_adds_its_terms():
    inp = gen.make_layer_inputs(T=16, d=8, E=4, k=2, f=6, dtype="f32", seed=12, weight_std=0.3)
    idx, gate = gen.uniform_random_routing(16, 4, 2, seed=1)
    sh = _shared(8, 6, 7)
    fwd = ref.layer_fwd_routed(inp.x, idx, gate, inp.w_gate, inp.w_up, inp.w_down, shared=sh)
    base = ref.layer_fwd_routed(inp.x, idx, gate, inp.w_gate, inp.w_up, inp.w_down)
    b = ref.layer_bwd_routed(fwd, inp.dy, inp.w_gate, inp.w_up, inp.w_down, x=inp.x, shared=sh)
    b0 = ref.layer_bwd_routed(base, inp.dy, inp.w_gate, inp.w_up, inp.w_down)
    ts = [torch.tensor(np.asarray(a, np.float64), requires_grad=True) for a in (inp.x, *sh)]
    (_dense_swiglu_torch(*ts) * torch.tensor(inp.dy, dtype=torch.float64)).sum().backward()
    np.testing.assert_allclose(b["dx"] - b0["dx"], ts[0].grad.numpy(), rtol=1e-10, atol=1e-12)
    for n, t in zip(["dw_shared_gate", "dw_shared_up", "dw_shared_down"], ts[1:]):
        np.testing.assert_allclose(b[n], t.grad.numpy(), rtol=1e-10, atol=1e-12, err_msg=n)
    np.testing.assert_array_equal(b["dw_gate"], b0["dw_gate"])
