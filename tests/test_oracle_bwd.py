"""Pins for the oracle's backward (CPU only): central finite differences in fp64,
torch autograd on an independently written dense layer, and closed forms."""
import numpy as np
import pytest
import torch

from oracle import moe_ref as ref
from routing_grouped_expert_softmax_b200 import inputs as gen

T, D, E, K, F = 5, 6, 4, 2, 5


def _inputs(seed):
    inp = gen.make_layer_inputs(T=T, d=D, E=E, k=K, f=F, dtype="f32", seed=seed, weight_std=0.5)
    # routing must not flip under the finite-difference step: demand clear top-k margins
    z = ref.router_logits(inp.x, inp.w_r)
    zs = -np.sort(-z, axis=1)
    assert np.min(zs[:, K - 1] - zs[:, K]) > 1e-3
    return inp


def _loss(x, w_r, wg, wu, wd, dy):
    return float(np.sum(ref.layer_fwd(x, w_r, wg, wu, wd, K)["y"] * dy))


@pytest.mark.parametrize("seed", [11, 12])
def test_layer_backward_matches_central_differences(seed):
    inp = _inputs(seed)
    params = dict(x=inp.x.astype(np.float64), w_r=inp.w_r.astype(np.float64),
                  wg=inp.w_gate.astype(np.float64), wu=inp.w_up.astype(np.float64),
                  wd=inp.w_down.astype(np.float64))
    dy = inp.dy.astype(np.float64)
    fwd = ref.layer_fwd(params["x"], params["w_r"], params["wg"], params["wu"], params["wd"], K)
    bwd = ref.layer_bwd(fwd, dy, params["x"], params["w_r"], params["wg"], params["wu"], params["wd"])
    analytic = dict(x=bwd["dx"], w_r=bwd["dw_r"], wg=bwd["dw_gate"], wu=bwd["dw_up"], wd=bwd["dw_down"])
    h = 1e-6
    for name, val in params.items():
        fd = np.zeros_like(val)
        it = np.nditer(val, flags=["multi_index"])
        for _ in it:
            i = it.multi_index
            old = val[i]
            val[i] = old + h
            lp = _loss(**params, dy=dy)
            val[i] = old - h
            lm = _loss(**params, dy=dy)
            val[i] = old
            fd[i] = (lp - lm) / (2 * h)
        scale = max(1.0, np.max(np.abs(fd)))
        assert np.max(np.abs(fd - analytic[name])) <= 1e-6 * scale, name


def test_gate_logit_grad_matches_differences_of_gates():
    z = gen.normal_logits(6, 7, seed=2).astype(np.float64)
    idx, g = ref.route_from_logits(z, 3)
    dg = np.random.default_rng(0).standard_normal(g.shape)
    dz = ref.gate_logit_grad(dg, g, idx, 7)
    np.testing.assert_allclose(dz.sum(axis=1), 0.0, atol=1e-15)      # sums to zero per token
    h = 1e-6
    for t in range(6):
        for e in range(7):
            zp, zm = z.copy(), z.copy()
            zp[t, e] += h
            zm[t, e] -= h
            ip, gp = ref.route_from_logits(zp, 3)
            im, gm = ref.route_from_logits(zm, 3)
            assert np.array_equal(ip, idx) and np.array_equal(im, idx)
            fd = np.sum((gp - gm) * dg) / (2 * h)
            assert abs(fd - dz[t, e]) < 1e-8


def _torch_moe_loss(x, w_r, wg, wu, wd, dy, k):
    """Independent dense formulation: every expert on every token, masked by the routing weights."""
    z = x @ w_r
    topv, topi = torch.topk(z, k, dim=1)             # library top-k (no ties in these inputs)
    gates = torch.softmax(topv, dim=1)
    weight = torch.zeros_like(z).scatter(1, topi, gates)      # [T, E]
    y = torch.zeros_like(x)
    for e in range(w_r.shape[1]):
        ye = (torch.nn.functional.silu(x @ wg[e]) * (x @ wu[e])) @ wd[e]
        y = y + weight[:, e:e + 1] * ye
    return (y * dy).sum()


def test_layer_backward_matches_torch_autograd():
    inp = gen.make_layer_inputs(T=32, d=16, E=8, k=3, f=12, dtype="f32", seed=21, weight_std=0.3)
    fwd = ref.layer_fwd(inp.x, inp.w_r, inp.w_gate, inp.w_up, inp.w_down, 3)
    bwd = ref.layer_bwd(fwd, inp.dy, inp.x, inp.w_r, inp.w_gate, inp.w_up, inp.w_down)
    ts = [torch.tensor(np.asarray(a, np.float64), requires_grad=True)
          for a in (inp.x, inp.w_r, inp.w_gate, inp.w_up, inp.w_down)]
    loss = _torch_moe_loss(*ts, torch.tensor(inp.dy, dtype=torch.float64), 3)
    loss.backward()
    names = ["dx", "dw_r", "dw_gate", "dw_up", "dw_down"]
    for n, t in zip(names, ts):
        np.testing.assert_allclose(bwd[n], t.grad.numpy(), rtol=1e-10, atol=1e-12, err_msg=n)


def test_identical_experts_gradients_sum_to_dense():
    inp = gen.make_layer_inputs(T=16, d=8, E=4, k=2, f=6, dtype="f32", seed=8, weight_std=0.4)
    wg = np.repeat(inp.w_gate[:1], 4, axis=0).astype(np.float64)
    wu = np.repeat(inp.w_up[:1], 4, axis=0).astype(np.float64)
    wd = np.repeat(inp.w_down[:1], 4, axis=0).astype(np.float64)
    fwd = ref.layer_fwd(inp.x, inp.w_r, wg, wu, wd, 2)
    bwd = ref.layer_bwd(fwd, inp.dy, inp.x, inp.w_r, wg, wu, wd)
    tx = torch.tensor(inp.x, dtype=torch.float64, requires_grad=True)
    tw = [torch.tensor(w[0], requires_grad=True) for w in (wg, wu, wd)]
    y = (torch.nn.functional.silu(tx @ tw[0]) * (tx @ tw[1])) @ tw[2]
    (y * torch.tensor(inp.dy, dtype=torch.float64)).sum().backward()
    np.testing.assert_allclose(bwd["dw_gate"].sum(0), tw[0].grad.numpy(), rtol=1e-11, atol=1e-13)
    np.testing.assert_allclose(bwd["dw_up"].sum(0), tw[1].grad.numpy(), rtol=1e-11, atol=1e-13)
    np.testing.assert_allclose(bwd["dw_down"].sum(0), tw[2].grad.numpy(), rtol=1e-11, atol=1e-13)
    np.testing.assert_allclose(bwd["dx"], tx.grad.numpy(), rtol=1e-11, atol=1e-13)
    np.testing.assert_allclose(bwd["dz"], 0.0, atol=1e-13)    # equal experts: router gets no gradient


def test_swiglu_bwd_special_values():
    # silu'(0) = 1/2 and silu(0) = 0: dh = da * u / 2, du = 0 at h = 0
    dh, du = ref.swiglu_bwd(np.array([2.0]), np.array([0.0]), np.array([3.0]))
    assert dh[0] == 3.0 and du[0] == 0.0


def test_unpermute_sum_and_combine_bwd_are_adjoints():
    # <combine(y), dY> == <y, dy_perm> and <unpermute_sum(v), w> == <v, permute(w)>
    rng = np.random.default_rng(4)
    idx = gen.skewed_routing_idx(12, 5, 2, seed=4)
    _, _, sop, pos = ref.routing_metadata(idx, 5)
    g = rng.random((12, 2))
    y = rng.standard_normal((24, 3))
    dY = rng.standard_normal((12, 3))
    dy_perm, dgate = ref.combine_bwd(dY, y, sop, g)
    assert np.isclose(np.sum(ref.combine(y, sop, g) * dY), np.sum(y * dy_perm), rtol=1e-13)
    np.testing.assert_allclose(np.sum(g * dgate), np.sum(y * dy_perm), rtol=1e-13)
    v = rng.standard_normal((24, 3))
    w = rng.standard_normal((12, 3))
    assert np.isclose(np.sum(ref.unpermute_sum(v, sop, 12, 2) * w), np.sum(v * ref.permute(w, pos, 2)),
                      rtol=1e-13)
