"""Pins for the oracle's MXFP8 layer step, its fixed-routing backward and the grouped
token-axis quantiser (CPU only).

  * layer_fwd_mx / layer_bwd_mx are the bf16 layer's steps with the MXFP8 GEMMs in place:
    with the quantiser and the bf16 rounding made the identity they must give exactly the
    float64 layer, which finite differences and torch autograd pin
    (tests/test_oracle_bwd.py); a spy checks that the five tensors the layer keeps in
    bf16 reach the GEMMs on the bf16 grid; on MX-grid inputs the first GEMM is exact;
    the whole step stays within the quantisation error of the exact layer.
  * layer_bwd_routed against torch autograd on an independently written dense layer with
    the routing held fixed.
  * mx_quantize_grouped_rows against an element-by-element brute force that finds each
    element's group and 32-row block and rounds with ml_dtypes' float8_e4m3fn.
"""
import math

import ml_dtypes
import numpy as np
import pytest
import torch

from oracle import moe_ref as ref
from routing_grouped_expert_softmax_b200 import inputs as gen


def _identity_quantiser(monkeypatch):
    monkeypatch.setattr(ref, "mx_quantize", lambda v, axis=-1: (None, None, np.asarray(v, np.float64)))
    monkeypatch.setattr(ref, "bf16_rne", lambda v: np.asarray(v, np.float64))


def _close(a, b, name):
    scale = max(1.0, float(np.max(np.abs(b))))
    assert np.max(np.abs(np.asarray(a) - np.asarray(b))) <= 1e-12 * scale, name


@pytest.mark.parametrize("routed,shared", [(False, False), (True, False), (False, True)])
def test_mx_layer_is_the_exact_layer_when_quantisation_is_the_identity(monkeypatch, routed, shared):
    T, d, E, k, f = 40, 64, 5, 2, 32
    inp = gen.make_layer_inputs(T, d, E, k, f, dtype="f32", seed=31, weight_std=0.3, skew=True)
    sh = gen.make_shared_expert(d, f, dtype="f32", seed=32, weight_std=0.3) if shared else None
    routing = gen.uniform_random_routing(T, E, k, seed=33) if routed else None
    if routed:
        fwd = ref.layer_fwd_routed(inp.x, *routing, inp.w_gate, inp.w_up, inp.w_down, shared=sh)
        bwd = ref.layer_bwd_routed(fwd, inp.dy, inp.w_gate, inp.w_up, inp.w_down, x=inp.x, shared=sh)
    else:
        fwd = ref.layer_fwd(inp.x, inp.w_r, inp.w_gate, inp.w_up, inp.w_down, k, inp.bias, shared=sh)
        bwd = ref.layer_bwd(fwd, inp.dy, inp.x, inp.w_r, inp.w_gate, inp.w_up, inp.w_down, shared=sh)
    _identity_quantiser(monkeypatch)
    mf = ref.layer_fwd_mx(inp.x, inp.w_r, inp.w_gate, inp.w_up, inp.w_down, k, inp.bias, routing=routing,
                          shared=sh)
    mb = ref.layer_bwd_mx(mf, inp.dy, inp.x, inp.w_r, inp.w_gate, inp.w_up, inp.w_down, router=not routed,
                          shared=sh)
    for n in ("idx", "offsets", "slot_of_pair"):
        assert np.array_equal(mf[n], fwd[n]), n
    for n in ("h", "u", "a", "y_perm", "y"):
        _close(mf[n], fwd[n], n)
    names = ["dy_perm", "dgate", "dh", "du", "dx_perm", "dx", "dw_gate", "dw_up", "dw_down"]
    names += [] if routed else ["dw_r", "dz"]
    names += ["dw_shared_gate", "dw_shared_up", "dw_shared_down", "shared_dx"] if shared else []
    for n in names:
        _close(mb[n], bwd[n], n)


def test_mx_layer_keeps_its_stored_tensors_in_bf16(monkeypatch):
    T, d, E, k, f = 64, 64, 4, 2, 32
    inp = gen.make_layer_inputs(T, d, E, k, f, dtype="bf16", seed=41)
    seen = {}
    real_bwd = ref.grouped_swiglu_bwd_mx

    def spy(dy_perm, x_perm, h, u, a, *rest):
        seen.update(dy_perm=dy_perm, x_perm=x_perm, h=h, u=u, a=a)
        return real_bwd(dy_perm, x_perm, h, u, a, *rest)

    monkeypatch.setattr(ref, "grouped_swiglu_bwd_mx", spy)
    fwd = ref.layer_fwd_mx(inp.x, inp.w_r, inp.w_gate, inp.w_up, inp.w_down, k)
    ref.layer_bwd_mx(fwd, inp.dy, inp.x, inp.w_r, inp.w_gate, inp.w_up, inp.w_down)
    on_bf16_grid = lambda v: np.array_equal(gen.bf16_round(np.asarray(v, np.float32)).astype(np.float64), v)
    for n in ("dy_perm", "h", "u", "a"):
        assert on_bf16_grid(seen[n]), n
    for n in ("h", "u", "a"):        # the forward's own values are unrounded float64
        assert not on_bf16_grid(fwd[n]), n
    # x_perm is a bit copy of the (bf16) layer input
    assert np.array_equal(seen["x_perm"], inp.x[fwd["pair_of_slot"] // k])


def _mx_grid(shape, axis, rng):
    """Values on the E4M3 grid with a 448 in every 32-block along `axis`: exact under MX."""
    g = ref.e4m3_grid()
    v = rng.choice(g, size=shape) * rng.choice([-1.0, 1.0], size=shape)
    v = np.moveaxis(v, axis, -1).copy()
    v[..., ::32] = 448.0
    return np.moveaxis(v, -1, axis) * 2.0 ** -12


def test_mx_layer_first_gemm_is_exact_on_grid_inputs():
    rng = np.random.default_rng(7)
    T, d, E, k, f = 48, 64, 4, 2, 32
    inp = gen.make_layer_inputs(T, d, E, k, f, dtype="f32", seed=7)
    x = _mx_grid((T, d), 1, rng)
    wg, wu = _mx_grid((E, d, f), 1, rng), _mx_grid((E, d, f), 1, rng)
    routing = gen.uniform_random_routing(T, E, k, seed=7)
    mf = ref.layer_fwd_mx(x, inp.w_r, wg, wu, inp.w_down, k, routing=routing)
    ef = ref.layer_fwd_routed(x, *routing, wg, wu, inp.w_down)
    np.testing.assert_array_equal(mf["h"], ef["h"])
    np.testing.assert_array_equal(mf["u"], ef["u"])


def test_mx_layer_within_quantisation_error_of_the_exact_layer():
    T, d, E, k, f = 128, 128, 8, 2, 64
    inp = gen.make_layer_inputs(T, d, E, k, f, dtype="bf16", seed=51)
    fwd = ref.layer_fwd(inp.x, inp.w_r, inp.w_gate, inp.w_up, inp.w_down, k)
    bwd = ref.layer_bwd(fwd, inp.dy, inp.x, inp.w_r, inp.w_gate, inp.w_up, inp.w_down)
    mf = ref.layer_fwd_mx(inp.x, inp.w_r, inp.w_gate, inp.w_up, inp.w_down, k)
    mb = ref.layer_bwd_mx(mf, inp.dy, inp.x, inp.w_r, inp.w_gate, inp.w_up, inp.w_down)
    rel = lambda a, b: float(np.max(np.abs(a - b)) / np.max(np.abs(b)))
    # every quantised operand carries at most 2^-4 relative rounding (3 mantissa bits, plus the
    # saturation of a block's largest values to 448 X, at most 1/8 below them): a product of two
    # quantised operands is off by at most ~2^-2 of its magnitude, and two GEMMs in a row at most
    # ~1/2 of the sum of |terms|.  Per tensor the error must be non-zero (quantisation happened)
    # and well inside that bound (random signs average it down).
    for got, want, n in ((mf["y"], fwd["y"], "y"), (mb["dx"], bwd["dx"], "dx"),
                         (mb["dw_gate"], bwd["dw_gate"], "dw_gate"), (mb["dw_down"], bwd["dw_down"], "dw_down"),
                         (mb["dw_r"], bwd["dw_r"], "dw_r")):
        e = rel(got, want)
        assert 1e-4 < e < 0.25, (n, e)


def _dense_routed_torch(x, wg, wu, wd, idx, gate):
    """Independent dense formulation with fixed routing: every expert on every token,
    weighted by a [T, E] matrix that holds the given gates at the given experts."""
    T, E = x.shape[0], wg.shape[0]
    weight = torch.zeros(T, E, dtype=x.dtype)
    weight[torch.arange(T)[:, None], torch.as_tensor(idx, dtype=torch.long)] = torch.as_tensor(gate, dtype=x.dtype)
    y = torch.zeros(T, wd.shape[2], dtype=x.dtype)
    for e in range(E):
        y = y + weight[:, e:e + 1] * ((torch.nn.functional.silu(x @ wg[e]) * (x @ wu[e])) @ wd[e])
    return y


@pytest.mark.parametrize("gates", ["uniform", "random"])
def test_layer_bwd_routed_matches_torch_autograd(gates):
    T, d, E, k, f = 24, 12, 6, 3, 10
    inp = gen.make_layer_inputs(T, d, E, k, f, dtype="f32", seed=61, weight_std=0.3)
    idx, gate = gen.uniform_random_routing(T, E, k, seed=62)
    if gates == "random":
        gate = np.random.default_rng(63).random((T, k)) + 0.1
    fwd = ref.layer_fwd_routed(inp.x, idx, gate, inp.w_gate, inp.w_up, inp.w_down)
    bwd = ref.layer_bwd_routed(fwd, inp.dy, inp.w_gate, inp.w_up, inp.w_down)
    ts = [torch.tensor(np.asarray(a, np.float64), requires_grad=True)
          for a in (inp.x, inp.w_gate, inp.w_up, inp.w_down)]
    y = _dense_routed_torch(*ts, idx, gate)
    np.testing.assert_allclose(fwd["y"], y.detach().numpy(), rtol=1e-12, atol=1e-14)
    (y * torch.tensor(inp.dy, dtype=torch.float64)).sum().backward()
    for n, t in zip(["dx", "dw_gate", "dw_up", "dw_down"], ts):
        np.testing.assert_allclose(bwd[n], t.grad.numpy(), rtol=1e-10, atol=1e-12, err_msg=n)
    # an expert nobody routes to gets exactly zero weight gradients
    unused = np.setdiff1d(np.arange(E), idx.ravel())
    for e in unused:
        assert np.all(bwd["dw_gate"][e] == 0) and np.all(bwd["dw_down"][e] == 0)


def _brute_grouped_rows(v, offsets):
    """Element by element: the element's group [lo, hi), its 32-row block inside the group
    (rows past hi count as zeros), the block's amax in that column, the OCP scale
    2^(floor(log2 amax) - 8), and ml_dtypes' float8_e4m3fn rounding of v / X (|v / X| capped
    at 448)."""
    out = np.zeros_like(v)
    for e in range(len(offsets) - 1):
        lo, hi = int(offsets[e]), int(offsets[e + 1])
        for r in range(lo, hi):
            b0 = lo + (r - lo) // 32 * 32
            for c in range(v.shape[1]):
                amax = max(abs(float(v[i, c])) for i in range(b0, min(b0 + 32, hi)))
                if amax == 0:
                    out[r, c] = 0.0
                    continue
                X = 2.0 ** (math.frexp(amax)[1] - 1 - 8)
                q = np.clip(np.float32(v[r, c] / X), -448.0, 448.0).astype(ml_dtypes.float8_e4m3fn)
                out[r, c] = float(q) * X
    return out


def test_grouped_rows_quantiser_against_brute_force():
    rng = np.random.default_rng(71)
    offsets = np.array([0, 0, 33, 103, 108, 108, 140])   # empty groups, tails of 1, 6, 5 and 0 rows
    v = rng.standard_normal((140, 3)) * np.exp(rng.standard_normal((140, 1)) * 2)
    v[40:72, 1] = 0.0                                     # an all-zero block
    got = ref.mx_quantize_grouped_rows(v, offsets)
    np.testing.assert_array_equal(got, _brute_grouped_rows(v, offsets))
