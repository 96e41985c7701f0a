"""Parity at the benchmark's full sizes, in the launch configuration bench.py times
(moe_layer_fwd + moe_layer_bwd on one stream):

  * E=8:   T=8192, d=2048, k=4, ffn=1024 (near-uniform load)
  * E=128: T=8192, d=2048, k=4, ffn=1024
  * E=128: T=16384 with the Zipf-like logit bias, and with uniform random routing

The whole-tensor oracle is too slow here, so the checks are (a) properties that hold at
any size (routing and metadata invariants, exact permute), (b) oracle values computed one
token at a time (y and dx of sampled tokens) or one expert at a time (the weight
gradients of sampled experts), each from the oracle's own routing of those tokens.
"""
import numpy as np
import pytest

import routing_grouped_expert_softmax_b200 as moe
from oracle import moe_ref as ref
from routing_grouped_expert_softmax_b200 import inputs as gen
from tests.gpu_util import dev, dev_f32, host, rel_err

pytestmark = pytest.mark.gpu

TOL = 2e-2
TOL_COMBINE = 1e-2

FULL_SIZE_CASES = {
    "e8": dict(T=8192, d=2048, E=8, k=4, f=1024, skew=False, routing="router"),
    "e128": dict(T=8192, d=2048, E=128, k=4, f=1024, skew=False, routing="router"),
    "e128_t16k_skew": dict(T=16384, d=2048, E=128, k=4, f=1024, skew=True, routing="router"),
    "e128_t16k_uniform": dict(T=16384, d=2048, E=128, k=4, f=1024, skew=False, routing="uniform"),
    "e128_t16k_mxfp8": dict(T=16384, d=2048, E=128, k=4, f=1024, skew=False, routing="router", prec="mxfp8"),
}
TOL_MX = 6e-2


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    import torch
    assert torch.cuda.is_available()
    from routing_grouped_expert_softmax_b200 import build
    build.build()


def clear_tokens(z, delta, k):
    """Tokens whose top-(k+1) logits are pairwise separated by more than 2*delta."""
    zs = np.sort(z, axis=1)[:, ::-1][:, :k + 1]
    gaps = -np.diff(zs, axis=1)
    return np.all(gaps > 2 * delta[:, None], axis=1)


class _MxWeights:
    """The oracle's MXFP8 copies of one expert's weights, along each GEMM's own K."""

    def __init__(self, inp):
        self.inp, self.cache = inp, {}

    def __call__(self, e):
        if e not in self.cache:
            q = lambda w, ax: ref.mx_quantize(np.asarray(w, np.float64), axis=ax)[2]
            i = self.inp
            self.cache[e] = dict(g=q(i.w_gate[e], 0), u=q(i.w_up[e], 0), d=q(i.w_down[e], 0),
                                 dT=q(i.w_down[e], 1), gT=q(i.w_gate[e], 1), uT=q(i.w_up[e], 1))
        return self.cache[e]


def _token_oracle(inp, t, idx_t, g_t, router, mx=None):
    """Oracle y[t] and dx[t] of one token from its routing (experts idx_t, gates g_t).
    With mx, every GEMM operand is MXFP8-quantised along its own K, as the MXFP8 layer
    does (row-wise blocks of one token's vectors, and the bf16 tensors it stores)."""
    x = inp.x[t:t + 1].astype(np.float64)
    dY = inp.dy[t].astype(np.float64)
    y = np.zeros(inp.d)
    dx = np.zeros(inp.d)
    dg = np.zeros(len(idx_t))
    q = lambda v: ref.mx_quantize(v, axis=1)[2]
    b = ref.bf16_rne
    for j, e in enumerate(idx_t):
        if mx is None:
            h, u, a, ye = ref.expert_swiglu(x, inp.w_gate[e], inp.w_up[e], inp.w_down[e])
            da = (g_t[j] * dY)[None, :] @ inp.w_down[e].astype(np.float64).T
            dh, du = ref.swiglu_bwd(da, h, u)
            dx += (dh @ inp.w_gate[e].astype(np.float64).T + du @ inp.w_up[e].astype(np.float64).T)[0]
        else:
            w = mx(e)
            xq = q(x)
            h, u = xq @ w["g"], xq @ w["u"]
            a = ref.silu(h) * u
            ye = q(b(a)) @ w["d"]
            da = q(b(g_t[j] * dY)[None, :]) @ w["dT"].T
            dh, du = ref.swiglu_bwd(da, b(h), b(u))
            dhu = q(b(np.concatenate([dh, du], axis=1)))
            f = inp.f
            dx += (dhu[:, :f] @ w["gT"].T + dhu[:, f:] @ w["uT"].T)[0]
        y += g_t[j] * ye[0]
        dg[j] = dY @ ye[0]
    if router:
        dz = ref.gate_logit_grad(dg[None, :], np.asarray(g_t)[None, :], np.asarray(idx_t)[None, :], inp.E)
        dx += (dz @ inp.w_r.astype(np.float64).T)[0]
    return y, dx


def _expert_oracle(inp, e, idx, gate, mx=None):
    """Oracle weight gradients of expert e from the routing of every token (with mx: the
    MXFP8 layer's operands, the token-axis operands blocked 32 rows at a time from the
    expert's first row)."""
    pairs = np.nonzero(idx.ravel() == e)[0]           # pair order = the stable slot order
    toks = pairs // inp.k
    g = gate.ravel()[pairs].astype(np.float64)
    X = inp.x[toks].astype(np.float64)
    if mx is None:
        h, u, a, _ = ref.expert_swiglu(X, inp.w_gate[e], inp.w_up[e], inp.w_down[e])
        dy = g[:, None] * inp.dy[toks].astype(np.float64)
        da = dy @ inp.w_down[e].astype(np.float64).T
        dh, du = ref.swiglu_bwd(da, h, u)
        return X.T @ dh, X.T @ du, a.T @ dy
    w, b, f = mx(e), ref.bf16_rne, inp.f
    q = lambda v: ref.mx_quantize(v, axis=1)[2]
    qt = lambda v: ref.mx_quantize_grouped_rows(v, np.array([0, v.shape[0]]))
    xq = q(X)
    h, u = xq @ w["g"], xq @ w["u"]
    a = b(ref.silu(h) * u)
    dy = b(g[:, None] * inp.dy[toks].astype(np.float64))
    da = q(dy) @ w["dT"].T
    dh, du = ref.swiglu_bwd(da, b(h), b(u))
    dhu = b(np.concatenate([dh, du], axis=1))
    dwgu = qt(X).T @ qt(dhu)
    return dwgu[:, :f], dwgu[:, f:], qt(a).T @ qt(dy)


@pytest.mark.parametrize("name", list(FULL_SIZE_CASES))
def test_fullsize(name):
    import torch
    c = FULL_SIZE_CASES[name]
    T, d, E, k, f = c["T"], c["d"], c["E"], c["k"], c["f"]
    inp = gen.make_layer_inputs(T, d, E, k, f, dtype="bf16", seed=0, skew=c["skew"])
    prec = c.get("prec", "native")
    cfg = moe.config(T, d, E, k, f, dtype="bf16", prec=prec)
    mx = _MxWeights(inp) if prec == "mxfp8" else None
    tol, tol_c = (TOL_MX, TOL_MX) if mx else (TOL, TOL_COMBINE)
    ws = moe.alloc_workspace(cfg)
    saved = moe.alloc_saved(cfg)
    router = c["routing"] == "router"
    grads = moe.alloc_grads(cfg, router=router)
    w = [dev(a, "bf16") for a in (inp.w_r, inp.w_gate, inp.w_up, inp.w_down)]
    bias = dev_f32(inp.bias) if inp.bias is not None else None
    wts = moe.layer_weights(w[0], bias, w[1], w[2], w[3])
    x = dev(inp.x, "bf16")
    y = torch.empty(T, d, dtype=torch.bfloat16, device="cuda")
    if router:
        moe.moe_layer_fwd(cfg, wts, x, y, saved, ws)
    else:
        ridx, rgate = gen.uniform_random_routing(T, E, k, seed=0)
        saved["topk_idx"].copy_(torch.from_numpy(ridx))
        saved["topk_gate"].copy_(torch.from_numpy(rgate))
        moe.moe_layer_fwd_routed(cfg, wts, x, y, saved, ws)
    moe.moe_layer_bwd(cfg, wts, x, dev(inp.dy, "bf16"), saved, grads, ws)
    assert moe.moe_get_error(ws) == 0

    # (a) invariants at any size
    gi = host(saved["topk_idx"]).astype(np.int64)
    gg = host(saved["topk_gate"])
    counts, offsets = host(saved["counts"]), host(saved["offsets"])
    sop, pos = host(saved["slot_of_pair"]).astype(np.int64), host(saved["pair_of_slot"]).astype(np.int64)
    assert gi.min() >= 0 and gi.max() < E
    assert all(len(set(r)) == k for r in gi[:: max(1, T // 512)])
    np.testing.assert_allclose(gg.sum(axis=1), 1.0, atol=1e-5)
    assert np.all(np.diff(gg, axis=1) <= 1e-7)
    assert counts.sum() == T * k and offsets[0] == 0 and np.array_equal(offsets[1:], np.cumsum(counts))
    assert np.array_equal(counts, np.bincount(gi.ravel(), minlength=E))
    assert np.array_equal(pos[sop], np.arange(T * k))
    assert np.array_equal(pos, np.argsort(gi.ravel(), kind="stable"))
    xp = host(saved["x_perm"])
    rows = np.random.default_rng(1).choice(T * k, size=256, replace=False)
    assert np.array_equal(xp[rows], inp.x[pos[rows] // k])
    load = counts / counts.mean()
    print(f"{name}: max/mean expert load {load.max():.3f}, empty experts {(counts == 0).sum()}")

    # (b) oracle routing, then sampled tokens
    if router:
        z, p, ridx, rgate = ref.route(inp.x, inp.w_r, k, inp.bias)
        # the logits are checked against the rigorous fp32 dot-product bound ...
        bound = d * 2.0 ** -24 * (np.abs(inp.x.astype(np.float64)) @ np.abs(inp.w_r.astype(np.float64)))
        zg = host(saved["logits"])
        assert np.all(np.abs(zg - z) <= bound + 2.0 ** -24 * np.abs(z) + 1e-30)
        # ... and a token's routing is fixed wherever every gap among its k+1 largest oracle
        # logits exceeds twice that token's largest logit error: then the order must agree
        clear = clear_tokens(z, np.max(np.abs(zg - z), axis=1), k)
        assert clear.mean() > 0.99
        assert np.array_equal(gi[clear], ridx[clear])
        print(f"{name}: {(~clear).sum()} near-tie tokens of {T}; "
              f"routing flips among them: {(gi[~clear] != ridx[~clear]).any(axis=1).sum()}")
    else:
        ridx, rgate, clear = ridx.astype(np.int64), rgate.astype(np.float64), np.ones(T, bool)
    rng = np.random.default_rng(2)
    toks = rng.choice(np.nonzero(clear)[0], size=24, replace=False)
    gy, gdx = host(y), host(grads["dx"])
    ys, dxs = [], []
    for t in toks:
        yt, dxt = _token_oracle(inp, t, ridx[t], rgate[t], router, mx)
        ys.append(yt)
        dxs.append(dxt)
    assert rel_err(gy[toks], np.array(ys)) <= tol_c
    assert rel_err(gdx[toks], np.array(dxs)) <= tol

    # sampled experts' weight gradients (only experts all of whose tokens route clearly)
    touch = (ridx[:, :, None] == np.arange(E)).any(axis=1) | (gi[:, :, None] == np.arange(E)).any(axis=1)
    owners = [e for e in range(E) if clear[touch[:, e]].all()]
    picks = [owners[0], owners[len(owners) // 2], owners[-1]] if E > 8 else owners[:1]
    for e in picks:
        dwg, dwu, dwd = _expert_oracle(inp, e, ridx, rgate, mx)
        assert rel_err(host(grads["dw_gate"][e]), dwg) <= tol, e
        assert rel_err(host(grads["dw_up"][e]), dwu) <= tol, e
        assert rel_err(host(grads["dw_down"][e]), dwd) <= tol, e
