"""The shared expert and the recomputing backward through moe_layer_fwd / moe_layer_bwd.

Shared expert: parity with the oracle (every output and gradient, including the shared
expert's activations and weight gradients).  Recompute (saved h | u left out): parity with
the oracle (bf16 and MXFP8), and, since the same kernels run on the same inputs, forward
outputs and every gradient bit for bit equal to those of the saving path."""
import numpy as np
import pytest

import routing_grouped_expert_softmax_b200 as moe
from routing_grouped_expert_softmax_b200 import inputs as gen
from tests.gpu_util import check_layer, check_logits_and_routing, dev, dev_f32, gpu_decided_oracle, host

pytestmark = pytest.mark.gpu

TOL = 2e-2
TOL_COMBINE = 1e-2
TOL_MX = 6e-2


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    import torch
    assert torch.cuda.is_available()
    from routing_grouped_expert_softmax_b200 import build
    build.build()


def _run(inp, shared=None, recompute=False, prec="native", routed=None):
    import torch
    T, d, E, k, f = inp.T, inp.d, inp.E, inp.k, inp.f
    cfg = moe.config(T, d, E, k, f, prec=prec)
    ws = moe.alloc_workspace(cfg)
    saved = moe.alloc_saved(cfg, shared=shared is not None, recompute=recompute)
    w = [dev(a, "bf16") for a in (inp.w_r, inp.w_gate, inp.w_up, inp.w_down)]
    sh = tuple(dev(a, "bf16") for a in shared) if shared is not None else None
    bias = dev_f32(inp.bias) if inp.bias is not None else None
    wts = moe.layer_weights(w[0], bias, w[1], w[2], w[3], shared=sh)
    x = dev(inp.x, "bf16")
    y = torch.empty(T, d, dtype=torch.bfloat16, device="cuda")
    if routed is not None:
        saved["topk_idx"].copy_(torch.from_numpy(routed[0]))
        saved["topk_gate"].copy_(torch.from_numpy(routed[1]))
        moe.moe_layer_fwd_routed(cfg, wts, x, y, saved, ws)
    else:
        moe.moe_layer_fwd(cfg, wts, x, y, saved, ws)
    grads = moe.alloc_grads(cfg, router=routed is None, shared=shared is not None)
    moe.moe_layer_bwd(cfg, wts, x, dev(inp.dy, "bf16"), saved, grads, ws)
    assert moe.moe_get_error(ws) == 0
    return y, saved, grads


@pytest.mark.parametrize("T,d,E,k,f,skew", [
    (256, 128, 8, 2, 256, False),
    (600, 256, 16, 4, 256, True),
    (300, 128, 128, 4, 128, False),
    (1100, 256, 4, 2, 128, False),     # experts large enough for 256-row tile pairs
])
def test_layer_with_shared_expert_against_oracle(T, d, E, k, f, skew):
    inp = gen.make_layer_inputs(T, d, E, k, f, seed=T + 7, skew=skew)
    sh = gen.make_shared_expert(d, f, seed=T + 8)
    y, sv, g = _run(inp, shared=sh)
    zg = check_logits_and_routing(inp, sv)
    fwd, bwd_fn = gpu_decided_oracle(inp, zg, shared=sh)
    check_layer(y, sv, g, fwd, bwd_fn(fwd), f, TOL, TOL_COMBINE)


def test_shared_expert_with_uniform_random_routing():
    T, d, E, k, f = 512, 256, 16, 4, 256
    inp = gen.make_layer_inputs(T, d, E, k, f, seed=5)
    sh = gen.make_shared_expert(d, f, seed=6)
    idx, gate = gen.uniform_random_routing(T, E, k, seed=5)
    y, sv, g = _run(inp, shared=sh, routed=(idx, gate))
    fwd, bwd_fn = gpu_decided_oracle(inp, None, shared=sh, routed=(idx, gate))
    check_layer(y, sv, g, fwd, bwd_fn(fwd), f, TOL, TOL_COMBINE)


@pytest.mark.parametrize("T,d,E,k,f,shared,prec", [
    (600, 256, 16, 4, 256, False, "native"),
    (1100, 256, 4, 2, 128, True, "native"),
    (300, 128, 128, 4, 128, True, "native"),
    (256, 256, 8, 2, 256, True, "mxfp8"),
    (700, 256, 16, 4, 256, False, "mxfp8"),
])
def test_recompute_against_oracle_and_saving_path(T, d, E, k, f, shared, prec):
    """The recomputing backward against the oracle, and bit for bit against the saving path
    (the same kernels on the same inputs)."""
    inp = gen.make_layer_inputs(T, d, E, k, f, seed=T + 1)
    sh = gen.make_shared_expert(d, f, seed=T + 2) if shared else None
    y0, s0, g0 = _run(inp, shared=sh, prec=prec)
    y1, s1, g1 = _run(inp, shared=sh, recompute=True, prec=prec)
    assert s1["hu"] is None and s1["shared_hu"] is None
    # against the oracle (the MXFP8 layer's oracle for prec="mxfp8")
    mx = prec == "mxfp8"
    zg = check_logits_and_routing(inp, s1)
    fwd, bwd_fn = gpu_decided_oracle(inp, zg, shared=sh, mx=mx)
    tol, tol_c = (TOL_MX, TOL_MX) if mx else (TOL, TOL_COMBINE)
    check_layer(y1, s1, g1, fwd, bwd_fn(fwd), f, tol, tol_c, tag="recompute ", dhu=not mx)
    # and bit for bit against the path that keeps h | u
    assert np.array_equal(host(y0), host(y1))
    for n in ("a", "y_perm", "x_perm") + (("shared_a",) if shared else ()):
        if s0[n] is None:             # x_perm: the MXFP8 layer moves the rows in MXFP8 only
            assert s1[n] is None, n
            continue
        assert np.array_equal(host(s0[n]), host(s1[n])), n
    names = ["dx", "dw_router", "dw_gate", "dw_up", "dw_down", "dx_perm", "dgate"] + ([] if mx else ["dhu"])
    if shared:
        names += ["dw_shared_gate", "dw_shared_up", "dw_shared_down", "shared_dhu"]
    for n in names:
        assert np.array_equal(host(g0[n]), host(g1[n])), n


def test_partial_shared_expert_is_rejected():
    import torch
    cfg = moe.config(16, 128, 8, 2, 128)
    ws = moe.alloc_workspace(cfg)
    saved = moe.alloc_saved(cfg, shared=True)
    z = torch.zeros(8, 128, 128, dtype=torch.bfloat16, device="cuda")
    s = torch.zeros(128, 128, dtype=torch.bfloat16, device="cuda")
    wts = moe.layer_weights(torch.zeros(128, 8, dtype=torch.bfloat16, device="cuda"), None, z, z, z,
                            shared=(s, s, None))
    x = torch.zeros(16, 128, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(moe.MoeError) as e:
        moe.moe_layer_fwd(cfg, wts, x, x.clone(), saved, ws)
    assert e.value.code == moe.MOE_ERR_INVALID_ARG
