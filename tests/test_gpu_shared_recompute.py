"""The shared expert and the recomputing backward through moe_layer_fwd / moe_layer_bwd.

Shared expert: parity with the oracle (every output and gradient, including the shared
expert's activations and weight gradients).  Recompute (saved h | u left out): the same
kernels on the same inputs, so forward outputs and every gradient must equal those of the
saving path bit for bit."""
import numpy as np
import pytest

import routing_grouped_expert_softmax_b200 as moe
from oracle import moe_ref as ref
from routing_grouped_expert_softmax_b200 import inputs as gen
from tests.gpu_util import dev, dev_f32, host, rel_err

pytestmark = pytest.mark.gpu

TOL = 2e-2


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
    fwd = ref.layer_fwd(inp.x, inp.w_r, inp.w_gate, inp.w_up, inp.w_down, k, inp.bias, shared=sh)
    gi = host(sv["topk_idx"])
    if not np.array_equal(gi, fwd["idx"]):
        pytest.skip("near-tie routing differs from the fp64 oracle; the whole-layer comparison needs it equal")
    shu = host(sv["shared_hu"])
    assert rel_err(shu[:, :f], fwd["shared_h"]) <= TOL and rel_err(shu[:, f:], fwd["shared_u"]) <= TOL
    assert rel_err(host(sv["shared_a"]), fwd["shared_a"]) <= TOL
    assert rel_err(host(y), fwd["y"]) <= TOL
    bwd = ref.layer_bwd(fwd, inp.dy, inp.x, inp.w_r, inp.w_gate, inp.w_up, inp.w_down, shared=sh)
    sdhu = host(g["shared_dhu"])
    assert rel_err(sdhu[:, :f], bwd["shared_dh"]) <= TOL and rel_err(sdhu[:, f:], bwd["shared_du"]) <= TOL
    for n, key in (("dx", "dx"), ("dw_gate", "dw_gate"), ("dw_up", "dw_up"), ("dw_down", "dw_down"),
                   ("dw_router", "dw_r"), ("dw_shared_gate", "dw_shared_gate"),
                   ("dw_shared_up", "dw_shared_up"), ("dw_shared_down", "dw_shared_down")):
        assert rel_err(host(g[n]), bwd[key]) <= TOL, n


def test_shared_expert_with_uniform_random_routing():
    T, d, E, k, f = 512, 256, 16, 4, 256
    inp = gen.make_layer_inputs(T, d, E, k, f, seed=5)
    sh = gen.make_shared_expert(d, f, seed=6)
    idx, gate = gen.uniform_random_routing(T, E, k, seed=5)
    y, sv, g = _run(inp, shared=sh, routed=(idx, gate))
    fwd = ref.layer_fwd_routed(inp.x, idx, gate, inp.w_gate, inp.w_up, inp.w_down, shared=sh)
    bwd = ref.layer_bwd_routed(fwd, inp.dy, inp.w_gate, inp.w_up, inp.w_down, x=inp.x, shared=sh)
    assert rel_err(host(y), fwd["y"]) <= TOL
    for n in ("dx", "dw_gate", "dw_up", "dw_down", "dw_shared_gate", "dw_shared_up", "dw_shared_down"):
        assert rel_err(host(g[n]), bwd[n]) <= TOL, n


@pytest.mark.parametrize("T,d,E,k,f,shared,prec", [
    (600, 256, 16, 4, 256, False, "native"),
    (1100, 256, 4, 2, 128, True, "native"),
    (300, 128, 128, 4, 128, True, "native"),
    (256, 256, 8, 2, 256, True, "mxfp8"),
])
def test_recompute_equals_saving_bit_for_bit(T, d, E, k, f, shared, prec):
    inp = gen.make_layer_inputs(T, d, E, k, f, seed=T + 1)
    sh = gen.make_shared_expert(d, f, seed=T + 2) if shared else None
    y0, s0, g0 = _run(inp, shared=sh, prec=prec)
    y1, s1, g1 = _run(inp, shared=sh, recompute=True, prec=prec)
    assert s1["hu"] is None and s1["shared_hu"] is None
    assert np.array_equal(host(y0), host(y1))
    for n in ("a", "y_perm", "x_perm") + (("shared_a",) if shared else ()):
        assert np.array_equal(host(s0[n]), host(s1[n])), n
    names = ["dx", "dw_router", "dw_gate", "dw_up", "dw_down", "dhu", "dx_perm", "dgate"]
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
