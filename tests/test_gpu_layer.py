"""Whole-layer parity through moe_layer_fwd / moe_layer_bwd at sizes the oracle finishes
in seconds: every intermediate the C ABI exposes is compared with the oracle.  The routing
decision is taken on both sides by the same rule on the GPU's fp32 logits, which are first
checked against the oracle's float64 logits (and the routing against the oracle's own on every
token whose decision is clear of the logit error), so near-ties never skip a comparison."""
import numpy as np
import pytest

import routing_grouped_expert_softmax_b200 as moe
from oracle import moe_ref as ref
from routing_grouped_expert_softmax_b200 import inputs as gen
from tests.gpu_util import (check_layer, check_logits_and_routing, dev, dev_f32, gpu_decided_oracle,
                             host)

pytestmark = pytest.mark.gpu

TOL = 2e-2
TOL_COMBINE = 1e-2


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    import torch
    assert torch.cuda.is_available()
    from routing_grouped_expert_softmax_b200 import build
    build.build()


def _run_layer(inp, backward=True, routed=None):
    import torch
    T, d, E, k, f, dtype = inp.T, inp.d, inp.E, inp.k, inp.f, inp.dtype
    cfg = moe.config(T, d, E, k, f, dtype=dtype)
    ws = moe.alloc_workspace(cfg)
    saved = moe.alloc_saved(cfg)
    w = [dev(a, dtype) for a in (inp.w_r, inp.w_gate, inp.w_up, inp.w_down)]
    bias = dev_f32(inp.bias) if inp.bias is not None else None
    wts = moe.layer_weights(w[0], bias, w[1], w[2], w[3])
    x = dev(inp.x, dtype)
    y = torch.empty(T, d, dtype=moe.torch_dtype(cfg), device="cuda")
    if routed is not None:
        saved["topk_idx"].copy_(torch.from_numpy(routed[0]))
        saved["topk_gate"].copy_(torch.from_numpy(routed[1]))
        moe.moe_layer_fwd_routed(cfg, wts, x, y, saved, ws)
    else:
        moe.moe_layer_fwd(cfg, wts, x, y, saved, ws)
    grads = None
    if backward:
        grads = moe.alloc_grads(cfg, router=routed is None)
        moe.moe_layer_bwd(cfg, wts, x, dev(inp.dy, dtype), saved, grads, ws)
    assert moe.moe_get_error(ws) == 0
    return y, saved, grads


@pytest.mark.parametrize("T,d,E,k,f,dtype,skew", [
    (256, 128, 8, 2, 256, "f32", False),          # the tiny fp32 forward configuration
    (256, 128, 8, 2, 256, "bf16", False),
    (600, 256, 16, 4, 256, "bf16", True),
    (1000, 384, 128, 4, 128, "bf16", False),
    (130, 256, 256, 8, 384, "bf16", True),
    (64, 128, 2, 2, 128, "bf16", False),
    (2000, 256, 4, 2, 256, "bf16", False),        # 1000 rows per expert: 256-row CTA-pair tiles
])
def test_layer_against_oracle(T, d, E, k, f, dtype, skew):
    inp = gen.make_layer_inputs(T, d, E, k, f, dtype=dtype, seed=T + E, skew=skew)
    backward = dtype == "bf16"
    y, sv, g = _run_layer(inp, backward=backward)
    zg = check_logits_and_routing(inp, sv)
    fwd, bwd_fn = gpu_decided_oracle(inp, zg)
    check_layer(y, sv, g, fwd, bwd_fn(fwd) if backward else None, f, TOL, TOL_COMBINE)


@pytest.mark.parametrize("T,d,E,k,f", [(512, 256, 16, 4, 256), (300, 128, 128, 4, 128)])
def test_layer_uniform_random_routing(T, d, E, k, f):
    inp = gen.make_layer_inputs(T, d, E, k, f, dtype="bf16", seed=3)
    idx, gate = gen.uniform_random_routing(T, E, k, seed=3)
    y, sv, g = _run_layer(inp, routed=(idx, gate))
    fwd, bwd_fn = gpu_decided_oracle(inp, None, routed=(idx, gate))
    check_layer(y, sv, g, fwd, bwd_fn(fwd), f, TOL, TOL_COMBINE)


def test_layer_empty_batch():
    import torch
    cfg = moe.config(0, 128, 8, 2, 128)
    ws = moe.alloc_workspace(cfg)
    saved = moe.alloc_saved(cfg)
    grads = moe.alloc_grads(cfg)
    z = torch.zeros(8, 128, 128, dtype=torch.bfloat16, device="cuda")
    wts = moe.layer_weights(torch.zeros(128, 8, dtype=torch.bfloat16, device="cuda"), None, z, z, z)
    for n in ("dw_gate", "dw_up", "dw_down", "dw_router"):
        grads[n].fill_(5)
    moe.moe_layer_fwd(cfg, wts, None, None, saved, ws)
    moe.moe_layer_bwd(cfg, wts, None, None, saved, grads, ws)
    torch.cuda.synchronize()
    assert host(saved["offsets"]).tolist() == [0] * 9
    for n in ("dw_gate", "dw_up", "dw_down", "dw_router"):
        assert float(grads[n].abs().max()) == 0.0
