"""Parity at the benchmark's full sizes, in the launch configuration bench.py times
(moe_layer_fwd + moe_layer_bwd on one stream):

  * E=8:   T=8192, d=2048, k=4, ffn=1024 (near-uniform load)
  * E=128: T=8192, d=2048, k=4, ffn=1024
  * E=128: T=16384 with the Zipf-like logit bias, and with uniform random routing

Checks: (a) properties that hold at any size (routing and metadata invariants); (b) the
logits against the fp32 dot-product bound and the routing against the oracle's own on every
token whose decision is clear of the logit error; (c) bf16: every tensor the C ABI exposes
against the whole float64 oracle (about 15 s and 15 GB of host memory per case), on the
routing decided by the oracle's rule on the GPU's logits; MXFP8: the oracle's MXFP8 layer on
sub-batches of tokens (y, dx and every row of their pairs; the last rows of several experts
among them) and on the rows of three experts (their weight gradients).
"""
import dataclasses

import numpy as np
import pytest

import routing_grouped_expert_softmax_b200 as moe
from oracle import moe_ref as ref
from routing_grouped_expert_softmax_b200 import inputs as gen
from tests.gpu_util import check, check_layer, check_logits_and_routing, dev, dev_f32, gpu_decided_oracle, host

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


def _sub(inp, toks):
    """The layer inputs restricted to the tokens `toks` (weights unchanged)."""
    return dataclasses.replace(inp, T=len(toks), x=inp.x[toks], dy=inp.dy[toks])


def _mx_sampled(inp, y, saved, grads, zg, routed):
    """MXFP8 at full size: the oracle's MXFP8 layer on sub-batches.  Every quantity compared
    depends only on the rows that enter it: a token's y and dx on its own k pairs (row-wise
    blocks along d, f or 2f), an expert's weight gradients on the rows routed to it, in slot
    order (token-axis blocks of 32 from the expert's first row).  So a sub-batch with the same
    routing for its tokens gives those values exactly as the whole batch would."""
    T, E, k, f = inp.T, inp.E, inp.k, inp.f
    if routed is None:
        p = ref.softmax(ref.router_logits(inp.x, inp.w_r, inp.bias))
        idx = ref.topk_experts(zg, k)
        gate = ref.renormalised_gates(p, idx)
    else:
        idx, gate = routed[0].astype(np.int64), routed[1].astype(np.float64)
    offsets = host(saved["offsets"]).astype(np.int64)
    sop = host(saved["slot_of_pair"]).astype(np.int64)
    pos = host(saved["pair_of_slot"]).astype(np.int64)
    counts = np.diff(offsets)
    # tokens: two at random and the ones holding the last row of the four largest experts and
    # of four experts whose row count is not a multiple of 128 (their last tile is partial)
    rng = np.random.default_rng(2)
    tails = [e for e in np.argsort(-counts)[:4]] + [e for e in range(E) if counts[e] % 128][:4]
    toks = sorted(set(rng.choice(T, 2, replace=False).tolist() +
                      [int(pos[offsets[e + 1] - 1] // k) for e in tails if counts[e] > 0]))
    sub = _sub(inp, toks)
    fwd = ref.layer_fwd_mx(sub.x, inp.w_r, inp.w_gate, inp.w_up, inp.w_down, k, routing=(idx[toks], gate[toks]))
    bwd = ref.layer_bwd_mx(fwd, sub.dy, sub.x, inp.w_r, inp.w_gate, inp.w_up, inp.w_down, router=routed is None)
    check(host(y)[toks], fwd["y"], TOL_MX, "mxfp8 full-size sampled y")
    check(host(grads["dx"])[toks], bwd["dx"], TOL_MX, "mxfp8 full-size sampled dx")
    # the sampled tokens' pairs: GPU rows at their slots, oracle rows at the sub-batch's slots
    full_slot = np.array([sop[t * k + j] for t in toks for j in range(k)])
    sub_slot = fwd["slot_of_pair"]
    # ([dh | du] stays in MXFP8 in the layer: it is checked through dx_perm and the weight
    # gradients here, and in bf16 by the grouped-GEMM tests)
    hu = host(saved["hu"])[full_slot]
    rows = dict(h=(hu[:, :f], fwd["h"]), u=(hu[:, f:], fwd["u"]), a=(host(saved["a"])[full_slot], fwd["a"]),
                y_perm=(host(saved["y_perm"])[full_slot], fwd["y_perm"]),
                dx_perm=(host(grads["dx_perm"])[full_slot], bwd["dx_perm"]))
    if grads["dy_perm"] is not None:      # (None: dy_perm moved in MXFP8 only)
        rows["dy_perm"] = (host(grads["dy_perm"])[full_slot], bwd["dy_perm"])
    for n, (g_rows, o_rows) in rows.items():
        check(g_rows, o_rows[sub_slot], TOL_MX, f"mxfp8 full-size sampled {n}")
    # three experts' weight gradients from their own rows (k = 1 sub-batches, same gates)
    picks = [int(np.argmax(counts)), int(np.nonzero(counts)[0][len(np.nonzero(counts)[0]) // 2]), tails[-1]]
    for e in picks:
        pairs = pos[offsets[e]:offsets[e + 1]]           # slot order
        te = pairs // k
        g_e = gate.reshape(-1)[pairs][:, None]
        sub = _sub(inp, te)
        fe = ref.layer_fwd_mx(sub.x, inp.w_r, inp.w_gate, inp.w_up, inp.w_down, 1,
                              routing=(np.full((len(te), 1), e), g_e))
        be = ref.layer_bwd_mx(fe, sub.dy, sub.x, inp.w_r, inp.w_gate, inp.w_up, inp.w_down, router=False)
        for n in ("dw_gate", "dw_up", "dw_down"):
            check(host(grads[n][e]), be[n][e], TOL_MX, f"mxfp8 full-size expert {e} {n}")


@pytest.mark.parametrize("name", list(FULL_SIZE_CASES))
def test_fullsize(name):
    import torch
    c = FULL_SIZE_CASES[name]
    T, d, E, k, f = c["T"], c["d"], c["E"], c["k"], c["f"]
    inp = gen.make_layer_inputs(T, d, E, k, f, dtype="bf16", seed=0, skew=c["skew"])
    prec = c.get("prec", "native")
    mx = prec == "mxfp8"
    cfg = moe.config(T, d, E, k, f, dtype="bf16", prec=prec)
    ws = moe.alloc_workspace(cfg)
    saved = moe.alloc_saved(cfg)
    router = c["routing"] == "router"
    grads = moe.alloc_grads(cfg, router=router)
    w = [dev(a, "bf16") for a in (inp.w_r, inp.w_gate, inp.w_up, inp.w_down)]
    bias = dev_f32(inp.bias) if inp.bias is not None else None
    wts = moe.layer_weights(w[0], bias, w[1], w[2], w[3])
    x = dev(inp.x, "bf16")
    y = torch.empty(T, d, dtype=torch.bfloat16, device="cuda")
    routed = None
    if router:
        moe.moe_layer_fwd(cfg, wts, x, y, saved, ws)
    else:
        routed = gen.uniform_random_routing(T, E, k, seed=0)
        saved["topk_idx"].copy_(torch.from_numpy(routed[0]))
        saved["topk_gate"].copy_(torch.from_numpy(routed[1]))
        moe.moe_layer_fwd_routed(cfg, wts, x, y, saved, ws)
    moe.moe_layer_bwd(cfg, wts, x, dev(inp.dy, "bf16"), saved, grads, ws)
    assert moe.moe_get_error(ws) == 0

    # (a) invariants at any size
    gi = host(saved["topk_idx"]).astype(np.int64)
    gg = host(saved["topk_gate"])
    counts, offsets = host(saved["counts"]), host(saved["offsets"])
    sop, pos = host(saved["slot_of_pair"]).astype(np.int64), host(saved["pair_of_slot"]).astype(np.int64)
    assert gi.min() >= 0 and gi.max() < E
    assert all(len(set(r)) == k for r in gi)
    np.testing.assert_allclose(gg.sum(axis=1), 1.0, atol=1e-5)
    assert np.all(np.diff(gg, axis=1) <= 1e-7)
    assert counts.sum() == T * k and offsets[0] == 0 and np.array_equal(offsets[1:], np.cumsum(counts))
    assert np.array_equal(counts, np.bincount(gi.ravel(), minlength=E))
    assert np.array_equal(pos[sop], np.arange(T * k))
    assert np.array_equal(pos, np.argsort(gi.ravel(), kind="stable"))
    load = counts / counts.mean()
    print(f"{name}: max/mean expert load {load.max():.3f}, empty experts {(counts == 0).sum()}")

    # (b) logits within the fp32 bound, routing equal to the oracle's wherever it is clear
    zg = check_logits_and_routing(inp, saved) if router else None

    # (c) the oracle on the routing decided as the GPU decides it
    if mx:
        _mx_sampled(inp, y, saved, grads, zg, routed)
        return
    fwd, bwd_fn = gpu_decided_oracle(inp, zg, routed=routed)
    check_layer(y, saved, grads, fwd, bwd_fn(fwd), f, TOL, TOL_COMBINE, tag=f"{name} ")
