"""Helpers shared by the GPU tests: move generator arrays to the device and back, and the
error measures the tolerances are written in."""
import numpy as np

from routing_grouped_expert_softmax_b200 import inputs as gen


def dev(a, dtype):
    """fp32 numpy values (already on the dtype's grid) -> a CUDA tensor of that dtype."""
    import torch
    a = np.ascontiguousarray(a, np.float32)
    if dtype == "bf16":
        bits = gen.bf16_bits(a)
        return torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).cuda()
    return torch.from_numpy(a).cuda()


def dev_f32(a):
    import torch
    return torch.from_numpy(np.ascontiguousarray(a, np.float32)).cuda()


def dev_i32(a):
    import torch
    return torch.from_numpy(np.ascontiguousarray(a, np.int32)).cuda()


def host(t):
    """A CUDA tensor -> float64 numpy (bf16 converts exactly)."""
    import torch
    if t.dtype in (torch.bfloat16, torch.float16):
        t = t.float()
    return t.detach().cpu().numpy().astype(np.float64) if t.is_floating_point() else t.cpu().numpy()


def rel_err(got, ref):
    """max |got - ref| / max |ref| over the whole tensor."""
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    scale = np.max(np.abs(ref)) if ref.size else 0.0
    if scale == 0:
        return float(np.max(np.abs(got))) if got.size else 0.0
    return float(np.max(np.abs(got - ref)) / scale)


def grid(a, dtype):
    """Round to the dtype's grid (the values the GPU will receive)."""
    return gen.bf16_round(a) if dtype == "bf16" else np.asarray(a, np.float32)


def random_counts(E, total_hint, rng, zero_some=True, cap=None):
    """Per-expert row counts with empty experts, counts off the 128-row tiles, and a tail."""
    c = rng.integers(0, max(2, 2 * total_hint // max(E, 1)), size=E)
    if zero_some and E > 2:
        c[rng.choice(E, size=max(1, E // 5), replace=False)] = 0
    if cap is not None:
        c = np.minimum(c, cap)
    if c.sum() == 0:
        c[0] = 1
    return c.astype(np.int64)


def offsets_of(counts):
    return np.concatenate([[0], np.cumsum(counts)]).astype(np.int64)


# ---------------------------------------------------------------- layer comparisons
# Elementwise report next to the per-tensor bar: an element counts as outside when
# |got - ref| > tol |ref| + 1e-3 max|ref| (atol = 1e-3 of the tensor's scale).  The bar the
# tests assert is the per-tensor max relative error; the elementwise figures are collected in
# PARITY_REPORT and printed (pytest -s), and written as JSON lines to the file named by the
# environment variable MOE_PARITY_REPORT when it is set.
PARITY_REPORT = []


def check(got, ref_v, tol, name):
    import json
    import os
    got = np.asarray(got, np.float64)
    ref_v = np.asarray(ref_v, np.float64)
    assert got.shape == ref_v.shape, (name, got.shape, ref_v.shape)
    e = rel_err(got, ref_v)
    scale = float(np.max(np.abs(ref_v))) if ref_v.size else 0.0
    diff = np.abs(got - ref_v)
    over = int(np.count_nonzero(diff > tol * np.abs(ref_v) + 1e-3 * scale))
    ratio = float(np.max(diff / (np.abs(ref_v) + 1e-3 * scale))) if scale > 0 else float(np.max(diff, initial=0))
    row = dict(name=name, rel_err=e, tol=tol, elems=int(ref_v.size), elems_outside=over,
               max_elem_err_over_abs_ref_plus_atol=ratio)
    PARITY_REPORT.append(row)
    print(f"parity {name}: rel_err {e:.3e} (bar {tol}), elementwise outside {over}/{ref_v.size}, "
          f"max |d|/(|ref|+atol) {ratio:.3e}")
    path = os.environ.get("MOE_PARITY_REPORT")
    if path:
        with open(path, "a") as fh:
            fh.write(json.dumps(row) + "\n")
    assert e <= tol, (name, e, tol)


def gpu_decided_oracle(inp, logits_gpu, shared=None, mx=False, routed=None, router=True):
    """The oracle's forward and backward with the routing decision taken the way the GPU takes
    it: the oracle's own top-k rule applied to the GPU's fp32 logits (which the tests first
    check against the oracle's float64 logits within the fp32 dot-product bound); gates are
    the oracle's float64 softmax renormalised over that selection.  routed=(idx, gate): fixed
    routing instead (no logits).  mx: the MXFP8 layer (layer_fwd_mx / layer_bwd_mx)."""
    from oracle import moe_ref as ref
    k = inp.k
    if routed is not None:
        idx, gate = routed
        z = p = None
    else:
        z = ref.router_logits(inp.x, inp.w_r, inp.bias)
        p = ref.softmax(z)
        idx = ref.topk_experts(np.asarray(logits_gpu, np.float64), k)
        gate = ref.renormalised_gates(p, idx)
    if mx:
        fwd = ref.layer_fwd_mx(inp.x, inp.w_r, inp.w_gate, inp.w_up, inp.w_down, k, inp.bias,
                               routing=(idx, gate), shared=shared)
        bwd_fn = lambda f: ref.layer_bwd_mx(f, inp.dy, inp.x, inp.w_r, inp.w_gate, inp.w_up, inp.w_down,
                                            router=router and routed is None, shared=shared)
    else:
        fwd = ref.layer_fwd_routed(inp.x, idx, gate, inp.w_gate, inp.w_up, inp.w_down, shared=shared)
        if router and routed is None:
            bwd_fn = lambda f: ref.layer_bwd(f, inp.dy, inp.x, inp.w_r, inp.w_gate, inp.w_up, inp.w_down,
                                             shared=shared)
        else:
            bwd_fn = lambda f: ref.layer_bwd_routed(f, inp.dy, inp.w_gate, inp.w_up, inp.w_down, x=inp.x,
                                                    shared=shared)
    if z is not None:
        fwd.update(z=z, p=p)
    return fwd, bwd_fn


def check_layer(y, saved, grads, fwd, bwd, f, tol, tol_combine, tag="", dhu=True):
    """Every tensor the layer's C ABI exposes against the oracle's (bit-exact for the integer
    metadata and the permuted rows, the stated tolerances for floating point).  dhu=False: the
    layer kept [dh | du] in MXFP8 only (its GEMM-level test checks the bf16 values)."""
    for key in ("counts", "offsets", "slot_of_pair", "pair_of_slot"):
        assert np.array_equal(host(saved[key]), fwd[key]), key
    if saved.get("x_perm") is not None:      # (None: the rows moved in MXFP8 only)
        assert np.array_equal(host(saved["x_perm"]), fwd["x_perm"])
    assert np.max(np.abs(host(saved["topk_gate"]) - fwd["gate"])) <= 1e-5
    if saved.get("hu") is not None:
        hu = host(saved["hu"])
        check(hu[:, :f], fwd["h"], tol, tag + "h")
        check(hu[:, f:], fwd["u"], tol, tag + "u")
    check(host(saved["a"]), fwd["a"], tol, tag + "a")
    check(host(saved["y_perm"]), fwd["y_perm"], tol, tag + "y_perm")
    check(host(y), fwd["y"], tol_combine, tag + "y")
    if saved.get("shared_a") is not None:
        check(host(saved["shared_a"]), fwd["shared_a"], tol, tag + "shared_a")
        if saved.get("shared_hu") is not None:
            shu = host(saved["shared_hu"])
            check(shu[:, :f], fwd["shared_h"], tol, tag + "shared_h")
            check(shu[:, f:], fwd["shared_u"], tol, tag + "shared_u")
    if grads is None:
        return
    if grads.get("dy_perm") is not None:
        check(host(grads["dy_perm"]), bwd["dy_perm"], tol_combine, tag + "dy_perm")
    check(host(grads["dgate"]), bwd["dgate"], tol, tag + "dgate")
    if dhu:
        dhu_g = host(grads["dhu"])
        check(dhu_g[:, :f], bwd["dh"], tol, tag + "dh")
        check(dhu_g[:, f:], bwd["du"], tol, tag + "du")
    check(host(grads["dx_perm"]), bwd["dx_perm"], tol, tag + "dx_perm")
    for n, key in (("dx", "dx"), ("dw_gate", "dw_gate"), ("dw_up", "dw_up"), ("dw_down", "dw_down")):
        check(host(grads[n]), bwd[key], tol, tag + n)
    if grads.get("dw_router") is not None and "dw_r" in bwd:
        check(host(grads["dw_router"]), bwd["dw_r"], tol, tag + "dw_router")
    if grads.get("dw_shared_gate") is not None:
        sdhu = host(grads["shared_dhu"])
        check(sdhu[:, :f], bwd["shared_dh"], tol, tag + "shared_dh")
        check(sdhu[:, f:], bwd["shared_du"], tol, tag + "shared_du")
        for n in ("dw_shared_gate", "dw_shared_up", "dw_shared_down"):
            check(host(grads[n]), bwd[n], tol, tag + n)


def check_logits_and_routing(inp, saved):
    """The GPU's fp32 logits within the rigorous fp32 dot-product bound of the oracle's float64
    logits, and its routing bit for bit equal to the oracle's own wherever every gap among the
    k+1 largest oracle logits exceeds twice the token's measured logit error.  Returns the GPU
    logits (float64)."""
    from oracle import moe_ref as ref
    z = ref.router_logits(inp.x, inp.w_r, inp.bias)
    zg = host(saved["logits"])
    bound = inp.d * 2.0 ** -24 * (np.abs(inp.x.astype(np.float64)) @ np.abs(inp.w_r.astype(np.float64)))
    assert np.all(np.abs(zg - z) <= bound + 2.0 ** -24 * np.abs(z) + 1e-30)
    zs = np.sort(z, axis=1)[:, ::-1][:, :inp.k + 1]
    delta = np.max(np.abs(zg - z), axis=1)
    clear = np.all(-np.diff(zs, axis=1) > 2 * delta[:, None], axis=1)
    gi = host(saved["topk_idx"])
    own = ref.topk_experts(z, inp.k)
    assert np.array_equal(gi[clear], own[clear])
    # where the decision is not clear, the GPU's choice is the oracle's rule on the GPU's logits
    assert np.array_equal(gi, ref.topk_experts(zg, inp.k))
    print(f"routing: {(~clear).sum()} near-tie tokens of {inp.T}; "
          f"flips against float64 among them: {(gi[~clear] != own[~clear]).any(axis=1).sum()}")
    return zg
