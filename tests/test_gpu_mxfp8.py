"""MXFP8 on the GPU: the quantisers bit for bit against the oracle's OCP MX rule, and the
block-scaled grouped GEMMs (forward and backward) against the oracle run on the same
quantised operands, within 6e-2 max relative error."""
import numpy as np
import pytest

import routing_grouped_expert_softmax_b200 as moe
from oracle import moe_ref as ref
from routing_grouped_expert_softmax_b200 import inputs as gen
from tests.gpu_util import (check_layer, check_logits_and_routing, dev, dev_f32, dev_i32, gpu_decided_oracle, grid,
                             host, offsets_of, random_counts, rel_err)

pytestmark = pytest.mark.gpu

TOL_MX = 6e-2


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    import torch
    assert torch.cuda.is_available()
    from routing_grouped_expert_softmax_b200 import build
    build.build()


def _special_data(rows, cols, seed):
    """bf16 values with the quantiser's edge cases planted in some 32-blocks."""
    rng = np.random.default_rng(seed)
    v = rng.standard_normal((rows, cols)).astype(np.float32) * np.exp(rng.standard_normal((rows, 1)) * 2)
    g = ref.e4m3_grid()
    if rows >= 8 and cols >= 64:
        v[0, :32] = 0.0                                   # amax = 0 -> scale 2^-127, codes 0
        v[1, :32] = 1e-30 * rng.standard_normal(32)       # tiny block
        v[2, :32] = 500.0 * rng.standard_normal(32)       # large values, saturating at 448 X
        v[3, :32] = -0.0                                  # signed zero
        mids = (g[:-1] + g[1:]) / 2                       # exact midpoints between codes (X = 1)
        v[4, :32] = np.concatenate([[256.0], rng.choice(mids[mids < 256], 31)])
        v[5, 32:64] = -v[4, :32]
    return gen.bf16_round(v)


def _codes_scales_rows(v):
    codes, scales, _ = ref.mx_quantize(v.astype(np.float64), axis=1)
    return codes, scales


@pytest.mark.parametrize("rows,cols", [(1, 32), (37, 128), (300, 2048), (8, 4096)])
def test_mx_quantize_rows_identity(rows, cols):
    import torch
    v = _special_data(rows, cols, rows)
    codes = torch.empty(rows, cols, dtype=torch.uint8, device="cuda")
    scales = torch.empty(rows, cols // 32, dtype=torch.uint8, device="cuda")
    moe.moe_mx_quantize_rows(dev(v, "bf16"), rows, cols, None, 0, rows, codes, scales)
    rc, rs = _codes_scales_rows(v)
    assert np.array_equal(host(codes), rc)
    assert np.array_equal(host(scales), rs)


@pytest.mark.parametrize("rows,cols", [(32, 32), (96, 256), (4096, 128), (100, 64)])
def test_mx_quantize_cols_identity(rows, cols):
    import torch
    v = _special_data(rows, cols, rows + 1).T.copy().T.copy()
    nb = (rows + 31) // 32
    codes = torch.empty(nb * 32, cols, dtype=torch.uint8, device="cuda")
    scales = torch.empty(nb, cols, dtype=torch.uint8, device="cuda")
    moe.moe_mx_quantize_cols(dev(v, "bf16"), rows, cols, None, 0, rows, codes, scales)
    pad = np.zeros((nb * 32, cols))
    pad[:rows] = v
    rc, rs, _ = ref.mx_quantize(pad, axis=0)
    assert np.array_equal(host(codes)[:rows], rc[:rows])
    assert np.array_equal(host(scales), rs)


def _padded(v, offsets):
    """The expert-padded layout: each expert's rows start at a multiple of 128."""
    E = len(offsets) - 1
    counts = np.diff(offsets)
    pre = np.concatenate([[0], np.cumsum((counts + 127) // 128)])
    out = np.zeros((int(pre[-1]) * 128, v.shape[1]))
    for e in range(E):
        out[pre[e] * 128: pre[e] * 128 + counts[e]] = v[offsets[e]:offsets[e + 1]]
    return out


@pytest.mark.parametrize("E,cols", [(8, 256), (128, 128), (3, 512)])
def test_mx_quantize_expert_padded(E, cols):
    import torch
    rng = np.random.default_rng(E)
    counts = random_counts(E, 150, rng)
    offsets = offsets_of(counts)
    P = int(offsets[-1])
    v = _special_data(P, cols, E)
    bound = P + 127 * E
    d_off = dev_i32(offsets)
    cr = torch.full((bound, cols), 0xAB, dtype=torch.uint8, device="cuda")
    sr = torch.full((bound, cols // 32), 0xAB, dtype=torch.uint8, device="cuda")
    moe.moe_mx_quantize_rows(dev(v, "bf16"), P, cols, d_off, E, bound, cr, sr)
    pv = _padded(v, offsets)
    n = pv.shape[0]
    rc, rs, _ = ref.mx_quantize(pv, axis=1)
    assert np.array_equal(host(cr)[:n], rc) and np.array_equal(host(sr)[:n], rs)
    ct = torch.full((bound, cols), 0xAB, dtype=torch.uint8, device="cuda")
    st = torch.full(((bound + 31) // 32, cols), 0xAB, dtype=torch.uint8, device="cuda")
    moe.moe_mx_quantize_cols(dev(v, "bf16"), P, cols, d_off, E, bound, ct, st)
    tc, ts, _ = ref.mx_quantize(pv, axis=0)
    assert np.array_equal(host(ct)[:n], tc) and np.array_equal(host(st)[:n // 32], ts)


@pytest.mark.parametrize("T,d,E,k", [(300, 256, 8, 2), (1000, 2048, 128, 4), (77, 128, 5, 3),
                                     (513, 1024, 16, 8)])
def test_permute_mxfp8_is_the_permute_and_the_row_quantiser(T, d, E, k):
    """FP8 dispatch: x_perm bit for bit as the oracle's permute, and every routed row's
    codes and scales bit for bit as the oracle's OCP MX rule on the expert-padded layout;
    the padding rows past each expert's count are left untouched."""
    import torch
    idx, _ = gen.uniform_random_routing(T, E, k, seed=T)
    counts, offsets, sop, pos = ref.routing_metadata(idx, E)
    x = _special_data(T, d, T)
    cfg = moe.config(T, d, E, k, 128)
    bound = T * k + 127 * E
    xp = torch.empty(T * k, d, dtype=torch.bfloat16, device="cuda")
    codes = torch.full((bound, d), 0xAB, dtype=torch.uint8, device="cuda")
    scales = torch.full((bound, d // 32), 0xAB, dtype=torch.uint8, device="cuda")
    moe.moe_permute_mxfp8(cfg, dev(x, "bf16"), dev_i32(sop), dev_i32(offsets), xp, bound, codes, scales)
    xpr = ref.permute(x, pos, k)
    assert np.array_equal(host(xp), xpr)
    pv = _padded(xpr, offsets)
    rc, rs, _ = ref.mx_quantize(pv, axis=1)
    pre = np.concatenate([[0], np.cumsum((np.diff(offsets) + 127) // 128)])
    valid = np.zeros(bound, bool)
    for e in range(E):
        valid[pre[e] * 128: pre[e] * 128 + int(offsets[e + 1] - offsets[e])] = True
    hc, hs = host(codes), host(scales)
    n = pv.shape[0]
    assert np.array_equal(hc[:n][valid[:n]], rc[valid[:n]])
    assert np.array_equal(hs[:n][valid[:n]], rs[valid[:n]])
    assert np.all(hc[~valid] == 0xAB) and np.all(hs[~valid] == 0xAB)


def _both_orientations(bound, d):
    import torch
    u8 = dict(dtype=torch.uint8, device="cuda")
    return (torch.full((bound, d), 0xAB, **u8), torch.full((bound, d // 32), 0xAB, **u8),
            torch.full((bound, d), 0xAB, **u8), torch.full(((bound + 31) // 32, d), 0xAB, **u8))


def _check_both_orientations(rows, offsets, cr, sr, cc, sc):
    """codes/scales along d and down the padded token axis bit for bit as the oracle's OCP MX
    rule on the expert-padded layout of `rows` (pad rows: zero codes, scale byte 0); the rows
    past the last expert's 128-row block untouched."""
    pv = _padded(rows, offsets)
    n = pv.shape[0]
    rc, rs, _ = ref.mx_quantize(pv, axis=1)
    tc, ts, _ = ref.mx_quantize(pv, axis=0)
    hcr, hsr, hcc, hsc = host(cr), host(sr), host(cc), host(sc)
    assert np.array_equal(hcr[:n], rc) and np.array_equal(hsr[:n], rs)
    assert np.array_equal(hcc[:n], tc) and np.array_equal(hsc[:n // 32], ts)
    assert np.all(hcr[n:] == 0xAB) and np.all(hsr[n:] == 0xAB)
    assert np.all(hcc[n:] == 0xAB) and np.all(hsc[n // 32:] == 0xAB)


@pytest.mark.parametrize("T,d,E,k,bf16_copy", [(300, 256, 8, 2, True), (1000, 2048, 128, 4, False),
                                               (77, 128, 5, 3, True), (513, 1024, 16, 8, False)])
def test_dispatch_mxfp8_writes_both_orientations(T, d, E, k, bf16_copy):
    """FP8 dispatch from x itself: each routed row read once through pair_of_slot and written
    in MXFP8 along d and down the padded token axis, bit for bit as the oracle quantises its
    own permute; the bf16 copy, when asked for, bit for bit as the oracle's permute."""
    import torch
    idx, _ = gen.uniform_random_routing(T, E, k, seed=T + 1)
    counts, offsets, sop, pos = ref.routing_metadata(idx, E)
    x = _special_data(T, d, T + 2)
    cfg = moe.config(T, d, E, k, 128)
    bound = T * k + 127 * E
    xp = torch.empty(T * k, d, dtype=torch.bfloat16, device="cuda") if bf16_copy else None
    cr, sr, cc, sc = _both_orientations(bound, d)
    moe.moe_dispatch_mxfp8(cfg, dev(x, "bf16"), dev_i32(pos), dev_i32(offsets), bound, xp, cr, sr, cc, sc)
    xpr = ref.permute(x, pos, k)
    if bf16_copy:
        assert np.array_equal(host(xp), xpr)
    _check_both_orientations(xpr, offsets, cr, sr, cc, sc)


@pytest.mark.parametrize("T,d,E,k", [(300, 256, 8, 2), (1000, 2048, 128, 4), (77, 128, 5, 3)])
def test_combine_bwd_mxfp8_against_oracle(T, d, E, k):
    """The combine's backward dispatched in MXFP8: dgate against the oracle within fp32
    rounding, the bf16 dy_perm and both MXFP8 orientations of it bit for bit.  The rounding of
    g * dY to bf16 decides the codes, so the oracle takes that product in the kernel's float32
    (its working precision for this call) before rounding it to bf16."""
    import torch
    idx, gate = gen.uniform_random_routing(T, E, k, seed=T + 3)
    counts, offsets, sop, pos = ref.routing_metadata(idx, E)
    rng = np.random.default_rng(T)
    gate = (gate * rng.uniform(0.2, 1.8, gate.shape)).astype(np.float32)
    dY = _special_data(T, d, T + 4)
    y_perm = grid(rng.standard_normal((T * k, d), dtype=np.float32), "bf16")
    cfg = moe.config(T, d, E, k, 128)
    bound = T * k + 127 * E
    dyp = torch.empty(T * k, d, dtype=torch.bfloat16, device="cuda")
    dgate = torch.empty(T, k, dtype=torch.float32, device="cuda")
    cr, sr, cc, sc = _both_orientations(bound, d)
    moe.moe_combine_bwd_mxfp8(cfg, dev(dY, "bf16"), dev(y_perm, "bf16"), dev_i32(pos), dev_i32(offsets),
                              dev_f32(gate), bound, dyp, dgate, cr, sr, cc, sc)
    with ref.working_precision(np.float32):
        r_dyp, _ = ref.combine_bwd(dY, y_perm, sop, gate)
    _, r_dg = ref.combine_bwd(dY, y_perm, sop, gate)
    r_dyp = ref.bf16_rne(r_dyp)
    assert np.array_equal(host(dyp), r_dyp)
    assert rel_err(host(dgate), r_dg) <= 1e-4
    _check_both_orientations(r_dyp, offsets, cr, sr, cc, sc)
    # without the bf16 copy: the same codes
    cr2, sr2, cc2, sc2 = _both_orientations(bound, d)
    moe.moe_combine_bwd_mxfp8(cfg, dev(dY, "bf16"), dev(y_perm, "bf16"), dev_i32(pos), dev_i32(offsets),
                              dev_f32(gate), bound, None, dgate, cr2, sr2, cc2, sc2)
    for a_, b_ in ((cr, cr2), (sr, sr2), (cc, cc2), (sc, sc2)):
        assert torch.equal(a_, b_)


# ------------------------------------------------------------------ grouped GEMMs

MX_CASES = [
    # d, f, E, counts kind
    (256, 256, 8, "random"),
    (128, 128, 4, "random"),
    (384, 256, 3, "one"),
    (2048, 1024, 8, "random"),
]


def _mx_counts(kind, E, rng):
    if kind == "one":
        c = np.zeros(E, np.int64)
        c[1] = 300
        return c
    return random_counts(E, 300, rng)


@pytest.mark.parametrize("d,f,E,kind", MX_CASES)
def test_mx_grouped_swiglu_fwd(d, f, E, kind):
    import torch
    rng = np.random.default_rng(d + f + E)
    offsets = offsets_of(_mx_counts(kind, E, rng))
    P = int(offsets[-1])
    x = grid(rng.standard_normal((P, d), dtype=np.float32), "bf16")
    wg = grid(rng.standard_normal((E, d, f), dtype=np.float32) / np.sqrt(d), "bf16")
    wu = grid(rng.standard_normal((E, d, f), dtype=np.float32) / np.sqrt(d), "bf16")
    wd = grid(rng.standard_normal((E, f, d), dtype=np.float32) / np.sqrt(f), "bf16")
    cfg = moe.config(P, d, E, 1, f, dtype="bf16", prec="mxfp8")
    ws = moe.alloc_workspace(cfg)
    hu = torch.empty(P, 2 * f, dtype=torch.bfloat16, device="cuda")
    a = torch.empty(P, f, dtype=torch.bfloat16, device="cuda")
    y = torch.empty(P, d, dtype=torch.bfloat16, device="cuda")
    moe.moe_grouped_swiglu_fwd(cfg, dev(x, "bf16"), dev_i32(offsets), dev(wg, "bf16"), dev(wu, "bf16"),
                               dev(wd, "bf16"), hu, a, y, ws)
    assert moe.moe_get_error(ws) == 0
    h, u, ra, ry = ref.grouped_swiglu_mx(x, offsets, wg, wu, wd)
    g = host(hu)
    assert rel_err(g[:, :f], h) <= TOL_MX
    assert rel_err(g[:, f:], u) <= TOL_MX
    assert rel_err(host(a), ra) <= TOL_MX
    assert rel_err(host(y), ry) <= TOL_MX
    # h and u come from exactly quantised operands: far tighter than the MX bar
    assert rel_err(g[:, :f], h) <= 1e-2


@pytest.mark.parametrize("d,f,E,kind", MX_CASES)
def test_mx_grouped_swiglu_bwd(d, f, E, kind):
    import torch
    rng = np.random.default_rng(3 * d + f + E)
    counts = _mx_counts(kind, E, rng)
    offsets = offsets_of(counts)
    P = int(offsets[-1])
    x = grid(rng.standard_normal((P, d), dtype=np.float32), "bf16")
    dy = grid(rng.standard_normal((P, d), dtype=np.float32), "bf16")
    h = grid(rng.standard_normal((P, f), dtype=np.float32), "bf16")
    u = grid(rng.standard_normal((P, f), dtype=np.float32), "bf16")
    a = grid(rng.standard_normal((P, f), dtype=np.float32), "bf16")
    wg = grid(rng.standard_normal((E, d, f), dtype=np.float32) / np.sqrt(d), "bf16")
    wu = grid(rng.standard_normal((E, d, f), dtype=np.float32) / np.sqrt(d), "bf16")
    wd = grid(rng.standard_normal((E, f, d), dtype=np.float32) / np.sqrt(f), "bf16")
    cfg = moe.config(P, d, E, 1, f, dtype="bf16", prec="mxfp8")
    ws = moe.alloc_workspace(cfg)
    dhu = torch.empty(P, 2 * f, dtype=torch.bfloat16, device="cuda")
    dxp = torch.empty(P, d, dtype=torch.bfloat16, device="cuda")
    dwg = torch.full((E, d, f), 7.0, dtype=torch.bfloat16, device="cuda")
    dwu = torch.full((E, d, f), 7.0, dtype=torch.bfloat16, device="cuda")
    dwd = torch.full((E, f, d), 7.0, dtype=torch.bfloat16, device="cuda")
    moe.moe_grouped_swiglu_bwd(cfg, dev(dy, "bf16"), dev(x, "bf16"), dev(np.concatenate([h, u], 1), "bf16"),
                               dev(a, "bf16"), dev_i32(offsets), dev(wg, "bf16"), dev(wu, "bf16"), dev(wd, "bf16"),
                               dhu, dxp, dwg, dwu, dwd, ws)
    assert moe.moe_get_error(ws) == 0
    r = ref.grouped_swiglu_bwd_mx(dy, x, h, u, a, offsets, wg, wu, wd)
    g = host(dhu)
    assert rel_err(g[:, :f], r["dh"]) <= TOL_MX
    assert rel_err(g[:, f:], r["du"]) <= TOL_MX
    assert rel_err(host(dxp), r["dx_perm"]) <= TOL_MX
    for name, t in (("dw_gate", dwg), ("dw_up", dwu), ("dw_down", dwd)):
        assert rel_err(host(t), r[name]) <= TOL_MX, name
    for e in np.nonzero(counts == 0)[0]:
        assert np.all(host(dwg[e]) == 0) and np.all(host(dwd[e]) == 0)


@pytest.mark.parametrize("T,d,E,k,f,skew", [(512, 256, 16, 4, 256, False), (700, 384, 8, 2, 256, True)])
def test_mx_layer_against_oracle_and_bf16_path(T, d, E, k, f, skew):
    import torch
    inp = gen.make_layer_inputs(T, d, E, k, f, dtype="bf16", seed=5, skew=skew)
    outs = {}
    for prec in ("native", "mxfp8"):
        cfg = moe.config(T, d, E, k, f, dtype="bf16", prec=prec)
        ws = moe.alloc_workspace(cfg)
        saved = moe.alloc_saved(cfg)
        grads = moe.alloc_grads(cfg)
        w = [dev(a_, "bf16") for a_ in (inp.w_r, inp.w_gate, inp.w_up, inp.w_down)]
        bias = dev_f32(inp.bias) if inp.bias is not None else None
        wts = moe.layer_weights(w[0], bias, w[1], w[2], w[3])
        x = dev(inp.x, "bf16")
        y = torch.empty(T, d, dtype=torch.bfloat16, device="cuda")
        moe.moe_layer_fwd(cfg, wts, x, y, saved, ws)
        moe.moe_layer_bwd(cfg, wts, x, dev(inp.dy, "bf16"), saved, grads, ws)
        assert moe.moe_get_error(ws) == 0
        outs[prec] = (y, saved, grads)
    # the oracle's MXFP8 layer (every GEMM operand quantised along its own K, the five stored
    # tensors in bf16), on the routing decided as the GPU decides it
    y, sv, g = outs["mxfp8"]
    zg = check_logits_and_routing(inp, sv)
    fwd, bwd_fn = gpu_decided_oracle(inp, zg, mx=True)
    check_layer(y, sv, g, fwd, bwd_fn(fwd), f, TOL_MX, TOL_MX, tag="mxfp8 ", dhu=False)
    # and MXFP8 stays close to the bf16 path (quantisation error only)
    ybf, _, gbf = outs["native"]
    assert 0 < rel_err(host(y), host(ybf)) <= 0.1
    for n in ("dx", "dw_gate", "dw_down"):
        assert rel_err(host(g[n]), host(gbf[n])) <= 0.15, n


@pytest.mark.parametrize("recompute", [False, True])
def test_mx_saved_weights_give_the_same_bits(recompute):
    """The forward's MXFP8 weight copies (all four orientations from one read of each weight)
    reused by the backward give exactly what quantising each orientation where it is used
    gives."""
    import torch
    T, d, E, k, f = 600, 256, 8, 4, 256
    inp = gen.make_layer_inputs(T, d, E, k, f, dtype="bf16", seed=17)
    outs = []
    for keep in (False, True):
        cfg = moe.config(T, d, E, k, f, dtype="bf16", prec="mxfp8")
        ws = moe.alloc_workspace(cfg)
        saved = moe.alloc_saved(cfg, recompute=recompute, mx_saved=keep)
        assert (saved["mx_saved"] is not None) == keep
        grads = moe.alloc_grads(cfg)
        w = [dev(a_, "bf16") for a_ in (inp.w_r, inp.w_gate, inp.w_up, inp.w_down)]
        wts = moe.layer_weights(w[0], None, w[1], w[2], w[3])
        x = dev(inp.x, "bf16")
        y = torch.empty(T, d, dtype=torch.bfloat16, device="cuda")
        moe.moe_layer_fwd(cfg, wts, x, y, saved, ws)
        moe.moe_layer_bwd(cfg, wts, x, dev(inp.dy, "bf16"), saved, grads, ws)
        assert moe.moe_get_error(ws) == 0
        outs.append([host(y)] + [host(grads[n]) for n in ("dx", "dw_gate", "dw_up", "dw_down", "dw_router")])
    for a_, b_ in zip(*outs):
        assert np.array_equal(a_, b_)
