"""GPU parity of every C-ABI call against the CPU oracle, on seeded generator inputs.

Bars: bit-exact for indices, counts, offsets and slot maps; bit-exact copies for the
permute; gates within 1e-6 of the oracle on the same fp32 logits; floats within the
stated max relative error (2e-2, 1e-2 on the combine).
"""
import numpy as np
import pytest

import routing_grouped_expert_softmax_b200 as moe
from oracle import moe_ref as ref
from routing_grouped_expert_softmax_b200 import inputs as gen
from tests.gpu_util import dev, dev_f32, dev_i32, grid, host, offsets_of, random_counts, rel_err

pytestmark = pytest.mark.gpu

TOL = 2e-2
TOL_COMBINE = 1e-2


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    import torch
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from routing_grouped_expert_softmax_b200 import build
    build.build()
    moe.lib()


def _ws(cfg):
    return moe.alloc_workspace(cfg)


def _check_no_device_error(ws):
    assert moe.moe_get_error(ws) == 0


# ------------------------------------------------------------------ routing

@pytest.mark.parametrize("T,E,k,kind", [
    (1, 1, 1, "normal"), (37, 8, 2, "tied"), (1000, 128, 4, "normal"), (513, 128, 4, "tied"),
    (300, 256, 8, "tied"), (64, 64, 8, "equal"), (100, 2, 2, "normal"), (257, 33, 3, "tied"),
    (4096, 128, 4, "normal"),
])
def test_topk_gating_bit_exact(T, E, k, kind):
    import torch
    if kind == "normal":
        z = gen.normal_logits(T, E, seed=T + E)
    elif kind == "tied":
        z = gen.tied_logits(T, E, levels=3, seed=T)
    else:
        z = np.full((T, E), 0.5, np.float32)
    cfg = moe.config(T, 128, E, k, 128)
    ws = _ws(cfg)
    idx = torch.empty(T, k, dtype=torch.int32, device="cuda")
    g = torch.empty(T, k, dtype=torch.float32, device="cuda")
    moe.moe_topk_gating(cfg, dev_f32(z), idx, g, ws)
    ri, rg = ref.route_from_logits(z.astype(np.float64), k)
    assert np.array_equal(host(idx), ri)
    assert np.max(np.abs(host(g) - rg)) <= 1e-6
    _check_no_device_error(ws)


@pytest.mark.parametrize("T,d,E,k,dtype,bias", [
    (256, 128, 8, 2, "f32", False),       # the tiny fp32 configuration
    (1000, 256, 64, 4, "bf16", True),
    (333, 384, 128, 4, "bf16", False),
    (129, 128, 256, 8, "bf16", True),
    (300, 256, 36, 4, "bf16", False),     # E not a multiple of 8: the CUDA-core router
    (8192, 2048, 8, 4, "bf16", False),    # E below one 64-column MMA tile
])
def test_route_topk(T, d, E, k, dtype, bias):
    import torch
    inp = gen.make_layer_inputs(T, d, E, k, 128, dtype=dtype, seed=7, skew=bias, with_grad=False)
    cfg = moe.config(T, d, E, k, 128, dtype=dtype)
    ws = _ws(cfg)
    logits = torch.empty(T, E, dtype=torch.float32, device="cuda")
    idx = torch.empty(T, k, dtype=torch.int32, device="cuda")
    g = torch.empty(T, k, dtype=torch.float32, device="cuda")
    b = dev_f32(inp.bias) if bias else None
    moe.moe_route_topk(cfg, dev(inp.x, dtype), dev(inp.w_r, dtype), b, logits, idx, g, ws)
    z, p, ri, rg = ref.route(inp.x, inp.w_r, k, inp.bias)
    # fp32 dot products of length d: |error| <= d * 2^-24 * sum_i |x_i w_i| (+ the bias add)
    bound = d * 2.0 ** -24 * (np.abs(inp.x.astype(np.float64)) @ np.abs(inp.w_r.astype(np.float64)))
    bound = bound + 2.0 ** -24 * np.abs(z) + 1e-30
    zg = host(logits)
    assert np.all(np.abs(zg - z) <= bound)
    # routing bit-exact wherever every gap among the k+1 largest oracle logits exceeds
    # twice the token's largest logit error (then set and order must agree)
    zs = np.sort(z, axis=1)[:, ::-1][:, :k + 1]
    delta = np.max(np.abs(zg - z), axis=1)
    clear = np.all(-np.diff(zs, axis=1) > 2 * delta[:, None], axis=1)
    gi = host(idx)
    assert clear.mean() > 0.95
    assert np.array_equal(gi[clear], ri[clear])
    gerr = np.max(np.abs(host(g)[clear] - rg[clear]))
    assert gerr <= 2 * np.max(delta) + 1e-6
    _check_no_device_error(ws)


@pytest.mark.parametrize("T,d,E,k,bias,nan_rows", [
    (1000, 256, 64, 4, True, 0),
    (333, 384, 128, 4, False, 3),
    (129, 128, 256, 8, True, 2),
    (700, 128, 8, 8, False, 0),        # k = E: every expert, in order
    (515, 256, 16, 8, True, 1),
    (300, 128, 192, 6, False, 0),      # the second half of a 256-column tile is ragged
    (2000, 512, 128, 1, False, 0),
    (300, 128, 36, 4, False, 2),       # the CUDA-core router
    (20000, 256, 128, 4, True, 1),     # more 128-token tiles than CTA clusters: several per cluster
])
def test_route_topk_selects_exactly_on_its_own_logits(T, d, E, k, bias, nan_rows):
    """Given the fp32 logits the router wrote, the selection is unique: on every row the
    experts must be the oracle's top k of those logits (larger first, the lower index on
    equal logits, NaN below every number) and the gates their renormalised softmax.  Each
    router column is used by three experts, so exact ties are common."""
    import torch
    inp = gen.make_layer_inputs(T, d, E, k, 128, seed=23, skew=bias, with_grad=False)
    w = np.ascontiguousarray(inp.w_r[:, np.arange(E) // 3])
    x = inp.x.copy()
    bad = (np.arange(nan_rows) * 97) % T
    x[bad, 5] = np.nan
    cfg = moe.config(T, d, E, k, 128)
    ws = _ws(cfg)
    logits = torch.empty(T, E, dtype=torch.float32, device="cuda")
    idx = torch.empty(T, k, dtype=torch.int32, device="cuda")
    g = torch.empty(T, k, dtype=torch.float32, device="cuda")
    b = dev_f32(inp.bias) if bias else None
    moe.moe_route_topk(cfg, dev(x, "bf16"), dev(w, "bf16"), b, logits, idx, g, ws)
    zg = host(logits)
    gi = host(idx)
    assert np.array_equal(gi, ref.topk_experts(zg, k))
    if not bias and E >= 3:
        # exact ties decided the selection on many rows
        zs = np.take_along_axis(zg, gi.astype(np.int64), axis=1)
        assert np.mean(np.any(zs[:, :-1] == zs[:, 1:], axis=1) if k > 1 else zs[:, 0] == zg.max(1)) > 0.5
    fine = ~np.isnan(zg).any(axis=1)
    assert fine.sum() == T - nan_rows
    rg = ref.renormalised_gates(ref.softmax(zg[fine]), gi[fine])
    assert np.max(np.abs(host(g)[fine] - rg)) <= 1e-6
    code = moe.moe_get_error(ws)
    assert code == (moe.MOE_ERR_DEVICE_NAN if nan_rows else 0)


@pytest.mark.parametrize("T,E,k,kind", [
    (1, 1, 1, "uniform"), (3000, 8, 4, "uniform"), (777, 128, 4, "skewed"), (2048, 256, 8, "skewed"),
    (500, 16, 2, "one_expert"), (4097, 128, 4, "uniform"), (16384, 128, 4, "skewed"),
])
def test_build_offsets_bit_exact(T, E, k, kind):
    import torch
    if kind == "uniform":
        idx, _ = gen.uniform_random_routing(T, E, k, seed=T)
    elif kind == "skewed":
        idx = gen.skewed_routing_idx(T, E, k, seed=T)
    else:
        idx = np.tile(np.arange(k, dtype=np.int32), (T, 1))   # experts >= k stay empty
    cfg = moe.config(T, 128, E, k, 128)
    ws = _ws(cfg)
    P = T * k
    counts = torch.empty(E, dtype=torch.int32, device="cuda")
    offsets = torch.empty(E + 1, dtype=torch.int32, device="cuda")
    sop = torch.empty(P, dtype=torch.int32, device="cuda")
    pos = torch.empty(P, dtype=torch.int32, device="cuda")
    moe.moe_build_offsets(cfg, dev_i32(idx), counts, offsets, sop, pos, ws)
    rc, ro, rs, rp = ref.routing_metadata(idx, E)
    assert np.array_equal(host(counts), rc)
    assert np.array_equal(host(offsets), ro)
    assert np.array_equal(host(sop), rs)
    assert np.array_equal(host(pos), rp)
    _check_no_device_error(ws)


def test_build_offsets_flags_out_of_range_index():
    import torch
    T, E, k = 100, 8, 2
    idx, _ = gen.uniform_random_routing(T, E, k, seed=1)
    idx[17, 1] = E          # out of range: the kernels skip it and raise the error bit
    cfg = moe.config(T, 128, E, k, 128)
    ws = _ws(cfg)
    P = T * k
    bufs = [torch.empty(n, dtype=torch.int32, device="cuda") for n in (E, E + 1, P, P)]
    moe.moe_build_offsets(cfg, dev_i32(idx), *bufs, ws)
    assert moe.moe_get_error(ws) & moe.MOE_ERR_DEVICE_INDEX
    assert moe.moe_get_error(ws) == 0      # reading clears it


def test_build_offsets_empty_batch():
    import torch
    cfg = moe.config(0, 128, 8, 2, 128)
    ws = _ws(cfg)
    counts = torch.full((8,), -1, dtype=torch.int32, device="cuda")
    offsets = torch.full((9,), -1, dtype=torch.int32, device="cuda")
    moe.moe_build_offsets(cfg, None, counts, offsets, None, None, ws)
    assert host(counts).tolist() == [0] * 8 and host(offsets).tolist() == [0] * 9


# ------------------------------------------------------------------ row ops

def _routing(T, E, k, seed):
    idx, _ = gen.uniform_random_routing(T, E, k, seed=seed)
    z = gen.normal_logits(T, k, seed=seed + 1)
    g = np.exp(z) / np.exp(z).sum(axis=1, keepdims=True)       # any positive weights will do
    _, _, sop, pos = ref.routing_metadata(idx, E)
    return idx, g.astype(np.float32), sop, pos


@pytest.mark.parametrize("T,d,E,k,dtype", [(37, 128, 8, 1, "bf16"), (1000, 2048, 128, 4, "bf16"),
                                           (256, 128, 8, 2, "f32"), (300, 384, 16, 8, "bf16")])
def test_permute_is_a_bit_copy(T, d, E, k, dtype):
    import torch
    rng = np.random.default_rng(0)
    x = grid(rng.standard_normal((T, d), dtype=np.float32), dtype)
    idx, g, sop, pos = _routing(T, E, k, 3)
    cfg = moe.config(T, d, E, k, 128, dtype=dtype)
    xp = torch.empty(T * k, d, dtype=moe.torch_dtype(cfg), device="cuda")
    moe.moe_permute(cfg, dev(x, dtype), dev_i32(sop), xp)
    assert np.array_equal(host(xp), ref.permute(x, pos, k))


@pytest.mark.parametrize("T,d,E,k,dtype", [(37, 128, 8, 1, "bf16"), (1000, 2048, 128, 4, "bf16"),
                                           (256, 128, 8, 2, "f32"), (300, 384, 16, 8, "bf16")])
def test_combine_and_its_backward(T, d, E, k, dtype):
    import torch
    rng = np.random.default_rng(1)
    P = T * k
    y_perm = grid(rng.standard_normal((P, d), dtype=np.float32), dtype)
    dY = grid(rng.standard_normal((T, d), dtype=np.float32), dtype)
    idx, g, sop, pos = _routing(T, E, k, 5)
    cfg = moe.config(T, d, E, k, 128, dtype=dtype)
    dt = moe.torch_dtype(cfg)
    y = torch.empty(T, d, dtype=dt, device="cuda")
    moe.moe_unpermute_combine(cfg, dev(y_perm, dtype), dev_i32(sop), dev_f32(g), y)
    assert rel_err(host(y), ref.combine(y_perm, sop, g)) <= TOL_COMBINE
    dy_perm = torch.empty(P, d, dtype=dt, device="cuda")
    dgate = torch.empty(T, k, dtype=torch.float32, device="cuda")
    moe.moe_combine_bwd(cfg, dev(dY, dtype), dev(y_perm, dtype), dev_i32(sop), dev_f32(g), dy_perm, dgate)
    r_dyp, r_dg = ref.combine_bwd(dY, y_perm, sop, g)
    assert rel_err(host(dy_perm), r_dyp) <= TOL_COMBINE
    assert rel_err(host(dgate), r_dg) <= 1e-4
    dx = torch.empty(T, d, dtype=dt, device="cuda")
    moe.moe_unpermute_sum(cfg, dev(y_perm, dtype), dev_i32(sop), dx)
    assert rel_err(host(dx), ref.unpermute_sum(y_perm, sop, T, k)) <= TOL_COMBINE


@pytest.mark.parametrize("T,d,E,k,dtype", [(256, 128, 8, 2, "f32"), (1000, 512, 64, 4, "bf16"),
                                           (77, 256, 256, 8, "bf16")])
def test_route_bwd(T, d, E, k, dtype):
    import torch
    inp = gen.make_layer_inputs(T, d, E, k, 128, dtype=dtype, seed=11, with_grad=True)
    z, p, idx, gate = ref.route(inp.x, inp.w_r, k)
    gate32 = gate.astype(np.float32)
    rng = np.random.default_rng(2)
    dgate = rng.standard_normal((T, k)).astype(np.float32)
    dx0 = grid(rng.standard_normal((T, d), dtype=np.float32), dtype)
    cfg = moe.config(T, d, E, k, 128, dtype=dtype)
    ws = _ws(cfg)
    dx = dev(dx0, dtype)
    dwr = torch.empty(d, E, dtype=torch.float32, device="cuda")
    moe.moe_route_bwd(cfg, dev_f32(dgate), dev_f32(gate32), dev_i32(idx), dev(inp.x, dtype),
                      dev(inp.w_r, dtype), dx, dwr, ws)
    dz, r_dwr, r_dx = ref.route_bwd(dgate, gate32, idx, inp.x, inp.w_r)
    assert rel_err(host(dwr), r_dwr) <= 1e-4
    assert rel_err(host(dx), dx0 + r_dx) <= TOL
    _check_no_device_error(ws)


# ------------------------------------------------------------------ grouped GEMMs

GEMM_CASES = [
    # dtype, d, f, E, counts kind
    ("bf16", 256, 256, 8, "random"),
    ("bf16", 128, 128, 4, "random"),
    ("bf16", 384, 256, 3, "one_expert"),
    ("bf16", 512, 384, 16, "random"),
    ("bf16", 256, 512, 1, "tiny"),
    ("f32", 128, 256, 8, "random"),
    ("bf16", 2048, 1024, 8, "random"),
    # large groups: 256-row CTA-pair tiles for the row-grouped GEMMs (P >= 768 E), with an
    # empty expert and tails that leave the second CTA of a pair without rows
    ("bf16", 256, 256, 3, "big"),
    ("bf16", 512, 512, 2, "big2"),
]


def _counts(kind, E, rng):
    if kind == "big":
        return np.array([1000, 0, 1400], np.int64)
    if kind == "big2":
        return np.array([1537, 129], np.int64)
    if kind == "random":
        return random_counts(E, 300, rng)
    if kind == "one_expert":
        c = np.zeros(E, np.int64)
        c[E // 2] = 517
        return c
    return np.array([5] * E, np.int64)


@pytest.mark.parametrize("dtype,d,f,E,kind", GEMM_CASES)
def test_grouped_swiglu_fwd(dtype, d, f, E, kind):
    import torch
    rng = np.random.default_rng(d + f + E)
    counts = _counts(kind, E, rng)
    offsets = offsets_of(counts)
    P = int(offsets[-1])
    x_perm = grid(rng.standard_normal((P, d), dtype=np.float32), dtype)
    sd = 1.0 / np.sqrt(d)
    wg = grid(sd * rng.standard_normal((E, d, f), dtype=np.float32), dtype)
    wu = grid(sd * rng.standard_normal((E, d, f), dtype=np.float32), dtype)
    wd = grid((1.0 / np.sqrt(f)) * rng.standard_normal((E, f, d), dtype=np.float32), dtype)
    # P rows, k = 1 view: the grouped call only looks at P = T*k
    cfg = moe.config(P, d, E, 1, f, dtype=dtype)
    ws = _ws(cfg)
    dt = moe.torch_dtype(cfg)
    hu = torch.empty(P, 2 * f, dtype=dt, device="cuda")
    a = torch.empty(P, f, dtype=dt, device="cuda")
    y = torch.empty(P, d, dtype=dt, device="cuda")
    moe.moe_grouped_swiglu_fwd(cfg, dev(x_perm, dtype), dev_i32(offsets), dev(wg, dtype), dev(wu, dtype),
                               dev(wd, dtype), hu, a, y, ws)
    torch.cuda.synchronize()
    h, u, ra, ry = ref.grouped_swiglu(x_perm, offsets, wg, wu, wd)
    ghu = host(hu)
    assert rel_err(ghu[:, :f], h) <= TOL
    assert rel_err(ghu[:, f:], u) <= TOL
    assert rel_err(host(a), ra) <= TOL
    assert rel_err(host(y), ry) <= TOL
    _check_no_device_error(ws)


@pytest.mark.parametrize("dtype,d,f,E,kind", GEMM_CASES)
def test_grouped_swiglu_bwd(dtype, d, f, E, kind):
    import torch
    rng = np.random.default_rng(d * 3 + f + E)
    counts = _counts(kind, E, rng)
    offsets = offsets_of(counts)
    P = int(offsets[-1])
    x_perm = grid(rng.standard_normal((P, d), dtype=np.float32), dtype)
    dy = grid(rng.standard_normal((P, d), dtype=np.float32), dtype)
    h = grid(rng.standard_normal((P, f), dtype=np.float32), dtype)
    u = grid(rng.standard_normal((P, f), dtype=np.float32), dtype)
    a = grid(rng.standard_normal((P, f), dtype=np.float32), dtype)
    sd = 1.0 / np.sqrt(d)
    wg = grid(sd * rng.standard_normal((E, d, f), dtype=np.float32), dtype)
    wu = grid(sd * rng.standard_normal((E, d, f), dtype=np.float32), dtype)
    wd = grid((1.0 / np.sqrt(f)) * rng.standard_normal((E, f, d), dtype=np.float32), dtype)
    cfg = moe.config(P, d, E, 1, f, dtype=dtype)
    ws = _ws(cfg)
    dt = moe.torch_dtype(cfg)
    if dtype == "f32":
        # tf32 tensor-core operands are K-major only; the token-reduction GEMMs are not offered
        z = torch.zeros(16, dtype=torch.float32, device="cuda")
        with pytest.raises(moe.MoeError) as ex:
            moe.moe_grouped_swiglu_bwd(cfg, z, z, z, z, dev_i32(offsets), z, z, z, z, z, z, z, z, ws)
        assert ex.value.code == moe.MOE_ERR_UNSUPPORTED
        return
    dhu = torch.empty(P, 2 * f, dtype=dt, device="cuda")
    dxp = torch.empty(P, d, dtype=dt, device="cuda")
    dwg = torch.full((E, d, f), 7.0, dtype=dt, device="cuda")   # must be overwritten (zeros for empty experts)
    dwu = torch.full((E, d, f), 7.0, dtype=dt, device="cuda")
    dwd = torch.full((E, f, d), 7.0, dtype=dt, device="cuda")
    moe.moe_grouped_swiglu_bwd(cfg, dev(dy, dtype), dev(x_perm, dtype),
                               dev(np.concatenate([h, u], axis=1), dtype), dev(a, dtype), dev_i32(offsets),
                               dev(wg, dtype), dev(wu, dtype), dev(wd, dtype), dhu, dxp, dwg, dwu, dwd, ws)
    torch.cuda.synchronize()
    r = ref.grouped_swiglu_bwd(dy, x_perm, h, u, a, offsets, wg, wu, wd)
    g = host(dhu)
    assert rel_err(g[:, :f], r["dh"]) <= TOL
    assert rel_err(g[:, f:], r["du"]) <= TOL
    assert rel_err(host(dxp), r["dx_perm"]) <= TOL
    assert rel_err(host(dwg), r["dw_gate"]) <= TOL
    assert rel_err(host(dwu), r["dw_up"]) <= TOL
    assert rel_err(host(dwd), r["dw_down"]) <= TOL
    for e in np.nonzero(counts == 0)[0]:
        assert np.all(host(dwg[e]) == 0) and np.all(host(dwd[e]) == 0)
    _check_no_device_error(ws)
