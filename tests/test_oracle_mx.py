"""Pins for the oracle's MXFP8 quantiser and MXFP8 expert FFN (CPU only).

Against: the OCP FP8 spec's code table (tests/golden/e4m3_ocp.txt), the
ml_dtypes / torch float8_e4m3fn conversions (library round-to-nearest-even),
the OCP MX scale rule's special cases, exact round trips of values already on
the MX grid, and the quantisation error bound.
"""
import os

import ml_dtypes
import numpy as np
import pytest
import torch

from oracle import moe_ref as ref
from routing_grouped_expert_softmax_b200 import inputs as gen

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "e4m3_ocp.txt")


def _golden_pairs():
    pairs = []
    for line in open(GOLDEN):
        line = line.split("#")[0].strip()
        if line:
            c, v = line.split()
            pairs.append((int(c, 16), float(v)))
    return pairs


def test_bf16_rne_matches_torch():
    rng = np.random.default_rng(9)
    v = np.concatenate([rng.standard_normal(50000) * 10.0 ** rng.integers(-20, 20, 50000),
                        [0.0, -0.0, 1.0, 1.00390625, 1.01171875, 65504.0]])
    want = torch.from_numpy(v.astype(np.float32)).to(torch.bfloat16).to(torch.float64).numpy()
    np.testing.assert_array_equal(ref.bf16_rne(v), want)


def test_e4m3_codes_match_ocp_table():
    for code, val in _golden_pairs():
        got = ref.e4m3_value(code)
        assert got == val and np.signbit(got) == np.signbit(val)
        codes, vals = ref.round_to_e4m3(np.array([val]))
        assert codes[0] == code
    assert np.isnan(ref.e4m3_value(0x7F)) and np.isnan(ref.e4m3_value(0xFF))


def test_e4m3_grid_matches_ml_dtypes_decoding():
    codes = np.arange(0x7F, dtype=np.uint8)
    lib = codes.view(ml_dtypes.float8_e4m3fn).astype(np.float64)
    np.testing.assert_array_equal(ref.e4m3_grid(), lib)


def test_rounding_matches_library_conversion_in_range():
    rng = np.random.default_rng(0)
    v = np.concatenate([rng.standard_normal(20000) * s for s in (1e-3, 0.05, 1.0, 30.0, 150.0)])
    v = v[np.abs(v) <= 448.0]
    # also every midpoint between neighbouring grid values (the ties)
    g = ref.e4m3_grid()
    mids = (g[:-1] + g[1:]) / 2
    v = np.concatenate([v, mids, -mids, g, -g])
    codes, vals = ref.round_to_e4m3(v)
    lib = v.astype(np.float32).astype(ml_dtypes.float8_e4m3fn)
    np.testing.assert_array_equal(codes, lib.view(np.uint8))
    t = torch.from_numpy(v.astype(np.float32)).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    np.testing.assert_array_equal(codes, t)


def test_saturation_to_448():
    codes, vals = ref.round_to_e4m3(np.array([449.0, 464.0, 500.0, 1e6, -1e6]))
    assert codes.tolist() == [0x7E, 0x7E, 0x7E, 0x7E, 0xFE]
    assert vals.tolist() == [448.0, 448.0, 448.0, 448.0, -448.0]


def test_scale_rule_special_cases():
    # X = 2^(floor(log2 amax) - 8); amax in [256, 512) -> X = 1; amax = 1 -> X = 2^-8
    assert ref.mx_scale_exponent(np.array([256.0, 511.0, 1.0, 1.5, 0.0])).tolist() == [0, 0, -8, -8, -127]
    assert ref.mx_scale_exponent(np.array([2.0 ** 200])).tolist() == [127]
    v = np.zeros((1, 32))
    codes, scales, deq = ref.mx_quantize(v, axis=1)
    assert scales.tolist() == [[0]] and np.all(codes == 0) and np.all(deq == 0)


def test_values_on_the_mx_grid_round_trip_exactly():
    rng = np.random.default_rng(1)
    g = ref.e4m3_grid()
    # each block: grid values with the block's max forced into [256, 448] so X = 2^s exactly
    blocks = rng.choice(g, size=(64, 32)) * rng.choice([-1.0, 1.0], size=(64, 32))
    blocks[:, 0] = rng.choice(g[(g >= 256)], size=64)
    s = rng.integers(-20, 20, size=(64, 1))
    v = blocks * np.ldexp(1.0, s)
    codes, scales, deq = ref.mx_quantize(v, axis=1)
    np.testing.assert_array_equal(deq, v)
    np.testing.assert_array_equal(scales[:, 0].astype(np.int64) - 127, s[:, 0])
    np.testing.assert_array_equal(ref.mx_dequantize(codes, scales, axis=1), v)


def test_quantisation_error_bound():
    # normal-range elements: |q - v| <= 2^-4 |v|; below 2^-6 X: |q - v| <= 2^-10 X
    rng = np.random.default_rng(2)
    v = rng.standard_normal((256, 64)) * np.exp(rng.standard_normal((256, 1)) * 3)
    codes, scales, deq = ref.mx_quantize(v, axis=1)
    X = np.repeat(np.ldexp(1.0, scales.astype(np.int64) - 127), 32, axis=1)
    err = np.abs(deq - v)
    # the rule puts each block's amax in [256, 512) X, so elements above 448 X saturate
    sat = np.abs(v) > 448.0 * X
    assert np.all(np.abs(deq[sat]) == 448.0 * X[sat])
    normal = (np.abs(v) >= X * 2.0 ** -6) & ~sat
    sub = np.abs(v) < X * 2.0 ** -6
    assert np.all(err[normal] <= 2.0 ** -4 * np.abs(v[normal]) * (1 + 1e-12))
    assert np.all(err[sub] <= 2.0 ** -10 * X[sub] * (1 + 1e-12))
    # the block maximum never saturates by more than the rounding step near 448
    assert np.all(np.abs(deq) <= 448.0 * X)


def test_quantise_along_axis_0_equals_transposed_axis_1():
    v = np.random.default_rng(3).standard_normal((64, 5))
    c0, s0, d0 = ref.mx_quantize(v, axis=0)
    c1, s1, d1 = ref.mx_quantize(v.T, axis=1)
    np.testing.assert_array_equal(c0, c1.T)
    np.testing.assert_array_equal(s0, s1.T)


def test_grouped_rows_padding_is_neutral():
    v = np.random.default_rng(4).standard_normal((70, 8))
    offsets = np.array([0, 32, 32, 70])           # groups of 32, 0 and 38 rows
    out = ref.mx_quantize_grouped_rows(v, offsets)
    np.testing.assert_array_equal(out[:32], ref.mx_quantize(v[:32], axis=0)[2])
    pad = np.zeros((64, 8))
    pad[:38] = v[32:]
    np.testing.assert_array_equal(out[32:], ref.mx_quantize(pad, axis=0)[2][:38])


def test_mx_ffn_equals_exact_ffn_on_grid_inputs():
    # x and weights on the MX grid: GEMM-1 outputs (h, u) must equal the exact FFN's
    rng = np.random.default_rng(5)
    g = ref.e4m3_grid()
    E, d, f, P = 3, 64, 32, 40

    def grid(shape, axis):
        v = rng.choice(g, size=shape) * rng.choice([-1.0, 1.0], size=shape)
        v = np.moveaxis(v, axis, -1).copy()
        v[..., ::32] = 448.0                       # fix each block's scale at 2^0
        return np.moveaxis(v, -1, axis) * 2.0 ** -10

    x = grid((P, d), 1)
    wg, wu = grid((E, d, f), 1), grid((E, d, f), 1)
    wd = grid((E, f, d), 1)
    offsets = np.array([0, 10, 10, 40])
    h, u, a, y = ref.grouped_swiglu_mx(x, offsets, wg, wu, wd)
    h0, u0, a0, y0 = ref.grouped_swiglu(x, offsets, wg, wu, wd)
    np.testing.assert_array_equal(h, h0)
    np.testing.assert_array_equal(u, u0)
    # GEMM 2 quantises a: the result stays within the MX error bound of the exact FFN
    assert np.max(np.abs(y - y0)) <= (2.0 ** -4 + 2.0 ** -8) * np.sum(np.abs(a0)[:, :, None] * np.abs(
        wd[np.searchsorted(offsets, np.arange(P), side="right") - 1]), axis=1).max() + 1e-300


def _diag_grid(shape, rng):
    """Values on the E4M3 grid times 2^-10, with 448 * 2^-10 on every position whose
    last two indices agree mod 32: each 32-block along either of the last two axes
    then has scale 2^-10 and quantises exactly."""
    g = ref.e4m3_grid()
    v = rng.choice(g[g <= 256], size=shape) * rng.choice([-1.0, 1.0], size=shape)
    i = np.arange(shape[-2])[:, None] % 32
    j = np.arange(shape[-1])[None, :] % 32
    v = np.where(i == j, 448.0, v)
    return v * 2.0 ** -10


def test_mx_backward_on_grid_inputs():
    rng = np.random.default_rng(6)
    E, d, f, P = 3, 64, 32, 96
    offsets = np.array([0, 32, 32, 96])          # groups on 32-row boundaries
    x = _diag_grid((P, d), rng)
    a = _diag_grid((P, f), rng)
    dy = _diag_grid((P, d), rng)
    h = rng.standard_normal((P, f))
    u = rng.standard_normal((P, f))
    wg = rng.standard_normal((E, d, f)) * 0.1
    wu = rng.standard_normal((E, d, f)) * 0.1
    wd = _diag_grid((E, f, d), rng)
    exact = ref.grouped_swiglu_bwd(dy, x, h, u, a, offsets, wg, wu, wd)
    mx = ref.grouped_swiglu_bwd_mx(dy, x, h, u, a, offsets, wg, wu, wd)
    # operands already on the grid along their reduction axes: exact
    for n in ("dh", "du", "dw_down"):
        np.testing.assert_array_equal(mx[n], exact[n], err_msg=n)
    # [dh|du] and the gate/up weights are not on the grid: a-priori bound.  A quantised
    # element is off by at most 1/7 of its magnitude (saturation of [448, 512) X to 448 X)
    # plus 2^-10 X below the normal range; the grid operand x is exact.
    dhu = np.concatenate([exact["dh"], exact["du"]], axis=1)
    wgu = np.concatenate([wg, wu], axis=2)
    for e in range(E):
        lo, hi = offsets[e], offsets[e + 1]
        if hi == lo:
            continue
        # (+ 2^-8 for the bf16 rounding of [dh | du] before it is quantised)
        bx = (np.abs(dhu[lo:hi]) @ np.abs(wgu[e]).T) * (2 / 7 + 1 / 49 + 2 ** -8 * 1.5) + 1e-9
        assert np.all(np.abs(mx["dx_perm"][lo:hi] - exact["dx_perm"][lo:hi]) <= bx)
        bw = (np.abs(x[lo:hi]).T @ np.abs(dhu[lo:hi])) * (1 / 7 + 2 ** -8 * 1.2) + 1e-9
        got = np.concatenate([mx["dw_gate"][e], mx["dw_up"][e]], axis=1)
        want = np.concatenate([exact["dw_gate"][e], exact["dw_up"][e]], axis=1)
        assert np.all(np.abs(got - want) <= bw)
    assert np.max(np.abs(mx["dx_perm"] - exact["dx_perm"])) > 0     # quantisation did happen
