"""The C-ABI library loads and exports every symbol include/moe.h declares; host-side
argument validation rejects bad calls before any CUDA call (CPU only, no GPU needed)."""
import ctypes
import os
import re

import pytest

import routing_grouped_expert_softmax_b200 as moe
from routing_grouped_expert_softmax_b200 import build as moe_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    src = open(os.path.join(ROOT, "include", "moe.h")).read()
    return sorted(set(re.findall(r"MOE_API\s+\w+\s+(moe_\w+)\s*\(", src)))


@pytest.fixture(scope="module")
def lib():
    moe_build.build()
    return moe.lib()


def test_every_declared_symbol_is_exported(lib):
    names = _declared()
    assert len(names) >= 15
    for n in names:
        assert hasattr(lib, n), n
    assert sorted(moe.EXPORTED) == names


def test_no_unresolved_library_symbols():
    # every internal launcher the C ABI calls is defined inside the library
    import subprocess
    out = subprocess.run(["nm", "-D", "--undefined-only", moe.LIB_PATH], capture_output=True, text=True).stdout
    assert "moe" not in out, out


def test_workspace_size_is_host_only(lib):
    cfg = moe.config(8192, 2048, 128, 4, 1024)
    ws = moe.moe_workspace_size(cfg)
    assert ws >= 256 and ws % 256 == 0
    assert moe.moe_workspace_size(moe.config(0, 128, 8, 2, 256)) >= 256


@pytest.mark.parametrize("bad", [
    dict(T=-1), dict(d=0), dict(E=0), dict(k=0), dict(f=-5), dict(dtype=7), dict(prec=9),
])
def test_invalid_config_rejected(lib, bad):
    base = dict(T=16, d=128, E=8, k=2, f=128, dtype=moe.MOE_BF16, prec=moe.MOE_PREC_NATIVE)
    base.update(bad)
    cfg = moe.MoeConfig(**base)
    rc = lib.moe_permute(ctypes.byref(cfg), 16, 16, 16, None)
    assert rc == moe.MOE_ERR_INVALID_ARG


@pytest.mark.parametrize("bad", [dict(E=257), dict(k=9), dict(k=9, E=8), dict(d=192), dict(f=200),
                                 dict(prec=moe.MOE_PREC_MXFP8, dtype=moe.MOE_F32)])
def test_unsupported_config_rejected(lib, bad):
    base = dict(T=16, d=128, E=8, k=2, f=128, dtype=moe.MOE_BF16, prec=moe.MOE_PREC_NATIVE)
    base.update(bad)
    cfg = moe.MoeConfig(**base)
    assert lib.moe_permute(ctypes.byref(cfg), 16, 16, 16, None) == moe.MOE_ERR_UNSUPPORTED


def test_null_and_misaligned_pointers_rejected(lib):
    cfg = moe.config(16, 128, 8, 2, 128)
    assert lib.moe_permute(ctypes.byref(cfg), None, 16, 16, None) == moe.MOE_ERR_INVALID_ARG
    assert lib.moe_permute(ctypes.byref(cfg), 16, 16, 24, None) == moe.MOE_ERR_INVALID_ARG
    assert lib.moe_build_offsets(ctypes.byref(cfg), 16, 16, 16, 16, 16, None, None) == moe.MOE_ERR_WORKSPACE
    code = ctypes.c_int32()
    assert lib.moe_get_error(None, None, ctypes.byref(code)) == moe.MOE_ERR_INVALID_ARG


def test_empty_batch_launches_nothing(lib):
    # T = 0 returns MOE_OK before any launch, so it is valid even without a GPU
    cfg = moe.config(0, 128, 8, 2, 128)
    assert lib.moe_permute(ctypes.byref(cfg), None, None, None, None) == moe.MOE_OK
    assert lib.moe_unpermute_combine(ctypes.byref(cfg), None, None, None, None, None) == moe.MOE_OK


def test_partial_shared_expert_rejected_on_host(lib):
    # shared gate and up given, down missing: rejected before anything is launched
    cfg = moe.config(16, 128, 8, 2, 128)
    w = moe.LayerWeights(16, None, 16, 16, 16, 16, 16, None)
    sv = moe.LayerSaved(*([16] * len(moe.SAVED_FIELDS)))
    gr = moe.LayerGrads(*([16] * len(moe.GRAD_FIELDS)))
    assert lib.moe_layer_fwd(ctypes.byref(cfg), ctypes.byref(w), 16, 16, ctypes.byref(sv), 16, None) \
        == moe.MOE_ERR_INVALID_ARG
    assert lib.moe_layer_bwd(ctypes.byref(cfg), ctypes.byref(w), 16, 16, ctypes.byref(sv), ctypes.byref(gr),
                             16, None) == moe.MOE_ERR_INVALID_ARG


def test_permute_mxfp8_host_validation(lib):
    cfg = moe.config(16, 128, 8, 2, 128)
    bound = 16 * 2 + 127 * 8
    ok = (ctypes.byref(cfg), 16, 16, 16, 16, bound, 16, 16, None)
    # fp32 storage has no MXFP8 path
    c32 = moe.config(16, 128, 8, 2, 128, dtype="f32")
    assert lib.moe_permute_mxfp8(ctypes.byref(c32), *ok[1:]) == moe.MOE_ERR_UNSUPPORTED
    # the padded buffers must hold T*k + 127*E rows
    assert lib.moe_permute_mxfp8(ctypes.byref(cfg), 16, 16, 16, 16, bound - 1, 16, 16, None) \
        == moe.MOE_ERR_INVALID_ARG
    # x, x_perm and codes move as 16-byte vectors
    assert lib.moe_permute_mxfp8(ctypes.byref(cfg), 24, 16, 16, 16, bound, 16, 16, None) == moe.MOE_ERR_INVALID_ARG
    assert lib.moe_permute_mxfp8(ctypes.byref(cfg), 16, 16, 16, 16, bound, 8, 16, None) == moe.MOE_ERR_INVALID_ARG
    assert lib.moe_permute_mxfp8(ctypes.byref(cfg), 16, 16, None, 16, bound, 16, 16, None) \
        == moe.MOE_ERR_INVALID_ARG
    # an empty batch launches nothing
    c0 = moe.config(0, 128, 8, 2, 128)
    assert lib.moe_permute_mxfp8(ctypes.byref(c0), None, None, None, None, 0, None, None, None) == moe.MOE_OK


def test_mx_quantize_cols_alignment(lib):
    assert lib.moe_mx_quantize_cols(24, 64, 64, None, 0, 64, 16, 16, None) == moe.MOE_ERR_INVALID_ARG
    assert lib.moe_mx_quantize_cols(16, 64, 64, None, 0, 64, 16, 6, None) == moe.MOE_ERR_INVALID_ARG
    assert lib.moe_mx_quantize_cols(16, 64, 48, None, 0, 64, 16, 16, None) == moe.MOE_ERR_INVALID_ARG


def test_shared_expert_and_recompute_host_validation(lib):
    cfg = moe.config(16, 128, 8, 2, 128)
    w = moe.LayerWeights(16, None, 16, 16, 16, 16, 16, 16)      # a complete shared expert
    fields = {n: 16 for n in moe.SAVED_FIELDS}
    fields["shared_a"] = None                                     # ... but no room for its a
    sv = moe.LayerSaved(*[fields[n] for n in moe.SAVED_FIELDS])
    assert lib.moe_layer_fwd(ctypes.byref(cfg), ctypes.byref(w), 16, 16, ctypes.byref(sv), 16, None) \
        == moe.MOE_ERR_INVALID_ARG
    # recompute: hu may be NULL but, when given, must be 16-byte aligned
    fields = {n: 16 for n in moe.SAVED_FIELDS}
    fields["hu"] = 24
    sv = moe.LayerSaved(*[fields[n] for n in moe.SAVED_FIELDS])
    w0 = moe.LayerWeights(16, None, 16, 16, 16, None, None, None)
    assert lib.moe_layer_fwd(ctypes.byref(cfg), ctypes.byref(w0), 16, 16, ctypes.byref(sv), 16, None) \
        == moe.MOE_ERR_INVALID_ARG


def test_debug_stall_hook_validates_its_limit(lib):
    # host only: the hook is a process-wide setting read at the next launch
    assert lib.moe_debug_set_gemm_stall_ns(2_000_000_000) == moe.MOE_ERR_INVALID_ARG
    assert lib.moe_debug_set_gemm_stall_ns(1_000_000) == moe.MOE_OK
    assert lib.moe_debug_set_gemm_stall_ns(0) == moe.MOE_OK


def test_dispatch_mxfp8_host_validation(lib):
    cfg = moe.config(16, 128, 8, 2, 128)
    bound = 16 * 2 + 127 * 8
    # (cfg, x, pair_of_slot, offsets, rows_bound, x_perm, codes_r, scales_r, codes_c, scales_c, stream)
    c32 = moe.config(16, 128, 8, 2, 128, dtype="f32")
    assert lib.moe_dispatch_mxfp8(ctypes.byref(c32), 16, 16, 16, bound, None, 16, 16, 16, 16, None) \
        == moe.MOE_ERR_UNSUPPORTED
    assert lib.moe_dispatch_mxfp8(ctypes.byref(cfg), 16, 16, 16, bound - 1, None, 16, 16, 16, 16, None) \
        == moe.MOE_ERR_INVALID_ARG
    assert lib.moe_dispatch_mxfp8(ctypes.byref(cfg), 16, 16, 16, bound, 24, 16, 16, 16, 16, None) \
        == moe.MOE_ERR_INVALID_ARG                                   # x_perm, when given, 16-byte aligned
    assert lib.moe_dispatch_mxfp8(ctypes.byref(cfg), 16, 16, 16, bound, None, None, 16, 16, 16, None) \
        == moe.MOE_ERR_INVALID_ARG                                   # both orientations are outputs
    assert lib.moe_dispatch_mxfp8(ctypes.byref(cfg), 16, 16, 16, bound, None, 16, 16, 16, 6, None) \
        == moe.MOE_ERR_INVALID_ARG                                   # scales 4-byte aligned
    c0 = moe.config(0, 128, 8, 2, 128)
    assert lib.moe_dispatch_mxfp8(ctypes.byref(c0), None, None, None, 0, None, None, None, None, None, None) \
        == moe.MOE_OK
    # (cfg, dy, y_perm, pair_of_slot, offsets, topk_gate, rows_bound, dy_perm, dgate, codes_r, scales_r,
    #  codes_c, scales_c, stream)
    assert lib.moe_combine_bwd_mxfp8(ctypes.byref(c32), 16, 16, 16, 16, 16, bound, None, 16, 16, 16, 16, 16,
                                     None) == moe.MOE_ERR_UNSUPPORTED
    assert lib.moe_combine_bwd_mxfp8(ctypes.byref(cfg), 16, 16, 16, 16, 16, bound - 1, None, 16, 16, 16, 16, 16,
                                     None) == moe.MOE_ERR_INVALID_ARG
    assert lib.moe_combine_bwd_mxfp8(ctypes.byref(cfg), 16, 16, 16, 16, 16, bound, None, None, 16, 16, 16, 16,
                                     None) == moe.MOE_ERR_INVALID_ARG  # dgate is an output
    assert lib.moe_combine_bwd_mxfp8(ctypes.byref(c0), None, None, None, None, None, 0, None, None, None, None,
                                     None, None, None) == moe.MOE_OK


def test_layer_bf16_rows_are_optional_only_in_mxfp8(lib):
    w = moe.LayerWeights(16, None, 16, 16, 16, None, None, None)
    # bf16 layer: x_perm is required
    cfg = moe.config(16, 128, 8, 2, 128)
    fields = {n: 16 for n in moe.SAVED_FIELDS}
    fields["x_perm"] = None
    fields["mx_saved"] = None
    sv = moe.LayerSaved(*[fields[n] for n in moe.SAVED_FIELDS])
    assert lib.moe_layer_fwd(ctypes.byref(cfg), ctypes.byref(w), 16, 16, ctypes.byref(sv), 16, None) \
        == moe.MOE_ERR_INVALID_ARG
    # MXFP8 without the saved copies: the forward writes x_perm, so it is required too
    cmx = moe.config(16, 128, 8, 2, 128, prec="mxfp8")
    assert lib.moe_layer_fwd(ctypes.byref(cmx), ctypes.byref(w), 16, 16, ctypes.byref(sv), 16, None) \
        == moe.MOE_ERR_INVALID_ARG
    # bf16 backward: dy_perm is required (MXFP8 keeps it in MXFP8 only)
    fields = {n: 16 for n in moe.SAVED_FIELDS}
    sv = moe.LayerSaved(*[fields[n] for n in moe.SAVED_FIELDS])
    gf = {n: 16 for n in moe.GRAD_FIELDS}
    gf["dy_perm"] = None
    for n in ("dw_shared_gate", "dw_shared_up", "dw_shared_down", "shared_dhu"):
        gf[n] = None
    g = moe.LayerGrads(*[gf[n] for n in moe.GRAD_FIELDS])
    assert lib.moe_layer_bwd(ctypes.byref(cfg), ctypes.byref(w), 16, 16, ctypes.byref(sv), ctypes.byref(g), 16,
                             None) == moe.MOE_ERR_INVALID_ARG
