"""Python binding of libmoe, the B200 (sm_100a) MoE layer-step library.

Argument marshalling only: every call passes device pointers and a CUDA stream to the
C ABI declared in include/moe.h, and every step of the layer runs in libmoe's CUDA
kernels.  There is no CPU path: if libmoe.so has not been built, or no GPU is
present, the calls raise.

Tensors are torch tensors (used only as device memory); any argument may also be a raw
integer device address.  Streams default to torch's current stream.
"""
from __future__ import annotations

import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmoe.so")

# status codes (enum moe_status)
MOE_OK = 0
MOE_ERR_INVALID_ARG = 1
MOE_ERR_UNSUPPORTED = 2
MOE_ERR_WORKSPACE = 3
MOE_ERR_CUDA = 4
MOE_ERR_DEVICE_INDEX = 16
MOE_ERR_DEVICE_TIMEOUT = 32
MOE_ERR_DEVICE_NAN = 64

MOE_F32 = 0
MOE_BF16 = 1
MOE_PREC_NATIVE = 0
MOE_PREC_MXFP8 = 1

EXPORTED = [
    "moe_workspace_size", "moe_get_error", "moe_route_topk", "moe_topk_gating",
    "moe_build_offsets", "moe_build_offsets_noalloc", "moe_permute", "moe_grouped_swiglu_fwd", "moe_grouped_swiglu_bwd",
    "moe_unpermute_combine", "moe_combine_bwd", "moe_unpermute_sum", "moe_route_bwd",
    "moe_layer_fwd", "moe_layer_fwd_routed", "moe_layer_bwd", "moe_mx_quantize_rows",
    "moe_mx_quantize_cols", "moe_permute_mxfp8", "moe_debug_set_gemm_stall_ns", "moe_mx_saved_bytes",
    "moe_dispatch_mxfp8", "moe_combine_bwd_mxfp8",
]


class MoeConfig(ctypes.Structure):
    _fields_ = [("T", ctypes.c_int64), ("d", ctypes.c_int32), ("E", ctypes.c_int32),
                ("k", ctypes.c_int32), ("f", ctypes.c_int32), ("dtype", ctypes.c_int32),
                ("prec", ctypes.c_int32)]

    @property
    def P(self) -> int:
        return self.T * self.k


WEIGHT_FIELDS = ("w_router", "bias", "w_gate", "w_up", "w_down", "w_shared_gate", "w_shared_up",
                 "w_shared_down")
SAVED_FIELDS = ("logits", "topk_idx", "topk_gate", "counts", "offsets", "slot_of_pair",
                "pair_of_slot", "x_perm", "hu", "a", "y_perm", "shared_hu", "shared_a", "mx_saved")
GRAD_FIELDS = ("dx", "dw_router", "dw_gate", "dw_up", "dw_down", "dy_perm", "dgate", "dhu",
               "dx_perm", "dw_shared_gate", "dw_shared_up", "dw_shared_down", "shared_dhu")


class LayerWeights(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in WEIGHT_FIELDS]


class LayerSaved(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in SAVED_FIELDS]


class LayerGrads(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in GRAD_FIELDS]


class MoeError(RuntimeError):
    def __init__(self, name: str, code: int):
        super().__init__(f"{name} failed with status {code}")
        self.code = code


_lib = None
_P = ctypes.c_void_p
_CFG = ctypes.POINTER(MoeConfig)


def lib() -> ctypes.CDLL:
    """Load libmoe.so (built in-tree by routing_grouped_expert_softmax_b200.build)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is not built; run python -m "
                               "routing_grouped_expert_softmax_b200.build")
        L = ctypes.CDLL(LIB_PATH)
        sig = {
            "moe_workspace_size": (ctypes.c_size_t, [_CFG]),
            "moe_mx_saved_bytes": (ctypes.c_size_t, [_CFG]),
            "moe_get_error": (ctypes.c_int, [_P, _P, ctypes.POINTER(ctypes.c_int32)]),
            "moe_debug_set_gemm_stall_ns": (ctypes.c_int, [ctypes.c_uint64]),
            "moe_route_topk": (ctypes.c_int, [_CFG, _P, _P, _P, _P, _P, _P, _P, _P]),
            "moe_topk_gating": (ctypes.c_int, [_CFG, _P, _P, _P, _P, _P]),
            "moe_build_offsets": (ctypes.c_int, [_CFG, _P, _P, _P, _P, _P, _P, _P]),
            "moe_build_offsets_noalloc": (ctypes.c_int, [_CFG, _P, _P, _P, _P, _P, _P]),
            "moe_permute": (ctypes.c_int, [_CFG, _P, _P, _P, _P]),
            "moe_grouped_swiglu_fwd": (ctypes.c_int, [_CFG] + [_P] * 10),
            "moe_grouped_swiglu_bwd": (ctypes.c_int, [_CFG] + [_P] * 15),
            "moe_unpermute_combine": (ctypes.c_int, [_CFG, _P, _P, _P, _P, _P]),
            "moe_combine_bwd": (ctypes.c_int, [_CFG, _P, _P, _P, _P, _P, _P, _P]),
            "moe_unpermute_sum": (ctypes.c_int, [_CFG, _P, _P, _P, _P]),
            "moe_route_bwd": (ctypes.c_int, [_CFG] + [_P] * 9),
            "moe_mx_quantize_rows": (ctypes.c_int, [_P, ctypes.c_int64, ctypes.c_int32, _P, ctypes.c_int32,
                                                    ctypes.c_int64, _P, _P, _P]),
            "moe_mx_quantize_cols": (ctypes.c_int, [_P, ctypes.c_int64, ctypes.c_int32, _P, ctypes.c_int32,
                                                    ctypes.c_int64, _P, _P, _P]),
            "moe_permute_mxfp8": (ctypes.c_int, [_CFG, _P, _P, _P, _P, ctypes.c_int64, _P, _P, _P]),
            "moe_dispatch_mxfp8": (ctypes.c_int, [_CFG, _P, _P, _P, ctypes.c_int64, _P, _P, _P, _P, _P, _P]),
            "moe_combine_bwd_mxfp8": (ctypes.c_int, [_CFG, _P, _P, _P, _P, _P, ctypes.c_int64, _P, _P, _P, _P,
                                                     _P, _P, _P]),
            "moe_layer_fwd": (ctypes.c_int, [_CFG, ctypes.POINTER(LayerWeights), _P, _P,
                                             ctypes.POINTER(LayerSaved), _P, _P]),
            "moe_layer_fwd_routed": (ctypes.c_int, [_CFG, ctypes.POINTER(LayerWeights), _P, _P,
                                                    ctypes.POINTER(LayerSaved), _P, _P]),
            "moe_layer_bwd": (ctypes.c_int, [_CFG, ctypes.POINTER(LayerWeights), _P, _P,
                                             ctypes.POINTER(LayerSaved),
                                             ctypes.POINTER(LayerGrads), _P, _P]),
        }
        for name, (res, args) in sig.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _lib = L
    return _lib


def ptr(t):
    """Device address of a tensor (or None / a raw integer address)."""
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def stream_handle(s=None):
    if s is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(s, int):
        return s
    return s.cuda_stream


def _call(name, *args):
    rc = getattr(lib(), name)(*args)
    if rc != MOE_OK:
        raise MoeError(name, rc)


def config(T, d, E, k, f, dtype="bf16", prec="native") -> MoeConfig:
    return MoeConfig(T, d, E, k, f, MOE_BF16 if dtype == "bf16" else MOE_F32,
                     MOE_PREC_NATIVE if prec == "native" else MOE_PREC_MXFP8)


def moe_workspace_size(cfg: MoeConfig) -> int:
    return lib().moe_workspace_size(ctypes.byref(cfg))


def moe_mx_saved_bytes(cfg: MoeConfig) -> int:
    return lib().moe_mx_saved_bytes(ctypes.byref(cfg))


def moe_get_error(ws, stream=None) -> int:
    code = ctypes.c_int32(0)
    _call("moe_get_error", ptr(ws), stream_handle(stream), ctypes.byref(code))
    return code.value


def moe_debug_set_gemm_stall_ns(ns: int):
    """Failure-detection test hook: later single-CTA grouped GEMM launches wait up to ns on a
    barrier nothing arrives on and take their abort path (0 turns it off)."""
    _call("moe_debug_set_gemm_stall_ns", ns)


def moe_route_topk(cfg, x, w_router, bias, logits, topk_idx, topk_gate, ws, stream=None):
    _call("moe_route_topk", ctypes.byref(cfg), ptr(x), ptr(w_router), ptr(bias), ptr(logits),
          ptr(topk_idx), ptr(topk_gate), ptr(ws), stream_handle(stream))


def moe_topk_gating(cfg, logits, topk_idx, topk_gate, ws, stream=None):
    _call("moe_topk_gating", ctypes.byref(cfg), ptr(logits), ptr(topk_idx), ptr(topk_gate),
          ptr(ws), stream_handle(stream))


def moe_build_offsets(cfg, topk_idx, counts, offsets, slot_of_pair, pair_of_slot, ws, stream=None):
    _call("moe_build_offsets", ctypes.byref(cfg), ptr(topk_idx), ptr(counts), ptr(offsets),
          ptr(slot_of_pair), ptr(pair_of_slot), ptr(ws), stream_handle(stream))


def moe_build_offsets_noalloc(cfg, topk_idx, counts, offsets, slot_of_pair, pair_of_slot,
                              stream=None):
    """moe_build_offsets with its scratch inside the library: for callers that cannot
    allocate a workspace.  Calls that may overlap on the GPU must be ordered."""
    _call("moe_build_offsets_noalloc", ctypes.byref(cfg), ptr(topk_idx), ptr(counts), ptr(offsets),
          ptr(slot_of_pair), ptr(pair_of_slot), stream_handle(stream))


def moe_permute(cfg, x, slot_of_pair, x_perm, stream=None):
    _call("moe_permute", ctypes.byref(cfg), ptr(x), ptr(slot_of_pair), ptr(x_perm),
          stream_handle(stream))


def moe_grouped_swiglu_fwd(cfg, x_perm, offsets, w_gate, w_up, w_down, hu, a, y_perm, ws,
                           stream=None):
    _call("moe_grouped_swiglu_fwd", ctypes.byref(cfg), ptr(x_perm), ptr(offsets), ptr(w_gate),
          ptr(w_up), ptr(w_down), ptr(hu), ptr(a), ptr(y_perm), ptr(ws), stream_handle(stream))


def moe_grouped_swiglu_bwd(cfg, dy_perm, x_perm, hu, a, offsets, w_gate, w_up, w_down, dhu,
                           dx_perm, dw_gate, dw_up, dw_down, ws, stream=None):
    _call("moe_grouped_swiglu_bwd", ctypes.byref(cfg), ptr(dy_perm), ptr(x_perm), ptr(hu), ptr(a),
          ptr(offsets), ptr(w_gate), ptr(w_up), ptr(w_down), ptr(dhu), ptr(dx_perm),
          ptr(dw_gate), ptr(dw_up), ptr(dw_down), ptr(ws), stream_handle(stream))


def moe_unpermute_combine(cfg, y_perm, slot_of_pair, topk_gate, y, stream=None):
    _call("moe_unpermute_combine", ctypes.byref(cfg), ptr(y_perm), ptr(slot_of_pair),
          ptr(topk_gate), ptr(y), stream_handle(stream))


def moe_combine_bwd(cfg, dy, y_perm, slot_of_pair, topk_gate, dy_perm, dgate, stream=None):
    _call("moe_combine_bwd", ctypes.byref(cfg), ptr(dy), ptr(y_perm), ptr(slot_of_pair),
          ptr(topk_gate), ptr(dy_perm), ptr(dgate), stream_handle(stream))


def moe_unpermute_sum(cfg, dx_perm, slot_of_pair, dx, stream=None):
    _call("moe_unpermute_sum", ctypes.byref(cfg), ptr(dx_perm), ptr(slot_of_pair), ptr(dx),
          stream_handle(stream))


def moe_route_bwd(cfg, dgate, topk_gate, topk_idx, x, w_router, dx, dw_router, ws, stream=None):
    _call("moe_route_bwd", ctypes.byref(cfg), ptr(dgate), ptr(topk_gate), ptr(topk_idx), ptr(x),
          ptr(w_router), ptr(dx), ptr(dw_router), ptr(ws), stream_handle(stream))


def moe_mx_quantize_rows(src, rows, cols, offsets, E, rows_bound, codes, scales, stream=None):
    _call("moe_mx_quantize_rows", ptr(src), rows, cols, ptr(offsets), E, rows_bound, ptr(codes),
          ptr(scales), stream_handle(stream))


def moe_permute_mxfp8(cfg, x, slot_of_pair, offsets, x_perm, rows_bound, codes, scales, stream=None):
    _call("moe_permute_mxfp8", ctypes.byref(cfg), ptr(x), ptr(slot_of_pair), ptr(offsets), ptr(x_perm),
          rows_bound, ptr(codes), ptr(scales), stream_handle(stream))


def moe_dispatch_mxfp8(cfg, x, pair_of_slot, offsets, rows_bound, x_perm, codes_r, scales_r, codes_c, scales_c,
                       stream=None):
    _call("moe_dispatch_mxfp8", ctypes.byref(cfg), ptr(x), ptr(pair_of_slot), ptr(offsets), rows_bound,
          ptr(x_perm), ptr(codes_r), ptr(scales_r), ptr(codes_c), ptr(scales_c), stream_handle(stream))


def moe_combine_bwd_mxfp8(cfg, dy, y_perm, pair_of_slot, offsets, topk_gate, rows_bound, dy_perm, dgate, codes_r,
                          scales_r, codes_c, scales_c, stream=None):
    _call("moe_combine_bwd_mxfp8", ctypes.byref(cfg), ptr(dy), ptr(y_perm), ptr(pair_of_slot), ptr(offsets),
          ptr(topk_gate), rows_bound, ptr(dy_perm), ptr(dgate), ptr(codes_r), ptr(scales_r), ptr(codes_c),
          ptr(scales_c), stream_handle(stream))


def moe_mx_quantize_cols(src, rows, cols, offsets, E, rows_bound, codes, scales, stream=None):
    _call("moe_mx_quantize_cols", ptr(src), rows, cols, ptr(offsets), E, rows_bound, ptr(codes),
          ptr(scales), stream_handle(stream))


def _struct(cls, fields, d):
    return cls(*[ptr(d.get(n)) for n in fields])


def layer_weights(w_router, bias, w_gate, w_up, w_down, shared=None) -> LayerWeights:
    """shared: None, or (w_shared_gate [d,f], w_shared_up [d,f], w_shared_down [f,d])."""
    sg, su, sd = shared if shared is not None else (None, None, None)
    return LayerWeights(ptr(w_router), ptr(bias), ptr(w_gate), ptr(w_up), ptr(w_down), ptr(sg), ptr(su),
                        ptr(sd))


def moe_layer_fwd(cfg, weights: LayerWeights, x, y, saved: dict, ws, stream=None):
    sv = _struct(LayerSaved, SAVED_FIELDS, saved)
    _call("moe_layer_fwd", ctypes.byref(cfg), ctypes.byref(weights), ptr(x), ptr(y),
          ctypes.byref(sv), ptr(ws), stream_handle(stream))


def moe_layer_fwd_routed(cfg, weights: LayerWeights, x, y, saved: dict, ws, stream=None):
    sv = _struct(LayerSaved, SAVED_FIELDS, saved)
    _call("moe_layer_fwd_routed", ctypes.byref(cfg), ctypes.byref(weights), ptr(x), ptr(y),
          ctypes.byref(sv), ptr(ws), stream_handle(stream))


def moe_layer_bwd(cfg, weights: LayerWeights, x, dy, saved: dict, grads: dict, ws, stream=None):
    sv = _struct(LayerSaved, SAVED_FIELDS, saved)
    gr = _struct(LayerGrads, GRAD_FIELDS, grads)
    _call("moe_layer_bwd", ctypes.byref(cfg), ctypes.byref(weights), ptr(x), ptr(dy),
          ctypes.byref(sv), ctypes.byref(gr), ptr(ws), stream_handle(stream))


# ------------------------------------------------------------------ buffer helpers
# Device-memory plumbing for callers that use torch as their allocator.

def torch_dtype(cfg):
    import torch
    return torch.bfloat16 if cfg.dtype == MOE_BF16 else torch.float32


def alloc_workspace(cfg, device="cuda"):
    import torch
    return torch.zeros(max(moe_workspace_size(cfg), 256), dtype=torch.uint8, device=device)


def alloc_saved(cfg, device="cuda", logits=True, shared=False, recompute=False, mx_saved=True) -> dict:
    """Forward buffers.  shared: room for a shared expert's activations; recompute: keep no
    [h | u] (the backward recomputes them), which leaves hu (and shared_hu) None; mx_saved
    (MXFP8 only): keep the MXFP8 copies of the weights and the routed rows from the forward
    for the backward, which leaves x_perm None (the rows move in MXFP8 only)."""
    import torch
    dt = torch_dtype(cfg)
    T, d, E, k, f, P = cfg.T, cfg.d, cfg.E, cfg.k, cfg.f, cfg.T * cfg.k
    i32 = dict(dtype=torch.int32, device=device)
    keep_hu = not recompute
    fp8_rows = mx_saved and cfg.prec == MOE_PREC_MXFP8
    return dict(
        logits=torch.empty(T, E, dtype=torch.float32, device=device) if logits else None,
        topk_idx=torch.empty(T, k, **i32),
        topk_gate=torch.empty(T, k, dtype=torch.float32, device=device),
        counts=torch.empty(E, **i32), offsets=torch.empty(E + 1, **i32),
        slot_of_pair=torch.empty(P, **i32), pair_of_slot=torch.empty(P, **i32),
        x_perm=None if fp8_rows else torch.empty(P, d, dtype=dt, device=device),
        hu=torch.empty(P, 2 * f, dtype=dt, device=device) if keep_hu else None,
        a=torch.empty(P, f, dtype=dt, device=device),
        y_perm=torch.empty(P, d, dtype=dt, device=device),
        shared_hu=torch.empty(T, 2 * f, dtype=dt, device=device) if shared and keep_hu else None,
        shared_a=torch.empty(T, f, dtype=dt, device=device) if shared else None,
        mx_saved=torch.empty(moe_mx_saved_bytes(cfg), dtype=torch.uint8, device=device) if fp8_rows else None,
    )


def alloc_grads(cfg, device="cuda", router=True, shared=False) -> dict:
    """Backward buffers.  MXFP8 leaves dy_perm None (the combine's backward writes it in
    MXFP8 only, into the workspace)."""
    import torch
    dt = torch_dtype(cfg)
    T, d, E, k, f, P = cfg.T, cfg.d, cfg.E, cfg.k, cfg.f, cfg.T * cfg.k
    return dict(
        dx=torch.empty(T, d, dtype=dt, device=device),
        dw_router=torch.empty(d, E, dtype=torch.float32, device=device) if router else None,
        dw_gate=torch.empty(E, d, f, dtype=dt, device=device),
        dw_up=torch.empty(E, d, f, dtype=dt, device=device),
        dw_down=torch.empty(E, f, d, dtype=dt, device=device),
        dy_perm=None if cfg.prec == MOE_PREC_MXFP8 else torch.empty(P, d, dtype=dt, device=device),
        dgate=torch.empty(T, k, dtype=torch.float32, device=device),
        dhu=torch.empty(P, 2 * f, dtype=dt, device=device),
        dx_perm=torch.empty(P, d, dtype=dt, device=device),
        dw_shared_gate=torch.empty(d, f, dtype=dt, device=device) if shared else None,
        dw_shared_up=torch.empty(d, f, dtype=dt, device=device) if shared else None,
        dw_shared_down=torch.empty(f, d, dtype=dt, device=device) if shared else None,
        shared_dhu=torch.empty(T, 2 * f, dtype=dt, device=device) if shared else None,
    )
