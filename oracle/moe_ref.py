"""Plain CPU oracle for one MoE layer step (forward and backward).

TEST INFRASTRUCTURE ONLY.  Only the test suite, the smoke check and the
benchmark's CPU-baseline leg may import this module.  The library never calls
it, and it shares no code with the CUDA path.

Every function is written for a reader to check by eye: NumPy in float64 (the
routed layer can also run in float32, only to time it as the CPU baseline), an
explicit loop over experts, a library matmul or sort as a single step, no
blocking or fusion.

Sources.  The method is described, in prose only, by five web pages about
Ai2's Olmo-core 3 MoE training stack:
  [qidao123] "Ai2开源Olmo-core 3：把万亿参数MoE训练栈交给小团队，8卡吞吐达旧实现2.7倍",
             section "新闻原文" (news text);
  [bigchange] "Olmo-core 3 открывает стек обучения MoE от Ai2, но результаты GPU
             ограничены", sections "Главное изменение", "Три числа, три знаменателя";
  [kitmori]  "Introducing Olmo-core 3: Open, Scalable Training Infrastructure for
             Trillion-Parameter MoEs", "Key points";
  [unite.ai] "Ai2 κυκλοφορεί το Olmo-Core 3, ανοιχτό σύνολο εκπαίδευσης για MoE
             τρισεκατομμυρίων παραμέτρων", section "Παραλληλισμός, Ακρίβεια και
             Τεχνικές Μνήμης" (parallelism, precision and memory techniques);
  [ettayeb]  "Olmo-core 3 ouvre l'entraînement des MoE à l'échelle du trillion de
             paramètres", section "Trois parallélismes, trois optimisations de routage".
The pages say that each token is sent to 4 of E experts, that routed rows are
written straight into per-expert input buffers, that routing metadata stays on
the GPU, that the experts' small matmuls run as one grouped GEMM, and that
MXFP8 is used for the feed-forward compute.  They never write the layer's
arithmetic out.  Where they are silent this oracle takes the plainest reading:
  * router: softmax over all E logits, top-k on the logits, gates renormalised
    over the k selected experts; equal logits go to the lower expert index;
    selected experts are listed in descending logit order;
  * expert FFN: SwiGLU without biases, y = (silu(x W_gate) * (x W_up)) W_down;
  * rows inside one expert's buffer keep the order of the routed pairs
    (pair i = t*k + j), i.e. a stable counting sort by expert;
  * MXFP8: OCP Microscaling v1.0 with E4M3 elements and an E8M0 scale per
    32-element block along each GEMM's reduction axis;
  * shared expert ([bigchange], section "Что инженер может попробовать на
    практике": the production rows use top-four routing and one shared expert):
    a SwiGLU of the routed experts' shape that every token passes through, its
    output added to the routed experts' gate-weighted sum with weight 1.

Parity pins for every function live in tests/test_oracle_*.py.  Nothing here
is "parity unpinned".
"""
from __future__ import annotations

import contextlib

import numpy as np

F64 = np.float64

# Working precision of the routed layer's arithmetic (routing, FFN, combine and their
# backward): float64 for parity, the default; float32 only to time the same code as the CPU
# baseline (working_precision).  The MXFP8 quantisers below always work in float64.
_PRECISION = [F64]


def _wdt():
    return _PRECISION[0]


def _work(a):
    """a as an array in the working precision."""
    return np.asarray(a, _PRECISION[0])


@contextlib.contextmanager
def working_precision(dtype):
    """Run the routed layer's functions in another floating type (np.float32 for timing)."""
    old = _PRECISION[0]
    _PRECISION[0] = np.dtype(dtype).type
    try:
        yield
    finally:
        _PRECISION[0] = old


# ---------------------------------------------------------------------------
# Routing: [unite.ai] / [ettayeb] routing paragraph; [qidao123] news text
# ("8 -> 128 experts, 4 selected per token").
# ---------------------------------------------------------------------------

def router_logits(x, w_r, bias=None):
    """z = x W_r (+ b): one logit per (token, expert).  x [T,d], w_r [d,E], bias [E]."""
    z = _work(x) @ _work(w_r)
    if bias is not None:
        z = z + _work(bias)[None, :]
    return z


def softmax(z):
    """Row-wise softmax over the last axis."""
    z = _work(z)
    m = z.max(axis=-1, keepdims=True)
    e = np.exp(z - m)
    return e / e.sum(axis=-1, keepdims=True)


def topk_experts(z, k):
    """The k experts with the largest logits, per token.

    Order: descending logit; equal logits (including +0 and -0) put the lower
    expert index first.  Selection is done on the logits themselves, which is
    the same as selecting on softmax probabilities (softmax is monotone) but
    does not invent ties through rounding of exp.  Returns int32 [T,k].
    """
    z = _work(z)
    T, E = z.shape
    index = np.broadcast_to(np.arange(E), (T, E))
    # np.lexsort sorts by the last key first: primary key -z, then expert index.
    order = np.lexsort((index, -z), axis=-1)
    return order[:, :k].astype(np.int32)


def renormalised_gates(p, idx):
    """g_j = p_{S_j} / sum_{j'} p_{S_j'}: softmax probabilities renormalised over the selection."""
    sel = np.take_along_axis(_work(p), np.asarray(idx, np.int64), axis=1)
    return sel / sel.sum(axis=1, keepdims=True)


def route(x, w_r, k, bias=None):
    """Router forward: logits, full softmax, top-k indices and renormalised gates."""
    z = router_logits(x, w_r, bias)
    p = softmax(z)
    idx = topk_experts(z, k)
    return z, p, idx, renormalised_gates(p, idx)


def route_from_logits(z, k):
    """Top-k indices and renormalised gates from given logits (the router's second half)."""
    p = softmax(z)
    idx = topk_experts(z, k)
    return idx, renormalised_gates(p, idx)


# ---------------------------------------------------------------------------
# GPU-resident routing metadata and rowwise placement: [unite.ai] / [ettayeb]
# ("routed rows go straight into the experts' input buffers", "routing
# metadata stays on the GPU").
# ---------------------------------------------------------------------------

def routing_metadata(idx, E):
    """Per-expert counts, exclusive-scan offsets, and the slot of every routed pair.

    Pair i = t*k + j (token t, choice j) goes to expert e = idx[t, j].  Its slot
    is offsets[e] + (number of earlier pairs that chose e): a stable counting
    sort by expert.  pair_of_slot is the inverse permutation.
    """
    flat = np.asarray(idx, np.int64).ravel()
    P = flat.size
    counts = np.zeros(E, np.int64)
    for e in flat:
        counts[e] += 1
    offsets = np.zeros(E + 1, np.int64)
    for e in range(E):
        offsets[e + 1] = offsets[e] + counts[e]
    cursor = offsets[:E].copy()
    slot_of_pair = np.empty(P, np.int64)
    for i in range(P):
        e = flat[i]
        slot_of_pair[i] = cursor[e]
        cursor[e] += 1
    pair_of_slot = np.empty(P, np.int64)
    pair_of_slot[slot_of_pair] = np.arange(P)
    return counts, offsets, slot_of_pair, pair_of_slot


def permute(x, pair_of_slot, k):
    """Rowwise dispatch: x_perm[s] = x[token of the pair in slot s]."""
    return _work(x)[np.asarray(pair_of_slot) // k]


# ---------------------------------------------------------------------------
# Grouped expert FFN: [unite.ai] / [ettayeb] ("grouped GEMM combines the
# experts' many small matmuls"); [bigchange] "Три числа" (feed-forward compute).
# ---------------------------------------------------------------------------

def silu(h):
    return h / (1.0 + np.exp(-h))


def sigmoid(h):
    return 1.0 / (1.0 + np.exp(-h))


def expert_swiglu(xr, w_gate_e, w_up_e, w_down_e):
    """One expert on its rows: h = x Wg, u = x Wu, a = silu(h) * u, y = a Wd."""
    xr = _work(xr)
    h = xr @ _work(w_gate_e)
    u = xr @ _work(w_up_e)
    a = silu(h) * u
    y = a @ _work(w_down_e)
    return h, u, a, y


def grouped_swiglu(x_perm, offsets, w_gate, w_up, w_down):
    """Every expert's SwiGLU on its contiguous row range [offsets[e], offsets[e+1])."""
    x_perm = _work(x_perm)
    P = x_perm.shape[0]
    f = w_gate.shape[2]
    d = w_down.shape[2]
    h = np.zeros((P, f), _wdt())
    u = np.zeros((P, f), _wdt())
    a = np.zeros((P, f), _wdt())
    y = np.zeros((P, d), _wdt())
    for e in range(w_gate.shape[0]):
        lo, hi = int(offsets[e]), int(offsets[e + 1])
        if hi > lo:
            h[lo:hi], u[lo:hi], a[lo:hi], y[lo:hi] = expert_swiglu(
                x_perm[lo:hi], w_gate[e], w_up[e], w_down[e])
    return h, u, a, y


def combine(y_perm, slot_of_pair, gate):
    """Gate-weighted unpermute: Y[t] = sum_j g[t,j] * y_perm[slot(t,j)]."""
    gate = _work(gate)
    T, k = gate.shape
    slots = np.asarray(slot_of_pair).reshape(T, k)
    y_perm = _work(y_perm)
    Y = np.zeros((T, y_perm.shape[1]), _wdt())
    for j in range(k):
        Y += gate[:, j:j + 1] * y_perm[slots[:, j]]
    return Y


def shared_expert_fwd(x, shared):
    """The shared expert on every token: shared = (W_gate [d,f], W_up [d,f], W_down [f,d])."""
    h, u, a, y = expert_swiglu(x, *shared)
    return dict(shared_h=h, shared_u=u, shared_a=a, shared_y=y)


def layer_fwd(x, w_r, w_gate, w_up, w_down, k, bias=None, shared=None):
    """Whole forward step.  Returns a dict with every intermediate.  shared: None or the
    shared expert's (W_gate, W_up, W_down)."""
    E = w_gate.shape[0]
    z, p, idx, gate = route(x, w_r, k, bias)
    counts, offsets, slot_of_pair, pair_of_slot = routing_metadata(idx, E)
    x_perm = permute(x, pair_of_slot, k)
    h, u, a, y_perm = grouped_swiglu(x_perm, offsets, w_gate, w_up, w_down)
    Y = combine(y_perm, slot_of_pair, gate)
    out = dict(z=z, p=p, idx=idx, gate=gate, counts=counts, offsets=offsets,
               slot_of_pair=slot_of_pair, pair_of_slot=pair_of_slot, x_perm=x_perm,
               h=h, u=u, a=a, y_perm=y_perm, y=Y)
    if shared is not None:
        out.update(shared_expert_fwd(x, shared))
        out["y"] = Y + out["shared_y"]
    return out


def layer_fwd_routed(x, idx, gate, w_gate, w_up, w_down, shared=None):
    """Forward step from given routing (uniform random routing enters here)."""
    E = w_gate.shape[0]
    k = idx.shape[1]
    counts, offsets, slot_of_pair, pair_of_slot = routing_metadata(idx, E)
    x_perm = permute(x, pair_of_slot, k)
    h, u, a, y_perm = grouped_swiglu(x_perm, offsets, w_gate, w_up, w_down)
    Y = combine(y_perm, slot_of_pair, gate)
    out = dict(idx=np.asarray(idx), gate=_work(gate), counts=counts,
               offsets=offsets, slot_of_pair=slot_of_pair, pair_of_slot=pair_of_slot,
               x_perm=x_perm, h=h, u=u, a=a, y_perm=y_perm, y=Y)
    if shared is not None:
        out.update(shared_expert_fwd(x, shared))
        out["y"] = Y + out["shared_y"]
    return out


# ---------------------------------------------------------------------------
# Backward (chain rule through each forward step, in reverse order).
# ---------------------------------------------------------------------------

def combine_bwd(dY, y_perm, slot_of_pair, gate):
    """dy_perm[slot(t,j)] = g[t,j] dY[t];  dgate[t,j] = <dY[t], y_perm[slot(t,j)]>."""
    dY = _work(dY)
    gate = _work(gate)
    T, k = gate.shape
    slots = np.asarray(slot_of_pair).reshape(T, k)
    y_perm = _work(y_perm)
    dy_perm = np.zeros_like(y_perm)
    dgate = np.zeros((T, k), _wdt())
    for j in range(k):
        dy_perm[slots[:, j]] = gate[:, j:j + 1] * dY
        dgate[:, j] = np.sum(dY * y_perm[slots[:, j]], axis=1)
    return dy_perm, dgate


def swiglu_bwd(da, h, u):
    """From da = dL/da with a = silu(h) * u: dh = da u silu'(h), du = da silu(h).

    silu'(h) = s (1 + h (1 - s)) with s = sigmoid(h).
    """
    s = sigmoid(h)
    dh = da * u * s * (1.0 + h * (1.0 - s))
    du = da * h * s
    return dh, du


def grouped_swiglu_bwd(dy_perm, x_perm, h, u, a, offsets, w_gate, w_up, w_down):
    """Per expert: da = dy Wd^T; (dh, du) = SwiGLU'; dx = dh Wg^T + du Wu^T;
    dWd = a^T dy; dWg = x^T dh; dWu = x^T du."""
    dy_perm = _work(dy_perm)
    x_perm = _work(x_perm)
    E = w_gate.shape[0]
    dh = np.zeros_like(h)
    du = np.zeros_like(u)
    dx_perm = np.zeros_like(x_perm)
    dw_gate = np.zeros(w_gate.shape, _wdt())
    dw_up = np.zeros(w_up.shape, _wdt())
    dw_down = np.zeros(w_down.shape, _wdt())
    for e in range(E):
        lo, hi = int(offsets[e]), int(offsets[e + 1])
        if hi == lo:
            continue
        wg, wu, wd = (_work(w[e]) for w in (w_gate, w_up, w_down))
        da = dy_perm[lo:hi] @ wd.T
        dh[lo:hi], du[lo:hi] = swiglu_bwd(da, h[lo:hi], u[lo:hi])
        dw_down[e] = a[lo:hi].T @ dy_perm[lo:hi]
        dx_perm[lo:hi] = dh[lo:hi] @ wg.T + du[lo:hi] @ wu.T
        dw_gate[e] = x_perm[lo:hi].T @ dh[lo:hi]
        dw_up[e] = x_perm[lo:hi].T @ du[lo:hi]
    return dict(dh=dh, du=du, dx_perm=dx_perm, dw_gate=dw_gate, dw_up=dw_up, dw_down=dw_down)


def unpermute_sum(dx_perm, slot_of_pair, T, k):
    """dx[t] = sum_j dx_perm[slot(t,j)] (the gate was already applied in combine_bwd)."""
    slots = np.asarray(slot_of_pair).reshape(T, k)
    dx_perm = _work(dx_perm)
    dx = np.zeros((T, dx_perm.shape[1]), _wdt())
    for j in range(k):
        dx += dx_perm[slots[:, j]]
    return dx


def gate_logit_grad(dgate, gate, idx, E):
    """dL/dz for renormalised top-k gates (softmax over the selected logits).

    dz[t, S_j] = g_j (dg_j - sum_j' g_j' dg_j'); zero for experts not selected
    (the selection is piecewise constant in z).
    """
    dgate = _work(dgate)
    gate = _work(gate)
    T, k = gate.shape
    inner = np.sum(gate * dgate, axis=1, keepdims=True)
    dz_sel = gate * (dgate - inner)
    dz = np.zeros((T, E), _wdt())
    np.put_along_axis(dz, np.asarray(idx, np.int64), dz_sel, axis=1)
    return dz


def route_bwd(dgate, gate, idx, x, w_r):
    """Router backward: dz as above, dW_r = x^T dz, dx_router = dz W_r^T."""
    E = w_r.shape[1]
    dz = gate_logit_grad(dgate, gate, idx, E)
    dw_r = _work(x).T @ dz
    dx = dz @ _work(w_r).T
    return dz, dw_r, dx


def shared_expert_bwd(dY, x, fwd, shared):
    """The shared expert's backward: its output gradient is dY itself (weight 1).  The
    SwiGLU backward of one expert holding every token, in the same steps as the routed
    experts'.  Returns dx and the three weight gradients."""
    T = np.asarray(x).shape[0]
    one = [_work(w)[None] for w in shared]     # one expert [1, ...]
    g = grouped_swiglu_bwd(dY, x, fwd["shared_h"], fwd["shared_u"], fwd["shared_a"],
                           np.array([0, T]), *one)
    return dict(shared_dx=g["dx_perm"], dw_shared_gate=g["dw_gate"][0],
                dw_shared_up=g["dw_up"][0], dw_shared_down=g["dw_down"][0],
                shared_dh=g["dh"], shared_du=g["du"])


def layer_bwd(fwd, dY, x, w_r, w_gate, w_up, w_down, shared=None):
    """Whole backward step, given the forward dict from layer_fwd."""
    T, k = fwd["gate"].shape
    dy_perm, dgate = combine_bwd(dY, fwd["y_perm"], fwd["slot_of_pair"], fwd["gate"])
    g = grouped_swiglu_bwd(dy_perm, fwd["x_perm"], fwd["h"], fwd["u"], fwd["a"],
                           fwd["offsets"], w_gate, w_up, w_down)
    dx = unpermute_sum(g["dx_perm"], fwd["slot_of_pair"], T, k)
    dz, dw_r, dx_r = route_bwd(dgate, fwd["gate"], fwd["idx"], x, w_r)
    out = dict(dy_perm=dy_perm, dgate=dgate, dz=dz, dw_r=dw_r, dx=dx + dx_r,
               dx_experts=dx, **g)
    if shared is not None:
        out.update(shared_expert_bwd(dY, x, fwd, shared))
        out["dx"] = out["dx"] + out["shared_dx"]
    return out


def layer_bwd_routed(fwd, dY, w_gate, w_up, w_down, x=None, shared=None):
    """Backward with routing held fixed (no router gradient): uniform-random routing.
    With a shared expert, x (the layer input) is needed too."""
    T, k = fwd["gate"].shape
    dy_perm, dgate = combine_bwd(dY, fwd["y_perm"], fwd["slot_of_pair"], fwd["gate"])
    g = grouped_swiglu_bwd(dy_perm, fwd["x_perm"], fwd["h"], fwd["u"], fwd["a"],
                           fwd["offsets"], w_gate, w_up, w_down)
    dx = unpermute_sum(g["dx_perm"], fwd["slot_of_pair"], T, k)
    out = dict(dy_perm=dy_perm, dgate=dgate, dx=dx, **g)
    if shared is not None:
        out.update(shared_expert_bwd(dY, x, fwd, shared))
        out["dx"] = out["dx"] + out["shared_dx"]
    return out

# ---------------------------------------------------------------------------
# MXFP8: [unite.ai] / [ettayeb] / [kitmori] ("MXFP8 for selected operations,
# mostly feed-forward compute and data movement between experts").  Element
# and scale formats follow the OCP Microscaling Formats (MX) v1.0 spec:
# E4M3 elements (bias 7, max 448, no infinities) and one E8M0 power-of-two
# scale per block of 32 consecutive elements along the reduction axis.
# ---------------------------------------------------------------------------

def bf16_rne(v):
    """Round to bf16 (nearest, ties to even) through fp32, as a GEMM output stored in bf16
    after fp32 accumulation: the bf16 tensors the MXFP8 GEMMs quantise."""
    f = np.asarray(v, F64).astype(np.float32)
    u = f.view(np.uint32).astype(np.uint64)
    u = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    return (u.astype(np.uint32) << 16).view(np.float32).astype(F64)


MX_BLOCK = 32
E4M3_EMAX = 8          # exponent of the largest normal E4M3 value, 448 = 1.75 * 2^8
E4M3_MAX = 448.0


def e4m3_value(code):
    """Value of an E4M3 byte (codes 0x7F / 0xFF are NaN)."""
    code = int(code)
    sign = -1.0 if code & 0x80 else 1.0
    e = (code >> 3) & 0xF
    m = code & 0x7
    if e == 0xF and m == 0x7:
        return float("nan")
    if e == 0:
        return sign * (m / 8.0) * 2.0 ** -6
    return sign * (1.0 + m / 8.0) * 2.0 ** (e - 7)


def e4m3_grid():
    """All non-negative finite E4M3 values, indexed by their code 0x00..0x7E."""
    return np.array([e4m3_value(c) for c in range(0x7F)], F64)


_E4M3 = e4m3_grid()


def round_to_e4m3(v):
    """Nearest E4M3 code (ties to the even code), saturating |v| > 448 to 448;
    a negative input that rounds to zero keeps its sign (code 0x80).

    Returns (codes uint8, values float64).
    """
    v = np.asarray(v, F64)
    mag = np.minimum(np.abs(v), E4M3_MAX)
    hi = np.searchsorted(_E4M3, mag, side="left")          # first grid value >= mag
    hi = np.minimum(hi, _E4M3.size - 1)
    lo = np.maximum(hi - 1, 0)
    d_lo = mag - _E4M3[lo]
    d_hi = _E4M3[hi] - mag
    pick_hi = (d_hi < d_lo) | ((d_hi == d_lo) & (hi % 2 == 0))
    code = np.where(pick_hi, hi, lo)
    code = np.where(mag == _E4M3[hi], hi, code)
    # The sign is kept even when the magnitude rounds to zero (IEEE-style -0).
    neg = np.signbit(v)
    codes = (code | np.where(neg, 0x80, 0)).astype(np.uint8)
    vals = np.where(neg, -_E4M3[code], _E4M3[code])
    return codes, vals


def mx_scale_exponent(amax):
    """Shared block exponent s = floor(log2(amax)) - 8, clamped to E8M0's [-127, 127];
    amax = 0 gives the smallest scale, s = -127."""
    amax = np.asarray(amax, F64)
    mant, ex = np.frexp(np.where(amax > 0, amax, 1.0))      # amax = mant * 2^ex, mant in [0.5, 1)
    s = (ex - 1) - E4M3_EMAX
    s = np.where(amax > 0, s, -127)
    return np.clip(s, -127, 127).astype(np.int64)


def mx_quantize(v, axis=-1):
    """Quantise to MXFP8 along ``axis`` (its length a multiple of 32).

    Returns (codes uint8 with v's shape, scales uint8 E8M0 with the axis
    divided by 32, dequantised float64 values).
    """
    v = np.moveaxis(np.asarray(v, F64), axis, -1)
    n = v.shape[-1]
    if n % MX_BLOCK:
        raise ValueError("length along the block axis must be a multiple of 32")
    blocks = v.reshape(v.shape[:-1] + (n // MX_BLOCK, MX_BLOCK))
    s = mx_scale_exponent(np.max(np.abs(blocks), axis=-1))
    scaled = blocks / np.ldexp(1.0, s)[..., None]
    codes, q = round_to_e4m3(scaled)
    deq = q * np.ldexp(1.0, s)[..., None]
    codes = np.moveaxis(codes.reshape(v.shape), -1, axis)
    deq = np.moveaxis(deq.reshape(v.shape), -1, axis)
    scales = np.moveaxis((s + 127).astype(np.uint8), -1, axis)
    return codes, scales, deq


def mx_dequantize(codes, scales, axis=-1):
    """Inverse of mx_quantize's storage: value = E4M3(code) * 2^(scale - 127)."""
    codes = np.moveaxis(np.asarray(codes), axis, -1)
    scales = np.moveaxis(np.asarray(scales), axis, -1).astype(np.int64)
    vals = np.vectorize(e4m3_value, otypes=[F64])(codes)
    vals = vals * np.repeat(np.ldexp(1.0, scales - 127), MX_BLOCK, axis=-1)
    return np.moveaxis(vals, -1, axis)


def mx_quantize_grouped_rows(v, offsets):
    """Quantise a row-grouped operand along its rows (the reduction axis of a
    weight-gradient GEMM), one 32-row block at a time inside each group.

    Each group [offsets[e], offsets[e+1]) is zero-padded to a multiple of 32
    rows; zero rows do not change any block's amax.  Returns the dequantised
    values with v's shape.
    """
    v = np.asarray(v, F64)
    out = np.zeros_like(v)
    for e in range(len(offsets) - 1):
        lo, hi = int(offsets[e]), int(offsets[e + 1])
        n = hi - lo
        if n == 0:
            continue
        padded = np.zeros(((n + MX_BLOCK - 1) // MX_BLOCK * MX_BLOCK, v.shape[1]))
        padded[:n] = v[lo:hi]
        out[lo:hi] = mx_quantize(padded, axis=0)[2][:n]
    return out


def grouped_swiglu_mx(x_perm, offsets, w_gate, w_up, w_down):
    """Forward expert FFN with every GEMM operand MXFP8-quantised along its own K.

    GEMM 1: x_perm (K = d, along rows' columns) with W_gate/W_up (K = d, down
    their rows).  GEMM 2: a (K = f) with W_down (K = f).  Products and sums in
    float64 on the dequantised values.  The MXFP8 GEMMs output bf16, so GEMM 2
    quantises a as stored: bf16(a).  Returns h, u, a unrounded.  Each expert's
    weights are quantised inside the loop (blocks never cross experts), so only
    experts holding rows are quantised.
    """
    xq = mx_quantize(x_perm, axis=1)[2]
    P = xq.shape[0]
    f = w_gate.shape[2]
    d = w_down.shape[2]
    h = np.zeros((P, f))
    u = np.zeros((P, f))
    a = np.zeros((P, f))
    y = np.zeros((P, d))
    for e in range(w_gate.shape[0]):
        lo, hi = int(offsets[e]), int(offsets[e + 1])
        if hi == lo:
            continue
        h[lo:hi] = xq[lo:hi] @ mx_quantize(w_gate[e], axis=0)[2]
        u[lo:hi] = xq[lo:hi] @ mx_quantize(w_up[e], axis=0)[2]
        a[lo:hi] = silu(h[lo:hi]) * u[lo:hi]
    aq = mx_quantize(bf16_rne(a), axis=1)[2]
    for e in range(w_gate.shape[0]):
        lo, hi = int(offsets[e]), int(offsets[e + 1])
        if hi > lo:
            y[lo:hi] = aq[lo:hi] @ mx_quantize(w_down[e], axis=0)[2]
    return h, u, a, y


def grouped_swiglu_bwd_mx(dy_perm, x_perm, h, u, a, offsets, w_gate, w_up, w_down):
    """Backward expert FFN with every GEMM operand MXFP8-quantised along its own K.

    dgrad GEMMs reduce over the feature axis (dy: K = d with W_down^T; [dh|du]:
    K = 2f with [W_gate|W_up]^T); weight-gradient GEMMs reduce over the tokens
    of one expert (blocks of 32 rows inside each expert, zero-padded).  [dh|du]
    is the bf16 output of the first GEMM's epilogue, so both GEMMs that read it
    quantise bf16([dh|du]).  Returns dh, du unrounded.  Weights are quantised per
    expert, as in grouped_swiglu_mx.
    """
    dy_perm = np.asarray(dy_perm, F64)
    x_perm = np.asarray(x_perm, F64)
    E = w_gate.shape[0]
    f = w_gate.shape[2]
    dyq_k = mx_quantize(dy_perm, axis=1)[2]
    dh = np.zeros_like(h)
    du = np.zeros_like(u)
    for e in range(E):
        lo, hi = int(offsets[e]), int(offsets[e + 1])
        if hi == lo:
            continue
        wdq_t = mx_quantize(w_down[e], axis=1)[2]     # W_down^T has K = d along W_down's columns
        da = dyq_k[lo:hi] @ wdq_t.T
        dh[lo:hi], du[lo:hi] = swiglu_bwd(da, h[lo:hi], u[lo:hi])
    dhu = bf16_rne(np.concatenate([dh, du], axis=1))
    dhuq_k = mx_quantize(dhu, axis=1)[2]
    # weight-gradient operands: reduction over tokens inside each expert
    aq_t = mx_quantize_grouped_rows(a, offsets)
    dyq_t = mx_quantize_grouped_rows(dy_perm, offsets)
    xq_t = mx_quantize_grouped_rows(x_perm, offsets)
    dhuq_t = mx_quantize_grouped_rows(dhu, offsets)
    dx_perm = np.zeros_like(x_perm)
    dw_gate = np.zeros(w_gate.shape)
    dw_up = np.zeros(w_up.shape)
    dw_down = np.zeros(w_down.shape)
    for e in range(E):
        lo, hi = int(offsets[e]), int(offsets[e + 1])
        if hi == lo:
            continue
        wgu = np.concatenate([np.asarray(w_gate[e], F64), np.asarray(w_up[e], F64)], axis=1)  # [d, 2f]
        wguq_t = mx_quantize(wgu, axis=1)[2]
        dx_perm[lo:hi] = dhuq_k[lo:hi] @ wguq_t.T
        dw_down[e] = aq_t[lo:hi].T @ dyq_t[lo:hi]
        dwgu = xq_t[lo:hi].T @ dhuq_t[lo:hi]
        dw_gate[e] = dwgu[:, :f]
        dw_up[e] = dwgu[:, f:]
    return dict(dh=dh, du=du, dx_perm=dx_perm, dw_gate=dw_gate, dw_up=dw_up, dw_down=dw_down)


# ---------------------------------------------------------------------------
# The MXFP8 layer step: the steps of layer_fwd / layer_bwd in the same order, with the
# grouped GEMMs above in place of the bf16 ones.  The MXFP8 GEMMs write bf16, and the layer
# keeps five tensors in that storage between its GEMMs; each later step reads the stored
# bf16 value, so the oracle rounds exactly these (and nothing else) to bf16:
#   h, u     GEMM 1's outputs, read by the SwiGLU backward;
#   a        silu(h) * u from GEMM 1's unrounded outputs, quantised by GEMM 2 and by
#            the down projection's weight-gradient GEMM (rounded inside the GEMM steps);
#   dy_perm  g * dY, quantised by both GEMMs that read it;
#   [dh|du]  the SwiGLU backward's output, quantised by both GEMMs that read it
#            (rounded inside grouped_swiglu_bwd_mx).
# y_perm, dgate, dx_perm and the weight gradients stay unrounded, as in the bf16 oracle.
# ---------------------------------------------------------------------------

def shared_expert_fwd_mx(x, shared):
    """The shared expert with MXFP8 GEMMs: one group holding every token."""
    T = np.asarray(x).shape[0]
    one = [np.asarray(w, F64)[None] for w in shared]
    h, u, a, y = grouped_swiglu_mx(x, np.array([0, T]), *one)
    return dict(shared_h=h, shared_u=u, shared_a=a, shared_y=y)


def shared_expert_bwd_mx(dY, x, fwd, shared):
    """Its backward: output gradient dY (weight 1), the stored bf16 h, u, a as for the
    routed experts."""
    T = np.asarray(x).shape[0]
    one = [np.asarray(w, F64)[None] for w in shared]
    b = bf16_rne
    g = grouped_swiglu_bwd_mx(dY, x, b(fwd["shared_h"]), b(fwd["shared_u"]), b(fwd["shared_a"]),
                              np.array([0, T]), *one)
    return dict(shared_dx=g["dx_perm"], dw_shared_gate=g["dw_gate"][0], dw_shared_up=g["dw_up"][0],
                dw_shared_down=g["dw_down"][0], shared_dh=g["dh"], shared_du=g["du"])


def layer_fwd_mx(x, w_r, w_gate, w_up, w_down, k, bias=None, routing=None, shared=None):
    """Whole forward step with MXFP8 grouped GEMMs.  routing: None (the router runs), or
    (idx, gate) given (uniform random routing; then no router logits).  shared: None or
    the shared expert's (W_gate, W_up, W_down)."""
    E = w_gate.shape[0]
    out = {}
    if routing is None:
        z, p, idx, gate = route(x, w_r, k, bias)
        out.update(z=z, p=p)
    else:
        idx, gate = np.asarray(routing[0]), np.asarray(routing[1], F64)
        k = idx.shape[1]
    counts, offsets, slot_of_pair, pair_of_slot = routing_metadata(idx, E)
    x_perm = permute(x, pair_of_slot, k)
    h, u, a, y_perm = grouped_swiglu_mx(x_perm, offsets, w_gate, w_up, w_down)
    Y = combine(y_perm, slot_of_pair, gate)
    out.update(idx=idx, gate=gate, counts=counts, offsets=offsets, slot_of_pair=slot_of_pair,
               pair_of_slot=pair_of_slot, x_perm=x_perm, h=h, u=u, a=a, y_perm=y_perm, y=Y)
    if shared is not None:
        out.update(shared_expert_fwd_mx(x, shared))
        out["y"] = Y + out["shared_y"]
    return out


def layer_bwd_mx(fwd, dY, x, w_r, w_gate, w_up, w_down, router=True, shared=None):
    """Whole backward step with MXFP8 grouped GEMMs, given the forward dict from
    layer_fwd_mx.  router=False: routing held fixed (no router gradient)."""
    T, k = fwd["gate"].shape
    dy_perm, dgate = combine_bwd(dY, fwd["y_perm"], fwd["slot_of_pair"], fwd["gate"])
    b = bf16_rne
    g = grouped_swiglu_bwd_mx(b(dy_perm), fwd["x_perm"], b(fwd["h"]), b(fwd["u"]), b(fwd["a"]),
                              fwd["offsets"], w_gate, w_up, w_down)
    dx = unpermute_sum(g["dx_perm"], fwd["slot_of_pair"], T, k)
    out = dict(dy_perm=dy_perm, dgate=dgate, dx_experts=dx, **g)
    if router:
        dz, dw_r, dx_r = route_bwd(dgate, fwd["gate"], fwd["idx"], x, w_r)
        out.update(dz=dz, dw_r=dw_r)
        dx = dx + dx_r
    if shared is not None:
        out.update(shared_expert_bwd_mx(dY, x, fwd, shared))
        dx = dx + out["shared_dx"]
    out["dx"] = dx
    return out
