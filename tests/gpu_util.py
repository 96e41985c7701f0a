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
