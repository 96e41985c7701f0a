"""moe_build_offsets_noalloc against moe_build_offsets.

Callers that cannot allocate device memory (their memory is all handed to their own pool,
or their interface has no way to pass a workspace) use the allocation-free entry point,
whose scratch lives in a fixed array inside the library.  It must give exactly the
workspace version's outputs, on consecutive calls that reuse the array.  This file is
collected last, so a run that stops at the first failure has already run every other test.
"""
import numpy as np
import pytest

import routing_grouped_expert_softmax_b200 as moe
from routing_grouped_expert_softmax_b200 import inputs as gen

pytestmark = pytest.mark.gpu


def _bufs(T, E, k):
    import torch
    P = T * k
    return [torch.full((n,), -7, dtype=torch.int32, device="cuda") for n in (E, E + 1, P, P)]


def test_noalloc_matches_workspace_version_twice():
    import torch
    from routing_grouped_expert_softmax_b200 import build
    assert torch.cuda.is_available()
    build.build()
    cases = [(4097, 128, 4, "skewed"), (3000, 8, 4, "uniform")]   # different shapes, back to back
    for T, E, k, kind in cases:
        if kind == "skewed":
            idx = gen.skewed_routing_idx(T, E, k, seed=T)
        else:
            idx, _ = gen.uniform_random_routing(T, E, k, seed=T)
        cfg = moe.config(T, 128, E, k, 128)
        d_idx = torch.from_numpy(idx).cuda()
        ref_out = _bufs(T, E, k)
        ws = moe.alloc_workspace(cfg)
        moe.moe_build_offsets(cfg, d_idx, *ref_out, ws)
        for _ in range(2):
            out = _bufs(T, E, k)
            moe.moe_build_offsets_noalloc(cfg, d_idx, *out)
            torch.cuda.synchronize()
            for a, b in zip(out, ref_out):
                assert torch.equal(a, b)


def test_noalloc_rejects_shapes_beyond_its_scratch():
    cfg = moe.config(262144, 128, 256, 1, 128)      # ceil(262144/1024) * 256 = 65536 fits
    cfg_big = moe.config(262145, 128, 256, 1, 128)  # one more block does not
    import ctypes
    L = moe.lib()
    assert L.moe_build_offsets_noalloc(ctypes.byref(cfg_big), 16, 16, 16, 16, 16, None) == \
        moe.MOE_ERR_UNSUPPORTED
    assert moe.moe_workspace_size(cfg) > 0
