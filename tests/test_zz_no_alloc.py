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

# the library's fixed scratch: ceil(T*k / 1024) * E int32 histogram entries at most
SCRATCH_ENTRIES = 65536


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    import torch
    assert torch.cuda.is_available()
    from routing_grouped_expert_softmax_b200 import build
    build.build()


def _bufs(T, E, k):
    import torch
    P = T * k
    return [torch.full((max(n, 1),), -7, dtype=torch.int32, device="cuda") for n in (E, E + 1, P, P)]


def _compare_twice(T, E, k, idx):
    """The workspace version once, then the allocation-free version twice in a row."""
    import torch
    cfg = moe.config(T, 128, E, k, 128)
    d_idx = torch.from_numpy(np.ascontiguousarray(idx, np.int32).reshape(-1)).cuda() if T else \
        torch.zeros(1, dtype=torch.int32, device="cuda")
    ref_out = _bufs(T, E, k)
    ws = moe.alloc_workspace(cfg)
    moe.moe_build_offsets(cfg, d_idx, *ref_out, ws)
    assert moe.moe_get_error(ws) == 0
    for _ in range(2):
        out = _bufs(T, E, k)
        moe.moe_build_offsets_noalloc(cfg, d_idx, *out)
        torch.cuda.synchronize()
        for a, b in zip(out, ref_out):
            assert torch.equal(a, b)


def test_noalloc_matches_workspace_version_twice():
    cases = [(4097, 128, 4, "skewed"), (3000, 8, 4, "uniform")]   # different shapes, back to back
    for T, E, k, kind in cases:
        if kind == "skewed":
            idx = gen.skewed_routing_idx(T, E, k, seed=T)
        else:
            idx, _ = gen.uniform_random_routing(T, E, k, seed=T)
        _compare_twice(T, E, k, idx)


def test_noalloc_largest_admitted_shape_and_empty_batch():
    # T*k = 262144 pairs at E = 256: exactly 256 blocks x 256 experts = 65536 entries
    T, E, k = 262144, 256, 1
    assert -(-T * k // 1024) * E == SCRATCH_ENTRIES
    idx = gen.skewed_routing_idx(T, E, k, seed=11)
    _compare_twice(T, E, k, idx)
    _compare_twice(0, 8, 2, None)


def test_noalloc_rejects_shapes_beyond_its_scratch():
    import torch
    # one pair more than the largest admitted shape needs a 257th block of 256 entries
    T, E, k = 262145, 256, 1
    cfg = moe.config(T, 128, E, k, 128)
    # real buffers of the right sizes, with valid expert indices, so that the call would
    # still be well defined if the size check ever stopped rejecting it
    idx = torch.zeros(T * k, dtype=torch.int32, device="cuda")
    out = _bufs(T, E, k)
    with pytest.raises(moe.MoeError) as e:
        moe.moe_build_offsets_noalloc(cfg, idx, *out)
    assert e.value.code == moe.MOE_ERR_UNSUPPORTED
    torch.cuda.synchronize()
    for b in out:
        assert int(b.min()) == -7 and int(b.max()) == -7   # nothing was launched
