"""Failure detection on the GPU without a fault: a bounded wait that nothing ends runs out.

The library's test hook makes each later single-CTA grouped GEMM launch wait on a barrier
that nothing arrives on, with a 20 ms limit.  The wait runs out, every role of the kernel
stops, the copies and MMAs already issued are drained, the kernel returns, and the error word
reports MOE_ERR_DEVICE_TIMEOUT.  The test then turns the hook off and checks that the next
calls on the same context run normally and match the oracle.  All shapes here use single-CTA
tiles (the hook does not apply to CTA pairs).
"""
import numpy as np
import pytest

import routing_grouped_expert_softmax_b200 as moe
from oracle import moe_ref as ref
from tests.gpu_util import check, dev, dev_i32, grid, host, offsets_of, random_counts

pytestmark = pytest.mark.gpu

STALL_NS = 20_000_000     # 20 ms


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    import torch
    assert torch.cuda.is_available()
    from routing_grouped_expert_softmax_b200 import build
    build.build()


def _problem(seed=3):
    rng = np.random.default_rng(seed)
    d, f, E = 128, 128, 8
    counts = random_counts(E, 200, rng)
    offsets = offsets_of(counts)
    P = int(offsets[-1])
    x = grid(rng.standard_normal((P, d), dtype=np.float32), "bf16")
    dy = grid(rng.standard_normal((P, d), dtype=np.float32), "bf16")
    w = [grid(rng.standard_normal(shape, dtype=np.float32) / 8, "bf16") for shape in ((E, d, f), (E, d, f), (E, f, d))]
    return d, f, E, P, offsets, x, dy, w


def _run(cfg, ws, bufs):
    (xd, offd, wgd, wud, wdd, dyd, hu, a, y, dhu, dxp, dwg, dwu, dwd) = bufs
    moe.moe_grouped_swiglu_fwd(cfg, xd, offd, wgd, wud, wdd, hu, a, y, ws)
    moe.moe_grouped_swiglu_bwd(cfg, dyd, xd, hu, a, offd, wgd, wud, wdd, dhu, dxp, dwg, dwu, dwd, ws)


def test_wait_that_nothing_ends_times_out_and_the_context_stays_usable():
    import torch
    d, f, E, P, offsets, x, dy, (wg, wu, wd) = _problem()
    cfg = moe.config(P, d, E, 1, f)
    ws = moe.alloc_workspace(cfg)
    bf = dict(dtype=torch.bfloat16, device="cuda")
    bufs = (dev(x, "bf16"), dev_i32(offsets), dev(wg, "bf16"), dev(wu, "bf16"), dev(wd, "bf16"), dev(dy, "bf16"),
            torch.empty(P, 2 * f, **bf), torch.empty(P, f, **bf), torch.empty(P, d, **bf),
            torch.empty(P, 2 * f, **bf), torch.empty(P, d, **bf), torch.empty(E, d, f, **bf),
            torch.empty(E, d, f, **bf), torch.empty(E, f, d, **bf))
    assert moe.moe_get_error(ws) == 0
    moe.moe_debug_set_gemm_stall_ns(STALL_NS)
    try:
        _run(cfg, ws, bufs)          # six launches, each stops at its first wait
        code = moe.moe_get_error(ws)
    finally:
        moe.moe_debug_set_gemm_stall_ns(0)
    assert code & moe.MOE_ERR_DEVICE_TIMEOUT
    assert not code & ~(moe.MOE_ERR_DEVICE_TIMEOUT | moe.MOE_ERR_DEVICE_INDEX | moe.MOE_ERR_DEVICE_NAN)

    # the same context, hook off: the normal path runs and agrees with the oracle
    _run(cfg, ws, bufs)
    assert moe.moe_get_error(ws) == 0
    h, u, a, y = ref.grouped_swiglu(x, offsets, wg, wu, wd)
    hu_g = host(bufs[6])
    check(hu_g[:, :f], h, 2e-2, "after timeout h")
    check(host(bufs[8]), y, 2e-2, "after timeout y_perm")
    g = ref.grouped_swiglu_bwd(dy, x, ref.bf16_rne(h), ref.bf16_rne(u), ref.bf16_rne(a), offsets, wg, wu, wd)
    check(host(bufs[10]), g["dx_perm"], 2e-2, "after timeout dx_perm")
    for n, t in (("dw_gate", bufs[11]), ("dw_up", bufs[12]), ("dw_down", bufs[13])):
        check(host(t), g[n], 2e-2, f"after timeout {n}")

