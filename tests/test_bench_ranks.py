"""bench.py's multi-rank plumbing on two gloo ranks (CPU, no GPU): the time reported is the
slowest rank's, the value is the whole job's tokens over that time, and the reference arm
runs on rank 0 only."""
import argparse
import contextlib
import io
import os
import socket
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE="2", LOCAL_RANK=str(rank))
    import datetime

    import torch.distributed as dist
    dist.init_process_group("gloo", rank=rank, world_size=2, timeout=datetime.timedelta(seconds=60))
    sys.path.insert(0, ROOT)
    import bench
    try:
        ws, r, _ = bench.dist_env()
        ms = bench.max_over_ranks(1.5 + 2.0 * rank, "cpu")       # rank 1 is the slower one
        value = bench.job_tokens_per_s(8192, ws, ms)
        out = io.StringIO()
        args = argparse.Namespace(workload="e128_fwd_bwd", steps=1, warmup=0, cpu_tokens=4)
        printed = None
        if rank == 1:                                             # rank 0 would run the oracle
            with contextlib.redirect_stdout(out):
                bench.run_reference(args)
            printed = out.getvalue()
        dist.barrier()
        q.put((rank, ws, r, ms, value, printed))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_take_the_slowest_time():
    import multiprocessing as mp
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    ps = [ctx.Process(target=_worker, args=(r, port, q)) for r in range(2)]
    for p in ps:
        p.start()
    res = sorted(q.get(timeout=120) for _ in ps)
    for p in ps:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, ws, r, ms, value, printed in res:
        assert (ws, r) == (2, rank)
        assert ms == 3.5                          # the max over ranks
        assert value == pytest.approx(8192 * 2 / 3.5e-3)
    assert res[1][5] == ""                        # the reference arm prints nothing off rank 0


def test_single_process_keeps_its_own_time():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(2.25, "cpu") == 2.25
    assert bench.job_tokens_per_s(8192, 1, 2.0) == pytest.approx(4.096e6)


def test_gemm_algorithmic_bytes_and_binding_roof():
    sys.path.insert(0, ROOT)
    import bench
    P, d, f = 8192 * 4, 2048, 1024
    MB = 2 ** 20
    # C3: weights [Wg|Wu] 1024 MiB and Wd 512 MiB (bf16); x_perm, dy_perm, dx_perm 128 MiB;
    # [h|u], [dh|du] 128 MiB; a 64 MiB.  Forward: GU reads W 1024 + x 128, writes hu 128 + a 64;
    # down reads Wd 512 + a 64, writes y 128.
    fwd, bwd = bench.gemm_algorithmic_bytes(P, d, f, 128, "native")
    assert fwd == (1024 + 128 + 128 + 64 + 512 + 64 + 128) * MB
    # backward: dgrad-down 512 + 128 + 128 read, 128 written; wgrad-down 64 + 128 read, 512
    # written; dgrad-gu 128 + 1024 read, 128 written; wgrad-gu 128 + 128 read, 1024 written
    assert bwd == (512 + 128 + 128 + 128 + 64 + 128 + 512 + 128 + 1024 + 128 + 128 + 128 + 1024) * MB
    flops = 18.0 * P * d * f
    pk = dict(hbm=6551.4, bf16=1636.8)
    t_byte = (fwd + bwd) / (pk["hbm"] * 1e9)
    assert t_byte > flops / (pk["bf16"] * 1e12)                 # E=128: HBM-bound
    f8, b8 = bench.gemm_algorithmic_bytes(P, d, f, 8, "native")
    assert (f8 + b8) / (pk["hbm"] * 1e9) < flops / (pk["bf16"] * 1e12)    # E=8: tensor-bound
    # MXFP8 operands are read as codes plus one scale byte per 32
    fm, bm = bench.gemm_algorithmic_bytes(P, d, f, 128, "mxfp8")
    assert fm < fwd and bm < bwd


def test_launch_count():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.count_launches("router") == 20
    assert bench.count_launches("uniform") == 15
    assert bench.count_launches("router", "mxfp8") == 22
    assert bench.count_launches("router", "native", shared=True) == 30
    assert bench.count_launches("router", "native", recompute=True) == 21
