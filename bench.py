"""Benchmark: one MoE layer step (forward + backward) on B200, through libmoe's C ABI.

Workload (default): T=8192 tokens, d=2048, E=128 experts, top-4, SwiGLU ffn=1024, bf16,
seeded synthetic inputs (x ~ N(0,1), weights ~ N(0,0.02), dY ~ N(0,1)).  A step is
moe_layer_fwd + moe_layer_bwd: router, routing metadata, permute, grouped SwiGLU GEMMs,
combine, and the backward of each.  The expert weights (1.6 GB) exceed L2 (126 MB), so
no L2 flush is needed between steps.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

N > 1 runs one independent replica per GPU (weak scaling; the layer step has no
data-path exchange), launched by torchrun.  Rank 0 prints one JSON line.
"""
from __future__ import annotations

import argparse
import json
import os
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

WORKLOADS = {
    # name: (T, d, E, k, f, skew, routing)
    "e128_fwd_bwd": (8192, 2048, 128, 4, 1024, False, "router"),
    "e8_fwd_bwd": (8192, 2048, 8, 4, 1024, False, "router"),
    "e128_t16k_skew_fwd_bwd": (16384, 2048, 128, 4, 1024, True, "router"),
    "e128_t16k_uniform_fwd_bwd": (16384, 2048, 128, 4, 1024, False, "uniform"),
    # the MXFP8 workload's shapes and inputs in bf16 (the pair that MXFP8 is compared within)
    "e128_t16k_fwd_bwd": (16384, 2048, 128, 4, 1024, False, "router"),
    # a smaller case of the same kernels for profiler captures (still larger than L2)
    "profile_e32_t4k": (4096, 2048, 32, 4, 1024, False, "router"),
    # 256 rows per expert, as at T=8192, E=128, k=4
    "profile_e32_t2k": (2048, 2048, 32, 4, 1024, False, "router"),
    "profile_e32_t2k_mxfp8": (2048, 2048, 32, 4, 1024, False, "router", "mxfp8"),
    # the same shapes with every grouped-GEMM operand in MXFP8 (E4M3 + E8M0 per 32)
    "e128_t16k_mxfp8_fwd_bwd": (16384, 2048, 128, 4, 1024, False, "router", "mxfp8"),
    "e128_mxfp8_fwd_bwd": (8192, 2048, 128, 4, 1024, False, "router", "mxfp8"),
    # E=8 (4096 rows per expert: the GEMMs are compute-bound) with MXFP8 grouped GEMMs
    "e8_mxfp8_fwd_bwd": (8192, 2048, 8, 4, 1024, False, "router", "mxfp8"),
    # the C3 shapes plus one shared expert (every token, weight 1) of the routed experts' shape
    "e128_shared_fwd_bwd": (8192, 2048, 128, 4, 1024, False, "router", "native", {"shared": True}),
    # the C3 shapes keeping no [h | u] between forward and backward (recomputed there)
    "e128_recompute_fwd_bwd": (8192, 2048, 128, 4, 1024, False, "router", "native", {"recompute": True}),
}
DEFAULT = "e128_fwd_bwd"
# Timed after the main workload, each in a short run of its own, and reported beside it: the
# pages' two comparisons -- 8 against 128 experts at equal active FLOPs (qidao123.com, section
# "新闻原文"), and MXFP8 against bf16 (unite.ai, section "Παραλληλισμός, Ακρίβεια και
# Τεχνικές Μνήμης") -- on this layer.
SWEEP = ("e128_fwd_bwd", "e8_fwd_bwd", "e8_mxfp8_fwd_bwd", "e128_t16k_fwd_bwd", "e128_t16k_mxfp8_fwd_bwd")


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as fh:
            j = json.load(fh)
        return dict(hbm=j["hbm_gbs"], bf16=j["bf16_tflops"], bf16_sus=j.get("bf16_tflops_sustained"),
                    src="measured")
    return dict(hbm=6650.0, bf16=1590.0, bf16_sus=1400.0, src="fallback")


class ClockSampler:
    """nvidia-smi clock/throttle samples during the timed region."""

    def __init__(self, index):
        self.index = index
        self.samples = []
        self.proc = None

    def __enter__(self):
        q = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
             "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
             "clocks_event_reasons.sw_power_cap")
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), f"--query-gpu={q}", "--format=csv,noheader,nounits",
                 "-lms", "50"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except (FileNotFoundError, OSError):
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            parts = [s.strip() for s in line.split(",")]
            if len(parts) >= 7:
                self.samples.append((time.time(), parts))

    def window(self, t0, t1):
        self.t0, self.t1 = t0, t1

    def __exit__(self, *a):
        if self.proc:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        t0, t1 = getattr(self, "t0", 0.0), getattr(self, "t1", 1e30)
        rows = [p for (t, p) in self.samples if t0 <= t <= t1 + 0.15]
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"], "samples": 0}

        def num(v):
            try:
                return float(v)
            except ValueError:
                return None
        sm = [v for v in (num(r[0]) for r in rows) if v is not None]
        mx = [v for v in (num(r[1]) for r in rows) if v is not None]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[3 + i] == "Active"})
        return {"sm_mhz": float(np.median(sm)) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(rows)}


def dist_env():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


def max_over_ranks(x: float, device: str) -> float:
    """The largest x over all ranks of the process group (x itself on one process): a
    multi-GPU time is the slowest rank's."""
    import torch
    import torch.distributed as dist
    if not dist.is_initialized() or dist.get_world_size() == 1:
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_tokens_per_s(tokens_per_rank: int, world: int, ms: float) -> float:
    """Whole-job throughput: the tokens all ranks processed over the slowest rank's time."""
    return tokens_per_rank * world / (ms * 1e-3)


def make_inputs(name, seed):
    from routing_grouped_expert_softmax_b200 import inputs as gen
    T, d, E, k, f, skew, routing = WORKLOADS[name][:7]
    inp = gen.make_layer_inputs(T, d, E, k, f, dtype="bf16", seed=seed, skew=skew)
    if routing == "uniform":
        inp.extra["idx"], inp.extra["gate"] = gen.uniform_random_routing(T, E, k, seed=seed)
    return inp


def to_dev_bf16(a, torch):
    from routing_grouped_expert_softmax_b200 import inputs as gen
    return torch.from_numpy(gen.bf16_bits(a).view(np.int16)).view(torch.bfloat16).cuda()


def _workload_spec(name):
    T, d, E, k, f, skew, routing = WORKLOADS[name][:7]
    prec = WORKLOADS[name][7] if len(WORKLOADS[name]) > 7 else "native"
    opts = WORKLOADS[name][8] if len(WORKLOADS[name]) > 8 else {}
    return T, d, E, k, f, skew, routing, prec, bool(opts.get("shared")), bool(opts.get("recompute"))


class Layer:
    """One workload's device buffers and its step (moe_layer_fwd + moe_layer_bwd)."""

    def __init__(self, name, inp):
        import torch

        import routing_grouped_expert_softmax_b200 as moe
        self.moe, self.name, self.inp = moe, name, inp
        T, d, E, k, f, skew, routing, prec, shared, recompute = _workload_spec(name)
        self.T, self.d, self.E, self.k, self.f, self.prec = T, d, E, k, f, prec
        self.routing, self.shared, self.recompute = routing, shared, recompute
        self.cfg = moe.config(T, d, E, k, f, dtype="bf16", prec=prec)
        self.st = torch.cuda.current_stream()
        self.ws = moe.alloc_workspace(self.cfg)
        self.saved = moe.alloc_saved(self.cfg, logits=False, shared=shared, recompute=recompute)
        self.grads = moe.alloc_grads(self.cfg, router=(routing == "router"), shared=shared)
        self.x = to_dev_bf16(inp.x, torch)
        self.dy = to_dev_bf16(inp.dy, torch)
        self.wr, self.wg, self.wu, self.wd = (to_dev_bf16(a, torch) for a in (inp.w_r, inp.w_gate, inp.w_up,
                                                                              inp.w_down))
        self.bias = torch.from_numpy(inp.bias).cuda() if inp.bias is not None else None
        sh = None
        if shared:
            from routing_grouped_expert_softmax_b200 import inputs as gen
            sh = tuple(to_dev_bf16(a, torch) for a in gen.make_shared_expert(d, f, seed=1))
        self.w = moe.layer_weights(self.wr, self.bias, self.wg, self.wu, self.wd, shared=sh)
        self.y = torch.empty(T, d, dtype=torch.bfloat16, device="cuda")
        self.fwd_fn = moe.moe_layer_fwd
        if routing == "uniform":
            self.saved["topk_idx"].copy_(torch.from_numpy(inp.extra["idx"]))
            self.saved["topk_gate"].copy_(torch.from_numpy(inp.extra["gate"]))
            self.fwd_fn = moe.moe_layer_fwd_routed
        self.launches_per_step = count_launches(routing, prec, shared, recompute)

    def step(self, x=None, dy=None, y=None, grads=None):
        self.fwd_fn(self.cfg, self.w, self.x if x is None else x, self.y if y is None else y, self.saved, self.ws,
                    self.st)
        self.moe.moe_layer_bwd(self.cfg, self.w, self.x if x is None else x, self.dy if dy is None else dy,
                               self.saved, self.grads if grads is None else grads, self.ws, self.st)

    def layer_bytes(self):
        """Device bytes the layer's own buffers hold: workspace, forward context, gradients."""
        n = self.ws.numel()
        for dct in (self.saved, self.grads):
            n += sum(t.numel() * t.element_size() for t in dct.values() if t is not None)
        return n

    def load(self):
        c = self.saved["counts"].cpu().numpy().astype(np.int64)
        m = c.mean()
        return {"max_over_mean": float(c.max() / m), "min_over_mean": float(c.min() / m),
                "empty_experts": int((c == 0).sum()), "counts": c.tolist()}


def profiled_launches(step):
    """Kernels of this library (namespace moe) that one step launches, counted by CUPTI through
    torch.profiler on one untimed step; None if the profiler is unavailable."""
    import torch
    try:
        from torch.profiler import ProfilerActivity, profile
        torch.cuda.synchronize()
        with profile(activities=[ProfilerActivity.CUDA]) as prof:
            step()
            torch.cuda.synchronize()
        names = [e.name for e in prof.events() if e.device_type == torch.autograd.DeviceType.CUDA]
        n = sum(1 for nm in names if "moe::" in nm)
        return n if n > 0 else None
    except Exception:
        return None


def time_steps(layer, steps, warmup, barrier):
    """Device time of `steps` back-to-back steps (CUDA events on the launching stream), ms per step."""
    import torch
    for _ in range(warmup):
        layer.step()
    torch.cuda.synchronize()
    assert layer.moe.moe_get_error(layer.ws) == 0
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier()
    e0.record(layer.st)
    for _ in range(steps):
        layer.step()
    e1.record(layer.st)
    barrier()
    assert layer.moe.moe_get_error(layer.ws) == 0
    return e0.elapsed_time(e1) / steps


def run_ours(args):
    import torch
    import torch.distributed as dist

    import routing_grouped_expert_softmax_b200 as moe
    from routing_grouped_expert_softmax_b200 import build
    ws_n, rank, local = dist_env()
    if ws_n > 1:
        dist.init_process_group("nccl", timeout=__import__("datetime").timedelta(seconds=120))
    torch.cuda.set_device(local)
    build.build()
    name = args.workload
    T, d, E, k, f, skew, routing, prec, shared, recompute = _workload_spec(name)
    inp = make_inputs(name, seed=0)
    torch.cuda.reset_peak_memory_stats()
    base_mem = torch.cuda.memory_allocated()
    L = Layer(name, inp)
    st = L.st
    cfg, saved, grads, ws = L.cfg, L.saved, L.grads, L.ws
    wg, wu, wd = L.wg, L.wu, L.wd
    x, dy, y = L.x, L.dy, L.y
    step = L.step
    launches_per_step = L.launches_per_step

    def barrier():
        if ws_n > 1:
            dist.barrier()
        torch.cuda.synchronize()

    clk = ClockSampler(local)
    clk.__enter__()
    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    assert moe.moe_get_error(ws) == 0
    time.sleep(0.3)     # let the sampler start reporting before the timed region

    # ---- headline: K whole steps, device-timed with CUDA events on the launching stream
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier()
    t_start = time.time()
    e0.record(st)
    for _ in range(args.steps):
        step()
    e1.record(st)
    barrier()
    clk.window(t_start, time.time())
    clk.__exit__()
    ms_max = max_over_ranks(e0.elapsed_time(e1) / args.steps, "cuda")
    peak_mem = torch.cuda.max_memory_allocated() - base_mem
    load = L.load()
    counted = None if args.no_cupti else profiled_launches(step)
    if counted is not None:
        launches_per_step = counted

    # ---- step-time spread: up to 50 more steps, each between its own pair of events
    n_spread = min(args.steps, 50)
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(n_spread)]
    for a_ev, b_ev in evs:
        a_ev.record(st)
        step()
        b_ev.record(st)
    torch.cuda.synchronize()
    per_step = sorted(a_ev.elapsed_time(b_ev) for a_ev, b_ev in evs)
    p50 = max_over_ranks(float(np.percentile(per_step, 50)), "cuda") if per_step else None
    p90 = max_over_ranks(float(np.percentile(per_step, 90)), "cuda") if per_step else None

    # ---- the grouped GEMMs alone (6 tcgen05 launches per step), same stream and inputs
    g0, g1, g2 = (torch.cuda.Event(enable_timing=True) for _ in range(3))
    hu_buf = saved["hu"] if saved["hu"] is not None else grads["dhu"]   # recompute keeps no h | u
    x_perm, dy_perm = saved["x_perm"], grads["dy_perm"]
    if x_perm is None:     # the MXFP8 layer moved the rows in MXFP8 only: make the bf16 ones
        x_perm = torch.empty(L.T * L.k, L.d, dtype=torch.bfloat16, device="cuda")
        moe.moe_permute(cfg, L.x, saved["slot_of_pair"], x_perm, st)
    if dy_perm is None:
        dy_perm = torch.empty(L.T * L.k, L.d, dtype=torch.bfloat16, device="cuda")
        moe.moe_combine_bwd(cfg, L.dy, saved["y_perm"], saved["slot_of_pair"], saved["topk_gate"], dy_perm,
                            grads["dgate"], st)
    fwd_ms = bwd_ms = 0.0
    for _ in range(args.steps):
        g0.record(st)
        moe.moe_grouped_swiglu_fwd(cfg, x_perm, saved["offsets"], wg, wu, wd, hu_buf,
                                   saved["a"], saved["y_perm"], ws, st)
        g1.record(st)
        moe.moe_grouped_swiglu_bwd(cfg, dy_perm, x_perm, hu_buf, saved["a"],
                                   saved["offsets"], wg, wu, wd, grads["dhu"], grads["dx_perm"],
                                   grads["dw_gate"], grads["dw_up"], grads["dw_down"], ws, st)
        g2.record(st)
        g2.synchronize()
        fwd_ms += g0.elapsed_time(g1)
        bwd_ms += g1.elapsed_time(g2)
    fwd_ms /= args.steps
    bwd_ms /= args.steps

    # ---- end to end through the public API with host buffers: x, dY in; y, dx out.
    # Inputs and outputs are double-buffered on the device so that step i+1's upload and
    # step i's download run on their own streams while step i computes; every step's copies
    # are inside the timed region.
    hx = torch.from_numpy(gen_bits(inp.x)).pin_memory()
    hdy = torch.from_numpy(gen_bits(inp.dy)).pin_memory()
    hy = torch.empty(T * d, dtype=torch.int16).pin_memory()
    hdx = torch.empty(T * d, dtype=torch.int16).pin_memory()
    xs = [x, torch.empty_like(x)]
    dys = [dy, torch.empty_like(dy)]
    ys = [y, torch.empty_like(y)]
    gs = [grads, dict(grads, dx=torch.empty_like(grads["dx"]))]
    s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()
    ev = {n: [torch.cuda.Event(), torch.cuda.Event()] for n in ("in", "comp", "out")}

    def upload(b):
        xs[b].view(torch.int16).view(-1).copy_(hx, non_blocking=True)
        dys[b].view(torch.int16).view(-1).copy_(hdy, non_blocking=True)
        ev["in"][b].record(s_in)

    barrier()
    e0.record(st)
    s_in.wait_stream(st)
    s_out.wait_stream(st)
    with torch.cuda.stream(s_in):
        upload(0)
    for i in range(args.steps):
        b, nb = i % 2, (i + 1) % 2
        if i + 1 < args.steps:
            with torch.cuda.stream(s_in):
                if i >= 1:
                    s_in.wait_event(ev["comp"][nb])      # step i-1 is done with buffers nb
                upload(nb)
        st.wait_event(ev["in"][b])
        if i >= 2:
            st.wait_event(ev["out"][b])                  # step i-2's outputs have left
        step(xs[b], dys[b], ys[b], gs[b])
        ev["comp"][b].record(st)
        with torch.cuda.stream(s_out):
            s_out.wait_event(ev["comp"][b])
            hy.copy_(ys[b].view(torch.int16).view(-1), non_blocking=True)
            hdx.copy_(gs[b]["dx"].view(torch.int16).view(-1), non_blocking=True)
            ev["out"][b].record(s_out)
    st.wait_stream(s_out)
    e1.record(st)
    barrier()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1) / args.steps, "cuda")
    assert moe.moe_get_error(ws) == 0
    layer_gib = L.layer_bytes() / 2 ** 30
    del L, xs, dys, ys, gs, saved, grads, ws, x, dy, y, hx, hdy, hy, hdx
    torch.cuda.empty_cache()

    # ---- the sweep's other points, each in its own short timed run: E=8 at equal active
    # FLOPs (the pages' 8 -> 128 experts comparison) and the T=16384 shapes in bf16 and in
    # MXFP8 (the pages' MXFP8 against bf16 comparison)
    sweep = {}
    if not args.no_sweep:
        cache = {}
        for other in SWEEP:
            if other == name:
                sweep[other] = ms_max
                continue
            key = _workload_spec(other)[:7]
            if key not in cache:
                cache.clear()
                cache[key] = make_inputs(other, seed=0)
            lo = Layer(other, cache[key])
            sweep[other] = max_over_ranks(time_steps(lo, min(args.steps, 30), max(args.warmup, 3), barrier), "cuda")
            del lo
            torch.cuda.empty_cache()
        cache.clear()

    P = T * k
    flops_fwd = 6.0 * P * d * f
    flops_bwd = 12.0 * P * d * f
    pk = peaks()
    gemm_ms = fwd_ms + bwd_ms
    tflops = (flops_fwd + flops_bwd) / (gemm_ms * 1e-3) / 1e12
    # The six GEMMs are timed per step between events, a loop of well under a second: the
    # tensor roof is the burst bf16 figure.  An MXFP8 contraction is measured against the fp8
    # peak: the measured bf16 peak times the nominal fp8 / bf16 ratio (4.5 / 2.25).
    peak_tc = pk["bf16"] * (2.0 if prec == "mxfp8" else 1.0)
    bytes_fwd, bytes_bwd = gemm_algorithmic_bytes(P, d, f, E, prec)
    gbs = (bytes_fwd + bytes_bwd) / (gemm_ms * 1e-3) / 1e9
    # the binding roof: whichever of the FLOP time and the byte time is longer
    t_flop = (flops_fwd + flops_bwd) / (peak_tc * 1e12)
    t_byte = (bytes_fwd + bytes_bwd) / (pk["hbm"] * 1e9)
    hbm_bound = t_byte > t_flop
    tr = GEMM_TRAFFIC.get(name)
    traffic = tr["bytes"] if tr and tr["sources_sha1"] == gemm_sources_sha1() else None
    out = {
        "metric": "MoE-layer tokens/s (E=128,k=4,bf16 fwd+bwd) 1xB200; grouped-GEMM % TC peak",
        "value": job_tokens_per_s(T, ws_n, ms_max),
        "unit": "tokens/s",
        "n_gpus": ws_n,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": ms_max,
        "ms_per_step_p50": p50, "ms_per_step_p90": p90,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16" if prec == "native" else "mxfp8 (e4m3 + e8m0/32) GEMMs, bf16 storage",
        "data": "synthetic (seeded N(0,1) activations, N(0,0.02) weights)",
        "config": {"workload": name, "T": T, "d_model": d, "experts": E, "top_k": k, "ffn": f,
                   "routing": "skewed (Zipf bias)" if skew else routing, "gemm_precision": prec,
                   "parallelism": f"replicas x{ws_n}" if ws_n > 1 else "single GPU",
                   "shared_expert": shared, "recompute_hu": recompute,
                   "l2": "no flush: 1.6 GB of expert weights per step exceed the 126 MB L2"},
        "roofline": {"kernel": "grouped SwiGLU GEMMs (6 tcgen05 launches per step: fwd gate/up, fwd down, "
                               "dgrad down, wgrad down, dgrad gate/up, wgrad gate/up)",
                     "bound": "hbm" if hbm_bound else "tensor",
                     "achieved": gbs if hbm_bound else tflops,
                     "peak": pk["hbm"] if hbm_bound else peak_tc,
                     "unit": "GB/s" if hbm_bound else "TFLOP/s",
                     "frac": gbs / pk["hbm"] if hbm_bound else tflops / peak_tc,
                     "peak_source": (f"{pk['src']} HBM copy" if hbm_bound else
                                     f"{pk['src']} bf16 burst" + (" x 2 (nominal fp8/bf16)" if prec == "mxfp8" else "")),
                     "traffic": traffic,
                     "algorithmic_bytes_per_step": bytes_fwd + bytes_bwd,
                     "flops_per_step": flops_fwd + flops_bwd,
                     "tensor_tflops": tflops, "tensor_frac": tflops / peak_tc,
                     "tensor_peak_source": f"{pk['src']} bf16 burst" + (" x 2" if prec == "mxfp8" else ""),
                     "hbm_gbs": gbs, "hbm_frac": gbs / pk["hbm"],
                     "fwd_ms": fwd_ms, "bwd_ms": bwd_ms,
                     "fwd_tflops": flops_fwd / (fwd_ms * 1e-3) / 1e12,
                     "bwd_tflops": flops_bwd / (bwd_ms * 1e-3) / 1e12},
        "e2e": {"value": job_tokens_per_s(T, ws_n, e2e_ms), "unit": "tokens/s",
                "h2d_bytes_per_step": 2 * T * d * 2, "d2h_bytes_per_step": 2 * T * d * 2},
        "gpu_launches": launches_per_step * args.steps,
        "gpu_launches_per_step": launches_per_step,
        "gpu_launches_source": "CUPTI count of one untimed step" if counted is not None else "formula",
        "clocks": clk.summary(),
        "load": load,
        "memory": {"peak_gib": peak_mem / 2 ** 30, "layer_buffers_gib": layer_gib,
                   "what": "peak torch-allocated device memory of the workload (inputs, weights, forward "
                           "context, gradients, workspace; the library allocates nothing)"},
    }
    if sweep:
        out["sweep_ms_per_step"] = sweep
        r = {}
        if "e8_fwd_bwd" in sweep and "e128_fwd_bwd" in sweep:
            r["e128_over_e8_time"] = sweep["e128_fwd_bwd"] / sweep["e8_fwd_bwd"]
        if "e128_t16k_fwd_bwd" in sweep and "e128_t16k_mxfp8_fwd_bwd" in sweep:
            r["mxfp8_speedup_over_bf16"] = sweep["e128_t16k_fwd_bwd"] / sweep["e128_t16k_mxfp8_fwd_bwd"]
        if "e8_fwd_bwd" in sweep and "e8_mxfp8_fwd_bwd" in sweep:
            r["mxfp8_speedup_over_bf16_e8"] = sweep["e8_fwd_bwd"] / sweep["e8_mxfp8_fwd_bwd"]
        out["sweep_ratios"] = r
    if rank == 0 and not args.no_cpu_baseline:
        out["cpu_baseline"] = cpu_baseline(inp, k, routing)
    if ws_n > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(out))


def gen_bits(a):
    from routing_grouped_expert_softmax_b200 import inputs as gen
    return gen.bf16_bits(a).view(np.int16).reshape(-1)


# DRAM bytes (read + write) of the six grouped-GEMM launches of one step, from one ncu
# capture (dram__bytes_read.sum + dram__bytes_write.sum, a one-pass metric) of the full-size
# workload, with the SHA-1 of the kernel sources it was taken on; a report carries it only
# while those sources are unchanged.
GEMM_TRAFFIC = {
    "e128_fwd_bwd": {"bytes": 6430130432, "sources_sha1": "3f56a09854c19adcc9f50d038b6e135376632e47"},
}
GEMM_SOURCES = ("grouped_gemm.cu", "tc_ptx.cuh", "common.cuh")


def gemm_sources_sha1():
    import hashlib
    h = hashlib.sha1()
    for f in GEMM_SOURCES:
        with open(os.path.join(ROOT, "routing_grouped_expert_softmax_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()


def gemm_algorithmic_bytes(P, d, f, E, prec):
    """Bytes the six grouped GEMMs of one step must move at least: every operand read once
    and every output written once per GEMM (fwd: gate/up, down; bwd: down-dgrad with the
    SwiGLU backward, down-wgrad, gate/up-dgrad, gate/up-wgrad).  MXFP8 operands are read as
    1-byte codes plus one scale byte per 32; outputs are bf16."""
    r = 1.0 + 1.0 / 32 if prec == "mxfp8" else 2.0   # bytes per operand element read
    w = 2.0                                          # bytes per output element written
    wgu, wd = E * d * 2 * f, E * f * d               # weight elements: [Wg | Wu], Wd
    fwd = (wgu * r + P * d * r + P * 2 * f * w + P * f * w) + (wd * r + P * f * r + P * d * w)
    bwd = ((wd * r + P * d * r + P * 2 * f * 2 + P * 2 * f * w)      # hu read in bf16
           + (P * f * r + P * d * r + wd * w)
           + (P * 2 * f * r + wgu * r + P * d * w)
           + (P * d * r + P * 2 * f * r + wgu * w))
    return fwd, bwd


def count_launches(routing, prec="native", shared=False, recompute=False):
    """Kernels one step launches (the fallback when the CUPTI count is unavailable): forward
    (router 1, metadata 3, permute 1, grouped GEMMs 2, combine 1) and backward (combine-bwd 1,
    grouped GEMMs 4, router transpose 1, router weight-gradient 3, unpermute-sum 1; bf16: one
    tail-buffer copy before each weight-gradient GEMM, per expert set).  MXFP8
    with the forward's weight copies kept for the backward adds 2 weight quantisers forward
    (the permute and the gate/up epilogue quantise x and a) and 2 token-axis quantisers
    backward (the combine's backward and the down projection's epilogue quantise dy and
    [dh | du]).  A shared expert adds its group offsets and 2 GEMMs forward, offsets and 4
    GEMMs backward (MXFP8: its operands through 3 + 7 quantisers); recompute adds one GEMM per
    expert set backward (MXFP8: with the quantiser of its input)."""
    fwd = (1 if routing == "router" else 0) + 3 + 1 + 2 + 1
    bwd = 1 + 4 + (5 if routing == "router" else 1)
    mx = prec == "mxfp8"
    sets = 2 if shared else 1
    n = fwd + bwd + (4 if mx else 2 * sets)
    if shared:
        n += 1 + 2 + 1 + 4 + (10 if mx else 0)
    if recompute:
        n += sets * (1 + (1 if mx else 0))
    return n


def _oracle_step(ref, inp, k, routing, fwd_only=False):
    """One layer step of the oracle on inp (the whole batch it holds)."""
    if routing == "uniform":
        fwd = ref.layer_fwd_routed(inp.x, inp.extra["idx"], inp.extra["gate"], inp.w_gate, inp.w_up, inp.w_down)
        if not fwd_only:
            ref.layer_bwd_routed(fwd, inp.dy, inp.w_gate, inp.w_up, inp.w_down)
    else:
        fwd = ref.layer_fwd(inp.x, inp.w_r, inp.w_gate, inp.w_up, inp.w_down, k, inp.bias)
        if not fwd_only:
            ref.layer_bwd(fwd, inp.dy, inp.x, inp.w_r, inp.w_gate, inp.w_up, inp.w_down)


def _token_sample(inp, n):
    import dataclasses
    extra = dict(inp.extra)
    if "idx" in extra:
        extra["idx"], extra["gate"] = extra["idx"][:n], extra["gate"][:n]
    return dataclasses.replace(inp, T=n, x=inp.x[:n], dy=inp.dy[:n], extra=extra)


def _blas_threads():
    try:
        from threadpoolctl import threadpool_info
        return max((i.get("num_threads", 1) for i in threadpool_info()), default=1)
    except Exception:
        return len(os.sched_getaffinity(0))


def cpu_baseline(inp, k, routing):
    """The CPU oracle (NumPy, per-expert loops, BLAS matmuls) in its float32 working precision
    on the host cores: the workload's whole batch, forward and forward + backward (median of
    two timed runs after one warm-up), and a 512-token sample of it on one thread."""
    from oracle import moe_ref as ref
    with ref.working_precision(np.float32):
        _oracle_step(ref, inp, k, routing)
        tf, tb = [], []
        for _ in range(2):
            t0 = time.perf_counter()
            _oracle_step(ref, inp, k, routing, fwd_only=True)
            tf.append(time.perf_counter() - t0)
            t0 = time.perf_counter()
            _oracle_step(ref, inp, k, routing)
            tb.append(time.perf_counter() - t0)
        one = None
        try:
            from threadpoolctl import threadpool_limits
            small = _token_sample(inp, min(512, inp.T))
            with threadpool_limits(limits=1):
                _oracle_step(ref, small, k, routing)
                t0 = time.perf_counter()
                _oracle_step(ref, small, k, routing)
                one = {"value": small.T / (time.perf_counter() - t0), "unit": "tokens/s", "cores": 1,
                       "sample": f"first {small.T} tokens of the workload, all weights, fwd+bwd, float32"}
        except ImportError:
            pass
    t_fb, t_f = float(np.median(tb)), float(np.median(tf))
    return {"value": inp.T / t_fb, "unit": "tokens/s", "cores": _blas_threads(), "kind": "oracle",
            "sample": f"the whole workload ({inp.T} tokens), fwd+bwd, float32 NumPy with BLAS, "
                      "median of 2 runs after 1 warm-up",
            "seconds_per_step": t_fb, "fwd_tokens_per_s": inp.T / t_f, "affinity_cores": len(os.sched_getaffinity(0)),
            "one_thread": one}


def run_reference(args):
    """The reference arm is the CPU oracle itself (float32 working precision, BLAS matmuls),
    timed on the host cores."""
    ws_n, rank, local = dist_env()
    if rank != 0:
        return
    name = args.workload
    T, d, E, k, f, skew, routing = WORKLOADS[name][:7]
    inp = make_inputs(name, seed=0)
    from oracle import moe_ref as ref
    with ref.working_precision(np.float32):
        # size each step's token sample so that the W warm-up and K timed steps take about two
        # minutes together
        probe = _token_sample(inp, min(1024, T))
        t0 = time.perf_counter()
        _oracle_step(ref, probe, k, routing)
        t_probe = time.perf_counter() - t0
        n_steps = max(args.steps + args.warmup, 1)
        n = int(max(64, min(T, probe.T * (120.0 / n_steps) / max(t_probe, 1e-3))))
        sample = _token_sample(inp, n)
        for _ in range(args.warmup):
            _oracle_step(ref, sample, k, routing)
        times = []
        for _ in range(args.steps):
            t0 = time.perf_counter()
            _oracle_step(ref, sample, k, routing)
            times.append(time.perf_counter() - t0)
    dt = float(np.mean(times))
    v = n / dt
    print(json.dumps({
        "impl": "reference", "metric": "MoE-layer tokens/s (E=128,k=4,bf16 fwd+bwd) 1xB200; grouped-GEMM % TC peak",
        "value": v, "unit": "tokens/s", "n_gpus": ws_n, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": dt * 1e3, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "f32", "data": "synthetic", "config": {"workload": name, "T": T, "d_model": d, "experts": E,
                                                          "top_k": k, "ffn": f},
        "cpu_baseline": {"value": v, "unit": "tokens/s", "cores": _blas_threads(), "kind": "oracle",
                         "sample": f"first {n} tokens of the workload per step, all weights, fwd+bwd, float32 "
                                   "NumPy with BLAS"},
        "e2e": {"value": v, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }))


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default=DEFAULT, choices=sorted(WORKLOADS))
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-sweep", action="store_true", help="time the main workload only")
    ap.add_argument("--no-cupti", action="store_true",
                    help="count launches by formula, not with the CUDA profiler (e.g. under ncu)")
    args = ap.parse_args()
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
