"""Benchmark of the routed MoE block (route -> plan -> grouped experts -> combine).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

One step = one moe_forward over one batch of the workload's synthetic tokens
(all stages of the block).  Default workload: the LFM2-8B-A1B-shaped decode
block (T=8, H=2048, E=32, top-4, I=1792, SwiGLU, bf16).  N > 1 (torchrun) runs
independent replicas, one per GPU, with no data-path collective (the block has
none): value = tokens all ranks processed / max-over-ranks time (weak scaling).

Timing: W warm-up steps, then exactly K steps replayed from CUDA graphs,
bracketed by a barrier + synchronize, timed with CUDA events on the stream.
Inputs larger than L2: the steps rotate over several copies of the expert
weights whose total is at least 4x the 126 MB L2, so every step streams its
experts from HBM.  The roofline entry times the dominant kernel (the expert
up-projection) with CUDA events recorded around it inside the timed graphs.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "MoE-block routed tokens/s and % of BF16/HBM roofline, 1×B200"
L2_BYTES = 126 * 1024 * 1024
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=0, help="timed steps (0: about 2 s of work)")
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default="lfm2_decode_t8")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--dispatch", default="auto", choices=["auto", "gemv", "gemm"],
                    help="expert kernels: the library's choice, the grouped GEMV or the tcgen05 GEMM")
    ap.add_argument("--combine", default="atomic", choices=["atomic", "ordered"],
                    help="combine of the k expert outputs: fp32 atomics, or slot-ordered (reproducible)")
    ap.add_argument("--profile", action="store_true",
                    help="only W + K plain forward calls (for a profiler); prints the work model")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-stages", action="store_true", help="skip the per-stage time breakdown")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=12.0, help="budget of the CPU-baseline sample")
    return ap.parse_args()


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return FALLBACK_PEAKS, "fallback"


# ----------------------------------------------------------------------------- algorithmic work

def work_model(inp, counts):
    """Algorithmic FLOPs and bytes of one step, and of one launch of the
    expert up kernel, given the plan's per-expert counts."""
    wl = inp.wl
    from sigmoid_top_routing_b200.device_inputs import weight_bytes
    active = [e for e in range(wl.E) if counts[e] > 0]
    A = len(active)
    n1 = (2 if wl.act == "swiglu" else 1) * wl.I
    P = wl.T * wl.k
    if wl.fmt == "bf16":
        w1_per = n1 * wl.H * 2
    else:
        w1_per = n1 * wl.H // 2 + (n1 * wl.H // 64) * 4
    flops = 2.0 * P * (n1 * wl.H + wl.H * wl.I)
    x_b, h_b, yacc_b, y_b = wl.T * wl.H * 2, P * wl.I * 2, wl.T * wl.H * 4, wl.T * wl.H * 2
    step_bytes = (weight_bytes(inp, active) + x_b + wl.E * wl.H * 4 + 2 * h_b + 3 * yacc_b + y_b)
    up_bytes = A * w1_per + x_b + h_b
    up_flops = 2.0 * P * n1 * wl.H
    return {"active_experts": A, "flops": flops, "step_bytes": step_bytes, "up_bytes": up_bytes,
            "up_flops": up_flops, "w1_bytes_per_expert": w1_per}


# ----------------------------------------------------------------------------- clocks

class ClockSampler:
    """nvidia-smi sampling of SM clocks and throttle reasons while running."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, bus_id: str):
        self.samples = []
        self.proc = None
        self.bus_id = bus_id
        self.t0 = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits", "-lms", "100",
                 "-i", self.bus_id], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except (OSError, FileNotFoundError):
            self.proc = None
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()

    def _read(self):
        for line in self.proc.stdout:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) >= 9:
                self.samples.append((time.time(), parts))

    def stop(self):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self, t_from: float, t_to: float):
        win = [p for (t, p) in self.samples if t_from <= t <= t_to]
        if not win:
            win = [p for (_, p) in self.samples]
        if not win:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no nvidia-smi samples"], "samples": 0}

        def num(v):
            try:
                return float(v)
            except ValueError:
                return None
        sm = [num(p[1]) for p in win if num(p[1]) is not None]
        smax = [num(p[2]) for p in win if num(p[2]) is not None]
        reasons = set()
        for p in win:
            for name, v in zip(("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"),
                               p[5:9]):
                if v.strip().lower() == "active":
                    reasons.add(name)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(smax) if smax else None,
                "reasons": sorted(reasons), "samples": len(win),
                "power_w_max": max((num(p[3]) or 0.0) for p in win)}


def bus_id_of(torch, dev):
    p = torch.cuda.get_device_properties(dev)
    try:
        return f"{p.pci_domain_id:08X}:{p.pci_bus_id:02X}:{p.pci_device_id:02X}.0"
    except AttributeError:
        return str(dev)


# ----------------------------------------------------------------------------- CPU oracle

def cpu_oracle_rate(inp, budget_s: float):
    """Time the float64 oracle (as it stands) on a bounded sample of the
    workload's tokens; returns (tokens/s, sample description, threads)."""
    import numpy as np
    import oracle as O
    wl = inp.wl
    try:
        from threadpoolctl import threadpool_info
        threads = max([i.get("num_threads", 1) for i in threadpool_info()] or [1])
    except Exception:  # pragma: no cover
        threads = os.cpu_count() or 1
    rng = np.random.default_rng(1)
    n = min(wl.T, 8)
    done_tokens, t_used, calls = 0, 0.0, 0
    while t_used < budget_s and calls < 64:
        tok = np.sort(rng.choice(wl.T, n, replace=False))
        t0 = time.perf_counter()
        O.moe_block(inp, tok)
        t_used += time.perf_counter() - t0
        done_tokens += n
        calls += 1
        if t_used > budget_s * 0.5 and calls >= 1 and t_used / calls > budget_s / 2:
            break
    return done_tokens / t_used, f"{calls} oracle calls x {n} tokens of the workload ({t_used:.1f} s)", threads


# ----------------------------------------------------------------------------- ranks

def max_over_ranks(v, dist, world: int, device, dtype):
    """The maximum of v over all ranks.  Every rank calls it at the same
    point (a collective); with one rank it returns v unchanged."""
    if world <= 1:
        return v
    import torch
    t = torch.tensor([v], device=device, dtype=dtype)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t.item()


def job_rate(units_per_rank: float, world: int, seconds: float) -> float:
    """Whole-job throughput: the units all ranks processed over the slowest
    rank's time (weak scaling: every rank runs the same per-rank work)."""
    return units_per_rank * world / seconds


# ----------------------------------------------------------------------------- reference arm

def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    from sigmoid_top_routing_b200 import inputs as G
    wl = G.WORKLOADS[args.workload]
    inp = G.make_inputs(wl)
    steps = args.steps or 3
    budget = max(2.0, min(20.0, 120.0 / max(1, steps + args.warmup)))
    for _ in range(args.warmup):
        cpu_oracle_rate(inp, budget * 0.25)
    rates, desc, threads = [], "", 1
    t0 = time.perf_counter()
    for _ in range(steps):
        r, desc, threads = cpu_oracle_rate(inp, budget)
        rates.append(r)
    el = time.perf_counter() - t0
    value = statistics.median(rates)
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": args.gpus,
            "steps": steps, "warmup": args.warmup, "ms_per_step": 1e3 * el / steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": config_of(wl),
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": threads, "kind": "oracle",
                             "sample": desc},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line))
    return 0


def config_of(wl):
    return {"workload": wl.name, "T": wl.T, "H": wl.H, "E": wl.E, "k": wl.k, "I": wl.I, "act": wl.act,
            "weights": wl.fmt, "eps": wl.eps, "router_scale": wl.router_scale, "out_scale": wl.out_scale,
            "parallelism": "replicas (one independent block per GPU)"}


# ----------------------------------------------------------------------------- our arm

def main():
    args = parse()
    if args.impl == "reference":
        return run_reference(args)

    import numpy as np
    import torch
    import torch.distributed as dist

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))

    from sigmoid_top_routing_b200 import abi, api
    from sigmoid_top_routing_b200 import build as B
    from sigmoid_top_routing_b200 import inputs as G
    from sigmoid_top_routing_b200.device_inputs import to_device
    if rank == 0 or world == 1:
        B.build(quiet=True)
    if world > 1:
        dist.barrier()
    api.load()

    wl = G.WORKLOADS[args.workload]
    api.moe_set_combine({"atomic": abi.MOE_COMBINE_ATOMIC, "ordered": abi.MOE_COMBINE_ORDERED}[args.combine])
    api.moe_set_dispatch({"auto": abi.MOE_DISPATCH_AUTO, "gemv": abi.MOE_DISPATCH_GEMV,
                          "gemm": abi.MOE_DISPATCH_GEMM}[args.dispatch])
    inp = G.make_inputs(wl)
    D = to_device(inp)
    d = api.dims(wl.T, wl.H, wl.E, wl.k, wl.I)
    stream = torch.cuda.Stream()

    # weight copies rotated across steps so the step's experts stream from HBM
    from sigmoid_top_routing_b200.device_inputs import weight_bytes
    all_w = weight_bytes(inp, range(wl.E))
    n_sets = max(1, math.ceil(4 * L2_BYTES / all_w)) if all_w < 4 * L2_BYTES else 2
    n_sets = min(max(n_sets, 2), 16)
    Ws = [D.W]
    for _ in range(n_sets - 1):
        W = D.W
        Ws.append(api.ExpertWeights(act=W.act, fmt=W.fmt, w1=W.w1.clone(), w2=W.w2.clone(),
                                    w1_scale=None if W.w1_scale is None else W.w1_scale.clone(),
                                    w1_bias=None if W.w1_bias is None else W.w1_bias.clone(),
                                    w2_scale=None if W.w2_scale is None else W.w2_scale.clone(),
                                    w2_bias=None if W.w2_bias is None else W.w2_bias.clone()))
    ws = api.new_workspace(d, D.W.fmt)
    plan = api.new_plan(wl.T, wl.E, wl.k)
    y = torch.empty((wl.T, wl.H), dtype=torch.bfloat16, device="cuda")
    idx = torch.empty((wl.T, wl.k), dtype=torch.int32, device="cuda")
    tw = torch.empty((wl.T, wl.k), dtype=torch.float32, device="cuda")

    def forward(W):
        api.moe_forward(D.x, W, D.w_router, D.expert_bias, E=wl.E, k=wl.k, I=wl.I, eps=wl.eps,
                        router_scale=wl.router_scale, out_scale=wl.out_scale, topk_idx=idx, topk_w=tw,
                        plan=plan, y=y, ws=ws, stream=stream)

    with torch.cuda.stream(stream):
        forward(Ws[0])
    stream.synchronize()
    assert api.moe_device_error(stream) == 0
    launches_per_step = api.moe_last_launch_count()
    counts = plan.counts.cpu().numpy()
    wm = work_model(inp, counts)

    if args.profile:
        # plain launches for a profiler: W + K forward calls, nothing else
        with torch.cuda.stream(stream):
            for j in range(args.warmup + max(1, args.steps)):
                forward(Ws[j % n_sets])
        stream.synchronize()
        assert api.moe_device_error(stream) == 0
        if rank == 0:
            print(json.dumps({"profile_run": wl.name, "steps": args.warmup + max(1, args.steps),
                              "launches_per_step": launches_per_step, "work": wm}))
        return 0

    # graphs: one block of B steps (rotating the weight sets), with an event
    # pair around the expert up kernel of every step
    B_steps = n_sets * max(1, 32 // n_sets)
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(B_steps)]
    single = []
    with torch.cuda.stream(stream):
        for j in range(n_sets):                      # warm the allocator/caches before capture
            forward(Ws[j])
        for a, b in ev:                              # create the events before capture
            a.record(stream)
            b.record(stream)
    stream.synchronize()
    block = torch.cuda.CUDAGraph()
    with torch.cuda.graph(block, stream=stream):
        for j in range(B_steps):
            api.moe_profile_hook(ev[j][0], ev[j][1], abi.MOE_STAGE_UP)
            forward(Ws[j % n_sets])
    for j in range(n_sets):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            forward(Ws[j])
        single.append(g)

    def run_steps(n):
        full, rest = divmod(n, B_steps)
        for _ in range(full):
            block.replay()
        for j in range(rest):
            single[j % n_sets].replay()

    with torch.cuda.stream(stream):
        run_steps(max(3, args.warmup))
    stream.synchronize()

    # size K to about 2 s of work unless given
    K = args.steps
    if K <= 0:
        t0 = time.perf_counter()
        with torch.cuda.stream(stream):
            run_steps(B_steps * 4)
        stream.synchronize()
        per = (time.perf_counter() - t0) / (B_steps * 4)
        K = int(max(B_steps, min(200000, 2.0 / per)))
        K = (K // B_steps) * B_steps
    K = int(max_over_ranks(K, dist, world, "cuda", torch.int64))

    sampler = ClockSampler(bus_id_of(torch, local))
    sampler.start()
    # soak so the sampler sees the clocks under load, then the timed region
    with torch.cuda.stream(stream):
        t_soak = time.time()
        while time.time() - t_soak < 1.0:
            run_steps(B_steps)
            stream.synchronize()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t_a = time.time()
    with torch.cuda.stream(stream):
        e0.record(stream)
        run_steps(K)
        e1.record(stream)
    stream.synchronize()
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    t_b = time.time()
    sampler.stop()
    ms = e0.elapsed_time(e1)
    ms = float(max_over_ranks(ms, dist, world, "cuda", torch.float64))
    assert api.moe_device_error(stream) == 0

    # up-kernel durations from the last block replay inside the timed region
    up_ms = [a.elapsed_time(b) for (a, b) in ev] if K >= B_steps else []
    clocks = sampler.summary(t_a - 0.5, t_b)

    value = job_rate(wl.T * K, world, ms / 1e3)
    pk, pk_kind = peaks()
    line = {"metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": K,
            "warmup": args.warmup, "ms_per_step": ms / K, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16" if wl.fmt == "bf16" else "u4+bf16", "data": "synthetic",
            "config": dict(config_of(wl), l2=f"inputs larger than L2: {n_sets} weight copies rotated "
                                             f"({n_sets * all_w / 1e9:.2f} GB, {wm['active_experts']} "
                                             f"active experts per step)",
                           graphs=f"CUDA graphs of {B_steps} steps", expert_kernels=args.dispatch,
                           combine=args.combine),
            "gpu_launches": launches_per_step * K, "clocks": clocks}

    # roofline of the dominant kernel (expert up-projection + activation)
    if up_ms:
        up_avg = statistics.mean(up_ms)
        if wl.fmt == "bf16" and wl.T <= 64 or wm["up_flops"] / wm["up_bytes"] < 281:
            bound, achieved, peak = "hbm", wm["up_bytes"] / (up_avg / 1e3) / 1e9, pk["hbm_gbs"]
            unit = "GB/s"
        else:   # timed back to back for seconds: the sustained (power-capped) GEMM figure
            bound, achieved = "tensor", wm["up_flops"] / (up_avg / 1e3) / 1e12
            peak = pk.get("bf16_tflops_sustained", pk["bf16_tflops"])
            unit = "TFLOP/s"
        line["roofline"] = {"bound": bound, "achieved": achieved, "peak": peak, "unit": unit,
                            "frac": achieved / peak, "traffic": traffic_of("up", wl.name),
                            "kernel": "expert up-projection + activation", "us_per_launch": up_avg * 1e3,
                            "peak_source": pk_kind}
    step_s = ms / K / 1e3
    t_hbm = wm["step_bytes"] / (pk["hbm_gbs"] * 1e9)
    t_tc = wm["flops"] / (pk.get("bf16_tflops_sustained", pk["bf16_tflops"]) * 1e12)
    line["step_roofline"] = {"bound": "hbm" if t_hbm >= t_tc else "tensor",
                             "roofline_us": max(t_hbm, t_tc) * 1e6, "measured_us": step_s * 1e6,
                             "frac": max(t_hbm, t_tc) / step_s, "bytes": wm["step_bytes"], "flops": wm["flops"]}

    # in-situ time of each stage: graphs of B steps with events around one stage
    if not args.no_stages:
        names = [(abi.MOE_STAGE_ROUTE, "route"), (abi.MOE_STAGE_PLAN, "plan"),
                 (abi.MOE_STAGE_GATHER, "gather"), (abi.MOE_STAGE_UP, "up"),
                 (abi.MOE_STAGE_DOWN, "down"), (abi.MOE_STAGE_FINAL, "finalize")]
        # the library's AUTO choice: affine 4-bit experts at <= 8 pairs per expert take the GEMV
        gemv_path = args.dispatch == "gemv" or (
            args.dispatch == "auto" and wl.fmt != "bf16" and wl.T * wl.k <= 8 * wl.E
            and wl.H <= 8192 and wl.I <= 8192)
        stage_us = {}
        for sid, nm in names:
            if sid == abi.MOE_STAGE_PLAN and wl.T <= 32:
                stage_us[nm] = "fused into route"     # one CTA routes and plans at T <= 32
                continue
            if sid == abi.MOE_STAGE_GATHER and gemv_path:
                stage_us[nm] = "not launched (GEMV path)"
                continue
            evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                   for _ in range(B_steps)]
            with torch.cuda.stream(stream):
                for a_, b_ in evs:
                    a_.record(stream)
                    b_.record(stream)
            stream.synchronize()
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=stream):
                for j in range(B_steps):
                    api.moe_profile_hook(evs[j][0], evs[j][1], sid)
                    forward(Ws[j % n_sets])
            api.moe_profile_hook(None, None, 0)
            with torch.cuda.stream(stream):
                for _ in range(3):
                    g.replay()
            stream.synchronize()
            vals = [a_.elapsed_time(b_) for a_, b_ in evs]
            stage_us[nm] = round(1e3 * statistics.mean(vals), 2)
            del g
        line["stage_us"] = stage_us

    # end to end through the public host-buffer call
    if not args.no_e2e:
        x_host = torch.from_numpy(inp.x_bits.view(np.int16)).view(torch.bfloat16).pin_memory()
        y_host = torch.empty((wl.T, wl.H), dtype=torch.bfloat16).pin_memory()
        x_dev = torch.empty_like(D.x)
        n_e2e = max(10, min(K, 2000))

        def host_call(W):
            api.moe_forward_host(x_host, x_dev, W, D.w_router, D.expert_bias, E=wl.E, k=wl.k, I=wl.I,
                                 y_dev=y, y_host=y_host, topk_idx=idx, topk_w=tw, plan=plan, ws=ws,
                                 eps=wl.eps, router_scale=wl.router_scale, out_scale=wl.out_scale,
                                 stream=stream)
        for j in range(3):
            host_call(Ws[j % n_sets])
        if world > 1:
            dist.barrier()
        t0 = time.perf_counter()
        for j in range(n_e2e):
            host_call(Ws[j % n_sets])
        el = time.perf_counter() - t0
        el = float(max_over_ranks(el, dist, world, "cuda", torch.float64))
        line["e2e"] = {"value": job_rate(wl.T * n_e2e, world, el), "unit": "tokens/s",
                       "h2d_bytes_per_step": wl.T * wl.H * 2, "d2h_bytes_per_step": wl.T * wl.H * 2,
                       "steps": n_e2e, "timing": "host wall clock around synchronous moe_forward_host calls"}

    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        rate, desc, threads = cpu_oracle_rate(inp, args.cpu_seconds)
        line["cpu_baseline"] = {"value": rate, "unit": "tokens/s", "cores": threads, "kind": "oracle",
                                "sample": desc}
    if rank == 0:
        print(json.dumps(line))
    if world > 1:
        dist.destroy_process_group()
    return 0


def code_hash(text: str) -> str:
    """sha256 prefix of C++ source with comments and whitespace removed: a
    comment edit leaves it unchanged, any code change moves it."""
    import hashlib
    import re
    text = re.sub(r"/\*.*?\*/", " ", text, flags=re.S)
    text = re.sub(r"//[^\n]*", " ", text)
    return hashlib.sha256(" ".join(text.split()).encode()).hexdigest()[:16]


def traffic_of(kernel: str, workload: str):
    """DRAM bytes per launch from the committed ncu summary, if it was taken on
    the current code of that kernel's source file; else None."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    try:
        with open(p) as f:
            d = json.load(f)
        rec = d.get(f"{kernel}:{workload}")
        if not rec:
            return None
        src = os.path.join(ROOT, "sigmoid_top_routing_b200", "csrc", rec["source"])
        with open(src) as f:
            if code_hash(f.read()) != rec["code_sha256_16"]:
                return None
        return rec["bytes_per_launch"]
    except Exception:
        return None


if __name__ == "__main__":
    sys.exit(main())
