"""Benchmark of the routed MoE block (route -> plan -> grouped experts -> combine).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
                  [--workloads LIST|all|none] [--impl ours|reference]

One step = one moe_forward over one batch of the workload's synthetic tokens
(all stages of the block).  Default workload: the LFM2-8B-A1B-shaped MoE block
at prefill (T=4096, H=2048, E=32, top-4, I=1792, SwiGLU, bf16, 41 all-NaN
router rows), the largest single-GPU configuration.  N > 1 (torchrun) runs
independent replicas, one per GPU, with no data-path collective (the block has
none): value = tokens all ranks processed / max-over-ranks time (weak scaling).

Timing: W warm-up steps, then exactly K steps replayed from CUDA graphs,
bracketed by a barrier + synchronize, timed with CUDA events on the stream.
Inputs larger than L2: the steps rotate over several copies of the expert
weights whose total is at least 4x the 126 MB L2, so every step streams its
experts from HBM.  Every captured step carries a CUDA-event pair around the
dominant kernel (the expert up-projection), so the `roofline` entry is the
average duration of the launches replayed inside the timed region, whatever K.

The same process then measures the other configurations (`workloads` key: the
decode block, the relu^2 block and the affine 4-bit and NVFP4 token sweeps), each with its
own value, roofline and step roofline, on its own step count (about 0.3 s of
work, at least 20 steps); the driver's K and W apply to the headline line.
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
# B200's published dense figures (HGX): context for the measured fractions
NOMINAL_PEAKS = {"hbm_gbs": 7700.0, "bf16_tflops": 2250.0}
DEFAULT_WORKLOAD = "lfm2_prefill_t4096"
SIDE_WORKLOADS = ("lfm2_decode_t8", "nemotron_relu2_t2048", "affine4_t1", "affine4_t8", "affine4_t64",
                  "affine4_t512", "affine4_t8192", "nvfp4_t1", "nvfp4_t8", "nvfp4_t64", "nvfp4_t512",
                  "nvfp4_t8192")
GRAPH_BLOCK = 32      # steps per captured graph (at most; fewer when K is smaller)


def parse(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=0, help="timed steps (0: about 2 s of work)")
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD)
    ap.add_argument("--workloads", default="all",
                    help="other configurations measured after the headline one: 'all', 'none' or a "
                         "comma-separated list of workload names")
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
    return ap.parse_args(argv)


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return FALLBACK_PEAKS, "fallback"


def sustained_tflops(pk) -> float:
    return float(pk.get("bf16_tflops_sustained", pk["bf16_tflops"]))


def ridge_flop_per_byte(pk) -> float:
    """Machine balance of the peaks: a kernel whose FLOPs per algorithmic byte
    exceed it is tensor-bound, else HBM-bound."""
    return sustained_tflops(pk) * 1e3 / float(pk["hbm_gbs"])


def config_of(wl, args) -> dict:
    """The workload's configuration, identical in both arms of the benchmark."""
    return {"workload": wl.name, "T": wl.T, "H": wl.H, "E": wl.E, "k": wl.k, "I": wl.I, "act": wl.act,
            "weights": wl.fmt, "eps": wl.eps, "router_scale": wl.router_scale, "out_scale": wl.out_scale,
            "nan_rows": wl.nan_rows, "hot_experts": wl.hot_experts,
            "parallelism": "replicas (one independent block per GPU)",
            "l2": "inputs larger than L2: the steps rotate over copies of the expert weights totalling "
                  ">= 4x the 126 MB L2, so each step streams its experts from HBM",
            "graphs": f"CUDA graphs of up to {GRAPH_BLOCK} steps", "expert_kernels": args.dispatch,
            "combine": args.combine}


# ----------------------------------------------------------------------------- algorithmic work

def expert_bytes(wl) -> tuple:
    """(W1 bytes, W2 bytes) of one expert: bf16; affine 4-bit codes + bf16 scale and
    bias per 64; NVFP4 codes + an e4m3 scale per 16 + an fp32 global scale."""
    n1 = (2 if wl.act == "swiglu" else 1) * wl.I
    if wl.fmt == "bf16":
        return n1 * wl.H * 2, wl.H * wl.I * 2
    if wl.fmt == "nvfp4":
        return n1 * wl.H // 2 + n1 * wl.H // 16 + 4, wl.H * wl.I // 2 + wl.H * wl.I // 16 + 4
    return n1 * wl.H // 2 + (n1 * wl.H // 64) * 4, wl.H * wl.I // 2 + (wl.H * wl.I // 64) * 4


def work_model(inp, counts):
    """Algorithmic FLOPs and bytes of one step, and of one launch of the
    expert up kernel, given the plan's per-expert counts."""
    wl = inp.wl
    active = [e for e in range(wl.E) if counts[e] > 0]
    A = len(active)
    n1 = (2 if wl.act == "swiglu" else 1) * wl.I
    P = wl.T * wl.k
    w1_per, w2_per = expert_bytes(wl)
    flops = 2.0 * P * (n1 * wl.H + wl.H * wl.I)
    x_b, h_b, yacc_b, y_b = wl.T * wl.H * 2, P * wl.I * 2, wl.T * wl.H * 4, wl.T * wl.H * 2
    step_bytes = (A * (w1_per + w2_per) + x_b + wl.E * wl.H * 4 + 2 * h_b + 3 * yacc_b + y_b)
    up_bytes = A * w1_per + x_b + h_b
    up_flops = 2.0 * P * n1 * wl.H
    return {"active_experts": A, "flops": flops, "step_bytes": step_bytes, "up_bytes": up_bytes,
            "up_flops": up_flops, "w1_bytes_per_expert": w1_per}


def roofline_of(wm, up_us: float, pk, pk_kind: str, traffic):
    """The dominant kernel's roofline entry: HBM-bound when its FLOPs per
    algorithmic byte are under the peaks' ridge, else tensor-bound (against
    the sustained GEMM figure: the kernel runs inside a long timed loop)."""
    ridge = ridge_flop_per_byte(pk)
    intensity = wm["up_flops"] / wm["up_bytes"]
    sec = up_us / 1e6
    if intensity < ridge:
        bound, unit = "hbm", "GB/s"
        achieved, peak, nominal = wm["up_bytes"] / sec / 1e9, float(pk["hbm_gbs"]), NOMINAL_PEAKS["hbm_gbs"]
    else:
        bound, unit = "tensor", "TFLOP/s"
        achieved, peak, nominal = wm["up_flops"] / sec / 1e12, sustained_tflops(pk), NOMINAL_PEAKS["bf16_tflops"]
    return {"bound": bound, "achieved": achieved, "peak": peak, "unit": unit, "frac": achieved / peak,
            "traffic": traffic, "kernel": "expert up-projection + activation", "us_per_launch": up_us,
            "peak_source": pk_kind, "frac_of_nominal": achieved / nominal, "nominal_peak": nominal,
            "intensity_flop_per_byte": intensity, "ridge_flop_per_byte": ridge,
            "targets_judged_on": "peak (" + pk_kind + ")"}


def step_roofline_of(wm, step_us: float, pk):
    t_hbm = wm["step_bytes"] / (float(pk["hbm_gbs"]) * 1e9)
    t_tc = wm["flops"] / (sustained_tflops(pk) * 1e12)
    s = step_us / 1e6
    return {"bound": "hbm" if t_hbm >= t_tc else "tensor", "roofline_us": max(t_hbm, t_tc) * 1e6,
            "measured_us": step_us, "frac": max(t_hbm, t_tc) / s, "bytes": wm["step_bytes"], "flops": wm["flops"]}


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

def cpu_model() -> str:
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.lower().startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    import platform
    return platform.processor() or "unknown"


def blas_threads() -> int:
    try:
        from threadpoolctl import threadpool_info
        return max([i.get("num_threads", 1) for i in threadpool_info()] or [1])
    except Exception:  # pragma: no cover
        return os.cpu_count() or 1


def cpu_oracle_rate(inp, budget_s: float):
    """Time the float64 oracle (as it stands) on a bounded sample of the
    workload's tokens; returns (tokens/s, sample description, threads)."""
    import numpy as np
    import oracle as O
    wl = inp.wl
    threads = blas_threads()
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


def cpu_baseline_entry(inp, budget_s: float) -> dict:
    """The oracle on every BLAS thread of the host, then on one thread."""
    rate, desc, threads = cpu_oracle_rate(inp, budget_s)
    entry = {"value": rate, "unit": "tokens/s", "cores": threads, "kind": "oracle", "sample": desc,
             "cpu_model": cpu_model(), "host_cpus": os.cpu_count()}
    try:
        from threadpoolctl import threadpool_limits
        with threadpool_limits(limits=1):
            r1, d1, _ = cpu_oracle_rate(inp, max(2.0, budget_s / 3))
        entry["value_1_thread"] = r1
        entry["sample_1_thread"] = d1
    except Exception as ex:  # pragma: no cover
        entry["value_1_thread"] = None
        entry["sample_1_thread"] = f"not run: {ex}"
    return entry


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


def block_steps(K: int, n_sets: int, cap: int = GRAPH_BLOCK) -> int:
    """Steps per captured graph block: a multiple of the weight-set count, at
    most `cap`, and at most K when K >= n_sets (so the block is replayed
    inside any timed region of K steps)."""
    return n_sets * max(1, min(cap, max(K, 1)) // n_sets)


def replayed_events(K: int, B: int, n_block: int, n_single: int):
    """Which event pairs the last replays of a timed region of K steps left
    behind: ('block', range) for the block's pairs when it was replayed, and
    ('single', range) for the trailing single-step graphs."""
    full, rest = divmod(K, B)
    out = []
    if full > 0:
        out.append(("block", range(n_block)))
    if rest > 0:
        out.append(("single", range(min(rest, n_single))))
    return out


def side_workloads(arg: str, main: str):
    if arg == "none":
        return []
    if arg == "all":
        return [w for w in SIDE_WORKLOADS if w != main]
    return [w for w in arg.split(",") if w and w != main]


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
            "data": "synthetic", "config": config_of(wl, args),
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": threads, "kind": "oracle",
                             "sample": desc, "cpu_model": cpu_model(), "host_cpus": os.cpu_count()},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line))
    return 0


# ----------------------------------------------------------------------------- our arm

class Inputs:
    """Host and device inputs, sharing expert weights between workloads that
    draw the same ones (same H, E, I, activation, format and seed)."""

    def __init__(self, G, api, torch):
        self.G, self.api, self.torch = G, api, torch
        self.host = {}
        self.dev = {}

    @staticmethod
    def key(wl):
        return (wl.H, wl.E, wl.I, wl.act, wl.fmt, wl.seed, wl.shared_I)

    def host_inputs(self, wl):
        k = self.key(wl)
        if k not in self.host:
            self.host[k] = self.G.make_inputs(wl)
            return self.host[k]
        src = self.host[k]
        inp = self.G.make_inputs(wl, with_experts=False)
        for f in ("w1_bits", "w2_bits", "w1_q", "w1_scale", "w1_bias", "w2_q", "w2_scale", "w2_bias", "w1_global",
                  "w2_global", "shared"):
            setattr(inp, f, getattr(src, f))
        return inp

    def weight_sets(self, inp):
        """Copies of the experts' device weights, rotated across steps."""
        from sigmoid_top_routing_b200.device_inputs import to_device
        k = self.key(inp.wl)
        if k not in self.dev:
            W = to_device(inp, with_x=False).W
            w1, w2 = expert_bytes(inp.wl)
            all_w = (w1 + w2) * inp.wl.E
            n_sets = max(2, min(16, math.ceil(4 * L2_BYTES / all_w)))
            sets = [W] + [W.clone() for _ in range(n_sets - 1)]
            self.dev[k] = (sets, all_w)
        return self.dev[k]


class Runner:
    """One workload on the device: buffers, the forward call, graphs with the
    up-kernel event pairs, and the timing of K steps."""

    def __init__(self, wl, inp, sets, all_w, api, abi, torch, stream):
        from sigmoid_top_routing_b200.device_inputs import bf16_tensor
        self.wl, self.inp, self.api, self.abi, self.torch, self.stream = wl, inp, api, abi, torch, stream
        self.Ws, self.all_w = sets, all_w
        self.n_sets = len(sets)
        self.x = bf16_tensor(inp.x_bits, "cuda")
        self.w_router = torch.from_numpy(inp.w_router).cuda()
        self.bias = torch.from_numpy(inp.expert_bias).cuda()
        d = api.dims(wl.T, wl.H, wl.E, wl.k, wl.I)
        self.ws = api.new_workspace(d, sets[0].fmt)
        self.plan = api.new_plan(wl.T, wl.E, wl.k)
        self.y = torch.empty((wl.T, wl.H), dtype=torch.bfloat16, device="cuda")
        self.idx = torch.empty((wl.T, wl.k), dtype=torch.int32, device="cuda")
        self.tw = torch.empty((wl.T, wl.k), dtype=torch.float32, device="cuda")

    def forward(self, W):
        wl = self.wl
        self.api.moe_forward(self.x, W, self.w_router, self.bias, E=wl.E, k=wl.k, I=wl.I, eps=wl.eps,
                             router_scale=wl.router_scale, out_scale=wl.out_scale, topk_idx=self.idx,
                             topk_w=self.tw, plan=self.plan, y=self.y, ws=self.ws, stream=self.stream)

    def first_call(self):
        torch = self.torch
        with torch.cuda.stream(self.stream):
            self.forward(self.Ws[0])
        self.stream.synchronize()
        assert self.api.moe_device_error(self.stream) == 0
        self.launches = self.api.moe_last_launch_count()
        self.counts = self.plan.counts.cpu().numpy()
        self.wm = work_model(self.inp, self.counts)

    def _events(self, n):
        torch = self.torch
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(n)]
        with torch.cuda.stream(self.stream):
            for a, b in evs:      # created and recorded once before capture
                a.record(self.stream)
                b.record(self.stream)
        return evs

    def capture(self, K: int, stage: int):
        """Graphs: a block of B steps and n_sets single steps, each step with
        an event pair around `stage`'s kernel."""
        torch, api = self.torch, self.api
        self.B = block_steps(K, self.n_sets)
        with torch.cuda.stream(self.stream):
            for j in range(self.n_sets):
                self.forward(self.Ws[j])
        self.ev_block = self._events(self.B)
        self.ev_single = self._events(self.n_sets)
        self.stream.synchronize()
        self.block = torch.cuda.CUDAGraph()
        with torch.cuda.graph(self.block, stream=self.stream):
            for j in range(self.B):
                api.moe_profile_hook(self.ev_block[j][0], self.ev_block[j][1], stage)
                self.forward(self.Ws[j % self.n_sets])
        self.single = []
        for j in range(self.n_sets):
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=self.stream):
                api.moe_profile_hook(self.ev_single[j][0], self.ev_single[j][1], stage)
                self.forward(self.Ws[j])
            self.single.append(g)
        api.moe_profile_hook(None, None, 0)

    def run_steps(self, n: int):
        full, rest = divmod(n, self.B)
        with self.torch.cuda.stream(self.stream):
            for _ in range(full):
                self.block.replay()
            for j in range(rest):
                self.single[j % self.n_sets].replay()

    def stage_ms(self, K: int):
        """Mean duration of the hooked stage over the launches the last K-step
        region replayed."""
        vals = []
        for kind, rng in replayed_events(K, self.B, len(self.ev_block), len(self.ev_single)):
            evs = self.ev_block if kind == "block" else self.ev_single
            vals += [evs[i][0].elapsed_time(evs[i][1]) for i in rng]
        return statistics.mean(vals) if vals else None

    def timed(self, K: int, dist, world: int):
        torch = self.torch
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(self.stream):
            e0.record(self.stream)
        self.run_steps(K)
        with torch.cuda.stream(self.stream):
            e1.record(self.stream)
        self.stream.synchronize()
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        return e0.elapsed_time(e1)

    def per_step_s(self) -> float:
        t0 = time.perf_counter()
        self.run_steps(self.B * 2)
        self.stream.synchronize()
        return (time.perf_counter() - t0) / (self.B * 2)

    def stage_breakdown(self, gemv_path: bool):
        abi, torch, api = self.abi, self.torch, self.api
        names = [(abi.MOE_STAGE_ROUTE, "route"), (abi.MOE_STAGE_PLAN, "plan"),
                 (abi.MOE_STAGE_GATHER, "gather"), (abi.MOE_STAGE_UP, "up"),
                 (abi.MOE_STAGE_DOWN, "down"), (abi.MOE_STAGE_FINAL, "finalize")]
        B = self.B
        out = {}
        for sid, nm in names:
            if sid == abi.MOE_STAGE_PLAN and self.wl.T <= 32:
                out[nm] = "fused into route"     # one CTA routes and plans at T <= 32
                continue
            if sid == abi.MOE_STAGE_GATHER and gemv_path:
                out[nm] = "not launched (GEMV path)"
                continue
            if sid == abi.MOE_STAGE_GATHER and self.wl.fmt == "bf16" and self.wl.T <= 16:
                out[nm] = "not launched (the up GEMM reads x itself at T <= 16)"
                continue
            evs = self._events(B)
            self.stream.synchronize()
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=self.stream):
                for j in range(B):
                    api.moe_profile_hook(evs[j][0], evs[j][1], sid)
                    self.forward(self.Ws[j % self.n_sets])
            api.moe_profile_hook(None, None, 0)
            with torch.cuda.stream(self.stream):
                for _ in range(3):
                    g.replay()
            self.stream.synchronize()
            try:
                out[nm] = round(1e3 * statistics.mean(a.elapsed_time(b) for a, b in evs), 2)
            except RuntimeError:      # the stage launched no kernel of its own (events never recorded)
                out[nm] = "not launched"
            del g
        return out


def dtype_of(wl) -> str:
    """The arithmetic the path computes in: bf16 operands, or 4-bit weight codes
    dequantised on chip against bf16 activations; fp32 accumulation throughout."""
    return {"bf16": "bf16", "affine4": "u4+bf16", "nvfp4": "e2m1+bf16"}[wl.fmt]


def gemv_path_of(wl, dispatch: str) -> bool:
    """The library's AUTO choice: 4-bit experts at <= 8 pairs per expert take a GEMV."""
    return dispatch == "gemv" or (dispatch == "auto" and wl.fmt != "bf16" and wl.T * wl.k <= 8 * wl.E
                                  and wl.H <= 8192 and wl.I <= 8192)


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
    if rank == 0 or world == 1:
        B.build(quiet=True)
    if world > 1:
        dist.barrier()
    api.load()

    api.moe_set_combine({"atomic": abi.MOE_COMBINE_ATOMIC, "ordered": abi.MOE_COMBINE_ORDERED}[args.combine])
    api.moe_set_dispatch({"auto": abi.MOE_DISPATCH_AUTO, "gemv": abi.MOE_DISPATCH_GEMV,
                          "gemm": abi.MOE_DISPATCH_GEMM}[args.dispatch])
    stream = torch.cuda.Stream()
    store = Inputs(G, api, torch)
    pk, pk_kind = peaks()

    def runner_for(name):
        wl = G.WORKLOADS[name]
        inp = store.host_inputs(wl)
        sets, all_w = store.weight_sets(inp)
        r = Runner(wl, inp, sets, all_w, api, abi, torch, stream)
        r.first_call()
        return r

    wl = G.WORKLOADS[args.workload]
    R = runner_for(args.workload)

    if args.profile:
        # plain launches for a profiler: W + K forward calls, nothing else
        with torch.cuda.stream(stream):
            for j in range(args.warmup + max(1, args.steps)):
                R.forward(R.Ws[j % R.n_sets])
        stream.synchronize()
        assert api.moe_device_error(stream) == 0
        if rank == 0:
            print(json.dumps({"profile_run": wl.name, "steps": args.warmup + max(1, args.steps),
                              "launches_per_step": R.launches, "work": R.wm}))
        return 0

    K = args.steps
    R.capture(max(K, GRAPH_BLOCK) if K <= 0 else K, abi.MOE_STAGE_UP)
    R.run_steps(max(3, args.warmup))
    stream.synchronize()
    if K <= 0:      # about 2 s of work, a whole number of blocks
        K = int(max(R.B, min(200000, 2.0 / R.per_step_s())))
        K = (K // R.B) * R.B
    K = int(max_over_ranks(K, dist, world, "cuda", torch.int64))

    sampler = ClockSampler(bus_id_of(torch, local))
    sampler.start()
    t_soak = time.time()           # soak so the sampler sees the clocks under load
    while time.time() - t_soak < 1.0:
        R.run_steps(R.B)
        stream.synchronize()
    t_a = time.time()
    ms = R.timed(K, dist, world)
    t_b = time.time()
    ms = float(max_over_ranks(ms, dist, world, "cuda", torch.float64))
    assert api.moe_device_error(stream) == 0
    up_ms = R.stage_ms(K)
    clocks = sampler.summary(t_a - 0.5, t_b)

    value = job_rate(wl.T * K, world, ms / 1e3)
    line = {"metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": K,
            "warmup": args.warmup, "ms_per_step": ms / K, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": dtype_of(wl), "data": "synthetic",
            "config": config_of(wl, args),
            "l2_detail": f"{R.n_sets} weight copies rotated ({R.n_sets * R.all_w / 1e9:.2f} GB), "
                         f"{R.wm['active_experts']} active experts per step",
            "gpu_launches": R.launches * K, "clocks": clocks}
    up_us = float(max_over_ranks(up_ms * 1e3, dist, world, "cuda", torch.float64))
    line["roofline"] = roofline_of(R.wm, up_us, pk, pk_kind, traffic_of("up", wl.name))
    line["step_roofline"] = step_roofline_of(R.wm, 1e3 * ms / K, pk)
    if not args.no_stages:
        line["stage_us"] = R.stage_breakdown(gemv_path_of(wl, args.dispatch))

    # end to end through the public host-buffer call
    if not args.no_e2e:
        x_host = torch.from_numpy(R.inp.x_bits.view(np.int16)).view(torch.bfloat16).pin_memory()
        y_host = torch.empty((wl.T, wl.H), dtype=torch.bfloat16).pin_memory()
        x_dev = torch.empty_like(R.x)
        n_e2e = max(10, min(K, 2000))

        def host_call(W):
            api.moe_forward_host(x_host, x_dev, W, R.w_router, R.bias, E=wl.E, k=wl.k, I=wl.I,
                                 y_dev=R.y, y_host=y_host, topk_idx=R.idx, topk_w=R.tw, plan=R.plan, ws=R.ws,
                                 eps=wl.eps, router_scale=wl.router_scale, out_scale=wl.out_scale,
                                 stream=stream)
        for j in range(3):
            host_call(R.Ws[j % R.n_sets])
        if world > 1:
            dist.barrier()
        t0 = time.perf_counter()
        for j in range(n_e2e):
            host_call(R.Ws[j % R.n_sets])
        el = time.perf_counter() - t0
        el = float(max_over_ranks(el, dist, world, "cuda", torch.float64))
        line["e2e"] = {"value": job_rate(wl.T * n_e2e, world, el), "unit": "tokens/s",
                       "h2d_bytes_per_step": wl.T * wl.H * 2, "d2h_bytes_per_step": wl.T * wl.H * 2,
                       "steps": n_e2e, "timing": "host wall clock around synchronous moe_forward_host calls"}

    # the other configurations, each on its own step count
    others = {}
    for name in side_workloads(args.workloads, wl.name):
        w2 = G.WORKLOADS[name]
        r = runner_for(name)
        r.capture(GRAPH_BLOCK, abi.MOE_STAGE_UP)
        r.run_steps(max(3, args.warmup))
        stream.synchronize()
        k2 = int(max(20, min(20000, 0.3 / r.per_step_s())))
        k2 = int(max_over_ranks(k2, dist, world, "cuda", torch.int64))
        ta = time.time()
        ms2 = float(max_over_ranks(r.timed(k2, dist, world), dist, world, "cuda", torch.float64))
        tb = time.time()
        assert api.moe_device_error(stream) == 0
        up2 = float(max_over_ranks(r.stage_ms(k2) * 1e3, dist, world, "cuda", torch.float64))
        c2 = sampler.summary(ta, tb)
        entry = {"value": job_rate(w2.T * k2, world, ms2 / 1e3), "unit": "tokens/s", "steps": k2,
                 "ms_per_step": ms2 / k2, "dtype": dtype_of(w2),
                 "config": config_of(w2, args), "gpu_launches": r.launches * k2,
                 "roofline": roofline_of(r.wm, up2, pk, pk_kind, traffic_of("up", name)),
                 "step_roofline": step_roofline_of(r.wm, 1e3 * ms2 / k2, pk),
                 "clocks": {"sm_mhz": c2.get("sm_mhz"), "reasons": c2.get("reasons")},
                 "active_experts": r.wm["active_experts"]}
        if not args.no_stages:
            entry["stage_us"] = r.stage_breakdown(gemv_path_of(w2, args.dispatch))
        others[name] = entry
        del r
    sampler.stop()
    if others:
        line["workloads"] = others

    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline_entry(R.inp, args.cpu_seconds)
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
